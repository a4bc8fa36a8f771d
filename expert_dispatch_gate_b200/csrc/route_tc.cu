// route_tc.cu — router gate GEMM on the tensor cores (tcgen05 + TMEM + TMA), sm_100a.
//
// [P4] "MoE Router" (2048ai.net), section "Router 就是一个小型网络": the gate is a bias-free
// Linear layer, logits[t, e] = sum_h x[t, h] * Wr[h, e].
//
// Orientation: tokens on the MMA's M side (128 per CTA, one TMEM lane each), experts on N
// (E <= 256, padded to a multiple of 16). A = x rows (K-major, 128-byte swizzle), B = Wr
// (expert-contiguous rows, so MN-major; 64-expert chunks of 8 KB per 64-row k-block). The
// hidden dimension is split into `ksplit` ranges, one per CTA along grid.y, so that small T
// still spreads over the SMs; each CTA writes its fp32 partial logits, and the top-k kernel
// sums the ranges in ascending order. When N <= 128 the four 16-deep MMAs of a k-block
// alternate between two accumulators (even / odd K steps), which keeps two independent
// accumulate chains in flight; the epilogue adds the two.
//
// When E % 128 == 0, two CTAs of a cluster share each 256-token tile (cta_group::2, below).
//
// Warps: 0 TMA producer, 1 MMA issuer (converged warp, elected lane), 2-5 epilogue (one TMEM
// lane quadrant each).
#include <cuda.h>

#include <mutex>
#include <string>
#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace moe {
namespace {

constexpr int kRtM = 128;          // tokens per CTA
constexpr int kRtBK = 64;          // K per stage (one 128-byte swizzle row of bf16)
constexpr int kRtMaxStages = 8;
constexpr int kRtThreads = 192;    // 6 warps
constexpr int kRtTmemCols = 256;
constexpr int kRtSmemLimit = 227 * 1024;
constexpr int kRtCtrl = 256;

struct RtParams {
  int T, H, E;
  int npad;            // N of the MMA: E rounded up to 16
  int nch;             // 64-expert chunks of B loaded per stage by this CTA
  int kb_per_split;    // k-blocks of one K range
  int two_acc;         // 1: alternate two accumulators over K steps
  int stages;
  int64_t split_stride;  // elements between consecutive K-range partial arrays
  float* out;            // partials [ksplit][T][E]
  int* err;
};

// PAIR: two CTAs of a cluster share one 256-token tile with tcgen05.mma.cta_group::2 (M = 256):
// each CTA loads its own 128 token rows (A) and half of the expert chunks of Wr (B, so E % 128
// == 0); both CTAs' loads complete on the even CTA's `full` barrier, the even CTA issues the
// MMAs, and its commits arrive on both CTAs' `empty` and `done` barriers. Each CTA's TMEM holds
// its own 128 tokens x N experts, drained by its own epilogue. Per CTA and k-block that is
// 16 KB of x and 16 KB of Wr instead of 16 + 32 KB: a third less L2-to-SM traffic, and more
// k-blocks in flight in the same shared memory.
template <bool PAIR>
__global__ void __launch_bounds__(kRtThreads, 1)
    route_gemm_kernel(const __grid_constant__ CUtensorMap tmX,
                      const __grid_constant__ CUtensorMap tmW, const RtParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int b_bytes = p.nch * 8192;
  const int stage_bytes = 16384 + b_bytes;
  const int S = p.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(S) * stage_bytes);
  uint64_t* empty = full + kRtMaxStages;
  uint64_t* done = empty + kRtMaxStages;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = (rank == 0);
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(done), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(smem_u32(tmem_holder), kRtTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_holder), kRtTmemCols);
      tmem_relinquish();
    }
  }
  pdl_enter<false>();
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync_all();  // both CTAs' barriers are initialised
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int row0 = PAIR ? static_cast<int>(blockIdx.x >> 1) * (2 * kRtM) +
                               static_cast<int>(rank) * kRtM
                        : static_cast<int>(blockIdx.x) * kRtM;
  const int ks = static_cast<int>(blockIdx.y);
  const int kb0 = ks * p.kb_per_split;
  const int nkb = p.kb_per_split;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t s = 0, ph = 0;
      // in PAIR mode the even CTA's barrier expects both CTAs' bytes
      const uint32_t tx = static_cast<uint32_t>(stage_bytes) * (PAIR ? 2u : 1u);
      const int c0 = static_cast<int>(rank) * p.nch;  // first expert chunk this CTA loads
      bool ok = true;
      int issued = 0;
      for (int i = 0; i < nkb; ++i) {
        if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t sa = smem_u32(smem + static_cast<size_t>(s) * stage_bytes);
        const int kc = (kb0 + i) * kRtBK;
        if constexpr (PAIR) {
          const uint32_t fb = mapa_shared(smem_u32(&full[s]), 0);
          if (leader) mbar_arrive_expect_tx(smem_u32(&full[s]), tx);
          tma_load_2d_pair(sa, &tmX, kc, row0, fb);
          for (int c = 0; c < p.nch; ++c)
            tma_load_2d_pair(sa + 16384 + c * 8192, &tmW, (c0 + c) * 64, kc, fb);
        } else {
          const uint32_t fb = smem_u32(&full[s]);
          mbar_arrive_expect_tx(fb, tx);
          tma_load_2d(sa, &tmX, kc, row0, fb);
          for (int c = 0; c < p.nch; ++c) tma_load_2d(sa + 16384 + c * 8192, &tmW, c * 64, kc, fb);
        }
        ++issued;
        if (++s == static_cast<uint32_t>(S)) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (!ok) {
        *abort_flag = 1;
        flag_error(p.err, kDevWaitTimeout);
      }
      // Every load issued lands before the CTA may exit. In PAIR mode the loads complete on the
      // even CTA's barriers; the cluster barrier at the end keeps the odd CTA alive until then.
      if (!PAIR || leader) {
        for (int i = (issued > S ? issued - S : 0); i < issued; ++i)
          mbar_wait_cluster(smem_u32(&full[i % S]), static_cast<uint32_t>(i / S) & 1u, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (whole warp)
    if (leader) {
      constexpr uint32_t kFull = 0xffffffffu;
      const uint32_t sbase = smem_u32(smem);
      const uint64_t adesc0 = smem_desc_sw128(sbase, 16, 1024);            // x rows, K-major
      const uint64_t bdesc0 = smem_desc_sw128(sbase + 16384, 8192, 1024);  // Wr, MN-major
      const uint32_t idesc = idesc_bf16(PAIR ? 2 * kRtM : kRtM, p.npad, /*a_mn_major=*/false,
                                        /*b_mn_major=*/true);
      const uint32_t d1 = tmem_base + (p.two_acc ? static_cast<uint32_t>(p.npad) : 0u);
      uint32_t s = 0, ph = 0, soff = 0;
      uint32_t acc0 = 0, acc1 = 0;
      bool ok = true;
      for (int i = 0; i < nkb; ++i) {
        if (!__all_sync(kFull, mbar_wait_cluster(smem_u32(&full[s]), ph, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t ad = adesc0 + (soff >> 4);
        const uint64_t bd = bdesc0 + (soff >> 4);
#pragma unroll
        for (int kk = 0; kk < kRtBK / 16; ++kk) {
          // A advances 16 K-columns (32 B) per step, B 16 K-rows (2 KB)
          const bool second = p.two_acc && (kk & 1);
          const uint32_t d = second ? d1 : tmem_base;
          const uint32_t acc = second ? acc1 : acc0;
          if constexpr (PAIR) tc_mma_bf16_pair_elect(d, ad + kk * 2, bd + kk * 128, idesc, acc);
          else tc_mma_bf16_elect(d, ad + kk * 2, bd + kk * 128, idesc, acc);
          if (second) acc1 = 1u;
          else acc0 = 1u;
        }
        if constexpr (PAIR) tc_commit_pair_mc_elect(smem_u32(&empty[s]), 0x3);
        else tc_commit_elect(smem_u32(&empty[s]));
        if (++s == static_cast<uint32_t>(S)) {
          s = 0;
          ph ^= 1u;
          soff = 0;
        } else {
          soff += static_cast<uint32_t>(stage_bytes);
        }
      }
      if (!ok && lane == 0) {
        *abort_flag = 1;
        flag_error(p.err, kDevWaitTimeout);
      }
      // completes once every MMA issued has finished (also when the loop stopped early)
      if constexpr (PAIR) tc_commit_pair_mc_elect(smem_u32(done), 0x3);
      else tc_commit_elect(smem_u32(done));
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;
    const int t = row0 + q * 32 + lane;
    int got = 1;
    if (lane == 0) got = mbar_wait_cluster(smem_u32(done), 0u, abort_flag) ? 1 : 0;
    got = __shfl_sync(0xffffffffu, got, 0);
    if (!got) {
      if (lane == 0) {
        *abort_flag = 1;
        flag_error(p.err, kDevWaitTimeout);
      }
    } else {
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
      float* orow = p.out + static_cast<int64_t>(ks) * p.split_stride +
                    static_cast<int64_t>(t) * p.E;
      for (int c0 = 0; c0 < p.E; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tb + static_cast<uint32_t>(c0), v);
        if (p.two_acc) {
          uint32_t u[32];
          tmem_ld32(tb + static_cast<uint32_t>(p.npad + c0), u);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j)
            v[j] = __float_as_uint(__uint_as_float(v[j]) + __uint_as_float(u[j]));
        } else {
          tmem_wait_ld();
        }
        if (t < p.T) {
          // E % 8 == 0: whole 16-byte groups
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            if (c0 + j < p.E) {
              const float4 f = make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                                           __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
              *reinterpret_cast<float4*>(orow + c0 + j) = f;
            }
          }
        }
      }
    }
  }

  // The MMA completion barrier also guards TMEM release when the epilogue gave up early.
  if (warp == 1 && lane == 0) mbar_wait_cluster(smem_u32(done), 0u, nullptr);
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync_all();  // no CTA leaves while its peer may still signal it
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, kRtTmemCols);
    else tmem_dealloc(tmem_base, kRtTmemCols);
  }
}

// Gate GEMM and plain top-k in one persistent kernel, for the whole hidden dimension in one K
// range (large T): E = 64 on single CTAs, or E = 128 / 256 on CTA pairs (the pair protocol of
// route_gemm_kernel). The selection that a top-k kernel would run after a round trip of fp32
// logits through memory runs in the epilogue warps instead, on one tile's logits while the MMAs
// of the CTA's next tile run: two TMEM accumulator buffers (each the even/odd K-step pair of
// route_gemm_kernel when N <= 128, else one accumulator of N columns). Epilogue thread
// q * 32 + lane owns TMEM lane (token) q * 32 + lane of its CTA's rows: it reads its logits 32
// experts at a time (the two K-step accumulators added, as in route_gemm_kernel), adds the
// bias, writes the logits when asked and inserts them in ascending expert order into a
// TopList, then writes the picks and their weights; the result equals the two-kernel router's
// bit for bit. The buffer goes back to the MMA issuer after the last 32-expert chunk is read.
template <int KL, bool PAIR>
__global__ void __launch_bounds__(kRtThreads, 1)
    route_gemm_topk_kernel(const __grid_constant__ CUtensorMap tmX,
                           const __grid_constant__ CUtensorMap tmW, const RtParams p,
                           int tmem_cols, const float* __restrict__ bias,
                           float* __restrict__ logits_out, int k, int32_t* __restrict__ topk_idx,
                           float* __restrict__ topk_w) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int b_bytes = p.nch * 8192;
  const int stage_bytes = 16384 + b_bytes;
  const int S = p.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(S) * stage_bytes);
  uint64_t* empty = full + kRtMaxStages;
  uint64_t* tfull = empty + kRtMaxStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* done = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = (rank == 0);
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&tfull[b]), 1);
      // one arrival per epilogue warp (of both CTAs in PAIR mode, on the even CTA's barrier)
      mbar_init(smem_u32(&tempty[b]), PAIR ? 8 : 4);
    }
    mbar_init(smem_u32(done), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(smem_u32(tmem_holder), static_cast<uint32_t>(tmem_cols));
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_holder), static_cast<uint32_t>(tmem_cols));
      tmem_relinquish();
    }
  }
  pdl_enter<false>();
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync_all();  // both CTAs' barriers are initialised
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  constexpr int kTileRows = PAIR ? 2 * kRtM : kRtM;
  const int ntiles = (p.T + kTileRows - 1) / kTileRows;
  const int tile0 = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int tstep = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  const int nkb = p.kb_per_split;  // the whole hidden dimension
  const int cb = p.two_acc ? 2 * p.npad : p.npad;  // TMEM columns per accumulator buffer

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t s = 0, ph = 0;
      // in PAIR mode the even CTA's barrier expects both CTAs' bytes
      const uint32_t tx = static_cast<uint32_t>(stage_bytes) * (PAIR ? 2u : 1u);
      const int c0 = static_cast<int>(rank) * p.nch;  // first expert chunk this CTA loads
      bool ok = true;
      int issued = 0;
      for (int tile = tile0; ok && tile < ntiles; tile += tstep) {
        const int row0 = tile * kTileRows + static_cast<int>(rank) * kRtM;
        for (int i = 0; i < nkb; ++i) {
          if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t sa = smem_u32(smem + static_cast<size_t>(s) * stage_bytes);
          const int kc = i * kRtBK;
          if constexpr (PAIR) {
            const uint32_t fb = mapa_shared(smem_u32(&full[s]), 0);
            if (leader) mbar_arrive_expect_tx(smem_u32(&full[s]), tx);
            tma_load_2d_pair(sa, &tmX, kc, row0, fb);
            for (int c = 0; c < p.nch; ++c)
              tma_load_2d_pair(sa + 16384 + c * 8192, &tmW, (c0 + c) * 64, kc, fb);
          } else {
            const uint32_t fb = smem_u32(&full[s]);
            mbar_arrive_expect_tx(fb, tx);
            tma_load_2d(sa, &tmX, kc, row0, fb);
            for (int c = 0; c < p.nch; ++c)
              tma_load_2d(sa + 16384 + c * 8192, &tmW, (c0 + c) * 64, kc, fb);
          }
          ++issued;
          if (++s == static_cast<uint32_t>(S)) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        flag_error(p.err, kDevWaitTimeout);
      }
      // Every load issued lands before the CTA may exit. In PAIR mode the loads complete on the
      // even CTA's barriers; the cluster barrier at the end keeps the odd CTA alive until then.
      if (!PAIR || leader) {
        for (int i = (issued > S ? issued - S : 0); i < issued; ++i)
          mbar_wait_cluster(smem_u32(&full[i % S]), static_cast<uint32_t>(i / S) & 1u, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (whole warp)
    if (leader) {
      constexpr uint32_t kFull = 0xffffffffu;
      const uint32_t sbase = smem_u32(smem);
      const uint64_t adesc0 = smem_desc_sw128(sbase, 16, 1024);            // x rows, K-major
      const uint64_t bdesc0 = smem_desc_sw128(sbase + 16384, 8192, 1024);  // Wr, MN-major
      const uint32_t idesc = idesc_bf16(kTileRows, p.npad, /*a_mn_major=*/false,
                                        /*b_mn_major=*/true);
      uint32_t s = 0, ph = 0, soff = 0;
      bool ok = true;
      int tc = 0;
      for (int tile = tile0; ok && tile < ntiles; tile += tstep, ++tc) {
        const int buf = tc & 1;
        const uint32_t use = static_cast<uint32_t>(tc >> 1);
        if (!__all_sync(kFull, mbar_wait_cluster(smem_u32(&tempty[buf]), (use & 1u) ^ 1u,
                                                 abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d0 = tmem_base + static_cast<uint32_t>(buf * cb);
        const uint32_t d1 = d0 + static_cast<uint32_t>(p.npad);
        uint32_t acc0 = 0, acc1 = 0;
        for (int i = 0; i < nkb; ++i) {
          if (!__all_sync(kFull, mbar_wait_cluster(smem_u32(&full[s]), ph, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = adesc0 + (soff >> 4);
          const uint64_t bd = bdesc0 + (soff >> 4);
#pragma unroll
          for (int kk = 0; kk < kRtBK / 16; ++kk) {
            const bool second = p.two_acc && (kk & 1);
            const uint32_t d = second ? d1 : d0;
            const uint32_t acc = second ? acc1 : acc0;
            if constexpr (PAIR) tc_mma_bf16_pair_elect(d, ad + kk * 2, bd + kk * 128, idesc, acc);
            else tc_mma_bf16_elect(d, ad + kk * 2, bd + kk * 128, idesc, acc);
            if (second) acc1 = 1u;
            else acc0 = 1u;
          }
          if constexpr (PAIR) tc_commit_pair_mc_elect(smem_u32(&empty[s]), 0x3);
          else tc_commit_elect(smem_u32(&empty[s]));
          if (++s == static_cast<uint32_t>(S)) {
            s = 0;
            ph ^= 1u;
            soff = 0;
          } else {
            soff += static_cast<uint32_t>(stage_bytes);
          }
        }
        if (!ok) break;
        if constexpr (PAIR) tc_commit_pair_mc_elect(smem_u32(&tfull[buf]), 0x3);
        else tc_commit_elect(smem_u32(&tfull[buf]));
      }
      if (!ok && lane == 0) {
        *abort_flag = 1;
        flag_error(p.err, kDevWaitTimeout);
      }
      // completes once every MMA issued has finished (also when the loop stopped early)
      if constexpr (PAIR) tc_commit_pair_mc_elect(smem_u32(done), 0x3);
      else tc_commit_elect(smem_u32(done));
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue + top-k (warps 2..5)
    const int q = warp & 3;
    int tc = 0;
    for (int tile = tile0; tile < ntiles; tile += tstep, ++tc) {
      const int buf = tc & 1;
      const uint32_t use = static_cast<uint32_t>(tc >> 1);
      int got = 1;
      if (lane == 0) got = mbar_wait_cluster(smem_u32(&tfull[buf]), use & 1u, abort_flag) ? 1 : 0;
      got = __shfl_sync(0xffffffffu, got, 0);
      if (!got) {
        if (lane == 0) {
          *abort_flag = 1;
          flag_error(p.err, kDevWaitTimeout);
        }
        break;
      }
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                          static_cast<uint32_t>(buf * cb);
      const int64_t t = static_cast<int64_t>(tile) * kTileRows + static_cast<int>(rank) * kRtM +
                        q * 32 + lane;
      const bool mine = t < p.T;
      TopList<KL> L;
      L.clear();
      for (int c0 = 0; c0 < p.E; c0 += 32) {  // uniform; E % 32 == 0
        uint32_t v[32];
        tmem_ld32(tb + static_cast<uint32_t>(c0), v);
        if (p.two_acc) {
          uint32_t u[32];
          tmem_ld32(tb + static_cast<uint32_t>(p.npad + c0), u);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j)
            v[j] = __float_as_uint(__uint_as_float(v[j]) + __uint_as_float(u[j]));
        } else {
          tmem_wait_ld();
        }
        if (mine) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int e = c0 + j;
            float val = __uint_as_float(v[j]);
            if (bias != nullptr) val += __ldg(bias + e);
            if (logits_out != nullptr) logits_out[t * p.E + e] = val;
            L.insert(order_key(val), e);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (PAIR) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[buf]), 0));
        else mbar_arrive(smem_u32(&tempty[buf]));
      }
      if (mine) thread_write_selection<KL>(L.key, L.idx, k, 0, 1, topk_idx + t * k, topk_w + t * k);
    }
  }

  // TMEM is released only after every MMA issued has completed (the commit reaches both CTAs)
  if (warp == 1 && lane == 0) mbar_wait_cluster(smem_u32(done), 0u, nullptr);
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync_all();  // no CTA leaves while its peer may still signal it
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, static_cast<uint32_t>(tmem_cols));
    else tmem_dealloc(tmem_base, static_cast<uint32_t>(tmem_cols));
  }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// bf16 [rows, cols] row-major, box {64 columns, box_rows rows}, 128-byte swizzle; elements
// outside the tensor read as zero.
bool map_2d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows,
            std::string* d) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) {
    if (d) *d = "cuTensorMapEncodeTiled is not available from the driver";
    return false;
  }
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS && d)
    *d = "cuTensorMapEncodeTiled(router operand) failed with code " + std::to_string(r);
  return r == CUDA_SUCCESS;
}

}  // namespace

// CTA pairs need whole 64-expert chunks in each half of B.
bool route_uses_pairs(int E) { return E % 128 == 0; }

int route_ksplit(int64_t T, int H, int E) {
  const int64_t kb_total = H / kRtBK;
  // CTAs per K range: one per 128 tokens, rounded up to whole pairs when pairs are used
  int64_t ctas = (T + kRtM - 1) / kRtM;
  if (route_uses_pairs(E)) ctas = 2 * ((T + 2 * kRtM - 1) / (2 * kRtM));
  int ks = 1;
  // split K while the grid stays within about 128 CTAs and each range keeps >= 4 k-blocks
  while (ks * 2 <= 16 && kb_total % (ks * 2) == 0 && kb_total / (ks * 2) >= 4 &&
         ctas * ks * 2 <= 128)
    ks *= 2;
  return ks;
}

cudaError_t launch_route_gemm_tc(const void* x, const void* w_router, int T, int H, int E,
                                 float* partials, int ksplit, int* err, int num_sms,
                                 cudaStream_t stream, std::string* detail) {
  (void)num_sms;
  if (T == 0) return cudaSuccess;
  if (E < 16 || E > 256 || E % 8 != 0 || H % kRtBK != 0 || (H / kRtBK) % ksplit != 0) {
    if (detail) *detail = "router GEMM shape outside the tensor-core path";
    return cudaErrorInvalidValue;
  }
  const bool pair = route_uses_pairs(E);
  CUtensorMap mx, mw;
  if (!map_2d(&mx, x, static_cast<uint64_t>(H), static_cast<uint64_t>(T), kRtM, detail) ||
      !map_2d(&mw, w_router, static_cast<uint64_t>(E), static_cast<uint64_t>(H), kRtBK, detail))
    return cudaErrorInvalidValue;
  RtParams p{};
  p.T = T;
  p.H = H;
  p.E = E;
  p.npad = (E + 15) & ~15;
  p.nch = pair ? E / 128 : (E + 63) / 64;
  p.kb_per_split = H / kRtBK / ksplit;
  p.two_acc = (2 * p.npad <= kRtTmemCols) ? 1 : 0;
  p.split_stride = static_cast<int64_t>(T) * E;
  p.out = partials;
  p.err = err;
  const int stage_bytes = 16384 + p.nch * 8192;
  int stages = (kRtSmemLimit - 1024 - kRtCtrl) / stage_bytes;
  if (stages > kRtMaxStages) stages = kRtMaxStages;
  if (stages > p.kb_per_split) stages = p.kb_per_split;
  if (stages < 2) stages = 2;
  p.stages = stages;
  const size_t smem = 1024 + static_cast<size_t>(stages) * stage_bytes + kRtCtrl;
  auto kernel = pair ? route_gemm_kernel<true> : route_gemm_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const unsigned tiles = pair ? 2u * static_cast<unsigned>((T + 2 * kRtM - 1) / (2 * kRtM))
                              : static_cast<unsigned>((T + kRtM - 1) / kRtM);
  const dim3 grid(tiles, static_cast<unsigned>(ksplit));
  return launch_kernel(kernel, grid, dim3(kRtThreads), smem, stream, pair ? 2 : 1, mx, mw, p);
}

bool route_fuses_topk(int64_t T, int H, int E, int k, int n_group) {
  const bool shape_ok = E == 64 || (E % 128 == 0 && E <= 256);
  return shape_ok && n_group <= 1 && k <= 16 && H % kRtBK == 0 && route_ksplit(T, H, E) == 1;
}

cudaError_t launch_route_gemm_topk_tc(const void* x, const void* w_router, int T, int H, int E,
                                      int k, const float* bias, float* logits_out,
                                      int32_t* topk_idx, float* topk_w, int* err, int num_sms,
                                      cudaStream_t stream, std::string* detail) {
  if (T == 0) return cudaSuccess;
  const bool pair = route_uses_pairs(E);
  if (!(E == 64 || (pair && E <= 256)) || H % kRtBK != 0 || k < 1 || k > 16) {
    if (detail) *detail = "fused router shape outside the tensor-core path";
    return cudaErrorInvalidValue;
  }
  CUtensorMap mx, mw;
  if (!map_2d(&mx, x, static_cast<uint64_t>(H), static_cast<uint64_t>(T), kRtM, detail) ||
      !map_2d(&mw, w_router, static_cast<uint64_t>(E), static_cast<uint64_t>(H), kRtBK, detail))
    return cudaErrorInvalidValue;
  RtParams p{};
  p.T = T;
  p.H = H;
  p.E = E;
  p.npad = E;
  p.nch = pair ? E / 128 : E / 64;
  p.kb_per_split = H / kRtBK;
  p.two_acc = (E <= 128) ? 1 : 0;  // two K-step accumulators per buffer while 2E <= 256
  p.split_stride = 0;
  p.out = nullptr;
  p.err = err;
  // two accumulator buffers: 2 * (2E or E) columns, a power of two (256 or 512)
  const int tmem_cols = 2 * (p.two_acc ? 2 * E : E);
  const int stage_bytes = 16384 + p.nch * 8192;
  int stages = (kRtSmemLimit - 1024 - kRtCtrl) / stage_bytes;
  if (stages > kRtMaxStages) stages = kRtMaxStages;
  if (stages > p.kb_per_split) stages = p.kb_per_split;
  if (stages < 2) stages = 2;
  p.stages = stages;
  const size_t smem = 1024 + static_cast<size_t>(stages) * stage_bytes + kRtCtrl;
  auto pick = [&](auto tag) {
    constexpr bool P = decltype(tag)::value;
    auto kernel = route_gemm_topk_kernel<16, P>;
    if (k <= 2) kernel = route_gemm_topk_kernel<2, P>;
    else if (k <= 4) kernel = route_gemm_topk_kernel<4, P>;
    else if (k <= 6) kernel = route_gemm_topk_kernel<6, P>;
    else if (k <= 8) kernel = route_gemm_topk_kernel<8, P>;
    return kernel;
  };
  auto kernel = pair ? pick(std::true_type{}) : pick(std::false_type{});
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int tiles = pair ? (T + 2 * kRtM - 1) / (2 * kRtM) : (T + kRtM - 1) / kRtM;
  const int units = pair ? num_sms / 2 : num_sms;
  const int grid = (tiles < units ? tiles : units) * (pair ? 2 : 1);
  return launch_kernel(kernel, dim3(static_cast<unsigned>(grid)), dim3(kRtThreads), smem, stream,
                       pair ? 2 : 1, mx, mw, p, tmem_cols, bias, logits_out, k, topk_idx, topk_w);
}

}  // namespace moe
