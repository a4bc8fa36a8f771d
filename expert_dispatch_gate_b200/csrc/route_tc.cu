// route_tc.cu — the router in one launch on the tensor cores (tcgen05 + TMEM + TMA), sm_100a:
// gate GEMM, softmax/top-k selection and the renormalised weights.
//
// [P4] "MoE Router" (2048ai.net), section "Router 就是一个小型网络": the gate is a bias-free
// Linear layer, logits[t, e] = sum_h x[t, h] * Wr[h, e], then softmax, top-k and division of the
// k kept weights by their sum. [P5] "大模型推理加速200%+？…", section "3.1 Moe Fuse Gate & Softmax
// TopK": gate, softmax and top-k fused in one kernel, exp only for the k selected logits.
//
// Orientation: tokens on the MMA's M side (128 per CTA, one TMEM lane each), experts on N
// (E <= 256, padded to a multiple of 16). A = x rows (K-major, 128-byte swizzle), B = Wr
// (expert-contiguous rows, so MN-major; 64-expert chunks of 8 KB per 64-row k-block). When
// N <= 128 the four 16-deep MMAs of a k-block alternate between two accumulators (even / odd K
// steps), which keeps two accumulate chains in flight; the drain adds the two.
//
// One cluster covers one token tile: `ks` K ranges (cluster y) x (1 CTA, or a CTA pair along
// cluster x when E % 128 == 0). Each CTA accumulates its K range of its 128 tokens x E experts in
// TMEM, then
//   1. drains TMEM into shared memory (fp32 [128][E + 4]), reusing the operand ring;
//   2. after a cluster barrier, takes 128 / ks of the tile's tokens and sums their logits over
//      the ks CTAs holding the same tokens (ascending K range) through distributed shared memory,
//      adds the optional bias, writes the logits when asked, and selects the top k with one warp
//      per token (select.cuh), writing topk_idx and topk_w;
//   3. waits at a second cluster barrier so that no CTA's shared memory goes away while a peer
//      still reads it.
// Partial logits never reach global memory, and the selection needs no second launch.
//
// CTA pairs (E % 128 == 0): the two CTAs of a pair share a 256-token tile with
// tcgen05.mma.cta_group::2 (M = 256). Each loads its own 128 token rows (A) and half of the
// expert chunks of Wr (B); both CTAs' loads complete on the even CTA's `full` barrier, the even
// CTA issues the MMAs, and its commits arrive on both CTAs' `empty` and `done` barriers. Per CTA
// and k-block that is 16 KB of x and 16 KB of Wr instead of 16 + 32 KB.
//
// Warps: 0 TMA producer, 1 MMA issuer (converged warp, elected lane), 2-9 TMEM drain (two warps
// per lane quadrant, alternate 32-column chunks), all 12 select.
#include <cuda.h>

#include <math.h>

#include <map>
#include <mutex>
#include <string>
#include <utility>

#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace moe {
namespace {

constexpr int kRtM = 128;          // tokens per CTA
constexpr int kRtBK = 64;          // K per stage (one 128-byte swizzle row of bf16)
constexpr int kRtMaxStages = 8;
constexpr int kRtWarps = 12;
constexpr int kRtThreads = 32 * kRtWarps;
constexpr int kRtTmemCols = 256;
constexpr int kRtSmemLimit = 227 * 1024;
constexpr int kRtCtrl = 256;
constexpr int kRtMaxCluster = 8;   // portable cluster size: CTAs per tile x K ranges

struct RtParams {
  int T, H, E;
  int npad;            // N of the MMA: E rounded up to 16
  int nch;             // 64-expert chunks of B loaded per stage by this CTA
  int kb_per_split;    // k-blocks of one K range
  int ks;              // K ranges (cluster y extent)
  int two_acc;         // 1: alternate two accumulators over K steps
  int stages;
  int srow;            // staging row stride in floats (E + 4)
  const float* bias;   // [E] or null
  float* logits_out;   // [T][E] or null
  int32_t* topk_idx;   // [T][k]
  float* topk_w;       // [T][k]
  int k, n_group, topk_group;
  int* err;
};

template <bool PAIR, int VPL>
__global__ void __launch_bounds__(kRtThreads, 1)
    route_fused_kernel(const __grid_constant__ CUtensorMap tmX,
                       const __grid_constant__ CUtensorMap tmW, const RtParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int b_bytes = p.nch * 8192;
  const int stage_bytes = 16384 + b_bytes;
  const int S = p.stages;
  const size_t ring = static_cast<size_t>(S) * stage_bytes;
  const size_t staging = static_cast<size_t>(kRtM) * p.srow * 4;
  uint8_t* ctrl = smem + (ring > staging ? ring : staging);
  uint64_t* full = reinterpret_cast<uint64_t*>(ctrl);
  uint64_t* empty = full + kRtMaxStages;
  uint64_t* done = empty + kRtMaxStages;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  float* stage_f = reinterpret_cast<float*>(smem);  // staging [kRtM][srow], after the mainloop

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t half = PAIR ? (rank & 1u) : 0u;
  const uint32_t pair0 = rank - half;              // cluster rank of the pair's even CTA
  const bool leader = (half == 0);
  const uint16_t pair_mask = static_cast<uint16_t>(3u << pair0);
  const bool clustered = PAIR || p.ks > 1;
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
  if (clustered) cluster_sync_all();  // every CTA's barriers are initialised
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int row0 = PAIR ? static_cast<int>(blockIdx.x >> 1) * (2 * kRtM) +
                              static_cast<int>(half) * kRtM
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
      const int c0 = static_cast<int>(half) * p.nch;  // first expert chunk this CTA loads
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
          const uint32_t fb = mapa_shared(smem_u32(&full[s]), pair0);
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
      // Every load issued lands before the shared memory is reused or the CTA exits. In PAIR
      // mode the loads complete on the even CTA's barriers; the odd CTA's loads are covered by
      // the even CTA's wait here and the cluster barriers that follow.
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
        if constexpr (PAIR) tc_commit_pair_mc_elect(smem_u32(&empty[s]), pair_mask);
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
      if constexpr (PAIR) tc_commit_pair_mc_elect(smem_u32(done), pair_mask);
      else tc_commit_elect(smem_u32(done));
    }
    __syncwarp();
  }

  // ---------------------------------------------------------------- 1. drain TMEM -> staging
  // The ring is free once `done` has completed (every load was consumed by a finished MMA) and
  // the producer has seen its last loads land (the barrier below).
  __syncthreads();
  if (warp >= 2 && warp < 10) {
    const int q = warp & 3;            // TMEM lane quadrant this warp may read
    const int hf = (warp - 2) >> 2;    // which alternate 32-column chunks it drains
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
      float* srow = stage_f + static_cast<size_t>(q * 32 + lane) * p.srow;
      for (int c0 = 32 * hf; c0 < p.E; c0 += 64) {
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
        // E % 8 == 0: whole 16-byte groups
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          if (c0 + j < p.E)
            *reinterpret_cast<float4*>(srow + c0 + j) =
                make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                            __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (clustered) cluster_sync_all();  // every CTA of the tile has staged its partial logits

  // ---------------------------------------------------------------- 2. reduce + select
  // This CTA takes rows [r0, r1) of its 128 tokens; the ks CTAs holding the same tokens (same
  // pair half) are cluster ranks half + (PAIR ? 2 : 1) * y, y = 0 .. ks-1.
  if (!*abort_flag) {
    const int per = kRtM / p.ks;
    const int r0 = ks * per;
    const int e0 = VPL * lane;
    const bool mine = e0 < p.E;  // E % VPL == 0 on this path: a lane's run is whole or absent
    const uint32_t stage_u32 = smem_u32(stage_f);
    for (int r = r0 + warp; r < r0 + per; r += kRtWarps) {
      const int t = row0 + r;
      if (t >= p.T) break;
      float v[VPL];
      uint32_t taken = 0;
#pragma unroll
      for (int i = 0; i < VPL; ++i) v[i] = 0.f;
      if (mine) {
        const uint32_t off = stage_u32 + static_cast<uint32_t>((r * p.srow + e0) * 4);
        for (int y = 0; y < p.ks; ++y) {
          const uint32_t src = mapa_shared(off, half + (PAIR ? 2u : 1u) * static_cast<uint32_t>(y));
          float part[VPL];
          if constexpr (VPL >= 4) {
#pragma unroll
            for (int i = 0; i < VPL; i += 4) {
              const float4 f = ld_shared_cluster_f32x4(src + i * 4);
              part[i] = f.x;
              part[i + 1] = f.y;
              part[i + 2] = f.z;
              part[i + 3] = f.w;
            }
          } else if constexpr (VPL == 2) {
            const float2 f = ld_shared_cluster_f32x2(src);
            part[0] = f.x;
            part[1] = f.y;
          } else {
            part[0] = ld_shared_cluster_f32(src);
          }
#pragma unroll
          for (int i = 0; i < VPL; ++i) v[i] = (y == 0) ? part[i] : v[i] + part[i];
        }
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
          if (p.bias != nullptr) v[i] += __ldg(p.bias + e0 + i);
        }
        if (p.logits_out != nullptr) {
          float* lo = p.logits_out + static_cast<size_t>(t) * p.E + e0;
          if constexpr (VPL >= 4) {
#pragma unroll
            for (int i = 0; i < VPL; i += 4)
              *reinterpret_cast<float4*>(lo + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
          } else {
#pragma unroll
            for (int i = 0; i < VPL; ++i) lo[i] = v[i];
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < VPL; ++i) v[i] = -INFINITY;
        taken = (1u << VPL) - 1u;
      }
      if (p.n_group > 1) taken |= warp_group_exclude<VPL>(v, p.E, p.n_group, p.topk_group, lane);
      warp_select_topk<VPL>(v, taken, p.k, lane, p.topk_idx + static_cast<size_t>(t) * p.k,
                            p.topk_w + static_cast<size_t>(t) * p.k);
    }
  }

  // ---------------------------------------------------------------- teardown
  // The MMA completion barrier also guards TMEM release when the drain gave up early.
  if (warp == 1 && lane == 0) mbar_wait_cluster(smem_u32(done), 0u, nullptr);
  tc_fence_before();
  __syncthreads();
  if (clustered) cluster_sync_all();  // no CTA leaves while a peer may still read or signal it
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, kRtTmemCols);
    else tmem_dealloc(tmem_base, kRtTmemCols);
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


// CTA pairs need whole 64-expert chunks in each half of B.
bool route_uses_pairs(int E) { return E % 128 == 0; }

struct RtConfig {
  bool pair;
  int ks, stages;
  size_t smem;
};

// Shared memory of one CTA: the operand ring, or the logit staging that reuses it, plus control.
RtConfig rt_config(bool pair, int ks, int H, int E) {
  RtConfig c{pair, ks, 0, 0};
  const int nch = pair ? E / 128 : (E + 63) / 64;
  const int stage_bytes = 16384 + nch * 8192;
  const int kb_per_split = H / kRtBK / ks;
  int stages = (kRtSmemLimit - 1024 - kRtCtrl) / stage_bytes;
  if (stages > kRtMaxStages) stages = kRtMaxStages;
  if (stages > kb_per_split) stages = kb_per_split;
  if (stages < 2) stages = 2;
  c.stages = stages;
  const size_t ring = static_cast<size_t>(stages) * stage_bytes;
  const size_t staging = static_cast<size_t>(kRtM) * (E + 4) * 4;
  c.smem = 1024 + (ring > staging ? ring : staging) + kRtCtrl;
  return c;
}

template <bool PAIR, int VPL>
cudaError_t rt_launch(const RtConfig& c, const CUtensorMap& mx, const CUtensorMap& mw,
                      const RtParams& p, unsigned tiles, cudaStream_t stream) {
  auto kernel = route_fused_kernel<PAIR, VPL>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(c.smem));
  if (e != cudaSuccess) return e;
  const dim3 grid(tiles * (PAIR ? 2u : 1u), static_cast<unsigned>(c.ks));
  const dim3 cluster(PAIR ? 2u : 1u, static_cast<unsigned>(c.ks), 1u);
  return launch_kernel_clusters(kernel, grid, dim3(kRtThreads), c.smem, stream, cluster, mx, mw,
                                p);
}

// Clusters of this configuration that the GPU holds at once (cudaOccupancyMaxActiveClusters),
// cached per configuration; 0 when the query fails.
template <bool PAIR, int VPL>
int rt_max_clusters(const RtConfig& c) {
  static std::mutex mu;
  static std::map<std::pair<int, size_t>, int> cache;  // (ks, shared memory bytes) -> clusters
  std::lock_guard<std::mutex> lk(mu);
  int& slot = cache[{c.ks, c.smem}];
  if (slot != 0) return slot - 1;
  auto kernel = route_fused_kernel<PAIR, VPL>;
  int n = 0;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(c.smem)) == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    const unsigned cl = (PAIR ? 2u : 1u) * static_cast<unsigned>(c.ks);
    cfg.gridDim = dim3(cl * 64u, 1, 1);
    cfg.blockDim = dim3(kRtThreads);
    cfg.dynamicSmemBytes = c.smem;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = cl;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
  }
  slot = n + 1;
  return n;
}

// The launch layout for T tokens: among CTA pairs (E % 128 == 0) or single CTAs, and K split
// into ks = 1, 2, 4 or 8 ranges (one tile's cluster <= 8 CTAs, each range >= 4 k-blocks), the one
// with the most CTAs whose clusters all fit on the GPU at once (one wave), pairs first on a tie.
// When no layout fits in one wave (large T), the tiles run in waves with ks = 1.
template <int VPL>
RtConfig choose_config(int T, int H, int E, bool can_pair) {
  const int kb_total = H / kRtBK;
  RtConfig best{};
  long best_ctas = -1;
  for (int pi = 0; pi < 2; ++pi) {
    const bool pair = (pi == 0);
    if (pair && !can_pair) continue;
    const long tiles = pair ? (T + 2 * kRtM - 1) / (2 * kRtM) : (T + kRtM - 1) / kRtM;
    for (int ks = 1; ks <= 8; ks *= 2) {
      if ((pair ? 2 : 1) * ks > kRtMaxCluster || kb_total % ks != 0) continue;
      if (ks > 1 && kb_total / ks < 4) continue;
      if (ks > 1 && kRtM % ks != 0) continue;
      const RtConfig c = rt_config(pair, ks, H, E);
      if (c.smem > static_cast<size_t>(kRtSmemLimit)) continue;
      const int maxc = pair ? rt_max_clusters<true, VPL>(c) : rt_max_clusters<false, VPL>(c);
      if (tiles > maxc) continue;
      const long ctas = tiles * (pair ? 2 : 1) * ks;
      if (ctas > best_ctas) {
        best = c;
        best_ctas = ctas;
      }
    }
  }
  if (best_ctas < 0) best = rt_config(can_pair, 1, H, E);
  return best;
}

}  // namespace

cudaError_t launch_route_tc(const void* x, const void* w_router, const float* bias, int T, int H,
                            int E, int k, int n_group, int topk_group, float* logits_out,
                            int32_t* topk_idx, float* topk_w, int* err, cudaStream_t stream,
                            std::string* detail) {
  if (T == 0) return cudaSuccess;
  if (E < 16 || E > 256 || E % 8 != 0 || H % kRtBK != 0) {
    if (detail) *detail = "router shape outside the tensor-core path";
    return cudaErrorInvalidValue;
  }
  const bool can_pair = route_uses_pairs(E);
  const int vpl = E <= 32 ? 1 : E <= 64 ? 2 : E <= 128 ? 4 : 8;  // experts per lane (select)
  RtConfig c;
  switch (vpl) {
    case 1: c = choose_config<1>(T, H, E, can_pair); break;
    case 2: c = choose_config<2>(T, H, E, can_pair); break;
    case 4: c = choose_config<4>(T, H, E, can_pair); break;
    default: c = choose_config<8>(T, H, E, can_pair); break;
  }
  if (c.smem > static_cast<size_t>(kRtSmemLimit)) {
    if (detail) *detail = "router tile does not fit in shared memory";
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
  p.npad = (E + 15) & ~15;
  p.nch = c.pair ? E / 128 : (E + 63) / 64;
  p.kb_per_split = H / kRtBK / c.ks;
  p.ks = c.ks;
  p.two_acc = (2 * p.npad <= kRtTmemCols) ? 1 : 0;
  p.stages = c.stages;
  p.srow = E + 4;
  p.bias = bias;
  p.logits_out = logits_out;
  p.topk_idx = topk_idx;
  p.topk_w = topk_w;
  p.k = k;
  p.n_group = n_group;
  p.topk_group = topk_group;
  p.err = err;
  const unsigned tiles = c.pair ? static_cast<unsigned>((T + 2 * kRtM - 1) / (2 * kRtM))
                                : static_cast<unsigned>((T + kRtM - 1) / kRtM);
  // lane l of a selecting warp holds experts VPL*l ... VPL*l + VPL - 1
  if (c.pair) {
    if (vpl == 4) return rt_launch<true, 4>(c, mx, mw, p, tiles, stream);
    return rt_launch<true, 8>(c, mx, mw, p, tiles, stream);
  }
  switch (vpl) {
    case 1: return rt_launch<false, 1>(c, mx, mw, p, tiles, stream);
    case 2: return rt_launch<false, 2>(c, mx, mw, p, tiles, stream);
    case 4: return rt_launch<false, 4>(c, mx, mw, p, tiles, stream);
    default: return rt_launch<false, 8>(c, mx, mw, p, tiles, stream);
  }
}

}  // namespace moe
