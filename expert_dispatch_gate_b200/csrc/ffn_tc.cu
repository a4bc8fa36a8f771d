// ffn_tc.cu — grouped expert GEMMs (and the E >= 64 router GEMM) on the B200 tensor cores.
//
// [P1] "MoE 模型的 FlashAttention 跟普通模型有什么不一样？", section "FlashAttention 在 MoE 模型里的位置",
// step 4: each expert runs its FFN on the tokens grouped to it. Here the FFN is SwiGLU,
// h = silu(x Wg) * (x Wu), y = h Wd ([P1] section "手动编译 MoE 融合算子": activation="silu").
//
// Design (sm_100a):
//   * swap-AB: the weight matrix is the MMA's A operand (M = 128 output features per tile) and
//     the expert's tokens are the B operand (N = tokens of the tile, padded to 16). An expert's
//     weights are streamed from HBM once per tile, whatever its token count; a decode step with
//     one token per expert pays for N = 16 columns of MMA, not 128 rows.
//   * A (weights, MN-major: features contiguous) arrives by 3-D TMA tiles of 64x64 bf16 with
//     128-byte swizzle. B (token rows, K-major, same swizzle) arrives in one of three ways:
//       - contiguous rows (router: x rows; GEMM2: slot-major h rows): 2-D TMA boxes of 32 rows;
//       - gathered rows by cp.async from four producer warps that read the grouping's
//         slot -> token map and write the swizzled layout themselves (GEMM1: x rows straight
//         from the unpermuted activations, so no permuted copy of x is ever written);
//       - gathered rows by TMA tile::gather4 (four rows per instruction; kept as an option).
//   * tcgen05.mma accumulates in TMEM (fp32); GEMM1 keeps gate and up accumulators side by side
//     so one epilogue thread owns both values of a (feature, token) pair and applies SwiGLU.
//   * Persistent CTAs (one per SM), warp-specialised: warp 0 issues TMA, warp 1 issues MMAs,
//     warps 2-5 drain TMEM. Tiles are ordered (expert, feature block, token block) so the token
//     blocks that share a weight slice run at the same time and hit it in L2.
//   * Every mbarrier wait is bounded; on timeout the CTA raises an error word and winds down.
#include <mutex>

#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kBM = 128;        // MMA M: output features per tile
constexpr int kBK = 64;         // K per pipeline stage: one 128-byte swizzle row of bf16
constexpr int kMaxStages = 8;
constexpr int kMaxGroups = 256;
constexpr int kTmemCols = 512;
constexpr int kSmemLimit = 232448;  // 227 KB opt-in dynamic shared memory per block
constexpr int kCtrlBytes = 2560;    // barriers + group tables

// Epilogue / operand modes:
//   kEpiSwiGLU: two A operands (gate, up) of the same 128 features; h = silu(g) * u (bf16).
//   kEpiBF16:   one A operand, 128 features; y stored as bf16.
//   kEpiBF16x2: two A operands = features [m0, m0+128) and [m0+128, m0+256) of one weight; both
//               accumulators share the B tile, halving B traffic per weight byte; bf16 out.
enum EpiMode { kEpiSwiGLU = 0, kEpiBF16 = 1, kEpiBF16x2 = 3 };
template <int MODE>
constexpr bool dual_a() { return MODE == kEpiSwiGLU || MODE == kEpiBF16x2; }
template <int MODE>
constexpr int tile_features() { return MODE == kEpiBF16x2 ? 256 : 128; }
// How the B operand (token rows) reaches shared memory.
enum BMode { kBGather4 = 0, kBTiled = 1, kBCpAsync = 2 };

// Warps: 0 TMA producer, 1 MMA issuer, 2-9 epilogue (two warps per TMEM lane quadrant, each
// draining half of the token columns), 10-13 cp.async row gatherers (kBCpAsync).
constexpr int kEpiWarps = 8;
// 32-column chunks one epilogue warp drains per tile: columns 32*half + 64*i, i < 4, cover
// every token block of up to 256 rows.
constexpr int kEpiChunks = 4;
constexpr int kMaxTokenBlock = 256;
constexpr int kGatherWarp0 = 2 + kEpiWarps;
// W8: FP8 (e4m3) weights, converted to bf16 in shared memory by four converter warps
// (warps 10-13) before the bf16 MMA; the per-channel scale is applied in the epilogue.
template <int BMODE, bool W8 = false>
constexpr int threads_of() { return 32 * (kGatherWarp0 + ((BMODE == kBCpAsync || W8) ? 4 : 0)); }

// Token rows of B one CTA keeps per stage: all TB, or the half it holds in a CTA pair (rounded
// up to whole 32-row TMA boxes).
__host__ __device__ constexpr int b_rows_smem(bool pair, int TB) {
  return pair ? (((TB >> 1) + 31) & ~31) : TB;
}

struct TcParams {
  int K;          // reduction length (multiple of 64)
  int num_fb;     // feature blocks of 128
  int m_valid;    // features stored by the epilogue
  int m_base;     // first feature of feature block 0
  int TB;         // max tokens per tile, multiple of 32, <= 256
  int groups;     // experts
  int k_top;      // GEMM1: B row = sorted_ids[slot] / k_top
  int rows_b;     // rows of the B tensor
  const __nv_bfloat16* b_ptr;  // B tensor [rows_b, K] (cp.async gather)
  const int32_t* sorted_ids;
  const int32_t* offsets;     // [groups+1] slot offsets
  const int32_t* blk_prefix;  // [groups+1] token blocks before each group
  void* out;
  int64_t ldo;
  int* err;
  int stages;
  int nbuf;       // TMEM accumulator buffers (1 or 2, 256 columns apart)
  int b_box_rows; // rows per B box (contiguous-rows mode)
  const float* scale0;  // W8: per-channel scales [groups][scale_ld] of A0 (gate, or down)
  const float* scale1;  // W8: of A1 (up)
  int scale_ld;
  const float* act_scale;  // F8: per-row scale of the B operand (token / slot rows), [rows_b]
};

struct Tile {
  int group, fb, n, row0, kb0, kb1;
};

// Tile order: K range fastest, then token block, then feature block, then group (expert).
__device__ __forceinline__ Tile decode_tile(int tile, int num_fb, int groups, int TB,
                                            const int* s_off, const int* s_blk, int kblocks) {
  int lo = 0, hi = groups;  // largest lo with num_fb * s_blk[lo] <= tile
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (num_fb * s_blk[mid] <= tile) lo = mid; else hi = mid;
  }
  Tile t;
  t.group = lo;
  const int nb = s_blk[lo + 1] - s_blk[lo];
  const int local = tile - num_fb * s_blk[lo];
  t.fb = local / nb;
  const int b = local - t.fb * nb;
  // nb = ceil(cnt / TB) blocks of equal size bs = ceil(cnt / nb) <= TB; every block is non-empty
  // because (nb - 1) * bs <= (nb - 1) * TB < cnt
  const int cnt = s_off[lo + 1] - s_off[lo];
  const int bs = (cnt + nb - 1) / nb;
  t.n = min(bs, cnt - b * bs);
  t.row0 = s_off[lo] + b * bs;
  t.kb0 = 0;
  t.kb1 = kblocks;
  return t;
}

// SiLU(g) = g * sigmoid(g) = g / (1 + e^-g), with the fast-division intrinsic (at most 2 ulp
// in fp32; the result is rounded to bf16 right after). The IEEE-exact division made the
// SwiGLU epilogue hold the accumulator several times longer on tensor-bound shapes. For
// g below about -85 the denominator reaches 2^126 or overflows and the quotient is 0, where
// SiLU itself is below 1e-35 in magnitude.
__device__ __forceinline__ float silu_f32(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// Two e4m3 codes (first in the low byte) as two bf16 (first in the low half). The hardware
// e4m3 -> f16 conversion is exact, and so is f16 -> f32 -> bf16 for these values (at most 4
// significant bits, exponents within bf16's range).
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint16_t codes) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(codes),
                                                    __NV_E4M3);
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
  const __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);
  return *reinterpret_cast<const uint32_t*>(&b);
}

// Round two floats to bf16 (nearest-even) and pack them, the first in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ uint16_t bf16_half(uint32_t w, int hi) {
  return static_cast<uint16_t>(hi ? (w >> 16) : (w & 0xffffu));
}

// PAIR: two CTAs of a cluster cooperate on each tile with tcgen05.mma.cta_group::2 (M = 256).
// Each CTA holds its own feature rows of A (its 128 features, or 256 in kEpiBF16x2) and half of
// the tile's token rows of B; the even CTA issues the MMAs, every CTA reads back its own TMEM
// rows. B traffic per weight byte halves. Stage bookkeeping lives in the even CTA: its full[s]
// counts both CTAs' A bytes (TMA completes there), and its tempty[b] counts both epilogues;
// MMA completions are signalled to both CTAs at once (commit with a two-CTA mask).
//
// W8: A arrives as e4m3 boxes (128 features x 64 K, one byte each) in the stage ring; the
// converter warps rewrite each stage's A as bf16 into a two-slot ring in the layout the bf16
// TMA boxes have (MN-major, 128-byte swizzle), and the MMA reads A from there. Every e4m3 value
// is exactly a bf16 value, so the MMA sees decode(code) exactly; the channel scale multiplies
// the fp32 accumulator in the epilogue.
//
// F8: both operands e4m3 (weights and activations, W8A8) on the native kind::f8f6f4 MMA. The
// weight codes are stored K-major ([E][M][K], the repacked layout), so A and B are both K-major
// 128-byte-swizzled boxes of 128 K values; a stage covers K = 128 with the same bytes as a
// bf16 stage of K = 64, and each of its four MMAs takes K = 32. The epilogue multiplies the fp32
// accumulator by the channel scale of the weights and the row scale of the activations.
template <int MODE, int BMODE, bool PAIR, bool W8 = false, bool F8 = false>
__global__ void __launch_bounds__(threads_of<BMODE, W8>(), 1)
    tc_grouped_gemm(const __grid_constant__ CUtensorMap tmA0,
                    const __grid_constant__ CUtensorMap tmA1,
                    const __grid_constant__ CUtensorMap tmB, const TcParams p) {
  constexpr bool kSwiGLU = (MODE == kEpiSwiGLU);
  constexpr bool kDual = dual_a<MODE>();
  constexpr bool kCp = (BMODE == kBCpAsync);
  // full[s] arrivals: the producer's expect_tx (+ one completion-tracked arrival per cp.async
  // gatherer thread). Pairs stream B by TMA only.
  static_assert(!(PAIR && BMODE != kBTiled), "CTA pairs take the B operand by TMA boxes");
  static_assert(!(W8 && (PAIR || BMODE != kBTiled)), "FP8 weights: single CTAs, TMA-streamed B");
  static_assert(!(F8 && (W8 || BMODE != kBTiled)), "e4m3 operands: TMA-streamed B rows");
  constexpr int kStageK = F8 ? 128 : kBK;  // K elements per stage (128 bytes of a row)
  constexpr uint32_t kFullCount = 1u + (kCp ? 128u : 0u);
  // one arrival per epilogue warp (both CTAs' warps in PAIR mode)
  constexpr uint32_t kTemptyCount = PAIR ? 2u * kEpiWarps : kEpiWarps;
  constexpr int kCtaFeatures = tile_features<MODE>();
  constexpr int kTileFeatures = kCtaFeatures * (PAIR ? 2 : 1);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int a_bytes = kDual ? 32768 : 16384;         // bf16 A of one k-block, as the MMA reads it
  constexpr int a8_bytes = kDual ? 16384 : 8192;     // W8: the same A as e4m3 codes
  const int stage_bytes = (W8 ? a8_bytes : a_bytes) + b_rows_smem(PAIR, p.TB) * 128;
  const int S = p.stages;
  uint8_t* a16 = smem + static_cast<size_t>(S) * stage_bytes;  // W8: two bf16 A slots
  uint8_t* ctrl = a16 + (W8 ? 2 * a_bytes : 0);
  uint64_t* full = reinterpret_cast<uint64_t*>(ctrl);
  uint64_t* empty = full + kMaxStages;
  uint64_t* tfull = empty + kMaxStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  uint64_t* cfull = reinterpret_cast<uint64_t*>(ctrl + 176);  // W8: bf16 slot written
  uint64_t* cempty = cfull + 2;                                // W8: bf16 slot consumed
  int* s_off = reinterpret_cast<int*>(ctrl + 256);
  int* s_blk = s_off + (kMaxGroups + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int groups = p.groups;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = (rank == 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full[s]), kFullCount);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&tfull[b]), 1);
      mbar_init(smem_u32(&tempty[b]), kTemptyCount);
    }
    mbar_init(smem_u32(drain), 1);
    if constexpr (W8) {
      for (int j = 0; j < 2; ++j) {
        mbar_init(smem_u32(&cfull[j]), 4);  // one arrival per converter warp
        mbar_init(smem_u32(&cempty[j]), 1);
      }
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(smem_u32(tmem_holder), kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_holder), kTmemCols);
      tmem_relinquish();
    }
  }
  // Barriers and TMEM are set up while the previous kernel may still be finishing; the group
  // tables (written by the grouping kernels) are read only after the dependency wait.
  pdl_enter<true>();
  for (int i = threadIdx.x; i <= groups; i += blockDim.x) {
    s_off[i] = p.offsets[i];
    s_blk[i] = p.blk_prefix[i];
  }
  if constexpr (kDebugChecks) {
    // the group tables must describe token blocks inside the B rows; otherwise no tile runs
    __syncthreads();
    if (threadIdx.x == 0) {
      bool bad = s_off[0] != 0 || s_blk[0] != 0 || s_off[groups] > p.rows_b;
      for (int g = 0; g < groups && !bad; ++g) {
        const int cnt = s_off[g + 1] - s_off[g], nb = s_blk[g + 1] - s_blk[g];
        bad = cnt < 0 || nb < (cnt + p.TB - 1) / p.TB || nb > cnt;
      }
      if (bad) {
        flag_error(p.err, kDevDebugBounds);
        for (int g = 0; g <= groups; ++g) s_off[g] = s_blk[g] = 0;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync_all();  // barriers of both CTAs are initialised
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int num_tiles = p.num_fb * s_blk[groups];
  // the last stage of an e4m3 operand may reach past K (K % 128 == 64): TMA fills it with zeros
  const int kblocks = (p.K + kStageK - 1) / kStageK;
  const int tile0 = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int tstep = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  // B rows of a tile held by this CTA: all npad rows, or half of them per CTA in PAIR mode
  auto b_rows = [&](int npad) { return PAIR ? (npad >> 1) : npad; };
  auto b_first = [&](int npad) { return PAIR ? static_cast<int>(rank) * (npad >> 1) : 0; };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    int it = 0;
    bool ok = true;
    for (int tile = tile0; ok && tile < num_tiles; tile += tstep) {
      const Tile t = decode_tile(tile, p.num_fb, groups, p.TB, s_off, s_blk, kblocks);
      const int npad = (t.n + 15) & ~15;
      int rows[8];
      if constexpr (BMODE == kBGather4) {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int nn = (lane + 32 * q) * 4 + r;
            const int src = t.row0 + min(nn, t.n - 1);
            int row = (p.sorted_ids != nullptr) ? (p.sorted_ids[src] / p.k_top) : src;
            rows[q * 4 + r] = min(max(row, 0), p.rows_b - 1);
          }
        }
      }
      const int m0 = p.m_base + t.fb * kTileFeatures + static_cast<int>(rank) * kCtaFeatures;
      // A: one box per weight operand (all feature chunks of this CTA's rows); B: one box of
      // b_box_rows token rows, or npad gathered rows
      uint32_t tx = static_cast<uint32_t>(W8 ? a8_bytes : a_bytes);
      if constexpr (BMODE == kBGather4) tx += static_cast<uint32_t>(npad) * 128u;
      if constexpr (BMODE == kBTiled) tx += static_cast<uint32_t>(p.b_box_rows) * 128u;
      if constexpr (PAIR) tx *= 2u;  // both CTAs' loads complete on the even CTA's barrier
      const int brow0 = t.row0 + b_first(npad);
      for (int kb = t.kb0; kb < t.kb1; ++kb) {
        const int s = it % S;
        const uint32_t ph = static_cast<uint32_t>(it / S) & 1u;
        int got = 1;
        if (lane == 0) got = mbar_wait(smem_u32(&empty[s]), ph ^ 1u, abort_flag) ? 1 : 0;
        got = __shfl_sync(0xffffffffu, got, 0);
        if (!got) {
          ok = false;
          break;
        }
        const uint32_t sa = smem_u32(smem + static_cast<size_t>(s) * stage_bytes);
        const uint32_t sb = sa + (W8 ? a8_bytes : a_bytes);
        if constexpr (W8) {
          // e4m3 boxes of 128 features x 64 K per weight operand, then the token rows
          const uint32_t fbar = smem_u32(&full[s]);
          if (lane == 0) {
            mbar_arrive_expect_tx(fbar, tx);
            tma_load_3d(sa, &tmA0, m0, kb * kBK, t.group, fbar);
            if constexpr (kSwiGLU) tma_load_3d(sa + 8192, &tmA1, m0, kb * kBK, t.group, fbar);
            else if constexpr (kDual) tma_load_3d(sa + 8192, &tmA0, m0 + 128, kb * kBK, t.group, fbar);
            tma_load_2d(sb, &tmB, kb * kBK, brow0, fbar);
          }
          __syncwarp();
        } else if constexpr (F8) {
          // K-major e4m3 boxes: 128 K bytes x 128 feature rows per weight operand (256 rows in
          // one box for the two feature blocks of kEpiBF16x2), then the token rows
          const int kc = kb * kStageK;
          if constexpr (PAIR) {
            const uint32_t fbar = mapa_shared(smem_u32(&full[s]), 0);
            if (lane == 0) {
              if (leader) mbar_arrive_expect_tx(smem_u32(&full[s]), tx);
              tma_load_3d_pair(sa, &tmA0, kc, m0, t.group, fbar);
              if constexpr (kSwiGLU) tma_load_3d_pair(sa + 16384, &tmA1, kc, m0, t.group, fbar);
              tma_load_2d_pair(sb, &tmB, kc, brow0, fbar);
            }
          } else {
            const uint32_t fbar = smem_u32(&full[s]);
            if (lane == 0) {
              mbar_arrive_expect_tx(fbar, tx);
              tma_load_3d(sa, &tmA0, kc, m0, t.group, fbar);
              if constexpr (kSwiGLU) tma_load_3d(sa + 16384, &tmA1, kc, m0, t.group, fbar);
              tma_load_2d(sb, &tmB, kc, brow0, fbar);
            }
          }
          __syncwarp();
        } else if constexpr (PAIR) {
          const uint32_t fbar = mapa_shared(smem_u32(&full[s]), 0);
          if (lane == 0) {
            if (leader) mbar_arrive_expect_tx(smem_u32(&full[s]), tx);
            tma_load_4d_pair(sa, &tmA0, 0, kb * kBK, m0 >> 6, t.group, fbar);
            if constexpr (kSwiGLU) tma_load_4d_pair(sa + 16384, &tmA1, 0, kb * kBK, m0 >> 6, t.group, fbar);
            tma_load_2d_pair(sb, &tmB, kb * kBK, brow0, fbar);
          }
          __syncwarp();
        } else {
          const uint32_t fbar = smem_u32(&full[s]);
          if (lane == 0) {
            mbar_arrive_expect_tx(fbar, tx);
            tma_load_4d(sa, &tmA0, 0, kb * kBK, m0 >> 6, t.group, fbar);
            if constexpr (kSwiGLU) tma_load_4d(sa + 16384, &tmA1, 0, kb * kBK, m0 >> 6, t.group, fbar);
            if constexpr (BMODE == kBTiled) tma_load_2d(sb, &tmB, kb * kBK, brow0, fbar);
          }
          __syncwarp();
          if constexpr (BMODE == kBGather4) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const int grp = lane + 32 * q;
              if (grp * 4 < npad)
                tma_gather4(sb + grp * 512, &tmB, kb * kBK, rows[q * 4], rows[q * 4 + 1],
                            rows[q * 4 + 2], rows[q * 4 + 3], fbar);
            }
          }
        }
        ++it;
      }
    }
    if (!ok) {
      *abort_flag = 1;
      if (lane == 0) flag_error(p.err, kDevWaitTimeout);
    }
    // Every load issued must land before the CTA may exit. In PAIR mode the loads complete on
    // the even CTA's barriers; the cluster barrier at the end covers the odd CTA.
    if (lane == 0 && (!PAIR || leader)) {
      for (int i = max(0, it - S); i < it; ++i)
        mbar_wait_cluster(smem_u32(&full[i % S]), static_cast<uint32_t>(i / S) & 1u, nullptr);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (leader) {
      // ---------------------------------------------------------- MMA issuer (one warp)
      // The whole warp runs this loop so that its control flow, counters and descriptors stay
      // warp-uniform; one elected lane issues each tcgen05.mma / commit. Stage index, phase and
      // stage byte offset advance incrementally, and the smem descriptors are the stage-0 ones
      // plus the offset (in 16-byte units), so nothing but the MMAs sits between two MMAs.
      constexpr uint32_t kFull = 0xffffffffu;
      const uint32_t S = static_cast<uint32_t>(p.stages);
      const uint32_t sbase = smem_u32(smem);
      // W8: A comes from the bf16 slots; the stage ring holds the e4m3 codes and B
      // A: MN-major bf16 (weights [E][K][M]) or K-major e4m3 (F8: repacked [E][M][K])
      const uint64_t adesc0 = F8 ? smem_desc_sw128(sbase, 16, 1024)
                                 : smem_desc_sw128(W8 ? smem_u32(a16) : sbase, 8192, 1024);
      const uint64_t bdesc0 = smem_desc_sw128(sbase + (W8 ? a8_bytes : a_bytes), 16, 1024);
      uint32_t s = 0, ph = 0, soff = 0;
      uint32_t kbi = 0;  // W8: k-blocks issued (bf16 slot kbi & 1, its use count kbi >> 1)
      int tc = 0;
      bool ok = true;
      for (int tile = tile0; ok && tile < num_tiles; tile += tstep) {
        const Tile t = decode_tile(tile, p.num_fb, groups, p.TB, s_off, s_blk, kblocks);
        const int npad = (t.n + 15) & ~15;
        const int buf = tc % p.nbuf;
        const uint32_t use = static_cast<uint32_t>(tc / p.nbuf);
        if (!__all_sync(kFull, mbar_wait_cluster(smem_u32(&tempty[buf]), (use & 1u) ^ 1u,
                                                 abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d0 = tmem_base + static_cast<uint32_t>(buf * 256);
        const uint32_t d1 = d0 + static_cast<uint32_t>(p.TB);
        const uint32_t idesc =
            F8 ? idesc_e4m3(PAIR ? 2 * kBM : kBM, npad)
               : idesc_bf16(PAIR ? 2 * kBM : kBM, npad, /*a_mn_major=*/true, /*b_mn_major=*/false);
        uint32_t acc = 0;
#pragma unroll 2
        for (int kb = t.kb0; kb < t.kb1; ++kb) {
          if (!__all_sync(kFull, mbar_wait_cluster(smem_u32(&full[s]), ph, abort_flag))) {
            ok = false;
            break;
          }
          if constexpr (W8) {
            if (!__all_sync(kFull, mbar_wait(smem_u32(&cfull[kbi & 1]), (kbi >> 1) & 1u,
                                             abort_flag))) {
              ok = false;
              break;
            }
          }
          tc_fence_after();
          const uint64_t ad =
              W8 ? adesc0 + (kbi & 1) * static_cast<uint32_t>(a_bytes >> 4) : adesc0 + (soff >> 4);
          const uint64_t bd = bdesc0 + (soff >> 4);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            // bf16: A advances 16 K-rows (2 KB), B 16 K-columns (32 B) per step; F8: both
            // advance 32 K-columns (32 B) per step. The second A operand sits 16 KB after the
            // first.
            constexpr uint32_t kAStep = F8 ? 2u : 128u;
            if constexpr (F8) {
              if constexpr (PAIR) tc_mma_f8_pair_elect(d0, ad + kk * kAStep, bd + kk * 2, idesc, acc);
              else tc_mma_f8_elect(d0, ad + kk * kAStep, bd + kk * 2, idesc, acc);
              if constexpr (kDual) {
                if constexpr (PAIR)
                  tc_mma_f8_pair_elect(d1, ad + 1024 + kk * kAStep, bd + kk * 2, idesc, acc);
                else
                  tc_mma_f8_elect(d1, ad + 1024 + kk * kAStep, bd + kk * 2, idesc, acc);
              }
            } else {
              if constexpr (PAIR) tc_mma_bf16_pair_elect(d0, ad + kk * kAStep, bd + kk * 2, idesc, acc);
              else tc_mma_bf16_elect(d0, ad + kk * kAStep, bd + kk * 2, idesc, acc);
              if constexpr (kDual) {
                if constexpr (PAIR)
                  tc_mma_bf16_pair_elect(d1, ad + 1024 + kk * kAStep, bd + kk * 2, idesc, acc);
                else
                  tc_mma_bf16_elect(d1, ad + 1024 + kk * kAStep, bd + kk * 2, idesc, acc);
              }
            }
            acc = 1u;
          }
          if constexpr (PAIR) tc_commit_pair_mc_elect(smem_u32(&empty[s]), 0x3);
          else tc_commit_elect(smem_u32(&empty[s]));
          if constexpr (W8) tc_commit_elect(smem_u32(&cempty[kbi & 1]));
          ++kbi;
          if (++s == S) {
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
        ++tc;
      }
      if (!ok && lane == 0) {
        *abort_flag = 1;
        flag_error(p.err, kDevWaitTimeout);
      }
      // Every MMA issued must complete before TMEM is released.
      if constexpr (PAIR) tc_commit_pair_mc_elect(smem_u32(drain), 0x3);
      else tc_commit_elect(smem_u32(drain));
      mbar_wait(smem_u32(drain), 0u, nullptr);
    }
    __syncwarp();
  } else if (kCp && warp >= kGatherWarp0) {
    // ------------------------------------------------------------ cp.async row gatherers
    // Thread g (0..127) copies 16-byte chunk (g % 8) of rows g/8, g/8 + 16, ... of this CTA's
    // B rows of each stage, writing the 128-byte-swizzled K-major layout the MMA expects.
    const int g = threadIdx.x - kGatherWarp0 * 32;
    const int chunk = g & 7;
    int it = 0;
    bool ok = true;
    for (int tile = tile0; ok && tile < num_tiles; tile += tstep) {
      const Tile t = decode_tile(tile, p.num_fb, groups, p.TB, s_off, s_blk, kblocks);
      const int npad = (t.n + 15) & ~15;
      const int bn = b_rows(npad);
      const int first = b_first(npad);
      const __nv_bfloat16* src[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = (g >> 3) + 16 * i;
        const int slot = t.row0 + min(first + r, t.n - 1);
        int row = (p.sorted_ids != nullptr) ? (p.sorted_ids[slot] / p.k_top) : slot;
        row = min(max(row, 0), p.rows_b - 1);
        src[i] = p.b_ptr + static_cast<size_t>(row) * p.K + chunk * 8;
      }
      for (int kb = t.kb0; kb < t.kb1; ++kb) {
        const int s = it % S;
        const uint32_t ph = static_cast<uint32_t>(it / S) & 1u;
        int got = 1;
        if (lane == 0) got = mbar_wait(smem_u32(&empty[s]), ph ^ 1u, abort_flag) ? 1 : 0;
        got = __shfl_sync(0xffffffffu, got, 0);
        if (!got) {
          ok = false;
          break;
        }
        const uint32_t sb = smem_u32(smem + static_cast<size_t>(s) * stage_bytes) + a_bytes;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int r = (g >> 3) + 16 * i;
          if (r < bn) cp_async_16(sb + r * 128 + ((chunk ^ (r & 7)) << 4), src[i] + kb * kBK);
        }
        cp_async_arrive_noinc(smem_u32(&full[s]));
        ++it;
      }
    }
    if (!ok) {
      *abort_flag = 1;
      if (lane == 0) flag_error(p.err, kDevWaitTimeout);
    }
    cp_async_wait_all();
  } else if (W8 && warp >= kGatherWarp0) {
    // ------------------------------------------------------------ e4m3 -> bf16 converters
    // Thread g (0..127) takes 16-byte units g, g+128, ... of the stage's e4m3 A: unit u is
    // operand u / 512, K row (u % 512) / 8 and features 16 * (u % 8) .. +15 of that row. Each
    // unit becomes two 16-byte bf16 units at the same K row of the 64-feature chunk holding
    // those features, with the 128-byte swizzle (16-byte unit index XOR K row % 8) of both
    // layouts.
    constexpr uint32_t kFull = 0xffffffffu;
    constexpr int kUnits = a8_bytes / 16;
    const int g = threadIdx.x - kGatherWarp0 * 32;
    const uint32_t sbase = smem_u32(smem);
    const uint32_t a16base = smem_u32(a16);
    uint32_t s = 0, ph = 0, kbi = 0;
    bool ok = true;
    for (int tile = tile0; ok && tile < num_tiles; tile += tstep) {
      const Tile t = decode_tile(tile, p.num_fb, groups, p.TB, s_off, s_blk, kblocks);
      for (int kb = t.kb0; kb < t.kb1; ++kb) {
        const uint32_t j = kbi & 1u;
        const bool got = mbar_wait(smem_u32(&full[s]), ph, abort_flag) &&
                         mbar_wait(smem_u32(&cempty[j]), ((kbi >> 1) & 1u) ^ 1u, abort_flag);
        if (!__all_sync(kFull, got)) {
          ok = false;
          break;
        }
        const uint32_t src0 = sbase + s * static_cast<uint32_t>(stage_bytes);
        const uint32_t dst0 = a16base + j * static_cast<uint32_t>(a_bytes);
#pragma unroll 2
        for (int u = g; u < kUnits; u += 128) {
          const int o = u >> 9, k = (u >> 3) & 63, v = u & 7;
          uint32_t w[4];
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                       : "r"(src0 + o * 8192 + k * 128 + ((v ^ (k & 7)) << 4)));
          uint32_t b[8];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            b[2 * i] = e4m3x2_to_bf16x2(static_cast<uint16_t>(w[i] & 0xffffu));
            b[2 * i + 1] = e4m3x2_to_bf16x2(static_cast<uint16_t>(w[i] >> 16));
          }
          const uint32_t d = dst0 + o * 16384 + (v >> 2) * 8192 + k * 128;
          const int u0 = (v & 3) * 2;
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(d + ((u0 ^ (k & 7)) << 4)),
                       "r"(b[0]), "r"(b[1]), "r"(b[2]), "r"(b[3])
                       : "memory");
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(
                           d + (((u0 + 1) ^ (k & 7)) << 4)),
                       "r"(b[4]), "r"(b[5]), "r"(b[6]), "r"(b[7])
                       : "memory");
        }
        fence_proxy_async_smem();  // generic-proxy writes, read next by the tensor core
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&cfull[j]));
        ++kbi;
        if (++s == static_cast<uint32_t>(S)) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
    if (!ok) {
      *abort_flag = 1;
      if (lane == 0) flag_error(p.err, kDevWaitTimeout);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..9)
    const int q = warp & 3;               // TMEM lane quadrant this warp may read
    const int half = (warp - 2) >> 2;     // which alternate 32-column chunks it drains
    int tc = 0;
    bool ok = true;
    for (int tile = tile0; tile < num_tiles; tile += tstep) {
      const Tile t = decode_tile(tile, p.num_fb, groups, p.TB, s_off, s_blk, kblocks);
      const int buf = tc % p.nbuf;
      const uint32_t use = static_cast<uint32_t>(tc / p.nbuf);
      int got = 1;
      if (lane == 0) got = mbar_wait_cluster(smem_u32(&tfull[buf]), use & 1u, abort_flag) ? 1 : 0;
      got = __shfl_sync(0xffffffffu, got, 0);
      if (!got) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int m = p.m_base + t.fb * kTileFeatures + static_cast<int>(rank) * kCtaFeatures +
                    q * 32 + lane;
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                          static_cast<uint32_t>(buf * 256);
      // Read every accumulator chunk this warp owns into registers, already rounded to bf16
      // (two values per word), hand the TMEM buffer back to the MMA issuer, and only then
      // write the rows out: the next tile's MMAs run under these stores.
      constexpr int kW = (MODE == kEpiBF16x2) ? 32 : 16;  // words held per 32-column chunk
      uint32_t pk[kEpiChunks][kW];
      // W8 / F8: channel scales of this lane's feature rows (1 otherwise, and then unused)
      float sc0 = 1.0f, sc1 = 1.0f;
      if constexpr (W8 || F8) {
        // feature rows past the weight's extent (a partial last tile) have no scale and no
        // output
        const size_t so = static_cast<size_t>(t.group) * p.scale_ld + m;
        if (m < p.m_valid) {
          sc0 = p.scale0[so];
          if constexpr (kSwiGLU) sc1 = p.scale1[so];
        }
        if constexpr (kDual && !kSwiGLU) {
          if (m + 128 < p.m_valid) sc1 = p.scale0[so + 128];
        }
      }
      auto scl0 = [&](uint32_t a) {
        return (W8 || F8) ? __uint_as_float(a) * sc0 : __uint_as_float(a);
      };
      auto scl1 = [&](uint32_t a) {
        return (W8 || F8) ? __uint_as_float(a) * sc1 : __uint_as_float(a);
      };
#pragma unroll
      for (int i = 0; i < kEpiChunks; ++i) {
        const int c0 = 32 * half + 64 * i;
        if (c0 < t.n) {
          // F8: the row scale of column (token row) c0 + lane, broadcast to the warp per column
          float csv = 1.0f;
          if constexpr (F8) csv = (c0 + lane < t.n) ? p.act_scale[t.row0 + c0 + lane] : 0.0f;
          auto cs = [&](int col) { return F8 ? __shfl_sync(0xffffffffu, csv, col) : 1.0f; };
          uint32_t v[32];
          tmem_ld32(tb + static_cast<uint32_t>(c0), v);
          if constexpr (kSwiGLU) {
            uint32_t u[32];
            tmem_ld32(tb + static_cast<uint32_t>(p.TB + c0), u);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float ca = cs(2 * j), cb = cs(2 * j + 1);
              pk[i][j] = pack_bf16x2(silu_f32(scl0(v[2 * j]) * ca) * (scl1(u[2 * j]) * ca),
                                     silu_f32(scl0(v[2 * j + 1]) * cb) * (scl1(u[2 * j + 1]) * cb));
            }
          } else {
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j)
              pk[i][j] = pack_bf16x2(scl0(v[2 * j]) * cs(2 * j), scl0(v[2 * j + 1]) * cs(2 * j + 1));
            if constexpr (kDual) {
              tmem_ld32(tb + static_cast<uint32_t>(p.TB + c0), v);
              tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 16; ++j)
                pk[i][16 + j] =
                    pack_bf16x2(scl1(v[2 * j]) * cs(2 * j), scl1(v[2 * j + 1]) * cs(2 * j + 1));
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (PAIR) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[buf]), 0));
        else mbar_arrive(smem_u32(&tempty[buf]));
      }
      // The last tile of a CTA pair may reach past the weight's feature extent (the second
      // CTA's rows were loaded as zeros): those feature rows have no output.
      const bool keep0 = m < p.m_valid;
      const bool keep1 = (MODE == kEpiBF16x2) && (m + 128 < p.m_valid);
#pragma unroll
      for (int i = 0; i < kEpiChunks; ++i) {
        const int c0 = 32 * half + 64 * i;
        if (c0 < t.n && keep0) {
          const int cmax = min(32, t.n - c0);
          uint16_t* o = reinterpret_cast<uint16_t*>(p.out) +
                        static_cast<size_t>(t.row0 + c0) * p.ldo + m;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if (j < cmax) {
              o[static_cast<size_t>(j) * p.ldo] = bf16_half(pk[i][j >> 1], j & 1);
              if constexpr (MODE == kEpiBF16x2)
                if (keep1)
                  o[static_cast<size_t>(j) * p.ldo + 128] =
                      bf16_half(pk[i][16 + (j >> 1)], j & 1);
            }
          }
        }
      }
      ++tc;
    }
    if (!ok) {
      *abort_flag = 1;
      if (lane == 0) flag_error(p.err, kDevWaitTimeout);
    }
  }

  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync_all();  // no CTA leaves while its peer may still signal it
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, kTmemCols);
    else tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ------------------------------------------------------------------ host side

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

// bf16 [rows, cols] row-major, box = {64 columns, 1 row}, 128-byte swizzle: for tile::gather4.
bool map_rows(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, std::string* d) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) {
    if (d) *d = "cuTensorMapEncodeTiled is not available from the driver";
    return false;
  }
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, 1};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS && d) *d = "cuTensorMapEncodeTiled(rows) failed with code " + std::to_string(r);
  return r == CUDA_SUCCESS;
}

// bf16 [rows, cols] row-major, box = {64 columns, box_rows rows}, 128-byte swizzle: contiguous rows.
bool map_row_boxes(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, std::string* d,
                   uint32_t box_rows) {
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
  if (r != CUDA_SUCCESS && d) *d = "cuTensorMapEncodeTiled(row boxes) failed with code " + std::to_string(r);
  return r == CUDA_SUCCESS;
}

// bf16 [groups, kdim, mdim] (mdim contiguous) seen as 4-D {64, kdim, mdim/64, groups}, so that one
// box {64, 64, chunks, 1} brings `chunks` consecutive 64-feature chunks of 64 K rows, laid out
// chunk after chunk (8 KB apart) as the MN-major operand expects. 128-byte swizzle.
bool map_weights_wide(CUtensorMap* m, const void* base, uint64_t mdim, uint64_t kdim,
                      uint64_t groups, uint32_t chunks, std::string* d) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) {
    if (d) *d = "cuTensorMapEncodeTiled is not available from the driver";
    return false;
  }
  cuuint64_t dims[4] = {64, kdim, mdim / 64, groups};
  cuuint64_t strides[3] = {mdim * 2, 128, mdim * kdim * 2};
  cuuint32_t box[4] = {64, 64, chunks, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS && d) *d = "cuTensorMapEncodeTiled(wide weights) failed with code " + std::to_string(r);
  return r == CUDA_SUCCESS;
}


// e4m3 weights [G][K][M] (one byte each): box {128 features, 64 K, 1 group}, 128-byte
// swizzle (a box row is one K index: 128 bytes).
bool map_weights_fp8(CUtensorMap* m, const void* base, uint64_t mdim, uint64_t kdim,
                     uint64_t groups, std::string* d) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) {
    if (d) *d = "cuTensorMapEncodeTiled is not available from the driver";
    return false;
  }
  cuuint64_t dims[3] = {mdim, kdim, groups};
  cuuint64_t strides[2] = {mdim, mdim * kdim};
  cuuint32_t box[3] = {128, 64, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS && d)
    *d = "cuTensorMapEncodeTiled(e4m3 weights) failed with code " + std::to_string(r);
  return r == CUDA_SUCCESS;
}

// K-major e4m3 weight codes [groups][mdim][kdim] (K contiguous): box {128 K bytes, box_rows
// feature rows, 1 group}, 128-byte swizzle.
bool map_weights_kmajor_e4m3(CUtensorMap* m, const void* base, uint64_t kdim, uint64_t mdim,
                             uint64_t groups, uint32_t box_rows, std::string* d) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) {
    if (d) *d = "cuTensorMapEncodeTiled is not available from the driver";
    return false;
  }
  cuuint64_t dims[3] = {kdim, mdim, groups};
  cuuint64_t strides[2] = {kdim, kdim * mdim};
  cuuint32_t box[3] = {128, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS && d)
    *d = "cuTensorMapEncodeTiled(K-major e4m3 weights) failed with code " + std::to_string(r);
  return r == CUDA_SUCCESS;
}

// e4m3 rows [rows][cols] (one byte each): box {128 columns, box_rows rows}, 128-byte swizzle.
bool map_rows_e4m3(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows,
                   uint32_t box_rows, std::string* d) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) {
    if (d) *d = "cuTensorMapEncodeTiled is not available from the driver";
    return false;
  }
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS && d)
    *d = "cuTensorMapEncodeTiled(e4m3 rows) failed with code " + std::to_string(r);
  return r == CUDA_SUCCESS;
}

template <int MODE, int BMODE, bool PAIR, bool W8 = false, bool F8 = false>
cudaError_t launch_mode(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b,
                        TcParams p, int64_t tiles_ub, int num_sms, cudaStream_t stream,
                        std::string* d) {
  const int a_bytes = dual_a<MODE>() ? 32768 : 16384;
  const int a8_bytes = dual_a<MODE>() ? 16384 : 8192;
  const int stage_bytes = (W8 ? a8_bytes : a_bytes) + b_rows_smem(PAIR, p.TB) * 128;
  const int extra = W8 ? 2 * a_bytes : 0;  // the two bf16 A slots
  int stages = (kSmemLimit - 1024 - kCtrlBytes - extra) / stage_bytes;
  if (stages > kMaxStages) stages = kMaxStages;
  if (stages < 2) {
    if (d) *d = "tile too large for shared memory";
    return cudaErrorInvalidValue;
  }
  if (p.TB < 32 || p.TB > kMaxTokenBlock || (p.TB & 31) != 0) {
    if (d) *d = "token block must be a multiple of 32 in [32, 256]";
    return cudaErrorInvalidValue;
  }
  p.stages = stages;
  p.nbuf = ((dual_a<MODE>() ? 2 : 1) * p.TB <= 256) ? 2 : 1;
  const size_t smem = 1024 + static_cast<size_t>(stages) * stage_bytes + extra + kCtrlBytes;
  const int64_t units = PAIR ? num_sms / 2 : num_sms;  // CTA pairs or CTAs, one per SM
  int64_t grid = tiles_ub < units ? tiles_ub : units;
  if (grid < 1) grid = 1;
  if (PAIR) grid *= 2;
  auto kernel = tc_grouped_gemm<MODE, BMODE, PAIR, W8, F8>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_kernel(kernel, dim3(static_cast<unsigned>(grid)), dim3(threads_of<BMODE, W8>()),
                       smem, stream, PAIR ? 2 : 1, a0, a1, b, p);
}

// CTA pairs (cta_group::2) for the expert GEMMs unless the build opts out.
constexpr bool kUsePairs =
#ifdef MOE_NO_CTA_PAIRS
    false;
#else
    true;
#endif

}  // namespace

bool gemm1_uses_row_copy(int /*I*/) { return kUsePairs; }

cudaError_t launch_gemm1_tc(const void* x, int T, const void* xs, const int32_t* sorted_ids,
                            const int32_t* offsets, const int32_t* blk_prefix, const void* w_gate,
                            const void* w_up, void* hbuf, int64_t hbuf_rows, int H, int E, int k,
                            int I, int TB, int64_t ub_blocks, int* err, int num_sms,
                            cudaStream_t stream, std::string* detail) {
  CUtensorMap a0, a1, b;
  // gate and up slices of a CTA's 128 features arrive as one box each
  if (!map_weights_wide(&a0, w_gate, I, H, E, 2, detail) ||
      !map_weights_wide(&a1, w_up, I, H, E, 2, detail))
    return cudaErrorInvalidValue;
  if (xs != nullptr) {
    // token rows already in expert-major order: contiguous rows like GEMM2's B operand, so
    // both CTAs of a pair can take their halves by TMA, one box per stage
    // CTA pairs cover 256 features. When I % 256 == 128 a last pair tile would give its second
    // CTA only zero-filled weight rows (an eighth of the work wasted at I = 1408), so the pairs
    // take the first I - 128 features and a second launch of single CTAs the last 128.
    const bool pair = kUsePairs;
    const bool split = pair && I % 256 == 128 && I >= 384;
    const int box_rows = b_rows_smem(pair, TB);
    if (!map_row_boxes(&b, xs, static_cast<uint64_t>(H), static_cast<uint64_t>(hbuf_rows), detail,
                       static_cast<uint32_t>(box_rows)))
      return cudaErrorInvalidValue;
    TcParams p{};
    p.b_box_rows = box_rows;
    p.K = H;
    p.num_fb = pair ? (split ? I / 256 : (I + 255) / 256) : (I + kBM - 1) / kBM;
    p.m_valid = split ? I - 128 : I;
    p.m_base = 0;
    p.TB = TB;
    p.groups = E;
    p.k_top = 1;
    p.rows_b = static_cast<int>(hbuf_rows);
    p.sorted_ids = nullptr;
    p.offsets = offsets;
    p.blk_prefix = blk_prefix;
    p.out = hbuf;
    p.ldo = I;
    p.err = err;
    p.b_ptr = nullptr;
    const int64_t tiles = static_cast<int64_t>(p.num_fb) * ub_blocks;
    if (!pair)
      return launch_mode<kEpiSwiGLU, kBTiled, false>(a0, a1, b, p, tiles, num_sms, stream, detail);
    cudaError_t e =
        launch_mode<kEpiSwiGLU, kBTiled, true>(a0, a1, b, p, tiles, num_sms, stream, detail);
    if (e != cudaSuccess || !split) return e;
    // the last 128 features on single CTAs, each taking its token block's rows whole
    CUtensorMap b1;
    const int box1 = b_rows_smem(false, TB);
    if (!map_row_boxes(&b1, xs, static_cast<uint64_t>(H), static_cast<uint64_t>(hbuf_rows),
                       detail, static_cast<uint32_t>(box1)))
      return cudaErrorInvalidValue;
    TcParams p1 = p;
    p1.b_box_rows = box1;
    p1.num_fb = 1;
    p1.m_base = I - 128;
    p1.m_valid = I;
    return launch_mode<kEpiSwiGLU, kBTiled, false>(a0, a1, b1, p1, ub_blocks, num_sms, stream,
                                                    detail);
  }
  if (!map_rows(&b, x, static_cast<uint64_t>(H), static_cast<uint64_t>(T), detail))
    return cudaErrorInvalidValue;
#ifdef MOE_GEMM1_GATHER4
  const bool use_gather4 = true;   // TMA tile::gather4 row gather (build-time choice)
#else
  const bool use_gather4 = false;  // cp.async row gather
#endif
  TcParams p{};
  p.b_box_rows = 0;
  p.K = H;
  p.num_fb = (I + kBM - 1) / kBM;
  p.m_valid = I;
  p.TB = TB;
  p.groups = E;
  p.k_top = k;
  p.rows_b = T;
  p.sorted_ids = sorted_ids;
  p.offsets = offsets;
  p.blk_prefix = blk_prefix;
  p.out = hbuf;
  p.ldo = I;
  p.err = err;
  p.b_ptr = static_cast<const __nv_bfloat16*>(x);
  const int64_t tiles = static_cast<int64_t>(p.num_fb) * ub_blocks;
  if (use_gather4)
    return launch_mode<kEpiSwiGLU, kBGather4, false>(a0, a1, b, p, tiles, num_sms, stream, detail);
  return launch_mode<kEpiSwiGLU, kBCpAsync, false>(a0, a1, b, p, tiles, num_sms, stream, detail);
}

cudaError_t launch_gemm2_tc(const void* hbuf, int64_t hbuf_rows, const int32_t* offsets,
                            const int32_t* blk_prefix, const void* w_down, void* y, int H, int E,
                            int I, int TB, int64_t ub_blocks, int* err, int num_sms,
                            cudaStream_t stream, std::string* detail) {
  CUtensorMap a0, b;
  const bool dual = (H % 256) == 0;
  const bool pair = kUsePairs && dual;  // 512 features per pair tile; a partial last tile is masked
  const int box_rows = b_rows_smem(pair, TB);
  // a CTA's 256 (dual) or 128 feature rows of Wd arrive as one box; its token rows as another
  if (!map_weights_wide(&a0, w_down, H, I, E, dual ? 4 : 2, detail) ||
      !map_row_boxes(&b, hbuf, static_cast<uint64_t>(I), static_cast<uint64_t>(hbuf_rows), detail,
                     static_cast<uint32_t>(box_rows)))
    return cudaErrorInvalidValue;
  TcParams p{};
  p.b_box_rows = box_rows;
  p.K = I;
  p.num_fb = pair ? (H + 511) / 512 : (dual ? H / 256 : (H + kBM - 1) / kBM);
  p.m_valid = H;
  p.TB = TB;
  p.groups = E;
  p.k_top = 1;
  p.rows_b = static_cast<int>(hbuf_rows);
  p.sorted_ids = nullptr;
  p.offsets = offsets;
  p.blk_prefix = blk_prefix;
  p.out = y;
  p.ldo = H;
  p.err = err;
  const int64_t tiles = static_cast<int64_t>(p.num_fb) * ub_blocks;
  if (pair)
    return launch_mode<kEpiBF16x2, kBTiled, true>(a0, a0, b, p, tiles, num_sms, stream, detail);
  if (dual)
    return launch_mode<kEpiBF16x2, kBTiled, false>(a0, a0, b, p, tiles, num_sms, stream, detail);
  return launch_mode<kEpiBF16, kBTiled, false>(a0, a0, b, p, tiles, num_sms, stream, detail);
}

// ---- FP8 (e4m3) expert weights: single CTAs, B streamed by TMA from contiguous rows.

cudaError_t launch_gemm1_w8(const void* xs, const int32_t* offsets, const int32_t* blk_prefix,
                            const uint8_t* q_gate, const uint8_t* q_up, const float* s_gate,
                            const float* s_up, void* hbuf, int64_t hbuf_rows, int H, int E,
                            int I, int TB, int64_t ub_blocks, int* err, int num_sms,
                            cudaStream_t stream, std::string* detail) {
  CUtensorMap a0, a1, b;
  if (!map_weights_fp8(&a0, q_gate, I, H, E, detail) ||
      !map_weights_fp8(&a1, q_up, I, H, E, detail) ||
      !map_row_boxes(&b, xs, static_cast<uint64_t>(H), static_cast<uint64_t>(hbuf_rows), detail,
                     static_cast<uint32_t>(TB)))
    return cudaErrorInvalidValue;
  TcParams p{};
  p.b_box_rows = TB;
  p.K = H;
  p.num_fb = (I + kBM - 1) / kBM;
  p.m_valid = I;
  p.TB = TB;
  p.groups = E;
  p.k_top = 1;
  p.rows_b = static_cast<int>(hbuf_rows);
  p.sorted_ids = nullptr;
  p.offsets = offsets;
  p.blk_prefix = blk_prefix;
  p.out = hbuf;
  p.ldo = I;
  p.err = err;
  p.b_ptr = nullptr;
  p.scale0 = s_gate;
  p.scale1 = s_up;
  p.scale_ld = I;
  const int64_t tiles = static_cast<int64_t>(p.num_fb) * ub_blocks;
  return launch_mode<kEpiSwiGLU, kBTiled, false, true>(a0, a1, b, p, tiles, num_sms, stream,
                                                       detail);
}

cudaError_t launch_gemm2_w8(const void* hbuf, int64_t hbuf_rows, const int32_t* offsets,
                            const int32_t* blk_prefix, const uint8_t* q_down, const float* s_down,
                            void* y, int H, int E, int I, int TB, int64_t ub_blocks, int* err,
                            int num_sms, cudaStream_t stream, std::string* detail) {
  CUtensorMap a0, b;
  const bool dual = (H % 256) == 0;
  if (!map_weights_fp8(&a0, q_down, H, I, E, detail) ||
      !map_row_boxes(&b, hbuf, static_cast<uint64_t>(I), static_cast<uint64_t>(hbuf_rows), detail,
                     static_cast<uint32_t>(TB)))
    return cudaErrorInvalidValue;
  TcParams p{};
  p.b_box_rows = TB;
  p.K = I;
  p.num_fb = dual ? H / 256 : (H + kBM - 1) / kBM;
  p.m_valid = H;
  p.TB = TB;
  p.groups = E;
  p.k_top = 1;
  p.rows_b = static_cast<int>(hbuf_rows);
  p.sorted_ids = nullptr;
  p.offsets = offsets;
  p.blk_prefix = blk_prefix;
  p.out = y;
  p.ldo = H;
  p.err = err;
  p.scale0 = s_down;
  p.scale1 = nullptr;
  p.scale_ld = H;
  const int64_t tiles = static_cast<int64_t>(p.num_fb) * ub_blocks;
  if (dual)
    return launch_mode<kEpiBF16x2, kBTiled, false, true>(a0, a0, b, p, tiles, num_sms, stream,
                                                         detail);
  return launch_mode<kEpiBF16, kBTiled, false, true>(a0, a0, b, p, tiles, num_sms, stream,
                                                     detail);
}

// ---- FP8 weights and activations (W8A8): native e4m3 MMAs on CTA pairs, B streamed by TMA
// from expert-major e4m3 rows.

cudaError_t launch_gemm1_f8(const void* xs8, const float* sx, const int32_t* offsets,
                            const int32_t* blk_prefix, const uint8_t* qk_gate,
                            const uint8_t* qk_up, const float* s_gate, const float* s_up,
                            void* hbuf, int64_t hbuf_rows, int H, int E, int I, int TB,
                            int64_t ub_blocks, int* err, int num_sms, cudaStream_t stream,
                            std::string* detail) {
  CUtensorMap a0, a1, b;
  const bool pair = kUsePairs;
  const int box_rows = b_rows_smem(pair, TB);
  if (!map_weights_kmajor_e4m3(&a0, qk_gate, H, I, E, 128, detail) ||
      !map_weights_kmajor_e4m3(&a1, qk_up, H, I, E, 128, detail) ||
      !map_rows_e4m3(&b, xs8, static_cast<uint64_t>(H), static_cast<uint64_t>(hbuf_rows),
                     static_cast<uint32_t>(box_rows), detail))
    return cudaErrorInvalidValue;
  TcParams p{};
  p.b_box_rows = box_rows;
  p.K = H;
  p.num_fb = pair ? (I + 255) / 256 : (I + kBM - 1) / kBM;
  p.m_valid = I;
  p.TB = TB;
  p.groups = E;
  p.k_top = 1;
  p.rows_b = static_cast<int>(hbuf_rows);
  p.offsets = offsets;
  p.blk_prefix = blk_prefix;
  p.out = hbuf;
  p.ldo = I;
  p.err = err;
  p.scale0 = s_gate;
  p.scale1 = s_up;
  p.scale_ld = I;
  p.act_scale = sx;
  const int64_t tiles = static_cast<int64_t>(p.num_fb) * ub_blocks;
  if (pair)
    return launch_mode<kEpiSwiGLU, kBTiled, true, false, true>(a0, a1, b, p, tiles, num_sms,
                                                               stream, detail);
  return launch_mode<kEpiSwiGLU, kBTiled, false, false, true>(a0, a1, b, p, tiles, num_sms, stream,
                                                              detail);
}

cudaError_t launch_gemm2_f8(const void* h8, const float* sh, int64_t hbuf_rows,
                            const int32_t* offsets, const int32_t* blk_prefix,
                            const uint8_t* qk_down, const float* s_down, void* y, int H, int E,
                            int I, int TB, int64_t ub_blocks, int* err, int num_sms,
                            cudaStream_t stream, std::string* detail) {
  CUtensorMap a0, b;
  const bool dual = (H % 256) == 0;
  const bool pair = kUsePairs && dual;
  const int box_rows = b_rows_smem(pair, TB);
  // a CTA's 256 (dual) or 128 feature rows of the down projection as one box
  if (!map_weights_kmajor_e4m3(&a0, qk_down, I, H, E, dual ? 256 : 128, detail) ||
      !map_rows_e4m3(&b, h8, static_cast<uint64_t>(I), static_cast<uint64_t>(hbuf_rows),
                     static_cast<uint32_t>(box_rows), detail))
    return cudaErrorInvalidValue;
  TcParams p{};
  p.b_box_rows = box_rows;
  p.K = I;
  p.num_fb = pair ? (H + 511) / 512 : (dual ? H / 256 : (H + kBM - 1) / kBM);
  p.m_valid = H;
  p.TB = TB;
  p.groups = E;
  p.k_top = 1;
  p.rows_b = static_cast<int>(hbuf_rows);
  p.offsets = offsets;
  p.blk_prefix = blk_prefix;
  p.out = y;
  p.ldo = H;
  p.err = err;
  p.scale0 = s_down;
  p.scale1 = nullptr;
  p.scale_ld = H;
  p.act_scale = sh;
  const int64_t tiles = static_cast<int64_t>(p.num_fb) * ub_blocks;
  if (pair)
    return launch_mode<kEpiBF16x2, kBTiled, true, false, true>(a0, a0, b, p, tiles, num_sms,
                                                               stream, detail);
  if (dual)
    return launch_mode<kEpiBF16x2, kBTiled, false, false, true>(a0, a0, b, p, tiles, num_sms,
                                                                stream, detail);
  return launch_mode<kEpiBF16, kBTiled, false, false, true>(a0, a0, b, p, tiles, num_sms, stream,
                                                            detail);
}

}  // namespace moe
