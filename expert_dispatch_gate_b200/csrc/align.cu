// align.cu — capacity-limited grouping of the T*k assignments by expert.
//
// [P1] "MoE 模型的 FlashAttention 跟普通模型有什么不一样？", section "FlashAttention 在 MoE 模型里的位置",
// step 3 (pick out the tokens that go to the same expert); [P4] "MoE Router" (2048ai.net),
// section "Token 分发的通信瓶颈" (per-destination counts) and section "昇腾NPU的通信计算重叠"
// (at most C per expert, overflow dropped to the residual path); [P5] "大模型推理加速200%+？…",
// section "3.2 Fuse RMS RoPE & MoE Align & MoE Sum" (prefix sums for the index calculation,
// hierarchical atomics, expert map / mask / fill fused).
//
// Rank of assignment a = t*k + j inside expert e = idx[t,j]: number of earlier assignments (in
// a order, i.e. token order) routed to e. Kept iff rank < C. The result is deterministic and
// identical to the sequential definition:
//   1. hist:    per 2048-assignment chunk, per-expert counts (shared-memory atomics).
//   2. scan:    one block; per expert, exclusive prefix over chunks (chunk bases), raw totals,
//               counts = min(raw, C), offsets = exclusive scan of counts, and the token-block
//               plan blk_prefix used by the expert GEMMs.
//   3. scatter: per chunk, stable in-chunk ranks (warp __match_any_sync + per-warp prefix),
//               then slot = offsets[e] + rank for kept assignments; fills the -1 tail.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kSinglePerWarp = kAlignSingle / kWarps;  // one-block path: 256 per warp
constexpr int kMaxE = 256;

__global__ void __launch_bounds__(kThreads)
    align_hist_kernel(const int32_t* __restrict__ idx, int64_t A, int E, int chunk,
                      int32_t* __restrict__ blk_hist, int* err) {
  pdl_enter<false>();
  __shared__ int h[kMaxE];
  for (int e = threadIdx.x; e < E; e += kThreads) h[e] = 0;
  __syncthreads();
  const int64_t base = static_cast<int64_t>(blockIdx.x) * chunk;
  const int64_t end = min(A, base + chunk);
  for (int64_t a = base + threadIdx.x; a < end; a += kThreads) {
    const int e = idx[a];
    if (e >= 0 && e < E) atomicAdd(&h[e], 1);
    else flag_error(err, kDevBadExpert);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kThreads)
    blk_hist[static_cast<size_t>(blockIdx.x) * E + e] = h[e];
}

// Exclusive block-wide scan of one int per thread (kThreads threads).
__device__ __forceinline__ int block_exclusive_scan(int v, int* sh, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int inc = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, inc, off);
    if (lane >= off) inc += o;
  }
  if (lane == 31) sh[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int w = (lane < kWarps) ? sh[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, w, off);
      if (lane >= off) w += o;
    }
    if (lane < kWarps) sh[lane] = w;  // inclusive warp totals
  }
  __syncthreads();
  const int warp_base = (warp > 0) ? sh[warp - 1] : 0;
  total = sh[kWarps - 1];
  __syncthreads();
  return warp_base + inc - v;
}

__global__ void __launch_bounds__(kThreads)
    align_scan_kernel(int32_t* __restrict__ blk_hist, int nblk, int E, int C, int TB,
                      int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                      int32_t* __restrict__ blk_prefix) {
  pdl_enter<false>();
  __shared__ int sh[kWarps];
  const int e = threadIdx.x;
  int run = 0;
  if (e < E) {
    // chunk bases in place; loads batched so they overlap
    for (int b0 = 0; b0 < nblk; b0 += 8) {
      int c[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        c[i] = (b0 + i < nblk) ? blk_hist[static_cast<size_t>(b0 + i) * E + e] : 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (b0 + i < nblk) blk_hist[static_cast<size_t>(b0 + i) * E + e] = run;
        run += c[i];
      }
    }
  }
  const int cnt = (e < E) ? min(run, C) : 0;
  const int nb = (cnt + TB - 1) / TB;
  int tot_cnt, tot_nb;
  const int off = block_exclusive_scan(cnt, sh, tot_cnt);
  const int bp = block_exclusive_scan(nb, sh, tot_nb);
  if (e < E) {
    counts[e] = cnt;
    offsets[e] = off;
    if (blk_prefix != nullptr) blk_prefix[e] = bp;
  }
  if (e == 0) {
    offsets[E] = tot_cnt;
    if (blk_prefix != nullptr) blk_prefix[E] = tot_nb;
  }
}

__global__ void __launch_bounds__(kThreads)
    align_scatter_kernel(const int32_t* __restrict__ idx, int64_t A, int E, int C, int chunk,
                         const int32_t* __restrict__ blk_base, const int32_t* __restrict__ offsets,
                         int32_t* __restrict__ sorted_ids, int32_t* __restrict__ slot_of,
                         uint8_t* __restrict__ drop_mask) {
  pdl_enter<false>();
  __shared__ int wrun[kWarps][kMaxE];
  __shared__ int s_off[kMaxE];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < kWarps * kMaxE; i += kThreads) (&wrun[0][0])[i] = 0;
  for (int e = threadIdx.x; e < E; e += kThreads) s_off[e] = offsets[e];
  __syncthreads();
  const int per_warp = chunk / kWarps;  // a multiple of 32
  const int64_t wbase = static_cast<int64_t>(blockIdx.x) * chunk + warp * per_warp;

  // pass 1: per-warp per-expert counts of this warp's assignments
  for (int step = 0; step < per_warp / 32; ++step) {
    const int64_t a = wbase + step * 32 + lane;
    const int e = (a < A) ? idx[a] : -1;
    const bool ok = (e >= 0 && e < E);
    const uint32_t peers = __match_any_sync(0xffffffffu, ok ? e : (E + lane));
    if (ok && lane == __ffs(peers) - 1) wrun[warp][e] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // per expert: exclusive prefix across the warps, seeded with this chunk's base
  for (int e = threadIdx.x; e < E; e += kThreads) {
    int run = blk_base[static_cast<size_t>(blockIdx.x) * E + e];
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const int c = wrun[w][e];
      wrun[w][e] = run;
      run += c;
    }
  }
  __syncthreads();
  // pass 2: stable ranks in assignment order
  for (int step = 0; step < per_warp / 32; ++step) {
    const int64_t a = wbase + step * 32 + lane;
    const bool in = a < A;
    const int e = in ? idx[a] : -1;
    const bool ok = (e >= 0 && e < E);
    const uint32_t peers = __match_any_sync(0xffffffffu, ok ? e : (E + lane));
    int rank = 0;
    if (ok) rank = wrun[warp][e] + __popc(peers & lanemask_lt());
    __syncwarp();
    if (ok && lane == __ffs(peers) - 1) wrun[warp][e] += __popc(peers);
    __syncwarp();
    if (in) {
      if (ok && rank < C) {
        const int slot = s_off[e] + rank;
        sorted_ids[slot] = static_cast<int32_t>(a);
        slot_of[a] = slot;
        drop_mask[a] = 0;
      } else {
        slot_of[a] = -1;
        drop_mask[a] = 1;
      }
    }
  }
  // slots past the kept total
  const int64_t kept = offsets[E];
  for (int64_t s = kept + static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; s < A;
       s += static_cast<int64_t>(gridDim.x) * kThreads)
    sorted_ids[s] = -1;
}

// Whole grouping in one block when every assignment fits one chunk (A <= kAlignSingle): the
// histogram, scan and stable scatter of the three kernels above, without two launches.
__global__ void __launch_bounds__(kThreads)
    align_single_chunk_kernel(const int32_t* __restrict__ idx, int64_t A, int E, int C, int TB,
                              int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                              int32_t* __restrict__ blk_prefix, int32_t* __restrict__ sorted_ids,
                              int32_t* __restrict__ slot_of, uint8_t* __restrict__ drop_mask,
                              int* err) {
  pdl_enter<false>();
  __shared__ int wrun[kWarps][kMaxE];
  __shared__ int s_off[kMaxE + 1];
  __shared__ int sh[kWarps];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < kWarps * kMaxE; i += kThreads) (&wrun[0][0])[i] = 0;
  __syncthreads();
  const int64_t wbase = static_cast<int64_t>(warp) * kSinglePerWarp;
  // per-warp per-expert counts
  for (int step = 0; step < kSinglePerWarp / 32; ++step) {
    const int64_t a = wbase + step * 32 + lane;
    const int e = (a < A) ? idx[a] : -1;
    const bool ok = (e >= 0 && e < E);
    if (a < A && !ok) flag_error(err, kDevBadExpert);
    const uint32_t peers = __match_any_sync(0xffffffffu, ok ? e : (E + lane));
    if (ok && lane == __ffs(peers) - 1) wrun[warp][e] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // per expert: exclusive prefix across warps and the raw total
  const int e = threadIdx.x;
  int raw = 0;
  if (e < E) {
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const int c = wrun[w][e];
      wrun[w][e] = raw;
      raw += c;
    }
  }
  const int cnt = (e < E) ? min(raw, C) : 0;
  const int nb = (cnt + TB - 1) / TB;
  int tot_cnt, tot_nb;
  const int off = block_exclusive_scan(cnt, sh, tot_cnt);
  const int bp = block_exclusive_scan(nb, sh, tot_nb);
  if (e < E) {
    counts[e] = cnt;
    offsets[e] = off;
    s_off[e] = off;
    if (blk_prefix != nullptr) blk_prefix[e] = bp;
  }
  if (e == 0) {
    offsets[E] = tot_cnt;
    if (blk_prefix != nullptr) blk_prefix[E] = tot_nb;
  }
  __syncthreads();
  // stable ranks in assignment order, then the scatter
  for (int step = 0; step < kSinglePerWarp / 32; ++step) {
    const int64_t a = wbase + step * 32 + lane;
    const bool in = a < A;
    const int ea = in ? idx[a] : -1;
    const bool ok = (ea >= 0 && ea < E);
    const uint32_t peers = __match_any_sync(0xffffffffu, ok ? ea : (E + lane));
    int rank = 0;
    if (ok) rank = wrun[warp][ea] + __popc(peers & lanemask_lt());
    __syncwarp();
    if (ok && lane == __ffs(peers) - 1) wrun[warp][ea] += __popc(peers);
    __syncwarp();
    if (in) {
      if (ok && rank < C) {
        const int slot = s_off[ea] + rank;
        sorted_ids[slot] = static_cast<int32_t>(a);
        slot_of[a] = slot;
        drop_mask[a] = 0;
      } else {
        slot_of[a] = -1;
        drop_mask[a] = 1;
      }
    }
  }
  for (int64_t sl = tot_cnt + threadIdx.x; sl < A; sl += kThreads) sorted_ids[sl] = -1;
}

__global__ void __launch_bounds__(kThreads)
    plan_from_offsets_kernel(const int32_t* __restrict__ offsets, int E, int TB,
                             int32_t* __restrict__ blk_prefix) {
  pdl_enter<false>();
  __shared__ int sh[kWarps];
  const int e = threadIdx.x;
  const int cnt = (e < E) ? (offsets[e + 1] - offsets[e]) : 0;
  const int nb = (cnt + TB - 1) / TB;
  int tot;
  const int bp = block_exclusive_scan(nb, sh, tot);
  if (e < E) blk_prefix[e] = bp;
  if (e == 0) blk_prefix[E] = tot;
}

}  // namespace

cudaError_t launch_align(const int32_t* topk_idx, int64_t A, int E, int C, int TB,
                         int32_t* blk_hist, int32_t* counts, int32_t* offsets,
                         int32_t* blk_prefix, int32_t* sorted_ids, int32_t* slot_of,
                         uint8_t* drop_mask, int* err, cudaStream_t stream) {
  if (A == 0) return cudaSuccess;
  if (A <= kAlignSingle)
    return launch_kernel(align_single_chunk_kernel, dim3(1), dim3(kThreads), 0, stream, 1,
                         topk_idx, A, E, C, TB, counts, offsets, blk_prefix, sorted_ids, slot_of,
                         drop_mask, err);
  const int chunk = align_chunk(A);
  const int nblk = static_cast<int>((A + chunk - 1) / chunk);
  cudaError_t e = launch_kernel(align_hist_kernel, dim3(nblk), dim3(kThreads), 0, stream, 1,
                                topk_idx, A, E, chunk, blk_hist, err);
  if (e == cudaSuccess)
    e = launch_kernel(align_scan_kernel, dim3(1), dim3(kThreads), 0, stream, 1, blk_hist, nblk, E,
                      C, TB, counts, offsets, blk_prefix);
  if (e == cudaSuccess)
    e = launch_kernel(align_scatter_kernel, dim3(nblk), dim3(kThreads), 0, stream, 1, topk_idx, A,
                      E, C, chunk, blk_hist, offsets, sorted_ids, slot_of, drop_mask);
  return e;
}

// ---- grouping without a caller workspace
//
// Scratch of moe_align_noalloc, a variant of the launch sequence above for callers that may
// not allocate device memory. It holds the per-chunk histograms of up to
// kNoAllocMaxAssignments assignments for up to 256 experts, the token-block plan and an
// error word: about 130 KB, resident on every device that loads the library until the
// process exits. All calls share it, so calls that overlap on the GPU (different streams,
// different host threads) race on it and must be serialised by the caller.
namespace {
struct NoAllocScratch {
  int err[64];
  int blk_prefix[320];
  int blk_hist[kNoAllocMaxBlocks * 256];
};
static __device__ __align__(256) NoAllocScratch g_noalloc_scratch;

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {};
}  // namespace

cudaError_t launch_align_noalloc(const int32_t* topk_idx, int64_t A, int E, int C, int TB,
                                 int32_t* counts, int32_t* offsets, int32_t* sorted_ids,
                                 int32_t* slot_of, uint8_t* drop_mask, cudaStream_t stream) {
  if (A > kNoAllocMaxAssignments || E > 256) return cudaErrorInvalidValue;
  if (A > kAlignSingle && (A + align_chunk(A) - 1) / align_chunk(A) > kNoAllocMaxBlocks)
    return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  void* base = nullptr;
  {
    // In host code g_noalloc_scratch names a host-side stand-in, not device memory: the
    // device address is looked up once per device, with that device current.
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess) return e;
      g_noalloc_ptr[dev] = p;
    }
    base = g_noalloc_ptr[dev];
  }
  NoAllocScratch* sc = static_cast<NoAllocScratch*>(base);
  // The error word must start at zero; the histograms and the plan are fully rewritten.
  e = cudaMemsetAsync(sc->err, 0, sizeof(int), stream);
  if (e != cudaSuccess) return e;
  return launch_align(topk_idx, A, E, C, TB, sc->blk_hist, counts, offsets, sc->blk_prefix,
                      sorted_ids, slot_of, drop_mask, sc->err, stream);
}

cudaError_t launch_plan_from_offsets(const int32_t* offsets, int E, int TB, int32_t* blk_prefix,
                                     cudaStream_t stream) {
  return launch_kernel(plan_from_offsets_kernel, dim3(1), dim3(kThreads), 0, stream, 1, offsets, E,
                       TB, blk_prefix);
}

}  // namespace moe
