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
// identical to the sequential definition. Up to kAlignCluster assignments one launch does all
// of it (one block up to kAlignSingle, one cluster of CTAs above); beyond that one cooperative
// launch with a grid barrier (align_grid_kernel), or, when its CTAs cannot all be resident,
// three kernels:
//   1. hist:    per chunk of align_chunk(A) assignments, per-expert counts (shared-memory
//               atomics).
//   2. scan:    one block; per expert, exclusive prefix over chunks (chunk bases; the chunks
//               of an expert split over several threads), raw totals, counts = min(raw, C),
//               offsets = exclusive scan of counts, and the token-block plan blk_prefix used by
//               the expert GEMMs.
//   3. scatter: per chunk, stable in-chunk ranks (warp_peers + per-warp prefix),
//               then slot = offsets[e] + rank for kept assignments; fills the -1 tail.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kBlockThreads = 1024;  // threads of each CTA of the one-launch cluster grouping
constexpr int kMaxE = 256;
constexpr int kClusterCtas = 8;       // CTAs of the one-launch grouping's cluster (portable size)

// Lanes of the warp whose key equals this lane's, for keys below 2^nbits (nbits <= 8); lanes
// with ok == false belong to no group and get 0. Warp-level multisplit by ballots over the
// key's bits (S. Ashkiani et al., "GPU Multisplit", PPoPP 2016): a lane's peers are the
// intersection, over the bits, of the lanes that agree with it on that bit.
__device__ __forceinline__ uint32_t warp_peers(uint32_t key, bool ok, int nbits) {
  uint32_t peers = __ballot_sync(0xffffffffu, ok);
#pragma unroll
  for (int b = 0; b < 8; ++b) {
    if (b < nbits) {  // uniform across the warp
      const bool bit = (key >> b) & 1u;
      const uint32_t m = __ballot_sync(0xffffffffu, bit);
      peers &= bit ? m : ~m;
    }
  }
  return ok ? peers : 0u;
}

// The two halves of a cluster-wide barrier, for work between arriving and waiting.
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// 32-bit load from another CTA's shared memory (a shared::cluster address from mapa_shared).
__device__ __forceinline__ int ld_shared_cluster_s32(uint32_t cluster_addr) {
  int v;
  asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(cluster_addr) : "memory");
  return v;
}

__global__ void __launch_bounds__(kThreads)
    align_hist_kernel(const int32_t* __restrict__ idx, int64_t A, int E, int chunk,
                      int32_t* __restrict__ blk_hist, int* err) {
  pdl_enter<false>();
  __shared__ int h[kMaxE];
  for (int e = threadIdx.x; e < E; e += kThreads) h[e] = 0;
  __syncthreads();
  const int64_t base = static_cast<int64_t>(blockIdx.x) * chunk;
  const int64_t end = min(A, base + chunk);
  // a thread's ids of the chunk (at most kAlignChunkMax / kThreads = 8) are loaded together
  constexpr int kPer = kAlignChunkMax / kThreads;
  int ids[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int64_t a = base + threadIdx.x + static_cast<int64_t>(i) * kThreads;
    ids[i] = (a < end) ? __ldg(idx + a) : -1;
  }
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int64_t a = base + threadIdx.x + static_cast<int64_t>(i) * kThreads;
    if (a >= end) continue;
    const int e = ids[i];
    if (e >= 0 && e < E) atomicAdd(&h[e], 1);
    else flag_error(err, kDevBadExpert);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kThreads)
    blk_hist[static_cast<size_t>(blockIdx.x) * E + e] = h[e];
}

// Exclusive block-wide scan of one int per thread (NW warps, NW <= 32; sh holds NW ints).
template <int NW = kWarps>
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
    int w = (lane < NW) ? sh[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, w, off);
      if (lane >= off) w += o;
    }
    if (lane < NW) sh[lane] = w;  // inclusive warp totals
  }
  __syncthreads();
  const int warp_base = (warp > 0) ? sh[warp - 1] : 0;
  total = sh[NW - 1];
  __syncthreads();
  return warp_base + inc - v;
}

// Two exclusive block-wide scans at once (NW warps, NW <= 32; sh2 holds NW int2): returns the
// prefix of a, sets b_prefix, and the totals of a and b.
template <int NW>
__device__ __forceinline__ int block_exclusive_scan2(int a, int b, int2* sh2, int& total_a,
                                                     int& total_b, int& b_prefix) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int ia = a, ib = b;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int oa = __shfl_up_sync(0xffffffffu, ia, off);
    const int ob = __shfl_up_sync(0xffffffffu, ib, off);
    if (lane >= off) {
      ia += oa;
      ib += ob;
    }
  }
  if (lane == 31) sh2[warp] = make_int2(ia, ib);
  __syncthreads();
  if (warp == 0) {
    int2 w = (lane < NW) ? sh2[lane] : make_int2(0, 0);
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int oa = __shfl_up_sync(0xffffffffu, w.x, off);
      const int ob = __shfl_up_sync(0xffffffffu, w.y, off);
      if (lane >= off) {
        w.x += oa;
        w.y += ob;
      }
    }
    if (lane < NW) sh2[lane] = w;  // inclusive warp totals
  }
  __syncthreads();
  const int2 wb = (warp > 0) ? sh2[warp - 1] : make_int2(0, 0);
  total_a = sh2[NW - 1].x;
  total_b = sh2[NW - 1].y;
  __syncthreads();
  b_prefix = wb.y + ib - b;
  return wb.x + ia - a;
}

// Chunk bases, counts, offsets and the token-block plan, one block of kScanThreads threads.
// Thread (s, e), tid = s * Ep + e (Ep = E rounded up to a power of two, S = kScanThreads / Ep
// splits capped at kScanMaxSplit), owns the chunks [s*per, (s+1)*per) of expert e: it sums them
// (pass 1), takes the sums of the splits before it as its base, then rewrites each chunk's count
// as the running base (pass 2). Every chain of dependent loads is per/8 batches long instead of
// nblk/8 for one thread per expert.
constexpr int kScanThreads = 1024;
constexpr int kScanMaxSplit = 64;

__global__ void __launch_bounds__(kScanThreads)
    align_scan_kernel(int32_t* __restrict__ blk_hist, int nblk, int E, int C, int TB,
                      int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                      int32_t* __restrict__ blk_prefix) {
  pdl_enter<false>();
  __shared__ int part[kScanThreads];
  __shared__ int sh[kScanThreads / 32];
  int Ep = 1;
  while (Ep < E) Ep <<= 1;
  int S = kScanThreads / Ep;
  if (S > kScanMaxSplit) S = kScanMaxSplit;
  const int tid = threadIdx.x;
  const int e = tid % Ep, sp = tid / Ep;
  const bool act = sp < S && e < E;
  const int per = (nblk + S - 1) / S;
  const int c0 = sp * per;
  const int c1 = min(nblk, c0 + per);
  int sum = 0;
  if (act) {
    for (int b0 = c0; b0 < c1; b0 += 8) {
      int c[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        c[i] = (b0 + i < c1) ? blk_hist[static_cast<size_t>(b0 + i) * E + e] : 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) sum += c[i];
    }
  }
  part[tid] = sum;
  __syncthreads();
  int base = 0, raw = 0;
  if (act) {
    for (int q = 0; q < S; ++q) {
      const int v = part[q * Ep + e];
      if (q < sp) base += v;
      raw += v;
    }
    int run = base;
    for (int b0 = c0; b0 < c1; b0 += 8) {
      int c[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        c[i] = (b0 + i < c1) ? blk_hist[static_cast<size_t>(b0 + i) * E + e] : 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (b0 + i < c1) blk_hist[static_cast<size_t>(b0 + i) * E + e] = run;
        run += c[i];
      }
    }
  }
  // counts, offsets and the plan: threads tid < Ep hold experts e = tid (split 0)
  const int cnt = (sp == 0 && e < E) ? min(raw, C) : 0;
  const int nb = (cnt + TB - 1) / TB;
  int tot_cnt, tot_nb;
  const int off = block_exclusive_scan<kScanThreads / 32>(cnt, sh, tot_cnt);
  const int bp = block_exclusive_scan<kScanThreads / 32>(nb, sh, tot_nb);
  if (sp == 0 && e < E) {
    counts[e] = cnt;
    offsets[e] = off;
    if (blk_prefix != nullptr) blk_prefix[e] = bp;
  }
  if (tid == 0) {
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
  __shared__ uint16_t code[kAlignChunkMax];  // the chunk's ids (0xFFFF: none or invalid)
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < kWarps * kMaxE; i += kThreads) (&wrun[0][0])[i] = 0;
  for (int e = threadIdx.x; e < E; e += kThreads) s_off[e] = offsets[e];
  const int per_warp = chunk / kWarps;  // a multiple of 32
  const int64_t cbase = static_cast<int64_t>(blockIdx.x) * chunk;
  const int64_t wbase = cbase + warp * per_warp;
  {
    // the chunk's ids, read once (a thread's loads in flight together)
    constexpr int kPer = kAlignChunkMax / kThreads;
    int ids[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int o = threadIdx.x + i * kThreads;
      const int64_t a = cbase + o;
      ids[i] = (o < chunk && a < A) ? __ldg(idx + a) : -1;
    }
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int o = threadIdx.x + i * kThreads;
      if (o < chunk)
        code[o] = (ids[i] >= 0 && ids[i] < E) ? static_cast<uint16_t>(ids[i]) : uint16_t{0xFFFF};
    }
  }
  __syncthreads();

  const int nbits = (E > 1) ? 32 - __clz(E - 1) : 0;
  const int wofs = warp * per_warp;  // this warp's first id in `code`
  // pass 1: per-warp per-expert counts of this warp's assignments
  for (int step = 0; step < per_warp / 32; ++step) {
    const uint32_t c = code[wofs + step * 32 + lane];
    if (c != 0xFFFFu) atomicAdd(&wrun[warp][c], 1);
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
    const uint32_t c = code[wofs + step * 32 + lane];
    const bool ok = in && c != 0xFFFFu;
    const int e = ok ? static_cast<int>(c) : -1;
    const uint32_t peers = warp_peers(static_cast<uint32_t>(e), ok, nbits);
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

// Whole grouping in one launch of one cluster of CS CTAs of NT threads (CS = 1: a single
// block), for A <= CS * NT * MAXS. CTA r of the cluster owns a contiguous slice of the
// assignments and warp w of it a contiguous segment of `steps` rounds of 32. idx is read once,
// 8 loads of a lane in flight together, into 16-bit codes in dynamic shared memory
// (code_sm[round * NT + thread], NT * MAXS * 2 bytes; 0xFFFF: no assignment or an invalid id).
//   1. per-warp per-expert counts (shared-memory atomics: counting needs no order);
//   2. per expert, the exclusive prefix over this CTA's warps and the CTA's total;
//   3. cluster barrier; every CTA reads all CTAs' totals through distributed shared memory,
//      giving its own base (CTAs of lower rank) and the raw totals; each derives counts,
//      offsets and the token-block plan (CTA 0 writes them);
//   4. stable ranks in assignment order (warp_peers) and the scatter.
// A second cluster barrier, arrived on after the remote reads and waited on at exit, keeps
// every CTA's totals alive until no CTA reads them any more.
template <int NT, int CS, int MAXS>
__global__ void __launch_bounds__(NT, 1)
    align_cluster_kernel(const int32_t* __restrict__ idx, int64_t A, int E, int C, int TB,
                         int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                         int32_t* __restrict__ blk_prefix, int32_t* __restrict__ sorted_ids,
                         int32_t* __restrict__ slot_of, uint8_t* __restrict__ drop_mask,
                         int* err) {
  constexpr int NW = NT / 32;
  static_assert(MAXS % 8 == 0, "ids are loaded 8 rounds at a time");
  constexpr int kBatch = 8;
  pdl_enter<false>();
  __shared__ int wrun[NW][kMaxE];
  __shared__ int cta_tot[kMaxE];
  __shared__ int s_off[kMaxE];
  __shared__ int sh[NW];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r = (CS > 1) ? static_cast<int>(cluster_ctarank()) : 0;
  for (int i = threadIdx.x; i < NW * kMaxE; i += NT) (&wrun[0][0])[i] = 0;
  // rounds per warp: ceil(ceil(A / (CS * NW)) / 32) <= MAXS; A <= CS * NT * MAXS (checked by
  // the launcher), so 32-bit indices suffice
  const int An = static_cast<int>(A);
  const int steps = ((An + CS * NW - 1) / (CS * NW) + 31) / 32;
  const int wbase = (r * NW + warp) * steps * 32;
  const int nbits = (E > 1) ? 32 - __clz(E - 1) : 0;
  extern __shared__ uint16_t code_sm[];
#pragma unroll
  for (int s0 = 0; s0 < MAXS; s0 += kBatch) {
    if (s0 >= steps) break;  // uniform across the block
    int raw[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int a = wbase + (s0 + j) * 32 + lane;
      raw[j] = (s0 + j < steps && a < An) ? __ldg(idx + a) : -1;
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int s = s0 + j;
      const int a = wbase + s * 32 + lane;
      const bool ok = (raw[j] >= 0 && raw[j] < E);
      if (s < steps && a < An && !ok) flag_error(err, kDevBadExpert);
      code_sm[s * NT + threadIdx.x] = ok ? static_cast<uint16_t>(raw[j]) : uint16_t{0xFFFF};
    }
  }
  __syncthreads();
  // 1. per-warp per-expert counts
  for (int s = 0; s < steps; ++s) {
    const uint32_t c = code_sm[s * NT + threadIdx.x];
    if (c != 0xFFFFu) atomicAdd(&wrun[warp][c], 1);
  }
  __syncthreads();
  // 2. per expert: exclusive prefix across this CTA's warps, and the CTA's total
  const int e = threadIdx.x;
  int mine = 0;
  if (e < E) {
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const int c = wrun[w][e];
      wrun[w][e] = mine;
      mine += c;
    }
    cta_tot[e] = mine;
  }
  // 3. this CTA's base and the raw totals over the cluster, in CTA-rank order
  int before = 0, raw_tot = mine;
  if constexpr (CS > 1) {
    cluster_sync_all();
    if (e < E) {
      const uint32_t loc = smem_u32(&cta_tot[e]);
      raw_tot = 0;
#pragma unroll
      for (int q = 0; q < CS; ++q) {
        const int v = ld_shared_cluster_s32(mapa_shared(loc, q));
        if (q < r) before += v;
        raw_tot += v;
      }
    }
    cluster_arrive();
  }
  const int cnt = (e < E) ? min(raw_tot, C) : 0;
  const int nb = (cnt + TB - 1) / TB;
  int tot_cnt, tot_nb;
  const int off = block_exclusive_scan<NW>(cnt, sh, tot_cnt);
  const int bp = block_exclusive_scan<NW>(nb, sh, tot_nb);
  if (e < E) {
    s_off[e] = off;
    if (r == 0) {
      counts[e] = cnt;
      offsets[e] = off;
      if (blk_prefix != nullptr) blk_prefix[e] = bp;
    }
    if (before != 0) {
#pragma unroll
      for (int w = 0; w < NW; ++w) wrun[w][e] += before;
    }
  }
  if (e == 0 && r == 0) {
    offsets[E] = tot_cnt;
    if (blk_prefix != nullptr) blk_prefix[E] = tot_nb;
  }
  __syncthreads();
  // 4. stable ranks in assignment order, then the scatter
  for (int s = 0; s < steps; ++s) {  // uniform across the block
    const int a = wbase + s * 32 + lane;
    const bool in = a < An;
    const uint32_t c = code_sm[s * NT + threadIdx.x];
    const bool ok = c != 0xFFFFu;
    const int ea = static_cast<int>(c);
    const uint32_t peers = warp_peers(c, ok, nbits);
    int rank = 0;
    if (ok) rank = wrun[warp][ea] + __popc(peers & lanemask_lt());
    __syncwarp();
    if (ok && lane == __ffs(peers) - 1) wrun[warp][ea] += __popc(peers);
    __syncwarp();
    if (in) {
      if (ok && rank < C) {
        const int slot = s_off[ea] + rank;
        sorted_ids[slot] = a;
        slot_of[a] = slot;
        drop_mask[a] = 0;
      } else {
        slot_of[a] = -1;
        drop_mask[a] = 1;
      }
    }
  }
  for (int sl = tot_cnt + r * NT + threadIdx.x; sl < An; sl += CS * NT) sorted_ids[sl] = -1;
  if constexpr (CS > 1) cluster_wait();
}

// Whole grouping in one cooperative launch of G CTAs (at most one per SM, all resident at
// once), for kAlignCluster < A <= G * kGridThreads * kGridMaxSteps. Same steps as the cluster
// form; the per-CTA expert totals go through global memory (hist[r][e]) and a grid barrier
// instead of distributed shared memory:
//   1. ids into 16-bit codes in shared memory, per-warp per-expert counts;
//   2. per expert, the exclusive prefix over this CTA's warps; the CTA's totals to hist[r];
//   3. grid barrier (bounded wait); each CTA sums hist over the CTAs before it (its base) and
//      over all of them (raw totals), in CTA order, split over several threads per expert;
//      counts, offsets and the token-block plan as in the cluster form (CTA 0 writes them);
//   4. stable ranks in assignment order and the scatter.
// The barrier's two counters (arrivals, departures; bar[0], bar[1]) are zero between launches:
// the last CTA to leave the barrier resets both.
constexpr int kGridThreads = 1024;
constexpr int kGridMaxSteps = 64;  // rounds of 32 ids per warp: 128 KB of codes per CTA

__global__ void __launch_bounds__(kGridThreads, 1)
    align_grid_kernel(const int32_t* __restrict__ idx, int64_t A, int E, int C, int TB,
                      int32_t* __restrict__ hist, int* bar, int32_t* __restrict__ counts,
                      int32_t* __restrict__ offsets, int32_t* __restrict__ blk_prefix,
                      int32_t* __restrict__ sorted_ids, int32_t* __restrict__ slot_of,
                      uint8_t* __restrict__ drop_mask, int* err) {
  constexpr int NT = kGridThreads, NW = NT / 32, kBatch = 8;
  pdl_enter<false>();
  __shared__ int wrun[NW][kMaxE + 1];  // padded: a warp reads one column without conflicts
  __shared__ int s_off[kMaxE];
  __shared__ int s_base[kMaxE];        // this CTA's base per expert (totals of CTAs before it)
  __shared__ int part[2][NT];
  __shared__ int2 sh2[NW];
  __shared__ int s_ok;
  extern __shared__ uint16_t code_sm[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r = static_cast<int>(blockIdx.x), G = static_cast<int>(gridDim.x);
  for (int i = threadIdx.x; i < NW * (kMaxE + 1); i += NT) (&wrun[0][0])[i] = 0;
  // A <= G * NT * kGridMaxSteps (checked by the launcher): 32-bit indices suffice
  const int An = static_cast<int>(A);
  const int steps = ((An + G * NW - 1) / (G * NW) + 31) / 32;
  const int wbase = (r * NW + warp) * steps * 32;
  const int nbits = (E > 1) ? 32 - __clz(E - 1) : 0;
  for (int s0 = 0; s0 < steps; s0 += kBatch) {  // uniform across the block
    int raw[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int a = wbase + (s0 + j) * 32 + lane;
      raw[j] = (s0 + j < steps && a < An) ? __ldg(idx + a) : -1;
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int st = s0 + j;
      const int a = wbase + st * 32 + lane;
      const bool ok = (raw[j] >= 0 && raw[j] < E);
      if (st < steps && a < An && !ok) flag_error(err, kDevBadExpert);
      if (st < steps)
        code_sm[st * NT + threadIdx.x] = ok ? static_cast<uint16_t>(raw[j]) : uint16_t{0xFFFF};
    }
  }
  __syncthreads();
  // 1. per-warp per-expert counts
  for (int st = 0; st < steps; ++st) {
    const uint32_t c = code_sm[st * NT + threadIdx.x];
    if (c != 0xFFFFu) atomicAdd(&wrun[warp][c], 1);
  }
  __syncthreads();
  // 2. per expert: exclusive prefix across this CTA's warps, warp-parallel (warp w takes
  //    experts w, w + 32, ...; lane = source warp); the CTA's total to hist[r]
  for (int e = warp; e < E; e += NW) {
    const int c = wrun[lane][e];
    int inc = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, inc, off);
      if (lane >= off) inc += o;
    }
    wrun[lane][e] = inc - c;
    if (lane == 31) hist[static_cast<size_t>(r) * E + e] = inc;
  }
  // 3. grid barrier: every CTA's totals are written before any CTA reads them
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(&bar[0], 1);
    const unsigned long long t0 = global_ns();
    int ok = 1, v;
    for (;;) {
      asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(bar) : "memory");
      if (v >= G) break;
      if (global_ns() - t0 > kWaitLimitNs) {
        ok = 0;
        break;
      }
      __nanosleep(64);
    }
    if (!ok) flag_error(err, kDevWaitTimeout);
    __threadfence();
    s_ok = ok;
  }
  __syncthreads();
  if (!s_ok) return;  // the grouping is abandoned; the error word says so
  // thread (sp, e), tid = sp * Ep + e, sums the totals of CTAs [sp * per, (sp + 1) * per)
  int Ep = 1;
  while (Ep < E) Ep <<= 1;
  const int S = NT / Ep;
  const int e = threadIdx.x % Ep, sp = threadIdx.x / Ep;
  const int per = (G + S - 1) / S;
  int below = 0, all = 0;
  if (e < E) {
    const int q1 = min(G, (sp + 1) * per);
#pragma unroll 8
    for (int q = sp * per; q < q1; ++q) {
      const int v = __ldcg(hist + static_cast<size_t>(q) * E + e);
      all += v;
      below += (q < r) ? v : 0;
    }
  }
  part[0][threadIdx.x] = below;
  part[1][threadIdx.x] = all;
  __syncthreads();
  // every CTA has read what it needs from the counters: the last one out resets them
  if (threadIdx.x == 0 && atomicAdd(&bar[1], 1) == G - 1) {
    bar[0] = 0;
    bar[1] = 0;
  }
  int before = 0, raw_tot = 0;
  if (threadIdx.x < E) {
    for (int q = 0; q < S; ++q) {
      before += part[0][q * Ep + threadIdx.x];
      raw_tot += part[1][q * Ep + threadIdx.x];
    }
  }
  const int cnt = (threadIdx.x < E) ? min(raw_tot, C) : 0;
  const int nb = (cnt + TB - 1) / TB;
  int tot_cnt, tot_nb;
  int bp;
  const int off = block_exclusive_scan2<NW>(cnt, nb, sh2, tot_cnt, tot_nb, bp);
  if (threadIdx.x < E) {
    const int ee = threadIdx.x;
    s_off[ee] = off;
    s_base[ee] = before;
    if (r == 0) {
      counts[ee] = cnt;
      offsets[ee] = off;
      if (blk_prefix != nullptr) blk_prefix[ee] = bp;
    }
  }
  if (threadIdx.x == 0 && r == 0) {
    offsets[E] = tot_cnt;
    if (blk_prefix != nullptr) blk_prefix[E] = tot_nb;
  }
  __syncthreads();
  // 4. stable ranks in assignment order, then the scatter
  for (int st = 0; st < steps; ++st) {  // uniform across the block
    const int a = wbase + st * 32 + lane;
    const bool in = a < An;
    const uint32_t c = code_sm[st * NT + threadIdx.x];
    const bool ok = c != 0xFFFFu;
    const int ea = static_cast<int>(c);
    const uint32_t peers = warp_peers(c, ok, nbits);
    int rank = 0;
    if (ok) rank = s_base[ea] + wrun[warp][ea] + __popc(peers & lanemask_lt());
    __syncwarp();
    if (ok && lane == __ffs(peers) - 1) wrun[warp][ea] += __popc(peers);
    __syncwarp();
    if (in) {
      if (ok && rank < C) {
        const int slot = s_off[ea] + rank;
        sorted_ids[slot] = a;
        slot_of[a] = slot;
        drop_mask[a] = 0;
      } else {
        slot_of[a] = -1;
        drop_mask[a] = 1;
      }
    }
  }
  for (int sl = tot_cnt + r * NT + threadIdx.x; sl < An; sl += G * NT) sorted_ids[sl] = -1;
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
  if (A <= kAlignSingle) {
    constexpr int kMaxs = kAlignSingle / kThreads;
    return launch_kernel(align_cluster_kernel<kThreads, 1, kMaxs>, dim3(1), dim3(kThreads),
                         size_t{kThreads} * kMaxs * 2, stream, 1, topk_idx, A, E, C, TB, counts,
                         offsets, blk_prefix, sorted_ids, slot_of, drop_mask, err);
  }
  if (A <= kAlignCluster) {
    constexpr int kMaxs = kAlignCluster / (kClusterCtas * kBlockThreads);
    static_assert(kMaxs * kClusterCtas * kBlockThreads == kAlignCluster, "cluster capacity");
    auto kernel = align_cluster_kernel<kBlockThreads, kClusterCtas, kMaxs>;
    constexpr size_t kCodeBytes = size_t{kBlockThreads} * kMaxs * 2;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kCodeBytes));
    if (e != cudaSuccess) return e;
    return launch_kernel(kernel, dim3(kClusterCtas), dim3(kBlockThreads), kCodeBytes, stream,
                         kClusterCtas, topk_idx, A, E, C, TB, counts, offsets, blk_prefix,
                         sorted_ids, slot_of, drop_mask, err);
  }
  const int chunk = align_chunk(A);
  const int nblk = static_cast<int>((A + chunk - 1) / chunk);
  // one cooperative launch when every CTA (one per SM, at most one per chunk histogram row of
  // blk_hist) can be resident and hold its share of the codes
  {
    int dev = 0, sms = 0, per_sm = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int G = nblk < sms ? nblk : sms;
    const int64_t steps = ((A + int64_t{G} * (kGridThreads / 32) - 1) /
                               (int64_t{G} * (kGridThreads / 32)) + 31) / 32;
    if (G > 0 && steps <= kGridMaxSteps) {
      const size_t code_bytes = static_cast<size_t>(steps) * kGridThreads * 2;
      e = cudaFuncSetAttribute(align_grid_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(code_bytes));
      if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, align_grid_kernel,
                                                          kGridThreads, code_bytes);
      if (e != cudaSuccess) return e;
      if (per_sm >= 1) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(G));
        cfg.blockDim = dim3(kGridThreads);
        cfg.dynamicSmemBytes = code_bytes;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, align_grid_kernel, topk_idx, A, E, C, TB, blk_hist,
                               err + kAlignBarrierWord, counts, offsets, blk_prefix, sorted_ids,
                               slot_of, drop_mask, err);
        // the GPU cannot hold every CTA at once (other work resident): the chunked kernels
        if (e != cudaErrorCooperativeLaunchTooLarge) return e;
        (void)cudaGetLastError();
      }
    }
  }
  cudaError_t e = launch_kernel(align_hist_kernel, dim3(nblk), dim3(kThreads), 0, stream, 1,
                                topk_idx, A, E, chunk, blk_hist, err);
  if (e == cudaSuccess)
    e = launch_kernel(align_scan_kernel, dim3(1), dim3(kScanThreads), 0, stream, 1, blk_hist,
                      nblk, E, C, TB, counts, offsets, blk_prefix);
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
void* g_noalloc_ctx[64] = {};  // the context each cached address belongs to

// The current driver context (CUcontext as void*), through the runtime's driver entry point so
// that the library does not link libcuda itself; nullptr if it cannot be queried.
void* current_context() {
  using CtxGetCurrentFn = int (*)(void**);
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(ptr);
  });
  void* ctx = nullptr;
  if (fn == nullptr || fn(&ctx) != 0) return nullptr;
  return ctx;
}
}  // namespace

cudaError_t launch_align_noalloc(const int32_t* topk_idx, int64_t A, int E, int C, int TB,
                                 int32_t* counts, int32_t* offsets, int32_t* sorted_ids,
                                 int32_t* slot_of, uint8_t* drop_mask, cudaStream_t stream) {
  if (A > kNoAllocMaxAssignments || E > 256) return cudaErrorInvalidValue;
  if (A > kAlignCluster && (A + align_chunk(A) - 1) / align_chunk(A) > kNoAllocMaxBlocks)
    return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  void* base = nullptr;
  {
    // In host code g_noalloc_scratch names a host-side stand-in, not device memory: the
    // device address is looked up once per device and context, with that device current. A
    // new context on the device (after cudaDeviceReset, say) loads the module again, so the
    // address is looked up again then; with no context query available it is looked up on
    // every call.
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    void* ctx = current_context();
    if (g_noalloc_ptr[dev] == nullptr || ctx == nullptr || g_noalloc_ctx[dev] != ctx) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess) return e;
      g_noalloc_ptr[dev] = p;
      g_noalloc_ctx[dev] = ctx;
    }
    base = g_noalloc_ptr[dev];
  }
  NoAllocScratch* sc = static_cast<NoAllocScratch*>(base);
  // The error word and the grid barrier's counters must start at zero; the histograms and the
  // plan are fully rewritten.
  e = cudaMemsetAsync(sc->err, 0, sizeof(sc->err), stream);
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
