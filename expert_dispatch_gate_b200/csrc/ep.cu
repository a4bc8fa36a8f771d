// ep.cu — expert parallelism over R ranks: placement plan, dispatch of token rows to the experts'
// owners, and the combine that reads the expert outputs back from the owners.
//
// [P4] "MoE Router" (2048ai.net), section "Token 分发的通信瓶颈": with experts spread over devices,
// every token row goes to the devices that own its experts and the outputs come back (AlltoAllV);
// section "昇腾NPU的通信计算重叠": at most C assignments per expert, the overflow dropped.
//
// Rank r holds its own tokens and the experts [r*El, (r+1)*El), El = E/R. The ranks compute what
// one device computes on the concatenated batch (rank 0's tokens first): with counts_all[q][e]
// the number of assignments of rank q's tokens to expert e, rank r's assignment a to e has the
// global rank  g = sum_{q<r} counts_all[q][e] + (its rank among rank r's assignments to e), and
// is kept iff g < C. Its row goes to owner e / El at slot  own_off[e] + g, own_off being the
// exclusive prefix of min(total[e], C) over the owner's own experts: the owner's rows come out
// expert-major and in global token order, as a one-device grouping would lay them out.
//
// Rows move by plain stores into, and plain loads from, the other ranks' buffers through the
// pointers in peer_xs / peer_y (peer memory mapped into this device's address space, or, when R
// ranks are emulated on one device, the other ranks' buffers there). No TMA touches peer memory.
// Ordering between ranks uses one flag word per (announcing rank, receiving rank): the announcing
// rank stores a step number (epoch) with a system-scope release after its stores, and the
// receiving rank waits for it with a bounded system-scope acquire loop.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxE = 256;

// owner / slot of every local assignment, and (block 0) the offsets of this rank's experts.
__global__ void __launch_bounds__(kThreads)
    ep_plan_kernel(const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ slot_of_local,
                   const int32_t* __restrict__ offsets_local,
                   const int32_t* __restrict__ counts_all, int64_t A, int E, int R, int rank, int C,
                   int32_t* __restrict__ owner, int32_t* __restrict__ slot,
                   int32_t* __restrict__ own_offsets, int* err) {
  pdl_enter<false>();
  __shared__ int before[kMaxE];
  __shared__ int own_off[kMaxE];
  __shared__ int cnt[kMaxE];
  const int El = E / R;
  for (int e = threadIdx.x; e < E; e += kThreads) {
    int b = 0, tot = 0;
    for (int q = 0; q < R; ++q) {
      const int c = counts_all[static_cast<size_t>(q) * E + e];
      if (q < rank) b += c;
      tot += c;
    }
    before[e] = b;
    cnt[e] = min(tot, C);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kThreads) {
    int off = 0;
    for (int e2 = (e / El) * El; e2 < e; ++e2) off += cnt[e2];
    own_off[e] = off;
  }
  __syncthreads();
  if (blockIdx.x == 0) {
    for (int le = threadIdx.x; le <= El; le += kThreads)
      own_offsets[le] = (le < El) ? own_off[rank * El + le]
                                  : own_off[rank * El + El - 1] + cnt[rank * El + El - 1];
  }
  for (int64_t a = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; a < A;
       a += static_cast<int64_t>(gridDim.x) * kThreads) {
    const int e = topk_idx[a];
    int o = -1, s = -1;
    if (e >= 0 && e < E) {
      const int g = before[e] + (slot_of_local[a] - offsets_local[e]);
      if (g < C) {
        o = e / El;
        s = own_off[e] + g;
      }
    } else {
      flag_error(err, kDevBadExpert);
    }
    owner[a] = o;
    slot[a] = s;
  }
}

// One warp per local assignment: its token row, 16 bytes per lane access, to the owner's slot.
__global__ void __launch_bounds__(kThreads)
    ep_dispatch_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ owner,
                       const int32_t* __restrict__ slot, uint4* const* __restrict__ peer_xs,
                       int64_t A, int k, int row_chunks) {
  pdl_enter<false>();
  const int lane = threadIdx.x & 31;
  const int64_t a = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  if (a >= A) return;
  const int o = owner[a];
  if (o < 0) return;
  const uint4* src = x + (a / k) * row_chunks;
  uint4* dst = peer_xs[o] + static_cast<int64_t>(slot[a]) * row_chunks;
  for (int c = lane; c < row_chunks; c += 32) dst[c] = __ldg(src + c);
  // the rows reach the owner's memory before any later signal of this stream
  __threadfence_system();
}

// Step signal: stores `epoch` into slot `rank` of every rank's flag array (peer_flags[q] is rank
// q's array of R words), with release semantics at system scope, after a system-scope fence.
// Launched after the work it announces (the dispatch stores, or the owner's expert outputs), in
// stream order, so that work is complete and visible before any rank can see the new epoch.
__global__ void __launch_bounds__(32) ep_signal_kernel(uint32_t* const* __restrict__ peer_flags,
                                                       int R, int rank, uint32_t epoch) {
  pdl_enter<false>();
  __threadfence_system();
  for (int q = threadIdx.x; q < R; q += 32) {
    uint32_t* f = peer_flags[q] + rank;
    asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(f), "r"(epoch) : "memory");
  }
}

// Bounded wait until every rank q < R has signalled `epoch` in flags[q] (epochs compared modulo
// 2^32). A rank that never signals ends the wait after kWaitLimitNs: the kernel records
// kDevWaitTimeout in the error word and returns, so the host reads a status instead of a hang.
__global__ void __launch_bounds__(32) ep_wait_kernel(const uint32_t* __restrict__ flags, int R,
                                                     uint32_t epoch, int* err) {
  pdl_enter<false>();
  bool ok = true;
  for (int q = threadIdx.x; q < R; q += 32) {
    const unsigned long long t0 = global_ns();
    for (uint32_t i = 0;; ++i) {
      uint32_t v;
      asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(flags + q) : "memory");
      if (static_cast<int32_t>(v - epoch) >= 0) break;
      if ((i & 15u) == 15u && global_ns() - t0 > kWaitLimitNs) {
        ok = false;
        break;
      }
      __nanosleep(256);
    }
  }
  if (!ok) flag_error(err, kDevWaitTimeout);
}

template <typename T>
struct Vec;
template <>
struct Vec<float> {
  static constexpr int N = 4;
  __device__ static void widen(const uint4& r, float (&o)[4]) {
    o[0] = __uint_as_float(r.x); o[1] = __uint_as_float(r.y);
    o[2] = __uint_as_float(r.z); o[3] = __uint_as_float(r.w);
  }
  __device__ static void store(float* p, const float (&o)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(o[0], o[1], o[2], o[3]);
  }
};
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void widen(const uint4& r, float (&o)[8]) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      o[2 * i] = __uint_as_float(w[i] << 16);
      o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  __device__ static void store(__nv_bfloat16* p, const float (&o)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 b = __floats2bfloat162_rn(o[2 * i], o[2 * i + 1]);
      w[i] = *reinterpret_cast<const uint32_t*>(&b);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
  }
};

// out[t,:] = sum over kept j, ascending, of topk_w[t,j] * peer_y[owner][slot,:] in fp32, rounded
// once: the one-device combine with each expert row read from its owner. One warp per (token,
// segment of 32*kG 16-byte chunks); lane j < k holds assignment j's owner, slot and weight.
constexpr int kG = 4;

template <typename T>
__global__ void __launch_bounds__(kThreads, 2)
    ep_combine_kernel(const T* const* __restrict__ peer_y, const int32_t* __restrict__ owner,
                      const int32_t* __restrict__ slot, const float* __restrict__ topk_w,
                      T* __restrict__ out, int64_t Ttok, int H, int k, int segs) {
  pdl_enter<false>();
  constexpr int N = Vec<T>::N;
  const int lane = threadIdx.x & 31;
  const int64_t wid = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  const int64_t t = wid / segs;
  if (t >= Ttok) return;
  const int seg = static_cast<int>(wid - t * segs);
  const int my_owner = (lane < k) ? owner[t * k + lane] : -1;
  const int my_slot = (lane < k) ? slot[t * k + lane] : -1;
  const float my_w = (lane < k) ? topk_w[t * k + lane] : 0.f;
  const int nchunk = H / N;
  const int c0 = seg * 32 * kG + lane;
  float acc[kG][N];
#pragma unroll
  for (int g = 0; g < kG; ++g)
#pragma unroll
    for (int i = 0; i < N; ++i) acc[g][i] = 0.f;
  for (int j0 = 0; j0 < k; j0 += 4) {
    uint4 raw[4][kG];
    int ow[4];
    float wj[4];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      ow[jj] = __shfl_sync(0xffffffffu, my_owner, (j0 + jj) & 31);
      const int sl = __shfl_sync(0xffffffffu, my_slot, (j0 + jj) & 31);
      wj[jj] = __shfl_sync(0xffffffffu, my_w, (j0 + jj) & 31);
      if (j0 + jj >= k) ow[jj] = -1;
      if (ow[jj] >= 0) {
        const uint4* row =
            reinterpret_cast<const uint4*>(peer_y[ow[jj]] + static_cast<size_t>(sl) * H);
#pragma unroll
        for (int g = 0; g < kG; ++g) {
          const int c = c0 + 32 * g;
          if (c < nchunk) raw[jj][g] = row[c];
        }
      }
    }
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      if (ow[jj] < 0) continue;
#pragma unroll
      for (int g = 0; g < kG; ++g) {
        float v[N];
        Vec<T>::widen(raw[jj][g], v);
#pragma unroll
        for (int i = 0; i < N; ++i) acc[g][i] = fmaf(wj[jj], v[i], acc[g][i]);
      }
    }
  }
  T* orow = out + static_cast<size_t>(t) * H;
#pragma unroll
  for (int g = 0; g < kG; ++g) {
    const int c = c0 + 32 * g;
    if (c < nchunk) Vec<T>::store(orow + static_cast<size_t>(c) * N, acc[g]);
  }
}

}  // namespace

cudaError_t launch_ep_plan(const int32_t* topk_idx, const int32_t* slot_of_local,
                           const int32_t* offsets_local, const int32_t* counts_all, int64_t A,
                           int E, int R, int rank, int C, int32_t* owner, int32_t* slot,
                           int32_t* own_offsets, int* err, int num_sms, cudaStream_t stream) {
  int64_t blocks = (A + kThreads - 1) / kThreads;
  if (blocks < 1) blocks = 1;  // block 0 also writes own_offsets
  if (blocks > 4LL * num_sms) blocks = 4LL * num_sms;
  return launch_kernel(ep_plan_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kThreads), 0,
                       stream, 1, topk_idx, slot_of_local, offsets_local, counts_all, A, E, R,
                       rank, C, owner, slot, own_offsets, err);
}

cudaError_t launch_ep_dispatch(int dtype, const void* x, const int32_t* owner, const int32_t* slot,
                               void* const* peer_xs, int64_t A, int k, int H,
                               cudaStream_t stream) {
  if (A == 0) return cudaSuccess;
  const int row_chunks = H * (dtype == 0 ? 4 : 2) / 16;
  const unsigned grid = static_cast<unsigned>((A + kWarps - 1) / kWarps);
  return launch_kernel(ep_dispatch_kernel, dim3(grid), dim3(kThreads), 0, stream, 1,
                       static_cast<const uint4*>(x), owner, slot,
                       reinterpret_cast<uint4* const*>(peer_xs), A, k, row_chunks);
}

cudaError_t launch_ep_signal(uint32_t* const* peer_flags, int R, int rank, uint32_t epoch,
                             cudaStream_t stream) {
  return launch_kernel(ep_signal_kernel, dim3(1), dim3(32), 0, stream, 1, peer_flags, R, rank,
                       epoch);
}

cudaError_t launch_ep_wait(const uint32_t* flags, int R, uint32_t epoch, int* err,
                           cudaStream_t stream) {
  return launch_kernel(ep_wait_kernel, dim3(1), dim3(32), 0, stream, 1, flags, R, epoch, err);
}

cudaError_t launch_ep_combine(int dtype, const void* const* peer_y, const int32_t* owner,
                              const int32_t* slot, const float* topk_w, void* out, int64_t T,
                              int H, int k, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const int n = (dtype == 0) ? 4 : 8;
  const int segs = static_cast<int>((H / n + 32 * kG - 1) / (32 * kG));
  const int64_t blocks = (T * segs + kWarps - 1) / kWarps;
  const dim3 grid(static_cast<unsigned>(blocks));
  if (dtype == 0)
    return launch_kernel(ep_combine_kernel<float>, grid, dim3(kThreads), 0, stream, 1,
                         reinterpret_cast<const float* const*>(peer_y), owner, slot, topk_w,
                         static_cast<float*>(out), T, H, k, segs);
  return launch_kernel(ep_combine_kernel<__nv_bfloat16>, grid, dim3(kThreads), 0, stream, 1,
                       reinterpret_cast<const __nv_bfloat16* const*>(peer_y), owner, slot, topk_w,
                       static_cast<__nv_bfloat16*>(out), T, H, k, segs);
}

}  // namespace moe
