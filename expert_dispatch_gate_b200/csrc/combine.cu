// combine.cu — weighted merge of the expert outputs back into token order.
//
// [P1] "MoE 模型的 FlashAttention 跟普通模型有什么不一样？", section "融合二：expert 计算的输出 + 合并结果":
// accum += route_weight * expert_output; [P5] "大模型推理加速200%+？…", section "3.2 Fuse RMS RoPE &
// MoE Align & MoE Sum" (128-bit vector reads/writes).
//
// out[t,:] = sum over kept j of topk_w[t,j] * y_slots[slot_of[t*k+j],:]
//            (+ shared_factor * shared[t,:]) (+ out_bias[:]),
// fp32 accumulation in ascending j, then the shared-expert term, then the bias, rounded once
// ([P5] section 3.2: the MoE sum fuses the shared expert's factor and the bias add).
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 256;

template <typename T>
struct Vec;  // a 16-byte chunk of T: raw load, widen to float, narrow-and-store
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

// One warp per (token, row segment of 32*kG 16-byte chunks). Lane j < k holds slot_of/topk_w
// of assignment j (broadcast by shuffle); lane l owns chunks l, l+32, ... of the segment, and
// every expert row's loads for those chunks are issued before they are accumulated.
constexpr int kWarps = kThreads / 32;
constexpr int kG = 4;

// Two blocks per SM (registers capped accordingly) keep enough row loads in flight.
template <typename T>
__global__ void __launch_bounds__(kThreads, 2)
    combine_kernel(const T* __restrict__ y, const int32_t* __restrict__ slot_of,
                   const float* __restrict__ topk_w, const T* __restrict__ shared,
                   float shared_factor, const float* __restrict__ out_bias, T* __restrict__ out,
                   int64_t Ttok, int H, int k, int segs, int* err) {
  pdl_enter<false>();
  constexpr int N = Vec<T>::N;
  const int lane = threadIdx.x & 31;
  const int64_t wid = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  const int64_t t = wid / segs;
  if (t >= Ttok) return;
  const int seg = static_cast<int>(wid - t * segs);
  int my_slot = (lane < k) ? slot_of[t * k + lane] : -1;
  if (kDebugChecks && my_slot >= Ttok * k) {  // y_slots holds T*k rows
    if (seg == 0) flag_error(err, kDevDebugBounds);
    my_slot = -1;
  }
  const float my_w = (lane < k) ? topk_w[t * k + lane] : 0.f;
  const int nchunk = H / N;
  T* orow = out + static_cast<size_t>(t) * H;
  {
    const int c0 = seg * 32 * kG + lane;
    float acc[kG][N];
#pragma unroll
    for (int g = 0; g < kG; ++g)
#pragma unroll
      for (int i = 0; i < N; ++i) acc[g][i] = 0.f;
    for (int j0 = 0; j0 < k; j0 += 4) {
      uint4 raw[4][kG];
      int sl[4];
      float wj[4];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        sl[jj] = __shfl_sync(0xffffffffu, my_slot, (j0 + jj) & 31);
        wj[jj] = __shfl_sync(0xffffffffu, my_w, (j0 + jj) & 31);
        if (j0 + jj >= k) sl[jj] = -1;
#pragma unroll
        for (int g = 0; g < kG; ++g) {
          const int c = c0 + 32 * g;
          if (sl[jj] >= 0 && c < nchunk)
            raw[jj][g] = __ldg(reinterpret_cast<const uint4*>(y + static_cast<size_t>(sl[jj]) * H) + c);
        }
      }
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        if (sl[jj] < 0) continue;
#pragma unroll
        for (int g = 0; g < kG; ++g) {
          float v[N];
          Vec<T>::widen(raw[jj][g], v);
#pragma unroll
          for (int i = 0; i < N; ++i) acc[g][i] = fmaf(wj[jj], v[i], acc[g][i]);
        }
      }
    }
    if (shared != nullptr) {
      const T* srow = shared + static_cast<size_t>(t) * H;
#pragma unroll
      for (int g = 0; g < kG; ++g) {
        const int c = c0 + 32 * g;
        if (c < nchunk) {
          float v[N];
          Vec<T>::widen(__ldg(reinterpret_cast<const uint4*>(srow) + c), v);
#pragma unroll
          for (int i = 0; i < N; ++i) acc[g][i] = fmaf(shared_factor, v[i], acc[g][i]);
        }
      }
    }
    if (out_bias != nullptr) {
#pragma unroll
      for (int g = 0; g < kG; ++g) {
        const int c = c0 + 32 * g;
        if (c < nchunk) {
#pragma unroll
          for (int i = 0; i < N; ++i) acc[g][i] += __ldg(out_bias + static_cast<size_t>(c) * N + i);
        }
      }
    }
#pragma unroll
    for (int g = 0; g < kG; ++g) {
      const int c = c0 + 32 * g;
      if (c < nchunk) Vec<T>::store(orow + static_cast<size_t>(c) * N, acc[g]);
    }
  }
}

// xs[s, :] = x[sorted_ids[s] / k, :] for every kept slot s < offsets[E]: the token rows in
// expert-major order, so a GEMM can stream them as contiguous rows. One warp per slot row.
template <typename T>
__global__ void __launch_bounds__(kThreads)
    dispatch_rows_kernel(const T* __restrict__ x, const int32_t* __restrict__ sorted_ids,
                         const int32_t* __restrict__ offsets, int E, int k, int H, int64_t rows,
                         int64_t Ttok, T* __restrict__ xs, int* err) {
  pdl_enter<false>();
  const int lane = threadIdx.x & 31;
  const int64_t s = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  if (s >= rows || s >= offsets[E]) return;
  const int64_t t = sorted_ids[s] / k;
  if (kDebugChecks && (sorted_ids[s] < 0 || t >= Ttok)) {
    if (lane == 0) flag_error(err, kDevDebugBounds);
    return;
  }
  const uint4* src = reinterpret_cast<const uint4*>(x + t * H);
  uint4* dst = reinterpret_cast<uint4*>(xs + s * H);
  const int n = H * static_cast<int>(sizeof(T)) / 16;
  for (int c = lane; c < n; c += 32) dst[c] = __ldg(src + c);
}

}  // namespace

cudaError_t launch_dispatch_rows(int dtype, const void* x, const int32_t* sorted_ids,
                                 const int32_t* offsets, int E, int k, int H, int64_t rows,
                                 int64_t T, void* xs, int* err, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>((rows + kWarps - 1) / kWarps);
  if (dtype == 0)
    return launch_kernel(dispatch_rows_kernel<float>, dim3(grid), dim3(kThreads), 0, stream, 1,
                         static_cast<const float*>(x), sorted_ids, offsets, E, k, H, rows, T,
                         static_cast<float*>(xs), err);
  return launch_kernel(dispatch_rows_kernel<__nv_bfloat16>, dim3(grid), dim3(kThreads), 0, stream,
                       1, static_cast<const __nv_bfloat16*>(x), sorted_ids, offsets, E, k, H, rows,
                       T, static_cast<__nv_bfloat16*>(xs), err);
}

cudaError_t launch_combine(int dtype, const void* y_slots, const int32_t* slot_of,
                           const float* topk_w, const void* shared, float shared_factor,
                           const float* out_bias, void* out, int64_t T, int H, int k,
                           int* err, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const int n = (dtype == 0) ? 4 : 8;  // elements per 16-byte chunk
  const int segs = static_cast<int>((H / n + 32 * kG - 1) / (32 * kG));
  const int64_t blocks = (T * segs + kWarps - 1) / kWarps;
  const dim3 grid(static_cast<unsigned>(blocks));
  if (dtype == 0)
    return launch_kernel(combine_kernel<float>, grid, dim3(kThreads), 0, stream, 1,
                         static_cast<const float*>(y_slots), slot_of, topk_w,
                         static_cast<const float*>(shared), shared_factor, out_bias,
                         static_cast<float*>(out), T, H, k, segs, err);
  return launch_kernel(combine_kernel<__nv_bfloat16>, grid, dim3(kThreads), 0, stream, 1,
                       static_cast<const __nv_bfloat16*>(y_slots), slot_of, topk_w,
                       static_cast<const __nv_bfloat16*>(shared), shared_factor, out_bias,
                       static_cast<__nv_bfloat16*>(out), T, H, k, segs, err);
}

}  // namespace moe
