// combine.cu — weighted merge of the expert outputs back into token order.
//
// [P1] "MoE 模型的 FlashAttention 跟普通模型有什么不一样？", section "融合二：expert 计算的输出 + 合并结果":
// accum += route_weight * expert_output; [P5] "大模型推理加速200%+？…", section "3.2 Fuse RMS RoPE &
// MoE Align & MoE Sum" (128-bit vector reads/writes).
//
// out[t,:] = sum over kept j of topk_w[t,j] * y_slots[slot_of[t*k+j],:], fp32 accumulation in
// ascending j, rounded once. One block per token; each thread owns 16-byte chunks of the row
// and issues the (up to 16) expert-row loads of a chunk back to back before accumulating.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxK = 16;

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

template <typename T>
__global__ void __launch_bounds__(kThreads)
    combine_kernel(const T* __restrict__ y, const int32_t* __restrict__ slot_of,
                   const float* __restrict__ topk_w, T* __restrict__ out, int64_t Ttok, int H,
                   int k) {
  constexpr int N = Vec<T>::N;
  __shared__ int s_slot[kMaxK];
  __shared__ float s_w[kMaxK];
  for (int64_t t = blockIdx.x; t < Ttok; t += gridDim.x) {
    if (threadIdx.x < k) {
      s_slot[threadIdx.x] = slot_of[t * k + threadIdx.x];
      s_w[threadIdx.x] = topk_w[t * k + threadIdx.x];
    }
    __syncthreads();
    for (int c = threadIdx.x * N; c < H; c += kThreads * N) {
      uint4 raw[kMaxK];
#pragma unroll
      for (int j = 0; j < kMaxK; ++j) {
        if (j < k && s_slot[j] >= 0)
          raw[j] = __ldg(reinterpret_cast<const uint4*>(y + static_cast<size_t>(s_slot[j]) * H + c));
      }
      float acc[N];
#pragma unroll
      for (int i = 0; i < N; ++i) acc[i] = 0.f;
#pragma unroll
      for (int j = 0; j < kMaxK; ++j) {
        if (j < k && s_slot[j] >= 0) {
          const float wj = s_w[j];
          float v[N];
          Vec<T>::widen(raw[j], v);
#pragma unroll
          for (int i = 0; i < N; ++i) acc[i] = fmaf(wj, v[i], acc[i]);
        }
      }
      Vec<T>::store(out + static_cast<size_t>(t) * H + c, acc);
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_combine(int dtype, const void* y_slots, const int32_t* slot_of,
                           const float* topk_w, void* out, int64_t T, int H, int k,
                           cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const int64_t blocks = T < 65535 * 8 ? T : 65535 * 8;
  if (dtype == 0)
    combine_kernel<float><<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(
        static_cast<const float*>(y_slots), slot_of, topk_w, static_cast<float*>(out), T, H, k);
  else
    combine_kernel<__nv_bfloat16><<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(y_slots), slot_of, topk_w,
        static_cast<__nv_bfloat16*>(out), T, H, k);
  return cudaGetLastError();
}

}  // namespace moe
