// quant.cu — FP8 (e4m3) quantisation of expert weights, one float32 scale per output channel.
//
// [P5] "大模型推理加速200%+？…", section "4.3 MOE量化方案矩阵" lists quantised expert GEMMs
// (W16A16, W8A8 with INT8/FP8, W4A8, W4A16) with offline weight repacking, without a numeric
// scheme. The scheme here takes the FP8 weights of W8A8 with the 16-bit activations of W4A16
// (W8A16): for weights w [E][K][M] (K the reduction dimension, M the output channels)
//   scale[e][m] = max_k |w[e][k][m]| / 448   (1 when the column is all zero), float32
//   code[e][k][m] = e4m3(w[e][k][m] / scale[e][m]), nearest-even, saturating at +-448
// Both divisions are IEEE float32 divisions; the e4m3 rounding is the hardware conversion.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 256;

// One thread per (expert, output channel): the column's largest magnitude over K.
__global__ void __launch_bounds__(kThreads)
    fp8_scale_kernel(const __nv_bfloat16* __restrict__ w, int K, int M, float* __restrict__ scale) {
  pdl_enter<false>();
  const int e = blockIdx.y;
  const int m = blockIdx.x * kThreads + threadIdx.x;
  if (m >= M) return;
  const __nv_bfloat16* col = w + static_cast<size_t>(e) * K * M + m;
  float amax = 0.0f;
  for (int k = 0; k < K; ++k) amax = fmaxf(amax, fabsf(__bfloat162float(col[static_cast<size_t>(k) * M])));
  scale[static_cast<size_t>(e) * M + m] = amax > 0.0f ? amax / 448.0f : 1.0f;
}

// Two adjacent output channels per thread (M is even), grid-stride over all weights.
__global__ void __launch_bounds__(kThreads)
    fp8_quant_kernel(const __nv_bfloat16* __restrict__ w, const float* __restrict__ scale,
                     int64_t pairs, int M, int64_t KM, uint16_t* __restrict__ codes) {
  pdl_enter<false>();
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; i < pairs;
       i += static_cast<int64_t>(gridDim.x) * kThreads) {
    const int64_t idx = 2 * i;
    const int64_t e = idx / KM;
    const int m = static_cast<int>(idx % M);
    const float* sc = scale + e * M + m;
    float2 v;
    v.x = __bfloat162float(w[idx]) / sc[0];
    v.y = __bfloat162float(w[idx + 1]) / sc[1];
    codes[i] = static_cast<uint16_t>(__nv_cvt_float2_to_fp8x2(v, __NV_SATFINITE, __NV_E4M3));
  }
}

}  // namespace

cudaError_t launch_quantize_fp8(const void* w, int64_t E, int K, int M, uint8_t* codes,
                                float* scale, int num_sms, cudaStream_t stream) {
  if (E == 0 || K == 0 || M == 0) return cudaSuccess;
  const dim3 g1(static_cast<unsigned>((M + kThreads - 1) / kThreads), static_cast<unsigned>(E));
  cudaError_t e = launch_kernel(fp8_scale_kernel, g1, dim3(kThreads), 0, stream, 1,
                                static_cast<const __nv_bfloat16*>(w), K, M, scale);
  if (e != cudaSuccess) return e;
  const int64_t pairs = E * static_cast<int64_t>(K) * M / 2;
  int64_t blocks = (pairs + kThreads - 1) / kThreads;
  const int64_t cap = static_cast<int64_t>(num_sms) * 16;
  if (blocks > cap) blocks = cap;
  return launch_kernel(fp8_quant_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kThreads), 0,
                       stream, 1, static_cast<const __nv_bfloat16*>(w), scale, pairs, M,
                       static_cast<int64_t>(K) * M, reinterpret_cast<uint16_t*>(codes));
}

}  // namespace moe
