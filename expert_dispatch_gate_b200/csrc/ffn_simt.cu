// ffn_simt.cu — float32 grouped SwiGLU expert FFN on CUDA cores.
//
// [P1] "MoE 模型的 FlashAttention 跟普通模型有什么不一样？", section "FlashAttention 在 MoE 模型里的位置",
// step 4, with the SwiGLU expert of section "手动编译 MoE 融合算子" (activation "silu").
//
// The float32 contract (1e-4 relative to the output's max) rules out the tf32 tensor-core kinds,
// so float32 layers run here: one block per (kept slot, 128-feature block); the slot's input row
// is staged in shared memory and each thread owns one output feature, reading the weight matrix
// along its contiguous feature dimension (coalesced across the block).
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 128;

__device__ __forceinline__ int expert_of_slot(const int32_t* offsets, int E, int s) {
  int lo = 0, hi = E;  // largest e with offsets[e] <= s
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (offsets[mid] <= s) lo = mid; else hi = mid;
  }
  return lo;
}

__global__ void __launch_bounds__(kThreads)
    gemm1_simt_kernel(const float* __restrict__ x, const int32_t* __restrict__ sorted_ids,
                      const int32_t* __restrict__ offsets, const float* __restrict__ wg,
                      const float* __restrict__ wu, float* __restrict__ hbuf, int H, int E, int k,
                      int I) {
  pdl_enter<false>();
  extern __shared__ float xs[];
  const int s = blockIdx.x;
  if (s >= offsets[E]) return;  // uniform across the block
  const int e = expert_of_slot(offsets, E, s);
  const int t = sorted_ids[s] / k;
  for (int h = threadIdx.x; h < H; h += kThreads) xs[h] = x[static_cast<size_t>(t) * H + h];
  __syncthreads();
  const int i = blockIdx.y * kThreads + threadIdx.x;
  if (i >= I) return;
  const float* g_col = wg + static_cast<size_t>(e) * H * I + i;
  const float* u_col = wu + static_cast<size_t>(e) * H * I + i;
  float g = 0.f, u = 0.f;
  for (int h = 0; h < H; ++h) {
    g = fmaf(xs[h], __ldg(g_col + static_cast<size_t>(h) * I), g);
    u = fmaf(xs[h], __ldg(u_col + static_cast<size_t>(h) * I), u);
  }
  hbuf[static_cast<size_t>(s) * I + i] = g / (1.0f + expf(-g)) * u;
}

__global__ void __launch_bounds__(kThreads)
    gemm2_simt_kernel(const float* __restrict__ hbuf, const int32_t* __restrict__ offsets,
                      const float* __restrict__ wd, float* __restrict__ y, int H, int E, int I) {
  pdl_enter<false>();
  extern __shared__ float hs[];
  const int s = blockIdx.x;
  if (s >= offsets[E]) return;
  const int e = expert_of_slot(offsets, E, s);
  for (int i = threadIdx.x; i < I; i += kThreads) hs[i] = hbuf[static_cast<size_t>(s) * I + i];
  __syncthreads();
  const int c = blockIdx.y * kThreads + threadIdx.x;
  if (c >= H) return;
  const float* d_col = wd + static_cast<size_t>(e) * I * H + c;
  float acc = 0.f;
  for (int i = 0; i < I; ++i) acc = fmaf(hs[i], __ldg(d_col + static_cast<size_t>(i) * H), acc);
  y[static_cast<size_t>(s) * H + c] = acc;
}

}  // namespace

cudaError_t launch_gemm1_simt(const float* x, const int32_t* sorted_ids, const int32_t* offsets,
                              const float* w_gate, const float* w_up, float* hbuf, int64_t A,
                              int H, int E, int k, int I, cudaStream_t stream) {
  if (A == 0) return cudaSuccess;
  const size_t smem = static_cast<size_t>(H) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(gemm1_simt_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  dim3 grid(static_cast<unsigned>(A), static_cast<unsigned>((I + kThreads - 1) / kThreads));
  return launch_kernel(gemm1_simt_kernel, grid, dim3(kThreads), smem, stream, 1, x, sorted_ids,
                       offsets, w_gate, w_up, hbuf, H, E, k, I);
}

cudaError_t launch_gemm2_simt(const float* hbuf, const int32_t* offsets, const float* w_down,
                              float* y, int64_t A, int H, int E, int I, cudaStream_t stream) {
  if (A == 0) return cudaSuccess;
  const size_t smem = static_cast<size_t>(I) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(gemm2_simt_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  dim3 grid(static_cast<unsigned>(A), static_cast<unsigned>((H + kThreads - 1) / kThreads));
  return launch_kernel(gemm2_simt_kernel, grid, dim3(kThreads), smem, stream, 1, hbuf, offsets,
                       w_down, y, H, E, I);
}

}  // namespace moe
