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

// ---- FP8 weights and activations (W8A8): K-major weight codes and per-row activation codes
//
// W8A8 takes the weights of W8A16 stored transposed, codes[e][m][k] (the reduction dimension
// contiguous, as the tensor cores' e4m3 operands are read), and quantises the activations that
// enter each expert GEMM per row with the same rule: scale[r] = max_k |a[r][k]| / 448 (1 for a
// zero row), code[r][k] = e4m3(a[r][k] / scale[r]).

constexpr int kPackTile = 64;

// One block per (expert, 64 output channels, 64 K rows): reads the tile (a 128-byte run of
// channels per K row), converts, transposes through shared memory and writes 64 bytes of K per
// channel.
__global__ void __launch_bounds__(kThreads)
    pack_w8a8_kernel(const __nv_bfloat16* __restrict__ w, const float* __restrict__ scale, int K,
                     int M, uint8_t* __restrict__ codes) {
  pdl_enter<false>();
  __shared__ __align__(16) uint8_t tile[kPackTile][kPackTile + 16];
  const int e = blockIdx.z;
  const int m0 = blockIdx.x * kPackTile, k0 = blockIdx.y * kPackTile;
  const int tm = threadIdx.x % kPackTile, tk = threadIdx.x / kPackTile;
  const float sc = scale[static_cast<size_t>(e) * M + m0 + tm];
  const __nv_bfloat16* src = w + (static_cast<size_t>(e) * K + k0) * M + m0 + tm;
  for (int k = tk; k < kPackTile; k += kThreads / kPackTile) {
    const float v = __bfloat162float(src[static_cast<size_t>(k) * M]) / sc;
    tile[tm][k] = static_cast<uint8_t>(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
  }
  __syncthreads();
  const int row = threadIdx.x / 4, seg = threadIdx.x % 4;  // 64 channels x 4 16-byte segments
  const uint4 v = *reinterpret_cast<const uint4*>(&tile[row][seg * 16]);
  *reinterpret_cast<uint4*>(codes + (static_cast<size_t>(e) * M + m0 + row) * K + k0 + seg * 16) = v;
}

// The codes of one row of K values (bf16) held by one warp: lane l converts 16-byte chunks
// l, l + 32, ... (8 values each) after the warp has found the row's largest magnitude.
// Returns the row's scale.
__device__ __forceinline__ float warp_row_scale(const uint4* __restrict__ row, int nchunk,
                                                int lane) {
  uint32_t amax = 0;  // |v| as float bits: non-negative floats order like their bit patterns
  for (int c = lane; c < nchunk; c += 32) {
    const uint4 r = __ldg(row + c);
    const uint32_t w4[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      amax = max(amax, (w4[i] << 16) & 0x7fffffffu);
      amax = max(amax, w4[i] & 0x7fff0000u);
    }
  }
  amax = __reduce_max_sync(0xffffffffu, amax);
  const float a = __uint_as_float(amax);
  return a > 0.0f ? a / 448.0f : 1.0f;
}

// Eight bf16 values (one 16-byte chunk) divided by `sc` and converted to e4m3, as 8 bytes.
__device__ __forceinline__ uint2 chunk_codes(const uint4 r, float sc) {
  const uint32_t w4[4] = {r.x, r.y, r.z, r.w};
  uint32_t out[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float2 lo, hi;
    lo.x = __uint_as_float(w4[2 * h] << 16) / sc;
    lo.y = __uint_as_float(w4[2 * h] & 0xffff0000u) / sc;
    hi.x = __uint_as_float(w4[2 * h + 1] << 16) / sc;
    hi.y = __uint_as_float(w4[2 * h + 1] & 0xffff0000u) / sc;
    const uint32_t a = __nv_cvt_float2_to_fp8x2(lo, __NV_SATFINITE, __NV_E4M3);
    const uint32_t b = __nv_cvt_float2_to_fp8x2(hi, __NV_SATFINITE, __NV_E4M3);
    out[h] = (a & 0xffffu) | (b << 16);
  }
  return make_uint2(out[0], out[1]);
}

// Per-row quantisation of rows [N][K] (bf16, K % 8 == 0), one warp per row; rows at or past
// *n_dev (when given) are skipped.
__global__ void __launch_bounds__(kThreads)
    quant_rows_kernel(const __nv_bfloat16* __restrict__ a, int64_t N, const int32_t* n_dev,
                      int K, uint8_t* __restrict__ codes, float* __restrict__ scale) {
  pdl_enter<false>();
  const int lane = threadIdx.x & 31;
  const int64_t r = static_cast<int64_t>(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5);
  if (r >= N || (n_dev != nullptr && r >= *n_dev)) return;
  const int nchunk = K / 8;
  const uint4* row = reinterpret_cast<const uint4*>(a + r * K);
  const float sc = warp_row_scale(row, nchunk, lane);
  uint2* dst = reinterpret_cast<uint2*>(codes + r * K);
  for (int c = lane; c < nchunk; c += 32) dst[c] = chunk_codes(__ldg(row + c), sc);
  if (lane == 0) scale[r] = sc;
}

// W8A8 dispatch: the expert-major copy of the quantised token rows. Slot s of expert e takes the
// e4m3 row and the scale of token sorted_ids[s] / k from x8 / sxt (moe_quantize_rows of x, each
// token quantised once). One warp per slot row; rows past offsets[E] are not written.
__global__ void __launch_bounds__(kThreads)
    dispatch_rows_q8_kernel(const uint8_t* __restrict__ x8, const float* __restrict__ sxt,
                            const int32_t* __restrict__ sorted_ids,
                            const int32_t* __restrict__ offsets, int E, int k, int H, int64_t rows,
                            int64_t Ttok, uint8_t* __restrict__ xs8, float* __restrict__ sx,
                            int* err) {
  pdl_enter<false>();
  const int lane = threadIdx.x & 31;
  const int64_t s = static_cast<int64_t>(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5);
  if (s >= rows || s >= offsets[E]) return;
  const int64_t t = sorted_ids[s] / k;
  if (kDebugChecks && (sorted_ids[s] < 0 || t >= Ttok)) {
    if (lane == 0) flag_error(err, kDevDebugBounds);
    return;
  }
  const uint4* src = reinterpret_cast<const uint4*>(x8 + t * H);
  uint4* dst = reinterpret_cast<uint4*>(xs8 + s * H);
  for (int c = lane; c < H / 16; c += 32) dst[c] = __ldg(src + c);
  if (lane == 0) sx[s] = sxt[t];
}

}  // namespace

cudaError_t launch_pack_w8a8(const void* w, int64_t E, int K, int M, uint8_t* codes, float* scale,
                             cudaStream_t stream) {
  if (E == 0 || K == 0 || M == 0) return cudaSuccess;
  if (K % kPackTile != 0 || M % kPackTile != 0) return cudaErrorInvalidValue;
  const dim3 g1(static_cast<unsigned>((M + kThreads - 1) / kThreads), static_cast<unsigned>(E));
  cudaError_t e = launch_kernel(fp8_scale_kernel, g1, dim3(kThreads), 0, stream, 1,
                                static_cast<const __nv_bfloat16*>(w), K, M, scale);
  if (e != cudaSuccess) return e;
  const dim3 g2(static_cast<unsigned>(M / kPackTile), static_cast<unsigned>(K / kPackTile),
                static_cast<unsigned>(E));
  return launch_kernel(pack_w8a8_kernel, g2, dim3(kThreads), 0, stream, 1,
                       static_cast<const __nv_bfloat16*>(w), scale, K, M, codes);
}

cudaError_t launch_quantize_rows(const void* a, int64_t N, const int32_t* n_dev, int K,
                                 uint8_t* codes, float* scale, cudaStream_t stream) {
  if (N == 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>((N + kThreads / 32 - 1) / (kThreads / 32));
  return launch_kernel(quant_rows_kernel, dim3(grid), dim3(kThreads), 0, stream, 1,
                       static_cast<const __nv_bfloat16*>(a), N, n_dev, K, codes, scale);
}

cudaError_t launch_dispatch_rows_q8(const uint8_t* x8, const float* sxt, const int32_t* sorted_ids,
                                    const int32_t* offsets, int E, int k, int H, int64_t rows,
                                    int64_t T, uint8_t* xs8, float* sx, int* err,
                                    cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>((rows + kThreads / 32 - 1) / (kThreads / 32));
  return launch_kernel(dispatch_rows_q8_kernel, dim3(grid), dim3(kThreads), 0, stream, 1, x8, sxt,
                       sorted_ids, offsets, E, k, H, rows, T, xs8, sx, err);
}

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
