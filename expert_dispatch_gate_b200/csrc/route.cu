// route.cu — router: gate logits, top-k selection and renormalised weights.
//
// [P4] "MoE Router" (2048ai.net), section "Router 就是一个小型网络": logits = x Wr (bias-free
// Linear), softmax, top-k, divide the k selected weights by their sum.
// [P5] "大模型推理加速200%+？…", section "3.1 Moe Fuse Gate & Softmax TopK": gate + softmax + top-k
// in one kernel, a warp-level arg-max with the winner erased each round, exp evaluated only for
// the k selected logits (exp(l - m) / sum over the selection equals the renormalised softmax).
// With E >= 64 in bf16 the gate GEMM runs on the tensor cores (route_tc.cu) and topk_kernel
// below does the selection; the CUDA-core kernel further down fuses both for small E.
//
// Selection rule: the k largest float32 logits, ties to the lower expert index (-0 == +0);
// listed by descending logit then ascending index. Logits must be finite.
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace moe {
namespace {

constexpr int kWarpsPerBlock = 8;

// Logits distributed over lanes: lane l holds experts VPL*l ... VPL*l + VPL - 1. Each logit is
// the sum of the K-range partials in ascending order plus the optional bias. With n_group > 1
// the selection is group-limited (select.cuh).
template <int VPL>
__device__ __forceinline__ void load_run(const float* p, bool vec, bool in, float (&o)[VPL]) {
  if (!in) {
#pragma unroll
    for (int i = 0; i < VPL; ++i) o[i] = 0.f;
  } else if (VPL >= 4 && vec) {
#pragma unroll
    for (int i = 0; i < VPL; i += 4) {
      const float4 q = __ldg(reinterpret_cast<const float4*>(p + i));
      o[i] = q.x;
      o[i + 1] = q.y;
      o[i + 2] = q.z;
      o[i + 3] = q.w;
    }
  } else if (VPL == 2 && vec) {
    const float2 q = __ldg(reinterpret_cast<const float2*>(p));
    o[0] = q.x;
    o[VPL - 1] = q.y;
  } else {
#pragma unroll
    for (int i = 0; i < VPL; ++i) o[i] = __ldg(p + i);
  }
}

// Partial sums in ascending K-range order. Four K ranges are loaded per group with no branch
// between the loads, so one group costs one memory latency. vec: E % VPL == 0, so a lane's run
// of VPL logits is one or two aligned vector loads (rows start on 16-byte boundaries then);
// otherwise a lane with experts past E reads only those below E.
template <int VPL>
__global__ void __launch_bounds__(kWarpsPerBlock * 32, 4)
    topk_kernel(const float* __restrict__ partials, int ksplit, int64_t split_stride,
                const float* __restrict__ bias, float* __restrict__ logits_out, int64_t T, int E,
                int k, int n_group, int topk_group, int32_t* __restrict__ topk_idx,
                float* __restrict__ topk_w) {
  pdl_enter<false>();
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kWarpsPerBlock + (threadIdx.x >> 5);
  if (t >= T) return;
  const int e0 = VPL * lane;
  const bool vec = (E % VPL) == 0;
  const bool full = e0 + VPL <= E;  // every expert of this lane exists
  const float* row = partials + t * E + e0;
  float v[VPL];
  uint32_t taken = 0;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    v[i] = 0.f;
    if (e0 + i >= E) taken |= 1u << i;
  }
  for (int ks0 = 0; ks0 < ksplit; ks0 += 4) {
    float p[4][VPL];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const bool in = ks0 + j < ksplit;
      if (full) {
        load_run<VPL>(row + (ks0 + j) * split_stride, vec, in, p[j]);
      } else {
#pragma unroll
        for (int i = 0; i < VPL; ++i)
          p[j][i] = (in && e0 + i < E) ? __ldg(row + (ks0 + j) * split_stride + i) : 0.f;
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (ks0 + j < ksplit) {
#pragma unroll
        for (int i = 0; i < VPL; ++i) v[i] = (ks0 + j == 0) ? p[j][i] : v[i] + p[j][i];
      }
    }
  }
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = e0 + i;
    if (e < E) {
      if (bias != nullptr) v[i] += __ldg(bias + e);
      if (logits_out != nullptr) logits_out[t * E + e] = v[i];
    } else {
      v[i] = -INFINITY;
    }
  }
  if (n_group > 1) taken |= warp_group_exclude<VPL>(v, E, n_group, topk_group, lane);
  warp_select_topk<VPL>(v, taken, k, lane, topk_idx + t * k, topk_w + t * k);
}

template <typename Tin>
__device__ __forceinline__ float ld_f(const Tin* p);
template <>
__device__ __forceinline__ float ld_f<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float ld_f<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

template <typename Tin>
__device__ __forceinline__ void load8(const Tin* p, float (&o)[8]);
template <>
__device__ __forceinline__ void load8<float>(const float* p, float (&o)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
  o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
}
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&o)[8]) {
  const uint4 r = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    o[2 * i] = __uint_as_float(w[i] << 16);
    o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// 16 bytes of Tin widened to float.
template <typename Tin>
struct Vec16;
template <>
struct Vec16<float> {
  static constexpr int N = 4;
  __device__ static void load(const float* p, float (&o)[4]) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(p));
    o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
  }
};
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void load(const __nv_bfloat16* p, float (&o)[8]) {
    const uint4 r = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      o[2 * i] = __uint_as_float(w[i] << 16);
      o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};

// Gate GEMM on CUDA cores + selection, one warp per token; E <= EMAX <= 64, H % 8 == 0.
// Lane l owns x[h] for h in [8l + 256i, 8l + 256i + 8): one 128-bit x load, then the matching
// 8 rows of Wr (contiguous, 8*E values) as 128-bit loads when a row is a whole number of
// 16-byte vectors (VEC), else element by element. Every lane accumulates all E partial dot
// products; a butterfly reduction gives every lane all E logits.
template <typename Tin, int EMAX, bool VEC>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    route_simt_kernel(const Tin* __restrict__ x, const Tin* __restrict__ wr,
                      const float* __restrict__ bias, int64_t T, int H, int E, int k,
                      float* __restrict__ logits_out, int32_t* __restrict__ topk_idx,
                      float* __restrict__ topk_w) {
  pdl_enter<false>();
  constexpr int VN = Vec16<Tin>::N;
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kWarpsPerBlock + (threadIdx.x >> 5);
  if (t >= T) return;
  float acc[EMAX];
#pragma unroll
  for (int e = 0; e < EMAX; ++e) acc[e] = 0.f;
  const Tin* xr = x + t * H;
  for (int h0 = lane * 8; h0 < H; h0 += 256) {
    float xv[8];
    load8<Tin>(xr + h0, xv);
    const Tin* wb = wr + static_cast<size_t>(h0) * E;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if constexpr (VEC) {
#pragma unroll
        for (int e0 = 0; e0 < EMAX; e0 += VN) {
          if (e0 < E) {
            float wv[VN];
            Vec16<Tin>::load(wb + u * E + e0, wv);
#pragma unroll
            for (int i = 0; i < VN; ++i) acc[e0 + i] = fmaf(xv[u], wv[i], acc[e0 + i]);
          }
        }
      } else {
#pragma unroll
        for (int e = 0; e < EMAX; ++e)
          if (e < E) acc[e] = fmaf(xv[u], ld_f<Tin>(wb + u * E + e), acc[e]);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < EMAX; ++e) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
    if (bias != nullptr && e < E) acc[e] += __ldg(bias + e);
  }
  if (logits_out != nullptr) {
#pragma unroll
    for (int e = 0; e < EMAX; ++e)
      if (e < E && (e & 31) == lane) logits_out[t * E + e] = acc[e];
  }
  // Every lane holds the same E logits: select redundantly, lane j keeps the j-th pick.
  uint64_t taken = 0;
  float my_v = 0.f, top = 0.f;
  int my_i = 0;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int e = 0; e < EMAX; ++e) {
      if (e < E && !((taken >> e) & 1ull) && (acc[e] > bv || (acc[e] == bv && e < bi))) {
        bv = acc[e];
        bi = e;
      }
    }
    taken |= 1ull << (bi & 63);
    if (lane == j) {
      my_v = bv;
      my_i = bi;
    }
    if (j == 0) top = bv;
  }
  write_selection(lane, k, my_v, my_i, top, topk_idx + t * k, topk_w + t * k);
}

template <typename Tin, int EMAX>
cudaError_t route_simt_launch(const Tin* x, const Tin* wr, const float* bias, int64_t T, int H, int E,
                       int k, float* logits_out, int32_t* idx, float* w, cudaStream_t st) {
  const unsigned grid = static_cast<unsigned>((T + kWarpsPerBlock - 1) / kWarpsPerBlock);
  const unsigned block = kWarpsPerBlock * 32;
  if ((E * sizeof(Tin)) % 16 == 0)
    return launch_kernel(route_simt_kernel<Tin, EMAX, true>, dim3(grid), dim3(block), 0, st, 1, x,
                         wr, bias, T, H, E, k, logits_out, idx, w);
  return launch_kernel(route_simt_kernel<Tin, EMAX, false>, dim3(grid), dim3(block), 0, st, 1, x,
                       wr, bias, T, H, E, k, logits_out, idx, w);
}

template <typename Tin>
cudaError_t route_simt_dispatch(const Tin* x, const Tin* wr, const float* bias, int64_t T, int H,
                                int E, int k, float* logits_out, int32_t* idx, float* w,
                                cudaStream_t st) {
  if (E <= 8) return route_simt_launch<Tin, 8>(x, wr, bias, T, H, E, k, logits_out, idx, w, st);
  if (E <= 16) return route_simt_launch<Tin, 16>(x, wr, bias, T, H, E, k, logits_out, idx, w, st);
  if (E <= 32) return route_simt_launch<Tin, 32>(x, wr, bias, T, H, E, k, logits_out, idx, w, st);
  return route_simt_launch<Tin, 64>(x, wr, bias, T, H, E, k, logits_out, idx, w, st);
}

}  // namespace

cudaError_t launch_route_simt(int dtype, const void* x, const void* w_router, const float* bias,
                              int64_t T, int H, int E, int k, float* logits_out, int32_t* topk_idx,
                              float* topk_w, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  if (dtype == 0)
    return route_simt_dispatch<float>(static_cast<const float*>(x),
                                      static_cast<const float*>(w_router), bias, T, H, E, k,
                                      logits_out, topk_idx, topk_w, stream);
  return route_simt_dispatch<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(x),
                                            static_cast<const __nv_bfloat16*>(w_router), bias, T,
                                            H, E, k, logits_out, topk_idx, topk_w, stream);
}

cudaError_t launch_topk(const float* partials, int ksplit, int64_t split_stride,
                        const float* bias, float* logits_out, int64_t T, int E, int k,
                        int n_group, int topk_group, int32_t* topk_idx, float* topk_w,
                        cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>((T + kWarpsPerBlock - 1) / kWarpsPerBlock);
  const unsigned block = kWarpsPerBlock * 32;
  auto kernel = topk_kernel<8>;
  if (E <= 32) kernel = topk_kernel<1>;
  else if (E <= 64) kernel = topk_kernel<2>;
  else if (E <= 128) kernel = topk_kernel<4>;
  return launch_kernel(kernel, dim3(grid), dim3(block), 0, stream, 1, partials, ksplit,
                       split_stride, bias, logits_out, T, E, k, n_group, topk_group, topk_idx,
                       topk_w);
}

}  // namespace moe
