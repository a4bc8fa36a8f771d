// route.cu — router: gate logits, top-k selection and renormalised weights.
//
// [P4] "MoE Router" (2048ai.net), section "Router 就是一个小型网络": logits = x Wr (bias-free
// Linear), softmax, top-k, divide the k selected weights by their sum.
// [P5] "大模型推理加速200%+？…", section "3.1 Moe Fuse Gate & Softmax TopK": gate + softmax + top-k
// in one kernel, a warp-level arg-max with the winner erased each round, exp evaluated only for
// the k selected logits (exp(l - m) / sum over the selection equals the renormalised softmax).
// With E >= 64 in bf16 the gate GEMM runs on the tensor cores (route_tc.cu); with the hidden
// dimension in one K range it also selects, otherwise a kernel below does: topk_kernel (one
// warp per token) for E > 64, topk_lanes_kernel (G lanes per token) for E <= 64. For smaller E
// or float32 the CUDA-core kernels further down (route_slab_kernel, route_simt_kernel) compute
// the logits and select in one pass.
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

// Partial sums in ascending K-range order. GROUP K ranges are loaded per group with no branch
// between the loads, so one group costs one memory latency: 4 for the usual split, 16 (every
// range of a short batch at once, where few warps run and registers are plentiful) when the
// K split is deeper. vec: E % VPL == 0, so a lane's run of VPL logits is one or two aligned
// vector loads (rows start on 16-byte boundaries then); otherwise a lane with experts past E
// reads only those below E.
template <int VPL, int GROUP>
__global__ void __launch_bounds__(kWarpsPerBlock * 32, GROUP == 4 ? 4 : 1)
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
  for (int ks0 = 0; ks0 < ksplit; ks0 += GROUP) {
    float p[GROUP][VPL];
#pragma unroll
    for (int j = 0; j < GROUP; ++j) {
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
    for (int j = 0; j < GROUP; ++j) {
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

// Plain top-k with G lanes per token (G = 1 ... 16), for E <= 64.
//
// Stage: the block's TPB = 256 / G tokens are a contiguous [TPB, E] slice of every K-range
// partial array; all threads sum it in ascending range order with 128-bit loads (many loads in
// flight per thread), add the bias, write the logits when asked and store them in shared
// memory (row stride E + G, so the lanes reading below hit distinct banks).
// Select: lane g of a token takes experts g, g + G, g + 2G, ... in ascending order and inserts
// each order-preserving key into a list of its KL largest (KL >= k), kept in (key descending,
// index ascending) order: an entry moves ahead of a listed one only on a strictly larger key,
// and from the place it takes the entries below shift down one place each. Then k merge
// rounds over the G lanes: a butterfly finds the largest head (ties to the lower index), and
// the lane holding it pops it. Picks therefore come out in descending key order with ties to
// the lower index: the rule of select_topk. One thread per token (G = 1) gives a warp
// instruction 32 tokens; G > 1 keeps enough threads busy when T is small.
template <int G, int KL>
__global__ void __launch_bounds__(256)
    topk_lanes_kernel(const float* __restrict__ partials, int ksplit, int64_t split_stride,
                      const float* __restrict__ bias, float* __restrict__ logits_out, int64_t T,
                      int E, int k, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w) {
  constexpr int TPB = 256 / G;
  extern __shared__ float s_log[];
  pdl_enter<false>();
  const int stride = E + G;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * TPB;
  const int nt = static_cast<int>(T - t0 < TPB ? T - t0 : static_cast<int64_t>(TPB));
  {
    const int n = nt * E;  // the slice's elements, contiguous in each partial array
    const float* base = partials + t0 * E;
    // one 16-byte group: its ksplit partials in ascending order, + bias; out to logits_out and
    // shared memory
    auto finish = [&](int i, float4 v) {
      const int tl = i / E, e = i - tl * E;
      if (bias != nullptr) {
        v.x += __ldg(bias + e);
        v.y += __ldg(bias + e + 1);
        v.z += __ldg(bias + e + 2);
        v.w += __ldg(bias + e + 3);
      }
      if (logits_out != nullptr) *reinterpret_cast<float4*>(logits_out + t0 * E + i) = v;
      float* d = s_log + tl * stride + e;
      d[0] = v.x;
      d[1] = v.y;
      d[2] = v.z;
      d[3] = v.w;
    };
    auto add4 = [](float4& a, const float4& b) {
      a.x += b.x;
      a.y += b.y;
      a.z += b.z;
      a.w += b.w;
    };
    const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
    if ((E & 3) == 0 && ksplit == 1) {
      // eight groups per thread in flight
      for (int i0 = 4 * static_cast<int>(threadIdx.x); i0 < n; i0 += 8 * 4 * 256) {
        float4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = i0 + u * 4 * 256;
          v[u] = i < n ? __ldg(reinterpret_cast<const float4*>(base + i)) : zero;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (i0 + u * 4 * 256 < n) finish(i0 + u * 4 * 256, v[u]);
      }
    } else if ((E & 3) == 0) {
      // two groups per thread, four K ranges of each loaded together
      for (int i0 = 4 * static_cast<int>(threadIdx.x); i0 < n; i0 += 2 * 4 * 256) {
        float4 v[2];
        for (int ks0 = 0; ks0 < ksplit; ks0 += 4) {
          float4 p[2][4];
#pragma unroll
          for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int i = i0 + u * 4 * 256;
              p[u][j] = (i < n && ks0 + j < ksplit)
                            ? __ldg(reinterpret_cast<const float4*>(base + (ks0 + j) * split_stride + i))
                            : zero;
            }
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            if (ks0 == 0) v[u] = p[u][0];
            else add4(v[u], p[u][0]);
#pragma unroll
            for (int j = 1; j < 4; ++j)
              if (ks0 + j < ksplit) add4(v[u], p[u][j]);
          }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u)
          if (i0 + u * 4 * 256 < n) finish(i0 + u * 4 * 256, v[u]);
      }
    } else {
#pragma unroll 4
      for (int i = static_cast<int>(threadIdx.x); i < n; i += 256) {
        float v = __ldg(base + i);
        for (int ks = 1; ks < ksplit; ++ks) v += __ldg(base + ks * split_stride + i);
        const int tl = i / E, e = i - tl * E;
        if (bias != nullptr) v += __ldg(bias + e);
        if (logits_out != nullptr) logits_out[t0 * E + i] = v;
        s_log[tl * stride + e] = v;
      }
    }
  }
  __syncthreads();
  const int g = static_cast<int>(threadIdx.x) % G;
  const int tl = static_cast<int>(threadIdx.x) / G;
  TopList<KL> L;
  L.clear();
  if (tl < nt) {
    const float* row = s_log + tl * stride;
    for (int e = g; e < E; e += G) L.insert(order_key(row[e]), e);
  }
  // k merge rounds over the token's G lanes (every lane of the warp takes part)
  uint32_t pk[KL];
  int pi[KL];
#pragma unroll
  for (int j = 0; j < KL; ++j) {
    pk[j] = 0u;
    pi[j] = 0;
    if (j < k) {
      uint32_t hk = L.key[0];
      int hi = L.idx[0];
#pragma unroll
      for (int off = 1; off < G; off <<= 1) {
        const uint32_t ok = __shfl_xor_sync(0xffffffffu, hk, off);
        const int oi = __shfl_xor_sync(0xffffffffu, hi, off);
        const bool better = ok > hk || (ok == hk && oi < hi);
        hk = better ? ok : hk;
        hi = better ? oi : hi;
      }
      pk[j] = hk;
      pi[j] = hi;
      const bool pop = L.idx[0] == hi;  // expert ids are unique: only the holder pops
#pragma unroll
      for (int q = 0; q + 1 < KL; ++q) {
        L.key[q] = pop ? L.key[q + 1] : L.key[q];
        L.idx[q] = pop ? L.idx[q + 1] : L.idx[q];
      }
      L.key[KL - 1] = pop ? 0u : L.key[KL - 1];
      L.idx[KL - 1] = pop ? 0x7fffffff : L.idx[KL - 1];
    }
  }
  if (tl >= nt) return;
  const int64_t t = t0 + tl;
  thread_write_selection<KL>(pk, pi, k, g, G, topk_idx + t * k, topk_w + t * k);
}

template <int G>
cudaError_t launch_topk_lanes(const float* partials, int ksplit, int64_t split_stride,
                              const float* bias, float* logits_out, int64_t T, int E, int k,
                              int32_t* topk_idx, float* topk_w, cudaStream_t stream) {
  auto kern = topk_lanes_kernel<G, 16>;
  if (k <= 2) kern = topk_lanes_kernel<G, 2>;
  else if (k <= 4) kern = topk_lanes_kernel<G, 4>;
  else if (k <= 6) kern = topk_lanes_kernel<G, 6>;
  else if (k <= 8) kern = topk_lanes_kernel<G, 8>;
  const size_t smem = static_cast<size_t>(256 / G) * (E + G) * sizeof(float);
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  const unsigned grid = static_cast<unsigned>((T + 256 / G - 1) / (256 / G));
  return launch_kernel(kern, dim3(grid), dim3(256), smem, stream, 1, partials, ksplit,
                       split_stride, bias, logits_out, T, E, k, topk_idx, topk_w);
}

// Lanes per token for the plain top-k with E <= 64: one, doubled while the batch leaves fewer
// than about 16 warps per SM busy and each lane would still scan at least 4 experts. 0 for
// E > 64 or k > 16: the warp-per-token topk_kernel, which measured faster for E = 256 at every
// batch size from 1 to 32768 tokens (its k warp reductions cost less than 256 / G insertions
// per lane).
int topk_lanes_for(int64_t T, int E, int k) {
  if (k > 16 || E > 64) return 0;
  int G = 1;
  while (G < 16 && (E + 2 * G - 1) / (2 * G) >= 4 && T * G < 148 * 512) G *= 2;
  return G;
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
  __device__ static void unpack(const uint4 r, float (&o)[4]) {
    o[0] = __uint_as_float(r.x); o[1] = __uint_as_float(r.y);
    o[2] = __uint_as_float(r.z); o[3] = __uint_as_float(r.w);
  }
};
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void load(const __nv_bfloat16* p, float (&o)[8]) {
    unpack(__ldg(reinterpret_cast<const uint4*>(p)), o);
  }
  __device__ static void unpack(const uint4 r, float (&o)[8]) {
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

// 16-byte global -> shared copy through L2 (cp.async.cg); bytes = 0 fills the 16 bytes with
// zeros and reads nothing.
__device__ __forceinline__ void cp16_zfill(uint32_t dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// The same gate GEMM + selection with Wr and x staged in shared memory, for rows of Wr that are
// whole 16-byte granules (E * es % 16 == 0) and H % 8 == 0. Each block runs 8 warps of TPW
// tokens and walks H in slabs of 256 rows through a ring of kSlabStages buffers filled by
// cp.async, two slabs ahead of the one in use. Lane l owns rows 8l ... 8l + 7 of every slab
// (the same rows, in the same order, as in route_simt_kernel, so the logits agree bit for
// bit): its x values of each token, and its 8 rows of Wr, which are GPL = E * es / 2
// contiguous granules stored with the granule index XORed by (l & 7) so that the lanes of a
// quarter-warp read distinct banks. One Wr read serves TPW tokens; route_simt_kernel reads Wr
// from L1 once per token, and its per-lane 16-byte loads from 32 different lines each take one
// L1 pass per lane.
constexpr int kSlabRows = 256;
constexpr int kSlabStages = 3;

template <typename Tin, int EMAX, int TPW>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    route_slab_kernel(const Tin* __restrict__ x, const Tin* __restrict__ wr,
                      const float* __restrict__ bias, int64_t T, int H, int E, int k,
                      float* __restrict__ logits_out, int32_t* __restrict__ topk_idx,
                      float* __restrict__ topk_w) {
  constexpr int VN = Vec16<Tin>::N;  // elements per 16-byte granule
  constexpr int XG = 8 / VN;         // x granules per lane and token (8 rows)
  constexpr int NT = kWarpsPerBlock * 32;
  constexpr int S = kSlabStages;
  // Wr granules a thread copies per slab: gps / NT <= PRE (gps = 256 * E * es / 16)
  constexpr int PRE = EMAX * static_cast<int>(sizeof(Tin)) / 16 > 1
                          ? EMAX * static_cast<int>(sizeof(Tin)) / 16 : 1;
  extern __shared__ uint4 s_w[];     // [S][gps] Wr ring, then the x ring [S][warps][TPW][XG][32]
  pdl_enter<false>();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gpr = E / VN;            // granules per Wr row
  const int gpl = 8 * gpr;           // granules per lane (8 rows); a multiple of 8
  const int gps = 32 * gpl;          // granules per slab
  uint4* s_x = s_w + S * gps;
  const int64_t tw = (static_cast<int64_t>(blockIdx.x) * kWarpsPerBlock + warp) * TPW;
  const int nslab = (H + kSlabRows - 1) / kSlabRows;
  const uint4* wg = reinterpret_cast<const uint4*>(wr);
  const int64_t w_gran = static_cast<int64_t>(H) * gpr;  // granules in Wr
  // the ring position of each slab granule this thread copies (the same for every slab)
  int wdst[PRE];
#pragma unroll
  for (int j = 0; j < PRE; ++j) {
    const int g = static_cast<int>(threadIdx.x) + j * NT;
    wdst[j] = g ^ ((g / gpl) & 7);
  }
  auto x_slot = [&](int b, int q, int c) {
    return s_x + ((((b * kWarpsPerBlock + warp) * TPW + q) * XG + c) * 32 + lane);
  };
  // one commit group per slab (empty past the last, so the group count stays uniform)
  auto issue = [&](int sl) {
    if (sl < nslab) {
      const int b = sl % S;
#pragma unroll
      for (int j = 0; j < PRE; ++j) {
        const int g = static_cast<int>(threadIdx.x) + j * NT;
        if (g < gps) {
          const int64_t src = static_cast<int64_t>(sl) * gps + g;
          const bool ok = src < w_gran;
          cp16_zfill(smem_u32(s_w + b * gps + wdst[j]), ok ? wg + src : wg, ok ? 16u : 0u);
        }
      }
      const int h0 = sl * kSlabRows + 8 * lane;
#pragma unroll
      for (int q = 0; q < TPW; ++q) {
        const int64_t t = tw + q;
        const bool ok = t < T && h0 < H;
#pragma unroll
        for (int c = 0; c < XG; ++c)
          cp16_zfill(smem_u32(x_slot(b, q, c)), ok ? x + t * H + h0 + c * VN : x, ok ? 16u : 0u);
      }
    }
    cp_commit();
  };
  float acc[TPW][EMAX];
#pragma unroll
  for (int q = 0; q < TPW; ++q)
#pragma unroll
    for (int e = 0; e < EMAX; ++e) acc[q][e] = 0.f;
#pragma unroll
  for (int p = 0; p < S - 1; ++p) issue(p);
  for (int sl = 0; sl < nslab; ++sl) {
    issue(sl + S - 1);
    cp_wait<S - 1>();  // this thread's copies of slab sl have landed
    __syncthreads();   // and every thread's
    const int b = sl % S;
    const int h0 = sl * kSlabRows + 8 * lane;
    if (h0 < H) {  // rows past H (last slab): nothing to add
      float xv[TPW][8];
#pragma unroll
      for (int q = 0; q < TPW; ++q)
#pragma unroll
        for (int c = 0; c < XG; ++c) {
          float v[VN];
          Vec16<Tin>::unpack(*x_slot(b, q, c), v);
#pragma unroll
          for (int i = 0; i < VN; ++i) xv[q][c * VN + i] = v[i];
        }
      // this lane's granules: lane * gpl + i with i < gpl, stored at lane * gpl + (i ^ (lane & 7))
      const uint4* sw = s_w + b * gps + lane * gpl;
      const int lx = lane & 7;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
#pragma unroll
        for (int e0 = 0; e0 < EMAX; e0 += VN) {
          if (e0 < E) {
            float wv[VN];
            Vec16<Tin>::unpack(sw[(u * gpr + e0 / VN) ^ lx], wv);
#pragma unroll
            for (int q = 0; q < TPW; ++q)
#pragma unroll
              for (int i = 0; i < VN; ++i)
                acc[q][e0 + i] = fmaf(xv[q][u], wv[i], acc[q][e0 + i]);
          }
        }
      }
    }
    __syncthreads();  // slot b is refilled by the next iteration's issue
  }
#pragma unroll
  for (int q = 0; q < TPW; ++q) {
    const int64_t t = tw + q;
#pragma unroll
    for (int e = 0; e < EMAX; ++e) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1)
        acc[q][e] += __shfl_xor_sync(0xffffffffu, acc[q][e], off);
      if (bias != nullptr && e < E) acc[q][e] += __ldg(bias + e);
    }
    if (t >= T) continue;  // uniform across the warp
    if (logits_out != nullptr) {
#pragma unroll
      for (int e = 0; e < EMAX; ++e)
        if (e < E && (e & 31) == lane) logits_out[t * E + e] = acc[q][e];
    }
    // every lane holds the same E logits: select redundantly, lane j keeps the j-th pick
    uint64_t taken = 0;
    float my_v = 0.f, top = 0.f;
    int my_i = 0;
    for (int j = 0; j < k; ++j) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int e = 0; e < EMAX; ++e) {
        if (e < E && !((taken >> e) & 1ull) && (acc[q][e] > bv || (acc[q][e] == bv && e < bi))) {
          bv = acc[q][e];
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
}

template <typename Tin, int EMAX>
cudaError_t route_simt_launch(const Tin* x, const Tin* wr, const float* bias, int64_t T, int H, int E,
                       int k, float* logits_out, int32_t* idx, float* w, cudaStream_t st) {
  const unsigned block = kWarpsPerBlock * 32;
  if ((E * sizeof(Tin)) % 16 == 0 && H % 8 == 0) {
    // Wr rows of whole granules: the shared-memory slab kernel, two tokens per warp for E <= 8
    constexpr int kTpw = EMAX <= 8 ? 2 : 1;
    // the Wr ring (stages x 256 rows x E) and the x ring (stages x 8 warps x kTpw tokens x 256)
    const size_t smem = kSlabStages * (size_t{kSlabRows} * E * sizeof(Tin) +
                                       size_t{kWarpsPerBlock} * kTpw * kSlabRows * sizeof(Tin));
    auto kern = route_slab_kernel<Tin, EMAX, kTpw>;
    if (smem > 48 * 1024) {
      const cudaError_t e = cudaFuncSetAttribute(
          kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      if (e != cudaSuccess) return e;
    }
    const unsigned g = static_cast<unsigned>((T + kWarpsPerBlock * kTpw - 1) /
                                             (kWarpsPerBlock * kTpw));
    return launch_kernel(kern, dim3(g), dim3(block), smem, st, 1, x, wr, bias, T, H, E, k,
                         logits_out, idx, w);
  }
  const unsigned grid = static_cast<unsigned>((T + kWarpsPerBlock - 1) / kWarpsPerBlock);
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
  if (n_group <= 1) {
    switch (topk_lanes_for(T, E, k)) {
      case 1: return launch_topk_lanes<1>(partials, ksplit, split_stride, bias, logits_out, T, E,
                                          k, topk_idx, topk_w, stream);
      case 2: return launch_topk_lanes<2>(partials, ksplit, split_stride, bias, logits_out, T, E,
                                          k, topk_idx, topk_w, stream);
      case 4: return launch_topk_lanes<4>(partials, ksplit, split_stride, bias, logits_out, T, E,
                                          k, topk_idx, topk_w, stream);
      case 8: return launch_topk_lanes<8>(partials, ksplit, split_stride, bias, logits_out, T, E,
                                          k, topk_idx, topk_w, stream);
      case 16: return launch_topk_lanes<16>(partials, ksplit, split_stride, bias, logits_out, T,
                                            E, k, topk_idx, topk_w, stream);
      default: break;  // warp-per-token kernel below
    }
  }
  const unsigned grid = static_cast<unsigned>((T + kWarpsPerBlock - 1) / kWarpsPerBlock);
  const unsigned block = kWarpsPerBlock * 32;
  // short batch (at most one warp per token for 1024 tokens: one block per SM suffices): every
  // K range in one batch of loads
  const bool deep = ksplit > 4 && T <= 1024;
  auto kernel = deep ? topk_kernel<8, 16> : topk_kernel<8, 4>;
  if (E <= 32) kernel = deep ? topk_kernel<1, 16> : topk_kernel<1, 4>;
  else if (E <= 64) kernel = deep ? topk_kernel<2, 16> : topk_kernel<2, 4>;
  else if (E <= 128) kernel = deep ? topk_kernel<4, 16> : topk_kernel<4, 4>;
  return launch_kernel(kernel, dim3(grid), dim3(block), 0, stream, 1, partials, ksplit,
                       split_stride, bias, logits_out, T, E, k, n_group, topk_group, topk_idx,
                       topk_w);
}

}  // namespace moe
