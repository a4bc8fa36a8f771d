// select.cuh — top-k selection and renormalised routing weights for one token per warp.
//
// [P4] "MoE Router" (2048ai.net), section "Router 就是一个小型网络": softmax over the logits, keep
// the top k, divide the k kept weights by their sum.
// [P5] "大模型推理加速200%+？…", section "3.1 Moe Fuse Gate & Softmax TopK": a warp-level arg-max
// per round with the winner erased, and exp only for the k selected logits
// (exp(l - m) / sum over the selection equals the renormalised softmax). Here each round's
// arg-max is one redux.sync max-reduction over order-preserving integer keys plus a ballot,
// instead of a shuffle tree (warp_select_topk).
//
// Selection rule: the k largest float32 logits, ties to the lower expert index (-0 == +0);
// listed by descending logit then ascending index. Logits must be finite.
#pragma once

#include <math.h>
#include <stdint.h>

namespace moe {

// Winner of (value desc, index asc) across the warp; every lane ends with the same pair.
__device__ __forceinline__ void warp_argmax(float& bv, int& bi) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
    if (ov > bv || (ov == bv && oi < bi)) {
      bv = ov;
      bi = oi;
    }
  }
}

// Lane j < k holds the j-th selected (value, index); `top` is the largest logit. Writes
// topk_idx and the weights exp(l_j - top) / sum_i exp(l_i - top).
__device__ __forceinline__ void write_selection(int lane, int k, float my_v, int my_i, float top,
                                                int32_t* idx_row, float* w_row) {
  const float ex = (lane < k) ? expf(my_v - top) : 0.0f;
  float s = ex;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane < k) {
    idx_row[lane] = my_i;
    w_row[lane] = ex / s;
  }
}

// Group-limited selection ([P5] section 3.1, "select groups first"): the E experts form
// n_group equal contiguous groups (n_group <= 32); a group's score is the float32 sum of its
// two largest logits (its only logit when a group holds one expert); the topk_group groups
// with the highest scores (ties to the lower group index) stay selectable. Lane l holds
// experts VPL*l ... VPL*l + VPL - 1 in v[]. Returns the bit mask of v[] entries of this lane to
// exclude (experts outside the kept groups).
template <int VPL>
__device__ __forceinline__ uint32_t warp_group_exclude(const float (&v)[VPL], int E, int n_group,
                                                       int topk_group, int lane) {
  const int gs = E / n_group;
  float my_score = -INFINITY;
  for (int g = 0; g < n_group; ++g) {
    // this lane's two largest members of group g, then the warp's (multiset top-2)
    float a1 = -INFINITY, a2 = -INFINITY;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int e = VPL * lane + i;
      if (e < E && e / gs == g) {
        const float x = v[i];
        if (x > a1) {
          a2 = a1;
          a1 = x;
        } else if (x > a2) {
          a2 = x;
        }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float b1 = __shfl_xor_sync(0xffffffffu, a1, off);
      const float b2 = __shfl_xor_sync(0xffffffffu, a2, off);
      if (b1 > a1) {
        a2 = fmaxf(a1, b2);
        a1 = b1;
      } else {
        a2 = fmaxf(a2, b1);
      }
    }
    if (lane == g) my_score = (gs == 1) ? a1 : a1 + a2;
  }
  uint32_t keep = 0;
  bool mine_taken = false;
  for (int j = 0; j < topk_group; ++j) {
    float bv = (lane < n_group && !mine_taken) ? my_score : -INFINITY;
    int bi = (lane < n_group && !mine_taken) ? lane : 0x7fffffff;
    warp_argmax(bv, bi);
    keep |= 1u << (bi & 31);
    if (lane == bi) mine_taken = true;
  }
  uint32_t excl = 0;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = VPL * lane + i;
    if (e < E && !((keep >> (e / gs)) & 1u)) excl |= 1u << i;
  }
  return excl;
}

// Order-preserving 32-bit key of a finite float: key(a) < key(b) iff a < b, with -0 mapped to
// +0 so that the two zeros rank equal. key 0 belongs to no finite float.
__device__ __forceinline__ uint32_t order_key(float v) {
  uint32_t u = __float_as_uint(v);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// A thread's list of its KL largest candidates in (key descending, index ascending) order.
// Candidates must arrive in ascending index order: an entry moves ahead of a listed one only on
// a strictly larger key, and from the place it takes the entries below shift down one place
// each, so equal keys keep the lower index first. Key 0 (no finite float) marks an empty place.
template <int KL>
struct TopList {
  uint32_t key[KL];
  int idx[KL];
  __device__ __forceinline__ void clear() {
#pragma unroll
    for (int j = 0; j < KL; ++j) {
      key[j] = 0u;
      idx[j] = 0x7fffffff;
    }
  }
  __device__ __forceinline__ void insert(uint32_t ck, int ci) {
    bool shift = false;
#pragma unroll
    for (int q = 0; q < KL; ++q) {
      const bool gt = shift || ck > key[q];
      shift = gt;
      const uint32_t hk = gt ? ck : key[q];
      const int hi = gt ? ci : idx[q];
      ck = gt ? key[q] : ck;
      ci = gt ? idx[q] : ci;
      key[q] = hk;
      idx[q] = hi;
    }
  }
};

// Renormalised weights of k picks held by one thread (keys pk, indices pi; k <= KL):
// w_j = exp(l_j - l_0) / sum_i exp(l_i - l_0), the sum taken in the pairwise order of
// write_selection's butterfly (halving strides; adding the zeros of unused places is exact), so
// the weights equal the warp kernels' bit for bit. Writes the picks j with j % stride == first.
template <int KL>
__device__ __forceinline__ void thread_write_selection(const uint32_t (&pk)[KL],
                                                       const int (&pi)[KL], int k, int first,
                                                       int stride, int32_t* idx_row,
                                                       float* w_row) {
  constexpr int PW = KL <= 2 ? 2 : KL <= 4 ? 4 : KL <= 8 ? 8 : 16;
  const float top = key_value(pk[0]);
  float ex[KL], acc[PW];
#pragma unroll
  for (int j = 0; j < PW; ++j) acc[j] = 0.f;
#pragma unroll
  for (int j = 0; j < KL; ++j) {
    ex[j] = (j < k) ? expf(key_value(pk[j]) - top) : 0.f;
    acc[j] = ex[j];
  }
#pragma unroll
  for (int off = PW / 2; off > 0; off >>= 1) {
#pragma unroll
    for (int j = 0; j < off; ++j) acc[j] += acc[j + off];
  }
#pragma unroll
  for (int j = 0; j < KL; ++j) {
    if (j < k && j % stride == first) {
      idx_row[j] = pi[j];
      w_row[j] = ex[j] / acc[0];
    }
  }
}

// This lane's two best entries not yet taken, in (key descending, index ascending) order:
// entries are scanned in ascending index order and only a strictly larger key displaces one.
// Lane l holds experts VPL*l + i. Key 0 (no finite float) marks "none".
template <int VPL>
__device__ __forceinline__ void lane_best2(const uint32_t (&key)[VPL], uint32_t taken, int lane,
                                           uint32_t& bk, int& bi, uint32_t& sk, int& si) {
  bk = 0u;
  bi = 0x7fffffff;
  sk = 0u;
  si = 0x7fffffff;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    if (!((taken >> i) & 1u)) {
      const uint32_t kk = key[i];
      if (kk > bk) {
        sk = bk;
        si = bi;
        bk = kk;
        bi = VPL * lane + i;
      } else if (kk > sk) {
        sk = kk;
        si = VPL * lane + i;
      }
    }
  }
}

// One token's logits spread over the warp: lane l holds experts VPL*l ... VPL*l + VPL - 1 in
// v[]; bit i of `taken` marks v[i] as absent (expert id >= E, or excluded). Selects the top k
// and writes idx_row[0..k) and w_row[0..k). Each round takes the warp's largest key with one
// max-reduction (redux.sync). Lanes hold disjoint ascending index ranges, so among the lanes
// holding that key the lowest lane has the lowest expert index (ballot + find-first); one
// shuffle broadcasts it. Each lane keeps its two best remaining entries: the winning lane
// promotes its second, and rescans only when it wins while holding no second (its second
// was promoted on an earlier win), which with k picks spread over 32 lanes is rare.
template <int VPL>
__device__ __forceinline__ void warp_select_topk(const float (&v)[VPL], uint32_t taken, int k,
                                                 int lane, int32_t* idx_row, float* w_row) {
  uint32_t key[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) key[i] = order_key(v[i]);
  uint32_t bk, sk;
  int bi, si;
  lane_best2<VPL>(key, taken, lane, bk, bi, sk, si);
  float my_v = 0.f, top = 0.f;
  int my_i = 0;
  for (int j = 0; j < k; ++j) {
    const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
    const int wl = __ffs(__ballot_sync(0xffffffffu, bk == m)) - 1;
    const int win = __shfl_sync(0xffffffffu, bi, wl);
    const float val = key_value(m);
    if (lane == j) {
      my_v = val;
      my_i = win;
    }
    if (j == 0) top = val;
    if (lane == wl) {
      taken |= 1u << (win - VPL * lane);
      if (sk != 0u) {
        bk = sk;
        bi = si;
        sk = 0u;
        si = 0x7fffffff;
      } else {
        lane_best2<VPL>(key, taken, lane, bk, bi, sk, si);
      }
    }
  }
  write_selection(lane, k, my_v, my_i, top, idx_row, w_row);
}

}  // namespace moe
