// select.cuh — top-k selection and renormalised routing weights for one token per warp.
//
// [P4] "MoE Router" (2048ai.net), section "Router 就是一个小型网络": softmax over the logits, keep
// the top k, divide the k kept weights by their sum.
// [P5] "大模型推理加速200%+？…", section "3.1 Moe Fuse Gate & Softmax TopK": warp-shuffle arg-max
// with the winner erased each round; exp only for the k selected logits
// (exp(l - m) / sum over the selection equals the renormalised softmax).
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
// with the highest scores (ties to the lower group index) stay selectable. Returns the bit
// mask of v[] entries of this lane to exclude (experts outside the kept groups).
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
      const int e = lane + 32 * i;
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
    const int e = lane + 32 * i;
    if (e < E && !((keep >> (e / gs)) & 1u)) excl |= 1u << i;
  }
  return excl;
}

// One token's logits spread over the warp: lane holds experts lane, lane + 32, ... in v[]
// (VPL per lane); bit i of `taken` marks v[i] as absent (expert id >= E). Selects the top k
// and writes idx_row[0..k) and w_row[0..k).
template <int VPL>
__device__ __forceinline__ void warp_select_topk(const float (&v)[VPL], uint32_t taken, int k,
                                                 int lane, int32_t* idx_row, float* w_row) {
  float my_v = 0.f, top = 0.f;
  int my_i = 0;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int e = lane + 32 * i;
      if (!((taken >> i) & 1u) && (v[i] > bv || (v[i] == bv && e < bi))) {
        bv = v[i];
        bi = e;
      }
    }
    warp_argmax(bv, bi);
    if ((bi & 31) == lane) taken |= 1u << ((bi >> 5) & 31);
    if (lane == j) {
      my_v = bv;
      my_i = bi;
    }
    if (j == 0) top = bv;
  }
  write_selection(lane, k, my_v, my_i, top, idx_row, w_row);
}

}  // namespace moe
