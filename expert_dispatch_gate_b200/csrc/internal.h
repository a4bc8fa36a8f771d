// internal.h — launchers shared between the C-ABI layer (moe_api.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <string>

namespace moe {

// ---- route.cu
// Fused gate GEMM (CUDA cores) + top-k + renormalise, one warp per token; E <= 64.
cudaError_t launch_route_simt(int dtype, const void* x, const void* w_router, const float* bias,
                              int64_t T, int H, int E, int k, float* logits_out, int32_t* topk_idx,
                              float* topk_w, cudaStream_t stream);
// Top-k + renormalise, one warp per token, E <= 256: logits[t,e] = sum over ks of
// partials[ks * split_stride + t*E + e] (ascending ks) + bias[e] (bias optional); the logits
// are written to logits_out when it is non-null.
// With n_group > 1 the selection is group-limited (n_group <= 32 groups, topk_group kept).
cudaError_t launch_topk(const float* partials, int ksplit, int64_t split_stride,
                        const float* bias, float* logits_out, int64_t T, int E, int k,
                        int n_group, int topk_group, int32_t* topk_idx, float* topk_w,
                        cudaStream_t stream);

// ---- route_tc.cu (tcgen05 / TMEM / TMA, bf16)
// Gate logits on the tensor cores (tokens on the MMA's M side, experts on N, E in [16, 256],
// E % 8 == 0), K split into `ksplit` ranges:
// partials[ks][t][e] = sum over h in range ks of x[t,h] * w_router[h,e].
int route_ksplit(int64_t T, int H, int E);
cudaError_t launch_route_gemm_tc(const void* x, const void* w_router, int T, int H, int E,
                                 float* partials, int ksplit, int* err, int num_sms,
                                 cudaStream_t stream, std::string* detail);
// Gate GEMM + plain top-k in one persistent kernel (E = 64, one K range, n_group = 1, k <= 16):
// the same logits, picks and weights as launch_route_gemm_tc followed by launch_topk.
bool route_fuses_topk(int64_t T, int H, int E, int k, int n_group);
cudaError_t launch_route_gemm_topk_tc(const void* x, const void* w_router, int T, int H, int E,
                                      int k, const float* bias, float* logits_out,
                                      int32_t* topk_idx, float* topk_w, int* err, int num_sms,
                                      cudaStream_t stream, std::string* detail);

// ---- ffn_tc.cu (tcgen05 / TMEM / TMA, bf16)
// Expert GEMM1: h[s, :] = silu(x[t] Wg[e]) * (x[t] Wu[e]) for kept slots; h rows = hbuf_rows.
// With xs != nullptr the token rows come from the expert-major copy xs (contiguous per expert,
// streamed by TMA, CTA pairs); otherwise they are gathered from x through
// sorted_ids by cp.async (single CTAs).
bool gemm1_uses_row_copy(int I);
cudaError_t launch_gemm1_tc(const void* x, int T, const void* xs, const int32_t* sorted_ids,
                            const int32_t* offsets, const int32_t* blk_prefix, const void* w_gate,
                            const void* w_up, void* hbuf, int64_t hbuf_rows, int H, int E, int k,
                            int I, int TB, int64_t ub_blocks, int* err, int num_sms,
                            cudaStream_t stream, std::string* detail);
// Expert GEMM2: y[s, :] = h[s] Wd[e].
cudaError_t launch_gemm2_tc(const void* hbuf, int64_t hbuf_rows, const int32_t* offsets,
                            const int32_t* blk_prefix, const void* w_down, void* y, int H, int E,
                            int I, int TB, int64_t ub_blocks, int* err, int num_sms,
                            cudaStream_t stream, std::string* detail);

// FP8 weights and activations (W8A8): GEMM1 from expert-major e4m3 rows xs8 [rows][H] with row
// scales sx, K-major weight codes [E][I][H] and channel scales [E][I]; h written as bf16.
// GEMM2 from e4m3 rows h8 [rows][I] with row scales sh, K-major codes [E][H][I], scales [E][H].
cudaError_t launch_gemm1_f8(const void* xs8, const float* sx, const int32_t* offsets,
                            const int32_t* blk_prefix, const uint8_t* qk_gate,
                            const uint8_t* qk_up, const float* s_gate, const float* s_up,
                            void* hbuf, int64_t hbuf_rows, int H, int E, int I, int TB,
                            int64_t ub_blocks, int* err, int num_sms, cudaStream_t stream,
                            std::string* detail);
cudaError_t launch_gemm2_f8(const void* h8, const float* sh, int64_t hbuf_rows,
                            const int32_t* offsets, const int32_t* blk_prefix,
                            const uint8_t* qk_down, const float* s_down, void* y, int H, int E,
                            int I, int TB, int64_t ub_blocks, int* err, int num_sms,
                            cudaStream_t stream, std::string* detail);

// ---- ffn_simt.cu (float32 CUDA-core path)
cudaError_t launch_gemm1_simt(const float* x, const int32_t* sorted_ids, const int32_t* offsets,
                              const float* w_gate, const float* w_up, float* hbuf, int64_t A,
                              int H, int E, int k, int I, cudaStream_t stream);
cudaError_t launch_gemm2_simt(const float* hbuf, const int32_t* offsets, const float* w_down,
                              float* y, int64_t A, int H, int E, int I, cudaStream_t stream);

// ---- align.cu
// Grouping: one launch does everything up to kAlignCluster assignments (one 256-thread block up
// to kAlignSingle, one cluster of 8 CTAs of 1024 threads above); beyond that one cooperative
// launch of min(chunks, SMs) CTAs with a grid barrier, or, when those CTAs cannot all be
// resident, three kernels (histogram / scan / scatter) whose blocks take align_chunk(A)
// assignments each (a multiple of 256 between kAlignChunkMin and kAlignChunkMax, aiming at
// about 128 blocks). Measured on B200, the cluster's time grows by about 0.11 us per 1000
// assignments on its 8 SMs, so the cluster form stops at 65536.
constexpr int kAlignSingle = 2048;
constexpr int kAlignCluster = 65536;
constexpr int kAlignChunkMin = 512;
constexpr int kAlignChunkMax = 2048;
inline int align_chunk(int64_t A) {
  int64_t c = (A + 127) / 128;
  c = (c + 255) / 256 * 256;
  if (c < kAlignChunkMin) c = kAlignChunkMin;
  if (c > kAlignChunkMax) c = kAlignChunkMax;
  return static_cast<int>(c);
}
// `err` points at the error word, the first of 64 ints (256 bytes) that start out zero:
// err[kAlignBarrierWord] and the int after it are the one-launch grid barrier's counters, which
// the grouping leaves at zero.
constexpr int kAlignBarrierWord = 32;
cudaError_t launch_align(const int32_t* topk_idx, int64_t A, int E, int C, int TB,
                         int32_t* blk_hist, int32_t* counts, int32_t* offsets,
                         int32_t* blk_prefix, int32_t* sorted_ids, int32_t* slot_of,
                         uint8_t* drop_mask, int* err, cudaStream_t stream);
// Same grouping with its scratch in a file-scope device array instead of a workspace;
// at most kNoAllocMaxAssignments assignments and 256 experts.
constexpr int64_t kNoAllocMaxAssignments = 262144;
// align_chunk(A) >= ceil(A / 128) up to 128 * kAlignChunkMax = 262144 assignments, so the
// grouping of at most kNoAllocMaxAssignments uses at most 128 chunk histograms.
constexpr int kNoAllocMaxBlocks = 128;
static_assert(kNoAllocMaxAssignments <= int64_t{kNoAllocMaxBlocks} * kAlignChunkMax,
              "the no-allocation scratch holds 128 chunk histograms");
cudaError_t launch_align_noalloc(const int32_t* topk_idx, int64_t A, int E, int C, int TB,
                                 int32_t* counts, int32_t* offsets, int32_t* sorted_ids,
                                 int32_t* slot_of, uint8_t* drop_mask, cudaStream_t stream);
// blk_prefix[e] = sum over e' < e of ceil(count[e'] / TB), count from offsets.
cudaError_t launch_plan_from_offsets(const int32_t* offsets, int E, int TB, int32_t* blk_prefix,
                                     cudaStream_t stream);

// ---- quant.cu: FP8 weights and activations (W8A8)
// Weights w [E][K][M] bf16 -> K-major e4m3 codes [E][M][K] and per-channel scales [E][M]
// (K % 64 == 0, M % 64 == 0).
cudaError_t launch_pack_w8a8(const void* w, int64_t E, int K, int M, uint8_t* codes, float* scale,
                             cudaStream_t stream);
// Per-row e4m3 codes [N][K] and scales [N] of bf16 rows a [N][K] (K % 8 == 0); rows at or past
// *n_dev (a device count, when non-null) are skipped.
cudaError_t launch_quantize_rows(const void* a, int64_t N, const int32_t* n_dev, int K,
                                 uint8_t* codes, float* scale, cudaStream_t stream);
// Expert-major copy of quantised token rows: xs8[s] = x8[sorted_ids[s] / k], sx[s] likewise, for
// the kept slots s < offsets[E] (H % 16 == 0).
cudaError_t launch_dispatch_rows_q8(const uint8_t* x8, const float* sxt, const int32_t* sorted_ids,
                                    const int32_t* offsets, int E, int k, int H, int64_t rows,
                                    int64_t T, uint8_t* xs8, float* sx, int* err,
                                    cudaStream_t stream);

// ---- probe.cu: one bounded wait that nothing satisfies (failure-detection test)
cudaError_t launch_stalled_wait(int* err, cudaStream_t stream);

// ---- ep.cu (expert parallelism over R ranks; see the entry points in moe.h)
cudaError_t launch_ep_plan(const int32_t* topk_idx, const int32_t* slot_of_local,
                           const int32_t* offsets_local, const int32_t* counts_all, int64_t A,
                           int E, int R, int rank, int C, int32_t* owner, int32_t* slot,
                           int32_t* own_offsets, int* err, int num_sms, cudaStream_t stream);
cudaError_t launch_ep_dispatch(int dtype, const void* x, const int32_t* owner, const int32_t* slot,
                               void* const* peer_xs, int64_t A, int k, int H, cudaStream_t stream);
cudaError_t launch_ep_signal(uint32_t* const* peer_flags, int R, int rank, uint32_t epoch,
                             cudaStream_t stream);
cudaError_t launch_ep_wait(const uint32_t* flags, int R, uint32_t epoch, int* err,
                           cudaStream_t stream);
cudaError_t launch_ep_combine(int dtype, const void* const* peer_y, const int32_t* owner,
                              const int32_t* slot, const float* topk_w, void* out, int64_t T,
                              int H, int k, cudaStream_t stream);

// ---- combine.cu
// Expert-major copy of the token rows: xs[s,:] = x[sorted_ids[s]/k,:] for kept slots.
// T: rows of x (debug builds check sorted_ids[s] / k < T; err receives the failure).
cudaError_t launch_dispatch_rows(int dtype, const void* x, const int32_t* sorted_ids,
                                 const int32_t* offsets, int E, int k, int H, int64_t rows,
                                 int64_t T, void* xs, int* err, cudaStream_t stream);
// err (may be null): debug builds record a slot outside the T*k rows of y_slots there.
cudaError_t launch_combine(int dtype, const void* y_slots, const int32_t* slot_of,
                           const float* topk_w, const void* shared, float shared_factor,
                           const float* out_bias, void* out, int64_t T, int H, int k, int* err,
                           cudaStream_t stream);

// ---- FP8 (e4m3) expert weights (quant.cu, ffn_tc.cu)
// codes[e][k][m] = e4m3(w / scale[e][m]), scale[e][m] = max_k |w[e][k][m]| / 448 (w bf16 [E][K][M]).
cudaError_t launch_quantize_fp8(const void* w, int64_t E, int K, int M, uint8_t* codes,
                                float* scale, int num_sms, cudaStream_t stream);
// The expert GEMMs with e4m3 weights and their per-channel scales (xs: expert-major rows).
cudaError_t launch_gemm1_w8(const void* xs, const int32_t* offsets, const int32_t* blk_prefix,
                            const uint8_t* q_gate, const uint8_t* q_up, const float* s_gate,
                            const float* s_up, void* hbuf, int64_t hbuf_rows, int H, int E,
                            int I, int TB, int64_t ub_blocks, int* err, int num_sms,
                            cudaStream_t stream, std::string* detail);
cudaError_t launch_gemm2_w8(const void* hbuf, int64_t hbuf_rows, const int32_t* offsets,
                            const int32_t* blk_prefix, const uint8_t* q_down, const float* s_down,
                            void* y, int H, int E, int I, int TB, int64_t ub_blocks, int* err,
                            int num_sms, cudaStream_t stream, std::string* detail);

}  // namespace moe
