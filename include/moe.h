/*
 * moe.h — C ABI of libmoe.so: the MoE layer forward hot path on one NVIDIA B200 (sm_100a).
 *
 * The layer (router gate -> softmax/top-k/renormalise -> capacity-limited grouping by expert
 * -> grouped SwiGLU expert FFN -> weighted combine) follows these pages:
 *   [P1] "MoE 模型的 FlashAttention 跟普通模型有什么不一样？" (framerc.cn):
 *        section "FlashAttention 在 MoE 模型里的位置" (the five steps), section
 *        "融合二：expert 计算的输出 + 合并结果" (accum += route_weight * expert_output),
 *        section "手动编译 MoE 融合算子" (npu_moe_fusion(x, router_weight[H,E],
 *        expert_weights[E,...], num_experts, top_k, activation="silu")).
 *   [P4] "MoE Router" on Ascend CANN (2048ai.net): section "Router 就是一个小型网络" (gate
 *        Linear(H,E,bias=False), softmax, topk, renormalise), section "Token 分发的通信瓶颈"
 *        (per-destination counts), section "昇腾NPU的通信计算重叠" (capacity C = total/E x 1.25,
 *        overflow dropped to the residual path).
 *   [P5] "大模型推理加速200%+？这套国产融合算子库把CUDA/Triton全替换了" (csdn.net): sections
 *        "3.1 Moe Fuse Gate & Softmax TopK" and "3.2 Fuse RMS RoPE & MoE Align & MoE Sum".
 *
 * Conventions (all entry points):
 *   - Notation: T tokens, H hidden size, E experts, k experts per token, I SwiGLU intermediate
 *     size, C per-expert capacity (moe_capacity), A = T*k assignments; assignment a = t*k + j.
 *   - Pointers named x, w_*, out, y_slots, logits*, topk_*, counts, offsets, sorted_ids,
 *     slot_of, drop_mask and ws are DEVICE pointers owned by the caller; the library never
 *     allocates, frees or synchronises (except moe_check_error). Every device pointer must be
 *     16-byte aligned; tensors are dense row-major with the shapes given below.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream). All calls are
 *     asynchronous on that stream; outputs are valid once the stream reaches them.
 *   - Arguments are validated on the host before any launch; an invalid call returns an error
 *     status and launches nothing. A failed launch returns MOE_ERR_CUDA. Device-side faults
 *     that the kernels detect (an expert id out of range, a bounded wait that ran out) are
 *     recorded in the first word of `ws` and reported by moe_check_error.
 *   - The first 256 bytes of `ws` are the library's control block (the error word, and the
 *     counters of the grid barrier the one-launch grouping uses above 65536 assignments). They
 *     must be zero before the first call on a workspace; the library leaves them zero, and
 *     moe_check_error clears all of them when it reports a device error.
 *   - Float dtype: MOE_F32 or MOE_BF16 for x, the weights, y_slots and out. Gate logits,
 *     routing weights and the logit bias are always float32.
 *   - Weight layout (x @ W convention): w_router [H,E]; w_gate, w_up [E,H,I]; w_down [E,I,H]
 *     (one tensor per kind with a leading expert dimension, [P1] "手动编译 MoE 融合算子").
 *   - Outputs are the MoE contribution only; the residual add belongs to the caller.
 *   - Limits: 1 <= E <= 256, 1 <= k <= min(E,16), 0 <= T < 2^24, H % 8 == 0, I >= 1.
 *     BF16: H % 64 == 0 and I % 64 == 0 (tensor-core expert GEMMs); E <= 64 or E % 8 == 0.
 *     F32: E <= 64.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* null pointer, bad size, misaligned pointer, k > E ... */
  MOE_ERR_UNSUPPORTED = 2, /* valid layer, but outside the limits listed above */
  MOE_ERR_WORKSPACE = 3,   /* ws missing or ws_bytes below the required size */
  MOE_ERR_CUDA = 4,        /* a CUDA runtime call or kernel launch failed */
  MOE_ERR_DEVICE = 5       /* a kernel reported a fault through the workspace error word */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

typedef struct {
  int64_t T;             /* tokens (rows of x); 0 is valid and launches nothing */
  int32_t H;             /* hidden size */
  int32_t E;             /* number of experts */
  int32_t k;             /* experts per token */
  int32_t I;             /* SwiGLU intermediate size per expert */
  float capacity_factor; /* C = ceil(cf*T*k/E) capped at T; cf <= 0 means no limit (C = T) */
  int32_t dtype;         /* moe_dtype */
} moe_shape;

/* Workspace bytes that moe_layer_forward needs for `shape`; it also covers every other call
 * on the same shape. 0 if the shape is invalid. */
size_t moe_workspace_bytes(const moe_shape* shape);

/* Per-expert capacity C, [P4] section "昇腾NPU的通信计算重叠", reading "total tokens" as the
 * T*k assignments: C = ceil(cf*T*k/E) in exact integer arithmetic on the float32 cf, capped at
 * T; cf <= 0 gives T. Returns -1 for an invalid shape. */
int32_t moe_capacity(const moe_shape* shape);

/* Router, [P4] section "Router 就是一个小型网络" and [P5] section "3.1 Moe Fuse Gate &
 * Softmax TopK": logits[t,e] = sum_h x[t,h]*w_router[h,e] (+ logit_bias[e]) accumulated in
 * float32; topk_idx[t,:] = the k largest logits in (logit desc, index asc) order, ties to the
 * lower index; topk_w[t,j] = exp(l_j - m) / sum over the selected i of exp(l_i - m), m = row
 * max (the renormalised softmax over the selected experts).
 *   x [T,H] dtype; w_router [H,E] dtype; logit_bias [E] float32 or NULL;
 *   logits_out [T,E] float32 or NULL (when given, receives the logits the selection used);
 *   topk_idx [T,k] int32; topk_w [T,k] float32; ws/ws_bytes: workspace (moe_workspace_bytes). */
moe_status moe_route(const moe_shape* shape, const void* x, const void* w_router,
                     const float* logit_bias, float* logits_out, int32_t* topk_idx,
                     float* topk_w, void* ws, size_t ws_bytes, void* stream);

/* Selection only, from given float32 logits [T,E] (same rule as moe_route). No workspace.
 * Logits must be finite. */
moe_status moe_route_from_logits(const moe_shape* shape, const float* logits,
                                 int32_t* topk_idx, float* topk_w, void* stream);

/* Capacity-limited grouping, [P1] section "FlashAttention 在 MoE 模型里的位置" step 3, [P4]
 * sections "Token 分发的通信瓶颈" and "昇腾NPU的通信计算重叠", [P5] "MoE Align". The rank of
 * assignment a = t*k+j within expert e = idx[t,j] counts earlier tokens routed to e; a is kept
 * iff rank < C. counts[e] = min(#assignments to e, C); offsets = exclusive scan of counts
 * (offsets[E] = kept total); slot = offsets[e] + rank; sorted_ids[slot] = a (slots past the
 * kept total hold -1); slot_of[a] = slot or -1; drop_mask[a] = 1 iff dropped.
 *   topk_idx [T,k] int32 (distinct experts per token; an id outside [0,E) is treated as
 *   dropped and flagged in the error word); counts [E], offsets [E+1], sorted_ids [T*k],
 *   slot_of [T*k] int32; drop_mask [T*k] uint8. */
moe_status moe_align(const moe_shape* shape, const int32_t* topk_idx, int32_t* counts,
                     int32_t* offsets, int32_t* sorted_ids, int32_t* slot_of,
                     uint8_t* drop_mask, void* ws, size_t ws_bytes, void* stream);

/* moe_align without a workspace, for callers that cannot allocate device memory: code that
 * runs inside another framework's memory planner, which hands out only the tensors it owns,
 * or on a latency-critical path where a cudaMalloc could stall the device or fail under memory
 * pressure. The pages have no counterpart to this call: it is a deployment variant of
 * moe_align with identical arguments and results, minus ws/ws_bytes.
 *   Its scratch (per-chunk histograms, the token-block plan, an error word; about 130 KB) is
 *   a file-scope __device__ array inside libmoe.so that every device loading the library keeps
 *   until the process exits. The first call on a device looks up that array's device address
 *   (cudaGetSymbolAddress) with the device current, and looks it up again when the device's
 *   context has changed (after cudaDeviceReset); make the first call after any such change
 *   before any stream capture. The call itself allocates nothing: no cudaMalloc, cudaFree or allocating library
 *   routine.
 *   Limits: T*k <= 262144 assignments and E <= 256; larger batches return MOE_ERR_UNSUPPORTED
 *   (use moe_align with a workspace). All calls share the one scratch array, which keeps the
 *   last call's contents: calls that overlap on the GPU (other streams or host threads) race on
 *   it and must be serialised by the caller. Expert ids outside [0,E) are treated as dropped;
 *   this call does not report them (moe_check_error reads a workspace, which it has none of). */
moe_status moe_align_noalloc(const moe_shape* shape, const int32_t* topk_idx, int32_t* counts,
                             int32_t* offsets, int32_t* sorted_ids, int32_t* slot_of,
                             uint8_t* drop_mask, void* stream);

/* Grouped SwiGLU expert FFN, [P1] section "FlashAttention 在 MoE 模型里的位置" step 4 and
 * section "手动编译 MoE 融合算子" (activation "silu"): for every kept slot s of expert e (offsets[e]
 * <= s < offsets[e+1]) with token t = sorted_ids[s] / k:
 *   y_slots[s,:] = (silu(x[t] @ w_gate[e]) * (x[t] @ w_up[e])) @ w_down[e], silu(z) = z*sigmoid(z),
 * float32 accumulation; BF16 rounds the intermediate and y to bf16. Rows of y_slots past
 * offsets[E] are not written.
 *   x [T,H]; sorted_ids [T*k], offsets [E+1] as produced by moe_align; w_gate, w_up [E,H,I];
 *   w_down [E,I,H]; y_slots [T*k,H] dtype. */
moe_status moe_grouped_ffn(const moe_shape* shape, const void* x, const int32_t* sorted_ids,
                           const int32_t* offsets, const void* w_gate, const void* w_up,
                           const void* w_down, void* y_slots, void* ws, size_t ws_bytes,
                           void* stream);

/* Weighted combine, [P1] section "融合二：expert 计算的输出 + 合并结果" and [P5] "MoE Sum":
 * out[t,:] = sum over j with slot_of[t*k+j] >= 0 of topk_w[t,j] * y_slots[slot_of[t*k+j],:],
 * accumulated in float32 and rounded once; a fully dropped token gives a zero row.
 *   y_slots [T*k,H] dtype; slot_of [T*k] int32; topk_w [T,k] float32; out [T,H] dtype. */
moe_status moe_combine(const moe_shape* shape, const void* y_slots, const int32_t* slot_of,
                       const float* topk_w, void* out, void* stream);

/* The whole layer on one stream: moe_route -> moe_align -> moe_grouped_ffn -> moe_combine,
 * with the intermediates (logits unless logits_out is given, offsets, sorted_ids, slot_of, the
 * SwiGLU intermediate, y_slots) in the workspace. Outputs: out [T,H] dtype, topk_idx [T,k],
 * topk_w [T,k], counts [E], drop_mask [T*k]; logits_out [T,E] float32 or NULL. No host
 * synchronisation: launch grids come from upper bounds and kernels read counts on the device. */
moe_status moe_layer_forward(const moe_shape* shape, const void* x, const void* w_router,
                             const float* logit_bias, const void* w_gate, const void* w_up,
                             const void* w_down, void* out, float* logits_out,
                             int32_t* topk_idx, float* topk_w, int32_t* counts,
                             uint8_t* drop_mask, void* ws, size_t ws_bytes, void* stream);

/* ---- Extensions of the routing and the combine.
 *
 * Group-limited routing, [P5] "大模型推理加速200%+？…", section "3.1 Moe Fuse Gate & Softmax
 * TopK" (the gate selects expert groups first and keeps each group's top-1/top-2; the page
 * gives no formula, this is the reading taken): the E experts form n_group equal contiguous
 * groups; a group's score is the float32 sum of its two largest logits (its only logit when a
 * group holds one expert); the topk_group best groups are kept (ties to the lower group
 * index); the k largest logits among their experts are selected with the plain rule; weights
 * are renormalised over the k as in moe_route.
 *
 * Shared expert and bias in the combine, [P5] section "3.2 Fuse RMS RoPE & MoE Align & MoE
 * Sum" (the MoE sum fuses the shared expert's factor and a bias add):
 *   out[t,:] = sum_j w[t,j] y[slot,:] + shared_factor * shared_out[t,:] + out_bias[:]
 * accumulated in float32 in that order and rounded once; shared_out is the shared expert's
 * output computed by the caller, [T,H] in the layer dtype, 16-byte aligned. Both terms apply
 * to every token, a fully dropped one included. */
typedef struct {
  int32_t n_group;        /* >= 1, divides E, <= 32; 1 = plain top-k */
  int32_t topk_group;     /* groups kept per token, 1..n_group; k <= topk_group * E / n_group */
  const void* shared_out; /* [T,H] (dtype of the layer) or NULL */
  float shared_factor;    /* multiplies shared_out */
  const float* out_bias;  /* [H] float32 or NULL */
} moe_layer_opts;

/* moe_route / moe_route_from_logits / moe_combine / moe_layer_forward with `opts` (NULL or all
 * defaults: identical to the plain call). Invalid options return MOE_ERR_INVALID_ARG before any
 * launch. */
moe_status moe_route_ex(const moe_shape* shape, const moe_layer_opts* opts, const void* x,
                        const void* w_router, const float* logit_bias, float* logits_out,
                        int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes,
                        void* stream);
moe_status moe_route_from_logits_ex(const moe_shape* shape, const moe_layer_opts* opts,
                                    const float* logits, int32_t* topk_idx, float* topk_w,
                                    void* stream);
moe_status moe_combine_ex(const moe_shape* shape, const moe_layer_opts* opts,
                          const void* y_slots, const int32_t* slot_of, const float* topk_w,
                          void* out, void* stream);
moe_status moe_layer_forward_ex(const moe_shape* shape, const moe_layer_opts* opts,
                                const void* x, const void* w_router, const float* logit_bias,
                                const void* w_gate, const void* w_up, const void* w_down,
                                void* out, float* logits_out, int32_t* topk_idx, float* topk_w,
                                int32_t* counts, uint8_t* drop_mask, void* ws, size_t ws_bytes,
                                void* stream);

/* ---- FP8 (e4m3) expert weights, weight-only (W8A16).
 *
 * [P5] section "4.3 MOE量化方案矩阵" lists W16A16, W8A8 (INT8/FP8), W4A8 and W4A16 expert GEMMs
 * with offline weight repacking, without a numeric scheme. The reading taken: the FP8 weights
 * of W8A8 with the 16-bit activations of W4A16. For one weight tensor w [E][K][M] (K the
 * reduction dimension, M the output channels: K = H, M = I for gate/up; K = I, M = H for down)
 *   scale[e][m] = max_k |w[e][k][m]| / 448 (1 for an all-zero column), float32
 *   codes[e][k][m] = e4m3(w[e][k][m] / scale[e][m]): OCP FP8 E4M3 (bias 7, subnormals, 448 the
 *                    largest finite value), nearest-even, saturating
 * The expert GEMMs apply decode(codes) * scale: every e4m3 value is exactly a bf16 value, so
 * the tensor cores see decode(codes) exactly and the scale multiplies the float32 accumulator.
 * Halves the expert-weight bytes the layer streams. */

/* Quantises bf16 weights w [E][K][M] (M even) into codes [E][K][M] (uint8, 16-byte aligned)
 * and scale [E][M] (float32). Asynchronous on `stream`. */
moe_status moe_quantize_weights_fp8(const void* w, int64_t E, int64_t K, int64_t M,
                                    uint8_t* codes, float* scale, void* stream);

/* moe_grouped_ffn / moe_layer_forward_ex with e4m3 expert weights (bf16 shapes only):
 * q_gate, q_up [E][H][I] and s_gate, s_up [E][I]; q_down [E][I][H] and s_down [E][H]. */
moe_status moe_grouped_ffn_w8(const moe_shape* shape, const void* x, const int32_t* sorted_ids,
                              const int32_t* offsets, const uint8_t* q_gate, const uint8_t* q_up,
                              const uint8_t* q_down, const float* s_gate, const float* s_up,
                              const float* s_down, void* y_slots, void* ws, size_t ws_bytes,
                              void* stream);
moe_status moe_layer_forward_w8(const moe_shape* shape, const moe_layer_opts* opts,
                                const void* x, const void* w_router, const float* logit_bias,
                                const uint8_t* q_gate, const uint8_t* q_up, const uint8_t* q_down,
                                const float* s_gate, const float* s_up, const float* s_down,
                                void* out, float* logits_out, int32_t* topk_idx, float* topk_w,
                                int32_t* counts, uint8_t* drop_mask, void* ws, size_t ws_bytes,
                                void* stream);

/* ---- FP8 weights and activations (W8A8).
 *
 * [P5] section "4.3 MOE量化方案矩阵": W8A8 with FP8, and offline weight repacking. The reading
 * taken: the weights as in W8A16 (e4m3, one float32 scale per output channel), repacked with the
 * reduction dimension contiguous; the activations entering each expert GEMM quantised per row to
 * e4m3 with the same rule (one float32 scale per token row of x and per slot row of the SwiGLU
 * intermediate h, which is rounded to bf16 first). Both GEMMs then run as e4m3 x e4m3 products on
 * the tensor cores, and the fp32 accumulator is multiplied by the channel scale and the row scale:
 *   y[s,m] = s_act[s] * s_w[e][m] * sum_k decode(q_act[s][k]) * decode(q_w[e][m][k]).
 * Halves the expert-weight bytes the layer streams and the activation bytes the GEMMs read. */

/* Repacks bf16 weights w [E][K][M] (K the reduction dimension; K, M multiples of 64) into K-major
 * e4m3 codes [E][M][K] (uint8, 16-byte aligned) and per-channel scales [E][M] (float32), with the
 * rule of moe_quantize_weights_fp8 (the same codes, transposed). */
moe_status moe_pack_weights_w8a8(const void* w, int64_t E, int64_t K, int64_t M, uint8_t* codes,
                                 float* scale, void* stream);

/* Per-row e4m3 quantisation of bf16 rows a [N][K] (K a multiple of 8): scale[n] = max_k
 * |a[n][k]| / 448 (1 for an all-zero row, float32 division), codes[n][k] = e4m3(a[n][k] /
 * scale[n]) (float32 division, nearest-even, saturating). codes [N][K] uint8, scale [N] float32. */
moe_status moe_quantize_rows_fp8(const void* a, int64_t N, int64_t K, uint8_t* codes,
                                 float* scale, void* stream);

/* moe_grouped_ffn / moe_layer_forward_ex with W8A8 expert GEMMs (bf16 shapes only): qk_gate, qk_up
 * [E][I][H] and s_gate, s_up [E][I]; qk_down [E][H][I] and s_down [E][H] (moe_pack_weights_w8a8
 * of w_gate, w_up [E][H][I] and w_down [E][I][H]). y_slots and out stay bf16. */
moe_status moe_grouped_ffn_w8a8(const moe_shape* shape, const void* x, const int32_t* sorted_ids,
                                const int32_t* offsets, const uint8_t* qk_gate,
                                const uint8_t* qk_up, const uint8_t* qk_down, const float* s_gate,
                                const float* s_up, const float* s_down, void* y_slots, void* ws,
                                size_t ws_bytes, void* stream);
moe_status moe_layer_forward_w8a8(const moe_shape* shape, const moe_layer_opts* opts,
                                  const void* x, const void* w_router, const float* logit_bias,
                                  const uint8_t* qk_gate, const uint8_t* qk_up,
                                  const uint8_t* qk_down, const float* s_gate, const float* s_up,
                                  const float* s_down, void* out, float* logits_out,
                                  int32_t* topk_idx, float* topk_w, int32_t* counts,
                                  uint8_t* drop_mask, void* ws, size_t ws_bytes, void* stream);

/* Expert parallelism over R ranks, [P4] section "Token 分发的通信瓶颈" (rows go to the devices
 * that own their experts and the outputs come back) with the capacity of section
 * "昇腾NPU的通信计算重叠". Rank r holds its own T tokens (shape->T) and the experts
 * [r*E/R, (r+1)*E/R); shape->E is the total E, which R must divide. The ranks compute what one
 * device computes on the concatenated batch (rank 0's tokens first): capacity C from T_total,
 * drops by the global token order, each expert's rows expert-major in that order at its owner.
 * Steps on rank r: moe_route; moe_align with capacity_factor <= 0 (the local grouping);
 * gather every rank's `counts` into counts_all [R,E] (a collective between devices);
 * moe_ep_plan; moe_ep_dispatch; moe_ep_signal (rows sent) and moe_ep_wait (every rank's rows
 * arrived); moe_grouped_ffn on the owner's rows (E/R experts, k = 1, identity sorted_ids,
 * own_offsets); moe_ep_signal (outputs ready) and moe_ep_wait; moe_ep_combine. Before a buffer
 * is reused by the next step, a third signal/wait pair (or a host barrier) orders the reuse
 * after the last remote read. Rows move only by plain loads and stores through peer pointers.
 *
 * moe_ep_plan: owner [T*k] (rank owning the expert, -1 if dropped) and slot [T*k] (row in the
 * owner's slot-major buffer, -1 if dropped) of this rank's assignments, and own_offsets
 * [E/R + 1], the first slot of each of this rank's experts and the total. topk_idx [T,k],
 * slot_of_local [T*k], offsets_local [E+1] are moe_align's outputs for this rank's tokens
 * without a capacity limit; counts_all [R,E] int32 holds every rank's local counts. An expert
 * id outside [0, E) sets the error word at the start of `ws` (ws_bytes >= 256) and that
 * assignment is dropped. */
moe_status moe_ep_plan(const moe_shape* shape, int32_t R, int32_t rank, int64_t T_total,
                       const int32_t* topk_idx, const int32_t* slot_of_local,
                       const int32_t* offsets_local, const int32_t* counts_all, int32_t* owner,
                       int32_t* slot, int32_t* own_offsets, void* ws, size_t ws_bytes,
                       void* stream);

/* Stores the token row x[a/k,:] of every kept assignment a into peer_xs[owner[a]] at row
 * slot[a]. peer_xs is a device array of R device pointers to the ranks' slot-major row buffers
 * ([rows, H] dtype, 16-byte aligned; the other ranks' buffers mapped into this device's address
 * space, or other buffers of the same device when ranks are emulated on one device). The
 * stores are plain global stores, fenced at system scope by each block before it exits; the
 * owners read them after moe_ep_signal / moe_ep_wait. */
moe_status moe_ep_dispatch(const moe_shape* shape, int32_t R, const void* x,
                           const int32_t* owner, const int32_t* slot, void* const* peer_xs,
                           void* stream);

/* Step signal between ranks (the ordering of [P4] section "昇腾NPU的通信计算重叠", where compute
 * on arrived rows overlaps the transfer of the rest): after all earlier work on `stream`, stores
 * `epoch` into word `rank` of every rank's flag array, with a system-scope fence before it and
 * release semantics. peer_flags is a device array of R device pointers; peer_flags[q] points to
 * rank q's flag array of R uint32 words (mapped into this device's address space). Use a new
 * epoch per step and per kind of signal (flag arrays start at 0; epochs compare modulo 2^32). */
moe_status moe_ep_signal(int32_t R, int32_t rank, uint32_t epoch, uint32_t* const* peer_flags,
                         void* stream);

/* Waits on `stream` until every one of the R words of this rank's flag array `flags` (device
 * memory, 4-byte aligned; the flag arrays are exempt from the 16-byte rule) holds at least
 * `epoch` (system-scope acquire loads). The wait is bounded: if a rank
 * has not signalled within 2 s, the kernel records device error 2 in the error word at the start
 * of `ws` (ws_bytes >= 256) and returns; moe_check_error then reports MOE_ERR_DEVICE. Launch it
 * only after every signal it waits for has been launched, on this device or another: kernels
 * that wait on one another are never run as separate launches that must overlap on one GPU. */
moe_status moe_ep_wait(int32_t R, uint32_t epoch, const uint32_t* flags, void* ws,
                       size_t ws_bytes, void* stream);

/* out[t,:] = sum over kept j, ascending, of topk_w[t,j] * peer_y[owner][slot,:], accumulated in
 * float32 and rounded once (a fully dropped token gives a zero row): moe_combine with each
 * expert output row read from its owner. peer_y is a device array of R device pointers to the
 * ranks' expert outputs ([rows, H] dtype, slot-major, as moe_grouped_ffn writes them). */
moe_status moe_ep_combine(const moe_shape* shape, int32_t R, const void* const* peer_y,
                          const int32_t* owner, const int32_t* slot, const float* topk_w,
                          void* out, void* stream);

/* Synchronises `stream`, reads and clears the device error word at the start of `ws`.
 * Returns MOE_OK, MOE_ERR_DEVICE (a kernel flagged a fault; see moe_last_error_detail) or
 * MOE_ERR_CUDA. */
moe_status moe_check_error(void* ws, void* stream);

/* Failure-detection check: launches one kernel whose single wait (the bounded mbarrier wait
 * every pipelined kernel of the library uses) is never satisfied. After the wait limit (2 s)
 * the kernel records device error 2 in the error word at the start of `ws` (ws_bytes >= 256)
 * and returns, so moe_check_error then reports MOE_ERR_DEVICE and clears the word; the
 * context stays usable. Returns MOE_ERR_WORKSPACE without launching when ws is NULL or too
 * small. */
moe_status moe_probe_stalled_wait(void* ws, size_t ws_bytes, void* stream);

/* 1 in the debug build (libmoe_debug.so, compiled with -DMOE_DEBUG), 0 otherwise. The debug build
 * checks every slot, token-row and group-table index a kernel reads from device data before
 * using it; a failed check records device error 3 in the workspace error word (moe_check_error
 * reports it) and the access is skipped. Its results are otherwise those of the release build. */
int32_t moe_debug_checks(void);

/* Static description of a status code. */
const char* moe_status_string(moe_status status);

/* Human-readable detail of the last error returned on the calling thread (which argument
 * failed validation, the CUDA error string, the device error code). Never NULL. */
const char* moe_last_error_detail(void);

/* Profiling hook. When `events` is non-NULL, moe_layer_forward records events[i] (cudaEvent_t
 * passed as void*) on its stream after stage i: 0 route, 1 align, 2 expert GEMM1 (gate/up +
 * SwiGLU), 3 expert GEMM2 (down projection), 4 combine. n_events must be 5 (or 0 with NULL to
 * switch recording off). The setting is process-wide. */
moe_status moe_set_stage_events(void** events, int32_t n_events);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
