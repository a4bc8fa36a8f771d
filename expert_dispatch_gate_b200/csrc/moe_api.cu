// moe_api.cu — the C ABI of libmoe.so (declared in include/moe.h): host-side validation,
// workspace layout and the launch sequence of the MoE layer forward path.
//
// Nothing here allocates, frees or synchronises device memory (moe_check_error excepted).
// Invalid calls fail loudly with a status and a detail string and launch nothing; there is no
// fallback path.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <cmath>
#include <mutex>
#include <string>

#include "moe.h"
#include "internal.h"

namespace {

thread_local std::string g_detail = "";

std::mutex g_events_mu;
void* g_events[5] = {nullptr, nullptr, nullptr, nullptr, nullptr};
bool g_events_on = false;

moe_status fail(moe_status s, const std::string& why) {
  g_detail = why;
  return s;
}

moe_status cuda_fail(cudaError_t e, const char* where, const std::string& extra = "") {
  g_detail = std::string(where) + ": " + cudaGetErrorString(e) + (extra.empty() ? "" : " (" + extra + ")");
  return MOE_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t elem_size(int32_t dtype) { return dtype == MOE_F32 ? 4 : 2; }

size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

// Shape checks shared by every entry point.
moe_status check_shape(const moe_shape* s) {
  if (s == nullptr) return fail(MOE_ERR_INVALID_ARG, "shape is NULL");
  if (s->T < 0) return fail(MOE_ERR_INVALID_ARG, "T < 0");
  if (s->T >= (int64_t(1) << 24)) return fail(MOE_ERR_UNSUPPORTED, "T >= 2^24");
  if (s->H < 1 || s->I < 1) return fail(MOE_ERR_INVALID_ARG, "H and I must be >= 1");
  if (s->E < 1) return fail(MOE_ERR_INVALID_ARG, "E must be >= 1");
  if (s->E > 256) return fail(MOE_ERR_UNSUPPORTED, "E > 256");
  if (s->k < 1 || s->k > s->E) return fail(MOE_ERR_INVALID_ARG, "need 1 <= k <= E");
  if (s->k > 16) return fail(MOE_ERR_UNSUPPORTED, "k > 16");
  if (s->dtype != MOE_F32 && s->dtype != MOE_BF16)
    return fail(MOE_ERR_INVALID_ARG, "dtype must be MOE_F32 or MOE_BF16");
  if (!(s->capacity_factor == s->capacity_factor))
    return fail(MOE_ERR_INVALID_ARG, "capacity_factor is NaN");
  if (s->H % 8 != 0) return fail(MOE_ERR_UNSUPPORTED, "H % 8 != 0");
  if (s->dtype == MOE_BF16) {
    if (s->H % 64 != 0 || s->I % 64 != 0)
      return fail(MOE_ERR_UNSUPPORTED, "bf16 needs H % 64 == 0 and I % 64 == 0");
    if (s->E > 64 && s->E % 8 != 0) return fail(MOE_ERR_UNSUPPORTED, "bf16 with E > 64 needs E % 8 == 0");
  } else {
    if (s->E > 64) return fail(MOE_ERR_UNSUPPORTED, "f32 needs E <= 64");
  }
  return MOE_OK;
}

// Capacity C = ceil(cf*T*k/E), cf taken exactly as the float32 it is, capped at T.
int32_t capacity_of(const moe_shape& s) {
  if (!(s.capacity_factor > 0.0f)) return static_cast<int32_t>(s.T);
  int exp2 = 0;
  const double frac = frexp(static_cast<double>(s.capacity_factor), &exp2);  // cf = frac*2^exp2
  // frac in [0.5, 1) has a 24-bit mantissa: cf = m * 2^(exp2-24), m integer
  const unsigned __int128 m = static_cast<unsigned __int128>(ldexp(frac, 24));
  const int sh = exp2 - 24;
  unsigned __int128 num = m * static_cast<unsigned __int128>(s.T) * static_cast<unsigned>(s.k);
  unsigned __int128 den = static_cast<unsigned>(s.E);
  if (sh >= 0) {
    if (sh > 60) return static_cast<int32_t>(s.T);
    num <<= sh;
  } else {
    if (-sh > 60) return s.T > 0 ? 1 : 0;  // positive but tiny: ceil of a tiny positive value
    den <<= -sh;
  }
  const unsigned __int128 c = (num + den - 1) / den;
  return c >= static_cast<unsigned __int128>(s.T) ? static_cast<int32_t>(s.T) : static_cast<int32_t>(c);
}

// Largest token block of the expert GEMMs (a multiple of 32 in [32, 256]). It only shapes the
// work: an expert with n kept tokens runs as ceil(n / TB) blocks of equal size, whatever n is.
// Sized from the largest expected group, min(C, T, 2 * T*k/E): the shared-memory stages and
// TMEM accumulators are reserved for TB rows, so a TB far above the real groups (decode) wastes
// pipeline depth, and one far below splits experts and re-reads their weights.
int token_block(const moe_shape& s, int32_t C) {
  int64_t rows = C < s.T ? C : s.T;
  const int64_t mean2 = 2 * ((s.T * s.k + s.E - 1) / s.E);
  if (mean2 < rows) rows = mean2;
  if (rows < 1) rows = 1;
  int64_t tb = ((rows + 31) / 32) * 32;
  if (tb > 256) tb = 256;
  return static_cast<int>(tb);
}

// GEMM1 reads the token rows from an expert-major copy made right after the grouping when it
// runs on CTA pairs (every bf16 layer unless the build opts out of pairs): the copy is
// streamed by TMA, half per CTA. Otherwise GEMM1 gathers the rows straight from x.
bool gemm1_from_copy(const moe_shape& s) {
  return s.dtype == MOE_BF16 && moe::gemm1_uses_row_copy(s.I);
}

struct Layout {
  size_t err, logits, blk_hist, offsets, blk_prefix, sorted_ids, slot_of, hbuf, yslots, xs, total;
  size_t logits_bytes;
  size_t x8, h8;  // W8A8 (bf16 shapes): e4m3 token rows + scales, e4m3 h rows + scales
  int64_t A, a_cap;
  int nblk;
  int32_t C;
  int TB;
  int ksplit;  // router K split (tensor-core router only)
};

Layout layout_of(const moe_shape& s) {
  Layout L{};
  L.C = capacity_of(s);
  L.TB = token_block(s, L.C);
  L.A = s.T * s.k;
  const int64_t ec = static_cast<int64_t>(s.E) * L.C;
  L.a_cap = L.A < ec ? L.A : ec;
  L.nblk = static_cast<int>((L.A + moe::align_chunk(L.A) - 1) / moe::align_chunk(L.A));
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  const size_t es = elem_size(s.dtype);
  L.err = take(256);
  L.ksplit = (s.dtype == MOE_BF16 && s.E >= 64 && s.E % 8 == 0 && s.T > 0)
                 ? moe::route_ksplit(s.T, s.H, s.E) : 1;
  // the router's partial logits [ksplit][T][E] (or the CUDA-core router's logits before a
  // group-limited selection)
  L.logits_bytes = static_cast<size_t>(s.T) * s.E * 4 * L.ksplit;
  L.logits = take(L.logits_bytes);
  L.blk_hist = take(static_cast<size_t>(L.nblk) * s.E * 4);
  L.offsets = take(static_cast<size_t>(s.E + 1) * 4);
  L.blk_prefix = take(static_cast<size_t>(s.E + 1) * 4);
  L.sorted_ids = take(static_cast<size_t>(L.A) * 4);
  L.slot_of = take(static_cast<size_t>(L.A) * 4);
  L.hbuf = take(static_cast<size_t>(L.a_cap) * s.I * es);
  L.yslots = take(static_cast<size_t>(L.a_cap) * s.H * es);
  L.xs = s.dtype == MOE_BF16 ? take(static_cast<size_t>(L.a_cap) * s.H * es) : 0;
  // W8A8: x quantised per token ([T][H] codes, then T scales) and h per slot ([a_cap][I] codes,
  // then a_cap scales); the expert-major e4m3 rows and their scales reuse the xs region
  L.x8 = s.dtype == MOE_BF16 ? take(static_cast<size_t>(s.T) * s.H + static_cast<size_t>(s.T) * 4)
                             : 0;
  L.h8 = s.dtype == MOE_BF16
             ? take(static_cast<size_t>(L.a_cap) * s.I + static_cast<size_t>(L.a_cap) * 4)
             : 0;
  L.total = off;
  return L;
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
    return 148;
  return n;
}

#define REQUIRE_PTR(p, name)                                                  \
  do {                                                                        \
    if ((p) == nullptr) return fail(MOE_ERR_INVALID_ARG, name " is NULL");    \
    if (!aligned16(p)) return fail(MOE_ERR_INVALID_ARG, name " is not 16-byte aligned"); \
  } while (0)

#define OPT_PTR(p, name)                                                      \
  do {                                                                        \
    if ((p) != nullptr && !aligned16(p))                                      \
      return fail(MOE_ERR_INVALID_ARG, name " is not 16-byte aligned");       \
  } while (0)

moe_status check_ws(const void* ws, size_t ws_bytes, size_t need) {
  if (ws == nullptr) return fail(MOE_ERR_WORKSPACE, "workspace is NULL");
  if (!aligned16(ws)) return fail(MOE_ERR_INVALID_ARG, "workspace is not 16-byte aligned");
  if (ws_bytes < need)
    return fail(MOE_ERR_WORKSPACE, "workspace too small: need " + std::to_string(need) +
                                       " bytes, got " + std::to_string(ws_bytes));
  return MOE_OK;
}

template <typename P>
P* at(void* ws, size_t off) {
  return reinterpret_cast<P*>(static_cast<char*>(ws) + off);
}

void record_stage(int i, cudaStream_t st) {
  std::lock_guard<std::mutex> lk(g_events_mu);
  if (g_events_on && g_events[i] != nullptr)
    cudaEventRecord(static_cast<cudaEvent_t>(g_events[i]), st);
}

// ---- routing / combine options (moe_layer_opts), validated once per call

struct Opts {
  int n_group = 1, topk_group = 1;
  const void* shared = nullptr;
  float shared_factor = 0.f;
  const float* out_bias = nullptr;
};

moe_status read_opts(const moe_shape& s, const moe_layer_opts* o, Opts* out) {
  *out = Opts{};
  if (o == nullptr) return MOE_OK;
  if (o->n_group < 1 || o->n_group > 32 || s.E % o->n_group != 0)
    return fail(MOE_ERR_INVALID_ARG, "n_group must be in [1, 32] and divide E");
  if (o->topk_group < 1 || o->topk_group > o->n_group)
    return fail(MOE_ERR_INVALID_ARG, "topk_group must be in [1, n_group]");
  if (o->n_group > 1 && s.k > o->topk_group * (s.E / o->n_group))
    return fail(MOE_ERR_INVALID_ARG, "k exceeds the experts of the kept groups");
  if (!std::isfinite(o->shared_factor))
    return fail(MOE_ERR_INVALID_ARG, "shared_factor is not finite");
  OPT_PTR(o->shared_out, "shared_out");
  OPT_PTR(o->out_bias, "out_bias");
  out->n_group = o->n_group;
  out->topk_group = o->n_group > 1 ? o->topk_group : 1;
  out->shared = o->shared_out;
  out->shared_factor = o->shared_factor;
  out->out_bias = o->out_bias;
  return MOE_OK;
}

// ---- stage bodies (arguments already validated)

moe_status do_route(const moe_shape& s, const Layout& L, const Opts& o, const void* x,
                    const void* w_router, const float* bias, float* logits_out, int32_t* topk_idx,
                    float* topk_w, void* ws, cudaStream_t st) {
  cudaError_t e;
  if (s.dtype == MOE_BF16 && s.E >= 64 && s.E % 8 == 0 &&
      moe::route_fuses_topk(s.T, s.H, s.E, s.k, o.n_group)) {
    std::string d;
    e = moe::launch_route_gemm_topk_tc(x, w_router, static_cast<int>(s.T), s.H, s.E, s.k, bias,
                                       logits_out, topk_idx, topk_w, at<int>(ws, L.err),
                                       num_sms(), st, &d);
    if (e != cudaSuccess) return cuda_fail(e, "router gate GEMM + top-k (tcgen05)", d);
  } else if (s.dtype == MOE_BF16 && s.E >= 64 && s.E % 8 == 0) {
    float* partials = at<float>(ws, L.logits);
    std::string d;
    e = moe::launch_route_gemm_tc(x, w_router, static_cast<int>(s.T), s.H, s.E, partials,
                                  L.ksplit, at<int>(ws, L.err), num_sms(), st, &d);
    if (e != cudaSuccess) return cuda_fail(e, "router gate GEMM (tcgen05)", d);
    e = moe::launch_topk(partials, L.ksplit, s.T * s.E, bias, logits_out, s.T, s.E, s.k,
                         o.n_group, o.topk_group, topk_idx, topk_w, st);
    if (e != cudaSuccess) return cuda_fail(e, "router top-k");
  } else {
    // the fused CUDA-core router selects plain top-k; with groups its logits (bias included)
    // go through the group-limited top-k kernel
    float* lg = logits_out;
    if (o.n_group > 1 && lg == nullptr) lg = at<float>(ws, L.logits);
    e = moe::launch_route_simt(s.dtype, x, w_router, bias, s.T, s.H, s.E, s.k, lg, topk_idx,
                               topk_w, st);
    if (e != cudaSuccess) return cuda_fail(e, "router (CUDA cores)");
    if (o.n_group > 1) {
      e = moe::launch_topk(lg, 1, 0, nullptr, nullptr, s.T, s.E, s.k, o.n_group, o.topk_group,
                           topk_idx, topk_w, st);
      if (e != cudaSuccess) return cuda_fail(e, "router group-limited top-k");
    }
  }
  return MOE_OK;
}

// Expert weights: bf16 / f32 tensors, or e4m3 codes with per-channel scales (w8).
struct FfnWeights {
  const void* w_gate = nullptr;
  const void* w_up = nullptr;
  const void* w_down = nullptr;
  const uint8_t* q_gate = nullptr;
  const uint8_t* q_up = nullptr;
  const uint8_t* q_down = nullptr;
  const float* s_gate = nullptr;
  const float* s_up = nullptr;
  const float* s_down = nullptr;
  bool w8 = false;   // e4m3 weights [E][K][M], bf16 activations (W8A16)
  bool a8 = false;   // K-major e4m3 weights [E][M][K] and e4m3 activations (W8A8)
};

moe_status do_ffn(const moe_shape& s, const Layout& L, const void* x, const int32_t* sorted_ids,
                  const int32_t* offsets, const FfnWeights& fw, void* y, void* ws, cudaStream_t st,
                  bool stage_events) {
  const void* w_gate = fw.w_gate;
  const void* w_up = fw.w_up;
  const void* w_down = fw.w_down;
  cudaError_t e;
  if (fw.a8) {
    // x quantised once per token, copied expert-major with its scales; GEMM1 on e4m3 rows; h
    // (bf16) quantised per slot row; GEMM2 on e4m3 rows
    const int64_t ub_blocks = (s.E < L.a_cap ? s.E : L.a_cap) + L.a_cap / L.TB;
    std::string d;
    uint8_t* x8 = at<uint8_t>(ws, L.x8);
    float* sxt = reinterpret_cast<float*>(x8 + static_cast<size_t>(s.T) * s.H);
    uint8_t* xs8 = at<uint8_t>(ws, L.xs);
    float* sx = reinterpret_cast<float*>(xs8 + static_cast<size_t>(L.a_cap) * s.H);
    uint8_t* h8 = at<uint8_t>(ws, L.h8);
    float* sh = reinterpret_cast<float*>(h8 + static_cast<size_t>(L.a_cap) * s.I);
    e = moe::launch_quantize_rows(x, s.T, nullptr, s.H, x8, sxt, st);
    if (e != cudaSuccess) return cuda_fail(e, "e4m3 quantisation of the token rows");
    e = moe::launch_dispatch_rows_q8(x8, sxt, sorted_ids, offsets, s.E, s.k, s.H, L.a_cap, s.T,
                                     xs8, sx, at<int>(ws, L.err), st);
    if (e != cudaSuccess) return cuda_fail(e, "expert-major copy of the e4m3 rows");
    e = moe::launch_gemm1_f8(xs8, sx, offsets, at<int32_t>(ws, L.blk_prefix), fw.q_gate, fw.q_up,
                             fw.s_gate, fw.s_up, at<void>(ws, L.hbuf), L.a_cap, s.H, s.E, s.I,
                             L.TB, ub_blocks, at<int>(ws, L.err), num_sms(), st, &d);
    if (e != cudaSuccess) return cuda_fail(e, "expert GEMM1 (tcgen05, e4m3 x e4m3)", d);
    if (stage_events) record_stage(2, st);
    e = moe::launch_quantize_rows(at<void>(ws, L.hbuf), L.a_cap, offsets + s.E, s.I, h8, sh, st);
    if (e != cudaSuccess) return cuda_fail(e, "e4m3 quantisation of the SwiGLU rows");
    e = moe::launch_gemm2_f8(h8, sh, L.a_cap, offsets, at<int32_t>(ws, L.blk_prefix), fw.q_down,
                             fw.s_down, y, s.H, s.E, s.I, L.TB, ub_blocks, at<int>(ws, L.err),
                             num_sms(), st, &d);
    if (e != cudaSuccess) return cuda_fail(e, "expert GEMM2 (tcgen05, e4m3 x e4m3)", d);
  } else if (fw.w8) {
    const int64_t ub_blocks = (s.E < L.a_cap ? s.E : L.a_cap) + L.a_cap / L.TB;
    std::string d;
    void* xs = at<void>(ws, L.xs);
    e = moe::launch_dispatch_rows(s.dtype, x, sorted_ids, offsets, s.E, s.k, s.H, L.a_cap, s.T,
                                     xs, at<int>(ws, L.err), st);
    if (e != cudaSuccess) return cuda_fail(e, "expert-major row copy");
    e = moe::launch_gemm1_w8(xs, offsets, at<int32_t>(ws, L.blk_prefix), fw.q_gate, fw.q_up,
                             fw.s_gate, fw.s_up, at<void>(ws, L.hbuf), L.a_cap, s.H, s.E, s.I,
                             L.TB, ub_blocks, at<int>(ws, L.err), num_sms(), st, &d);
    if (e != cudaSuccess) return cuda_fail(e, "expert GEMM1 (tcgen05, e4m3 weights)", d);
    if (stage_events) record_stage(2, st);
    e = moe::launch_gemm2_w8(at<void>(ws, L.hbuf), L.a_cap, offsets, at<int32_t>(ws, L.blk_prefix),
                             fw.q_down, fw.s_down, y, s.H, s.E, s.I, L.TB, ub_blocks,
                             at<int>(ws, L.err), num_sms(), st, &d);
    if (e != cudaSuccess) return cuda_fail(e, "expert GEMM2 (tcgen05, e4m3 weights)", d);
  } else if (s.dtype == MOE_BF16) {
    const int64_t ub_blocks = (s.E < L.a_cap ? s.E : L.a_cap) + L.a_cap / L.TB;
    std::string d;
    void* xs = nullptr;
    if (gemm1_from_copy(s)) {
      xs = at<void>(ws, L.xs);
      e = moe::launch_dispatch_rows(s.dtype, x, sorted_ids, offsets, s.E, s.k, s.H, L.a_cap, s.T,
                                     xs, at<int>(ws, L.err), st);
      if (e != cudaSuccess) return cuda_fail(e, "expert-major row copy");
    }
    e = moe::launch_gemm1_tc(x, static_cast<int>(s.T), xs, sorted_ids, offsets,
                             at<int32_t>(ws, L.blk_prefix), w_gate, w_up, at<void>(ws, L.hbuf),
                             L.a_cap, s.H, s.E, s.k, s.I, L.TB, ub_blocks, at<int>(ws, L.err),
                             num_sms(), st, &d);
    if (e != cudaSuccess) return cuda_fail(e, "expert GEMM1 (tcgen05)", d);
    if (stage_events) record_stage(2, st);
    e = moe::launch_gemm2_tc(at<void>(ws, L.hbuf), L.a_cap, offsets, at<int32_t>(ws, L.blk_prefix),
                             w_down, y, s.H, s.E, s.I, L.TB, ub_blocks, at<int>(ws, L.err),
                             num_sms(), st, &d);
    if (e != cudaSuccess) return cuda_fail(e, "expert GEMM2 (tcgen05)", d);
  } else {
    e = moe::launch_gemm1_simt(static_cast<const float*>(x), sorted_ids, offsets,
                               static_cast<const float*>(w_gate), static_cast<const float*>(w_up),
                               at<float>(ws, L.hbuf), L.a_cap, s.H, s.E, s.k, s.I, st);
    if (e != cudaSuccess) return cuda_fail(e, "expert GEMM1 (CUDA cores)");
    if (stage_events) record_stage(2, st);
    e = moe::launch_gemm2_simt(at<float>(ws, L.hbuf), offsets, static_cast<const float*>(w_down),
                               static_cast<float*>(y), L.a_cap, s.H, s.E, s.I, st);
    if (e != cudaSuccess) return cuda_fail(e, "expert GEMM2 (CUDA cores)");
  }
  if (stage_events) record_stage(3, st);
  return MOE_OK;
}

}  // namespace

extern "C" {

int32_t moe_debug_checks(void) {
#ifdef MOE_DEBUG
  return 1;
#else
  return 0;
#endif
}

size_t moe_workspace_bytes(const moe_shape* shape) {
  if (check_shape(shape) != MOE_OK) return 0;
  return layout_of(*shape).total;
}

int32_t moe_capacity(const moe_shape* shape) {
  if (check_shape(shape) != MOE_OK) return -1;
  return capacity_of(*shape);
}

moe_status moe_route_ex(const moe_shape* shape, const moe_layer_opts* opts, const void* x,
                        const void* w_router, const float* logit_bias, float* logits_out,
                        int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes,
                        void* stream) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  Opts o;
  st = read_opts(*shape, opts, &o);
  if (st != MOE_OK) return st;
  if (shape->T == 0) return MOE_OK;
  REQUIRE_PTR(x, "x");
  REQUIRE_PTR(w_router, "w_router");
  REQUIRE_PTR(topk_idx, "topk_idx");
  REQUIRE_PTR(topk_w, "topk_w");
  OPT_PTR(logit_bias, "logit_bias");
  OPT_PTR(logits_out, "logits_out");
  const Layout L = layout_of(*shape);
  st = check_ws(ws, ws_bytes, L.logits + L.logits_bytes);
  if (st != MOE_OK) return st;
  return do_route(*shape, L, o, x, w_router, logit_bias, logits_out, topk_idx, topk_w, ws,
                  static_cast<cudaStream_t>(stream));
}

moe_status moe_route(const moe_shape* shape, const void* x, const void* w_router,
                     const float* logit_bias, float* logits_out, int32_t* topk_idx,
                     float* topk_w, void* ws, size_t ws_bytes, void* stream) {
  return moe_route_ex(shape, nullptr, x, w_router, logit_bias, logits_out, topk_idx, topk_w, ws,
                      ws_bytes, stream);
}

moe_status moe_route_from_logits_ex(const moe_shape* shape, const moe_layer_opts* opts,
                                    const float* logits, int32_t* topk_idx, float* topk_w,
                                    void* stream) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  Opts o;
  st = read_opts(*shape, opts, &o);
  if (st != MOE_OK) return st;
  if (shape->T == 0) return MOE_OK;
  REQUIRE_PTR(logits, "logits");
  REQUIRE_PTR(topk_idx, "topk_idx");
  REQUIRE_PTR(topk_w, "topk_w");
  cudaError_t e = moe::launch_topk(logits, 1, 0, nullptr, nullptr, shape->T, shape->E, shape->k,
                                   o.n_group, o.topk_group, topk_idx, topk_w,
                                   static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "router top-k");
  return MOE_OK;
}

moe_status moe_route_from_logits(const moe_shape* shape, const float* logits, int32_t* topk_idx,
                                 float* topk_w, void* stream) {
  return moe_route_from_logits_ex(shape, nullptr, logits, topk_idx, topk_w, stream);
}

moe_status moe_align(const moe_shape* shape, const int32_t* topk_idx, int32_t* counts,
                     int32_t* offsets, int32_t* sorted_ids, int32_t* slot_of, uint8_t* drop_mask,
                     void* ws, size_t ws_bytes, void* stream) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  REQUIRE_PTR(counts, "counts");
  REQUIRE_PTR(offsets, "offsets");
  const Layout L = layout_of(*shape);
  st = check_ws(ws, ws_bytes, L.blk_prefix + static_cast<size_t>(shape->E + 1) * 4);
  if (st != MOE_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (shape->T == 0) {
    // empty batch: zero counts and offsets, nothing else to write
    cudaError_t e = cudaMemsetAsync(counts, 0, static_cast<size_t>(shape->E) * 4, cs);
    if (e == cudaSuccess) e = cudaMemsetAsync(offsets, 0, static_cast<size_t>(shape->E + 1) * 4, cs);
    if (e != cudaSuccess) return cuda_fail(e, "align (empty batch)");
    return MOE_OK;
  }
  REQUIRE_PTR(topk_idx, "topk_idx");
  REQUIRE_PTR(sorted_ids, "sorted_ids");
  REQUIRE_PTR(slot_of, "slot_of");
  REQUIRE_PTR(drop_mask, "drop_mask");
  cudaError_t e = moe::launch_align(topk_idx, L.A, shape->E, L.C, L.TB, at<int32_t>(ws, L.blk_hist),
                                    counts, offsets, at<int32_t>(ws, L.blk_prefix), sorted_ids,
                                    slot_of, drop_mask, at<int>(ws, L.err), cs);
  if (e != cudaSuccess) return cuda_fail(e, "align");
  return MOE_OK;
}

moe_status moe_align_noalloc(const moe_shape* shape, const int32_t* topk_idx, int32_t* counts,
                             int32_t* offsets, int32_t* sorted_ids, int32_t* slot_of,
                             uint8_t* drop_mask, void* stream) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  REQUIRE_PTR(counts, "counts");
  REQUIRE_PTR(offsets, "offsets");
  const Layout L = layout_of(*shape);
  if (L.A > moe::kNoAllocMaxAssignments)
    return fail(MOE_ERR_UNSUPPORTED,
                "moe_align_noalloc handles at most " + std::to_string(moe::kNoAllocMaxAssignments) +
                    " assignments (T*k); got " + std::to_string(L.A) +
                    ": use moe_align with a workspace");
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (shape->T == 0) {
    cudaError_t e = cudaMemsetAsync(counts, 0, static_cast<size_t>(shape->E) * 4, cs);
    if (e == cudaSuccess) e = cudaMemsetAsync(offsets, 0, static_cast<size_t>(shape->E + 1) * 4, cs);
    if (e != cudaSuccess) return cuda_fail(e, "align without workspace (empty batch)");
    return MOE_OK;
  }
  REQUIRE_PTR(topk_idx, "topk_idx");
  REQUIRE_PTR(sorted_ids, "sorted_ids");
  REQUIRE_PTR(slot_of, "slot_of");
  REQUIRE_PTR(drop_mask, "drop_mask");
  cudaError_t e = moe::launch_align_noalloc(topk_idx, L.A, shape->E, L.C, L.TB, counts, offsets,
                                            sorted_ids, slot_of, drop_mask, cs);
  if (e != cudaSuccess) return cuda_fail(e, "align without workspace");
  return MOE_OK;
}

moe_status moe_grouped_ffn(const moe_shape* shape, const void* x, const int32_t* sorted_ids,
                           const int32_t* offsets, const void* w_gate, const void* w_up,
                           const void* w_down, void* y_slots, void* ws, size_t ws_bytes,
                           void* stream) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (shape->T == 0) return MOE_OK;
  REQUIRE_PTR(x, "x");
  REQUIRE_PTR(sorted_ids, "sorted_ids");
  REQUIRE_PTR(offsets, "offsets");
  REQUIRE_PTR(w_gate, "w_gate");
  REQUIRE_PTR(w_up, "w_up");
  REQUIRE_PTR(w_down, "w_down");
  REQUIRE_PTR(y_slots, "y_slots");
  const Layout L = layout_of(*shape);
  st = check_ws(ws, ws_bytes, L.total);
  if (st != MOE_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (shape->dtype == MOE_BF16) {
    cudaError_t e = moe::launch_plan_from_offsets(offsets, shape->E, L.TB,
                                                  at<int32_t>(ws, L.blk_prefix), cs);
    if (e != cudaSuccess) return cuda_fail(e, "expert GEMM tile plan");
  }
  FfnWeights fw;
  fw.w_gate = w_gate;
  fw.w_up = w_up;
  fw.w_down = w_down;
  return do_ffn(*shape, L, x, sorted_ids, offsets, fw, y_slots, ws, cs, false);
}

moe_status moe_combine_ex(const moe_shape* shape, const moe_layer_opts* opts,
                          const void* y_slots, const int32_t* slot_of, const float* topk_w,
                          void* out, void* stream) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  Opts o;
  st = read_opts(*shape, opts, &o);
  if (st != MOE_OK) return st;
  if (shape->T == 0) return MOE_OK;
  REQUIRE_PTR(y_slots, "y_slots");
  REQUIRE_PTR(slot_of, "slot_of");
  REQUIRE_PTR(topk_w, "topk_w");
  REQUIRE_PTR(out, "out");
  cudaError_t e = moe::launch_combine(shape->dtype, y_slots, slot_of, topk_w, o.shared,
                                      o.shared_factor, o.out_bias, out, shape->T, shape->H,
                                      shape->k, nullptr, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "combine");
  return MOE_OK;
}

moe_status moe_combine(const moe_shape* shape, const void* y_slots, const int32_t* slot_of,
                       const float* topk_w, void* out, void* stream) {
  return moe_combine_ex(shape, nullptr, y_slots, slot_of, topk_w, out, stream);
}

// ---- expert parallelism (ep.cu)

static moe_status check_ep(const moe_shape* shape, int32_t R) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (R < 1 || R > shape->E || shape->E % R != 0)
    return fail(MOE_ERR_INVALID_ARG, "the E experts must split evenly over R >= 1 ranks");
  return MOE_OK;
}

moe_status moe_ep_plan(const moe_shape* shape, int32_t R, int32_t rank, int64_t T_total,
                       const int32_t* topk_idx, const int32_t* slot_of_local,
                       const int32_t* offsets_local, const int32_t* counts_all, int32_t* owner,
                       int32_t* slot, int32_t* own_offsets, void* ws, size_t ws_bytes,
                       void* stream) {
  moe_status st = check_ep(shape, R);
  if (st != MOE_OK) return st;
  if (rank < 0 || rank >= R) return fail(MOE_ERR_INVALID_ARG, "rank outside [0, R)");
  if (T_total < shape->T) return fail(MOE_ERR_INVALID_ARG, "T_total below this rank's T");
  st = check_ws(ws, ws_bytes, 256);
  if (st != MOE_OK) return st;
  REQUIRE_PTR(counts_all, "counts_all");
  REQUIRE_PTR(own_offsets, "own_offsets");
  if (shape->T > 0) {
    REQUIRE_PTR(topk_idx, "topk_idx");
    REQUIRE_PTR(slot_of_local, "slot_of_local");
    REQUIRE_PTR(offsets_local, "offsets_local");
    REQUIRE_PTR(owner, "owner");
    REQUIRE_PTR(slot, "slot");
  }
  moe_shape whole = *shape;
  whole.T = T_total;
  const int C = capacity_of(whole);
  cudaError_t e = moe::launch_ep_plan(topk_idx, slot_of_local, offsets_local, counts_all,
                                      shape->T * shape->k, shape->E, R, rank, C, owner, slot,
                                      own_offsets, at<int>(ws, 0), num_sms(),
                                      static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "expert-parallel plan");
  return MOE_OK;
}

moe_status moe_ep_dispatch(const moe_shape* shape, int32_t R, const void* x,
                           const int32_t* owner, const int32_t* slot, void* const* peer_xs,
                           void* stream) {
  moe_status st = check_ep(shape, R);
  if (st != MOE_OK) return st;
  if (shape->T == 0) return MOE_OK;
  REQUIRE_PTR(x, "x");
  REQUIRE_PTR(owner, "owner");
  REQUIRE_PTR(slot, "slot");
  REQUIRE_PTR(peer_xs, "peer_xs");
  cudaError_t e = moe::launch_ep_dispatch(shape->dtype, x, owner, slot, peer_xs,
                                          shape->T * shape->k, shape->k, shape->H,
                                          static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "expert-parallel dispatch");
  return MOE_OK;
}

moe_status moe_ep_signal(int32_t R, int32_t rank, uint32_t epoch, uint32_t* const* peer_flags,
                         void* stream) {
  if (R < 1 || R > 256) return fail(MOE_ERR_INVALID_ARG, "R must be in [1, 256]");
  if (rank < 0 || rank >= R) return fail(MOE_ERR_INVALID_ARG, "rank outside [0, R)");
  REQUIRE_PTR(peer_flags, "peer_flags");
  cudaError_t e = moe::launch_ep_signal(peer_flags, R, rank, epoch,
                                        static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "expert-parallel signal");
  return MOE_OK;
}

moe_status moe_ep_wait(int32_t R, uint32_t epoch, const uint32_t* flags, void* ws,
                       size_t ws_bytes, void* stream) {
  if (R < 1 || R > 256) return fail(MOE_ERR_INVALID_ARG, "R must be in [1, 256]");
  if (flags == nullptr) return fail(MOE_ERR_INVALID_ARG, "flags is NULL");
  if ((reinterpret_cast<uintptr_t>(flags) & 3u) != 0)
    return fail(MOE_ERR_INVALID_ARG, "flags is not 4-byte aligned");
  moe_status st = check_ws(ws, ws_bytes, 256);
  if (st != MOE_OK) return st;
  cudaError_t e = moe::launch_ep_wait(flags, R, epoch, at<int>(ws, 0),
                                      static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "expert-parallel wait");
  return MOE_OK;
}

moe_status moe_ep_combine(const moe_shape* shape, int32_t R, const void* const* peer_y,
                          const int32_t* owner, const int32_t* slot, const float* topk_w,
                          void* out, void* stream) {
  moe_status st = check_ep(shape, R);
  if (st != MOE_OK) return st;
  if (shape->T == 0) return MOE_OK;
  REQUIRE_PTR(peer_y, "peer_y");
  REQUIRE_PTR(owner, "owner");
  REQUIRE_PTR(slot, "slot");
  REQUIRE_PTR(topk_w, "topk_w");
  REQUIRE_PTR(out, "out");
  cudaError_t e = moe::launch_ep_combine(shape->dtype, peer_y, owner, slot, topk_w, out, shape->T,
                                         shape->H, shape->k, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "expert-parallel combine");
  return MOE_OK;
}

}  // extern "C"

namespace {

moe_status layer_impl(const moe_shape* shape, const moe_layer_opts* opts, const void* x,
                      const void* w_router, const float* logit_bias, const FfnWeights& fw,
                      void* out, float* logits_out, int32_t* topk_idx, float* topk_w,
                      int32_t* counts, uint8_t* drop_mask, void* ws, size_t ws_bytes,
                      void* stream) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  const moe_shape& s = *shape;
  Opts o;
  st = read_opts(s, opts, &o);
  if (st != MOE_OK) return st;
  REQUIRE_PTR(counts, "counts");
  const Layout L = layout_of(s);
  st = check_ws(ws, ws_bytes, L.total);
  if (st != MOE_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (s.T == 0) {
    cudaError_t e = cudaMemsetAsync(counts, 0, static_cast<size_t>(s.E) * 4, cs);
    if (e != cudaSuccess) return cuda_fail(e, "layer (empty batch)");
    return MOE_OK;
  }
  REQUIRE_PTR(x, "x");
  REQUIRE_PTR(w_router, "w_router");
  if (fw.w8 || fw.a8) {
    if (s.dtype != MOE_BF16) return fail(MOE_ERR_UNSUPPORTED, "e4m3 expert weights need bf16");
    REQUIRE_PTR(fw.q_gate, "q_gate");
    REQUIRE_PTR(fw.q_up, "q_up");
    REQUIRE_PTR(fw.q_down, "q_down");
    REQUIRE_PTR(fw.s_gate, "s_gate");
    REQUIRE_PTR(fw.s_up, "s_up");
    REQUIRE_PTR(fw.s_down, "s_down");
  } else {
    REQUIRE_PTR(fw.w_gate, "w_gate");
    REQUIRE_PTR(fw.w_up, "w_up");
    REQUIRE_PTR(fw.w_down, "w_down");
  }
  REQUIRE_PTR(out, "out");
  REQUIRE_PTR(topk_idx, "topk_idx");
  REQUIRE_PTR(topk_w, "topk_w");
  REQUIRE_PTR(drop_mask, "drop_mask");
  OPT_PTR(logit_bias, "logit_bias");
  OPT_PTR(logits_out, "logits_out");

  st = do_route(s, L, o, x, w_router, logit_bias, logits_out, topk_idx, topk_w, ws, cs);
  if (st != MOE_OK) return st;
  record_stage(0, cs);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* sorted_ids = at<int32_t>(ws, L.sorted_ids);
  int32_t* slot_of = at<int32_t>(ws, L.slot_of);
  cudaError_t e = moe::launch_align(topk_idx, L.A, s.E, L.C, L.TB, at<int32_t>(ws, L.blk_hist),
                                    counts, offsets, at<int32_t>(ws, L.blk_prefix), sorted_ids,
                                    slot_of, drop_mask, at<int>(ws, L.err), cs);
  if (e != cudaSuccess) return cuda_fail(e, "align");
  record_stage(1, cs);
  void* y = at<void>(ws, L.yslots);
  st = do_ffn(s, L, x, sorted_ids, offsets, fw, y, ws, cs, true);
  if (st != MOE_OK) return st;
  e = moe::launch_combine(s.dtype, y, slot_of, topk_w, o.shared, o.shared_factor, o.out_bias, out,
                          s.T, s.H, s.k, at<int>(ws, L.err), cs);
  if (e != cudaSuccess) return cuda_fail(e, "combine");
  record_stage(4, cs);
  return MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_layer_forward_ex(const moe_shape* shape, const moe_layer_opts* opts,
                                const void* x, const void* w_router, const float* logit_bias,
                                const void* w_gate, const void* w_up, const void* w_down,
                                void* out, float* logits_out, int32_t* topk_idx, float* topk_w,
                                int32_t* counts, uint8_t* drop_mask, void* ws, size_t ws_bytes,
                                void* stream) {
  FfnWeights fw;
  fw.w_gate = w_gate;
  fw.w_up = w_up;
  fw.w_down = w_down;
  return layer_impl(shape, opts, x, w_router, logit_bias, fw, out, logits_out, topk_idx, topk_w,
                    counts, drop_mask, ws, ws_bytes, stream);
}

moe_status moe_layer_forward_w8(const moe_shape* shape, const moe_layer_opts* opts,
                                const void* x, const void* w_router, const float* logit_bias,
                                const uint8_t* q_gate, const uint8_t* q_up, const uint8_t* q_down,
                                const float* s_gate, const float* s_up, const float* s_down,
                                void* out, float* logits_out, int32_t* topk_idx, float* topk_w,
                                int32_t* counts, uint8_t* drop_mask, void* ws, size_t ws_bytes,
                                void* stream) {
  FfnWeights fw;
  fw.q_gate = q_gate;
  fw.q_up = q_up;
  fw.q_down = q_down;
  fw.s_gate = s_gate;
  fw.s_up = s_up;
  fw.s_down = s_down;
  fw.w8 = true;
  return layer_impl(shape, opts, x, w_router, logit_bias, fw, out, logits_out, topk_idx, topk_w,
                    counts, drop_mask, ws, ws_bytes, stream);
}

moe_status moe_grouped_ffn_w8(const moe_shape* shape, const void* x, const int32_t* sorted_ids,
                              const int32_t* offsets, const uint8_t* q_gate, const uint8_t* q_up,
                              const uint8_t* q_down, const float* s_gate, const float* s_up,
                              const float* s_down, void* y_slots, void* ws, size_t ws_bytes,
                              void* stream) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (shape->dtype != MOE_BF16) return fail(MOE_ERR_UNSUPPORTED, "e4m3 expert weights need bf16");
  if (shape->T == 0) return MOE_OK;
  REQUIRE_PTR(x, "x");
  REQUIRE_PTR(sorted_ids, "sorted_ids");
  REQUIRE_PTR(offsets, "offsets");
  REQUIRE_PTR(q_gate, "q_gate");
  REQUIRE_PTR(q_up, "q_up");
  REQUIRE_PTR(q_down, "q_down");
  REQUIRE_PTR(s_gate, "s_gate");
  REQUIRE_PTR(s_up, "s_up");
  REQUIRE_PTR(s_down, "s_down");
  REQUIRE_PTR(y_slots, "y_slots");
  const Layout L = layout_of(*shape);
  st = check_ws(ws, ws_bytes, L.total);
  if (st != MOE_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  cudaError_t e = moe::launch_plan_from_offsets(offsets, shape->E, L.TB,
                                                at<int32_t>(ws, L.blk_prefix), cs);
  if (e != cudaSuccess) return cuda_fail(e, "expert GEMM tile plan");
  FfnWeights fw;
  fw.q_gate = q_gate;
  fw.q_up = q_up;
  fw.q_down = q_down;
  fw.s_gate = s_gate;
  fw.s_up = s_up;
  fw.s_down = s_down;
  fw.w8 = true;
  return do_ffn(*shape, L, x, sorted_ids, offsets, fw, y_slots, ws, cs, false);
}

moe_status moe_quantize_weights_fp8(const void* w, int64_t E, int64_t K, int64_t M,
                                    uint8_t* codes, float* scale, void* stream) {
  if (E < 0 || K < 1 || M < 2 || M % 2 != 0 || K > (1 << 30) || M > (1 << 30))
    return fail(MOE_ERR_INVALID_ARG, "need E >= 0, K >= 1 and an even M >= 2");
  if (E == 0) return MOE_OK;
  REQUIRE_PTR(w, "w");
  REQUIRE_PTR(codes, "codes");
  REQUIRE_PTR(scale, "scale");
  cudaError_t e = moe::launch_quantize_fp8(w, E, static_cast<int>(K), static_cast<int>(M), codes,
                                           scale, num_sms(), static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "e4m3 weight quantisation");
  return MOE_OK;
}

moe_status moe_pack_weights_w8a8(const void* w, int64_t E, int64_t K, int64_t M, uint8_t* codes,
                                 float* scale, void* stream) {
  if (E < 0 || K < 64 || M < 64 || K % 64 != 0 || M % 64 != 0 || K > (1 << 30) || M > (1 << 30))
    return fail(MOE_ERR_INVALID_ARG, "need E >= 0 and K, M positive multiples of 64");
  if (E == 0) return MOE_OK;
  REQUIRE_PTR(w, "w");
  REQUIRE_PTR(codes, "codes");
  REQUIRE_PTR(scale, "scale");
  cudaError_t e = moe::launch_pack_w8a8(w, E, static_cast<int>(K), static_cast<int>(M), codes,
                                        scale, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "W8A8 weight packing");
  return MOE_OK;
}

moe_status moe_quantize_rows_fp8(const void* a, int64_t N, int64_t K, uint8_t* codes,
                                 float* scale, void* stream) {
  if (N < 0 || K < 8 || K % 8 != 0 || K > (1 << 30))
    return fail(MOE_ERR_INVALID_ARG, "need N >= 0 and K a positive multiple of 8");
  if (N == 0) return MOE_OK;
  REQUIRE_PTR(a, "a");
  REQUIRE_PTR(codes, "codes");
  REQUIRE_PTR(scale, "scale");
  cudaError_t e = moe::launch_quantize_rows(a, N, nullptr, static_cast<int>(K), codes, scale,
                                            static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "e4m3 row quantisation");
  return MOE_OK;
}

moe_status moe_grouped_ffn_w8a8(const moe_shape* shape, const void* x, const int32_t* sorted_ids,
                                const int32_t* offsets, const uint8_t* qk_gate,
                                const uint8_t* qk_up, const uint8_t* qk_down, const float* s_gate,
                                const float* s_up, const float* s_down, void* y_slots, void* ws,
                                size_t ws_bytes, void* stream) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (shape->dtype != MOE_BF16) return fail(MOE_ERR_UNSUPPORTED, "e4m3 expert weights need bf16");
  if (shape->T == 0) return MOE_OK;
  REQUIRE_PTR(x, "x");
  REQUIRE_PTR(sorted_ids, "sorted_ids");
  REQUIRE_PTR(offsets, "offsets");
  REQUIRE_PTR(qk_gate, "qk_gate");
  REQUIRE_PTR(qk_up, "qk_up");
  REQUIRE_PTR(qk_down, "qk_down");
  REQUIRE_PTR(s_gate, "s_gate");
  REQUIRE_PTR(s_up, "s_up");
  REQUIRE_PTR(s_down, "s_down");
  REQUIRE_PTR(y_slots, "y_slots");
  const Layout L = layout_of(*shape);
  st = check_ws(ws, ws_bytes, L.total);
  if (st != MOE_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  cudaError_t e = moe::launch_plan_from_offsets(offsets, shape->E, L.TB,
                                                at<int32_t>(ws, L.blk_prefix), cs);
  if (e != cudaSuccess) return cuda_fail(e, "expert GEMM tile plan");
  FfnWeights fw;
  fw.q_gate = qk_gate;
  fw.q_up = qk_up;
  fw.q_down = qk_down;
  fw.s_gate = s_gate;
  fw.s_up = s_up;
  fw.s_down = s_down;
  fw.a8 = true;
  return do_ffn(*shape, L, x, sorted_ids, offsets, fw, y_slots, ws, cs, false);
}

moe_status moe_layer_forward_w8a8(const moe_shape* shape, const moe_layer_opts* opts,
                                  const void* x, const void* w_router, const float* logit_bias,
                                  const uint8_t* qk_gate, const uint8_t* qk_up,
                                  const uint8_t* qk_down, const float* s_gate, const float* s_up,
                                  const float* s_down, void* out, float* logits_out,
                                  int32_t* topk_idx, float* topk_w, int32_t* counts,
                                  uint8_t* drop_mask, void* ws, size_t ws_bytes, void* stream) {
  FfnWeights fw;
  fw.q_gate = qk_gate;
  fw.q_up = qk_up;
  fw.q_down = qk_down;
  fw.s_gate = s_gate;
  fw.s_up = s_up;
  fw.s_down = s_down;
  fw.a8 = true;
  return layer_impl(shape, opts, x, w_router, logit_bias, fw, out, logits_out, topk_idx, topk_w,
                    counts, drop_mask, ws, ws_bytes, stream);
}

moe_status moe_layer_forward(const moe_shape* shape, const void* x, const void* w_router,
                             const float* logit_bias, const void* w_gate, const void* w_up,
                             const void* w_down, void* out, float* logits_out, int32_t* topk_idx,
                             float* topk_w, int32_t* counts, uint8_t* drop_mask, void* ws,
                             size_t ws_bytes, void* stream) {
  return moe_layer_forward_ex(shape, nullptr, x, w_router, logit_bias, w_gate, w_up, w_down, out,
                              logits_out, topk_idx, topk_w, counts, drop_mask, ws, ws_bytes,
                              stream);
}

moe_status moe_probe_stalled_wait(void* ws, size_t ws_bytes, void* stream) {
  moe_status st = check_ws(ws, ws_bytes, 256);
  if (st != MOE_OK) return st;
  cudaError_t e = moe::launch_stalled_wait(at<int>(ws, 0), static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stalled-wait probe");
  return MOE_OK;
}

moe_status moe_check_error(void* ws, void* stream) {
  if (ws == nullptr) return fail(MOE_ERR_INVALID_ARG, "workspace is NULL");
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, ws, sizeof(int), cudaMemcpyDeviceToHost, cs);
  if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
  if (e != cudaSuccess) return cuda_fail(e, "moe_check_error");
  if (word != 0) {
    // the whole 256-byte control block: a wait that ran out may have left the grouping's grid
    // barrier counters (words 32 and 33) off zero
    e = cudaMemsetAsync(ws, 0, 256, cs);
    if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
    if (e != cudaSuccess) return cuda_fail(e, "moe_check_error (clear)");
    const char* what = word == 1 ? "an expert id outside [0, E) in topk_idx"
                       : word == 3 ? "debug bounds check: a slot, token row or group offset read "
                                     "from device data was out of range"
                       : word == 2 ? "a bounded wait ran out in a pipelined kernel (stalled pipeline)"
                                   : "unknown device error";
    return fail(MOE_ERR_DEVICE, std::string("device error ") + std::to_string(word) + ": " + what);
  }
  return MOE_OK;
}

const char* moe_status_string(moe_status status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: invalid argument";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: shape outside the supported limits";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace missing or too small";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: CUDA runtime or launch failure";
    case MOE_ERR_DEVICE: return "MOE_ERR_DEVICE: a kernel reported a device-side fault";
  }
  return "unknown moe_status";
}

const char* moe_last_error_detail(void) { return g_detail.c_str(); }

moe_status moe_set_stage_events(void** events, int32_t n_events) {
  std::lock_guard<std::mutex> lk(g_events_mu);
  if (events == nullptr) {
    if (n_events != 0) return fail(MOE_ERR_INVALID_ARG, "events is NULL but n_events != 0");
    for (int i = 0; i < 5; ++i) g_events[i] = nullptr;
    g_events_on = false;
    return MOE_OK;
  }
  if (n_events != 5) return fail(MOE_ERR_INVALID_ARG, "n_events must be 5");
  for (int i = 0; i < 5; ++i) g_events[i] = events[i];
  g_events_on = true;
  return MOE_OK;
}

}  // extern "C"
