// C ABI of the MoE FFN layer: host-side validation, workspace layout and kernel sequencing.
// Every entry point validates its arguments before enqueuing anything and reports errors
// as a moe_status; nothing here allocates, frees or synchronises on the compute path.
#include <cstring>

#include "common.cuh"

using namespace moe;

namespace {

constexpr size_t kAlign = 256;
constexpr int kTcMinTokens = 33;
inline size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool bank_ok(const moe_bank& b, int expect_n, int d, int f) {
  if (b.n_exp != expect_n) return false;
  if (expect_n == 0) return true;
  if (b.fmt != MOE_W_BF16 && b.fmt != MOE_W_INT8 && b.fmt != MOE_W_INT4 && b.fmt != MOE_W_NVFP4)
    return false;
  const void* w[3] = {b.w_gate, b.w_up, b.w_down};
  for (const void* p : w)
    if (!p || !aligned(p, 16)) return false;
  if (b.fmt == MOE_W_BF16) return true;
  if (b.fmt == MOE_W_NVFP4) {
    // packed block scales (bulk copies: 16-byte aligned) and the tensor scales
    if (b.group != 16) return false;
    const void* s[3] = {b.s_gate, b.s_up, b.s_down};
    for (const void* p : s)
      if (!p || !aligned(p, 16)) return false;
    const float* g[3] = {b.g_gate, b.g_up, b.g_down};
    for (const float* p : g)
      if (!p || !aligned(p, 4)) return false;
    return true;
  }
  if (b.group != kGroup) return false;
  const void* s[3] = {b.s_gate, b.s_up, b.s_down};
  for (const void* p : s)
    if (!p || !aligned(p, 2)) return false;
  (void)d;
  (void)f;
  return true;
}

moe_status validate(const moe_layer* L) {
  if (!L) return MOE_ERR_INVALID_ARG;
  if (L->T < 1 || L->d < 128 || L->f < 128 || L->E < 1 || L->k < 1) return MOE_ERR_INVALID_ARG;
  if (L->d % 128 || L->f % 128) return MOE_ERR_INVALID_ARG;
  if (L->d > 8192 || L->f > 8192) return MOE_ERR_UNSUPPORTED;
  if (L->E > kMaxE || L->k > kMaxK || L->k > L->E) return MOE_ERR_UNSUPPORTED;
  if ((long long)L->T * L->k > (1LL << 30)) return MOE_ERR_UNSUPPORTED;
  if (L->path < MOE_PATH_AUTO || L->path > MOE_PATH_FUSED) return MOE_ERR_INVALID_ARG;
  if (!L->router_w || !aligned(L->router_w, 16)) return MOE_ERR_INVALID_ARG;
  if (L->router_bias && !aligned(L->router_bias, 4)) return MOE_ERR_INVALID_ARG;
  if (!bank_ok(L->routed, L->E, L->d, L->f)) return MOE_ERR_INVALID_ARG;
  if (L->shared.n_exp != 0 && L->shared.n_exp != 1) return MOE_ERR_UNSUPPORTED;
  if (!bank_ok(L->shared, L->shared.n_exp, L->d, L->f)) return MOE_ERR_INVALID_ARG;
  if (L->shared.n_exp && L->shared.fmt == MOE_W_NVFP4) return MOE_ERR_UNSUPPORTED;
  if (L->routed.fmt == MOE_W_NVFP4) {
    // the FP4 tensor-core kernels only; stages of 256 K values
    if (L->path == MOE_PATH_GEMV || L->path == MOE_PATH_FUSED) return MOE_ERR_UNSUPPORTED;
    if (L->d % 256 || L->f % 256) return MOE_ERR_UNSUPPORTED;
  }
  return MOE_OK;
}

inline bool is_nvfp4(const moe_layer* L) { return L->routed.fmt == MOE_W_NVFP4; }

// Workspace layout (offsets from the 256-byte aligned base).
struct WsLayout {
  size_t status, logits, topk_idx, topk_w, offsets, perm, inv, active, cta_hist, h, y_assign,
      y_shared, xg, tc_sched, xq, xsf, gx, h32, hq, hsf, gh, total;
};

WsLayout layout(const moe_layer* L) {
  WsLayout w{};
  const size_t T = L->T, k = L->k, E = L->E, d = L->d, f = L->f;
  const size_t n = T * k;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes); return at; };
  w.status = take(sync_bytes(L->d));
  w.logits = take(T * E * sizeof(float));
  w.topk_idx = take(n * sizeof(int32_t));
  w.topk_w = take(n * sizeof(float));
  w.offsets = take((E + 1) * sizeof(int32_t));
  w.perm = take(n * sizeof(int32_t));
  w.inv = take(n * sizeof(int32_t));
  w.active = take((E + 2) * sizeof(int32_t));
  w.cta_hist = take((size_t)perm_chunks(L->T, L->k) * E * sizeof(int32_t));
  w.h = take((n + T) * f * sizeof(uint16_t));
  w.y_assign = take(n * d * sizeof(float));
  w.y_shared = take(T * d * sizeof(float));
  w.xg = take((n + T) * d * sizeof(uint16_t));
  w.tc_sched = take(tc_sched_bytes(L->E));
  // NVFP4 routed experts: quantised activations, block scales by token tile, fp32 h
  const bool nv = is_nvfp4(L);
  const size_t tiles = nv ? nv_tile_cap(L->T, L->k, L->E) : 0;
  w.xq = take(nv ? n * d / 2 : 0);
  w.xsf = take(tiles * (d / 64) * 512);
  w.gx = take(nv ? n * sizeof(float) : 0);
  w.h32 = take(nv ? n * f * sizeof(float) : 0);
  w.hq = take(nv ? n * f / 2 : 0);
  w.hsf = take(tiles * (f / 64) * 512);
  w.gh = take(nv ? n * sizeof(float) : 0);
  w.total = o;
  return w;
}

Bank to_bank(const moe_bank& b) {
  Bank r;
  r.fmt = b.fmt;
  r.w[0] = b.w_gate;
  r.w[1] = b.w_up;
  r.w[2] = b.w_down;
  r.s[0] = static_cast<const uint16_t*>(b.s_gate);
  r.s[1] = static_cast<const uint16_t*>(b.s_up);
  r.s[2] = static_cast<const uint16_t*>(b.s_down);
  if (b.fmt == MOE_W_BF16) r.s[0] = r.s[1] = r.s[2] = nullptr;
  r.g[0] = b.fmt == MOE_W_NVFP4 ? b.g_gate : nullptr;
  r.g[1] = b.fmt == MOE_W_NVFP4 ? b.g_up : nullptr;
  r.g[2] = b.fmt == MOE_W_NVFP4 ? b.g_down : nullptr;
  return r;
}

moe_status check_ws(const moe_layer* L, void* ws, size_t ws_bytes) {
  if (!ws || !aligned(ws, kAlign)) return MOE_ERR_WORKSPACE;
  if (ws_bytes < layout(L).total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

Plan make_plan(const moe_layer* L, void* ws) {
  const WsLayout w = layout(L);
  uint8_t* b = static_cast<uint8_t*>(ws);
  Plan p{};
  p.T = L->T;
  p.d = L->d;
  p.f = L->f;
  p.E = L->E;
  p.k = L->k;
  p.has_shared = L->shared.n_exp;
  p.router_w = static_cast<const uint16_t*>(L->router_w);
  p.router_bias = L->router_bias;
  p.routed = to_bank(L->routed);
  p.shared = to_bank(L->shared);
  p.status = reinterpret_cast<int32_t*>(b + w.status + kSyncStatus);
  p.ticket = reinterpret_cast<int32_t*>(b + w.status + kSyncTicket);
  p.gbar = reinterpret_cast<uint32_t*>(b + w.status + kSyncGbar);
  p.test_ctl = reinterpret_cast<const int32_t*>(b + w.status + kSyncTest);
  p.tile_cnt = reinterpret_cast<int32_t*>(b + w.status + kSyncTiles);
  p.logits = reinterpret_cast<float*>(b + w.logits);
  p.topk_idx = reinterpret_cast<int32_t*>(b + w.topk_idx);
  p.topk_w = reinterpret_cast<float*>(b + w.topk_w);
  p.offsets = reinterpret_cast<int32_t*>(b + w.offsets);
  p.perm = reinterpret_cast<int32_t*>(b + w.perm);
  p.inv = reinterpret_cast<int32_t*>(b + w.inv);
  p.active = reinterpret_cast<int32_t*>(b + w.active);
  p.cta_hist = reinterpret_cast<int32_t*>(b + w.cta_hist);
  p.h = reinterpret_cast<uint16_t*>(b + w.h);
  p.y_assign = reinterpret_cast<float*>(b + w.y_assign);
  p.y_shared = reinterpret_cast<float*>(b + w.y_shared);
  p.xg = reinterpret_cast<uint16_t*>(b + w.xg);
  p.tc_sched = reinterpret_cast<int32_t*>(b + w.tc_sched);
  if (is_nvfp4(L)) {
    p.xq = b + w.xq;
    p.xsf = b + w.xsf;
    p.gx = reinterpret_cast<float*>(b + w.gx);
    p.h32 = reinterpret_cast<float*>(b + w.h32);
    p.hq = b + w.hq;
    p.hsf = b + w.hsf;
    p.gh = reinterpret_cast<float*>(b + w.gh);
  }
  p.path = L->path;
  return p;
}

#define MOE_TRY(expr)                                  \
  do {                                                 \
    cudaError_t _e = (expr);                           \
    if (_e != cudaSuccess) return MOE_ERR_CUDA;        \
  } while (0)

// Records mark i on the stream. The external flag makes the record a node of its own when
// the stream is being captured into a CUDA graph, so the mark also fires on every replay.
cudaError_t record_mark(void* const* marks, int n_marks, int i, cudaStream_t st) {
  if (i >= n_marks || !marks[i]) return cudaSuccess;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  cudaError_t err = cudaStreamIsCapturing(st, &cap);
  if (err != cudaSuccess) return err;
  cudaEvent_t ev = static_cast<cudaEvent_t>(marks[i]);
  if (cap == cudaStreamCaptureStatusActive)
    return cudaEventRecordWithFlags(ev, st, cudaEventRecordExternal);
  return cudaEventRecord(ev, st);
}

bool scales_aligned16(const Bank& b) {
  for (int i = 0; i < 3; ++i)
    if (b.s[i] && !aligned(b.s[i], 16)) return false;
  return true;
}

// Grouped FFN kernels for the call: the tensor-core grouped GEMMs from kTcMinTokens tokens
// up, the TMA-pipelined GEMV for smaller int4 calls, the register-streaming GEMV otherwise.
// Up to 32 rows (decode and speculative-verify calls) the automatic choice keeps a token's
// output bits independent of the call: the GEMV kernels and the single-kernel 1-token layer
// share one arithmetic order (TandemLLM docs, "17 Qwen3.8-Flash-Next", §17.3: decode rows
// must equal the rows of a verify chain bit for bit); they are also the faster choice
// there (measured on B200: 16 / 32 rows 233 / 387 us against 289 / 473 us on the tensor
// cores, which sum in another order; MOE_PATH_TC asks for them). Kernels after the first of
// a call use programmatic dependent launch.
bool use_tc(const Plan& p) {
  if (p.path == MOE_PATH_GEMV || p.path == MOE_PATH_FUSED) return false;
  if (p.path == MOE_PATH_TC) return true;
  return p.T >= kTcMinTokens;
}

// The single-kernel 1-token layer (decode_fused.cu) when the call allows it.
bool use_fused(const Plan& p) {
  if (p.path != MOE_PATH_AUTO && p.path != MOE_PATH_FUSED) return false;
  return decode_fused_supported(p);
}

// NVFP4 routed experts: the FP4 tensor-core kernels for them, the shared expert (another
// format) on the integer/bf16 tensor-core kernels.
moe_status run_ffn_nvfp4(const Plan& p, cudaStream_t st, void* const* marks, int n_marks) {
  if (!nv_supported(p) || !tc_supported(p)) return MOE_ERR_UNSUPPORTED;
  if (p.has_shared && !scales_aligned16(p.shared)) return MOE_ERR_UNSUPPORTED;
  const TcSched S = tc_sched_view(p.tc_sched, p.E);
  MOE_TRY(launch_tc_prep(p, S, p.xg, st, /*shared_rows_only=*/true));
  MOE_TRY(launch_nv_quant_x(p, S, st));
  MOE_TRY(launch_nv_gate_up(p, S, st));
  if (p.has_shared) MOE_TRY(launch_tc_shared_gate_up(p, S, p.xg, st));
  MOE_TRY(record_mark(marks, n_marks, 3, st));
  MOE_TRY(launch_nv_quant_h(p, S, st));
  MOE_TRY(launch_nv_down(p, S, st));
  if (p.has_shared) MOE_TRY(launch_tc_shared_down(p, S, st));
  MOE_TRY(record_mark(marks, n_marks, 4, st));
  return MOE_OK;
}

moe_status run_ffn(const Plan& p, cudaStream_t st, void* const* marks, int n_marks) {
  if (p.routed.fmt == kNvfp4) return run_ffn_nvfp4(p, st, marks, n_marks);
  if (use_tc(p)) {
    if (!tc_supported(p) || !scales_aligned16(p.routed) ||
        (p.has_shared && !scales_aligned16(p.shared)))
      return MOE_ERR_UNSUPPORTED;
    const TcSched S = tc_sched_view(p.tc_sched, p.E);
    MOE_TRY(launch_tc_prep(p, S, p.xg, st));
    MOE_TRY(launch_tc_gate_up(p, S, p.xg, st));
    MOE_TRY(record_mark(marks, n_marks, 3, st));
    MOE_TRY(launch_tc_down(p, S, st));
    MOE_TRY(record_mark(marks, n_marks, 4, st));
    return MOE_OK;
  }
  const bool tma = tma_gemv_supported(p) && scales_aligned16(p.routed) &&
                   (!p.has_shared || scales_aligned16(p.shared));
  if (tma) {
    MOE_TRY(launch_tma_gate_up(p, st, true));
    MOE_TRY(record_mark(marks, n_marks, 3, st));
    MOE_TRY(launch_tma_down(p, st, true));
  } else {
    MOE_TRY(launch_gemv_gate_up(p, st));
    MOE_TRY(record_mark(marks, n_marks, 3, st));
    MOE_TRY(launch_gemv_down(p, st));
  }
  MOE_TRY(record_mark(marks, n_marks, 4, st));
  return MOE_OK;
}

// Routing (+ the plan when the fused kernel applies). Returns whether the plan is done.
moe_status run_route(const Plan& p, cudaStream_t st, bool* plan_done) {
  if (route_fused_supported(p)) {
    MOE_TRY(launch_route_fused(p, p.ticket, st));
    *plan_done = true;
  } else {
    MOE_TRY(launch_router(p, st));
    MOE_TRY(launch_topk(p, st));
    *plan_done = false;
  }
  return MOE_OK;
}

}  // namespace

extern "C" {

int32_t moe_abi_version(void) { return MOE_ABI_VERSION; }

const char* moe_status_str(int32_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape or format";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_TIMEOUT: return "device-side wait timed out";
    case MOE_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case MOE_ERR_DEVICE: return "device-side check failed";
    case MOE_ERR_TOO_LARGE: return "request exceeds the library's built-in scratch buffer";
    default: return "unknown status";
  }
}

moe_status moe_validate(const moe_layer* L) { return validate(L); }

size_t moe_workspace_size(const moe_layer* L) {
  if (validate(L) != MOE_OK) return 0;
  return layout(L).total;
}

moe_status moe_route(const moe_layer* L, const void* x, int32_t* topk_idx, float* topk_w,
                     void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status s = validate(L);
  if (s != MOE_OK) return s;
  if (!x || !aligned(x, 16) || !topk_idx || !topk_w || !aligned(topk_idx, 4) ||
      !aligned(topk_w, 4))
    return MOE_ERR_INVALID_ARG;
  if ((s = check_ws(L, ws, ws_bytes)) != MOE_OK) return s;
  Plan p = make_plan(L, ws);
  p.x = static_cast<const uint16_t*>(x);
  p.topk_idx = topk_idx;
  p.topk_w = topk_w;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  bool plan_done = false;
  return run_route(p, st, &plan_done);
}

moe_status moe_permute(const moe_layer* L, const int32_t* topk_idx, int32_t* expert_offsets,
                       int32_t* perm, int32_t* inv, void* ws, size_t ws_bytes,
                       moe_stream_t stream) {
  moe_status s = validate(L);
  if (s != MOE_OK) return s;
  if (!topk_idx || !expert_offsets || !perm || !inv || !aligned(topk_idx, 4) ||
      !aligned(expert_offsets, 4) || !aligned(perm, 4) || !aligned(inv, 4))
    return MOE_ERR_INVALID_ARG;
  if ((s = check_ws(L, ws, ws_bytes)) != MOE_OK) return s;
  Plan p = make_plan(L, ws);
  p.topk_idx = const_cast<int32_t*>(topk_idx);
  p.offsets = expert_offsets;
  p.perm = perm;
  p.inv = inv;
  MOE_TRY(launch_permute(p, reinterpret_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_grouped_ffn(const moe_layer* L, const void* x, const int32_t* expert_offsets,
                           const int32_t* perm, float* y_assign, float* y_shared, void* ws,
                           size_t ws_bytes, moe_stream_t stream) {
  moe_status s = validate(L);
  if (s != MOE_OK) return s;
  if (!x || !aligned(x, 16) || !expert_offsets || !perm || !y_assign || !aligned(y_assign, 16))
    return MOE_ERR_INVALID_ARG;
  if (L->shared.n_exp && (!y_shared || !aligned(y_shared, 16))) return MOE_ERR_INVALID_ARG;
  if ((s = check_ws(L, ws, ws_bytes)) != MOE_OK) return s;
  Plan p = make_plan(L, ws);
  p.x = static_cast<const uint16_t*>(x);
  p.offsets = const_cast<int32_t*>(expert_offsets);
  p.perm = const_cast<int32_t*>(perm);
  p.y_assign = y_assign;
  if (y_shared) p.y_shared = y_shared;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  MOE_TRY(launch_schedule_from_offsets(p, st));
  return run_ffn(p, st, nullptr, 0);
}

moe_status moe_combine(const moe_layer* L, const float* y_assign, const float* y_shared,
                       const int32_t* inv, const float* topk_w, void* out,
                       moe_stream_t stream) {
  moe_status s = validate(L);
  if (s != MOE_OK) return s;
  if (!y_assign || !aligned(y_assign, 16) || !inv || !topk_w || !out || !aligned(out, 16))
    return MOE_ERR_INVALID_ARG;
  if (L->shared.n_exp && (!y_shared || !aligned(y_shared, 16))) return MOE_ERR_INVALID_ARG;
  Plan p{};
  p.T = L->T;
  p.d = L->d;
  p.k = L->k;
  p.has_shared = L->shared.n_exp;
  p.y_assign = const_cast<float*>(y_assign);
  p.y_shared = const_cast<float*>(y_shared);
  p.inv = const_cast<int32_t*>(inv);
  p.topk_w = const_cast<float*>(topk_w);
  MOE_TRY(launch_combine(p, out, reinterpret_cast<cudaStream_t>(stream), false));
  return MOE_OK;
}

moe_status moe_layer_forward_marked(const moe_layer* L, const void* x, void* out,
                                    int32_t* topk_idx, float* topk_w, int32_t* expert_offsets,
                                    int32_t* perm, void* ws, size_t ws_bytes,
                                    moe_stream_t stream, void* const* marks, int32_t n_marks) {
  moe_status s = validate(L);
  if (s != MOE_OK) return s;
  if (!x || !aligned(x, 16) || !out || !aligned(out, 16)) return MOE_ERR_INVALID_ARG;
  if ((topk_idx && !aligned(topk_idx, 4)) || (topk_w && !aligned(topk_w, 4)) ||
      (expert_offsets && !aligned(expert_offsets, 4)) || (perm && !aligned(perm, 4)))
    return MOE_ERR_INVALID_ARG;
  if (n_marks < 0 || (n_marks > 0 && !marks)) return MOE_ERR_INVALID_ARG;
  if ((s = check_ws(L, ws, ws_bytes)) != MOE_OK) return s;
  Plan p = make_plan(L, ws);
  p.x = static_cast<const uint16_t*>(x);
  if (topk_idx) p.topk_idx = topk_idx;
  if (topk_w) p.topk_w = topk_w;
  if (expert_offsets) p.offsets = expert_offsets;
  if (perm) p.perm = perm;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  auto mark = [&](int i) -> cudaError_t { return record_mark(marks, n_marks, i, st); };
  MOE_TRY(mark(0));
  if (use_fused(p)) {
    // one kernel: every stage mark after it
    MOE_TRY(launch_decode_fused(p, out, st));
    for (int i = 1; i < MOE_N_MARKS; ++i) MOE_TRY(mark(i));
    return MOE_OK;
  }
  if (p.path == MOE_PATH_FUSED) return MOE_ERR_UNSUPPORTED;
  bool plan_done = false;
  if ((s = run_route(p, st, &plan_done)) != MOE_OK) return s;
  MOE_TRY(mark(1));
  if (!plan_done) MOE_TRY(launch_permute(p, st));
  MOE_TRY(mark(2));
  if ((s = run_ffn(p, st, marks, n_marks)) != MOE_OK) return s;
  MOE_TRY(launch_combine(p, out, st, true));
  MOE_TRY(mark(5));
  return MOE_OK;
}

moe_status moe_layer_forward(const moe_layer* L, const void* x, void* out, int32_t* topk_idx,
                             float* topk_w, int32_t* expert_offsets, int32_t* perm, void* ws,
                             size_t ws_bytes, moe_stream_t stream) {
  return moe_layer_forward_marked(L, x, out, topk_idx, topk_w, expert_offsets, perm, ws,
                                  ws_bytes, stream, nullptr, 0);
}

int32_t moe_launches_per_call(const moe_layer* L) {
  if (validate(L) != MOE_OK) return 0;
  Plan p{};
  p.T = L->T;
  p.E = L->E;
  p.k = L->k;
  p.path = L->path;
  p.d = L->d;
  p.f = L->f;
  p.has_shared = L->shared.n_exp;
  p.routed.fmt = L->routed.fmt;
  p.shared.fmt = L->shared.fmt;
  for (int i = 0; i < 3; ++i) {
    p.routed.s[i] = static_cast<const uint16_t*>(i == 0 ? L->routed.s_gate : i == 1 ? L->routed.s_up : L->routed.s_down);
    p.shared.s[i] = static_cast<const uint16_t*>(i == 0 ? L->shared.s_gate : i == 1 ? L->shared.s_up : L->shared.s_down);
  }
  if (use_fused(p)) return 1;
  const int route = route_fused_supported(p) ? 1 : (2 + (L->T * L->k <= 1024 ? 1 : 3));
  if (L->routed.fmt == MOE_W_NVFP4)  // prep, quantise x, gate/up, quantise h, down (+ shared)
    return route + 5 + (p.has_shared ? 2 : 0) + 1;
  int ffn = use_tc(p) ? 3 : 2;  // (+ gather/schedule) gate/up, down
  if (p.has_shared && p.shared.fmt != p.routed.fmt) ffn += 2;  // each GEMM once per bank
  return route + ffn + 1;       // + combine
}

moe_status moe_test_inject_hold(const moe_layer* L, void* ws, size_t ws_bytes, int32_t hold,
                                int32_t budget_cycles, moe_stream_t stream) {
  moe_status s = validate(L);
  if (s != MOE_OK) return s;
  if (budget_cycles < 0) return MOE_ERR_INVALID_ARG;
  if ((s = check_ws(L, ws, ws_bytes)) != MOE_OK) return s;
  int32_t* dev = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + layout(L).status + kSyncTest);
  const int32_t words[2] = {hold ? 1 : 0, budget_cycles};
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // pageable source: the call returns once the words are staged, so a stack array is fine
  MOE_TRY(cudaMemcpyAsync(dev, words, sizeof(words), cudaMemcpyHostToDevice, st));
  return MOE_OK;
}

moe_status moe_nvfp4_pack_scales(const void* src, void* dst, int32_t n_mats, int32_t rows,
                                 int32_t K, moe_stream_t stream) {
  if (!src || !dst || !aligned(src, 16) || !aligned(dst, 16)) return MOE_ERR_INVALID_ARG;
  if (n_mats < 1 || rows < 128 || rows % 128 || K < 64 || K % 64) return MOE_ERR_INVALID_ARG;
  const size_t bytes = (size_t)n_mats * rows * (K / 16);
  const uint8_t* a = static_cast<const uint8_t*>(src);
  const uint8_t* b = static_cast<const uint8_t*>(dst);
  if (a < b + bytes && b < a + bytes) return MOE_ERR_INVALID_ARG;  // overlap
  MOE_TRY(launch_nv_pack_scales(a, static_cast<uint8_t*>(dst), n_mats, rows, K,
                                reinterpret_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_nvfp4_quantize_rows(const float* v, int32_t rows, int32_t K, void* codes,
                                   void* scales, float* g, moe_stream_t stream) {
  if (!v || !codes || !scales || !g) return MOE_ERR_INVALID_ARG;
  if (!aligned(v, 16) || !aligned(codes, 16) || !aligned(scales, 16) || !aligned(g, 4))
    return MOE_ERR_INVALID_ARG;
  if (rows < 1 || K < 16 || K % 16 || K > 8192) return MOE_ERR_INVALID_ARG;
  MOE_TRY(launch_nv_quant_rows(v, rows, K, static_cast<uint8_t*>(codes),
                               static_cast<uint8_t*>(scales), g,
                               reinterpret_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_device_wait_site(const moe_layer* L, void* ws, size_t ws_bytes, int32_t* site,
                                moe_stream_t stream) {
  moe_status s = validate(L);
  if (s != MOE_OK) return s;
  if (!site) return MOE_ERR_INVALID_ARG;
  if ((s = check_ws(L, ws, ws_bytes)) != MOE_OK) return s;
  int32_t* dev = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + layout(L).status) + kSiteWord;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t h = 0;
  MOE_TRY(cudaMemcpyAsync(&h, dev, sizeof(int32_t), cudaMemcpyDeviceToHost, st));
  MOE_TRY(cudaStreamSynchronize(st));
  MOE_TRY(cudaMemsetAsync(dev, 0, sizeof(int32_t), st));
  *site = h;
  return MOE_OK;
}

moe_status moe_device_status(const moe_layer* L, void* ws, size_t ws_bytes, int32_t* code,
                             moe_stream_t stream) {
  moe_status s = validate(L);
  if (s != MOE_OK) return s;
  if (!code) return MOE_ERR_INVALID_ARG;
  if ((s = check_ws(L, ws, ws_bytes)) != MOE_OK) return s;
  int32_t* dev = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + layout(L).status);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t h = 0;
  MOE_TRY(cudaMemcpyAsync(&h, dev, sizeof(int32_t), cudaMemcpyDeviceToHost, st));
  MOE_TRY(cudaStreamSynchronize(st));
  MOE_TRY(cudaMemsetAsync(dev, 0, sizeof(int32_t), st));
  *code = (h == DEV_OK) ? MOE_OK : (h == DEV_TIMEOUT ? MOE_ERR_TIMEOUT : MOE_ERR_DEVICE);
  return MOE_OK;
}

}  // extern "C"
