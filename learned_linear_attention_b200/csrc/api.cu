// api.cu -- the C ABI (include/ttt.h): host-side validation, workspace
// sizing, state copies and kernel dispatch.
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>

#include <algorithm>

#include "../../include/ttt.h"
#include "kernels.h"

using namespace ttt;

namespace {

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;  // 2 s per wait

uint64_t wait_timeout_ns() {
  static uint64_t v = 0;
  if (v == 0) {
    const char* e = getenv("TTT_WAIT_TIMEOUT_MS");
    v = (e && atoll(e) > 0) ? (uint64_t)atoll(e) * 1000000ull : kDefaultTimeoutNs;
  }
  return v;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

DevStatus status_of(void* ws, uint32_t kernel_id) {
  DevStatus st;
  st.word = reinterpret_cast<uint32_t*>(ws);
  st.timeout_ns = wait_timeout_ns();
  st.kernel_id = kernel_id;
  return st;
}

int cuda_ok(cudaError_t e) { return e == cudaSuccess ? TTT_OK : TTT_ERR_CUDA; }

int check_linear(const ttt_linear_desc* d) {
  if (!d) return TTT_ERR_ARG;
  if (d->B < 1 || d->H < 1 || d->N < 0 || d->dk < 1 || d->dv < 1) return TTT_ERR_SHAPE;
  if (d->chunk < 1) return TTT_ERR_ARG;
  if (d->order != TTT_CAUSAL && d->order != TTT_BIDIRECTIONAL) return TTT_ERR_ARG;
  if ((d->in_dtype != TTT_F32 && d->in_dtype != TTT_BF16) ||
      (d->out_dtype != TTT_F32 && d->out_dtype != TTT_BF16))
    return TTT_ERR_DTYPE;
  if (d->dk > 128 || d->dv > 128) return TTT_ERR_UNSUPPORTED;
  return TTT_OK;
}

int check_lact(const lact_desc* d) {
  if (!d) return TTT_ERR_ARG;
  if (d->B < 1 || d->H < 1 || d->N_in < 0 || d->N_q < 0) return TTT_ERR_SHAPE;
  if (d->chunk < 1) return TTT_ERR_ARG;
  if (d->order != TTT_CAUSAL && d->order != TTT_BIDIRECTIONAL) return TTT_ERR_ARG;
  if (d->opt != TTT_OPT_GD && d->opt != TTT_OPT_MOMENTUM && d->opt != TTT_OPT_MUON)
    return TTT_ERR_ARG;
  if (d->order == TTT_CAUSAL && d->N_q != d->N_in) return TTT_ERR_SHAPE;
  if (d->update_mask < 1 || d->update_mask > 7) return TTT_ERR_ARG;
  if (d->opt == TTT_OPT_MUON && d->ns_steps < 0) return TTT_ERR_ARG;
  if (d->in_dtype != TTT_BF16) return TTT_ERR_DTYPE;
  if (d->out_dtype != TTT_F32 && d->out_dtype != TTT_BF16) return TTT_ERR_DTYPE;
  if (d->d < 128 || d->dh < 128 || d->d % 128 != 0 || d->dh % 128 != 0 || d->d > 1024 ||
      d->dh > 1024)
    return TTT_ERR_UNSUPPORTED;
  const long long rows = (long long)d->B * d->H * std::max(d->N_in, d->N_q);
  if (rows > (1ll << 31)) return TTT_ERR_SHAPE;
  return TTT_OK;
}

LactWorkspace layout_of(const lact_desc* d, int allow_parallel) {
  return lact_workspace_layout(d->B, d->H, d->N_in, d->N_q, d->d, d->dh, d->chunk,
                               d->order == TTT_CAUSAL, (int)d->opt, d->split_operands ? 1 : 0,
                               d->update_mask, d->normalize_rows, allow_parallel);
}

size_t lact_state_elems(const lact_desc* d) {
  const size_t per = (size_t)d->B * d->H * d->d * d->dh;
  return per * (d->opt == TTT_OPT_GD ? 3 : 6);
}

}  // namespace

extern "C" {

const char* ttt_status_string(int s) {
  switch (s) {
    case TTT_OK: return "TTT_OK";
    case TTT_ERR_ARG: return "TTT_ERR_ARG";
    case TTT_ERR_SHAPE: return "TTT_ERR_SHAPE";
    case TTT_ERR_ALIGN: return "TTT_ERR_ALIGN";
    case TTT_ERR_DTYPE: return "TTT_ERR_DTYPE";
    case TTT_ERR_UNSUPPORTED: return "TTT_ERR_UNSUPPORTED";
    case TTT_ERR_WORKSPACE: return "TTT_ERR_WORKSPACE";
    case TTT_ERR_CUDA: return "TTT_ERR_CUDA";
    case TTT_ERR_TIMEOUT: return "TTT_ERR_TIMEOUT";
    default: return "TTT_ERR_UNKNOWN";
  }
}

const char* ttt_build_info(void) {
  static char buf[128];
  snprintf(buf, sizeof(buf), "libttt_b200 sm_100a nvcc %d.%d", __CUDACC_VER_MAJOR__,
           __CUDACC_VER_MINOR__);
  return buf;
}

// ------------------------------------------------------------------ linear
static int device_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
    cudaGetLastError();
    sms = 148;
  }
  return sms;
}
static bool linear_uses_umma(const ttt_linear_desc* d) {
  return d->in_dtype == TTT_BF16 && d->dk == 64 && d->dv == 64;
}

int ttt_linear_workspace_bytes(const ttt_linear_desc* d, size_t* bytes) {
  int e = check_linear(d);
  if (e) return e;
  if (!bytes) return TTT_ERR_ARG;
  size_t seg = 0;
  if (linear_uses_umma(d))
    seg = (d->order == TTT_BIDIRECTIONAL
               ? ttt_linear_state_sum_floats(d->B * d->H, d->N, device_sms())
               : ttt_linear_plan(d->B * d->H, d->N, device_sms()).ws_floats) *
          sizeof(float);
  *bytes = TTT_STATUS_BYTES + seg;
  return TTT_OK;
}

int ttt_linear_state_init(const ttt_linear_desc* d, const float* S0, float* S, void* stream) {
  int e = check_linear(d);
  if (e) return e;
  if (!S) return TTT_ERR_ARG;
  const size_t bytes = (size_t)d->B * d->H * d->dk * d->dv * sizeof(float);
  if (S0) return cuda_ok(cudaMemcpyAsync(S, S0, bytes, cudaMemcpyDefault, as_stream(stream)));
  return cuda_ok(cudaMemsetAsync(S, 0, bytes, as_stream(stream)));
}

int ttt_linear_state_readout(const ttt_linear_desc* d, const float* S, float* dst, void* stream) {
  int e = check_linear(d);
  if (e) return e;
  if (!S || !dst) return TTT_ERR_ARG;
  const size_t bytes = (size_t)d->B * d->H * d->dk * d->dv * sizeof(float);
  return cuda_ok(cudaMemcpyAsync(dst, S, bytes, cudaMemcpyDefault, as_stream(stream)));
}

int ttt_linear_fwd(const ttt_linear_desc* d, const void* q, const void* k, const void* v,
                   const float* lr, float* S, void* out, void* ws, size_t ws_bytes, void* stream) {
  int e = check_linear(d);
  if (e) return e;
  if (!S || !ws) return TTT_ERR_ARG;
  if (ws_bytes < TTT_STATUS_BYTES) return TTT_ERR_WORKSPACE;
  if (d->N == 0) return TTT_OK;
  if (!q || !k || !v || !lr || !out) return TTT_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(lr) || !aligned16(S) ||
      !aligned16(out) || !aligned16(ws))
    return TTT_ERR_ALIGN;
  LinearLaunch L{};
  L.B = d->B; L.H = d->H; L.N = d->N; L.dk = d->dk; L.dv = d->dv; L.chunk = d->chunk;
  L.include_diag = d->include_diag ? 1 : 0;
  L.bidir = d->order == TTT_BIDIRECTIONAL ? 1 : 0;
  L.in_bf16 = d->in_dtype == TTT_BF16;
  L.out_bf16 = d->out_dtype == TTT_BF16;
  L.q = q; L.k = k; L.v = v; L.lr = lr; L.S = S; L.out = out;
  L.st = status_of(ws, 1);
  bool umma = linear_uses_umma(d);
  // the bidirectional tensor-core path needs the state pass's partial sums
  // in the workspace; with less it runs on CUDA cores
  if (umma && L.bidir &&
      ws_bytes - TTT_STATUS_BYTES <
          ttt_linear_state_sum_floats(d->B * d->H, d->N, device_sms()) * sizeof(float))
    umma = false;
  if (umma) {
    L.plan = ttt_linear_plan(d->B * d->H, d->N, device_sms());
    L.seg_state = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + TTT_STATUS_BYTES);
    L.seg_state_floats = (ws_bytes - TTT_STATUS_BYTES) / sizeof(float);
  }
  const int r = umma ? launch_ttt_linear_umma(L, as_stream(stream))
                     : launch_ttt_linear_simt(L, as_stream(stream));
  return r == 0 ? TTT_OK : TTT_ERR_CUDA;
}

LinearBwdWorkspace linear_bwd_layout(const ttt_linear_desc* d, LinearPlan* plan) {
  const int BH = d->B * d->H, sms = device_sms();
  size_t seg = 0;
  if (linear_uses_umma(d)) {
    *plan = ttt_linear_plan(BH, d->N, sms);
    seg = std::max(plan->ws_floats, ttt_linear_state_sum_floats(BH, d->N, sms));
  }
  return ttt_linear_bwd_layout(BH, d->N, d->dk, d->dv, seg);
}

int ttt_linear_bwd_workspace_bytes(const ttt_linear_desc* d, size_t* bytes) {
  int e = check_linear(d);
  if (e) return e;
  if (d->order != TTT_CAUSAL) return TTT_ERR_UNSUPPORTED;
  if (!bytes) return TTT_ERR_ARG;
  LinearPlan plan{};
  *bytes = linear_bwd_layout(d, &plan).total;
  return TTT_OK;
}

int ttt_linear_bwd(const ttt_linear_desc* d, const void* q, const void* k, const void* v,
                   const float* lr, const float* S0, const void* dout, const float* dS_end,
                   float* dq, float* dk, float* dv, float* dlr, float* dS0, void* ws,
                   size_t ws_bytes, void* stream) {
  int e = check_linear(d);
  if (e) return e;
  if (d->order != TTT_CAUSAL) return TTT_ERR_UNSUPPORTED;
  if (!ws || !dS0) return TTT_ERR_ARG;
  LinearPlan plan{};
  const LinearBwdWorkspace w = linear_bwd_layout(d, &plan);
  if (ws_bytes < w.total) return TTT_ERR_WORKSPACE;
  if (d->N > 0 && (!q || !k || !v || !lr || !dout || !dq || !dk || !dv || !dlr))
    return TTT_ERR_ARG;
  const void* ptrs[] = {q, k, v, lr, S0, dout, dS_end, dq, dk, dv, dlr, dS0, ws};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return TTT_ERR_ALIGN;
  LinearBwdLaunch L{};
  L.B = d->B; L.H = d->H; L.N = d->N; L.dk = d->dk; L.dv = d->dv; L.chunk = d->chunk;
  L.include_diag = d->include_diag ? 1 : 0;
  L.in_bf16 = d->in_dtype == TTT_BF16;
  L.umma = linear_uses_umma(d) ? 1 : 0;
  L.sms = device_sms();
  L.q = q; L.k = k; L.v = v; L.dout = dout; L.lr = lr; L.S0 = S0; L.dS_end = dS_end;
  L.gq = dq; L.gk = dk; L.gv = dv; L.glr = dlr; L.gS0 = dS0;
  L.ws = static_cast<uint8_t*>(ws);
  L.w = w;
  L.plan = plan;
  L.st = status_of(ws, 1);
  return launch_ttt_linear_bwd(L, as_stream(stream)) == 0 ? TTT_OK : TTT_ERR_CUDA;
}

// ------------------------------------------------------------------ window attention
static int check_window(const ttt_window_desc* d) {
  if (!d) return TTT_ERR_ARG;
  if (d->B < 1 || d->H < 1 || d->N < 0) return TTT_ERR_SHAPE;
  if (d->window < 1) return TTT_ERR_ARG;
  if (d->in_dtype != TTT_BF16) return TTT_ERR_DTYPE;
  if (d->out_dtype != TTT_F32 && d->out_dtype != TTT_BF16) return TTT_ERR_DTYPE;
  if (d->d != 128) return TTT_ERR_UNSUPPORTED;
  if ((long long)d->B * d->H * d->N > (1ll << 31)) return TTT_ERR_SHAPE;
  return TTT_OK;
}

static int run_window(const ttt_window_desc* d, const void* q, const void* k, const void* v,
                      void* out, void* ws, void* stream) {
  WindowAttnLaunch L{};
  L.B = d->B; L.H = d->H; L.N = d->N; L.window = d->window;
  L.scale = d->scale > 0.f ? d->scale : 1.f / sqrtf((float)d->d);
  L.out_bf16 = d->out_dtype == TTT_BF16;
  L.accumulate = d->accumulate ? 1 : 0;
  L.q = q; L.k = k; L.v = v; L.out = out;
  L.st = status_of(ws, 3);
  return launch_window_attention(L, as_stream(stream)) == 0 ? TTT_OK : TTT_ERR_CUDA;
}

int ttt_window_attn_fwd(const ttt_window_desc* d, const void* q, const void* k, const void* v,
                        void* out, void* ws, size_t ws_bytes, void* stream) {
  int e = check_window(d);
  if (e) return e;
  if (!ws) return TTT_ERR_ARG;
  if (ws_bytes < TTT_STATUS_BYTES) return TTT_ERR_WORKSPACE;
  if (d->N == 0) return TTT_OK;
  if (!q || !k || !v || !out) return TTT_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(ws))
    return TTT_ERR_ALIGN;
  return run_window(d, q, k, v, out, ws, stream);
}

// ------------------------------------------------------------------ LaCT
int lact_state_bytes(const lact_desc* d, size_t* bytes) {
  int e = check_lact(d);
  if (e) return e;
  if (!bytes) return TTT_ERR_ARG;
  *bytes = lact_state_elems(d) * sizeof(float);
  return TTT_OK;
}

int lact_workspace_bytes(const lact_desc* d, size_t* bytes) {
  int e = check_lact(d);
  if (e) return e;
  if (!bytes) return TTT_ERR_ARG;
  // the fastest form's layout, and never less than the chunk loop's, which
  // every call accepts (for short sequences the parallel form can be smaller)
  *bytes = std::max(layout_of(d, 1).total, layout_of(d, 0).total);
  return TTT_OK;
}

int lact_workspace_bytes_min(const lact_desc* d, size_t* bytes) {
  int e = check_lact(d);
  if (e) return e;
  if (!bytes) return TTT_ERR_ARG;
  *bytes = layout_of(d, 0).total;
  return TTT_OK;
}

int lact_state_init(const lact_desc* d, const float* W1, const float* W3, const float* W2,
                    int w_per_batch, void* state, void* stream) {
  int e = check_lact(d);
  if (e) return e;
  if (!W1 || !W3 || !W2 || !state) return TTT_ERR_ARG;
  cudaStream_t s = as_stream(stream);
  const size_t per_head = (size_t)d->d * d->dh;
  const size_t per_mat = (size_t)d->B * d->H * per_head;
  float* st = reinterpret_cast<float*>(state);
  const float* src[3] = {W1, W3, W2};
  for (int m = 0; m < 3; ++m) {
    float* dst = st + m * per_mat;
    if (w_per_batch) {
      e = cuda_ok(cudaMemcpyAsync(dst, src[m], per_mat * 4, cudaMemcpyDefault, s));
      if (e) return e;
    } else {
      for (int b = 0; b < d->B; ++b) {
        e = cuda_ok(cudaMemcpyAsync(dst + (size_t)b * d->H * per_head, src[m],
                                    (size_t)d->H * per_head * 4, cudaMemcpyDefault, s));
        if (e) return e;
      }
    }
  }
  if (d->opt != TTT_OPT_GD) return cuda_ok(cudaMemsetAsync(st + 3 * per_mat, 0, 3 * per_mat * 4, s));
  return TTT_OK;
}

int lact_state_readout(const lact_desc* d, const void* state, float* W1, float* W3, float* W2,
                       float* M, void* stream) {
  int e = check_lact(d);
  if (e) return e;
  if (!state || !W1 || !W3 || !W2) return TTT_ERR_ARG;
  cudaStream_t s = as_stream(stream);
  const size_t per_mat = (size_t)d->B * d->H * d->d * d->dh;
  const float* st = reinterpret_cast<const float*>(state);
  float* dst[3] = {W1, W3, W2};
  for (int m = 0; m < 3; ++m) {
    e = cuda_ok(cudaMemcpyAsync(dst[m], st + m * per_mat, per_mat * 4, cudaMemcpyDefault, s));
    if (e) return e;
  }
  if (M && d->opt != TTT_OPT_GD)
    return cuda_ok(cudaMemcpyAsync(M, st + 3 * per_mat, 3 * per_mat * 4, cudaMemcpyDefault, s));
  return TTT_OK;
}

int lact_chunk_fwd(const lact_desc* d, const void* q, const void* k, const void* v,
                   const float* lr, void* state, void* out, void* ws, size_t ws_bytes,
                   void* stream) {
  int e = check_lact(d);
  if (e) return e;
  if (!state || !ws) return TTT_ERR_ARG;
  // the smallest workspace runs the chunk loop; launch_lact takes the
  // parallel form of the W2-only layer when ws_bytes holds its layout
  if (ws_bytes < layout_of(d, 0).total) return TTT_ERR_WORKSPACE;
  const bool causal = d->order == TTT_CAUSAL;
  const int n_out = causal ? d->N_in : d->N_q;
  if (d->N_in > 0 && (!k || !v || !lr)) return TTT_ERR_ARG;
  if (n_out > 0 && (!q || !out)) return TTT_ERR_ARG;
  if ((k && !aligned16(k)) || (v && !aligned16(v)) || (q && !aligned16(q)) ||
      (lr && !aligned16(lr)) || (out && !aligned16(out)) || !aligned16(state) || !aligned16(ws))
    return TTT_ERR_ALIGN;
  if (d->N_in == 0 && n_out == 0) return TTT_OK;
  LactLaunch L{};
  L.B = d->B; L.H = d->H; L.N_in = d->N_in; L.N_q = causal ? d->N_in : d->N_q;
  L.d = d->d; L.dh = d->dh; L.chunk = d->chunk; L.causal = causal ? 1 : 0;
  L.opt = (int)d->opt; L.beta = d->beta; L.ns_steps = d->ns_steps;
  L.ns_a = d->ns_coef[0]; L.ns_b = d->ns_coef[1]; L.ns_c = d->ns_coef[2]; L.ns_eps = d->ns_eps;
  L.normalize_rows = d->normalize_rows ? 1 : 0; L.norm_eps = d->norm_eps;
  L.update_mask = d->update_mask; L.out_bf16 = d->out_dtype == TTT_BF16;
  L.split = d->split_operands ? 1 : 0;
  L.q = q; L.k = k; L.v = v; L.lr = lr;
  L.state = reinterpret_cast<float*>(state);
  L.out = out;
  L.ws = reinterpret_cast<uint8_t*>(ws);
  L.ws_bytes = ws_bytes;
  L.st = status_of(ws, 2);
  return launch_lact(L, as_stream(stream)) == 0 ? TTT_OK : TTT_ERR_CUDA;
}

// ------------------------------------------------------------------ context parallelism
static void fill_lact_launch(const lact_desc* d, LactLaunch& L) {
  const bool causal = d->order == TTT_CAUSAL;
  L.B = d->B; L.H = d->H; L.N_in = d->N_in; L.N_q = causal ? d->N_in : d->N_q;
  L.d = d->d; L.dh = d->dh; L.chunk = d->chunk; L.causal = causal ? 1 : 0;
  L.opt = (int)d->opt; L.beta = d->beta; L.ns_steps = d->ns_steps;
  L.ns_a = d->ns_coef[0]; L.ns_b = d->ns_coef[1]; L.ns_c = d->ns_coef[2]; L.ns_eps = d->ns_eps;
  L.normalize_rows = d->normalize_rows ? 1 : 0; L.norm_eps = d->norm_eps;
  L.update_mask = d->update_mask; L.out_bf16 = d->out_dtype == TTT_BF16;
  L.split = d->split_operands ? 1 : 0;
}

int lact_grad_bytes(const lact_desc* d, size_t* bytes) {
  int e = check_lact(d);
  if (e) return e;
  if (!bytes) return TTT_ERR_ARG;
  *bytes = 3 * (size_t)d->B * d->H * d->d * d->dh * sizeof(float);
  return TTT_OK;
}

int lact_chunk_grad(const lact_desc* d, int t0, int n, const void* k, const void* v,
                    const float* lr, const void* state, float* G, void* ws, size_t ws_bytes,
                    void* stream) {
  int e = check_lact(d);
  if (e) return e;
  if (!state || !G || !ws) return TTT_ERR_ARG;
  if (t0 < 0 || n < 0 || (long long)t0 + n > d->N_in || n > d->chunk) return TTT_ERR_SHAPE;
  if (ws_bytes < layout_of(d, 0).total) return TTT_ERR_WORKSPACE;
  if (n > 0 && (!k || !v || !lr)) return TTT_ERR_ARG;
  if ((k && !aligned16(k)) || (v && !aligned16(v)) || (lr && !aligned16(lr)) ||
      !aligned16(state) || !aligned16(G) || !aligned16(ws))
    return TTT_ERR_ALIGN;
  LactLaunch L{};
  fill_lact_launch(d, L);
  L.k = k; L.v = v; L.lr = lr;
  L.state = reinterpret_cast<float*>(const_cast<void*>(state));
  L.ws = reinterpret_cast<uint8_t*>(ws);
  L.ws_bytes = ws_bytes;
  L.st = status_of(ws, 2);
  L.mode = LACT_GRAD; L.t0 = t0; L.n = n; L.G = G;
  return launch_lact(L, as_stream(stream)) == 0 ? TTT_OK : TTT_ERR_CUDA;
}

int lact_apply_grad(const lact_desc* d, const float* G, void* state, void* ws, size_t ws_bytes,
                    void* stream) {
  int e = check_lact(d);
  if (e) return e;
  if (!state || !G || !ws) return TTT_ERR_ARG;
  if (ws_bytes < layout_of(d, 0).total) return TTT_ERR_WORKSPACE;
  if (!aligned16(state) || !aligned16(G) || !aligned16(ws)) return TTT_ERR_ALIGN;
  LactLaunch L{};
  fill_lact_launch(d, L);
  L.state = reinterpret_cast<float*>(state);
  L.ws = reinterpret_cast<uint8_t*>(ws);
  L.ws_bytes = ws_bytes;
  L.st = status_of(ws, 2);
  L.mode = LACT_APPLY; L.G = const_cast<float*>(G);
  return launch_lact(L, as_stream(stream)) == 0 ? TTT_OK : TTT_ERR_CUDA;
}

int lact_read(const lact_desc* d, int t0, int n, const void* q, const void* state, void* out,
              void* ws, size_t ws_bytes, void* stream) {
  int e = check_lact(d);
  if (e) return e;
  if (!state || !ws) return TTT_ERR_ARG;
  const int rows = d->order == TTT_CAUSAL ? d->N_in : d->N_q;
  if (t0 < 0 || n < 0 || (long long)t0 + n > rows) return TTT_ERR_SHAPE;
  if (ws_bytes < layout_of(d, 0).total) return TTT_ERR_WORKSPACE;
  if (n == 0) return TTT_OK;
  if (!q || !out) return TTT_ERR_ARG;
  if (!aligned16(q) || !aligned16(out) || !aligned16(state) || !aligned16(ws)) return TTT_ERR_ALIGN;
  // the read's intermediates hold at most one chunk (causal) or N_q rows
  if (n > layout_of(d, 0).cmax) return TTT_ERR_SHAPE;
  LactLaunch L{};
  fill_lact_launch(d, L);
  L.q = q;
  L.state = reinterpret_cast<float*>(const_cast<void*>(state));
  L.out = out;
  L.ws = reinterpret_cast<uint8_t*>(ws);
  L.ws_bytes = ws_bytes;
  L.st = status_of(ws, 2);
  L.mode = LACT_READ; L.t0 = t0; L.n = n;
  return launch_lact(L, as_stream(stream)) == 0 ? TTT_OK : TTT_ERR_CUDA;
}

// ------------------------------------------------------------------ LaCT backward
static int check_lact_bwd(const lact_desc* d) {
  int e = check_lact(d);
  if (e) return e;
  if (d->opt == TTT_OPT_MUON) return TTT_ERR_UNSUPPORTED;
  return TTT_OK;
}

int lact_bwd_workspace_bytes(const lact_desc* d, size_t* bytes) {
  int e = check_lact_bwd(d);
  if (e) return e;
  if (!bytes) return TTT_ERR_ARG;
  LactLaunch f{};
  fill_lact_launch(d, f);
  *bytes = lact_bwd_layout(f).total;
  return TTT_OK;
}

int lact_chunk_bwd(const lact_desc* d, const void* q, const void* k, const void* v,
                   const float* lr, const void* state0, const void* dout, const float* dW_end,
                   float* dq, float* dk, float* dv, float* dlr, float* dW0, void* ws,
                   size_t ws_bytes, void* stream) {
  int e = check_lact_bwd(d);
  if (e) return e;
  if (!state0 || !dW0 || !ws) return TTT_ERR_ARG;
  LactLaunch f{};
  fill_lact_launch(d, f);
  if (ws_bytes < lact_bwd_layout(f).total) return TTT_ERR_WORKSPACE;
  const int rows = d->order == TTT_CAUSAL ? d->N_in : d->N_q;
  if (d->N_in > 0 && (!k || !v || !lr || !dk || !dv || !dlr)) return TTT_ERR_ARG;
  if (rows > 0 && (!q || !dout || !dq)) return TTT_ERR_ARG;
  const void* ptrs[] = {q, k, v, lr, state0, dout, dW_end, dq, dk, dv, dlr, dW0, ws};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return TTT_ERR_ALIGN;
  f.q = q; f.k = k; f.v = v; f.lr = lr;
  f.st = status_of(ws, 4);
  LactBwdLaunch L{};
  L.f = f;
  L.W0 = reinterpret_cast<const float*>(state0);
  L.dout = dout; L.dW_end = dW_end;
  L.dq = dq; L.dk = dk; L.dv = dv; L.dlr = dlr; L.dW0 = dW0;
  L.ws = reinterpret_cast<uint8_t*>(ws);
  L.st = f.st;
  return launch_lact_bwd(L, as_stream(stream)) == 0 ? TTT_OK : TTT_ERR_CUDA;
}

int lact_layer_fwd(const lact_desc* d, int window, float scale, const void* q, const void* k,
                   const void* v, const float* lr, void* state, void* out, void* ws,
                   size_t ws_bytes, void* stream) {
  int e = check_lact(d);
  if (e) return e;
  if (d->order != TTT_CAUSAL) return TTT_ERR_ARG;
  ttt_window_desc wd{};
  wd.B = d->B; wd.H = d->H; wd.N = d->N_in; wd.d = d->d; wd.window = window; wd.scale = scale;
  wd.in_dtype = d->in_dtype; wd.out_dtype = d->out_dtype; wd.accumulate = 1;
  e = check_window(&wd);
  if (e) return e;
  e = lact_chunk_fwd(d, q, k, v, lr, state, out, ws, ws_bytes, stream);
  if (e || d->N_in == 0) return e;
  return run_window(&wd, q, k, v, out, ws, stream);
}

// ------------------------------------------------------------------ status
int ttt_check_device_status(void* ws, void* stream) {
  if (!ws) return TTT_ERR_ARG;
  cudaStream_t s = as_stream(stream);
  uint32_t h[4] = {0, 0, 0, 0};
  if (cudaStreamSynchronize(s) != cudaSuccess) return TTT_ERR_CUDA;
  if (cudaMemcpy(h, ws, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return TTT_ERR_CUDA;
  if (h[0] == DEV_OK) return TTT_OK;
  if (cudaMemset(ws, 0, sizeof(h)) != cudaSuccess) return TTT_ERR_CUDA;
  return h[0] == DEV_TIMEOUT ? TTT_ERR_TIMEOUT : TTT_ERR_CUDA;
}

int ttt_selftest_wait_timeout(void* ws, size_t ws_bytes, int timeout_us, void* stream) {
  if (!ws || timeout_us < 1 || timeout_us > 10000000) return TTT_ERR_ARG;
  if (ws_bytes < TTT_STATUS_BYTES) return TTT_ERR_WORKSPACE;
  DevStatus st = status_of(ws, 9);
  st.timeout_ns = (uint64_t)timeout_us * 1000ull;
  return launch_wait_timeout_probe(st, as_stream(stream)) == 0 ? TTT_OK : TTT_ERR_CUDA;
}

}  // extern "C"

// ------------------------------------------------------------------ probe kernel
namespace ttt {
// One CTA waits on an mbarrier whose phase never completes (nobody arrives);
// the bounded wait must give up, record DEV_TIMEOUT and let the CTA exit.
__global__ void wait_timeout_probe_kernel(DevStatus st) {
  __shared__ uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    Waiter W{&abort_flag, st, 900};
    (void)W.wait(&bar, 0, 0);
  }
  __syncthreads();
}

int launch_wait_timeout_probe(DevStatus st, cudaStream_t stream) {
  wait_timeout_probe_kernel<<<1, 32, 0, stream>>>(st);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}
}  // namespace ttt
