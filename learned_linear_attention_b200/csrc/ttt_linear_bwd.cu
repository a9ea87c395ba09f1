// ttt_linear_bwd.cu -- backward pass of the linear fast-weight layer.
//
// "Test-Time Training with KV Binding Is Secretly Linear Attention" (summary
// "B. Reformulación Teórica"): the layer is causal linear attention,
//   S_t = S0 + sum_{s <= t} eta_s k_s v_s^T,   o_t = S_t^T q_t
// (S_{t-1} with the exclusive diagonal).  For the scalar
// L = sum_t <dout_t, o_t> + <dS_end, S_end>, with
//   R_s = dS_end + sum over the reads t that see token s of q_t dout_t^T
//       = R_tot - sum over the other reads t of q_t dout_t^T,
//   R_tot = dS_end + sum_t q_t dout_t^T,
// the gradients are
//   dq_t = S_t dout_t,  dk_s = eta_s R_s v_s,  dv_s = eta_s R_s^T k_s,
//   dlr_s = v_s . (R_s^T k_s),  dS0 = R_tot.
// Every one of them is a forward-time causal scan of the same form as the
// layer itself, with the roles of q, k, v and dout exchanged:
//   R_tot:      keys q,    values dout, lr = 1, start dS_end   (its end state)
//   -R_s v_s:   queries v, keys dout,  values q,    lr = 1, start -R_tot^T
//   -R_s^T k_s: queries k, keys q,     values dout, lr = 1, start -R_tot
//   dq:         queries dout, keys v,  values k,    lr,     start S0^T
// with the opposite diagonal for the two R_s scans (a read that sees token s
// is one that the scan leaves out).  So the forward kernels do all the
// token work (R_tot, an end state only, comes from the state pre-pass on
// tensor cores); the dk scan scales its output rows by -lr, and two small
// kernels prepare the start states and finish dv and dlr.
#include "../../include/ttt.h"
#include "kernels.h"

namespace ttt {

namespace {

constexpr int EW_THREADS = 256;

__global__ void lin_bwd_fill_kernel(float* p, size_t n, float value) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    p[i] = value;
}

// R_tot [BH][dk][dv] -> -R_tot^T [BH][dv][dk], -R_tot, S0^T (zeros if S0 is
// null) and dS0 = R_tot.
__global__ void lin_bwd_states_kernel(const float* __restrict__ R, const float* __restrict__ S0,
                                      float* __restrict__ neg_rt, float* __restrict__ neg_r,
                                      float* __restrict__ s0t, float* __restrict__ dS0, int BH,
                                      int dk, int dv) {
  const size_t per = (size_t)dk * dv, n = (size_t)BH * per;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (size_t)gridDim.x * blockDim.x) {
    const size_t bh = e / per, r = e % per;
    const size_t i = r / dv, j = r % dv;        // element (i, j) of a [dk][dv] matrix
    const size_t et = bh * per + j * dk + i;    // element (j, i) of a [dv][dk] matrix
    const float x = R[e];
    neg_rt[et] = -x;
    neg_r[e] = -x;
    s0t[et] = S0 ? S0[e] : 0.f;
    dS0[e] = x;
  }
}

template <typename TV>
__device__ __forceinline__ float load_f(const TV* p, size_t i);
template <>
__device__ __forceinline__ float load_f<float>(const float* p, size_t i) { return p[i]; }
template <>
__device__ __forceinline__ float load_f<__nv_bfloat16>(const __nv_bfloat16* p, size_t i) {
  return __bfloat162float(p[i]);
}

// One warp per token row.  The scan gave w = -R_s^T k_s = -u in dv:
// dlr = v . u,  dv <- eta * u.  (dk comes out of its scan already scaled.)
template <typename TV>
__global__ void lin_bwd_finish_kernel(const float* __restrict__ lr, const TV* __restrict__ v,
                                      float* __restrict__ dv, float* __restrict__ dlr, size_t rows,
                                      int dv_dim) {
  const int lane = threadIdx.x & 31;
  const size_t warps = (size_t)gridDim.x * (blockDim.x >> 5);
  for (size_t row = (size_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < rows;
       row += warps) {
    const float eta = lr[row];
    float* dvr = dv + row * dv_dim;
    float dot = 0.f;
    if (dv_dim == 64) {   // two adjacent columns per lane, one pass
      float2 w = reinterpret_cast<float2*>(dvr)[lane];
      float v0, v1;
      if constexpr (sizeof(TV) == 2) {
        const __nv_bfloat162 b = reinterpret_cast<const __nv_bfloat162*>(v + row * 64)[lane];
        v0 = __low2float(b);
        v1 = __high2float(b);
      } else {
        const float2 f = reinterpret_cast<const float2*>(v + row * 64)[lane];
        v0 = f.x;
        v1 = f.y;
      }
      dot = -(v0 * w.x + v1 * w.y);
      reinterpret_cast<float2*>(dvr)[lane] = make_float2(-eta * w.x, -eta * w.y);
    } else {
      for (int c = lane; c < dv_dim; c += 32) {
        const float u = -dvr[c];
        dot = fmaf(load_f(v, row * dv_dim + c), u, dot);
        dvr[c] = eta * u;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    if (lane == 0) dlr[row] = dot;
  }
}

unsigned ew_grid(size_t n, int per_block) {
  const size_t b = (n + per_block - 1) / per_block;
  return (unsigned)(b < 1 ? 1 : (b > 148 * 16 ? 148 * 16 : b));
}

}  // namespace

LinearBwdWorkspace ttt_linear_bwd_layout(int BH, int N, int dk, int dv, size_t seg_floats) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  LinearBwdWorkspace w{};
  size_t o = 0;
  w.status = o; o = up(o + TTT_STATUS_BYTES);
  w.ones = o; o = up(o + (size_t)BH * N * sizeof(float));
  const size_t st = (size_t)BH * dk * dv * sizeof(float);
  w.r = o; o = up(o + st);
  w.neg_rt = o; o = up(o + st);
  w.neg_r = o; o = up(o + st);
  w.s0t = o; o = up(o + st);
  w.seg = o;
  w.seg_floats = seg_floats;
  o = up(o + w.seg_floats * sizeof(float));
  w.total = o;
  return w;
}

int launch_ttt_linear_bwd(const LinearBwdLaunch& L, cudaStream_t stream) {
  const int BH = L.B * L.H;
  const size_t rows = (size_t)BH * L.N, st_elems = (size_t)BH * L.dk * L.dv;
  const LinearBwdWorkspace& w = L.w;
  float* ones = reinterpret_cast<float*>(L.ws + w.ones);
  float* R = reinterpret_cast<float*>(L.ws + w.r);
  float* neg_rt = reinterpret_cast<float*>(L.ws + w.neg_rt);
  float* neg_r = reinterpret_cast<float*>(L.ws + w.neg_r);
  float* s0t = reinterpret_cast<float*>(L.ws + w.s0t);
  float* seg = reinterpret_cast<float*>(L.ws + w.seg);

  // R_tot starts from dS_end
  if (L.dS_end) {
    if (cudaMemcpyAsync(R, L.dS_end, st_elems * sizeof(float), cudaMemcpyDeviceToDevice, stream) !=
        cudaSuccess)
      return -1;
  } else if (cudaMemsetAsync(R, 0, st_elems * sizeof(float), stream) != cudaSuccess) {
    return -1;
  }
  if (L.N == 0) {   // dS0 = dS_end; nothing else to write
    return cudaMemcpyAsync(L.gS0, R, st_elems * sizeof(float), cudaMemcpyDeviceToDevice, stream) ==
                   cudaSuccess
               ? 0
               : -1;
  }
  prof_before(K_LIN_BWD_EW, stream);
  lin_bwd_fill_kernel<<<ew_grid(rows, EW_THREADS), EW_THREADS, 0, stream>>>(ones, rows, 1.f);
  prof_after(K_LIN_BWD_EW, stream);

  // one forward scan; dims are those of its (query/key, value) operands
  auto scan = [&](const void* q, const void* k, const void* v, const float* lr, float* S,
                  float* out, int dkk, int dvv, int include_diag, const float* out_scale) -> int {
    LinearLaunch F{};
    F.B = L.B; F.H = L.H; F.N = L.N; F.dk = dkk; F.dv = dvv; F.chunk = L.chunk;
    F.include_diag = include_diag;
    F.in_bf16 = L.in_bf16;
    F.out_bf16 = 0;
    F.q = q; F.k = k; F.v = v; F.lr = lr; F.S = S; F.out = out;
    F.st = L.st;
    F.out_scale = out_scale;
    F.out_mul = -1.f;
    if (L.umma) {
      F.plan = L.plan;
      F.seg_state = seg;
      F.seg_state_floats = w.seg_floats;
      return launch_ttt_linear_umma(F, stream);
    }
    return launch_ttt_linear_simt(F, stream);
  };
  const int inc = L.include_diag ? 1 : 0;
  // R_tot = dS_end + sum_t q_t dout_t^T: on tensor cores the state-only
  // pre-pass over the whole sequence; otherwise the end state of a scan with
  // keys q and values dout, whose outputs land in dv (a later scan
  // overwrites them)
  if (L.umma) {
    LinearLaunch F{};
    F.B = L.B; F.H = L.H; F.N = L.N; F.dk = L.dk; F.dv = L.dv;
    F.k = L.q; F.v = L.dout; F.lr = ones; F.S = R;
    F.st = L.st;
    F.seg_state = seg;
    F.seg_state_floats = w.seg_floats;
    if (launch_ttt_linear_state_sum(F, L.sms, stream)) return -1;
  } else if (scan(L.q, L.q, L.dout, ones, R, L.gv, L.dk, L.dv, 1, nullptr)) {
    return -1;
  }
  prof_before(K_LIN_BWD_EW, stream);
  lin_bwd_states_kernel<<<ew_grid(st_elems, EW_THREADS), EW_THREADS, 0, stream>>>(
      R, L.S0, neg_rt, neg_r, s0t, L.gS0, BH, L.dk, L.dv);
  prof_after(K_LIN_BWD_EW, stream);
  // dk_s = eta_s R_s v_s: the scan (queries v, keys dout, values q; state
  // [dv][dk]) gives -R_s v_s and scales its rows by -eta_s
  if (scan(L.v, L.dout, L.q, ones, neg_rt, L.gk, L.dv, L.dk, 1 - inc, L.lr)) return -1;
  // -R_s^T k_s -> dv (queries k, keys q, values dout; state [dk][dv])
  if (scan(L.k, L.q, L.dout, ones, neg_r, L.gv, L.dk, L.dv, 1 - inc, nullptr)) return -1;
  // dq_t = S_t dout_t (queries dout, keys v, values k, lr; state S0^T [dv][dk])
  if (scan(L.dout, L.v, L.k, L.lr, s0t, L.gq, L.dv, L.dk, inc, nullptr)) return -1;
  prof_before(K_LIN_BWD_EW, stream);
  const unsigned g = ew_grid(rows, EW_THREADS / 32);
  if (L.in_bf16)
    lin_bwd_finish_kernel<<<g, EW_THREADS, 0, stream>>>(
        L.lr, static_cast<const __nv_bfloat16*>(L.v), L.gv, L.glr, rows, L.dv);
  else
    lin_bwd_finish_kernel<<<g, EW_THREADS, 0, stream>>>(
        L.lr, static_cast<const float*>(L.v), L.gv, L.glr, rows, L.dv);
  prof_after(K_LIN_BWD_EW, stream);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace ttt
