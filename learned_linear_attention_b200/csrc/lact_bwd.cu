// lact_bwd.cu -- backward pass of the LaCT layer through its chunk loop
// ("Test-Time Training Done Right" review: the layer is trained end to end,
// "Lenguaje: calidad y velocidad no son equivalentes" reports its training
// throughput with GD, momentum and Muon updates).
//
// Gradients of  L = sum <dout, out> + sum_m <dW_end[m], W_m(end)>  with
// respect to q, k, v, lr and the start weights W0 (GD and momentum, causal
// or bidirectional, with or without row normalisation, any update mask).
//
// 1. Forward replay, chunk by chunk, with the layer's own pieces (the chunk
//    gradient and the update of the context-parallel calls): it keeps every
//    chunk's start weights W_c and the row norms of the pre-normalisation
//    update U_c = W_c - (G_c or M_c).
// 2. Reverse over the chunks, per chunk c with upstream dW = dL/dW_{c+1}:
//      row step   dU = (dW - w <w, dW>) / |U| (w = W_{c+1} rows; dW / eps
//                 for a row whose norm was below eps; dU = dW without the
//                 normalisation); momentum: dM -= dU, R = dM, dM *= beta;
//                 GD: R = -dU; then dW = dU.  R = dL/dG_c.
//      chunk gradient VJP at W_c over the chunk's tokens (per token: h1 = W1 k,
//                 h3 = W3 k, a = silu(h1), s = silu'(h1), g = a h3,
//                 dy = -lr v, dg = W2^T dy; r1 = R1 k, r3 = R3 k, r2 = R2^T dy):
//                 d_h3 = r2 a + dg s r1,
//                 d_h1 = (r2 h3 + dg r3) s + dg h3 r1 silu''(h1),
//                 d_dg = a r3 + h3 s r1,
//                 dW1 += d_h1^T K, dW3 += d_h3^T K, dW2 += V^T (-lr d_dg),
//                 dk = d_h1 W1 + d_h3 W3 + (dg h3 s) R1 + (dg a) R3,
//                 d_dy = d_dg W2^T + g R2^T, dv = -lr d_dy, dlr = -v . d_dy;
//      causal read VJP at W_c for the chunk's queries (per query: hq1, hq3,
//                 aq = silu(hq1), gq = aq hq3, dgq = W2^T dout):
//                 dW1 += (dgq hq3 s)^T Q, dW3 += (dgq aq)^T Q,
//                 dW2 += dout^T gq, dq = (dgq hq3 s) W1 + (dgq aq) W3.
//    The bidirectional read VJP runs once, before the reverse loop, with the
//    final weights.  dW0 = dW after the first chunk.
// Every product is a batched tcgen05 GEMM (bf16 operands, fp32 accumulators)
// of gemm.cuh; the elementwise steps are the kernels below.
#include <algorithm>

#include "gemm.cuh"
#include "kernels.h"
#include "gemm_group.cuh"

namespace ttt {

namespace {

TTT_DEVICE_INLINE float sig(float x) { return 1.f / (1.f + __expf(-x)); }

int num_sms_bwd() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// bf16 copies of fp32 matrices (the GEMMs' weight and R operands)
__global__ void bwd_cast_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                                size_t n4) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (size_t)gridDim.x * blockDim.x) {
    const float4 x = reinterpret_cast<const float4*>(src)[i];
    reinterpret_cast<uint2*>(dst)[i] = make_uint2(pack_bf16x2(x.x, x.y), pack_bf16x2(x.z, x.w));
  }
}

struct RowStepArgs {
  int BH, d, dh, mask, normalize, momentum;
  float beta, norm_eps;
  float* dW;             // [3 mats][BH][rows][cols], in: dL/dW_{c+1}, out: dL/dU
  float* dM;             // momentum carry (momentum only)
  const float* Wn;       // W_{c+1}
  const float* rn;       // row norms of U_c, [BH][2 dh + d]
  float* R;              // out: dL/dG_c (fp32)
  __nv_bfloat16* Rb;     // out: bf16 copy
  const float* Wc;       // W_c (the chunk's start weights), cast to Wb alongside
  __nv_bfloat16* Wb;
  // nullable: the later chunk's split weight-gradient partials, added to dW
  // first ([BH][splits][rows][cols] per matrix, in split order)
  const float* part[3];
  int splits;
};
// One warp per row of one matrix of one head (rows of 128 to 1024 columns,
// a multiple of 128): each lane holds four-column slices of the row in
// registers across the two passes (projection onto W_{c+1}, then the step).
// The same warp writes the bf16 copy of the row of W_c the chunk's products
// read.
__global__ void bwd_row_step_kernel(RowStepArgs a) {
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  const int per = 2 * a.dh + a.d;
  if (gw >= a.BH * per) return;
  const int bh = gw / per, rr = gw % per;
  const int mat = rr < a.dh ? 0 : (rr < 2 * a.dh ? 1 : 2);
  const int row = mat == 0 ? rr : (mat == 1 ? rr - a.dh : rr - 2 * a.dh);
  const int rows = mat < 2 ? a.dh : a.d, cols = mat < 2 ? a.d : a.dh;
  const size_t mat_elems = (size_t)a.BH * a.d * a.dh;
  const size_t off = mat * mat_elems + ((size_t)bh * rows + row) * cols;
  const int nv = cols / 128;   // float4 slices per lane (<= 8)
  {
    const float4* wc = reinterpret_cast<const float4*>(a.Wc + off);
    uint2* wb = reinterpret_cast<uint2*>(a.Wb + off);
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (k < nv) {
        const float4 x = wc[k * 32 + lane];
        wb[k * 32 + lane] = make_uint2(pack_bf16x2(x.x, x.y), pack_bf16x2(x.z, x.w));
      }
  }
  float4* R4 = reinterpret_cast<float4*>(a.R + off);
  uint2* Rb2 = reinterpret_cast<uint2*>(a.Rb + off);
  float4* dW4 = reinterpret_cast<float4*>(a.dW + off);
  // dW of this chunk's end weights: the later chunk's partial products
  // still to be added (in split order, as a separate summing pass would)
  const float4* P4 = a.part[mat] != nullptr
                         ? reinterpret_cast<const float4*>(a.part[mat] + ((size_t)bh * a.splits * rows + row) * cols)
                         : nullptr;
  const size_t pstride4 = (size_t)rows * cols / 4;
  auto dw_in = [&](int k) {
    float4 u = dW4[k * 32 + lane];
    if (P4 != nullptr)
      for (int sp = 0; sp < a.splits; ++sp) {
        const float4 x = P4[sp * pstride4 + k * 32 + lane];
        u.x += x.x; u.y += x.y; u.z += x.z; u.w += x.w;
      }
    return u;
  };
  if (!(a.mask & (1 << mat))) {   // not updated: no dependence on G, dW passes through
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (k < nv) {
        if (P4 != nullptr) dW4[k * 32 + lane] = dw_in(k);
        R4[k * 32 + lane] = make_float4(0.f, 0.f, 0.f, 0.f);
        Rb2[k * 32 + lane] = make_uint2(0u, 0u);
      }
    return;
  }
  const float4* Wn4 = reinterpret_cast<const float4*>(a.Wn + off);
  float4 du[8], wn[8];
  float proj = 0.f, inv = 1.f;
  bool big = true;
#pragma unroll
  for (int k = 0; k < 8; ++k)
    if (k < nv) {
      du[k] = dw_in(k);
      if (a.normalize) {
        wn[k] = Wn4[k * 32 + lane];
        proj += wn[k].x * du[k].x + wn[k].y * du[k].y + wn[k].z * du[k].z + wn[k].w * du[k].w;
      }
    }
  if (a.normalize) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) proj += __shfl_xor_sync(0xffffffffu, proj, o);
    const float n = a.rn[gw];
    big = n > a.norm_eps;
    inv = 1.f / (big ? n : a.norm_eps);
  }
  float4* dM4 = reinterpret_cast<float4*>(a.dM + off);
#pragma unroll
  for (int k = 0; k < 8; ++k)
    if (k < nv) {
      float4 u = du[k];
      if (a.normalize) {
        if (big) {
          u.x = (u.x - wn[k].x * proj) * inv; u.y = (u.y - wn[k].y * proj) * inv;
          u.z = (u.z - wn[k].z * proj) * inv; u.w = (u.w - wn[k].w * proj) * inv;
        } else {
          u.x *= inv; u.y *= inv; u.z *= inv; u.w *= inv;
        }
      }
      float4 r;
      if (a.momentum) {
        const float4 m0 = dM4[k * 32 + lane];
        r = make_float4(m0.x - u.x, m0.y - u.y, m0.z - u.z, m0.w - u.w);
        dM4[k * 32 + lane] = make_float4(a.beta * r.x, a.beta * r.y, a.beta * r.z, a.beta * r.w);
      } else {
        r = make_float4(-u.x, -u.y, -u.z, -u.w);
      }
      dW4[k * 32 + lane] = u;
      R4[k * 32 + lane] = r;
      Rb2[k * 32 + lane] = make_uint2(pack_bf16x2(r.x, r.y), pack_bf16x2(r.z, r.w));
    }
}

struct KeyEwArgs {
  int BH, C, cmax, dh, lr_len, t0;
  const float* lr;       // [BH][lr_len]
  // fp32 [BH][cmax][dh]: K W1^T, K W3^T, V W2, K R1^T, K R3^T, V R2
  const float *h1, *h3, *vw2, *r1, *r3, *vr2;
  // bf16 [BH][cmax][dh] outputs
  __nv_bfloat16 *d_h1, *d_h3, *d_dg, *d_dgn, *e1, *e3, *g;
};
// The chunk gradient's elementwise VJP step; rows past the chunk are zero.
__global__ void bwd_key_ew_kernel(KeyEwArgs a) {
  const size_t n = (size_t)a.BH * a.cmax * a.dh;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    const size_t bh = i / ((size_t)a.cmax * a.dh);
    const int t = (int)((i / a.dh) % a.cmax);
    float vdh1 = 0.f, vdh3 = 0.f, vddg = 0.f, vddgn = 0.f, ve1 = 0.f, ve3 = 0.f, vg = 0.f;
    if (t < a.C) {
      const float eta = a.lr[bh * a.lr_len + a.t0 + t];
      const float x = a.h1[i], y = a.h3[i];
      const float sg = sig(x);
      const float act = x * sg;                                   // silu
      const float s1 = sg * (1.f + x * (1.f - sg));               // silu'
      const float s2 = sg * (1.f - sg) * (2.f + x * (1.f - 2.f * sg));   // silu''
      const float dg = -eta * a.vw2[i], r2 = -eta * a.vr2[i];
      const float r1 = a.r1[i], r3 = a.r3[i];
      vdh3 = r2 * act + dg * s1 * r1;
      vdh1 = (r2 * y + dg * r3) * s1 + dg * y * r1 * s2;
      vddg = act * r3 + y * s1 * r1;
      vddgn = -eta * vddg;
      ve1 = dg * y * s1;
      ve3 = dg * act;
      vg = act * y;
    }
    a.d_h1[i] = __float2bfloat16_rn(vdh1);
    a.d_h3[i] = __float2bfloat16_rn(vdh3);
    a.d_dg[i] = __float2bfloat16_rn(vddg);
    a.d_dgn[i] = __float2bfloat16_rn(vddgn);
    a.e1[i] = __float2bfloat16_rn(ve1);
    a.e3[i] = __float2bfloat16_rn(ve3);
    a.g[i] = __float2bfloat16_rn(vg);
  }
}

struct ReadEwArgs {
  int BH, C, cmax, dh;
  const float *hq1, *hq3, *dgq;   // fp32 [BH][cmax][dh]: Q W1^T, Q W3^T, dout W2
  __nv_bfloat16 *dhq1, *dhq3, *gq;
};
__global__ void bwd_read_ew_kernel(ReadEwArgs a) {
  const size_t n = (size_t)a.BH * a.cmax * a.dh;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    const int t = (int)((i / a.dh) % a.cmax);
    float v1 = 0.f, v3 = 0.f, vg = 0.f;
    if (t < a.C) {
      const float x = a.hq1[i], y = a.hq3[i], dg = a.dgq[i];
      const float sg = sig(x);
      const float act = x * sg;
      v1 = dg * y * sg * (1.f + x * (1.f - sg));
      v3 = dg * act;
      vg = act * y;
    }
    a.dhq1[i] = __float2bfloat16_rn(v1);
    a.dhq3[i] = __float2bfloat16_rn(v3);
    a.gq[i] = __float2bfloat16_rn(vg);
  }
}

// dv = -lr d_dy, dlr = -v . d_dy for the chunk's tokens (one warp per token).
__global__ void bwd_dv_kernel(int BH, int C, int cmax, int d, int N, int t0, const float* lr,
                              const __nv_bfloat16* v, const float* ddy, float* dv, float* dlr) {
  // one warp per token row, four consecutive columns per lane (d % 128 == 0)
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (gw >= BH * C) return;
  const int bh = gw / C, t = gw % C;
  const size_t tok = (size_t)bh * N + t0 + t;
  const float eta = lr[tok];
  const float4* src = reinterpret_cast<const float4*>(ddy + ((size_t)bh * cmax + t) * d);
  const uint2* vr = reinterpret_cast<const uint2*>(v + tok * d);
  float4* dst = reinterpret_cast<float4*>(dv + tok * d);
  float acc = 0.f;
  for (int c = lane; c < d / 4; c += 32) {
    const float4 x = src[c];
    const uint2 vv = vr[c];
    dst[c] = make_float4(-eta * x.x, -eta * x.y, -eta * x.z, -eta * x.w);
    acc += bf16lo(vv.x) * x.x + bf16hi(vv.x) * x.y + bf16lo(vv.y) * x.z + bf16hi(vv.y) * x.w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) dlr[tok] = -acc;
}


// dW[m] += sum over the splits of the split-K partial products (the three
// weight-gradient matrices of a chunk, each [BH][splits][rows x cols]).
struct WgradSumArgs {
  int BH, splits;
  long long mat;             // rows x cols of one head's matrix (equal for the three)
  const float* part[3];
  float* dW[3];              // [BH][rows x cols]
};
__global__ void bwd_wgrad_sum_kernel(WgradSumArgs a) {
  const long long per = (long long)a.BH * a.mat / 4;   // float4 per matrix
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < 3 * per;
       i += (long long)gridDim.x * blockDim.x) {
    const int m = (int)(i / per);
    const long long e = (i % per) * 4;
    const long long b = e / a.mat, o = e % a.mat;
    const float* src = a.part[m] + (b * a.splits) * a.mat + o;
    float4 u = *reinterpret_cast<float4*>(a.dW[m] + e);
    for (int sp = 0; sp < a.splits; ++sp) {
      const float4 x = *reinterpret_cast<const float4*>(src + sp * a.mat);
      u.x += x.x; u.y += x.y; u.z += x.z; u.w += x.w;
    }
    *reinterpret_cast<float4*>(a.dW[m] + e) = u;
  }
}

// ---------------------------------------------------------------- fused forward products + elementwise step
// d = 128.  One CTA per (head, 128-token tile, 64 hidden units J): all
// operands in shared memory at once, the products into TMEM, then the
// elementwise step of the chain rule straight from TMEM to the bf16 outputs
// (no fp32 intermediates in memory).
//   key:  [h1 | h3] = K [W1_J; W3_J]^T, [r1 | r3] = K [R1_J; R3_J]^T,
//         [vw2 | vr2] = V [W2[:, J] | R2[:, J]]  -> d_h1, d_h3, d_dg, -lr d_dg,
//         e1, e3, g (the chunk gradient's VJP step above)
//   read: [hq1 | hq3] = Q [W1_J; W3_J]^T, dgq = dout W2[:, J] -> (dgq hq3 s),
//         (dgq aq), gq
namespace bf {
constexpr int BM = 128, HB = 64, D = 128;
constexpr uint32_t ATILE = BM * D * 2;      // 32 KB: 128 token rows x 128 d, two 64-column boxes
constexpr uint32_t ASTAGE = 2 * ATILE;      // K | V (key) or Q | dout (read)
constexpr uint32_t B2 = 2 * HB * D * 2;     // 32 KB: two weight blocks of 64 hidden x 128 d
constexpr uint32_t STG_OUT = BM * 32 * 2;   // 8 KB: one output's 128 rows x 32 columns (staging)
constexpr int EPI_WARPS = 8;
constexpr int THREADS = (2 + EPI_WARPS) * 32;
// Shared memory.  Key: one token stage (the next tile's loads only have to
// beat the elementwise step), [W1|W3], [R1|R3], [W2|R2], staging for seven
// outputs.  Read: two token stages, [W1|W3], W2, staging for three.
struct Layout {
  uint32_t nst, b13, r13, b2, stg, bar, bytes;
};
__host__ __device__ inline Layout layout(bool key) {
  Layout l;
  l.nst = key ? 1u : 2u;
  l.b13 = l.nst * ASTAGE;
  l.r13 = l.b13 + B2;
  l.b2 = key ? l.r13 + B2 : l.r13;          // read: W2 alone where [R1|R3] would go
  l.stg = key ? l.b2 + B2 : l.r13 + B2 / 2;
  l.bar = l.stg + (key ? 7u : 3u) * STG_OUT;
  l.bytes = l.bar + 256 + 1024;
  return l;
}
constexpr uint32_t TM_COLS = 512;
}  // namespace bf

struct BwdFwdMaps {
  CUtensorMap a0, a1;        // K / V (key) or Q / dout (read): token maps, box {64, 128}
  CUtensorMap w1, w3, w2;    // bf16 weights: W1, W3 box {64 d, 64 rows}; W2 box {64 hidden, 64 d rows}
  CUtensorMap r1, r3, r2;    // key: bf16 R (same shapes)
  CUtensorMap o[7];          // outputs [BH][cmax][dh] bf16, box {32, 128}, 64-byte swizzle
};
struct BwdFwdArgs {
  int BH, C, cmax, dh, t0, lr_len, n_mt, key;
  const float* lr;           // key: [BH][lr_len]
  DevStatus st;
};

// TMEM column of product j (0: [h1|h3], 1: [r1|r3], 2: [vw2|vr2]) of the
// CTA's tile t in the key step: three 128-column products rotate over four
// slots, so product 0 of tile t + 1 lands in the slot tile t left free
TTT_DEVICE_INLINE uint32_t key_slot(uint32_t t, int j) { return ((3u * t + (uint32_t)j) & 3u) * 128u; }

// Byte offset of 16-byte chunk `c` (0..3) of row `r` in a 64-byte-row tile
// under the 64-byte swizzle of the tensor store (chunk ^= bits 1-2 of the row)
TTT_DEVICE_INLINE uint32_t sw64_offset(int r, int c) {
  return (uint32_t)(r * 64 + ((c ^ ((r >> 1) & 3)) << 4));
}

// Persistent: CTA c takes a contiguous range of the (head, hidden block,
// token tile) tiles, token tile fastest, so consecutive tiles share their
// weight blocks (reloaded only when the block changes).  The next tile's
// loads and products overlap this tile's elementwise step; one set of
// accumulators in TMEM (the next tile's products wait until the epilogue has
// read them out).  The epilogue stages each half tile (32 hidden columns) of
// every output in shared memory and one lane per output writes it with a
// tensor store, so the rows leave as whole 64-byte segments.
__global__ void __launch_bounds__(bf::THREADS, 1)
    bwd_fwd_fused_kernel(const __grid_constant__ BwdFwdMaps maps, const BwdFwdArgs a) {
  using namespace bf;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const bool key = a.key != 0;
  const Layout lay = layout(key);
  const uint32_t nst = lay.nst;
  const int nout = key ? 7 : 3;
  uint64_t* a_full = reinterpret_cast<uint64_t*>(smem + lay.bar);   // [2]
  uint64_t* a_empty = a_full + 2;     // [2]
  uint64_t* w_full = a_empty + 2;
  uint64_t* w_empty = w_full + 1;
  uint64_t* acc_full = w_empty + 1;   // [2]
  uint64_t* acc_empty = acc_full + 2;  // [2]
  uint64_t* fin = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  uint32_t* abort_flag = tmem_slot + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_hb = a.dh / HB;
  const int total = a.n_mt * n_hb * a.BH;
  const int lo = (int)((long long)blockIdx.x * total / gridDim.x);
  const int hi = (int)((long long)(blockIdx.x + 1) * total / gridDim.x);
  auto decode = [&](int t, int& bh, int& hb, int& mt) {
    mt = t % a.n_mt;
    hb = (t / a.n_mt) % n_hb;
    bh = t / (a.n_mt * n_hb);
  };
  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&a_full[b], 1);
      mbar_init(&a_empty[b], 1);
    }
    mbar_init(w_full, 1);
    mbar_init(w_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], EPI_WARPS * 32);
    }
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  Waiter W{abort_flag, a.st, 400};
  const uint32_t wbytes = key ? 3 * B2 : B2 + B2 / 2;
  uint32_t at = 0, wl = 0;   // copies issued (producer lane)
  if (warp == 0) {
    if (lane == 0) {
      int cur = -1;
      bool ok = true;
      for (int t = lo; ok && t < hi; ++t) {
        int bh, hb, mt;
        decode(t, bh, hb, mt);
        const int grpw = bh * n_hb + hb;
        if (grpw != cur) {   // the weight blocks of (head, hidden block)
          if (wl >= 1 && !W.wait(w_empty, (wl - 1) & 1, 1)) { ok = false; break; }
          const int j0 = hb * HB;
          mbar_arrive_expect_tx(w_full, wbytes);
          // K-major weight blocks: atom h (d 64h .. 64h + 63) = [first 64 rows | second 64 rows]
          for (int h = 0; h < 2; ++h) {
            tma_load_3d(smem + lay.b13 + h * (B2 / 2), &maps.w1, w_full, h * 64, j0, bh);
            tma_load_3d(smem + lay.b13 + h * (B2 / 2) + B2 / 4, &maps.w3, w_full, h * 64, j0, bh);
          }
          // MN-major W2[:, J] (and R2[:, J]): 128 d rows of 64 hidden units, two 64-row boxes
          uint8_t* b2 = smem + lay.b2;
          for (int h = 0; h < 2; ++h) tma_load_3d(b2 + h * (B2 / 4), &maps.w2, w_full, j0, h * 64, bh);
          if (key) {
            for (int h = 0; h < 2; ++h) {
              tma_load_3d(smem + lay.r13 + h * (B2 / 2), &maps.r1, w_full, h * 64, j0, bh);
              tma_load_3d(smem + lay.r13 + h * (B2 / 2) + B2 / 4, &maps.r3, w_full, h * 64, j0, bh);
              tma_load_3d(b2 + B2 / 2 + h * (B2 / 4), &maps.r2, w_full, j0, h * 64, bh);
            }
          }
          ++wl;
          cur = grpw;
        }
        const uint32_t s = at % nst, u = at / nst;
        if (at >= nst && !W.wait(&a_empty[s], (u - 1) & 1, 2)) { ok = false; break; }
        const int row = a.t0 + mt * BM;
        uint8_t* st = smem + s * ASTAGE;
        mbar_arrive_expect_tx(&a_full[s], ASTAGE);
        for (int h = 0; h < 2; ++h) {
          tma_load_3d(st + h * (ATILE / 2), &maps.a0, &a_full[s], h * 64, row, bh);
          tma_load_3d(st + ATILE + h * (ATILE / 2), &maps.a1, &a_full[s], h * 64, row, bh);
        }
        ++at;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_k = make_idesc(128, 128, false, false);          // K-major B, N = 128
      const uint32_t id_mn = make_idesc(128, key ? 128 : 64, false, true);   // MN-major B
      const uint64_t da = make_sdesc(smem_u32(smem), 16, 1024);
      const uint64_t db13 = make_sdesc(smem_u32(smem + lay.b13), 16, 1024);
      const uint64_t dr13 = make_sdesc(smem_u32(smem + lay.r13), 16, 1024);
      // [W2_J | R2_J]: two 64-wide N blocks 16 KB apart
      const uint64_t db2 = make_sdesc(smem_u32(smem + lay.b2), B2 / 2, 1024);
      uint32_t am = 0, wu = 0;
      int cur = -1;
      bool ok = true;
      for (int t = lo; ok && t < hi; ++t) {
        int bh, hb, mt;
        decode(t, bh, hb, mt);
        const int grpw = bh * n_hb + hb;
        if (grpw != cur) {
          if (wu >= 1) mma_commit(w_empty);   // after every product on the previous blocks
          if (!W.wait(w_full, wu & 1, 3)) { ok = false; break; }
          ++wu;
          cur = grpw;
        }
        const uint32_t s = am % nst, u = am / nst;
        if (!W.wait(&a_full[s], u & 1, 4)) { ok = false; break; }
        tc_fence_after();
        const uint64_t da0 = sdesc_add(da, s * ASTAGE), da1 = sdesc_add(da0, ATILE);
        auto off_a = [](int kk) -> uint32_t { return (kk >> 2) * (ATILE / 2) + (kk & 3) * 32; };
        auto off_b = [](int kk) -> uint32_t { return (kk >> 2) * (B2 / 2) + (kk & 3) * 32; };
        if (key) {
          // three 128-column products in four TMEM slots, rotating: the
          // first goes to the slot the previous tile left free and starts
          // before the epilogue has read that tile out
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16(tmem + key_slot(am, 0), sdesc_add(da0, off_a(kk)), sdesc_add(db13, off_b(kk)), id_k, kk > 0);
          if (am >= 1 && !W.wait(&acc_empty[0], (am - 1) & 1, 5)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            mma_bf16(tmem + key_slot(am, 1), sdesc_add(da0, off_a(kk)), sdesc_add(dr13, off_b(kk)), id_k, kk > 0);
            mma_bf16(tmem + key_slot(am, 2), sdesc_add(da1, off_a(kk)), sdesc_add(db2, kk * 2048), id_mn, kk > 0);
          }
          mma_commit(&a_empty[s]);
          mma_commit(&acc_full[0]);
        } else {
          // two accumulator sets of 256 columns: a tile's products only wait
          // for the epilogue of the tile two back
          const uint32_t ab = am & 1;
          if (am >= 2 && !W.wait(&acc_empty[ab], ((am >> 1) - 1) & 1, 5)) { ok = false; break; }
          tc_fence_after();
          const uint32_t tb = tmem + ab * 256;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            mma_bf16(tb, sdesc_add(da0, off_a(kk)), sdesc_add(db13, off_b(kk)), id_k, kk > 0);
            mma_bf16(tb + 128, sdesc_add(da1, off_a(kk)), sdesc_add(db2, kk * 2048), id_mn, kk > 0);
          }
          mma_commit(&a_empty[s]);
          mma_commit(&acc_full[ab]);
        }
        ++am;
      }
      mma_commit(fin);
      W.drain(fin, 0);
    }
    __syncwarp();
  } else {
    const int q4 = warp & 3;
    const int cg = (warp - 2) >> 2;                 // 16 columns of each 32-column half
    const int r = q4 * 32 + lane;
    const uint32_t lb = (uint32_t)(q4 * 32) << 16;
    const int ew = warp - 2;                        // epilogue warp 0..7: output ew's store lane
    const bool issuer = lane == 0 && ew < nout;
    uint8_t* stg = smem + lay.stg;
    uint32_t ae = 0;
    for (int t = lo; t < hi; ++t, ++ae) {
      int bh, hb, mt;
      decode(t, bh, hb, mt);
      const int j0 = hb * HB;
      const int tok = mt * BM + r;                  // row of the chunk
      const bool valid = tok < a.C;
      const float eta = (key && valid) ? a.lr[(size_t)bh * a.lr_len + a.t0 + tok] : 0.f;
      // accumulators of this tile: key, slots rotating over four; read, the
      // set of the tile's parity
      const uint32_t eb = key ? 0u : (ae & 1u);
      const uint32_t e_par = key ? (ae & 1u) : ((ae >> 1) & 1u);
      const uint32_t p13 = key ? key_slot(ae, 0) : eb * 256;
      const uint32_t pr13 = key ? key_slot(ae, 1) : 0;
      const uint32_t p2 = key ? key_slot(ae, 2) : eb * 256 + 128;
      // the epilogue warps meet at named barriers below: they leave together
      if (!named_bar_all(1, EPI_WARPS * 32, W.wait(&acc_full[eb], e_par, 6))) break;
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t c0 = (uint32_t)(h * 32 + cg * 16);
        uint32_t x1[16], x3[16], x5[16], y1[16], y3[16], y5[16];
        // every lane takes part in the warp-collective loads
        tmem_ld16_issue(tmem + lb + p13 + c0, x1);          // h1 / hq1
        tmem_ld16_issue(tmem + lb + p13 + 64 + c0, x3);     // h3 / hq3
        tmem_ld16_issue(tmem + lb + p2 + c0, x5);           // vw2 / dgq
        if (key) {
          tmem_ld16_issue(tmem + lb + pr13 + c0, y1);       // r1
          tmem_ld16_issue(tmem + lb + pr13 + 64 + c0, y3);  // r3
          tmem_ld16_issue(tmem + lb + p2 + 64 + c0, y5);    // vr2
        }
        tmem_wait_ld();
        if (h == 1) {   // the accumulators are read out: later products may reuse them
          tc_fence_before();
          mbar_arrive(&acc_empty[eb]);
        }
        auto f2 = [](const uint32_t* rr, int j) {
          return make_float2(__uint_as_float(rr[j]), __uint_as_float(rr[j + 1]));
        };
        const float2 one = x2_splat(1.f);
        uint32_t o[7][8];
        if (key) {
          // pairs of adjacent hidden columns on the packed fp32 instructions
          const float2 ne = x2_splat(-eta);
#pragma unroll
          for (int j = 0; j < 16; j += 2) {
            const float2 x = f2(x1, j), y = f2(x3, j);
            const float2 r1 = f2(y1, j), r3 = f2(y3, j);
            const float2 sg = x2_sigmoid(x);
            const float2 act = x2_mul(x, sg);
            const float2 oms = x2_sub(one, sg);
            const float2 s1 = x2_fma(sg, x2_mul(x, oms), sg);                       // sg (1 + x (1 - sg))
            const float2 w = x2_fma(x, x2_fma(sg, x2_splat(-2.f), one), x2_splat(2.f));   // 2 + x (1 - 2 sg)
            const float2 s2 = x2_mul(x2_mul(sg, oms), w);
            const float2 dg = x2_mul(ne, f2(x5, j)), r2 = x2_mul(ne, f2(y5, j));
            const float2 dgy = x2_mul(dg, y);
            const float2 vdh3 = x2_fma(r2, act, x2_mul(x2_mul(dg, s1), r1));
            const float2 vdh1 = x2_fma(x2_fma(r2, y, x2_mul(dg, r3)), s1, x2_mul(x2_mul(dgy, r1), s2));
            const float2 vddg = x2_fma(act, r3, x2_mul(x2_mul(y, s1), r1));
            const float2 vddgn = x2_mul(ne, vddg);
            const float2 ve1 = x2_mul(dgy, s1);
            const float2 ve3 = x2_mul(dg, act);
            const float2 vg = x2_mul(act, y);
            o[0][j >> 1] = pack_bf16x2(vdh1.x, vdh1.y);
            o[1][j >> 1] = pack_bf16x2(vdh3.x, vdh3.y);
            o[2][j >> 1] = pack_bf16x2(vddg.x, vddg.y);
            o[3][j >> 1] = pack_bf16x2(vddgn.x, vddgn.y);
            o[4][j >> 1] = pack_bf16x2(ve1.x, ve1.y);
            o[5][j >> 1] = pack_bf16x2(ve3.x, ve3.y);
            o[6][j >> 1] = pack_bf16x2(vg.x, vg.y);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 16; j += 2) {
            const float2 x = f2(x1, j), y = f2(x3, j), dg = f2(x5, j);
            const float2 sg = x2_sigmoid(x);
            const float2 act = x2_mul(x, sg);
            const float2 s1 = x2_fma(sg, x2_mul(x, x2_sub(one, sg)), sg);
            const float2 v1 = x2_mul(x2_mul(dg, y), s1);
            const float2 v3 = x2_mul(dg, act);
            const float2 vg = x2_mul(act, y);
            o[0][j >> 1] = pack_bf16x2(v1.x, v1.y);
            o[1][j >> 1] = pack_bf16x2(v3.x, v3.y);
            o[2][j >> 1] = pack_bf16x2(vg.x, vg.y);
          }
        }
        if (!valid) {   // rows past the chunk hold zeros
#pragma unroll
          for (int q = 0; q < 7; ++q)
#pragma unroll
            for (int u = 0; u < 8; ++u) o[q][u] = 0u;
        }
        // the staging buffer is free once the previous half's stores have read it
        if (issuer) bulk_wait_read();
        named_bar_sync(1, EPI_WARPS * 32);
        const uint32_t sb = smem_u32(stg);
#pragma unroll
        for (int q = 0; q < 7; ++q) {
          if (q < nout) {
            st_shared_v4(sb + q * STG_OUT + sw64_offset(r, 2 * cg), o[q][0], o[q][1], o[q][2], o[q][3]);
            st_shared_v4(sb + q * STG_OUT + sw64_offset(r, 2 * cg + 1), o[q][4], o[q][5], o[q][6], o[q][7]);
          }
        }
        fence_async_smem();   // the tensor store (async proxy) reads what these threads wrote
        named_bar_sync(1, EPI_WARPS * 32);
        if (issuer) {
          tma_store_3d(&maps.o[ew], stg + ew * STG_OUT, j0 + h * 32, mt * BM, bh);
          bulk_commit();
        }
      }
    }
    if (issuer) bulk_wait_all();   // every tensor store is complete before the CTA exits
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0 && lane == 0 && W.aborted()) {   // an aborted CTA: its copies land before it leaves
    for (uint32_t i = at > nst ? at - nst : 0; i < at; ++i) W.drain(&a_full[i % nst], (i / nst) & 1);
    if (wl >= 1) W.drain(w_full, (wl - 1) & 1);
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TM_COLS);
  }
}

}  // namespace

LactBwdWorkspace lact_bwd_layout(const LactLaunch& f) {
  LactBwdWorkspace w{};
  const size_t BH = (size_t)f.B * f.H, mat = BH * f.d * f.dh;
  const int nch = f.N_in > 0 ? (f.N_in + f.chunk - 1) / f.chunk : 0;
  const int cin = std::min(f.chunk, std::max(f.N_in, 1));
  w.cmax = (std::max(cin, f.causal ? 0 : f.N_q) + 127) / 128 * 128;
  w.nch = nch;
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  size_t o = 0;
  w.status = o; o = al(o + 256);
  w.fws_bytes = lact_workspace_layout(f.B, f.H, f.N_in, f.N_q, f.d, f.dh, f.chunk, f.causal,
                                      f.opt, 0, f.update_mask, f.normalize_rows, 0).total;
  w.fws = o; o = al(o + w.fws_bytes);
  w.state = o; o = al(o + (f.opt == 0 ? 3 : 6) * mat * 4);
  w.wsave = o; o = al(o + (size_t)(nch + 1) * 3 * mat * 4);
  w.rn = o; o = al(o + (size_t)std::max(nch, 1) * BH * (2 * f.dh + f.d) * 4);
  w.G = o; o = al(o + 3 * mat * 4);
  w.dW = o; o = al(o + 3 * mat * 4);
  w.dM = o; o = al(o + 3 * mat * 4);
  w.R = o; o = al(o + 3 * mat * 4);
  w.Rb = o; o = al(o + 3 * mat * 2);
  w.Wb = o; o = al(o + 3 * mat * 2);
  const size_t inter = BH * w.cmax * f.dh;
  for (int i = 0; i < 6; ++i) { w.f32[i] = o; o = al(o + inter * 4); }
  for (int i = 0; i < 7; ++i) { w.b16[i] = o; o = al(o + inter * 2); }
  w.ddy = o; o = al(o + BH * w.cmax * f.d * 4);
  w.gctr = o; o = al(o + (size_t)std::max(nch, 1) * 4);   // unit counters of the grouped launches
  w.total = o;
  return w;
}

#define BWD_TRY(...)                      \
  do {                                    \
    if ((__VA_ARGS__) != 0) return -1;    \
  } while (0)

int launch_lact_bwd(const LactBwdLaunch& L, cudaStream_t stream) {
  const LactLaunch& f = L.f;
  const LactBwdWorkspace w = lact_bwd_layout(f);
  const int BH = f.B * f.H, d = f.d, dh = f.dh;
  const size_t mat = (size_t)BH * d * dh;
  uint8_t* ws = L.ws;
  auto F = [&](size_t off) { return reinterpret_cast<float*>(ws + off); };
  auto Hb = [&](size_t off) { return reinterpret_cast<__nv_bfloat16*>(ws + off); };
  float* state = F(w.state);
  float* wsave = F(w.wsave);
  float* rn = F(w.rn);
  const int nch = w.nch;
  const int q_rows = f.causal ? f.N_in : f.N_q;

  // ---------------------------------------------------------------- 1. forward replay
  BWD_TRY(cudaMemcpyAsync(state, L.W0, 3 * mat * 4, cudaMemcpyDeviceToDevice, stream) == cudaSuccess ? 0 : -1);
  if (f.opt != 0)
    BWD_TRY(cudaMemsetAsync(state + 3 * mat, 0, 3 * mat * 4, stream) == cudaSuccess ? 0 : -1);
  LactLaunch p = f;
  p.state = state;
  p.ws = ws + w.fws;
  p.ws_bytes = w.fws_bytes;
  p.split = 0;
  p.rownorm_out = nullptr;
  p.out = nullptr;
  p.mode = LACT_REPLAY;
  p.wsave = wsave;
  p.rownorm_all = rn;
  BWD_TRY(launch_lact(p, stream));

  // ---------------------------------------------------------------- maps and helpers
  const uint64_t BHu = (uint64_t)BH;
  auto tok = [&](CUtensorMap* m, const void* ptr, int rows, uint32_t box_rows) {   // [BH][rows][d]
    return make_tmap_bf16_3d(m, ptr, d, rows, BHu, (uint64_t)d * 2, (uint64_t)d * 2 * rows, 64, box_rows);
  };
  auto inter = [&](CUtensorMap* m, const void* ptr, uint32_t box_rows) {            // [BH][cmax][dh]
    return make_tmap_bf16_3d(m, ptr, dh, w.cmax, BHu, (uint64_t)dh * 2, (uint64_t)dh * 2 * w.cmax, 64,
                             box_rows);
  };
  // weights and R, bf16 [BH][rows][cols]: W1/W3-shaped [dh][d], W2-shaped [d][dh]
  auto w13 = [&](CUtensorMap* m, const void* ptr, uint32_t box_rows) {
    return make_tmap_bf16_3d(m, ptr, d, dh, BHu, (uint64_t)d * 2, (uint64_t)d * dh * 2, 64, box_rows);
  };
  auto w2m = [&](CUtensorMap* m, const void* ptr, uint32_t box_rows) {
    return make_tmap_bf16_3d(m, ptr, dh, d, BHu, (uint64_t)dh * 2, (uint64_t)d * dh * 2, 64, box_rows);
  };
  __nv_bfloat16* Wb = Hb(w.Wb);
  __nv_bfloat16* Rb = Hb(w.Rb);
  auto cast = [&](const float* src, __nv_bfloat16* dst, size_t n) -> int {
    const size_t n4 = n / 4;
    bwd_cast_kernel<<<(unsigned)std::min<size_t>((n4 + 255) / 256, 4096), 256, 0, stream>>>(src, dst, n4);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
  };
  float* dW = F(w.dW);
  float* dM = F(w.dM);
  // C[b][m][n] (+)= sum_p A_p B_p^T  into fp32 `o` (ld, batch stride), optionally accumulating
  // TMA coordinate offsets: am (A rows, K-major A), ak / bk (the K coordinate
  // of an MN-major A / B: token rows of a token tensor)
  auto gemm = [&](int variant, const CUtensorMap* A, const CUtensorMap* B, int np, int M, int N,
                  int ksteps, float* o, int ld, long long bs, bool acc, int row_off, int am,
                  int ak, int bk) -> int {
    GemmMaps m{};
    GemmArgs g = gemm_args_default(L.st);
    for (int i = 0; i < np; ++i) {
      m.a[i] = A[i];
      m.b[i] = B[i];
      g.a_m_off[i] = am;
      g.a_k_off[i] = ak;
      g.b_k_off[i] = bk;
    }
    g.npairs = np; g.M = M; g.N = N; g.batch = BH; g.k_steps = ksteps;
    g.o32 = o; g.ld32 = ld; g.o32_bs = bs; g.out_row_off = row_off;
    if (acc) { g.beta = 1.f; g.cin = o + 0; g.cin_bs = bs; g.ldc = ld; }
    return gemm_launch(variant, m, g, stream, K_GEMM_GRAD);
  };
  // cin of an accumulating GEMM is read at row m (no row offset), so
  // accumulating outputs always start at row 0 of their buffer


  CUtensorMap mq_k{}, mq_mn{}, mk_k{}, mk_mn{}, mv_k{}, mv_mn{}, mdo_k{}, mdo_mn{};
  if (f.N_in > 0) {
    BWD_TRY(tok(&mk_k, f.k, f.N_in, 128));
    BWD_TRY(tok(&mk_mn, f.k, f.N_in, 64));
    BWD_TRY(tok(&mv_k, f.v, f.N_in, 128));
    BWD_TRY(tok(&mv_mn, f.v, f.N_in, 64));
  }
  if (q_rows > 0) {
    BWD_TRY(tok(&mq_k, f.q, q_rows, 128));
    BWD_TRY(tok(&mq_mn, f.q, q_rows, 64));
    BWD_TRY(tok(&mdo_k, L.dout, q_rows, 128));
    BWD_TRY(tok(&mdo_mn, L.dout, q_rows, 64));
  }
  CUtensorMap mW1k, mW3k, mW2mn, mW1mn, mW3mn, mW2k, mR1k, mR3k, mR2mn, mR1mn, mR3mn, mR2k;
  BWD_TRY(w13(&mW1k, Wb, 128) | w13(&mW3k, Wb + mat, 128) | w2m(&mW2mn, Wb + 2 * mat, 64));
  BWD_TRY(w13(&mW1mn, Wb, 64) | w13(&mW3mn, Wb + mat, 64) | w2m(&mW2k, Wb + 2 * mat, 128));
  BWD_TRY(w13(&mR1k, Rb, 128) | w13(&mR3k, Rb + mat, 128) | w2m(&mR2mn, Rb + 2 * mat, 64));
  BWD_TRY(w13(&mR1mn, Rb, 64) | w13(&mR3mn, Rb + mat, 64) | w2m(&mR2k, Rb + 2 * mat, 128));
  float* f32[6];
  __nv_bfloat16* b16[7];
  for (int i = 0; i < 6; ++i) f32[i] = F(w.f32[i]);
  for (int i = 0; i < 7; ++i) b16[i] = Hb(w.b16[i]);
  CUtensorMap mb_k[7], mb_mn[7];
  for (int i = 0; i < 7; ++i) BWD_TRY(inter(&mb_k[i], b16[i], 128) | inter(&mb_mn[i], b16[i], 64));
  const long long ibs = (long long)w.cmax * dh;
  // d = 128: the forward products and the elementwise step of a chunk in one
  // kernel (bwd_fwd_fused_kernel); other shapes take the GEMMs + elementwise
  // kernels below
  const bool fused_fwd = d == 128 && dh % 64 == 0;
  // the read VJP's bf16 dhq1, dhq3, gq on the fused path: in the fp32
  // intermediates' memory (each region holds two bf16 buffers), so a causal
  // chunk's key and read steps can feed the same weight-gradient products
  __nv_bfloat16* rb16[3];
  CUtensorMap mrb_k[3], mrb_mn[3];
  for (int i = 0; i < 3; ++i) {
    rb16[i] = reinterpret_cast<__nv_bfloat16*>(f32[i]);
    BWD_TRY(inter(&mrb_k[i], rb16[i], 128) | inter(&mrb_mn[i], rb16[i], 64));
  }
  static std::atomic<uint64_t> fused_attr{0};
  const int fused_smem = (int)std::max(bf::layout(true).bytes, bf::layout(false).bytes);
  if (fused_fwd && allow_dynamic_smem(bwd_fwd_fused_kernel, fused_smem, fused_attr)) return -1;
  // the fused kernel's outputs as tensor-store targets: boxes of 32 hidden
  // columns x 128 token rows, 64-byte swizzle (its staging layout)
  CUtensorMap mo_key[7], mo_read[3];
  if (fused_fwd) {
    for (int i = 0; i < 7; ++i)
      BWD_TRY(make_tmap_bf16_3d_sw(&mo_key[i], b16[i], dh, w.cmax, BHu, (uint64_t)dh * 2,
                                   (uint64_t)dh * 2 * w.cmax, 32, 128, 64));
    for (int i = 0; i < 3; ++i)
      BWD_TRY(make_tmap_bf16_3d_sw(&mo_read[i], rb16[i], dh, w.cmax, BHu, (uint64_t)dh * 2,
                                   (uint64_t)dh * 2 * w.cmax, 32, 128, 64));
  }
  auto fused = [&](bool key, const CUtensorMap& a0, const CUtensorMap& a1, int t0, int C) -> int {
    BwdFwdMaps m{};
    m.a0 = a0; m.a1 = a1;
    m.w1 = mW1mn; m.w3 = mW3mn; m.w2 = mW2mn;
    m.r1 = mR1mn; m.r3 = mR3mn; m.r2 = mR2mn;
    for (int i = 0; i < (key ? 7 : 3); ++i) m.o[i] = key ? mo_key[i] : mo_read[i];
    BwdFwdArgs ba{};
    ba.BH = BH; ba.C = C; ba.cmax = w.cmax; ba.dh = dh; ba.t0 = t0; ba.lr_len = f.N_in;
    ba.n_mt = w.cmax / bf::BM; ba.key = key ? 1 : 0; ba.lr = f.lr; ba.st = L.st;
    prof_before(K_BWD_FWD, stream);
    bwd_fwd_fused_kernel<<<dim3((unsigned)std::min(ba.n_mt * (dh / bf::HB) * BH, num_sms_bwd())),
                           dim3(bf::THREADS), bf::layout(key).bytes, stream>>>(m, ba);
    prof_after(K_BWD_FWD, stream);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
  };

  float* dW1 = dW;
  float* dW3 = dW + mat;
  float* dW2 = dW + 2 * mat;
  const long long w13bs = (long long)dh * d, w2bs = (long long)d * dh;

  // dq rows [t0, t0 + C) = dhq1 W1 + dhq3 W3  (M = C, N = d, K = dh)
  auto read_dq = [&](int t0, int C) -> int {
    const CUtensorMap A[2] = {fused_fwd ? mrb_k[0] : mb_k[0], fused_fwd ? mrb_k[1] : mb_k[1]},
                      B[2] = {mW1mn, mW3mn};
    return gemm(GEMM_AK_BMN, A, B, 2, C, d, dh / 64, L.dq, d, (long long)q_rows * d, false, t0,
                0, 0, 0);
  };
  // read VJP for query rows [t0, t0 + C) with the weights in Wb: dq rows and dW
  auto read_vjp = [&](int t0, int C) -> int {
    const int ks = (C + 63) / 64;
    if (fused_fwd) {
      BWD_TRY(fused(false, mq_k, mdo_k, t0, C));
    } else {
      // hq1 = Q W1^T, hq3 = Q W3^T, dgq = dout W2   (M = C, N = dh, K = d)
      BWD_TRY(gemm(GEMM_AK_BK, &mq_k, &mW1k, 1, C, dh, d / 64, f32[0], dh, ibs, false, 0, t0, 0, 0));
      BWD_TRY(gemm(GEMM_AK_BK, &mq_k, &mW3k, 1, C, dh, d / 64, f32[1], dh, ibs, false, 0, t0, 0, 0));
      BWD_TRY(gemm(GEMM_AK_BMN, &mdo_k, &mW2mn, 1, C, dh, d / 64, f32[2], dh, ibs, false, 0, t0, 0, 0));
      ReadEwArgs ra{BH, C, w.cmax, dh, f32[0], f32[1], f32[2], b16[0], b16[1], b16[6]};
      const size_t n = (size_t)BH * w.cmax * dh;
      bwd_read_ew_kernel<<<(unsigned)std::min<size_t>((n + 255) / 256, 8192), 256, 0, stream>>>(ra);
      BWD_TRY(cudaGetLastError() == cudaSuccess ? 0 : -1);
    }
    const CUtensorMap& dhq1_mn = fused_fwd ? mrb_mn[0] : mb_mn[0];
    const CUtensorMap& dhq3_mn = fused_fwd ? mrb_mn[1] : mb_mn[1];
    const CUtensorMap& gq_mn = fused_fwd ? mrb_mn[2] : mb_mn[6];
    // dW1 += dhq1^T Q, dW3 += dhq3^T Q  (M = dh, N = d, K = C tokens)
    BWD_TRY(gemm(GEMM_AMN_BMN, &dhq1_mn, &mq_mn, 1, dh, d, ks, dW1, d, w13bs, true, 0, 0, 0, t0));
    BWD_TRY(gemm(GEMM_AMN_BMN, &dhq3_mn, &mq_mn, 1, dh, d, ks, dW3, d, w13bs, true, 0, 0, 0, t0));
    // dW2 += dout^T gq  (M = d, N = dh)
    BWD_TRY(gemm(GEMM_AMN_BMN, &mdo_mn, &gq_mn, 1, d, dh, ks, dW2, dh, w2bs, true, 0, 0, t0, 0));
    return read_dq(t0, C);
  };

  // maps of the grouped launch: K-major token-row operands in boxes of 256
  // rows, MN-major operands through blocked views (one copy per block)
  CUtensorMap gk_b16[7], gk_rb16[3], gm_b16[7], gm_rb16[3], gm_w[4], gm_tok[4];
  if (fused_fwd) {
    for (int i = 0; i < 7; ++i)
      BWD_TRY(make_tmap_bf16_3d(&gk_b16[i], b16[i], dh, w.cmax, BHu, (uint64_t)dh * 2,
                                (uint64_t)dh * 2 * w.cmax, 64, 256) |
              make_tmap_bf16_blocked(&gm_b16[i], b16[i], dh, w.cmax, BHu, (uint64_t)dh * 2,
                                     (uint64_t)dh * 2 * w.cmax, 64, 4));
    for (int i = 0; i < 3; ++i)
      BWD_TRY(make_tmap_bf16_3d(&gk_rb16[i], rb16[i], dh, w.cmax, BHu, (uint64_t)dh * 2,
                                (uint64_t)dh * 2 * w.cmax, 64, 256) |
              make_tmap_bf16_blocked(&gm_rb16[i], rb16[i], dh, w.cmax, BHu, (uint64_t)dh * 2,
                                     (uint64_t)dh * 2 * w.cmax, 64, 4));
    // W1, W3, R1, R3 as [m = d][k = hidden] (MN-major A)
    const __nv_bfloat16* wsrc[4] = {Wb, Wb + mat, Rb, Rb + mat};
    for (int i = 0; i < 4; ++i)
      BWD_TRY(make_tmap_bf16_blocked(&gm_w[i], wsrc[i], d, dh, BHu, (uint64_t)d * 2,
                                     (uint64_t)d * dh * 2, 64, 2));
    // K, V (N_in rows), Q, dout (q_rows rows) as [m = d][k = token] (MN-major A)
    const void* tsrc[4] = {f.k, f.v, f.q, L.dout};
    const int trows[4] = {f.N_in, f.N_in, q_rows, q_rows};
    for (int i = 0; i < 4; ++i)
      if (tsrc[i] != nullptr && trows[i] > 0)
        BWD_TRY(make_tmap_bf16_blocked(&gm_tok[i], tsrc[i], d, trows[i], BHu, (uint64_t)d * 2,
                                       (uint64_t)d * 2 * trows[i], 64, 2));
  }
  // The products of a chunk on the fused path, in one grouped launch, each
  // posed with M = d and N the long side (tokens or hidden units):
  //   dk rows^T  = W1^T d_h1^T + W3^T d_h3^T + R1^T e1^T + R3^T e3^T   (N = C, K = 4 dh)
  //   d_dy^T     = W2 d_dg^T + R2 g^T                                   (N = C, K = 2 dh)
  //   dq rows^T  = W1^T dhq1^T + W3^T dhq3^T                            (with the read)
  //   dW1^T, dW3^T partials = K^T d_h1 (+ Q^T dhq1), K^T d_h3 (+ Q^T dhq3)   (N = dh)
  //   dW2 partial           = V^T (-lr d_dg) (+ dout^T gq)                   (N = dh)
  // the weight-gradient products split over the chunk's tokens into the
  // (free) fp32 intermediates, then one pass adds the splits to dW (a few
  // output tiles per matrix would leave most SMs idle); steps past the chunk
  // read zero rows of the bf16 intermediates.  Each split's partial is
  // d x dh per head, so S splits fit the region while S d <= cmax.
  static std::atomic<uint64_t> group_attr{0};
  if (fused_fwd && allow_dynamic_smem(gemm_group_kernel, (int)gg::SMEM, group_attr)) return -1;
  int pending_splits = 0;   // partials of the last grouped launch not yet in dW
  auto chunk_products = [&](int t0, int C, bool with_read) -> int {
    const int ks = (C + 63) / 64;
    const int S = std::max(1, std::min(std::min(8, ks), w.cmax / d)), kps = (ks + S - 1) / S;
    GroupMaps m{};
    GroupArgs g{};
    g.st = L.st;
    g.ctr = reinterpret_cast<unsigned int*>(ws + w.gctr) + t0 / f.chunk;
    int units = 0;
    auto add = [&](int N, int splits, int k_steps, int np, bool a_mn, bool b_mn,
                   const CUtensorMap* A, const CUtensorMap* B, int a_k_off, int b_k_off, float* o,
                   long long o_bs, long long o_ss, int ld, bool out_t, int row_off) {
      GroupProblem& q = g.p[g.nprob];
      q.M = d; q.N = N;
      q.tiles_m = d / 128; q.tiles_n = (N + gg::BN - 1) / gg::BN; q.splits = splits;
      q.k_steps = k_steps; q.npairs = np; q.a_mn = a_mn ? 1 : 0; q.b_mn = b_mn ? 1 : 0;
      q.unit0 = units;
      for (int i = 0; i < np; ++i) {
        m.a[g.nprob][i] = A[i];
        m.b[g.nprob][i] = B[i];
        q.a_k_off[i] = a_k_off;
        q.b_k_off[i] = b_k_off;
      }
      q.o = o; q.o_bs = o_bs; q.o_ss = o_ss; q.ld = ld; q.out_t = out_t ? 1 : 0; q.row_off = row_off;
      q.v8 = (reinterpret_cast<uintptr_t>(o) % 32 == 0 && ld % 8 == 0 && o_bs % 8 == 0 &&
              o_ss % 8 == 0) ? 1 : 0;
      units += q.tiles_m * q.tiles_n * splits * BH;
      ++g.nprob;
    };
    const int kd = dh / 64;
    {
      const CUtensorMap A[4] = {gm_w[0], gm_w[1], gm_w[2], gm_w[3]};
      const CUtensorMap B[4] = {gk_b16[0], gk_b16[1], gk_b16[4], gk_b16[5]};
      add(C, 1, kd, 4, true, false, A, B, 0, 0, L.dk, (long long)f.N_in * d, 0, d, true, t0);
    }
    {
      const CUtensorMap A[2] = {mW2k, mR2k}, B[2] = {gk_b16[2], gk_b16[6]};
      add(C, 1, kd, 2, false, false, A, B, 0, 0, F(w.ddy), (long long)w.cmax * d, 0, d, true, 0);
    }
    if (with_read) {
      const CUtensorMap A[2] = {gm_w[0], gm_w[1]}, B[2] = {gk_rb16[0], gk_rb16[1]};
      add(C, 1, kd, 2, true, false, A, B, 0, 0, L.dq, (long long)q_rows * d, 0, d, true, t0);
    }
    const int np = with_read ? 2 : 1;
    const long long wsz = (long long)d * dh;
    {
      const CUtensorMap A13[2] = {gm_tok[0], gm_tok[2]};
      const CUtensorMap B1[2] = {gm_b16[0], gm_rb16[0]}, B3[2] = {gm_b16[1], gm_rb16[1]};
      add(dh, S, kps, np, true, true, A13, B1, t0, 0, f32[3], S * wsz, wsz, d, true, 0);
      add(dh, S, kps, np, true, true, A13, B3, t0, 0, f32[4], S * wsz, wsz, d, true, 0);
    }
    {
      const CUtensorMap A2[2] = {gm_tok[1], gm_tok[3]}, B2[2] = {gm_b16[3], gm_rb16[2]};
      add(dh, S, kps, np, true, true, A2, B2, t0, 0, f32[5], S * wsz, wsz, dh, false, 0);
    }
    g.units = units;
    prof_before(K_BWD_GROUP, stream);
    const cudaError_t e = launch_pdl(gemm_group_kernel, dim3((unsigned)std::min(units, num_sms_bwd())),
                                     dim3(gg::THREADS), gg::SMEM, stream, m, g);
    prof_after(K_BWD_GROUP, stream);
    if (e != cudaSuccess || cudaGetLastError() != cudaSuccess) return -1;
    // the splits are added to dW by the next chunk's row step (or the final
    // sum after the last chunk)
    pending_splits = S;
    return 0;
  };

  // ---------------------------------------------------------------- 2. reverse
  if (L.dW_end)
    BWD_TRY(cudaMemcpyAsync(dW, L.dW_end, 3 * mat * 4, cudaMemcpyDeviceToDevice, stream) == cudaSuccess ? 0 : -1);
  else
    BWD_TRY(cudaMemsetAsync(dW, 0, 3 * mat * 4, stream) == cudaSuccess ? 0 : -1);
  BWD_TRY(cudaMemsetAsync(dM, 0, 3 * mat * 4, stream) == cudaSuccess ? 0 : -1);
  if (fused_fwd && nch > 0)
    BWD_TRY(cudaMemsetAsync(ws + w.gctr, 0, (size_t)nch * 4, stream) == cudaSuccess ? 0 : -1);
  if (!f.causal && f.N_q > 0) {   // the queries read the final weights
    BWD_TRY(cast(wsave + (size_t)nch * 3 * mat, Wb, 3 * mat));
    BWD_TRY(read_vjp(0, f.N_q));
  }
  RowStepArgs rs{};
  rs.BH = BH; rs.d = d; rs.dh = dh; rs.mask = f.update_mask; rs.normalize = f.normalize_rows;
  rs.momentum = f.opt == 1; rs.beta = f.beta; rs.norm_eps = f.norm_eps;
  rs.dW = dW; rs.dM = dM; rs.R = F(w.R); rs.Rb = Rb; rs.Wb = Wb;
  const int row_warps = BH * (2 * dh + d);
  for (int c = nch - 1; c >= 0; --c) {
    const int t0 = c * f.chunk, C = std::min(f.chunk, f.N_in - t0);
    const int ks = (C + 63) / 64;
    rs.Wn = wsave + (size_t)(c + 1) * 3 * mat;
    rs.rn = rn + (size_t)c * BH * (2 * dh + d);
    rs.Wc = wsave + (size_t)c * 3 * mat;   // its bf16 copy is the chunk's product operand
    for (int m = 0; m < 3; ++m) rs.part[m] = pending_splits > 0 ? f32[3 + m] : nullptr;
    rs.splits = pending_splits;
    pending_splits = 0;
    bwd_row_step_kernel<<<(row_warps * 32 + 255) / 256, 256, 0, stream>>>(rs);
    BWD_TRY(cudaGetLastError() == cudaSuccess ? 0 : -1);
    // a causal chunk on the fused path: the read's elementwise step too, so
    // both feed the weight-gradient products below
    const bool both = fused_fwd && f.causal;
    if (fused_fwd) {
      BWD_TRY(fused(true, mk_k, mv_k, t0, C));
      if (both) BWD_TRY(fused(false, mq_k, mdo_k, t0, C));
    } else {
      // h1 = K W1^T, h3 = K W3^T, vw2 = V W2, r1 = K R1^T, r3 = K R3^T, vr2 = V R2
      BWD_TRY(gemm(GEMM_AK_BK, &mk_k, &mW1k, 1, C, dh, d / 64, f32[0], dh, ibs, false, 0, t0, 0, 0));
      BWD_TRY(gemm(GEMM_AK_BK, &mk_k, &mW3k, 1, C, dh, d / 64, f32[1], dh, ibs, false, 0, t0, 0, 0));
      BWD_TRY(gemm(GEMM_AK_BMN, &mv_k, &mW2mn, 1, C, dh, d / 64, f32[2], dh, ibs, false, 0, t0, 0, 0));
      BWD_TRY(gemm(GEMM_AK_BK, &mk_k, &mR1k, 1, C, dh, d / 64, f32[3], dh, ibs, false, 0, t0, 0, 0));
      BWD_TRY(gemm(GEMM_AK_BK, &mk_k, &mR3k, 1, C, dh, d / 64, f32[4], dh, ibs, false, 0, t0, 0, 0));
      BWD_TRY(gemm(GEMM_AK_BMN, &mv_k, &mR2mn, 1, C, dh, d / 64, f32[5], dh, ibs, false, 0, t0, 0, 0));
      KeyEwArgs ka{BH, C, w.cmax, dh, f.N_in, t0, f.lr, f32[0], f32[1], f32[2], f32[3], f32[4], f32[5],
                   b16[0], b16[1], b16[2], b16[3], b16[4], b16[5], b16[6]};
      const size_t n = (size_t)BH * w.cmax * dh;
      bwd_key_ew_kernel<<<(unsigned)std::min<size_t>((n + 255) / 256, 8192), 256, 0, stream>>>(ka);
      BWD_TRY(cudaGetLastError() == cudaSuccess ? 0 : -1);
    }
    if (fused_fwd) {
      BWD_TRY(chunk_products(t0, C, both));
    } else {
      // dk rows = d_h1 W1 + d_h3 W3 + e1 R1, then + e3 R3   (M = C, N = d, K = dh)
      const CUtensorMap A[3] = {mb_k[0], mb_k[1], mb_k[4]}, B[3] = {mW1mn, mW3mn, mR1mn};
      BWD_TRY(gemm(GEMM_AK_BMN, A, B, 3, C, d, dh / 64, F(w.ddy), d, (long long)w.cmax * d, false, 0,
                   0, 0, 0));
      BWD_TRY(gemm(GEMM_AK_BMN, &mb_k[5], &mR3mn, 1, C, d, dh / 64, F(w.ddy), d, (long long)w.cmax * d,
                   true, 0, 0, 0, 0));
      // the chunk's dk rows: copy out of the temporary (rows t0.. of dk)
      BWD_TRY(cudaMemcpy2DAsync(L.dk + (size_t)t0 * d, (size_t)f.N_in * d * 4, F(w.ddy),
                                (size_t)w.cmax * d * 4, (size_t)C * d * 4, BH, cudaMemcpyDeviceToDevice,
                                stream) == cudaSuccess ? 0 : -1);
      // weight gradients: dW1 += d_h1^T K, dW3 += d_h3^T K, dW2 += V^T (-lr d_dg)
      BWD_TRY(gemm(GEMM_AMN_BMN, &mb_mn[0], &mk_mn, 1, dh, d, ks, dW1, d, w13bs, true, 0, 0, 0, t0));
      BWD_TRY(gemm(GEMM_AMN_BMN, &mb_mn[1], &mk_mn, 1, dh, d, ks, dW3, d, w13bs, true, 0, 0, 0, t0));
      BWD_TRY(gemm(GEMM_AMN_BMN, &mv_mn, &mb_mn[3], 1, d, dh, ks, dW2, dh, w2bs, true, 0, 0, t0, 0));
      // d_dy = d_dg W2^T + g R2^T   (M = C, N = d, K = dh)
      const CUtensorMap A2[2] = {mb_k[2], mb_k[6]}, B2[2] = {mW2k, mR2k};
      BWD_TRY(gemm(GEMM_AK_BK, A2, B2, 2, C, d, dh / 64, F(w.ddy), d, (long long)w.cmax * d, false, 0,
                   0, 0, 0));
    }
    {
      const int warps = BH * C;
      bwd_dv_kernel<<<(warps * 32 + 255) / 256, 256, 0, stream>>>(
          BH, C, w.cmax, d, f.N_in, t0, f.lr, reinterpret_cast<const __nv_bfloat16*>(f.v), F(w.ddy),
          L.dv, L.dlr);
      BWD_TRY(cudaGetLastError() == cudaSuccess ? 0 : -1);
    }
    if (!both && f.causal) BWD_TRY(read_vjp(t0, C));
  }
  if (pending_splits > 0) {   // the first chunk's partial products
    WgradSumArgs sa{BH, pending_splits, (long long)d * dh, {f32[3], f32[4], f32[5]}, {dW1, dW3, dW2}};
    const long long n4 = 3LL * BH * d * dh / 4;
    bwd_wgrad_sum_kernel<<<(unsigned)std::min<long long>((n4 + 255) / 256, 4096), 256, 0, stream>>>(sa);
    BWD_TRY(cudaGetLastError() == cudaSuccess ? 0 : -1);
  }
  return cudaMemcpyAsync(L.dW0, dW, 3 * mat * 4, cudaMemcpyDeviceToDevice, stream) == cudaSuccess
             ? 0 : -1;
}

}  // namespace ttt
