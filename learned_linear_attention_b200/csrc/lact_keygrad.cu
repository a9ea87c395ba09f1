// lact_keygrad.cu -- fused key pass + chunk gradient for head dim d = 128
// ("Test-Time Training Done Right" review, "Memoria no lineal y atención
// local": the chunk's lr-weighted gradients of -<f_W(k), v> are summed at
// the chunk-start weights).
//
// One work item = (head, 64 hidden units J, a group of token tiles of the
// chunk).  For every 128-token tile of the group:
//   MMA   H13 = K [W1_J; W3_J]^T   (128 x 128),   dGr = V W2[:, J]  (128 x 64)
//   epi   dG = -eta dGr, dH3 = dG silu(H1), dH1 = dG H3 silu'(H1),
//         Gm' = -eta silu(H1) H3           -> bf16 operands in shared memory
//   MMA   [G1_J | G3_J]^T += K^T [dH1 | dH3] (one N = 128 product),
//         G2[:, J] += V^T Gm'
// with the K and V tiles reused from shared memory (as MN-major operands)
// and the three gradient accumulators resident in TMEM across the group.
// H13 alternates between two TMEM buffers, so a tile's forward product runs
// while the epilogue still works on the previous tile.
// At the end of the item the partial gradients are stored (plain stores,
// one slot per token group) and the row update kernel sums the groups in a
// fixed order.  Nothing of the chunk's intermediates goes to global memory.
#include <algorithm>

#include "kernels.h"

namespace ttt {
namespace kg {
constexpr int D = 128, HB = 64, BM = 128;
constexpr uint32_t HALF = BM * 64 * 2;                 // 16 KB: 128 rows x 64 bf16
constexpr uint32_t TILE = 2 * HALF;                    // 32 KB: 128 tokens x 128 d
constexpr uint32_t OFF_KV = 0;                         // 2 stages x (K tile | V tile)
constexpr uint32_t KV_STAGE = 2 * TILE;                // 64 KB
constexpr uint32_t OFF_W13 = 2 * KV_STAGE;             // [W1_J | W3_J] x d: two K atoms
constexpr uint32_t OFF_W2 = OFF_W13 + 2 * HALF;        // W2[:, J]: 128 d-rows x 64 hidden
constexpr uint32_t OFF_DH = OFF_W2 + 2 * 8192;         // dH1 | dH3 | Gm' (16 KB each)
constexpr uint32_t OFF_BAR = OFF_DH + 3 * HALF;
constexpr uint32_t SMEM = OFF_BAR + 256 + 1024;
constexpr int EPI_WARPS = 16;                          // four per TMEM lane quadrant
constexpr int THREADS = (2 + EPI_WARPS) * 32;
constexpr int CW = HB / (EPI_WARPS / 4);              // hidden columns per epilogue warp (16)
// TMEM columns: H13 in two buffers, dGr (key tiles), G2, [G1 | G3]
constexpr uint32_t TM_H13A = 0, TM_DG = 128, TM_G2 = 192, TM_G13 = 256, TM_H13B = 384, TM_COLS = 512;
// chunk loop: room for the row update's partial sums (weight tiles + dH)
constexpr uint32_t LOOP_PART_BYTES = OFF_BAR - OFF_W13;
}  // namespace kg

struct KeyGradArgs {
  int BH, C, t0, lr_len, dh;
  int n_hb, n_groups, tiles_total, tiles_per_group;
  const float* lr;
  float* part[3];        // [group][BH][rows][cols] partial gradients (G1, G3, G2)
  int queries;           // causal order: also form Aq = silu(Q W1^T) (Q W3^T) for the tiles
  __nv_bfloat16* Aq;     // [BH][cmax][dh] (queries)
  long long aq_bs;       // cmax * dh
  DevStatus st;
};
// Chunk loop only (one launch runs the whole causal chunk sequence); a
// separate parameter, so the one-chunk kernel's arguments stay small.
struct KeyGradLoopArgs {
  int n_chunks, N;       // chunks of C tokens (the last one may be shorter); tokens
  int n_workers;         // CTAs [0, n_workers) take the items, the others read out
  long long aq_buf;      // elements between the two Aq buffers
  unsigned* ctr;         // per head bh: [bh] its CTAs' partial sums of a chunk
                         // written, [BH + bh] their row updates done, [2 BH +
                         // bh] their Aq written; [3 BH] reader chunks done,
                         // [3 BH + 1] grid-wide abort word; all zero at launch
  float* W[3];           // fp32 weights W1, W3, W2 (updated in place)
  float* M[3];           // momentum (opt == 1)
  __nv_bfloat16* Wb[3][3];   // [buffer][matrix] bf16 copies; chunk c reads buffer c % 3
  int opt, normalize, mask;
  float beta, norm_eps;
  void* out;             // [BH][N][128] bf16 or fp32
  int out_bf16;
  long long out_bs;      // N * 128
  int cast_first;        // workers write the start weights' bf16 copies first (counted
                         // on the heads' update counters like an update)
  // the backward pass's replay (nullable): the weights after chunk c go to
  // wsave + (c + 1) [W1 | W3 | W2], and each updated row's norm before the
  // normalisation to rownorm + c [BH][2 dh + 128]
  float* wsave;
  float* rownorm;
};
struct KeyGradMaps {
  CUtensorMap k, v, q;
  CUtensorMap w1[3], w3[3], w2[3];   // per bf16 weight buffer (one buffer unless chunk loop)
  CUtensorMap aq[2], w2k[3];         // chunk loop readers: Aq buffers, W2 as K-major B
};

TTT_DEVICE_INLINE void tma_prefetch_l2_3d(const CUtensorMap* m, int x, int y, int z) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(x), "r"(y), "r"(z)
               : "memory");
}


// Epilogue operand arithmetic on two hidden columns of one token row at a
// time, with the packed two-lane fp32 instructions of sm_100 (each lane
// rounds exactly like the scalar instruction), so the per-tile math issues
// about half as many instructions.  sg = sigmoid(x) = 0.5 tanh(x / 2) + 0.5.
// Key tiles, with the row's -eta and dGr = g:
//   dH3 = -eta g silu(x),  Gm' = -eta silu(x) y,
//   dH1 = -eta g sg y (1 + x (1 - sg))  (x (1 - sg) = x - silu(x)).
TTT_DEVICE_INLINE void key_ops_x2(uint32_t x0, uint32_t x1, uint32_t y0, uint32_t y1, uint32_t g0,
                                  uint32_t g1, float neta, uint32_t& o1, uint32_t& o3, uint32_t& om) {
  asm("{\n\t"
      ".reg .b64 X, Y, G, N, HF, H, T, SG, XS, NX, NG, Q, QY, U, A;\n\t"
      ".reg .f32 h0, h1, t0, t1, a0, a1;\n\t"
      ".reg .b32 c;\n\t"
      "mov.b32 c, 0f3F000000;\n\t"
      "mov.b64 HF, {c, c};\n\t"
      "mov.b64 X, {%3, %4};\n\t"
      "mov.b64 Y, {%5, %6};\n\t"
      "mov.b64 G, {%7, %8};\n\t"
      "mov.b64 N, {%9, %9};\n\t"
      "mul.rn.f32x2 H, X, HF;\n\t"
      "mov.b64 {h0, h1}, H;\n\t"
      "tanh.approx.f32 t0, h0;\n\t"
      "tanh.approx.f32 t1, h1;\n\t"
      "mov.b64 T, {t0, t1};\n\t"
      "fma.rn.f32x2 SG, T, HF, HF;\n\t"
      "mul.rn.f32x2 XS, X, SG;\n\t"
      "mul.rn.f32x2 NX, N, XS;\n\t"
      "mul.rn.f32x2 A, NX, G;\n\t"
      "mov.b64 {a0, a1}, A;\n\t"
      "cvt.rn.bf16x2.f32 %1, a1, a0;\n\t"
      "mul.rn.f32x2 A, NX, Y;\n\t"
      "mov.b64 {a0, a1}, A;\n\t"
      "cvt.rn.bf16x2.f32 %2, a1, a0;\n\t"
      "mul.rn.f32x2 NG, N, G;\n\t"
      "mul.rn.f32x2 Q, NG, SG;\n\t"
      "mul.rn.f32x2 QY, Q, Y;\n\t"
      "sub.rn.f32x2 U, X, XS;\n\t"
      "fma.rn.f32x2 A, QY, U, QY;\n\t"
      "mov.b64 {a0, a1}, A;\n\t"
      "cvt.rn.bf16x2.f32 %0, a1, a0;\n\t"
      "}"
      : "=r"(o1), "=r"(o3), "=r"(om)
      : "r"(x0), "r"(x1), "r"(y0), "r"(y1), "r"(g0), "r"(g1), "f"(neta));
}
// Query tiles: Aq = silu(x) y.
TTT_DEVICE_INLINE uint32_t query_ops_x2(uint32_t x0, uint32_t x1, uint32_t y0, uint32_t y1) {
  uint32_t o;
  asm("{\n\t"
      ".reg .b64 X, Y, HF, H, T, SG, A;\n\t"
      ".reg .f32 h0, h1, t0, t1, a0, a1;\n\t"
      ".reg .b32 c;\n\t"
      "mov.b32 c, 0f3F000000;\n\t"
      "mov.b64 HF, {c, c};\n\t"
      "mov.b64 X, {%1, %2};\n\t"
      "mov.b64 Y, {%3, %4};\n\t"
      "mul.rn.f32x2 H, X, HF;\n\t"
      "mov.b64 {h0, h1}, H;\n\t"
      "tanh.approx.f32 t0, h0;\n\t"
      "tanh.approx.f32 t1, h1;\n\t"
      "mov.b64 T, {t0, t1};\n\t"
      "fma.rn.f32x2 SG, T, HF, HF;\n\t"
      "mul.rn.f32x2 A, X, SG;\n\t"
      "mul.rn.f32x2 A, A, Y;\n\t"
      "mov.b64 {a0, a1}, A;\n\t"
      "cvt.rn.bf16x2.f32 %0, a1, a0;\n\t"
      "}"
      : "=r"(o)
      : "r"(x0), "r"(x1), "r"(y0), "r"(y1));
  return o;
}
TTT_DEVICE_INLINE void mbar_arrive_n(uint64_t* bar, uint32_t n) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(n) : "memory");
}
// The row update of chunk c inside the chunk loop.  The worker of item
// (head bh, hidden block hb, token group grp) owns an even share (by token
// group) of the 64 rows of W1 and of W3 in block hb, and an even share (by
// item) of the head's 128 rows of W2, so the update waits only for the
// head's own items.  One epilogue warp per row, lane = four columns of each
// 128-column chunk; a warp's W1 and W3 rows go out together.  The token
// groups' partial sums are added in group order, then momentum, the step,
// the row L2 norm and the fp32 / bf16 stores: the arithmetic of the
// stand-alone GD / momentum row update.
TTT_DEVICE_INLINE float kg_warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}
TTT_DEVICE_INLINE float4 row_step(const KeyGradArgs& a, const KeyGradLoopArgs& la, int m, size_t c, float4 u, float4 w, float& ss) {
  if (la.opt == 1) {
    float4 mo = *reinterpret_cast<const float4*>(la.M[m] + c);
    mo.x = la.beta * mo.x + u.x; mo.y = la.beta * mo.y + u.y;
    mo.z = la.beta * mo.z + u.z; mo.w = la.beta * mo.w + u.w;
    *reinterpret_cast<float4*>(la.M[m] + c) = mo;
    u = mo;
  }
  w = make_float4(w.x - u.x, w.y - u.y, w.z - u.z, w.w - u.w);
  ss += w.x * w.x + w.y * w.y + w.z * w.z + w.w * w.w;
  return w;
}
// the scale of an updated row (1 without the row norm); with `norm`, the
// row's norm before the normalisation is recorded by lane 0
TTT_DEVICE_INLINE float row_scale(const KeyGradArgs& a, const KeyGradLoopArgs& la, float ss, float* norm) {
  if (!la.normalize) return 1.f;
  const float n = sqrtf(kg_warp_sum(ss));
  if (norm != nullptr && (threadIdx.x & 31) == 0) *norm = n;
  return 1.f / fmaxf(n, la.norm_eps);
}
TTT_DEVICE_INLINE void row_store(const KeyGradArgs& a, const KeyGradLoopArgs& la, int m, int nb, size_t c, float4 w, float scale,
                                 float* snap) {
  const float4 x = make_float4(w.x * scale, w.y * scale, w.z * scale, w.w * scale);
  *reinterpret_cast<float4*>(la.W[m] + c) = x;
  *reinterpret_cast<uint2*>(la.Wb[nb][m] + c) = make_uint2(pack_bf16x2(x.x, x.y), pack_bf16x2(x.z, x.w));
  if (snap != nullptr) *reinterpret_cast<float4*>(snap + c) = x;
}
TTT_DEVICE_INLINE void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// The rows a worker owns: W1 / W3 rows [lo13, lo13 + n13) of the head (its
// token group's share of hidden block hb) and W2 rows [lo2, lo2 + n2).
struct OwnRows {
  int lo13, n13, lo2, n2;
};
__host__ __device__ __forceinline__ OwnRows own_rows(const KeyGradArgs& a, const KeyGradLoopArgs& la, int hb, int grp) {
  const int G = a.n_groups, K = a.n_hb * G, k = hb * G + grp;
  OwnRows o;
  o.lo13 = hb * kg::HB + kg::HB * grp / G;
  o.n13 = kg::HB * (grp + 1) / G - kg::HB * grp / G;
  o.lo2 = kg::D * k / K;
  o.n2 = kg::D * (k + 1) / K - o.lo2;
  return o;
}
// bytes of one token group's partial sums for the owned rows (masked
// matrices take no room): [W1 rows | W3 rows | W2 rows], fp32
__host__ __device__ __forceinline__ uint32_t own_group_bytes(const KeyGradArgs& a, const KeyGradLoopArgs& la, const OwnRows& o) {
  return (uint32_t)(((la.mask & 1) ? o.n13 * kg::D : 0) + ((la.mask & 2) ? o.n13 * kg::D : 0) +
                    ((la.mask & 4) ? o.n2 * a.dh : 0)) * 4u;
}
// one thread: bring every token group's partial sums of the owned rows into
// shared memory (one bulk copy per group and matrix, completing on `bar`)
TTT_DEVICE_INLINE void own_partials_load(const KeyGradArgs& a, const KeyGradLoopArgs& la, int bh, const OwnRows& o, uint8_t* dst,
                                         uint64_t* bar) {
  const size_t mat_stride = (size_t)a.BH * a.dh * kg::D;
  const uint32_t gb = own_group_bytes(a, la, o);
  mbar_arrive_expect_tx(bar, gb * (uint32_t)a.n_groups);
  for (int sp = 0; sp < a.n_groups; ++sp) {
    uint8_t* d = dst + (size_t)sp * gb;
    for (int m = 0; m < 3; ++m) {
      if (!(la.mask & (1 << m))) continue;
      const size_t off = m < 2 ? ((size_t)bh * a.dh + o.lo13) * kg::D : ((size_t)bh * kg::D + o.lo2) * a.dh;
      const uint32_t bytes = (uint32_t)(m < 2 ? o.n13 * kg::D : o.n2 * a.dh) * 4u;
      bulk_g2s(d, a.part[m] + sp * mat_stride + off, bytes, bar);
      d += bytes;
    }
  }
}
// The row update of the owned rows, one epilogue warp per row (lane = four
// columns of each 128-column chunk), with the partial sums from shared
// memory (added in token-group order): momentum, the step, the row L2 norm
// and the fp32 / bf16 stores, the arithmetic of the stand-alone GD /
// momentum row update.
TTT_DEVICE_INLINE void loop_cast_rows(const KeyGradArgs& a, const KeyGradLoopArgs& la, int bh,
                                      const OwnRows& o, int e, int lane) {
  for (int m = 0; m < 3; ++m) {
    const int n = m < 2 ? o.n13 : o.n2, cols = m < 2 ? kg::D : a.dh;
    const size_t row0 = m < 2 ? (size_t)bh * a.dh + o.lo13 : (size_t)bh * kg::D + o.lo2;
    const int nb = (la.mask & (1 << m)) ? 1 : 3;
    for (int i = e; i < n; i += kg::EPI_WARPS)
      for (int c = 4 * lane; c < cols; c += 128) {
        const size_t off = (row0 + i) * cols + c;
        const float4 x = *reinterpret_cast<const float4*>(la.W[m] + off);
        const uint2 h = make_uint2(pack_bf16x2(x.x, x.y), pack_bf16x2(x.z, x.w));
        for (int b = 0; b < nb; ++b) *reinterpret_cast<uint2*>(la.Wb[b][m] + off) = h;
      }
  }
}
template <bool SNAP>
TTT_DEVICE_INLINE void loop_row_update(const KeyGradArgs& a, const KeyGradLoopArgs& la, int bh, const OwnRows& o, int e, int lane,
                                       int nb, const uint8_t* sp0, int c) {
  // SNAP (the backward's replay): the chunk's updated weights and row norms
  // are also kept; the forward's build of the kernel carries none of it
  const size_t mat_elems = (size_t)a.BH * a.dh * kg::D;
  auto snap = [&](int m) -> float* {
    if constexpr (SNAP)
      return la.wsave != nullptr ? la.wsave + (size_t)(c + 1) * 3 * mat_elems + (size_t)m * mat_elems : nullptr;
    return nullptr;
  };
  // row norms of chunk c: [BH][W1 rows | W3 rows | W2 rows]
  float* rn = nullptr;
  if constexpr (SNAP)
    if (la.rownorm != nullptr) rn = la.rownorm + ((size_t)c * a.BH + bh) * (2 * a.dh + kg::D);
  const uint32_t gb = own_group_bytes(a, la, o);
  auto psum = [&](uint32_t byte_off) {   // byte offset within one group's block
    float4 u = *reinterpret_cast<const float4*>(sp0 + byte_off);
    for (int sp = 1; sp < a.n_groups; ++sp) {
      const float4 x = *reinterpret_cast<const float4*>(sp0 + (size_t)sp * gb + byte_off);
      u.x += x.x; u.y += x.y; u.z += x.z; u.w += x.w;
    }
    return u;
  };
  uint32_t base = 0;   // this matrix's rows within a group's block
  for (int m = 0; m < 2; ++m) {
    if (!(la.mask & (1 << m))) continue;
    for (int i = e; i < o.n13; i += kg::EPI_WARPS) {
      const size_t c = ((size_t)bh * a.dh + o.lo13 + i) * kg::D + 4 * lane;
      const float4 w = *reinterpret_cast<const float4*>(la.W[m] + c);
      const float4 u = psum(base + (uint32_t)(i * kg::D + 4 * lane) * 4u);
      float ss = 0.f;
      const float4 x = row_step(a, la, m, c, u, w, ss);
      row_store(a, la, m, nb, c, x, row_scale(a, la, ss, rn ? rn + m * a.dh + o.lo13 + i : nullptr), snap(m));
    }
    base += (uint32_t)o.n13 * kg::D * 4u;
  }
  if (la.mask & 4) {
    const bool two = a.dh > 128;
    for (int i = e; i < o.n2; i += kg::EPI_WARPS) {
      const size_t c0 = ((size_t)bh * kg::D + o.lo2 + i) * a.dh + 4 * lane, c1 = c0 + 128;
      const uint32_t b0 = base + (uint32_t)(i * a.dh + 4 * lane) * 4u, b1 = b0 + 512u;
      float4 w0 = *reinterpret_cast<const float4*>(la.W[2] + c0);
      float4 w1 = two ? *reinterpret_cast<const float4*>(la.W[2] + c1) : w0;
      const float4 u0 = psum(b0);
      const float4 u1 = two ? psum(b1) : u0;
      float ss = 0.f;
      w0 = row_step(a, la, 2, c0, u0, w0, ss);
      if (two) w1 = row_step(a, la, 2, c1, u1, w1, ss);
      const float sc = row_scale(a, la, ss, rn ? rn + 2 * a.dh + o.lo2 + i : nullptr);
      row_store(a, la, 2, nb, c0, w0, sc, snap(2));
      if (two) row_store(a, la, 2, nb, c1, w1, sc, snap(2));
    }
  }
}

// LOOP = false: one chunk per launch (items over the grid, the row update is
// a separate kernel).  LOOP = true: one cooperative launch runs every chunk
// of a causal call.  CTAs [0, n_workers) each own one item and, after each
// chunk, a share of its head's weight rows: partial sums and Aq written ->
// the head's counter -> row update into the next bf16 buffer -> the head's
// update counter -> the next chunk's weights.  Heads never wait for each
// other.  The remaining CTAs are readers: once a head's counter shows its
// Aq of a chunk complete they form out = Aq W2^T for their share of the
// chunk's 128-token tiles (W2 of the chunk start, still in its bf16 buffer)
// and count themselves done on the readers' counter; a worker starts chunk
// c once the readers are done with chunk c - 2, whose Aq and W2 buffers
// chunk c reuses.
template <bool LOOP, bool SNAP = false>
__global__ void __launch_bounds__(kg::THREADS, 1)
    lact_keygrad_kernel(const __grid_constant__ KeyGradMaps maps, const KeyGradArgs a,
                        const __grid_constant__ KeyGradLoopArgs la) {
  using namespace kg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* kv_full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);   // [2]
  uint64_t* kv_empty = kv_full + 2;                                   // [2]
  uint64_t* w_full = kv_empty + 2;
  uint64_t* w_empty = w_full + 1;
  uint64_t* acc_full = w_empty + 1;    // [2]: per H13 buffer
  uint64_t* acc_empty = acc_full + 2;   // [2]
  uint64_t* dh_ready = acc_empty + 2;
  uint64_t* dh_free = dh_ready + 1;
  uint64_t* g_full = dh_free + 1;
  uint64_t* g_empty = g_full + 1;
  uint64_t* fin = g_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  uint32_t* abort_flag = tmem_slot + 1;
  // readers (chunk loop): W2 loaded, W2 free, Aq stage full / empty [2],
  // accumulator full / empty [2]
  uint64_t* r_w2_full = reinterpret_cast<uint64_t*>(smem + OFF_BAR + 128);
  uint64_t* r_w2_empty = r_w2_full + 1;
  uint64_t* r_a_full = r_w2_empty + 1;
  uint64_t* r_a_empty = r_a_full + 2;
  uint64_t* r_acc_full = r_a_empty + 2;
  uint64_t* r_acc_empty = r_acc_full + 2;
  uint64_t* upd_full = r_w2_full;   // workers (chunk loop): the row update's partial sums landed

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int items_per_bh = a.n_hb * a.n_groups;
  const int n_items = items_per_bh * a.BH;
  const int n_chunks = LOOP ? la.n_chunks : 1;
  const int stride = LOOP ? la.n_workers : (int)gridDim.x;
  const bool reader = LOOP && (int)blockIdx.x >= la.n_workers;
  unsigned* const gabort = LOOP ? la.ctr + 3 * a.BH + 1 : nullptr;
  auto ctr_part = [&](int bh) { return la.ctr + bh; };
  auto ctr_upd = [&](int bh) { return la.ctr + a.BH + bh; };
  auto ctr_aq = [&](int bh) { return la.ctr + 2 * a.BH + bh; };
  unsigned* const ctr_read = LOOP ? la.ctr + 3 * a.BH : nullptr;
  const unsigned per_head = (unsigned)items_per_bh;   // items (worker CTAs) of one head

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(w_full, 1);
    mbar_init(w_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], EPI_WARPS * 32);
    }
    mbar_init(dh_ready, EPI_WARPS * 32);
    mbar_init(dh_free, 1);
    mbar_init(g_full, 1);
    mbar_init(g_empty, EPI_WARPS * 32);
    mbar_init(fin, 1);
    if (LOOP) {
      mbar_init(r_w2_full, 1);
      mbar_init(r_w2_empty, 1);
      for (int b = 0; b < 2; ++b) {
        mbar_init(&r_a_full[b], 1);
        mbar_init(&r_a_empty[b], 1);
        mbar_init(&r_acc_full[b], 1);
        mbar_init(&r_acc_empty[b], EPI_WARPS * 32);
      }
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&maps.k);
    tma_prefetch_desc(&maps.v);
    if (a.queries) tma_prefetch_desc(&maps.q);
    for (int b = 0; b < (LOOP ? 3 : 1); ++b) {
      tma_prefetch_desc(&maps.w1[b]);
      tma_prefetch_desc(&maps.w3[b]);
      tma_prefetch_desc(&maps.w2[b]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // The TMA thread waits for the preceding kernels after it has issued its
  // first token tile (an input of the call, which no kernel of the call
  // writes); everything else waits here.
  if (warp != 0 || lane != 0) pdl_wait();
  const uint32_t tmem = *tmem_slot;
  Waiter W{abort_flag, a.st, 300};

  // the chunk a loop iteration works on (without the loop these read the
  // arguments directly, so nothing extra stays in registers)
  auto ct0 = [&](int c) { return LOOP ? a.t0 + c * a.C : a.t0; };
  auto cC = [&](int c) { return LOOP ? min(a.C, la.N - ct0(c)) : a.C; };
  auto ctiles = [&](int c) { return LOOP ? (cC(c) + BM - 1) / BM : a.tiles_total; };
  auto ctpg = [&](int c) { return LOOP ? (ctiles(c) + a.n_groups - 1) / a.n_groups : a.tiles_per_group; };
  auto cwb = [&](int c) { return LOOP ? c % 3 : 0; };
  auto caq = [&](int c) { return LOOP ? a.Aq + (size_t)(c & 1) * la.aq_buf : a.Aq; };
  auto decode = [&](int item, int& bh, int& hb, int& grp) {
    hb = item % a.n_hb;
    grp = (item / a.n_hb) % a.n_groups;
    bh = item / items_per_bh;
  };
  auto group_tiles = [&](int c, int grp) {
    const int tpg = ctpg(c);
    return std::max(0, std::min(tpg, ctiles(c) - grp * tpg));
  };

  if (reader) {
    // ============================================================ reader
    // Per tile of 128 tokens: out = Aq [128 x dh] W2^T [dh -> 128], K-major
    // operands (Aq rows, W2 rows of the bf16 copy), fp32 accumulator in
    // TMEM (two buffers), 16 epilogue warps convert and store.
    const int rr = (int)blockIdx.x - la.n_workers, R = (int)gridDim.x - la.n_workers;
    const uint32_t A_OFF = 65536, A_STAGE = 65536;   // W2 at 0 (64 KB), two Aq stages
    const int kblocks = a.dh / 64;
    auto tile_range = [&](int c, int& lo, int& hi) {
      const int T = a.BH * ctiles(c);
      lo = (int)((long long)rr * T / R);
      hi = (int)((long long)(rr + 1) * T / R);
    };
    if (warp == 0) {
      if (lane == 0) {
        uint32_t at = 0, wl = 0;
        bool ok = true;
        for (int c = 0; ok && c < n_chunks; ++c) {
            int lo, hi;
          tile_range(c, lo, hi);
          int cur_bh = -1;
          for (int t = lo; ok && t < hi; ++t) {
            const int bh = t / ctiles(c), mt = t % ctiles(c);
            if (bh != cur_bh) {
              // the head's Aq of this chunk is complete (and W2 of its start
              // was written before the head began the chunk)
              if (!grid_wait(ctr_aq(bh), per_head * (c + 1), W, 20, gabort)) { ok = false; break; }
              fence_proxy_async_global();
              if (wl >= 1 && !W.wait(r_w2_empty, (wl - 1) & 1, 21)) { ok = false; break; }
              mbar_arrive_expect_tx(r_w2_full, (uint32_t)kblocks * 16384u);
              for (int kb = 0; kb < kblocks; ++kb)
                tma_load_3d(smem + kb * 16384, &maps.w2k[cwb(c)], r_w2_full, kb * 64, 0, bh);
              ++wl;
              cur_bh = bh;
            }
            const uint32_t s = at & 1;
            if (at >= 2 && !W.wait(&r_a_empty[s], ((at >> 1) - 1) & 1, 22)) { ok = false; break; }
            mbar_arrive_expect_tx(&r_a_full[s], (uint32_t)kblocks * 16384u);
            for (int kb = 0; kb < kblocks; ++kb)
              tma_load_3d(smem + A_OFF + s * A_STAGE + kb * 16384, &maps.aq[c & 1], &r_a_full[s],
                          kb * 64, mt * BM, bh);
            ++at;
          }
        }
        if (W.aborted()) {   // copies still in flight land before the CTA exits
          const uint32_t first = at > 2 ? at - 2 : 0;
          for (uint32_t i = first; i < at; ++i) W.drain(&r_a_full[i & 1], (i >> 1) & 1);
          if (wl >= 1) W.drain(r_w2_full, (wl - 1) & 1);
        }
      }
      __syncwarp();
    } else if (warp == 1) {
      if (lane == 0) {
        const uint32_t idr = make_idesc(128, 128, false, false);
        const uint64_t dw2 = make_sdesc(smem_u32(smem), 16, 1024);
        const uint64_t dat = make_sdesc(smem_u32(smem + A_OFF), 16, 1024);
        uint32_t at = 0, wu = 0;
        bool ok = true;
        for (int c = 0; ok && c < n_chunks; ++c) {
            int lo, hi;
          tile_range(c, lo, hi);
          int cur_bh = -1;
          for (int t = lo; ok && t < hi; ++t) {
            const int bh = t / ctiles(c);
            if (bh != cur_bh) {
              if (wu >= 1) mma_commit(r_w2_empty);   // after every product on the previous W2
              if (!W.wait(r_w2_full, wu & 1, 23)) { ok = false; break; }
              ++wu;
              cur_bh = bh;
            }
            const uint32_t s = at & 1;
            if (!W.wait(&r_a_full[s], (at >> 1) & 1, 24)) { ok = false; break; }
            if (at >= 2 && !W.wait(&r_acc_empty[s], ((at >> 1) - 1) & 1, 25)) { ok = false; break; }
            tc_fence_after();
            for (int kk = 0; kk < kblocks * 4; ++kk) {
              const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
              mma_bf16(tmem + s * 128, sdesc_add(dat, s * A_STAGE + off), sdesc_add(dw2, off), idr, kk > 0);
            }
            mma_commit(&r_a_empty[s]);
            mma_commit(&r_acc_full[s]);
            ++at;
          }
        }
        mma_commit(fin);
        W.drain(fin, 0);
      }
      __syncwarp();
    } else {
      const int q4 = warp & 3;
      const int cg = (warp - 2) >> 2;                 // 32-column group of the 128 outputs
      const int r = q4 * 32 + lane;
      const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
      uint32_t at = 0;
      for (int c = 0; c < n_chunks; ++c) {
        int lo, hi;
        tile_range(c, lo, hi);
        bool ok = true;
        for (int t = lo; t < hi; ++t, ++at) {
          const int bh = t / ctiles(c), mt = t % ctiles(c);
          const uint32_t s = at & 1;
          if (!W.wait(&r_acc_full[s], (at >> 1) & 1, 26)) { ok = false; break; }
          tc_fence_after();
          float o[32];
          tmem_ld32(tmem + lane_base + s * 128 + cg * 32, o);
          tc_fence_before();
          mbar_arrive(&r_acc_empty[s]);
          const int row = mt * BM + r;
          if (row < cC(c)) {
            const size_t base = (size_t)bh * la.out_bs + (size_t)(ct0(c) + row) * D + cg * 32;
            if (la.out_bf16) {
              uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(la.out) + base);
#pragma unroll
              for (int j = 0; j < 4; ++j)
                dst[j] = make_uint4(pack_bf16x2(o[8 * j], o[8 * j + 1]), pack_bf16x2(o[8 * j + 2], o[8 * j + 3]),
                                    pack_bf16x2(o[8 * j + 4], o[8 * j + 5]), pack_bf16x2(o[8 * j + 6], o[8 * j + 7]));
            } else {
              float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(la.out) + base);
#pragma unroll
              for (int j = 0; j < 8; ++j) dst[j] = make_float4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
            }
          }
        }
        // every product of this chunk has completed (its accumulators were
        // read), so the chunk's Aq and W2 buffers may be reused
        named_bar_sync(1, EPI_WARPS * 32);
        if (!ok || W.aborted()) break;
        if (threadIdx.x == 64) red_release_gpu_add(ctr_read, 1u);
      }
    }
  } else if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      uint32_t tile = 0, item_ctr = 0;
      bool ok = true;
      for (int c = 0; ok && c < n_chunks; ++c) {
        // tile i of an item: key tiles (K and V) first, then query tiles (Q
        // in the K slot)
        auto issue_tile = [&](uint32_t t, int i, int nt, int bh, int grp) {
          const uint32_t s = t & 1;
          const bool is_q = i >= nt;
          const int row = ct0(c) + (grp * ctpg(c) + (is_q ? i - nt : i)) * BM;
          uint8_t* st = smem + OFF_KV + s * KV_STAGE;
          if (is_q) {
            mbar_arrive_expect_tx(&kv_full[s], TILE);
            tma_load_3d(st, &maps.q, &kv_full[s], 0, row, bh);
            tma_load_3d(st + HALF, &maps.q, &kv_full[s], 64, row, bh);
          } else {
            mbar_arrive_expect_tx(&kv_full[s], KV_STAGE);
            tma_load_3d(st, &maps.k, &kv_full[s], 0, row, bh);
            tma_load_3d(st + HALF, &maps.k, &kv_full[s], 64, row, bh);
            tma_load_3d(st + TILE, &maps.v, &kv_full[s], 0, row, bh);
            tma_load_3d(st + TILE + HALF, &maps.v, &kv_full[s], 64, row, bh);
          }
        };
        for (int item = blockIdx.x; ok && item < n_items; item += stride, ++item_ctr) {
          int bh, hb, grp;
          decode(item, bh, hb, grp);
          const int j0 = hb * HB;
          const int nt = group_tiles(c, grp);
          const int n_all = nt + (a.queries ? nt : 0);
          // the item's first tile goes out before any wait on other work (it
          // overlaps the preceding kernel's tail or the last row update); the
          // second follows the weights, so they do not queue behind it
          if (n_all > 0) {
            if (tile >= 2 && !W.wait(&kv_empty[tile & 1], ((tile >> 1) - 1) & 1, 2)) { ok = false; break; }
            issue_tile(tile, 0, nt, bh, grp);
            ++tile;
          }
          if (c == 0 && item_ctr == 0) pdl_wait();
          if (LOOP && (c > 0 || la.cast_first) && item == (int)blockIdx.x) {
            // the head's row updates of chunk c - 1 (and the start copies)
            if (!grid_wait(ctr_upd(bh), per_head * (c + la.cast_first), W, 3, gabort)) { ok = false; break; }
            fence_proxy_async_global();
          }
          if (item_ctr >= 1 && !W.wait(w_empty, (item_ctr - 1) & 1, 1)) { ok = false; break; }
          // weights of the item: [W1_J; W3_J] as two K atoms (d 0-63, 64-127),
          // W2[:, J] as 128 d-rows of 64 hidden units
          mbar_arrive_expect_tx(w_full, 2 * HALF + 2 * 8192);
          for (int atom = 0; atom < 2; ++atom) {
            tma_load_3d(smem + OFF_W13 + atom * HALF, &maps.w1[cwb(c)], w_full, atom * 64, j0, bh);
            tma_load_3d(smem + OFF_W13 + atom * HALF + HALF / 2, &maps.w3[cwb(c)], w_full, atom * 64, j0, bh);
            tma_load_3d(smem + OFF_W2 + atom * 8192, &maps.w2[cwb(c)], w_full, j0, atom * 64, bh);
          }
          for (int i = 1; ok && i < n_all; ++i, ++tile) {
            const uint32_t s = tile & 1;
            if (tile >= 2 && !W.wait(&kv_empty[s], ((tile >> 1) - 1) & 1, 2)) { ok = false; break; }
            issue_tile(tile, i, nt, bh, grp);
            if (i == 1)   // warm L2 with the later key tiles; their loads then hit it
              for (int k = 2; k < nt; ++k)
                for (int h = 0; h < 2; ++h) {
                  const int row = ct0(c) + (grp * ctpg(c) + k) * BM;
                  tma_prefetch_l2_3d(&maps.k, h * 64, row, bh);
                  tma_prefetch_l2_3d(&maps.v, h * 64, row, bh);
                }
          }
        }
      }
      if (W.aborted()) {
        const uint32_t first = tile > 2 ? tile - 2 : 0;
        for (uint32_t i = first; i < tile; ++i) W.drain(&kv_full[i & 1], (i >> 1) & 1);
      }
    }
    // the other lanes wait here for lane 0 (not at the block barrier below)
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    // One thread issues every MMA.  Within an item it polls the readiness of
    // the next forward product and of the next gradient product and issues
    // whichever can go, so a gradient whose operands are ready never waits
    // behind a forward product that waits for its tile.
    if (lane == 0) {
      const uint32_t id_h = make_idesc(128, 128, false, false);
      const uint32_t id_g = make_idesc(128, 64, false, true);
      const uint32_t id_g13 = make_idesc(128, 128, true, true);
      const uint32_t id_g2 = make_idesc(128, 64, true, true);
      const uint32_t kvb = smem_u32(smem + OFF_KV);
      const uint32_t w13 = smem_u32(smem + OFF_W13), w2 = smem_u32(smem + OFF_W2);
      const uint32_t dhb = smem_u32(smem + OFF_DH);
      uint32_t tile = 0, ktile = 0, item_ctr = 0;   // all tiles / key tiles of this CTA
      bool ok = true;
      // tile t can take its forward product: its tile has landed, its H13
      // buffer was read by the epilogue (tile t - 2) and, for a key tile, so
      // was dGr (tile t - 1)
      auto fwd_ready = [&](uint32_t t, bool is_key) -> bool {
        if (!mbar_test(&kv_full[t & 1], (t >> 1) & 1)) return false;
        if (t >= 2 && !mbar_test(&acc_empty[t & 1], ((t >> 1) - 1) & 1)) return false;
        if (is_key && t >= 1 && !mbar_test(&acc_empty[(t - 1) & 1], ((t - 1) >> 1) & 1)) return false;
        return true;
      };
      // H13 (+ dGr for key tiles) of tile t into its H13 buffer
      // descriptor bases, advanced by constant byte offsets
      const uint64_t dkv_k = make_sdesc(kvb, 16, 1024), dkv_mn = make_sdesc(kvb, HALF, 1024);
      const uint64_t dw13 = make_sdesc(w13, 16, 1024), dw2 = make_sdesc(w2, 8192, 1024);
      const uint64_t ddh13 = make_sdesc(dhb, HALF, 1024), dgm = make_sdesc(dhb + 2 * HALF, 8192, 1024);
      auto forward = [&](uint32_t t, bool is_key) {
        tc_fence_after();
        const uint32_t s = t & 1;
        const uint64_t dk = sdesc_add(dkv_k, s * KV_STAGE), dv = sdesc_add(dk, TILE);
        const uint32_t acc = tmem + (s ? TM_H13B : TM_H13A);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * HALF + (kk & 3) * 32;
          mma_bf16(acc, sdesc_add(dk, off), sdesc_add(dw13, off), id_h, kk > 0);
          if (is_key) mma_bf16(tmem + TM_DG, sdesc_add(dv, off), sdesc_add(dw2, kk * 2048), id_g, kk > 0);
        }
        mma_commit(&acc_full[s]);
        if (!is_key) mma_commit(&kv_empty[s]);   // a query tile is done with its stage
      };
      // gradient products of the key tile in stage t & 1
      auto grads = [&](uint32_t t, bool first) {
        tc_fence_after();
        const uint64_t dk = sdesc_add(dkv_mn, (t & 1) * KV_STAGE), dv = sdesc_add(dk, TILE);
        // K^T / V^T as MN-major A: M = d in two 64-wide blocks 16 KB apart,
        // K = tokens (rows of 128 B); [dH1 | dH3] as MN-major B with its two
        // 64-wide blocks 16 KB apart (N = 128), Gm' as N = 64
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t acc = (first && kk == 0) ? 0u : 1u;
          mma_bf16(tmem + TM_G13, sdesc_add(dk, kk * 2048), sdesc_add(ddh13, kk * 2048), id_g13, acc);
          mma_bf16(tmem + TM_G2, sdesc_add(dv, kk * 2048), sdesc_add(dgm, kk * 2048), id_g2, acc);
        }
        mma_commit(dh_free);
        mma_commit(&kv_empty[t & 1]);
      };
      for (int c = 0; ok && c < n_chunks; ++c) {
        for (int item = blockIdx.x; ok && item < n_items; item += stride, ++item_ctr) {
          int bh, hb, grp;
          decode(item, bh, hb, grp);
          const int nt = group_tiles(c, grp);
          const int nq = a.queries ? nt : 0;
          if (!W.wait(w_full, item_ctr & 1, 5)) { ok = false; break; }
          // key tiles first, then the query tiles
          int nf = 0, ng = 0;   // forward / gradient products issued in this item
          uint64_t t_idle = 0;
          uint32_t spins = 0;
          while (nf < nt + nq || ng < nt) {
            bool prog = false;
            // the next key tile's gradient: its forward is issued and its dH is
            // staged (the accumulators were read out after the previous item)
            if (ng < nt && ng < nf) {
              const bool first = ng == 0;
              if ((!first || item_ctr == 0 || mbar_test(g_empty, (item_ctr - 1) & 1)) &&
                  mbar_test(dh_ready, (ktile + ng) & 1)) {
                grads(tile + ng, first);
                ++ng;
                prog = true;
                if (ng == nt) mma_commit(g_full);
              }
            }
            if (nf < nt + nq) {
              const bool is_key = nf < nt;
              if (fwd_ready(tile + nf, is_key)) {
                forward(tile + nf, is_key);
                ++nf;
                prog = true;
              }
            }
            if (prog) {
              spins = 0;
              t_idle = 0;
              continue;
            }
            // plain polling (a short sleep here measured slower: every issue on
            // the per-tile chain waits for the wake-up)
            if ((++spins & 255u) == 0u) {   // bounded: give up after the wait timeout
              if (W.aborted()) { ok = false; break; }
              const uint64_t now = globaltimer_ns();
              if (t_idle == 0) t_idle = now;
              else if (now - t_idle > W.st.timeout_ns) { W.fail(15); ok = false; break; }
            }
          }
          if (!ok) break;
          if (nt == 0) mma_commit(g_full);
          tile += nt + nq;
          ktile += nt;
          mma_commit(w_empty);
        }
      }
      mma_commit(fin);
      W.drain(fin, 0);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q4 = warp & 3;
    const int cg = (warp - 2) >> 2;                 // 16-column group of the 64 hidden
    const int r = q4 * 32 + lane;                   // token row of the tile / d row of G
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    uint8_t* dh1s = smem + OFF_DH;
    const uint32_t dh1 = smem_u32(dh1s), dh3 = dh1 + HALF, gms = dh1 + 2 * HALF;
    uint32_t tile = 0, ktile = 0, item_ctr = 0;
    if (LOOP && la.cast_first) {
      // the start weights' bf16 copies of the owned rows (buffer 0, and every
      // buffer for a matrix the update leaves alone), published like an update
      int bh, hb, grp;
      decode((int)blockIdx.x, bh, hb, grp);
      loop_cast_rows(a, la, bh, own_rows(a, la, hb, grp), warp - 2, lane);
      fence_proxy_async_global();
      named_bar_sync(1, EPI_WARPS * 32);
      if (threadIdx.x == 64) red_release_gpu_add(ctr_upd(bh), 1u);
    }
    for (int c = 0; c < n_chunks; ++c) {
      if (LOOP && c >= 2) {
        // chunk c rewrites the Aq buffer and (in its update) the W buffer of
        // chunk c - 2: the readers must be done with that chunk
        if (threadIdx.x == 64)
          grid_wait(ctr_read, (unsigned)((int)gridDim.x - la.n_workers) * (c - 1), W, 12, gabort);
        named_bar_sync(1, EPI_WARPS * 32);
        if (W.aborted()) break;
      }
      bool ok = true;
      for (int item = blockIdx.x; item < n_items; item += stride, ++item_ctr) {
        int bh, hb, grp;
        decode(item, bh, hb, grp);
        const int nt = group_tiles(c, grp);
        const int nq = a.queries ? nt : 0;
        for (int i = 0; i < nt; ++i, ++tile, ++ktile) {
          const int tc = (grp * ctpg(c) + i) * BM + r;   // token row in the chunk
          const bool valid = tc < cC(c);
          // -eta, zero for rows past the chunk (their H and dGr are finite, so
          // every gradient operand of such a row comes out zero)
          const float neta = valid ? -a.lr[(size_t)bh * a.lr_len + ct0(c) + tc] : 0.f;
          if (!W.wait(&acc_full[tile & 1], (tile >> 1) & 1, 8)) { ok = false; break; }
          tc_fence_after();
          uint32_t rh1[CW], rh3[CW], rg[CW];
          const uint32_t tb = tmem + lane_base + cg * CW;
          const uint32_t th = tb + ((tile & 1) ? TM_H13B : TM_H13A);
          tmem_ld16_issue(th, rh1);
          tmem_ld16_issue(th + 64, rh3);
          tmem_ld16_issue(tb + TM_DG, rg);
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(&acc_empty[tile & 1]);
          uint32_t o1[CW / 2], o3[CW / 2], om[CW / 2];
#pragma unroll
          for (int j = 0; j < CW; j += 2)
            key_ops_x2(rh1[j], rh1[j + 1], rh3[j], rh3[j + 1], rg[j], rg[j + 1], neta, o1[j >> 1],
                       o3[j >> 1], om[j >> 1]);
          // the previous key tile's gradient MMAs must be done reading dH
          if (ktile >= 1 && !W.wait(dh_free, (ktile - 1) & 1, 9)) { ok = false; break; }
#pragma unroll
          for (int j = 0; j < CW; j += 8) {
            const uint32_t off = sw128_offset(r, cg * CW + j);
            st_shared_v4(dh1 + off, o1[j / 2], o1[j / 2 + 1], o1[j / 2 + 2], o1[j / 2 + 3]);
            st_shared_v4(dh3 + off, o3[j / 2], o3[j / 2 + 1], o3[j / 2 + 2], o3[j / 2 + 3]);
            st_shared_v4(gms + off, om[j / 2], om[j / 2 + 1], om[j / 2 + 2], om[j / 2 + 3]);
          }
          fence_async_smem();
          tc_fence_before();
          mbar_arrive(dh_ready);
        }
        // After the key tiles the epilogue splits: column groups 0-1 move the
        // item's gradient sums to its token-group slot while groups 2-3 form
        // the query tiles' Aq, each for all 64 hidden columns (two 16-column
        // blocks per warp), so the two streams of stores overlap.
        if (ok && nt > 0) {
          if (cg < 2) {
            if (!W.wait(g_full, item_ctr & 1, 10)) {
              ok = false;
            } else {
              tc_fence_after();
              const size_t mat_stride = (size_t)a.BH * a.dh * D;
              const size_t slot = (size_t)grp * mat_stride;
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int c0 = (cg * 2 + h) * CW;
                const int j0 = hb * HB + c0;
                uint32_t g1[CW], g3[CW], g2[CW];
                tmem_ld16_issue(tmem + lane_base + TM_G13 + c0, g1);
                tmem_ld16_issue(tmem + lane_base + TM_G13 + HB + c0, g3);
                tmem_ld16_issue(tmem + lane_base + TM_G2 + c0, g2);
                tmem_wait_ld();
                if (h == 1) {
                  tc_fence_before();
                  mbar_arrive_n(g_empty, 2);
                }
                // G1, G3 [BH][dh][d]: this thread is d row r -> element (j0 + j, r)
                float* p1 = a.part[0] + slot + ((size_t)bh * a.dh + j0) * D + r;
                float* p3 = a.part[1] + slot + ((size_t)bh * a.dh + j0) * D + r;
#pragma unroll
                for (int j = 0; j < CW; ++j) {
                  p1[(size_t)j * D] = __uint_as_float(g1[j]);
                  p3[(size_t)j * D] = __uint_as_float(g3[j]);
                }
                // G2 [BH][d][dh]: row r, columns j0 .. j0 + CW - 1
                float4* p2 = reinterpret_cast<float4*>(a.part[2] + slot + ((size_t)bh * D + r) * a.dh + j0);
#pragma unroll
                for (int j = 0; j < CW / 4; ++j)
                  p2[j] = make_float4(__uint_as_float(g2[4 * j]), __uint_as_float(g2[4 * j + 1]),
                                      __uint_as_float(g2[4 * j + 2]), __uint_as_float(g2[4 * j + 3]));
              }
            }
            tile += nq;
          } else {
            // query tiles (causal): Aq = silu(Q W1^T) * (Q W3^T) -> bf16
            for (int i = 0; i < nq; ++i, ++tile) {
              const int tc = (grp * ctpg(c) + i) * BM + r;
              const bool valid = tc < cC(c);
              if (!W.wait(&acc_full[tile & 1], (tile >> 1) & 1, 11)) { ok = false; break; }
              tc_fence_after();
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int c0 = ((cg - 2) * 2 + h) * CW;
                uint32_t rh1[CW], rh3[CW];
                const uint32_t tb = tmem + lane_base + c0 + ((tile & 1) ? TM_H13B : TM_H13A);
                tmem_ld16_issue(tb, rh1);
                tmem_ld16_issue(tb + 64, rh3);
                tmem_wait_ld();
                if (h == 1) {
                  tc_fence_before();
                  mbar_arrive_n(&acc_empty[tile & 1], 2);
                }
                if (valid) {
                  uint32_t oq[CW / 2];
#pragma unroll
                  for (int j = 0; j < CW; j += 2)
                    oq[j >> 1] = query_ops_x2(rh1[j], rh1[j + 1], rh3[j], rh3[j + 1]);
                  uint4* dq = reinterpret_cast<uint4*>(caq(c) + (size_t)bh * a.aq_bs + (size_t)tc * a.dh +
                                                       hb * HB + c0);
#pragma unroll
                  for (int j = 0; j < CW / 8; ++j) dq[j] = make_uint4(oq[4 * j], oq[4 * j + 1], oq[4 * j + 2], oq[4 * j + 3]);
                }
              }
            }
          }
        }
        if (LOOP) {
          // Each half publishes what it wrote as soon as it is done: the
          // partial sums (read by the head's row updates) and Aq (read by
          // the readers).  The half's barrier orders its threads' stores
          // before the one release add; the proxy fence orders them before
          // the bulk / TMA copies that read them.  Every thread of a half
          // reaches its barrier, also after a failed wait.
          fence_proxy_async_global();
          if (cg < 2) {
            named_bar_sync(2, EPI_WARPS * 16);
            if (threadIdx.x == 64 && !W.aborted()) red_release_gpu_add(ctr_part(bh), 1u);
          } else {
            named_bar_sync(3, EPI_WARPS * 16);
            if (threadIdx.x == 320 && !W.aborted()) red_release_gpu_add(ctr_aq(bh), 1u);
          }
        }
        // both halves finish the item before either starts the next one, so no
        // epilogue warp waits on an accumulator phase two uses ahead; every
        // epilogue thread reaches this barrier, also after a failed wait
        named_bar_sync(1, EPI_WARPS * 32);
        if (!ok || W.aborted()) break;
      }
      if (!ok || W.aborted()) break;
      if (LOOP) {
        // the row update: once every item of the head has published its
        // partial sums, bring the owned rows' sums into shared memory (the
        // weight tiles' and dH's, free until the next chunk's weights load,
        // which waits for this update)
        int bh, hb, grp;
        decode((int)blockIdx.x, bh, hb, grp);
        const OwnRows own = own_rows(a, la, hb, grp);
        if (threadIdx.x == 64) {
          if (own_group_bytes(a, la, own) * (uint32_t)a.n_groups > LOOP_PART_BYTES) {
            W.fail(16);   // the host plan rules this out
          } else if (grid_wait(ctr_part(bh), per_head * (c + 1), W, 13, gabort)) {
            fence_proxy_async_global();
            own_partials_load(a, la, bh, own, smem + OFF_W13, upd_full);
          }
        }
        named_bar_sync(1, EPI_WARPS * 32);
        if (W.aborted()) break;
        if (!W.wait(upd_full, c & 1, 14)) break;
        loop_row_update<SNAP>(a, la, bh, own, warp - 2, lane, (c + 1) % 3, smem + OFF_W13, c);
        // the next chunk's weights: read by TMA in the head's workers
        fence_proxy_async_global();
        named_bar_sync(1, EPI_WARPS * 32);
        if (threadIdx.x == 64) red_release_gpu_add(ctr_upd(bh), 1u);
        if (W.aborted()) break;
      }
    }
  }
  // dependents (the row update) may start launching once this CTA is done
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TM_COLS);
  }
}

// Token groups per chunk: enough items (BH x dh/64 x groups) to fill the
// SMs, and never an empty group (every slot of the partial sums is written).
int keygrad_groups(int BH, int dh, int C, int max_groups) {
  const int n_hb = dh / kg::HB;
  const int tiles = std::max(1, (C + kg::BM - 1) / kg::BM);
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (sms <= 0) sms = 148;
  int g = std::max(1, std::min(sms / std::max(1, BH * n_hb), tiles));
  if (max_groups > 0) g = std::min(g, max_groups);
  const int tpg = (tiles + g - 1) / g;
  return (tiles + tpg - 1) / tpg;
}

static int keygrad_maps(KeyGradMaps& m, int BH_, int N_in, int dh, const void* k, const void* v,
                        const void* q) {
  const uint64_t BH = (uint64_t)BH_;
  const uint64_t tok_row = (uint64_t)kg::D * 2;
  if (make_tmap_bf16_3d(&m.k, k, kg::D, N_in, BH, tok_row, tok_row * N_in, 64, 128) ||
      make_tmap_bf16_3d(&m.v, v, kg::D, N_in, BH, tok_row, tok_row * N_in, 64, 128) ||
      make_tmap_bf16_3d(&m.q, q ? q : k, kg::D, N_in, BH, tok_row, tok_row * N_in, 64, 128))
    return -1;
  (void)dh;
  return 0;
}
static int keygrad_weight_maps(KeyGradMaps& m, int b, int BH_, int dh, const void* w1b,
                               const void* w3b, const void* w2b) {
  const uint64_t BH = (uint64_t)BH_;
  const uint64_t tok_row = (uint64_t)kg::D * 2;
  return make_tmap_bf16_3d(&m.w1[b], w1b, kg::D, dh, BH, tok_row, tok_row * dh, 64, 64) ||
                 make_tmap_bf16_3d(&m.w3[b], w3b, kg::D, dh, BH, tok_row, tok_row * dh, 64, 64) ||
                 make_tmap_bf16_3d(&m.w2[b], w2b, dh, kg::D, BH, (uint64_t)dh * 2,
                                   (uint64_t)dh * 2 * kg::D, 64, 64)
             ? -1
             : 0;
}

int launch_lact_keygrad(const KeyGradLaunch& L, cudaStream_t stream) {
  KeyGradMaps m{};
  if (keygrad_maps(m, L.BH, L.N_in, L.dh, L.k, L.v, L.q) ||
      keygrad_weight_maps(m, 0, L.BH, L.dh, L.w1b, L.w3b, L.w2b))
    return -1;
  KeyGradArgs a{};
  a.BH = L.BH; a.C = L.C; a.t0 = L.t0; a.lr_len = L.N_in; a.dh = L.dh;
  a.n_hb = L.dh / kg::HB;
  a.tiles_total = (L.C + kg::BM - 1) / kg::BM;
  a.n_groups = L.groups;
  a.tiles_per_group = (a.tiles_total + a.n_groups - 1) / a.n_groups;
  if ((a.n_groups - 1) * a.tiles_per_group >= a.tiles_total) return -1;   // empty group
  a.lr = L.lr;
  a.part[0] = L.part[0]; a.part[1] = L.part[1]; a.part[2] = L.part[2];
  a.queries = L.q != nullptr ? 1 : 0;
  a.Aq = L.Aq;
  a.aq_bs = L.aq_bs;
  a.st = L.st;
  static std::atomic<uint64_t> attr{0};
  if (allow_dynamic_smem(lact_keygrad_kernel<false>, (int)kg::SMEM, attr)) return -1;
  const int items = a.n_hb * a.n_groups * L.BH;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  prof_before(K_KEYGRAD, stream);
  if (launch_pdl(lact_keygrad_kernel<false>, dim3(std::min(items, sms)), dim3(kg::THREADS), kg::SMEM,
                 stream, m, a, KeyGradLoopArgs{}) != cudaSuccess)
    return -1;
  prof_after(K_KEYGRAD, stream);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

// Readers the chunk loop needs at least: fewer spare SMs than this and the
// per-chunk launches (reads on the SMs the fused kernel leaves free) win.
constexpr int kLoopMinReaders = 8;

int lact_loop_plan(int BH, int N_in, int C, int dh, int max_groups, int* groups, int* workers,
                   int* readers) {
  if (dh % 128 != 0 || dh > 256 || C <= 0 || N_in <= 0) return -1;
  int sms = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    return -1;
  int coop = 0;
  if (cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess || !coop) return -1;
  const int g = keygrad_groups(BH, dh, C, max_groups);
  // every chunk, the last (possibly shorter) one included, must fill all g
  // token groups, since each group's slot of the partial sums is read back
  const int n_chunks = (N_in + C - 1) / C;
  for (const int len : {std::min(C, N_in), N_in - (n_chunks - 1) * C}) {   // full chunks and the last
    const int tiles = (len + kg::BM - 1) / kg::BM;
    const int tpg = (tiles + g - 1) / g;
    if ((g - 1) * tpg >= tiles) return -1;
  }
  const int items = BH * (dh / kg::HB) * g;
  if (items + kLoopMinReaders > sms) return -1;
  // every worker's share of the partial sums fits the shared memory the
  // update uses (all three matrices counted)
  {
    KeyGradArgs t{};
    KeyGradLoopArgs tl{};
    t.BH = BH; t.dh = dh; t.n_hb = dh / kg::HB; t.n_groups = g; tl.mask = 7;
    for (int hb = 0; hb < t.n_hb; ++hb)
      for (int grp = 0; grp < g; ++grp)
        if (own_group_bytes(t, tl, own_rows(t, tl, hb, grp)) * (uint32_t)g > kg::LOOP_PART_BYTES) return -1;
  }
  static std::atomic<uint64_t> attr{0};
  if (allow_dynamic_smem(lact_keygrad_kernel<true>, (int)kg::SMEM, attr)) return -1;
  static std::atomic<uint64_t> attr_snap{0};
  if (allow_dynamic_smem(lact_keygrad_kernel<true, true>, (int)kg::SMEM, attr_snap)) return -1;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, lact_keygrad_kernel<true>, kg::THREADS,
                                                    kg::SMEM) != cudaSuccess ||
      per_sm < 1)
    return -1;
  *groups = g;
  *workers = items;
  *readers = sms - items;
  return 0;
}

int launch_lact_loop(const KeyGradLoopLaunch& L, cudaStream_t stream) {
  // the caller's plan (lact_loop_plan), else this call's
  int g = L.groups, nw = L.workers, nr = L.readers;
  const bool reads = L.q != nullptr;   // without queries there is nothing to read out
  if ((g <= 0 || nw <= 0 || (reads && nr <= 0)) &&
      lact_loop_plan(L.BH, L.N_in, L.C, L.dh, L.max_groups, &g, &nw, &nr))
    return -1;
  if (!reads) nr = 0;
  KeyGradMaps m{};
  if (keygrad_maps(m, L.BH, L.N_in, L.dh, L.k, L.v, L.q)) return -1;
  const uint64_t BH = (uint64_t)L.BH;
  for (int b = 0; b < 3; ++b) {
    if (keygrad_weight_maps(m, b, L.BH, L.dh, L.Wb[b][0], L.Wb[b][1], L.Wb[b][2])) return -1;
    // W2 [BH][d][dh] as the K-major B of the read (N = d, K = dh)
    if (make_tmap_bf16_3d(&m.w2k[b], L.Wb[b][2], L.dh, kg::D, BH, (uint64_t)L.dh * 2,
                          (uint64_t)L.dh * 2 * kg::D, 64, 128))
      return -1;
  }
  for (int b = 0; b < 2; ++b)
    if (make_tmap_bf16_3d(&m.aq[b], L.Aq + (size_t)b * L.aq_buf, L.dh, L.cmax, BH,
                          (uint64_t)L.dh * 2, (uint64_t)L.cmax * L.dh * 2, 64, 128))
      return -1;
  KeyGradArgs a{};
  KeyGradLoopArgs la{};
  a.BH = L.BH; a.C = L.C; a.t0 = 0; a.lr_len = L.N_in; a.dh = L.dh;
  a.n_hb = L.dh / kg::HB;
  a.n_groups = g;
  a.lr = L.lr;
  for (int i = 0; i < 3; ++i) {
    a.part[i] = L.part[i];
    la.W[i] = L.W[i];
    la.M[i] = L.M[i];
    for (int b = 0; b < 3; ++b) la.Wb[b][i] = L.Wb[b][i];
  }
  a.queries = reads ? 1 : 0;
  a.Aq = L.Aq;
  a.aq_bs = (long long)L.cmax * L.dh;
  la.aq_buf = L.aq_buf;
  a.st = L.st;
  la.n_chunks = (L.N_in + L.C - 1) / L.C;
  la.N = L.N_in;
  la.n_workers = nw;
  la.ctr = L.ctr;
  la.opt = L.opt; la.normalize = L.normalize; la.mask = L.mask;
  la.beta = L.beta; la.norm_eps = L.norm_eps;
  la.out = L.out; la.out_bf16 = L.out_bf16; la.out_bs = (long long)L.N_in * kg::D;
  la.cast_first = L.cast_first;
  la.wsave = L.wsave;
  la.rownorm = L.rownorm;
  if (cudaMemsetAsync(L.ctr, 0, (3 * (size_t)L.BH + 2) * sizeof(unsigned), stream) != cudaSuccess) return -1;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(nw + nr);
  cfg.blockDim = dim3(kg::THREADS);
  cfg.dynamicSmemBytes = kg::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeCooperative;
  attrs[0].val.cooperative = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  prof_before(K_LOOP, stream);
  const bool snap = L.wsave != nullptr || L.rownorm != nullptr;
  const cudaError_t e = snap ? cudaLaunchKernelEx(&cfg, lact_keygrad_kernel<true, true>, m, a, la)
                             : cudaLaunchKernelEx(&cfg, lact_keygrad_kernel<true>, m, a, la);
  prof_after(K_LOOP, stream);
  return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace ttt
