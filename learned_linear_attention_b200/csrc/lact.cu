// lact.cu -- LaCT fast-weight layer: SwiGLU memory with large chunks
// ("Test-Time Training Done Right" review: "Memoria no lineal y atención
// local", "El orden de lectura evita información futura").
//
// Per chunk c of C input tokens (all heads at once, every step on the GPU):
//   1. key pass   (tcgen05):  [H1|H3] = K_c [W1;W3]^T, dGr = V_c W2 and, for
//      the causal order, [Hq1|Hq3] = Q_c [W1;W3]^T.  The epilogue forms
//        dH3 = dG*silu(H1), dH1 = dG*H3*silu'(H1), Gm' = -eta*silu(H1)*H3
//      with dG = -eta*dGr (token rows), and Aq = silu(Hq1)*Hq3; all bf16.
//   2. read       (tcgen05):  out_c = Aq W2^T             (causal order)
//   3. gradients  (tcgen05, split-K over tokens):
//        G1 = dH1^T K_c,  G3 = dH3^T K_c,  G2 = V_c^T Gm'
//   4. update: GD / momentum in one row kernel with the row L2
//      normalisation; Muon: momentum, Newton-Schulz on tensor cores, apply +
//      normalisation.  Each writes the fp32 state and the bf16 operand copy
//      used by the next chunk.
// Bidirectional order: steps 1 (keys only), 3, 4 for every chunk, then the
// queries run step 1 (queries only) and step 2 with the final weights.
#include <algorithm>
#include <cstdlib>
#include <functional>
#include <vector>

#include "gemm.cuh"
#include "kernels.h"

namespace ttt {

// =====================================================================
// key pass
// =====================================================================
namespace kp {
constexpr int BM = 128, HB = 64;          // token rows, hidden units per tile
constexpr uint32_t X_BYTES = BM * 64 * 2;            // 16 KB (K or Q tile)
constexpr uint32_t V_BYTES = BM * 64 * 2;            // 16 KB
constexpr uint32_t W13_BYTES = 2 * HB * 64 * 2;      // 16 KB (W1 rows | W3 rows)
constexpr uint32_t W2_BYTES = 64 * HB * 2;           // 8 KB  (W2 block, MN-major)
constexpr uint32_t STAGE = X_BYTES + V_BYTES + W13_BYTES + W2_BYTES;
constexpr int STAGES = 3;
constexpr uint32_t STG_OUT = BM * HB * 2;            // 16 KB: one output tile, 128-byte swizzle
constexpr uint32_t STG_HALF = BM * 32 * 2;           // 8 KB: half an output tile (split operands)
constexpr uint32_t STG_OFF = STAGES * STAGE;         // [dH1 | dH3 | Gm'] or [Aq] staging
constexpr uint32_t BAR_OFF = STG_OFF + 3 * STG_OUT;
constexpr uint32_t SMEM = BAR_OFF + 256 + 1024;
constexpr uint32_t ACC_COLS = 256;                   // [H1 64 | H3 64 | dG 64 | pad]
constexpr int EPI_WARPS = 8;                         // two per TMEM lane quadrant
constexpr int THREADS = (2 + EPI_WARPS) * 32;
}  // namespace kp

struct KeyPassArgs {
  int C;            // rows of this pass (chunk length or N_q)
  int t0;           // first token row in the token tensors
  int n_key_tiles, n_q_tiles;
  int n_hb;         // dh / 64
  int BH;
  int d_steps;      // d / 64
  int dh;
  int lr_len;       // row length of lr ([BH][lr_len])
  const float* lr;
  // dH1 | dH3 side by side in D13 [BH][cmax][2*dh]; Gm', Aq [BH][cmax][dh]
  __nv_bfloat16 *D13, *Gm, *Aq;
  // split operands: W = W_hi + W_lo (the K loop runs twice) and the
  // intermediates are written as hi and lo bf16 parts
  int split;
  __nv_bfloat16 *D13lo, *Gmlo, *Aqlo;
  // key tiles form only Gm' = -eta silu(H1) H3 (no V W2 product, no dH1 and
  // dH3): only W2 is updated
  int feat_only;
  long long inter_bs;      // cmax * dh (Gm', Aq); D13 uses twice that
  DevStatus st;
};

struct KeyPassMaps {
  CUtensorMap k, v, q, w1, w3, w2, w1lo, w3lo, w2lo;
  // tensor-store views of the intermediates: D13 {2 dh, cmax, BH}, Gm' and
  // Aq {dh, cmax, BH}.  Box 64 hidden x 128 rows, 128-byte swizzle; with split
  // operands [hi, lo] pairs with box 32 x 128, 64-byte swizzle.
  CUtensorMap od13, ogm, oaq;
  CUtensorMap sd13[2], sgm[2], saq[2];
};

// Byte offset of 16-byte chunk c (0..7) of row r in a tile of 128-byte rows
// laid out with the 128-byte swizzle (chunk index XOR row mod 8).
TTT_DEVICE_INLINE uint32_t sw128_offset(int r, int c) {
  return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
}
// The same for 64-byte rows and the 64-byte swizzle (chunk c = 0..3).
TTT_DEVICE_INLINE uint32_t kp_sw64_offset(int r, int c) {
  return (uint32_t)(r * 64 + ((c ^ ((r >> 1) & 3)) << 4));
}

// bf16 residual of x given its bf16 rounding h: the "lo" part of x = hi + lo.
TTT_DEVICE_INLINE __nv_bfloat16 bf16_residual(float x, __nv_bfloat16 h) {
  return __float2bfloat16_rn(x - __bfloat162float(h));
}

TTT_DEVICE_INLINE float sigmoidf_fast(float x) { return __fdividef(1.f, 1.f + __expf(-x)); }
// sigma(x) = 1/2 + tanh(x/2)/2 with the hardware tanh approximation (one
// MUFU op, max relative error about 2^-11): used when the outputs are
// rounded to bf16 anyway.
TTT_DEVICE_INLINE float sigmoidf_tanh(float x) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
  return fmaf(0.5f, t, 0.5f);
}

// SP: split operands (a.split != 0); one instance per mode, so each keeps
// only its own epilogue's registers
template <bool SP>
__global__ void __launch_bounds__(kp::THREADS, 1)
    lact_keypass_kernel(const __grid_constant__ KeyPassMaps maps, const KeyPassArgs a) {
  using namespace kp;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* empty = full + STAGES;
  uint64_t* afull = empty + STAGES;
  uint64_t* aempty = afull + 2;
  uint64_t* fin = aempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_per_bh = (a.n_key_tiles + a.n_q_tiles) * a.n_hb;
  const int n_tiles = tiles_per_bh * a.BH;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&afull[s], 1);
      mbar_init(&aempty[s], EPI_WARPS * 32);
    }
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * ACC_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&maps.k);
    tma_prefetch_desc(&maps.v);
    tma_prefetch_desc(&maps.q);
    tma_prefetch_desc(&maps.w1);
    tma_prefetch_desc(&maps.w3);
    tma_prefetch_desc(&maps.w2);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  pdl_launch_dependents();
  const uint32_t tmem = *tmem_slot;
  Waiter W{abort_flag, a.st, 200};

  // tile id -> (bh, token tile, hidden block); hidden block fastest so the
  // CTAs sharing a token tile run together and its K/V rows hit in L2.
  auto decode = [&](int t, int& bh, int& tt, int& hb) {
    hb = t % a.n_hb;
    tt = (t / a.n_hb) % (a.n_key_tiles + a.n_q_tiles);
    bh = t / tiles_per_bh;
  };

  if (warp == 0) {
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
        int bh, tt, hb;
        decode(t, bh, tt, hb);
        const bool is_key = tt < a.n_key_tiles;
        const int row = a.t0 + (is_key ? tt : tt - a.n_key_tiles) * BM;
        const int j0 = hb * HB;
        const int steps = a.d_steps * (a.split ? 2 : 1);
        for (int kk = 0; kk < steps; ++kk, ++it) {
          const bool lo = kk >= a.d_steps;
          const int ks = lo ? kk - a.d_steps : kk;
          const uint32_t s = it % STAGES;
          if (it >= (uint32_t)STAGES && !W.wait(&empty[s], ((it / STAGES) - 1) & 1, 1)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * STAGE;
          const bool with_v = is_key && !a.feat_only;
          mbar_arrive_expect_tx(&full[s], with_v ? STAGE : X_BYTES + W13_BYTES);
          tma_load_3d(st, is_key ? &maps.k : &maps.q, &full[s], ks * 64, row, bh);
          tma_load_3d(st + X_BYTES + V_BYTES, lo ? &maps.w1lo : &maps.w1, &full[s], ks * 64, j0, bh);
          tma_load_3d(st + X_BYTES + V_BYTES + W13_BYTES / 2, lo ? &maps.w3lo : &maps.w3, &full[s],
                      ks * 64, j0, bh);
          if (with_v) {
            tma_load_3d(st + X_BYTES, &maps.v, &full[s], ks * 64, row, bh);
            tma_load_3d(st + X_BYTES + V_BYTES + W13_BYTES, lo ? &maps.w2lo : &maps.w2, &full[s],
                        j0, ks * 64, bh);
          }
        }
      }
      if (W.aborted()) {
        const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0;
        for (uint32_t i = first; i < it; ++i) W.drain(&full[i % STAGES], (i / STAGES) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_h = make_idesc(128, 128, false, false);
      const uint32_t id_g = make_idesc(128, 64, false, true);
      uint32_t it = 0, lt = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++lt) {
        int bh, tt, hb;
        decode(t, bh, tt, hb);
        const bool is_key = tt < a.n_key_tiles;
        const uint32_t ab = lt & 1;
        if (lt >= 2 && !W.wait(&aempty[ab], ((lt >> 1) - 1) & 1, 2)) break;
        tc_fence_after();
        const uint32_t d = tmem + ab * ACC_COLS;
        const int steps = a.d_steps * (a.split ? 2 : 1);
        for (int ks = 0; ks < steps; ++ks, ++it) {
          const uint32_t s = it % STAGES;
          if (!W.wait(&full[s], (it / STAGES) & 1, 3)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sx = smem_u32(smem + s * STAGE);
          const uint32_t sv = sx + X_BYTES;
          const uint32_t sw13 = sv + V_BYTES;
          const uint32_t sw2 = sw13 + W13_BYTES;
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            mma_bf16(d, make_sdesc(sx + k4 * 32, 16, 1024), make_sdesc(sw13 + k4 * 32, 16, 1024),
                     id_h, (ks | k4) != 0);
            if (is_key && !a.feat_only)
              mma_bf16(d + 128, make_sdesc(sv + k4 * 32, 16, 1024),
                       make_sdesc(sw2 + k4 * 2048, 8192, 1024), id_g, (ks | k4) != 0);
          }
          mma_commit(&empty[s]);
        }
        if (!ok) break;
        mma_commit(&afull[ab]);
      }
      mma_commit(fin);
      W.drain(fin, 0);
    }
  } else {
    // epilogue: warps 2..9; quadrant q4 = TMEM lanes, column group cg, two
    // halves of 16 columns per thread.  Every output tile is staged in shared
    // memory and leaves by tensor stores, issued by lane 0 of epilogue warp ew
    // for staged output ew, so the rows go out as whole lines; rows past the
    // pass are staged as zeros (the intermediates hold cmax rows and their
    // readers stop at the pass length).
    //  - bf16 operands: cg takes 32 of the 64 hidden units, the halves 16 each;
    //    each output (dH1, dH3, Gm' or Aq) is one 128 x 64 tile with the
    //    128-byte swizzle, stored once per tile;
    //  - split operands: half h is hidden units [32h, 32h + 32), cg 16 of
    //    them; the hi and lo parts of each output are 128 x 32 tiles with the
    //    64-byte swizzle, stored once per half.
    const int q4 = warp & 3;
    const int cg = (warp - 2) >> 2;
    const int ew = warp - 2;
    const int r = q4 * 32 + lane;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    constexpr bool sp = SP;
    const uint32_t stg = smem_u32(smem + STG_OFF);
    uint32_t lt = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++lt) {
      int bh, tt, hb;
      decode(t, bh, tt, hb);
      const bool is_key = tt < a.n_key_tiles;
      const bool full_key = is_key && !a.feat_only;
      const int nout = full_key ? 3 : 1;
      // staged outputs: the hi parts, then (split operands) the lo parts;
      // only W2 updated (no split operands) writes Gm' alone
      const int nst = sp && (full_key || !is_key) ? 2 * nout : nout;
      const int prow = (is_key ? tt : tt - a.n_key_tiles) * BM;   // first row within the pass
      const int tc = prow + r;
      const bool valid = tc < a.C;
      const uint32_t ab = lt & 1;
      // the learning rate is fetched before waiting for the accumulator
      const float eta = (is_key && valid) ? a.lr[(size_t)bh * a.lr_len + a.t0 + tc] : 0.f;
      if (!named_bar_all(1, EPI_WARPS * 32, W.wait(&afull[ab], (lt >> 1) & 1, 4))) break;
      tc_fence_after();
      const uint32_t base = tmem + lane_base + ab * ACC_COLS;
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        const int jc = sp ? half * 32 + cg * 16 : cg * 32 + half * 16;
        uint32_t rh1[16], rh3[16], rg[16];
        tmem_ld16_issue(base + jc, rh1);
        tmem_ld16_issue(base + 64 + jc, rh3);
        if (full_key) tmem_ld16_issue(base + 128 + jc, rg);
        tmem_wait_ld();
        if (half == 1) {   // this thread's last read of the accumulators
          tc_fence_before();
          mbar_arrive(&aempty[ab]);
        }
        float h1[16], h3[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          h1[j] = __uint_as_float(rh1[j]);
          h3[j] = __uint_as_float(rh3[j]);
        }
        uint32_t o[3][8];   // hi part of output q for this row's 16 columns, bf16 pairs
        uint32_t l[3][8];   // lo part (split operands)
        if (is_key && a.feat_only) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float x0 = h1[2 * j], x1 = h1[2 * j + 1];
            o[0][j] = pack_bf16x2(-eta * x0 * sigmoidf_tanh(x0) * h3[2 * j],
                                  -eta * x1 * sigmoidf_tanh(x1) * h3[2 * j + 1]);
          }
        } else if (is_key) {
          float r1[16], r3[16], rm[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float x = h1[j], y = h3[j];
            const float sg = sp ? sigmoidf_fast(x) : sigmoidf_tanh(x);
            const float act = x * sg;
            const float dg = -eta * __uint_as_float(rg[j]);
            r3[j] = dg * act;
            r1[j] = dg * y * (sg * (1.f + x * (1.f - sg)));
            rm[j] = -eta * act * y;
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            o[0][j] = pack_bf16x2(r1[2 * j], r1[2 * j + 1]);
            o[1][j] = pack_bf16x2(r3[2 * j], r3[2 * j + 1]);
            o[2][j] = pack_bf16x2(rm[2 * j], rm[2 * j + 1]);
          }
          if (sp) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              l[0][j] = pack_bf16x2(r1[2 * j] - bf16lo(o[0][j]), r1[2 * j + 1] - bf16hi(o[0][j]));
              l[1][j] = pack_bf16x2(r3[2 * j] - bf16lo(o[1][j]), r3[2 * j + 1] - bf16hi(o[1][j]));
              l[2][j] = pack_bf16x2(rm[2 * j] - bf16lo(o[2][j]), rm[2 * j + 1] - bf16hi(o[2][j]));
            }
          }
        } else {
          float aq[16];
#pragma unroll
          for (int j = 0; j < 16; ++j)
            aq[j] = h1[j] * (sp ? sigmoidf_fast(h1[j]) : sigmoidf_tanh(h1[j])) * h3[j];
#pragma unroll
          for (int j = 0; j < 8; ++j) o[0][j] = pack_bf16x2(aq[2 * j], aq[2 * j + 1]);
          if (sp) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
              l[0][j] = pack_bf16x2(aq[2 * j] - bf16lo(o[0][j]), aq[2 * j + 1] - bf16hi(o[0][j]));
          }
        }
        if (!valid) {
#pragma unroll
          for (int q = 0; q < 3; ++q)
#pragma unroll
            for (int j = 0; j < 8; ++j) o[q][j] = l[q][j] = 0u;
        }
        if (!sp) {
          if (half == 0) {   // the staging tiles are free once the previous tile's stores have read them
            if (lane == 0 && ew < 3) bulk_wait_read();
            named_bar_sync(1, EPI_WARPS * 32);
          }
#pragma unroll
          for (int q = 0; q < 3; ++q) {
            if (q < nout) {
              st_shared_v4(stg + q * STG_OUT + sw128_offset(r, jc >> 3), o[q][0], o[q][1], o[q][2], o[q][3]);
              st_shared_v4(stg + q * STG_OUT + sw128_offset(r, (jc >> 3) + 1), o[q][4], o[q][5], o[q][6],
                           o[q][7]);
            }
          }
        } else {
          // the staging tiles are free once the previous half's stores have read them
          if (lane == 0 && ew < 6) bulk_wait_read();
          named_bar_sync(1, EPI_WARPS * 32);
#pragma unroll
          for (int q = 0; q < 3; ++q) {
            if (q < nout) {
              st_shared_v4(stg + q * STG_HALF + kp_sw64_offset(r, 2 * cg), o[q][0], o[q][1], o[q][2], o[q][3]);
              st_shared_v4(stg + q * STG_HALF + kp_sw64_offset(r, 2 * cg + 1), o[q][4], o[q][5], o[q][6],
                           o[q][7]);
              if (nst > nout) {
                const uint32_t sl = stg + (nout + q) * STG_HALF;
                st_shared_v4(sl + kp_sw64_offset(r, 2 * cg), l[q][0], l[q][1], l[q][2], l[q][3]);
                st_shared_v4(sl + kp_sw64_offset(r, 2 * cg + 1), l[q][4], l[q][5], l[q][6], l[q][7]);
              }
            }
          }
          fence_async_smem();   // the tensor stores (async proxy) read what these threads wrote
          named_bar_sync(1, EPI_WARPS * 32);
          if (lane == 0 && ew < nst) {
            // staged output ew: kind 0 dH1, 1 dH3, 2 Gm', 3 Aq; part 0 hi, 1 lo
            const int kind = full_key ? ew % 3 : is_key ? 2 : 3;
            const int part = full_key ? ew / 3 : is_key ? 0 : ew;
            const CUtensorMap* m = kind == 3 ? &maps.saq[part] : kind == 2 ? &maps.sgm[part] : &maps.sd13[part];
            const int x = hb * HB + half * 32 + (kind == 1 ? a.dh : 0);
            tma_store_3d(m, smem + STG_OFF + ew * STG_HALF, x, prow, bh);
            bulk_commit();
          }
        }
      }
      if (!sp) {
        fence_async_smem();   // the tensor stores (async proxy) read what these threads wrote
        named_bar_sync(1, EPI_WARPS * 32);
        if (lane == 0 && ew < nout) {
          const CUtensorMap* m = !is_key ? &maps.oaq : (full_key && ew < 2) ? &maps.od13 : &maps.ogm;
          const int x = hb * HB + ((full_key && ew == 1) ? a.dh : 0);
          tma_store_3d(m, smem + STG_OFF + ew * STG_OUT, x, prow, bh);
          bulk_commit();
        }
      }
    }
    if (lane == 0 && ew < 6) bulk_wait_all();   // every tensor store is complete before the CTA exits
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * ACC_COLS);
  }
}

// =====================================================================
// row kernels: bf16 copies, GD / momentum update, Muon pieces
// =====================================================================
struct RowArgs {
  int BH, d, dh, splits, opt, normalize, mask;
  float beta, norm_eps, ns_eps;
  float* W[3];              // fp32 state per matrix [BH][rows][cols]
  float* M[3];              // momentum (nullable)
  __nv_bfloat16* Wb[3];     // bf16 copies
  __nv_bfloat16* Wlo[3];    // bf16 residual copies (split operands; nullable)
  const float* part[3];     // split-K partial gradients [splits][BH][rows][cols]
  float* rowss;             // [3][BH][rows] row sums of squares (Muon)
  const float* X32;         // NS result [3][BH][r][c] (Muon apply)
  DevStatus st;
  int nbuf;                 // cast: copies written, buf_stride elements apart
  size_t buf_stride;
  float* rownorm;           // nullable: norm of each updated row before normalisation
};

constexpr int ROW_MAXV = 32;  // columns per lane (cols <= 1024)

TTT_DEVICE_INLINE void row_decode(const RowArgs& a, int gw, int& mat, int& bh, int& row, int& rows,
                                  int& cols) {
  const int per_bh = 2 * a.dh + a.d;
  bh = gw / per_bh;
  int rr = gw % per_bh;
  if (rr < a.dh) {
    mat = 0; row = rr; rows = a.dh; cols = a.d;
  } else if (rr < 2 * a.dh) {
    mat = 1; row = rr - a.dh; rows = a.dh; cols = a.d;
  } else {
    mat = 2; row = rr - 2 * a.dh; rows = a.d; cols = a.dh;
  }
}

TTT_DEVICE_INLINE float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// bf16 operand copies of all three matrices.
__global__ void lact_cast_kernel(RowArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (gw >= a.BH * (2 * a.dh + a.d)) return;
  int mat, bh, row, rows, cols;
  row_decode(a, gw, mat, bh, row, rows, cols);
  const size_t off = ((size_t)bh * rows + row) * cols;
  for (int c = lane; c < cols; c += 32) {
    const float x = a.W[mat][off + c];
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    for (int b = 0; b < a.nbuf; ++b) {
      a.Wb[mat][b * a.buf_stride + off + c] = h;
      if (a.Wlo[mat] != nullptr) a.Wlo[mat][b * a.buf_stride + off + c] = bf16_residual(x, h);
    }
  }
}

// Row kernels run one 128-thread block per weight row; each thread owns up
// to ROW_PER_THREAD columns so the split-K partial loads are independent.
constexpr int ROW_THREADS = 128, ROW_PER_THREAD = 8;   // cols <= 1024

TTT_DEVICE_INLINE float block_sum128(float x, float* red) {
  x = warp_sum(x);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = x;
  __syncthreads();
  const float t = red[0] + red[1] + red[2] + red[3];
  __syncthreads();
  return t;
}

TTT_DEVICE_INLINE void sum_partials(const RowArgs& a, int mat, size_t off, size_t split_stride,
                                    int cols, float* g) {
#pragma unroll
  for (int i = 0; i < ROW_PER_THREAD; ++i) g[i] = 0.f;
  for (int s = 0; s < a.splits; ++s) {
    const float* p = a.part[mat] + s * split_stride + off;
#pragma unroll
    for (int i = 0; i < ROW_PER_THREAD; ++i) {
      const int c = threadIdx.x + ROW_THREADS * i;
      if (c < cols) g[i] += __ldcg(p + c);
    }
  }
}

// GD / momentum: sum the split-K partials, update, normalise the row.  One
// warp per UPD_RPW rows; lanes own 4 consecutive columns per 128-column chunk
// (16-byte loads).  All partial sums of all the warp's rows are requested
// before any is used, so many loads are in flight per warp.
constexpr int UPD_ROWS_PER_BLOCK = 8;   // warps per block
constexpr int UPD_RPW = 1;              // rows per warp
__global__ void __launch_bounds__(UPD_ROWS_PER_BLOCK * 32) lact_update_kernel(RowArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int total = a.BH * (2 * a.dh + a.d);
  const int gw0 = (blockIdx.x * UPD_ROWS_PER_BLOCK + (threadIdx.x >> 5)) * UPD_RPW;
  if (gw0 >= total) return;
  int mat[UPD_RPW], rows[UPD_RPW], cols[UPD_RPW];
  size_t off[UPD_RPW];
  bool live[UPD_RPW];
#pragma unroll
  for (int q = 0; q < UPD_RPW; ++q) {
    int bh, row;
    live[q] = gw0 + q < total;
    row_decode(a, live[q] ? gw0 + q : gw0, mat[q], bh, row, rows[q], cols[q]);
    live[q] = live[q] && (a.mask & (1 << mat[q]));
    off[q] = ((size_t)bh * rows[q] + row) * cols[q];
  }
  float4 w[UPD_RPW][8];
#pragma unroll
  for (int q = 0; q < UPD_RPW; ++q)
#pragma unroll
    for (int i = 0; i < 8; ++i) w[q][i] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = 0; s < a.splits; ++s) {
#pragma unroll
    for (int q = 0; q < UPD_RPW; ++q) {
      if (!live[q]) continue;
      const size_t split_stride = (size_t)a.BH * rows[q] * cols[q];
      const float4* p = reinterpret_cast<const float4*>(a.part[mat[q]] + s * split_stride + off[q]) + lane;
      const int nch = cols[q] >> 7;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (i < nch) {
          const float4 x = __ldcg(p + 32 * i);
          w[q][i].x += x.x; w[q][i].y += x.y; w[q][i].z += x.z; w[q][i].w += x.w;
        }
      }
    }
  }
#pragma unroll
  for (int q = 0; q < UPD_RPW; ++q) {
    if (!live[q]) continue;
    const int nch = cols[q] >> 7;
    float4* Wr = reinterpret_cast<float4*>(a.W[mat[q]] + off[q]) + lane;
    float4* Mr = a.opt == 1 ? reinterpret_cast<float4*>(a.M[mat[q]] + off[q]) + lane : nullptr;
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i < nch) {
        float4 u = w[q][i];
        if (Mr != nullptr) {
          float4 m = Mr[32 * i];
          m.x = a.beta * m.x + u.x; m.y = a.beta * m.y + u.y;
          m.z = a.beta * m.z + u.z; m.w = a.beta * m.w + u.w;
          Mr[32 * i] = m;
          u = m;
        }
        const float4 x = Wr[32 * i];
        w[q][i] = make_float4(x.x - u.x, x.y - u.y, x.z - u.z, x.w - u.w);
        ss += w[q][i].x * w[q][i].x + w[q][i].y * w[q][i].y + w[q][i].z * w[q][i].z +
              w[q][i].w * w[q][i].w;
      }
    }
    float scale = 1.f;
    if (a.normalize) {
      const float nrm = sqrtf(warp_sum(ss));
      scale = 1.f / fmaxf(nrm, a.norm_eps);
      if (a.rownorm != nullptr && lane == 0) a.rownorm[gw0 + q] = nrm;
    }
    uint2* Br = reinterpret_cast<uint2*>(a.Wb[mat[q]] + off[q]) + lane;
    uint2* Lr = a.Wlo[mat[q]] != nullptr ? reinterpret_cast<uint2*>(a.Wlo[mat[q]] + off[q]) + lane : nullptr;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i < nch) {
        const float4 x = make_float4(w[q][i].x * scale, w[q][i].y * scale, w[q][i].z * scale,
                                     w[q][i].w * scale);
        Wr[32 * i] = x;
        const uint32_t h0 = pack_bf16x2(x.x, x.y), h1 = pack_bf16x2(x.z, x.w);
        Br[32 * i] = make_uint2(h0, h1);
        if (Lr != nullptr)
          Lr[32 * i] = make_uint2(pack_bf16x2(x.x - bf16lo(h0), x.y - bf16hi(h0)),
                                  pack_bf16x2(x.z - bf16lo(h1), x.w - bf16hi(h1)));
      }
    }
  }
}

// GD / momentum on slabs of whole rows (about 8 KB of one matrix of one
// head).  One thread brings the slab's split-K partial sums, its fp32
// weights and its momentum into shared memory with bulk copies completing
// on one mbarrier, so every byte a block needs is in flight at once; then
// each warp sums its rows' partials in split order, updates, normalises
// and writes fp32 weights and bf16 copies.
constexpr int UPB_THREADS = 256;
constexpr uint32_t UPB_SLAB = 8192;
constexpr int UPB_MAX_SPLITS = 8;
__host__ __device__ __forceinline__ int upb_rows(int cols) { return cols * 4 >= (int)UPB_SLAB ? 1 : (int)UPB_SLAB / (cols * 4); }

TTT_DEVICE_INLINE void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__global__ void __launch_bounds__(UPB_THREADS) lact_update_bulk_kernel(RowArgs a) {
  extern __shared__ __align__(128) uint8_t upb_smem[];
  __shared__ uint64_t bar;
  __shared__ uint32_t abort_flag;
  const int r13 = upb_rows(a.d), r2 = upb_rows(a.dh);
  const int s13 = (a.dh + r13 - 1) / r13, s2 = (a.d + r2 - 1) / r2;
  const int per_bh = 2 * s13 + s2;
  const int bh = blockIdx.x / per_bh, rr = blockIdx.x % per_bh;
  const int mat = rr < s13 ? 0 : (rr < 2 * s13 ? 1 : 2);
  const int slab = mat == 0 ? rr : (mat == 1 ? rr - s13 : rr - 2 * s13);
  const int rows = mat < 2 ? a.dh : a.d, cols = mat < 2 ? a.d : a.dh;
  const int R = mat < 2 ? r13 : r2;
  const int row0 = slab * R, nrows = min(R, rows - row0);
  if (bh >= a.BH || nrows <= 0 || !(a.mask & (1 << mat))) {
    pdl_wait();
    pdl_launch_dependents();
    return;
  }
  const size_t off = ((size_t)bh * rows + row0) * cols;
  const uint32_t bytes = (uint32_t)nrows * cols * 4;
  float* const Wg = mat == 0 ? a.W[0] : (mat == 1 ? a.W[1] : a.W[2]);
  float* const Mg = a.opt == 1 ? (mat == 0 ? a.M[0] : (mat == 1 ? a.M[1] : a.M[2])) : nullptr;
  const float* const Pg = mat == 0 ? a.part[0] : (mat == 1 ? a.part[1] : a.part[2]);
  __nv_bfloat16* const Bg = mat == 0 ? a.Wb[0] : (mat == 1 ? a.Wb[1] : a.Wb[2]);
  __nv_bfloat16* const Lg = mat == 0 ? a.Wlo[0] : (mat == 1 ? a.Wlo[1] : a.Wlo[2]);
  const size_t split_stride = (size_t)a.BH * rows * cols;
  float* sp = reinterpret_cast<float*>(upb_smem);                  // [splits][R][cols]
  float* sw = sp + (size_t)a.splits * UPB_SLAB / 4;                 // [R][cols]
  float* sm = sw + UPB_SLAB / 4;                                    // [R][cols]
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  // The fp32 weights and momentum were last written by an update that had
  // completed before the preceding kernel started, so their copies go out
  // before the wait for that kernel (whose partial sums come after it).
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&bar, bytes * (a.splits + 1 + (Mg != nullptr ? 1 : 0)));
    bulk_load(sw, Wg + off, bytes, &bar);
    if (Mg != nullptr) bulk_load(sm, Mg + off, bytes, &bar);
  }
  pdl_wait();
  pdl_launch_dependents();
  if (threadIdx.x == 0)
    for (int s = 0; s < a.splits; ++s)
      bulk_load(sp + (size_t)s * UPB_SLAB / 4, Pg + s * split_stride + off, bytes, &bar);
  Waiter W{&abort_flag, a.st, 500};
  if (!W.wait(&bar, 0, 0)) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nch = cols >> 7;   // 128-column chunks; lane owns 4 columns of each
  for (int r = warp; r < nrows; r += UPB_THREADS / 32) {
    float4 w[8];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i >= nch) break;
      const int c = r * cols + 128 * i + 4 * lane;
      float4 u = *reinterpret_cast<const float4*>(sp + c);
      for (int s = 1; s < a.splits; ++s) {
        const float4 x = *reinterpret_cast<const float4*>(sp + (size_t)s * UPB_SLAB / 4 + c);
        u.x += x.x; u.y += x.y; u.z += x.z; u.w += x.w;
      }
      if (Mg != nullptr) {
        float4 m = *reinterpret_cast<const float4*>(sm + c);
        m.x = a.beta * m.x + u.x; m.y = a.beta * m.y + u.y;
        m.z = a.beta * m.z + u.z; m.w = a.beta * m.w + u.w;
        *reinterpret_cast<float4*>(Mg + off + c) = m;
        u = m;
      }
      const float4 x = *reinterpret_cast<const float4*>(sw + c);
      w[i] = make_float4(x.x - u.x, x.y - u.y, x.z - u.z, x.w - u.w);
      ss += w[i].x * w[i].x + w[i].y * w[i].y + w[i].z * w[i].z + w[i].w * w[i].w;
    }
    float scale = 1.f;
    if (a.normalize) {
      const float nrm = sqrtf(warp_sum(ss));
      scale = 1.f / fmaxf(nrm, a.norm_eps);
      if (a.rownorm != nullptr && lane == 0)
        a.rownorm[(size_t)bh * (2 * a.dh + a.d) + (mat == 0 ? 0 : mat == 1 ? a.dh : 2 * a.dh) +
                  row0 + r] = nrm;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i >= nch) break;
      const int c = r * cols + 128 * i + 4 * lane;
      const float4 x = make_float4(w[i].x * scale, w[i].y * scale, w[i].z * scale, w[i].w * scale);
      *reinterpret_cast<float4*>(Wg + off + c) = x;
      const uint32_t h0 = pack_bf16x2(x.x, x.y), h1 = pack_bf16x2(x.z, x.w);
      *reinterpret_cast<uint2*>(Bg + off + c) = make_uint2(h0, h1);
      if (Lg != nullptr)
        *reinterpret_cast<uint2*>(Lg + off + c) =
            make_uint2(pack_bf16x2(x.x - bf16lo(h0), x.y - bf16hi(h0)),
                       pack_bf16x2(x.z - bf16lo(h1), x.w - bf16hi(h1)));
    }
  }
}
static int update_bulk_blocks(int BH, int d, int dh) {
  const int r13 = upb_rows(d), r2 = upb_rows(dh);
  return BH * (2 * ((dh + r13 - 1) / r13) + (d + r2 - 1) / r2);
}

// Muon step 1: M = beta M + G, and the row sums of squares of M.
__global__ void __launch_bounds__(ROW_THREADS) muon_momentum_kernel(RowArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ float red[4];
  int mat, bh, row, rows, cols;
  row_decode(a, blockIdx.x, mat, bh, row, rows, cols);
  if (!(a.mask & (1 << mat))) return;
  const size_t off = ((size_t)bh * rows + row) * cols;
  const size_t split_stride = (size_t)a.BH * rows * cols;
  float g[ROW_PER_THREAD];
  sum_partials(a, mat, off, split_stride, cols, g);
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < ROW_PER_THREAD; ++i) {
    const int c = threadIdx.x + ROW_THREADS * i;
    if (c < cols) {
      const float m = a.beta * a.M[mat][off + c] + g[i];
      a.M[mat][off + c] = m;
      ss += m * m;
    }
  }
  ss = block_sum128(ss, red);
  if (threadIdx.x == 0) a.rowss[(size_t)mat * a.BH * a.dh + (size_t)bh * rows + row] = ss;
}

// Muon step 2: X = M / (||M||_F + eps) in the wide orientation (r x c with
// r = min(d, dh)), fp32 and bf16.  One CTA row-block per (mat, bh, x-row).
struct NsPrepArgs {
  int BH, d, dh, r, c;
  float eps;
  const float* M[3];
  const float* rowss;
  float* X32;              // [3*BH][r][c]
  __nv_bfloat16* Xb;       // [3*BH][r][c]
  __nv_bfloat16* Xlo;      // residual (split operands; nullable)
  unsigned* counter;       // phase counter of the fused Newton-Schulz kernel (zeroed here)
};
__global__ void ns_prep_kernel(NsPrepArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  if (a.counter != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *a.counter = 0u;
  const int mb = blockIdx.y;                 // mat * BH + bh
  const int mat = mb / a.BH, bh = mb % a.BH;
  const int rows = mat < 2 ? a.dh : a.d, cols = mat < 2 ? a.d : a.dh;
  __shared__ float s_scale;
  if (threadIdx.x < 32) {
    float ss = 0.f;
    const float* rs = a.rowss + (size_t)mat * a.BH * a.dh + (size_t)bh * rows;
    for (int i = threadIdx.x; i < rows; i += 32) ss += rs[i];
    ss = warp_sum(ss);
    if (threadIdx.x == 0) s_scale = 1.f / (sqrtf(ss) + a.eps);
  }
  __syncthreads();
  const float scale = s_scale;
  const bool tall = rows > cols;
  const float* Mm = a.M[mat] + (size_t)bh * rows * cols;
  float* x32 = a.X32 + (size_t)mb * a.r * a.c;
  __nv_bfloat16* xb = a.Xb + (size_t)mb * a.r * a.c;
  const int xr = blockIdx.x;  // row of X
  for (int xc = threadIdx.x; xc < a.c; xc += blockDim.x) {
    const float v = (tall ? Mm[(size_t)xc * cols + xr] : Mm[(size_t)xr * cols + xc]) * scale;
    x32[(size_t)xr * a.c + xc] = v;
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    xb[(size_t)xr * a.c + xc] = h;
    if (a.Xlo != nullptr) a.Xlo[(size_t)mb * a.r * a.c + (size_t)xr * a.c + xc] = bf16_residual(v, h);
  }
}

// Muon step 4: W -= NS(M) (orientation restored), normalise the row.
__global__ void muon_apply_kernel(RowArgs a, int r, int c) {
  pdl_wait();
  pdl_launch_dependents();
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (gw >= a.BH * (2 * a.dh + a.d)) return;
  int mat, bh, row, rows, cols;
  row_decode(a, gw, mat, bh, row, rows, cols);
  if (!(a.mask & (1 << mat))) return;
  const bool tall = rows > cols;
  const float* X = a.X32 + (size_t)(mat * a.BH + bh) * r * c;
  const size_t off = ((size_t)bh * rows + row) * cols;
  float w[ROW_MAXV];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < ROW_MAXV; ++i) {
    const int cc = lane + 32 * i;
    w[i] = 0.f;
    if (cc < cols) {
      const float u = tall ? X[(size_t)cc * c + row] : X[(size_t)row * c + cc];
      w[i] = a.W[mat][off + cc] - u;
      ss += w[i] * w[i];
    }
  }
  float scale = 1.f;
  if (a.normalize) scale = 1.f / fmaxf(sqrtf(warp_sum(ss)), a.norm_eps);
#pragma unroll
  for (int i = 0; i < ROW_MAXV; ++i) {
    const int cc = lane + 32 * i;
    if (cc < cols) {
      const float x = w[i] * scale;
      const __nv_bfloat16 h = __float2bfloat16_rn(x);
      a.W[mat][off + cc] = x;
      a.Wb[mat][off + cc] = h;
      if (a.Wlo[mat] != nullptr) a.Wlo[mat][off + cc] = bf16_residual(x, h);
    }
  }
}

// =====================================================================
// host side
// =====================================================================
// SMs of the current device (asked on every call: a process may drive
// devices of different sizes)
static int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = 148;
  }
  return n;
}

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Helper streams (per device, created once) on which the independent GEMMs
// of a chunk run concurrently; fork/join with events keeps every call
// ordered on the caller's stream.
struct SideStreams {
  cudaStream_t s[3] = {nullptr, nullptr, nullptr};
  cudaEvent_t fork = nullptr, join[3] = {nullptr, nullptr, nullptr},
              read_done[3] = {nullptr, nullptr, nullptr};
  bool ok = false;
};
// Helper streams and their events belong to the calling host thread (one set
// per device), so calls made concurrently from several threads never record
// or wait on each other's events.
static SideStreams* side_streams() {
  thread_local SideStreams per_dev[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  SideStreams& x = per_dev[dev];
  if (!x.ok) {
    bool good = cudaEventCreateWithFlags(&x.fork, cudaEventDisableTiming) == cudaSuccess &&
                cudaEventCreateWithFlags(&x.read_done[0], cudaEventDisableTiming) == cudaSuccess &&
                cudaEventCreateWithFlags(&x.read_done[1], cudaEventDisableTiming) == cudaSuccess &&
                cudaEventCreateWithFlags(&x.read_done[2], cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; i < 3 && good; ++i)
      good = cudaStreamCreateWithFlags(&x.s[i], cudaStreamNonBlocking) == cudaSuccess &&
             cudaEventCreateWithFlags(&x.join[i], cudaEventDisableTiming) == cudaSuccess;
    x.ok = good;
  }
  return x.ok ? &x : nullptr;
}

static int grad_splits(int BH, int d, int dh, int cmax) {
  const int tiles = BH * 3 * (dh / 128) * (d / 128);
  const int ksteps = (cmax + 63) / 64;
  int s = (2 * num_sms() + tiles - 1) / tiles;
  s = std::max(1, std::min(s, std::max(1, ksteps / 8)));
  return s;
}

// Tile widths of the split-K gradient products: [G1; G3] (N = d) and G2 (N = dh).
static int grad_bn13(int d) { return d % 192 == 0 ? 192 : 128; }
static int grad_bn2(int dh) { return dh % 256 == 0 ? 256 : 128; }

// Split count of the unfused path's three gradient products.  They run side
// by side on three streams, one CTA per SM, G2 launched first (its tiles are
// the wider ones where dh > d).  The count taken is the one whose greedy
// schedule of those CTAs, in launch order on the SMs, ends first (a CTA's time
// taken as its tile width times its k-steps plus a few for the prologue and
// the epilogue); at most UPB_MAX_SPLITS, so the slab update still sums the
// partials, and at least eight k-steps per split.
static int grad_splits_sched(int BH, int d, int dh, int cmax) {
  const int ksteps = (cmax + 63) / 64;
  const int bn13 = grad_bn13(d), bn2 = grad_bn2(dh);
  const long long t13 = (long long)BH * ((dh + 127) / 128) * (d / bn13);
  const long long t2 = (long long)BH * ((d + 127) / 128) * (dh / bn2);
  const int sms = num_sms();
  const int smax = std::max(1, std::min(UPB_MAX_SPLITS, ksteps / 8));
  int best = 1;
  double best_t = 0.0;
  std::vector<double> free_at;
  for (int s = 1; s <= smax; ++s) {
    const int kps = (ksteps + s - 1) / s;
    free_at.assign(sms, 0.0);   // min-heap of the times the SMs come free
    auto place = [&](long long n, int bn) {
      for (long long i = 0; i < n; ++i) {
        std::pop_heap(free_at.begin(), free_at.end(), std::greater<double>());
        free_at.back() += (double)bn * (kps + 4);
        std::push_heap(free_at.begin(), free_at.end(), std::greater<double>());
      }
    };
    place(t2 * s, bn2);
    place(2 * t13 * s, bn13);
    const double t = *std::max_element(free_at.begin(), free_at.end());
    if (s == 1 || t < best_t) { best = s; best_t = t; }
  }
  return best;
}

// head dim 128 (dh a multiple of 64), no split operands, GD or momentum: the
// key pass and the chunk gradient run as one fused kernel (lact_keygrad.cu)
// The chunk-loop launch is on unless TTT_LACT_CHUNK_LOOP=0 (read once).
bool lact_chunk_loop_enabled() {
  static const bool on = [] {
    const char* e = getenv("TTT_LACT_CHUNK_LOOP");
    return !(e != nullptr && e[0] == '0');
  }();
  return on;
}

bool lact_uses_keygrad(int d, int dh, int opt, int split) {
  return d == 128 && dh % 64 == 0 && !split && opt != 2;
}

// W2 alone updated by plain GD without row normalisation, causal order,
// whole chunks of whole tiles: W1 and W3 stay fixed, so the layer is
// block-causal linear attention on the features silu(W1 x) * (W3 x) and no
// chunk depends on an earlier chunk's weights ("Test-Time Training with KV
// Binding Is Secretly Linear Attention", Resumen técnico §4: with only the
// last layer updated and no normalisation the layer reduces to linear
// attention, which has a parallel form).  It runs as one key pass over all
// tokens, one split-K GEMM whose splits are the chunks (the per-chunk W2
// increments), a prefix over chunks and one batched read.
bool lact_uses_w2_parallel(int N_in, int chunk, int d, int dh, int causal, int opt, int split,
                           int update_mask, int normalize) {
  return causal && opt == 0 && !split && update_mask == 4 && !normalize && N_in > 0 &&
         chunk % 128 == 0 && N_in % chunk == 0 && d % 128 == 0 && dh % 128 == 0;
}

LactWorkspace lact_workspace_layout(int B, int H, int N_in, int N_q, int d, int dh, int chunk,
                                    int causal, int opt, int split, int update_mask,
                                    int normalize, int allow_parallel) {
  LactWorkspace w{};
  const size_t BH = (size_t)B * H;
  const int cin = std::min(chunk, std::max(N_in, 1));
  int cmax = std::max(cin, causal ? 0 : N_q);
  cmax = (cmax + 127) / 128 * 128;
  w.cmax = cmax;
  w.w2par = allow_parallel &&
                    lact_uses_w2_parallel(N_in, chunk, d, dh, causal, opt, split, update_mask, normalize)
                ? 1 : 0;
  if (w.w2par) {   // every token at once: features, increments per chunk, chunk-start weights
    const int nch = N_in / chunk;
    w.cmax = (N_in + 127) / 128 * 128;
    w.splits = nch;
    w.keygrad = 0;
    w.nbuf = 1;
    w.naq = 1;
    size_t o = 0;
    w.status = o; o = align256(o + 256);
    w.w1b = o; o = align256(o + BH * dh * d * 2);
    w.w3b = o; o = align256(o + BH * dh * d * 2);
    w.w2b = o; o = align256(o + BH * d * dh * 2);
    w.aq = o; o = align256(o + BH * w.cmax * dh * 2);
    w.gm = o; o = align256(o + BH * w.cmax * dh * 2);
    w.d13 = o;
    w.part = o; o = align256(o + (size_t)nch * BH * d * dh * 4);
    w.pmb = o; o = align256(o + (size_t)nch * BH * d * dh * 2);
    w.rowss = w.nsx32 = w.nsxb = w.nsa32 = w.nsab = w.nsbb = o;
    w.w1lo = w.w3lo = w.w2lo = w.d13lo = w.gmlo = w.aqlo = w.nsxlo = w.nsalo = w.nsblo = o;
    w.total = o;
    return w;
  }
  w.keygrad = lact_uses_keygrad(d, dh, opt, split) ? 1 : 0;
  w.splits = w.keygrad ? std::max(grad_splits((int)BH, d, dh, cin), keygrad_groups((int)BH, dh, cin, 0))
                       : grad_splits_sched((int)BH, d, dh, cin);
  // bf16 operand copies: chunk c reads buffer c mod nbuf while its update
  // writes the next one.  On the fused causal path the read of chunk c runs
  // beside the next chunk, so a third buffer (and a second Aq) keeps what it
  // reads intact.
  w.nbuf = w.keygrad && causal ? 3 : 2;
  w.naq = w.keygrad && causal ? 2 : 1;
  size_t o = 0;
  w.status = o; o = align256(o + 256);
  w.w1b = o; o = align256(o + w.nbuf * BH * dh * d * 2);
  w.w3b = o; o = align256(o + w.nbuf * BH * dh * d * 2);
  w.w2b = o; o = align256(o + w.nbuf * BH * d * dh * 2);
  w.aq = o; o = align256(o + w.naq * BH * cmax * dh * 2);
  w.d13 = w.gm = o;
  if (!w.keygrad) {   // key-pass intermediates of the unfused path
    w.d13 = o; o = align256(o + BH * cmax * 2 * dh * 2);
    w.gm = o; o = align256(o + BH * cmax * dh * 2);
  }
  w.part = o; o = align256(o + (size_t)w.splits * BH * 3 * d * dh * 4);
  w.loopctr = o;
  if (w.keygrad && causal) o = align256(o + 4 * (3 * BH + 2));
  w.rowss = w.nsx32 = w.nsxb = w.nsa32 = w.nsab = w.nsbb = o;
  if (opt == 2) {
    const size_t r = std::min(d, dh), c = std::max(d, dh);
    w.rowss = o; o = align256(o + 3 * BH * std::max(d, dh) * 4);
    w.nsx32 = o; o = align256(o + 3 * BH * r * c * 4);
    w.nsxb = o; o = align256(o + 2 * 3 * BH * r * c * 2);
    w.nsa32 = o; o = align256(o + 3 * BH * r * r * 4);
    w.nsab = o; o = align256(o + 3 * BH * r * r * 2);
    w.nsbb = o; o = align256(o + 3 * BH * r * r * 2);
    w.nsctr = o; o = align256(o + 256);
  }
  w.w1lo = w.w3lo = w.w2lo = w.d13lo = w.gmlo = w.aqlo = w.nsxlo = w.nsalo = w.nsblo = o;
  if (split) {
    w.w1lo = o; o = align256(o + 2 * BH * dh * d * 2);
    w.w3lo = o; o = align256(o + 2 * BH * dh * d * 2);
    w.w2lo = o; o = align256(o + 2 * BH * d * dh * 2);
    w.d13lo = o; o = align256(o + BH * cmax * 2 * dh * 2);
    w.gmlo = o; o = align256(o + BH * cmax * dh * 2);
    w.aqlo = o; o = align256(o + BH * cmax * dh * 2);
    if (opt == 2) {
      const size_t r = std::min(d, dh), c = std::max(d, dh);
      w.nsxlo = o; o = align256(o + 2 * 3 * BH * r * c * 2);
      w.nsalo = o; o = align256(o + 3 * BH * r * r * 2);
      w.nsblo = o; o = align256(o + 3 * BH * r * r * 2);
    }
  }
  w.total = o;
  return w;
}

template <int BN, bool A_MN, bool B_MN, int STAGES, bool BLK = false>
static int run_gemm(const GemmMaps& maps, const GemmArgs& g, cudaStream_t stream, int kind,
                    int max_grid = 0) {
  auto kfn = gemm_bf16_kernel<BN, A_MN, B_MN, STAGES, BLK>;
  const int smem = (int)GemmSmem<BN, STAGES>::BYTES;
  static std::atomic<uint64_t> attr_done{0};
  if (allow_dynamic_smem(kfn, smem, attr_done)) return -1;
  const int tiles = ((g.M + 127) / 128) * (g.N / BN) * g.splits * g.batch;
  if (tiles <= 0) return 0;
  // cluster mode: one tile per CTA, N tiles of a row block in one cluster
  const int cl = g.cluster_n > 1 ? g.cluster_n : 1;
  if (cl > 1 && (g.N / BN != cl || g.splits != 1)) return -1;
  const int grid = cl > 1 ? tiles : std::min(tiles, max_grid > 0 ? max_grid : num_sms());
  prof_before(kind, stream);
  if (launch_pdl_cluster(kfn, dim3(grid), dim3(192), smem, stream, cl, maps, g) != cudaSuccess)
    return -1;
  prof_after(kind, stream);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

static GemmArgs gemm_defaults(const DevStatus& st) {
  GemmArgs g{};
  g.splits = 1;
  g.npairs = 1;
  g.alpha = 1.f;
  g.st = st;
  return g;
}

// The batched GEMM for other files of the library (the LaCT backward pass):
// operand majorness by variant, 128-wide N tiles, four stages.
int gemm_launch(int variant, const GemmMaps& maps, const GemmArgs& g, cudaStream_t stream,
                int kind) {
  switch (variant) {
    case GEMM_AK_BK: return run_gemm<128, false, false, 4>(maps, g, stream, kind);
    case GEMM_AK_BMN: return run_gemm<128, false, true, 4>(maps, g, stream, kind);
    case GEMM_AMN_BMN: return run_gemm<128, true, true, 4>(maps, g, stream, kind);
    default: return -1;
  }
}
GemmArgs gemm_args_default(const DevStatus& st) { return gemm_defaults(st); }

#define TTT_TRY(...)                      \
  do {                                    \
    if ((__VA_ARGS__) != 0) return -1;    \
  } while (0)

// Parallel form of the W2-only layer: W2 before chunk c (bf16, the read's
// operand) and W2 after the last chunk, from W2_0 and the chunks' gradient
// sums part[c] = sum_t (-eta_t v_t) phi(k_t)^T, summed in chunk order.
__global__ void w2_prefix_kernel(float* W2, const float* part, __nv_bfloat16* Mb, int BH, int dd,
                                 int nch) {
  pdl_wait();
  pdl_launch_dependents();
  const size_t n4 = (size_t)BH * dd / 4;
  for (size_t e4 = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e4 < n4;
       e4 += (size_t)gridDim.x * blockDim.x) {
    const size_t e = e4 * 4;
    const size_t bh = e / dd, r = e % dd;
    float4 m = *reinterpret_cast<const float4*>(W2 + e);
    for (int c = 0; c < nch; ++c) {
      *reinterpret_cast<uint2*>(Mb + (bh * nch + c) * dd + r) =
          make_uint2(pack_bf16x2(m.x, m.y), pack_bf16x2(m.z, m.w));
      const float4 p = __ldcg(reinterpret_cast<const float4*>(part + ((size_t)c * BH + bh) * dd + r));
      m.x -= p.x; m.y -= p.y; m.z -= p.z; m.w -= p.w;
    }
    *reinterpret_cast<float4*>(W2 + e) = m;
  }
}

// Chunk gradient of a token range: G[m] = sum over the partial-sum slots of
// matrix m, in slot order (the update kernels sum them the same way).
__global__ void lact_grad_sum_kernel_strided(const float* __restrict__ part, float* __restrict__ G,
                                             size_t mat_elems, int slots, int used) {
  pdl_wait();
  pdl_launch_dependents();
  const size_t n4 = mat_elems / 4;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < 3 * n4;
       i += (size_t)gridDim.x * blockDim.x) {
    const size_t m = i / n4, e = (i % n4) * 4;
    const float* p = part + m * (size_t)slots * mat_elems + e;
    float4 acc = __ldcg(reinterpret_cast<const float4*>(p));
    for (int sp = 1; sp < used; ++sp) {
      const float4 x = __ldcg(reinterpret_cast<const float4*>(p + (size_t)sp * mat_elems));
      acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
    }
    *reinterpret_cast<float4*>(G + m * mat_elems + e) = acc;
  }
}

int launch_lact(const LactLaunch& L, cudaStream_t stream) {
  const int BH = L.B * L.H, d = L.d, dh = L.dh;
  const bool split = L.split != 0;
  // the parallel form of the W2-only layer runs when the workspace holds it,
  // else the chunk loop; the per-chunk pieces of context parallelism (and the
  // backward pass built on them) always use the chunk loop's layout
  LactWorkspace w =
      lact_workspace_layout(L.B, L.H, L.N_in, L.N_q, d, dh, L.chunk, L.causal, L.opt, L.split,
                            L.update_mask, L.normalize_rows, L.mode == LACT_FULL ? 1 : 0);
  if (w.w2par && w.total > L.ws_bytes)
    w = lact_workspace_layout(L.B, L.H, L.N_in, L.N_q, d, dh, L.chunk, L.causal, L.opt, L.split,
                              L.update_mask, L.normalize_rows, 0);
  uint8_t* ws = L.ws;
  auto bf = [&](size_t off) { return reinterpret_cast<__nv_bfloat16*>(ws + off); };
  const size_t wsz = (size_t)BH * d * dh;
  const int nbuf = w.nbuf;
  __nv_bfloat16* wbuf[3][3];
  __nv_bfloat16* lbuf[3][3];
  for (int b = 0; b < nbuf; ++b) {
    wbuf[b][0] = bf(w.w1b) + b * wsz;
    wbuf[b][1] = bf(w.w3b) + b * wsz;
    wbuf[b][2] = bf(w.w2b) + b * wsz;
    lbuf[b][0] = split ? bf(w.w1lo) + b * wsz : nullptr;
    lbuf[b][1] = split ? bf(w.w3lo) + b * wsz : nullptr;
    lbuf[b][2] = split ? bf(w.w2lo) + b * wsz : nullptr;
  }
  __nv_bfloat16 *D13 = w.w2par ? nullptr : bf(w.d13), *Gm = bf(w.gm), *Aq = bf(w.aq);
  __nv_bfloat16 *D13lo = split ? bf(w.d13lo) : nullptr, *Gmlo = split ? bf(w.gmlo) : nullptr, *Aqlo = split ? bf(w.aqlo) : nullptr;
  float* part = reinterpret_cast<float*>(ws + w.part);
  const size_t mat_elems = (size_t)BH * d * dh;
  float* W1 = L.state;
  float* W3 = W1 + mat_elems;
  float* W2 = W3 + mat_elems;
  float* M1 = L.opt != 0 ? W2 + mat_elems : nullptr;
  float* M3 = M1 ? M1 + mat_elems : nullptr;
  float* M2 = M3 ? M3 + mat_elems : nullptr;

  RowArgs ra{};
  ra.BH = BH; ra.d = d; ra.dh = dh; ra.splits = w.splits; ra.opt = L.opt;
  ra.normalize = L.normalize_rows; ra.mask = L.update_mask; ra.beta = L.beta;
  ra.norm_eps = L.norm_eps; ra.ns_eps = L.ns_eps; ra.st = L.st;
  ra.W[0] = W1; ra.W[1] = W3; ra.W[2] = W2;
  ra.M[0] = M1; ra.M[1] = M3; ra.M[2] = M2;
  auto set_out_buf = [&](int b) {
    for (int i = 0; i < 3; ++i) {
      ra.Wb[i] = wbuf[b][i];
      ra.Wlo[i] = lbuf[b][i];
    }
  };
  ra.part[0] = part;
  ra.part[1] = part + (size_t)w.splits * mat_elems;
  ra.part[2] = part + 2 * (size_t)w.splits * mat_elems;
  ra.rowss = reinterpret_cast<float*>(ws + w.rowss);
  ra.X32 = reinterpret_cast<float*>(ws + w.nsx32);
  const int row_warps = BH * (2 * dh + d);
  const int row_blocks = (row_warps * 32 + 255) / 256;
  // GD / momentum row update: slab kernel with bulk copies (split count
  // bounded by its shared memory), else one warp per row
  auto row_update = [&](cudaStream_t st) -> int {
    prof_before(K_UPDATE, st);
    cudaError_t e;
    if (ra.splits <= UPB_MAX_SPLITS && d % 128 == 0 && dh % 128 == 0) {
      static std::atomic<uint64_t> upb_attr{0};
      if (allow_dynamic_smem(lact_update_bulk_kernel, (int)((UPB_MAX_SPLITS + 2) * UPB_SLAB),
                             upb_attr))
        return -1;
      e = launch_pdl(lact_update_bulk_kernel, dim3(update_bulk_blocks(BH, d, dh)), dim3(UPB_THREADS),
                     (size_t)(ra.splits + 2) * UPB_SLAB, st, ra);
    } else {
      e = launch_pdl(lact_update_kernel,
                     dim3((row_warps + UPD_ROWS_PER_BLOCK * UPD_RPW - 1) / (UPD_ROWS_PER_BLOCK * UPD_RPW)),
                     dim3(UPD_ROWS_PER_BLOCK * 32), 0, st, ra);
    }
    if (e != cudaSuccess) return -1;
    prof_after(K_UPDATE, st);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
  };

  set_out_buf(0);
  // only buffer 0 is read before an update writes it, unless a matrix is
  // never updated (update_mask): then every buffer must hold it
  ra.nbuf = (L.update_mask & 7) == 7 ? 1 : nbuf;
  ra.buf_stride = wsz;
  // Where the shape allows, one cooperative launch runs the whole causal
  // sequence (lact_keygrad.cu): no kernel boundary between a chunk's
  // gradient, its row update and the next chunk, and the reads on the spare
  // SMs; it also makes the start weights' bf16 copies itself.
  // TTT_LACT_CHUNK_LOOP=0 in the environment keeps the per-chunk launches.
  int loop_g = 0, loop_nw = 0, loop_nr = 0;
  // the backward's replay runs the loop too (no queries, no read), when every
  // matrix is updated (a matrix the update leaves alone is not snapshotted)
  const bool loop_mode = (L.mode == LACT_FULL && L.out != nullptr) ||
                         (L.mode == LACT_REPLAY && (L.update_mask & 7) == 7);
  const bool use_loop = w.keygrad && L.causal && loop_mode && !split && L.opt != 2 &&
                        L.N_in > 0 && w.nbuf == 3 && w.naq == 2 &&
                        lact_chunk_loop_enabled() &&
                        lact_loop_plan(BH, L.N_in, L.chunk, dh, w.splits, &loop_g, &loop_nw, &loop_nr) == 0;
  if (L.mode != LACT_APPLY && !use_loop) {   // the update of an APPLY call writes its own copies
    prof_before(K_LACT_CAST, stream);
    if (launch_pdl(lact_cast_kernel, dim3(row_blocks), dim3(256), 0, stream, ra) != cudaSuccess)
      return -1;
    prof_after(K_LACT_CAST, stream);
  }
  ra.nbuf = 1;
  TTT_TRY(cudaGetLastError() == cudaSuccess ? 0 : -1);
  // replay: the chunk's start weights are kept, and its update records the
  // row norms
  auto replay_save = [&](int chunk) -> int {
    if (L.mode != LACT_REPLAY) return 0;
    ra.rownorm = L.rownorm_all ? L.rownorm_all + (size_t)chunk * BH * (2 * dh + d) : nullptr;
    if (L.wsave == nullptr) return 0;
    return cudaMemcpyAsync(L.wsave + (size_t)chunk * 3 * mat_elems, L.state, 3 * mat_elems * sizeof(float),
                           cudaMemcpyDeviceToDevice, stream) == cudaSuccess ? 0 : -1;
  };

  // ---- tensor maps.  Token tensors {d, rows, BH}; K-major boxes {64, 128},
  // MN-major boxes {64, 64}.  Weights (bf16 copies): W1, W3 [BH][dh][d],
  // W2 [BH][d][dh].
  const uint64_t tok_row = (uint64_t)d * 2;
  const int q_rows = L.causal ? L.N_in : L.N_q;
  auto tok_map = [&](CUtensorMap* m, const void* p, int rows, uint32_t box_rows) {
    return make_tmap_bf16_3d(m, p, d, rows, BH, tok_row, tok_row * rows, 64, box_rows);
  };
  auto w13_map = [&](CUtensorMap* m, const void* p) {    // K-major, 64 hidden rows per box
    return make_tmap_bf16_3d(m, p, d, dh, BH, (uint64_t)d * 2, (uint64_t)d * dh * 2, 64, 64);
  };
  auto w2_mn_map = [&](CUtensorMap* m, const void* p) {  // MN-major (hidden contiguous)
    return make_tmap_bf16_3d(m, p, dh, d, BH, (uint64_t)dh * 2, (uint64_t)d * dh * 2, 64, 64);
  };
  auto w2_k_map = [&](CUtensorMap* m, const void* p) {   // K-major B for the read (N = d)
    return make_tmap_bf16_3d(m, p, dh, d, BH, (uint64_t)dh * 2, (uint64_t)d * dh * 2, 64, 128);
  };
  auto inter_map = [&](CUtensorMap* m, const void* p, int rows, uint32_t box_rows) {
    return make_tmap_bf16_3d(m, p, dh, rows, BH, (uint64_t)dh * 2, (uint64_t)w.cmax * dh * 2, 64,
                             box_rows);
  };
  // which token tensors this call reads (the context-parallel pieces read a
  // subset and may leave the others null)
  const bool uses_kv =
      L.N_in > 0 && (L.mode == LACT_FULL || L.mode == LACT_GRAD || L.mode == LACT_REPLAY);
  const bool uses_q = q_rows > 0 && (L.mode == LACT_FULL || L.mode == LACT_READ);
  KeyPassMaps km{};
  if (uses_kv) {
    TTT_TRY(tok_map(&km.k, L.k, L.N_in, 128));
    TTT_TRY(tok_map(&km.v, L.v, L.N_in, 128));
  }
  if (uses_q) TTT_TRY(tok_map(&km.q, L.q, q_rows, 128));
  else km.q = km.k;
  if (!uses_kv) { km.k = km.q; km.v = km.q; }
  // the key pass's tensor-store views (its staged epilogue: no split
  // operands); a workspace laid out for the fused key-gradient kernel has no
  // key-pass intermediates and gets none
  const bool kp_staged = !w.keygrad;
  if (kp_staged) {
    const uint64_t ibs = (uint64_t)w.cmax * dh * 2;   // bytes per head of Gm' / Aq
    if (!split) {
      if (D13 != nullptr)
        TTT_TRY(make_tmap_bf16_3d_sw(&km.od13, D13, 2 * dh, w.cmax, BH, (uint64_t)dh * 4, 2 * ibs, 64, 128, 128));
      TTT_TRY(make_tmap_bf16_3d_sw(&km.ogm, Gm, dh, w.cmax, BH, (uint64_t)dh * 2, ibs, 64, 128, 128));
      TTT_TRY(make_tmap_bf16_3d_sw(&km.oaq, Aq, dh, w.cmax, BH, (uint64_t)dh * 2, ibs, 64, 128, 128));
    } else {
      __nv_bfloat16* d13p[2] = {D13, D13lo};
      __nv_bfloat16* gmp[2] = {Gm, Gmlo};
      __nv_bfloat16* aqp[2] = {Aq, Aqlo};
      for (int p = 0; p < 2; ++p) {
        if (d13p[p] != nullptr)
          TTT_TRY(make_tmap_bf16_3d_sw(&km.sd13[p], d13p[p], 2 * dh, w.cmax, BH, (uint64_t)dh * 4, 2 * ibs, 32, 128, 64));
        TTT_TRY(make_tmap_bf16_3d_sw(&km.sgm[p], gmp[p], dh, w.cmax, BH, (uint64_t)dh * 2, ibs, 32, 128, 64));
        TTT_TRY(make_tmap_bf16_3d_sw(&km.saq[p], aqp[p], dh, w.cmax, BH, (uint64_t)dh * 2, ibs, 32, 128, 64));
      }
    }
  }
  KeyPassMaps kmb[3] = {km, km, km};
  CUtensorMap mw2k[3], mw2klo[3];
  for (int b = 0; b < nbuf; ++b) {
    TTT_TRY(w13_map(&kmb[b].w1, wbuf[b][0]));
    TTT_TRY(w13_map(&kmb[b].w3, wbuf[b][1]));
    TTT_TRY(w2_mn_map(&kmb[b].w2, wbuf[b][2]));
    TTT_TRY(w2_k_map(&mw2k[b], wbuf[b][2]));
    if (split) {
      TTT_TRY(w13_map(&kmb[b].w1lo, lbuf[b][0]));
      TTT_TRY(w13_map(&kmb[b].w3lo, lbuf[b][1]));
      TTT_TRY(w2_mn_map(&kmb[b].w2lo, lbuf[b][2]));
      TTT_TRY(w2_k_map(&mw2klo[b], lbuf[b][2]));
    } else {
      kmb[b].w1lo = kmb[b].w1; kmb[b].w3lo = kmb[b].w3; kmb[b].w2lo = kmb[b].w2;
      mw2klo[b] = mw2k[b];
    }
  }
  int cur = 0;   // buffer holding the chunk-start weights
  auto nxt = [&](int b) { return b + 1 == nbuf ? 0 : b + 1; };   // buffer its update writes
  CUtensorMap mk_mn{}, mv_mn{};   // token tensors as MN-major operands
  if (uses_kv) {
    TTT_TRY(tok_map(&mk_mn, L.k, L.N_in, 64));
    TTT_TRY(tok_map(&mv_mn, L.v, L.N_in, 64));
  }

  static std::atomic<uint64_t> kp_attr[2];
  if (split ? allow_dynamic_smem(lact_keypass_kernel<true>, (int)kp::SMEM, kp_attr[1])
            : allow_dynamic_smem(lact_keypass_kernel<false>, (int)kp::SMEM, kp_attr[0]))
    return -1;

  auto key_pass_on = [&](int t0, int C, int nkt, int nqt, cudaStream_t kstream) -> int {
    // never launch on a token or store map this call did not encode
    if ((nkt > 0 && !uses_kv) || (nqt > 0 && !uses_q) || !kp_staged) return -1;
    KeyPassArgs a{};
    a.C = C; a.t0 = t0; a.n_key_tiles = nkt; a.n_q_tiles = nqt; a.n_hb = dh / 64; a.BH = BH;
    a.d_steps = d / 64; a.dh = dh; a.lr_len = L.N_in; a.lr = L.lr;
    a.D13 = D13; a.Gm = Gm; a.Aq = Aq;
    a.split = split ? 1 : 0; a.D13lo = D13lo; a.Gmlo = Gmlo; a.Aqlo = Aqlo;
    a.feat_only = D13 == nullptr ? 1 : 0;
    a.inter_bs = (long long)w.cmax * dh; a.st = L.st;
    const int tiles = (nkt + nqt) * a.n_hb * BH;
    if (tiles <= 0) return 0;
    prof_before(K_KEYPASS, kstream);
    const cudaError_t e =
        split ? launch_pdl(lact_keypass_kernel<true>, dim3(std::min(tiles, num_sms())), dim3(kp::THREADS),
                           kp::SMEM, kstream, kmb[cur], a)
              : launch_pdl(lact_keypass_kernel<false>, dim3(std::min(tiles, num_sms())), dim3(kp::THREADS),
                           kp::SMEM, kstream, kmb[cur], a);
    if (e != cudaSuccess) return -1;
    prof_after(K_KEYPASS, kstream);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
  };
  auto key_pass = [&](int t0, int C, int nkt, int nqt) -> int {
    return key_pass_on(t0, C, nkt, nqt, stream);
  };
  // out rows [t0, t0 + C) = Aq W2^T (split: hi*hi + hi*lo + lo*hi)
  auto read_out = [&](int t0, int C, cudaStream_t rstream, const __nv_bfloat16* aq,
                      int max_grid = 0) -> int {
    GemmArgs g = gemm_defaults(L.st);
    g.M = C; g.N = d; g.batch = BH; g.k_steps = dh / 64;
    g.out_row_off = t0;
    const int orows = L.causal ? L.N_in : L.N_q;
    if (L.out_bf16) {
      g.o16 = reinterpret_cast<__nv_bfloat16*>(L.out);
      g.o16_bs = (long long)orows * d;
      g.ld16 = d;
    } else {
      g.o32 = reinterpret_cast<float*>(L.out);
      g.o32_bs = (long long)orows * d;
      g.ld32 = d;
    }
    GemmMaps m{};
    TTT_TRY(inter_map(&m.a[0], aq, C, 128));
    m.b[0] = mw2k[cur];
    if (split) {
      g.npairs = 3;
      m.a[1] = m.a[0];
      m.b[1] = mw2klo[cur];
      TTT_TRY(inter_map(&m.a[2], Aqlo, C, 128));
      m.b[2] = mw2k[cur];
    }
    return run_gemm<128, false, false, 4>(m, g, rstream, K_GEMM_READ, max_grid);
  };
  // Chunk gradients G1 = dH1^T K, G3 = dH3^T K (rows = hidden units, N = d)
  // and G2 = V^T Gm' (rows = d, N = dh), contracted over the chunk's tokens.
  // fused (GD / momentum, d in {128, 256}, dh <= 256, chunk <= 8192): one
  // launch for [G1; G3] (stacked rows of D13^T) and one for G2 (N tiles of
  // a W2 row block in one cluster), each with the weight update, row
  // normalisation and bf16 copies in the epilogue.  Otherwise split-K
  // partial sums go to the row update kernels.
  const int cmax_chunk = std::min(L.chunk, std::max(L.N_in, 1));
  const bool fused_update = L.opt != 2 && (d == 128 || d == 256) && (dh == 128 || dh == 256) &&
                            cmax_chunk <= 8192 && L.mode != LACT_REPLAY;
  auto d13_map = [&](CUtensorMap* m, const void* p, int rows) {
    return make_tmap_bf16_3d(m, p, 2 * dh, rows, BH, (uint64_t)dh * 4, (uint64_t)w.cmax * dh * 4,
                             64, 64);
  };
  auto gradients = [&](int t0, int C, cudaStream_t* mstream, bool partials_only) -> int {
    if (!uses_kv) return -1;   // the K / V maps were not encoded for this call
    CUtensorMap md, mdl, mg, mgl;
    TTT_TRY(d13_map(&md, D13, C));
    TTT_TRY(inter_map(&mg, Gm, C, 64));
    if (split) {
      TTT_TRY(d13_map(&mdl, D13lo, C));
      TTT_TRY(inter_map(&mgl, Gmlo, C, 64));
    }
    const int ksteps_total = (C + 63) / 64;
    const int np = split ? 2 : 1;
    if (fused_update && !partials_only) {
      GemmArgs g = gemm_defaults(L.st);
      g.batch = BH; g.splits = 1; g.k_steps = ksteps_total; g.npairs = np; g.epi = 1;
      g.mom_beta = L.beta; g.norm_eps = L.norm_eps; g.normalize = L.normalize_rows;
      GemmMaps m{};
      // [G1; G3]: rows 0..dh-1 update W1, rows dh..2dh-1 update W3
      if ((L.update_mask & 3) != 0) {
        GemmArgs g13 = g;
        g13.M = 2 * dh; g13.N = d; g13.ldw = d; g13.rows_first = dh;
        g13.W[0] = W1; g13.W[1] = W3; g13.Mom[0] = M1; g13.Mom[1] = M3;
        g13.Wb[0] = wbuf[nxt(cur)][0]; g13.Wb[1] = wbuf[nxt(cur)][1];
        g13.Wlo[0] = lbuf[nxt(cur)][0]; g13.Wlo[1] = lbuf[nxt(cur)][1];
        if ((L.update_mask & 3) == 2) { g13.a_m_off[0] = g13.a_m_off[1] = dh; g13.M = dh; g13.rows_first = 0; }
        if ((L.update_mask & 3) == 1) { g13.M = dh; }
        for (int p = 0; p < np; ++p) {
          m.a[p] = p == 0 ? md : mdl;
          m.b[p] = mk_mn;
          g13.b_k_off[p] = t0;
        }
        if (d == 128) TTT_TRY(run_gemm<128, true, true, 6>(m, g13, mstream[0], K_GEMM_GRAD));
        else TTT_TRY(run_gemm<256, true, true, 4>(m, g13, mstream[0], K_GEMM_GRAD));
      }
      if (L.update_mask & 4) {
        GemmArgs g2 = g;
        g2.M = d; g2.N = dh; g2.ldw = dh; g2.rows_first = d; g2.cluster_n = dh / 128;
        g2.W[0] = W2; g2.Mom[0] = M2; g2.Wb[0] = wbuf[nxt(cur)][2]; g2.Wlo[0] = lbuf[nxt(cur)][2];
        for (int p = 0; p < np; ++p) {
          m.a[p] = mv_mn;
          m.b[p] = p == 0 ? mg : mgl;
          g2.a_k_off[p] = t0;
          g2.b_k_off[p] = 0;
        }
        TTT_TRY(run_gemm<128, true, true, 6>(m, g2, mstream[1], K_GEMM_GRAD));
      }
      return 1;
    }
    const int splits = std::min(w.splits, ksteps_total);
    const int kps = (ksteps_total + splits - 1) / splits;
    // the same operands through blocked views: one copy per operand per stage
    // (A blocks of 128 rows, B blocks of the tile width)
    const int bn13 = grad_bn13(d), bn2 = grad_bn2(dh);
    CUtensorMap bd13[2], bk13, bv, bg[2];
    TTT_TRY(make_tmap_bf16_blocked(&bd13[0], D13, 2 * dh, C, BH, (uint64_t)dh * 4,
                                   (uint64_t)w.cmax * dh * 4, 64, 2));
    TTT_TRY(make_tmap_bf16_blocked(&bg[0], Gm, dh, C, BH, (uint64_t)dh * 2,
                                   (uint64_t)w.cmax * dh * 2, 64, bn2 / 64));
    if (split) {
      TTT_TRY(make_tmap_bf16_blocked(&bd13[1], D13lo, 2 * dh, C, BH, (uint64_t)dh * 4,
                                     (uint64_t)w.cmax * dh * 4, 64, 2));
      TTT_TRY(make_tmap_bf16_blocked(&bg[1], Gmlo, dh, C, BH, (uint64_t)dh * 2,
                                     (uint64_t)w.cmax * dh * 2, 64, bn2 / 64));
    }
    TTT_TRY(make_tmap_bf16_blocked(&bk13, L.k, d, L.N_in, BH, tok_row, tok_row * L.N_in, 64, bn13 / 64));
    TTT_TRY(make_tmap_bf16_blocked(&bv, L.v, d, L.N_in, BH, tok_row, tok_row * L.N_in, 64, 2));
    GemmArgs g = gemm_defaults(L.st);
    g.batch = BH; g.splits = splits; g.k_steps = kps; g.npairs = np;
    g.o32_ss = (long long)BH * d * dh;
    g.o32_bs = (long long)d * dh;
    // G2 first (grad_splits_sched models this order): where dh > d its CTAs
    // are the longest, and the shorter ones fill in behind them
    for (int mi = 0; mi < 3; ++mi) {
      const int mat = (mi + 2) % 3;
      GemmMaps m{};
      if (mat < 2) {
        g.M = dh; g.N = d; g.ld32 = d;
        for (int p = 0; p < np; ++p) {
          m.a[p] = bd13[p];
          m.b[p] = bk13;
          g.a_m_off[p] = mat * dh; g.a_k_off[p] = 0; g.b_k_off[p] = t0;
        }
      } else {
        g.M = d; g.N = dh; g.ld32 = dh;
        for (int p = 0; p < np; ++p) {
          m.a[p] = bv;
          m.b[p] = bg[p];
          g.a_m_off[p] = 0; g.a_k_off[p] = t0; g.b_k_off[p] = 0;
        }
      }
      g.o32 = const_cast<float*>(ra.part[mat]);
      // wide N tiles read the long token-major operands fewer times: 192 for
      // [G1; G3] (N = d), 256 for G2 (N = dh)
      if (mat < 2 && bn13 == 192)
        TTT_TRY((run_gemm<192, true, true, 5, true>(m, g, mstream[mat], K_GEMM_GRAD)));
      else if (mat == 2 && bn2 == 256)
        TTT_TRY((run_gemm<256, true, true, 4, true>(m, g, mstream[mat], K_GEMM_GRAD)));
      else
        TTT_TRY((run_gemm<128, true, true, 4, true>(m, g, mstream[mat], K_GEMM_GRAD)));
    }
    return splits;
  };
  // Muon: momentum, Newton-Schulz on the wide orientation, apply + norm.
  auto muon = [&]() -> int {
    const int r = std::min(d, dh), c = std::max(d, dh);
    const int nb = 3 * BH;
    float* X32 = reinterpret_cast<float*>(ws + w.nsx32);
    __nv_bfloat16* Xb[2] = {bf(w.nsxb), bf(w.nsxb) + (size_t)nb * r * c};
    __nv_bfloat16* Xl[2] = {split ? bf(w.nsxlo) : nullptr,
                            split ? bf(w.nsxlo) + (size_t)nb * r * c : nullptr};
    float* A32 = reinterpret_cast<float*>(ws + w.nsa32);
    __nv_bfloat16 *Ab = bf(w.nsab), *Bb = bf(w.nsbb);
    __nv_bfloat16 *Al = split ? bf(w.nsalo) : nullptr, *Bl = split ? bf(w.nsblo) : nullptr;
    prof_before(K_MUON_MOM, stream);
    if (launch_pdl(muon_momentum_kernel, dim3(row_warps), dim3(ROW_THREADS), 0, stream, ra) !=
        cudaSuccess)
      return -1;
    prof_after(K_MUON_MOM, stream);
    NsPrepArgs pa{};
    pa.BH = BH; pa.d = d; pa.dh = dh; pa.r = r; pa.c = c; pa.eps = L.ns_eps;
    pa.M[0] = M1; pa.M[1] = M3; pa.M[2] = M2; pa.rowss = ra.rowss; pa.X32 = X32;
    pa.Xb = Xb[0]; pa.Xlo = Xl[0];
    unsigned* ctr = reinterpret_cast<unsigned*>(ws + w.nsctr);
    pa.counter = ctr;
    prof_before(K_NS_PREP, stream);
    if (launch_pdl(ns_prep_kernel, dim3(r, nb), dim3(256), 0, stream, pa) != cudaSuccess)
      return -1;
    prof_after(K_NS_PREP, stream);
    TTT_TRY(cudaGetLastError() == cudaSuccess ? 0 : -1);
    bool fused_ns = L.ns_steps > 0;
    if (fused_ns) {   // every Newton-Schulz step in one cooperative launch
      NsFusedLaunch nl{};
      nl.r = r; nl.c = c; nl.nb = nb; nl.steps = L.ns_steps; nl.split = split ? 1 : 0;
      nl.coef_a = L.ns_a; nl.coef_b = L.ns_b; nl.coef_c = L.ns_c;
      nl.X32 = X32;
      nl.Xb[0] = Xb[0]; nl.Xb[1] = Xb[1]; nl.Xl[0] = Xl[0]; nl.Xl[1] = Xl[1];
      nl.A32 = A32; nl.Ab = Ab; nl.Al = Al; nl.Bb = Bb; nl.Bl = Bl;
      nl.counter = ctr;
      nl.st = L.st;
      TTT_TRY(launch_ns_fused(nl, stream));
    }
    auto sq_map = [&](CUtensorMap* m, const void* p) {
      return make_tmap_bf16_3d(m, p, r, r, nb, (uint64_t)r * 2, (uint64_t)r * r * 2, 64, 128);
    };
    CUtensorMap mab, mbb, mal, mbl, mxk[2], mxn[2], mxkl[2], mxnl[2];
    TTT_TRY(sq_map(&mab, Ab));
    TTT_TRY(sq_map(&mbb, Bb));
    if (split) {
      TTT_TRY(sq_map(&mal, Al));
      TTT_TRY(sq_map(&mbl, Bl));
    }
    for (int i = 0; i < 2; ++i) {
      TTT_TRY(make_tmap_bf16_3d(&mxk[i], Xb[i], c, r, nb, (uint64_t)c * 2, (uint64_t)r * c * 2, 64, 128));
      TTT_TRY(make_tmap_bf16_3d(&mxn[i], Xb[i], c, r, nb, (uint64_t)c * 2, (uint64_t)r * c * 2, 64, 64));
      if (split) {
        TTT_TRY(make_tmap_bf16_3d(&mxkl[i], Xl[i], c, r, nb, (uint64_t)c * 2, (uint64_t)r * c * 2, 64, 128));
        TTT_TRY(make_tmap_bf16_3d(&mxnl[i], Xl[i], c, r, nb, (uint64_t)c * 2, (uint64_t)r * c * 2, 64, 64));
      }
    }
    // products of split operands: hi*hi + hi*lo + lo*hi
    auto pairs = [&](GemmMaps& m, GemmArgs& g, const CUtensorMap& ah, const CUtensorMap& al,
                     const CUtensorMap& bh, const CUtensorMap& bl) {
      m.a[0] = ah; m.b[0] = bh;
      if (split) {
        m.a[1] = ah; m.b[1] = bl;
        m.a[2] = al; m.b[2] = bh;
        g.npairs = 3;
      }
    };
    for (int it = 0; !fused_ns && it < L.ns_steps; ++it) {
      const int cur = it & 1;
      GemmMaps m{};
      // A = X X^T  (fp32 + bf16 hi/lo)
      GemmArgs g = gemm_defaults(L.st);
      g.M = r; g.N = r; g.batch = nb; g.k_steps = c / 64;
      g.o32 = A32; g.o32_bs = (long long)r * r; g.ld32 = r;
      g.o16 = Ab; g.o16lo = Al; g.o16_bs = (long long)r * r; g.ld16 = r;
      pairs(m, g, mxk[cur], mxkl[cur], mxk[cur], mxkl[cur]);
      TTT_TRY(run_gemm<128, false, false, 4>(m, g, stream, K_GEMM_NS));
      // B = b A + c A A
      m = GemmMaps{};
      g = gemm_defaults(L.st);
      g.M = r; g.N = r; g.batch = nb; g.k_steps = r / 64;
      g.alpha = L.ns_c; g.beta = L.ns_b; g.cin = A32; g.cin_bs = (long long)r * r; g.ldc = r;
      g.o16 = Bb; g.o16lo = Bl; g.o16_bs = (long long)r * r; g.ld16 = r;
      pairs(m, g, mab, mal, mab, mal);
      TTT_TRY(run_gemm<128, false, false, 4>(m, g, stream, K_GEMM_NS));
      // X <- a X + B X  (fp32 in place; bf16 hi/lo into the other buffers)
      m = GemmMaps{};
      g = gemm_defaults(L.st);
      g.M = r; g.N = c; g.batch = nb; g.k_steps = r / 64;
      g.alpha = 1.f; g.beta = L.ns_a; g.cin = X32; g.cin_bs = (long long)r * c; g.ldc = c;
      g.o32 = X32; g.o32_bs = (long long)r * c; g.ld32 = c;
      g.o16 = Xb[cur ^ 1]; g.o16lo = Xl[cur ^ 1]; g.o16_bs = (long long)r * c; g.ld16 = c;
      pairs(m, g, mbb, mbl, mxn[cur], mxnl[cur]);
      TTT_TRY(run_gemm<128, false, true, 4>(m, g, stream, K_GEMM_NS));
    }
    prof_before(K_MUON_APPLY, stream);
    if (launch_pdl(muon_apply_kernel, dim3(row_blocks), dim3(256), 0, stream, ra, r, c) !=
        cudaSuccess)
      return -1;
    prof_after(K_MUON_APPLY, stream);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
  };

  // ------------------------------------------------------------ chunk loop
  // Per chunk: key pass; then the memory read and the three gradient GEMMs,
  // which are independent, run concurrently on the caller's stream and the
  // helper streams; then (unfused path) the update.
  SideStreams* ss = side_streams();
  cudaStream_t gstream[3] = {stream, ss ? ss->s[0] : stream, ss ? ss->s[1] : stream};
  cudaStream_t rstream = ss ? ss->s[2] : stream;
  auto fork = [&]() -> int {
    if (!ss) return 0;
    if (cudaEventRecord(ss->fork, stream) != cudaSuccess) return -1;
    for (int i = 0; i < 3; ++i)
      if (cudaStreamWaitEvent(ss->s[i], ss->fork, 0) != cudaSuccess) return -1;
    return 0;
  };
  auto join = [&]() -> int {
    if (!ss) return 0;
    for (int i = 0; i < 3; ++i)
      if (cudaEventRecord(ss->join[i], ss->s[i]) != cudaSuccess ||
          cudaStreamWaitEvent(stream, ss->join[i], 0) != cudaSuccess)
        return -1;
    return 0;
  };
  // ------------------------------------------------------------ context-parallel pieces
  if (L.mode == LACT_APPLY) {
    // the optimizer step and row normalisation with the caller's summed chunk
    // gradient, which takes the place of the partial sums (one slot)
    ra.part[0] = L.G;
    ra.part[1] = L.G + mat_elems;
    ra.part[2] = L.G + 2 * mat_elems;
    ra.splits = 1;
    ra.rownorm = L.rownorm_out;
    set_out_buf(nxt(cur));
    return L.opt == 2 ? muon() : row_update(stream);
  }
  if (L.mode == LACT_READ) {   // queries [t0, t0 + n) read the current weights
    if (L.n <= 0) return 0;
    if (d == 128 && !split) {
      ReadFusedLaunch rl{};
      rl.BH = BH; rl.rows = q_rows; rl.t0 = L.t0; rl.C = L.n; rl.dh = dh; rl.out_bf16 = L.out_bf16;
      rl.max_grid = num_sms();
      rl.q = L.q; rl.w1b = wbuf[cur][0]; rl.w3b = wbuf[cur][1]; rl.w2b = wbuf[cur][2];
      rl.out = L.out; rl.st = L.st;
      return launch_lact_read_fused(rl, stream);
    }
    TTT_TRY(key_pass(L.t0, L.n, 0, (L.n + 127) / 128));
    return read_out(L.t0, L.n, stream, Aq);
  }
  if (L.mode == LACT_GRAD) {   // gradient sum of tokens [t0, t0 + n), no update
    int splits = 1;
    if (L.n > 0 && w.keygrad) {
      KeyGradLaunch kgl{};
      kgl.BH = BH; kgl.N_in = L.N_in; kgl.C = L.n; kgl.t0 = L.t0; kgl.dh = dh;
      kgl.groups = keygrad_groups(BH, dh, L.n, w.splits);
      kgl.k = L.k; kgl.v = L.v; kgl.lr = L.lr; kgl.q = nullptr;
      kgl.Aq = Aq; kgl.aq_bs = (long long)w.cmax * dh;
      kgl.w1b = wbuf[cur][0]; kgl.w3b = wbuf[cur][1]; kgl.w2b = wbuf[cur][2];
      kgl.part[0] = const_cast<float*>(ra.part[0]);
      kgl.part[1] = const_cast<float*>(ra.part[1]);
      kgl.part[2] = const_cast<float*>(ra.part[2]);
      kgl.st = L.st;
      TTT_TRY(launch_lact_keygrad(kgl, stream));
      splits = kgl.groups;
    } else if (L.n > 0) {
      const int nt = (L.n + 127) / 128;
      TTT_TRY(key_pass(L.t0, L.n, nt, 0));
      TTT_TRY(fork());
      splits = gradients(L.t0, L.n, gstream, /*partials_only=*/true);
      if (splits < 0) return -1;
      TTT_TRY(join());
    } else {   // no tokens: a zero gradient
      return cudaMemsetAsync(L.G, 0, 3 * mat_elems * sizeof(float), stream) == cudaSuccess ? 0 : -1;
    }
    // slot s of matrix m sits at part + (m * w.splits + s) * mat_elems
    const size_t n4 = 3 * mat_elems / 4;
    const int blocks = (int)std::min<size_t>((n4 + 255) / 256, 8 * (size_t)num_sms());
    if (launch_pdl(lact_grad_sum_kernel_strided, dim3(blocks), dim3(256), 0, stream,
                   (const float*)part, L.G, mat_elems, w.splits, splits) != cudaSuccess)
      return -1;
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
  }

  if (w.w2par) {
    // ---- parallel form of the W2-only layer (see lact_uses_w2_parallel)
    const int nch = L.N_in / L.chunk;
    const int nt = L.N_in / 128;
    TTT_TRY(key_pass(0, L.N_in, nt, nt));   // phi(q) -> Aq, -eta phi(k) -> Gm'
    {   // per-chunk gradient sums G2_c = V_c^T Gm'_c: the chunks are the splits
      CUtensorMap mg;
      TTT_TRY(inter_map(&mg, Gm, L.N_in, 64));
      GemmArgs g = gemm_defaults(L.st);
      g.M = d; g.N = dh; g.batch = BH; g.splits = nch; g.k_steps = L.chunk / 64; g.npairs = 1;
      g.o32 = part; g.o32_ss = (long long)BH * d * dh; g.o32_bs = (long long)d * dh; g.ld32 = dh;
      GemmMaps m{};
      m.a[0] = mv_mn;
      m.b[0] = mg;
      if (dh % 256 == 0) TTT_TRY(run_gemm<256, true, true, 4>(m, g, stream, K_GEMM_GRAD));
      else TTT_TRY(run_gemm<128, true, true, 4>(m, g, stream, K_GEMM_GRAD));
    }
    __nv_bfloat16* Mb = bf(w.pmb);
    {
      const int dd = d * dh;
      const int blocks = std::min(4 * num_sms(), (int)(((size_t)BH * dd / 4 + 255) / 256));
      prof_before(K_UPDATE, stream);
      if (launch_pdl(w2_prefix_kernel, dim3(blocks), dim3(256), 0, stream, W2, (const float*)part, Mb, BH,
                     dd, nch) != cudaSuccess)
        return -1;
      prof_after(K_UPDATE, stream);
    }
    {   // out rows of chunk c = Aq_c (W2 before chunk c)^T, all chunks at once
      GemmArgs g = gemm_defaults(L.st);
      g.M = L.chunk; g.N = d; g.batch = BH * nch; g.k_steps = dh / 64;
      if (L.out_bf16) {
        g.o16 = reinterpret_cast<__nv_bfloat16*>(L.out);
        g.o16_bs = (long long)L.chunk * d;
        g.ld16 = d;
      } else {
        g.o32 = reinterpret_cast<float*>(L.out);
        g.o32_bs = (long long)L.chunk * d;
        g.ld32 = d;
      }
      GemmMaps m{};
      TTT_TRY(make_tmap_bf16_3d(&m.a[0], Aq, dh, L.chunk, (uint64_t)BH * nch, (uint64_t)dh * 2,
                                (uint64_t)L.chunk * dh * 2, 64, 128));
      TTT_TRY(make_tmap_bf16_3d(&m.b[0], Mb, dh, d, (uint64_t)BH * nch, (uint64_t)dh * 2,
                                (uint64_t)d * dh * 2, 64, 128));
      TTT_TRY(run_gemm<128, false, false, 4>(m, g, stream, K_GEMM_READ));
    }
    return 0;
  }
  // Head dim 128, GD / momentum: per chunk the fused kernel forms Aq (causal)
  // and the gradient partial sums on the chunk-start weights (buffer cur);
  // the row update writes buffer nxt(cur).  The read of chunk c (helper
  // stream; Aq buffer c % 2, W2 buffer cur) runs beside the update and the
  // next chunk on the SMs the fused kernel leaves free; the kernel of chunk
  // c + 2 rewrites both, so it first waits for that read.  (Forming Aq in the
  // fused kernel reuses the [W1_J; W3_J] tiles already in its shared memory:
  // measured faster than a separate Q -> out read kernel on the free SMs.)
  const bool keygrad = w.keygrad != 0;
  int ci = 0;
  // the chunk loop (decided above, before the bf16 copies)
  bool looped = false;
  if (use_loop) {
    {
      KeyGradLoopLaunch ll{};
      ll.BH = BH; ll.N_in = L.N_in; ll.C = L.chunk; ll.dh = dh; ll.max_groups = w.splits;
      ll.cmax = w.cmax;
      ll.k = L.k; ll.v = L.v; ll.q = L.q; ll.lr = L.lr;
      ll.Aq = Aq; ll.aq_buf = (long long)BH * w.cmax * dh;
      for (int b = 0; b < 3; ++b)
        for (int i = 0; i < 3; ++i) ll.Wb[b][i] = wbuf[b][i];
      for (int i = 0; i < 3; ++i) {
        ll.W[i] = ra.W[i];
        ll.M[i] = ra.M[i];
        ll.part[i] = const_cast<float*>(ra.part[i]);
      }
      ll.opt = L.opt; ll.normalize = L.normalize_rows; ll.mask = L.update_mask;
      ll.beta = L.beta; ll.norm_eps = L.norm_eps;
      ll.out = L.out; ll.out_bf16 = L.out_bf16;
      ll.ctr = reinterpret_cast<unsigned*>(ws + w.loopctr);
      ll.cast_first = 1;
      ll.groups = loop_g; ll.workers = loop_nw; ll.readers = loop_nr;
      ll.st = L.st;
      if (L.mode == LACT_REPLAY) {   // keys only; the updates keep every chunk's weights and norms
        ll.q = nullptr;
        ll.out = nullptr;
        ll.readers = 0;
        ll.wsave = L.wsave;
        ll.rownorm = L.normalize_rows ? L.rownorm_all : nullptr;
        if (L.wsave != nullptr)
          TTT_TRY(cudaMemcpyAsync(L.wsave, L.state, 3 * mat_elems * sizeof(float), cudaMemcpyDeviceToDevice,
                                  stream) == cudaSuccess ? 0 : -1);
      }
      TTT_TRY(launch_lact_loop(ll, stream));
      looped = true;
    }
  }
  for (int t0 = 0; keygrad && !looped && t0 < L.N_in; t0 += L.chunk, ++ci) {
    const int C = std::min(L.chunk, L.N_in - t0);
    __nv_bfloat16* aq = Aq + (size_t)(ci % w.naq) * BH * w.cmax * dh;
    KeyGradLaunch kgl{};
    kgl.BH = BH; kgl.N_in = L.N_in; kgl.C = C; kgl.t0 = t0; kgl.dh = dh;
    kgl.groups = keygrad_groups(BH, dh, C, w.splits);
    kgl.k = L.k; kgl.v = L.v; kgl.lr = L.lr;
    const bool reads = L.causal && L.mode != LACT_REPLAY;
    kgl.q = reads ? L.q : nullptr;
    kgl.Aq = aq; kgl.aq_bs = (long long)w.cmax * dh;
    kgl.w1b = wbuf[cur][0]; kgl.w3b = wbuf[cur][1]; kgl.w2b = wbuf[cur][2];
    kgl.part[0] = const_cast<float*>(ra.part[0]);
    kgl.part[1] = const_cast<float*>(ra.part[1]);
    kgl.part[2] = const_cast<float*>(ra.part[2]);
    kgl.st = L.st;
    if (reads && ss && ci >= w.naq)
      TTT_TRY(cudaStreamWaitEvent(stream, ss->read_done[ci & 1], 0) == cudaSuccess ? 0 : -1);
    TTT_TRY(launch_lact_keygrad(kgl, stream));
    if (reads) {   // the read of this chunk runs beside the update and the next chunk
      if (ss) {
        TTT_TRY(cudaEventRecord(ss->fork, stream) == cudaSuccess ? 0 : -1);
        TTT_TRY(cudaStreamWaitEvent(rstream, ss->fork, 0) == cudaSuccess ? 0 : -1);
      }
      const int kg_grid = std::min(BH * (dh / 64) * kgl.groups, num_sms());
      TTT_TRY(read_out(t0, C, rstream, aq, ss ? std::max(8, num_sms() - kg_grid) : 0));
      if (ss) TTT_TRY(cudaEventRecord(ss->read_done[ci & 1], rstream) == cudaSuccess ? 0 : -1);
    }
    ra.splits = kgl.groups;
    set_out_buf(nxt(cur));
    TTT_TRY(replay_save(ci));
    TTT_TRY(row_update(stream));
    cur = nxt(cur);
  }
  if (keygrad && L.causal && L.mode != LACT_REPLAY && ss && ci >= 1)   // the reads join the caller's stream
    TTT_TRY(cudaStreamWaitEvent(stream, ss->read_done[(ci - 1) & 1], 0) == cudaSuccess ? 0 : -1);
  for (int t0 = 0; !keygrad && t0 < L.N_in; t0 += L.chunk, ++ci) {
    const int C = std::min(L.chunk, L.N_in - t0);
    const int nt = (C + 127) / 128;
    const bool reads = L.causal && L.mode != LACT_REPLAY;
    TTT_TRY(key_pass(t0, C, nt, reads ? nt : 0));
    TTT_TRY(fork());
    if (reads) TTT_TRY(read_out(t0, C, rstream, Aq));
    const int splits = gradients(t0, C, gstream, false);
    if (splits < 0) return -1;
    TTT_TRY(join());
    if (fused_update) {   // the epilogues wrote buffer nxt(cur)
      cur = nxt(cur);
      continue;
    }
    ra.splits = splits;
    set_out_buf(nxt(cur));
    TTT_TRY(replay_save(ci));
    if (L.opt == 2) {
      TTT_TRY(muon());
    } else {
      TTT_TRY(row_update(stream));
    }
    cur = nxt(cur);
  }
  if (L.mode == LACT_REPLAY && L.wsave != nullptr && !looped)   // the weights after the last chunk
    TTT_TRY(cudaMemcpyAsync(L.wsave + (size_t)ci * 3 * mat_elems, L.state, 3 * mat_elems * sizeof(float),
                            cudaMemcpyDeviceToDevice, stream) == cudaSuccess ? 0 : -1);
  if (!L.causal && L.N_q > 0 && L.mode != LACT_REPLAY) {
    if (d == 128 && !split) {   // the fused read: Q -> out in one kernel
      ReadFusedLaunch rl{};
      rl.BH = BH; rl.rows = L.N_q; rl.t0 = 0; rl.C = L.N_q; rl.dh = dh; rl.out_bf16 = L.out_bf16;
      rl.max_grid = num_sms();
      rl.q = L.q; rl.w1b = wbuf[cur][0]; rl.w3b = wbuf[cur][1]; rl.w2b = wbuf[cur][2];
      rl.out = L.out; rl.st = L.st;
      TTT_TRY(launch_lact_read_fused(rl, stream));
    } else {
      TTT_TRY(key_pass(0, L.N_q, 0, (L.N_q + 127) / 128));
      TTT_TRY(read_out(0, L.N_q, stream, Aq));
    }
  }
  return 0;
}

}  // namespace ttt
