// window_attention.cu -- causal sliding-window softmax attention, the local
// branch of the LaCT language layer ("Test-Time Training Done Right" review,
// "Memoria no lineal y atención local" and "El orden de lectura evita
// información futura": windowed attention and the fast-weight memory share
// Q, K and V and their outputs are summed; the causal sliding window keeps
// future tokens out).
//
// o_i = sum over j in (i - W, i] of softmax_j(scale q_i . k_j) v_j, head dim
// 128, bf16 q, k, v, fp32 accumulation.
//
// One CTA per (head, 128-query tile) walks the window's 128-key tiles twice:
//   pass 1   S = Q K^T (tcgen05, TMEM)  -> row max m and row sum l (online)
//   pass 2   S = Q K^T again            -> P = exp(S - m) / l, bf16 in smem
//            O += P V (tcgen05, TMEM)
// so O accumulates already-normalised terms and is never rescaled.  Each
// query row is shared by four epilogue threads (32 key columns each), whose
// partial row statistics are combined through shared memory between the
// passes.  S
// alternates between two TMEM buffers and P between two shared buffers, so
// the tensor cores work on one key tile while the epilogue warps work on the
// previous one.  K and V tiles sit in separate two-slot rings, so a K slot
// is refilled as soon as its scores are computed, while the V slot waits for
// its P V product (pass 1 loads K only).
#include <algorithm>

#include "kernels.h"

namespace ttt {
namespace swa {
constexpr int D = 128, BM = 128, BN = 128;
constexpr uint32_t HALF = 128 * 64 * 2;          // 16 KB: 128 rows x 64 bf16 (one swizzle atom wide)
constexpr uint32_t TILE = 2 * HALF;              // 32 KB: 128 rows x 128 bf16
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = TILE;                 // 2 K slots
constexpr uint32_t OFF_V = OFF_K + 2 * TILE;     // 2 V slots (pass 2)
constexpr uint32_t OFF_P = OFF_V + 2 * TILE;     // 2 x P (128 queries x 128 keys)
constexpr uint32_t OFF_BAR = OFF_P + 2 * TILE;
constexpr uint32_t SMEM = OFF_BAR + 256 + 1024;
// four per TMEM lane quadrant: a thread takes 32 key columns of one query row
constexpr int EPI_WARPS = 16;
constexpr int THREADS = (2 + EPI_WARPS) * 32;
constexpr int CW = 32;                            // columns per epilogue thread
constexpr uint32_t TM_S0 = 0, TM_S1 = 128, TM_O = 256, TM_COLS = 512;
}  // namespace swa

struct SwaArgs {
  int N, window, n_qt;
  float scale_log2;     // scale * log2(e): scores go through exp2
  int out_bf16, accumulate;
  void* out;            // [BH][N][128]
  DevStatus st;
};
struct SwaMaps {
  CUtensorMap q, k, v;
};

__global__ void __launch_bounds__(swa::THREADS, 1)
    window_attention_kernel(const __grid_constant__ SwaMaps maps, const SwaArgs a) {
  using namespace swa;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* q_full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* k_full = q_full + 1;      // [2]
  uint64_t* k_empty = k_full + 2;     // [2]
  uint64_t* v_full = k_empty + 2;     // [2]
  uint64_t* v_empty = v_full + 2;     // [2]
  uint64_t* s_full = v_empty + 2;     // [2]
  uint64_t* s_empty = s_full + 2;     // [2]
  uint64_t* p_full = s_empty + 2;     // [2]
  uint64_t* p_empty = p_full + 2;     // [2]
  uint64_t* o_full = p_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_full + 1);
  uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the tiles with the most keys (late in the sequence) first
  const int bh = blockIdx.x / a.n_qt;
  const int qt = a.n_qt - 1 - (int)(blockIdx.x % a.n_qt);
  const int q0 = qt * BM;
  const int kt_lo = max(0, q0 - a.window + 1) / BN;   // first key tile of the window
  const int nk = qt - kt_lo + 1;                            // key tiles per pass
  const int G = 2 * nk;                                     // pass 1, then pass 2

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&s_empty[s], EPI_WARPS * 32);
      mbar_init(&p_full[s], EPI_WARPS * 32);
      mbar_init(&p_empty[s], 1);
    }
    mbar_init(o_full, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&maps.q);
    tma_prefetch_desc(&maps.k);
    tma_prefetch_desc(&maps.v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  Waiter W{abort_flag, a.st, 400};

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, TILE);
      tma_load_3d(smem + OFF_Q, &maps.q, q_full, 0, q0, bh);
      tma_load_3d(smem + OFF_Q + HALF, &maps.q, q_full, 64, q0, bh);
      int k_issued = 0, v_issued = 0;
      for (int g = 0; g < G; ++g) {
        // K of tile g into slot g & 1, free once the scores of tile g - 2 are done
        const int s = g & 1;
        if (g >= 2 && !W.wait(&k_empty[s], ((g >> 1) - 1) & 1, 1)) break;
        const bool pass2 = g >= nk;
        const int i = g - nk;
        const int row = (kt_lo + (pass2 ? i : g)) * BN;
        mbar_arrive_expect_tx(&k_full[s], TILE);
        tma_load_3d(smem + OFF_K + s * TILE, &maps.k, &k_full[s], 0, row, bh);
        tma_load_3d(smem + OFF_K + s * TILE + HALF, &maps.k, &k_full[s], 64, row, bh);
        k_issued = g + 1;
        if (pass2) {
          // V of pass-2 tile i into slot i & 1, free once P V of tile i - 2 is done
          const int sv = i & 1;
          if (i >= 2 && !W.wait(&v_empty[sv], ((i >> 1) - 1) & 1, 9)) break;
          mbar_arrive_expect_tx(&v_full[sv], TILE);
          tma_load_3d(smem + OFF_V + sv * TILE, &maps.v, &v_full[sv], 0, row, bh);
          tma_load_3d(smem + OFF_V + sv * TILE + HALF, &maps.v, &v_full[sv], 64, row, bh);
          v_issued = i + 1;
        }
      }
      if (W.aborted()) {
        W.drain(q_full, 0);
        for (int g = max(0, k_issued - 2); g < k_issued; ++g) W.drain(&k_full[g & 1], (g >> 1) & 1);
        for (int i = max(0, v_issued - 2); i < v_issued; ++i) W.drain(&v_full[i & 1], (i >> 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t id_s = make_idesc(128, 128, false, false);   // Q, K both K-major (d)
      const uint32_t id_o = make_idesc(128, 128, false, true);    // P K-major (keys), V MN-major
      const uint64_t dq = make_sdesc(smem_u32(smem + OFF_Q), 16, 1024);
      const uint64_t dk0 = make_sdesc(smem_u32(smem + OFF_K), 16, 1024);
      const uint64_t dv0 = make_sdesc(smem_u32(smem + OFF_V), HALF, 1024);
      const uint64_t dp0 = make_sdesc(smem_u32(smem + OFF_P), 16, 1024);
      bool ok = W.wait(q_full, 0, 2);
      tc_fence_after();
      // S(g) = Q K(g)^T into S buffer g & 1
      auto issue_s = [&](int g) -> bool {
        const int s = g & 1;
        if (!W.wait(&k_full[s], (g >> 1) & 1, 3)) return false;
        if (g >= 2 && !W.wait(&s_empty[s], ((g >> 1) - 1) & 1, 4)) return false;
        tc_fence_after();
        const uint64_t dk = sdesc_add(dk0, s * TILE);
        const uint32_t acc = tmem + (s ? TM_S1 : TM_S0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * HALF + (kk & 3) * 32;
          mma_bf16(acc, sdesc_add(dq, off), sdesc_add(dk, off), id_s, kk > 0);
        }
        mma_commit(&s_full[s]);
        mma_commit(&k_empty[s]);   // the scores are done with this K tile
        return true;
      };
      if (ok && G > 0) ok = issue_s(0);
      for (int g = 0; ok && g < G; ++g) {
        // the next tile's scores first, so they run while the epilogue
        // turns this tile's scores into P
        if (g + 1 < G && !issue_s(g + 1)) { ok = false; break; }
        if (g >= nk) {
          // pass-2 tile i: P buffer i & 1, filled for the (i >> 1)-th time
          const int i = g - nk, pb = i & 1, sv = i & 1;
          if (!W.wait(&p_full[pb], (i >> 1) & 1, 5)) { ok = false; break; }
          if (!W.wait(&v_full[sv], (i >> 1) & 1, 10)) { ok = false; break; }
          tc_fence_after();
          const uint64_t dv = sdesc_add(dv0, sv * TILE);
          const uint64_t dp = sdesc_add(dp0, pb * TILE);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t offp = (kk >> 2) * HALF + (kk & 3) * 32;
            mma_bf16(tmem + TM_O, sdesc_add(dp, offp), sdesc_add(dv, kk * 2048), id_o,
                     (i > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&v_empty[sv]);
          mma_commit(&p_empty[pb]);
        }
      }
      mma_commit(o_full);
      W.drain(o_full, 0);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q4 = warp & 3;
    const int cg = (warp - 2) >> 2;             // 32-column group of the key tile
    const int c0 = cg * CW;
    const int r = q4 * 32 + lane;               // query row of the tile
    const int qi = q0 + r;                      // query token
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    const bool row_ok = qi < a.N;
    float m = -INFINITY, l = 0.f;               // running max (log2 units) and sum of this slice
    bool ok = true;
    // key tile kt lies inside every row's window (no mask needed): uniform
    // across the CTA, so the branches below never split a warp
    auto inside = [&](int kt) {
      return kt * BN + BN - 1 <= q0 && kt * BN > q0 + BM - 1 - a.window && q0 + BM <= a.N;
    };
    // ---- pass 1: statistics of this thread's 32 columns
    for (int g = 0; ok && g < nk; ++g) {
      const int kt = kt_lo + g, sb = g & 1;
      if (!W.wait(&s_full[sb], (g >> 1) & 1, 6)) { ok = false; break; }
      tc_fence_after();
      float x[CW];
      // tcgen05.ld is warp-collective: every lane reaches it, converged
      __syncwarp();
      tmem_ld32(tmem + lane_base + (sb ? TM_S1 : TM_S0) + c0, x);
      tc_fence_before();
      mbar_arrive(&s_empty[sb]);
      float cm = -INFINITY;
      if (inside(kt)) {
#pragma unroll
        for (int j = 0; j < CW; ++j) {
          x[j] *= a.scale_log2;
          cm = fmaxf(cm, x[j]);
        }
      } else {
#pragma unroll
        for (int j = 0; j < CW; ++j) {
          const int kj = kt * BN + c0 + j;
          const bool valid = row_ok && kj <= qi && kj > qi - a.window;
          x[j] = valid ? x[j] * a.scale_log2 : -INFINITY;
          cm = fmaxf(cm, x[j]);
        }
      }
      const float mn = fmaxf(m, cm);
      if (mn != -INFINITY) {   // no valid key yet: m and l stay as they are
        float add = 0.f;
#pragma unroll
        for (int j = 0; j < CW; ++j) add += exp2f(x[j] - mn);
        l = l * exp2f(m - mn) + add;
        m = mn;
      }
    }
    // ---- the row's statistics from its four slices.  Every epilogue thread
    // passes both barriers exactly once (also after a failed wait), so no
    // thread is left waiting.  The scratch is P buffer 1, first written by
    // pass-2 tile 1, after the second barrier.
    float2* stats = reinterpret_cast<float2*>(smem + OFF_P + TILE);   // [4 slices][128 rows]
    stats[cg * BM + r] = make_float2(m, l);
    asm volatile("bar.sync 1, %0;" ::"n"(EPI_WARPS * 32) : "memory");
    {
      float M = -INFINITY;
#pragma unroll
      for (int u = 0; u < 4; ++u) M = fmaxf(M, stats[u * BM + r].x);
      float L = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float2 t = stats[u * BM + r];
          if (t.x != -INFINITY) L += t.y * exp2f(t.x - M);
        }
      }
      m = M;
      l = L;
    }
    asm volatile("bar.sync 1, %0;" ::"n"(EPI_WARPS * 32) : "memory");
    // ---- pass 2: P = exp(S - m) / l for this thread's 32 columns
    const float inv_l = row_ok ? 1.f / l : 0.f;
    for (int i = 0; ok && i < nk; ++i) {
      const int g = nk + i, kt = kt_lo + i, sb = g & 1, pb = i & 1;
      if (!W.wait(&s_full[sb], (g >> 1) & 1, 6)) { ok = false; break; }
      // P buffer i & 1 is free once the P V product of pass-2 tile i - 2 is done
      if (i >= 2 && !W.wait(&p_empty[pb], ((i >> 1) - 1) & 1, 7)) { ok = false; break; }
      tc_fence_after();
      float x[CW];
      __syncwarp();
      tmem_ld32(tmem + lane_base + (sb ? TM_S1 : TM_S0) + c0, x);
      tc_fence_before();
      mbar_arrive(&s_empty[sb]);
      uint32_t pk[CW / 2];
      if (inside(kt)) {
#pragma unroll
        for (int j = 0; j < CW; j += 2)
          pk[j >> 1] = pack_bf16x2(exp2f(x[j] * a.scale_log2 - m) * inv_l,
                                   exp2f(x[j + 1] * a.scale_log2 - m) * inv_l);
      } else {
#pragma unroll
        for (int j = 0; j < CW; j += 2) {
          float p2[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int kj = kt * BN + c0 + j + u;
            const bool valid = row_ok && kj <= qi && kj > qi - a.window;
            p2[u] = valid ? exp2f(x[j + u] * a.scale_log2 - m) * inv_l : 0.f;
          }
          pk[j >> 1] = pack_bf16x2(p2[0], p2[1]);
        }
      }
      // keys c0 .. c0 + 31 of row r: half c0 / 64, columns (c0 % 64) ..
      const uint32_t hb = smem_u32(smem + OFF_P + pb * TILE) + (uint32_t)(c0 >> 6) * HALF;
#pragma unroll
      for (int j = 0; j < CW; j += 8)
        st_shared_v4(hb + sw128_offset(r, (c0 & 63) + j), pk[j / 2], pk[j / 2 + 1], pk[j / 2 + 2],
                     pk[j / 2 + 3]);
      fence_async_smem();
      mbar_arrive(&p_full[pb]);
    }
    if (ok && W.wait(o_full, 0, 8)) {
      tc_fence_after();
      float o[CW];
      // every lane loads (warp-collective); only rows inside the sequence store
      __syncwarp();
      tmem_ld32(tmem + lane_base + TM_O + c0, o);
      if (row_ok) {
        const size_t base = ((size_t)bh * a.N + qi) * D + c0;
        if (a.out_bf16) {
          uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) + base);
#pragma unroll
          for (int j = 0; j < CW / 8; ++j) {
            float v8[8];
            if (a.accumulate) {
              const uint4 w = dst[j];
              const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                v8[2 * u] = o[8 * j + 2 * u] + bf16lo(ww[u]);
                v8[2 * u + 1] = o[8 * j + 2 * u + 1] + bf16hi(ww[u]);
              }
            } else {
#pragma unroll
              for (int u = 0; u < 8; ++u) v8[u] = o[8 * j + u];
            }
            dst[j] = make_uint4(pack_bf16x2(v8[0], v8[1]), pack_bf16x2(v8[2], v8[3]),
                                pack_bf16x2(v8[4], v8[5]), pack_bf16x2(v8[6], v8[7]));
          }
        } else {
          float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + base);
#pragma unroll
          for (int j = 0; j < CW / 4; ++j) {
            float4 v4 = make_float4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
            if (a.accumulate) {
              const float4 w = dst[j];
              v4.x += w.x; v4.y += w.y; v4.z += w.z; v4.w += w.w;
            }
            dst[j] = v4;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Single pass with an online softmax.  One thread per query row holds the
// row's 128 scores of a key tile; the row keeps a running maximum m (log2
// units) and sum l, and P = exp2(s - m) goes straight into the P V product.
// When a tile raises a row's maximum by more than 8 (a factor 256), the row
// of O accumulated so far in TMEM is rescaled by exp2(m_old - m_new) before
// that tile's P V product; smaller rises keep the old m (P stays below 256).
// O is divided by l once, at the end.  Each key tile costs one Q K^T and one
// P V product and one exponential per score.
// ---------------------------------------------------------------------------
// (x0, x1) -> (2^(s x0 + b), 2^(s x1 + b)): one packed two-lane fp32 FMA
// (sm_100 f32x2, each lane rounded like the scalar instruction) and the
// hardware base-2 exponential per lane (ex2.approx, a few ulp; the result
// is rounded to bf16 next).  2^-inf = 0 for masked columns.
TTT_DEVICE_INLINE float2 exp2_scaled_x2(float x0, float x1, float sc, float b) {
  float2 r;
  asm("{\n\t.reg .b64 X, S, B, T;\n\t.reg .f32 t0, t1;\n\t"
      "mov.b64 X, {%2, %3};\n\t"
      "mov.b64 S, {%4, %4};\n\t"
      "mov.b64 B, {%5, %5};\n\t"
      "fma.rn.f32x2 T, X, S, B;\n\t"
      "mov.b64 {t0, t1}, T;\n\t"
      "ex2.approx.ftz.f32 %0, t0;\n\t"
      "ex2.approx.ftz.f32 %1, t1;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(x0), "f"(x1), "f"(sc), "f"(b));
  return r;
}
TTT_DEVICE_INLINE float2 add_x2(float2 a, float2 b) {
  float2 r;
  asm("{\n\t.reg .b64 A, B, R;\n\t"
      "mov.b64 A, {%2, %3};\n\t"
      "mov.b64 B, {%4, %5};\n\t"
      "add.rn.f32x2 R, A, B;\n\t"
      "mov.b64 {%0, %1}, R;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}

namespace swa1 {
constexpr int D = 128, BM = 128, BN = 128;
constexpr uint32_t HALF = 128 * 64 * 2;
constexpr uint32_t TILE = 2 * HALF;
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = TILE;                 // 2 K slots
constexpr uint32_t OFF_V = OFF_K + 2 * TILE;     // 2 V slots
constexpr uint32_t OFF_P = OFF_V + 2 * TILE;     // 2 P buffers
constexpr uint32_t OFF_BAR = OFF_P + 2 * TILE;
constexpr uint32_t SMEM = OFF_BAR + 256 + 1024;
constexpr int EPI_WARPS = 4;                      // one per TMEM lane quadrant: a thread per row
constexpr int THREADS = (2 + EPI_WARPS) * 32;
constexpr float RESCALE = 8.f;                    // lazy rescale threshold (log2 units)
constexpr uint32_t TM_S0 = 0, TM_S1 = 128, TM_O = 256, TM_COLS = 512;
}  // namespace swa1

__global__ void __launch_bounds__(swa1::THREADS, 1)
    window_attention_1p_kernel(const __grid_constant__ SwaMaps maps, const SwaArgs a) {
  using namespace swa1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* q_full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* k_full = q_full + 1;      // [2]
  uint64_t* k_empty = k_full + 2;     // [2]
  uint64_t* v_full = k_empty + 2;     // [2]
  uint64_t* v_empty = v_full + 2;     // [2]
  uint64_t* s_full = v_empty + 2;     // [2]
  uint64_t* s_empty = s_full + 2;     // [2]
  uint64_t* p_full = s_empty + 2;     // [2]
  uint64_t* p_empty = p_full + 2;     // [2]
  uint64_t* o_done = p_empty + 2;     // one phase per P V product
  uint64_t* fin = o_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x / a.n_qt;
  const int qt = a.n_qt - 1 - (int)(blockIdx.x % a.n_qt);   // the longest windows first
  const int q0 = qt * BM;
  const int kt_lo = max(0, q0 - a.window + 1) / BN;
  const int nk = qt - kt_lo + 1;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&s_empty[s], EPI_WARPS * 32);
      mbar_init(&p_full[s], EPI_WARPS * 32);
      mbar_init(&p_empty[s], 1);
    }
    mbar_init(o_done, 1);
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&maps.q);
    tma_prefetch_desc(&maps.k);
    tma_prefetch_desc(&maps.v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  Waiter W{abort_flag, a.st, 450};

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, TILE);
      tma_load_3d(smem + OFF_Q, &maps.q, q_full, 0, q0, bh);
      tma_load_3d(smem + OFF_Q + HALF, &maps.q, q_full, 64, q0, bh);
      int k_issued = 0, v_issued = 0;
      for (int g = 0; g < nk; ++g) {
        const int s = g & 1, row = (kt_lo + g) * BN;
        // K slot free once the scores of tile g - 2 are done
        if (g >= 2 && !W.wait(&k_empty[s], ((g >> 1) - 1) & 1, 1)) break;
        mbar_arrive_expect_tx(&k_full[s], TILE);
        tma_load_3d(smem + OFF_K + s * TILE, &maps.k, &k_full[s], 0, row, bh);
        tma_load_3d(smem + OFF_K + s * TILE + HALF, &maps.k, &k_full[s], 64, row, bh);
        k_issued = g + 1;
        // V slot free once the P V product of tile g - 2 is done
        if (g >= 2 && !W.wait(&v_empty[s], ((g >> 1) - 1) & 1, 2)) break;
        mbar_arrive_expect_tx(&v_full[s], TILE);
        tma_load_3d(smem + OFF_V + s * TILE, &maps.v, &v_full[s], 0, row, bh);
        tma_load_3d(smem + OFF_V + s * TILE + HALF, &maps.v, &v_full[s], 64, row, bh);
        v_issued = g + 1;
      }
      if (W.aborted()) {
        W.drain(q_full, 0);
        for (int g = max(0, k_issued - 2); g < k_issued; ++g) W.drain(&k_full[g & 1], (g >> 1) & 1);
        for (int g = max(0, v_issued - 2); g < v_issued; ++g) W.drain(&v_full[g & 1], (g >> 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t id_s = make_idesc(128, 128, false, false);
      const uint32_t id_o = make_idesc(128, 128, false, true);
      const uint64_t dq = make_sdesc(smem_u32(smem + OFF_Q), 16, 1024);
      const uint64_t dk0 = make_sdesc(smem_u32(smem + OFF_K), 16, 1024);
      const uint64_t dv0 = make_sdesc(smem_u32(smem + OFF_V), HALF, 1024);
      const uint64_t dp0 = make_sdesc(smem_u32(smem + OFF_P), 16, 1024);
      bool ok = W.wait(q_full, 0, 3);
      tc_fence_after();
      auto issue_s = [&](int g) -> bool {
        const int s = g & 1;
        if (!W.wait(&k_full[s], (g >> 1) & 1, 4)) return false;
        if (g >= 2 && !W.wait(&s_empty[s], ((g >> 1) - 1) & 1, 5)) return false;
        tc_fence_after();
        const uint64_t dk = sdesc_add(dk0, s * TILE);
        const uint32_t acc = tmem + (s ? TM_S1 : TM_S0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * HALF + (kk & 3) * 32;
          mma_bf16(acc, sdesc_add(dq, off), sdesc_add(dk, off), id_s, kk > 0);
        }
        mma_commit(&s_full[s]);
        mma_commit(&k_empty[s]);
        return true;
      };
      if (ok && nk > 0) ok = issue_s(0);
      for (int g = 0; ok && g < nk; ++g) {
        // the next tile's scores run while the softmax warps work on this one
        if (g + 1 < nk && !issue_s(g + 1)) { ok = false; break; }
        const int s = g & 1;
        if (!W.wait(&p_full[s], (g >> 1) & 1, 6)) { ok = false; break; }
        if (!W.wait(&v_full[s], (g >> 1) & 1, 7)) { ok = false; break; }
        tc_fence_after();
        const uint64_t dv = sdesc_add(dv0, s * TILE);
        const uint64_t dp = sdesc_add(dp0, s * TILE);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t offp = (kk >> 2) * HALF + (kk & 3) * 32;
          mma_bf16(tmem + TM_O, sdesc_add(dp, offp), sdesc_add(dv, kk * 2048), id_o,
                   (g > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&v_empty[s]);
        mma_commit(&p_empty[s]);
        mma_commit(o_done);
      }
      mma_commit(fin);
      W.drain(fin, 0);
    }
  } else {
    // ---------------------------------------------------------------- softmax
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;                // query row of the tile
    const int qi = q0 + r;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    const bool row_ok = qi < a.N;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    auto inside = [&](int kt) {
      return kt * BN + BN - 1 <= q0 && kt * BN > q0 + BM - 1 - a.window && q0 + BM <= a.N;
    };
    for (int g = 0; ok && g < nk; ++g) {
      const int kt = kt_lo + g, s = g & 1;
      if (!W.wait(&s_full[s], (g >> 1) & 1, 8)) { ok = false; break; }
      tc_fence_after();
      float x[BN];
      {
        uint32_t xr[BN];
        __syncwarp();   // tcgen05.ld is warp-collective: every lane, converged
        // all eight loads in flight before one wait
#pragma unroll
        for (int c = 0; c < BN; c += 16) tmem_ld16_issue(tmem + lane_base + (s ? TM_S1 : TM_S0) + c, xr + c);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < BN; ++j) x[j] = __uint_as_float(xr[j]);
      }
      tc_fence_before();
      mbar_arrive(&s_empty[s]);
      // the row maximum on the raw scores (the scale is positive), masked
      // keys set to -inf
      float mx = -INFINITY;
      if (inside(kt)) {
#pragma unroll
        for (int j = 0; j < BN; ++j) mx = fmaxf(mx, x[j]);
      } else {
#pragma unroll
        for (int j = 0; j < BN; ++j) {
          const int kj = kt * BN + j;
          const bool valid = row_ok && kj <= qi && kj > qi - a.window;
          x[j] = valid ? x[j] : -INFINITY;
          mx = fmaxf(mx, x[j]);
        }
      }
      mx *= a.scale_log2;
      // lazy rescale: keep m unless the tile raises it by more than RESCALE
      float alpha = 1.f;
      if (mx > m + RESCALE || (m == -INFINITY && mx != -INFINITY)) {
        alpha = m == -INFINITY ? 0.f : exp2f(m - mx);
        m = mx;
      }
      // the rows of O a warp rescales: P V of tile g - 1 must be done first;
      // every lane of the warp takes part in the TMEM load and store
      const bool any = __any_sync(0xffffffffu, alpha != 1.f) && g > 0;
      if (any) {
        if (!W.wait(o_done, (g - 1) & 1, 9)) { ok = false; }
        __syncwarp();
        if (ok) {
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < D; c += 32) {
            float o[32];
            tmem_ld32(tmem + lane_base + TM_O + c, o);
#pragma unroll
            for (int j = 0; j < 32; j += 16) {
              float t16[16];
#pragma unroll
              for (int u = 0; u < 16; ++u) t16[u] = o[j + u] * alpha;
              tmem_st16(tmem + lane_base + TM_O + c + j, t16);
            }
          }
          tc_fence_before();
        }
      }
      if (!ok) break;
      l *= alpha;
      // P = exp2(s - m) (zero where masked or before any valid key)
      uint32_t pk[BN / 2];
      float add = 0.f;
      if (m == -INFINITY) {
#pragma unroll
        for (int j = 0; j < BN / 2; ++j) pk[j] = 0u;
      } else {
        // two columns per packed fp32 instruction: t = scale x - m, then
        // the hardware base-2 exponential of each lane
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < BN; j += 2) {
          const float2 p = exp2_scaled_x2(x[j], x[j + 1], a.scale_log2, -m);
          acc = add_x2(acc, p);
          pk[j >> 1] = pack_bf16x2(p.x, p.y);
        }
        add = acc.x + acc.y;
      }
      l += add;
      // P buffer s is free once the P V product of tile g - 2 is done (its own
      // barrier: o_done may already be a phase further on)
      if (g >= 2 && !W.wait(&p_empty[s], ((g >> 1) - 1) & 1, 10)) { ok = false; break; }
      const uint32_t pb = smem_u32(smem + OFF_P + s * TILE);
#pragma unroll
      for (int j = 0; j < BN; j += 8)
        st_shared_v4(pb + (uint32_t)(j >> 6) * HALF + sw128_offset(r, j & 63), pk[j / 2],
                     pk[j / 2 + 1], pk[j / 2 + 2], pk[j / 2 + 3]);
      fence_async_smem();
      mbar_arrive(&p_full[s]);
    }
    if (ok && nk > 0 && W.wait(o_done, (nk - 1) & 1, 11)) {
      tc_fence_after();
      const float inv_l = (row_ok && l > 0.f) ? 1.f / l : 0.f;
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        float o[32];
        __syncwarp();
        tmem_ld32(tmem + lane_base + TM_O + c, o);   // every lane (warp-collective)
        if (!row_ok) continue;
        const size_t base = ((size_t)bh * a.N + qi) * D + c;
        if (a.out_bf16) {
          uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) + base);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float v8[8];
            if (a.accumulate) {
              const uint4 w = dst[j];
              const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                v8[2 * u] = o[8 * j + 2 * u] * inv_l + bf16lo(ww[u]);
                v8[2 * u + 1] = o[8 * j + 2 * u + 1] * inv_l + bf16hi(ww[u]);
              }
            } else {
#pragma unroll
              for (int u = 0; u < 8; ++u) v8[u] = o[8 * j + u] * inv_l;
            }
            dst[j] = make_uint4(pack_bf16x2(v8[0], v8[1]), pack_bf16x2(v8[2], v8[3]),
                                pack_bf16x2(v8[4], v8[5]), pack_bf16x2(v8[6], v8[7]));
          }
        } else {
          float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + base);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            float4 v4 = make_float4(o[4 * j] * inv_l, o[4 * j + 1] * inv_l, o[4 * j + 2] * inv_l,
                                    o[4 * j + 3] * inv_l);
            if (a.accumulate) {
              const float4 w = dst[j];
              v4.x += w.x; v4.y += w.y; v4.z += w.z; v4.w += w.w;
            }
            dst[j] = v4;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TM_COLS);
  }
}

// The single-pass kernel is the default; the two-pass kernel is kept as the
// reference design it replaced.
constexpr bool kSinglePass = true;

int launch_window_attention(const WindowAttnLaunch& L, cudaStream_t stream) {
  using namespace swa;
  const uint64_t BH = (uint64_t)L.B * L.H;
  if (L.N == 0) return 0;
  SwaMaps m;
  const uint64_t row = D * 2;
  if (make_tmap_bf16_3d(&m.q, L.q, D, L.N, BH, row, row * L.N, 64, 128) ||
      make_tmap_bf16_3d(&m.k, L.k, D, L.N, BH, row, row * L.N, 64, 128) ||
      make_tmap_bf16_3d(&m.v, L.v, D, L.N, BH, row, row * L.N, 64, 128))
    return -1;
  SwaArgs a{};
  a.N = L.N;
  a.window = L.window;
  a.n_qt = (L.N + BM - 1) / BM;
  a.scale_log2 = L.scale * 1.4426950408889634f;
  a.out_bf16 = L.out_bf16;
  a.accumulate = L.accumulate;
  a.out = L.out;
  a.st = L.st;
  prof_before(K_SWA, stream);
  if (kSinglePass) {
    static std::atomic<uint64_t> attr1{0};
    if (allow_dynamic_smem(window_attention_1p_kernel, (int)swa1::SMEM, attr1)) return -1;
    window_attention_1p_kernel<<<dim3((unsigned)(BH * a.n_qt)), dim3(swa1::THREADS), swa1::SMEM,
                                 stream>>>(m, a);
  } else {
    static std::atomic<uint64_t> attr{0};
    if (allow_dynamic_smem(window_attention_kernel, (int)SMEM, attr)) return -1;
    window_attention_kernel<<<dim3((unsigned)(BH * a.n_qt)), dim3(THREADS), SMEM, stream>>>(m, a);
  }
  prof_after(K_SWA, stream);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace ttt
