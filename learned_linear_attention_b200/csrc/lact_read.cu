// lact_read.cu -- the LaCT memory read as one fused kernel for head dim 128
// ("Test-Time Training Done Right" review, "Memoria no lineal y atención
// local" and "El orden de lectura evita información futura": a query reads
// the SwiGLU memory, o = W2 (silu(W1 q) * (W3 q)), with the weights left by
// the earlier chunks).
//
// One work item = (head, 128-query tile).  The Q tile stays in shared
// memory; the hidden units are walked in blocks J of 64:
//   MMA   H13_J = Q [W1_J; W3_J]^T              (128 x 128, TMEM, two buffers)
//   epi   Aq_J = silu(H1_J) * H3_J              -> bf16 in shared memory
//   MMA   O += Aq_J W2[:, J]^T                  (128 x 128, TMEM)
// with the weight blocks streamed through a three-stage ring (the next
// item's first blocks load while this item finishes), so the product of
// block J runs while the epilogue forms Aq of block J - 1.  At the end of the
// item the epilogue stores O.  Nothing between Q and O goes to global memory.
#include <algorithm>

#include "kernels.h"

namespace ttt {
namespace rd {
constexpr int D = 128, HB = 64, BM = 128;
constexpr uint32_t HALF = BM * 64 * 2;                 // 16 KB: 128 rows x 64 bf16
constexpr uint32_t OFF_Q = 0;                          // Q tile: two K atoms (32 KB)
constexpr uint32_t W_STAGE = 3 * HALF;                 // [W1_J; W3_J] 32 KB + W2[:, J] 16 KB
constexpr int WS = 3;                                  // weight stages
constexpr uint32_t OFF_W = 2 * HALF;
constexpr uint32_t OFF_AQ = OFF_W + WS * W_STAGE;      // two Aq_J buffers (16 KB each)
constexpr uint32_t OFF_BAR = OFF_AQ + 2 * HALF;
constexpr uint32_t SMEM = OFF_BAR + 256 + 1024;
constexpr int EPI_WARPS = 8;                           // two per TMEM lane quadrant
constexpr int THREADS = (2 + EPI_WARPS) * 32;
constexpr int CW = HB / (EPI_WARPS / 4);               // hidden columns per epilogue thread (32)
constexpr uint32_t TM_H0 = 0, TM_H1 = 128, TM_O = 256, TM_COLS = 512;
}  // namespace rd

struct ReadFusedArgs {
  int BH, rows, t0, C;   // q / out rows per head; the tiles cover rows [t0, t0 + C)
  int n_hb;              // dh / 64
  int n_tiles;           // query tiles per head
  int out_bf16;
  void* out;             // [BH][rows][128]
  DevStatus st;
};
struct ReadFusedMaps {
  CUtensorMap q, w1, w3, w2;
};

TTT_DEVICE_INLINE float rd_sigmoid(float x) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
  return fmaf(0.5f, t, 0.5f);
}

__global__ void __launch_bounds__(rd::THREADS, 1)
    lact_read_fused_kernel(const __grid_constant__ ReadFusedMaps maps, const ReadFusedArgs a) {
  using namespace rd;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* q_full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* q_empty = q_full + 1;
  uint64_t* w_full = q_empty + 1;     // [WS]
  uint64_t* w_empty = w_full + WS;    // [WS]
  uint64_t* h_full = w_empty + WS;    // [2]
  uint64_t* h_empty = h_full + 2;     // [2]
  uint64_t* aq_full = h_empty + 2;    // [2]
  uint64_t* aq_empty = aq_full + 2;   // [2]
  uint64_t* o_full = aq_empty + 2;
  uint64_t* o_empty = o_full + 1;
  uint64_t* fin = o_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = a.BH * a.n_tiles;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < WS; ++s) {
      mbar_init(&w_full[s], 1);
      mbar_init(&w_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&h_full[s], 1);
      mbar_init(&h_empty[s], EPI_WARPS * 32);
      mbar_init(&aq_full[s], EPI_WARPS * 32);
      mbar_init(&aq_empty[s], 1);
    }
    mbar_init(o_full, 1);
    mbar_init(o_empty, EPI_WARPS * 32);
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
    tma_prefetch_desc(&maps.w1);
    tma_prefetch_desc(&maps.w3);
    tma_prefetch_desc(&maps.w2);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  const uint32_t tmem = *tmem_slot;
  Waiter W{abort_flag, a.st, 800};

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      uint32_t gj = 0, it = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x, ++it) {
        const int bh = item / a.n_tiles, qt = item % a.n_tiles;
        // the Q tile is free once every H13 product of the previous item is done
        if (it >= 1 && !W.wait(q_empty, (it - 1) & 1, 1)) { ok = false; break; }
        mbar_arrive_expect_tx(q_full, 2 * HALF);
        const int row = a.t0 + qt * BM;
        tma_load_3d(smem + OFF_Q, &maps.q, q_full, 0, row, bh);
        tma_load_3d(smem + OFF_Q + HALF, &maps.q, q_full, 64, row, bh);
        for (int j = 0; j < a.n_hb; ++j, ++gj) {
          const uint32_t s = gj % WS;
          if (gj >= (uint32_t)WS && !W.wait(&w_empty[s], ((gj / WS) - 1) & 1, 2)) { ok = false; break; }
          uint8_t* st = smem + OFF_W + s * W_STAGE;
          mbar_arrive_expect_tx(&w_full[s], W_STAGE);
          for (int atom = 0; atom < 2; ++atom) {
            tma_load_3d(st + atom * HALF, &maps.w1, &w_full[s], atom * 64, j * HB, bh);
            tma_load_3d(st + atom * HALF + HALF / 2, &maps.w3, &w_full[s], atom * 64, j * HB, bh);
          }
          // W2[:, J] as a K-major B operand: 128 d-rows of 64 hidden units
          tma_load_3d(st + 2 * HALF, &maps.w2, &w_full[s], j * HB, 0, bh);
        }
      }
      if (W.aborted()) {
        W.drain(q_full, it & 1);
        const uint32_t first = gj > (uint32_t)WS ? gj - WS : 0;
        for (uint32_t i = first; i < gj; ++i) W.drain(&w_full[i % WS], (i / WS) & 1);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t id_h = make_idesc(128, 128, false, false);
      const uint32_t id_o = make_idesc(128, 128, false, false);
      const uint64_t dq = make_sdesc(smem_u32(smem + OFF_Q), 16, 1024);
      const uint64_t dw = make_sdesc(smem_u32(smem + OFF_W), 16, 1024);
      const uint64_t daq = make_sdesc(smem_u32(smem + OFF_AQ), 16, 1024);
      uint32_t gj = 0, it = 0;
      bool ok = true;
      // O += Aq_J W2[:, J]^T for the block in stage s, Aq buffer b
      auto issue_o = [&](uint32_t g, bool first) -> bool {
        const uint32_t s = g & 1, ws = g % WS;
        if (!W.wait(&aq_full[s], (g >> 1) & 1, 3)) return false;
        // the first product of an item overwrites O: the epilogue must have
        // stored the previous item's
        if (first && it >= 1 && !W.wait(o_empty, (it - 1) & 1, 5)) return false;
        tc_fence_after();
        const uint64_t dw2 = sdesc_add(dw, ws * W_STAGE + 2 * HALF);
        const uint64_t da = sdesc_add(daq, s * HALF);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + TM_O, sdesc_add(da, kk * 32), sdesc_add(dw2, kk * 32), id_o,
                   (first && kk == 0) ? 0u : 1u);
        mma_commit(&w_empty[ws]);
        mma_commit(&aq_empty[s]);
        return true;
      };
      for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x, ++it) {
        if (!W.wait(q_full, it & 1, 4)) { ok = false; break; }
        const uint32_t g0 = gj;
        for (int j = 0; j < a.n_hb; ++j, ++gj) {
          const uint32_t s = gj & 1, ws = gj % WS;
          if (!W.wait(&w_full[ws], (gj / WS) & 1, 6)) { ok = false; break; }
          if (gj >= 2 && !W.wait(&h_empty[s], ((gj >> 1) - 1) & 1, 7)) { ok = false; break; }
          tc_fence_after();
          const uint64_t dws = sdesc_add(dw, ws * W_STAGE);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * HALF + (kk & 3) * 32;
            mma_bf16(tmem + (s ? TM_H1 : TM_H0), sdesc_add(dq, off), sdesc_add(dws, off), id_h,
                     kk > 0);
          }
          mma_commit(&h_full[s]);
          if (j == a.n_hb - 1) mma_commit(q_empty);   // the item's last read of Q
          // the previous block's O product, whose Aq the epilogue is forming
          if (j >= 1 && !issue_o(gj - 1, gj - 1 == g0)) { ok = false; break; }
        }
        if (!ok) break;
        if (!issue_o(gj - 1, gj - 1 == g0)) { ok = false; break; }
        mma_commit(o_full);
      }
      mma_commit(fin);
      W.drain(fin, 0);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q4 = warp & 3;
    const int cg = (warp - 2) >> 2;               // which 32 of the 64 hidden units
    const int r = q4 * 32 + lane;                 // query row of the tile
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    uint32_t gj = 0, it = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x, ++it) {
      const int bh = item / a.n_tiles, qt = item % a.n_tiles;
      for (int j = 0; j < a.n_hb; ++j, ++gj) {
        const uint32_t s = gj & 1;
        if (!W.wait(&h_full[s], (gj >> 1) & 1, 8)) { ok = false; break; }
        tc_fence_after();
        uint32_t rh1[CW], rh3[CW];
        const uint32_t th = tmem + lane_base + (s ? TM_H1 : TM_H0) + cg * CW;
        tmem_ld16_issue(th, rh1);
        tmem_ld16_issue(th + 16, rh1 + 16);
        tmem_ld16_issue(th + 64, rh3);
        tmem_ld16_issue(th + 80, rh3 + 16);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&h_empty[s]);
        uint32_t pk[CW / 2];
#pragma unroll
        for (int c = 0; c < CW; c += 2) {
          const float x0 = __uint_as_float(rh1[c]), x1 = __uint_as_float(rh1[c + 1]);
          pk[c >> 1] = pack_bf16x2(x0 * rd_sigmoid(x0) * __uint_as_float(rh3[c]),
                                   x1 * rd_sigmoid(x1) * __uint_as_float(rh3[c + 1]));
        }
        // Aq buffer s is free once the O product of block gj - 2 is done
        if (gj >= 2 && !W.wait(&aq_empty[s], ((gj >> 1) - 1) & 1, 9)) { ok = false; break; }
        const uint32_t dst = smem_u32(smem + OFF_AQ + s * HALF);
#pragma unroll
        for (int c = 0; c < CW; c += 8)
          st_shared_v4(dst + sw128_offset(r, cg * CW + c), pk[c / 2], pk[c / 2 + 1], pk[c / 2 + 2],
                       pk[c / 2 + 3]);
        fence_async_smem();
        mbar_arrive(&aq_full[s]);
      }
      if (!ok || !W.wait(o_full, it & 1, 10)) { ok = false; break; }
      tc_fence_after();
      // this thread's row, d columns cg * 64 .. cg * 64 + 63
      const int t = qt * BM + r;
      const bool valid = t < a.C;
      const size_t base = ((size_t)bh * a.rows + a.t0 + t) * D + cg * 64;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        float o[32];
        tmem_ld32(tmem + lane_base + TM_O + cg * 64 + h * 32, o);   // every lane: warp-collective
        if (!valid) continue;
        if (a.out_bf16) {
          uint4* dstp = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) + base + h * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dstp[q] = make_uint4(pack_bf16x2(o[8 * q], o[8 * q + 1]), pack_bf16x2(o[8 * q + 2], o[8 * q + 3]),
                                 pack_bf16x2(o[8 * q + 4], o[8 * q + 5]), pack_bf16x2(o[8 * q + 6], o[8 * q + 7]));
        } else {
          float4* dstp = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + base + h * 32);
#pragma unroll
          for (int q = 0; q < 8; ++q) dstp[q] = make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(o_empty);
    }
  }
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TM_COLS);
  }
}

int launch_lact_read_fused(const ReadFusedLaunch& L, cudaStream_t stream) {
  using namespace rd;
  ReadFusedMaps m{};
  const uint64_t BH = (uint64_t)L.BH, row = (uint64_t)D * 2;
  if (make_tmap_bf16_3d(&m.q, L.q, D, L.rows, BH, row, row * L.rows, 64, 128) ||
      make_tmap_bf16_3d(&m.w1, L.w1b, D, L.dh, BH, row, row * L.dh, 64, 64) ||
      make_tmap_bf16_3d(&m.w3, L.w3b, D, L.dh, BH, row, row * L.dh, 64, 64) ||
      make_tmap_bf16_3d(&m.w2, L.w2b, L.dh, D, BH, (uint64_t)L.dh * 2, (uint64_t)L.dh * 2 * D, 64, 128))
    return -1;
  ReadFusedArgs a{};
  a.BH = L.BH; a.rows = L.rows; a.t0 = L.t0; a.C = L.C;
  a.n_hb = L.dh / HB;
  a.n_tiles = (L.C + BM - 1) / BM;
  a.out_bf16 = L.out_bf16;
  a.out = L.out;
  a.st = L.st;
  const int items = a.BH * a.n_tiles;
  if (items <= 0) return 0;
  static std::atomic<uint64_t> attr{0};
  if (allow_dynamic_smem(lact_read_fused_kernel, (int)SMEM, attr)) return -1;
  const int grid = std::max(1, std::min(items, L.max_grid));
  prof_before(K_GEMM_READ, stream);
  if (launch_pdl(lact_read_fused_kernel, dim3(grid), dim3(THREADS), SMEM, stream, m, a) != cudaSuccess)
    return -1;
  prof_after(K_GEMM_READ, stream);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace ttt
