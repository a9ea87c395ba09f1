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
struct KeyGradMaps {
  CUtensorMap k, v, q, w1, w3, w2;
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
TTT_DEVICE_INLINE void named_bar_sync(uint32_t id, uint32_t n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__global__ void __launch_bounds__(kg::THREADS, 1)
    lact_keygrad_kernel(const __grid_constant__ KeyGradMaps maps, const KeyGradArgs a) {
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

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int items_per_bh = a.n_hb * a.n_groups;
  const int n_items = items_per_bh * a.BH;

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
    tma_prefetch_desc(&maps.w1);
    tma_prefetch_desc(&maps.w3);
    tma_prefetch_desc(&maps.w2);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // The TMA thread waits for the preceding kernels after it has issued its
  // first token tiles (inputs of the call, which no kernel of the call
  // writes); everything else waits here.
  if (warp != 0 || lane != 0) pdl_wait();
  const uint32_t tmem = *tmem_slot;
  Waiter W{abort_flag, a.st, 300};

  auto decode = [&](int item, int& bh, int& hb, int& grp) {
    hb = item % a.n_hb;
    grp = (item / a.n_hb) % a.n_groups;
    bh = item / items_per_bh;
  };
  auto group_tiles = [&](int grp) {
    const int first = grp * a.tiles_per_group;
    return std::max(0, std::min(a.tiles_per_group, a.tiles_total - first));
  };

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      uint32_t tile = 0, item_ctr = 0;
      bool ok = true;
      // tile i of an item: key tiles (K and V) first, then query tiles (Q in
      // the K slot)
      auto issue_tile = [&](uint32_t t, int i, int nt, int bh, int grp) {
        const uint32_t s = t & 1;
        const bool is_q = i >= nt;
        const int row = a.t0 + (grp * a.tiles_per_group + (is_q ? i - nt : i)) * BM;
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
      // the first item's first tile goes out before the wait for the
      // preceding kernels (it overlaps that kernel's tail); its second one
      // follows the weights, so the weights do not queue behind 128 KB of
      // token tiles
      int pre = 0;
      if ((int)blockIdx.x < n_items) {
        int bh, hb, grp;
        decode(blockIdx.x, bh, hb, grp);
        const int nt = group_tiles(grp);
        const int n_all = nt + (a.queries ? nt : 0);
        for (; pre < 1 && pre < n_all; ++pre, ++tile) issue_tile(tile, pre, nt, bh, grp);
      }
      pdl_wait();
      for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x, ++item_ctr) {
        int bh, hb, grp;
        decode(item, bh, hb, grp);
        const int j0 = hb * HB;
        const int nt = group_tiles(grp);
        if (item_ctr >= 1 && !W.wait(w_empty, (item_ctr - 1) & 1, 1)) { ok = false; break; }
        // weights of the item: [W1_J; W3_J] as two K atoms (d 0-63, 64-127),
        // W2[:, J] as 128 d-rows of 64 hidden units
        mbar_arrive_expect_tx(w_full, 2 * HALF + 2 * 8192);
        for (int atom = 0; atom < 2; ++atom) {
          tma_load_3d(smem + OFF_W13 + atom * HALF, &maps.w1, w_full, atom * 64, j0, bh);
          tma_load_3d(smem + OFF_W13 + atom * HALF + HALF / 2, &maps.w3, w_full, atom * 64, j0, bh);
          tma_load_3d(smem + OFF_W2 + atom * 8192, &maps.w2, w_full, j0, atom * 64, bh);
        }
        if (item_ctr == 0 && pre == 1 && nt + (a.queries ? nt : 0) > 1) {   // second tile
          issue_tile(tile, 1, nt, bh, grp);
          ++tile;
          ++pre;
        }
        // warm L2 with the item's later tiles; their loads then hit it
        for (int i = 2; i < nt; ++i)
          for (int h = 0; h < 2; ++h) {
            const int row = a.t0 + (grp * a.tiles_per_group + i) * BM;
            tma_prefetch_l2_3d(&maps.k, h * 64, row, bh);
            tma_prefetch_l2_3d(&maps.v, h * 64, row, bh);
          }
        const int nq = a.queries ? nt : 0;
        for (int i = item_ctr == 0 ? pre : 0; ok && i < nt + nq; ++i, ++tile) {
          const uint32_t s = tile & 1;
          if (tile >= 2 && !W.wait(&kv_empty[s], ((tile >> 1) - 1) & 1, 2)) { ok = false; break; }
          issue_tile(tile, i, nt, bh, grp);
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
      for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x, ++item_ctr) {
        int bh, hb, grp;
        decode(item, bh, hb, grp);
        const int nt = group_tiles(grp);
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
    for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++item_ctr) {
      int bh, hb, grp;
      decode(item, bh, hb, grp);
      const int nt = group_tiles(grp);
      const int nq = a.queries ? nt : 0;
      bool ok = true;
      for (int i = 0; i < nt; ++i, ++tile, ++ktile) {
        const int tc = (grp * a.tiles_per_group + i) * BM + r;   // token row in the chunk
        const bool valid = tc < a.C;
        // -eta, zero for rows past the chunk (their H and dGr are finite, so
        // every gradient operand of such a row comes out zero)
        const float neta = valid ? -a.lr[(size_t)bh * a.lr_len + a.t0 + tc] : 0.f;
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
            const int tc = (grp * a.tiles_per_group + i) * BM + r;
            const bool valid = tc < a.C;
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
                uint4* dq = reinterpret_cast<uint4*>(a.Aq + (size_t)bh * a.aq_bs + (size_t)tc * a.dh +
                                                     hb * HB + c0);
#pragma unroll
                for (int j = 0; j < CW / 8; ++j) dq[j] = make_uint4(oq[4 * j], oq[4 * j + 1], oq[4 * j + 2], oq[4 * j + 3]);
              }
            }
          }
        }
      }
      // both halves finish the item before either starts the next one, so no
      // epilogue warp waits on an accumulator phase two uses ahead; every
      // epilogue thread reaches this barrier, also after a failed wait
      named_bar_sync(1, EPI_WARPS * 32);
      if (!ok || W.aborted()) break;
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

int launch_lact_keygrad(const KeyGradLaunch& L, cudaStream_t stream) {
  KeyGradMaps m{};
  const uint64_t BH = (uint64_t)L.BH;
  const uint64_t tok_row = (uint64_t)kg::D * 2;
  if (make_tmap_bf16_3d(&m.k, L.k, kg::D, L.N_in, BH, tok_row, tok_row * L.N_in, 64, 128) ||
      make_tmap_bf16_3d(&m.v, L.v, kg::D, L.N_in, BH, tok_row, tok_row * L.N_in, 64, 128) ||
      make_tmap_bf16_3d(&m.q, L.q ? L.q : L.k, kg::D, L.N_in, BH, tok_row, tok_row * L.N_in, 64, 128) ||
      make_tmap_bf16_3d(&m.w1, L.w1b, kg::D, L.dh, BH, tok_row, tok_row * L.dh, 64, 64) ||
      make_tmap_bf16_3d(&m.w3, L.w3b, kg::D, L.dh, BH, tok_row, tok_row * L.dh, 64, 64) ||
      make_tmap_bf16_3d(&m.w2, L.w2b, L.dh, kg::D, BH, (uint64_t)L.dh * 2, (uint64_t)L.dh * 2 * kg::D,
                        64, 64))
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
  if (allow_dynamic_smem(lact_keygrad_kernel, (int)kg::SMEM, attr)) return -1;
  const int items = a.n_hb * a.n_groups * L.BH;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  prof_before(K_KEYGRAD, stream);
  if (launch_pdl(lact_keygrad_kernel, dim3(std::min(items, sms)), dim3(kg::THREADS), kg::SMEM, stream,
                 m, a) != cudaSuccess)
    return -1;
  prof_after(K_KEYGRAD, stream);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace ttt
