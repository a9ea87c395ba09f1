// gemm_group.cuh -- several independent batched GEMMs in one persistent
// tcgen05 launch: the products of one chunk of the LaCT backward pass (input
// gradients of the keys, the values' upstream term, the queries, and the
// split-K weight gradients), which are all fed by the same elementwise step
// and are independent of one another.
//
//   problem p:  C_p[b][s][m][n] = sum_pair A_pair[b][m][:] . B_pair[b][n][:]
//
// * Each problem has its own shape, operand majorness (K- or MN-major, as
//   in gemm.cuh), up to four operand pairs concatenated along K, an optional
//   split of K (split s covers K steps [s k_steps, (s + 1) k_steps) of every
//   pair and writes its own output slice) and an fp32 output with its own
//   leading dimension, batch / split strides and row offset.
// * Work units are 128 x 128 output tiles, numbered problem by problem
//   (largest K first); CTA c takes units c, c + grid, ...  One launch keeps
//   every SM busy where each product alone would fill one wave of
//   single-tile CTAs with nothing to overlap.
// * Warp 0: TMA producer over a STAGES-deep ring of 32 KB stages; warp 1:
//   MMA issuer and TMEM owner (two 128-column accumulators, so a tile's
//   epilogue overlaps the next tile's products); warps 2-5: epilogue.
#pragma once
#include "common.cuh"

namespace ttt {

namespace gg {
constexpr int MAXP = 6, MAXPAIR = 4, BN = 128, STAGES = 6;
constexpr uint32_t A_BYTES = 128 * 64 * 2, B_BYTES = BN * 64 * 2, STAGE = A_BYTES + B_BYTES;
constexpr uint32_t BAR_OFF = STAGES * STAGE;
constexpr uint32_t SMEM = BAR_OFF + 256 + 1024;
constexpr uint32_t TM_COLS = 2 * BN;
}  // namespace gg

struct GroupProblem {
  int M, N;                 // output extent per (batch, split); N % 128 == 0, rows masked
  int tiles_m, tiles_n, splits;
  int k_steps;              // 64-wide K steps per pair per split
  int npairs;               // 1..4
  int a_mn, b_mn;           // operand majorness (1 = MN-major)
  int unit0;                // first work unit of this problem
  int a_m_off[gg::MAXPAIR], a_k_off[gg::MAXPAIR];   // TMA coordinate offsets per pair
  int b_n_off[gg::MAXPAIR], b_k_off[gg::MAXPAIR];
  float* o;                 // fp32 output
  long long o_bs, o_ss;     // batch and split strides (elements)
  int ld, out_row_off;      // row length; added to the output row index
  int v8;                   // rows start on 32-byte boundaries: 256-bit stores
};

struct GroupMaps {
  CUtensorMap a[gg::MAXP][gg::MAXPAIR], b[gg::MAXP][gg::MAXPAIR];
};

struct GroupArgs {
  int nprob, units;
  GroupProblem p[gg::MAXP];
  DevStatus st;
};

struct GroupUnit {
  int p, tm, tn, b, sp;
};

TTT_DEVICE_INLINE GroupUnit group_unit(const GroupArgs& g, int u) {
  int p = 0;
  while (p + 1 < g.nprob && u >= g.p[p + 1].unit0) ++p;
  const GroupProblem& q = g.p[p];
  const int l = u - q.unit0;
  GroupUnit r;
  r.p = p;
  r.tm = l % q.tiles_m;
  r.tn = (l / q.tiles_m) % q.tiles_n;
  const int bs = l / (q.tiles_m * q.tiles_n);
  r.b = bs / q.splits;
  r.sp = bs % q.splits;
  return r;
}

__global__ void __launch_bounds__(192, 1)
    gemm_group_kernel(const __grid_constant__ GroupMaps maps, const __grid_constant__ GroupArgs g) {
  using namespace gg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* empty = full + STAGES;
  uint64_t* afull = empty + STAGES;   // [2]
  uint64_t* aempty = afull + 2;       // [2]
  uint64_t* fin = aempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  uint32_t* abort_flag = tmem_slot + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&afull[s], 1);
      mbar_init(&aempty[s], 128);
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
  pdl_wait();
  pdl_launch_dependents();
  const uint32_t tmem = *tmem_slot;
  Waiter W{abort_flag, g.st, 700};
  uint32_t it_issued = 0;   // stages filled (producer lane)

  if (warp == 0) {
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < g.units; u += gridDim.x) {
        const GroupUnit w = group_unit(g, u);
        const GroupProblem& q = g.p[w.p];
        const int total_k = q.k_steps * q.npairs;
        for (int kk = 0; kk < total_k; ++kk, ++it) {
          const int pr = kk / q.k_steps;
          const int ks = (kk % q.k_steps) + w.sp * q.k_steps;
          const uint32_t s = it % STAGES;
          if (it >= (uint32_t)STAGES && !W.wait(&empty[s], ((it / STAGES) - 1) & 1, 1)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + s * STAGE;
          uint8_t* sb = sa + A_BYTES;
          const CUtensorMap* ma = &maps.a[w.p][pr];
          const CUtensorMap* mb = &maps.b[w.p][pr];
          mbar_arrive_expect_tx(&full[s], STAGE);
          const int am = q.a_m_off[pr] + w.tm * 128, ak = q.a_k_off[pr] + ks * 64;
          const int bn = q.b_n_off[pr] + w.tn * BN, bk = q.b_k_off[pr] + ks * 64;
          if (!q.a_mn) {
            tma_load_3d(sa, ma, &full[s], ak, am, w.b);
          } else {
            tma_load_3d(sa, ma, &full[s], am, ak, w.b);
            tma_load_3d(sa + 8192, ma, &full[s], am + 64, ak, w.b);
          }
          if (!q.b_mn) {
            tma_load_3d(sb, mb, &full[s], bk, bn, w.b);
          } else {
            tma_load_3d(sb, mb, &full[s], bn, bk, w.b);
            tma_load_3d(sb + 8192, mb, &full[s], bn + 64, bk, w.b);
          }
        }
      }
      it_issued = it;
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      uint32_t it = 0, lt = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < g.units; u += gridDim.x, ++lt) {
        const GroupUnit w = group_unit(g, u);
        const GroupProblem& q = g.p[w.p];
        const int total_k = q.k_steps * q.npairs;
        const uint32_t ab = lt & 1;
        if (lt >= 2 && !W.wait(&aempty[ab], ((lt >> 1) - 1) & 1, 2)) break;
        tc_fence_after();
        const uint32_t d = tmem + ab * BN;
        const uint32_t idesc = make_idesc(128, BN, q.a_mn != 0, q.b_mn != 0);
        // the four K = 16 slices of a stage advance the start address by 32 B
        // (K-major) or 2 KB (MN-major); MN-major blocks of 64 are 8 KB apart
        const uint32_t alo = q.a_mn ? 8192u : 16u, blo = q.b_mn ? 8192u : 16u;
        const uint32_t astep = q.a_mn ? 2048u : 32u, bstep = q.b_mn ? 2048u : 32u;
        for (int kk = 0; kk < total_k; ++kk, ++it) {
          const uint32_t s = it % STAGES;
          if (!W.wait(&full[s], (it / STAGES) & 1, 3)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * STAGE);
          const uint64_t ad0 = make_sdesc(sa, alo, 1024), bd0 = make_sdesc(sa + A_BYTES, blo, 1024);
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4)
            mma_bf16(d, sdesc_add(ad0, k4 * astep), sdesc_add(bd0, k4 * bstep), idesc,
                     (kk | k4) != 0 ? 1u : 0u);
          mma_commit(&empty[s]);
        }
        if (!ok) break;
        mma_commit(&afull[ab]);
      }
      mma_commit(fin);
      W.drain(fin, 0);
    }
    __syncwarp();
  } else {
    // epilogue: warps 2..5 -> TMEM lane quadrants 2,3,0,1
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    uint32_t lt = 0;
    for (int u = blockIdx.x; u < g.units; u += gridDim.x, ++lt) {
      const GroupUnit w = group_unit(g, u);
      const GroupProblem& q = g.p[w.p];
      const uint32_t ab = lt & 1;
      if (!W.wait(&afull[ab], (lt >> 1) & 1, 4)) break;
      tc_fence_after();
      const int m = w.tm * 128 + row;
      const bool valid = m < q.M;
      float* orow = q.o + w.b * q.o_bs + w.sp * q.o_ss + (long long)(m + q.out_row_off) * q.ld +
                    w.tn * BN;
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        float v[32];
        tmem_ld32(tmem + lane_base + ab * BN + c, v);
        if (c == BN - 32) {   // the accumulator is read out: the next tile may start
          tc_fence_before();
          mbar_arrive(&aempty[ab]);
        }
        if (valid && q.v8) {
#pragma unroll
          for (int j = 0; j < 4; ++j) st_global_v8(orow + c + 8 * j, reinterpret_cast<const uint32_t*>(v + 8 * j));
        } else if (valid) {
          float4* dst = reinterpret_cast<float4*>(orow + c);
#pragma unroll
          for (int j = 0; j < 8; ++j) dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0 && lane == 0 && W.aborted()) {   // copies still in flight land before the CTA exits
    for (uint32_t i = it_issued > (uint32_t)STAGES ? it_issued - STAGES : 0; i < it_issued; ++i)
      W.drain(&full[i % STAGES], (i / STAGES) & 1);
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TM_COLS);
  }
}

}  // namespace ttt
