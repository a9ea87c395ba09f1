// gemm_group.cuh -- several independent batched GEMMs in one persistent
// tcgen05 launch: the products of one chunk of the LaCT backward pass (input
// gradients of the keys, the values' upstream term, the queries, and the
// split-K weight gradients), which are all fed by the same elementwise step
// and are independent of one another.
//
//   problem p:  D_p[b][s][m][n] = sum_pair A_pair[b][m][:] . B_pair[b][n][:]
//
// * Every problem is posed with M = 128 (the head dimension d) and N the
//   long side (tokens or hidden units), so each unit is one 128 x 256 tile
//   and every product is a 128 x 256 x 16 tcgen05.mma: per instruction and
//   per barrier hand-off, the most work the single-CTA tensor core takes.
//   A product whose natural output is [tokens][d] or [hidden][d] writes D
//   transposed: TMEM lane = d, so a warp stores 32 consecutive d values
//   (128 bytes) of one output row per instruction.
// * Each problem has its own operand majorness (K-major: rows contiguous
//   along K; MN-major: contiguous along M/N), up to four operand pairs
//   concatenated along K, an optional split of K (split s covers K steps
//   [s k_steps, (s + 1) k_steps) of every pair and writes its own output
//   slice) and an fp32 output with its own leading dimension, strides and
//   row offset.
// * A stage is one 128 x 64 A block (16 KB) and one 256 x 64 B block
//   (32 KB), each brought by ONE tensor copy: K-major blocks as one box of
//   64 K x 128 or 256 rows, MN-major blocks through a blocked 4-D view
//   whose box holds 2 or 4 blocks of 64 M/N elements x 64 K rows.  The
//   issuing lane and the barrier hand-offs cost a fixed time per copy and
//   per stage, not per byte, so a stage is two copies and one wait.
// * Units are handed out by a global counter (one per launch, zero before
//   it), numbered problem by problem, largest K first, so the CTAs finish
//   together; the producer lane draws the next unit and passes its number
//   through a small shared-memory ring to the MMA issuer and the epilogue.
// * Warp 0: TMA producer; warp 1: MMA issuer and TMEM owner (two 256-column
//   accumulators, so a unit's epilogue overlaps the next unit's products);
//   warps 2-9: epilogue, one 128-column half per group of four warps.
#pragma once
#include "common.cuh"

namespace ttt {

namespace gg {
constexpr int MAXP = 6, MAXPAIR = 4, STAGES = 4, EPI_WARPS = 8, RING = 4;
constexpr int BN = 256;                                    // unit width (N)
constexpr uint32_t A_BYTES = 128 * 64 * 2, B_BYTES = BN * 64 * 2, STAGE = A_BYTES + B_BYTES;
constexpr uint32_t BAR_OFF = STAGES * STAGE;
constexpr uint32_t SMEM = BAR_OFF + 512 + 1024;
constexpr uint32_t TM_COLS = 2 * BN;
constexpr int THREADS = (2 + EPI_WARPS) * 32;
}  // namespace gg

struct GroupProblem {
  int M, N;                 // extent of D per (batch, split); M % 128 == 0, N masked
  int tiles_m, tiles_n, splits;
  int k_steps;              // 64-wide K steps per pair per split
  int npairs;               // 1..4
  int a_mn, b_mn;           // operand majorness (1 = MN-major, blocked 4-D map)
  int unit0;                // first work unit of this problem
  int a_k_off[gg::MAXPAIR], b_k_off[gg::MAXPAIR];   // K coordinate offsets per pair
  float* o;                 // fp32 output
  long long o_bs, o_ss;     // batch and split strides (elements)
  int ld;                   // output row length
  int out_t;                // 1: D[m][n] goes to o[(n + row_off) ld + m]; 0: to o[m ld + n]
  int row_off;              // added to n (transposed outputs)
  int v8;                   // untransposed rows start on 32-byte boundaries: 256-bit stores
};

struct GroupMaps {
  CUtensorMap a[gg::MAXP][gg::MAXPAIR], b[gg::MAXP][gg::MAXPAIR];
};

struct GroupArgs {
  int nprob, units;
  unsigned int* ctr;        // unit counter of this launch (zero before it)
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

// one operand block of `rows` M/N rows x 64 K: K-major as a box {64 K, rows}
// of a 3-D map, MN-major as a box {64, 64 K, rows / 64, 1} of a blocked map
TTT_DEVICE_INLINE void group_load(uint8_t* dst, const CUtensorMap* m, uint64_t* bar, bool mn,
                                  int row, int k, int b) {
  if (!mn) tma_load_3d(dst, m, bar, k, row, b);
  else tma_load_4d(dst, m, bar, 0, k, row >> 6, b);
}

__global__ void __launch_bounds__(gg::THREADS, 1)
    gemm_group_kernel(const __grid_constant__ GroupMaps maps, const __grid_constant__ GroupArgs g) {
  using namespace gg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* empty = full + STAGES;
  uint64_t* afull = empty + STAGES;   // [2]
  uint64_t* aempty = afull + 2;       // [2]
  uint64_t* ufull = aempty + 2;       // [RING]
  uint64_t* uempty = ufull + RING;    // [RING]
  uint64_t* fin = uempty + RING;
  int* unit_ring = reinterpret_cast<int*>(fin + 1);   // [RING]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(unit_ring + RING);
  uint32_t* abort_flag = tmem_slot + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&afull[s], 1);
      mbar_init(&aempty[s], EPI_WARPS * 32);
    }
    for (int s = 0; s < RING; ++s) {
      mbar_init(&ufull[s], 1);
      mbar_init(&uempty[s], 1 + EPI_WARPS);   // the MMA lane and one lane per epilogue warp
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
      for (uint32_t j = 0; ok; ++j) {
        // the next unit, published to the other roles (a number past the
        // last unit ends every role's loop)
        const uint32_t r = j % RING;
        if (j >= (uint32_t)RING && !W.wait(&uempty[r], ((j / RING) - 1) & 1, 1)) break;
        int u = (int)atomicAdd(g.ctr, 1u);
        if (u >= g.units) u = -1;
        unit_ring[r] = u;
        mbar_arrive(&ufull[r]);   // release: the number is visible to the waiters
        if (u < 0) break;
        const GroupUnit w = group_unit(g, u);
        const GroupProblem& q = g.p[w.p];
        const int total_k = q.k_steps * q.npairs;
        for (int kk = 0; kk < total_k; ++kk, ++it) {
          const int pr = kk / q.k_steps;
          const int ks = (kk % q.k_steps) + w.sp * q.k_steps;
          const uint32_t s = it % STAGES;
          if (it >= (uint32_t)STAGES && !W.wait(&empty[s], ((it / STAGES) - 1) & 1, 2)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * STAGE;
          mbar_arrive_expect_tx(&full[s], STAGE);
          group_load(st, &maps.a[w.p][pr], &full[s], q.a_mn, w.tm * 128, q.a_k_off[pr] + ks * 64, w.b);
          group_load(st + A_BYTES, &maps.b[w.p][pr], &full[s], q.b_mn, w.tn * BN,
                     q.b_k_off[pr] + ks * 64, w.b);
        }
      }
      it_issued = it;
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (uint32_t lt = 0; ok; ++lt) {
        const uint32_t r = lt % RING;
        if (!W.wait(&ufull[r], (lt / RING) & 1, 3)) break;
        const int u = *reinterpret_cast<volatile int*>(&unit_ring[r]);
        mbar_arrive(&uempty[r]);
        if (u < 0) break;
        const GroupUnit w = group_unit(g, u);
        const GroupProblem& q = g.p[w.p];
        const int total_k = q.k_steps * q.npairs;
        const uint32_t ab = lt & 1;
        if (lt >= 2 && !W.wait(&aempty[ab], ((lt >> 1) - 1) & 1, 4)) break;
        tc_fence_after();
        const uint32_t d = tmem + ab * BN;
        const uint32_t idesc = make_idesc(128, BN, q.a_mn != 0, q.b_mn != 0);
        // the four K = 16 slices of a stage advance the start address by 32 B
        // (K-major) or 2 KB (MN-major); MN-major blocks of 64 are 8 KB apart
        const uint32_t alo = q.a_mn ? 8192u : 16u, blo = q.b_mn ? 8192u : 16u;
        const uint32_t astep = q.a_mn ? 2048u : 32u, bstep = q.b_mn ? 2048u : 32u;
        for (int kk = 0; kk < total_k; ++kk, ++it) {
          const uint32_t s = it % STAGES;
          if (!W.wait(&full[s], (it / STAGES) & 1, 5)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * STAGE);
          const uint64_t ad = make_sdesc(sa, alo, 1024), bd = make_sdesc(sa + A_BYTES, blo, 1024);
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4)
            mma_bf16(d, sdesc_add(ad, k4 * astep), sdesc_add(bd, k4 * bstep), idesc,
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
    // epilogue: warps 2..9 -> TMEM lane quadrant (warp & 3), column half (warp - 2) / 4
    const int q4 = warp & 3;
    const int half = (warp - 2) >> 2;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    for (uint32_t lt = 0;; ++lt) {
      const uint32_t r = lt % RING;
      if (!W.wait(&ufull[r], (lt / RING) & 1, 6)) break;
      const int u = *reinterpret_cast<volatile int*>(&unit_ring[r]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&uempty[r]);
      if (u < 0) break;
      const GroupUnit w = group_unit(g, u);
      const GroupProblem& q = g.p[w.p];
      const uint32_t ab = lt & 1;
      if (!W.wait(&afull[ab], (lt >> 1) & 1, 7)) break;
      tc_fence_after();
      const int m = w.tm * 128 + q4 * 32 + lane;
      const int n0 = w.tn * BN + half * 128;
      float* ob = q.o + w.b * q.o_bs + w.sp * q.o_ss;
#pragma unroll 1
      for (int c = 0; c < 128; c += 32) {
        float v[32];
        tmem_ld32(tmem + lane_base + ab * BN + half * 128 + c, v);
        if (c == 96) {   // the accumulator is read out: the next unit may start
          tc_fence_before();
          mbar_arrive(&aempty[ab]);
        }
        const int n = n0 + c;
        if (m >= q.M || n >= q.N) continue;
        if (q.out_t) {
          // one output row per column: the warp writes 32 consecutive d values
          float* dst = ob + (long long)(n + q.row_off) * q.ld + m;
          const int cnt = min(32, q.N - n);
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < cnt) dst[(long long)j * q.ld] = v[j];
        } else if (q.v8) {
          float* dst = ob + (long long)m * q.ld + n;
#pragma unroll
          for (int j = 0; j < 4; ++j) st_global_v8(dst + 8 * j, reinterpret_cast<const uint32_t*>(v + 8 * j));
        } else {
          float4* dst = reinterpret_cast<float4*>(ob + (long long)m * q.ld + n);
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
