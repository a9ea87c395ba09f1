// gemm.cuh -- persistent, warp-specialised tcgen05 GEMM used by the LaCT
// path (chunk gradients, memory read, Newton-Schulz).
//
//   C[b][m][n] = alpha * sum_p A_p[b][m][:] . B_p[b][n][:]  + beta * Cin[b][m][n]
//
// * bf16 operands, fp32 accumulation in TMEM (tcgen05.mma kind::f16).
// * Up to three operand pairs (A_p, B_p) are concatenated along K; a split
//   precision product (x_hi + x_lo) * y is two pairs.
// * A and B are loaded by TMA with 128-byte swizzle, either K-major (rows of
//   the operand are contiguous along K) or MN-major (contiguous along M/N).
// * Warp 0: TMA producer; warp 1: MMA issuer + TMEM owner; warps 2-5:
//   epilogue (TMEM -> registers -> global).  TMEM holds two accumulators so
//   the epilogue of one tile overlaps the MMAs of the next.
// * Tiles: tile = ((b*splits + s) * tiles_n + tn) * tiles_m + tm; each CTA
//   walks tiles with stride gridDim.x.  In cluster mode (cluster_n > 1) the
//   cluster_n CTAs of a cluster take the N tiles of one output row block
//   (tn fastest) and exchange per-row partial sums over distributed shared
//   memory; one tile per CTA.
// * epi == 1: the epilogue is the weight update of a chunk -- optimizer step
//   on the fp32 weights, row L2 normalisation, bf16 operand copies -- with
//   the output rows being weight rows (rows >= rows_first go to the second
//   matrix, so [W1; W3] can be updated by one launch).
#pragma once
#include "common.cuh"

namespace ttt {

struct GemmArgs {
  int M, N;              // output extent per batch (rows masked, N % BN == 0)
  int batch, splits;
  int k_steps;           // 64-wide K steps per split per pair
  int npairs;            // 1..3
  int a_m_off[3], a_k_off[3];   // TMA coordinate offsets per pair
  int b_n_off[3], b_k_off[3];
  int a_b_off, b_b_off;  // batch coordinate offsets
  float alpha, beta;
  const float* cin;      // [batch][M][ldc] (beta != 0)
  long long cin_bs;
  int ldc;
  float* o32;            // [batch][splits][..][ld32] (nullable)
  long long o32_bs, o32_ss;
  int ld32;
  __nv_bfloat16* o16;    // (nullable)
  __nv_bfloat16* o16lo;  // (nullable) residual v - bf16(v), same layout as o16
  long long o16_bs;
  int ld16;
  int out_row_off;       // added to the output row index
  int cluster_n;         // > 1: N tiles of a row block form one cluster
  // ---- epi == 1: weight update (splits == 1).  Row m of batch b is row m of
  // matrix 0 ([batch][rows_first][ldw]) or row m - rows_first of matrix 1.
  int epi;
  int rows_first;
  float* W[2];           // fp32 weights
  float* Mom[2];         // momentum (nullable: plain GD)
  __nv_bfloat16* Wb[2];  // bf16 operand copies
  __nv_bfloat16* Wlo[2]; // bf16 residual copies (nullable)
  int ldw;               // row length of the weights (= N)
  float mom_beta, norm_eps;
  int normalize;
  DevStatus st;
};

struct GemmMaps {
  CUtensorMap a[3], b[3];
};

// TMEM columns for the two accumulators (allocations are powers of two >= 32)
template <int BN>
struct GemmTmem {
  static constexpr uint32_t COLS = 2 * BN <= 32 ? 32 : 2 * BN <= 64 ? 64 : 2 * BN <= 128 ? 128
                                   : 2 * BN <= 256 ? 256 : 512;
  static_assert(2 * BN <= 512, "two accumulators fit in TMEM");
};

template <int BN, int STAGES>
struct GemmSmem {
  static constexpr uint32_t A_BYTES = 128 * 64 * 2;
  static constexpr uint32_t B_BYTES = BN * 64 * 2;
  static constexpr uint32_t STAGE = A_BYTES + B_BYTES;
  static constexpr uint32_t BAR_OFF = STAGES * STAGE;
  static constexpr uint32_t RED_OFF = BAR_OFF + 256;          // 128 floats (row sums)
  static constexpr uint32_t BYTES = RED_OFF + 512 + 1024;
};

TTT_DEVICE_INLINE void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
TTT_DEVICE_INLINE float ld_dsmem_f32(const float* local, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

// Weight update from one accumulator tile (epi == 1).  One thread owns one
// row (its TMEM lane): pass 1 reads G from TMEM and the fp32 weights (and
// momentum) from global, forms the unnormalised row, writes it back into
// TMEM and accumulates its squared norm; in cluster mode the partial norms
// of the N tiles are added over distributed shared memory; pass 2 scales
// the row and stores fp32 weights and bf16 copies.
template <int BN>
TTT_DEVICE_INLINE void epilogue_update(const GemmArgs& g, uint32_t tacc, int b, int m, int n0,
                                       bool valid, float* red) {
  const int mat = m >= g.rows_first ? 1 : 0;
  const int mr = m - mat * g.rows_first;
  const size_t ro = ((size_t)b * g.rows_first + mr) * g.ldw + n0;
  float* Wr = g.W[mat] + ro;
  float* Mr = g.Mom[mat] != nullptr ? g.Mom[mat] + ro : nullptr;
  float ss = 0.f;
  float4 wn[8];
  if (valid) {
#pragma unroll
    for (int j = 0; j < 8; ++j) wn[j] = reinterpret_cast<const float4*>(Wr)[j];
  }
#pragma unroll 1
  for (int c = 0; c < BN; c += 32) {
    uint32_t r0[16], r1[16];
    tmem_ld16_issue(tacc + c, r0);
    tmem_ld16_issue(tacc + c + 16, r1);
    float4 wc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) wc[j] = wn[j];
    if (valid && c + 32 < BN) {   // prefetch the next 32 weights
#pragma unroll
      for (int j = 0; j < 8; ++j) wn[j] = reinterpret_cast<const float4*>(Wr + c + 32)[j];
    }
    float4 mc[8];
    if (valid && Mr != nullptr) {
#pragma unroll
      for (int j = 0; j < 8; ++j) mc[j] = reinterpret_cast<const float4*>(Mr + c)[j];
    }
    tmem_wait_ld();
    float u[32];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      u[j] = __uint_as_float(r0[j]);
      u[16 + j] = __uint_as_float(r1[j]);
    }
    if (valid && Mr != nullptr) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        mc[j].x = g.mom_beta * mc[j].x + u[4 * j];
        mc[j].y = g.mom_beta * mc[j].y + u[4 * j + 1];
        mc[j].z = g.mom_beta * mc[j].z + u[4 * j + 2];
        mc[j].w = g.mom_beta * mc[j].w + u[4 * j + 3];
        reinterpret_cast<float4*>(Mr + c)[j] = mc[j];
        u[4 * j] = mc[j].x; u[4 * j + 1] = mc[j].y; u[4 * j + 2] = mc[j].z; u[4 * j + 3] = mc[j].w;
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      u[4 * j] = wc[j].x - u[4 * j];
      u[4 * j + 1] = wc[j].y - u[4 * j + 1];
      u[4 * j + 2] = wc[j].z - u[4 * j + 2];
      u[4 * j + 3] = wc[j].w - u[4 * j + 3];
    }
    if (valid) {
#pragma unroll
      for (int j = 0; j < 32; ++j) ss += u[j] * u[j];
    }
    tmem_st16(tacc + c, u);
    tmem_st16(tacc + c + 16, u + 16);
  }
  if (g.cluster_n > 1) {
    const int row = threadIdx.x - 64;
    red[row] = ss;
    // warps 0-1 join this cluster barrier at the end of their roles
    cluster_sync_all();
    float tot = 0.f;
    for (int r = 0; r < g.cluster_n; ++r) tot += ld_dsmem_f32(&red[row], (uint32_t)r);
    ss = tot;
  }
  // pass 2 (tcgen05.ld is warp-collective: every lane runs it, stores are
  // guarded by the row's validity)
  const float scale = g.normalize ? 1.f / fmaxf(sqrtf(ss), g.norm_eps) : 1.f;
  __nv_bfloat16* Br = g.Wb[mat] + ro;
  __nv_bfloat16* Lr = g.Wlo[mat] != nullptr ? g.Wlo[mat] + ro : nullptr;
#pragma unroll 1
  for (int c = 0; c < BN; c += 32) {
    float v[32];
    tmem_ld32(tacc + c, v);
    if (!valid) continue;
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] *= scale;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      reinterpret_cast<float4*>(Wr + c)[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    uint32_t h[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) h[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
#pragma unroll
    for (int j = 0; j < 4; ++j)
      reinterpret_cast<uint4*>(Br + c)[j] = make_uint4(h[4 * j], h[4 * j + 1], h[4 * j + 2], h[4 * j + 3]);
    if (Lr != nullptr) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t l[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int e = 8 * j + 2 * q;
          l[q] = pack_bf16x2(v[e] - bf16lo(h[e >> 1]), v[e + 1] - bf16hi(h[e >> 1]));
        }
        reinterpret_cast<uint4*>(Lr + c)[j] = make_uint4(l[0], l[1], l[2], l[3]);
      }
    }
  }
}

// BLK: the MN-major operands come through blocked 4-D maps (make_tmap_bf16_blocked,
// boxes of 2 blocks for A and BN / 64 for B), one copy per operand per stage.
template <int BN, bool A_MN, bool B_MN, int STAGES, bool BLK = false>
__global__ void __launch_bounds__(192, 1)
    gemm_bf16_kernel(const __grid_constant__ GemmMaps maps, const GemmArgs g) {
  using L = GemmSmem<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* empty = full + STAGES;
  uint64_t* afull = empty + STAGES;   // [2]
  uint64_t* aempty = afull + 2;       // [2]
  uint64_t* fin = aempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  uint32_t* abort_flag = tmem_slot + 1;
  float* red = reinterpret_cast<float*>(smem + L::RED_OFF);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_m = (g.M + 127) / 128, tiles_n = g.N / BN;
  const int n_tiles = tiles_m * tiles_n * g.splits * g.batch;
  const int total_k = g.k_steps * g.npairs;
  const bool clustered = g.cluster_n > 1;

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
    tmem_alloc(tmem_slot, GemmTmem<BN>::COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    for (int p = 0; p < g.npairs; ++p) {
      tma_prefetch_desc(&maps.a[p]);
      tma_prefetch_desc(&maps.b[p]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  pdl_launch_dependents();
  const uint32_t tmem = *tmem_slot;
  Waiter W{abort_flag, g.st, 100};

  auto decode = [&](int t, int& tm, int& tn, int& b, int& sp) {
    if (clustered) {
      tn = t % tiles_n;
      tm = (t / tiles_n) % tiles_m;
    } else {
      tm = t % tiles_m;
      tn = (t / tiles_m) % tiles_n;
    }
    const int bs = t / (tiles_m * tiles_n);
    b = bs / g.splits;
    sp = bs % g.splits;
  };

  if (warp == 0) {
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
        int tm, tn, b, sp;
        decode(t, tm, tn, b, sp);
        for (int kk = 0; kk < total_k; ++kk, ++it) {
          const int p = kk / g.k_steps;
          const int ks = (kk % g.k_steps) + sp * g.k_steps;
          const uint32_t s = it % STAGES;
          if (it >= (uint32_t)STAGES && !W.wait(&empty[s], ((it / STAGES) - 1) & 1, 1)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + s * L::STAGE;
          uint8_t* sb = sa + L::A_BYTES;
          mbar_arrive_expect_tx(&full[s], L::STAGE);
          const int am = g.a_m_off[p] + tm * 128, ak = g.a_k_off[p] + ks * 64;
          const int bn = g.b_n_off[p] + tn * BN, bk = g.b_k_off[p] + ks * 64;
          if (!A_MN) {
            tma_load_3d(sa, &maps.a[p], &full[s], ak, am, b + g.a_b_off);
          } else if (BLK) {
            tma_load_4d(sa, &maps.a[p], &full[s], 0, ak, am >> 6, b + g.a_b_off);
          } else {
            tma_load_3d(sa, &maps.a[p], &full[s], am, ak, b + g.a_b_off);
            tma_load_3d(sa + 8192, &maps.a[p], &full[s], am + 64, ak, b + g.a_b_off);
          }
          if (!B_MN) {
            tma_load_3d(sb, &maps.b[p], &full[s], bk, bn, b + g.b_b_off);
          } else if (BLK) {
            tma_load_4d(sb, &maps.b[p], &full[s], 0, bk, bn >> 6, b + g.b_b_off);
          } else {
#pragma unroll
            for (int j = 0; j < BN / 64; ++j)
              tma_load_3d(sb + j * 8192, &maps.b[p], &full[s], bn + 64 * j, bk, b + g.b_b_off);
          }
        }
      }
      if (W.aborted()) {
        const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0;
        for (uint32_t i = first; i < it; ++i) W.drain(&full[i % STAGES], (i / STAGES) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = make_idesc(128, BN, A_MN, B_MN);
      uint32_t it = 0, lt = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++lt) {
        const uint32_t ab = lt & 1;
        if (lt >= 2 && !W.wait(&aempty[ab], ((lt >> 1) - 1) & 1, 2)) break;
        tc_fence_after();
        const uint32_t d = tmem + ab * BN;
        for (int kk = 0; kk < total_k; ++kk, ++it) {
          const uint32_t s = it % STAGES;
          if (!W.wait(&full[s], (it / STAGES) & 1, 3)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * L::STAGE);
          const uint32_t sb = sa + L::A_BYTES;
          // descriptors of the stage; the four K=16 slices advance the start
          // address field (16-byte units) by 32 B (K-major) or 2 KB (MN-major)
          const uint64_t ad0 = A_MN ? make_sdesc(sa, 8192, 1024) : make_sdesc(sa, 16, 1024);
          const uint64_t bd0 = B_MN ? make_sdesc(sb, 8192, 1024) : make_sdesc(sb, 16, 1024);
          constexpr uint64_t ASTEP = A_MN ? (2048 >> 4) : (32 >> 4);
          constexpr uint64_t BSTEP = B_MN ? (2048 >> 4) : (32 >> 4);
          mma_bf16(d, ad0, bd0, idesc, kk != 0);
#pragma unroll
          for (int k4 = 1; k4 < 4; ++k4)
            mma_bf16(d, ad0 + k4 * ASTEP, bd0 + k4 * BSTEP, idesc, 1u);
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
    bool synced = false;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++lt) {
      int tm, tn, b, sp;
      decode(t, tm, tn, b, sp);
      const uint32_t ab = lt & 1;
      if (!W.wait(&afull[ab], (lt >> 1) & 1, 4)) break;
      tc_fence_after();
      const int m = tm * 128 + row;
      const bool valid = m < g.M;
      const int orow = m + g.out_row_off;
      if (g.epi == 1) {
        epilogue_update<BN>(g, tmem + lane_base + ab * BN, b, m, tn * BN, valid, red);
        synced = clustered;
        tc_fence_before();
        mbar_arrive(&aempty[ab]);
        continue;
      }
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        float v[32];
        tmem_ld32(tmem + lane_base + ab * BN + c, v);
        if (valid) {
          const int n = tn * BN + c;
          if (g.beta != 0.f) {
            const float4* cp =
                reinterpret_cast<const float4*>(g.cin + b * g.cin_bs + (size_t)m * g.ldc + n);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float4 x = cp[j];
              v[4 * j + 0] = g.alpha * v[4 * j + 0] + g.beta * x.x;
              v[4 * j + 1] = g.alpha * v[4 * j + 1] + g.beta * x.y;
              v[4 * j + 2] = g.alpha * v[4 * j + 2] + g.beta * x.z;
              v[4 * j + 3] = g.alpha * v[4 * j + 3] + g.beta * x.w;
            }
          } else if (g.alpha != 1.f) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] *= g.alpha;
          }
          if (g.o32 != nullptr) {
            float4* dst = reinterpret_cast<float4*>(g.o32 + b * g.o32_bs + sp * g.o32_ss +
                                                    (size_t)orow * g.ld32 + n);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
          }
          if (g.o16 != nullptr) {
            const size_t o = b * g.o16_bs + (size_t)orow * g.ld16 + n;
            uint32_t hv[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) hv[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
            uint4* dst = reinterpret_cast<uint4*>(g.o16 + o);
#pragma unroll
            for (int j = 0; j < 4; ++j) dst[j] = make_uint4(hv[4 * j], hv[4 * j + 1], hv[4 * j + 2], hv[4 * j + 3]);
            if (g.o16lo != nullptr) {
              uint4* dlo = reinterpret_cast<uint4*>(g.o16lo + o);
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                uint32_t l[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                  const int e = 8 * j + 2 * u;
                  l[u] = pack_bf16x2(v[e] - bf16lo(hv[e >> 1]), v[e + 1] - bf16hi(hv[e >> 1]));
                }
                dlo[j] = make_uint4(l[0], l[1], l[2], l[3]);
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&aempty[ab]);
    }
    // an epilogue that never reached the update (abort) still joins the
    // cluster barrier its peers wait on
    if (clustered && !synced) cluster_sync_all();
  }
  // cluster mode: warps 0-1 join the row-sum barrier here; then every
  // thread waits until the peers have finished reading this CTA's row sums
  if (clustered) {
    if (warp < 2) cluster_sync_all();
    cluster_sync_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, GemmTmem<BN>::COLS);
  }
}

}  // namespace ttt
