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
// * Split-K over blockIdx-independent tile ids: tile = ((b*splits + s) *
//   tiles_n + tn) * tiles_m + tm; each CTA walks tiles with stride gridDim.x.
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
  // ---- fused split-K reduction + optimizer + row normalisation (epi == 1);
  // requires one N tile per row (N == BN).  W rows are the output rows.
  int epi;               // 0: store (alpha/beta/cin/o32/o16), 1: update
  float* W;              // fp32 weights [batch][M][N]
  float* Mom;            // momentum [batch][M][N] (nullable: plain GD)
  __nv_bfloat16* Wb;     // bf16 operand copy [batch][M][N]
  __nv_bfloat16* Wlo;    // residual copy W - bf16(W) (nullable)
  float* part;           // split-K partials [splits][batch][M][N] (splits > 1)
  int* counters;         // [batch][tiles_m], zero on entry, left zero on exit
  float mom_beta, norm_eps;
  int normalize;
  DevStatus st;
};

struct GemmMaps {
  CUtensorMap a[3], b[3];
};

template <int BN, int STAGES>
struct GemmSmem {
  static constexpr uint32_t A_BYTES = 128 * 64 * 2;
  static constexpr uint32_t B_BYTES = BN * 64 * 2;
  static constexpr uint32_t STAGE = A_BYTES + B_BYTES;
  static constexpr uint32_t BAR_OFF = STAGES * STAGE;
  static constexpr uint32_t BYTES = BAR_OFF + 256 + 1024;
};

// Named barrier of the four epilogue warps (ids 0 is __syncthreads).
TTT_DEVICE_INLINE void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Split-K reduction + GD / momentum update + row L2 normalisation of one
// output tile whose N extent is a whole weight row.  Every split CTA stores
// its partial; the last one to arrive (per-tile counter) sums them with its
// own accumulator, applies the optimizer to the fp32 weights, normalises the
// rows and refreshes the bf16 operand copy.
template <int BN>
TTT_DEVICE_INLINE void epilogue_update(const GemmArgs& g, uint32_t tacc, int b, int sp, int tm,
                                       int m, bool valid, uint32_t* epi_flag) {
  const size_t row_off = ((size_t)b * g.M + m) * BN;
  const size_t split_stride = (size_t)g.batch * g.M * BN;
  if (g.splits > 1) {
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      float v[32];
      tmem_ld32(tacc + c, v);
      if (valid) {
        float4* dst = reinterpret_cast<float4*>(g.part + sp * split_stride + row_off + c);
#pragma unroll
        for (int j = 0; j < 8; ++j) dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
      }
    }
    __threadfence();
    epi_bar();
    if (threadIdx.x == 64) {
      int* cnt = g.counters + (size_t)b * ((g.M + 127) / 128) + tm;
      const int prev = atomicAdd(cnt, 1);
      const bool last = prev == g.splits - 1;
      if (last) *cnt = 0;
      *epi_flag = last ? 1u : 0u;
    }
    epi_bar();
    if (*epi_flag == 0u) return;
    __threadfence();
  }
  float ss = 0.f;
#pragma unroll 1
  for (int c = 0; c < BN; c += 32) {
    float v[32];
    tmem_ld32(tacc + c, v);
    if (!valid) continue;
    for (int s = 0; s < g.splits; ++s) {
      if (s == sp) continue;
      const float4* src = reinterpret_cast<const float4*>(g.part + s * split_stride + row_off + c);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float4 x = __ldcg(src + j);
        v[4 * j] += x.x; v[4 * j + 1] += x.y; v[4 * j + 2] += x.z; v[4 * j + 3] += x.w;
      }
    }
    float* wr = g.W + row_off + c;
    if (g.Mom != nullptr) {
      float* mr = g.Mom + row_off + c;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float mm = g.mom_beta * mr[j] + v[j];
        mr[j] = mm;
        v[j] = mm;
      }
    }
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float w = wr[j] - v[j];
      v[j] = w;
      ss += w * w;
    }
    if (g.normalize) {
#pragma unroll
      for (int j = 0; j < 32; ++j) wr[j] = v[j];
    } else {
      __nv_bfloat16* br = g.Wb + row_off + c;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        wr[j] = v[j];
        br[j] = __float2bfloat16_rn(v[j]);
        if (g.Wlo != nullptr) g.Wlo[row_off + c + j] = __float2bfloat16_rn(v[j] - __bfloat162float(br[j]));
      }
    }
  }
  if (g.normalize && valid) {
    const float scale = 1.f / fmaxf(sqrtf(ss), g.norm_eps);
    float* wr = g.W + row_off;
    __nv_bfloat16* br = g.Wb + row_off;
#pragma unroll 4
    for (int c = 0; c < BN; ++c) {
      const float w = wr[c] * scale;
      wr[c] = w;
      const __nv_bfloat16 h = __float2bfloat16_rn(w);
      br[c] = h;
      if (g.Wlo != nullptr) g.Wlo[row_off + c] = __float2bfloat16_rn(w - __bfloat162float(h));
    }
  }
}

template <int BN, bool A_MN, bool B_MN, int STAGES>
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
  uint32_t* epi_flag = abort_flag + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_m = (g.M + 127) / 128, tiles_n = g.N / BN;
  const int n_tiles = tiles_m * tiles_n * g.splits * g.batch;
  const int total_k = g.k_steps * g.npairs;

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
    tmem_alloc(tmem_slot, 2 * BN);
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
  const uint32_t tmem = *tmem_slot;
  Waiter W{abort_flag, g.st, 100};

  if (warp == 0) {
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
        const int tm = t % tiles_m;
        const int tn = (t / tiles_m) % tiles_n;
        const int bs = t / (tiles_m * tiles_n);
        const int b = bs / g.splits, sp = bs % g.splits;
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
          } else {
            tma_load_3d(sa, &maps.a[p], &full[s], am, ak, b + g.a_b_off);
            tma_load_3d(sa + 8192, &maps.a[p], &full[s], am + 64, ak, b + g.a_b_off);
          }
          if (!B_MN) {
            tma_load_3d(sb, &maps.b[p], &full[s], bk, bn, b + g.b_b_off);
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
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const uint64_t ad = A_MN ? make_sdesc(sa + k4 * 2048, 8192, 1024)
                                     : make_sdesc(sa + k4 * 32, 16, 1024);
            const uint64_t bd = B_MN ? make_sdesc(sb + k4 * 2048, 8192, 1024)
                                     : make_sdesc(sb + k4 * 32, 16, 1024);
            mma_bf16(d, ad, bd, idesc, (kk | k4) != 0);
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
    // epilogue: warps 2..5 -> TMEM lane quadrants 2,3,0,1
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    uint32_t lt = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++lt) {
      const int tm = t % tiles_m;
      const int tn = (t / tiles_m) % tiles_n;
      const int bs = t / (tiles_m * tiles_n);
      const int b = bs / g.splits, sp = bs % g.splits;
      const uint32_t ab = lt & 1;
      if (!W.wait(&afull[ab], (lt >> 1) & 1, 4)) break;
      tc_fence_after();
      const int m = tm * 128 + row;
      const bool valid = m < g.M;
      const int orow = m + g.out_row_off;
      if (g.epi == 1) {
        epilogue_update<BN>(g, tmem + lane_base + ab * BN, b, sp, tm, m, valid, epi_flag);
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
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * BN);
  }
}

}  // namespace ttt
