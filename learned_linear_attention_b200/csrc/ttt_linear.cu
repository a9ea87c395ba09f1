// ttt_linear.cu -- linear fast weight trained on -<W k, v> == causal linear
// attention ("Test-Time Training with KV Binding Is Secretly Linear
// Attention", summary "B. Reformulación Teórica", "Formulación Paralela").
//
// Chunked form per (b, h), state S = W^T [dk, dv] in fp32:
//   O_c   = (Q_c K_c^T  o  causal mask) (diag(eta_c) V_c) + Q_c S_{c-1}
//   S_c   = S_{c-1} + K_c^T diag(eta_c) V_c
//
// Two kernels:
//  * ttt_linear_simt_kernel   -- exact fp32 FFMA on CUDA cores; any dk, dv <=
//    128, fp32 or bf16 inputs; honours the caller's chunk (capped at 32).
//  * ttt_linear_umma_kernel   -- bf16, dk = dv = 64, one persistent CTA per
//    (b, h) chain walking 128-token tiles: TMA loads Q/K/V, tcgen05 MMAs with
//    fp32 accumulators in TMEM, the fp32 state S resident in TMEM for the
//    whole sequence, causal mask and per-token lr applied by the epilogue
//    warps between the MMAs.
#include "common.cuh"
#include <algorithm>

#include "kernels.h"

namespace ttt {

// =====================================================================
// CUDA-core kernel
// =====================================================================
constexpr int SIMT_THREADS = 256;
constexpr int SIMT_MAXC = 32;

template <typename Tin>
TTT_DEVICE_INLINE float load_in(const Tin* p, size_t i);
template <>
TTT_DEVICE_INLINE float load_in<float>(const float* p, size_t i) { return p[i]; }
template <>
TTT_DEVICE_INLINE float load_in<__nv_bfloat16>(const __nv_bfloat16* p, size_t i) {
  return __bfloat162float(p[i]);
}

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(SIMT_THREADS)
    ttt_linear_simt_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                           const Tin* __restrict__ v, const float* __restrict__ lr,
                           float* __restrict__ S, Tout* __restrict__ out, int N, int dk, int dv,
                           int C, int include_diag, int bidir, const float* __restrict__ out_scale,
                           float out_mul) {
  extern __shared__ float sm[];
  float* Ss = sm;                       // [dk][dv]
  float* Qs = Ss + dk * dv;             // [C][dk]
  float* Ks = Qs + SIMT_MAXC * dk;      // [C][dk]
  float* Vs = Ks + SIMT_MAXC * dk;      // [C][dv]  (pre-scaled by eta)
  float* Ps = Vs + SIMT_MAXC * dv;      // [C][C]
  const int bh = blockIdx.x;
  const size_t qk_base = (size_t)bh * N * dk;
  const size_t v_base = (size_t)bh * N * dv;
  float* Sg = S + (size_t)bh * dk * dv;

  for (int i = threadIdx.x; i < dk * dv; i += blockDim.x) Ss[i] = Sg[i];
  __syncthreads();

  // Bidirectional order: every token's update first (S += K^T diag(eta) V
  // chunk by chunk), then the reads below with the final S and no P term.
  for (int t0 = 0; bidir && t0 < N; t0 += C) {
    const int Cc = min(C, N - t0);
    for (int i = threadIdx.x; i < Cc * dk; i += blockDim.x)
      Ks[i] = load_in(k, qk_base + (size_t)t0 * dk + i);
    for (int i = threadIdx.x; i < Cc * dv; i += blockDim.x) {
      const int t = i / dv;
      Vs[i] = lr[(size_t)bh * N + t0 + t] * load_in(v, v_base + (size_t)t0 * dv + i);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < dk * dv; e += blockDim.x) {
      const int r = e / dv, c = e % dv;
      float acc = Ss[e];
      for (int j = 0; j < Cc; ++j) acc = fmaf(Ks[j * dk + r], Vs[j * dv + c], acc);
      Ss[e] = acc;
    }
    __syncthreads();
  }

  for (int t0 = 0; t0 < N; t0 += C) {
    const int Cc = min(C, N - t0);
    for (int i = threadIdx.x; i < Cc * dk; i += blockDim.x) {
      Qs[i] = load_in(q, qk_base + (size_t)t0 * dk + i);
      Ks[i] = load_in(k, qk_base + (size_t)t0 * dk + i);
    }
    for (int i = threadIdx.x; i < Cc * dv; i += blockDim.x) {
      const int t = i / dv;
      Vs[i] = lr[(size_t)bh * N + t0 + t] * load_in(v, v_base + (size_t)t0 * dv + i);
    }
    __syncthreads();
    // P[i][j] = q_i . k_j for j <= i (j < i without the diagonal); no
    // within-chunk term in bidirectional order (S already holds every update)
    for (int e = threadIdx.x; e < Cc * Cc; e += blockDim.x) {
      const int i = e / Cc, j = e % Cc;
      float acc = 0.f;
      if (!bidir && (j < i || (include_diag && j == i))) {
        for (int r = 0; r < dk; ++r) acc = fmaf(Qs[i * dk + r], Ks[j * dk + r], acc);
      }
      Ps[i * SIMT_MAXC + j] = acc;
    }
    __syncthreads();
    // out_i = sum_j P[i][j] (eta_j v_j) + S^T q_i
    for (int e = threadIdx.x; e < Cc * dv; e += blockDim.x) {
      const int i = e / dv, c = e % dv;
      float acc = 0.f;
      for (int r = 0; r < dk; ++r) acc = fmaf(Qs[i * dk + r], Ss[r * dv + c], acc);
      for (int j = 0; j < Cc; ++j) acc = fmaf(Ps[i * SIMT_MAXC + j], Vs[j * dv + c], acc);
      if (out_scale) acc *= out_mul * out_scale[(size_t)bh * N + t0 + i];
      out[v_base + (size_t)(t0 + i) * dv + c] = static_cast<Tout>(acc);
    }
    __syncthreads();
    // S += K^T diag(eta) V
    for (int e = threadIdx.x; !bidir && e < dk * dv; e += blockDim.x) {
      const int r = e / dv, c = e % dv;
      float acc = Ss[e];
      for (int j = 0; j < Cc; ++j) acc = fmaf(Ks[j * dk + r], Vs[j * dv + c], acc);
      Ss[e] = acc;
    }
    __syncthreads();
  }
  for (int i = threadIdx.x; i < dk * dv; i += blockDim.x) Sg[i] = Ss[i];
}

size_t ttt_linear_simt_smem(int dk, int dv) {
  return sizeof(float) *
         ((size_t)dk * dv + 2 * SIMT_MAXC * dk + SIMT_MAXC * dv + SIMT_MAXC * SIMT_MAXC);
}

int launch_ttt_linear_simt(const LinearLaunch& L, cudaStream_t stream) {
  const int C = L.chunk < SIMT_MAXC ? L.chunk : SIMT_MAXC;
  const size_t smem = ttt_linear_simt_smem(L.dk, L.dv);
  dim3 grid(L.B * L.H), block(SIMT_THREADS);
#define TTT_SIMT_LAUNCH(TI, TO)                                                              \
  do {                                                                                       \
    auto kfn = ttt_linear_simt_kernel<TI, TO>;                                               \
    if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != \
        cudaSuccess)                                                                         \
      return -1;                                                                             \
    prof_before(K_LIN_SIMT, stream);                                                         \
    kfn<<<grid, block, smem, stream>>>((const TI*)L.q, (const TI*)L.k, (const TI*)L.v, L.lr, \
                                       L.S, (TO*)L.out, L.N, L.dk, L.dv, C, L.include_diag,   \
                                       L.bidir, L.out_scale, L.out_mul);                      \
    prof_after(K_LIN_SIMT, stream);                                                          \
  } while (0)
  if (L.in_bf16) {
    if (L.out_bf16) TTT_SIMT_LAUNCH(__nv_bfloat16, __nv_bfloat16);
    else TTT_SIMT_LAUNCH(__nv_bfloat16, float);
  } else {
    if (L.out_bf16) TTT_SIMT_LAUNCH(float, __nv_bfloat16);
    else TTT_SIMT_LAUNCH(float, float);
  }
#undef TTT_SIMT_LAUNCH
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

// =====================================================================
// tcgen05 kernel, bf16, dk = dv = 64
// =====================================================================
namespace lin {
constexpr int T = 128;          // tokens per tile
constexpr int D = 64;           // dk = dv
constexpr int NUM_EPI_WARPS = 8;
constexpr int THREADS = (2 + NUM_EPI_WARPS) * 32;
constexpr uint32_t TILE_BYTES = T * D * 2;          // 16 KB (Q, K, V, eta*V tiles)
constexpr uint32_t STAGE_BYTES = 3 * TILE_BYTES;    // Q, K, V
// Three Q/K/V stages keep about two tiles of loads in flight per SM; the
// masked P and eta V operands are single-buffered: the epilogue builds the
// next tile's in registers while this tile's products run and stores them
// once those products are done.
constexpr int STAGES = 3;
constexpr uint32_t OFF_STAGE = 0;
constexpr uint32_t OFF_PT = OFF_STAGE + STAGES * STAGE_BYTES;      // 32 KB (masked P, bf16)
constexpr uint32_t OFF_EV = OFF_PT + 2 * TILE_BYTES;              // 16 KB (eta*V, bf16)
constexpr uint32_t OFF_SB = OFF_EV + TILE_BYTES;                  // 8 KB (S, bf16)
constexpr uint32_t OFF_BAR = OFF_SB + D * D * 2;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;             // + alignment slack
// TMEM columns
constexpr uint32_t TM_P0 = 0, TM_P1 = 128, TM_O0 = 256, TM_S = 320, TM_O1 = 384, TM_COLS = 512;
}  // namespace lin

struct LinUmmaArgs {
  const float* lr;
  float* S;           // [BH][64][64] fp32, in/out
  void* out;          // [BH][N][64]
  int N;
  int include_diag;
  int out_bf16;
  DevStatus st;
  // Sequence split: CTA (bh, p) takes tiles [p seg_tiles, (p + 1) seg_tiles)
  // of head bh.  With P > 1 its start state is S0 (copied to seg_state by
  // the pre-pass) plus the state increments of the R units of every
  // earlier segment, and only the last segment writes S.
  int P, R, seg_tiles;
  const float* seg_state;   // [BH][1 + (P - 1) R][64][64]: S0, then the units' increments
  const float* out_scale;   // nullable: output row t is multiplied by out_mul * out_scale[bh][t]
  float out_mul;
  // Reads only: out = Q S with S fixed (the bidirectional order, after the
  // state pass has summed every update into S).  Only Q is loaded, there is
  // no masked term and no state update, every segment starts from S and
  // none writes it back.
  int read_only;
};

__global__ void __launch_bounds__(lin::THREADS, 1)
    ttt_linear_umma_kernel(const __grid_constant__ CUtensorMap mapQ,
                           const __grid_constant__ CUtensorMap mapK,
                           const __grid_constant__ CUtensorMap mapV, LinUmmaArgs a) {
  using namespace lin;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);   // [STAGES]
  uint64_t* empty = full + STAGES;                                  // [STAGES]
  uint64_t* pfull = empty + STAGES;                                 // [2]: per P buffer
  uint64_t* ops = pfull + 2;                                        // [1]
  uint64_t* ofull = ops + 1;                                        // [1]
  uint64_t* fin = ofull + 1;                                        // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x / a.P, seg = blockIdx.x % a.P;
  const int t_first = seg * a.seg_tiles;   // first tile of this CTA's segment
  const int n_tiles = max(0, min(a.seg_tiles, (a.N + T - 1) / T - t_first));

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) mbar_init(&pfull[s], 1);
    mbar_init(ops, NUM_EPI_WARPS * 32);
    mbar_init(ofull, 1);
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mapQ);
    tma_prefetch_desc(&mapK);
    tma_prefetch_desc(&mapV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  Waiter W{abort_flag, a.st, 0};

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i % STAGES;
        if (i >= STAGES && !W.wait(&empty[s], ((i / STAGES) - 1) & 1, 1)) break;
        uint8_t* st = smem + OFF_STAGE + s * STAGE_BYTES;
        mbar_arrive_expect_tx(&full[s], a.read_only ? TILE_BYTES : STAGE_BYTES);
        tma_load_3d(st, &mapQ, &full[s], 0, (t_first + i) * T, bh);
        if (!a.read_only) {
          tma_load_3d(st + TILE_BYTES, &mapK, &full[s], 0, (t_first + i) * T, bh);
          tma_load_3d(st + 2 * TILE_BYTES, &mapV, &full[s], 0, (t_first + i) * T, bh);
        }
        issued = i + 1;
      }
      if (W.aborted()) {  // drain the copies still in flight into our smem
        for (int i = issued - STAGES < 0 ? 0 : issued - STAGES; i < issued; ++i)
          W.drain(&full[i % STAGES], (i / STAGES) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // It polls the next tile's QK^T product (its Q/K tiles landed, its P
    // buffer was read by the epilogue two tiles back) and the current tile's
    // O and S products (the epilogue staged its operands) and issues
    // whichever can go, so the O/S chain never waits for a tile load.
    if (lane == 0 && n_tiles > 0) {
      const uint32_t id_qk = make_idesc(128, 128, false, false);
      const uint32_t id_o = make_idesc(128, 64, false, true);
      const uint32_t id_s = make_idesc(64, 64, true, true);
      const uint32_t pt_base = smem_u32(smem + OFF_PT);
      const uint32_t ev_base = smem_u32(smem + OFF_EV);
      const uint32_t sb_base = smem_u32(smem + OFF_SB);
      // descriptors: per-stage bases, advanced by constant byte offsets
      const uint64_t dq0 = make_sdesc(smem_u32(smem + OFF_STAGE), 16, 1024);
      const uint64_t dk_mn0 = make_sdesc(smem_u32(smem + OFF_STAGE) + TILE_BYTES, 8192, 1024);
      const uint64_t dpt = make_sdesc(pt_base, 16, 1024);
      const uint64_t dev_mn = make_sdesc(ev_base, 8192, 1024);
      const uint64_t dsb = make_sdesc(sb_base, 8192, 1024);
      auto issue_p = [&](int i) {
        tc_fence_after();
        const int s = i % STAGES, pb = i & 1;
        const uint64_t dq = sdesc_add(dq0, s * STAGE_BYTES), dk = sdesc_add(dq, TILE_BYTES);
        if (!a.read_only) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmem + (pb ? TM_P1 : TM_P0), sdesc_add(dq, kk * 32), sdesc_add(dk, kk * 32),
                     id_qk, kk > 0);
        }
        mma_commit(&pfull[pb]);   // read-only: only tells the epilogue the tile is in
      };
      auto issue_o = [&](int i) {
        tc_fence_after();
        const int s = i % STAGES;
        const uint64_t dq = sdesc_add(dq0, s * STAGE_BYTES);
        const uint64_t dk = sdesc_add(dk_mn0, s * STAGE_BYTES);
        // O = mask(P) (eta V): K = 128 keys, two 64-key atoms of the P tile.
        // O alternates between two TMEM buffers so the epilogue can store the
        // previous tile's O while this tile's products run.
        const uint32_t tm_o = (i & 1) ? TM_O1 : TM_O0;
        if (!a.read_only) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16(tmem + tm_o, sdesc_add(dpt, (kk >> 2) * TILE_BYTES + (kk & 3) * 32),
                     sdesc_add(dev_mn, kk * 2048), id_o, kk > 0);
        }
        // O += Q S_{prev}
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + tm_o, sdesc_add(dq, kk * 32), sdesc_add(dsb, kk * 2048), id_o,
                   (a.read_only && kk == 0) ? 0u : 1u);
        // S += K^T (eta V)   (M = 64: rows live in lanes 0-15 of each quadrant)
        if (!a.read_only) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16(tmem + TM_S, sdesc_add(dk, kk * 2048), sdesc_add(dev_mn, kk * 2048), id_s, 1);
        }
        mma_commit(ofull);
        mma_commit(&empty[s]);
      };
      int np = 0, no = 0;   // QK^T products / O and S products issued
      uint64_t t_idle = 0;
      uint32_t spins = 0;
      while (no < n_tiles) {
        bool prog = false;
        if (no < np && mbar_test(ops, no & 1)) {
          issue_o(no);
          ++no;
          prog = true;
        }
        if (np < n_tiles && np <= no + 1 && mbar_test(&full[np % STAGES], (np / STAGES) & 1)) {
          issue_p(np);
          ++np;
          prog = true;
        }
        if (prog) {
          spins = 0;
          t_idle = 0;
          continue;
        }
        // plain polling: a sleep here put its wake-up on the per-tile chain
        if ((++spins & 255u) == 0u) {   // bounded: give up after the wait timeout
          if (W.aborted()) break;
          const uint64_t now = globaltimer_ns();
          if (t_idle == 0) t_idle = now;
          else if (now - t_idle > W.st.timeout_ns) { W.fail(3); break; }
        }
      }
    }
    if (lane == 0) {  // every MMA issued by this thread completes before teardown
      mma_commit(fin);
      W.drain(fin, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q4 = warp & 3;                  // TMEM lane quadrant
    const int hf = (warp - 2) >> 2;           // column half
    const int r = q4 * 32 + lane;             // row of the tile
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    float* Sg = a.S + (size_t)bh * D * D;
    const float* lrg = a.lr + (size_t)bh * a.N;
    uint8_t* sb = smem + OFF_SB;
    // S rows of the M = 64 accumulator: lanes 0-15 of quadrant q4 hold rows 16*q4 + lane
    const bool s_owner = lane < 16;
    const int srow = q4 * 16 + lane;
    {
      float vals[32];
      if (a.P == 1 || a.read_only) {
#pragma unroll
        for (int j = 0; j < 32; ++j) vals[j] = s_owner ? Sg[srow * D + hf * 32 + j] : 0.f;
      } else {   // S0 + the increments of the earlier segments' units, in order
        const int nu = 1 + seg * a.R;
        const float* ss = a.seg_state + (size_t)bh * (1 + (a.P - 1) * a.R) * D * D + srow * D + hf * 32;
#pragma unroll
        for (int j = 0; j < 32; ++j) vals[j] = 0.f;
        for (int u = 0; u < nu; ++u)
#pragma unroll
          for (int j = 0; j < 32; ++j) vals[j] += s_owner ? ss[(size_t)u * D * D + j] : 0.f;
      }
      tmem_st16(tmem + lane_base + TM_S + hf * 32, vals);
      tmem_st16(tmem + lane_base + TM_S + hf * 32 + 16, vals + 16);
      if (s_owner) {
#pragma unroll
        for (int j = 0; j < 32; j += 8)
          st_shared_v4(smem_u32(sb) + sw128_offset(srow, hf * 32 + j),
                       pack_bf16x2(vals[j], vals[j + 1]), pack_bf16x2(vals[j + 2], vals[j + 3]),
                       pack_bf16x2(vals[j + 4], vals[j + 5]), pack_bf16x2(vals[j + 6], vals[j + 7]));
      }
    }
    auto store_out = [&](int tile) {
      const int t = (t_first + tile) * T + r;
      float o[32];
      tmem_ld32(tmem + lane_base + ((tile & 1) ? TM_O1 : TM_O0) + hf * 32, o);
      if (t < a.N) {
        if (a.out_scale) {
          const float f = a.out_mul * a.out_scale[(size_t)bh * a.N + t];
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] *= f;
        }
        const size_t base = ((size_t)bh * a.N + t) * D + hf * 32;
        if (a.out_bf16) {
          uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) + base);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            dst[j] = make_uint4(pack_bf16x2(o[8 * j], o[8 * j + 1]), pack_bf16x2(o[8 * j + 2], o[8 * j + 3]),
                                pack_bf16x2(o[8 * j + 4], o[8 * j + 5]), pack_bf16x2(o[8 * j + 6], o[8 * j + 7]));
        } else {
          float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + base);
#pragma unroll
          for (int j = 0; j < 8; ++j) dst[j] = make_float4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
        }
      }
    };
    bool ok = true;
    for (int i = 0; a.read_only && i < n_tiles; ++i) {
      // reads only: the operands (Q in the stage, S in shared memory) are in
      // place; keep the O buffers' order and store the previous tile's O
      if (!W.wait(&pfull[i & 1], (i >> 1) & 1, 5)) { ok = false; break; }
      if (i > 0 && !W.wait(ofull, (i - 1) & 1, 6)) { ok = false; break; }
      tc_fence_after();
      // the bf16 S operand this thread stored before the loop must be visible
      // to the tensor core (async proxy) before the first product reads it
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(ops);
      if (i > 0) store_out(i - 1);
    }
    for (int i = 0; !a.read_only && i < n_tiles; ++i) {
      const int s = i % STAGES, pb = i & 1;
      if (!W.wait(&pfull[pb], (i >> 1) & 1, 5)) { ok = false; break; }
      tc_fence_after();
      const int t = (t_first + i) * T + r;
      const float eta = (t < a.N) ? lrg[t] : 0.f;
      // eta * V of this row's 32 columns (bf16 pairs), from the stage
      uint32_t evr[16];
      {
        const uint32_t vsrc = smem_u32(smem + OFF_STAGE + s * STAGE_BYTES + 2 * TILE_BYTES);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t w0, w1, w2, w3;
          ld_shared_v4(vsrc + sw128_offset(r, hf * 32 + 8 * j), w0, w1, w2, w3);
          evr[4 * j] = pack_bf16x2(eta * bf16lo(w0), eta * bf16hi(w0));
          evr[4 * j + 1] = pack_bf16x2(eta * bf16lo(w1), eta * bf16hi(w1));
          evr[4 * j + 2] = pack_bf16x2(eta * bf16lo(w2), eta * bf16hi(w2));
          evr[4 * j + 3] = pack_bf16x2(eta * bf16lo(w3), eta * bf16hi(w3));
        }
      }
      // masked P of this row's 64 keys hf*64 .. hf*64+63 (bf16 pairs)
      uint32_t pr[32];
      {
        const uint32_t pcol = (pb ? TM_P1 : TM_P0) + hf * 64;
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          float p[32];
          tmem_ld32(tmem + lane_base + pcol + h2 * 32, p);
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const int key = hf * 64 + h2 * 32 + j;
            const bool k0 = a.include_diag ? (key <= r) : (key < r);
            const bool k1 = a.include_diag ? (key + 1 <= r) : (key + 1 < r);
            pr[h2 * 16 + j / 2] = pack_bf16x2(k0 ? p[j] : 0.f, k1 ? p[j + 1] : 0.f);
          }
        }
      }
      // the previous tile's products are done with the single P, eta V and
      // S operand buffers; S after tile i-1 becomes tile i's operand
      float sv[32];
      if (i > 0) {
        if (!W.wait(ofull, (i - 1) & 1, 6)) { ok = false; break; }
        tc_fence_after();
        tmem_ld32(tmem + lane_base + TM_S + hf * 32, sv);
      }
      {
        const uint32_t evdst = smem_u32(smem + OFF_EV);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          st_shared_v4(evdst + sw128_offset(r, hf * 32 + 8 * j), evr[4 * j], evr[4 * j + 1],
                       evr[4 * j + 2], evr[4 * j + 3]);
        const uint32_t pdst = smem_u32(smem + OFF_PT + hf * TILE_BYTES);
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
          for (int j = 0; j < 32; j += 8)
            st_shared_v4(pdst + sw128_offset(r, h2 * 32 + j), pr[h2 * 16 + j / 2], pr[h2 * 16 + j / 2 + 1],
                         pr[h2 * 16 + j / 2 + 2], pr[h2 * 16 + j / 2 + 3]);
      }
      if (i > 0 && s_owner) {
#pragma unroll
        for (int j = 0; j < 32; j += 8)
          st_shared_v4(smem_u32(sb) + sw128_offset(srow, hf * 32 + j),
                       pack_bf16x2(sv[j], sv[j + 1]), pack_bf16x2(sv[j + 2], sv[j + 3]),
                       pack_bf16x2(sv[j + 4], sv[j + 5]), pack_bf16x2(sv[j + 6], sv[j + 7]));
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(ops);
      // the previous tile's output leaves the critical path: stored while
      // this tile's products run (its TMEM buffer is next written by tile i+1)
      if (i > 0) store_out(i - 1);
    }
    if (ok && n_tiles > 0 && W.wait(ofull, (n_tiles - 1) & 1, 7)) {
      tc_fence_after();
      store_out(n_tiles - 1);
      float sv[32];
      tmem_ld32(tmem + lane_base + TM_S + hf * 32, sv);
      if (s_owner && seg == a.P - 1 && !a.read_only) {
#pragma unroll
        for (int j = 0; j < 32; ++j) Sg[srow * D + hf * 32 + j] = sv[j];
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

// =====================================================================
// sequence split: state increments of the earlier segments
// =====================================================================
// Causal linear attention is a prefix scan of S (the state after a token is
// S0 plus the sum of eta k v^T before it), so a head's sequence can be cut
// into segments that run on different SMs once each knows its start state.
// This pre-pass forms, per unit of tiles of every segment but the last,
// dS_u = sum_t k_t^T (eta_t v_t) with the same bf16 operands and fp32
// tensor-core accumulation as the main kernel, and copies S0 beside them.
namespace lss {
constexpr int T = 128, D = 64;
constexpr int EPI_WARPS = 4;
constexpr int THREADS = (2 + EPI_WARPS) * 32;
constexpr uint32_t TILE = T * D * 2;                 // 16 KB
constexpr uint32_t STAGE = 2 * TILE;                 // K, V
constexpr int STAGES = 5;                            // ~128 KB of loads in flight per SM
constexpr uint32_t OFF_EV = STAGES * STAGE;          // 2 x 16 KB (eta V, bf16)
constexpr uint32_t OFF_BAR = OFF_EV + 2 * TILE;
constexpr uint32_t SMEM = OFF_BAR + 256 + 1024;
constexpr uint32_t TM_S = 0, TM_COLS = 64;
}  // namespace lss

struct SegStateArgs {
  const float* lr;
  const float* S0;    // [BH][64][64]
  float* seg_state;   // [BH][1 + U][64][64]
  int N, U, R, seg_tiles, unit_tiles;
  DevStatus st;
};

__global__ void __launch_bounds__(lss::THREADS, 1)
    ttt_linear_segstate_kernel(const __grid_constant__ CUtensorMap mapK,
                               const __grid_constant__ CUtensorMap mapV, SegStateArgs a) {
  using namespace lss;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);   // [STAGES]
  uint64_t* empty = full + STAGES;                                  // [STAGES]
  uint64_t* evfull = empty + STAGES;                                // [2]
  uint64_t* evempty = evfull + 2;                                   // [2]
  uint64_t* fin = evempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x / a.U, u = blockIdx.x % a.U;
  const int p = u / a.R, rr = u % a.R;
  const int total = (a.N + T - 1) / T;
  const int t0 = p * a.seg_tiles + rr * a.unit_tiles;
  const int t1 = min(min(t0 + a.unit_tiles, (p + 1) * a.seg_tiles), total);
  const int nt = max(0, t1 - t0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&evfull[s], EPI_WARPS * 32);
      mbar_init(&evempty[s], 1);
    }
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mapK);
    tma_prefetch_desc(&mapV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  Waiter W{abort_flag, a.st, 600};
  float* out = a.seg_state + (size_t)bh * (1 + a.U) * D * D;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nt; ++i) {
        const int s = i % STAGES;
        if (i >= STAGES && !W.wait(&empty[s], ((i / STAGES) - 1) & 1, 1)) break;
        uint8_t* st = smem + s * STAGE;
        mbar_arrive_expect_tx(&full[s], STAGE);
        tma_load_3d(st, &mapK, &full[s], 0, (t0 + i) * T, bh);
        tma_load_3d(st + TILE, &mapV, &full[s], 0, (t0 + i) * T, bh);
        issued = i + 1;
      }
      if (W.aborted())
        for (int i = issued > STAGES ? issued - STAGES : 0; i < issued; ++i)
          W.drain(&full[i % STAGES], (i / STAGES) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_s = make_idesc(64, 64, true, true);
      for (int i = 0; i < nt; ++i) {
        const int s = i % STAGES, e = i & 1;
        if (!W.wait(&evfull[e], (i >> 1) & 1, 2)) break;
        tc_fence_after();
        const uint32_t ks = smem_u32(smem + s * STAGE);
        const uint32_t ev = smem_u32(smem + OFF_EV + e * TILE);
        // S += K^T (eta V): M = 64 (d), K = 128 tokens, N = 64
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16(tmem + TM_S, make_sdesc(ks + kk * 2048, 8192, 1024),
                   make_sdesc(ev + kk * 2048, 8192, 1024), id_s, (i > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&empty[s]);
        mma_commit(&evempty[e]);
      }
      mma_commit(fin);
      W.drain(fin, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue: eta V
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;   // token row of the tile
    const float* lrg = a.lr + (size_t)bh * a.N;
    bool ok = true;
    for (int i = 0; i < nt; ++i) {
      const int s = i % STAGES, e = i & 1;
      const int t = (t0 + i) * T + r;
      const float eta = t < a.N ? lrg[t] : 0.f;
      if (!W.wait(&full[s], (i / STAGES) & 1, 3)) { ok = false; break; }
      if (i >= 2 && !W.wait(&evempty[e], ((i >> 1) - 1) & 1, 4)) { ok = false; break; }
      const uint32_t vsrc = smem_u32(smem + s * STAGE + TILE);
      const uint32_t evdst = smem_u32(smem + OFF_EV + e * TILE);
#pragma unroll
      for (int j = 0; j < 64; j += 8) {
        const uint32_t off = sw128_offset(r, j);
        uint32_t w0, w1, w2, w3;
        ld_shared_v4(vsrc + off, w0, w1, w2, w3);
        st_shared_v4(evdst + off, pack_bf16x2(eta * bf16lo(w0), eta * bf16hi(w0)),
                     pack_bf16x2(eta * bf16lo(w1), eta * bf16hi(w1)),
                     pack_bf16x2(eta * bf16lo(w2), eta * bf16hi(w2)),
                     pack_bf16x2(eta * bf16lo(w3), eta * bf16hi(w3)));
      }
      fence_async_smem();
      mbar_arrive(&evfull[e]);
    }
    // increment of the unit (rows of the M = 64 accumulator: lanes 0-15 of
    // quadrant q4 hold rows 16 q4 + lane)
    if (ok && W.wait(fin, 0, 5)) {
      tc_fence_after();
      const int srow = q4 * 16 + lane;
      float sv[32];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        tmem_ld32(tmem + ((uint32_t)(q4 * 32) << 16) + TM_S + h * 32, sv);
        if (lane < 16) {
          float* dst = out + (size_t)(1 + u) * D * D + srow * D + h * 32;
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4*>(dst + j) =
                nt > 0 ? make_float4(sv[j], sv[j + 1], sv[j + 2], sv[j + 3]) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
    }
    // the first unit of the head also copies S0 beside the increments
    if (u == 0) {
      const float4* src = reinterpret_cast<const float4*>(a.S0 + (size_t)bh * D * D);
      float4* dst = reinterpret_cast<float4*>(out);
      for (int k = threadIdx.x - 64; k < D * D / 4; k += EPI_WARPS * 32) dst[k] = src[k];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TM_COLS);
  }
}

// Segments per head P, units per segment R, tiles per segment and per unit.
// P fills the SMs with one CTA per (head, segment) (at least 8 tiles per
// segment); the pre-pass fills them again with (head, unit) CTAs.
LinearPlan ttt_linear_plan(int BH, int N, int sms) {
  LinearPlan pl{};
  const int total = (N + 127) / 128;
  pl.P = std::max(1, std::min(std::min(8, sms / std::max(1, BH)), total / 8));
  pl.seg_tiles = (total + pl.P - 1) / std::max(1, pl.P);
  if (pl.seg_tiles < 1) pl.seg_tiles = 1;
  pl.P = std::max(1, (total + pl.seg_tiles - 1) / pl.seg_tiles);
  pl.R = 1;
  if (pl.P > 1) pl.R = std::max(1, std::min(std::min(8, sms / (BH * (pl.P - 1))), pl.seg_tiles / 4));
  pl.unit_tiles = (pl.seg_tiles + pl.R - 1) / pl.R;
  pl.ws_floats = pl.P > 1 ? (size_t)BH * (1 + (size_t)(pl.P - 1) * pl.R) * 64 * 64 : 0;
  return pl;
}

// SMs of the current device
static int num_sms_current() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = 148;
  }
  return n;
}

int launch_ttt_linear_umma(const LinearLaunch& L, cudaStream_t stream) {
  CUtensorMap mq, mk, mv;
  const uint64_t BH = (uint64_t)L.B * L.H;
  if (make_tmap_bf16_3d(&mq, L.q, 64, L.N, BH, 64 * 2, (uint64_t)L.N * 64 * 2, 64, 128) ||
      make_tmap_bf16_3d(&mk, L.k, 64, L.N, BH, 64 * 2, (uint64_t)L.N * 64 * 2, 64, 128) ||
      make_tmap_bf16_3d(&mv, L.v, 64, L.N, BH, 64 * 2, (uint64_t)L.N * 64 * 2, 64, 128))
    return -1;
  LinearPlan pl = L.plan;
  if (pl.P > 1 && (L.seg_state == nullptr || L.seg_state_floats < pl.ws_floats)) {
    pl.P = 1;   // no room for the segment states: one CTA per head
    pl.seg_tiles = (L.N + 127) / 128;
  }
  LinUmmaArgs a{L.lr, L.S, L.out, L.N, L.include_diag, L.out_bf16, L.st,
                pl.P, pl.R, pl.seg_tiles, L.seg_state, L.out_scale, L.out_mul, 0};
  if (L.bidir) {
    // every update first: S <- S + sum over all tokens (state pass), then
    // reads only, in segments that all start from that S
    if (launch_ttt_linear_state_sum(L, num_sms_current(), stream) != 0) return -1;
    const int total = (L.N + 127) / 128;
    a.read_only = 1;
    a.P = std::max(1, std::min(total, num_sms_current() / (int)BH));
    a.seg_tiles = (total + a.P - 1) / a.P;
    a.P = (total + a.seg_tiles - 1) / a.seg_tiles;
    a.R = 1;
    pl.P = 1;   // no segment pre-pass
  }
  if (pl.P > 1) {
    SegStateArgs sa{L.lr, L.S, L.seg_state, L.N, (pl.P - 1) * pl.R, pl.R, pl.seg_tiles, pl.unit_tiles, L.st};
    static std::atomic<uint64_t> ss_attr{0};
    if (allow_dynamic_smem(ttt_linear_segstate_kernel, (int)lss::SMEM, ss_attr)) return -1;
    prof_before(K_LIN_SEG, stream);
    ttt_linear_segstate_kernel<<<dim3((unsigned)(BH * sa.U)), dim3(lss::THREADS), lss::SMEM, stream>>>(
        mk, mv, sa);
    prof_after(K_LIN_SEG, stream);
  }
  static std::atomic<uint64_t> attr{0};
  if (allow_dynamic_smem(ttt_linear_umma_kernel, (int)lin::SMEM_BYTES, attr)) return -1;
  prof_before(K_LIN_UMMA, stream);
  ttt_linear_umma_kernel<<<dim3((unsigned)(BH * a.P)), dim3(lin::THREADS), lin::SMEM_BYTES, stream>>>(
      mq, mk, mv, a);
  prof_after(K_LIN_UMMA, stream);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

// ---------------------------------------------------------------- state sum
namespace {
// Units of the whole-sequence pre-pass: enough (head, unit) CTAs to fill the
// SMs, at least 4 tiles per unit.
int state_sum_units(int BH, int N, int sms) {
  const int total = (N + 127) / 128;
  return std::max(1, std::min(std::min(8, sms / std::max(1, BH)), total / 4));
}

// S[bh] = seg[bh][0] + sum_u seg[bh][1 + u]  (slot 0 holds the start state)
__global__ void lin_state_sum_kernel(const float* __restrict__ seg, float* __restrict__ S, int BH,
                                     int U) {
  constexpr int DD = 64 * 64;
  const size_t n = (size_t)BH * DD;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (size_t)gridDim.x * blockDim.x) {
    const size_t bh = e / DD, i = e % DD;
    const float* p = seg + bh * (size_t)(1 + U) * DD + i;
    float acc = p[0];
    for (int u = 1; u <= U; ++u) acc += p[(size_t)u * DD];
    S[e] = acc;
  }
}
}  // namespace

size_t ttt_linear_state_sum_floats(int BH, int N, int sms) {
  return (size_t)BH * (1 + state_sum_units(BH, N, sms)) * 64 * 64;
}

int launch_ttt_linear_state_sum(const LinearLaunch& L, int sms, cudaStream_t stream) {
  const int BH = L.B * L.H;
  const int U = state_sum_units(BH, L.N, sms);
  if (L.seg_state == nullptr || L.seg_state_floats < ttt_linear_state_sum_floats(BH, L.N, sms))
    return -1;
  CUtensorMap mk, mv;
  if (make_tmap_bf16_3d(&mk, L.k, 64, L.N, BH, 64 * 2, (uint64_t)L.N * 64 * 2, 64, 128) ||
      make_tmap_bf16_3d(&mv, L.v, 64, L.N, BH, 64 * 2, (uint64_t)L.N * 64 * 2, 64, 128))
    return -1;
  const int total = (L.N + 127) / 128;
  // one segment of `total` tiles split into U units
  SegStateArgs sa{L.lr, L.S, L.seg_state, L.N, U, U, total, (total + U - 1) / U, L.st};
  static std::atomic<uint64_t> attr{0};
  if (allow_dynamic_smem(ttt_linear_segstate_kernel, (int)lss::SMEM, attr)) return -1;
  prof_before(K_LIN_SEG, stream);
  ttt_linear_segstate_kernel<<<dim3((unsigned)(BH * U)), dim3(lss::THREADS), lss::SMEM, stream>>>(
      mk, mv, sa);
  prof_after(K_LIN_SEG, stream);
  const size_t n = (size_t)BH * 64 * 64;
  prof_before(K_LIN_BWD_EW, stream);
  lin_state_sum_kernel<<<(unsigned)std::min<size_t>((n + 255) / 256, 148 * 8), 256, 0, stream>>>(
      L.seg_state, L.S, BH, U);
  prof_after(K_LIN_BWD_EW, stream);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace ttt
