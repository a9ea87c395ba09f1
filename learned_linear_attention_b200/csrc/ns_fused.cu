// ns_fused.cu -- the Newton-Schulz iteration of the Muon update as one fused,
// batched small-matrix kernel ("Test-Time Training Done Right" review,
// "Memoria no lineal y atención local": Muon orthogonalises each weight's
// gradient with Newton-Schulz iterations).
//
// For every matrix X of the batch (the three weights of every head, in the
// wide orientation r x c, r <= c) and each of `steps` quintic steps
//   phase 0:  A  = X X^T                      (r x r, contraction over c)
//   phase 1:  B  = c A A + b A                (r x r, contraction over r)
//   phase 2:  X <- B X + a X                  (r x c, contraction over r)
// All 3 * steps phases run in one persistent launch: every CTA walks the
// 128 x 128 output tiles of a phase (TMA loads, tcgen05 MMAs with fp32
// accumulators in TMEM, epilogue from TMEM), and the phases are separated by
// a grid-wide barrier on one monotone counter (a phase's outputs are the next
// phase's operands).  The launch is cooperative, so every CTA is resident
// and the barrier can complete; every wait on it is bounded.  X, A and B
// stay in L2 between phases (six 384 x 768 matrices: 3.5 MB of fp32 X).
//
// Operands are bf16 with fp32 accumulation; in split-operand mode every
// operand is carried as hi + lo bf16 parts and each product is the three
// products hi*hi + hi*lo + lo*hi.  X is kept in fp32 as well (its update is
// X <- BX + aX in fp32), and each phase writes the bf16 copies the next one
// reads.
#include <algorithm>

#include "gemm.cuh"
#include "kernels.h"

namespace ttt {

namespace nsf {
constexpr int BN = 128, STAGES = 4;
constexpr uint32_t A_BYTES = 128 * 64 * 2, B_BYTES = BN * 64 * 2;
constexpr uint32_t STAGE = A_BYTES + B_BYTES;
constexpr uint32_t BAR_OFF = STAGES * STAGE;
constexpr uint32_t SMEM = BAR_OFF + 256 + 1024;
constexpr int THREADS = 192;
}  // namespace nsf

// One phase of one step parity: C = alpha * sum_p A_p B_p^T + beta * Cin.
struct NsPhase {
  CUtensorMap a[3], b[3];
  int M, N, batch, k_steps, npairs, b_mn;
  float alpha, beta;
  const float* cin;          // [batch][M][ldc] (beta != 0)
  long long cin_bs;
  int ldc;
  float* o32;                // nullable
  long long o32_bs;
  int ld32;
  __nv_bfloat16* o16;        // hi part (bf16 copy)
  __nv_bfloat16* o16lo;      // lo part (nullable)
  long long o16_bs;
  int ld16;
};
struct NsFusedParams {
  NsPhase ph[3][2];          // [kind][step parity]
  int steps;
  unsigned* counter;         // zero at launch
  DevStatus st;
};

// the epilogue warps (threads 64..191) only
TTT_DEVICE_INLINE void epilogue_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__global__ void __launch_bounds__(nsf::THREADS, 1)
    ns_fused_kernel(const __grid_constant__ NsFusedParams P) {
  using namespace nsf;
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
  const int nph = 3 * P.steps;
  const unsigned G = gridDim.x;

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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  Waiter W{abort_flag, P.st, 700};

  auto phase = [&](int p) -> const NsPhase& { return P.ph[p % 3][(p / 3) & 1]; };
  auto tiles_of = [&](const NsPhase& ph) { return ((ph.M + 127) / 128) * (ph.N / BN) * ph.batch; };
  auto decode = [&](const NsPhase& ph, int t, int& tm, int& tn, int& b) {
    const int tiles_m = (ph.M + 127) / 128, tiles_n = ph.N / BN;
    tm = t % tiles_m;
    tn = (t / tiles_m) % tiles_n;
    b = t / (tiles_m * tiles_n);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int p = 0; ok && p < nph; ++p) {
        const NsPhase& ph = phase(p);
        // the previous phase's outputs (written by every CTA's epilogue
        // through the generic proxy) are this phase's TMA operands
        if (p > 0) {
          if (!grid_wait(P.counter, (unsigned)p * G, W, 1)) { ok = false; break; }
          fence_proxy_async_global();
        }
        const int total_k = ph.k_steps * ph.npairs;
        for (int t = blockIdx.x; ok && t < tiles_of(ph); t += gridDim.x) {
          int tm, tn, b;
          decode(ph, t, tm, tn, b);
          for (int kk = 0; kk < total_k; ++kk, ++it) {
            const int pr = kk / ph.k_steps, ks = kk % ph.k_steps;
            const uint32_t s = it % STAGES;
            if (it >= (uint32_t)STAGES && !W.wait(&empty[s], ((it / STAGES) - 1) & 1, 2)) {
              ok = false;
              break;
            }
            uint8_t* sa = smem + s * STAGE;
            uint8_t* sb = sa + A_BYTES;
            mbar_arrive_expect_tx(&full[s], STAGE);
            tma_load_3d(sa, &ph.a[pr], &full[s], ks * 64, tm * 128, b);
            if (!ph.b_mn) {
              tma_load_3d(sb, &ph.b[pr], &full[s], ks * 64, tn * BN, b);
            } else {
              tma_load_3d(sb, &ph.b[pr], &full[s], tn * BN, ks * 64, b);
              tma_load_3d(sb + 8192, &ph.b[pr], &full[s], tn * BN + 64, ks * 64, b);
            }
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
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, lt = 0;
      bool ok = true;
      for (int p = 0; ok && p < nph; ++p) {
        const NsPhase& ph = phase(p);
        const uint32_t idesc = make_idesc(128, BN, false, ph.b_mn != 0);
        const int total_k = ph.k_steps * ph.npairs;
        for (int t = blockIdx.x; ok && t < tiles_of(ph); t += gridDim.x, ++lt) {
          const uint32_t ab = lt & 1;
          if (lt >= 2 && !W.wait(&aempty[ab], ((lt >> 1) - 1) & 1, 3)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d = tmem + ab * BN;
          for (int kk = 0; kk < total_k; ++kk, ++it) {
            const uint32_t s = it % STAGES;
            if (!W.wait(&full[s], (it / STAGES) & 1, 4)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sa = smem_u32(smem + s * STAGE);
            const uint32_t sb = sa + A_BYTES;
            // four K = 16 slices: 32 B along a K-major row, 2 KB (eight
            // 128-B rows) along an MN-major tile
            const uint64_t ad0 = make_sdesc(sa, 16, 1024);
            const uint64_t bd0 = ph.b_mn ? make_sdesc(sb, 8192, 1024) : make_sdesc(sb, 16, 1024);
            const uint64_t bstep = ph.b_mn ? (2048 >> 4) : (32 >> 4);
            for (int k4 = 0; k4 < 4; ++k4)
              mma_bf16(d, ad0 + k4 * (32 >> 4), bd0 + k4 * bstep, idesc, (kk | k4) != 0);
            mma_commit(&empty[s]);
          }
          if (!ok) break;
          mma_commit(&afull[ab]);
        }
      }
      mma_commit(fin);
      W.drain(fin, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    uint32_t lt = 0;
    bool ok = true;
    // Every epilogue warp runs every phase up to the named barrier at its end,
    // also after a failed wait (it then skips the work), so that no warp is
    // left waiting at that barrier for one that gave up.
    for (int p = 0; p < nph; ++p) {
      const NsPhase& ph = phase(p);
      // Cin of this phase may be another CTA's output of the phase before
      if (ok && p > 0 && !grid_wait(P.counter, (unsigned)p * G, W, 5)) ok = false;
      for (int t = blockIdx.x; ok && t < tiles_of(ph); t += gridDim.x, ++lt) {
        int tm, tn, b;
        decode(ph, t, tm, tn, b);
        const uint32_t ab = lt & 1;
        if (!W.wait(&afull[ab], (lt >> 1) & 1, 6)) { ok = false; break; }
        tc_fence_after();
        const int m = tm * 128 + row;
        const bool valid = m < ph.M;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          float v[32];
          tmem_ld32(tmem + lane_base + ab * BN + c, v);   // every lane: warp-collective
          if (!valid) continue;
          const int n = tn * BN + c;
          if (ph.beta != 0.f) {
            const float4* cp =
                reinterpret_cast<const float4*>(ph.cin + b * ph.cin_bs + (size_t)m * ph.ldc + n);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float4 x = cp[j];
              v[4 * j + 0] = ph.alpha * v[4 * j + 0] + ph.beta * x.x;
              v[4 * j + 1] = ph.alpha * v[4 * j + 1] + ph.beta * x.y;
              v[4 * j + 2] = ph.alpha * v[4 * j + 2] + ph.beta * x.z;
              v[4 * j + 3] = ph.alpha * v[4 * j + 3] + ph.beta * x.w;
            }
          } else if (ph.alpha != 1.f) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] *= ph.alpha;
          }
          if (ph.o32 != nullptr) {
            float4* dst = reinterpret_cast<float4*>(ph.o32 + b * ph.o32_bs + (size_t)m * ph.ld32 + n);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
          }
          const size_t o = b * ph.o16_bs + (size_t)m * ph.ld16 + n;
          uint32_t hv[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) hv[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
          uint4* dst = reinterpret_cast<uint4*>(ph.o16 + o);
#pragma unroll
          for (int j = 0; j < 4; ++j) dst[j] = make_uint4(hv[4 * j], hv[4 * j + 1], hv[4 * j + 2], hv[4 * j + 3]);
          if (ph.o16lo != nullptr) {
            uint4* dlo = reinterpret_cast<uint4*>(ph.o16lo + o);
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
        tc_fence_before();
        mbar_arrive(&aempty[ab]);
      }
      // this CTA's outputs of phase p are written: make them visible to the
      // other CTAs' TMA loads and plain loads, then count the CTA in (not
      // after a failure: the other CTAs then run out their bounded waits)
      fence_proxy_async_global();
      __threadfence();
      epilogue_bar();
      if (threadIdx.x == 64 && !W.aborted()) red_release_gpu_add(P.counter, 1u);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * BN);
  }
}

// Host side: the six (kind, parity) phases of the Newton-Schulz loop of
// launch_lact's Muon step, launched cooperatively.  Returns 0 on success.
int launch_ns_fused(const NsFusedLaunch& L, cudaStream_t stream) {
  static_assert(sizeof(NsFusedParams) < 32000, "kernel parameters fit the launch limit");
  NsFusedParams* P = new NsFusedParams();
  const int r = L.r, c = L.c, nb = L.nb;
  const bool split = L.split;
  auto sq_map = [&](CUtensorMap* m, const void* p) {   // r x r, K-major boxes {64, 128}
    return make_tmap_bf16_3d(m, p, r, r, nb, (uint64_t)r * 2, (uint64_t)r * r * 2, 64, 128);
  };
  auto xk_map = [&](CUtensorMap* m, const void* p) {   // r x c, K-major (K = c)
    return make_tmap_bf16_3d(m, p, c, r, nb, (uint64_t)c * 2, (uint64_t)r * c * 2, 64, 128);
  };
  auto xn_map = [&](CUtensorMap* m, const void* p) {   // r x c as an MN-major B (N = c)
    return make_tmap_bf16_3d(m, p, c, r, nb, (uint64_t)c * 2, (uint64_t)r * c * 2, 64, 64);
  };
  int err = 0;
  for (int par = 0; par < 2 && !err; ++par) {
    // products of split operands: hi*hi + hi*lo + lo*hi
    NsPhase& A = P->ph[0][par];
    err |= xk_map(&A.a[0], L.Xb[par]) | xk_map(&A.b[0], L.Xb[par]);
    if (split) {
      A.a[1] = A.a[0];
      err |= xk_map(&A.b[1], L.Xl[par]) | xk_map(&A.a[2], L.Xl[par]);
      A.b[2] = A.b[0];
    }
    A.M = r; A.N = r; A.batch = nb; A.k_steps = c / 64; A.npairs = split ? 3 : 1; A.b_mn = 0;
    A.alpha = 1.f; A.beta = 0.f;
    A.o32 = L.A32; A.o32_bs = (long long)r * r; A.ld32 = r;
    A.o16 = L.Ab; A.o16lo = L.Al; A.o16_bs = (long long)r * r; A.ld16 = r;

    NsPhase& B = P->ph[1][par];
    err |= sq_map(&B.a[0], L.Ab);
    B.b[0] = B.a[0];
    if (split) {
      B.a[1] = B.a[0];
      err |= sq_map(&B.b[1], L.Al);
      B.a[2] = B.b[1];
      B.b[2] = B.a[0];
    }
    B.M = r; B.N = r; B.batch = nb; B.k_steps = r / 64; B.npairs = split ? 3 : 1; B.b_mn = 0;
    B.alpha = L.coef_c; B.beta = L.coef_b; B.cin = L.A32; B.cin_bs = (long long)r * r; B.ldc = r;
    B.o16 = L.Bb; B.o16lo = L.Bl; B.o16_bs = (long long)r * r; B.ld16 = r;

    NsPhase& X = P->ph[2][par];
    err |= sq_map(&X.a[0], L.Bb) | xn_map(&X.b[0], L.Xb[par]);
    if (split) {
      X.a[1] = X.a[0];
      err |= xn_map(&X.b[1], L.Xl[par]) | sq_map(&X.a[2], L.Bl);
      X.b[2] = X.b[0];
    }
    X.M = r; X.N = c; X.batch = nb; X.k_steps = r / 64; X.npairs = split ? 3 : 1; X.b_mn = 1;
    X.alpha = 1.f; X.beta = L.coef_a; X.cin = L.X32; X.cin_bs = (long long)r * c; X.ldc = c;
    X.o32 = L.X32; X.o32_bs = (long long)r * c; X.ld32 = c;
    X.o16 = const_cast<__nv_bfloat16*>(L.Xb[par ^ 1]);
    X.o16lo = const_cast<__nv_bfloat16*>(L.Xl[par ^ 1]); X.o16_bs = (long long)r * c; X.ld16 = c;
  }
  if (err) {
    delete P;
    return -1;
  }
  P->steps = L.steps;
  P->counter = L.counter;
  P->st = L.st;
  static std::atomic<uint64_t> attr{0};
  if (allow_dynamic_smem(ns_fused_kernel, (int)nsf::SMEM, attr)) {
    delete P;
    return -1;
  }
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int most = 0;
  for (int k = 0; k < 3; ++k) {
    const NsPhase& ph = P->ph[k][0];
    most = std::max(most, ((ph.M + 127) / 128) * (ph.N / nsf::BN) * ph.batch);
  }
  const int grid = std::max(1, std::min(sms, most));
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(nsf::THREADS);
  cfg.dynamicSmemBytes = nsf::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeCooperative;
  attrs[0].val.cooperative = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  prof_before(K_GEMM_NS, stream);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, ns_fused_kernel, *P);
  prof_after(K_GEMM_NS, stream);
  delete P;
  return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace ttt
