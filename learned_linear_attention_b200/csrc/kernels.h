// kernels.h -- internal interface between the C ABI (api.cu) and the kernel
// launchers.  Not part of the public ABI.
#pragma once

#include <stdio.h>

#include <atomic>
#include <utility>

#include "common.cuh"

namespace ttt {

// ----------------------------------------------------------------- launches
// Launch with programmatic stream serialisation (the kernel calls pdl_wait()
// before reading what earlier work on the stream wrote).
// cluster_x > 1 additionally groups consecutive CTAs into clusters.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block,
                                      size_t smem, cudaStream_t stream, int cluster_x,
                                      Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  int n = 1;
  if (cluster_x > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster_x;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args&&... args) {
  return launch_pdl_cluster(kernel, grid, block, smem, stream, 1, std::forward<Args>(args)...);
}

// Let `kernel` use `bytes` of dynamic shared memory on the current device.
// The attribute belongs to each device, so `done` keeps one bit per device
// that already has it (devices 64 and up are set on every call).
template <typename... KArgs>
inline int allow_dynamic_smem(void (*kernel)(KArgs...), int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  const uint64_t bit = (dev >= 0 && dev < 64) ? (uint64_t(1) << dev) : 0;
  if (bit != 0 && (done.load(std::memory_order_acquire) & bit) != 0) return 0;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return -1;
  done.fetch_or(bit, std::memory_order_release);
  return 0;
}

// ----------------------------------------------------------------- tensor maps
// 3-D bf16 tensor map {inner, rows, batch} with 128-byte swizzle; strides in
// bytes; box {box_inner, box_rows, 1}.  Out-of-range elements read as zero.
// Returns 0 on success.
int make_tmap_bf16_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                      uint64_t batch, uint64_t row_stride, uint64_t batch_stride,
                      uint32_t box_inner, uint32_t box_rows);
// The same bf16 matrices [batch][rows][inner] seen as 4-D {64, rows,
// inner / 64, batch}: the third dimension steps 128 bytes, one 64-element
// block of a row.  A box {64, box_rows, box_blocks, 1} lands in shared
// memory as box_blocks blocks of box_rows 128-byte rows (8 KB apart for 64
// rows), the MN-major operand layout of the tensor cores with 128-byte
// swizzle, so one copy brings a whole MN-major operand block.
// As make_tmap_bf16_3d with the swizzle given in bytes (0, 32, 64 or 128).
int make_tmap_bf16_3d_sw(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                         uint64_t batch, uint64_t row_stride, uint64_t batch_stride,
                         uint32_t box_inner, uint32_t box_rows, int swizzle_bytes);
int make_tmap_bf16_blocked(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                           uint64_t batch, uint64_t row_stride, uint64_t batch_stride,
                           uint32_t box_rows, uint32_t box_blocks);

// ----------------------------------------------------------------- TTT-linear
// Sequence split of the tensor-core linear kernel (see ttt_linear.cu).
struct LinearPlan {
  int P, R, seg_tiles, unit_tiles;
  size_t ws_floats;   // segment-state floats the split needs in the workspace
};
LinearPlan ttt_linear_plan(int BH, int N, int sms);
struct LinearLaunch {
  int B, H, N, dk, dv, chunk, include_diag;
  int bidir;    // bidirectional order: every update first, then every read
  int in_bf16, out_bf16;
  const void *q, *k, *v;
  const float* lr;
  float* S;
  void* out;
  DevStatus st;
  LinearPlan plan;
  float* seg_state;           // workspace after the status block
  size_t seg_state_floats;
  const float* out_scale;     // nullable: output row t is multiplied by out_mul * out_scale[bh][t]
  float out_mul;
};
// S <- S + sum_t lr_t k_t v_t^T over all N tokens (bf16, dk = dv = 64), with
// no outputs: the segment pre-pass run over the whole sequence, then a sum of
// its unit increments.  Needs L.seg_state_floats >= ttt_linear_state_sum_floats.
size_t ttt_linear_state_sum_floats(int BH, int N, int sms);
int launch_ttt_linear_state_sum(const LinearLaunch& L, int sms, cudaStream_t stream);
int launch_ttt_linear_simt(const LinearLaunch& L, cudaStream_t stream);
int launch_ttt_linear_umma(const LinearLaunch& L, cudaStream_t stream);
size_t ttt_linear_simt_smem(int dk, int dv);

// Backward pass (ttt_linear_bwd.cu): four forward scans with exchanged roles.
struct LinearBwdWorkspace {
  size_t status, ones, r, neg_rt, neg_r, s0t, seg, total;   // byte offsets
  size_t seg_floats;                                         // segment states of one scan
};
// seg_floats: segment states of one tensor-core scan or of the state pre-pass
LinearBwdWorkspace ttt_linear_bwd_layout(int BH, int N, int dk, int dv, size_t seg_floats);
struct LinearBwdLaunch {
  int B, H, N, dk, dv, chunk, include_diag, in_bf16, umma, sms;
  const void *q, *k, *v, *dout;
  const float *lr, *S0, *dS_end;       // S0, dS_end nullable (zeros)
  float *gq, *gk, *gv, *glr, *gS0;     // gradients of q, k, v, lr, S0 (float32)
  uint8_t* ws;
  LinearBwdWorkspace w;
  LinearPlan plan;
  DevStatus st;
};
int launch_ttt_linear_bwd(const LinearBwdLaunch& L, cudaStream_t stream);

// ----------------------------------------------------------------- window attention
// Causal sliding-window softmax attention, head dim 128, bf16 q, k, v
// [B,H,N,128]; out fp32 or bf16, overwritten or (accumulate) added to.
struct WindowAttnLaunch {
  int B, H, N, window;
  float scale;
  int out_bf16, accumulate;
  const void *q, *k, *v;
  void* out;
  DevStatus st;
};
int launch_window_attention(const WindowAttnLaunch& L, cudaStream_t stream);

// ----------------------------------------------------------------- LaCT
struct LactLaunch {
  int B, H, N_in, N_q, d, dh, chunk;
  int causal;
  int opt;                 // 0 GD, 1 momentum, 2 Muon
  float beta;
  int ns_steps;
  float ns_a, ns_b, ns_c, ns_eps;
  int normalize_rows;
  float norm_eps;
  int update_mask;
  int out_bf16;
  int split;               // split-bf16 operands (hi + lo)
  const void *q, *k, *v;
  const float* lr;
  float* state;            // [W1 | W3 | W2 | M1 | M3 | M2] fp32
  void* out;
  uint8_t* ws;             // workspace (status block first)
  size_t ws_bytes;
  DevStatus st;
  // Pieces of the chunk loop for context parallelism (a chunk's tokens split
  // across devices): LACT_FULL runs the whole layer; LACT_GRAD writes to G
  // the lr-weighted gradient sum of tokens [t0, t0 + n) (n <= chunk) at the
  // current weights; LACT_APPLY applies the optimizer step and row
  // normalisation with the (summed) chunk gradient G; LACT_READ writes out
  // rows [t0, t0 + n) = f_W(q rows) with the current weights.
  int mode;
  int t0, n;
  float* G;                // [G1 | G3 | G2] fp32, laid out like the weights of the state
  float* rownorm_out;      // APPLY, nullable: each updated row's norm before the
                           // normalisation, [BH][2 dh + d] (W1 rows, W3 rows, W2 rows)
  // LACT_REPLAY (the backward pass's forward replay): the chunk sequence
  // without the read, keeping the fp32 weights at the start of every chunk
  // and after the last ([chunks + 1][W1 | W3 | W2]) and the row norms of
  // every update ([chunks][BH][2 dh + d]).
  float* wsave;
  float* rownorm_all;
};
enum LactMode { LACT_FULL = 0, LACT_GRAD = 1, LACT_APPLY = 2, LACT_READ = 3, LACT_REPLAY = 4 };
// The batched tcgen05 GEMM of gemm.cuh (operand majorness by variant).
struct GemmMaps;
struct GemmArgs;
enum { GEMM_AK_BK = 0, GEMM_AK_BMN = 1, GEMM_AMN_BMN = 2 };
int gemm_launch(int variant, const GemmMaps& maps, const GemmArgs& g, cudaStream_t stream,
                int kind);
GemmArgs gemm_args_default(const DevStatus& st);
// Workspace layout (byte offsets) for a given problem.
struct LactWorkspace {
  size_t status, w1b, w3b, w2b, d13, gm, aq, part, rowss, nsx32, nsxb, nsa32, nsab, nsbb, total;
  // split operands (hi + lo bf16): residual copies
  size_t w1lo, w3lo, w2lo, d13lo, gmlo, aqlo, nsxlo, nsalo, nsblo;
  int cmax;                // rows of the per-chunk intermediates
  int splits;              // split-K factor of the gradient GEMMs
  int keygrad;             // head dim 128, GD / momentum: fused key/gradient path
  int w2par;               // W2-only GD without normalisation: parallel form over chunks
  size_t pmb;              // parallel form: bf16 chunk-start W2 [chunks][BH][d][dh]
  int nbuf;                // bf16 weight buffers (3 on the fused causal path, else 2)
  int naq;                 // Aq buffers (2 on the fused causal path, else 1)
  size_t nsctr;            // Muon: phase counter of the fused Newton-Schulz kernel
  size_t loopctr;          // causal chunk loop: per-head arrival counters (3 BH + 2 words)
};
// The Newton-Schulz loop of the Muon step as one cooperative launch
// (ns_fused.cu): `steps` quintic steps on nb matrices r x c (r <= c).
struct NsFusedLaunch {
  int r, c, nb, steps, split;
  float coef_a, coef_b, coef_c;
  float* X32;                       // [nb][r][c] fp32, in/out
  const __nv_bfloat16* Xb[2];       // bf16 hi copies of X (step parity)
  const __nv_bfloat16* Xl[2];       // lo copies (split operands)
  float* A32;                       // [nb][r][r]
  __nv_bfloat16 *Ab, *Al, *Bb, *Bl;
  unsigned* counter;                // zeroed before the launch
  DevStatus st;
};
int launch_ns_fused(const NsFusedLaunch& L, cudaStream_t stream);
bool lact_uses_keygrad(int d, int dh, int opt, int split);
bool lact_uses_w2_parallel(int N_in, int chunk, int d, int dh, int causal, int opt, int split,
                           int update_mask, int normalize);
// allow_parallel = 0 lays out the chunk loop even where the parallel form of
// the W2-only layer applies (its workspace holds every chunk at once).
LactWorkspace lact_workspace_layout(int B, int H, int N_in, int N_q, int d, int dh, int chunk,
                                    int causal, int opt, int split, int update_mask, int normalize,
                                    int allow_parallel);
int launch_lact(const LactLaunch& L, cudaStream_t stream);

// Backward pass of the LaCT layer (lact_bwd.cu).
struct LactBwdWorkspace {
  size_t status, fws, fws_bytes, state, wsave, rn, G, dW, dM, R, Rb, Wb, ddy, gctr, total;
  size_t f32[6], b16[7];   // per-chunk intermediates [BH][cmax][dh]
  int cmax, nch;
};
struct LactBwdLaunch {
  LactLaunch f;            // the forward problem (shapes, optimizer, q, k, v, lr)
  const float* W0;         // [W1 | W3 | W2] at the start of the call
  const void* dout;        // [B,H,R,d] bf16 (R = N_in causal, N_q bidirectional)
  const float* dW_end;     // nullable: [dW1 | dW3 | dW2] of the end weights
  float *dq, *dk, *dv, *dlr, *dW0;
  uint8_t* ws;
  DevStatus st;
};
LactBwdWorkspace lact_bwd_layout(const LactLaunch& f);
int launch_lact_bwd(const LactBwdLaunch& L, cudaStream_t stream);

// Fused key pass + chunk gradient (head dim 128): partial sums per token group.
struct KeyGradLaunch {
  int BH, N_in, C, t0, dh, groups;
  const void *k, *v, *q;      // q != nullptr: also form Aq for the chunk's queries
  __nv_bfloat16* Aq;
  long long aq_bs;
  const float* lr;
  const void *w1b, *w3b, *w2b;
  float* part[3];
  DevStatus st;
};
int keygrad_groups(int BH, int dh, int C, int max_groups);
// The whole causal chunk sequence of a head-dim-128 GD / momentum layer in
// one cooperative launch (lact_keygrad.cu): the fused key/gradient work, the
// row update and the read, with grid counters between the chunks.
struct KeyGradLoopLaunch {
  int BH, N_in, C, dh, max_groups, cmax;
  const void *k, *v, *q;
  const float* lr;
  __nv_bfloat16* Aq;          // two buffers of [BH][cmax][dh], aq_buf elements apart
  long long aq_buf;
  __nv_bfloat16* Wb[3][3];    // [buffer][matrix] bf16 copies, buffer 0 holds the start weights
  float* W[3];
  float* M[3];
  float* part[3];             // >= groups slots of partial sums
  int opt, normalize, mask;
  float beta, norm_eps;
  void* out;
  int out_bf16;
  unsigned* ctr;              // 3 BH + 2 words of workspace (zeroed by the launch)
  int groups, workers, readers;   // from lact_loop_plan (0: the launch plans itself)
  int cast_first;             // the kernel writes the start weights' bf16 copies (every buffer
                              // for a matrix the update leaves alone) before the first chunk
  float* wsave;               // nullable: the weights after every chunk (slots 1 .. chunks)
  float* rownorm;             // nullable: every update's row norms (normalising layers)
  DevStatus st;
};
// 0 when the chunk loop can run this shape on the current device (groups,
// worker and reader CTA counts returned), -1 otherwise.
int lact_loop_plan(int BH, int N_in, int C, int dh, int max_groups, int* groups, int* workers,
                   int* readers);
int launch_lact_loop(const KeyGradLoopLaunch& L, cudaStream_t stream);
// The fused memory read for head dim 128 (lact_read.cu): out rows [t0, t0 + C)
// = W2 (silu(W1 q) * (W3 q)) with bf16 weight copies, on at most max_grid CTAs.
struct ReadFusedLaunch {
  int BH, rows, t0, C, dh, out_bf16, max_grid;
  const void* q;                       // [BH][rows][128] bf16
  const __nv_bfloat16 *w1b, *w3b, *w2b;
  void* out;                           // [BH][rows][128]
  DevStatus st;
};
int launch_lact_read_fused(const ReadFusedLaunch& L, cudaStream_t stream);
int launch_lact_keygrad(const KeyGradLaunch& L, cudaStream_t stream);

// ----------------------------------------------------------------- profiling
enum KernelKind {
  K_LIN_SIMT, K_LIN_UMMA, K_LACT_CAST, K_KEYPASS, K_GEMM_READ, K_GEMM_GRAD, K_UPDATE,
  K_MUON_MOM, K_NS_PREP, K_GEMM_NS, K_MUON_APPLY, K_KEYGRAD, K_LIN_SEG, K_LIN_BWD_EW, K_SWA, K_LOOP,
  K_BWD_FWD, K_BWD_GROUP, K_NUM
};
void prof_before(int kind, cudaStream_t s);
void prof_after(int kind, cudaStream_t s);

// ----------------------------------------------------------------- self test
int launch_wait_timeout_probe(DevStatus st, cudaStream_t stream);

}  // namespace ttt
