// common.cuh -- sm_100a building blocks shared by the kernels of this
// library: mbarriers with bounded waits, TMA tile loads, tcgen05 (5th-gen
// tensor core) MMA / TMEM helpers, UMMA shared-memory descriptors and the
// device status word.  Inline PTX written for this library.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#ifndef TTT_DEVICE_INLINE
#define TTT_DEVICE_INLINE __device__ __forceinline__
#endif

namespace ttt {

// ----------------------------------------------------------------- status
// Status word layout (first 256 bytes of every workspace):
//   [0] error code (0 = ok; 1 = bounded wait ran out)
//   [1] kernel id that recorded it, [2] wait site, [3] block id
enum : uint32_t { DEV_OK = 0, DEV_TIMEOUT = 1 };

struct DevStatus {
  uint32_t* word;          // global status block (may be null: no reporting)
  uint64_t timeout_ns;     // wall-clock bound of every wait
  uint32_t kernel_id;
};

TTT_DEVICE_INLINE uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

TTT_DEVICE_INLINE uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ----------------------------------------------------------------- mbarrier
TTT_DEVICE_INLINE void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
TTT_DEVICE_INLINE void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
TTT_DEVICE_INLINE void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
TTT_DEVICE_INLINE void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
TTT_DEVICE_INLINE bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of a phase (no suspend): for issuers that poll several
// barriers and act on whichever is ready.
TTT_DEVICE_INLINE bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Per-CTA abort flag lives in shared memory; once any thread of the CTA gives
// up on a wait, every later wait of the CTA returns false immediately so that
// all roles drain to the common teardown.
struct Waiter {
  volatile uint32_t* abort_flag;  // shared memory
  DevStatus st;
  uint32_t site_base;

  // Bounded wait on (bar, parity).  Returns false on abort/timeout.
  TTT_DEVICE_INLINE bool wait(uint64_t* bar, uint32_t parity, uint32_t site) const {
    if (*abort_flag) return false;
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
      if (mbar_try_wait(bar, parity)) return true;
      if ((it & 255u) == 0u) {
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > st.timeout_ns) {
          fail(site);
          return false;
        }
      }
    }
  }
  // Wait that ignores the abort flag (used while draining copies in flight);
  // still bounded by the timeout.
  TTT_DEVICE_INLINE bool drain(uint64_t* bar, uint32_t parity) const {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
      if (globaltimer_ns() - t0 > st.timeout_ns) return false;
    }
    return true;
  }
  TTT_DEVICE_INLINE void fail(uint32_t site) const {
    *abort_flag = 1u;
    if (st.word != nullptr) {
      if (atomicCAS(st.word, DEV_OK, DEV_TIMEOUT) == DEV_OK) {
        st.word[1] = st.kernel_id;
        st.word[2] = site_base + site;
        st.word[3] = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
      }
    }
  }
  TTT_DEVICE_INLINE bool aborted() const { return *abort_flag != 0u; }
};

// ------------------------------------------------- grid-wide counters
// Monotone arrival counters in global memory: a CTA publishes its writes
// with a release add, a waiter polls with acquire loads.  Generic-proxy
// writes that a TMA load reads later are ordered by a proxy fence on both
// sides.
TTT_DEVICE_INLINE unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
TTT_DEVICE_INLINE void red_release_gpu_add(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
TTT_DEVICE_INLINE void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Bounded wait until the counter reaches `target`.  False on abort (this
// CTA's flag, or the grid-wide word `gabort` when given) or timeout; a
// timeout records the site and raises `gabort`, so the other CTAs stop
// waiting too.
TTT_DEVICE_INLINE bool grid_wait(const unsigned* ctr, unsigned target, const Waiter& W,
                                 uint32_t site, unsigned* gabort = nullptr) {
  if (ld_acquire_gpu(ctr) >= target) return true;
  const uint64_t t0 = globaltimer_ns();
  // plain polling (one thread per CTA waits)
  for (uint32_t it = 1;; ++it) {
    if (ld_acquire_gpu(ctr) >= target) return true;
    if ((it & 63u) == 0u) {
      if (W.aborted()) return false;
      if (gabort != nullptr && *reinterpret_cast<volatile unsigned*>(gabort) != 0u) {
        *W.abort_flag = 1u;
        return false;
      }
      if (globaltimer_ns() - t0 > W.st.timeout_ns) {
        W.fail(site);
        if (gabort != nullptr) atomicExch(gabort, 1u);
        return false;
      }
    }
  }
}

// ----------------------------------------------------------------- PDL
// Programmatic dependent launch: a kernel launched with programmatic stream
// serialisation may start while its predecessor drains; it must wait for the
// predecessor's memory before touching global data.
TTT_DEVICE_INLINE void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
TTT_DEVICE_INLINE void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ----------------------------------------------------------------- TMA
TTT_DEVICE_INLINE void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}
// 3-D tiled load (no multicast) into this CTA's shared memory; completion is
// signalled as transaction bytes on `bar`.
TTT_DEVICE_INLINE void tma_load_3d(void* dst, const CUtensorMap* m, uint64_t* bar, int x, int y,
                                   int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

TTT_DEVICE_INLINE void tma_load_4d(void* dst, const CUtensorMap* m, uint64_t* bar, int x, int y,
                                   int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}

// Barrier `id` (1..15) over `n` threads (a multiple of 32): every thread of
// the participating warps must reach it on every path.
TTT_DEVICE_INLINE void named_bar_sync(uint32_t id, uint32_t n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Barrier `id` over `n` threads that also ANDs a per-thread flag: every
// participant gets the same answer, so a loop can leave on it uniformly.
TTT_DEVICE_INLINE bool named_bar_all(uint32_t id, uint32_t n, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

// Tensor store shared -> global (bulk async group of the issuing thread).
// The shared source must not be rewritten before bulk_wait_read() returns;
// every group is waited for (bulk_wait_all) before the CTA exits.
TTT_DEVICE_INLINE void tma_store_3d(const CUtensorMap* m, const void* src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
               : "memory");
}
TTT_DEVICE_INLINE void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
TTT_DEVICE_INLINE void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
TTT_DEVICE_INLINE void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Make generic-proxy shared-memory writes visible to the async proxy
// (tcgen05.mma operand reads, TMA stores).
TTT_DEVICE_INLINE void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ----------------------------------------------------------------- tcgen05
TTT_DEVICE_INLINE void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
TTT_DEVICE_INLINE void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
TTT_DEVICE_INLINE void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
TTT_DEVICE_INLINE void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
TTT_DEVICE_INLINE void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 inputs, fp32 accumulate.
TTT_DEVICE_INLINE void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T, tf32 inputs (fp32 in shared memory).
TTT_DEVICE_INLINE void mma_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` once every tcgen05 op issued so far by this thread is done.
TTT_DEVICE_INLINE void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Instruction descriptor, kind::f16 / kind::tf32 with fp32 accumulation.
// bits: [4,6) D fmt (1=f32), [7,10) A fmt, [10,13) B fmt (bf16=1, tf32=2),
// 15 A major (1 = MN), 16 B major, [17,23) N>>3, [24,29) M>>4.
__host__ __device__ constexpr uint32_t make_idesc(int M, int N, bool a_mn, bool b_mn,
                                                  uint32_t ab_fmt = 1u) {
  return (1u << 4) | (ab_fmt << 7) | (ab_fmt << 10) | ((a_mn ? 1u : 0u) << 15) |
         ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version bits.
// K-major tiles: rows of 128 B, 8-row groups 1024 B apart (sbo), lbo unused.
// MN-major tiles: 64-element (128 B) MN blocks `lbo` bytes apart, 8-row K
// groups `sbo` bytes apart.
TTT_DEVICE_INLINE uint64_t make_sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;   // descriptor version for sm_100
  d |= (uint64_t)2u << 61;   // SWIZZLE_128B
  return d;
}

// The same descriptor for an operand `bytes` further on (the start address
// field holds addr >> 4 in 14 bits; shared addresses stay below 2^18, so the
// sum never carries out of the field).
TTT_DEVICE_INLINE uint64_t sdesc_add(uint64_t d, uint32_t bytes) { return d + (bytes >> 4); }

// 32 lanes x 32 consecutive 32-bit columns per warp (one row per thread).
TTT_DEVICE_INLINE void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
TTT_DEVICE_INLINE void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
// Issue-only variants: several loads may be in flight before one wait.
TTT_DEVICE_INLINE void tmem_ld16_issue(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
TTT_DEVICE_INLINE void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

TTT_DEVICE_INLINE void tmem_st16(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ----------------------------------------------------------------- layouts
// Byte offset of element (row, col) of a bf16 tile stored with 128-byte rows
// in the 128B-swizzled layout produced by TMA (tile base 1024-B aligned):
// the 16-byte chunk index is XOR-ed with (row mod 8).
TTT_DEVICE_INLINE uint32_t sw128_offset(uint32_t row, uint32_t col_bf16) {
  return row * 128u + ((((col_bf16 >> 3) ^ row) & 7u) << 4) + ((col_bf16 & 7u) << 1);
}

TTT_DEVICE_INLINE uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Two-lane fp32 arithmetic with sm_100's packed instructions (each lane
// rounds exactly like the scalar instruction): half the issue slots.
TTT_DEVICE_INLINE float2 x2_mul(float2 a, float2 b) {
  float2 r;
  asm("{\n\t.reg .b64 A, B, R;\n\tmov.b64 A, {%2, %3};\n\tmov.b64 B, {%4, %5};\n\t"
      "mul.rn.f32x2 R, A, B;\n\tmov.b64 {%0, %1}, R;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}
TTT_DEVICE_INLINE float2 x2_fma(float2 a, float2 b, float2 c) {
  float2 r;
  asm("{\n\t.reg .b64 A, B, C, R;\n\tmov.b64 A, {%2, %3};\n\tmov.b64 B, {%4, %5};\n\t"
      "mov.b64 C, {%6, %7};\n\tfma.rn.f32x2 R, A, B, C;\n\tmov.b64 {%0, %1}, R;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return r;
}
TTT_DEVICE_INLINE float2 x2_sub(float2 a, float2 b) {
  float2 r;
  asm("{\n\t.reg .b64 A, B, R;\n\tmov.b64 A, {%2, %3};\n\tmov.b64 B, {%4, %5};\n\t"
      "sub.rn.f32x2 R, A, B;\n\tmov.b64 {%0, %1}, R;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}
TTT_DEVICE_INLINE float2 x2_splat(float a) { return make_float2(a, a); }
// sigmoid(x) = 0.5 tanh(x / 2) + 0.5 on both lanes (hardware tanh
// approximation, relative error about 2^-11)
TTT_DEVICE_INLINE float2 x2_sigmoid(float2 x) {
  const float2 h = x2_mul(x, x2_splat(0.5f));
  float2 t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t.x) : "f"(h.x));
  asm("tanh.approx.f32 %0, %1;" : "=f"(t.y) : "f"(h.y));
  return x2_fma(t, x2_splat(0.5f), x2_splat(0.5f));
}

// 32 bytes to global memory in one 256-bit access (dst 32-byte aligned):
// a warp storing one row per thread then writes whole 32-byte sectors
TTT_DEVICE_INLINE void st_global_v8(void* dst, const uint32_t* a) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "r"(a[0]),
               "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(a[4]), "r"(a[5]), "r"(a[6]), "r"(a[7])
               : "memory");
}

TTT_DEVICE_INLINE void st_shared_v4(uint32_t saddr, uint32_t a, uint32_t b, uint32_t c,
                                    uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(saddr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}
TTT_DEVICE_INLINE void ld_shared_v4(uint32_t saddr, uint32_t& a, uint32_t& b, uint32_t& c,
                                    uint32_t& d) {
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(a), "=r"(b), "=r"(c), "=r"(d)
               : "r"(saddr)
               : "memory");
}

TTT_DEVICE_INLINE float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
TTT_DEVICE_INLINE float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

}  // namespace ttt
