// Device helpers shared by the sm_100a kernels of the TTT trunk+branch attention:
// mbarriers with bounded waits, TMA tile loads, tcgen05 (UMMA) descriptors and
// instructions, TMEM loads/stores.  Inline PTX only; no library kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ttt_internal.h"

namespace ttt {

// ---------------------------------------------------------------------------
// Kernel timeline trace (profiling builds only: -DTTT_KERNEL_TRACE).  CTA 0 of a
// launch records %clock64 at numbered points, per loop iteration; the trace build
// exports ttt_trace_read_<kernel>() to copy the table out.  In normal builds every
// trace point compiles to nothing.
// ---------------------------------------------------------------------------
#ifdef TTT_KERNEL_TRACE
constexpr int kTraceSlots = 24;
constexpr int kTraceIters = 1024;
static __device__ long long g_trace[kTraceSlots][kTraceIters];
__device__ __forceinline__ void trace_point(int slot, int j) {
  if (blockIdx.x == 0 && j < kTraceIters) {
    long long t;
    asm volatile("mov.u64 %0, %%clock64;" : "=l"(t));
    g_trace[slot][j] = t;
  }
}
// Every CTA (up to kCtaTrace) also records its SM, its work count and %clock64 /
// %globaltimer at four points: entry, first tile ready, last tile done, exit.
constexpr int kCtaTrace = 8192;
static __device__ long long g_cta[kCtaTrace][10];
__device__ __forceinline__ void cta_mark(int point) {
  if (blockIdx.x < kCtaTrace) {
    long long t;
    asm volatile("mov.u64 %0, %%clock64;" : "=l"(t));
    g_cta[blockIdx.x][point] = t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    g_cta[blockIdx.x][4 + point] = t;
  }
}
__device__ __forceinline__ void cta_info(int work) {
  if (blockIdx.x < kCtaTrace) {
    unsigned sm;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));
    g_cta[blockIdx.x][8] = sm;
    g_cta[blockIdx.x][9] = work;
  }
}
#define TTT_TRACE(slot, j) ::ttt::trace_point((slot), (j))
#define TTT_CTA_MARK(point) ::ttt::cta_mark(point)
#define TTT_CTA_INFO(work) ::ttt::cta_info(work)
#define TTT_TRACE_READER(name)                                                                       \
  extern "C" int name(void* host) {                                                                  \
    return static_cast<int>(cudaMemcpyFromSymbol(host, ::ttt::g_trace, sizeof(::ttt::g_trace)));     \
  }                                                                                                  \
  extern "C" int name##_cta(void* host) {                                                            \
    return static_cast<int>(cudaMemcpyFromSymbol(host, ::ttt::g_cta, sizeof(::ttt::g_cta)));         \
  }
#else
#define TTT_TRACE(slot, j) ((void)0)
#define TTT_CTA_MARK(point) ((void)0)
#define TTT_CTA_INFO(work) ((void)0)
#define TTT_TRACE_READER(name)
#endif

// ---------------------------------------------------------------------------
// generic
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ float exp2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Every wait in these kernels is bounded.  On expiry the waiting thread raises the
// CTA-wide abort flag (shared memory) and records the wait site in the per-call
// status word (global memory, first word of the workspace); every later wait in
// the CTA then returns at once, so all roles fall through to the common exit,
// which releases TMEM.  The host reads the status word with
// ttt_attn_device_status().
struct Watchdog {
  uint32_t* abort_smem;   // CTA-wide abort flag
  uint32_t* status_gmem;  // per-call device status (0 = ok)
  uint64_t budget_ns;     // per-wait limit
};

static __device__ __noinline__ bool wait_slow(uint64_t* bar, uint32_t parity, const Watchdog& wd, uint32_t site) {
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*reinterpret_cast<volatile uint32_t*>(wd.abort_smem)) return false;
    if (globaltimer_ns() - t0 > wd.budget_ns) {
      atomicExch(wd.abort_smem, 1u);
      if (wd.status_gmem) atomicCAS(wd.status_gmem, 0u, kStatusTimeoutBase | site);
      return false;
    }
  }
}

__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, const Watchdog& wd, uint32_t site) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_slow(bar, parity, wd, site);
}

// Warp-uniform bounded wait: every lane waits (and acquires); the result is agreed
// across the warp so that control flow stays uniform.
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, const Watchdog& wd, uint32_t site) {
  const bool ok = wait_bounded(bar, parity, wd, site);
  return __all_sync(0xffffffffu, ok);
}

// Bounded wait until a global counter that other CTAs advance equals `expect`
// (acquire: their writes before the increment are visible afterwards).
static __device__ __noinline__ bool wait_counter(const int* counter, int expect, const Watchdog& wd, uint32_t site) {
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(counter) : "memory");
    if (v == expect) return true;
    if (*reinterpret_cast<volatile uint32_t*>(wd.abort_smem)) return false;
    if (globaltimer_ns() - t0 > wd.budget_ns) {
      atomicExch(wd.abort_smem, 1u);
      if (wd.status_gmem) atomicCAS(wd.status_gmem, 0u, kStatusTimeoutBase | site);
      return false;
    }
    __nanosleep(128);
  }
}

// Bounded wait that ignores the abort flag: used on the exit path to let operations
// already issued to the tensor cores finish before TMEM is released.
static __device__ __noinline__ bool wait_drain(uint64_t* bar, uint32_t parity, const Watchdog& wd, uint32_t site) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > wd.budget_ns) {
      atomicExch(wd.abort_smem, 1u);
      if (wd.status_gmem) atomicCAS(wd.status_gmem, 0u, kStatusTimeoutBase | site);
      return false;
    }
  }
  return true;
}

// ---------------------------------------------------------------------------
// TMA (tiled bulk tensor copies, global -> shared of this CTA only)
// ---------------------------------------------------------------------------

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

// Tiled bulk tensor store shared -> global (bulk-group completion; coordinates >= 0).
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, const void* src, int c0, int c1, int c2,
                                             int c3) {
  asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
               : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Bulk (untiled) copy global -> shared, completion on an mbarrier (16-byte aligned,
// size a multiple of 16).
__device__ __forceinline__ void bulk_load(void* sdst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(sdst)),
               "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Slot of the 64-row query tile containing position pos of sequence n (see ld_slots).
__device__ __forceinline__ int ld_slot(int seq_start, int n, int pos) { return (seq_start >> 6) + n + (pos >> 6); }

// Bulk (untiled) reduce-add of fp32 from shared to global memory.
__device__ __forceinline__ void bulk_reduce_add_f32(float* gdst, const void* ssrc, uint32_t bytes) {
  asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(gdst),
               "r"(smem_u32(ssrc)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// ---------------------------------------------------------------------------
// paired fp32 arithmetic (sm_100: one instruction on two floats held in a 64-bit
// register pair; each lane is rounded exactly like the scalar instruction)
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// three-input maximum (one instruction on sm_100)
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// asynchronous copies global -> shared of this thread (16 or 4 bytes, aligned), completed
// by cp.async.wait_group
__device__ __forceinline__ void cp_async16(void* sdst, const void* gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(sdst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async4(void* sdst, const void* gsrc) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(sdst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// all but the most recent bulk group have finished reading their shared-memory source
__device__ __forceinline__ void bulk_wait_read1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// every bulk group has finished reading its shared-memory source
__device__ __forceinline__ void bulk_wait_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: shared-memory matrix descriptors, instruction descriptor, MMA
// ---------------------------------------------------------------------------

// Shared-memory matrix descriptor, 128-byte swizzle (operand tiles are 1024-byte
// aligned, rows of 128 bytes, 8-row swizzle atoms).  Field positions: start
// address >> 4 in bits 0-13, leading byte offset >> 4 in 16-29, stride byte offset
// >> 4 in 32-45, descriptor version 1 in bits 46-47, swizzle mode in 61-63
// (2 = 128-byte swizzle).
//   K-major operand: rows of the M/N dimension, 64 bf16 of K per 128-byte row;
//     SBO = byte distance between 8-row groups (1024), LBO unused (16).
//   MN-major operand: 64 bf16 of M/N per 128-byte row, rows along K;
//     LBO = byte distance between 64-element M/N chunks, SBO = distance between
//     8-row K groups (1024).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// Instruction descriptor for kind::f16 with bf16 A/B and an fp32 accumulator:
// D format in bits 4-5 (1 = f32), A format 7-9 and B format 10-12 (1 = bf16),
// A/B major in bits 15/16 (0 = K-major, 1 = MN-major), N >> 3 in 17-22,
// M >> 4 in 24-28.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem] (umma_ss_warp) or A[tmem] * B[smem] (umma_ts_warp;
// A one row per lane, two bf16 per column).  The whole warp executes them with
// identical (warp-uniform) operands and one elected lane issues, so that descriptors
// stay in the uniform datapath and the issuing warp spends few instructions per MMA.
__device__ __forceinline__ void umma_ss_warp(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_ts_warp(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on `bar` when every tcgen05 operation issued so far by the issuing
// thread has completed (elected lane).
__device__ __forceinline__ void umma_commit_warp(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// TMEM allocation: whole warp.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// 32 consecutive 32-bit columns of the calling thread's TMEM lane (32x32b shape:
// warp w reads lanes 32*(w%4) .. 32*(w%4)+31; the lane is part of taddr).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
        "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// Wait for this thread's outstanding TMEM loads, then tie the loaded registers to
// the wait so that no use of them can be scheduled above it.
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void reg_fence32(uint32_t (&r)[32]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                 "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                 "+r"(r[29]), "+r"(r[30]), "+r"(r[31]));
}

// ---------------------------------------------------------------------------
// sequence geometry
// ---------------------------------------------------------------------------

// Start token and length of sequence n: dense batches have B equal lengths S;
// packed (THD) batches read cu_seqlens.
__device__ __forceinline__ void seq_bounds(const SeqInfo& si, int n, int& start, int& len) {
  if (si.cu_seqlens) {
    start = si.cu_seqlens[n] * si.mult;
    len = si.cu_seqlens[n + 1] * si.mult - start;
  } else {
    start = n * si.S;
    len = si.S;
  }
}

// Sequence index and in-sequence position of packed token tau.
__device__ __forceinline__ void token_position(const SeqInfo& si, int tau, int& n, int& pos) {
  if (si.cu_seqlens) {
    int lo = 0, hi = si.nseq - 1;
    while (lo < hi) {
      int mid = (lo + hi + 1) >> 1;
      if (si.cu_seqlens[mid] * si.mult <= tau)
        lo = mid;
      else
        hi = mid - 1;
    }
    n = lo;
    pos = tau - si.cu_seqlens[lo] * si.mult;
  } else {
    n = tau / si.S;
    pos = tau - n * si.S;
  }
}

// Offset of lse / delta entry (pass p, head h, token tau in sequence n at position
// pos) in the public lse layout: dense [P][B][H][S], packed [P][H][T].
__device__ __forceinline__ int64_t lse_index(const SeqInfo& si, int H, int p, int h, int n, int tau, int pos) {
  if (si.cu_seqlens) return (static_cast<int64_t>(p) * H + h) * si.T + tau;
  return ((static_cast<int64_t>(p) * si.nseq + n) * H + h) * si.S + pos;
}

// cos/sin of pos * inv_freq: the angle in double, reduced by whole turns in double,
// then the single-precision sincosf of the remainder (|remainder| <= pi).
__device__ __forceinline__ void angle_cos_sin(int pos, double inv_freq, float& c, float& s) {
  const double ang = static_cast<double>(pos) * inv_freq;
  const double turns = rint(ang * 0.15915494309189535);  // 1 / (2 pi)
  const double red = fma(-turns, 6.283185307179586, ang);
  sincosf(static_cast<float>(red), &s, &c);
}

// cos and sin of one rotation angle, each split into a float pair (hi + lo carries
// about 48 significant bits of the double value): hi = {c_hi, s_hi}, lo = {c_lo, s_lo}.
// Kept as two float2 arrays in shared memory (8-byte entries: a warp reading 32
// consecutive entries spreads over the banks; 16-byte entries at a stride of 8 would
// put every lane on the same four banks).
__device__ __forceinline__ void cos_sin_split(double c, double s, float2& hi, float2& lo) {
  const float ch = static_cast<float>(c), sh = static_cast<float>(s);
  hi = make_float2(ch, sh);
  lo = make_float2(static_cast<float>(c - static_cast<double>(ch)), static_cast<float>(s - static_cast<double>(sh)));
}

// One output of the rotate-half rotation of the pair (x1, x2) by (cos, sin):
// x1 cos - x2 sin (first half) or x2 cos + x1 sin (second half), rounded to fp32 and then
// to bf16 (round to nearest even), the chain of an fp64 evaluation.  The value is formed
// to about 2^-48 relative in float-float arithmetic: each product of a bf16 input with
// the high part of cos / sin is split exactly into a rounded product and its error
// (fma), the two products are added with an exact two-sum, and the small terms (the
// errors and the low parts) are added to the error; the final fp32 addition then rounds
// the value the way an fp64 evaluation would, except within ~2^-48 of an fp32 rounding
// midpoint, and the bf16 result differs only if that also sits on a bf16 tie.
__device__ __forceinline__ __nv_bfloat16 rotate_round_exact(float x1, float x2, float2 hi, float2 lo, bool second) {
  const float4 cs = make_float4(hi.x, lo.x, hi.y, lo.y);
  // first half: a*c - b*s with (a, b) = (x1, x2); second half: a*c + b*s with (a, b) = (x2, x1)
  const float a = second ? x2 : x1;
  const float bneg = second ? -x1 : x2;  // the term subtracted: b * s with b = bneg
  const float p1 = __fmul_rn(a, cs.x);
  const float e1 = __fmaf_rn(a, cs.x, -p1);
  const float p2 = __fmul_rn(bneg, cs.z);
  const float e2 = __fmaf_rn(bneg, cs.z, -p2);
  // two-sum of p1 - p2
  const float t = __fsub_rn(p1, p2);
  const float bv = __fsub_rn(t, p1);
  const float err = __fadd_rn(__fsub_rn(p1, __fsub_rn(t, bv)), __fsub_rn(-p2, bv));
  const float small = __fmaf_rn(a, cs.y, __fmaf_rn(-bneg, cs.w, __fsub_rn(e1, e2)));
  return __float2bfloat16_rn(__fadd_rn(t, __fadd_rn(err, small)));
}

// The same rounding, fast in the common case.  The plain fp32 evaluation differs from
// the exact value by less than (|x1| + |x2|) * 2^-21 (two rounded products, cos / sin
// rounded to fp32), so its bf16 rounding is the exact value's unless it lies that close
// to a bf16 rounding midpoint (the value with the dropped 16 bits equal to 0x8000);
// about 1.4e-3 of the elements do, and take the float-float path above.
__device__ __forceinline__ __nv_bfloat16 rotate_round(__nv_bfloat16 x1b, __nv_bfloat16 x2b, float2 hi, float2 lo,
                                                      bool second) {
  const float x1 = __bfloat162float(x1b), x2 = __bfloat162float(x2b);
  const float y = second ? fmaf(x2, hi.x, x1 * hi.y) : fmaf(x1, hi.x, -x2 * hi.y);
  const float mid = __uint_as_float((__float_as_uint(y) & 0xFFFF0000u) | 0x8000u);
  if (fabsf(y - mid) > (fabsf(x1) + fabsf(x2)) * 4.76837158203125e-07f) return __float2bfloat16_rn(y);  // 2^-21
  return rotate_round_exact(x1, x2, hi, lo, second);
}

// Eight (x1, x2) pairs of one head row (x1 = a[e] in the first half, x2 = b[e] in the
// second): oa[e] = x1 c - x2 s, ob[e] = x2 c + x1 s, rounded as rotate_round rounds them.
// All sixteen results are first evaluated in plain fp32 and packed; the elements within
// the error bound of a bf16 midpoint are only flagged, and redone after the packing in
// float-float arithmetic, so the common path carries no branch per element.
// lo is read in the rare path only: a register array or a pointer to shared memory.
template <typename LoT>
__device__ __forceinline__ void rotate8_round(const uint4& av, const uint4& bv, const float2 (&hi)[8], const LoT& lo,
                                              uint4& oa, uint4& ob) {
  const __nv_bfloat16* xa = reinterpret_cast<const __nv_bfloat16*>(&av);
  const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(&bv);
  float y1[8], y2[8];
  uint32_t near = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float x1 = __bfloat162float(xa[e]), x2 = __bfloat162float(xb[e]);
    y1[e] = fmaf(x1, hi[e].x, -x2 * hi[e].y);
    y2[e] = fmaf(x2, hi[e].x, x1 * hi[e].y);
    const float bound = (fabsf(x1) + fabsf(x2)) * 4.76837158203125e-07f;  // 2^-21
    const float m1 = __uint_as_float((__float_as_uint(y1[e]) & 0xFFFF0000u) | 0x8000u);
    const float m2 = __uint_as_float((__float_as_uint(y2[e]) & 0xFFFF0000u) | 0x8000u);
    near |= (fabsf(y1[e] - m1) > bound ? 0u : 1u) << e;
    near |= (fabsf(y2[e] - m2) > bound ? 0u : 1u) << (8 + e);
  }
  oa = make_uint4(pack_bf16x2(y1[0], y1[1]), pack_bf16x2(y1[2], y1[3]), pack_bf16x2(y1[4], y1[5]),
                  pack_bf16x2(y1[6], y1[7]));
  ob = make_uint4(pack_bf16x2(y2[0], y2[1]), pack_bf16x2(y2[2], y2[3]), pack_bf16x2(y2[4], y2[5]),
                  pack_bf16x2(y2[6], y2[7]));
  if (near != 0u) {
    __nv_bfloat16* ya = reinterpret_cast<__nv_bfloat16*>(&oa);
    __nv_bfloat16* yb = reinterpret_cast<__nv_bfloat16*>(&ob);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float x1 = __bfloat162float(xa[e]), x2 = __bfloat162float(xb[e]);
      if (near & (1u << e)) ya[e] = rotate_round_exact(x1, x2, hi[e], lo[e], false);
      if (near & (1u << (8 + e))) yb[e] = rotate_round_exact(x1, x2, hi[e], lo[e], true);
    }
  }
}

// Trunk-key limit of block-draft query row r of a sequence whose block rows start at
// qstart (a multiple of Bs) and whose context has klen keys: its block's anchor,
// clamped to [0, klen - 1] (-1, no trunk key, for an empty context).
__device__ __forceinline__ int block_row_limit(const Geometry& g, int qstart, int r, int klen) {
  const int a = __ldg(g.anchors + (qstart + r) / g.Bs);
  return min(max(a, 0), klen - 1);
}

// First trunk key of a block-draft row whose last trunk key is lim: 0, or for a
// sliding-window layer lim - window + 1 (at least 0).
__device__ __forceinline__ int block_row_start(const Geometry& g, int lim) {
  return g.window > 0 ? max(0, lim - g.window + 1) : 0;
}

// RoPE position of that row: the clamped anchor (0 for an empty context) plus the
// row's index in its block.
__device__ __forceinline__ int block_row_position(const Geometry& g, int qstart, int r, int klen) {
  return max(block_row_limit(g, qstart, r, klen), 0) + r % g.Bs;
}

}  // namespace ttt
