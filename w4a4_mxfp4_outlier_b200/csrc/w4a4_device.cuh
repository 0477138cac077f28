// Device-side helpers shared by the sm_100a kernels of libw4a4: mbarriers with
// bounded waits, TMA / bulk copies, tcgen05 (TMEM allocation, MMA, copies,
// loads) and the shared-memory / instruction descriptors the 5th-generation
// tensor cores read.  Everything here is inline PTX written for sm_100a.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace w4a4 {

// ---------------------------------------------------------------------------
// Error word.  Kernels that give up a bounded wait set a bit here and return;
// the host reads it with w4a4_last_error().  Never a trap.
// ---------------------------------------------------------------------------
enum : uint32_t {
  DEVERR_TIMEOUT_PRODUCER = 1u << 0,
  DEVERR_TIMEOUT_MMA = 1u << 1,
  DEVERR_TIMEOUT_EPILOGUE = 1u << 2,
  DEVERR_TIMEOUT_PREP = 1u << 3,
  DEVERR_NONFINITE_CALIB = 1u << 4,   // calibration magnitude was inf or NaN
  DEVERR_BAD_ARG = 1u << 8,
};
// The library is compiled as one translation unit (csrc/libw4a4.cu), so this
// single definition is the word every kernel and the host accessor use.
static __device__ uint32_t g_device_error = 0u;

// Wall time on %globaltimer before a wait is abandoned: about 2 s, unless a
// failure-detection test shortened it (w4a4_test_fault).
constexpr uint64_t kWaitLimitNs = 2000000000ull;
static __device__ uint64_t g_wait_limit_ns = kWaitLimitNs;

// Failure-detection test hook (w4a4_test_fault): while bit 0 is set, the
// activation-prep producer issues no row copies, so its consumers' waits run
// out.  Zero in normal use.
enum : uint32_t { FAULT_PREP_SKIP_LOADS = 1u << 0 };
static __device__ uint32_t g_fault_mask = 0u;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking check: has the phase with the given parity completed?
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete.  Gives up after
// g_wait_limit_ns, or as soon as *abort becomes non-zero (another role gave
// up): returns false then, after recording `err_bit` in the device error word.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  volatile uint32_t* abort, uint32_t err_bit) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(a, parity)) return true;
    if ((it & 63u) == 0) {
      if (abort != nullptr && *abort) return false;
      if (globaltimer_ns() - t0 > *static_cast<volatile uint64_t*>(&g_wait_limit_ns)) {
        atomicOr(&g_device_error, err_bit);
        if (abort != nullptr) *abort = 1u;
        return false;
      }
    }
  }
}

// The same wait run by every lane of a converged warp; the result is made
// warp-uniform (a lane that timed out makes the whole warp give up).
__device__ __forceinline__ bool warp_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  volatile uint32_t* abort, uint32_t err_bit) {
  const bool ok = mbar_wait_bounded(bar, parity, abort, err_bit);
  return __all_sync(0xFFFFFFFFu, ok);
}

// Programmatic dependent launch.  A kernel launched with the attribute may
// start (its CTAs take SMs as the previous kernel's CTAs leave) before the
// previous kernel in the stream has finished; it runs only shared-memory and
// tensor-memory setup until pdl_wait(), which returns once the grids it
// depends on have completed and their memory is visible, and touches global
// memory only after it.  Without the attribute both are no-ops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// lets the next kernel in the stream start launching
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// One lane of a converged warp (always the same lane for a full mask).  The
// single-thread tcgen05 and TMA instructions are issued under it while the
// rest of the warp stays converged with the issuer: a lone lane running the
// issue loop in a divergent branch was measured to leave the tensor pipe idle
// for about a third of the time at every barrier wait of that lane.
__device__ __forceinline__ bool elect_one() {
  uint32_t p = 0;
  asm volatile(
      "{\n\t.reg .pred P;\n\telect.sync _|P, 0xffffffff;\n\tselp.b32 %0, 1, 0, P;\n\t}"
      : "=r"(p));
  return p != 0;
}

// ---------------------------------------------------------------------------
// GELU of the FFN between the two projections, for a bf16 input y, as the
// bf16 value nearest the exact
//   gelu(y) = 0.5 y (1 + tanh(u)) = y / (1 + exp(-2u)),  u = sqrt(2/pi) (y + 0.044715 y^3)
// (tanh form), ties to even.  It is a function of 16 bits, so kernels may
// evaluate it any way that returns that value:
//  * 2^-12 <= |y| < 16: a 4096-entry table (sign, 16 binades, 128
//    mantissas) in shared memory, filled per CTA with gelu_bf16_exact;
//  * |y| < 2^-12: gelu(y) = y/2 + d with 0 < d <= 0.4 y^2, far below half a
//    bf16 spacing of y/2, so the result is y/2, except that when y/2 falls
//    exactly between two bf16 values (only below 2^-125) d breaks the tie
//    toward +inf;
//  * |y| >= 16: gelu(y) = y (1 - e), e < 1e-137, rounds to y; for y <= -16
//    |gelu(y)| < 1e-136 rounds to -0.  +inf -> +inf, -inf and NaN -> NaN
//    (the value of the second form).
// ---------------------------------------------------------------------------
constexpr uint32_t kGeluTabExp0 = 115;      // biased exponent of 2^-12
constexpr int kGeluTabEntries = 4096;       // 2 signs x 16 binades x 128 mantissas
constexpr uint32_t kGeluTabBase = kGeluTabExp0 << 7;

// float64 -> bf16 bits, round to nearest even, in one rounding: truncate to
// float32 and set its last bit if anything was cut off (round to odd keeps
// the information a second rounding to 8 bits needs), then round to bf16
__device__ __forceinline__ uint32_t f64_to_bf16_rn(double g) {
  float f = __double2float_rz(g);
  if (static_cast<double>(f) != g) f = __uint_as_float(__float_as_uint(f) | 1u);
  return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(f)));
}

// gelu of the bf16 value with bits b (low 16 bits), for 2^-12 <= |y| < 16:
// float64 evaluation (relative error below 2^-40; every such input's value
// lies at least 1e-4 of a bf16 spacing from a rounding boundary) rounded once
__device__ __noinline__ uint32_t gelu_bf16_exact(uint32_t b) {
  const double y = static_cast<double>(__uint_as_float(b << 16));
  const double u = 0.7978845608028654 * (y + 0.044715 * (y * y * y));
  return f64_to_bf16_rn(y / (1.0 + exp(-2.0 * u)));
}

// the inputs outside the table (see above)
__device__ __forceinline__ uint32_t gelu_bf16_outside(uint32_t b) {
  const uint32_t mag = b & 0x7FFFu;
  if (mag < kGeluTabBase) {
    if (mag == 0u) return b;                                   // +-0
    uint32_t f = __float_as_uint(__fmul_rn(__uint_as_float(b << 16), 0.5f));   // exact
    f += (f >> 31) ? 0xFFFFFFFFu : 1u;                         // one float ulp toward +inf
    return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(f))));
  }
  if (mag > 0x7F80u || b == 0xFF80u) return 0x7FC0u;          // NaN, -inf
  return (b & 0x8000u) ? 0x8000u : b;
}

// entry i of the table: sign (i >> 11), offset (i & 2047) from 2^-12
__device__ __forceinline__ void gelu_table_fill(uint16_t* tab, int tid, int nthreads) {
  for (int i = tid; i < kGeluTabEntries; i += nthreads) {
    const uint32_t b = (static_cast<uint32_t>(i & 0x800) << 4) | (kGeluTabBase + (i & 0x7FF));
    tab[i] = static_cast<uint16_t>(gelu_bf16_exact(b));
  }
}

// barrier `id` (1..15) over the first `nthreads` threads that reach it (a
// multiple of 32; the other warps of the block do not take part)
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}

// table lookup for an input inside the table's range; `rel` = (b & 0x7FFF) -
// kGeluTabBase (< 2048 there).  Outside the range the index wraps and the
// caller must use gelu_bf16_outside instead.
__device__ __forceinline__ uint32_t gelu_bf16_table(uint32_t tab, uint32_t b, uint32_t rel) {
  return lds_u16(tab + 2u * ((rel & 0x7FFu) | ((b >> 4) & 0x800u)));
}

__device__ __forceinline__ uint32_t gelu_bf16(uint32_t tab, uint32_t b) {
  const uint32_t rel = (b & 0x7FFFu) - kGeluTabBase;
  return rel < 2048u ? gelu_bf16_table(tab, b, rel) : gelu_bf16_outside(b);
}

// ---------------------------------------------------------------------------
// TMA and bulk copies (global -> shared, completion counted on an mbarrier)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

// TMA tile store shared -> global (bulk-group completion, issuing thread only)
__device__ __forceinline__ void tma_store_2d(const void* tmap, uint32_t smem_src, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
               ::"l"(tmap), "r"(smem_src), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// this thread's committed bulk stores have finished reading shared memory
__device__ __forceinline__ void bulk_wait_group_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// this thread's committed bulk stores are complete
__device__ __forceinline__ void bulk_wait_group0() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
// generic-proxy shared-memory writes become visible to the async proxy (TMA)
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tma_load_2d(void* smem_dst, const void* tmap, uint64_t* bar,
                                            int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(tmap), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(smem_dst)),
      "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory, MMA, copies, loads
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_result)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 x bf16 -> f32.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= (A * SFA) (B * SFB)^T with packed E2M1 operands and one E8M0
// scale per 32 K (scale factors read from tensor memory).
__device__ __forceinline__ void mma_mxf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%5], "
      "[%6], p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Arrive once on `bar` when every tcgen05 operation issued so far by this
// thread has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Copy 32 rows x 16 bytes from shared memory into 32 lanes x 4 columns of
// tensor memory, replicated into all four 32-lane sub-partitions.
__device__ __forceinline__ void tc_cp_32x128b_warpx4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// Each thread of the warp reads 32 consecutive 32-bit columns of its lane.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// Each thread of the warp reads 16 consecutive 32-bit columns of its lane.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------
// CTA pairs (cluster of 2): tcgen05 cta_group::2 and cluster plumbing
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address of the same shared variable in CTA `cta` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t cta) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(cta));
  return r;
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}

// TMA load into this CTA's shared memory whose completion is counted on an
// mbarrier that may live in the pair's leader CTA (cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const void* tmap,
                                                 uint32_t mbar_cluster, int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(tmap), "r"(mbar_cluster), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_result)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_mxf4_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                              uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%5], "
      "[%6], p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Scale atoms into the tensor memory of both CTAs of the pair (each CTA's
// copy comes from the same shared-memory offset of that CTA).
__device__ __forceinline__ void tc_cp_pair_32x128b_warpx4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// Arrive on the mbarrier at the same offset in every CTA of `mask` once all
// tcgen05 operations issued so far by this thread have completed.
__device__ __forceinline__ void tc_commit_pair_multicast(uint64_t* bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"(mask)
      : "memory");
}

__device__ __forceinline__ void tc_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void spin_ns(uint64_t ns) {
  const uint64_t t0 = globaltimer_ns();
  while (globaltimer_ns() - t0 < ns) {
  }
}

// ---------------------------------------------------------------------------
// Descriptors
// ---------------------------------------------------------------------------
// Shared-memory matrix descriptor for a K-major operand tile stored with the
// 128-byte swizzle: rows of 128 bytes, 8-row groups 1024 bytes apart.  The
// tile base must be 1024-byte aligned; advancing along K inside the 128-byte
// row adds (bytes >> 4) to the start address.
__device__ __forceinline__ uint64_t sdesc_kmajor_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);      // start address
  d |= static_cast<uint64_t>(1u) << 16;                     // leading byte offset (unused)
  d |= static_cast<uint64_t>(1024u >> 4) << 32;             // stride byte offset: 8 rows
  d |= static_cast<uint64_t>(1u) << 46;                     // descriptor version (sm_100)
  d |= static_cast<uint64_t>(2u) << 61;                     // 128-byte swizzle
  return d;
}

// Descriptor for tcgen05.cp source data: 16-byte rows, contiguous, no swizzle
// (8-row core matrices 128 bytes apart, a single core matrix along K).
__device__ __forceinline__ uint64_t sdesc_sf_rows16(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(128u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  return d;
}

// Instruction descriptor, kind::f16 with bf16 inputs and f32 accumulation,
// both operands K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4)                                   // D format: f32
         | (1u << 7)                                 // A format: bf16
         | (1u << 10)                                // B format: bf16
         | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

// Instruction descriptor, kind::mxf4 (packed E2M1 x E2M1, E8M0 scales,
// K = 64 per instruction), both operands K-major.  sf ids pick the byte of
// the 32-bit tensor-memory word the scales start at.
__host__ __device__ constexpr uint32_t idesc_mxf4(int M, int N, uint32_t a_sf_id,
                                                  uint32_t b_sf_id) {
  return (b_sf_id << 4)                              // B scale byte
         | (1u << 7)                                 // A format: E2M1
         | (1u << 10)                                // B format: E2M1
         | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
         | (1u << 23)                                // scale format: E8M0
         | (static_cast<uint32_t>(M >> 4) << 24)     // M / 16
         | (a_sf_id << 29);                          // A scale byte
}

// ---------------------------------------------------------------------------
// Small numeric helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16_lo_to_f32(uint32_t pair) { return __uint_as_float(pair << 16); }
__device__ __forceinline__ float bf16_hi_to_f32(uint32_t pair) {
  return __uint_as_float(pair & 0xFFFF0000u);
}

// Eight f32 -> eight E2M1 codes packed in 32 bits, element i in bits
// [4i+3:4i].  Round to nearest even, saturating at +-6 (cvt.rn.satfinite;
// the first source operand of each cvt lands in the high nibble).
__device__ __forceinline__ uint32_t cvt_e2m1x8(float v0, float v1, float v2, float v3, float v4,
                                               float v5, float v6, float v7) {
  uint32_t r;
  asm("{\n\t.reg .b8 c0, c1, c2, c3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c3, %8, %7;\n\t"
      "mov.b32 %0, {c0, c1, c2, c3};\n\t}"
      : "=r"(r)
      : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
  return r;
}

// Maxima of magnitudes with NaN propagation (IEEE 754-2019 maximum): the
// maximum of a block that holds a NaN is NaN, of one that holds an infinity
// (and no NaN) +inf.  Three-input form: one instruction for three values.
__device__ __forceinline__ float max_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float max3_nan(float a, float b, float c) {
  float r;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// max |v| over 32 values, NaN-propagating (16 instructions)
__device__ __forceinline__ float block_absmax32(const float2 (&v)[16]) {
  float m[12];
#pragma unroll
  for (int i = 0; i < 5; ++i) {
    m[2 * i] = max3_nan(fabsf(v[3 * i].x), fabsf(v[3 * i].y), fabsf(v[3 * i + 1].x));
    m[2 * i + 1] = max3_nan(fabsf(v[3 * i + 1].y), fabsf(v[3 * i + 2].x), fabsf(v[3 * i + 2].y));
  }
  m[10] = fabsf(v[15].x);
  m[11] = fabsf(v[15].y);
  const float n0 = max3_nan(m[0], m[1], m[2]), n1 = max3_nan(m[3], m[4], m[5]);
  const float n2 = max3_nan(m[6], m[7], m[8]), n3 = max3_nan(m[9], m[10], m[11]);
  return max_nan(max3_nan(n0, n1, n2), n3);
}

// E8M0 scale code for a block maximum amax (>= 0, +inf or NaN):
// clamp(floor(log2 amax) - 2, -127, 127) + 127, read from the exponent field
// (0 for zero / subnormal maxima).  amax = +inf gives e = 127, code 254;
// amax = NaN gives 0xFF, E8M0's NaN, and the block's element codes are all
// zero (mx_nan_block_mask).
__device__ __forceinline__ uint32_t mx_scale_code(float amax) {
  const uint32_t b = __float_as_uint(amax) & 0x7FFFFFFFu;
  const uint32_t ebits = b >> 23;
  if (ebits == 255u) return b == 0x7F800000u ? 254u : 255u;
  return ebits > 2u ? ebits - 2u : 0u;
}

// 2^-e as a float for the scale code c = e + 127: exact for e <= 126, and
// 2^-127 (a subnormal float) for code 254 (and for the NaN code, whose
// element codes are zeroed anyway).
__device__ __forceinline__ float mx_inv_scale(uint32_t code) {
  return __uint_as_float(code < 254u ? (254u - code) << 23 : 0x00400000u);
}

// AND mask for a block's code words: 0 for a NaN block (scale code 0xFF).
__device__ __forceinline__ uint32_t mx_nan_block_mask(uint32_t code) {
  return code == 255u ? 0u : 0xFFFFFFFFu;
}

// bf16 bits of v rounded to nearest even; every NaN becomes 0x7FC0, the
// quiet NaN without payload (a NaN's sign and payload are not carried).
__device__ __forceinline__ uint32_t bf16_rn_bits(float v) {
  const uint32_t b = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v)));
  return v != v ? 0x7FC0u : b;
}

}  // namespace w4a4
