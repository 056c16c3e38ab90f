// Device-side helpers for the sm_100a kernels: status word, bounded
// mbarrier waits, TMA (cp.async.bulk[.tensor]) and tcgen05/TMEM wrappers.
// Everything here is inline PTX written for this library.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/qsa.h"

namespace qsa {

// ---------------------------------------------------------------- status
// First error recorded wins; the host reads and clears it with
// qsa_get_device_status().
__device__ int g_status = 0;
__device__ int g_status_detail = 0;
// Global time (ns) of the latest timeout any wait recorded: a wait gives up
// early only on a timeout recorded after it started, so a timeout left in the
// status word by an earlier kernel does not cut short the waits of later ones.
__device__ unsigned long long g_timeout_at = 0;

__device__ __forceinline__ uint64_t globaltimer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void report(int code, int detail)
{
    if (code == QSA_ERR_TIMEOUT) atomicMax(&g_timeout_at, (unsigned long long)globaltimer_ns());
    if (atomicCAS(&g_status, 0, code) == 0) atomicExch(&g_status_detail, detail);
}

// Default limit of every bounded wait: 1 s of wall time.
constexpr uint64_t kWaitLimitNs = 1000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// --------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------- register redistribution
// Every warp of a warpgroup executes the same one; an increase waits until
// the warpgroups that decrease have released enough of the CTA's launch
// registers, so the kernel's split must fit its launch allocation.
template <int N>
__device__ __forceinline__ void setmaxnreg_inc()
{
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

template <int N>
__device__ __forceinline__ void setmaxnreg_dec()
{
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// ------------------------------------------------- split cluster barrier
// Every thread of every CTA in the cluster arrives once, then waits once,
// before the next barrier of the cluster.
__device__ __forceinline__ void cluster_arrive_release()
{
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}

__device__ __forceinline__ void cluster_wait_acquire()
{
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// ---------------------------------------------- programmatic dependent launch
// A kernel launched with programmatic stream serialization may start while
// the previous kernel on the stream is still running.  It must not touch
// global memory that earlier work on the stream writes or reads before
// grid_dependency_wait() returns (which is immediate without such a
// dependency).
__device__ __forceinline__ void grid_dependency_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Lets the next kernel on the stream be scheduled early; it still waits for
// this grid's completion in its grid_dependency_wait().
__device__ __forceinline__ void grid_launch_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" :::);
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile(
        "{\n\t.reg .b64 st;\n\t"
        "mbarrier.arrive.release.cta.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile(
        "{\n\t.reg .b64 st;\n\t"
        "mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
            smem_u32(bar)),
        "r"(bytes)
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// try_wait that lets the hardware park the thread for up to `hint_ns`
// (woken early when the phase completes), so a waiting warp does not spin
// on the issue slots the working warps need.
__device__ __forceinline__ bool mbar_try_wait_hint(uint32_t bar, uint32_t parity, uint32_t hint_ns)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase of `parity` to complete.  Returns false (and
// records QSA_ERR_TIMEOUT with `where`) when the limit runs out, or early if
// *abort is set (another wait of this CTA gave up) or, after the first
// millisecond, if any CTA has recorded a timeout since this wait began.
// Sets *abort on a timeout so that the other waits of the CTA give up
// immediately.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort,
                                          int where, uint64_t limit_ns = kWaitLimitNs)
{
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait(a, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (abort && *abort) return false;
        if (mbar_try_wait_hint(a, parity, 200000u)) return true;
        const uint64_t dt = globaltimer_ns() - t0;
        if (dt > 1000000ull && *(volatile unsigned long long *)&g_timeout_at >= t0) {
            if (abort) *abort = 1;
            return false;
        }
        if (dt > limit_ns) {
            if (abort) *abort = 1;
            report(QSA_ERR_TIMEOUT, where);
            return false;
        }
    }
}

// ------------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int c0, int c1)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cta.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int c0, int c1, int c2)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cta.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

// Untiled bulk copy global -> this CTA's shared memory, completing on an
// mbarrier (both addresses 16-byte aligned, bytes a multiple of 16).
// Barrier `id` (1..15) among `count` threads (a multiple of 32) of the CTA.
__device__ __forceinline__ void named_barrier_sync(int id, int count)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// 16-byte asynchronous copy global -> shared (both 16-byte aligned); with
// valid false nothing is read and the 16 bytes are zero-filled.
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src, bool valid)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src),
                 "r"(valid ? 16 : 0)
                 : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

// Waits until at most N of this thread's committed groups are pending.
template <int N>
__device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- tcgen05
// Shared-memory matrix descriptor (sm_100 UMMA): start address, leading and
// stride byte offsets (16-byte units), version 1, layout type in bits 61-63.
constexpr uint32_t kLayoutSwizzle128B = 2;

__host__ __device__ __forceinline__ uint64_t umma_smem_desc(uint32_t saddr, uint32_t lbo_bytes,
                                                   uint32_t sbo_bytes)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;                       // descriptor version (sm_100)
    d |= (uint64_t)kLayoutSwizzle128B << 61;
    return d;
}

// Instruction descriptor for kind::f16 with bf16 A/B and fp32 accumulate.
// a_mn / b_mn select MN-major operands.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N, int a_mn, int b_mn)
{
    return (1u << 4)                 // D format: f32
           | (1u << 7)               // A format: bf16
           | (1u << 10)              // B format: bf16
           | ((uint32_t)a_mn << 15)  // A major
           | ((uint32_t)b_mn << 16)  // B major
           | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]^T  (both K-major unless the idesc says otherwise)
__device__ __forceinline__ void umma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// The mbarrier completes once every tcgen05 op issued so far by this thread
// has completed.
__device__ __forceinline__ void umma_commit(uint64_t *bar)
{
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets lane
// (warp's lane quarter + i), columns [col, col+32).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
        : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}

// Nonzero in one lane (the same one every time) of a converged warp: an
// MMA warp runs its waits and descriptor arithmetic together, warp-uniform,
// and lets the elected lane issue the single-thread tcgen05 ops.
__device__ __forceinline__ uint32_t elect_one()
{
    uint32_t pred = 0;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "elect.sync _|p, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(pred));
    return pred;
}

// ------------------------------------------------------------- misc math
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);   // .x = lo (low half)
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi)
{
    __half2 v = __floats2half2_rn(lo, hi);   // .x = lo (low half)
    return *reinterpret_cast<uint32_t *>(&v);
}

// ---------------------------------------------- rotated fp8 KV (decode option)
// Unnormalised Walsh-Hadamard transform of a warp's 32*V values, element
// e = V*lane + k in x[k], in place: for len = 1, 2, ..., 16V every pair
// (j, j + len) with j mod 2 len < len becomes (x_j + x_{j+len},
// x_j - x_{j+len}) -- stage by stage in increasing len, so every output is
// a fixed sequence of fp32 additions and the codes derived from it are
// reproducible on any implementation that follows the same order.
template <int V>
__device__ __forceinline__ void fwht_warp(float (&x)[V])
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int len = 1; len < V; len <<= 1) {
#pragma unroll
        for (int k = 0; k < V; k++) {
            if (k & len) continue;
            const float a = x[k], b = x[k + len];
            x[k] = a + b;
            x[k + len] = a - b;
        }
    }
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {   // len = V * m
#pragma unroll
        for (int k = 0; k < V; k++) {
            const float y = __shfl_xor_sync(0xffffffffu, x[k], m);
            x[k] = (lane & m) ? y - x[k] : x[k] + y;
        }
    }
}

// Two fp32 values -> fp8 e4m3 codes (lo in the low byte): nearest, ties to
// even, saturating to +-448.
__device__ __forceinline__ uint16_t cvt_e4m3x2(float lo, float hi)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Two fp8 e4m3 codes (low byte first) -> f16x2 (exact).
__device__ __forceinline__ uint32_t cvt_e4m3x2_f16x2(uint16_t v)
{
    uint32_t r;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(v));
    return r;
}

__device__ __forceinline__ float fast_exp2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float max3f(float a, float b, float c)
{
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Largest of 32 values: a tree of 3-input maxima (depth 4, 16 instructions).
__device__ __forceinline__ float max32(const float (&x)[32])
{
    float t[11];
#pragma unroll
    for (int q = 0; q < 10; q++) t[q] = max3f(x[3 * q], x[3 * q + 1], x[3 * q + 2]);
    t[10] = fmaxf(x[30], x[31]);
    const float u0 = max3f(t[0], t[1], t[2]), u1 = max3f(t[3], t[4], t[5]);
    const float u2 = max3f(t[6], t[7], t[8]), u3 = fmaxf(t[9], t[10]);
    return fmaxf(max3f(u0, u1, u2), u3);
}

// ---- packed fp32 pairs (sm_100 f32x2 arithmetic)
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float &lo, float &hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// 2^x for a pair of fp32 values with x <= 8, on the FMA pipe instead of the
// MUFU unit.  Cody-Waite style argument reduction: x = n + f with
// n = round(x) (obtained by adding 1.5 * 2^23, which leaves n in the low
// mantissa bits) and f in [-1/2, 1/2]; 2^f from a degree-3 polynomial whose
// coefficients were fitted for this library (Chebyshev-node weighted least
// squares towards minimax relative error; max relative error 7.5e-5 on
// [-1/2, 1/2], far below the 2^-9 of the bf16 rounding that follows); 2^n
// is applied by adding n to the exponent field.  x is clamped at -126 so
// the exponent never underflows (2^-126 is negligible next to the row's
// largest term, which is >= 1).
__device__ __forceinline__ uint64_t exp2_poly_x2(uint64_t x2)
{
    float x0, x1;
    f2_unpack(x2, x0, x1);
    const uint64_t x = f2_pack(fmaxf(x0, -126.f), fmaxf(x1, -126.f));
    const uint64_t round_c = f2_pack(12582912.f, 12582912.f);
    const uint64_t t = f2_add(x, round_c);
    const uint64_t f = f2_sub(x, f2_sub(t, round_c));
    uint64_t p = f2_fma(f2_pack(5.517164618e-02f, 5.517164618e-02f), f,
                        f2_pack(2.426111251e-01f, 2.426111251e-01f));
    p = f2_fma(p, f, f2_pack(6.932609677e-01f, 6.932609677e-01f));
    p = f2_fma(p, f, f2_pack(9.999280572e-01f, 9.999280572e-01f));
    float t0, t1, p0, p1;
    f2_unpack(t, t0, t1);
    f2_unpack(p, p0, p1);
    // p * 2^n: n's low bits sit in t's mantissa; one multiply-add per value
    // moves them into the exponent field (the wrap-around of the product
    // is the intended modular arithmetic)
    return f2_pack(__uint_as_float(__float_as_uint(t0) * 8388608u + __float_as_uint(p0)),
                   __uint_as_float(__float_as_uint(t1) * 8388608u + __float_as_uint(p1)));
}

// 2^x for a pair of fp32 values with x <= 0 (a softmax weight), on the FMA
// pipe, accurate enough to stand in for ex2.approx in sums that decide a
// selection: the same argument reduction as exp2_poly_x2 (x = n + f, n =
// round(x), f in [-1/2, 1/2]), then 2^f from a degree-5 polynomial with
// coefficients fitted for this library (Lawson-weighted least squares on
// Chebyshev nodes towards minimax relative error: 7.5e-8 in exact
// arithmetic, 2.1e-7 with fp32 Horner steps, against 2^-22 for ex2.approx);
// x is clamped at -126 (a weight below 2^-126 is negligible in the sum).
__device__ __forceinline__ uint64_t exp2_poly5_x2(uint64_t x2)
{
    float x0, x1;
    f2_unpack(x2, x0, x1);
    const uint64_t x = f2_pack(fmaxf(x0, -126.f), fmaxf(x1, -126.f));
    const uint64_t round_c = f2_pack(12582912.f, 12582912.f);
    const uint64_t t = f2_add(x, round_c);
    const uint64_t f = f2_sub(x, f2_sub(t, round_c));
    uint64_t p = f2_fma(f2_pack(1.327647152e-03f, 1.327647152e-03f), f,
                        f2_pack(9.6755413307e-03f, 9.6755413307e-03f));
    p = f2_fma(p, f, f2_pack(5.550713275e-02f, 5.550713275e-02f));
    p = f2_fma(p, f, f2_pack(2.4022119724e-01f, 2.4022119724e-01f));
    p = f2_fma(p, f, f2_pack(6.9314696706e-01f, 6.9314696706e-01f));
    p = f2_fma(p, f, f2_pack(1.0000000717f, 1.0000000717f));
    float t0, t1, p0, p1;
    f2_unpack(t, t0, t1);
    f2_unpack(p, p0, p1);
    return f2_pack(__uint_as_float(__float_as_uint(t0) * 8388608u + __float_as_uint(p0)),
                   __uint_as_float(__float_as_uint(t1) * 8388608u + __float_as_uint(p1)));
}

// 2^x of a pair: on the FMA pipe (exp2_poly5_x2) when poly, else on MUFU
// (in unrolled loops the choice folds away at compile time).
__device__ __forceinline__ uint64_t exp2_pair(bool poly, uint64_t x2)
{
    if (poly) return exp2_poly5_x2(x2);
    float a, b;
    f2_unpack(x2, a, b);
    return f2_pack(fast_exp2(a), fast_exp2(b));
}

}  // namespace qsa
