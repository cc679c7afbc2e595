// common.cuh -- small device helpers shared by the kernels of libmoe.so:
// bf16 unpacking, mbarrier / bulk-copy / programmatic-dependent-launch PTX
// wrappers, bounded waits and the workspace header.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/moe.h"

#define MOE_DEVINL __device__ __forceinline__

// MOE_CHECKS=1 builds the checked library (libmoe_checks.so): kernels also
// verify the index tables they otherwise trust -- caller-supplied expert
// offsets and slot ids on the grouped path, the route the one-token kernel
// forms -- and record MOE_ERR_DEVICE_CHECK in the status word, skipping the
// access, instead of reading or writing out of range.  The checks the normal
// build always makes (expert ids in the permutation, slot ids in the gather,
// the combine and the streaming kernel) stay as they are.
#ifndef MOE_CHECKS
#define MOE_CHECKS 0
#endif

// ---------------------------------------------------------------------------
// Workspace header: the first 12 KiB of every workspace.
constexpr int kMaxGridCtas = 960;  // most CTAs a grid barrier can serve
constexpr int kMaxExperts = 1024;
constexpr int kSpread = 8;         // counters one cross-CTA count is spread over
// One count of the one-token layer kernel, spread over kSpread counters on
// separate 128-byte lines (arrival i adds to counter i % kSpread), so that
// arrivals from many SMs do not queue on one L2 line.
struct SpreadCount {
    unsigned c[kSpread][32];
};
struct WsHeader {
    int status;             // device status word (moe_status), 0 = OK
    unsigned route_arrive;  // last-block hand-off counter of the top-k kernel
    unsigned decode_arrive; // last-block hand-off counter of the decode kernel
    unsigned sched[8];      // work-item counters of the grouped GEMMs (next, done) x 3
    unsigned decode_seq;    // one-token layer: number of the last call on this workspace
    unsigned pad0[20];
    unsigned bar_go;        // grid barrier: generation released so far (own 128-byte line)
    unsigned pad1[31];
    unsigned bar_flag[kMaxGridCtas];  // grid barrier: generation each CTA has reached
    // one-token layer: router logits published, per call (call number mod 4;
    // each call clears the count two calls ahead)
    SpreadCount xcnt[4];
    unsigned pad2[1024];
};
static_assert(sizeof(WsHeader) == 12288, "header is 12 KiB");
static_assert(offsetof(WsHeader, xcnt) == 4096, "spread counters on whole lines");

// Bounded waits give up after this many nanoseconds (globaltimer) and record
// MOE_ERR_TIMEOUT; no correct launch comes anywhere near it.  The limit is a
// device variable (2 s) that a test hook may shorten.
#define MOE_WAIT_LIMIT_NS 2000000000ull
__device__ unsigned long long g_moe_wait_limit_ns = MOE_WAIT_LIMIT_NS;

MOE_DEVINL unsigned long long wait_limit_ns()
{
    return *(volatile unsigned long long *)&g_moe_wait_limit_ns;
}

MOE_DEVINL uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

MOE_DEVINL void set_status(int *status, int code)
{
    if (status)
        atomicCAS(status, 0, code);
}

// ---------------------------------------------------------------------------
// bf16 helpers: a bf16 value is the upper half of a float32.
MOE_DEVINL float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
MOE_DEVINL float bf16hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

MOE_DEVINL uint16_t f32_to_bf16_rn(float f)
{
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x7fffffu))  // NaN stays NaN
        return (uint16_t)((u >> 16) | 0x40u);
    uint32_t r = u + 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(r >> 16);
}

// 8 bf16 (one 16-byte vector) times 8 floats, accumulated into acc.
MOE_DEVINL float dot8_bf16(const uint4 w, const float *x, float acc)
{
    acc = fmaf(bf16lo(w.x), x[0], acc);
    acc = fmaf(bf16hi(w.x), x[1], acc);
    acc = fmaf(bf16lo(w.y), x[2], acc);
    acc = fmaf(bf16hi(w.y), x[3], acc);
    acc = fmaf(bf16lo(w.z), x[4], acc);
    acc = fmaf(bf16hi(w.z), x[5], acc);
    acc = fmaf(bf16lo(w.w), x[6], acc);
    acc = fmaf(bf16hi(w.w), x[7], acc);
    return acc;
}

// Paired float32 arithmetic (sm_100): two float32 lanes in one 64-bit
// register, low half first.  ffma2: both halves a*b + c, each rounded once.
MOE_DEVINL uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
// The two bf16 of a 32-bit word (element 0 in the low half) as a float32 pair.
MOE_DEVINL uint64_t bf16x2_pair(uint32_t v)
{
    return ((uint64_t)(v & 0xffff0000u) << 32) | (uint64_t)(v << 16);
}
MOE_DEVINL uint64_t f32_pair(float lo, float hi)
{
    return ((uint64_t)__float_as_uint(hi) << 32) | (uint64_t)__float_as_uint(lo);
}
MOE_DEVINL float pair_lo(uint64_t p) { return __uint_as_float((uint32_t)p); }
MOE_DEVINL float pair_hi(uint64_t p) { return __uint_as_float((uint32_t)(p >> 32)); }

MOE_DEVINL float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch.  griddepcontrol.wait returns once every
// grid this one depends on has completed and its memory is visible; it is a
// no-op when the kernel was launched without the attribute.
MOE_DEVINL void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
MOE_DEVINL void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------------------
// Shared-memory mbarriers and bulk asynchronous copies (no multicast).
MOE_DEVINL uint32_t smem_addr(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

MOE_DEVINL void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

MOE_DEVINL void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

MOE_DEVINL void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

MOE_DEVINL void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

MOE_DEVINL bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase of `bar` with the given parity to complete.  Gives up
// after the wait limit, records MOE_ERR_TIMEOUT and returns false.
MOE_DEVINL bool mbar_wait(uint64_t *bar, uint32_t parity, int *status)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = global_ns();
    const uint64_t lim = wait_limit_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_ns() - t0 > lim) {
            set_status(status, MOE_ERR_TIMEOUT);
            return false;
        }
    }
    return true;
}

// mbar_wait that also ends (false) once the CTA's abort flag is set, so a
// warp that waits on a slot other warps gave up on leaves promptly.
MOE_DEVINL bool mbar_wait_live(uint64_t *bar, uint32_t parity, const int *abort, int *status)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = global_ns();
    const uint64_t lim = wait_limit_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (*(const volatile int *)abort)
            return false;
        if (global_ns() - t0 > lim) {
            set_status(status, MOE_ERR_TIMEOUT);
            return false;
        }
    }
    return true;
}

// L2 policy for weights streamed exactly once: evict first.
MOE_DEVINL uint64_t l2_evict_first_policy()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// L2 policy for small weights every call reads again (the router): evict last.
MOE_DEVINL uint64_t l2_evict_last_policy()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// Global -> shared bulk copy of `bytes` (multiple of 16, both addresses
// 16-byte aligned); completion is counted on `bar` as transaction bytes.
MOE_DEVINL void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar, uint64_t pol)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(pol)
        : "memory");
}

// The same without a cache hint (data other calls read again soon).
MOE_DEVINL void bulk_g2s_plain(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1], %2, [%3];" ::"r"(smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

MOE_DEVINL void named_bar_sync(int id, int nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

MOE_DEVINL unsigned ld_acquire_u32(const unsigned *p)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

MOE_DEVINL unsigned ld_relaxed_u32(const unsigned *p)
{
    unsigned v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

MOE_DEVINL void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }
// One-sided fences: release orders this thread's earlier accesses (and, by
// cumulativity, those it has observed, e.g. through a CTA barrier) before its
// later writes; acquire orders its earlier reads before its later accesses.
MOE_DEVINL void fence_release_gpu() { asm volatile("fence.release.gpu;" ::: "memory"); }
MOE_DEVINL void fence_acquire_gpu() { asm volatile("fence.acquire.gpu;" ::: "memory"); }

// Release store: a gpu-scope acq_rel fence, then a relaxed store.
MOE_DEVINL void st_release_u32(unsigned *p, unsigned v)
{
    fence_acq_rel_gpu();
    asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

MOE_DEVINL unsigned long long ld_relaxed_u64(const unsigned long long *p)
{
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

MOE_DEVINL void st_relaxed_u64(unsigned long long *p, unsigned long long v)
{
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Spin (bounded) on relaxed loads until *p == want, then one acq_rel fence
// (acquire).  Records MOE_ERR_TIMEOUT and returns false when
// wait limit passes first.
MOE_DEVINL bool wait_flag_eq(const unsigned *p, unsigned want, int *status)
{
    if (ld_relaxed_u32(p) != want) {
        const uint64_t t0 = global_ns();
        const uint64_t lim = wait_limit_ns();
        while (ld_relaxed_u32(p) != want) {
            if (global_ns() - t0 > lim) {
                set_status(status, MOE_ERR_TIMEOUT);
                return false;
            }
            __nanosleep(20);
        }
    }
    fence_acq_rel_gpu();
    return true;
}

// Balanced split of n items over G parts: part b gets [split_lo(n,G,b), split_lo(n,G,b+1)).
MOE_DEVINL unsigned split_lo(unsigned n, unsigned G, unsigned b)
{
    const unsigned q = n / G, r = n % G;
    return q * b + (b < r ? b : r);
}

// Shared -> global bulk reduction: dst[i] += src[i] for `bytes` of float32
// (both 16-byte aligned, bytes a multiple of 16), done by the TMA unit at L2 in
// line-sized pieces; tracked as a bulk async-group of the issuing thread.
MOE_DEVINL void bulk_reduce_add_f32(float *dst, const float *src, uint32_t bytes)
{
    asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(
                     dst),
                 "r"(smem_addr(src)), "r"(bytes)
                 : "memory");
}
// Shared -> global bulk copy (TMA) of `bytes` (16-byte aligned, a multiple of
// 16), tracked as a bulk async-group of the issuing thread.
MOE_DEVINL void bulk_s2g(void *dst, const void *src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
                 "r"(smem_addr(src)), "r"(bytes)
                 : "memory");
}
MOE_DEVINL void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until every bulk async-group of this thread is complete (its writes done).
MOE_DEVINL void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Generic-proxy writes to shared memory become visible to the async proxy.
MOE_DEVINL void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
// Async-proxy writes to global memory ordered before later generic accesses.
MOE_DEVINL void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

// y[0..3] += v (16-byte aligned float32 vector), one vector reduction.
MOE_DEVINL void red_add_v4(float *y, float v0, float v1, float v2, float v3)
{
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(y), "f"(v0), "f"(v1),
                 "f"(v2), "f"(v3)
                 : "memory");
}

MOE_DEVINL uint4 ld_nc_v4(const void *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}
