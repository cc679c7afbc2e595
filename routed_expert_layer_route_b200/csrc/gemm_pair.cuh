// gemm_pair.cuh -- the gate/up grouped GEMM of the large-batch expert FFN on
// CTA pairs: tcgen05.mma with cta_group::2, one 256-row weight tile per MMA.
//
// Expert structure ("Channel Selection for Mixture-of-Experts Decoding Needs
// No Calibration Data", section 2 "Background"): for expert e with n_e routed
// token rows X_e, G = W_gate[e] X_e^T and U = W_up[e] X_e^T ([I x n_e],
// K = d), H = silu(G) * U stored bf16 in the slot order of the counting sort
// -- the contraction k_gemm1 (grouped.cuh) computes on single CTAs.
//
// Here the two CTAs of a cluster share one MMA of M = 256 weight rows x
// N <= 256 tokens: CTA r holds weight rows [128 r, 128 r + 128) of the tile
// (gate and up) and tokens [N/2 r, N/2 r + N/2) in its shared memory; the
// product lands in each CTA's tensor memory for its own 128 rows and all N
// tokens.  Per CTA and K step that is 48 KB of operands for the work the
// single-CTA kernel feeds with 64 KB, so four stages fit where three did.
//
// Roles (576 threads per CTA):
//   warps 0-3, 6-17 epilogue of this CTA's 128 rows (both CTAs);
//   warp 4          TMA producer of this CTA's halves; in CTA 0 it also takes
//                   the work items and publishes them to both CTAs' queues;
//   warp 5          tensor memory (allocated for the pair); in CTA 0 one
//                   thread issues the MMAs.
// Both CTAs' copies of a stage complete on CTA 0's full barrier; each commit
// of the MMA thread arrives on the same barrier in both CTAs; the
// epilogues of both CTAs, and the consumers of both queues, report to CTA 0.
// Remote barriers and queue slots are reached through shared::cluster
// addresses (mapa).  Every wait is bounded; at the end each CTA waits
// (bounded) for the other's farewell before its shared memory may go away.
#pragma once
#include "grouped.cuh"

namespace moe {

constexpr int kGPTileB = (kGBN / 2) * kGBK * 2;  // 16 KB: half of a token tile
constexpr int kGPRows = 2 * kGBM;                 // weight rows of one pair item
// gate/up: A_gate + A_up + half B per stage (48 KB), four stages
constexpr int kGP1Stages = 4;
constexpr int kGP1Stage = 2 * kGTileA + kGPTileB;
constexpr int kGPMaxStages = kGP1Stages;
// gate/up epilogue: four warps per quarter of the tensor-memory lanes, each
// for 64 of the token columns (one accumulator set: the MMAs wait while
// tensor memory drains, so the drain gets the warps)
constexpr int kGP1EpiWarps = 16;
constexpr int kGP1Threads = (kGP1EpiWarps + 2) * 32;  // 576

// silu(g) * u as g * u * (1 + tanh(g / 2)) / 2 with the hardware tanh (one
// special-function operation; relative error about 2^-11, well inside the
// bf16 rounding of h that follows)
MOE_DEVINL float silu_mul_tanh(float g, float u)
{
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * g));
    return g * u * fmaf(0.5f, t, 0.5f);
}

// ---------------------------------------------------------------------------
// cluster wrappers
MOE_DEVINL uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// shared::cluster address of the variable at local address `p` in CTA `rank`
MOE_DEVINL uint32_t cluster_addr(const void *p, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr(p)), "r"(rank));
    return r;
}

MOE_DEVINL void mbar_arrive_cluster(uint32_t caddr)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(caddr)
                 : "memory");
}

MOE_DEVINL void st_cluster_u32(uint32_t caddr, int v)
{
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(caddr), "r"(v) : "memory");
}

MOE_DEVINL bool mbar_try_wait_cluster(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// mbar_wait whose acquire covers arrivals released by the other CTA
MOE_DEVINL bool mbar_wait_cluster(uint64_t *bar, uint32_t parity, int *status)
{
    if (mbar_try_wait_cluster(bar, parity))
        return true;
    const uint64_t t0 = global_ns();
    const uint64_t lim = wait_limit_ns();
    while (!mbar_try_wait_cluster(bar, parity)) {
        if (global_ns() - t0 > lim) {
            set_status(status, MOE_ERR_TIMEOUT);
            return false;
        }
    }
    return true;
}

MOE_DEVINL void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

MOE_DEVINL void tmem_alloc_pair(uint32_t *dst, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(dst)),
                 "r"(ncols)
                 : "memory");
}
MOE_DEVINL void tmem_relinquish_pair()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
MOE_DEVINL void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// M = 256 across the pair: A rows [0,128) and B columns [0, N/2) from CTA 0's
// shared memory at these descriptors' addresses, the rest from CTA 1's at the
// same addresses; D rows split the same way over the two tensor memories.
MOE_DEVINL void umma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                               uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on the barrier at this shared-memory offset in both CTAs of the
// pair when every pair MMA this thread issued so far has completed (the
// commit's own CTA mask; no data moves).
MOE_DEVINL void umma_commit_pair_both(const uint64_t *bar)
{
    const uint16_t mask = 3;
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(smem_addr(bar)),
        "h"(mask)
        : "memory");
}

// 2-D tiled TMA load (no multicast) into this CTA's shared memory whose bytes
// complete on a barrier of either CTA of the pair (shared::cluster address).
MOE_DEVINL void tma_load_2d_pair(void *dst, const CUtensorMap *map, int x, int y, uint32_t bar_caddr)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_caddr), "r"(x), "r"(y)
        : "memory");
}

// ---------------------------------------------------------------------------
struct GPSync {
    uint64_t full[kGPMaxStages];   // CTA 0: both CTAs' tiles of stage s landed
    uint64_t empty[kGPMaxStages];  // each CTA: the MMAs reading stage s finished
    uint64_t acc_full[2];          // each CTA: accumulator set b of the item is complete
    uint64_t acc_empty[2];         // CTA 0: both epilogues have read accumulator set b
    uint64_t q_full[kGQ];          // each CTA: CTA 0 published q_item[slot]
    uint64_t q_empty[kGQ];         // CTA 0: every consumer of both CTAs is done with it
    uint64_t drained;              // each CTA: every MMA has completed
    uint64_t bye;                  // each CTA: the other CTA has finished
    int q_item[kGQ];
    uint32_t tmem_base;
    int abort;
};

MOE_DEVINL bool gp_aborted(const GPSync &sy) { return *(volatile const int *)&sy.abort != 0; }

inline size_t gemm1_pair_smem_bytes()
{
    return 1024 + (size_t)kGP1Stages * kGP1Stage + sizeof(GPSync) + sizeof(GTable);
}

// Set-up of a pair kernel: barriers (thread 0), tensor memory for the pair
// (warp kGWarpMma of both CTAs, all 512 columns), then a cluster barrier so
// that no remote arrival reaches a barrier before it exists.  nepi: the
// epilogue warps of one CTA.
MOE_DEVINL void gp_setup(GPSync &sy, int stages, int nepi, int tid, int warp)
{
    if (tid == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&sy.full[s], 1);
            mbar_init(&sy.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sy.acc_full[b], 1);
            mbar_init(&sy.acc_empty[b], 2 * nepi);
        }
        // queue consumers: per CTA the epilogue warps, plus the MMA thread
        // (CTA 0) or the TMA producer (CTA 1)
        for (int q = 0; q < kGQ; ++q) {
            mbar_init(&sy.q_full[q], 1);
            mbar_init(&sy.q_empty[q], 2 * (nepi + 1));
        }
        mbar_init(&sy.drained, 1);
        mbar_init(&sy.bye, 1);
        sy.abort = 0;
        fence_mbar_init();
    }
    if (warp == kGWarpMma) {
        tmem_alloc_pair(&sy.tmem_base, 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    tc_fence_after();
}

// The TMA warp's next item (lane 0): CTA 0 takes `next` (or -1 to end) and
// publishes it to both CTAs' queues once every consumer of both CTAs is done
// with the slot; CTA 1 takes it from its queue and hands the slot back to
// CTA 0.  Returns the item, -1 at the end, -2 if a wait gave up.
MOE_DEVINL int gp_producer_item(GPSync &sy, GQueue &q, bool lead, uint32_t peer, int next,
                                int *status)
{
    int cur;
    if (lead) {
        cur = next;
        if (!mbar_wait_cluster(&sy.q_empty[q.slot], q.ph ^ 1u, status))
            return -2;
        sy.q_item[q.slot] = cur;
        st_cluster_u32(cluster_addr(&sy.q_item[q.slot], peer), cur);
        mbar_arrive(&sy.q_full[q.slot]);
        mbar_arrive_cluster(cluster_addr(&sy.q_full[q.slot], peer));
    } else {
        if (!mbar_wait_cluster(&sy.q_full[q.slot], q.ph, status))
            return -2;
        cur = *(volatile int *)&sy.q_item[q.slot];
        mbar_arrive_cluster(cluster_addr(&sy.q_empty[q.slot], 0));
    }
    q.advance();
    return cur;
}

// An epilogue warp's next item: lane 0 waits, the warp gets one answer (-1:
// none left, or the wait gave up and the CTA aborts).
MOE_DEVINL int gp_take_warp(GPSync &sy, GQueue &q, int *status, int lane)
{
    int cur = -1;
    if (lane == 0) {
        if (mbar_wait_cluster(&sy.q_full[q.slot], q.ph, status))
            cur = *(volatile int *)&sy.q_item[q.slot];
        else
            sy.abort = 1;
    }
    return __shfl_sync(0xffffffffu, cur, 0);
}

// An epilogue warp is done with its item: accumulator set `buf` read (CTA 0's
// barrier) and the queue slot handed back (CTA 0's barrier).
MOE_DEVINL void gp_release_warp(GPSync &sy, GQueue &q, int buf, int lane)
{
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
        mbar_arrive_cluster(cluster_addr(&sy.acc_empty[buf], 0));
        mbar_arrive_cluster(cluster_addr(&sy.q_empty[q.slot], 0));
    }
    q.advance();
}

// End of a pair kernel: free tensor memory once every MMA has completed (CTA
// 0's MMA thread waited already), the farewell handshake -- neither CTA's
// shared memory goes away while the other may still reach it -- and the
// last CTA resets the item counters.
MOE_DEVINL void gp_teardown(GPSync &sy, uint32_t tmem, GSched sc, bool lead, uint32_t peer,
                            int tid, int warp, int lane, int *status)
{
    tc_fence_before();
    __syncthreads();
    if (warp == kGWarpMma) {
        if (lane == 0 && !lead)
            mbar_wait(&sy.drained, 0, status);
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_pair(tmem, 512);
    }
    if (tid == 0) {
        mbar_arrive_cluster(cluster_addr(&sy.bye, peer));
        mbar_wait_cluster(&sy.bye, 0, status);
        __threadfence();
        if (atomicAdd(sc.done, 1u) == gridDim.x - 1) {
            *sc.next = 0u;
            *sc.done = 0u;
        }
    }
}

// ---------------------------------------------------------------------------
// Gate/up GEMM on CTA pairs with the SwiGLU epilogue (I % 256 == 0).  Tensor
// memory of each CTA: its rows' gate accumulator in columns [0, 256), up in
// [256, 512).
__global__ void __launch_bounds__(kGP1Threads, 1)
    k_gemm1_pair(const __grid_constant__ CUtensorMap tm_gate,
                 const __grid_constant__ CUtensorMap tm_up,
                 const __grid_constant__ CUtensorMap tm_xs, Gemm1Args a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *ring = g_align1024(smem_raw);
    GPSync &sy = *reinterpret_cast<GPSync *>(ring + (size_t)kGP1Stages * kGP1Stage);
    GTable &tb = *reinterpret_cast<GTable *>(&sy + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_rank(), peer = rank ^ 1u;
    const bool lead = rank == 0;
    int *status = &a.hdr->status;

    gp_setup(sy, kGP1Stages, kGP1EpiWarps, tid, warp);
    const uint32_t tmem = sy.tmem_base;

    pdl_wait();
    pdl_trigger();
    const int d = a.d, E = a.E, I = a.I;
    const int nrt = I / kGPRows;
    const int nkb = d / kGBK;
    g_build_items(a.offsets, E, nrt, tb, a.T * a.k1, status);
    const int n_items = tb.ibase[E];
    GQueue q = {0, 0u};

    if (warp == kGWarpTma) {
        // -------------------------------------------------------- items (CTA 0), tiles
        if (lane == 0) {
            uint32_t g = 0;
            int i = lead ? (int)atomicAdd(a.sched.next, 1u) : 0;
            while (true) {
                const int cur = gp_producer_item(sy, q, lead, peer,
                                                 i < n_items && !gp_aborted(sy) ? i : -1, status);
                if (cur == -2)
                    sy.abort = 1;
                if (cur < 0)
                    break;
                if (lead)
                    i = (int)atomicAdd(a.sched.next, 1u);  // the next one, in flight meanwhile
                const GItem it = g_item(tb, E, cur);
                const int row = it.e * I + it.rt * kGPRows + (int)rank * kGBM;
                const int nh = pad16(it.n) / 2;         // this CTA's tokens (multiple of 8)
                const int t0 = it.p0 + (int)rank * nh;  // its first token row
                const int nb = (nh + 63) / 64;          // 64-row boxes of them
                const uint32_t stage_bytes = 2u * (2 * kGTileA + nb * (kGTileB / 4));
                for (int kb = 0; kb < nkb; ++kb, ++g) {
                    const int s = g % kGP1Stages;
                    if (!mbar_wait_cluster(&sy.empty[s], ((g / kGP1Stages) & 1) ^ 1, status)) {
                        sy.abort = 1;
                        break;
                    }
                    uint8_t *st = ring + (size_t)s * kGP1Stage;
                    const uint32_t fb = cluster_addr(&sy.full[s], 0);
                    if (lead)  // both CTAs' bytes of the stage
                        mbar_arrive_expect_tx(&sy.full[s], stage_bytes);
                    tma_load_2d_pair(st, &tm_gate, kb * kGBK, row, fb);
                    tma_load_2d_pair(st + kGTileA, &tm_up, kb * kGBK, row, fb);
                    for (int bx = 0; bx < nb; ++bx)
                        tma_load_2d_pair(st + 2 * kGTileA + bx * (kGTileB / 4), &tm_xs, kb * kGBK,
                                         t0 + 64 * bx, fb);
                }
                if (gp_aborted(sy))
                    break;
            }
            // drain (CTA 0): every stage issued has landed before the CTA may leave;
            // CTA 1's copies complete on CTA 0's barriers, which the MMAs waited for
            if (lead) {
                const uint32_t n_iss = g;
                for (uint32_t r = n_iss > (uint32_t)kGP1Stages ? n_iss - kGP1Stages : 0; r < n_iss;
                     ++r)
                    mbar_wait(&sy.full[r % kGP1Stages], (r / kGP1Stages) & 1, status);
            }
        }
    } else if (warp == kGWarpMma) {
        // -------------------------------------------------------- MMA issue (CTA 0)
        if (lane == 0 && lead) {
            uint32_t g = 0, itc = 0;
            while (true) {
                if (!mbar_wait(&sy.q_full[q.slot], q.ph, status)) {
                    sy.abort = 1;
                    break;
                }
                const int cur = *(volatile int *)&sy.q_item[q.slot];
                if (cur < 0)
                    break;
                const GItem it = g_item(tb, E, cur);
                if (!mbar_wait_cluster(&sy.acc_empty[0], (itc & 1) ^ 1, status)) {
                    sy.abort = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t idesc = umma_idesc_bf16(kGPRows, pad16(it.n));
                for (int kb = 0; kb < nkb; ++kb, ++g) {
                    const int s = g % kGP1Stages;
                    if (!mbar_wait(&sy.full[s], (g / kGP1Stages) & 1, status)) {
                        sy.abort = 1;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = smem_addr(ring + (size_t)s * kGP1Stage);
#pragma unroll
                    for (int kk = 0; kk < kGBK / 16; ++kk) {
                        const uint64_t ag = umma_desc_sw128(st + kk * 32);
                        const uint64_t au = umma_desc_sw128(st + kGTileA + kk * 32);
                        const uint64_t bd = umma_desc_sw128(st + 2 * kGTileA + kk * 32);
                        const uint32_t acc = (kb | kk) != 0;
                        umma_bf16_pair(tmem, ag, bd, idesc, acc);
                        umma_bf16_pair(tmem + 256, au, bd, idesc, acc);
                    }
                    umma_commit_pair_both(&sy.empty[s]);
                }
                if (gp_aborted(sy))
                    break;
                umma_commit_pair_both(&sy.acc_full[0]);
                mbar_arrive(&sy.q_empty[q.slot]);
                q.advance();
                ++itc;
            }
            // every MMA issued has completed before tensor memory is freed
            umma_commit_pair_both(&sy.drained);
            mbar_wait(&sy.drained, 0, status);
        }
    } else {
        // -------------------------------------------------------- epilogue (both CTAs)
        const int lq = warp & 3;  // tensor-memory lane quarter
        // which quarter of the token columns: warps 0-3 the first, then
        // warps 6-9, 10-13, 14-17 (each set covers the four lane quarters)
        const int eh = warp < 4 ? 0 : (warp - 6) / 4 + 1;
        uint32_t itc = 0;
        const uint32_t lane_addr = tmem + ((uint32_t)(lq * 32) << 16);
        while (true) {
            const int cur = gp_take_warp(sy, q, status, lane);
            if (cur < 0)
                break;
            const GItem it = g_item(tb, E, cur);
            int ok = 1;
            if (lane == 0)
                ok = mbar_wait_cluster(&sy.acc_full[0], itc & 1, status);
            if (!__shfl_sync(0xffffffffu, ok, 0)) {
                sy.abort = 1;
                break;
            }
            tc_fence_after();
            // lane pairs (2m, 2m+1) store channels 2m, 2m+1 together: the even lane
            // for token j, the odd lane for token j+1
            const int odd = lane & 1;
            uint16_t *hrow = a.h + (size_t)it.p0 * I + it.rt * kGPRows + (int)rank * kGBM +
                             lq * 32 + (lane & ~1);
            for (int c0 = 64 * eh; c0 < it.n && c0 < 64 * eh + 64; c0 += 32) {
                float gv[32], uv[32];
                tmem_ld32x2(lane_addr + c0, lane_addr + 256 + c0, gv, uv);
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    const float h0 = silu_mul_tanh(gv[j], uv[j]);
                    const float h1 = silu_mul_tanh(gv[j + 1], uv[j + 1]);
                    const float other = __shfl_xor_sync(0xffffffffu, odd ? h0 : h1, 1);
                    const uint32_t pair = odd ? pack_bf16x2(other, h1) : pack_bf16x2(h0, other);
                    const int tj = c0 + j + odd;
                    if (tj < it.n)
                        *reinterpret_cast<uint32_t *>(hrow + (size_t)tj * I) = pair;
                }
            }
            gp_release_warp(sy, q, 0, lane);
            ++itc;
        }
    }
    gp_teardown(sy, tmem, a.sched, lead, peer, tid, warp, lane, status);
}

}  // namespace moe
