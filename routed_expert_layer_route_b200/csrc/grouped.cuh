// grouped.cuh -- the large-batch expert FFN as two grouped GEMMs on the
// fifth-generation tensor cores (tcgen05.mma, accumulators in tensor memory).
//
// Expert structure ("Channel Selection for Mixture-of-Experts Decoding Needs
// No Calibration Data", section 2 "Background"): a gated MLP; with the
// routed slots grouped by expert (the counting sort of route.cuh), expert
// e's n_e token rows X_e form two dense contractions:
//     GEMM 1:  G = W_gate[e] X_e^T,  U = W_up[e] X_e^T   ([I x n_e], K = d)
//              H = silu(G) * U, stored bf16 as rows of the slot-ordered H
//     GEMM 2:  O = W_down[e] H_e^T                         ([d x n_e], K = I)
//              y[t] += w[t, s] * O[:, slot]   (Eq. 2 weight, "Paper of the
//              Week #3", section "The Receipt"), or O stored per slot.
// The weight matrix is the MMA's M side (128 rows per tile) and the tokens
// its N side (up to 256 per tile, padded to 16), so an expert with few tokens
// costs little padding.  Both operands are K-major bf16 tiles of 64 K values
// (one 128-byte row) in the 128-byte swizzled shared-memory layout.
//
// One persistent CTA per SM takes work items (expert, weight-row tile, token
// tile; token tile fastest) from a device-wide counter, so items are handed
// out in order to whichever SM is free: neighbours in the order, which share
// weight tiles and token rows, run at the same time and read them once from
// DRAM, and the load balances itself.  Warp roles:
//   warps 0-3, 6-9  epilogue: tensor memory -> registers (tcgen05.ld),
//               SwiGLU or the weighted combine, global stores / float32
//               red.add; warp w reads lane quarter w % 4, the two warps of a
//               quarter split the token columns;
//   warp 4      takes the items and publishes them to the other roles
//               through a shared-memory queue; TMA producer, no multicast:
//               weight tiles and token tiles (GEMM 1: the routed tokens' x
//               rows, copied into expert order by k_gather_rows; GEMM 2: H);
//   warp 5      allocates tensor memory and issues the MMAs (one thread).
// The same down-GEMM kernel computes the router logits of large batches
// (one group of T rows, W_r as the weight matrix, bias added).
// Every wait is bounded: a wait that gives up records MOE_ERR_TIMEOUT and the
// CTA drains what it issued and leaves.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "route.cuh"
#include "stream.cuh"

namespace moe {

constexpr int kGBM = 128;                 // weight rows per tile (MMA M)
constexpr int kGBK = 64;                  // K values per stage (one 128-byte row)
constexpr int kGBN = 256;                 // most tokens per tile (MMA N)
constexpr int kGTileA = kGBM * kGBK * 2;  // 16 KB
constexpr int kGTileB = kGBN * kGBK * 2;  // 32 KB
constexpr int kG1Stages = 3;              // A_gate + A_up + B = 64 KB per stage
constexpr int kG2Stages = 4;              // A_down + B = 48 KB per stage
constexpr int kG1Stage = 2 * kGTileA + kGTileB;
constexpr int kG2Stage = kGTileA + kGTileB;
constexpr int kGEpiWarps = 8;  // two per quarter of the tensor-memory lanes
constexpr int kGEpiThreads = kGEpiWarps * 32;
constexpr int kG1Threads = kGEpiThreads + 64;  // 320
constexpr int kG2Threads = kGEpiThreads + 64;  // 320
constexpr int kGMaxE = 1024;
constexpr int kGWarpTma = 4, kGWarpMma = 5;

// ---------------------------------------------------------------------------
// tcgen05 / TMA wrappers
MOE_DEVINL void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
MOE_DEVINL void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

MOE_DEVINL void tmem_alloc(uint32_t *dst, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(dst)),
                 "r"(ncols)
                 : "memory");
}
MOE_DEVINL void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
MOE_DEVINL void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// Shared-memory matrix descriptor: K-major operand in the 128-byte swizzled
// layout (rows of 128 bytes, 8-row groups 1024 bytes apart), tile base
// 1024-byte aligned; the K step inside a row advances the start address.
MOE_DEVINL uint64_t umma_desc_sw128(uint32_t saddr)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu)     // start address
           | ((uint64_t)1 << 16)                  // leading byte offset (unused here), 16 B
           | ((uint64_t)(1024 >> 4) << 32)        // stride byte offset: 8 rows x 128 B
           | ((uint64_t)1 << 46)                  // descriptor version of this architecture
           | ((uint64_t)2 << 61);                 // 128-byte swizzle
}

// Instruction descriptor of kind::f16: bf16 A and B, float32 accumulator,
// both K-major, M x N.
MOE_DEVINL uint32_t umma_idesc_bf16(int M, int N)
{
    return (1u << 4)                        // D float32
           | (1u << 7)                      // A bf16
           | (1u << 10)                     // B bf16
           | ((uint32_t)(N >> 3) << 17)     // N / 8
           | ((uint32_t)(M >> 4) << 24);    // M / 16
}

MOE_DEVINL void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                          uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on `bar` when every MMA this thread issued so far has completed.
MOE_DEVINL void umma_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_addr(bar))
                 : "memory");
}

// 32 lanes x 32 consecutive float32 columns: thread i of the warp gets lane
// (taddr.lane + i), columns taddr.col .. +31.
MOE_DEVINL void tmem_ld32(uint32_t taddr, float (&v)[32])
{
    uint32_t r[32];
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
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i)
        v[i] = __uint_as_float(r[i]);
}

// Two 32-column loads (columns ta.. and tb..) with one wait: the wait is part
// of the same asm statement, so no use of the outputs can move above it.
MOE_DEVINL void tmem_ld32x2(uint32_t ta, uint32_t tb, float (&a)[32], float (&b)[32])
{
    uint32_t r[64];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%64];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
        "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%65];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]),
          "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]),
          "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]),
          "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]),
          "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]),
          "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(ta), "r"(tb)
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        a[i] = __uint_as_float(r[i]);
        b[i] = __uint_as_float(r[32 + i]);
    }
}

// silu(g) * u for the tensor-core path, whose h is rounded to bf16 next:
// fast exp and divide (a few ulp of float32, far below the bf16 step).
MOE_DEVINL float silu_mul_fast(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

// Two floats to a bf16x2 word (round to nearest even), lo in the low half.
MOE_DEVINL uint32_t pack_bf16x2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// 32 lanes x 16 consecutive float32 columns.
MOE_DEVINL void tmem_ld16(uint32_t taddr, float (&v)[16])
{
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i)
        v[i] = __uint_as_float(r[i]);
}

// 2-D tiled TMA load (no multicast) of box {64 K values, rows} at (x, y).
MOE_DEVINL void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(x), "r"(y)
        : "memory");
}

// ---------------------------------------------------------------------------
// Work items: expert e contributes nrt x ceil(n_e / kGBN) items (weight-row
// tile rt, token tile tt; tt fastest).
struct GItem {
    int e, rt, n, p0;
};

struct GTable {
    int ibase[kGMaxE + 1];  // first item of each expert; ibase[E] = item count
    int offs[kGMaxE + 1];   // expert offsets into the slot order
    int bn;                 // tokens per tile (<= kGBN, multiple of 64)
    int bad;                // checked build: the offsets failed their check
    int scan[40];
};

// All threads of the CTA: fill the table from the expert offsets (or, with
// offsets == nullptr, one group of single_n rows).  nmax: the rows the
// offsets may address; the checked build verifies 0 <= offs[0] <= ... <=
// offs[E] <= nmax and, if not, records MOE_ERR_DEVICE_CHECK and leaves no
// items.
__device__ void g_build_items(const int32_t *offsets, int E, int nrt, GTable &tb, int nmax,
                              int *status, int single_n = 0, int bn = kGBN)
{
    for (int e = threadIdx.x; e <= E; e += blockDim.x)
        tb.offs[e] = offsets ? __ldcg(&offsets[e]) : (e == 0 ? 0 : single_n);
    if (threadIdx.x == 0) {
        tb.bn = bn;
        tb.bad = 0;
    }
    __syncthreads();
    if (MOE_CHECKS) {
        for (int e = threadIdx.x; e <= E; e += blockDim.x) {
            const int o = tb.offs[e];
            if (o < 0 || o > nmax || (e < E && o > tb.offs[e + 1]))
                tb.bad = 1;
        }
        __syncthreads();
        if (tb.bad) {
            if (threadIdx.x == 0)
                set_status(status, MOE_ERR_DEVICE_CHECK);
            for (int e = threadIdx.x; e <= E; e += blockDim.x)
                tb.offs[e] = 0;
        }
        __syncthreads();
    }
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const int n = tb.offs[e + 1] - tb.offs[e];
        tb.ibase[e] = n > 0 ? nrt * ((n + bn - 1) / bn) : 0;
    }
    __syncthreads();
    const int total = block_exclusive_scan(tb.ibase, E, tb.scan);
    if (threadIdx.x == 0)
        tb.ibase[E] = total;
    __syncthreads();
}

MOE_DEVINL GItem g_item(const GTable &tb, int E, int i)
{
    int lo = 0, hi = E;  // ibase[lo] <= i < ibase[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (tb.ibase[mid] <= i)
            lo = mid;
        else
            hi = mid;
    }
    GItem it;
    it.e = lo;
    const int ne = tb.offs[lo + 1] - tb.offs[lo];
    const int bn = tb.bn;
    const int nt = (ne + bn - 1) / bn;
    const int local = i - tb.ibase[lo];
    it.rt = local / nt;
    const int tt = local - it.rt * nt;
    it.n = min(bn, ne - tt * bn);
    it.p0 = tb.offs[lo] + tt * bn;
    return it;
}

MOE_DEVINL int pad16(int n) { return (n + 15) & ~15; }

// ---------------------------------------------------------------------------
constexpr int kGQ = 4;  // depth of the work-item queue between the roles

struct GSync {
    uint64_t full[kG2Stages];
    uint64_t empty[kG2Stages];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t q_full[kGQ];   // the producer published item q_item[slot]
    uint64_t q_empty[kGQ];  // the MMA thread and every epilogue warp are done with it
    uint64_t drained;
    int q_item[kGQ];        // item index, -1: no more items
    uint32_t tmem_base;
    int abort;
};

// Position in the item queue: slot and phase parity.
struct GQueue {
    int slot;
    uint32_t ph;
    __device__ void advance()
    {
        if (++slot == kGQ) {
            slot = 0;
            ph ^= 1u;
        }
    }
};

// Device-wide item counters of one grouped launch: `next` hands out items,
// `done` counts the CTAs that have left; the last CTA resets both, so each
// launch finds them at zero (the workspace header starts zeroed).
struct GSched {
    unsigned *next;
    unsigned *done;
};

MOE_DEVINL uint8_t *g_align1024(uint8_t *p)
{
    const uint32_t a = smem_addr(p);
    return p + (((a + 1023u) & ~1023u) - a);
}

MOE_DEVINL bool g_aborted(const GSync &sy) { return *(volatile const int *)&sy.abort != 0; }

// Barrier set-up shared by the kernels (thread 0) and the tensor-memory
// allocation (warp kGWarpMma, all 512 columns).
MOE_DEVINL void g_setup(GSync &sy, int stages, int nacc, int tid, int warp)
{
    if (tid == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&sy.full[s], 1);
            mbar_init(&sy.empty[s], 1);
        }
        for (int b = 0; b < nacc; ++b) {
            mbar_init(&sy.acc_full[b], 1);
            mbar_init(&sy.acc_empty[b], kGEpiWarps);
        }
        for (int q = 0; q < kGQ; ++q) {
            mbar_init(&sy.q_full[q], 1);
            mbar_init(&sy.q_empty[q], 1 + kGEpiWarps);
        }
        mbar_init(&sy.drained, 1);
        sy.abort = 0;
        fence_mbar_init();
    }
    if (warp == kGWarpMma) {
        tmem_alloc(&sy.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
}

// Producer side of the queue: publish item `cur` (-1 ends the stream).
MOE_DEVINL bool g_publish(GSync &sy, GQueue &q, int cur, int *status)
{
    if (!mbar_wait(&sy.q_empty[q.slot], q.ph ^ 1u, status))
        return false;
    sy.q_item[q.slot] = cur;
    mbar_arrive(&sy.q_full[q.slot]);
    q.advance();
    return true;
}

// Consumer side, one thread (the MMA issuer): the next item index (-1: none
// left, or a wait gave up).
MOE_DEVINL int g_take(GSync &sy, GQueue &q, int *status)
{
    if (!mbar_wait(&sy.q_full[q.slot], q.ph, status)) {
        sy.abort = 1;
        return -1;
    }
    return *(volatile int *)&sy.q_item[q.slot];
}

MOE_DEVINL void g_release(GSync &sy, GQueue &q)
{
    mbar_arrive(&sy.q_empty[q.slot]);
    q.advance();
}

// Consumer side, a whole warp (epilogue): lane 0 waits, every lane gets the
// same answer, so the warp never splits before its warp-wide tcgen05.ld.
MOE_DEVINL int g_take_warp(GSync &sy, GQueue &q, int *status, int lane)
{
    int cur = -1;
    if (lane == 0)
        cur = g_take(sy, q, status);
    return __shfl_sync(0xffffffffu, cur, 0);
}

MOE_DEVINL void g_release_warp(GSync &sy, GQueue &q, int lane)
{
    __syncwarp();
    if (lane == 0)
        mbar_arrive(&sy.q_empty[q.slot]);
    q.advance();
}

// Bounded wait by lane 0 for the whole warp.
MOE_DEVINL bool g_wait_warp(uint64_t *bar, uint32_t parity, int *status, int lane)
{
    int ok = 1;
    if (lane == 0)
        ok = mbar_wait(bar, parity, status);
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// End of a grouped kernel: free tensor memory; the last CTA resets the counters.
MOE_DEVINL void g_teardown(GSync &sy, uint32_t tmem, GSched sc, int tid, int warp)
{
    tc_fence_before();
    __syncthreads();
    if (warp == kGWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    if (tid == 0) {
        __threadfence();
        if (atomicAdd(sc.done, 1u) == gridDim.x - 1) {
            *sc.next = 0u;
            *sc.done = 0u;
        }
    }
}

struct Gemm1Args {
    const int32_t *offsets;      // [E + 1]
    const int32_t *sorted_slot;  // [T*k1] slot ids (t*k1 + s) in expert order
    uint16_t *h;                 // [T*k1 x I] bf16, row p = sorted position p
    int T, d, E, I, k1;
    GSched sched;
    WsHeader *hdr;
};

inline size_t gemm1_smem_bytes() { return 1024 + (size_t)kG1Stages * kG1Stage + sizeof(GSync) + sizeof(GTable); }
inline size_t gemm2_smem_bytes() { return 1024 + (size_t)kG2Stages * kG2Stage + sizeof(GSync) + sizeof(GTable); }

// Gate/up GEMM with the SwiGLU epilogue.  Tensor memory: gate accumulator in
// columns [0, 256), up accumulator in [256, 512).
__global__ void __launch_bounds__(kG1Threads, 1)
    k_gemm1(const __grid_constant__ CUtensorMap tm_gate, const __grid_constant__ CUtensorMap tm_up,
            const __grid_constant__ CUtensorMap tm_xs, Gemm1Args a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *ring = g_align1024(smem_raw);
    GSync &sy = *reinterpret_cast<GSync *>(ring + (size_t)kG1Stages * kG1Stage);
    GTable &tb = *reinterpret_cast<GTable *>(&sy + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int *status = &a.hdr->status;

    g_setup(sy, kG1Stages, 1, tid, warp);
    const uint32_t tmem = sy.tmem_base;

    pdl_wait();
    pdl_trigger();
    const int d = a.d, E = a.E, I = a.I;
    const int nrt = I / kGBM;
    const int nkb = d / kGBK;
    g_build_items(a.offsets, E, nrt, tb, a.T * a.k1, status);
    const int n_items = tb.ibase[E];
    GQueue q = {0, 0u};

    if (warp == kGWarpTma) {
        // -------------------------------------------------------- items, weight and token tiles
        if (lane == 0) {
            uint32_t g = 0;
            int i = (int)atomicAdd(a.sched.next, 1u);
            while (true) {
                const int cur = i < n_items && !g_aborted(sy) ? i : -1;
                if (!g_publish(sy, q, cur, status)) {
                    sy.abort = 1;
                    break;
                }
                if (cur < 0)
                    break;
                i = (int)atomicAdd(a.sched.next, 1u);  // the next one, in flight meanwhile
                const GItem it = g_item(tb, E, cur);
                const int row = it.e * I + it.rt * kGBM;
                const int nb = (it.n + 63) / 64;  // 64-row boxes of the sorted x rows
                for (int kb = 0; kb < nkb; ++kb, ++g) {
                    const int s = g % kG1Stages;
                    if (!mbar_wait(&sy.empty[s], ((g / kG1Stages) & 1) ^ 1, status)) {
                        sy.abort = 1;
                        break;
                    }
                    uint8_t *st = ring + (size_t)s * kG1Stage;
                    mbar_arrive_expect_tx(&sy.full[s], 2 * kGTileA + nb * (kGTileB / 4));
                    tma_load_2d(st, &tm_gate, kb * kGBK, row, &sy.full[s]);
                    tma_load_2d(st + kGTileA, &tm_up, kb * kGBK, row, &sy.full[s]);
                    for (int b = 0; b < nb; ++b)
                        tma_load_2d(st + 2 * kGTileA + b * (kGTileB / 4), &tm_xs, kb * kGBK,
                                    it.p0 + 64 * b, &sy.full[s]);
                }
            }
            // drain: every stage issued has landed before the CTA may leave
            const uint32_t n_iss = g;
            for (uint32_t r = n_iss > (uint32_t)kG1Stages ? n_iss - kG1Stages : 0; r < n_iss; ++r)
                mbar_wait(&sy.full[r % kG1Stages], (r / kG1Stages) & 1, status);
        }
    } else if (warp == kGWarpMma) {
        // -------------------------------------------------------- MMA issue
        if (lane == 0) {
            uint32_t g = 0, itc = 0;
            while (true) {
                const int cur = g_take(sy, q, status);
                if (cur < 0)
                    break;
                const GItem it = g_item(tb, E, cur);
                if (!mbar_wait(&sy.acc_empty[0], (itc & 1) ^ 1, status)) {
                    sy.abort = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t idesc = umma_idesc_bf16(kGBM, pad16(it.n));
                for (int kb = 0; kb < nkb; ++kb, ++g) {
                    const int s = g % kG1Stages;
                    if (!mbar_wait(&sy.full[s], (g / kG1Stages) & 1, status)) {
                        sy.abort = 1;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = smem_addr(ring + (size_t)s * kG1Stage);
#pragma unroll
                    for (int kk = 0; kk < kGBK / 16; ++kk) {
                        const uint64_t ag = umma_desc_sw128(st + kk * 32);
                        const uint64_t au = umma_desc_sw128(st + kGTileA + kk * 32);
                        const uint64_t bd = umma_desc_sw128(st + 2 * kGTileA + kk * 32);
                        const uint32_t acc = (kb | kk) != 0;
                        umma_bf16(tmem, ag, bd, idesc, acc);
                        umma_bf16(tmem + 256, au, bd, idesc, acc);
                    }
                    umma_commit(&sy.empty[s]);
                }
                if (g_aborted(sy))
                    break;
                umma_commit(&sy.acc_full[0]);
                g_release(sy, q);
                ++itc;
            }
            // every MMA issued has completed before tensor memory is freed
            umma_commit(&sy.drained);
            mbar_wait(&sy.drained, 0, status);
        }
    } else {
        // -------------------------------------------------------- epilogue (warps 0-3, 6-9)
        const int lq = warp & 3;                    // tensor-memory lane quarter
        const int eh = warp >= 6;                   // which half of the token columns
        uint32_t itc = 0;
        const uint32_t lane_addr = tmem + ((uint32_t)(lq * 32) << 16);
        while (true) {
            const int cur = g_take_warp(sy, q, status, lane);
            if (cur < 0)
                break;
            const GItem it = g_item(tb, E, cur);
            if (!g_wait_warp(&sy.acc_full[0], itc & 1, status, lane)) {
                sy.abort = 1;
                break;
            }
            tc_fence_after();
            // lane pairs (2m, 2m+1) store channels 2m, 2m+1 together: the even lane
            // for token j, the odd lane for token j+1
            const int odd = lane & 1;
            uint16_t *hrow = a.h + (size_t)it.p0 * I + it.rt * kGBM + lq * 32 + (lane & ~1);
            for (int c0 = 32 * eh; c0 < it.n; c0 += 64) {
                float gv[32], uv[32];
                tmem_ld32x2(lane_addr + c0, lane_addr + 256 + c0, gv, uv);
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    const float h0 = silu_mul_fast(gv[j], uv[j]);
                    const float h1 = silu_mul_fast(gv[j + 1], uv[j + 1]);
                    const float other = __shfl_xor_sync(0xffffffffu, odd ? h0 : h1, 1);
                    const uint32_t pair = odd ? pack_bf16x2(other, h1) : pack_bf16x2(h0, other);
                    const int tj = c0 + j + odd;
                    if (tj < it.n)
                        *reinterpret_cast<uint32_t *>(hrow + (size_t)tj * I) = pair;
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sy.acc_empty[0]);
            g_release_warp(sy, q, lane);
            ++itc;
        }
    }
    g_teardown(sy, tmem, a.sched, tid, warp);
}

// ---------------------------------------------------------------------------
struct Gemm2Args {
    const int32_t *offsets;      // [E + 1]; nullptr: one group of single_n rows
    const int32_t *sorted_slot;  // [T*k1]
    const float *topk_w;         // [T*k1] Eq. 2 weights by slot (combine mode)
    float *y_acc;                // [T x d] float32, zero on entry (combine mode)
    float *out;                  // [rows x d] float32 per sorted position (store mode)
    float *out_copy;             // nullable second destination of the store mode
    const float *bias;           // nullable [d], added in the store mode
    int single_n;
    int bn;                      // tokens per tile: kGBN, or 64 to spread a small job
    int T, d, E, I, k1;          // d: output rows of the weight matrix, I: K
    int combine;                 // 1: weighted red.add into y_acc; 0: store rows of out
    GSched sched;
    WsHeader *hdr;
};

// Down GEMM with the combine epilogue.  Two accumulator buffers of 256
// columns each, so the epilogue of one item overlaps the MMAs of the next.
__global__ void __launch_bounds__(kG2Threads, 1)
    k_gemm2(const __grid_constant__ CUtensorMap tm_down, const __grid_constant__ CUtensorMap tm_h,
            Gemm2Args a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *ring = g_align1024(smem_raw);
    GSync &sy = *reinterpret_cast<GSync *>(ring + (size_t)kG2Stages * kG2Stage);
    GTable &tb = *reinterpret_cast<GTable *>(&sy + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int *status = &a.hdr->status;

    g_setup(sy, kG2Stages, 2, tid, warp);
    const uint32_t tmem = sy.tmem_base;

    pdl_wait();
    pdl_trigger();
    const int d = a.d, E = a.E, I = a.I;
    const int nrt = d / kGBM;
    const int nkb = I / kGBK;
    g_build_items(a.offsets, E, nrt, tb, a.offsets ? a.T * a.k1 : a.single_n, status, a.single_n,
                  a.bn > 0 ? a.bn : kGBN);
    const int n_items = tb.ibase[E];
    GQueue q = {0, 0u};

    if (warp == kGWarpTma) {
        if (lane == 0) {
            uint32_t g = 0;
            int i = (int)atomicAdd(a.sched.next, 1u);
            while (true) {
                const int cur = i < n_items && !g_aborted(sy) ? i : -1;
                if (!g_publish(sy, q, cur, status)) {
                    sy.abort = 1;
                    break;
                }
                if (cur < 0)
                    break;
                i = (int)atomicAdd(a.sched.next, 1u);
                const GItem it = g_item(tb, E, cur);
                const int row = it.e * d + it.rt * kGBM;
                const int nb = (it.n + 63) / 64;  // 64-row boxes of H
                for (int kb = 0; kb < nkb; ++kb, ++g) {
                    const int s = g % kG2Stages;
                    if (!mbar_wait(&sy.empty[s], ((g / kG2Stages) & 1) ^ 1, status)) {
                        sy.abort = 1;
                        break;
                    }
                    uint8_t *st = ring + (size_t)s * kG2Stage;
                    mbar_arrive_expect_tx(&sy.full[s], kGTileA + nb * (kGTileB / 4));
                    tma_load_2d(st, &tm_down, kb * kGBK, row, &sy.full[s]);
                    for (int b = 0; b < nb; ++b)
                        tma_load_2d(st + kGTileA + b * (kGTileB / 4), &tm_h, kb * kGBK,
                                    it.p0 + 64 * b, &sy.full[s]);
                }
            }
            const uint32_t n_iss = g;
            for (uint32_t r = n_iss > (uint32_t)kG2Stages ? n_iss - kG2Stages : 0; r < n_iss; ++r)
                mbar_wait(&sy.full[r % kG2Stages], (r / kG2Stages) & 1, status);
        }
    } else if (warp == kGWarpMma) {
        if (lane == 0) {
            uint32_t g = 0, itc = 0;
            while (true) {
                const int cur = g_take(sy, q, status);
                if (cur < 0)
                    break;
                const GItem it = g_item(tb, E, cur);
                const int buf = itc & 1;
                if (!mbar_wait(&sy.acc_empty[buf], ((itc >> 1) & 1) ^ 1, status)) {
                    sy.abort = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t idesc = umma_idesc_bf16(kGBM, pad16(it.n));
                const uint32_t dt = tmem + buf * 256;
                for (int kb = 0; kb < nkb; ++kb, ++g) {
                    const int s = g % kG2Stages;
                    if (!mbar_wait(&sy.full[s], (g / kG2Stages) & 1, status)) {
                        sy.abort = 1;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = smem_addr(ring + (size_t)s * kG2Stage);
#pragma unroll
                    for (int kk = 0; kk < kGBK / 16; ++kk)
                        umma_bf16(dt, umma_desc_sw128(st + kk * 32),
                                  umma_desc_sw128(st + kGTileA + kk * 32), idesc, (kb | kk) != 0);
                    umma_commit(&sy.empty[s]);
                }
                if (g_aborted(sy))
                    break;
                umma_commit(&sy.acc_full[buf]);
                g_release(sy, q);
                ++itc;
            }
            umma_commit(&sy.drained);
            mbar_wait(&sy.drained, 0, status);
        }
    } else {
        // -------------------------------------------------------- epilogue (warps 0-3, 6-9)
        const int lq = warp & 3;   // tensor-memory lane quarter
        const int eh = warp >= 6;  // which half of the token column chunks
        uint32_t itc = 0;
        const int k1 = a.k1;
        while (true) {
            const int cur = g_take_warp(sy, q, status, lane);
            if (cur < 0)
                break;
            const GItem it = g_item(tb, E, cur);
            const int buf = itc & 1;
            // this lane's columns c*32 + lane: token and Eq. 2 weight (before the wait)
            int tk[kGBN / 32];
            float wt[kGBN / 32];
#pragma unroll
            for (int c = 0; c < kGBN / 32; ++c) {
                const int col = c * 32 + lane;
                tk[c] = 0;
                wt[c] = 0.0f;
                if (a.combine && (c & 1) == eh && col < it.n) {
                    const int slot = __ldcg(&a.sorted_slot[it.p0 + col]);
                    if (MOE_CHECKS && (slot < 0 || slot >= a.T * k1)) {
                        set_status(status, MOE_ERR_DEVICE_CHECK);
                        continue;  // weight 0 into token 0: adds nothing
                    }
                    tk[c] = slot / k1;
                    wt[c] = __ldcg(&a.topk_w[slot]);
                }
            }
            if (!g_wait_warp(&sy.acc_full[buf], (itc >> 1) & 1, status, lane)) {
                sy.abort = 1;
                break;
            }
            tc_fence_after();
            const uint32_t taddr = tmem + buf * 256 + ((uint32_t)(lq * 32) << 16);
            const int r = it.rt * kGBM + lq * 32 + lane;  // this thread's output row
            const int qd = lane & 3;                       // position in the lane quad
            const int rq = it.rt * kGBM + lq * 32 + (lane & ~3);  // the quad's first row
#pragma unroll
            for (int c = 0; c < kGBN / 32; ++c) {
                if ((c & 1) == eh && c * 32 < it.n) {
                    float v[32];
                    tmem_ld32(taddr + c * 32, v);
                    if (a.combine) {
                        // 4 x 4 transposes inside each lane quad: lane 4m+q gets rows
                        // 4m..4m+3 of token column j0+q and adds them with one vector red
#pragma unroll
                        for (int j0 = 0; j0 < 32; j0 += 4) {
                            float s0 = v[j0], s1 = v[j0 + 1], s2 = v[j0 + 2], s3 = v[j0 + 3];
                            const bool hi = qd & 2, od = qd & 1;
                            float t0 = __shfl_xor_sync(0xffffffffu, hi ? s0 : s2, 2);
                            float t1 = __shfl_xor_sync(0xffffffffu, hi ? s1 : s3, 2);
                            if (hi) {
                                s0 = t0;
                                s1 = t1;
                            } else {
                                s2 = t0;
                                s3 = t1;
                            }
                            t0 = __shfl_xor_sync(0xffffffffu, od ? s0 : s1, 1);
                            t1 = __shfl_xor_sync(0xffffffffu, od ? s2 : s3, 1);
                            const float o0 = od ? t0 : s0, o1 = od ? s1 : t0;
                            const float o2 = od ? t1 : s2, o3 = od ? s3 : t1;
                            const int col = j0 + qd;
                            const int t = __shfl_sync(0xffffffffu, tk[c], col);
                            const float w = __shfl_sync(0xffffffffu, wt[c], col);
                            if (c * 32 + col < it.n)
                                red_add_v4(a.y_acc + (size_t)t * d + rq, w * o0, w * o1, w * o2,
                                           w * o3);
                        }
                    } else {
                        const float b = a.bias ? __ldg(&a.bias[r]) : 0.0f;
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (c * 32 + j < it.n) {
                                const size_t o = (size_t)(it.p0 + c * 32 + j) * d + r;
                                const float val = a.bias ? __fadd_rn(v[j], b) : v[j];
                                a.out[o] = val;
                                if (a.out_copy)
                                    a.out_copy[o] = val;
                            }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sy.acc_empty[buf]);
            g_release_warp(sy, q, lane);
            ++itc;
        }
    }
    g_teardown(sy, tmem, a.sched, tid, warp);
}

// xs[p] = x[sorted_slot[p] / k1]: the routed tokens' rows in expert order, the
// token operand of the gate/up GEMM.  One warp per row, 16-byte vectors; only
// the offsets[E] placed slots (empty or dropped slots are not in the order),
// and a slot id beyond the T*k1 slots records MOE_ERR_DEVICE_CHECK and is
// skipped.  Also clears the down GEMM's float32 accumulator (zero: nullable,
// zero_n4 float4s).
__global__ void __launch_bounds__(256) k_gather_rows(const uint16_t *x, const int32_t *sorted_slot,
                                                     const int32_t *offsets, int E, int n, int d,
                                                     int k1, uint16_t *xs, float4 *zero,
                                                     int zero_n4, int *status)
{
    pdl_wait();
    pdl_trigger();
    if (zero)
        for (int q = blockIdx.x * 256 + threadIdx.x; q < zero_n4; q += gridDim.x * 256)
            zero[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    const int lane = threadIdx.x & 31;
    const int nv = d >> 3;
    const int placed = min(n, __ldcg(&offsets[E]));
    for (int p = blockIdx.x * 8 + (threadIdx.x >> 5); p < placed; p += gridDim.x * 8) {
        const int slot = __ldcg(&sorted_slot[p]);
        if (slot < 0 || slot >= n) {
            if (lane == 0)
                set_status(status, MOE_ERR_DEVICE_CHECK);
            continue;
        }
        const int t = slot / k1;
        const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)t * d);
        uint4 *dst = reinterpret_cast<uint4 *>(xs + (size_t)p * d);
        // eight 16-byte loads of the row in flight before their stores
        for (int v0 = lane; v0 < nv; v0 += 8 * 32) {
            uint4 r[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (v0 + 32 * u < nv)
                    r[u] = __ldg(&src[v0 + 32 * u]);
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (v0 + 32 * u < nv)
                    dst[v0 + 32 * u] = r[u];
        }
    }
}

// The grouped path's shapes: whole 128-row weight tiles on both GEMMs.
inline bool grouped_fits(int d, int E, int I) { return d % kGBM == 0 && I % kGBM == 0 && E <= kGMaxE; }

}  // namespace moe
