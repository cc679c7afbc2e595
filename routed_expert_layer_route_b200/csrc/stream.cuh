// stream.cuh -- small-batch expert FFN that streams only the activated
// experts' weights from HBM, each byte once.
//
// Structure of an expert ("Channel Selection for Mixture-of-Experts Decoding
// Needs No Calibration Data", section 2 "Background"): a gated MLP whose
// channel c owns gate row c, up row c and down column c.  SwiGLU:
//     h_c = silu(W_gate[c,:] . x) * (W_up[c,:] . x),   o = W_down h.
//
// Design (one persistent CTA per SM, grid = number of SMs):
//  * routing state first: either the CTA routes the single token itself from
//    its float32 logits (T == 1, every CTA redundantly, with the same fixed
//    float32 operation sequence as the router kernels), or it loads the
//    routing tables written by the permutation kernel -- in both cases in one
//    round of independent loads, into shared memory, together with the
//    tokens' x rows when they fit;
//  * the U activated experts (ascending ids) are laid end to end as U*I
//    channels; CTA b owns a contiguous channel range of floor(U*I/G) or one
//    more channels, so every CTA streams the same number of gate/up bytes
//    (within one channel) whatever k1, U or the batch;
//  * one producer thread moves the CTA's weights with bulk asynchronous
//    copies (cp.async.bulk, no multicast) into a ring of kStages shared-memory
//    stages; stage s lands in slot s % kStages and is consumed by the
//    consumer warps bound to that slot, each warp owning whole work units
//    (one channel = its gate row and up row; or one down row), so no stage
//    needs a cross-warp reduction or barrier;
//  * phase 1: gate/up rows of the CTA's channels -> h (float32) for them;
//  * one grid-wide barrier (bounded spins on per-CTA generation flags that
//    CTA 0 gathers, then one release flag; no same-address atomics) makes
//    every h visible;
//  * phase 2: CTA b owns a contiguous range of about d/G output rows of every
//    activated expert; its W_down rows (contiguous, I elements each) go
//    through the same ring -- the producer issues them before the barrier
//    completes, so the barrier hides under copies in flight;
//  * the combine with Eq. 2's weights runs on the CTA's own rows: y[t, r] =
//    sum_s w[t, s] o[slot(t, s), r] in slot order, float32, no atomics, so
//    the output is deterministic.
#pragma once
#include "common.cuh"
#include "route.cuh"

namespace moe {

constexpr int kSC = 12;                    // consumer warps (13 warps in all: <= 4 per SM
                                           // sub-partition, so up to 128 registers each)
constexpr int kSThreads = (kSC + 1) * 32;  // + one producer warp
constexpr int kStages = 4;
constexpr int kWPS = kSC / kStages;        // consumer warps bound to each ring slot
constexpr int kStageBytes = 32 * 1024;
constexpr int kTokChunk = 4;               // most tokens per dot-product pass
constexpr int kAreaBytes = 48 * 1024;      // x rows (phase 1) or h rows (phase 2)
constexpr int kMaxRows = 128;              // rows of one stage
constexpr int kMetaU = 1024;               // activated experts kept in shared memory
constexpr int kSlotMax = 1024;             // routed slots kept in shared memory
constexpr int kObufFloats = 4096;          // per-slot down outputs of this CTA's rows
constexpr int kConsumerBar = 1;            // named barrier id of the consumer warps

static_assert(kSC % kStages == 0, "consumer warps split evenly over the ring slots");

struct StreamArgs {
    const uint16_t *x;   // [T x d]
    const uint16_t *wg;  // [E x I x d]
    const uint16_t *wu;  // [E x I x d]
    const uint16_t *wd;  // [E x d x I]
    int T, d, E, I, k1, k2;
    // route_in_kernel (T == 1): route from logits[0..E) and write the routing
    // tables below (CTA 0); otherwise the tables are inputs.
    int route_in_kernel;
    const float *logits;
    int32_t *topk_idx;     // [T x k1]  (route mode: output)
    float *topk_w;         // [T x k1]  (route mode: output; combine: input)
    int32_t *idx_copy;     // nullable user copies (route mode)
    float *w_copy;
    int32_t *offsets;      // [E+1]
    int32_t *sorted_slot;  // [T*k1]
    int32_t *slot_pos;     // [T*k1]
    int32_t *uniq_count;   // [1]
    int32_t *uniq_list;    // [E]
    float *h;              // [T*k1 x I] scratch
    float *out;            // [T*k1 x d] per-slot outputs, sorted order (nullable when y is set)
    void *y;               // nullable: combine into y [T x d]
    int y_dtype;
    WsHeader *hdr;
};

// The ordered list of stages a CTA works through; the producer and every
// consumer warp walk it independently and identically.
struct Stage {
    int phase;  // 1: gate/up rows of channels [c, c+n); 2: W_down rows [r, r+n)
    int u;      // index into the activated-expert list
    int c;      // first channel (phase 1) or first row (phase 2)
    int n;      // channels (phase 1) or rows (phase 2)
};

struct StageIter {
    unsigned c_cur, c_hi;  // phase-1 channel cursor over [0, U*I)
    int r_lo, r_hi;        // phase-2 rows of this CTA
    int u2, r2;            // phase-2 cursor
    int U, I, nch, nrows;
    int phase;

    __device__ void init(int U_, int I_, int d, int b, int G)
    {
        U = U_;
        I = I_;
        const unsigned tot = (unsigned)U * (unsigned)I;
        c_cur = split_lo(tot, G, b);
        c_hi = split_lo(tot, G, b + 1);
        r_lo = (int)split_lo(d, G, b);
        r_hi = (int)split_lo(d, G, b + 1);
        // channels per stage: a multiple of the warps serving a slot when the
        // stage holds that many, so each warp owns the same number of units
        nch = max(1, min(kMaxRows / 2, kStageBytes / (4 * d)));
        if (nch >= kWPS)
            nch -= nch % kWPS;
        nrows = max(1, min(kMaxRows, kStageBytes / (2 * I)));
        u2 = 0;
        r2 = r_lo;
        phase = c_cur < c_hi ? 1 : 2;
        if (phase == 2 && (r_lo >= r_hi || U == 0))
            phase = 0;
    }
    __device__ bool valid() const { return phase != 0; }
    __device__ Stage get() const
    {
        Stage s;
        if (phase == 1) {
            s.phase = 1;
            s.u = (int)(c_cur / (unsigned)I);
            s.c = (int)(c_cur % (unsigned)I);
            const unsigned lim = min((unsigned)(I - s.c), c_hi - c_cur);
            s.n = (int)min((unsigned)nch, lim);
        } else {
            s.phase = 2;
            s.u = u2;
            s.c = r2;
            s.n = min(nrows, r_hi - r2);
        }
        return s;
    }
    __device__ void next()
    {
        const Stage s = get();
        if (phase == 1) {
            c_cur += s.n;
            if (c_cur >= c_hi)
                phase = (r_lo < r_hi && U > 0) ? 2 : 0;
        } else {
            r2 += s.n;
            if (r2 >= r_hi) {
                r2 = r_lo;
                if (++u2 >= U)
                    phase = 0;
            }
        }
    }
};

// Shared memory besides the ring (dynamic, right after the ring's barriers).
struct __align__(16) StreamSmem {
    float obuf[kObufFloats];  // o[p][r - r_lo] when it fits
    int ue[kMetaU];           // activated experts, ascending
    int up0[kMetaU];          // first sorted position of each
    int uM[kMetaU];           // tokens of each
    int stok[kSlotMax];       // token of each sorted position
    float sw[kSlotMax];       // Eq. 2 weight of each slot t*k1+s
    int spos[kSlotMax];       // sorted position of each slot
    int U;
    int abort;
    int issued;    // stages issued by the producer
    unsigned gen;  // grid-barrier generation of this launch
};

__device__ __forceinline__ void consumer_sync() { named_bar_sync(kConsumerBar, kSC * 32); }

__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.0f + __expf(-g)) * u; }

__device__ __forceinline__ void bf16x8(const uint4 v, float f[8])
{
    f[0] = bf16lo(v.x);
    f[1] = bf16hi(v.x);
    f[2] = bf16lo(v.y);
    f[3] = bf16hi(v.y);
    f[4] = bf16lo(v.z);
    f[5] = bf16hi(v.z);
    f[6] = bf16lo(v.w);
    f[7] = bf16hi(v.w);
}

// Row pointers of up to kTokChunk tokens, passed by value so they stay in
// registers.
struct XRows {
    const uint4 *r[kTokChunk];
};
struct HRows {
    const float4 *r[kTokChunk];
};

// One channel: g_t = W_gate[c,:] . x_t and u_t = W_up[c,:] . x_t for NT
// tokens (rows xr.r[t], bf16), reduced over the warp (every lane gets the sums).
template <int NT>
__device__ __forceinline__ void unit_gate_up(const uint4 *grow, const uint4 *urow, const XRows xr,
                                             int nvec, int lane, float (&g)[kTokChunk],
                                             float (&u)[kTokChunk])
{
    float ag[NT], au[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t)
        ag[t] = au[t] = 0.0f;
    for (int v = lane; v < nvec; v += 32) {
        const uint4 wg = grow[v], wu = urow[v];
        float fg[8], fu[8];
        bf16x8(wg, fg);
        bf16x8(wu, fu);
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            float xf[8];
            bf16x8(xr.r[t][v], xf);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                ag[t] = fmaf(fg[k], xf[k], ag[t]);
                au[t] = fmaf(fu[k], xf[k], au[t]);
            }
        }
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        g[t] = warp_sum(ag[t]);
        u[t] = warp_sum(au[t]);
    }
}

// One down row: o_t = W_down[r,:] . h_t for NT tokens (rows hr.r[t], float32).
template <int NT>
__device__ __forceinline__ void unit_down(const uint4 *wrow, const HRows hr, int nvec, int lane,
                                          float (&o)[kTokChunk])
{
    float acc[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t)
        acc[t] = 0.0f;
    for (int v = lane; v < nvec; v += 32) {
        float fw[8];
        bf16x8(wrow[v], fw);
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            const float4 h0 = hr.r[t][2 * v], h1 = hr.r[t][2 * v + 1];
            acc[t] = fmaf(fw[0], h0.x, acc[t]);
            acc[t] = fmaf(fw[1], h0.y, acc[t]);
            acc[t] = fmaf(fw[2], h0.z, acc[t]);
            acc[t] = fmaf(fw[3], h0.w, acc[t]);
            acc[t] = fmaf(fw[4], h1.x, acc[t]);
            acc[t] = fmaf(fw[5], h1.y, acc[t]);
            acc[t] = fmaf(fw[6], h1.z, acc[t]);
            acc[t] = fmaf(fw[7], h1.w, acc[t]);
        }
    }
#pragma unroll
    for (int t = 0; t < NT; ++t)
        o[t] = warp_sum(acc[t]);
}

// ---------------------------------------------------------------------------
// Single-token fast path (T == 1, d = 256*VPL, I = 256*VPLI): lane l always
// handles the 16-byte vectors l, l+32, ... of a row, so the token's x (phase
// 1) and the expert's h (phase 2) stay in registers and each warp's units run
// as long independent load/FMA streams with interleaved warp reductions.

// x of the single token: in registers for d <= 2048, else read from shared
// memory inside the loop (register budget).
constexpr int kXRegMax = 8;

// One channel: h = silu(W_gate[c,:] . x) * (W_up[c,:] . x), both rows at once.
template <int VPL>
__device__ __forceinline__ float fast_channel(const uint4 *grow, const uint4 *urow,
                                              const uint4 (&xv)[VPL <= kXRegMax ? VPL : 1],
                                              const uint4 *xs, int lane)
{
    float g0 = 0.f, g1 = 0.f, u0 = 0.f, u1 = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const uint4 wg = grow[lane + 32 * i];
        const uint4 wu = urow[lane + 32 * i];
        float xf[8], fg[8], fu[8];
        if constexpr (VPL <= kXRegMax)
            bf16x8(xv[i], xf);
        else
            bf16x8(xs[lane + 32 * i], xf);
        bf16x8(wg, fg);
        bf16x8(wu, fu);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            if (i & 1) {
                g1 = fmaf(fg[k], xf[k], g1);
                u1 = fmaf(fu[k], xf[k], u1);
            } else {
                g0 = fmaf(fg[k], xf[k], g0);
                u0 = fmaf(fu[k], xf[k], u0);
            }
        }
    }
    float g = g0 + g1, u = u0 + u1;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        g += __shfl_xor_sync(0xffffffffu, g, o);
        u += __shfl_xor_sync(0xffffffffu, u, o);
    }
    return silu_mul(g, u);
}

// Up to four down rows of one warp at once: o_r = W_down[row_r,:] . h.
template <int VPLI>
__device__ __forceinline__ void fast_rows(const uint8_t *stg, int I, int u0, int n,
                                          const float (&hv)[VPLI][8], int lane, float (&o)[4])
{
#pragma unroll
    for (int r = 0; r < 4; ++r)
        o[r] = 0.f;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int unit = u0 + r * kWPS;
        if (unit < n) {
            const uint4 *wrow = reinterpret_cast<const uint4 *>(stg + (size_t)unit * I * 2);
#pragma unroll
            for (int i = 0; i < VPLI; ++i) {
                float fw[8];
                bf16x8(wrow[lane + 32 * i], fw);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    o[r] = fmaf(fw[k], hv[i][k], o[r]);
            }
        }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
#pragma unroll
        for (int r = 0; r < 4; ++r)
            o[r] += __shfl_xor_sync(0xffffffffu, o[r], off);
    }
}

// The streaming kernel.  VPL/VPLI > 0 selects the single-token fast path for
// d = 256*VPL and I = 256*VPLI (x and h held in registers); VPL = VPLI = 0 is
// the general path (any T, d, I).
template <int VPL, int VPLI>
__global__ void __launch_bounds__(kSThreads, 1) k_stream(StreamArgs a)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *ring = smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kStages * kStageBytes);
    uint64_t *empty = full + kStages;
    StreamSmem *ss = reinterpret_cast<StreamSmem *>(empty + kStages);
    uint8_t *area = reinterpret_cast<uint8_t *>(ss + 1);  // kAreaBytes, 16-byte aligned

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x, b = blockIdx.x;
    int *status = &a.hdr->status;
    const int T = a.T, d = a.d, E = a.E, I = a.I, k1 = a.k1;
    const int nslots = T * k1;
    const bool slots_in_smem = nslots <= kSlotMax;
    const bool x_in_smem = (size_t)T * d * 2 <= (size_t)kAreaBytes;
    const bool h_in_smem = (size_t)nslots * I * 4 <= (size_t)kAreaBytes;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kWPS);
        }
        ss->abort = 0;
        ss->issued = 0;
        fence_mbar_init();
    }
    __syncthreads();

    pdl_wait();
    pdl_trigger();
    if (tid == 0)
        ss->gen = ld_relaxed_u32(&a.hdr->bar_go);  // cannot advance before this CTA arrives

    // ------------------------------------------------------------ routing state
    // the tokens' x rows (independent of routing) go out in the same round
    if (x_in_smem) {
        const int nv = T * (d >> 3);
        for (int i = tid; i < nv; i += kSThreads)
            reinterpret_cast<uint4 *>(area)[i] = reinterpret_cast<const uint4 *>(a.x)[i];
    }
    if (a.route_in_kernel) {
        // T == 1: every CTA ranks the E probabilities itself (the ring is idle
        // until routing is known, so the routing scratch lives there)
        RouteSmem &rs = *reinterpret_cast<RouteSmem *>(ring);
        float *zs = reinterpret_cast<float *>(ring + sizeof(RouteSmem));
        for (int j = tid; j < E; j += kSThreads)
            zs[j] = __ldcg(&a.logits[j]);
        __syncthreads();
        route_token_block(zs, E, k1, a.k2, rs, b == 0 ? a.topk_idx : nullptr,
                          b == 0 ? a.topk_w : nullptr, b == 0 ? a.idx_copy : nullptr,
                          b == 0 ? a.w_copy : nullptr);
        if (tid < k1) {
            const int e = rs.out_j[tid];
            int p = 0;
            for (int s = 0; s < k1; ++s)
                p += rs.out_j[s] < e;
            ss->ue[p] = e;
            ss->up0[p] = p;
            ss->uM[p] = 1;
            ss->stok[p] = 0;
            ss->sw[tid] = rs.out_w[tid];
            ss->spos[tid] = p;
            if (b == 0) {
                a.uniq_list[p] = e;
                a.sorted_slot[p] = tid;
                a.slot_pos[tid] = p;
            }
        }
        if (tid == 0) {
            ss->U = k1;
            if (b == 0)
                *a.uniq_count = k1;
        }
        if (b == 0) {
            for (int e = tid; e <= E; e += kSThreads) {
                int c = 0;
                for (int s = 0; s < k1; ++s)
                    c += rs.out_j[s] < e;
                a.offsets[e] = c;
            }
        }
        __syncthreads();
    } else {
        // tables written by the permutation kernel: one round of loads
        int *t_uniq = reinterpret_cast<int *>(ring);  // [E]
        int *t_off = t_uniq + 1024;                   // [E+1]
        for (int i = tid; i < E; i += kSThreads)
            t_uniq[i] = __ldcg(&a.uniq_list[i]);
        for (int i = tid; i <= E; i += kSThreads)
            t_off[i] = __ldcg(&a.offsets[i]);
        if (slots_in_smem) {
            for (int i = tid; i < nslots; i += kSThreads) {
                const int sl = __ldcg(&a.sorted_slot[i]);
                int t = sl / k1;
                if (sl < 0 || t >= T) {
                    set_status(status, MOE_ERR_DEVICE_CHECK);
                    t = 0;
                }
                ss->stok[i] = t;
                if (a.y) {
                    ss->sw[i] = __ldcg(&a.topk_w[i]);
                    int p = __ldcg(&a.slot_pos[i]);
                    if (p < 0 || p >= nslots) {
                        set_status(status, MOE_ERR_DEVICE_CHECK);
                        p = 0;
                    }
                    ss->spos[i] = p;
                }
            }
        }
        if (tid == 0) {
            int U = __ldcg(a.uniq_count);
            if (U < 0 || U > E || U > kMetaU) {
                set_status(status, MOE_ERR_DEVICE_CHECK);
                U = 0;
            }
            ss->U = U;
        }
        __syncthreads();
        const int U = ss->U;
        for (int u = tid; u < U; u += kSThreads) {
            const int e = min(max(t_uniq[u], 0), E - 1);
            int p0 = t_off[e], M = t_off[e + 1] - p0;
            if (p0 < 0 || M < 0 || p0 + M > nslots) {  // inconsistent routing state
                set_status(status, MOE_ERR_DEVICE_CHECK);
                p0 = 0;
                M = 0;
            }
            ss->ue[u] = e;
            ss->up0[u] = p0;
            ss->uM[u] = M;
        }
        __syncthreads();
    }
    const int U = ss->U;
    const int r_lo = (int)split_lo(d, G, b), r_hi = (int)split_lo(d, G, b + 1);
    const int nr = r_hi - r_lo;
    const bool obuf_ok = a.y && (size_t)nslots * nr <= (size_t)kObufFloats;

    if (warp == kSC) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol = l2_evict_first_policy();
            StageIter it;
            it.init(U, I, d, b, G);
            int slot = 0;
            uint32_t ph = 0;
            int issued = 0;
            while (it.valid()) {
                if (*(volatile int *)&ss->abort)
                    break;
                if (!mbar_wait_live(&empty[slot], ph ^ 1u, &ss->abort, status)) {
                    ss->abort = 1;
                    break;
                }
                const Stage st = it.get();
                const int e = ss->ue[st.u];
                uint8_t *dst = ring + (size_t)slot * kStageBytes;
                if (st.phase == 1) {
                    const uint32_t bytes = (uint32_t)st.n * d * 2;
                    const size_t row0 = (size_t)e * I + st.c;
                    mbar_arrive_expect_tx(&full[slot], 2 * bytes);
                    bulk_g2s(dst, a.wg + row0 * d, bytes, &full[slot], pol);
                    bulk_g2s(dst + bytes, a.wu + row0 * d, bytes, &full[slot], pol);
                } else {
                    const uint32_t bytes = (uint32_t)st.n * I * 2;
                    mbar_arrive_expect_tx(&full[slot], bytes);
                    bulk_g2s(dst, a.wd + ((size_t)e * d + st.c) * I, bytes, &full[slot], pol);
                }
                ++issued;
                it.next();
                if (++slot == kStages) {
                    slot = 0;
                    ph ^= 1u;
                }
            }
            ss->issued = issued;
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ consumers
        const int group = warp / kWPS;  // the ring slot this warp serves
        const int gl = warp % kWPS;     // this warp's index inside its group
        StageIter it;
        it.init(U, I, d, b, G);
        int sidx = 0;  // global stage index

        // Wait for stage sidx if this warp serves its slot; returns the stage
        // buffer, or nullptr when this warp skips the stage (not its slot) or
        // the launch aborted.  Every stage acquired is handed back with
        // release(); one not acquired is not, so the producer refills a slot
        // only once its copies have landed.
        auto acquire = [&](bool &mine) -> const uint8_t * {
            mine = (sidx % kStages) == group;
            if (!mine)
                return nullptr;
            const uint32_t parity = (uint32_t)((sidx / kStages) & 1);
            bool ok = !*(volatile int *)&ss->abort &&
                      mbar_wait_live(&full[group], parity, &ss->abort, status);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) {
                if (lane == 0)
                    ss->abort = 1;
                return nullptr;
            }
            return ring + (size_t)group * kStageBytes;
        };
        auto release = [&]() {
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&empty[group]);
        };
        auto x_row = [&](int p) -> const uint4 * {
            int t;
            if (slots_in_smem) {
                t = ss->stok[p];
            } else {
                const int sl = __ldcg(&a.sorted_slot[p]);
                t = sl / k1;
                if (sl < 0 || t >= T)
                    t = 0;
            }
            return x_in_smem ? reinterpret_cast<const uint4 *>(area + (size_t)t * d * 2)
                             : reinterpret_cast<const uint4 *>(a.x + (size_t)t * d);
        };
        auto h_row = [&](int p) -> const float4 * {
            return h_in_smem ? reinterpret_cast<const float4 *>(area + (size_t)p * I * 4)
                             : reinterpret_cast<const float4 *>(a.h + (size_t)p * I);
        };

        // ---------------------------------------------------- phase 1: h
        {
            uint4 xv[VPL > 0 && VPL <= kXRegMax ? VPL : 1];
            const uint4 *xs = reinterpret_cast<const uint4 *>(area);
            if constexpr (VPL > 0 && VPL <= kXRegMax) {
#pragma unroll
                for (int i = 0; i < VPL; ++i)
                    xv[i] = xs[lane + 32 * i];
            }
            while (it.valid() && it.phase == 1) {
                const Stage st = it.get();
                bool mine;
                const uint8_t *stg = acquire(mine);
                if (stg) {
                    const int p0 = ss->up0[st.u];
                    const int M = ss->uM[st.u];
                    for (int unit = gl; unit < st.n; unit += kWPS) {
                        const uint4 *grow = reinterpret_cast<const uint4 *>(stg + (size_t)unit * d * 2);
                        const uint4 *urow =
                            reinterpret_cast<const uint4 *>(stg + (size_t)(st.n + unit) * d * 2);
                        if constexpr (VPL > 0) {
                            const float hval = fast_channel<VPL>(grow, urow, xv, xs, lane);
                            if (lane == 0)
                                a.h[(size_t)p0 * I + st.c + unit] = hval;
                        } else {
                            for (int m0 = 0; m0 < M; m0 += kTokChunk) {
                                const int mt = min(kTokChunk, M - m0);
                                float r0[kTokChunk], r1[kTokChunk];
                                XRows xr;
#pragma unroll
                                for (int t = 0; t < kTokChunk; ++t)
                                    xr.r[t] = x_row(p0 + m0 + min(t, mt - 1));
                                const int nvec = d >> 3;
                                if (mt == 1)
                                    unit_gate_up<1>(grow, urow, xr, nvec, lane, r0, r1);
                                else if (mt == 2)
                                    unit_gate_up<2>(grow, urow, xr, nvec, lane, r0, r1);
                                else
                                    unit_gate_up<4>(grow, urow, xr, nvec, lane, r0, r1);
#pragma unroll
                                for (int t = 0; t < kTokChunk; ++t)
                                    if (lane == t && t < mt)
                                        a.h[(size_t)(p0 + m0 + t) * I + st.c + unit] =
                                            silu_mul(r0[t], r1[t]);
                            }
                        }
                    }
                }
                if (stg)
                    release();
                ++sidx;
                it.next();
            }
        }

        // ---------------------------------------------------- grid barrier
        // every CTA's h is written before any is read
        consumer_sync();
        {
            const unsigned target = ss->gen + 1u;
            if (tid == 0)
                st_release_u32(&a.hdr->bar_flag[b], target);
            if (b == 0) {
                // CTA 0 gathers every CTA's arrival flag, then releases all
                for (int i = tid; i < G; i += kSC * 32)
                    if (!wait_flag_eq(&a.hdr->bar_flag[i], target, status))
                        ss->abort = 1;
                consumer_sync();
                if (tid == 0)
                    st_release_u32(&a.hdr->bar_go, target);
            }
            if (tid == 0 && !wait_flag_eq(&a.hdr->bar_go, target, status))
                ss->abort = 1;
        }
        consumer_sync();
        if (h_in_smem && it.valid()) {
            const int n4 = nslots * (I >> 2);
            for (int i = tid; i < n4; i += kSC * 32)
                reinterpret_cast<float4 *>(area)[i] = __ldcg(reinterpret_cast<const float4 *>(a.h) + i);
            consumer_sync();
        }

        // ---------------------------------------------------- phase 2: o
        {
            float hv[VPLI > 0 ? VPLI : 1][8];
            int hv_pos = -1;
            while (it.valid()) {
                const Stage st = it.get();
                bool mine;
                const uint8_t *stg = acquire(mine);
                if (stg) {
                    const int p0 = ss->up0[st.u];
                    const int M = ss->uM[st.u];
                    if constexpr (VPLI > 0) {
                        if (hv_pos != p0) {  // this expert's h into registers
                            const float4 *hs = reinterpret_cast<const float4 *>(area + (size_t)p0 * I * 4);
#pragma unroll
                            for (int i = 0; i < VPLI; ++i) {
                                const float4 q0 = hs[2 * (lane + 32 * i)];
                                const float4 q1 = hs[2 * (lane + 32 * i) + 1];
                                hv[i][0] = q0.x;
                                hv[i][1] = q0.y;
                                hv[i][2] = q0.z;
                                hv[i][3] = q0.w;
                                hv[i][4] = q1.x;
                                hv[i][5] = q1.y;
                                hv[i][6] = q1.z;
                                hv[i][7] = q1.w;
                            }
                            hv_pos = p0;
                        }
                        for (int u0 = gl; u0 < st.n; u0 += 4 * kWPS) {
                            float o[4];
                            fast_rows<VPLI>(stg, I, u0, st.n, hv, lane, o);
#pragma unroll
                            for (int r = 0; r < 4; ++r) {
                                const int unit = u0 + r * kWPS;
                                if (lane == r && unit < st.n) {
                                    const int row = st.c + unit;
                                    if (obuf_ok)
                                        ss->obuf[p0 * nr + (row - r_lo)] = o[r];
                                    else
                                        a.out[(size_t)p0 * d + row] = o[r];
                                }
                            }
                        }
                    } else {
                        for (int unit = gl; unit < st.n; unit += kWPS) {
                            const uint4 *wrow = reinterpret_cast<const uint4 *>(stg + (size_t)unit * I * 2);
                            const int row = st.c + unit;
                            for (int m0 = 0; m0 < M; m0 += kTokChunk) {
                                const int mt = min(kTokChunk, M - m0);
                                float r0[kTokChunk];
                                HRows hr;
#pragma unroll
                                for (int t = 0; t < kTokChunk; ++t)
                                    hr.r[t] = h_row(p0 + m0 + min(t, mt - 1));
                                const int nvec = I >> 3;
                                if (mt == 1)
                                    unit_down<1>(wrow, hr, nvec, lane, r0);
                                else if (mt == 2)
                                    unit_down<2>(wrow, hr, nvec, lane, r0);
                                else
                                    unit_down<4>(wrow, hr, nvec, lane, r0);
#pragma unroll
                                for (int t = 0; t < kTokChunk; ++t) {
                                    if (lane == t && t < mt) {
                                        const int p = p0 + m0 + t;
                                        if (obuf_ok)
                                            ss->obuf[p * nr + (row - r_lo)] = r0[t];
                                        else
                                            a.out[(size_t)p * d + row] = r0[t];
                                    }
                                }
                            }
                        }
                    }
                }
                if (stg)
                    release();
                ++sidx;
                it.next();
            }
        }

        // ------------------------------------------------------------ combine
        if (a.y) {
            consumer_sync();  // every o of this CTA's rows is written
            for (int i = tid; i < T * nr; i += kSC * 32) {
                const int t = i / nr, r = r_lo + i % nr;
                float acc = 0.0f;
                for (int s = 0; s < k1; ++s) {
                    const int sl = t * k1 + s;
                    int pos;
                    float w;
                    if (slots_in_smem) {
                        pos = ss->spos[sl];
                        w = ss->sw[sl];
                    } else {
                        pos = __ldcg(&a.slot_pos[sl]);
                        w = __ldcg(&a.topk_w[sl]);
                        if (pos < 0 || pos >= nslots) {
                            set_status(status, MOE_ERR_DEVICE_CHECK);
                            continue;
                        }
                    }
                    const float o = obuf_ok ? ss->obuf[pos * nr + (r - r_lo)] : a.out[(size_t)pos * d + r];
                    const float prod = w * o;
                    acc = acc + prod;
                }
                if (a.y_dtype == MOE_DTYPE_BF16)
                    reinterpret_cast<uint16_t *>(a.y)[(size_t)t * d + r] = f32_to_bf16_rn(acc);
                else
                    reinterpret_cast<float *>(a.y)[(size_t)t * d + r] = acc;
            }
        }
    }

    __syncthreads();
    // After an abort, wait (bounded) for copies that may still be in flight
    // before the CTA's shared memory is released.
    if (tid == 0 && ss->abort) {
        const int issued = ss->issued;
        for (int s = 0; s < kStages && s < issued; ++s) {
            const int last = issued - 1 - ((issued - 1 - s) % kStages);  // last stage on slot s
            const uint32_t parity = (uint32_t)((last / kStages) & 1);
            mbar_wait(&full[s], parity, status);
        }
    }
}

// Which instantiation serves these shapes: the single-token fast path when x
// and every routed slot's h fit the shared-memory staging area.
inline int stream_variant(int T, int d, int I, int k1)
{
    if (T != 1 || (size_t)d * 2 > (size_t)kAreaBytes || (size_t)k1 * I * 4 > (size_t)kAreaBytes)
        return 0;
    if (d == 2048 && I == 768)
        return 1;
    if (d == 4096 && I == 1024)
        return 2;
    return 0;
}

inline size_t stream_smem_bytes()
{
    return (size_t)kStages * kStageBytes + 2 * kStages * sizeof(uint64_t) + sizeof(StreamSmem) +
           kAreaBytes;
}

}  // namespace moe
