// decode_mt.cuh -- the few-token layer kernel (2 <= T <= 8 tokens per call):
// router logits, routing, the routed experts' SwiGLU FFN and the weighted
// combine in one launch, each activated expert's weight bytes read once from
// HBM however many of the tokens route to it.
//
// An expert is read as in the one-token kernel (decode.cuh): with the down
// matrix stored channel-major, channel c of expert e is three contiguous rows
// (gate row c, up row c, down column c; "Channel Selection for
// Mixture-of-Experts Decoding Needs No Calibration Data", section 2
// "Background"), and
//     y_t[:] += w_{t,e} * h_{t,c} * down_row_c
// for every token t routed to e, w the Eq. 2 weight ("Paper of the Week #3",
// section "The Receipt").
//
// Design (one CTA per SM, cooperative launch; 11 consumer warps + 1 producer):
//  * every CTA stages the T tokens' x rows in shared memory; router CTA b
//    fetches router rows R*b .. R*b+R-1 (R = ceil(E / grid)) before the
//    programmatic-launch wait, and its consumer warps share the R*T dot
//    products (row, token), each in the order of k_logits; every logit is
//    one arrival (number t*E + e) on the spread release counters;
//  * warps t < T wait (bounded) for all E*T arrivals and route token t
//    (warp_route_vals: the float32 softmax, top-k2, Eq. 2); warp 0 then forms
//    the union of the routed experts, ascending, each with its tokens (a bit
//    mask) and their weights;
//  * the U activated experts are laid end to end as U*I channels, CTA b takes
//    a balanced contiguous range, and the producer streams stages of whole
//    channels (up to eight: two slots of the largest size that fits) through
//    the bulk-copy ring;
//  * all 11 consumer warps serve every stage: first the gate and up dot
//    products of the stage's (channel, token) pairs -- a job per channel and
//    chunk of at most two of the expert's tokens (a gate/up vector read once
//    for both), dealt over the warps -- with w*h into shared memory (two buffers by
//    stage parity); after the consumer barrier each warp adds w*h*down_row
//    into the register partials of its own output rows, one set per token
//    slot of the current expert -- the warps own disjoint rows, so no partial
//    meets another inside the CTA.  Stage bookkeeping takes no division.
//  * when the stage's expert changes (a CTA's range spans one to a few
//    experts), and at the end, each warp adds its partials into the float32
//    accumulator [T x d] with 16-byte vector reductions; one ticket per CTA;
//    the last converts the accumulator to y and clears it.
// The accumulation order across CTAs is the order of their reductions, so y
// can differ between runs in the last bits (as in the one-token kernel).
#pragma once
#include "decode.cuh"

namespace moe {

constexpr int kMtMaxT = 8;        // tokens per call
constexpr int kMtMaxSlots = 64;   // T * k1
constexpr int kMtMaxRowVec = 2;   // 16-byte row vectors per lane (d <= 5632)
constexpr int kMtMaxCh = 8;       // channels per stage
// 11 consumer warps and the producer: 12 warps, three per scheduler, so a
// thread may hold up to 168 registers (the per-token row partials)
constexpr int kMtC = 11;
constexpr int kMtThreads = (kMtC + 1) * 32;

struct MtArgs {
    const uint16_t *x;    // [T x d]
    const uint16_t *wg;   // [E x I x d]
    const uint16_t *wu;   // [E x I x d]
    const uint16_t *wdt;  // [E x I x d]: down matrix, channel-major
    const uint16_t *wr;   // [E x d] router
    const float *bias;    // [E], nullable
    float *logits;        // [T x E] float32 (workspace)
    float *logits_out;    // [T x E], nullable
    int32_t *topk_idx;    // [T x k1] (workspace)
    float *topk_w;
    int32_t *idx_copy;    // nullable
    float *w_copy;        // nullable
    int32_t *count;       // [T], nullable: slots taken per token
    float *yacc;          // [T x d] float32, zero on entry; the last CTA clears it again
    void *y;              // [T x d] output (y_dtype)
    int y_dtype;
    int T, d, E, I, k1, k2;
    int rrows;            // router rows per router CTA (at least ceil(E / grid))
    int nslots;           // ring slots (mt_layout)
    VarK vk;              // fixed k, cascade or skip
    WsHeader *hdr;
};

struct __align__(16) MtSmem {
    float hs[2][kMtMaxCh][kMtMaxT];   // w*h of the stage's channels per token slot, by stage parity
    float uw[kMtMaxSlots][kMtMaxT];   // activated expert u, token slot k: the Eq. 2 weight
    uint8_t utok[kMtMaxSlots][kMtMaxT];  //   the token (slots k < popc(tmask[u]), ascending)
    int sj[kMtMaxSlots];              // the route by slot t*k1 + s: expert (or MOE_EMPTY_SLOT),
    float sw[kMtMaxSlots];            //   weight
    unsigned bits[kMaxExperts / 32];  // the activated experts
    int wpre[kMaxExperts / 32];       // activated experts in the words before
    int ue[kMtMaxSlots];              // the activated experts, ascending
    unsigned tmask[kMtMaxSlots];      // the tokens routed to each
    int ktok[kMtMaxT];                // slots taken per token
    DSeg seg[kDMaxSeg];
    int nseg;
    int U;
    int abort;
    int issued;
    int last;
    unsigned call;
};

// Shared memory of the few-token kernel: MtSmem, the barriers, the T tokens'
// x rows (widened to float32 once), then the ring.  A stage is nch whole
// channels (three d-element bf16 rows each, 6d bytes): the most, up to
// kMtMaxCh, of which two slots fit -- a stage's cost is dominated by one dot
// job's latency and grows slowly with its channels, so two large slots move
// more bytes per stage than more small ones (measured at T = 2, 4, 8).
struct MtLayout {
    size_t bar_off, x_off, ring_off, stage, total;
    int nch, nslots;
};
__host__ __device__ inline MtLayout mt_layout(int T, int d)
{
    MtLayout L;
    L.bar_off = sizeof(MtSmem);
    L.x_off = L.bar_off + (2 * kDSlots + 2) * sizeof(uint64_t);
    L.ring_off = (L.x_off + (size_t)T * d * 4 + 127) & ~(size_t)127;  // x as float32
    const size_t cap = 227 * 1024;
    const size_t room = cap > L.ring_off ? cap - L.ring_off : 0;
    const size_t ch = (size_t)6 * d;  // one channel's rows
    const int n = (int)(room / 2 / ch);
    L.nch = n > kMtMaxCh ? kMtMaxCh : n;
    L.stage = (size_t)L.nch * ch;
    const int ns = L.nch > 0 ? (int)(room / L.stage) : 0;
    L.nslots = ns > kDSlots ? kDSlots : ns;
    L.total = L.ring_off + (size_t)L.nslots * L.stage;
    return L;
}

// This CTA's channel segments of the U activated experts (the split of the
// one-token kernel).
__device__ void mt_segments(MtSmem *ms, int U, int I, int G, int b, int *status)
{
    const unsigned tot = (unsigned)U * (unsigned)I;
    const unsigned c_lo = split_lo(tot, G, b), c_hi = split_lo(tot, G, b + 1);
    int ns = 0;
    unsigned c = c_lo;
    for (; c < c_hi && ns < kDMaxSeg;) {
        const int u = (int)(c / (unsigned)I);
        DSeg sg;
        sg.u = u;
        sg.a = (int)(c % (unsigned)I);
        sg.b = (int)min((unsigned)I, c_hi - (unsigned)u * I);
        ms->seg[ns++] = sg;
        c = (unsigned)u * I + sg.b;
    }
    if (c < c_hi) {  // more segments than kDMaxSeg: the host rules this out
        set_status(status, MOE_ERR_DEVICE_CHECK);
        ns = 0;
    }
    ms->nseg = ns;
}

MOE_DEVINL void mt_sync() { named_bar_sync(kConsumerBar, kMtC * 32); }

// j / n for 1 <= n <= kMtMaxCh and 0 <= j < 40: (j * ceil(256 / n)) >> 8.
MOE_DEVINL int div_small(int j, int n)
{
    const int mul = n == 1 ? 256 : n == 2 ? 128 : n == 3 ? 86 : n == 4 ? 64 : n == 5 ? 52
                  : n == 6 ? 43 : n == 7 ? 37 : 32;
    return (j * mul) >> 8;
}

// Token position of the r-th set bit of m (r < popc(m)).
MOE_DEVINL int nth_bit(unsigned m, int r)
{
    for (int k = 0; k < r; ++k)
        m &= m - 1u;
    return __ffs(m) - 1;
}

// One step of a gate/up dot pair with paired float32 FMAs: 16-byte weight
// vectors wg, wu against the token's 8 x values (float32 pairs xa, xb).
MOE_DEVINL void mt_step(uint64_t &g, uint64_t &u, const uint4 wg, const uint4 wu,
                        const ulonglong2 xa, const ulonglong2 xb)
{
    const uint64_t x0 = xa.x, x1 = xa.y, x2 = xb.x, x3 = xb.y;
    g = ffma2(bf16x2_pair(wg.x), x0, g);
    u = ffma2(bf16x2_pair(wu.x), x0, u);
    g = ffma2(bf16x2_pair(wg.y), x1, g);
    u = ffma2(bf16x2_pair(wu.y), x1, u);
    g = ffma2(bf16x2_pair(wg.z), x2, g);
    u = ffma2(bf16x2_pair(wu.z), x2, u);
    g = ffma2(bf16x2_pair(wg.w), x3, g);
    u = ffma2(bf16x2_pair(wu.w), x3, u);
}

MOE_DEVINL float pair_total(uint64_t a, uint64_t b)
{
    return (pair_lo(a) + pair_hi(a)) + (pair_lo(b) + pair_hi(b));
}

// h = SiLU(gate_row . x_t) * (up_row . x_t) for NT tokens (1 or 2) of one
// channel, the weight vectors read once for both; two partial chains per dot
// product (vectors lane + 64i and lane + 64i + 32).  x0, x1: the tokens' rows
// as two planes of float32 pairs, elements 0-3 of 16-byte vector v at [v],
// elements 4-7 at [v + nvec] (consecutive lanes read consecutive 16 bytes).
template <int NT>
MOE_DEVINL void mt_channel(const uint4 *grow, const uint4 *urow, const ulonglong2 *x0,
                           const ulonglong2 *x1, int nvec, int lane, float (&h)[2])
{
    uint64_t g[NT][2], u[NT][2];
#pragma unroll
    for (int t = 0; t < NT; ++t)
        g[t][0] = g[t][1] = u[t][0] = u[t][1] = 0;
    for (int v = lane; v < nvec; v += 64) {
        const bool second = v + 32 < nvec;
        const uint4 z = make_uint4(0, 0, 0, 0);
        const uint4 wg0 = grow[v], wu0 = urow[v];
        const uint4 wg1 = second ? grow[v + 32] : z, wu1 = second ? urow[v + 32] : z;
        mt_step(g[0][0], u[0][0], wg0, wu0, x0[v], x0[v + nvec]);
        if (second)
            mt_step(g[0][1], u[0][1], wg1, wu1, x0[v + 32], x0[v + 32 + nvec]);
        if constexpr (NT > 1) {
            mt_step(g[1][0], u[1][0], wg0, wu0, x1[v], x1[v + nvec]);
            if (second)
                mt_step(g[1][1], u[1][1], wg1, wu1, x1[v + 32], x1[v + 32 + nvec]);
        }
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        float gs = pair_total(g[t][0], g[t][1]);
        float us = pair_total(u[t][0], u[t][1]);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            gs += __shfl_xor_sync(0xffffffffu, gs, o);
            us += __shfl_xor_sync(0xffffffffu, us, o);
        }
        h[t] = silu_mul(gs, us);
    }
}

// Token t's route (one warp): its E logits, read once the exchange has
// counted them all (or zeros after a failed wait), through warp_route_vals.
template <int R>
__device__ __forceinline__ void mt_route(const MtArgs &a, int t, bool ok, int lane, int &my_j,
                                         float &my_w, int &kt)
{
    const int E = a.E;
    float p[R];
#pragma unroll
    for (int i = 0; i < R; ++i) {
        const int j = lane + 32 * i;
        p[i] = j < E && ok ? __ldcg(&a.logits[(size_t)t * E + j]) : 0.0f;
    }
    warp_route_vals<R>(p, E, a.k1, a.k2, lane, my_j, my_w, a.vk, &kt);
}

// The down phase of one stage for one warp: y partials += w*h * down row for
// the warp's rows (vectors v = warp*32 + lane + kMtC*32*j) and token slots
// k < MM, every slot branch-free with w*h = 0 at k >= m (those slots are
// dropped, not added, at the next flush).  MM >= m is chosen per stage, so
// an expert with one or two tokens costs one or two slots' FMAs, not TM's.
template <int MM, int TM, int RVM>
MOE_DEVINL void mt_down(uint64_t (&yq)[TM][RVM][4], const float (&hs)[kMtMaxCh][kMtMaxT],
                        const uint8_t *drows, int n, int m, int d, int nvec, int warp, int lane)
{
#pragma unroll
    for (int c = 0; c < kMtMaxCh; ++c) {
        if (c < n) {
            const uint4 *drow = reinterpret_cast<const uint4 *>(drows + (size_t)c * d * 2);
#pragma unroll
            for (int j = 0; j < RVM; ++j) {
                const int v = warp * 32 + lane + kMtC * 32 * j;
                if (v < nvec) {
                    const uint4 w = drow[v];
                    const uint64_t w0 = bf16x2_pair(w.x), w1 = bf16x2_pair(w.y);
                    const uint64_t w2 = bf16x2_pair(w.z), w3 = bf16x2_pair(w.w);
#pragma unroll
                    for (int k = 0; k < MM; ++k) {
                        const float hv = k < m ? hs[c][k] : 0.0f;
                        const uint64_t h2 = f32_pair(hv, hv);
                        yq[k][j][0] = ffma2(w0, h2, yq[k][j][0]);
                        yq[k][j][1] = ffma2(w1, h2, yq[k][j][1]);
                        yq[k][j][2] = ffma2(w2, h2, yq[k][j][2]);
                        yq[k][j][3] = ffma2(w3, h2, yq[k][j][3]);
                    }
                }
            }
        }
    }
}

// TM: tokens the partials cover (T <= TM); RVM: 16-byte output-row vectors per
// lane (d <= RVM * kMtC * 256).
template <int TM, int RVM>
__global__ void __launch_bounds__(kMtThreads, 1) k_decode_mt(MtArgs a)
{
    static_assert(TM <= kMtMaxT && RVM <= kMtMaxRowVec, "few-token kernel: partials");
    extern __shared__ __align__(1024) uint8_t smem[];
    MtSmem *ms = reinterpret_cast<MtSmem *>(smem);
    const MtLayout L = mt_layout(a.T, a.d);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    uint64_t *empty = full + kDSlots;
    uint64_t *rbar = empty + kDSlots;  // the router rows' bulk copies
    float *xs = reinterpret_cast<float *>(smem + L.x_off);  // [T][2 planes][d/2] float32
    uint8_t *ring = smem + L.ring_off;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x, b = blockIdx.x;
    int *status = &a.hdr->status;
    const int T = a.T, d = a.d, E = a.E, I = a.I, k1 = a.k1;
    const int NS = a.nslots;
    const int R = max(a.rrows, (E + G - 1) / G);                // the grid covers all E rows
    const int nr = b * R < E ? min(R, E - b * R) : 0;           // router rows e = R*b + i
    const int nvec = d >> 3;                                    // 16-byte vectors per row

    if (tid == 0) {
        for (int s = 0; s < kDSlots; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kMtC);
        }
        mbar_init(rbar, 1);
        ms->abort = 0;
        ms->issued = 0;
        fence_mbar_init();
    }
    __syncthreads();
    // this CTA's router rows: weights no earlier kernel writes, so they are
    // fetched before the dependency wait and overlap the previous kernel
    if (warp == kMtC && lane == 0 && nr > 0) {
        const uint64_t keep = l2_evict_last_policy();  // the router, read by every call
        mbar_arrive_expect_tx(rbar, (uint32_t)(nr * d * 2));
        for (int i = 0; i < nr; ++i)
            bulk_g2s(ring + (size_t)i * d * 2, a.wr + (size_t)(b * R + i) * d, (uint32_t)(d * 2),
                     rbar, keep);
    }

    pdl_wait();
    pdl_trigger();

    if (warp < kMtC) {
        const unsigned call = ld_relaxed_u32(&a.hdr->decode_seq) + 1u;
        const unsigned slot = call & 3u;
        if (b == 0 && tid < kSpread)  // the count of the call two ahead starts at zero
            a.hdr->xcnt[(call + 2u) & 3u].c[tid][0] = 0u;
        // ------------------------------------------------------------ x rows
        // widened to float32 once (exact), for the router and the dot jobs
        {
            const uint4 *xg = reinterpret_cast<const uint4 *>(a.x);
            for (int i = tid; i < T * nvec; i += kMtC * 32) {
                const int t = i / nvec, v = i - t * nvec;
                const uint4 w = xg[i];
                float4 *row = reinterpret_cast<float4 *>(xs + (size_t)t * d);
                row[v] = make_float4(bf16lo(w.x), bf16hi(w.x), bf16lo(w.y), bf16hi(w.y));
                row[v + nvec] = make_float4(bf16lo(w.z), bf16hi(w.z), bf16lo(w.w), bf16hi(w.w));
            }
        }
        mt_sync();
        // ------------------------------------------------------------ router logits
        // dot product (row i, token t) = job i*T + t, shared by the consumer
        // warps; each in router_step's order (the order of k_logits)
        if (warp < nr * T) {
            if (!mbar_wait(rbar, 0, status))
                ms->abort = 1;
            for (int job = warp; job < nr * T; job += kMtC) {
                const int i = job / T, t = job % T;
                const uint4 *row = reinterpret_cast<const uint4 *>(ring + (size_t)i * d * 2);
                const float *xt = xs + (size_t)t * d;
                float a0 = 0.0f, a1 = 0.0f;
                int q = 0;
                for (int v = lane; v < nvec; v += 32, ++q) {
                    // router_step's order (k_logits): vectors alternate between a0 and a1
                    float xf[8];
                    *reinterpret_cast<float4 *>(xf) = reinterpret_cast<const float4 *>(xt)[v];
                    *reinterpret_cast<float4 *>(xf + 4) =
                        reinterpret_cast<const float4 *>(xt)[v + nvec];
                    if (q & 1)
                        a1 = dot8_bf16(row[v], xf, a1);
                    else
                        a0 = dot8_bf16(row[v], xf, a0);
                }
                float z = warp_sum(a0 + a1);
                const int e = b * R + i;
                if (a.bias)
                    z = z + a.bias[e];
                if (lane == 0) {
                    a.logits[(size_t)t * E + e] = z;
                    if (a.logits_out)
                        a.logits_out[(size_t)t * E + e] = z;
                    spread_arrive(&a.hdr->xcnt[slot], (unsigned)(t * E + e));  // logit, then count
                }
            }
        }

        // ------------------------------------------------------------ routing (warp t: token t)
        if (warp < T) {
            const bool ok = warp_wait_spread(&a.hdr->xcnt[slot], (unsigned)(E * T), lane, status);
            if (!ok && lane == 0)
                ms->abort = 1;
            int j, kt;
            float wv;
            if (E <= 128)
                mt_route<4>(a, warp, ok, lane, j, wv, kt);
            else if (E <= 256)
                mt_route<8>(a, warp, ok, lane, j, wv, kt);
            else if (E <= 512)
                mt_route<16>(a, warp, ok, lane, j, wv, kt);
            else
                mt_route<32>(a, warp, ok, lane, j, wv, kt);
            if (MOE_CHECKS) {  // the route: experts in range, kt slots taken
                const bool bad = (lane < k1 && j != MOE_EMPTY_SLOT && (j < 0 || j >= E)) ||
                                 kt < 0 || kt > k1;
                if (__any_sync(0xffffffffu, bad)) {
                    if (lane == 0) {
                        set_status(status, MOE_ERR_DEVICE_CHECK);
                        ms->abort = 1;
                    }
                    j = MOE_EMPTY_SLOT;
                    wv = 0.0f;
                    kt = 0;
                }
            }
            if (lane < k1) {
                ms->sj[warp * k1 + lane] = j;
                ms->sw[warp * k1 + lane] = wv;
            }
            if (lane == 0)
                ms->ktok[warp] = kt;
        }
        mt_sync();

        // ------------------------------------------------------------ the union (warp 0)
        if (warp == 0) {
            const int nw = (E + 31) >> 5;  // <= 32
            const int n = T * k1;
            if (lane < nw)
                ms->bits[lane] = 0u;
            for (int i = lane; i < kMtMaxSlots; i += 32)
                ms->tmask[i] = 0u;
            __syncwarp();
            for (int i = lane; i < n; i += 32) {
                const int j = ms->sj[i];
                if (j != MOE_EMPTY_SLOT)
                    atomicOr(&ms->bits[j >> 5], 1u << (j & 31));
            }
            __syncwarp();
            const int c = lane < nw ? __popc(ms->bits[lane]) : 0;
            int incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o)
                    incl += y;
            }
            if (lane < nw)
                ms->wpre[lane] = incl - c;
            const int U = __shfl_sync(0xffffffffu, incl, 31);
            __syncwarp();
            // each slot's expert at its rank u among the activated experts (an
            // expert two tokens share is written twice, with the same value),
            // its token in u's mask; then the token's slot k among u's tokens
            // (ascending) with its Eq. 2 weight
            for (int i = lane; i < n; i += 32) {
                const int j = ms->sj[i];
                if (j != MOE_EMPTY_SLOT) {
                    const int u = ms->wpre[j >> 5] + __popc(ms->bits[j >> 5] & ((1u << (j & 31)) - 1u));
                    ms->ue[u] = j;
                    atomicOr(&ms->tmask[u], 1u << (i / k1));
                }
            }
            __syncwarp();
            for (int i = lane; i < n; i += 32) {
                const int j = ms->sj[i];
                if (j != MOE_EMPTY_SLOT) {
                    const int u = ms->wpre[j >> 5] + __popc(ms->bits[j >> 5] & ((1u << (j & 31)) - 1u));
                    const int t = i / k1;
                    const int k = __popc(ms->tmask[u] & ((1u << t) - 1u));
                    ms->utok[u][k] = (uint8_t)t;
                    ms->uw[u][k] = ms->sw[i];
                }
            }
            __syncwarp();
            if (lane == 0) {
                ms->U = U;
                ms->call = call;
                mt_segments(ms, U, I, G, b, status);
            }
        }
    }
    __syncthreads();
    const int nseg = ms->nseg;
    const int nch = L.nch;
    const size_t stage_bytes = L.stage;

    if (warp == kMtC) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol = l2_evict_first_policy();
            DIter it;
            it.init(ms->seg, nseg, nch);
            int slot_r = 0;
            uint32_t ph = 0;
            int issued = 0;
            while (it.valid()) {
                if (*(volatile int *)&ms->abort)
                    break;
                if (!mbar_wait_live(&empty[slot_r], ph ^ 1u, &ms->abort, status)) {
                    ms->abort = 1;
                    break;
                }
                const int n = it.count();
                const int e = ms->ue[ms->seg[it.s].u];
                const size_t row0 = (size_t)e * I + it.c;
                const uint32_t bytes = (uint32_t)n * d * 2;
                uint8_t *dst = ring + (size_t)slot_r * stage_bytes;
                mbar_arrive_expect_tx(&full[slot_r], 3 * bytes);
                bulk_g2s(dst, a.wg + row0 * d, bytes, &full[slot_r], pol);
                bulk_g2s(dst + bytes, a.wu + row0 * d, bytes, &full[slot_r], pol);
                bulk_g2s(dst + 2 * bytes, a.wdt + row0 * d, bytes, &full[slot_r], pol);
                ++issued;
                it.next();
                if (++slot_r == NS) {
                    slot_r = 0;
                    ph ^= 1u;
                }
            }
            ms->issued = issued;
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ consumers
        // this warp's output rows: vectors v = warp*32 + lane + kMtC*32*j, j < RVM;
        // partials as float32 pairs, per token slot k of the current expert
        // (its k-th token), added into the accumulator when the expert changes
        uint64_t yq[TM][RVM][4];
#pragma unroll
        for (int k = 0; k < TM; ++k)
#pragma unroll
            for (int j = 0; j < RVM; ++j)
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    yq[k][j][q] = 0;
        int cur_u = -1, cur_m = 0;
        auto flush = [&]() {
#pragma unroll
            for (int k = 0; k < TM; ++k) {
                if (k < cur_m) {
                    const int t = ms->utok[cur_u][k];
#pragma unroll
                    for (int j = 0; j < RVM; ++j) {
                        const int v = warp * 32 + lane + kMtC * 32 * j;
                        if (v < nvec) {
                            float *dst = a.yacc + (size_t)t * d + (size_t)v * 8;
                            red_add_v4(dst, pair_lo(yq[k][j][0]), pair_hi(yq[k][j][0]),
                                       pair_lo(yq[k][j][1]), pair_hi(yq[k][j][1]));
                            red_add_v4(dst + 4, pair_lo(yq[k][j][2]), pair_hi(yq[k][j][2]),
                                       pair_lo(yq[k][j][3]), pair_hi(yq[k][j][3]));
                        }
                    }
                }
#pragma unroll
                for (int j = 0; j < RVM; ++j)
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        yq[k][j][q] = 0;  // every slot: those past cur_m held only w*0
            }
        };

        DIter it;
        it.init(ms->seg, nseg, nch);
        int sidx = 0, slot = 0;
        uint32_t par = 0;  // parity of the slot's current use
        while (it.valid()) {
            // stage sidx: slot sidx % NS, parity of its use sidx / NS.  Every
            // consumer warp takes every stage in order and hands the slot back
            // after it, so the producer cannot refill a slot a warp has not
            // consumed, and one parity per use suffices.
            const int n = it.count();
            const int u = ms->seg[it.s].u;
            if (u != cur_u) {
                if (cur_u >= 0)
                    flush();
                cur_u = u;
                cur_m = __popc(ms->tmask[u]);
            }
            const int m = cur_m;
            const int hb = sidx & 1;
            bool ok = !*(volatile int *)&ms->abort;
            if (ok)
                ok = mbar_wait_live(&full[slot], par, &ms->abort, status);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok && lane == 0)
                ms->abort = 1;
            const uint8_t *stg = ring + (size_t)slot * stage_bytes;
            const size_t rb = (size_t)n * d * 2;  // bytes of one of the three row blocks
            // (1) w*h: a job per (channel c, chunk of the expert's m tokens),
            // job j = chunk * n + c on warp j % kMtC; a chunk holds one token,
            // or two (a gate/up vector read once for both) when the n*m pairs
            // outnumber the warps; J = n * chunks <= kMtMaxCh * 4 jobs
            const int tpc = n * m > kMtC && m > 1 ? 2 : 1;
            const int nq = tpc == 1 ? m : (m + 1) >> 1;
            for (int j = warp; ok && j < n * nq; j += kMtC) {
                const int ch = div_small(j, n);
                const int c = j - ch * n;
                const int k0 = ch * tpc;
                const bool two = tpc == 2 && k0 + 1 < m;
                const int t0 = ms->utok[u][k0];
                const int t1 = two ? ms->utok[u][k0 + 1] : t0;
                const uint4 *grow = reinterpret_cast<const uint4 *>(stg + (size_t)c * d * 2);
                const uint4 *urow = reinterpret_cast<const uint4 *>(stg + rb + (size_t)c * d * 2);
                const ulonglong2 *x0 = reinterpret_cast<const ulonglong2 *>(xs + (size_t)t0 * d);
                const ulonglong2 *x1 = reinterpret_cast<const ulonglong2 *>(xs + (size_t)t1 * d);
                float h[2];
                if (two)
                    mt_channel<2>(grow, urow, x0, x1, nvec, lane, h);
                else
                    mt_channel<1>(grow, urow, x0, nullptr, nvec, lane, h);
                if (lane == 0) {
                    ms->hs[hb][c][k0] = h[0] * ms->uw[u][k0];
                    if (two)
                        ms->hs[hb][c][k0 + 1] = h[1] * ms->uw[u][k0 + 1];
                }
            }
            mt_sync();  // the stage's w*h are in shared memory
            // (2) y partials += w*h * down row (mt_down), for this warp's rows
            // and the expert's m token slots.  hs alternates by stage parity: a warp
            // writes the buffer again two stages later, past the next stage's
            // barrier, which every warp reaches only after this read.
            if (ok) {
                const uint8_t *drows = stg + 2 * rb;
                constexpr int M2 = TM < 2 ? TM : 2, M4 = TM < 4 ? TM : 4;
                if (m <= 1)
                    mt_down<1, TM, RVM>(yq, ms->hs[hb], drows, n, m, d, nvec, warp, lane);
                else if (m <= M2)
                    mt_down<M2, TM, RVM>(yq, ms->hs[hb], drows, n, m, d, nvec, warp, lane);
                else if (m <= M4)
                    mt_down<M4, TM, RVM>(yq, ms->hs[hb], drows, n, m, d, nvec, warp, lane);
                else
                    mt_down<TM, TM, RVM>(yq, ms->hs[hb], drows, n, m, d, nvec, warp, lane);
            }
            __syncwarp();
            if (ok && lane == 0)
                mbar_arrive(&empty[slot]);
            ++sidx;
            if (++slot == NS) {
                slot = 0;
                par ^= 1u;
            }
            it.next();
        }
        // the last expert's partials (CTAs that finish early add theirs while
        // the others still stream)
        if (cur_u >= 0)
            flush();
    }

    __syncthreads();
    if (tid == 0 && ms->abort) {
        // wait (bounded) for the copies still in flight into this CTA's ring
        const int issued = ms->issued;
        for (int s = 0; s < NS && s < issued; ++s) {
            const int last = issued - 1 - ((issued - 1 - s) % NS);
            const uint32_t parity = (uint32_t)((last / NS) & 1);
            mbar_wait(&full[s], parity, status);
        }
    }
    if (warp == kMtC)
        return;

    // ------------------------------------------------------------ y (last CTA to check in)
    if (tid == 0) {
        // release: this CTA's reductions before its ticket; acquire: the
        // reductions of every CTA that took a ticket before, for the last one
        unsigned prev;
        asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
                     : "=r"(prev)
                     : "l"(&a.hdr->decode_arrive)
                     : "memory");
        ms->last = prev == (unsigned)G - 1;
    }
    mt_sync();
    if (ms->last) {
        const int tot = T * d;
        for (int i = tid * 4; i < tot; i += kMtC * 32 * 4) {
            const float4 v = __ldcg(reinterpret_cast<const float4 *>(a.yacc + i));
            if (a.y_dtype == MOE_DTYPE_BF16) {
                const uint32_t lo = f32_to_bf16_rn(v.x) | ((uint32_t)f32_to_bf16_rn(v.y) << 16);
                const uint32_t hi = f32_to_bf16_rn(v.z) | ((uint32_t)f32_to_bf16_rn(v.w) << 16);
                *reinterpret_cast<uint2 *>(reinterpret_cast<uint16_t *>(a.y) + i) =
                    make_uint2(lo, hi);
            } else {
                *reinterpret_cast<float4 *>(reinterpret_cast<float *>(a.y) + i) = v;
            }
            __stcg(reinterpret_cast<float4 *>(a.yacc + i), make_float4(0.f, 0.f, 0.f, 0.f));
        }
        if (tid == 0) {
            a.hdr->decode_arrive = 0u;
            // every CTA read the call number before it took its ticket
            a.hdr->decode_seq = ms->call;
        }
    }

    if (b == 0 && warp == 0) {
        // the routing outputs
        for (int i = lane; i < T * k1; i += 32) {
            const int j = ms->sj[i];
            const float wv = ms->sw[i];
            a.topk_idx[i] = j;
            a.topk_w[i] = wv;
            if (a.idx_copy)
                a.idx_copy[i] = j;
            if (a.w_copy)
                a.w_copy[i] = wv;
        }
        if (a.count && lane < T)
            a.count[lane] = ms->ktok[lane];
    }
}

// Router rows per router CTA of the few-token kernel: as few as cover E.
inline int mt_router_rows(int E, int G) { return (E + G - 1) / G; }

// Partials of the few-token kernel: (TM, RVM) for T tokens of width d, or
// TM = 0 when they do not fit.
inline void mt_shape(int T, int d, int &TM, int &RVM)
{
    const int nvec = d >> 3;
    TM = T <= 2 ? 2 : (T <= 4 ? 4 : 8);
    RVM = nvec <= kMtC * 32 ? 1 : (nvec <= 2 * kMtC * 32 ? 2 : 0);
    if (T < 2 || T > kMtMaxT || RVM == 0 || TM * RVM > 8)
        TM = 0;
}

// The few-token path serves 2 <= T <= 8 tokens (T*k1 <= 64) with the down
// matrix channel-major: the per-token row partials fit the registers (at most
// 8 row vectors of 8 floats per lane), three channels' rows fit a ring slot,
// at least two ring slots and the router rows fit beside the x rows, and no
// CTA's channel range crosses more than kDMaxSeg experts.
inline bool mt_fits(int T, int d, int E, int I, int k1, int G)
{
    int TM, RVM;
    mt_shape(T, d, TM, RVM);
    if (TM == 0 || T * k1 > kMtMaxSlots || k1 > kDMaxK1 || E > kMaxExperts)
        return false;
    const MtLayout L = mt_layout(T, d);
    if (L.nslots < 2)
        return false;
    const int rows = mt_router_rows(E, G);
    if ((size_t)rows * d * 2 > (size_t)L.nslots * L.stage)
        return false;
    const int umax = T * k1 < E ? T * k1 : E;
    const long chmax = ((long)umax * I + G - 1) / G;
    const long nseg = (chmax + I - 1) / I + 1;
    return nseg <= kDMaxSeg;
}

}  // namespace moe
