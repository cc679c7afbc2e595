// decode.cuh -- the one-token layer kernel: router logits, routing, the
// routed experts' SwiGLU FFN and the weighted combine in one launch, each
// weight byte read once from HBM.
//
// Structure of an expert ("Channel Selection for Mixture-of-Experts Decoding
// Needs No Calibration Data", section 2 "Background"): a gated MLP whose
// channel c owns gate row c, up row c and down column c.  With the down
// matrix stored channel-major (down column c contiguous, [E x I x d], see
// k_pack_w_down), a channel is three contiguous rows, and a CTA that owns
// channels [c0, c1) of an expert finishes that expert's share of the output
// alone:
//     y[:] += w_e * sum_{c in [c0, c1)} h_c(x) * down_row_c
// (Eq. 2 weight w_e, "Paper of the Week #3", section "The Receipt").
//
// Design (one CTA per SM, cooperative launch; 12 consumer warps + 1 producer
// warp):
//  * router: CTA b dots x with router rows R*b .. R*b+R-1 (R rows per
//    router CTA, chosen on the host: fewer router CTAs each with more rows
//    make fewer arrivals to wait for), fetched into shared memory before the
//    programmatic-launch wait -- weights no earlier kernel writes -- with an
//    L2 evict-last policy; it writes the logits and counts
//    them on a release counter in the workspace header (spread over lines);
//    warp 0 of every CTA waits for all E, reads them back, forms the float32
//    softmax, takes the top min(k2, E) in rank order by repeated warp arg-max
//    and applies Eq. 2 -- the fixed float32 sequence the oracle follows;
//  * the U activated experts are laid end to end as U*I channels and CTA b
//    owns a contiguous range of floor(U*I/G) or one more channels;
//  * the producer streams stages of n whole channels (gate rows, up rows,
//    down rows: three contiguous bulk copies) through a ring of kDStages
//    shared-memory slots; each slot is served by kWPS consumer warps;
//  * per stage, warp i of the slot's group forms h for channel i (times the
//    token's Eq. 2 weight), the group meets at a named barrier, and each warp
//    adds h * down_row into register partials for its fixed third of the
//    output rows;
//  * combine: the four groups' partials are summed in shared memory and added
//    into a float32 accumulator with 16-byte vector reductions (CTAs that
//    finish early add theirs while others still stream); one fence and one
//    ticket per CTA; the last CTA converts the accumulator to y and clears it
//    for the next call.  Partial sums reach the accumulator in a
//    timing-dependent order, so y can differ between runs in the last bits.
// Call numbers (decode_seq in the header) pick one of four counters per call;
// each call clears the counter two calls ahead, so no counter is reset on the
// critical path.
#pragma once
#include "common.cuh"
#include "route.cuh"
#include "stream.cuh"

namespace moe {

constexpr int kDStageBytes = 36 * 1024;   // one ring slot of the decode kernel
constexpr int kDSlots = 6;                // ring slots (stages in flight)
constexpr int kDStages = 4;               // consumer groups (kWPS warps each)
constexpr int kDMaxRowVec = 6;            // 16-byte row vectors per lane (d <= 4608)
constexpr int kDMaxK1 = 32;
constexpr int kDMaxSeg = 8;               // expert segments of one CTA's channels
constexpr int kGroupBar0 = 2;             // named barriers 2..5: one per slot group

static_assert(kSC == kDStages * kWPS, "decode kernel: the consumer warps split into groups");

struct DecodeArgs {
    const uint16_t *x;    // [1 x d]
    const uint16_t *wg;   // [E x I x d]
    const uint16_t *wu;   // [E x I x d]
    const uint16_t *wdt;  // [E x I x d]: down matrix, channel-major
    int d, E, I, k1, k2;
    // router: wr [E x d] (+ bias [E], nullable) -- the kernel forms the
    // logits itself, writes them to `logits` (and logits_out, nullable); with
    // wr null it routes from the float32 logits already in `logits`
    const uint16_t *wr;
    const float *bias;
    float *logits_out;
    const float *logits;  // [E] float32
    int32_t *topk_idx;
    float *topk_w;
    int32_t *idx_copy;
    float *w_copy;
    int32_t *offsets;
    int32_t *sorted_slot;
    int32_t *slot_pos;
    int32_t *uniq_count;
    int32_t *uniq_list;
    float *yacc;   // [d] float32 accumulator, zero on entry; the last CTA clears it again
    void *y;       // [d] output (y_dtype)
    int y_dtype;
    VarK vk;       // variable k: cascade or skip (kind 0 with the fixed-k kernel)
    int32_t *count;  // nullable: kt
    int rrows;       // router rows per router CTA: decode_router_rows(d, E, G)
    WsHeader *hdr;
};

// One expert's share of this CTA's channel range.
struct DSeg {
    int u;  // index into the activated-expert list
    int a;  // first channel (within the expert)
    int b;  // one past the last channel
};

constexpr int kDMaxRouterRows = 8;          // router rows one CTA dots with x
constexpr int kDRouterBytes = 128 * 1024;   // ring bytes the router rows may use

struct __align__(16) DecodeSmem {
    float hs[kDStages][2][kWPS];  // w*h of the stage's channels, per group and stage parity
    int ue[kDMaxK1];           // the activated experts, ascending
    float uw[kDMaxK1];         // their Eq. 2 weights
    int sj[kDMaxK1];           // the route by slot: expert (or MOE_EMPTY_SLOT),
    float sw[kDMaxK1];         //   weight,
    int sp[kDMaxK1];           //   position among the taken experts (-1: empty)
    DSeg seg[kDMaxSeg];
    int nseg;
    int kt;                    // slots taken
    int abort;
    int issued;
    int last;                  // this CTA checked in last: it writes y
    unsigned call;             // this call's number (decode_seq + 1)
};

struct DIter {
    int s, c, nseg, nch;
    const DSeg *seg;
    __device__ void init(const DSeg *sg, int ns, int n)
    {
        seg = sg;
        nseg = ns;
        nch = n;
        s = 0;
        c = ns > 0 ? sg[0].a : 0;
    }
    __device__ bool valid() const { return s < nseg; }
    __device__ int count() const { return min(nch, seg[s].b - c); }
    __device__ void next()
    {
        c += count();
        if (c >= seg[s].b && ++s < nseg)
            c = seg[s].a;
    }
};

// channels per stage: kWPS when three channels' rows fit a stage, else fewer
__host__ __device__ inline int decode_channels_per_stage(int d)
{
    const int n = kDStageBytes / (6 * d);
    return n >= kWPS ? kWPS : (n < 1 ? 1 : n);
}

// This CTA's channel segments: the U activated experts laid end to end as
// U*I channels, CTA b taking a balanced contiguous range.
__device__ void decode_segments(DecodeSmem *ds, int U, int I, int G, int b, int *status)
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
        ds->seg[ns++] = sg;
        c = (unsigned)u * I + sg.b;
    }
    if (c < c_hi) {  // more segments than kDMaxSeg: the host rules this out
        set_status(status, MOE_ERR_DEVICE_CHECK);
        ns = 0;
    }
    ds->nseg = ns;
}

// Arrival i of a spread count (release: this thread's earlier accesses, and
// those it observed through a CTA barrier, come first).
MOE_DEVINL void spread_arrive(SpreadCount *sc, unsigned i)
{
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(&sc->c[i % kSpread][0])
                 : "memory");
}

// One warp waits (bounded) until a spread count has seen n arrivals numbered
// 0..n-1: lane l reads counter l % kSpread, whose share is the arrivals i
// with i % kSpread == l % kSpread; then every lane acquires.  Gives up at the
// wait limit: records MOE_ERR_TIMEOUT and returns false (on every lane).
MOE_DEVINL bool warp_wait_spread(const SpreadCount *sc, unsigned n, int lane, int *status)
{
    const unsigned q = (unsigned)lane % kSpread;
    const unsigned want = n > q ? (n - q + kSpread - 1) / kSpread : 0u;
    const unsigned *p = &sc->c[q][0];
    bool ok = true;
    if (!__all_sync(0xffffffffu, ld_relaxed_u32(p) >= want)) {
        const uint64_t t0 = global_ns();
        const uint64_t lim = wait_limit_ns();
        while (!__all_sync(0xffffffffu, ld_relaxed_u32(p) >= want)) {
            // the whole warp gives up together (lanes read the clock apart)
            if (__any_sync(0xffffffffu, global_ns() - t0 > lim)) {
                if (lane == 0)
                    set_status(status, MOE_ERR_TIMEOUT);
                ok = false;
                break;
            }
            __nanosleep(32);
        }
    }
    fence_acquire_gpu();
    return ok;
}

// Warp 0 routes the token: its E logits into registers -- once the router
// exchange counts all E published (bounded wait; every lane acquires, so each
// lane's reads follow the logits), or directly when the logits were given --
// then warp_route_vals: the float32 softmax, the top min(k2, E) by repeated
// warp arg-max in rank order, Eq. 2 (lane s < k1: slot s).
template <int R>
__device__ __forceinline__ void decode_route(const DecodeArgs &a, bool fused, unsigned slot,
                                             int lane, DecodeSmem *ds, int *status, VarK vk,
                                             int &my_j, float &my_w, int &kt)
{
    const int E = a.E;
    float p[R];
    bool ok = true;
    if (fused)
        ok = warp_wait_spread(&a.hdr->xcnt[slot], (unsigned)E, lane, status);
    if (!ok && lane == 0)
        ds->abort = 1;
#pragma unroll
    for (int i = 0; i < R; ++i) {
        const int j = lane + 32 * i;
        p[i] = j < E && ok ? __ldcg(&a.logits[j]) : 0.0f;
    }
    warp_route_vals<R>(p, E, a.k1, a.k2, lane, my_j, my_w, vk, &kt);
}

// One channel of the single-token register path with paired float32 FMAs:
// g = gate_row . x, u = up_row . x with x held as float32 pairs, four partial
// chains per dot product (pairs of 16-byte vectors alternate), then SiLU(g)*u.
template <int VPL>
__device__ __forceinline__ float pair_channel(const uint4 *grow, const uint4 *urow,
                                              const uint64_t (&xp)[VPL][4], int lane)
{
    uint64_t g0 = 0, g1 = 0, u0 = 0, u1 = 0;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const uint4 wg = grow[lane + 32 * i];
        const uint4 wu = urow[lane + 32 * i];
        uint64_t &g = (i & 1) ? g1 : g0;
        uint64_t &u = (i & 1) ? u1 : u0;
        g = ffma2(bf16x2_pair(wg.x), xp[i][0], g);
        u = ffma2(bf16x2_pair(wu.x), xp[i][0], u);
        g = ffma2(bf16x2_pair(wg.y), xp[i][1], g);
        u = ffma2(bf16x2_pair(wu.y), xp[i][1], u);
        g = ffma2(bf16x2_pair(wg.z), xp[i][2], g);
        u = ffma2(bf16x2_pair(wu.z), xp[i][2], u);
        g = ffma2(bf16x2_pair(wg.w), xp[i][3], g);
        u = ffma2(bf16x2_pair(wu.w), xp[i][3], u);
    }
    float g = (pair_lo(g0) + pair_hi(g0)) + (pair_lo(g1) + pair_hi(g1));
    float u = (pair_lo(u0) + pair_hi(u0)) + (pair_lo(u1) + pair_hi(u1));
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        g += __shfl_xor_sync(0xffffffffu, g, o);
        u += __shfl_xor_sync(0xffffffffu, u, o);
    }
    return silu_mul(g, u);
}

// VPL: d = 256*VPL for the single-token register path (x in registers when
// VPL <= kXRegMax), 0 for the general token loop.  CASCADE: the variable-k
// route (a.vk: cascade or skip).
template <int VPL, bool CASCADE>
__global__ void __launch_bounds__(kSThreads, 1) k_decode(DecodeArgs a)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *ring = smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kDSlots * kDStageBytes);
    uint64_t *empty = full + kDSlots;
    uint64_t *rbar = empty + kDSlots;  // the router rows' bulk copies (2 slots: alignment)
    DecodeSmem *ds = reinterpret_cast<DecodeSmem *>(rbar + 2);
    uint8_t *area = reinterpret_cast<uint8_t *>(ds + 1);  // the token's x row, d bf16

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x, b = blockIdx.x;
    int *status = &a.hdr->status;
    const int d = a.d, E = a.E, I = a.I, k1 = a.k1;
    const bool fused = a.wr != nullptr;
    const int R = max(a.rrows, (E + G - 1) / G);  // the grid covers all E rows
    const int nr = fused && b * R < E ? min(R, E - b * R) : 0;  // router rows e = R*b + i
    const int nvec = d >> 3;                                   // 16-byte vectors per row

    if (tid == 0) {
        for (int s = 0; s < kDSlots; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kWPS);
        }
        mbar_init(rbar, 1);
        ds->abort = 0;
        ds->issued = 0;
        fence_mbar_init();
        // this CTA's channel segments depend only on k1, I and the grid (with
        // the cascade, on the routed count: computed after routing)
        if constexpr (!CASCADE)
            decode_segments(ds, k1, I, G, b, status);
    }
    __syncthreads();
    // this CTA's router rows: weights no earlier kernel writes, so they are
    // fetched before the dependency wait and overlap the previous kernel
    if (warp == kSC && lane == 0 && nr > 0) {
        const uint64_t keep = l2_evict_last_policy();  // the router, read by every call
        mbar_arrive_expect_tx(rbar, (uint32_t)(nr * d * 2));
        for (int i = 0; i < nr; ++i)
            bulk_g2s(ring + (size_t)i * d * 2, a.wr + (size_t)(b * R + i) * d, (uint32_t)(d * 2),
                     rbar, keep);
    }

    pdl_wait();
    pdl_trigger();

    if (warp < kSC) {
        const unsigned call = ld_relaxed_u32(&a.hdr->decode_seq) + 1u;
        const unsigned slot = call & 3u;
        if (b == 0 && tid < kSpread)  // the count of the call two ahead starts at zero
            a.hdr->xcnt[(call + 2u) & 3u].c[tid][0] = 0u;
        // ------------------------------------------------------------ router logits
        // warp i < nr: router row R*b + i in router_step's order (the order of
        // k_logits), its x vectors all in flight at once; warp 0 also keeps
        // the token's x row in shared memory for the FFN
        const uint4 *xg = reinterpret_cast<const uint4 *>(a.x);
        const bool xreg = nvec <= 32 * kLogitsMaxVec;
        uint4 xq[kLogitsMaxVec];
        if ((warp == 0 || warp < nr) && xreg) {
#pragma unroll
            for (int i = 0; i < kLogitsMaxVec; ++i) {
                const int v = lane + 32 * i;
                xq[i] = v < nvec ? xg[v] : make_uint4(0, 0, 0, 0);
            }
        }
        if (warp == 0) {
            if (xreg) {
#pragma unroll
                for (int i = 0; i < kLogitsMaxVec; ++i)
                    if (lane + 32 * i < nvec)
                        reinterpret_cast<uint4 *>(area)[lane + 32 * i] = xq[i];
            } else {
                for (int v = lane; v < nvec; v += 32)
                    reinterpret_cast<uint4 *>(area)[v] = xg[v];
            }
        }
        if (warp < nr) {
            if (!mbar_wait(rbar, 0, status))
                ds->abort = 1;
            const uint4 *row = reinterpret_cast<const uint4 *>(ring + (size_t)warp * d * 2);
            float a0 = 0.0f, a1 = 0.0f;
            if (xreg) {
#pragma unroll
                for (int i = 0; i < kLogitsMaxVec; ++i)
                    if (lane + 32 * i < nvec)
                        router_step(a0, a1, i, row[lane + 32 * i], xq[i]);
            } else {
                int i = 0;
                for (int v = lane; v < nvec; v += 32, ++i)
                    router_step(a0, a1, i, row[v], xg[v]);
            }
            float z = warp_sum(a0 + a1);
            const int e = b * R + warp;
            if (a.bias)
                z = z + a.bias[e];
            if (lane == 0) {
                const_cast<float *>(a.logits)[e] = z;
                if (a.logits_out)
                    a.logits_out[e] = z;
                spread_arrive(&a.hdr->xcnt[slot], (unsigned)e);  // the logit before the count
            }
        }

        // ------------------------------------------------------------ routing (warp 0)
        if (warp == 0) {
            int j, kt;
            float wv;
            const VarK vk = CASCADE ? a.vk : VarK();
            if (E <= 128)
                decode_route<4>(a, fused, slot, lane, ds, status, vk, j, wv, kt);
            else if (E <= 256)
                decode_route<8>(a, fused, slot, lane, ds, status, vk, j, wv, kt);
            else if (E <= 512)
                decode_route<16>(a, fused, slot, lane, ds, status, vk, j, wv, kt);
            else
                decode_route<32>(a, fused, slot, lane, ds, status, vk, j, wv, kt);
            if (MOE_CHECKS) {  // the route: experts in range, kt slots taken
                const bool bad = (lane < k1 && j != MOE_EMPTY_SLOT && (j < 0 || j >= E)) ||
                                 kt < 0 || kt > k1;
                if (__any_sync(0xffffffffu, bad)) {
                    if (lane == 0) {
                        set_status(status, MOE_ERR_DEVICE_CHECK);
                        ds->abort = 1;
                    }
                    j = lane < k1 ? MOE_EMPTY_SLOT : 0;
                    kt = 0;
                }
            }
            int p = 0;  // position of this lane's expert among the kt taken, ascending
            for (int q = 0; q < k1; ++q)
                p += __shfl_sync(0xffffffffu, j, q) < j;  // empty slots never count
            if (lane < k1) {
                if (j != MOE_EMPTY_SLOT) {  // taken (kt of the k1 slots)
                    ds->ue[p] = j;
                    ds->uw[p] = wv;
                }
                // kept for the routing outputs, which CTA 0 writes at the end
                // (off the path the layer's time waits on)
                ds->sj[lane] = j;
                ds->sw[lane] = wv;
                ds->sp[lane] = j != MOE_EMPTY_SLOT ? p : -1;
            }
            if (lane == 0) {
                ds->kt = kt;
                ds->call = call;
            }
            __syncwarp();
            if constexpr (CASCADE) {
                if (lane == 0)
                    decode_segments(ds, kt, I, G, b, status);
            }
        }
    }
    __syncthreads();
    const int nseg = ds->nseg;
    const int nch = decode_channels_per_stage(d);

    if (warp == kSC) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol = l2_evict_first_policy();
            DIter it;
            it.init(ds->seg, nseg, nch);
            int slot_r = 0;
            uint32_t ph = 0;
            int issued = 0;
            while (it.valid()) {
                if (*(volatile int *)&ds->abort)
                    break;
                if (!mbar_wait_live(&empty[slot_r], ph ^ 1u, &ds->abort, status)) {
                    ds->abort = 1;
                    break;
                }
                const int n = it.count();
                const int e = ds->ue[ds->seg[it.s].u];
                const size_t row0 = (size_t)e * I + it.c;
                const uint32_t bytes = (uint32_t)n * d * 2;
                uint8_t *dst = ring + (size_t)slot_r * kDStageBytes;
                mbar_arrive_expect_tx(&full[slot_r], 3 * bytes);
                bulk_g2s(dst, a.wg + row0 * d, bytes, &full[slot_r], pol);
                bulk_g2s(dst + bytes, a.wu + row0 * d, bytes, &full[slot_r], pol);
                bulk_g2s(dst + 2 * bytes, a.wdt + row0 * d, bytes, &full[slot_r], pol);
                ++issued;
                it.next();
                if (++slot_r == kDSlots) {
                    slot_r = 0;
                    ph ^= 1u;
                }
            }
            ds->issued = issued;
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ consumers
        const int group = warp / kWPS;
        const int gl = warp % kWPS;
        // this warp's output rows: vectors v = gl*32 + lane + kWPS*32*j, j < RV
        constexpr int RV = VPL > 0 ? (VPL * 32 + kWPS * 32 - 1) / (kWPS * 32) : kDMaxRowVec;
        static_assert(RV <= kDMaxRowVec, "row partials");
        float yp[RV][8];
#pragma unroll
        for (int j = 0; j < RV; ++j)
#pragma unroll
            for (int k = 0; k < 8; ++k)
                yp[j][k] = 0.0f;

        // x: float32 pairs in registers (register path), else read from shared memory
        constexpr bool kPairs = VPL > 0 && VPL <= kXRegMax;
        uint64_t xp[kPairs ? VPL : 1][4];
        uint64_t yq[kPairs ? RV : 1][4];  // the row partials as pairs (register path)
        const uint4 *xs = reinterpret_cast<const uint4 *>(area);
        if constexpr (kPairs) {
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                const uint4 v = xs[lane + 32 * i];
                xp[i][0] = bf16x2_pair(v.x);
                xp[i][1] = bf16x2_pair(v.y);
                xp[i][2] = bf16x2_pair(v.z);
                xp[i][3] = bf16x2_pair(v.w);
            }
#pragma unroll
            for (int j = 0; j < RV; ++j)
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    yq[j][q] = 0;
        }
        uint4 xv[1];  // unused by the pair path

        DIter it;
        it.init(ds->seg, nseg, nch);
        int sidx = 0;
        while (it.valid()) {
            const int n = it.count();
            if (sidx % kDStages == group) {
                // stage sidx: group sidx % kDStages, slot sidx % kDSlots, the
                // slot's use number rnd.  A slot's stages alternate between two
                // groups, so a group comes back to a slot two phases of its
                // full barrier later, which parity alone cannot tell from the
                // phase before: it first waits until the other group has
                // consumed the slot's previous stage (that stage's full phase
                // done), then on this stage's full phase.  A warp hands a slot
                // back only after a successful wait, so the producer refills a
                // slot only once its previous copies have landed.
                const int slot = sidx % kDSlots;
                const int rnd = sidx / kDSlots;
                const int hb = (sidx / kDStages) & 1;  // the group's h buffer
                bool ok = !*(volatile int *)&ds->abort;
                if (ok && rnd > 0)
                    ok = mbar_wait_live(&empty[slot], (uint32_t)((rnd - 1) & 1), &ds->abort,
                                        status);
                if (ok)
                    ok = mbar_wait_live(&full[slot], (uint32_t)(rnd & 1), &ds->abort, status);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok && lane == 0)
                    ds->abort = 1;
                const uint8_t *stg = ring + (size_t)slot * kDStageBytes;
                const size_t rb = (size_t)n * d * 2;  // bytes of one of the three row blocks
                const float wgt = ds->uw[ds->seg[it.s].u];
                // (1) w * h for channel gl of the stage
                if (ok && gl < n) {
                    const uint4 *grow = reinterpret_cast<const uint4 *>(stg + (size_t)gl * d * 2);
                    const uint4 *urow = reinterpret_cast<const uint4 *>(stg + rb + (size_t)gl * d * 2);
                    float hval;
                    if constexpr (kPairs) {
                        hval = pair_channel<VPL>(grow, urow, xp, lane);
                    } else if constexpr (VPL > 0) {
                        hval = fast_channel<VPL>(grow, urow, xv, xs, lane);
                    } else {
                        float r0[kTokChunk], r1[kTokChunk];
                        XRows xr;
#pragma unroll
                        for (int t = 0; t < kTokChunk; ++t)
                            xr.r[t] = xs;
                        unit_gate_up<1>(grow, urow, xr, nvec, lane, r0, r1);
                        hval = silu_mul(r0[0], r1[0]);
                    }
                    if (lane == 0)
                        ds->hs[group][hb][gl] = hval * wgt;
                }
                named_bar_sync(kGroupBar0 + group, kWPS * 32);  // the group's h are in shared memory
                // (2) y partial += w*h * down row, for this warp's rows
                if (ok && kPairs) {
                    const uint8_t *drows = stg + 2 * rb;
                    for (int i = 0; i < n; ++i) {
                        const float hv = ds->hs[group][hb][i];
                        const uint64_t h2 = f32_pair(hv, hv);
                        const uint4 *drow = reinterpret_cast<const uint4 *>(drows + (size_t)i * d * 2);
#pragma unroll
                        for (int j = 0; j < (kPairs ? RV : 1); ++j) {
                            const int v = gl * 32 + lane + kWPS * 32 * j;
                            if (v < nvec) {
                                const uint4 w = drow[v];
                                yq[j][0] = ffma2(bf16x2_pair(w.x), h2, yq[j][0]);
                                yq[j][1] = ffma2(bf16x2_pair(w.y), h2, yq[j][1]);
                                yq[j][2] = ffma2(bf16x2_pair(w.z), h2, yq[j][2]);
                                yq[j][3] = ffma2(bf16x2_pair(w.w), h2, yq[j][3]);
                            }
                        }
                    }
                } else if (ok) {
                    const uint8_t *drows = stg + 2 * rb;
                    for (int i = 0; i < n; ++i) {
                        const float hv = ds->hs[group][hb][i];
                        const uint4 *drow = reinterpret_cast<const uint4 *>(drows + (size_t)i * d * 2);
#pragma unroll
                        for (int j = 0; j < RV; ++j) {
                            const int v = gl * 32 + lane + kWPS * 32 * j;
                            if (v < nvec) {
                                float f[8];
                                bf16x8(drow[v], f);
#pragma unroll
                                for (int k = 0; k < 8; ++k)
                                    yp[j][k] = fmaf(f[k], hv, yp[j][k]);
                            }
                        }
                    }
                }
                // hand the slot back; hs[group] alternates by stage parity, and a
                // warp reaches the group's stage after next only past the next
                // stage's group barrier, which every warp of the group passes
                // after it has read this stage's values
                __syncwarp();
                if (ok && lane == 0)
                    mbar_arrive(&empty[slot]);
            }
            ++sidx;
            it.next();
        }

        if constexpr (kPairs) {
#pragma unroll
            for (int j = 0; j < RV; ++j)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    yp[j][2 * q] = pair_lo(yq[j][q]);
                    yp[j][2 * q + 1] = pair_hi(yq[j][q]);
                }
        }
        // ------------------------------------------------------------ this CTA's partial row
        consumer_sync();  // every warp is past its last stage: the ring is free
        float *red = reinterpret_cast<float *>(ring);  // [kDStages][d]
#pragma unroll
        for (int j = 0; j < RV; ++j) {
            const int v = gl * 32 + lane + kWPS * 32 * j;
            if (v < nvec) {
                float4 *dst = reinterpret_cast<float4 *>(red + (size_t)group * d + v * 8);
                dst[0] = make_float4(yp[j][0], yp[j][1], yp[j][2], yp[j][3]);
                dst[1] = make_float4(yp[j][4], yp[j][5], yp[j][6], yp[j][7]);
            }
        }
        consumer_sync();
        // the four groups' partials summed and added into the accumulator with
        // 16-byte vector reductions; CTAs that finish early add theirs while
        // the others still stream
        if (nseg > 0) {
            for (int r = tid * 4; r < d; r += kSC * 32 * 4) {
                float4 sum = *reinterpret_cast<const float4 *>(red + r);
#pragma unroll
                for (int g = 1; g < kDStages; ++g) {
                    const float4 v = *reinterpret_cast<const float4 *>(red + (size_t)g * d + r);
                    sum.x += v.x;
                    sum.y += v.y;
                    sum.z += v.z;
                    sum.w += v.w;
                }
                red_add_v4(a.yacc + r, sum.x, sum.y, sum.z, sum.w);
            }
        }
    }

    __syncthreads();
    if (tid == 0 && ds->abort) {
        const int issued = ds->issued;
        for (int s = 0; s < kDSlots && s < issued; ++s) {
            const int last = issued - 1 - ((issued - 1 - s) % kDSlots);
            const uint32_t parity = (uint32_t)((last / kDSlots) & 1);
            mbar_wait(&full[s], parity, status);
        }
    }
    if (warp == kSC)
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
        ds->last = prev == (unsigned)G - 1;
    }
    consumer_sync();
    if (ds->last) {
        for (int i = tid * 4; i < d; i += kSC * 32 * 4) {
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
            a.hdr->decode_seq = ds->call;
        }
    }

    if (b == 0 && warp == 0) {
        // the routing outputs and the permutation tables of the one token
        const int kt = ds->kt;
        if (lane < k1) {
            const int j = ds->sj[lane], p = ds->sp[lane];
            const float wv = ds->sw[lane];
            a.topk_idx[lane] = j;
            a.topk_w[lane] = wv;
            if (a.idx_copy)
                a.idx_copy[lane] = j;
            if (a.w_copy)
                a.w_copy[lane] = wv;
            if (p >= 0) {
                a.uniq_list[p] = j;
                a.sorted_slot[p] = lane;
            }
            a.slot_pos[lane] = p;
        }
        if (lane == 0) {
            *a.uniq_count = kt;
            if (a.count)
                *a.count = kt;
        }
        for (int e = lane; e <= E; e += 32) {
            int c = 0;
            for (int q = 0; q < kt; ++q)
                c += ds->ue[q] < e;
            a.offsets[e] = c;
        }
    }
}

inline size_t decode_smem_bytes(int d)
{
    return (size_t)kDSlots * kDStageBytes + (2 * kDSlots + 2) * sizeof(uint64_t) +
           sizeof(DecodeSmem) + (size_t)d * 2;
}

// The single-pass path serves one token per call (T == 1) whose output rows
// fit the register partials, with the down matrix channel-major; each CTA's
// router rows fit the ring.
// Router rows per router CTA: about 32 KB of them (at most kDMaxRouterRows),
// and enough for the grid to cover all E rows.
inline int decode_router_rows(int d, int E, int G)
{
    int r = (32 * 1024) / (2 * d);
    r = r < 1 ? 1 : (r > kDMaxRouterRows ? kDMaxRouterRows : r);
    const int need = (E + G - 1) / G;
    return r > need ? r : need;
}

inline bool decode_fits(int T, int d, int E, int I, int k1, int G)
{
    if (T != 1 || k1 > kDMaxK1 || (d >> 3) > kWPS * 32 * kDMaxRowVec || E > kMaxExperts)
        return false;
    if (decode_smem_bytes(d) > 227 * 1024 || (size_t)kDStages * d * 4 > (size_t)kDSlots * kDStageBytes)
        return false;
    const int rows = decode_router_rows(d, E, G);
    if (rows > kDMaxRouterRows || (size_t)rows * d * 2 > (size_t)kDRouterBytes)
        return false;
    const long chmax = ((long)k1 * I + G - 1) / G;
    const long nseg = (chmax + I - 1) / I + 1;
    return nseg <= kDMaxSeg;
}

// y = y_acc in the output type.  T*d elements, four per thread.
__global__ void __launch_bounds__(256) k_finalize(const float *y_acc, int n, void *y, int y_dtype)
{
    pdl_wait();
    pdl_trigger();
    const int i = (blockIdx.x * 256 + threadIdx.x) * 4;
    if (i >= n)
        return;
    const float4 v = __ldcg(reinterpret_cast<const float4 *>(y_acc + i));
    if (y_dtype == MOE_DTYPE_BF16) {
        const uint32_t lo = f32_to_bf16_rn(v.x) | ((uint32_t)f32_to_bf16_rn(v.y) << 16);
        const uint32_t hi = f32_to_bf16_rn(v.z) | ((uint32_t)f32_to_bf16_rn(v.w) << 16);
        *reinterpret_cast<uint2 *>(reinterpret_cast<uint16_t *>(y) + i) = make_uint2(lo, hi);
    } else {
        *reinterpret_cast<float4 *>(reinterpret_cast<float *>(y) + i) = v;
    }
}

// Channel-major copy of the down matrix: wdt[e][c][r] = wd[e][r][c]
// (wd [E x d x I] -> wdt [E x I x d]), 64 x 64 tiles through shared memory.
__global__ void __launch_bounds__(256) k_pack_w_down(const uint16_t *wd, uint16_t *wdt, int d,
                                                     int I)
{
    __shared__ uint16_t tile[64][65];
    pdl_wait();
    pdl_trigger();
    const int e = blockIdx.z;
    const int r0 = blockIdx.y * 64, c0 = blockIdx.x * 64;
    const uint16_t *src = wd + (size_t)e * d * I;
    uint16_t *dst = wdt + (size_t)e * I * d;
    for (int i = threadIdx.x; i < 64 * 64; i += 256) {
        const int rr = i / 64, cc = i % 64;
        if (r0 + rr < d && c0 + cc < I)
            tile[rr][cc] = src[(size_t)(r0 + rr) * I + c0 + cc];
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 64 * 64; i += 256) {
        const int cc = i / 64, rr = i % 64;
        if (r0 + rr < d && c0 + cc < I)
            dst[(size_t)(c0 + cc) * d + r0 + rr] = tile[rr][cc];
    }
}

}  // namespace moe
