// decode.cuh -- the small-batch layer kernel: one pass over the routed
// experts' weights, each byte read once from HBM, no grid-wide barrier.
//
// Structure of an expert ("Channel Selection for Mixture-of-Experts Decoding
// Needs No Calibration Data", section 2 "Background"): a gated MLP whose
// channel c owns gate row c, up row c and down column c.  With the down
// matrix stored channel-major (down column c contiguous, [E x I x d], see
// k_pack_w_down), a channel is three contiguous rows, and a CTA that owns
// channels [c0, c1) of an expert finishes that expert's share of the output
// alone:
//     y[t, :] += w[t, e] * sum_{c in [c0, c1)} h_c(x_t) * down_row_c
// (Eq. 2 weight w, "Paper of the Week #3", section "The Receipt").
//
// Design (one persistent CTA per SM, 12 consumer warps + 1 producer warp):
//  * one token per call (T == 1): one warp of every CTA routes it from the
//    router's logits in registers (warp_route: the same fixed float32
//    sequence as the router kernels) while the others load x; each CTA's
//    channel ranges are fixed before the kernel waits on the router;
//  * the U activated experts are laid end to end as U*I channels and CTA b
//    owns a contiguous range of floor(U*I/G) or one more channels;
//  * the producer streams stages of n whole channels (gate rows, up rows,
//    down rows: three contiguous bulk copies) through a ring of kStages
//    shared-memory slots; each slot is served by kWPS consumer warps;
//  * per stage, warp i of the slot's group forms h for channel i (times the
//    token's Eq. 2 weight), the group meets at a named barrier, and each warp
//    adds h * down_row into register partials for its fixed third of the
//    output rows;
//  * at the end the four groups' partials are summed in shared memory and
//    added into the float32 accumulator y_acc with 16-byte vector reductions
//    (red.global.add.v4.f32); the last CTA to check in (a counter in the
//    workspace header) converts y_acc to the output y, and the first one
//    writes the routing outputs and permutation tables (every CTA holds the
//    route; writing them out before the stream delayed that CTA, and the
//    layer, by a microsecond or more).
// Partial sums from different CTAs reach y_acc in a timing-dependent order,
// so y can differ between runs in the last bits (stream.cuh holds the
// deterministic two-phase kernel).
#pragma once
#include "common.cuh"
#include "route.cuh"
#include "stream.cuh"

namespace moe {

constexpr int kDStageBytes = 48 * 1024;   // one ring stage of the decode kernel
constexpr int kDStages = 4;
constexpr int kDMaxRowVec = 6;            // 16-byte row vectors per lane (d <= 4608)
constexpr int kDMaxK1 = 32;
constexpr int kDMaxSeg = 8;               // expert segments of one CTA's channels
constexpr int kGroupBar0 = 2;             // named barriers 2..5: one per slot group

static_assert(kSC == kDStages * kWPS, "decode kernel: one group of consumer warps per slot");

struct DecodeArgs {
    const uint16_t *x;    // [1 x d]
    const uint16_t *wg;   // [E x I x d]
    const uint16_t *wu;   // [E x I x d]
    const uint16_t *wdt;  // [E x I x d]: down matrix, channel-major
    int d, E, I, k1, k2;
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
    float *y_acc;  // [d] float32, zero on entry
    void *y;       // [d] output (y_dtype); written by the last CTA to finish
    int y_dtype;
    VarK vk;       // variable k: cascade or skip (kind 0 with the fixed-k kernel)
    int32_t *count;  // nullable: kt
    WsHeader *hdr;
};

// One expert's share of this CTA's channel range.
struct DSeg {
    int u;  // index into the activated-expert list
    int a;  // first channel (within the expert)
    int b;  // one past the last channel
};

struct __align__(16) DecodeSmem {
    float hs[kDStages][kWPS];  // w*h of the stage's channels, per group
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
    int first;                 // this CTA checked in first: it writes the route out
    int last;                  // this CTA checked in last: it writes y
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

// VPL: d = 256*VPL for the single-token register path (x in registers when
// VPL <= kXRegMax), 0 for the general token loop.  CASCADE: the variable-k
// route (a.vk: cascade or skip).
template <int VPL, bool CASCADE>
__global__ void __launch_bounds__(kSThreads, 1) k_decode(DecodeArgs a)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *ring = smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kDStages * kDStageBytes);
    uint64_t *empty = full + kDStages;
    DecodeSmem *ds = reinterpret_cast<DecodeSmem *>(empty + kDStages);
    uint8_t *area = reinterpret_cast<uint8_t *>(ds + 1);  // the token's x row, d bf16

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x, b = blockIdx.x;
    int *status = &a.hdr->status;
    const int d = a.d, E = a.E, I = a.I, k1 = a.k1;

    if (tid == 0) {
        for (int s = 0; s < kDStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kWPS);
        }
        ds->abort = 0;
        ds->issued = 0;
        fence_mbar_init();
        // this CTA's channel segments depend only on k1, I and the grid (with
        // the cascade, on the routed count: computed after routing)
        if constexpr (!CASCADE)
            decode_segments(ds, k1, I, G, b, status);
    }
    __syncthreads();

    pdl_wait();
    pdl_trigger();

    // ------------------------------------------------------------ routing (one warp)
    if (warp == 0) {
        int j, kt;
        float wv;
        const VarK vk = CASCADE ? a.vk : VarK();
        if (E <= 128)
            warp_route<4>(a.logits, E, k1, a.k2, lane, j, wv, vk, &kt);
        else if (E <= 256)
            warp_route<8>(a.logits, E, k1, a.k2, lane, j, wv, vk, &kt);
        else if (E <= 512)
            warp_route<16>(a.logits, E, k1, a.k2, lane, j, wv, vk, &kt);
        else
            warp_route<32>(a.logits, E, k1, a.k2, lane, j, wv, vk, &kt);
        int p = 0;  // position of this lane's expert among the kt taken, ascending
        for (int q = 0; q < k1; ++q)
            p += __shfl_sync(0xffffffffu, j, q) < j;  // empty slots never count
        if (lane < k1) {
            if (j != MOE_EMPTY_SLOT) {  // taken (kt of the k1 slots)
                ds->ue[p] = j;
                ds->uw[p] = wv;
            }
            // kept for the routing outputs, written after the stream by the
            // first CTA to finish (off the path the layer's time waits on)
            ds->sj[lane] = j;
            ds->sw[lane] = wv;
            ds->sp[lane] = j != MOE_EMPTY_SLOT ? p : -1;
        }
        if (lane == 0)
            ds->kt = kt;
        __syncwarp();
        if constexpr (CASCADE) {
            if (lane == 0)
                decode_segments(ds, kt, I, G, b, status);
        }
    } else {
        // the token's x row, meanwhile
        for (int i = tid - 32; i < (d >> 3); i += kSThreads - 32)
            reinterpret_cast<uint4 *>(area)[i] = reinterpret_cast<const uint4 *>(a.x)[i];
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
            int slot = 0;
            uint32_t ph = 0;
            int issued = 0;
            while (it.valid()) {
                if (*(volatile int *)&ds->abort)
                    break;
                if (!mbar_wait(&empty[slot], ph ^ 1u, status)) {
                    ds->abort = 1;
                    break;
                }
                const int n = it.count();
                const int e = ds->ue[ds->seg[it.s].u];
                const size_t row0 = (size_t)e * I + it.c;
                const uint32_t bytes = (uint32_t)n * d * 2;
                uint8_t *dst = ring + (size_t)slot * kDStageBytes;
                mbar_arrive_expect_tx(&full[slot], 3 * bytes);
                bulk_g2s(dst, a.wg + row0 * d, bytes, &full[slot], pol);
                bulk_g2s(dst + bytes, a.wu + row0 * d, bytes, &full[slot], pol);
                bulk_g2s(dst + 2 * bytes, a.wdt + row0 * d, bytes, &full[slot], pol);
                ++issued;
                it.next();
                if (++slot == kDStages) {
                    slot = 0;
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
        const int nvec = d >> 3;  // 16-byte vectors per row
        // this warp's output rows: vectors v = gl*32 + lane + kWPS*32*j, j < RV
        constexpr int RV = VPL > 0 ? (VPL * 32 + kWPS * 32 - 1) / (kWPS * 32) : kDMaxRowVec;
        static_assert(RV <= kDMaxRowVec, "row partials");
        float yp[RV][8];
#pragma unroll
        for (int j = 0; j < RV; ++j)
#pragma unroll
            for (int k = 0; k < 8; ++k)
                yp[j][k] = 0.0f;

        uint4 xv[VPL > 0 && VPL <= kXRegMax ? VPL : 1];
        const uint4 *xs = reinterpret_cast<const uint4 *>(area);
        if constexpr (VPL > 0 && VPL <= kXRegMax) {
#pragma unroll
            for (int i = 0; i < VPL; ++i)
                xv[i] = xs[lane + 32 * i];
        }

        DIter it;
        it.init(ds->seg, nseg, nch);
        int sidx = 0;
        while (it.valid()) {
            const int n = it.count();
            if (sidx % kDStages == group) {
                const uint32_t parity = (uint32_t)((sidx / kDStages) & 1);
                const bool ok =
                    !*(volatile int *)&ds->abort && mbar_wait(&full[group], parity, status);
                if (!ok)
                    ds->abort = 1;
                const uint8_t *stg = ring + (size_t)group * kDStageBytes;
                const size_t rb = (size_t)n * d * 2;  // bytes of one of the three row blocks
                const float wgt = ds->uw[ds->seg[it.s].u];
                // (1) w * h for channel gl of the stage
                if (ok && gl < n) {
                    const uint4 *grow = reinterpret_cast<const uint4 *>(stg + (size_t)gl * d * 2);
                    const uint4 *urow = reinterpret_cast<const uint4 *>(stg + rb + (size_t)gl * d * 2);
                    float hval;
                    if constexpr (VPL > 0) {
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
                        ds->hs[group][gl] = hval * wgt;
                }
                named_bar_sync(kGroupBar0 + group, kWPS * 32);  // the group's h are in shared memory
                // (2) y partial += w*h * down row, for this warp's rows
                if (ok) {
                    const uint8_t *drows = stg + 2 * rb;
                    for (int i = 0; i < n; ++i) {
                        const float hv = ds->hs[group][i];
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
                // hand the slot back (hs[group] is next written after this
                // group's next stage wait, which needs these arrivals)
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&empty[group]);
            }
            ++sidx;
            it.next();
        }

        // ------------------------------------------------------------ reduce and add
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
        if (nseg > 0) {  // one 16-byte vector reduction per four output rows
            for (int r = tid * 4; r < d; r += kSC * 32 * 4) {
                float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int g = 0; g < kDStages; ++g) {
                    const float4 v = *reinterpret_cast<const float4 *>(red + (size_t)g * d + r);
                    sum.x += v.x;
                    sum.y += v.y;
                    sum.z += v.z;
                    sum.w += v.w;
                }
                red_add_v4(a.y_acc + r, sum.x, sum.y, sum.z, sum.w);
            }
        }
        __threadfence();  // the adds are visible before this CTA checks in below
    }

    __syncthreads();
    if (tid == 0 && ds->abort) {
        const int issued = ds->issued;
        for (int s = 0; s < kDStages && s < issued; ++s) {
            const int last = issued - 1 - ((issued - 1 - s) % kDStages);
            const uint32_t parity = (uint32_t)((last / kDStages) & 1);
            mbar_wait(&full[s], parity, status);
        }
    }

    // ------------------------------------------------------------ y (last CTA to finish)
    if (tid == 0) {
        const unsigned prev = atomicAdd(&a.hdr->decode_arrive, 1u);
        ds->first = prev == 0u;
        ds->last = prev == (unsigned)G - 1;
    }
    __syncthreads();
    if (ds->first && warp == 0) {
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
            int cnt = 0;
            for (int q = 0; q < kt; ++q)
                cnt += ds->ue[q] < e;
            a.offsets[e] = cnt;
        }
    }
    if (ds->last) {
        __threadfence();
        for (int i = tid * 4; i < d; i += kSThreads * 4) {
            const float4 v = __ldcg(reinterpret_cast<const float4 *>(a.y_acc + i));
            if (a.y_dtype == MOE_DTYPE_BF16) {
                const uint32_t lo = f32_to_bf16_rn(v.x) | ((uint32_t)f32_to_bf16_rn(v.y) << 16);
                const uint32_t hi = f32_to_bf16_rn(v.z) | ((uint32_t)f32_to_bf16_rn(v.w) << 16);
                *reinterpret_cast<uint2 *>(reinterpret_cast<uint16_t *>(a.y) + i) =
                    make_uint2(lo, hi);
            } else {
                *reinterpret_cast<float4 *>(reinterpret_cast<float *>(a.y) + i) = v;
            }
        }
        if (tid == 0)
            a.hdr->decode_arrive = 0u;
    }
}

inline size_t decode_smem_bytes(int d)
{
    return (size_t)kDStages * kDStageBytes + 2 * kDStages * sizeof(uint64_t) + sizeof(DecodeSmem) +
           (size_t)d * 2;
}

// The single-pass path serves one token per call (T == 1) whose output rows
// fit the register partials, with the down matrix channel-major.
inline bool decode_fits(int T, int d, int E, int I, int k1, int G)
{
    if (T != 1 || k1 > kDMaxK1 || (d >> 3) > kWPS * 32 * kDMaxRowVec)
        return false;
    if (decode_smem_bytes(d) > 227 * 1024 || (size_t)kDStages * d * 4 > (size_t)kDStages * kDStageBytes)
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
