// ctopk.cuh -- channel top-k inside the activated experts, one token at a
// time ("Channel Selection for Mixture-of-Experts Decoding Needs No
// Calibration Data", paperlayer.ai):
//  * section 2 "Background": channel c of a routed expert owns gate row c,
//    up row c and down column c; h_c = silu(W_gate[c,:] . x) * (W_up[c,:] . x);
//  * section 5.2: each channel is scored in output units,
//        score(s, c) = w_s * ||W_down_s[:, c]|| * |h_c|,
//    so channels of different experts compare, and the token keeps the
//    `keep` best of its k1 * I channels;
//  * section 5.3: kept channels are computed exactly.  The ternary sketch
//    that screens channels before h is known, and the low-rank recovery of
//    skipped channels, are not built: h is computed exactly for every channel
//    (all gate and up rows are read) and skipped channels add nothing, so the
//    bytes saved are the skipped channels' down columns.
//
// Two kernels per token, one persistent CTA per SM each:
//  k_ctk_gateup: one warp of every CTA routes the token from its logits
//      (warp_route, the same float32 sequence as every router kernel); the
//      token's k1 * I channels, flat index q = s * I + c (slot s in rank
//      order), are split into balanced contiguous ranges over the CTAs and
//      each warp forms h_q and score_q for one channel at a time, reading the
//      gate and up rows with 16-byte no-L1 loads;
//  k_ctk_down: every CTA loads all k1 * I scores, finds the keep-th largest
//      by a 4 x 8-bit radix select on the float32 bit patterns (scores are
//      non-negative, so bit order is numeric order), marks the kept channels
//      in flat order (equal scores to the lower q) with one block scan, and
//      streams its balanced share of the kept channels' down columns
//      (contiguous rows of the channel-major down matrix), adding
//      w_s * h_q * column into y_acc with 16-byte float32 vector reductions;
//      the last CTA to check in writes y.
// Like the decode kernel, partial sums reach y_acc in a timing-dependent
// order, so y can differ between runs in the last bits; h, the scores and
// the kept set are deterministic.
#pragma once
#include "common.cuh"
#include "route.cuh"
#include "stream.cuh"

namespace moe {

constexpr int kCtkThreads = 512;
constexpr int kCtkWarps = kCtkThreads / 32;
constexpr int kCtkMaxN = 16384;    // k1 * I of one token: its scores sit in shared memory
constexpr int kCtkMaxMine = 1024;  // kept channels one CTA may own: ceil(keep / G)
constexpr int kCtkUnroll = 4;      // down rows in flight per thread
constexpr int kCtkMaxK1 = 32;
constexpr int kCtkCand = 64;       // candidates ranked directly by the selection
constexpr int kCtkBuckets = 4096;  // first selection pass: key bits 30..19
static_assert(kCtkBuckets == 8 * kCtkThreads, "eight first-pass buckets per thread");

struct CtkArgs {
    const uint16_t *x;    // [d] this token's row
    const uint16_t *wg;   // [E x I x d]
    const uint16_t *wu;   // [E x I x d]
    const uint16_t *wdt;  // [E x I x d]: down matrix, channel-major
    const float *norms;   // [E x I] float32 down-column norms
    const float *logits;  // [E] this token's logits
    int d, E, I, k1, k2, keep;
    int32_t *topk_idx;    // [k1] routing outputs (workspace)
    float *topk_w;
    int32_t *idx_copy;    // nullable caller copies
    float *w_copy;
    float *h;             // [k1 * I] workspace
    float *score;         // [k1 * I] workspace
    float *h_copy;        // nullable caller copies
    float *score_copy;
    int32_t *kept_out;    // nullable [keep]: kept flat indices, ascending
    float *y_acc;         // [d] float32, zero on entry
    void *y;              // [d] output (y_dtype), written by the last CTA of k_ctk_down
    int y_dtype;
    WsHeader *hdr;
};

// h of one channel from its gate and up rows in global memory and the
// token's x in shared memory (nvec = d / 8 vectors of 8 bf16).
MOE_DEVINL float ctk_channel(const uint16_t *grow, const uint16_t *urow, const uint4 *xs, int nvec,
                             int lane)
{
    float g0 = 0.f, g1 = 0.f, u0 = 0.f, u1 = 0.f;
    for (int base = 0; base < nvec; base += 256) {
        uint4 gv[8], uv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int v = base + lane + 32 * i;
            if (v < nvec) {
                gv[i] = ld_nc_v4(grow + 8 * (size_t)v);
                uv[i] = ld_nc_v4(urow + 8 * (size_t)v);
            }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int v = base + lane + 32 * i;
            if (v < nvec) {
                float xf[8], fg[8], fu[8];
                bf16x8(xs[v], xf);
                bf16x8(gv[i], fg);
                bf16x8(uv[i], fu);
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
        }
    }
    return silu_mul(warp_sum(g0 + g1), warp_sum(u0 + u1));
}

__global__ void __launch_bounds__(kCtkThreads, 1) k_ctk_gateup(CtkArgs a)
{
    extern __shared__ __align__(16) uint4 ctk_xs[];  // the token's x, d / 8 vectors
    __shared__ int se[kCtkMaxK1];
    __shared__ float sw[kCtkMaxK1];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x, b = blockIdx.x;
    const int d = a.d, E = a.E, I = a.I, k1 = a.k1;
    const int nvec = d >> 3;

    pdl_wait();
    pdl_trigger();
    if (warp == 0) {
        int j;
        float wv;
        if (E <= 128)
            warp_route<4>(a.logits, E, k1, a.k2, lane, j, wv);
        else if (E <= 256)
            warp_route<8>(a.logits, E, k1, a.k2, lane, j, wv);
        else if (E <= 512)
            warp_route<16>(a.logits, E, k1, a.k2, lane, j, wv);
        else
            warp_route<32>(a.logits, E, k1, a.k2, lane, j, wv);
        if (lane < k1) {
            se[lane] = j;
            sw[lane] = wv;
            if (b == 0) {
                a.topk_idx[lane] = j;
                a.topk_w[lane] = wv;
                if (a.idx_copy)
                    a.idx_copy[lane] = j;
                if (a.w_copy)
                    a.w_copy[lane] = wv;
            }
        }
    } else {
        for (int i = tid - 32; i < nvec; i += kCtkThreads - 32)
            ctk_xs[i] = reinterpret_cast<const uint4 *>(a.x)[i];
    }
    __syncthreads();

    const unsigned N = (unsigned)k1 * (unsigned)I;
    const unsigned lo = split_lo(N, G, b), hi = split_lo(N, G, b + 1);
    for (unsigned q = lo + warp; q < hi; q += kCtkWarps) {
        const int s = (int)(q / (unsigned)I), c = (int)(q % (unsigned)I);
        const size_t row = (size_t)se[s] * I + c;
        const float h = ctk_channel(a.wg + row * d, a.wu + row * d, ctk_xs, nvec, lane);
        if (lane == 0) {
            const float sc = __fmul_rn(__fmul_rn(sw[s], __ldg(&a.norms[row])), fabsf(h));
            a.h[q] = h;
            a.score[q] = sc;
            if (a.h_copy)
                a.h_copy[q] = h;
            if (a.score_copy)
                a.score_copy[q] = sc;
        }
    }
}

// Exclusive block scan of two counters (kCtkThreads threads); total gets
// the block-wide sums.
MOE_DEVINL int2 ctk_block_scan2(int x, int y, int2 *wtot, int2 &total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int ix = x, iy = y;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int vx = __shfl_up_sync(0xffffffffu, ix, o);
        const int vy = __shfl_up_sync(0xffffffffu, iy, o);
        if (lane >= o) {
            ix += vx;
            iy += vy;
        }
    }
    if (lane == 31)
        wtot[warp] = make_int2(ix, iy);
    __syncthreads();
    int bx = 0, by = 0, tx = 0, ty = 0;
    for (int w = 0; w < kCtkWarps; ++w) {
        const int2 v = wtot[w];
        if (w < warp) {
            bx += v.x;
            by += v.y;
        }
        tx += v.x;
        ty += v.y;
    }
    total = make_int2(tx, ty);
    return make_int2(bx + ix - x, by + iy - y);
}

__global__ void __launch_bounds__(kCtkThreads, 1) k_ctk_down(CtkArgs a)
{
    extern __shared__ __align__(16) uint8_t ctk_smem[];
    __shared__ unsigned hist[256];
    __shared__ int2 wtot[kCtkWarps];
    __shared__ int mine[kCtkMaxMine];          // this CTA's kept channels (flat q)
    __shared__ const uint16_t *mrow[kCtkMaxMine];
    __shared__ float mcoef[kCtkMaxMine];
    __shared__ unsigned hist0[kCtkBuckets];
    __shared__ unsigned s_digit, s_rem, s_cnt, s_ncand;
    __shared__ unsigned cand[kCtkCand];
    __shared__ int s_e[kCtkMaxK1];
    __shared__ float s_w[kCtkMaxK1];
    __shared__ int s_last;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x, b = blockIdx.x;
    const int d = a.d, I = a.I;
    const int N = a.k1 * I, K = a.keep;
    unsigned *key = reinterpret_cast<unsigned *>(ctk_smem);               // [N]
    float *red = reinterpret_cast<float *>(ctk_smem + (((size_t)N * 4 + 15) & ~(size_t)15));

    for (int i = tid; i < kCtkBuckets; i += kCtkThreads)
        hist0[i] = 0;
    pdl_wait();
    pdl_trigger();
    if (tid < a.k1) {
        s_e[tid] = __ldcg(&a.topk_idx[tid]);
        s_w[tid] = __ldcg(&a.topk_w[tid]);
    }
    __syncthreads();  // hist0 is clear
    // first pass: 4096 buckets on bits 30..19 of the key (the exponent and the
    // top four mantissa bits: sixteen buckets per binade), no range needed
#pragma unroll 4
    for (int i = tid; i < N; i += kCtkThreads) {
        const unsigned k = __float_as_uint(__ldcg(&a.score[i]));
        key[i] = k;
        atomicAdd(&hist0[k >> 19], 1u);
    }
    __syncthreads();
    {
        // thread t holds buckets 4095 - 8t - j, j < 8 (thread 0 the top ones)
        unsigned c[8], tot = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            c[j] = hist0[kCtkBuckets - 1 - 8 * tid - j];
            tot += c[j];
        }
        int2 total;
        const unsigned above0 = (unsigned)ctk_block_scan2((int)tot, 0, wtot, total).x;
        if (above0 < (unsigned)K && above0 + tot >= (unsigned)K) {  // exactly one thread
            unsigned above = above0;
            for (int j = 0; j < 8; ++j) {
                if (above + c[j] >= (unsigned)K) {
                    s_digit = (unsigned)(kCtkBuckets - 1 - 8 * tid - j);
                    s_rem = (unsigned)K - above;
                    s_cnt = c[j];
                    break;
                }
                above += c[j];
            }
        }
        __syncthreads();
    }

    // ---------------------------------------------------- the keep-th largest key
    // Then a range-adaptive radix select inside that bucket.  The candidates
    // are the keys in [lo, hi]
    // (cnt of them) and the answer is the rem-th largest candidate; every key
    // above hi is kept.  A pass buckets the candidates by (k - lo) >> shift
    // into at most 256 buckets (linear in the bit pattern, so the buckets
    // spread over the scores' decades and the shared atomics rarely collide)
    // and keeps the bucket that holds the rem-th largest; hi - lo shrinks by
    // 2^8 per pass, so at most four passes run before lo == hi, and as soon as
    // at most kCtkCand candidates are left they are ranked directly.
    unsigned lo = s_digit << 19, hi = lo + ((1u << 19) - 1), rem = s_rem, cnt = s_cnt;
    unsigned thr;
    for (;;) {
        if (lo == hi) {
            thr = lo;
            break;
        }
        if (cnt <= (unsigned)kCtkCand) {
            if (tid == 0)
                s_ncand = 0;
            __syncthreads();
            for (int i = tid; i < N; i += kCtkThreads) {
                const unsigned k = key[i];
                if (k >= lo && k <= hi)
                    cand[atomicAdd(&s_ncand, 1u)] = k;
            }
            __syncthreads();
            const int nc = (int)s_ncand;
            for (int j = tid; j < nc; j += kCtkThreads) {
                const unsigned c = cand[j];
                unsigned gt = 0, eq = 0;
#pragma unroll 16
                for (int m = 0; m < kCtkCand; ++m) {
                    const unsigned v = m < nc ? cand[m] : 0u;
                    gt += m < nc && v > c;
                    eq += m < nc && v == c;
                }
                if (gt < rem && gt + eq >= rem)
                    s_digit = c;  // every writer writes the same value
            }
            __syncthreads();
            thr = s_digit;
            break;
        }
        const int bits = 32 - __clz(hi - lo);
        const int shift = bits > 8 ? bits - 8 : 0;
        for (int i = tid; i < 256; i += kCtkThreads)
            hist[i] = 0;
        __syncthreads();
        for (int i = tid; i < N; i += kCtkThreads) {
            const unsigned k = key[i];
            if (k >= lo && k <= hi)
                atomicAdd(&hist[(k - lo) >> shift], 1u);
        }
        __syncthreads();
        if (warp == 0) {
            unsigned c[8], tot = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                c[j] = hist[8 * lane + j];
                tot += c[j];
            }
            unsigned suf = tot;  // candidates in the buckets of this lane and the lanes above
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned v = __shfl_down_sync(0xffffffffu, suf, o);
                if (lane + o < 32)
                    suf += v;
            }
            unsigned above = suf - tot;
            if (above < rem && suf >= rem) {  // exactly one lane
                for (int j = 7; j >= 0; --j) {
                    if (above + c[j] >= rem) {
                        s_digit = (unsigned)(8 * lane + j);
                        s_rem = rem - above;
                        s_cnt = c[j];
                        break;
                    }
                    above += c[j];
                }
            }
        }
        __syncthreads();
        const unsigned long long nlo = (unsigned long long)lo + ((unsigned long long)s_digit << shift);
        const unsigned long long nhi = nlo + ((1ull << shift) - 1);
        lo = (unsigned)nlo;
        hi = nhi < hi ? (unsigned)nhi : hi;
        rem = s_rem;
        cnt = s_cnt;
    }
    // ---------------------------------------------------- kept set, in flat order
    // warp w walks the contiguous segment [w*seg, (w+1)*seg) 32 keys at a
    // time (coalesced); ballots give the in-order ranks of the keys above
    // thr and of the keys equal to it
    const int seg = (((N + kCtkWarps - 1) / kCtkWarps) + 31) & ~31;
    const int s0 = min(N, warp * seg), s1 = min(N, s0 + seg);
    const unsigned lt = (1u << lane) - 1u;
    int ngt = 0, neq = 0;
#pragma unroll 4
    for (int i0 = s0; i0 < s1; i0 += 32) {
        const int i = i0 + lane;
        const unsigned k = i < s1 ? key[i] : 0u;
        ngt += __popc(__ballot_sync(0xffffffffu, i < s1 && k > thr));
        neq += __popc(__ballot_sync(0xffffffffu, i < s1 && k == thr));
    }
    if (lane == 0)
        wtot[warp] = make_int2(ngt, neq);
    __syncthreads();
    int gt_before = 0, eq_before = 0, tot_gt = 0;
    for (int w = 0; w < kCtkWarps; ++w) {
        const int2 v = wtot[w];
        if (w < warp) {
            gt_before += v.x;
            eq_before += v.y;
        }
        tot_gt += v.x;
    }
    const int n_eq = K - tot_gt;  // keys equal to thr that are kept: the first n_eq
    const int p_lo = (int)split_lo((unsigned)K, G, b), p_hi = (int)split_lo((unsigned)K, G, b + 1);
    int pos = gt_before + min(eq_before, n_eq);
#pragma unroll 4
    for (int i0 = s0; i0 < s1; i0 += 32) {
        const int i = i0 + lane;
        const unsigned k = i < s1 ? key[i] : 0u;
        const unsigned eqb = __ballot_sync(0xffffffffu, i < s1 && k == thr);
        const bool kp = i < s1 && (k > thr || (k == thr && eq_before + __popc(eqb & lt) < n_eq));
        const unsigned kb = __ballot_sync(0xffffffffu, kp);
        if (kp) {
            const int my = pos + __popc(kb & lt);
            if (my >= p_lo && my < p_hi)
                mine[my - p_lo] = i;
            if (b == 0 && a.kept_out)
                a.kept_out[my] = i;
        }
        pos += __popc(kb);
        eq_before += __popc(eqb);
    }
    __syncthreads();
    const int nm = p_hi - p_lo;
    for (int i = tid; i < nm; i += kCtkThreads) {
        const int q = mine[i];
        const int s = q / I, c = q - s * I;
        mrow[i] = a.wdt + ((size_t)s_e[s] * I + c) * d;
        mcoef[i] = __fmul_rn(s_w[s], __ldcg(&a.h[q]));
    }
    __syncthreads();

    // ---------------------------------------------------- y_acc += sum coef * column
    const int C = d >> 3;                                   // 16-byte vectors per row
    const int P = C >= kCtkThreads ? 1 : kCtkThreads / C;   // rows side by side
    const int pr = tid / C;
    const int v0 = tid - pr * C;
    float acc[2][8];
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int k = 0; k < 8; ++k)
            acc[u][k] = 0.f;
    if (pr < P) {
        for (int i0 = pr; i0 < nm; i0 += kCtkUnroll * P) {
            uint4 rv[kCtkUnroll][2];
#pragma unroll
            for (int r = 0; r < kCtkUnroll; ++r) {
                const int i = i0 + r * P;
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int v = v0 + u * kCtkThreads;
                    if (i < nm && v < C)
                        rv[r][u] = ld_nc_v4(mrow[i] + 8 * (size_t)v);
                }
            }
#pragma unroll
            for (int r = 0; r < kCtkUnroll; ++r) {
                const int i = i0 + r * P;
                if (i < nm) {
                    const float cf = mcoef[i];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int v = v0 + u * kCtkThreads;
                        if (v < C) {
                            float f[8];
                            bf16x8(rv[r][u], f);
#pragma unroll
                            for (int k = 0; k < 8; ++k)
                                acc[u][k] = fmaf(f[k], cf, acc[u][k]);
                        }
                    }
                }
            }
        }
    }
    if (nm > 0) {
        // the P side-by-side partials of each output row, then one atomic per row
        if (P > 1) {
            if (pr < P) {
                float4 *dst = reinterpret_cast<float4 *>(red + (size_t)pr * d + 8 * v0);
                dst[0] = make_float4(acc[0][0], acc[0][1], acc[0][2], acc[0][3]);
                dst[1] = make_float4(acc[0][4], acc[0][5], acc[0][6], acc[0][7]);
            }
            __syncthreads();
            for (int r = tid * 4; r < d; r += kCtkThreads * 4) {
                float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int p = 0; p < P; ++p) {
                    const float4 v = *reinterpret_cast<const float4 *>(red + (size_t)p * d + r);
                    sum.x += v.x;
                    sum.y += v.y;
                    sum.z += v.z;
                    sum.w += v.w;
                }
                red_add_v4(a.y_acc + r, sum.x, sum.y, sum.z, sum.w);
            }
        } else if (pr < P) {
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int v = v0 + u * kCtkThreads;
                if (v < C) {
                    red_add_v4(a.y_acc + 8 * v, acc[u][0], acc[u][1], acc[u][2], acc[u][3]);
                    red_add_v4(a.y_acc + 8 * v + 4, acc[u][4], acc[u][5], acc[u][6], acc[u][7]);
                }
            }
        }
    }
    __threadfence();  // the adds are visible before this CTA checks in
    __syncthreads();

    // ---------------------------------------------------- y (last CTA to finish)
    if (tid == 0)
        s_last = atomicAdd(&a.hdr->decode_arrive, 1u) == (unsigned)G - 1;
    __syncthreads();
    if (s_last) {
        __threadfence();
        for (int i = tid * 4; i < d; i += kCtkThreads * 4) {
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

inline size_t ctk_down_smem_bytes(int N, int d)
{
    const int C = d >> 3;
    const int P = C >= kCtkThreads ? 1 : kCtkThreads / C;
    return (((size_t)N * 4 + 15) & ~(size_t)15) + (P > 1 ? (size_t)P * d * 4 : 0);
}

// Down-column norms n[e][c] = ||W_down_e[:, c]|| in float32 (sum of squares
// in float32, then an IEEE square root).  Channel-major input [E x I x d]:
// one warp per channel row.
__global__ void __launch_bounds__(512) k_norms_cm(const uint16_t *wdt, int E, int I, int d,
                                                   float *norms)
{
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const long row = (long)blockIdx.x * 16 + (threadIdx.x >> 5);
    if (row >= (long)E * I)
        return;
    const uint16_t *p = wdt + row * d;
    float s = 0.f;
    for (int v = lane; v < (d >> 3); v += 32) {
        float f[8];
        bf16x8(ld_nc_v4(p + 8 * (size_t)v), f);
#pragma unroll
        for (int k = 0; k < 8; ++k)
            s = fmaf(f[k], f[k], s);
    }
    s = warp_sum(s);
    if (lane == 0)
        norms[row] = __fsqrt_rn(s);
}

// The same from the HF layout [E x d x I]: one thread per column, rows in order.
__global__ void __launch_bounds__(256) k_norms_hf(const uint16_t *wd, int E, int I, int d,
                                                   float *norms)
{
    pdl_wait();
    pdl_trigger();
    const int e = blockIdx.y;
    const int c = blockIdx.x * 256 + threadIdx.x;
    if (c >= I)
        return;
    const uint16_t *p = wd + (size_t)e * d * I + c;
    float s = 0.f;
    for (int r = 0; r < d; ++r) {
        const float f = __uint_as_float((uint32_t)__ldg(p + (size_t)r * I) << 16);
        s = fmaf(f, f, s);
    }
    norms[(size_t)e * I + c] = __fsqrt_rn(s);
}

}  // namespace moe
