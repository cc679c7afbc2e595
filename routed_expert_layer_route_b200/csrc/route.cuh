// route.cuh -- router logits, float32 softmax, top-k1/top-k2 selection with
// the decoupled renormalisation of Eq. 2, and the stable counting sort that
// groups routed slots by expert.
//
// Eq. 2 ("Paper of the Week #3 -- Half the FLOPs Is Not Half the Time",
// section "The Receipt"): w_i = p_i / sum_{j in Top-k2} p_j, i in Top-k1;
// k2 >= E means no division.  Order of operations ("Code of the Week"
// section of the same page): float32 softmax, top min(k2, E) in descending
// order, first k1 kept, divided by the sum of all min(k2, E) taken values.
//
// The float32 softmax and the top-k2 mass follow one fixed sequence of
// IEEE-754 binary32 operations so the result is reproducible bit for bit:
//   m   = max_j z_j
//   e_j = expc(z_j - m)                       (expc: see below)
//   Z   : 32 partial sums, partial q adds e_q, e_{q+32}, ... in order from +0;
//         then five butterfly rounds P[q] <- P[q] + P[q ^ o], o = 16..1
//   p_j = e_j / Z                             (round-to-nearest division)
//   rank by (p descending, j ascending); K = min(k2, E)
//   S   = (((p_(0) + p_(1)) + ...) + p_(K-1)) in rank order (k2 < E only)
//   w_s = p_(s) / S   (k2 < E)   or   p_(s)   (k2 >= E),   s < k1.
// Every float operation below that takes part in this sequence is written
// with an explicit round-to-nearest intrinsic so the compiler cannot fuse or
// reorder it.
#pragma once
#include "common.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// expc: float32 exponential for x <= 88, from Cody & Waite's two-constant
// argument reduction (W. J. Cody, W. Waite, "Software Manual for the
// Elementary Functions", 1980) and the Taylor series of e^r up to r^7 in
// Horner form with fused multiply-adds; 2^n applied through exponent bits.
// ln2 split: the high part is ln 2 cut to 12 significant bits (n * hi is
// exact for |n| < 2^12), the low part is float32(ln 2 - hi).  Below -87 (and
// for NaN) the result is +0, so results are never subnormal.
__device__ __forceinline__ float expc(float x)
{
    const float kLog2e = 0x1.715476p+0f;
    const float kLn2Hi = 0x1.62ep-1f;
    const float kLn2Lo = 0x1.0bfbe8p-15f;
    if (!(x >= -87.0f))
        return 0.0f;
    if (x > 88.0f)
        return __int_as_float(0x7f800000);
    const float n = rintf(__fmul_rn(x, kLog2e));
    float r = __fmaf_rn(-n, kLn2Hi, x);
    r = __fmaf_rn(-n, kLn2Lo, r);
    float p = 0x1.a01a02p-13f;             // 1/7!
    p = __fmaf_rn(p, r, 0x1.6c16c2p-10f);  // 1/6!
    p = __fmaf_rn(p, r, 0x1.111112p-7f);   // 1/5!
    p = __fmaf_rn(p, r, 0x1.555556p-5f);   // 1/4!
    p = __fmaf_rn(p, r, 0x1.555556p-3f);   // 1/3!
    p = __fmaf_rn(p, r, 0x1p-1f);          // 1/2!
    p = __fmaf_rn(p, r, 1.0f);
    p = __fmaf_rn(p, r, 1.0f);
    const int ni = (int)n;
    return __fmul_rn(p, __int_as_float((ni + 127) << 23));
}

__global__ void k_test_expc(const float *x, float *y, int64_t n)
{
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        y[i] = expc(x[i]);
}

// ---------------------------------------------------------------------------
struct __align__(16) RouteSmem {
    float ps[1024];    // e_j = expc(z_j - m)
    float pp[1024];    // p_j = e_j / Z
    float sel_p[1024]; // probabilities in rank order (ranks < Kneed)
    int sel_j[1024];   // their expert ids
    float red[64];
    int out_j[32];     // the k1 selected experts, rank order
    float out_w[32];   // their Eq. 2 weights
};

// One CTA routes one token whose E logits sit in shared memory (E <= 1024).
// Leaves the k1 selected experts and weights in sm.out_j / sm.out_w and
// writes them to idx_out / w_out and the optional copies (each pointer
// nullable).  All threads of the CTA must call it; blockDim.x is a multiple
// of 32.  Five block barriers: the normaliser Z is formed by every warp
// redundantly, in the same fixed order, so no barrier is needed after it.
__device__ void route_token_block(const float *zs, int E, int k1, int k2, RouteSmem &sm,
                                  int32_t *idx_out, float *w_out, int32_t *idx_copy,
                                  float *w_copy)
{
    const int tid = threadIdx.x, nt = blockDim.x;
    const int lane = tid & 31, warp = tid >> 5, nw = nt >> 5;
    const int K = k2 < E ? k2 : E;
    const bool renorm = k2 < E;
    const int Kneed = renorm ? K : k1;

    // m = max_j z_j (exact in any order)
    float m = -__int_as_float(0x7f800000);
    for (int j = tid; j < E; j += nt)
        m = fmaxf(m, zs[j]);
    for (int o = 16; o >= 1; o >>= 1)
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0)
        sm.red[warp] = m;
    __syncthreads();  // 1
    m = sm.red[0];
    for (int w = 1; w < nw; ++w)
        m = fmaxf(m, sm.red[w]);

    for (int j = tid; j < E; j += nt)
        sm.ps[j] = expc(__fsub_rn(zs[j], m));
    __syncthreads();  // 2

    // Z in the canonical 32-partial order, then the butterfly (every warp)
    float Z = 0.0f;
    for (int j = lane; j < E; j += 32)
        Z = __fadd_rn(Z, sm.ps[j]);
    for (int o = 16; o >= 1; o >>= 1)
        Z = __fadd_rn(Z, __shfl_xor_sync(0xffffffffu, Z, o));
    for (int j = tid; j < E; j += nt)
        sm.pp[j] = __fdiv_rn(sm.ps[j], Z);
    __syncthreads();  // 3

    // rank_j = #{i : p_i > p_j} + #{i < j : p_i == p_j}; keep rank < Kneed
    for (int j = tid; j < E; j += nt) {
        const float pj = sm.pp[j];
        int r = 0;
        int i = 0;
        for (; i + 4 <= E; i += 4) {
            const float4 v = *reinterpret_cast<const float4 *>(&sm.pp[i]);
            r += (v.x > pj) | ((v.x == pj) & (i + 0 < j));
            r += (v.y > pj) | ((v.y == pj) & (i + 1 < j));
            r += (v.z > pj) | ((v.z == pj) & (i + 2 < j));
            r += (v.w > pj) | ((v.w == pj) & (i + 3 < j));
        }
        for (; i < E; ++i) {
            const float v = sm.pp[i];
            r += (v > pj) | ((v == pj) & (i < j));
        }
        if (r < Kneed) {
            sm.sel_p[r] = pj;
            sm.sel_j[r] = j;
        }
    }
    __syncthreads();  // 4

    // S = (((p_(0) + p_(1)) + ...) + p_(K-1)) in rank order; Eq. 2 weights
    if (tid == 0) {
        float S = 0.0f;
        if (renorm)
            for (int r = 0; r < K; ++r)
                S = __fadd_rn(S, sm.sel_p[r]);
        for (int s = 0; s < k1; ++s) {
            const float p = sm.sel_p[s];
            sm.out_j[s] = sm.sel_j[s];
            sm.out_w[s] = renorm ? __fdiv_rn(p, S) : p;
        }
    }
    __syncthreads();  // 5
    if (tid < k1) {
        const int j = sm.out_j[tid];
        const float wv = sm.out_w[tid];
        if (idx_out)
            idx_out[tid] = j;
        if (w_out)
            w_out[tid] = wv;
        if (idx_copy)
            idx_copy[tid] = j;
        if (w_copy)
            w_copy[tid] = wv;
    }
}

// ---------------------------------------------------------------------------
// Block-wide exclusive scan of n ints (in place in smem), returns the total.
// scratch: >= 33 ints.
__device__ int block_exclusive_scan(int *v, int n, int *scratch)
{
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
    const int per = (n + nt - 1) / nt;
    const int b = tid * per, e = min(n, b + per);
    int local = 0;
    for (int i = b; i < e; ++i)
        local += v[i];
    int incl = local;
    for (int o = 1; o < 32; o <<= 1) {
        int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o)
            incl += t;
    }
    if (lane == 31)
        scratch[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int nw = nt >> 5;
        int t = lane < nw ? scratch[lane] : 0;
        int s = t;
        for (int o = 1; o < 32; o <<= 1) {
            int u = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o)
                s += u;
        }
        scratch[lane] = s - t;  // exclusive prefix of warp totals
        if (lane == 31)
            scratch[32] = s;
    }
    __syncthreads();
    int run = scratch[warp] + incl - local;
    for (int i = b; i < e; ++i) {
        const int t = v[i];
        v[i] = run;
        run += t;
    }
    const int total = scratch[32];
    __syncthreads();
    return total;
}

// ---------------------------------------------------------------------------
// Stable counting sort of the n = T*k1 slots by expert, one CTA.
// Token chunks of 32*WC tokens are marked in a per-expert bitmap (bit l of
// word w of expert e = token t0 + 32w + l routes to e); the stable position
// of slot (t, s) is offsets[e] + (#tokens before t routed to e), counted with
// popc over the bitmap rows.
// smem (dynamic, ints): cnt[E+1] | run[E] | bits[E*WC] | pref[E*WC] | scan[40]
// Outputs: expert_offsets[E+1], sorted_slot[n], slot_pos[n],
// uniq_count[1], uniq_list[U] (activated experts, ascending).
struct PermOut {
    int32_t *offsets;
    int32_t *sorted_slot;
    int32_t *slot_pos;
    int32_t *uniq_count;  // nullable
    int32_t *uniq_list;   // nullable
};

// 32-token words of the bitmap handled per chunk: bounded by 32, by a 4096-word
// bitmap, and by the tokens there are.
__host__ __device__ inline int permute_words_per_chunk(int E, int T)
{
    int wc = 4096 / (E > 0 ? E : 1);
    const int need = (T + 31) / 32;
    if (wc > 32)
        wc = 32;
    if (wc > need)
        wc = need;
    return wc < 1 ? 1 : wc;
}

__device__ void permute_block(const int32_t *idx, int T, int k1, int E, PermOut out, int *smem,
                              int *status)
{
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5, nw = nt >> 5;
    const int WC = permute_words_per_chunk(E, T);
    int *cnt = smem;
    int *run = cnt + (E + 1);
    unsigned *bits = reinterpret_cast<unsigned *>(run + E);
    int *pref = reinterpret_cast<int *>(bits + E * WC);
    int *scan = pref + E * WC;
    const int n = T * k1;

    for (int e = tid; e <= E; e += nt)
        cnt[e] = 0;
    __syncthreads();
    // pass 1: per-expert counts, warp-aggregated
    for (int base = warp * 32; base < n; base += nt) {
        const int i = base + lane;
        int e = i < n ? __ldcg(&idx[i]) : -1;
        const bool valid = (e >= 0) & (e < E);
        if (i < n && !valid && e != MOE_EMPTY_SLOT)
            set_status(status, MOE_ERR_DEVICE_CHECK);
        const int key = valid ? e : -1;
        const unsigned grp = __match_any_sync(0xffffffffu, key);
        if (valid && lane == __ffs(grp) - 1)
            atomicAdd(&cnt[e], __popc(grp));
    }
    __syncthreads();
    // uniq list from the counts (before the scan overwrites them)
    for (int e = tid; e < E; e += nt)
        run[e] = cnt[e] > 0 ? 1 : 0;
    __syncthreads();
    const int U = block_exclusive_scan(run, E, scan);
    if (out.uniq_list)
        for (int e = tid; e < E; e += nt)
            if (cnt[e] > 0)
                out.uniq_list[run[e]] = e;
    if (out.uniq_count && tid == 0)
        *out.uniq_count = U;
    __syncthreads();
    block_exclusive_scan(cnt, E + 1, scan);  // cnt[e] = offsets[e], cnt[E] = n
    for (int e = tid; e <= E; e += nt)
        out.offsets[e] = cnt[e];
    for (int e = tid; e < E; e += nt)
        run[e] = 0;
    __syncthreads();

    const unsigned lt_mask = (1u << lane) - 1u;
    for (int t0 = 0; t0 < T; t0 += 32 * WC) {
        for (int i = tid; i < E * WC; i += nt)
            bits[i] = 0u;
        __syncthreads();
        for (int w = warp; w < WC; w += nw) {
            const int t = t0 + 32 * w + lane;
            for (int s = 0; s < k1; ++s) {
                int e = t < T ? __ldcg(&idx[t * k1 + s]) : -1;
                const bool valid = (e >= 0) & (e < E);
                const int key = valid ? e : -1;
                const unsigned grp = __match_any_sync(0xffffffffu, key);
                if (valid && lane == __ffs(grp) - 1) {
                    if (bits[e * WC + w] & grp)
                        set_status(status, MOE_ERR_DEVICE_CHECK);  // repeated expert in a token
                    bits[e * WC + w] |= grp;
                }
                __syncwarp();
            }
        }
        __syncthreads();
        for (int e = tid; e < E; e += nt) {
            int acc = run[e];
            for (int w = 0; w < WC; ++w) {
                pref[e * WC + w] = acc;
                acc += __popc(bits[e * WC + w]);
            }
            run[e] = acc;
        }
        __syncthreads();
        for (int w = warp; w < WC; w += nw) {
            const int t = t0 + 32 * w + lane;
            if (t < T) {
                for (int s = 0; s < k1; ++s) {
                    const int e = __ldcg(&idx[t * k1 + s]);
                    if (e < 0 || e >= E)
                        continue;
                    const int pos = cnt[e] + pref[e * WC + w] + __popc(bits[e * WC + w] & lt_mask);
                    out.sorted_slot[pos] = t * k1 + s;
                    out.slot_pos[t * k1 + s] = pos;
                }
            }
        }
        __syncthreads();
    }
}

__host__ __device__ inline size_t permute_smem_bytes(int E, int T)
{
    const int WC = permute_words_per_chunk(E, T);
    return sizeof(int) * ((size_t)(E + 1) + E + 2 * (size_t)E * WC + 40);
}

// ---------------------------------------------------------------------------
// k_permute: standalone permutation (one CTA).
__global__ void __launch_bounds__(1024) k_permute(const int32_t *idx, int T, int k1, int E,
                                                  PermOut out, int *status)
{
    extern __shared__ int dsm[];
    pdl_wait();
    pdl_trigger();
    permute_block(idx, T, k1, E, out, dsm, status);
}

// ---------------------------------------------------------------------------
// k_topk: one CTA per token routes from float32 logits [T x E].  With
// `perm.offsets` non-null, the last CTA to finish also runs the permutation
// of all T*k1 slots (last-block hand-off through hdr->route_arrive).
__global__ void __launch_bounds__(1024) k_topk(const float *logits, int T, int E, int k1, int k2,
                                               int32_t *idx, float *w, int32_t *idx_copy,
                                               float *w_copy, PermOut perm, WsHeader *hdr)
{
    __shared__ RouteSmem sm;
    __shared__ float zs[1024];
    __shared__ int is_last;
    extern __shared__ int dsm[];
    pdl_wait();
    pdl_trigger();
    int *status = hdr ? &hdr->status : nullptr;
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        for (int j = threadIdx.x; j < E; j += blockDim.x)
            zs[j] = logits[(size_t)t * E + j];
        __syncthreads();
        route_token_block(zs, E, k1, k2, sm, idx + (size_t)t * k1, w + (size_t)t * k1,
                          idx_copy ? idx_copy + (size_t)t * k1 : nullptr,
                          w_copy ? w_copy + (size_t)t * k1 : nullptr);
        __syncthreads();
    }
    if (perm.offsets == nullptr)
        return;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(&hdr->route_arrive, 1u);
        is_last = (prev == gridDim.x - 1);
    }
    __syncthreads();
    if (!is_last)
        return;
    if (threadIdx.x == 0)
        hdr->route_arrive = 0u;
    __threadfence();
    permute_block(idx, T, k1, E, perm, dsm, status);
}

// ---------------------------------------------------------------------------
// Variable experts per token.  kind 0: the fixed k1.  kind 1, cascade (the
// "cascade ... cover" arm of "Reading the MoE measurement defects", sections
// 4 and 6.2-6.3): the first kt <= k1 ranked experts whose mass reaches tau.
// kind 2, skip (the expert-skipping shell of "ACE", aimodeling.com, section
// "How ACE decides what to skip: GSP + RCR": two views must both call a slot
// low before it is skipped, and the top-1 expert is always kept): slot
// s >= 1 is skipped when tab[e_s] < th_e (the per-expert offline scalar,
// looked up) and its Eq. 2 weight w_s < th_w (the token's router-conditioned
// view); kept slots keep their Eq. 2 weights.  Unused slots hold
// MOE_EMPTY_SLOT with weight 0 -- a suffix for the cascade, anywhere after
// slot 0 for skip.
struct VarK {
    int kind;
    float tau;
    const float *tab;  // [E] (skip)
    float th_e, th_w;
};
constexpr int kVarFixed = 0, kVarCascade = 1, kVarSkip = 2;

// ---------------------------------------------------------------------------
// warp_route_vals: one warp routes one token from its E float32 logits, held
// as p[i] = z[lane + 32 i], everything in registers.  That assignment is
// exactly the canonical partial-sum assignment of the normaliser Z; the
// top-Kneed probabilities come out in rank order by repeated warp arg-max on
// (p descending, j ascending) -- two redux.sync per rank: the largest key,
// then the lowest index holding it -- so the top-k2 mass S is summed in rank
// order as it is found.  Same float sequence, same bits as
// route_token_block.  Lane s < k1 returns the rank-s expert in my_j and its
// Eq. 2 weight in my_w.
// With a VarK (above): for the cascade the experts are taken in rank order
// until their mass -- the same float32 rank-order partial sums as S --
// reaches tau; kt = the smallest such k <= k1, else k1, and lanes
// kt <= s < k1 return MOE_EMPTY_SLOT and weight 0; for skip the skipped lanes
// return MOE_EMPTY_SLOT and weight 0.  kt = the slots taken (k1 when fixed).
// k_route_warp: one warp per token.
template <int R>
__device__ __forceinline__ void warp_route_vals(float (&p)[R], int E, int k1, int k2, int lane,
                                                int &my_j, float &my_w, VarK vk = VarK(),
                                                int *kt_out = nullptr)
{
    const bool cascade = vk.kind == kVarCascade;
    const float tau = vk.tau;
    const float kNegInf = -__int_as_float(0x7f800000);
    float m = kNegInf;
#pragma unroll
    for (int i = 0; i < R; ++i)
        if (lane + 32 * i < E)
            m = fmaxf(m, p[i]);
    asm volatile("redux.sync.max.f32 %0, %0, 0xffffffff;" : "+f"(m));  // exact in any order
    float Z = 0.0f;
#pragma unroll
    for (int i = 0; i < R; ++i)
        if (lane + 32 * i < E) {
            p[i] = expc(__fsub_rn(p[i], m));
            Z = __fadd_rn(Z, p[i]);
        }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1)
        Z = __fadd_rn(Z, __shfl_xor_sync(0xffffffffu, Z, o));
    // key = bits of p + 1 (p >= 0, so the bits order like the values); 0 = taken / absent
    unsigned key[R];
#pragma unroll
    for (int i = 0; i < R; ++i)
        key[i] = lane + 32 * i < E ? __float_as_uint(__fdiv_rn(p[i], Z)) + 1u : 0u;

    const int K = k2 < E ? k2 : E;
    const bool renorm = k2 < E;
    const int Kneed = renorm ? K : k1;
    float S = 0.0f, my_p = 0.0f;
    int kt = k1;
    bool covered = false;
    my_j = 0;
    for (int r = 0; r < Kneed; ++r) {
        unsigned kl = 0u;
        int jl = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < R; ++i)
            if (key[i] > kl) {  // strict: the lowest j among equal p in this lane
                kl = key[i];
                jl = lane + 32 * i;
            }
        const unsigned km = __reduce_max_sync(0xffffffffu, kl);
        const int bj = (int)__reduce_min_sync(0xffffffffu, kl == km ? (unsigned)jl : 0xffffffffu);
        const float bp = __uint_as_float(km - 1u);
        if (lane == r) {
            my_j = bj;
            my_p = bp;
        }
        S = __fadd_rn(S, bp);  // mass of the first r+1 ranks
        if (cascade && !covered && r < k1 && S >= tau) {
            covered = true;
            kt = r + 1;
        }
#pragma unroll
        for (int i = 0; i < R; ++i)
            if (lane + 32 * i == bj)
                key[i] = 0u;
    }
    my_w = renorm ? __fdiv_rn(my_p, S) : my_p;
    if (lane >= kt && lane < k1) {
        my_j = MOE_EMPTY_SLOT;
        my_w = 0.0f;
    }
    if (vk.kind == kVarSkip) {
        if (lane >= 1 && lane < k1 && __ldg(&vk.tab[my_j]) < vk.th_e && my_w < vk.th_w) {
            my_j = MOE_EMPTY_SLOT;
            my_w = 0.0f;
        }
        kt = __popc(__ballot_sync(0xffffffffu, lane < k1 && my_j != MOE_EMPTY_SLOT));
    }
    if (kt_out)
        *kt_out = kt;
}

// The same from E logits in global memory.
template <int R>
__device__ __forceinline__ void warp_route(const float *z, int E, int k1, int k2, int lane,
                                           int &my_j, float &my_w, VarK vk = VarK(),
                                           int *kt_out = nullptr)
{
    float p[R];
#pragma unroll
    for (int i = 0; i < R; ++i) {
        const int j = lane + 32 * i;
        p[i] = j < E ? __ldcg(&z[j]) : 0.0f;
    }
    warp_route_vals<R>(p, E, k1, k2, lane, my_j, my_w, vk, kt_out);
}

template <int R>
__global__ void __launch_bounds__(256) k_route_warp(const float *logits, int T, int E, int k1,
                                                    int k2, int32_t *idx, float *w,
                                                    int32_t *idx_copy, float *w_copy,
                                                    VarK vk, int32_t *count)
{
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T)
        return;
    int my_j, kt;
    float my_w;
    warp_route<R>(logits + (size_t)t * E, E, k1, k2, lane, my_j, my_w, vk, &kt);
    if (count && lane == 0)
        count[t] = kt;
    if (lane < k1) {
        const size_t o = (size_t)t * k1 + lane;
        idx[o] = my_j;
        w[o] = my_w;
        if (idx_copy)
            idx_copy[o] = my_j;
        if (w_copy)
            w_copy[o] = my_w;
    }
}

// ---------------------------------------------------------------------------
// Large-batch permutation in two kernels over chunks of kPermTok tokens.
// k_perm_hist: per-chunk expert counts into hist[chunk][E] (and the range /
// repeat checks of the expert ids).  k_perm_scatter: every chunk turns the
// counts into its starting position per expert (offsets of all experts plus
// the counts of earlier chunks) and one warp walks the chunk's slots in
// order, so the sort is stable by slot index.
constexpr int kPermTok = 128;

__global__ void __launch_bounds__(256) k_perm_hist(const int32_t *idx, int T, int k1, int E,
                                                   int *hist, int *status)
{
    extern __shared__ int hsm[];  // cnt[E], ids[kPermTok * k1]
    int *cnt = hsm, *ids = hsm + E;
    pdl_wait();
    pdl_trigger();
    const int tid = threadIdx.x, nt = blockDim.x, b = blockIdx.x;
    for (int e = tid; e < E; e += nt)
        cnt[e] = 0;
    const int t0 = b * kPermTok, t1 = min(T, t0 + kPermTok);
    const int i0 = t0 * k1, m = (t1 - t0) * k1;
    for (int i = tid; i < m; i += nt)
        ids[i] = __ldcg(&idx[i0 + i]);
    __syncthreads();
    for (int i = tid; i < m; i += nt) {
        const int e = ids[i];
        if (e < 0 || e >= E) {
            if (e != MOE_EMPTY_SLOT)
                set_status(status, MOE_ERR_DEVICE_CHECK);
            continue;
        }
        atomicAdd(&cnt[e], 1);
        for (int q = i - i % k1; q < i; ++q)  // the same expert earlier in this token
            if (ids[q] == e)
                set_status(status, MOE_ERR_DEVICE_CHECK);
    }
    __syncthreads();
    for (int e = tid; e < E; e += nt)
        hist[(size_t)b * E + e] = cnt[e];
}

__global__ void __launch_bounds__(256) k_perm_scatter(const int32_t *idx, int T, int k1, int E,
                                                      const int *hist, PermOut out)
{
    extern __shared__ int psm[];  // base[E], run[E], tot[E + 1], scan[40], ids[kPermTok * k1]
    pdl_wait();
    pdl_trigger();
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, b = blockIdx.x;
    const int nch = gridDim.x;
    int *base = psm, *run = base + E, *tot = run + E, *scan = tot + E + 1, *ids = scan + 40;
    const int i0 = b * kPermTok * k1, i1 = min(T, (b + 1) * kPermTok) * k1;
    for (int i = tid; i < i1 - i0; i += nt)
        ids[i] = __ldcg(&idx[i0 + i]);
    for (int e = tid; e < E; e += nt) {
        int before = 0, all = 0;
        // the chunks' counts are independent loads: eight in flight at a time
#pragma unroll 8
        for (int c = 0; c < nch; ++c) {
            const int h = __ldcg(&hist[(size_t)c * E + e]);
            all += h;
            before += c < b ? h : 0;
        }
        base[e] = before;
        tot[e] = all;
        run[e] = 0;
    }
    if (tid == 0)
        tot[E] = 0;
    __syncthreads();
    block_exclusive_scan(tot, E + 1, scan);  // tot[e] = offsets[e], tot[E] = T*k1 (valid ids)
    if (b == 0)
        for (int e = tid; e <= E; e += nt)
            out.offsets[e] = tot[e];
    for (int e = tid; e < E; e += nt)
        base[e] += tot[e];
    __syncthreads();
    if (tid < 32) {
        const unsigned lt = (1u << lane) - 1u;
        for (int i = i0; i < i1; i += 32) {
            const int slot = i + lane;
            const int e = slot < i1 ? ids[slot - i0] : -1;
            const bool valid = e >= 0 && e < E;
            const unsigned grp = __match_any_sync(0xffffffffu, valid ? e : -1);
            if (valid) {
                const int pos = base[e] + run[e] + __popc(grp & lt);
                out.sorted_slot[pos] = slot;
                out.slot_pos[slot] = pos;
            }
            __syncwarp();
            if (valid && lane == __ffs(grp) - 1)
                run[e] += __popc(grp);
            __syncwarp();
        }
    }
}

inline size_t perm_hist_smem_bytes(int E, int k1) { return sizeof(int) * ((size_t)E + kPermTok * k1); }
inline size_t perm_scatter_smem_bytes(int E, int k1)
{
    return sizeof(int) * ((size_t)3 * E + 1 + 40 + kPermTok * k1);
}

// ---------------------------------------------------------------------------
// One router logit, x . W_r[e], in one fixed float32 order: lane l takes the
// 16-byte vectors v = l + 32 i of both rows in turn (i = 0, 1, ...), i even
// into accumulator a0, i odd into a1 (two dependent chains instead of one),
// then a0 + a1 and the xor butterfly 16..1 (warp_sum); the bias is added
// after.  k_logits and the one-token layer kernel both use it, so a layer
// call routes on the same bits as moe_route.
MOE_DEVINL void router_step(float &a0, float &a1, int i, const uint4 w, const uint4 x)
{
    const float xf[8] = {bf16lo(x.x), bf16hi(x.x), bf16lo(x.y), bf16hi(x.y),
                         bf16lo(x.z), bf16hi(x.z), bf16lo(x.w), bf16hi(x.w)};
    if (i & 1)
        a1 = dot8_bf16(w, xf, a1);
    else
        a0 = dot8_bf16(w, xf, a0);
}

// ---------------------------------------------------------------------------
// k_logits: z[t, e] = sum_k x[t, k] W_r[e, k] (+ b[e]) with float32
// accumulation.  One warp per (expert, chunk of up to 8 tokens).  The warp's
// W_r row is loaded into registers before the programmatic-launch wait (the
// router weights never depend on earlier kernels), so its HBM latency
// overlaps the previous kernel.
constexpr int kLogitsWarps = 8;
constexpr int kLogitsTok = 8;
constexpr int kLogitsMaxVec = 16;  // register prefetch covers d <= 4096

struct LogitsArgs {
    const uint16_t *x;
    const uint16_t *wr;
    const float *bias;
    float *z;       // [T x E] output (workspace or caller)
    float *z_copy;  // nullable second copy (caller's logits_out)
    int T, d, E;
    float4 *zero;   // nullable: float4 buffer the grid clears (the layer's y accumulator)
    int zero_n4;
};

__global__ void __launch_bounds__(kLogitsWarps * 32) k_logits(LogitsArgs a)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nchunk = (a.T + kLogitsTok - 1) / kLogitsTok;
    const int item = blockIdx.x * kLogitsWarps + warp;
    const int nitems = a.E * nchunk;
    const int nvec = a.d >> 3;  // 16-byte vectors per row
    const bool has_item = item < nitems;
    const int e = has_item ? item % a.E : 0;
    const int chunk = has_item ? item / a.E : 0;

    uint4 wv[kLogitsMaxVec];
    const bool prefetch = nvec <= 32 * kLogitsMaxVec;
    if (has_item && prefetch) {
        const uint4 *row = reinterpret_cast<const uint4 *>(a.wr + (size_t)e * a.d);
#pragma unroll
        for (int i = 0; i < kLogitsMaxVec; ++i) {
            const int v = lane + 32 * i;
            wv[i] = v < nvec ? ld_nc_v4(row + v) : make_uint4(0, 0, 0, 0);
        }
    }
    pdl_wait();
    pdl_trigger();
    if (a.zero) {
        for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < a.zero_n4; i += gridDim.x * blockDim.x)
            a.zero[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (!has_item)
        return;

    const uint4 *row = reinterpret_cast<const uint4 *>(a.wr + (size_t)e * a.d);
    const int t0 = chunk * kLogitsTok;
    const int nt = min(kLogitsTok, a.T - t0);
#pragma unroll 1
    for (int t = 0; t < nt; ++t) {
        const uint4 *xr = reinterpret_cast<const uint4 *>(a.x + (size_t)(t0 + t) * a.d);
        float a0 = 0.0f, a1 = 0.0f;
        if (prefetch) {
            // all x vectors of this lane first (independent loads), then the math
            uint4 xv[kLogitsMaxVec];
#pragma unroll
            for (int i = 0; i < kLogitsMaxVec; ++i) {
                const int v = lane + 32 * i;
                xv[i] = v < nvec ? xr[v] : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int i = 0; i < kLogitsMaxVec; ++i)
                if (lane + 32 * i < nvec)
                    router_step(a0, a1, i, wv[i], xv[i]);
        } else {
            int i = 0;
            for (int v = lane; v < nvec; v += 32, ++i)
                router_step(a0, a1, i, ld_nc_v4(row + v), xr[v]);
        }
        float sum = warp_sum(a0 + a1);
        if (lane == 0) {
            if (a.bias)
                sum = sum + a.bias[e];
            a.z[(size_t)(t0 + t) * a.E + e] = sum;
            if (a.z_copy)
                a.z_copy[(size_t)(t0 + t) * a.E + e] = sum;
        }
    }
}

}  // namespace moe
