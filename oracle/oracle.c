/*
 * oracle.c -- plain, slow CPU reference for the routed-expert MoE layer with
 * decoupled top-k1 / top-k2 renormalisation.
 *
 * THIS IS TEST INFRASTRUCTURE.  Only the test-suite, the smoke check and the
 * CPU-baseline leg of the benchmark load it.  The GPU library never links,
 * includes or calls anything here, and nothing here comes from the GPU code.
 *
 * What it follows (page = the source web page, cited by title and section):
 *  - "Paper of the Week #3 -- Half the FLOPs Is Not Half the Time"
 *    (sotaaz.com), section "The Receipt", Eq. 2:
 *        w_i = p_i / sum_{j in Top-k2} p_j   for i in Top-k1,
 *    with k2 = k1 the standard renormalisation and k2 = E no renormalisation.
 *  - same page, section "Ship It / Code of the Week": logits are a bias-free
 *    linear map of the hidden state, probabilities are a softmax taken in
 *    float32, the top min(k2, E) probabilities are taken in descending order,
 *    the first k1 are kept, and they are divided by the sum of all min(k2, E)
 *    taken values unless k2 >= E (then no division).  k2 >= k1 is required.
 *  - "Channel Selection for Mixture-of-Experts Decoding Needs No Calibration
 *    Data" (paperlayer.ai), section 2 "Background": a routed expert is a gated
 *    MLP; channel c owns gate row c, up row c and down column c.
 *  - The gated MLP is SwiGLU: h_c = silu(g_c) * u_c, silu(a) = a / (1 + e^-a),
 *    o = W_down h; the layer output is y = sum_s w_s o_s.
 *
 * Readings taken where the pages are silent (each one is listed in the design
 * notes of the repository):
 *  - ties in the top-k are broken by the lower expert index; selection is on p;
 *  - the float32 softmax and the top-k2 mass follow one fixed ("canonical")
 *    sequence of float32 operations so that a GPU implementation can be
 *    compared bit for bit (see oracle_route_f32 below);
 *  - the top-k2 mass is summed sequentially in rank order;
 *  - the returned weights stay in float32 (the page casts them to the logits
 *    dtype; that cast is not applied here);
 *  - an optional per-expert float32 router bias is added once after the dot
 *    product.
 *
 * Compile with contraction and fast-math OFF (-ffp-contract=off
 * -fno-fast-math): every float operation below is one IEEE-754 binary32
 * operation rounded to nearest even, and fmaf is the correctly rounded fused
 * multiply-add of C99.
 *
 * Parity status of each exported function (pins live in tests/):
 *  oracle_exp_c            pinned: exhaustive error bound vs double exp, exp(0)=1
 *  oracle_softmax_f32      pinned: uniform logits -> 1/E exactly, sum within E ulp,
 *                          agreement with the double softmax
 *  oracle_route_f32/_f64   pinned: Eq. 2 special cases and invariants,
 *                          brute-force subset enumeration, tie rule, the page's
 *                          router restated with library top-k
 *  oracle_route_cascade_f32  pinned: tau below the top probability gives k = 1,
 *                          tau above any reachable mass gives kmax, uniform
 *                          logits give k = ceil(tau E) exactly, minimality by
 *                          brute force (mass of the first k-1 < tau), equality
 *                          with the fixed-k route on the taken prefix
 *  oracle_logits           pinned: library matmul (numpy) on exactly
 *                          representable inputs, bias shift
 *  oracle_expert           pinned: I=1 closed form, zero weights, library
 *                          matmul + silu in double, linearity in W_down
 *  oracle_combine          pinned: k1=1 gives w*o, slot-order permutation
 *  oracle_permute          pinned: scan/stability/inverse properties, brute force
 *  oracle_layer            pinned: identical experts give (sum w) * FFN(x),
 *                          E=1 reduces to a plain SwiGLU MLP, zero experts give 0.
 *                          The pages print no worked example of a full layer,
 *                          so no page value pins its end-to-end output.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_OK 0
#define OR_BAD_ARG (-1)
#define ORACLE_EMPTY_SLOT 0x7fffffff /* an unused slot of a variable-k route */

/* ------------------------------------------------------------------------ */
/* element access: dtype 0 = float32, 1 = bfloat16 (upper half of a float32) */

static float bf16_bits_to_f32(uint16_t v)
{
    uint32_t u = ((uint32_t)v) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static float elem(const void *base, int dtype, size_t i)
{
    if (dtype == 1)
        return bf16_bits_to_f32(((const uint16_t *)base)[i]);
    return ((const float *)base)[i];
}

/* ------------------------------------------------------------------------ */
/* exp_c: the canonical float32 exponential used by the routing softmax.
 *
 * Method: Cody & Waite argument reduction (W. J. Cody, W. Waite, "Software
 * Manual for the Elementary Functions", 1980) followed by the Taylor series
 * of e^r truncated after the r^7 term, evaluated in Horner form with fused
 * multiply-adds, and an exact scaling by 2^n built from exponent bits.
 *
 *   n = rint(x * log2(e))                 (float32 multiply, round-half-even)
 *   r = (x - n*LN2_HI) - n*LN2_LO         (two fmaf; n*LN2_HI is exact because
 *                                          LN2_HI has 12 significant bits)
 *   p = 1 + r(1 + r(1/2 + r(1/6 + ... + r/5040)))   (Horner, fmaf each step)
 *   exp_c(x) = p * 2^n
 *
 * |r| <= ln2/2 + 2^-10, so the first dropped Taylor term r^8/8! is below
 * 6e-9, a small fraction of an ulp.  Domain: x <= 88; the softmax only calls
 * it with x = z - max(z) <= 0.  x < -87 (and NaN) returns +0, which keeps
 * every result a normal number (e^-87 > FLT_MIN).  x = 0 gives exactly 1.
 */
static const float EXPC_LOG2E = 0x1.715476p+0f;   /* fp32(1/ln 2)                      */
static const float EXPC_LN2_HI = 0x1.62ep-1f;     /* ln 2 cut to 12 significant bits   */
static const float EXPC_LN2_LO = 0x1.0bfbe8p-15f; /* fp32(ln 2 - EXPC_LN2_HI)          */
static const float EXPC_C2 = 0x1p-1f;             /* 1/2!                              */
static const float EXPC_C3 = 0x1.555556p-3f;      /* fp32(1/3!)                        */
static const float EXPC_C4 = 0x1.555556p-5f;      /* fp32(1/4!)                        */
static const float EXPC_C5 = 0x1.111112p-7f;      /* fp32(1/5!)                        */
static const float EXPC_C6 = 0x1.6c16c2p-10f;     /* fp32(1/6!)                        */
static const float EXPC_C7 = 0x1.a01a02p-13f;     /* fp32(1/7!)                        */

float oracle_exp_c(float x)
{
    if (!(x >= -87.0f))
        return 0.0f;
    if (x > 88.0f)
        return INFINITY;
    float t = x * EXPC_LOG2E;
    float n = rintf(t);
    float r = fmaf(-n, EXPC_LN2_HI, x);
    r = fmaf(-n, EXPC_LN2_LO, r);
    float p = EXPC_C7;
    p = fmaf(p, r, EXPC_C6);
    p = fmaf(p, r, EXPC_C5);
    p = fmaf(p, r, EXPC_C4);
    p = fmaf(p, r, EXPC_C3);
    p = fmaf(p, r, EXPC_C2);
    p = fmaf(p, r, 1.0f);
    p = fmaf(p, r, 1.0f);
    int ni = (int)n;
    uint32_t sb = (uint32_t)(ni + 127) << 23;
    float s;
    memcpy(&s, &sb, sizeof s);
    return p * s;
}

void oracle_exp_c_array(const float *x, float *y, int64_t n)
{
#pragma omp parallel for schedule(static) if (n > 100000)
    for (int64_t i = 0; i < n; ++i)
        y[i] = oracle_exp_c(x[i]);
}

/* Distance in units in the last place between a float result and the exact
 * value v (given in double): |res - v| / ulp(v), ulp taken at v's binade. */
static double ulp_error(float res, double v)
{
    if (v == 0.0)
        return res == 0.0f ? 0.0 : INFINITY;
    int e;
    frexp(v, &e); /* v = m * 2^e, m in [0.5, 1) */
    double ulp = ldexp(1.0, e - 24);
    if (ulp < ldexp(1.0, -149))
        ulp = ldexp(1.0, -149);
    return fabs((double)res - v) / ulp;
}

/* Sweep every float32 bit pattern from -0 down to -87 (inclusive) and return
 * the largest ulp error of exp_c against the double-precision exp.  Also
 * counts results that are not normal numbers (must be 0). */
double oracle_exp_c_sweep(uint32_t stride, int64_t *n_checked, int64_t *n_not_normal)
{
    const uint32_t lo = 0x80000000u;               /* -0.0  */
    uint32_t hi;                                   /* -87.0 */
    {
        float m87 = -87.0f;
        memcpy(&hi, &m87, sizeof hi);
    }
    if (stride == 0)
        stride = 1;
    double worst = 0.0;
    int64_t cnt = 0, bad = 0;
#pragma omp parallel for reduction(max : worst) reduction(+ : cnt, bad) schedule(static)
    for (int64_t b = lo; b <= (int64_t)hi; b += stride) {
        uint32_t u = (uint32_t)b;
        float x;
        memcpy(&x, &u, sizeof x);
        float y = oracle_exp_c(x);
        double ref = exp((double)x);
        double err = ulp_error(y, ref);
        if (err > worst)
            worst = err;
        if (!isnormal(y))
            ++bad;
        ++cnt;
    }
    if (n_checked)
        *n_checked = cnt;
    if (n_not_normal)
        *n_not_normal = bad;
    return worst;
}

/* ------------------------------------------------------------------------ */
/* Canonical float32 softmax of one row of E logits.
 *
 *   m   = max_j z_j                         (exact)
 *   e_j = exp_c(z_j - m)                    (float32 subtraction, then exp_c)
 *   Z   : 32 partial sums; partial q (q = 0..31) starts at +0 and adds
 *         e_q, e_{q+32}, e_{q+64}, ... in that order; then five butterfly
 *         rounds P[q] <- P[q] + P[q xor o] for o = 16, 8, 4, 2, 1 (all q at
 *         once); Z = P[0] (all 32 end equal).
 *   p_j = e_j / Z                           (IEEE division, round to nearest)
 */
void oracle_softmax_f32(const float *z, int E, float *p)
{
    float m = z[0];
    for (int j = 1; j < E; ++j)
        if (z[j] > m)
            m = z[j];
    for (int j = 0; j < E; ++j)
        p[j] = oracle_exp_c(z[j] - m);
    float P[32];
    for (int q = 0; q < 32; ++q) {
        float acc = 0.0f;
        for (int j = q; j < E; j += 32)
            acc = acc + p[j];
        P[q] = acc;
    }
    for (int o = 16; o >= 1; o >>= 1) {
        float Q[32];
        for (int q = 0; q < 32; ++q)
            Q[q] = P[q] + P[q ^ o];
        memcpy(P, Q, sizeof P);
    }
    float Z = P[0];
    for (int j = 0; j < E; ++j)
        p[j] = p[j] / Z;
}

/* key order: a before b when p_a > p_b, or p_a == p_b and a < b */
static int before_f32(const float *p, int a, int b)
{
    return p[a] > p[b] || (p[a] == p[b] && a < b);
}

static int before_f64(const double *p, int a, int b)
{
    return p[a] > p[b] || (p[a] == p[b] && a < b);
}

/* Canonical float32 routing of T tokens (Eq. 2 on the float32 softmax).
 * logits [T x E] row-major.  Writes idx [T x k1] (rank order) and w [T x k1].
 * K = min(k2, E) experts are ranked; the first k1 are emitted.
 *   k2 >= E : w_s = p_{idx_s}
 *   else    : S = ((p_(0) + p_(1)) + ...) + p_(K-1)   (rank order)
 *             w_s = p_{idx_s} / S
 * Returns OR_BAD_ARG unless 1 <= k1 <= k2 and k1 <= E. */
int oracle_route_f32(const float *logits, int T, int E, int k1, int k2, int32_t *idx, float *w)
{
    if (T < 0 || E < 1 || k1 < 1 || k2 < k1 || k1 > E)
        return OR_BAD_ARG;
    const int K = k2 < E ? k2 : E;
    float *p = (float *)malloc(sizeof(float) * (size_t)E);
    int *rank = (int *)malloc(sizeof(int) * (size_t)K);
    char *taken = (char *)malloc((size_t)E);
    if (!p || !rank || !taken) {
        free(p);
        free(rank);
        free(taken);
        return OR_BAD_ARG;
    }
    for (int t = 0; t < T; ++t) {
        oracle_softmax_f32(logits + (size_t)t * E, E, p);
        memset(taken, 0, (size_t)E);
        for (int s = 0; s < K; ++s) {
            int best = -1;
            for (int j = 0; j < E; ++j)
                if (!taken[j] && (best < 0 || before_f32(p, j, best)))
                    best = j;
            taken[best] = 1;
            rank[s] = best;
        }
        float S = 0.0f;
        if (k2 < E)
            for (int s = 0; s < K; ++s)
                S = S + p[rank[s]];
        for (int s = 0; s < k1; ++s) {
            idx[(size_t)t * k1 + s] = rank[s];
            w[(size_t)t * k1 + s] = (k2 >= E) ? p[rank[s]] : p[rank[s]] / S;
        }
    }
    free(p);
    free(rank);
    free(taken);
    return OR_OK;
}

/* Double-precision twin: libm exp, plain index-order sums, the same ranking
 * and Eq. 2.  p_out (nullable) receives the [T x E] probabilities. */
/* Variable k per token (the "cascade ... cover" arm of "Reading the MoE
 * measurement defects", kozo-lab, sections 4 and 6.2-6.3): the experts are
 * taken in rank order until their probability mass reaches tau.  Reading
 * used here: the mass after k experts is the float32 sequential sum
 * (((p_(0) + p_(1)) + ...) + p_(k-1)) from +0, the same partial sums as the
 * top-k2 mass S; k_t = the smallest k <= kmax with mass >= tau, else kmax
 * (so k_t >= 1).  Weights are Eq. 2 with the fixed k2 (kmax <= k2).  Output
 * rows have kmax slots; slots s >= k_t hold ORACLE_EMPTY_SLOT and weight 0;
 * count[t] = k_t (count nullable). */
int oracle_route_cascade_f32(const float *logits, int T, int E, int kmax, int k2, float tau,
                             int32_t *idx, float *w, int32_t *count)
{
    if (T < 0 || E < 1 || kmax < 1 || k2 < kmax || kmax > E)
        return OR_BAD_ARG;
    const int K = k2 < E ? k2 : E;
    float *p = (float *)malloc(sizeof(float) * (size_t)E);
    int *rank = (int *)malloc(sizeof(int) * (size_t)K);
    char *taken = (char *)malloc((size_t)E);
    if (!p || !rank || !taken) {
        free(p);
        free(rank);
        free(taken);
        return OR_BAD_ARG;
    }
    for (int t = 0; t < T; ++t) {
        oracle_softmax_f32(logits + (size_t)t * E, E, p);
        memset(taken, 0, (size_t)E);
        for (int s = 0; s < K; ++s) {
            int best = -1;
            for (int j = 0; j < E; ++j)
                if (!taken[j] && (best < 0 || before_f32(p, j, best)))
                    best = j;
            taken[best] = 1;
            rank[s] = best;
        }
        int kt = kmax;
        float M = 0.0f;
        for (int s = 0; s < kmax; ++s) {
            M = M + p[rank[s]];
            if (M >= tau) {
                kt = s + 1;
                break;
            }
        }
        float S = 0.0f;
        if (k2 < E)
            for (int s = 0; s < K; ++s)
                S = S + p[rank[s]];
        for (int s = 0; s < kmax; ++s) {
            const size_t o = (size_t)t * kmax + s;
            if (s < kt) {
                idx[o] = rank[s];
                w[o] = (k2 >= E) ? p[rank[s]] : p[rank[s]] / S;
            } else {
                idx[o] = ORACLE_EMPTY_SLOT;
                w[o] = 0.0f;
            }
        }
        if (count)
            count[t] = kt;
    }
    free(p);
    free(rank);
    free(taken);
    return OR_OK;
}

int oracle_route_f64(const double *logits, int T, int E, int k1, int k2, int32_t *idx, double *w,
                     double *p_out)
{
    if (T < 0 || E < 1 || k1 < 1 || k2 < k1 || k1 > E)
        return OR_BAD_ARG;
    const int K = k2 < E ? k2 : E;
    double *p = (double *)malloc(sizeof(double) * (size_t)E);
    int *rank = (int *)malloc(sizeof(int) * (size_t)K);
    char *taken = (char *)malloc((size_t)E);
    if (!p || !rank || !taken) {
        free(p);
        free(rank);
        free(taken);
        return OR_BAD_ARG;
    }
    for (int t = 0; t < T; ++t) {
        const double *z = logits + (size_t)t * E;
        double m = z[0];
        for (int j = 1; j < E; ++j)
            if (z[j] > m)
                m = z[j];
        double Z = 0.0;
        for (int j = 0; j < E; ++j) {
            p[j] = exp(z[j] - m);
            Z += p[j];
        }
        for (int j = 0; j < E; ++j)
            p[j] /= Z;
        if (p_out)
            memcpy(p_out + (size_t)t * E, p, sizeof(double) * (size_t)E);
        memset(taken, 0, (size_t)E);
        for (int s = 0; s < K; ++s) {
            int best = -1;
            for (int j = 0; j < E; ++j)
                if (!taken[j] && (best < 0 || before_f64(p, j, best)))
                    best = j;
            taken[best] = 1;
            rank[s] = best;
        }
        double S = 0.0;
        for (int s = 0; s < K; ++s)
            S += p[rank[s]];
        for (int s = 0; s < k1; ++s) {
            idx[(size_t)t * k1 + s] = rank[s];
            w[(size_t)t * k1 + s] = (k2 >= E) ? p[rank[s]] : p[rank[s]] / S;
        }
    }
    free(p);
    free(rank);
    free(taken);
    return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* Router logits: z[t][e] = (sum_k x[t][k] * Wr[e][k]) + b[e], float32,
 * k ascending, each product and sum rounded separately; bias nullable. */
void oracle_logits(const void *x, int x_dtype, const void *wr, int w_dtype, const float *bias, int T,
                   int d, int E, float *z)
{
#pragma omp parallel for collapse(2) schedule(static)
    for (int t = 0; t < T; ++t)
        for (int e = 0; e < E; ++e) {
            float acc = 0.0f;
            for (int k = 0; k < d; ++k) {
                float prod = elem(x, x_dtype, (size_t)t * d + k) * elem(wr, w_dtype, (size_t)e * d + k);
                acc = acc + prod;
            }
            if (bias)
                acc = acc + bias[e];
            z[(size_t)t * E + e] = acc;
        }
}

/* ------------------------------------------------------------------------ */
/* One token through one SwiGLU expert, float32 throughout.
 *   xf [d]          the token (already widened to float32)
 *   wg, wu [I x d]  this expert's gate and up rows (channel c = row c)
 *   wd     [d x I]  this expert's down matrix (channel c = column c)
 *   g_c = sum_k wg[c][k] xf[k];  u_c = sum_k wu[c][k] xf[k]      (k ascending)
 *   h_c = (g_c / (1 + expf(-g_c))) * u_c
 *   o_j = sum_c wd[j][c] h_c                                      (c ascending)
 * h (nullable) receives the I channel activations.  par != 0 splits the
 * rows over OpenMP threads (results do not depend on the thread count). */
void oracle_expert(const float *xf, const void *wg, const void *wu, const void *wd, int w_dtype, int d,
                   int I, float *h, float *o, int par)
{
    float *hh = h ? h : (float *)malloc(sizeof(float) * (size_t)I);
#pragma omp parallel for schedule(static) if (par)
    for (int c = 0; c < I; ++c) {
        float g = 0.0f, u = 0.0f;
        for (int k = 0; k < d; ++k) {
            float pg = elem(wg, w_dtype, (size_t)c * d + k) * xf[k];
            float pu = elem(wu, w_dtype, (size_t)c * d + k) * xf[k];
            g = g + pg;
            u = u + pu;
        }
        float silu = g / (1.0f + expf(-g));
        hh[c] = silu * u;
    }
#pragma omp parallel for schedule(static) if (par)
    for (int j = 0; j < d; ++j) {
        float acc = 0.0f;
        for (int c = 0; c < I; ++c) {
            float prod = elem(wd, w_dtype, (size_t)j * I + c) * hh[c];
            acc = acc + prod;
        }
        o[j] = acc;
    }
    if (!h)
        free(hh);
}

/* y[j] = sum_{s=0}^{k1-1} w[s] * o[s][j], s ascending, float32. */
void oracle_combine(const float *o, const float *w, int k1, int d, float *y)
{
    for (int j = 0; j < d; ++j) {
        float acc = 0.0f;
        for (int s = 0; s < k1; ++s) {
            float prod = w[s] * o[(size_t)s * d + j];
            acc = acc + prod;
        }
        y[j] = acc;
    }
}

/* ------------------------------------------------------------------------ */
/* Stable counting sort of the T*k1 slots (slot i = t*k1 + s) by expert.
 *   offsets[E+1]     exclusive scan of the per-expert counts
 *   sorted_slot[n]   slots in (expert ascending, slot index ascending) order
 *   slot_pos[n]      inverse: sorted_slot[slot_pos[i]] == i
 * Returns OR_BAD_ARG on an expert index outside [0, E). */
int oracle_permute(const int32_t *idx, int T, int k1, int E, int32_t *offsets, int32_t *sorted_slot,
                   int32_t *slot_pos)
{
    const int64_t n = (int64_t)T * k1;
    for (int e = 0; e <= E; ++e)
        offsets[e] = 0;
    for (int64_t i = 0; i < n; ++i) {
        if (idx[i] == ORACLE_EMPTY_SLOT)
            continue; /* an unused slot of a variable-k route: not placed */
        if (idx[i] < 0 || idx[i] >= E)
            return OR_BAD_ARG;
        offsets[idx[i] + 1] += 1;
    }
    for (int e = 0; e < E; ++e)
        offsets[e + 1] += offsets[e];
    int32_t *next = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E > 0 ? E : 1));
    if (!next)
        return OR_BAD_ARG;
    for (int e = 0; e < E; ++e)
        next[e] = offsets[e];
    for (int64_t i = 0; i < n; ++i) {
        if (idx[i] == ORACLE_EMPTY_SLOT) {
            slot_pos[i] = -1;
            continue;
        }
        int32_t pos = next[idx[i]]++;
        sorted_slot[pos] = (int32_t)i;
        slot_pos[i] = pos;
    }
    free(next);
    return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* The whole layer for T tokens, float32, on the given (possibly bf16) inputs.
 *   x [T x d], wr [E x d], bias [E] (nullable), wg/wu [E x I x d], wd [E x d x I]
 *   logits_in [T x E] (nullable): when given, routing starts from these
 *   float32 logits instead of the oracle's own (used to route from another
 *   implementation's logits, so a near-tie at the k1 boundary cannot turn
 *   into an O(1) output difference).
 * Outputs: y [T x d] float32; idx/w [T x k1] (nullable); z_out [T x E]
 * (nullable, the logits actually routed on). */
int oracle_layer(const void *x, int x_dtype, const void *wr, const float *bias, const void *wg,
                 const void *wu, const void *wd, int w_dtype, int T, int d, int E, int I, int k1,
                 int k2, const float *logits_in, float *y, int32_t *idx_out, float *w_out,
                 float *z_out)
{
    if (T < 0 || d < 1 || E < 1 || I < 1 || k1 < 1 || k2 < k1 || k1 > E)
        return OR_BAD_ARG;
    size_t TE = (size_t)T * E;
    float *z = (float *)malloc(sizeof(float) * (TE ? TE : 1));
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)T * k1 + 1);
    float *w = (float *)malloc(sizeof(float) * (size_t)T * k1 + 1);
    if (!z || !idx || !w) {
        free(z);
        free(idx);
        free(w);
        return OR_BAD_ARG;
    }
    if (logits_in)
        memcpy(z, logits_in, sizeof(float) * TE);
    else
        oracle_logits(x, x_dtype, wr, w_dtype, bias, T, d, E, z);
    int rc = oracle_route_f32(z, T, E, k1, k2, idx, w);
    if (rc != OR_OK) {
        free(z);
        free(idx);
        free(w);
        return rc;
    }
    const int par_rows = T < 8;
#pragma omp parallel for schedule(dynamic, 1) if (!par_rows)
    for (int t = 0; t < T; ++t) {
        float *xf = (float *)malloc(sizeof(float) * (size_t)d);
        float *o = (float *)malloc(sizeof(float) * (size_t)k1 * d);
        for (int k = 0; k < d; ++k)
            xf[k] = elem(x, x_dtype, (size_t)t * d + k);
        for (int s = 0; s < k1; ++s) {
            size_t e = (size_t)idx[(size_t)t * k1 + s];
            oracle_expert(xf, (const char *)wg + e * (size_t)I * d * (w_dtype == 1 ? 2 : 4),
                          (const char *)wu + e * (size_t)I * d * (w_dtype == 1 ? 2 : 4),
                          (const char *)wd + e * (size_t)d * I * (w_dtype == 1 ? 2 : 4), w_dtype, d, I,
                          NULL, o + (size_t)s * d, par_rows);
        }
        oracle_combine(o, w + (size_t)t * k1, k1, d, y + (size_t)t * d);
        free(xf);
        free(o);
    }
    if (idx_out)
        memcpy(idx_out, idx, sizeof(int32_t) * (size_t)T * k1);
    if (w_out)
        memcpy(w_out, w, sizeof(float) * (size_t)T * k1);
    if (z_out)
        memcpy(z_out, z, sizeof(float) * TE);
    free(z);
    free(idx);
    free(w);
    return OR_OK;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
