// stream.cuh -- small-batch expert FFN that streams only the activated
// experts' weights from HBM, each byte once.
//
// Structure of an expert ("Channel Selection for Mixture-of-Experts Decoding
// Needs No Calibration Data", section 2 "Background"): a gated MLP whose
// channel c owns gate row c, up row c and down column c.  SwiGLU:
//     h_c = silu(W_gate[c,:] . x) * (W_up[c,:] . x),   o = W_down h.
//
// Design (one persistent CTA per SM, grid = number of SMs):
//  * the U activated experts (ascending ids) are laid end to end as U*I
//    channels; CTA b owns the contiguous channel range
//    [b*U*I/G, (b+1)*U*I/G), so every CTA streams the same number of gate/up
//    bytes (within one channel) whatever k1, U or the batch;
//  * phase 1: gate and up rows of the CTA's channels (contiguous in HBM) are
//    moved by bulk asynchronous copies (cp.async.bulk, no multicast) into a
//    ring of shared-memory stages by one producer thread; 16 consumer warps
//    form the dot products with the expert's tokens (staged in shared
//    memory) and write h (float32) for their channels;
//  * one grid-wide barrier (bounded spin) makes every h visible;
//  * phase 2: CTA b owns the output rows [b*d/G, (b+1)*d/G) of every
//    activated expert; its W_down rows (contiguous, I elements each) stream
//    through the same ring -- the producer issues them before the barrier
//    completes, so the barrier hides under copies in flight -- and the
//    consumers write o = W_down h for the expert's tokens;
//  * the combine of Eq. 2's weights runs on the CTA's own rows: y[t, r] =
//    sum_s w[t, s] o[slot(t, s), r] in slot order, float32, no atomics, so
//    the output is deterministic.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int kSC = 16;                      // consumer warps
constexpr int kSThreads = (kSC + 1) * 32;    // + one producer warp
constexpr int kStages = 5;
constexpr int kStageBytes = 32 * 1024;
constexpr int kTokChunk = 8;                 // most tokens staged in shared memory at once
constexpr int kTokBytes = 32 * 1024;         // staging area for one token chunk
constexpr int kMaxRows = 128;                // rows of one stage
constexpr int kPartItems = 128;              // (row, slice) items of one stage
constexpr int kConsumerBar = 1;              // named barrier id of the consumer warps

struct StreamArgs {
    const uint16_t *x;   // [T x d]
    const uint16_t *wg;  // [E x I x d]
    const uint16_t *wu;  // [E x I x d]
    const uint16_t *wd;  // [E x d x I]
    int T, d, E, I, k1;
    const int32_t *offsets;      // [E+1]
    const int32_t *sorted_slot;  // [T*k1]
    const int32_t *uniq_count;   // [1]
    const int32_t *uniq_list;    // [E]
    float *h;                    // [T*k1 x I] scratch
    float *out;                  // [T*k1 x d] per-slot outputs, sorted order
    void *y;                     // nullable: combine into y [T x d]
    int y_dtype;
    const float *topk_w;         // [T x k1]
    const int32_t *slot_pos;     // [T*k1]
    WsHeader *hdr;
};

// The ordered list of stages a CTA works through; the producer and the
// consumers walk it independently and identically.
struct Stage {
    int phase;  // 1: gate/up rows of channels [c, c+n); 2: W_down rows [r, r+n)
    int u;      // index into uniq_list
    int c;      // first channel (phase 1) or first row (phase 2)
    int n;      // channels (phase 1) or rows (phase 2)
};

struct StageIter {
    int64_t c_cur, c_hi;  // phase-1 channel cursor over [0, U*I)
    int r_lo, r_hi;       // phase-2 rows of this CTA
    int u2, r2;           // phase-2 cursor
    int U, I, nch, nrows;
    int phase;

    __device__ void init(int U_, int I_, int d, int b, int G)
    {
        U = U_;
        I = I_;
        const int64_t tot = (int64_t)U * I;
        c_cur = tot * b / G;
        c_hi = tot * (b + 1) / G;
        r_lo = (int)((int64_t)d * b / G);
        r_hi = (int)((int64_t)d * (b + 1) / G);
        nch = max(1, min(kMaxRows / 2, kStageBytes / (4 * d)));
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
            s.u = (int)(c_cur / I);
            s.c = (int)(c_cur % I);
            int64_t lim = min((int64_t)(I - s.c), c_hi - c_cur);
            s.n = (int)min((int64_t)nch, lim);
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

__device__ __forceinline__ int floor_pow2(int v)
{
    int p = 1;
    while (p * 2 <= v)
        p *= 2;
    return p;
}

struct __align__(16) ConsumerSmem {
    float part[2][kPartItems * kTokChunk];
    int tok_pos0;  // first sorted position of the staged expert
    int tok_cnt;   // tokens of the staged expert
    int abort;
    int issued;    // stages issued by the producer
};

__device__ __forceinline__ void consumer_sync() { named_bar_sync(kConsumerBar, kSC * 32); }

// tokens per staged chunk: as many rows of x (bf16, d) or h (float32, I) as
// fit the staging area, at most kTokChunk
__host__ __device__ __forceinline__ int tok_chunk(int d, int I)
{
    const int row = 2 * d > 4 * I ? 2 * d : 4 * I;
    const int n = kTokBytes / row;
    return n < 1 ? 1 : (n > kTokChunk ? kTokChunk : n);
}

__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.0f + __expf(-g)) * u; }

__global__ void __launch_bounds__(kSThreads, 1) k_stream(StreamArgs a)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *ring = smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kStages * kStageBytes);
    uint64_t *empty = full + kStages;
    ConsumerSmem *cs = reinterpret_cast<ConsumerSmem *>(empty + kStages);
    // staging area for one token chunk: x rows (bf16, phase 1) or h rows
    // (float32, phase 2); 16-byte aligned
    uint8_t *tok_area = reinterpret_cast<uint8_t *>(cs + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x, b = blockIdx.x;
    int *status = &a.hdr->status;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kSC);
        }
        cs->abort = 0;
        cs->issued = 0;
        fence_mbar_init();
    }
    __syncthreads();

    pdl_wait();
    pdl_trigger();

    const int nslots = a.T * a.k1;
    int U = __ldcg(a.uniq_count);
    if (U < 0 || U > a.E) {
        if (tid == 0)
            set_status(status, MOE_ERR_DEVICE_CHECK);
        U = 0;
    }
    const int d = a.d, I = a.I, k1 = a.k1;
    const int mtc = tok_chunk(d, I);

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
                if (*(volatile int *)&cs->abort)
                    break;
                if (!mbar_wait(&empty[slot], ph ^ 1u, status)) {
                    cs->abort = 1;
                    break;
                }
                const Stage st = it.get();
                const int e = min(max(__ldcg(&a.uniq_list[st.u]), 0), a.E - 1);
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
            cs->issued = issued;
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ consumers
        StageIter it;
        it.init(U, I, d, b, G);
        int slot = 0;
        uint32_t ph = 0;
        int iter = 0;       // part[] double-buffer parity
        int staged_u = -1;  // expert whose token chunk sits in tok_area
        int staged_m0 = -1;
        int staged_phase = 0;
        bool arrived = false;

        auto do_grid_barrier = [&]() {
            __threadfence();  // this thread's h stores are visible device-wide
            consumer_sync();
            if (tid == 0) {
                unsigned gen0 = ld_acquire_u32(&a.hdr->bar_gen);
                // the generation read above was taken before this CTA
                // arrives, so it cannot have advanced yet
                __threadfence();
                const unsigned prev = atomicAdd(&a.hdr->bar_count, 1u);
                if (prev == (unsigned)G - 1) {
                    atomicExch(&a.hdr->bar_count, 0u);
                    __threadfence();
                    atomicAdd(&a.hdr->bar_gen, 1u);
                } else {
                    const uint64_t t0 = global_ns();
                    while (ld_acquire_u32(&a.hdr->bar_gen) == gen0) {
                        if (global_ns() - t0 > MOE_WAIT_LIMIT_NS) {
                            set_status(status, MOE_ERR_TIMEOUT);
                            cs->abort = 1;
                            break;
                        }
                        __nanosleep(64);
                    }
                }
                __threadfence();
            }
            consumer_sync();
        };

        while (true) {
            const bool have = it.valid();
            const Stage st = have ? it.get() : Stage{0, 0, 0, 0};
            if (!arrived && (!have || st.phase == 2)) {
                do_grid_barrier();
                arrived = true;
                staged_u = -1;
            }
            if (!have)
                break;

            const int e = min(max(__ldcg(&a.uniq_list[st.u]), 0), a.E - 1);
            int p0 = __ldcg(&a.offsets[e]);
            int M = __ldcg(&a.offsets[e + 1]) - p0;
            if (p0 < 0 || M < 0 || p0 + M > nslots) {  // inconsistent routing state
                if (tid == 0)
                    set_status(status, MOE_ERR_DEVICE_CHECK);
                p0 = 0;
                M = 0;
            }

            const bool ok = !*(volatile int *)&cs->abort && mbar_wait(&full[slot], ph, status);
            if (!ok)
                cs->abort = 1;

            const int rows = st.phase == 1 ? 2 * st.n : st.n;
            const int rowlen = st.phase == 1 ? d : I;  // elements per row
            const int nvec = rowlen >> 3;
            int S = floor_pow2(max(1, kSC / rows));
            S = min(S, max(1, nvec / 32));
            const int items = rows * S;
            const int vper = (nvec + S - 1) / S;  // vectors per slice
            const uint8_t *stg = ring + (size_t)slot * kStageBytes;

            for (int m0 = 0; m0 < M; m0 += mtc) {
                const int mt = min(mtc, M - m0);
                // stage this expert's token chunk (x for phase 1, h for phase 2)
                if (staged_u != st.u || staged_m0 != m0 || staged_phase != st.phase) {
                    consumer_sync();  // nobody still reads tok_area
                    if (st.phase == 1) {
                        const int vpr = d >> 3;
                        for (int i = tid; i < mt * vpr; i += kSC * 32) {
                            const int m = i / vpr, v = i % vpr;
                            const int slotid = __ldcg(&a.sorted_slot[p0 + m0 + m]);
                            int t = slotid / k1;
                            if (slotid < 0 || t >= a.T) {
                                set_status(status, MOE_ERR_DEVICE_CHECK);
                                t = 0;
                            }
                            reinterpret_cast<uint4 *>(tok_area)[m * vpr + v] =
                                reinterpret_cast<const uint4 *>(a.x + (size_t)t * d)[v];
                        }
                    } else {
                        const int vpr = I >> 2;  // float4 per h row
                        for (int i = tid; i < mt * vpr; i += kSC * 32) {
                            const int m = i / vpr, v = i % vpr;
                            reinterpret_cast<float4 *>(tok_area)[m * vpr + v] = __ldcg(
                                reinterpret_cast<const float4 *>(a.h + (size_t)(p0 + m0 + m) * I) + v);
                        }
                    }
                    consumer_sync();
                    staged_u = st.u;
                    staged_m0 = m0;
                    staged_phase = st.phase;
                }
                float *part = cs->part[iter & 1];
                if (ok) {
                    for (int item = warp; item < items; item += kSC) {
                        const int r = item / S, sl = item % S;
                        const uint4 *wrow =
                            reinterpret_cast<const uint4 *>(stg + (size_t)r * rowlen * 2);
                        float acc[kTokChunk];
#pragma unroll
                        for (int m = 0; m < kTokChunk; ++m)
                            acc[m] = 0.0f;
                        const int vb = sl * vper, ve = min(nvec, vb + vper);
                        for (int v = vb + lane; v < ve; v += 32) {
                            const uint4 wv = wrow[v];
                            if (st.phase == 1) {
#pragma unroll
                                for (int m = 0; m < kTokChunk; ++m) {
                                    if (m < mt) {
                                        const uint4 xv =
                                            reinterpret_cast<const uint4 *>(tok_area)[m * nvec + v];
                                        float xf[8] = {bf16lo(xv.x), bf16hi(xv.x), bf16lo(xv.y),
                                                       bf16hi(xv.y), bf16lo(xv.z), bf16hi(xv.z),
                                                       bf16lo(xv.w), bf16hi(xv.w)};
                                        acc[m] = dot8_bf16(wv, xf, acc[m]);
                                    }
                                }
                            } else {
#pragma unroll
                                for (int m = 0; m < kTokChunk; ++m) {
                                    if (m < mt) {
                                        const float4 *hp = reinterpret_cast<const float4 *>(
                                            tok_area + ((size_t)m * I + (size_t)v * 8) * 4);
                                        const float4 h0 = hp[0], h1 = hp[1];
                                        float hf[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
                                        acc[m] = dot8_bf16(wv, hf, acc[m]);
                                    }
                                }
                            }
                        }
#pragma unroll
                        for (int m = 0; m < kTokChunk; ++m) {
                            if (m < mt) {
                                const float s = warp_sum(acc[m]);
                                if (lane == 0)
                                    part[item * kTokChunk + m] = s;
                            }
                        }
                    }
                }
                if (m0 + mtc >= M) {
                    // last read of this stage's weights: hand the slot back
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&empty[slot]);
                }
                consumer_sync();
                if (ok) {
                    if (st.phase == 1) {
                        for (int i = tid; i < st.n * mt; i += kSC * 32) {
                            const int ch = i / mt, m = i % mt;
                            float g = 0.0f, u = 0.0f;
                            for (int sl = 0; sl < S; ++sl) {
                                g += part[((ch)*S + sl) * kTokChunk + m];
                                u += part[((st.n + ch) * S + sl) * kTokChunk + m];
                            }
                            a.h[(size_t)(p0 + m0 + m) * I + st.c + ch] = silu_mul(g, u);
                        }
                    } else {
                        for (int i = tid; i < st.n * mt; i += kSC * 32) {
                            const int r = i / mt, m = i % mt;
                            float o = 0.0f;
                            for (int sl = 0; sl < S; ++sl)
                                o += part[(r * S + sl) * kTokChunk + m];
                            a.out[(size_t)(p0 + m0 + m) * d + st.c + r] = o;
                        }
                    }
                }
                ++iter;
            }
            if (M == 0) {  // cannot happen for an activated expert; keep the ring moving
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&empty[slot]);
            }
            it.next();
            if (++slot == kStages) {
                slot = 0;
                ph ^= 1u;
            }
        }

        // ------------------------------------------------------------ combine
        if (a.y) {
            consumer_sync();  // every out[] row of this CTA is written
            const int r_lo = (int)((int64_t)d * b / G), r_hi = (int)((int64_t)d * (b + 1) / G);
            const int nr = r_hi - r_lo;
            for (int i = tid; i < a.T * nr; i += kSC * 32) {
                const int t = i / nr, r = r_lo + i % nr;
                float acc = 0.0f;
                for (int s = 0; s < k1; ++s) {
                    const int pos = __ldcg(&a.slot_pos[t * k1 + s]);
                    if (pos < 0 || pos >= nslots) {
                        set_status(status, MOE_ERR_DEVICE_CHECK);
                        continue;
                    }
                    const float prod = __ldcg(&a.topk_w[t * k1 + s]) * a.out[(size_t)pos * d + r];
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
    if (tid == 0 && cs->abort) {
        const int issued = cs->issued;
        for (int s = 0; s < kStages && s < issued; ++s) {
            const int last = issued - 1 - ((issued - 1 - s) % kStages);  // last stage on slot s
            const uint32_t parity = (uint32_t)((last / kStages) & 1);
            mbar_wait(&full[s], parity, status);
        }
    }
}

size_t stream_smem_bytes(int d, int I)
{
    const size_t tok = (size_t)tok_chunk(d, I) * (size_t)(d * 2 > I * 4 ? d * 2 : I * 4);
    return (size_t)kStages * kStageBytes + 2 * kStages * sizeof(uint64_t) + sizeof(ConsumerSmem) +
           16 + tok;
}

}  // namespace moe
