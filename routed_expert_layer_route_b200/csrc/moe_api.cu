// moe_api.cu -- the C ABI of libmoe.so (declared in include/moe.h): argument
// checks, workspace layout and kernel launches.  All work is enqueued on the
// caller's stream; consecutive kernels are chained with programmatic
// dependent launch so each kernel's prologue (and the router's weight
// prefetch) overlaps the tail of the previous one.  Every kernel waits
// (griddepcontrol.wait) before it touches data written by earlier work.
#include <cuda_runtime.h>

#include <mutex>
#include <utility>

#include "../../include/moe.h"
#include "../../include/moe_testing.h"
#include "combine.cuh"
#include "ctopk.cuh"
#include "decode.cuh"
#include "decode_mt.cuh"
#include "gemm_pair.cuh"
#include "grouped.cuh"
#include "route.cuh"
#include "stream.cuh"

namespace moe {

// ------------------------------------------------------------------ limits
constexpr int kMaxE = 1024;
constexpr int kMaxK1 = 32;
constexpr int kMinD = 64, kMaxD = 8192;
constexpr int kMinI = 16, kMaxI = 8192;
constexpr int kMaxT = 1 << 20;

static inline size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

struct WsLayout {
    size_t logits, idx, w, offsets, sorted_slot, slot_pos, uniq_count, uniq_list, h, out, y_acc,
        hist, ctk, dyacc, total;
};

static inline int perm_chunks(int T) { return (T + kPermTok - 1) / kPermTok; }

static WsLayout ws_layout(int T, int d, int E, int I, int k1)
{
    WsLayout L;
    size_t o = sizeof(WsHeader);
    const size_t n = (size_t)T * k1;
    // the decode kernels' accumulator (kMtMaxT tokens, kept zero between
    // calls), first after the header: the same place for every T
    L.dyacc = o;       o = align256(o + sizeof(float) * (size_t)kMtMaxT * d);
    L.logits = o;      o = align256(o + sizeof(float) * (size_t)T * E);
    L.idx = o;         o = align256(o + sizeof(int32_t) * n);
    L.w = o;           o = align256(o + sizeof(float) * n);
    L.offsets = o;     o = align256(o + sizeof(int32_t) * (size_t)(E + 1));
    L.sorted_slot = o; o = align256(o + sizeof(int32_t) * n);
    L.slot_pos = o;    o = align256(o + sizeof(int32_t) * n);
    L.uniq_count = o;  o = align256(o + sizeof(int32_t));
    L.uniq_list = o;   o = align256(o + sizeof(int32_t) * (size_t)E);
    L.h = o;           o = align256(o + sizeof(float) * n * (size_t)I);
    L.out = o;         o = align256(o + sizeof(float) * n * (size_t)d);
    L.y_acc = o;       o = align256(o + sizeof(float) * (size_t)T * d);
    L.hist = o;        o = align256(o + sizeof(int32_t) * (size_t)perm_chunks(T) * E);
    L.ctk = o;         o = align256(o + 2 * sizeof(float) * (size_t)k1 * I);  // one token's h, scores
    L.total = o;
    return L;
}

template <typename P>
static inline P *at(void *ws, size_t off)
{
    return reinterpret_cast<P *>(reinterpret_cast<char *>(ws) + off);
}

static inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

static int check_shape(int T, int d, int E, int I, int k1)
{
    if (T < 0 || T > kMaxT)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (E < 1 || E > kMaxE)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (d < kMinD || d > kMaxD || d % 64)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (I < kMinI || I > kMaxI || I % 16)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (k1 < 1 || k1 > kMaxK1 || k1 > E)
        return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

static int check_route(int E, int k1, int k2)
{
    if (E < 1 || E > kMaxE)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (k1 < 1 || k1 > kMaxK1 || k1 > E || k2 < k1)
        return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

// ------------------------------------------------------------------ device info
struct DevInfo {
    bool ready = false;
    int num_sms = 0;
    int gemm1_pairs = 0;  // CTA pairs of k_gemm1_pair resident at once (0: not launchable)
};

// Which grouped GEMM kernels the grouped path uses (test hook): 0 the pair
// kernel for the gate/up GEMM where the shapes allow it, 1 always the
// single-CTA kernels.
static int g_grouped_single = 0;

// CTA pairs of a pair kernel the device holds at once (0: not launchable).
template <typename K>
static int pair_occupancy(K kern, int threads, size_t smem, int num_sms)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (num_sms / 2));
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute at;
    at.id = cudaLaunchAttributeClusterDimension;
    at.val.clusterDim.x = 2;
    at.val.clusterDim.y = 1;
    at.val.clusterDim.z = 1;
    cfg.attrs = &at;
    cfg.numAttrs = 1;
    int nc = 0;
    if (cudaOccupancyMaxActiveClusters(&nc, kern, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return nc < num_sms / 2 ? nc : num_sms / 2;
}
static DevInfo g_dev[64];
static std::mutex g_dev_mu;

static int device_info(DevInfo *&out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_dev_mu);
    DevInfo &di = g_dev[dev];
    if (!di.ready) {
        if (cudaDeviceGetAttribute(&di.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return MOE_ERR_CUDA;
        const int stream_smem = (int)stream_smem_bytes();
        if (cudaFuncSetAttribute(k_stream<0, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 stream_smem) != cudaSuccess ||
            cudaFuncSetAttribute(k_stream<8, 3>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 stream_smem) != cudaSuccess ||
            cudaFuncSetAttribute(k_stream<16, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 stream_smem) != cudaSuccess)
            return MOE_ERR_CUDA;
        const int decode_smem = 227 * 1024;
        const cudaFuncAttribute dsm = cudaFuncAttributeMaxDynamicSharedMemorySize;
        if (cudaFuncSetAttribute(k_decode<0, false>, dsm, decode_smem) != cudaSuccess ||
            cudaFuncSetAttribute(k_decode<8, false>, dsm, decode_smem) != cudaSuccess ||
            cudaFuncSetAttribute(k_decode<16, false>, dsm, decode_smem) != cudaSuccess ||
            cudaFuncSetAttribute(k_decode<0, true>, dsm, decode_smem) != cudaSuccess ||
            cudaFuncSetAttribute(k_decode<8, true>, dsm, decode_smem) != cudaSuccess ||
            cudaFuncSetAttribute(k_decode<16, true>, dsm, decode_smem) != cudaSuccess ||
            cudaFuncSetAttribute(k_decode_mt<2, 1>, dsm, decode_smem) != cudaSuccess ||
            cudaFuncSetAttribute(k_decode_mt<4, 1>, dsm, decode_smem) != cudaSuccess ||
            cudaFuncSetAttribute(k_decode_mt<8, 1>, dsm, decode_smem) != cudaSuccess ||
            cudaFuncSetAttribute(k_decode_mt<2, 2>, dsm, decode_smem) != cudaSuccess ||
            cudaFuncSetAttribute(k_decode_mt<4, 2>, dsm, decode_smem) != cudaSuccess)
            return MOE_ERR_CUDA;
        if (cudaFuncSetAttribute(k_gemm1, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)gemm1_smem_bytes()) != cudaSuccess ||
            cudaFuncSetAttribute(k_gemm2, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)gemm2_smem_bytes()) != cudaSuccess ||
            cudaFuncSetAttribute(k_gemm1_pair, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)gemm1_pair_smem_bytes()) != cudaSuccess)
            return MOE_ERR_CUDA;
        di.gemm1_pairs = pair_occupancy(k_gemm1_pair, kGP1Threads, gemm1_pair_smem_bytes(),
                                        di.num_sms);
        // scores of kCtkMaxN channels + at most 16 KiB of side-by-side row partials
        if (cudaFuncSetAttribute(k_ctk_down, dsm, kCtkMaxN * 4 + 16 * 1024) != cudaSuccess)
            return MOE_ERR_CUDA;
        const int small = 96 * 1024;
        if (cudaFuncSetAttribute(k_logits, cudaFuncAttributeMaxDynamicSharedMemorySize, small) !=
                cudaSuccess ||
            cudaFuncSetAttribute(k_topk, cudaFuncAttributeMaxDynamicSharedMemorySize, small) !=
                cudaSuccess ||
            cudaFuncSetAttribute(k_permute, cudaFuncAttributeMaxDynamicSharedMemorySize, small) !=
                cudaSuccess)
            return MOE_ERR_CUDA;
        di.ready = true;
    }
    out = &di;
    return MOE_OK;
}

// ------------------------------------------------------------------ launch
// Launch options: kPdl chains the kernel to the previous one on the stream by
// programmatic dependent launch (the kernel calls griddepcontrol.wait before
// it reads anything an earlier kernel wrote); kCoop makes it a cooperative
// launch, which the runtime places only when every CTA of the grid can be
// resident at once (kernels whose CTAs wait on one another need that);
// kPair launches clusters of two CTAs (the pair kernels).
constexpr int kPdl = 1, kCoop = 2, kPair = 4;

template <typename... KArgs, typename... Args>
static int launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                  int opts, Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[3];
    int n = 0;
    if (opts & kPdl) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    if (opts & kCoop) {
        attr[n].id = cudaLaunchAttributeCooperative;
        attr[n].val.cooperative = 1;
        ++n;
    }
    if (opts & kPair) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = 2;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = n ? attr : nullptr;
    cfg.numAttrs = n;
    const cudaError_t err = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
    return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

static int topk_threads(int E)
{
    int t = ((E + 31) / 32) * 32;
    if (t < 128)
        t = 128;
    if (t > 1024)
        t = 1024;
    return t;
}

// logits for T tokens (no routing tail)
static int enqueue_logits(const void *x, const void *wr, const float *bias, float *z, float *z_copy,
                          int T, int d, int E, cudaStream_t s, float4 *zero = nullptr,
                          int zero_n4 = 0)
{
    LogitsArgs a = {};
    a.x = static_cast<const uint16_t *>(x);
    a.wr = static_cast<const uint16_t *>(wr);
    a.bias = bias;
    a.z = z;
    a.z_copy = z_copy;
    a.T = T;
    a.d = d;
    a.E = E;
    a.zero = zero;
    a.zero_n4 = zero_n4;
    const int items = E * ((T + kLogitsTok - 1) / kLogitsTok);
    const int grid = (items + kLogitsWarps - 1) / kLogitsWarps;
    return launch(k_logits, dim3(grid), dim3(kLogitsWarps * 32), 0, s, true, a);
}

// The single-pass decode path of moe_layer (T == 1, down matrix
// channel-major): one kernel -- router logits, routing, gate/up, down
// partials into y_acc, y written by its last CTA.
static int enqueue_decode(const void *x, const void *wr, const float *bias, float *logits_out,
                          const void *wg, const void *wu, const void *wdt, int d,
                          int E, int I, int k1, int k2, void *y, int y_dtype, int32_t *idx_copy,
                          float *w_copy, void *ws, int G, cudaStream_t s, VarK vk = VarK(),
                          int32_t *count = nullptr)
{
    const WsLayout L = ws_layout(1, d, E, I, k1);
    DecodeArgs a = {};
    a.x = static_cast<const uint16_t *>(x);
    a.wg = static_cast<const uint16_t *>(wg);
    a.wu = static_cast<const uint16_t *>(wu);
    a.wdt = static_cast<const uint16_t *>(wdt);
    a.d = d;
    a.E = E;
    a.I = I;
    a.k1 = k1;
    a.k2 = k2;
    a.wr = static_cast<const uint16_t *>(wr);
    a.bias = bias;
    a.logits_out = logits_out;
    a.logits = at<float>(ws, L.logits);
    a.topk_idx = at<int32_t>(ws, L.idx);
    a.topk_w = at<float>(ws, L.w);
    a.idx_copy = idx_copy;
    a.w_copy = w_copy;
    a.offsets = at<int32_t>(ws, L.offsets);
    a.sorted_slot = at<int32_t>(ws, L.sorted_slot);
    a.slot_pos = at<int32_t>(ws, L.slot_pos);
    a.uniq_count = at<int32_t>(ws, L.uniq_count);
    a.uniq_list = at<int32_t>(ws, L.uniq_list);
    a.yacc = at<float>(ws, L.dyacc);
    a.y = y;
    a.y_dtype = y_dtype;
    a.vk = vk;
    a.count = count;
    a.rrows = decode_router_rows(d, E, G);
    a.hdr = static_cast<WsHeader *>(ws);
    const size_t smem = decode_smem_bytes(d);
    const dim3 grid(G), block(kSThreads);
    if (vk.kind != kVarFixed) {
        if (d == 2048)
            return launch(k_decode<8, true>, grid, block, smem, s, kPdl | kCoop, a);
        if (d == 4096)
            return launch(k_decode<16, true>, grid, block, smem, s, kPdl | kCoop, a);
        return launch(k_decode<0, true>, grid, block, smem, s, kPdl | kCoop, a);
    }
    if (d == 2048)
        return launch(k_decode<8, false>, grid, block, smem, s, kPdl | kCoop, a);
    if (d == 4096)
        return launch(k_decode<16, false>, grid, block, smem, s, kPdl | kCoop, a);
    return launch(k_decode<0, false>, grid, block, smem, s, kPdl | kCoop, a);
}

// The few-token decode path of moe_layer (2 <= T <= 8, down matrix
// channel-major): one kernel -- router logits, routing, the union of the
// routed experts streamed once, per-token partials into y_acc, y written by
// its last CTA.
static int enqueue_decode_mt(const void *x, const void *wr, const float *bias, float *logits_out,
                             const void *wg, const void *wu, const void *wdt, int T, int d, int E,
                             int I, int k1, int k2, void *y, int y_dtype, int32_t *idx_copy,
                             float *w_copy, void *ws, int G, cudaStream_t s, VarK vk,
                             int32_t *count)
{
    const WsLayout L = ws_layout(T, d, E, I, k1);
    const MtLayout ML = mt_layout(T, d);
    MtArgs a = {};
    a.x = static_cast<const uint16_t *>(x);
    a.wg = static_cast<const uint16_t *>(wg);
    a.wu = static_cast<const uint16_t *>(wu);
    a.wdt = static_cast<const uint16_t *>(wdt);
    a.wr = static_cast<const uint16_t *>(wr);
    a.bias = bias;
    a.logits = at<float>(ws, L.logits);
    a.logits_out = logits_out;
    a.topk_idx = at<int32_t>(ws, L.idx);
    a.topk_w = at<float>(ws, L.w);
    a.idx_copy = idx_copy;
    a.w_copy = w_copy;
    a.count = count;
    a.yacc = at<float>(ws, L.dyacc);
    a.y = y;
    a.y_dtype = y_dtype;
    a.T = T;
    a.d = d;
    a.E = E;
    a.I = I;
    a.k1 = k1;
    a.k2 = k2;
    a.rrows = mt_router_rows(E, G);
    a.nslots = ML.nslots;
    a.vk = vk;
    a.hdr = static_cast<WsHeader *>(ws);
    int TM, RVM;
    mt_shape(T, d, TM, RVM);
    const dim3 grid(G), block(kMtThreads);
    const int opts = kPdl | kCoop;
    if (RVM == 1) {
        if (TM == 2)
            return launch(k_decode_mt<2, 1>, grid, block, ML.total, s, opts, a);
        if (TM == 4)
            return launch(k_decode_mt<4, 1>, grid, block, ML.total, s, opts, a);
        return launch(k_decode_mt<8, 1>, grid, block, ML.total, s, opts, a);
    }
    if (TM == 2)
        return launch(k_decode_mt<2, 2>, grid, block, ML.total, s, opts, a);
    return launch(k_decode_mt<4, 2>, grid, block, ML.total, s, opts, a);
}

// ------------------------------------------------------------------ grouped GEMM path
// cuTensorMapEncodeTiled from the driver, looked up once through the runtime
// (no link-time dependence on the driver library).
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_tiled_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Row-major bf16 matrix [rows x inner] read in boxes of 64 inner values x
// box_rows rows, 128-byte swizzle (the K-major operand layout of the MMAs).
static int bf16_tile_map(CUtensorMap *m, const void *base, uint64_t inner, uint64_t rows,
                         uint32_t box_rows)
{
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc)
        return MOE_ERR_CUDA;
    const cuuint64_t dims[2] = {inner, rows};
    const cuuint64_t strides[1] = {inner * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kGBK, box_rows};
    const cuuint32_t es[2] = {1, 1};
    const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                           strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

// The two grouped GEMMs over routed slots already grouped by expert
// (offsets / sorted_slot).  combine: weighted red.add into y_acc (zeroed
// before); otherwise per-slot rows of `out` in sorted order.
// which: 4 gathers the token rows into expert order (xs), 1 runs the gate/up
// GEMM, 2 the down GEMM (7: the whole expert FFN).
static int enqueue_grouped(const void *x, const void *wg, const void *wu, const void *wd, int T,
                           int d, int E, int I, int k1, const int32_t *offsets,
                           const int32_t *sorted_slot, const float *topk_w, uint16_t *xs,
                           uint16_t *h, float *y_acc, float *out, WsHeader *hdr, int G,
                           cudaStream_t s, int which = 7, bool pdl = true)
{
    CUtensorMap tg, tu, tx, td, th;
    int rc;
    const uint64_t n = (uint64_t)T * k1;
    if ((rc = bf16_tile_map(&tg, wg, d, (uint64_t)E * I, kGBM)) != MOE_OK ||
        (rc = bf16_tile_map(&tu, wu, d, (uint64_t)E * I, kGBM)) != MOE_OK ||
        (rc = bf16_tile_map(&tx, xs, d, n, 64)) != MOE_OK ||
        (rc = bf16_tile_map(&td, wd, I, (uint64_t)E * d, kGBM)) != MOE_OK ||
        (rc = bf16_tile_map(&th, h, I, n, 64)) != MOE_OK)
        return rc;
    if (which & 4) {
        const int rows = (int)n;
        const int grid = (rows + 7) / 8 < 8 * G ? (rows + 7) / 8 : 8 * G;
        if ((rc = launch(k_gather_rows, dim3(grid), dim3(256), 0, s, pdl,
                         static_cast<const uint16_t *>(x), sorted_slot, offsets, E, rows, d, k1,
                         xs, reinterpret_cast<float4 *>(y_acc), y_acc ? T * d / 4 : 0,
                         &hdr->status)) != MOE_OK)
            return rc;
    }
    Gemm1Args a1 = {};
    a1.offsets = offsets;
    a1.sorted_slot = sorted_slot;
    a1.h = h;
    a1.sched = {&hdr->sched[0], &hdr->sched[1]};
    a1.T = T;
    a1.d = d;
    a1.E = E;
    a1.I = I;
    a1.k1 = k1;
    a1.hdr = hdr;
    DevInfo *di;
    if ((rc = device_info(di)) != MOE_OK)
        return rc;
    if (which & 1) {
        // the pair kernel when the weight rows come in whole 256-row tiles
        if (I % kGPRows == 0 && di->gemm1_pairs > 0 && !g_grouped_single)
            rc = launch(k_gemm1_pair, dim3(2 * di->gemm1_pairs), dim3(kGP1Threads),
                        gemm1_pair_smem_bytes(), s, (pdl ? kPdl : 0) | kPair, tg, tu, tx, a1);
        else
            rc = launch(k_gemm1, dim3(G), dim3(kG1Threads), gemm1_smem_bytes(), s, pdl, tg, tu,
                        tx, a1);
        if (rc != MOE_OK)
            return rc;
    }
    if (!(which & 2))
        return MOE_OK;
    Gemm2Args a2 = {};
    a2.offsets = offsets;
    a2.sorted_slot = sorted_slot;
    a2.topk_w = topk_w;
    a2.y_acc = y_acc;
    a2.out = out;
    a2.T = T;
    a2.d = d;
    a2.E = E;
    a2.I = I;
    a2.k1 = k1;
    a2.combine = y_acc != nullptr;
    a2.sched = {&hdr->sched[2], &hdr->sched[3]};
    a2.hdr = hdr;
    return launch(k_gemm2, dim3(G), dim3(kG2Threads), gemm2_smem_bytes(), s, pdl, td, th, a2);
}

// Router logits of a large batch as a tensor-core GEMM (the down-GEMM kernel
// with W_r as the weight matrix, the tokens in order as one group, bias added
// in the epilogue): needs whole 128-row tiles of experts.
static bool gemm_logits_ok(int T, int d, int E) { return E % kGBM == 0 && E <= kGMaxE && T >= 256; }

static int enqueue_logits_gemm(const void *x, const void *wr, const float *bias, float *z,
                               float *z_copy, int T, int d, int E, WsHeader *hdr, int G,
                               cudaStream_t s)
{
    CUtensorMap tw, tx;
    int rc;
    if ((rc = bf16_tile_map(&tw, wr, d, E, kGBM)) != MOE_OK ||
        (rc = bf16_tile_map(&tx, x, d, T, 64)) != MOE_OK)
        return rc;
    Gemm2Args a = {};
    a.out = z;
    a.out_copy = z_copy;
    a.bias = bias;
    a.single_n = T;
    a.bn = 64;  // 64-token tiles: enough work items to spread over the SMs
    a.T = T;
    a.d = E;  // output rows: the experts
    a.I = d;  // K: the hidden size
    a.E = 1;  // one group: every token
    a.k1 = 1;
    a.combine = 0;
    a.sched = {&hdr->sched[4], &hdr->sched[5]};
    a.hdr = hdr;
    return launch(k_gemm2, dim3(G), dim3(kG2Threads), gemm2_smem_bytes(), s, true, tw, tx, a);
}

// Warp-per-token routing of T tokens from float32 logits.
static int enqueue_route_warp(const float *z, int T, int E, int k1, int k2, int32_t *idx, float *w,
                              int32_t *idx_copy, float *w_copy, cudaStream_t s,
                              VarK vk = VarK(), int32_t *count = nullptr)
{
    const dim3 grid((T + 7) / 8), block(256);
#define MOE_ROUTE_WARP(R)                                                                        \
    return launch(k_route_warp<R>, grid, block, 0, s, true, z, T, E, k1, k2, idx, w, idx_copy, \
                  w_copy, vk, count)
    if (E <= 32) MOE_ROUTE_WARP(1);
    if (E <= 64) MOE_ROUTE_WARP(2);
    if (E <= 128) MOE_ROUTE_WARP(4);
    if (E <= 256) MOE_ROUTE_WARP(8);
    if (E <= 512) MOE_ROUTE_WARP(16);
    MOE_ROUTE_WARP(32);
#undef MOE_ROUTE_WARP
}

// Stable counting sort of T*k1 slots over chunks of kPermTok tokens (no
// unique-expert list); hist: perm_chunks(T) x E ints of scratch.
static int enqueue_perm_parallel(const int32_t *idx, int T, int k1, int E, int *hist, PermOut po,
                                 int *status, cudaStream_t s)
{
    const int nch = perm_chunks(T);
    int rc;
    if ((rc = launch(k_perm_hist, dim3(nch), dim3(256), perm_hist_smem_bytes(E, k1), s, true, idx,
                     T, k1, E, hist, status)) != MOE_OK)
        return rc;
    return launch(k_perm_scatter, dim3(nch), dim3(256), perm_scatter_smem_bytes(E, k1), s, true,
                  idx, T, k1, E, (const int *)hist, po);
}

// AUTO's choice of the tensor-core path: every batch of two or more tokens
// whose weights fill whole 128-row tiles (measured on B200 it beats the
// CUDA-core streaming kernel from T = 4 up: 58 vs 68 us per layer at d = 2048,
// E = 128, I = 768, k1 = 4, and 162 vs 872 us at T = 64).
static bool auto_grouped(int T, int d, int E, int I, int k1)
{
    (void)k1;
    (void)E;
    return grouped_fits(d, E, I) && T >= 2;
}

}  // namespace moe

using namespace moe;

// ========================================================================== ABI
extern "C" {

const char *moe_status_string(int status)
{
    switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_TIMEOUT: return "device wait timed out";
    case MOE_ERR_DEVICE_CHECK: return "device-side check failed";
    case MOE_ERR_SCRATCH_LIMIT:
        return "shapes exceed the fixed scratch of moe_expert_ffn_noalloc (T*k1*I > 1047424)";
    default: return "unknown status";
    }
}

int moe_version(void) { return 10000; }

size_t moe_workspace_size(int T, int d, int E, int I, int k1)
{
    if (check_shape(T, d, E, I, k1) != MOE_OK)
        return 0;
    return ws_layout(T, d, E, I, k1).total;
}

int moe_workspace_init(void *ws, size_t ws_bytes, void *stream)
{
    if (!ws || ws_bytes < sizeof(WsHeader) || (reinterpret_cast<uintptr_t>(ws) & 255))
        return MOE_ERR_INVALID_ARG;
    // all of it: the header's counters and the accumulators that kernels keep
    // zero between calls
    return cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

int moe_read_device_status(void *ws, int *status_out, void *stream)
{
    if (!ws || !status_out)
        return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int v = 0;
    if (cudaMemcpyAsync(&v, ws, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (cudaMemsetAsync(ws, 0, sizeof(int), s) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess)
        return MOE_ERR_CUDA;
    *status_out = v;
    return MOE_OK;
}

}  // extern "C" (route_impl below is internal)

static int route_impl(const void *x_bf16, const void *w_router_bf16, const float *bias,
                      float *logits, int T, int d, int E, int k1, int k2, int32_t *topk_idx,
                      float *topk_w, void *ws, size_t ws_bytes, void *stream, VarK vk,
                      int32_t *count)
{
    int rc = check_route(E, k1, k2);
    if (rc != MOE_OK)
        return rc;
    if (T < 0 || T > kMaxT)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!topk_idx || !topk_w)
        return MOE_ERR_INVALID_ARG;
    if (!x_bf16 && !logits)
        return MOE_ERR_INVALID_ARG;
    if (x_bf16) {
        if (!w_router_bf16)
            return MOE_ERR_INVALID_ARG;
        if (d < kMinD || d > kMaxD || d % 64)
            return MOE_ERR_UNSUPPORTED_SHAPE;
        if (!aligned16(x_bf16) || !aligned16(w_router_bf16))
            return MOE_ERR_INVALID_ARG;
        if (!logits) {
            if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255))
                return MOE_ERR_INVALID_ARG;
            const size_t need = sizeof(WsHeader) + align256(sizeof(float) * (size_t)T * E);
            if (ws_bytes < need)
                return MOE_ERR_WORKSPACE_TOO_SMALL;
        }
    }
    if (ws && ws_bytes < sizeof(WsHeader))
        return MOE_ERR_WORKSPACE_TOO_SMALL;
    if (T == 0)
        return MOE_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    DevInfo *di;
    if ((rc = device_info(di)) != MOE_OK)
        return rc;
    const float *z = logits;
    if (x_bf16) {
        float *zbuf = logits ? logits : at<float>(ws, sizeof(WsHeader));
        if ((rc = enqueue_logits(x_bf16, w_router_bf16, bias, zbuf, nullptr, T, d, E, s)) != MOE_OK)
            return rc;
        z = zbuf;
    }
    return enqueue_route_warp(z, T, E, k1, k2, topk_idx, topk_w, nullptr, nullptr, s, vk, count);
}

extern "C" {

int moe_route(const void *x_bf16, const void *w_router_bf16, const float *bias, float *logits,
              int T, int d, int E, int k1, int k2, int32_t *topk_idx, float *topk_w, void *ws,
              size_t ws_bytes, void *stream)
{
    return route_impl(x_bf16, w_router_bf16, bias, logits, T, d, E, k1, k2, topk_idx, topk_w, ws,
                      ws_bytes, stream, VarK(), nullptr);
}

int moe_route_cascade(const void *x_bf16, const void *w_router_bf16, const float *bias,
                      float *logits, int T, int d, int E, int k1, int k2, float tau,
                      int32_t *topk_idx, float *topk_w, int32_t *topk_count, void *ws,
                      size_t ws_bytes, void *stream)
{
    if (tau != tau)
        return MOE_ERR_INVALID_ARG;  // NaN
    VarK vk = {};
    vk.kind = kVarCascade;
    vk.tau = tau;
    return route_impl(x_bf16, w_router_bf16, bias, logits, T, d, E, k1, k2, topk_idx, topk_w, ws,
                      ws_bytes, stream, vk, topk_count);
}

// The skip rule's arguments: a 16-byte aligned table and two thresholds, not NaN.
static int skip_args(const float *tab, float th_e, float th_w, VarK &vk)
{
    if (!tab || !aligned16(tab) || th_e != th_e || th_w != th_w)
        return MOE_ERR_INVALID_ARG;
    vk = {};
    vk.kind = kVarSkip;
    vk.tab = tab;
    vk.th_e = th_e;
    vk.th_w = th_w;
    return MOE_OK;
}

int moe_route_skip(const void *x_bf16, const void *w_router_bf16, const float *bias,
                   float *logits, int T, int d, int E, int k1, int k2, const float *expert_score,
                   float theta_expert, float theta_weight, int32_t *topk_idx, float *topk_w,
                   int32_t *topk_count, void *ws, size_t ws_bytes, void *stream)
{
    VarK vk;
    const int rc = skip_args(expert_score, theta_expert, theta_weight, vk);
    if (rc != MOE_OK)
        return rc;
    return route_impl(x_bf16, w_router_bf16, bias, logits, T, d, E, k1, k2, topk_idx, topk_w, ws,
                      ws_bytes, stream, vk, topk_count);
}

int moe_permute(const int32_t *topk_idx, int T, int k1, int E, int32_t *expert_offsets,
                int32_t *sorted_slot, int32_t *slot_pos, void *ws, size_t ws_bytes, void *stream)
{
    if (E < 1 || E > kMaxE)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (k1 < 1 || k1 > kMaxK1 || k1 > E)
        return MOE_ERR_INVALID_ARG;
    if (T < 0 || T > kMaxT)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!expert_offsets || (T > 0 && (!topk_idx || !sorted_slot || !slot_pos)))
        return MOE_ERR_INVALID_ARG;
    if (ws && ws_bytes < sizeof(WsHeader))
        return MOE_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    DevInfo *di;
    int rc;
    if ((rc = device_info(di)) != MOE_OK)
        return rc;
    PermOut po = {expert_offsets, sorted_slot, slot_pos, nullptr, nullptr};
    int *status = ws ? &static_cast<WsHeader *>(ws)->status : nullptr;
    // many slots and room for the chunk counts after the header: chunked kernels
    const size_t hist_bytes = sizeof(int) * (size_t)perm_chunks(T) * E;
    if ((long)T * k1 > 4096 && ws && ws_bytes >= sizeof(WsHeader) + hist_bytes)
        return enqueue_perm_parallel(topk_idx, T, k1, E, at<int>(ws, sizeof(WsHeader)), po, status,
                                     s);
    return launch(k_permute, dim3(1), dim3(1024), permute_smem_bytes(E, T), s, true, topk_idx, T,
                  k1, E, po, status);
}

struct StreamCall {
    const void *x, *wg, *wu, *wd;
    int T, d, E, I, k1, k2;
    int route_in_kernel;
    const float *logits;
    int32_t *topk_idx;
    float *topk_w;
    int32_t *idx_copy;
    float *w_copy;
    int32_t *offsets, *sorted_slot, *slot_pos, *uniq_count, *uniq_list;
    float *h, *out;
    void *y;
    int y_dtype;
    WsHeader *hdr;
};

static int enqueue_stream(const StreamCall &c, cudaStream_t s, bool pdl = true)
{
    DevInfo *di;
    int rc;
    if ((rc = device_info(di)) != MOE_OK)
        return rc;
    StreamArgs a = {};
    a.x = static_cast<const uint16_t *>(c.x);
    a.wg = static_cast<const uint16_t *>(c.wg);
    a.wu = static_cast<const uint16_t *>(c.wu);
    a.wd = static_cast<const uint16_t *>(c.wd);
    a.T = c.T;
    a.d = c.d;
    a.E = c.E;
    a.I = c.I;
    a.k1 = c.k1;
    a.k2 = c.k2;
    a.route_in_kernel = c.route_in_kernel;
    a.logits = c.logits;
    a.topk_idx = c.topk_idx;
    a.topk_w = c.topk_w;
    a.idx_copy = c.idx_copy;
    a.w_copy = c.w_copy;
    a.offsets = c.offsets;
    a.sorted_slot = c.sorted_slot;
    a.slot_pos = c.slot_pos;
    a.uniq_count = c.uniq_count;
    a.uniq_list = c.uniq_list;
    a.h = c.h;
    a.out = c.out;
    a.y = c.y;
    a.y_dtype = c.y_dtype;
    a.hdr = c.hdr;
    // One CTA per SM, and the CTAs meet at a grid-wide barrier between the
    // two phases: the launch is cooperative, so the runtime places the grid
    // only when all of it can be resident at once (else the launch fails
    // instead of the barrier timing out).
    const unsigned grid = (unsigned)(di->num_sms < kMaxGridCtas ? di->num_sms : kMaxGridCtas);
    const int opts = (pdl ? kPdl : 0) | kCoop;
    switch (stream_variant(c.T, c.d, c.I, c.k1)) {
    case 1:
        return launch(k_stream<8, 3>, dim3(grid), dim3(kSThreads), stream_smem_bytes(), s,
                      opts, a);
    case 2:
        return launch(k_stream<16, 4>, dim3(grid), dim3(kSThreads), stream_smem_bytes(), s,
                      opts, a);
    default:
        return launch(k_stream<0, 0>, dim3(grid), dim3(kSThreads), stream_smem_bytes(), s,
                      opts, a);
    }
}

// The streaming call of a moe_layer on workspace ws (routing tables there).
static StreamCall layer_stream_call(const void *x, const void *wg, const void *wu, const void *wd,
                                    int T, int d, int E, int I, int k1, int k2, void *y,
                                    int y_dtype, int32_t *idx_copy, float *w_copy, void *ws)
{
    const WsLayout L = ws_layout(T, d, E, I, k1);
    StreamCall c = {};
    c.x = x;
    c.wg = wg;
    c.wu = wu;
    c.wd = wd;
    c.T = T;
    c.d = d;
    c.E = E;
    c.I = I;
    c.k1 = k1;
    c.k2 = k2;
    c.route_in_kernel = T == 1;
    c.logits = at<float>(ws, L.logits);
    c.topk_idx = at<int32_t>(ws, L.idx);
    c.topk_w = at<float>(ws, L.w);
    c.idx_copy = idx_copy;
    c.w_copy = w_copy;
    c.offsets = at<int32_t>(ws, L.offsets);
    c.sorted_slot = at<int32_t>(ws, L.sorted_slot);
    c.slot_pos = at<int32_t>(ws, L.slot_pos);
    c.uniq_count = at<int32_t>(ws, L.uniq_count);
    c.uniq_list = at<int32_t>(ws, L.uniq_list);
    c.h = at<float>(ws, L.h);
    c.out = at<float>(ws, L.out);
    c.y = y;
    c.y_dtype = y_dtype;
    c.hdr = static_cast<WsHeader *>(ws);
    return c;
}

int moe_expert_ffn(const void *x_bf16, const int32_t *expert_offsets, const int32_t *sorted_slot,
                   const void *w_gate_bf16, const void *w_up_bf16, const void *w_down_bf16, int T,
                   int d, int E, int I, int k1, float *out, int flags, void *ws, size_t ws_bytes,
                   void *stream)
{
    int rc = check_shape(T, d, E, I, k1);
    if (rc != MOE_OK)
        return rc;
    if (flags < MOE_PATH_AUTO || flags > MOE_PATH_GROUPED)
        return MOE_ERR_INVALID_ARG;
    if (T == 0)
        return MOE_OK;
    if (!x_bf16 || !expert_offsets || !sorted_slot || !w_gate_bf16 || !w_up_bf16 ||
        !w_down_bf16 || !out || !ws)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x_bf16) || !aligned16(w_gate_bf16) || !aligned16(w_up_bf16) ||
        !aligned16(w_down_bf16) || !aligned16(out) || (reinterpret_cast<uintptr_t>(ws) & 255))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(T, d, E, I, k1);
    if (ws_bytes < L.total)
        return MOE_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    DevInfo *di;
    if ((rc = device_info(di)) != MOE_OK)
        return rc;
    const bool grouped = flags == MOE_PATH_GROUPED || (flags == MOE_PATH_AUTO && auto_grouped(T, d, E, I, k1));
    if (grouped) {
        if (!grouped_fits(d, E, I))
            return MOE_ERR_UNSUPPORTED_SHAPE;
        return enqueue_grouped(x_bf16, w_gate_bf16, w_up_bf16, w_down_bf16, T, d, E, I, k1,
                               expert_offsets, sorted_slot, nullptr, at<uint16_t>(ws, L.out),
                               at<uint16_t>(ws, L.h), nullptr, out, static_cast<WsHeader *>(ws),
                               di->num_sms, s);
    }
    if ((rc = launch(k_uniq_from_offsets, dim3(1), dim3(1024), 0, s, true, expert_offsets, E,
                     at<int32_t>(ws, L.uniq_count), at<int32_t>(ws, L.uniq_list))) != MOE_OK)
        return rc;
    StreamCall c = {};
    c.x = x_bf16;
    c.wg = w_gate_bf16;
    c.wu = w_up_bf16;
    c.wd = w_down_bf16;
    c.T = T;
    c.d = d;
    c.E = E;
    c.I = I;
    c.k1 = k1;
    c.k2 = k1;
    c.offsets = const_cast<int32_t *>(expert_offsets);
    c.sorted_slot = const_cast<int32_t *>(sorted_slot);
    c.uniq_count = at<int32_t>(ws, L.uniq_count);
    c.uniq_list = at<int32_t>(ws, L.uniq_list);
    c.h = at<float>(ws, L.h);
    c.out = out;
    c.hdr = static_cast<WsHeader *>(ws);
    return enqueue_stream(c, s);
}

int moe_combine(const float *expert_out, const int32_t *slot_pos, const float *topk_w, int T,
                int d, int k1, void *y, int y_dtype, void *stream)
{
    if (T < 0 || T > kMaxT || d < kMinD || d > kMaxD || d % 64)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (k1 < 1 || k1 > kMaxK1 || (y_dtype != MOE_DTYPE_F32 && y_dtype != MOE_DTYPE_BF16))
        return MOE_ERR_INVALID_ARG;
    if (T == 0)
        return MOE_OK;
    if (!expert_out || !slot_pos || !topk_w || !y || !aligned16(expert_out) || !aligned16(y))
        return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int per_block = 4 * kCombineThreads;
    return launch(k_combine, dim3((d + per_block - 1) / per_block, T), dim3(kCombineThreads), 0, s,
                  true, expert_out, slot_pos, topk_w, T, d, k1, y, y_dtype, (int *)nullptr);
}

}  // extern "C" (layer_impl below is internal)

static int layer_impl(const void *x_bf16, const void *w_router_bf16, const float *bias,
                      const void *w_gate_bf16, const void *w_up_bf16, const void *w_down_bf16,
                      int T, int d, int E, int I, int k1, int k2, void *y, int y_dtype,
                      int32_t *topk_idx_out, float *topk_w_out, float *logits_out, int flags,
                      void *ws, size_t ws_bytes, void *stream, VarK vk, int32_t *count_out)
{
    const bool cascade = vk.kind != kVarFixed;  // a variable-k route (cascade or skip)
    int rc = check_shape(T, d, E, I, k1);
    if (rc != MOE_OK)
        return rc;
    if ((rc = check_route(E, k1, k2)) != MOE_OK)
        return rc;
    const int path = flags & MOE_PATH_MASK;
    const bool down_cm = (flags & MOE_WDOWN_CHANNEL_MAJOR) != 0;
    if (path > MOE_PATH_DECODE || (flags & ~(MOE_PATH_MASK | MOE_WDOWN_CHANNEL_MAJOR)))
        return MOE_ERR_INVALID_ARG;
    if (path == MOE_PATH_DECODE && !down_cm)
        return MOE_ERR_INVALID_ARG;  // the decode kernel reads the channel-major down matrix
    if (down_cm && path != MOE_PATH_AUTO && path != MOE_PATH_DECODE)
        return MOE_ERR_INVALID_ARG;
    if (y_dtype != MOE_DTYPE_F32 && y_dtype != MOE_DTYPE_BF16)
        return MOE_ERR_INVALID_ARG;
    if (T == 0)
        return MOE_OK;
    if (!x_bf16 || !w_router_bf16 || !w_gate_bf16 || !w_up_bf16 || !w_down_bf16 || !y || !ws)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x_bf16) || !aligned16(w_router_bf16) || !aligned16(w_gate_bf16) ||
        !aligned16(w_up_bf16) || !aligned16(w_down_bf16) || (reinterpret_cast<uintptr_t>(ws) & 255))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(T, d, E, I, k1);
    if (ws_bytes < L.total)
        return MOE_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    DevInfo *di;
    if ((rc = device_info(di)) != MOE_OK)
        return rc;
    WsHeader *hdr = static_cast<WsHeader *>(ws);
    float *z = at<float>(ws, L.logits);
    int32_t *idx = at<int32_t>(ws, L.idx);
    float *w = at<float>(ws, L.w);
    PermOut po = {at<int32_t>(ws, L.offsets), at<int32_t>(ws, L.sorted_slot),
                  at<int32_t>(ws, L.slot_pos), at<int32_t>(ws, L.uniq_count),
                  at<int32_t>(ws, L.uniq_list)};

    const int G = di->num_sms;
    const bool decode = down_cm && decode_fits(T, d, E, I, k1, G);
    const bool decode_mt = down_cm && !decode && mt_fits(T, d, E, I, k1, G);
    if (down_cm && !decode && !decode_mt)
        return MOE_ERR_UNSUPPORTED_SHAPE;  // channel-major down matrix: up to kMtMaxT tokens
    const bool grouped = !down_cm && (path == MOE_PATH_GROUPED ||
                                      (path == MOE_PATH_AUTO && auto_grouped(T, d, E, I, k1)));
    if (grouped && !grouped_fits(d, E, I))
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (cascade && !decode && !decode_mt && !grouped)
        return MOE_ERR_UNSUPPORTED_SHAPE;  // the variable-k route runs on those two paths
    if (grouped) {
        // router logits (tensor-core GEMM when the experts fill 128-row tiles),
        // warp-per-token routing, the chunked stable permutation, the two
        // grouped GEMMs (the first clears y_acc for the second's combine), y
        if (gemm_logits_ok(T, d, E))
            rc = enqueue_logits_gemm(x_bf16, w_router_bf16, bias, z, logits_out, T, d, E, hdr, G, s);
        else
            rc = enqueue_logits(x_bf16, w_router_bf16, bias, z, logits_out, T, d, E, s);
        if (rc != MOE_OK)
            return rc;
        if ((rc = enqueue_route_warp(z, T, E, k1, k2, idx, w, topk_idx_out, topk_w_out, s, vk,
                                     count_out)) != MOE_OK)
            return rc;
        if ((rc = enqueue_perm_parallel(idx, T, k1, E, at<int>(ws, L.hist), po, &hdr->status, s)) !=
            MOE_OK)
            return rc;
        if ((rc = enqueue_grouped(x_bf16, w_gate_bf16, w_up_bf16, w_down_bf16, T, d, E, I, k1,
                                  po.offsets, po.sorted_slot, w, at<uint16_t>(ws, L.out),
                                  at<uint16_t>(ws, L.h), at<float>(ws, L.y_acc), nullptr, hdr, G,
                                  s)) != MOE_OK)
            return rc;
        const int n = T * d;
        return launch(k_finalize, dim3((n / 4 + 255) / 256), dim3(256), 0, s, true,
                      (const float *)at<float>(ws, L.y_acc), n, y, y_dtype);
    }
    if (decode)
        return enqueue_decode(x_bf16, w_router_bf16, bias, logits_out, w_gate_bf16, w_up_bf16,
                              w_down_bf16, d, E, I, k1, k2, y, y_dtype, topk_idx_out, topk_w_out,
                              ws, G, s, vk, count_out);
    if (decode_mt)
        return enqueue_decode_mt(x_bf16, w_router_bf16, bias, logits_out, w_gate_bf16, w_up_bf16,
                                 w_down_bf16, T, d, E, I, k1, k2, y, y_dtype, topk_idx_out,
                                 topk_w_out, ws, G, s, vk, count_out);
    if ((rc = enqueue_logits(x_bf16, w_router_bf16, bias, z, logits_out, T, d, E, s)) != MOE_OK)
        return rc;
    if (T > 1) {
        // one CTA per token ranks its probabilities; the last one to finish
        // builds the permutation tables
        if ((rc = launch(k_topk, dim3(T), dim3(topk_threads(E)), permute_smem_bytes(E, T), s, true,
                         (const float *)z, T, E, k1, k2, idx, w, topk_idx_out, topk_w_out, po,
                         hdr)) != MOE_OK)
            return rc;
    }
    // T == 1: the streaming kernel routes the token itself
    return enqueue_stream(layer_stream_call(x_bf16, w_gate_bf16, w_up_bf16, w_down_bf16, T, d, E, I,
                                            k1, k2, y, y_dtype, topk_idx_out, topk_w_out, ws),
                          s);
}

extern "C" {

int moe_layer(const void *x_bf16, const void *w_router_bf16, const float *bias,
              const void *w_gate_bf16, const void *w_up_bf16, const void *w_down_bf16, int T, int d,
              int E, int I, int k1, int k2, void *y, int y_dtype, int32_t *topk_idx_out,
              float *topk_w_out, float *logits_out, int flags, void *ws, size_t ws_bytes,
              void *stream)
{
    return layer_impl(x_bf16, w_router_bf16, bias, w_gate_bf16, w_up_bf16, w_down_bf16, T, d, E, I,
                      k1, k2, y, y_dtype, topk_idx_out, topk_w_out, logits_out, flags, ws, ws_bytes,
                      stream, VarK(), nullptr);
}

int moe_layer_cascade(const void *x_bf16, const void *w_router_bf16, const float *bias,
                      const void *w_gate_bf16, const void *w_up_bf16, const void *w_down_bf16,
                      int T, int d, int E, int I, int k1, int k2, float tau, void *y, int y_dtype,
                      int32_t *topk_idx_out, float *topk_w_out, int32_t *topk_count_out,
                      float *logits_out, int flags, void *ws, size_t ws_bytes, void *stream)
{
    if (tau != tau)
        return MOE_ERR_INVALID_ARG;  // NaN
    VarK vk = {};
    vk.kind = kVarCascade;
    vk.tau = tau;
    return layer_impl(x_bf16, w_router_bf16, bias, w_gate_bf16, w_up_bf16, w_down_bf16, T, d, E, I,
                      k1, k2, y, y_dtype, topk_idx_out, topk_w_out, logits_out, flags, ws, ws_bytes,
                      stream, vk, topk_count_out);
}

int moe_layer_skip(const void *x_bf16, const void *w_router_bf16, const float *bias,
                   const void *w_gate_bf16, const void *w_up_bf16, const void *w_down_bf16, int T,
                   int d, int E, int I, int k1, int k2, const float *expert_score,
                   float theta_expert, float theta_weight, void *y, int y_dtype,
                   int32_t *topk_idx_out, float *topk_w_out, int32_t *topk_count_out,
                   float *logits_out, int flags, void *ws, size_t ws_bytes, void *stream)
{
    VarK vk;
    const int rc = skip_args(expert_score, theta_expert, theta_weight, vk);
    if (rc != MOE_OK)
        return rc;
    return layer_impl(x_bf16, w_router_bf16, bias, w_gate_bf16, w_up_bf16, w_down_bf16, T, d, E, I,
                      k1, k2, y, y_dtype, topk_idx_out, topk_w_out, logits_out, flags, ws, ws_bytes,
                      stream, vk, topk_count_out);
}

int moe_channel_norms(const void *w_down_bf16, int E, int d, int I, int flags, float *norms,
                      void *stream)
{
    if (E < 1 || E > kMaxE || d < kMinD || d > kMaxD || d % 64 || I < kMinI || I > kMaxI || I % 16)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if ((flags & ~MOE_WDOWN_CHANNEL_MAJOR) || !w_down_bf16 || !norms || !aligned16(w_down_bf16))
        return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const uint16_t *wd = static_cast<const uint16_t *>(w_down_bf16);
    if (flags & MOE_WDOWN_CHANNEL_MAJOR)
        return launch(k_norms_cm, dim3((unsigned)(((long)E * I + 15) / 16)), dim3(512), 0, s, true,
                      wd, E, I, d, norms);
    return launch(k_norms_hf, dim3((I + 255) / 256, E), dim3(256), 0, s, true, wd, E, I, d, norms);
}

int moe_layer_channel_topk(const void *x_bf16, const void *w_router_bf16, const float *bias,
                           const void *w_gate_bf16, const void *w_up_bf16, const void *w_down_cm_bf16,
                           const float *norms, int T, int d, int E, int I, int k1, int k2, int keep,
                           void *y, int y_dtype, int32_t *topk_idx_out, float *topk_w_out,
                           float *logits_out, float *h_out, float *scores_out, int32_t *kept_out,
                           void *ws, size_t ws_bytes, void *stream)
{
    int rc = check_shape(T, d, E, I, k1);
    if (rc != MOE_OK)
        return rc;
    if ((rc = check_route(E, k1, k2)) != MOE_OK)
        return rc;
    const int N = k1 * I;
    if (keep < 1 || keep > N || (y_dtype != MOE_DTYPE_F32 && y_dtype != MOE_DTYPE_BF16))
        return MOE_ERR_INVALID_ARG;
    if (N > kCtkMaxN)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (T == 0)
        return MOE_OK;
    if (!x_bf16 || !w_router_bf16 || !w_gate_bf16 || !w_up_bf16 || !w_down_cm_bf16 || !norms ||
        !y || !ws)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x_bf16) || !aligned16(w_router_bf16) || !aligned16(w_gate_bf16) ||
        !aligned16(w_up_bf16) || !aligned16(w_down_cm_bf16) || !aligned16(y) ||
        (reinterpret_cast<uintptr_t>(ws) & 255))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(T, d, E, I, k1);
    if (ws_bytes < L.total)
        return MOE_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    DevInfo *di;
    if ((rc = device_info(di)) != MOE_OK)
        return rc;
    const int G = di->num_sms;
    if ((keep + G - 1) / G > kCtkMaxMine)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    float *z = at<float>(ws, L.logits);
    float *y_acc = at<float>(ws, L.y_acc);
    if ((rc = enqueue_logits(x_bf16, w_router_bf16, bias, z, logits_out, T, d, E, s,
                             reinterpret_cast<float4 *>(y_acc), T * d / 4)) != MOE_OK)
        return rc;
    const size_t ysz = y_dtype == MOE_DTYPE_BF16 ? 2 : 4;
    for (int t = 0; t < T; ++t) {  // one token after another (two kernels each)
        CtkArgs a = {};
        a.x = static_cast<const uint16_t *>(x_bf16) + (size_t)t * d;
        a.wg = static_cast<const uint16_t *>(w_gate_bf16);
        a.wu = static_cast<const uint16_t *>(w_up_bf16);
        a.wdt = static_cast<const uint16_t *>(w_down_cm_bf16);
        a.norms = norms;
        a.logits = z + (size_t)t * E;
        a.d = d;
        a.E = E;
        a.I = I;
        a.k1 = k1;
        a.k2 = k2;
        a.keep = keep;
        a.topk_idx = at<int32_t>(ws, L.idx) + (size_t)t * k1;
        a.topk_w = at<float>(ws, L.w) + (size_t)t * k1;
        a.idx_copy = topk_idx_out ? topk_idx_out + (size_t)t * k1 : nullptr;
        a.w_copy = topk_w_out ? topk_w_out + (size_t)t * k1 : nullptr;
        a.h = at<float>(ws, L.ctk);
        a.score = a.h + N;
        a.h_copy = h_out ? h_out + (size_t)t * N : nullptr;
        a.score_copy = scores_out ? scores_out + (size_t)t * N : nullptr;
        a.kept_out = kept_out ? kept_out + (size_t)t * keep : nullptr;
        a.y_acc = y_acc + (size_t)t * d;
        a.y = static_cast<char *>(y) + (size_t)t * d * ysz;
        a.y_dtype = y_dtype;
        a.hdr = static_cast<WsHeader *>(ws);
        if ((rc = launch(k_ctk_gateup, dim3(G), dim3(kCtkThreads), (size_t)d * 2, s, true, a)) !=
                MOE_OK ||
            (rc = launch(k_ctk_down, dim3(G), dim3(kCtkThreads), ctk_down_smem_bytes(N, d), s, true,
                         a)) != MOE_OK)
            return rc;
    }
    return MOE_OK;
}

int moe_pack_w_down(const void *w_down_bf16, void *w_down_cm_bf16, int E, int d, int I,
                    void *stream)
{
    if (E < 1 || E > kMaxE || d < kMinD || d > kMaxD || d % 64 || I < kMinI || I > kMaxI || I % 16)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!w_down_bf16 || !w_down_cm_bf16 || w_down_bf16 == w_down_cm_bf16)
        return MOE_ERR_INVALID_ARG;
    return launch(k_pack_w_down, dim3((I + 63) / 64, (d + 63) / 64, E), dim3(256), 0,
                  static_cast<cudaStream_t>(stream), true,
                  static_cast<const uint16_t *>(w_down_bf16), static_cast<uint16_t *>(w_down_cm_bf16),
                  d, I);
}

int moe_test_exp_c(const float *x, float *y, int64_t n, void *stream)
{
    if (n < 0 || (n > 0 && (!x || !y)))
        return MOE_ERR_INVALID_ARG;
    if (n == 0)
        return MOE_OK;
    int64_t blocks = (n + 255) / 256;
    if (blocks > 65535 * 16)
        blocks = 65535 * 16;
    return launch(k_test_expc, dim3((unsigned)blocks), dim3(256), 0,
                  static_cast<cudaStream_t>(stream), false, x, y, n);
}

int moe_test_expert_stream(const void *x_bf16, const void *w_gate_bf16, const void *w_up_bf16,
                           const void *w_down_bf16, int T, int d, int E, int I, int k1, int k2,
                           void *y, int y_dtype, int flags, void *ws, size_t ws_bytes,
                           void *stream)
{
    int rc = check_shape(T, d, E, I, k1);
    if (rc != MOE_OK)
        return rc;
    if ((rc = check_route(E, k1, k2)) != MOE_OK)
        return rc;
    if (T == 0)
        return MOE_OK;
    if (!x_bf16 || !w_gate_bf16 || !w_up_bf16 || !w_down_bf16 || !y || !ws)
        return MOE_ERR_INVALID_ARG;
    if (y_dtype != MOE_DTYPE_F32 && y_dtype != MOE_DTYPE_BF16)
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(T, d, E, I, k1);
    if (ws_bytes < L.total)
        return MOE_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    DevInfo *di;
    if ((rc = device_info(di)) != MOE_OK)
        return rc;
    if (flags & MOE_WDOWN_CHANNEL_MAJOR) {
        if (!decode_fits(T, d, E, I, k1, di->num_sms))
            return MOE_ERR_UNSUPPORTED_SHAPE;
        DecodeArgs a = {};
        a.x = static_cast<const uint16_t *>(x_bf16);
        a.wg = static_cast<const uint16_t *>(w_gate_bf16);
        a.wu = static_cast<const uint16_t *>(w_up_bf16);
        a.wdt = static_cast<const uint16_t *>(w_down_bf16);
        a.d = d;
        a.E = E;
        a.I = I;
        a.k1 = k1;
        a.k2 = k2;
        a.logits = at<float>(ws, L.logits);
        a.topk_idx = at<int32_t>(ws, L.idx);
        a.topk_w = at<float>(ws, L.w);
        a.offsets = at<int32_t>(ws, L.offsets);
        a.sorted_slot = at<int32_t>(ws, L.sorted_slot);
        a.slot_pos = at<int32_t>(ws, L.slot_pos);
        a.uniq_count = at<int32_t>(ws, L.uniq_count);
        a.uniq_list = at<int32_t>(ws, L.uniq_list);
            a.yacc = at<float>(ws, L.dyacc);
        a.y = y;
        a.y_dtype = y_dtype;
        a.hdr = static_cast<WsHeader *>(ws);
        const size_t smem = decode_smem_bytes(d);
        if (d == 2048)
            return launch(k_decode<8, false>, dim3(di->num_sms), dim3(kSThreads), smem, s, kCoop,
                          a);
        if (d == 4096)
            return launch(k_decode<16, false>, dim3(di->num_sms), dim3(kSThreads), smem, s, kCoop,
                          a);
        return launch(k_decode<0, false>, dim3(di->num_sms), dim3(kSThreads), smem, s, kCoop, a);
    }
    return enqueue_stream(layer_stream_call(x_bf16, w_gate_bf16, w_up_bf16, w_down_bf16, T, d, E, I,
                                            k1, k2, y, y_dtype, nullptr, nullptr, ws),
                          s, false);
}

int moe_test_set_wait_limit_ns(uint64_t ns)
{
    if (ns == 0)
        return MOE_ERR_INVALID_ARG;
    const unsigned long long v = ns;
    return cudaMemcpyToSymbol(g_moe_wait_limit_ns, &v, sizeof(v)) == cudaSuccess ? MOE_OK
                                                                                 : MOE_ERR_CUDA;
}

}  // extern "C" (the wait kernel below is internal)

namespace moe {
// One CTA waits on something nothing will ever complete, with the library's
// own bounded waits: which 0, a header flag (the grid barrier's release flag,
// one generation ahead); 1, an mbarrier phase nobody arrives on; 2, the
// one-token layer's router exchange, for a tag no CTA publishes.  Each wait
// gives up at the wait limit and records MOE_ERR_TIMEOUT.
__global__ void k_test_wait_never_set(WsHeader *hdr, int which)
{
    __shared__ uint64_t bar;
    __shared__ DecodeSmem ds;
    int *status = &hdr->status;
    if (which == 0) {
        if (threadIdx.x == 0)
            wait_flag_eq(&hdr->bar_go, ld_relaxed_u32(&hdr->bar_go) + 1u, status);
    } else if (which == 1) {
        if (threadIdx.x == 0) {
            mbar_init(&bar, 1);
            fence_mbar_init();
            mbar_wait(&bar, 0, status);
        }
    } else if (threadIdx.x < 32) {
        DecodeArgs a = {};
        a.hdr = hdr;
        a.E = 16;
        a.k1 = 2;
        a.k2 = 4;
        // not read (the wait gives up first), but a valid global address
        a.logits = reinterpret_cast<const float *>(hdr->bar_flag);
        // the counter pair of the call two ahead: zero until that call runs
        const unsigned slot = (ld_relaxed_u32(&hdr->decode_seq) + 3u) & 3u;
        int j, kt;
        float wv;
        decode_route<4>(a, true, slot, threadIdx.x, &ds, status, VarK(), j, wv, kt);
    }
}
}  // namespace moe

extern "C" {

int moe_test_wait_never_set(void *ws, size_t ws_bytes, int which, void *stream)
{
    if (!ws || ws_bytes < sizeof(WsHeader) || (reinterpret_cast<uintptr_t>(ws) & 255) ||
        which < 0 || which > 2)
        return MOE_ERR_INVALID_ARG;
    return launch(k_test_wait_never_set, dim3(1), dim3(64), 0, static_cast<cudaStream_t>(stream),
                  0, static_cast<WsHeader *>(ws), which);
}

int moe_test_set_grouped_single(int single)
{
    if (single != 0 && single != 1)
        return MOE_ERR_INVALID_ARG;
    g_grouped_single = single;
    return MOE_OK;
}

int moe_test_grouped_pairs(int which)
{
    if (which != 1)
        return -1;
    DevInfo *di;
    if (device_info(di) != MOE_OK)
        return -1;
    return di->gemm1_pairs;
}

int moe_test_num_sms(void)
{
    DevInfo *di;
    if (device_info(di) != MOE_OK)
        return 0;
    return di->num_sms;
}

int moe_test_expert_grouped(const void *x_bf16, const void *w_gate_bf16, const void *w_up_bf16,
                            const void *w_down_bf16, int T, int d, int E, int I, int k1, int which,
                            void *ws, size_t ws_bytes, void *stream)
{
    int rc = check_shape(T, d, E, I, k1);
    if (rc != MOE_OK)
        return rc;
    if (which < 1 || which > 8)
        return MOE_ERR_INVALID_ARG;
    if (!grouped_fits(d, E, I))
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (T == 0)
        return MOE_OK;
    if (!x_bf16 || !w_gate_bf16 || !w_up_bf16 || !w_down_bf16 || !ws)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x_bf16) || !aligned16(w_gate_bf16) || !aligned16(w_up_bf16) ||
        !aligned16(w_down_bf16) || (reinterpret_cast<uintptr_t>(ws) & 255))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(T, d, E, I, k1);
    if (ws_bytes < L.total)
        return MOE_ERR_WORKSPACE_TOO_SMALL;
    DevInfo *di;
    if ((rc = device_info(di)) != MOE_OK)
        return rc;
    if (which & 8)  // the down GEMM storing per-slot rows (the moe_expert_ffn epilogue)
        return enqueue_grouped(x_bf16, w_gate_bf16, w_up_bf16, w_down_bf16, T, d, E, I, k1,
                               at<int32_t>(ws, L.offsets), at<int32_t>(ws, L.sorted_slot),
                               nullptr, at<uint16_t>(ws, L.out), at<uint16_t>(ws, L.h), nullptr,
                               at<float>(ws, L.out), static_cast<WsHeader *>(ws), di->num_sms,
                               static_cast<cudaStream_t>(stream), 2, false);
    return enqueue_grouped(x_bf16, w_gate_bf16, w_up_bf16, w_down_bf16, T, d, E, I, k1,
                           at<int32_t>(ws, L.offsets), at<int32_t>(ws, L.sorted_slot),
                           at<float>(ws, L.w), at<uint16_t>(ws, L.out), at<uint16_t>(ws, L.h),
                           at<float>(ws, L.y_acc), nullptr, static_cast<WsHeader *>(ws),
                           di->num_sms, static_cast<cudaStream_t>(stream), which, false);
}

}  // extern "C"

// ====================================================================== no-alloc
// Scratch for moe_expert_ffn_noalloc: a fixed array in the library image, so
// callers that cannot give the library device memory can still run the
// expert FFN.  Layout: header (grid-barrier flags, status) | activated
// expert count | activated expert list (E <= 1024) | float32 channel
// activations of every routed slot [T*k1 x I].
namespace moe {
constexpr size_t kNoAllocMaxH = 1047424;  // float32 channel activations that fit
constexpr size_t kNoAllocUOffset = sizeof(WsHeader);
constexpr size_t kNoAllocHOffset = kNoAllocUOffset + 256 + sizeof(int32_t) * 1024;
constexpr size_t kNoAllocBytes = kNoAllocHOffset + sizeof(float) * kNoAllocMaxH;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

// Device address of g_noalloc_scratch per device (the host-side name is only
// a stand-in, so kernels get this address instead).
static void *g_noalloc_ptr[64];
static std::mutex g_noalloc_mu;

static int noalloc_scratch(void *&out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p)
            return MOE_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    out = g_noalloc_ptr[dev];
    return MOE_OK;
}
}  // namespace moe

extern "C" int moe_expert_ffn_noalloc(const void *x_bf16, const int32_t *expert_offsets,
                                      const int32_t *sorted_slot, const void *w_gate_bf16,
                                      const void *w_up_bf16, const void *w_down_bf16, int T, int d,
                                      int E, int I, int k1, float *out, void *stream)
{
    int rc = check_shape(T, d, E, I, k1);
    if (rc != MOE_OK)
        return rc;
    if ((size_t)T * (size_t)k1 * (size_t)I > kNoAllocMaxH)
        return MOE_ERR_SCRATCH_LIMIT;
    if (T == 0)
        return MOE_OK;
    if (!x_bf16 || !expert_offsets || !sorted_slot || !w_gate_bf16 || !w_up_bf16 ||
        !w_down_bf16 || !out)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x_bf16) || !aligned16(w_gate_bf16) || !aligned16(w_up_bf16) ||
        !aligned16(w_down_bf16) || !aligned16(out))
        return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    DevInfo *di;
    if ((rc = device_info(di)) != MOE_OK)
        return rc;
    void *scratch = nullptr;
    if ((rc = noalloc_scratch(scratch)) != MOE_OK)
        return rc;
    // the grid-barrier counters and flags must start at zero; the status word
    // (the header's first int) is kept, so problems of earlier calls stay
    // visible until moe_noalloc_read_status reads and clears it
    if (cudaMemsetAsync(static_cast<char *>(scratch) + sizeof(int), 0,
                        sizeof(WsHeader) - sizeof(int), s) != cudaSuccess)
        return MOE_ERR_CUDA;
    int32_t *uniq_count = at<int32_t>(scratch, kNoAllocUOffset);
    int32_t *uniq_list = at<int32_t>(scratch, kNoAllocUOffset + 256);
    float *h = at<float>(scratch, kNoAllocHOffset);
    if ((rc = launch(k_uniq_from_offsets, dim3(1), dim3(1024), 0, s, true, expert_offsets, E,
                     uniq_count, uniq_list)) != MOE_OK)
        return rc;
    StreamCall c = {};
    c.x = x_bf16;
    c.wg = w_gate_bf16;
    c.wu = w_up_bf16;
    c.wd = w_down_bf16;
    c.T = T;
    c.d = d;
    c.E = E;
    c.I = I;
    c.k1 = k1;
    c.k2 = k1;
    c.offsets = const_cast<int32_t *>(expert_offsets);
    c.sorted_slot = const_cast<int32_t *>(sorted_slot);
    c.uniq_count = uniq_count;
    c.uniq_list = uniq_list;
    c.h = h;
    c.out = out;
    c.hdr = static_cast<WsHeader *>(scratch);
    return enqueue_stream(c, s);
}

extern "C" int moe_noalloc_read_status(int *status_out, void *stream)
{
    if (!status_out)
        return MOE_ERR_INVALID_ARG;
    void *scratch = nullptr;
    int rc = noalloc_scratch(scratch);
    if (rc != MOE_OK)
        return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int v = 0;
    if (cudaMemcpyAsync(&v, scratch, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (cudaMemsetAsync(scratch, 0, sizeof(int), s) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess)
        return MOE_ERR_CUDA;
    *status_out = v;
    return MOE_OK;
}
