// combine.cuh -- weighted combine of per-slot expert outputs with the Eq. 2
// weights ("Paper of the Week #3", section "The Receipt"):
//     y[t, :] = sum_{s=0}^{k1-1} w[t, s] * out[slot_pos[t*k1 + s], :]
// summed in slot order in float32; y in bf16 or float32.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int kCombineThreads = 256;

// grid (ceil(d / (4 * kCombineThreads)), T); four columns per thread
__global__ void __launch_bounds__(kCombineThreads) k_combine(const float *out,
                                                             const int32_t *slot_pos,
                                                             const float *topk_w, int T, int d,
                                                             int k1, void *y, int y_dtype,
                                                             int *status)
{
    pdl_wait();
    pdl_trigger();
    const int t = blockIdx.y;
    const int j = (blockIdx.x * kCombineThreads + threadIdx.x) * 4;
    if (t >= T || j >= d)
        return;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < k1; ++s) {
        const int pos = slot_pos[t * k1 + s];
        if (pos < 0 || pos >= T * k1) {
            set_status(status, MOE_ERR_DEVICE_CHECK);
            continue;
        }
        const float w = topk_w[t * k1 + s];
        const float4 o = *reinterpret_cast<const float4 *>(out + (size_t)pos * d + j);
        float p;
        p = w * o.x; acc.x = acc.x + p;
        p = w * o.y; acc.y = acc.y + p;
        p = w * o.z; acc.z = acc.z + p;
        p = w * o.w; acc.w = acc.w + p;
    }
    if (y_dtype == MOE_DTYPE_BF16) {
        uint16_t *yb = reinterpret_cast<uint16_t *>(y) + (size_t)t * d + j;
        const uint32_t lo = f32_to_bf16_rn(acc.x) | ((uint32_t)f32_to_bf16_rn(acc.y) << 16);
        const uint32_t hi = f32_to_bf16_rn(acc.z) | ((uint32_t)f32_to_bf16_rn(acc.w) << 16);
        *reinterpret_cast<uint2 *>(yb) = make_uint2(lo, hi);
    } else {
        *reinterpret_cast<float4 *>(reinterpret_cast<float *>(y) + (size_t)t * d + j) = acc;
    }
}

// Activated experts (ascending) from per-expert offsets; one CTA.
__global__ void __launch_bounds__(1024) k_uniq_from_offsets(const int32_t *offsets, int E,
                                                            int32_t *uniq_count,
                                                            int32_t *uniq_list)
{
    __shared__ int flag[1024];
    __shared__ int scan[40];
    pdl_wait();
    pdl_trigger();
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        flag[e] = offsets[e + 1] > offsets[e] ? 1 : 0;
    __syncthreads();
    // exclusive scan (E <= 1024, one element per thread)
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int v = tid < E ? flag[tid] : 0;
    int incl = v;
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o)
            incl += u;
    }
    if (lane == 31)
        scan[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int nw = blockDim.x >> 5;
        const int t = lane < nw ? scan[lane] : 0;
        int s = t;
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o)
                s += u;
        }
        scan[lane] = s - t;
        if (lane == 31)
            scan[32] = s;
    }
    __syncthreads();
    if (tid < E && v)
        uniq_list[scan[warp] + incl - v] = tid;
    if (tid == 0)
        *uniq_count = scan[32];
}

}  // namespace moe
