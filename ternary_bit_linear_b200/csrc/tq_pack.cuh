// tq_pack.cuh -- absmean ternarisation and 2-bit packing.
//
// Foundry, docs/quantization.md, "Ternary Quantization / How It Works" 1-3 and
// "Ternary Format / Encoding"; Hetman-2b, src/quantization.py, section 2
// (AbsmeanWeightQuantizer.forward) and section 5 (export_packed_weights).
//
// gamma is the fp32 nearest to the exact mean of |w|: every CTA sums |w| as a
// double-double (TwoSum per element, error ~2^-100 relative), so the rounding
// to fp32 does not depend on the reduction tree.  Codes come from a single
// fp32 threshold per gamma (code_threshold), which is equivalent to rounding
// the fp32 quotient w / gamma and clamping, without a divide per element.
//
// HBM traffic: read 4 B and write 0.25 B per weight (per-row gamma: one pass;
// per-tensor gamma: a reduction pass, then the packing pass, which walks the
// rows in reverse so the tail of the first pass is still in L2).
#pragma once

#include "tq_common.cuh"

namespace tq {

constexpr int kPackThreads = 256;

__device__ __forceinline__ float4 sanitize_w(float4 v) {
    auto f = [](float x) {
        if (x != x) return 0.0f;
        if (isinf(x)) return x > 0.0f ? 1.0f : -1.0f;
        return x;
    };
    return make_float4(f(v.x), f(v.y), f(v.z), f(v.w));
}

__device__ __forceinline__ void acc_abs4(DD &a, float4 v) {
    dd_acc(a, (double)fabsf(v.x));
    dd_acc(a, (double)fabsf(v.y));
    dd_acc(a, (double)fabsf(v.z));
    dd_acc(a, (double)fabsf(v.w));
}

__device__ __forceinline__ uint32_t pack4(float4 v, float t) {
    return ternary_field(v.x, t) | (ternary_field(v.y, t) << 2) | (ternary_field(v.z, t) << 4) |
           (ternary_field(v.w, t) << 6);
}

// Sum over the CTA in a fixed order; the result is valid in every thread.
__device__ __forceinline__ DD dd_block_sum(DD a, DD *red /* [kPackThreads/32] */) {
    a = dd_warp_sum(a);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = a;
    __syncthreads();
    DD t = {0.0, 0.0};
    if (lane < kPackThreads / 32) t = red[lane];
    t = dd_warp_sum(t);
    __syncthreads();
    return t;
}

// One CTA per row.  VEC > 0: each thread keeps VEC float4 of the row in
// registers (K <= 1024 * VEC); VEC == 0: the row is streamed twice (any K).
// per_tensor_t != nullptr: use that precomputed threshold instead of a row gamma.
template <int VEC>
__global__ void __launch_bounds__(kPackThreads)
    pack_rows_kernel(const float *__restrict__ w, int64_t N, int K, int sanitize,
                     uint8_t *__restrict__ packed, float *__restrict__ gamma,
                     const float *__restrict__ per_tensor_t, int reverse) {
    __shared__ DD red[kPackThreads / 32];
    __shared__ float s_t;
    const int64_t n = reverse ? (N - 1 - (int64_t)blockIdx.x) : (int64_t)blockIdx.x;
    const int nv = K >> 2;
    const float4 *src = reinterpret_cast<const float4 *>(w + n * (int64_t)K);
    uint8_t *dst = packed + n * (int64_t)(K >> 2);
    const int tid = threadIdx.x;

    float4 v[VEC > 0 ? VEC : 1];
    if (VEC > 0) {
#pragma unroll
        for (int i = 0; i < VEC; ++i) {
            const int idx = tid + i * kPackThreads;
            v[i] = idx < nv ? __ldcs(src + idx) : make_float4(0.f, 0.f, 0.f, 0.f);
            if (sanitize) v[i] = sanitize_w(v[i]);
        }
    }

    float t;
    if (per_tensor_t != nullptr) {
        t = __ldg(per_tensor_t);
    } else {
        DD a = {0.0, 0.0};
        if (VEC > 0) {
#pragma unroll
            for (int i = 0; i < VEC; ++i) acc_abs4(a, v[i]);
        } else {
            for (int idx = tid; idx < nv; idx += kPackThreads) {
                float4 x = __ldg(src + idx);
                if (sanitize) x = sanitize_w(x);
                acc_abs4(a, x);
            }
        }
        a = dd_block_sum(a, red);
        if (tid == 0) {
            float g = dd_mean_to_f32(a, (double)K);
            g = g > 1e-6f ? g : 1e-6f;
            gamma[n] = g;
            s_t = code_threshold(g);
        }
        __syncthreads();
        t = s_t;
    }

    if (VEC > 0) {
#pragma unroll
        for (int i = 0; i < VEC; ++i) {
            const int idx = tid + i * kPackThreads;
            if (idx < nv) dst[idx] = (uint8_t)pack4(v[i], t);
        }
    } else {
        for (int idx = tid; idx < nv; idx += kPackThreads) {
            float4 x = __ldcs(src + idx);
            if (sanitize) x = sanitize_w(x);
            dst[idx] = (uint8_t)pack4(x, t);
        }
    }
}

// Per-tensor gamma, pass 1: CTA b sums |w| over float4 range [b*chunk, ...)
// into partial[b] (double-double).
__global__ void __launch_bounds__(kPackThreads)
    absum_partial_kernel(const float *__restrict__ w, int64_t nv, int64_t chunk, int sanitize,
                         DD *__restrict__ partial) {
    __shared__ DD red[kPackThreads / 32];
    const float4 *src = reinterpret_cast<const float4 *>(w);
    const int64_t beg = (int64_t)blockIdx.x * chunk;
    const int64_t end = min(nv, beg + chunk);
    DD a = {0.0, 0.0};
    int64_t idx = beg + threadIdx.x;
    for (; idx + 3 * kPackThreads < end; idx += 4 * kPackThreads) {
        float4 x0 = __ldg(src + idx), x1 = __ldg(src + idx + kPackThreads),
               x2 = __ldg(src + idx + 2 * kPackThreads), x3 = __ldg(src + idx + 3 * kPackThreads);
        if (sanitize) {
            x0 = sanitize_w(x0);
            x1 = sanitize_w(x1);
            x2 = sanitize_w(x2);
            x3 = sanitize_w(x3);
        }
        acc_abs4(a, x0);
        acc_abs4(a, x1);
        acc_abs4(a, x2);
        acc_abs4(a, x3);
    }
    for (; idx < end; idx += kPackThreads) {
        float4 x = __ldg(src + idx);
        if (sanitize) x = sanitize_w(x);
        acc_abs4(a, x);
    }
    a = dd_block_sum(a, red);
    if (threadIdx.x == 0) partial[blockIdx.x] = a;
}

// Per-tensor gamma, pass 2: one CTA folds the partials in a fixed order and
// writes gamma[0] and the code threshold.
__global__ void __launch_bounds__(kPackThreads)
    absum_finalize_kernel(const DD *__restrict__ partial, int nparts, double n,
                          float *__restrict__ gamma, float *__restrict__ t_out) {
    __shared__ DD red[kPackThreads / 32];
    DD a = {0.0, 0.0};
    for (int i = threadIdx.x; i < nparts; i += kPackThreads) a = dd_add(a, partial[i]);
    a = dd_block_sum(a, red);
    if (threadIdx.x == 0) {
        float g = dd_mean_to_f32(a, n);
        g = g > 1e-6f ? g : 1e-6f;
        gamma[0] = g;
        *t_out = code_threshold(g);
    }
}

}  // namespace tq
