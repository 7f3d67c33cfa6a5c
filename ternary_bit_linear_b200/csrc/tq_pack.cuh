// tq_pack.cuh -- absmean ternarisation and 2-bit packing.
//
// Foundry, docs/quantization.md, "Ternary Quantization / How It Works" 1-3 and
// "Ternary Format / Encoding"; Hetman-2b, src/quantization.py, section 2
// (AbsmeanWeightQuantizer.forward) and section 5 (export_packed_weights).
//
// gamma is the fp32 nearest to the exact mean of |w| (ties to even), then
// max(., 1e-6).  Fast path: |w| is summed in plain fp64 over a fixed tree of
// known height h, so the computed mean q is within eps = (h + 2) * 2^-53 * q of
// the exact mean.  If q is farther than 2 * eps from both fp32 rounding
// midpoints around fp32(q), fp32(q) is the correctly rounded mean.  Otherwise
// (about one row in ten million on random data, and every row whose mean is an
// exact midpoint) the sum is redone as a double-double (TwoSum per element,
// ~2^-100 relative) and rounded with an explicit midpoint test.
//
// Codes come from one fp32 threshold per gamma (code_threshold), equivalent to
// rounding the fp32 quotient w / gamma and clamping, without a divide; or, for
// the threshold rule (Foundry "Absmean Thresholding", BitRASP ternarize_weight),
// from w > fp32(ratio * gamma) (pack_threshold); or, for Foundry's manual
// threshold (fq_quantize_ternary_threshold), from w > t with gamma = t.
//
// HBM traffic: read 4 B and write 0.25 B per weight.  Per-row gamma is one
// pass; per-tensor gamma reads W twice (reduction, then packing walking the
// rows in reverse so the tail of the first pass is still in L2).
#pragma once

#include "tq_common.cuh"

namespace tq {

constexpr int kPackThreads = 256;
constexpr int kPackWarps = kPackThreads / 32;

__device__ __forceinline__ float4 sanitize_w(float4 v) {
    auto f = [](float x) {
        if (x != x) return 0.0f;
        if (isinf(x)) return x > 0.0f ? 1.0f : -1.0f;
        return x;
    };
    return make_float4(f(v.x), f(v.y), f(v.z), f(v.w));
}

__device__ __forceinline__ double abs_sum4(float4 v) {
    // left-to-right: ((|x| + |y|) + |z|) + |w|
    return __dadd_rn(__dadd_rn(__dadd_rn((double)fabsf(v.x), (double)fabsf(v.y)),
                               (double)fabsf(v.z)),
                     (double)fabsf(v.w));
}

__device__ __forceinline__ void acc_abs4(DD &a, float4 v) {
    dd_acc(a, (double)fabsf(v.x));
    dd_acc(a, (double)fabsf(v.y));
    dd_acc(a, (double)fabsf(v.z));
    dd_acc(a, (double)fabsf(v.w));
}

// Byte of four 2-bit codes: start from 0b01010101 (all zero codes) and move
// each field up (+1 -> 0b10) or down (-1 -> 0b00).  NaN compares false: code 0.
// The packed byte in the requested layout (CONV: one of Hetman-2b's).
template <bool CONV>
__device__ __forceinline__ uint32_t out_codes(uint32_t foundry_byte, int enc) {
    return CONV ? codes_from_foundry(foundry_byte, enc) : foundry_byte;
}

__device__ __forceinline__ uint32_t pack4(float4 v, float t) {
    uint32_t b = 0x55u;
    b += (v.x >= t) ? 1u : 0u;
    b -= (v.x <= -t) ? 1u : 0u;
    b += (v.y >= t) ? 4u : 0u;
    b -= (v.y <= -t) ? 4u : 0u;
    b += (v.z >= t) ? 16u : 0u;
    b -= (v.z <= -t) ? 16u : 0u;
    b += (v.w >= t) ? 64u : 0u;
    b -= (v.w <= -t) ? 64u : 0u;
    return b;
}

__device__ __forceinline__ double warp_sum_dbl(double v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = __dadd_rn(v, __shfl_xor_sync(0xffffffffu, v, off));
    return v;
}

// Plain fp64 block sum in a fixed order (5 + 3 tree levels); valid in every thread.
__device__ __forceinline__ double block_sum_dbl(double a, double *red) {
    a = warp_sum_dbl(a);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = a;
    __syncthreads();
    // lanes >= kPackWarps add exact zeros; every lane ends with the same value
    double t = warp_sum_dbl(lane < kPackWarps ? red[lane] : 0.0);
    __syncthreads();
    return t;
}

// Double-double block sum in a fixed order; valid in every thread.
__device__ __forceinline__ DD dd_block_sum(DD a, DD *red) {
    a = dd_warp_sum(a);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = a;
    __syncthreads();
    DD t = {0.0, 0.0};
    if (lane < kPackWarps) t = red[lane];
    t = dd_warp_sum(t);
    __syncthreads();
    return t;
}

// fp32(q) if the exact mean, known to lie within q * (1 +- eps), must round to
// it; otherwise a negative value (caller falls back to the exact sum).
__device__ __forceinline__ float mean_fast_or_fail(double q, double eps) {
    if (!(q > 0.0)) return 0.0f;  // all zero: exact
    const float f = __double2float_rn(q);
    if (!(f > 0.0f) || isinf(f)) return -1.0f;  // tiny or huge: let the exact path decide
    const float up = __int_as_float(__float_as_int(f) + 1);  // neighbours of a positive finite f
    const float dn = __int_as_float(__float_as_int(f) - 1);
    const double mu = 0.5 * ((double)f + (double)up);
    const double ml = 0.5 * ((double)f + (double)dn);
    const double margin = 2.0 * eps * q;
    if (mu - q > margin && q - ml > margin) return f;
    return -1.0f;
}

// Relative error bound of a plain fp64 sum of non-negative terms over a tree of
// height h, followed by a multiply with a rounded reciprocal of n: h + 2
// roundings of relative error 2^-53 each, with slack.
__device__ __forceinline__ double sum_error_bound(int h) { return (double)(h + 3) * 0x1p-53 * 1.01; }

// ---------------------------------------------------------------------------
// Per-row gamma (or a precomputed per-tensor threshold) + packing, one warp per
// row, persistent warps walking rows (warp id, + total warps, ...).
//   pass 1: stream the row once (8 float4 per lane in flight), sum |w| in plain
//           fp64 per lane, fold the 32 lanes with shuffles (fixed order);
//           every lane derives the same gamma and code threshold; the rare
//           rows whose mean sits within the error bound of a midpoint are
//           re-summed exactly (double-double) by the same warp.
//   pass 2: re-read the row (L2 hit: pass 1 left it there) and write one byte
//           per float4; a warp stores 32 consecutive bytes per instruction.
// ---------------------------------------------------------------------------
// Per-tensor gamma from the partial sums of tq_absum_partial_kernel, computed by
// every CTA of the pack pass (all kPackThreads threads take part): a fixed
// thread-strided chain over the partials and a fixed block tree, then the
// rounding-margin check of mean_fast_or_fail with the error bound of the
// whole summation tree (height); in the rare case that the mean lies too close
// to an fp32 rounding boundary, an exact double-double re-sum of the tensor.
// All CTAs therefore agree on gamma (it is the correctly rounded exact mean).
// CTA 0 writes gamma[0].  Returns the code threshold.
// ---------------------------------------------------------------------------
__device__ __noinline__ float per_tensor_threshold(const double *__restrict__ partial, int nparts, int height,
                                                   const float *__restrict__ w, int64_t nv, int sanitize,
                                                   float *__restrict__ gamma, float ratio) {
    __shared__ double red[kPackWarps];
    __shared__ DD redd[kPackWarps];
    __shared__ float g_s;
    double a = 0.0;
    for (int i = threadIdx.x; i < nparts; i += kPackThreads) a = __dadd_rn(a, partial[i]);
    const double S = block_sum_dbl(a, red);
    const double n = 4.0 * (double)nv;
    float g = mean_fast_or_fail(__ddiv_rn(S, n), sum_error_bound(height));
    if (g < 0.0f) {  // CTA-uniform: every thread holds the same S
        const float4 *src = reinterpret_cast<const float4 *>(w);
        DD d = {0.0, 0.0};
        for (int64_t idx = threadIdx.x; idx < nv; idx += kPackThreads) {
            float4 x = __ldg(src + idx);
            acc_abs4(d, sanitize ? sanitize_w(x) : x);
        }
        d = dd_warp_sum(d);
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        if (lane == 0) redd[warp] = d;
        __syncthreads();
        if (threadIdx.x == 0) {
            DD e = {0.0, 0.0};
            for (int u = 0; u < kPackWarps; ++u) e = dd_add(e, redd[u]);
            g_s = dd_mean_to_f32(e, n);
        }
        __syncthreads();
        g = g_s;
    }
    g = g > 1e-6f ? g : 1e-6f;
    if (blockIdx.x == 0 && threadIdx.x == 0) gamma[0] = g;
    return pack_threshold(g, ratio);
}

// Foundry's manual threshold: gamma is the caller's threshold t (CTA 0 writes
// it), and a weight is +1 iff w > t, i.e. w >= the next float above t.
__device__ __forceinline__ float fixed_threshold(float t, float *__restrict__ gamma) {
    if (blockIdx.x == 0 && threadIdx.x == 0) gamma[0] = t;
    return nextafterf(t, __int_as_float(0x7f800000));
}

// Options word of the pack kernels: bit 0 inputs ready, bits 1-2 the packed-code
// layout, bit 3 a fixed scale (the manual threshold, passed in `ratio`).
constexpr int kPackOptFixed = 8;

// No block-level synchronisation: warps are independent.
// ---------------------------------------------------------------------------
constexpr int kPackUnroll = 8;

template <bool SAN, bool CONV>
__global__ void __launch_bounds__(kPackThreads)
    tq_pack_rows_kernel(const float *__restrict__ w, int64_t N, int K, double inv_k,
                     uint8_t *__restrict__ packed, float *__restrict__ gamma,
                     const double *__restrict__ partial, int nparts, int height, int reverse,
                     int opts, float ratio) {
    const int ready = opts & 1, enc = (opts >> 1) & 3;  // inputs ready; packed-code layout
    const bool fixed = (opts & kPackOptFixed) != 0;
    if (!ready) pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (int64_t)gridDim.x * kPackWarps;
    const int nv = K >> 2;
    const bool per_tensor = partial != nullptr || fixed;
    const float t_tensor =
        fixed ? fixed_threshold(ratio, gamma)
              : per_tensor ? per_tensor_threshold(partial, nparts, height, w, (int64_t)nv * N, SAN, gamma, ratio)
                           : 0.0f;
    // per-lane chain length (float4) of pass 1, for the error bound
    const int chain = (nv + 31) / 32;
    const double eps = sum_error_bound(4 * chain + 5);

    for (int64_t i = (int64_t)blockIdx.x * kPackWarps + (threadIdx.x >> 5); i < N; i += nwarps) {
        const int64_t n = reverse ? (N - 1 - i) : i;
        const float4 *src = reinterpret_cast<const float4 *>(w + n * (int64_t)K);
        float t = t_tensor;
        if (!per_tensor) {
            double a = 0.0;
            int c = lane;
            for (; c + 32 * (kPackUnroll - 1) < nv; c += 32 * kPackUnroll) {
                float4 x[kPackUnroll];
#pragma unroll
                for (int u = 0; u < kPackUnroll; ++u) x[u] = __ldg(src + c + 32 * u);
#pragma unroll
                for (int u = 0; u < kPackUnroll; ++u) a = __dadd_rn(a, abs_sum4(SAN ? sanitize_w(x[u]) : x[u]));
            }
            for (; c < nv; c += 32) {
                const float4 x = __ldg(src + c);
                a = __dadd_rn(a, abs_sum4(SAN ? sanitize_w(x) : x));
            }
            const double S = warp_sum_dbl(a);  // identical in every lane
            float g = mean_fast_or_fail(__dmul_rn(S, inv_k), eps);
            if (g < 0.0f) {  // rare: redo the sum exactly
                DD d = {0.0, 0.0};
                for (int cc = lane; cc < nv; cc += 32) {
                    const float4 x = __ldg(src + cc);
                    acc_abs4(d, SAN ? sanitize_w(x) : x);
                }
                d = dd_warp_sum(d);
                g = dd_mean_to_f32(d, (double)K);
            }
            g = g > 1e-6f ? g : 1e-6f;
            if (lane == 0) gamma[n] = g;
            t = pack_threshold(g, ratio);
        }
        uint8_t *dst = packed + n * (int64_t)nv;
        int c = lane;
        for (; c + 32 * (kPackUnroll - 1) < nv; c += 32 * kPackUnroll) {
            float4 x[kPackUnroll];
#pragma unroll
            for (int u = 0; u < kPackUnroll; ++u) x[u] = __ldcs(src + c + 32 * u);
#pragma unroll
            for (int u = 0; u < kPackUnroll; ++u)
                dst[c + 32 * u] = (uint8_t)out_codes<CONV>(pack4(SAN ? sanitize_w(x[u]) : x[u], t), enc);
        }
        for (; c < nv; c += 32) {
            const float4 x = __ldcs(src + c);
            dst[c] = (uint8_t)out_codes<CONV>(pack4(SAN ? sanitize_w(x) : x, t), enc);
        }
    }
    if (ready) pdl_wait();  // complete no earlier than the previous kernel
}

// ---------------------------------------------------------------------------
// Team kernel (K <= 8192): T warps share a row.  The team's leader streams
// its rows with 1-D bulk copies into a ring of kPackRing shared-memory row
// buffers, kPackRing - 1 rows ahead, so HBM latency is hidden behind the
// work on earlier rows; every thread takes 8 float4 of the row into
// registers.  Per row: per-lane fp64 chain, warp shuffles, one named barrier
// for the T warp sums (double-buffered by row parity; it also tells the
// leader that the buffer is free again), then each thread packs its values.
// ---------------------------------------------------------------------------
constexpr int kTeamVec = 8;
constexpr int kPackRing = 3;

__device__ __forceinline__ void team_barrier(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Named barrier that also returns the AND of every participant's flag.
__device__ __forceinline__ bool team_all(int id, int threads, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(threads)
        : "memory");
    return r != 0;
}

__host__ __device__ constexpr int pack_team_smem(int T, int K) {
    return (kPackWarps / T) * kPackRing * (K / 4) * 16;
}

template <int T, bool SAN, bool CONV>
__global__ void __launch_bounds__(kPackThreads, 2)
    tq_pack_team_kernel(const float *__restrict__ w, int64_t N, int K, double inv_k,
                     uint8_t *__restrict__ packed, float *__restrict__ gamma,
                     const double *__restrict__ partial, int nparts, int height, int reverse,
                     int opts, float ratio) {
    const int ready = opts & 1, enc = (opts >> 1) & 3;  // inputs ready; packed-code layout
    const bool fixed = (opts & kPackOptFixed) != 0;
    constexpr int TEAMS = kPackWarps / T;
    extern __shared__ __align__(16) float4 rowbuf[];  // [TEAMS][kPackRing][nv]
    __shared__ uint64_t rbar[TEAMS][kPackRing];
    __shared__ double tred[2][kPackWarps];
    __shared__ DD tredd[kPackWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int team = warp / T, tw = warp % T;
    const int bar_id = 1 + team;
    const int nv = K >> 2;
    const int64_t nteams = (int64_t)gridDim.x * TEAMS;
    const int64_t first = (int64_t)blockIdx.x * TEAMS + team;
    const int64_t nmine = first < N ? (N - 1 - first) / nteams + 1 : 0;
    const bool leader = tw == 0 && lane == 0;
    float4 *ring = rowbuf + (size_t)team * kPackRing * nv;
    if (threadIdx.x == 0) {
        for (int u = 0; u < TEAMS; ++u)
            for (int r = 0; r < kPackRing; ++r) mbar_init(smem_u32(&rbar[u][r]), 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (!ready) pdl_wait();
    pdl_trigger();
    auto row_of = [&](int64_t k) {
        const int64_t i = first + k * nteams;
        return reverse ? (N - 1 - i) : i;
    };
    auto issue = [&](int64_t k) {  // leader: row k of this team into buffer k % kPackRing
        const uint32_t bar = smem_u32(&rbar[team][k % kPackRing]);
        mbar_arrive_expect_tx(bar, (uint32_t)(nv * 16));
        bulk_g2s(smem_u32(ring + (k % kPackRing) * nv), w + row_of(k) * (int64_t)K, (uint32_t)(nv * 16), bar);
    };
    int64_t issued = nmine < kPackRing ? nmine : kPackRing;
    if (leader)
        for (int64_t k = 0; k < issued; ++k) issue(k);
    // the first rows are in flight: now the per-tensor threshold (if any)
    const bool per_tensor = partial != nullptr || fixed;
    const float t_tensor =
        fixed ? fixed_threshold(ratio, gamma)
              : per_tensor ? per_tensor_threshold(partial, nparts, height, w, (int64_t)nv * N, SAN, gamma, ratio)
                           : 0.0f;
    const double eps = sum_error_bound(4 * kTeamVec + 5 + T);
    int parity = 0;
    int64_t k = 0;
    for (; k < nmine; ++k) {
        const int64_t n = row_of(k);
        const bool ok = warp_wait_sleep(smem_u32(&rbar[team][k % kPackRing]), (uint32_t)((k / kPackRing) & 1), lane);
        const float4 *src = ring + (k % kPackRing) * nv;
        float4 v[kTeamVec];
#pragma unroll
        for (int j = 0; j < kTeamVec; ++j) {
            const int idx = j * 32 * T + tw * 32 + lane;
            v[j] = idx < nv ? src[idx] : make_float4(0.f, 0.f, 0.f, 0.f);
            if (SAN) v[j] = sanitize_w(v[j]);
        }
        float t = t_tensor;
        bool all_ok;
        if (!per_tensor) {
            double a = 0.0;
#pragma unroll
            for (int j = 0; j < kTeamVec; ++j) a = __dadd_rn(a, abs_sum4(v[j]));
            a = warp_sum_dbl(a);
            if (lane == 0) tred[parity][warp] = a;
            all_ok = team_all(bar_id, 32 * T, ok);  // the buffer has been read, sums are in
            double S = 0.0;
#pragma unroll
            for (int u = 0; u < T; ++u) S = __dadd_rn(S, tred[parity][team * T + u]);
            parity ^= 1;
            float g = mean_fast_or_fail(__dmul_rn(S, inv_k), eps);
            if (g < 0.0f) {  // rare: redo the sum exactly (team-uniform branch)
                DD d = {0.0, 0.0};
#pragma unroll
                for (int j = 0; j < kTeamVec; ++j) acc_abs4(d, v[j]);
                d = dd_warp_sum(d);
                if (lane == 0) tredd[warp] = d;
                team_barrier(bar_id, 32 * T);
                DD e = {0.0, 0.0};
                for (int u = 0; u < T; ++u) e = dd_add(e, tredd[team * T + u]);
                team_barrier(bar_id, 32 * T);  // tredd may be rewritten by the next fallback
                g = dd_mean_to_f32(e, (double)K);
            }
            g = g > 1e-6f ? g : 1e-6f;
            if (all_ok && tw == 0 && lane == 0) gamma[n] = g;
            t = pack_threshold(g, ratio);
        } else {
            all_ok = team_all(bar_id, 32 * T, ok);  // the buffer has been read
        }
        if (!all_ok) break;  // a copy never landed (timeout recorded)
        if (leader && issued < nmine) issue(issued);
        issued = issued < nmine ? issued + 1 : issued;
        uint8_t *dst = packed + n * (int64_t)nv;
#pragma unroll
        for (int j = 0; j < kTeamVec; ++j) {
            const int idx = j * 32 * T + tw * 32 + lane;
            if (idx < nv) dst[idx] = (uint8_t)out_codes<CONV>(pack4(v[j], t), enc);
        }
    }
    // Copies in flight must land before the CTA exits (already true unless a
    // wait gave up).
    if (leader)
        for (int64_t j = k; j < issued; ++j)
            mbar_wait(smem_u32(&rbar[team][j % kPackRing]), (uint32_t)((j / kPackRing) & 1));
    if (ready) pdl_wait();  // complete no earlier than the previous kernel
}

// Per-tensor gamma, pass 1: CTA b sums |w| over float4 range [b*chunk, ...) in
// plain fp64 (each thread sequentially, then a fixed block tree).
__global__ void __launch_bounds__(kPackThreads)
    tq_absum_partial_kernel(const float *__restrict__ w, int64_t nv, int64_t chunk, int sanitize,
                         double *__restrict__ partial, int ready) {
    __shared__ double red[kPackWarps];
    if (!ready) pdl_wait();
    pdl_trigger();
    const float4 *src = reinterpret_cast<const float4 *>(w);
    const int64_t beg = (int64_t)blockIdx.x * chunk;
    const int64_t end = min(nv, beg + chunk);
    double a0 = 0.0, a1 = 0.0;
    int64_t idx = beg + threadIdx.x;
    for (; idx + 3 * kPackThreads < end; idx += 4 * kPackThreads) {
        float4 x[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) x[u] = __ldg(src + idx + u * kPackThreads);
        if (sanitize) {
#pragma unroll
            for (int u = 0; u < 4; ++u) x[u] = sanitize_w(x[u]);
        }
#pragma unroll
        for (int u = 0; u < 4; u += 2) {
            a0 = __dadd_rn(a0, abs_sum4(x[u]));
            a1 = __dadd_rn(a1, abs_sum4(x[u + 1]));
        }
    }
    for (; idx < end; idx += kPackThreads) {
        float4 x = __ldg(src + idx);
        if (sanitize) x = sanitize_w(x);
        a0 = __dadd_rn(a0, abs_sum4(x));
    }
    const double S = block_sum_dbl(__dadd_rn(a0, a1), red);
    if (threadIdx.x == 0) partial[blockIdx.x] = S;
    if (ready) pdl_wait();  // complete no earlier than the previous kernel
}

// Tree height of the per-tensor sum (the longest chain of additions any term
// goes through): a thread's chain over its float4 of a chunk (each float4
// adds 4 levels, two interleaved chains joined once), the partial kernel's
// block tree (8), the pack CTA's chain over partials and its block tree (8).
__host__ __device__ inline int absum_tree_height(int64_t chunk, int nparts) {
    const int64_t per_thread = (chunk + kPackThreads - 1) / kPackThreads;  // float4
    const int64_t parts_per_thread = (nparts + kPackThreads - 1) / kPackThreads;
    return (int)(per_thread + 4 + 1 + 8 + parts_per_thread + 8);
}

}  // namespace tq
