// tq_act.cuh -- per-token int8 quantisation, RMSNorm and the blockwise
// FWHT-512 (standalone, and fused as the prologue of the whole layer).
//
// Hetman-2b, src/quantization.py:
//   section 1  fast_walsh_hadamard_transform_512 / blockwise_fwht_forward:
//              stages h = 1, 2, ..., 256 of (a + b, a - b) in fp32, then a
//              multiply by fp32(1/sqrt(512)).  The kernels below perform
//              exactly these fp32 operations on the same operands, so their
//              results are bit-identical to that stage order.
//   section 2  SymmetricActivationQuantizer.forward: eta = max|x| (>= 1e-6,
//              optionally clamped), scale = 127/eta, x_q = clamp(round(x*scale)).
//   section 4  SubLayerRMSNorm.forward: x * rsqrt(mean(x^2) + eps) * g.
//   section 5  BitLinear.forward step 0: quench nan -> 0, +-inf -> +-eta_max.
//
// Layout of a 512-block inside one warp: lane l holds the 16 elements
//   i = 128*j + 4*l + e   (j, e in 0..3)
// loaded as four coalesced float4 (one per j).  Stages h = 1, 2 pair elements
// inside a float4 (bit 0/1 of i = e), h = 4..64 pair lanes (bits 2..6 = lane
// bits 0..4, exchanged with shfl.xor), h = 128, 256 pair float4s (j bits).
#pragma once

#include "tq_common.cuh"

namespace tq {

constexpr int kActThreads = 256;

struct ActParams {
    int sanitize;    // quench non-finite inputs (nan -> 0, +-inf -> +-eta_max)
    int clamp_eta;   // clamp eta to [eta_min, eta_max]
    float eta_min, eta_max;
    int rmsnorm;     // (fused prologue only)
    float rms_eps;
    const float *rms_gain;  // [K] or nullptr
    int ready;       // inputs complete and outputs untouched by work in flight:
                     // read at once, wait for the previous kernel before exiting
};

__device__ __forceinline__ float quench(float x, float eta_max) {
    if (x != x) return 0.0f;
    if (isinf(x)) return x > 0.0f ? eta_max : -eta_max;
    return x;
}

// round half to even, clamp to [-127, 127]; NaN -> 0
__device__ __forceinline__ int quant_code(float x, float scale) {
    const float t = rintf(__fmul_rn(x, scale));
    if (t != t) return 0;
    return (int)fminf(fmaxf(t, -127.0f), 127.0f);
}

__device__ __forceinline__ float eta_of(float amax, const ActParams &p) {
    float eta = amax > 1e-6f ? amax : 1e-6f;
    if (p.clamp_eta) eta = fminf(fmaxf(eta, p.eta_min), p.eta_max);
    return eta;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
    return v;
}
__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// Block-wide reductions in a fixed order; result valid in every thread.
// `red` needs 32 slots.
template <int NT>
__device__ __forceinline__ float block_max(float v, float *red) {
    v = warp_max(v);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float t = lane < NT / 32 ? red[lane] : 0.0f;
    t = warp_max(t);
    __syncthreads();
    return t;
}
template <int NT>
__device__ __forceinline__ int block_sum_i(int v, int *red) {
    v = warp_sum_i(v);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    int t = lane < NT / 32 ? red[lane] : 0;
    t = warp_sum_i(t);
    __syncthreads();
    return t;
}
template <int NT>
__device__ __forceinline__ double block_sum_d(double v, double *red) {
    v = warp_sum_d(v);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    double t = lane < NT / 32 ? red[lane] : 0.0;
    t = warp_sum_d(t);
    __syncthreads();
    return t;
}

__device__ __forceinline__ uint32_t pack_codes4(int a, int b, int c, int d) {
    return (uint32_t)(a & 0xff) | ((uint32_t)(b & 0xff) << 8) | ((uint32_t)(c & 0xff) << 16) |
           ((uint32_t)(d & 0xff) << 24);
}

// x * r * g in fp64, rounded once (RMSNorm output of one element).
__device__ __forceinline__ float rms_apply(float x, double r, const float *gain, int k) {
    const double g = gain ? (double)__ldg(gain + k) : 1.0;
    return __double2float_rn(__dmul_rn(__dmul_rn((double)x, r), g));
}

// ---------------------------------------------------------------------------
// Per-token quantisation (optionally after RMSNorm) of one row that a CTA of
// kActThreads holds in registers: thread tid has float4 tid + i * kActThreads
// (i < VEC; zeros past the row).  Writes x_q, s_x[m] and rowsum[m].
//
// XT: x_q in the layout the grouped small-M GEMV copies straight into shared
// memory -- each 16-byte chunk 4x4-byte transposed (word j holds elements
// 16c + j, 16c + 4 + j, 16c + 8 + j, 16c + 12 + j) and stored at chunk position
// gemv_chunk_pos(c).  The four words of a chunk sit in four consecutive lanes
// (kActThreads is a multiple of 4), which exchange them by shuffles.
// ---------------------------------------------------------------------------
template <int VEC, bool XT = false>
__device__ __forceinline__ void act_row_regs(float4 (&v)[VEC], int K, const ActParams &p, int64_t m,
                                             int8_t *__restrict__ xq, float *__restrict__ s_x,
                                             int32_t *__restrict__ rowsum, float *redf, int *redi,
                                             double *redd) {
    const int nv = K >> 2, tid = threadIdx.x;
    uint32_t *dst = reinterpret_cast<uint32_t *>(xq + m * (int64_t)K);
    if (p.rmsnorm) {
        double ss = 0.0;
#pragma unroll
        for (int i = 0; i < VEC; ++i) {
            ss = __fma_rn((double)v[i].x, (double)v[i].x, ss);
            ss = __fma_rn((double)v[i].y, (double)v[i].y, ss);
            ss = __fma_rn((double)v[i].z, (double)v[i].z, ss);
            ss = __fma_rn((double)v[i].w, (double)v[i].w, ss);
        }
        ss = block_sum_d<kActThreads>(ss, redd);
        const double r = __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(__ddiv_rn(ss, (double)K), (double)p.rms_eps)));
#pragma unroll
        for (int i = 0; i < VEC; ++i) {
            const int k = 4 * (tid + i * kActThreads);
            v[i] = make_float4(rms_apply(v[i].x, r, p.rms_gain, k), rms_apply(v[i].y, r, p.rms_gain, k + 1),
                               rms_apply(v[i].z, r, p.rms_gain, k + 2),
                               rms_apply(v[i].w, r, p.rms_gain, k + 3));
        }
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < VEC; ++i)
        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v[i].x), fabsf(v[i].y)), fmaxf(fabsf(v[i].z), fabsf(v[i].w))));
    amax = block_max<kActThreads>(amax, redf);
    const float eta = eta_of(amax, p);
    const float scale = __fdiv_rn(127.0f, eta);
    int sum = 0;
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
        const int idx = tid + i * kActThreads;
        // past the row (K % 64 == 0: whole chunks, whole lane quads) the codes are 0
        const int a = quant_code(v[i].x, scale), b = quant_code(v[i].y, scale),
                  c = quant_code(v[i].z, scale), d = quant_code(v[i].w, scale);
        uint32_t word = pack_codes4(a, b, c, d);
        if (XT) {
            const int q0 = (threadIdx.x & 31) & ~3;
            uint4 q;
            q.x = __shfl_sync(0xffffffffu, word, q0);
            q.y = __shfl_sync(0xffffffffu, word, q0 + 1);
            q.z = __shfl_sync(0xffffffffu, word, q0 + 2);
            q.w = __shfl_sync(0xffffffffu, word, q0 + 3);
            const uint4 t = transpose_bytes4x4(q);
            const int j = idx & 3;
            word = j == 0 ? t.x : j == 1 ? t.y : j == 2 ? t.z : t.w;
        }
        if (idx < nv) {
            dst[XT ? 4 * gemv_chunk_pos(idx >> 2) + (idx & 3) : idx] = word;
            sum += a + b + c + d;
        }
    }
    sum = block_sum_i<kActThreads>(sum, redi);
    if (tid == 0) {
        s_x[m] = __fdiv_rn(eta, 127.0f);
        if (rowsum) rowsum[m] = sum;
    }
}

__device__ __forceinline__ float4 quench4(float4 v, const ActParams &p) {
    return make_float4(quench(v.x, p.eta_max), quench(v.y, p.eta_max), quench(v.z, p.eta_max),
                       quench(v.w, p.eta_max));
}

// One CTA per token.  VEC > 0: the row lives in registers (K <= 1024*VEC);
// VEC == 0: streamed (two passes over the row, the second from cache).
// XT: x_q in the grouped GEMV's layout (see act_row_regs; VEC > 0 only).
template <int VEC, bool XT = false>
__global__ void __launch_bounds__(kActThreads)
    tq_act_quant_kernel(const float *__restrict__ x, int K, ActParams p, int8_t *__restrict__ xq,
                     float *__restrict__ s_x, int32_t *__restrict__ rowsum) {
    static_assert(!XT || VEC > 0, "the GEMV layout is written from registers");
    __shared__ float redf[32];
    __shared__ int redi[32];
    __shared__ double redd[32];
    if (!p.ready) pdl_wait();
    pdl_trigger();
    const int64_t m = blockIdx.x;
    const int nv = K >> 2, tid = threadIdx.x;
    const float4 *src = reinterpret_cast<const float4 *>(x + m * (int64_t)K);
    auto load = [&](int idx) {
        float4 v = __ldg(src + idx);
        if (p.sanitize) v = quench4(v, p);
        return v;
    };
    if (VEC > 0) {
        constexpr int V = VEC > 0 ? VEC : 1;
        float4 v[V];
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int idx = tid + i * kActThreads;
            v[i] = idx < nv ? load(idx) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        act_row_regs<V, XT>(v, K, p, m, xq, s_x, rowsum, redf, redi, redd);
        if (p.ready) pdl_wait();  // complete no earlier than the previous kernel
        return;
    }
    uint32_t *dst = reinterpret_cast<uint32_t *>(xq + m * (int64_t)K);
    double r = 1.0;
    if (p.rmsnorm) {
        double ss = 0.0;
        for (int idx = tid; idx < nv; idx += kActThreads) {
            const float4 t = load(idx);
            ss = __fma_rn((double)t.x, (double)t.x, ss);
            ss = __fma_rn((double)t.y, (double)t.y, ss);
            ss = __fma_rn((double)t.z, (double)t.z, ss);
            ss = __fma_rn((double)t.w, (double)t.w, ss);
        }
        ss = block_sum_d<kActThreads>(ss, redd);
        r = __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(__ddiv_rn(ss, (double)K), (double)p.rms_eps)));
    }
    auto normed = [&](int idx) {
        float4 t = load(idx);
        if (p.rmsnorm) {
            const int k = 4 * idx;
            t = make_float4(rms_apply(t.x, r, p.rms_gain, k), rms_apply(t.y, r, p.rms_gain, k + 1),
                            rms_apply(t.z, r, p.rms_gain, k + 2), rms_apply(t.w, r, p.rms_gain, k + 3));
        }
        return t;
    };
    float amax = 0.0f;
    for (int idx = tid; idx < nv; idx += kActThreads) {
        const float4 t = normed(idx);
        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(t.x), fabsf(t.y)), fmaxf(fabsf(t.z), fabsf(t.w))));
    }
    amax = block_max<kActThreads>(amax, redf);
    const float eta = eta_of(amax, p);
    const float scale = __fdiv_rn(127.0f, eta);
    int sum = 0;
    for (int idx = tid; idx < nv; idx += kActThreads) {
        const float4 t = normed(idx);
        const int a = quant_code(t.x, scale), b = quant_code(t.y, scale), c = quant_code(t.z, scale),
                  d = quant_code(t.w, scale);
        dst[idx] = pack_codes4(a, b, c, d);
        sum += a + b + c + d;
    }
    sum = block_sum_i<kActThreads>(sum, redi);
    if (tid == 0) {
        s_x[m] = __fdiv_rn(eta, 127.0f);
        if (rowsum) rowsum[m] = sum;
    }
    if (p.ready) pdl_wait();  // complete no earlier than the previous kernel
}

// Many tokens (K <= 1024*VEC): a persistent grid; each CTA streams its tokens
// m = blockIdx.x + j * gridDim.x through a ring of kActRing shared-memory row
// buffers filled by 1-D bulk copies kActRing - 1 rows ahead, so HBM latency
// hides behind the work on earlier rows.
constexpr int kActRing = 4;

template <int VEC>
__global__ void __launch_bounds__(kActThreads)
    tq_act_ring_kernel(const float *__restrict__ x, int64_t M, int K, ActParams p,
                    int8_t *__restrict__ xq, float *__restrict__ s_x, int32_t *__restrict__ rowsum) {
    extern __shared__ __align__(16) float4 rowbuf[];  // [kActRing][nv]
    __shared__ uint64_t rbar[kActRing];
    __shared__ float redf[32];
    __shared__ int redi[32];
    __shared__ double redd[32];
    const int nv = K >> 2, tid = threadIdx.x, lane = tid & 31;
    const int64_t nmine = (int64_t)blockIdx.x < M ? (M - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    if (tid == 0) {
        for (int r = 0; r < kActRing; ++r) mbar_init(smem_u32(&rbar[r]), 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (!p.ready) pdl_wait();
    pdl_trigger();
    auto issue = [&](int64_t j) {  // thread 0: token j of this CTA into buffer j % kActRing
        const uint32_t bar = smem_u32(&rbar[j % kActRing]);
        mbar_arrive_expect_tx(bar, (uint32_t)(nv * 16));
        bulk_g2s(smem_u32(rowbuf + (j % kActRing) * nv), x + ((int64_t)blockIdx.x + j * gridDim.x) * K,
                 (uint32_t)(nv * 16), bar);
    };
    int64_t issued = nmine < kActRing ? nmine : kActRing;
    if (tid == 0)
        for (int64_t j = 0; j < issued; ++j) issue(j);
    int64_t j = 0;
    for (; j < nmine; ++j) {
        const bool ok = warp_wait(smem_u32(&rbar[j % kActRing]), (uint32_t)((j / kActRing) & 1), lane);
        const float4 *src = rowbuf + (j % kActRing) * nv;
        float4 v[VEC];
#pragma unroll
        for (int i = 0; i < VEC; ++i) {
            const int idx = tid + i * kActThreads;
            v[i] = idx < nv ? src[idx] : make_float4(0.f, 0.f, 0.f, 0.f);
            if (p.sanitize) v[i] = quench4(v[i], p);
        }
        if (!__syncthreads_and(ok)) break;  // buffer read by all; CTA-uniform timeout decision
        if (tid == 0 && issued < nmine) issue(issued);
        issued = issued < nmine ? issued + 1 : issued;
        act_row_regs<VEC>(v, K, p, (int64_t)blockIdx.x + j * gridDim.x, xq, s_x, rowsum, redf, redi, redd);
    }
    // Copies in flight must land before the CTA exits (already true unless a
    // wait gave up).
    if (tid == 0)
        for (int64_t u = j; u < issued; ++u) mbar_wait(smem_u32(&rbar[u % kActRing]), (uint32_t)((u / kActRing) & 1));
    if (p.ready) pdl_wait();  // complete no earlier than the previous kernel
}

// ---------------------------------------------------------------------------
// FWHT-512 of the 16 values a warp lane holds (layout in the file header).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void butterfly(float &a, float &b) {
    const float s = __fadd_rn(a, b), d = __fsub_rn(a, b);
    a = s;
    b = d;
}

__device__ __forceinline__ void fwht512_regs(float (&f)[16], bool normalize) {
    const int lane = threadIdx.x & 31;
    // h = 1 (e bit 0), h = 2 (e bit 1)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        butterfly(f[4 * j + 0], f[4 * j + 1]);
        butterfly(f[4 * j + 2], f[4 * j + 3]);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        butterfly(f[4 * j + 0], f[4 * j + 2]);
        butterfly(f[4 * j + 1], f[4 * j + 3]);
    }
    // h = 4 .. 64: partner lane = lane ^ s; the lane with the bit clear holds a
#pragma unroll
    for (int s = 1; s < 32; s <<= 1) {
        const bool upper = (lane & s) != 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float o = __shfl_xor_sync(0xffffffffu, f[i], s);
            f[i] = upper ? __fsub_rn(o, f[i]) : __fadd_rn(f[i], o);
        }
    }
    // h = 128 (j bit 0), h = 256 (j bit 1)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        butterfly(f[0 + e], f[4 + e]);
        butterfly(f[8 + e], f[12 + e]);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        butterfly(f[0 + e], f[8 + e]);
        butterfly(f[4 + e], f[12 + e]);
    }
    if (normalize) {
        const float c = __int_as_float(0x3D3504F3);  // fp32(1/sqrt(512))
#pragma unroll
        for (int i = 0; i < 16; ++i) f[i] = __fmul_rn(f[i], c);
    }
}

// Standalone transform: one warp per 512-block, 8 warps per CTA.
__global__ void __launch_bounds__(256)
    tq_fwht512_kernel(const float *x, float *y, int64_t nblocks, int normalize) {
    pdl_wait();
    pdl_trigger();
    const int64_t blk = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (blk >= nblocks) return;
    const int lane = threadIdx.x & 31;
    const float4 *src = reinterpret_cast<const float4 *>(x + blk * 512);
    float4 *dst = reinterpret_cast<float4 *>(y + blk * 512);
    float f[16];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float4 v = src[j * 32 + lane];
        f[4 * j + 0] = v.x;
        f[4 * j + 1] = v.y;
        f[4 * j + 2] = v.z;
        f[4 * j + 3] = v.w;
    }
    fwht512_regs(f, normalize != 0);
#pragma unroll
    for (int j = 0; j < 4; ++j)
        dst[j * 32 + lane] = make_float4(f[4 * j + 0], f[4 * j + 1], f[4 * j + 2], f[4 * j + 3]);
}

// ---------------------------------------------------------------------------
// Hetman-2b section 1 FastWalshHadamardTransform.forward: the module's int8
// round trip between two rotations.  One CTA per row, one warp per 512-block
// (K = 512 * blockDim.x / 32): quench (nan -> 0, +-inf -> +-eta_max), FWHT,
// eta = max|x_rot| + 1e-5 clamped to [eta_min, eta_max], x_q =
// clamp(round(x_rot * fp32(127 / eta)), +-127), dequantised by fp32(eta / 127),
// FWHT again -- every step the fp32 operation the definition names, so the
// result is bit-identical to it.  y may alias x (a CTA reads its row before
// it writes it).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024)
    tq_fwht_roundtrip_kernel(const float *x, float *y, float eta_min, float eta_max,
                          float *__restrict__ eta_out) {
    __shared__ float redf[32];
    pdl_wait();
    pdl_trigger();
    const int nw = blockDim.x >> 5, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t K = 512 * (int64_t)nw;
    const float *row = x + (int64_t)blockIdx.x * K + warp * 512;
    float f[16];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float4 v = reinterpret_cast<const float4 *>(row)[j * 32 + lane];
        f[4 * j + 0] = quench(v.x, eta_max);
        f[4 * j + 1] = quench(v.y, eta_max);
        f[4 * j + 2] = quench(v.z, eta_max);
        f[4 * j + 3] = quench(v.w, eta_max);
    }
    fwht512_regs(f, true);
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(f[i]));
    amax = warp_max(amax);
    if (lane == 0) redf[warp] = amax;
    __syncthreads();
    amax = warp_max(lane < nw ? redf[lane] : 0.0f);
    const float eta = fminf(fmaxf(__fadd_rn(amax, 1e-5f), eta_min), eta_max);
    const float scale = __fdiv_rn(127.0f, eta), back = __fdiv_rn(eta, 127.0f);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float q = fminf(fmaxf(rintf(__fmul_rn(f[i], scale)), -127.0f), 127.0f);
        f[i] = __fmul_rn(q, back);
    }
    fwht512_regs(f, true);
    float4 *dst = reinterpret_cast<float4 *>(y + (int64_t)blockIdx.x * K + warp * 512);
#pragma unroll
    for (int j = 0; j < 4; ++j) dst[j * 32 + lane] = make_float4(f[4 * j + 0], f[4 * j + 1], f[4 * j + 2], f[4 * j + 3]);
    if (eta_out && threadIdx.x == 0) eta_out[blockIdx.x] = eta;
}

// ---------------------------------------------------------------------------
// Between the projections of Hetman-2b's clamped SwiGLU (section 6,
// SwiGLUClamped.forward), fused with the down projection's activation pass:
// a = clamp(SiLU(gate) * up, +-clamp_val) (SiLU(v) = v / (1 + e^-v), fp32),
// then [quench] -> [RMSNorm] -> FWHT-512 -> per-token int8, as
// tq_prologue_fwht_kernel.  One CTA per token, one warp per 512-block
// (K = 512 * blockDim.x / 32).  act_out (or NULL) receives a.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float swiglu_one(float g, float u, float c) {
    const float a = __fmul_rn(__fdiv_rn(g, __fadd_rn(1.0f, expf(-g))), u);
    return fminf(fmaxf(a, -c), c);
}

__global__ void __launch_bounds__(1024)
    tq_swiglu_prologue_kernel(const float *__restrict__ gate, const float *__restrict__ up, float clamp_val,
                           ActParams p, int8_t *__restrict__ xq, float *__restrict__ s_x,
                           int32_t *__restrict__ rowsum, float *__restrict__ act_out) {
    __shared__ float redf[32];
    __shared__ int redi[32];
    __shared__ double redd[32];
    pdl_wait();
    pdl_trigger();
    const int nw = blockDim.x >> 5, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t K = 512 * (int64_t)nw;
    const int64_t m = blockIdx.x;
    const int64_t off = m * K + warp * 512;
    float f[16];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float4 g = reinterpret_cast<const float4 *>(gate + off)[j * 32 + lane];
        const float4 u = reinterpret_cast<const float4 *>(up + off)[j * 32 + lane];
        float4 a = make_float4(swiglu_one(g.x, u.x, clamp_val), swiglu_one(g.y, u.y, clamp_val),
                               swiglu_one(g.z, u.z, clamp_val), swiglu_one(g.w, u.w, clamp_val));
        if (act_out) reinterpret_cast<float4 *>(act_out + off)[j * 32 + lane] = a;
        if (p.sanitize)
            a = make_float4(quench(a.x, p.eta_max), quench(a.y, p.eta_max), quench(a.z, p.eta_max),
                            quench(a.w, p.eta_max));
        f[4 * j + 0] = a.x;
        f[4 * j + 1] = a.y;
        f[4 * j + 2] = a.z;
        f[4 * j + 3] = a.w;
    }
    if (p.rmsnorm) {
        double ss = 0.0;
#pragma unroll
        for (int i = 0; i < 16; ++i) ss = __fma_rn((double)f[i], (double)f[i], ss);
        ss = warp_sum_d(ss);
        if (lane == 0) redd[warp] = ss;
        __syncthreads();
        ss = warp_sum_d(lane < nw ? redd[lane] : 0.0);
        const double r =
            __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(__ddiv_rn(ss, (double)K), (double)p.rms_eps)));
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int k = warp * 512 + j * 128 + lane * 4 + e;
                f[4 * j + e] = rms_apply(f[4 * j + e], r, p.rms_gain, k);
            }
    }
    fwht512_regs(f, true);
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(f[i]));
    amax = warp_max(amax);
    if (lane == 0) redf[warp] = amax;
    __syncthreads();
    amax = warp_max(lane < nw ? redf[lane] : 0.0f);
    const float eta = eta_of(amax, p);
    const float scale = __fdiv_rn(127.0f, eta);
    int sum = 0;
    uint32_t *dst = reinterpret_cast<uint32_t *>(xq + off);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int a = quant_code(f[4 * j + 0], scale), b = quant_code(f[4 * j + 1], scale),
                  c = quant_code(f[4 * j + 2], scale), d = quant_code(f[4 * j + 3], scale);
        dst[j * 32 + lane] = pack_codes4(a, b, c, d);
        sum += a + b + c + d;
    }
    sum = warp_sum_i(sum);
    if (lane == 0) redi[warp] = sum;
    __syncthreads();
    if (threadIdx.x < 32) {
        sum = warp_sum_i(lane < nw ? redi[lane] : 0);
        if (lane == 0) {
            s_x[m] = __fdiv_rn(eta, 127.0f);
            rowsum[m] = sum;
        }
    }
}

// ---------------------------------------------------------------------------
// Fused prologue of the whole layer: [quench] -> [RMSNorm] -> FWHT-512 ->
// per-token int8.  One CTA per token, one warp per 512-block (K = 512 * NW).
// ---------------------------------------------------------------------------
template <int NW>
__global__ void __launch_bounds__(NW * 32)
    tq_prologue_fwht_kernel(const float *__restrict__ x, ActParams p, int8_t *__restrict__ xq,
                         float *__restrict__ s_x, int32_t *__restrict__ rowsum) {
    __shared__ float redf[32];
    __shared__ int redi[32];
    __shared__ double redd[32];
    constexpr int K = 512 * NW;
    if (!p.ready) pdl_wait();
    pdl_trigger();
    const int64_t m = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float *row = x + m * (int64_t)K + warp * 512;
    float f[16];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float4 v = __ldg(reinterpret_cast<const float4 *>(row) + j * 32 + lane);
        if (p.sanitize)
            v = make_float4(quench(v.x, p.eta_max), quench(v.y, p.eta_max), quench(v.z, p.eta_max),
                            quench(v.w, p.eta_max));
        f[4 * j + 0] = v.x;
        f[4 * j + 1] = v.y;
        f[4 * j + 2] = v.z;
        f[4 * j + 3] = v.w;
    }
    if (p.rmsnorm) {
        double ss = 0.0;
#pragma unroll
        for (int i = 0; i < 16; ++i) ss = __fma_rn((double)f[i], (double)f[i], ss);
        ss = block_sum_d<NW * 32>(ss, redd);
        const double r =
            __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(__ddiv_rn(ss, (double)K), (double)p.rms_eps)));
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int k = warp * 512 + j * 128 + lane * 4 + e;
                f[4 * j + e] = rms_apply(f[4 * j + e], r, p.rms_gain, k);
            }
    }
    fwht512_regs(f, true);
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(f[i]));
    amax = block_max<NW * 32>(amax, redf);
    const float eta = eta_of(amax, p);
    const float scale = __fdiv_rn(127.0f, eta);
    int sum = 0;
    uint32_t *dst = reinterpret_cast<uint32_t *>(xq + m * (int64_t)K + warp * 512);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int a = quant_code(f[4 * j + 0], scale), b = quant_code(f[4 * j + 1], scale),
                  c = quant_code(f[4 * j + 2], scale), d = quant_code(f[4 * j + 3], scale);
        dst[j * 32 + lane] = pack_codes4(a, b, c, d);
        sum += a + b + c + d;
    }
    sum = block_sum_i<NW * 32>(sum, redi);
    if (threadIdx.x == 0) {
        s_x[m] = __fdiv_rn(eta, 127.0f);
        rowsum[m] = sum;
    }
    // Inputs ready: complete no earlier than the previous kernel (one CTA
    // waits; the others free their slots at once).
    if (p.ready && blockIdx.x == gridDim.x - 1) pdl_wait();
}

}  // namespace tq
