// tq_gemv.cuh -- small-M (decode) ternary GEMV: y = (x_q . q) * gamma * s_x.
//
// Hetman-2b, src/quantization.py, section 7 (simulate_hardware_bitnet_gemv:
// per output row, decode the packed bytes branch-free and accumulate in
// int32, then one fp32 rescale); Foundry, docs/quantization.md, "Native Matmul
// Kernel".  Here the add/subtract loop becomes an integer MMA.
//
// The kernel is bound by HBM reads of the packed weights (N*K/4 bytes), so it
// is organised around streaming them once, 16 bytes per thread per load:
//   * A CTA of 8 warps walks 16-row strips of W.  Warp w owns the fixed set of
//     64-byte column steps s = w, w + 8, ... of every row, so the activation
//     fragments it needs never change: they are loaded once into registers.
//   * Thread (g = lane/4, t = lane%4) loads 16 bytes (64 codes) of rows g and
//     g+8 per step.  A 32-bit word holds 16 codes; (word >> 2j) & 0x03030303
//     spreads codes {j, 4+j, 8+j, 12+j} into bytes as unsigned values
//     c = q + 1 in {0, 1, 2}.  The activation group is transposed the same way
//     once at start-up, so the pairing of codes and activations is exact.
//   * mma.sync m16n8k32 (u8 x s8 -> s32) reduces 32 codes per row and token;
//     sum_k x*c - sum_k x = sum_k x*q removes the offset (rowsum).
//   * The 8 warps' partial sums meet in shared memory; warp 0 writes y.
#pragma once

#include "tq_common.cuh"

namespace tq {

constexpr int kGemvWarps = 8;
constexpr int kGemvMaxK = 8192;  // 8 warps x 4 steps x 256 codes

__device__ __forceinline__ uint4 ldg_stream_u4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// 4x4 byte transpose: out word j = (in0.byte j, in1.byte j, in2.byte j, in3.byte j).
__device__ __forceinline__ uint4 transpose_bytes4x4(uint4 q) {
    const uint32_t t0 = __byte_perm(q.x, q.y, 0x5140), t1 = __byte_perm(q.x, q.y, 0x7362);
    const uint32_t t2 = __byte_perm(q.z, q.w, 0x5140), t3 = __byte_perm(q.z, q.w, 0x7362);
    return make_uint4(__byte_perm(t0, t2, 0x5410), __byte_perm(t0, t2, 0x7632),
                      __byte_perm(t1, t3, 0x5410), __byte_perm(t1, t3, 0x7632));
}

template <int NB, int MAXSTEP>
__global__ void __launch_bounds__(kGemvWarps * 32)
    gemv_kernel(const int8_t *__restrict__ xq, const float *__restrict__ s_x,
                const int32_t *__restrict__ rowsum, const uint8_t *__restrict__ packed,
                const float *__restrict__ gamma, int per_row, int M, int64_t N, int K,
                float *__restrict__ y, int32_t *__restrict__ acc_out) {
    __shared__ int red[2][kGemvWarps][32][4 * NB];
    __shared__ float sx_s[16];
    __shared__ int rs_s[16];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int KB = K >> 2;                    // packed bytes per row
    const int nsteps = (KB + 63) >> 6;        // 64-byte column steps per row
    const int64_t nstrips = (N + 15) >> 4;

    // Activation fragments for this thread's token(s) and column steps.
    uint32_t xf[NB][MAXSTEP][4][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int j = 0; j < MAXSTEP; ++j)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int step = warp + kGemvWarps * j;
                const int b = step * 64 + t * 16 + 4 * i;  // packed byte of this word
                const int m = g + 8 * nb;
                uint4 q = make_uint4(0u, 0u, 0u, 0u);
                if (step < nsteps && b < KB && m < M)
                    q = __ldg(reinterpret_cast<const uint4 *>(xq + (int64_t)m * K + 4 * b));
                const uint4 tr = transpose_bytes4x4(q);
                xf[nb][j][i][0] = tr.x;
                xf[nb][j][i][1] = tr.y;
                xf[nb][j][i][2] = tr.z;
                xf[nb][j][i][3] = tr.w;
            }
    if (threadIdx.x < 16) {
        const int m = threadIdx.x;
        sx_s[m] = m < M ? s_x[m] : 0.0f;
        rs_s[m] = m < M ? rowsum[m] : 0;
    }
    __syncthreads();

    int buf = 0;
    for (int64_t s = blockIdx.x; s < nstrips; s += gridDim.x) {
        const int64_t row0 = s * 16;
        const int64_t ra = row0 + g, rb = row0 + g + 8;
        uint4 wa[MAXSTEP], wb[MAXSTEP];
#pragma unroll
        for (int j = 0; j < MAXSTEP; ++j) {
            const int step = warp + kGemvWarps * j;
            const int b = step * 64 + t * 16;
            const bool ok = step < nsteps && b < KB;
            wa[j] = (ok && ra < N) ? ldg_stream_u4(packed + ra * KB + b) : make_uint4(0u, 0u, 0u, 0u);
            wb[j] = (ok && rb < N) ? ldg_stream_u4(packed + rb * KB + b) : make_uint4(0u, 0u, 0u, 0u);
        }
        int d[NB][4];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) d[nb][0] = d[nb][1] = d[nb][2] = d[nb][3] = 0;
#pragma unroll
        for (int j = 0; j < MAXSTEP; ++j) {
            const uint32_t wav[4] = {wa[j].x, wa[j].y, wa[j].z, wa[j].w};
            const uint32_t wbv[4] = {wb[j].x, wb[j].y, wb[j].z, wb[j].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint32_t ua[4], ub[4];
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    ua[jj] = (wav[i] >> (2 * jj)) & 0x03030303u;
                    ub[jj] = (wbv[i] >> (2 * jj)) & 0x03030303u;
                }
#pragma unroll
                for (int nb = 0; nb < NB; ++nb) {
                    mma_16x8x32_u8s8(d[nb], ua[0], ub[0], ua[1], ub[1], xf[nb][j][i][0],
                                     xf[nb][j][i][1]);
                    mma_16x8x32_u8s8(d[nb], ua[2], ub[2], ua[3], ub[3], xf[nb][j][i][2],
                                     xf[nb][j][i][3]);
                }
            }
        }
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
            for (int c = 0; c < 4; ++c) red[buf][warp][lane][nb * 4 + c] = d[nb][c];
        __syncthreads();
        if (warp == 0) {
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    int tot = 0;
#pragma unroll
                    for (int w = 0; w < kGemvWarps; ++w) tot += red[buf][w][lane][nb * 4 + c];
                    // fragment c: row g (+8 for c >= 2), token 2t + (c & 1)
                    const int m = 8 * nb + 2 * t + (c & 1);
                    const int64_t n = row0 + g + ((c & 2) ? 8 : 0);
                    if (m < M && n < N) {
                        const int a = tot - rs_s[m];
                        const float gn = per_row ? __ldg(gamma + n) : __ldg(gamma);
                        y[(int64_t)m * N + n] = __fmul_rn(__int2float_rn(a), __fmul_rn(gn, sx_s[m]));
                        if (acc_out) acc_out[(int64_t)m * N + n] = a;
                    }
                }
        }
        buf ^= 1;
    }
}

}  // namespace tq
