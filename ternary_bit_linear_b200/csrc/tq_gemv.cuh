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

constexpr int kGemvSmemCap = 96 * 1024;  // weight ring per CTA (two CTAs fit on an SM)
constexpr int kGemvMaxStages = 32;

// Shared-memory bytes of the weight ring for K (the launcher passes this as
// dynamic shared memory): as many 16-row strips as fit in kGemvSmemCap.
__host__ __device__ inline int gemv_stage_bytes(int K) { return 16 * (K / 4); }
__host__ __device__ inline int gemv_stages(int K, int64_t strips_per_cta) {
    int s = kGemvSmemCap / gemv_stage_bytes(K);
    if (s < 1) s = 1;
    if (s > kGemvMaxStages) s = kGemvMaxStages;
    return strips_per_cta < s ? (int)strips_per_cta : s;
}

// NB: token blocks of 8 (M <= 8 * NB).  W: warps per CTA; warp w owns the
// 64-byte column steps w, w + W, ... (MAXSTEP of them, K <= 256 * W * MAXSTEP).
//
// CTA b owns the contiguous strips [s0, s1) of W (a contiguous byte range of
// the packed matrix).  Thread 0 streams them, one 16-row strip per 1-D bulk
// copy, through a ring of `nstage` shared-memory stages.  With static_w (the
// packed weights are not written by the work just before this kernel on the
// stream) the first copies are issued before the programmatic-dependent-launch
// wait, so they overlap the previous kernel.
template <int NB, int MAXSTEP, int W>
__global__ void __launch_bounds__(W * 32, 1)
    gemv_kernel(const int8_t *__restrict__ xq, const float *__restrict__ s_x,
                const int32_t *__restrict__ rowsum, const uint8_t *__restrict__ packed,
                const float *__restrict__ gamma, int per_row, int M, int64_t N, int K,
                float *__restrict__ y, int32_t *__restrict__ acc_out, int static_w, int nstage) {
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ uint64_t bars[kGemvMaxStages];
    __shared__ int red[2][W][32][4 * NB];
    __shared__ float sx_s[16];
    __shared__ int rs_s[16];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int KB = K >> 2;                    // packed bytes per row
    const int nsteps = (KB + 63) >> 6;        // 64-byte column steps per row
    const int64_t nstrips = (N + 15) >> 4;
    const int64_t s0 = (int64_t)blockIdx.x * nstrips / gridDim.x;
    const int64_t s1 = (int64_t)(blockIdx.x + 1) * nstrips / gridDim.x;
    const int nmine = (int)(s1 - s0);
    const int sbytes = 16 * KB;

    pdl_trigger();
    if (threadIdx.x == 0) {
        for (int i = 0; i < nstage; ++i) mbar_init(smem_u32(&bars[i]), 1);
        fence_barrier_init();
    }
    __syncthreads();

    // thread 0: copy strip k (k-th of this CTA) into stage k % nstage
    auto issue = [&](int k) {
        const int64_t r0 = (s0 + k) * 16;
        const int64_t rows = (N - r0) < 16 ? (N - r0) : 16;
        const uint32_t bytes = (uint32_t)(rows * KB);
        const uint32_t bar = smem_u32(&bars[k % nstage]);
        mbar_arrive_expect_tx(bar, bytes);
        bulk_g2s(smem_u32(ring + (size_t)(k % nstage) * sbytes), packed + r0 * KB, bytes, bar);
    };
    const int first = nmine < nstage ? nmine : nstage;
    if (static_w && threadIdx.x == 0)
        for (int k = 0; k < first; ++k) issue(k);
    pdl_wait();
    if (!static_w && threadIdx.x == 0)
        for (int k = 0; k < first; ++k) issue(k);

    // Activation fragments for this thread's token(s) and column steps.
    uint32_t xf[NB][MAXSTEP][4][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int j = 0; j < MAXSTEP; ++j)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int step = warp + W * j;
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

    int buf = 0, issued = first, consumed = 0;
    for (int k = 0; k < nmine; ++k) {
        const bool ok = warp_wait(smem_u32(&bars[k % nstage]), (uint32_t)((k / nstage) & 1), lane);
        if (!__syncthreads_and(ok)) break;  // CTA-uniform decision
        const uint8_t *stage = ring + (size_t)(k % nstage) * sbytes;
        const int64_t row0 = (s0 + k) * 16;
        // one accumulator set per word position: four independent MMA chains
        int d4[4][NB][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) d4[i][nb][0] = d4[i][nb][1] = d4[i][nb][2] = d4[i][nb][3] = 0;
#pragma unroll
        for (int j = 0; j < MAXSTEP; ++j) {
            const int step = warp + W * j;
            const int bo = step * 64 + t * 16;
            uint4 wa = make_uint4(0u, 0u, 0u, 0u), wb = make_uint4(0u, 0u, 0u, 0u);
            if (step < nsteps && bo < KB) {
                wa = *reinterpret_cast<const uint4 *>(stage + g * KB + bo);
                wb = *reinterpret_cast<const uint4 *>(stage + (g + 8) * KB + bo);
            }
            const uint32_t wav[4] = {wa.x, wa.y, wa.z, wa.w};
            const uint32_t wbv[4] = {wb.x, wb.y, wb.z, wb.w};
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
                    mma_16x8x32_u8s8(d4[i][nb], ua[0], ub[0], ua[1], ub[1], xf[nb][j][i][0],
                                     xf[nb][j][i][1]);
                    mma_16x8x32_u8s8(d4[i][nb], ua[2], ub[2], ua[3], ub[3], xf[nb][j][i][2],
                                     xf[nb][j][i][3]);
                }
            }
        }
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
            for (int c = 0; c < 4; ++c)
                red[buf][warp][lane][nb * 4 + c] = (d4[0][nb][c] + d4[1][nb][c]) + (d4[2][nb][c] + d4[3][nb][c]);
        __syncthreads();  // every warp is done with this stage and wrote its sums
        consumed = k + 1;
        if (threadIdx.x == 0 && issued < nmine) issue(issued);
        issued = issued < nmine ? issued + 1 : issued;
        if (warp == 0) {
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    int tot = 0;
#pragma unroll
                    for (int w = 0; w < W; ++w) tot += red[buf][w][lane][nb * 4 + c];
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
    // Copies this CTA issued must have landed before it exits (already true
    // unless a wait above gave up).
    if (threadIdx.x == 0)
        for (int k = consumed; k < issued; ++k)
            mbar_wait(smem_u32(&bars[k % nstage]), (uint32_t)((k / nstage) & 1));
}

}  // namespace tq
