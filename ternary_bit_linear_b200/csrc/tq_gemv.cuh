// tq_gemv.cuh -- small-M (decode) ternary GEMV: y = (x_q . q) * gamma * s_x.
//
// Hetman-2b, src/quantization.py, section 7 (simulate_hardware_bitnet_gemv:
// per output row, decode the packed bytes branch-free and accumulate in
// int32, then one fp32 rescale); Foundry, docs/quantization.md, "Native Matmul
// Kernel".  Here the add/subtract loop becomes an integer MMA.
//
// The kernel is bound by HBM reads of the packed weights (N*K/4 bytes), and in
// a chain of layers by the latency from "previous kernel done" to "y stored",
// so it is organised around streaming the weights once and keeping that chain
// short:
//   * A CTA owns a contiguous run of 16-row strips of W.  Warp 0 requests them
//     with 1-D bulk copies, one per row, into a shared-memory ring whose rows
//     are padded so that rows g and g + 8 fall in different banks.
//   * x_q (M rows, at most 16) is bulk-copied once into shared memory (padded
//     rows); nothing of it lives in registers, which keeps the kernel small
//     enough for several layers' CTAs to be resident at once.
//   * Warp w takes the 64-byte column steps w, w + W, ... of the strip.
//     Thread (g = lane/4, t = lane%4) reads 16 bytes (64 codes) of rows g and
//     g + 8 per step.  A 32-bit word holds 16 codes; (word >> 2j) & 0x03030303
//     spreads codes {j, 4+j, 8+j, 12+j} into bytes as unsigned values
//     c = q + 1 in {0, 1, 2}; the matching 16 activations are transposed the
//     same way, so the pairing of codes and activations is exact.
//   * mma.sync m16n8k32 (u8 x s8 -> s32) reduces 32 codes per row and token;
//     sum_k x*c - sum_k x = sum_k x*q removes the offset (rowsum).
//   * The W warps' partial sums meet in shared memory; warp 0 writes y.
#pragma once

#include "tq_common.cuh"

namespace tq {

constexpr int kGemvMaxK = 8192;
constexpr int kGemvMaxStages = 8;
constexpr int kGemvSmemCap = 200 * 1024;

// Padded shared-memory row strides: weight rows are 64 bytes off a multiple of
// 128 (rows g and g + 8 of one quarter-warp then use disjoint banks), x rows 32.
__host__ __device__ inline int gemv_w_stride(int K) {
    const int kb = K / 4;
    return kb + ((64 - kb % 128) + 128) % 128;
}
__host__ __device__ inline int gemv_x_stride(int K) { return K + ((32 - K % 128) + 128) % 128; }
__host__ __device__ inline int gemv_stage_bytes(int K) { return 16 * gemv_w_stride(K); }
__host__ __device__ inline int gemv_x_bytes(int M, int K) { return M * gemv_x_stride(K); }

// 4x4 byte transpose: out word j = (in0.byte j, in1.byte j, in2.byte j, in3.byte j).
__device__ __forceinline__ uint4 transpose_bytes4x4(uint4 q) {
    const uint32_t t0 = __byte_perm(q.x, q.y, 0x5140), t1 = __byte_perm(q.x, q.y, 0x7362);
    const uint32_t t2 = __byte_perm(q.z, q.w, 0x5140), t3 = __byte_perm(q.z, q.w, 0x7362);
    return make_uint4(__byte_perm(t0, t2, 0x5410), __byte_perm(t0, t2, 0x7632),
                      __byte_perm(t1, t3, 0x5410), __byte_perm(t1, t3, 0x7632));
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "r"(addr)
                 : "memory");
    return r;
}

// NB: token blocks of 8 (M <= 8 * NB).  W: warps per CTA (at least 2).
//
// CTA b owns strips [b * per_cta, min((b + 1) * per_cta, nstrips)) and streams
// them through `nstage` ring stages.
//
// mode & kModeWeightsStatic: the packed weights and gamma are not written by
// work still in flight on the stream, so the first copies and the first
// strip's gamma are requested before the programmatic-dependent-launch wait
// and overlap the previous kernel.  mode & kModeInputsReady: no input is
// written, and no output touched, by work still in flight; the kernel then
// does not wait before reading at all, and waits for its predecessor only
// before it exits, which keeps the stream's completion order.
template <int NB, int W>
__global__ void __launch_bounds__(W * 32, (NB == 1 ? 1024 : 512) / (W * 32))
    gemv_kernel(const int8_t *__restrict__ xq, const float *__restrict__ s_x,
                const int32_t *__restrict__ rowsum, const uint8_t *__restrict__ packed,
                const float *__restrict__ gamma, int per_row, int M, int64_t N, int K,
                float *__restrict__ y, int32_t *__restrict__ acc_out, int mode, int nstage,
                int per_cta) {
    static_assert(W >= 2, "warp 1 copies x_q");
    extern __shared__ __align__(128) uint8_t dsm[];
    __shared__ uint64_t bars[kGemvMaxStages];
    __shared__ uint64_t xbar;
    __shared__ int red[2][W][32][4 * NB];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int KB = K >> 2;               // packed bytes per row
    const int nsteps = (KB + 63) >> 6;   // 64-byte column steps per row
    const int WS = gemv_w_stride(K), XS = gemv_x_stride(K);
    const int64_t nstrips = (N + 15) >> 4;
    const int64_t s0 = (int64_t)blockIdx.x * per_cta;
    const int64_t s1 = (s0 + per_cta) < nstrips ? (s0 + per_cta) : nstrips;
    const int nmine = (int)(s1 - s0);
    const uint32_t x_s = smem_u32(dsm);
    const uint32_t ring = x_s + (uint32_t)gemv_x_bytes(M, K);
    const int sbytes = 16 * WS;

    pdl_trigger();
    if (threadIdx.x == 0) {
        for (int i = 0; i < nstage; ++i) mbar_init(smem_u32(&bars[i]), 1);
        mbar_init(smem_u32(&xbar), 1);
        fence_barrier_init();
    }
    __syncthreads();

    // warp 0: copy strip k (k-th of this CTA) into stage k % nstage, one row per lane
    auto issue = [&](int k) {
        const int64_t r0 = (s0 + k) * 16;
        const int rows = (N - r0) < 16 ? (int)(N - r0) : 16;
        const uint32_t bar = smem_u32(&bars[k % nstage]);
        if (lane == 0) mbar_arrive_expect_tx(bar, (uint32_t)(rows * KB));
        __syncwarp();
        if (lane < rows)
            bulk_g2s(ring + (uint32_t)((k % nstage) * sbytes + lane * WS), packed + (r0 + lane) * KB,
                     (uint32_t)KB, bar);
    };
    // warp 1: x_q rows into padded shared memory, one row per lane
    auto issue_x = [&]() {
        if (lane == 0) mbar_arrive_expect_tx(smem_u32(&xbar), (uint32_t)(M * K));
        __syncwarp();
        if (lane < M)
            bulk_g2s(x_s + (uint32_t)(lane * XS), xq + (int64_t)lane * K, (uint32_t)K, smem_u32(&xbar));
    };
    auto gamma_of = [&](int64_t n) { return n < N ? __ldg(gamma + (per_row ? n : 0)) : 0.0f; };

    const int first = nmine < nstage ? nmine : nstage;
    const bool early_w = (mode & (kModeWeightsStatic | kModeInputsReady)) != 0;
    float ga = 0.0f, gb = 0.0f;  // gamma of rows g and g + 8 of the current strip (warp 0)
    if (early_w && warp == 0) {
        for (int k = 0; k < first; ++k) issue(k);
        ga = gamma_of(s0 * 16 + g);
        gb = gamma_of(s0 * 16 + g + 8);
    }
    if (!(mode & kModeInputsReady)) pdl_wait();
    if (warp == 1) issue_x();
    if (!early_w && warp == 0) {
        for (int k = 0; k < first; ++k) issue(k);
        ga = gamma_of(s0 * 16 + g);
        gb = gamma_of(s0 * 16 + g + 8);
    }
    // token scales for warp 0's outputs: fragment c -> token 8 nb + 2 t + (c & 1)
    float sxv[NB][2];
    int rsv[NB][2];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const int m = 8 * nb + 2 * t + c;
            sxv[nb][c] = (warp == 0 && m < M) ? __ldg(s_x + m) : 0.0f;
            rsv[nb][c] = (warp == 0 && m < M) ? __ldg(rowsum + m) : 0;
        }

    const bool x_ok = warp_wait(smem_u32(&xbar), 0, lane);
    int buf = 0, issued = first, consumed = 0;
    for (int k = 0; k < nmine; ++k) {
        const bool ok = x_ok && warp_wait(smem_u32(&bars[k % nstage]), (uint32_t)((k / nstage) & 1), lane);
        if (!__syncthreads_and(ok)) break;  // CTA-uniform decision
        const uint32_t stage = ring + (uint32_t)((k % nstage) * sbytes);
        const int64_t row0 = (s0 + k) * 16;
        float na = 0.0f, nbg = 0.0f;  // next strip's gamma, requested now
        if (warp == 0 && k + 1 < nmine) {
            na = gamma_of(row0 + 16 + g);
            nbg = gamma_of(row0 + 16 + g + 8);
        }
        // one accumulator set per word position: four independent MMA chains
        int d4[4][NB][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) d4[i][nb][0] = d4[i][nb][1] = d4[i][nb][2] = d4[i][nb][3] = 0;
#pragma unroll 2
        for (int step = warp; step < nsteps; step += W) {
            const int bo = step * 64 + t * 16;  // packed byte of this thread's 16 bytes
            uint4 wa = make_uint4(0u, 0u, 0u, 0u), wb = wa;
            if (bo < KB) {
                wa = lds128(stage + (uint32_t)(g * WS + bo));
                wb = lds128(stage + (uint32_t)((g + 8) * WS + bo));
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
                    const int m = g + 8 * nb;
                    uint4 xv = make_uint4(0u, 0u, 0u, 0u);
                    if (m < M && bo < KB) xv = lds128(x_s + (uint32_t)(m * XS + 4 * (bo + 4 * i)));
                    const uint4 xt = transpose_bytes4x4(xv);
                    mma_16x8x32_u8s8(d4[i][nb], ua[0], ub[0], ua[1], ub[1], xt.x, xt.y);
                    mma_16x8x32_u8s8(d4[i][nb], ua[2], ub[2], ua[3], ub[3], xt.z, xt.w);
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
        if (warp == 0 && issued < nmine) issue(issued);
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
                        const int a = tot - rsv[nb][c & 1];
                        const float gn = (c & 2) ? gb : ga;
                        y[(int64_t)m * N + n] = __fmul_rn(__int2float_rn(a), __fmul_rn(gn, sxv[nb][c & 1]));
                        if (acc_out) acc_out[(int64_t)m * N + n] = a;
                    }
                }
        }
        ga = na;
        gb = nbg;
        buf ^= 1;
    }
    // Copies this CTA issued must have landed before it exits (already true
    // unless a wait above gave up).
    if (threadIdx.x == 0) {
        for (int k = consumed; k < issued; ++k)
            mbar_wait(smem_u32(&bars[k % nstage]), (uint32_t)((k / nstage) & 1));
        mbar_wait(smem_u32(&xbar), 0);
    }
    // Inputs-ready mode skipped the wait above: finish no earlier than the
    // previous kernel, so later work still sees the stream's results in order.
    if (mode & kModeInputsReady) pdl_wait();
}

}  // namespace tq
