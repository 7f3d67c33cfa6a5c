// tq_gemv.cuh -- small-M (decode) ternary GEMV: y = (x_q . q) * gamma * s_x.
//
// Hetman-2b, src/quantization.py, section 7 (simulate_hardware_bitnet_gemv:
// per output row, decode the packed bytes branch-free and accumulate in
// int32, then one fp32 rescale); Foundry, docs/quantization.md, "Native Matmul
// Kernel".  Here the add/subtract loop becomes an integer MMA.
//
// The GEMV is bound by HBM reads of the packed weights (N*K/4 bytes).  A
// 4096 x 4096 layer is 4 MiB, about 0.65 us of HBM time -- less than the
// latency of one launch.  Two kernels share the per-strip arithmetic:
//
//   tq_gemv_kernel (a layer that waits for its predecessor): one CTA per 16-row
//     strip over the whole GPU, so the time from "inputs ready" to "y stored"
//     -- the critical path of a chain of dependent layers -- is as short as
//     possible.
//   tq_gemv_stream_kernel (independent calls, TQ_FLAG_INPUTS_READY): a narrow
//     grid of 32-odd CTAs that stream runs of strips.  Under programmatic
//     dependent launch the next kernel starts only once every CTA of this one
//     is resident; a narrow grid is resident at once, so several layers'
//     kernels run side by side on different SMs and the launch rate, not the
//     latency of one launch, sets the pace.
//
// Per strip, as both kernels do it:
//   * Thread (g = lane/4, t = lane%4) of warp w owns the 16-byte pieces at byte
//     64*step + 16*t of rows g and g + 8 for the column steps step = w + j*W,
//     j < SPW, and loads them straight into registers (no shared-memory
//     staging, no barrier in front of the weight stream).
//   * x_q (M <= 16 rows) is copied into shared memory with cp.async (no
//     registers held); gamma, s_x and rowsum are requested early.
//   * A 32-bit word holds 16 codes; (word >> 2j) & 0x03030303 spreads codes
//     {j, 4+j, 8+j, 12+j} into bytes as unsigned values c = q + 1 in
//     {0, 1, 2}.  The matching 16 activations are the 16-byte chunk of x_q
//     transposed 4 x 4 the same way, so the pairing of codes and activations
//     is exact.  The streaming kernel, whose CTAs use x_q for many strips,
//     transposes every chunk once, in place, right after it lands.  Chunk c
//     of a row sits at position c ^ (((c >> 3) & 1) << 1) and rows are 16
//     bytes past a multiple of 128 apart, which makes a quarter-warp's chunk
//     reads (8 threads, 2 rows x 4 column offsets) free of bank conflicts.
//   * mma.sync m16n8k32 (u8 x s8 -> s32) reduces 32 codes per row and token;
//     sum_k x*c - sum_k x = sum_k x*q removes the offset (rowsum).
//   * The warps' partial sums meet in shared memory; each thread finishes one
//     or two (row, token) outputs.
#pragma once

#include "tq_common.cuh"

namespace tq {

constexpr int kGemvMaxK = 8192;

// Shared-memory row stride of x_q (16 bytes past a multiple of 128) and the
// swizzled position of 16-byte chunk c inside a row.
__host__ __device__ inline int gemv_x_stride(int K) { return K + ((16 - K % 128) + 128) % 128; }
__device__ __forceinline__ uint32_t x_chunk(int c) { return (uint32_t)gemv_chunk_pos(c) << 4; }
__host__ __device__ inline int gemv_x_bytes(int M, int K) { return M * gemv_x_stride(K); }

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "r"(addr)
                 : "memory");
    return r;
}

// 16-byte streaming load of packed weights (read-only for the kernel's
// lifetime, not kept in L1); volatile, so it is issued where it is written.
__device__ __forceinline__ uint4 ldg_stream16(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p)
                 : "memory");
    return r;
}

// 16-byte asynchronous global -> shared copy (cached in L2 only), and the
// wait for all of this thread's copies.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// Registers per thread bound the CTAs per SM: lean shapes aim at 8 CTAs of
// 4 warps, the others at 4 CTAs of 8 warps (half of that with 16 tokens).
__host__ __device__ constexpr int gemv_min_blocks(int NB, int W) {
    return (W <= 4 ? 8 : W <= 8 ? 4 : 2) / NB;
}

// Weights of one strip held by one thread: rows g and g + 8, column steps
// w + j * W (w = warp in its group, W = warps per strip).
template <int SPW>
struct StripRegs {
    uint4 a[SPW], b[SPW];
};

template <int SPW, int W>
__device__ __forceinline__ void load_strip(StripRegs<SPW> &r, const uint8_t *__restrict__ packed,
                                           int64_t n0, int64_t N, int KB, int w, int lane) {
    const int g = lane >> 2, t = lane & 3;
    const int64_t ra = n0 + g, rb = n0 + g + 8;
#pragma unroll
    for (int j = 0; j < SPW; ++j) {
        const int bo = (w + j * W) * 64 + t * 16;
        r.a[j] = make_uint4(0u, 0u, 0u, 0u);
        r.b[j] = r.a[j];
        if (bo < KB) {
            if (ra < N) r.a[j] = ldg_stream16(packed + ra * KB + bo);
            if (rb < N) r.b[j] = ldg_stream16(packed + rb * KB + bo);
        }
    }
}

// Partial sums of one warp over its column steps: d[chain][nb][fragment].
// XT: the x_q chunks in shared memory are already transposed (else each
// chunk is transposed here, after it is read).
template <int NB, int W, int SPW, int CH, bool XT, bool CONV>
__device__ __forceinline__ void strip_mma(const StripRegs<SPW> &r, int (&d)[CH][NB][4], int w, int lane,
                                          uint32_t x_s, int XS, int M, int KB, int enc) {
    const int g = lane >> 2, t = lane & 3;
    const int nsteps = (KB + 63) >> 6;
    const uint32_t xsw = (uint32_t)(t & 2) << 4;  // chunk swizzle of this thread's columns
#pragma unroll
    for (int i = 0; i < CH; ++i)
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) d[i][nb][0] = d[i][nb][1] = d[i][nb][2] = d[i][nb][3] = 0;
#pragma unroll
    for (int j = 0; j < SPW; ++j) {
        const int step = w + j * W;
        if (step < nsteps) {  // warp-uniform
            const int bo = step * 64 + t * 16;
            const uint32_t a4[4] = {r.a[j].x, r.a[j].y, r.a[j].z, r.a[j].w};
            const uint32_t b4[4] = {r.b[j].x, r.b[j].y, r.b[j].z, r.b[j].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                // codes in Foundry's layout (field = q + 1); other layouts (CONV) converted here
                const uint32_t ar = CONV ? codes_to_foundry(a4[i], enc) : a4[i];
                const uint32_t br = CONV ? codes_to_foundry(b4[i], enc) : b4[i];
                uint32_t ua[4], ub[4];
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    ua[jj] = (ar >> (2 * jj)) & 0x03030303u;
                    ub[jj] = (br >> (2 * jj)) & 0x03030303u;
                }
#pragma unroll
                for (int nb = 0; nb < NB; ++nb) {
                    const int m = g + 8 * nb;
                    // chunk c = bo / 4 + i, at x_chunk(c) = 16 * (bo / 4 + (i ^ (t & 2)))
                    uint4 xt = make_uint4(0u, 0u, 0u, 0u);
                    if (m < M && bo < KB)
                        xt = lds128(x_s + (uint32_t)(m * XS + 4 * bo) + ((uint32_t)(i << 4) ^ xsw));
                    if (!XT) xt = transpose_bytes4x4(xt);
                    mma_16x8x32_u8s8(d[i % CH][nb], ua[0], ub[0], ua[1], ub[1], xt.x, xt.y);
                    mma_16x8x32_u8s8(d[i % CH][nb], ua[2], ub[2], ua[3], ub[3], xt.z, xt.w);
                }
            }
        }
    }
}

// Finishing role: output e (< 128 * NB) of a strip is fragment value
// c = (e/32)%4 of lane l = e%32 in token block nb = e/128: row g(l) (+8 if
// c >= 2) of the strip, token 8 nb + 2 t(l) + (c & 1).
__device__ __forceinline__ int fin_row(int e) { return ((e & 31) >> 2) + (((e >> 5) & 2) ? 8 : 0); }
__device__ __forceinline__ int fin_tok(int e) { return 8 * (e >> 7) + 2 * (e & 3) + ((e >> 5) & 1); }

// x_q rows into shared memory (swizzled chunks), 16 bytes per copy, by
// `nthr` threads; then, once landed, each thread transposes the chunks it
// copied (its own cp.async writes are complete after the wait).
__device__ __forceinline__ void copy_x(uint32_t x_s, const int8_t *__restrict__ xq, int M, int K, int XS,
                                       int tid, int nthr) {
    const int cpr = K >> 4;
    for (int i = tid; i < M * cpr; i += nthr) {
        const int m = i / cpr, c = i - m * cpr;
        cp_async16(x_s + (uint32_t)(m * XS) + x_chunk(c), xq + (int64_t)m * K + 16 * c);
    }
}
__device__ __forceinline__ void transpose_x(uint32_t x_s, int M, int K, int XS, int tid, int nthr) {
    const int cpr = K >> 4;
    for (int i = tid; i < M * cpr; i += nthr) {
        const int m = i / cpr, c = i - m * cpr;
        const uint32_t a = x_s + (uint32_t)(m * XS) + x_chunk(c);
        const uint4 v = transpose_bytes4x4(lds128(a));
        asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                     : "memory");
    }
}

// NB: token blocks of 8 (M <= 8 * NB).  W: warps per CTA.  SPW: 64-byte
// column steps per warp (K <= 256 * W * SPW).  CONV: weights in one of
// Hetman-2b's layouts (mode bits 2-3), rewritten in Foundry's as they are used.
// EPI: the extra epilogue `ep` (bias, integer bias and shift) is applied.
//
// mode & kModeWeightsStatic: the packed weights and gamma are not written by
// work still in flight on the stream, so they are requested before the
// programmatic-dependent-launch wait and overlap the previous kernel.
// mode & kModeInputsReady: no input is written, and no output touched, by
// work still in flight; the kernel then does not wait before reading at all.
// One CTA (the last) waits for the previous kernel before it exits, so this
// kernel still completes after its predecessor and later work sees the
// stream's results in order; the other CTAs leave as soon as they are done.
template <int NB, int W, int SPW, bool CONV, bool EPI>
__global__ void __launch_bounds__(W * 32, gemv_min_blocks(NB, W))
    tq_gemv_kernel(const int8_t *__restrict__ xq, const float *__restrict__ s_x,
                const int32_t *__restrict__ rowsum, const uint8_t *__restrict__ packed,
                const float *__restrict__ gamma, int per_row, int M, int64_t N, int K,
                float *__restrict__ y, int32_t *__restrict__ acc_out, int mode, Epilogue ep) {
    constexpr int CH = 8 / SPW;                              // independent MMA chains
    constexpr int FPT = (128 * NB + W * 32 - 1) / (W * 32);  // outputs finished per thread
    extern __shared__ __align__(128) uint8_t dsm[];
    __shared__ int red[W][4 * NB][32];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KB = K >> 2;  // packed bytes per row
    const int XS = gemv_x_stride(K);
    const uint32_t x_s = smem_u32(dsm);
    const int64_t r0 = (int64_t)blockIdx.x * 16;

    pdl_trigger();
    const bool ready = (mode & kModeInputsReady) != 0;
    const bool early_w = (mode & (kModeWeightsStatic | kModeInputsReady)) != 0;

    float gv[FPT], sxv[FPT], bv[FPT];
    int rsv[FPT], abv[FPT];
    auto load_gamma = [&]() {  // and, with EPI, the row's biases
#pragma unroll
        for (int q = 0; q < FPT; ++q) {
            const int e = threadIdx.x + q * W * 32;
            const int64_t n = r0 + fin_row(e);
            const bool ok = e < 128 * NB && n < N;
            gv[q] = ok ? __ldg(gamma + (per_row ? n : 0)) : 0.0f;
            if (EPI) {
                bv[q] = (ok && ep.bias) ? __ldg(ep.bias + n) : 0.0f;
                abv[q] = (ok && ep.acc_bias) ? __ldg(ep.acc_bias + n) : 0;
            }
        }
    };
    auto load_tok = [&]() {
#pragma unroll
        for (int q = 0; q < FPT; ++q) {
            const int e = threadIdx.x + q * W * 32;
            const int m = fin_tok(e);
            sxv[q] = (e < 128 * NB && m < M) ? __ldcg(s_x + m) : 0.0f;
            rsv[q] = (e < 128 * NB && m < M) ? __ldcg(rowsum + m) : 0;
        }
    };
    StripRegs<SPW> wr;
    if (early_w) load_gamma();
    if (ready) {
        load_tok();
        copy_x(x_s, xq, M, K, XS, threadIdx.x, W * 32);
    }
    if (early_w) load_strip<SPW, W>(wr, packed, r0, N, KB, warp, lane);
    if (!ready) pdl_wait();
    if (!ready) {
        load_tok();
        copy_x(x_s, xq, M, K, XS, threadIdx.x, W * 32);
    }
    if (!early_w) {
        load_gamma();
        load_strip<SPW, W>(wr, packed, r0, N, KB, warp, lane);
    }
    cp_async_wait_all();
    __syncthreads();  // x_q is in shared memory (each chunk is used once here:
                      // transposed where it is read, off the wait's critical path)

    int d[CH][NB][4];
    strip_mma<NB, W, SPW, CH, false, CONV>(wr, d, warp, lane, x_s, XS, M, KB, (mode >> kModeEncShift) & 3);
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            int sum = 0;
#pragma unroll
            for (int i = 0; i < CH; ++i) sum += d[i][nb][c];
            red[warp][nb * 4 + c][lane] = sum;
        }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < FPT; ++q) {
        const int e = threadIdx.x + q * W * 32;
        if (e < 128 * NB) {
            const int64_t n = r0 + fin_row(e);
            const int m = fin_tok(e);
            int tot = 0;
#pragma unroll
            for (int ww = 0; ww < W; ++ww) tot += red[ww][(e >> 7) * 4 + ((e >> 5) & 3)][e & 31];
            if (m < M && n < N) {
                const int a = tot - rsv[q];
                const float v = __fmul_rn(__int2float_rn(a), __fmul_rn(gv[q], sxv[q]));
                y[(int64_t)m * N + n] = EPI ? __fadd_rn(v, bv[q]) : v;
                if (acc_out) acc_out[(int64_t)m * N + n] = EPI ? (a + abv[q]) >> ep.shift : a;
            }
        }
    }
    if (ready && blockIdx.x == gridDim.x - 1) pdl_wait();
}

// ---------------------------------------------------------------------------
// Streaming GEMV for independent calls (inputs ready), M <= 8, K <= 4096.
// A CTA of kStreamGroups groups of four warps owns `per_cta` consecutive
// strips; group q takes strips q, q + G, q + 2G, ... of the run and requests
// the next one as soon as it has computed the current one (one register set:
// two CTAs fit on an SM, and the other groups, CTAs and layers keep the
// memory system busy meanwhile -- a second register set per group measured
// slower).  x_q is copied once per CTA.  Groups synchronise on their own
// named barrier; the partial sums are double-buffered by strip.
// ---------------------------------------------------------------------------
constexpr int kStreamGroups = 4;
constexpr int kStreamThreads = kStreamGroups * 128;
constexpr int kStreamMaxK = 4096;

__device__ __forceinline__ void group_sync(int group) {
    asm volatile("bar.sync %0, 128;" ::"r"(1 + group) : "memory");
}

// ENC: packed-code layout (kEnc*), a template argument here: registers are at
// the two-CTAs-per-SM limit.
template <int ENC>
__global__ void __launch_bounds__(kStreamThreads, 2)
    tq_gemv_stream_kernel(const int8_t *__restrict__ xq, const float *__restrict__ s_x,
                       const int32_t *__restrict__ rowsum, const uint8_t *__restrict__ packed,
                       const float *__restrict__ gamma, int per_row, int M, int64_t N, int K,
                       float *__restrict__ y, int32_t *__restrict__ acc_out, int per_cta) {
    constexpr int SPW = 4, CH = 2, GW = 4;  // 4 warps per strip, 4 steps each
    extern __shared__ __align__(128) uint8_t dsm[];
    __shared__ int red[kStreamGroups][2][GW][4][32];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int group = warp / GW, gw = warp % GW, gt = threadIdx.x & 127;
    const int KB = K >> 2;
    const int XS = gemv_x_stride(K);
    const uint32_t x_s = smem_u32(dsm);
    const int64_t nstrips = (N + 15) >> 4;
    const int64_t s0 = (int64_t)blockIdx.x * per_cta;
    const int nmine = (int)((s0 + per_cta) < nstrips ? per_cta : nstrips - s0);

    pdl_trigger();
    // finishing role inside the group: output gt of each strip
    const int f_m = fin_tok(gt), f_r = fin_row(gt);
    const float f_sx = f_m < M ? __ldcg(s_x + f_m) : 0.0f;
    const int f_rs = f_m < M ? __ldcg(rowsum + f_m) : 0;
    auto gamma_of = [&](int k) {
        const int64_t n = (s0 + k) * 16 + f_r;
        return (k < nmine && n < N) ? __ldg(gamma + (per_row ? n : 0)) : 0.0f;
    };
    copy_x(x_s, xq, M, K, XS, threadIdx.x, kStreamThreads);
    StripRegs<SPW> w0;
    int k = group;
    if (k < nmine) load_strip<SPW, GW>(w0, packed, (s0 + k) * 16, N, KB, gw, lane);
    float g0 = gamma_of(k);
    cp_async_wait_all();
    transpose_x(x_s, M, K, XS, threadIdx.x, kStreamThreads);
    __syncthreads();  // x_q is in shared memory, transposed

    int par = 0;
    auto one = [&](const StripRegs<SPW> &w, int kk, float gn) {
        int d[CH][1][4];
        strip_mma<1, GW, SPW, CH, true, ENC != kEncFoundry>(w, d, gw, lane, x_s, XS, M, KB, ENC);
#pragma unroll
        for (int c = 0; c < 4; ++c) red[group][par][gw][c][lane] = d[0][0][c] + d[1][0][c];
        group_sync(group);
        const int64_t n = (s0 + kk) * 16 + f_r;
        int tot = 0;
#pragma unroll
        for (int ww = 0; ww < GW; ++ww) tot += red[group][par][ww][(gt >> 5) & 3][gt & 31];
        if (f_m < M && n < N) {
            const int a = tot - f_rs;
            y[(int64_t)f_m * N + n] = __fmul_rn(__int2float_rn(a), __fmul_rn(gn, f_sx));
            if (acc_out) acc_out[(int64_t)f_m * N + n] = a;
        }
        par ^= 1;
    };
    for (; k < nmine; k += kStreamGroups) {
        one(w0, k, g0);
        if (k + kStreamGroups < nmine) {
            load_strip<SPW, GW>(w0, packed, (s0 + k + kStreamGroups) * 16, N, KB, gw, lane);
            g0 = gamma_of(k + kStreamGroups);
        }
    }
    // One CTA waits for the previous kernel before exiting (stream order).
    if (blockIdx.x == gridDim.x - 1) pdl_wait();
}

}  // namespace tq
