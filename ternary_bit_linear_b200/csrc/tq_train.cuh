// tq_train.cuh -- training kernels of the ternary layer: the gradient with
// respect to the layer input, the straight-through estimator of the latent
// weights, and the stochastic ternary flip.
//
//   Foundry, docs/quantization.md, "Ternary Training (Backward Pass +
//   Stochastic Flip)": fq_matmul_ternary_backward_input (dX += dY W_ternary,
//   same unpacking as the forward, summed over the output features) and
//   fq_ternary_stochastic_flip (p = clamp(|grad| T, 0, 1), one step toward
//   -grad, caller-owned xorshift64 state).
//   Hetman-2b, src/quantization.py, section 2 AbsmeanWeightQuantizer.backward
//   (grad / gamma, damped by 0.1 outside |w / gamma| <= tau).
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>

#include "tq_common.cuh"
#include "tq_gemm.cuh"
#include "tq_gemv.cuh"
#include "tq_xorshift_jump.h"

namespace tq {

// ===========================================================================
// Straight-through estimator (elementwise, HBM-bound: 12 bytes per weight)
// ===========================================================================
constexpr int kSteThreads = 256;

__device__ __forceinline__ float ste_one(float g, float w, float gm, float tau, bool san) {
    if (san) {
        if (isnan(w)) w = 0.0f;
        else if (isinf(w)) w = w > 0.0f ? 1.0f : -1.0f;
    }
    const float ws = __fdiv_rn(w, gm);
    const float damp = fabsf(ws) <= tau ? 1.0f : 0.1f;  // NaN compares false: damped
    return __fmul_rn(__fdiv_rn(g, gm), damp);
}

// grad, w, out: [N][K] fp32 viewed as float4 (K % 4 == 0, so a vector never
// crosses a row); gamma [N] (per_row) or [1].  out may be grad or w.
template <bool SAN>
__global__ void __launch_bounds__(kSteThreads)
    tq_ste_backward_kernel(const float4 *grad, const float4 *w, const float *__restrict__ gamma, int per_row,
                        int64_t nvec, int64_t kvec, float tau, float4 *out) {
    pdl_wait();
    pdl_trigger();
    const int64_t stride = (int64_t)gridDim.x * kSteThreads;
    for (int64_t i = (int64_t)blockIdx.x * kSteThreads + threadIdx.x; i < nvec; i += stride) {
        const float gm = __ldg(gamma + (per_row ? i / kvec : 0));
        const float4 g = __ldcs(grad + i), x = __ldcs(w + i);
        float4 r;
        r.x = ste_one(g.x, x.x, gm, tau, SAN);
        r.y = ste_one(g.y, x.y, gm, tau, SAN);
        r.z = ste_one(g.z, x.z, gm, tau, SAN);
        r.w = ste_one(g.w, x.w, gm, tau, SAN);
        __stcs(out + i, r);
    }
}

// ===========================================================================
// Stochastic flip
// ===========================================================================
// The stream of draws is Foundry's sequential one: weight i (row-major over
// [N][K]) compares against the (i+1)-th xorshift64 output after the caller's
// state.  xorshift64 is linear over GF(2), so the state i steps ahead is
// A^i x0; the tables of tq_xorshift_jump.h hold the powers of A needed to
// start every lane's run of kFlipRun weights at its own point of the stream:
//   CTA    first chunk c: A^(16384 c) from the binary powers TQ_XS_CHUNK
//          (one warp, 64-column matrix-vector products split over the lanes);
//          later chunks continue from the end state of the previous one;
//   warp   w: A^(2048 w) x_chunk (TQ_XS_WARP, same cooperative product);
//   lane   l: A^(64 l) x_warp (TQ_XS_LANE, copied to shared memory, one
//          product per lane).
// Each lane then runs its 64 draws sequentially.  Gradients are staged per
// warp in shared memory with cp.async (coalesced), packed codes are read and
// written as one 16-byte vector per lane.
constexpr int kFlipWarps = TQ_XS_WARPS;
constexpr int kFlipThreads = 32 * kFlipWarps;
constexpr int kFlipRun = TQ_XS_RUN;                          // weights per lane
constexpr int kFlipWarpRun = 32 * kFlipRun;                  // weights per warp
constexpr int64_t kFlipChunk = (int64_t)kFlipWarps * kFlipWarpRun;  // weights per CTA pass
constexpr int kFlipTabBytes = 64 * 32 * 8;
constexpr int kFlipSmem = kFlipTabBytes + kFlipWarps * kFlipWarpRun * 4;
static_assert(kFlipRun == 64, "one 16-byte packed vector per lane");

__device__ const uint64_t kXsChunk[TQ_XS_CHUNK_BITS][64] = TQ_XS_CHUNK_INIT;
__device__ const uint64_t kXsWarp[TQ_XS_WARPS][64] = TQ_XS_WARP_INIT;
__device__ const uint64_t kXsLane[64][32] = TQ_XS_LANE_INIT;

// y = M x for a warp-uniform x: lane l folds columns 2l and 2l+1, then an
// XOR reduction over the warp gives every lane the product.
__device__ __forceinline__ uint64_t warp_matvec(const uint64_t *__restrict__ cols, uint64_t x, int lane) {
    const int b = 2 * lane;
    uint64_t r = 0;
    if ((x >> b) & 1ull) r ^= __ldg(cols + b);
    if ((x >> (b + 1)) & 1ull) r ^= __ldg(cols + b + 1);
#pragma unroll
    for (int off = 16; off; off >>= 1) r ^= __shfl_xor_sync(0xffffffffu, r, off);
    return r;
}

// y = A^(64 lane) x, each lane its own matrix (column-major table in shared
// memory: column b of every lane's matrix in 32 consecutive words).
__device__ __forceinline__ uint64_t lane_matvec(const uint64_t *tab, uint64_t x, int lane) {
    uint64_t r = 0;
#pragma unroll 16
    for (int b = 0; b < 64; ++b) r ^= tab[b * 32 + lane] & (0ull - ((x >> b) & 1ull));
    return r;
}

// New field of a weight, two bits per entry at index field + 4 * action, with
// the field read as q + 1 (the unassigned 0b11 as q = 0) and q clamped to
// [-1, 1]:  keep 0 1 2 1 | down 0 0 1 0 | up 1 2 2 2.
constexpr uint32_t kFlipTable = 0x00A91064u;

// Four weights (one packed byte in Foundry's layout) against the next four draws.
__device__ __forceinline__ uint32_t flip_byte(uint32_t byte, const float4 g4, float temp, uint64_t &x) {
    const float gs[4] = {g4.x, g4.y, g4.z, g4.w};
    uint32_t out = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x ^= x << 13;
        x ^= x >> 7;
        x ^= x << 17;
        const float u = __fmul_rn(__uint2float_rn((uint32_t)(x >> 40)), 0x1p-24f);  // exact
        const float a = __fmul_rn(fabsf(gs[i]), temp);
        const float p = a > 1.0f ? 1.0f : a;  // NaN stays NaN: u < p is false
        // action: 0 keep, 1 one step down (grad > 0), 2 one step up (grad < 0)
        const uint32_t act = u < p ? (gs[i] > 0.0f ? 1u : (gs[i] < 0.0f ? 2u : 0u)) : 0u;
        const uint32_t f = (byte >> (2 * i)) & 3u;
        out |= ((kFlipTable >> (2 * (f + 4 * act))) & 3u) << (2 * i);
    }
    return out;
}

// packed [nw / 4] bytes (in place), grad [nw] fp32, nw % 64 == 0.  CTA b
// owns chunks [b * per_cta, (b + 1) * per_cta).
template <bool CONV>
__global__ void __launch_bounds__(kFlipThreads, 2)
    tq_flip_kernel(uint8_t *packed, const float *__restrict__ grad, int64_t nw, float temp, uint64_t x0,
                int64_t per_cta, int mode) {
    extern __shared__ __align__(16) uint8_t flip_smem[];
    __shared__ uint64_t chunk_state;
    uint64_t *tab = reinterpret_cast<uint64_t *>(flip_smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float4 *stage = reinterpret_cast<float4 *>(flip_smem + kFlipTabBytes) + warp * (kFlipWarpRun / 4);
    const int enc = (mode >> kModeEncShift) & 3;
    const int64_t nchunks = (nw + kFlipChunk - 1) / kFlipChunk;
    const int64_t c_begin = (int64_t)blockIdx.x * per_cta;
    const int64_t c_end = c_begin + per_cta < nchunks ? c_begin + per_cta : nchunks;

    // constant tables only: no dependence on earlier kernels yet
    for (int i = threadIdx.x; i < 64 * 32; i += kFlipThreads) tab[i] = (&kXsLane[0][0])[i];
    if (warp == 0) {
        uint64_t x = x0;
        for (int j = 0; j < TQ_XS_CHUNK_BITS; ++j)
            if ((c_begin >> j) & 1) x = warp_matvec(kXsChunk[j], x, lane);
        if (lane == 0) chunk_state = x;
    }
    pdl_wait();  // grad and packed may be written by the previous kernel
    pdl_trigger();
    __syncthreads();

    for (int64_t c = c_begin; c < c_end; ++c) {
        const int64_t wbase = c * kFlipChunk + (int64_t)warp * kFlipWarpRun;  // this warp's first weight
        const int64_t left = nw - wbase;
        const int nruns = left <= 0 ? 0 : (left >= kFlipWarpRun ? 32 : (int)(left / kFlipRun));
        // stage the warp's gradients: float4 g of the warp = run g / 16, vector
        // g % 16, stored at run * 16 + (vector ^ (run & 7)) (conflict-free reads)
        for (int i = 0; i < 16; ++i) {
            const int g = i * 32 + lane, r = g >> 4, j = g & 15;
            if (r < nruns)
                cp_async16(smem_u32(stage + r * 16 + (j ^ (r & 7))), grad + wbase + 4 * (int64_t)g);
        }
        uint64_t x = warp_matvec(kXsWarp[warp], chunk_state, lane);
        x = lane_matvec(tab, x, lane);
        cp_async_wait_all();
        __syncwarp();
        if (lane < nruns) {
            uint8_t *pk = packed + (wbase + (int64_t)lane * kFlipRun) / 4;
            const uint4 v = *reinterpret_cast<const uint4 *>(pk);
            uint32_t words[4] = {v.x, v.y, v.z, v.w};
            if (CONV) {
#pragma unroll
                for (int i = 0; i < 4; ++i) words[i] = codes_to_foundry(words[i], enc);
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float4 g4 = stage[lane * 16 + (j ^ (lane & 7))];
                const int sh = (j & 3) * 8;
                const uint32_t b = flip_byte((words[j >> 2] >> sh) & 0xFFu, g4, temp, x);
                words[j >> 2] = (words[j >> 2] & ~(0xFFu << sh)) | (b << sh);
            }
            if (CONV) {
#pragma unroll
                for (int i = 0; i < 4; ++i) words[i] = codes_from_foundry(words[i], enc);
            }
            *reinterpret_cast<uint4 *>(pk) = make_uint4(words[0], words[1], words[2], words[3]);
        }
        // A chunk followed by another one is full: its last lane ends where
        // the next chunk starts.
        __syncthreads();
        if (threadIdx.x == kFlipThreads - 1) chunk_state = x;
        __syncthreads();
    }
}

// ===========================================================================
// Gradient with respect to the input: dX = row_scale * (dY * gamma) W_ternary
// ===========================================================================
// The contraction runs over the N output features with fp32 operands on one
// side and codes in {-1, 0, +1} on the other.  It is a dense GEMM, so it runs
// on the tensor cores (tcgen05 kind::f16, fp16 operands, fp32 accumulation in
// tensor memory).  The fp32 side is scaled per token by a power of two that
// puts the row's largest |g| in [2^14, 2^15), then split into two fp16 parts:
//   g = fp32(dY * gamma_n),  v = g * 2^e_t (exact),
//   hi = fp16(v),  lo = fp16(v - hi)           (v - hi is exact in fp32)
// hi + lo keeps 22 of fp32's 24 significant bits (|v - hi - lo| <= 2^-22 |v|,
// or 2^-25 absolute where lo is subnormal, i.e. 2^-39 of the row's largest
// term).  Products with a code are exact, the tensor core accumulates in
// fp32, and the epilogue multiplies by 2^-e_t (exact) and row_scale.

// --- split pass: planes [2][M][Np] fp16 (columns N .. Np - 1 zero), then
// inv_scale [M] fp32 = 2^-e_t.  One CTA per token row. --------------------
constexpr int kSplitThreads = 256;

// 8 columns of row `row` starting at c0 (zero beyond N), times the column scale.
template <bool VEC>
__device__ __forceinline__ void load_g8(const float *row, const float *gamma, int per_row, float g0, int N, int c0,
                                        float (&v)[8]) {
    if (VEC && c0 + 8 <= N) {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(row + c0));
        const float4 b = __ldg(reinterpret_cast<const float4 *>(row + c0 + 4));
        v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = c0 + j < N ? __ldg(row + c0 + j) : 0.0f;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float sc = per_row ? (c0 + j < N ? __ldg(gamma + c0 + j) : 0.0f) : g0;
        v[j] = c0 + j < N ? __fmul_rn(v[j], sc) : 0.0f;
    }
}

// VEC: rows are 16-byte aligned (N % 4 == 0).
template <bool VEC>
__global__ void __launch_bounds__(kSplitThreads)
    tq_bwd_split_kernel(const float *__restrict__ dY, const float *__restrict__ gamma, int per_row, int M, int N,
                     int Np, __half *__restrict__ planes, float *__restrict__ inv_scale) {
    __shared__ float red[kSplitThreads / 32];
    pdl_wait();
    pdl_trigger();
    const int64_t plane = (int64_t)M * Np;
    const float g0 = __ldg(gamma);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int t = blockIdx.x; t < M; t += gridDim.x) {
        const float *row = dY + (int64_t)t * N;
        float mx = 0.0f;
        for (int c0 = threadIdx.x * 8; c0 < N; c0 += kSplitThreads * 8) {
            float v[8];
            load_g8<VEC>(row, gamma, per_row, g0, N, c0, v);
#pragma unroll
            for (int j = 0; j < 8; ++j) mx = fmaxf(mx, fabsf(v[j]));
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        if (lane == 0) red[warp] = mx;
        __syncthreads();
        mx = red[0];
#pragma unroll
        for (int w = 1; w < kSplitThreads / 32; ++w) mx = fmaxf(mx, red[w]);
        __syncthreads();  // red is reused by the next row
        // scale 2^e with mx * 2^e in [2^14, 2^15); 1 for a zero or non-finite row
        float sc = 1.0f, inv = 1.0f;
        if (mx > 0.0f && mx <= 3.4028235e38f) {
            int E;
            frexpf(mx, &E);  // mx = m 2^E, m in [0.5, 1)
            sc = ldexpf(1.0f, 15 - E);
            inv = ldexpf(1.0f, E - 15);
        }
        if (threadIdx.x == 0) inv_scale[t] = inv;
        __half *o = planes + (int64_t)t * Np;
        for (int c0 = threadIdx.x * 8; c0 < Np; c0 += kSplitThreads * 8) {
            float v[8];
            load_g8<VEC>(row, gamma, per_row, g0, N, c0, v);
            __align__(16) __half hi[8], lo[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float x = __fmul_rn(v[j], sc);
                hi[j] = __float2half_rn(x);
                lo[j] = __float2half_rn(__fsub_rn(x, __half2float(hi[j])));
            }
            *reinterpret_cast<uint4 *>(o + c0) = *reinterpret_cast<const uint4 *>(hi);
            *reinterpret_cast<uint4 *>(o + plane + c0) = *reinterpret_cast<const uint4 *>(lo);
        }
    }
}

// --- the GEMM ---------------------------------------------------------------
// Persistent, one CTA per SM.  Output tile: 256 input features (two MMAs of
// M = 128, taken by the unpacked codes, A = W^T) x 256 tokens (the MMA's N,
// taken by the fp16 planes, B = g).  The contraction dimension is the layer's
// N, in steps of 32.  Per step: the two plane tiles [256 tokens][32 n]
// (64-byte rows, 64-byte swizzle, K-major, by TMA), the packed tile
// [32 n][64 B] (by TMA), and the code tiles A [32 n][2 x 128 features] in
// fp16, written by the unpackers in the 128-byte-swizzled MN-major layout
// (features contiguous: the packed rows already are).  Eight MMAs of K = 16
// per step (two halves of the step x two feature halves x two planes) into
// two fp32 accumulators of 256 columns (all of tensor memory, so the next
// tile's MMAs wait for the epilogue).  Both feature halves share each plane
// tile, which halves the plane bytes each MMA needs from L2 against a
// 128-feature tile.  Feature tiles run fastest, so concurrently running CTAs
// share the token block's planes in L2.  Warp roles as in the forward GEMM:
// 0 plane producer, 1 MMA issuer and TMEM owner, 2 packed-weight producer,
// 4-11 unpackers (two groups taking alternate steps), 12-19 epilogue.
constexpr int kBwdTileF = 256;   // features per tile (two MMAs of M = 128)
constexpr int kBwdTileT = 256;   // tokens per tile (MMA N)
constexpr int kBwdStepN = 32;    // contraction rows per step
constexpr int kBwdPlanes = 2;
constexpr int kBwdPlaneBytes = kBwdTileT * kBwdStepN * 2;             // 16 KB
constexpr int kBwdAHalf = 128 * kBwdStepN * 2;                        // 8 KB per feature half
constexpr int kBwdABytes = 2 * kBwdAHalf;
constexpr int kBwdStage = kBwdPlanes * kBwdPlaneBytes + kBwdABytes;   // 48 KB
constexpr int kBwdStages = 4;
constexpr int kBwdWBytes = kBwdStepN * kBwdTileF / 4;                 // 2 KB packed per step
constexpr int kBwdWStages = 8;
constexpr int kBwdOffW = kBwdStages * kBwdStage;
constexpr int kBwdOffBar = kBwdOffW + kBwdWStages * kBwdWBytes;
constexpr int kBwdBars = 2 * kBwdStages + 2 * kBwdWStages + 3;
constexpr int kBwdOffTmem = kBwdOffBar + kBwdBars * 8;
constexpr int kBwdDynamic = kBwdOffTmem + 16 + 1024;
constexpr uint32_t kBwdTmemCols = 2 * kBwdTileT;  // two feature halves x 256 fp32 columns
static_assert(kBwdDynamic <= 232448, "shared memory per CTA");
static_assert(kBwdPlaneBytes % 1024 == 0 && kBwdAHalf % 1024 == 0 && kBwdStage % 1024 == 0, "atoms aligned");

// Instruction descriptor, kind::f16: D f32, A and B f16, A MN-major, B K-major.
__host__ __device__ constexpr uint32_t idesc_f16_amn(int M, int N) {
    return (1u << 4)                        // D format: f32
           | (0u << 7)                      // A: f16
           | (0u << 10)                     // B: f16
           | (1u << 15)                     // A MN-major
           | ((uint32_t)(N >> 3) << 17)     // N / 8
           | ((uint32_t)(M >> 4) << 24);    // M / 16
}

// MN-major 16-bit operand, 128-byte swizzle: atoms of 8 contraction rows x 64
// elements (128 B per row, 16-byte chunk index XOR row % 8); atoms along M
// are `lbo` bytes apart, atoms along the contraction (8-row groups) `sbo`.
__device__ __forceinline__ uint64_t smem_desc_mn_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;  // 128-byte swizzle
    return d;
}

// K-major operand, 64-byte swizzle: rows of 64 B, 8-row groups 512 B apart.
__device__ __forceinline__ uint64_t smem_desc_k_sw64(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;             // leading byte offset (unused)
    d |= (uint64_t)(512u >> 4) << 32;    // stride byte offset: 8 rows x 64 B
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)4u << 61;             // 64-byte swizzle
    return d;
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Four codes (one packed byte, Foundry's layout) -> four fp16 of q = field - 1
// (0b00 -> -1.0 = 0xBC00, 0b01 -> 0, 0b10 -> +1.0 = 0x3C00; the unassigned
// 0b11 gives 2.0 = 0x4000).  A byte permute picks the high byte of each fp16
// from the four-entry table BC 00 3C 40 and a zero low byte.
__device__ __forceinline__ uint2 codes4_to_f16(uint32_t byte) {
    const uint32_t n0 = byte & 0xFu, n1 = (byte >> 4) & 0xFu;
    const uint32_t s0 = 0x0404u + (n0 & 3u) * 0x11u + (n0 >> 2) * 0x1100u;
    const uint32_t s1 = 0x0404u + (n1 & 3u) * 0x11u + (n1 >> 2) * 0x1100u;
    return make_uint2(__byte_perm(0x403C00BCu, 0u, s0), __byte_perm(0x403C00BCu, 0u, s1));
}

// planes: tensor map over [2 M][Np] fp16 (plane p of token t is row p M + t);
// packed: tensor map over [N][K / 4] bytes; inv_scale [M] = 2^-e_t.  dX [M][K] fp32.
template <bool CONV>
__global__ void __launch_bounds__(kGemmThreads, 1)
    tq_bwd_gemm_kernel(const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_w,
                    const float *__restrict__ inv_scale, const float *__restrict__ row_scale, int accumulate, int M,
                    int N, int K, float *__restrict__ dX, int mode) {
    constexpr int S = kBwdStages, SW = kBwdWStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + kBwdOffBar;
    auto full = [&](int s) { return bar0 + 8u * s; };
    auto empty = [&](int s) { return bar0 + 8u * (S + s); };
    auto w_full = [&](int s) { return bar0 + 8u * (2 * S + s); };
    auto w_empty = [&](int s) { return bar0 + 8u * (2 * S + SW + s); };
    const uint32_t d_full = bar0 + 8u * (2 * S + 2 * SW);
    const uint32_t d_empty = bar0 + 8u * (2 * S + 2 * SW + 1);
    const uint32_t mma_done = bar0 + 8u * (2 * S + 2 * SW + 2);
    auto g_stage = [&](int s) { return sbase + (uint32_t)(s * kBwdStage); };
    auto a_stage = [&](int s) { return g_stage(s) + (uint32_t)(kBwdPlanes * kBwdPlaneBytes); };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kBwdOffTmem);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_f = (K + kBwdTileF - 1) / kBwdTileF, num_t = (M + kBwdTileT - 1) / kBwdTileT;
    const int ntiles = num_f * num_t;
    const int nkb = (N + kBwdStepN - 1) / kBwdStepN;
    const int my_tiles =
        ntiles > (int)blockIdx.x ? (ntiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
    const int total = my_tiles * nkb;

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full(s), 1 + kUnpackWarps / 2);
            mbar_init(empty(s), 1);
        }
        for (int s = 0; s < SW; ++s) {
            mbar_init(w_full(s), 1);
            mbar_init(w_empty(s), kUnpackWarps / 2);
        }
        mbar_init(d_full, 1);
        mbar_init(d_empty, kEpiWarps);
        mbar_init(mma_done, 1);
        fence_barrier_init();
        prefetch_tmap(&tm_g);
        prefetch_tmap(&tm_w);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), kBwdTmemCols);
        tmem_relinquish();
    }
    pdl_wait();  // the planes come from the split pass just before
    pdl_trigger();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------- plane producer ----------------
        if (lane == 0) {
            int g = 0;
            for (; g < total; ++g) {
                const int s = g % S, r = g / S;
                const int t = (int)blockIdx.x + (g / nkb) * (int)gridDim.x;
                const int kb = g % nkb;
                const int t0 = (t / num_f) * kBwdTileT;
                if (!mbar_wait_sleep(empty(s), (r & 1) ^ 1)) break;
                mbar_arrive_expect_tx(full(s), kBwdPlanes * kBwdPlaneBytes);
#pragma unroll
                for (int p = 0; p < kBwdPlanes; ++p)
                    tma_load_2d(g_stage(s) + (uint32_t)(p * kBwdPlaneBytes), &tm_g, kb * kBwdStepN, p * M + t0,
                                full(s));
            }
            for (int j = g - S < 0 ? 0 : g - S; j < g; ++j) mbar_wait(full(j % S), (j / S) & 1);
        }
        __syncwarp();
    } else if (warp == 2) {
        // ---------------- packed-weight producer ----------------
        if (lane == 0) {
            int g = 0;
            for (; g < total; ++g) {
                const int s = g % SW, r = g / SW;
                const int t = (int)blockIdx.x + (g / nkb) * (int)gridDim.x;
                const int kb = g % nkb;
                if (!mbar_wait_sleep(w_empty(s), (r & 1) ^ 1)) break;
                mbar_arrive_expect_tx(w_full(s), kBwdWBytes);
                tma_load_2d(sbase + (uint32_t)(kBwdOffW + s * kBwdWBytes), &tm_w, (t % num_f) * (kBwdTileF / 4),
                            kb * kBwdStepN, w_full(s));
            }
            for (int j = g - SW < 0 ? 0 : g - SW; j < g; ++j) mbar_wait(w_full(j % SW), (j / SW) & 1);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_f16_amn(128, kBwdTileT);
            int g = 0;
            bool ok = true;
            for (int tl = 0; tl < my_tiles && ok; ++tl) {
                if (!mbar_wait(d_empty, (tl & 1) ^ 1)) break;  // the epilogue drained the accumulators
                tc_fence_after();
                for (int kb = 0; kb < nkb; ++kb, ++g) {
                    const int s = g % S;
                    if (!mbar_wait(full(s), (g / S) & 1)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kBwdStepN / 16; ++kk) {
#pragma unroll
                        for (int p = 0; p < kBwdPlanes; ++p) {
                            const uint64_t bd =
                                smem_desc_k_sw64(g_stage(s) + (uint32_t)(p * kBwdPlaneBytes + kk * 32));
#pragma unroll
                            for (int h = 0; h < 2; ++h)
                                mma_f16(tmem + (uint32_t)(h * kBwdTileT),
                                         smem_desc_mn_sw128(a_stage(s) + (uint32_t)(h * kBwdAHalf + kk * 4096),
                                                            1024u, 2048u),
                                         bd, idesc, (kb | kk | p) != 0 ? 1u : 0u);
                        }
                    }
                    mma_commit(empty(s));
                }
                if (ok) mma_commit(d_full);
            }
            mma_commit(mma_done);
            mbar_wait(mma_done, 0);
        }
        __syncwarp();
    } else if (warp >= 4 && warp < 4 + kUnpackWarps) {
        // ---------------- unpack codes into the MN-major fp16 tiles ----------------
        // Group thread: contraction row c = 8 (warp % 4) + lane % 8, features
        // 64 (lane / 8) .. + 64 (16 packed bytes -> eight 16-byte chunks).
        const int par = (warp - 4) >> 2;
        const int enc = (mode >> kModeEncShift) & 3;
        const int c = 8 * (warp & 3) + (lane & 7), fq = lane >> 3;
        const uint32_t r8 = (uint32_t)(c & 7);
        const uint32_t a_off = (uint32_t)((fq >> 1) * kBwdAHalf + (c >> 3) * 2048 + (fq & 1) * 1024) + r8 * 128u;
        for (int g = par; g < total; g += 2) {
            const int ws = g % SW, s = g % S;
            if (!warp_wait_sleep(w_full(ws), (g / SW) & 1, lane)) break;
            uint32_t w[4];
            asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                         : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                         : "r"(sbase + (uint32_t)(kBwdOffW + ws * kBwdWBytes + c * 64 + fq * 16))
                         : "memory");
            if (CONV) {
#pragma unroll
                for (int i = 0; i < 4; ++i) w[i] = codes_to_foundry(w[i], enc);
            }
            uint2 e[16];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int k = 0; k < 4; ++k) e[4 * i + k] = codes4_to_f16((w[i] >> (8 * k)) & 0xFFu);
            if (!warp_wait_sleep(empty(s), ((g / S) & 1) ^ 1, lane)) break;
            const uint32_t base = a_stage(s) + a_off;
#pragma unroll
            for (int k = 0; k < 8; ++k)  // chunk k: features 8k .. 8k + 7 of this thread's 64
                asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(base + ((((uint32_t)k) ^ r8) << 4)),
                             "r"(e[2 * k].x), "r"(e[2 * k].y), "r"(e[2 * k + 1].x), "r"(e[2 * k + 1].y)
                             : "memory");
            fence_proxy_async_smem();
            __syncwarp();
            // The packed slot is released only now: the stores above consume the
            // loaded words, so every lane's read of the slot is complete before
            // the producer may refill it (an arrive right after the loads let a
            // refill overtake a lane's read).
            if (lane == 0) {
                mbar_arrive(w_empty(ws));
                mbar_arrive(full(s));
            }
        }
    } else if (warp >= 12) {
        // ---------------- epilogue ----------------
        constexpr int kChunks = kBwdTileT / 32;
        const int q = warp & 3;
        const int h = (warp - 12) >> 2;  // feature half
        const uint32_t lane_addr = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(h * kBwdTileT);
        for (int tl = 0; tl < my_tiles; ++tl) {
            const int t = (int)blockIdx.x + tl * (int)gridDim.x;
            const int f = (t % num_f) * kBwdTileF + 128 * h + 32 * q + lane;
            const int m0 = (t / num_f) * kBwdTileT;
            if (!warp_wait_sleep(d_full, tl & 1, lane)) break;
            tc_fence_after();
#pragma unroll 1
            for (int cc = 0; cc < kChunks; ++cc) {
                uint32_t v[32];
                tmem_ld32(lane_addr + (uint32_t)(cc * 32), v);
                tmem_ld_wait();
                if (cc == kChunks - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(d_empty);
                }
                const int mb = m0 + cc * 32;
                const int jmax = M - mb;
                const bool in = mb + lane < M;
                const float isl = in ? __ldg(inv_scale + mb + lane) : 1.0f;
                const float rsl = (row_scale && in) ? __ldg(row_scale + mb + lane) : 1.0f;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    float o = __fmul_rn(__uint_as_float(v[j]), __shfl_sync(0xffffffffu, isl, j));  // exact
                    if (row_scale) o = __fmul_rn(o, __shfl_sync(0xffffffffu, rsl, j));
                    v[j] = __float_as_uint(o);
                }
                // 4 x 4 transposes inside each lane quad: lane 4g + r then holds token
                // 4k + r of features 4g .. 4g + 3, stored as one 16-byte vector
                // (K % 64 == 0 keeps every row 16-byte aligned).
                const int r = lane & 3;
                float *xq = dX + (int64_t)(mb + r) * K + (f - r);
                const bool fin = f - r < K;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    float a0 = __uint_as_float(v[4 * k]), a1 = __uint_as_float(v[4 * k + 1]);
                    float a2 = __uint_as_float(v[4 * k + 2]), a3 = __uint_as_float(v[4 * k + 3]);
                    const bool o1 = r & 1;
                    const float x1 = __shfl_xor_sync(0xffffffffu, o1 ? a0 : a1, 1);
                    const float y1 = __shfl_xor_sync(0xffffffffu, o1 ? a2 : a3, 1);
                    if (o1) { a0 = x1; a2 = y1; } else { a1 = x1; a3 = y1; }
                    const bool o2 = r & 2;
                    const float x2 = __shfl_xor_sync(0xffffffffu, o2 ? a0 : a2, 2);
                    const float y2 = __shfl_xor_sync(0xffffffffu, o2 ? a1 : a3, 2);
                    if (o2) { a0 = x2; a1 = y2; } else { a2 = x2; a3 = y2; }
                    if (fin && 4 * k + r < jmax) {
                        float4 *p = reinterpret_cast<float4 *>(xq + (int64_t)(4 * k) * K);
                        if (accumulate) {
                            const float4 b = *p;
                            a0 = __fadd_rn(b.x, a0), a1 = __fadd_rn(b.y, a1);
                            a2 = __fadd_rn(b.z, a2), a3 = __fadd_rn(b.w, a3);
                        }
                        __stcs(p, make_float4(a0, a1, a2, a3));
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kBwdTmemCols);
    }
}

}  // namespace tq
