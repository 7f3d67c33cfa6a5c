// tq_gemm.cuh -- prefill ternary GEMM on the 5th-generation tensor cores.
//
// Hetman-2b, src/quantization.py, section 5 steps 5-6 (y_int32 = x_q W^T,
// then y = y_int32 * gamma / scale_x); Foundry, docs/quantization.md,
// "Native Matmul Kernel".  The contraction is a dense int8 GEMM, so it runs
// as tcgen05.mma kind::i8 with int32 accumulators in tensor memory.
//
// Persistent: one CTA per SM walks output tiles of 128 features (the MMA's M,
// taken by the weights) x BT tokens (the MMA's N), token blocks fastest so
// that concurrently running CTAs share x_q and weight tiles in L2.  K is
// consumed in steps of 128 codes.  Sixteen warps:
//
//   warp 0      TMA producer: x_q tile [BT][128 B] (128-byte swizzle, the
//               canonical K-major operand layout) into a shared-memory ring.
//   warp 1      TMEM owner and single-thread MMA issuer: per step 4 MMAs of
//               K = 32 with the weight operand read from tensor memory; the
//               accumulator alternates between two TMEM buffers per tile.
//   warps 4-11  unpackers.  Warps 4-7 take even steps, 8-11 odd steps; thread
//               r of quarter q owns TMEM lane 32q + r = weight row r of the
//               tile: it loads its 32 packed bytes (prefetched one step ahead
//               with 16-byte non-coherent loads), expands them to 128 unsigned
//               codes c = q + 1 in natural K order and writes them with
//               tcgen05.st into one of 8 TMEM operand slots.
//   warps 12-15 epilogue: wait for a finished accumulator, read it with
//               tcgen05.ld (lane = feature, column = token), release it, and
//               write y = (acc - rowsum) * gamma * s_x with evict-first
//               128-byte stores -- overlapping the next tile's MMAs.
//
// Tensor memory: accumulators in columns [0, 2 BT), operand slots after them.
// Every mbarrier wait is bounded (see mbar_wait); on a timeout the kernel
// records it in the status word, skips the remaining work and still frees
// its tensor memory.
#pragma once

#include <cuda.h>

#include "tq_common.cuh"

namespace tq {

constexpr int kGemmThreads = 512;
constexpr int kGemmAStages = 8;  // tensor-memory slots for the unpacked weights
constexpr int kTileN = 128;      // features per tile (MMA M)
constexpr int kTileK = 128;      // codes (bytes of x_q) per step

__host__ __device__ constexpr uint32_t pow2_at_least(uint32_t v) {
    uint32_t p = 32;
    while (p < v) p <<= 1;
    return p;
}

template <int BT>
struct GemmLayout {
    static constexpr int kStages = BT >= 128 ? 10 : 12;  // x_q ring
    static constexpr int kB = BT * kTileK;               // x_q bytes per stage
    static constexpr int offB = 0;
    static constexpr int offBar = offB + kStages * kB;
    // barriers: full[S], empty[S], a_full[SA], a_empty[SA], d_full[2], d_empty[2], mma_done
    static constexpr int kBars = 2 * kStages + 2 * kGemmAStages + 5;
    static constexpr int offTmem = offBar + kBars * 8;
    static constexpr int kBytes = offTmem + 16;
    static constexpr int kDynamic = kBytes + 1024;  // slack for 1024-byte alignment
    static constexpr uint32_t kACol = 2 * BT;       // first TMEM column of the operand slots
    static constexpr uint32_t kTmemCols = pow2_at_least(2 * BT + kGemmAStages * (kTileK / 4));
};

// Natural-order expansion of one 32-bit packed word (16 codes) into 16
// unsigned bytes c_i = field_i (0, 1, 2), as four 32-bit words.
__device__ __forceinline__ uint4 expand_word(uint32_t w) {
    const uint32_t e0 = w & 0x03030303u;          // fields 0, 4, 8, 12
    const uint32_t e1 = (w >> 2) & 0x03030303u;   // fields 1, 5, 9, 13
    const uint32_t e2 = (w >> 4) & 0x03030303u;   // fields 2, 6, 10, 14
    const uint32_t e3 = (w >> 6) & 0x03030303u;   // fields 3, 7, 11, 15
    const uint32_t t0 = __byte_perm(e0, e1, 0x5140), t1 = __byte_perm(e0, e1, 0x7362);
    const uint32_t t2 = __byte_perm(e2, e3, 0x5140), t3 = __byte_perm(e2, e3, 0x7362);
    return make_uint4(__byte_perm(t0, t2, 0x5410), __byte_perm(t0, t2, 0x7632),
                      __byte_perm(t1, t3, 0x5410), __byte_perm(t1, t3, 0x7632));
}

__device__ __forceinline__ uint4 ldg_nc_u4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

template <int BT>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const uint8_t *__restrict__ packed,
                const float *__restrict__ s_x, const int32_t *__restrict__ rowsum,
                const float *__restrict__ gamma, int per_row, int M, int N, int K,
                float *__restrict__ y, int32_t *__restrict__ acc_out) {
    using L = GemmLayout<BT>;
    constexpr int S = L::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + L::offBar;
    auto full = [&](int s) { return bar0 + 8u * s; };
    auto empty = [&](int s) { return bar0 + 8u * (S + s); };
    auto a_full = [&](int s) { return bar0 + 8u * (2 * S + s); };
    auto a_empty = [&](int s) { return bar0 + 8u * (2 * S + kGemmAStages + s); };
    auto d_full = [&](int b) { return bar0 + 8u * (2 * S + 2 * kGemmAStages + b); };
    auto d_empty = [&](int b) { return bar0 + 8u * (2 * S + 2 * kGemmAStages + 2 + b); };
    const uint32_t mma_done = bar0 + 8u * (2 * S + 2 * kGemmAStages + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::offTmem);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_m = (M + BT - 1) / BT, num_n = (N + kTileN - 1) / kTileN;
    const int ntiles = num_m * num_n;
    const int nkb = (K + kTileK - 1) / kTileK;
    const int KB = K / 4;  // packed bytes per weight row

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        for (int s = 0; s < kGemmAStages; ++s) {
            mbar_init(a_full(s), 4);
            mbar_init(a_empty(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(d_full(b), 1);
            mbar_init(d_empty(b), 4);
        }
        mbar_init(mma_done, 1);
        fence_barrier_init();
        prefetch_tmap(&tm_x);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
        tmem_relinquish();
    }
    // Everything above touched no global memory; inputs of the previous kernel
    // on the stream are visible after this wait.
    pdl_wait();
    pdl_trigger();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------- TMA producer (lane 0 issues; the warp stays converged) ----------------
        int g = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            const int m0 = (t % num_m) * BT;
            for (int kb = 0; kb < nkb; ++kb, ++g) {
                const int s = g % S, r = g / S;
                if (!warp_wait(empty(s), (r & 1) ^ 1, lane)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    mbar_arrive_expect_tx(full(s), L::kB);
                    tma_load_2d(sbase + L::offB + s * L::kB, &tm_x, kb * kTileK, m0, full(s));
                }
                __syncwarp();
            }
        }
        // Own copies must have landed before the CTA may exit (already true
        // unless a wait above gave up).
        for (int j = g - S < 0 ? 0 : g - S; j < g; ++j) warp_wait(full(j % S), (j / S) & 1, lane);
    } else if (warp == 1) {
        // ---------------- MMA issuer (lane 0 issues) ----------------
        constexpr uint32_t idesc = idesc_i8_u8s8(kTileN, BT);
        int g = 0, tl = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++tl) {
            const int b = tl & 1;
            if (!warp_wait(d_empty(b), ((tl >> 1) & 1) ^ 1, lane)) break;
            tc_fence_after();
            const uint32_t d_col = tmem + (uint32_t)(b * BT);
            for (int kb = 0; kb < nkb; ++kb, ++g) {
                const int s = g % S, r = g / S;
                const int sa = g % kGemmAStages, ra = g / kGemmAStages;
                if (!warp_wait(full(s), r & 1, lane) || !warp_wait(a_full(sa), ra & 1, lane)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t a_col = tmem + L::kACol + (uint32_t)sa * (kTileK / 4);
                    const uint32_t b_addr = sbase + L::offB + s * L::kB;
#pragma unroll
                    for (int kk = 0; kk < kTileK / 32; ++kk)
                        mma_i8_ts(d_col, a_col + kk * 8, smem_desc_sw128(b_addr + kk * 32), idesc,
                                  (kb | kk) != 0 ? 1u : 0u);
                    mma_commit(empty(s));
                    mma_commit(a_empty(sa));
                }
                __syncwarp();
            }
            if (ok && lane == 0) mma_commit(d_full(b));  // accumulator b complete
            __syncwarp();
        }
        // No MMA may still use TMEM when it is freed: this commit fires once
        // every MMA issued above has completed.
        if (lane == 0) mma_commit(mma_done);
        __syncwarp();
        warp_wait(mma_done, 0, lane);
    } else if (warp >= 4 && warp < 12) {
        // ---------------- unpack into tensor memory ----------------
        const int q = warp & 3;            // TMEM lane quarter
        const int par = (warp - 4) >> 2;   // steps g with g % 2 == par
        const int r = 32 * q + lane;       // row of the tile = TMEM lane
        const uint32_t lane_addr = tmem + ((uint32_t)(32 * q) << 16);
        const int total = ((ntiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x) * nkb;
        // packed bytes of step g for this thread's row (zeros past N or K)
        auto load_step = [&](int gg, uint4 &v0, uint4 &v1) {
            v0 = make_uint4(0u, 0u, 0u, 0u);
            v1 = v0;
            if (gg >= total) return;
            const int tt = (int)blockIdx.x + (gg / nkb) * (int)gridDim.x;
            const int kb = gg % nkb;
            const int n = (tt / num_m) * kTileN + r;
            if (n >= N) return;
            const uint8_t *src = packed + (int64_t)n * KB + kb * 32;
            if (kb * 32 + 16 <= KB) v0 = ldg_nc_u4(src);
            if (kb * 32 + 32 <= KB) v1 = ldg_nc_u4(src + 16);
        };
        uint4 c0, c1, n0_, n1_;
        load_step(par, c0, c1);
        for (int g = par; g < total; g += 2) {
            load_step(g + 2, n0_, n1_);  // prefetch this warp's next step
            const int sa = g % kGemmAStages, ra = g / kGemmAStages;
            const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
            uint32_t cols[32];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 e = expand_word(words[c]);
                cols[4 * c + 0] = e.x;
                cols[4 * c + 1] = e.y;
                cols[4 * c + 2] = e.z;
                cols[4 * c + 3] = e.w;
            }
            if (!warp_wait(a_empty(sa), (ra & 1) ^ 1, lane)) break;
            tc_fence_after();
            tmem_st32(lane_addr + L::kACol + (uint32_t)sa * (kTileK / 4), cols);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(a_full(sa));
            c0 = n0_;
            c1 = n1_;
        }
    } else if (warp >= 12) {
        // ---------------- epilogue ----------------
        const int q = warp & 3;
        const uint32_t lane_addr = tmem + ((uint32_t)(32 * q) << 16);
        int tl = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++tl) {
            const int b = tl & 1;
            if (!warp_wait(d_full(b), (tl >> 1) & 1, lane)) break;
            tc_fence_after();
            const int m0 = (t % num_m) * BT, n0 = (t / num_m) * kTileN;
            const int n = n0 + 32 * q + lane;
            const float gn = n < N ? __ldg(gamma + (per_row ? n : 0)) : 0.0f;
#pragma unroll 1
            for (int cc = 0; cc < BT / 32; ++cc) {
                uint32_t v[32];
                tmem_ld32(lane_addr + (uint32_t)(b * BT + cc * 32), v);
                // this chunk's 32 tokens: lane j holds token m0 + 32 cc + j
                const int mj = m0 + cc * 32 + lane;
                const float sxj = mj < M ? __ldg(s_x + mj) : 0.0f;
                const int rsj = mj < M ? __ldg(rowsum + mj) : 0;
                tmem_ld_wait();
                if (cc == BT / 32 - 1) {  // accumulator fully read: hand it back to the MMA warp
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(d_empty(b));
                }
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float sxm = __shfl_sync(0xffffffffu, sxj, j);
                    const int rsm = __shfl_sync(0xffffffffu, rsj, j);
                    const int m = m0 + cc * 32 + j;
                    if (m < M && n < N) {
                        const int a = (int)v[j] - rsm;
                        __stcs(y + (int64_t)m * N + n, __fmul_rn(__int2float_rn(a), __fmul_rn(gn, sxm)));
                        if (acc_out) __stcs(acc_out + (int64_t)m * N + n, a);
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, L::kTmemCols);
    }
}

}  // namespace tq
