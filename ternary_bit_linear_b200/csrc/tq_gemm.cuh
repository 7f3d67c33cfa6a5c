// tq_gemm.cuh -- prefill ternary GEMM on the 5th-generation tensor cores.
//
// Hetman-2b, src/quantization.py, section 5 steps 5-6 (y_int32 = x_q W^T,
// then y = y_int32 * gamma / scale_x); Foundry, docs/quantization.md,
// "Native Matmul Kernel".  The contraction is a dense int8 GEMM, so it runs
// as tcgen05.mma kind::i8 with int32 accumulators in tensor memory.
//
// Tile: 128 output features (the MMA's M, taken by the weights) x BT tokens
// (the MMA's N, 64..256) x 128 codes of K per pipeline stage.
//
//   warp 0      TMA producer: x_q tile [BT][128] (128-byte swizzle, the
//               canonical K-major layout) and packed tile [128][32 B].
//   warp 1      TMEM owner and single-thread MMA issuer (4 MMAs of K = 32
//               per stage); tcgen05.commit frees the stage.
//   warps 4-7   unpackers, then epilogue.  Thread r unpacks row r of the
//               packed tile: the 2-bit fields become unsigned bytes c = q + 1
//               in natural K order (four 16-code words -> 4x4 byte transpose),
//               written in the 128-byte-swizzle K-major layout the MMA reads.
//               The epilogue reads D (lane = feature, column = token) with
//               tcgen05.ld and writes y = (D - rowsum) * gamma * s_x with
//               one coalesced 128-byte store per token and warp.
//
// Every mbarrier wait is bounded (see mbar_wait); on a timeout the kernel
// records it in the status word, skips the remaining work and still frees
// its tensor memory.
#pragma once

#include <cuda.h>

#include "tq_common.cuh"

namespace tq {

constexpr int kGemmThreads = 256;
constexpr int kGemmStages = 4;
constexpr int kTileN = 128;   // features per tile (MMA M)
constexpr int kTileK = 128;   // codes (bytes of x_q) per stage

template <int BT>
struct GemmLayout {
    static constexpr int kA = kTileN * kTileK;   // unpacked weights per stage
    static constexpr int kB = BT * kTileK;       // x_q per stage
    static constexpr int kP = kTileN * kTileK / 4;  // packed weights per stage
    static constexpr int offA = 0;
    static constexpr int offB = offA + kGemmStages * kA;
    static constexpr int offP = offB + kGemmStages * kB;
    static constexpr int offBar = offP + kGemmStages * kP;
    // barriers: full_tma[S], full_a[S], empty[S], tmem_full
    static constexpr int offTmem = offBar + (3 * kGemmStages + 1) * 8;
    static constexpr int offSx = offTmem + 16;
    static constexpr int offRs = offSx + BT * 4;
    static constexpr int offG = offRs + BT * 4;
    static constexpr int kBytes = offG + kTileN * 4;
    static constexpr int kDynamic = kBytes + 1024;  // slack for 1024-byte alignment
    static constexpr uint32_t kTx = kB + kP;
    static constexpr uint32_t kTmemCols = BT < 32 ? 32 : BT;
};

// Natural-order expansion of one 32-bit packed word (16 codes) into 16
// unsigned bytes c_i = field_i (0, 1, 2), as a 16-byte chunk.
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

template <int BT>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                const float *__restrict__ s_x, const int32_t *__restrict__ rowsum,
                const float *__restrict__ gamma, int per_row, int M, int N, int K,
                float *__restrict__ y, int32_t *__restrict__ acc_out) {
    using L = GemmLayout<BT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + L::offBar;
    auto full_tma = [&](int s) { return bar0 + 8u * s; };
    auto full_a = [&](int s) { return bar0 + 8u * (kGemmStages + s); };
    auto empty = [&](int s) { return bar0 + 8u * (2 * kGemmStages + s); };
    const uint32_t tmem_full = bar0 + 8u * (3 * kGemmStages);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::offTmem);
    float *sx_s = reinterpret_cast<float *>(smem + L::offSx);
    int *rs_s = reinterpret_cast<int *>(smem + L::offRs);
    float *g_s = reinterpret_cast<float *>(smem + L::offG);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * kTileN, m0 = blockIdx.y * BT;
    const int nkb = (K + kTileK - 1) / kTileK;

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < kGemmStages; ++s) {
            mbar_init(full_tma(s), 1);
            mbar_init(full_a(s), 4);
            mbar_init(empty(s), 1);
        }
        mbar_init(tmem_full, 1);
        fence_barrier_init();
        prefetch_tmap(&tm_x);
        prefetch_tmap(&tm_w);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
        tmem_relinquish();
    }
    if (warp >= 4) {
        const int i = threadIdx.x - 128;
        for (int j = i; j < BT; j += 128) {
            const int m = m0 + j;
            sx_s[j] = m < M ? s_x[m] : 0.0f;
            rs_s[j] = m < M ? rowsum[m] : 0;
        }
        const int n = n0 + i;
        g_s[i] = n < N ? (per_row ? gamma[n] : gamma[0]) : 0.0f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_d = *tmem_slot;

    if (warp == 0) {
        // ---------------- TMA producer (lane 0 issues; the warp stays converged) ----------------
        int issued = 0;
        for (int kb = 0; kb < nkb; ++kb) {
            const int s = kb % kGemmStages, r = kb / kGemmStages;
            if (!warp_wait(empty(s), (r & 1) ^ 1, lane)) break;
            if (lane == 0) {
                mbar_arrive_expect_tx(full_tma(s), L::kTx);
                tma_load_2d(sbase + L::offB + s * L::kB, &tm_x, kb * kTileK, m0, full_tma(s));
                tma_load_2d(sbase + L::offP + s * L::kP, &tm_w, kb * (kTileK / 4), n0, full_tma(s));
            }
            __syncwarp();
            issued = kb + 1;
        }
        // Own copies must have landed before the CTA may exit (already true
        // unless a wait above gave up).
        for (int kb = issued - kGemmStages < 0 ? 0 : issued - kGemmStages; kb < issued; ++kb)
            warp_wait(full_tma(kb % kGemmStages), (kb / kGemmStages) & 1, lane);
    } else if (warp == 1) {
        // ---------------- MMA issuer (lane 0 issues) ----------------
        constexpr uint32_t idesc = idesc_i8_u8s8(kTileN, BT);
        for (int kb = 0; kb < nkb; ++kb) {
            const int s = kb % kGemmStages, r = kb / kGemmStages;
            if (!warp_wait(full_a(s), r & 1, lane) || !warp_wait(full_tma(s), r & 1, lane)) break;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t a_addr = sbase + L::offA + s * L::kA;
                const uint32_t b_addr = sbase + L::offB + s * L::kB;
#pragma unroll
                for (int kk = 0; kk < kTileK / 32; ++kk)
                    mma_i8(tmem_d, smem_desc_sw128(a_addr + kk * 32),
                           smem_desc_sw128(b_addr + kk * 32), idesc, (kb | kk) != 0 ? 1u : 0u);
                mma_commit(empty(s));
            }
            __syncwarp();
        }
        if (lane == 0) mma_commit(tmem_full);  // fires once every MMA issued above has completed
        __syncwarp();
        warp_wait(tmem_full, 0, lane);  // no MMA may still write TMEM when it is freed
    } else if (warp >= 4) {
        // ---------------- unpack ----------------
        const int r = threadIdx.x - 128;  // row of the tile, 0..127
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
            const int s = kb % kGemmStages, rr = kb / kGemmStages;
            if (!warp_wait(full_tma(s), rr & 1, lane)) {
                ok = false;
                break;
            }
            const uint8_t *prow = smem + L::offP + s * L::kP + r * 32;
            const uint4 p0 = *reinterpret_cast<const uint4 *>(prow);
            const uint4 p1 = *reinterpret_cast<const uint4 *>(prow + 16);
            const uint32_t words[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
            uint8_t *arow = smem + L::offA + s * L::kA + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c)
                *reinterpret_cast<uint4 *>(arow + ((c ^ (r & 7)) << 4)) = expand_word(words[c]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(full_a(s));
        }
        // ---------------- epilogue ----------------
        const int q = warp - 4;  // TMEM lane quarter of this warp
        if (ok && warp_wait(tmem_full, 0, lane)) {
            tc_fence_after();
            const int n = n0 + 32 * q + lane;
            const float gn = g_s[32 * q + lane];
#pragma unroll 1
            for (int cc = 0; cc < BT / 32; ++cc) {
                uint32_t v[32];
                tmem_ld32(tmem_d + ((uint32_t)(32 * q) << 16) + (uint32_t)(cc * 32), v);
                tmem_ld_wait();
                if (n < N) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int mj = cc * 32 + j;
                        const int m = m0 + mj;
                        if (m < M) {
                            const int a = (int)v[j] - rs_s[mj];
                            y[(int64_t)m * N + n] =
                                __fmul_rn(__int2float_rn(a), __fmul_rn(gn, sx_s[mj]));
                            if (acc_out) acc_out[(int64_t)m * N + n] = a;
                        }
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_d, L::kTmemCols);
    }
}

}  // namespace tq
