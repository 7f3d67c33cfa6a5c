// tq_gemm.cuh -- prefill ternary GEMM on the 5th-generation tensor cores.
//
// Hetman-2b, src/quantization.py, section 5 steps 5-6 (y_int32 = x_q W^T,
// then y = y_int32 * gamma / scale_x); Foundry, docs/quantization.md,
// "Native Matmul Kernel".  The contraction is a dense int8 GEMM, so it runs
// as tcgen05.mma kind::i8 with int32 accumulators in tensor memory.
//
// Persistent: one CTA per SM walks output tiles of 128 features (the MMA's M,
// taken by the weights) x BT tokens (the MMA's N: 64, 128 or 256, chosen
// per problem by the launcher to fill the SMs), token blocks
// fastest so that concurrently running CTAs share weight tiles in L2.  K is
// consumed in steps of 128 codes; one step is four MMAs of K = 32, the codes
// (A) read from tensor memory and x_q (B) from shared memory (128-byte
// swizzled, K-major).  Twenty warps:
//
//   warp 0      x_q producer (lane 0): TMA of the x_q tile [BT][128 B] into
//               stage s of the operand ring.
//   warp 1      TMEM owner; lane 0 issues the MMAs.  Per step: one wait on
//               full(s), four MMAs, one commit that frees stage s.  The
//               accumulator alternates between two TMEM buffers per tile
//               (BT <= 128) or is a single buffer (BT = 256).
//   warp 2      weight producer (lane 0): TMA of the packed tile [128][32 B]
//               into a deeper ring of its own, so that weights coming from
//               HBM are requested well before they are needed.
//   warps 4-11  unpackers, two groups of four taking alternate steps: thread
//               r of a group expands row r's 32 packed bytes to 128 unsigned
//               codes c = q + 1 in {0, 1, 2} and stores them into TMEM lane r
//               of stage s's code tile (tcgen05.st).
//   warps 12-19 epilogue: wait for a finished accumulator, read it with
//               tcgen05.ld (lane = feature, column = token), release it, and
//               write y = (acc - rowsum) * gamma * s_x with evict-first
//               stores -- overlapping the next tile's MMAs where there are
//               two accumulator buffers.
//
// The single-thread issue loops matter: an MMA-issuing warp that waits with
// warp-wide votes or commits twice per step leaves the tensor pipe idle for
// longer than a K = 32 MMA lasts.
//
// sum_k x * c = sum_k x * q + sum_k x, so the epilogue subtracts the token's
// rowsum.  Zero-filled tails (tokens >= M, features >= N, codes >= K) carry
// x = 0 or c = 0 and add nothing.  Every mbarrier wait is bounded (see
// mbar_wait); on a timeout the kernel records it in the status word, skips
// the remaining work, lets its copies land and still frees its tensor memory.
#pragma once

#include <cuda.h>

#include "tq_common.cuh"

namespace tq {

constexpr int kGemmWarps = 20;
constexpr int kGemmThreads = 32 * kGemmWarps;
constexpr int kUnpackWarps = 8;  // warps 4 .. 11
constexpr int kEpiWarps = 8;     // warps 12 .. 19
constexpr int kTileN = 128;      // features per tile (MMA M)
constexpr int kTileK = 128;      // codes (bytes of x_q) per step
constexpr int kWStageBytes = kTileN * kTileK / 4;  // packed bytes of one step's weight tile

__host__ __device__ constexpr uint32_t pow2_at_least(uint32_t v) {
    uint32_t p = 32;
    while (p < v) p <<= 1;
    return p;
}

// The unpacked codes (the A operand) live in tensor memory -- written by the
// unpackers with tcgen05.st, read by the MMA from TMEM -- so neither their
// stores nor the MMA's A reads take shared-memory bandwidth.  TMEM holds the
// accumulators and one 32-column code tile (128 lanes x 128 codes) per stage:
// two accumulators up to BT = 128, one for larger tiles (the MMAs of a tile
// then start once the epilogue has read the previous tile's accumulator).
// Shared memory holds the x_q ring (the B operand) and the packed-weight ring.
template <int BT>
struct GemmLayout {
    static constexpr int kAccBufs = BT > 128 ? 1 : 2;
    static constexpr int kWStages = 8;      // packed-weight ring
    static constexpr int kB = BT * kTileK;  // x_q bytes per stage
    static constexpr int kStage = kB;
    // x_q ring: as many stages as fit beside the weight ring, at most 8
    // (6 for BT = 256, 8 for the smaller tiles)
    static constexpr int kStagesFit = (232448 - 1024 - 512 - kWStages * kWStageBytes) / kStage;
    static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
    static constexpr int kACols = kTileK / 4;  // TMEM columns of one stage's code tile
    static constexpr int offStage = 0;  // stage s: x_q tile (1024-aligned)
    static constexpr int offW = kStages * kStage;
    static constexpr int offBar = offW + kWStages * kWStageBytes;
    // barriers: full[S], empty[S], w_full[SW], w_empty[SW], d_full[2], d_empty[2], mma_done
    static constexpr int kBars = 2 * kStages + 2 * kWStages + 5;
    static constexpr int offTmem = offBar + kBars * 8;
    static constexpr int kBytes = offTmem + 16;
    static constexpr int kDynamic = kBytes + 1024;  // slack for 1024-byte alignment
    // accumulator buffers start at multiples of kDStride TMEM columns; the
    // code stages follow them
    static constexpr int kDStride = BT <= 128 ? BT : 256;
    static constexpr int kAColBase = kAccBufs * kDStride;
    static constexpr uint32_t kTmemCols = pow2_at_least(kAColBase + kStages * kACols);
    static_assert(kTmemCols <= 512, "tensor memory columns");
    static_assert(kDynamic <= 232448, "shared memory per CTA");
    static_assert(kB % 1024 == 0, "swizzle atoms stay aligned");
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

// CONV: the weights are packed in one of Hetman-2b's layouts (mode bits
// 2-3) and every word is rewritten in Foundry's layout before the unpack; the
// default layout compiles without that step.  EPI: the extra epilogue `ep`
// (bias, integer bias and shift) is applied.
template <int BT, bool CONV, bool EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
    tq_gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                const float *__restrict__ s_x, const int32_t *__restrict__ rowsum,
                const float *__restrict__ gamma, int per_row, int M, int N, int K,
                float *__restrict__ y, int32_t *__restrict__ acc_out, int mode, Epilogue ep) {
    using L = GemmLayout<BT>;
    constexpr int S = L::kStages, SW = L::kWStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + L::offBar;
    auto full = [&](int s) { return bar0 + 8u * s; };
    auto empty = [&](int s) { return bar0 + 8u * (S + s); };
    auto w_full = [&](int s) { return bar0 + 8u * (2 * S + s); };
    auto w_empty = [&](int s) { return bar0 + 8u * (2 * S + SW + s); };
    auto d_full = [&](int b) { return bar0 + 8u * (2 * S + 2 * SW + b); };
    auto d_empty = [&](int b) { return bar0 + 8u * (2 * S + 2 * SW + 2 + b); };
    const uint32_t mma_done = bar0 + 8u * (2 * S + 2 * SW + 4);
    auto x_stage = [&](int s) { return sbase + (uint32_t)(L::offStage + s * L::kStage); };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::offTmem);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_m = (M + BT - 1) / BT, num_n = (N + kTileN - 1) / kTileN;
    const int ntiles = num_m * num_n;
    const int nkb = (K + kTileK - 1) / kTileK;
    // steps this CTA runs: its tiles times the steps per tile
    const int my_tiles = ntiles > (int)blockIdx.x
                             ? (ntiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x
                             : 0;
    const int total = my_tiles * nkb;

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full(s), 1 + kUnpackWarps / 2);  // TMA bytes + the step's four unpacker warps
            mbar_init(empty(s), 1);
        }
        for (int s = 0; s < SW; ++s) {
            mbar_init(w_full(s), 1);
            mbar_init(w_empty(s), kUnpackWarps / 2);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(d_full(b), 1);
            mbar_init(d_empty(b), kEpiWarps);
        }
        mbar_init(mma_done, 1);
        fence_barrier_init();
        prefetch_tmap(&tm_x);
        prefetch_tmap(&tm_w);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
        tmem_relinquish();
    }
    // Everything above touched no global memory; inputs of the previous kernel
    // on the stream are visible after this wait.  With static weights only the
    // roles that read x_q, s_x, rowsum or write y wait (the weight producer,
    // the unpackers and the MMA issuer start at once); with ready inputs no
    // role waits here and the kernel waits before exiting instead (stream
    // completion order).
    const bool ready = (mode & kModeInputsReady) != 0;
    const bool w_early = (mode & (kModeWeightsStatic | kModeInputsReady)) != 0;
    if (!w_early) pdl_wait();
    pdl_trigger();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------- x_q producer ----------------
        if (w_early && !ready) pdl_wait();
        if (lane == 0) {
            int g = 0;
            for (; g < total; ++g) {
                const int s = g % S, r = g / S;
                const int t = (int)blockIdx.x + (g / nkb) * (int)gridDim.x;
                const int kb = g % nkb;
                if (!mbar_wait_sleep(empty(s), (r & 1) ^ 1)) break;
                mbar_arrive_expect_tx(full(s), L::kB);
                tma_load_2d(x_stage(s), &tm_x, kb * kTileK, (t % num_m) * BT, full(s));
            }
            // Own copies must have landed before the CTA may exit (already
            // true unless a wait gave up).
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
                mbar_arrive_expect_tx(w_full(s), kWStageBytes);
                tma_load_2d(sbase + (uint32_t)(L::offW + s * kWStageBytes), &tm_w, kb * (kTileK / 4),
                            (t / num_m) * kTileN, w_full(s));
            }
            for (int j = g - SW < 0 ? 0 : g - SW; j < g; ++j) mbar_wait(w_full(j % SW), (j / SW) & 1);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_i8_u8s8(kTileN, BT);
            int g = 0;
            bool ok = true;
            for (int tl = 0; tl < my_tiles && ok; ++tl) {
                const int b = tl % L::kAccBufs;
                if (!mbar_wait(d_empty(b), ((tl / L::kAccBufs) & 1) ^ 1)) break;
                tc_fence_after();
                const uint32_t d_col = tmem + (uint32_t)(b * L::kDStride);
                for (int kb = 0; kb < nkb; ++kb, ++g) {
                    const int s = g % S;
                    if (!mbar_wait(full(s), (g / S) & 1)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t b_addr = x_stage(s);
                    // codes of stage s: TMEM columns kAColBase + 32 s ..., 8 columns per K = 32
                    const uint32_t a_col = tmem + (uint32_t)(L::kAColBase + s * L::kACols);
#pragma unroll
                    for (int kk = 0; kk < kTileK / 32; ++kk)
                        mma_i8_ts(d_col, a_col + (uint32_t)(kk * 8), smem_desc_sw128(b_addr + kk * 32), idesc,
                                  (kb | kk) != 0 ? 1u : 0u);
                    mma_commit(empty(s));
                }
                if (ok) mma_commit(d_full(b));  // accumulator b complete
            }
            // No MMA may still use TMEM when it is freed: this commit fires
            // once every MMA issued above has completed.
            mma_commit(mma_done);
            mbar_wait(mma_done, 0);
        }
        __syncwarp();
    } else if (warp >= 4 && warp < 4 + kUnpackWarps) {
        // ---------------- unpack codes into the TMEM operand tile ----------------
        // Two groups of four warps take alternate steps, so each has two steps'
        // time for its waits, loads and stores; thread r of a group owns row r.
        const int par = (warp - 4) >> 2;
        const int enc = (mode >> kModeEncShift) & 3;  // packed-code layout
        const int r = 32 * (warp & 3) + lane;  // weight row of the tile
        const uint32_t w_row = sbase + (uint32_t)(L::offW + r * (kTileK / 4));
        for (int g = par; g < total; g += 2) {
            const int ws = g % SW, s = g % S;
            if (!warp_wait_sleep(w_full(ws), (g / SW) & 1, lane)) break;
            uint4 p0, p1;
            const uint32_t src = w_row + (uint32_t)(ws * kWStageBytes);
            // Rows are 32 bytes apart, so rows r and r + 4 share banks: threads
            // with (r >> 2) odd read their second half first, which makes each
            // quarter warp's 16-byte loads hit eight distinct bank groups.
            const uint32_t h = (uint32_t)((r >> 2) & 1) << 4;
            asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                         : "=r"(p0.x), "=r"(p0.y), "=r"(p0.z), "=r"(p0.w)
                         : "r"(src + h)
                         : "memory");
            asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                         : "=r"(p1.x), "=r"(p1.y), "=r"(p1.z), "=r"(p1.w)
                         : "r"(src + (h ^ 16u))
                         : "memory");
            if (h) {  // back to natural order
                const uint4 tmp = p0;
                p0 = p1;
                p1 = tmp;
            }
            uint32_t words[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
            if (CONV) {
#pragma unroll
                for (int c = 0; c < 8; ++c) words[c] = codes_to_foundry(words[c], enc);
            }
            uint4 e[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) e[c] = expand_word(words[c]);
            if (!warp_wait_sleep(empty(s), ((g / S) & 1) ^ 1, lane)) break;
            // row r's 128 codes -> TMEM lane r (this warp's lane quarter is
            // 32 (warp % 4) .. + 31), 32 consecutive columns of 4 codes each
            uint32_t cw[32];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                cw[4 * c] = e[c].x;
                cw[4 * c + 1] = e[c].y;
                cw[4 * c + 2] = e[c].z;
                cw[4 * c + 3] = e[c].w;
            }
            tmem_st32(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(L::kAColBase + s * L::kACols), cw);
            tmem_st_wait();
            tc_fence_before();  // the stores are complete before the MMA warp is told
            __syncwarp();
            // The packed slot is released only now: the stores above consume the
            // loaded words, so every lane's read of the slot is complete before
            // the producer may refill it.
            if (lane == 0) {
                mbar_arrive(w_empty(ws));
                mbar_arrive(full(s));
            }
        }
    } else if (warp >= 12) {
        // ---------------- epilogue ----------------
        if (w_early && !ready) pdl_wait();
        constexpr int kHalf = BT / 2;          // tokens per epilogue warp and tile
        constexpr int kChunks = kHalf / 32;
        const int q = warp & 3;                // TMEM lane quarter
        const int half = (warp - 12) >> 2;     // token half of the tile
        const uint32_t lane_addr = tmem + ((uint32_t)(32 * q) << 16);
        const bool vec4 = (N & 3) == 0;  // rows of y are 16-byte multiples
        // vec4 layout: after a 4 x 4 transpose inside each lane quad, lane 4g + r
        // holds token 4k + r of the quad's features 4g .. 4g + 3 (one 16-byte store)
        const int r = lane & 3;
        for (int tl = 0; tl < my_tiles; ++tl) {
            const int t = (int)blockIdx.x + tl * (int)gridDim.x;
            const int b = tl % L::kAccBufs;
            const int m0 = (t % num_m) * BT + half * kHalf, n0 = (t / num_m) * kTileN;
            const int n = n0 + 32 * q + lane;
            const int nq = n - r;  // first feature of the lane's quad
            // per-tile scalars, loaded while the accumulator is still being computed
            float gn = 0.0f, bn = 0.0f;
            int abn = 0;
            float g4[4] = {0.0f, 0.0f, 0.0f, 0.0f}, b4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            float sxc[kChunks];
            int rsc[kChunks];
            const bool quads = vec4 && !acc_out;
            if (quads) {
                if (nq < N) {  // N % 4 == 0: the quad's four features are all < N
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        g4[i] = __ldg(gamma + (per_row ? nq + i : 0));
                        if (EPI && ep.bias) b4[i] = __ldg(ep.bias + nq + i);
                    }
                }
            } else {
                gn = n < N ? __ldg(gamma + (per_row ? n : 0)) : 0.0f;
                bn = (EPI && n < N && ep.bias) ? __ldg(ep.bias + n) : 0.0f;
                abn = (EPI && n < N && ep.acc_bias) ? __ldg(ep.acc_bias + n) : 0;
#pragma unroll
                for (int cc = 0; cc < kChunks; ++cc) {
                    const int mj = m0 + cc * 32 + lane;  // lane j holds token m0 + 32 cc + j
                    sxc[cc] = mj < M ? __ldg(s_x + mj) : 0.0f;
                    rsc[cc] = mj < M ? __ldg(rowsum + mj) : 0;
                }
            }
            if (!warp_wait_sleep(d_full(b), (tl / L::kAccBufs) & 1, lane)) break;
            tc_fence_after();
#pragma unroll
            for (int cc = 0; cc < kChunks; ++cc) {
                const int mb = m0 + cc * 32;
                const int jmax = M - mb;  // tokens of this chunk inside [0, M)
                uint32_t v[32];
                tmem_ld32(lane_addr + (uint32_t)(b * L::kDStride + half * kHalf + cc * 32), v);
                // the lane's own tokens of the transposed layout (quads), fetched
                // while the accumulator load is in flight
                float sxk[8];
                int rsk[8];
                if (quads) {
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int mk = mb + 4 * k + r;
                        sxk[k] = mk < M ? __ldg(s_x + mk) : 0.0f;
                        rsk[k] = mk < M ? __ldg(rowsum + mk) : 0;
                    }
                }
                tmem_ld_wait();
                if (cc == kChunks - 1) {  // accumulator fully read: hand it back to the MMA warp
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(d_empty(b));
                }
                if (quads) {
                    float *yq = y + (int64_t)(mb + r) * N + nq;
                    const bool fin = nq < N;
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        // lane 4g + r holds feature 4g + r of tokens 4k .. 4k + 3;
                        // transpose the raw accumulators inside the quad
                        uint32_t a0 = v[4 * k], a1 = v[4 * k + 1], a2 = v[4 * k + 2], a3 = v[4 * k + 3];
                        // distance 1: swap the odd/even off-diagonal elements of lane pairs
                        const bool o1 = r & 1;
                        const uint32_t x1 = __shfl_xor_sync(0xffffffffu, o1 ? a0 : a1, 1);
                        const uint32_t y1 = __shfl_xor_sync(0xffffffffu, o1 ? a2 : a3, 1);
                        if (o1) { a0 = x1; a2 = y1; } else { a1 = x1; a3 = y1; }
                        // distance 2: swap the off-diagonal 2 x 2 blocks of lane pairs
                        const bool o2 = r & 2;
                        const uint32_t x2 = __shfl_xor_sync(0xffffffffu, o2 ? a0 : a2, 2);
                        const uint32_t y2 = __shfl_xor_sync(0xffffffffu, o2 ? a1 : a3, 2);
                        if (o2) { a0 = x2; a1 = y2; } else { a2 = x2; a3 = y2; }
                        // now token 4k + r of features 4g + i: y = fp32(acc - rowsum) * (gamma * s_x)
                        const uint32_t ai[4] = {a0, a1, a2, a3};
                        float yv[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            yv[i] = __fmul_rn(__int2float_rn((int)ai[i] - rsk[k]), __fmul_rn(g4[i], sxk[k]));
                            if (EPI) yv[i] = __fadd_rn(yv[i], b4[i]);
                        }
                        if (fin && 4 * k + r < jmax)
                            __stcs(reinterpret_cast<float4 *>(yq + (int64_t)(4 * k) * N),
                                   make_float4(yv[0], yv[1], yv[2], yv[3]));
                    }
                } else if (!acc_out) {
                    float *yp = y + (int64_t)mb * N + n;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {  // every lane takes part in the shuffles
                        const float sxm = __shfl_sync(0xffffffffu, sxc[cc], j);
                        const int rsm = __shfl_sync(0xffffffffu, rsc[cc], j);
                        const float yv = __fmul_rn(__int2float_rn((int)v[j] - rsm), __fmul_rn(gn, sxm));
                        if (j < jmax && n < N) __stcs(yp + (int64_t)j * N, EPI ? __fadd_rn(yv, bn) : yv);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float sxm = __shfl_sync(0xffffffffu, sxc[cc], j);
                        const int rsm = __shfl_sync(0xffffffffu, rsc[cc], j);
                        const int a = (int)v[j] - rsm;
                        if (j < jmax && n < N) {
                            const float yv = __fmul_rn(__int2float_rn(a), __fmul_rn(gn, sxm));
                            __stcs(y + (int64_t)(mb + j) * N + n, EPI ? __fadd_rn(yv, bn) : yv);
                            __stcs(acc_out + (int64_t)(mb + j) * N + n, EPI ? (a + abn) >> ep.shift : a);
                        }
                    }
                }
            }
        }
    }
    if (ready || w_early) pdl_wait();  // no-op for roles that already waited
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, L::kTmemCols);
    }
}

}  // namespace tq
