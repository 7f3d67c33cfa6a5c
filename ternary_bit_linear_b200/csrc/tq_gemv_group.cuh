// tq_gemv_group.cuh -- grouped small-M (decode) ternary GEMV: G independent
// layers of one shape, y_g = (x_q,g . q_g) * gamma_g * s_x,g, in one launch.
//
// The per-strip arithmetic is the small-M GEMV's (tq_gemv.cuh; Hetman-2b,
// src/quantization.py, section 7 simulate_hardware_bitnet_gemv: decode the
// packed codes branch-free and accumulate in int32, then one fp32 rescale).
// What changes is how the bytes move: a 4096 x 4096 layer is 4 MiB, less HBM
// time than one launch takes, so G layers share one persistent launch that
// streams all of their packed weights back to back.
//
//   * Work unit: a strip of 16 consecutive weight rows of one problem (16 x
//     K/4 contiguous bytes).  The G * ceil(N/16) strips are split into
//     contiguous runs, one per CTA (one CTA per SM).
//   * Warp 8 (lane 0) is the producer: one 1-D bulk copy (TMA engine) brings
//     each strip (and, with per-row gamma, the strip's 16 gammas) into a ring
//     of `stages` shared-memory slots; the copies of the first slots are
//     issued before the wait for the previous kernel when the weights are
//     static.  The same
//     thread copies each problem's x_q rows (written by the activation pass in
//     the GEMV's transposed, chunk-swizzled layout) into one of two x buffers.
//   * Warps 0-7 form teams of `ksplit` warps; team q takes strips q, q + T,
//     ... of the run; warp j of a team takes the strip's 64-byte column steps
//     j, j + ksplit, ...; the team's partial sums meet in shared memory
//     (double-buffered by strip) and its first warp finishes the outputs.
//   * Synchronisation: full/empty mbarriers per ring slot; xfull/xempty per x
//     buffer (every consumer warp passes every problem of the run in order,
//     so a buffer is refilled only after all warps are done with it).  All
//     waits are bounded; a wait that gives up records TQ_ERR_TIMEOUT, and the
//     CTA skips the rest of its work but keeps the barrier protocol, and the
//     producer lets its copies land before it exits.
#pragma once

#include "tq_common.cuh"
#include "tq_gemv.cuh"

namespace tq {

constexpr int kGroupMax = 64;  // problems per launch
constexpr int kGrpConsumerWarps = 8;
constexpr int kGrpThreads = (kGrpConsumerWarps + 1) * 32;
constexpr int kGrpStagesMax = 8;
constexpr int kGammaSlot = 64;  // bytes after a slot's 16 rows: the strip's per-row gammas

// Per-problem pointers (device), read by dynamic index from parameter space.
struct GroupTable {
    const uint8_t *packed[kGroupMax];
    const float *gamma[kGroupMax];
};

// Host-computed shape and shared-memory plan of one launch.
struct GroupPlan {
    int M, K, KB;           // tokens, contraction length, packed bytes per row
    int64_t N;              // rows per problem
    int64_t spp;            // strips per problem
    int64_t nstrips;        // G * spp
    int x_shared;           // one x_q batch serves every problem
    int per_row;            // gamma per row (else one per problem)
    int weights_static;     // weight copies may start before the wait
    int enc;                // packed-code layout (kEnc*)
    int ksplit;             // warps per strip (1, 2, 4, 8)
    int stages, xbufs;      // ring slots, x buffers (1 or 2)
    int RS, XS;             // shared-memory row strides: strip rows, x_q rows
    int off_x, off_red, off_bar;  // byte offsets of the x buffers, partial sums, barriers
    int smem;               // dynamic shared memory bytes
};

__host__ __device__ inline int grp_red_bytes(int NB) { return 2 * kGrpConsumerWarps * 4 * NB * 32 * 4; }

// Shared-memory plan; returns false if even one x buffer and two slots do not fit.
inline bool grp_plan(GroupPlan &p, int NB, int budget) {
    p.KB = p.K / 4;
    p.RS = p.KB;
    p.XS = gemv_x_stride(p.K);
    const int stage = 16 * p.RS + kGammaSlot, xbytes = p.M * p.XS, red = grp_red_bytes(NB);
    const int bars = (2 * kGrpStagesMax + 4) * 8 + 16;
    for (int xb = 2; xb >= 1; --xb) {
        const int avail = budget - xb * xbytes - red - bars;
        int st = avail / stage;
        if (st > kGrpStagesMax) st = kGrpStagesMax;
        if (st >= (xb == 2 ? 3 : 2)) {
            p.stages = st;
            p.xbufs = xb;
            p.off_x = st * stage;
            p.off_red = p.off_x + xb * xbytes;
            p.off_bar = p.off_red + red;
            p.smem = p.off_bar + bars;
            // warps per strip: keep about half of the slots in flight
            const int nsteps = (p.KB + 63) / 64;
            int teams = st / 2 < 1 ? 1 : st / 2;
            if (teams > kGrpConsumerWarps) teams = kGrpConsumerWarps;
            int ks = (kGrpConsumerWarps + teams - 1) / teams;
            int k2 = 1;
            while (k2 < ks) k2 <<= 1;  // a power of two dividing the consumer warps
            if (k2 > kGrpConsumerWarps) k2 = kGrpConsumerWarps;
            while (k2 > 1 && k2 > nsteps) k2 >>= 1;
            p.ksplit = k2;
            // slots: a multiple of the team count (each slot's strips stay with one team)
            const int T = kGrpConsumerWarps / k2;
            st = st / T * T;
            if (st < T) return false;
            p.stages = st;
            p.off_x = st * stage;
            p.off_red = p.off_x + xb * xbytes;
            p.off_bar = p.off_red + red;
            p.smem = p.off_bar + bars;
            return true;
        }
    }
    return false;
}

// Partial sums of one warp over the column steps j0, j0 + ks, ... of a strip
// in shared memory (rows at stride RS; x_q chunks transposed and swizzled).
//
// Codes enter the MMA in place: field j of a packed word is kept where it is,
// masked by 0x03030303 << 2j, so byte b holds c * 4^j for the code c of
// element 4b + j of its 4-code group -- one logic op per 16 codes and field
// instead of a shift and a mask.  Each field has its own accumulator d[j]
// (its sums are exact multiples of 4^j), and the caller combines them as
// d[0] + d[1]/4 + d[2]/16 + d[3]/64, exact shifts.  One MMA pairs words 2pr
// and 2pr + 1 of a row (K = 32: k < 16 from the first, k >= 16 from the
// second) with word j of the matching transposed x_q chunks.  The next step's
// weight words and the current step's x chunks are loaded before the
// current step's MMAs, so the loads' latency overlaps the arithmetic.
template <int NB, bool CONV, bool FULL>
__device__ __forceinline__ void strip_mma_fields(int (&d)[4][NB][4], uint32_t w_s, int RS, uint32_t x_s, int XS,
                                                 int M, int KB, int j0, int ks, int lane, int enc) {
    const int g = lane >> 2, t = lane & 3;
    // FULL: K % 256 == 0, every 64-byte step lies inside the row.  Otherwise the
    // last step is partial: past the row the weight words are padding and the
    // x chunks are taken as 0, so they add nothing.
    const int nsteps = (KB + 63) >> 6;
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) d[j][nb][0] = d[j][nb][1] = d[j][nb][2] = d[j][nb][3] = 0;
    if (j0 >= nsteps) return;
    // per-lane bases: weight rows g and g + 8 at column 16 t; token rows g + 8 nb
    // (rows past M read row M - 1: those outputs are never stored) at column
    // 64 t; the x chunk swizzle gives the lane's four chunk offsets
    const uint32_t ra = w_s + (uint32_t)(g * RS + t * 16), rb = ra + (uint32_t)(8 * RS);
    uint32_t xr[NB];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
        const int m = g + 8 * nb < M ? g + 8 * nb : M - 1;
        xr[nb] = x_s + (uint32_t)(m * XS + 64 * t);
    }
    const uint32_t xsw = (uint32_t)(t & 2) << 4;
    const uint32_t c0 = 0u ^ xsw, c1 = 16u ^ xsw, c2 = 32u ^ xsw, c3 = 48u ^ xsw;
    uint4 wa = lds128(ra + (uint32_t)(j0 * 64)), wb = lds128(rb + (uint32_t)(j0 * 64));
    for (int step = j0; step < nsteps; step += ks) {
        const uint32_t xo = (uint32_t)step * 256u;
        const bool in_row = FULL || step * 64 + t * 16 < KB;
        uint4 xt[NB][4];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
            xt[nb][0] = lds128(xr[nb] + xo + c0);
            xt[nb][1] = lds128(xr[nb] + xo + c1);
            xt[nb][2] = lds128(xr[nb] + xo + c2);
            xt[nb][3] = lds128(xr[nb] + xo + c3);
            if (!FULL && !in_row)
#pragma unroll
                for (int i = 0; i < 4; ++i) xt[nb][i] = make_uint4(0u, 0u, 0u, 0u);
        }
        uint4 na = wa, nbw = wb;
        if (step + ks < nsteps) {
            na = lds128(ra + (uint32_t)((step + ks) * 64));
            nbw = lds128(rb + (uint32_t)((step + ks) * 64));
        }
        uint32_t a4[4] = {wa.x, wa.y, wa.z, wa.w};
        uint32_t b4[4] = {wb.x, wb.y, wb.z, wb.w};
        if (CONV) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                a4[i] = codes_to_foundry(a4[i], enc);
                b4[i] = codes_to_foundry(b4[i], enc);
            }
        }
#pragma unroll
        for (int pr = 0; pr < 2; ++pr)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t msk = 0x03030303u << (2 * j);
                const uint32_t a0 = a4[2 * pr] & msk, a1 = b4[2 * pr] & msk;
                const uint32_t a2 = a4[2 * pr + 1] & msk, a3 = b4[2 * pr + 1] & msk;
#pragma unroll
                for (int nb = 0; nb < NB; ++nb) {
                    const uint4 &u = xt[nb][2 * pr], &v = xt[nb][2 * pr + 1];
                    const uint32_t x0 = j == 0 ? u.x : j == 1 ? u.y : j == 2 ? u.z : u.w;
                    const uint32_t x1 = j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w;
                    mma_16x8x32_u8s8_pure(d[j][nb], a0, a1, a2, a3, x0, x1);
                }
            }
        wa = na;
        wb = nbw;
    }
}

// NB: token blocks of 8 (M <= 8 NB).  ENC: packed-code layout.
// FULL: K % 256 == 0 (no partial column step).
template <int NB, int ENC, bool FULL>
__global__ void __launch_bounds__(kGrpThreads, 1)
    tq_gemv_group_kernel(const __grid_constant__ GroupTable tab, const __grid_constant__ GroupPlan pl,
                         const int8_t *__restrict__ xq, const float *__restrict__ s_x,
                         const int32_t *__restrict__ rowsum, float *__restrict__ y) {
    constexpr bool CONV = ENC != kEncFoundry;
    extern __shared__ __align__(128) uint8_t dsm[];
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t sbase = smem_u32(dsm);
    const int S = pl.stages, M = pl.M, KB = pl.KB, RS = pl.RS, XS = pl.XS;
    const int64_t spp = pl.spp;
    const uint32_t bar0 = sbase + (uint32_t)pl.off_bar;
    auto full = [&](int s) { return bar0 + 8u * (uint32_t)s; };
    auto empty = [&](int s) { return bar0 + 8u * (uint32_t)(kGrpStagesMax + s); };
    auto xfull = [&](int b) { return bar0 + 8u * (uint32_t)(2 * kGrpStagesMax + b); };
    auto xempty = [&](int b) { return bar0 + 8u * (uint32_t)(2 * kGrpStagesMax + 2 + b); };
    const uint32_t stage_bytes = 16u * (uint32_t)RS + kGammaSlot;
    auto stage_addr = [&](int s) { return sbase + (uint32_t)s * stage_bytes; };
    auto xbuf_addr = [&](int b) { return sbase + (uint32_t)pl.off_x + (uint32_t)(b * M * XS); };

    // contiguous run of strips of this CTA
    const int64_t s0 = (int64_t)blockIdx.x * pl.nstrips / gridDim.x;
    const int64_t s1 = (int64_t)(blockIdx.x + 1) * pl.nstrips / gridDim.x;
    const int nloc = (int)(s1 - s0);
    const int64_t p_first = s0 / spp;
    const int np = nloc > 0 ? (int)((s1 - 1) / spp - p_first + 1) : 0;
    // teams of ks warps; the host makes S a multiple of T, so strips i and i + S
    // (the same slot, consecutive phases) belong to the same team, which
    // takes its strips in order: no wait ever targets a phase two ahead
    const int ks = pl.ksplit, T = kGrpConsumerWarps / ks;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGrpStagesMax; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), (uint32_t)ks);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(xfull(b), 1);
            mbar_init(xempty(b), kGrpConsumerWarps);
        }
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    pdl_trigger();

    volatile int *abrt = &abort_flag;
    auto wait_spin = [&](uint32_t bar, uint32_t par) {
        if (*abrt) return false;
        if (mbar_wait(bar, par)) return true;
        *abrt = 1;
        return false;
    };

    if (warp == kGrpConsumerWarps) {
        // ---------------- producer ----------------
        if (lane == 0 && nloc > 0) {
            auto issue_x = [&](int pi) {
                const int bb = pl.xbufs == 1 ? 0 : (pi & 1);
                const int prev = pi - pl.xbufs;  // the problem buffer bb held before
                if (prev >= 0 && !wait_spin(xempty(bb), (uint32_t)((prev / pl.xbufs) & 1))) return false;
                const int8_t *src = xq + (pl.x_shared ? 0 : p_first + pi) * (int64_t)M * pl.K;
                mbar_arrive_expect_tx(xfull(bb), (uint32_t)(M * pl.K));
                for (int m = 0; m < M; ++m)
                    bulk_g2s(xbuf_addr(bb) + (uint32_t)(m * XS), src + (int64_t)m * pl.K, (uint32_t)pl.K, xfull(bb));
                return true;
            };
            // cursor of the next strip to issue: index, slot, use of the slot, problem, strip in problem
            int wi = 0, ws = 0, wk = 0;
            int64_t wp = p_first, wls = s0 - p_first * spp;
            auto issue_w = [&]() {
                if (wi >= S && !wait_spin(empty(ws), (uint32_t)((wk - 1) & 1))) return false;
                const int64_t r0 = wls * 16;
                const int rows = (int)(pl.N - r0 < 16 ? pl.N - r0 : 16);
                const bool gslot = pl.per_row && rows == 16;  // 64 gamma bytes, 16-byte aligned
                mbar_arrive_expect_tx(full(ws), (uint32_t)(rows * KB) + (gslot ? kGammaSlot : 0u));
                bulk_g2s(stage_addr(ws), tab.packed[wp] + r0 * KB, (uint32_t)(rows * KB), full(ws));
                if (gslot) bulk_g2s(stage_addr(ws) + 16u * (uint32_t)RS, tab.gamma[wp] + r0, kGammaSlot, full(ws));
                ++wi;
                if (++ws == S) {
                    ws = 0;
                    ++wk;
                }
                if (++wls == spp) {
                    wls = 0;
                    ++wp;
                }
                return true;
            };
            const int pre = pl.weights_static ? (nloc < S ? nloc : S) : 0;
            while (wi < pre) issue_w();
            pdl_wait();
            int next_x = 0;
            bool ok = true;
            // x for the problems of the strips already issued, then strip by strip
            const int xpre = wi > 0 ? (int)((wls == 0 ? wp - 1 : wp) - p_first) : -1;
            while (ok && next_x <= xpre) ok = issue_x(next_x++);
            while (ok && wi < nloc) {
                const int pi = (int)(wp - p_first);
                while (ok && next_x <= pi) ok = issue_x(next_x++);
                if (ok) ok = issue_w();
            }
            // Every copy lands before this thread exits.  In normal operation
            // the consumers have waited for (or will wait for) each one; after
            // a timeout they may have skipped theirs, and then only the last
            // copy issued into each slot and buffer can still be in flight (no
            // copy is issued once a wait has given up).
            for (int s = 0; s < S && s < wi; ++s) {
                const int last = s + ((wi - 1 - s) / S) * S;
                mbar_wait_sleep(full(s), (uint32_t)((last / S) & 1));
            }
            for (int b = 0; b < pl.xbufs && b < next_x; ++b) {
                const int last = b + ((next_x - 1 - b) / pl.xbufs) * pl.xbufs;
                mbar_wait_sleep(xfull(b), (uint32_t)((last / pl.xbufs) & 1));
            }
        }
        return;
    }

    // ---------------- consumers ----------------
    pdl_wait();  // s_x, rowsum (and y) belong to work before this kernel
    const int team = warp / ks, kw = warp % ks;
    int *red = reinterpret_cast<int *>(dsm + pl.off_red);  // [2][consumer warps][4 NB][32]
    int par = 0;
    const int g = lane >> 2, tt = lane & 3;
    // cursor of this team's next strip: index, slot, use of the slot, problem, strip in problem
    int i = team, cs = team % S, ck = team / S;
    int64_t cp = (s0 + team) / spp, cls = s0 + team - cp * spp;
    for (int pi = 0; pi < np; ++pi) {
        const int bb = pl.xbufs == 1 ? 0 : (pi & 1);
        const int64_t p = p_first + pi;
        const bool xok = !*abrt && warp_wait(xfull(bb), (uint32_t)((pi / pl.xbufs) & 1), lane);
        if (!xok && lane == 0) *abrt = 1;
        const uint32_t x_s = xbuf_addr(bb);
        const float *sx_p = s_x + (pl.x_shared ? 0 : p) * (int64_t)M;
        const int32_t *rs_p = rowsum + (pl.x_shared ? 0 : p) * (int64_t)M;
        const float *gam = tab.gamma[p];
        const float g_tensor = pl.per_row ? 0.0f : __ldg(gam);
        // the finishing lanes' token scales and offsets: tokens 8 nb + 2 tt + e
        float sxv[NB][2];
        int rsv[NB][2];
        if (kw == 0)
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int m = 8 * nb + 2 * tt + e;
                    sxv[nb][e] = m < M ? __ldcg(sx_p + m) : 0.0f;
                    rsv[nb][e] = m < M ? __ldcg(rs_p + m) : 0;
                }
        for (; i < nloc && cp == p;) {
            const int s = cs;
            const int64_t ls = cls;
            const bool ok = !*abrt && warp_wait(full(s), (uint32_t)(ck & 1), lane);
            if (!ok && lane == 0) *abrt = 1;
            // gamma of rows g and g + 8: from the slot (full strips, per row), else from memory
            float gv[2] = {g_tensor, g_tensor};
            if (kw == 0 && pl.per_row) {
                if (ls * 16 + 16 <= pl.N) {
                    const float *gs = reinterpret_cast<const float *>(dsm + (size_t)s * stage_bytes + 16 * RS);
                    gv[0] = gs[g];
                    gv[1] = gs[g + 8];
                } else {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int64_t n = ls * 16 + g + 8 * h;
                        gv[h] = n < pl.N ? __ldg(gam + n) : 0.0f;
                    }
                }
            }
            int d[4][NB][4];
            if (ok && !*abrt)
                strip_mma_fields<NB, CONV, FULL>(d, stage_addr(s), RS, x_s, XS, M, KB, kw, ks, lane, ENC);
            else
#pragma unroll
                for (int j = 0; j < 4; ++j)
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb) d[j][nb][0] = d[j][nb][1] = d[j][nb][2] = d[j][nb][3] = 0;
            __syncwarp();
            if (lane == 0) mbar_arrive(empty(s));  // the slot's words are in registers (consumed)
            int acc[NB][4];
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                for (int c = 0; c < 4; ++c)  // exact: d[j] is a multiple of 4^j
                    acc[nb][c] = d[0][nb][c] + (d[1][nb][c] >> 2) + (d[2][nb][c] >> 4) + (d[3][nb][c] >> 6);
            if (ks > 1) {
                int *rb = red + par * (kGrpConsumerWarps * 4 * NB * 32);
                if (kw != 0) {
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                        for (int c = 0; c < 4; ++c) rb[(warp * 4 * NB + nb * 4 + c) * 32 + lane] = acc[nb][c];
                }
                asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "r"(ks * 32) : "memory");
                if (kw == 0) {
                    for (int w2 = warp + 1; w2 < warp + ks; ++w2)
#pragma unroll
                        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                            for (int c = 0; c < 4; ++c) acc[nb][c] += rb[(w2 * 4 * NB + nb * 4 + c) * 32 + lane];
                }
                par ^= 1;
            }
            if (kw == 0 && !*abrt) {
                // fragment c of lane (g, tt): row g (+8 for c >= 2), token 8 nb + 2 tt + (c & 1)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int64_t n = ls * 16 + g + ((c & 2) ? 8 : 0);
                    if (n >= pl.N) continue;
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb) {
                        const int m = 8 * nb + 2 * tt + (c & 1);
                        if (m < M) {
                            const int a = acc[nb][c] - rsv[nb][c & 1];
                            y[(p * M + m) * pl.N + n] =
                                __fmul_rn(__int2float_rn(a), __fmul_rn(gv[c >> 1], sxv[nb][c & 1]));
                        }
                    }
                }
            }
            // advance the cursor by T strips
            i += T;
            cls += T;
            while (cls >= spp) {
                cls -= spp;
                ++cp;
            }
            cs += T;
            if (cs >= S) {
                cs -= S;
                ++ck;
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(xempty(bb));
    }
}

}  // namespace tq
