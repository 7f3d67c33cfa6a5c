// tq_common.cuh -- device helpers shared by the libtq kernels (sm_100a only).
//
// Everything here is written for this library: PTX wrappers for mbarriers,
// bulk/tensor copies and tcgen05, the bounded-wait policy, and the
// double-double arithmetic that makes gamma the correctly rounded mean.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ != 1000)
#error "libtq is written for sm_100a only"
#endif

namespace tq {

// ---------------------------------------------------------------------------
// Per-device status word.  Kernels OR error bits into it; the host reads and
// clears it in tq_get_device_status().
// ---------------------------------------------------------------------------
static __device__ unsigned int g_status;
constexpr unsigned kStatusTimeout = 1u;

// A wait gives up after this much wall time (ns, %globaltimer).
constexpr unsigned long long kWaitLimitNs = 1000000000ull;
// Longest single sleep of a waiting thread (ns); the phase completing wakes it earlier.
constexpr uint32_t kWaitHintNs = 1000000u;

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void flag_timeout() { atomicOr(&g_status, kStatusTimeout); }

// ---------------------------------------------------------------------------
// Programmatic dependent launch.  Every kernel of the library waits (pdl_wait)
// before it reads anything an earlier kernel on the stream may have written,
// and lets the next kernel be scheduled early (pdl_trigger).  Without the
// launch attribute both are no-ops.
// ---------------------------------------------------------------------------
// Launch modes of the contraction kernels (set from TQ_FLAG_WEIGHTS_STATIC and
// TQ_FLAG_INPUTS_READY): weights may be read before the wait; no wait at all
// before reading, only before exiting.
constexpr int kModeWeightsStatic = 1;
constexpr int kModeInputsReady = 2;
constexpr int kModeEncShift = 2;  // bits 2-3: packed-code layout (kEnc*, below)

// Extra epilogue of a contraction (tq_ternary_gemm_ex): y gets + bias[n]
// (Hetman-2b BitLinear's bias), the int32 accumulator output (acc + acc_bias[n])
// >> shift (BitRASP's integer epilogue).  NULL pointers add nothing.
struct Epilogue {
    const float *bias;
    const int32_t *acc_bias;
    int shift;
};

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Shared-memory addresses and mbarriers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// try_wait with a suspend-time hint: a thread whose phase is not complete
// sleeps until it completes (or the hint runs out) instead of spinning, so
// waiting warps leave the issue slots to the warps doing work.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(kWaitHintNs)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity.  Returns false (and sets
// the timeout bit) if it did not complete within kWaitLimitNs.  The spinning
// form is for waits on a kernel's critical path; the sleeping form for warps
// that wait long while others on the SM do the work.
template <bool SLEEP>
__device__ __forceinline__ bool mbar_wait_t(uint32_t bar, uint32_t parity,
                                            unsigned long long limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    for (;;) {
        for (int i = 0; i < (SLEEP ? 8 : 64); ++i)
            if (SLEEP ? mbar_try_wait_sleep(bar, parity) : mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > limit_ns) {
            flag_timeout();
            return false;
        }
    }
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    return mbar_wait_t<false>(bar, parity);
}
__device__ __forceinline__ bool mbar_wait_sleep(uint32_t bar, uint32_t parity) {
    return mbar_wait_t<true>(bar, parity);
}

// Warp-uniform bounded wait: lane 0 polls, every lane gets the same answer,
// and the warp leaves converged.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, int lane) {
    int ok = 0;
    if (lane == 0) ok = mbar_wait(bar, parity) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}
__device__ __forceinline__ bool warp_wait_sleep(uint32_t bar, uint32_t parity, int lane) {
    int ok = 0;
    if (lane == 0) ok = mbar_wait_sleep(bar, parity) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// Self-test of the bounded wait: one warp waits (as the kernels' waits do, with
// the given limit) on an mbarrier that nothing ever completes, gives up, and
// records the timeout in the status word.  Touches no memory but its own
// shared mbarrier; exits normally.
__global__ void __launch_bounds__(32) tq_selftest_wait_kernel(unsigned long long limit_ns, int sleeping) {
    __shared__ uint64_t bar;
    const uint32_t b = smem_u32(&bar);
    if (threadIdx.x == 0) mbar_init(b, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    __syncwarp();
    int ok = 1;
    if (threadIdx.x == 0) ok = (sleeping ? mbar_wait_t<true>(b, 0, limit_ns) : mbar_wait_t<false>(b, 0, limit_ns)) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    (void)ok;
}

// Generic-proxy writes to shared memory become visible to the async proxy
// (TMA, tensor core) after this fence.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Bulk copies (TMA engine)
// ---------------------------------------------------------------------------
// 1-D bulk copy global -> shared, completion counted on `bar` in bytes.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes,
                                         uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// 2-D tiled tensor copy global -> shared (no multicast).
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void *tmap, int32_t c0, int32_t c1,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(tmap), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const void *tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05 (5th-generation tensor core, tensor memory)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T, int8 kind, one CTA; A is M lanes x
// (K/4) columns of four 8-bit values each, starting at column a_tmem.
__device__ __forceinline__ void mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns from registers: thread t of the
// warp writes lane (base lane + t), columns col..col+31.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Arrive once on `bar` when all previously issued tcgen05.mma of this thread
// have completed.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns; thread t of the warp receives
// lane (base lane + t), columns col..col+31.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major operand stored in the
// 128-byte-swizzle canonical layout: rows of 128 bytes, 8-row groups 1024 B
// apart, 16-byte chunk index XOR (row % 8).  Base must be 1024-byte aligned
// (the start address may be advanced by k*32 bytes inside the row).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);   // start address, bits 0-13
    d |= (uint64_t)(16u >> 4) << 16;            // leading byte offset (unused here)
    d |= (uint64_t)(1024u >> 4) << 32;          // stride byte offset: 8 rows x 128 B
    d |= (uint64_t)1u << 46;                    // descriptor version for sm_100
    d |= (uint64_t)2u << 61;                    // layout: 128-byte swizzle
    return d;
}

// Instruction descriptor, kind::i8: D s32, A u8, B s8, both K-major, M x N.
__host__ __device__ constexpr uint32_t idesc_i8_u8s8(int M, int N) {
    return (2u << 4)                        // D format: s32
           | (0u << 7)                      // A: unsigned 8-bit
           | (1u << 10)                     // B: signed 8-bit
           | ((uint32_t)(N >> 3) << 17)     // N / 8
           | ((uint32_t)(M >> 4) << 24);    // M / 16
}

// ---------------------------------------------------------------------------
// Legacy warp-level MMA used by the small-M GEMV (HBM-bound; the tensor rate
// is irrelevant there): D[16x8] += A[16x32] (u8) * B[32x8] (s8).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_16x8x32_u8s8(int (&d)[4], uint32_t a0, uint32_t a1,
                                                  uint32_t a2, uint32_t a3, uint32_t b0,
                                                  uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 4x4 byte transpose: out word j = (in0.byte j, in1.byte j, in2.byte j, in3.byte j).
__device__ __forceinline__ uint4 transpose_bytes4x4(uint4 q) {
    const uint32_t t0 = __byte_perm(q.x, q.y, 0x5140), t1 = __byte_perm(q.x, q.y, 0x7362);
    const uint32_t t2 = __byte_perm(q.z, q.w, 0x5140), t3 = __byte_perm(q.z, q.w, 0x7362);
    return make_uint4(__byte_perm(t0, t2, 0x5410), __byte_perm(t0, t2, 0x7632),
                      __byte_perm(t1, t3, 0x5410), __byte_perm(t1, t3, 0x7632));
}

// Position of 16-byte chunk c inside an x_q row as the small-M GEMV keeps it
// in shared memory: chunks 8..15 of every 16 swap in pairs, so the chunk reads
// of a quarter warp (two rows, four column offsets) hit distinct banks.
__host__ __device__ __forceinline__ int gemv_chunk_pos(int c) { return c ^ (((c >> 3) & 1) << 1); }

// The same MMA as a plain (non-volatile) asm: a pure function of its register
// operands, so the compiler may schedule it among independent work (used where
// the operands come from registers only).
__device__ __forceinline__ void mma_16x8x32_u8s8_pure(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                                       uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------------------
// Double-double accumulation of non-negative terms, and the correctly
// rounded fp32 mean derived from it.
// ---------------------------------------------------------------------------
struct DD {
    double hi, lo;
};

// s + e == a + b exactly (Knuth's TwoSum).
__device__ __forceinline__ void two_sum(double a, double b, double &s, double &e) {
    s = __dadd_rn(a, b);
    const double bb = __dsub_rn(s, a);
    e = __dadd_rn(__dsub_rn(a, __dsub_rn(s, bb)), __dsub_rn(b, bb));
}

// Running sum (hi) plus the exact sum of the rounding errors so far (lo,
// itself summed in plain fp64 -- its own error is negligible at this scale).
__device__ __forceinline__ void dd_acc(DD &x, double v) {
    double s, e;
    two_sum(x.hi, v, s, e);
    x.hi = s;
    x.lo = __dadd_rn(x.lo, e);
}

__device__ __forceinline__ DD dd_add(DD x, DD y) {
    double s, e;
    two_sum(x.hi, y.hi, s, e);
    e = __dadd_rn(e, __dadd_rn(x.lo, y.lo));
    DD r;
    r.hi = __dadd_rn(s, e);
    r.lo = __dsub_rn(e, __dsub_rn(r.hi, s));
    return r;
}

__device__ __forceinline__ DD dd_shfl_xor(DD x, int off) {
    DD r;
    r.hi = __shfl_xor_sync(0xffffffffu, x.hi, off);
    r.lo = __shfl_xor_sync(0xffffffffu, x.lo, off);
    return r;
}

__device__ __forceinline__ DD dd_warp_sum(DD x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x = dd_add(x, dd_shfl_xor(x, off));
    return x;
}

// fp32 nearest (ties to even) to (hi + lo) / n for hi + lo >= 0, assuming the
// double-double holds the sum to ~2^-100 relative.
__device__ __forceinline__ float dd_mean_to_f32(DD s, double n) {
    if (!(s.hi > 0.0)) return 0.0f;
    const double q1 = __ddiv_rn(s.hi, n);
    const double rem = __fma_rn(-q1, n, s.hi);  // exact remainder of the division
    const double q2 = __ddiv_rn(__dadd_rn(rem, s.lo), n);
    float f = __double2float_rn(q1);
    const float up = nextafterf(f, __int_as_float(0x7f800000));
    const float dn = nextafterf(f, 0.0f);
    const double mu = 0.5 * ((double)f + (double)up);  // fp32 midpoints are exact in fp64
    const double ml = 0.5 * ((double)f + (double)dn);
    const double du = __dadd_rn(__dsub_rn(q1, mu), q2);  // sign of (value - mu)
    const double dl = __dadd_rn(__dsub_rn(q1, ml), q2);
    const bool odd = (__float_as_uint(f) & 1u) != 0;
    if (du > 0.0 || (du == 0.0 && odd))
        f = up;
    else if (dl < 0.0 || (dl == 0.0 && odd))
        f = dn;
    return f;
}

// Smallest fp32 t with: w >= t  <=>  fp32(w / gamma) rounds (half to even)
// above 0.5, i.e. w / gamma > 0.5 + 2^-25 exactly.  gamma * (0.5 + 2^-25) is
// exact in fp64 (24-bit times 25-bit significand).
__device__ __forceinline__ float code_threshold(float gamma) {
    const double T = (double)gamma * (0.5 + 0x1p-25);
    float t = __double2float_ru(T);
    if ((double)t == T) t = nextafterf(t, __int_as_float(0x7f800000));
    return t;
}

// Code threshold t for one gamma (a weight is +1 iff w >= t, -1 iff w <= -t):
// the round rule (ratio <= 0; code_threshold) or the threshold rule
// w > fp32(ratio * gamma), strict, i.e. t = the next float above it.
__device__ __forceinline__ float pack_threshold(float gamma, float ratio) {
    if (ratio > 0.0f) return nextafterf(__fmul_rn(ratio, gamma), __int_as_float(0x7f800000));
    return code_threshold(gamma);
}

// 2-bit code (-1 -> 0b00, 0 -> 0b01, +1 -> 0b10) of one weight.
__device__ __forceinline__ uint32_t ternary_field(float w, float t) {
    return 1u + (w >= t ? 1u : 0u) - (w <= -t ? 1u : 0u);
}

// Packed-code layouts.  Foundry (docs/quantization.md, "Ternary Format /
// Encoding"): -1 = 0b00, 0 = 0b01, +1 = 0b10, the field being q + 1 -- the
// form the kernels compute with.  Hetman-2b (src/quantization.py, section 3,
// PackedTernaryStorage) "Format 0": 0 = 0b00, +1 = 0b01, -1 = 0b11 (0b10 reads
// as 0); "Format 1": 0 = 0b00, +1 = 0b01, -1 = 0b10 (0b11 reads as 0).
constexpr int kEncFoundry = 0, kEncFormat0 = 1, kEncFormat1 = 2;

// The 16 fields of a word in layout `enc`, rewritten in Foundry's layout.
// With p, n the low and high bit of a field, Foundry's field is
// (p & ~n) << 1 | (Format 0: ~p, Format 1: ~(p ^ n)) -- the page's decodes
// p - 2(p & n) and p - n, plus one.  A warp-uniform branch for the default.
__device__ __forceinline__ uint32_t codes_to_foundry(uint32_t w, int enc) {
    if (enc == kEncFoundry) return w;
    const uint32_t M = 0x55555555u;
    const uint32_t p = w & M, n = (w >> 1) & M;
    const uint32_t lo = enc == kEncFormat0 ? (~p & M) : (~(p ^ n) & M);
    return ((p & ~n) << 1) | lo;
}

// Inverse for the packer (its Foundry-layout fields are never 0b11): with
// f0, f1 the low and high bit, a -1 (both clear) gets the high bit, and the
// low bit is ~f0 (Format 0) or f1 (Format 1).
__device__ __forceinline__ uint32_t codes_from_foundry(uint32_t f, int enc) {
    if (enc == kEncFoundry) return f;
    const uint32_t M = 0x55555555u;
    const uint32_t f0 = f & M, f1 = (f >> 1) & M;
    const uint32_t lo = enc == kEncFormat0 ? (~f0 & M) : f1;
    return lo | ((~f0 & ~f1 & M) << 1);
}

}  // namespace tq
