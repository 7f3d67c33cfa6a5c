// tq_api.cu -- the C ABI of libtq (declared in include/tq.h).
//
// Host side only: argument checks (before anything is enqueued), tensor-map
// encoding for the TMA copies, launch configuration and dispatch.  All
// arithmetic of the method runs in the kernels included below.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "tq.h"
#include "tq_act.cuh"
#include "tq_common.cuh"
#include "tq_gemm.cuh"
#include "tq_gemv.cuh"
#include "tq_gemv_group.cuh"
#include "tq_pack.cuh"
#include "tq_train.cuh"

namespace {

using namespace tq;

constexpr int kMaxDevices = 64;
constexpr int64_t kMaxK = 65536;

inline cudaStream_t cs(tq_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool overlap(const void *a, size_t na, const void *b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

struct DeviceInfo {
    int checked = 0;  // 0 unknown, 1 ok, -1 wrong arch
    int sms = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

// Current device must be compute capability 10.0 (sm_100a code only).
tq_status check_device(int *sms_out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return TQ_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return TQ_ERR_DEVICE;
    DeviceInfo &d = g_dev[dev];
    if (d.checked == 0) {
        std::lock_guard<std::mutex> lk(g_mu);
        if (d.checked == 0) {
            int maj = 0, min = 0, sms = 0;
            if (cudaDeviceGetAttribute(&maj, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
                cudaDeviceGetAttribute(&min, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
                cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
                return TQ_ERR_CUDA;
            d.sms = sms;
            d.checked = (maj == 10 && min == 0) ? 1 : -1;
        }
    }
    if (d.checked < 0) return TQ_ERR_DEVICE;
    if (sms_out) *sms_out = d.sms;
    return TQ_OK;
}

inline tq_status launch_status() {
    return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

// Every kernel is launched with programmatic dependent launch allowed; each
// kernel waits (griddepcontrol.wait) before touching memory an earlier kernel
// may have produced, so the attribute only lets launches overlap.
template <typename... KArgs, typename... Args>
tq_status launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                     cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...) == cudaSuccess
               ? TQ_OK
               : TQ_ERR_CUDA;
}

// Packed-code layout from the flags (kEnc*), or -1 for the reserved value.
inline int flag_encoding(unsigned flags) {
    const int e = (int)((flags & TQ_ENC_MASK) >> 7);
    return e == 3 ? -1 : e;
}

inline tq_status check_k(int64_t K) {
    if (K < 64 || K > kMaxK || (K % 64) != 0) return TQ_ERR_SHAPE;
    return TQ_OK;
}

// ---------------------------------------------------------------------------
// Tensor maps (driver entry point fetched through the runtime, no -lcuda)
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static std::atomic<EncodeTiledFn> fn{nullptr};
    EncodeTiledFn f = fn.load();
    if (!f) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        f = reinterpret_cast<EncodeTiledFn>(p);
        fn.store(f);
    }
    return f;
}

// 2-D uint8 tensor [rows][cols] (row stride = cols bytes), box [box_rows][box_cols].
bool make_tmap_u8(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows, uint32_t box_cols,
                  uint32_t box_rows, CUtensorMapSwizzle swz) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------------------
// Launch helpers
// ---------------------------------------------------------------------------
// Arguments of one contraction call, as the kernels take them.
struct GemmArgs {
    const int8_t *xq;
    const float *s_x;
    const int32_t *rowsum;
    const uint8_t *packed;
    const float *gamma;
    int per_row;
    int64_t M, N, K;
    float *y;
    int32_t *acc;
    int mode;
    Epilogue ep;
};

template <int BT, bool CONV, bool EPI>
tq_status launch_gemm(const GemmArgs &a, int sms, cudaStream_t st) {
    using L = GemmLayout<BT>;
    static std::atomic<int> attr_done[kMaxDevices];
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr_done[dev].load()) {
        if (cudaFuncSetAttribute(tq_gemm_kernel<BT, CONV, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 L::kDynamic) != cudaSuccess)
            return TQ_ERR_CUDA;
        attr_done[dev].store(1);
    }
    // x_q [M][K] in 128-byte-swizzled [BT][128] boxes; packed weights [N][K/4]
    // in plain [128][32] boxes (K % 64 == 0 keeps both row strides 16-byte multiples).
    CUtensorMap tx, tw;
    if (!make_tmap_u8(&tx, a.xq, (uint64_t)a.K, (uint64_t)a.M, kTileK, BT, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_u8(&tw, a.packed, (uint64_t)(a.K / 4), (uint64_t)a.N, kTileK / 4, kTileN,
                      CU_TENSOR_MAP_SWIZZLE_NONE))
        return TQ_ERR_CUDA;
    const int64_t tiles = ((a.M + BT - 1) / BT) * ((a.N + kTileN - 1) / kTileN);
    const unsigned grid = (unsigned)(tiles < sms ? tiles : sms);  // persistent, one CTA per SM
    return launch_pdl(tq_gemm_kernel<BT, CONV, EPI>, dim3(grid), dim3(kGemmThreads), L::kDynamic, st, tx, tw,
                      a.s_x, a.rowsum, a.gamma, a.per_row, (int)a.M, (int)a.N, (int)a.K, a.y, a.acc, a.mode,
                      a.ep);
}

// Grid: one CTA per 16-row strip.  Dynamic shared memory holds x_q only.
template <int NB, int W, int SPW, bool CONV, bool EPI>
tq_status launch_gemv(const GemmArgs &a, cudaStream_t st) {
    static_assert(256 * W * SPW >= kGemvMaxK / 2, "shape covers K");
    static std::atomic<int> attr_done[kMaxDevices];
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr_done[dev].load()) {
        if (cudaFuncSetAttribute(tq_gemv_kernel<NB, W, SPW, CONV, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 gemv_x_bytes(8 * NB, kGemvMaxK)) != cudaSuccess)
            return TQ_ERR_CUDA;
        attr_done[dev].store(1);
    }
    const int64_t grid = (a.N + 15) / 16;
    const size_t smem = (size_t)gemv_x_bytes((int)a.M, (int)a.K);
    return launch_pdl(tq_gemv_kernel<NB, W, SPW, CONV, EPI>, dim3((unsigned)grid), dim3(W * 32), smem, st, a.xq,
                      a.s_x, a.rowsum, a.packed, a.gamma, a.per_row, (int)a.M, a.N, (int)a.K, a.y, a.acc,
                      a.mode, a.ep);
}

// Independent calls: a narrow grid of about 32 CTAs streaming runs of strips
// (at least one strip per group), so that consecutive calls run side by side.
template <int ENC>
tq_status launch_gemv_stream_t(const int8_t *xq, const float *s_x, const int32_t *rowsum,
                               const uint8_t *packed, const float *gamma, int per_row, int64_t M,
                               int64_t N, int64_t K, float *y, int32_t *acc, cudaStream_t st) {
    static std::atomic<int> attr_done[kMaxDevices];
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr_done[dev].load()) {
        if (cudaFuncSetAttribute(tq_gemv_stream_kernel<ENC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 gemv_x_bytes(8, kStreamMaxK)) != cudaSuccess)
            return TQ_ERR_CUDA;
        attr_done[dev].store(1);
    }
    const int64_t nstrips = (N + 15) / 16;
    int64_t per_cta = (nstrips + 31) / 32;
    if (per_cta < kStreamGroups) per_cta = kStreamGroups;
    const int64_t grid = (nstrips + per_cta - 1) / per_cta;
    const size_t smem = (size_t)gemv_x_bytes((int)M, (int)K);
    return launch_pdl(tq_gemv_stream_kernel<ENC>, dim3((unsigned)grid), dim3(kStreamThreads), smem, st, xq,
                      s_x, rowsum, packed, gamma, per_row, (int)M, N, (int)K, y, acc, (int)per_cta);
}

tq_status launch_gemv_stream(const int8_t *xq, const float *s_x, const int32_t *rowsum,
                             const uint8_t *packed, const float *gamma, int per_row, int64_t M,
                             int64_t N, int64_t K, float *y, int32_t *acc, int enc, cudaStream_t st) {
    if (enc == kEncFormat0)
        return launch_gemv_stream_t<kEncFormat0>(xq, s_x, rowsum, packed, gamma, per_row, M, N, K, y, acc, st);
    if (enc == kEncFormat1)
        return launch_gemv_stream_t<kEncFormat1>(xq, s_x, rowsum, packed, gamma, per_row, M, N, K, y, acc, st);
    return launch_gemv_stream_t<kEncFoundry>(xq, s_x, rowsum, packed, gamma, per_row, M, N, K, y, acc, st);
}

// Independent calls (inputs ready) overlap one another: lean CTAs (four
// steps per warp) keep several layers resident.  Otherwise, for K <= 4096,
// the time after the wait is the critical path: twice the warps, two steps
// each.  Larger K keeps the lean shape (16-warp CTAs measured slower).
template <int NB, bool CONV, bool EPI>
tq_status gemv_shape(const GemmArgs &a, cudaStream_t st) {
    const bool lean = (a.mode & kModeInputsReady) != 0;
    if (a.K <= kGemvMaxK / 2)
        return lean ? launch_gemv<NB, 4, 4, CONV, EPI>(a, st) : launch_gemv<NB, 8, 2, CONV, EPI>(a, st);
    return launch_gemv<NB, 8, 4, CONV, EPI>(a, st);
}

template <int NW>
void launch_prologue(const float *x, const ActParams &p, int64_t M, int8_t *xq, float *sx,
                     int32_t *rs, cudaStream_t st) {
    launch_pdl(tq_prologue_fwht_kernel<NW>, dim3((unsigned)M), dim3(NW * 32), 0, st, x, p, xq, sx, rs);
}

typedef void (*PrologueFn)(const float *, const ActParams &, int64_t, int8_t *, float *, int32_t *,
                           cudaStream_t);

template <int... NWs>
struct PrologueTable {
    static constexpr PrologueFn fns[sizeof...(NWs)] = {&launch_prologue<NWs>...};
};
template <int... NWs>
constexpr PrologueFn PrologueTable<NWs...>::fns[sizeof...(NWs)];
using Prologues = PrologueTable<1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11, 12, 13, 14, 15, 16, 17, 18, 19,
                                20, 21, 22, 23, 24, 25, 26, 27, 28, 29, 30, 31, 32>;
constexpr int64_t kMaxFwhtFusedK = 512 * 32;

// Many tokens: persistent ring kernel (one CTA per SM share, rows streamed
// through shared memory); few tokens: one CTA per token.
template <int VEC>
void launch_act_ring(const float *x, const ActParams &p, int64_t M, int64_t K, int8_t *xq, float *sx,
                     int32_t *rs, int sms, cudaStream_t st) {
    static std::atomic<int> per_sm_c[kMaxDevices];
    int dev = 0;
    cudaGetDevice(&dev);
    const int smem = kActRing * (int)(K / 4) * 16;
    const int key = per_sm_c[dev].load();
    int per_sm = 0;
    if ((key >> 8) == smem + 1) {
        per_sm = key & 0xff;
    } else {
        if (cudaFuncSetAttribute(tq_act_ring_kernel<VEC>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
                cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, tq_act_ring_kernel<VEC>, kActThreads,
                                                          (size_t)smem) != cudaSuccess)
            per_sm = 1;
        if (per_sm < 1) per_sm = 1;
        per_sm_c[dev].store(((smem + 1) << 8) | (per_sm & 0xff));
    }
    const int64_t cap = (int64_t)per_sm * sms;
    const unsigned grid = (unsigned)(M < cap ? M : cap);
    launch_pdl(tq_act_ring_kernel<VEC>, dim3(grid), dim3(kActThreads), (size_t)smem, st, x, M, (int)K, p, xq,
               sx, rs);
}

void launch_act(const float *x, const ActParams &p, int64_t M, int64_t K, int8_t *xq, float *sx,
                int32_t *rs, cudaStream_t st) {
    const int nv = (int)(K / 4);
    int sms = 0;
    check_device(&sms);
    if (M >= 2 * (int64_t)sms && nv <= 2048) {
        if (nv <= 256) return launch_act_ring<1>(x, p, M, K, xq, sx, rs, sms, st);
        if (nv <= 512) return launch_act_ring<2>(x, p, M, K, xq, sx, rs, sms, st);
        if (nv <= 1024) return launch_act_ring<4>(x, p, M, K, xq, sx, rs, sms, st);
        return launch_act_ring<8>(x, p, M, K, xq, sx, rs, sms, st);
    }
    const dim3 grid((unsigned)M), block(kActThreads);
    if (nv <= 256)
        launch_pdl(tq_act_quant_kernel<1>, grid, block, 0, st, x, (int)K, p, xq, sx, rs);
    else if (nv <= 512)
        launch_pdl(tq_act_quant_kernel<2>, grid, block, 0, st, x, (int)K, p, xq, sx, rs);
    else if (nv <= 1024)
        launch_pdl(tq_act_quant_kernel<4>, grid, block, 0, st, x, (int)K, p, xq, sx, rs);
    else if (nv <= 2048)
        launch_pdl(tq_act_quant_kernel<8>, grid, block, 0, st, x, (int)K, p, xq, sx, rs);
    else
        launch_pdl(tq_act_quant_kernel<0>, grid, block, 0, st, x, (int)K, p, xq, sx, rs);
}

// Per-tensor mode of the pack pass: the partial sums of tq_absum_partial_kernel
// and the height of the whole summation tree (partial == nullptr: per row).
struct PerTensor {
    const double *partial = nullptr;
    int nparts = 0;
    int height = 0;
};

// Persistent pack grid: as many CTAs as fit on the device, at most one row per
// team.  K <= 8192: a team of T warps streams its rows through a shared-memory
// ring (smem bytes per CTA); larger K: one warp streams each row twice.
template <typename Kern>
tq_status launch_pack_grid(Kern kern, std::atomic<int> *occ, int64_t rows_per_cta, int smem,
                           const float *w, int64_t N, int64_t K, uint8_t *packed, float *gamma,
                           const PerTensor &pt, int reverse, int opts, float ratio, cudaStream_t st) {
    int dev = 0, sms = 0;
    if (tq_status e = check_device(&sms)) return e;
    cudaGetDevice(&dev);
    // occupancy depends on smem, i.e. on K: cache it per (device, smem)
    const int key = occ[dev].load();
    int per_sm = 0;
    if ((key >> 8) == smem + 1) {
        per_sm = key & 0xff;
    } else {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kPackThreads, (size_t)smem) !=
                cudaSuccess)
            return TQ_ERR_CUDA;
        if (per_sm < 1) per_sm = 1;
        occ[dev].store(((smem + 1) << 8) | (per_sm & 0xff));
    }
    const int64_t need = (N + rows_per_cta - 1) / rows_per_cta;
    const int64_t cap = (int64_t)per_sm * sms;
    const unsigned grid = (unsigned)(need < cap ? need : cap);
    return launch_pdl(kern, dim3(grid), dim3(kPackThreads), (size_t)smem, st, w, N, (int)K,
                      1.0 / (double)K, packed, gamma, pt.partial, pt.nparts, pt.height, reverse, opts, ratio);
}

template <bool SAN, bool CONV>
tq_status launch_pack_rows_s(const float *w, int64_t N, int64_t K, uint8_t *packed, float *gamma,
                             const PerTensor &pt, int reverse, int opts, float ratio, cudaStream_t st) {
    static std::atomic<int> occ[5][kMaxDevices];
    const int64_t nv = K / 4;
    const int k = (int)K;
    if (nv <= 32 * kTeamVec * 1)
        return launch_pack_grid(tq_pack_team_kernel<1, SAN, CONV>, occ[0], kPackWarps / 1, pack_team_smem(1, k), w, N, K, packed, gamma, pt, reverse, opts, ratio, st);
    if (nv <= 32 * kTeamVec * 2)
        return launch_pack_grid(tq_pack_team_kernel<2, SAN, CONV>, occ[1], kPackWarps / 2, pack_team_smem(2, k), w, N, K, packed, gamma, pt, reverse, opts, ratio, st);
    if (nv <= 32 * kTeamVec * 4)
        return launch_pack_grid(tq_pack_team_kernel<4, SAN, CONV>, occ[2], kPackWarps / 4, pack_team_smem(4, k), w, N, K, packed, gamma, pt, reverse, opts, ratio, st);
    if (nv <= 32 * kTeamVec * 8)
        return launch_pack_grid(tq_pack_team_kernel<8, SAN, CONV>, occ[3], kPackWarps / 8, pack_team_smem(8, k), w, N, K, packed, gamma, pt, reverse, opts, ratio, st);
    return launch_pack_grid(tq_pack_rows_kernel<SAN, CONV>, occ[4], kPackWarps, 0, w, N, K, packed, gamma, pt, reverse, opts, ratio, st);
}

// Options word of the pack kernels: bit 0 inputs ready, bits 1-2 layout (bit 3:
// kPackOptFixed).
inline int pack_opts(int ready, int enc) { return (ready ? 1 : 0) | (enc << 1); }

tq_status launch_pack_rows(const float *w, int64_t N, int64_t K, int sanitize, uint8_t *packed,
                           float *gamma, const PerTensor &pt, int reverse, int opts, float ratio, cudaStream_t st) {
    if ((opts >> 1) & 3)  // a layout other than Foundry's
        return sanitize ? launch_pack_rows_s<true, true>(w, N, K, packed, gamma, pt, reverse, opts, ratio, st)
                        : launch_pack_rows_s<false, true>(w, N, K, packed, gamma, pt, reverse, opts, ratio, st);
    return sanitize ? launch_pack_rows_s<true, false>(w, N, K, packed, gamma, pt, reverse, opts, ratio, st)
                    : launch_pack_rows_s<false, false>(w, N, K, packed, gamma, pt, reverse, opts, ratio, st);
}

size_t pack_parts(int64_t nv) {
    const int64_t chunk_min = 4096;  // float4 per CTA, at least
    int64_t chunk = (nv + 1183) / 1184;
    if (chunk < chunk_min) chunk = chunk_min;
    return (size_t)((nv + chunk - 1) / chunk);
}

// Tokens per GEMM tile.  Cost model: rounds of tiles over the SMs times the
// time of one K-step, 4 MMAs of BT/2 cycles each but no faster than the
// single-thread issue rate (about 72 cycles per MMA); ties go to the smaller
// tile (less padding and x_q traffic).  No 192-token tiles: where the model
// preferred them (one round of tiles either way) the 256-token tile measured
// faster or close (fused 512 x 5632 x 2048 layer 19.8 -> 15.8 us; SwiGLU
// block 67.7 -> 70.3 us), and with more rounds 256 wins the model anyway.
int gemm_tile_tokens(int64_t M, int64_t N, int sms) {
    int best = 64;
    int64_t best_cost = -1;
    for (int bt : {64, 128, 256}) {
        const int64_t tiles = ((M + bt - 1) / bt) * ((N + kTileN - 1) / kTileN);
        const int64_t rounds = (tiles + sms - 1) / sms;
        const int64_t cost = rounds * (bt / 2 > 72 ? bt / 2 : 72);
        if (best_cost < 0 || cost < best_cost) {
            best = bt;
            best_cost = cost;
        }
    }
    return best;
}

template <bool CONV, bool EPI>
tq_status contraction(const GemmArgs &a, int sms, cudaStream_t st) {
    if (a.M <= 16 && a.K <= kGemvMaxK)
        return a.M <= 8 ? gemv_shape<1, CONV, EPI>(a, st) : gemv_shape<2, CONV, EPI>(a, st);
    switch (gemm_tile_tokens(a.M, a.N, sms)) {
    case 64: return launch_gemm<64, CONV, EPI>(a, sms, st);
    case 128: return launch_gemm<128, CONV, EPI>(a, sms, st);
    default: return launch_gemm<256, CONV, EPI>(a, sms, st);
    }
}

// ep: the extra epilogue of tq_ternary_gemm_ex, or nullptr.
tq_status gemm_dispatch(const int8_t *xq, const float *s_x, const int32_t *rowsum,
                        const uint8_t *packed, const float *gamma, unsigned flags, int64_t M,
                        int64_t N, int64_t K, float *y, int32_t *acc, int sms, cudaStream_t st,
                        const Epilogue *ep = nullptr) {
    const int per_row = (flags & TQ_GAMMA_PER_ROW) ? 1 : 0;
    const int enc = flag_encoding(flags);
    const int mode = ((flags & TQ_FLAG_WEIGHTS_STATIC) ? kModeWeightsStatic : 0) |
                     ((flags & TQ_FLAG_INPUTS_READY) ? kModeInputsReady : 0) | (enc << kModeEncShift);
    if (!ep && M <= 8 && K <= kStreamMaxK && (mode & kModeInputsReady))
        return launch_gemv_stream(xq, s_x, rowsum, packed, gamma, per_row, M, N, K, y, acc, enc, st);
    const GemmArgs a{xq, s_x, rowsum, packed, gamma, per_row, M, N, K, y, acc, mode,
                     ep ? *ep : Epilogue{nullptr, nullptr, 0}};
    const bool conv = enc != kEncFoundry;
    if (ep) return conv ? contraction<true, true>(a, sms, st) : contraction<false, true>(a, sms, st);
    return conv ? contraction<true, false>(a, sms, st) : contraction<false, false>(a, sms, st);
}


// ---------------------------------------------------------------------------
// Training helpers
// ---------------------------------------------------------------------------
// 2-D fp16 tensor [rows][cols] (row stride = 2 cols bytes), box [box_rows][box_cols].
bool make_tmap_f16(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows, uint32_t box_cols,
                    uint32_t box_rows, CUtensorMapSwizzle swz) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Row length of the fp16 planes of the backward pass: N rounded up to a step.
inline int64_t bwd_plane_cols(int64_t N) { return (N + kBwdStepN - 1) / kBwdStepN * kBwdStepN; }

// Host copies of the xorshift64 jump tables: the state after a flip call.
const uint64_t kXsChunkHost[TQ_XS_CHUNK_BITS][64] = TQ_XS_CHUNK_INIT;
const uint64_t kXsWarpHost[TQ_XS_WARPS][64] = TQ_XS_WARP_INIT;
const uint64_t kXsLaneHost[64][32] = TQ_XS_LANE_INIT;

inline uint64_t xs_apply(const uint64_t *cols, int stride, uint64_t x) {
    uint64_t r = 0;
    for (int b = 0; b < 64; ++b)
        if ((x >> b) & 1ull) r ^= cols[b * stride];
    return r;
}

// A^n x for n % 64 == 0, n < 2^40.
uint64_t xs_jump(uint64_t x, int64_t n) {
    const int64_t chunks = n / kFlipChunk;
    int64_t rem = n % kFlipChunk;
    for (int j = 0; j < TQ_XS_CHUNK_BITS; ++j)
        if ((chunks >> j) & 1) x = xs_apply(kXsChunkHost[j], 1, x);
    x = xs_apply(kXsWarpHost[rem / kFlipWarpRun], 1, x);
    rem %= kFlipWarpRun;
    return xs_apply(&kXsLaneHost[0][rem / kFlipRun], 32, x);
}

template <typename Kern>
tq_status set_smem_once(Kern kern, int bytes, std::atomic<int> *done) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TQ_ERR_CUDA;
    if (!done[dev].load()) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
            return TQ_ERR_CUDA;
        done[dev].store(1);
    }
    return TQ_OK;
}

template <bool CONV>
tq_status launch_flip(uint8_t *packed, const float *grad, int64_t nw, float temp, uint64_t x0, int mode,
                      int sms, cudaStream_t st) {
    static std::atomic<int> done[kMaxDevices];
    if (tq_status e = set_smem_once(tq_flip_kernel<CONV>, kFlipSmem, done)) return e;
    const int64_t nchunks = (nw + kFlipChunk - 1) / kFlipChunk;
    const int64_t target = 2 * (int64_t)sms;  // two CTAs per SM
    const int64_t per_cta = (nchunks + target - 1) / target;
    const int64_t grid = (nchunks + per_cta - 1) / per_cta;
    return launch_pdl(tq_flip_kernel<CONV>, dim3((unsigned)grid), dim3(kFlipThreads), (size_t)kFlipSmem, st, packed,
                      grad, nw, temp, x0, per_cta, mode);
}

template <bool CONV>
tq_status launch_bwd_gemm(const __half *planes, const float *inv_scale, const uint8_t *packed,
                          const float *row_scale, int accumulate,
                          int64_t M, int64_t N, int64_t K, float *dX, int mode, int sms, cudaStream_t st) {
    static std::atomic<int> done[kMaxDevices];
    if (tq_status e = set_smem_once(tq_bwd_gemm_kernel<CONV>, kBwdDynamic, done)) return e;
    // planes [2 M][Np] fp16 in 64-byte-swizzled [256][32] boxes; packed [N][K/4]
    // in plain [32][32 B] boxes.
    CUtensorMap tg, tw;
    if (!make_tmap_f16(&tg, planes, (uint64_t)bwd_plane_cols(N), (uint64_t)(kBwdPlanes * M), kBwdStepN, kBwdTileT,
                        CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_tmap_u8(&tw, packed, (uint64_t)(K / 4), (uint64_t)N, kBwdTileF / 4, kBwdStepN,
                      CU_TENSOR_MAP_SWIZZLE_NONE))
        return TQ_ERR_CUDA;
    const int64_t tiles = ((M + kBwdTileT - 1) / kBwdTileT) * ((K + kBwdTileF - 1) / kBwdTileF);
    const unsigned grid = (unsigned)(tiles < sms ? tiles : sms);
    return launch_pdl(tq_bwd_gemm_kernel<CONV>, dim3(grid), dim3(kGemmThreads), (size_t)kBwdDynamic, st, tg, tw,
                      inv_scale, row_scale, accumulate, (int)M, (int)N, (int)K, dX, mode);
}

// ---------------------------------------------------------------------------
// Grouped small-M contraction
// ---------------------------------------------------------------------------
constexpr int kGroupSmemBudget = 226 * 1024;  // dynamic; the opt-in limit is 227 KiB including static

// Workspace of tq_bitlinear_grouped: x_q [Gx][M][K] (in the grouped GEMV's
// layout), s_x [Gx][M], rowsum [Gx][M], each part 256-byte aligned.
inline size_t grouped_parts(int64_t Gx, int64_t M, int64_t K, size_t off[3]) {
    auto al = [](size_t b) { return (b + 255) & ~(size_t)255; };
    off[0] = 0;
    off[1] = al((size_t)(Gx * M * K));
    off[2] = off[1] + al((size_t)(Gx * M) * 4);
    return off[2] + al((size_t)(Gx * M) * 4);
}

template <int NB, int ENC, bool FULL>
tq_status launch_group_gemv_k(const GroupTable &tab, const GroupPlan &pl, const int8_t *xq, const float *sx,
                              const int32_t *rs, float *y, int sms, cudaStream_t st) {
    static std::atomic<int> done[kMaxDevices];
    if (tq_status e = set_smem_once(tq_gemv_group_kernel<NB, ENC, FULL>, kGroupSmemBudget, done)) return e;
    const int64_t grid = pl.nstrips < sms ? pl.nstrips : sms;
    return launch_pdl(tq_gemv_group_kernel<NB, ENC, FULL>, dim3((unsigned)grid), dim3(kGrpThreads), (size_t)pl.smem,
                      st, tab, pl, xq, sx, rs, y);
}

template <int NB, int ENC>
tq_status launch_group_gemv(const GroupTable &tab, const GroupPlan &pl, const int8_t *xq, const float *sx,
                            const int32_t *rs, float *y, int sms, cudaStream_t st) {
    return pl.K % 256 == 0 ? launch_group_gemv_k<NB, ENC, true>(tab, pl, xq, sx, rs, y, sms, st)
                           : launch_group_gemv_k<NB, ENC, false>(tab, pl, xq, sx, rs, y, sms, st);
}

template <int NB>
tq_status launch_group_gemv_enc(const GroupTable &tab, const GroupPlan &pl, const int8_t *xq, const float *sx,
                                const int32_t *rs, float *y, int sms, cudaStream_t st) {
    if (pl.enc == kEncFormat0) return launch_group_gemv<NB, kEncFormat0>(tab, pl, xq, sx, rs, y, sms, st);
    if (pl.enc == kEncFormat1) return launch_group_gemv<NB, kEncFormat1>(tab, pl, xq, sx, rs, y, sms, st);
    return launch_group_gemv<NB, kEncFoundry>(tab, pl, xq, sx, rs, y, sms, st);
}

// Activation pass of the grouped call: rows of x quantised per token, x_q
// written in the grouped GEMV's layout.
inline tq_status launch_act_group(const float *x, const ActParams &p, int64_t rows, int64_t K, int8_t *xq,
                                  float *sx, int32_t *rs, cudaStream_t st) {
    const int nv = (int)(K / 4);
    const dim3 grid((unsigned)rows), block(kActThreads);
    if (nv <= 256) return launch_pdl(tq_act_quant_kernel<1, true>, grid, block, 0, st, x, (int)K, p, xq, sx, rs);
    if (nv <= 512) return launch_pdl(tq_act_quant_kernel<2, true>, grid, block, 0, st, x, (int)K, p, xq, sx, rs);
    if (nv <= 1024) return launch_pdl(tq_act_quant_kernel<4, true>, grid, block, 0, st, x, (int)K, p, xq, sx, rs);
    return launch_pdl(tq_act_quant_kernel<8, true>, grid, block, 0, st, x, (int)K, p, xq, sx, rs);
}

}  // namespace

extern "C" {

int tq_version(void) { return 100; }

const char *tq_status_string(tq_status s) {
    switch (s) {
        case TQ_OK: return "ok";
        case TQ_ERR_NULL: return "a required pointer is NULL";
        case TQ_ERR_SHAPE: return "a size is out of range or breaks a divisibility rule";
        case TQ_ERR_ALIGN: return "a pointer is not 16-byte aligned";
        case TQ_ERR_ARG: return "unknown flag, overlapping buffers, or workspace too small";
        case TQ_ERR_CUDA: return "a CUDA runtime call or kernel launch failed";
        case TQ_ERR_DEVICE: return "the current device is not compute capability 10.0 (sm_100a)";
        case TQ_ERR_TIMEOUT: return "a bounded wait inside a kernel gave up";
    }
    return "unknown status";
}

size_t tq_pack_workspace_bytes(int64_t N, int64_t K, unsigned flags) {
    if (flags & TQ_GAMMA_PER_ROW) return 0;
    if (N <= 0 || K <= 0) return 0;
    return pack_parts(N * K / 4) * sizeof(DD) + 16;
}

// Shared body of the two packing entry points; ratio 0 selects the round rule.
static tq_status pack_impl(const float *w, int64_t N, int64_t K, unsigned flags, float ratio,
                           uint8_t *packed, float *gamma, void *workspace, size_t workspace_bytes,
                           tq_stream_t stream) {
    if (!w || !packed || !gamma) return TQ_ERR_NULL;
    if (N < 1 || N > INT32_MAX) return TQ_ERR_SHAPE;
    if (tq_status e = check_k(K)) return e;
    if (flags & ~(TQ_GAMMA_PER_ROW | TQ_FLAG_SANITIZE_NONFINITE | TQ_FLAG_INPUTS_READY | TQ_ENC_MASK))
        return TQ_ERR_ARG;
    const int enc = flag_encoding(flags);
    if (enc < 0) return TQ_ERR_ARG;
    if (!aligned16(w) || !aligned16(packed) || !aligned16(gamma)) return TQ_ERR_ALIGN;
    const bool per_row = flags & TQ_GAMMA_PER_ROW;
    const int ready = (flags & TQ_FLAG_INPUTS_READY) ? 1 : 0;
    const size_t wbytes = (size_t)(N * K) * 4, pbytes = (size_t)(N * K / 4),
                 gbytes = (per_row ? (size_t)N : 1) * 4;
    if (overlap(w, wbytes, packed, pbytes) || overlap(w, wbytes, gamma, gbytes) ||
        overlap(packed, pbytes, gamma, gbytes))
        return TQ_ERR_ARG;
    const size_t need = tq_pack_workspace_bytes(N, K, flags);
    if (need) {
        if (!workspace) return TQ_ERR_NULL;
        if (!aligned16(workspace)) return TQ_ERR_ALIGN;
        if (workspace_bytes < need) return TQ_ERR_ARG;
        if (overlap(workspace, need, w, wbytes) || overlap(workspace, need, packed, pbytes) ||
            overlap(workspace, need, gamma, gbytes))
            return TQ_ERR_ARG;
    }
    if (tq_status e = check_device(nullptr)) return e;
    const int sanitize = (flags & TQ_FLAG_SANITIZE_NONFINITE) ? 1 : 0;
    cudaStream_t st = cs(stream);
    if (per_row) {
        if (tq_status e = launch_pack_rows(w, N, K, sanitize, packed, gamma, PerTensor{}, 0,
                                           pack_opts(ready, enc), ratio, st))
            return e;
        return launch_status();
    }
    const int64_t total_v = N * K / 4;
    const size_t nparts = pack_parts(total_v);
    const int64_t chunk = (total_v + (int64_t)nparts - 1) / (int64_t)nparts;
    double *partial = reinterpret_cast<double *>(workspace);
    if (tq_status e = launch_pdl(tq_absum_partial_kernel, dim3((unsigned)nparts), dim3(kPackThreads), 0,
                                 st, w, total_v, chunk, sanitize, partial, ready))
        return e;
    PerTensor pt;
    pt.partial = partial;
    pt.nparts = (int)nparts;
    pt.height = absum_tree_height(chunk, (int)nparts);
    if (tq_status e = launch_pack_rows(w, N, K, sanitize, packed, gamma, pt, 1, pack_opts(0, enc), ratio, st))
        return e;
    return launch_status();
}

tq_status tq_quantize_ternary_pack(const float *w, int64_t N, int64_t K, unsigned flags,
                                   uint8_t *packed, float *gamma, void *workspace,
                                   size_t workspace_bytes, tq_stream_t stream) {
    return pack_impl(w, N, K, flags, 0.0f, packed, gamma, workspace, workspace_bytes, stream);
}

tq_status tq_quantize_ternary_pack_threshold(const float *w, int64_t N, int64_t K, unsigned flags,
                                             float ratio, uint8_t *packed, float *gamma,
                                             void *workspace, size_t workspace_bytes,
                                             tq_stream_t stream) {
    if (!(ratio > 0.0f && ratio <= 64.0f)) return TQ_ERR_ARG;  // NaN fails too
    return pack_impl(w, N, K, flags, ratio, packed, gamma, workspace, workspace_bytes, stream);
}

tq_status tq_quantize_ternary_pack_abs_threshold(const float *w, int64_t N, int64_t K, unsigned flags,
                                                 float threshold, uint8_t *packed, float *gamma,
                                                 tq_stream_t stream) {
    if (!w || !packed || !gamma) return TQ_ERR_NULL;
    if (N < 1 || N > INT32_MAX) return TQ_ERR_SHAPE;
    if (tq_status e = check_k(K)) return e;
    if (flags & ~(TQ_FLAG_SANITIZE_NONFINITE | TQ_FLAG_INPUTS_READY | TQ_ENC_MASK)) return TQ_ERR_ARG;
    const int enc = flag_encoding(flags);
    if (enc < 0) return TQ_ERR_ARG;
    if (!(threshold >= 0.0f && threshold <= 3.4028235e38f)) return TQ_ERR_ARG;  // NaN fails too
    if (!aligned16(w) || !aligned16(packed) || !aligned16(gamma)) return TQ_ERR_ALIGN;
    const size_t wbytes = (size_t)(N * K) * 4, pbytes = (size_t)(N * K / 4);
    if (overlap(w, wbytes, packed, pbytes) || overlap(w, wbytes, gamma, 4) || overlap(packed, pbytes, gamma, 4))
        return TQ_ERR_ARG;
    if (tq_status e = check_device(nullptr)) return e;
    const int sanitize = (flags & TQ_FLAG_SANITIZE_NONFINITE) ? 1 : 0;
    const int opts = pack_opts((flags & TQ_FLAG_INPUTS_READY) ? 1 : 0, enc) | kPackOptFixed;
    if (tq_status e = launch_pack_rows(w, N, K, sanitize, packed, gamma, PerTensor{}, 0, opts, threshold, cs(stream)))
        return e;
    return launch_status();
}

tq_status tq_quantize_act_int8(const float *x, int64_t M, int64_t K, unsigned flags, float eta_min,
                               float eta_max, int8_t *xq, float *s_x, int32_t *rowsum,
                               tq_stream_t stream) {
    if (!x || !xq || !s_x || !rowsum) return TQ_ERR_NULL;
    if (M < 1 || M > INT32_MAX) return TQ_ERR_SHAPE;
    if (tq_status e = check_k(K)) return e;
    if (flags & ~(TQ_FLAG_ETA_CLAMP | TQ_FLAG_SANITIZE_NONFINITE | TQ_FLAG_INPUTS_READY)) return TQ_ERR_ARG;
    if ((flags & TQ_FLAG_ETA_CLAMP) && !(eta_min > 0.0f && eta_min <= eta_max)) return TQ_ERR_ARG;
    if ((flags & TQ_FLAG_SANITIZE_NONFINITE) && !(eta_max > 0.0f && eta_max < 3.0e38f)) return TQ_ERR_ARG;
    if (!aligned16(x) || !aligned16(xq) || !aligned16(s_x) || !aligned16(rowsum)) return TQ_ERR_ALIGN;
    const size_t xb = (size_t)(M * K) * 4, qb = (size_t)(M * K), mb = (size_t)M * 4;
    if (overlap(x, xb, xq, qb) || overlap(x, xb, s_x, mb) || overlap(x, xb, rowsum, mb) ||
        overlap(xq, qb, s_x, mb) || overlap(xq, qb, rowsum, mb) || overlap(s_x, mb, rowsum, mb))
        return TQ_ERR_ARG;
    if (tq_status e = check_device(nullptr)) return e;
    ActParams p{};
    p.sanitize = (flags & TQ_FLAG_SANITIZE_NONFINITE) ? 1 : 0;
    p.clamp_eta = (flags & TQ_FLAG_ETA_CLAMP) ? 1 : 0;
    p.eta_min = eta_min;
    p.eta_max = eta_max;
    p.ready = (flags & TQ_FLAG_INPUTS_READY) ? 1 : 0;
    launch_act(x, p, M, K, xq, s_x, rowsum, cs(stream));
    return launch_status();
}

tq_status tq_fwht512(const float *x, float *y, int64_t rows, int64_t K, int normalize,
                     tq_stream_t stream) {
    if (!x || !y) return TQ_ERR_NULL;
    if (rows < 1 || K < 512 || K % 512 != 0 || K > kMaxK) return TQ_ERR_SHAPE;
    if (!aligned16(x) || !aligned16(y)) return TQ_ERR_ALIGN;
    const size_t b = (size_t)(rows * K) * 4;
    if (x != y && overlap(x, b, y, b)) return TQ_ERR_ARG;
    if (tq_status e = check_device(nullptr)) return e;
    const int64_t nblocks = rows * (K / 512);
    return launch_pdl(tq_fwht512_kernel, dim3((unsigned)((nblocks + 7) / 8)), dim3(256), 0, cs(stream),
                      x, y, nblocks, normalize);
}

tq_status tq_fwht_roundtrip(const float *x, float *y, int64_t rows, int64_t K, float eta_min,
                            float eta_max, float *eta_out, tq_stream_t stream) {
    if (!x || !y) return TQ_ERR_NULL;
    if (rows < 1 || rows > INT32_MAX || K < 512 || K % 512 != 0 || K > kMaxFwhtFusedK) return TQ_ERR_SHAPE;
    if (!(eta_min > 0.0f && eta_min <= eta_max && eta_max < 3.0e38f)) return TQ_ERR_ARG;
    if (!aligned16(x) || !aligned16(y) || (eta_out && !aligned16(eta_out))) return TQ_ERR_ALIGN;
    const size_t b = (size_t)(rows * K) * 4;
    if (x != y && overlap(x, b, y, b)) return TQ_ERR_ARG;
    if (eta_out && (overlap(eta_out, (size_t)rows * 4, x, b) || overlap(eta_out, (size_t)rows * 4, y, b)))
        return TQ_ERR_ARG;
    if (tq_status e = check_device(nullptr)) return e;
    return launch_pdl(tq_fwht_roundtrip_kernel, dim3((unsigned)rows), dim3((unsigned)(K / 512 * 32)), 0, cs(stream),
                      x, y, eta_min, eta_max, eta_out);
}

// Shared body of tq_ternary_gemm and tq_ternary_gemm_ex (ep: the extra epilogue or nullptr).
static tq_status gemm_impl(const int8_t *xq, const float *s_x, const int32_t *rowsum,
                           const uint8_t *packed, const float *gamma, unsigned flags, int64_t M,
                           int64_t N, int64_t K, float *y, int32_t *acc, tq_stream_t stream,
                           const Epilogue *ep) {
    if (!xq || !s_x || !rowsum || !packed || !gamma || !y) return TQ_ERR_NULL;
    if (M < 1 || N < 1 || M > INT32_MAX || N > INT32_MAX) return TQ_ERR_SHAPE;
    if (tq_status e = check_k(K)) return e;
    if (flags & ~(TQ_GAMMA_PER_ROW | TQ_FLAG_WEIGHTS_STATIC | TQ_FLAG_INPUTS_READY | TQ_ENC_MASK))
        return TQ_ERR_ARG;
    if (flag_encoding(flags) < 0) return TQ_ERR_ARG;
    if (!aligned16(xq) || !aligned16(s_x) || !aligned16(rowsum) || !aligned16(packed) ||
        !aligned16(gamma) || !aligned16(y) || (acc && !aligned16(acc)))
        return TQ_ERR_ALIGN;
    const size_t yb = (size_t)(M * N) * 4;
    const size_t gb = ((flags & TQ_GAMMA_PER_ROW) ? (size_t)N : 1) * 4;
    const void *ins[5] = {xq, s_x, rowsum, packed, gamma};
    const size_t inb[5] = {(size_t)(M * K), (size_t)M * 4, (size_t)M * 4, (size_t)(N * K / 4), gb};
    for (int i = 0; i < 5; ++i)
        if (overlap(ins[i], inb[i], y, yb) || (acc && overlap(ins[i], inb[i], acc, yb))) return TQ_ERR_ARG;
    if (acc && overlap(acc, yb, y, yb)) return TQ_ERR_ARG;
    int sms = 0;
    if (tq_status e = check_device(&sms)) return e;
    return gemm_dispatch(xq, s_x, rowsum, packed, gamma, flags, M, N, K, y, acc, sms, cs(stream), ep);
}

tq_status tq_ternary_gemm(const int8_t *xq, const float *s_x, const int32_t *rowsum,
                          const uint8_t *packed, const float *gamma, unsigned flags, int64_t M,
                          int64_t N, int64_t K, float *y, int32_t *acc, tq_stream_t stream) {
    return gemm_impl(xq, s_x, rowsum, packed, gamma, flags, M, N, K, y, acc, stream, nullptr);
}

tq_status tq_ternary_gemm_ex(const int8_t *xq, const float *s_x, const int32_t *rowsum,
                             const uint8_t *packed, const float *gamma, unsigned flags, int64_t M,
                             int64_t N, int64_t K, const float *bias, const int32_t *acc_bias,
                             int out_shift, float *y, int32_t *acc, tq_stream_t stream) {
    if (out_shift < 0 || out_shift > 31) return TQ_ERR_ARG;
    if ((bias && !aligned16(bias)) || (acc_bias && !aligned16(acc_bias))) return TQ_ERR_ALIGN;
    const size_t yb = (size_t)(M > 0 && N > 0 ? M * N : 0) * 4, nb = (size_t)(N > 0 ? N : 0) * 4;
    if ((bias && (overlap(bias, nb, y, yb) || (acc && overlap(bias, nb, acc, yb)))) ||
        (acc_bias && (overlap(acc_bias, nb, y, yb) || (acc && overlap(acc_bias, nb, acc, yb)))))
        return TQ_ERR_ARG;
    const Epilogue ep{bias, acc_bias, out_shift};
    return gemm_impl(xq, s_x, rowsum, packed, gamma, flags, M, N, K, y, acc, stream, &ep);
}

size_t tq_fused_workspace_bytes(int64_t M, int64_t K, unsigned flags) {
    (void)flags;
    if (M <= 0 || K <= 0) return 0;
    const size_t xq = ((size_t)(M * K) + 255) & ~(size_t)255;
    const size_t v = (((size_t)M * 4) + 255) & ~(size_t)255;
    return xq + 2 * v;
}

tq_status tq_bitlinear_fused(const float *x, const float *rms_gain, float rms_eps, float eta_min,
                             float eta_max, unsigned flags, const uint8_t *packed,
                             const float *gamma, int64_t M, int64_t N, int64_t K, float *y,
                             int8_t *xq_out, float *s_x_out, void *workspace,
                             size_t workspace_bytes, tq_stream_t stream) {
    if (!x || !packed || !gamma || !y || !workspace) return TQ_ERR_NULL;
    if (M < 1 || N < 1 || M > INT32_MAX || N > INT32_MAX) return TQ_ERR_SHAPE;
    if (tq_status e = check_k(K)) return e;
    const unsigned known = TQ_GAMMA_PER_ROW | TQ_FLAG_FWHT | TQ_FLAG_RMSNORM | TQ_FLAG_ETA_CLAMP |
                           TQ_FLAG_SANITIZE_NONFINITE | TQ_FLAG_WEIGHTS_STATIC | TQ_FLAG_INPUTS_READY |
                           TQ_ENC_MASK;
    if (flags & ~known) return TQ_ERR_ARG;
    if (flag_encoding(flags) < 0) return TQ_ERR_ARG;
    if ((flags & TQ_FLAG_FWHT) && (K % 512 != 0 || K > kMaxFwhtFusedK)) return TQ_ERR_SHAPE;
    if ((flags & TQ_FLAG_ETA_CLAMP) && !(eta_min > 0.0f && eta_min <= eta_max)) return TQ_ERR_ARG;
    if ((flags & TQ_FLAG_SANITIZE_NONFINITE) && !(eta_max > 0.0f && eta_max < 3.0e38f)) return TQ_ERR_ARG;
    if ((flags & TQ_FLAG_RMSNORM) && !(rms_eps >= 0.0f)) return TQ_ERR_ARG;
    if (!aligned16(x) || !aligned16(packed) || !aligned16(gamma) || !aligned16(y) ||
        !aligned16(workspace) || (rms_gain && !aligned16(rms_gain)) || (xq_out && !aligned16(xq_out)) ||
        (s_x_out && !aligned16(s_x_out)))
        return TQ_ERR_ALIGN;
    const size_t need = tq_fused_workspace_bytes(M, K, flags);
    if (workspace_bytes < need) return TQ_ERR_ARG;
    const size_t xb = (size_t)(M * K) * 4, yb = (size_t)(M * N) * 4, qb = (size_t)(M * K),
                 pb = (size_t)(N * K / 4), gb = ((flags & TQ_GAMMA_PER_ROW) ? (size_t)N : 1) * 4;
    const void *outs[4] = {y, workspace, xq_out, s_x_out};
    const size_t outb[4] = {yb, need, qb, (size_t)M * 4};
    const void *ins[4] = {x, packed, gamma, rms_gain};
    const size_t inb[4] = {xb, pb, gb, (size_t)K * 4};
    for (int o = 0; o < 4; ++o) {
        if (!outs[o]) continue;
        for (int i = 0; i < 4; ++i)
            if (ins[i] && overlap(outs[o], outb[o], ins[i], inb[i])) return TQ_ERR_ARG;
        for (int o2 = o + 1; o2 < 4; ++o2)
            if (outs[o2] && overlap(outs[o], outb[o], outs[o2], outb[o2])) return TQ_ERR_ARG;
    }
    int sms = 0;
    if (tq_status e = check_device(&sms)) return e;
    cudaStream_t st = cs(stream);

    uint8_t *ws = reinterpret_cast<uint8_t *>(workspace);
    const size_t xq_sz = ((size_t)(M * K) + 255) & ~(size_t)255;
    const size_t v_sz = (((size_t)M * 4) + 255) & ~(size_t)255;
    int8_t *xq = xq_out ? xq_out : reinterpret_cast<int8_t *>(ws);
    float *sx = s_x_out ? s_x_out : reinterpret_cast<float *>(ws + xq_sz);
    int32_t *rs = reinterpret_cast<int32_t *>(ws + xq_sz + v_sz);

    ActParams p{};
    p.sanitize = (flags & TQ_FLAG_SANITIZE_NONFINITE) ? 1 : 0;
    p.clamp_eta = (flags & TQ_FLAG_ETA_CLAMP) ? 1 : 0;
    p.eta_min = eta_min;
    p.eta_max = eta_max;
    p.rmsnorm = (flags & TQ_FLAG_RMSNORM) ? 1 : 0;
    p.rms_eps = rms_eps;
    p.rms_gain = rms_gain;
    // Inputs ready: the activation pass reads x at once; the contraction still
    // waits for it (x_q is made here), but may stream its weights early.
    p.ready = (flags & TQ_FLAG_INPUTS_READY) ? 1 : 0;
    if (flags & TQ_FLAG_FWHT)
        Prologues::fns[K / 512 - 1](x, p, M, xq, sx, rs, st);
    else
        launch_act(x, p, M, K, xq, sx, rs, st);
    if (tq_status e = launch_status()) return e;
    const unsigned cflags = (flags & (TQ_GAMMA_PER_ROW | TQ_FLAG_WEIGHTS_STATIC | TQ_ENC_MASK)) |
                            ((flags & TQ_FLAG_INPUTS_READY) ? TQ_FLAG_WEIGHTS_STATIC : 0u);
    return gemm_dispatch(xq, sx, rs, packed, gamma, cflags, M, N, K, y, nullptr, sms, st);
}

// Workspace of tq_swiglu_mlp: the first projection's x_q, s_x, rowsum; the
// gate and up outputs; the down projection's x_q, s_x, rowsum (each 256-byte
// aligned).
static size_t swiglu_parts(int64_t M, int64_t D, int64_t F, size_t off[8]) {
    auto al = [](size_t b) { return (b + 255) & ~(size_t)255; };
    const size_t sz[8] = {al((size_t)(M * D)), al((size_t)M * 4), al((size_t)M * 4), al((size_t)(M * F) * 4),
                          al((size_t)(M * F) * 4), al((size_t)(M * F)), al((size_t)M * 4), al((size_t)M * 4)};
    size_t t = 0;
    for (int i = 0; i < 8; ++i) {
        off[i] = t;
        t += sz[i];
    }
    return t;
}

size_t tq_swiglu_workspace_bytes(int64_t M, int64_t d_model, int64_t d_ffn, unsigned flags) {
    (void)flags;
    if (M <= 0 || d_model <= 0 || d_ffn <= 0) return 0;
    size_t off[8];
    return swiglu_parts(M, d_model, d_ffn, off);
}

tq_status tq_swiglu_mlp(const float *x, int64_t M, int64_t d_model, int64_t d_ffn, unsigned flags,
                        float clamp_val, const uint8_t *gate_packed, const float *gate_gamma,
                        const uint8_t *up_packed, const float *up_gamma, const uint8_t *down_packed,
                        const float *down_gamma, float *y, float *act_out, void *workspace,
                        size_t workspace_bytes, tq_stream_t stream) {
    if (!x || !gate_packed || !gate_gamma || !up_packed || !up_gamma || !down_packed || !down_gamma || !y ||
        !workspace)
        return TQ_ERR_NULL;
    if (M < 1 || M > INT32_MAX) return TQ_ERR_SHAPE;
    if (tq_status e = check_k(d_model)) return e;
    if (tq_status e = check_k(d_ffn)) return e;
    if (d_model % 512 || d_ffn % 512 || d_model > kMaxFwhtFusedK || d_ffn > kMaxFwhtFusedK) return TQ_ERR_SHAPE;
    const unsigned known = TQ_GAMMA_PER_ROW | TQ_FLAG_FWHT | TQ_FLAG_RMSNORM | TQ_FLAG_SANITIZE_NONFINITE |
                           TQ_FLAG_WEIGHTS_STATIC | TQ_ENC_MASK;
    if ((flags & ~known) || !(flags & TQ_FLAG_FWHT) || flag_encoding(flags) < 0) return TQ_ERR_ARG;
    if (!(clamp_val > 0.0f && clamp_val < 3.0e38f)) return TQ_ERR_ARG;
    const void *al16[10] = {x, gate_packed, gate_gamma, up_packed, up_gamma, down_packed, down_gamma, y, workspace,
                            act_out};
    for (const void *q : al16)
        if (q && !aligned16(q)) return TQ_ERR_ALIGN;
    size_t off[8];
    const size_t need = swiglu_parts(M, d_model, d_ffn, off);
    if (workspace_bytes < need) return TQ_ERR_ARG;
    const size_t yb = (size_t)(M * d_model) * 4, ab = (size_t)(M * d_ffn) * 4;
    const bool pr = flags & TQ_GAMMA_PER_ROW;
    const void *ins[7] = {x, gate_packed, gate_gamma, up_packed, up_gamma, down_packed, down_gamma};
    const size_t inb[7] = {yb, (size_t)(d_ffn * d_model / 4), (pr ? (size_t)d_ffn : 1) * 4,
                           (size_t)(d_ffn * d_model / 4), (pr ? (size_t)d_ffn : 1) * 4,
                           (size_t)(d_model * d_ffn / 4), (pr ? (size_t)d_model : 1) * 4};
    const void *outs[3] = {y, workspace, act_out};
    const size_t outb[3] = {yb, need, ab};
    for (int o = 0; o < 3; ++o) {
        if (!outs[o]) continue;
        for (int i = 0; i < 7; ++i)
            if (overlap(outs[o], outb[o], ins[i], inb[i])) return TQ_ERR_ARG;
        for (int o2 = o + 1; o2 < 3; ++o2)
            if (outs[o2] && overlap(outs[o], outb[o], outs[o2], outb[o2])) return TQ_ERR_ARG;
    }
    int sms = 0;
    if (tq_status e = check_device(&sms)) return e;
    cudaStream_t st = cs(stream);
    uint8_t *ws = reinterpret_cast<uint8_t *>(workspace);
    int8_t *xq1 = reinterpret_cast<int8_t *>(ws + off[0]);
    float *sx1 = reinterpret_cast<float *>(ws + off[1]);
    int32_t *rs1 = reinterpret_cast<int32_t *>(ws + off[2]);
    float *yg = reinterpret_cast<float *>(ws + off[3]);
    float *yu = reinterpret_cast<float *>(ws + off[4]);
    int8_t *xq2 = reinterpret_cast<int8_t *>(ws + off[5]);
    float *sx2 = reinterpret_cast<float *>(ws + off[6]);
    int32_t *rs2 = reinterpret_cast<int32_t *>(ws + off[7]);
    ActParams p{};
    p.sanitize = (flags & TQ_FLAG_SANITIZE_NONFINITE) ? 1 : 0;
    p.eta_max = 40.0f;  // the quench bound of Hetman-2b's BitLinear (step 0)
    p.eta_min = 0.05f;
    p.rmsnorm = (flags & TQ_FLAG_RMSNORM) ? 1 : 0;
    p.rms_eps = 1e-6f;
    const unsigned cflags = flags & (TQ_GAMMA_PER_ROW | TQ_FLAG_WEIGHTS_STATIC | TQ_ENC_MASK);
    // gate and up see the same x: one activation pass for both
    Prologues::fns[d_model / 512 - 1](x, p, M, xq1, sx1, rs1, st);
    if (tq_status e = launch_status()) return e;
    if (tq_status e = gemm_dispatch(xq1, sx1, rs1, gate_packed, gate_gamma, cflags, M, d_ffn, d_model, yg,
                                    nullptr, sms, st))
        return e;
    if (tq_status e = gemm_dispatch(xq1, sx1, rs1, up_packed, up_gamma, cflags, M, d_ffn, d_model, yu, nullptr,
                                    sms, st))
        return e;
    if (tq_status e = launch_pdl(tq_swiglu_prologue_kernel, dim3((unsigned)M), dim3((unsigned)(d_ffn / 512 * 32)), 0,
                                 st, (const float *)yg, (const float *)yu, clamp_val, p, xq2, sx2, rs2, act_out))
        return e;
    return gemm_dispatch(xq2, sx2, rs2, down_packed, down_gamma, cflags, M, d_model, d_ffn, y, nullptr, sms, st);
}

// ---------------------------------------------------------------------------
// Training
// ---------------------------------------------------------------------------
size_t tq_backward_input_workspace_bytes(int64_t M, int64_t N) {
    if (M <= 0 || N <= 0) return 0;
    const size_t planes = ((size_t)(kBwdPlanes * M * bwd_plane_cols(N)) * 2 + 255) & ~(size_t)255;
    return planes + (((size_t)M * 4 + 255) & ~(size_t)255);
}

tq_status tq_ternary_backward_input(const float *dY, const uint8_t *packed, const float *gamma,
                                    const float *row_scale, unsigned flags, int64_t M, int64_t N, int64_t K,
                                    float *dX, void *workspace, size_t workspace_bytes, tq_stream_t stream) {
    if (!dY || !packed || !gamma || !dX || !workspace) return TQ_ERR_NULL;
    if (M < 1 || N < 1 || M > INT32_MAX / kBwdPlanes || N > INT32_MAX) return TQ_ERR_SHAPE;
    if (tq_status e = check_k(K)) return e;
    if (flags & ~(TQ_GAMMA_PER_ROW | TQ_FLAG_ACCUMULATE | TQ_ENC_MASK)) return TQ_ERR_ARG;
    const int enc = flag_encoding(flags);
    if (enc < 0) return TQ_ERR_ARG;
    if (!aligned16(dY) || !aligned16(packed) || !aligned16(gamma) || !aligned16(dX) || !aligned16(workspace) ||
        (row_scale && !aligned16(row_scale)))
        return TQ_ERR_ALIGN;
    const size_t need = tq_backward_input_workspace_bytes(M, N);
    if (workspace_bytes < need) return TQ_ERR_ARG;
    const size_t xb = (size_t)(M * K) * 4;
    const void *ins[4] = {dY, packed, gamma, row_scale};
    const size_t inb[4] = {(size_t)(M * N) * 4, (size_t)(N * K / 4),
                           ((flags & TQ_GAMMA_PER_ROW) ? (size_t)N : 1) * 4, (size_t)M * 4};
    for (int i = 0; i < 4; ++i)
        if (ins[i] && (overlap(ins[i], inb[i], dX, xb) || overlap(ins[i], inb[i], workspace, need)))
            return TQ_ERR_ARG;
    if (overlap(dX, xb, workspace, need)) return TQ_ERR_ARG;
    int sms = 0;
    if (tq_status e = check_device(&sms)) return e;
    cudaStream_t st = cs(stream);
    __half *planes = reinterpret_cast<__half *>(workspace);
    const int64_t Np = bwd_plane_cols(N);
    float *inv_scale = reinterpret_cast<float *>(
        reinterpret_cast<uint8_t *>(workspace) + (((size_t)(kBwdPlanes * M * Np) * 2 + 255) & ~(size_t)255));
    const int per_row = (flags & TQ_GAMMA_PER_ROW) ? 1 : 0;
    const unsigned sgrid = (unsigned)(M < 8 * (int64_t)sms ? M : 8 * (int64_t)sms);  // one CTA per token row
    tq_status e = (N % 4 == 0)
                      ? launch_pdl(tq_bwd_split_kernel<true>, dim3(sgrid), dim3(kSplitThreads), 0, st, dY, gamma,
                                   per_row, (int)M, (int)N, (int)Np, planes, inv_scale)
                      : launch_pdl(tq_bwd_split_kernel<false>, dim3(sgrid), dim3(kSplitThreads), 0, st, dY, gamma,
                                   per_row, (int)M, (int)N, (int)Np, planes, inv_scale);
    if (e) return e;
    const int mode = enc << kModeEncShift;
    const int acc = (flags & TQ_FLAG_ACCUMULATE) ? 1 : 0;
    return enc != kEncFoundry
               ? launch_bwd_gemm<true>(planes, inv_scale, packed, row_scale, acc, M, N, K, dX, mode, sms, st)
               : launch_bwd_gemm<false>(planes, inv_scale, packed, row_scale, acc, M, N, K, dX, mode, sms, st);
}

tq_status tq_ste_backward(const float *grad, const float *w, const float *gamma, int64_t N, int64_t K,
                          float tau, unsigned flags, float *out, tq_stream_t stream) {
    if (!grad || !w || !gamma || !out) return TQ_ERR_NULL;
    if (N < 1) return TQ_ERR_SHAPE;
    if (tq_status e = check_k(K)) return e;
    if (flags & ~(TQ_GAMMA_PER_ROW | TQ_FLAG_SANITIZE_NONFINITE)) return TQ_ERR_ARG;
    if (!(tau >= 0.0f)) return TQ_ERR_ARG;
    if (!aligned16(grad) || !aligned16(w) || !aligned16(gamma) || !aligned16(out)) return TQ_ERR_ALIGN;
    const size_t nb = (size_t)(N * K) * 4, gb = ((flags & TQ_GAMMA_PER_ROW) ? (size_t)N : 1) * 4;
    // in place on grad or on w is allowed; any other overlap is not
    if ((out != grad && overlap(out, nb, grad, nb)) || (out != w && overlap(out, nb, w, nb)) ||
        overlap(out, nb, gamma, gb))
        return TQ_ERR_ARG;
    int sms = 0;
    if (tq_status e = check_device(&sms)) return e;
    const int64_t nvec = N * K / 4;
    const int64_t g64 = (nvec + kSteThreads - 1) / kSteThreads;
    const unsigned grid = (unsigned)(g64 < 8 * (int64_t)sms ? g64 : 8 * (int64_t)sms);
    const int per_row = (flags & TQ_GAMMA_PER_ROW) ? 1 : 0;
    const float4 *g4 = reinterpret_cast<const float4 *>(grad), *w4 = reinterpret_cast<const float4 *>(w);
    float4 *o4 = reinterpret_cast<float4 *>(out);
    return (flags & TQ_FLAG_SANITIZE_NONFINITE)
               ? launch_pdl(tq_ste_backward_kernel<true>, dim3(grid), dim3(kSteThreads), 0, cs(stream), g4, w4, gamma,
                            per_row, nvec, K / 4, tau, o4)
               : launch_pdl(tq_ste_backward_kernel<false>, dim3(grid), dim3(kSteThreads), 0, cs(stream), g4, w4,
                            gamma, per_row, nvec, K / 4, tau, o4);
}

void tq_seed(uint64_t *state, uint64_t seed) {
    if (state) *state = seed ? seed : 0x9E3779B97F4A7C15ull;
}

tq_status tq_ternary_stochastic_flip(uint8_t *packed, const float *grad, int64_t N, int64_t K,
                                     float temperature, uint64_t *rng_state, unsigned flags,
                                     tq_stream_t stream) {
    if (!packed || !grad || !rng_state) return TQ_ERR_NULL;
    if (N < 1) return TQ_ERR_SHAPE;
    if (tq_status e = check_k(K)) return e;
    if (N > ((int64_t)1 << 40) / K) return TQ_ERR_SHAPE;
    if (flags & ~TQ_ENC_MASK) return TQ_ERR_ARG;
    const int enc = flag_encoding(flags);
    if (enc < 0) return TQ_ERR_ARG;
    if (!(temperature >= 0.0f && temperature <= 3.4028235e38f)) return TQ_ERR_ARG;
    if (!aligned16(packed) || !aligned16(grad)) return TQ_ERR_ALIGN;
    const int64_t nw = N * K;
    if (overlap(packed, (size_t)(nw / 4), grad, (size_t)nw * 4)) return TQ_ERR_ARG;
    int sms = 0;
    if (tq_status e = check_device(&sms)) return e;
    const uint64_t x0 = *rng_state;
    const int mode = enc << kModeEncShift;
    tq_status e = enc != kEncFoundry ? launch_flip<true>(packed, grad, nw, temperature, x0, mode, sms, cs(stream))
                                     : launch_flip<false>(packed, grad, nw, temperature, x0, mode, sms, cs(stream));
    if (e) return e;
    *rng_state = xs_jump(x0, nw);
    return TQ_OK;
}

size_t tq_grouped_workspace_bytes(int64_t G, int64_t M, int64_t K, unsigned flags) {
    if (G <= 0 || M <= 0 || K <= 0) return 0;
    size_t off[3];
    return grouped_parts((flags & TQ_FLAG_SHARED_INPUT) ? 1 : G, M, K, off);
}

tq_status tq_bitlinear_grouped(const float *x, int64_t G, const uint8_t *const *packed, const float *const *gamma,
                               unsigned flags, int64_t M, int64_t N, int64_t K, float *y, void *workspace,
                               size_t workspace_bytes, tq_stream_t stream) {
    if (!x || !packed || !gamma || !y || !workspace) return TQ_ERR_NULL;
    if (G < 1 || G > kGroupMax || M < 1 || M > 16 || N < 1 || N > INT32_MAX) return TQ_ERR_SHAPE;
    if (tq_status e = check_k(K)) return e;
    if (K > kGemvMaxK) return TQ_ERR_SHAPE;
    if (flags & ~(TQ_GAMMA_PER_ROW | TQ_FLAG_SHARED_INPUT | TQ_FLAG_WEIGHTS_STATIC | TQ_FLAG_INPUTS_READY |
                  TQ_ENC_MASK))
        return TQ_ERR_ARG;
    const int enc = flag_encoding(flags);
    if (enc < 0) return TQ_ERR_ARG;
    const bool shared = flags & TQ_FLAG_SHARED_INPUT;
    const int64_t Gx = shared ? 1 : G;
    for (int64_t g = 0; g < G; ++g)
        if (!packed[g] || !gamma[g]) return TQ_ERR_NULL;
    if (!aligned16(x) || !aligned16(y) || !aligned16(workspace)) return TQ_ERR_ALIGN;
    for (int64_t g = 0; g < G; ++g)
        if (!aligned16(packed[g]) || !aligned16(gamma[g])) return TQ_ERR_ALIGN;
    size_t off[3];
    const size_t need = grouped_parts(Gx, M, K, off);
    if (workspace_bytes < need) return TQ_ERR_ARG;
    const size_t xb = (size_t)(Gx * M * K) * 4, yb = (size_t)(G * M * N) * 4, pb = (size_t)(N * K / 4),
                 gb = ((flags & TQ_GAMMA_PER_ROW) ? (size_t)N : 1) * 4;
    if (overlap(x, xb, y, yb) || overlap(x, xb, workspace, need) || overlap(y, yb, workspace, need)) return TQ_ERR_ARG;
    for (int64_t g = 0; g < G; ++g)
        if (overlap(packed[g], pb, y, yb) || overlap(packed[g], pb, workspace, need) ||
            overlap(gamma[g], gb, y, yb) || overlap(gamma[g], gb, workspace, need))
            return TQ_ERR_ARG;
    int sms = 0;
    if (tq_status e = check_device(&sms)) return e;
    cudaStream_t st = cs(stream);
    uint8_t *ws = reinterpret_cast<uint8_t *>(workspace);
    int8_t *xq = reinterpret_cast<int8_t *>(ws + off[0]);
    float *sx = reinterpret_cast<float *>(ws + off[1]);
    int32_t *rs = reinterpret_cast<int32_t *>(ws + off[2]);

    GroupPlan pl{};
    pl.M = (int)M;
    pl.K = (int)K;
    pl.N = N;
    pl.spp = (N + 15) / 16;
    pl.nstrips = G * pl.spp;
    pl.x_shared = shared ? 1 : 0;
    pl.per_row = (flags & TQ_GAMMA_PER_ROW) ? 1 : 0;
    pl.weights_static = (flags & (TQ_FLAG_WEIGHTS_STATIC | TQ_FLAG_INPUTS_READY)) ? 1 : 0;
    pl.enc = enc;
    const int NB = M <= 8 ? 1 : 2;
    if (!grp_plan(pl, NB, kGroupSmemBudget)) return TQ_ERR_SHAPE;
    GroupTable tab{};
    for (int64_t g = 0; g < G; ++g) {
        tab.packed[g] = packed[g];
        tab.gamma[g] = gamma[g];
    }
    ActParams p{};
    p.ready = (flags & TQ_FLAG_INPUTS_READY) ? 1 : 0;
    if (tq_status e = launch_act_group(x, p, Gx * M, K, xq, sx, rs, st)) return e;
    if (tq_status e = NB == 1 ? launch_group_gemv_enc<1>(tab, pl, xq, sx, rs, y, sms, st)
                              : launch_group_gemv_enc<2>(tab, pl, xq, sx, rs, y, sms, st))
        return e;
    return launch_status();
}

tq_status tq_selftest_wait_timeout(uint64_t limit_ns, int sleeping, tq_stream_t stream) {
    if (limit_ns < 1000 || limit_ns > 1000000000ull) return TQ_ERR_ARG;
    if (sleeping != 0 && sleeping != 1) return TQ_ERR_ARG;
    if (tq_status e = check_device(nullptr)) return e;
    return launch_pdl(tq_selftest_wait_kernel, dim3(1), dim3(32), 0, cs(stream), (unsigned long long)limit_ns,
                      sleeping);
}

tq_status tq_get_device_status(tq_stream_t stream) {
    if (cudaStreamSynchronize(cs(stream)) != cudaSuccess) return TQ_ERR_CUDA;
    unsigned v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, tq::g_status, sizeof v) != cudaSuccess) return TQ_ERR_CUDA;
    if (v && cudaMemcpyToSymbol(tq::g_status, &zero, sizeof zero) != cudaSuccess) return TQ_ERR_CUDA;
    return (v & tq::kStatusTimeout) ? TQ_ERR_TIMEOUT : TQ_OK;
}

}  // extern "C"

// ===========================================================================
// Allocation-free variant of tq_quantize_ternary_pack.
//
// Per-tensor gamma needs scratch for the partial sums of |w|; the regular entry
// point takes it from the caller.  Some callers cannot provide it: a runtime
// whose allocator has reserved all device memory up front and forbids new
// reservations, a host that only holds device pointers handed to it by someone
// else and has no allocator of its own, or code on a path where a cudaMalloc
// (which may synchronise the device) is not allowed.  This variant keeps that
// scratch in a fixed array compiled into the library instead.
//
// Limits and sharing rules:
//   * the array holds kNoAllocSlots partial sums of kNoAllocChunk float4 each,
//     so per-tensor gamma is limited to N*K <= kNoAllocMaxElems weights
//     (134,217,728, e.g. 8192 x 16384); larger calls return TQ_ERR_SHAPE
//     before launching anything.  Per-row gamma needs no scratch and has no
//     extra limit.
//   * every GPU that loads the library holds the array (16 KB: one fp64
//     partial sum per slot) until the process exits.
//   * all calls share the one array: calls whose work overlaps on the GPU (for
//     example on two streams at once) race and give wrong results.  Each call
//     writes every slot it reads before reading it, so nothing needs clearing
//     and leftovers from a previous call are harmless.
//   * the device address of the array is looked up (cudaGetSymbolAddress) on
//     the first call made on each device, with that device current; make that
//     first call before capturing work into a CUDA graph.
// ===========================================================================
namespace {

constexpr int kNoAllocSlots = 2048;
constexpr int64_t kNoAllocChunk = 16384;  // float4 per partial sum (65,536 weights)
constexpr int64_t kNoAllocMaxElems = (int64_t)kNoAllocSlots * kNoAllocChunk * 4;
constexpr size_t kNoAllocBytes = (size_t)kNoAllocSlots * sizeof(double);  // tq_absum_partial_kernel's output

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

void *g_noalloc_addr[kMaxDevices];
std::mutex g_noalloc_mu;

// Device address of g_noalloc_scratch on the current device (looked up once).
tq_status noalloc_scratch_addr(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return TQ_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return TQ_ERR_DEVICE;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (g_noalloc_addr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
            return TQ_ERR_CUDA;
        g_noalloc_addr[dev] = p;
    }
    *out = g_noalloc_addr[dev];
    return TQ_OK;
}

}  // namespace

extern "C" tq_status tq_quantize_ternary_pack_noalloc(const float *w, int64_t N, int64_t K,
                                                     unsigned flags, uint8_t *packed,
                                                     float *gamma, tq_stream_t stream) {
    if (!w || !packed || !gamma) return TQ_ERR_NULL;
    if (N < 1 || N > INT32_MAX) return TQ_ERR_SHAPE;
    if (tq_status e = check_k(K)) return e;
    if (flags & ~(TQ_GAMMA_PER_ROW | TQ_FLAG_SANITIZE_NONFINITE | TQ_ENC_MASK)) return TQ_ERR_ARG;
    const int enc = flag_encoding(flags);
    if (enc < 0) return TQ_ERR_ARG;
    const bool per_row = flags & TQ_GAMMA_PER_ROW;
    if (!per_row && N * K > kNoAllocMaxElems) return TQ_ERR_SHAPE;
    if (!aligned16(w) || !aligned16(packed) || !aligned16(gamma)) return TQ_ERR_ALIGN;
    const size_t wbytes = (size_t)(N * K) * 4, pbytes = (size_t)(N * K / 4),
                 gbytes = (per_row ? (size_t)N : 1) * 4;
    if (overlap(w, wbytes, packed, pbytes) || overlap(w, wbytes, gamma, gbytes) ||
        overlap(packed, pbytes, gamma, gbytes))
        return TQ_ERR_ARG;
    if (tq_status e = check_device(nullptr)) return e;
    const int sanitize = (flags & TQ_FLAG_SANITIZE_NONFINITE) ? 1 : 0;
    cudaStream_t st = cs(stream);
    if (per_row) {
        if (tq_status e = launch_pack_rows(w, N, K, sanitize, packed, gamma, PerTensor{}, 0, pack_opts(0, enc),
                                           0.0f, st))
            return e;
        return launch_status();
    }
    void *scratch = nullptr;
    if (tq_status e = noalloc_scratch_addr(&scratch)) return e;
    const int64_t total_v = N * K / 4;
    const int64_t nparts = (total_v + kNoAllocChunk - 1) / kNoAllocChunk;  // <= kNoAllocSlots
    double *partial = reinterpret_cast<double *>(scratch);
    if (tq_status e = launch_pdl(tq_absum_partial_kernel, dim3((unsigned)nparts), dim3(kPackThreads), 0,
                                 st, w, total_v, kNoAllocChunk, sanitize, partial, 0))
        return e;
    PerTensor pt;
    pt.partial = partial;
    pt.nparts = (int)nparts;
    pt.height = absum_tree_height(kNoAllocChunk, (int)nparts);
    if (tq_status e = launch_pack_rows(w, N, K, sanitize, packed, gamma, pt, 1, pack_opts(0, enc), 0.0f, st))
        return e;
    return launch_status();
}
