/*
 * tq.h -- C ABI of libtq, a B200 (sm_100a) implementation of the ternary
 * (BitNet b1.58 style) linear layer.
 *
 *   weights:     gamma = mean|w| (per tensor, or per output row),
 *                q = clamp(round(w / gamma), -1, 1), packed 2 bits per value,
 *                four per byte, LSB first, -1 = 0b00, 0 = 0b01, +1 = 0b10.
 *   activations: per token, eta = max|x| (>= 1e-6), x_q = clamp(round(x * 127/eta),
 *                -127, 127), s_x = eta / 127.
 *   output:      y[m][n] = (sum_k x_q[m][k] * q[n][k]) * gamma_n * s_x[m].
 *   optional prologue: RMSNorm, then a blockwise 512-point fast Walsh-Hadamard
 *                rotation, before the activation quantisation.
 *
 * Sources (page title, section):
 *   Foundry, docs/quantization.md: "Ternary Format / Encoding" (bit codes and
 *     byte layout), "Ternary Quantization (BitNet b1.58) / How It Works"
 *     (absmean gamma, round and clamp, add/subtract matmul scaled by gamma).
 *   Hetman-2b, src/quantization.py: section 1 (FWHT B=512), section 2
 *     (AbsmeanWeightQuantizer, SymmetricActivationQuantizer), section 4
 *     (SubLayerRMSNorm), section 5 (BitLinear.forward and export_packed_weights),
 *     section 7 (simulate_hardware_bitnet_gemv).
 *
 * Conventions for every entry point
 *   - All array arguments are DEVICE pointers on the current CUDA device, owned
 *     by the caller; the library allocates nothing on these paths.  Work is
 *     enqueued on `stream` (NULL = legacy default stream) and the call returns
 *     without waiting for it.
 *   - Layouts are row-major and dense: W / x are [rows][K] with K contiguous;
 *     packed weights are [N][K/4] bytes; y is [M][N].
 *   - Every pointer must be 16-byte aligned (TQ_ERR_ALIGN otherwise).
 *   - Shape rules: 1 <= M, N; 64 <= K <= 65536 and K % 64 == 0 (the packed row
 *     of K/4 bytes is then a whole number of 16-byte vectors); K % 512 == 0
 *     when the FWHT is requested.  Violations return TQ_ERR_SHAPE.
 *   - Arguments are checked before anything is enqueued: a call that returns an
 *     error has launched nothing and written nothing.  Launch failures return
 *     TQ_ERR_CUDA.  Waits inside kernels are bounded; a wait that gives up
 *     records TQ_ERR_TIMEOUT in a per-device status word read (and cleared) by
 *     tq_get_device_status().
 *   - Inputs and outputs must not overlap, except where an entry point says so.
 *   - Non-finite inputs give unspecified (but memory-safe) results unless
 *     TQ_FLAG_SANITIZE_NONFINITE is set.
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define TQ_API __attribute__((visibility("default")))
#else
#define TQ_API
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *tq_stream_t;

typedef enum tq_status {
    TQ_OK = 0,
    TQ_ERR_NULL = 1,    /* a required pointer is NULL                        */
    TQ_ERR_SHAPE = 2,   /* a size is out of range or breaks a divisibility rule */
    TQ_ERR_ALIGN = 3,   /* a pointer is not 16-byte aligned                   */
    TQ_ERR_ARG = 4,     /* unknown flag, overlap, or workspace too small      */
    TQ_ERR_CUDA = 5,    /* a CUDA runtime call or a kernel launch failed      */
    TQ_ERR_DEVICE = 6,  /* the current device is not compute capability 10.0  */
    TQ_ERR_TIMEOUT = 7  /* a bounded wait inside a kernel gave up             */
} tq_status;

/* flags */
#define TQ_GAMMA_PER_ROW (1u << 0)           /* one gamma per output row (else one per tensor) */
#define TQ_FLAG_FWHT (1u << 1)               /* blockwise FWHT-512 before act. quantisation    */
#define TQ_FLAG_RMSNORM (1u << 2)            /* RMSNorm before the FWHT                        */
#define TQ_FLAG_ETA_CLAMP (1u << 3)          /* clamp eta to [eta_min, eta_max]                */
#define TQ_FLAG_SANITIZE_NONFINITE (1u << 4) /* quench NaN / +-Inf inputs first                */
#define TQ_FLAG_WEIGHTS_STATIC (1u << 5)     /* see "Launch overlap" below                      */
#define TQ_FLAG_INPUTS_READY (1u << 6)       /* see "Launch overlap" below                      */
#define TQ_FLAG_ACCUMULATE (1u << 9)         /* tq_ternary_backward_input: dX += result         */
#define TQ_FLAG_SHARED_INPUT (1u << 10)      /* tq_bitlinear_grouped: one x for all G layers    */

/* Packed-code layout (flag bits 7-8; tq_quantize_ternary_pack[_noalloc],
 * tq_ternary_gemm, tq_bitlinear_fused).  Four codes per byte, LSB first.
 *   TQ_ENC_FOUNDRY  -1 = 0b00, 0 = 0b01, +1 = 0b10 (Foundry, docs/quantization.md,
 *                   "Ternary Format / Encoding"; the default; 0b11 is never
 *                   produced and undefined on input).
 *   TQ_ENC_FORMAT0  0 = 0b00, +1 = 0b01, -1 = 0b11, 0b10 reads as 0 (Hetman-2b,
 *                   src/quantization.py, section 3, "Format 0").
 *   TQ_ENC_FORMAT1  0 = 0b00, +1 = 0b01, -1 = 0b10, 0b11 reads as 0 (same, "Format 1").
 * A contraction must be given the layout its weights were packed in.  The
 * value 3 << 7 is rejected (TQ_ERR_ARG). */
#define TQ_ENC_FOUNDRY (0u << 7)
#define TQ_ENC_FORMAT0 (1u << 7)
#define TQ_ENC_FORMAT1 (2u << 7)
#define TQ_ENC_MASK (3u << 7)

/*
 * Launch overlap.  Every kernel is launched with programmatic dependent launch:
 * it may be scheduled while earlier kernels on the stream are still finishing,
 * and waits for the previous kernel's completion before reading or writing
 * any buffer.  "In flight" below means: enqueued on the stream since the last
 * point at which the stream was drained (a host synchronisation, an event
 * wait, the start of a CUDA graph launch).
 *
 * TQ_FLAG_WEIGHTS_STATIC (tq_ternary_gemm, tq_bitlinear_fused): the caller
 * promises that no work in flight writes the packed weights or gamma (true for
 * the layers of a model during inference).  The small-M GEMV then starts
 * streaming weights and gamma before the wait.
 *
 * TQ_FLAG_INPUTS_READY (tq_ternary_gemm, tq_quantize_ternary_pack,
 * tq_quantize_act_int8, tq_bitlinear_fused): the caller promises that no work
 * in flight writes any input of the call or reads or writes its outputs or
 * workspace -- e.g. the independent projections of one decode step that share
 * an activation (q/k/v, gate/up), each with its own output, or the packing of
 * a model's layers, each with its own buffers.  The first kernel of the call
 * then reads and computes at once and waits for the previous kernel only
 * before it exits, so any later call still sees every earlier result (it
 * implies TQ_FLAG_WEIGHTS_STATIC).  For the small-M contraction it also
 * selects a narrow streaming grid built for many such calls in flight; a
 * lone call is quicker without the flag.  Without either flag nothing is read
 * early.  A flagged call may still be running while later calls on the stream
 * start, so its buffers must not be recycled by a stream-ordered allocator
 * (which assumes that work on one stream runs in order) until the stream has
 * been drained.
 */

/*
 * Absmean ternarisation and 2-bit packing of an fp32 weight matrix.
 * Foundry docs/quantization.md, "How It Works" steps 1-3 and "Ternary Format /
 * Encoding"; Hetman-2b section 5 BitLinear.export_packed_weights; the per-row
 * variant is Foundry's per-channel granularity (fq_quantize_ternary_per_channel).
 *
 *   w       [N][K] fp32, read only.
 *   flags   TQ_GAMMA_PER_ROW, TQ_FLAG_SANITIZE_NONFINITE (nan -> 0,
 *           +-inf -> +-1 before anything else, Hetman-2b section 2),
 *           TQ_FLAG_INPUTS_READY (see "Launch overlap").
 *   packed  [N][K/4] bytes, written: byte j of row n holds codes 4j..4j+3 in bits
 *           (0,1) (2,3) (4,5) (6,7); 0b11 is never produced.
 *   gamma   [N] (per row) or [1] (per tensor) fp32, written: the fp32 nearest to
 *           the exact mean of |w| (ties to even), then max(., 1e-6).
 *   workspace / workspace_bytes: device scratch of at least
 *           tq_pack_workspace_bytes(N, K, flags) bytes (0 for per-row gamma, where
 *           workspace may be NULL).  Contents on entry are ignored.
 * Codes: q = +1 iff the fp32 quotient w / gamma rounds (half to even) above 0.5,
 * -1 iff below -0.5, else 0.
 */
TQ_API tq_status tq_quantize_ternary_pack(const float *w, int64_t N, int64_t K, unsigned flags,
                                   uint8_t *packed, float *gamma, void *workspace,
                                   size_t workspace_bytes, tq_stream_t stream);

/* Scratch bytes tq_quantize_ternary_pack needs for these arguments (the same
 * for tq_quantize_ternary_pack_threshold). */
TQ_API size_t tq_pack_workspace_bytes(int64_t N, int64_t K, unsigned flags);

/*
 * Threshold ternarisation with the same gamma: tau = fp32(ratio * gamma),
 * code = +1 if w > tau, -1 if w < -tau, else 0 (strict).  Foundry,
 * docs/quantization.md, "Absmean Thresholding (BitNet b1.58)" is ratio = 1
 * (threshold = mean |w|, scale = threshold); BitRASP, core_math.py,
 * ternarize_weight is ratio = 0.55 with TQ_GAMMA_PER_ROW (scale = the row's
 * mean |w|).  Arguments, flags, layout, workspace and errors as for
 * tq_quantize_ternary_pack; ratio must lie in (0, 64] (else TQ_ERR_ARG).
 */
TQ_API tq_status tq_quantize_ternary_pack_threshold(const float *w, int64_t N, int64_t K,
                                             unsigned flags, float ratio, uint8_t *packed,
                                             float *gamma, void *workspace,
                                             size_t workspace_bytes, tq_stream_t stream);

/*
 * Ternarisation with a manual (absolute) threshold, and 2-bit packing.
 * Foundry, docs/quantization.md, "Ternary Quantization":
 * fq_quantize_ternary_threshold(weights, shape, 2, 0.05f) ("Or with manual
 * threshold"), read with the page's "Absmean Thresholding (BitNet b1.58)"
 * rule with the caller's threshold t in place of mean |w|:
 *
 *   q = +1 if w > t, -1 if w < -t, else 0 (strict);  gamma[0] = t (the scale).
 *
 *   w, N, K, packed, stream: as for tq_quantize_ternary_pack.
 *   gamma      [1] fp32, written: t.
 *   threshold  t >= 0 and finite (else TQ_ERR_ARG); t = 0 gives sign(w).
 *   flags      TQ_FLAG_SANITIZE_NONFINITE, TQ_FLAG_INPUTS_READY, TQ_ENC_*.
 * One pass over W (no reduction, no workspace).
 */
TQ_API tq_status tq_quantize_ternary_pack_abs_threshold(const float *w, int64_t N, int64_t K, unsigned flags,
                                                        float threshold, uint8_t *packed, float *gamma,
                                                        tq_stream_t stream);

/*
 * Same result as tq_quantize_ternary_pack, for callers that cannot allocate
 * device memory (a runtime whose allocator owns all of HBM and refuses new
 * reservations, a host that only receives device pointers, or a path where a
 * cudaMalloc and the synchronisation it may cause are not allowed).  It takes
 * no workspace: the per-tensor partial sums live in a fixed 16 KB array inside
 * the library, held on every GPU that loads it until the process exits.  The
 * pages have no counterpart of this entry point; it only moves scratch memory.
 *
 *   w, N, K, packed, gamma, stream: as for tq_quantize_ternary_pack.
 *   flags: TQ_GAMMA_PER_ROW, TQ_FLAG_SANITIZE_NONFINITE and the layout bits
 *   TQ_ENC_*, as for tq_quantize_ternary_pack.  TQ_FLAG_INPUTS_READY is
 *   rejected (TQ_ERR_ARG): a call must not overlap the one before it, which
 *   may still be using the shared array.
 *   Limit: with per-tensor gamma, N * K <= 134,217,728 weights (2048 partial
 *   sums of 65,536 weights); larger calls return TQ_ERR_SHAPE and launch
 *   nothing.  Per-row gamma uses no scratch and has no extra limit.
 *   Sharing: every call uses the same array, so calls whose work overlaps on the
 *   GPU (e.g. on two streams at once) race; serialise them.  Each call writes
 *   the scratch before reading it, so nothing needs clearing between calls.
 *   Set-up: the first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before capturing work into a CUDA graph.
 */
TQ_API tq_status tq_quantize_ternary_pack_noalloc(const float *w, int64_t N, int64_t K,
                                                  unsigned flags, uint8_t *packed, float *gamma,
                                                  tq_stream_t stream);

/*
 * Per-token symmetric int8 quantisation.
 * Hetman-2b section 2 SymmetricActivationQuantizer.forward (reduction over the
 * last dimension); s_x = eta / 127 is the scale the output is multiplied by.
 *
 *   x       [M][K] fp32, read only.
 *   flags   TQ_FLAG_ETA_CLAMP (eta clamped to [eta_min, eta_max] after the 1e-6
 *           floor), TQ_FLAG_SANITIZE_NONFINITE (nan -> 0, +-inf -> +-eta_max),
 *           TQ_FLAG_INPUTS_READY (see "Launch overlap").
 *   xq      [M][K] int8, written, values in [-127, 127].
 *   s_x     [M] fp32, written.
 *   rowsum  [M] int32, written: sum_k xq[m][k].  tq_ternary_gemm needs it.
 */
TQ_API tq_status tq_quantize_act_int8(const float *x, int64_t M, int64_t K, unsigned flags,
                               float eta_min, float eta_max, int8_t *xq, float *s_x,
                               int32_t *rowsum, tq_stream_t stream);

/*
 * Blockwise fast Walsh-Hadamard transform over 512-element blocks of each row,
 * fp32: stages h = 1, 2, ..., 256 of (a + b, a - b), then, if normalize != 0,
 * a multiply by the fp32 value of 1/sqrt(512).  Hetman-2b section 1
 * (fast_walsh_hadamard_transform_512, blockwise_fwht_forward).
 *
 *   x  [rows][K] fp32 (K % 512 == 0), read;  y [rows][K] fp32, written.
 *   y == x (in place) is allowed; any other overlap is not.
 * Results are bit-identical to that stage order.
 */
TQ_API tq_status tq_fwht512(const float *x, float *y, int64_t rows, int64_t K, int normalize,
                     tq_stream_t stream);

/*
 * Ternary x int8 contraction with the fp32 rescale fused in its epilogue.
 * Hetman-2b section 5 steps 5-6 and section 7; Foundry "Native Matmul Kernel".
 *
 *   xq, s_x, rowsum  quantised activations as written by tq_quantize_act_int8
 *                    ([M][K] int8, [M] fp32, [M] int32).
 *   packed, gamma    as written by tq_quantize_ternary_pack ([N][K/4], [N] or [1]).
 *   flags            TQ_GAMMA_PER_ROW selects gamma[N] (else gamma[0]);
 *                    TQ_FLAG_WEIGHTS_STATIC, TQ_FLAG_INPUTS_READY as described
 *                    under "Launch overlap".
 *   y                [M][N] fp32, written: y = fp32(acc) * (gamma_n * s_x[m]).
 *   acc              [M][N] int32 or NULL: if given, the exact integer sums
 *                    acc[m][n] = sum_k xq[m][k] * q[n][k] are written too.
 * M <= 16 runs an HBM-bound GEMV; larger M runs a tcgen05 int8 tensor-core GEMM.
 */
TQ_API tq_status tq_ternary_gemm(const int8_t *xq, const float *s_x, const int32_t *rowsum,
                          const uint8_t *packed, const float *gamma, unsigned flags,
                          int64_t M, int64_t N, int64_t K, float *y, int32_t *acc,
                          tq_stream_t stream);

/*
 * tq_ternary_gemm with the pages' other epilogues.
 *   bias      [N] fp32 or NULL: y = acc * gamma * s_x + bias[n] (Hetman-2b
 *             section 5, BitLinear.forward, "y_out + self.bias").
 *   acc_bias  [N] int32 or NULL, out_shift in [0, 31]: the int32 output becomes
 *             (acc + acc_bias[n]) >> out_shift, an arithmetic shift (BitRASP,
 *             core_math.py, additive_ternary_linear_int8: acc += bias[o];
 *             acc >>= out_shift).  Applies to `acc` only; y uses the plain sum.
 * Other arguments, flags and errors as for tq_ternary_gemm (bias and acc_bias
 * 16-byte aligned, not overlapping the outputs; out_shift outside [0, 31] is
 * TQ_ERR_ARG).  Small M runs the per-strip GEMV shapes even with
 * TQ_FLAG_INPUTS_READY.
 */
TQ_API tq_status tq_ternary_gemm_ex(const int8_t *xq, const float *s_x, const int32_t *rowsum,
                                    const uint8_t *packed, const float *gamma, unsigned flags,
                                    int64_t M, int64_t N, int64_t K, const float *bias,
                                    const int32_t *acc_bias, int out_shift, float *y, int32_t *acc,
                                    tq_stream_t stream);

/*
 * Whole layer on pre-packed weights: [quench] -> [RMSNorm] -> [FWHT-512] ->
 * per-token int8 -> contraction -> rescale.  Hetman-2b section 5
 * BitLinear.forward steps 0-6.
 *
 *   x           [M][K] fp32, read.
 *   rms_gain    [K] fp32 or NULL (unit gain); used with TQ_FLAG_RMSNORM.
 *   rms_eps     RMSNorm epsilon (1e-6 in the pages).
 *   eta_min/max used with TQ_FLAG_ETA_CLAMP (0.05 / 40 in the pages).
 *   flags       any of the TQ_* flags above.
 *   packed, gamma, M, N, K as for tq_ternary_gemm.
 *   y           [M][N] fp32, written.
 *   xq_out      [M][K] int8 or NULL; s_x_out [M] fp32 or NULL: if given, the
 *               quantised activations are left there.
 *   workspace   at least tq_fused_workspace_bytes(M, K, flags) bytes of device
 *               scratch (x_q, s_x, rowsum live there when xq_out / s_x_out are
 *               NULL).  Contents on entry are ignored.
 * RMSNorm sums squares in fp64; the FWHT and the quantiser are bit-identical to
 * the fp32 definitions.
 */
TQ_API tq_status tq_bitlinear_fused(const float *x, const float *rms_gain, float rms_eps,
                             float eta_min, float eta_max, unsigned flags,
                             const uint8_t *packed, const float *gamma, int64_t M, int64_t N,
                             int64_t K, float *y, int8_t *xq_out, float *s_x_out,
                             void *workspace, size_t workspace_bytes, tq_stream_t stream);

/* Scratch bytes tq_bitlinear_fused needs for these arguments. */
TQ_API size_t tq_fused_workspace_bytes(int64_t M, int64_t K, unsigned flags);

/*
 * The FWHT module's quantisation round trip.  Hetman-2b section 1,
 * FastWalshHadamardTransform.forward: per row of K, nan -> 0 and +-inf ->
 * +-eta_max, then x_rot = FWHT-512 (normalised) of every 512-block, eta =
 * max_k |x_rot| + 1e-5 clamped to [eta_min, eta_max] (the Hadamard gain
 * clamp; 0.05 and 40 on the page), x_q = clamp(round(x_rot * 127 / eta),
 * -127, 127) half to even, y = FWHT-512 of x_q * (eta / 127).  All in fp32, in
 * the definition's order (bit-identical to it).
 *
 *   x, y      [rows][K] fp32; y may equal x (in place), else no overlap.
 *   K         multiple of 512, at most 16384.
 *   eta_out   [rows] fp32 or NULL: each row's clamped eta (the module reports
 *             their mean).
 * Errors: TQ_ERR_SHAPE, TQ_ERR_ARG (eta bounds not 0 < min <= max < 3e38, or
 * overlap), TQ_ERR_ALIGN (16 bytes).
 */
TQ_API tq_status tq_fwht_roundtrip(const float *x, float *y, int64_t rows, int64_t K, float eta_min,
                                   float eta_max, float *eta_out, tq_stream_t stream);

/*
 * Clamped SwiGLU feed-forward block of three BitLinear layers.  Hetman-2b
 * section 6, SwiGLUClamped.forward: gate = SiLU(W_gate(x)), up = W_up(x),
 * y = W_down(clamp(gate * up, -clamp_val, +clamp_val)) (clamp_val 10 on the
 * page), every W_* a BitLinear as in tq_bitlinear_fused (with TQ_FLAG_FWHT,
 * which is required here, and TQ_FLAG_RMSNORM if given, eps 1e-6, unit gain).
 *
 *   x          [M][d_model] fp32.  d_model, d_ffn multiples of 512, at most 16384.
 *   gate_*, up_*   packed [d_ffn][d_model/4] and gamma; down_* packed
 *              [d_model][d_ffn/4] and gamma (all per row with TQ_GAMMA_PER_ROW,
 *              in the layout the flags name).
 *   y          [M][d_model] fp32, written.
 *   act_out    [M][d_ffn] fp32 or NULL: the clamped activation.
 *   workspace  tq_swiglu_workspace_bytes(M, d_model, d_ffn, flags) bytes.
 *              After the call it holds the block's intermediates, eight
 *              parts in this order, each starting on a 256-byte boundary:
 *              the gate/up input codes x_q [M][d_model] int8, their s_x [M]
 *              fp32 and rowsum [M] int32; the gate and up projections
 *              [M][d_ffn] fp32 each; the down projection's input codes
 *              [M][d_ffn] int8, s_x [M] fp32 and rowsum [M] int32.
 * flags: TQ_FLAG_FWHT (required), TQ_FLAG_RMSNORM, TQ_GAMMA_PER_ROW,
 * TQ_FLAG_SANITIZE_NONFINITE, TQ_FLAG_WEIGHTS_STATIC, TQ_ENC_*.  SiLU is
 * computed in fp32 (v / (1 + e^-v)), within a few ulp of its exact value.
 */
TQ_API tq_status tq_swiglu_mlp(const float *x, int64_t M, int64_t d_model, int64_t d_ffn, unsigned flags,
                               float clamp_val, const uint8_t *gate_packed, const float *gate_gamma,
                               const uint8_t *up_packed, const float *up_gamma, const uint8_t *down_packed,
                               const float *down_gamma, float *y, float *act_out, void *workspace,
                               size_t workspace_bytes, tq_stream_t stream);
TQ_API size_t tq_swiglu_workspace_bytes(int64_t M, int64_t d_model, int64_t d_ffn, unsigned flags);

/*
 * Grouped small-M layer: G independent layers of one shape (N x K, packed
 * weights and gamma of their own) applied to their activation batches in two
 * launches -- one activation pass (per-token int8, Hetman-2b section 2
 * SymmetricActivationQuantizer) over all batches, then one persistent GEMV
 * that streams every layer's packed weights back to back (Hetman-2b section 7
 * simulate_hardware_bitnet_gemv; Foundry "Native Matmul Kernel"):
 *
 *   y[g][m][n] = (sum_k x_q[g][m][k] * q_g[n][k]) * gamma_g[n or 0] * s_x[g][m]
 *
 * with x_q, s_x the per-token quantisation of x[g] (no RMSNorm, no FWHT, eta
 * floor 1e-6, no clamp).  For the independent projections of a decode step
 * (q/k/v or gate/up over one input: TQ_FLAG_SHARED_INPUT), the experts of a
 * mixture-of-experts layer, or any set of same-shape layers whose inputs are
 * ready together.  Each y[g] equals what tq_quantize_act_int8 followed by
 * tq_ternary_gemm computes for that layer.
 *
 *   x          [G][M][K] fp32, or [M][K] with TQ_FLAG_SHARED_INPUT.
 *   packed     HOST array of G device pointers, each [N][K/4] bytes in the
 *              layout the flags name; gamma: HOST array of G device
 *              pointers, each [N] (TQ_GAMMA_PER_ROW) or [1] fp32.  The arrays
 *              are read during the call only.
 *   y          [G][M][N] fp32, written.
 *   workspace  tq_grouped_workspace_bytes(G, M, K, flags) bytes, 16-byte
 *              aligned.  After the call it holds x_q [Gx][M][K] int8 (Gx = 1
 *              with TQ_FLAG_SHARED_INPUT, else G) with each 16-byte chunk c of a
 *              row stored 4x4-byte transposed (word j = elements 16c + j,
 *              16c + 4 + j, 16c + 8 + j, 16c + 12 + j) at chunk position
 *              c ^ (2 * ((c >> 3) & 1)), then s_x [Gx][M] fp32 and rowsum
 *              [Gx][M] int32, each part starting on a 256-byte boundary.
 *   Shapes: 1 <= G <= 64, 1 <= M <= 16, 64 <= K <= 8192 (K % 64 == 0);
 *   otherwise TQ_ERR_SHAPE.
 *   flags: TQ_GAMMA_PER_ROW, TQ_FLAG_SHARED_INPUT, TQ_FLAG_WEIGHTS_STATIC,
 *   TQ_FLAG_INPUTS_READY (see "Launch overlap"), TQ_ENC_*.
 */
TQ_API tq_status tq_bitlinear_grouped(const float *x, int64_t G, const uint8_t *const *packed,
                                      const float *const *gamma, unsigned flags, int64_t M, int64_t N,
                                      int64_t K, float *y, void *workspace, size_t workspace_bytes,
                                      tq_stream_t stream);
TQ_API size_t tq_grouped_workspace_bytes(int64_t G, int64_t M, int64_t K, unsigned flags);

/* ------------------------------------------------------------------------
 * Training
 * ------------------------------------------------------------------------ */

/*
 * Gradient with respect to the layer input.  Foundry, docs/quantization.md,
 * "Ternary Training (Backward Pass + Stochastic Flip) / Backward Pass",
 * fq_matmul_ternary_backward_input: for the forward Y = scale * X W_ternary,
 *
 *   dX[m][k] = (TQ_FLAG_ACCUMULATE ? dX[m][k] : 0)
 *            + row_scale[m] * sum_n fp32(dY[m][n] * gamma_n) * q[n][k]
 *
 * with the codes q of the packed weights [N][K/4] (the layout the flags
 * name) and gamma_n = gamma[n] (TQ_GAMMA_PER_ROW) or gamma[0].  The page's
 * "+=" form (caller zeroes d_input) is TQ_FLAG_ACCUMULATE.  row_scale (NULL
 * = 1) is a per-token factor: Hetman-2b's BitLinear scales the contraction
 * by gamma * s_x per token (section 5 step 6) and its activation STE passes
 * the gradient of x_q on unchanged (section 2), so row_scale = s_x gives
 * that gradient.  Each row of g = fp32(dY * gamma) is scaled by the power
 * of two that puts its largest |g| in [2^14, 2^15) and split into two fp16
 * parts (22 significant bits: error <= 2^-22 of each term, or 2^-39 of the
 * row's largest term), contracted on the tensor cores with fp32
 * accumulation and scaled back exactly (the result is within 1e-5 of
 * sum_n |g q| of the exact sum).
 *
 *   dY         [M][N] fp32.          dX [M][K] fp32 (written, or updated).
 *   workspace  tq_backward_input_workspace_bytes(M, N) bytes (two fp16
 *              planes of the scaled dY * gamma and one scale per token),
 *              16-byte aligned, owned by the caller.
 * K % 64 == 0, 64 <= K <= 65536; N >= 1; 1 <= M <= 1073741823.
 * flags: TQ_GAMMA_PER_ROW, TQ_FLAG_ACCUMULATE, TQ_ENC_*.
 * Errors: TQ_ERR_NULL, TQ_ERR_SHAPE, TQ_ERR_ALIGN (16 bytes), TQ_ERR_ARG
 * (flags, workspace too small, any overlap between dX or the workspace and
 * another buffer).
 */
TQ_API tq_status tq_ternary_backward_input(const float *dY, const uint8_t *packed, const float *gamma,
                                           const float *row_scale, unsigned flags, int64_t M, int64_t N,
                                           int64_t K, float *dX, void *workspace, size_t workspace_bytes,
                                           tq_stream_t stream);
TQ_API size_t tq_backward_input_workspace_bytes(int64_t M, int64_t N);

/*
 * Straight-through estimator of the latent weights.  Hetman-2b,
 * src/quantization.py, section 2, AbsmeanWeightQuantizer.backward:
 *
 *   out[n][k] = (grad[n][k] / gamma_n) * (|w[n][k] / gamma_n| <= tau ? 1 : 0.1)
 *
 * in fp32 as written (IEEE division; 0.1 is the fp32 constant).  The page
 * uses tau = 1 and one gamma per tensor; TQ_GAMMA_PER_ROW takes gamma[n].
 * TQ_FLAG_SANITIZE_NONFINITE applies the forward's quarantine to w first
 * (nan -> 0, +-inf -> +-1).
 *
 *   grad, w, out  [N][K] fp32; out may be grad or w (in place), no other overlap.
 * K % 64 == 0, 64 <= K <= 65536; N >= 1; tau >= 0.
 * Errors: TQ_ERR_NULL, TQ_ERR_SHAPE, TQ_ERR_ALIGN, TQ_ERR_ARG.
 */
TQ_API tq_status tq_ste_backward(const float *grad, const float *w, const float *gamma, int64_t N, int64_t K,
                                 float tau, unsigned flags, float *out, tq_stream_t stream);

/*
 * Stochastic ternary flip (replaces the optimiser).  Foundry,
 * docs/quantization.md, "Stochastic Weight Flip", fq_ternary_stochastic_flip:
 * for every weight i in storage order (row n, then k), one draw each,
 *
 *   x = xorshift64(state)      (x ^= x << 13; x ^= x >> 7; x ^= x << 17)
 *   u = (x >> 40) * 2^-24      (fp32, in [0, 1))
 *   p = min(|grad_i| * temperature, 1)   (fp32; a NaN gradient never flips)
 *   if u < p: q_i = clamp(q_i - sign(grad_i), -1, 1)
 *
 * packed [N][K/4] is updated in place in the layout the flags name (reserved
 * fields read as 0).  rng_state is a HOST pointer to the caller's 64-bit
 * state: the launch takes its value and the call advances it by N*K draws
 * before returning (the kernel may still be running).  The draws are those
 * of the sequential loop, bit for bit: each lane of the kernel starts its run
 * at the right point of the stream by jumping ahead with powers of the
 * generator's GF(2) matrix.  A CUDA graph that captures this call replays
 * the draws of the captured state.
 *
 *   grad  [N][K] fp32, not overlapping packed.
 * K % 64 == 0, 64 <= K <= 65536; N >= 1; N * K <= 2^40; 0 <= temperature < inf.
 * flags: TQ_ENC_*.  Errors: TQ_ERR_NULL, TQ_ERR_SHAPE, TQ_ERR_ALIGN, TQ_ERR_ARG.
 */
TQ_API tq_status tq_ternary_stochastic_flip(uint8_t *packed, const float *grad, int64_t N, int64_t K,
                                            float temperature, uint64_t *rng_state, unsigned flags,
                                            tq_stream_t stream);

/* fq_seed: state = seed, or 0x9E3779B97F4A7C15 for seed 0 (xorshift's fixed
 * point).  The page leaves the mapping open.  Host only; NULL is ignored. */
TQ_API void tq_seed(uint64_t *state, uint64_t seed);

/*
 * Self-test of the failure-detection path (no counterpart on the pages).  One
 * warp of a one-CTA kernel waits on a shared-memory mbarrier that nothing ever
 * completes, through the same bounded wait every kernel of the library uses
 * (spinning, or with sleeping = 1 the suspending form), gives up after
 * limit_ns nanoseconds of %globaltimer, records TQ_ERR_TIMEOUT in the
 * per-device status word and exits normally -- the context stays usable.  The
 * next tq_get_device_status() returns TQ_ERR_TIMEOUT and clears the word.
 *   limit_ns  in [1000, 1e9] (1 us .. 1 s), else TQ_ERR_ARG.
 *   sleeping  0 or 1, else TQ_ERR_ARG.
 */
TQ_API tq_status tq_selftest_wait_timeout(uint64_t limit_ns, int sleeping, tq_stream_t stream);

/*
 * Waits for `stream`, then returns and clears the current device's status word:
 * TQ_OK, or TQ_ERR_TIMEOUT if a bounded wait inside a kernel gave up since the
 * last call.  TQ_ERR_CUDA if the synchronisation itself failed.
 */
TQ_API tq_status tq_get_device_status(tq_stream_t stream);

/* Static, NUL-terminated description of a status code. */
TQ_API const char *tq_status_string(tq_status status);

/* Library version as major * 10000 + minor * 100 + patch. */
TQ_API int tq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */
