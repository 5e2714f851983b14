/*
 * bitnet.h -- C ABI of the B200 BitLinear (W1.58A8) library.
 *
 * The method (BitNet b1.58): a projection whose weights are ternary
 * {-1, 0, +1} times one per-tensor scale gamma = mean|W| ("absmean"), stored
 * four codes to a byte, and whose input is quantised per token to int8 with
 * scale s = 127 / max|x| ("absmax").  Its output is the integer contraction of
 * the two code matrices, dequantised by gamma / s.  Sources (web pages):
 *   - nnterp encyclopedia "bitnet", "The projections quantize their inputs and
 *     weights": per-token round(x * 127 / max|x|) to 255 levels; weights
 *     rounded to {-1, 0, 1} * mean|W|, stored ternary four to a byte with a
 *     weight_scale; the output equals the linear map of the rounded input by
 *     the ternarised weight exactly.
 *   - same page, "The block, in order", "The MLP gates with a squared ReLU",
 *     "Scaling inside a sublayer is undone by the sub-norm", "Config": the
 *     RMSNorm sub-norms (eps 1e-5) and the gated ReLU^2 FFN.
 *   - "BitNet b1.58 2B4T - Scaling Native 1-bit LLM", "Model Details": W1.58A8,
 *     absmean weights, per-token absmax int8 activations, no bias.
 *   - "bitnetv2-model" README, "Special Features" / "Architecture Overview":
 *     H-BitLinear (a Hadamard transform before the quantised linear, on
 *     power-of-two widths) and its 512 -> 2048 -> 512 SiLU FFN.
 *
 * Conventions shared by every call
 *   Pointers   All tensor pointers are DEVICE pointers owned by the caller.
 *              The library never allocates, frees or retains them.  Scratch
 *              space is passed in as `workspace`; its size comes from the
 *              matching *_workspace_size() call.
 *   Layout     Matrices are row-major with the contiguous dimension last:
 *              activations [M][K] (M tokens), weights [N][K] (N outputs,
 *              K inputs, the Linear(in=K, out=N) convention), outputs [M][N].
 *   Alignment  Every tensor pointer must be 16-byte aligned.
 *   Sizes      M, N >= 0 (0 is a no-op), K >= 16 and K % 16 == 0, K <= 16384.
 *   Streams    Every call is asynchronous and stream-ordered on `stream` (a
 *              cudaStream_t; NULL means the legacy default stream).  Nothing
 *              synchronises the host except bitnet_check_device_error().
 *   Errors     Every call returns a status code.  Arguments are validated on
 *              the host before any launch, so a call that returns
 *              BITNET_ERR_INVALID_ARG / _UNSUPPORTED / _WORKSPACE has no device
 *              side effect.  bitnet_last_error() gives a message (per host
 *              thread).  Device-side failures (a bounded wait that gave up)
 *              are recorded in a device error word that
 *              bitnet_check_device_error() reads.
 *   Inputs     Inputs must be finite; with NaN or Inf in an input the codes
 *              are unspecified.
 *   Launch     The quantiser and the prefill GEMM (M > 16) are launched with
 *              programmatic dependent launch: their CTAs may do on-chip setup
 *              while the preceding work on the stream finishes, and touch no
 *              global memory before that work has completed, so stream order
 *              is preserved whatever precedes them.
 *
 * Packed ternary layout (the pages fix only "four to a byte"; this layout is
 * this library's convention)
 *   A packed row holds bitnet_packed_row_bytes(K) = 16 * ceil(K / 64) bytes.
 *   Weight k of row n lives in byte  n * row_bytes + 4 * (k / 16) + (k % 4),
 *   at bits 2 * ((k % 16) / 4) and up, as the code c = t + 1 in {0, 1, 2}.
 *   So each little-endian 32-bit word holds 16 consecutive weights, and
 *   (word >> 2*i) & 0x03030303 yields the four codes of weights 4i..4i+3 of
 *   that group, one per byte.  Padding positions k >= K hold code 1 (t = 0).
 *   Code 3 is never written.  gamma is one fp32 in device memory.
 */
#ifndef BITNET_B200_H
#define BITNET_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---------------------------------------------------------------- status */
#define BITNET_OK               0
#define BITNET_ERR_INVALID_ARG  1  /* null pointer, bad size, misaligned pointer */
#define BITNET_ERR_UNSUPPORTED  2  /* a shape / flag combination not handled     */
#define BITNET_ERR_CUDA         3  /* a CUDA call or launch failed               */
#define BITNET_ERR_WORKSPACE    4  /* workspace missing or too small             */
#define BITNET_ERR_TIMEOUT      5  /* a bounded device-side wait gave up         */

/* ----------------------------------------------------------- element types */
#define BITNET_F32   0
#define BITNET_BF16  1
#define BITNET_I32   2

/* ---------------------------------------------------- activation preludes */
#define BITNET_PRELUDE_NONE     0
#define BITNET_PRELUDE_RMSNORM  1  /* x * g / sqrt(mean(x^2) + eps)             */
#define BITNET_PRELUDE_FWHT     2  /* normalised Walsh-Hadamard, K power of two */

/* ------------------------------------------------------ linear epilogues */
/* Low 4 bits: output element type (BITNET_F32 / BITNET_BF16 / BITNET_I32).
 * BITNET_I32 writes the raw int32 contraction sum_k q[m,k] * t[n,k]. */
#define BITNET_EPI_TYPE_MASK  0x0f
#define BITNET_EPI_RESIDUAL   0x10  /* y = residual[m][n] + y (residual has Y's type; F32/BF16) */
#define BITNET_EPI_SILU       0x20  /* y = silu(y) = y / (1 + exp(-y)) (F32/BF16)               */
/* Launch hint for the decode path (M <= 16): the kernel may start before the
 * preceding work on the stream has finished (programmatic dependent launch)
 * and stream its packed weights early; activation codes, scales, code sums,
 * gamma, residual and Y are touched only after that work has completed.  Set
 * it only when the preceding work does not write the packed weights, e.g. in
 * a decode loop over static weights.  For M > 16 (the prefill GEMM, always a
 * dependent launch) it lets the GEMM load its first weight tiles before the
 * preceding work has completed. */
#define BITNET_LAUNCH_PDL     0x100
/* Stronger launch hint for the decode path (implies BITNET_LAUNCH_PDL): the
 * preceding work on the stream writes none of this call's inputs (packed
 * weights, gamma, activation codes, scales, code sums, residual), as for the
 * q/k/v or gate/up projections of a decode step, which read one quantised
 * input.  Everything up to the output stores (loads, MMAs, the cross-CTA
 * reduction, dequantisation) may then overlap the preceding work; only the
 * writes of Y wait for it to finish.  Ignored for M > 16. */
#define BITNET_LAUNCH_PDL_INPUTS 0x200

/* ----------------------------------------------------------- FFN variants */
#define BITNET_FFN_RELU2_GLU      0  /* x + down(subnorm(relu(gate(z))^2 * up(z))), z = RMSNorm(x) */
#define BITNET_FFN_HADAMARD_SILU  1  /* W2 . silu(W1 . x), each projection an H-BitLinear          */
/* Launch option, OR-ed into the variant: run the decode-size GLU FFN (M <= 16,
 * H and I multiples of 128) as one persistent cooperative launch instead of
 * four launches (see bitnet_ffn).  It needs every SM at once, so callers
 * whose other kernels run concurrently should leave it off.  No effect on
 * other sizes or on the results' tolerance. */
#define BITNET_FFN_SINGLE_LAUNCH 0x200

typedef void *bitnet_stream_t;       /* a cudaStream_t */

#if defined(BITNET_BUILD) && defined(__GNUC__)
#define BITNET_API __attribute__((visibility("default")))
#else
#define BITNET_API
#endif

/* Bytes per packed weight row for K inputs: 16 * ceil(K / 64).  Pure host
 * function; returns 0 for K <= 0. */
BITNET_API size_t bitnet_packed_row_bytes(int K);

/* Workspace bytes bitnet_pack_weights() needs for an N x K weight. */
BITNET_API size_t bitnet_pack_workspace_size(int N, int K);

/* Ternarise and pack one weight matrix (nnterp "bitnet", "The projections
 * quantize their inputs and weights": weights rounded to {-1, 0, 1} *
 * mean|W| and stored four to a byte with a weight_scale).
 *   W         [N][K] row-major, element type w_dtype (BITNET_F32 or BITNET_BF16).
 *   packed    out: [N][bitnet_packed_row_bytes(K)] bytes in the layout above.
 *   gamma     out: one fp32 = mean|W| (accumulated in fp64, rounded once).
 *             Codes are t = clamp(rint(W / gamma), -1, 1) with IEEE fp32
 *             division and ties to even; gamma == 0 gives t = 0.
 *   workspace at least bitnet_pack_workspace_size(N, K) bytes, 16-B aligned.
 * Errors: INVALID_ARG (null, sizes, alignment), WORKSPACE, CUDA. */
BITNET_API int bitnet_pack_weights(const void *W, int w_dtype, int N, int K,
                        uint8_t *packed, float *gamma,
                        void *workspace, size_t ws_bytes, bitnet_stream_t stream);

/* The canonical exchange layout TW2 and this library's device layout.
 * TW2: [N][K/4] bytes, weight k of row n is the code t + 1 at bits 2 (k % 4)
 * of byte n K/4 + k/4 (four to a byte, [NN] "stored ternary, four to a byte";
 * low bits first is this library's convention).  bitnet_pack_weights() and
 * bitnet_linear() use the device layout above (16 codes per 32-bit word
 * arranged so that two ALU ops expand four of them); these two calls convert.
 *   packed  [N][bitnet_packed_row_bytes(K)] device layout.
 *   tw2     [N][K/4] TW2.  An input code 3 is invalid (unspecified result).
 * K must be a multiple of 16 in [16, 16384]; pointers 16-byte aligned; N = 0
 * is a no-op.  Errors: INVALID_ARG, CUDA. */
BITNET_API int bitnet_export_tw2(const uint8_t *packed, int N, int K, uint8_t *tw2,
                                 bitnet_stream_t stream);
BITNET_API int bitnet_import_tw2(const uint8_t *tw2, int N, int K, uint8_t *packed,
                                 bitnet_stream_t stream);

/* Per-token int8 absmax quantisation with an optional fused prelude
 * (nnterp "bitnet", same section: round(x * 127 / max|x|) per token; "BitNet
 * b1.58 2B4T", "Model Details": absmax per token; sub-norm RMSNorm, nnterp
 * "The block, in order"; Hadamard prelude, "bitnetv2-model" README).
 *   X         [M][K], element type x_dtype (BITNET_F32 or BITNET_BF16).
 *   prelude   BITNET_PRELUDE_*; FWHT needs K to be a power of two.
 *   norm_gain [K] fp32 RMSNorm gain, or NULL for all ones (RMSNORM only).
 *   eps       RMSNorm epsilon (1e-5 in the model).
 *   Xq        out: [M][K] int8 codes q = clamp(rint(xh * s), -128, 127).
 *   x_scale   out: [M] fp32 s = 127 / max|xh| (1 for an all-zero row).
 *   x_rowsum  out: [M] int32 sum_k q[m,k], or NULL to skip.
 * RMSNorm: r = 1/sqrt(mean(x^2) + eps) with the mean square accumulated in
 * fp64 and rounded once to fp32, xh = (x * r) * g in fp32.  FWHT: butterfly
 * stages h = 1, 2, ..., K/2 in that order, then one multiply by
 * fp32(1/sqrt(K)).  Errors: INVALID_ARG, CUDA. */
BITNET_API int bitnet_quant_act(const void *X, int x_dtype, int M, int K,
                     int prelude, const float *norm_gain, float eps,
                     int8_t *Xq, float *x_scale, int32_t *x_rowsum,
                     bitnet_stream_t stream);

/* The BitLinear contraction with its dequantising epilogue (nnterp "bitnet",
 * same section: the output equals the linear map of the rounded input by the
 * ternarised weight exactly).
 *   Xq, x_scale, x_rowsum  outputs of bitnet_quant_act() for the M tokens
 *             (x_rowsum is REQUIRED: the kernels multiply by the stored
 *             codes c = t + 1 and subtract sum_k q).
 *   packed, gamma          outputs of bitnet_pack_weights() for [N][K].
 *   Y         out: [M][N] of the type in (epilogue & BITNET_EPI_TYPE_MASK):
 *             y = fp32( acc * gamma / s[m] ), formed to ~2^-47 relative and
 *             rounded once (the correctly rounded value except within ~2^-46
 *             of an fp32 midpoint), then the optional SiLU / residual add in
 *             fp32, then the cast.
 *   residual  [M][N] of Y's type when BITNET_EPI_RESIDUAL is set, else NULL.
 * M <= 2 (K a multiple of 64), M <= 4 in a call without BITNET_LAUNCH_PDL_INPUTS
 * and K <= 4096, or M <= 8 with N K <= 2^20, runs a dp4a streaming GEMV, M <= 16
 * otherwise the cluster tensor-core GEMV (all HBM-bound), larger M the tcgen05
 * GEMM.
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA. */
BITNET_API int bitnet_linear(const int8_t *Xq, const float *x_scale, const int32_t *x_rowsum,
                  const uint8_t *packed, const float *gamma,
                  int M, int N, int K,
                  void *Y, int epilogue, const void *residual,
                  bitnet_stream_t stream);

/* Kernels of a launch plan (bitnet_plan_linear). */
#define BITNET_PLAN_STREAM   1  /* row-group dp4a streaming GEMV                 */
#define BITNET_PLAN_FLAT     2  /* flat dp4a streaming GEMV                      */
#define BITNET_PLAN_GEMV_TC  3  /* cluster split-K tensor-core GEMV              */
#define BITNET_PLAN_GEMV     4  /* plain dp4a GEMV (decode K the others refuse)  */
#define BITNET_PLAN_GEMM_TC  5  /* persistent tcgen05 GEMM                       */

/* The launch plan bitnet_linear() follows for one projection on a device with
 * `sms` SMs: host logic only (no launch, no device access), for tests and
 * tooling.  epilogue as bitnet_linear() (its flags choose the plan).
 *   out[0]  kernel, BITNET_PLAN_*
 *   out[1]  tokens per pass: decode kernels' token tile (1, 2, 4, 8, 16), the
 *           GEMM's tile (128, 96 or 64 tokens)
 *   out[2]  CTAs (the plain GEMV: before its occupancy cap)
 *   out[3], out[4]
 *           STREAM: lanes per row, warps per CTA; FLAT: rows per warp, bulk
 *           weight copies (0 / 1); GEMV_TC: cluster size, 128-row tiles;
 *           GEMM_TC: tiles, 0; GEMV: 0, 0
 * Errors: INVALID_ARG (out NULL, M, N or sms not positive, K as for
 * bitnet_linear()). */
BITNET_API int bitnet_plan_linear(int M, int N, int K, int epilogue, int sms, int *out);

/* Several projections of one quantised input in one call -- the q, k and v
 * projections of an attention block (2560 -> 2560 + 640 + 640 in the 2B
 * model, nnterp "bitnet", "Printout"), or gate and up -- as bitnet_linear()
 * for each, with one launch for all of them on the decode path (M <= 16).
 *   count       projections, 1..4
 *   packed[i], gamma[i], N[i], Y[i]
 *               weight i [N[i]][K] (device layout) with its gamma, and its
 *               output [M][N[i]]; host arrays of device pointers
 *   epilogue    as bitnet_linear() without BITNET_EPI_RESIDUAL
 * M > 16 runs the projections as consecutive prefill GEMMs.
 * Errors: INVALID_ARG, UNSUPPORTED (residual requested), CUDA. */
BITNET_API int bitnet_linear_multi(const int8_t *Xq, const float *x_scale,
                                   const int32_t *x_rowsum, int count,
                                   const uint8_t *const *packed, const float *const *gamma,
                                   const int *N, int M, int K, void *const *Y, int epilogue,
                                   bitnet_stream_t stream);

/* Workspace bytes bitnet_ffn() needs. */
BITNET_API size_t bitnet_ffn_workspace_size(int M, int H, int I, int variant);

/* One FFN built from BitLinear projections.
 * BITNET_FFN_RELU2_GLU (nnterp "bitnet", "The block, in order" and "The MLP
 * gates with a squared ReLU"):
 *   z = RMSNorm(x; pre_norm_gain, eps)              (post_attention_layernorm)
 *   m = relu(gate_proj(z))^2 * up_proj(z)           (fp32)
 *   Y = x + down_proj(RMSNorm(m; sub_norm_gain, eps))   (ffn_sub_norm)
 *   X, Y [M][H] of x_dtype / y_dtype (F32 or BF16); W_gate, W_up [I][H] and
 *   W_down [H][I] packed; gains may be NULL (all ones).
 *   Decode (M <= 16): four launches -- the RMSNorm quantiser, gate and up as
 *   two projections of one decode launch (fp32 outputs), the sub-norm
 *   quantiser forming m from them as it loads them (the workspace is then
 *   larger by M * I * 4 bytes), down with the residual.  With
 *   BITNET_FFN_SINGLE_LAUNCH (H and I multiples of 128) the whole FFN runs
 *   as one persistent cooperative launch with one CTA per SM (weights of
 *   every projection bulk-copied into shared memory at start, x quantised by
 *   every CTA, gate and up on mma.sync, one grid-wide exchange of m's sums of
 *   squares through the workspace, the sub-norm codes formed by every CTA,
 *   down with the residual); the exchange uses a fresh 64-bit epoch per
 *   launch, so the workspace needs no initialisation, and calls sharing a
 *   workspace must not overlap on the GPU.  Larger M runs the fused gate/up
 *   GEMM, whose epilogue forms m.
 * BITNET_FFN_HADAMARD_SILU ("bitnetv2-model" README, "Architecture
 * Overview"): Y = W2 . silu(W1 . x), each an H-BitLinear (FWHT prelude);
 *   W_gate = W1 [I][H], W_down = W2 [H][I], W_up / gamma_up must be NULL,
 *   H and I powers of two, gains and eps unused.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
BITNET_API int bitnet_ffn(const void *X, int x_dtype, int M, int H, int I,
               const uint8_t *W_gate, const float *gamma_gate,
               const uint8_t *W_up, const float *gamma_up,
               const uint8_t *W_down, const float *gamma_down,
               const float *pre_norm_gain, const float *sub_norm_gain, float eps,
               int variant, void *Y, int y_dtype,
               void *workspace, size_t ws_bytes, bitnet_stream_t stream);

/* Workspace bytes bitnet_block_tail() needs. */
BITNET_API size_t bitnet_block_tail_workspace_size(int M, int H, int I);

/* The part of a W1.58A8 block after attention, at decode sizes, in one
 * persistent launch (nnterp "bitnet", "The block, in order"):
 *   h = x + o_proj(attn_sub_norm(a))                       (h kept in fp32)
 *   Y = h + down_proj(ffn_sub_norm(relu(gate_proj(z))^2 * up_proj(z))),
 *       z = post_attention_layernorm(h)
 * every norm an RMSNorm with eps and a gain (NULL for all ones), every
 * projection a BitLinear ("The projections quantize their inputs and
 * weights").  A (attention output) and X (residual stream), H_out and Y are
 * [M][H] of `dtype` (F32 or BF16); W_o [H][H], W_gate, W_up [I][H], W_down
 * [H][I] packed.  H_out receives h in `dtype` (NULL to skip).
 * One cooperative launch, one CTA per SM, two bounded grid-wide exchanges
 * through the workspace (epochs, as bitnet_ffn at decode sizes): o_proj rows,
 * then gate/up features, then down rows split over the CTAs; the codes of a,
 * h and m formed by every CTA.  Supported: 1 <= M <= 16, H and I multiples
 * of 128, staged weights and codes within an SM's shared memory (for the 2B
 * model's 2560 / 6912, M <= 8); otherwise BITNET_ERR_UNSUPPORTED before any
 * launch -- compose bitnet_quant_act (RMSNorm), bitnet_linear (fp32 output
 * with the residual) and bitnet_ffn instead.  Calls sharing a workspace must
 * not overlap on the GPU.  Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
BITNET_API int bitnet_block_tail(const void *A, const void *X, int dtype, int M, int H, int I,
                                 const uint8_t *W_o, const float *gamma_o,
                                 const uint8_t *W_gate, const float *gamma_gate,
                                 const uint8_t *W_up, const float *gamma_up,
                                 const uint8_t *W_down, const float *gamma_down,
                                 const float *attn_norm_gain, const float *post_norm_gain,
                                 const float *sub_norm_gain, float eps, void *H_out, void *Y,
                                 void *workspace, size_t ws_bytes, bitnet_stream_t stream);

/* bitnet_ffn without a workspace argument, for callers that cannot allocate
 * device memory: code running inside a CUDA stream capture whose mode forbids
 * cudaMalloc, or plugins whose host application owns every device buffer and
 * hands the library no allocator.  (No counterpart on the method's pages:
 * this is a property of the library, not of BitLinear.)
 *   Scratch    The intermediate buffers live in one file-scope device array of
 *              BITNET_FFN_NOALLOC_SCRATCH_BYTES (8 MiB) inside the library.
 *              Every GPU that loads the library holds it until the process
 *              exits.  The request must fit:
 *              bitnet_ffn_workspace_size(M, H, I, variant) <= that size (about
 *              225 tokens of the 2560 -> 6912 -> 2560 FFN); a larger request
 *              returns BITNET_ERR_WORKSPACE and launches nothing.
 *   Set-up     The first call on each device looks up the device address of
 *              the array (cudaGetSymbolAddress) with that device current; make
 *              that first call before any stream capture begins.  The address
 *              belongs to the device's context: after cudaDeviceReset call
 *              bitnet_release_cache(), and the next call looks it up again.
 *   Sharing    All calls on a device share the one array and it keeps the last
 *              call's contents (nothing in it needs to start at zero).  Calls
 *              that can overlap on the GPU (different streams, no ordering
 *              between them) race on it: order them on one stream.
 *   It allocates and frees nothing and calls no allocating routine.  All other
 *   arguments, results and errors are those of bitnet_ffn(). */
#define BITNET_FFN_NOALLOC_SCRATCH_BYTES (8u << 20)
BITNET_API int bitnet_ffn_noalloc(const void *X, int x_dtype, int M, int H, int I,
                                  const uint8_t *W_gate, const float *gamma_gate,
                                  const uint8_t *W_up, const float *gamma_up,
                                  const uint8_t *W_down, const float *gamma_down,
                                  const float *pre_norm_gain, const float *sub_norm_gain,
                                  float eps, int variant, void *Y, int y_dtype,
                                  bitnet_stream_t stream);

/* Message for the last non-OK status on this host thread ("" if none). */
BITNET_API const char *bitnet_last_error(void);

/* Synchronise `stream`, then read and clear the device error word.  Returns
 * BITNET_OK, BITNET_ERR_TIMEOUT (a bounded wait inside a kernel gave up) or
 * BITNET_ERR_CUDA.  Debug / test call: it blocks the host. */
BITNET_API int bitnet_check_device_error(bitnet_stream_t stream);

/* Diagnostic: launch one block that waits on a barrier no thread ever
 * arrives at, with the same bounded wait the kernels use but a limit of
 * `timeout_us` microseconds (1 .. 1000000).  The kernel gives up, records
 * BITNET_ERR_TIMEOUT in the device error word and returns, leaving the
 * context usable.  Returns BITNET_OK if the launch succeeded. */
BITNET_API int bitnet_debug_wait_timeout(unsigned timeout_us, bitnet_stream_t stream);

/* Empty the host-side cache of TMA tensor descriptors and forget the
 * per-context state the library keeps: the device address of the
 * no-allocation FFN scratch, the kernels' shared-memory attributes it has set
 * and the occupancies it has looked up (per device, so that warm calls make
 * no driver query).  The descriptor cache is keyed by device,
 * pointer, shape, box and swizzle, so it stays correct when an address is
 * reused; it holds at most 16384 descriptors (it starts over when full).
 * After cudaDeviceReset (which ends the context those addresses and
 * attributes belong to) call this before the next call into the library. */
BITNET_API void bitnet_release_cache(void);

/* Library version string. */
BITNET_API const char *bitnet_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BITNET_B200_H */
