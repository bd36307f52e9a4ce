/*
 * qk.h -- C ABI of the W8A8 INT8 quantized linear layer for NVIDIA B200
 * (sm_100a).  Library: libqk.so (built from w8a8_int8_quantized_qk_b200/csrc).
 *
 * The layer has three stages, one entry point each:
 *   1. qk_quantize_per_token / qk_silu_mul_quant_per_token -- dynamic
 *      per-token symmetric INT8 quantisation of the activation, optionally
 *      fused with silu(gate) * up;
 *   2. + 3. qk_w8a8_gemm -- INT8 x INT8 GEMM with INT32 accumulation and a
 *      fused dequantisation epilogue (per-token x per-output-channel, or
 *      per-token x per-(channel, 128-wide K group) fp32 scales).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every tensor pointer is DEVICE memory owned by the caller.  The library
 *   never allocates, frees or retains caller memory, and keeps no state
 *   between calls except one device status word (qk_device_status) and the
 *   cached properties (SM count, compute capability) of each device used.
 * - Matrices are row-major and densely packed: x, q [m, k]; b (weights)
 *   [n, k] with K contiguous (one output channel per row, nn.Linear layout);
 *   out, c [m, n].
 * - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *   stream) and the call returns without synchronising.  Arguments are
 *   checked on the host before anything is launched; a rejected call
 *   launches nothing and writes nothing.
 * - The return value is a qk_status.  No entry point throws, aborts, traps
 *   or asserts on the device.
 * - Kernels are launched with programmatic dependent launch: a kernel may
 *   start while the kernel before it on the stream is finishing, if that one
 *   allows it early (this library's kernels do; a kernel that does not is
 *   waited for in full).  Each kernel waits for its predecessor before it
 *   reads anything the predecessor may write or writes anything it may read,
 *   with one exception: the GEMMs (qk_w8a8_gemm and its variants) and the
 *   linear layer request their first weight tiles b (never scale_b or any
 *   other input) before that wait.  So the kernel launched just before a GEMM
 *   on the same stream must not write that GEMM's b if it triggers its
 *   dependents early; the quantisers of this library never write weights.
 * - Values of int8 operands are in [-127, 127] (what the quantisers
 *   produce); -128 and non-finite floating-point inputs are outside the
 *   contract and are not checked.
 * - The library keeps per-device state for the life of the process: the
 *   properties above, kernel attributes, cached tensor maps and the device
 *   address of qk_w8a8_gemm_noalloc's scratch array.  A cudaDeviceReset
 *   invalidates that state: do not call the library on a device after
 *   resetting it in the same process.
 */
#ifndef QK_H_
#define QK_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Symbols of the C ABI are the only ones the library exports. */
#if defined(__GNUC__)
#define QK_API __attribute__((visibility("default")))
#else
#define QK_API
#endif

/* Version of this ABI.  qk_abi_version() returns the value the library was
 * built with; a binding must refuse to use a library whose number differs
 * (an idea taken from the dynquant-kernels package page, "Variants": an ABI
 * number baked into the binary and checked at import). */
#define QK_ABI_VERSION 12

typedef enum qk_status {
  QK_OK = 0,
  QK_ERR_INVALID_ARG = 1,    /* bad size, dtype, group size or NULL pointer */
  QK_ERR_MISALIGNED = 2,     /* a pointer or row stride breaks its alignment rule */
  QK_ERR_UNSUPPORTED = 3,    /* valid request the library does not implement
                                (e.g. no sm_100 device) */
  QK_ERR_OVERFLOW_BOUND = 4, /* k * 127^2 >= 2^31: the INT32 sum could overflow */
  QK_ERR_CUDA = 5,           /* a CUDA runtime/driver call or launch failed */
  QK_ERR_TIMEOUT = 6,        /* a kernel's bounded wait expired (device status) */
  QK_ERR_WORKSPACE = 7       /* workspace NULL or smaller than the size query */
} qk_status;

typedef enum qk_dtype { QK_F32 = 0, QK_BF16 = 1 } qk_dtype;

/* cudaStream_t is `struct CUstream_st *`; this alias keeps the header free of
 * CUDA includes while staying the same type. */
typedef struct CUstream_st* qk_stream;

/* ABI number the library was built with (== QK_ABI_VERSION of its header). */
QK_API int qk_abi_version(void);

/* Static, NUL-terminated description of a status code (never NULL). */
QK_API const char* qk_status_string(int status);

/*
 * qk_quantize_per_token -- dynamic per-token symmetric INT8 quantisation.
 *
 * Defined by: "write-int8-quantized-kernel" (agentmods skill), section
 * "Inputs the agent should gather first": per-token granularity (one scale per
 * activation row) and the symmetric range [-127, 127] with zero-point 0; and
 * the vLLM PR "fused silu_and_mul + dynamic per-token FP8 quantization",
 * Purpose / Algorithm: the scale of a token is max(absmax, 1e-12) / qmax of its
 * own row, and values are quantised with the per-token inverse scale.  With
 * qmax = 127, for every row r:
 *     amax     = max_i |x[r, i]|                       (exact)
 *     scale[r] = max(amax, 1e-12f) / 127.0f            (binary32, RN)
 *     inv      = 1.0f / scale[r]                       (binary32, RN)
 *     q[r, i]  = clamp(rint_half_even(x[r, i] * inv), -127, 127)
 * scale is the DEQUANT multiplier: x ~= q * scale.
 *
 * m        rows (tokens), >= 0 (m == 0 is a no-op)
 * k        row length, > 0 and a multiple of 16
 * x        [m, k] fp32 or bf16 (x_dtype), 16-byte aligned
 * q        [m, k] int8 output, 16-byte aligned
 * scale    [m] fp32 output, 4-byte aligned
 * Errors: QK_ERR_INVALID_ARG (m < 0, k <= 0, k % 16, NULL, bad dtype),
 *         QK_ERR_MISALIGNED, QK_ERR_CUDA.
 */
QK_API qk_status qk_quantize_per_token(int m, int k, const void* x, qk_dtype x_dtype, int8_t* q,
                                float* scale, qk_stream stream);

/*
 * qk_silu_mul_quant_per_token -- h = silu(gate) * up, then the per-token
 * quantisation above applied to h.
 *
 * Defined by: the vLLM PR "fused silu_and_mul + dynamic per-token FP8
 * quantization", Purpose / Algorithm (SiLU gating fused with dynamic
 * per-token quantisation, scale from the row's own absmax), with qmax = 127.
 * h is computed in fp32 and is not rounded to bf16 before quantisation:
 *     e = exp(-g) (the library's fixed binary32 exp: Cody-Waite reduction,
 *                  degree-7 Taylor polynomial, clamp to [-87, 88]);
 *     silu = g / (1 + e);   h = silu * u          (binary32, RN)
 * The kernel keeps h on chip, so gate and up are read from memory once.
 *
 * gate, up [m, k] with row stride ld_in ELEMENTS (ld_in >= k).  Pass the
 * halves of one [m, 2k] buffer as gate = base, up = base + k, ld_in = 2k, or
 * two separate [m, k] tensors with ld_in = k.  Both 16-byte aligned, and
 * ld_in * element size a multiple of 16 bytes.
 * q [m, k] int8, scale [m] fp32 as for qk_quantize_per_token.
 * Errors: as qk_quantize_per_token, plus QK_ERR_INVALID_ARG if ld_in < k.
 */
QK_API qk_status qk_silu_mul_quant_per_token(int m, int k, const void* gate, const void* up,
                                      int64_t ld_in, qk_dtype in_dtype, int8_t* q, float* scale,
                                      qk_stream stream);

/*
 * qk_quantize_per_token_fp8 / qk_silu_mul_quant_per_token_fp8 -- the same
 * two quantisers with float8 e4m3 output: the form of the vLLM PR "fused
 * silu_and_mul + dynamic per-token FP8 quantization" itself (Purpose /
 * Algorithm: float8_e4m3fn, scale = max(absmax, 1e-12) / fp8_max, optionally
 * clamped by scale_ub, quantisation with the per-token inverse scale).
 *
 * Per row: amax = max |x| (or |h|, h = silu(gate) * up in fp32);
 * scale = max(amax, 1e-12f) / 448 (fp32 RN), then scale = min(scale,
 * *scale_ub) when scale_ub is given; inv = 1 / scale (fp32 RN);
 * q = e4m3(clamp(x * inv, -448, 448)) rounded to nearest, ties to even.
 * e4m3 is the OCP E4M3FN format (no infinities, largest finite 448).
 *
 * scale_ub       optional device pointer to one fp32 upper bound of the
 *                written scale (NULL: none), 4-byte aligned
 * q              [m, k] e4m3 codes (one byte each), 16-B aligned
 * other arguments, layouts and errors as the int8 forms above.
 */
QK_API qk_status qk_quantize_per_token_fp8(int m, int k, const void* x, qk_dtype x_dtype,
                                           const float* scale_ub, uint8_t* q, float* scale,
                                           qk_stream stream);
QK_API qk_status qk_silu_mul_quant_per_token_fp8(int m, int k, const void* gate, const void* up,
                                                 int64_t ld_in, qk_dtype in_dtype,
                                                 const float* scale_ub, uint8_t* q, float* scale,
                                                 qk_stream stream);

/*
 * qk_w8a8_gemm -- INT8 x INT8 GEMM with INT32 accumulation and a fused
 * dequantisation epilogue.
 *
 * Defined by: "16. Deploying Custom Kernels", section "C++ Kernel
 * Interface" (GemmConfig: m, n, k, int8 a and b, int32 c, fp32 scale_a and
 * scale_b, float output_scale, stream; status-returning quantized_gemm);
 * "write-int8-quantized-kernel", Inputs (INT32 accumulation, FP32/FP16 output
 * after dequantisation); "KV-cache kernels" (day 26), section 02 (int8
 * products accumulate in int32 and are scaled by a_scale * b_scale at the
 * end) and section 03 (per-group scales every 64-128 channels).
 *
 *   acc[i, j] = sum_k a[i, k] * b[j, k]                     (int32, exact)
 *   group_k == 0   (per-token x per-channel):
 *     out[i, j] = (((float)acc[i, j] * scale_a[i]) * scale_b[j]) * output_scale
 *   group_k == 128 (per-token x per-(channel, K group)):
 *     P_g = sum_{k in group g} a[i, k] * b[j, k]            (int32)
 *     f = 0; for g = 0, 1, ...: f = fmaf((float)P_g, scale_b[j, g], f)
 *     out[i, j] = (f * scale_a[i]) * output_scale
 *   Each step is one binary32 RN operation, in the order written; a bf16
 *   output is the round-to-nearest-even of the fp32 value.
 *
 * m, n, k        m >= 0, n >= 0 (either 0: no-op); k > 0, k % 16 == 0,
 *                n % 8 == 0, and k <= 133144 so that k * 127^2 < 2^31
 * a              [m, k] int8 activations (e.g. q of the quantiser), 16-B aligned
 * b              [n, k] int8 weights, K contiguous, 16-B aligned
 * scale_a        [m] fp32 per-token dequant scales
 * scale_b        [n] fp32 (group_k == 0) or [n, k / 128] fp32 row-major
 *                (group_k == 128); scale_a and scale_b 16-byte aligned
 * group_k        0 or 128 (128 requires k % 128 == 0)
 * output_scale   extra fp32 multiplier applied last (GemmConfig.output_scale)
 * c              optional [m, n] int32 output of the full-K sum acc (in group
 *                mode the sum of the group partials); NULL to skip; 16-B aligned
 * out            optional [m, n] output in out_dtype (QK_BF16 or QK_F32);
 *                NULL to skip; 16-B aligned.  At least one of c, out non-NULL.
 * workspace      device scratch of at least qk_w8a8_gemm_workspace_size()
 *                bytes, 256-B aligned; may be NULL when that size is 0.  When
 *                the output has too few tiles to occupy the GPU, K is split
 *                across CTA pairs; if the pairs of a tile can share a
 *                cluster, the partial sums meet in distributed shared memory
 *                and no workspace is needed (size 0), otherwise they meet in
 *                the workspace (a 4 KB header of arrival counters, then one
 *                INT32 accumulator per output tile that the K slices add
 *                into).  When there are more tiles than CTA pairs but not a
 *                whole number of waves, the tiles of the last partial wave
 *                are cut into 2 to 4 K slices that run first; every slice
 *                stores its INT32 partial in the workspace and the last to
 *                finish adds them up (the same 4 KB header, 16 MB left for
 *                the split-K accumulators, then 256 KB per partial).  In
 *                group mode (the output-only form) the last partial wave's
 *                tiles are instead cut at their middle K group: the first
 *                part runs early on one CTA pair (or CTA, for m <= 128) and
 *                leaves its fp32 running sums in the workspace, the second
 *                runs last on another and continues them in the same group
 *                order, so the result is unchanged (one counter per cut tile
 *                and CTA in the 4 KB header, then the sums, 256 KB per cut
 *                256 x 256 tile or 128 KB per cut 128 x 256 tile, past the
 *                16 MB of split-K accumulators).  The workspace
 *                must be zero-filled before its first use; every completed
 *                call leaves the header, the flags and the split-K
 *                accumulators zero again (the partials and sums need no
 *                initialisation), so
 *                one workspace (sized for the largest problem) can be
 *                reused across calls and shapes.  The call
 *                owns it until the work on `stream` completes: calls that
 *                may overlap need separate workspaces.  After a call that
 *                ended in QK_ERR_TIMEOUT, zero-fill it again.
 * Errors: QK_ERR_INVALID_ARG, QK_ERR_MISALIGNED, QK_ERR_OVERFLOW_BOUND,
 *         QK_ERR_WORKSPACE, QK_ERR_UNSUPPORTED, QK_ERR_CUDA.
 */
QK_API qk_status qk_w8a8_gemm(int m, int n, int k, const int8_t* a, const int8_t* b,
                       const float* scale_a, const float* scale_b, int group_k,
                       float output_scale, int32_t* c, void* out, qk_dtype out_dtype,
                       void* workspace, size_t workspace_bytes, qk_stream stream);

/*
 * qk_fp8_gemm -- float8 e4m3 x e4m3 GEMM (tcgen05.mma kind::f8f6f4, fp32
 * accumulation in the tensor core) with the per-token x per-channel
 * dequantisation epilogue: out = ((acc * scale_a[m]) * scale_b[n]) *
 * output_scale, rounded to out_dtype.  The FP8 counterpart of qk_w8a8_gemm
 * for the e4m3 codes of qk_quantize_per_token_fp8 (the vLLM PR's W8A8-FP8
 * use; "KV-cache kernels" section 02 for the epilogue order).
 *
 * a              [m, k] e4m3 codes, K contiguous, 16-B aligned
 * b              [n, k] e4m3 codes (one output channel per row), 16-B aligned
 * scale_a, scale_b   [m] and [n] fp32 dequant scales, 16-B aligned
 * out            [m, n] in out_dtype (QK_BF16 or QK_F32), 16-B aligned
 * m, n, k        k % 16 == 0, n % 8 == 0 (either of m, n 0: no-op)
 * The accumulation order inside the tensor core is the hardware's, so the
 * results match the exact dot product to within fp32 summation error, not
 * bit for bit.  No workspace.  When the output tiles are too few to fill
 * the GPU, each tile's K range is split over the CTAs of one cluster and
 * the fp32 partials are added in ascending slice order through distributed
 * shared memory, so the result does not depend on which CTA finishes first.
 * Errors: QK_ERR_INVALID_ARG, QK_ERR_MISALIGNED, QK_ERR_UNSUPPORTED,
 *         QK_ERR_CUDA.
 */
QK_API qk_status qk_fp8_gemm(int m, int n, int k, const uint8_t* a, const uint8_t* b,
                             const float* scale_a, const float* scale_b, float output_scale,
                             void* out, qk_dtype out_dtype, qk_stream stream);

/*
 * Asymmetric per-token INT8 ("write-int8-quantized-kernel", Inputs the agent
 * should gather first: asymmetric quantisation maps [-128, 127] to an
 * arbitrary range with a non-zero zero-point; the zero-point adds
 * arithmetic to the hot loop).
 *
 * qk_quantize_per_token_asym: per row, the range [lo, hi] = [min(min x, 0),
 * max(max x, 0)]; scale = max(hi - lo, 1e-12f) / 255; inv = 1 / scale;
 * zero_point = clamp(rne(-128 - lo * inv), -128, 127);
 * q = clamp(rne(x * inv) + zero_point, -128, 127), so x ~ (q - zp) * scale.
 *   x [m, k] (QK_BF16 / QK_F32, 16-B aligned, k % 16 == 0); q [m, k] int8
 *   (16-B aligned); scale [m] fp32; zero_point [m] int32.
 *
 * qk_weight_row_sums: wsum[r] = sum_k w[r][k] (int32), the term the
 *   zero-point correction needs; computed once per weight.  w [n, k] int8,
 *   16-B aligned, k % 16 == 0.
 *
 * qk_w8a8_gemm_asym: qk_w8a8_gemm (per channel, group_k 0) for asymmetric
 *   activations: acc = sum_k (a[m][k] - zero_point_a[m]) * b[n][k], formed
 *   as the tensor-core sum minus zero_point_a[m] * wsum_b[n]; the epilogue
 *   and c as qk_w8a8_gemm.  wsum_b [n] int32 (16-B aligned) from
 *   qk_weight_row_sums.  k <= 66311, so that k * 255 * 127 < 2^31 (else
 *   QK_ERR_OVERFLOW_BOUND).  Workspace as qk_w8a8_gemm.
 */
/*
 * qk_w8a8_moe_gemm -- the W8A8 GEMM of a mixture-of-experts layer in one
 * launch (grouped GEMM): tokens already grouped by expert, expert e owning
 * rows [expert_offsets[e], expert_offsets[e + 1]) of a; each group times
 * its own expert's int8 weights, with the per-token x per-channel epilogue.
 *
 * num_experts    E >= 1
 * total_m        rows of a and out (the tokens of all experts)
 * n, k           per expert: b is [E, n, k] (row e * n + j is expert e's
 *                output channel j), k % 16 == 0, n % 8 == 0, k <= 133144
 * max_m_per_expert   an upper bound on every expert's token count: it sizes
 *                the tile space (E x ceil(max / T) x ceil(n / 256) tiles of
 *                T rows, the empty ones skipped; T = 256 on CTA pairs when
 *                total_m >= 128 E, else T = 128 on single SMs); rows of an
 *                expert beyond it are not computed
 * expert_offsets [E + 1] int32 device array, non-decreasing, offsets[0] = 0,
 *                offsets[E] = total_m (rows outside [0, total_m) are never
 *                written)
 * a              [total_m, k] int8, 16-B aligned; scale_a [total_m] fp32
 * b              [E * n, k] int8, 16-B aligned; scale_b [E, n] fp32, 16-B
 *                aligned
 * out            [total_m, n] bf16 or fp32, 16-B aligned
 * Errors as qk_w8a8_gemm (per channel only, no workspace, no c).
 */
QK_API qk_status qk_w8a8_moe_gemm(int num_experts, int total_m, int n, int k, int max_m_per_expert,
                                  const int32_t* expert_offsets, const int8_t* a, const int8_t* b,
                                  const float* scale_a, const float* scale_b, float output_scale,
                                  void* out, qk_dtype out_dtype, qk_stream stream);

/*
 * qk_quantize_static -- static per-tensor INT8 ("write-int8-quantized-
 * kernel", Inputs the agent should gather first: per-tensor granularity, one
 * scale for the entire tensor, computed offline): inv = 1 / *scale (fp32
 * RN), q = clamp(rne(x * inv), -127, 127); values beyond 127 * scale
 * saturate.  scale: device pointer to one fp32 (> 0), 4-byte aligned; x, q
 * as qk_quantize_per_token.  The GEMM then takes scale_a as an [m] vector
 * holding that one value.
 */
QK_API qk_status qk_quantize_static(int m, int k, const void* x, qk_dtype x_dtype,
                                    const float* scale, int8_t* q, qk_stream stream);

QK_API qk_status qk_quantize_per_token_asym(int m, int k, const void* x, qk_dtype x_dtype,
                                            int8_t* q, float* scale, int32_t* zero_point,
                                            qk_stream stream);
QK_API qk_status qk_weight_row_sums(int n, int k, const int8_t* w, int32_t* wsum,
                                    qk_stream stream);
QK_API qk_status qk_w8a8_gemm_asym(int m, int n, int k, const int8_t* a,
                                   const int32_t* zero_point_a, const int8_t* b,
                                   const int32_t* wsum_b, const float* scale_a,
                                   const float* scale_b, float output_scale, int32_t* c,
                                   void* out, qk_dtype out_dtype, void* workspace,
                                   size_t workspace_bytes, qk_stream stream);

/* Bytes of workspace qk_w8a8_gemm needs for this problem on the current
 * device (0 when none; the split depends on the device's SM count).
 * Returns 0 for arguments qk_w8a8_gemm would reject. */
QK_API size_t qk_w8a8_gemm_workspace_size(int m, int n, int k, int group_k);

/* qk_w8a8_gemm_kernel -- diagnostic: which kernel, tile shape and split form
 * qk_w8a8_gemm launches for this problem on the current device (the choice
 * depends on m, n, k, group_k, whether the int32 sums c are requested
 * (with_c != 0), and the device's SM count).  Returns a NUL-terminated
 * string, never null: "unsupported" for shapes qk_w8a8_gemm rejects, "no
 * device" without a usable sm_100 device.  The string is owned by the
 * library and stays valid until the next call of this function on the same
 * host thread. */
QK_API const char* qk_w8a8_gemm_kernel(int m, int n, int k, int group_k, int with_c);

/*
 * qk_w8a8_linear -- the whole W8A8 linear layer in one call: dynamic
 * per-token quantisation of x (as qk_quantize_per_token) into the
 * workspace, then the INT8 GEMM and dequant epilogue (as qk_w8a8_gemm) on
 * the same stream.  The int8 values, scales and outputs are bit-identical to
 * the two-call form.  The two kernels are launched with programmatic
 * dependent launch, so the GEMM's set-up overlaps the quantiser's tail.
 *
 * x              [m, k] activations, x_dtype QK_BF16 or QK_F32, 16-B aligned
 * b, scale_b, group_k, output_scale   as qk_w8a8_gemm
 * scale_a_out    optional [m] fp32: receives the per-token scales; NULL to skip
 * out            [m, n] output in out_dtype, 16-B aligned (required)
 * workspace      qk_w8a8_linear_workspace_size() bytes, 256-B aligned: the
 *                GEMM's workspace and 256 bytes of flags used by
 *                qk_w8a8_linear_fused (both must be zero-filled before the
 *                first use and are left zero by every completed call;
 *                zero-fill again after a call that ended in QK_ERR_TIMEOUT),
 *                then q and the scales.  Calls that may overlap need
 *                separate workspaces.
 * Errors: those of qk_quantize_per_token and qk_w8a8_gemm.
 */
QK_API qk_status qk_w8a8_linear(int m, int n, int k, const void* x, qk_dtype x_dtype,
                                const int8_t* b, const float* scale_b, int group_k,
                                float output_scale, float* scale_a_out, void* out,
                                qk_dtype out_dtype, void* workspace, size_t workspace_bytes,
                                qk_stream stream);

/* Bytes of workspace qk_w8a8_linear needs (0 for arguments it would reject). */
QK_API size_t qk_w8a8_linear_workspace_size(int m, int n, int k, int group_k);

/*
 * qk_w8a8_linear_fused -- the decode linear layer (per-channel scales) in ONE
 * launch: the quantiser inside the GEMV's grid ("dynquant-kernels" 0.2.0,
 * What is in here: the decode GEMV as the memory-bound serving case;
 * "KV-cache kernels" section 04: the same fusion instincts).  The grid's first
 * m CTAs quantise one token each (the rule of qk_quantize_per_token) into the
 * workspace and count it in a flag word there; the other CTAs run the GEMV,
 * start the weight stream at once and wait (bounded, about a second) for the
 * count to reach m before they read the tokens.  The grid never exceeds what
 * the device holds at once; other work running on the device at the same
 * time can make the wait expire (QK_ERR_TIMEOUT in qk_device_status, outputs
 * incomplete).  Results are bit-identical to qk_w8a8_linear.
 *
 * On a B200, at 4 x 14336 x 4096 in CUDA graphs of back-to-back calls, it
 * takes 14.9 us against 13.0 us for qk_w8a8_linear's two overlapped kernels:
 * the weight requests queue in DRAM ahead of the tokens' own loads.  It saves
 * the host one kernel launch per layer, which matters when decode steps are
 * launched eagerly.
 *
 * Arguments, layouts and the workspace are those of qk_w8a8_linear with
 * group_k = 0; the workspace's flag words must be zero before the call and
 * are zero again after it.  Shapes: m <= 4 with k <= 16384, or 4 < m <= 8
 * with k <= 8192 (k % 16 == 0, n % 8 == 0); others give QK_ERR_UNSUPPORTED.
 * Errors: those of qk_w8a8_linear, and QK_ERR_UNSUPPORTED.
 */
QK_API qk_status qk_w8a8_linear_fused(int m, int n, int k, const void* x, qk_dtype x_dtype,
                                      const int8_t* b, const float* scale_b, float output_scale,
                                      float* scale_a_out, void* out, qk_dtype out_dtype,
                                      void* workspace, size_t workspace_bytes, qk_stream stream);

/*
 * qk_w8a8_gemm_noalloc -- qk_w8a8_gemm without a caller-provided workspace.
 *
 * (No counterpart on the pages: an addition for callers that cannot allocate
 * device memory.)  Some callers cannot call cudaMalloc on the path that runs
 * the layer: a plugin inside an inference runtime that owns all device
 * memory, a latency-critical path where an allocation would synchronise the
 * device, or an embedded caller with a fixed memory budget.  This entry point
 * takes the same arguments as qk_w8a8_gemm minus the workspace, and when the
 * problem needs split-K scratch it uses a scratch array built into the
 * library instead: QK_NOALLOC_SCRATCH_BYTES bytes of device memory that every
 * GPU which loads the library holds until the process exits.
 *
 * - Nothing is allocated or freed: no cudaMalloc, cudaFree or allocating
 *   library routine.  The inputs and outputs are still the caller's.
 * - The first call on a device looks up the scratch array's device address
 *   (once per device, with that device current); make that first call before
 *   any stream capture on the device.
 * - Each call clears the part of the scratch array that must start at zero
 *   (counters and split-K accumulators) on `stream` before its kernel, so it
 *   does not depend on what an earlier call left there.
 * - Every call shares the one array: calls that can overlap on the GPU (on
 *   different streams, or from different threads) race and give wrong
 *   results.  Serialise them.
 * - QK_NOALLOC_SCRATCH_BYTES covers every split-K problem (a 4 KB header,
 *   at most 64 split-K accumulator tiles and 128 tail-split partial tiles,
 *   each 256 KB), and group mode's cut tiles (256 KB of running sums per cut
 *   256 x 256 tile, at most a quarter of the SM count of them, or 128 KB per
 *   cut 128 x 256 tile, at most half the SM count, past the same 4 KB +
 *   16 MB); a problem
 *   whose qk_w8a8_gemm_workspace_size exceeded it would be rejected with
 *   QK_ERR_WORKSPACE and nothing launched.  Other errors are those of
 *   qk_w8a8_gemm.
 */
#define QK_NOALLOC_SCRATCH_BYTES (48u * 1024u * 1024u + 4096u)

QK_API qk_status qk_w8a8_gemm_noalloc(int m, int n, int k, const int8_t* a, const int8_t* b,
                                      const float* scale_a, const float* scale_b, int group_k,
                                      float output_scale, int32_t* c, void* out,
                                      qk_dtype out_dtype, qk_stream stream);

/*
 * qk_device_status -- read and clear the library's device status word on the
 * current device.  Kernels that wait on a barrier give up after a bounded
 * time (about one second) instead of hanging; when that happens they record
 * QK_ERR_TIMEOUT there, release what they hold and return early, so their
 * outputs are incomplete.  This call synchronises `stream` first; it returns
 * QK_OK, QK_ERR_TIMEOUT or QK_ERR_CUDA.
 */
QK_API qk_status qk_device_status(qk_stream stream);

/*
 * qk_selftest_bounded_wait -- diagnostic: launch one block that waits on a
 * barrier nobody arrives at, with a limit of `timeout_us` microseconds
 * (1 .. 2,000,000).  When the limit passes the kernel records QK_ERR_TIMEOUT in
 * the device status word and returns.  Lets a caller check, without any fault,
 * that the bounded-wait path works on this device.
 */
QK_API qk_status qk_selftest_bounded_wait(int timeout_us, qk_stream stream);

/*
 * qk_selftest_silu -- diagnostic: checks the fused SiLU arithmetic of the
 * silu quantisers.  For every binary32 bit pattern g in [first, first +
 * count) that is finite, it computes silu(g) * 1 the way the quantisers do
 * (two values at a time: the exp's reduction, polynomial, the divide -- by
 * Markstein's method -- and the final multiply on packed binary32 pairs) and
 * the way the definition reads (one value at a time, every step a scalar
 * IEEE round-to-nearest operation, the divide IEEE's), and
 * counts the g whose two results differ in any bit.  g is the only input of that
 * arithmetic, so first = 0, count = 2^32 covers every value it can see.
 * Defined by the fused silu_and_mul quantisation of the vLLM PR "fused
 * silu_and_mul + dynamic per-token FP8 quantization", Algorithm (silu(gate)
 * computed in fp32 before the per-token absmax).
 *
 * first, count     the range of bit patterns; 1 <= count, first + count <= 2^32
 * mismatches       device uint64 the kernel adds its count to (the caller
 *                  zero-fills it), 8-byte aligned
 * first_mismatch   optional device uint32 lowered (atomic minimum) to the
 *                  smallest mismatching bit pattern; the caller sets it to
 *                  0xFFFFFFFF first; NULL to skip
 * Errors: QK_ERR_INVALID_ARG, QK_ERR_MISALIGNED, QK_ERR_UNSUPPORTED,
 *         QK_ERR_CUDA.
 */
QK_API qk_status qk_selftest_silu(uint32_t first, uint64_t count, unsigned long long* mismatches,
                                  uint32_t* first_mismatch, qk_stream stream);

/*
 * qk_selftest_mma_rate -- diagnostic: the INT8 tensor-core rate of the
 * current device.  Launches `ctas` CTAs (cta_group 1: one per SM, M = 128;
 * cta_group 2: clusters of two CTAs on an SM pair, M = 256, the pair's
 * leader issuing tcgen05.mma.cta_group::2) that each issue `iters`
 * tcgen05.mma.kind::i8 instructions of M x n x 32 back to back on fixed
 * shared-memory operands into one TMEM accumulator: no global-memory traffic,
 * so the kernel's duration is the tensor pipe's time.  Defined by the
 * roofline reading of "KV-cache kernels" (day 26) section 01 (a kernel's
 * achieved rate is read against the hardware's compute ceiling): the
 * library's GEMM fractions divide by the rate this kernel reaches.
 *
 * Work per launch: (ctas / cta_group) * iters * M * n * 32 multiply-adds
 * (2 int8 ops each); the caller times the launch with CUDA events.
 * cta_group   1 or 2
 * n           32 .. 256, a multiple of 16
 * iters       1 .. 1048576 instructions per CTA (pair)
 * ctas        1 .. 65535 CTAs, a multiple of cta_group; at most what the
 *             device holds at once (one CTA per SM) for a meaningful rate
 * operand_seed  0: the operand tiles are zero; otherwise every CTA fills
 *             them with bytes from a counter-based hash of the seed (close to
 *             uniform over the int8 range).  The rate depends on the values:
 *             on a B200 random operands run measurably slower than zeros at
 *             the same SM clock, so a GEMM on random data is also read
 *             against the random-operand rate
 * cycles      optional device array [ctas] of uint64, 8-byte aligned: the
 *             issuing CTA's SM clock cycles from its first issue to the
 *             completion of its last MMA (0 for a pair's second CTA); NULL
 *             to skip
 * The completion wait is bounded like every other wait of the library.
 * Errors: QK_ERR_INVALID_ARG, QK_ERR_MISALIGNED, QK_ERR_UNSUPPORTED,
 *         QK_ERR_CUDA.
 */
QK_API qk_status qk_selftest_mma_rate(int cta_group, int n, int iters, int ctas,
                                      uint32_t operand_seed, unsigned long long* cycles,
                                      qk_stream stream);

/*
 * qk_selftest_mma_interference -- diagnostic: how much arithmetic on the
 * CUDA cores slows the tensor core of the same SM.  Launches `ctas` CTAs of
 * 384 threads in clusters of two (one pair per SM pair).  In each pair the
 * leader issues `groups` groups of four tcgen05.mma.cta_group::2.kind::i8
 * 256 x 256 x 32 (the group-128 GEMM's unit of work, 512 SM cycles at the
 * full rate) on fixed pseudo-random shared-memory operands into alternating
 * TMEM buffers.  Meanwhile warps 4..11 of both CTAs run a companion loop
 * until the MMAs are done:
 *   0 none; 1 fp32 fused multiply-add; 2 fp32 multiply; 3 int32 -> fp32
 *   conversion and a logic op; 4 int32 multiply-add; 5 conversion and fused
 *   multiply-add (the group-128 epilogue's arithmetic); 6 fp32 pair ->
 *   bf16x2 conversion (the epilogues' output packing).
 * Defined, like qk_selftest_mma_rate, by the roofline reading of
 * "KV-cache kernels" (day 26) section 01: it tells whether an epilogue that
 * overlaps the MMAs can be hidden under them.
 *
 * groups      1 .. 262144 groups of four MMAs per pair
 * ctas        2 .. 65535, even; at most what the device holds at once
 * cycles      optional device array [ctas] of uint64, 8-byte aligned: the
 *             leader's SM clock cycles from its first MMA to the completion
 *             of its last (0 on the second CTA of a pair); cycles / groups is
 *             the time of one group
 * The companion loops and the completion wait are bounded.
 * Errors: QK_ERR_INVALID_ARG, QK_ERR_MISALIGNED, QK_ERR_UNSUPPORTED,
 *         QK_ERR_CUDA.
 */
QK_API qk_status qk_selftest_mma_interference(int companion, int groups, int ctas,
                                              unsigned long long* cycles, qk_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* QK_H_ */
