/*
 * fp4q.h — C ABI of the fused block-Hadamard rotation + microscaling FP4 quantizer.
 *
 * What it computes.  The online activation path of MR-GPTQ-style FP4 inference
 * ("Bridging the Gap Between Promise and Performance for Microscaling FP4 Quantization",
 * gist.science/de/paper/2509.23202, Technische Zusammenfassung, 2. Methodik,
 * GPU-Kernel-Unterstützung: the activation's block Hadamard rotation is fused into a
 * lightweight quantization kernel computed online).  For a bf16 activation matrix X
 * (M rows x K columns, row-major):
 *
 *   1. rotate every contiguous b-block of each row:  y = x_blk * H_b / sqrt(b), with the
 *      Sylvester Hadamard matrix H_b in natural order (b = 1 means no rotation);
 *   2. split each row into groups of g consecutive rotated values (g = 32 for MXFP4,
 *      16 for NVFP4 — same page, 1. Problemstellung) and take the group amax A;
 *   3. pick the group scale:
 *        MXFP4: X = 2^e stored as the E8M0 byte e + 127 ("Unveiling the Potential of
 *               Quantization with MXFP4", gist.science/nl/paper/2603.08713, Technische
 *               samenvatting, Probleemstelling: E8M0, powers of two), with e by rule
 *                 FP4Q_SCALE_FLOOR_OCP    e = floor(log2 A) - 2
 *                 FP4Q_SCALE_CEIL_NOCLIP  e = ceil(log2(A / 6))   (A/X in (3, 6])
 *                 FP4Q_SCALE_OAS          the ceil rule, then e - 1 when A/X is in
 *                                         [3, 3.5] (same page, Methodologie 1,
 *                                         Overflow-Aware Scaling)
 *               e clamped to [-127, 127]; A = 0 gives byte 0;
 *        NVFP4: an fp32 tensor scale s_g and E4M3 block scales
 *               s_b = E4M3_RNE_satfinite(A / fp32(6 s_g)), element divisor
 *               S = fp32(E4M3(s_b) s_g) (same page, Probleemstelling: E4M3 scales;
 *               gist.science/es/paper/2509.23202, Resumen técnico 2.B: group and
 *               tensor scales).  s_g = fp32(A_t / 2688) from the amax A_t of the whole
 *               rotated tensor (1 when A_t = 0);
 *   4. divide by the scale and round to E2M1 (magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6),
 *      nearest with ties to the even code, saturating at 6, sign bit = sign of y;
 *      a zero NV block scale gives all-zero codes;
 *   5. pack two codes per byte, element 2j in the low nibble.
 *
 * Layout (all row-major, contiguous):
 *   x        bf16  [M][K]          device memory, 16-byte aligned
 *   codes    uint8 [M][K/2]        device memory, 16-byte aligned
 *   scales   uint8 [M][K/g]        device memory, 16-byte aligned
 *                                  (E8M0 bytes for MXFP4, E4M3 bytes for NVFP4)
 *   tensor_scale  one fp32 in device memory (NVFP4 only; NULL for MXFP4)
 *
 * Shape rules: M >= 0, K >= 0, K a multiple of lcm(g, b), M*K < 2^40.  M*K = 0 is a valid
 * empty call that launches nothing.
 *
 * Ownership.  The caller owns every buffer passed in.  A plan owns two small device
 * arrays that fp4q_plan_create allocates and fp4q_plan_destroy frees: the per-CTA partial
 * maxima of NV plans (for FP4Q_SCALE_NV_DYNAMIC and fp4q_amax), and the per-CTA partial
 * sums of fp4q_quant_error (every plan made on a machine with a CUDA device).  Calls
 * allocate nothing.
 *
 * Streams.  Every call is asynchronous and stream-ordered on the given stream (a
 * cudaStream_t passed as void*; NULL is the legacy default stream).  A plan's format, group,
 * block and rule are fixed at creation; fp4q_plan_set_kernel and fp4q_plan_set_signs change
 * its kernel choice and channel signs for later calls and must not race with calls in
 * flight on it.  Two calls that share a DYNAMIC plan, or two fp4q_quant_error calls on one
 * plan, must be ordered on one stream (they share the plan's scratch arrays).
 *
 * Errors.  Argument problems are found on the host before anything is launched and
 * return FP4Q_ERR_ARG / _SHAPE / _ALIGN / _UNSUPPORTED.  A CUDA launch failure returns
 * FP4Q_ERR_CUDA (fp4q_last_cuda_error gives the message).  No C++ exception crosses the
 * ABI.  Every wait inside a kernel is bounded in time; a wait that runs out records a
 * code that fp4q_device_status reads back (and clears) instead of hanging.
 */
#ifndef FP4Q_H_
#define FP4Q_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FP4Q_OK = 0,
  FP4Q_ERR_ARG = 1,          /* null pointer where one is required, bad plan handle  */
  FP4Q_ERR_SHAPE = 2,        /* M, K outside the shape rules                          */
  FP4Q_ERR_ALIGN = 3,        /* a pointer is not 16-byte aligned                      */
  FP4Q_ERR_UNSUPPORTED = 4,  /* format / group / block / rule combination not offered */
  FP4Q_ERR_CUDA = 5,         /* a CUDA runtime call failed                            */
  FP4Q_ERR_TIMEOUT = 6       /* a bounded wait inside a kernel ran out                */
} fp4q_status;

/* FP4Q_MXFP4_MBS: MXFP4 under MBS-Static macro-block scales ("Unveiling the Potential of
 * Quantization with MXFP4", Methodologie 2, Macro Block Scaling).  Every 128-element macro
 * block of a row gets one extra scale with 8 mantissa bits, taken directly from the block's
 * maximum A_M: with fp32(A_M / 6) = 2^E (1 + f), the byte m8 = ceil(256 f) mod 256 and
 * s_M = 1 + m8 / 256 (so the block maximum lands on the top E2M1 value, never above it;
 * 256 wraps to 0, the same quantization with every group exponent one higher).  The rotated
 * values are divided by s_M (fp32, correctly rounded) and then quantized as MXFP4 with the
 * plan's MX rule; a value decodes as E2M1 * 2^(byte - 127) * s_M.  Group 32, K a multiple of
 * 128.  Served by fp4q_rotate_quantize_mbs, fp4q_dequantize_mbs and fp4q_quant_error, on
 * either rotate + quantize kernel (the tensor-core kernel for b >= 32). */
typedef enum { FP4Q_MXFP4 = 0, FP4Q_NVFP4 = 1, FP4Q_MXFP4_MBS = 2 } fp4q_format;

typedef enum {
  FP4Q_SCALE_FLOOR_OCP = 0,   /* MX: e = floor(log2 A) - 2; values above 6 X saturate  */
  FP4Q_SCALE_CEIL_NOCLIP = 1, /* MX: e = ceil(log2(A/6)); overflow-aware, never clips  */
  FP4Q_SCALE_OAS = 2,         /* MX: ceil rule, A/X in [3, 3.5] pushed to [6, 7]        */
  FP4Q_SCALE_NV_STATIC = 3,   /* NV: caller supplies s_g in *tensor_scale (read only)  */
  FP4Q_SCALE_NV_DYNAMIC = 4   /* NV: the call computes s_g from X and writes it        */
} fp4q_scale_rule;

typedef struct fp4q_plan_s* fp4q_plan;

/* Create a plan.  format: fp4q_format; group: 32 (MXFP4) or 16 (NVFP4); hadamard_block:
 * 1, 2, 4, ..., 128 (1 = no rotation); scale_rule: an fp4q_scale_rule valid for the
 * format.  Writes the plan to *out.
 *
 * Device binding.  A plan made while a CUDA device is current belongs to the CUDA context
 * current at creation (the device's primary context, unless the caller made another one
 * current through the driver API): its scratch arrays (see Ownership) are allocated there.
 * fp4q_rotate_quantize(_dump, _mbs), fp4q_amax, fp4q_quant_error and fp4q_dequantize(_mbs)
 * must then be called with that context current; with another device or another context
 * current they return FP4Q_ERR_ARG before launching anything (and before their shape and
 * pointer checks), and fp4q_last_cuda_error() says so.  After cudaDeviceReset a plan made before it
 * is unusable: destroy it and make a new one.  A plan made on a machine without a CUDA
 * device owns no device memory and is bound to none. */
fp4q_status fp4q_plan_create(fp4q_plan* out, int format, int group, int hadamard_block,
                             int scale_rule);

/* Which kernel a plan's rotate + quantize calls run on. */
typedef enum {
  FP4Q_KERNEL_AUTO = 0,        /* the tensor-core kernel when every Hadamard block holds whole
                                  scale groups (b >= 16 and b >= g) and M*K >= 2^22, else the
                                  butterfly kernel (which starts faster on small tensors); MXFP4
                                  plans with channel signs and b = 128 take the butterfly
                                  kernel from M*K >= 3 * 2^26 on (faster there, by
                                  measurement)                                                 */
  FP4Q_KERNEL_BUTTERFLY = 1,   /* in-register fast Walsh-Hadamard butterfly on CUDA cores    */
  FP4Q_KERNEL_TENSOR_CORE = 2  /* tcgen05 MMA against H_b with TMEM accumulators; tensors of
                                  2^31 - 1024 or more Hadamard blocks (the limit of its 32-bit
                                  TMA row coordinates) still run on the butterfly kernel      */
} fp4q_kernel;

/* Choose the kernel for later rotate + quantize calls of this plan (not thread-safe against
 * calls running on the same plan).  Returns FP4Q_ERR_UNSUPPORTED for FP4Q_KERNEL_TENSOR_CORE
 * when b < 16 or b < g.  Both kernels compute the same function (see fp4q_rotate_quantize);
 * they round the butterfly sums differently, so rare codes within the parity tolerance of a
 * rounding boundary can differ between them. */
fp4q_status fp4q_plan_set_kernel(fp4q_plan plan, int kernel);

/* Free a plan (NULL is accepted).  Synchronizes nothing: the caller must make sure no
 * call using the plan is still running on the device. */
fp4q_status fp4q_plan_destroy(fp4q_plan plan);

/* Per-channel random signs for the rotation (a randomised Hadamard transform, "wie in
 * QuIP/QuaRot": "Bridging the Gap Between Promise and Performance for Microscaling FP4
 * Quantization", Technische Zusammenfassung, 2. Methodik).  With signs s the rotation of
 * every row is Q = diag(s) (I kron H_b / sqrt(b)): channel k is negated before the block
 * rotation.  The same s must be used on the activations (online) and on the weights (offline,
 * rotate + quantize of W with the same plan settings), so that (X Q)(W Q)^T = X W^T.
 *
 * signs: device uint32 [ceil(K / 32)]; bit (k mod 32) of word k / 32 set negates channel k.
 * Borrowed: the caller keeps the array alive and unchanged while the plan uses it.  NULL
 * clears the signs.  K: the row length the signs are for; a multiple of max(g, b), at most
 * 2^34.  Afterwards every call on the plan must have this K (FP4Q_ERR_SHAPE otherwise), and
 * fp4q_rotate_quantize(_dump), fp4q_amax, fp4q_quant_error and fp4q_dequantize (with
 * unrotate) all use the signs, on either rotate + quantize kernel (the tensor-core kernel
 * flips the signs in shared memory before its product; the butterfly kernel as it loads).
 * signs must be 4-byte aligned. */
fp4q_status fp4q_plan_set_signs(fp4q_plan plan, const uint32_t* signs, int64_t K);

/* Rotate and quantize X in one pass over HBM (steps 1-5 above).
 * x_bf16: device bf16 [M][K]; codes_out: device uint8 [M][K/2]; scales_out: device
 * uint8 [M][K/g]; tensor_scale: device fp32 — NV static: read; NV dynamic: written with
 * the s_g the call used; MX: ignored (may be NULL). */
fp4q_status fp4q_rotate_quantize(fp4q_plan plan, const void* x_bf16, int64_t M, int64_t K,
                                 void* codes_out, void* scales_out, float* tensor_scale,
                                 void* stream);

/* Rotate and quantize X under an FP4Q_MXFP4_MBS plan: codes_out uint8 [M][K/2] and
 * scales_out uint8 [M][K/32] (E8M0 bytes of the scaled groups) as for MXFP4, and macro_out
 * uint8 [M][K/128] (the macro-scale bytes m8; any alignment).  Returns FP4Q_ERR_UNSUPPORTED
 * for a plan of another format; fp4q_rotate_quantize(_dump) return it for an MBS plan. */
fp4q_status fp4q_rotate_quantize_mbs(fp4q_plan plan, const void* x_bf16, int64_t M, int64_t K,
                                     void* codes_out, void* scales_out, void* macro_out, void* stream);

/* Same as fp4q_rotate_quantize, and also stores the fp32 rotated values y (before any
 * scaling) to y_out (device fp32 [M][K]).  A debugging and testing aid: the same kernel
 * body with one extra store. */
fp4q_status fp4q_rotate_quantize_dump(fp4q_plan plan, const void* x_bf16, int64_t M, int64_t K,
                                      void* codes_out, void* scales_out, float* tensor_scale,
                                      float* y_out, void* stream);

/* NVFP4 per-tensor scale: s_g = fp32(max|y| / 2688) over the rotated X (1 for an all-zero
 * X), written to *tensor_scale_out (device fp32).  Uses the plan's block size; needs a
 * plan made with an NV rule.  The pass runs on the kernel the plan's rotate + quantize calls
 * would use (see fp4q_kernel), so max|y| is taken over the same fp32 sums. */
fp4q_status fp4q_amax(fp4q_plan plan, const void* x_bf16, int64_t M, int64_t K,
                      float* tensor_scale_out, void* stream);

/* Decode: out[r][k] = E2M1(code) * scale (MX: 2^(byte-127); NV: fp32(E4M3(byte) * s_g)),
 * then, when unrotate != 0, the inverse rotation (H_b / sqrt(b) again, it is its own
 * inverse).  codes, scales: device, layout as produced above; tensor_scale: device fp32
 * (NV only); out_f32: device fp32 [M][K]. */
fp4q_status fp4q_dequantize(fp4q_plan plan, const void* codes, const void* scales,
                            const float* tensor_scale, int64_t M, int64_t K, int unrotate,
                            float* out_f32, void* stream);

/* Quantization error of rotate + quantize on X, without storing codes or scales: the
 * signal and error energies sum y^2 and sum (y - yhat)^2 over all M*K elements and the QSNR
 * 10 log10(signal / error) in dB.  y are the rotated values and yhat the dequantized codes
 * the plan's fp4q_rotate_quantize would produce (the same scale decisions and codes).  The
 * rotation is orthonormal, so both energies are also those of X against its dequantized,
 * rotated-back copy.  This is the measure of the error analysis in "Bridging the Gap Between
 * Promise and Performance for Microscaling FP4 Quantization" (Technische Zusammenfassung,
 * 2. Methodik: quantization MSE = error / (M*K)) and of the QSNR gains in "Unveiling the
 * Potential of Quantization with MXFP4" (Methodologie 1).
 *
 * x_bf16: device bf16 [M][K]; tensor_scale: device fp32 as for fp4q_rotate_quantize (NV
 * static: read; NV dynamic: written; MX: ignored, may be NULL); out: device fp64 [3] =
 * {signal, error, QSNR dB}, +inf dB when the error is 0 (an empty X gives {0, 0, +inf}).
 * The result is deterministic: per-CTA partial sums in fp64 (in a scratch array the plan
 * owns, allocated when the plan is made on a machine with a CUDA device), then one
 * fixed-order reduction.  Calls on one plan must not overlap on the GPU.  Returns
 * FP4Q_ERR_UNSUPPORTED for a plan made without a CUDA device; argument errors as for
 * fp4q_rotate_quantize, and out must be 8-byte aligned. */
fp4q_status fp4q_quant_error(fp4q_plan plan, const void* x_bf16, int64_t M, int64_t K,
                             float* tensor_scale, double* out, void* stream);

/* Decode an FP4Q_MXFP4_MBS result: out[r][k] = E2M1(code) * 2^(byte - 127) * s_M (exact in
 * fp32), rotated back when unrotate != 0.  macro: the bytes fp4q_rotate_quantize_mbs wrote.
 * Returns FP4Q_ERR_UNSUPPORTED for other plans; fp4q_dequantize returns it for MBS plans. */
fp4q_status fp4q_dequantize_mbs(fp4q_plan plan, const void* codes, const void* scales, const void* macro,
                                int64_t M, int64_t K, int unrotate, float* out_f32, void* stream);

/* Block-scaled FP4 GEMM on the tensor cores: D = alpha * A * B^T, the product the rotated,
 * quantized activations and weights meet in ("Bridging the Gap Between Promise and Performance
 * for Microscaling FP4 Quantization", Technische Zusammenfassung, 2. Methodik,
 * GPU-Kernel-Unterstützung; the weights absorb the rotation, so no inverse rotation is needed).
 *
 * format: FP4Q_MXFP4 (E8M0 scales per 32) or FP4Q_NVFP4 (E4M3 scales per 16).  A: the output of
 * fp4q_rotate_quantize on an activation X [M][K]: a_codes uint8 [M][K/2], a_scales uint8
 * [M][K/g]; B: the same for the weights W [N][K] (quantized with the same block and signs, so
 * that (X Q)(W Q)^T = X W^T): b_codes uint8 [N][K/2], b_scales uint8 [N][K/g].  NVFP4: alpha =
 * *a_tensor_scale * *b_tensor_scale (device fp32); MXFP4: alpha = 1 (the pointers are
 * ignored).  d_bf16: device bf16 [M][N], row-major, the fp32 accumulator times alpha rounded
 * to nearest even.  Shapes: M >= 0 any; N a multiple of 32; K a positive multiple of 256 (an
 * empty M or N launches nothing).  Arrays 16-byte aligned, tensor scales 4-byte aligned.  The
 * MMA is tcgen05 kind::mxf4 / kind::mxf4nvf4 with fp32 accumulation in tensor memory. */
fp4q_status fp4q_gemm(int format, const void* a_codes, const void* a_scales, const float* a_tensor_scale,
                      const void* b_codes, const void* b_scales, const float* b_tensor_scale, int64_t M,
                      int64_t N, int64_t K, void* d_bf16, void* stream);

/* No-allocation NVFP4 dynamic-scale path.  The paper has no counterpart: this exists for
 * callers that cannot allocate device memory themselves — for example a library loaded into
 * a framework or serving runtime whose own allocator owns all device memory, or a service that
 * must not allocate after start-up — and so cannot create an FP4Q_SCALE_NV_DYNAMIC plan, whose
 * creation allocates the plan's partial-maximum array.
 *
 * Same computation and output layout as fp4q_rotate_quantize with a plan
 * (FP4Q_NVFP4, 16, hadamard_block, FP4Q_SCALE_NV_DYNAMIC): x_bf16 device bf16 [M][K];
 * codes_out device uint8 [M][K/2]; scales_out device uint8 [M][K/16]; tensor_scale_out
 * device fp32, written with the s_g the call used.  The caller still owns and passes every
 * input and output.  Both passes run on the butterfly kernel, so the outputs are those of such
 * a plan held to FP4Q_KERNEL_BUTTERFLY.
 *
 * Scratch: the per-CTA partial maxima live in a fixed array inside this library (4096 fp32
 * values, 16 KB), reserved on every GPU that loads the library until the process exits.
 * The call needs one value per CTA of its amax pass (a full wave: SM count x resident CTAs
 * per SM); when that exceeds 4096 it returns FP4Q_ERR_UNSUPPORTED before launching anything
 * and fp4q_last_cuda_error() names the limit.  Every call overwrites the values it reads, so
 * nothing carries over from earlier calls; calls that overlap on the GPU (other streams, other
 * host threads) share the array and race.
 *
 * Allocation: none — no cudaMalloc, cudaFree or allocating library routine.  Every call looks
 * up the array's device address in the context current at the time (a host-side lookup), so
 * it stays right after cudaDeviceReset or under a context the caller made current.  The first
 * call in each context also configures the kernels there (shared-memory attributes); make
 * that first call outside any stream capture. */
fp4q_status fp4q_rotate_quantize_nvfp4_dynamic_noalloc(const void* x_bf16, int64_t M, int64_t K,
                                                       int hadamard_block, void* codes_out,
                                                       void* scales_out, float* tensor_scale_out,
                                                       void* stream);

/* Read and clear the device-side status word (FP4Q_OK, or FP4Q_ERR_TIMEOUT when a bounded
 * wait ran out in a kernel since the last read).  Synchronizes the current device. */
fp4q_status fp4q_device_status(void);

/* Self-test of the failure path: launches one warp that waits on a shared-memory barrier
 * nothing arrives on.  The wait is bounded like every wait in the library; after about one
 * second it records FP4Q_ERR_TIMEOUT in the device status word and the kernel returns, so
 * the CUDA context stays usable and the next fp4q_device_status returns FP4Q_ERR_TIMEOUT.
 * No fault, trap or unbounded wait is involved.  stream: as for the other calls. */
fp4q_status fp4q_selftest_wait_timeout(void* stream);

/* Static string for a status code. */
const char* fp4q_status_string(fp4q_status status);

/* Message of the last CUDA error seen by this library on the calling thread (or ""). */
const char* fp4q_last_cuda_error(void);

/* Library version, major * 10000 + minor * 100 + patch. */
int fp4q_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FP4Q_H_ */
