/*
 * nvfp4.h -- C ABI of the B200 (sm_100a) NVFP4 W4A4 linear-layer library.
 *
 * The operation: an NVFP4 linear layer as run on Blackwell, i.e. runtime
 * quantization of bf16 activations to NVFP4 followed by an NVFP4 x NVFP4
 * block-scaled GEMM against ModelOpt-layout weights ("BFL (fp8r / nvfp4)"
 * diffusers doc, section "Kernels", table row `nvfp4`: `nvfp4_quantize` on the
 * activations, `mm_fp4` for the GEMM).
 *
 * NVFP4 format ("NVIDIA FP4 format" news page, paragraph 1; BFL doc, `nvfp4`
 * bullet): 4-bit E2M1 elements, two per byte, one E4M3 scale per 16 elements
 * along K, plus one fp32 per-tensor scale.  This library uses the DECODE
 * convention for the per-tensor scale everywhere:
 *     x_hat = e2m1(code) * e4m3(block_scale) * g,   g = amax / (6 * 448)
 * so g is ModelOpt's `input_scale` for activations and `weight_scale_2` for
 * weights, and the GEMM's alpha is input_scale * weight_scale_2.
 *
 * Layouts (all row-major, all buffers owned by the caller):
 *   bf16 activations  x      [M, K]      2 bytes/elem
 *   codes             q      [rows, K/2] uint8; element 2j in bits 0-3 of
 *                                        byte j, element 2j+1 in bits 4-7
 *   linear scales            [rows, K/16] uint8 E4M3 (ModelOpt `weight_scale`)
 *   swizzled scales          nvfp4_sf_bytes(rows, K) bytes: rows padded to a
 *                            multiple of 128, scale columns (K/16) padded to a
 *                            multiple of 4, cut into 512-byte atoms of
 *                            128 rows x 4 scale columns stored atom-row-major;
 *                            logical (r, c) sits at byte
 *         ((r/128)*(Cp/4) + c/4)*512 + (r%32)*16 + ((r%128)/32)*4 + c%4
 *                            with Cp = padded scale columns.  Padding is 0.
 *                            This is the layout the tcgen05 block-scaled MMA
 *                            reads scale factors in.
 *   bf16 output       y      [M, N]  (GEMM; B is the weight [N, K], i.e.
 *                                     PyTorch's [out_features, in_features])
 *
 * Common contract of every entry point:
 *   - Pointers are device pointers on the current CUDA device, 16-byte
 *     aligned, unless stated otherwise.  The library allocates nothing and
 *     keeps no state besides per-device caches (device properties, the
 *     address of its device fault word and of its no-allocation scratch,
 *     each kernel's co-resident grid size).  These caches assume each
 *     device's primary context lives as long as the process: calls after a
 *     cudaDeviceReset of a device the library has already used are not
 *     supported (the cached addresses would be stale).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and is asynchronous: a return of NVFP4_OK means the work was
 *     validated and launched, not that it finished.
 *   - Arguments are validated on the host before anything is launched; an
 *     invalid call launches nothing and returns a non-zero status with a
 *     message available from nvfp4_last_error() (thread-local).
 *   - The current device must be compute capability 10.0 (B200, sm_100a);
 *     otherwise NVFP4_EARCH.  There is no CPU fallback.
 *   - K is a multiple of 64 and at least 64.
 *   - Row counts (M, N, rows) and K are at most 2^30 - 1, which keeps every
 *     row index and tile coordinate inside int32; larger sizes, and sizes
 *     whose one-dimensional launch grid would exceed 2^31 - 1 blocks, return
 *     NVFP4_EINVAL.
 *   - Per-tensor scales (g, alpha) must be finite; g must lie in
 *     [2^-64, 2^64] so that no intermediate of the quantizer overflows.
 */
#ifndef NVFP4_H_
#define NVFP4_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum nvfp4_status {
  NVFP4_OK = 0,
  NVFP4_EINVAL = 1,   /* bad size, null pointer, bad scale or range list   */
  NVFP4_EALIGN = 2,   /* a pointer or leading dimension is misaligned     */
  NVFP4_EARCH = 3,    /* current device is not compute capability 10.0    */
  NVFP4_ECUDA = 4,    /* a CUDA runtime / driver call or launch failed     */
  NVFP4_ETIMEOUT = 5  /* a kernel gave up waiting on one of its barriers   */
} nvfp4_status;

/* Activation applied by the fused epilogue to a column range. */
enum { NVFP4_ACT_NONE = 0, NVFP4_ACT_GELU_TANH = 1 };
/* Destination of a column range in the fused epilogue. */
enum { NVFP4_DST_BF16 = 0, NVFP4_DST_NVFP4 = 1 };

/* Most column ranges nvfp4_gemm_quant accepts. */
#define NVFP4_MAX_RANGES 8

/*
 * Size in bytes of the swizzled scale buffer for a [rows, k] NVFP4 tensor:
 * ceil(rows/128)*128 * ceil(k/64)*4.  Returns 0 if rows < 1 or k < 16 or
 * k % 16 != 0.  Host-only, no CUDA call.
 */
size_t nvfp4_sf_bytes(int64_t rows, int64_t k);

/*
 * Per-tensor scale calibration (BFL doc, `nvfp4` bullet: the calibrated fp32
 * `input_scale` and the global fp32 `weight_scale_2`):
 *     out[0] = amax = max |x_i| over the n bf16 values (exact)
 *     out[1] = g    = fl(amax / 2688)          (2688 = 6 * 448)
 * x is [n] bf16 with n % 8 == 0, n >= 8; out is 2 device floats (8 bytes,
 * 4-byte aligned), written.  Errors: EINVAL, EALIGN, EARCH, ECUDA.
 */
nvfp4_status nvfp4_calibrate(const void* x, int64_t n, float* out, void* stream);

/*
 * Runtime activation quantization, bf16 -> NVFP4 (BFL doc, "Kernels",
 * `nvfp4_quantize`).  For each row and each 16-element block along K, with
 * every step one IEEE fp32 operation rounded to nearest even:
 *     amax = max |x_i|;  s = E4M3_satfinite(amax / (6*g))
 *     s == 0  ->  all 16 codes 0x0
 *     else       r = 1 / (e4m3(s) * g);  code_i = E2M1_satfinite(x_i * r)
 * E2M1 rounding is to nearest, ties to the even code, saturating at +-6; the
 * code's sign bit is the sign of x_i * r (so -0 inputs give 0x8).  E4M3 never
 * produces NaN (saturates at 448).
 *   x      [M, K] bf16, read only.
 *   g      per-tensor decode scale (calibrated input_scale), in [2^-64, 2^64].
 *   codes  [M, K/2] uint8, written.
 *   sf     nvfp4_sf_bytes(M, K) bytes, written in the swizzled layout,
 *          including its zero padding rows.
 * M >= 1.  Errors: EINVAL (sizes, null, g), EALIGN, EARCH, ECUDA.
 */
nvfp4_status nvfp4_quantize(const void* x, int64_t M, int64_t K, float g,
                            uint8_t* codes, uint8_t* sf, void* stream);

/* Bytes of caller workspace one nvfp4_quantize_dynamic call uses. */
#define NVFP4_DYNAMIC_WORKSPACE_BYTES 8

/*
 * Runtime activation quantization with the per-tensor scale measured on the
 * activation itself, for a layer that has no calibrated `input_scale` (BFL
 * doc, `nvfp4` bullet: the calibrated fp32 activation scale is the default;
 * measuring it per call is the variant).  In one launch:
 *     amax = max |x_i| over the whole tensor (exact)
 *     g    = 0                                   if amax == 0
 *            min(max(fl(amax / 2688), 2^-64), 2^64)  otherwise
 *     codes, sf = nvfp4_quantize(x, g)   (all zero when g == 0)
 *   x, M, K, codes, sf  as nvfp4_quantize.
 *   scale_out  2 device floats (4-byte aligned), written: [0] = amax,
 *              [1] = g (pass &scale_out[1] to nvfp4_gemm_dynamic).
 *   workspace  device memory of at least NVFP4_DYNAMIC_WORKSPACE_BYTES
 *              (4-byte aligned) that no other work uses while the call
 *              runs; its contents on entry do not matter (the call zeroes
 *              it on the stream before the kernel), on exit they are
 *              unspecified.
 * The kernel is a cooperative launch of at most one CTA per SM: every CTA
 * folds its own tiles' maximum into the grid-wide one, then quantizes its
 * tiles once all CTAs have arrived (a bounded wait: on time-out the kernel
 * writes nothing more and records NVFP4_ETIMEOUT in the fault word).
 * Errors: EINVAL (sizes, null, workspace too small), EALIGN, EARCH, ECUDA.
 */
nvfp4_status nvfp4_quantize_dynamic(const void* x, int64_t M, int64_t K,
                                    uint8_t* codes, uint8_t* sf, float* scale_out,
                                    void* workspace, size_t workspace_bytes,
                                    void* stream);

/*
 * The dynamic-scale quantize in one pass, for an activation whose amax was
 * measured already (by nvfp4_gemm_amax when the previous layer produced it):
 *     g = 0                                   if amax[0] == 0
 *         min(max(fl(amax[0] / 2688), 2^-64), 2^64)  otherwise
 *     codes, sf = nvfp4_quantize(x, g)   (all zero when g == 0)
 * -- the rule of nvfp4_quantize_dynamic, with the amax given instead of
 * measured.  The kernel reads amax on the device (work earlier on `stream`
 * may write it); nothing is read back to the host.
 *   x, M, K, codes, sf  as nvfp4_quantize.
 *   amax       device pointer to one non-negative float (4-byte aligned).
 *   scale_out  2 device floats (4-byte aligned), written: [0] = amax,
 *              [1] = g (pass &scale_out[1] to nvfp4_gemm_dynamic).
 * One launch of the static quantizer's grid; no workspace.
 * Errors: EINVAL (sizes, null), EALIGN, EARCH, ECUDA.
 */
nvfp4_status nvfp4_quantize_from_amax(const void* x, int64_t M, int64_t K, const float* amax,
                                      uint8_t* codes, uint8_t* sf, float* scale_out,
                                      void* stream);

/* Bytes of device scratch nvfp4_quantize_dynamic_noalloc holds per device. *//* Bytes of device scratch nvfp4_quantize_dynamic_noalloc holds per device. */
#define NVFP4_NOALLOC_SCRATCH_BYTES 256

/*
 * nvfp4_quantize_dynamic without a workspace argument.  The source pages have
 * no counterpart to this entry point: it exists for callers that cannot hand
 * the library device memory of their own -- e.g. a host program or a plugin
 * that is given only its input and output buffers and has no device
 * allocator to draw a workspace from.
 *   The call allocates nothing.  Its grid state (NVFP4_DYNAMIC_WORKSPACE_BYTES)
 *   lives in a fixed array in the library's own device memory,
 *   NVFP4_NOALLOC_SCRATCH_BYTES per device; a call that would need more
 *   returns EINVAL.  The call zeroes what must start at zero on `stream`
 *   before the kernel.
 *   First call on each device: looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current, once; make that first
 *   call outside any stream capture.
 *   Calls that overlap in time on the same device (other streams, other host
 *   threads) share the array and race: order them, e.g. on one stream.
 * Arguments, results and errors as nvfp4_quantize_dynamic (ECUDA also if the
 * address lookup fails).
 */
nvfp4_status nvfp4_quantize_dynamic_noalloc(const void* x, int64_t M, int64_t K,
                                            uint8_t* codes, uint8_t* sf, float* scale_out,
                                            void* stream);

/*
 * Weight preparation: scatter ModelOpt's row-major E4M3 `weight_scale`
 * [rows, k/16] into the swizzled layout the GEMM reads (a byte permutation;
 * padding bytes are written as 0).  sf_linear needs no alignment;
 * sf_swizzled (nvfp4_sf_bytes(rows, k) bytes) must be 16-byte aligned.
 * rows >= 1, k % 64 == 0.  Errors: EINVAL, EALIGN, EARCH, ECUDA.
 */
nvfp4_status nvfp4_swizzle_sf(const uint8_t* sf_linear, int64_t rows, int64_t k,
                              uint8_t* sf_swizzled, void* stream);

/*
 * Block-scaled NVFP4 GEMM with the dequant folded into the epilogue
 * (BFL doc, "Kernels", `mm_fp4`):
 *     y[m, n] = bf16_rn( alpha * sum_k a_hat[m,k] * b_hat[n,k] + bias[n] )
 * with a_hat = e2m1(a) * e4m3(sfa) and b_hat likewise; the sum is
 * accumulated in fp32 by the tensor cores (tcgen05, kind::mxf4nvf4, one
 * E4M3 scale per 16 elements).
 *   a     [M, K/2] codes (activations), sfa swizzled nvfp4_sf_bytes(M, K)
 *   b     [N, K/2] codes (weights),     sfb swizzled nvfp4_sf_bytes(N, K)
 *   alpha input_scale * weight_scale_2 (finite)
 *   bias  [N] bf16 or NULL
 *   y     [M, N] bf16, written
 * M >= 1, N >= 8 with N % 8 == 0.  Errors: EINVAL, EALIGN, EARCH, ECUDA.
 * A barrier wait inside the kernel that exceeds its time limit makes the
 * kernel return early and record NVFP4_ETIMEOUT in the device fault word
 * (see nvfp4_check_fault).
 */
nvfp4_status nvfp4_gemm(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                        const uint8_t* sfb, int64_t M, int64_t N, int64_t K,
                        float alpha, const void* bias, void* y, void* stream);

/*
 * nvfp4_gemm with the two per-tensor scales passed apart, as a ModelOpt layer
 * stores them (BFL doc, `nvfp4` bullet: `input_scale` and `weight_scale_2`):
 * the epilogue forms alpha = fl(g_a * g_b) itself (one fp32 product, the same
 * value a caller computing input_scale * weight_scale_2 in fp32 passes to
 * nvfp4_gemm).
 *   g_a  the activation's per-tensor scale (input_scale), finite
 *   g_b  the weight's per-tensor scale (weight_scale_2), finite
 *   with g_a * g_b finite.  Other arguments and errors as nvfp4_gemm.
 */
nvfp4_status nvfp4_gemm_scaled(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                               const uint8_t* sfb, int64_t M, int64_t N, int64_t K,
                               float g_a, float g_b, const void* bias, void* y,
                               void* stream);

/*
 * nvfp4_gemm for an activation whose per-tensor scale was measured on the
 * device (nvfp4_quantize_dynamic): the epilogue reads g_a from device memory
 * and uses alpha = fl(g_a[0] * g_b) (the same single fp32 product as
 * input_scale * weight_scale_2).
 *   g_a  device pointer to one float (4-byte aligned), read by the kernel;
 *        work earlier on `stream` may write it.
 *   g_b  the weight's per-tensor scale (weight_scale_2), finite.
 * Other arguments and errors as nvfp4_gemm.
 */
nvfp4_status nvfp4_gemm_dynamic(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                                const uint8_t* sfb, int64_t M, int64_t N, int64_t K,
                                float g_b, const float* g_a, const void* bias, void* y,
                                void* stream);

/*
 * The GEMM of nvfp4_gemm_scaled / nvfp4_gemm_dynamic that also measures its
 * output for the next layer's dynamic scale (a measured activation scale in
 * place of the calibrated input_scale, "BFL (fp8r / nvfp4)" doc, nvfp4
 * bullet, with the amax taken by the previous layer's epilogue: the next
 * layer then quantizes in one pass with nvfp4_quantize_from_amax instead of
 * the two passes of nvfp4_quantize_dynamic).
 *     Y = bf16( fl(g * g_b) * acc + bias ),  g = g_a_device ? g_a_device[0] : g_a
 *     amax_out[0] = max(amax_out[0], max |Y[m, n]|)  over the M x N outputs
 * The maximum is taken over the bf16 values written (a NaN counts as +inf)
 * and folded in with an atomic max on the float's bit pattern, so amax_out[0]
 * must hold a non-negative float on entry (zero it to measure one GEMM; leave
 * it to take the maximum over several).
 *   g_a         the activation's per-tensor scale (used when g_a_device is
 *               NULL; then g_a * g_b must be finite)
 *   g_a_device  nullable device pointer to one float (4-byte aligned), e.g.
 *               &scale_out[1] of a dynamic or one-pass quantize
 *   g_b         the weight's per-tensor scale, finite
 *   amax_out    device pointer to one float (4-byte aligned)
 * Other arguments and errors as nvfp4_gemm.
 */
nvfp4_status nvfp4_gemm_amax(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                             const uint8_t* sfb, int64_t M, int64_t N, int64_t K,
                             float g_a, const float* g_a_device, float g_b,
                             const void* bias, void* y, float* amax_out, void* stream);

/* One column range of the fused epilogue. *//* One column range of the fused epilogue. */
typedef struct nvfp4_colrange {
  int64_t begin;   /* first GEMM output column of the range              */
  int64_t end;     /* one past the last column                           */
  int32_t act;     /* NVFP4_ACT_NONE or NVFP4_ACT_GELU_TANH              */
  int32_t dst;     /* NVFP4_DST_BF16 or NVFP4_DST_NVFP4                  */
  int64_t dst_col; /* first column written in the destination tensor     */
} nvfp4_colrange;

/*
 * GEMM with a fused epilogue that writes the next layer's input.  For every
 * output column n in range i:
 *     v = bf16_rn(alpha * acc[m,n] + bias[n])
 *     if act == GELU_TANH:  v = bf16_rn(gelu_tanh(v))
 *       (0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3))), fp32)
 *     dst == BF16:   y_bf16[m, dst_col + n - begin] = v
 *     dst == NVFP4:  v (bf16) is quantized exactly as nvfp4_quantize does,
 *                    with scale g_next, into column dst_col + n - begin of
 *                    the [M, k_next] NVFP4 tensor (codes_next, sf_next).
 * Columns outside every range are dropped.  Ranges must not overlap; at most
 * NVFP4_MAX_RANGES; begin, end and dst_col multiples of 64; end <= N;
 * dst_col + (end - begin) <= ldy (BF16) or <= k_next (NVFP4).  The NVFP4
 * destination's scale padding rows are written as zero; its scale columns
 * belonging to no range are left untouched.
 *   y_bf16     [M, ldy] bf16 (NULL if no BF16 range), ldy % 8 == 0
 *   codes_next [M, k_next/2] uint8, sf_next nvfp4_sf_bytes(M, k_next)
 *              (NULL if no NVFP4 range), k_next % 64 == 0
 * Other arguments as nvfp4_gemm.  Errors: EINVAL, EALIGN, EARCH, ECUDA.
 */
nvfp4_status nvfp4_gemm_quant(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                              const uint8_t* sfb, int64_t M, int64_t N, int64_t K,
                              float alpha, const void* bias,
                              const nvfp4_colrange* ranges, int32_t n_ranges,
                              void* y_bf16, int64_t ldy,
                              float g_next, uint8_t* codes_next, uint8_t* sf_next,
                              int64_t k_next, void* stream);

/*
 * nvfp4_gemm_quant with the two per-tensor scales passed apart (alpha =
 * fl(g_a * g_b) formed by the epilogue, as in nvfp4_gemm_scaled).  Arguments
 * and errors as nvfp4_gemm_quant, with g_a, g_b finite and their product
 * finite in place of alpha.
 */
nvfp4_status nvfp4_gemm_quant_scaled(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                                     const uint8_t* sfb, int64_t M, int64_t N, int64_t K,
                                     float g_a, float g_b, const void* bias,
                                     const nvfp4_colrange* ranges, int32_t n_ranges,
                                     void* y_bf16, int64_t ldy,
                                     float g_next, uint8_t* codes_next, uint8_t* sf_next,
                                     int64_t k_next, void* stream);

/*
 * ------------------------------------------------------------------------
 * MXFP8 variant ("NVIDIA FP4 format" news page, paragraph 1: 8-bit E4M3/E5M2
 * elements in 32-element blocks, Open Compute Project microscaling; the
 * page's 1.26x end-to-end figure for MXFP8 next to NVFP4's 1.68x).  E4M3
 * elements, one E8M0 scale (a power of two, 2^(byte - 127)) per 32 elements
 * along K, no per-tensor scale.
 *   codes   [rows, K] uint8, one E4M3 byte per element
 *   scales  nvfp4_mxfp8_sf_bytes(rows, K) bytes: the same 512-byte atom
 *           layout as the NVFP4 scales, with one scale column per 32
 *           elements (K/32 columns padded to a multiple of 4; padding 0)
 * ------------------------------------------------------------------------
 */

/* Size of the swizzled MXFP8 scale buffer: ceil(rows/128)*128 *
 * ceil(k/128)*4.  0 if rows < 1 or k < 32 or k % 32 != 0.  Host-only. */
size_t nvfp4_mxfp8_sf_bytes(int64_t rows, int64_t k);

/*
 * bf16 -> MXFP8.  For each row and each 32-element block along K:
 *     amax = max |x_i|
 *     amax == 0:  scale byte 0;  codes E4M3(x_i) (zeros, sign kept)
 *     else        s = clamp(floor(log2 amax) - 8, -127, 127);  scale byte s + 127
 *                 code_i = E4M3_satfinite(fl(x_i * 2^-s))   (RNE, +-448)
 * (the microscaling conversion: 8 is the exponent of E4M3's largest normal,
 * 448 = 1.75 * 2^8, so the block maximum lands in [256, 448]).
 *   x      [M, K] bf16, finite
 *   codes  [M, K] uint8, written;  sf  nvfp4_mxfp8_sf_bytes(M, K), written
 *          including its zero padding.
 * M >= 1, K % 64 == 0.  Errors: EINVAL, EALIGN, EARCH, ECUDA.
 */
nvfp4_status nvfp4_mxfp8_quantize(const void* x, int64_t M, int64_t K,
                                  uint8_t* codes, uint8_t* sf, void* stream);

/*
 * Block-scaled MXFP8 GEMM on the tensor cores (tcgen05, kind::mxf8f6f4, one
 * E8M0 scale per 32 elements), dequant folded into the epilogue:
 *     y[m, n] = bf16_rn( alpha * sum_k a_hat[m,k] * b_hat[n,k] + bias[n] )
 * with a_hat = e4m3(a) * 2^(sfa - 127), b_hat likewise.
 *   a  [M, K] codes, sfa nvfp4_mxfp8_sf_bytes(M, K);  b [N, K] codes (the
 *   weight, PyTorch [out, in]), sfb nvfp4_mxfp8_sf_bytes(N, K);
 *   alpha finite (1 for a plain MXFP8 layer);  bias [N] bf16 or NULL;
 *   y [M, N] bf16, written.
 * M >= 1, N >= 8 with N % 8 == 0, K % 64 == 0.  Errors: EINVAL, EALIGN,
 * EARCH, ECUDA; a barrier time-out records NVFP4_ETIMEOUT (nvfp4_check_fault).
 */
nvfp4_status nvfp4_mxfp8_gemm(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                              const uint8_t* sfb, int64_t M, int64_t N, int64_t K,
                              float alpha, const void* bias, void* y, void* stream);

/*
 * ------------------------------------------------------------------------
 * Row-wise FP8 (W8A8) variant (BFL doc, `fp8r` bullet and "Kernels" row
 * `fp8r`: an E4M3 `weight` with one fp32 `weight_scale` per row;
 * activations quantized to E4M3 row by row at run time; the GEMM applies the
 * row scales).  No block scales, no per-tensor scale.
 * ------------------------------------------------------------------------
 */

/*
 * bf16 -> row-wise FP8, for activations at run time (and for weights once):
 *     s[m] = fl(amax(|x[m, :]|) / 448)
 *     code = E4M3_satfinite(fl(x[m, k] / s[m]))   (RNE, +-448)
 *   a row of zeros gets s = 0 and the codes of +-0.
 *   x      [M, K] bf16, finite
 *   codes  [M, K] uint8 E4M3, written;  scale  [M] fp32, written
 * M >= 1, K % 64 == 0, all pointers 16-byte aligned.
 * Errors: EINVAL, EALIGN, EARCH, ECUDA.
 */
nvfp4_status nvfp4_fp8row_quantize(const void* x, int64_t M, int64_t K,
                                   uint8_t* codes, float* scale, void* stream);

/*
 * Row-wise FP8 GEMM on the tensor cores (tcgen05, kind::f8f6f4, E4M3 x E4M3
 * -> fp32 accumulation), scales folded into the epilogue:
 *     y[m, n] = bf16_rn( fl(a_scale[m] * b_scale[n]) * acc[m, n] + bias[n] )
 *   a [M, K] codes, a_scale [M];  b [N, K] codes (the weight, PyTorch
 *   [out, in]), b_scale [N] (16-byte aligned);  bias [N] bf16 or NULL;
 *   y [M, N] bf16, written.
 * M >= 1, N >= 8 with N % 8 == 0, K % 64 == 0.  Errors: EINVAL, EALIGN,
 * EARCH, ECUDA; a barrier time-out records NVFP4_ETIMEOUT.
 */
nvfp4_status nvfp4_fp8row_gemm(const uint8_t* a, const float* a_scale, const uint8_t* b,
                               const float* b_scale, int64_t M, int64_t N, int64_t K,
                               const void* bias, void* y, void* stream);

/*
 * W4A16 path (BFL doc, "Kernels", last paragraph: where the fused kernels do
 * not run, the NVFP4 weights are dequantized to the compute dtype on every
 * forward and the layer runs as a regular linear with bf16 activations):
 * NVFP4 -> bf16,
 *     out[r, k] = bf16_rn( fl( fl(e2m1(code) * e4m3(scale)) * g ) )
 * (the first product is exact in fp32).  nvfp4_w4a16_gemm runs the whole
 * layer without storing these values; this call materializes them.
 *   codes [rows, K/2], sf swizzled nvfp4_sf_bytes(rows, K), g finite;
 *   out   [rows, K] bf16, written.
 * rows >= 1, K % 64 == 0.  Errors: EINVAL, EALIGN, EARCH, ECUDA.
 */
nvfp4_status nvfp4_dequantize(const uint8_t* codes, const uint8_t* sf, float g,
                              int64_t rows, int64_t K, void* out, void* stream);

/*
 * W4A16 linear layer in one kernel (BFL doc, "Kernels", last paragraph: the
 * NVFP4 weights dequantized to the compute dtype, the activations left in
 * bf16, a regular linear):
 *     y[m, n] = bf16_rn( sum_k x[m, k] * w[n, k] + bias[n] )
 *     w[n, k] = bf16_rn( fl( fl(e2m1(code) * e4m3(scale)) * g_w ) )
 * -- exactly the values nvfp4_dequantize writes, formed tile by tile in shared
 * memory and never stored -- with the sum accumulated in fp32 by the tensor
 * cores (tcgen05, kind::f16, bf16 x bf16).
 *   x        [M, K] bf16 activations
 *   w_codes  [N, K/2] NVFP4 weight codes, w_sf swizzled nvfp4_sf_bytes(N, K),
 *   g_w      the weight's per-tensor scale (weight_scale_2), finite
 *   bias     [N] bf16 or NULL;  y  [M, N] bf16, written
 * M >= 1, N >= 8 with N % 8 == 0, K % 64 == 0; the same tile shapes as
 * nvfp4_gemm.  Errors: EINVAL, EALIGN, EARCH, ECUDA; a barrier time-out
 * records NVFP4_ETIMEOUT (nvfp4_check_fault).
 */
nvfp4_status nvfp4_w4a16_gemm(const void* x, const uint8_t* w_codes, const uint8_t* w_sf,
                              int64_t M, int64_t N, int64_t K, float g_w, const void* bias,
                              void* y, void* stream);

/*
 * Synchronize the current device, then read and clear its fault word.
 * Returns NVFP4_ETIMEOUT if any kernel of this library gave up on a barrier
 * wait since the last check, NVFP4_ECUDA if the synchronize failed, else
 * NVFP4_OK.
 */
nvfp4_status nvfp4_check_fault(void);

/*
 * For tests of the failure path only: sets, for the dynamic quantizes
 * (nvfp4_quantize_dynamic, nvfp4_quantize_dynamic_noalloc) that the calling
 * host thread launches from now on, how long the kernel's grid-wide wait
 * lasts (limit_ns; 0 restores the default of one second) and how many
 * arrivals beyond the grid size it waits for (extra_arrivals; 0 restores the
 * default).  With extra_arrivals > 0 the wait cannot complete: every CTA gives
 * up after limit_ns, writes no codes, scales or scale_out, and records
 * NVFP4_ETIMEOUT in the device fault word (nvfp4_check_fault reports it).  No
 * other wait and no other entry point is affected.  The pages have no
 * counterpart; the failure behaviour it exercises is this library's own.
 * limit_ns <= 10^9, extra_arrivals <= 1024.  Host only.  Errors: EINVAL.
 */
nvfp4_status nvfp4_testing_set_grid_wait(uint64_t limit_ns, uint32_t extra_arrivals);

/*
 * Launch shapes the library picks, for callers that size work around them
 * and for tests (host only: nothing touches a device).  Every GEMM entry point
 * (NVFP4, fused, dynamic, MXFP8, row-wise FP8) takes the same tile shape for
 * the same M, N and SM count:
 *   out[0] = CTAs per output tile (1, or 2 for a CTA pair),
 *   out[1] = tile width in output columns (128, 192 or 256),
 *   out[2] = accumulator buffers in TMEM (1 or 2);
 * the tile height is 128 * out[0] rows.  The rule: M <= 128 takes one CTA and
 * 192 columns; otherwise 256 x 256 pair tiles when there are at least
 * num_sms / 2 of them, else 256 x 128 when those still fit in one wave and
 * 256 x 192 ones would not fill it, else 256 x 192.
 * Errors: EINVAL (null out, M or N out of range, num_sms < 2).
 */
nvfp4_status nvfp4_gemm_tile_shape(int64_t M, int64_t N, int32_t num_sms, int32_t* out);

/*
 * Launch plan of the GEMMs with the plain epilogue -- nvfp4_gemm,
 * nvfp4_gemm_scaled, nvfp4_gemm_dynamic, nvfp4_gemm_amax (w4a16 = 0) and nvfp4_w4a16_gemm
 * (w4a16 = 1) -- for an M x N x K problem on num_sms SMs (host only):
 *   out[0..2] = tile shape as nvfp4_gemm_tile_shape reports it,
 *   out[3]    = K split: tile groups (CTAs or CTA pairs) that share one
 *               output tile over disjoint ranges of k-tiles (1, 2 or 4).
 * When the tiles cannot fill the SMs (a few hundred tokens or fewer) and K is
 * long enough for the split to pay for its own work, up to 4 CTAs of a
 * thread-block cluster work on one tile, each over its own k-tile range
 * (k-tiles of 256 elements for NVFP4, 64 for W4A16), and sum their fp32
 * partial tiles through distributed shared memory in a fixed order before the
 * epilogue (so results are deterministic; they may differ from the unsplit
 * sum in the last bits, within the GEMM's tolerance).  The shape is then the
 * one of 256 x 192 or 256 x 128 (M > 128) that leaves each CTA group the
 * fewest k-tiles.  The fused, MXFP8 and row-wise FP8 GEMMs never split K.
 * Errors: EINVAL (null out, sizes out of range).
 */
nvfp4_status nvfp4_gemm_plan(int64_t M, int64_t N, int64_t K, int32_t num_sms, int32_t w4a16,
                             int32_t* out);

/*
 * Rows per tile of the NVFP4 and MXFP8 quantizers for an [M, K] input on a
 * device with num_sms SMs: 256 once every SM gets at least eight 256-row
 * tiles of 64 columns, else 128.  0 for invalid sizes (M or K out of range,
 * K not a multiple of 64, num_sms < 1).  Host only.
 */
int32_t nvfp4_quantize_tile_rows(int64_t M, int64_t K, int32_t num_sms);

/* Message describing the last error of the calling thread ("" if none).
 * The pointer stays valid until the thread's next call into the library. */
const char* nvfp4_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H_ */
