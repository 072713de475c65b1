/*
 * signrot.h -- C ABI of the SignRot online down-projection activation path on B200 (sm_100a).
 *
 * Per token row x in R^n (the input of a LLaMA MLP's down projection) the path computes
 *
 *     y = diag(s) . H . diag(D) . x / sqrt(n)                       (rotation + sign adjustment)
 *     lo, hi = min_j y_j, max_j y_j
 *     scale = (hi - lo) / 15,  zero = rne(-lo / scale)              (asymmetric per-token grid)
 *     q_j = clamp(rne(y_j / scale) + zero, 0, 15)                   (INT4 codes, two per byte)
 *
 * Sources. "SignRot: LLM Quantization with Massive Outlier-Aware Sign-Adjusted Rotation" (arXiv
 * 2611.16502, abstract): the randomized Hadamard rotation applied online at the down-projection
 * input by the fast Walsh-Hadamard transform, the sign adjustment vector built from the massive
 * outlier channel found in one calibration pass, and asymmetric activation quantization. "SignRot
 * for 4-bit LLM quantization -- Sign-adjusted Hadamard rotation" (learnaivisually.com explainer),
 * paragraphs "Picture the photographer" (16 levels from the token's smallest to largest value),
 * "The standard fix is rotation" (entries +/-1/sqrt(n)), "SignRot asks one crowd to walk across
 * the hall" (largest absolute calibration activation; per-output sign of the outlier's entry),
 * "The flip alone does nothing for a symmetric quantizer" (asymmetric zero-point) and "Worked
 * example" (steps are range/15, no clipping).
 *
 * H = H_F kron H_M with n = F * M, F in {1, 28, 344}, M = 2^m, channel j = a * M + b. H_M is
 * Sylvester's (H_M[b][e] = (-1)^popcount(b & e)); H_28 and H_344 are Paley's construction I
 * over GF(27) = GF(3)[t]/(t^3 + 2t + 1) and GF(343) = GF(7)[t]/(t^3 + t + 1): row 0 all +1,
 * column 0 = (1, -1, ..., -1), H[1+e][1+f] = [e == f] + chi(e - f) with field element
 * e = c0 + p c1 + p^2 c2 and chi the quadratic character (see signrot_get_h28/_h344).
 * Supported n: 2^m for 1 <= m <= 15, 28 * 2^m for 0 <= m <= 10, and 344 * 2^m for
 * 0 <= m <= 5 (n = 11008 = 344 * 32 is LLaMA-2-7B's MLP width, the example in the
 * explainer's paragraph "Here is how it breaks"). F = 344 runs on the generic kernel (fp64
 * accumulation on the CUDA cores).
 *
 * Conventions shared by every call:
 *   - Every call returns a signrot_status; nothing is thrown across the ABI.
 *   - Tensors are caller-owned DEVICE pointers unless a parameter says host. The library
 *     allocates no device memory.
 *   - Work is enqueued on `stream` (a cudaStream_t passed as void*, NULL = legacy default stream)
 *     and is asynchronous: a return of SIGNROT_OK means the launch was accepted. Device-side
 *     faults surface on the caller's next synchronisation, as for any CUDA kernel.
 *   - Activation rows are row-major: row t starts at element t * ld (ld >= n, in elements).
 *   - T == 0 is a no-op that returns SIGNROT_OK.
 *   - Inputs must be finite; a NaN or Inf in x gives unspecified codes (no fault).
 */
#ifndef SIGNROT_H
#define SIGNROT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t signrot_status;
#define SIGNROT_OK 0
#define SIGNROT_ERR_INVALID_ARG 1   /* null pointer, negative size, ld < n, bad dtype, ... */
#define SIGNROT_ERR_UNSUPPORTED_N 2 /* n not of a supported form (see above)              */
#define SIGNROT_ERR_ALIGNMENT 3     /* pointer not aligned to its element type            */
#define SIGNROT_ERR_CUDA 4          /* a CUDA runtime call failed; see signrot_last_error */
#define SIGNROT_ERR_UNSUPPORTED 5   /* e.g. bits != 4, clip outside (0, 1]                 */

/* Storage type of the activations x. */
#define SIGNROT_BF16 0
#define SIGNROT_F32 1

/*
 * signrot_calibrate -- per-channel max |x| over calibration tokens, then the outlier channel.
 *
 * Follows the abstract's "single calibration forward pass" and the explainer's "finds the channel
 * with the largest absolute activation". Reads x[T, n] (dtype, leading dimension ld) and folds it
 * into the workspace ws[n] (uint64, device, caller-owned, 8 * n bytes), which keeps for every
 * channel i the largest |x_{t,i}| seen, the first token index attaining it and that value's sign.
 * Token indices are t_offset + t, so a calibration set streamed in chunks keeps "first token"
 * global (0 <= t_offset, t_offset + T <= 2^31 - 1).
 *   accumulate == 0: ws is reset first (this call starts a new calibration);
 *   accumulate != 0: this chunk is folded into what ws already holds.
 * After folding, writes k_out[0] (int32, device) = the lowest channel index attaining
 * max_i max_t |x_{t,i}|, and xk_out[0] (float, device) = the signed value x_{t*,k} at the first
 * token t* attaining it. T == 0 with accumulate != 0 only recomputes k and x_k from ws.
 */
signrot_status signrot_calibrate(const void* x, int32_t dtype, int64_t T, int32_t n, int64_t ld,
                                 int64_t t_offset, uint64_t* ws, int32_t accumulate,
                                 int32_t* k_out, float* xk_out, void* stream);

/*
 * signrot_calibrate_static -- signrot_calibrate without a caller workspace. (Not from the SignRot
 * pages, which have no counterpart: it exists for callers that cannot allocate device memory.)
 *
 * Some callers cannot hand the library an 8 * n byte device workspace: runtimes that reserve all
 * device memory in one pool at start-up and forbid later cudaMalloc calls, plugins whose host
 * framework owns the allocator and passes them only inputs and outputs, and latency-bound code
 * that must not risk the device-wide synchronisation a cudaMalloc or cudaFree can cause. This call
 * takes the same arguments as signrot_calibrate minus ws, and keeps the per-channel keys in a
 * fixed array inside the library's device image (SIGNROT_STATIC_SCRATCH_MAX_N channels, 256 KB,
 * held on every GPU that loads the library until the process exits). It allocates nothing.
 *   - Arguments are checked as for signrot_calibrate, before any CUDA call. The array holds
 *     every supported row length; an n beyond SIGNROT_STATIC_SCRATCH_MAX_N is not a supported
 *     form and returns SIGNROT_ERR_UNSUPPORTED_N with a message.
 *   - The first call on a device looks the array's device address up (cudaGetSymbolAddress with
 *     that device current) and caches it; make that first call before any stream capture. The
 *     cache assumes the device's primary context is never reset: after cudaDeviceReset the
 *     library image is reloaded and this entry point must not be called again in that process.
 *   - All calls on a device share the one array, and it keeps the last call's contents:
 *     accumulate == 0 clears it first; accumulate != 0 folds into whatever the previous call on
 *     that device left there. Calls that overlap on the GPU (other streams, other host threads)
 *     race on the array; serialise them.
 */
#define SIGNROT_STATIC_SCRATCH_MAX_N 32768
signrot_status signrot_calibrate_static(const void* x, int32_t dtype, int64_t T, int32_t n, int64_t ld,
                                        int64_t t_offset, int32_t accumulate, int32_t* k_out,
                                        float* xk_out, void* stream);

/*
 * signrot_build_sign -- the sign adjustment vector s.
 *
 * Follows the explainer's "SignRot asks one crowd to walk across the hall": every output j is
 * multiplied by the sign of the outlier column's entry, so the outlier adds the same +|M|/sqrt(n)
 * to every output. Here s_j = +1 if H[j][k] * D_k * x_k >= 0 else -1, with k = k[0] and
 * x_k = xk[0] read on the device (as written by signrot_calibrate). d[n] and s_out[n] are int8
 * +/-1, device. Passing x_k > 0 gives the literal "sign of that row's entry" form.
 */
signrot_status signrot_build_sign(int32_t n, const int32_t* k, const float* xk, const int8_t* d,
                                  int8_t* s_out, void* stream);

/*
 * signrot_rotate -- the rotated, sign-adjusted rows in fp32 (the check path).
 *
 * y[t * ldy + j] = s_j * (H . diag(D) . x_t)_j / sqrt(n) for t < T, j < n. d[n] int8 +/-1;
 * s[n] int8 +/-1 or NULL (all +1); y float, device, ldy >= n. Follows "The standard fix is
 * rotation" (entries +/-1/sqrt(n), every output a signed sum of all inputs) and the abstract's
 * fast Walsh-Hadamard transform.
 */
signrot_status signrot_rotate(const void* x, int32_t dtype, int64_t T, int32_t n, int64_t ld,
                              const int8_t* d, const int8_t* s, float* y, int64_t ldy,
                              void* stream);

/*
 * signrot_rotate_quant -- the fused online path: rotate, sign-adjust, quantize to packed INT4.
 *
 * For each row t: y as in signrot_rotate, then with c = clip, lo = c * min y, hi = c * max y:
 *   scale[t] = (hi - lo) / 15, zero[t] = rne(-lo / scale[t])   (fp32; zero is integer-valued and
 *   usually far outside [0, 15], which is why it is stored as fp32)
 *   code_j = clamp(rne(y_j / scale[t]) + zero[t], 0, 15)       (rne: nearest, ties to even)
 *   a row with hi == lo gets scale = 1, zero = rne(-lo).
 * q[t * (n / 2) + i] = code_{2i} | code_{2i+1} << 4 (uint8, device, [T, n/2] row-major; n even).
 * Dequantize with (code - zero) * scale. clip in (0, 1] (1 = no clipping, as in the worked
 * example). s may be NULL (plain rotation, no sign adjustment).
 * bits = 8 gives the same grid with 255 levels (/ 255 and clamp(., 0, 255) above) and one code per
 * byte: q[t * n + j] = code_j ([T, n]). Any other bits -> SIGNROT_ERR_UNSUPPORTED.
 * The codes are decided in fp32 with the reciprocal of the scale, so a code may differ by one
 * from the formula above where y / scale lies within an ulp of a half-integer.
 */
signrot_status signrot_rotate_quant(const void* x, int32_t dtype, int64_t T, int32_t n, int64_t ld,
                                    const int8_t* d, const int8_t* s, int32_t bits, float clip,
                                    uint8_t* q, float* scale, float* zero, void* stream);

/*
 * signrot_rotate_outlier / signrot_rotate_quant_outlier -- the same two calls with the sign
 * adjustment given by its outlier channel instead of a materialised s: k[0] (int32, device) and
 * x_k = xk[0] (float, device), as written by signrot_calibrate. The result equals calling
 * signrot_rotate(_quant) with s = signrot_build_sign(n, k, xk, d), bit for bit on the fused
 * kernels for n >= 7168 (F = 28) or n >= 8192. For the short rows n = 3584 and 4096 (bf16) the
 * outlier form runs a kernel that tiles four tokens per tensor-core tile, keeping channel k out
 * of its fp32 sums and adding its exact contribution once at the end; for n = 512, 1024 and 2048
 * (fp32 or bf16, rows 16-byte aligned) it runs one that gives each token one warp and fp64 sums.
 * A sign vector takes the exact generic kernel on these shapes; all give the formula's codes
 * except at rounding ties.
 * Because
 * s_j = sgn(H[j][k] D_k x_k) is a signed column of H, it factorises along the
 * Kronecker structure and is folded into the rotation itself, so the sign adjustment costs no
 * per-element work (the explainer's "at inference the only new work is an element-wise sign
 * flip", taken to zero). x_k == 0 means s = +1 everywhere.
 */
signrot_status signrot_rotate_outlier(const void* x, int32_t dtype, int64_t T, int32_t n, int64_t ld,
                                      const int8_t* d, const int32_t* k, const float* xk, float* y,
                                      int64_t ldy, void* stream);
signrot_status signrot_rotate_quant_outlier(const void* x, int32_t dtype, int64_t T, int32_t n,
                                            int64_t ld, const int8_t* d, const int32_t* k,
                                            const float* xk, int32_t bits, float clip, uint8_t* q,
                                            float* scale, float* zero, void* stream);

/*
 * signrot_rotate_quant_sym / signrot_rotate_quant_sym_outlier -- the same path with the
 * symmetric per-token grid instead (the explainer's comparison grid, "Worked example": levels
 * spaced evenly on both sides of zero): L = 2^(bits-1) - 1 (7 for bits = 4, 127 for bits = 8),
 *   scale[t] = max_j |y_j| / L  (1 for an all-zero row),  code_j = clamp(rne(y_j / scale[t]), -L, L).
 * bits = 4: q [T, n/2], q[t * (n/2) + i] = (code_{2i} & 15) | (code_{2i+1} & 15) << 4 (two's
 * complement nibbles); bits = 8: q [T, n] as int8. No zero-point and no clip. The sign
 * adjustment is s (or NULL) or, in the _outlier form, k and xk as for
 * signrot_rotate_quant_outlier. Codes are decided as in signrot_rotate_quant (reciprocal of the
 * scale on the fused kernel: a code may differ by one where y / scale is within an ulp of a
 * half-integer).
 */
signrot_status signrot_rotate_quant_sym(const void* x, int32_t dtype, int64_t T, int32_t n, int64_t ld,
                                        const int8_t* d, const int8_t* s, int32_t bits, uint8_t* q,
                                        float* scale, void* stream);
signrot_status signrot_rotate_quant_sym_outlier(const void* x, int32_t dtype, int64_t T, int32_t n,
                                                int64_t ld, const int8_t* d, const int32_t* k,
                                                const float* xk, int32_t bits, uint8_t* q, float* scale,
                                                void* stream);

/*
 * signrot_rotate_quant_host -- the fused path between HOST buffers: x_host [T, ld] (pinned for
 * overlap; pageable works but serialises) -> q_host [T, n/2], scale_host [T], zero_host [T].
 * d (device, [n]) as above; the sign adjustment is s (device [n], or NULL) or, when k and xk
 * (device) are both given, the outlier channel (then s must be NULL). The rows are streamed
 * through the caller's device workspace in chunks: each chunk's host-to-device copy, kernel and
 * device-to-host copy are enqueued on one of two library streams (created once per device), so
 * copies in both directions overlap the neighbouring chunks. workspace must hold at least
 * 2 * signrot_host_bytes_per_token(n, dtype) bytes (16-byte aligned); the chunk length is what
 * fits in half of it. The caller's stream waits for all of it before its next work; the host
 * outputs are complete once that stream is synchronised.
 */
signrot_status signrot_rotate_quant_host(const void* x_host, int32_t dtype, int64_t T, int32_t n,
                                         int64_t ld, const int8_t* d, const int8_t* s,
                                         const int32_t* k, const float* xk, int32_t bits, float clip,
                                         uint8_t* q_host, float* scale_host, float* zero_host,
                                         void* workspace, size_t workspace_bytes, void* stream);

/* Device workspace bytes one token needs in signrot_rotate_quant_host (input row + outputs). */
size_t signrot_host_bytes_per_token(int32_t n, int32_t dtype);

/*
 * Host, synchronous: writes the device error word of the current device to *code (0 = none;
 * bit 0 = a fused kernel's (or the W4A4 product's) bounded wait on its own pipeline expired and
 * the kernel stopped early, leaving its outputs incomplete; bit 1 = an outlier channel index out
 * of range) and clears it when clear != 0.
 */
signrot_status signrot_device_error(int32_t* code, int32_t clear);

/*
 * signrot_w4a4_prepare_weights -- offline step of the consumer side: unpack the down projection's
 * 4-bit weight codes and sum each output row.
 *
 * Follows the explainer's "SignRot asks one crowd to walk across the hall" (the rotation and the
 * sign flip are folded into the weights offline: W' = W R^T, which is signrot_rotate applied to
 * the rows of W with the same d and sign adjustment) and "The flip alone does nothing for a
 * symmetric quantizer" (the zero-point's correction is the zero-point times a precomputed column
 * sum of the weights). wq4 [N, K/2] (device, row stride ldw4 bytes) holds per-output-row symmetric
 * 4-bit codes as signrot_rotate_quant_sym(bits = 4) writes them (two's complement nibbles,
 * element 2i low); writes wq8 [N, K] int8 (row stride ldw8 bytes), one code per byte, and
 * colsum[N] int32, colsum[o] = sum_j wq8[o][j]. K even.
 */
signrot_status signrot_w4a4_prepare_weights(const uint8_t* wq4, int32_t N, int32_t K, int64_t ldw4,
                                            int8_t* wq8, int64_t ldw8, int32_t* colsum, void* stream);

/*
 * signrot_w4a4_matmul -- the down projection on the packed codes (tcgen05 int8 tensor cores):
 *
 *     out[t][o] = scale[t] * wscale[o] * (sum_j code_tj * wq8[o][j] - zero[t] * colsum[o])
 *
 * for t < T, o < N, j < K: code_tj the activation codes 0..15 as signrot_rotate_quant writes them
 * (q [T, K/2], row stride ldq bytes, element 2i in the low nibble) with their scale[T] and zero[T];
 * zero = NULL means the symmetric grid instead: code_tj is the signed nibble (-8..7, two's
 * complement) that signrot_rotate_quant_sym(bits = 4) writes and the zero term is absent.
 * wq8 [N, K] int8 weight codes in [-8, 7] (row
 * stride ldw bytes) with per-row scales wscale[N] and colsum[N] from
 * signrot_w4a4_prepare_weights; out [T, N] fp32 (row stride ldo elements). The integer sums are
 * exact; the bracket is rounded once to fp32 and multiplied by the two scales. K a multiple of 128
 * and at most 2^18 (else SIGNROT_ERR_UNSUPPORTED); q and wq8 16-byte aligned with row strides
 * multiples of 16 bytes (else SIGNROT_ERR_ALIGNMENT). All pointers are device pointers.
 */
signrot_status signrot_w4a4_matmul(const uint8_t* q, int64_t T, int32_t K, int64_t ldq, const float* scale,
                                   const float* zero, const int8_t* wq8, int32_t N, int64_t ldw,
                                   const float* wscale, const int32_t* colsum, float* out, int64_t ldo,
                                   void* stream);

/* Host: writes H_28 (Paley, GF(27), the orientation described above) row-major into out[784]. */
signrot_status signrot_get_h28(int8_t* out);

/* Host: writes H_344 (Paley, GF(343), the orientation described above) row-major into
 * out[344 * 344]. */
signrot_status signrot_get_h344(int8_t* out);

/* 1 if n is a supported row length, else 0. */
int32_t signrot_supported_n(int32_t n);

/* Static English text for a status code. */
const char* signrot_status_string(signrot_status status);

/* Details of the last failure on the calling host thread ("" if none). */
const char* signrot_last_error(void);

/* Number of kernels this library has launched in this process (all threads, all devices). */
uint64_t signrot_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* SIGNROT_H */
