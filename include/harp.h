/*
 * harp.h -- C ABI of the B200 (sm_100a) rotated low-bit linear library.
 *
 * The method: "HARP: Hadamard-Preconditioned Adaptive Rotation Processor for
 * Extreme LLM Quantization" (gist.science explanation of arXiv 2605.29843).
 * A linear layer W (n_out x n_in) is stored as a low-bit quantization of the
 * rotated matrix W' = U W V^T, where V and U^T are butterfly transforms:
 *   F(theta, s, w) = S_{m-1} ... S_1 S_0 D,  m = log2(w),
 *   D = diag(s), s_i in {+1,-1}; stage S_t pairs (i, i + 2^t) inside every w-wide
 *   block with the 2x2 block Givens(theta) * H_2 = [[cos p, sin p], [sin p, -cos p]],
 *   p = pi/4 + theta (Sec. 2.1 "Arquitetura Central": stride stages of block-diagonal
 *   orthogonal B_t; Sec. 2.2: B = Q(theta) G_2, Theta = 0 gives the randomized
 *   Hadamard transform). Pairs of stage t are numbered in increasing order of their
 *   first index; theta is stored stage-major, [m][n/2] fp32.
 *   n that is not a power of two uses w-wide blocks (block-diagonal butterfly).
 * Online the layer computes y = U^T dequant(codes) V x = F_U(dequant(codes) F_V(x))
 * with V = F(theta_V, s_V, w_in) and U^T = F(theta_U, s_U, w_out).
 *
 * Quantizer (a stand-in: the pages leave the codebook to the backend, Sec. 2.4):
 * per output row and group of `group` = 64 consecutive columns of W',
 * zero16 = fp16(min), scale16 = fp16((max-min)/(2^b-1)) (1 when that is 0),
 * q = clamp(round_half_even((w - zero16)/scale16), 0, 2^b-1), dequant = scale16*q + zero16.
 *
 * Canonical layouts (device memory, row-major by output row, e = r*n_in + j):
 *   codes, b = 2 or 4: code e in little-endian 32-bit word (e*b)/32, bits [(e*b)%32, +b);
 *   codes, b = 3: a 2-bit plane of (q & 3) laid out as for b = 2 (n_out*n_in/4 bytes)
 *                 followed by a 1-bit plane of (q >> 2): word e/32, bit e%32;
 *   scale_zero: [n_out][n_in/group] half2, .x = scale16, .y = zero16.
 *
 * Conventions for every entry point:
 *   - Pointers named "device" must be device memory of the current device; every
 *     device pointer must be 16-byte aligned. `stream` is a cudaStream_t (0 = the
 *     legacy default stream). All work is enqueued on `stream` and returns at once.
 *   - Arguments are validated before anything is launched; on failure nothing is
 *     launched, the call returns a non-zero status and harp_last_error() (a
 *     thread-local string) says why. No C++ exception crosses this boundary.
 *   - Device-side failures (a bounded wait that ran out, a failed bounds check) set
 *     a per-device status word; harp_device_status() reads and clears it.
 *   - Calls on different layer handles may run from different host threads.
 */
#ifndef HARP_H
#define HARP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HARP_OK = 0,
  HARP_ERR_INVALID_ARG = 1, /* bad size, alignment, null pointer, unsupported width */
  HARP_ERR_UNSUPPORTED = 2, /* a valid request the library does not implement */
  HARP_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
  HARP_ERR_WORKSPACE = 4,   /* workspace missing or smaller than the query returned */
  HARP_ERR_TIMEOUT = 5,     /* a bounded device-side wait ran out (device status) */
  HARP_ERR_DEVICE_CHECK = 6 /* a device-side bounds/consistency check failed */
} harp_status;

typedef enum { HARP_F32 = 0, HARP_BF16 = 1, HARP_F16 = 2 } harp_dtype;

typedef struct harp_layer_s* harp_layer;
typedef struct harp_stack_s* harp_stack;

/* Thread-local description of the last failure on this host thread ("" if none). */
const char* harp_last_error(void);

/* Reads and clears the device status word of the current device (HARP_OK if clean).
 * Synchronises `stream` first. */
harp_status harp_device_status(void* stream);

/* Testing hook for the failure paths; everything is off by default and the paper has no
 * counterpart. It applies process-wide to launches made after it:
 *   wait_limit_us   : > 0 bounds the device-side waits of harp_linear_fwd's dequant-GEMV and of
 *                     the fused decode step by that many microseconds (0 restores the default,
 *                     about 1-2 s);
 *   gemv_skip_stage : >= 0 makes the first CTA of the dequant-GEMV skip issuing that stage of
 *                     its weight ring, so its consumers' wait runs out (-1: off);
 *   decode_barrier  : >= 0 raises the arrival target of that grid barrier of the fused decode
 *                     step (index 5 * block + phase) by one, so no CTA passes it (-1: off).
 * A wait that runs out records HARP_ERR_TIMEOUT and its site in the device status word and
 * ends the kernel after waiting (bounded) for its copies in flight; no GPU fault is raised.
 * Returns HARP_ERR_INVALID_ARG for negative values other than -1. */
harp_status harp_test_set_faults(int wait_limit_us, int gemv_skip_stage, int decode_barrier);

/* ---------------------------------------------------------------- butterfly
 * y = F(theta, s, w) x for `batch` rows of n (row-major, contiguous).
 * Sec. 2.1-2.2 of the HARP page: signs, then stages of stride 1, 2, ..., w/2.
 *   n      : vector length, n % w == 0, n <= 2^30.
 *   w      : block width, a power of two, 2 <= w <= 8192.
 *   theta  : device fp32 [log2 w][n/2] angle offsets (the pi/4 is added inside), or
 *            NULL for Theta == 0: the fixed randomized Hadamard transform H_w D / sqrt(w)
 *            per block (every 2x2 block [[1, 1], [1, -1]] / sqrt 2; no angles are read).
 *   sign   : device int8 [n], each +1 or -1.
 *   x, y   : device, dtypes xt / yt (f32, bf16, f16); y may equal x when xt == yt.
 * Arithmetic is fp32; sin/cos are evaluated in fp32 from pi/4 + theta.
 */
harp_status harp_butterfly_fwd(int64_t n, int w, int batch, const float* theta, const int8_t* sign,
                               const void* x, harp_dtype xt, void* y, harp_dtype yt, void* stream);

/* y = F(theta, s, w)^T x: the same stages in reverse order, then the signs
 * (every 2x2 block is symmetric). Same arguments as harp_butterfly_fwd. */
harp_status harp_butterfly_inv(int64_t n, int w, int batch, const float* theta, const int8_t* sign,
                               const void* x, harp_dtype xt, void* y, harp_dtype yt, void* stream);

/* ---------------------------------------------------------------- quantize
 * Quantizes an already rotated matrix W' (device fp32 [n_out][n_in], row-major) into
 * the canonical codes and scale_zero buffers (device, caller-owned, sizes
 * n_out*n_in*bits/8 and n_out*(n_in/group)*4 bytes). bits in {2,3,4}, group == 64,
 * n_in % 64 == 0. The arithmetic of the rule above is done in fp64 on the device, so
 * the codes equal those of an fp64 evaluation of the same fp32 input.
 */
harp_status harp_quantize_weights(int64_t n_out, int64_t n_in, int bits, int group,
                                  const float* W_rot, void* codes, void* scale_zero, void* stream);

/* ---------------------------------------------------------------- mixed-radix schedules
 * HARP page, Sec. 2.1 (Suporte a Misto-Raiz) and 2.2: for d = b_0 b_1 ... b_{m-1} the
 * rotation is signs, then stages t = 0..m-1, stage t mixing the b_t coordinates that differ
 * only in mixed-radix digit t (stride b_0 ... b_{t-1}; group c starts at
 * (c mod s_t) + (c div s_t) s_t b_t) with B_{t,c} = Q_{t,c}(theta) G_{b_t}:
 *   b = 2: the Givens block of the radix-2 butterfly (one angle offset, pi/4 added inside);
 *   b > 2: Q = (I - A)(I + A)^-1 (Cayley) of the skew-symmetric A whose strict upper
 *          triangle holds the group's b(b-1)/2 parameters row by row; G_b = H_b / sqrt(b)
 *          (Sylvester) for powers of two, else the orthogonal factor of the QR
 *          factorisation of the stage's fixed Gaussian matrix, R's diagonal positive.
 * With every b_t = 2 this is harp_butterfly_fwd with w = d.
 * A plan computes every block once (fp64, stored fp32) and owns them.
 *   d      : 2..16384, the product of the radices.    m: 1..32 stages.
 *   radix  : HOST int [m], each in [2, 64].
 *   theta  : device fp32, stage after stage, group after group, the group's parameters.
 *   sign   : device int8 [d] (copied).
 *   gauss  : device fp32, one b_t x b_t row-major matrix per stage, stage after stage
 *            (entries of power-of-two stages are not read); NULL when every radix is a
 *            power of two. The pages give no seed for it: it is the caller's input.
 * Synchronises `stream` (the set-up is checked before returning). Errors:
 * HARP_ERR_INVALID_ARG (sizes, radices, pointers, a singular Gaussian), HARP_ERR_CUDA. */
typedef struct harp_mr_plan_s* harp_mr_plan;
harp_status harp_mr_plan_create(harp_mr_plan* out, int64_t d, int m, const int* radix, const float* theta,
                                const int8_t* sign, const float* gauss, void* stream);
harp_status harp_mr_plan_destroy(harp_mr_plan plan);

/* y = F x (fwd) or F^T x (inv: the stage transposes from t = m-1 down to 0, then the signs)
 * for `batch` rows of d, row-major; dtypes f32/bf16/f16; y may equal x when xt == yt;
 * pointers 16-byte aligned. Arithmetic is fp32. */
harp_status harp_mr_butterfly_fwd(harp_mr_plan plan, int batch, const void* x, harp_dtype xt, void* y,
                                  harp_dtype yt, void* stream);
harp_status harp_mr_butterfly_inv(harp_mr_plan plan, int batch, const void* x, harp_dtype xt, void* y,
                                  harp_dtype yt, void* stream);

/* A layer whose two sides are mixed-radix butterflies (HARP page, Sec. 2.1, Suporte a
 * Misto-Raiz): y = F_U(dequant(codes) F_V(x)) with F_V the plan V's forward transform and
 * F_U the plan U's. For a width such as 11008 = 2^8 * 43 this mixes all coordinates, where a
 * radix-2 layer uses independent 256-wide blocks. codes/scale_zero must come from
 * W' = F_U^T W F_V^T rotated with the same plans (canonical layouts as for harp_create_layer).
 *   n_in  : a multiple of 256, <= 16384, equal to V's length;  n_out: <= 16384, U's length.
 *   V, U  : plans of harp_mr_plan_create on the current device. BORROWED, like codes and
 *           scale_zero: keep all four alive and unchanged until harp_destroy_layer.
 * harp_linear_fwd runs the plans' transforms (fp32) around the same dequant-GEMV (1..15
 * tokens; the transformed input is brought to the int16 group operand) or tcgen05 path (16+
 * tokens; the split partials are summed before the output transform). Stacks of such layers
 * take the per-linear path. Errors: HARP_ERR_INVALID_ARG (sizes, lengths, pointers, device),
 * HARP_ERR_UNSUPPORTED (group), HARP_ERR_CUDA. */
harp_status harp_create_layer_mr(harp_layer* out, int64_t n_in, int64_t n_out, int bits, int group,
                                 harp_mr_plan V, harp_mr_plan U, const void* codes, const void* scale_zero,
                                 void* stream);

/* ---------------------------------------------------------------- int8 angles
 * The HARP page stores its parameters in int8 (Sec. 2.4, Armazenamento, and Sec. 4:
 * 2.00 -> 2.05 bits per parameter at 2 bits); the format is this library's:
 * one symmetric step per butterfly stage,
 *   delta_t = fp32(max_p |theta_tp| / 127),
 *   q_tp    = clamp(round_half_even(theta_tp / delta_t), -127, 127)   (0 when delta_t = 0),
 * and the layer applies theta^ = delta_t * q_tp. The codes and steps are computed in fp64
 * from the fp32 angles, so they equal those of an fp64 evaluation exactly.
 *   m      : stages, 1..16.    half_n: pairs per stage (n/2).
 *   theta  : device fp32 [m][half_n], finite.
 *   q      : device int8 [m][half_n] (out).    delta: device fp32 [m] (out).
 * All pointers 16-byte aligned. */
harp_status harp_quantize_angles(int m, int64_t half_n, const float* theta, int8_t* q, float* delta,
                                 void* stream);

/* A layer whose butterflies keep their angles in int8: the same as harp_create_layer, with
 * each side's theta replaced by (q [log2 w][n/2] int8, delta [log2 w] fp32) from
 * harp_quantize_angles. The layer copies both (1 byte per angle plus a 64-byte head), and
 * its kernels evaluate cos/sin of pi/4 + delta_t q as they rotate, instead of reading
 * 8-byte (cos, sin) pairs. codes/scale_zero must come from W rotated with the dequantized
 * angles theta^ (the exact change of basis holds for theta^, not theta). q NULL makes that
 * side Theta = 0 (delta ignored). The fused decode step runs when every butterfly of a
 * stack uses int8 angles, like when all use fp32 angles or all are Theta = 0. */
harp_status harp_create_layer_q8(harp_layer* out, int64_t n_in, int64_t n_out, int bits, int group,
                                 int w_in, int w_out, const int8_t* q_V, const float* delta_V,
                                 const int8_t* sign_V, const int8_t* q_U, const float* delta_U,
                                 const int8_t* sign_U, const void* codes, const void* scale_zero,
                                 void* stream);

/* ---------------------------------------------------------------- calibration
 * The per-layer fitting loss that calibration minimises over the angles (HARP page,
 * Sec. 2.3, Objetivo de Otimizacao), and its gradient:
 *   W' = U W V^T,  T = deq(Q(W')),  H' = V H V^T,  d = diag(H')
 *   L_diag = sum_{r,j} d_j (W'_rj - T_rj)^2
 *   R_bd   = sum of H'_ij^2 over i, j in different 64-column quantizer groups
 *   L_fit  = L_diag + lambda_bd * R_bd
 * Here V = F(theta_V, sign_V, w_in) and U = F(theta_U, sign_U, w_out)^T. Q and deq are the
 * quantizer above: the codes and their fp16 scale and zero, exactly as the linear stores
 * them. The gradient holds T constant (no gradient through the code assignment).
 *   n_out, n_in : n_in % 256 == 0, n_out % 32 == 0, each < 65536 (each side is the other
 *                 side's butterfly batch).
 *   bits, group : {2, 3, 4}, 64.    w_in, w_out: butterfly widths dividing n_in, n_out.
 *   W           : device fp32 [n_out][n_in], row-major, not modified.
 *   theta_V/U   : device fp32 [log2 w][n/2] angle offsets, or NULL for Theta = 0.
 *   sign_V/U    : device int8 [n].
 *   H           : device fp32 [n_in][n_in] symmetric Hessian proxy of the layer's inputs
 *                 (e.g. X^T X / N), or NULL for the identity (then d = 1 and R_bd = 0).
 *   lambda_bd   : >= 0.
 *   loss        : device fp64 [3] = {L_fit, L_diag, R_bd}, written on `stream`.
 *   grad_theta_V/U : device fp32, shaped like theta, receive dL_fit/dtheta; NULL skips
 *                 that side (both NULL: no backward pass). A NULL theta still gets its
 *                 gradient at Theta = 0, where calibration starts.
 *   workspace   : device, 256-byte aligned, at least harp_calib_workspace_size bytes for
 *                 the same sizes, with_hessian = (H != NULL) and with_grad; overwritten.
 *                 Roughly 3 fp32 copies of W, plus 3 of H when H is given.
 * Rotations and the backward stages run in fp32. Sums of squares and the angle-gradient
 * sums are fp64 and run in a fixed order, so a call repeats its results exactly.
 * Pointers must be 16-byte aligned (loss 8).
 * Errors:
 *   HARP_ERR_INVALID_ARG for sizes, widths, a negative lambda, null or misaligned pointers;
 *   HARP_ERR_WORKSPACE;
 *   HARP_ERR_CUDA on a launch failure.
 */
harp_status harp_calib_workspace_size(int64_t n_out, int64_t n_in, int bits, int w_in, int w_out,
                                      int with_hessian, int with_grad, size_t* bytes);

harp_status harp_calib_fit(int64_t n_out, int64_t n_in, int bits, int group, int w_in, int w_out,
                           const float* W, const float* theta_V, const int8_t* sign_V,
                           const float* theta_U, const int8_t* sign_U, const float* H, double lambda_bd,
                           double* loss, float* grad_theta_V, float* grad_theta_U, void* workspace,
                           size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- layer
 * Creates a layer handle.
 *   n_in, n_out : multiples of 64, each <= 65536.
 *   bits        : 2, 3 or 4.   group: 64.
 *   w_in, w_out : butterfly block widths: powers of two, 64 <= w <= 8192, w | n.
 *   theta_V, sign_V : device [log2 w_in][n_in/2] fp32, [n_in] int8 (input side V).
 *   theta_U, sign_U : device [log2 w_out][n_out/2] fp32, [n_out] int8 (U^T side).
 *   A NULL theta_V or theta_U makes that side the fixed randomized Hadamard transform
 *   (Theta == 0, "RHT"): its kernels use the constant 1/sqrt 2 blocks and load no
 *   per-stage parameters. The codes must then come from a W' rotated with Theta == 0.
 *   codes, scale_zero : device, canonical layout above.
 * Ownership: the layer COPIES theta/sign (it stores cos/sin tables of pi/4 + theta in
 * its own device memory) and BORROWS codes and scale_zero, which the caller keeps
 * alive and unchanged until harp_destroy_layer. The copies are enqueued on `stream`.
 */
harp_status harp_create_layer(harp_layer* out, int64_t n_in, int64_t n_out, int bits, int group,
                              int w_in, int w_out, const float* theta_V, const int8_t* sign_V,
                              const float* theta_U, const int8_t* sign_U, const void* codes,
                              const void* scale_zero, void* stream);

/* Frees the layer's own device memory (synchronises the device first). Null is a no-op. */
harp_status harp_destroy_layer(harp_layer layer);

/* Bytes of device workspace harp_linear_fwd needs for `batch` rows (batch 1..65535). */
harp_status harp_linear_workspace_size(harp_layer layer, int batch, size_t* bytes);

/* y = F_U(dequant(codes) F_V(x)) for `batch` rows.
 *   x : device [batch][n_in] of dtype xt;  y : device [batch][n_out] of dtype yt.
 *   workspace : device scratch of at least harp_linear_workspace_size bytes, 256-byte
 *               aligned; its contents are overwritten. y must not alias x or workspace.
 * Batches 1..15 run the CUDA-core dequant-GEMV: the transformed activations as int16 with
 * a power-of-two scale per 64-column group, and exact integer dot products per group,
 * in passes of 8 rows.
 * Batches 16..65535 run the tcgen05 tensor-core path:
 *   - the transformed activations as fp16 with a power-of-two scale per row, and the
 *     weights as fp16 s*q;
 *   - fp32 accumulation in tensor memory;
 *   - the zero term m * (group sum) as one more K block;
 *   - in chunks of 256 rows.
 * Both paths take the same workspace call; its size depends on the path.
 */
harp_status harp_linear_fwd(harp_layer layer, int batch, const void* x, harp_dtype xt, void* y,
                            harp_dtype yt, void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- linear, no allocation
 * harp_linear_fwd for callers that cannot allocate device memory: code that runs inside
 * another framework's memory pool, real-time paths where an allocation may block or
 * fail, and hosts that hand the library only pre-registered buffers. The paper has no
 * counterpart; this is a library convenience. Its scratch is a 2 MiB array in the
 * library's device image, which every GPU that loads the library holds until exit.
 *   x, y  : as for harp_linear_fwd (caller-owned device memory); no workspace argument.
 *   Fails with HARP_ERR_WORKSPACE when the layer and batch need more than 2 MiB of
 *   scratch (harp_linear_workspace_size says how much).
 *   The first call on a device looks up the array's device address; under CUDA's lazy
 *   module loading that lookup also loads the part of the library holding the array, so
 *   the 2 MiB are taken from the device at that first call. Make that first call before
 *   any stream capture; later calls take no device memory. Batches as for
 *   harp_linear_fwd (1..65535), as far as their scratch fits. All calls on a device
 *   share the array and it keeps
 *   the last call's contents (nothing in it must start at zero): calls that overlap on
 *   the GPU (other streams, other host threads) race, so serialise them.
 *   Allocates nothing (no cudaMalloc, cudaFree or allocating library routine); for the
 *   same reason a device-side wait that runs out ends the kernel without a status report.
 */
harp_status harp_linear_fwd_static(harp_layer layer, int batch, const void* x, harp_dtype xt, void* y,
                                   harp_dtype yt, void* stream);

/* ---------------------------------------------------------------- decoder stack
 * A Llama-shaped stack of n_layers blocks, each with seven rotated linears in the
 * order q, k, v, o, gate, up, down (layers[7*l + i]). One decode step computes, per
 * block: n1 = rms(x); v = v_proj(n1) (q_proj and k_proj are evaluated too; a one-key
 * attention returns its value); a = v repeated per key/value group (head h reads kv
 * head h / (n_heads/n_kv_heads)); h = x + o_proj(a); n2 = rms(h);
 * x' = h + down(silu(gate(n2)) * up(n2)); rms(u) = u / sqrt(mean(u^2) + eps).
 * The stack borrows the layer handles (they must outlive it).
 * Shapes: q n_heads*head_dim x hidden, k/v n_kv_heads*head_dim x hidden,
 * o hidden x n_heads*head_dim, gate/up ffn x hidden, down hidden x ffn; the output-side
 * block width of gate and up must equal the input-side block width of down.
 */
harp_status harp_stack_create(harp_stack* out, int n_layers, int hidden, int ffn, int n_heads,
                              int n_kv_heads, int head_dim, float eps, const harp_layer* layers,
                              void* stream);
harp_status harp_stack_destroy(harp_stack stack);
harp_status harp_stack_workspace_size(harp_stack stack, int batch, size_t* bytes);

/* 1 when harp_stack_step with this batch runs the fused single-kernel decode step
 * (batch 1, hidden a power of two in [4096, 8192], n_heads*head_dim == hidden, single-block
 * q/k/v/o/down butterflies, gate/up output blocks 64..512, 4096 or 8192 wide, one bit width,
 * one form of the angles), else 0
 * (the step then runs one launch sequence per linear; harp_last_error() then says why). */
int harp_stack_uses_fused_step(harp_stack stack, int batch);

/* One decode step: out = stack(x). x, out: device [batch][hidden] of dtypes xt / ot
 * (batch 1..256); out may equal x. workspace as for harp_linear_fwd. */
harp_status harp_stack_step(harp_stack stack, int batch, const void* x, harp_dtype xt, void* out,
                            harp_dtype ot, void* workspace, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* HARP_H */
