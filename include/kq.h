/*
 * kq.h -- C ABI of the B200 (sm_100a) KroQuant online activation quantizer.
 *
 * What it computes (KroQuant review on pith.science, "What carries the
 * argument" and section 3.2 Eq. 4 / Eq. 6; abstract): every 32-channel block j
 * of a bf16 activation row x is multiplied on the right by a learned
 * invertible 32x32 block
 *
 *     K^(j) = G1 (x) G2 (x) G3 (x) G4 (x) G5,
 *     G_k   = [[1, 0], [a_k, 1]] . [[b_k, c_k], [0, 1/b_k]]   (det G_k = 1),
 *
 * (y = x T with T = diag(K^(1), ..., K^(d/32)); Eq. 1 of the paper folds T^-1
 * into the weights offline), and the transformed block is quantized to MXFP4:
 * one E8M0 scale byte per 32 elements and one E2M1 code per element, two codes
 * per byte.  G1 acts on the most significant bit of the 5-bit in-block index.
 *
 * Quantization rule (OCP Microscaling MXFP4, which the paper's "MXFP4e2"
 * names):  e = clamp(floor(log2(max_c |y_c|)) - 2, -127, 127)  (e = -127 for
 * an all-zero block), scale byte = e + 127, code = nearest E2M1 value of
 * y_c / 2^e in {0, .5, 1, 1.5, 2, 3, 4, 6} with ties to the even code,
 * saturating at 6, sign bit 0x8 set for negative values (also when they round
 * to zero).  Element 2i goes to the low nibble of byte i, element 2i+1 to the
 * high nibble.  The transform runs in float32; the decision is taken on the
 * float32 value.
 *
 * Conventions for every entry point:
 *   - All data pointers are DEVICE pointers that the caller allocates and
 *     owns; nothing is allocated, freed or retained by the library.
 *   - Arrays are dense and row-major: x and y are [M][d], q_packed is
 *     [M][d/2] bytes, scales is [M][d/32] bytes, params is [d/32][5][3]
 *     float32 holding (a, b, c) for factors k = 1..5, inv_s is [d] float32.
 *   - d must be a positive multiple of 32.  M == 0 is a no-op returning
 *     KQ_OK; M < 0 is KQ_ERR_INVALID.  M * d must not exceed 2^40.
 *   - x, q_packed, y (float32 in or out) must be 16-byte aligned; params and
 *     inv_s 4-byte aligned; scales has no alignment requirement.
 *   - stream is a cudaStream_t (NULL = the legacy default stream).  Calls are
 *     asynchronous: they enqueue kernels and return without synchronising.
 *   - Results for non-finite inputs or parameters (b_k == 0, NaN, Inf), for a
 *     transform that overflows float32, or for |x| >= 2^100 (intermediate
 *     butterfly values may overflow) are unspecified.
 *   - Return value: KQ_OK, KQ_ERR_INVALID (argument check failed, nothing
 *     enqueued), KQ_ERR_CUDA (a CUDA call or launch failed; see
 *     kq_last_cuda_error) or KQ_ERR_DEVICE (current device is not sm_100).
 */
#ifndef KQ_H_
#define KQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
    KQ_OK = 0,
    KQ_ERR_INVALID = 1,
    KQ_ERR_CUDA = 2,
    KQ_ERR_DEVICE = 3,
    KQ_ERR_TIMEOUT = 4
};

/* Implementation selector for kq_quantize_ex (for measurements). */
enum {
    KQ_IMPL_AUTO = 0,       /* what kq_quantize uses */
    KQ_IMPL_TMA = 1,        /* TMA-staged, persistent, thread per 32-block */
    KQ_IMPL_DIRECT = 2,     /* direct 32-byte global loads, thread per 32-block */
    KQ_IMPL_WARP = 3,       /* one 32-block per warp, lane = element, shuffle butterfly */
    KQ_IMPL_PANEL = 4,      /* TMA-staged column panels, factors in registers */
    KQ_IMPL_MMA = 5         /* tensor cores: dense K^(j) as three bf16 terms, tcgen05.mma */
};

/* KroQuant quantizer, the hot path: q_packed/scales = MXFP4(x T).
 * KroQuant review, "What carries the argument"; section 3.2 Eq. 4 and 6. */
int kq_quantize(const uint16_t* x, int64_t M, int64_t d, const float* params,
                uint8_t* q_packed, uint8_t* scales, void* stream);

/* Same computation with an explicit implementation choice (KQ_IMPL_*).
 * KQ_ERR_INVALID if the implementation cannot take this shape. */
int kq_quantize_ex(const uint16_t* x, int64_t M, int64_t d, const float* params,
                   uint8_t* q_packed, uint8_t* scales, int impl, void* stream);

/* Comparator: fixed orthonormal block Hadamard H_32/sqrt(32) (Sylvester
 * order) in place of K^(j), then the same MXFP4 quantizer.  KroQuant review,
 * "Core claim" (the Hadamard initialisation) and abstract. */
int kq_quantize_hadamard(const uint16_t* x, int64_t M, int64_t d,
                         uint8_t* q_packed, uint8_t* scales, void* stream);

/* Comparator: per-channel scaling y[c] = x[c] * inv_s[c] (SmoothQuant's
 * X diag(s)^-1 with the caller's float32 reciprocal scale), then the same
 * MXFP4 quantizer.  Handbook page "Quantization: where diffusion differs from
 * an LLM", section "SmoothQuant"; KroQuant abstract. */
int kq_quantize_smooth(const uint16_t* x, int64_t M, int64_t d, const float* inv_s,
                       uint8_t* q_packed, uint8_t* scales, void* stream);

/* y = x T in float32: the Kronecker block transform of kq_quantize (KroQuant
 * review, "What carries the argument": K^(j) = G1 (x) ... (x) G5 per 32-channel
 * block; "Circularity Check", Eq. 1: the activations are multiplied on the
 * right, A T), stopped before the quantizer, for parity checks, round trips
 * and the calibration.  Computed in double (every factor entry and every
 * stage) and rounded once to float32, so each value is within 2^-24 of
 * itself but where its terms cancel by about ten decimal orders.  Same
 * arguments and layout as kq_quantize; y: [M][d] float32, 16-byte aligned,
 * written by the call.  KQ_ERR_INVALID for the same argument errors.  The
 * transform, inverse and fold calls below are computed the same way. */
int kq_transform(const uint16_t* x, int64_t M, int64_t d, const float* params,
                 float* y, void* stream);

/* 16-element variant (KroQuant review, "Where Pith is reading between the
 * lines": other block formats by changing the number of Kronecker factors):
 * every 16-channel block j of x is multiplied on the right by
 * K16^(j) = G1 (x) G2 (x) G3 (x) G4 (G1 on bit 3 of the 4-bit in-block
 * index, each G_k of the same unit-determinant LU form as above), and each
 * transformed 16-block gets its own E8M0 scale (the same floor rule, amax over
 * 16 elements) and 16 E2M1 codes.
 *   params16: [d/16][4][3] float32, (a, b, c) per factor, 4-byte aligned.
 *   q_packed: [M][d/2] bytes as for kq_quantize (element 2i low nibble).
 *   scales16: [M][d/16] bytes, 2-byte aligned.
 * d must be a positive multiple of 32 and at most 32 * 65535; M at most
 * 2^31 - 1024.  Other conventions as above. */
int kq_quantize16(const uint16_t* x, int64_t M, int64_t d, const float* params16,
                  uint8_t* q_packed, uint8_t* scales16, void* stream);

/* The block-16 weight side and W4A4 product (Eq. 1 with 16-element
 * blocks): kq_quantize_weight16 writes MXFP4 of W T16^-T with a scale per 16
 * (codes [N][d/2], scales16 [N][d/16], 2-byte aligned), kq_fold_weight16
 * writes W T16^-T in float32.  The _tiled variants (and kq_quantize16_tiled)
 * write the scales in the tiled layout of kq_gemm_mxfp4_tiled with d/16
 * scales a row (kq_scales16_tiled_bytes(rows, d) bytes, 16-byte aligned).
 * kq_gemm_mxfp4_16_tiled is C = A B^T for such operands on the tensor cores
 * (tcgen05.mma kind::mxf4nvf4, block16 scaling with E8M0 scales). */
int kq_quantize_weight16(const uint16_t* w, int64_t N, int64_t d, const float* params16,
                         uint8_t* q_packed, uint8_t* scales16, void* stream);
int kq_fold_weight16(const uint16_t* w, int64_t N, int64_t d, const float* params16,
                     float* w_folded, void* stream);
int kq_quantize16_tiled(const uint16_t* x, int64_t M, int64_t d, const float* params16,
                        uint8_t* q_packed, uint8_t* scales16_tiled, void* stream);
int kq_quantize_weight16_tiled(const uint16_t* w, int64_t N, int64_t d, const float* params16,
                               uint8_t* q_packed, uint8_t* scales16_tiled, void* stream);
size_t kq_scales16_tiled_bytes(int64_t rows, int64_t K);
int kq_gemm_mxfp4_16_tiled(const uint8_t* qa, const uint8_t* sa16_tiled, const uint8_t* qb,
                           const uint8_t* sb16_tiled, int64_t M, int64_t N, int64_t K, void* c,
                           int c_dtype, void* stream);

/* y = x T16 in float32 (the kq_quantize16 transform without quantization). */
int kq_transform16(const uint16_t* x, int64_t M, int64_t d, const float* params16,
                   float* y, void* stream);

/* LayerNorm + AdaLN modulation fused in front of the quantizer: the
 * normalization that forces the transform to run online (review, "Core
 * claim" and the axiom ledger; handbook page "Quantization: where diffusion
 * differs from an LLM", AdaLN's per-timestep scales and shifts):
 *   h[m][c] = (x[m][c] - mean_m) / sqrt(var_m + eps) * (1 + scale[b][c])
 *             + shift[b][c],   b = m / tokens_per_sample,
 * mean and biased variance over the row's d channels (LayerNorm without an
 * affine part), then q_packed/scales = MXFP4(h T) exactly as kq_quantize
 * (kq_transform_adaln writes h T in float32 instead).
 *   shift, scale: bf16 [B][d], B = ceil(M / tokens_per_sample), 16-byte
 *   aligned; tokens_per_sample >= 1; 0 <= eps (finite).
 * d must be a positive multiple of 32 and at most 12288 (384 blocks).  The
 * statistics are float32 (two-pass per block, combined pairwise across the
 * row in a fixed order); h, the transform and the decision are float32.
 * With eps = 0 a row whose d values are all equal has no normalized value
 * (0 / 0): its codes and scale bytes are unspecified, nothing else is
 * affected and no error is raised; any eps > 0 maps such a row to shift. */
int kq_quantize_adaln(const uint16_t* x, int64_t M, int64_t d, const uint16_t* shift,
                      const uint16_t* scale, int64_t tokens_per_sample, float eps,
                      const float* params, uint8_t* q_packed, uint8_t* scales, void* stream);
/* kq_quantize_adaln with the scales in the tiled layout of
 * kq_gemm_mxfp4_tiled (scales_tiled: kq_scales_tiled_bytes(M, d) bytes; the
 * padding of each row's last 4-scale column is written as 0). */
int kq_quantize_adaln_tiled(const uint16_t* x, int64_t M, int64_t d, const uint16_t* shift,
                            const uint16_t* scale, int64_t tokens_per_sample, float eps,
                            const float* params, uint8_t* q_packed, uint8_t* scales_tiled,
                            void* stream);
int kq_transform_adaln(const uint16_t* x, int64_t M, int64_t d, const uint16_t* shift,
                       const uint16_t* scale, int64_t tokens_per_sample, float eps,
                       const float* params, float* y, void* stream);

/* Weight side of the transformed layer (review, "Circularity Check", Eq. 1:
 * A T (W T^-T)^T = A W^T, the inverse folded into the weights offline).
 * w is the bf16 weight matrix [N][d] of a linear layer y = x W^T (row n holds
 * output channel n, d = input channels, the same d and params as the
 * activations it meets).  kq_quantize_weight writes MXFP4(W T^-T): each
 * 32-column block of a row is multiplied on the right by
 * (K^(j))^-T = (G1^-1)^T (x) ... (x) (G5^-1)^T, then quantized exactly as
 * kq_quantize does (codes [N][d/2], scales [N][d/32], 16-byte aligned w and
 * q_packed).  kq_fold_weight writes W T^-T in float32 [N][d] (16-byte
 * aligned).  d at most 32 * 65535; N at most 2^31 - 1024. */
int kq_quantize_weight(const uint16_t* w, int64_t N, int64_t d, const float* params,
                       uint8_t* q_packed, uint8_t* scales, void* stream);
int kq_fold_weight(const uint16_t* w, int64_t N, int64_t d, const float* params,
                   float* w_folded, void* stream);

/* Output types of kq_gemm_mxfp4. */
enum {
    KQ_OUT_F32 = 0,
    KQ_OUT_BF16 = 1
};

/* W4A4 product of the transformed layer (review, "Circularity Check",
 * Eq. 1): C = A B^T for A = kq_quantize(x) and B = kq_quantize_weight(W),
 * so that C approximates x W^T.  On the tensor cores (block-scaled
 * tcgen05.mma, kind::mxf4), accumulating in float32.
 *   qa: [M][K/2] packed E2M1 codes, sa: [M][K/32] E8M0 scale bytes;
 *   qb: [N][K/2] codes, sb: [N][K/32] scales (same layout as kq_quantize);
 *   c:  [M][N] row-major, float32 (c_dtype KQ_OUT_F32) or bf16
 *       (KQ_OUT_BF16, rounded to nearest even once from the float32 sum).
 * K must be a positive multiple of 32; M and N any size up to about 2^31
 * (each below 2^31 - 256).  qa, qb and c 16-byte aligned.  Each output is
 * the float32 accumulation of the exact products A[m][k] B[n][k]; scale byte
 * 0xFF (NaN) gives NaN. */
int kq_gemm_mxfp4(const uint8_t* qa, const uint8_t* sa, const uint8_t* qb, const uint8_t* sb,
                  int64_t M, int64_t N, int64_t K, void* c, int c_dtype, void* stream);

/* Calibration of the transform on one linear layer (review, "What carries
 * the argument" and the free-parameter ledger: per-layer minimization of the
 * quantized output error plus per-operand regularization, Adam with a
 * straight-through estimator through the quantizer).
 *
 * kq_transform_params_grad: for Z = X K(theta) per 32-block (K = T, or
 * K = T^-T with inverse_transpose != 0, the weight side), the gradient of
 * L with respect to the [d/32][5][3] parameters given
 *   dL/dZ = g + 2 lambda (Z - Zq)   (g = dL_out/dZq, straight-through),
 * written to dparams (float32 [d/32][5][3], overwritten), and
 * reg = sum (Zq - Z)^2 (one float).  z, zq, g: float32 [M][d], 16-byte
 * aligned; z must be the transform of the layer's operand at `params`
 * (the stage inputs are recovered from it).  workspace: device memory of at
 * least kq_transform_params_grad_workspace_bytes(M, d) bytes, 256-byte
 * aligned, zero before its first use (each call leaves it reusable); calls
 * sharing a workspace must be ordered.  The result is deterministic. */
size_t kq_transform_params_grad_workspace_bytes(int64_t M, int64_t d);
int kq_transform_params_grad(const float* z, const float* zq, const float* g, int64_t M,
                             int64_t d, const float* params, int inverse_transpose,
                             float lambda, float* dparams, float* reg, void* workspace,
                             size_t workspace_bytes, void* stream);

/* out[i] = scale (y[i] - y_ref[i]) and *sumsq = sum (y - y_ref)^2 (double,
 * deterministic); out may alias y.  workspace as above, of
 * kq_residual_workspace_bytes() bytes, zero before first use. */
size_t kq_residual_workspace_bytes(void);
int kq_residual(const float* y, const float* y_ref, int64_t n, float scale, float* out,
                double* sumsq, void* workspace, size_t workspace_bytes, void* stream);

/* One Adam step (bias-corrected; step counts from 1) on n float32
 * parameters with gradient grad0 + grad1 (grad1 may be NULL); m and v are
 * the float32 moment buffers, updated in place.  The hyperparameters are
 * double so that 1 - beta is formed exactly before the float32 update. */
int kq_adam_step(float* params, const float* grad0, const float* grad1, float* m, float* v,
                 int64_t n, int step, double lr, double beta1, double beta2, double eps,
                 void* stream);

/* The same product with both scale arrays in the tiled layout the tensor
 * cores read: 128-row x 4-scale tiles of 512 bytes, row-tile major then
 * along K; inside a tile row r = r0 + 32 r1 (r0 < 32, r1 < 4) and scale i
 * (< 4) sit at byte 16 r0 + 4 r1 + i; rows are padded to a multiple of 128
 * and the K/32 scales of a row to a multiple of 4 (zero bytes).  sa_tiled:
 * kq_scales_tiled_bytes(M, K) bytes, sb_tiled: kq_scales_tiled_bytes(N, K),
 * both 16-byte aligned.  The scale tiles reach the GEMM as whole bulk
 * copies, which is faster than gathering row-major scale bytes. */
int kq_gemm_mxfp4_tiled(const uint8_t* qa, const uint8_t* sa_tiled, const uint8_t* qb,
                        const uint8_t* sb_tiled, int64_t M, int64_t N, int64_t K, void* c,
                        int c_dtype, void* stream);

/* Bytes of the tiled scale layout for `rows` rows of K/32 scales (0 for an
 * invalid K or rows < 1). */
size_t kq_scales_tiled_bytes(int64_t rows, int64_t K);

/* kq_quantize and kq_quantize_weight with the scale bytes written straight
 * into the tiled layout above (scales_tiled: kq_scales_tiled_bytes(M, d)
 * bytes).  Every real entry and the padding of each row's last 4-scale
 * column are written; the padding rows of the last 128-row tile are not
 * (they only meet zero-filled code rows in the product).  Codes as for the
 * row-major entry points. */
int kq_quantize_tiled(const uint16_t* x, int64_t M, int64_t d, const float* params,
                      uint8_t* q_packed, uint8_t* scales_tiled, void* stream);
int kq_quantize_weight_tiled(const uint16_t* w, int64_t N, int64_t d, const float* params,
                             uint8_t* q_packed, uint8_t* scales_tiled, void* stream);

/* Row-major scales [rows][K/32] -> the tiled layout above (tiled: 16-byte
 * aligned, kq_scales_tiled_bytes(rows, K) bytes, padding written as 0). */
int kq_scales_to_tiled(const uint8_t* scales, int64_t rows, int64_t K, uint8_t* tiled,
                       void* stream);

/* x = y T^-1 in float32 with T^-1 = diag(G1^-1 (x) ... (x) G5^-1) (review,
 * axiom ledger: the inverse of a Kronecker product factorizes), computed in
 * double and rounded once as kq_transform is.  y: [M][d] float32, x: [M][d]
 * float32, both 16-byte aligned; params as for kq_quantize. */
int kq_inverse_transform(const float* y, int64_t M, int64_t d, const float* params,
                         float* x, void* stream);

/* y = E2M1(code) * 2^(scale - 127) in float32: the value MXFP4 codes and
 * their shared E8M0 scale stand for (the OCP Microscaling definition the
 * review cites for MXFP4: E2M1 elements with magnitudes {0, 0.5, 1, 1.5, 2,
 * 3, 4, 6}, an E8M0 power-of-two scale per 32 elements).  Exact; scale byte
 * 0xFF gives NaN, results beyond the float32 range give +-Inf.  q_packed
 * [M][d/2] and scales [M][d/32] as kq_quantize writes them; y [M][d] float32,
 * 16-byte aligned. */
int kq_dequantize(const uint8_t* q_packed, const uint8_t* scales, int64_t M, int64_t d,
                  float* y, void* stream);

/* End-to-end quantization of activations in HOST memory: the same result as
 * kq_quantize, with x_host [M][d] bf16 read from host memory and q_host
 * [M][d/2] and scales_host [M][d/32] written to host memory.  Rows move in
 * chunks through `workspace` (device memory the caller allocates, 256-byte
 * aligned; two chunks live in it at a time), so that the host-to-device copy
 * of one chunk, the quantizer on the previous one and the device-to-host copy
 * of the one before overlap.  The host buffers should be page-locked (pinned)
 * for the copies to overlap.  params is a device pointer.  The call is
 * asynchronous: it returns once the work is queued, and `stream` completes
 * when the last outputs have reached host memory; the host buffers must stay
 * valid until then.  The library keeps two copy streams and a few events per
 * device, created on the first call; calls for the same device are queued
 * one at a time.  KQ_ERR_INVALID if the workspace cannot hold two chunks of
 * one row (kq_quantize_host_workspace_bytes(d, 1)). */
int kq_quantize_host(const uint16_t* x_host, int64_t M, int64_t d, const float* params,
                     uint8_t* q_host, uint8_t* scales_host, void* workspace,
                     size_t workspace_bytes, void* stream);

/* Workspace bytes kq_quantize_host needs for chunks of rows_per_chunk rows
 * of width d (0 for an invalid d or rows_per_chunk < 1). */
size_t kq_quantize_host_workspace_bytes(int64_t d, int64_t rows_per_chunk);

/* Size of the staging area built into the library for
 * kq_quantize_host_static: 16 MiB of device memory. */
#define KQ_STATIC_STAGING_BYTES (16u << 20)

/* The same result as kq_quantize_host, for callers that cannot allocate
 * device memory: a serving process whose memory pool already holds nearly
 * all of the GPU can see cudaMalloc fail, and cudaMalloc / cudaFree may
 * synchronise the whole device.  This call takes no workspace and allocates
 * nothing (no cudaMalloc, no streams, no events): rows are copied in,
 * quantized and copied out chunk by chunk, in order on `stream` alone,
 * through a KQ_STATIC_STAGING_BYTES staging area that is part of the library
 * itself.  Each GPU on which that area is loaded keeps it until the process
 * exits.  The first call on a device looks up the area's device address
 * (cudaGetSymbolAddress) and keeps it for later calls; make that first call
 * before any stream capture.  The kept address belongs to the device's
 * primary context: it is valid only while that context lives, so a process
 * that resets the device (cudaDeviceReset) must not call this entry point
 * again.  The call uses the current device; `stream` must belong to it.
 * The call is asynchronous, like kq_quantize_host: it returns once the work
 * is queued, and `stream` completes when the last outputs have reached host
 * memory; the host buffers must stay valid until then.
 * All calls share the one area and the last call's data stays in it: calls
 * that overlap on the GPU (on different streams, or from several host
 * threads) race and must be serialised by the caller.  KQ_ERR_INVALID for
 * rows too wide for the area: 2 d + d/2 + d/32 bytes plus rounding must fit
 * in KQ_STATIC_STAGING_BYTES (d up to about 6.6 million).  The pages have no
 * counterpart of this entry point. */
int kq_quantize_host_static(const uint16_t* x_host, int64_t M, int64_t d, const float* params,
                            uint8_t* q_host, uint8_t* scales_host, void* stream);

/* Human-readable name of a status code (static string, never NULL). */
const char* kq_status_string(int status);

/* The cudaError_t of the last KQ_ERR_CUDA on this thread (0 if none). */
int kq_last_cuda_error(void);

/* Synchronises the current device, then reads and clears the library's
 * device-side error word: 0 if every bounded in-kernel wait finished,
 * otherwise a bit mask of the waits that gave up (kernels that give up stop
 * early and leave their outputs incomplete).  Returns KQ_OK or KQ_ERR_CUDA. */
int kq_device_status(int* flags);

/* Device-side error word bits (kq_device_status). */
#define KQ_DEVERR_CONSUMER_WAIT 1  /* a consumer gave up waiting for its data */
#define KQ_DEVERR_PRODUCER_WAIT 2  /* a producer gave up waiting for a free stage */
#define KQ_DEVERR_SELFTEST 4       /* set by kq_selftest_wait_timeout */

/* Self-test of the bounded waits: launches one tiny kernel that waits (at
 * most 64 polls of about 1 us) on a barrier nothing completes, gives up and
 * sets KQ_DEVERR_SELFTEST in the device error word, which kq_device_status
 * then reports and clears.  The device stays usable afterwards. */
int kq_selftest_wait_timeout(void* stream);

/* ABI version, (major << 16) | minor. */
int kq_version(void);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* KQ_H_ */
