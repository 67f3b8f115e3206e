/*
 * svdq.h -- C ABI of the B200 (sm_100a) SVDQuant W4A4 rank-corrected smoothed linear layer.
 *
 *   Y = Q4(X diag(lam)^-1) (x) Q4(R) + (X diag(lam)^-1 L1) L2 + b
 *
 * Sources (the pages this library restates):
 *   [MC]  SVDQuant model card, huggingface mit-han-lab/svdq-int4-flux.1-depth-dev:
 *         "Quantization Method -- SVDQuant" (stages 1-3: smoothing migrates outliers
 *         from X into W, SVD splits the smoothed W into a 16-bit low-rank branch
 *         L1 L2 and a 4-bit residual R) and "Nunchaku Engine Design" (a)(b)
 *         (Down Projection fused with Quantize on the shared input; Up Projection
 *         fused with 4-Bit Compute on the shared output).
 *   [ND]  "Nunchaku in Diffusers" blog: "Introducing Nunchaku Lite" (svdq_w4a4 kernel
 *         family, INT4 and NVFP4 variants), "Native loading in Diffusers"
 *         (quantization_config: precision nvfp4, group_size 16, rank 32,
 *         compute_dtype bfloat16), "Hardware support" (the GPU capability is checked at
 *         load time and a clear error is raised instead of wrong outputs).
 *
 * Conventions for every call
 *   - Shapes are nn.Linear shapes: X is M x K, W is N x K (output x input features),
 *     Y is M x N.  bf16 tensors are passed as uint16_t bit patterns (host) or as
 *     untyped device pointers.
 *   - "host" pointers are ordinary CPU memory; "device" pointers are global memory of
 *     the device the weights were prepared on.  The library never frees caller memory.
 *   - Every call returns an svdq_status.  Nothing aborts, traps or throws across the
 *     ABI; svdq_last_error() gives a human-readable message for the calling thread.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *     Device calls are asynchronous on that stream and never synchronise it, except
 *     where stated.
 *   - Precisions: SVDQ_NVFP4 = E2M1 values with one UE4M3 scale per 16 elements along
 *     K; SVDQ_INT4 = signed 4-bit integers with one fp32 scale per 64 elements along K.
 *   - Shape limits: K % 256 == 0, N % 8 == 0, 0 <= rank <= 128 with rank % 16 == 0,
 *     rank <= min(N, K); M >= 0 (any M; row tails are masked); ldx, ldy multiples of 8
 *     elements; X, Y and workspace 16-byte aligned.
 */
#ifndef SVDQ_H_
#define SVDQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SVDQ_ABI_VERSION 1

typedef enum {
  SVDQ_OK = 0,
  SVDQ_ERR_INVALID_ARG = 1,        /* null pointer, bad shape, misalignment, workspace too small */
  SVDQ_ERR_UNSUPPORTED_DEVICE = 2, /* device is not compute capability 10.0 ([ND] "Hardware support") */
  SVDQ_ERR_CUDA = 3,               /* a CUDA runtime call failed (message in svdq_last_error) */
  SVDQ_ERR_OOM = 4,                /* a device or host allocation in svdq_prepare_weights failed */
  SVDQ_ERR_TIMEOUT = 5,            /* a kernel's bounded wait gave up (see svdq_get_device_error) */
  SVDQ_ERR_INTERNAL = 6
} svdq_status;

/* SVDQ_NVFP4 and SVDQ_INT4: the W4A4 layer with its low-rank branch.  SVDQ_W4A16: 4-bit weights
 * (the INT4 quantizer, group 64, of the smoothed weight) with 16-bit activations and no low-rank
 * branch, the pages' "awq_w4a16" family ("Introducing Nunchaku Lite"; quantization_config
 * precision int4, group_size 64) for small-M, memory-bound layers: rank must be 0, K <= 49152, the
 * forward is one kernel that needs no workspace (svdq_workspace_size returns 0), and
 * svdq_quant_down, svdq_gemm_up and svdq_export_activations return SVDQ_ERR_INVALID_ARG. */
typedef enum { SVDQ_NVFP4 = 0, SVDQ_INT4 = 1, SVDQ_W4A16 = 2 } svdq_precision;

/* Opaque prepared layer: device buffers owned by the library until svdq_free_weights. */
typedef struct svdq_weights svdq_weights;

/* Offline parameters, the C mirror of [ND] quantization_config's svdq_w4a4 block. */
typedef struct {
  int precision;   /* svdq_precision */
  int rank;        /* r of the low-rank branch; 0 disables it ([MC] stage 3) */
  float alpha;     /* smoothing exponent: lam_k = a_k^alpha * w_k^(alpha-1); 0.5 gives sqrt(a/w) */
  int svd_iters;   /* subspace iterations of the randomized SVD; <= 0 selects the default (12) */
  uint64_t seed;   /* seed of the randomized SVD's Gaussian test matrix */
} svdq_prepare_params;

/* Shapes and group size of a prepared layer. */
typedef struct {
  int N, K, rank, precision, group, device;
} svdq_weights_info;

/* ------------------------------------------------------------------ status / device */

/* Static string for a status code; never NULL. */
const char* svdq_status_string(svdq_status s);

/* Detailed message of the last failing call on this thread ("" if none).  The pointer
 * stays valid until the next call on the same thread. */
const char* svdq_last_error(void);

/* Load-time capability validation ([ND] "Hardware support": raise a clear error instead
 * of producing incorrect outputs).  OK only for compute capability 10.0 (B200/GB200). */
svdq_status svdq_check_device(int device);

/* Synchronises `stream`, then reads and clears the device error word that kernels set
 * when a bounded wait gives up.  SVDQ_ERR_TIMEOUT if any bit was set, else SVDQ_OK. */
svdq_status svdq_get_device_error(void* stream);

/* ------------------------------------------------------------------ offline prepare */

/* [MC] stages 2-3, once per layer, on the host except the final uploads:
 *   lam_k = a_k^alpha w_k^(alpha-1) (a_k = act_absmax[k], w_k = max_n |W[n,k]|; 1 if either is 0),
 *   W_hat = W diag(lam) (fp64),  top-`rank` SVD of W_hat by randomized subspace iteration,
 *   L1 = U_r sqrt(S), L2 = sqrt(S) V_r^T (bf16),  R = W_hat - U_r S V_r^T (fp32),
 *   R quantized per group along K (same quantizer as the activations).
 * W_bf16:     host, N x K row-major bf16 bits (nn.Linear weight).
 * bias_bf16:  host, N bf16 bits, or NULL for no bias.
 * act_absmax: host, K fp32, the calibration statistic max_m |X[m,k]|.
 * device:     CUDA ordinal that will run the forward; `stream` orders the uploads, and the
 *             call synchronises it before returning.
 * out:        receives the handle; free it with svdq_free_weights.
 * Errors: INVALID_ARG (shape/params), UNSUPPORTED_DEVICE, OOM, CUDA. */
svdq_status svdq_prepare_weights(const uint16_t* W_bf16, int N, int K, const uint16_t* bias_bf16,
                                 const float* act_absmax, const svdq_prepare_params* params,
                                 int device, void* stream, svdq_weights** out);

svdq_status svdq_free_weights(svdq_weights* w);

/* A second, independent handle holding device copies of `src`'s buffers (same device, same
 * operands; copies ordered on `stream`, which the call synchronises).  Useful to run several
 * instances of a layer without repeating the offline SVD.  Errors: INVALID_ARG, OOM, CUDA. */
svdq_status svdq_clone_weights(const svdq_weights* src, void* stream, svdq_weights** out);

svdq_status svdq_get_weights_info(const svdq_weights* w, svdq_weights_info* info);

/* Canonical (row-major, untiled) host copies of the prepared operands, for checking the
 * layer against an independent implementation.  Any pointer may be NULL to skip it.
 *   inv_lambda: K fp32 (fp32 of 1/lam)         codes_w: N x K/2 bytes (element 2i in bits 3:0)
 *   scales_w:   NVFP4 N x K/16 UE4M3 bytes;   INT4 N x K/64 fp32
 *   L1: K x rank bf16    L2: rank x N bf16    bias: N bf16 (zeros when prepared without bias)
 *   sigma: rank fp64 singular values of W_hat (descending). */
svdq_status svdq_export_weights(const svdq_weights* w, float* inv_lambda, uint8_t* codes_w,
                                void* scales_w, uint16_t* L1, uint16_t* L2, uint16_t* bias,
                                double* sigma);

/* ------------------------------------------------------------------ the hot path */

/* Bytes of device workspace svdq_linear_forward needs for M rows (0 when M == 0). */
svdq_status svdq_workspace_size(const svdq_weights* w, int M, size_t* bytes);

/* The forward ([MC] "Nunchaku Engine Design"): two kernels on `stream`.
 *   kernel 1 (Quantize + Down Projection): reads X once; per token and K-group computes
 *     x_hat = fp32(x) * inv_lambda_k, the group scale and the 4-bit codes, and the bf16
 *     low-rank product T = bf16(x_hat) L1 (fp32 accumulation, rounded to bf16);
 *   kernel 2 (4-Bit Compute + Up Projection): block-scaled 4-bit GEMM of the codes against
 *     Q4(R) on the tensor cores, plus T L2 and the bias into the same fp32 accumulator;
 *     writes Y = bf16_rn(acc) once.
 * X:  device, M rows of K bf16, row stride ldx elements.   Y: device, M x N bf16, stride ldy.
 * workspace: device, >= svdq_workspace_size(w, M) bytes, 256-byte aligned; holds the codes,
 *   scales and T between the two kernels (every row up to M rounded up to a multiple of 256)
 *   and, when kernel 1 splits K, the fp32 partials of T and one arrival counter per 16-row block;
 *   contents are scratch and need no initialisation (kernel 1 writes every byte kernel 2 reads; a
 *   counter tagged with another launch restarts, the last slice resets it).  One workspace must
 *   not be used by two forwards whose kernels overlap on the GPU.
 * No allocation, no synchronisation.  Errors: INVALID_ARG, CUDA (launch failure). */
svdq_status svdq_linear_forward(const svdq_weights* w, const void* X, int M, int ldx, void* Y, int ldy,
                                void* workspace, size_t workspace_bytes, void* stream);

/* The forward without a caller workspace and without any device allocation.  The pages have no
 * counterpart to this call: it exists for callers that cannot allocate device memory while they
 * run, for instance code inside a host framework that owns all device memory and hands its
 * plugins no allocator, or a latency-critical path where cudaMalloc (which may synchronise the
 * device) is not acceptable.  The scratch between the two kernels is a fixed 20 MiB array in the
 * library's own device module, which every GPU that loads the library keeps until the process
 * exits.  The first call on a device looks up that array's device address (cudaGetSymbolAddress,
 * with the device current) and caches it; make that first call before any stream capture.  The
 * cache is keyed by the device's current context as well, so after cudaDeviceReset the next call
 * looks the address up again (in the new context, again before any capture).
 * All calls on a device share the one array and it keeps the contents of the last call: calls
 * whose kernels overlap on the GPU (different streams, no ordering between them) race and give
 * wrong results, so order them on one stream or use svdq_linear_forward with separate
 * workspaces.  Nothing in the array has to start at zero.  Shapes whose workspace
 * (svdq_workspace_size) exceeds 20 MiB are rejected with SVDQ_ERR_INVALID_ARG: a shape is
 * accepted exactly when its svdq_workspace_size fits in 20 MiB (at K = 3072 and rank 32 today every
 * M up to 9984 does; the size is not monotonic in M, since kernel 1's K-split partials vanish once
 * a 128-row tile gets a single slice; it moves with the workspace layout, so query
 * svdq_workspace_size rather than relying on that figure).  A W4A16 layer uses no scratch and has no such limit.
 * Other arguments and errors as svdq_linear_forward. */
svdq_status svdq_linear_forward_noalloc(const svdq_weights* w, const void* X, int M, int ldx, void* Y, int ldy,
                                        void* stream);

/* Bytes of the packed rotary table of M tokens (M rounded up to a multiple of 32 rows of
 * head_dim fp32).  head_dim must be 128.  Errors: INVALID_ARG. */
svdq_status svdq_rope_packed_size(int M, int head_dim, size_t* bytes);

/* Packs a rotary table for svdq_linear_forward_qkv_norm_rope.  rope: device, M rows of head_dim/2
 * (cos, sin) fp32 pairs (row stride head_dim floats), 16-byte aligned: row m holds the angles of
 * token m.  packed: device, >= svdq_rope_packed_size(M) bytes, 16-byte aligned, caller-owned.  The
 * packed layout puts the same 16 bytes of 32 consecutive rows side by side, so that the epilogue's
 * warps (one row per lane) read whole 512-byte segments; rows past M repeat row M - 1.  Asynchronous
 * on `stream`; no allocation.  A layout change only, not in the pages.  Errors: INVALID_ARG (head_dim
 * other than 128, NULL or misaligned pointer, buffer too small), CUDA. */
svdq_status svdq_pack_rope(const float* rope, int M, int head_dim, float* packed, size_t packed_bytes, void* stream);

/* The grouped QKV projection with its Q/K normalization and rotary embedding in one operator
 * ([ND] "Quantizing models with structural rewrites": the fused operator consumes the QKV
 * projection, norm_q, norm_k and the rotary embedding; Q, K and V are concatenated along the
 * output dimension in that order).  The pages name the steps only; the library reads them as:
 * the layer's output row (before its rounding to bf16) holds H heads of Q, then H of K, then H
 * of V, `head_dim` channels each; every Q and K head vector x becomes
 *   x / sqrt(mean(x^2) + eps) * gamma   (RMS normalization, gamma_q for Q, gamma_k for K),
 * and then each channel pair (2i, 2i+1) of it is turned by the row's angle i:
 *   (a, b) -> (a cos - b sin, a sin + b cos);
 * V passes unchanged.  Y is rounded to bf16 once, as in svdq_linear_forward.
 * The normalization and rotation run in the epilogue of kernel 2 (NVFP4: one thread holds one
 * row of one head; INT4: half of it, the two halves exchanging their sums of squares).  NVFP4 or
 * INT4 layer, head_dim = 128 and N a multiple of 3 * 128.
 * gamma_q, gamma_k: device, head_dim fp32 each, 16-byte aligned.
 * rope: device, the rotary table of the M tokens packed by svdq_pack_rope (for this M), 16-byte
 *       aligned.  A model computes its table once per resolution and every QKV layer reuses it.
 * eps:  >= 0 and finite (FLUX uses 1e-6).
 * Other arguments, workspace rules and errors as svdq_linear_forward; INVALID_ARG also for a
 * W4A16 layer, another head_dim, N not a multiple of 3 * head_dim, or a bad pointer. */
svdq_status svdq_linear_forward_qkv_norm_rope(const svdq_weights* w, const void* X, int M, int ldx, void* Y,
                                              int ldy, const float* gamma_q, const float* gamma_k, float eps,
                                              const float* rope, int head_dim, void* workspace,
                                              size_t workspace_bytes, void* stream);

/* The fused MLP pair ([ND] "Introducing Nunchaku Lite": fused GELU/MLP kernels; the pages give no
 * formula).  The library reads it as the unfused module sequence: Y = down(h) with
 *   h = bf16(GELU(bf16(up(X)))),  GELU(x) = x Phi(x) (Phi the standard normal distribution),
 * fused so that h never goes through memory: the up layer's kernel 2 computes h in its epilogue
 * and writes, instead of its output, the down layer's activation codes and scales of h and the
 * fp32 partials of the down layer's T (warp-level bf16 MMAs per half tile); a small kernel adds
 * the partials in a fixed order into T; the down layer's kernel 2 then runs as usual.  GELU is
 * rounded correctly to bf16 (a shared-memory table of exact values for |x| in [2^-10, 16), closed
 * forms outside it; svdq_selftest_gelu_bf16 runs the same path).
 * Both layers NVFP4, up->N == down->K, the down layer's rank 0, 16 or 32, same device.
 * ws_up: the up layer's workspace (svdq_workspace_size(up, M)).  ws_mid: the down layer's
 * workspace followed by the T partials, svdq_mlp_workspace_size(up, down, M) bytes, 256-byte
 * aligned (after the call it holds the down layer's kernel-1 outputs: svdq_export_activations
 * (down, ws_mid, ...) reads them).  Y: M x down->N bf16, row stride ldy.
 * No allocation, no synchronisation.  Errors: INVALID_ARG, CUDA. */
svdq_status svdq_mlp_workspace_size(const svdq_weights* up, const svdq_weights* down, int M, size_t* bytes);
svdq_status svdq_mlp_forward(const svdq_weights* up, const svdq_weights* down, const void* X, int M, int ldx,
                             void* Y, int ldy, void* ws_up, size_t ws_up_bytes, void* ws_mid,
                             size_t ws_mid_bytes, void* stream);

/* The forward with GELU on its output: Y = bf16(GELU(bf16(acc + bias))), GELU as in
 * svdq_mlp_forward (correctly rounded).  The lighter of the two fusions of an MLP pair ([ND]
 * "Introducing Nunchaku Lite" names fused GELU/MLP kernels): GELU in the up layer's kernel 2
 * epilogue, Y (the hidden activation) written once and read by the down layer's own forward,
 * whose kernel 1 quantizes it; svdq_mlp_forward instead keeps the hidden activation out of memory
 * but does the quantization in the up layer's epilogue.  NVFP4 layers only (INVALID_ARG
 * otherwise).  Arguments, workspace and errors as svdq_linear_forward. */
svdq_status svdq_linear_forward_gelu(const svdq_weights* w, const void* X, int M, int ldx, void* Y, int ldy,
                                     void* workspace, size_t workspace_bytes, void* stream);

/* Kernel 1 alone (same arguments as the forward minus Y): fills the workspace. */
svdq_status svdq_quant_down(const svdq_weights* w, const void* X, int M, int ldx, void* workspace,
                            size_t workspace_bytes, void* stream);

/* Kernel 2 alone: consumes a workspace filled by svdq_quant_down for the same M. */
svdq_status svdq_gemm_up(const svdq_weights* w, int M, void* Y, int ldy, const void* workspace,
                         size_t workspace_bytes, void* stream);

/* Copies kernel 1's outputs out of `workspace` into canonical host layouts (synchronises
 * `stream`): codes_x M x K/2 bytes, scales_x (NVFP4: M x K/16 UE4M3 bytes; INT4: M x K/64
 * fp32), T M x rank bf16.  Any output pointer may be NULL. */
svdq_status svdq_export_activations(const svdq_weights* w, const void* workspace, size_t workspace_bytes,
                                    int M, uint8_t* codes_x, void* scales_x, uint16_t* T, void* stream);

/* ------------------------------------------------------------------ host-only helpers */

/* The library's host quantizer on fp32 rows (the one svdq_prepare_weights applies to R):
 * V host rows x K fp32; codes rows x K/2; scales as in svdq_export_weights.  No GPU. */
svdq_status svdq_quantize_rows_host(const float* V, int rows, int K, int precision, uint8_t* codes,
                                    void* scales);

/* The offline prepare without a device: same arithmetic as svdq_prepare_weights, results
 * in the canonical layouts of svdq_export_weights (each output may be NULL). */
svdq_status svdq_prepare_host(const uint16_t* W_bf16, int N, int K, const uint16_t* bias_bf16,
                              const float* act_absmax, const svdq_prepare_params* params,
                              float* inv_lambda, uint8_t* codes_w, void* scales_w, uint16_t* L1,
                              uint16_t* L2, double* sigma, float* R_out);

/* ------------------------------------------------------------------ failure detection */

/* Launches a one-block kernel that waits, with the library's bounded-wait routine, on a
 * shared-memory barrier that nothing signals, for at most `spin_limit` polls; on giving up
 * it sets the device error word and returns.  Lets a test check that a wait that runs out
 * is reported as SVDQ_ERR_TIMEOUT by svdq_get_device_error while the context stays usable. */
svdq_status svdq_selftest_wait_timeout(int spin_limit, void* stream);

/* The bf16 GELU of the fused MLP pair's epilogue (svdq_mlp_forward), applied to n bf16 values:
 * out[i] = the nearest bf16 (ties to even) of y Phi(y), y = in[i], Phi the standard normal
 * distribution function ([ND] "Introducing Nunchaku Lite": fused GELU/MLP kernels; the library
 * reads GELU as the exact erf form).  in, out: device, n uint16 bf16 patterns each; asynchronous
 * on `stream`.  A test hook: a bf16 input has only 2^16 values, so a test can check the epilogue's
 * GELU on every one of them.  Errors: INVALID_ARG (n < 0, NULL buffer with n > 0), CUDA. */
svdq_status svdq_selftest_gelu_bf16(const uint16_t* in, uint16_t* out, int n, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SVDQ_H_ */
