/*
 * autoround.h — C ABI of libautoround.so: the AutoRound weight-quantization
 * tuning step, INT4 export and the W4A16 matmul on one NVIDIA B200 (sm_100a).
 *
 * Sources cited below (page title, then section):
 *  [AR] "Low-Bit Quantization in Practice with vLLM: Core Mechanisms and
 *       Architectural Optimizations of AutoRound" — §2 "Minimal Example",
 *       §3 "Optimization Variables" table, §3 "Algorithm Flow", §3 "SignSGD",
 *       §4 "QDQ Fake Quantization vs. Real Inference" (comparison table and
 *       "Minimal State Evolution" table), §8 preset-mode table.
 *  [QC] "量化：从 Scale 到 W4A8 的完整坐标" — §1.2 basic integer mapping.
 *  [IA] "Intel AutoRound 高级量化" (hotdry blog) — sign-gradient mechanism
 *       (STE), production parameter advice (int4 g128 lr 0.005; int8 g256 lr 0.002).
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers on the current CUDA device unless
 *    stated otherwise, row-major, densely packed, 16-byte aligned.
 *  - bf16 / fp16 tensors are passed as uint16_t bit patterns.
 *  - The caller owns every buffer.  The library never allocates or frees
 *    device memory; scratch comes from the caller's workspace.
 *  - Calls are asynchronous on `stream` (NULL = legacy default stream).  The
 *    return value covers host-side validation and kernel launch only.
 *    Device-side problems (non-finite inputs or gradients, a pipeline wait that
 *    timed out) set a sticky status word read by ar_get_device_status().
 *  - No silent fallback: an unsupported combination returns
 *    AR_ERR_UNSUPPORTED and launches nothing.
 *  - On any error return nothing has been launched and ar_last_error() holds
 *    a one-line reason.
 */
#ifndef AUTOROUND_H_
#define AUTOROUND_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define AR_API __attribute__((visibility("default")))
#else
#define AR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* ar_stream_t; /* same handle as cudaStream_t */

typedef enum {
  AR_OK = 0,
  AR_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size or shape */
  AR_ERR_UNSUPPORTED = 2, /* valid request the library does not implement */
  AR_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed */
  AR_ERR_NONFINITE = 4,   /* device status: NaN/Inf seen in an input or gradient */
  AR_ERR_TIMEOUT = 5,     /* device status: a pipeline wait gave up */
  AR_ERR_WORKSPACE = 6    /* workspace missing or smaller than required */
} ar_status;

/* Quantizer and optimiser settings ([AR] §3 table and §8 presets; [IA]).
 *  bits        2..8 (ar_pack_int4 and ar_w4a16_gemm: 4 only)
 *  group_size  weights per group along in_features (K); must divide K.
 *              ar_qdq: 8, 16, ..., 1024 (power of two);
 *              ar_tune_step: 32, 64, 128 or 256.
 *  symmetric   0: asymmetric (s = (hi-lo)/(2^b-1), zp = round(-lo/s));
 *              1: symmetric  (s = max(hi,-lo)/(2^(b-1)-1), zp = 2^(b-1)).
 *  lr          SignSGD step ([AR] §3 "SignSGD"; 5e-3 in all presets).
 *  iters       default step count for drivers; ar_tune_step takes n_steps.
 *  v_min/v_max bounds of the rounding offsets V ([AR] §3 table: -0.5, 0.5).
 *  clip_min/clip_max bounds of the clip factors alpha, beta (0.5, 1.0).     */
typedef struct {
  int bits;
  int group_size;
  int symmetric;
  float lr;
  int iters;
  float v_min, v_max;
  float clip_min, clip_max;
} ar_qconfig;

/* Fills *cfg with the defaults: 4 bits, group 128, asymmetric, lr 5e-3,
 * 200 iterations, V in [-0.5, 0.5], alpha/beta in [0.5, 1]. */
AR_API void ar_qconfig_default(ar_qconfig* cfg);

/* One quantized linear layer of a block.
 *  W      bf16 [N][K], original weights (read only)
 *  V      fp32 [N][K], rounding offsets (in/out for ar_tune_step)
 *  alpha  fp32 [N][K/group_size], multiplier of the group maximum (in/out)
 *  beta   fp32 [N][K/group_size], multiplier of the group minimum (in/out) */
typedef struct {
  const uint16_t* W;
  float* V;
  float* alpha;
  float* beta;
  int64_t N; /* out_features */
  int64_t K; /* in_features */
} ar_layer;

/* Optional gradient outputs of the LAST step of an ar_tune_step call (any
 * pointer may be NULL).  Same shapes as V, alpha, beta of each layer. */
typedef struct {
  float* dV;
  float* dalpha;
  float* dbeta;
} ar_grads;

typedef enum {
  AR_BLOCK_LINEAR = 0,    /* one linear layer: Y = X W^T (n_layers = 1) */
  AR_BLOCK_SWIGLU_MLP = 1 /* SwiGLU MLP: Y = (silu(X Wg^T) * (X Wu^T)) Wd^T; layers = {gate, up, down},
                             gate/up [F][H], down [H][F] (n_layers = 3) */
} ar_block_kind;

/* ------------------------------------------------------------------------ */

/* fp32 -> bf16 (round to nearest even) of n values: src fp32 [n], dst bf16 [n].
 * Marshalling for fp32 workloads: the tuning path runs on bf16 X and W
 * ([AR] §3 "Algorithm Flow" step 2: the reference uses the BF16 weights). */
AR_API ar_status ar_f32_to_bf16(const float* src, uint16_t* dst, int64_t n, ar_stream_t stream);

/* Fake-quant (QDQ) forward of one weight matrix ([AR] §4 comparison table,
 * "QDQ" column; [AR] §2 "Minimal Example"; [QC] §1.2):
 *   mx = max(0, max_group W),  mn = min(0, min_group W)
 *   hi = alpha*mx, lo = beta*mn, s = (hi-lo)/(2^b-1) (>= 1e-8), zp = round(-lo/s)
 *   q  = clamp(round(W/s + V) + zp, 0, 2^b-1),  W_hat = s*(q - zp)
 * All arithmetic in fp32 IEEE operations (no contraction), round() is half
 * away from zero.
 * Inputs:  W bf16 [N][K]; V fp32 [N][K]; alpha, beta fp32 [N][K/g].
 * Outputs (each may be NULL, at least one non-NULL):
 *   W_hat bf16 [N][K] (round to nearest even); codes uint8 [N][K];
 *   scale fp32 [N][K/g]; zero fp32 [N][K/g] (integer valued).
 * Errors: AR_ERR_INVALID_ARG (shape, alignment, K % g), AR_ERR_UNSUPPORTED
 * (bits or group_size outside the ranges above). */
AR_API ar_status ar_qdq(const uint16_t* W, const float* V, const float* alpha, const float* beta, int64_t N, int64_t K,
                 const ar_qconfig* cfg, uint16_t* W_hat, uint8_t* codes, float* scale, float* zero,
                 ar_stream_t stream);

/* Reference forward of one linear layer with its original weights ([AR] §3
 * "Algorithm Flow" step 2): Y fp32 [M][N] = X bf16 [M][K] x W bf16 [N][K]^T,
 * fp32 accumulation on the tensor cores.  Needs N % 8 == 0, K % 8 == 0.
 * No workspace. */
AR_API ar_status ar_linear_forward(const uint16_t* X, int64_t M, const uint16_t* W, int64_t N, int64_t K, float* Y,
                            ar_stream_t stream);

/* Bytes of workspace ar_block_forward needs (0 on invalid input). */
AR_API size_t ar_block_forward_workspace(int block_kind, const ar_layer* layers, int n_layers, int64_t M);

/* Reference output of a block with its original weights ([AR] §3 "Algorithm
 * Flow" step 2; for the SwiGLU block [AR] §3 "Why Block-Wise Optimization").
 * AR_BLOCK_LINEAR: as ar_linear_forward.  AR_BLOCK_SWIGLU_MLP: a = bf16(X Wg^T),
 * b = bf16(X Wu^T), h = bf16(silu(a) b) (workspace holds h, M x F bf16),
 * Y fp32 [M][H] = h Wd^T.  Only layers[i].W are read. */
AR_API ar_status ar_block_forward(int block_kind, const ar_layer* layers, int n_layers, const uint16_t* X, int64_t M,
                                  float* Y, void* workspace, size_t workspace_bytes, ar_stream_t stream);

/* Bytes of workspace ar_tune_step needs for this block, M tokens and
 * n_steps steps (0 on invalid input; see ar_last_error()). */
AR_API size_t ar_tune_step_workspace(int block_kind, const ar_layer* layers, int n_layers, int64_t M,
                              const ar_qconfig* cfg, int n_steps);

/* n_steps SignSGD tuning steps of one block ([AR] §3 "Algorithm Flow" steps
 * 3-5, "SignSGD"; [IA] STE):
 *   QDQ forward -> Y_hat = X W_hat^T -> R = Y_hat - Y, loss = sum R^2/(M N),
 *   G = bf16(2R/(M N)) -> dW_hat = G^T X -> straight-through fold:
 *     dV = g s m,  c = g((q-zp) - m W/s - (1-m) lo/s),
 *     dalpha = mx sum_group(c)/Q,  dbeta = mn (-sum_group(c)/Q + sum_group g(1-m))
 *   (m = 1 where 0 <= round(W/s+V)+zp <= Q) -> p <- clamp(p - lr sign(dp)).
 * X: bf16 [M][K] calibration activations (all M rows are used every step).
 * Y: fp32 [M][N], the reference output of ar_linear_forward (required).
 * layers[0].V/alpha/beta are updated in place after every step.
 * loss_per_step: device fp32 [max(n_steps,1)]; entry i is the loss of the
 *   state before update i.  n_steps = 0 evaluates the loss of the current
 *   state into loss_per_step[0] and updates nothing.
 * grads: NULL, or an array of n_layers gradient outputs of the last step.
 * AR_BLOCK_SWIGLU_MLP (n_layers = 3: gate, up, down) tunes the three weights
 *   jointly against the block output ([AR] §3 "Why Block-Wise Optimization"):
 *   h = bf16(silu(a) b) with a, b the bf16 gate/up products; G as above on the
 *   block output (M x H); dWd = G^T h; dH = G Wd_hat; dA = bf16(dH b silu'(a)),
 *   dB = bf16(dH silu(a)); dWg = dA^T X, dWu = dB^T X; each folded and
 *   updated as above.  X [M][H] bf16, Y [M][H] fp32 from ar_block_forward.
 * workspace: device buffer of at least ar_tune_step_workspace() bytes.
 * Where the fold runs (the same values either way, up to the order of a
 * group's sums): from 8192 tokens the weight-gradient GEMM folds and updates
 * in its epilogue (dW_hat never leaves the SM); an AR_BLOCK_LINEAR step with
 * fewer tokens and group_size <= 128 writes dW_hat (fp32 [N][K]) to the
 * workspace and a separate kernel folds, updates and takes the next step's QDQ,
 * so that only the first step runs the QDQ kernel.
 * Supported: AR_BLOCK_LINEAR with n_layers = 1 and AR_BLOCK_SWIGLU_MLP with
 * n_layers = 3; bits 2..8; group_size 32, 64, 128, 256 dividing every K;
 * N % 8 == 0 (H, F % 8 == 0 for the MLP).
 * Errors: AR_ERR_INVALID_ARG, AR_ERR_UNSUPPORTED, AR_ERR_WORKSPACE. */
AR_API ar_status ar_tune_step(int block_kind, const ar_layer* layers, int n_layers, const uint16_t* X, int64_t M,
                       const float* Y, const ar_qconfig* cfg, int n_steps, float* loss_per_step,
                       const ar_grads* grads, void* workspace, size_t workspace_bytes, ar_stream_t stream);

/* ar_tune_step for a shard of one linear layer's output rows (AR_BLOCK_LINEAR;
 * [AR] §3 "Algorithm Flow" steps 3-5).  Output rows of a linear layer are
 * independent: row n of W, V, alpha, beta only meets column n of Y and of G.
 * So a layer of N_total rows splits over GPUs by rows with no exchange on the
 * data path; each GPU passes its rows (*layer: W, V, alpha, beta [N][K], N
 * rows of the N_total), the full X [M][K] and its columns of the reference
 * output Y [M][N] (ar_linear_forward of its rows).  The only difference from
 * ar_tune_step is the loss normaliser: M * n_total instead of M * N, so
 *   G = bf16(2 R / (M n_total))
 * is bit for bit the whole layer's G on these rows, and every update matches
 * the unsharded call's rows exactly.  loss_per_step[i] is this shard's part of
 * the layer's loss, sum_shard R^2 / (M n_total): the shards' values add up to
 * the layer's loss (a one-float all-reduce, for reporting only).
 * Workspace: ar_tune_step_workspace of the shard (AR_BLOCK_LINEAR, *layer).
 * Errors: as ar_tune_step; AR_ERR_INVALID_ARG if n_total < layer->N. */
AR_API ar_status ar_tune_step_shard(const ar_layer* layer, const uint16_t* X, int64_t M, const float* Y,
                                    int64_t n_total, const ar_qconfig* cfg, int n_steps, float* loss_per_step,
                                    const ar_grads* grads, void* workspace, size_t workspace_bytes,
                                    ar_stream_t stream);

/* ---- the decoder block ([AR] §3 "Why Block-Wise Optimization", "Algorithm
 * Flow": the decoder block, not the layer, is the unit of tuning) ----------
 * The pages name the block but not its layers; this is the Llama family's
 * pre-norm block on X [M][H] bf16, M = samples * seq_len tokens:
 *   r1 = bf16(rmsnorm(X) gamma1), rmsnorm(x) = x / sqrt(mean(x^2) + 1e-6)
 *   Q, K, V = r1 Wq^T, r1 Wk^T, r1 Wv^T  (n_heads heads of d = H / n_heads)
 *   Qr, Kr = Q, K with the rotary embedding: in every head, (x_i, x_{i+d/2})
 *            -> (x_i c - x_{i+d/2} s, x_{i+d/2} c + x_i s), c, s = cos, sin of
 *            t 10000^(-2i/d), t the token's position in its sample
 *   O      = softmax(Qr Kr^T / sqrt(d) + causal mask) V per sample and head
 *   X2     = X + O Wo^T;  r2 = bf16(rmsnorm(X2) gamma2)
 *   Y      = X2 + (silu(r2 Wg^T) * (r2 Wu^T)) Wd^T
 * Rounding points (each operand of a product is bf16, the rest fp32): r1, Qr,
 * Kr, V, the attention probabilities P = bf16(exp(z - lse)) (z the scaled
 * scores, lse the row's log-sum-exp over its keys), O, r2, the MLP's a, b, h;
 * X2 and Y are fp32.  In the backward: G, dA, dB, dX2 (the gradient at X2),
 * dO, dS (the softmax gradient times 1/sqrt(d)), dQ, dK (after the inverse
 * rotation) and dV are bf16.
 * layers: seven ar_layer in the order q, k, v, o, gate, up, down; q, k, v, o
 * [H][H], gate, up [F][H], down [H][F]. */
typedef struct {
  int64_t hidden;       /* H: a multiple of 128 */
  int64_t intermediate; /* F: a multiple of 8 */
  int n_heads;          /* head dim d = H / n_heads, 64 or 128 */
  int64_t seq_len;      /* L: tokens per sample, a multiple of 64; M % L == 0 */
  const float* gamma1;  /* device fp32 [H], the two norms' scales (not tuned) */
  const float* gamma2;
} ar_decoder_cfg;

/* Bytes of workspace ar_decoder_forward needs (0 on invalid input). */
AR_API size_t ar_decoder_forward_workspace(const ar_decoder_cfg* dcfg, int64_t M);

/* The block's output with its original weights ([AR] §3 "Algorithm Flow" step
 * 2): Y fp32 [M][H].  Only layers[i].W are read.  Workspace: device, 256-byte
 * aligned.  Errors: AR_ERR_INVALID_ARG / AR_ERR_UNSUPPORTED /
 * AR_ERR_WORKSPACE before any launch. */
AR_API ar_status ar_decoder_forward(const ar_decoder_cfg* dcfg, const ar_layer* layers, const uint16_t* X, int64_t M,
                                    float* Y, void* workspace, size_t workspace_bytes, ar_stream_t stream);

/* Bytes of workspace ar_tune_step_decoder needs (0 on invalid input). */
AR_API size_t ar_tune_step_decoder_workspace(const ar_decoder_cfg* dcfg, const ar_layer* layers, int64_t M,
                                             const ar_qconfig* cfg, int n_steps);

/* n_steps joint SignSGD steps on the block's seven weights ([AR] §3
 * "Algorithm Flow" steps 3-5, "SignSGD"; straight-through fold as in
 * ar_tune_step): QDQ of the seven weights, the block forward above with the
 * fake-quantized weights, R = Y_hat - Y, loss = sum R^2 / (M H),
 * G = bf16(2R/(M H)), the block's backward to the seven dW_hat, each folded
 * into dV, dalpha, dbeta and applied as p <- clamp(p - lr sign(dp)).
 * Y: fp32 [M][H] from ar_decoder_forward.  loss_per_step, n_steps, grads (an
 * array of seven, or NULL) and the in-place updates as in ar_tune_step.
 * Supported: bits 2..8, group_size 32..256 dividing H and F, the shapes of
 * ar_decoder_cfg.  Errors before any launch as ar_tune_step. */
AR_API ar_status ar_tune_step_decoder(const ar_decoder_cfg* dcfg, const ar_layer* layers, const uint16_t* X,
                                      int64_t M, const float* Y, const ar_qconfig* cfg, int n_steps,
                                      float* loss_per_step, const ar_grads* grads, void* workspace,
                                      size_t workspace_bytes, ar_stream_t stream);

/* The block's parts on their own (the tuning step runs exactly these kernels):
 * r [M][H] bf16 = bf16(rmsnorm(x) gamma) and inv [M] fp32 = 1/sqrt(mean(x^2) +
 * 1e-6) (inv may be NULL); x bf16 (x_is_f32 = 0) or fp32 [M][H]; H % 8 == 0. */
AR_API ar_status ar_rmsnorm(const void* x, int x_is_f32, const float* gamma, int64_t M, int64_t H, uint16_t* r,
                            float* inv, ar_stream_t stream);

/* Causal softmax attention per sample and head on qkv [S*L][3H] bf16 (columns
 * Qr | Kr | V, the rotation already applied): out [S*L][H] bf16 = P V with
 * P = bf16(exp(z - lse)), z = Qr Kr^T / sqrt(d) (fp32), and lse fp32 [S][nh][L].
 * Needs L % 64 == 0, d = H / n_heads in {64, 128}.  d = 128 with L % 128 == 0
 * runs on tcgen05 (128-query CTAs, S and O in tensor memory, the exponential
 * as 2^x by the hardware after one fused multiply-add); other shapes on
 * mma.sync.  Both compute the two passes the same way (lse, then P). */
AR_API ar_status ar_attention_forward(const uint16_t* qkv, int64_t S, int64_t L, int64_t H, int n_heads,
                                      uint16_t* out, float* lse, ar_stream_t stream);

/* Its backward from dO [S*L][H] bf16: dqkv [S*L][3H] bf16 = dQ | dK | dV, with
 * dQ and dK taken back through the rotation (dQ = R^T dQr).  out and lse are
 * the forward's.  d = 128 with L % 128 == 0 runs two tcgen05 kernels (dQ per
 * 128 queries, dK and dV per 128 keys; no atomics, deterministic); other
 * shapes mma.sync.  Workspace: ar_attention_backward_workspace bytes (device,
 * 256-byte aligned). */
AR_API size_t ar_attention_backward_workspace(int64_t S, int64_t L, int64_t H, int n_heads);
AR_API ar_status ar_attention_backward(const uint16_t* qkv, const uint16_t* out, const uint16_t* dout,
                                       const float* lse, int64_t S, int64_t L, int64_t H, int n_heads,
                                       uint16_t* dqkv, void* workspace, size_t workspace_bytes,
                                       ar_stream_t stream);

/* Fixed scratch size of ar_tune_step_noalloc, in bytes (16 MiB per GPU). */
#define AR_NOALLOC_SCRATCH_BYTES (16 * 1024 * 1024)

/* ar_tune_step without a caller workspace.  The pages have no counterpart:
 * this entry point exists for callers that cannot allocate device memory —
 * a process whose GPU memory is owned by another allocator (for example a
 * framework's caching allocator that has reserved it), or a latency-critical
 * loop that cannot take the implicit device synchronisation of
 * cudaMalloc/cudaFree.  It runs exactly the kernels of ar_tune_step, with
 * the same arguments minus the workspace, and allocates nothing: its scratch
 * is one file-scope device array of AR_NOALLOC_SCRATCH_BYTES that every GPU
 * loading this library holds until the process exits.
 *  - Problems whose ar_tune_step_workspace() exceeds AR_NOALLOC_SCRATCH_BYTES
 *    return AR_ERR_WORKSPACE with the sizes in ar_last_error(); at 4-bit g128
 *    this admits e.g. a 1024x1024 layer with 2048 tokens, not a 4096x4096
 *    layer with 16384 tokens.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current) and keeps it for later
 *    calls; make that first call before any stream capture.  The address is
 *    not looked up again, so do not call this entry point on a device after
 *    cudaDeviceReset() on it in the same process.
 *  - Every call on a device shares the one array and leaves its contents
 *    behind; nothing in it needs to start at zero (each step writes every
 *    scratch byte it later reads).  Calls that overlap on the GPU (other
 *    streams, other host threads) race on the array: serialise them. */
AR_API ar_status ar_tune_step_noalloc(int block_kind, const ar_layer* layers, int n_layers, const uint16_t* X,
                                      int64_t M, const float* Y, const ar_qconfig* cfg, int n_steps,
                                      float* loss_per_step, const ar_grads* grads, ar_stream_t stream);

/* Export the tuned codes as INT4 ([AR] §4 comparison table, "Real INT4
 * Kernel" column: weights stored as 4-bit integers with per-group metadata).
 * Recomputes the codes exactly as ar_qdq does, then writes
 *   packed  uint32 [N][K/8]: element k at bits 4*(k mod 8) of word k/8
 *   scale   fp16  [N][K/g]: fp16(s), round to nearest even
 *   zero    fp16  [N][K/g]: fp16(zp) (exact: integer <= 15)
 * Needs cfg->bits == 4, asymmetric or symmetric, K % 8 == 0. */
AR_API ar_status ar_pack_int4(const uint16_t* W, const float* V, const float* alpha, const float* beta, int64_t N,
                       int64_t K, const ar_qconfig* cfg, uint32_t* packed, uint16_t* scale_f16,
                       uint16_t* zero_f16, ar_stream_t stream);

/* W4A16 matmul ([AR] §4: dequantization fused into the kernel):
 *   out[t][n] = sum_k A[t][k] (q[n][k] - zero[n][k/g]) scale[n][k/g]
 * A bf16 [T][K]; packed/scale/zero as written by ar_pack_int4 (zero must hold
 * integers 0..15, as ar_pack_int4 writes them); out bf16 [T][N] (round to
 * nearest even of the fp32 accumulation).  (q - zero) is exact in bf16; the
 * products are accumulated in fp32 on the tensor cores, one group (or 32-k
 * slice of a group) at a time, and scaled by the group's scale in fp32.
 * T <= 16 runs a decode kernel (mma.sync fragments built in registers, one
 * range of weight rows per SM; when K/g is not a multiple of 8 or scale/zero
 * are not 16-byte aligned, an older decode kernel with 64-row tiles); larger
 * T a tcgen05 GEMM whose dequantization warps write each 128-row tile of
 * (q - zero) into tensor memory as the MMA's A operand.  Results are
 * deterministic for a given T.
 * Supported: 1 <= T < 2^31, group_size 32..1024 (power of two) dividing K,
 * K % 128 == 0; anything else returns AR_ERR_UNSUPPORTED or
 * AR_ERR_INVALID_ARG before any launch. */
AR_API ar_status ar_w4a16_gemm(const uint16_t* A, int64_t T, const uint32_t* packed, const uint16_t* scale_f16,
                        const uint16_t* zero_f16, int64_t N, int64_t K, int group_size, uint16_t* out,
                        ar_stream_t stream);

/* Packed export of the tuned codes at 2, 3, 4 or 8 bits (cfg->bits): the INT4
 * layout of ar_pack_int4 for other widths (the pages define no packing for
 * them; the low-bit tunings need one).  Each row is one little-endian bit
 * stream: element k at stream bits [bits*k, bits*k + bits), stream bit i in
 * bit i mod 32 of the row's word i/32.
 *   packed  uint32 [N][K*bits/32]: for 2, 4, 8 bits element k at bits
 *           bits*(k mod 32/bits) of word k/(32/bits); for 3 bits 32 codes in
 *           3 words, codes 10 and 21 of every 32 straddling two words
 *   scale   fp16  [N][K/g]: fp16(s), round to nearest even
 *   zero    fp16  [N][K/g]: fp16(zp) (exact: integer < 2^bits)
 * Same codes as ar_qdq.  Needs K % (32/bits) == 0 (3 bits: K % 32 == 0) and
 * group_size 8..1024 (power of two) dividing K; other widths return
 * AR_ERR_UNSUPPORTED. */
AR_API ar_status ar_pack_codes(const uint16_t* W, const float* V, const float* alpha, const float* beta, int64_t N,
                               int64_t K, const ar_qconfig* cfg, uint32_t* packed, uint16_t* scale_f16,
                               uint16_t* zero_f16, ar_stream_t stream);

/* WbA16 matmul for codes packed by ar_pack_codes (bits 2, 3, 4 or 8):
 *   out[t][n] = sum_k A[t][k] (q[n][k] - zero[n][k/g]) scale[n][k/g]
 * A bf16 [T][K]; zero must hold integers 0..2^bits-1; out bf16 [T][N].  bits 4
 * is ar_w4a16_gemm.  At T <= 8 with K/group_size a multiple of 8, 2 and 3
 * bits (group_size >= 64, K >= 512) and 8 bits run the W4A16 decode kernel's
 * 2, 3 and 8-bit forms (codes taken at mantissa positions of a bf16 with the
 * paired activations scaled to match; an 8-bit code as its two nibbles); other 2 and
 * 3-bit shapes at T <= 8 run a generic decode kernel (mma.sync, one range of
 * weight rows per SM, the codes read straight from the bit stream); the rest,
 * and every width from 9 tokens, run the tcgen05 dequant
 * GEMM (a 3-bit stage of 128 k is 48 bytes of a row: its code slots hold
 * three 128-byte boxes, eight stages).  (q - z) is exact in bf16 for every width and
 * each group's sum is scaled once in fp32.  Needs 1 <= T < 2^31, group_size
 * 32..1024 (power of two) dividing K, K % 128 == 0; otherwise
 * AR_ERR_UNSUPPORTED or AR_ERR_INVALID_ARG before any launch. */
AR_API ar_status ar_wxa16_gemm(const uint16_t* A, int64_t T, const uint32_t* packed, const uint16_t* scale_f16,
                               const uint16_t* zero_f16, int64_t N, int64_t K, int group_size, int bits,
                               uint16_t* out, ar_stream_t stream);

/* Absolute maximum of n bf16 values: *amax = max_i |x[i]| (device fp32
 * scalar, written; exact, as it is one of the inputs).  The per-tensor
 * statistic of ar_qdq_nvfp4.  Needs n > 0, n % 8 == 0, x 16-byte aligned,
 * amax 4-byte aligned; otherwise AR_ERR_INVALID_ARG before any launch.  A NaN
 * or Inf input raises AR_ERR_NONFINITE in the device status
 * (ar_get_device_status); *amax is then not meaningful. */
AR_API ar_status ar_absmax_bf16(const uint16_t* x, int64_t n, float* amax, ar_stream_t stream);

/* NVFP4 fake quantization: a QDQ function for a new data type ([AR] §4 "Why
 * the Tuning Stage Must Take the QDQ Path", point 3).  Format: E2M1 values (1
 * sign, 2 exponent, 1 mantissa bits; largest 6) with one E4M3 scale (largest
 * finite 448) per block of 16 values and a per-tensor scale ([QC] "量化：从
 * Scale 到 W4A8 的完整坐标" §2 table and §5 row "NVFP4 recipe"; [NQ] "量化",
 * section "低比特浮点：FP8 与 NVFP4").  In fp32, in this order:
 *   S = amax / 2688                         (2688 = 6 * 448; amax = max |W|)
 *   per block b of 16 consecutive values along K:
 *     s_b = E4M3((alpha_b * max_b |W|) / 6 / S) * S
 *     q = E2M1(W / s_b + V),  W_hat = q * s_b     (q = 0, W_hat = 0 if s_b = 0)
 * E4M3 and E2M1 round to nearest, ties to even, and saturate.
 *   W      bf16 [N][K], K % 16 == 0, 16-byte aligned
 *   V      fp32 [N][K] offsets, or NULL (0); 16-byte aligned
 *   alpha  fp32 [N][K/16] clip factors, or NULL (1)
 *   amax   device fp32 scalar, max |W| (ar_absmax_bf16 of W)
 * Outputs, each optional (at least one):
 *   W_hat         bf16 [N][K], round to nearest even; 16-byte aligned
 *   codes         uint8 [N][K/2]: two E2M1 codes per byte along K, element k
 *                 in the low nibble when k is even; 16-byte aligned
 *   scales        uint8 [N][K/16]: the E4M3 codes of s_b / S
 *   global_scale  device fp32 scalar S
 * All device memory is the caller's.  Invalid shapes, pointers or alignment
 * return AR_ERR_INVALID_ARG before any launch. */
AR_API ar_status ar_qdq_nvfp4(const uint16_t* W, const float* V, const float* alpha, int64_t N, int64_t K,
                              const float* amax, uint16_t* W_hat, uint8_t* codes, uint8_t* scales,
                              float* global_scale, ar_stream_t stream);

/* Matmul with NVFP4 weights as ar_qdq_nvfp4 exports them, for bf16 activations:
 *   out[t][n] = S * sum_k A[t][k] * E4M3(scales[n][k/16]) * E2M1(codes[n][k])
 * the real-kernel side of the NVFP4 format ([QC] "量化：从 Scale 到 W4A8 的完整坐标"
 * §2 table and §5 row "NVFP4 recipe"; [NQ] "量化", section "低比特浮点：FP8 与
 * NVFP4": E2M1 values, an E4M3 scale per 16-value block, a per-tensor scale, on
 * Blackwell).  Reading: the pages list the format for weights and activations;
 * this call keeps the activations in bf16 (weight-only NVFP4, like W4A16), so that
 * it consumes exactly what the tuning exports.  Each E2M1 value times its block
 * scale is exact in bf16; the tensor cores (tcgen05) accumulate in fp32 and S
 * scales the fp32 sums; out is rounded to bf16 (nearest even).
 *   A       bf16 [T][K], 16-byte aligned
 *   codes   uint8 [N][K/2]: two E2M1 codes per byte along K, element k in the
 *           low nibble when k is even (ar_qdq_nvfp4's codes); 16-byte aligned
 *   scales  uint8 [N][K/16]: E4M3 codes of the block scales (ar_qdq_nvfp4's
 *           scales); 16-byte aligned
 *   global_scale  device fp32 scalar S (ar_qdq_nvfp4's global_scale)
 *   out     bf16 [T][N], 16-byte aligned
 * Needs 1 <= T < 2^31, N >= 1, K % 128 == 0; otherwise AR_ERR_INVALID_ARG or
 * AR_ERR_UNSUPPORTED before any launch.  All memory is the caller's. */
AR_API ar_status ar_nvfp4_gemm(const uint16_t* A, int64_t T, const uint8_t* codes, const uint8_t* scales,
                               const float* global_scale, int64_t N, int64_t K, uint16_t* out,
                               ar_stream_t stream);

/* Tuning steps of one linear layer on NVFP4: the SignSGD step of ar_tune_step
 * ([AR] §3 "Algorithm Flow" steps 3-5, "SignSGD") with ar_qdq_nvfp4 as its QDQ
 * function ([AR] §4 "Why the Tuning Stage Must Take the QDQ Path", point 3).
 * Per step: W_hat = NVFP4 QDQ of W (V, alpha); Y_hat = X W_hat^T; loss = mean
 * (Y_hat - Y)^2; G = bf16(2 (Y_hat - Y) / (M N)); dW_hat = G^T X; straight-
 * through fold with both roundings (E4M3, E2M1) as the identity and the
 * gradient passed where |W/s_b + V| <= 6:
 *   dV = dW_hat s_b m,   dalpha_b = (amax_b / 6) sum_block dW_hat (q - m W / s_b)
 * then V <- clamp(V - lr sign(dV), v_min, v_max), alpha <- clamp(alpha -
 * lr sign(dalpha), clip_min, clip_max) (cfg's lr and bounds; bits, group_size
 * and symmetric are not used).
 *   W      bf16 [N][K] (K % 16 == 0, N % 8 == 0)
 *   V      fp32 [N][K], alpha fp32 [N][K/16]: the state, updated in place
 *   amax   device fp32 scalar, max |W| (ar_absmax_bf16)
 *   X      bf16 [M][K] (M % 8 == 0), Y fp32 [M][N] the reference output
 *   loss_per_step  device fp32 [max(n_steps, 1)]: each step's loss before its
 *                  update (n_steps = 0: the loss of the current state only)
 *   dV_out [N][K], dalpha_out [N][K/16]: optional, the last step's gradients
 *   workspace      device, 256-byte aligned, ar_tune_step_nvfp4_workspace bytes
 * Errors: AR_ERR_INVALID_ARG / AR_ERR_UNSUPPORTED / AR_ERR_WORKSPACE before any
 * launch. */
AR_API size_t ar_tune_step_nvfp4_workspace(int64_t M, int64_t N, int64_t K, int n_steps);
AR_API ar_status ar_tune_step_nvfp4(const uint16_t* W, float* V, float* alpha, int64_t N, int64_t K, const float* amax,
                                    const uint16_t* X, int64_t M, const float* Y, const ar_qconfig* cfg, int n_steps,
                                    float* loss_per_step, float* dV_out, float* dalpha_out, void* workspace,
                                    size_t workspace_bytes, ar_stream_t stream);

/* Minibatch assembly for block-by-block tuning ([AR] §8 preset table: each
 * iteration works on a batch of 8 -- 4 in the "fast" preset -- of the 128
 * calibration samples; [AR] §3 "Algorithm Flow" steps 3-6 iterate on such
 * batches).  Copies samples idx[0..n_idx-1] of src (n_src_samples samples of
 * sample_bytes each, contiguous) to dst in that order:
 *   dst[i*sample_bytes .. +sample_bytes) = src[idx[i]*sample_bytes .. ).
 * idx is a HOST array, read before the call returns.  Needs 1 <= n_idx <= 64,
 * every idx in [0, n_src_samples), sample_bytes a positive multiple of 16,
 * 16-byte aligned device pointers, dst not overlapping src; otherwise
 * AR_ERR_INVALID_ARG before any launch. */
AR_API ar_status ar_gather_samples(const void* src, int64_t n_src_samples, int64_t sample_bytes, const int32_t* idx,
                                   int n_idx, void* dst, ar_stream_t stream);

/* Plain tensor-core GEMM, fp32 out: D[M][N] = sum_k A(m,k) B(n,k).
 * A is [M][K] (a_mn_major = 0) or [K][M] (a_mn_major = 1); B is [N][K]
 * (b_mn_major = 0) or [K][N] (b_mn_major = 1); all bf16.  The same
 * tcgen05 mainloop as the tuning step, exposed for testing the operand
 * layouts.  Needs N % 8 == 0, K % 8 == 0 and, when A is MN-major, M % 8 == 0. */
AR_API ar_status ar_gemm_bf16(const uint16_t* A, int a_mn_major, const uint16_t* B, int b_mn_major, float* D, int64_t M,
                       int64_t N, int64_t K, ar_stream_t stream);

/* Diagnostic of the failure path (the pages have no counterpart): one warp
 * waits on a device barrier that nothing completes, with the same bounded-wait
 * mechanism the pipelined kernels use but a limit of limit_ns (at most 1 s).
 * The wait gives up, writes 1 to *gave_up (device int) and raises the sticky
 * AR_ERR_TIMEOUT status; the kernel returns normally and the context stays
 * usable.  No fault, trap or hang is involved. */
AR_API ar_status ar_debug_wait_timeout(uint64_t limit_ns, int* gave_up, ar_stream_t stream);

/* Synchronizes `stream`, then returns and clears the sticky device status:
 * AR_OK, AR_ERR_NONFINITE or AR_ERR_TIMEOUT (timeout wins if both are set),
 * or AR_ERR_CUDA if the synchronization itself failed. */
AR_API ar_status ar_get_device_status(ar_stream_t stream);

/* One line describing the last error of this host thread ("" if none). */
AR_API const char* ar_last_error(void);

/* Names of the kernels the last successful call of this host thread launched,
 * separated by ';' (tracing: shows which kernel variant ran). */
AR_API const char* ar_last_kernels(void);

/* Device-time profiling.  Between ar_profile_start() and ar_profile_stop()
 * every kernel launch of this library (any host thread) is bracketed by two
 * CUDA events recorded on its launch stream.  ar_profile_stop() waits for
 * those events and writes one line per kernel name into buf (NUL-terminated,
 * truncated to buf_len):  "<kernel name> <launches> <total device ms>\n".
 * Events come from a pool the library keeps; no device memory is allocated. */
AR_API ar_status ar_profile_start(void);
AR_API ar_status ar_profile_stop(char* buf, size_t buf_len);

/* Library version string. */
AR_API const char* ar_version(void);

#ifdef __cplusplus
}
#endif

#endif /* AUTOROUND_H_ */
