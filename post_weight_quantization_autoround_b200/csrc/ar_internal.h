// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ar_device.cuh"

namespace ar {

constexpr float kScaleGuard = 1e-8f;  // lower bound on a group's scale

// Sets the text ar_last_error() returns on this host thread.
void set_last_error(const char* msg);

// Records the name of a kernel launched by the current API call (tracing).
void trace_kernel(const char* name);

// Wraps one kernel launch: traces its name and, while device profiling is on
// (ar_profile_start), records CUDA events around it on the launch stream.
// `name` must have static storage (a string literal or a static table): it is
// kept after the launch.
class LaunchScope {
 public:
  LaunchScope(cudaStream_t stream, const char* name);
  ~LaunchScope();
  LaunchScope(const LaunchScope&) = delete;
  LaunchScope& operator=(const LaunchScope&) = delete;

 private:
  cudaStream_t stream_;
  const char* name_;
  cudaEvent_t start_;
};

int num_sms();

cudaError_t launch_qdq(const uint16_t* W, const float* V, const float* alpha, const float* beta, int64_t N,
                       int64_t K, int group_size, int bits, int symmetric, uint16_t* W_hat, uint8_t* codes,
                       float* scale, float* zero, float* mx, float* mn, cudaStream_t stream);

cudaError_t launch_pack_int4(const uint16_t* W, const float* V, const float* alpha, const float* beta, int64_t N,
                             int64_t K, int group_size, int symmetric, uint32_t* packed, uint16_t* scale16,
                             uint16_t* zero16, cudaStream_t stream);
// 2, 4 or 8 bits per code, 32/bits codes per uint32 (ar_quant.cu)
cudaError_t launch_pack_codes(const uint16_t* W, const float* V, const float* alpha, const float* beta, int64_t N,
                              int64_t K, int group_size, int bits, int symmetric, uint32_t* packed,
                              uint16_t* scale16, uint16_t* zero16, cudaStream_t stream);

cudaError_t launch_f32_to_bf16(const float* src, uint16_t* dst, int64_t n, cudaStream_t stream);

// 2-D tensor map over a row-major [rows][cols] array (cols contiguous) with a
// box of box_rows x box_cols elements; zero fill out of bounds.
cudaError_t make_tmap_2d(CUtensorMap* tm, CUtensorMapDataType dtype, uint32_t elem_bytes, const void* ptr,
                         uint64_t rows, uint64_t cols, uint32_t box_cols, uint32_t box_rows,
                         CUtensorMapSwizzle swizzle, uint64_t ld = 0);

// ---- tensor-core GEMMs (ar_gemm.cu) ----
struct FoldArgs {
  const uint16_t* W;  // bf16 [N][K] original weights
  float* V;           // fp32 [N][K], updated in place
  float* alpha;       // fp32 [N][G], updated in place
  float* beta;        // fp32 [N][G], updated in place
  const float* s;     // fp32 [N][G] from the QDQ of this step
  const float* zp;
  const float* mx;
  const float* mn;
  float* dV_out;      // optional gradient outputs
  float* da_out;
  float* db_out;
  int group_size, bits, symmetric;
  float lr, v_min, v_max, c_min, c_max;
};

// Y[M][N] fp32 = X[M][K] * W[N][K]^T (both K-major bf16).
cudaError_t launch_gemm_store(const uint16_t* X, const uint16_t* W, float* Y, int M, int N, int K,
                              cudaStream_t stream);

// Forward of the tuning step with the residual epilogue:
//   R = X W_hat^T - Y, G = bf16(R * gscale), partial[tile*4+warp] = sum R^2 (fp64).
// With Yadd (fp32 [M][N]), R = (X W_hat^T + Yadd) - Y.
cudaError_t launch_gemm_resid(const uint16_t* X, const uint16_t* W_hat, const float* Y, uint16_t* G, float gscale,
                              double* loss_partial, int M, int N, int K, cudaStream_t stream,
                              const float* Yadd = nullptr);
int resid_partials(int M, int N);

// Backward of the tuning step: dW_hat = G^T X (reduction over the M tokens),
// folded through the straight-through estimator and applied as a SignSGD step.
// ldg, ldx: row strides of G and X when they are column slices of wider matrices (0: dense).
// Standalone fold + SignSGD from a materialised dL/dW_hat (fp32 [N][K]) (ar_fold.cu),
// group sizes 32, 64, 128, 256; used for short token counts instead of the
// weight-gradient GEMM's fold epilogue.  With W_hat_next it also writes the next
// step's QDQ (W_hat_next bf16, and the new scale / zero-point into fa.s, fa.zp).
bool fold_int_supported(int group_size);
// The linear step's choice: the split fold below kFoldSplitTokens tokens for g <= 128.
bool use_split_fold(int64_t M, int group_size);
cudaError_t launch_fold_int(const float* dW, const FoldArgs& fa, int64_t N, int64_t K, uint16_t* W_hat_next,
                            cudaStream_t stream);
// Below this many tokens a linear layer's step writes dL/dW_hat and folds in a
// separate kernel (the fold epilogue would pace the weight-gradient GEMM).
constexpr int64_t kFoldSplitTokens = 8192;
cudaError_t launch_gemm_fold(const uint16_t* G, const uint16_t* X, const FoldArgs& fa, int M, int N, int K,
                             cudaStream_t stream, int64_t ldg = 0, int64_t ldx = 0);

// SwiGLU forward of X[M][Hd] with gate/up weights [F][Hd]: a, b, h [M][F]
// bf16 (a, b nullable).
cudaError_t launch_gemm_swiglu_fwd(const uint16_t* X, const uint16_t* Wg, const uint16_t* Wu, uint16_t* A_out,
                                   uint16_t* B_out, uint16_t* H_out, int M, int F, int Hd, cudaStream_t stream);

// dH = G[M][Hd] W_down[Hd][F] with the SiLU backward epilogue -> dA, dB [M][F] bf16
// (rows ld_grad elements apart; 0: F).
cudaError_t launch_gemm_swiglu_bwd(const uint16_t* G, const uint16_t* Wd_hat, const uint16_t* A_in,
                                   const uint16_t* B_in, uint16_t* dA, uint16_t* dB, int M, int F, int Hd,
                                   cudaStream_t stream, int ld_grad = 0);

// ---- decoder block (ar_gemm.cu epilogues, ar_decoder.cu kernels) ----
// out [M][3H] bf16 = X [M][H] Wqkv [3H][H]^T, the Q and K columns (the first 2H)
// rotated by the position (row % L) angles of rope_cs ((cos, sin) [L][head_dim/2]).
cudaError_t launch_gemm_qkv(const uint16_t* X, const uint16_t* Wqkv, uint16_t* out, const float* rope_cs, int M,
                            int H, int L, int head_dim, cudaStream_t stream);
// out [M][N] fp32 = residual (bf16 res [M][N], else fp32 res_f32) + A [M][K] W [N][K]^T
cudaError_t launch_gemm_resadd(const uint16_t* A, const uint16_t* W, const uint16_t* res, const float* res_f32,
                               float* out, int M, int N, int K, cudaStream_t stream);
// out [M][N] bf16 = A [M][K] B, B stored [K][N]
cudaError_t launch_gemm_store_bf16_kmn(const uint16_t* A, const uint16_t* B_kn, uint16_t* out, int M, int N, int K,
                                       cudaStream_t stream);
// causal attention per sample and head over qkv [S*L][3H] (Q, K rotated; V): O [S*L][H] bf16, lse [S][nh][L]
cudaError_t launch_attn_fwd(const uint16_t* qkv, int S, int L, int H, int head_dim, uint16_t* out, float* lse,
                            cudaStream_t st);
// the same on tcgen05 for head dimension 128 and L % 128 == 0 (cudaErrorNotSupported otherwise)
cudaError_t launch_attn_fwd_tc(const uint16_t* qkv, int S, int L, int H, uint16_t* out, float* lse, cudaStream_t st);
// the dQ, dK, dV kernels on tcgen05 for head dimension 128 and L % 128 == 0, Dsum already = rowsum(dO O)
cudaError_t launch_attn_bwd_tc(const uint16_t* qkv, const uint16_t* dO, const float* lse, const float* Dsum,
                               const float* rope_cs, int S, int L, int H, uint16_t* dqkv, cudaStream_t st);
// its backward from dO: dqkv [S*L][3H] bf16 (dQ, dK with the inverse rotation applied; dV); Dsum [S][nh][L] scratch
cudaError_t launch_attn_bwd(const uint16_t* qkv, const uint16_t* O, const uint16_t* dO, const float* lse,
                            float* Dsum, const float* rope_cs, int S, int L, int H, int head_dim, uint16_t* dqkv,
                            cudaStream_t st);
// r [M][H] bf16 = x inv gamma, inv [M] = 1/sqrt(mean(x^2) + 1e-6) (x bf16 or fp32)
cudaError_t launch_rmsnorm_fwd(const void* x, bool x_f32, const float* gamma, int64_t M, int H, uint16_t* r,
                               float* inv, cudaStream_t st);
// dx [M][H] bf16 = G + RMSNorm backward of dr (fp32) at x (fp32) with inv, gamma
cudaError_t launch_rmsnorm_bwd(const float* x, const float* inv, const float* gamma, const float* dr,
                               const uint16_t* G, int64_t M, int H, uint16_t* dx, cudaStream_t st);
// (cos, sin) [L][head_dim/2] fp32 of t 10000^(-2i/head_dim)
cudaError_t launch_rope_table(int L, int head_dim, float* cs, cudaStream_t st);

// Plain D[M][N] fp32 = op(A) op(B)^T, with A given K-major ([M][K]) or
// MN-major ([K][M]) and B given K-major ([N][K]) or MN-major ([K][N]).
cudaError_t launch_gemm_plain(const uint16_t* A, bool a_mn, const uint16_t* B, bool b_mn, float* D, int M, int N,
                              int K, cudaStream_t stream);

// Fixed-order reduction of the loss partials, `n` per step for `steps` steps:
// loss[i] = sum(partials[i*n .. i*n+n)) * inv_count.
cudaError_t launch_loss_reduce(const double* partials, int n, int steps, double inv_count, float* loss,
                               cudaStream_t stream);

// Diagnostic wait that is bound to time out (see ar_debug_wait_timeout).
cudaError_t launch_wait_timeout(uint64_t limit_ns, int* gave_up, cudaStream_t stream);

// Synchronizes `stream`, copies the sticky device status to *out and clears it.
cudaError_t read_and_clear_status(unsigned int* out, cudaStream_t stream);

// ---- W4A16 (ar_w4a16.cu) ----
cudaError_t launch_w4a16(const uint16_t* A, int T, const uint32_t* packed, const uint16_t* scale16,
                         const uint16_t* zero16, int N, int K, int group_size, uint16_t* out, cudaStream_t stream);
// decode kernel over per-SM row ranges (ar_w4a16_dec.cu); cudaErrorNotSupported
// (nothing launched) for shapes whose scale/zero rows are not 16-byte multiples
cudaError_t launch_w4a16_dec(const uint16_t* A, int T, const uint32_t* packed, const uint16_t* scale16,
                             const uint16_t* zero16, int N, int K, int group_size, uint16_t* out,
                             cudaStream_t stream);
// the same kernel on 2-bit codes (ar_pack_codes' layout): T <= 8 and g >= 64,
// else cudaErrorNotSupported (nothing launched)
cudaError_t launch_w2a16_dec(const uint16_t* A, int T, const uint32_t* packed, const uint16_t* scale16,
                             const uint16_t* zero16, int N, int K, int group_size, uint16_t* out,
                             cudaStream_t stream);
// ... and on 8-bit codes (each code split into nibbles): T <= 8, else cudaErrorNotSupported
cudaError_t launch_w8a16_dec(const uint16_t* A, int T, const uint32_t* packed, const uint16_t* scale16,
                             const uint16_t* zero16, int N, int K, int group_size, uint16_t* out,
                             cudaStream_t stream);
// ... and on 3-bit codes (ar_pack_codes' 32-codes-in-3-words stream): T <= 8, g >= 64, K >= 512
cudaError_t launch_w3a16_dec(const uint16_t* A, int T, const uint32_t* packed, const uint16_t* scale16,
                             const uint16_t* zero16, int N, int K, int group_size, uint16_t* out,
                             cudaStream_t stream);
// NVFP4 QDQ (ar_nvfp4.cu): absmax into a zeroed device scalar, then the block QDQ
cudaError_t launch_absmax_bf16(const uint16_t* x, int64_t n, float* amax, cudaStream_t stream);
cudaError_t launch_qdq_nvfp4(const uint16_t* W, const float* V, const float* alpha, int64_t n, const float* amax,
                             uint16_t* W_hat, uint8_t* codes, uint8_t* scales, float* global_scale,
                             cudaStream_t stream);
// ... and the straight-through fold + SignSGD update of one NVFP4 tuning step from dL/dW_hat
cudaError_t launch_fold_nvfp4(const float* dW, const uint16_t* W, float* V, float* alpha, int64_t n, const float* amax,
                              float lr, float v_min, float v_max, float c_min, float c_max, float* dV_out,
                              float* da_out, cudaStream_t stream);
// minibatch assembly (ar_gather.cu): n <= kMaxGatherSamples samples of sample_bytes each
constexpr int kMaxGatherSamples = 64;
cudaError_t launch_gather_samples(const void* src, int64_t sample_bytes, const int32_t* idx, int n, void* dst,
                                  cudaStream_t stream);
// T > 16: tcgen05 dequant GEMM (ar_w4a16_tc.cu)
cudaError_t launch_w4a16_tc(const uint16_t* A, int T, const uint32_t* packed, const uint16_t* scale16,
                            const uint16_t* zero16, int N, int K, int group_size, uint16_t* out, cudaStream_t stream);
// 2, 3 or 8-bit codes (ar_wbx_dec.cu): mma.sync decode kernel, 16 tokens at a time
cudaError_t launch_wbx_dec(const uint16_t* A, int T, const uint32_t* packed, const uint16_t* scale16,
                           const uint16_t* zero16, int N, int K, int group_size, int bits, uint16_t* out,
                           cudaStream_t stream);
// NVFP4 weights (E2M1 codes uint8 [N][K/2], E4M3 block scales uint8 [N][K/16],
// device per-tensor scale), any T: the same tcgen05 GEMM (ar_w4a16_tc.cu)
cudaError_t launch_nvfp4_tc(const uint16_t* A, int T, const uint8_t* codes, const uint8_t* scales, const float* gscale,
                            int N, int K, uint16_t* out, cudaStream_t stream);
// 2, 4 or 8-bit codes (32/bits per uint32), any T: the same tcgen05 GEMM
cudaError_t launch_wxa16_tc(const uint16_t* A, int T, const uint32_t* packed, const uint16_t* scale16,
                            const uint16_t* zero16, int N, int K, int group_size, int bits, uint16_t* out,
                            cudaStream_t stream);

}  // namespace ar
