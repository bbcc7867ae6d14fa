// C ABI of libautoround.so (declared in include/autoround.h): argument
// validation, workspace layout and the launch sequence of each entry point.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "../../include/autoround.h"
#include "ar_internal.h"

namespace ar {

namespace {
thread_local std::string t_error;
thread_local std::string t_kernels;
thread_local std::string t_kernels_last;

ar_status fail(ar_status code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_error = buf;
  return code;
}

ar_status cuda_fail(cudaError_t e, const char* what) {
  return fail(AR_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

void begin_call() {
  t_error.clear();
  t_kernels.clear();
}

ar_status end_call() {
  t_kernels_last = t_kernels;
  return AR_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

ar_status check_cfg(const ar_qconfig* cfg) {
  if (!cfg) return fail(AR_ERR_INVALID_ARG, "cfg is NULL");
  if (cfg->bits < 2 || cfg->bits > 8) return fail(AR_ERR_UNSUPPORTED, "bits=%d outside 2..8", cfg->bits);
  if (cfg->symmetric != 0 && cfg->symmetric != 1) return fail(AR_ERR_INVALID_ARG, "symmetric must be 0 or 1");
  if (!(cfg->lr >= 0.0f) || !(cfg->lr < 1e30f)) return fail(AR_ERR_INVALID_ARG, "lr must be finite and >= 0");
  if (!(cfg->v_min <= cfg->v_max) || !(cfg->clip_min <= cfg->clip_max))
    return fail(AR_ERR_INVALID_ARG, "bounds must satisfy min <= max");
  return AR_OK;
}

// Layout of the tuning workspace for one linear layer.
struct LinearWs {
  size_t what, g, s, zp, mx, mn, dw, partial, total;
  int partials_per_step;
  bool split_fold;  // dL/dW_hat materialised in dw and folded by the standalone kernel
};

LinearWs linear_ws(int64_t M, int64_t N, int64_t K, int g, int n_steps) {
  LinearWs w{};
  const int64_t groups = N * (K / g);
  size_t off = 0;
  w.what = off;
  off = align_up(off + static_cast<size_t>(N * K) * 2, 256);
  w.g = off;
  off = align_up(off + static_cast<size_t>(M * N) * 2, 256);
  w.s = off;
  off = align_up(off + static_cast<size_t>(groups) * 4, 256);
  w.zp = off;
  off = align_up(off + static_cast<size_t>(groups) * 4, 256);
  w.mx = off;
  off = align_up(off + static_cast<size_t>(groups) * 4, 256);
  w.mn = off;
  off = align_up(off + static_cast<size_t>(groups) * 4, 256);
  w.split_fold = use_split_fold(M, g);
  w.dw = off;
  if (w.split_fold) off = align_up(off + static_cast<size_t>(N * K) * 4, 256);
  w.partials_per_step = resid_partials(static_cast<int>(M), static_cast<int>(N));
  w.partial = off;
  off = align_up(off + static_cast<size_t>(w.partials_per_step) * (n_steps > 0 ? n_steps : 1) * 8, 256);
  w.total = off;
  return w;
}

ar_status check_linear(const ar_layer* layers, int n_layers, int64_t M, const ar_qconfig* cfg, bool for_tune) {
  ar_status st = check_cfg(cfg);
  if (st != AR_OK) return st;
  if (!layers || n_layers != 1) return fail(AR_ERR_UNSUPPORTED, "AR_BLOCK_LINEAR needs exactly one layer");
  const ar_layer& L = layers[0];
  if (L.N <= 0 || L.K <= 0 || M <= 0) return fail(AR_ERR_INVALID_ARG, "sizes must be positive (M=%lld N=%lld K=%lld)",
                                                  (long long)M, (long long)L.N, (long long)L.K);
  const int g = cfg->group_size;
  if (for_tune && g != 32 && g != 64 && g != 128 && g != 256)
    return fail(AR_ERR_UNSUPPORTED, "ar_tune_step supports group_size 32, 64, 128, 256 (got %d)", g);
  if (L.K % g != 0) return fail(AR_ERR_INVALID_ARG, "K=%lld is not a multiple of group_size=%d", (long long)L.K, g);
  if (L.N % 8 != 0) return fail(AR_ERR_INVALID_ARG, "N=%lld must be a multiple of 8", (long long)L.N);
  if (M > INT32_MAX || L.N > INT32_MAX || L.K > INT32_MAX) return fail(AR_ERR_UNSUPPORTED, "dimension exceeds 2^31-1");
  if (!L.W || !L.V || !L.alpha || !L.beta) return fail(AR_ERR_INVALID_ARG, "layer pointer is NULL");
  if (!aligned16(L.W) || !aligned16(L.V) || !aligned16(L.alpha) || !aligned16(L.beta))
    return fail(AR_ERR_INVALID_ARG, "layer pointers must be 16-byte aligned");
  return AR_OK;
}


// Layout of the tuning workspace for a SwiGLU block (gate, up: [F][H]; down: [H][F]).
struct MlpWs {
  size_t what[3], s[3], zp[3], mx[3], mn[3];
  size_t a, b, h, da, db, g, partial, total;
  int partials_per_step;
};

MlpWs mlp_ws(int64_t M, int64_t Hd, int64_t F, int g, int n_steps) {
  MlpWs w{};
  size_t off = 0;
  const int64_t NK = F * Hd;
  for (int i = 0; i < 3; ++i) {
    w.what[i] = off;
    off = align_up(off + static_cast<size_t>(NK) * 2, 256);
  }
  for (int i = 0; i < 3; ++i) {
    const int64_t groups = NK / g;
    size_t* dst[4] = {&w.s[i], &w.zp[i], &w.mx[i], &w.mn[i]};
    for (size_t* d : dst) {
      *d = off;
      off = align_up(off + static_cast<size_t>(groups) * 4, 256);
    }
  }
  size_t* acts[5] = {&w.a, &w.b, &w.h, &w.da, &w.db};
  for (size_t* d : acts) {
    *d = off;
    off = align_up(off + static_cast<size_t>(M * F) * 2, 256);
  }
  w.g = off;
  off = align_up(off + static_cast<size_t>(M * Hd) * 2, 256);
  w.partials_per_step = resid_partials(static_cast<int>(M), static_cast<int>(Hd));
  w.partial = off;
  off = align_up(off + static_cast<size_t>(w.partials_per_step) * (n_steps > 0 ? n_steps : 1) * 8, 256);
  w.total = off;
  return w;
}

// gate [F][H], up [F][H], down [H][F]; returns H and F.
ar_status check_mlp(const ar_layer* layers, int n_layers, int64_t M, const ar_qconfig* cfg, bool for_tune,
                    int64_t* Hd, int64_t* F) {
  if (!layers || n_layers != 3) return fail(AR_ERR_UNSUPPORTED, "AR_BLOCK_SWIGLU_MLP needs three layers (gate, up, down)");
  const ar_layer &lg = layers[0], &lu = layers[1], &ld = layers[2];
  if (lg.N <= 0 || lg.K <= 0 || M <= 0) return fail(AR_ERR_INVALID_ARG, "sizes must be positive");
  if (lu.N != lg.N || lu.K != lg.K || ld.N != lg.K || ld.K != lg.N)
    return fail(AR_ERR_INVALID_ARG, "SwiGLU shapes: gate and up [F][H], down [H][F]");
  *F = lg.N;
  *Hd = lg.K;
  if (cfg) {
    ar_status st = check_cfg(cfg);
    if (st != AR_OK) return st;
    const int g = cfg->group_size;
    if (for_tune && g != 32 && g != 64 && g != 128 && g != 256)
      return fail(AR_ERR_UNSUPPORTED, "ar_tune_step supports group_size 32, 64, 128, 256 (got %d)", g);
    if (*Hd % g != 0 || *F % g != 0) return fail(AR_ERR_INVALID_ARG, "H and F must be multiples of group_size");
  }
  if (*Hd % 8 != 0 || *F % 8 != 0) return fail(AR_ERR_INVALID_ARG, "H and F must be multiples of 8");
  if (M > INT32_MAX || *Hd > INT32_MAX || *F > INT32_MAX) return fail(AR_ERR_UNSUPPORTED, "dimension exceeds 2^31-1");
  for (int i = 0; i < 3; ++i) {
    const ar_layer& L = layers[i];
    if (!L.W || (for_tune && (!L.V || !L.alpha || !L.beta))) return fail(AR_ERR_INVALID_ARG, "layer pointer is NULL");
    if (!aligned16(L.W) || (for_tune && (!aligned16(L.V) || !aligned16(L.alpha) || !aligned16(L.beta))))
      return fail(AR_ERR_INVALID_ARG, "layer pointers must be 16-byte aligned");
  }
  return AR_OK;
}

FoldArgs fold_args(const ar_layer& L, const ar_qconfig* cfg, float* sc, float* zp, float* mx, float* mn,
                   const ar_grads* gr) {
  FoldArgs fa{};
  fa.W = L.W;
  fa.V = L.V;
  fa.alpha = L.alpha;
  fa.beta = L.beta;
  fa.s = sc;
  fa.zp = zp;
  fa.mx = mx;
  fa.mn = mn;
  fa.dV_out = gr ? gr->dV : nullptr;
  fa.da_out = gr ? gr->dalpha : nullptr;
  fa.db_out = gr ? gr->dbeta : nullptr;
  fa.group_size = cfg->group_size;
  fa.bits = cfg->bits;
  fa.symmetric = cfg->symmetric;
  fa.lr = cfg->lr;
  fa.v_min = cfg->v_min;
  fa.v_max = cfg->v_max;
  fa.c_min = cfg->clip_min;
  fa.c_max = cfg->clip_max;
  return fa;
}

ar_status tune_mlp(const ar_layer* L, const uint16_t* X, int64_t M, const float* Y, const ar_qconfig* cfg,
                   int n_steps, float* loss_per_step, const ar_grads* grads, void* workspace,
                   size_t workspace_bytes, cudaStream_t s) {
  int64_t Hd = 0, F = 0;
  ar_status st = check_mlp(L, 3, M, cfg, true, &Hd, &F);
  if (st != AR_OK) return st;
  const MlpWs w = mlp_ws(M, Hd, F, cfg->group_size, n_steps);
  if (!workspace || workspace_bytes < w.total)
    return fail(AR_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", w.total, workspace_bytes);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return fail(AR_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (grads) {
    for (int i = 0; i < 3; ++i) {
      const void* gp[] = {grads[i].dV, grads[i].dalpha, grads[i].dbeta};
      for (const void* p : gp)
        if (p && !aligned16(p)) return fail(AR_ERR_INVALID_ARG, "gradient outputs must be 16-byte aligned");
    }
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  auto bf = [&](size_t off) { return reinterpret_cast<uint16_t*>(ws + off); };
  auto f32p = [&](size_t off) { return reinterpret_cast<float*>(ws + off); };
  const int Mi = static_cast<int>(M), Hi = static_cast<int>(Hd), Fi = static_cast<int>(F);
  const float gscale = static_cast<float>(2.0 / (static_cast<double>(M) * static_cast<double>(Hd)));
  double* partial = reinterpret_cast<double*>(ws + w.partial);
  const int steps = n_steps > 0 ? n_steps : 1;
  cudaError_t e;
  for (int step = 0; step < steps; ++step) {
    for (int i = 0; i < 3; ++i) {
      e = launch_qdq(L[i].W, L[i].V, L[i].alpha, L[i].beta, L[i].N, L[i].K, cfg->group_size, cfg->bits,
                     cfg->symmetric, bf(w.what[i]), nullptr, f32p(w.s[i]), f32p(w.zp[i]), f32p(w.mx[i]),
                     f32p(w.mn[i]), s);
      if (e != cudaSuccess) return cuda_fail(e, "qdq launch");
    }
    e = launch_gemm_swiglu_fwd(X, bf(w.what[0]), bf(w.what[1]), bf(w.a), bf(w.b), bf(w.h), Mi, Fi, Hi, s);
    if (e != cudaSuccess) return cuda_fail(e, "SwiGLU forward GEMM launch");
    e = launch_gemm_resid(bf(w.h), bf(w.what[2]), Y, bf(w.g), gscale,
                          partial + static_cast<size_t>(step) * w.partials_per_step, Mi, Hi, Fi, s);
    if (e != cudaSuccess) return cuda_fail(e, "down-projection GEMM launch");
    if (n_steps == 0) break;
    const bool last = step == steps - 1;
    FoldArgs fd = fold_args(L[2], cfg, f32p(w.s[2]), f32p(w.zp[2]), f32p(w.mx[2]), f32p(w.mn[2]),
                            (last && grads) ? &grads[2] : nullptr);
    e = launch_gemm_fold(bf(w.g), bf(w.h), fd, Mi, Hi, Fi, s);
    if (e != cudaSuccess) return cuda_fail(e, "down weight-gradient GEMM launch");
    e = launch_gemm_swiglu_bwd(bf(w.g), bf(w.what[2]), bf(w.a), bf(w.b), bf(w.da), bf(w.db), Mi, Fi, Hi, s);
    if (e != cudaSuccess) return cuda_fail(e, "SwiGLU backward GEMM launch");
    FoldArgs fg = fold_args(L[0], cfg, f32p(w.s[0]), f32p(w.zp[0]), f32p(w.mx[0]), f32p(w.mn[0]),
                            (last && grads) ? &grads[0] : nullptr);
    e = launch_gemm_fold(bf(w.da), X, fg, Mi, Fi, Hi, s);
    if (e != cudaSuccess) return cuda_fail(e, "gate weight-gradient GEMM launch");
    FoldArgs fu = fold_args(L[1], cfg, f32p(w.s[1]), f32p(w.zp[1]), f32p(w.mx[1]), f32p(w.mn[1]),
                            (last && grads) ? &grads[1] : nullptr);
    e = launch_gemm_fold(bf(w.db), X, fu, Mi, Fi, Hi, s);
    if (e != cudaSuccess) return cuda_fail(e, "up weight-gradient GEMM launch");
  }
  e = launch_loss_reduce(partial, w.partials_per_step, steps,
                         1.0 / (static_cast<double>(M) * static_cast<double>(Hd)), loss_per_step, s);
  if (e != cudaSuccess) return cuda_fail(e, "loss reduction launch");
  return end_call();
}

// n_steps tuning steps of one linear layer (or of a shard of its output rows:
// n_total > 0 is the whole layer's row count, which sets the loss normaliser).
ar_status tune_linear(const ar_layer* layers, int n_layers, const uint16_t* X, int64_t M, const float* Y,
                      const ar_qconfig* cfg, int n_steps, float* loss_per_step, const ar_grads* grads,
                      void* workspace, size_t workspace_bytes, int64_t n_total, cudaStream_t s) {
  ar_status st = check_linear(layers, n_layers, M, cfg, true);
  if (st != AR_OK) return st;
  if (n_steps < 0) return fail(AR_ERR_INVALID_ARG, "n_steps must be >= 0");
  if (!X || !Y || !loss_per_step) return fail(AR_ERR_INVALID_ARG, "X, Y and loss_per_step are required");
  if (!aligned16(X) || !aligned16(Y)) return fail(AR_ERR_INVALID_ARG, "X and Y must be 16-byte aligned");
  const ar_layer& L = layers[0];
  const LinearWs w = linear_ws(M, L.N, L.K, cfg->group_size, n_steps);
  if (!workspace || workspace_bytes < w.total)
    return fail(AR_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", w.total, workspace_bytes);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return fail(AR_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (grads) {
    const void* gp[] = {grads->dV, grads->dalpha, grads->dbeta};
    for (const void* p : gp)
      if (p && !aligned16(p)) return fail(AR_ERR_INVALID_ARG, "gradient outputs must be 16-byte aligned");
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint16_t* W_hat = reinterpret_cast<uint16_t*>(ws + w.what);
  uint16_t* G = reinterpret_cast<uint16_t*>(ws + w.g);
  float* sc = reinterpret_cast<float*>(ws + w.s);
  float* zp = reinterpret_cast<float*>(ws + w.zp);
  float* mx = reinterpret_cast<float*>(ws + w.mx);
  float* mn = reinterpret_cast<float*>(ws + w.mn);
  double* partial = reinterpret_cast<double*>(ws + w.partial);
  const int Mi = static_cast<int>(M), Ni = static_cast<int>(L.N), Ki = static_cast<int>(L.K);
  // loss normaliser M * N_total: the whole layer's output count (N_total = N unless this is a row shard)
  const double count = static_cast<double>(M) * static_cast<double>(n_total > 0 ? n_total : L.N);
  const float gscale = static_cast<float>(2.0 / count);
  const int steps = n_steps > 0 ? n_steps : 1;
  cudaError_t e;
  for (int step = 0; step < steps; ++step) {
    // on the split-fold path the previous step's fold kernel already took this step's QDQ
    if (step == 0 || !w.split_fold) {
      e = launch_qdq(L.W, L.V, L.alpha, L.beta, L.N, L.K, cfg->group_size, cfg->bits, cfg->symmetric, W_hat, nullptr,
                     sc, zp, mx, mn, s);
      if (e != cudaSuccess) return cuda_fail(e, "qdq launch");
    }
    e = launch_gemm_resid(X, W_hat, Y, G, gscale, partial + static_cast<size_t>(step) * w.partials_per_step, Mi, Ni,
                          Ki, s);
    if (e != cudaSuccess) return cuda_fail(e, "forward GEMM launch");
    if (n_steps == 0) break;
    const bool last = step == steps - 1;
    const FoldArgs fa = fold_args(L, cfg, sc, zp, mx, mn, (last && grads) ? grads : nullptr);
    if (w.split_fold) {
      // short token reduction: dL/dW_hat = G^T X to the workspace, then the fold at full occupancy
      float* dW = reinterpret_cast<float*>(ws + w.dw);
      e = launch_gemm_plain(G, true, X, true, dW, Ni, Ki, Mi, s);
      if (e != cudaSuccess) return cuda_fail(e, "weight-gradient GEMM launch");
      e = launch_fold_int(dW, fa, L.N, L.K, last ? nullptr : W_hat, s);
      if (e != cudaSuccess) return cuda_fail(e, "fold launch");
    } else {
      e = launch_gemm_fold(G, X, fa, Mi, Ni, Ki, s);
      if (e != cudaSuccess) return cuda_fail(e, "weight-gradient GEMM launch");
    }
  }
  e = launch_loss_reduce(partial, w.partials_per_step, steps, 1.0 / count, loss_per_step, s);
  if (e != cudaSuccess) return cuda_fail(e, "loss reduction launch");
  return end_call();
}

// ---- decoder block ----------------------------------------------------------
// Workspace of the decoder block (H hidden, F intermediate, M tokens, L per sample).
struct DecWs {
  size_t wqkv, wo, wgu, wd;             // bf16 fake-quantized (or original) weights, stacked where one GEMM reads them
  size_t sc[7], zp[7], mx[7], mn[7];    // per-layer group parameters
  size_t rope, r1, qkv, o, lse, x2, inv2, r2, a, b, h, g, dab, dr2, dx2, dout, dsum, dqkv, partial, total;
  int partials_per_step;
};

constexpr int kDecLayers = 7;  // q, k, v, o, gate, up, down

DecWs dec_ws(int64_t M, int64_t H, int64_t F, int64_t L, int head_dim, int g, int n_steps, bool tune) {
  DecWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, 256);
    return at;
  };
  w.wqkv = take(static_cast<size_t>(3 * H * H) * 2);
  w.wo = take(static_cast<size_t>(H * H) * 2);
  w.wgu = take(static_cast<size_t>(2 * F * H) * 2);
  w.wd = take(static_cast<size_t>(H * F) * 2);
  if (tune) {
    const int64_t NK[kDecLayers] = {H * H, H * H, H * H, H * H, F * H, F * H, H * F};
    for (int i = 0; i < kDecLayers; ++i) {
      const size_t groups = static_cast<size_t>(NK[i] / g) * 4;
      w.sc[i] = take(groups);
      w.zp[i] = take(groups);
      w.mx[i] = take(groups);
      w.mn[i] = take(groups);
    }
  }
  const size_t MH = static_cast<size_t>(M * H), MF = static_cast<size_t>(M * F);
  const size_t rows = static_cast<size_t>(M / L) * static_cast<size_t>(H / head_dim) * static_cast<size_t>(L);
  w.rope = take(static_cast<size_t>(L) * head_dim / 2 * 8);
  w.r1 = take(MH * 2);
  w.qkv = take(3 * MH * 2);
  w.o = take(MH * 2);
  w.lse = take(rows * 4);
  w.x2 = take(MH * 4);
  w.inv2 = take(static_cast<size_t>(M) * 4);
  w.r2 = take(MH * 2);
  w.a = take(MF * 2);
  w.b = take(MF * 2);
  w.h = take(MF * 2);
  if (tune) {
    w.g = take(MH * 2);
    w.dab = take(2 * MF * 2);
    w.dr2 = take(MH * 4);
    w.dx2 = take(MH * 2);
    w.dout = take(MH * 2);
    w.dsum = take(rows * 4);
    w.dqkv = take(3 * MH * 2);
    w.partials_per_step = resid_partials(static_cast<int>(M), static_cast<int>(H));
    w.partial = take(static_cast<size_t>(w.partials_per_step) * (n_steps > 0 ? n_steps : 1) * 8);
  }
  w.total = off;
  return w;
}

ar_status check_decoder(const ar_decoder_cfg* d, const ar_layer* L, int64_t M, const ar_qconfig* cfg, bool tune) {
  if (!d) return fail(AR_ERR_INVALID_ARG, "decoder config is NULL");
  const int64_t H = d->hidden, F = d->intermediate, Ls = d->seq_len;
  if (H <= 0 || F <= 0 || Ls <= 0 || M <= 0 || d->n_heads <= 0)
    return fail(AR_ERR_INVALID_ARG, "sizes must be positive");
  if (H % d->n_heads != 0) return fail(AR_ERR_INVALID_ARG, "H=%lld is not a multiple of n_heads", (long long)H);
  const int64_t hd = H / d->n_heads;
  if (hd != 64 && hd != 128) return fail(AR_ERR_UNSUPPORTED, "head dim %lld: needs 64 or 128", (long long)hd);
  if (H % 128 != 0 || F % 8 != 0) return fail(AR_ERR_INVALID_ARG, "H must be a multiple of 128 and F of 8");
  if (Ls % 64 != 0 || M % Ls != 0) return fail(AR_ERR_INVALID_ARG, "seq_len must be a multiple of 64 dividing M");
  if (3 * H * M > INT32_MAX * 8ll || 3 * H > INT32_MAX || M > INT32_MAX || F > INT32_MAX)
    return fail(AR_ERR_UNSUPPORTED, "dimension exceeds 2^31-1");
  if (!d->gamma1 || !d->gamma2 || !aligned16(d->gamma1) || !aligned16(d->gamma2))
    return fail(AR_ERR_INVALID_ARG, "gamma1, gamma2 must be 16-byte aligned device pointers");
  if (!L) return fail(AR_ERR_INVALID_ARG, "layers is NULL");
  const int64_t shp[kDecLayers][2] = {{H, H}, {H, H}, {H, H}, {H, H}, {F, H}, {F, H}, {H, F}};
  for (int i = 0; i < kDecLayers; ++i) {
    if (L[i].N != shp[i][0] || L[i].K != shp[i][1])
      return fail(AR_ERR_INVALID_ARG, "layer %d: shape [%lld][%lld], expected [%lld][%lld] (q, k, v, o, gate, up, down)",
                  i, (long long)L[i].N, (long long)L[i].K, (long long)shp[i][0], (long long)shp[i][1]);
    if (!L[i].W || !aligned16(L[i].W)) return fail(AR_ERR_INVALID_ARG, "layer %d: W must be 16-byte aligned", i);
    if (tune && (!L[i].V || !L[i].alpha || !L[i].beta || !aligned16(L[i].V) || !aligned16(L[i].alpha) ||
                 !aligned16(L[i].beta)))
      return fail(AR_ERR_INVALID_ARG, "layer %d: V, alpha, beta must be 16-byte aligned", i);
  }
  if (tune) {
    ar_status st = check_cfg(cfg);
    if (st != AR_OK) return st;
    const int g = cfg->group_size;
    if (g != 32 && g != 64 && g != 128 && g != 256)
      return fail(AR_ERR_UNSUPPORTED, "group_size %d: needs 32, 64, 128 or 256", g);
    if (H % g != 0 || F % g != 0) return fail(AR_ERR_INVALID_ARG, "H and F must be multiples of group_size");
  }
  return AR_OK;
}

// The block forward from r1 on (the QKV, attention, residual, norm and MLP launches);
// with G != nullptr the last GEMM is the loss epilogue, else Y = X2 + h Wd^T.
ar_status decoder_forward_launches(const ar_decoder_cfg* d, const DecWs& w, uint8_t* ws, const uint16_t* X, int64_t M,
                                   float* Y_out, const float* Y_ref, uint16_t* G, float gscale, double* partial,
                                   cudaStream_t s) {
  auto bf = [&](size_t off) { return reinterpret_cast<uint16_t*>(ws + off); };
  auto f32p = [&](size_t off) { return reinterpret_cast<float*>(ws + off); };
  const int Mi = static_cast<int>(M), Hi = static_cast<int>(d->hidden), Fi = static_cast<int>(d->intermediate);
  const int Li = static_cast<int>(d->seq_len), hd = static_cast<int>(d->hidden / d->n_heads);
  const int S = Mi / Li;
  cudaError_t e = launch_gemm_qkv(bf(w.r1), bf(w.wqkv), bf(w.qkv), f32p(w.rope), Mi, Hi, Li, hd, s);
  if (e != cudaSuccess) return cuda_fail(e, "QKV GEMM launch");
  e = launch_attn_fwd(bf(w.qkv), S, Li, Hi, hd, bf(w.o), f32p(w.lse), s);
  if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  e = launch_gemm_resadd(bf(w.o), bf(w.wo), X, nullptr, f32p(w.x2), Mi, Hi, Hi, s);
  if (e != cudaSuccess) return cuda_fail(e, "output projection GEMM launch");
  e = launch_rmsnorm_fwd(f32p(w.x2), true, d->gamma2, M, Hi, bf(w.r2), f32p(w.inv2), s);
  if (e != cudaSuccess) return cuda_fail(e, "rmsnorm launch");
  e = launch_gemm_swiglu_fwd(bf(w.r2), bf(w.wgu), bf(w.wgu) + static_cast<size_t>(Fi) * Hi, bf(w.a), bf(w.b),
                             bf(w.h), Mi, Fi, Hi, s);
  if (e != cudaSuccess) return cuda_fail(e, "SwiGLU forward GEMM launch");
  if (G) e = launch_gemm_resid(bf(w.h), bf(w.wd), Y_ref, G, gscale, partial, Mi, Hi, Fi, s, f32p(w.x2));
  else e = launch_gemm_resadd(bf(w.h), bf(w.wd), nullptr, f32p(w.x2), Y_out, Mi, Hi, Fi, s);
  if (e != cudaSuccess) return cuda_fail(e, "down-projection GEMM launch");
  return AR_OK;
}

ar_status decoder_tune(const ar_decoder_cfg* d, const ar_layer* L, const uint16_t* X, int64_t M, const float* Y,
                       const ar_qconfig* cfg, int n_steps, float* loss_per_step, const ar_grads* grads,
                       void* workspace, size_t workspace_bytes, cudaStream_t s) {
  ar_status st = check_decoder(d, L, M, cfg, true);
  if (st != AR_OK) return st;
  if (n_steps < 0) return fail(AR_ERR_INVALID_ARG, "n_steps must be >= 0");
  if (!X || !Y || !loss_per_step || !aligned16(X) || !aligned16(Y))
    return fail(AR_ERR_INVALID_ARG, "X, Y (16-byte aligned) and loss_per_step are required");
  const int64_t H = d->hidden, F = d->intermediate;
  const int hd = static_cast<int>(H / d->n_heads);
  const DecWs w = dec_ws(M, H, F, d->seq_len, hd, cfg->group_size, n_steps, true);
  if (!workspace || workspace_bytes < w.total)
    return fail(AR_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", w.total, workspace_bytes);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return fail(AR_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (grads) {
    for (int i = 0; i < kDecLayers; ++i) {
      const void* gp[] = {grads[i].dV, grads[i].dalpha, grads[i].dbeta};
      for (const void* p : gp)
        if (p && !aligned16(p)) return fail(AR_ERR_INVALID_ARG, "gradient outputs must be 16-byte aligned");
    }
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  auto bf = [&](size_t off) { return reinterpret_cast<uint16_t*>(ws + off); };
  auto f32p = [&](size_t off) { return reinterpret_cast<float*>(ws + off); };
  const int Mi = static_cast<int>(M), Hi = static_cast<int>(H), Fi = static_cast<int>(F);
  const int Li = static_cast<int>(d->seq_len), S = Mi / Li;
  // Where each layer's W_hat goes: q, k, v stacked, gate and up stacked.
  uint16_t* what[kDecLayers] = {bf(w.wqkv), bf(w.wqkv) + static_cast<size_t>(H) * H,
                                bf(w.wqkv) + 2 * static_cast<size_t>(H) * H, bf(w.wo), bf(w.wgu),
                                bf(w.wgu) + static_cast<size_t>(F) * H, bf(w.wd)};
  const double count = static_cast<double>(M) * static_cast<double>(H);
  const float gscale = static_cast<float>(2.0 / count);
  double* partial = reinterpret_cast<double*>(ws + w.partial);
  cudaError_t e = launch_rope_table(Li, hd, f32p(w.rope), s);
  if (e != cudaSuccess) return cuda_fail(e, "rope table launch");
  // r1 = rmsnorm(X) gamma1 does not depend on the tuned parameters: once per call
  e = launch_rmsnorm_fwd(X, false, d->gamma1, M, Hi, bf(w.r1), nullptr, s);
  if (e != cudaSuccess) return cuda_fail(e, "rmsnorm launch");
  const int steps = n_steps > 0 ? n_steps : 1;
  for (int step = 0; step < steps; ++step) {
    for (int i = 0; i < kDecLayers; ++i) {
      e = launch_qdq(L[i].W, L[i].V, L[i].alpha, L[i].beta, L[i].N, L[i].K, cfg->group_size, cfg->bits,
                     cfg->symmetric, what[i], nullptr, f32p(w.sc[i]), f32p(w.zp[i]), f32p(w.mx[i]), f32p(w.mn[i]), s);
      if (e != cudaSuccess) return cuda_fail(e, "qdq launch");
    }
    st = decoder_forward_launches(d, w, ws, X, M, nullptr, Y, bf(w.g), gscale,
                                  partial + static_cast<size_t>(step) * w.partials_per_step, s);
    if (st != AR_OK) return st;
    if (n_steps == 0) break;
    const bool last = step == steps - 1;
    auto fa = [&](int i) {
      return fold_args(L[i], cfg, f32p(w.sc[i]), f32p(w.zp[i]), f32p(w.mx[i]), f32p(w.mn[i]),
                       (last && grads) ? &grads[i] : nullptr);
    };
    // MLP: dWd = G^T h; dH = G Wd -> dA, dB (one [M][2F] buffer); dWg = dA^T r2, dWu = dB^T r2
    e = launch_gemm_fold(bf(w.g), bf(w.h), fa(6), Mi, Hi, Fi, s);
    if (e != cudaSuccess) return cuda_fail(e, "down weight-gradient GEMM launch");
    e = launch_gemm_swiglu_bwd(bf(w.g), bf(w.wd), bf(w.a), bf(w.b), bf(w.dab), bf(w.dab) + Fi, Mi, Fi, Hi, s, 2 * Fi);
    if (e != cudaSuccess) return cuda_fail(e, "SwiGLU backward GEMM launch");
    e = launch_gemm_fold(bf(w.dab), bf(w.r2), fa(4), Mi, Fi, Hi, s, 2 * F, 0);
    if (e != cudaSuccess) return cuda_fail(e, "gate weight-gradient GEMM launch");
    e = launch_gemm_fold(bf(w.dab) + Fi, bf(w.r2), fa(5), Mi, Fi, Hi, s, 2 * F, 0);
    if (e != cudaSuccess) return cuda_fail(e, "up weight-gradient GEMM launch");
    // dr2 = [dA | dB] [Wg ; Wu] (fp32), then the norm's backward plus the residual path: dX2 (bf16)
    e = launch_gemm_plain(bf(w.dab), false, bf(w.wgu), true, f32p(w.dr2), Mi, Hi, 2 * Fi, s);
    if (e != cudaSuccess) return cuda_fail(e, "norm-input gradient GEMM launch");
    e = launch_rmsnorm_bwd(f32p(w.x2), f32p(w.inv2), d->gamma2, f32p(w.dr2), bf(w.g), M, Hi, bf(w.dx2), s);
    if (e != cudaSuccess) return cuda_fail(e, "rmsnorm backward launch");
    // attention output projection: dWo = dX2^T O; dO = dX2 Wo
    e = launch_gemm_fold(bf(w.dx2), bf(w.o), fa(3), Mi, Hi, Hi, s);
    if (e != cudaSuccess) return cuda_fail(e, "o weight-gradient GEMM launch");
    e = launch_gemm_store_bf16_kmn(bf(w.dx2), bf(w.wo), bf(w.dout), Mi, Hi, Hi, s);
    if (e != cudaSuccess) return cuda_fail(e, "attention-output gradient GEMM launch");
    // attention backward -> dQ | dK | dV, then dWq, dWk, dWv = d(.)^T r1
    e = launch_attn_bwd(bf(w.qkv), bf(w.o), bf(w.dout), f32p(w.lse), f32p(w.dsum), f32p(w.rope), S, Li, Hi, hd,
                        bf(w.dqkv), s);
    if (e != cudaSuccess) return cuda_fail(e, "attention backward launch");
    for (int i = 0; i < 3; ++i) {
      e = launch_gemm_fold(bf(w.dqkv) + static_cast<size_t>(i) * Hi, bf(w.r1), fa(i), Mi, Hi, Hi, s, 3 * H, 0);
      if (e != cudaSuccess) return cuda_fail(e, "q/k/v weight-gradient GEMM launch");
    }
  }
  e = launch_loss_reduce(partial, w.partials_per_step, steps, 1.0 / count, loss_per_step, s);
  if (e != cudaSuccess) return cuda_fail(e, "loss reduction launch");
  return end_call();
}

ar_status decoder_reference(const ar_decoder_cfg* d, const ar_layer* L, const uint16_t* X, int64_t M, float* Y,
                            void* workspace, size_t workspace_bytes, cudaStream_t s) {
  ar_status st = check_decoder(d, L, M, nullptr, false);
  if (st != AR_OK) return st;
  if (!X || !Y || !aligned16(X) || !aligned16(Y)) return fail(AR_ERR_INVALID_ARG, "X, Y must be 16-byte aligned");
  const int64_t H = d->hidden, F = d->intermediate;
  const int hd = static_cast<int>(H / d->n_heads);
  const DecWs w = dec_ws(M, H, F, d->seq_len, hd, 32, 0, false);
  if (!workspace || workspace_bytes < w.total)
    return fail(AR_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", w.total, workspace_bytes);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return fail(AR_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t HH = static_cast<size_t>(H) * H * 2, FH = static_cast<size_t>(F) * H * 2;
  // the original weights, stacked where one GEMM reads them
  const struct {
    size_t dst;
    int layer;
    size_t bytes;
  } copies[] = {{w.wqkv, 0, HH}, {w.wqkv + HH, 1, HH}, {w.wqkv + 2 * HH, 2, HH}, {w.wo, 3, HH},
                {w.wgu, 4, FH},  {w.wgu + FH, 5, FH},  {w.wd, 6, FH}};
  for (const auto& c : copies) {
    cudaError_t e = cudaMemcpyAsync(ws + c.dst, L[c.layer].W, c.bytes, cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "weight copy");
  }
  cudaError_t e = launch_rope_table(static_cast<int>(d->seq_len), hd, reinterpret_cast<float*>(ws + w.rope), s);
  if (e != cudaSuccess) return cuda_fail(e, "rope table launch");
  e = launch_rmsnorm_fwd(X, false, d->gamma1, M, static_cast<int>(H), reinterpret_cast<uint16_t*>(ws + w.r1), nullptr, s);
  if (e != cudaSuccess) return cuda_fail(e, "rmsnorm launch");
  st = decoder_forward_launches(d, w, ws, X, M, Y, nullptr, nullptr, 0.f, nullptr, s);
  if (st != AR_OK) return st;
  return end_call();
}
}  // namespace

void set_last_error(const char* msg) { t_error = msg; }

void trace_kernel(const char* name) {
  if (!t_kernels.empty()) t_kernels += ";";
  t_kernels += name;
}

// ---- device-time profiler: events around every launch while enabled ----
namespace {
struct ProfRecord {
  const char* name;
  cudaEvent_t start, stop;
};
std::atomic<bool> g_prof_on{false};
std::mutex g_prof_mu;
std::vector<ProfRecord> g_prof_records;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t take_event() {
  cudaEvent_t e = nullptr;
  if (!g_event_pool.empty()) {
    e = g_event_pool.back();
    g_event_pool.pop_back();
  } else if (cudaEventCreate(&e) != cudaSuccess) {
    e = nullptr;
  }
  return e;
}
}  // namespace

// Every launch is also an NVTX range named after the kernel, so a timeline
// profiler shows which library kernel ran (a no-op without a profiler attached).
LaunchScope::LaunchScope(cudaStream_t stream, const char* name) : stream_(stream), name_(name), start_(nullptr) {
  nvtxRangePushA(name);
  if (g_prof_on.load(std::memory_order_relaxed)) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    start_ = take_event();
    if (start_) cudaEventRecord(start_, stream_);
  }
}

LaunchScope::~LaunchScope() {
  nvtxRangePop();
  trace_kernel(name_);
  if (start_) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    cudaEvent_t stop = take_event();
    if (stop) {
      cudaEventRecord(stop, stream_);
      g_prof_records.push_back({name_, start_, stop});
    } else {
      g_event_pool.push_back(start_);
    }
  }
}

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (cache[dev] == 0) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = v > 0 ? v : 1;
  }
  return cache[dev];
}

}  // namespace ar

using namespace ar;

extern "C" {

void ar_qconfig_default(ar_qconfig* cfg) {
  if (!cfg) return;
  cfg->bits = 4;
  cfg->group_size = 128;
  cfg->symmetric = 0;
  cfg->lr = 0.005f;
  cfg->iters = 200;
  cfg->v_min = -0.5f;
  cfg->v_max = 0.5f;
  cfg->clip_min = 0.5f;
  cfg->clip_max = 1.0f;
}

ar_status ar_f32_to_bf16(const float* src, uint16_t* dst, int64_t n, ar_stream_t stream) {
  begin_call();
  if (n < 0) return fail(AR_ERR_INVALID_ARG, "n must be >= 0");
  if (n == 0) return end_call();
  if (!src || !dst) return fail(AR_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(src) || !aligned16(dst)) return fail(AR_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  cudaError_t e = launch_f32_to_bf16(src, dst, n, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "f32_to_bf16 launch");
  return end_call();
}

ar_status ar_qdq(const uint16_t* W, const float* V, const float* alpha, const float* beta, int64_t N, int64_t K,
                 const ar_qconfig* cfg, uint16_t* W_hat, uint8_t* codes, float* scale, float* zero,
                 ar_stream_t stream) {
  begin_call();
  ar_status st = check_cfg(cfg);
  if (st != AR_OK) return st;
  const int g = cfg->group_size;
  if (!pow2(g) || g < 8 || g > 1024) return fail(AR_ERR_UNSUPPORTED, "group_size %d: ar_qdq needs a power of two in 8..1024", g);
  if (N <= 0 || K <= 0) return fail(AR_ERR_INVALID_ARG, "N, K must be positive");
  if (K % g != 0) return fail(AR_ERR_INVALID_ARG, "K=%lld is not a multiple of group_size=%d", (long long)K, g);
  if (!W || !V || !alpha || !beta) return fail(AR_ERR_INVALID_ARG, "NULL input pointer");
  if (!W_hat && !codes && !scale && !zero) return fail(AR_ERR_INVALID_ARG, "no output requested");
  const void* ptrs[] = {W, V, alpha, beta, W_hat, codes, scale, zero};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(AR_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  cudaError_t e = launch_qdq(W, V, alpha, beta, N, K, g, cfg->bits, cfg->symmetric, W_hat, codes, scale, zero,
                             nullptr, nullptr, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "qdq launch");
  return end_call();
}

ar_status ar_linear_forward(const uint16_t* X, int64_t M, const uint16_t* W, int64_t N, int64_t K, float* Y,
                            ar_stream_t stream) {
  begin_call();
  if (M <= 0 || N <= 0 || K <= 0) return fail(AR_ERR_INVALID_ARG, "sizes must be positive");
  if (N % 8 != 0 || K % 8 != 0) return fail(AR_ERR_INVALID_ARG, "N and K must be multiples of 8");
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return fail(AR_ERR_UNSUPPORTED, "dimension exceeds 2^31-1");
  if (!X || !W || !Y) return fail(AR_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(X) || !aligned16(W) || !aligned16(Y)) return fail(AR_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  cudaError_t e = launch_gemm_store(X, W, Y, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K),
                                    reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "reference forward launch");
  return end_call();
}

size_t ar_tune_step_workspace(int block_kind, const ar_layer* layers, int n_layers, int64_t M, const ar_qconfig* cfg,
                              int n_steps) {
  begin_call();
  if (block_kind == AR_BLOCK_SWIGLU_MLP) {
    int64_t Hd = 0, F = 0;
    if (n_steps < 0 || check_cfg(cfg) != AR_OK || check_mlp(layers, n_layers, M, nullptr, false, &Hd, &F) != AR_OK ||
        cfg->group_size <= 0 || Hd % cfg->group_size != 0 || F % cfg->group_size != 0) {
      if (t_error.empty()) fail(AR_ERR_INVALID_ARG, "invalid SwiGLU block");
      return 0;
    }
    return mlp_ws(M, Hd, F, cfg->group_size, n_steps).total;
  }
  if (block_kind != AR_BLOCK_LINEAR) {
    fail(AR_ERR_UNSUPPORTED, "block_kind %d not supported", block_kind);
    return 0;
  }
  if (n_steps < 0) {
    fail(AR_ERR_INVALID_ARG, "n_steps must be >= 0");
    return 0;
  }
  if (check_cfg(cfg) != AR_OK) return 0;
  if (!layers || n_layers != 1 || layers[0].N <= 0 || layers[0].K <= 0 || M <= 0 || cfg->group_size <= 0 ||
      layers[0].K % cfg->group_size != 0) {
    fail(AR_ERR_INVALID_ARG, "invalid layer shapes");
    return 0;
  }
  return linear_ws(M, layers[0].N, layers[0].K, cfg->group_size, n_steps).total;
}

ar_status ar_tune_step(int block_kind, const ar_layer* layers, int n_layers, const uint16_t* X, int64_t M,
                       const float* Y, const ar_qconfig* cfg, int n_steps, float* loss_per_step, const ar_grads* grads,
                       void* workspace, size_t workspace_bytes, ar_stream_t stream) {
  begin_call();
  if (block_kind == AR_BLOCK_SWIGLU_MLP) {
    if (n_steps < 0) return fail(AR_ERR_INVALID_ARG, "n_steps must be >= 0");
    if (!X || !Y || !loss_per_step) return fail(AR_ERR_INVALID_ARG, "X, Y and loss_per_step are required");
    if (!aligned16(X) || !aligned16(Y)) return fail(AR_ERR_INVALID_ARG, "X and Y must be 16-byte aligned");
    return tune_mlp(layers, X, M, Y, cfg, n_steps, loss_per_step, grads, workspace, workspace_bytes,
                    reinterpret_cast<cudaStream_t>(stream));
  }
  if (block_kind != AR_BLOCK_LINEAR) return fail(AR_ERR_UNSUPPORTED, "block_kind %d not supported", block_kind);
  return tune_linear(layers, n_layers, X, M, Y, cfg, n_steps, loss_per_step, grads, workspace, workspace_bytes,
                     0, reinterpret_cast<cudaStream_t>(stream));
}

ar_status ar_tune_step_shard(const ar_layer* layer, const uint16_t* X, int64_t M, const float* Y, int64_t n_total,
                             const ar_qconfig* cfg, int n_steps, float* loss_per_step, const ar_grads* grads,
                             void* workspace, size_t workspace_bytes, ar_stream_t stream) {
  begin_call();
  if (!layer) return fail(AR_ERR_INVALID_ARG, "layer is NULL");
  if (n_total < layer->N || n_total > INT32_MAX)
    return fail(AR_ERR_INVALID_ARG, "n_total=%lld must be in [N=%lld, 2^31-1]", (long long)n_total,
                (long long)layer->N);
  return tune_linear(layer, 1, X, M, Y, cfg, n_steps, loss_per_step, grads, workspace, workspace_bytes, n_total,
                     reinterpret_cast<cudaStream_t>(stream));
}

size_t ar_block_forward_workspace(int block_kind, const ar_layer* layers, int n_layers, int64_t M) {
  begin_call();
  if (block_kind == AR_BLOCK_LINEAR) {
    if (!layers || n_layers != 1) {
      fail(AR_ERR_INVALID_ARG, "AR_BLOCK_LINEAR needs one layer");
      return 0;
    }
    return 256;  // no scratch needed; a non-zero size keeps 0 for errors
  }
  if (block_kind != AR_BLOCK_SWIGLU_MLP) {
    fail(AR_ERR_UNSUPPORTED, "block_kind %d not supported", block_kind);
    return 0;
  }
  int64_t Hd = 0, F = 0;
  if (check_mlp(layers, n_layers, M, nullptr, false, &Hd, &F) != AR_OK) return 0;
  return align_up(static_cast<size_t>(M * F) * 2, 256);
}

ar_status ar_block_forward(int block_kind, const ar_layer* layers, int n_layers, const uint16_t* X, int64_t M,
                           float* Y, void* workspace, size_t workspace_bytes, ar_stream_t stream) {
  begin_call();
  if (!X || !Y) return fail(AR_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(X) || !aligned16(Y)) return fail(AR_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (block_kind == AR_BLOCK_LINEAR) {
    if (!layers || n_layers != 1) return fail(AR_ERR_INVALID_ARG, "AR_BLOCK_LINEAR needs one layer");
    return ar_linear_forward(X, M, layers[0].W, layers[0].N, layers[0].K, Y, stream);
  }
  if (block_kind != AR_BLOCK_SWIGLU_MLP) return fail(AR_ERR_UNSUPPORTED, "block_kind %d not supported", block_kind);
  int64_t Hd = 0, F = 0;
  ar_status st = check_mlp(layers, n_layers, M, nullptr, false, &Hd, &F);
  if (st != AR_OK) return st;
  const size_t need = align_up(static_cast<size_t>(M * F) * 2, 256);
  if (!workspace || workspace_bytes < need)
    return fail(AR_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, workspace_bytes);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return fail(AR_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  uint16_t* H = static_cast<uint16_t*>(workspace);
  cudaError_t e = launch_gemm_swiglu_fwd(X, layers[0].W, layers[1].W, nullptr, nullptr, H, static_cast<int>(M),
                                         static_cast<int>(F), static_cast<int>(Hd), s);
  if (e != cudaSuccess) return cuda_fail(e, "SwiGLU forward GEMM launch");
  e = launch_gemm_store(H, layers[2].W, Y, static_cast<int>(M), static_cast<int>(Hd), static_cast<int>(F), s);
  if (e != cudaSuccess) return cuda_fail(e, "down-projection GEMM launch");
  return end_call();
}

ar_status ar_pack_int4(const uint16_t* W, const float* V, const float* alpha, const float* beta, int64_t N, int64_t K,
                       const ar_qconfig* cfg, uint32_t* packed, uint16_t* scale_f16, uint16_t* zero_f16,
                       ar_stream_t stream) {
  begin_call();
  ar_status st = check_cfg(cfg);
  if (st != AR_OK) return st;
  if (cfg->bits != 4) return fail(AR_ERR_UNSUPPORTED, "ar_pack_int4 needs bits == 4 (got %d)", cfg->bits);
  const int g = cfg->group_size;
  if (!pow2(g) || g < 8 || g > 1024) return fail(AR_ERR_UNSUPPORTED, "group_size %d: needs a power of two in 8..1024", g);
  if (N <= 0 || K <= 0) return fail(AR_ERR_INVALID_ARG, "N, K must be positive");
  if (K % g != 0 || K % 8 != 0) return fail(AR_ERR_INVALID_ARG, "K must be a multiple of group_size and of 8");
  const void* ptrs[] = {W, V, alpha, beta, packed, scale_f16, zero_f16};
  for (const void* p : ptrs) {
    if (!p) return fail(AR_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned16(p)) return fail(AR_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  }
  cudaError_t e = launch_pack_int4(W, V, alpha, beta, N, K, g, cfg->symmetric, packed, scale_f16, zero_f16,
                                   reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "pack launch");
  return end_call();
}

ar_status ar_w4a16_gemm(const uint16_t* A, int64_t T, const uint32_t* packed, const uint16_t* scale_f16,
                        const uint16_t* zero_f16, int64_t N, int64_t K, int group_size, uint16_t* out,
                        ar_stream_t stream) {
  begin_call();
  if (T < 1 || N <= 0 || K <= 0) return fail(AR_ERR_INVALID_ARG, "T, N, K must be positive");
  if (!pow2(group_size) || group_size < 32 || group_size > 1024)
    return fail(AR_ERR_UNSUPPORTED, "group_size %d: needs a power of two in 32..1024", group_size);
  if (K % group_size != 0 || K % 128 != 0) return fail(AR_ERR_INVALID_ARG, "K must be a multiple of group_size and 128");
  if (N > INT32_MAX || K > INT32_MAX || T > INT32_MAX) return fail(AR_ERR_UNSUPPORTED, "dimension exceeds 2^31-1");
  const void* ptrs[] = {A, packed, scale_f16, zero_f16, out};
  for (const void* p : ptrs) {
    if (!p) return fail(AR_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned16(p)) return fail(AR_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  }
  // decode batches: CUDA-core dequant into mma.sync fragments; larger: tcgen05 dequant GEMM
  auto launch = T <= 16 ? launch_w4a16 : launch_w4a16_tc;
  cudaError_t e = launch(A, static_cast<int>(T), packed, scale_f16, zero_f16, static_cast<int>(N), static_cast<int>(K),
                         group_size, out, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "w4a16 launch");
  return end_call();
}

ar_status ar_pack_codes(const uint16_t* W, const float* V, const float* alpha, const float* beta, int64_t N,
                        int64_t K, const ar_qconfig* cfg, uint32_t* packed, uint16_t* scale_f16, uint16_t* zero_f16,
                        ar_stream_t stream) {
  begin_call();
  ar_status st = check_cfg(cfg);
  if (st != AR_OK) return st;
  const int bits = cfg->bits;
  if (bits != 2 && bits != 3 && bits != 4 && bits != 8)
    return fail(AR_ERR_UNSUPPORTED, "ar_pack_codes packs 2, 3, 4 or 8-bit codes (got %d)", bits);
  const int g = cfg->group_size;
  if (N <= 0 || K <= 0) return fail(AR_ERR_INVALID_ARG, "N, K must be positive");
  if (!pow2(g) || g < 8 || g > 1024) return fail(AR_ERR_UNSUPPORTED, "group_size %d: needs a power of two in 8..1024", g);
  // every row holds a whole number of 32-bit words: K bits / 32
  const int kmul = bits == 3 ? 32 : 32 / bits;
  if (K % g != 0 || K % kmul != 0) return fail(AR_ERR_INVALID_ARG, "K must be a multiple of group_size and of %d", kmul);
  const void* ptrs[] = {W, V, alpha, beta, packed, scale_f16, zero_f16};
  for (const void* p : ptrs) {
    if (!p) return fail(AR_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned16(p)) return fail(AR_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  }
  cudaError_t e = launch_pack_codes(W, V, alpha, beta, N, K, g, bits, cfg->symmetric, packed, scale_f16, zero_f16,
                                    reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "pack launch");
  return end_call();
}

ar_status ar_wxa16_gemm(const uint16_t* A, int64_t T, const uint32_t* packed, const uint16_t* scale_f16,
                        const uint16_t* zero_f16, int64_t N, int64_t K, int group_size, int bits, uint16_t* out,
                        ar_stream_t stream) {
  if (bits == 4) return ar_w4a16_gemm(A, T, packed, scale_f16, zero_f16, N, K, group_size, out, stream);
  begin_call();
  if (bits != 2 && bits != 3 && bits != 8) return fail(AR_ERR_UNSUPPORTED, "bits=%d: needs 2, 3, 4 or 8", bits);
  if (T < 1 || N <= 0 || K <= 0) return fail(AR_ERR_INVALID_ARG, "T, N, K must be positive");
  if (!pow2(group_size) || group_size < 32 || group_size > 1024)
    return fail(AR_ERR_UNSUPPORTED, "group_size %d: needs a power of two in 32..1024", group_size);
  if (K % group_size != 0 || K % 128 != 0) return fail(AR_ERR_INVALID_ARG, "K must be a multiple of group_size and 128");
  if (N > INT32_MAX || K > INT32_MAX || T > INT32_MAX) return fail(AR_ERR_UNSUPPORTED, "dimension exceeds 2^31-1");
  const void* ptrs[] = {A, packed, scale_f16, zero_f16, out};
  for (const void* p : ptrs) {
    if (!p) return fail(AR_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned16(p)) return fail(AR_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  }
  // Up to 8 tokens with K/g a multiple of 8: the W4A16 decode kernel's 2-bit, 3-bit (g >= 64)
  // and 8-bit forms (measured on 8192 x 28672, T = 1: 30.7, 38.9 and 59.4 us against 79.7 and
  // 79.9 us on the generic decode kernel and 90 us on the tcgen05 GEMM); other 2 and 3-bit shapes up to 8
  // tokens: the generic mma.sync decode kernel (80 us at T <= 8 against 88-90 us for the GEMM,
  // but 90-96 us at T = 16); the rest, and everything from 9 tokens: the tcgen05 dequant GEMM
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int t = static_cast<int>(T), n = static_cast<int>(N), k = static_cast<int>(K);
  cudaError_t e = cudaErrorNotSupported;
  // cudaErrorNotSupported comes from shape checks before any CUDA call: nothing to clear
  if (bits == 2 && T <= 8) e = launch_w2a16_dec(A, t, packed, scale_f16, zero_f16, n, k, group_size, out, s);
  if (bits == 8 && T <= 8) e = launch_w8a16_dec(A, t, packed, scale_f16, zero_f16, n, k, group_size, out, s);
  if (bits == 3 && T <= 8) e = launch_w3a16_dec(A, t, packed, scale_f16, zero_f16, n, k, group_size, out, s);
  if (e == cudaErrorNotSupported)
    e = ((bits == 2 || bits == 3) && T <= 8)
            ? launch_wbx_dec(A, t, packed, scale_f16, zero_f16, n, k, group_size, bits, out, s)
            : launch_wxa16_tc(A, t, packed, scale_f16, zero_f16, n, k, group_size, bits, out, s);
  if (e != cudaSuccess) return cuda_fail(e, "wxa16 launch");
  return end_call();
}

ar_status ar_nvfp4_gemm(const uint16_t* A, int64_t T, const uint8_t* codes, const uint8_t* scales,
                        const float* global_scale, int64_t N, int64_t K, uint16_t* out, ar_stream_t stream) {
  begin_call();
  if (T < 1 || N <= 0 || K <= 0) return fail(AR_ERR_INVALID_ARG, "T, N, K must be positive");
  if (K % 128 != 0) return fail(AR_ERR_INVALID_ARG, "K must be a multiple of 128");
  if (N > INT32_MAX || K > INT32_MAX || T > INT32_MAX) return fail(AR_ERR_UNSUPPORTED, "dimension exceeds 2^31-1");
  const void* ptrs[] = {A, codes, scales, out};
  for (const void* p : ptrs) {
    if (!p) return fail(AR_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned16(p)) return fail(AR_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  }
  if (!global_scale) return fail(AR_ERR_INVALID_ARG, "NULL pointer");
  cudaError_t e = launch_nvfp4_tc(A, static_cast<int>(T), codes, scales, global_scale, static_cast<int>(N),
                                  static_cast<int>(K), out, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "nvfp4 gemm launch");
  return end_call();
}

ar_status ar_gather_samples(const void* src, int64_t n_src_samples, int64_t sample_bytes, const int32_t* idx,
                            int n_idx, void* dst, ar_stream_t stream) {
  begin_call();
  if (!src || !dst || !idx) return fail(AR_ERR_INVALID_ARG, "NULL pointer");
  if (n_idx < 1 || n_idx > kMaxGatherSamples) return fail(AR_ERR_INVALID_ARG, "n_idx must be in 1..%d", kMaxGatherSamples);
  if (sample_bytes <= 0 || sample_bytes % 16 != 0) return fail(AR_ERR_INVALID_ARG, "sample_bytes must be a positive multiple of 16");
  if (n_src_samples <= 0) return fail(AR_ERR_INVALID_ARG, "n_src_samples must be positive");
  if (!aligned16(src) || !aligned16(dst)) return fail(AR_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  for (int i = 0; i < n_idx; ++i)
    if (idx[i] < 0 || idx[i] >= n_src_samples) return fail(AR_ERR_INVALID_ARG, "idx[%d] = %d out of range", i, idx[i]);
  const uintptr_t s0 = reinterpret_cast<uintptr_t>(src), s1 = s0 + static_cast<uintptr_t>(n_src_samples * sample_bytes);
  const uintptr_t d0 = reinterpret_cast<uintptr_t>(dst), d1 = d0 + static_cast<uintptr_t>(n_idx * sample_bytes);
  if (d0 < s1 && s0 < d1) return fail(AR_ERR_INVALID_ARG, "dst overlaps src");
  cudaError_t e = launch_gather_samples(src, sample_bytes, idx, n_idx, dst, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "gather launch");
  return end_call();
}

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

ar_status ar_absmax_bf16(const uint16_t* x, int64_t n, float* amax, ar_stream_t stream) {
  begin_call();
  if (!x || !amax) return fail(AR_ERR_INVALID_ARG, "NULL pointer");
  if (n <= 0 || n % 8 != 0) return fail(AR_ERR_INVALID_ARG, "n must be a positive multiple of 8");
  if (!aligned16(x) || !aligned4(amax)) return fail(AR_ERR_INVALID_ARG, "x must be 16-byte and amax 4-byte aligned");
  cudaError_t e = launch_absmax_bf16(x, n, amax, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "absmax launch");
  return end_call();
}

ar_status ar_qdq_nvfp4(const uint16_t* W, const float* V, const float* alpha, int64_t N, int64_t K, const float* amax,
                       uint16_t* W_hat, uint8_t* codes, uint8_t* scales, float* global_scale, ar_stream_t stream) {
  begin_call();
  if (N <= 0 || K <= 0) return fail(AR_ERR_INVALID_ARG, "N, K must be positive");
  if (K % 16 != 0) return fail(AR_ERR_INVALID_ARG, "K=%lld is not a multiple of the 16-value block", (long long)K);
  if (N > INT64_MAX / K) return fail(AR_ERR_INVALID_ARG, "N*K overflows");
  if (!W || !amax) return fail(AR_ERR_INVALID_ARG, "NULL input pointer");
  if (!W_hat && !codes && !scales && !global_scale) return fail(AR_ERR_INVALID_ARG, "no output requested");
  const void* a16[] = {W, V, W_hat, codes};
  for (const void* p : a16)
    if (p && !aligned16(p)) return fail(AR_ERR_INVALID_ARG, "W, V, W_hat and codes must be 16-byte aligned");
  if ((alpha && !aligned4(alpha)) || !aligned4(amax) || (global_scale && !aligned4(global_scale)))
    return fail(AR_ERR_INVALID_ARG, "alpha, amax and global_scale must be 4-byte aligned");
  cudaError_t e = launch_qdq_nvfp4(W, V, alpha, N * K, amax, W_hat, codes, scales, global_scale,
                                   reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "qdq_nvfp4 launch");
  return end_call();
}

struct Nvfp4Ws {
  size_t what, g, dw, partial, total;
  int partials_per_step;
};

Nvfp4Ws nvfp4_ws(int64_t M, int64_t N, int64_t K, int n_steps) {
  Nvfp4Ws w{};
  size_t off = 0;
  w.what = off;
  off = align_up(off + static_cast<size_t>(N * K) * 2, 256);
  w.g = off;
  off = align_up(off + static_cast<size_t>(M * N) * 2, 256);
  w.dw = off;
  off = align_up(off + static_cast<size_t>(N * K) * 4, 256);
  w.partials_per_step = resid_partials(static_cast<int>(M), static_cast<int>(N));
  w.partial = off;
  off = align_up(off + static_cast<size_t>(w.partials_per_step) * (n_steps > 0 ? n_steps : 1) * 8, 256);
  w.total = off;
  return w;
}

ar_status check_nvfp4_step(int64_t N, int64_t K, int64_t M, int n_steps) {
  if (N <= 0 || K <= 0 || M <= 0) return fail(AR_ERR_INVALID_ARG, "sizes must be positive");
  if (K % 16 != 0) return fail(AR_ERR_INVALID_ARG, "K=%lld is not a multiple of the 16-value block", (long long)K);
  if (N % 8 != 0 || M % 8 != 0) return fail(AR_ERR_INVALID_ARG, "N and M must be multiples of 8");
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return fail(AR_ERR_UNSUPPORTED, "dimension exceeds 2^31-1");
  if (n_steps < 0) return fail(AR_ERR_INVALID_ARG, "n_steps must be >= 0");
  return AR_OK;
}

size_t ar_tune_step_nvfp4_workspace(int64_t M, int64_t N, int64_t K, int n_steps) {
  begin_call();
  if (check_nvfp4_step(N, K, M, n_steps) != AR_OK) return 0;
  return nvfp4_ws(M, N, K, n_steps).total;
}

ar_status ar_tune_step_nvfp4(const uint16_t* W, float* V, float* alpha, int64_t N, int64_t K, const float* amax,
                             const uint16_t* X, int64_t M, const float* Y, const ar_qconfig* cfg, int n_steps,
                             float* loss_per_step, float* dV_out, float* dalpha_out, void* workspace,
                             size_t workspace_bytes, ar_stream_t stream) {
  begin_call();
  ar_status st = check_cfg(cfg);
  if (st != AR_OK) return st;
  st = check_nvfp4_step(N, K, M, n_steps);
  if (st != AR_OK) return st;
  if (!W || !V || !alpha || !amax || !X || !Y || !loss_per_step) return fail(AR_ERR_INVALID_ARG, "NULL pointer");
  const void* a16[] = {W, V, alpha, X, Y, dV_out};
  for (const void* p : a16)
    if (p && !aligned16(p)) return fail(AR_ERR_INVALID_ARG, "W, V, alpha, X, Y and dV_out must be 16-byte aligned");
  if (!aligned4(amax) || !aligned4(loss_per_step) || (dalpha_out && !aligned4(dalpha_out)))
    return fail(AR_ERR_INVALID_ARG, "amax, loss_per_step and dalpha_out must be 4-byte aligned");
  const Nvfp4Ws w = nvfp4_ws(M, N, K, n_steps);
  if (!workspace || workspace_bytes < w.total)
    return fail(AR_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", w.total, workspace_bytes);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return fail(AR_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint16_t* W_hat = reinterpret_cast<uint16_t*>(ws + w.what);
  uint16_t* G = reinterpret_cast<uint16_t*>(ws + w.g);
  float* dW = reinterpret_cast<float*>(ws + w.dw);
  double* partial = reinterpret_cast<double*>(ws + w.partial);
  const int Mi = static_cast<int>(M), Ni = static_cast<int>(N), Ki = static_cast<int>(K);
  const float gscale = static_cast<float>(2.0 / (static_cast<double>(M) * static_cast<double>(N)));
  const int steps = n_steps > 0 ? n_steps : 1;
  cudaError_t e;
  for (int step = 0; step < steps; ++step) {
    e = launch_qdq_nvfp4(W, V, alpha, N * K, amax, W_hat, nullptr, nullptr, nullptr, s);
    if (e != cudaSuccess) return cuda_fail(e, "qdq_nvfp4 launch");
    e = launch_gemm_resid(X, W_hat, Y, G, gscale, partial + static_cast<size_t>(step) * w.partials_per_step, Mi, Ni,
                          Ki, s);
    if (e != cudaSuccess) return cuda_fail(e, "forward GEMM launch");
    if (n_steps == 0) break;
    // dL/dW_hat [N][K] = G^T X: both operands as stored, MN-major, reduced over the M tokens
    e = launch_gemm_plain(G, true, X, true, dW, Ni, Ki, Mi, s);
    if (e != cudaSuccess) return cuda_fail(e, "weight-gradient GEMM launch");
    const bool last = step == steps - 1;
    e = launch_fold_nvfp4(dW, W, V, alpha, N * K, amax, cfg->lr, cfg->v_min, cfg->v_max, cfg->clip_min,
                          cfg->clip_max, last ? dV_out : nullptr, last ? dalpha_out : nullptr, s);
    if (e != cudaSuccess) return cuda_fail(e, "fold_nvfp4 launch");
  }
  e = launch_loss_reduce(partial, w.partials_per_step, steps, 1.0 / (static_cast<double>(M) * static_cast<double>(N)),
                         loss_per_step, s);
  if (e != cudaSuccess) return cuda_fail(e, "loss reduction launch");
  return end_call();
}

ar_status ar_gemm_bf16(const uint16_t* A, int a_mn_major, const uint16_t* B, int b_mn_major, float* D, int64_t M,
                       int64_t N, int64_t K, ar_stream_t stream) {
  begin_call();
  if (M <= 0 || N <= 0 || K <= 0) return fail(AR_ERR_INVALID_ARG, "sizes must be positive");
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return fail(AR_ERR_UNSUPPORTED, "dimension exceeds 2^31-1");
  if (N % 8 != 0 || K % 8 != 0 || (a_mn_major && M % 8 != 0))
    return fail(AR_ERR_INVALID_ARG, "row strides must be multiples of 16 bytes");
  if (!A || !B || !D) return fail(AR_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(A) || !aligned16(B) || !aligned16(D)) return fail(AR_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  cudaError_t e = launch_gemm_plain(A, a_mn_major != 0, B, b_mn_major != 0, D, static_cast<int>(M),
                                    static_cast<int>(N), static_cast<int>(K), reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "gemm launch");
  return end_call();
}

ar_status ar_debug_wait_timeout(uint64_t limit_ns, int* gave_up, ar_stream_t stream) {
  begin_call();
  if (!gave_up) return fail(AR_ERR_INVALID_ARG, "gave_up is NULL");
  if (limit_ns == 0 || limit_ns > 1000000000ull) return fail(AR_ERR_INVALID_ARG, "limit_ns must be in (0, 1e9]");
  cudaError_t e = launch_wait_timeout(limit_ns, gave_up, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "wait-timeout launch");
  return end_call();
}

ar_status ar_get_device_status(ar_stream_t stream) {
  unsigned int v = 0;
  cudaError_t e = read_and_clear_status(&v, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(AR_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
  if (v & kStatusTimeout) return fail(AR_ERR_TIMEOUT, "a pipeline wait timed out on the device");
  if (v & kStatusNonFinite) return fail(AR_ERR_NONFINITE, "non-finite value seen on the device");
  return AR_OK;
}

ar_status ar_profile_start(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (const ProfRecord& r : g_prof_records) {
    g_event_pool.push_back(r.start);
    g_event_pool.push_back(r.stop);
  }
  g_prof_records.clear();
  g_prof_on.store(true);
  return AR_OK;
}

ar_status ar_profile_stop(char* buf, size_t buf_len) {
  g_prof_on.store(false);
  std::lock_guard<std::mutex> lk(g_prof_mu);
  std::map<std::string, std::pair<long, double>> agg;
  ar_status st = AR_OK;
  for (const ProfRecord& r : g_prof_records) {
    float ms = 0.f;
    cudaError_t e = cudaEventSynchronize(r.stop);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, r.start, r.stop);
    if (e != cudaSuccess) {
      st = fail(AR_ERR_CUDA, "profile events: %s", cudaGetErrorString(e));
      continue;
    }
    auto& a = agg[r.name];
    a.first += 1;
    a.second += ms;
    g_event_pool.push_back(r.start);
    g_event_pool.push_back(r.stop);
  }
  g_prof_records.clear();
  std::string out;
  char line[256];
  for (const auto& kv : agg) {
    snprintf(line, sizeof(line), "%s %ld %.6f\n", kv.first.c_str(), kv.second.first, kv.second.second);
    out += line;
  }
  if (buf && buf_len > 0) {
    const size_t n = out.size() < buf_len - 1 ? out.size() : buf_len - 1;
    memcpy(buf, out.data(), n);
    buf[n] = 0;
  }
  return st;
}

size_t ar_decoder_forward_workspace(const ar_decoder_cfg* dcfg, int64_t M) {
  begin_call();
  if (!dcfg || dcfg->n_heads <= 0 || dcfg->hidden <= 0 || dcfg->hidden % dcfg->n_heads != 0 || dcfg->seq_len <= 0 ||
      M <= 0 || M % dcfg->seq_len != 0) {
    fail(AR_ERR_INVALID_ARG, "invalid decoder shapes");
    return 0;
  }
  return dec_ws(M, dcfg->hidden, dcfg->intermediate, dcfg->seq_len, static_cast<int>(dcfg->hidden / dcfg->n_heads),
                32, 0, false)
      .total;
}

ar_status ar_decoder_forward(const ar_decoder_cfg* dcfg, const ar_layer* layers, const uint16_t* X, int64_t M,
                             float* Y, void* workspace, size_t workspace_bytes, ar_stream_t stream) {
  begin_call();
  return decoder_reference(dcfg, layers, X, M, Y, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

size_t ar_tune_step_decoder_workspace(const ar_decoder_cfg* dcfg, const ar_layer* layers, int64_t M,
                                      const ar_qconfig* cfg, int n_steps) {
  begin_call();
  if (n_steps < 0 || check_decoder(dcfg, layers, M, cfg, true) != AR_OK) {
    if (t_error.empty()) fail(AR_ERR_INVALID_ARG, "invalid decoder block");
    return 0;
  }
  return dec_ws(M, dcfg->hidden, dcfg->intermediate, dcfg->seq_len, static_cast<int>(dcfg->hidden / dcfg->n_heads),
                cfg->group_size, n_steps, true)
      .total;
}

ar_status ar_tune_step_decoder(const ar_decoder_cfg* dcfg, const ar_layer* layers, const uint16_t* X, int64_t M,
                               const float* Y, const ar_qconfig* cfg, int n_steps, float* loss_per_step,
                               const ar_grads* grads, void* workspace, size_t workspace_bytes, ar_stream_t stream) {
  begin_call();
  return decoder_tune(dcfg, layers, X, M, Y, cfg, n_steps, loss_per_step, grads, workspace, workspace_bytes,
                      reinterpret_cast<cudaStream_t>(stream));
}

ar_status ar_rmsnorm(const void* x, int x_is_f32, const float* gamma, int64_t M, int64_t H, uint16_t* r, float* inv,
                     ar_stream_t stream) {
  begin_call();
  if (M <= 0 || H <= 0 || H % 8 != 0 || H > INT32_MAX) return fail(AR_ERR_INVALID_ARG, "M > 0 and H a positive multiple of 8");
  if (!x || !gamma || !r || !aligned16(x) || !aligned16(gamma) || !aligned16(r) || (inv && !aligned4(inv)))
    return fail(AR_ERR_INVALID_ARG, "x, gamma, r must be 16-byte aligned device pointers");
  cudaError_t e = launch_rmsnorm_fwd(x, x_is_f32 != 0, gamma, M, static_cast<int>(H), r, inv,
                                     reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "rmsnorm launch");
  return end_call();
}

static ar_status check_attention(int64_t S, int64_t L, int64_t H, int n_heads) {
  if (S <= 0 || L <= 0 || H <= 0 || n_heads <= 0) return fail(AR_ERR_INVALID_ARG, "sizes must be positive");
  if (L % 64 != 0) return fail(AR_ERR_INVALID_ARG, "L=%lld must be a multiple of 64", (long long)L);
  if (H % n_heads != 0 || (H / n_heads != 64 && H / n_heads != 128))
    return fail(AR_ERR_UNSUPPORTED, "head dim H/n_heads must be 64 or 128");
  if (S > 65535 || n_heads > 65535 || S * L * 3 * H > (int64_t(1) << 40)) return fail(AR_ERR_UNSUPPORTED, "too large");
  return AR_OK;
}

ar_status ar_attention_forward(const uint16_t* qkv, int64_t S, int64_t L, int64_t H, int n_heads, uint16_t* out,
                               float* lse, ar_stream_t stream) {
  begin_call();
  ar_status st = check_attention(S, L, H, n_heads);
  if (st != AR_OK) return st;
  if (!qkv || !out || !lse || !aligned16(qkv) || !aligned16(out) || !aligned16(lse))
    return fail(AR_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  cudaError_t e = launch_attn_fwd(qkv, static_cast<int>(S), static_cast<int>(L), static_cast<int>(H),
                                  static_cast<int>(H / n_heads), out, lse, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  return end_call();
}

size_t ar_attention_backward_workspace(int64_t S, int64_t L, int64_t H, int n_heads) {
  begin_call();
  if (check_attention(S, L, H, n_heads) != AR_OK) return 0;
  const int64_t hd = H / n_heads;
  return align_up(static_cast<size_t>(L * hd / 2) * 8, 256) + align_up(static_cast<size_t>(S * n_heads * L) * 4, 256);
}

ar_status ar_attention_backward(const uint16_t* qkv, const uint16_t* out, const uint16_t* dout, const float* lse,
                                int64_t S, int64_t L, int64_t H, int n_heads, uint16_t* dqkv, void* workspace,
                                size_t workspace_bytes, ar_stream_t stream) {
  begin_call();
  ar_status st = check_attention(S, L, H, n_heads);
  if (st != AR_OK) return st;
  const void* ptrs[] = {qkv, out, dout, lse, dqkv};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return fail(AR_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  const int64_t hd = H / n_heads;
  const size_t rope_bytes = align_up(static_cast<size_t>(L * hd / 2) * 8, 256);
  const size_t need = rope_bytes + align_up(static_cast<size_t>(S * n_heads * L) * 4, 256);
  if (!workspace || workspace_bytes < need)
    return fail(AR_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, workspace_bytes);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return fail(AR_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float* cs = static_cast<float*>(workspace);
  float* dsum = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + rope_bytes);
  cudaError_t e = launch_rope_table(static_cast<int>(L), static_cast<int>(hd), cs, s);
  if (e != cudaSuccess) return cuda_fail(e, "rope table launch");
  e = launch_attn_bwd(qkv, out, dout, lse, dsum, cs, static_cast<int>(S), static_cast<int>(L), static_cast<int>(H),
                      static_cast<int>(hd), dqkv, s);
  if (e != cudaSuccess) return cuda_fail(e, "attention backward launch");
  return end_call();
}

const char* ar_last_error(void) { return t_error.c_str(); }

const char* ar_last_kernels(void) { return t_kernels_last.c_str(); }

const char* ar_version(void) { return "autoround-b200 0.1 (sm_100a)"; }

}  // extern "C"
