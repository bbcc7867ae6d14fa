// Shared arithmetic of the straight-through fold and the SignSGD step of the
// integer quantizer ([AR] "Low-Bit Quantization in Practice with vLLM: Core
// Mechanisms and Architectural Optimizations of AutoRound", §3 "Algorithm Flow"
// steps 4-5 and "SignSGD"): the group parameters of one quantization group, the
// per-group quantities of the backward pass, and the clamped sign step.  Used by
// the weight-gradient GEMM's fold epilogue and by the standalone fold kernel, so
// that both take the same steps in the same order.
#pragma once

#include "ar_internal.h"

namespace ar {

struct QParams {
  float s, zp, lo, mx, mn;
  bool guarded;
};

// Scale / zero-point of a group; identical arithmetic in every kernel that needs it.
__device__ __forceinline__ QParams group_qparams(float mx, float mn, float alpha, float beta, int bits,
                                                 int symmetric) {
  QParams p;
  p.mx = mx;
  p.mn = mn;
  const float hi = __fmul_rn(alpha, mx);
  const float lo = __fmul_rn(beta, mn);
  float s;
  if (!symmetric) {
    s = __fdiv_rn(__fsub_rn(hi, lo), static_cast<float>((1 << bits) - 1));
  } else {
    s = __fdiv_rn(fmaxf(hi, -lo), static_cast<float>((1 << (bits - 1)) - 1));
  }
  p.guarded = s < kScaleGuard;
  if (p.guarded) s = kScaleGuard;
  p.s = s;
  p.lo = lo;
  p.zp = symmetric ? static_cast<float>(1 << (bits - 1)) : roundf(__fdiv_rn(-lo, s));
  return p;
}

// One element's fake quantization with its group's parameters:
// u = w/s + v, t = round(u) + zp (round half away from zero), q = clamp(t, 0, Q),
// returns W_hat = s (q - zp) and the code q.
__device__ __forceinline__ float qdq_elem(float w, float v, const QParams& p, float Q, float& q) {
  const float u = __fadd_rn(__fdiv_rn(w, p.s), v);
  const float t = __fadd_rn(roundf(u), p.zp);
  q = fminf(fmaxf(t, 0.0f), Q);
  return __fmul_rn(p.s, __fsub_rn(q, p.zp));
}

// p - lr*sign(d), clamped; sign(0) = sign(NaN) = 0.  p - (-lr) is the same
// IEEE result as p + lr.
__device__ __forceinline__ float sign_step(float p, float d, float lr, float lo, float hi) {
  const float step = d > 0.0f ? lr : (d < 0.0f ? -lr : 0.0f);
  return fminf(fmaxf(__fsub_rn(p, step), lo), hi);
}

struct GroupParams {
  float s, zp, lo_s, mx, mn, al, be;
  bool guarded, take_hi;
  size_t gidx;
};

__device__ __forceinline__ void group_load(const FoldArgs& f, size_t gidx, GroupParams& gp) {
  gp.gidx = gidx;
  gp.s = f.s[gidx];
  gp.zp = f.zp[gidx];
  gp.mx = f.mx[gidx];
  gp.mn = f.mn[gidx];
  gp.al = f.alpha[gidx];
  gp.be = f.beta[gidx];
}

__device__ __forceinline__ void group_prepare(const FoldArgs& f, GroupParams& gp) {
  const float Q = static_cast<float>((1 << f.bits) - 1);
  const float Qs = static_cast<float>((1 << (f.bits - 1)) - 1);
  const float hi = __fmul_rn(gp.al, gp.mx);
  const float lo = __fmul_rn(gp.be, gp.mn);
  const float s_raw = f.symmetric ? __fdiv_rn(fmaxf(hi, -lo), Qs) : __fdiv_rn(__fsub_rn(hi, lo), Q);
  gp.guarded = s_raw < kScaleGuard;
  gp.take_hi = hi >= -lo;
  gp.lo_s = __fdiv_rn(lo, gp.s);
}

// Finishes a group: dalpha, dbeta from the (full) sums and the SignSGD step of
// alpha, beta, written when `write`; the stepped values also go to *al_new and
// *be_new when given.  Returns true when a sum or gradient is not finite.
__device__ __forceinline__ bool group_finish(const FoldArgs& f, const GroupParams& gp, float csum, float osum,
                                             bool write, float* al_new = nullptr, float* be_new = nullptr) {
  const float Q = static_cast<float>((1 << f.bits) - 1);
  const float Qs = static_cast<float>((1 << (f.bits - 1)) - 1);
  if (gp.guarded) csum = 0.0f;
  float dhi, dlo;
  if (f.symmetric) {
    const float ds = __fdiv_rn(csum, Qs);
    dhi = gp.take_hi ? ds : 0.0f;
    dlo = gp.take_hi ? 0.0f : -ds;
  } else {
    const float cq = __fdiv_rn(csum, Q);
    dhi = cq;
    dlo = __fsub_rn(osum, cq);
  }
  const bool sums_bad = !isfinite(csum) || !isfinite(osum);
  const float da = __fmul_rn(gp.mx, dhi);
  const float db = __fmul_rn(gp.mn, dlo);
  const float a1 = sign_step(gp.al, da, f.lr, f.c_min, f.c_max);
  const float b1 = sign_step(gp.be, db, f.lr, f.c_min, f.c_max);
  if (al_new) *al_new = a1;
  if (be_new) *be_new = b1;
  if (write) {
    f.alpha[gp.gidx] = a1;
    f.beta[gp.gidx] = b1;
    if (f.da_out) f.da_out[gp.gidx] = da;
    if (f.db_out) f.db_out[gp.gidx] = db;
  }
  return sums_bad || !isfinite(da) || !isfinite(db);
}

}  // namespace ar
