// Straight-through fold + SignSGD of one tuning step from a materialised
// dL/dŴ (fp32 [N][K], the weight-gradient GEMM's plain output), for short token
// counts.  [AR] = "Low-Bit Quantization in Practice with vLLM: Core Mechanisms and
// Architectural Optimizations of AutoRound", §3 "Algorithm Flow" steps 4-5 and
// "SignSGD".
//
// The weight-gradient GEMM normally folds in its epilogue, where dŴ never leaves
// the SM.  That epilogue runs on the GEMM's eight epilogue warps per SM and
// overlaps the next tile's MMAs; with a short token reduction (a 2048-token
// calibration batch: 32 k-blocks per tile) the MMAs finish long before the fold,
// and the GEMM waits on it.  Writing dŴ and folding here instead costs 8 bytes
// per weight of traffic but runs the fold at full occupancy, streaming W, V and
// dŴ at HBM speed.
//
// Per element the same steps as the epilogue, in the same order (ar_fold.cuh):
// Q = 2^b - 1; w/s, t = round(w/s + v) + zp, m = 1[0 <= t <= Q], dV = g s m,
// c = g ((clamp(t) - zp) - (m ? w/s : lo/s)) (symmetric: g (m ? qz - w/s : qz)),
// o = g (1 - m); per group the sums of c and o give dalpha, dbeta; then the
// sign steps of V, alpha, beta.  Layout: each lane takes 8 consecutive weights of
// the flat [N][K] array (a group never crosses a row, since g divides K), so a
// group of g weights is g / 8 lanes of one warp, whose sums meet through a fixed
// xor-shuffle tree (deterministic; the epilogue sums a group in column order,
// so the two paths agree to rounding, not bit for bit).
#include "ar_fold.cuh"
#include "ar_internal.h"

namespace ar {
namespace {

// With W_hat_next, the kernel also takes the next step's QDQ (the group's new
// alpha, beta and the elements' new V): W_hat_next (bf16), and the group's scale
// and zero-point in place of this step's in f.s, f.zp (each group's entries are
// read by its own lanes before its leader writes them).  The arithmetic is
// qdq_kernel's (group_qparams, qdq_elem), so W_hat_next is the QDQ of the
// updated state, bit for bit.
// Three blocks an SM (at most 80 registers a thread): the stream needs the
// occupancy more than the registers (measured: 88 -> 78 us for 4096 x 4096).
template <int G>
__global__ void __launch_bounds__(256, 3) fold_int_kernel(const float* __restrict__ dW, const FoldArgs f, int64_t n,
                                                       uint16_t* __restrict__ W_hat_next) {
  constexpr int kLanes = G / 8;  // lanes per group: 4, 8, 16 or 32
  const float Q = static_cast<float>((1 << f.bits) - 1);
  const int lane = threadIdx.x & 31;
  const int64_t warp = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
  const int64_t warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  bool bad = false;
  for (int64_t base = warp * 256; base < n; base += warps * 256) {
    const int64_t e0 = base + 8 * lane;
    const bool live = e0 < n;  // n is a multiple of G, so a group is all live or all dead
    uint4 w = make_uint4(0u, 0u, 0u, 0u);
    float vv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float gw[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    GroupParams gp{};
    if (live) {
      w = __ldcs(reinterpret_cast<const uint4*>(f.W + e0));
      const float4 v0 = __ldcs(reinterpret_cast<const float4*>(f.V + e0));
      const float4 v1 = __ldcs(reinterpret_cast<const float4*>(f.V + e0 + 4));
      const float4 g0 = __ldcs(reinterpret_cast<const float4*>(dW + e0));
      const float4 g1 = __ldcs(reinterpret_cast<const float4*>(dW + e0 + 4));
      vv[0] = v0.x; vv[1] = v0.y; vv[2] = v0.z; vv[3] = v0.w;
      vv[4] = v1.x; vv[5] = v1.y; vv[6] = v1.z; vv[7] = v1.w;
      gw[0] = g0.x; gw[1] = g0.y; gw[2] = g0.z; gw[3] = g0.w;
      gw[4] = g1.x; gw[5] = g1.y; gw[6] = g1.z; gw[7] = g1.w;
      group_load(f, static_cast<size_t>(e0 / G), gp);
      group_prepare(f, gp);
    }
    const uint32_t wr[4] = {w.x, w.y, w.z, w.w};
    float dv[8];
    float csum = 0.f, osum = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      dv[i] = 0.f;
      if (!live) continue;
      const float wi = (i & 1) ? bf16_hi(wr[i >> 1]) : bf16_lo(wr[i >> 1]);
      const float wq = __fdiv_rn(wi, gp.s);
      const float t = __fadd_rn(roundf(__fadd_rn(wq, vv[i])), gp.zp);
      const bool in = (t >= 0.0f) && (t <= Q);
      const float qz = __fsub_rn(fminf(fmaxf(t, 0.0f), Q), gp.zp);
      const float gi = gw[i];
      dv[i] = in ? __fmul_rn(gi, gp.s) : 0.0f;
      float ci;
      if (f.symmetric) ci = __fmul_rn(gi, in ? __fsub_rn(qz, wq) : qz);
      else ci = __fmul_rn(gi, __fsub_rn(qz, in ? wq : gp.lo_s));
      // a NaN/Inf gradient reaches csum (or osum) and is reported at the group's end
      csum = __fadd_rn(csum, ci);
      osum = in ? osum : __fadd_rn(osum, gi);
      vv[i] = sign_step(vv[i], dv[i], f.lr, f.v_min, f.v_max);
    }
    // the group's sums: butterfly over its kLanes lanes (aligned, consecutive), the same on each
#pragma unroll
    for (int off = kLanes / 2; off > 0; off >>= 1) {
      csum = __fadd_rn(csum, __shfl_xor_sync(0xFFFFFFFFu, csum, off));
      osum = __fadd_rn(osum, __shfl_xor_sync(0xFFFFFFFFu, osum, off));
    }
    if (!live) continue;
    __stcs(reinterpret_cast<float4*>(f.V + e0), make_float4(vv[0], vv[1], vv[2], vv[3]));
    __stcs(reinterpret_cast<float4*>(f.V + e0 + 4), make_float4(vv[4], vv[5], vv[6], vv[7]));
    if (f.dV_out) {
      __stcs(reinterpret_cast<float4*>(f.dV_out + e0), make_float4(dv[0], dv[1], dv[2], dv[3]));
      __stcs(reinterpret_cast<float4*>(f.dV_out + e0 + 4), make_float4(dv[4], dv[5], dv[6], dv[7]));
    }
    // every lane of the group holds the same sums: each steps alpha, beta; the leader writes them
    const bool leader = (lane & (kLanes - 1)) == 0;
    float al1, be1;
    const bool gbad = group_finish(f, gp, csum, osum, leader, &al1, &be1);
    if (leader) bad |= gbad;
    if (W_hat_next) {
      const QParams pn = group_qparams(gp.mx, gp.mn, al1, be1, f.bits, f.symmetric);
      float wh[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float wi = (i & 1) ? bf16_hi(wr[i >> 1]) : bf16_lo(wr[i >> 1]);
        float q;
        wh[i] = qdq_elem(wi, vv[i], pn, Q, q);
      }
      uint4 o;
      o.x = pack_bf16x2(wh[0], wh[1]);
      o.y = pack_bf16x2(wh[2], wh[3]);
      o.z = pack_bf16x2(wh[4], wh[5]);
      o.w = pack_bf16x2(wh[6], wh[7]);
      *reinterpret_cast<uint4*>(W_hat_next + e0) = o;
      if (leader) {
        const_cast<float*>(f.s)[gp.gidx] = pn.s;
        const_cast<float*>(f.zp)[gp.gidx] = pn.zp;
      }
    }
  }
  if (bad) raise_status(kStatusNonFinite);
}

}  // namespace

bool fold_int_supported(int group_size) {
  return group_size == 32 || group_size == 64 || group_size == 128 || group_size == 256;
}

// Measured on the 4096 x 4096 layer with 2048 tokens (step time, GEMM fold epilogue
// vs plain GEMM + this kernel): g 32 250.8 vs 193.6 us, g 64 219.2 vs 194.1, g 128
// 200.5 vs 193.9, g 256 195.0 vs 199.7; at 16384 tokens the epilogue keeps up with the
// MMAs and the fused fold is the faster.
bool use_split_fold(int64_t M, int group_size) {
  return M < kFoldSplitTokens && group_size <= 128 && fold_int_supported(group_size);
}

cudaError_t launch_fold_int(const float* dW, const FoldArgs& fa, int64_t N, int64_t K, uint16_t* W_hat_next,
                            cudaStream_t stream) {
  if (!fold_int_supported(fa.group_size) || K % fa.group_size != 0) return cudaErrorInvalidValue;
  const int64_t n = N * K;
  int64_t blocks = (n / 256 + 7) / 8;  // eight warps a block, 256 weights a warp pass
  const int64_t cap = static_cast<int64_t>(num_sms()) * 16;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  LaunchScope scope(stream, "fold_int_kernel");
  switch (fa.group_size) {
    case 32: fold_int_kernel<32><<<static_cast<int>(blocks), 256, 0, stream>>>(dW, fa, n, W_hat_next); break;
    case 64: fold_int_kernel<64><<<static_cast<int>(blocks), 256, 0, stream>>>(dW, fa, n, W_hat_next); break;
    case 128: fold_int_kernel<128><<<static_cast<int>(blocks), 256, 0, stream>>>(dW, fa, n, W_hat_next); break;
    default: fold_int_kernel<256><<<static_cast<int>(blocks), 256, 0, stream>>>(dW, fa, n, W_hat_next); break;
  }
  return cudaGetLastError();
}

}  // namespace ar
