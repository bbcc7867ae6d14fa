// NVFP4 fake quantization (QDQ) of a bf16 weight matrix, and the per-tensor
// absolute maximum it needs.
//
// A new data type enters the tuning through one tensor-level QDQ function
// ([AR] §4 "Why the Tuning Stage Must Take the QDQ Path", point 3; [AR] = "Low-Bit
// Quantization in Practice with vLLM: Core Mechanisms and Architectural
// Optimizations of AutoRound").  The format: E2M1 values (1 sign, 2 exponent, 1
// mantissa bits) and E4M3 scales ([QC] "量化：从 Scale 到 W4A8 的完整坐标" §2
// table), one E4M3 scale per block of 16 values and a per-tensor scale ([QC] §5
// table, row "NVFP4 recipe"; [NQ] "量化" (note.yj-dis.top), section
// "低比特浮点：FP8 与 NVFP4").  In fp32, per block b of 16 along K:
//   S = amax(|W|) / (6 * 448)
//   s_b = E4M3((alpha_b * amax_b) / 6 / S) * S
//   q = E2M1(W / s_b + V),  Ŵ = q * s_b  (q = 0, Ŵ = 0 where s_b = 0)
// with round-to-nearest-even, saturating conversions (the hardware cvt of
// sm_100a).  alpha (the learnable clip factor) and V (the learnable offset) act
// as in the integer quantizer.
//
// Both kernels stream: each warp moves 512 consecutive weights per step (one
// 16-byte load of 8 bf16 per lane and chunk), and the two lanes that hold the
// halves of a 16-value block combine their maxima with one shuffle.
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "ar_internal.h"

namespace ar {
namespace {

constexpr int kNvBlock = 16;
constexpr float kE2M1Max = 6.0f;
constexpr float kE2M1xE4M3Max = 2688.0f;  // 6 * 448

// max of the magnitudes of the eight bf16 in v (as bf16 bit patterns, which
// order like the values for non-negative numbers)
__device__ __forceinline__ uint32_t max_mag8(const uint4& v) {
  uint32_t m = __vmaxu2(__vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu), __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu));
  return max(m & 0xFFFFu, m >> 16);
}

__global__ void absmax_bf16_kernel(const uint4* __restrict__ x, int64_t n_vec, unsigned int* __restrict__ amax_bits) {
  uint32_t m = 0;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n_vec;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    m = max(m, max_mag8(__ldcs(x + i)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((threadIdx.x & 31) == 0 && m != 0) {
    if (m >= 0x7F80u) raise_status(kStatusNonFinite);  // Inf or NaN among the inputs
    atomicMax(amax_bits, m << 16);                      // the fp32 bits of the bf16 maximum
  }
}

__device__ __forceinline__ float bf16_lo_f(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi_f(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
  const __nv_bfloat16 l = __float2bfloat16_rn(lo);
  const __nv_bfloat16 h = __float2bfloat16_rn(hi);
  return static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(&l)) |
         (static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(&h)) << 16);
}

// One warp step covers 512 weights = 32 blocks; lane l holds elements
// [8l, 8l + 8) of chunk c (c = 0, 1: the step's first and second 256), i.e.
// half of block 16c + l/2.
__global__ void __launch_bounds__(256) qdq_nvfp4_kernel(const uint16_t* __restrict__ W, const float* __restrict__ V,
                                                        const float* __restrict__ alpha, int64_t n,
                                                        const unsigned int* __restrict__ amax_bits,
                                                        uint16_t* __restrict__ W_hat, uint8_t* __restrict__ codes,
                                                        uint8_t* __restrict__ scales, float* __restrict__ global_scale) {
  const float amax = __uint_as_float(*amax_bits);
  const float S = __fdiv_rn(amax, kE2M1xE4M3Max);
  if (global_scale && blockIdx.x == 0 && threadIdx.x == 0) *global_scale = S;
  const int lane = threadIdx.x & 31;
  const int64_t warp = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
  const int64_t warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t base = warp * 512; base < n; base += warps * 512) {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int64_t e0 = base + c * 256 + 8 * lane;  // first of this lane's 8 elements
      const bool live = e0 < n;                      // n is a multiple of 16: a block is all in or all out
      uint4 w = make_uint4(0, 0, 0, 0);
      if (live) w = __ldcs(reinterpret_cast<const uint4*>(W + e0));
      // block maximum: this lane's half, then its partner's (lanes 2j and 2j+1 share block j)
      uint32_t m = max_mag8(w);
      m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
      if (!live) continue;
      const float amax_b = __uint_as_float(m << 16);
      const int64_t blk = e0 / kNvBlock;
      const float a = alpha ? __ldg(alpha + blk) : 1.0f;
      const float sb = __fdiv_rn(__fmul_rn(a, amax_b), kE2M1Max);
      const float ratio = S > 0.0f ? __fdiv_rn(sb, S) : 0.0f;
      const __nv_fp8_storage_t s8 = __nv_cvt_float_to_fp8(ratio, __NV_SATFINITE, __NV_E4M3);
      const float s_eff = __fmul_rn(__half2float(__half(__nv_cvt_fp8_to_halfraw(s8, __NV_E4M3))), S);
      float x[8] = {bf16_lo_f(w.x), bf16_hi_f(w.x), bf16_lo_f(w.y), bf16_hi_f(w.y),
                    bf16_lo_f(w.z), bf16_hi_f(w.z), bf16_lo_f(w.w), bf16_hi_f(w.w)};
      float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (V) {
        const float4 v0 = __ldcs(reinterpret_cast<const float4*>(V + e0));
        const float4 v1 = __ldcs(reinterpret_cast<const float4*>(V + e0 + 4));
        v[0] = v0.x; v[1] = v0.y; v[2] = v0.z; v[3] = v0.w;
        v[4] = v1.x; v[5] = v1.y; v[6] = v1.z; v[7] = v1.w;
      }
      uint32_t code_word = 0;
      float wq[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        uint32_t q = 0;
        float qf = 0.0f;
        if (s_eff > 0.0f) {
          const float t = __fadd_rn(__fdiv_rn(x[i], s_eff), v[i]);
          q = static_cast<uint32_t>(__nv_cvt_float_to_fp4(t, __NV_E2M1, cudaRoundNearest)) & 0xFu;
          qf = __half2float(__half(__nv_cvt_fp4_to_halfraw(static_cast<__nv_fp4_storage_t>(q), __NV_E2M1)));
        }
        wq[i] = s_eff > 0.0f ? __fmul_rn(qf, s_eff) : 0.0f;
        code_word |= q << (4 * i);
      }
      if (W_hat) {
        uint4 o;
        o.x = bf16x2_rn(wq[0], wq[1]);
        o.y = bf16x2_rn(wq[2], wq[3]);
        o.z = bf16x2_rn(wq[4], wq[5]);
        o.w = bf16x2_rn(wq[6], wq[7]);
        __stcs(reinterpret_cast<uint4*>(W_hat + e0), o);
      }
      if (codes) __stcs(reinterpret_cast<unsigned int*>(codes + e0 / 2), code_word);
      if (scales && (lane & 1) == 0) scales[blk] = static_cast<uint8_t>(s8);
    }
  }
}

// Backward and update of one tuning step on NVFP4, from dL/dŴ (fp32 [N][K], the
// weight-gradient GEMM's output).  The forward's values are recomputed exactly
// as qdq_nvfp4_kernel computes them; the straight-through fold counts both
// roundings as the identity and passes the gradient where |W/s + V| <= 6:
//   dV_i = g_i s_b m_i,   dalpha_b = (amax_b / 6) sum_i g_i (q_i - m_i W_i / s_b)
// then V <- clamp(V - lr sign(dV)), alpha <- clamp(alpha - lr sign(dalpha))
// ([AR] §3 "SignSGD"; sign(0) = 0, a NaN gradient counts as 0 and raises the
// non-finite status).  Same lane layout as the QDQ: the two lanes of a block add
// their halves of the block sum with one shuffle (a + b on both lanes).
__device__ __forceinline__ float sign0f(float d) { return d > 0.f ? 1.f : (d < 0.f ? -1.f : 0.f); }

__global__ void __launch_bounds__(256) fold_nvfp4_kernel(const float* __restrict__ dW, const uint16_t* __restrict__ W,
                                                         float* __restrict__ V, float* __restrict__ alpha, int64_t n,
                                                         const unsigned int* __restrict__ amax_bits, float lr,
                                                         float v_min, float v_max, float c_min, float c_max,
                                                         float* __restrict__ dV_out, float* __restrict__ da_out) {
  const float S = __fdiv_rn(__uint_as_float(*amax_bits), kE2M1xE4M3Max);
  const int lane = threadIdx.x & 31;
  const int64_t warp = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
  const int64_t warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t base = warp * 512; base < n; base += warps * 512) {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int64_t e0 = base + c * 256 + 8 * lane;
      const bool live = e0 < n;
      uint4 w = make_uint4(0, 0, 0, 0);
      float4 v0 = make_float4(0.f, 0.f, 0.f, 0.f), v1 = v0, g0 = v0, g1 = v0;
      float a = 1.0f;
      const int64_t blk = e0 / kNvBlock;
      if (live) {
        w = __ldcs(reinterpret_cast<const uint4*>(W + e0));
        v0 = __ldcs(reinterpret_cast<const float4*>(V + e0));
        v1 = __ldcs(reinterpret_cast<const float4*>(V + e0 + 4));
        g0 = __ldcs(reinterpret_cast<const float4*>(dW + e0));
        g1 = __ldcs(reinterpret_cast<const float4*>(dW + e0 + 4));
        a = alpha[blk];
      }
      uint32_t m = max_mag8(w);
      m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
      const float amax_b = __uint_as_float(m << 16);
      const float sb = __fdiv_rn(__fmul_rn(a, amax_b), kE2M1Max);
      const float ratio = S > 0.0f ? __fdiv_rn(sb, S) : 0.0f;
      const __nv_fp8_storage_t s8 = __nv_cvt_float_to_fp8(ratio, __NV_SATFINITE, __NV_E4M3);
      const float s_eff = __fmul_rn(__half2float(__half(__nv_cvt_fp8_to_halfraw(s8, __NV_E4M3))), S);
      const float x[8] = {bf16_lo_f(w.x), bf16_hi_f(w.x), bf16_lo_f(w.y), bf16_hi_f(w.y),
                          bf16_lo_f(w.z), bf16_hi_f(w.z), bf16_lo_f(w.w), bf16_hi_f(w.w)};
      const float v[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
      const float g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
      float dv[8];
      float csum = 0.0f;
      bool bad = false;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        dv[i] = 0.0f;
        if (s_eff > 0.0f) {
          const float ws = __fdiv_rn(x[i], s_eff);
          const float t = __fadd_rn(ws, v[i]);
          const uint32_t q = static_cast<uint32_t>(__nv_cvt_float_to_fp4(t, __NV_E2M1, cudaRoundNearest)) & 0xFu;
          const float qf = __half2float(__half(__nv_cvt_fp4_to_halfraw(static_cast<__nv_fp4_storage_t>(q), __NV_E2M1)));
          const bool mi = fabsf(t) <= kE2M1Max;
          dv[i] = mi ? __fmul_rn(g[i], s_eff) : 0.0f;
          csum = __fadd_rn(csum, __fmul_rn(g[i], __fsub_rn(qf, mi ? ws : 0.0f)));
        }
        bad |= !(fabsf(g[i]) <= 3.0e38f);
      }
      // the block sum: this lane's half plus its partner's (the same sum on both lanes)
      const float other = __shfl_xor_sync(0xFFFFFFFFu, csum, 1);
      const float cblk = (lane & 1) ? __fadd_rn(other, csum) : __fadd_rn(csum, other);
      if (!live) continue;
      if (bad) raise_status(kStatusNonFinite);
      const float da = __fmul_rn(__fdiv_rn(amax_b, kE2M1Max), cblk);
      float vo[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        vo[i] = fminf(fmaxf(__fsub_rn(v[i], lr * sign0f(dv[i])), v_min), v_max);
      __stcs(reinterpret_cast<float4*>(V + e0), make_float4(vo[0], vo[1], vo[2], vo[3]));
      __stcs(reinterpret_cast<float4*>(V + e0 + 4), make_float4(vo[4], vo[5], vo[6], vo[7]));
      if (dV_out) {
        __stcs(reinterpret_cast<float4*>(dV_out + e0), make_float4(dv[0], dv[1], dv[2], dv[3]));
        __stcs(reinterpret_cast<float4*>(dV_out + e0 + 4), make_float4(dv[4], dv[5], dv[6], dv[7]));
      }
      if ((lane & 1) == 0) {
        alpha[blk] = fminf(fmaxf(__fsub_rn(a, lr * sign0f(da)), c_min), c_max);
        if (da_out) da_out[blk] = da;
      }
    }
  }
}

int grid_for(int64_t units, int per_block) {
  int64_t b = (units + per_block - 1) / per_block;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 16;
  if (b > cap) b = cap;
  return static_cast<int>(b < 1 ? 1 : b);
}

}  // namespace

cudaError_t launch_absmax_bf16(const uint16_t* x, int64_t n, float* amax, cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(float), stream);
  if (e != cudaSuccess) return e;
  const int64_t n_vec = n / 8;
  {
    LaunchScope scope(stream, "absmax_bf16_kernel");
    absmax_bf16_kernel<<<grid_for(n_vec, 256), 256, 0, stream>>>(reinterpret_cast<const uint4*>(x), n_vec,
                                                                 reinterpret_cast<unsigned int*>(amax));
  }
  return cudaGetLastError();
}

cudaError_t launch_qdq_nvfp4(const uint16_t* W, const float* V, const float* alpha, int64_t n, const float* amax,
                             uint16_t* W_hat, uint8_t* codes, uint8_t* scales, float* global_scale,
                             cudaStream_t stream) {
  {
    LaunchScope scope(stream, "qdq_nvfp4_kernel");
    qdq_nvfp4_kernel<<<grid_for((n + 511) / 512, 8), 256, 0, stream>>>(
        W, V, alpha, n, reinterpret_cast<const unsigned int*>(amax), W_hat, codes, scales, global_scale);
  }
  return cudaGetLastError();
}

cudaError_t launch_fold_nvfp4(const float* dW, const uint16_t* W, float* V, float* alpha, int64_t n, const float* amax,
                              float lr, float v_min, float v_max, float c_min, float c_max, float* dV_out,
                              float* da_out, cudaStream_t stream) {
  {
    LaunchScope scope(stream, "fold_nvfp4_kernel");
    fold_nvfp4_kernel<<<grid_for((n + 511) / 512, 8), 256, 0, stream>>>(
        dW, W, V, alpha, n, reinterpret_cast<const unsigned int*>(amax), lr, v_min, v_max, c_min, c_max, dV_out,
        da_out);
  }
  return cudaGetLastError();
}

}  // namespace ar
