// Group-wise fake quantization (QDQ), INT4 packing and fp32->bf16 conversion.
//
// QDQ follows [AR] §4 ("QDQ / Fake Quantization" column of the comparison
// table) and the worked examples of [AR] §2 and §4: per group of g weights
// along in_features, with the range always containing zero,
//   hi = alpha*max(0, max W), lo = beta*min(0, min W), s = (hi-lo)/(2^b-1),
//   zp = round(-lo/s), q = clamp(round(W/s + V) + zp, 0, 2^b-1), W_hat = s*(q-zp).
// ([AR] = "Low-Bit Quantization in Practice with vLLM: Core Mechanisms and
// Architectural Optimizations of AutoRound".)
//
// Every operation is an explicit IEEE fp32 intrinsic (no FMA contraction) so
// that the integer codes are a pure function of (W, V, alpha, beta).
//
// Layout: one group is handled by TPG = min(g/8, 32) consecutive threads of
// a warp; each thread owns 8 consecutive weights per chunk (one 16-byte load
// of bf16 W, two 16-byte loads of fp32 V) and g/(8*TPG) chunks.  The group's
// min/max are reduced with xor-shuffles inside the TPG lanes.
#include "ar_fold.cuh"
#include "ar_internal.h"

namespace ar {

__device__ unsigned int g_status = 0;

cudaError_t read_and_clear_status(unsigned int* out, cudaStream_t stream) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  e = cudaMemcpyFromSymbol(out, g_status, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  const unsigned int zero = 0;
  return cudaMemcpyToSymbol(g_status, &zero, sizeof(unsigned int));
}

// Diagnostic: one warp waits on an mbarrier that nothing arrives on, with a
// limit of `limit_ns`; the bounded wait gives up, raises the timeout status
// and the kernel returns normally.
__global__ void wait_timeout_kernel(uint64_t limit_ns, int* gave_up) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  const uint32_t addr = smem_u32(&bar);
  const uint64_t t0 = globaltimer_ns();
  bool done = false;
  while (!done) {
    if (mbar_try_wait(addr, 0)) break;
    if (globaltimer_ns() - t0 > limit_ns) {
      done = true;
      if (threadIdx.x == 0) {
        raise_status(kStatusTimeout);
        *gave_up = 1;
      }
    }
  }
}

cudaError_t launch_wait_timeout(uint64_t limit_ns, int* gave_up, cudaStream_t stream) {
  LaunchScope scope(stream, "wait_timeout_kernel");
  wait_timeout_kernel<<<1, 32, 0, stream>>>(limit_ns, gave_up);
  return cudaGetLastError();
}

template <int TPG, int CHUNKS>
__global__ void __launch_bounds__(256) qdq_kernel(const uint16_t* __restrict__ W, const float* __restrict__ V,
                                                  const float* __restrict__ alpha, const float* __restrict__ beta,
                                                  int64_t n_groups, int groups_per_row, int bits, int symmetric,
                                                  uint16_t* __restrict__ W_hat, uint8_t* __restrict__ codes,
                                                  float* __restrict__ scale_out, float* __restrict__ zero_out,
                                                  float* __restrict__ mx_out, float* __restrict__ mn_out) {
  constexpr int G = TPG * 8 * CHUNKS;  // group size
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t grp = tid / TPG;
  const int li = static_cast<int>(tid % TPG);
  const bool active = grp < n_groups;
  const int64_t gbase = (active ? grp : 0) * static_cast<int64_t>(G);  // element offset of the group

  // Every load is issued before the group reduction, so the V, alpha and beta
  // round trips overlap the W one instead of following it.
  uint4 wv[CHUNKS];
  float4 v0[CHUNKS], v1[CHUNKS];
#pragma unroll
  for (int c = 0; c < CHUNKS; ++c) {
    const int64_t e = gbase + (static_cast<int64_t>(c) * TPG + li) * 8;
    wv[c] = active ? __ldcs(reinterpret_cast<const uint4*>(W + e)) : make_uint4(0, 0, 0, 0);
    v0[c] = active ? __ldcs(reinterpret_cast<const float4*>(V + e)) : make_float4(0.f, 0.f, 0.f, 0.f);
    v1[c] = active ? __ldcs(reinterpret_cast<const float4*>(V + e + 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const float ga = active ? alpha[grp] : 1.0f;
  const float gb = active ? beta[grp] : 1.0f;
  float lmax = -INFINITY, lmin = INFINITY;
  bool bad = false;
#pragma unroll
  for (int c = 0; c < CHUNKS; ++c) {
    const uint32_t wr[4] = {wv[c].x, wv[c].y, wv[c].z, wv[c].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float a = bf16_lo(wr[i]), b = bf16_hi(wr[i]);
      lmax = fmaxf(lmax, fmaxf(a, b));
      lmin = fminf(lmin, fminf(a, b));
      bad |= !isfinite(a) || !isfinite(b);
    }
  }
#pragma unroll
  for (int off = TPG / 2; off > 0; off >>= 1) {
    lmax = fmaxf(lmax, __shfl_xor_sync(0xFFFFFFFFu, lmax, off));
    lmin = fminf(lmin, __shfl_xor_sync(0xFFFFFFFFu, lmin, off));
  }
  if (!active) return;
  if (bad) raise_status(kStatusNonFinite);

  const float mx = fmaxf(lmax, 0.0f);
  const float mn = fminf(lmin, 0.0f);
  const QParams p = group_qparams(mx, mn, ga, gb, bits, symmetric);
  const float Q = static_cast<float>((1 << bits) - 1);

#pragma unroll
  for (int c = 0; c < CHUNKS; ++c) {
    const int64_t e = gbase + (static_cast<int64_t>(c) * TPG + li) * 8;
    const float vv[8] = {v0[c].x, v0[c].y, v0[c].z, v0[c].w, v1[c].x, v1[c].y, v1[c].z, v1[c].w};
    const uint32_t wr[4] = {wv[c].x, wv[c].y, wv[c].z, wv[c].w};
    float wh[8];
    uint32_t qb[2] = {0, 0};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float w = (i & 1) ? bf16_hi(wr[i >> 1]) : bf16_lo(wr[i >> 1]);
      float q;
      wh[i] = qdq_elem(w, vv[i], p, Q, q);
      qb[i >> 2] |= static_cast<uint32_t>(q) << (8 * (i & 3));
    }
    if (W_hat) {
      uint4 o;
      o.x = pack_bf16x2(wh[0], wh[1]);
      o.y = pack_bf16x2(wh[2], wh[3]);
      o.z = pack_bf16x2(wh[4], wh[5]);
      o.w = pack_bf16x2(wh[6], wh[7]);
      *reinterpret_cast<uint4*>(W_hat + e) = o;
    }
    if (codes) *reinterpret_cast<uint2*>(codes + e) = make_uint2(qb[0], qb[1]);
  }
  if (li == 0) {
    if (scale_out) scale_out[grp] = p.s;
    if (zero_out) zero_out[grp] = p.zp;
    if (mx_out) mx_out[grp] = p.mx;
    if (mn_out) mn_out[grp] = p.mn;
  }
  (void)groups_per_row;
}

// Packed export: the same codes as qdq_kernel, BITS (2, 3, 4 or 8) bits each, as
// one little-endian bit stream per row: element k at stream bits [BITS k,
// BITS k + BITS), stream bit i in bit i mod 32 of word i / 32 (2, 4, 8 bits:
// element k at bits BITS*(k mod 32/BITS) of word k/(32/BITS); INT4: nibbles;
// 3 bits: 32 codes in 3 words, codes 10 and 21 straddling two), plus fp16
// scale / zero per group.  A thread's 8 codes fill BITS whole bytes.
template <int TPG, int CHUNKS, int BITS>
__global__ void __launch_bounds__(256) pack_codes_kernel(const uint16_t* __restrict__ W, const float* __restrict__ V,
                                                         const float* __restrict__ alpha,
                                                         const float* __restrict__ beta, int64_t n_groups,
                                                         int symmetric, uint8_t* __restrict__ packed,
                                                         __half* __restrict__ scale16, __half* __restrict__ zero16) {
  constexpr int G = TPG * 8 * CHUNKS;
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t grp = tid / TPG;
  const int li = static_cast<int>(tid % TPG);
  const bool active = grp < n_groups;
  const int64_t gbase = (active ? grp : 0) * static_cast<int64_t>(G);

  uint4 wv[CHUNKS];
  float lmax = -INFINITY, lmin = INFINITY;
  bool bad = false;
#pragma unroll
  for (int c = 0; c < CHUNKS; ++c) {
    const int64_t e = gbase + (static_cast<int64_t>(c) * TPG + li) * 8;
    wv[c] = active ? *reinterpret_cast<const uint4*>(W + e) : make_uint4(0, 0, 0, 0);
    const uint32_t wr[4] = {wv[c].x, wv[c].y, wv[c].z, wv[c].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float a = bf16_lo(wr[i]), b = bf16_hi(wr[i]);
      lmax = fmaxf(lmax, fmaxf(a, b));
      lmin = fminf(lmin, fminf(a, b));
      bad |= !isfinite(a) || !isfinite(b);
    }
  }
#pragma unroll
  for (int off = TPG / 2; off > 0; off >>= 1) {
    lmax = fmaxf(lmax, __shfl_xor_sync(0xFFFFFFFFu, lmax, off));
    lmin = fminf(lmin, __shfl_xor_sync(0xFFFFFFFFu, lmin, off));
  }
  if (!active) return;
  if (bad) raise_status(kStatusNonFinite);
  const QParams p = group_qparams(fmaxf(lmax, 0.0f), fminf(lmin, 0.0f), alpha[grp], beta[grp], BITS, symmetric);
  constexpr float Q = static_cast<float>((1 << BITS) - 1);

#pragma unroll
  for (int c = 0; c < CHUNKS; ++c) {
    const int64_t e = gbase + (static_cast<int64_t>(c) * TPG + li) * 8;
    const float4 v0 = *reinterpret_cast<const float4*>(V + e);
    const float4 v1 = *reinterpret_cast<const float4*>(V + e + 4);
    const float vv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    const uint32_t wr[4] = {wv[c].x, wv[c].y, wv[c].z, wv[c].w};
    uint64_t bits = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float w = (i & 1) ? bf16_hi(wr[i >> 1]) : bf16_lo(wr[i >> 1]);
      float q;
      (void)qdq_elem(w, vv[i], p, Q, q);
      bits |= static_cast<uint64_t>(q) << (BITS * i);
    }
    uint8_t* dst = packed + (e * BITS) / 8;
    if (BITS == 2) {
      *reinterpret_cast<uint16_t*>(dst) = static_cast<uint16_t>(bits);
    } else if (BITS == 3) {  // 24 bits at byte offset 3 (e / 8): three byte stores
      dst[0] = static_cast<uint8_t>(bits);
      dst[1] = static_cast<uint8_t>(bits >> 8);
      dst[2] = static_cast<uint8_t>(bits >> 16);
    } else if (BITS == 4) {
      *reinterpret_cast<uint32_t*>(dst) = static_cast<uint32_t>(bits);
    } else {
      *reinterpret_cast<uint2*>(dst) = make_uint2(static_cast<uint32_t>(bits), static_cast<uint32_t>(bits >> 32));
    }
  }
  if (li == 0) {
    scale16[grp] = __float2half_rn(p.s);
    zero16[grp] = __float2half_rn(p.zp);
  }
}

__global__ void f32_to_bf16_kernel(const float* __restrict__ src, uint16_t* __restrict__ dst, int64_t n) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x * 4;
  for (int64_t i = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 4; i < n; i += stride) {
    if (i + 4 <= n && (reinterpret_cast<uintptr_t>(src + i) & 15) == 0) {
      const float4 v = *reinterpret_cast<const float4*>(src + i);
      uint2 o;
      o.x = pack_bf16x2(v.x, v.y);
      o.y = pack_bf16x2(v.z, v.w);
      *reinterpret_cast<uint2*>(dst + i) = o;
    } else {
      for (int64_t j = i; j < n && j < i + 4; ++j) {
        __nv_bfloat16 h = __float2bfloat16_rn(src[j]);
        dst[j] = *reinterpret_cast<uint16_t*>(&h);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// host launchers
// ---------------------------------------------------------------------------
#define AR_QDQ_CASE(TPG_, CH_)                                                                                  \
  case (TPG_ * 8 * CH_): {                                                                                      \
    const int64_t threads = n_groups * TPG_;                                                                    \
    const int blocks = static_cast<int>((threads + 255) / 256);                                                 \
    LaunchScope scope(stream, "qdq_kernel<g=" #TPG_ "x8x" #CH_ ">");                                           \
    qdq_kernel<TPG_, CH_><<<blocks, 256, 0, stream>>>(W, V, alpha, beta, n_groups, groups_per_row, bits,      \
                                                      symmetric, W_hat, codes, scale, zero, mx, mn);           \
    break;                                                                                                      \
  }

cudaError_t launch_qdq(const uint16_t* W, const float* V, const float* alpha, const float* beta, int64_t N,
                       int64_t K, int group_size, int bits, int symmetric, uint16_t* W_hat, uint8_t* codes,
                       float* scale, float* zero, float* mx, float* mn, cudaStream_t stream) {
  const int64_t n_groups = N * (K / group_size);
  const int groups_per_row = static_cast<int>(K / group_size);
  switch (group_size) {
    // two 8-element chunks per thread from g = 16 up: twice the loads in flight
    // per thread at the same occupancy (HBM latency needs ~44 KB in flight per SM)
    AR_QDQ_CASE(1, 1)
    AR_QDQ_CASE(1, 2)
    AR_QDQ_CASE(2, 2)
    AR_QDQ_CASE(4, 2)
    AR_QDQ_CASE(8, 2)
    AR_QDQ_CASE(16, 2)
    AR_QDQ_CASE(32, 2)
    AR_QDQ_CASE(32, 4)
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}
#undef AR_QDQ_CASE

template <int BITS>
cudaError_t launch_pack_bits(const uint16_t* W, const float* V, const float* alpha, const float* beta, int64_t N,
                             int64_t K, int group_size, int symmetric, uint8_t* packed, uint16_t* scale16,
                             uint16_t* zero16, cudaStream_t stream) {
  const int64_t n_groups = N * (K / group_size);
  __half* s16 = reinterpret_cast<__half*>(scale16);
  __half* z16 = reinterpret_cast<__half*>(zero16);
#define AR_PACK_CASE(TPG_, CH_)                                                                               \
  case (TPG_ * 8 * CH_): {                                                                                    \
    const int64_t threads = n_groups * TPG_;                                                                  \
    const int blocks = static_cast<int>((threads + 255) / 256);                                               \
    LaunchScope scope(stream, BITS == 4   ? "pack_codes_kernel<b=4,g=" #TPG_ "x8x" #CH_ ">"                    \
                              : BITS == 2 ? "pack_codes_kernel<b=2,g=" #TPG_ "x8x" #CH_ ">"                    \
                              : BITS == 3 ? "pack_codes_kernel<b=3,g=" #TPG_ "x8x" #CH_ ">"                    \
                                          : "pack_codes_kernel<b=8,g=" #TPG_ "x8x" #CH_ ">");                  \
    pack_codes_kernel<TPG_, CH_, BITS><<<blocks, 256, 0, stream>>>(W, V, alpha, beta, n_groups, symmetric,    \
                                                                   packed, s16, z16);                         \
    break;                                                                                                    \
  }
  switch (group_size) {
    AR_PACK_CASE(1, 1)
    AR_PACK_CASE(2, 1)
    AR_PACK_CASE(4, 1)
    AR_PACK_CASE(8, 1)
    AR_PACK_CASE(16, 1)
    AR_PACK_CASE(32, 1)
    AR_PACK_CASE(32, 2)
    AR_PACK_CASE(32, 4)
    default:
      return cudaErrorInvalidValue;
  }
#undef AR_PACK_CASE
  return cudaGetLastError();
}

cudaError_t launch_pack_int4(const uint16_t* W, const float* V, const float* alpha, const float* beta, int64_t N,
                             int64_t K, int group_size, int symmetric, uint32_t* packed, uint16_t* scale16,
                             uint16_t* zero16, cudaStream_t stream) {
  return launch_pack_bits<4>(W, V, alpha, beta, N, K, group_size, symmetric, reinterpret_cast<uint8_t*>(packed),
                             scale16, zero16, stream);
}

cudaError_t launch_pack_codes(const uint16_t* W, const float* V, const float* alpha, const float* beta, int64_t N,
                              int64_t K, int group_size, int bits, int symmetric, uint32_t* packed,
                              uint16_t* scale16, uint16_t* zero16, cudaStream_t stream) {
  uint8_t* dst = reinterpret_cast<uint8_t*>(packed);
  if (bits == 2) return launch_pack_bits<2>(W, V, alpha, beta, N, K, group_size, symmetric, dst, scale16, zero16, stream);
  if (bits == 3) return launch_pack_bits<3>(W, V, alpha, beta, N, K, group_size, symmetric, dst, scale16, zero16, stream);
  if (bits == 4) return launch_pack_bits<4>(W, V, alpha, beta, N, K, group_size, symmetric, dst, scale16, zero16, stream);
  if (bits == 8) return launch_pack_bits<8>(W, V, alpha, beta, N, K, group_size, symmetric, dst, scale16, zero16, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_f32_to_bf16(const float* src, uint16_t* dst, int64_t n, cudaStream_t stream) {
  const int64_t vec = (n + 3) / 4;
  int blocks = static_cast<int>((vec + 255) / 256);
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  {
    LaunchScope scope(stream, "f32_to_bf16_kernel");
    f32_to_bf16_kernel<<<blocks, 256, 0, stream>>>(src, dst, n);
  }
  return cudaGetLastError();
}

}  // namespace ar
