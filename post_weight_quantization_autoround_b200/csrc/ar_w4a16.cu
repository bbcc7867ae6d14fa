// W4A16 matmul for decode-shaped batches: out[t][n] = sum_k A[t][k] (q[n][k] - z) s.
//
// [AR] §4 (comparison table, "Real INT4 Kernel" column): the weights stay
// 4-bit in memory and are dequantized inside the kernel; activations are
// 16-bit ([AR] = "Low-Bit Quantization in Practice with vLLM: Core Mechanisms
// and Architectural Optimizations of AutoRound").
//
// HBM-bound for T <= 16 (0.5 byte per weight plus 4 bytes of metadata per
// group).  One warp owns one output row at a time; each lane streams 16-byte
// words of packed codes (32 codes, always inside one group because g >= 32)
// so that a warp reads 512 contiguous bytes per step.  The code is turned
// into (q - z) exactly in fp32 with the 2^23 mantissa trick, and the group
// scale multiplies the per-chunk dot product once:
//   acc_t += s * sum_i a_t,i (q_i - z).
#include "ar_internal.h"

namespace ar {
namespace {

template <int T>
__global__ void __launch_bounds__(256) w4a16_kernel(const uint16_t* __restrict__ A, const uint32_t* __restrict__ packed,
                                                    const __half* __restrict__ scale16,
                                                    const __half* __restrict__ zero16, int N, int K, int group_shift,
                                                    int t_valid, uint16_t* __restrict__ out) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int chunks = K >> 5;  // 32 codes per 16-byte word group
  const int groups_per_row = K >> group_shift;
  for (int n = blockIdx.x * 8 + warp; n < N; n += gridDim.x * 8) {
    float acc[T];
#pragma unroll
    for (int t = 0; t < T; ++t) acc[t] = 0.0f;
    const uint4* wrow = reinterpret_cast<const uint4*>(packed + static_cast<size_t>(n) * (K >> 3));
    for (int c = lane; c < chunks; c += 32) {
      const uint4 wv = __ldcs(wrow + c);
      const int gi = (c << 5) >> group_shift;
      const float s = __half2float(scale16[static_cast<size_t>(n) * groups_per_row + gi]);
      const float z = __half2float(zero16[static_cast<size_t>(n) * groups_per_row + gi]);
      const float bias = 8388608.0f + z;  // (2^23 + q) - (2^23 + z) = q - z exactly
      float d[32];
      const uint32_t ws[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t nib = (ws[j] >> (4 * i)) & 0xFu;
          d[8 * j + i] = __uint_as_float(0x4B000000u | nib) - bias;
        }
      }
#pragma unroll
      for (int t = 0; t < T; ++t) {
        if (t < t_valid) {
          const uint4* ap = reinterpret_cast<const uint4*>(A + static_cast<size_t>(t) * K + (c << 5));
          float dot = 0.0f;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 av = __ldg(ap + j);
            const uint32_t as[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              dot = fmaf(bf16_lo(as[i]), d[8 * j + 2 * i], dot);
              dot = fmaf(bf16_hi(as[i]), d[8 * j + 2 * i + 1], dot);
            }
          }
          acc[t] = fmaf(s, dot, acc[t]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < T; ++t) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc[t] += __shfl_xor_sync(0xFFFFFFFFu, acc[t], off);
    }
    if (lane == 0) {
#pragma unroll
      for (int t = 0; t < T; ++t) {
        if (t < t_valid) {
          __nv_bfloat16 h = __float2bfloat16_rn(acc[t]);
          out[static_cast<size_t>(t) * N + n] = *reinterpret_cast<uint16_t*>(&h);
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_w4a16(const uint16_t* A, int T, const uint32_t* packed, const uint16_t* scale16,
                         const uint16_t* zero16, int N, int K, int group_size, uint16_t* out, cudaStream_t stream) {
  int group_shift = 0;
  while ((1 << group_shift) < group_size) ++group_shift;
  const int rows_per_block = 8;
  int blocks = (N + rows_per_block - 1) / rows_per_block;
  const int cap = num_sms() * 8;
  if (blocks > cap) blocks = cap;
  const __half* s16 = reinterpret_cast<const __half*>(scale16);
  const __half* z16 = reinterpret_cast<const __half*>(zero16);
#define AR_W4_CASE(TT)                                                                                 \
  {                                                                                                    \
    LaunchScope scope(stream, "w4a16_kernel<T=" #TT ">");                                              \
    w4a16_kernel<TT><<<blocks, 256, 0, stream>>>(A, packed, s16, z16, N, K, group_shift, T, out);     \
  }
  if (T <= 1) {
    AR_W4_CASE(1)
  } else if (T <= 2) {
    AR_W4_CASE(2)
  } else if (T <= 4) {
    AR_W4_CASE(4)
  } else if (T <= 8) {
    AR_W4_CASE(8)
  } else {
    AR_W4_CASE(16)
  }
#undef AR_W4_CASE
  return cudaGetLastError();
}

}  // namespace ar
