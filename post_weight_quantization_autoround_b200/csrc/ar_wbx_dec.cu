// WbA16 matmul at decode batches (T <= 16 tokens) for codes packed at 2, 3 or 8
// bits (the per-row little-endian bit stream of ar_pack_codes); the launcher
// takes any T, 16 tokens at a time:
//   out[t][n] = sum_k A[t][k] (q[n][k] - zero[n][k/g]) scale[n][k/g].
//
// [AR] §4 (comparison table, "Real INT4 Kernel" column): the weights stay
// low-bit in memory and are dequantized inside the kernel; the pages define no
// layout for other widths, so the packing is ar_pack_codes' bit stream ([AR] =
// "Low-Bit Quantization in Practice with vLLM: Core Mechanisms and
// Architectural Optimizations of AutoRound").
//
// One CTA per SM over a contiguous range of weight rows (a multiple of 8) and
// all of K; its 12 warps take the K blocks in turn and add their sums in a
// fixed order through shared memory at the end, so results are deterministic
// and no workspace is needed.  The weights are the B operand of mma.sync
// m16n8k16 (an n8 tile is eight weight rows), the activations the A operand.
//
// A block is the smaller of the group and 128 k.  In a block, lane (g, c) of a
// warp takes the CH = block/4 consecutive codes CH c .. CH c + CH - 1 of weight
// row g; MMA step j of the block feeds that lane's codes 4j .. 4j + 3 into the
// k-slots (2c, 2c+1, 2c+8, 2c+9), so every step stays inside one group and the
// activations it needs are the lane's own consecutive k (no permutes).  A lane
// loads the 32-bit words that hold its CH*BITS bits, funnel-shifts them to bit
// 0 and extracts each code at a compile-time position; (q - zero) is an
// integer of magnitude <= 255, exact in bf16.  Each group's sum is scaled once
// in fp32.
#include <algorithm>

#include "ar_internal.h"

namespace ar {
namespace {

constexpr int kWbxWarps = 12;
constexpr int kWbxThreads = kWbxWarps * 32;
constexpr int kWbxMaxTiles = 8;  // rows per CTA <= 64

struct WbxParams {
  const uint16_t* A;  // bf16 [T][K]
  const uint32_t* packed;  // [N][K*BITS/32]
  const __half* scale;
  const __half* zero;
  uint16_t* out;  // bf16 [T][N], row stride ldo
  int N, K, T, ldo, group_shift, rows_per_cta;
};

__device__ __forceinline__ void wbx_mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// BITS per code, CH codes per lane per block, TB = 8 (T <= 8) or 16 token rows, NT n8 tiles.
template <int BITS, int CH, int TB, int NT>
__global__ void __launch_bounds__(kWbxThreads, 1) wbx_dec_kernel(const WbxParams p) {
  constexpr int kBlock = 4 * CH;                 // k per block
  constexpr int kLaneBits = CH * BITS;           // bits per lane per block
  // a lane's bits start on a word boundary when CH*BITS is a multiple of 32; else
  // one more word covers any start offset, plus one for the funnel shift
  constexpr bool kAligned = kLaneBits % 32 == 0;
  constexpr int kWords = kAligned ? kLaneBits / 32 : kLaneBits / 32 + 2;  // words loaded
  constexpr int kUsed = kAligned ? kWords : kWords - 1;                    // words after the shift
  constexpr int kSteps = CH / 4;                 // MMA k16 steps per block
  extern __shared__ float wbx_red[];  // [warp][64 rows][TB tokens]
  auto red = [&](int w, int r, int t) -> float& { return wbx_red[(w * kWbxMaxTiles * 8 + r) * TB + t]; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  const int row0 = blockIdx.x * p.rows_per_cta;
  const int n_blocks = p.K / kBlock;
  const int64_t row_words = static_cast<int64_t>(p.K) * BITS / 32;
  const int tok_lo = min(g, p.T - 1);
  const int tok_hi = min(g + 8, p.T - 1);

  float acc[NT][4];
#pragma unroll
  for (int i = 0; i < NT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  bool bad = false;

  for (int blk = warp; blk < n_blocks; blk += kWbxWarps) {
    // activations: token g (and g + 8) at this lane's CH consecutive k
    const int kbase = blk * kBlock + CH * c;
    uint32_t alo[CH / 2], ahi[CH / 2];
#pragma unroll
    for (int i = 0; i < CH / 8; ++i) {
      const uint4 v = *reinterpret_cast<const uint4*>(p.A + static_cast<int64_t>(tok_lo) * p.K + kbase + 8 * i);
      alo[4 * i] = v.x;
      alo[4 * i + 1] = v.y;
      alo[4 * i + 2] = v.z;
      alo[4 * i + 3] = v.w;
      if (TB == 16) {
        const uint4 u = *reinterpret_cast<const uint4*>(p.A + static_cast<int64_t>(tok_hi) * p.K + kbase + 8 * i);
        ahi[4 * i] = u.x;
        ahi[4 * i + 1] = u.y;
        ahi[4 * i + 2] = u.z;
        ahi[4 * i + 3] = u.w;
      } else {
        ahi[4 * i] = ahi[4 * i + 1] = ahi[4 * i + 2] = ahi[4 * i + 3] = 0u;
      }
    }
    // this lane's bits of row g of every tile: words from bit offset blk*4*CH*BITS + c*CH*BITS
    const int64_t bit0 = static_cast<int64_t>(blk) * kBlock * BITS + static_cast<int64_t>(c) * kLaneBits;
    const int64_t w0 = bit0 >> 5;
    const int sh = static_cast<int>(bit0 & 31);
    const int grp = (blk * kBlock) >> p.group_shift;
    uint32_t wd[NT][kWords];
#pragma unroll
    for (int jt = 0; jt < NT; ++jt) {
      const int row = min(row0 + 8 * jt + g, p.N - 1);
      const uint32_t* src = p.packed + static_cast<int64_t>(row) * row_words + w0;
#pragma unroll
      for (int w = 0; w < kWords; ++w) wd[jt][w] = (w0 + w < row_words) ? src[w] : 0u;
    }
#pragma unroll
    for (int jt = 0; jt < NT; ++jt) {
      const int row = min(row0 + 8 * jt + g, p.N - 1);
      const float z = __half2float(p.zero[static_cast<int64_t>(row) * (p.K >> p.group_shift) + grp]);
      // the lane's bit stream shifted to bit 0
      uint32_t u[kUsed];
#pragma unroll
      for (int w = 0; w < kUsed; ++w) u[w] = kAligned ? wd[jt][w] : __funnelshift_r(wd[jt][w], wd[jt][w + 1], sh);
      float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < kSteps; ++j) {
        float qz[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          constexpr uint32_t mask = (1u << BITS) - 1u;
          const int pos = (4 * j + e) * BITS;  // compile-time
          uint32_t q;
          if ((pos & 31) + BITS <= 32) q = (u[pos >> 5] >> (pos & 31)) & mask;
          else q = __funnelshift_r(u[pos >> 5], u[(pos >> 5) + 1], pos & 31) & mask;
          qz[e] = __fsub_rn(static_cast<float>(q), z);
        }
        const uint32_t a[4] = {alo[2 * j], ahi[2 * j], alo[2 * j + 1], ahi[2 * j + 1]};
        wbx_mma(d, a, pack_bf16x2(qz[0], qz[1]), pack_bf16x2(qz[2], qz[3]));
      }
      // scale of rows 2c, 2c+1 of the tile (the columns of this lane's accumulators)
      const int r0 = min(row0 + 8 * jt + 2 * c, p.N - 1), r1 = min(row0 + 8 * jt + 2 * c + 1, p.N - 1);
      const int gpr = p.K >> p.group_shift;
      const float s0 = __half2float(p.scale[static_cast<int64_t>(r0) * gpr + grp]);
      const float s1 = __half2float(p.scale[static_cast<int64_t>(r1) * gpr + grp]);
      acc[jt][0] = fmaf(s0, d[0], acc[jt][0]);
      acc[jt][1] = fmaf(s1, d[1], acc[jt][1]);
      acc[jt][2] = fmaf(s0, d[2], acc[jt][2]);
      acc[jt][3] = fmaf(s1, d[3], acc[jt][3]);
    }
  }
  // fixed-order sum over the warps
#pragma unroll
  for (int jt = 0; jt < NT; ++jt) {
    red(warp, 8 * jt + 2 * c, g) = acc[jt][0];
    red(warp, 8 * jt + 2 * c + 1, g) = acc[jt][1];
    if (TB == 16) {
      red(warp, 8 * jt + 2 * c, (g + 8) % TB) = acc[jt][2];
      red(warp, 8 * jt + 2 * c + 1, (g + 8) % TB) = acc[jt][3];
    }
  }
  __syncthreads();
  const int rows_here = min(p.rows_per_cta, p.N - row0);
  for (int e = threadIdx.x; e < p.T * rows_here; e += kWbxThreads) {
    const int t = e / rows_here;
    const int r = e - t * rows_here;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kWbxWarps; ++w) v += red(w, r, t);
    bad |= !isfinite(v);
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    p.out[static_cast<int64_t>(t) * p.ldo + row0 + r] = *reinterpret_cast<const uint16_t*>(&h);
  }
  if (bad) raise_status(kStatusNonFinite);
}

const char* wbx_name(int bits, int tb) {
  static const char* names[3][2] = {{"wbx_dec_kernel<b=2,T<=8>", "wbx_dec_kernel<b=2,T<=16>"},
                                    {"wbx_dec_kernel<b=3,T<=8>", "wbx_dec_kernel<b=3,T<=16>"},
                                    {"wbx_dec_kernel<b=8,T<=8>", "wbx_dec_kernel<b=8,T<=16>"}};
  return names[bits == 2 ? 0 : (bits == 3 ? 1 : 2)][tb == 16 ? 1 : 0];
}

template <int BITS, int CH, int TB, int NT>
cudaError_t wbx_launch_one(const WbxParams& p, int grid, cudaStream_t st) {
  constexpr int smem = kWbxWarps * kWbxMaxTiles * 8 * TB * 4;
  auto k = wbx_dec_kernel<BITS, CH, TB, NT>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  LaunchScope scope(st, wbx_name(BITS, TB));
  k<<<grid, kWbxThreads, smem, st>>>(p);
  return cudaGetLastError();
}

template <int BITS, int CH, int TB>
cudaError_t wbx_launch_nt(int nt, const WbxParams& p, int grid, cudaStream_t st) {
  switch (nt) {
    case 1: return wbx_launch_one<BITS, CH, TB, 1>(p, grid, st);
    case 2: return wbx_launch_one<BITS, CH, TB, 2>(p, grid, st);
    case 3: return wbx_launch_one<BITS, CH, TB, 3>(p, grid, st);
    case 4: return wbx_launch_one<BITS, CH, TB, 4>(p, grid, st);
    case 5: return wbx_launch_one<BITS, CH, TB, 5>(p, grid, st);
    case 6: return wbx_launch_one<BITS, CH, TB, 6>(p, grid, st);
    case 7: return wbx_launch_one<BITS, CH, TB, 7>(p, grid, st);
    default: return wbx_launch_one<BITS, CH, TB, 8>(p, grid, st);
  }
}

template <int BITS>
cudaError_t wbx_launch_bits(int ch, int tb, int nt, const WbxParams& p, int grid, cudaStream_t st) {
  if (ch == 8) return tb == 16 ? wbx_launch_nt<BITS, 8, 16>(nt, p, grid, st) : wbx_launch_nt<BITS, 8, 8>(nt, p, grid, st);
  if (ch == 16)
    return tb == 16 ? wbx_launch_nt<BITS, 16, 16>(nt, p, grid, st) : wbx_launch_nt<BITS, 16, 8>(nt, p, grid, st);
  return tb == 16 ? wbx_launch_nt<BITS, 32, 16>(nt, p, grid, st) : wbx_launch_nt<BITS, 32, 8>(nt, p, grid, st);
}

}  // namespace

// bits 2, 3 or 8; group_size a power of two >= 32 dividing K; K % 128 == 0;
// T >= 1 (chunks of 16 tokens).
cudaError_t launch_wbx_dec(const uint16_t* A, int T, const uint32_t* packed, const uint16_t* scale16,
                           const uint16_t* zero16, int N, int K, int group_size, int bits, uint16_t* out,
                           cudaStream_t stream) {
  if (bits != 2 && bits != 3 && bits != 8) return cudaErrorInvalidValue;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  int gs = 0;
  while ((1 << gs) < group_size) ++gs;
  const int ch = group_size >= 128 ? 32 : group_size / 4;
  // rows per CTA: a multiple of 8 with one CTA per SM, at most 64
  const int units = (N + 7) / 8;
  const int nt = std::min(kWbxMaxTiles, std::max(1, (units + sms - 1) / sms));
  const int rows = 8 * nt;
  const int grid = (N + rows - 1) / rows;
  for (int t0 = 0; t0 < T; t0 += 16) {
    WbxParams p{};
    p.A = A + static_cast<int64_t>(t0) * K;
    p.packed = packed;
    p.scale = reinterpret_cast<const __half*>(scale16);
    p.zero = reinterpret_cast<const __half*>(zero16);
    p.out = out + static_cast<int64_t>(t0) * N;
    p.N = N;
    p.K = K;
    p.T = std::min(16, T - t0);
    p.ldo = N;
    p.group_shift = gs;
    p.rows_per_cta = rows;
    const int tb = p.T > 8 ? 16 : 8;
    if (bits == 2) e = wbx_launch_bits<2>(ch, tb, nt, p, grid, stream);
    else if (bits == 3) e = wbx_launch_bits<3>(ch, tb, nt, p, grid, stream);
    else e = wbx_launch_bits<8>(ch, tb, nt, p, grid, stream);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace ar
