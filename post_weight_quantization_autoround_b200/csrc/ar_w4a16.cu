// W4A16 matmul for decode-shaped batches: out[t][n] = sum_k A[t][k] (q[n][k] - z) s.
//
// [AR] §4 (comparison table, "Real INT4 Kernel" column): the weights stay
// 4-bit in memory and are dequantized inside the kernel; activations are
// 16-bit ([AR] = "Low-Bit Quantization in Practice with vLLM: Core Mechanisms
// and Architectural Optimizations of AutoRound").
//
// For T <= 16 tokens the kernel is bound by HBM (0.5 byte per weight), and a
// CUDA-core dot product would spend ~3 instructions per weight and token.
// Here the dequantized weights go straight from registers into tensor-core
// fragments (mma.sync m16n8k16, bf16 in, fp32 out), so a weight costs about
// 1.5 instructions whatever T is:
//
//  * Codes -> bf16 without arithmetic: (word >> 4i) & 0x000F000F | 0x43004300
//    is the exact bf16 pair (128 + q_i, 128 + q_{i+4}).  The MMA sums
//    D = sum (128 + q) a; one extra MMA against a fragment of ones gives
//    O = sum a over the same k (shared by all 64 rows), and the zero-point is
//    applied once per group span: sum (q - z) a = D - (128 + z) O.
//  * The reduction index of the MMA is permuted: lane (g = lane/4, c = lane%4)
//    feeds k-slots {2c, 2c+1, 2c+8, 2c+9} of two consecutive MMAs from one
//    32-bit word (8 codes, k = 32j + 8c + 0..7) of each of its two rows, and
//    the activations are permuted the same way with byte permutes.  Each
//    32-k slice j lies inside one quantization group (g >= 32), so each
//    group span's fp32 partial is scaled once: acc += s * (D - (128 + z) O).
//  * A CTA owns 64 rows (four 16-row MMA tiles) and half of K; one warp
//    streams the packed weights into a 4-stage shared-memory ring with TMA
//    (64 rows x 512 k per stage, 128-byte swizzle so that the fragment reads
//    are free of bank conflicts) and 8 warps consume it, so memory latency is
//    hidden by the ring rather than by registers.  The two CTAs of a cluster
//    cover all of K and their partial sums are added in a fixed order through
//    distributed shared memory: no workspace, deterministic results.
//
// Packed layout (as ar_pack_int4 writes it): uint32 [N][K/8], element k at
// bits 4*(k mod 8) of word k/8; scale/zero fp16 [N][K/g].
#include <cooperative_groups.h>

#include "ar_internal.h"

namespace cg = cooperative_groups;

namespace ar {
namespace {

constexpr int kRows = 64;      // rows of W per CTA
constexpr int kSplit = 2;      // CTAs per cluster, each half of K
constexpr int kWarps = 8;
constexpr int kChunk = 128;    // k per warp iteration (four 32-k slices)

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Shared memory of one CTA: a ring of stages, each holding
//   * the weight tile: 64 rows x 64 words (512 k), two 64 x 32-word TMA boxes
//     with 128-byte swizzle (16-byte chunk q of row p sits at chunk q ^ (p % 8)),
//   * the activation tile: 8*TH tokens x 512 k bf16 (two TMA boxes, rows past T
//     are zero-filled),
// plus the reduction buffers and, loaded once per CTA, the fp16 (scale, zero)
// of its 64 rows over its half of K.
constexpr int kWBoxBytes = kRows * 32 * 4;        // 8 KiB
constexpr int kThreadsW4 = (kWarps + 1) * 32;     // 8 consumer warps + 1 producer warp

template <int TH>
struct W4Cfg {
  static constexpr int kStages = TH == 1 ? 3 : 4;
  static constexpr int kABoxBytes = 8 * TH * 256 * 2;  // 8*TH tokens x 256 k
};

template <int TH>
struct alignas(1024) W4Stage {
  uint8_t w[2 * kWBoxBytes];
  uint8_t a[2 * W4Cfg<TH>::kABoxBytes];
};

template <int TH>
struct W4Smem {
  W4Stage<TH> stage[W4Cfg<TH>::kStages];
  uint64_t full[W4Cfg<TH>::kStages];
  uint64_t empty[W4Cfg<TH>::kStages];
  float part[kRows][16];
  int abort_flag;
  // followed by the CTA's scales and zeros: __half2 (scale, zero) [kRows][max_groups]
};

template <int TH>
int w4_smem_bytes(int max_groups) {
  return static_cast<int>(sizeof(W4Smem<TH>)) + 1024 + kRows * max_groups * 4;
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
               : "memory");
  return v;
}

// TH: token halves of 8 (1 for T <= 8, 2 for T <= 16).  GROUP_CHUNK: the
// group size is >= 128, so one (scale, zero) serves a whole 128-k chunk.
template <int TH, bool GROUP_CHUNK>
__global__ void __cluster_dims__(kSplit, 1, 1) __launch_bounds__(kThreadsW4, 1)
    w4a16_tma_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmA, int T,
                     const __half* __restrict__ scale16, const __half* __restrict__ zero16, int N, int K,
                     int group_shift, int max_groups, uint16_t* __restrict__ out) {
  constexpr int S = W4Cfg<TH>::kStages;
  constexpr int kABox = W4Cfg<TH>::kABoxBytes;
  extern __shared__ uint8_t smem_raw[];
  W4Smem<TH>& sm = *reinterpret_cast<W4Smem<TH>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  volatile int* abort_flag = &sm.abort_flag;
  static_assert(sizeof(sm.stage) >= sizeof(float) * kWarps * 4 * TH * 4 * 32, "reduction buffer must fit the ring");

  cg::cluster_group cluster = cg::this_cluster();
  const int split = static_cast<int>(cluster.block_rank());
  const int row0 = (blockIdx.x / kSplit) * kRows;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int chunks = K / kChunk;
  const int ch_begin = (chunks * split) / kSplit;
  const int ch_end = (chunks * (split + 1)) / kSplit;
  const int n_iters = (ch_end - ch_begin + 3) / 4;  // four 128-k chunks per stage
  const int groups_per_row = K >> group_shift;

  // (scale, zero) of rows row0..row0+63 for groups [grp0, grp0 + n_grp), after the ring
  __half2* sz = reinterpret_cast<__half2*>(&sm + 1);
  const int grp0 = (ch_begin * kChunk) >> group_shift;
  const int n_grp = ch_end > ch_begin ? (((ch_end * kChunk - 1) >> group_shift) - grp0 + 1) : 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kWarps);
    }
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kWarps) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmW);
      tma_prefetch_desc(&tmA);
      uint32_t issued = 0;
      for (int it = 0; it < n_iters; ++it) {
        const int s = it % S;
        const uint32_t ph = static_cast<uint32_t>(it / S) & 1u;
        if (!mbar_wait_sleep(&sm.empty[s], ph ^ 1u, abort_flag)) break;
        W4Stage<TH>& st = sm.stage[s];
        const int k0 = (ch_begin + 4 * it) * kChunk;
        mbar_arrive_expect_tx(&sm.full[s], 2 * kWBoxBytes + 2 * kABox);
        tma_load_2d(st.w, &tmW, &sm.full[s], k0 / 8, row0);
        tma_load_2d(st.w + kWBoxBytes, &tmW, &sm.full[s], k0 / 8 + 32, row0);
        tma_load_2d(st.a, &tmA, &sm.full[s], k0, 0);
        tma_load_2d(st.a + kABox, &tmA, &sm.full[s], k0 + 256, 0);
        ++issued;
      }
      const uint32_t first = issued > static_cast<uint32_t>(S) ? issued - S : 0;
      for (uint32_t i = first; i < issued; ++i) mbar_wait_drain(&sm.full[i % S], (i / S) & 1u);
    }
  } else {
    // ---------------------------------------------------------------- consumers
    // scales and zeros of the CTA, loaded while the first stages stream in
    for (int e = threadIdx.x; e < kRows * n_grp; e += kWarps * 32) {
      const int row = e / n_grp;
      const int gg = e - row * n_grp;
      const int n = row0 + row;
      __half2 v = __halves2half2(__float2half_rn(0.f), __float2half_rn(0.f));
      if (n < N) {
        const size_t gi = static_cast<size_t>(n) * groups_per_row + grp0 + gg;
        v = __halves2half2(scale16[gi], zero16[gi]);
      }
      sz[row * max_groups + gg] = v;
    }
    asm volatile("bar.sync 1, %0;" ::"r"(kWarps * 32) : "memory");

    // warp -> chunk cw of the stage (weight box cw/2, chunk cw%2 in it) and slices 2jp, 2jp+1;
    // every warp covers all four 16-row tiles, so activation fragments serve 64 rows
    const int cw = warp >> 1;
    const int jp = warp & 1;
    const int g = lane >> 2;
    const int c = lane & 3;
    float acc[4][TH][4];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int h = 0; h < TH; ++h)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[r][h][i] = 0.0f;

    for (int it = 0; it < n_iters; ++it) {
      const int s = it % S;
      const uint32_t ph = static_cast<uint32_t>(it / S) & 1u;
      const bool got = mbar_wait_sleep(&sm.full[s], ph, abort_flag);
      if (!__all_sync(0xFFFFFFFFu, got)) break;
      const int ch = ch_begin + 4 * it + cw;
      if (ch < ch_end) {  // warp-uniform
        W4Stage<TH>& st = sm.stage[s];
        const uint32_t wbox = smem_u32(st.w + (cw >> 1) * kWBoxBytes) + static_cast<uint32_t>(g) * 128u;
        const uint32_t a_base = smem_u32(st.a);
        // D = sum (128 + q) a over the k of one group span, O = sum a over the same k
        // (the "ones" MMA); the span's contribution is s * (D - (128 + z) O).
        float s_lo[4], s_hi[4], z_lo[4], z_hi[4];
        float dsum[4][TH][4], dones[TH][4];
        auto load_sz = [&](int gg) {
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const __half2 vlo = sz[(16 * r + g) * max_groups + gg];
            const __half2 vhi = sz[(16 * r + g + 8) * max_groups + gg];
            s_lo[r] = __low2float(vlo);
            s_hi[r] = __low2float(vhi);
            z_lo[r] = 128.0f + __high2float(vlo);
            z_hi[r] = 128.0f + __high2float(vhi);
          }
        };
        auto clear = [&]() {
#pragma unroll
          for (int h = 0; h < TH; ++h) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              dones[h][i] = 0.f;
#pragma unroll
              for (int r = 0; r < 4; ++r) dsum[r][h][i] = 0.f;
            }
          }
        };
        auto flush = [&]() {
#pragma unroll
          for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int h = 0; h < TH; ++h) {
              acc[r][h][0] = fmaf(s_lo[r], fmaf(-z_lo[r], dones[h][0], dsum[r][h][0]), acc[r][h][0]);
              acc[r][h][1] = fmaf(s_lo[r], fmaf(-z_lo[r], dones[h][1], dsum[r][h][1]), acc[r][h][1]);
              acc[r][h][2] = fmaf(s_hi[r], fmaf(-z_hi[r], dones[h][2], dsum[r][h][2]), acc[r][h][2]);
              acc[r][h][3] = fmaf(s_hi[r], fmaf(-z_hi[r], dones[h][3], dsum[r][h][3]), acc[r][h][3]);
            }
        };
        constexpr uint32_t kOne2 = 0x3F803F80u;  // bf16 pair (1, 1)
        const uint32_t ones[4] = {kOne2, kOne2, kOne2, kOne2};
        if (GROUP_CHUNK) {
          load_sz(((ch * kChunk) >> group_shift) - grp0);
          clear();
        }
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int j = 2 * jp + jj;
          const int kl = cw * kChunk + 32 * j + 8 * c;  // k within the stage
          if (!GROUP_CHUNK) {
            load_sz(((ch * kChunk + 32 * j) >> group_shift) - grp0);
            clear();
          }
          uint32_t b[TH][4];
#pragma unroll
          for (int h = 0; h < TH; ++h) {
            // activation box (kl / 256) holds 8*TH rows of 256 k
            const uint4 v = lds128(a_base + static_cast<uint32_t>((kl >> 8) * kABox + (8 * h + g) * 512 + (kl & 255) * 2));
            b[h][0] = __byte_perm(v.x, v.z, 0x5410);  // (k0, k4)
            b[h][1] = __byte_perm(v.x, v.z, 0x7632);  // (k1, k5)
            b[h][2] = __byte_perm(v.y, v.w, 0x5410);  // (k2, k6)
            b[h][3] = __byte_perm(v.y, v.w, 0x7632);  // (k3, k7)
            mma_bf16_16816(dones[h], ones, b[h][0], b[h][1]);
            mma_bf16_16816(dones[h], ones, b[h][2], b[h][3]);
          }
          const uint32_t off = static_cast<uint32_t>((((4 * (cw & 1) + j) ^ g) * 16) + 4 * c);
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const uint32_t row_lo = wbox + static_cast<uint32_t>(16 * r) * 128u;
            const uint32_t xl = lds32(row_lo + off);
            const uint32_t xh = lds32(row_lo + 8u * 128u + off);
            // step 2j: slots (2c, 2c+1) <- nibbles (0, 4); (2c+8, 2c+9) <- (1, 5)
            // step 2j+1: slots (2c, 2c+1) <- nibbles (2, 6); (2c+8, 2c+9) <- (3, 7)
            const uint32_t a0[4] = {(xl & 0x000F000Fu) | 0x43004300u, (xh & 0x000F000Fu) | 0x43004300u,
                                    ((xl >> 4) & 0x000F000Fu) | 0x43004300u, ((xh >> 4) & 0x000F000Fu) | 0x43004300u};
            const uint32_t a1[4] = {((xl >> 8) & 0x000F000Fu) | 0x43004300u, ((xh >> 8) & 0x000F000Fu) | 0x43004300u,
                                    ((xl >> 12) & 0x000F000Fu) | 0x43004300u, ((xh >> 12) & 0x000F000Fu) | 0x43004300u};
#pragma unroll
            for (int h = 0; h < TH; ++h) {
              mma_bf16_16816(dsum[r][h], a0, b[h][0], b[h][1]);
              mma_bf16_16816(dsum[r][h], a1, b[h][2], b[h][3]);
            }
          }
          if (!GROUP_CHUNK) flush();
        }
        if (GROUP_CHUNK) flush();
      }
      // every value read from this stage has been consumed above
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[s]);
    }
    // the ring is drained once every consumer has left the loop
    asm volatile("bar.sync 1, %0;" ::"r"(kWarps * 32) : "memory");
    float* red = reinterpret_cast<float*>(sm.stage);  // [warp][r][h][i][lane]
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int h = 0; h < TH; ++h)
#pragma unroll
        for (int i = 0; i < 4; ++i) red[(((warp * 4 + r) * TH + h) * 4 + i) * 32 + lane] = acc[r][h][i];
  }
  __syncthreads();

  // fixed-order reduction: the eight warps of each tile -> CTA partial -> cluster
  {
    const float* red = reinterpret_cast<const float*>(sm.stage);
    for (int e = threadIdx.x; e < 4 * TH * 4 * 32; e += kThreadsW4) {
      const int ln = e & 31;
      const int i = (e >> 5) & 3;
      const int h = (e >> 7) % TH;
      const int r = (e >> 7) / TH;
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) v += red[(((w * 4 + r) * TH + h) * 4 + i) * 32 + ln];
      const int row = 16 * r + (ln >> 2) + ((i & 2) ? 8 : 0);
      const int tok = 8 * h + 2 * (ln & 3) + (i & 1);
      sm.part[row][tok] = v;
    }
  }
  cluster.sync();
  if (split == 0) {
    for (int e = threadIdx.x; e < kRows * 8 * TH; e += kThreadsW4) {
      const int row = e / (8 * TH);
      const int tok = e % (8 * TH);
      float v = 0.f;
#pragma unroll
      for (int q = 0; q < kSplit; ++q) v += cluster.map_shared_rank(&sm.part[0][0], q)[row * 16 + tok];
      const int n = row0 + row;
      if (n < N && tok < T) {
        __nv_bfloat16 hv = __float2bfloat16_rn(v);
        out[static_cast<size_t>(tok) * N + n] = *reinterpret_cast<uint16_t*>(&hv);
      }
    }
  }
  cluster.sync();  // peers keep their shared memory until rank 0 has read it
}

template <int TH, bool GROUP_CHUNK>
cudaError_t launch_tma(const CUtensorMap& tmW, const uint16_t* A, int T, const __half* s16, const __half* z16, int N,
                       int K, int group_shift, uint16_t* out, cudaStream_t stream, const char* name) {
  CUtensorMap tmA;
  cudaError_t e = make_tmap_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, A, static_cast<uint64_t>(T),
                               static_cast<uint64_t>(K), 256, 8 * TH, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (e != cudaSuccess) return e;
  // groups touched by one CTA's share of K (at most): ceil(chunks/kSplit) chunks, plus one straddled group
  const int chunks = K / kChunk;
  const int max_groups = (((chunks + kSplit - 1) / kSplit) * kChunk + (1 << group_shift) - 1) / (1 << group_shift) + 1;
  const int smem = w4_smem_bytes<TH>(max_groups);
  if (smem > 227 * 1024) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(w4a16_tma_kernel<TH, GROUP_CHUNK>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int blocks = ((N + kRows - 1) / kRows) * kSplit;
  LaunchScope scope(stream, name);
  w4a16_tma_kernel<TH, GROUP_CHUNK><<<blocks, kThreadsW4, smem, stream>>>(tmW, tmA, T, s16, z16, N, K, group_shift, max_groups,
                                                             out);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_w4a16(const uint16_t* A, int T, const uint32_t* packed, const uint16_t* scale16,
                         const uint16_t* zero16, int N, int K, int group_size, uint16_t* out, cudaStream_t stream) {
  cudaError_t e = launch_w4a16_dec(A, T, packed, scale16, zero16, N, K, group_size, out, stream);
  // cudaErrorNotSupported comes from the shape checks before any CUDA call, so
  // no runtime error state is set and none is cleared here
  if (e != cudaErrorNotSupported) return e;
  int group_shift = 0;
  while ((1 << group_shift) < group_size) ++group_shift;
  CUtensorMap tmW;
  e = make_tmap_2d(&tmW, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, packed, static_cast<uint64_t>(N),
                   static_cast<uint64_t>(K / 8), 32, kRows, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  const __half* s16 = reinterpret_cast<const __half*>(scale16);
  const __half* z16 = reinterpret_cast<const __half*>(zero16);
  const bool gc = group_shift >= 7;
  if (T <= 8) {
    return gc ? launch_tma<1, true>(tmW, A, T, s16, z16, N, K, group_shift, out, stream, "w4a16_tma_kernel<T<=8,g>=128>")
              : launch_tma<1, false>(tmW, A, T, s16, z16, N, K, group_shift, out, stream, "w4a16_tma_kernel<T<=8,g<128>");
  }
  return gc ? launch_tma<2, true>(tmW, A, T, s16, z16, N, K, group_shift, out, stream, "w4a16_tma_kernel<T<=16,g>=128>")
            : launch_tma<2, false>(tmW, A, T, s16, z16, N, K, group_shift, out, stream, "w4a16_tma_kernel<T<=16,g<128>");
}

}  // namespace ar
