// Decoder-block kernels of the AutoRound tuning step that are not tuned GEMMs:
// RMSNorm forward and backward, the rotary-embedding table, and causal softmax
// attention forward and backward per sample and head.
//
// [AR] §3 "Why Block-Wise Optimization" and "Algorithm Flow" make the decoder
// block the unit of tuning: the block output's error reaches every weight of
// the block, through attention and the norms.  The pages name the block but
// not its layers; the block here is the Llama family's pre-norm block:
//   r1 = rmsnorm(X) g1;  Q, K, V = r1 Wq^T, r1 Wk^T, r1 Wv^T;  rotary embedding
//   on Q and K (head halves (x_i, x_{i+d/2}) rotate by t 10000^(-2i/d), t the
//   position in the sample);  O = softmax(Q K^T / sqrt(d) + causal mask) V per
//   head;  X2 = X + O Wo^T;  r2 = rmsnorm(X2) g2;  Y = X2 + SwiGLU(r2).
// ([AR] = "Low-Bit Quantization in Practice with vLLM: Core Mechanisms and
// Architectural Optimizations of AutoRound".)
//
// Precision (shared with the oracle): every operand of a product is bf16,
// accumulators and the residual stream are fp32.  The attention probabilities
// come from two passes, P = bf16(exp(z - lse)) with lse the row's log-sum-exp
// over its keys, so that their rounding does not depend on the order in which
// keys are visited; O = P V needs no division afterwards.
//
// The exponentials are CUDA's fast exponential intrinsic (__expf, accurate to
// a few fp32 ulp), much cheaper per score than the accurate expf; a
// probability's bf16 rounding changes only within ~1e-7 of a rounding midpoint,
// the size of a summation-order difference.
//
// The attention kernels here run on mma.sync m16n8k16 (bf16, fp32 accumulation)
// over 64-row tiles staged in shared memory with cp.async (double-buffered,
// 16-byte row padding so that ldmatrix reads are free of bank conflicts); the
// forward and backward at head dimension 128 on whole 128-row blocks run on
// tcgen05 instead (ar_attn_tc.cu, ar_attn_bwd_tc.cu).  No kernel here waits on
// another CTA: every wait is a cp.async group wait or a CTA barrier.
#include "ar_internal.h"

namespace ar {
namespace {

constexpr int kAttnRows = 64;  // query (or key) rows per CTA
constexpr int kAttnThreads = 128;  // four warps of 16 rows

template <int D>
struct Tile {
  static constexpr int kPitch = D + 8;  // elements per shared-memory row
  static constexpr int kElems = kAttnRows * kPitch;
  static constexpr int kBytes = kElems * 2;
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// 64 rows x D bf16 columns starting at (row0, col0) of a matrix with row stride ld -> tile.
template <int D>
__device__ __forceinline__ void load_tile(uint16_t* sm, const uint16_t* g, int64_t row0, int64_t ld, int col0) {
  constexpr int kChunks = D / 8;
  for (int i = threadIdx.x; i < kAttnRows * kChunks; i += kAttnThreads) {
    const int r = i / kChunks;
    const int c = i - r * kChunks;
    cp_async16(sm + r * Tile<D>::kPitch + c * 8, g + (row0 + r) * ld + col0 + c * 8);
  }
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const uint16_t* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const uint16_t* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float round_bf16(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }

// A fragment (16 rows x 16 k) of a row-major tile: rows r0.., k 16*kk..
__device__ __forceinline__ void frag_a(uint32_t (&a)[4], const uint16_t* tile, int pitch, int r0, int kk) {
  const int l = threadIdx.x & 31;
  ldsm_x4(a, tile + (r0 + (l & 7) + 8 * ((l >> 3) & 1)) * pitch + 16 * kk + 8 * (l >> 4));
}
// B fragments of two n8 tiles (n0.., n0+8..) x k16 when the tile is stored [n][k]
// (keys x d for Q K^T): b[0], b[1] for n-tile n0; b[2], b[3] for n0 + 8.
__device__ __forceinline__ void frag_b_nk(uint32_t (&b)[4], const uint16_t* tile, int pitch, int n0, int kk) {
  const int l = threadIdx.x & 31;
  ldsm_x4(b, tile + (n0 + (l & 7) + 8 * (l >> 4)) * pitch + 16 * kk + 8 * ((l >> 3) & 1));
}
// B fragments of two n8 tiles x k16 when the tile is stored [k][n] (keys x d for P V).
__device__ __forceinline__ void frag_b_kn(uint32_t (&b)[4], const uint16_t* tile, int pitch, int n0, int kk) {
  const int l = threadIdx.x & 31;
  ldsm_x4_t(b, tile + (16 * kk + (l & 7) + 8 * ((l >> 3) & 1)) * pitch + n0 + 8 * (l >> 4));
}

// Accumulators of n-tiles 2kk, 2kk+1 (16 rows x 16 columns) as the A fragment of a
// product over those columns.
__device__ __forceinline__ void acc_to_a(uint32_t (&a)[4], const float (&c0)[4], const float (&c1)[4]) {
  a[0] = pack_bf16x2(c0[0], c0[1]);
  a[1] = pack_bf16x2(c0[2], c0[3]);
  a[2] = pack_bf16x2(c1[0], c1[1]);
  a[3] = pack_bf16x2(c1[2], c1[3]);
}

// ---------------------------------------------------------------------------
// attention forward: one CTA per (64-query block, head, sample)
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_kernel(const uint16_t* __restrict__ qkv, int H, int L, int nh, float scale, uint16_t* __restrict__ out,
                    float* __restrict__ lse_out) {
  constexpr int P = Tile<D>::kPitch;
  constexpr int NT = D / 8;   // n8 tiles of the output
  constexpr int KS = D / 16;  // k16 steps over d
  extern __shared__ __align__(128) uint8_t attn_smem[];
  uint16_t* sQ = reinterpret_cast<uint16_t*>(attn_smem);
  uint16_t* sK = sQ + Tile<D>::kElems;      // two buffers
  uint16_t* sV = sK + 2 * Tile<D>::kElems;  // two buffers
  const int nqb = L / kAttnRows;
  const int qb = nqb - 1 - static_cast<int>(blockIdx.x);  // the longest rows first
  const int h = blockIdx.y;
  const int s = blockIdx.z;
  const int64_t ld = 3 * static_cast<int64_t>(H);
  const int64_t rows0 = static_cast<int64_t>(s) * L;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  const int r0 = warp * 16;

  load_tile<D>(sQ, qkv, rows0 + qb * kAttnRows, ld, h * D);
  load_tile<D>(sK, qkv, rows0, ld, H + h * D);
  cp_async_commit();

  // ---- pass 1: row maximum and sum of exponentials over the row's keys -> lse
  float m[2] = {-INFINITY, -INFINITY}, lsum[2] = {0.f, 0.f};
  for (int kb = 0; kb <= qb; ++kb) {
    if (kb + 1 <= qb) load_tile<D>(sK + ((kb + 1) & 1) * Tile<D>::kElems, qkv, rows0 + (kb + 1) * kAttnRows, ld, H + h * D);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint16_t* kt = sK + (kb & 1) * Tile<D>::kElems;
    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      uint32_t a[4];
      frag_a(a, sQ, P, r0, kk);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b[4];
        frag_b_nk(b, kt, P, 16 * np, kk);
        mma_bf16(acc[2 * np], a, b[0], b[1]);
        mma_bf16(acc[2 * np + 1], a, b[2], b[3]);
      }
    }
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int qi = r0 + g + 8 * hr;  // query row within the block
      float z[16];
      float mx = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int kj = 8 * nt + 2 * c + e;
          float v = __fmul_rn(acc[nt][2 * hr + e], scale);
          if (kb == qb && kj > qi) v = -INFINITY;
          z[2 * nt + e] = v;
          mx = fmaxf(mx, v);
        }
      mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 2));
      const float mn = fmaxf(m[hr], mx);
      float t = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) t += __expf(z[i] - mn);
      t += __shfl_xor_sync(0xFFFFFFFFu, t, 1);
      t += __shfl_xor_sync(0xFFFFFFFFu, t, 2);
      lsum[hr] = lsum[hr] * __expf(m[hr] - mn) + t;
      m[hr] = mn;
    }
    __syncthreads();  // the next iteration refills the buffer read here
  }
  float lse[2];
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) lse[hr] = m[hr] + logf(lsum[hr]);

  // ---- pass 2: P = bf16(exp(z - lse)), O = P V
  float o[NT][4];
#pragma unroll
  for (int i = 0; i < NT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  load_tile<D>(sK, qkv, rows0, ld, H + h * D);
  load_tile<D>(sV, qkv, rows0, ld, 2 * H + h * D);
  cp_async_commit();
  for (int kb = 0; kb <= qb; ++kb) {
    if (kb + 1 <= qb) {
      const int nb = (kb + 1) & 1;
      load_tile<D>(sK + nb * Tile<D>::kElems, qkv, rows0 + (kb + 1) * kAttnRows, ld, H + h * D);
      load_tile<D>(sV + nb * Tile<D>::kElems, qkv, rows0 + (kb + 1) * kAttnRows, ld, 2 * H + h * D);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint16_t* kt = sK + (kb & 1) * Tile<D>::kElems;
    const uint16_t* vt = sV + (kb & 1) * Tile<D>::kElems;
    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      uint32_t a[4];
      frag_a(a, sQ, P, r0, kk);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b[4];
        frag_b_nk(b, kt, P, 16 * np, kk);
        mma_bf16(acc[2 * np], a, b[0], b[1]);
        mma_bf16(acc[2 * np + 1], a, b[2], b[3]);
      }
    }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int qi = r0 + g + 8 * (i >> 1);
        const int kj = 8 * nt + 2 * c + (i & 1);
        const float z = __fmul_rn(acc[nt][i], scale);
        acc[nt][i] = (kb == qb && kj > qi) ? 0.f : __expf(z - lse[i >> 1]);
      }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {  // keys 16 kk .. 16 kk + 15
      uint32_t a[4];
      acc_to_a(a, acc[2 * kk], acc[2 * kk + 1]);
#pragma unroll
      for (int np = 0; np < NT / 2; ++np) {
        uint32_t b[4];
        frag_b_kn(b, vt, P, 16 * np, kk);
        mma_bf16(o[2 * np], a, b[0], b[1]);
        mma_bf16(o[2 * np + 1], a, b[2], b[3]);
      }
    }
    __syncthreads();
  }
  // ---- O (bf16) and lse
  bool bad = false;
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int qi = qb * kAttnRows + r0 + g + 8 * hr;
    uint16_t* orow = out + (rows0 + qi) * static_cast<int64_t>(H) + h * D;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const float v0 = o[nt][2 * hr], v1 = o[nt][2 * hr + 1];
      bad |= !isfinite(v0) || !isfinite(v1);
      *reinterpret_cast<uint32_t*>(orow + 8 * nt + 2 * c) = pack_bf16x2(v0, v1);
    }
    if (c == 0) lse_out[(static_cast<int64_t>(s) * nh + h) * L + qi] = lse[hr];
  }
  if (bad) raise_status(kStatusNonFinite);
}

// D[s][h][t] = sum over the head's columns of dO * O (fp32 from bf16): one warp per (token, head).
__global__ void attn_bwd_prep_kernel(const uint16_t* __restrict__ dO, const uint16_t* __restrict__ O, int64_t M,
                                     int H, int L, int nh, int d, float* __restrict__ Dout) {
  const int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= M * nh) return;
  const int64_t m = w / nh;
  const int h = static_cast<int>(w - m * nh);
  const uint16_t* a = dO + m * H + h * d;
  const uint16_t* b = O + m * H + h * d;
  float acc = 0.f;
  for (int i = 2 * lane; i < d; i += 64) {
    const uint32_t x = *reinterpret_cast<const uint32_t*>(a + i);
    const uint32_t y = *reinterpret_cast<const uint32_t*>(b + i);
    acc = fmaf(bf16_lo(x), bf16_lo(y), acc);
    acc = fmaf(bf16_hi(x), bf16_hi(y), acc);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, off);
  if (lane == 0) {
    const int64_t s = m / L;
    const int t = static_cast<int>(m - s * L);
    Dout[(s * nh + h) * L + t] = acc;
  }
}

// Inverse rotation of a head's row held as n8-tile accumulator pairs: column i and
// i + D/2 (n-tiles nt and nt + D/16) at position t; cs = (cos, sin) [L][D/2].
template <int D>
__device__ __forceinline__ void rope_back_row(float (&v)[D / 8][4], int hr, int t, const float2* __restrict__ cs) {
  const int c = threadIdx.x & 3;
#pragma unroll
  for (int nt = 0; nt < D / 16; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int i = 8 * nt + 2 * c + e;
      const float2 r = cs[static_cast<int64_t>(t) * (D / 2) + i];
      const float x1 = v[nt][2 * hr + e], x2 = v[nt + D / 16][2 * hr + e];
      // rotation by -angle: (x1 c + x2 s, x2 c - x1 s)
      v[nt][2 * hr + e] = __fadd_rn(__fmul_rn(x1, r.x), __fmul_rn(x2, r.y));
      v[nt + D / 16][2 * hr + e] = __fsub_rn(__fmul_rn(x2, r.x), __fmul_rn(x1, r.y));
    }
}

// ---------------------------------------------------------------------------
// attention backward, dQ: one CTA per (64-query block, head, sample), keys up to the diagonal
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_bwd_dq_kernel(const uint16_t* __restrict__ qkv, const uint16_t* __restrict__ dO, const float* __restrict__ lse,
                       const float* __restrict__ Dsum, const float2* __restrict__ cs, int H, int L, int nh, float scale,
                       uint16_t* __restrict__ dqkv) {
  constexpr int P = Tile<D>::kPitch;
  constexpr int NT = D / 8;
  constexpr int KS = D / 16;
  extern __shared__ __align__(128) uint8_t attn_smem[];
  uint16_t* sQ = reinterpret_cast<uint16_t*>(attn_smem);
  uint16_t* sdO = sQ + Tile<D>::kElems;
  uint16_t* sK = sdO + Tile<D>::kElems;     // two buffers
  uint16_t* sV = sK + 2 * Tile<D>::kElems;  // two buffers
  const int nqb = L / kAttnRows;
  const int qb = nqb - 1 - static_cast<int>(blockIdx.x);
  const int h = blockIdx.y;
  const int s = blockIdx.z;
  const int64_t ld = 3 * static_cast<int64_t>(H);
  const int64_t rows0 = static_cast<int64_t>(s) * L;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  const int r0 = warp * 16;
  float lr[2], dr[2];
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int64_t idx = (static_cast<int64_t>(s) * nh + h) * L + qb * kAttnRows + r0 + g + 8 * hr;
    lr[hr] = lse[idx];
    dr[hr] = Dsum[idx];
  }
  load_tile<D>(sQ, qkv, rows0 + qb * kAttnRows, ld, h * D);
  load_tile<D>(sdO, dO, rows0 + qb * kAttnRows, H, h * D);
  load_tile<D>(sK, qkv, rows0, ld, H + h * D);
  load_tile<D>(sV, qkv, rows0, ld, 2 * H + h * D);
  cp_async_commit();
  float dq[NT][4];
#pragma unroll
  for (int i = 0; i < NT; ++i) dq[i][0] = dq[i][1] = dq[i][2] = dq[i][3] = 0.f;
  for (int kb = 0; kb <= qb; ++kb) {
    if (kb + 1 <= qb) {
      const int nb = (kb + 1) & 1;
      load_tile<D>(sK + nb * Tile<D>::kElems, qkv, rows0 + (kb + 1) * kAttnRows, ld, H + h * D);
      load_tile<D>(sV + nb * Tile<D>::kElems, qkv, rows0 + (kb + 1) * kAttnRows, ld, 2 * H + h * D);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint16_t* kt = sK + (kb & 1) * Tile<D>::kElems;
    const uint16_t* vt = sV + (kb & 1) * Tile<D>::kElems;
    float sc[8][4], dp[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) sc[i][j] = dp[i][j] = 0.f;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      uint32_t aq[4], ao[4];
      frag_a(aq, sQ, P, r0, kk);
      frag_a(ao, sdO, P, r0, kk);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b[4];
        frag_b_nk(b, kt, P, 16 * np, kk);
        mma_bf16(sc[2 * np], aq, b[0], b[1]);
        mma_bf16(sc[2 * np + 1], aq, b[2], b[3]);
        frag_b_nk(b, vt, P, 16 * np, kk);  // dP = dO V^T: V stored [key][d] like K
        mma_bf16(dp[2 * np], ao, b[0], b[1]);
        mma_bf16(dp[2 * np + 1], ao, b[2], b[3]);
      }
    }
    // dS = bf16(P (dP - D) scale), P = bf16(exp(z - lse)); masked entries are 0
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int hr = i >> 1;
        const int qi = r0 + g + 8 * hr;
        const int kj = 8 * nt + 2 * c + (i & 1);
        const float z = __fmul_rn(sc[nt][i], scale);
        const float p = (kb == qb && kj > qi) ? 0.f : round_bf16(__expf(z - lr[hr]));
        sc[nt][i] = __fmul_rn(__fmul_rn(p, __fsub_rn(dp[nt][i], dr[hr])), scale);
      }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t a[4];
      acc_to_a(a, sc[2 * kk], sc[2 * kk + 1]);
#pragma unroll
      for (int np = 0; np < NT / 2; ++np) {
        uint32_t b[4];
        frag_b_kn(b, kt, P, 16 * np, kk);  // dQ = dS K: K as [key][d] = [k][n]
        mma_bf16(dq[2 * np], a, b[0], b[1]);
        mma_bf16(dq[2 * np + 1], a, b[2], b[3]);
      }
    }
    __syncthreads();
  }
  bool bad = false;
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int t = qb * kAttnRows + r0 + g + 8 * hr;
    rope_back_row<D>(dq, hr, t, cs);
    uint16_t* row = dqkv + (rows0 + t) * ld + h * D;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      bad |= !isfinite(dq[nt][2 * hr]) || !isfinite(dq[nt][2 * hr + 1]);
      *reinterpret_cast<uint32_t*>(row + 8 * nt + 2 * c) = pack_bf16x2(dq[nt][2 * hr], dq[nt][2 * hr + 1]);
    }
  }
  if (bad) raise_status(kStatusNonFinite);
}

// ---------------------------------------------------------------------------
// attention backward, dK and dV: one CTA per (64-key block, head, sample), queries from the diagonal on
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_bwd_dkdv_kernel(const uint16_t* __restrict__ qkv, const uint16_t* __restrict__ dO,
                         const float* __restrict__ lse, const float* __restrict__ Dsum,
                         const float2* __restrict__ cs, int H, int L, int nh, float scale,
                         uint16_t* __restrict__ dqkv) {
  constexpr int P = Tile<D>::kPitch;
  constexpr int NT = D / 8;
  constexpr int KS = D / 16;
  extern __shared__ __align__(128) uint8_t attn_smem[];
  uint16_t* sK = reinterpret_cast<uint16_t*>(attn_smem);
  uint16_t* sV = sK + Tile<D>::kElems;
  uint16_t* sQ = sV + Tile<D>::kElems;        // two buffers
  uint16_t* sdO = sQ + 2 * Tile<D>::kElems;   // two buffers
  float* sL = reinterpret_cast<float*>(sdO + 2 * Tile<D>::kElems);  // [2][64] lse, then [2][64] D
  float* sD = sL + 2 * kAttnRows;
  const int nkb = L / kAttnRows;
  const int kb = static_cast<int>(blockIdx.x);  // key blocks near the start see the most queries
  const int h = blockIdx.y;
  const int s = blockIdx.z;
  const int64_t ld = 3 * static_cast<int64_t>(H);
  const int64_t rows0 = static_cast<int64_t>(s) * L;
  const int64_t lrow0 = (static_cast<int64_t>(s) * nh + h) * L;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  const int r0 = warp * 16;  // this warp's keys within the block

  auto load_q = [&](int qb, int buf) {
    load_tile<D>(sQ + buf * Tile<D>::kElems, qkv, rows0 + qb * kAttnRows, ld, h * D);
    load_tile<D>(sdO + buf * Tile<D>::kElems, dO, rows0 + qb * kAttnRows, H, h * D);
    for (int i = threadIdx.x; i < kAttnRows / 4; i += kAttnThreads) {
      cp_async16(sL + buf * kAttnRows + 4 * i, lse + lrow0 + qb * kAttnRows + 4 * i);
      cp_async16(sD + buf * kAttnRows + 4 * i, Dsum + lrow0 + qb * kAttnRows + 4 * i);
    }
  };
  load_tile<D>(sK, qkv, rows0 + kb * kAttnRows, ld, H + h * D);
  load_tile<D>(sV, qkv, rows0 + kb * kAttnRows, ld, 2 * H + h * D);
  load_q(kb, 0);
  cp_async_commit();
  float dk[NT][4], dv[NT][4];
#pragma unroll
  for (int i = 0; i < NT; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) dk[i][j] = dv[i][j] = 0.f;
  for (int qb = kb; qb < nkb; ++qb) {
    const int buf = (qb - kb) & 1;
    if (qb + 1 < nkb) load_q(qb + 1, buf ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint16_t* qt = sQ + buf * Tile<D>::kElems;
    const uint16_t* ot = sdO + buf * Tile<D>::kElems;
    const float* lq = sL + buf * kAttnRows;
    const float* dq = sD + buf * kAttnRows;
#pragma unroll
    for (int half = 0; half < 2; ++half) {  // queries 32 half .. 32 half + 31
      float st[4][4], dpt[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) st[i][j] = dpt[i][j] = 0.f;
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
        uint32_t ak[4], av[4];
        frag_a(ak, sK, P, r0, kk);
        frag_a(av, sV, P, r0, kk);
#pragma unroll
        for (int np = 0; np < 2; ++np) {
          uint32_t b[4];
          frag_b_nk(b, qt, P, 32 * half + 16 * np, kk);  // S^T = K Q^T: Q as [query][d] = [n][k]
          mma_bf16(st[2 * np], ak, b[0], b[1]);
          mma_bf16(st[2 * np + 1], ak, b[2], b[3]);
          frag_b_nk(b, ot, P, 32 * half + 16 * np, kk);  // dP^T = V dO^T
          mma_bf16(dpt[2 * np], av, b[0], b[1]);
          mma_bf16(dpt[2 * np + 1], av, b[2], b[3]);
        }
      }
      // P^T = bf16(exp(z - lse[q])), dS^T = bf16(P^T (dP^T - D[q]) scale); queries before the key are masked
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int kj = r0 + g + 8 * (i >> 1);                  // key within the block
          const int qi = 32 * half + 8 * nt + 2 * c + (i & 1);   // query within its block
          const float z = __fmul_rn(st[nt][i], scale);
          const float p = (qb == kb && qi < kj) ? 0.f : round_bf16(__expf(z - lq[qi]));
          st[nt][i] = p;
          dpt[nt][i] = __fmul_rn(__fmul_rn(p, __fsub_rn(dpt[nt][i], dq[qi])), scale);
        }
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {  // queries 32 half + 16 kk ..
        uint32_t ap[4], as[4];
        acc_to_a(ap, st[2 * kk], st[2 * kk + 1]);
        acc_to_a(as, dpt[2 * kk], dpt[2 * kk + 1]);
#pragma unroll
        for (int np = 0; np < NT / 2; ++np) {
          uint32_t b[4];
          frag_b_kn(b, ot, P, 16 * np, 2 * half + kk);  // dV += P^T dO: dO as [query][d] = [k][n]
          mma_bf16(dv[2 * np], ap, b[0], b[1]);
          mma_bf16(dv[2 * np + 1], ap, b[2], b[3]);
          frag_b_kn(b, qt, P, 16 * np, 2 * half + kk);  // dK += dS^T Q
          mma_bf16(dk[2 * np], as, b[0], b[1]);
          mma_bf16(dk[2 * np + 1], as, b[2], b[3]);
        }
      }
    }
    __syncthreads();
  }
  bool bad = false;
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int t = kb * kAttnRows + r0 + g + 8 * hr;
    rope_back_row<D>(dk, hr, t, cs);
    uint16_t* row = dqkv + (rows0 + t) * ld;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      bad |= !isfinite(dk[nt][2 * hr]) || !isfinite(dv[nt][2 * hr]);
      *reinterpret_cast<uint32_t*>(row + H + h * D + 8 * nt + 2 * c) = pack_bf16x2(dk[nt][2 * hr], dk[nt][2 * hr + 1]);
      *reinterpret_cast<uint32_t*>(row + 2 * H + h * D + 8 * nt + 2 * c) =
          pack_bf16x2(dv[nt][2 * hr], dv[nt][2 * hr + 1]);
    }
  }
  if (bad) raise_status(kStatusNonFinite);
}

// ---------------------------------------------------------------------------
// RMSNorm
// ---------------------------------------------------------------------------
// r = bf16(x inv gamma), inv = 1 / sqrt(sum(x^2) / H + eps), one warp per row; the
// sum of squares runs over the lane's 8-column chunks in order, then a fixed xor tree.
template <bool IN_F32>
__global__ void rmsnorm_fwd_kernel(const void* __restrict__ x, const float* __restrict__ gamma, int64_t M, int H,
                                   float eps, uint16_t* __restrict__ r, float* __restrict__ inv_out) {
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  auto load8 = [&](int chunk, float (&v)[8]) {
    if (IN_F32) {
      const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(x) + row * H + 8 * chunk);
      const float4 a = p[0], b = p[1];
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
      const uint4 w = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + row * H + 8 * chunk);
      const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[2 * i] = bf16_lo(u[i]);
        v[2 * i + 1] = bf16_hi(u[i]);
      }
    }
  };
  float ss = 0.f;
  bool bad = false;
  for (int ch = lane; ch < H / 8; ch += 32) {
    float v[8];
    load8(ch, v);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      ss = __fadd_rn(ss, __fmul_rn(v[i], v[i]));
      bad |= !isfinite(v[i]);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xFFFFFFFFu, ss, off));
  const float inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(ss, static_cast<float>(H)), eps)));
  for (int ch = lane; ch < H / 8; ch += 32) {
    float v[8];
    load8(ch, v);
    const float4 g0 = *reinterpret_cast<const float4*>(gamma + 8 * ch);
    const float4 g1 = *reinterpret_cast<const float4*>(gamma + 8 * ch + 4);
    const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      o[i] = pack_bf16x2(__fmul_rn(__fmul_rn(v[2 * i], inv), gg[2 * i]),
                         __fmul_rn(__fmul_rn(v[2 * i + 1], inv), gg[2 * i + 1]));
    *reinterpret_cast<uint4*>(r + row * H + 8 * ch) = make_uint4(o[0], o[1], o[2], o[3]);
  }
  if (lane == 0 && inv_out) inv_out[row] = inv;
  if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) raise_status(kStatusNonFinite);
}

// dX2 = bf16(G + inv gdy - x inv^3 mean(gdy x)), gdy = dr gamma: the RMSNorm backward
// added to the residual path's gradient G; one warp per row.
__global__ void rmsnorm_bwd_kernel(const float* __restrict__ x, const float* __restrict__ inv,
                                   const float* __restrict__ gamma, const float* __restrict__ dr,
                                   const uint16_t* __restrict__ G, int64_t M, int H, uint16_t* __restrict__ dx) {
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  const float* xr = x + row * H;
  const float* drr = dr + row * H;
  float acc = 0.f;
  for (int ch = lane; ch < H / 4; ch += 32) {
    const float4 a = *reinterpret_cast<const float4*>(xr + 4 * ch);
    const float4 b = *reinterpret_cast<const float4*>(drr + 4 * ch);
    const float4 gm = *reinterpret_cast<const float4*>(gamma + 4 * ch);
    acc = __fadd_rn(acc, __fmul_rn(__fmul_rn(b.x, gm.x), a.x));
    acc = __fadd_rn(acc, __fmul_rn(__fmul_rn(b.y, gm.y), a.y));
    acc = __fadd_rn(acc, __fmul_rn(__fmul_rn(b.z, gm.z), a.z));
    acc = __fadd_rn(acc, __fmul_rn(__fmul_rn(b.w, gm.w), a.w));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xFFFFFFFFu, acc, off));
  const float mean = __fdiv_rn(acc, static_cast<float>(H));
  const float iv = inv[row];
  const float i3m = __fmul_rn(__fmul_rn(__fmul_rn(iv, iv), iv), mean);
  bool bad = !isfinite(mean);
  for (int ch = lane; ch < H / 4; ch += 32) {
    const float4 a = *reinterpret_cast<const float4*>(xr + 4 * ch);
    const float4 b = *reinterpret_cast<const float4*>(drr + 4 * ch);
    const float4 gm = *reinterpret_cast<const float4*>(gamma + 4 * ch);
    const uint2 gw = *reinterpret_cast<const uint2*>(G + row * H + 4 * ch);
    const float xs[4] = {a.x, a.y, a.z, a.w}, ds[4] = {b.x, b.y, b.z, b.w}, gs[4] = {gm.x, gm.y, gm.z, gm.w};
    const float gg[4] = {bf16_lo(gw.x), bf16_hi(gw.x), bf16_lo(gw.y), bf16_hi(gw.y)};
    float o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float t = __fsub_rn(__fmul_rn(iv, __fmul_rn(ds[i], gs[i])), __fmul_rn(xs[i], i3m));
      o[i] = __fadd_rn(gg[i], t);
      bad |= !isfinite(o[i]);
    }
    *reinterpret_cast<uint2*>(dx + row * H + 4 * ch) = make_uint2(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]));
  }
  if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) raise_status(kStatusNonFinite);
}

// (cos, sin) of t 10000^(-2i/d), computed in fp64 and rounded to fp32: [L][d/2].
__global__ void rope_table_kernel(int L, int d, float2* __restrict__ cs) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  const int half = d / 2;
  if (idx >= L * half) return;
  const int t = idx / half;
  const int i = idx - t * half;
  const double ang = static_cast<double>(t) * pow(10000.0, -2.0 * i / d);
  cs[idx] = make_float2(static_cast<float>(cos(ang)), static_cast<float>(sin(ang)));
}

template <int D>
cudaError_t attn_fwd_launch(const uint16_t* qkv, int S, int L, int H, uint16_t* out, float* lse, cudaStream_t st) {
  const int nh = H / D;
  const int smem = 5 * Tile<D>::kBytes;
  auto k = attn_fwd_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  LaunchScope scope(st, D == 128 ? "attn_fwd_kernel<d128>" : "attn_fwd_kernel<d64>");
  k<<<dim3(L / kAttnRows, nh, S), kAttnThreads, smem, st>>>(qkv, H, L, nh, 1.0f / sqrtf(static_cast<float>(D)), out,
                                                             lse);
  return cudaGetLastError();
}

// D[s][h][t] = rowsum(dO * O) over each head's columns
cudaError_t attn_bwd_prep(const uint16_t* O, const uint16_t* dO, int S, int L, int H, int D, float* Dsum,
                          cudaStream_t st) {
  const int nh = H / D;
  const int64_t M = static_cast<int64_t>(S) * L;
  const int64_t warps = M * nh;
  LaunchScope scope(st, "attn_bwd_prep_kernel");
  attn_bwd_prep_kernel<<<static_cast<unsigned>((warps * 32 + 255) / 256), 256, 0, st>>>(dO, O, M, H, L, nh, D, Dsum);
  return cudaGetLastError();
}

template <int D>
cudaError_t attn_bwd_launch(const uint16_t* qkv, const uint16_t* O, const uint16_t* dO, const float* lse,
                            float* Dsum, const float2* cs, int S, int L, int H, uint16_t* dqkv, cudaStream_t st) {
  const int nh = H / D;
  const float scale = 1.0f / sqrtf(static_cast<float>(D));
  cudaError_t e = attn_bwd_prep(O, dO, S, L, H, D, Dsum, st);
  if (e != cudaSuccess) return e;
  const int smem_dq = 6 * Tile<D>::kBytes;
  e = cudaFuncSetAttribute(attn_bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_dq);
  if (e != cudaSuccess) return e;
  {
    LaunchScope scope(st, D == 128 ? "attn_bwd_dq_kernel<d128>" : "attn_bwd_dq_kernel<d64>");
    attn_bwd_dq_kernel<D><<<dim3(L / kAttnRows, nh, S), kAttnThreads, smem_dq, st>>>(qkv, dO, lse, Dsum, cs, H, L,
                                                                                     nh, scale, dqkv);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int smem_kv = 6 * Tile<D>::kBytes + 4 * kAttnRows * 4;
  e = cudaFuncSetAttribute(attn_bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_kv);
  if (e != cudaSuccess) return e;
  {
    LaunchScope scope(st, D == 128 ? "attn_bwd_dkdv_kernel<d128>" : "attn_bwd_dkdv_kernel<d64>");
    attn_bwd_dkdv_kernel<D><<<dim3(L / kAttnRows, nh, S), kAttnThreads, smem_kv, st>>>(qkv, dO, lse, Dsum, cs, H, L,
                                                                                       nh, scale, dqkv);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd(const uint16_t* qkv, int S, int L, int H, int head_dim, uint16_t* out, float* lse,
                            cudaStream_t st) {
  // head dimension 128 and whole 128-row blocks: the tcgen05 kernel (ar_attn_tc.cu)
  if (head_dim == 128 && L % 128 == 0) return launch_attn_fwd_tc(qkv, S, L, H, out, lse, st);
  if (head_dim == 128) return attn_fwd_launch<128>(qkv, S, L, H, out, lse, st);
  if (head_dim == 64) return attn_fwd_launch<64>(qkv, S, L, H, out, lse, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_attn_bwd(const uint16_t* qkv, const uint16_t* O, const uint16_t* dO, const float* lse,
                            float* Dsum, const float* rope_cs, int S, int L, int H, int head_dim, uint16_t* dqkv,
                            cudaStream_t st) {
  const float2* cs = reinterpret_cast<const float2*>(rope_cs);
  if (head_dim == 128 && L % 128 == 0) {  // the tcgen05 kernels (ar_attn_bwd_tc.cu)
    const cudaError_t e = attn_bwd_prep(O, dO, S, L, H, head_dim, Dsum, st);
    if (e != cudaSuccess) return e;
    return launch_attn_bwd_tc(qkv, dO, lse, Dsum, rope_cs, S, L, H, dqkv, st);
  }
  if (head_dim == 128) return attn_bwd_launch<128>(qkv, O, dO, lse, Dsum, cs, S, L, H, dqkv, st);
  if (head_dim == 64) return attn_bwd_launch<64>(qkv, O, dO, lse, Dsum, cs, S, L, H, dqkv, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_rmsnorm_fwd(const void* x, bool x_f32, const float* gamma, int64_t M, int H, uint16_t* r,
                               float* inv, cudaStream_t st) {
  const int64_t threads = M * 32;
  const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
  LaunchScope scope(st, x_f32 ? "rmsnorm_fwd_kernel<f32>" : "rmsnorm_fwd_kernel<bf16>");
  if (x_f32) rmsnorm_fwd_kernel<true><<<blocks, 256, 0, st>>>(x, gamma, M, H, 1e-6f, r, inv);
  else rmsnorm_fwd_kernel<false><<<blocks, 256, 0, st>>>(x, gamma, M, H, 1e-6f, r, inv);
  return cudaGetLastError();
}

cudaError_t launch_rmsnorm_bwd(const float* x, const float* inv, const float* gamma, const float* dr,
                               const uint16_t* G, int64_t M, int H, uint16_t* dx, cudaStream_t st) {
  const int64_t threads = M * 32;
  LaunchScope scope(st, "rmsnorm_bwd_kernel");
  rmsnorm_bwd_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, st>>>(x, inv, gamma, dr, G, M, H, dx);
  return cudaGetLastError();
}

cudaError_t launch_rope_table(int L, int head_dim, float* cs, cudaStream_t st) {
  const int n = L * (head_dim / 2);
  LaunchScope scope(st, "rope_table_kernel");
  rope_table_kernel<<<(n + 255) / 256, 256, 0, st>>>(L, head_dim, reinterpret_cast<float2*>(cs));
  return cudaGetLastError();
}

}  // namespace ar
