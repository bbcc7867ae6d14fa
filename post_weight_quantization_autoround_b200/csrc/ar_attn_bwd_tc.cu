// Causal softmax attention backward of the decoder block on tcgen05, head
// dimension 128, sample lengths a multiple of 128.  The mma.sync kernels'
// method (ar_decoder.cu), with D = rowsum(dO * O) from their prep kernel and
// the forward's lse:
//   P = bf16(exp(s scale - lse)),  dS = bf16(P (dP - D) scale),  dP = dO V^T,
//   dV = P^T dO,  dK = dS^T Q,  dQ = dS K,
// fp32 accumulation of bf16 products, the exponential as in the tcgen05
// forward (2^x by the hardware after one fused multiply-add); dQ and dK leave
// through the inverse rotary rotation (the forward rotated Q and K).
//
// [AR] §3 "Why Block-Wise Optimization" and "Algorithm Flow": the block output's
// error reaches every weight of the decoder block, through attention ([AR] =
// "Low-Bit Quantization in Practice with vLLM: Core Mechanisms and
// Architectural Optimizations of AutoRound").
//
// Two kernels, no atomics, deterministic:
//  * dK, dV: one CTA per 128 keys of one (sample, head) (the MMA's M, one TMEM
//    lane per key), over the 64-query blocks from the diagonal on.  Per block:
//    S^T = K Q^T and dP^T = V dO^T (N = 64 queries) into one of two buffer
//    pairs; the softmax warps write P^T and dS^T as bf16 pairs back over the
//    columns they read; then dV += P^T dO and dK += dS^T Q with those as the A
//    operand from tensor memory and dO, Q as MN-major B operands.  The next
//    block's S^T, dP^T run while this block's elementwise work does.
//  * dQ: one CTA per 128 queries, over the 64-key blocks up to the diagonal:
//    S = Q K^T, dP = dO V^T, dS written back over dP, dQ += dS K.
// Warp roles: warp 0 TMA producer (the resident operands once, then a 3-deep
// ring of the streamed pair); warp 1 TMEM owner and issuer of the S chain;
// warps 2-17 the elementwise work (four per TMEM lane quarter, 16 of each
// block's 64 columns each) and the epilogue; warp 18 issuer of the dP chain;
// warp 19 issuer of the accumulating products.  Three issuing threads on three
// sub-partitions, because one thread issuing every MMA of a block (20-24 per
// 64-column block) was the limit.
// TMEM columns: S buffers 0 and 64, dP buffers 128 and 192, then the fp32
// accumulators (dV at 256 and dK at 384; dQ at 256).
#include <type_traits>

#include "ar_attn_tc.cuh"

namespace ar {
namespace {

constexpr int kBwD = 128;                   // head dimension
constexpr int kBwRows = 128;                // keys (dK, dV) or queries (dQ) per CTA
constexpr int kBwCols = 64;                 // streamed queries (dK, dV) or keys (dQ) per block
constexpr int kBwBig = kBwRows * kBwD * 2;  // 32 KiB: a resident 128 x 128 tile
constexpr int kBwSmall = kBwCols * kBwD * 2;  // 16 KiB: a streamed 64 x 128 tile
constexpr int kBwStages = 3;
constexpr int kBwSmWarps = 16;                     // four per TMEM lane quarter
constexpr int kBwWCols = kBwCols / (kBwSmWarps / 4);  // streamed columns per elementwise warp
static_assert(kBwWCols == 16, "the elementwise role loads and stores 16-column slices");
constexpr int kBwDpWarp = 2 + kBwSmWarps;          // MMA issuer of the dP chain
constexpr int kBwAccWarp = 3 + kBwSmWarps;         // MMA issuer of the accumulating products
constexpr int kBwThreads = (4 + kBwSmWarps) * 32;
constexpr uint32_t kBwColS = 0, kBwColDP = 128, kBwColAcc = 256;
constexpr uint32_t kBwTmemCols = 512;

struct BwCtl {
  uint64_t res_full;              // resident tiles landed
  uint64_t full[kBwStages];       // streamed pair landed
  uint64_t empty[kBwStages];      // streamed pair no longer read (one commit from each of three issuers)
  uint64_t st_full[2];            // MMA: S and dP of the buffer pair written (one commit from each issuer)
  uint64_t ds_full[2];            // elementwise warps: their bf16 operands written (one arrival per warp)
  uint64_t st_empty[2];           // MMA: the accumulating products of the pair done
  uint64_t acc_full;
  uint64_t mma_done;
  uint64_t mma_done_dp;           // the dP issuer's MMAs all complete
  uint64_t mma_done_acc;          // the accumulating issuer's MMAs all complete
  uint32_t tmem_base;
  int abort_flag;
};

constexpr int kBwSmem = 2 * kBwBig + kBwStages * 2 * kBwSmall + static_cast<int>(sizeof(BwCtl)) + 1024;
static_assert(kBwSmem <= 227 * 1024, "shared memory per CTA");

__device__ __forceinline__ void bw_init(BwCtl* ctl) {
  mbar_init(&ctl->res_full, 1);
  for (int i = 0; i < kBwStages; ++i) {
    mbar_init(&ctl->full[i], 1);
    mbar_init(&ctl->empty[i], 3);
  }
  for (int i = 0; i < 2; ++i) {
    mbar_init(&ctl->st_full[i], 2);
    mbar_init(&ctl->ds_full[i], kBwSmWarps);
    mbar_init(&ctl->st_empty[i], 1);
  }
  mbar_init(&ctl->acc_full, 1);
  mbar_init(&ctl->mma_done, 1);
  mbar_init(&ctl->mma_done_dp, 1);
  mbar_init(&ctl->mma_done_acc, 1);
  ctl->abort_flag = 0;
  fence_barrier_init();
}

// Producer: two resident 128-row tiles (columns c0a, c0b of tmBig at row rres),
// then n blocks of two 64-row tiles (columns c1a of tmA and c1b of tmB at row
// rstream + 64 j) into the ring.  Every issued copy lands before it returns.
__device__ __forceinline__ void bw_produce(BwCtl* ctl, uint8_t* resA, uint8_t* resB, uint8_t* ring,
                                           const CUtensorMap* tmBig, int c0a, int c0b, int rres,
                                           const CUtensorMap* tmA, int c1a, const CUtensorMap* tmB, int c1b,
                                           int rstream, int n, volatile int* abort_flag) {
  mbar_arrive_expect_tx(&ctl->res_full, 2 * kBwBig);
  tma_load_2d(resA, tmBig, &ctl->res_full, c0a, rres);
  tma_load_2d(resA + kBwBig / 2, tmBig, &ctl->res_full, c0a + 64, rres);
  tma_load_2d(resB, tmBig, &ctl->res_full, c0b, rres);
  tma_load_2d(resB + kBwBig / 2, tmBig, &ctl->res_full, c0b + 64, rres);
  uint32_t issued = 0;
  for (int j = 0; j < n; ++j) {
    const uint32_t slot = static_cast<uint32_t>(j) % kBwStages;
    if (!mbar_wait(&ctl->empty[slot], ((static_cast<uint32_t>(j) / kBwStages) & 1u) ^ 1u, abort_flag)) break;
    uint8_t* dst = ring + slot * 2 * kBwSmall;
    const int row = rstream + kBwCols * j;
    mbar_arrive_expect_tx(&ctl->full[slot], 2 * kBwSmall);
    tma_load_2d(dst, tmA, &ctl->full[slot], c1a, row);
    tma_load_2d(dst + kBwSmall / 2, tmA, &ctl->full[slot], c1a + 64, row);
    tma_load_2d(dst + kBwSmall, tmB, &ctl->full[slot], c1b, row);
    tma_load_2d(dst + kBwSmall + kBwSmall / 2, tmB, &ctl->full[slot], c1b + 64, row);
    ++issued;
  }
  mbar_wait_drain(&ctl->res_full, 0);
  for (uint32_t i = issued > kBwStages ? issued - kBwStages : 0; i < issued; ++i)
    mbar_wait_drain(&ctl->full[i % kBwStages], (i / kBwStages) & 1u);
}

// Three MMA-issuing threads on three sub-partitions (one thread issuing all of a
// block's MMAs was the kernel's limit: ~80 cycles per N = 64 MMA against 48 of
// tensor work).  Resident A1 (K, or Q for dQ) and A2 (V, or dO); streamed X (Q,
// or K) and Y (dO, or V) per block, in ring slot it % 3; buffer pair it % 2.
//  * bw_mma_st<false>: S = A1 X^T;  bw_mma_st<true>: dP = A2 Y^T (each commits to
//    st_full, which counts both, and to the slot's empty barrier);
//  * bw_mma_acc: after the elementwise warps have written their bf16 operands over
//    the pair, DKDV: dV += P^T Y and dK += dS^T X; else dQ += dS X; commits
//    st_empty (the pair may be overwritten) and the slot's empty barrier.
// Every issuer waits on each phase of its barriers in order.
template <bool DP>
__device__ __forceinline__ void bw_mma_st(BwCtl* ctl, uint32_t tmem, const uint8_t* res, const uint8_t* ring, int n,
                                          uint64_t* done, volatile int* abort_flag) {
  constexpr uint32_t idesc_st = idesc_bf16_f32(kBwRows, kBwCols, false, false);
  const uint64_t a = sdesc_sw128(smem_u32(res), 16, 1024);  // K = 16 steps add compile-time offsets
  const uint32_t col = DP ? kBwColDP : kBwColS;
  bool ok = mbar_wait(&ctl->res_full, 0, abort_flag);
  tc_fence_after();
  for (int it = 0; ok && it < n; ++it) {
    const uint32_t slot = static_cast<uint32_t>(it) % kBwStages;
    const uint32_t buf = static_cast<uint32_t>(it) & 1u;
    if (!mbar_wait(&ctl->full[slot], (static_cast<uint32_t>(it) / kBwStages) & 1u, abort_flag) ||
        !mbar_wait(&ctl->st_empty[buf], ((static_cast<uint32_t>(it) >> 1) & 1u) ^ 1u, abort_flag))
      break;
    tc_fence_after();
    const uint64_t b = sdesc_sw128(smem_u32(ring + slot * 2 * kBwSmall) + (DP ? kBwSmall : 0), 16, 1024);
    // K-major steps: 32 bytes inside a 128-byte swizzle row, the second 64-column box from kk = 4 on
#pragma unroll
    for (int kk = 0; kk < kBwD / 16; ++kk) {
      const uint32_t oa = (kk >> 2) * kBwRows * 128 + (kk & 3) * 32;
      const uint32_t ob = (kk >> 2) * kBwCols * 128 + (kk & 3) * 32;
      umma_bf16(tmem + col + buf * kBwCols, at_desc_add(a, oa), at_desc_add(b, ob), idesc_st, kk > 0 ? 1u : 0u);
    }
    umma_commit(&ctl->st_full[buf]);
    umma_commit(&ctl->empty[slot]);
  }
  umma_commit(done);  // every issued MMA completes before TMEM is released
  mbar_wait_drain(done, 0);
}

template <bool DKDV>
__device__ __forceinline__ void bw_mma_acc(BwCtl* ctl, uint32_t tmem, const uint8_t* ring, int n,
                                           volatile int* abort_flag) {
  constexpr uint32_t idesc_acc = idesc_bf16_f32(kBwRows, kBwD, false, true);
  bool ok = true;
  for (int p = 0; p < n; ++p) {
    const uint32_t pbuf = static_cast<uint32_t>(p) & 1u;
    const uint32_t pslot = static_cast<uint32_t>(p) % kBwStages;
    if (!mbar_wait(&ctl->ds_full[pbuf], (static_cast<uint32_t>(p) >> 1) & 1u, abort_flag)) {
      ok = false;
      break;
    }
    tc_fence_after();
    // MN-major views of the streamed tiles (64 rows x 128 columns as two 64-column boxes):
    // 64-column chunks one box apart, 8-row groups 1 KiB apart, a K = 16 step 2 KiB
    const uint32_t xs = smem_u32(ring + pslot * 2 * kBwSmall);
    const uint64_t x = sdesc_sw128(xs, kBwCols * 128, 1024), y = sdesc_sw128(xs + kBwSmall, kBwCols * 128, 1024);
#pragma unroll
    for (int kk = 0; kk < kBwCols / 16; ++kk) {
      // streamed rows 16 kk .. 16 kk + 15: written by the lane quarter's warp kk over its own first 8 columns
      const uint32_t c = pbuf * kBwCols + kBwWCols * kk;
      const uint32_t acc = (p > 0 || kk > 0) ? 1u : 0u;
      if (DKDV) {
        at_mma_ta(tmem + kBwColAcc, tmem + kBwColS + c, at_desc_add(y, kk * 2048), idesc_acc, acc);
        at_mma_ta(tmem + kBwColAcc + kBwD, tmem + kBwColDP + c, at_desc_add(x, kk * 2048), idesc_acc, acc);
      } else {
        at_mma_ta(tmem + kBwColAcc, tmem + kBwColDP + c, at_desc_add(x, kk * 2048), idesc_acc, acc);
      }
    }
    umma_commit(&ctl->st_empty[pbuf]);
    umma_commit(&ctl->empty[pslot]);
  }
  if (ok) umma_commit(&ctl->acc_full);
  umma_commit(&ctl->mma_done_acc);
  mbar_wait_drain(&ctl->mma_done_acc, 0);
}

// 32 fp32 accumulator values of a row -> 32 bf16 at dst (16-byte aligned); returns
// true when one is not finite.
__device__ __forceinline__ bool bw_store32(uint16_t* dst, const float (&v)[32]) {
  bool bad = false;
  uint32_t w[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    bad |= !isfinite(v[2 * i]) || !isfinite(v[2 * i + 1]);
    w[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
    *reinterpret_cast<uint4*>(dst + 8 * i) = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
  return bad;
}

// 16 fp32 accumulator values of a row -> 16 bf16 at dst (16-byte aligned); returns
// true when one is not finite.
__device__ __forceinline__ bool bw_store16(uint16_t* dst, const float (&v)[16]) {
  bool bad = false;
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    bad |= !isfinite(v[2 * i]) || !isfinite(v[2 * i + 1]);
    w[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
  }
  *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  *reinterpret_cast<uint4*>(dst + 8) = make_uint4(w[4], w[5], w[6], w[7]);
  return bad;
}

// A head row's accumulator columns c and c + 64 (c = 16 sub .. + 15) through the
// inverse rotary rotation at position t (cs = (cos, sin) [L][64]), to dst and
// dst + 64.
__device__ __forceinline__ bool bw_store_rope(uint32_t taddr, int sub, int t, const float2* __restrict__ cs,
                                              uint16_t* dst) {
  float x1[16], x2[16];
  at_ld16x2(taddr + 16 * sub, x1, taddr + 64 + 16 * sub, x2);
  const float4* c4 = reinterpret_cast<const float4*>(cs + static_cast<size_t>(t) * (kBwD / 2) + 16 * sub);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 r = __ldg(c4 + i);  // (cos, sin) of columns 2i, 2i + 1
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float cv = e ? r.z : r.x, sv = e ? r.w : r.y;
      const float a = x1[2 * i + e], b = x2[2 * i + e];
      // rotation by -angle: (a c + b s, b c - a s)
      x1[2 * i + e] = __fadd_rn(__fmul_rn(a, cv), __fmul_rn(b, sv));
      x2[2 * i + e] = __fsub_rn(__fmul_rn(b, cv), __fmul_rn(a, sv));
    }
  }
  bool bad = bw_store16(dst + 16 * sub, x1);
  bad |= bw_store16(dst + 64 + 16 * sub, x2);
  return bad;
}

// Elementwise warps: per block, P = bf16(exp(fl(s scale) - lse)) and
// dS = bf16(P (dP - D) scale) for this warp's 16 of the block's 64 streamed
// columns, written as bf16 pairs over the columns read (P over S only for DKDV,
// where dV needs it).  DKDV: the rows are keys, the columns queries (lse and D
// per column); else the rows are queries (lse and D per row), the columns keys.
// `row_pos` is the row's position in the sample, `col_pos0` the position of the
// first streamed column of block 0.
template <bool DKDV>
__device__ __forceinline__ bool bw_elementwise(BwCtl* ctl, uint32_t tmem, uint32_t lane_off, int sub, int n,
                                               int row_pos, int col_pos0, const float* __restrict__ lse_row,
                                               const float* __restrict__ D_row, float scale,
                                               volatile int* abort_flag) {
  const int lane = threadIdx.x & 31;
  // exp(fl(s scale) - lse) as 2^(s c2 - lse log2 e) with the hardware ex2, one fused
  // multiply-add per score (a few fp32 ulp, far below the bf16 rounding of P)
  constexpr float kLog2e = 1.4426950408889634f;
  const float c2 = scale * kLog2e;
  float l_own2 = 0.f, d_own = 0.f;
  if (!DKDV) {
    l_own2 = lse_row[row_pos] * kLog2e;
    d_own = D_row[row_pos];
  }
  for (int it = 0; it < n; ++it) {
    const uint32_t buf = static_cast<uint32_t>(it) & 1u;
    const int c0 = col_pos0 + kBwCols * it + kBwWCols * sub;  // position of this warp's first column
    float lc[kBwWCols], dc[kBwWCols];
    if (DKDV) {  // the columns' lse and D (the same addresses in every lane: broadcast loads)
      const float4* l4 = reinterpret_cast<const float4*>(lse_row + c0);
      const float4* d4 = reinterpret_cast<const float4*>(D_row + c0);
#pragma unroll
      for (int i = 0; i < kBwWCols / 4; ++i) {
        const float4 a = __ldg(l4 + i), b = __ldg(d4 + i);
        lc[4 * i] = a.x, lc[4 * i + 1] = a.y, lc[4 * i + 2] = a.z, lc[4 * i + 3] = a.w;
        dc[4 * i] = b.x, dc[4 * i + 1] = b.y, dc[4 * i + 2] = b.z, dc[4 * i + 3] = b.w;
      }
    }
    if (!__all_sync(0xFFFFFFFFu, mbar_wait(&ctl->st_full[buf], (static_cast<uint32_t>(it) >> 1) & 1u, abort_flag)))
      return false;
    tc_fence_after();
    const uint32_t cs = kBwColS + buf * kBwCols + kBwWCols * sub;
    const uint32_t cd = kBwColDP + buf * kBwCols + kBwWCols * sub;
    float sv[kBwWCols], dpv[kBwWCols];
    at_ld16x2(tmem + lane_off + cs, sv, tmem + lane_off + cd, dpv);
    uint32_t pp[kBwWCols / 2], dd[kBwWCols / 2];
    // causal: a query sees the keys at or before its position; only the two blocks
    // that overlap the diagonal hold masked entries
    const bool near_diag = DKDV ? it < 2 : it >= n - 2;
    auto body = [&](auto masked_tag) {
      constexpr bool kMask = decltype(masked_tag)::value;
#pragma unroll
      for (int i = 0; i < kBwWCols / 2; ++i) {
        float pe[2], de[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int c = 2 * i + e;
          const float lx2 = DKDV ? lc[c] * kLog2e : l_own2;
          const float dx = DKDV ? dc[c] : d_own;
          float p = at_round_bf16(at_ex2(fmaf(sv[c], c2, -lx2)));
          if (kMask) {
            const int cpos = c0 + c;
            if (DKDV ? (cpos < row_pos) : (cpos > row_pos)) p = 0.f;
          }
          pe[e] = p;
          de[e] = __fmul_rn(__fmul_rn(p, __fsub_rn(dpv[c], dx)), scale);
        }
        pp[i] = pack_bf16x2(pe[0], pe[1]);
        dd[i] = pack_bf16x2(de[0], de[1]);
      }
    };
    if (near_diag) body(std::true_type{});
    else body(std::false_type{});
    // pair column j of the slice holds streamed columns 2j, 2j + 1 (over the slice's first 8 columns)
    if (DKDV) at_tmem_st8(tmem + lane_off + cs, pp);
    at_tmem_st8(tmem + lane_off + cd, dd);
    at_tmem_st_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl->ds_full[buf]);
  }
  return true;
}

// dK, dV: CTA (key block kb of 128, head, sample); query blocks of 64 from 2 kb on.
__global__ void __launch_bounds__(kBwThreads, 1)
    attn_bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tmBig, const __grid_constant__ CUtensorMap tmQ64,
                            const __grid_constant__ CUtensorMap tmDO64, const float* __restrict__ lse,
                            const float* __restrict__ Dsum, const float2* __restrict__ cs, int H, int L, int nh,
                            float scale, uint16_t* __restrict__ dqkv) {
  extern __shared__ uint8_t bw_smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(bw_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = base;
  uint8_t* sV = sK + kBwBig;
  uint8_t* ring = sV + kBwBig;
  BwCtl* ctl = reinterpret_cast<BwCtl*>(ring + kBwStages * 2 * kBwSmall);
  volatile int* abort_flag = &ctl->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kb = static_cast<int>(blockIdx.x);  // key blocks near the start see the most queries
  const int h = blockIdx.y, s = blockIdx.z;
  const int row0 = s * L;
  const int q0 = 2 * kb;                        // first 64-query block at or after the keys
  const int n = L / kBwCols - q0;
  if (threadIdx.x == 0) bw_init(ctl);
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmBig);
    tma_prefetch_desc(&tmQ64);
    tma_prefetch_desc(&tmDO64);
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, kBwTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  if (warp == 0) {
    if (lane == 0)
      bw_produce(ctl, sK, sV, ring, &tmBig, H + h * kBwD, 2 * H + h * kBwD, row0 + kb * kBwRows, &tmQ64, h * kBwD,
                 &tmDO64, h * kBwD, row0 + q0 * kBwCols, n, abort_flag);
  } else if (warp == 1) {
    if (lane == 0) bw_mma_st<false>(ctl, tmem, sK, ring, n, &ctl->mma_done, abort_flag);
  } else if (warp == kBwDpWarp) {
    if (lane == 0) bw_mma_st<true>(ctl, tmem, sV, ring, n, &ctl->mma_done_dp, abort_flag);
  } else if (warp == kBwAccWarp) {
    if (lane == 0) bw_mma_acc<true>(ctl, tmem, ring, n, abort_flag);
  } else {
    const int quarter = warp & 3;
    const int sub = (warp - 2) >> 2;  // the warp's part of its lane quarter's columns
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int t = kb * kBwRows + r;  // key position in the sample
    const size_t lrow = (static_cast<size_t>(s) * nh + h) * L;
    bool ok = bw_elementwise<true>(ctl, tmem, lane_off, sub, n, t, q0 * kBwCols, lse + lrow, Dsum + lrow, scale,
                                   abort_flag);
    if (ok) ok = __all_sync(0xFFFFFFFFu, mbar_wait(&ctl->acc_full, 0, abort_flag));
    bool bad = false;
    if (ok) {
      tc_fence_after();
      uint16_t* row = dqkv + static_cast<size_t>(row0 + t) * (3 * H);
      bad |= bw_store_rope(tmem + lane_off + kBwColAcc + kBwD, sub, t, cs, row + H + h * kBwD);  // dK
      float v[32];  // dV: this warp's 32 head columns
      tmem_ld32(tmem + lane_off + kBwColAcc + 32 * sub, v);
      bad |= bw_store32(row + 2 * H + h * kBwD + 32 * sub, v);
      tc_fence_before();
    }
    if (bad) raise_status(kStatusNonFinite);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kBwTmemCols);
  }
}

// dQ: CTA (query block qb of 128, head, sample); key blocks of 64 up to the diagonal.
__global__ void __launch_bounds__(kBwThreads, 1)
    attn_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tmBig, const __grid_constant__ CUtensorMap tmDOBig,
                          const __grid_constant__ CUtensorMap tmK64, const float* __restrict__ lse,
                          const float* __restrict__ Dsum, const float2* __restrict__ cs, int H, int L, int nh,
                          float scale, uint16_t* __restrict__ dqkv) {
  extern __shared__ uint8_t bw_smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(bw_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;
  uint8_t* sDO = sQ + kBwBig;
  uint8_t* ring = sDO + kBwBig;
  BwCtl* ctl = reinterpret_cast<BwCtl*>(ring + kBwStages * 2 * kBwSmall);
  volatile int* abort_flag = &ctl->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = L / kBwRows - 1 - static_cast<int>(blockIdx.x);  // the longest rows first
  const int h = blockIdx.y, s = blockIdx.z;
  const int row0 = s * L;
  const int n = 2 * (qb + 1);  // 64-key blocks up to the diagonal
  if (threadIdx.x == 0) bw_init(ctl);
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmBig);
    tma_prefetch_desc(&tmDOBig);
    tma_prefetch_desc(&tmK64);
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, kBwTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  if (warp == 0) {
    if (lane == 0) {
      // resident: Q from qkv and dO (its own map); bw_produce takes both from one map, so load dO here
      mbar_arrive_expect_tx(&ctl->res_full, 2 * kBwBig);
      tma_load_2d(sQ, &tmBig, &ctl->res_full, h * kBwD, row0 + qb * kBwRows);
      tma_load_2d(sQ + kBwBig / 2, &tmBig, &ctl->res_full, h * kBwD + 64, row0 + qb * kBwRows);
      tma_load_2d(sDO, &tmDOBig, &ctl->res_full, h * kBwD, row0 + qb * kBwRows);
      tma_load_2d(sDO + kBwBig / 2, &tmDOBig, &ctl->res_full, h * kBwD + 64, row0 + qb * kBwRows);
      uint32_t issued = 0;
      for (int j = 0; j < n; ++j) {
        const uint32_t slot = static_cast<uint32_t>(j) % kBwStages;
        if (!mbar_wait(&ctl->empty[slot], ((static_cast<uint32_t>(j) / kBwStages) & 1u) ^ 1u, abort_flag)) break;
        uint8_t* dst = ring + slot * 2 * kBwSmall;
        const int row = row0 + kBwCols * j;
        mbar_arrive_expect_tx(&ctl->full[slot], 2 * kBwSmall);
        tma_load_2d(dst, &tmK64, &ctl->full[slot], H + h * kBwD, row);                            // K
        tma_load_2d(dst + kBwSmall / 2, &tmK64, &ctl->full[slot], H + h * kBwD + 64, row);
        tma_load_2d(dst + kBwSmall, &tmK64, &ctl->full[slot], 2 * H + h * kBwD, row);             // V
        tma_load_2d(dst + kBwSmall + kBwSmall / 2, &tmK64, &ctl->full[slot], 2 * H + h * kBwD + 64, row);
        ++issued;
      }
      mbar_wait_drain(&ctl->res_full, 0);
      for (uint32_t i = issued > kBwStages ? issued - kBwStages : 0; i < issued; ++i)
        mbar_wait_drain(&ctl->full[i % kBwStages], (i / kBwStages) & 1u);
    }
  } else if (warp == 1) {
    if (lane == 0) bw_mma_st<false>(ctl, tmem, sQ, ring, n, &ctl->mma_done, abort_flag);
  } else if (warp == kBwDpWarp) {
    if (lane == 0) bw_mma_st<true>(ctl, tmem, sDO, ring, n, &ctl->mma_done_dp, abort_flag);
  } else if (warp == kBwAccWarp) {
    if (lane == 0) bw_mma_acc<false>(ctl, tmem, ring, n, abort_flag);
  } else {
    const int quarter = warp & 3;
    const int sub = (warp - 2) >> 2;  // the warp's part of its lane quarter's columns
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int t = qb * kBwRows + r;  // query position in the sample
    const size_t lrow = (static_cast<size_t>(s) * nh + h) * L;
    bool ok = bw_elementwise<false>(ctl, tmem, lane_off, sub, n, t, 0, lse + lrow, Dsum + lrow, scale, abort_flag);
    if (ok) ok = __all_sync(0xFFFFFFFFu, mbar_wait(&ctl->acc_full, 0, abort_flag));
    bool bad = false;
    if (ok) {
      tc_fence_after();
      uint16_t* row = dqkv + static_cast<size_t>(row0 + t) * (3 * H);
      bad |= bw_store_rope(tmem + lane_off + kBwColAcc, sub, t, cs, row + h * kBwD);  // dQ
      tc_fence_before();
    }
    if (bad) raise_status(kStatusNonFinite);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kBwTmemCols);
  }
}

}  // namespace

// dQ, dK, dV of causal attention for head dimension 128 and L % 128 == 0 (qkv,
// dO bf16; lse and Dsum fp32 [S][H / 128][L], Dsum already holding rowsum(dO O);
// cs the rotary table [L][64]; dqkv bf16 [S L][3 H]).  cudaErrorNotSupported for
// other shapes.
cudaError_t launch_attn_bwd_tc(const uint16_t* qkv, const uint16_t* dO, const float* lse, const float* Dsum,
                               const float* rope_cs, int S, int L, int H, uint16_t* dqkv, cudaStream_t st) {
  if (L % kBwRows != 0 || H % kBwD != 0 || L <= 0 || S <= 0) return cudaErrorNotSupported;
  const uint64_t M = static_cast<uint64_t>(S) * L;
  CUtensorMap tmBig, tm64, tmDOBig, tmDO64;
  cudaError_t e = make_tmap_2d(&tmBig, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, qkv, M, 3ull * H, 64, kBwRows,
                               CU_TENSOR_MAP_SWIZZLE_128B);
  if (e == cudaSuccess)
    e = make_tmap_2d(&tm64, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, qkv, M, 3ull * H, 64, kBwCols, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e == cudaSuccess)
    e = make_tmap_2d(&tmDOBig, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dO, M, H, 64, kBwRows, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e == cudaSuccess)
    e = make_tmap_2d(&tmDO64, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dO, M, H, 64, kBwCols, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(attn_bwd_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kBwSmem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attn_bwd_dkdv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kBwSmem);
  if (e != cudaSuccess) return e;
  const int nh = H / kBwD;
  const float scale = 1.0f / sqrtf(static_cast<float>(kBwD));
  const float2* cs = reinterpret_cast<const float2*>(rope_cs);
  {
    LaunchScope scope(st, "attn_bwd_dq_tc_kernel<d128>");
    attn_bwd_dq_tc_kernel<<<dim3(L / kBwRows, nh, S), kBwThreads, kBwSmem, st>>>(tmBig, tmDOBig, tm64, lse, Dsum, cs,
                                                                                 H, L, nh, scale, dqkv);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  {
    LaunchScope scope(st, "attn_bwd_dkdv_tc_kernel<d128>");
    attn_bwd_dkdv_tc_kernel<<<dim3(L / kBwRows, nh, S), kBwThreads, kBwSmem, st>>>(tmBig, tm64, tmDO64, lse, Dsum,
                                                                                   cs, H, L, nh, scale, dqkv);
  }
  return cudaGetLastError();
}

}  // namespace ar
