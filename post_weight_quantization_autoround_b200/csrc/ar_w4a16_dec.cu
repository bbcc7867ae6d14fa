// W4A16 matmul for decode batches (T <= 16 tokens), one CTA per SM over a
// contiguous range of weight rows: out[t][n] = sum_k A[t][k] (q[n][k] - z) s.
//
// [AR] §4 (comparison table, "Real INT4 Kernel" column): the weights stay
// 4-bit in memory and are dequantized inside the kernel, activations are
// 16-bit ([AR] = "Low-Bit Quantization in Practice with vLLM: Core Mechanisms
// and Architectural Optimizations of AutoRound").
//
// At T <= 16 the kernel moves 0.5 byte per weight from HBM and its cost on the
// SM is the 4-bit -> bf16 conversion (about 7 integer instructions per eight
// codes).  The layout is chosen so that nothing else costs per weight:
//
//  * Rows are handed out in groups of eight, so every SM owns the same number
//    of rows (8192 rows -> 147 CTAs of 56 rows).  Up to 8 tokens, the weights
//    are the A operand of mma.sync m16n8k16 (a 16-row tile is two row groups;
//    each lane converts one word of row g and one of row g + 8, so a word
//    costs one MMA) and the activations the B operand (8 token columns,
//    columns past T repeat the last token and are discarded).  From 9 to 16
//    tokens the roles swap: the weights are the B operand (an n8 tile is one
//    row group, two MMAs a word) and the activations the A operand (16 token
//    rows).
//  * Codes -> bf16 pairs without arithmetic: (word >> 4i) & 0x000F000F |
//    0x43004300 is the bf16 pair (128 + q_i, 128 + q_{i+4}).  One more MMA
//    against a fragment of ones gives O = sum of the activations over the same
//    k, so a group's contribution is s (D - (128 + z) O), applied once per
//    group span in fp32.
//  * The reduction index of the MMA is permuted: lane (g = lane/4, c = lane%4)
//    feeds k-slots {2c, 2c+1, 2c+8, 2c+9} of two consecutive MMAs from one
//    32-bit word (eight codes, k = 32j + 8c + 0..7) of a weight row, and the
//    activations are permuted the same way with byte permutes.  Both operand
//    arrangements use the same k-slots, so they give bit-identical sums.
//  * One producer warp streams stages of 1024 k (up to 8 tokens, where four
//    stages fit in shared memory) or 512 k with TMA: the codes of the pass's
//    rows (256-k boxes, 128-byte swizzle, so that the fragment reads are free
//    of bank conflicts), the activations, and the window of fp16 (scale, zero)
//    groups the stage touches.  Consumer warps work in groups of four (one
//    quarter of the stage each) and the groups take stages in turn, so each
//    warp owns whole group spans of its chunk.  The costs per stage (barrier
//    waits, the table boxes) are what 1024-k stages halve: 42 -> 36 us for the
//    8192 x 28672 layer at T = 1.  The ring depth is a multiple
//    of the number of groups, so a slot is always taken by the same group and
//    its waits on the slot's barrier follow the barrier's phases in order (a
//    parity wait cannot tell a phase from the one two before it: were two
//    groups to share a slot, one could pass its wait on a fill that another
//    group's previous phase completed).
//  * A CTA's rows are cut into passes of at most 64; the consumer warps' sums
//    are added in a fixed order through shared memory at the end of a pass.
//    For small N the two CTAs of a cluster split K and rank 0 adds the
//    partial sums in a fixed order through distributed shared memory.
//    Results are deterministic and no workspace is needed.
//
// Packed layout (as ar_pack_int4 writes it): uint32 [N][K/8], element k at
// bits 4*(k mod 8) of word k/8; scale/zero fp16 [N][K/g].
//
// The same kernel takes 2-bit codes (ar_pack_codes' stream: element k at bits
// 2*(k mod 16) of word k/16) up to 8 tokens for g >= 64.  A stage is 1024 k
// (two 128-byte boxes per row), or 2048 k for one token at g >= 128 where four
// such stages fit (30.8 against 32.8 us on the 8192 x 28672 layer), and a
// lane's 32-bit word holds 16 codes, so a warp's quarter of a stage is 64-k
// slices of four MMAs each (weights as the A operand).  The codes are not
// shifted down one by one: (x & (3 << 2m)) | 0x4300 for
// m = 0, 1, 2 is the bf16 128 + 4^m q, since bits 0..6 are the mantissa of a
// bf16 in [128, 256), so one word needs two shifts (by 6 and 12) and eight
// logic ops to give its eight pairs (q_i, q_{i+8}).  The activation paired
// with a code at scale 4^m is multiplied by 4^-m (exact in bf16), so each
// product is (128 / 4^m) a + q a.  One MMA of the scaled activations against a
// constant fragment gives both corrections: rows 0..7 hold the class weights
// 4^m (Oa = sum of a), rows 8..15 ones (Ob = sum of a / 4^m), and a group adds
// s (D - 128 Ob) - s z Oa.
//
// 8-bit codes (T <= 8; 512-k stages, four boxes per row) are split into their
// nibbles: (x & 0x000F000F) | 0x4300 is (128 + lo_0, 128 + lo_2), and
// ((x >> 1) & 0x00780078) | 0x4300, the high nibbles at mantissa bits 3..6, is
// (128 + 8 hi_0, 128 + 8 hi_2), paired with doubled activations; a code then
// contributes 384 a + q a, and a group adds s D - s (384 + z) O.
//
// 3-bit codes (T <= 8, g >= 64; 1024-k stages, three boxes per row): a lane's
// 16 codes are 6 bytes of the bit stream, read as the two aligned words that
// hold them and funnel-shifted into place; two byte permutes put codes 0..7
// and 8..15 side by side, and masks at mantissa bits 0-2 and 3-5 give the
// pairs at scales 1 and 8, corrected as at 2 bits.
#include <cooperative_groups.h>

#include <cstdio>

#include "ar_internal.h"

namespace cg = cooperative_groups;

namespace ar {
namespace {

constexpr int kDecStageK = 512;                 // k per stage
constexpr int kDecPassRows = 64;                // rows per pass (eight n8 tiles)
constexpr int kDecCodeBox = kDecPassRows * 128; // one 256-k box of codes: 64 rows x 128 bytes
constexpr int kDecMaxStages = 8;               // ring depth cap, 4-bit codes (two boxes per stage)
constexpr int kDecMaxStages2 = 16;             // ... 2-bit codes
constexpr int kDecSmemLimit = 227 * 1024;

template <bool TBIG>
struct DecCfg {
  static constexpr int kWarps = 8;              // consumer warps
  static constexpr int kGroups = kWarps / 4;    // stages in consumption at once
  static constexpr int kThreads = (kWarps + 1) * 32;
  // registers per thread: the warps are spread over the SM's four 16K-register
  // partitions, so the partition with the most warps (ceil(warps / 4)) sets the cap
  static constexpr int kMaxRegs = ((16384 / (32 * ((kWarps + 1 + 3) / 4))) / 8) * 8;
  static constexpr int kTokPad = TBIG ? 16 : 8;
  static constexpr int kAcc = TBIG ? 4 : 2;     // accumulators per n8 tile and lane
  static constexpr int kRedBytes = kWarps * kDecPassRows * kTokPad * 4;
};

struct DecParams {
  int N, K, T;
  int rows_per_cta;  // multiple of 8
  int passes;        // ceil(rows_per_cta / 64)
  int last_rows;     // box height of the last pass
  int n_stages;      // ceil(K / 512)
  int group_shift;
  int wg;            // groups per table window (8, or 16 when g = 32)
  int act_off;       // stage layout: codes at 0, activations, scale table, zero table
  int tab_off;
  int stage_bytes;
  int S;             // ring depth
};

struct alignas(16) DecTail {
  float2 sm[8][kDecPassRows];   // per consumer warp: (s, -s (128 + z)) of the pass's rows for one group
  uint64_t full[kDecMaxStages2];
  uint64_t empty[kDecMaxStages2];
  float part[kDecPassRows][16];
  int abort_flag;
};

__host__ __device__ constexpr int dec_tail_offset(int S, int stage_bytes, int red_bytes) {
  return S * stage_bytes + red_bytes;
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Same with a zero accumulator input (the first MMA of a group span).
__device__ __forceinline__ void mma16816_z(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%10, %10, %10, %10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
}

// (x & 0x000F000F) | 0x43004300 as one three-input logic op: the bf16 pair
// (128 + nibble 0, 128 + nibble 4) of x.
__device__ __forceinline__ uint32_t nib_pair(uint32_t x) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(x), "r"(0x000F000Fu), "r"(0x43004300u));
  return d;
}

__device__ __forceinline__ uint32_t shr(uint32_t x, uint32_t n) {
  uint32_t d;
  asm("shf.r.clamp.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(x), "r"(0u), "r"(n));
  return d;
}

// (x & m) | 0x43004300 for a mask m inside bits 0..5 of each half: the bf16
// pair (128 + code, 128 + code') scaled by the mask's position.
template <uint32_t M>
__device__ __forceinline__ uint32_t mask_pair(uint32_t x) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(x), "r"(M), "r"(0x43004300u));
  return d;
}

// The eight bf16 pairs of one word of 2-bit codes: r[i] = (128 + s_i q_i,
// 128 + s_i q_{i+8}) with s = (1, 4, 16, 1, 4, 16, 1, 4).
__device__ __forceinline__ void two_bit_pairs(uint32_t x, uint32_t (&r)[8]) {
  const uint32_t y = shr(x, 6);
  const uint32_t z = shr(x, 12);
  r[0] = mask_pair<0x00030003u>(x);
  r[1] = mask_pair<0x000C000Cu>(x);
  r[2] = mask_pair<0x00300030u>(x);
  r[3] = mask_pair<0x00030003u>(y);
  r[4] = mask_pair<0x000C000Cu>(y);
  r[5] = mask_pair<0x00300030u>(y);
  r[6] = mask_pair<0x00030003u>(z);
  r[7] = mask_pair<0x000C000Cu>(z);
}

// The eight bf16 pairs of 16 consecutive 3-bit codes that start at bit `sh` (0 or 16) of the
// 64-bit value (w1:w0): r[i] = (128 + s_i q_i, 128 + s_i q_{i+8}) with s = (1, 8, 1, 8, ...).
// u holds codes 0..7 at bits 3i, v codes 8..15; a byte permute puts the low 16 bits of each side
// by side, so each half carries codes at bits 0-2 and 3-5, both inside a bf16 mantissa.
__device__ __forceinline__ void three_bit_pairs(uint32_t w0, uint32_t w1, uint32_t sh, uint32_t (&r)[8]) {
  const uint32_t u = __funnelshift_r(w0, w1, sh);
  const uint32_t v = __funnelshift_r(u, shr(w1, sh), 24);
  const uint32_t a = __byte_perm(u, v, 0x5410);                    // codes 0, 1 | 8, 9 (+ 2, 3 | 10, 11 above)
  const uint32_t b = __byte_perm(shr(u, 12), shr(v, 12), 0x5410);  // codes 4, 5 | 12, 13 (+ 6, 7 | 14, 15)
  const uint32_t a6 = shr(a, 6), b6 = shr(b, 6);
  r[0] = mask_pair<0x00070007u>(a);
  r[1] = mask_pair<0x00380038u>(a);
  r[2] = mask_pair<0x00070007u>(a6);
  r[3] = mask_pair<0x00380038u>(a6);
  r[4] = mask_pair<0x00070007u>(b);
  r[5] = mask_pair<0x00380038u>(b);
  r[6] = mask_pair<0x00070007u>(b6);
  r[7] = mask_pair<0x00380038u>(b6);
}

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ float half_bits_to_float(uint16_t h) { return __half2float(__ushort_as_half(h)); }

// TBIG: 9..16 tokens (token rows g and g + 8 of the A fragment both live).
// SPAN: slices per group span inside a 128-k chunk; 4-bit codes: 32-k slices (4
// for g >= 128, 2 for g = 64, 1 for g = 32), 2-bit codes: 64-k slices (2 for
// g >= 128, 1 for g = 64).  KS: CTAs of a cluster splitting K (1 or 2).  NT: n8
// tiles per pass, a compile-time count so that the tile loops are straight-line
// code (tiles past a pass's rows read rows of the stage buffer that the pass
// does not own and are computed but never stored).  BITS: 4, or 2 (T <= 8 only).
template <bool TBIG, int SPAN, int KS, int NT, int BITS, int STAGEK>
__global__ void __maxnreg__(DecCfg<TBIG>::kMaxRegs)
    w4a16_dec_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmWl,
                     const __grid_constant__ CUtensorMap tmS, const __grid_constant__ CUtensorMap tmSl,
                     const __grid_constant__ CUtensorMap tmZ, const __grid_constant__ CUtensorMap tmZl,
                     const __grid_constant__ CUtensorMap tmA, const DecParams p, uint16_t* __restrict__ out) {
  using C = DecCfg<TBIG>;
  static_assert(BITS == 4 || ((BITS == 2 || BITS == 3 || BITS == 8) && !TBIG),
                "4-bit codes, or 2, 3 or 8-bit codes up to 8 tokens");
  // k per stage (512 or 1024; 2-bit codes: 1024); a stage holds kStageK * BITS / 1024 128-byte
  // boxes of codes per row, contiguous in the row
  constexpr int kStageK = STAGEK;
  static_assert(BITS == 4   ? (kStageK == 512 || kStageK == 1024)
                : BITS == 2 ? (kStageK == 1024 || kStageK == 2048)
                : BITS == 3 ? kStageK == 1024
                            : kStageK == 512,
                "stage size");
  constexpr int kCodeBoxes = kStageK * BITS / 1024;
  constexpr int kActBoxes = kStageK / 256;  // 256-k boxes of activations per stage
  extern __shared__ uint8_t dec_smem_raw[];
  // 1024-byte aligned base by pointer arithmetic on the shared array, so that
  // every access below stays a shared-memory access (ld.shared)
  uint8_t* smem = dec_smem_raw + ((1024u - (smem_u32(dec_smem_raw) & 1023u)) & 1023u);
  float* red = reinterpret_cast<float*>(smem + p.S * p.stage_bytes);  // [warp][row][token]
  DecTail& tl = *reinterpret_cast<DecTail*>(smem + dec_tail_offset(p.S, p.stage_bytes, C::kRedBytes));
  volatile int* abort_flag = &tl.abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = KS == 2 ? static_cast<int>(cluster_ctarank()) : 0;
  const int row_base = (blockIdx.x / KS) * p.rows_per_cta;
  const int rows_here = min(p.rows_per_cta, p.N - row_base);
  const int passes_here = (rows_here + kDecPassRows - 1) / kDecPassRows;
  const int ks0 = (p.n_stages * rank) / KS;
  const int nks = (p.n_stages * (rank + 1)) / KS - ks0;  // stages of one pass
  const int total = passes_here * nks;
  const int S = p.S;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&tl.full[s], 1);
      mbar_init(&tl.empty[s], 4);
    }
    tl.abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == C::kWarps) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmW);
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmS);
      tma_prefetch_desc(&tmZ);
      int issued = 0;
      for (int it = 0; it < total; ++it) {
        const int s = it % S;
        const uint32_t ph = static_cast<uint32_t>(it / S) & 1u;
        if (!mbar_wait_sleep(&tl.empty[s], ph ^ 1u, abort_flag)) break;
        const int pass = it / nks;
        const int ks = ks0 + (it - pass * nks);
        const bool last = pass == p.passes - 1;
        const int h = last ? p.last_rows : kDecPassRows;
        const int row0 = row_base + pass * kDecPassRows;
        uint8_t* st = smem + s * p.stage_bytes;
        const int gi0 = (ks * kStageK) >> p.group_shift;
        const int x0 = p.wg >= 16 ? gi0 : (gi0 & ~7);
        mbar_arrive_expect_tx(&tl.full[s], static_cast<uint32_t>(kCodeBoxes * 128 * h + kActBoxes * 512 * p.T +
                                                                 2 * 2 * p.wg * h));
        // kStageK * BITS / 32 words of codes per row and stage, in boxes of 32
#pragma unroll
        for (int b = 0; b < kCodeBoxes; ++b)
          tma_load_2d(st + b * kDecCodeBox, last ? &tmWl : &tmW, &tl.full[s], ks * 32 * kCodeBoxes + 32 * b, row0);
#pragma unroll
        for (int b = 0; b < kActBoxes; ++b)
          tma_load_2d(st + p.act_off + b * 512 * p.T, &tmA, &tl.full[s], ks * kStageK + 256 * b, 0);
        tma_load_2d(st + p.tab_off, last ? &tmSl : &tmS, &tl.full[s], x0, row0);
        tma_load_2d(st + p.tab_off + 2 * p.wg * kDecPassRows, last ? &tmZl : &tmZ, &tl.full[s], x0, row0);
        ++issued;
      }
      const int first = issued > S ? issued - S : 0;
      for (int i = first; i < issued; ++i) mbar_wait_drain(&tl.full[i % S], static_cast<uint32_t>(i / S) & 1u);
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int cw = warp & 3;     // 128-k chunk of the stage
    const int grp = warp >> 2;   // stages it == grp (mod kGroups)
    const int g = lane >> 2;
    const int c = lane & 3;
    const int T = p.T;
    const int tok_lo = min(g, T - 1);
    const int tok_hi = min(g + 8, T - 1);
    const int kw0 = cw * (kStageK / 4);  // k offset of the warp's quarter of a stage
    const uint32_t kOne2 = 0x3F803F80u;  // bf16 pair (1, 1)
    bool ok = true;

    float2* smw = tl.sm[warp];
    for (int pass = 0; pass < passes_here; ++pass) {
      const bool last = pass == p.passes - 1;
      const int h = min(last ? p.last_rows : kDecPassRows, rows_here - pass * kDecPassRows);
      // T <= 8: MT 16-row tiles x (row g, g + 8) x (token 2c, 2c + 1); else NT row groups x kAcc
      constexpr int MT = (NT + 1) / 2;
      constexpr int kTiles = TBIG ? NT : MT;
      constexpr int kAccN = TBIG ? C::kAcc : 4;
      float acc[kTiles][kAccN];
#pragma unroll
      for (int jt = 0; jt < kTiles; ++jt)
#pragma unroll
        for (int i = 0; i < kAccN; ++i) acc[jt][i] = 0.0f;

      const int it_begin = pass * nks;
      const int it_end = it_begin + nks;
      int it = it_begin + ((grp - it_begin % C::kGroups) + C::kGroups) % C::kGroups;
      for (; it < it_end; it += C::kGroups) {
        const int s = it % S;
        const uint32_t ph = static_cast<uint32_t>(it / S) & 1u;
        if (ok) ok = mbar_wait_sleep(&tl.full[s], ph, abort_flag);
        if (__all_sync(0xFFFFFFFFu, ok)) {
          const int ks = ks0 + (it - it_begin);
          const uint8_t* st = smem + s * p.stage_bytes;
          // 4-bit codes: a box is 256 k of a row; activations: a box is 256 k of each token
          const uint8_t* codes = st + (kw0 >> 8) * kDecCodeBox + g * 128 + 4 * c;
          const uint8_t* act = st + p.act_off + (kw0 >> 8) * 512 * T + (((kw0 & 255) + 8 * c) * 2);
          const uint16_t* sc = reinterpret_cast<const uint16_t*>(st + p.tab_off);
          const uint16_t* zr = sc + p.wg * kDecPassRows;
          const int gi0 = (ks * kStageK) >> p.group_shift;
          const int x0 = p.wg >= 16 ? gi0 : (gi0 & ~7);
          if constexpr (BITS == 8) {
            // weights as the A operand as below; warp cw takes k kw0 .. kw0 + 127 (code box cw of
            // 128 k, half of activation box cw / 2).  Per 16-k chunk j a lane takes word c of the
            // chunk (codes k = 16 j + 4 c + 0..3) of its rows; each code is split into nibbles:
            // (x & 0x000F000F) | 0x4300 is the pair (128 + lo_0, 128 + lo_2) and
            // ((x >> 1) & 0x00780078) | 0x4300 the pair (128 + 8 hi_0, 128 + 8 hi_2), paired with
            // the activations (a_0, a_2) and (2 a_0, 2 a_2) in k-slots (2c, 2c+1) and (2c+8, 2c+9) of
            // MMA 0 (codes 1, 3 likewise in MMA 1), so a code contributes 384 a + q a
            float d[MT][4], o[4];
            const uint8_t* codes8 = st + (kw0 >> 7) * kDecCodeBox + g * 128 + 4 * c;
            const uint8_t* act8 = st + p.act_off + (kw0 >> 8) * 512 * T + ((kw0 & 255) + 4 * c) * 2;
            constexpr uint32_t kTwo2 = 0x40004000u;  // bf16 pair (2, 2)
#pragma unroll
            for (int j = 0; j < kStageK / 64; ++j) {
              const uint2 v = *reinterpret_cast<const uint2*>(act8 + tok_lo * 512 + 32 * j);
              const uint32_t p02 = __byte_perm(v.x, v.y, 0x5410);  // (a_0, a_2)
              const uint32_t p13 = __byte_perm(v.x, v.y, 0x7632);  // (a_1, a_3)
              const uint32_t b0[2] = {p02, bf16x2_mul(p02, kTwo2)};
              const uint32_t b1[2] = {p13, bf16x2_mul(p13, kTwo2)};
              const bool first = (j % SPAN) == 0;
              {
                // O = sum of the activations: ones against the low-nibble slots, zeros against the high
                const uint32_t ones[4] = {kOne2, kOne2, 0u, 0u};
                if (first) {
                  mma16816_z(o, ones, b0[0], b0[1]);
                } else {
                  mma16816(o, ones, b0[0], b0[1]);
                }
                mma16816(o, ones, b1[0], b1[1]);
              }
              const uint8_t* cj = codes8 + ((((kw0 & 127) >> 4) + j) ^ g) * 16;
#pragma unroll
              for (int mt = 0; mt < MT; ++mt) {
                const bool pair = 2 * mt + 1 < NT;
                const uint32_t xg = *reinterpret_cast<const uint32_t*>(cj + (2 * mt) * 8 * 128);
                const uint32_t xh = pair ? *reinterpret_cast<const uint32_t*>(cj + (2 * mt + 1) * 8 * 128) : 0u;
                const uint32_t yg = shr(xg, 8), yh = shr(xh, 8);
                uint32_t a0[4], a1[4];
                a0[0] = nib_pair(xg);
                a0[2] = mask_pair<0x00780078u>(shr(xg, 1));
                a1[0] = nib_pair(yg);
                a1[2] = mask_pair<0x00780078u>(shr(xg, 9));
                if (pair) {
                  a0[1] = nib_pair(xh);
                  a0[3] = mask_pair<0x00780078u>(shr(xh, 1));
                  a1[1] = nib_pair(yh);
                  a1[3] = mask_pair<0x00780078u>(shr(xh, 9));
                } else {
                  a0[1] = a0[3] = a1[1] = a1[3] = 0u;
                }
                if (first) {
                  mma16816_z(d[mt], a0, b0[0], b0[1]);
                } else {
                  mma16816(d[mt], a0, b0[0], b0[1]);
                }
                mma16816(d[mt], a1, b1[0], b1[1]);
              }
              if ((j % SPAN) == SPAN - 1) {
                // group span done: acc += s D - s (384 + z) O for rows g, g + 8 of each tile
                const int gl = ((ks * kStageK + kw0 + 16 * (j - SPAN + 1)) >> p.group_shift) - x0;
                __syncwarp();
#pragma unroll
                for (int rr = 0; rr < (8 * NT + 31) / 32; ++rr) {
                  const int row = lane + 32 * rr;
                  if (row < 8 * NT) {
                    const float sv = half_bits_to_float(sc[row * p.wg + gl]);
                    const float zv = half_bits_to_float(zr[row * p.wg + gl]);
                    smw[row] = make_float2(sv, -sv * (384.0f + zv));
                  }
                }
                __syncwarp();
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                  const float2 mg = smw[16 * mt + g];
                  acc[mt][0] = fmaf(mg.x, d[mt][0], fmaf(mg.y, o[0], acc[mt][0]));
                  acc[mt][1] = fmaf(mg.x, d[mt][1], fmaf(mg.y, o[1], acc[mt][1]));
                  if (2 * mt + 1 < NT) {
                    const float2 mh = smw[16 * mt + 8 + g];
                    acc[mt][2] = fmaf(mh.x, d[mt][2], fmaf(mh.y, o[2], acc[mt][2]));
                    acc[mt][3] = fmaf(mh.x, d[mt][3], fmaf(mh.y, o[3], acc[mt][3]));
                  }
                }
              }
            }
          } else if constexpr (BITS == 3) {
            // weights as the A operand as below.  A row's 1024-k stage is 384 bytes (three boxes);
            // warp cw takes its bytes 96 cw .. 96 cw + 95.  Per 64-k slice j (24 bytes) lane c takes
            // the 16 codes at bytes 24 j + 6 c .. + 5 of that range (k = 64 j + 16 c + 0..15), read as
            // the two aligned words that hold them; pair i of the lane (codes i, i + 8) feeds k-slots
            // (2c, 2c+1) of MMA i/2 when i is even, (2c+8, 2c+9) when odd, as at 2 bits
            float d[MT][4], o[4];
            const uint8_t* row3 = st + g * 128;
            const uint8_t* act3 = st + p.act_off + 16 * c * 2;
            constexpr uint32_t kEighth2 = 0x3E003E00u;  // bf16 pair (1/8, 1/8)
            constexpr uint32_t kEight2 = 0x41004100u;   // (8, 8)
#pragma unroll
            for (int j = 0; j < kStageK / 256; ++j) {
              const int kj = kw0 + 64 * j;
              const uint8_t* aj = act3 + (kj >> 8) * 512 * T + (kj & 255) * 2 + tok_lo * 512;
              const uint4 v = *reinterpret_cast<const uint4*>(aj);
              const uint4 u = *reinterpret_cast<const uint4*>(aj + 16);
              uint32_t b[8];
              b[0] = __byte_perm(v.x, u.x, 0x5410);
              b[1] = bf16x2_mul(__byte_perm(v.x, u.x, 0x7632), kEighth2);
              b[2] = __byte_perm(v.y, u.y, 0x5410);
              b[3] = bf16x2_mul(__byte_perm(v.y, u.y, 0x7632), kEighth2);
              b[4] = __byte_perm(v.z, u.z, 0x5410);
              b[5] = bf16x2_mul(__byte_perm(v.z, u.z, 0x7632), kEighth2);
              b[6] = __byte_perm(v.w, u.w, 0x5410);
              b[7] = bf16x2_mul(__byte_perm(v.w, u.w, 0x7632), kEighth2);
              const bool first = (j % SPAN) == 0;
              {
                // rows 0..7: Oa = sum of a (class weights 1, 8); rows 8..15: Ob = sum of the scaled a
                const uint32_t c0[4] = {kOne2, kOne2, kEight2, kOne2};
                if (first) {
                  mma16816_z(o, c0, b[0], b[1]);
                } else {
                  mma16816(o, c0, b[0], b[1]);
                }
                mma16816(o, c0, b[2], b[3]);
                mma16816(o, c0, b[4], b[5]);
                mma16816(o, c0, b[6], b[7]);
              }
              // the lane's two aligned words: byte x of the row segment is in box x / 128, 16-byte
              // chunk (x % 128) / 16 stored at chunk ((x % 128) / 16) ^ (row % 8)
              const int x = ((kw0 * 3) >> 3) + 24 * j + 6 * c;
              const int x0w = x & ~3, x1w = x0w + 4;
              const int off0 = (x0w >> 7) * kDecCodeBox + ((((x0w & 127) >> 4) ^ g) << 4) + (x0w & 15);
              const int off1 = (x1w >> 7) * kDecCodeBox + ((((x1w & 127) >> 4) ^ g) << 4) + (x1w & 15);
              const uint32_t sh = static_cast<uint32_t>(x & 3) * 8u;
#pragma unroll
              for (int mt = 0; mt < MT; ++mt) {
                const bool pair = 2 * mt + 1 < NT;
                const uint8_t* rg = row3 + (2 * mt) * 8 * 128;
                uint32_t qg[8], qh[8];
                three_bit_pairs(*reinterpret_cast<const uint32_t*>(rg + off0),
                                *reinterpret_cast<const uint32_t*>(rg + off1), sh, qg);
                if (pair) {
                  const uint8_t* rh = rg + 8 * 128;
                  three_bit_pairs(*reinterpret_cast<const uint32_t*>(rh + off0),
                                  *reinterpret_cast<const uint32_t*>(rh + off1), sh, qh);
                } else {
#pragma unroll
                  for (int i = 0; i < 8; ++i) qh[i] = 0u;
                }
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                  const uint32_t a[4] = {qg[2 * m], qh[2 * m], qg[2 * m + 1], qh[2 * m + 1]};
                  if (first && m == 0) {
                    mma16816_z(d[mt], a, b[0], b[1]);
                  } else {
                    mma16816(d[mt], a, b[2 * m], b[2 * m + 1]);
                  }
                }
              }
              if ((j % SPAN) == SPAN - 1) {
                // group span done: acc += s (D - 128 Ob) - s z Oa, as at 2 bits
                const int gl = ((ks * kStageK + kw0 + 64 * (j - SPAN + 1)) >> p.group_shift) - x0;
                __syncwarp();
#pragma unroll
                for (int rr = 0; rr < (8 * NT + 31) / 32; ++rr) {
                  const int row = lane + 32 * rr;
                  if (row < 8 * NT) {
                    const float sv = half_bits_to_float(sc[row * p.wg + gl]);
                    const float zv = half_bits_to_float(zr[row * p.wg + gl]);
                    smw[row] = make_float2(sv, -sv * zv);
                  }
                }
                __syncwarp();
                const float ob0 = -128.0f * o[2];
                const float ob1 = -128.0f * o[3];
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                  const float2 mg = smw[16 * mt + g];
                  acc[mt][0] = fmaf(mg.x, d[mt][0] + ob0, fmaf(mg.y, o[0], acc[mt][0]));
                  acc[mt][1] = fmaf(mg.x, d[mt][1] + ob1, fmaf(mg.y, o[1], acc[mt][1]));
                  if (2 * mt + 1 < NT) {
                    const float2 mh = smw[16 * mt + 8 + g];
                    acc[mt][2] = fmaf(mh.x, d[mt][2] + ob0, fmaf(mh.y, o[0], acc[mt][2]));
                    acc[mt][3] = fmaf(mh.x, d[mt][3] + ob1, fmaf(mh.y, o[1], acc[mt][3]));
                  }
                }
              }
            }
          } else if constexpr (BITS == 2) {
            // weights as the A operand as below; warp cw takes the k range kw0 .. kw0 + kStageK / 4 - 1
            // of the stage (code boxes hold 512 k, activation boxes 256 k).  Per 64-k slice j a lane
            // takes word c of the slice's 16-byte chunk of its rows (codes k = 64 j + 16 c + 0..15
            // of the warp's range) and feeds pair i of the word (codes i, i + 8) to k-slots
            // (2c, 2c+1) of MMA i/2 when i is even, (2c+8, 2c+9) when odd
            float d[MT][4], o[4];
            const uint8_t* codes2 = st + (kw0 >> 9) * kDecCodeBox + g * 128 + 4 * c;
            const uint8_t* act2 = st + p.act_off + 16 * c * 2;
            constexpr uint32_t kQuarter2 = 0x3E803E80u;    // bf16 pair (1/4, 1/4)
            constexpr uint32_t kSixteenth2 = 0x3D803D80u;  // (1/16, 1/16)
            constexpr uint32_t kFour2 = 0x40804080u;       // (4, 4)
            constexpr uint32_t kSixteen2 = 0x41804180u;    // (16, 16)
#pragma unroll
            for (int j = 0; j < kStageK / 256; ++j) {
              // the lane's 16 activations of token column g, paired (k_i, k_{i+8}) and divided by
              // the scale of code pair i
              const int kj = kw0 + 64 * j;  // k of the slice in the stage: box kj / 256 of each token
              const uint8_t* aj = act2 + (kj >> 8) * 512 * T + (kj & 255) * 2 + tok_lo * 512;
              const uint4 v = *reinterpret_cast<const uint4*>(aj);
              const uint4 u = *reinterpret_cast<const uint4*>(aj + 16);
              uint32_t b[8];
              b[0] = __byte_perm(v.x, u.x, 0x5410);
              b[1] = bf16x2_mul(__byte_perm(v.x, u.x, 0x7632), kQuarter2);
              b[2] = bf16x2_mul(__byte_perm(v.y, u.y, 0x5410), kSixteenth2);
              b[3] = __byte_perm(v.y, u.y, 0x7632);
              b[4] = bf16x2_mul(__byte_perm(v.z, u.z, 0x5410), kQuarter2);
              b[5] = bf16x2_mul(__byte_perm(v.z, u.z, 0x7632), kSixteenth2);
              b[6] = __byte_perm(v.w, u.w, 0x5410);
              b[7] = bf16x2_mul(__byte_perm(v.w, u.w, 0x7632), kQuarter2);
              const bool first = (j % SPAN) == 0;
              {
                // rows 0..7: Oa = sum of the activations (the scale of each pair against its scaled
                // activations); rows 8..15: Ob = sum of the scaled activations (ones)
                const uint32_t c0[4] = {kOne2, kOne2, kFour2, kOne2};
                const uint32_t c1[4] = {kSixteen2, kOne2, kOne2, kOne2};
                const uint32_t c2[4] = {kFour2, kOne2, kSixteen2, kOne2};
                if (first) {
                  mma16816_z(o, c0, b[0], b[1]);
                } else {
                  mma16816(o, c0, b[0], b[1]);
                }
                mma16816(o, c1, b[2], b[3]);
                mma16816(o, c2, b[4], b[5]);
                mma16816(o, c0, b[6], b[7]);
              }
              const int q = ((kw0 & 511) >> 6) + j;
              const uint8_t* cj = codes2 + ((q ^ g) << 4);
#pragma unroll
              for (int mt = 0; mt < MT; ++mt) {
                const bool pair = 2 * mt + 1 < NT;
                uint32_t rg[8], rh[8];
                two_bit_pairs(*reinterpret_cast<const uint32_t*>(cj + (2 * mt) * 8 * 128), rg);
                if (pair) {
                  two_bit_pairs(*reinterpret_cast<const uint32_t*>(cj + (2 * mt + 1) * 8 * 128), rh);
                } else {
#pragma unroll
                  for (int i = 0; i < 8; ++i) rh[i] = 0u;
                }
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                  const uint32_t a[4] = {rg[2 * m], rh[2 * m], rg[2 * m + 1], rh[2 * m + 1]};
                  if (first && m == 0) {
                    mma16816_z(d[mt], a, b[0], b[1]);
                  } else {
                    mma16816(d[mt], a, b[2 * m], b[2 * m + 1]);
                  }
                }
              }
              if ((j % SPAN) == SPAN - 1) {
                // group span done: D = sum (128 / s_k) a_k + sum q a, so acc += s D - s z Oa -
                // 128 s Ob for rows g, g + 8 of each tile (o[0..1]: Oa, o[2..3]: Ob of tokens 2c, 2c+1)
                const int gl = ((ks * kStageK + kw0 + 64 * (j - SPAN + 1)) >> p.group_shift) - x0;
                __syncwarp();
#pragma unroll
                for (int rr = 0; rr < (8 * NT + 31) / 32; ++rr) {
                  const int row = lane + 32 * rr;
                  if (row < 8 * NT) {
                    const float sv = half_bits_to_float(sc[row * p.wg + gl]);
                    const float zv = half_bits_to_float(zr[row * p.wg + gl]);
                    smw[row] = make_float2(sv, -sv * zv);
                  }
                }
                __syncwarp();
                const float ob0 = -128.0f * o[2];
                const float ob1 = -128.0f * o[3];
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                  const float2 mg = smw[16 * mt + g];
                  acc[mt][0] = fmaf(mg.x, d[mt][0] + ob0, fmaf(mg.y, o[0], acc[mt][0]));
                  acc[mt][1] = fmaf(mg.x, d[mt][1] + ob1, fmaf(mg.y, o[1], acc[mt][1]));
                  if (2 * mt + 1 < NT) {
                    const float2 mh = smw[16 * mt + 8 + g];
                    acc[mt][2] = fmaf(mh.x, d[mt][2] + ob0, fmaf(mh.y, o[0], acc[mt][2]));
                    acc[mt][3] = fmaf(mh.x, d[mt][3] + ob1, fmaf(mh.y, o[1], acc[mt][3]));
                  }
                }
              }
            }
          } else if constexpr (!TBIG) {
            // weights as the A operand: tile mt holds row groups 2 mt and 2 mt + 1 (rows g and g + 8
            // of the lane); an odd last row group leaves the tile's lower half zero
            float d[MT][4], o[4];
#pragma unroll
            for (int j = 0; j < kStageK / 128; ++j) {
              // activations of this lane's k-range (eight bf16) for token column g
              const uint4 v = *reinterpret_cast<const uint4*>(act + tok_lo * 512 + 64 * j);
              const uint32_t b0[2] = {__byte_perm(v.x, v.z, 0x5410), __byte_perm(v.x, v.z, 0x7632)};  // (k0,k4) (k1,k5)
              const uint32_t b1[2] = {__byte_perm(v.y, v.w, 0x5410), __byte_perm(v.y, v.w, 0x7632)};  // (k2,k6) (k3,k7)
              const uint32_t ones[4] = {kOne2, kOne2, kOne2, kOne2};
              const bool first = (j % SPAN) == 0;
              if (first) {
                mma16816_z(o, ones, b0[0], b0[1]);
              } else {
                mma16816(o, ones, b0[0], b0[1]);
              }
              mma16816(o, ones, b1[0], b1[1]);
              const int q = ((kw0 & 255) >> 5) + j;
              const uint8_t* cj = codes + ((q ^ g) << 4);
#pragma unroll
              for (int mt = 0; mt < MT; ++mt) {
                const bool pair = 2 * mt + 1 < NT;
                const uint32_t xg = *reinterpret_cast<const uint32_t*>(cj + (2 * mt) * 8 * 128);
                const uint32_t xh = pair ? *reinterpret_cast<const uint32_t*>(cj + (2 * mt + 1) * 8 * 128) : 0u;
                // MMA 0: k-slots (2c, 2c+1) <- nibbles (0, 4), (2c+8, 2c+9) <- (1, 5); MMA 1: (2, 6), (3, 7)
                uint32_t a0[4], a1[4];
                a0[0] = nib_pair(xg);
                a0[2] = nib_pair(shr(xg, 4));
                a1[0] = nib_pair(shr(xg, 8));
                a1[2] = nib_pair(shr(xg, 12));
                if (pair) {
                  a0[1] = nib_pair(xh);
                  a0[3] = nib_pair(shr(xh, 4));
                  a1[1] = nib_pair(shr(xh, 8));
                  a1[3] = nib_pair(shr(xh, 12));
                } else {
                  a0[1] = a0[3] = a1[1] = a1[3] = 0u;
                }
                if (first) {
                  mma16816_z(d[mt], a0, b0[0], b0[1]);
                } else {
                  mma16816(d[mt], a0, b0[0], b0[1]);
                }
                mma16816(d[mt], a1, b1[0], b1[1]);
              }
              if ((j % SPAN) == SPAN - 1) {
                // group span done: acc += s D - s (128 + z) O for rows g, g + 8 of each tile
                const int gl = ((ks * kStageK + kw0 + 32 * (j - SPAN + 1)) >> p.group_shift) - x0;
                __syncwarp();
#pragma unroll
                for (int rr = 0; rr < (8 * NT + 31) / 32; ++rr) {
                  const int row = lane + 32 * rr;
                  if (row < 8 * NT) {
                    const float sv = half_bits_to_float(sc[row * p.wg + gl]);
                    const float zv = half_bits_to_float(zr[row * p.wg + gl]);
                    smw[row] = make_float2(sv, -sv * (128.0f + zv));
                  }
                }
                __syncwarp();
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                  const float2 mg = smw[16 * mt + g];
                  acc[mt][0] = fmaf(mg.x, d[mt][0], fmaf(mg.y, o[0], acc[mt][0]));
                  acc[mt][1] = fmaf(mg.x, d[mt][1], fmaf(mg.y, o[1], acc[mt][1]));
                  if (2 * mt + 1 < NT) {
                    const float2 mh = smw[16 * mt + 8 + g];
                    acc[mt][2] = fmaf(mh.x, d[mt][2], fmaf(mh.y, o[2], acc[mt][2]));
                    acc[mt][3] = fmaf(mh.x, d[mt][3], fmaf(mh.y, o[3], acc[mt][3]));
                  }
                }
              }
            }
          } else {
          float d[NT][4], o[4];
#pragma unroll
          for (int j = 0; j < kStageK / 128; ++j) {
            // activations of this lane's k-range (eight bf16) for token rows g and g + 8
            const uint4 v = *reinterpret_cast<const uint4*>(act + tok_lo * 512 + 64 * j);
            uint32_t A0[4], A1[4];
            A0[0] = __byte_perm(v.x, v.z, 0x5410);  // (k0, k4)
            A0[2] = __byte_perm(v.x, v.z, 0x7632);  // (k1, k5)
            A1[0] = __byte_perm(v.y, v.w, 0x5410);  // (k2, k6)
            A1[2] = __byte_perm(v.y, v.w, 0x7632);  // (k3, k7)
            if (TBIG) {
              const uint4 u = *reinterpret_cast<const uint4*>(act + tok_hi * 512 + 64 * j);
              A0[1] = __byte_perm(u.x, u.z, 0x5410);
              A0[3] = __byte_perm(u.x, u.z, 0x7632);
              A1[1] = __byte_perm(u.y, u.w, 0x5410);
              A1[3] = __byte_perm(u.y, u.w, 0x7632);
            } else {
              A0[1] = A0[3] = A1[1] = A1[3] = 0u;
            }
            const bool first = (j % SPAN) == 0;
            if (first) {
              mma16816_z(o, A0, kOne2, kOne2);
            } else {
              mma16816(o, A0, kOne2, kOne2);
            }
            mma16816(o, A1, kOne2, kOne2);
            // 16-byte chunk q of the 128-byte row, stored at chunk q ^ (row % 8) = q ^ g
            const int q = ((kw0 & 255) >> 5) + j;
            const uint8_t* cj = codes + ((q ^ g) << 4);
#pragma unroll
            for (int jt = 0; jt < NT; ++jt) {
              {
                const uint32_t x = *reinterpret_cast<const uint32_t*>(cj + jt * 8 * 128);
                // MMA 0 slots (2c, 2c+1) <- nibbles (0, 4), (2c+8, 2c+9) <- (1, 5); MMA 1: (2, 6), (3, 7)
                const uint32_t b00 = nib_pair(x);
                const uint32_t b01 = nib_pair(shr(x, 4));
                const uint32_t b10 = nib_pair(shr(x, 8));
                const uint32_t b11 = nib_pair(shr(x, 12));
                if (first) {
                  mma16816_z(d[jt], A0, b00, b01);
                } else {
                  mma16816(d[jt], A0, b00, b01);
                }
                mma16816(d[jt], A1, b10, b11);
              }
            }
            if ((j % SPAN) == SPAN - 1) {
              // group span done: acc += s D - s (128 + z) O for weight rows 2c, 2c + 1 of each tile.
              // The warp first converts the group's fp16 (scale, zero) of the pass's rows once
              // (two rows per lane) into fp32 (s, -s (128 + z)) pairs.
              const int gl = ((ks * kStageK + kw0 + 32 * (j - SPAN + 1)) >> p.group_shift) - x0;
              __syncwarp();
#pragma unroll
              for (int rr = 0; rr < (8 * NT + 31) / 32; ++rr) {
                const int row = lane + 32 * rr;
                if (row < 8 * NT) {
                  const float sv = half_bits_to_float(sc[row * p.wg + gl]);
                  const float zv = half_bits_to_float(zr[row * p.wg + gl]);
                  smw[row] = make_float2(sv, -sv * (128.0f + zv));
                }
              }
              __syncwarp();
#pragma unroll
              for (int jt = 0; jt < NT; ++jt) {
                const float4 m4 = *reinterpret_cast<const float4*>(&smw[8 * jt + 2 * c]);
                acc[jt][0] = fmaf(m4.x, d[jt][0], fmaf(m4.y, o[0], acc[jt][0]));
                acc[jt][1] = fmaf(m4.z, d[jt][1], fmaf(m4.w, o[1], acc[jt][1]));
                if (TBIG) {
                  acc[jt][2 % C::kAcc] = fmaf(m4.x, d[jt][2], fmaf(m4.y, o[2], acc[jt][2 % C::kAcc]));
                  acc[jt][3 % C::kAcc] = fmaf(m4.z, d[jt][3], fmaf(m4.w, o[3], acc[jt][3 % C::kAcc]));
                }
              }
            }
          }
          }
        }
        // every value read from this stage has been consumed above
        __syncwarp();
        if (lane == 0) mbar_arrive(&tl.empty[s]);
      }

      // fixed-order reduction of the consumer warps' sums for this pass
      if constexpr (!TBIG) {
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          float* rw = red + (warp * kDecPassRows + 16 * mt + g) * C::kTokPad + 2 * c;
          if (2 * c < T) rw[0] = acc[mt][0];
          if (2 * c + 1 < T) rw[1] = acc[mt][1];
          if (2 * mt + 1 < NT) {
            if (2 * c < T) rw[8 * C::kTokPad] = acc[mt][2];
            if (2 * c + 1 < T) rw[8 * C::kTokPad + 1] = acc[mt][3];
          }
        }
      } else
#pragma unroll
      for (int jt = 0; jt < NT; ++jt) {
        {
          const int r0 = 8 * jt + 2 * c;
          if (g < T) {
            red[(warp * kDecPassRows + r0) * C::kTokPad + g] = acc[jt][0];
            red[(warp * kDecPassRows + r0 + 1) * C::kTokPad + g] = acc[jt][1];
          }
          if (TBIG && g + 8 < T) {
            red[(warp * kDecPassRows + r0) * C::kTokPad + g + 8] = acc[jt][2 % C::kAcc];
            red[(warp * kDecPassRows + r0 + 1) * C::kTokPad + g + 8] = acc[jt][3 % C::kAcc];
          }
        }
      }
      named_bar_sync(1, C::kWarps * 32);
      const int row0 = row_base + pass * kDecPassRows;
      for (int e = threadIdx.x; e < T * h; e += C::kWarps * 32) {
        const int t = e / h;
        const int r = e - t * h;
        float v = 0.0f;
#pragma unroll
        for (int w = 0; w < C::kWarps; ++w) v += red[(w * kDecPassRows + r) * C::kTokPad + t];
        if (KS == 1) {
          if (row0 + r < p.N) {
            const __nv_bfloat16 hv = __float2bfloat16_rn(v);
            out[static_cast<size_t>(t) * p.N + row0 + r] = *reinterpret_cast<const uint16_t*>(&hv);
          }
        } else {
          tl.part[r][t] = v;
        }
      }
      named_bar_sync(1, C::kWarps * 32);  // red is rewritten by the next pass
    }
  }

  if (KS == 2) {
    // one pass per CTA when K is split: rank 0 adds rank 1's partial sums in a fixed order
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    if (rank == 0 && warp < C::kWarps && passes_here > 0) {
      const int h = rows_here;
      const float* peer = cluster.map_shared_rank(&tl.part[0][0], 1);
      for (int e = threadIdx.x; e < p.T * h; e += C::kWarps * 32) {
        const int t = e / h;
        const int r = e - t * h;
        const float v = tl.part[r][t] + peer[r * 16 + t];
        const __nv_bfloat16 hv = __float2bfloat16_rn(v);
        out[static_cast<size_t>(t) * p.N + row_base + r] = *reinterpret_cast<const uint16_t*>(&hv);
      }
    }
    cluster.sync();  // rank 1 keeps its shared memory until rank 0 has read it
  }
}

// group-size class: 0 for g >= 128, 1 for g = 64, 2 for g = 32
template <int BITS, int SPAN>
constexpr int dec_gclass() {
  return BITS == 4                 ? (SPAN == 4 ? 0 : (SPAN == 2 ? 1 : 2))
         : (BITS == 2 || BITS == 3) ? (SPAN == 2 ? 0 : 1)
                                    : (SPAN == 8 ? 0 : (SPAN == 4 ? 1 : 2));
}

const char* dec_name(int bits, bool tbig, int gclass, int ks, int nt) {
  // "w4a16_dec_kernel<T<=8,g>=128,nt7>", "...,ksplit2,nt7>", "w2a16_dec_kernel<T<=8,g=64,nt8>";
  // built once, kept for the process
  static char names[4][2][3][2][9][64];
  static const bool filled = [] {
    const char* gs[3] = {"g>=128", "g=64", "g=32"};
    const int widths[4] = {4, 2, 8, 3};
    for (int w = 0; w < 4; ++w)
      for (int a = 0; a < 2; ++a)
        for (int b = 0; b < 3; ++b)
          for (int c = 0; c < 2; ++c)
            for (int d = 1; d <= 8; ++d)
              snprintf(names[w][a][b][c][d], sizeof(names[w][a][b][c][d]), "w%da16_dec_kernel<T<=%d,%s%s,nt%d>",
                       widths[w], a ? 16 : 8, gs[b], c ? ",ksplit2" : "", d);
    return true;
  }();
  (void)filled;
  return names[bits == 2 ? 1 : (bits == 8 ? 2 : (bits == 3 ? 3 : 0))][tbig ? 1 : 0][gclass][ks - 1][nt];
}

template <bool TBIG, int SPAN, int KS, int NT, int BITS, int STAGEK>
cudaError_t launch_dec(const CUtensorMap (&maps)[7], const DecParams& p, int grid, int smem, uint16_t* out,
                       cudaStream_t stream) {
  auto kern = w4a16_dec_kernel<TBIG, SPAN, KS, NT, BITS, STAGEK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(DecCfg<TBIG>::kThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = KS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  LaunchScope scope(stream, dec_name(BITS, TBIG, dec_gclass<BITS, SPAN>(), KS, NT));
  e = cudaLaunchKernelEx(&cfg, kern, maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], maps[6], p, out);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// g >= 128 (the common case) has a kernel per tile count; g = 32, 64 run eight tiles
template <bool TBIG, int SPAN, int KS, int BITS, int STAGEK>
cudaError_t launch_dec_nt(int nt, const CUtensorMap (&maps)[7], const DecParams& p, int grid, int smem,
                          uint16_t* out, cudaStream_t stream) {
  if constexpr (dec_gclass<BITS, SPAN>() == 0) {
    switch (nt) {
      case 1: return launch_dec<TBIG, SPAN, KS, 1, BITS, STAGEK>(maps, p, grid, smem, out, stream);
      case 2: return launch_dec<TBIG, SPAN, KS, 2, BITS, STAGEK>(maps, p, grid, smem, out, stream);
      case 3: return launch_dec<TBIG, SPAN, KS, 3, BITS, STAGEK>(maps, p, grid, smem, out, stream);
      case 4: return launch_dec<TBIG, SPAN, KS, 4, BITS, STAGEK>(maps, p, grid, smem, out, stream);
      case 5: return launch_dec<TBIG, SPAN, KS, 5, BITS, STAGEK>(maps, p, grid, smem, out, stream);
      case 6: return launch_dec<TBIG, SPAN, KS, 6, BITS, STAGEK>(maps, p, grid, smem, out, stream);
      case 7: return launch_dec<TBIG, SPAN, KS, 7, BITS, STAGEK>(maps, p, grid, smem, out, stream);
      default: return launch_dec<TBIG, SPAN, KS, 8, BITS, STAGEK>(maps, p, grid, smem, out, stream);
    }
  } else {
    (void)nt;
    return launch_dec<TBIG, SPAN, KS, 8, BITS, STAGEK>(maps, p, grid, smem, out, stream);
  }
}

// 4-bit codes
template <bool TBIG, int STAGEK>
cudaError_t launch_dec_span(int span, int ks, int nt, const CUtensorMap (&maps)[7], const DecParams& p, int grid,
                            int smem, uint16_t* out, cudaStream_t stream) {
  if (ks == 2) {
    if (span == 4) return launch_dec_nt<TBIG, 4, 2, 4, STAGEK>(nt, maps, p, grid, smem, out, stream);
    if (span == 2) return launch_dec_nt<TBIG, 2, 2, 4, STAGEK>(nt, maps, p, grid, smem, out, stream);
    return launch_dec_nt<TBIG, 1, 2, 4, STAGEK>(nt, maps, p, grid, smem, out, stream);
  }
  if (span == 4) return launch_dec_nt<TBIG, 4, 1, 4, STAGEK>(nt, maps, p, grid, smem, out, stream);
  if (span == 2) return launch_dec_nt<TBIG, 2, 1, 4, STAGEK>(nt, maps, p, grid, smem, out, stream);
  return launch_dec_nt<TBIG, 1, 1, 4, STAGEK>(nt, maps, p, grid, smem, out, stream);
}

// 2-bit codes, T <= 8, 1024-k stages: span 2 (g >= 128) or 1 (g = 64); 2048-k stages: g >= 128
template <int STAGEK>
cudaError_t launch_dec2_span(int span, int ks, int nt, const CUtensorMap (&maps)[7], const DecParams& p, int grid,
                             int smem, uint16_t* out, cudaStream_t stream) {
  if constexpr (STAGEK == 2048) {
    (void)span;
    return ks == 2 ? launch_dec_nt<false, 2, 2, 2, STAGEK>(nt, maps, p, grid, smem, out, stream)
                   : launch_dec_nt<false, 2, 1, 2, STAGEK>(nt, maps, p, grid, smem, out, stream);
  } else {
    if (ks == 2) {
      if (span == 2) return launch_dec_nt<false, 2, 2, 2, STAGEK>(nt, maps, p, grid, smem, out, stream);
      return launch_dec_nt<false, 1, 2, 2, STAGEK>(nt, maps, p, grid, smem, out, stream);
    }
    if (span == 2) return launch_dec_nt<false, 2, 1, 2, STAGEK>(nt, maps, p, grid, smem, out, stream);
    return launch_dec_nt<false, 1, 1, 2, STAGEK>(nt, maps, p, grid, smem, out, stream);
  }
}

// 8-bit codes, T <= 8, 512-k stages: span 8 (g >= 128), 4 (g = 64) or 2 (g = 32) 16-k chunks
cudaError_t launch_dec8_span(int span, int ks, int nt, const CUtensorMap (&maps)[7], const DecParams& p, int grid,
                             int smem, uint16_t* out, cudaStream_t stream) {
  if (ks == 2) {
    if (span == 8) return launch_dec_nt<false, 8, 2, 8, 512>(nt, maps, p, grid, smem, out, stream);
    if (span == 4) return launch_dec_nt<false, 4, 2, 8, 512>(nt, maps, p, grid, smem, out, stream);
    return launch_dec_nt<false, 2, 2, 8, 512>(nt, maps, p, grid, smem, out, stream);
  }
  if (span == 8) return launch_dec_nt<false, 8, 1, 8, 512>(nt, maps, p, grid, smem, out, stream);
  if (span == 4) return launch_dec_nt<false, 4, 1, 8, 512>(nt, maps, p, grid, smem, out, stream);
  return launch_dec_nt<false, 2, 1, 8, 512>(nt, maps, p, grid, smem, out, stream);
}

// 3-bit codes, T <= 8, 1024-k stages: span 2 (g >= 128) or 1 (g = 64)
cudaError_t launch_dec3_span(int span, int ks, int nt, const CUtensorMap (&maps)[7], const DecParams& p, int grid,
                             int smem, uint16_t* out, cudaStream_t stream) {
  if (ks == 2) {
    if (span == 2) return launch_dec_nt<false, 2, 2, 3, 1024>(nt, maps, p, grid, smem, out, stream);
    return launch_dec_nt<false, 1, 2, 3, 1024>(nt, maps, p, grid, smem, out, stream);
  }
  if (span == 2) return launch_dec_nt<false, 2, 1, 3, 1024>(nt, maps, p, grid, smem, out, stream);
  return launch_dec_nt<false, 1, 1, 3, 1024>(nt, maps, p, grid, smem, out, stream);
}

int round_up(int x, int m) { return (x + m - 1) / m * m; }

// Returns cudaErrorNotSupported (nothing launched) when the shape does not fit
// this kernel's tensor maps: the scale/zero row stride must be a multiple of 16
// bytes (K/g a multiple of 8) and the scale/zero arrays 16-byte aligned; 2-bit
// codes also need T <= 8, g >= 64 (a 64-k slice inside one group) and K >= 512
// (a row of codes at least one box wide).
cudaError_t launch_dec_bits(const uint16_t* A, int T, const uint32_t* packed, const uint16_t* scale16,
                            const uint16_t* zero16, int N, int K, int group_size, int bits, uint16_t* out,
                            cudaStream_t stream) {
  if (T < 1 || T > 16 || N < 1 || K < 128 || K % 128 != 0 || group_size < 32) return cudaErrorNotSupported;
  if (bits == 2 && (T > 8 || group_size < 64 || K < kDecStageK)) return cudaErrorNotSupported;
  if (bits == 3 && (T > 8 || group_size < 64 || K < kDecStageK)) return cudaErrorNotSupported;
  if (bits == 8 && T > 8) return cudaErrorNotSupported;
  if (bits != 2 && bits != 3 && bits != 4 && bits != 8) return cudaErrorNotSupported;
  const int G = K / group_size;
  if (G % 8 != 0 || (reinterpret_cast<uintptr_t>(scale16) & 15u) || (reinterpret_cast<uintptr_t>(zero16) & 15u))
    return cudaErrorNotSupported;
  int dev = 0, num_sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;

  DecParams p = {};
  p.N = N;
  p.K = K;
  p.T = T;
  int gs = 0;
  while ((1 << gs) < group_size) ++gs;
  p.group_shift = gs;

  const bool tbig = T > 8;
  const int red_bytes = tbig ? DecCfg<true>::kRedBytes : DecCfg<false>::kRedBytes;
  const int fixed = red_bytes + static_cast<int>(sizeof(DecTail)) + 1024;
  // ring depth: a multiple of the consumer groups (each slot always taken by the same group)
  const int groups = tbig ? DecCfg<true>::kGroups : DecCfg<false>::kGroups;
  // stage layout for stage_k k per stage: codes, activations, scale table, zero table; false
  // when fewer than two stages per consumer group fit
  auto layout = [&](int stage_k) {
    p.n_stages = (K + stage_k - 1) / stage_k;
    p.wg = std::max(8, stage_k / group_size);  // a window of the groups a stage touches
    p.act_off = (stage_k * bits / 1024) * kDecCodeBox;
    p.tab_off = p.act_off + round_up(2 * stage_k * T, 128);
    p.stage_bytes = round_up(p.tab_off + 2 * 2 * p.wg * kDecPassRows, 1024);
    p.S = std::min(bits == 4 ? kDecMaxStages : kDecMaxStages2, (kDecSmemLimit - fixed) / p.stage_bytes) / groups *
          groups;
    return p.S >= 2 * groups;
  };
  // 1024-k stages (half the per-stage costs) unless the ring would be too shallow; 9..16 tokens
  // keep 512-k stages.  2-bit codes: 2048-k stages for one token at g >= 128 where four fit and K
  // holds two of them (so a small N can still split K over a CTA pair), else 1024 (measured on the
  // 8192 x 28672 layer: T = 1 g 128 30.8 against 32.8 us; T = 2 the same; g = 64 slower, 38.9
  // against 34.8 us, from its 32-group table windows and spills)
  int stage_k = bits == 8 ? 512 : 1024;
  if (bits == 4 && (tbig || !layout(1024))) stage_k = 512;
  if (bits == 2 && T == 1 && group_size >= 128 && K >= 4096 && layout(2048)) stage_k = 2048;
  if (!layout(stage_k)) return cudaErrorNotSupported;

  // rows per CTA (multiple of 8) with one CTA per SM; a cluster pair splits K
  // instead when that halves the rows a CTA streams (small N)
  const int units = (N + 7) / 8;
  const int rows1 = 8 * ((units + num_sms - 1) / num_sms);
  const int rows2 = 8 * ((2 * units + num_sms - 1) / num_sms);
  int ks = 1, rows = rows1;
  if (p.n_stages >= 2 && rows2 <= kDecPassRows && 2 * rows1 > rows2 + 4) {
    ks = 2;
    rows = rows2;
  }
  p.rows_per_cta = rows;
  p.passes = (rows + kDecPassRows - 1) / kDecPassRows;
  p.last_rows = rows - (p.passes - 1) * kDecPassRows;
  const int grid = ks * ((N + rows - 1) / rows);
  const int smem = dec_tail_offset(p.S, p.stage_bytes, red_bytes) + static_cast<int>(sizeof(DecTail)) + 1024;

  CUtensorMap maps[7];
  const int heights[2] = {std::min(kDecPassRows, rows), p.last_rows};
  for (int m = 0; m < 2; ++m) {
    e = make_tmap_2d(&maps[m], CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, packed, static_cast<uint64_t>(N),
                     static_cast<uint64_t>(K) * bits / 32, 32, static_cast<uint32_t>(heights[m]),
                     CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    e = make_tmap_2d(&maps[2 + m], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, scale16, static_cast<uint64_t>(N),
                     static_cast<uint64_t>(G), static_cast<uint32_t>(p.wg), static_cast<uint32_t>(heights[m]),
                     CU_TENSOR_MAP_SWIZZLE_NONE);
    if (e != cudaSuccess) return e;
    e = make_tmap_2d(&maps[4 + m], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, zero16, static_cast<uint64_t>(N),
                     static_cast<uint64_t>(G), static_cast<uint32_t>(p.wg), static_cast<uint32_t>(heights[m]),
                     CU_TENSOR_MAP_SWIZZLE_NONE);
    if (e != cudaSuccess) return e;
  }
  e = make_tmap_2d(&maps[6], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, A, static_cast<uint64_t>(T), static_cast<uint64_t>(K),
                   256, static_cast<uint32_t>(T), CU_TENSOR_MAP_SWIZZLE_NONE);
  if (e != cudaSuccess) return e;

  const int nt = p.passes == 1 ? rows / 8 : 8;  // tiles of a full pass
  if (bits == 8) return launch_dec8_span(std::min(8, group_size / 16), ks, nt, maps, p, grid, smem, out, stream);
  if (bits == 3) return launch_dec3_span(group_size >= 128 ? 2 : 1, ks, nt, maps, p, grid, smem, out, stream);
  if (bits == 2) {
    const int span2 = group_size >= 128 ? 2 : 1;
    return stage_k == 2048 ? launch_dec2_span<2048>(span2, ks, nt, maps, p, grid, smem, out, stream)
                           : launch_dec2_span<1024>(span2, ks, nt, maps, p, grid, smem, out, stream);
  }
  const int span = group_size >= 128 ? 4 : group_size / 32;
  if (tbig) return launch_dec_span<true, 512>(span, ks, nt, maps, p, grid, smem, out, stream);
  return stage_k == 1024 ? launch_dec_span<false, 1024>(span, ks, nt, maps, p, grid, smem, out, stream)
                         : launch_dec_span<false, 512>(span, ks, nt, maps, p, grid, smem, out, stream);
}

}  // namespace

cudaError_t launch_w4a16_dec(const uint16_t* A, int T, const uint32_t* packed, const uint16_t* scale16,
                             const uint16_t* zero16, int N, int K, int group_size, uint16_t* out,
                             cudaStream_t stream) {
  return launch_dec_bits(A, T, packed, scale16, zero16, N, K, group_size, 4, out, stream);
}

cudaError_t launch_w2a16_dec(const uint16_t* A, int T, const uint32_t* packed, const uint16_t* scale16,
                             const uint16_t* zero16, int N, int K, int group_size, uint16_t* out,
                             cudaStream_t stream) {
  return launch_dec_bits(A, T, packed, scale16, zero16, N, K, group_size, 2, out, stream);
}

cudaError_t launch_w8a16_dec(const uint16_t* A, int T, const uint32_t* packed, const uint16_t* scale16,
                             const uint16_t* zero16, int N, int K, int group_size, uint16_t* out,
                             cudaStream_t stream) {
  return launch_dec_bits(A, T, packed, scale16, zero16, N, K, group_size, 8, out, stream);
}

cudaError_t launch_w3a16_dec(const uint16_t* A, int T, const uint32_t* packed, const uint16_t* scale16,
                             const uint16_t* zero16, int N, int K, int group_size, uint16_t* out,
                             cudaStream_t stream) {
  return launch_dec_bits(A, T, packed, scale16, zero16, N, K, group_size, 3, out, stream);
}

}  // namespace ar
