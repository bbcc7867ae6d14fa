// W4A16 matmul on the fifth-generation tensor cores (tcgen05), for batches
// past decode size: out[t][n] = sum_k A[t][k] (q[n][k] - z[n][k/g]) s[n][k/g].
//
// [AR] §4 (comparison table, "Real INT4 Kernel" column): the weights stay
// 4-bit in memory and are dequantized inside the kernel; the page notes that
// decode-sized batches are memory bound and prefill-sized ones compute bound
// ([AR] = "Low-Bit Quantization in Practice with vLLM: Core Mechanisms and
// Architectural Optimizations of AutoRound").
//
// At T = 256 tokens the product is 2 T N K FLOPs on 0.5 N K bytes of weights
// (1024 FLOP/byte), well past the ridge, so the tensor cores set the pace:
//
//  * One CTA owns 128 weight rows (the MMA's M, one TMEM lane per row) and a
//    tile of TN tokens (the MMA's N).  One TMA warp streams the packed codes
//    (128 rows x 256 k = 128 bytes a row, 128-byte swizzle) into a ring of
//    four slots that runs up to 16 stages ahead; another streams the bf16
//    activations (TN x 64 k per stage, 128-byte swizzle) into the stage
//    ring, as deep as shared memory allows.
//  * Four dequantization warps turn each stage's codes into the MMA's A
//    operand: (word >> 4i) & 0x000F000F | 0x43004300 is the exact bf16 pair
//    (128 + q_i, 128 + q_{i+4}); one bf16x2 subtraction of (128 + z) leaves
//    (q - z), exact in bf16; byte permutes restore k order, and tcgen05.st
//    writes the 128 x 64 tile straight into tensor memory (one lane per row),
//    where the MMA reads A.  Shared memory then carries only the codes and
//    the activations: an M = 128, N = 128 MMA reading both operands from
//    shared memory would take all of its bandwidth by itself.
//  * One thread issues tcgen05.mma (kind::f16, bf16 x bf16 -> fp32, M = 128,
//    N = TN, K = 16) into a TMEM accumulator that holds ONE quantization
//    group: sum_{k in group} a (q - z) is exact up to fp32 summation, and the
//    group's scale is applied once, in fp32, by the epilogue warps, which
//    read the accumulator (tcgen05.ld) and add s * D to register sums (8
//    warps, two per TMEM lane quarter, splitting columns or groups).  Four
//    accumulators rotate so that the MMAs of the next groups overlap the
//    epilogue of the last.
//  * When one token tile leaves SMs idle, the two CTAs of a cluster split K
//    and rank 0 adds rank 1's partial sums through distributed shared memory
//    in a fixed order: no workspace, deterministic results.
//
// Packed layout (as ar_pack_int4 writes it): uint32 [N][K/8], element k at
// bits 4*(k mod 8) of word k/8; scale/zero fp16 [N][K/g].  Other widths (2, 3,
// 8 bits, as ar_pack_codes writes them): each row a little-endian bit stream,
// element k at stream bits BITS k .. BITS k + BITS - 1.
#include <cooperative_groups.h>

#include <cuda_fp8.h>

#include "ar_internal.h"

namespace cg = cooperative_groups;

namespace ar {
namespace {

constexpr int kTcRows = 128;  // weight rows per CTA (MMA M, TMEM lanes)
constexpr int kTcK = 128;     // k per stage: 8 MMAs per barrier hand-off
constexpr int kSub = kTcK / 64;  // 64-k sub-tiles (one 128-byte swizzle row of bf16 each)
constexpr int kCodeBytes = kTcRows * 128;  // 16 KiB per TMA box of codes: a 128-byte row of packed words per weight row
// Code slots per width.  A 128-k stage takes 16 BITS bytes of a row.  At 2, 4 and 8
// bits a slot is one box (4, 2 or 1 stages); a 3-bit stage (48 bytes) does not divide
// a box, so a 3-bit slot is three boxes side by side, 384 bytes a row: eight stages.
template <int BITS>
struct CodeCfg {
  static constexpr int kBoxes = BITS == 3 ? 3 : 1;
  static constexpr int kChunksPerSlot = BITS == 3 ? 8 : 8 / BITS;  // stages of 128 k per slot
  static constexpr int kSlots = BITS == 3 ? 2 : 4;
  static constexpr int kSlotBytes = kBoxes * kCodeBytes;
  static_assert(kChunksPerSlot * 16 * BITS == kBoxes * 128, "a slot holds whole stages");
};
constexpr int kCodeSlotsMax = 4;
constexpr int kNBufMax = 4;   // TMEM accumulators, one group each
constexpr int kAStages = 4;   // A operand stages in TMEM (and activation stages in shared memory)
constexpr int kACols = kTcK / 2;  // TMEM columns per A stage (two bf16 per column)
constexpr int kACol0 = 256;   // TMEM column of A stage 0; stage s at kACol0 + kACols s
constexpr int kTmemCols = 512;
// Warp roles: 0 activation TMA, 1 TMEM owner + MMA issuer, 2 code TMA, then the
// dequantization warps, then the epilogue warps.
constexpr int kEpWarps = 8;   // a multiple of 4: kEpWarps / 4 per TMEM lane quarter
constexpr int kEpQ = kEpWarps / 4;
constexpr int kDqWarp0 = 3;

// True when sets of warps that take a ring's stages in turn (set i takes stages
// i, i + sets, ...), with `per_slot` consecutive stages sharing one slot of a
// `slots`-slot ring, each wait on a slot's phases in order.
__host__ __device__ constexpr bool slot_phases_in_order(int per_slot, int sets, int slots) {
  return per_slot % sets == 0 || (sets % per_slot == 0 && slots % (sets / per_slot) == 0);
}

template <int TN, int BITS, bool FP4 = false>
struct TcCfg {
  // One dequantization warp per TMEM lane quarter is latency bound (its nibble
  // and permute chains), so narrow tiles, whose epilogue needs few registers,
  // run two per quarter on alternating stages.  At TN = 128 a second set costs
  // epilogue spills (the 608 threads leave ~104 registers), which pays only where
  // the dequantization is long enough: measured on 8192 x 28672 at 256 tokens,
  // NVFP4 219 -> 176 us and 2 bits 221 -> 212 us, but 4 bits 227 -> 239 us,
  // 3 bits 223 -> 270 us, 8 bits unchanged.
  static constexpr int kDqWarps = (TN < 128 || FP4 || BITS == 2) ? 8 : 4;
  static constexpr int kEpWarp0 = kDqWarp0 + kDqWarps;
  static constexpr int kThreads = (kEpWarp0 + kEpWarps) * 32;
  static constexpr int kActBytes = TN * 128 * kSub;    // TN tokens x kTcK k bf16, kSub sub-tiles
  static constexpr int kStageBytes = kActBytes;
  static constexpr int kStages = kAStages;
  static constexpr int kRingBytes = kStages * kStageBytes + CodeCfg<BITS>::kSlots * CodeCfg<BITS>::kSlotBytes;
  static constexpr int kNBuf = TN >= 128 ? 2 : kNBufMax;  // accumulators fit below kACol0
  static_assert(kNBuf * TN <= kACol0, "accumulators and A stages share the 512 TMEM columns");
  static_assert(kACol0 + kACols * kAStages <= kTmemCols, "A stages fit in TMEM");
  // The epilogue warps of a lane quarter split the token columns
  // (kColSplit ways) and the groups (kGrpSplit ways, round robin).
  static constexpr int kColSplit = TN >= 128 ? kEpQ : TN >= 64 ? (kEpQ < 2 ? kEpQ : 2) : 1;
  static constexpr int kGrpSplit = kEpQ / kColSplit;
  static constexpr int kCols = TN / kColSplit;           // accumulator columns per epilogue thread (16 or 32)
  static constexpr int kRedStride = TN + 1;              // odd row stride: conflict-free transposes
  static constexpr int kRedPlanes = kGrpSplit;           // partial sums per row and column
  static constexpr int kRedBytes = kRedPlanes * kTcRows * kRedStride * 4;
  static constexpr int kFinBytes = kTcRows * kRedStride * 4;
  static_assert(kActBytes % 1024 == 0, "stage parts must keep 1024-byte alignment");
  static_assert(kRedBytes + kFinBytes <= kRingBytes, "reduction buffers reuse the rings");
  // Every waiter on a ring barrier must see the barrier's phases in order: a
  // parity wait cannot tell a phase from the one two before it.  So when
  // several warp sets take a ring's entries in turn, each entry is always
  // taken by the same set (the set count divides the entry count).
  static_assert(kStages % (kDqWarps / 4) == 0, "A stages: one dequantization set per stage");
  static_assert(kNBuf % kGrpSplit == 0, "accumulators: one epilogue set per accumulator");
};

struct TcCtl {
  uint64_t full[kAStages];      // TMA: activations of the stage landed
  uint64_t dq_full[kAStages];   // A operand written and activations landed (one arrival per row quarter)
  uint64_t empty[kAStages];     // MMAs of the stage done (tcgen05.commit)
  uint64_t code_full[kCodeSlotsMax];   // TMA: codes of the slot landed
  uint64_t code_empty[kCodeSlotsMax];  // codes of the slot read (one arrival per row quarter and stage)
  uint64_t tmem_full[kNBufMax];
  uint64_t tmem_empty[kNBufMax];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
};

struct TcParams {
  const uint16_t* s16;  // fp16 bits [N][G]
  const uint16_t* z16;
  const uint8_t* sc8;   // NVFP4: E4M3 block-scale codes [N][K/16]
  const float* gscale;  // NVFP4: device per-tensor scale S
  uint16_t* out;        // bf16 bits [T][N]
  int N, K, T, G;
  int group_shift;
  int t_tiles;
  int split_units;      // rank 0 of a split takes the first split_units (k units of max(g, 64))
  int unit_k;
  int vec_meta;         // every row's metadata starts 16-byte aligned for this CTA's range
};

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// A shared-memory descriptor from its two 32-bit halves (the start address sits
// in the low 14 bits; offsets inside the 227 KB window never carry out of them).
__device__ __forceinline__ uint64_t mk_desc(uint32_t lo, uint32_t hi) {
  return (static_cast<uint64_t>(hi) << 32) | lo;
}

// 32 lanes x 32 columns of 32-bit values into TMEM (this warp's lane quarter).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// D[tmem] (+)= A[tmem] x B[smem]^T, bf16 inputs, fp32 accumulate; A is M lanes x
// (K / 2) columns, two k-consecutive bf16 values per 32-bit column.
__device__ __forceinline__ void umma_bf16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// 8 codes of one word -> 8 bf16 values (q - z) in k order; zz = (128 + z) in both halves.
__device__ __forceinline__ uint4 dequant8(uint32_t x, uint32_t zz) {
  constexpr uint32_t kMask = 0x000F000Fu, kBias = 0x43004300u;
  const uint32_t e0 = bf16x2_sub((x & kMask) | kBias, zz);          // (k0, k4)
  const uint32_t e1 = bf16x2_sub(((x >> 4) & kMask) | kBias, zz);   // (k1, k5)
  const uint32_t e2 = bf16x2_sub(((x >> 8) & kMask) | kBias, zz);   // (k2, k6)
  const uint32_t e3 = bf16x2_sub(((x >> 12) & kMask) | kBias, zz);  // (k3, k7)
  uint4 o;
  o.x = __byte_perm(e0, e1, 0x5410);  // (k0, k1)
  o.y = __byte_perm(e2, e3, 0x5410);  // (k2, k3)
  o.z = __byte_perm(e0, e1, 0x7632);  // (k4, k5)
  o.w = __byte_perm(e2, e3, 0x7632);  // (k6, k7)
  return o;
}

// bf16 pair (128 + z, 128 + z) from the fp16 bits of an integer zero-point 0..15
// (128 + z is exact in bf16: its ulp is 1 in [128, 256)).
// 16 two-bit codes of one word -> 16 bf16 values (q - z) in k order (8 words);
// zz = (128 + z) in both halves.
__device__ __forceinline__ void dequant16(uint32_t x, uint32_t zz, uint32_t* o) {
  uint32_t e[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) e[i] = bf16x2_sub(((x >> (2 * i)) & 0x00030003u) | 0x43004300u, zz);  // (k_i, k_{i+8})
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    o[j] = __byte_perm(e[2 * j], e[2 * j + 1], 0x5410);      // (k_{2j}, k_{2j+1})
    o[4 + j] = __byte_perm(e[2 * j], e[2 * j + 1], 0x7632);  // (k_{8+2j}, k_{9+2j})
  }
}

// Component c (0..3, known at compile time) of a 16-byte vector.
__device__ __forceinline__ uint32_t vec_word(const uint4& v, int c) {
  return c == 0 ? v.x : c == 1 ? v.y : c == 2 ? v.z : v.w;
}

// 32 three-bit codes of three consecutive words (the row's bit stream: code m at
// bits 3m .. 3m + 2 of the 96 bits, words little-endian) -> 32 bf16 values (q - z)
// in k order (16 words); zz = (128 + z) in both halves.  For each four codes y (12
// bits), y (1 + 2^13) = y | y << 13 (the two do not overlap, so nothing carries)
// holds q0 at bit 0, q1 at bit 16, q2 at bit 6 and q3 at bit 22: one mask gives
// the pair (q0, q1) and, after a 6-bit shift, (q2, q3).
__device__ __forceinline__ void dequant3x32(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t zz, uint32_t* o) {
  constexpr uint32_t kMask = 0x00070007u, kBias = 0x43004300u;
#pragma unroll
  for (int j = 0; j < 8; ++j) {  // codes 4j .. 4j + 3: stream bits 12j .. 12j + 11
    const int b = 12 * j;
    uint32_t y;
    if (b + 12 <= 32) y = w0 >> b;
    else if (b < 32) y = __funnelshift_r(w0, w1, b);
    else if (b + 12 <= 64) y = w1 >> (b - 32);
    else if (b < 64) y = __funnelshift_r(w1, w2, b - 32);
    else y = w2 >> (b - 64);
    const uint32_t m = (y & 0xFFFu) * 0x2001u;
    o[2 * j] = bf16x2_sub((m & kMask) | kBias, zz);             // (k 4j, 4j + 1)
    o[2 * j + 1] = bf16x2_sub(((m >> 6) & kMask) | kBias, zz);  // (k 4j + 2, 4j + 3)
  }
}

// 4 eight-bit codes of one word -> 4 bf16 values (q - z) in k order (2 words):
// the byte under an fp32 exponent of 2^23 is 2^23 + q exactly, one subtraction
// of zf = 2^23 + z leaves q - z exactly (|q - z| <= 255 is exact in bf16).
__device__ __forceinline__ void dequant4b(uint32_t x, float zf, uint32_t* o) {
  float f[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) f[i] = __fsub_rn(__uint_as_float(__byte_perm(x, 0x4B000000u, 0x7540u | i)), zf);
  o[0] = pack_bf16x2(f[0], f[1]);
  o[1] = pack_bf16x2(f[2], f[3]);
}

// 8 E2M1 codes of one word (element k in bits 4k..4k+3; code = sign << 3 |
// magnitude index) -> 8 bf16 values in k order, each times the bf16 pair sc2 (the
// block scale in both halves).  The magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 are
// bf16 0x0000, 0x3F00, 0x3F80, 0x3FC0, 0x4000, 0x4040, 0x4080, 0x40C0: byte
// tables of their low and high bytes, indexed by the 3-bit magnitude index
// through byte permutes, give four values per permute; the sign bit of each
// code moves to bit 15 or 31 of its pair.  An E2M1 value times an E4M3 scale
// has at most 6 significant bits and stays in bf16's normal range, so every
// product is exact.
__device__ __forceinline__ uint4 dequant_e2m1x8(uint32_t x, uint32_t sc2) {
  constexpr uint32_t kL0 = 0xC0800000u, kL1 = 0xC0804000u;  // low bytes for magnitudes 0..3, 4..7
  constexpr uint32_t kH0 = 0x3F3F3F00u, kH1 = 0x40404040u;  // high bytes
  const uint32_t y = x & 0x77777777u;                       // magnitude indices (selector bit 3 cleared)
  const uint32_t y2 = y >> 16;
  const uint32_t l03 = __byte_perm(kL0, kL1, y), h03 = __byte_perm(kH0, kH1, y);
  const uint32_t l47 = __byte_perm(kL0, kL1, y2), h47 = __byte_perm(kH0, kH1, y2);
  // sign of code 2j: bit 7 of byte j of sx4; of code 2j + 1: bit 7 of byte j of sx
  const uint32_t sx = x & 0x88888888u;
  const uint32_t sx4 = (x << 4) & 0x88888888u;
  uint32_t m[4];
  m[0] = __byte_perm(l03, h03, 0x5140) | (__byte_perm(sx4, sx, 0x4000) & 0x80008000u);  // (k0, k1)
  m[1] = __byte_perm(l03, h03, 0x7362) | (__byte_perm(sx4, sx, 0x5111) & 0x80008000u);  // (k2, k3)
  m[2] = __byte_perm(l47, h47, 0x5140) | (__byte_perm(sx4, sx, 0x6222) & 0x80008000u);  // (k4, k5)
  m[3] = __byte_perm(l47, h47, 0x7362) | (__byte_perm(sx4, sx, 0x7333) & 0x80008000u);  // (k6, k7)
  uint4 o;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(o.x) : "r"(m[0]), "r"(sc2));
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(o.y) : "r"(m[1]), "r"(sc2));
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(o.z) : "r"(m[2]), "r"(sc2));
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(o.w) : "r"(m[3]), "r"(sc2));
  return o;
}

// The 8 E4M3 block-scale codes of one row's 128-k stage -> 8 bf16 pairs (each
// scale in both halves); E4M3 values are exact in bf16.
__device__ __forceinline__ void e4m3x8_to_bf16_pairs(uint2 c, uint32_t (&sc2)[8]) {
  const uint32_t w[2] = {c.x, c.y};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w[h] >> (16 * i)), __NV_E4M3);
      const float f0 = __half2float(__half(__half_raw{hr.x}));
      const float f1 = __half2float(__half(__half_raw{hr.y}));
      sc2[4 * h + 2 * i] = pack_bf16x2(f0, f0);
      sc2[4 * h + 2 * i + 1] = pack_bf16x2(f1, f1);
    }
  }
}

__device__ __forceinline__ uint32_t zero_pair(uint16_t z16) {
  const uint32_t z = static_cast<uint32_t>(__half2float(__ushort_as_half(z16)));
  return (0x4300u + z) * 0x00010001u;
}

// One row's fp16 metadata (scale or zero) in increasing group order.  Loads
// eight groups (16 bytes) at a time one batch ahead when the row's range is
// 16-byte aligned, else one group at a time one group ahead.
struct MetaRow {
  const uint16_t* row;
  int lim;    // groups in the row
  int held;   // batch (vector) or group (scalar) index in `cur`
  bool vec, live;
  uint4 cur, nxt;

  __device__ __forceinline__ uint4 load(int i) const {
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (!live) return v;
    if (vec) {
      if (8 * i < lim) v = __ldg(reinterpret_cast<const uint4*>(row) + i);
    } else if (i < lim) {
      v.x = __ldg(row + i);
    }
    return v;
  }
  __device__ __forceinline__ void start(const uint16_t* r, int g0, int groups, bool vector, bool valid) {
    row = r;
    lim = groups;
    vec = vector;
    live = valid;
    held = vec ? (g0 >> 3) : g0;
    cur = load(held);
    nxt = load(held + 1);
  }
  __device__ __forceinline__ uint16_t get(int gi) {
    const int want = vec ? (gi >> 3) : gi;
    while (held < want) {
      cur = nxt;
      ++held;
      nxt = load(held + 1);
    }
    if (!vec) return static_cast<uint16_t>(cur.x);
    const int h = gi & 7;
    const uint32_t w = (h >> 1) == 0 ? cur.x : (h >> 1) == 1 ? cur.y : (h >> 1) == 2 ? cur.z : cur.w;
    return static_cast<uint16_t>((h & 1) ? (w >> 16) : (w & 0xFFFFu));
  }
};

// 32 lanes x 16 columns of fp32 from TMEM (this warp's lane quarter), waited.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Grid: one CTA per (128-row tile, token tile, K half when split); the CTAs of
// a weight tile are adjacent so that its codes come from HBM once.
// FP4: NVFP4 weights (E2M1 codes in the 4-bit layout, E4M3 block scales folded
// into the dequantized operand, the per-tensor scale applied per group in the
// epilogue); BITS is then 4.
template <int TN, int KSPLIT, int BITS, bool FP4>
__global__ void __launch_bounds__(TcCfg<TN, BITS, FP4>::kThreads, 1)
    w4a16_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW,
                    const TcParams p) {
  using Cfg = TcCfg<TN, BITS, FP4>;
  using Code = CodeCfg<BITS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* codes = ring + Cfg::kStages * Cfg::kStageBytes;
  TcCtl* ctl = reinterpret_cast<TcCtl*>(ring + Cfg::kRingBytes);
  volatile int* abort_flag = &ctl->abort_flag;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int rank = KSPLIT == 2 ? static_cast<int>(cluster_ctarank()) : 0;
  const int tile = static_cast<int>(blockIdx.x) / KSPLIT;
  const int n_tile = tile / p.t_tiles;
  const int t_tile = tile - n_tile * p.t_tiles;
  const int n0 = n_tile * kTcRows;
  const int t0 = t_tile * TN;
  const int total_units = p.K / p.unit_k;
  const int u_begin = (KSPLIT == 2 && rank == 1) ? p.split_units : 0;
  const int u_end = (KSPLIT == 2 && rank == 0) ? p.split_units : total_units;
  const int k_begin = u_begin * p.unit_k;
  const int k_end = u_end * p.unit_k;
  const int c_begin = k_begin / kTcK;
  const int c_end = k_end / kTcK;
  const int g_begin = k_begin >> p.group_shift;
  const int n_groups = (k_end - k_begin) >> p.group_shift;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::kStages; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->dq_full[s], 4);  // the four warps that cover one stage's 128 rows
      mbar_init(&ctl->empty[s], 1);
    }
    for (int s = 0; s < Code::kSlots; ++s) {
      mbar_init(&ctl->code_full[s], 1);
      mbar_init(&ctl->code_empty[s], 4 * Code::kChunksPerSlot);
    }
    for (int b = 0; b < Cfg::kNBuf; ++b) {
      mbar_init(&ctl->tmem_full[b], 1);
      mbar_init(&ctl->tmem_empty[b], 4 * Cfg::kColSplit);  // the warps that read one group
    }
    mbar_init(&ctl->mma_done, 1);
    ctl->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  float acc[Cfg::kCols];
#pragma unroll
  for (int i = 0; i < Cfg::kCols; ++i) acc[i] = 0.f;
  const bool is_epi = warp >= Cfg::kEpWarp0;
  const int quarter = warp & 3;                      // TMEM lane quarter of an epilogue warp
  const int esub = (warp - Cfg::kEpWarp0) >> 2;           // 0..kEpQ-1 among the warps of a lane quarter
  const int ecol = esub % Cfg::kColSplit;            // column part
  const int egrp = esub / Cfg::kColSplit;            // group residue

  if (warp == 0) {
    // ------------------------------------------------------------ activation TMA
    // (every role that is not the bottleneck parks on its barrier instead of
    // spinning, leaving issue slots to the dequantization warps)
    if (lane == 0) {
      uint32_t stage = 0, phase = 0, issued = 0;
      for (int c = c_begin; c < c_end; ++c) {
        if (!mbar_wait_sleep(&ctl->empty[stage], phase ^ 1u, abort_flag)) break;
        mbar_arrive_expect_tx(&ctl->full[stage], Cfg::kActBytes);
#pragma unroll
        for (int sb = 0; sb < kSub; ++sb)
          tma_load_2d(ring + stage * Cfg::kStageBytes + sb * TN * 128, &tmA, &ctl->full[stage], c * kTcK + 64 * sb, t0);
        ++issued;
        if (++stage == Cfg::kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      // every issued copy must land before the CTA may exit
      const uint32_t first = issued > Cfg::kStages ? issued - Cfg::kStages : 0;
      for (uint32_t i = first; i < issued; ++i) mbar_wait_drain(&ctl->full[i % Cfg::kStages], (i / Cfg::kStages) & 1u);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Nothing but the MMAs may sit between consecutive MMAs: one issuing thread
    // needs ~45 cycles per instruction at best, and a descriptor rebuilt or a
    // branch taken per k-step doubles that.  B descriptors are a precomputed
    // low word plus a constant; group starts and ends are decided per stage.
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kTcRows, TN, false, false);
      constexpr int kSteps = kTcK / 16;
      const uint64_t bdesc0 = sdesc_sw128(smem_u32(ring), 16, 1024);
      const uint32_t blo0 = static_cast<uint32_t>(bdesc0), bhi = static_cast<uint32_t>(bdesc0 >> 32);
      const int gsteps = (1 << p.group_shift) >> 4;  // k16 steps per group: 2 .. 64
      uint32_t stage = 0, phase = 0, buf = 0, bphase = 0;
      int kstep = 0;
      bool ok = true;
      for (int c = c_begin; ok && c < c_end; ++c) {
        if (!mbar_wait_sleep(&ctl->dq_full[stage], phase, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_col = tmem + kACol0 + kACols * stage;
        const uint32_t blo = blo0 + stage * (Cfg::kStageBytes >> 4);
        if (gsteps >= kSteps) {
          // at most one group boundary per stage: at its first and/or last k-step
          const bool gstart = (kstep & (gsteps - 1)) == 0;
          const bool gend = ((kstep + kSteps) & (gsteps - 1)) == 0;
          if (gstart) {
            if (!mbar_wait_sleep(&ctl->tmem_empty[buf], bphase ^ 1u, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
          const uint32_t d = tmem + buf * TN;
          umma_bf16_ta(d, a_col, mk_desc(blo, bhi), idesc, gstart ? 0u : 1u);
#pragma unroll
          for (int k = 1; k < kSteps; ++k)
            umma_bf16_ta(d, a_col + 8 * k, mk_desc(blo + (((k >> 2) * TN * 128 + 32 * (k & 3)) >> 4), bhi), idesc, 1u);
          if (gend) {
            umma_commit(&ctl->tmem_full[buf]);
            if (++buf == Cfg::kNBuf) {
              buf = 0;
              bphase ^= 1u;
            }
          }
        } else {
          // g = 32 or 64: two or four groups per stage
#pragma unroll
          for (int k = 0; k < kSteps; ++k) {
            const bool gstart = ((kstep + k) & (gsteps - 1)) == 0;
            if (gstart) {
              if (!mbar_wait_sleep(&ctl->tmem_empty[buf], bphase ^ 1u, abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
            }
            umma_bf16_ta(tmem + buf * TN, a_col + 8 * k,
                         mk_desc(blo + (((k >> 2) * TN * 128 + 32 * (k & 3)) >> 4), bhi), idesc, gstart ? 0u : 1u);
            if (((kstep + k + 1) & (gsteps - 1)) == 0) {
              umma_commit(&ctl->tmem_full[buf]);
              if (++buf == Cfg::kNBuf) {
                buf = 0;
                bphase ^= 1u;
              }
            }
          }
          if (!ok) break;
        }
        kstep += kSteps;
        umma_commit(&ctl->empty[stage]);
        if (++stage == Cfg::kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      // all issued MMAs complete before TMEM is released
      umma_commit(&ctl->mma_done);
      mbar_wait_drain(&ctl->mma_done, 0);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ code TMA: up to 16 stages ahead
    if (lane == 0) {
      constexpr int kChunksPerSlot = Code::kChunksPerSlot;
      constexpr int kStageWords = kTcK * BITS / 32;  // 32-bit words of a row per stage
      const int n_slots = (c_end - c_begin + kChunksPerSlot - 1) / kChunksPerSlot;
      uint32_t slots = 0;
      for (int j = 0; j < n_slots; ++j) {
        const uint32_t cs = static_cast<uint32_t>(j % Code::kSlots);
        if (!mbar_wait_sleep(&ctl->code_empty[cs], ((j / Code::kSlots) & 1u) ^ 1u, abort_flag)) break;
        // a slot's boxes are consecutive 32-word spans of the rows; boxes that start past this
        // CTA's last stage hold nothing it reads and are not loaded (the first always is)
        const int x0 = (c_begin + j * kChunksPerSlot) * kStageWords;
        int boxes = 1;
        while (boxes < Code::kBoxes && x0 + 32 * boxes < c_end * kStageWords) ++boxes;
        mbar_arrive_expect_tx(&ctl->code_full[cs], boxes * kCodeBytes);
        for (int b = 0; b < boxes; ++b)
          tma_load_2d(codes + cs * Code::kSlotBytes + b * kCodeBytes, &tmW, &ctl->code_full[cs], x0 + 32 * b, n0);
        ++slots;
      }
      const uint32_t first_slot = slots > Code::kSlots ? slots - Code::kSlots : 0;
      for (uint32_t j = first_slot; j < slots; ++j)
        mbar_wait_drain(&ctl->code_full[j % Code::kSlots], (j / Code::kSlots) & 1u);
    }
  } else if (!is_epi) {
    // ------------------------------------------------------------ dequantization
    // warp -> the 32 rows of its TMEM lane quarter (warp % 4, hardware rule) and
    // every (kDqWarps / 4)-th stage
    const int dw = warp - kDqWarp0;
    const int r = (warp & 3) * 32 + lane;  // weight row within the tile = TMEM lane
    const int n = n0 + r;
    MetaRow zrow;
    if (!FP4) zrow.start(p.z16 + static_cast<size_t>(n < p.N ? n : 0) * p.G, g_begin, p.G, p.vec_meta != 0, n < p.N);
    const uint32_t sw = static_cast<uint32_t>(r & 7);
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + kACol0;
    // code slots: every dequantization set reads every phase of a slot (stages per slot a multiple
    // of the sets), or each slot is always read by the same set (the sets a multiple of the stages
    // per slot and their ratio dividing the slot count), so each set waits on a slot's phases in order
    static_assert(slot_phases_in_order(Code::kChunksPerSlot, Cfg::kDqWarps / 4, Code::kSlots),
                  "code slots: phases waited in order by every dequantization set");
    for (int i = dw >> 2; i < c_end - c_begin; i += Cfg::kDqWarps / 4) {
      const int c = c_begin + i;
      const uint32_t stage = static_cast<uint32_t>(i % Cfg::kStages);
      const uint32_t phase = static_cast<uint32_t>((i / Cfg::kStages) & 1);
      constexpr int kChunksPerSlot = Code::kChunksPerSlot;
      const uint32_t j = static_cast<uint32_t>(i / kChunksPerSlot);
      const uint32_t cs = j % Code::kSlots;
      // codes landed, the MMAs of this stage's previous use have released its A
      // operand, and the stage's activations landed (so the MMA thread waits once)
      const bool ok = mbar_wait_sleep(&ctl->code_full[cs], (j / Code::kSlots) & 1u, abort_flag) &&
                      mbar_wait_sleep(&ctl->empty[stage], phase ^ 1u, abort_flag);
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      tc_fence_after();
      // this stage's 16*BITS bytes of row r: 16-byte vectors qv..qv+BITS-1 of the slot's
      // row (vector v in box v / 8 at position v % 8), each box swizzled by r % 8
      const uint32_t qv = static_cast<uint32_t>(BITS * (i % kChunksPerSlot));
      const uint32_t pk = smem_u32(codes + cs * Code::kSlotBytes) + r * 128;
      const int k0 = c * kTcK;
      // the stage's codes: all loads issued before any conversion, except that
      // 8-bit stages (eight 16-byte vectors a row) load one half at a time
      constexpr int kPre = BITS == 8 ? BITS / 2 : BITS;
      uint4 pw[kPre];
#pragma unroll
      for (int v = 0; v < kPre; ++v) {
        const uint32_t qvv = qv + v;
        pw[v] = ld_shared_v4(pk + (qvv >> 3) * kCodeBytes + (((qvv & 7) ^ sw) << 4));
      }
      // NVFP4: the row's 8 block scales of this stage (one per two words)
      uint32_t sc2[8];
      if (FP4) {
        uint2 c8 = make_uint2(0u, 0u);
        if (n < p.N) c8 = __ldg(reinterpret_cast<const uint2*>(p.sc8 + static_cast<size_t>(n) * (p.K / 16) + k0 / 16));
        e4m3x8_to_bf16_pairs(c8, sc2);
      }
      // zero-points of the four 32-k quarters (equal when g >= 128), converted once:
      // (128 + z) bf16 pairs for 2 and 4 bits, 2^23 + z in fp32 for 8 bits
      uint32_t zz[4];
      float zf[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        if (FP4) {
          zz[h] = 0u;
          zf[h] = 0.f;
        } else if (h == 0 || p.group_shift < 7) {
          const uint16_t z = zrow.get((k0 + 32 * h) >> p.group_shift);
          if (BITS == 8) zf[h] = 8388608.0f + __half2float(__ushort_as_half(z));
          else zz[h] = zero_pair(z);
        } else {
          zz[h] = zz[0];
          zf[h] = zf[0];
        }
      }
      // column c of the stage holds k = 2c, 2c + 1
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t a[32];
        if (BITS == 8 && half == 1) {
#pragma unroll
          for (int v = 0; v < kPre; ++v) pw[v] = ld_shared_v4(pk + (((qv + kPre + v) ^ sw) << 4));
        }
        if constexpr (BITS == 3) {
          // the half's two 32-code units: words 3u .. 3u + 2 of the stage for unit u = 2 half, 2 half + 1
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int w = 3 * (2 * half + u);
            dequant3x32(vec_word(pw[w >> 2], w & 3), vec_word(pw[(w + 1) >> 2], (w + 1) & 3),
                        vec_word(pw[(w + 2) >> 2], (w + 2) & 3), zz[2 * half + u], &a[16 * u]);
          }
        } else {
#pragma unroll
        for (int v = 0; v < BITS / 2; ++v) {
          const uint4 pv = pw[BITS == 8 ? v : half * (BITS / 2) + v];
          const uint32_t xs[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int w = half * 2 * BITS + 4 * v + u;  // word of the stage; it covers k 32w/BITS ..
            const int quarter = w / BITS;
            const int col = (w - half * 2 * BITS) * (16 / BITS);  // first column of this word in the half
            if (FP4) {
              const uint4 o = dequant_e2m1x8(xs[u], sc2[w >> 1]);  // word w holds k 8w .. 8w + 7: block w / 2
              a[col] = o.x;
              a[col + 1] = o.y;
              a[col + 2] = o.z;
              a[col + 3] = o.w;
            } else if (BITS == 4) {
              const uint4 o = dequant8(xs[u], zz[quarter]);
              a[col] = o.x;
              a[col + 1] = o.y;
              a[col + 2] = o.z;
              a[col + 3] = o.w;
            } else if (BITS == 2) {
              dequant16(xs[u], zz[quarter], &a[col]);
            } else {
              dequant4b(xs[u], zf[quarter], &a[col]);
            }
          }
        }
        }
        tmem_st32(lane_base + kACols * stage + 32 * half, a);
      }
      const bool act_ok = mbar_wait_sleep(&ctl->full[stage], phase, abort_flag);
      tmem_st_wait();
      tc_fence_before();
      if (!__all_sync(0xFFFFFFFFu, act_ok)) break;
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&ctl->dq_full[stage]);
        mbar_arrive(&ctl->code_empty[cs]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue: acc += s * D per group
    const int r = quarter * 32 + lane;
    const int n = n0 + r;
    const int col0 = ecol * Cfg::kCols;
    const int gfirst = egrp;
    constexpr int gstep = Cfg::kGrpSplit;
    MetaRow srow;
    if (!FP4) srow.start(p.s16 + static_cast<size_t>(n < p.N ? n : 0) * p.G, g_begin + gfirst, p.G, p.vec_meta != 0, n < p.N);
    const float S = FP4 ? __ldg(p.gscale) : 0.f;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + col0;
    for (int li = gfirst; li < n_groups; li += gstep) {
      const uint32_t buf = static_cast<uint32_t>(li % Cfg::kNBuf);
      const uint32_t par = static_cast<uint32_t>((li / Cfg::kNBuf) & 1);
      if (!__all_sync(0xFFFFFFFFu, mbar_wait_sleep(&ctl->tmem_full[buf], par, abort_flag))) break;
      tc_fence_after();
      const float s = FP4 ? S : __half2float(__ushort_as_half(srow.get(g_begin + li)));
#pragma unroll
      for (int c = 0; c < Cfg::kCols; c += 16) {
        float v[16];
        tmem_ld16(lane_addr + buf * TN + c, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[c + i] = fmaf(s, v[i], acc[c + i]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->tmem_empty[buf]);
    }
  }

  // ------------------------------------------------------------ reduction and store
  tc_fence_before();
  __syncthreads();  // mainloop over: MMAs complete, copies landed, the ring is free
  float* red = reinterpret_cast<float*>(ring);
  float* fin = reinterpret_cast<float*>(ring + Cfg::kRedBytes);
  if (is_epi) {
    const int r = quarter * 32 + lane;
    float* dst = red + (egrp * kTcRows + r) * Cfg::kRedStride + ecol * Cfg::kCols;
#pragma unroll
    for (int i = 0; i < Cfg::kCols; ++i) dst[i] = acc[i];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < kTcRows * TN; e += Cfg::kThreads) {
    const int r = e % kTcRows;
    const int c = e / kTcRows;
    float v = red[r * Cfg::kRedStride + c];
#pragma unroll
    for (int q = 1; q < Cfg::kRedPlanes; ++q) v += red[(q * kTcRows + r) * Cfg::kRedStride + c];
    if (KSPLIT == 2) {
      fin[r * Cfg::kRedStride + c] = v;
    } else {
      const int n = n0 + r, t = t0 + c;
      if (n < p.N && t < p.T) p.out[static_cast<size_t>(t) * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
    }
  }
  if (KSPLIT == 2) {
    cluster_sync_all();
    if (rank == 0) {
      const float* peer = cg::this_cluster().map_shared_rank(fin, 1);
      for (int e = threadIdx.x; e < kTcRows * TN; e += Cfg::kThreads) {
        const int r = e % kTcRows;
        const int c = e / kTcRows;
        const float v = fin[r * Cfg::kRedStride + c] + peer[r * Cfg::kRedStride + c];
        const int n = n0 + r, t = t0 + c;
        if (n < p.N && t < p.T) p.out[static_cast<size_t>(t) * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
      }
    }
    cluster_sync_all();  // rank 1 keeps its shared memory until rank 0 has read it
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int TN, int KSPLIT, int BITS, bool FP4>
cudaError_t launch_tc(const uint16_t* A, const CUtensorMap& tmW, TcParams p, int n_tiles, cudaStream_t stream,
                      const char* name) {
  using Cfg = TcCfg<TN, BITS, FP4>;
  CUtensorMap tmA;
  cudaError_t e = make_tmap_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, A, static_cast<uint64_t>(p.T),
                               static_cast<uint64_t>(p.K), 64, TN, CU_TENSOR_MAP_SWIZZLE_128B);  // kSub boxes per stage
  if (e != cudaSuccess) return e;
  constexpr int smem = Cfg::kRingBytes + static_cast<int>(sizeof(TcCtl)) + 1024;
  static_assert(smem <= 227 * 1024, "shared memory per CTA");
  auto kern = w4a16_tc_kernel<TN, KSPLIT, BITS, FP4>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = KSPLIT;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(n_tiles * p.t_tiles * KSPLIT));
  cfg.blockDim = dim3(Cfg::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  LaunchScope scope(stream, name);
  e = cudaLaunchKernelEx(&cfg, kern, tmA, tmW, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int TN, int BITS, bool FP4 = false>
cudaError_t launch_tn(const uint16_t* A, const CUtensorMap& tmW, TcParams p, int n_tiles, cudaStream_t stream,
                      const char* name1, const char* name2) {
  // Split K over a CTA pair when one CTA per tile leaves more than half the SMs idle.
  const int tiles = n_tiles * p.t_tiles;
  const int total_units = p.K / p.unit_k;
  if (2 * tiles <= num_sms() && total_units >= 2) {
    p.split_units = (total_units + 1) / 2;
    const int g_split = (p.split_units * p.unit_k) >> p.group_shift;
    p.vec_meta = (p.G % 8 == 0 && g_split % 8 == 0) ? 1 : 0;
    return launch_tc<TN, 2, BITS, FP4>(A, tmW, p, n_tiles, stream, name2);
  }
  p.split_units = total_units;
  p.vec_meta = p.G % 8 == 0 ? 1 : 0;
  return launch_tc<TN, 1, BITS, FP4>(A, tmW, p, n_tiles, stream, name1);
}


// profiler / trace names per width: TN = 16, 32, 64, 128, each unsplit and split over a CTA pair
template <int BITS>
struct TcNames;
template <>
struct TcNames<2> {
  static constexpr const char* n[8] = {"wxa16_tc_kernel<b=2,TN=16>", "wxa16_tc_kernel<b=2,TN=16,split2>",
                                       "wxa16_tc_kernel<b=2,TN=32>", "wxa16_tc_kernel<b=2,TN=32,split2>",
                                       "wxa16_tc_kernel<b=2,TN=64>", "wxa16_tc_kernel<b=2,TN=64,split2>",
                                       "wxa16_tc_kernel<b=2,TN=128>", "wxa16_tc_kernel<b=2,TN=128,split2>"};
};
template <>
struct TcNames<3> {
  static constexpr const char* n[8] = {"wxa16_tc_kernel<b=3,TN=16>", "wxa16_tc_kernel<b=3,TN=16,split2>",
                                       "wxa16_tc_kernel<b=3,TN=32>", "wxa16_tc_kernel<b=3,TN=32,split2>",
                                       "wxa16_tc_kernel<b=3,TN=64>", "wxa16_tc_kernel<b=3,TN=64,split2>",
                                       "wxa16_tc_kernel<b=3,TN=128>", "wxa16_tc_kernel<b=3,TN=128,split2>"};
};
template <>
struct TcNames<4> {
  static constexpr const char* n[8] = {"w4a16_tc_kernel<TN=16>", "w4a16_tc_kernel<TN=16,split2>",
                                       "w4a16_tc_kernel<TN=32>", "w4a16_tc_kernel<TN=32,split2>",
                                       "w4a16_tc_kernel<TN=64>", "w4a16_tc_kernel<TN=64,split2>",
                                       "w4a16_tc_kernel<TN=128>", "w4a16_tc_kernel<TN=128,split2>"};
};
template <>
struct TcNames<8> {
  static constexpr const char* n[8] = {"wxa16_tc_kernel<b=8,TN=16>", "wxa16_tc_kernel<b=8,TN=16,split2>",
                                       "wxa16_tc_kernel<b=8,TN=32>", "wxa16_tc_kernel<b=8,TN=32,split2>",
                                       "wxa16_tc_kernel<b=8,TN=64>", "wxa16_tc_kernel<b=8,TN=64,split2>",
                                       "wxa16_tc_kernel<b=8,TN=128>", "wxa16_tc_kernel<b=8,TN=128,split2>"};
};

// NVFP4 names (TN = 16, 32, 64, 128, each unsplit and split over a CTA pair)
constexpr const char* kFp4Names[8] = {"nvfp4_tc_kernel<TN=16>", "nvfp4_tc_kernel<TN=16,split2>",
                                      "nvfp4_tc_kernel<TN=32>", "nvfp4_tc_kernel<TN=32,split2>",
                                      "nvfp4_tc_kernel<TN=64>", "nvfp4_tc_kernel<TN=64,split2>",
                                      "nvfp4_tc_kernel<TN=128>", "nvfp4_tc_kernel<TN=128,split2>"};

template <int BITS>
cudaError_t launch_bits_tc(const uint16_t* A, int T, const uint32_t* packed, const uint16_t* scale16,
                           const uint16_t* zero16, int N, int K, int group_size, uint16_t* out, cudaStream_t stream) {
  TcParams p{};
  p.s16 = scale16;
  p.z16 = zero16;
  p.out = out;
  p.N = N;
  p.K = K;
  p.T = T;
  p.G = K / group_size;
  while ((1 << p.group_shift) < group_size) ++p.group_shift;
  p.unit_k = group_size > kTcK ? group_size : kTcK;
  CUtensorMap tmW;
  cudaError_t e = make_tmap_2d(&tmW, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, packed, static_cast<uint64_t>(N),
                               static_cast<uint64_t>(K) * BITS / 32, 32, kTcRows, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  const int n_tiles = (N + kTcRows - 1) / kTcRows;
  if (T <= 16) {
    p.t_tiles = 1;
    return launch_tn<16, BITS>(A, tmW, p, n_tiles, stream, TcNames<BITS>::n[0], TcNames<BITS>::n[1]);
  }
  if (T <= 32) {
    p.t_tiles = 1;
    return launch_tn<32, BITS>(A, tmW, p, n_tiles, stream, TcNames<BITS>::n[2], TcNames<BITS>::n[3]);
  }
  if (T <= 64) {
    p.t_tiles = 1;
    return launch_tn<64, BITS>(A, tmW, p, n_tiles, stream, TcNames<BITS>::n[4], TcNames<BITS>::n[5]);
  }
  p.t_tiles = (T + 127) / 128;
  return launch_tn<128, BITS>(A, tmW, p, n_tiles, stream, TcNames<BITS>::n[6], TcNames<BITS>::n[7]);
}

}  // namespace

cudaError_t launch_w4a16_tc(const uint16_t* A, int T, const uint32_t* packed, const uint16_t* scale16,
                            const uint16_t* zero16, int N, int K, int group_size, uint16_t* out, cudaStream_t stream) {
  return launch_bits_tc<4>(A, T, packed, scale16, zero16, N, K, group_size, out, stream);
}

cudaError_t launch_nvfp4_tc(const uint16_t* A, int T, const uint8_t* codes, const uint8_t* scales, const float* gscale,
                            int N, int K, uint16_t* out, cudaStream_t stream) {
  if (T < 1 || N < 1 || K < kTcK || K % kTcK != 0) return cudaErrorInvalidValue;
  TcParams p{};
  p.sc8 = scales;
  p.gscale = gscale;
  p.out = out;
  p.N = N;
  p.K = K;
  p.T = T;
  // accumulation groups: the largest power of two up to 1024 that divides K (the per-tensor
  // scale is the same for all of them, so fewer groups mean fewer epilogue passes)
  p.group_shift = 7;
  while (p.group_shift < 10 && K % (1 << (p.group_shift + 1)) == 0) ++p.group_shift;
  p.G = K >> p.group_shift;
  p.unit_k = 1 << p.group_shift;
  CUtensorMap tmW;
  cudaError_t e = make_tmap_2d(&tmW, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, codes, static_cast<uint64_t>(N),
                               static_cast<uint64_t>(K) / 8, 32, kTcRows, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  const int n_tiles = (N + kTcRows - 1) / kTcRows;
  if (T <= 16) {
    p.t_tiles = 1;
    return launch_tn<16, 4, true>(A, tmW, p, n_tiles, stream, kFp4Names[0], kFp4Names[1]);
  }
  if (T <= 32) {
    p.t_tiles = 1;
    return launch_tn<32, 4, true>(A, tmW, p, n_tiles, stream, kFp4Names[2], kFp4Names[3]);
  }
  if (T <= 64) {
    p.t_tiles = 1;
    return launch_tn<64, 4, true>(A, tmW, p, n_tiles, stream, kFp4Names[4], kFp4Names[5]);
  }
  p.t_tiles = (T + 127) / 128;
  return launch_tn<128, 4, true>(A, tmW, p, n_tiles, stream, kFp4Names[6], kFp4Names[7]);
}

cudaError_t launch_wxa16_tc(const uint16_t* A, int T, const uint32_t* packed, const uint16_t* scale16,
                            const uint16_t* zero16, int N, int K, int group_size, int bits, uint16_t* out,
                            cudaStream_t stream) {
  if (bits == 2) return launch_bits_tc<2>(A, T, packed, scale16, zero16, N, K, group_size, out, stream);
  if (bits == 3) return launch_bits_tc<3>(A, T, packed, scale16, zero16, N, K, group_size, out, stream);
  if (bits == 4) return launch_bits_tc<4>(A, T, packed, scale16, zero16, N, K, group_size, out, stream);
  if (bits == 8) return launch_bits_tc<8>(A, T, packed, scale16, zero16, N, K, group_size, out, stream);
  return cudaErrorInvalidValue;
}

}  // namespace ar
