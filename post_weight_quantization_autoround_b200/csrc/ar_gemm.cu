// Tensor-core GEMMs of the AutoRound tuning step on sm_100a (tcgen05 + TMEM + TMA).
//
// The step ([AR] §3 "Algorithm Flow", steps 2-5) has two dense contractions
// per linear layer: the QDQ forward Y_hat = X W_hat^T and the weight gradient
// dW_hat = G^T X.  Both run in one persistent, warp-specialised kernel
// template; what differs is operand major-ness and the fused epilogue:
//
//   EPI_STORE  D (fp32) = A B^T                          (reference forward, tests)
//   EPI_RESID  R = A B^T - Y; G = bf16(R * 2/(MN)); per-tile sum R^2
//              (MSE loss and its gradient, [AR] §3 step 4)
//   EPI_FOLD   straight-through fold of dW_hat into dV (per element) and
//              dalpha/dbeta (per group), then the SignSGD step and clamp
//              ([AR] §3 "SignSGD"; STE as in [IA])
//   EPI_SWIGLU_FWD  gate and up products of a SwiGLU block in one 256-wide
//              tile (128 gate rows + the same 128 up rows of B): a, b -> bf16,
//              h = bf16(silu(a) b)  ([AR] §3 "Why Block-Wise Optimization")
//   EPI_SWIGLU_BWD  dH = G W_down; SiLU backward: dA = bf16(dH b silu'(a)),
//              dB = bf16(dH silu(a))
//   EPI_QKV    the decoder block's stacked Q, K, V projection: bf16 out, with the
//              rotary embedding applied to the Q and K columns (head halves
//              (x_i, x_{i+d/2}) rotated by the position's angle, from a table)
//   EPI_RESADD fp32 out = accumulator + a bf16 residual (X2 = X + O Wo^T)
//   EPI_STORE_BF16  bf16 out (the attention output's gradient dO = dX2 Wo)
// EPI_RESID optionally adds an fp32 residual before the difference: R = (acc +
// X2) - Y, the decoder block's output Y_hat = X2 + h Wd^T.
//
// ([AR] = "Low-Bit Quantization in Practice with vLLM: Core Mechanisms and
// Architectural Optimizations of AutoRound"; [IA] = "Intel AutoRound 高级量化".)
//
// Launch: persistent clusters of two CTAs (320 threads each, one CTA per SM).
// For the residual, reference-forward, plain, SwiGLU and (unsplit) weight-
// gradient GEMMs the pair computes one 256x256 output tile as a tcgen05 CTA
// pair: in each CTA warp 0 lane 0 issues TMA loads of its 128 A rows and its
// 128 of the tile's 256 B columns into a 6-stage ring (128-byte swizzle),
// completing on the even CTA's barrier; warp 1 allocates 512 TMEM columns
// together with the peer (two 128x256 fp32 accumulators) and, in the even CTA,
// lane 0 issues tcgen05.mma.cta_group::2.kind::f16 (M=256, N=256, K=16) and
// commits to both CTAs' barriers; warps 2-9 drain this CTA's accumulator rows
// with tcgen05.ld while the MMAs fill the other accumulator: warp w reads TMEM
// lanes 32*(w%4)..+31 (one output row per thread) and one half of the 256
// columns, so two warps share each lane quarter.  Tiles are strided over the
// clusters with the N index fastest so that concurrently running pairs share
// the A panel.  The weight-gradient GEMM from 32768 tokens on instead runs
// 128x256 one-CTA tiles whose reduction the two CTAs of a cluster split.
//
// Operands: A is [M][K] (K-major) or [K][M] (MN-major); B is [N][K] or [K][N].
// The weight-gradient GEMM reads G [tokens][N_w] and X [tokens][K_w] directly
// as MN-major operands, so no transpose is ever materialised.
//
// Every mbarrier wait is bounded (ar_device.cuh): on a timeout the kernel
// raises a block abort flag and the sticky device status, all roles leave
// their loops, in-flight TMA copies and MMAs are drained, TMEM is freed.
#include <algorithm>

#include "ar_fold.cuh"
#include "ar_internal.h"

namespace ar {
namespace {

constexpr int BM = 128;   // A rows per CTA (MMA M of one CTA)
constexpr int BN = 256;   // output columns per tile
constexpr int BK = 64;
constexpr int kMaxStages = 6;
constexpr int kEpiWarps = 8;                       // two per TMEM lane quarter
constexpr int kThreads = 64 + 32 * kEpiWarps;     // TMA warp, MMA warp, epilogue warps
constexpr int kAStage = BM * BK * 2;  // 16 KiB
constexpr int kTmemCols = 2 * BN;     // double-buffered accumulator

// CG = 1: one CTA per 128 x 256 tile.  CG = 2: a CTA pair per 256 x 256 tile
// (tcgen05 .cta_group::2): each CTA loads its 128 A rows and half of the B
// columns, so per SM the operand traffic from L2 falls from 48 to 32 KiB per
// 64-k block of the same MMA work.  Every CTA's accumulator still holds all
// 256 columns of its rows, so the epilogues are unchanged (the SwiGLU forward
// tile's gate half comes from the even CTA, its up half from the odd one).
template <int CG>
struct GemmCfg {
  static constexpr int kBStage = (BN / CG) * BK * 2;  // 32 or 16 KiB
  static constexpr int kStages = CG == 2 ? 6 : 4;
  static constexpr int kSmemBytes = kStages * (kAStage + kBStage) + 1024 + 24576;
  static_assert(kStages <= kMaxStages, "barrier arrays");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
};

enum {
  EPI_STORE = 0,
  EPI_RESID = 1,
  EPI_FOLD = 2,
  EPI_SWIGLU_FWD = 3,
  EPI_SWIGLU_BWD = 4,
  EPI_QKV = 5,
  EPI_RESADD = 6,
  EPI_STORE_BF16 = 7
};

struct Ctl {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
  float2 xch[4][2][32];  // fold epilogue: per lane quarter, the two halves' group sums
  uint64_t xbar[4];      // and the mbarrier that orders their exchange
  // split reduction (two CTAs of a cluster): rank 1 ships 32 rows x 16 columns
  // of its accumulator per message into rank 0's slot of the same epilogue warp
  uint64_t full_x[kEpiWarps];   // rank 0: message landed (32 remote arrivals)
  uint64_t empty_x[kEpiWarps];  // rank 1: slot free again (one remote arrival per message)
  float slot[kEpiWarps][32][20];  // 16 floats per lane, padded against bank conflicts
};
static_assert(sizeof(Ctl) <= 24576, "control block too large");

struct Params {
  int M, N, K;  // D is M x N, reduction over K
  int tiles_m, tiles_n, num_kb;
  int num_units;   // work units of this launch
  int full_units;  // units below this are whole tiles; from it on, two half-width units per tile
  int group_m;     // tile rows per raster group (columns swept inside a group, rows fastest)
  float* D;          // EPI_STORE
  const float* Y;    // EPI_RESID
  uint16_t* G;
  float gscale;
  double* partial;
  FoldArgs fold;     // EPI_FOLD
  uint16_t* act_a;   // EPI_SWIGLU_FWD outputs / EPI_SWIGLU_BWD inputs: a, b, h [M][N] bf16
  uint16_t* act_b;
  uint16_t* act_h;
  uint16_t* grad_a;  // EPI_SWIGLU_BWD outputs: dA, dB [M][ld_grad] bf16
  uint16_t* grad_b;
  int ld_grad;
  const float* Yadd;          // EPI_RESID: optional fp32 residual added before the difference
  const uint16_t* res;        // EPI_RESADD: bf16 residual [M][N]
  uint16_t* Dbf;              // EPI_QKV / EPI_STORE_BF16: bf16 out [M][N]
  const float2* rope;         // EPI_QKV: (cos, sin) [rope_L][head_dim / 2]
  int rope_cols, rope_L, head_dim;  // columns below rope_cols are rotated; position = row % rope_L
};

// Byte offsets of the MN-major canonical layout: the leading-dimension offset
// steps between 64-element (128 B) chunks of the contiguous dimension, which
// are 8 KiB apart (one 64-row TMA box each); the stride-dimension offset steps
// between 8-row groups along K, 1 KiB apart.
constexpr uint32_t kMnLbo = 8192;
constexpr uint32_t kMnSbo = 1024;

template <bool MN>
__device__ __forceinline__ uint64_t operand_desc(uint32_t stage_base, int kstep) {
  if (MN) {
    // K-step of 16 rows = two 8-row core groups = 2 KiB further.
    return sdesc_sw128(stage_base + kstep * 2048, kMnLbo, kMnSbo);
  } else {
    // K-major: a K-step of 16 bf16 is 32 bytes inside the 128-byte swizzle atom.
    return sdesc_sw128(stage_base + kstep * 32, 16, 1024);
  }
}

// ---------------------------------------------------------------------------
// epilogues: one thread = one output row, 32 columns per TMEM load
// ---------------------------------------------------------------------------
__device__ __forceinline__ void epi_store(const Params& p, uint32_t taddr, int row, int col_base, int c0, int c1) {
#pragma unroll 1
  for (int c = c0; c < c1; ++c) {
    float v[32];
    tmem_ld32(taddr + c * 32, v);
    const int col0 = col_base + c * 32;
    if (row >= p.M || col0 >= p.N) continue;
    float* d = p.D + static_cast<size_t>(row) * p.N + col0;
    if (col0 + 32 <= p.N) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        *reinterpret_cast<float4*>(d + 4 * i) = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    } else {
      for (int i = 0; i < 32 && col0 + i < p.N; ++i) d[i] = v[i];
    }
  }
}

__device__ __forceinline__ double epi_resid(const Params& p, uint32_t taddr, int row, int col_base, int c0,
                                            int c1) {
  double acc = 0.0;
#pragma unroll 1
  for (int c = c0; c < c1; ++c) {
    float v[32];
    tmem_ld32(taddr + c * 32, v);
    const int col0 = col_base + c * 32;
    if (row >= p.M || col0 >= p.N) continue;
    const float* y = p.Y + static_cast<size_t>(row) * p.N + col0;
    uint16_t* g = p.G + static_cast<size_t>(row) * p.N + col0;
    if (p.Yadd) {
      const float* ya = p.Yadd + static_cast<size_t>(row) * p.N + col0;
      for (int i = 0; i < 32 && col0 + i < p.N; ++i) v[i] = __fadd_rn(v[i], ya[i]);
    }
    float part = 0.0f;
    if (col0 + 32 <= p.N) {
      uint32_t gp[16];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 yv = *reinterpret_cast<const float4*>(y + 4 * i);
        const float r0 = __fsub_rn(v[4 * i + 0], yv.x);
        const float r1 = __fsub_rn(v[4 * i + 1], yv.y);
        const float r2 = __fsub_rn(v[4 * i + 2], yv.z);
        const float r3 = __fsub_rn(v[4 * i + 3], yv.w);
        part += r0 * r0 + r1 * r1 + r2 * r2 + r3 * r3;
        gp[2 * i] = pack_bf16x2(__fmul_rn(r0, p.gscale), __fmul_rn(r1, p.gscale));
        gp[2 * i + 1] = pack_bf16x2(__fmul_rn(r2, p.gscale), __fmul_rn(r3, p.gscale));
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
        *reinterpret_cast<uint4*>(g + 8 * i) = make_uint4(gp[4 * i], gp[4 * i + 1], gp[4 * i + 2], gp[4 * i + 3]);
    } else {
      for (int i = 0; i < 32 && col0 + i < p.N; ++i) {
        const float r = __fsub_rn(v[i], y[i]);
        part += r * r;
        __nv_bfloat16 h = __float2bfloat16_rn(__fmul_rn(r, p.gscale));
        g[i] = *reinterpret_cast<uint16_t*>(&h);
      }
    }
    acc += static_cast<double>(part);
  }
  return acc;
}

// Straight-through fold + SignSGD.  GEMM rows are weight rows n (M = N_w),
// GEMM columns are weight columns k (N = K_w).  Each epilogue warp owns 32
// rows and half of the unit's columns (chunks of 32: four of a whole 256-column
// tile, two of a half-width unit).  A group that fits in a warp's half keeps
// its sums in the thread; a group as wide as the unit (256 of a whole tile, 128
// of a half-width unit) spans both halves and the two warps of a lane quarter
// add their partial sums through shared memory (fixed order: half 0 + half 1).
//
// All global loads of the tile (group parameters, W and V of the first chunk)
// are issued before waiting for the accumulator, and each next chunk's W and
// V are loaded while the current chunk is computed.
struct FoldChunk {
  uint4 w[4];   // 32 bf16 weights
  float4 v[8];  // 32 rounding offsets
};

__device__ __forceinline__ void fold_load(const FoldArgs& f, size_t e, FoldChunk& ch) {
#pragma unroll
  for (int i = 0; i < 4; ++i) ch.w[i] = *reinterpret_cast<const uint4*>(f.W + e + 8 * i);
#pragma unroll
  for (int i = 0; i < 8; ++i) ch.v[i] = *reinterpret_cast<const float4*>(f.V + e + 4 * i);
}

// `wait_acc` waits for the accumulator (returns false on abort); `xch` is this
// lane quarter's exchange slot [2 halves][32 lanes] of float2 in shared memory
// and `xbar` its mbarrier (two arrivals per phase, two phases per exchange).
// Rank 0 of a split pair receives the peer's partial accumulator: per message
// 16 columns of this warp's 32 rows, added as own + peer.
struct SplitRecv {
  bool on;
  const float* slot;      // this lane's 16 floats
  uint64_t* full;         // local barrier the peer arrives on
  uint32_t peer_empty;    // the peer's slot-free barrier (cluster address)
  uint32_t* msg;          // messages received so far by this warp
};

// `nch`: 32-column chunks per warp, 4 for a whole tile and 2 for a half-width unit;
// a group of 2 nch chunks spans both warps of the lane quarter (the host never
// gives a half-width unit groups wider than the unit).
template <class WaitAcc>
__device__ __forceinline__ bool epi_fold(const Params& p, uint32_t taddr, int n, int col_base, int half, int nch,
                                         float2* xch, uint64_t* xbar, volatile int* abort_flag, WaitAcc wait_acc,
                                         bool* aborted, const SplitRecv& rx) {
  const FoldArgs& f = p.fold;
  const int g = f.group_size;
  const int cpg = g >> 5;  // chunks per group: 1, 2, 4 or 8
  const int groups_per_row = p.N / g;
  const float Q = static_cast<float>((1 << f.bits) - 1);
  const int c0 = nch * half;
  const bool row_ok = n < p.M;
  bool bad = false;

  GroupParams gp{};
  FoldChunk cur, nxt;
  // prefetch before the accumulator is ready
  if (row_ok && col_base + c0 * 32 < p.N) {
    const int col = col_base + c0 * 32;
    group_load(f, static_cast<size_t>(n) * groups_per_row + col / g, gp);
    fold_load(f, static_cast<size_t>(n) * p.N + col, nxt);
  }
  if (!wait_acc()) {
    *aborted = true;
    return false;
  }
  float csum = 0.f, osum = 0.f;
#pragma unroll 1
  for (int c = c0; c < c0 + nch; ++c) {
    const int col0 = col_base + c * 32;
    const bool ok = row_ok && col0 < p.N;
    cur = nxt;
    if (ok && c + 1 < c0 + nch && col0 + 32 < p.N) fold_load(f, static_cast<size_t>(n) * p.N + col0 + 32, nxt);
    if (ok && ((c % cpg) == 0 || c == c0)) {
      if (c != c0) group_load(f, static_cast<size_t>(n) * groups_per_row + col0 / g, gp);
      group_prepare(f, gp);
      csum = 0.f;
      osum = 0.f;
    }
    const size_t e = static_cast<size_t>(n) * p.N + col0;
    // two messages of 16 columns (split pairs), each two sub-blocks of 8 weights:
    // one 16-byte W word, two 16-byte V words and 8 accumulator columns
#pragma unroll
    for (int sc = 0; sc < 2; ++sc) {
      float part[16];
      if (rx.on) {
        if (!__all_sync(0xFFFFFFFFu, mbar_wait_cluster(rx.full, *rx.msg & 1u, abort_flag))) {
          *aborted = true;
          return bad;
        }
        const float4* src = reinterpret_cast<const float4*>(rx.slot);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 v = src[i];
          part[4 * i] = v.x;
          part[4 * i + 1] = v.y;
          part[4 * i + 2] = v.z;
          part[4 * i + 3] = v.w;
        }
        __syncwarp();
        if ((threadIdx.x & 31) == 0) mbar_arrive_remote(rx.peer_empty);
        ++*rx.msg;
      }
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int sb = 2 * sc + h2;
        float gw[8];
        tmem_ld8(taddr + c * 32 + 8 * sb, gw);
        if (rx.on) {
#pragma unroll
          for (int i = 0; i < 8; ++i) gw[i] = __fadd_rn(gw[i], part[8 * h2 + i]);
        }
        if (!ok) continue;
        const uint32_t wr[4] = {cur.w[sb].x, cur.w[sb].y, cur.w[sb].z, cur.w[sb].w};
        float vv[8] = {cur.v[2 * sb].x, cur.v[2 * sb].y, cur.v[2 * sb].z, cur.v[2 * sb].w,
                       cur.v[2 * sb + 1].x, cur.v[2 * sb + 1].y, cur.v[2 * sb + 1].z, cur.v[2 * sb + 1].w};
        float dv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float w = (i & 1) ? bf16_hi(wr[i >> 1]) : bf16_lo(wr[i >> 1]);
          const float wq = __fdiv_rn(w, gp.s);
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
        float* vp = f.V + e + 8 * sb;
        *reinterpret_cast<float4*>(vp) = make_float4(vv[0], vv[1], vv[2], vv[3]);
        *reinterpret_cast<float4*>(vp + 4) = make_float4(vv[4], vv[5], vv[6], vv[7]);
        if (f.dV_out) {
          float* dp = f.dV_out + e + 8 * sb;
          *reinterpret_cast<float4*>(dp) = make_float4(dv[0], dv[1], dv[2], dv[3]);
          *reinterpret_cast<float4*>(dp + 4) = make_float4(dv[4], dv[5], dv[6], dv[7]);
        }
      }
    }
    if (!ok) continue;
    if (cpg <= nch && (c % cpg) == cpg - 1) bad |= group_finish(f, gp, csum, osum, true);
  }
  if (cpg > nch) {
    // a group as wide as the unit: add the two halves' sums (the same order in both warps);
    // phase 0 publishes both halves, phase 1 frees the slot for the next tile
    const int lane = threadIdx.x & 31;
    xch[half * 32 + lane] = make_float2(csum, osum);
    __syncwarp();
    if (lane == 0) mbar_arrive(xbar);
    if (!__all_sync(0xFFFFFFFFu, mbar_wait(xbar, 0, abort_flag))) {
      *aborted = true;
      return bad;
    }
    const float2 a = xch[lane];
    const float2 b = xch[32 + lane];
    __syncwarp();
    if (lane == 0) mbar_arrive(xbar);
    if (!__all_sync(0xFFFFFFFFu, mbar_wait(xbar, 1, abort_flag))) {
      *aborted = true;
      return bad;
    }
    if (row_ok && col_base < p.N) bad |= group_finish(f, gp, __fadd_rn(a.x, b.x), __fadd_rn(a.y, b.y), half == 0);
  }
  return bad;
}

// out = acc + residual (bf16 res or fp32 Yadd), fp32 out.
__device__ __forceinline__ void epi_resadd(const Params& p, uint32_t taddr, int row, int col_base, int c0, int c1) {
#pragma unroll 1
  for (int c = c0; c < c1; ++c) {
    float v[32];
    tmem_ld32(taddr + c * 32, v);
    const int col0 = col_base + c * 32;
    if (row >= p.M || col0 >= p.N) continue;
    const size_t e = static_cast<size_t>(row) * p.N + col0;
    for (int i = 0; i < 32 && col0 + i < p.N; ++i) {
      const float x = p.res ? __uint_as_float(static_cast<uint32_t>(p.res[e + i]) << 16) : p.Yadd[e + i];
      p.D[e + i] = __fadd_rn(v[i], x);
    }
  }
}

// bf16 out of 32 accumulator columns (round to nearest even).
__device__ __forceinline__ void store_bf16_32(uint16_t* dst, const float (&v)[32], int n) {
  if (n == 32) {
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
#pragma unroll
    for (int i = 0; i < 4; ++i) *reinterpret_cast<uint4*>(dst + 8 * i) = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
  } else {
    for (int i = 0; i < n; ++i) {
      const __nv_bfloat16 h = __float2bfloat16_rn(v[i]);
      dst[i] = *reinterpret_cast<const uint16_t*>(&h);
    }
  }
}

__device__ __forceinline__ void epi_store_bf16(const Params& p, uint32_t taddr, int row, int col_base, int c0,
                                               int c1) {
#pragma unroll 1
  for (int c = c0; c < c1; ++c) {
    float v[32];
    tmem_ld32(taddr + c * 32, v);
    const int col0 = col_base + c * 32;
    if (row >= p.M || col0 >= p.N) continue;
    store_bf16_32(p.Dbf + static_cast<size_t>(row) * p.N + col0, v, min(32, p.N - col0));
  }
}

// Stacked Q, K, V projection with the rotary embedding on the Q and K columns.
// This thread's 128 columns (chunks c0..c0+3) start on a head boundary, so the
// head halves it rotates together, columns i and i + d/2, are both its own:
// chunk pairs (c0, c0+2), (c0+1, c0+3) for d = 128 and (c0, c0+1), (c0+2, c0+3)
// for d = 64.  (x1, x2) -> (x1 cos - x2 sin, x2 cos + x1 sin) in fp32, then bf16.
__device__ __forceinline__ void epi_qkv(const Params& p, uint32_t taddr, int row, int col_base, int c0) {
  const int dist = p.head_dim / 64;  // chunks between the two halves of a head
#pragma unroll 1
  for (int pr = 0; pr < 2; ++pr) {
    const int ca = c0 + (dist == 2 ? pr : 2 * pr);
    const int cb = ca + dist;
    float va[32], vb[32];
    tmem_ld32(taddr + ca * 32, va);
    tmem_ld32(taddr + cb * 32, vb);
    const int cola = col_base + ca * 32, colb = col_base + cb * 32;
    if (row >= p.M || cola >= p.N) continue;
    if (cola < p.rope_cols) {
      const int t = row % p.rope_L;
      const float2* cs = p.rope + static_cast<size_t>(t) * (p.head_dim / 2) + (cola % p.head_dim);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float2 r = cs[i];
        const float x1 = va[i], x2 = vb[i];
        va[i] = __fsub_rn(__fmul_rn(x1, r.x), __fmul_rn(x2, r.y));
        vb[i] = __fadd_rn(__fmul_rn(x2, r.x), __fmul_rn(x1, r.y));
      }
    }
    store_bf16_32(p.Dbf + static_cast<size_t>(row) * p.N + cola, va, 32);
    store_bf16_32(p.Dbf + static_cast<size_t>(row) * p.N + colb, vb, 32);
  }
}

__device__ __forceinline__ float bf16_round(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }
__device__ __forceinline__ float sigmoidf(float x) { return __fdiv_rn(1.0f, __fadd_rn(1.0f, expf(-x))); }

// SwiGLU forward: TMEM columns 0..127 hold the gate product a, 128..255 the
// up product b of the same 128 outputs f.  Writes a, b, h = silu(a) b (bf16).
__device__ __forceinline__ void epi_swiglu_fwd(const Params& p, uint32_t taddr, int row, int f_base, int c0,
                                               int c1) {
#pragma unroll 1
  for (int c = c0; c < c1; ++c) {
    float va[32], vb[32];
    tmem_ld32(taddr + c * 32, va);
    tmem_ld32(taddr + 128 + c * 32, vb);
    const int col0 = f_base + c * 32;
    if (row >= p.M || col0 >= p.N) continue;
    const size_t e = static_cast<size_t>(row) * p.N + col0;
    uint32_t pa[16], pb[16], ph[16];
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      const float a0 = bf16_round(va[i]), a1 = bf16_round(va[i + 1]);
      const float b0 = bf16_round(vb[i]), b1 = bf16_round(vb[i + 1]);
      pa[i / 2] = pack_bf16x2(a0, a1);
      pb[i / 2] = pack_bf16x2(b0, b1);
      ph[i / 2] = pack_bf16x2(__fmul_rn(__fmul_rn(a0, sigmoidf(a0)), b0), __fmul_rn(__fmul_rn(a1, sigmoidf(a1)), b1));
    }
    if (col0 + 32 <= p.N) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (p.act_a) *reinterpret_cast<uint4*>(p.act_a + e + 8 * i) = make_uint4(pa[4 * i], pa[4 * i + 1], pa[4 * i + 2], pa[4 * i + 3]);
        if (p.act_b) *reinterpret_cast<uint4*>(p.act_b + e + 8 * i) = make_uint4(pb[4 * i], pb[4 * i + 1], pb[4 * i + 2], pb[4 * i + 3]);
        *reinterpret_cast<uint4*>(p.act_h + e + 8 * i) = make_uint4(ph[4 * i], ph[4 * i + 1], ph[4 * i + 2], ph[4 * i + 3]);
      }
    } else {
      for (int i = 0; i < 32 && col0 + i < p.N; ++i) {
        const int sh = (i & 1) ? 16 : 0;
        if (p.act_a) p.act_a[e + i] = static_cast<uint16_t>(pa[i / 2] >> sh);
        if (p.act_b) p.act_b[e + i] = static_cast<uint16_t>(pb[i / 2] >> sh);
        p.act_h[e + i] = static_cast<uint16_t>(ph[i / 2] >> sh);
      }
    }
  }
}

// SiLU backward on dH (the accumulator): dA = dH b silu'(a), dB = dH silu(a).
__device__ __forceinline__ bool epi_swiglu_bwd(const Params& p, uint32_t taddr, int row, int col_base, int c0,
                                               int c1) {
  bool bad = false;
#pragma unroll 1
  for (int c = c0; c < c1; ++c) {
    float dh[32];
    tmem_ld32(taddr + c * 32, dh);
    const int col0 = col_base + c * 32;
    if (row >= p.M || col0 >= p.N) continue;
    const size_t e = static_cast<size_t>(row) * p.N + col0;
    const int n = col0 + 32 <= p.N ? 32 : p.N - col0;
    uint32_t ra[16], rb[16];
    if (n == 32) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 x = *reinterpret_cast<const uint4*>(p.act_a + e + 8 * i);
        const uint4 y = *reinterpret_cast<const uint4*>(p.act_b + e + 8 * i);
        ra[4 * i] = x.x; ra[4 * i + 1] = x.y; ra[4 * i + 2] = x.z; ra[4 * i + 3] = x.w;
        rb[4 * i] = y.x; rb[4 * i + 1] = y.y; rb[4 * i + 2] = y.z; rb[4 * i + 3] = y.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        ra[i] = 0;
        rb[i] = 0;
      }
      for (int i = 0; i < n; ++i) {
        ra[i / 2] |= static_cast<uint32_t>(p.act_a[e + i]) << ((i & 1) ? 16 : 0);
        rb[i / 2] |= static_cast<uint32_t>(p.act_b[e + i]) << ((i & 1) ? 16 : 0);
      }
    }
    uint32_t ga[16], gb[16];
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      float da[2], db[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const float a = u ? bf16_hi(ra[i / 2]) : bf16_lo(ra[i / 2]);
        const float b = u ? bf16_hi(rb[i / 2]) : bf16_lo(rb[i / 2]);
        const float sg = sigmoidf(a);
        const float ds = __fmul_rn(sg, __fadd_rn(1.0f, __fmul_rn(a, __fsub_rn(1.0f, sg))));
        da[u] = __fmul_rn(__fmul_rn(dh[i + u], b), ds);
        db[u] = __fmul_rn(dh[i + u], __fmul_rn(a, sg));
        bad |= !isfinite(dh[i + u]);
      }
      ga[i / 2] = pack_bf16x2(da[0], da[1]);
      gb[i / 2] = pack_bf16x2(db[0], db[1]);
    }
    const size_t eo = static_cast<size_t>(row) * p.ld_grad + col0;
    if (n == 32) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        *reinterpret_cast<uint4*>(p.grad_a + eo + 8 * i) = make_uint4(ga[4 * i], ga[4 * i + 1], ga[4 * i + 2], ga[4 * i + 3]);
        *reinterpret_cast<uint4*>(p.grad_b + eo + 8 * i) = make_uint4(gb[4 * i], gb[4 * i + 1], gb[4 * i + 2], gb[4 * i + 3]);
      }
    } else {
      for (int i = 0; i < n; ++i) {
        const int sh = (i & 1) ? 16 : 0;
        p.grad_a[eo + i] = static_cast<uint16_t>(ga[i / 2] >> sh);
        p.grad_b[eo + i] = static_cast<uint16_t>(gb[i / 2] >> sh);
      }
    }
  }
  return bad;
}

// Tile (tm, tn) of unit t of a grid of tiles_m x tiles_n tiles in raster order:
// groups of group_m tile rows, and inside a group the row index fastest (group_m
// = 1: rows one after another, columns fastest).
__host__ __device__ __forceinline__ void raster(int t, int tiles_m, int tiles_n, int group_m, int& tm, int& tn) {
  if (group_m <= 1) {
    tm = t / tiles_n;
    tn = t - tm * tiles_n;
    return;
  }
  const int per_group = group_m * tiles_n;
  const int grp = t / per_group;
  const int in = t - grp * per_group;
  const int rows = min(group_m, tiles_m - grp * group_m);
  tn = in / rows;
  tm = grp * group_m + (in - tn * rows);
}

// Work unit t: output tile (tm, tn) of this launch's BM * CG-row tiles, its first
// column and width.  Units below full_units are whole tiles in raster order; the
// tiles after them (the last wave's, when it would leave clusters idle) are run
// as two units of BN / 2 columns each, which other clusters take at the same time.
struct Unit {
  int tm, tn, col0;
  int tile;   // tile index in raster order
  int part;   // 0, or 1 for the right half of a split tile
  bool wide;  // BN columns (else BN / 2)
};

__device__ __forceinline__ Unit unit_of(const Params& p, int t) {
  Unit u;
  if (t < p.full_units) {
    u.tile = t;
    u.part = 0;
    u.wide = true;
  } else {
    u.tile = p.full_units + ((t - p.full_units) >> 1);
    u.part = (t - p.full_units) & 1;
    u.wide = false;
  }
  raster(u.tile, p.tiles_m, p.tiles_n, p.group_m, u.tm, u.tn);
  u.col0 = u.tn * BN + u.part * (BN / 2);
  return u;
}

// Raster group for a grid whose B operand has b_bytes: 1 while B fits in a share of
// L2 (B stays resident, A streams once), else as many tile rows as that share holds
// A panels of (A streams once, B once per group).
int raster_group(double b_bytes, double a_panel_bytes, int tiles_m) {
  constexpr double kL2Share = 64.0 * 1024 * 1024;
  if (b_bytes <= kL2Share) return 1;
  return std::max(1, std::min(tiles_m, static_cast<int>(kL2Share / a_panel_bytes)));
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
// KSPLIT = 2 (weight-gradient GEMM only): the two CTAs of a cluster share each
// tile, rank 0 reducing the first half of the k-blocks and rank 1 the second.
// CG = 2: the two CTAs of a cluster compute one 256 x 256 tile as a tcgen05
// pair; rank 0 issues the MMAs, each rank drains its own 128 rows.
template <bool A_MN, bool B_MN, int EPI, int KSPLIT, int CG>
__global__ void __launch_bounds__(kThreads, 1)
    umma_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmB2, const Params p) {
  static_assert(!(KSPLIT == 2 && CG == 2), "a cluster is either a split pair or a tcgen05 pair");
  constexpr int STAGES = GemmCfg<CG>::kStages;
  constexpr int kBStage = GemmCfg<CG>::kBStage;
  constexpr bool kPair = CG == 2;
  constexpr bool kCluster = KSPLIT == 2 || kPair;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* smA = base;
  uint8_t* smB = base + STAGES * kAStage;
  Ctl* ctl = reinterpret_cast<Ctl*>(smB + STAGES * kBStage);
  volatile int* abort_flag = &ctl->abort_flag;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_tiles = p.num_units;
  const int rank = kCluster ? static_cast<int>(cluster_ctarank()) : 0;
  const int tile0 = kCluster ? static_cast<int>(cluster_id_x()) : static_cast<int>(blockIdx.x);
  const int tile_step = kCluster ? static_cast<int>(cluster_count_x()) : static_cast<int>(gridDim.x);
  const int kb_begin = (KSPLIT == 2 && rank == 1) ? p.num_kb / 2 : 0;
  const int kb_end = (KSPLIT == 2 && rank == 0) ? p.num_kb / 2 : p.num_kb;
  const bool leader = !kPair || rank == 0;  // issues the MMAs (always, unless a pair's odd CTA)

  if (threadIdx.x == 0) {
    for (int w = 0; w < kEpiWarps; ++w) {
      mbar_init(&ctl->full_x[w], 32);
      mbar_init(&ctl->empty_x[w], 1);
    }
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&ctl->tmem_full[a], 1);
      mbar_init(&ctl->tmem_empty[a], kEpiWarps * CG);  // a pair's accumulator is drained by both CTAs
    }
    mbar_init(&ctl->mma_done, 1);
    for (int q = 0; q < 4; ++q) mbar_init(&ctl->xbar[q], 2);
    ctl->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (EPI == EPI_SWIGLU_FWD) tma_prefetch_desc(&tmB2);
  }
  if (warp == 1) {
    if (kPair) {
      tmem_alloc_pair(&ctl->tmem_base, kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(&ctl->tmem_base, kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (kCluster) cluster_sync_all();  // the peer's barriers are initialised before any remote arrival
  const uint32_t tmem = ctl->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      uint32_t issued = 0;
      bool ok = true;
      for (int t = tile0; ok && t < num_tiles; t += tile_step) {
        const Unit u = unit_of(p, t);
        const int tm = u.tm, tn = u.tn;
        // this CTA's A rows and B columns (a pair's CTA loads half of the unit's columns)
        const int b_cols = u.wide ? BN / CG : BN / (2 * CG);
        const int m0 = tm * (BM * CG) + rank * (kPair ? BM : 0);
        const int n0 = u.col0 + rank * (kPair ? b_cols : 0);
        for (int kb = kb_begin; kb < kb_end; ++kb) {
          if (!mbar_wait(&ctl->empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* a_dst = smA + stage * kAStage;
          uint8_t* b_dst = smB + stage * kBStage;
          if (kPair) {
            // both CTAs' bytes complete on the even CTA's barrier, which expects them all
            const uint32_t bar0 = mapa_shared(smem_u32(&ctl->full[stage]), 0);
            if (rank == 0) mbar_arrive_expect_tx(&ctl->full[stage], CG * (kAStage + b_cols * BK * 2));
            if (A_MN) {
#pragma unroll
              for (int i = 0; i < BM / 64; ++i) tma_load_2d_pair(a_dst + i * 8192, &tmA, bar0, m0 + 64 * i, kb * BK);
            } else {
              tma_load_2d_pair(a_dst, &tmA, bar0, kb * BK, m0);
            }
            if (EPI == EPI_SWIGLU_FWD) {
              // the tile's B columns are 128 gate rows then the same 128 up rows: one half each
              tma_load_2d_pair(b_dst, rank == 0 ? &tmB : &tmB2, bar0, kb * BK, tn * (BN / 2));
            } else if (B_MN) {
              // 64-column boxes: two for a whole tile's half, one for a half-width unit's
              for (int i = 0; i < b_cols / 64; ++i) tma_load_2d_pair(b_dst + i * 8192, &tmB, bar0, n0 + 64 * i, kb * BK);
            } else {
              // tmB: boxes of BN / 2 rows; tmB2: boxes of BN / 4 rows (half-width units)
              tma_load_2d_pair(b_dst, u.wide ? &tmB : &tmB2, bar0, kb * BK, n0);
            }
          } else {
            mbar_arrive_expect_tx(&ctl->full[stage], kAStage + kBStage);
            if (A_MN) {
#pragma unroll
              for (int i = 0; i < BM / 64; ++i) tma_load_2d(a_dst + i * 8192, &tmA, &ctl->full[stage], m0 + 64 * i, kb * BK);
            } else {
              tma_load_2d(a_dst, &tmA, &ctl->full[stage], kb * BK, m0);
            }
            if (EPI == EPI_SWIGLU_FWD) {
              // 128 gate rows then the same 128 up rows
              tma_load_2d(b_dst, &tmB, &ctl->full[stage], kb * BK, tn * (BN / 2));
              tma_load_2d(b_dst + kBStage / 2, &tmB2, &ctl->full[stage], kb * BK, tn * (BN / 2));
            } else if (B_MN) {
#pragma unroll
              for (int i = 0; i < BN / 64; ++i) tma_load_2d(b_dst + i * 8192, &tmB, &ctl->full[stage], n0 + 64 * i, kb * BK);
            } else {
              tma_load_2d(b_dst, &tmB, &ctl->full[stage], kb * BK, n0);
            }
          }
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Drain: every issued copy must have landed before the CTA may exit (a
      // pair's odd CTA signals the even CTA's barriers, which that CTA drains;
      // the closing cluster barrier keeps the odd CTA alive until then).
      if (leader) {
        const uint32_t first = issued > STAGES ? issued - STAGES : 0;
        for (uint32_t i = first; i < issued; ++i) mbar_wait_drain(&ctl->full[i % STAGES], (i / STAGES) & 1u);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && leader) {
      constexpr uint32_t idesc_wide = idesc_bf16_f32(BM * CG, BN, A_MN, B_MN);
      constexpr uint32_t idesc_half = idesc_bf16_f32(BM * CG, BN / 2, A_MN, B_MN);
      uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
      bool ok = true;
      for (int t = tile0; ok && t < num_tiles; t += tile_step) {
        const uint32_t idesc = t < p.full_units ? idesc_wide : idesc_half;
        // a pair's accumulator is free once both CTAs' epilogues have drained it
        const bool got = kPair ? mbar_wait_cluster(&ctl->tmem_empty[acc], acc_phase ^ 1u, abort_flag)
                               : mbar_wait(&ctl->tmem_empty[acc], acc_phase ^ 1u, abort_flag);
        if (!got) break;
        tc_fence_after();
        const uint32_t d = tmem + acc * BN;
        for (int kb = kb_begin; kb < kb_end; ++kb) {
          if (!mbar_wait(&ctl->full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smA + stage * kAStage);
          const uint32_t b_base = smem_u32(smB + stage * kBStage);
#pragma unroll
          for (int j = 0; j < BK / 16; ++j) {
            if (kPair)
              umma_bf16_pair(d, operand_desc<A_MN>(a_base, j), operand_desc<B_MN>(b_base, j), idesc,
                             (kb != kb_begin || j != 0) ? 1u : 0u);
            else
              umma_bf16(d, operand_desc<A_MN>(a_base, j), operand_desc<B_MN>(b_base, j), idesc,
                        (kb != kb_begin || j != 0) ? 1u : 0u);
          }
          if (kPair) umma_commit_pair(&ctl->empty[stage]);
          else umma_commit(&ctl->empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (kPair) umma_commit_pair(&ctl->tmem_full[acc]);
        else umma_commit(&ctl->tmem_full[acc]);
        acc ^= 1u;
        if (acc == 0) acc_phase ^= 1u;
      }
      // All issued MMAs must be complete before TMEM is released.
      if (kPair) umma_commit_pair(&ctl->mma_done);
      else umma_commit(&ctl->mma_done);
      mbar_wait_drain(&ctl->mma_done, 0);
    } else if (lane == 0) {
      // a pair's odd CTA: its TMEM is written by the even CTA's MMAs
      mbar_wait_drain(&ctl->mma_done, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // warp -> TMEM lane quarter (warp % 4, hardware rule) and column half
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    uint32_t acc = 0, acc_phase = 0;
    bool bad = false;
    const int ew = warp - 2;  // epilogue warp index 0..7
    uint32_t msg = 0;
    SplitRecv rx{};
    if (KSPLIT == 2 && rank == 0) {
      rx.on = true;
      rx.slot = &ctl->slot[ew][lane][0];
      rx.full = &ctl->full_x[ew];
      rx.peer_empty = mapa_shared(smem_u32(&ctl->empty_x[ew]), 1);
      rx.msg = &msg;
    }
    const uint32_t peer_slot = KSPLIT == 2 ? mapa_shared(smem_u32(&ctl->slot[ew][lane][0]), 0) : 0;
    const uint32_t peer_full = KSPLIT == 2 ? mapa_shared(smem_u32(&ctl->full_x[ew]), 0) : 0;
    for (int t = tile0; t < num_tiles; t += tile_step) {
      const Unit u = unit_of(p, t);
      const int tm = u.tm, tn = u.tn;
      const int nch = u.wide ? 4 : 2;  // 32-column chunks per warp: half of the unit's columns
      const int row = tm * (BM * CG) + rank * (kPair ? BM : 0) + quarter * 32 + lane;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + acc * BN;
      auto wait_acc = [&]() {
        const bool got = mbar_wait(&ctl->tmem_full[acc], acc_phase, abort_flag);
        if (!__all_sync(0xFFFFFFFFu, got)) return false;
        tc_fence_after();
        return true;
      };
      if (KSPLIT == 2 && rank == 1) {
        // ship this warp's 32 rows x 128 columns to rank 0, 16 columns per message
        if (!wait_acc()) break;
        bool aborted = false;
        for (int c = 4 * half; c < 4 * half + 4 && !aborted; ++c) {
          float v[32];
          tmem_ld32(taddr + c * 32, v);
#pragma unroll
          for (int sc = 0; sc < 2; ++sc) {
            if (!__all_sync(0xFFFFFFFFu, mbar_wait_cluster(&ctl->empty_x[ew], (msg & 1u) ^ 1u, abort_flag))) {
              aborted = true;
              break;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
              st_cluster_v4(peer_slot + 16 * i, v[16 * sc + 4 * i], v[16 * sc + 4 * i + 1], v[16 * sc + 4 * i + 2],
                            v[16 * sc + 4 * i + 3]);
            mbar_arrive_remote(peer_full);
            ++msg;
          }
        }
        if (aborted) break;
      } else if (EPI == EPI_FOLD) {
        bool aborted = false;
        bad |= epi_fold(p, taddr, row, u.col0, half, nch, &ctl->xch[quarter][0][0], &ctl->xbar[quarter], abort_flag,
                        wait_acc, &aborted, rx);
        if (aborted) break;
      } else {
        if (!wait_acc()) break;
        if (EPI == EPI_STORE) {
          epi_store(p, taddr, row, u.col0, nch * half, nch * half + nch);
        } else if (EPI == EPI_RESID) {
          double part = epi_resid(p, taddr, row, u.col0, nch * half, nch * half + nch);
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xFFFFFFFFu, part, off);
          // two partial slots per tile and warp, one per half: a whole tile fills the first
          // and zeroes the second, so every slot is written once whatever the split
          if (lane == 0) {
            const size_t slot = ((static_cast<size_t>(u.tile) * 2 + u.part) * CG + (kPair ? rank : 0)) * kEpiWarps +
                                half * 4 + quarter;
            p.partial[slot] = part;
            if (u.wide) p.partial[slot + static_cast<size_t>(CG) * kEpiWarps] = 0.0;
          }
        } else if (EPI == EPI_SWIGLU_FWD) {
          epi_swiglu_fwd(p, taddr, row, tn * (BN / 2), 2 * half, 2 * half + 2);
        } else if (EPI == EPI_SWIGLU_BWD) {
          bad |= epi_swiglu_bwd(p, taddr, row, tn * BN, 4 * half, 4 * half + 4);
        } else if (EPI == EPI_QKV) {
          epi_qkv(p, taddr, row, tn * BN, 4 * half);
        } else if (EPI == EPI_RESADD) {
          epi_resadd(p, taddr, row, tn * BN, 4 * half, 4 * half + 4);
        } else {
          epi_store_bf16(p, taddr, row, tn * BN, 4 * half, 4 * half + 4);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (kPair) mbar_arrive_remote(mapa_shared(smem_u32(&ctl->tmem_empty[acc]), 0));
        else mbar_arrive(&ctl->tmem_empty[acc]);
      }
      acc ^= 1u;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (bad) raise_status(kStatusNonFinite);
  }

  tc_fence_before();
  __syncthreads();
  if (kCluster) cluster_sync_all();  // the peer may still read or write this CTA's shared memory or barriers
  if (warp == 1) {
    tc_fence_after();
    if (kPair) tmem_dealloc_pair(tmem, kTmemCols);
    else tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
// bf16 matrix [rows][cols] (cols contiguous, rows ld elements apart; ld = 0: cols), box of
// box_rows x 64 columns, 128-byte swizzle.
cudaError_t make_tmap(CUtensorMap* tm, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows,
                      uint64_t ld = 0) {
  return make_tmap_2d(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, rows, cols, 64, box_rows,
                      CU_TENSOR_MAP_SWIZZLE_128B, ld);
}

// lda, ldb: row strides (elements) of A and B as stored, 0 for dense.
template <bool A_MN, bool B_MN, int EPI, int KSPLIT = 1, int CG = 1>
cudaError_t run(const uint16_t* A, const uint16_t* B, Params p, cudaStream_t stream, const char* name,
                const uint16_t* B2 = nullptr, uint64_t lda = 0, uint64_t ldb = 0) {
  CUtensorMap tmA, tmB, tmB2;
  // A: K-major [M][K] with 128-row boxes, or MN-major [K][M] with 64-row boxes.
  cudaError_t e = A_MN ? make_tmap(&tmA, A, p.K, p.M, 64, lda) : make_tmap(&tmA, A, p.M, p.K, BM, lda);
  if (e != cudaSuccess) return e;
  if (EPI == EPI_SWIGLU_FWD) {
    // gate and up weights [N][K], 128-row boxes each
    e = make_tmap(&tmB, B, p.N, p.K, BN / 2);
    if (e != cudaSuccess) return e;
    e = make_tmap(&tmB2, B2, p.N, p.K, BN / 2);
  } else {
    // a pair's CTA loads half of the unit's B columns: BN / CG rows of a K-major B for a
    // whole tile (tmB), half of that for a half-width unit (tmB2); MN-major B in 64-column boxes
    e = B_MN ? make_tmap(&tmB, B, p.K, p.N, 64, ldb) : make_tmap(&tmB, B, p.N, p.K, BN / CG, ldb);
    tmB2 = tmB;
    if (e == cudaSuccess && !B_MN && CG == 2) e = make_tmap(&tmB2, B, p.N, p.K, BN / (2 * CG), ldb);
  }
  if (e != cudaSuccess) return e;
  p.tiles_m = (p.M + BM * CG - 1) / (BM * CG);
  p.tiles_n = EPI == EPI_SWIGLU_FWD ? (p.N + BN / 2 - 1) / (BN / 2) : (p.N + BN - 1) / BN;
  p.num_kb = (p.K + BK - 1) / BK;
  p.num_units = p.tiles_m * p.tiles_n;
  p.full_units = p.num_units;
  // raster order
  {
    const double b_bytes = static_cast<double>(p.N) * p.K * 2 * (EPI == EPI_SWIGLU_FWD ? 2 : 1);
    p.group_m = raster_group(b_bytes, static_cast<double>(BM * CG) * p.K * 2, p.tiles_m);
  }
  auto kern = umma_gemm_kernel<A_MN, B_MN, EPI, KSPLIT, CG>;
  constexpr int kSmemBytes = GemmCfg<CG>::kSmemBytes;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  const int tiles = p.num_units;
  if (KSPLIT == 1 && CG == 1) {
    const int grid = tiles < num_sms() ? tiles : num_sms();
    LaunchScope scope(stream, name);
    kern<<<grid, kThreads, kSmemBytes, stream>>>(tmA, tmB, tmB2, p);
    return cudaGetLastError();
  }
  // pairs of CTAs: as many clusters as can be resident at once, at most one per tile
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int max_clusters = 0;
  cfg.gridDim = dim3(2 * (num_sms() / 2));
  e = cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg);
  if (e != cudaSuccess) return e;
  if (max_clusters < 1) return cudaErrorInvalidConfiguration;
  // A last wave of rem < clusters whole tiles leaves clusters idle while it runs: when its
  // tiles split in two fit one wave (2 rem <= clusters), they run as half-width units (same
  // rows, BN / 2 columns each), so that wave takes about half a tile's time.  Tcgen05 pair
  // tiles of the store, residual and fold epilogues only, with whole column tiles, and for
  // the fold groups no wider than the half unit.
  if (CG == 2 && KSPLIT == 1 && p.N % BN == 0 &&
      (EPI == EPI_STORE || EPI == EPI_RESID || (EPI == EPI_FOLD && p.fold.group_size <= BN / 2))) {
    const int rem = tiles % max_clusters;
    if (rem > 0 && 2 * rem <= max_clusters) {
      p.full_units = tiles - rem;
      p.num_units = tiles + rem;
    }
  }
  const int clusters = p.num_units < max_clusters ? p.num_units : max_clusters;
  cfg.gridDim = dim3(2 * clusters);
  LaunchScope scope(stream, name);
  e = cudaLaunchKernelEx(&cfg, kern, tmA, tmB, tmB2, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// One block per step; the partial sums of a step are added in a fixed order.
__global__ void loss_reduce_kernel(const double* __restrict__ partial, int n, double inv_count,
                                   float* __restrict__ loss) {
  __shared__ double sh[256];
  partial += static_cast<size_t>(blockIdx.x) * n;
  double acc = 0.0;
  for (int i = threadIdx.x; i < n; i += 256) acc += partial[i];
  sh[threadIdx.x] = acc;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) sh[threadIdx.x] += sh[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) loss[blockIdx.x] = static_cast<float>(sh[0] * inv_count);
}

}  // namespace

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

cudaError_t make_tmap_2d(CUtensorMap* tm, CUtensorMapDataType dtype, uint32_t elem_bytes, const void* ptr,
                         uint64_t rows, uint64_t cols, uint32_t box_cols, uint32_t box_rows,
                         CUtensorMapSwizzle swizzle, uint64_t ld) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {(ld ? ld : cols) * elem_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(tm, dtype, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// The residual, reference-forward, plain and (unsplit) weight-gradient GEMMs run
// as CTA pairs on 256 x 256 tiles; each CTA's eight epilogue warps write two
// loss partials per tile (one per half-width unit; a whole tile zeroes the second).
constexpr int kPairCG = 2;
int resid_partials(int M, int N) {
  return ((M + BM * kPairCG - 1) / (BM * kPairCG)) * ((N + BN - 1) / BN) * 2 * kPairCG * kEpiWarps;
}

cudaError_t launch_gemm_store(const uint16_t* X, const uint16_t* W, float* Y, int M, int N, int K,
                              cudaStream_t stream) {
  Params p{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.D = Y;
  return run<false, false, EPI_STORE, 1, kPairCG>(X, W, p, stream, "umma_gemm<K,K,store,pair>");
}

cudaError_t launch_gemm_resid(const uint16_t* X, const uint16_t* W_hat, const float* Y, uint16_t* G, float gscale,
                              double* loss_partial, int M, int N, int K, cudaStream_t stream, const float* Yadd) {
  Params p{};
  p.Yadd = Yadd;
  p.M = M;
  p.N = N;
  p.K = K;
  p.Y = Y;
  p.G = G;
  p.gscale = gscale;
  p.partial = loss_partial;
  return run<false, false, EPI_RESID, 1, kPairCG>(X, W_hat, p, stream, "umma_gemm<K,K,resid,pair>");
}

cudaError_t launch_gemm_fold(const uint16_t* G, const uint16_t* X, const FoldArgs& fa, int M, int N, int K,
                             cudaStream_t stream, int64_t ldg, int64_t ldx) {
  // dW_hat[N_w][K_w] = G[tokens][N_w]^T X[tokens][K_w]: GEMM M = N_w, N = K_w, reduction = tokens.
  Params p{};
  p.M = N;
  p.N = K;
  p.K = M;
  p.fold = fa;
  // Split the token reduction over CTA pairs when pairs fill the last wave
  // better and each half of the reduction still outlasts the fold epilogue of
  // a tile (~60 us, compute bound), i.e. from 32768 tokens on; below that the
  // epilogue paces the pair and the unsplit kernel is faster (measured on
  // 16384 tokens: 533 us split vs 511 us unsplit for a 4096 x 4096 layer).
  // Both variants run one cluster of two CTAs per work unit: a 256 x 256 tcgen05
  // pair tile, or a 128 x 256 tile whose reduction is split in halves.
  const int pairs = num_sms() / 2;
  const int tiles_pair = ((N + 2 * BM - 1) / (2 * BM)) * ((K + BN - 1) / BN);
  const int tiles_split = ((N + BM - 1) / BM) * ((K + BN - 1) / BN);
  const double eff1 = static_cast<double>(tiles_pair) / (((tiles_pair + pairs - 1) / pairs) * pairs);
  const double eff2 = static_cast<double>(tiles_split) / (((tiles_split + pairs - 1) / pairs) * pairs);
  if (M >= 32768 && eff2 > eff1 + 0.02)
    return run<true, true, EPI_FOLD, 2>(G, X, p, stream, "umma_gemm<MN,MN,fold,split2>", nullptr, ldg, ldx);
  return run<true, true, EPI_FOLD, 1, kPairCG>(G, X, p, stream, "umma_gemm<MN,MN,fold,pair>", nullptr, ldg, ldx);
}

cudaError_t launch_gemm_swiglu_fwd(const uint16_t* X, const uint16_t* Wg, const uint16_t* Wu, uint16_t* A_out,
                                   uint16_t* B_out, uint16_t* H_out, int M, int F, int Hd, cudaStream_t stream) {
  Params p{};
  p.M = M;
  p.N = F;
  p.K = Hd;
  p.act_a = A_out;
  p.act_b = B_out;
  p.act_h = H_out;
  return run<false, false, EPI_SWIGLU_FWD, 1, kPairCG>(X, Wg, p, stream, "umma_gemm<K,K,swiglu_fwd,pair>", Wu);
}

cudaError_t launch_gemm_swiglu_bwd(const uint16_t* G, const uint16_t* Wd_hat, const uint16_t* A_in,
                                   const uint16_t* B_in, uint16_t* dA, uint16_t* dB, int M, int F, int Hd,
                                   cudaStream_t stream, int ld_grad) {
  // dH[M][F] = G[M][Hd] W_down[Hd][F]: A = G (K-major over Hd), B = W_down as [K=Hd][N=F] (MN-major)
  Params p{};
  p.M = M;
  p.N = F;
  p.K = Hd;
  p.act_a = const_cast<uint16_t*>(A_in);
  p.act_b = const_cast<uint16_t*>(B_in);
  p.grad_a = dA;
  p.grad_b = dB;
  p.ld_grad = ld_grad > 0 ? ld_grad : F;
  return run<false, true, EPI_SWIGLU_BWD, 1, kPairCG>(G, Wd_hat, p, stream, "umma_gemm<K,MN,swiglu_bwd,pair>");
}

cudaError_t launch_gemm_plain(const uint16_t* A, bool a_mn, const uint16_t* B, bool b_mn, float* D, int M, int N,
                              int K, cudaStream_t stream) {
  Params p{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.D = D;
  if (!a_mn && !b_mn) return run<false, false, EPI_STORE, 1, kPairCG>(A, B, p, stream, "umma_gemm<K,K,store,pair>");
  if (!a_mn && b_mn) return run<false, true, EPI_STORE, 1, kPairCG>(A, B, p, stream, "umma_gemm<K,MN,store,pair>");
  if (a_mn && !b_mn) return run<true, false, EPI_STORE, 1, kPairCG>(A, B, p, stream, "umma_gemm<MN,K,store,pair>");
  return run<true, true, EPI_STORE, 1, kPairCG>(A, B, p, stream, "umma_gemm<MN,MN,store,pair>");
}

cudaError_t launch_gemm_qkv(const uint16_t* X, const uint16_t* Wqkv, uint16_t* out, const float* rope_cs, int M,
                            int H, int L, int head_dim, cudaStream_t stream) {
  // out [M][3H] = X [M][H] Wqkv [3H][H]^T, the first 2H columns rotated
  Params p{};
  p.M = M;
  p.N = 3 * H;
  p.K = H;
  p.Dbf = out;
  p.rope = reinterpret_cast<const float2*>(rope_cs);
  p.rope_cols = 2 * H;
  p.rope_L = L;
  p.head_dim = head_dim;
  return run<false, false, EPI_QKV, 1, kPairCG>(X, Wqkv, p, stream, "umma_gemm<K,K,qkv_rope,pair>");
}

cudaError_t launch_gemm_resadd(const uint16_t* A, const uint16_t* W, const uint16_t* res, const float* res_f32,
                               float* out, int M, int N, int K, cudaStream_t stream) {
  // out [M][N] fp32 = residual (bf16 res, else fp32 res_f32) + A [M][K] W [N][K]^T
  Params p{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.res = res;
  p.Yadd = res_f32;
  p.D = out;
  return run<false, false, EPI_RESADD, 1, kPairCG>(A, W, p, stream, "umma_gemm<K,K,resadd,pair>");
}

cudaError_t launch_gemm_store_bf16_kmn(const uint16_t* A, const uint16_t* B_kn, uint16_t* out, int M, int N, int K,
                                       cudaStream_t stream) {
  // out [M][N] bf16 = A [M][K] B with B stored [K][N] (MN-major)
  Params p{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.Dbf = out;
  return run<false, true, EPI_STORE_BF16, 1, kPairCG>(A, B_kn, p, stream, "umma_gemm<K,MN,store_bf16,pair>");
}

cudaError_t launch_loss_reduce(const double* partials, int n, int steps, double inv_count, float* loss,
                               cudaStream_t stream) {
  {
    LaunchScope scope(stream, "loss_reduce_kernel");
    loss_reduce_kernel<<<steps, 256, 0, stream>>>(partials, n, inv_count, loss);
  }
  return cudaGetLastError();
}

}  // namespace ar
