// Causal softmax attention forward of the decoder block on the fifth-generation
// tensor cores (tcgen05 + TMEM + TMA), head dimension 128, sample lengths a
// multiple of 128.  The mma.sync kernel's method (ar_decoder.cu): z = s * scale
// with s = q . k (fp32 accumulation of bf16 products), lse the row's log-sum-exp
// over its keys (pass 1), then P = bf16(exp(z - lse)) and O = P V (pass 2), so a
// probability's rounding does not depend on the order in which keys are
// visited.  Here every exp(z - a) is 2^(s scale log2 e - a log2 e) by the
// hardware's base-2 exponential after one fused multiply-add: a few fp32 ulp
// from the exact value, far below the bf16 rounding of P.
//
// [AR] §3 "Why Block-Wise Optimization" and "Algorithm Flow": the decoder block
// is the unit of tuning, its output's error reaches every weight through
// attention ([AR] = "Low-Bit Quantization in Practice with vLLM: Core Mechanisms
// and Architectural Optimizations of AutoRound").
//
// One CTA per 128 query rows of one (sample, head); the key blocks are the 128
// rows of the sample up to the diagonal.  Warp roles:
//  * warp 0: TMA producer.  Q once (two 64-column boxes of 128 rows, 128-byte
//    swizzle), then the K blocks of pass 1 and the K and V blocks of pass 2 in
//    the order the MMAs consume them, into a 3-deep K ring and a 2-deep V ring.
//  * warp 1: TMEM owner (512 columns) and, in lane 0, the S issuer: S = Q K^T
//    (M = 128 queries, N = 128 keys, K = 128, A and B K-major from shared
//    memory) into one of two fp32 S buffers, for pass 1 and then pass 2.
//  * warp 18, lane 0: the P V issuer: O += P V (A = P as bf16 pairs in tensor
//    memory, B = V as an MN-major operand from shared memory) into the fp32 O
//    accumulator.  Two issuing threads on two sub-partitions, so that neither
//    chain waits on the other's issue; the softmax of one block overlaps the
//    MMAs of the next.
//  * warps 2-17: softmax and epilogue.  Warp w reads TMEM lanes 32 (w % 4) ..
//    + 31 (one query row per thread, hardware rule) and 32 of the 128 key
//    columns (four warps per lane quarter).  Pass 1 keeps a running (max, sum)
//    per thread over its 32 keys; the four warps of a lane quarter combine them
//    once at the end through shared memory, in a fixed order.  Pass 2 writes
//    P = bf16(exp(z - lse)) into one of two P buffers in tensor memory (column
//    c holds keys 2c, 2c + 1).  At the end each warp drains 32 of O's 128
//    columns and stores bf16, and the lse.
//
// TMEM columns: S buffers [0, 256), P buffers [256, 384), O [384, 512).
// Every mbarrier wait is bounded (ar_device.cuh): on a timeout the kernel
// raises the abort flag and the sticky device status, every role leaves its
// loop, in-flight copies and MMAs are drained and TMEM is freed.
#include "ar_attn_tc.cuh"

namespace ar {
namespace {

constexpr int kAtD = 128;                  // head dimension
constexpr int kAtBlk = 128;                // query rows per CTA = keys per block
constexpr int kAtBox = kAtBlk * 128;       // 16 KiB: 128 rows x 64 bf16 columns (one 128-byte swizzle row each)
constexpr int kAtTile = 2 * kAtBox;        // 32 KiB: 128 rows x 128 columns
constexpr int kAtKStages = 3;
constexpr int kAtVStages = 2;
constexpr int kAtSmWarps = 16;             // four per TMEM lane quarter
constexpr int kAtPerQ = kAtSmWarps / 4;
constexpr int kAtWCols = kAtBlk / kAtPerQ;  // key columns of a block (and head columns of O) per warp
static_assert(kAtWCols == 32, "the softmax role loads and stores 32-column slices");
constexpr int kAtPvWarp = 2 + kAtSmWarps;   // issuer of the P V products
constexpr int kAtThreads = (3 + kAtSmWarps) * 32;
constexpr uint32_t kAtColS = 0;            // two S buffers of 128 fp32 columns
constexpr uint32_t kAtColP = 256;          // two P buffers of 64 columns (bf16 pairs)
constexpr uint32_t kAtColO = 384;          // O: 128 fp32 columns
constexpr uint32_t kAtTmemCols = 512;

struct AtCtl {
  uint64_t q_full;
  uint64_t k_full[kAtKStages];
  uint64_t k_empty[kAtKStages];
  uint64_t v_full[kAtVStages];
  uint64_t v_empty[kAtVStages];
  uint64_t s_full[2];   // MMA: S buffer written
  uint64_t s_empty[2];  // softmax warps: S buffer read (one arrival per softmax warp)
  uint64_t p_full[2];   // softmax warps: P buffer written (one arrival per softmax warp)
  uint64_t p_empty[2];  // P V issuer: P V of the buffer done
  uint64_t o_full;
  uint64_t mma_done;
  uint64_t mma_done_pv;
  uint32_t tmem_base;
  int abort_flag;
  float2 ml[4][kAtPerQ][32];  // pass 1: (max, sum) per lane quarter, column part and row
};

constexpr int kAtSmem = kAtTile * (1 + kAtKStages + kAtVStages) + static_cast<int>(sizeof(AtCtl)) + 1024;
static_assert(kAtSmem <= 227 * 1024, "shared memory per CTA");

// Operand layouts (descriptor offsets per K = 16 step kk, added to a descriptor
// built once per tile with at_desc_add):
//  * Q and K, K-major 128 rows x 128 columns as two 64-column swizzled boxes:
//    32 bytes inside a 128-byte swizzle row, box kk / 4 (16 KiB further);
//  * V as the MN-major B operand (N = head columns, K = keys): 64-column chunks
//    are the two boxes (leading offset 16 KiB), 8-key row groups 1 KiB apart,
//    step kk 16 rows = 2 KiB further.

__global__ void __launch_bounds__(kAtThreads, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQKV, int H, int L, int nh, float scale,
                       uint16_t* __restrict__ out, float* __restrict__ lse_out) {
  extern __shared__ uint8_t at_smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(at_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;
  uint8_t* sK = sQ + kAtTile;
  uint8_t* sV = sK + kAtKStages * kAtTile;
  AtCtl* ctl = reinterpret_cast<AtCtl*>(sV + kAtVStages * kAtTile);
  volatile int* abort_flag = &ctl->abort_flag;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nqb = L / kAtBlk;
  const int qb = nqb - 1 - static_cast<int>(blockIdx.x);  // the longest rows first
  const int h = blockIdx.y;
  const int s = blockIdx.z;
  const int n_kb = qb + 1;         // key blocks up to the diagonal
  const int row0 = s * L;          // the sample's first row of qkv

  if (threadIdx.x == 0) {
    mbar_init(&ctl->q_full, 1);
    for (int i = 0; i < kAtKStages; ++i) {
      mbar_init(&ctl->k_full[i], 1);
      mbar_init(&ctl->k_empty[i], 1);
    }
    for (int i = 0; i < kAtVStages; ++i) {
      mbar_init(&ctl->v_full[i], 1);
      mbar_init(&ctl->v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl->s_full[i], 1);
      mbar_init(&ctl->s_empty[i], kAtSmWarps);
      mbar_init(&ctl->p_full[i], kAtSmWarps);
      mbar_init(&ctl->p_empty[i], 1);
    }
    mbar_init(&ctl->o_full, 1);
    mbar_init(&ctl->mma_done, 1);
    mbar_init(&ctl->mma_done_pv, 1);
    ctl->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tmQKV);
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, kAtTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      mbar_arrive_expect_tx(&ctl->q_full, kAtTile);
      tma_load_2d(sQ, &tmQKV, &ctl->q_full, h * kAtD, row0 + qb * kAtBlk);
      tma_load_2d(sQ + kAtBox, &tmQKV, &ctl->q_full, h * kAtD + 64, row0 + qb * kAtBlk);
      uint32_t ki = 0, vi = 0;
      // one 128-row block of K (col0 = H) or V (col0 = 2 H) into its ring
      auto load = [&](uint8_t* ring, uint64_t* full, uint64_t* empty, int stages, uint32_t& idx, int col0,
                      int j) -> bool {
        const uint32_t slot = idx % stages;
        if (!mbar_wait_sleep(&empty[slot], ((idx / stages) & 1u) ^ 1u, abort_flag)) return false;
        uint8_t* dst = ring + slot * kAtTile;
        mbar_arrive_expect_tx(&full[slot], kAtTile);
        tma_load_2d(dst, &tmQKV, &full[slot], col0 + h * kAtD, row0 + j * kAtBlk);
        tma_load_2d(dst + kAtBox, &tmQKV, &full[slot], col0 + h * kAtD + 64, row0 + j * kAtBlk);
        ++idx;
        return true;
      };
      bool ok = true;
      for (int j = 0; ok && j < n_kb; ++j) ok = load(sK, ctl->k_full, ctl->k_empty, kAtKStages, ki, H, j);
      for (int j = 0; ok && j < n_kb; ++j)
        ok = load(sK, ctl->k_full, ctl->k_empty, kAtKStages, ki, H, j) &&
             load(sV, ctl->v_full, ctl->v_empty, kAtVStages, vi, 2 * H, j);
      // every issued copy lands before the CTA may exit
      mbar_wait_drain(&ctl->q_full, 0);
      for (uint32_t i = ki > kAtKStages ? ki - kAtKStages : 0; i < ki; ++i)
        mbar_wait_drain(&ctl->k_full[i % kAtKStages], (i / kAtKStages) & 1u);
      for (uint32_t i = vi > kAtVStages ? vi - kAtVStages : 0; i < vi; ++i)
        mbar_wait_drain(&ctl->v_full[i % kAtVStages], (i / kAtVStages) & 1u);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ S issuer
    // (two issuing threads on two sub-partitions: one thread issuing both the
    // S and the P V products of a block was a limit)
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kAtBlk, kAtBlk, false, false);
      const uint64_t q_desc = sdesc_sw128(smem_u32(sQ), 16, 1024);  // K = 16 steps: compile-time offsets
      bool ok = mbar_wait(&ctl->q_full, 0, abort_flag);
      tc_fence_after();
      // S buffer ns % 2 = Q K^T of the next K block in the ring: pass 1, then pass 2
      for (uint32_t ns = 0; ok && ns < static_cast<uint32_t>(2 * n_kb); ++ns) {
        const uint32_t slot = ns % kAtKStages;
        const uint32_t buf = ns & 1u;
        if (!mbar_wait(&ctl->k_full[slot], (ns / kAtKStages) & 1u, abort_flag) ||
            !mbar_wait(&ctl->s_empty[buf], ((ns >> 1) & 1u) ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t k_desc = sdesc_sw128(smem_u32(sK + slot * kAtTile), 16, 1024);
        const uint32_t d = tmem + kAtColS + buf * kAtBlk;
#pragma unroll
        for (int kk = 0; kk < kAtD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kAtBox + (kk & 3) * 32;
          umma_bf16(d, at_desc_add(q_desc, off), at_desc_add(k_desc, off), idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(&ctl->s_full[buf]);
        umma_commit(&ctl->k_empty[slot]);
      }
      // every issued MMA completes before TMEM is released
      umma_commit(&ctl->mma_done);
      mbar_wait_drain(&ctl->mma_done, 0);
    }
  } else if (warp == kAtPvWarp) {
    // ------------------------------------------------------------ P V issuer
    if (lane == 0) {
      constexpr uint32_t idesc_o = idesc_bf16_f32(kAtBlk, kAtD, false, true);
      bool ok = true;
      for (int j = 0; j < n_kb; ++j) {
        const uint32_t pbuf = static_cast<uint32_t>(j) & 1u;
        const uint32_t vslot = static_cast<uint32_t>(j) % kAtVStages;
        if (!mbar_wait(&ctl->p_full[pbuf], (static_cast<uint32_t>(j) >> 1) & 1u, abort_flag) ||
            !mbar_wait(&ctl->v_full[vslot], (static_cast<uint32_t>(j) / kAtVStages) & 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t v_desc = sdesc_sw128(smem_u32(sV + vslot * kAtTile), kAtBox, 1024);
#pragma unroll
        for (int kk = 0; kk < kAtBlk / 16; ++kk)
          at_mma_ta(tmem + kAtColO, tmem + kAtColP + pbuf * 64 + 8 * kk, at_desc_add(v_desc, kk * 2048), idesc_o,
                    (j > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&ctl->p_empty[pbuf]);
        umma_commit(&ctl->v_empty[vslot]);
      }
      if (ok) umma_commit(&ctl->o_full);
      umma_commit(&ctl->mma_done_pv);
      mbar_wait_drain(&ctl->mma_done_pv, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax and epilogue
    const int quarter = warp & 3;         // TMEM lane quarter (hardware rule: warp % 4)
    const int sub = (warp - 2) >> 2;      // 32-column part: keys of each block, head columns of O
    const int r = quarter * 32 + lane;    // query row within the block
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int k0 = sub * kAtWCols;        // first key column of this warp's part
    uint32_t ns = 0;
    bool ok = true;
    // Exponentials as 2^x with the hardware ex2: exp(z - a) = 2^(s c2 - a log2 e),
    // c2 = scale log2 e, one fused multiply-add per score (a few fp32 ulp from
    // exp(fl(s scale) - a), far below the bf16 rounding of P).  The row maximum is
    // taken over the raw scores (scale > 0).  Only the diagonal block is masked.
    const float c2 = scale * 1.4426950408889634f;
    // pass 1: running (max, sum of exp(scale (s - max))) over this part's keys
    float m = -INFINITY, l = 0.f;
    for (int j = 0; ok && j < n_kb; ++j, ++ns) {
      const uint32_t buf = ns & 1u;
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(&ctl->s_full[buf], (ns >> 1) & 1u, abort_flag));
      if (!ok) break;
      tc_fence_after();
      float v[kAtWCols];
      tmem_ld32(tmem + lane_off + kAtColS + buf * kAtBlk + k0, v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->s_empty[buf]);
      if (j == qb) {
#pragma unroll
        for (int i = 0; i < kAtWCols; ++i) v[i] = k0 + i > r ? -INFINITY : v[i];
      }
      float mx0 = v[0], mx1 = v[1];
#pragma unroll
      for (int i = 2; i < kAtWCols; i += 2) {
        mx0 = fmaxf(mx0, v[i]);
        mx1 = fmaxf(mx1, v[i + 1]);
      }
      const float mn = fmaxf(m, fmaxf(mx0, mx1));
      if (mn != -INFINITY) {  // else every key of the part so far is masked: nothing to add
        const float off = mn * c2;
        float t0 = 0.f, t1 = 0.f;
#pragma unroll
        for (int i = 0; i < kAtWCols; i += 2) {
          t0 += at_ex2(fmaf(v[i], c2, -off));
          t1 += at_ex2(fmaf(v[i + 1], c2, -off));
        }
        l = l * at_ex2((m - mn) * c2) + (t0 + t1);
        m = mn;
      }
    }
    // the row's lse from the parts (part 0 always holds key 0, so its max is finite);
    // every warp of the quarter adds in the same order and reaches this barrier once
    ctl->ml[quarter][sub][lane] = make_float2(m, l);
    at_bar_sync(1 + quarter, 32 * kAtPerQ);
    float mm = ctl->ml[quarter][0][lane].x;
#pragma unroll
    for (int q = 1; q < kAtPerQ; ++q) mm = fmaxf(mm, ctl->ml[quarter][q][lane].x);
    float lsum = 0.f;
#pragma unroll
    for (int q = 0; q < kAtPerQ; ++q) {
      const float2 a = ctl->ml[quarter][q][lane];
      lsum += a.y * at_ex2((a.x - mm) * c2);
    }
    const float lse = __fmul_rn(mm, scale) + logf(lsum);
    const float lse2 = lse * 1.4426950408889634f;
    ok = ok && *abort_flag == 0;
    // pass 2: P = bf16(exp(z - lse)) into a P buffer, read there by the P V MMAs
    for (int j = 0; ok && j < n_kb; ++j, ++ns) {
      const uint32_t buf = ns & 1u;
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(&ctl->s_full[buf], (ns >> 1) & 1u, abort_flag));
      if (!ok) break;
      tc_fence_after();
      float v[kAtWCols];
      tmem_ld32(tmem + lane_off + kAtColS + buf * kAtBlk + k0, v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->s_empty[buf]);
      uint32_t pk[kAtWCols / 2];
      if (j == qb) {
#pragma unroll
        for (int i = 0; i < kAtWCols / 2; ++i) {
          const float p0 = k0 + 2 * i > r ? 0.f : at_ex2(fmaf(v[2 * i], c2, -lse2));
          const float p1 = k0 + 2 * i + 1 > r ? 0.f : at_ex2(fmaf(v[2 * i + 1], c2, -lse2));
          pk[i] = pack_bf16x2(p0, p1);
        }
      } else {
#pragma unroll
        for (int i = 0; i < kAtWCols / 2; ++i)
          pk[i] = pack_bf16x2(at_ex2(fmaf(v[2 * i], c2, -lse2)), at_ex2(fmaf(v[2 * i + 1], c2, -lse2)));
      }
      const uint32_t pbuf = static_cast<uint32_t>(j) & 1u;
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(&ctl->p_empty[pbuf], ((static_cast<uint32_t>(j) >> 1) & 1u) ^ 1u,
                                             abort_flag));
      if (!ok) break;
      tc_fence_after();
      // pair column c of a P buffer holds keys 2c, 2c + 1
      at_tmem_st16(tmem + lane_off + kAtColP + pbuf * 64 + k0 / 2, pk);
      at_tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->p_full[pbuf]);
    }
    // epilogue: O (bf16) for this warp's 32 head columns, and the lse
    bool bad = false;
    if (ok) ok = __all_sync(0xFFFFFFFFu, mbar_wait(&ctl->o_full, 0, abort_flag));
    if (ok) {
      tc_fence_after();
      const int qi = qb * kAtBlk + r;
      uint16_t* orow = out + static_cast<size_t>(row0 + qi) * H + h * kAtD + k0;
      float o[kAtWCols];
      tmem_ld32(tmem + lane_off + kAtColO + k0, o);
      uint32_t w[kAtWCols / 2];
#pragma unroll
      for (int i = 0; i < kAtWCols / 2; ++i) {
        bad |= !isfinite(o[2 * i]) || !isfinite(o[2 * i + 1]);
        w[i] = pack_bf16x2(o[2 * i], o[2 * i + 1]);
      }
#pragma unroll
      for (int i = 0; i < kAtWCols / 8; ++i)
        *reinterpret_cast<uint4*>(orow + 8 * i) = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
      if (sub == 0) lse_out[(static_cast<size_t>(s) * nh + h) * L + qi] = lse;
      tc_fence_before();
    }
    if (bad) raise_status(kStatusNonFinite);
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kAtTmemCols);
  }
}

}  // namespace

// Causal attention forward for head dimension 128 and sample lengths a multiple
// of 128 (qkv bf16 [S L][3 H]: Q, K, V column blocks; out bf16 [S L][H]; lse fp32
// [S][H / 128][L]).  Returns cudaErrorNotSupported for other shapes.
cudaError_t launch_attn_fwd_tc(const uint16_t* qkv, int S, int L, int H, uint16_t* out, float* lse,
                               cudaStream_t st) {
  if (L % kAtBlk != 0 || H % kAtD != 0 || L <= 0 || S <= 0) return cudaErrorNotSupported;
  CUtensorMap tm;
  cudaError_t e = make_tmap_2d(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, qkv, static_cast<uint64_t>(S) * L,
                               static_cast<uint64_t>(3) * H, 64, kAtBlk, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(attn_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kAtSmem);
  if (e != cudaSuccess) return e;
  const int nh = H / kAtD;
  LaunchScope scope(st, "attn_fwd_tc_kernel<d128>");
  attn_fwd_tc_kernel<<<dim3(L / kAtBlk, nh, S), kAtThreads, kAtSmem, st>>>(
      tm, H, L, nh, 1.0f / sqrtf(static_cast<float>(kAtD)), out, lse);
  return cudaGetLastError();
}

}  // namespace ar
