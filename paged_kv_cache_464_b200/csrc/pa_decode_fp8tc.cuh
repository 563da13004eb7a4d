// pa_decode_fp8tc.cuh -- paged decode attention over a 1-byte E4M3 KV cache on
// the 5th-generation tensor cores (tcgen05, kind::f8f6f4): the tensor cores
// read the cache codes straight from the shared-memory tiles the TMA lands,
// so no code is ever converted on the CUDA cores.  Dispatched when the library
// is built with PA_FP8_TC=1; the default E4M3 path is the mma.sync block math
// of pa_decode.cuh, which measured faster on B200 (see pa.cu).
//
// What it computes is the decode of pa_decode.cuh for E4M3 caches (K = k_scale
// * code, V = v_scale * code), with the same grid, partitions and split-K
// partials, so the same reduce kernel finishes split sequences:
//   out[b, h] = sum_t softmax_t(scale * q[b, h] . K_t) V_t.
//
// Products.  A CTA (sequence b, KV head g, partition) walks its tokens in tiles
// of 128 (eight cache blocks).  Per tile
//   S^T[128 tok][N] = K[128 tok][128 d] . Qp[N][128 d]^T    (M=128, K=128 = 4 x 32)
//   O^T[128 d][N]   = V[128 tok][128 d]^T . Pp[N][128 tok]^T (M=128, K=128 = 4 x 32)
// with K read K-major and V MN-major from the same 128-byte-swizzled tiles.
// The N columns carry three E4M3 parts of each of the G query heads (column
// 3h + j, zero-padded to a multiple of 16):
//   q_h 2^e_h = x = x1 + x2 / 16 + x3 / 256,   x1 = e4m3(x), x2 = e4m3(16 (x - x1)), ...
// with e_h the power of two that puts max_d |q_h| in [128, 256), and likewise
// 256 P = p1 + p2 / 16 + p3 / 256 for the softmax weights.  Every part is a
// correctly rounded E4M3 value of an exact fp32 remainder, so the three hold q
// (and P) to about 2^-12 of its size (down to 2^-25 of the largest value), and
// the tensor cores form each part's products exactly and sum them in fp32.
//
// Roles (192 threads):
//   warps 0-3  softmax and epilogue; thread t = tensor-memory lane t.  Per tile:
//              tcgen05.ld of its token's N scores, the tile max per head
//              (redux.sync per warp, an mbarrier-guarded exchange between the
//              four warps), the online max/sum in base 2, the three parts of
//              P written to shared memory as the B operand of the PV product;
//              then, one tile behind, tcgen05.ld of O's row d = t, folded into
//              registers (o = o * alpha + O), so O is never rescaled in place;
//   warp 4     TMA: the K and V boxes of a tile (one 2 KiB box per cache block,
//              out-of-range blocks read as zeros) into a ring of 2 or 3 stages;
//   warp 5     tensor-core issue (one thread): QK(i+1) before PV(i) when tile
//              i+1 has landed, else PV(i) first.
// Tensor memory: S[2] and O[2], N columns each.  Every hand-over is an
// mbarrier; every wait is bounded, and a role that gives up raises a CTA-wide
// abort so that the others stop waiting.  Parity safety: S, P and O hand-overs
// are double-buffered by tile parity and each buffer's next phase needs an
// arrival that follows its waiter's wait (QK(i+2) waits for S(i) to be read,
// P(i+2) is written after the epilogue of tile i has seen PV(i) complete,
// PV(i+2) waits for O(i) to be read); the ring advances one phase per reuse
// that its waiter itself enables (TMA of tile i+3 after PV(i) completes).
#pragma once

#include "pa_common.cuh"
#include "pa_decode.cuh"
#include "pa_tcgen05.cuh"

namespace pa {

constexpr int kTcTok = 128;                          // tokens per tile
constexpr int kTcBlocks = kTcTok / kBlockSize;       // cache blocks per tile
#ifndef PA_FP8TC_STAGES
#define PA_FP8TC_STAGES 0
#endif
// K/V ring depth and resident CTAs an SM: two stages and three CTAs where the
// registers allow it (G <= 4), else three stages and two CTAs
constexpr int fp8tc_stages(int G) { return PA_FP8TC_STAGES > 0 ? PA_FP8TC_STAGES : G == 8 ? 3 : 2; }
constexpr int fp8tc_ctas(int G) { return fp8tc_stages(G) == 2 ? 3 : 2; }
constexpr int kTcTileBytes = kTcTok * 128;           // one K or V tile: 128 rows of 128 codes
constexpr int kTcLoadWarp = 4;
constexpr int kTcMmaWarp = 5;
constexpr int kTcThreads = 32 * (kTcMmaWarp + 1);

template <int G>
struct Fp8TcShape {
  static constexpr int kCols = 3 * G;                        // parts in use: column 3h + j
  static constexpr int N = (kCols + 15) / 16 * 16;           // 16 (G <= 4) or 32
  static constexpr int kTmemCols = 4 * N;                    // S[2], O[2]: 64 or 128
  static constexpr int kStage = 2 * kTcTileBytes;            // K tile, then V tile
  static constexpr int kStages = fp8tc_stages(G);
  static constexpr int kQp = kStages * kStage;             // q parts: N rows x 128 B, K-major, swizzled
  static constexpr int kPp = kQp + N * 128;                  // P parts [2]: N rows x 128 B
  static constexpr int kRed = kPp + 2 * N * 128;             // tile maxima [2][4 warps][G]
  static constexpr int kLsum = kRed + 2 * 4 * G * 4;         // row sums [4 warps][G]
  static constexpr int kQmax = kLsum + 4 * G * 4;            // max |q| [4 warps][G]
  static constexpr int kBar = (kQmax + 4 * G * 4 + 7) / 8 * 8;
  // full[S] free[S] s_full[2] s_free[2] p_full[2] o_full[2] o_free[2] red[2] q_ready drain
  static constexpr int kNumBars = 2 * kStages + 12 + 2;
  static constexpr int kTmemSlot = kBar + 8 * kNumBars;
  static constexpr int kFlag = kTmemSlot + 4;
  static constexpr int kBytes = kFlag + 4;
  static constexpr int kAlloc = kBytes + 1024;               // + alignment of the base (swizzle atoms)
  static_assert(kQp % 1024 == 0 && kPp % 1024 == 0 && (N * 128) % 1024 == 0, "operands on 1024-byte atoms");
  static_assert(kTmemCols >= 32 && (kTmemCols & (kTmemCols - 1)) == 0, "tensor memory: a power of two >= 32");
  static_assert(fp8tc_ctas(G) * (kAlloc + 1024) <= 228 * 1024, "resident CTAs an SM");
};

// Two floats -> two E4M3 codes (byte 0 from lo, byte 1 from hi), nearest even,
// saturating at +-448.
__device__ __forceinline__ uint32_t e4m3x2_from(float lo, float hi) {
  uint16_t c;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(c) : "f"(hi), "f"(lo));
  return c;
}

// Two E4M3 codes (byte 0, byte 1) -> their values (exact).
__device__ __forceinline__ float2 e4m3x2_value(uint32_t c) {
  uint32_t h;
  asm("{\n .reg .b16 t;\n cvt.u16.u32 t, %1;\n cvt.rn.f16x2.e4m3x2 %0, t;\n}" : "=r"(h) : "r"(c));
  return __half22float2(*reinterpret_cast<const __half2 *>(&h));
}

// Three E4M3 parts of each of a and b: a = a1 + a2 / 16 + a3 / 256 + r with
// each part the nearest E4M3 value of the remainder left by the ones before
// (remainders are exact in fp32).  |a|, |b| <= 256.  Returns the codes as
// c[j] = (part j of a) | (part j of b) << 8.
__device__ __forceinline__ void e4m3_split3(float a, float b, uint32_t (&c)[3]) {
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    c[j] = e4m3x2_from(a, b);
    if (j < 2) {
      const float2 v = e4m3x2_value(c[j]);
      a = (a - v.x) * 16.f;
      b = (b - v.y) * 16.f;
    }
  }
}

// Byte `col` (0..127) of row n of an N x 128 B K-major operand, 128-byte swizzled.
__device__ __forceinline__ int sw128_byte(int n, int col) {
  return (n >> 3) * 1024 + (n & 7) * 128 + ((((col >> 4) ^ n) & 7) << 4) + (col & 15);
}

template <typename T, int G>
__global__ void __launch_bounds__(kTcThreads, fp8tc_ctas(G))
    pa_decode_fp8tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                           const DecodeParams p) {
  using SH = Fp8TcShape<G>;
  constexpr int D = 128;
  constexpr int N = SH::N;
  constexpr int NS = SH::kStages;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SH::kBar);
  uint64_t *full = bars;             // [NS] TMA bytes of a tile
  uint64_t *free_ = full + NS;       // [NS] PV of the stage's tile complete
  uint64_t *s_full = free_ + NS;     // [2]  QK complete
  uint64_t *s_free = s_full + 2;     // [2]  S read (4 warps)
  uint64_t *p_full = s_free + 2;     // [2]  P parts written, V tail zeroed (4 warps)
  uint64_t *o_full = p_full + 2;     // [2]  PV complete
  uint64_t *o_free = o_full + 2;     // [2]  O read (4 warps)
  uint64_t *red = o_free + 2;        // [2]  tile maxima exchanged (4 warps)
  uint64_t *q_ready = red + 2;       // q parts written (4 warps)
  uint64_t *drain = q_ready + 1;     // the issuer's last operations complete
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + SH::kTmemSlot);
  volatile int *abort_s = reinterpret_cast<int *>(smem + SH::kFlag);
  float *red_s = reinterpret_cast<float *>(smem + SH::kRed);     // [2][4][G]
  float *lsum_s = reinterpret_cast<float *>(smem + SH::kLsum);   // [4][G]
  float *qmax_s = reinterpret_cast<float *>(smem + SH::kQmax);   // [4][G]

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const unsigned long long wait_limit = wait_limit_for(p.stall_cta, blockIdx.x);
  const bool stall_here = p.stall_cta != 0 && static_cast<int>(blockIdx.x) == p.stall_cta - 1;
  pdl_wait();      // the previous kernel's writes (caches, inputs) are visible from here on
  pdl_trigger();   // the reduce kernel may be scheduled once every CTA of this grid has started

  // ---- work item: blockIdx.x = ((b * Hkv) + g) * NPmax + part (as pa_decode_partition_kernel)
  int item = blockIdx.x;
  const int part = item % p.max_partitions;
  item /= p.max_partitions;
  const int g = item % p.num_kv_heads;
  const int b = item / p.num_kv_heads;
  const int L = p.context_lens[b];
  if (L < 0 || L > p.max_context_len || L > p.max_blocks_per_seq * kBlockSize) {
    if (part == 0 && g == 0 && tid == 0) record_error(4 /*PA_DEV_BAD_CONTEXT_LEN*/, b);
    return;
  }
  const int P = p.partition_size;
  const int nparts = (L + P - 1) / P;
  const int h0 = g * G;
  T *out = reinterpret_cast<T *>(p.out) + (static_cast<size_t>(b) * p.num_heads + h0) * D;
  if (L == 0) {   // empty context: the row is the empty sum, zeros
    if (part == 0)
      for (int i = tid; i < G * D; i += kTcThreads) Elem<T>::store1(out + i, 0.f);
    return;
  }
  if (part >= nparts) return;
  const int tok0 = part * P;
  const int tok1 = min(tok0 + P, L);
  const int nblk = (tok1 - tok0 + kBlockSize - 1) / kBlockSize;
  const int nt = (tok1 - tok0 + kTcTok - 1) / kTcTok;   // >= 1
  const int32_t *bt_row = p.block_tables + static_cast<size_t>(b) * p.max_blocks_per_seq + tok0 / kBlockSize;

  if (tid == 0) {
    prefetch_tensor_map(&tm_k);
    prefetch_tensor_map(&tm_v);
    for (int i = 0; i < NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&free_[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
      mbar_init(&p_full[i], 4);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_free[i], 4);
      mbar_init(&red[i], 4);
    }
    mbar_init(q_ready, 4);
    mbar_init(drain, 1);
    fence_mbar_init();
    *abort_s = 0;
  }
  if (warp == kTcMmaWarp) {
    tmem_alloc(tmem_slot, SH::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();   // barriers initialised, tensor memory allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  int last_issued[NS];   // TMA warp: last tile issued into each stage (for the abort drain)
#pragma unroll
  for (int i = 0; i < NS; ++i) last_issued[i] = -1;
  float o_acc[G], l_acc[G], m_run[G];   // softmax warps: row d = tid of each head's O, this token's sums, maxima

  if (warp == kTcLoadWarp) {
    // ================================================================ TMA producer
    const uint64_t policy = policy_evict_first();
    int grp = -1, my_id = 0;   // lane l holds the id of local block 32 * grp + l
    for (int i = 0; i < nt; ++i) {
      const int st = i % NS;
      if (i >= NS && !__all_sync(kFullMask, mbar_wait_or_abort(&free_[st], (i / NS - 1) & 1, abort_s, wait_limit, true)))
        break;
      if (((kTcBlocks * i) >> 5) != grp) {
        grp = (kTcBlocks * i) >> 5;
        const int lb = (grp << 5) + lane;
        my_id = static_cast<int>(p.num_blocks);   // past the end of the pool: the box reads zeros
        if (lb < nblk) {
          const int v = bt_row[lb];
          if (v < 0 || v >= p.num_blocks) record_error(1 /*PA_DEV_BAD_BLOCK_ID*/, v);
          else my_id = v;
        }
      }
      int ids[kTcBlocks];
#pragma unroll
      for (int k = 0; k < kTcBlocks; ++k) ids[k] = __shfl_sync(kFullMask, my_id, (kTcBlocks * i + k) & 31);
      const bool skip = stall_here && i == 0;   // test hook: tile 0 left unissued
      if (lane == 0 && !skip) {
        uint8_t *dst = smem + st * SH::kStage;
        mbar_arrive_expect_tx(&full[st], SH::kStage);
#pragma unroll
        for (int k = 0; k < kTcBlocks; ++k) {
          tma_load_5d(dst + k * (kBlockSize * 128), &tm_k, 0, 0, g, 0, ids[k], &full[st], policy);
          tma_load_5d(dst + kTcTileBytes + k * (kBlockSize * 128), &tm_v, 0, 0, g, 0, ids[k], &full[st], policy);
        }
      }
      if (!skip) last_issued[st] = i;
    }
  } else if (warp == kTcMmaWarp) {
    // ================================================================ tensor-core issue
    if (lane == 0) {
      constexpr uint32_t kIdescQK = instr_desc_e4m3(false, false, kTcTok, N);   // A = K tile, B = q parts
      constexpr uint32_t kIdescPV = instr_desc_e4m3(true, false, D, N);        // A = V tile (MN-major), B = P parts
      bool ok = true;
      auto wait = [&](uint64_t *bar, uint32_t parity) {
        if (!ok) return;
        ok = mbar_test_wait(bar, parity) || mbar_wait_or_abort(bar, parity, abort_s, wait_limit);
        if (!ok) {
          record_error(5 /*PA_DEV_WAIT_TIMEOUT*/, blockIdx.x);
          *abort_s = 1;
        }
        tc_fence_after();
      };
      // descriptors: an operand at byte offset `off` from a base has the base's
      // descriptor plus off / 16 in the start-address field
      const uint64_t tiles = smem_desc_sw128(smem, 16, 1024);                    // K (K-major) and V (MN-major)
      const uint64_t qd = smem_desc_sw128(smem + SH::kQp, 16, 1024);
      const uint64_t pd = smem_desc_sw128(smem + SH::kPp, 16, 1024);
      auto issue_qk = [&](int i) {
        const int st = i % NS;
        wait(&full[st], (i / NS) & 1);
        if (i >= 2) wait(&s_free[i & 1], ((i - 2) >> 1) & 1);   // S(i-2) read: buffer i&1 free
        if (!ok) return;
        const uint32_t d_tmem = tmem + (i & 1) * N;
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk)
          umma_f8(d_tmem, tiles + ((st * SH::kStage + kk * 32) >> 4), qd + ((kk * 32) >> 4), kIdescQK, kk > 0);
        umma_commit(&s_full[i & 1]);
      };
      auto issue_pv = [&](int i) {
        const int st = i % NS;
        wait(&p_full[i & 1], (i >> 1) & 1);                     // P(i) written, V(i) tail zeroed
        if (i >= 2) wait(&o_free[i & 1], ((i - 2) >> 1) & 1);   // O(i-2) read: buffer i&1 free
        if (!ok) return;
        const uint32_t d_tmem = tmem + 2 * N + (i & 1) * N;
#pragma unroll
        for (int kk = 0; kk < kTcTok / 32; ++kk)   // 32 tokens = four 8-row groups of the V tile
          umma_f8(d_tmem, tiles + ((st * SH::kStage + kTcTileBytes + kk * 4096) >> 4),
                  pd + (((i & 1) * N * 128 + kk * 32) >> 4), kIdescPV, kk > 0);
        umma_commit(&o_full[i & 1]);
        umma_commit(&free_[st]);   // the stage's K and V are consumed once these complete
      };
      wait(q_ready, 0);
      issue_qk(0);
      for (int i = 0; i < nt && ok; ++i) {
        // QK(i+1) goes first when its operands are there, so that its scores
        // are ready when the softmax finishes tile i; otherwise PV(i) is not
        // held back behind the copy of tile i+1 (PV(i) frees tile i's stage
        // for the copy of tile i+NS)
        const bool qk_first = i + 1 < nt && mbar_test_wait(&full[(i + 1) % NS], ((i + 1) / NS) & 1) &&
                              (i + 1 < 2 || mbar_test_wait(&s_free[(i + 1) & 1], ((i - 1) >> 1) & 1));
        if (qk_first) issue_qk(i + 1);
        if (!ok) break;
        issue_pv(i);
        if (!ok) break;
        if (!qk_first && i + 1 < nt) issue_qk(i + 1);
      }
    }
  } else {
    // ================================================================ softmax and epilogue (warps 0-3)
    const int t = tid;   // tensor-memory lane: token t of a tile, then output element d = t
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    bool ok = true;
    auto wait = [&](uint64_t *bar, uint32_t parity) {
      if (!ok) return;
      ok = __all_sync(kFullMask, mbar_wait_or_abort(bar, parity, abort_s, wait_limit));
      if (!ok && lane == 0) {
        record_error(5 /*PA_DEV_WAIT_TIMEOUT*/, blockIdx.x);
        *abort_s = 1;
      }
      tc_fence_after();
    };

    // -- q parts: x = q 2^e (max |x| in [128, 256)) -> rows 3h + j of the B operand of QK
    const T *qg = reinterpret_cast<const T *>(p.q) + (static_cast<size_t>(b) * p.num_heads + h0) * D;
    float qv[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      qv[h] = Elem<T>::load(qg + h * D + t);
      const float mx = warp_max(fabsf(qv[h]));
      if (lane == 0) qmax_s[warp * G + h] = mx;
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");   // the four warps' maxima
    float c_h[G];   // score of head h = (S1 + S2 / 16 + S3 / 256) * c_h, base 2
    uint8_t *qp = smem + SH::kQp;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float mx = fmaxf(fmaxf(qmax_s[h], qmax_s[G + h]), fmaxf(qmax_s[2 * G + h], qmax_s[3 * G + h]));
      const int e = mx > 0.f ? 7 - ilogbf(mx) : 0;
      c_h[h] = ldexpf(p.scale_log2, -e);
      qv[h] = ldexpf(qv[h], e);
      m_run[h] = -INFINITY;
      l_acc[h] = 0.f;
      o_acc[h] = 0.f;
    }
#pragma unroll
    for (int h = 0; h < G; h += 2) {
      uint32_t c[3];
      e4m3_split3(qv[h], h + 1 < G ? qv[h + 1] : 0.f, c);
#pragma unroll
      for (int j = 0; j < 3; ++j) {
        qp[sw128_byte(3 * h + j, t)] = static_cast<uint8_t>(c[j] & 0xFF);
        if (h + 1 < G) qp[sw128_byte(3 * (h + 1) + j, t)] = static_cast<uint8_t>(c[j] >> 8);
      }
    }
    // padding rows of the q parts and of both P buffers: zero
#pragma unroll
    for (int n = SH::kCols; n < N; ++n) {
      qp[sw128_byte(n, t)] = 0;
      smem[SH::kPp + sw128_byte(n, t)] = 0;
      smem[SH::kPp + N * 128 + sw128_byte(n, t)] = 0;
    }
    fence_proxy_async_smem();   // generic stores read by the tensor cores
    __syncwarp();
    if (lane == 0) mbar_arrive(q_ready);

    float alpha_prev[G];
#pragma unroll
    for (int h = 0; h < G; ++h) alpha_prev[h] = 0.f;
    // O(j) of row d = t folded in: o = o * alpha(j) + O(j)  (O(j) relative to tile j's max)
    auto epilogue = [&](int j) {
      wait(&o_full[j & 1], (j >> 1) & 1);
      if (!ok) return;
      float ov[N];
      if constexpr (N == 16) tmem_ld16(t_lane + 2 * N + (j & 1) * N, ov);
      else tmem_ld32(t_lane + 2 * N + (j & 1) * N, ov);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_free[j & 1]);
#pragma unroll
      for (int h = 0; h < G; ++h)
        o_acc[h] = fmaf(o_acc[h], alpha_prev[h], ov[3 * h] + ov[3 * h + 1] * 0.0625f + ov[3 * h + 2] * 0.00390625f);
    };

    for (int i = 0; i < nt && ok; ++i) {
      wait(&s_full[i & 1], (i >> 1) & 1);
      if (!ok) break;
      float sv[N];
      if constexpr (N == 16) tmem_ld16(t_lane + (i & 1) * N, sv);
      else tmem_ld32(t_lane + (i & 1) * N, sv);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[i & 1]);

      const bool valid = tok0 + i * kTcTok + t < tok1;
      float x[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        x[h] = valid ? (sv[3 * h] + sv[3 * h + 1] * 0.0625f + sv[3 * h + 2] * 0.00390625f) * c_h[h] : -INFINITY;
        const float wm = warp_max(x[h]);
        if (lane == 0) red_s[((i & 1) * 4 + warp) * G + h] = wm;
      }
      if (lane == 0) mbar_arrive(&red[i & 1]);
      wait(&red[i & 1], (i >> 1) & 1);
      if (!ok) break;
      float pv[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float *r = red_s + (i & 1) * 4 * G + h;
        const float mt = fmaxf(fmaxf(r[0], r[G]), fmaxf(r[2 * G], r[3 * G]));   // finite: token 0 of a tile is valid
        const float mn = fmaxf(m_run[h], mt);
        const float alpha = ex2(m_run[h] - mn);   // 0 on the first tile
        m_run[h] = mn;
        pv[h] = ex2(x[h] - mn);                   // 0 for tokens past the end
        l_acc[h] = fmaf(l_acc[h], alpha, pv[h]);
        x[h] = alpha;                             // kept for this tile's epilogue
      }
      // P(i) parts -> buffer i&1 (PV(i-2), its last reader, completed before
      // the epilogue of tile i-2, which this thread has run)
      uint8_t *pp = smem + SH::kPp + (i & 1) * N * 128;
#pragma unroll
      for (int h = 0; h < G; h += 2) {
        uint32_t c[3];
        e4m3_split3(pv[h] * 256.f, h + 1 < G ? pv[h + 1] * 256.f : 0.f, c);
#pragma unroll
        for (int j = 0; j < 3; ++j) {
          pp[sw128_byte(3 * h + j, t)] = static_cast<uint8_t>(c[j] & 0xFF);
          if (h + 1 < G) pp[sw128_byte(3 * (h + 1) + j, t)] = static_cast<uint8_t>(c[j] >> 8);
        }
      }
      if (tok0 + (i + 1) * kTcTok > tok1) {
        // the last tile: a token past the end has a V row that may hold anything
        // (NaN codes too) and 0 * V must stay 0.  Its copy has landed (QK(i)
        // waited for the stage); the wait orders this thread's stores after it.
        wait(&full[i % NS], (i / NS) & 1);
        if (!ok) break;
      }
      if (!valid) {
        uint4 *row = reinterpret_cast<uint4 *>(smem + (i % NS) * SH::kStage + kTcTileBytes +
                                               (t / kBlockSize) * (kBlockSize * 128) + (t % kBlockSize) * 128);
#pragma unroll
        for (int c = 0; c < 8; ++c) row[c] = make_uint4(0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[i & 1]);
      if (i > 0) epilogue(i - 1);
#pragma unroll
      for (int h = 0; h < G; ++h) alpha_prev[h] = x[h];
    }
    if (ok) epilogue(nt - 1);
    // this warp's share of each head's sum
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float l = l_acc[h];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(kFullMask, l, off);
      if (lane == 0) lsum_s[warp * G + h] = l;
    }
    tc_fence_before();
  }

  // ---- all roles done.  Every tensor-core operation, and every barrier arrival
  // that a commit makes, lands before the memory is released; after an abort
  // the copies in flight are let finish too (all bounded).
  __syncthreads();
  if (warp == kTcMmaWarp && lane == 0) {
    umma_commit(drain);
    mbar_wait(drain, 0, wait_limit);
  }
  if (*abort_s && warp == kTcLoadWarp && lane == 0) {
    for (int i = 0; i < NS; ++i)
      if (last_issued[i] >= 0) mbar_wait(&full[i], (last_issued[i] / NS) & 1, wait_limit);
  }
  __syncthreads();
  if (warp == kTcMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, SH::kTmemCols);
  }
  if (*abort_s || warp >= 4) return;

  // ---- output: row d = tid of each head; v_scale and the 2^-8 of P's parts applied here
  const int d = tid;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float l = (lsum_s[h] + lsum_s[G + h]) + (lsum_s[2 * G + h] + lsum_s[3 * G + h]);
    const float o = o_acc[h] * (p.v_scale * 0.00390625f);
    if (nparts == 1) {
      Elem<T>::store1(out + h * D + d, o / l);
    } else {
      const size_t row = (static_cast<size_t>(b) * p.num_heads + h0 + h) * p.max_partitions + part;
      p.ws_o[row * D + d] = o;
      if (d == 0) {
        p.ws_m[row] = m_run[h];
        p.ws_l[row] = l;
      }
    }
  }
}

}  // namespace pa
