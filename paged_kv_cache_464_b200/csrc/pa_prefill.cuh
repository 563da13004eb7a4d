// pa_prefill.cuh -- paged chunked-prefill attention on the 5th-generation
// tensor cores (tcgen05, accumulators in tensor memory).
//
// What it computes: the engine of "vLLM推理引擎深度实战：…" runs prompts in
// chunks (§5.3 推理优化配置 and §7.1 性能调优指南: enable_chunked_prefill);
// each new token's attention is the formula of "vLLM推理引擎深度解析：从
// PagedAttention原理到高吞吐量部署的工程实践" §五 (PagedAttention.forward) with
// the context cut at that token.  Sequence b holds L_b tokens in the paged
// cache, the last n_b of which are this step's chunk.  Query i of the chunk
// sits at position pos = L_b - n_b + i and attends, causally, to the cached
// tokens 0..pos of its KV head, read through the block table exactly like
// decode:
//   out[i, h] = sum_{t <= pos} softmax_t(scale * q[i, h] . K_t) V_t.
// A decode step is the chunk of one token.
//
// Work decomposition.  One CTA per (sequence, KV head, pair of query tiles).
// A query tile is 128 rows: the G query heads of each of 128 / G chunk queries
// (row = query * G + head), so every K/V tile read from the cache serves all
// grouped heads, and the two query tiles of a CTA share every K/V tile.  The
// KV walk runs over tiles of 64 tokens (four cache blocks) up to the last
// query's position.  Warp roles (512 threads):
//   warps 0-3, 4-7  one softmax warpgroup per query tile; thread = row.  Per KV
//                   tile: tcgen05.ld of its 64 scores, causal mask on diagonal
//                   tiles, online max/sum in base 2 (O rescaled in tensor
//                   memory only when a row's max grows by more than 2^8), P
//                   written back over its scores in tensor memory as fp16
//                   (relative rounding <= 2^-11); after the last tile, O / l
//                   staged through the tile's Q buffer (free once its last QK
//                   has completed) and copied out with coalesced 16-byte
//                   stores (a warp store covers two whole output rows instead
//                   of one 16-byte piece of 32 rows);
//   warps 8, 10     tensor-core issue, one thread per query tile: S = Q K^T
//                   (M=128 N=64, 8 x K=16, both operands in shared memory)
//                   into a double-buffered S, and O += P V (M=128 N=128,
//                   4 x K=16, fp16, P read from tensor memory, V from shared
//                   memory), QK(j+1) before PV(j); the tensor pipe runs one
//                   query tile's products while the other's issuer waits.  A
//                   product costs about the same below N=256 whatever its
//                   width (56-64 cycles at N=64 and at N=128, 128 at N=256);
//                   one fp16 pass of P V instead of two bf16 ones (hi + lo)
//                   takes a quarter of them away.  The pipe is busy about
//                   half of each step: the step is set by each query tile's
//                   chain through its two S buffers, QK(j+2) after PV(j)
//                   after softmax(j), and by the hand-overs;
//   warp 9          TMA: K and V tiles (four 2 KiB boxes per 128-byte half of
//                   the rows, 128-byte swizzled) into rings of 3 stages each,
//                   block ids read from the block table one per lane;
//   warps 12-15     bf16 caches: rewrite each landed V tile in place as fp16
//                   times 2^-8 (exact for 2^-6 <= |v| < 2^24, within 2^-17
//                   below) and zero the rows past the context end, then hand
//                   it to the issuers; f16 caches: idle (as are warp 11 and
//                   lanes 1-31 of warps 8 and 10).
// Before the barrier set-up the softmax warps already load their Q rows and the
// TMA warp its first 32 block ids, so that those loads overlap the set-up.
// Roles hand over through mbarriers (one arrival per warp) only; every wait is
// bounded, and a role that gives up raises a CTA-wide abort so that the others
// stop waiting.  Each barrier is waited on by parity, so no barrier may complete
// a phase twice before its waiter has seen the first: S and P hand-overs are
// double-buffered by tile parity (writing P(j+2) needs S(j+2), issued only
// after PV(j) has taken P(j)), and so is the PV-done hand-over (a waiter on
// PV(j) has seen S(j+1), which needed PV(j-2) done); the K/V ring barriers
// advance one phase per hand-over that their waiter itself enables.
// Tensor memory: per query tile, S[2] (2 x 64 columns; P of a tile replaces
// the first 32 columns of its S as fp16 pairs) and O (128 columns).
#pragma once

#include "pa_common.cuh"
#include "pa_tcgen05.cuh"

namespace pa {

struct PrefillParams {
  void *out;                          // [T][Hq][128]
  const void *q;                      // [T][Hq][128]
  const int32_t *block_tables;        // [S][MBS]
  const int32_t *context_lens;        // [S]   tokens in the cache, chunk included
  const int32_t *query_start_loc;     // [S+1] the chunk of sequence b is rows qsl[b] .. qsl[b+1]-1
  long long num_blocks;
  int num_seqs, num_heads, num_kv_heads, max_blocks_per_seq, max_query_len;
  float scale_log2;                   // scale * log2(e), > 0
  int stall_cta;                      // test hook (pa_common.cuh): 0 in every ordinary launch
};

constexpr int kPrefillRows = 128;        // M: rows of one query tile
constexpr int kPrefillTiles = 2;         // query tiles (softmax warpgroups) per CTA
constexpr int kPrefillMmaWarp = 4 * kPrefillTiles;
constexpr int kPrefillLoadWarp = kPrefillMmaWarp + 1;
constexpr int kPrefillConvWarp = 4 * (kPrefillTiles + 1);   // first of the four V converter warps
constexpr int kPrefillConvWarps = 4;
// four whole warpgroups: two softmax, one for the issuers and the TMA warp
// (warp 11 idle), one converting bf16 V tiles (idle for f16 caches)
constexpr int kPrefillThreads = 128 * (kPrefillTiles + 2);
constexpr int kPrefillKv = 64;           // N of S = Q K^T: tokens per KV tile
constexpr int kPrefillKStages = 3;
constexpr int kPrefillVStages = 3;
constexpr int kPrefillTmemCols = 512;    // per query tile: S/P double buffer (2 x 64) + O (128)
constexpr float kRescaleLog2 = 8.f;      // rescale O once a row's max grows by more than this (base-2 units)

struct PrefillSmem {
  static constexpr int kQTileBytes = 2 * kPrefillRows * 128;  // [2 halves][128 rows][128 B]
  static constexpr int kKvTileBytes = 2 * kPrefillKv * 128;   // [2 halves][64 tokens][128 B]
  static constexpr int kHalfBytes = kPrefillKv * 128;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kPrefillTiles * kQTileBytes;
  static constexpr int kV = kK + kPrefillKStages * kKvTileBytes;
  static constexpr int kBar = kV + kPrefillVStages * kKvTileBytes;
  // k_full[KS] v_full[VS] k_free[KS] v_free[VS]; per query tile: s_full[2] p_full[2] o_done[2]; drain,
  // tail_ready; v_conv[VS]
  static constexpr int kTileBars = 6;
  static constexpr int kNumBars = 2 * (kPrefillKStages + kPrefillVStages) + kPrefillTiles * kTileBars + 2 + kPrefillVStages;
  static constexpr int kTmemSlot = kBar + 8 * kNumBars;
  static constexpr int kFlag = kTmemSlot + 4;
  static constexpr int kBytes = kFlag + 4;
  static constexpr int kAlloc = kBytes + 1024;   // + alignment of the base to 1024 B (swizzle atoms)
};
static_assert(PrefillSmem::kAlloc <= 227 * 1024, "prefill shared memory exceeds the per-CTA limit");

template <typename T>
struct Pack16;
template <>
struct Pack16<__nv_bfloat16> {
  static constexpr int kFormat = 1;       // tcgen05 kind::f16 operand format of q and K
  static constexpr bool kConvertV = true; // V tiles rewritten as fp16 (times 2^-8) before PV
  __device__ __forceinline__ static uint32_t pack(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
  }
};
template <>
struct Pack16<__half> {
  static constexpr int kFormat = 0;
  static constexpr bool kConvertV = false; // V is fp16 already
  __device__ __forceinline__ static uint32_t pack(float a, float b) {
    __half2 v = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
  }
};

// Two softmax weights -> one fp16 pair (the A operand of P V), the first in the
// low half; relative rounding <= 2^-11.
__device__ __forceinline__ uint32_t pack_p(float2 e) {
  __half2 v = __floats2half2_rn(e.x, e.y);
  return *reinterpret_cast<uint32_t *>(&v);
}

// 64 consecutive fp32 columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&v)[64]) {
  uint32_t r[64];
#define PA_LD32(OFF)                                                                                              \
  asm volatile(                                                                                                   \
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, " \
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"              \
      : "=r"(r[OFF + 0]), "=r"(r[OFF + 1]), "=r"(r[OFF + 2]), "=r"(r[OFF + 3]), "=r"(r[OFF + 4]),                 \
        "=r"(r[OFF + 5]), "=r"(r[OFF + 6]), "=r"(r[OFF + 7]), "=r"(r[OFF + 8]), "=r"(r[OFF + 9]),                 \
        "=r"(r[OFF + 10]), "=r"(r[OFF + 11]), "=r"(r[OFF + 12]), "=r"(r[OFF + 13]), "=r"(r[OFF + 14]),            \
        "=r"(r[OFF + 15]), "=r"(r[OFF + 16]), "=r"(r[OFF + 17]), "=r"(r[OFF + 18]), "=r"(r[OFF + 19]),            \
        "=r"(r[OFF + 20]), "=r"(r[OFF + 21]), "=r"(r[OFF + 22]), "=r"(r[OFF + 23]), "=r"(r[OFF + 24]),            \
        "=r"(r[OFF + 25]), "=r"(r[OFF + 26]), "=r"(r[OFF + 27]), "=r"(r[OFF + 28]), "=r"(r[OFF + 29]),            \
        "=r"(r[OFF + 30]), "=r"(r[OFF + 31])                                                                      \
      : "r"(taddr + OFF)                                                                                          \
      : "memory")
  PA_LD32(0);
  PA_LD32(32);
#undef PA_LD32
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
}

// AND of `pred` over the 128 threads of one softmax warpgroup (named barrier kId).
template <int kId>
__device__ __forceinline__ bool warpgroup_all(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred p, %2, 128, p;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "n"(kId)
      : "memory");
  return r != 0;
}

template <typename T, int G>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    pa_prefill_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const PrefillParams p) {
  using SM = PrefillSmem;
  using PK = Pack16<T>;
  constexpr int D = 128;
  constexpr int QT = kPrefillRows / G;   // chunk queries per query tile
  constexpr int KS = kPrefillKStages;
  constexpr int VS = kPrefillVStages;
  constexpr int NT = kPrefillTiles;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::kBar);
  uint64_t *k_full = bars;
  uint64_t *v_full = k_full + KS;
  uint64_t *k_free = v_full + VS;
  uint64_t *v_free = k_free + KS;
  uint64_t *tile_bars = v_free + VS;   // query tile w: s_full[2], p_full[2], o_done[2] at w * kTileBars
  uint64_t *drain = tile_bars + NT * SM::kTileBars;
  uint64_t *tail_ready = drain + 1;
  uint64_t *v_conv = tail_ready + 1;   // [VS] bf16 caches: V tile rewritten as fp16
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + SM::kTmemSlot);
  volatile int *abort_s = reinterpret_cast<int *>(smem + SM::kFlag);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  // linear CTA index: reported with PA_DEV_WAIT_TIMEOUT, and the test hook's key
  const long long cta = blockIdx.x + static_cast<long long>(gridDim.x) * (blockIdx.y + static_cast<long long>(gridDim.y) * blockIdx.z);
  const unsigned long long wait_limit = wait_limit_for(p.stall_cta, cta);
  const bool stall_here = p.stall_cta != 0 && cta == p.stall_cta - 1;
  if (warp == kPrefillLoadWarp && lane == 0) {   // kernel parameters: independent of the previous grid
    prefetch_tensor_map(&tm_k);
    prefetch_tensor_map(&tm_v);
  }
  pdl_wait();
  pdl_trigger();

  // ---- work item; the longest query tiles are launched first
  const int ct = gridDim.x - 1 - blockIdx.x;
  const int g = blockIdx.y;
  const int b = blockIdx.z;
  const int L = p.context_lens[b];
  const int qs = p.query_start_loc[b];
  const int n = p.query_start_loc[b + 1] - qs;
  if (n < 0 || n > p.max_query_len || L < n || L > p.max_blocks_per_seq * kBlockSize) {
    if (ct == 0 && g == 0 && tid == 0) record_error(4 /*PA_DEV_BAD_CONTEXT_LEN*/, b);
    return;
  }
  if (ct * NT * QT >= n) return;
  // query tile w: queries q0(w) .. q0(w) + nq(w) - 1 of the chunk, KV tiles 0 .. nt(w) - 1
  int nt[NT];
  int pos_last_all = 0;
#pragma unroll
  for (int w = 0; w < NT; ++w) {
    const int q0 = (ct * NT + w) * QT;
    const int nq = max(0, min(QT, n - q0));
    const int pos_last = L - n + q0 + nq - 1;
    nt[w] = nq > 0 ? pos_last / kPrefillKv + 1 : 0;
    if (nq > 0) pos_last_all = pos_last;
  }
  const int ntiles = nt[NT - 1] > 0 ? nt[NT - 1] : nt[0];   // later tiles reach further
  const int nblk = pos_last_all / kBlockSize + 1;          // cache blocks covering tokens 0 .. pos_last_all
  const int32_t *bt_row = p.block_tables + static_cast<size_t>(b) * p.max_blocks_per_seq;

  // ---- started before the barrier set-up: the Q rows' loads (softmax
  // warps) and the first 32 block ids (TMA warp)
  uint4 qx[16];
  int tma_grp = -1, tma_id = 0;
  if (warp < kPrefillMmaWarp) {
    const int w = warp >> 2;
    const int q0 = (ct * NT + w) * QT;
    const int nq = max(0, min(QT, n - q0));
    const T *qg = reinterpret_cast<const T *>(p.q);
    const int c = tid & 15;              // this thread's 16-byte chunk of every row it moves
    const int row0 = (tid & 127) >> 4;   // rows row0, row0 + 8, ...
#pragma unroll
    for (int k = 0; k < 16; ++k) {   // every load in flight before the first store
      const int row = row0 + 8 * k;
      const int i = row / G, hl = row % G;
      qx[k] = make_uint4(0u, 0u, 0u, 0u);
      if (i < nq)
        qx[k] = *reinterpret_cast<const uint4 *>(
            qg + (static_cast<size_t>(qs + q0 + i) * p.num_heads + g * G + hl) * D + c * 8);
    }
  } else if (warp == kPrefillLoadWarp) {
    tma_grp = 0;
    tma_id = static_cast<int>(p.num_blocks);   // past the end of the pool: the box reads zeros
    if (lane < nblk) {
      const int v = bt_row[lane];
      if (v < 0 || v >= p.num_blocks) record_error(1 /*PA_DEV_BAD_BLOCK_ID*/, v);
      else tma_id = v;
    }
  }
  if (tid == 0) {
    for (int i = 0; i < KS; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_free[i], NT);   // one arrival per issuing thread
    }
    for (int i = 0; i < VS; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_free[i], NT);
    }
    for (int w = 0; w < NT; ++w) {
      uint64_t *tb = tile_bars + w * SM::kTileBars;
      mbar_init(&tb[0], 1);               // s_full[0], s_full[1]: tensor-core commit
      mbar_init(&tb[1], 1);
      mbar_init(&tb[2], 4);               // p_full[0], p_full[1]: every softmax warp
      mbar_init(&tb[3], 4);
      mbar_init(&tb[4], 1);               // o_done[0], o_done[1]: tensor-core commit
      mbar_init(&tb[5], 1);
    }
    mbar_init(drain, NT);
    mbar_init(tail_ready, 1);
    for (int i = 0; i < VS; ++i) mbar_init(&v_conv[i], kPrefillConvWarps);   // one arrival per converter warp
    fence_mbar_init();
    *abort_s = 0;
  }
  if (warp == kPrefillMmaWarp) {
    tmem_alloc(tmem_slot, kPrefillTmemCols);
    tmem_relinquish();
  }

  tc_fence_before();
  __syncthreads();   // barriers initialised, tensor memory allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // ---- Q tiles -> shared memory (rows loaded above), K-major 128-byte swizzled:
  // [d half][row][128 B].  The TMA warp streams K/V meanwhile; only the issuing
  // warps wait for Q (named barrier 1: the softmax warpgroups and warps 8 and 10).
  if (warp < kPrefillMmaWarp) {
    const int w = warp >> 2;
    uint8_t *q_s = smem + SM::kQ + w * SM::kQTileBytes;
    const int c = tid & 15;
    const int row0 = (tid & 127) >> 4;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const int row = row0 + 8 * k;
      *reinterpret_cast<uint4 *>(q_s + (c >> 3) * (kPrefillRows * 128) + row * 128 + (((c & 7) ^ (row & 7)) << 4)) =
          qx[k];
    }
    fence_proxy_async_smem();   // the generic stores of Q are read by the tensor cores
  }
  if (warp < kPrefillMmaWarp || warp == kPrefillMmaWarp || warp == kPrefillMmaWarp + 2)
    asm volatile("bar.sync 1, %0;" ::"n"(128 * kPrefillTiles + 64) : "memory");

  int last_k[KS], last_v[VS];   // TMA warp: last tile issued into each stage (for the abort drain)
#pragma unroll
  for (int i = 0; i < KS; ++i) last_k[i] = -1;
#pragma unroll
  for (int i = 0; i < VS; ++i) last_v[i] = -1;

  if (warp == kPrefillLoadWarp) {
    // ================================================================ TMA producer
    int grp = tma_grp, my_id = tma_id;
    auto issue = [&](int j, bool is_v) {   // all lanes; j uniform
      const int want = (4 * j) >> 5;
      if (want != grp) {
        grp = want;
        const int lb = (grp << 5) + lane;
        my_id = static_cast<int>(p.num_blocks);   // past the end of the pool: the box reads zeros
        if (lb < nblk) {
          const int v = bt_row[lb];
          if (v < 0 || v >= p.num_blocks) record_error(1 /*PA_DEV_BAD_BLOCK_ID*/, v);
          else my_id = v;
        }
      }
      int ids[4];
#pragma unroll
      for (int bi = 0; bi < 4; ++bi) ids[bi] = __shfl_sync(kFullMask, my_id, (4 * j + bi) & 31);
      const bool skip = stall_here && j == 0 && !is_v;   // test hook: K tile 0 left unissued
      if (lane == 0 && !skip) {
        const int st = j % (is_v ? VS : KS);
        uint8_t *dst = smem + (is_v ? SM::kV : SM::kK) + st * SM::kKvTileBytes;
        uint64_t *bar = is_v ? &v_full[st] : &k_full[st];
        mbar_arrive_expect_tx(bar, SM::kKvTileBytes);
#pragma unroll
        for (int bi = 0; bi < 4; ++bi)
#pragma unroll
          for (int half = 0; half < 2; ++half)
            tma_load_5d(dst + half * SM::kHalfBytes + bi * (kBlockSize * 128), is_v ? &tm_v : &tm_k, 0, half, g, 0,
                        ids[bi], bar);
      }
      if (is_v) last_v[j % VS] = j;
      else if (!skip) last_k[j % KS] = j;
    };
    for (int j = 0; j < ntiles; ++j) {
      if (j >= KS &&
          !__all_sync(kFullMask, mbar_wait_or_abort(&k_free[j % KS], (j / KS - 1) & 1, abort_s, wait_limit, true)))
        break;
      issue(j, false);
      if (j >= VS &&
          !__all_sync(kFullMask, mbar_wait_or_abort(&v_free[j % VS], (j / VS - 1) & 1, abort_s, wait_limit, true)))
        break;
      issue(j, true);
    }
  } else if ((warp == kPrefillMmaWarp || warp == kPrefillMmaWarp + 2) && lane == 0) {
    // ================================================================ tensor-core issue
    // One thread per query tile w (warps 8 and 10, on different schedulers).
    // The tensor pipe takes products about as fast as it runs them, so while
    // one issuer waits on a hand-over the other keeps the pipe busy.
    const int w = warp == kPrefillMmaWarp ? 0 : 1;
    const int ntw = nt[w];
    uint64_t *tb = tile_bars + w * SM::kTileBars;
    constexpr uint32_t kIdescQK = instr_desc_f16(PK::kFormat, false, kPrefillRows, kPrefillKv);
    constexpr uint32_t kIdescPV = instr_desc_f16(0 /* f16: P, and V after conversion */, true, kPrefillRows, D);
    bool ok = true;
    auto wait = [&](uint64_t *bar, uint32_t parity) {
      if (!ok) return;
      ok = mbar_test_wait(bar, parity) || mbar_wait_or_abort(bar, parity, abort_s, wait_limit);
      if (!ok) {
        record_error(5 /*PA_DEV_WAIT_TIMEOUT*/, cta);
        *abort_s = 1;
      }
      tc_fence_after();
    };
    // the K or V stage of tile t: an issuer with no product on t still arrives
    // once, after the stage's previous phase has completed (so that its
    // arrival counts toward tile t's phase)
    auto free_arrive = [&](uint64_t *ring, int t, int stages) {
      if (t >= stages) wait(&ring[t % stages], (t / stages - 1) & 1);
      if (ok) mbar_arrive(&ring[t % stages]);
    };
    const bool zero_tail = (L & (kBlockSize - 1)) != 0 && (L - 1) / kBlockSize == pos_last_all / kBlockSize;
    const int tail_owner = nt[NT - 1] > 0 ? NT - 1 : 0;   // a query tile that reaches the last KV tile
    // Per KV tile j: QK_w(j+1), then PV_w(j), so that the scores of the next
    // tile are computed while the softmax works on this one.
    //   S_w(j) = Q_w K_j^T goes to the S/P buffer j & 1 of query tile w, which
    //   last held P_w(j-2); PV_w(j-2) reads that as its A operand straight from
    //   tensor memory, and issue order does not keep a later product from
    //   overwriting it, so QK_w(j) waits until PV_w(j-2) has completed.
    // Descriptors are built once: an operand at byte offset `off` from a tile's
    // base has the base's descriptor with off / 16 added to the start-address
    // field (the field does not overflow: shared memory ends below 2^18 bytes).
    const uint64_t a_qk = smem_desc_sw128(smem + SM::kQ + w * SM::kQTileBytes, 16, 1024);
    const uint64_t k_desc = smem_desc_sw128(smem + SM::kK, 16, 1024);
    const uint64_t v_desc = smem_desc_sw128(smem + SM::kV, SM::kHalfBytes, 1024);
    auto issue_qk = [&](int j) {
      wait(&k_full[j % KS], (j / KS) & 1);
      if (j >= 2) wait(&tb[4 + (j & 1)], ((j - 2) >> 1) & 1);   // PV_w(j-2) complete: buffer j&1 free
      if (!ok) return;
      const uint64_t b0 = k_desc + (((j % KS) * SM::kKvTileBytes) >> 4);
      const uint32_t d_tmem = tmem + w * 256 + (j & 1) * kPrefillKv;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        umma_f16(d_tmem, a_qk + (((kk >> 2) * (kPrefillRows * 128) + (kk & 3) * 32) >> 4),
                 b0 + (((kk >> 2) * SM::kHalfBytes + (kk & 3) * 32) >> 4), kIdescQK, kk > 0);
      umma_commit(&tb[j & 1]);              // s_full
      umma_commit(&k_free[j % KS]);         // this issuer is done with the K stage once they complete
    };
    auto issue_pv = [&](int j) {   // O_w += P_w(j) V_j
      if constexpr (PK::kConvertV) wait(&v_conv[j % VS], (j / VS) & 1);   // rewritten as fp16, tail zeroed
      else wait(&v_full[j % VS], (j / VS) & 1);
      if (!ok) return;
      uint8_t *vt = smem + SM::kV + (j % VS) * SM::kKvTileBytes;
      if (!PK::kConvertV && zero_tail && j == ntiles - 1) {
        if (w == tail_owner) {
          // rows past the context end in its last block may hold anything (NaN
          // included); make them zero so that 0 * V stays 0
          const int t0 = j * kPrefillKv;
          const int r0 = L - t0, r1 = ((L + kBlockSize - 1) / kBlockSize) * kBlockSize - t0;
          for (int idx = 0; idx < (r1 - r0) * 16; ++idx) {
            const int r = r0 + (idx >> 4), c = idx & 15;
            *reinterpret_cast<uint4 *>(vt + (c >> 3) * SM::kHalfBytes + r * 128 + (c & 7) * 16) =
                make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
          mbar_arrive(tail_ready);
        } else {
          wait(tail_ready, 0);
          if (!ok) return;
        }
      }
      wait(&tb[2 + (j & 1)], (j >> 1) & 1);   // P_w(j) written
      if (!ok) return;
      const uint64_t b0 = v_desc + (((j % VS) * SM::kKvTileBytes) >> 4);
      const uint32_t a0 = tmem + w * 256 + (j & 1) * kPrefillKv;   // P_w(j): fp16 pairs in 32 columns
      const uint32_t o_tmem = tmem + w * 256 + 128;
      const bool acc = j > 0;
#pragma unroll
      for (int kk = 0; kk < kPrefillKv / 16; ++kk)   // 16 tokens = 8 columns of P per step
        umma_f16_ts(o_tmem, a0 + kk * 8, b0 + ((kk * 16 * 128) >> 4), kIdescPV, acc || kk > 0);
      umma_commit(&tb[4 + (j & 1)]);   // o_done
      umma_commit(&v_free[j % VS]);    // this issuer is done with the V stage once they complete
    };
    if (ntw > 0) issue_qk(0);
    else free_arrive(k_free, 0, KS);
    for (int j = 0; j < ntiles && ok; ++j) {
      if (j + 1 < ntiles) {
        if (j + 1 < ntw) issue_qk(j + 1);
        else free_arrive(k_free, j + 1, KS);
      }
      if (!ok) break;
      if (j < ntw) issue_pv(j);
      else free_arrive(v_free, j, VS);
    }
  } else if (warp >= kPrefillConvWarp) {
    if constexpr (PK::kConvertV) {
      // ================================================================ V converter (bf16 caches)
      // Every landed V tile is rewritten in place as fp16 times 2^-8 (exact for
      // 2^-6 <= |v| < 2^24, within 2^-17 absolute below; |v| >= 2^24 is out of
      // the kernel's stated range and recorded as PA_DEV_VALUE_RANGE), and the rows of tokens at or past the context end
      // (stale slots of the last block, possibly NaN) become zero, so that
      // 0 * V stays 0.  The element positions do not move, so the tile keeps
      // its swizzled layout.  Four warps, 8 16-byte chunks a lane per tile;
      // each warp arrives once on the stage's conversion barrier.
      const int ct = (warp - kPrefillConvWarp) * 32 + lane;   // converter thread 0..127
      bool ok = true;
      for (int j = 0; j < ntiles && ok; ++j) {
        ok = __all_sync(kFullMask, mbar_wait_or_abort(&v_full[j % VS], (j / VS) & 1, abort_s, wait_limit, true));
        if (!ok) {
          if (lane == 0) {
            record_error(5 /*PA_DEV_WAIT_TIMEOUT*/, cta);
            *abort_s = 1;
          }
          break;
        }
        uint4 *vt = reinterpret_cast<uint4 *>(smem + SM::kV + (j % VS) * SM::kKvTileBytes);
        const int valid_rows = L - j * kPrefillKv;   // rows at or past this are past the context end
        float vmax = 0.f;   // max |v| converted (fmaxf skips NaN, which passes through as NaN)
#pragma unroll
        for (int i = 0; i < SM::kKvTileBytes / 16 / 128; ++i) {
          const int c = ct + 128 * i;
          const int row = (c % (SM::kHalfBytes / 16)) >> 3;   // 8 chunks a 128-byte row, [half][row][128 B]
          uint4 x = vt[c];
          if (row >= valid_rows) {
            x = make_uint4(0u, 0u, 0u, 0u);
          } else {
            uint32_t *w = reinterpret_cast<uint32_t *>(&x);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float lo = __uint_as_float(w[k] << 16), hi = __uint_as_float(w[k] & 0xffff0000u);
              vmax = fmaxf(vmax, fmaxf(fabsf(lo), fabsf(hi)));
              w[k] = pack_p(make_float2(lo * 0.00390625f, hi * 0.00390625f));
            }
          }
          vt[c] = x;
        }
        const bool range_bad = vmax >= 16777216.f;   // |v| >= 2^24
        fence_proxy_async_smem();   // generic stores read by the tensor cores
        __syncwarp();
        if (lane == 0) mbar_arrive(&v_conv[j % VS]);
        if (__any_sync(kFullMask, range_bad) && lane == 0) record_error(6 /*PA_DEV_VALUE_RANGE*/, b);
      }
    }
  } else if (warp < kPrefillMmaWarp) {
    // ================================================================ softmax warpgroup w
    const int w = warp >> 2;
    const int r = tid & 127;             // row = tensor-memory lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t t_s = tmem + w * 256 + lane_base;
    const uint32_t t_o = t_s + 128;
    uint64_t *tb = tile_bars + w * SM::kTileBars;
    const int q0 = (ct * NT + w) * QT;
    const int nq = max(0, min(QT, n - q0));
    const int i_row = r / G;
    const int pos_first = L - n + q0;
    const int pos_r = pos_first + min(i_row, nq - 1);   // padding rows repeat the last query (never stored)
    const float c2 = p.scale_log2;
    const int ntw = nt[w];

    float m_run = -INFINITY;   // running max of this row's raw scores
    float l_run = 0.f;         // running sum of 2^((s - m_run) * c2)
    bool ok = true;
    auto wait = [&](uint64_t *bar, uint32_t parity) {
      if (!ok) return;
      ok = __all_sync(kFullMask, mbar_wait_or_abort(bar, parity, abort_s, wait_limit, true));
      if (!ok && lane == 0) {
        record_error(5 /*PA_DEV_WAIT_TIMEOUT*/, cta);
        *abort_s = 1;
      }
      tc_fence_after();
    };
    for (int j = 0; j < ntw && ok; ++j) {
      wait(&tb[j & 1], (j >> 1) & 1);
      if (!ok) break;
      float s[64];
      tmem_ld64(t_s + (j & 1) * kPrefillKv, s);
      const int t0 = j * kPrefillKv;
      if (t0 + kPrefillKv - 1 > pos_first) {   // a diagonal tile: mask tokens after each row's position
#pragma unroll
        for (int c = 0; c < 64; ++c) s[c] = (t0 + c <= pos_r) ? s[c] : -INFINITY;
      }
      float mx[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx[k] = fmaxf(fmaxf(fmaxf(s[8 * k], s[8 * k + 1]), fmaxf(s[8 * k + 2], s[8 * k + 3])),
                                                fmaxf(fmaxf(s[8 * k + 4], s[8 * k + 5]), fmaxf(s[8 * k + 6], s[8 * k + 7])));
      const float tmax = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      // token 0 is visible to every row, so after tile 0 m_run is finite
      float f = 1.f;
      bool need = false;
      if (j == 0) {
        m_run = tmax;
      } else if ((tmax - m_run) * c2 > kRescaleLog2) {
        need = true;
        f = ex2((m_run - tmax) * c2);
        m_run = tmax;
        l_run *= f;
      }
      const float2 nmc = make_float2(-m_run * c2, -m_run * c2);
      const float2 cc2 = make_float2(c2, c2);
      uint32_t ph[32];
      float2 sum[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const float2 x = __ffma2_rn(make_float2(s[2 * k], s[2 * k + 1]), cc2, nmc);
        const float2 e = make_float2(ex2(x.x), ex2(x.y));
        sum[k & 1] = __fadd2_rn(sum[k & 1], e);
        ph[k] = pack_p(e);
      }
      l_run += (sum[0].x + sum[0].y) + (sum[1].x + sum[1].y);

      // -- P(j) over S(j) in tensor memory (S(j) is in registers now)
      tmem_st32u(t_s + (j & 1) * kPrefillKv, ph);
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      // -- a row whose max grew: O, complete up to tile j-1, rescaled before PV(j)
      if (__any_sync(kFullMask, need)) {
        wait(&tb[4 + ((j - 1) & 1)], ((j - 1) >> 1) & 1);   // PV(j-1) done; need implies j > 0
        if (!ok) break;
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          float o[32];
          tmem_ld32(t_o + c, o);
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] *= f;
          tmem_st32(t_o + c, o);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tb[2 + (j & 1)]);   // P(j) written (and O rescaled)
    }
    if (ntw > 0) {
      // -- epilogue: O / l -> out, staged through this tile's Q buffer (its
      // last QK has completed: the softmax saw its scores).  Each thread puts
      // its row in shared memory (16-byte chunk c of row r at position
      // c ^ (r & 15): four wavefronts a warp store), then the warpgroup copies
      // the valid rows out with consecutive lanes on consecutive chunks, so
      // that a warp store covers two whole 256-byte rows.
      wait(&tb[4 + ((ntw - 1) & 1)], ((ntw - 1) >> 1) & 1);   // the last PV (and so every PV) done
      uint8_t *stage = smem + SM::kQ + w * SM::kQTileBytes;
      if (ok) {
        const float inv = (PK::kConvertV ? 256.f : 1.f) / l_run;   // V entered P V scaled by 2^-8
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          float o[32];
          tmem_ld32(t_o + c, o);
#pragma unroll
          for (int k = 0; k < 32; k += 8)
            *reinterpret_cast<uint4 *>(stage + r * 256 + ((((c + k) >> 3) ^ (r & 15)) << 4)) =
                make_uint4(PK::pack(o[k] * inv, o[k + 1] * inv), PK::pack(o[k + 2] * inv, o[k + 3] * inv),
                           PK::pack(o[k + 4] * inv, o[k + 5] * inv), PK::pack(o[k + 6] * inv, o[k + 7] * inv));
        }
      }
      // every warp of the warpgroup takes the barrier, and copies out only if all staged their rows
      const bool all_ok = w == 0 ? warpgroup_all<2>(ok) : warpgroup_all<3>(ok);   // named barriers 2, 3
      if (all_ok) {
        T *out_t = reinterpret_cast<T *>(p.out);
        const int units = nq * G * 16;   // 16-byte chunks of the valid rows
#pragma unroll 4
        for (int u = r; u < units; u += 128) {
          const int rr = u >> 4, ch = u & 15;
          const uint4 v = *reinterpret_cast<const uint4 *>(stage + rr * 256 + ((ch ^ (rr & 15)) << 4));
          *reinterpret_cast<uint4 *>(out_t + (static_cast<size_t>(qs + q0 + rr / G) * p.num_heads + g * G + rr % G) * D +
                                     ch * 8) = v;
        }
      }
    }
    tc_fence_before();
  }

  // ---- all roles done.  Every tensor-core operation, and every barrier arrival
  // that a commit makes, lands before the memory is released; after an abort
  // the copies in flight are let finish too (all bounded).
  __syncthreads();
  if ((warp == kPrefillMmaWarp || warp == kPrefillMmaWarp + 2) && lane == 0) {
    umma_commit(drain);   // both issuers: their own operations (and commit arrivals) complete
    mbar_wait(drain, 0, wait_limit);
  }
  if (*abort_s && warp == kPrefillLoadWarp && lane == 0) {
    // every stage: the last tile issued into it (its earlier phases completed before it was reissued)
    for (int i = 0; i < KS; ++i)
      if (last_k[i] >= 0) mbar_wait(&k_full[i], (last_k[i] / KS) & 1, wait_limit);
    for (int i = 0; i < VS; ++i)
      if (last_v[i] >= 0) mbar_wait(&v_full[i], (last_v[i] / VS) & 1, wait_limit);
  }
  __syncthreads();
  if (warp == kPrefillMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kPrefillTmemCols);
  }
}

}  // namespace pa
