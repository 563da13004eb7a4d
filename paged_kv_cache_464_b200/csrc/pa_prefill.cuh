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
// Work decomposition.  One CTA of 128 threads per (sequence, KV head, tile of
// 128 / G chunk queries): its 128 rows are the G query heads of each of the
// 128 / G queries (row = query * G + head), so every K/V tile read from the
// cache serves all grouped heads.  The KV walk runs over tiles of 64 tokens
// (four cache blocks) up to the last query's position:
//   S = Q K^T   tcgen05.mma M=128 N=64 K=16 (x8 over head_dim), fp32 in tensor memory;
//   softmax     each thread owns one row: tcgen05.ld of its 64 scores, causal
//               mask on the diagonal tiles, online max/sum in base 2, O rescaled
//               in tensor memory only when a row's max grows by more than 2^8;
//   O += P V    P written to shared memory as two 16-bit parts hi + lo
//               (hi = round(p), lo = round(p - hi)), so P carries ~16 bits like
//               the decode kernel; M=128 N=128 K=16 (x4 tokens, x2 parts).
// K and V tiles arrive by TMA (four 2 KiB boxes per 128-byte half of the rows,
// 128-byte swizzled) into rings of 3 stages each; the QK^T of tile j+1 is issued
// before the softmax of tile j, and the PV of tile j-1 runs under it.
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
  float scale_log2;                   // scale * log2(e)
};

constexpr int kPrefillThreads = 128;
constexpr int kPrefillRows = 128;       // M: rows of one CTA
constexpr int kPrefillKv = 64;          // N of S = Q K^T: tokens per KV tile
constexpr int kPrefillKStages = 3;
constexpr int kPrefillVStages = 3;
constexpr int kPrefillTmemCols = 256;   // S double buffer (2 x 64) + O (128)
constexpr float kRescaleLog2 = 8.f;     // rescale O once a row's max grows by more than this (base-2 units)

struct PrefillSmem {
  static constexpr int kQ = 0;                          // [2 halves][128 rows][128 B]
  static constexpr int kQBytes = 2 * kPrefillRows * 128;
  static constexpr int kKvTileBytes = 2 * kPrefillKv * 128;   // [2 halves][64 tokens][128 B]
  static constexpr int kHalfBytes = kPrefillKv * 128;
  static constexpr int kK = kQ + kQBytes;
  static constexpr int kV = kK + kPrefillKStages * kKvTileBytes;
  static constexpr int kP = kV + kPrefillVStages * kKvTileBytes;   // P hi [128][128 B], then P lo
  static constexpr int kPBytes = kPrefillRows * 128;
  static constexpr int kBar = kP + 2 * kPBytes;
  // k_full[KS], v_full[VS], s_full[2], o_done, drain
  static constexpr int kNumBars = kPrefillKStages + kPrefillVStages + 4;
  static constexpr int kTmemSlot = kBar + 8 * kNumBars;
  static constexpr int kFlag = kTmemSlot + 4;
  static constexpr int kBytes = kFlag + 4;
  static constexpr int kAlloc = kBytes + 1024;   // + alignment of the base to 1024 B (swizzle atoms)
};

template <typename T>
struct Pack16;
template <>
struct Pack16<__nv_bfloat16> {
  static constexpr int kFormat = 1;   // tcgen05 kind::f16 operand format
  __device__ __forceinline__ static uint32_t pack(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
  }
  __device__ __forceinline__ static float lo(uint32_t u) { return __uint_as_float(u << 16); }
  __device__ __forceinline__ static float hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }
};
template <>
struct Pack16<__half> {
  static constexpr int kFormat = 0;
  __device__ __forceinline__ static uint32_t pack(float a, float b) {
    __half2 v = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
  }
  __device__ __forceinline__ static float lo(uint32_t u) { return __half2float(__ushort_as_half((unsigned short)u)); }
  __device__ __forceinline__ static float hi(uint32_t u) {
    return __half2float(__ushort_as_half((unsigned short)(u >> 16)));
  }
};

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

template <typename T, int G>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    pa_prefill_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const PrefillParams p) {
  using SM = PrefillSmem;
  using PK = Pack16<T>;
  constexpr int D = 128;
  constexpr int QT = kPrefillRows / G;   // chunk queries per CTA
  constexpr int KS = kPrefillKStages;
  constexpr int VS = kPrefillVStages;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *q_s = smem + SM::kQ;
  uint8_t *p_s = smem + SM::kP;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::kBar);
  uint64_t *k_full = bars;
  uint64_t *v_full = bars + KS;
  uint64_t *s_full = bars + KS + VS;
  uint64_t *o_done = bars + KS + VS + 2;
  uint64_t *drain = bars + KS + VS + 3;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + SM::kTmemSlot);
  volatile int *abort_s = reinterpret_cast<int *>(smem + SM::kFlag);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  pdl_wait();
  pdl_trigger();

  // ---- work item; the longest query tiles are launched first
  const int qt = gridDim.x - 1 - blockIdx.x;
  const int g = blockIdx.y;
  const int b = blockIdx.z;
  const int L = p.context_lens[b];
  const int qs = p.query_start_loc[b];
  const int n = p.query_start_loc[b + 1] - qs;
  if (n < 0 || n > p.max_query_len || L < n || L > p.max_blocks_per_seq * kBlockSize) {
    if (qt == 0 && g == 0 && tid == 0) record_error(4 /*PA_DEV_BAD_CONTEXT_LEN*/, b);
    return;
  }
  const int q0 = qt * QT;
  if (q0 >= n) return;
  const int nq = min(QT, n - q0);                  // queries of this tile
  const int pos_first = L - n + q0;                // position of its first query
  const int pos_last = pos_first + nq - 1;         // ... and of its last
  const int ntiles = pos_last / kPrefillKv + 1;    // KV tiles covering tokens 0 .. pos_last
  const int nblk = pos_last / kBlockSize + 1;      // cache blocks covering them
  const int32_t *bt_row = p.block_tables + static_cast<size_t>(b) * p.max_blocks_per_seq;

  // ---- this thread's row
  const int i_row = tid / G;
  const bool row_valid = i_row < nq;
  const int pos_r = pos_first + min(i_row, nq - 1);   // padding rows repeat the last query (never stored)

  if (tid == 0) {
    prefetch_tensor_map(&tm_k);
    prefetch_tensor_map(&tm_v);
    for (int i = 0; i < SM::kNumBars; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
    *abort_s = 0;
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kPrefillTmemCols);
    tmem_relinquish();
  }

  // ---- Q tile -> shared memory, K-major 128-byte swizzled: [d half][row][128 B]
  {
    const T *qg = reinterpret_cast<const T *>(p.q);
    for (int idx = tid; idx < kPrefillRows * 16; idx += kPrefillThreads) {
      const int row = idx >> 4, c = idx & 15;
      const int i = row / G, hl = row % G;
      uint4 x = make_uint4(0u, 0u, 0u, 0u);
      if (i < nq)
        x = *reinterpret_cast<const uint4 *>(
            qg + (static_cast<size_t>(qs + q0 + i) * p.num_heads + g * G + hl) * D + c * 8);
      *reinterpret_cast<uint4 *>(q_s + (c >> 3) * (kPrefillRows * 128) + row * 128 + (((c & 7) ^ (row & 7)) << 4)) =
          x;
    }
  }
  fence_proxy_async_smem();   // the generic stores of Q are read by the tensor cores
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_s0 = tmem, t_o = tmem + 128;   // S buffers at columns 0 and 64, O at 128
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;

  // ---- TMA of K / V tiles (warp 0; the block ids of 8 tiles are held one per lane)
  int k_grp = -1, k_id = 0, v_grp = -1, v_id = 0;
  int k_issued = 0, v_issued = 0;   // tiles issued (warp 0)
  int k_waited = 0, v_waited = 0;   // tiles whose arrival was waited for (thread 0)
  auto tile_id = [&](int j, int bi, int &grp, int &id) -> int {   // warp 0, all lanes, j uniform
    const int want = (4 * j) >> 5;
    if (want != grp) {
      grp = want;
      const int lb = (grp << 5) + lane;
      id = static_cast<int>(p.num_blocks);   // past the end of the pool: the box reads zeros
      if (lb < nblk) {
        const int v = bt_row[lb];
        if (v < 0 || v >= p.num_blocks) record_error(1 /*PA_DEV_BAD_BLOCK_ID*/, v);
        else id = v;
      }
    }
    return __shfl_sync(kFullMask, id, (4 * j + bi) & 31);
  };
  auto issue_tile = [&](int j, bool is_v) {   // warp 0
    int ids[4];
#pragma unroll
    for (int bi = 0; bi < 4; ++bi)
      ids[bi] = is_v ? tile_id(j, bi, v_grp, v_id) : tile_id(j, bi, k_grp, k_id);
    if (lane == 0) {
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
    if (is_v) ++v_issued;
    else ++k_issued;
  };

  // ---- tensor-core issue (thread 0)
  constexpr uint32_t kIdescQK = instr_desc_f16(PK::kFormat, false, kPrefillRows, kPrefillKv);
  constexpr uint32_t kIdescPV = instr_desc_f16(PK::kFormat, true, kPrefillRows, D);
  auto issue_qk = [&](int j) {   // S[j & 1] = Q K_j^T
    const uint8_t *kt = smem + SM::kK + (j % KS) * SM::kKvTileBytes;
    const uint32_t d_tmem = t_s0 + (j & 1) * kPrefillKv;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint64_t a = smem_desc_sw128(q_s + (kk >> 2) * (kPrefillRows * 128) + (kk & 3) * 32, 16, 1024);
      const uint64_t bd = smem_desc_sw128(kt + (kk >> 2) * SM::kHalfBytes + (kk & 3) * 32, 16, 1024);
      umma_f16(d_tmem, a, bd, kIdescQK, kk > 0);
    }
    umma_commit(&s_full[j & 1]);
  };
  auto issue_pv = [&](int j) {   // O += P_hi V_j + P_lo V_j
    const uint8_t *vt = smem + SM::kV + (j % VS) * SM::kKvTileBytes;
#pragma unroll
    for (int part = 0; part < 2; ++part)
#pragma unroll
      for (int kk = 0; kk < kPrefillKv / 16; ++kk) {
        const uint64_t a = smem_desc_sw128(p_s + part * SM::kPBytes + kk * 32, 16, 1024);
        const uint64_t bd = smem_desc_sw128(vt + kk * 16 * 128, SM::kHalfBytes, 1024);
        umma_f16(t_o, a, bd, kIdescPV, j > 0 || part > 0 || kk > 0);
      }
    umma_commit(o_done);
  };

  if (warp == 0) {
    for (int j = 0; j < min(KS, ntiles); ++j) issue_tile(j, false);
    for (int j = 0; j < min(VS, ntiles); ++j) issue_tile(j, true);
  }
  bool ok = true;
  if (tid == 0) {
    ok = mbar_wait(&k_full[0], 0);
    if (ok) k_waited = 1;
    if (ok) {
      tc_fence_after();
      issue_qk(0);
    }
  }

  float m_run = -INFINITY;   // running max of this row, base-2 scaled units
  float l_run = 0.f;         // running sum of 2^(s - m_run)
  const float c2 = p.scale_log2;
  int j = 0;
  for (; j < ntiles; ++j) {
    if (tid == 0 && ok && j + 1 < ntiles) {
      ok = mbar_wait(&k_full[(j + 1) % KS], ((j + 1) / KS) & 1);
      if (ok) k_waited = j + 2;
      if (ok) {
        tc_fence_after();
        issue_qk(j + 1);
      }
    }
    // -- S_j
    const bool s_ok = mbar_wait(&s_full[j & 1], (j >> 1) & 1);
    tc_fence_after();
    if (warp == 0 && j + KS < ntiles && __all_sync(kFullMask, s_ok)) issue_tile(j + KS, false);   // K_j consumed
    float s[64];
    tmem_ld64(t_s0 + (j & 1) * kPrefillKv + lane_base, s);
    const int t0 = j * kPrefillKv;
    float mx = -INFINITY;
    if (t0 + kPrefillKv - 1 > pos_first) {   // a diagonal tile: mask tokens after each row's position
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        s[c] = (t0 + c <= pos_r) ? s[c] * c2 : -INFINITY;
        mx = fmaxf(mx, s[c]);
      }
    } else {
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        s[c] *= c2;
        mx = fmaxf(mx, s[c]);
      }
    }
    // token 0 is visible to every row, so after tile 0 m_run is finite
    float f = 1.f;
    bool need = false;
    if (j == 0) {
      m_run = mx;
    } else if (mx > m_run + kRescaleLog2) {
      need = true;
      f = ex2(m_run - mx);
      m_run = mx;
      l_run *= f;
    }
    uint32_t ph[32], pl[32];
    float sum = 0.f;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const float a = ex2(s[2 * k] - m_run);
      const float bb = ex2(s[2 * k + 1] - m_run);
      sum += a + bb;
      ph[k] = PK::pack(a, bb);
      pl[k] = PK::pack(a - PK::lo(ph[k]), bb - PK::hi(ph[k]));
    }
    l_run += sum;

    // -- PV_{j-1} done: P, O and the V stage of tile j-1 are free
    bool o_ok = true;
    if (j > 0) {
      o_ok = mbar_wait(o_done, (j - 1) & 1);
      tc_fence_after();
      if (warp == 0 && j - 1 + VS < ntiles && __all_sync(kFullMask, o_ok)) issue_tile(j - 1 + VS, true);
    }
    if (__any_sync(kFullMask, need)) {
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        float o[32];
        tmem_ld32(t_o + lane_base + c, o);
#pragma unroll
        for (int k = 0; k < 32; ++k) o[k] *= f;
        tmem_st32(t_o + lane_base + c, o);
      }
    }
    {
      uint8_t *rh = p_s + tid * 128;
      const int sw = tid & 7;
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        *reinterpret_cast<uint4 *>(rh + ((cc ^ sw) << 4)) =
            make_uint4(ph[4 * cc], ph[4 * cc + 1], ph[4 * cc + 2], ph[4 * cc + 3]);
        *reinterpret_cast<uint4 *>(rh + SM::kPBytes + ((cc ^ sw) << 4)) =
            make_uint4(pl[4 * cc], pl[4 * cc + 1], pl[4 * cc + 2], pl[4 * cc + 3]);
      }
    }
    // -- the tile holding token L-1: rows past the context end in its last block
    //    may hold anything (NaN included); make them zero so that 0 * V stays 0
    bool z_ok = true;
    if ((L & (kBlockSize - 1)) != 0 && (L - 1) / kBlockSize == pos_last / kBlockSize && j == ntiles - 1) {
      z_ok = mbar_wait(&v_full[j % VS], (j / VS) & 1);
      if (z_ok) {
        uint8_t *vt = smem + SM::kV + (j % VS) * SM::kKvTileBytes;
        const int r0 = L - t0, r1 = ((L + kBlockSize - 1) / kBlockSize) * kBlockSize - t0;   // rows r0 .. r1-1
        for (int idx = tid; idx < (r1 - r0) * 16; idx += kPrefillThreads) {
          const int r = r0 + (idx >> 4), c = idx & 15;
          *reinterpret_cast<uint4 *>(vt + (c >> 3) * SM::kHalfBytes + r * 128 + (c & 7) * 16) =
              make_uint4(0u, 0u, 0u, 0u);
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    if (!s_ok || !o_ok || !z_ok || !ok) *abort_s = 1;
    __syncthreads();
    if (*abort_s) break;
    tc_fence_after();
    if (tid == 0) {
      ok = mbar_wait(&v_full[j % VS], (j / VS) & 1);
      if (ok) {
        v_waited = j + 1;
        issue_pv(j);
      } else {
        *abort_s = 1;   // seen at the next barrier
      }
    }
  }

  bool failed = j < ntiles;
  if (!failed) {
    const bool fin = mbar_wait(o_done, (ntiles - 1) & 1);
    if (!fin) *abort_s = 1;
    __syncthreads();
    failed = *abort_s != 0;
  }
  if (failed) {
    if (tid == 0) {
      record_error(5 /*PA_DEV_WAIT_TIMEOUT*/, blockIdx.x);
      // let every copy and tensor-core operation in flight finish (bounded) before the memory is released
      for (int t = k_waited; t < k_issued; ++t) mbar_wait(&k_full[t % KS], (t / KS) & 1);
      for (int t = v_waited; t < v_issued; ++t) mbar_wait(&v_full[t % VS], (t / VS) & 1);
      umma_commit(drain);
      mbar_wait(drain, 0);
    }
  } else {
    tc_fence_after();
    // -- epilogue: O / l -> out
    const float inv = 1.f / l_run;
    T *orow = reinterpret_cast<T *>(p.out) +
              (static_cast<size_t>(qs + q0 + i_row) * p.num_heads + g * G + tid % G) * D;
#pragma unroll 1
    for (int c = 0; c < D; c += 32) {
      float o[32];
      tmem_ld32(t_o + lane_base + c, o);
      if (row_valid) {
#pragma unroll
        for (int k = 0; k < 32; k += 8)
          *reinterpret_cast<uint4 *>(orow + c + k) =
              make_uint4(PK::pack(o[k] * inv, o[k + 1] * inv), PK::pack(o[k + 2] * inv, o[k + 3] * inv),
                         PK::pack(o[k + 4] * inv, o[k + 5] * inv), PK::pack(o[k + 6] * inv, o[k + 7] * inv));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kPrefillTmemCols);
  }
}

}  // namespace pa
