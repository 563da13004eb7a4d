// pa_decode.cuh -- paged decode attention for sm_100a.
//
// What it computes ("vLLM推理引擎深度解析", §五 优化的注意力计算,
// PagedAttention.forward; "vLLM 原理与源码阅读", PagedAttention 核心思想):
// for each sequence b and query head h, softmax(scale * q K^T) V over the
// sequence's tokens, with K/V rows found through the sequence's block table
// (logical block j -> one physical block).  Unlike the page's sketch, the
// gathered K/V are never assembled in memory: each block is read once, straight
// from its physical location, as the page says the real kernel does.
//
// Work decomposition
//   One CTA = (sequence b, KV head g, partition p): the tokens
//   [p*P, min((p+1)*P, L_b)) of one KV head, serving all G = Hq/Hkv query heads
//   of that KV head from a single read of each K/V block.  Sequences longer
//   than P are split (split-K); each piece leaves an unnormalised partial
//   (running max m, sum l, vector o) in the workspace and reduce_kernel
//   combines them.  A sequence that fits in one partition is finished here.
//
// Inside a CTA (4 warps, no producer warp)
//   Warp w owns the partition's blocks w, w+4, w+8, ... and keeps its own
//   online-softmax state.  Each warp has kStagesPerWarp shared-memory stages;
//   one elected lane issues a TMA tensor load for the K tile and the V tile of
//   a block (16 tokens x 256 B each, a strided box of the [NB][16][Hkv][256 B]
//   cache) into a stage, completing on that stage's mbarrier.  After a warp has
//   used a stage it issues the load of its block kStagesPerWarp ahead into it.
//   The tiles land 128-byte swizzled: the 16-byte chunk c of 128-byte row r
//   sits at chunk position c ^ (r & 7), so the per-lane row reads below are
//   free of bank conflicts.
//
//   QK: lane = 128-byte row r (token t = r / 2, half = r & 1 of the 256-byte
//   row).  Each lane dots its half-row with the G query vectors (fp32,
//   pre-scaled by scale*log2(e), broadcast from shared memory) with packed
//   fp32x2 FMAs; one xor-shuffle joins the halves.
//   Softmax: block max by a single warp reduction per head (redux.sync.max.f32),
//   base-2 exponentials, running max/sum per warp (online softmax).
//   PV: lane = (16-byte chunk cc of the output row, token parity); each lane
//   accumulates G x (8 or 4) outputs over the block's tokens of its parity.
//   Rows past the sequence end are skipped in PV (they may hold anything) and
//   get weight 0 in QK.
//   Epilogue: parities and warps are merged through shared memory.
#pragma once

#include "pa_common.cuh"

namespace pa {

constexpr int kDecodeWarps = 4;
constexpr int kDecodeThreads = kDecodeWarps * 32;
constexpr int kStagesPerWarp = 2;
constexpr int kStages = kDecodeWarps * kStagesPerWarp;

struct DecodeParams {
  void *out;                      // [S][Hq][D]
  const void *q;                  // [S][Hq][D]
  const int32_t *block_tables;    // [S][MBS]
  const int32_t *context_lens;    // [S]
  float *ws_m;                    // [S][Hq][NPmax]
  float *ws_l;                    // [S][Hq][NPmax]
  float *ws_o;                    // [S][Hq][NPmax][D]
  long long num_blocks;
  int num_seqs, num_heads, num_kv_heads, max_blocks_per_seq;
  int max_context_len, partition_size, max_partitions;
  float scale_log2;               // scale * log2(e)
};

template <typename T, int G>
struct DecodeSmem {
  static constexpr int kPerChunk = Elem<T>::kPerChunk;
  static constexpr int D = kChunksPerRow * kPerChunk;
  static constexpr int kHalf = D / 2;
  static constexpr int kQStride = kHalf + 4;   // floats; pads the two halves onto different banks
  static constexpr int kTilesBytes = kStages * 2 * kTileBytes;
  static constexpr int kQOff = kTilesBytes;
  static constexpr int kPOff = kQOff + G * 2 * kQStride * 4;
  static constexpr int kMOff = kPOff + kDecodeWarps * kBlockSize * G * 4;
  static constexpr int kLOff = kMOff + kDecodeWarps * G * 4;
  static constexpr int kFlagOff = kLOff + kDecodeWarps * G * 4;
  static constexpr int kBarOff = (kFlagOff + 4 + 7) / 8 * 8;
  static constexpr int kBytes = kBarOff + kStages * 8;
  static constexpr int kAlloc = kBytes + 1024;   // room to align the base to 1024 B (128B swizzle atom)
  static_assert(kDecodeWarps * G * D * 4 <= kTilesBytes, "epilogue buffer must fit in the stage tiles");
};

template <typename T, int G>
__global__ void __launch_bounds__(kDecodeThreads, 3)
    pa_decode_partition_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                               const DecodeParams p) {
  using SM = DecodeSmem<T, G>;
  constexpr int EPC = SM::kPerChunk;
  constexpr int D = SM::D;
  constexpr int HALF = SM::kHalf;
  constexpr int QS = SM::kQStride;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float *q_s = reinterpret_cast<float *>(smem + SM::kQOff);
  float *p_s = reinterpret_cast<float *>(smem + SM::kPOff);
  float *m_s = reinterpret_cast<float *>(smem + SM::kMOff);
  float *l_s = reinterpret_cast<float *>(smem + SM::kLOff);
  int *abort_s = reinterpret_cast<int *>(smem + SM::kFlagOff);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + SM::kBarOff);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work item: blockIdx.x = ((b * Hkv) + g) * NPmax + part
  int item = blockIdx.x;
  const int part = item % p.max_partitions;
  item /= p.max_partitions;
  const int g = item % p.num_kv_heads;
  const int b = item / p.num_kv_heads;
  const int L = p.context_lens[b];
  if (L < 0 || L > p.max_context_len || L > p.max_blocks_per_seq * kBlockSize) {
    if (part == 0 && g == 0 && threadIdx.x == 0) record_error(4 /*PA_DEV_BAD_CONTEXT_LEN*/, b);
    return;
  }
  const int P = p.partition_size;
  const int nparts = (L + P - 1) / P;
  const int h0 = g * G;   // first query head of this KV head (contiguous groups)
  T *out = reinterpret_cast<T *>(p.out) + (static_cast<size_t>(b) * p.num_heads + h0) * D;
  if (L == 0) {   // empty context: the row is the empty sum, zeros
    if (part == 0)
      for (int i = threadIdx.x * 4; i < G * D; i += kDecodeThreads * 4) Elem<T>::store4(out + i, 0.f, 0.f, 0.f, 0.f);
    return;
  }
  if (part >= nparts) return;
  const int tok0 = part * P;
  const int tok1 = min(tok0 + P, L);
  const int nblk = (tok1 - tok0 + kBlockSize - 1) / kBlockSize;

  if (threadIdx.x == 0) {
    prefetch_tensor_map(&tm_k);
    prefetch_tensor_map(&tm_v);
    for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
    *abort_s = 0;
  }

  // ---- this warp's blocks: local block index lb = warp + j * 4, j = 0 .. nw-1
  const int nw = nblk > warp ? (nblk - warp + kDecodeWarps - 1) / kDecodeWarps : 0;
  const int32_t *bt_row = p.block_tables + static_cast<size_t>(b) * p.max_blocks_per_seq + tok0 / kBlockSize;
  int id_group = -1;   // which 32 consecutive j's the lanes' ids belong to
  int my_id = -1;      // lane l holds the physical id of j = 32 * id_group + l
  const uint64_t policy = policy_evict_first();

  auto issue = [&](int j) {   // called by all 32 lanes, j warp-uniform
    if ((j >> 5) != id_group) {
      id_group = j >> 5;
      const int jj = (id_group << 5) + lane;
      my_id = -1;
      if (jj < nw) {
        const int id = bt_row[warp + jj * kDecodeWarps];
        if (id < 0 || id >= p.num_blocks) record_error(1 /*PA_DEV_BAD_BLOCK_ID*/, id);
        else my_id = id;
      }
    }
    const int id = __shfl_sync(kFullMask, my_id, j & 31);
    const int s = warp + (j % kStagesPerWarp) * kDecodeWarps;
    if (lane == 0) {
      if (id >= 0) {
        uint8_t *tk = smem + s * 2 * kTileBytes;
        mbar_arrive_expect_tx(&full[s], 2 * kTileBytes);
        tma_load_5d(tk, &tm_k, 0, 0, g, 0, id, &full[s], policy);
        tma_load_5d(tk + kTileBytes, &tm_v, 0, 0, g, 0, id, &full[s], policy);
      } else {
        mbar_arrive(&full[s]);   // bad id: recorded above; complete the phase without data
      }
    }
  };

  // query vectors of the G heads, fp32, pre-scaled, halves padded apart
  {
    const T *qg = reinterpret_cast<const T *>(p.q) + (static_cast<size_t>(b) * p.num_heads + h0) * D;
    for (int i = threadIdx.x; i < G * D; i += kDecodeThreads) {
      const int hh = i / D, d = i % D;
      q_s[(hh * 2 + d / HALF) * QS + d % HALF] = Elem<T>::load(qg + i) * p.scale_log2;
    }
  }
  __syncthreads();   // barriers initialised, q staged

  for (int j = 0; j < min(nw, kStagesPerWarp); ++j) issue(j);

  float m_run[G], l_run[G];
  float2 o[G][EPC / 2];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    m_run[hh] = -INFINITY;
    l_run[hh] = 0.f;
#pragma unroll
    for (int e = 0; e < EPC / 2; ++e) o[hh][e] = make_float2(0.f, 0.f);
  }

  // lane roles
  const int r = lane;              // QK: 128-byte row of the tile
  const int t_qk = r >> 1;         // its token
  const int half = r & 1;          // which half of the 256-byte row
  const int cc = lane & 15;        // PV: output chunk
  const int par = lane >> 4;       // PV: token parity
  const int r_pv_hi = cc >> 3;     // which 128-byte half holds chunk cc
  const int c_pv = cc & 7;
  float *p_w = p_s + warp * kBlockSize * G;

  bool ok = true;
  int j = 0;
  for (; j < nw; ++j) {
    const int s = warp + (j % kStagesPerWarp) * kDecodeWarps;
    const bool landed = mbar_wait(&full[s], (j / kStagesPerWarp) & 1);
    if (!__all_sync(kFullMask, landed)) {
      if (lane == 0) {
        record_error(5 /*PA_DEV_WAIT_TIMEOUT*/, blockIdx.x);
        *abort_s = 1;
      }
      ok = false;
      break;
    }
    const uint8_t *tk = smem + s * 2 * kTileBytes;
    const uint8_t *tv = tk + kTileBytes;
    const int nvalid = min(kBlockSize, tok1 - (tok0 + (warp + j * kDecodeWarps) * kBlockSize));

    // ---- scores of this lane's token for the G heads (half row each)
    float2 acc[G];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) acc[hh] = make_float2(0.f, 0.f);
    const uint8_t *krow = tk + r * 128;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint4 raw = *reinterpret_cast<const uint4 *>(krow + ((c ^ (r & 7)) << 4));
      float kf[EPC];
      Elem<T>::unpack(raw, kf);
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        const float *qp = q_s + (hh * 2 + half) * QS + c * EPC;
#pragma unroll
        for (int e = 0; e < EPC; e += 4) {
          const float4 qv = *reinterpret_cast<const float4 *>(qp + e);
          acc[hh] = __ffma2_rn(make_float2(kf[e], kf[e + 1]), make_float2(qv.x, qv.y), acc[hh]);
          acc[hh] = __ffma2_rn(make_float2(kf[e + 2], kf[e + 3]), make_float2(qv.z, qv.w), acc[hh]);
        }
      }
    }
    const bool valid = t_qk < nvalid;
    float pr[G];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      float sc = acc[hh].x + acc[hh].y;
      sc += __shfl_xor_sync(kFullMask, sc, 1);
      sc = valid ? sc : -INFINITY;
      const float m_new = fmaxf(m_run[hh], warp_max(sc));
      if (m_new != m_run[hh]) {   // warp-uniform
        const float alpha = ex2(m_run[hh] - m_new);
        l_run[hh] *= alpha;
#pragma unroll
        for (int e = 0; e < EPC / 2; ++e) o[hh][e] = __fmul2_rn(o[hh][e], make_float2(alpha, alpha));
        m_run[hh] = m_new;
      }
      pr[hh] = ex2(sc - m_new);
      l_run[hh] += pr[hh];
    }
    if (half == 0) {
#pragma unroll
      for (int hh = 0; hh < G; ++hh) p_w[t_qk * G + hh] = pr[hh];
    }
    __syncwarp();

    // ---- o += p * V over this lane's parity of the block's tokens
#pragma unroll
    for (int i = 0; i < kBlockSize / 2; ++i) {
      const int tt = 2 * i + par;
      if (tt < nvalid) {
        const int rr = 2 * tt + r_pv_hi;
        const uint4 raw = *reinterpret_cast<const uint4 *>(tv + rr * 128 + ((c_pv ^ (rr & 7)) << 4));
        float vf[EPC];
        Elem<T>::unpack(raw, vf);
        float pv[G];
        if constexpr (G % 4 == 0) {
#pragma unroll
          for (int hh = 0; hh < G; hh += 4) {
            const float4 x = *reinterpret_cast<const float4 *>(p_w + tt * G + hh);
            pv[hh] = x.x; pv[hh + 1] = x.y; pv[hh + 2] = x.z; pv[hh + 3] = x.w;
          }
        } else if constexpr (G == 2) {
          const float2 x = *reinterpret_cast<const float2 *>(p_w + tt * 2);
          pv[0] = x.x; pv[1] = x.y;
        } else {
          pv[0] = p_w[tt];
        }
#pragma unroll
        for (int hh = 0; hh < G; ++hh)
#pragma unroll
          for (int e = 0; e < EPC / 2; ++e)
            o[hh][e] = __ffma2_rn(make_float2(vf[2 * e], vf[2 * e + 1]), make_float2(pv[hh], pv[hh]), o[hh][e]);
      }
    }
    __syncwarp();   // all lanes done with the stage and with p_w
    if (j + kStagesPerWarp < nw) {
      fence_proxy_async_smem();
      issue(j + kStagesPerWarp);
    }
  }
  if (!ok) {
    // let this warp's other copies in flight land (bounded) before the CTA can exit
    for (int jj = j + 1; jj < min(nw, j + kStagesPerWarp); ++jj)
      mbar_wait(&full[warp + (jj % kStagesPerWarp) * kDecodeWarps], (jj / kStagesPerWarp) & 1);
  }

  // ---- merge: l over the 16 tokens, o over the two parities
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    float l = l_run[hh];
    l += __shfl_xor_sync(kFullMask, l, 2);
    l += __shfl_xor_sync(kFullMask, l, 4);
    l += __shfl_xor_sync(kFullMask, l, 8);
    l += __shfl_xor_sync(kFullMask, l, 16);
    l_run[hh] = l;
#pragma unroll
    for (int e = 0; e < EPC / 2; ++e) {
      o[hh][e].x += __shfl_xor_sync(kFullMask, o[hh][e].x, 16);
      o[hh][e].y += __shfl_xor_sync(kFullMask, o[hh][e].y, 16);
    }
  }
  __syncthreads();   // every warp is done with the stage tiles: reuse them for the merge
  float *o_s = reinterpret_cast<float *>(smem);
  if (par == 0) {
#pragma unroll
    for (int hh = 0; hh < G; ++hh)
#pragma unroll
      for (int e = 0; e < EPC / 2; ++e)
        *reinterpret_cast<float2 *>(o_s + (warp * G + hh) * D + cc * EPC + 2 * e) = o[hh][e];
  }
  if (lane == 0) {
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      m_s[warp * G + hh] = m_run[hh];
      l_s[warp * G + hh] = l_run[hh];
    }
  }
  __syncthreads();
  if (*abort_s) return;

  for (int i = threadIdx.x * 4; i < G * D; i += kDecodeThreads * 4) {
    const int hh = i / D, d = i % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecodeWarps; ++w) M = fmaxf(M, m_s[w * G + hh]);
    float lsum = 0.f;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < kDecodeWarps; ++w) {
      const float f = ex2(m_s[w * G + hh] - M);   // 0 for a warp that saw no token
      lsum += f * l_s[w * G + hh];
      const float4 x = *reinterpret_cast<const float4 *>(o_s + (w * G + hh) * D + d);
      a.x += f * x.x;
      a.y += f * x.y;
      a.z += f * x.z;
      a.w += f * x.w;
    }
    if (nparts == 1) {
      const float inv = 1.f / lsum;
      Elem<T>::store4(out + i, a.x * inv, a.y * inv, a.z * inv, a.w * inv);
    } else {
      const size_t row = (static_cast<size_t>(b) * p.num_heads + h0 + hh) * p.max_partitions + part;
      *reinterpret_cast<float4 *>(p.ws_o + row * D + d) = a;
      if (d == 0) {
        p.ws_m[row] = M;
        p.ws_l[row] = lsum;
      }
    }
  }
}

// Combine the partitions of every (sequence, query head) that was split:
//   M = max_p m_p,  out = sum_p 2^(m_p - M) o_p / sum_p 2^(m_p - M) l_p
// (m_p are base-2 log-domain maxima; o_p and l_p are relative to m_p).
// One warp per (b, h); each lane owns D/32 consecutive outputs.
template <typename T>
__global__ void __launch_bounds__(128) pa_decode_reduce_kernel(const DecodeParams p) {
  constexpr int D = kChunksPerRow * Elem<T>::kPerChunk;
  constexpr int PER_LANE = D / 32;
  const int lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * 4 + (threadIdx.x >> 5);
  if (row >= static_cast<long long>(p.num_seqs) * p.num_heads) return;
  const int b = static_cast<int>(row / p.num_heads);
  const int L = p.context_lens[b];
  if (L < 0 || L > p.max_context_len || L > p.max_blocks_per_seq * kBlockSize) return;
  const int np = (L + p.partition_size - 1) / p.partition_size;
  if (np <= 1) return;   // finished by the partition kernel
  const float *m = p.ws_m + row * p.max_partitions;
  const float *l = p.ws_l + row * p.max_partitions;
  const float *o = p.ws_o + row * p.max_partitions * D;

  float M = -INFINITY;
  for (int i = lane; i < np; i += 32) M = fmaxf(M, m[i]);
  M = warp_max(M);
  float lsum = 0.f;
  float acc[PER_LANE];
#pragma unroll
  for (int e = 0; e < PER_LANE; ++e) acc[e] = 0.f;
  for (int base = 0; base < np; base += 32) {
    const int i = base + lane;
    const float w = i < np ? ex2(m[i] - M) : 0.f;
    lsum += i < np ? w * l[i] : 0.f;
    const int n = min(32, np - base);
    for (int k = 0; k < n; ++k) {
      const float wk = __shfl_sync(kFullMask, w, k);
      const float *src = o + static_cast<size_t>(base + k) * D + lane * PER_LANE;
      if constexpr (PER_LANE == 4) {
        const float4 x = *reinterpret_cast<const float4 *>(src);
        acc[0] += wk * x.x;
        acc[1] += wk * x.y;
        acc[2] += wk * x.z;
        acc[3] += wk * x.w;
      } else {
#pragma unroll
        for (int e = 0; e < PER_LANE; ++e) acc[e] += wk * src[e];
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) lsum += __shfl_xor_sync(kFullMask, lsum, off);
  const float inv = 1.f / lsum;
  T *out = reinterpret_cast<T *>(p.out) + row * D + lane * PER_LANE;
  if constexpr (PER_LANE == 4) {
    Elem<T>::store4(out, acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
  } else {
    static_assert(PER_LANE == 2, "D is 64 or 128");
    Elem<T>::store2(out, acc[0] * inv, acc[1] * inv);
  }
}

}  // namespace pa
