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
//   (running max m, sum l, vector o) in the workspace and the reduce kernel
//   combines them.  A sequence that fits in one partition is finished here.
//
// Inside a CTA (W warps, no producer warp; W = kDecodeWarps = 4, or 2 for the
// tensor-core block math when a call splits its sequences into partitions of
// at most 512 tokens: then six two-warp CTAs share an SM instead of three
// four-warp ones, which hides more of each CTA's fixed cost -- measured on B200
// 169.6 against 172.9 µs a call on the long-context workload, while the GQA
// workload with 1024-token partitions is 2% faster with four warps)
//   Warp w owns the partition's blocks w, w+W, w+2W, ... and keeps its own
//   online-softmax state.  Each warp has kStagesPerWarp shared-memory stages;
//   one elected lane issues a TMA tensor load for the K tile and the V tile of
//   a block into a stage, completing on that stage's mbarrier.  After a warp has
//   used a stage it issues the load of its block kStagesPerWarp ahead into it.
//   A tile is the 16 tokens x 256 B of one (block, KV head): a strided box of
//   the cache, landing as [half][token][128 B] (half = which 128-byte half of
//   the row) with the 128-byte swizzle: 16-byte chunk c of row r = half*16 + t
//   sits at chunk position c ^ (t & 7).  Eight consecutive tokens therefore
//   cover all 32 banks, so the row-per-lane reads (CUDA-core path) and the
//   8x8 ldmatrix reads (tensor-core path) are free of bank conflicts.
//
// Two ways to do a block's arithmetic (the pipeline is the same):
//   FmaMath (fp32 caches, and G = 1): CUDA cores.  QK: lane = (token, half);
//     each lane dots its half row with the G query vectors (fp32, pre-scaled
//     by scale*log2(e), broadcast from shared memory) with packed fp32x2 FMAs,
//     one shuffle joins the halves.  PV: lane = (output chunk, token parity).
//   MmaMath (fp16/bf16 caches, G = 2..8): warp-level tensor-core MMA
//     (m16n8k16, fp32 accumulate) on the transposed problem, so the G heads
//     are the narrow N = 8 side and tokens / head_dim are the M = 16 side:
//       S^T[16 tok][8 heads] = K[16 tok][128] . Q^T[128][8 heads]
//       O^T[128][8 heads]   += V^T[128][16 tok] . P^T[16 tok][8 heads]
//     K and V^T fragments come straight from the swizzled tiles (ldmatrix,
//     .trans for V); Q^T fragments stay in registers for the whole partition;
//     the S^T accumulator becomes the P^T operand with one 8x8 transpose
//     (movmatrix) per 8 tokens.  P is fed as hi + lo 16-bit parts (two MMAs)
//     so that rounding P to 16 bits costs nothing measurable (~2^-17).
//   Both use base-2 online softmax with fp32 running max and sum.  Rows past
//   the sequence end get weight 0 and never reach a multiply (their V rows
//   may hold anything).
#pragma once

#include "pa_common.cuh"

namespace pa {

// Launch shape (compile-time): warps per CTA, shared-memory stages per warp and
// the CTAs per SM the register budget is sized for.
#ifndef PA_DECODE_WARPS
#define PA_DECODE_WARPS 4
#endif
#ifndef PA_DECODE_STAGES_PER_WARP
#define PA_DECODE_STAGES_PER_WARP 2
#endif
#ifndef PA_DECODE_MIN_CTAS_PER_SM
#define PA_DECODE_MIN_CTAS_PER_SM 3
#endif
constexpr int kDecodeWarps = PA_DECODE_WARPS;
constexpr int kDecodeThreads = kDecodeWarps * 32;
constexpr int kStagesPerWarp = PA_DECODE_STAGES_PER_WARP;   // for 256-byte rows (128-byte rows: Fp8MmaMath)

struct DecodeParams {
  void *out;                      // [S][Hq][D]
  const void *q;                  // [S][Hq][D]
  const int32_t *block_tables;    // [S][MBS]
  const int32_t *context_lens;    // [S]
  float *ws_m;                    // [S][Hq][NPmax]
  float *ws_l;                    // [S][Hq][NPmax]
  float *ws_o;                    // [S][Hq][NPmax][D]
  unsigned *ws_count;             // [S][Hkv] partitions done (zeroed before the launch); null: separate reduce
  long long num_blocks;
  int num_seqs, num_heads, num_kv_heads, max_blocks_per_seq;
  int max_context_len, partition_size, max_partitions;
  float scale_log2;               // scale * log2(e) (* k_scale for 1-byte caches)
  float v_scale;                  // 1 for 16/32-bit caches
  // append mode (all non-null) or plain decode (all null): the step's new token
  // rows [S][Hkv][D], written at position context_len - 1 before it is attended
  const void *new_k, *new_v;
  void *k_cache, *v_cache;
  int stall_cta;                  // test hook (pa_common.cuh): 0 in every ordinary launch
};

// Byte offset of 16-byte chunk `c` (0..15) of token `t` in a swizzled tile.
__device__ __forceinline__ int tile_offset(int t, int c) {
  return ((c >> 3) * kBlockSize + t) * 128 + (((c & 7) ^ (t & 7)) << 4);
}

// ============================================================ CUDA-core math
template <typename T, int G>
struct FmaMath {
  static constexpr int EPC = Elem<T>::kPerChunk;   // elements per 16-byte chunk
  static constexpr int D = kChunksPerRow * EPC;
  static constexpr int HALF = D / 2;
  static constexpr int QS = HALF + 4;              // q row half stride (floats): halves on different banks
  static constexpr int kQBytes = G * 2 * QS * 4;
  static constexpr int kPBytes = kDecodeWarps * kBlockSize * G * 4;
  static constexpr int kScratchBytes = kQBytes + kPBytes;
  static constexpr bool kNeedsQInSmem = true;
  static constexpr int kRowBytes = 256;
  static constexpr int kStagesPerWarp = pa::kStagesPerWarp;

  float m_run[G], l_run[G];
  float2 o[G][EPC / 2];
  const float *q_s;
  float *p_w;

  // stage the G query vectors (fp32, pre-scaled, halves padded apart); CTA-wide
  __device__ static void stage_q(uint8_t *scratch, const T *qg, float scale_log2) {
    float *q_s = reinterpret_cast<float *>(scratch);
    for (int i = threadIdx.x; i < G * D; i += kDecodeThreads) {
      const int hh = i / D, d = i % D;
      q_s[(hh * 2 + d / HALF) * QS + d % HALF] = Elem<T>::load(qg + i) * scale_log2;
    }
  }

  __device__ void init(uint8_t *scratch, const T *, float, int warp, int) {
    q_s = reinterpret_cast<const float *>(scratch);
    p_w = reinterpret_cast<float *>(scratch + kQBytes) + warp * kBlockSize * G;
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      m_run[hh] = -INFINITY;
      l_run[hh] = 0.f;
#pragma unroll
      for (int e = 0; e < EPC / 2; ++e) o[hh][e] = make_float2(0.f, 0.f);
    }
  }

  __device__ void block(const uint8_t *tk, uint8_t *tv, int nvalid, int lane, float) {
    // ---- scores of this lane's token (half row) for the G heads
    const int t = lane & 15, half = lane >> 4;
    float2 acc[G];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) acc[hh] = make_float2(0.f, 0.f);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint4 raw = *reinterpret_cast<const uint4 *>(tk + tile_offset(t, half * 8 + c));
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
    const bool valid = t < nvalid;
    float pr[G];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      float sc = acc[hh].x + acc[hh].y;
      sc += __shfl_xor_sync(kFullMask, sc, 16);
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
      for (int hh = 0; hh < G; ++hh) p_w[t * G + hh] = pr[hh];
    }
    __syncwarp();

    // ---- o += p * V over this lane's token parity
    const int cc = lane & 15, par = lane >> 4;
#pragma unroll
    for (int i = 0; i < kBlockSize / 2; ++i) {
      const int tt = 2 * i + par;
      if (tt < nvalid) {
        const uint4 raw = *reinterpret_cast<const uint4 *>(tv + tile_offset(tt, cc));
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
  }

  // Merge the lane partials and write this warp's (m, l, o) for the G heads.
  __device__ void write_partials(float *o_s, float *m_s, float *l_s, int warp, int lane, float) {
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      float l = l_run[hh];   // lanes t and t+16 hold the same p: sum over one half
      l += __shfl_xor_sync(kFullMask, l, 1);
      l += __shfl_xor_sync(kFullMask, l, 2);
      l += __shfl_xor_sync(kFullMask, l, 4);
      l += __shfl_xor_sync(kFullMask, l, 8);
      l_run[hh] = l;
#pragma unroll
      for (int e = 0; e < EPC / 2; ++e) {
        o[hh][e].x += __shfl_xor_sync(kFullMask, o[hh][e].x, 16);
        o[hh][e].y += __shfl_xor_sync(kFullMask, o[hh][e].y, 16);
      }
    }
    if (lane < 16) {
#pragma unroll
      for (int hh = 0; hh < G; ++hh)
#pragma unroll
        for (int e = 0; e < EPC / 2; ++e)
          *reinterpret_cast<float2 *>(o_s + (warp * G + hh) * D + lane * EPC + 2 * e) = o[hh][e];
    }
    if (lane == 0) {
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        m_s[warp * G + hh] = m_run[hh];
        l_s[warp * G + hh] = l_run[hh];
      }
    }
  }
};

// ============================================================ tensor-core math
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const void *p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_addr(p)));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], const void *p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_addr(p)));
}
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

template <typename T>
struct MmaType;
template <>
struct MmaType<__nv_bfloat16> {
  __device__ __forceinline__ static void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
  // pack (lo, hi) into one register, rounding to nearest even; also return what was kept
  __device__ __forceinline__ static uint32_t pack(float lo, float hi, float &klo, float &khi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    const uint32_t u = *reinterpret_cast<uint32_t *>(&v);
    klo = __uint_as_float(u << 16);
    khi = __uint_as_float(u & 0xffff0000u);
    return u;
  }
  __device__ __forceinline__ static uint32_t pack(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
  }
};
template <>
struct MmaType<__half> {
  __device__ __forceinline__ static void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
  __device__ __forceinline__ static uint32_t pack(float lo, float hi, float &klo, float &khi) {
    __half2 v = __floats2half2_rn(lo, hi);
    const float2 k = __half22float2(v);
    klo = k.x;
    khi = k.y;
    return *reinterpret_cast<uint32_t *>(&v);
  }
  __device__ __forceinline__ static uint32_t pack(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
  }
};

template <typename T, int G>
struct MmaMath {
  static_assert(G >= 2 && G <= 8, "the N = 8 side holds up to 8 query heads");
  static constexpr int D = 128;
  static constexpr int kScratchBytes = 0;
  static constexpr bool kNeedsQInSmem = false;
  static constexpr int kRowBytes = 256;
  static constexpr int kStagesPerWarp = pa::kStagesPerWarp;

  // Fragment roles (m16n8k16): gid = lane / 4 is the row group, tig = lane % 4.
  //   S^T / P^T: this lane holds tokens gid and gid+8 for heads 2*tig, 2*tig+1.
  //   O^T:       this lane holds d = 16*m + gid (+8) for heads 2*tig, 2*tig+1.
  uint32_t qf[8][2];    // Q^T fragments, one pair per 16-wide k-step of head_dim
  float m_run[2], l_run[2];
  float o[8][4];        // O^T accumulators, 8 m-tiles of 16 d
  int k_off[8];         // this lane's ldmatrix row address offsets for the K tile
  int v_off[8];         // ... and for the V tile

  __device__ static void stage_q(uint8_t *, const T *, float) {}

  __device__ void init(uint8_t *, const T *qg, float, int, int lane) {
    const int gid = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      if (gid < G) {
        const uint32_t *row = reinterpret_cast<const uint32_t *>(qg + gid * D + 16 * c + 2 * tig);
        qf[c][0] = row[0];
        qf[c][1] = row[4];   // + 8 elements
      } else {
        qf[c][0] = qf[c][1] = 0u;   // padding heads: zero query
      }
    }
    m_run[0] = m_run[1] = -INFINITY;
    l_run[0] = l_run[1] = 0.f;
#pragma unroll
    for (int m = 0; m < 8; ++m) o[m][0] = o[m][1] = o[m][2] = o[m][3] = 0.f;
    // ldmatrix: thread i addresses row (i % 8) of matrix (i / 8)
    const int mi = lane >> 3, ri = lane & 7;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      // K as the A operand of k-step c: matrices (t0-7, d lo), (t8-15, d lo), (t0-7, d hi), (t8-15, d hi)
      k_off[c] = tile_offset(ri + 8 * (mi & 1), 2 * c + (mi >> 1));
      // V^T as the A operand of m-tile c: (t0-7, d lo), (t0-7, d hi), (t8-15, d lo), (t8-15, d hi), transposed
      v_off[c] = tile_offset(ri + 8 * (mi >> 1), 2 * c + (mi & 1));
    }
  }

  __device__ void block(const uint8_t *tk, uint8_t *tv, int nvalid, int lane, float scale_log2) {
    const int gid = lane >> 2;
    // ---- S^T = K Q^T for the block's 16 tokens
    float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      uint32_t a[4];
      ldmatrix_x4(a, tk + k_off[c]);
      MmaType<T>::mma(s, a, qf[c][0], qf[c][1]);
    }
    const bool v0 = gid < nvalid, v1 = gid + 8 < nvalid;
    const float x0 = v0 ? s[0] * scale_log2 : -INFINITY;
    const float x1 = v0 ? s[1] * scale_log2 : -INFINITY;
    const float x2 = v1 ? s[2] * scale_log2 : -INFINITY;
    const float x3 = v1 ? s[3] * scale_log2 : -INFINITY;
    // block max per head over the 16 tokens (lanes with equal tig)
    float mb0 = fmaxf(x0, x2), mb1 = fmaxf(x1, x3);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      mb0 = fmaxf(mb0, __shfl_xor_sync(kFullMask, mb0, off));
      mb1 = fmaxf(mb1, __shfl_xor_sync(kFullMask, mb1, off));
    }
    const float mn0 = fmaxf(m_run[0], mb0), mn1 = fmaxf(m_run[1], mb1);
    if (__any_sync(kFullMask, mn0 != m_run[0] || mn1 != m_run[1])) {
      const float a0 = ex2(m_run[0] - mn0), a1 = ex2(m_run[1] - mn1);
      l_run[0] *= a0;
      l_run[1] *= a1;
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        o[m][0] *= a0;
        o[m][1] *= a1;
        o[m][2] *= a0;
        o[m][3] *= a1;
      }
      m_run[0] = mn0;
      m_run[1] = mn1;
    }
    const float p0 = ex2(x0 - mn0), p1 = ex2(x1 - mn1), p2 = ex2(x2 - mn0), p3 = ex2(x3 - mn1);
    l_run[0] += p0 + p2;
    l_run[1] += p1 + p3;

    // rows past the end hold anything: zero them so that 0 * V stays 0
    if (nvalid < kBlockSize) {
      uint4 *rows = reinterpret_cast<uint4 *>(tv);
      const int n = (kBlockSize - nvalid) * 8;   // 16-byte chunks per half
      for (int i = lane; i < 2 * n; i += 32) {
        const int half = i / n, k = i % n;
        rows[half * kBlockSize * 8 + nvalid * 8 + k] = make_uint4(0u, 0u, 0u, 0u);
      }
      __syncwarp();
    }

    // ---- P^T fragments: hi and lo 16-bit parts, transposed from the S^T layout
    float k0, k1, k2, k3;
    const uint32_t h01 = MmaType<T>::pack(p0, p1, k0, k1);
    const uint32_t h23 = MmaType<T>::pack(p2, p3, k2, k3);
    const uint32_t l01 = MmaType<T>::pack(p0 - k0, p1 - k1);
    const uint32_t l23 = MmaType<T>::pack(p2 - k2, p3 - k3);
    const uint32_t bh0 = movmatrix_trans(h01), bh1 = movmatrix_trans(h23);
    const uint32_t bl0 = movmatrix_trans(l01), bl1 = movmatrix_trans(l23);

    // ---- O^T += V^T P^T
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      uint32_t a[4];
      ldmatrix_x4_trans(a, tv + v_off[m]);
      MmaType<T>::mma(o[m], a, bh0, bh1);
      MmaType<T>::mma(o[m], a, bl0, bl1);
    }
  }

  __device__ void write_partials(float *o_s, float *m_s, float *l_s, int warp, int lane, float) {
    const int gid = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      float l = l_run[j];   // sum over the 8 lanes that hold other tokens of the same heads
      l += __shfl_xor_sync(kFullMask, l, 4);
      l += __shfl_xor_sync(kFullMask, l, 8);
      l += __shfl_xor_sync(kFullMask, l, 16);
      l_run[j] = l;
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int hh = 2 * tig + j;
      if (hh < G) {
        float *dst = o_s + (warp * G + hh) * D + gid;
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          dst[16 * m] = o[m][j];
          dst[16 * m + 8] = o[m][2 + j];
        }
        if (gid == 0) {
          m_s[warp * G + hh] = m_run[j];
          l_s[warp * G + hh] = l_run[j];
        }
      }
    }
  }
};

// ============================================================ tensor-core math, 1-byte E4M3 caches
// Two E4M3 codes (low byte first) -> f16x2 (low half first); exact: every E4M3
// value is an f16.
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t x, uint32_t &lo, uint32_t &hi) {
  asm("{\n .reg .b16 l, h;\n mov.b32 {l, h}, %2;\n cvt.rn.f16x2.e4m3x2 %0, l;\n cvt.rn.f16x2.e4m3x2 %1, h;\n}"
      : "=r"(lo), "=r"(hi)
      : "r"(x));
}

__device__ __forceinline__ uint32_t f16x2_from(float a, float b) {
  __half2 v = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Block math for 1-byte E4M3 caches (rows of 128 bytes, head_dim 128), q and
// out in T (fp16 or bf16).  Same transposed MMA problem as MmaMath, in f16:
//  * QK: ldmatrix of the code tile gives each lane 4 consecutive codes of one
//    token; converted they fill the A fragment with head_dim permuted inside
//    every 16-wide k-step (k-slots 2t,2t+1,2t+8,2t+9 <-> d 4t..4t+3), and the
//    Q^T fragments use the same permutation.
//  * PV: ldmatrix.trans of the code tile (16-bit units = code pairs) gives two
//    tokens x two d; one byte permute makes (token pair at d0 | token pair at
//    d1), so the V^T A fragment holds rows d = 16c + 2*gid and 16c + 2*gid + 1
//    (a row permutation of the output tile, undone in write_partials).
//  * scores carry k_scale (folded into scale_log2), outputs v_scale.
//  * P is one f16 (relative rounding 2^-12).
// q is converted to f16 once (exact for |q| in the f16 normal range).
template <typename T, int G>
struct Fp8MmaMath {
  static_assert(G >= 1 && G <= 8, "the N = 8 side holds up to 8 query heads");
  static constexpr int D = 128;
  static constexpr int kScratchBytes = 0;
  static constexpr bool kNeedsQInSmem = false;
  static constexpr int kRowBytes = 128;
  // three 4 KiB stages a warp: 48 KiB a CTA, so four CTAs share an SM (the
  // conversions want the warps more than the deeper prefetch: 7% faster on
  // B200 than four stages with three CTAs an SM)
  static constexpr int kStagesPerWarp = 3;

  uint32_t qf[8][2];
  float m_run[2], l_run[2];
  float o[8][4];
  int off[4];           // ldmatrix row offsets: chunks 2x, 2x+1 (tokens 0-7, 8-15)

  __device__ static void stage_q(uint8_t *, const T *, float) {}

  __device__ void init(uint8_t *, const T *qg, float, int, int lane) {
    const int gid = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      if (gid < G) {
        const T *q4 = qg + gid * D + 16 * c + 4 * tig;
        qf[c][0] = f16x2_from(Elem<T>::load(q4), Elem<T>::load(q4 + 1));
        qf[c][1] = f16x2_from(Elem<T>::load(q4 + 2), Elem<T>::load(q4 + 3));
      } else {
        qf[c][0] = qf[c][1] = 0u;
      }
    }
    m_run[0] = m_run[1] = -INFINITY;
    l_run[0] = l_run[1] = 0.f;
#pragma unroll
    for (int m = 0; m < 8; ++m) o[m][0] = o[m][1] = o[m][2] = o[m][3] = 0.f;
    const int mi = lane >> 3, ri = lane & 7;
#pragma unroll
    for (int x = 0; x < 4; ++x) off[x] = tile_offset(ri + 8 * (mi & 1), 2 * x + (mi >> 1));
  }

  __device__ void block(const uint8_t *tk, uint8_t *tv, int nvalid, int lane, float scale_log2) {
    const int gid = lane >> 2;
    float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      uint32_t r[4];
      ldmatrix_x4(r, tk + off[x]);   // r0/r1: chunk 2x tokens 0-7 / 8-15; r2/r3: chunk 2x+1
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        uint32_t a[4];
        e4m3x4_to_f16x2x2(r[2 * kk], a[0], a[2]);
        e4m3x4_to_f16x2x2(r[2 * kk + 1], a[1], a[3]);
        mma_f16(s, a, qf[2 * x + kk][0], qf[2 * x + kk][1]);
      }
    }
    const bool v0 = gid < nvalid, v1 = gid + 8 < nvalid;
    const float x0 = v0 ? s[0] * scale_log2 : -INFINITY;
    const float x1 = v0 ? s[1] * scale_log2 : -INFINITY;
    const float x2 = v1 ? s[2] * scale_log2 : -INFINITY;
    const float x3 = v1 ? s[3] * scale_log2 : -INFINITY;
    float mb0 = fmaxf(x0, x2), mb1 = fmaxf(x1, x3);
#pragma unroll
    for (int d = 4; d < 32; d <<= 1) {
      mb0 = fmaxf(mb0, __shfl_xor_sync(kFullMask, mb0, d));
      mb1 = fmaxf(mb1, __shfl_xor_sync(kFullMask, mb1, d));
    }
    const float mn0 = fmaxf(m_run[0], mb0), mn1 = fmaxf(m_run[1], mb1);
    if (__any_sync(kFullMask, mn0 != m_run[0] || mn1 != m_run[1])) {
      const float a0 = ex2(m_run[0] - mn0), a1 = ex2(m_run[1] - mn1);
      l_run[0] *= a0;
      l_run[1] *= a1;
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        o[m][0] *= a0;
        o[m][1] *= a1;
        o[m][2] *= a0;
        o[m][3] *= a1;
      }
      m_run[0] = mn0;
      m_run[1] = mn1;
    }
    const float p0 = ex2(x0 - mn0), p1 = ex2(x1 - mn1), p2 = ex2(x2 - mn0), p3 = ex2(x3 - mn1);
    l_run[0] += p0 + p2;
    l_run[1] += p1 + p3;

    if (nvalid < kBlockSize) {   // rows past the end: code 0 (+0) so that 0 * V stays 0
      uint4 *rows = reinterpret_cast<uint4 *>(tv);
      for (int i = nvalid * 8 + lane; i < kBlockSize * 8; i += 32) rows[i] = make_uint4(0u, 0u, 0u, 0u);
      __syncwarp();
    }
    const uint32_t b0 = movmatrix_trans(f16x2_from(p0, p1));
    const uint32_t b1 = movmatrix_trans(f16x2_from(p2, p3));
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      uint32_t r[4];
      ldmatrix_x4_trans(r, tv + off[x]);
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        // (token 2t: d0 d1 | token 2t+1: d0 d1) -> (d0: 2t 2t+1 | d1: 2t 2t+1)
        const uint32_t lo = __byte_perm(r[2 * kk], 0u, 0x3120);
        const uint32_t hi = __byte_perm(r[2 * kk + 1], 0u, 0x3120);
        uint32_t a[4];
        e4m3x4_to_f16x2x2(lo, a[0], a[1]);
        e4m3x4_to_f16x2x2(hi, a[2], a[3]);
        mma_f16(o[2 * x + kk], a, b0, b1);
      }
    }
  }

  __device__ void write_partials(float *o_s, float *m_s, float *l_s, int warp, int lane, float v_scale) {
    const int gid = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      float l = l_run[j];
      l += __shfl_xor_sync(kFullMask, l, 4);
      l += __shfl_xor_sync(kFullMask, l, 8);
      l += __shfl_xor_sync(kFullMask, l, 16);
      l_run[j] = l;
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int hh = 2 * tig + j;
      if (hh < G) {
        float *dst = o_s + (warp * G + hh) * D + 2 * gid;
#pragma unroll
        for (int m = 0; m < 8; ++m) {   // m-tile m rows: d = 16m + 2*gid (c0,c1) and 16m + 2*gid + 1 (c2,c3)
          dst[16 * m] = o[m][j] * v_scale;
          dst[16 * m + 1] = o[m][2 + j] * v_scale;
        }
        if (gid == 0) {
          m_s[warp * G + hh] = m_run[j];
          l_s[warp * G + hh] = l_run[j];
        }
      }
    }
  }
};

// ============================================================ shared memory plan
template <typename T, int G, typename Math, int W = kDecodeWarps>
struct DecodeSmem {
  static constexpr int D = Math::D;
  static constexpr int kTile = kBlockSize * Math::kRowBytes;        // one K or V tile
  static constexpr int kStages = W * Math::kStagesPerWarp;
  static constexpr int kTilesBytes = kStages * 2 * kTile;
  static constexpr int kScratchOff = kTilesBytes;
  static constexpr int kMOff = kScratchOff + Math::kScratchBytes;
  static constexpr int kLOff = kMOff + W * G * 4;
  static constexpr int kFlagOff = kLOff + W * G * 4;
  static constexpr int kBarOff = (kFlagOff + 8 + 7) / 8 * 8;   // abort flag, last-partition flag
  static constexpr int kBytes = kBarOff + kStages * 8;
  static constexpr int kAlloc = kBytes + 1024;   // room to align the base to 1024 B (128B swizzle atom)
  static_assert(W * G * D * 4 <= kTilesBytes, "epilogue buffer must fit in the stage tiles");
};

// ============================================================ split-K combine
// out = sum_p 2^(m_p - M) o_p / sum_p 2^(m_p - M) l_p over the nparts partials of
// the G heads h0 .. h0+G-1 of sequence b (M = max_p m_p; m_p base-2 maxima, o_p
// and l_p relative to m_p).  Run by one CTA of the partition kernel, the last
// to finish for that (sequence, KV head).  Same arithmetic as
// pa_decode_reduce_kernel (the summation order differs): per head, a
// lane-strided max and sum over the partitions joined by shuffles, then o
// accumulated over the partitions in order.  Partials are read through L2
// (.cg): other SMs wrote them.
template <typename T, int G, int D, int W>
__device__ __forceinline__ void combine_partitions(const DecodeParams &p, int b, int h0, int nparts, float *M_s,
                                                   float *inv_s, T *out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int hh = warp; hh < G; hh += W) {
    const size_t row = static_cast<size_t>(b) * p.num_heads + h0 + hh;
    const float *m = p.ws_m + row * p.max_partitions;
    const float *l = p.ws_l + row * p.max_partitions;
    float M = -INFINITY;
    for (int i = lane; i < nparts; i += 32) M = fmaxf(M, __ldcg(m + i));
    M = warp_max(M);
    float lsum = 0.f;
    for (int i = lane; i < nparts; i += 32) lsum += ex2(__ldcg(m + i) - M) * __ldcg(l + i);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) lsum += __shfl_xor_sync(kFullMask, lsum, off);
    if (lane == 0) {
      M_s[hh] = M;
      inv_s[hh] = 1.f / lsum;
    }
  }
  __syncthreads();
  for (int i = threadIdx.x * 4; i < G * D; i += W * 32 * 4) {
    const int hh = i / D, d = i % D;
    const size_t row = static_cast<size_t>(b) * p.num_heads + h0 + hh;
    const float *m = p.ws_m + row * p.max_partitions;
    const float *o = p.ws_o + row * p.max_partitions * D + d;
    const float M = M_s[hh];
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    int k = 0;
    for (; k + 8 <= nparts; k += 8) {   // eight partials in flight
      float w[8];
      float4 x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        w[u] = __ldcg(m + k + u);
        x[u] = __ldcg(reinterpret_cast<const float4 *>(o + static_cast<size_t>(k + u) * D));
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float wk = ex2(w[u] - M);
        acc.x += wk * x[u].x;
        acc.y += wk * x[u].y;
        acc.z += wk * x[u].z;
        acc.w += wk * x[u].w;
      }
    }
    for (; k < nparts; ++k) {
      const float wk = ex2(__ldcg(m + k) - M);
      const float4 x = __ldcg(reinterpret_cast<const float4 *>(o + static_cast<size_t>(k) * D));
      acc.x += wk * x.x;
      acc.y += wk * x.y;
      acc.z += wk * x.z;
      acc.w += wk * x.w;
    }
    const float inv = inv_s[hh];
    Elem<T>::store4(out + i, acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  }
}

// Zero the per-(sequence, KV head) partition counters of a split call; launched
// (programmatically) just before the partition kernel of the same call.
__global__ void __launch_bounds__(256) zero_counts_kernel(unsigned *count, int n) {
  pdl_wait();   // the previous kernel in the stream (which may use the same workspace) is done
  pdl_trigger();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) count[i] = 0u;
}

// ============================================================ partition kernel
// Resident CTAs an SM the register budget is sized for: four-warp CTAs (the
// default launch shape), or six of the two-warp shape.
constexpr int decode_min_ctas(int warps) { return warps == 2 ? 6 : PA_DECODE_MIN_CTAS_PER_SM; }

template <typename T, int G, typename Math, int W = kDecodeWarps>
__global__ void __launch_bounds__(W * 32, decode_min_ctas(W))
    pa_decode_partition_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                               const DecodeParams p) {
  static_assert(!Math::kNeedsQInSmem || W == kDecodeWarps, "the CUDA-core block math stages q with kDecodeWarps warps");
  using SM = DecodeSmem<T, G, Math, W>;
  constexpr int D = SM::D;
  constexpr int kTile = SM::kTile;
  constexpr int kStages = SM::kStages;
  constexpr int kSPW = Math::kStagesPerWarp;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *scratch = smem + SM::kScratchOff;
  float *m_s = reinterpret_cast<float *>(smem + SM::kMOff);
  float *l_s = reinterpret_cast<float *>(smem + SM::kLOff);
  int *abort_s = reinterpret_cast<int *>(smem + SM::kFlagOff);
  int *last_s = abort_s + 1;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + SM::kBarOff);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const unsigned long long wait_limit = wait_limit_for(p.stall_cta, blockIdx.x);
  const bool stall_here = p.stall_cta != 0 && static_cast<int>(blockIdx.x) == p.stall_cta - 1;
  pdl_wait();      // the previous kernel's writes (caches, inputs) are visible from here on
  pdl_trigger();   // the reduce kernel may be scheduled once every CTA of this grid has started

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
      for (int i = threadIdx.x * 4; i < G * D; i += (W * 32) * 4) Elem<T>::store4(out + i, 0.f, 0.f, 0.f, 0.f);
    return;
  }
  if (part >= nparts) return;
  const int tok0 = part * P;
  const int tok1 = min(tok0 + P, L);
  const int nblk = (tok1 - tok0 + kBlockSize - 1) / kBlockSize;
  const T *qg = reinterpret_cast<const T *>(p.q) + (static_cast<size_t>(b) * p.num_heads + h0) * D;

  if (threadIdx.x == 0) {
    prefetch_tensor_map(&tm_k);
    prefetch_tensor_map(&tm_v);
    for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
    *abort_s = 0;
  }

  // ---- this warp's blocks: local block index warp + j * W, j = 0 .. nw-1
  const int nw = nblk > warp ? (nblk - warp + W - 1) / W : 0;
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
        const int id = bt_row[warp + jj * W];
        if (id < 0 || id >= p.num_blocks) record_error(1 /*PA_DEV_BAD_BLOCK_ID*/, id);
        else my_id = id;
      }
    }
    const int id = __shfl_sync(kFullMask, my_id, j & 31);
    const int s = warp + (j % kSPW) * W;
    if (lane == 0 && !(stall_here && warp == 0 && j == 0)) {   // (test hook: warp 0's first stage left unissued)
      if (id >= 0) {
        // one box per 128-byte part of the rows: the tile lands as [part][token][128 B]
        uint8_t *tk = smem + s * 2 * kTile;
        mbar_arrive_expect_tx(&full[s], 2 * kTile);
#pragma unroll
        for (int part = 0; part < Math::kRowBytes / 128; ++part) {
          tma_load_5d(tk + part * 2048, &tm_k, 0, part, g, 0, id, &full[s], policy);
          tma_load_5d(tk + kTile + part * 2048, &tm_v, 0, part, g, 0, id, &full[s], policy);
        }
      } else {
        mbar_arrive(&full[s]);   // bad id: recorded above; complete the phase without data
      }
    }
  };

  if constexpr (Math::kNeedsQInSmem) Math::stage_q(scratch, qg, p.scale_log2);
  __syncthreads();   // barriers initialised (and q staged)

  for (int j = 0; j < min(nw, kSPW); ++j) issue(j);

  Math math;
  math.init(scratch, qg, p.scale_log2, warp, lane);

  bool ok = true;
  int j = 0;
  for (; j < nw; ++j) {
    const int s = warp + (j % kSPW) * W;
    const bool landed = mbar_wait(&full[s], (j / kSPW) & 1, wait_limit);
    if (!__all_sync(kFullMask, landed)) {
      if (lane == 0) {
        record_error(5 /*PA_DEV_WAIT_TIMEOUT*/, blockIdx.x);
        *abort_s = 1;
      }
      ok = false;
      break;
    }
    uint8_t *tk = smem + s * 2 * kTile;
    const int lb = warp + j * W;   // local block index
    const int nvalid = min(kBlockSize, tok1 - (tok0 + lb * kBlockSize));
    if (Math::kRowBytes == 256 && p.new_k != nullptr && part == nparts - 1 && lb == nblk - 1) {
      // append mode: this block holds position L-1.  Store the new token's K/V
      // rows of head g in the cache and put them into the tile that just landed
      // (its copy of that row may predate the store).  Lanes 0-15 move the 16
      // chunks of the K row, lanes 16-31 those of the V row.
      const int t_new = (L - 1) % kBlockSize;
      const int c = lane & 15;
      const bool is_v = lane >= 16;
      const uint4 *src = reinterpret_cast<const uint4 *>(is_v ? p.new_v : p.new_k) +
                         (static_cast<size_t>(b) * p.num_kv_heads + g) * kChunksPerRow + c;
      const uint4 x = *src;
      const int id = bt_row[lb];
      if (id >= 0 && id < p.num_blocks) {
        uint4 *dst = reinterpret_cast<uint4 *>(is_v ? p.v_cache : p.k_cache) +
                     ((static_cast<size_t>(id) * kBlockSize + t_new) * p.num_kv_heads + g) * kChunksPerRow + c;
        *dst = x;
      }
      *reinterpret_cast<uint4 *>(tk + (is_v ? kTile : 0) + tile_offset(t_new, c)) = x;
      __syncwarp();
    }
    math.block(tk, tk + kTile, nvalid, lane, p.scale_log2);
    __syncwarp();   // all lanes done with the stage
    if (j + kSPW < nw) {
      fence_proxy_async_smem();
      issue(j + kSPW);
    }
  }
  if (!ok) {
    // let this warp's copies in flight land (bounded) before the CTA can exit:
    // the stages of blocks j .. j + kSPW - 1, the one that timed out included
    // (its copy may still arrive)
    for (int jj = j; jj < min(nw, j + kSPW); ++jj)
      mbar_wait(&full[warp + (jj % kSPW) * W], (jj / kSPW) & 1, wait_limit);
  }

  // ---- merge the warps through shared memory (the stage tiles are reused)
  __syncthreads();
  float *o_s = reinterpret_cast<float *>(smem);
  math.write_partials(o_s, m_s, l_s, warp, lane, p.v_scale);
  __syncthreads();
  if (*abort_s) return;

  for (int i = threadIdx.x * 4; i < G * D; i += (W * 32) * 4) {
    const int hh = i / D, d = i % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < W; ++w) M = fmaxf(M, m_s[w * G + hh]);
    float lsum = 0.f;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < W; ++w) {
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
  if (nparts == 1 || p.ws_count == nullptr) return;

  // ---- split sequence: the last of its nparts CTAs (per KV head) combines the
  // partials.  Publish this CTA's partial, then take a ticket; no CTA waits for
  // another, and the ticket that completes the count goes to exactly one CTA.
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0)
    *last_s = atomicAdd(p.ws_count + static_cast<size_t>(b) * p.num_kv_heads + g, 1u) == static_cast<unsigned>(nparts - 1);
  __syncthreads();
  if (!*last_s) return;
  __threadfence();   // the other CTAs' partials (published before their tickets) are visible from here on
  combine_partitions<T, G, D, W>(p, b, h0, nparts, m_s, l_s, out);
}

// Combine the partitions of every (sequence, query head) that was split:
//   M = max_p m_p,  out = sum_p 2^(m_p - M) o_p / sum_p 2^(m_p - M) l_p
// (m_p are base-2 log-domain maxima; o_p and l_p are relative to m_p).
// A CTA of kReduceWarps warps takes kReduceWarps / wpr rows at a time (grid
// stride); the wpr warps of a row split its partitions (warp k takes k, k + wpr,
// ...), each with all of its partials' loads in flight, and join their sums
// through shared memory.  wpr grows with the number of partitions (the host
// picks it), so a row of 64 partials is read by 8 warps at once instead of one.
// Lane l owns outputs [l*D/32, (l+1)*D/32): each partial vector is one
// coalesced row read.
constexpr int kReduceWarps = 8;
constexpr int kReduceBatch = 8;   // partials in flight per warp

template <typename T>
__global__ void __launch_bounds__(kReduceWarps * 32) pa_decode_reduce_kernel(const DecodeParams p, int wpr) {
  constexpr int D = kChunksPerRow * Elem<T>::kPerChunk;
  constexpr int PER_LANE = D / 32;
  __shared__ float acc_s[kReduceWarps][D];
  __shared__ float l_s[kReduceWarps];
  pdl_wait();   // the partition kernel's partials are visible from here on
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows_per_cta = kReduceWarps / wpr;
  const int sub = warp % wpr;    // this warp's share of the row's partitions
  const int rloc = warp / wpr;   // which of the CTA's rows
  const long long rows = static_cast<long long>(p.num_seqs) * p.num_heads;
  for (long long row0 = static_cast<long long>(blockIdx.x) * rows_per_cta; row0 < rows;
       row0 += static_cast<long long>(gridDim.x) * rows_per_cta) {   // CTA-uniform
    const long long row = row0 + rloc;
    int np = 0;
    if (row < rows) {
      const int b = static_cast<int>(row / p.num_heads);
      const int L = p.context_lens[b];
      if (L >= 0 && L <= p.max_context_len && L <= p.max_blocks_per_seq * kBlockSize)
        np = (L + p.partition_size - 1) / p.partition_size;
    }
    const bool split = np > 1;   // else finished by the partition kernel
    float lsum = 0.f;
    float acc[PER_LANE];
#pragma unroll
    for (int e = 0; e < PER_LANE; ++e) acc[e] = 0.f;
    if (split) {
      const float *m = p.ws_m + row * p.max_partitions;
      const float *l = p.ws_l + row * p.max_partitions;
      const float *o = p.ws_o + row * p.max_partitions * D + lane * PER_LANE;
      float M = -INFINITY;
      for (int i = lane; i < np; i += 32) M = fmaxf(M, m[i]);
      M = warp_max(M);
      for (int i0 = sub; i0 < np; i0 += kReduceBatch * wpr) {
        // the batch's m and l: lane u < kReduceBatch loads those of partition
        // i0 + u * wpr, then they are broadcast -- no thread reads two adjacent
        // partials, so no load of them can be merged into a wider one (a row's
        // m and l start only 4 * NP-byte aligned)
        const int iu = i0 + (lane % kReduceBatch) * wpr;
        const float m_u = lane < kReduceBatch && iu < np ? m[iu] : -INFINITY;
        const float l_u = lane < kReduceBatch && iu < np ? l[iu] : 0.f;
        float w[kReduceBatch], li[kReduceBatch], x[kReduceBatch][PER_LANE];
#pragma unroll
        for (int u = 0; u < kReduceBatch; ++u) {   // every load of the batch in flight
          const int i = i0 + u * wpr;
          w[u] = __shfl_sync(kFullMask, m_u, u);
          li[u] = __shfl_sync(kFullMask, l_u, u);
          const float *src = o + static_cast<size_t>(i < np ? i : 0) * D;
          if constexpr (PER_LANE == 4) {
            const float4 v = *reinterpret_cast<const float4 *>(src);
            x[u][0] = v.x; x[u][1] = v.y; x[u][2] = v.z; x[u][3] = v.w;
          } else {
            const float2 v = *reinterpret_cast<const float2 *>(src);
            x[u][0] = v.x; x[u][1] = v.y;
          }
        }
#pragma unroll
        for (int u = 0; u < kReduceBatch; ++u) {
          const float wk = ex2(w[u] - M);   // 0 past the end (m = -inf)
          lsum += wk * li[u];
#pragma unroll
          for (int e = 0; e < PER_LANE; ++e) acc[e] += wk * x[u][e];
        }
      }
    }
    if (wpr > 1) {   // join the row's warps
#pragma unroll
      for (int e = 0; e < PER_LANE; ++e) acc_s[warp][lane * PER_LANE + e] = acc[e];
      if (lane == 0) l_s[warp] = lsum;
      __syncthreads();
      if (sub == 0 && split) {
        for (int k = 1; k < wpr; ++k) {
          lsum += l_s[warp + k];
#pragma unroll
          for (int e = 0; e < PER_LANE; ++e) acc[e] += acc_s[warp + k][lane * PER_LANE + e];
        }
      }
      __syncthreads();   // acc_s is rewritten by the next rows
    }
    if (sub == 0 && split) {
      const float inv = 1.f / lsum;
      T *out = reinterpret_cast<T *>(p.out) + row * D + lane * PER_LANE;
      if constexpr (PER_LANE == 4) {
        Elem<T>::store4(out, acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
      } else {
        Elem<T>::store2(out, acc[0] * inv, acc[1] * inv);
      }
    }
  }
}

}  // namespace pa
