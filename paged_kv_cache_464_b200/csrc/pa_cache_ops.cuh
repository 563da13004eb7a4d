// pa_cache_ops.cuh -- the new token's slot write and the copy-on-write block
// copy.  Both are pure byte movement in 16-byte vectors; no arithmetic on the
// data.  Included only from pa.cu.
#pragma once

#include "pa_common.cuh"

namespace pa {

// Slot write of each new token's K/V rows ("vLLM推理引擎深度解析", §五: the
// current token's k/v join the cache; §三 append_token chooses the slot).
// One thread moves one 16-byte chunk of one row of K and the same chunk of V.
// Row (token i, head h) -> cache row (slot_i, h), i.e. chunk index
// slot * chunks_per_slot + h * 16 + c in the [NB*bs][Hkv][16 chunks] view.
__global__ void __launch_bounds__(256) reshape_and_cache_kernel(const uint4 *__restrict__ key,
                                                                const uint4 *__restrict__ value,
                                                                uint4 *__restrict__ k_cache,
                                                                uint4 *__restrict__ v_cache,
                                                                const int64_t *__restrict__ slot_mapping,
                                                                int num_tokens, int chunks_per_slot,
                                                                long long num_slots) {
  pdl_wait();
  pdl_trigger();
  const long long total = static_cast<long long>(num_tokens) * chunks_per_slot;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
    const int tok = static_cast<int>(i / chunks_per_slot);
    const int rem = static_cast<int>(i - static_cast<long long>(tok) * chunks_per_slot);
    const uint4 kx = key[i];   // issued before the slot load so the latencies overlap
    const uint4 vx = value[i];
    const long long slot = slot_mapping[tok];
    if (slot < 0) continue;   // padding token: nothing to write
    if (slot >= num_slots) {
      if (rem == 0) record_error(2 /*PA_DEV_BAD_SLOT*/, slot);
      continue;
    }
    const long long dst = slot * chunks_per_slot + rem;
    k_cache[dst] = kx;
    v_cache[dst] = vx;
  }
}

// Slot write into 1-byte E4M3 caches: each stored code is the E4M3 value
// nearest to the fp32 quotient x / scale (IEEE division), ties to even,
// saturating at +-448 (cvt.rn.satfinite).  One thread converts 8 elements (one
// 16-byte chunk of a 16-bit source row) into 8 codes.
template <typename T>
__global__ void __launch_bounds__(256) reshape_and_cache_fp8_kernel(const uint4 *__restrict__ key,
                                                                    const uint4 *__restrict__ value,
                                                                    uint2 *__restrict__ k_cache,
                                                                    uint2 *__restrict__ v_cache,
                                                                    const int64_t *__restrict__ slot_mapping,
                                                                    int num_tokens, int chunks_per_slot,
                                                                    long long num_slots, float k_scale,
                                                                    float v_scale) {
  pdl_wait();
  pdl_trigger();
  const long long total = static_cast<long long>(num_tokens) * chunks_per_slot;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
    const int tok = static_cast<int>(i / chunks_per_slot);
    const int rem = static_cast<int>(i - static_cast<long long>(tok) * chunks_per_slot);
    const uint4 kx = key[i];
    const uint4 vx = value[i];
    const long long slot = slot_mapping[tok];
    if (slot < 0) continue;
    if (slot >= num_slots) {
      if (rem == 0) record_error(2 /*PA_DEV_BAD_SLOT*/, slot);
      continue;
    }
    float kf[8], vf[8];
    Elem<T>::unpack(kx, kf);
    Elem<T>::unpack(vx, vf);
    uint32_t kc[4], vc[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint16_t a, b;
      // cvt packs its first source into the upper byte: element 2j goes low
      asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(a) : "f"(kf[2 * j + 1] / k_scale), "f"(kf[2 * j] / k_scale));
      asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(b) : "f"(vf[2 * j + 1] / v_scale), "f"(vf[2 * j] / v_scale));
      kc[j] = a;
      vc[j] = b;
    }
    const long long dst = slot * chunks_per_slot + rem;
    k_cache[dst] = make_uint2(kc[0] | (kc[1] << 16), kc[2] | (kc[3] << 16));
    v_cache[dst] = make_uint2(vc[0] | (vc[1] << 16), vc[2] | (vc[3] << 16));
  }
}

// Copy-on-write block copy ("vLLM 原理与源码阅读", Block 管理器, item 3).
// blockIdx.y = 0 for the K cache, 1 for the V cache; CTA x takes the pairs
// x, x + gridDim.x, ... (at most kCopyMaxPairsPerCta of them).  A pair is
// skipped when an id is out of range or when its dst is the dst of another pair
// or the src of any pair (the set of pairs decides, not their order).  The
// check streams all pairs once through shared memory in chunks of
// kCopyChunkPairs and compares them with this CTA's own pairs there: each CTA
// reads the mapping once (num_pairs x 16 bytes, from L2) and does
// (its pairs) x num_pairs comparisons in shared memory, so the whole check is
// num_pairs^2 shared-memory comparisons and gridDim x num_pairs x 16 bytes of
// reads.  Then each CTA copies its non-skipped blocks.
constexpr int kCopyThreads = 256;
constexpr int kCopyChunkPairs = 1024;      // pairs staged in shared memory at a time (16 KiB)
constexpr int kCopyMaxPairsPerCta = 256;   // with PA_MAX_COPY_PAIRS = 65536: at least 256 CTAs

__global__ void __launch_bounds__(kCopyThreads) copy_blocks_kernel(uint4 *__restrict__ k_cache,
                                                                   uint4 *__restrict__ v_cache,
                                                                   const longlong2 *__restrict__ block_mapping,
                                                                   int num_pairs, long long num_blocks,
                                                                   int chunks_per_block) {
  __shared__ longlong2 chunk[kCopyChunkPairs];
  __shared__ long long mine_dst[kCopyMaxPairsPerCta];
  __shared__ int mine_bad[kCopyMaxPairsPerCta];    // an id out of range
  __shared__ int mine_conf[kCopyMaxPairsPerCta];   // dst repeated or read by a pair
  pdl_wait();
  pdl_trigger();
  const int n_mine = (num_pairs - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1;
  for (int m = threadIdx.x; m < n_mine; m += kCopyThreads) {
    const longlong2 pr = block_mapping[blockIdx.x + static_cast<long long>(m) * gridDim.x];
    const bool bad = pr.x < 0 || pr.x >= num_blocks || pr.y < 0 || pr.y >= num_blocks;
    mine_dst[m] = pr.y;
    mine_bad[m] = bad ? 1 : 0;
    mine_conf[m] = 0;
    if (bad && blockIdx.y == 0) record_error(1 /*PA_DEV_BAD_BLOCK_ID*/, pr.x < 0 || pr.x >= num_blocks ? pr.x : pr.y);
  }
  for (int c0 = 0; c0 < num_pairs; c0 += kCopyChunkPairs) {
    const int n = min(kCopyChunkPairs, num_pairs - c0);
    __syncthreads();   // the previous chunk's comparisons are done (and mine_* are written)
    for (int e = threadIdx.x; e < n; e += kCopyThreads) chunk[e] = block_mapping[c0 + e];
    __syncthreads();
    for (int e = threadIdx.x; e < n; e += kCopyThreads) {
      const long long src = chunk[e].x, dst = chunk[e].y;
      const int pair_e = c0 + e;
      for (int m = 0; m < n_mine; ++m) {
        const long long d = mine_dst[m];
        const int pair_m = static_cast<int>(blockIdx.x) + m * static_cast<int>(gridDim.x);
        if (src == d || (dst == d && pair_e != pair_m)) mine_conf[m] = 1;   // every writer writes 1
      }
    }
  }
  __syncthreads();
  uint4 *cache = blockIdx.y == 0 ? k_cache : v_cache;
  for (int m = 0; m < n_mine; ++m) {
    const long long pair = blockIdx.x + static_cast<long long>(m) * gridDim.x;
    if (mine_bad[m]) continue;   // recorded above
    if (mine_conf[m]) {
      if (threadIdx.x == 0 && blockIdx.y == 0) record_error(3 /*PA_DEV_COPY_CONFLICT*/, pair);
      continue;
    }
    const longlong2 pr = block_mapping[pair];
    const uint4 *s = cache + pr.x * chunks_per_block;
    uint4 *d = cache + pr.y * chunks_per_block;
    for (int i = threadIdx.x; i < chunks_per_block; i += kCopyThreads) d[i] = s[i];
  }
}

}  // namespace pa
