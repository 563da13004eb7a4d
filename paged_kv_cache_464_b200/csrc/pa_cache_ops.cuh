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
// blockIdx.x = pair, blockIdx.y = 0 for the K cache, 1 for the V cache.
// Every CTA first checks its pair against all pairs (conflicting pairs are
// skipped, as are out-of-range ids), then copies one whole block.
__global__ void __launch_bounds__(256) copy_blocks_kernel(uint4 *__restrict__ k_cache, uint4 *__restrict__ v_cache,
                                                          const long long *__restrict__ block_mapping,
                                                          int num_pairs, long long num_blocks,
                                                          int chunks_per_block) {
  pdl_wait();
  pdl_trigger();
  const int pair = blockIdx.x;
  const long long src = block_mapping[2 * pair];
  const long long dst = block_mapping[2 * pair + 1];
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (threadIdx.x == 0 && blockIdx.y == 0) record_error(1 /*PA_DEV_BAD_BLOCK_ID*/, src < 0 || src >= num_blocks ? src : dst);
    return;
  }
  int conflict = 0;
  for (int j = threadIdx.x; j < num_pairs; j += blockDim.x) {
    const long long sj = block_mapping[2 * j], dj = block_mapping[2 * j + 1];
    conflict |= (j != pair && dj == dst) || sj == dst;
  }
  if (__syncthreads_or(conflict)) {
    if (threadIdx.x == 0 && blockIdx.y == 0) record_error(3 /*PA_DEV_COPY_CONFLICT*/, pair);
    return;
  }
  uint4 *cache = blockIdx.y == 0 ? k_cache : v_cache;
  const uint4 *s = cache + src * chunks_per_block;
  uint4 *d = cache + dst * chunks_per_block;
  for (int i = threadIdx.x; i < chunks_per_block; i += blockDim.x) d[i] = s[i];
}

}  // namespace pa
