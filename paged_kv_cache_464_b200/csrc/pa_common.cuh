// pa_common.cuh -- device helpers shared by the paged-KV kernels (sm_100a).
//
// mbarrier / TMA wrappers are inline PTX from the PTX ISA (mbarrier.*,
// cp.async.bulk.tensor.*, fence.proxy.async); nothing here is specific to
// attention.  Included only from pa.cu (one translation unit).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace pa {

constexpr int kBlockSize = 16;    // tokens per KV block (the pages' default; the only size built)
constexpr int kRowBytes = 256;    // bytes of one (token, KV head) row: head_dim * element bytes
constexpr int kChunksPerRow = kRowBytes / 16;
constexpr int kTileBytes = kBlockSize * kRowBytes;   // one block of one KV head: 4 KiB
constexpr unsigned kFullMask = 0xffffffffu;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // bounded waits give up after 2 s

// ---------------------------------------------------------------- error word
// One per device.  The first problem a kernel meets is kept until cleared.
__device__ int g_error_code;
__device__ long long g_error_detail;

__device__ __forceinline__ void record_error(int code, long long detail) {
  if (atomicCAS(&g_error_code, 0, code) == 0) {
    g_error_detail = detail;
    __threadfence();
  }
}

// ---------------------------------------------------------------- smem / mbarrier
__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for phase `parity` of `bar` to complete; false if it has not after
// `limit_ns` (kWaitLimitNs unless a test shortens it for one CTA).
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity,
                                          unsigned long long limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0 && global_ns() - t0 > limit_ns) return false;
  }
}

// Non-blocking: has phase `parity` of `bar` completed?
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Bounded wait (`limit_ns`) that also gives up once another role has raised
// the abort flag.  With `backoff` the waiting warp sleeps between polls,
// leaving the shared memory ports (which also feed the tensor cores' operands)
// to others.
__device__ __forceinline__ bool mbar_wait_or_abort(uint64_t *bar, uint32_t parity, const volatile int *abort_flag,
                                                   unsigned long long limit_ns, bool backoff = false) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (backoff) __nanosleep(64);
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0 && (*abort_flag || global_ns() - t0 > limit_ns)) return false;
  }
}

// Test hook for the bounded-wait error path.  A kernel launched with
// stall_cta = c + 1 (0 = off, the value of every ordinary launch) treats its CTA
// c specially: that CTA leaves one of its copies unissued -- no copy and no
// barrier arrival, so nothing is in flight for that stage -- and its waits give
// up after kTestWaitLimitNs instead of kWaitLimitNs.  The wait on the missing
// stage therefore runs out, and the CTA takes the same abort path a real
// timeout would.  Every other CTA runs as usual.
constexpr unsigned long long kTestWaitLimitNs = 1000000ull;   // 1 ms

__device__ __forceinline__ unsigned long long wait_limit_for(int stall_cta, long long cta) {
  return stall_cta != 0 && cta == stall_cta - 1 ? kTestWaitLimitNs : kWaitLimitNs;
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void prefetch_tensor_map(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// 5-D tiled bulk tensor load global -> this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_5d(void *dst, const CUtensorMap *map, int c0, int c1, int c2, int c3,
                                            int c4, uint64_t *bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7], %8;" ::"r"(smem_addr(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

// Same, with the default L2 policy (data that other CTAs read again).
__device__ __forceinline__ void tma_load_5d(void *dst, const CUtensorMap *map, int c0, int c1, int c2, int c3,
                                            int c4, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(smem_addr(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(smem_addr(bar))
      : "memory");
}

// L2 policy for data read exactly once (the KV stream).
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Order this thread's earlier generic-proxy shared-memory accesses before later
// async-proxy (TMA) accesses to the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- launch ordering
// Programmatic dependent launch: kernels are launched so that the next kernel
// in the stream may start before this one ends.  Each kernel calls pdl_wait()
// before its first global-memory access (it returns once the previous grid in
// the stream has completed and its writes are visible; a no-op when launched
// without the attribute), and pdl_trigger() to let its successor launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------- math
__device__ __forceinline__ float ex2(float x) {   // 2^x; ex2(-inf) = +0
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float warp_max(float x) {   // over all 32 lanes
  float y;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(y) : "f"(x));
  return y;
}

// ---------------------------------------------------------------- element types
// Unpack one 16-byte chunk of a row into fp32 values; pack fp32 back.
template <typename T>
struct Elem;

template <>
struct Elem<float> {
  static constexpr int kPerChunk = 4;
  __device__ __forceinline__ static void unpack(const uint4 &v, float *f) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
  }
  __device__ __forceinline__ static float load(const float *p) { return *p; }
  __device__ __forceinline__ static void store4(float *p, float a, float b, float c, float d) {
    *reinterpret_cast<float4 *>(p) = make_float4(a, b, c, d);
  }
  __device__ __forceinline__ static void store2(float *p, float a, float b) {
    *reinterpret_cast<float2 *>(p) = make_float2(a, b);
  }
  __device__ __forceinline__ static void store1(float *p, float a) { *p = a; }
};

template <>
struct Elem<__nv_bfloat16> {
  static constexpr int kPerChunk = 8;
  __device__ __forceinline__ static void unpack(const uint4 &v, float *f) {
    // a bf16 is the high half of an fp32: widening is exact
    f[0] = __uint_as_float(v.x << 16);
    f[1] = __uint_as_float(v.x & 0xffff0000u);
    f[2] = __uint_as_float(v.y << 16);
    f[3] = __uint_as_float(v.y & 0xffff0000u);
    f[4] = __uint_as_float(v.z << 16);
    f[5] = __uint_as_float(v.z & 0xffff0000u);
    f[6] = __uint_as_float(v.w << 16);
    f[7] = __uint_as_float(v.w & 0xffff0000u);
  }
  __device__ __forceinline__ static float load(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
  __device__ __forceinline__ static void store4(__nv_bfloat16 *p, float a, float b, float c, float d) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(a, b);
    __nv_bfloat162 hi = __floats2bfloat162_rn(c, d);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t *>(&lo);
    u.y = *reinterpret_cast<uint32_t *>(&hi);
    *reinterpret_cast<uint2 *>(p) = u;
  }
  __device__ __forceinline__ static void store2(__nv_bfloat16 *p, float a, float b) {
    *reinterpret_cast<__nv_bfloat162 *>(p) = __floats2bfloat162_rn(a, b);
  }
  __device__ __forceinline__ static void store1(__nv_bfloat16 *p, float a) { *p = __float2bfloat16_rn(a); }
};

template <>
struct Elem<__half> {
  static constexpr int kPerChunk = 8;
  __device__ __forceinline__ static void unpack(const uint4 &v, float *f) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __half2 h = *reinterpret_cast<const __half2 *>(&w[i]);
      float2 x = __half22float2(h);
      f[2 * i] = x.x;
      f[2 * i + 1] = x.y;
    }
  }
  __device__ __forceinline__ static float load(const __half *p) { return __half2float(*p); }
  __device__ __forceinline__ static void store4(__half *p, float a, float b, float c, float d) {
    __half2 lo = __floats2half2_rn(a, b);
    __half2 hi = __floats2half2_rn(c, d);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t *>(&lo);
    u.y = *reinterpret_cast<uint32_t *>(&hi);
    *reinterpret_cast<uint2 *>(p) = u;
  }
  __device__ __forceinline__ static void store2(__half *p, float a, float b) {
    *reinterpret_cast<__half2 *>(p) = __floats2half2_rn(a, b);
  }
  __device__ __forceinline__ static void store1(__half *p, float a) { *p = __float2half_rn(a); }
};

}  // namespace pa
