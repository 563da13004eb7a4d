// pa_probe.cuh -- a plain streaming read of a device buffer, used to measure
// the read-only HBM bandwidth of the GPU (the decode kernels only read the KV
// cache, while the usual bandwidth figure comes from a copy, which reads and
// writes).  No counterpart on the source pages.  Included only from pa.cu.
#pragma once

#include "pa_common.cuh"

namespace pa {

constexpr int kProbeThreads = 256;
constexpr int kProbeUnroll = 8;   // 16-byte loads in flight per thread

// XOR of every 8-byte word of buf[0 .. n16 * 16) into *sink (so the loads
// cannot be dropped, and a test can check that every byte was read once).
__global__ void __launch_bounds__(kProbeThreads) stream_read_kernel(const uint4 *__restrict__ buf, long long n16,
                                                                    unsigned long long *sink) {
  pdl_wait();
  pdl_trigger();
  unsigned long long acc = 0;
  const long long stride = static_cast<long long>(gridDim.x) * kProbeThreads;
  long long i = static_cast<long long>(blockIdx.x) * kProbeThreads + threadIdx.x;
  for (; i + (kProbeUnroll - 1) * stride < n16; i += kProbeUnroll * stride) {
    uint4 x[kProbeUnroll];
#pragma unroll
    for (int u = 0; u < kProbeUnroll; ++u) x[u] = __ldcs(buf + i + u * stride);
#pragma unroll
    for (int u = 0; u < kProbeUnroll; ++u)
      acc ^= (static_cast<unsigned long long>(x[u].y) << 32 | x[u].x) ^ (static_cast<unsigned long long>(x[u].w) << 32 | x[u].z);
  }
  for (; i < n16; i += stride) {
    const uint4 x = __ldcs(buf + i);
    acc ^= (static_cast<unsigned long long>(x.y) << 32 | x.x) ^ (static_cast<unsigned long long>(x.w) << 32 | x.z);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc ^= __shfl_xor_sync(kFullMask, acc, off);
  if ((threadIdx.x & 31) == 0 && acc != 0) atomicXor(sink, acc);
}

}  // namespace pa
