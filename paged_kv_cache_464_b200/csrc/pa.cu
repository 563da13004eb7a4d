// pa.cu -- the C ABI of libpa_b200.so (declared in include/pa.h): host-side
// argument checks, TMA descriptor encoding and kernel launches.  The kernels
// themselves live in pa_cache_ops.cuh, pa_decode.cuh and pa_prefill.cuh, compiled here as one
// translation unit so that the per-device error word needs no separate
// device linking.
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <type_traits>
#include <utility>

#include "pa.h"
#include "pa_cache_ops.cuh"
#include "pa_decode.cuh"
#include "pa_prefill.cuh"
#include "pa_decode_fp8tc.cuh"
#include "pa_probe.cuh"

#ifndef PA_PROGRAMMATIC_LAUNCH
#define PA_PROGRAMMATIC_LAUNCH 1
#endif
// Split sequences: 0 = a separate reduce kernel after the partition kernel
// (the default); 1 = the last partition CTA of each (sequence, KV head)
// combines the partials (one launch, plus a tiny counter-zeroing kernel).
// Measured on B200 the fused form is no faster on the GQA workload and ~5%
// slower on the long-context one: every split partition CTA then ends with a
// device-scope fence and an atomic round trip before it frees its SM slot.
#ifndef PA_FUSED_COMBINE
#define PA_FUSED_COMBINE 0
#endif

namespace {

using pa::kBlockSize;
using pa::kRowBytes;

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Streaming multiprocessors of the current device, queried once per device
// (grids of the cache operations and the reduce are sized from it).  Falls
// back to 148 (a full B200) if the query fails.
constexpr int kMaxDevices = 128;
std::atomic<int> g_sm_count[kMaxDevices];

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  int n = g_sm_count[dev].load(std::memory_order_relaxed);
  if (n > 0) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  g_sm_count[dev].store(n, std::memory_order_relaxed);
  return n;
}

// Test hook (pa_test_stall_next_launch): armed by a test, consumed by the next
// decode or prefill launch of the armed kind; 0 = not armed.
std::atomic<int> g_stall_decode{0};
std::atomic<int> g_stall_prefill{0};

int elem_bytes(pa_dtype_t dt) {
  switch (dt) {
    case PA_F32: return 4;
    case PA_F16:
    case PA_BF16: return 2;
    case PA_FP8_E4M3: return 1;
  }
  return 0;
}

// Bytes of one (token, KV head) row: 256 for 16/32-bit caches, 128 for E4M3.
int row_bytes(pa_dtype_t dt) { return dt == PA_FP8_E4M3 ? 128 : kRowBytes; }

pa_status_t cache_shape_status(int64_t num_blocks, int block_size, int num_kv_heads, int head_dim,
                               pa_dtype_t dtype) {
  const int es = elem_bytes(dtype);
  if (es == 0) return PA_ERR_DTYPE;
  if (num_blocks <= 0 || num_blocks > INT32_MAX || block_size != kBlockSize || num_kv_heads <= 0 ||
      head_dim * es != row_bytes(dtype))
    return PA_ERR_SHAPE;
  return PA_OK;
}

// Every kernel is launched with programmatic stream serialisation: it may be
// scheduled while the previous kernel in the stream is still running, and it
// waits (griddepcontrol.wait) before touching global memory, so stream order
// semantics are unchanged while the launch latency overlaps the previous tail.
template <typename... KArgs, typename... Args>
pa_status_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                   Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = PA_PROGRAMMATIC_LAUNCH ? 1 : 0;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// ---------------------------------------------------------------- TMA descriptors
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// The cache [NB][16][Hkv][R B] (R = 256 or 128) seen as a 5-D byte tensor
// {128 B, R/128 parts, Hkv, 16 tokens, NB}; the box is one 128-byte part of one
// (block, KV head) tile: {128, 1, 1, 16, 1} = 2 KiB (16 rows of 128 B),
// landing 128-byte swizzled.  R/128 boxes make the tile.
bool encode_cache_map(CUtensorMap *map, const void *cache, int64_t num_blocks, int num_kv_heads, int rb) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[5] = {128, (cuuint64_t)rb / 128, (cuuint64_t)num_kv_heads, (cuuint64_t)kBlockSize,
                              (cuuint64_t)num_blocks};
  const cuuint64_t strides[4] = {128, (cuuint64_t)rb, (cuuint64_t)num_kv_heads * rb,
                                 (cuuint64_t)kBlockSize * num_kv_heads * rb};
  const cuuint32_t box[5] = {128, 1, 1, kBlockSize, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, const_cast<void *>(cache), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- decode planning
// Library choice of the partition size: 1024 tokens for the tensor-core block
// math (16-bit caches, grouped heads), 512 for the CUDA-core one (measured best
// on B200 for the GQA and MHA workloads); one partition when the longest
// context fits.
int resolve_partition_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim, int max_context_len,
                           int requested) {
  (void)num_seqs;
  if (max_context_len < 0 || requested < 0 || num_kv_heads <= 0) return -1;
  if (requested > 0) return requested % kBlockSize == 0 ? requested : -1;
  const bool tensor_core_math = head_dim == 128 && num_heads / num_kv_heads >= 2;
  const int P = tensor_core_math ? 1024 : 512;
  if (max_context_len <= P)
    return max_context_len <= kBlockSize ? kBlockSize : (max_context_len + kBlockSize - 1) / kBlockSize * kBlockSize;
  return P;
}

int max_partitions(int max_context_len, int partition_size) {
  const int np = (max_context_len + partition_size - 1) / partition_size;
  return np < 1 ? 1 : np;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Split-K workspace: m, l [S][Hq][NP] fp32, o [S][Hq][NP][D] fp32, then one
// counter per (sequence, KV head); each section 256-byte aligned.
struct WorkspaceLayout {
  size_t m_off, l_off, o_off, c_off, bytes;
};

WorkspaceLayout workspace_layout(int num_seqs, int num_heads, int num_kv_heads, int head_dim, int np) {
  WorkspaceLayout w{};
  if (np <= 1) return w;
  const size_t rows = (size_t)num_seqs * num_heads * np;
  w.m_off = 0;
  w.l_off = align256(rows * sizeof(float));
  w.o_off = w.l_off + align256(rows * sizeof(float));
  w.c_off = w.o_off + align256(rows * head_dim * sizeof(float));
  w.bytes = w.c_off + align256((size_t)num_seqs * num_kv_heads * sizeof(unsigned));
  return w;
}

template <typename T>
pa_status_t launch_reduce(const pa::DecodeParams &p, cudaStream_t stream);

template <typename T, int G, typename Math, int W = pa::kDecodeWarps>
pa_status_t launch_decode(const CUtensorMap &mk, const CUtensorMap &mv, const pa::DecodeParams &p,
                          cudaStream_t stream) {
  using SM = pa::DecodeSmem<T, G, Math, W>;
  auto kernel = pa::pa_decode_partition_kernel<T, G, Math, W>;
  // the attribute is per device; setting it on every call costs ~a microsecond of host time
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kAlloc) != cudaSuccess)
    return PA_ERR_CUDA;
  const long long grid = (long long)p.num_seqs * p.num_kv_heads * p.max_partitions;
  if (grid == 0) return PA_OK;
  if (grid > INT32_MAX) return PA_ERR_SHAPE;
  if (p.ws_count != nullptr) {   // split call, combined in the partition kernel: counters start at 0
    const int n = p.num_seqs * p.num_kv_heads;
    const int ctas = (n + 255) / 256 < sm_count() ? (n + 255) / 256 : sm_count();
    pa_status_t st = launch(pa::zero_counts_kernel, dim3((unsigned)ctas), dim3(256), 0, stream, p.ws_count, n);
    if (st != PA_OK) return st;
  }
  pa_status_t st = launch(kernel, dim3((unsigned)grid), dim3(W * 32), SM::kAlloc, stream, mk, mv, p);
  if (st != PA_OK || p.max_partitions <= 1 || p.ws_count != nullptr) return st;
  return launch_reduce<T>(p, stream);
}

// Split-K reduce of a decode call's partials (after its partition kernel).
template <typename T>
pa_status_t launch_reduce(const pa::DecodeParams &p, cudaStream_t stream) {
  // warps per row: one per 8 partitions (at most kReduceWarps); a CTA takes
  // kReduceWarps / wpr rows at a time, the grid strides over the rest (at most
  // 8 CTAs of 8 warps per SM)
  int wpr = (p.max_partitions + pa::kReduceBatch - 1) / pa::kReduceBatch;
  wpr = wpr >= 8 ? 8 : wpr >= 4 ? 4 : wpr >= 2 ? 2 : 1;
  const long long rows = (long long)p.num_seqs * p.num_heads;
  const int rows_per_cta = pa::kReduceWarps / wpr;
  long long ctas = (rows + rows_per_cta - 1) / rows_per_cta;
  if (ctas > 8LL * sm_count()) ctas = 8LL * sm_count();
  return launch(pa::pa_decode_reduce_kernel<T>, dim3((unsigned)ctas), dim3(pa::kReduceWarps * 32), 0, stream, p,
                wpr);
}

// The tensor-core block math of a call that splits its sequences into
// partitions of at most 512 tokens runs as two-warp CTAs, six an SM (short
// CTAs: more of them resident hide more of each one's prologue and
// epilogue); every other call as four-warp CTAs, three an SM (see
// pa_decode.cuh).
template <typename T, int G, typename Math>
pa_status_t launch_mma(const CUtensorMap &mk, const CUtensorMap &mv, const pa::DecodeParams &p, cudaStream_t s) {
  if (p.max_partitions > 1 && p.partition_size <= 512) return launch_decode<T, G, Math, 2>(mk, mv, p, s);
  return launch_decode<T, G, Math>(mk, mv, p, s);
}

// fp32 caches and single-head groups run on the CUDA cores; 16-bit caches with
// grouped heads run the tensor-core block math.
template <typename T>
pa_status_t dispatch_group(int group, const CUtensorMap &mk, const CUtensorMap &mv, const pa::DecodeParams &p,
                           cudaStream_t s) {
  constexpr bool kMma = !std::is_same<T, float>::value;
  switch (group) {
    case 1: return launch_decode<T, 1, pa::FmaMath<T, 1>>(mk, mv, p, s);
    case 2:
      if constexpr (kMma) return launch_mma<T, 2, pa::MmaMath<T, 2>>(mk, mv, p, s);
      else return launch_decode<T, 2, pa::FmaMath<T, 2>>(mk, mv, p, s);
    case 4:
      if constexpr (kMma) return launch_mma<T, 4, pa::MmaMath<T, 4>>(mk, mv, p, s);
      else return launch_decode<T, 4, pa::FmaMath<T, 4>>(mk, mv, p, s);
    case 8:
      if constexpr (kMma) return launch_mma<T, 8, pa::MmaMath<T, 8>>(mk, mv, p, s);
      else return launch_decode<T, 8, pa::FmaMath<T, 8>>(mk, mv, p, s);
  }
  return PA_ERR_SHAPE;
}

// E4M3 caches on the tcgen05 path (pa_decode_fp8tc.cuh): the same grid and
// partials as launch_decode, combined by the same reduce.
template <typename T, int G>
pa_status_t launch_fp8tc(const CUtensorMap &mk, const CUtensorMap &mv, const pa::DecodeParams &p0,
                         cudaStream_t stream) {
  using SH = pa::Fp8TcShape<G>;
  auto kernel = pa::pa_decode_fp8tc_kernel<T, G>;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SH::kAlloc) != cudaSuccess)
    return PA_ERR_CUDA;
  pa::DecodeParams p = p0;
  p.ws_count = nullptr;   // partials always combined by the reduce kernel
  const long long grid = (long long)p.num_seqs * p.num_kv_heads * p.max_partitions;
  if (grid == 0) return PA_OK;
  if (grid > INT32_MAX) return PA_ERR_SHAPE;
  pa_status_t st = launch(kernel, dim3((unsigned)grid), dim3(pa::kTcThreads), SH::kAlloc, stream, mk, mv, p);
  if (st != PA_OK || p.max_partitions <= 1) return st;
  return launch_reduce<T>(p, stream);
}

// 1-byte E4M3 caches: the mma.sync block math in fp16 with the codes
// converted on the CUDA cores (the default), or, built with PA_FP8_TC=1, the
// tcgen05 kernel whose tensor cores read the codes as they land (parity-green,
// measured 1.45x slower on B200: each 128-token tile waits on a serial chain of
// products, softmax and hand-overs, so too few tiles are in flight an SM)
#ifndef PA_FP8_TC
#define PA_FP8_TC 0
#endif
template <typename T>
pa_status_t dispatch_group_fp8(int group, const CUtensorMap &mk, const CUtensorMap &mv, const pa::DecodeParams &p,
                               cudaStream_t s) {
  if (PA_FP8_TC) {
    switch (group) {
      case 1: return launch_fp8tc<T, 1>(mk, mv, p, s);
      case 2: return launch_fp8tc<T, 2>(mk, mv, p, s);
      case 4: return launch_fp8tc<T, 4>(mk, mv, p, s);
      case 8: return launch_fp8tc<T, 8>(mk, mv, p, s);
    }
    return PA_ERR_SHAPE;
  }
  switch (group) {
    case 1: return launch_decode<T, 1, pa::Fp8MmaMath<T, 1>>(mk, mv, p, s);
    case 2: return launch_decode<T, 2, pa::Fp8MmaMath<T, 2>>(mk, mv, p, s);
    case 4: return launch_decode<T, 4, pa::Fp8MmaMath<T, 4>>(mk, mv, p, s);
    case 8: return launch_decode<T, 8, pa::Fp8MmaMath<T, 8>>(mk, mv, p, s);
  }
  return PA_ERR_SHAPE;
}

}  // namespace

extern "C" {

pa_status_t pa_reshape_and_cache(const void *key, const void *value, void *k_cache, void *v_cache,
                                 const int64_t *slot_mapping, int num_tokens, int64_t num_blocks,
                                 int block_size, int num_kv_heads, int head_dim, pa_dtype_t dtype,
                                 void *stream) {
  pa_status_t st = cache_shape_status(num_blocks, block_size, num_kv_heads, head_dim, dtype);
  if (st != PA_OK) return st;
  if (num_tokens < 0) return PA_ERR_SHAPE;
  if (num_tokens == 0) return PA_OK;
  if (!key || !value || !k_cache || !v_cache || !slot_mapping) return PA_ERR_NULL;
  if (!aligned(key, 16) || !aligned(value, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(slot_mapping, 8))
    return PA_ERR_ALIGN;
  const int chunks_per_slot = num_kv_heads * (row_bytes(dtype) / 16);
  const long long total = (long long)num_tokens * chunks_per_slot;
  long long blocks = (total + 255) / 256;
  if (blocks > 16LL * sm_count()) blocks = 16LL * sm_count();
  return launch(pa::reshape_and_cache_kernel, dim3((unsigned)blocks), dim3(256), 0, (cudaStream_t)stream,
                (const uint4 *)key, (const uint4 *)value, (uint4 *)k_cache, (uint4 *)v_cache, slot_mapping,
                num_tokens, chunks_per_slot, (long long)num_blocks * block_size);
}

int pa_decode_partition_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim, int max_context_len,
                             int requested) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0) return -1;
  return resolve_partition_size(num_seqs, num_heads, num_kv_heads, head_dim, max_context_len, requested);
}

size_t pa_decode_workspace_bytes(int num_seqs, int num_heads, int num_kv_heads, int head_dim, int max_context_len,
                                 int requested_partition_size) {
  const int P = pa_decode_partition_size(num_seqs, num_heads, num_kv_heads, head_dim, max_context_len,
                                         requested_partition_size);
  if (P <= 0) return 0;
  return workspace_layout(num_seqs, num_heads, num_kv_heads, head_dim, max_partitions(max_context_len, P)).bytes;
}

}  // extern "C"

namespace {

// A decode call's arguments, checked, with the partition plan derived from them.
struct DecodePlan {
  pa::DecodeParams p;
  CUtensorMap mk, mv;
  const void *k_cache, *v_cache;
  WorkspaceLayout ws;
  int group;
  pa_dtype_t dtype, q_dtype;
  bool empty;   // nothing to launch (no sequences)
};

// Every host-side check of a decode call, in order, except the workspace's:
// dtype: the cache dtype; q_dtype: q and out (equal to dtype except for E4M3 caches).
pa_status_t plan_decode(DecodePlan &d, void *out, const void *q, const void *new_k, const void *new_v,
                        const void *k_cache, const void *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
                        const int32_t *context_lens, int num_seqs, int num_heads, int max_context_len, float scale,
                        int partition_size, int64_t num_blocks, int block_size, int num_kv_heads, int head_dim,
                        pa_dtype_t dtype, pa_dtype_t q_dtype, float k_scale, float v_scale) {
  pa_status_t st = cache_shape_status(num_blocks, block_size, num_kv_heads, head_dim, dtype);
  if (st != PA_OK) return st;
  if (dtype == PA_FP8_E4M3 ? (q_dtype != PA_F16 && q_dtype != PA_BF16) : q_dtype != dtype) return PA_ERR_DTYPE;
  if (!std::isfinite(k_scale) || !std::isfinite(v_scale) || k_scale <= 0.f || v_scale <= 0.f) return PA_ERR_SHAPE;
  if (num_seqs < 0 || num_heads <= 0 || max_context_len < 0 || max_blocks_per_seq < 0 ||
      num_heads % num_kv_heads != 0 || !std::isfinite(scale))
    return PA_ERR_SHAPE;
  const int group = num_heads / num_kv_heads;
  if (group != 1 && group != 2 && group != 4 && group != 8) return PA_ERR_SHAPE;
  if ((long long)max_blocks_per_seq * kBlockSize > INT32_MAX) return PA_ERR_SHAPE;
  const int P = resolve_partition_size(num_seqs, num_heads, num_kv_heads, head_dim, max_context_len,
                                       partition_size);
  if (P <= 0) return PA_ERR_SHAPE;
  d.empty = num_seqs == 0;
  if (d.empty) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !context_lens || (max_blocks_per_seq > 0 && !block_tables))
    return PA_ERR_NULL;
  if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(block_tables, 4) || !aligned(context_lens, 4))
    return PA_ERR_ALIGN;
  const int np = max_partitions(max_context_len, P);
  d.ws = workspace_layout(num_seqs, num_heads, num_kv_heads, head_dim, np);
  d.group = group;
  d.dtype = dtype;
  d.q_dtype = q_dtype;

  pa::DecodeParams &p = d.p;
  p = pa::DecodeParams{};
  p.out = out;
  p.q = q;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.num_blocks = num_blocks;
  p.num_seqs = num_seqs;
  p.num_heads = num_heads;
  p.num_kv_heads = num_kv_heads;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.max_context_len = max_context_len;
  p.partition_size = P;
  p.max_partitions = np;
  p.scale_log2 = (float)((double)scale * 1.4426950408889634 * (double)k_scale);
  p.v_scale = v_scale;
  p.new_k = new_k;
  p.new_v = new_v;
  p.k_cache = new_k ? const_cast<void *>(k_cache) : nullptr;
  p.v_cache = new_k ? const_cast<void *>(v_cache) : nullptr;
  d.k_cache = k_cache;
  d.v_cache = v_cache;
  return PA_OK;
}

// Launch a planned decode with its split-K workspace (checked by the caller).
pa_status_t launch_planned(DecodePlan &d, void *workspace, void *stream) {
  if (d.empty) return PA_OK;
  pa::DecodeParams &p = d.p;
  const int rb = row_bytes(d.dtype);
  if (!encode_cache_map(&d.mk, d.k_cache, p.num_blocks, p.num_kv_heads, rb) ||
      !encode_cache_map(&d.mv, d.v_cache, p.num_blocks, p.num_kv_heads, rb))
    return PA_ERR_CUDA;
  char *w = static_cast<char *>(workspace);
  p.ws_m = d.ws.bytes ? reinterpret_cast<float *>(w + d.ws.m_off) : nullptr;
  p.ws_l = d.ws.bytes ? reinterpret_cast<float *>(w + d.ws.l_off) : nullptr;
  p.ws_o = d.ws.bytes ? reinterpret_cast<float *>(w + d.ws.o_off) : nullptr;
  p.ws_count = d.ws.bytes && PA_FUSED_COMBINE ? reinterpret_cast<unsigned *>(w + d.ws.c_off) : nullptr;
  p.stall_cta = g_stall_decode.exchange(0);
  cudaStream_t s = (cudaStream_t)stream;
  const int group = d.group;
  if (d.dtype == PA_FP8_E4M3)
    return d.q_dtype == PA_F16 ? dispatch_group_fp8<__half>(group, d.mk, d.mv, p, s)
                               : dispatch_group_fp8<__nv_bfloat16>(group, d.mk, d.mv, p, s);
  switch (d.dtype) {
    case PA_F32: return dispatch_group<float>(group, d.mk, d.mv, p, s);
    case PA_F16: return dispatch_group<__half>(group, d.mk, d.mv, p, s);
    case PA_BF16: return dispatch_group<__nv_bfloat16>(group, d.mk, d.mv, p, s);
    case PA_FP8_E4M3: break;
  }
  return PA_ERR_DTYPE;
}

pa_status_t decode_impl(void *out, const void *q, const void *new_k, const void *new_v, const void *k_cache,
                        const void *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
                        const int32_t *context_lens, int num_seqs, int num_heads, int max_context_len, float scale,
                        int partition_size, void *workspace, size_t workspace_bytes, int64_t num_blocks,
                        int block_size, int num_kv_heads, int head_dim, pa_dtype_t dtype, void *stream,
                        pa_dtype_t q_dtype, float k_scale, float v_scale) {
  DecodePlan d;
  const pa_status_t st = plan_decode(d, out, q, new_k, new_v, k_cache, v_cache, block_tables, max_blocks_per_seq,
                                     context_lens, num_seqs, num_heads, max_context_len, scale, partition_size,
                                     num_blocks, block_size, num_kv_heads, head_dim, dtype, q_dtype, k_scale, v_scale);
  if (st != PA_OK || d.empty) return st;
  if (d.ws.bytes > 0) {
    if (!workspace || workspace_bytes < d.ws.bytes) return PA_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return PA_ERR_ALIGN;
  }
  return launch_planned(d, workspace, stream);
}

}  // namespace

extern "C" {

pa_status_t pa_decode(void *out, const void *q, const void *k_cache, const void *v_cache,
                      const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
                      int num_seqs, int num_heads, int max_context_len, float scale, int partition_size,
                      void *workspace, size_t workspace_bytes, int64_t num_blocks, int block_size,
                      int num_kv_heads, int head_dim, pa_dtype_t dtype, void *stream) {
  if (dtype == PA_FP8_E4M3) return PA_ERR_DTYPE;   // pa_decode_fp8
  return decode_impl(out, q, nullptr, nullptr, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                     num_seqs, num_heads, max_context_len, scale, partition_size, workspace, workspace_bytes,
                     num_blocks, block_size, num_kv_heads, head_dim, dtype, stream, dtype, 1.f, 1.f);
}

pa_status_t pa_decode_fp8(void *out, const void *q, const void *k_cache, const void *v_cache, float k_scale,
                          float v_scale, const int32_t *block_tables, int max_blocks_per_seq,
                          const int32_t *context_lens, int num_seqs, int num_heads, int max_context_len,
                          float scale, int partition_size, void *workspace, size_t workspace_bytes,
                          int64_t num_blocks, int block_size, int num_kv_heads, int head_dim, pa_dtype_t q_dtype,
                          void *stream) {
  return decode_impl(out, q, nullptr, nullptr, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                     num_seqs, num_heads, max_context_len, scale, partition_size, workspace, workspace_bytes,
                     num_blocks, block_size, num_kv_heads, head_dim, PA_FP8_E4M3, stream, q_dtype, k_scale, v_scale);
}

pa_status_t pa_reshape_and_cache_fp8(const void *key, const void *value, void *k_cache, void *v_cache,
                                     const int64_t *slot_mapping, int num_tokens, int64_t num_blocks,
                                     int block_size, int num_kv_heads, int head_dim, pa_dtype_t src_dtype,
                                     float k_scale, float v_scale, void *stream) {
  pa_status_t st = cache_shape_status(num_blocks, block_size, num_kv_heads, head_dim, PA_FP8_E4M3);
  if (st != PA_OK) return st;
  if (src_dtype != PA_F16 && src_dtype != PA_BF16) return PA_ERR_DTYPE;
  if (!std::isfinite(k_scale) || !std::isfinite(v_scale) || k_scale <= 0.f || v_scale <= 0.f) return PA_ERR_SHAPE;
  if (num_tokens < 0) return PA_ERR_SHAPE;
  if (num_tokens == 0) return PA_OK;
  if (!key || !value || !k_cache || !v_cache || !slot_mapping) return PA_ERR_NULL;
  if (!aligned(key, 16) || !aligned(value, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(slot_mapping, 8))
    return PA_ERR_ALIGN;
  const int chunks_per_slot = num_kv_heads * (head_dim / 8);   // 8 elements per thread
  const long long total = (long long)num_tokens * chunks_per_slot;
  long long blocks = (total + 255) / 256;
  if (blocks > 16LL * sm_count()) blocks = 16LL * sm_count();
  const long long slots = (long long)num_blocks * block_size;
  if (src_dtype == PA_F16)
    return launch(pa::reshape_and_cache_fp8_kernel<__half>, dim3((unsigned)blocks), dim3(256), 0,
                  (cudaStream_t)stream, (const uint4 *)key, (const uint4 *)value, (uint2 *)k_cache,
                  (uint2 *)v_cache, slot_mapping, num_tokens, chunks_per_slot, slots, k_scale, v_scale);
  return launch(pa::reshape_and_cache_fp8_kernel<__nv_bfloat16>, dim3((unsigned)blocks), dim3(256), 0,
                (cudaStream_t)stream, (const uint4 *)key, (const uint4 *)value, (uint2 *)k_cache, (uint2 *)v_cache,
                slot_mapping, num_tokens, chunks_per_slot, slots, k_scale, v_scale);
}

pa_status_t pa_decode_append(void *out, const void *q, const void *key, const void *value, void *k_cache,
                             void *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
                             const int32_t *context_lens, int num_seqs, int num_heads, int max_context_len,
                             float scale, int partition_size, void *workspace, size_t workspace_bytes,
                             int64_t num_blocks, int block_size, int num_kv_heads, int head_dim, pa_dtype_t dtype,
                             void *stream) {
  if (num_seqs > 0 && (!key || !value)) return PA_ERR_NULL;
  if (!aligned(key, 16) || !aligned(value, 16)) return PA_ERR_ALIGN;
  if (dtype == PA_FP8_E4M3) return PA_ERR_DTYPE;
  return decode_impl(out, q, key, value, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                     num_seqs, num_heads, max_context_len, scale, partition_size, workspace, workspace_bytes,
                     num_blocks, block_size, num_kv_heads, head_dim, dtype, stream, dtype, 1.f, 1.f);
}

pa_status_t pa_prefill(void *out, const void *q, const void *k_cache, const void *v_cache,
                       const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
                       const int32_t *query_start_loc, int num_seqs, int num_heads, int max_query_len,
                       float scale, int64_t num_blocks, int block_size, int num_kv_heads, int head_dim,
                       pa_dtype_t dtype, void *stream) {
  pa_status_t st = cache_shape_status(num_blocks, block_size, num_kv_heads, head_dim, dtype);
  if (st != PA_OK) return st;
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_DTYPE;
  if (head_dim != 128 || num_seqs < 0 || num_seqs > 65535 || num_heads <= 0 || num_kv_heads > 65535 ||
      num_heads % num_kv_heads != 0 || max_query_len < 0 || max_blocks_per_seq < 0 || !std::isfinite(scale) ||
      !(scale > 0.f))
    return PA_ERR_SHAPE;
  const int group = num_heads / num_kv_heads;
  if (group != 1 && group != 2 && group != 4 && group != 8) return PA_ERR_SHAPE;
  if ((long long)max_blocks_per_seq * kBlockSize > INT32_MAX) return PA_ERR_SHAPE;
  if (num_seqs == 0 || max_query_len == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !context_lens || !query_start_loc || (max_blocks_per_seq > 0 && !block_tables))
    return PA_ERR_NULL;
  if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(block_tables, 4) || !aligned(context_lens, 4) || !aligned(query_start_loc, 4))
    return PA_ERR_ALIGN;
  CUtensorMap mk, mv;
  if (!encode_cache_map(&mk, k_cache, num_blocks, num_kv_heads, kRowBytes) ||
      !encode_cache_map(&mv, v_cache, num_blocks, num_kv_heads, kRowBytes))
    return PA_ERR_CUDA;
  pa::PrefillParams p{};
  p.out = out;
  p.q = q;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.query_start_loc = query_start_loc;
  p.num_blocks = num_blocks;
  p.num_seqs = num_seqs;
  p.num_heads = num_heads;
  p.num_kv_heads = num_kv_heads;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.max_query_len = max_query_len;
  p.scale_log2 = (float)((double)scale * 1.4426950408889634);
  p.stall_cta = g_stall_prefill.exchange(0);
  const int qt = pa::kPrefillTiles * pa::kPrefillRows / group;   // chunk queries per CTA
  const dim3 grid((unsigned)((max_query_len + qt - 1) / qt), (unsigned)num_kv_heads, (unsigned)num_seqs);
  auto go = [&](auto kernel) -> pa_status_t {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, pa::PrefillSmem::kAlloc) !=
        cudaSuccess)
      return PA_ERR_CUDA;
    return launch(kernel, grid, dim3(pa::kPrefillThreads), pa::PrefillSmem::kAlloc, (cudaStream_t)stream, mk, mv, p);
  };
  if (dtype == PA_BF16) {
    switch (group) {
      case 1: return go(pa::pa_prefill_kernel<__nv_bfloat16, 1>);
      case 2: return go(pa::pa_prefill_kernel<__nv_bfloat16, 2>);
      case 4: return go(pa::pa_prefill_kernel<__nv_bfloat16, 4>);
      case 8: return go(pa::pa_prefill_kernel<__nv_bfloat16, 8>);
    }
  } else {
    switch (group) {
      case 1: return go(pa::pa_prefill_kernel<__half, 1>);
      case 2: return go(pa::pa_prefill_kernel<__half, 2>);
      case 4: return go(pa::pa_prefill_kernel<__half, 4>);
      case 8: return go(pa::pa_prefill_kernel<__half, 8>);
    }
  }
  return PA_ERR_SHAPE;
}

pa_status_t pa_copy_blocks(void *k_cache, void *v_cache, const int64_t *block_mapping, int num_pairs,
                           int64_t num_blocks, int block_size, int num_kv_heads, int head_dim, pa_dtype_t dtype,
                           void *stream) {
  pa_status_t st = cache_shape_status(num_blocks, block_size, num_kv_heads, head_dim, dtype);
  if (st != PA_OK) return st;
  if (num_pairs < 0 || num_pairs > PA_MAX_COPY_PAIRS) return PA_ERR_SHAPE;
  if (num_pairs == 0) return PA_OK;
  if (!k_cache || !v_cache || !block_mapping) return PA_ERR_NULL;
  if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(block_mapping, 8)) return PA_ERR_ALIGN;
  const int chunks_per_block = kBlockSize * num_kv_heads * (row_bytes(dtype) / 16);
  // one CTA per pair up to two per SM, then each CTA takes several pairs (at
  // most kCopyMaxPairsPerCta); blockIdx.y: 0 = K cache, 1 = V cache
  long long ctas = num_pairs < 2LL * sm_count() ? num_pairs : 2LL * sm_count();
  const long long min_ctas = (num_pairs + pa::kCopyMaxPairsPerCta - 1) / pa::kCopyMaxPairsPerCta;
  if (ctas < min_ctas) ctas = min_ctas;
  return launch(pa::copy_blocks_kernel, dim3((unsigned)ctas, 2), dim3(pa::kCopyThreads), 0, (cudaStream_t)stream,
                (uint4 *)k_cache, (uint4 *)v_cache, (const longlong2 *)block_mapping, num_pairs,
                (long long)num_blocks, chunks_per_block);
}

// ---------------------------------------------------------------- no-allocation decode
// Split-K scratch owned by the library, for callers that cannot allocate device
// memory themselves.  It lives in every device that loads this library, for
// the life of the process.  Host code must not use the array's name as a device
// address: the address is looked up per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_decode_scratch[PA_STATIC_WORKSPACE_BYTES];

namespace {
// Address of the current device's copy of g_decode_scratch, looked up on every
// call (cheap, allocates nothing), so that it is never stale -- e.g. after a
// cudaDeviceReset, which gives the device a new context and a new copy.  The
// first lookup on a device may load the library's device code there.
void *scratch_for_current_device() {
  void *ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess) return nullptr;
  return ptr;
}
}  // namespace

pa_status_t pa_decode_static_workspace(void *out, const void *q, const void *k_cache, const void *v_cache,
                                       const int32_t *block_tables, int max_blocks_per_seq,
                                       const int32_t *context_lens, int num_seqs, int num_heads,
                                       int max_context_len, float scale, int partition_size, int64_t num_blocks,
                                       int block_size, int num_kv_heads, int head_dim, pa_dtype_t dtype,
                                       void *stream) {
  if (dtype == PA_FP8_E4M3) return PA_ERR_DTYPE;   // as pa_decode
  // every check of pa_decode first, in its order; then the size of the scratch
  DecodePlan d;
  const pa_status_t st = plan_decode(d, out, q, nullptr, nullptr, k_cache, v_cache, block_tables, max_blocks_per_seq,
                                     context_lens, num_seqs, num_heads, max_context_len, scale, partition_size,
                                     num_blocks, block_size, num_kv_heads, head_dim, dtype, dtype, 1.f, 1.f);
  if (st != PA_OK || d.empty) return st;
  void *scratch = nullptr;
  if (d.ws.bytes > 0) {
    if (d.ws.bytes > PA_STATIC_WORKSPACE_BYTES) return PA_ERR_WORKSPACE;
    scratch = scratch_for_current_device();
    if (!scratch) return PA_ERR_CUDA;
  }
  return launch_planned(d, scratch, stream);
}

pa_status_t pa_stream_read(const void *buf, size_t bytes, uint64_t *sink, void *stream) {
  if (bytes % 16 != 0) return PA_ERR_SHAPE;
  if (bytes == 0) return PA_OK;
  if (!buf || !sink) return PA_ERR_NULL;
  if (!aligned(buf, 16) || !aligned(sink, 8)) return PA_ERR_ALIGN;
  // eight resident CTAs of 256 threads per SM: a full SM of threads
  const long long n16 = (long long)(bytes / 16);
  long long ctas = (n16 + pa::kProbeThreads - 1) / pa::kProbeThreads;
  if (ctas > 8LL * sm_count()) ctas = 8LL * sm_count();
  return launch(pa::stream_read_kernel, dim3((unsigned)ctas), dim3(pa::kProbeThreads), 0, (cudaStream_t)stream,
                (const uint4 *)buf, n16, (unsigned long long *)sink);
}

pa_status_t pa_test_stall_next_launch(int kernel, int64_t cta) {
  if (cta < -1 || cta >= INT32_MAX) return PA_ERR_SHAPE;
  const int armed = (int)cta + 1;   // cta -1: disarm
  switch (kernel) {
    case 0: g_stall_decode.store(armed); return PA_OK;
    case 1: g_stall_prefill.store(armed); return PA_OK;
  }
  return PA_ERR_SHAPE;
}

int pa_get_device_error(void *stream, int64_t *detail, int clear) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return -1;
  int code = 0;
  long long d = 0;
  if (cudaMemcpyFromSymbol(&code, pa::g_error_code, sizeof(int)) != cudaSuccess) return -1;
  if (cudaMemcpyFromSymbol(&d, pa::g_error_detail, sizeof(long long)) != cudaSuccess) return -1;
  if (detail) *detail = d;
  if (clear) {
    const int zero = 0;
    const long long zd = 0;
    if (cudaMemcpyToSymbol(pa::g_error_code, &zero, sizeof(int)) != cudaSuccess) return -1;
    if (cudaMemcpyToSymbol(pa::g_error_detail, &zd, sizeof(long long)) != cudaSuccess) return -1;
  }
  return code;
}

const char *pa_status_string(pa_status_t status) {
  switch (status) {
    case PA_OK: return "PA_OK";
    case PA_ERR_NULL: return "PA_ERR_NULL: a required pointer is NULL";
    case PA_ERR_DTYPE: return "PA_ERR_DTYPE: unknown dtype";
    case PA_ERR_SHAPE: return "PA_ERR_SHAPE: unsupported or inconsistent sizes";
    case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE: split-K workspace missing or too small";
    case PA_ERR_CUDA: return "PA_ERR_CUDA: a CUDA call or kernel launch failed";
    case PA_ERR_ALIGN: return "PA_ERR_ALIGN: a pointer is not aligned as required";
  }
  return "unknown status";
}

}  // extern "C"
