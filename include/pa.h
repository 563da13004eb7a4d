/*
 * pa.h -- C ABI of libpa_b200.so: paged-KV decode (and chunked-prefill)
 * attention on NVIDIA B200 (sm_100a).
 *
 * The library implements the decode-time hot path of a paged KV cache as
 * described by these web pages (cited by title and section):
 *   [A] "vLLM推理引擎深度解析：从PagedAttention原理到高吞吐量部署的工程实践"
 *       §三 PagedAttention：虚拟内存思想应用于KV Cache (block pool, per-request
 *       block table, append_token, share_prefix with reference counts);
 *       §五 优化的注意力计算 (PagedAttention.forward: gather K/V through the
 *       block table, scores, 1/sqrt(head_dim) scale, softmax, weighted V; the
 *       new token's K/V is written into the cache).
 *   [B] "vLLM 原理与源码阅读": PagedAttention 核心思想 (logical -> physical
 *       block map); Block 管理器 (block table per request, block size 16 by
 *       default, copy-on-write of a shared block).
 *   [C] "vLLM推理引擎深度实战：…" §1.2 PagedAttention原理 (block table, allocation
 *       failure reported as an error); §5.3 推理优化配置 and §7.1 性能调优指南
 *       (chunked prefill).
 *
 * Conventions shared by every call
 * --------------------------------
 * - Every pointer argument except `stream` and the `detail` out-parameter of
 *   pa_get_device_error is DEVICE memory owned by the caller.  The library
 *   allocates no device or host memory at run time.  What it keeps across
 *   calls: one device error word per GPU (see pa_get_device_error); the SM
 *   count of each GPU (queried once, to size grids); and two arrays that exist
 *   from load time in every GPU that loads the library -- the 64 MiB split-K
 *   scratch of pa_decode_static_workspace, which keeps the last such call's
 *   contents, and the error word.  pa_test_stall_next_launch arms a one-shot
 *   host-side flag (tests only).
 * - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *   NULL = the legacy default stream).  The returned status covers host-side
 *   argument checks and the launch itself (cudaGetLastError).  Problems that
 *   only the GPU can see (a block id or slot out of range, a context length
 *   beyond the table) never fault or trap: the kernel skips the bad access and
 *   records the first such problem in the device error word.
 * - KV cache layout: two separate tensors k_cache and v_cache, each
 *   [num_blocks][block_size][num_kv_heads][head_dim], row-major, contiguous
 *   (token-major inside a block, the per-block layout of [A] §五 with the K/V
 *   axis split into two tensors).  block_size must be 16.  One (token, KV head)
 *   row must be 256 bytes: head_dim 64 for PA_F32, 128 for PA_F16 / PA_BF16 --
 *   or 128 bytes for 1-byte PA_FP8_E4M3 caches (head_dim 128).
 *   Cache base addresses must be 16-byte aligned.
 * - A slot is a flat token index into the pool: slot = physical_block *
 *   block_size + offset ([A] §三 append_token: a new token goes to the next
 *   free offset of the sequence's last block, else to a newly allocated block).
 */
#ifndef PA_B200_PA_H
#define PA_B200_PA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* PA_FP8_E4M3: 1-byte OCP E4M3 codes with one fp32 scale per cache (see
 * pa_reshape_and_cache_fp8); only for caches. */
typedef enum { PA_F32 = 0, PA_F16 = 1, PA_BF16 = 2, PA_FP8_E4M3 = 3 } pa_dtype_t;

typedef enum {
  PA_OK = 0,
  PA_ERR_NULL = 1,       /* a required pointer is NULL */
  PA_ERR_DTYPE = 2,      /* unknown dtype */
  PA_ERR_SHAPE = 3,      /* unsupported or inconsistent sizes (see each call) */
  PA_ERR_WORKSPACE = 4,  /* split-K workspace missing or too small */
  PA_ERR_CUDA = 5,       /* a CUDA runtime/driver call or the launch failed */
  PA_ERR_ALIGN = 6,      /* a pointer is not aligned as required */
} pa_status_t;

/* Kinds recorded in the device error word (pa_get_device_error). */
typedef enum {
  PA_DEV_OK = 0,
  PA_DEV_BAD_BLOCK_ID = 1,     /* block id outside [0, num_blocks); detail = the id */
  PA_DEV_BAD_SLOT = 2,         /* slot >= num_blocks * block_size; detail = the slot */
  PA_DEV_COPY_CONFLICT = 3,    /* copy pair skipped (dst repeated or read by a pair); detail = pair index */
  PA_DEV_BAD_CONTEXT_LEN = 4,  /* context_len < 0, > max_context_len or > table capacity; detail = seq */
  PA_DEV_WAIT_TIMEOUT = 5,     /* an internal bounded wait gave up; detail = linear CTA index
                                  (blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z)) */
  PA_DEV_VALUE_RANGE = 6,      /* pa_prefill, bf16 caches: an attended V element with |v| >= 2^24
                                  (outside the kernel's fp16 range for V); detail = sequence */
} pa_device_error_t;

/*
 * pa_reshape_and_cache -- write each new token's K and V rows into its slot.
 * ([A] §五: the current token's k/v join the cache; [A] §三 append_token.)
 *
 * key, value    [num_tokens][num_kv_heads][head_dim], contiguous, cache dtype.
 * k_cache, v_cache  the caches (layout above); modified in place.
 * slot_mapping  [num_tokens] int64: destination slot of token i.  slot < 0
 *               means "no write" (padding).  slot >= num_blocks*block_size is
 *               skipped and recorded as PA_DEV_BAD_SLOT.  Slots must be
 *               distinct; with duplicates the written row is unspecified.
 * The copy is bit-exact: every byte of each row is moved unchanged, and no
 * other cache byte is touched.
 * Errors: PA_ERR_NULL, PA_ERR_DTYPE, PA_ERR_SHAPE (num_tokens < 0, block_size
 * != 16, row not 256 bytes, num_blocks <= 0), PA_ERR_ALIGN (16-byte
 * alignment of key/value/caches), PA_ERR_CUDA.  num_tokens == 0 is a no-op.
 */
pa_status_t pa_reshape_and_cache(const void *key, const void *value, void *k_cache, void *v_cache,
                                 const int64_t *slot_mapping, int num_tokens, int64_t num_blocks,
                                 int block_size, int num_kv_heads, int head_dim, pa_dtype_t dtype,
                                 void *stream);

/*
 * pa_reshape_and_cache_fp8 -- pa_reshape_and_cache into 1-byte E4M3 caches.
 * (An 8-bit KV cache: "vLLM推理引擎深度实战：…" §四 lists FP8 among vLLM's
 * quantisation options.)
 *
 * key, value    [num_tokens][num_kv_heads][128] in src_dtype (PA_F16 or PA_BF16).
 * k_cache, v_cache  [num_blocks][16][num_kv_heads][128] bytes.
 * Element x of a key row is stored as the OCP E4M3 code nearest to the fp32
 * quotient x / k_scale (IEEE division), ties to even, saturating at +-448
 * (NaN gives a NaN code); likewise value with v_scale.  Scales are finite and
 * > 0.  Slots as in pa_reshape_and_cache.
 * Errors: as pa_reshape_and_cache; PA_ERR_DTYPE for another src_dtype,
 * PA_ERR_SHAPE for head_dim != 128 or a bad scale.
 */
pa_status_t pa_reshape_and_cache_fp8(const void *key, const void *value, void *k_cache, void *v_cache,
                                     const int64_t *slot_mapping, int num_tokens, int64_t num_blocks,
                                     int block_size, int num_kv_heads, int head_dim, pa_dtype_t src_dtype,
                                     float k_scale, float v_scale, void *stream);

/*
 * pa_decode_partition_size -- the partition size (tokens per split-K piece)
 * that pa_decode will use for these arguments.  `requested` > 0 is returned
 * unchanged (it must be a positive multiple of block_size); 0 selects the
 * library's choice.  Returns -1 for invalid arguments.
 */
int pa_decode_partition_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                             int max_context_len, int requested);

/*
 * pa_decode_workspace_bytes -- bytes of split-K workspace pa_decode needs
 * (0 when no sequence can span more than one partition).  Same arguments as
 * pa_decode_partition_size.  Returns 0 for invalid arguments as well; callers
 * that care check pa_decode_partition_size first.
 */
size_t pa_decode_workspace_bytes(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                 int max_context_len, int requested_partition_size);

/*
 * pa_decode -- single-query attention for every sequence over its paged KV
 * cache ([A] §五 PagedAttention.forward; [B] PagedAttention 核心思想).
 *
 * For sequence b, query head h, KV head g = h / (num_heads / num_kv_heads):
 *   K_t, V_t  = row (physical block block_tables[b][t / 16], offset t % 16,
 *               head g) of k_cache / v_cache, for t < context_lens[b]
 *   out[b][h] = sum_t softmax_t(scale * <q[b][h], K_t>) * V_t
 * Accumulation is fp32; the output is rounded to the cache dtype (nearest
 * even).  context_lens[b] == 0 gives an all-zero row.
 *
 * out           [num_seqs][num_heads][head_dim], cache dtype (written).
 * q             [num_seqs][num_heads][head_dim], cache dtype.
 * block_tables  [num_seqs][max_blocks_per_seq] int32; entries at or past
 *               ceil(context_lens[b] / 16) are never read.
 * context_lens  [num_seqs] int32; each must be <= max_context_len and
 *               <= max_blocks_per_seq * 16 (else PA_DEV_BAD_CONTEXT_LEN and
 *               that row is not written).
 * max_context_len  host-side upper bound of context_lens (sizes the grid).
 * scale         softmax scale (1/sqrt(head_dim) in the pages).
 * partition_size   0 = library's choice, else a positive multiple of 16:
 *               sequences longer than it are split into pieces that are
 *               combined by a second (reduce) kernel through `workspace`.
 * workspace     device buffer of >= pa_decode_workspace_bytes(...) bytes,
 *               256-byte aligned (may be NULL when that is 0).  Its contents
 *               need no initialisation and are scratch after the call.
 * Errors: PA_ERR_NULL, PA_ERR_DTYPE, PA_ERR_SHAPE (num_heads % num_kv_heads,
 * group size not in {1,2,4,8}, row not 256 bytes, block_size != 16, bad
 * partition_size, negative sizes), PA_ERR_WORKSPACE, PA_ERR_ALIGN (16-byte
 * alignment of q/out/caches, 256 of workspace), PA_ERR_CUDA.
 */
pa_status_t pa_decode(void *out, const void *q, const void *k_cache, const void *v_cache,
                      const int32_t *block_tables, int max_blocks_per_seq,
                      const int32_t *context_lens, int num_seqs, int num_heads,
                      int max_context_len, float scale, int partition_size, void *workspace,
                      size_t workspace_bytes, int64_t num_blocks, int block_size, int num_kv_heads,
                      int head_dim, pa_dtype_t dtype, void *stream);

/*
 * pa_decode_fp8 -- pa_decode over 1-byte E4M3 caches (head_dim 128).
 *
 * K_t[d] = e4m3(k_cache code) * k_scale and V_t[d] = e4m3(v_cache code) *
 * v_scale; q and out are in q_dtype (PA_F16 or PA_BF16).  The tensor cores
 * compute in fp16 with fp32 accumulation: q is converted to fp16 once (exact
 * inside the fp16 normal range, |q| in [6.1e-5, 65504]); E4M3 codes convert to
 * fp16 exactly.  Everything else -- arguments, workspace, errors, group sizes
 * 1..8 -- as pa_decode.
 */
pa_status_t pa_decode_fp8(void *out, const void *q, const void *k_cache, const void *v_cache, float k_scale,
                          float v_scale, const int32_t *block_tables, int max_blocks_per_seq,
                          const int32_t *context_lens, int num_seqs, int num_heads, int max_context_len,
                          float scale, int partition_size, void *workspace, size_t workspace_bytes,
                          int64_t num_blocks, int block_size, int num_kv_heads, int head_dim,
                          pa_dtype_t q_dtype, void *stream);

/*
 * pa_decode_append -- the decode step's new-token write and decode in one
 * launch ([A] §五 PagedAttention.forward: the current token's k/v join the
 * cache and are attended together with it; [A] §三 append_token: the token
 * goes to the next offset of the sequence's last block).
 *
 * For every sequence with context_lens[b] >= 1, the new token is position
 * L = context_lens[b] - 1: its K and V rows key[b] and value[b]
 * ([num_seqs][num_kv_heads][head_dim], cache dtype) are written bit-exactly to
 * row (block_tables[b][L / 16], L % 16) of k_cache / v_cache, and the sequence
 * is then decoded over all context_lens[b] tokens exactly as pa_decode does.
 * Same result as pa_reshape_and_cache with slot = block_tables[b][L/16]*16 +
 * L%16 followed by pa_decode, in one kernel (plus the reduce when split).
 * Arguments and errors are those of pa_decode plus key/value (non-NULL,
 * 16-byte aligned); the caches are written, so they are not const here.
 */
pa_status_t pa_decode_append(void *out, const void *q, const void *key, const void *value, void *k_cache,
                             void *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
                             const int32_t *context_lens, int num_seqs, int num_heads, int max_context_len,
                             float scale, int partition_size, void *workspace, size_t workspace_bytes,
                             int64_t num_blocks, int block_size, int num_kv_heads, int head_dim,
                             pa_dtype_t dtype, void *stream);

/*
 * pa_prefill -- paged chunked-prefill attention ([C] §5.3 推理优化配置 and
 * §7.1 性能调优指南: the engine runs prompts in chunks, enable_chunked_prefill;
 * each token's attention is [A] §五's formula with the context cut at that
 * token).
 *
 * Sequence b's chunk is the query rows query_start_loc[b] ..
 * query_start_loc[b+1] - 1 of q; they are the LAST n_b = query_start_loc[b+1] -
 * query_start_loc[b] tokens of its L_b = context_lens[b] tokens, all of which
 * (chunk included) are already in the caches (pa_reshape_and_cache).  Query i
 * of the chunk is position pos = L_b - n_b + i; for each query head h
 *   out[row, h] = sum_{t <= pos} softmax_t(scale * q[row, h] . K_t[h / G]) V_t[h / G]
 * with K_t / V_t found through block_tables[b] as in pa_decode, G = num_heads /
 * num_kv_heads.
 *
 * q, out            [T][num_heads][head_dim], T = query_start_loc[num_seqs],
 *                   dtype PA_F16 or PA_BF16 (= the cache dtype), 16-byte aligned.
 * query_start_loc   [num_seqs + 1] int32, non-decreasing from 0.
 * max_query_len     an upper bound of every n_b (sizes the grid).
 * Other arguments as pa_decode.  head_dim must be 128 and G one of 1, 2, 4, 8.
 * Computed on the tensor cores (tcgen05) with fp32 accumulation; the softmax
 * weights enter P V as fp16 (relative rounding <= 2^-11), and so does V: bf16
 * caches are converted in shared memory, scaled by 2^-8 (exact for every bf16
 * value with 2^-6 <= |v| < 2^24, within 2^-17 absolute below 2^-6), the
 * scale undone in the output.  Device-side errors: PA_DEV_BAD_CONTEXT_LEN (n_b
 * < 0, n_b > max_query_len, L_b < n_b or L_b > max_blocks_per_seq * 16:
 * sequence skipped), PA_DEV_BAD_BLOCK_ID (the block reads as zeros),
 * PA_DEV_VALUE_RANGE (bf16 only: a V element at or above 2^24 in magnitude;
 * that sequence's outputs are not valid), PA_DEV_WAIT_TIMEOUT.
 * Errors: PA_ERR_NULL, PA_ERR_DTYPE, PA_ERR_SHAPE, PA_ERR_ALIGN, PA_ERR_CUDA.
 * num_seqs == 0 or max_query_len == 0 is a no-op.
 */
pa_status_t pa_prefill(void *out, const void *q, const void *k_cache, const void *v_cache,
                       const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
                       const int32_t *query_start_loc, int num_seqs, int num_heads, int max_query_len,
                       float scale, int64_t num_blocks, int block_size, int num_kv_heads, int head_dim,
                       pa_dtype_t dtype, void *stream);

/*
 * pa_copy_blocks -- copy-on-write block copies ([B] Block 管理器, item 3:
 * when a request writes to a block that several requests share, the block is
 * copied first and the request's table is pointed at the copy; the caller
 * keeps the reference counts and rewrites the tables).
 *
 * block_mapping [num_pairs][2] int64 (src, dst): block src of both caches is
 * copied whole (block_size * num_kv_heads * head_dim elements, bit-exact) to
 * block dst.  A pair is skipped and recorded as PA_DEV_BAD_BLOCK_ID if an id
 * is outside [0, num_blocks), or as PA_DEV_COPY_CONFLICT if its dst is the dst
 * of another pair or the src of any pair (itself included); all other pairs
 * are carried out, independently of their order.
 * Cost of the conflict check: each of the kernel's CTAs (up to 2 per SM, more
 * for large batches: one per 256 pairs) reads the mapping once through shared
 * memory, and the pairs are compared num_pairs^2 times in shared memory in
 * all.  num_pairs is capped at PA_MAX_COPY_PAIRS so that this stays bounded
 * (at the cap, about the time of copying the blocks themselves for 8 KV heads
 * of 256-byte rows); copy-on-write batches are far smaller in practice (one
 * block per sequence that writes into a shared block).
 * Errors: PA_ERR_NULL, PA_ERR_DTYPE, PA_ERR_SHAPE (incl. num_pairs < 0 or >
 * PA_MAX_COPY_PAIRS), PA_ERR_ALIGN, PA_ERR_CUDA.  num_pairs == 0 is a no-op.
 */
#define PA_MAX_COPY_PAIRS 65536

pa_status_t pa_copy_blocks(void *k_cache, void *v_cache, const int64_t *block_mapping, int num_pairs,
                           int64_t num_blocks, int block_size, int num_kv_heads, int head_dim,
                           pa_dtype_t dtype, void *stream);

/*
 * PA_STATIC_WORKSPACE_BYTES -- size of the split-K scratch that the library
 * itself owns for pa_decode_static_workspace: 64 MiB in every GPU that loads
 * the library, held until the process exits.
 */
#define PA_STATIC_WORKSPACE_BYTES ((size_t)64 << 20)

/*
 * pa_decode_static_workspace -- pa_decode without a caller-provided workspace
 * and without allocating anything.  The source pages have no counterpart to
 * this call: it exists for users of this library who cannot allocate device
 * memory at the point where they decode -- for example a plugin running inside
 * a serving process whose own allocator owns all device memory and hands out
 * no side buffers, or a latency-critical loop that must not call cudaMalloc or
 * cudaFree because those calls can synchronise the device.
 *
 * Arguments, results and errors are those of pa_decode, minus workspace and
 * workspace_bytes.  The split-K scratch is a library-owned device array of
 * PA_STATIC_WORKSPACE_BYTES; a call whose pa_decode_workspace_bytes(...)
 * exceeds it returns PA_ERR_WORKSPACE without launching anything (e.g. the
 * 256-sequence, 32-head, 4096-token workload at partition 512 needs 33 MiB and
 * fits; 4096 sequences of that shape would not).  The call allocates no device
 * or host memory: no cudaMalloc, no cudaFree, no allocating library routine.
 *
 * Checks: every check of pa_decode, in pa_decode's order, comes first (so a
 * call that is invalid in another way returns what pa_decode returns); then a
 * call whose split-K scratch need exceeds PA_STATIC_WORKSPACE_BYTES returns
 * PA_ERR_WORKSPACE without launching anything.
 *
 * Set-up: every call that needs scratch (one that splits a sequence) looks up
 * the array's address on the current device with cudaGetSymbolAddress, which
 * allocates nothing; the address is never cached, so a cudaDeviceReset (which
 * gives the device a new context and a new copy of the array) needs nothing
 * from the caller.  The first lookup on a device may load the library's
 * device code there, so make the first call on each device before any stream
 * capture.
 *
 * Sharing: every call on a device uses the same array, which keeps the last
 * call's contents.  Nothing in it needs clearing between calls (each call
 * writes every scratch entry it later reads), but calls whose kernels overlap
 * on the GPU -- on different streams, or from different host threads -- race on
 * the array and give wrong results.  Serialise them (one stream, or events).
 */
pa_status_t pa_decode_static_workspace(void *out, const void *q, const void *k_cache, const void *v_cache,
                                       const int32_t *block_tables, int max_blocks_per_seq,
                                       const int32_t *context_lens, int num_seqs, int num_heads,
                                       int max_context_len, float scale, int partition_size,
                                       int64_t num_blocks, int block_size, int num_kv_heads, int head_dim,
                                       pa_dtype_t dtype, void *stream);

/*
 * pa_stream_read -- measurement helper with no counterpart on the source
 * pages: read `bytes` of device memory once, as a plain streaming read (16-byte
 * loads, eight 256-thread CTAs per SM), and XOR every 8-byte little-endian word
 * of it into *sink (device memory, 8-byte aligned; the caller zeroes it first
 * if it wants the XOR itself).  Its duration gives the read-only bandwidth the
 * decode kernels are measured against.  bytes must be a multiple of 16 and buf
 * 16-byte aligned.  Errors: PA_ERR_SHAPE, PA_ERR_NULL, PA_ERR_ALIGN,
 * PA_ERR_CUDA.  bytes == 0 is a no-op.
 */
pa_status_t pa_stream_read(const void *buf, size_t bytes, uint64_t *sink, void *stream);

/*
 * pa_test_stall_next_launch -- test hook for the bounded-wait error path (no
 * counterpart on the source pages; ordinary callers never need it).
 *
 * Arms a one-shot flag in the host library: the next launch of `kernel`
 * (0 = the decode partition kernel of any pa_decode* call, 1 = pa_prefill),
 * from any thread, carries it and clears it.  In that launch, CTA `cta` (the
 * linear index of PA_DEV_WAIT_TIMEOUT) leaves one of its tile copies unissued
 * -- no copy and no barrier arrival, so nothing is in flight for it -- and its
 * waits give up after 1 ms instead of 2 s.  Its wait on the missing tile runs
 * out, it records PA_DEV_WAIT_TIMEOUT with detail = `cta`, lets its other
 * copies in flight land, and returns without writing its output rows; every
 * other CTA runs normally.  The GPU context stays usable.  cta = -1 disarms.
 * Errors: PA_ERR_SHAPE for an unknown kernel or cta < -1.
 */
pa_status_t pa_test_stall_next_launch(int kernel, int64_t cta);

/*
 * pa_get_device_error -- synchronise `stream`, then return the first problem a
 * kernel recorded on the current device since the last clear (a
 * pa_device_error_t; 0 = none).  `detail` (host pointer, may be NULL)
 * receives the offending value.  clear != 0 resets the word to 0.
 * Returns -1 if a CUDA call fails.
 */
int pa_get_device_error(void *stream, int64_t *detail, int clear);

/* pa_status_string -- a static, human-readable name of a status. */
const char *pa_status_string(pa_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* PA_B200_PA_H */
