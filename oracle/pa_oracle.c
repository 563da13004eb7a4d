/*
 * pa_oracle.c -- CPU oracle for paged decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA library; it is a plain, slow,
 * obviously correct restatement of what the method computes, in fp64.
 *
 * Sources (web pages; cited by title and section):
 *   [A] "vLLM推理引擎深度解析：从PagedAttention原理到高吞吐量部署的工程实践"
 *       (bbs.huaweicloud.cn/blogs/485029)
 *       §三 PagedAttention：虚拟内存思想应用于KV Cache -- PagedAttentionManager
 *           (block tables, append_token, share_prefix with ref counts)
 *       §五 优化的注意力计算 -- PagedAttention.forward (gather by block table,
 *           scores q.K, scale 1/sqrt(head_dim), softmax, weighted sum of V)
 *   [B] "vLLM 原理与源码阅读" (zhutianwuxian.top/ai/vllm-source.html)
 *       PagedAttention 核心思想 (logical -> physical block map),
 *       Block 管理器 (block table per request, default block size 16,
 *       copy-on-write of a shared block)
 *   [C] "vLLM推理引擎深度实战：…" (bbs.huaweicloud.cn/blogs/486472)
 *       §1.2 PagedAttention原理 (block table: logical block id -> physical
 *       block id; MemoryError when blocks run out)
 *
 * Readings where the pages are silent or garbled (each also listed in the
 * design notes):
 *   - GQA: the pages are multi-head only.  Query head h reads KV head
 *     h / (Hq/Hkv) (contiguous groups).
 *   - One logical block maps to exactly one physical block ([B]'s diagram that
 *     maps one logical block to two physical ids is read as garbled).
 *   - Each sequence has its own block-table row ([A]'s sketch shares one row
 *     across the batch); a block id outside [0, NB) is an error, never skipped.
 *   - context_len 0: the output row is all zeros (sum over an empty set).
 *   - A slot < 0 in the slot mapping means "no write" (padding token).
 *   - Copy-on-write pairs: a pair is carried out only if its ids are in range,
 *     its destination is not the destination of another pair and is not the
 *     source of any pair; every other pair is skipped and reported.
 *
 * Storage dtypes are widened exactly to double on read: fp32 directly, bf16 by
 * placing its 16 bits above 16 zero bits of an IEEE binary32, fp16 by decoding
 * the IEEE 754 binary16 fields (sign, 5-bit exponent with bias 15, 10-bit
 * fraction; subnormals, infinities and NaN included).
 *
 * Function pins (all in the CPU test suite):
 *   oracle_paged_decode      dense unpaged attention on the logical sequence,
 *                            block-permutation invariance, L=1 returns V,
 *                            sum of weights = 1, closed forms on 1-3 tokens,
 *                            GQA = MHA on repeated KV heads.
 *   oracle_reshape_and_cache reproduces the generator's placement of the
 *                            step's token; every other byte unchanged.
 *   oracle_copy_blocks       destination equals source byte for byte; every
 *                            other byte unchanged; conflict rule cases.
 *   oracle_slot_for_position the append rule against the generator's slots.
 *   oracle_widen             every fp16/bf16 bit pattern against numpy/torch.
 *   oracle_e4m3_decode       all 256 codes against torch's float8_e4m3fn.
 *   oracle_e4m3_quantize     torch's float8_e4m3fn cast (nearest, ties to even)
 *                            inside the finite range; saturation outside it.
 *   oracle_reshape_and_cache_fp8  the slot layout of oracle_reshape_and_cache.
 *   oracle_paged_decode_fp8  torch SDPA (fp64) on the dequantised logical K/V.
 *   oracle_paged_prefill     torch SDPA (fp64) with the causal mask at the
 *                            chunk's offset; later tokens do not matter.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_F32 = 0, ORACLE_F16 = 1, ORACLE_BF16 = 2 };

enum {
  ORACLE_OK = 0,
  ORACLE_BAD_ARGS = 1,
  ORACLE_BAD_BLOCK_ID = 2,
  ORACLE_BAD_SLOT = 3,
  ORACLE_COPY_CONFLICT = 4,
  ORACLE_BAD_CONTEXT_LEN = 5,
  ORACLE_NO_MEMORY = 6,
};

static int elem_bytes(int dtype) { return dtype == ORACLE_F32 ? 4 : 2; }

/* Exact widening of one stored element to double. */
static double widen_one(const void *base, int64_t i, int dtype) {
  if (dtype == ORACLE_F32) {
    float f;
    memcpy(&f, (const char *)base + 4 * i, 4);
    return (double)f;
  }
  uint16_t h;
  memcpy(&h, (const char *)base + 2 * i, 2);
  if (dtype == ORACLE_BF16) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
  }
  /* IEEE 754 binary16 */
  int sign = (h >> 15) & 1;
  int exp = (h >> 10) & 0x1f;
  int frac = h & 0x3ff;
  double v;
  if (exp == 0)
    v = ldexp((double)frac, -24);                  /* subnormal: frac * 2^-24 */
  else if (exp == 31)
    v = frac ? NAN : INFINITY;
  else
    v = ldexp((double)(1024 + frac), exp - 25);    /* (1 + frac/2^10) * 2^(exp-15) */
  return sign ? -v : v;
}

void oracle_widen(double *out, const void *src, int64_t n, int dtype) {
  for (int64_t i = 0; i < n; ++i) out[i] = widen_one(src, i, dtype);
}

/*
 * The append rule ([A] §三 append_token; [C] §1.2): token position `pos` of a
 * sequence lives in logical block pos / block_size at offset pos % block_size;
 * the block table gives the physical block.  Its flat slot number is
 * physical_block * block_size + offset.  Returns -1 if the table row has no
 * valid block for that position.
 */
int64_t oracle_slot_for_position(const int32_t *block_table_row, int row_len,
                                 int64_t pos, int block_size) {
  int64_t logical_block = pos / block_size;
  int64_t offset = pos % block_size;
  if (pos < 0 || logical_block >= row_len) return -1;
  int32_t physical_block = block_table_row[logical_block];
  if (physical_block < 0) return -1;
  return (int64_t)physical_block * block_size + offset;
}

/*
 * Paged decode attention ([A] §五 PagedAttention.forward; [B] PagedAttention
 * 核心思想).  For sequence b and query head h:
 *
 *   K_t, V_t = the row of token t (t < L_b) found through block_tables[b]:
 *              physical block block_tables[b][t / bs], offset t % bs, KV head g
 *   s_t      = scale * sum_d q[b][h][d] * K_t[d]
 *   w_t      = exp(s_t - max_u s_u) / sum_u exp(s_u - max_u s_u)   (softmax)
 *   out[b][h]= sum_t w_t * V_t
 *
 * q: [S][Hq][D], caches: [NB][bs][Hkv][D] in `dtype`; out: [S][Hq][D] double.
 * weights (optional): [S][Hq][max_len] double, the w_t of each row (zeros past
 * L_b).  Returns ORACLE_OK or an error code (nothing meaningful is written then).
 */
int oracle_paged_decode(double *out, double *weights, int max_len,
                        const void *q, const void *k_cache, const void *v_cache,
                        const int32_t *block_tables, int max_blocks_per_seq,
                        const int32_t *context_lens, int num_seqs, int num_heads,
                        int num_kv_heads, int head_dim, int block_size,
                        int num_blocks, double scale, int dtype) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
      block_size <= 0 || num_heads % num_kv_heads != 0)
    return ORACLE_BAD_ARGS;
  const int group = num_heads / num_kv_heads;
  const int64_t D = head_dim;

  /* validate every block id a row will read and every length first */
  for (int b = 0; b < num_seqs; ++b) {
    int L = context_lens[b];
    if (L < 0 || (int64_t)L > (int64_t)max_blocks_per_seq * block_size) return ORACLE_BAD_CONTEXT_LEN;
    if (weights && L > max_len) return ORACLE_BAD_ARGS;
    for (int j = 0; j < (L + block_size - 1) / block_size; ++j) {
      int32_t id = block_tables[(int64_t)b * max_blocks_per_seq + j];
      if (id < 0 || id >= num_blocks) return ORACLE_BAD_BLOCK_ID;
    }
  }

  int status = ORACLE_OK;
  const int64_t rows = (int64_t)num_seqs * num_heads;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < rows; ++r) {
    const int b = (int)(r / num_heads);
    const int h = (int)(r % num_heads);
    const int g = h / group;                       /* KV head of this query head */
    const int L = context_lens[b];
    double *o = out + r * D;
    for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
    if (weights)
      for (int t = 0; t < max_len; ++t) weights[r * max_len + t] = 0.0;
    if (L == 0) continue;

    double *s = (double *)malloc(sizeof(double) * (size_t)L);
    double *qv = (double *)malloc(sizeof(double) * (size_t)D);
    if (!s || !qv) {
      free(s);
      free(qv);
#pragma omp atomic write
      status = ORACLE_NO_MEMORY;
      continue;
    }
    for (int64_t d = 0; d < D; ++d) qv[d] = widen_one(q, r * D + d, dtype);

    /* scores: s_t = scale * <q, K_t>, K_t gathered through the block table */
    for (int t = 0; t < L; ++t) {
      int32_t physical_block = block_tables[(int64_t)b * max_blocks_per_seq + t / block_size];
      int offset = t % block_size;
      int64_t row = (((int64_t)physical_block * block_size + offset) * num_kv_heads + g) * D;
      double dot = 0.0;
      for (int64_t d = 0; d < D; ++d) dot += qv[d] * widen_one(k_cache, row + d, dtype);
      s[t] = scale * dot;
    }

    /* softmax over t < L */
    double m = s[0];
    for (int t = 1; t < L; ++t)
      if (s[t] > m) m = s[t];
    double z = 0.0;
    for (int t = 0; t < L; ++t) {
      s[t] = exp(s[t] - m);
      z += s[t];
    }
    for (int t = 0; t < L; ++t) s[t] = s[t] / z;
    if (weights)
      for (int t = 0; t < L; ++t) weights[r * max_len + t] = s[t];

    /* out = sum_t w_t * V_t, V_t gathered through the block table */
    for (int t = 0; t < L; ++t) {
      int32_t physical_block = block_tables[(int64_t)b * max_blocks_per_seq + t / block_size];
      int offset = t % block_size;
      int64_t row = (((int64_t)physical_block * block_size + offset) * num_kv_heads + g) * D;
      for (int64_t d = 0; d < D; ++d) o[d] += s[t] * widen_one(v_cache, row + d, dtype);
    }
    free(s);
    free(qv);
  }
  return status;
}

/*
 * Write the step's new K/V rows into their slots ([A] §五: the new k/v of the
 * current token are appended to the sequence's cache; [A] §三 append_token:
 * the token goes into the last block if it has room, else into a new block --
 * the caller has already turned that decision into a slot number).
 *
 * key, value: [T][Hkv][D]; caches [NB][bs][Hkv][D]; the row of token i and KV
 * head h is copied byte for byte to cache[slot / bs][slot % bs][h].  slot < 0:
 * no write.  A slot >= NB * bs is an error; rows are written in token order, so
 * with duplicate slots the last token wins.  Returns the first error seen (the
 * valid rows are still written).
 */
int oracle_reshape_and_cache(void *k_cache, void *v_cache, const void *key,
                             const void *value, const int64_t *slot_mapping,
                             int num_tokens, int num_kv_heads, int head_dim,
                             int block_size, int num_blocks, int dtype) {
  const int64_t row_bytes = (int64_t)head_dim * elem_bytes(dtype);
  int status = ORACLE_OK;
  for (int i = 0; i < num_tokens; ++i) {
    int64_t slot = slot_mapping[i];
    if (slot < 0) continue;
    if (slot >= (int64_t)num_blocks * block_size) {
      if (status == ORACLE_OK) status = ORACLE_BAD_SLOT;
      continue;
    }
    int64_t block = slot / block_size;
    int64_t offset = slot % block_size;
    for (int h = 0; h < num_kv_heads; ++h) {
      int64_t dst = ((block * block_size + offset) * num_kv_heads + h) * row_bytes;
      int64_t src = ((int64_t)i * num_kv_heads + h) * row_bytes;
      memcpy((char *)k_cache + dst, (const char *)key + src, (size_t)row_bytes);
      memcpy((char *)v_cache + dst, (const char *)value + src, (size_t)row_bytes);
    }
  }
  return status;
}

/*
 * Copy-on-write block copies ([B] Block 管理器, item 3: before a request writes
 * to a block that other requests share, the block is copied and the request
 * gets the copy).  block_mapping: [P][2] (src, dst).  For every valid pair the
 * whole block (bs * Hkv * D elements) of both caches is copied from src to dst.
 * Validity: 0 <= src, dst < NB; dst not the dst of another pair; dst not the
 * src of any pair (itself included).  Invalid pairs are skipped; the return
 * value is then the first error kind met.
 */
int oracle_copy_blocks(void *k_cache, void *v_cache, const int64_t *block_mapping,
                       int num_pairs, int num_kv_heads, int head_dim, int block_size,
                       int num_blocks, int dtype) {
  const int64_t block_bytes = (int64_t)block_size * num_kv_heads * head_dim * elem_bytes(dtype);
  int status = ORACLE_OK;
  /* decide every pair before copying anything: pairs are order-independent */
  char *ok = (char *)malloc((size_t)(num_pairs > 0 ? num_pairs : 1));
  if (!ok) return ORACLE_NO_MEMORY;
  for (int i = 0; i < num_pairs; ++i) {
    int64_t src = block_mapping[2 * i], dst = block_mapping[2 * i + 1];
    ok[i] = 1;
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
      ok[i] = 0;
      if (status == ORACLE_OK) status = ORACLE_BAD_BLOCK_ID;
      continue;
    }
    for (int j = 0; j < num_pairs; ++j) {
      if ((j != i && block_mapping[2 * j + 1] == dst) || block_mapping[2 * j] == dst) {
        ok[i] = 0;
        if (status == ORACLE_OK) status = ORACLE_COPY_CONFLICT;
        break;
      }
    }
  }
  for (int i = 0; i < num_pairs; ++i) {
    if (!ok[i]) continue;
    int64_t src = block_mapping[2 * i], dst = block_mapping[2 * i + 1];
    memcpy((char *)k_cache + dst * block_bytes, (const char *)k_cache + src * block_bytes, (size_t)block_bytes);
    memcpy((char *)v_cache + dst * block_bytes, (const char *)v_cache + src * block_bytes, (size_t)block_bytes);
  }
  free(ok);
  return status;
}

/*
 * ---------------------------------------------------------------- FP8 KV cache
 * An 8-bit KV cache ("vLLM推理引擎深度实战：…" §四 names FP8 among vLLM's
 * quantisation options).  Readings: the format is OCP FP8 E4M3 (sign, 4-bit
 * exponent with bias 7, 3-bit mantissa; no infinities; codes 0x7F / 0xFF are
 * NaN; largest finite 448); each cache has one fp32 scale; a stored code c
 * stands for e4m3(c) * scale; a value x is stored as the E4M3 value nearest to
 * the fp32 quotient x / scale (IEEE division), ties to the even code, values
 * of magnitude >= 448 saturating to +-448, NaN to 0x7F.
 */
static double e4m3_value(uint8_t c) {
  int sign = c >> 7, e = (c >> 3) & 15, m = c & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    v = ldexp((double)m, -9);          /* subnormal: m * 2^-9 */
  else
    v = ldexp(8.0 + m, e - 10);        /* (1 + m/8) * 2^(e-7) */
  return sign ? -v : v;
}

/* the values of the non-negative finite codes 0x00..0x7E (filled before use) */
static double e4m3_positive[0x7F];
static void e4m3_fill_table(void) {
  for (int c = 0; c <= 0x7E; ++c) e4m3_positive[c] = e4m3_value((uint8_t)c);
}

/* nearest E4M3 code by exhaustive search over the finite codes (ties: even code) */
static uint8_t e4m3_encode(float x) {
  if (isnan(x)) return 0x7F;
  int sign = signbit(x) ? 1 : 0;
  double a = fabs((double)x);
  if (a >= 448.0) return (uint8_t)(sign ? 0xFE : 0x7E);
  int best = 0;
  double best_d = INFINITY;
  for (int c = 0; c <= 0x7E; ++c) {
    double d = fabs(e4m3_positive[c] - a);
    if (d < best_d || (d == best_d && (c & 1) == 0)) {
      best = c;
      best_d = d;
    }
  }
  return (uint8_t)(best | (sign << 7));
}

void oracle_e4m3_decode(double *out, const uint8_t *in, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_value(in[i]);
}

/* codes of widen(src[i]) / scale, src in `dtype` (f32, f16 or bf16) */
void oracle_e4m3_quantize(uint8_t *out, const void *src, int64_t n, int dtype, float scale) {
  e4m3_fill_table();
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    float x = (float)widen_one(src, i, dtype);   /* exact: every f16 / bf16 value is an f32 */
    float q = x / scale;
    out[i] = e4m3_encode(q);
  }
}

/* oracle_reshape_and_cache with quantisation: rows of key / value ([T][Hkv][D]
 * in `dtype`) are stored as E4M3 codes (k_scale, v_scale) in the 1-byte caches. */
int oracle_reshape_and_cache_fp8(uint8_t *k_cache, uint8_t *v_cache, const void *key, const void *value,
                                 const int64_t *slot_mapping, int num_tokens, int num_kv_heads, int head_dim,
                                 int block_size, int num_blocks, int dtype, float k_scale, float v_scale) {
  int status = ORACLE_OK;
  e4m3_fill_table();
  for (int i = 0; i < num_tokens; ++i)
    if (slot_mapping[i] >= (int64_t)num_blocks * block_size) status = ORACLE_BAD_SLOT;
#pragma omp parallel for schedule(static)
  for (int i = 0; i < num_tokens; ++i) {
    int64_t slot = slot_mapping[i];
    if (slot < 0 || slot >= (int64_t)num_blocks * block_size) continue;
    int64_t block = slot / block_size;
    int64_t offset = slot % block_size;
    for (int h = 0; h < num_kv_heads; ++h) {
      int64_t dst = ((block * block_size + offset) * num_kv_heads + h) * head_dim;
      int64_t src = ((int64_t)i * num_kv_heads + h) * head_dim;
      for (int d = 0; d < head_dim; ++d) {
        k_cache[dst + d] = e4m3_encode((float)widen_one(key, src + d, dtype) / k_scale);
        v_cache[dst + d] = e4m3_encode((float)widen_one(value, src + d, dtype) / v_scale);
      }
    }
  }
  return status;
}

/*
 * Paged decode over 1-byte E4M3 caches: exactly oracle_paged_decode with
 * K_t[d] = e4m3(code) * k_scale and V_t[d] = e4m3(code) * v_scale (products in
 * fp64, exact), q in `q_dtype`.
 */
int oracle_paged_decode_fp8(double *out, const void *q, int q_dtype, const uint8_t *k_cache,
                            const uint8_t *v_cache, double k_scale, double v_scale,
                            const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
                            int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                            int num_blocks, double scale) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      num_heads % num_kv_heads != 0)
    return ORACLE_BAD_ARGS;
  const int group = num_heads / num_kv_heads;
  const int64_t D = head_dim;
  for (int b = 0; b < num_seqs; ++b) {
    int L = context_lens[b];
    if (L < 0 || (int64_t)L > (int64_t)max_blocks_per_seq * block_size) return ORACLE_BAD_CONTEXT_LEN;
    for (int j = 0; j < (L + block_size - 1) / block_size; ++j) {
      int32_t id = block_tables[(int64_t)b * max_blocks_per_seq + j];
      if (id < 0 || id >= num_blocks) return ORACLE_BAD_BLOCK_ID;
    }
  }
  int status = ORACLE_OK;
  const int64_t rows = (int64_t)num_seqs * num_heads;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < rows; ++r) {
    const int b = (int)(r / num_heads);
    const int h = (int)(r % num_heads);
    const int g = h / group;
    const int L = context_lens[b];
    double *o = out + r * D;
    for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
    if (L == 0) continue;
    double *s = (double *)malloc(sizeof(double) * (size_t)L);
    double *qv = (double *)malloc(sizeof(double) * (size_t)D);
    if (!s || !qv) {
      free(s);
      free(qv);
#pragma omp atomic write
      status = ORACLE_NO_MEMORY;
      continue;
    }
    for (int64_t d = 0; d < D; ++d) qv[d] = widen_one(q, r * D + d, q_dtype);
    for (int t = 0; t < L; ++t) {
      int32_t physical_block = block_tables[(int64_t)b * max_blocks_per_seq + t / block_size];
      int64_t row = (((int64_t)physical_block * block_size + t % block_size) * num_kv_heads + g) * D;
      double dot = 0.0;
      for (int64_t d = 0; d < D; ++d) dot += qv[d] * (e4m3_value(k_cache[row + d]) * k_scale);
      s[t] = scale * dot;
    }
    double m = s[0];
    for (int t = 1; t < L; ++t)
      if (s[t] > m) m = s[t];
    double z = 0.0;
    for (int t = 0; t < L; ++t) {
      s[t] = exp(s[t] - m);
      z += s[t];
    }
    for (int t = 0; t < L; ++t) s[t] = s[t] / z;
    for (int t = 0; t < L; ++t) {
      int32_t physical_block = block_tables[(int64_t)b * max_blocks_per_seq + t / block_size];
      int64_t row = (((int64_t)physical_block * block_size + t % block_size) * num_kv_heads + g) * D;
      for (int64_t d = 0; d < D; ++d) o[d] += s[t] * (e4m3_value(v_cache[row + d]) * v_scale);
    }
    free(s);
    free(qv);
  }
  return status;
}

/*
 * Paged prefill (a chunk of new tokens per sequence attending, causally, to the
 * sequence's cached tokens through its block table).  The pages' engine runs
 * prompts in chunks ("vLLM推理引擎深度实战：…" §五 / tuning: enable_chunked_prefill);
 * the attention of each new token is [A] §五's formula with the context cut at
 * that token.  Reading: sequence b's chunk holds n_b = query_start_loc[b+1] -
 * query_start_loc[b] queries, which are the last n_b of its context_lens[b]
 * tokens (their K/V are already in the cache); query i sits at position
 * p = L_b - n_b + i and attends to tokens 0..p.
 *
 * q, out: [T][Hq][D] with T = query_start_loc[num_seqs]; out double.
 */
int oracle_paged_prefill(double *out, const void *q, const void *k_cache, const void *v_cache,
                         const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
                         const int32_t *query_start_loc, int num_seqs, int num_heads, int num_kv_heads,
                         int head_dim, int block_size, int num_blocks, double scale, int dtype) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      num_heads % num_kv_heads != 0)
    return ORACLE_BAD_ARGS;
  const int group = num_heads / num_kv_heads;
  const int64_t D = head_dim;
  for (int b = 0; b < num_seqs; ++b) {
    int L = context_lens[b];
    int n = query_start_loc[b + 1] - query_start_loc[b];
    if (n < 0 || L < n || (int64_t)L > (int64_t)max_blocks_per_seq * block_size) return ORACLE_BAD_CONTEXT_LEN;
    for (int j = 0; j < (L + block_size - 1) / block_size; ++j) {
      int32_t id = block_tables[(int64_t)b * max_blocks_per_seq + j];
      if (id < 0 || id >= num_blocks) return ORACLE_BAD_BLOCK_ID;
    }
  }
  const int64_t T = query_start_loc[num_seqs];
  int status = ORACLE_OK;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < T * num_heads; ++r) {
    const int64_t tok = r / num_heads;
    const int h = (int)(r % num_heads);
    int b = 0;
    while (query_start_loc[b + 1] <= tok) ++b;
    const int L = context_lens[b];
    const int n = query_start_loc[b + 1] - query_start_loc[b];
    const int pos = L - n + (int)(tok - query_start_loc[b]);   /* this query's position */
    const int g = h / group;
    const int len = pos + 1;                                    /* tokens 0..pos */
    double *o = out + r * D;
    for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
    double *s = (double *)malloc(sizeof(double) * (size_t)len);
    double *qv = (double *)malloc(sizeof(double) * (size_t)D);
    if (!s || !qv) {
      free(s);
      free(qv);
#pragma omp atomic write
      status = ORACLE_NO_MEMORY;
      continue;
    }
    for (int64_t d = 0; d < D; ++d) qv[d] = widen_one(q, r * D + d, dtype);
    for (int t = 0; t < len; ++t) {
      int32_t physical_block = block_tables[(int64_t)b * max_blocks_per_seq + t / block_size];
      int64_t row = (((int64_t)physical_block * block_size + t % block_size) * num_kv_heads + g) * D;
      double dot = 0.0;
      for (int64_t d = 0; d < D; ++d) dot += qv[d] * widen_one(k_cache, row + d, dtype);
      s[t] = scale * dot;
    }
    double m = s[0];
    for (int t = 1; t < len; ++t)
      if (s[t] > m) m = s[t];
    double z = 0.0;
    for (int t = 0; t < len; ++t) {
      s[t] = exp(s[t] - m);
      z += s[t];
    }
    for (int t = 0; t < len; ++t) s[t] = s[t] / z;
    for (int t = 0; t < len; ++t) {
      int32_t physical_block = block_tables[(int64_t)b * max_blocks_per_seq + t / block_size];
      int64_t row = (((int64_t)physical_block * block_size + t % block_size) * num_kv_heads + g) * D;
      for (int64_t d = 0; d < D; ++d) o[d] += s[t] * widen_one(v_cache, row + d, dtype);
    }
    free(s);
    free(qv);
  }
  return status;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}
