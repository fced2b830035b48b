/*
 * attn.h -- C ABI of the B200 (sm_100a) exact-attention library with a KV cache.
 *
 * The library computes softmax(scale * Q K^T) V tile by tile with an online
 * softmax (running maximum m, running denominator l, rescale when m grows), so
 * the score matrix never reaches HBM; decode splits the keys into chunks that
 * are processed in parallel and merged by a log-sum-exp combine.
 *
 * Source pages (cited by title and section):
 *   [P1] "KV cache, flash attention and inference optimisation" lesson
 *        (AI Engineering from Scratch, Phase 07 · 12)
 *   [P2] "大模型面试笔记——Attention篇" (juejin)
 *   [P3] "[BEE-30062] FlashAttention 與高效注意力核心"
 *   [P5] "Effizienz" chapter (tokenwerk)
 *
 * Conventions shared by every entry point
 *   - Tensors are dense, row-major and token-major ("BSHD"), the layout of the
 *     [P3] "為長上下文推論啟用 FlashDecoding" section: q (batch, tokens, q_heads,
 *     head_dim), caches (batch, seqlen_cache, kv_heads, head_dim).
 *   - bf16 is IEEE bfloat16 stored as 2-byte little-endian words.
 *   - GQA/MQA: query head h reads K/V head h / (Hq / Hkv) ([P5] "GQA im leicht
 *     lesbaren Code": repeat_interleave along the head axis).  Hq % Hkv == 0.
 *   - Head dimension d is 64 or 128.
 *   - LSE outputs are natural-log log-sum-exp of the SCALED scores, fp32.
 *   - Paged caches ([P1] "页面注意 KV缓存作为虚拟内存"): pools of 16-token physical
 *     blocks laid out [num_blocks, 16, Hkv, d]; a page table int32
 *     [B, max_blocks_per_seq] maps logical block j/16 of sequence b to a
 *     physical block; token j sits in slot j % 16.
 *   - Pointers named "device" must be device (or managed) memory of the current
 *     device; the caller owns every buffer, including the decode workspace.  The
 *     library allocates nothing per call.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and returns a status.  Host-side argument checks run
 *     before anything is launched and return a negative status.  Checks that
 *     need device data (lengths, page ids) set bits of a sticky device status
 *     word instead of faulting; read it with attn_get_device_status().
 */
#ifndef KVATTN_ATTN_H
#define KVATTN_ATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ATTN_API __attribute__((visibility("default")))
#else
#define ATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- return codes -------------------------------------------------------- */
enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = -1, /* null pointer, inconsistent or non-positive sizes, bad dtype */
  ATTN_ERR_UNSUPPORTED = -2, /* valid request outside what is built (d, rows per KV head) */
  ATTN_ERR_WORKSPACE = -3,   /* decode workspace missing or smaller than required */
  ATTN_ERR_CUDA = -4,        /* a CUDA runtime/driver call failed (launch, tensor map, ...) */
  ATTN_ERR_DEVICE = -5,      /* the device status word is non-zero (attn_get_device_status) */
  ATTN_ERR_NO_BLOCKS = -6    /* the block pool cannot meet the request (nothing was changed) */
};

/* ---- output element types ------------------------------------------------ */
enum { ATTN_F32 = 0, ATTN_BF16 = 1 };

/* ---- device status bits (sticky until cleared) --------------------------- */
enum {
  ATTN_DEV_PAGE_ID = 1,      /* a page-table entry read was outside [0, num_blocks) */
  ATTN_DEV_SEQLEN = 2,       /* seqlens_k[b] < T, > max_seqlen_k or beyond the cache capacity */
  ATTN_DEV_APPEND_RANGE = 4, /* kv_append position beyond the cache capacity / page table */
  ATTN_DEV_TIMEOUT = 8,      /* a bounded wait inside a kernel gave up (no fault, results invalid) */
  ATTN_DEV_SCALE = 16        /* an FP8 cache scale was not a positive finite number */
};

/*
 * attn_prefill -- exact attention over a whole prompt, Nq == Nk == N.
 *
 * Defines: [P1] "片技巧" (standard attention S = Q K^T, P = softmax(S), O = P V,
 * computed per Q tile against K/V tiles with a running softmax so the N x N
 * matrix never reaches HBM) and [P2] section 2 (online safe softmax: keep the
 * running maximum m and denominator l, multiply l by a compensation factor when
 * m changes).  causal = 1 is [P3]'s SDPA is_causal: query i sees keys j <= i.
 *
 *   q    device bf16 [B, N, Hq, d]
 *   k, v device bf16 [B, N, Hkv, d]
 *   o    device [B, N, Hq, d], element type o_dtype (ATTN_F32 or ATTN_BF16)
 *   lse  device fp32 [B, Hq, N], or NULL to skip
 *   scale  multiplies q.k (e.g. 1/sqrt(d)); must be finite and > 0
 *   causal 0 or 1
 * Errors: ATTN_ERR_INVALID_ARG for null pointers / sizes < 1 / Hq % Hkv;
 * ATTN_ERR_UNSUPPORTED for d not in {64, 128}; ATTN_ERR_CUDA on launch failure.
 * Runs on tcgen05 tensor cores with TMEM accumulators and TMA-staged tiles.
 */
ATTN_API int attn_prefill(const void* q, const void* k, const void* v, void* o, int o_dtype, float* lse, int B, int Hq,
                 int Hkv, int N, int d, float scale, int causal, void* stream);

/*
 * attn_prefill_cache -- prefill against an existing KV cache: Nq new query
 * tokens per sequence (a prompt chunk, or a prompt after a cached prefix)
 * attend to every cached key plus themselves.
 *
 * Defines: attn_prefill's computation with the keys read from the cache;
 * [P5] "Der wichtige Maskenfehler beim Cache" (the Nq queries are the LAST Nq
 * positions: with causal = 1, query i sees keys j <= seqlens_k[b] - Nq + i) and
 * [P1] "用它" / exercise 2 of its "运动" (prefix caching: the prompt prefix's
 * K,V are computed once and reused).  Same result as attn_decode with T = Nq,
 * computed by the prefill kernel (no key split, no workspace): the faster
 * choice for chunks of some hundred tokens or more.
 *
 *   q           device bf16 [B, Nq, Hq, d]
 *   k_cache,    as for attn_decode (contiguous [B, cache_capacity, Hkv, d], or
 *   v_cache     paged pools [num_blocks, 16, Hkv, d] with page_table)
 *   seqlens_k   device int32 [B]: keys of sequence b INCLUDING the Nq new ones
 *               (append them with kv_append first, on the same stream)
 *   o, lse      [B, Nq, Hq, d] of o_dtype; fp32 [B, Hq, Nq] or NULL
 * Errors: ATTN_ERR_INVALID_ARG (including a capacity below Nq),
 * ATTN_ERR_UNSUPPORTED (d), ATTN_ERR_CUDA.  A length below Nq or beyond the
 * capacity sets ATTN_DEV_SEQLEN and makes that sequence's rows NaN; bad page ids
 * set ATTN_DEV_PAGE_ID.
 */
ATTN_API int attn_prefill_cache(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens_k,
                                const int32_t* page_table, int max_blocks_per_seq, int num_blocks, int cache_capacity,
                                void* o, int o_dtype, float* lse, int B, int Nq, int Hq, int Hkv, int d, float scale,
                                int causal, void* stream);

/*
 * attn_decode_workspace_bytes -- bytes of device workspace attn_decode and
 * attn_decode_fp8 need for these sizes (the per-chunk partial outputs and
 * log-sum-exps of the split along the keys; the larger of the two, whose key
 * chunking differs).  num_splits as for attn_decode.  Returns 0 for invalid sizes,
 * including max_seqlen_k above 2^30.
 */
ATTN_API size_t attn_decode_workspace_bytes(int B, int T, int Hq, int Hkv, int d, int max_seqlen_k, int num_splits);

/*
 * attn_decode -- T new query tokens per sequence against a KV cache.
 *
 * Defines: [P2] section 4 (next-token output softmax(t_Q x_K^T / sqrt(h)) x_V
 * over every cached key: no Q cache, O(N) per step), [P3] "背景" and
 * "為長上下文推論啟用 FlashDecoding" (Flash-Decoding: the keys are split into
 * chunks processed in parallel and the partial softmax results are reduced in a
 * numerically stable way; arguments q, k_cache, v_cache, cache_seqlens,
 * causal), and [P5] "Der wichtige Maskenfehler beim Cache" (the new queries are
 * the LAST T positions: with causal = 1, token t of T sees keys
 * j <= seqlens_k[b] - T + t; a single new token sees the whole cache).
 *
 *   q           device bf16 [B, T, Hq, d]
 *   k_cache,    contiguous (page_table == NULL): device bf16 [B, cache_capacity, Hkv, d]
 *   v_cache     paged: device bf16 pools [num_blocks, 16, Hkv, d]
 *   seqlens_k   device int32 [B]: valid keys of sequence b, INCLUDING the T new
 *               tokens (append them with kv_append first, on the same stream)
 *   page_table  device int32 [B, max_blocks_per_seq], or NULL for a contiguous cache
 *   max_blocks_per_seq, num_blocks   paged sizes (ignored when contiguous)
 *   cache_capacity  contiguous token capacity per sequence (ignored when paged)
 *   max_seqlen_k    host-side upper bound on every seqlens_k[b] (sizes the split
 *                   grid and the workspace), at most 2^30 (ATTN_ERR_UNSUPPORTED
 *                   above); 0 = the cache capacity, capped at 2^30
 *   o           device [B, T, Hq, d] of o_dtype;  lse  device fp32 [B, Hq, T] or NULL
 *   scale, causal   as for attn_prefill; causal with T == 1 equals non-causal
 *   num_splits  0 = automatic chunking (on the tensor-core kernel with one row
 *               tile per KV head and B <= 128: chunks apportioned over the
 *               sequences by their lengths on the device, so the work items fill
 *               the GPU's CTA slots evenly); n > 0 = split every sequence's keys
 *               into at most n chunks
 *   workspace   device memory of at least attn_decode_workspace_bytes(...) bytes,
 *               16-byte aligned; contents on entry do not matter
 * T may be large: a prompt chunk appended to a cached prefix (chunked prefill,
 * prefix caching; [P1] "用它" enable-prefix-caching) is this same call with T =
 * the chunk length, and T = seqlens_k[b] is a prefill from scratch.  With
 * R = (Hq / Hkv) * T query rows per KV head, R <= 16 runs on warp-level MMAs;
 * larger R on the tcgen05 tensor cores, in row tiles of whole tokens of at most
 * 128 rows, scores in TMEM.  With T >= 256 and num_splits == 0 the call runs
 * attn_prefill_cache's kernel instead (same rows, same length rules; the
 * workspace is then not written).  Hq / Hkv must be <= 128.
 * Errors: ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED (d, rows per KV head),
 * ATTN_ERR_WORKSPACE, ATTN_ERR_CUDA.  Bad lengths or page ids found on the
 * device set ATTN_DEV_SEQLEN / ATTN_DEV_PAGE_ID and make the affected rows NaN.
 */
ATTN_API int attn_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens_k,
                const int32_t* page_table, int max_blocks_per_seq, int num_blocks, int cache_capacity,
                int max_seqlen_k, void* o, int o_dtype, float* lse, int B, int T, int Hq, int Hkv, int d,
                float scale, int causal, int num_splits, void* workspace, size_t workspace_bytes, void* stream);

/*
 * kv_append -- write the K and V rows of T new tokens into the cache.
 *
 * Defines: [P2] section 4, x_K <- Concat(x_K, t W_K) and x_V <- Concat(x_V, t W_V)
 * (the projections t W are the caller's), and [P1] "步骤1" (the cache grows by
 * one K,V vector per token per layer per head).  Token t of sequence b goes to
 * position p = cache_lens[b] + t: contiguous row p, or paged block
 * page_table[b][p / 16], slot p % 16.
 *
 *   k_cache, v_cache  as for attn_decode (written)
 *   k_new, v_new      device bf16 [B, T, Hkv, d]
 *   cache_lens        device int32 [B]: lengths BEFORE the append (not modified;
 *                     the caller advances them)
 *   page_table, max_blocks_per_seq, num_blocks, cache_capacity  as for attn_decode
 * Errors: ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED (d), ATTN_ERR_CUDA.  A
 * position beyond the capacity / page table, or a bad page id, is skipped and
 * sets ATTN_DEV_APPEND_RANGE / ATTN_DEV_PAGE_ID.
 */
ATTN_API int kv_append(void* k_cache, void* v_cache, const void* k_new, const void* v_new, const int32_t* cache_lens,
              const int32_t* page_table, int max_blocks_per_seq, int num_blocks, int cache_capacity, int B, int T,
              int Hkv, int d, void* stream);

/*
 * attn_decode_fp8 -- attn_decode over an FP8 KV cache.
 *
 * Defines: [P1] "用它" (serving with an 8-bit float KV cache, --kv-cache-dtype
 * fp8) and [P3] FlashAttention-3 paragraph of "背景" (FP8 mode combines
 * quantisation with the tiled kernel); the attention itself is attn_decode's.
 * The pages fix no encoding; this library stores OCP E4M3 ("FN") codes: one
 * byte per element, exponent bias 7, largest finite +-448, no infinities.
 * Cached element (token, head g, i) stands for value(code) * k_scale[g] (K) or
 * value(code) * v_scale[g] (V); the result is exact attention over those values.
 *
 *   k_cache, v_cache  uint8 e4m3 codes in attn_decode's layouts (contiguous
 *                     [B, cache_capacity, Hkv, d] or paged pools
 *                     [num_blocks, 16, Hkv, d]): half the bytes of the bf16 cache
 *   k_scale, v_scale  device fp32 [Hkv]; positive and finite, else the affected
 *                     rows are NaN and ATTN_DEV_SCALE is set
 *   everything else   as for attn_decode, including the workspace size
 *                     (attn_decode_workspace_bytes with the same arguments)
 * Built for d = 128 (other d return ATTN_ERR_UNSUPPORTED) and, like
 * attn_decode, for Hq / Hkv <= 128 and any T.  Up to 32 query rows per KV head
 * ((Hq / Hkv) * T) run on warp-level f16 MMAs that convert the codes in
 * registers; more rows run on the tcgen05 tensor cores in row tiles of at most
 * 128 rows, the e4m3 tiles converted to f16 in shared memory.  Either way the
 * products are f16 x f16 with fp32 accumulation: every e4m3 value is exact in
 * f16, q is rounded to f16 (exact for bf16 values of magnitude 2^-14 .. 65504;
 * larger magnitudes overflow) and the softmax weights are rounded to f16 before
 * the P V product.
 */
ATTN_API int attn_decode_fp8(const void* q, const void* k_cache, const void* v_cache, const float* k_scale,
                             const float* v_scale, const int32_t* seqlens_k, const int32_t* page_table,
                             int max_blocks_per_seq, int num_blocks, int cache_capacity, int max_seqlen_k, void* o,
                             int o_dtype, float* lse, int B, int T, int Hq, int Hkv, int d, float scale, int causal,
                             int num_splits, void* workspace, size_t workspace_bytes, void* stream);

/*
 * kv_append_fp8 -- kv_append into an FP8 cache: quantise, then write.
 *
 * Each new value x (bf16) of KV head g is stored as the e4m3 code nearest to
 * x / scale[g] (the quotient computed in fp32 by one IEEE division; ties to the
 * even code; magnitudes beyond 448, infinities included, saturate to +-448;
 * NaN stays NaN).  Placement, arguments and errors are kv_append's; k_scale
 * and v_scale are device fp32 [Hkv] (positive and finite, else nothing is
 * written for that head and ATTN_DEV_SCALE is set).  d must be 64 or 128.
 */
ATTN_API int kv_append_fp8(void* k_cache, void* v_cache, const void* k_new, const void* v_new, const float* k_scale,
                           const float* v_scale, const int32_t* cache_lens, const int32_t* page_table,
                           int max_blocks_per_seq, int num_blocks, int cache_capacity, int B, int T, int Hkv, int d,
                           void* stream);

/*
 * kv_cache_bytes -- bytes held by a KV cache: 2 * n_layers * batch * tokens *
 * n_kv_heads * head_dim * elem_bytes, the K and V factor times every dimension.
 *
 * Defines: [P5] "Cachebedarf berechnen" (worked example L=6, B=1, T=1024,
 * Hkv=2, d=64, e=2 gives 3,145,728 bytes) and [P1] "预存计算" (bytes per token
 * per layer = 2 * n_kv_heads * d_head * dtype_size).  Host only, exact integer
 * arithmetic.  Returns -1 if any argument is <= 0 or the product overflows int64.
 */
ATTN_API int64_t kv_cache_bytes(int n_layers, int batch, int64_t tokens, int n_kv_heads, int head_dim, int elem_bytes);

/*
 * attn_get_device_status -- OR of the ATTN_DEV_* bits set by kernels on the
 * current device since the last clear.  Synchronises the device.  clear != 0
 * resets the word to 0 after reading.  Returns ATTN_ERR_CUDA (negative) if the
 * word cannot be read.  Not part of the pages' method: error reporting only.
 */
ATTN_API int attn_get_device_status(int clear);

/*
 * attn_selftest_wait_timeout -- check of the failure detection, not part of the
 * pages' method.  Launches one CTA on `stream` whose thread waits on an mbarrier
 * that nothing arrives at, through the same bounded wait every kernel of this
 * library uses (2 s of %globaltimer, or 4e9 SM cycles, whichever ends first).
 * The wait gives up and the kernel sets ATTN_DEV_TIMEOUT, as a kernel whose wait
 * ran out does; attn_get_device_status then reports it and the context stays
 * usable.  Returns ATTN_OK or ATTN_ERR_CUDA (launch failure).
 */
ATTN_API int attn_selftest_wait_timeout(void* stream);

/*
 * attn_decode_noalloc -- attn_decode for callers that cannot allocate device
 * memory.  The pages have no counterpart: this is a packaging variant only.
 *
 * Some callers have no way to hand the library a workspace: a plugin loaded by
 * a host program that passes it nothing but input and output pointers, or a
 * serving process that reserves every byte of device memory at start-up for
 * weights and its KV pool and treats any later cudaMalloc (which can also
 * synchronise the device) as an error.  This entry point takes exactly the
 * arguments of attn_decode except the workspace, and computes the same result
 * with the same kernels.  The per-chunk partials live in one file-scope device
 * array of ATTN_DECODE_NOALLOC_SCRATCH_BYTES bytes, which every GPU that loads
 * the library keeps from the first call on that device until the process
 * exits.  Nothing here calls cudaMalloc, cudaFree or an allocating library
 * routine.
 *
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture on the device.
 *   - All calls share the one array and leave the last call's partials in it.
 *     Nothing in it has to start at zero (every partial is written before it is
 *     read), but calls whose kernels overlap on the GPU -- on different streams,
 *     or from different host threads -- race on it: serialise them.
 *   - The request is checked exactly as attn_decode checks it, with a
 *     workspace of ATTN_DECODE_NOALLOC_SCRATCH_BYTES: argument errors come
 *     first, with attn_decode's codes; then ATTN_ERR_WORKSPACE, before anything
 *     is launched, when this request's own partials do not fit in the array
 *     (attn_decode_workspace_bytes reports the larger of the bf16 and FP8
 *     layouts, so it can exceed what this call needs); a smaller num_splits
 *     needs less.
 *   - The array's device address is looked up once per device and kept for the
 *     life of the process; like the library's status word and work-queue
 *     counters it does not survive cudaDeviceReset or the destruction of the
 *     device's primary context.
 */
#define ATTN_DECODE_NOALLOC_SCRATCH_BYTES (32u << 20) /* 32 MiB */

ATTN_API int attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens_k,
                                 const int32_t* page_table, int max_blocks_per_seq, int num_blocks,
                                 int cache_capacity, int max_seqlen_k, void* o, int o_dtype, float* lse, int B,
                                 int T, int Hq, int Hkv, int d, float scale, int causal, int num_splits,
                                 void* stream);

/* attn_status_string -- static text for a return code (never NULL). */
ATTN_API const char* attn_status_string(int status);

/*
 * ------------------------------------------------------------------ block pool
 * Host-side allocator of the 16-token physical blocks of a paged KV cache.
 *
 * Defines: [P1] "页面注意 KV缓存作为虚拟内存" (the cache is cut into fixed
 * 16-token blocks; a page table maps logical positions to physical blocks;
 * blocks are shared between parallel samples and reused prefixes) and its
 * exercises 2 (prefix caching: fill the cache for a prompt once, then branch
 * per completion) and 3 (a finished sequence returns its blocks to the pool).
 * Not on the device path: the pool only hands out block ids; the caller writes
 * the tables it produces into device memory for kv_append / attn_decode /
 * attn_prefill_cache.  Every call is thread-safe (one mutex per pool) and
 * all-or-nothing: a request that cannot be met returns a negative status and
 * changes nothing.  Free blocks form a LIFO stack with block 0 on top at
 * creation; a freed sequence pushes its blocks last-to-first.
 */
typedef struct attn_block_pool attn_block_pool;

/* A pool of num_blocks blocks of block_tokens tokens (16 for the kernels).
 * NULL if an argument is < 1 or memory runs out.  Owned by the caller. */
ATTN_API attn_block_pool* attn_block_pool_create(int num_blocks, int block_tokens);
ATTN_API void attn_block_pool_destroy(attn_block_pool* pool);
/* Blocks not referenced by any sequence. */
ATTN_API int attn_block_pool_free_blocks(attn_block_pool* pool);
/* Sequences that reference a block (0 = free). */
ATTN_API int attn_block_ref_count(attn_block_pool* pool, int32_t block);
/* A new empty sequence; returns its id (>= 0; the smallest freed id is reused first). */
ATTN_API int attn_seq_create(attn_block_pool* pool);
/* A new sequence sharing every block of `parent` (reference counts + 1), same length. */
ATTN_API int attn_seq_fork(attn_block_pool* pool, int parent);
/* Room for n_new more tokens at positions length .. length + n_new - 1.  If the
 * sequence's last block is partly filled and shared with another sequence, it is
 * first replaced by a private block: *n_cow = 1 and (*cow_src, *cow_dst) name the
 * block whose contents the caller must copy (attn_copy_blocks) before writing;
 * else *n_cow = 0.  Then the blocks the new length needs are taken.
 * ATTN_ERR_NO_BLOCKS if the pool is short (nothing changed). */
ATTN_API int attn_seq_reserve(attn_block_pool* pool, int seq, int n_new, int32_t* cow_src, int32_t* cow_dst,
                              int* n_cow);
/* Release a sequence: each of its blocks loses one reference; unreferenced blocks return to the pool. */
ATTN_API int attn_seq_free(attn_block_pool* pool, int seq);
/* Tokens the sequence holds (reserved so far). */
ATTN_API int64_t attn_seq_length(attn_block_pool* pool, int seq);
/* The sequence's physical block ids in logical order into out[capacity] (out may be
 * NULL to ask for the count); returns the number of blocks. */
ATTN_API int attn_seq_block_table(attn_block_pool* pool, int seq, int32_t* out, int capacity);
/* Host page table [n_seqs, max_blocks] (row i = seqs[i]'s blocks, -1 padded) and
 * int32 lengths [n_seqs] (lens may be NULL): the page_table / seqlens layout the
 * kernels read.  ATTN_ERR_INVALID_ARG if a sequence needs more than max_blocks. */
ATTN_API int attn_block_pool_page_table(attn_block_pool* pool, const int32_t* seqs, int n_seqs, int max_blocks,
                                        int32_t* table, int32_t* lens);

/*
 * attn_copy_blocks -- device copy of whole blocks of both pools, src[i] -> dst[i]
 * (the copy-on-write step above).  k_pool, v_pool: device [num_blocks, 16, Hkv, d]
 * with elem_bytes 2 (bf16) or 1 (e4m3); src, dst: device int32 [n], n <= 65535.
 * Ids outside [0, num_blocks) are skipped and set ATTN_DEV_PAGE_ID.  A pair must
 * not have its destination used as another pair's source in the same call.
 */
ATTN_API int attn_copy_blocks(void* k_pool, void* v_pool, const int32_t* src, const int32_t* dst, int n,
                              int num_blocks, int Hkv, int d, int elem_bytes, void* stream);

/*
 * attn_pool_simulate -- paged versus contiguous KV memory over a request trace
 * ([P1] exercise 3: many chat completions of different lengths, blocks returned
 * to the pool when a sequence finishes; compare the fragmentation with
 * contiguous allocation).  Host only.
 *
 * events: n_events triples (op, request, n): op 0 = the request starts holding n
 * tokens (its prompt), 1 = it grows by n tokens, 2 = it finishes.  Both
 * allocators see every event and an arena of arena_tokens tokens:
 *   paged       a block pool of arena_tokens / block_tokens blocks (attn_seq_*);
 *               a start that cannot get its blocks is rejected, a growth that
 *               cannot is dropped (its blocks are released, later events ignored);
 *   contiguous  every started request reserves reserve_tokens consecutive tokens
 *               (the worst-case length), or with reserve_tokens = 0 exactly its
 *               final length (the sum of its start and growth tokens in the
 *               trace; at least 1); first fit over the free extents, which
 *               merge when released; a start that finds no extent is rejected,
 *               a growth beyond the reservation is dropped.
 * After every event: reserved tokens (paged: blocks held x block_tokens;
 * contiguous: reservations held), stored tokens (lengths of live requests), and
 * for contiguous the free tokens outside the largest free extent (external
 * fragmentation).  metrics[ATTN_SIM_METRICS] receives, per allocator: rejected
 * starts, dropped requests, peak reserved tokens, and the sums over events of
 * reserved and of stored tokens (utilisation = stored sum / reserved sum), plus
 * the contiguous external-fragmentation sum.
 */
enum {
  ATTN_SIM_PAGED_REJECTED = 0,
  ATTN_SIM_PAGED_DROPPED = 1,
  ATTN_SIM_PAGED_PEAK_RESERVED = 2,
  ATTN_SIM_PAGED_SUM_RESERVED = 3,
  ATTN_SIM_PAGED_SUM_STORED = 4,
  ATTN_SIM_CONTIG_REJECTED = 5,
  ATTN_SIM_CONTIG_DROPPED = 6,
  ATTN_SIM_CONTIG_PEAK_RESERVED = 7,
  ATTN_SIM_CONTIG_SUM_RESERVED = 8,
  ATTN_SIM_CONTIG_SUM_STORED = 9,
  ATTN_SIM_CONTIG_SUM_EXTERNAL = 10,
  ATTN_SIM_METRICS = 11
};
ATTN_API int attn_pool_simulate(const int32_t* events, int n_events, int64_t arena_tokens, int block_tokens,
                                int64_t reserve_tokens, int64_t* metrics);

#ifdef __cplusplus
}
#endif

#endif /* KVATTN_ATTN_H */
