// Launchers shared between the C-ABI layer (api.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace kvattn {

constexpr int kPageTokens = 16;   // tokens per physical KV block
constexpr int kDecodeTile = 64;   // tokens per pipeline stage of the warp-MMA decode kernel
constexpr int kDecodeTcTile = 64;  // tokens per K/V tile of the tensor-core decode kernel
// Above this many query rows per KV head the tensor-core kernel runs (bf16
// caches).  Measured on B200 (paged Llama decode, 8 KV heads x 8 sequences):
// 32 rows ran at 5.7 TB/s there against 4.5 TB/s on the warp-MMA kernel, whose
// row groups each re-read the K/V fragments; up to 16 rows the warp-MMA kernel
// streams at the HBM rate.
constexpr int kDecodeMmaRows = 16;
// FP8 caches run the warp-MMA kernels up to this many rows per KV head, and the
// tensor-core kernel (converting each e4m3 tile to f16 in shared memory) above.
constexpr int kFp8MaxRows = 32;
// Whether attn_decode runs the tensor-core split kernel for R rows per KV head.
inline bool decode_uses_tc(int R, bool fp8) { return R > (fp8 ? kFp8MaxRows : kDecodeMmaRows); }

// Balanced split of the tensor-core decode kernel.  With one fixed chunk length the
// number of chunks of each sequence is its length rounded up, and the total over the
// batch falls anywhere against the 2 CTAs x SMs slots: measured on B200 (paged Llama
// decode, 8 x 8 sequence-heads, lengths 32K-131K, 4 seeds), one split count ran at
// 94-101 % of the HBM copy rate where the items came to just under a whole number of
// slot waves and at 62-80 % just over one.  The host knows only max_seqlen, so the
// kernel itself apportions kBalancedItemsPerSlot x slots chunks over the sequences in
// proportion to their lengths (at least one each, the rest by largest remainder), each
// sequence cut into its own number of equal chunks.
constexpr int kDecodeTcCtasPerSm = 2;      // shared memory and TMEM of one tensor-core decode CTA
constexpr int kBalancedItemsPerSlot = 2;
// Longest key range one decode call accepts (max_seqlen_k): keeps every token offset,
// chunk start and chunk end of the decode kernels inside int.
constexpr int kMaxDecodeSeqlen = 1 << 30;
constexpr int kBalancedMaxB = 128;         // the plan is built per CTA in shared memory
// Whether attn_decode with these sizes uses the balanced split (automatic splitting, the
// tensor-core kernel, one row tile per KV head).
inline bool decode_balanced(int B, int T, int G, int num_splits, bool fp8) {
  return num_splits == 0 && B <= kBalancedMaxB && decode_uses_tc(G * T, fp8) && G * T <= 128;
}
// Chunks over the whole batch (per KV head) of the balanced split on the current device.
int decode_balanced_chunks(int B, int Hkv);

// One CTA whose thread waits on an mbarrier nothing arrives at (bounded like every
// wait of the library) and then sets DEV_TIMEOUT (csrc/selftest.cu).
cudaError_t launch_wait_timeout_selftest(unsigned* status, cudaStream_t stream);

struct DecodeLaunch {
  const void* q;
  const void* k;          // contiguous cache or paged pool
  const void* v;
  const int32_t* seqlens;
  const int32_t* page_table;  // nullptr = contiguous
  int max_blocks, num_blocks, capacity, max_seqlen;
  void* o;
  int o_bf16;
  float* lse;
  int B, T, Hq, Hkv, d;
  float scale;
  int causal;
  int chunk;          // tokens per split (multiple of kDecodeTile)
  int max_chunks;     // ceil(max_seqlen / chunk)
  float* part_o;      // [B, Hkv, max_chunks, R, d]; balanced: [n_chunks * Hkv, R, d]
  float* part_lse;    // [B, Hkv, max_chunks, R];    balanced: [n_chunks * Hkv, R]
  unsigned* status;
  // balanced split (decode_balanced): chunks over the batch, and the per-sequence plan
  // (first chunk, chunks, chunk length) the split kernel writes for the combine
  int balanced = 0, n_chunks = 0;
  int* plan = nullptr;   // [B, 3]
  int fp8 = 0;                    // k/v hold e4m3 codes with per-KV-head scales
  const float* k_scale = nullptr;  // [Hkv]
  const float* v_scale = nullptr;
};

struct PrefillLaunch {
  const void* q;
  const void* k;          // dense [B, N, Hkv, d], or a contiguous cache / paged pool
  const void* v;
  void* o;
  int o_bf16;
  float* lse;
  int B, Hq, Hkv, N, d;   // N: queries per sequence
  float scale;
  int causal;
  unsigned* status;
  // prefill against an existing cache (seqlens == nullptr: dense K/V of N keys)
  const int32_t* seqlens = nullptr;     // [B] keys per sequence, including the N new ones
  const int32_t* page_table = nullptr;  // [B, max_blocks], or nullptr for a contiguous cache
  int capacity = 0, max_blocks = 0, num_blocks = 0;
  int max_seqlen = 0;   // > 0: lengths above it are invalid too (attn_decode's max_seqlen_k)
};

// attn_decode with at least this many new tokens (bf16 cache, automatic splitting)
// runs the prefill kernel's cached form: measured on B200 (Llama heads, 4K-16K cached
// keys, B 4 and 16, paged and contiguous), the split tensor-core path was faster up to
// T = 128 (decode 557-867 against 429-618 TFLOP/s) and slower from T = 256 (729-901
// against 873-1176), where each sequence has whole 256-row query blocks to stream.
constexpr int kDecodeViaPrefillT = 256;

struct AppendLaunch {
  void* k;
  void* v;
  const void* k_new;
  const void* v_new;
  const int32_t* cache_lens;
  const int32_t* page_table;
  int max_blocks, num_blocks, capacity;
  int B, T, Hkv, d;
  unsigned* status;
  int fp8 = 0;                    // quantise the new rows to e4m3 with per-KV-head scales
  const float* k_scale = nullptr;
  const float* v_scale = nullptr;
};

// Tokens per split for attn_decode (host heuristic, deterministic in its inputs).
// fp8: the call reads an FP8 cache (its kernels want other chunk lengths).
int decode_chunk_tokens(int B, int T, int G, int Hkv, int max_seqlen, int num_splits, bool fp8);

// Tokens per row tile of the tensor-core decode kernel (G query heads per KV head):
// as many whole tokens as fit in 128 rows, at most T.
inline int decode_tc_tile_tokens(int T, int G) { return T < 128 / G ? T : 128 / G; }
// Row tiles per KV head (1 unless the rows exceed one 128-row tensor-core tile).
inline int decode_row_tiles(int T, int G) {
  if (G * T <= kDecodeMmaRows) return 1;
  const int tt = decode_tc_tile_tokens(T, G);
  return (T + tt - 1) / tt;
}

// Encode a rank-N (1..5) tiled tensor map with 128-byte swizzle over bf16
// (elem_bytes 2) or bytes (elem_bytes 1); strides in bytes for dims 1..N-1.
// Returns 0 on success.
int encode_tmap_nd(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims,
                   const cuuint64_t* strides_bytes, const cuuint32_t* box, int elem_bytes = 2);

// Encode a 3-D tiled tensor map {inner, mid, rows} with 128-byte swizzle.
// Strides are in bytes for dims 1 and 2.  Returns 0 on success.
int encode_tmap_3d(CUtensorMap* map, const void* base, uint64_t dim0, uint64_t dim1, uint64_t dim2,
                   uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box0, uint32_t box1, uint32_t box2,
                   int elem_bytes = 2);

// Device address, on the current device, of the static array attn_decode_noalloc keeps
// its partials in (ATTN_DECODE_NOALLOC_SCRATCH_BYTES), or nullptr if it cannot be had.
void* noalloc_scratch();

cudaError_t launch_decode(const DecodeLaunch& a, cudaStream_t stream);
// tcgen05 split kernel for more than 16 query rows per KV head (K/V maps with 128-row boxes when contiguous)
cudaError_t launch_decode_tc(const DecodeLaunch& a, const CUtensorMap& tk, const CUtensorMap& tv, cudaStream_t stream);
cudaError_t launch_append(const AppendLaunch& a, cudaStream_t stream);
cudaError_t launch_prefill(const PrefillLaunch& a, cudaStream_t stream);
// copy n whole blocks (src[i] -> dst[i], device id lists) of both pools
cudaError_t launch_copy_blocks(void* k, void* v, const int32_t* src, const int32_t* dst, int n, int num_blocks,
                               int block_bytes, unsigned* status, cudaStream_t stream);

}  // namespace kvattn
