// Pieces shared by the split-KV decode kernels (decode.cu, decode_fp8.cu): the
// launch parameters, the length check, and the TMA producer loop that streams a
// work item's 64-token K/V tiles into a shared-memory ring.
#pragma once

#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace kvattn {

struct SplitParams {
  const __nv_bfloat16* q;
  const float* k_scale;   // FP8 caches: per-KV-head scales (else unused)
  const float* v_scale;
  const int32_t* seqlens;
  const int32_t* page_table;
  float* part_o;
  float* part_lse;
  unsigned* status;
  int T, Hq, Hkv, G, R;
  int chunk, max_chunks, capacity, max_blocks, num_blocks, max_seqlen;
  float scale_log2;
  int causal;
  int balanced = 0;            // tensor-core balanced split: partials indexed by the plan
  const int* plan = nullptr;   // [B, 3]: first chunk, chunks, chunk length per sequence
};

__device__ __forceinline__ bool seqlen_bad(int L, int T, int max_seqlen, bool paged, int capacity, int max_blocks) {
  if (L < T || L > max_seqlen) return true;
  if (!paged && L > capacity) return true;
  if (paged && (L + kPageTokens - 1) / kPageTokens > max_blocks) return true;
  return false;
}

// One thread: tiles 0 .. n_tiles-1 of keys [tok_begin, tok_end) into the ring of
// C::kStages stages (K then V, C::kHalves 128-byte swizzle spans per token row;
// contiguous: one 64-row box per span; paged: one 16-row box per physical
// block, its page-table entry bounds-checked first), evict-first L2 policy.  A
// stage is refilled once the consumers released it (empty barrier); a wait that
// gives up sets DEV_TIMEOUT and the abort flag.
template <class C, bool PAGED>
__device__ __forceinline__ void produce_split_tiles(uint8_t* smem, uint64_t* full, uint64_t* empty,
                                                    const CUtensorMap* tmK, const CUtensorMap* tmV,
                                                    const SplitParams& p, int b, int g, int tok_begin, int tok_end,
                                                    int n_tiles, int* abort_flag) {
  prefetch_tmap(tmK);
  prefetch_tmap(tmV);
  const uint64_t pol = policy_evict_first();
  for (int i = 0; i < n_tiles; ++i) {
    const int s = i % C::kStages;
    if (i >= C::kStages && !mbar_wait(&empty[s], ((i / C::kStages) - 1) & 1)) {
      atomicOr(p.status, DEV_TIMEOUT);
      *reinterpret_cast<volatile int*>(abort_flag) = 1;
      break;
    }
    uint8_t* kst = smem + s * C::kStageBytes;
    uint8_t* vst = kst + C::kTensorBytes;
    const int t0 = tok_begin + i * kDecodeTile;
    if (!PAGED) {
      mbar_arrive_expect_tx(&full[s], C::kStageBytes);
      const int row = b * p.capacity + t0;
#pragma unroll
      for (int h = 0; h < C::kHalves; ++h) {
        tma_load_3d(kst + h * C::kHalfBytes, tmK, &full[s], h * 64, g, row, pol);
        tma_load_3d(vst + h * C::kHalfBytes, tmV, &full[s], h * 64, g, row, pol);
      }
    } else {
      constexpr int kBlocks = kDecodeTile / kPageTokens;
      const int nb = min(kBlocks, (tok_end - t0 + kPageTokens - 1) / kPageTokens);
      const int32_t* row_tab = p.page_table + (size_t)b * p.max_blocks + t0 / kPageTokens;
      // read the stage's block ids together: the copies' memory clobbers would
      // otherwise serialise one table read per block
      int ids[kBlocks];
#pragma unroll
      for (int j = 0; j < kBlocks; ++j) ids[j] = j < nb ? __ldg(row_tab + j) : 0;
      mbar_arrive_expect_tx(&full[s], nb * 2 * C::kHalves * kPageTokens * 128);
#pragma unroll
      for (int j = 0; j < kBlocks; ++j) {
        if (j >= nb) break;
        int blk = ids[j];
        if (blk < 0 || blk >= p.num_blocks) {
          atomicOr(p.status, DEV_PAGE_ID);
          blk = 0;   // keep the byte count; the result is flagged invalid
        }
#pragma unroll
        for (int h = 0; h < C::kHalves; ++h) {
          tma_load_3d(kst + h * C::kHalfBytes + j * kPageTokens * 128, tmK, &full[s], h * 64, g, blk * kPageTokens,
                      pol);
          tma_load_3d(vst + h * C::kHalfBytes + j * kPageTokens * 128, tmV, &full[s], h * 64, g, blk * kPageTokens,
                      pol);
        }
      }
    }
  }
}

// FP8 caches, at most 8 query rows per KV head: the transposed-product split kernel (decode_fp8.cu)
cudaError_t launch_decode_fp8_rows8(const CUtensorMap& tk, const CUtensorMap& tv, const SplitParams& sp, int B,
                                    bool paged, cudaStream_t stream);

}  // namespace kvattn
