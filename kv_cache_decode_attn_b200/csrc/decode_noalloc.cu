// attn_decode_noalloc: attn_decode with its partials in a file-scope device
// array instead of a caller-provided workspace, for callers that cannot
// allocate device memory (see include/attn.h).
#include <mutex>

#include "../../include/attn.h"
#include "internal.h"

namespace {

// Shared by every call on a device; held from the module's load until exit.
static __device__ __align__(256) unsigned char g_decode_scratch[ATTN_DECODE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

// Device address of g_decode_scratch on the current device, looked up once per
// device with that device current.  In host code the array's name is only a
// host-side stand-in: passing it to a kernel would read the wrong memory.
void* scratch_on_current_device() {
  static void* ptrs[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return nullptr;
    ptrs[dev] = p;
  }
  return ptrs[dev];
}

}  // namespace

extern "C" ATTN_API int attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                            const int32_t* seqlens_k, const int32_t* page_table,
                                            int max_blocks_per_seq, int num_blocks, int cache_capacity,
                                            int max_seqlen_k, void* o, int o_dtype, float* lse, int B, int T,
                                            int Hq, int Hkv, int d, float scale, int causal, int num_splits,
                                            void* stream) {
  // the key-length bound attn_decode will use (0 means the cache capacity)
  long long bound = max_seqlen_k;
  if (bound == 0) bound = page_table ? (long long)max_blocks_per_seq * kvattn::kPageTokens : cache_capacity;
  if (bound > 0 && bound <= INT32_MAX) {
    const size_t need = attn_decode_workspace_bytes(B, T, Hq, Hkv, d, (int)bound, num_splits);
    if (need > ATTN_DECODE_NOALLOC_SCRATCH_BYTES) return ATTN_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  if (q && k_cache && v_cache && seqlens_k && o) {   // argument errors are reported by attn_decode itself
    scratch = scratch_on_current_device();
    if (!scratch) return ATTN_ERR_CUDA;
  }
  return attn_decode(q, k_cache, v_cache, seqlens_k, page_table, max_blocks_per_seq, num_blocks, cache_capacity,
                     max_seqlen_k, o, o_dtype, lse, B, T, Hq, Hkv, d, scale, causal, num_splits, scratch,
                     ATTN_DECODE_NOALLOC_SCRATCH_BYTES, stream);
}
