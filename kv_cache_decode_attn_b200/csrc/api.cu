// C ABI of the attention library: argument checks, workspace layout, tensor-map
// encoding and kernel dispatch.  The declarations and their contracts are in
// include/attn.h.  Nothing here allocates device memory.
#include <cudaTypedefs.h>
#include <math.h>
#include <stdio.h>
#include <stdlib.h>

#include <mutex>

#include "../../include/attn.h"
#include "internal.h"

namespace kvattn {

// Sticky device status word (ATTN_DEV_* bits), one per device that loads the library.
__device__ unsigned g_status_word;

namespace {

constexpr int kMaxDevices = 64;

unsigned* status_ptr() {
  static unsigned* ptrs[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<unsigned*>(p);
  }
  return ptrs[dev];
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

int encode_tmap_nd(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims,
                   const cuuint64_t* strides_bytes, const cuuint32_t* box, int elem_bytes) {
  auto fn = get_encode_fn();
  if (!fn || rank < 1 || rank > 5 || (elem_bytes != 1 && elem_bytes != 2)) return 1;
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUtensorMapDataType dt = elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUresult r = fn(map, dt, (cuuint32_t)rank, const_cast<void*>(base), dims,
                  strides_bytes, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : 1;
}

int encode_tmap_3d(CUtensorMap* map, const void* base, uint64_t dim0, uint64_t dim1, uint64_t dim2,
                   uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box0, uint32_t box1, uint32_t box2,
                   int elem_bytes) {
  cuuint64_t dims[3] = {dim0, dim1, dim2};
  cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  cuuint32_t box[3] = {box0, box1, box2};
  return encode_tmap_nd(map, base, 3, dims, strides, box, elem_bytes);
}

}  // namespace kvattn

using namespace kvattn;

namespace {

struct DecodeLayout {
  int R, chunk, max_chunks;
  int balanced, n_chunks;   // balanced split: chunks over the batch (per KV head)
  size_t o_bytes, lse_offset, plan_offset, total;
};

bool decode_layout(int B, int T, int Hq, int Hkv, int d, int max_seqlen_k, int num_splits, bool fp8,
                   DecodeLayout* out) {
  if (B < 1 || T < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || max_seqlen_k < 1 || num_splits < 0) return false;
  if (max_seqlen_k > kMaxDecodeSeqlen) return false;
  if (d != 64 && d != 128) return false;
  DecodeLayout L;
  L.R = (Hq / Hkv) * T;
  L.chunk = decode_chunk_tokens(B, T, Hq / Hkv, Hkv, max_seqlen_k, num_splits, fp8);
  L.max_chunks = (int)(((long long)max_seqlen_k + L.chunk - 1) / L.chunk);
  L.balanced = decode_balanced(B, T, Hq / Hkv, num_splits, fp8) ? 1 : 0;
  L.n_chunks = 0;
  size_t items = (size_t)B * Hkv * L.max_chunks;
  if (L.balanced) {
    // every sequence gets at least one chunk of the batch's n_chunks
    L.n_chunks = decode_balanced_chunks(B, Hkv);
    L.max_chunks = L.n_chunks - B + 1;   // most chunks one (sequence, KV head) can get
    items = (size_t)L.n_chunks * Hkv;
  }
  L.o_bytes = items * L.R * d * sizeof(float);
  L.lse_offset = (L.o_bytes + 255) & ~size_t(255);
  L.plan_offset = (L.lse_offset + items * L.R * sizeof(float) + 255) & ~size_t(255);
  L.total = L.plan_offset + (L.balanced ? (size_t)B * 3 * sizeof(int) : 0);
  *out = L;
  return true;
}

// With KVATTN_DEBUG set in the environment, CUDA failures are also printed to stderr.
int cuda_status(cudaError_t e, const char* where) {
  if (e == cudaSuccess) return ATTN_OK;
  static const bool debug = getenv("KVATTN_DEBUG") != nullptr;
  if (debug) fprintf(stderr, "[kvattn] %s: %s (%d)\n", where, cudaGetErrorString(e), (int)e);
  return ATTN_ERR_CUDA;
}

}  // namespace

extern "C" {

const char* attn_status_string(int status) {
  switch (status) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported configuration";
    case ATTN_ERR_WORKSPACE: return "workspace missing or too small";
    case ATTN_ERR_CUDA: return "CUDA error";
    case ATTN_ERR_DEVICE: return "device-side error flagged";
    case ATTN_ERR_NO_BLOCKS: return "block pool exhausted";
    default: return "unknown status";
  }
}

int64_t kv_cache_bytes(int n_layers, int batch, int64_t tokens, int n_kv_heads, int head_dim, int elem_bytes) {
  if (n_layers <= 0 || batch <= 0 || tokens <= 0 || n_kv_heads <= 0 || head_dim <= 0 || elem_bytes <= 0) return -1;
  const int64_t factors[6] = {n_layers, batch, tokens, n_kv_heads, head_dim, elem_bytes};
  int64_t r = 2;
  for (int i = 0; i < 6; ++i) {
    if (r > INT64_MAX / factors[i]) return -1;
    r *= factors[i];
  }
  return r;
}

int attn_get_device_status(int clear) {
  unsigned* p = status_ptr();
  if (!p) return ATTN_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return ATTN_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpy(&v, p, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return ATTN_ERR_CUDA;
  if (clear) {
    const unsigned zero = 0;
    if (cudaMemcpy(p, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return ATTN_ERR_CUDA;
  }
  return (int)v;
}

size_t attn_decode_workspace_bytes(int B, int T, int Hq, int Hkv, int d, int max_seqlen_k, int num_splits) {
  // enough for attn_decode and for attn_decode_fp8 with the same arguments (their chunking differs)
  DecodeLayout L, L8;
  if (!decode_layout(B, T, Hq, Hkv, d, max_seqlen_k, num_splits, false, &L)) return 0;
  if (!decode_layout(B, T, Hq, Hkv, d, max_seqlen_k, num_splits, true, &L8)) return 0;
  return L.total > L8.total ? L.total : L8.total;
}

int attn_prefill(const void* q, const void* k, const void* v, void* o, int o_dtype, float* lse, int B, int Hq,
                 int Hkv, int N, int d, float scale, int causal, void* stream) {
  if (!q || !k || !v || !o) return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || Hq % Hkv) return ATTN_ERR_INVALID_ARG;
  if (o_dtype != ATTN_F32 && o_dtype != ATTN_BF16) return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale) || (causal != 0 && causal != 1)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_ERR_INVALID_ARG;
  if ((long long)B * N * Hq > INT32_MAX || (long long)B * N * Hkv > INT32_MAX) return ATTN_ERR_UNSUPPORTED;
  unsigned* st = status_ptr();
  if (!st) return ATTN_ERR_CUDA;
  PrefillLaunch a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.o_bf16 = o_dtype == ATTN_BF16;
  a.lse = lse;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.N = N;
  a.d = d;
  a.scale = scale;
  a.causal = causal;
  a.status = st;
  return cuda_status(launch_prefill(a, static_cast<cudaStream_t>(stream)), "attn_prefill");
}

}  // extern "C"

namespace {

int decode_impl(const void* q, const void* k_cache, const void* v_cache, const float* k_scale, const float* v_scale,
                bool fp8, const int32_t* seqlens_k, const int32_t* page_table, int max_blocks_per_seq,
                int num_blocks, int cache_capacity, int max_seqlen_k, void* o, int o_dtype, float* lse, int B, int T,
                int Hq, int Hkv, int d, float scale, int causal, int num_splits, void* workspace,
                size_t workspace_bytes, void* stream, const char* name, bool static_scratch = false) {
  if (!q || !k_cache || !v_cache || !seqlens_k || !o) return ATTN_ERR_INVALID_ARG;
  if (fp8 && (!k_scale || !v_scale)) return ATTN_ERR_INVALID_ARG;
  if (B < 1 || T < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || num_splits < 0) return ATTN_ERR_INVALID_ARG;
  if (o_dtype != ATTN_F32 && o_dtype != ATTN_BF16) return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale) || (causal != 0 && causal != 1)) return ATTN_ERR_INVALID_ARG;
  const bool paged = page_table != nullptr;
  int capacity_tokens;
  if (paged) {
    if (max_blocks_per_seq < 1 || num_blocks < 1) return ATTN_ERR_INVALID_ARG;
    if ((long long)num_blocks * kPageTokens > INT32_MAX) return ATTN_ERR_UNSUPPORTED;
    capacity_tokens = (int)std::min<long long>((long long)max_blocks_per_seq * kPageTokens, INT32_MAX);
  } else {
    if (cache_capacity < 1) return ATTN_ERR_INVALID_ARG;
    if ((long long)B * cache_capacity > INT32_MAX) return ATTN_ERR_UNSUPPORTED;
    capacity_tokens = cache_capacity;
  }
  if (max_seqlen_k == 0) max_seqlen_k = std::min(capacity_tokens, kMaxDecodeSeqlen);
  if (max_seqlen_k < T || max_seqlen_k > capacity_tokens) return ATTN_ERR_INVALID_ARG;
  if (max_seqlen_k > kMaxDecodeSeqlen) return ATTN_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (Hq / Hkv > 128) return ATTN_ERR_UNSUPPORTED;                       // one token's heads must fit a row tile
  if (fp8 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o)) return ATTN_ERR_INVALID_ARG;
  DecodeLayout L;
  if (!decode_layout(B, T, Hq, Hkv, d, max_seqlen_k, num_splits, fp8, &L)) return ATTN_ERR_INVALID_ARG;
  if (workspace_bytes < L.total) return ATTN_ERR_WORKSPACE;
  if (static_scratch) {
    // attn_decode_noalloc: the library's own array, looked up only once the request is known to be valid
    workspace = noalloc_scratch();
    if (!workspace) return ATTN_ERR_CUDA;
  }
  if (!workspace || !aligned16(workspace)) return ATTN_ERR_WORKSPACE;
  unsigned* st = status_ptr();
  if (!st) return ATTN_ERR_CUDA;
  if (!fp8 && num_splits == 0 && T >= kDecodeViaPrefillT && (long long)B * T * Hq <= INT32_MAX) {
    // a prompt chunk against a cached prefix: the prefill kernel's cached form computes the
    // same rows (bottom-right causal alignment, the same length rules with max_seqlen_k) faster;
    // the workspace goes unused
    PrefillLaunch pa;
    pa.q = q;
    pa.k = k_cache;
    pa.v = v_cache;
    pa.o = o;
    pa.o_bf16 = o_dtype == ATTN_BF16;
    pa.lse = lse;
    pa.B = B;
    pa.Hq = Hq;
    pa.Hkv = Hkv;
    pa.N = T;
    pa.d = d;
    pa.scale = scale;
    pa.causal = causal;
    pa.status = st;
    pa.seqlens = seqlens_k;
    pa.page_table = page_table;
    pa.capacity = cache_capacity;
    pa.max_blocks = max_blocks_per_seq;
    pa.num_blocks = num_blocks;
    pa.max_seqlen = max_seqlen_k;
    return cuda_status(launch_prefill(pa, static_cast<cudaStream_t>(stream)), name);
  }
  DecodeLaunch a;
  a.q = q;
  a.k = k_cache;
  a.v = v_cache;
  a.seqlens = seqlens_k;
  a.page_table = page_table;
  a.max_blocks = max_blocks_per_seq;
  a.num_blocks = num_blocks;
  a.capacity = cache_capacity;
  a.max_seqlen = max_seqlen_k;
  a.o = o;
  a.o_bf16 = o_dtype == ATTN_BF16;
  a.lse = lse;
  a.B = B;
  a.T = T;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.d = d;
  a.scale = scale;
  a.causal = causal;
  a.chunk = L.chunk;
  a.max_chunks = L.max_chunks;
  a.part_o = static_cast<float*>(workspace);
  a.part_lse = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + L.lse_offset);
  a.balanced = L.balanced;
  a.n_chunks = L.n_chunks;
  a.plan = L.balanced ? reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + L.plan_offset) : nullptr;
  a.status = st;
  a.fp8 = fp8 ? 1 : 0;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  return cuda_status(launch_decode(a, static_cast<cudaStream_t>(stream)), name);
}

int append_impl(void* k_cache, void* v_cache, const void* k_new, const void* v_new, const float* k_scale,
                const float* v_scale, bool fp8, const int32_t* cache_lens, const int32_t* page_table,
                int max_blocks_per_seq, int num_blocks, int cache_capacity, int B, int T, int Hkv, int d, void* stream,
                const char* name) {
  if (!k_cache || !v_cache || !k_new || !v_new || !cache_lens) return ATTN_ERR_INVALID_ARG;
  if (fp8 && (!k_scale || !v_scale)) return ATTN_ERR_INVALID_ARG;
  if (B < 1 || T < 1 || Hkv < 1) return ATTN_ERR_INVALID_ARG;
  if (page_table) {
    if (max_blocks_per_seq < 1 || num_blocks < 1) return ATTN_ERR_INVALID_ARG;
  } else if (cache_capacity < 1) {
    return ATTN_ERR_INVALID_ARG;
  }
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k_new) || !aligned16(v_new))
    return ATTN_ERR_INVALID_ARG;
  unsigned* st = status_ptr();
  if (!st) return ATTN_ERR_CUDA;
  AppendLaunch a;
  a.k = k_cache;
  a.v = v_cache;
  a.k_new = k_new;
  a.v_new = v_new;
  a.cache_lens = cache_lens;
  a.page_table = page_table;
  a.max_blocks = max_blocks_per_seq;
  a.num_blocks = num_blocks;
  a.capacity = cache_capacity;
  a.B = B;
  a.T = T;
  a.Hkv = Hkv;
  a.d = d;
  a.status = st;
  a.fp8 = fp8 ? 1 : 0;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  return cuda_status(launch_append(a, static_cast<cudaStream_t>(stream)), name);
}

}  // namespace

extern "C" {

int attn_prefill_cache(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens_k,
                       const int32_t* page_table, int max_blocks_per_seq, int num_blocks, int cache_capacity, void* o,
                       int o_dtype, float* lse, int B, int Nq, int Hq, int Hkv, int d, float scale, int causal,
                       void* stream) {
  if (!q || !k_cache || !v_cache || !seqlens_k || !o) return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Nq < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv) return ATTN_ERR_INVALID_ARG;
  if (o_dtype != ATTN_F32 && o_dtype != ATTN_BF16) return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale) || (causal != 0 && causal != 1)) return ATTN_ERR_INVALID_ARG;
  if (page_table) {
    if (max_blocks_per_seq < 1 || num_blocks < 1) return ATTN_ERR_INVALID_ARG;
    if ((long long)num_blocks * kPageTokens > INT32_MAX || (long long)max_blocks_per_seq * kPageTokens > INT32_MAX)
      return ATTN_ERR_UNSUPPORTED;
    if ((long long)max_blocks_per_seq * kPageTokens < Nq) return ATTN_ERR_INVALID_ARG;
  } else {
    if (cache_capacity < Nq) return ATTN_ERR_INVALID_ARG;
  }
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o)) return ATTN_ERR_INVALID_ARG;
  if ((long long)B * Nq * Hq > INT32_MAX) return ATTN_ERR_UNSUPPORTED;
  unsigned* st = status_ptr();
  if (!st) return ATTN_ERR_CUDA;
  PrefillLaunch a;
  a.q = q;
  a.k = k_cache;
  a.v = v_cache;
  a.o = o;
  a.o_bf16 = o_dtype == ATTN_BF16;
  a.lse = lse;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.N = Nq;
  a.d = d;
  a.scale = scale;
  a.causal = causal;
  a.status = st;
  a.seqlens = seqlens_k;
  a.page_table = page_table;
  a.capacity = cache_capacity;
  a.max_blocks = max_blocks_per_seq;
  a.num_blocks = num_blocks;
  return cuda_status(launch_prefill(a, static_cast<cudaStream_t>(stream)), "attn_prefill_cache");
}

int attn_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens_k,
                const int32_t* page_table, int max_blocks_per_seq, int num_blocks, int cache_capacity,
                int max_seqlen_k, void* o, int o_dtype, float* lse, int B, int T, int Hq, int Hkv, int d,
                float scale, int causal, int num_splits, void* workspace, size_t workspace_bytes, void* stream) {
  return decode_impl(q, k_cache, v_cache, nullptr, nullptr, false, seqlens_k, page_table, max_blocks_per_seq,
                     num_blocks, cache_capacity, max_seqlen_k, o, o_dtype, lse, B, T, Hq, Hkv, d, scale, causal,
                     num_splits, workspace, workspace_bytes, stream, "attn_decode");
}

int attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens_k,
                        const int32_t* page_table, int max_blocks_per_seq, int num_blocks, int cache_capacity,
                        int max_seqlen_k, void* o, int o_dtype, float* lse, int B, int T, int Hq, int Hkv, int d,
                        float scale, int causal, int num_splits, void* stream) {
  return decode_impl(q, k_cache, v_cache, nullptr, nullptr, false, seqlens_k, page_table, max_blocks_per_seq,
                     num_blocks, cache_capacity, max_seqlen_k, o, o_dtype, lse, B, T, Hq, Hkv, d, scale, causal,
                     num_splits, nullptr, ATTN_DECODE_NOALLOC_SCRATCH_BYTES, stream, "attn_decode_noalloc", true);
}

int attn_decode_fp8(const void* q, const void* k_cache, const void* v_cache, const float* k_scale,
                    const float* v_scale, const int32_t* seqlens_k, const int32_t* page_table, int max_blocks_per_seq,
                    int num_blocks, int cache_capacity, int max_seqlen_k, void* o, int o_dtype, float* lse, int B,
                    int T, int Hq, int Hkv, int d, float scale, int causal, int num_splits, void* workspace,
                    size_t workspace_bytes, void* stream) {
  return decode_impl(q, k_cache, v_cache, k_scale, v_scale, true, seqlens_k, page_table, max_blocks_per_seq,
                     num_blocks, cache_capacity, max_seqlen_k, o, o_dtype, lse, B, T, Hq, Hkv, d, scale, causal,
                     num_splits, workspace, workspace_bytes, stream, "attn_decode_fp8");
}

int kv_append(void* k_cache, void* v_cache, const void* k_new, const void* v_new, const int32_t* cache_lens,
              const int32_t* page_table, int max_blocks_per_seq, int num_blocks, int cache_capacity, int B, int T,
              int Hkv, int d, void* stream) {
  return append_impl(k_cache, v_cache, k_new, v_new, nullptr, nullptr, false, cache_lens, page_table,
                     max_blocks_per_seq, num_blocks, cache_capacity, B, T, Hkv, d, stream, "kv_append");
}

int attn_copy_blocks(void* k_pool, void* v_pool, const int32_t* src, const int32_t* dst, int n, int num_blocks,
                     int Hkv, int d, int elem_bytes, void* stream) {
  if (!k_pool || !v_pool || n < 0 || num_blocks < 1 || Hkv < 1) return ATTN_ERR_INVALID_ARG;
  if (n > 0 && (!src || !dst)) return ATTN_ERR_INVALID_ARG;
  if (n > 65535) return ATTN_ERR_UNSUPPORTED;
  if ((d != 64 && d != 128) || (elem_bytes != 1 && elem_bytes != 2)) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(k_pool) || !aligned16(v_pool)) return ATTN_ERR_INVALID_ARG;
  if (n == 0) return ATTN_OK;
  const long long block_bytes = (long long)kPageTokens * Hkv * d * elem_bytes;
  if (block_bytes / 16 > INT32_MAX) return ATTN_ERR_UNSUPPORTED;
  unsigned* st = status_ptr();
  if (!st) return ATTN_ERR_CUDA;
  return cuda_status(launch_copy_blocks(k_pool, v_pool, src, dst, n, num_blocks, (int)block_bytes, st,
                                        static_cast<cudaStream_t>(stream)),
                     "attn_copy_blocks");
}

int attn_selftest_wait_timeout(void* stream) {
  unsigned* st = status_ptr();
  if (!st) return ATTN_ERR_CUDA;
  return cuda_status(launch_wait_timeout_selftest(st, static_cast<cudaStream_t>(stream)),
                     "attn_selftest_wait_timeout");
}

int kv_append_fp8(void* k_cache, void* v_cache, const void* k_new, const void* v_new, const float* k_scale,
                  const float* v_scale, const int32_t* cache_lens, const int32_t* page_table, int max_blocks_per_seq,
                  int num_blocks, int cache_capacity, int B, int T, int Hkv, int d, void* stream) {
  return append_impl(k_cache, v_cache, k_new, v_new, k_scale, v_scale, true, cache_lens, page_table,
                     max_blocks_per_seq, num_blocks, cache_capacity, B, T, Hkv, d, stream, "kv_append_fp8");
}

}  // extern "C"
