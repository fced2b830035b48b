// KV-cache append: write the K and V rows of T new tokens at positions
// cache_lens[b] .. cache_lens[b] + T - 1 of a contiguous cache or a paged pool.
//
// Method: "大模型面試笔记——Attention篇" section 4 (x_K <- Concat(x_K, t W_K),
// x_V <- Concat(x_V, t W_V)); paged placement per the PagedAttention section of
// the "KV cache, flash attention" lesson (16-token blocks behind a page table).
// Each (b, t, g) row is d bf16 values = d/8 16-byte vectors; one thread moves one
// vector of K and the matching vector of V with 128-bit loads and stores.
#include "internal.h"
#include "ptx.cuh"

namespace kvattn {
namespace {

__global__ void __launch_bounds__(256) kv_append_kernel(AppendLaunch a, int paged) {
  const int vec_per_row = a.d / 8;
  const long long total = (long long)a.B * a.T * a.Hkv * vec_per_row;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int vec = (int)(idx % vec_per_row);
  const long long row = idx / vec_per_row;                 // (b, t, g) row-major
  const int g = (int)(row % a.Hkv);
  const int t = (int)((row / a.Hkv) % a.T);
  const int b = (int)(row / ((long long)a.Hkv * a.T));
  const long long pos = (long long)a.cache_lens[b] + t;

  long long dst_row;   // row index in units of d elements, in the [rows, Hkv, d] view
  if (!paged) {
    if (pos < 0 || pos >= a.capacity) {
      if (vec == 0) atomicOr(a.status, DEV_APPEND_RANGE);
      return;
    }
    dst_row = ((long long)b * a.capacity + pos) * a.Hkv + g;
  } else {
    const long long blk_idx = pos / kPageTokens;
    if (pos < 0 || blk_idx >= a.max_blocks) {
      if (vec == 0) atomicOr(a.status, DEV_APPEND_RANGE);
      return;
    }
    const int blk = a.page_table[(long long)b * a.max_blocks + blk_idx];
    if (blk < 0 || blk >= a.num_blocks) {
      if (vec == 0) atomicOr(a.status, DEV_PAGE_ID);
      return;
    }
    dst_row = ((long long)blk * kPageTokens + pos % kPageTokens) * a.Hkv + g;
  }
  const uint4* ks = reinterpret_cast<const uint4*>(a.k_new) + row * vec_per_row + vec;
  const uint4* vs = reinterpret_cast<const uint4*>(a.v_new) + row * vec_per_row + vec;
  uint4* kd = reinterpret_cast<uint4*>(a.k) + dst_row * vec_per_row + vec;
  uint4* vd = reinterpret_cast<uint4*>(a.v) + dst_row * vec_per_row + vec;
  *kd = __ldg(ks);
  *vd = __ldg(vs);
}

}  // namespace

cudaError_t launch_append(const AppendLaunch& a, cudaStream_t stream) {
  const long long total = (long long)a.B * a.T * a.Hkv * (a.d / 8);
  const int threads = 256;
  const long long blocks = (total + threads - 1) / threads;
  kv_append_kernel<<<(unsigned)blocks, threads, 0, stream>>>(a, a.page_table != nullptr ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace kvattn
