// KV-cache append: write the K and V rows of T new tokens at positions
// cache_lens[b] .. cache_lens[b] + T - 1 of a contiguous cache or a paged pool.
//
// Method: "大模型面試笔记——Attention篇" section 4 (x_K <- Concat(x_K, t W_K),
// x_V <- Concat(x_V, t W_V)); paged placement per the PagedAttention section of
// the "KV cache, flash attention" lesson (16-token blocks behind a page table).
// Each (b, t, g) row is d bf16 values = d/8 16-byte vectors; one thread moves one
// vector of K and the matching vector of V with 128-bit loads and stores.
// FP8 caches (e4m3 codes, "KV cache, flash attention and inference optimisation"
// lesson, section "用它"): one thread quantises 16 values of K and of V, each
// divided by its KV head's scale in float32 (IEEE division) and rounded to the
// nearest e4m3 value with saturation to +-448, and stores 16 codes.
#include "internal.h"
#include "ptx.cuh"

namespace kvattn {
namespace {

// 16 bf16 values -> 16 e4m3 codes of x / s
__device__ __forceinline__ uint4 quantise16(const uint4* src, float s) {
  const uint4 lo = __ldg(src), hi = __ldg(src + 1);
  const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
  uint32_t out[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t codes[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t v = w[2 * i + h];
      const float x0 = __fdiv_rn(__uint_as_float(v << 16), s);
      const float x1 = __fdiv_rn(__uint_as_float(v & 0xffff0000u), s);
      codes[h] = f32x2_to_e4m3x2(x0, x1);
    }
    out[i] = codes[0] | (codes[1] << 16);
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

__global__ void __launch_bounds__(256) kv_append_kernel(AppendLaunch a, int paged) {
  const int vec_per_row = a.d / (a.fp8 ? 16 : 8);
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
  uint4* kd = reinterpret_cast<uint4*>(a.k) + dst_row * vec_per_row + vec;
  uint4* vd = reinterpret_cast<uint4*>(a.v) + dst_row * vec_per_row + vec;
  if (a.fp8) {
    // source: 16 bf16 = two 16-byte vectors per destination vector
    const uint4* ks = reinterpret_cast<const uint4*>(a.k_new) + (row * vec_per_row + vec) * 2;
    const uint4* vs = reinterpret_cast<const uint4*>(a.v_new) + (row * vec_per_row + vec) * 2;
    const float sk = __ldg(a.k_scale + g), sv = __ldg(a.v_scale + g);
    if (!(sk > 0.f && sk <= 3.402823466e38f && sv > 0.f && sv <= 3.402823466e38f)) {
      if (vec == 0) atomicOr(a.status, DEV_SCALE);
      return;
    }
    *kd = quantise16(ks, sk);
    *vd = quantise16(vs, sv);
    return;
  }
  const uint4* ks = reinterpret_cast<const uint4*>(a.k_new) + row * vec_per_row + vec;
  const uint4* vs = reinterpret_cast<const uint4*>(a.v_new) + row * vec_per_row + vec;
  *kd = __ldg(ks);
  *vd = __ldg(vs);
}

}  // namespace

cudaError_t launch_append(const AppendLaunch& a, cudaStream_t stream) {
  const long long total = (long long)a.B * a.T * a.Hkv * (a.d / (a.fp8 ? 16 : 8));
  const int threads = 256;
  const long long blocks = (total + threads - 1) / threads;
  kv_append_kernel<<<(unsigned)blocks, threads, 0, stream>>>(a, a.page_table != nullptr ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace kvattn
