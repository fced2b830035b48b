// Device copy of whole KV blocks (K and V pools together): the copy-on-write
// step of the host block pool, when a sequence that shares a partly filled last
// block with a fork is about to write into it.
//
// Method: "KV cache, flash attention and inference optimisation" lesson,
// section "页面注意 KV缓存作为虚拟内存" (blocks shared between parallel samples).
// One thread moves one 16-byte vector of K and the matching vector of V.
#include "../../include/attn.h"
#include "internal.h"
#include "ptx.cuh"

namespace kvattn {
namespace {

__global__ void __launch_bounds__(256) copy_blocks_kernel(uint4* k, uint4* v, const int32_t* src, const int32_t* dst,
                                                          int num_blocks, int vecs_per_block, unsigned* status) {
  const int pair = blockIdx.y;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= vecs_per_block) return;
  const int s = __ldg(src + pair), d = __ldg(dst + pair);
  if (s < 0 || s >= num_blocks || d < 0 || d >= num_blocks) {
    if (i == 0) atomicOr(status, DEV_PAGE_ID);
    return;
  }
  if (s == d) return;
  const size_t so = (size_t)s * vecs_per_block + i, dof = (size_t)d * vecs_per_block + i;
  k[dof] = k[so];
  v[dof] = v[so];
}

}  // namespace

cudaError_t launch_copy_blocks(void* k, void* v, const int32_t* src, const int32_t* dst, int n, int num_blocks,
                               int block_bytes, unsigned* status, cudaStream_t stream) {
  const int vecs = block_bytes / 16;
  dim3 grid((vecs + 255) / 256, n);
  copy_blocks_kernel<<<grid, 256, 0, stream>>>(static_cast<uint4*>(k), static_cast<uint4*>(v), src, dst, num_blocks,
                                               vecs, status);
  return cudaGetLastError();
}

}  // namespace kvattn
