// Split-KV decode over an FP8 (e4m3) cache for at most 8 query rows per KV head
// (grouped heads x new tokens, e.g. Llama decode: 4 or 8 heads, one token).
//
// With so few rows the usual orientation (query rows on the 16-row side of the
// m16n8k16 MMA) leaves most of every MMA empty.  This kernel transposes both
// products so that the 16-row side carries keys or output columns:
//   S^T = K Q^T   (A = 16 keys x 16 d from the cache, B = 16 d x 8 query rows)
//   O^T += V^T P^T (A = 16 output columns x 16 keys, B = 16 keys x 8 query rows)
// which halves the MMAs, exponentials and accumulators of the warp-level FP8
// kernel in decode.cu.  P^T's B fragments come from the S^T accumulators with
// one 8x8 register transpose (movmatrix) per 8 keys.  The cache bytes are read
// with 16-byte shared loads and converted exactly to f16 (cvt e4m3x2 -> f16x2);
// d is taken in the permuted order of the other FP8 kernel for Q K^T, and the
// output column of O^T row m of block j is d = 16 (m mod 8) + 2 j + (m >= 8), so
// a thread's 16 V bytes of a key cover its rows of every block.  The K scale is
// folded into the softmax scale and the V scale into the chunk's normalisation.
// Producer, work items, online softmax with the lazy rescale, the in-CTA merge
// of the four consumer warps and the partial layout are those of the other
// split kernels; the combine kernel merges the chunks.
//
// Method: "[BEE-30062] FlashAttention 與高效注意力核心", "背景" and
// "為長上下文推論啟用 FlashDecoding" (split along the KV length, stable merge);
// "大模型面試笔记——Attention篇" section 2 (online safe softmax); "KV cache, flash
// attention and inference optimisation" lesson, "用它" (an FP8 KV cache).
#include <cuda_bf16.h>
#include <math.h>

#include "internal.h"
#include "ptx.cuh"
#include "split.cuh"

namespace kvattn {
namespace {

constexpr float kLn2 = 0.6931471805599453f;

struct Fp8StCfg {
  static constexpr int kConsumerWarps = 4;
  static constexpr int kThreads = 32 * (kConsumerWarps + 1);
  static constexpr int kRows = 8;                       // query rows per KV head (MMA N)
  static constexpr int kHalves = 1;                     // one 128-byte span per token row (d = 128 bytes)
  static constexpr int kHalfBytes = kDecodeTile * 128;
  static constexpr int kTensorBytes = kHalfBytes;
  static constexpr int kStageBytes = 2 * kTensorBytes;  // 16 KB: 64 tokens of K and of V
  static constexpr int kStages = 4;
  static constexpr int kRedStride = 128 + 4;            // floats per row of the merge buffer
  static constexpr int kRedBytes = kConsumerWarps * kRows * kRedStride * 4;
  static_assert(kRedBytes <= kStages * kStageBytes, "merge buffer must fit in the ring");
  static constexpr int kBarOffset = kStages * kStageBytes;
  static constexpr int kStatsOffset = kBarOffset + 2 * kStages * 8;
  static constexpr int kSmemBytes = kStatsOffset + kConsumerWarps * kRows * 2 * 4 + 16 + 1024;
};

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v) {
  return pack_f16x2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
}

template <bool PAGED>
__global__ void __launch_bounds__(Fp8StCfg::kThreads, 3)
    decode_fp8_st_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                         const SplitParams p) {
  using C = Fp8StCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
  uint64_t* empty = full + C::kStages;
  float* stats = reinterpret_cast<float*>(smem + C::kStatsOffset);   // [4 warps][8 rows][2]: m, l
  int* abort_flag = reinterpret_cast<int*>(stats + C::kConsumerWarps * C::kRows * 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;

  const int L = p.seqlens[b];
  if (seqlen_bad(L, p.T, p.max_seqlen, PAGED, p.capacity, p.max_blocks)) {
    if (threadIdx.x == 0 && c == 0 && g == 0) atomicOr(p.status, DEV_SEQLEN);
    return;   // the combine kernel writes NaN rows for this sequence
  }
  const int tok_begin = c * p.chunk;
  if (tok_begin >= L) return;
  const int tok_end = min(tok_begin + p.chunk, L);
  const int n_tiles = (tok_end - tok_begin + kDecodeTile - 1) / kDecodeTile;
  const size_t item = ((size_t)b * p.Hkv + g) * p.max_chunks + c;
  const float ks = __ldg(p.k_scale + g), vs = __ldg(p.v_scale + g);
  if (!(ks > 0.f && ks <= 3.402823466e38f && vs > 0.f && vs <= 3.402823466e38f)) {
    if (threadIdx.x == 0 && c == 0) atomicOr(p.status, DEV_SCALE);
    for (int r = threadIdx.x; r < p.R; r += blockDim.x) p.part_lse[item * p.R + r] = NAN;
    return;   // the whole CTA leaves before any barrier: the scales are uniform across it
  }
  const float scale_log2 = p.scale_log2 * ks;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], C::kConsumerWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == C::kConsumerWarps) {
    if (lane == 0) produce_split_tiles<C, PAGED>(smem, full, empty, &tmK, &tmV, p, b, g, tok_begin, tok_end, n_tiles,
                                                abort_flag);
    return;
  }

  // -------------------------------------------------------------- consumers
  const int wsub = warp;                       // which 16 tokens of each tile
  const int gid = lane >> 2, tig = lane & 3;

  // Q^T (B operand, n = query row gid): k16 step kk takes d = 16 (tig + 4 (kk / 4)) + 4 (kk % 4) + {0, 1 | 2, 3}
  uint32_t qb[8][2];
  {
    const bool live = gid < p.R;
    const int t = gid / p.G, hh = gid - t * p.G;
    const __nv_bfloat16* qr = p.q + (((size_t)b * p.T + t) * p.Hq + (size_t)g * p.G + hh) * 128;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int d0 = 16 * (tig + 4 * (kk >> 2)) + 4 * (kk & 3);
      const uint2 x = live ? *reinterpret_cast<const uint2*>(qr + d0) : make_uint2(0u, 0u);
      qb[kk][0] = bf16x2_to_f16x2(x.x);
      qb[kk][1] = bf16x2_to_f16x2(x.y);
    }
  }
  // this thread's S^T columns are query rows 2 tig and 2 tig + 1: their first invisible keys
  const int r0 = 2 * tig, r1 = r0 + 1;
  const int end0 = r0 < p.R ? (p.causal ? L - p.T + r0 / p.G + 1 : L) : 0;
  const int end1 = r1 < p.R ? (p.causal ? L - p.T + r1 / p.G + 1 : L) : 0;

  float o[8][4];
#pragma unroll
  for (int j = 0; j < 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  for (int i = 0; i < n_tiles; ++i) {
    const int s = i % C::kStages;
    if (!mbar_wait(&full[s], (i / C::kStages) & 1)) {
      atomicOr(p.status, DEV_TIMEOUT);
      *reinterpret_cast<volatile int*>(abort_flag) = 1;   // every consumer sees it after the barrier below
      break;
    }
    if (*reinterpret_cast<volatile int*>(abort_flag)) break;
    const uint32_t kbase = smem_u32(smem + s * C::kStageBytes);
    const uint32_t vbase = kbase + C::kTensorBytes;
    const int tok_base = tok_begin + i * kDecodeTile + wsub * 16;

    // ---- S^T = K Q^T: A rows are keys gid and gid + 8 of this warp's 16 (token row & 7 == gid)
    uint32_t kw[2][8];
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const uint32_t ra = kbase + (wsub * 16 + rr * 8 + gid) * 128;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const uint4 x = lds128(ra + (((tig + 4 * hh) ^ gid) << 4));
        kw[rr][4 * hh + 0] = x.x;
        kw[rr][4 * hh + 1] = x.y;
        kw[rr][4 * hh + 2] = x.z;
        kw[rr][4 * hh + 3] = x.w;
      }
    }
    float sacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      uint32_t a[4];
      e4m3x4_to_f16x2x2(kw[0][kk], a[0], a[2]);
      e4m3x4_to_f16x2x2(kw[1][kk], a[1], a[3]);
      mma_f16_16816(sacc, a, qb[kk][0], qb[kk][1]);
    }

    // ---- V bytes d = 16 gid .. 16 gid + 15 of keys 2tig, 2tig+1, 2tig+8, 2tig+9, loaded before the
    //      softmax; keys at or past L may hold any bytes, so their rows are zeroed
    uint32_t vw[4][4];
    {
      const bool tail = tok_base + 16 > L;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int key = 2 * tig + (q & 1) + 8 * (q >> 1);
        const int vrow = wsub * 16 + key;
        uint4 x = lds128(vbase + vrow * 128 + ((gid ^ (vrow & 7)) << 4));
        if (tail && tok_base + key >= L) x = make_uint4(0u, 0u, 0u, 0u);
        vw[q][0] = x.x;
        vw[q][1] = x.y;
        vw[q][2] = x.z;
        vw[q][3] = x.w;
      }
    }

    // ---- online softmax over this warp's keys for query rows r0, r1 (base 2, lazy rescale)
    const int ka = tok_base + gid, kb = ka + 8;
    const float v00 = (ka < end0) ? sacc[0] * scale_log2 : -INFINITY;   // key gid,     row r0
    const float v01 = (ka < end1) ? sacc[1] * scale_log2 : -INFINITY;   // key gid,     row r1
    const float v10 = (kb < end0) ? sacc[2] * scale_log2 : -INFINITY;   // key gid + 8, row r0
    const float v11 = (kb < end1) ? sacc[3] * scale_log2 : -INFINITY;   // key gid + 8, row r1
    float mx0 = fmaxf(v00, v10), mx1 = fmaxf(v01, v11);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    if (__any_sync(0xffffffffu, mx0 > m0 + 8.f || mx1 > m1 + 8.f)) {
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
      const float al0 = ex2(m0 - ((mn0 == -INFINITY) ? 0.f : mn0));   // 0 while m is -inf
      const float al1 = ex2(m1 - ((mn1 == -INFINITY) ? 0.f : mn1));
      m0 = mn0;
      m1 = mn1;
      l0 *= al0;
      l1 *= al1;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        o[j][0] *= al0;
        o[j][2] *= al0;
        o[j][1] *= al1;
        o[j][3] *= al1;
      }
    }
    const float mu0 = (m0 == -INFINITY) ? 0.f : m0;
    const float mu1 = (m1 == -INFINITY) ? 0.f : m1;
    const float p00 = ex2(v00 - mu0), p10 = ex2(v10 - mu0);
    const float p01 = ex2(v01 - mu1), p11 = ex2(v11 - mu1);
    l0 += p00 + p10;
    l1 += p01 + p11;
    // P^T as the B operand: transpose the 8x8 (key, row) fragments of keys 0-7 and 8-15
    const uint32_t pb0 = movmatrix_trans(pack_f16x2(p00, p01));
    const uint32_t pb1 = movmatrix_trans(pack_f16x2(p10, p11));

    // ---- O^T += V^T P^T, 8 blocks of 16 output columns; block j row m is d = 16 (m mod 8) + 2 j + (m >= 8):
    //      bytes 2j and 2j+1 of this thread's V chunk, paired across keys by a byte permute
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int w = j >> 1;
      const uint32_t sel = (j & 1) ? 0x7362u : 0x5140u;
      uint32_t a[4];
      e4m3x4_to_f16x2x2(prmt(vw[0][w], vw[1][w], sel), a[0], a[1]);
      e4m3x4_to_f16x2x2(prmt(vw[2][w], vw[3][w], sel), a[2], a[3]);
      mma_f16_16816(o[j], a, pb0, pb1);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }

  // -------------------------------------------------- merge the four warps
  launch_dependents();   // the combine kernel may start launching (it waits for this grid)
  asm volatile("bar.sync 1, %0;" ::"n"(C::kConsumerWarps * 32) : "memory");
  // one decision for all consumers: a warp that gave up set the shared flag before the
  // barrier, so none of them can wait at a later named barrier for one that left
  if (*reinterpret_cast<volatile int*>(abort_flag)) {
    for (int r = threadIdx.x; r < p.R; r += C::kConsumerWarps * 32) p.part_lse[item * p.R + r] = NAN;
    return;
  }
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
  }
  float* st = stats + wsub * C::kRows * 2;
  if (gid == 0) {
    st[r0 * 2 + 0] = m0;
    st[r0 * 2 + 1] = l0;
    st[r1 * 2 + 0] = m1;
    st[r1 * 2 + 1] = l1;
  }
  asm volatile("bar.sync 1, %0;" ::"n"(C::kConsumerWarps * 32) : "memory");
  float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
  for (int w = 0; w < C::kConsumerWarps; ++w) {
    M0 = fmaxf(M0, stats[(w * C::kRows + r0) * 2]);
    M1 = fmaxf(M1, stats[(w * C::kRows + r1) * 2]);
  }
  const float f0 = (m0 == -INFINITY) ? 0.f : ex2(m0 - M0);
  const float f1 = (m1 == -INFINITY) ? 0.f : ex2(m1 - M1);
  float* red = reinterpret_cast<float*>(smem) + wsub * C::kRows * C::kRedStride;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int col = 16 * gid + 2 * j;
    *reinterpret_cast<float2*>(red + r0 * C::kRedStride + col) = make_float2(o[j][0] * f0, o[j][2] * f0);
    *reinterpret_cast<float2*>(red + r1 * C::kRedStride + col) = make_float2(o[j][1] * f1, o[j][3] * f1);
  }
  asm volatile("bar.sync 1, %0;" ::"n"(C::kConsumerWarps * 32) : "memory");

  float* out = p.part_o + item * (size_t)p.R * 128;
  for (int idx = threadIdx.x; idx < p.R * 32; idx += C::kConsumerWarps * 32) {
    const int r = idx >> 5, col = (idx & 31) * 4;
    float mrow = -INFINITY;
#pragma unroll
    for (int w = 0; w < C::kConsumerWarps; ++w) mrow = fmaxf(mrow, stats[(w * C::kRows + r) * 2]);
    float lsum = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < C::kConsumerWarps; ++w) {
      const float mw = stats[(w * C::kRows + r) * 2];
      const float fw = (mw == -INFINITY) ? 0.f : ex2(mw - mrow);
      lsum += stats[(w * C::kRows + r) * 2 + 1] * fw;
      const float4 x =
          *reinterpret_cast<const float4*>(reinterpret_cast<float*>(smem) + (w * C::kRows + r) * C::kRedStride + col);
      acc.x += x.x;
      acc.y += x.y;
      acc.z += x.z;
      acc.w += x.w;
    }
    const float inv = lsum > 0.f ? vs / lsum : 0.f;
    *reinterpret_cast<float4*>(out + (size_t)r * 128 + col) =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    if (col == 0) p.part_lse[item * p.R + r] = lsum > 0.f ? (mrow + log2f(lsum)) * kLn2 : -INFINITY;
  }
}

template <bool PAGED>
cudaError_t run(const CUtensorMap& tk, const CUtensorMap& tv, const SplitParams& sp, int B, cudaStream_t stream) {
  auto kern = decode_fp8_st_kernel<PAGED>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Fp8StCfg::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(sp.max_chunks, sp.Hkv, B);
  kern<<<grid, Fp8StCfg::kThreads, Fp8StCfg::kSmemBytes, stream>>>(tk, tv, sp);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_fp8_rows8(const CUtensorMap& tk, const CUtensorMap& tv, const SplitParams& sp, int B,
                                    bool paged, cudaStream_t stream) {
  return paged ? run<true>(tk, tv, sp, B, stream) : run<false>(tk, tv, sp, B, stream);
}

}  // namespace kvattn
