// Split-KV decode attention for sm_100a (memory-bound path).
//
// One CTA owns one work item (sequence b, KV head g, key chunk c).  All
// R = (Hq/Hkv) * T query rows that read KV head g are handled together, so each
// K/V byte is streamed from HBM once per step.  A producer warp moves 64-token
// K/V tiles into a shared-memory ring with TMA (128-byte swizzle, evict-first
// L2 policy); consumer warps compute S = Q K^T and O += P V with warp-level bf16
// tensor-core MMAs (fp32 accumulation), keeping a running maximum and running
// denominator per row and rescaling O when the maximum grows.  Each consumer
// warp owns 16 tokens of every tile, so the four warps of a row group are four
// independent online softmaxes that are merged at the end of the chunk.  The
// chunk's normalised output and log-sum-exp go to the workspace; a second
// kernel merges the chunks of each row with the log-sum-exp combine.
//
// FP8 caches (e4m3 codes with one float32 scale per KV head for K and for V):
// the tile is half as many bytes; each consumer thread reads its K and V bytes
// with 16-byte shared loads and converts them exactly to f16 with the hardware
// e4m3x2 -> f16x2 conversion, so the MMAs run in f16 (Q and P are rounded to
// f16).  The sum over d in Q K^T may take the d positions in any order as long
// as Q uses the same order, so a thread's four consecutive K bytes of a row
// feed one k16 step directly; for P V the output columns are permuted the same
// way (column n of the j-th 8-column block is d = 16 n + j) so that a thread's
// V bytes of two keys pair up with one byte permute.  The K scale is folded
// into the softmax scale and the V scale into the chunk's normalisation.
//
// Method: "[BEE-30062] FlashAttention 與高效注意力核心", sections "背景" and
// "為長上下文推論啟用 FlashDecoding" (split along the KV length, numerically
// stable reduction of partial softmax results); "大模型面試笔记——Attention篇"
// section 2 (online safe softmax); "Effizienz", "Der wichtige Maskenfehler beim
// Cache" (bottom-right aligned mask for several new tokens); "KV cache, flash
// attention and inference optimisation" lesson, section "用它" (an FP8 KV cache).
#include <cuda_bf16.h>
#include <math.h>

#include "internal.h"
#include "ptx.cuh"
#include "split.cuh"

namespace kvattn {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <int D, int MT, bool FP8>
struct DecodeCfg {
  static_assert(!FP8 || D == 128, "FP8 caches are built for d = 128");
  static_assert(MT == 1 || FP8, "bf16 caches with more than 16 rows run on the tensor-core kernel");
  static constexpr int kConsumerWarps = 4 * MT;
  static constexpr int kThreads = 32 * (kConsumerWarps + 1);
  static constexpr int kHalves = (FP8 ? D : 2 * D) / 128;   // 128-byte swizzle spans per token row
  static constexpr int kHalfBytes = kDecodeTile * 128;
  static constexpr int kTensorBytes = kHalves * kHalfBytes;   // one of K or V per stage
  static constexpr int kStageBytes = 2 * kTensorBytes;
  static constexpr int kBf16Stages = (MT == 1) ? (D == 128 ? 3 : 6) : (D == 128 ? 4 : 8);
  static constexpr int kStages = FP8 ? 2 * kBf16Stages : kBf16Stages;   // the same bytes in flight
  static constexpr int kRedStride = D + 8;            // floats per row of the merge buffer
  static constexpr int kRedBytes = MT * 4 * 16 * kRedStride * 4;
  static_assert(kRedBytes <= kStages * kStageBytes, "merge buffer must fit in the ring");
  static constexpr int kBarOffset = kStages * kStageBytes;
  static constexpr int kStatsOffset = kBarOffset + 2 * kStages * 8;
  static constexpr int kSmemBytes = kStatsOffset + MT * 4 * 16 * 2 * 4 + 16 + 1024;  // + alignment slack
  static constexpr int kMinBlocks = (kSmemBytes * 2 <= 227 * 1024) ? 2 : 1;
};

// bf16 pair (low = lower index) -> f16 pair
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v) {
  return pack_f16x2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
}

template <int D, int MT, bool PAGED, bool FP8>
__global__ void __launch_bounds__(DecodeCfg<D, MT, FP8>::kThreads, DecodeCfg<D, MT, FP8>::kMinBlocks)
    decode_split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const SplitParams p) {
  using C = DecodeCfg<D, MT, FP8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
  uint64_t* empty = full + C::kStages;
  float* stats = reinterpret_cast<float*>(smem + C::kStatsOffset);   // [MT][4][16][2]: m, l
  int* abort_flag = reinterpret_cast<int*>(stats + MT * 4 * 16 * 2);

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
  float scale_log2 = p.scale_log2, v_scale = 1.f;
  if constexpr (FP8) {
    const float ks = __ldg(p.k_scale + g), vs = __ldg(p.v_scale + g);
    if (!(ks > 0.f && ks <= 3.402823466e38f && vs > 0.f && vs <= 3.402823466e38f)) {
      if (threadIdx.x == 0 && c == 0) atomicOr(p.status, DEV_SCALE);
      const size_t item = ((size_t)b * p.Hkv + g) * p.max_chunks + c;
      for (int r = threadIdx.x; r < p.R; r += blockDim.x) p.part_lse[item * p.R + r] = NAN;
      return;   // the whole CTA leaves before any barrier: the scales are uniform across it
    }
    scale_log2 *= ks;
    v_scale = vs;
  }

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
    // ------------------------------------------------------------ producer
    if (lane == 0) produce_split_tiles<C, PAGED>(smem, full, empty, &tmK, &tmV, p, b, g, tok_begin, tok_end, n_tiles,
                                                abort_flag);
    return;
  }

  // -------------------------------------------------------------- consumers
  const int wsub = warp & 3;          // which 16 tokens of each tile
  const int mt = warp >> 2;           // which 16 query rows
  const int gid = lane >> 2, tig = lane & 3;

  // Query rows r0 = mt*16 + gid and r1 = r0 + 8; row r is (token t = r / G, head g*G + r % G).
  const int r0 = mt * 16 + gid, r1 = r0 + 8;
  int end0 = L, end1 = L;   // first invisible key of each row
  if (p.causal) {
    if (r0 < p.R) end0 = L - p.T + r0 / p.G + 1;
    if (r1 < p.R) end1 = L - p.T + r1 / p.G + 1;
  }

  // Q fragments (A operand, 16 x D, row-major) straight from global memory.
  uint32_t qa[D / 16][4];
  {
    auto qrow = [&](int r) -> const __nv_bfloat16* {
      const int t = r / p.G, hh = r - t * p.G;
      return p.q + (((size_t)b * p.T + t) * p.Hq + (size_t)g * p.G + hh) * D;
    };
    const __nv_bfloat16* qr0 = r0 < p.R ? qrow(r0) : nullptr;
    const __nv_bfloat16* qr1 = r1 < p.R ? qrow(r1) : nullptr;
    if constexpr (!FP8) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int c0 = kk * 16 + tig * 2;
        qa[kk][0] = qr0 ? *reinterpret_cast<const uint32_t*>(qr0 + c0) : 0u;
        qa[kk][1] = qr1 ? *reinterpret_cast<const uint32_t*>(qr1 + c0) : 0u;
        qa[kk][2] = qr0 ? *reinterpret_cast<const uint32_t*>(qr0 + c0 + 8) : 0u;
        qa[kk][3] = qr1 ? *reinterpret_cast<const uint32_t*>(qr1 + c0 + 8) : 0u;
      }
    } else {
      // k16 step kk takes d = 16 (tig + 4 (kk / 4)) + 4 (kk % 4) + {0, 1 | 2, 3}: the
      // four consecutive K bytes this thread reads for that step
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int d0 = 16 * (tig + 4 * (kk >> 2)) + 4 * (kk & 3);
        const uint2 x0 = qr0 ? *reinterpret_cast<const uint2*>(qr0 + d0) : make_uint2(0u, 0u);
        const uint2 x1 = qr1 ? *reinterpret_cast<const uint2*>(qr1 + d0) : make_uint2(0u, 0u);
        qa[kk][0] = bf16x2_to_f16x2(x0.x);
        qa[kk][1] = bf16x2_to_f16x2(x1.x);
        qa[kk][2] = bf16x2_to_f16x2(x0.y);
        qa[kk][3] = bf16x2_to_f16x2(x1.y);
      }
    }
  }

  float o_acc[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) o_acc[n][0] = o_acc[n][1] = o_acc[n][2] = o_acc[n][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  // ldmatrix lane roles
  const int lm = lane >> 3, lr = lane & 7;

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

    // ---- S = Q K^T for this warp's 16 tokens (two n8 tiles)
    float sacc[2][4];
#pragma unroll
    for (int n = 0; n < 2; ++n) sacc[n][0] = sacc[n][1] = sacc[n][2] = sacc[n][3] = 0.f;
    if constexpr (!FP8) {
      const int trow = wsub * 16 + (lm >> 1) * 8 + lr;   // token row inside the tile
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int chunk16 = kk * 2 + (lm & 1);             // 16-byte chunk along d
        const int h = chunk16 >> 3, cw = chunk16 & 7;
        const uint32_t addr = kbase + h * C::kHalfBytes + trow * 128 + ((cw ^ (trow & 7)) << 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(addr, b0, b1, b2, b3);
        mma_bf16_16816(sacc[0], qa[kk], b0, b1);
        mma_bf16_16816(sacc[1], qa[kk], b2, b3);
      }
    } else {
      // token rows gid (n8 block 0) and 8 + gid (block 1); 16-byte chunks tig and tig + 4
      uint32_t kw[2][8];
#pragma unroll
      for (int nb = 0; nb < 2; ++nb) {
        const int trow = wsub * 16 + nb * 8 + gid;       // trow & 7 == gid
        const uint32_t ra = kbase + trow * 128;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const uint4 x = lds128(ra + (((tig + 4 * hh) ^ gid) << 4));
          kw[nb][4 * hh + 0] = x.x;
          kw[nb][4 * hh + 1] = x.y;
          kw[nb][4 * hh + 2] = x.z;
          kw[nb][4 * hh + 3] = x.w;
        }
      }
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
        for (int nb = 0; nb < 2; ++nb) {
          uint32_t b0, b1;
          e4m3x4_to_f16x2x2(kw[nb][kk], b0, b1);
          mma_f16_16816(sacc[nb], qa[kk], b0, b1);
        }
      }
    }

    // ---- V fragments for this warp's 16 tokens, loaded before the softmax so the
    //      shared-memory latency overlaps it; keys at or past L may hold anything
    //      (even NaN), so their V rows are zeroed
    uint32_t vb[FP8 ? 1 : D / 16][4];
    uint32_t vw[FP8 ? 4 : 1][4];   // FP8: 16 bytes (d = 16 gid .. 16 gid + 15) of keys 2tig, 2tig+1, 2tig+8, 2tig+9
    if constexpr (FP8) {
      const bool tail = tok_base + 16 > L;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int key = 2 * tig + (i & 1) + 8 * (i >> 1);
        const int vrow = wsub * 16 + key;
        uint4 x = lds128(vbase + vrow * 128 + ((gid ^ (vrow & 7)) << 4));
        if (tail && tok_base + key >= L) x = make_uint4(0u, 0u, 0u, 0u);
        vw[i][0] = x.x;
        vw[i][1] = x.y;
        vw[i][2] = x.z;
        vw[i][3] = x.w;
      }
    } else {
      const bool tail = tok_base + 16 > L;
      const int vrow = wsub * 16 + (lm & 1) * 8 + lr;
      const int ta = tok_base + tig * 2, tb = ta + 8;
      const uint32_t keep_a = ((ta < L) ? 0x0000ffffu : 0u) | ((ta + 1 < L) ? 0xffff0000u : 0u);
      const uint32_t keep_b = ((tb < L) ? 0x0000ffffu : 0u) | ((tb + 1 < L) ? 0xffff0000u : 0u);
#pragma unroll
      for (int nn = 0; nn < D / 16; ++nn) {
        const int chunk16 = nn * 2 + (lm >> 1);
        const int h = chunk16 >> 3, cw = chunk16 & 7;
        const uint32_t addr = vbase + h * C::kHalfBytes + vrow * 128 + ((cw ^ (vrow & 7)) << 4);
        ldsm_x4_t(addr, vb[nn][0], vb[nn][1], vb[nn][2], vb[nn][3]);
        if (tail) {
          vb[nn][0] &= keep_a;
          vb[nn][2] &= keep_a;
          vb[nn][1] &= keep_b;
          vb[nn][3] &= keep_b;
        }
      }
    }

    // ---- online softmax (base-2 exponent, scale folded in).  A row's reference
    //      maximum is raised only when the tile maximum exceeds it by more than 8,
    //      so O is rescaled rarely; p = 2^(s - m) then stays <= 256, and the merge
    //      at the end uses the same reference, so the result is exact.
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int n = 0; n < 2; ++n) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tok = tok_base + n * 8 + tig * 2 + (e & 1);
        const int end = (e < 2) ? end0 : end1;
        const float v = (tok < end) ? sacc[n][e] * scale_log2 : -INFINITY;
        sacc[n][e] = v;
        if (e < 2) mx0 = fmaxf(mx0, v); else mx1 = fmaxf(mx1, v);
      }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    if (__any_sync(0xffffffffu, mx0 > m0 + 8.f || mx1 > m1 + 8.f)) {
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
      const float al0 = ex2(m0 - ((mn0 == -INFINITY) ? 0.f : mn0));   // 0 while m is -inf
      const float al1 = ex2(m1 - ((mn1 == -INFINITY) ? 0.f : mn1));
      m0 = mn0;
      m1 = mn1;
      l0 *= al0;
      l1 *= al1;
#pragma unroll
      for (int n = 0; n < D / 8; ++n) {
        o_acc[n][0] *= al0;
        o_acc[n][1] *= al0;
        o_acc[n][2] *= al1;
        o_acc[n][3] *= al1;
      }
    }
    const float mu0 = (m0 == -INFINITY) ? 0.f : m0;
    const float mu1 = (m1 == -INFINITY) ? 0.f : m1;
    float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
    for (int n = 0; n < 2; ++n) {
      sacc[n][0] = ex2(sacc[n][0] - mu0);
      sacc[n][1] = ex2(sacc[n][1] - mu0);
      sacc[n][2] = ex2(sacc[n][2] - mu1);
      sacc[n][3] = ex2(sacc[n][3] - mu1);
      ps0 += sacc[n][0] + sacc[n][1];
      ps1 += sacc[n][2] + sacc[n][3];
    }
    l0 += ps0;
    l1 += ps1;
    uint32_t pa[4];
    if constexpr (!FP8) {
      pa[0] = pack_bf16x2(sacc[0][0], sacc[0][1]);
      pa[1] = pack_bf16x2(sacc[0][2], sacc[0][3]);
      pa[2] = pack_bf16x2(sacc[1][0], sacc[1][1]);
      pa[3] = pack_bf16x2(sacc[1][2], sacc[1][3]);

      // ---- O += P V
#pragma unroll
      for (int nn = 0; nn < D / 16; ++nn) {
        mma_bf16_16816(o_acc[2 * nn], pa, vb[nn][0], vb[nn][1]);
        mma_bf16_16816(o_acc[2 * nn + 1], pa, vb[nn][2], vb[nn][3]);
      }
    } else {
      pa[0] = pack_f16x2(sacc[0][0], sacc[0][1]);
      pa[1] = pack_f16x2(sacc[0][2], sacc[0][3]);
      pa[2] = pack_f16x2(sacc[1][0], sacc[1][1]);
      pa[3] = pack_f16x2(sacc[1][2], sacc[1][3]);
      // ---- O += P V over 16 blocks of 8 output columns; block j, column n is d = 16 n + j,
      //      i.e. byte j of this thread's 16 V bytes; a byte permute pairs keys (2tig, 2tig+1)
      //      and (2tig+8, 2tig+9) for blocks j and j + 1
#pragma unroll
      for (int jj = 0; jj < D / 16; ++jj) {
        const int w = jj >> 1;
        const uint32_t sel = (jj & 1) ? 0x7362u : 0x5140u;
        uint32_t b01_j, b01_j1, b23_j, b23_j1;
        e4m3x4_to_f16x2x2(prmt(vw[0][w], vw[1][w], sel), b01_j, b01_j1);
        e4m3x4_to_f16x2x2(prmt(vw[2][w], vw[3][w], sel), b23_j, b23_j1);
        mma_f16_16816(o_acc[2 * jj], pa, b01_j, b23_j);
        mma_f16_16816(o_acc[2 * jj + 1], pa, b01_j1, b23_j1);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }

  // -------------------------------------------------- merge the four warps
  launch_dependents();   // the combine kernel may start launching (it waits for this grid)
  // every consumer reached here; the ring is idle (all issued tiles consumed)
  asm volatile("bar.sync 1, %0;" ::"n"(C::kConsumerWarps * 32) : "memory");
  // one decision for all consumers: a warp that gave up set the shared flag before the
  // barrier, so none of them can wait at a later named barrier for one that left
  if (*reinterpret_cast<volatile int*>(abort_flag)) {
    // a wait gave up: leave the partial as NaN so the result is visibly invalid
    const size_t item = ((size_t)b * p.Hkv + g) * p.max_chunks + c;
    for (int r = threadIdx.x; r < p.R; r += C::kConsumerWarps * 32) p.part_lse[item * p.R + r] = NAN;
    return;
  }
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  float* st = stats + ((mt * 4 + wsub) * 16) * 2;
  if (tig == 0) {
    st[gid * 2 + 0] = m0;
    st[gid * 2 + 1] = l0;
    st[(gid + 8) * 2 + 0] = m1;
    st[(gid + 8) * 2 + 1] = l1;
  }
  asm volatile("bar.sync 1, %0;" ::"n"(C::kConsumerWarps * 32) : "memory");
  float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const float* sw = stats + ((mt * 4 + w) * 16) * 2;
    M0 = fmaxf(M0, sw[gid * 2]);
    M1 = fmaxf(M1, sw[(gid + 8) * 2]);
  }
  const float f0 = (m0 == -INFINITY) ? 0.f : ex2(m0 - M0);
  const float f1 = (m1 == -INFINITY) ? 0.f : ex2(m1 - M1);
  float* red = reinterpret_cast<float*>(smem) + ((mt * 4 + wsub) * 16) * C::kRedStride;
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    if constexpr (!FP8) {
      const int col = n * 8 + tig * 2;
      *reinterpret_cast<float2*>(red + gid * C::kRedStride + col) = make_float2(o_acc[n][0] * f0, o_acc[n][1] * f0);
      *reinterpret_cast<float2*>(red + (gid + 8) * C::kRedStride + col) =
          make_float2(o_acc[n][2] * f1, o_acc[n][3] * f1);
    } else {
      const int col = 32 * tig + n;   // columns 2tig and 2tig + 1 of block n are d = 32 tig + n and + 16
      red[gid * C::kRedStride + col] = o_acc[n][0] * f0;
      red[gid * C::kRedStride + col + 16] = o_acc[n][1] * f0;
      red[(gid + 8) * C::kRedStride + col] = o_acc[n][2] * f1;
      red[(gid + 8) * C::kRedStride + col + 16] = o_acc[n][3] * f1;
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(C::kConsumerWarps * 32) : "memory");

  const size_t item = ((size_t)b * p.Hkv + g) * p.max_chunks + c;
  float* out = p.part_o + item * (size_t)p.R * D;
  constexpr int kVec = D / 4;   // float4 per row
  for (int idx = threadIdx.x; idx < p.R * kVec; idx += C::kConsumerWarps * 32) {
    const int r = idx / kVec, col = (idx - r * kVec) * 4;
    const int rm = r >> 4, rr = r & 15;
    float mrow = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) mrow = fmaxf(mrow, stats[((rm * 4 + w) * 16 + rr) * 2]);
    float lsum = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float mw = stats[((rm * 4 + w) * 16 + rr) * 2];
      const float fw = (mw == -INFINITY) ? 0.f : ex2(mw - mrow);
      lsum += stats[((rm * 4 + w) * 16 + rr) * 2 + 1] * fw;
      const float4 x = *reinterpret_cast<const float4*>(reinterpret_cast<float*>(smem) +
                                                        ((rm * 4 + w) * 16 + rr) * C::kRedStride + col);
      acc.x += x.x;
      acc.y += x.y;
      acc.z += x.z;
      acc.w += x.w;
    }
    const float inv = lsum > 0.f ? (FP8 ? v_scale / lsum : 1.f / lsum) : 0.f;
    *reinterpret_cast<float4*>(out + (size_t)r * D + col) =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    if (col == 0) p.part_lse[item * p.R + r] = lsum > 0.f ? (mrow + log2f(lsum)) * kLn2 : -INFINITY;
  }
}

// kPer consecutive partial-output floats of one lane (2 or 4), as a float4.
template <int kPer>
__device__ __forceinline__ float4 load_part(const float* src) {
  if constexpr (kPer == 4) {
    return __ldg(reinterpret_cast<const float4*>(src));
  } else {
    const float2 v = __ldg(reinterpret_cast<const float2*>(src));
    return make_float4(v.x, v.y, 0.f, 0.f);
  }
}

template <int kPer>
__device__ __forceinline__ void accumulate(float (&acc)[kPer], float w, float4 x) {
  acc[0] = fmaf(w, x.x, acc[0]);
  acc[1] = fmaf(w, x.y, acc[1]);
  if constexpr (kPer == 4) {
    acc[2] = fmaf(w, x.z, acc[2]);
    acc[3] = fmaf(w, x.w, acc[3]);
  }
}

// Merge the chunk partials of each output row (b, t, h).  wpr warps (1, 2, 4 or 8)
// share a row: warp w of the row takes chunks w, w + wpr, ...; their weighted sums
// meet in shared memory.  The sequence length is read before the wait on the split
// kernel (that kernel does not write it); after the wait every warp issues its first
// kBatch partial loads together with the row's LSE loads, so a row costs about two
// dependent memory round trips.  kBatch: partial loads in flight per lane -- 8 for
// long decode (many chunks per row), 2 for launches of at most two chunks (many rows,
// as in a prompt chunk), where a small register footprint buys five CTAs per SM.
template <int D, int kBatch>
__global__ void __launch_bounds__(256, kBatch >= 8 ? 2 : 5) decode_combine_kernel(const float* __restrict__ part_o,
                                                             const float* __restrict__ part_lse,
                                                             const int32_t* __restrict__ seqlens, void* o, int o_bf16,
                                                             float* lse, SplitParams p, int B, int paged, int wpr) {
  constexpr int kPer = D / 32;    // output columns per lane
  __shared__ float4 red[8][32];   // one float4 per lane of each of the 8 warps
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wi = warp & (wpr - 1);
  const int row = (blockIdx.x * 8 + warp) / wpr;
  const int rows = B * p.T * p.Hq;
  const bool live = row < rows;
  const int h = row % p.Hq;
  const int t = (row / p.Hq) % p.T;
  const int b = row / (p.Hq * p.T);
  const int g = h / p.G, r = t * p.G + (h - g * p.G);
  bool bad = true;
  int nc = 0, L = 0;
  if (live) {
    L = seqlens[b];
    bad = seqlen_bad(L, p.T, p.max_seqlen, paged != 0, p.capacity, p.max_blocks);
    if (!bad && !p.balanced) nc = (L + p.chunk - 1) / p.chunk;
  }
  grid_dependency_wait();   // launched early (programmatic dependent launch): the partials are ready after this
  // chunks of this (b, g): fixed length, or the balanced plan the split kernel wrote
  size_t item0 = ((size_t)b * p.Hkv + g) * p.max_chunks;
  if (p.balanced && live && !bad) {
    const int first = p.plan[3 * b], n_b = p.plan[3 * b + 1], chunk_b = p.plan[3 * b + 2];
    nc = (L + chunk_b - 1) / chunk_b;
    item0 = (size_t)p.Hkv * first + (size_t)g * n_b;
  }

  float acc[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
  float lse_row = -INFINITY;
  if (nc > 0) {
    const float* lse0 = part_lse + item0 * p.R + r;            // chunk c at lse0[c * R]
    const float* src0 = part_o + (item0 * p.R + r) * D + lane * kPer;
    const size_t cstride = (size_t)p.R * D;                    // floats between consecutive chunks of this row
    const int n0 = min(nc, 32);
    const float lc0 = lane < n0 ? __ldg(lse0 + (size_t)lane * p.R) : -INFINITY;
    float4 x[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int c = wi + u * wpr;
      x[u] = c < n0 ? load_part<kPer>(src0 + (size_t)c * cstride) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    // log-sum-exp over the chunks: every lane keeps a (max, sum) pair, then the pairs merge
    float m = lc0, sum = lc0 == -INFINITY ? 0.f : 1.f;
    for (int c = 32 + lane; c < nc; c += 32) {
      const float lc = __ldg(lse0 + (size_t)c * p.R);
      if (lc == -INFINITY) continue;
      if (lc > m) {
        sum = sum * expf(m - lc) + 1.f;
        m = lc;
      } else {
        sum += expf(lc - m);
      }
    }
    float M = m;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    float z = m == -INFINITY ? 0.f : sum * expf(m - M);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
    lse_row = M + logf(z);
    // chunk c of the first 32 has its weight on lane c
    const float wl0 = lc0 == -INFINITY ? 0.f : expf(lc0 - lse_row);
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int c = wi + u * wpr;
      const float w = __shfl_sync(0xffffffffu, wl0, c & 31);
      if (c < n0) accumulate<kPer>(acc, w, x[u]);
    }
    // what the first batch did not cover: more chunks of the first 32, later groups of 32
    for (int g0 = 0; g0 < nc; g0 += 32) {
      const int n = min(32, nc - g0);
      const int first = g0 == 0 ? wi + kBatch * wpr : wi;
      if (first >= n) continue;
      const float lc = g0 == 0 ? lc0 : (lane < n ? __ldg(lse0 + (size_t)(g0 + lane) * p.R) : -INFINITY);
      const float wl = lc == -INFINITY ? 0.f : expf(lc - lse_row);
      for (int j0 = first; j0 < n; j0 += kBatch * wpr) {
        float4 y[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          const int j = j0 + u * wpr;
          y[u] = j < n ? load_part<kPer>(src0 + (size_t)(g0 + j) * cstride) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          const int j = j0 + u * wpr;
          const float w = __shfl_sync(0xffffffffu, wl, j & 31);
          if (j < n) accumulate<kPer>(acc, w, y[u]);
        }
      }
    }
  }
  if (wpr > 1) {   // the row's warps add up in shared memory; its first warp writes
    if (wi != 0) {
      float4 v = make_float4(acc[0], acc[1], 0.f, 0.f);
      if constexpr (kPer == 4) {
        v.z = acc[2];
        v.w = acc[3];
      }
      red[warp][lane] = v;
    }
    __syncthreads();
    if (wi == 0) {
      for (int k = 1; k < wpr; ++k) {
        const float4 v = red[warp + k][lane];
        acc[0] += v.x;
        acc[1] += v.y;
        if constexpr (kPer == 4) {
          acc[2] += v.z;
          acc[3] += v.w;
        }
      }
    }
  }
  if (!live || wi != 0) return;
  if (bad) {
#pragma unroll
    for (int e = 0; e < kPer; ++e) acc[e] = NAN;
    lse_row = NAN;
  }
  const size_t orow = (((size_t)b * p.T + t) * p.Hq + h) * D + lane * kPer;
  if (o_bf16) {
    __nv_bfloat16* ob = reinterpret_cast<__nv_bfloat16*>(o) + orow;
#pragma unroll
    for (int e = 0; e < kPer; e += 2) *reinterpret_cast<__nv_bfloat162*>(ob + e) = __floats2bfloat162_rn(acc[e], acc[e + 1]);
  } else {
    float* of = reinterpret_cast<float*>(o) + orow;
#pragma unroll
    for (int e = 0; e < kPer; ++e) of[e] = acc[e];
  }
  if (lse && lane == 0) lse[((size_t)b * p.Hq + h) * p.T + t] = lse_row;
}

template <int D, int MT, bool PAGED, bool FP8 = false>
cudaError_t run_split(const CUtensorMap& tk, const CUtensorMap& tv, const SplitParams& sp, int B,
                      cudaStream_t stream) {
  using C = DecodeCfg<D, MT, FP8>;
  auto kern = decode_split_kernel<D, MT, PAGED, FP8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(sp.max_chunks, sp.Hkv, B);
  kern<<<grid, C::kThreads, C::kSmemBytes, stream>>>(tk, tv, sp);
  return cudaGetLastError();
}

}  // namespace

int decode_chunk_tokens(int B, int T, int G, int Hkv, int max_seqlen, int num_splits, bool fp8) {
  int chunk;
  if (num_splits > 0) {
    chunk = (int)(((long long)max_seqlen + num_splits - 1) / num_splits);
  } else {
    // Long chunks stream longer and leave fewer partials to merge; short ones
    // balance the grid.  Measured on B200: the warp-MMA kernel (2 CTAs per SM)
    // was best at 2048 tokens for 16 x 8 sequence-heads up to 32K keys and 4096
    // for 8 x 8 up to 128K, i.e. about 14 work items per SM; the FP8 kernel for
    // up to 8 rows (3 CTAs per SM) wants about 21; the tensor-core kernel
    // (2 CTAs per SM) about 9 for row tiles of up to 64 rows and about 4 for full
    // 128-row tiles, whose softmax makes each tile dearer.  Start long and halve
    // until the grid holds that many items (counted as if every sequence had
    // max_seqlen; row tiles of many new tokens count separately).
    const int R = G * T;
    const bool tc = decode_uses_tc(R, fp8);
    const long long units = (long long)B * Hkv * decode_row_tiles(T, G);
    const bool full_tiles = decode_tc_tile_tokens(T, G) * G > 64;
    const long long target = tc ? (full_tiles ? 640 : 1280) : (fp8 && R <= 8 ? 3072 : 2048);
    chunk = tc ? 16384 : 4096;
    while (chunk > 256 && units * (((long long)max_seqlen + chunk - 1) / chunk) < target) chunk >>= 1;
  }
  // a multiple of both kernels' tiles
  chunk = ((chunk + kDecodeTcTile - 1) / kDecodeTcTile) * kDecodeTcTile;
  return chunk < kDecodeTcTile ? kDecodeTcTile : chunk;
}

int decode_balanced_chunks(int B, int Hkv) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
    cudaGetLastError();   // no device here (workspace sizing on a host without one): a B200's 148 SMs
    sms = 148;
  }
  const int n = kBalancedItemsPerSlot * kDecodeTcCtasPerSm * sms / Hkv;
  return n > B ? n : B;
}

cudaError_t launch_decode(const DecodeLaunch& a, cudaStream_t stream) {
  const bool paged = a.page_table != nullptr;
  const int G = a.Hq / a.Hkv, R = G * a.T;
  SplitParams sp;
  sp.q = static_cast<const __nv_bfloat16*>(a.q);
  sp.k_scale = a.k_scale;
  sp.v_scale = a.v_scale;
  sp.seqlens = a.seqlens;
  sp.page_table = a.page_table;
  sp.part_o = a.part_o;
  sp.part_lse = a.part_lse;
  sp.status = a.status;
  sp.T = a.T;
  sp.Hq = a.Hq;
  sp.Hkv = a.Hkv;
  sp.G = G;
  sp.R = R;
  sp.chunk = a.chunk;
  sp.max_chunks = a.max_chunks;
  sp.capacity = a.capacity;
  sp.max_blocks = a.max_blocks;
  sp.num_blocks = a.num_blocks;
  sp.max_seqlen = a.max_seqlen;
  sp.scale_log2 = a.scale * kLog2e;
  sp.causal = a.causal;
  sp.balanced = a.balanced;
  sp.plan = a.plan;

  // K/V viewed as 3-D {d, Hkv, rows}: rows = B * capacity (contiguous) or num_blocks * 16 (paged)
  const uint64_t rows = paged ? (uint64_t)a.num_blocks * kPageTokens : (uint64_t)a.B * a.capacity;
  const bool tc = decode_uses_tc(R, a.fp8 != 0);
  const uint32_t box_rows = paged ? kPageTokens : (tc ? kDecodeTcTile : kDecodeTile);
  CUtensorMap tk, tv;
  const int eb = a.fp8 ? 1 : 2;   // bytes per cached element
  const uint64_t s1 = (uint64_t)a.d * eb, s2 = (uint64_t)a.Hkv * a.d * eb;
  const uint32_t box0 = 128 / eb;  // one 128-byte swizzle span
  if (encode_tmap_3d(&tk, a.k, a.d, a.Hkv, rows, s1, s2, box0, 1, box_rows, eb) ||
      encode_tmap_3d(&tv, a.v, a.d, a.Hkv, rows, s1, s2, box0, 1, box_rows, eb))
    return cudaErrorInvalidValue;

  cudaError_t e;
  if (tc) {
    e = launch_decode_tc(a, tk, tv, stream);   // bf16 above 16 rows per KV head, FP8 above 32
  } else if (a.fp8) {
    // api.cu admits FP8 caches with d == 128 only
    if (R <= 8) e = launch_decode_fp8_rows8(tk, tv, sp, a.B, paged, stream);
    else if (R <= 16) e = paged ? run_split<128, 1, true, true>(tk, tv, sp, a.B, stream)
                           : run_split<128, 1, false, true>(tk, tv, sp, a.B, stream);
    else e = paged ? run_split<128, 2, true, true>(tk, tv, sp, a.B, stream)
                   : run_split<128, 2, false, true>(tk, tv, sp, a.B, stream);
  } else if (a.d == 128) {   // at most kDecodeMmaRows (16) rows: one row group
    e = paged ? run_split<128, 1, true>(tk, tv, sp, a.B, stream) : run_split<128, 1, false>(tk, tv, sp, a.B, stream);
  } else {
    e = paged ? run_split<64, 1, true>(tk, tv, sp, a.B, stream) : run_split<64, 1, false>(tk, tv, sp, a.B, stream);
  }
  if (e != cudaSuccess) return e;

  // the combine kernel is launched as a programmatic dependent of the split kernel:
  // it starts launching while the split kernel's last CTAs finish and waits for them
  // warps per output row: enough that each warp merges at most four chunks
  int wpr = 1;
  while (wpr < 8 && wpr * 4 < sp.max_chunks) wpr *= 2;
  const long long rows_out = (long long)a.B * a.T * a.Hq;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((rows_out * wpr + 7) / 8));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const int paged_i = paged ? 1 : 0;
  const bool light = sp.max_chunks <= 2;
  auto kern = a.d == 128 ? (light ? decode_combine_kernel<128, 2> : decode_combine_kernel<128, 8>)
                         : (light ? decode_combine_kernel<64, 2> : decode_combine_kernel<64, 8>);
  e = cudaLaunchKernelEx(&cfg, kern, (const float*)a.part_o, (const float*)a.part_lse, a.seqlens, a.o, a.o_bf16,
                         a.lse, sp, a.B, paged_i, wpr);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace kvattn
