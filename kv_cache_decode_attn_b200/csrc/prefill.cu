// Prefill attention on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// One CTA computes a 128-row query tile of one (batch, query head).  Warp roles:
//   warps 0-3  softmax / correction / epilogue: thread i owns query row i, which
//              is TMEM lane i of the S and O accumulators;
//   warp 4     TMA producer: Q once, then K_j and V_j tiles into a 2-stage ring;
//   warp 5     MMA issuer: S_j = Q K_j^T into one of two TMEM S buffers, and
//              O += P_j V_j into the TMEM O accumulator.
// S is double-buffered, so the tensor core computes S_{j+1} while the softmax
// warps turn S_j into P_j.  P_j (bf16) goes to shared memory in the K-major
// 128-byte-swizzled layout the MMA reads as its A operand.
//
// Online softmax (running maximum m and denominator l per row, base-2 exponent
// with the scale folded in): a row's reference maximum is only raised when the
// tile maximum exceeds it by more than 8 (a factor 256), so O in TMEM is rescaled
// rarely; p = 2^(s - m) then stays <= 256, and the final O / l and
// LSE = m + log2(l) use the same reference, so the result is exact.
//
// Method: "KV cache, flash attention" lesson, "片技巧" (per Q tile, loop over
// K/V tiles kept on chip; running softmax aggregation; write O once) and
// "Numerical trick"; "大模型面試笔记——Attention篇" section 2 (online safe
// softmax with the compensation factor); "[BEE-30062]" "背景" (FA2: scaling
// moved out of the inner loop, parallel over query tiles).
#include <cuda_bf16.h>
#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace kvattn {
namespace {

constexpr int kBM = 128;          // query rows per CTA
constexpr int kBN = 128;          // keys per tile
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;   // log2 of the largest allowed p

template <int D>
struct PrefillCfg {
  static constexpr int kHalves = D / 64;
  static constexpr int kTileBytes = kBN * D * 2;          // one K or V tile (= one Q tile)
  static constexpr int kHalfBytes = kBN * 128;            // 128 rows x 128 B
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kTileBytes;
  static constexpr int kVOff = kKOff + 2 * kTileBytes;
  static constexpr int kPOff = kVOff + 2 * kTileBytes;
  static constexpr int kPBytes = kBM * kBN * 2;
  static constexpr int kBarOff = kPOff + kPBytes;
  static constexpr int kUsed = kBarOff + 256;
  // one CTA per SM: it owns all 512 TMEM columns
  static constexpr int kSmemBytes = (kUsed + 1024) > 120 * 1024 ? (kUsed + 1024) : 120 * 1024;
  static constexpr int kTmemCols = 512;
  static constexpr int kSCol0 = 0, kSCol1 = 128, kOCol = 256;
};

enum Bar {
  B_Q = 0,
  B_KFULL = 1,    // +stage
  B_VFULL = 3,    // +stage
  B_KVEMPTY = 5,  // +stage
  B_SFULL = 7,    // +buffer
  B_SFREE = 9,    // +buffer
  B_PFULL = 11,
  B_ODONE = 12,
  B_DRAIN = 13,   // only used when a bounded wait gave up
  B_COUNT = 14
};

struct PrefillParams {
  void* o;
  float* lse;
  unsigned* status;
  int N, Hq, Hkv, G, n_qtiles;
  float scale_log2;
  int causal, o_bf16;
};

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                              unsigned* status) {
  if (*abort_flag) return false;
  if (mbar_wait(bar, parity)) return true;
  atomicOr(status, DEV_TIMEOUT);
  *abort_flag = 1;
  return false;
}

template <int D>
__global__ void __launch_bounds__(192, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  using C = PrefillCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x, b = blockIdx.y;
  const int qt = p.n_qtiles - 1 - blockIdx.z;      // heaviest causal tiles launch first
  const int kvh = h / p.G;
  const int n_kv = p.causal ? (qt + 1) : (p.N + kBN - 1) / kBN;

  if (threadIdx.x == 0) {
    mbar_init(&bars[B_Q], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[B_KFULL + s], 1);
      mbar_init(&bars[B_VFULL + s], 1);
      mbar_init(&bars[B_KVEMPTY + s], 1);
      mbar_init(&bars[B_SFULL + s], 1);
      mbar_init(&bars[B_SFREE + s], 4);
    }
    mbar_init(&bars[B_PFULL], 4);
    mbar_init(&bars[B_ODONE], 1);
    mbar_init(&bars[B_DRAIN], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      const uint64_t keep = policy_evict_last();    // K/V tiles are re-read by other query tiles
      mbar_arrive_expect_tx(&bars[B_Q], C::kTileBytes);
#pragma unroll
      for (int hh = 0; hh < C::kHalves; ++hh)
        tma_load_4d(smem + C::kQOff + hh * C::kHalfBytes, &tmQ, &bars[B_Q], hh * 64, h, qt * kBM, b,
                    policy_evict_first());
      int last_t[2] = {-1, -1};
      for (int t = 0; t < n_kv; ++t) {
        const int st = t & 1;
        if (t >= 2 && !wait_or_abort(&bars[B_KVEMPTY + st], ((t >> 1) - 1) & 1, abort_flag, p.status)) break;
        last_t[st] = t;
        mbar_arrive_expect_tx(&bars[B_KFULL + st], C::kTileBytes);
#pragma unroll
        for (int hh = 0; hh < C::kHalves; ++hh)
          tma_load_4d(smem + C::kKOff + st * C::kTileBytes + hh * C::kHalfBytes, &tmK, &bars[B_KFULL + st], hh * 64,
                      kvh, t * kBN, b, keep);
        mbar_arrive_expect_tx(&bars[B_VFULL + st], C::kTileBytes);
#pragma unroll
        for (int hh = 0; hh < C::kHalves; ++hh)
          tma_load_4d(smem + C::kVOff + st * C::kTileBytes + hh * C::kHalfBytes, &tmV, &bars[B_VFULL + st], hh * 64,
                      kvh, t * kBN, b, keep);
      }
      // no copy may still be landing in shared memory when the CTA exits
      mbar_wait(&bars[B_Q], 0);
      for (int st = 0; st < 2; ++st) {
        if (last_t[st] < 0) continue;
        mbar_wait(&bars[B_KFULL + st], (last_t[st] >> 1) & 1);
        mbar_wait(&bars[B_VFULL + st], (last_t[st] >> 1) & 1);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(kBM, kBN, 0, 0);     // Q (K-major) x K^T (K-major)
      constexpr uint32_t idO = idesc_bf16(kBM, D, 0, 1);       // P (K-major) x V (N-major)
      const uint32_t q_s = smem_u32(smem + C::kQOff);
      const uint32_t p_s = smem_u32(smem + C::kPOff);
      auto issue_s = [&](int t) {
        const int st = t & 1;
        const uint32_t k_s = smem_u32(smem + C::kKOff + st * C::kTileBytes);
        const uint32_t d_tmem = tmem + (st ? C::kSCol1 : C::kSCol0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kHalfBytes + (kk & 3) * 32;
          tc_mma_ss(d_tmem, smem_desc(q_s + off, 16, 1024), smem_desc(k_s + off, 16, 1024), idS, kk > 0);
        }
        tc_commit(&bars[B_SFULL + st]);
      };
      bool ok = wait_or_abort(&bars[B_Q], 0, abort_flag, p.status) &&
                wait_or_abort(&bars[B_KFULL], 0, abort_flag, p.status);
      if (ok) {
        tc_fence_after();
        issue_s(0);
      }
      for (int j = 0; ok && j < n_kv; ++j) {
        const int t = j + 1;
        if (t < n_kv) {
          ok = wait_or_abort(&bars[B_KFULL + (t & 1)], (t >> 1) & 1, abort_flag, p.status) &&
               (t < 2 || wait_or_abort(&bars[B_SFREE + (t & 1)], ((t >> 1) - 1) & 1, abort_flag, p.status));
          if (!ok) break;
          tc_fence_after();
          issue_s(t);
        }
        ok = wait_or_abort(&bars[B_PFULL], j & 1, abort_flag, p.status) &&
             wait_or_abort(&bars[B_VFULL + (j & 1)], (j >> 1) & 1, abort_flag, p.status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t v_s = smem_u32(smem + C::kVOff + (j & 1) * C::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint32_t a_off = (kk >> 2) * (kBM * 128) + (kk & 3) * 32;
          tc_mma_ss(tmem + C::kOCol, smem_desc(p_s + a_off, 16, 1024),
                    smem_desc(v_s + kk * 16 * 128, C::kHalfBytes, 1024), idO, (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&bars[B_ODONE]);
        tc_commit(&bars[B_KVEMPTY + (j & 1)]);
      }
    }
  } else {
    // ------------------------------------------------------ softmax warps 0-3
    const int row = warp * 32 + lane;                   // TMEM lane == query row in the tile
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    const int q_row = qt * kBM + row;
    float m = -INFINITY, l = 0.f;
    uint8_t* p_tile = smem + C::kPOff;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int sb = j & 1;
      if (!wait_or_abort(&bars[B_SFULL + sb], (j >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
      tc_fence_after();
      float s[kBN];
#pragma unroll
      for (int c = 0; c < kBN; c += 32) {
        uint32_t r[32];
        tmem_ld32(lane_base + (sb ? C::kSCol1 : C::kSCol0) + c, r);
#pragma unroll
        for (int e = 0; e < 32; ++e) s[c + e] = __uint_as_float(r[e]);
      }
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_SFREE + sb]);

      // mask: causal diagonal tile, or keys past N
      const int key0 = j * kBN;
      const int lim = p.causal ? min(q_row - key0 + 1, p.N - key0) : (p.N - key0);   // visible keys: [0, lim)
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < kBN; ++c) {
        s[c] = (c < lim) ? s[c] * p.scale_log2 : -INFINITY;
        mx = fmaxf(mx, s[c]);
      }
      const bool raise = mx > m + kRescaleThreshold;          // also true on the first tile (m = -inf)
      const bool warp_raise = __any_sync(0xffffffffu, raise);
      float alpha = 1.f;
      if (warp_raise) {
        const float m_new = fmaxf(m, mx);
        alpha = ex2(m - m_new);                                 // 0 when m == -inf
        m = m_new;
      }
      const float mu = (m == -INFINITY) ? 0.f : m;
      float ls = 0.f;
      uint32_t pk[kBN / 2];
#pragma unroll
      for (int c = 0; c < kBN; c += 2) {
        const float p0 = ex2(s[c] - mu), p1 = ex2(s[c + 1] - mu);
        ls += p0 + p1;
        pk[c / 2] = pack_bf16x2(p0, p1);
      }
      l = l * alpha + ls;

      // PV of the previous tile must be done before P and O are touched
      if (j > 0) {
        if (!wait_or_abort(&bars[B_ODONE], (j - 1) & 1, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        if (warp_raise) {
#pragma unroll
          for (int c = 0; c < D; c += 32) {
            uint32_t r[32];
            tmem_ld32(lane_base + C::kOCol + c, r);
            tc_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st32(lane_base + C::kOCol + c, r);
          }
          tc_wait_st();
        }
      }
      // P row -> shared memory, K-major with the 128-byte swizzle (two 64-key halves)
#pragma unroll
      for (int ch = 0; ch < kBN / 8; ++ch) {
        const int half = ch >> 3, cw = ch & 7;
        uint4 v = make_uint4(pk[ch * 4 + 0], pk[ch * 4 + 1], pk[ch * 4 + 2], pk[ch * 4 + 3]);
        *reinterpret_cast<uint4*>(p_tile + half * (kBM * 128) + row * 128 + ((cw ^ (row & 7)) << 4)) = v;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_PFULL]);
    }

    // ---------------------------------------------------------- epilogue
    if (ok && wait_or_abort(&bars[B_ODONE], (n_kv - 1) & 1, abort_flag, p.status)) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      const bool store = q_row < p.N;
      const size_t obase = (((size_t)b * p.N + q_row) * p.Hq + h) * D;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t r[32];
        tmem_ld32(lane_base + C::kOCol + c, r);
        tc_wait_ld();
        if (store) {
          if (p.o_bf16) {
            __nv_bfloat16* ob = reinterpret_cast<__nv_bfloat16*>(p.o) + obase + c;
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              uint4 v = make_uint4(pack_bf16x2(__uint_as_float(r[e]) * inv_l, __uint_as_float(r[e + 1]) * inv_l),
                                   pack_bf16x2(__uint_as_float(r[e + 2]) * inv_l, __uint_as_float(r[e + 3]) * inv_l),
                                   pack_bf16x2(__uint_as_float(r[e + 4]) * inv_l, __uint_as_float(r[e + 5]) * inv_l),
                                   pack_bf16x2(__uint_as_float(r[e + 6]) * inv_l, __uint_as_float(r[e + 7]) * inv_l));
              *reinterpret_cast<uint4*>(ob + e) = v;
            }
          } else {
            float* of = reinterpret_cast<float*>(p.o) + obase + c;
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4*>(of + e) =
                  make_float4(__uint_as_float(r[e]) * inv_l, __uint_as_float(r[e + 1]) * inv_l,
                              __uint_as_float(r[e + 2]) * inv_l, __uint_as_float(r[e + 3]) * inv_l);
          }
        }
      }
      if (store && p.lse) p.lse[((size_t)b * p.Hq + h) * p.N + q_row] = (m + log2f(l)) * kLn2;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag && warp == 5 && lane == 0) {
    // a wait gave up: let every tensor-core op this CTA issued drain before TMEM is released
    tc_commit(&bars[B_DRAIN]);
    mbar_wait(&bars[B_DRAIN], 0);
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int D>
cudaError_t run_prefill(const PrefillLaunch& a, cudaStream_t stream) {
  using C = PrefillCfg<D>;
  CUtensorMap tq, tk, tv;
  // 4-D views {d, heads, N, B}; box {64, 1, 128, 1} with the 128-byte swizzle
  auto enc = [&](CUtensorMap* m, const void* base, int heads) {
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)a.N, (cuuint64_t)a.B};
    cuuint64_t str[3] = {(cuuint64_t)D * 2, (cuuint64_t)heads * D * 2, (cuuint64_t)a.N * heads * D * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)kBN, 1};
    return encode_tmap_nd(m, base, 4, dims, str, box);
  };
  if (enc(&tq, a.q, a.Hq) || enc(&tk, a.k, a.Hkv) || enc(&tv, a.v, a.Hkv)) return cudaErrorInvalidValue;
  PrefillParams p;
  p.o = a.o;
  p.lse = a.lse;
  p.status = a.status;
  p.N = a.N;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.G = a.Hq / a.Hkv;
  p.n_qtiles = (a.N + kBM - 1) / kBM;
  p.scale_log2 = a.scale * kLog2e;
  p.causal = a.causal;
  p.o_bf16 = a.o_bf16;
  auto kern = prefill_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(a.Hq, a.B, p.n_qtiles);
  kern<<<grid, 192, C::kSmemBytes, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const PrefillLaunch& a, cudaStream_t stream) {
  return a.d == 128 ? run_prefill<128>(a, stream) : run_prefill<64>(a, stream);
}

}  // namespace kvattn
