// Prefill attention on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// One CTA computes two 128-row query tiles (A: rows 256*qb .. +127, B: the next
// 128) of one (batch, query head); both tiles share every K/V tile it loads.
// Warp roles:
//   warps 0-3  softmax of tile A, warps 4-7 softmax of tile B: thread i of a
//              group owns query row i, which is TMEM lane i of its S and O;
//   warp 8     TMA producer: Q_A and Q_B once, then K_j, V_j into a 2-stage ring;
//   warp 9     MMA issuer (one thread).
// TMEM (512 columns): S_A | S_B | O_A | O_B.  Each softmax group reads its S row,
// turns it into bf16 probabilities P and writes P back over the first half of
// the same S columns; the PV MMA reads P straight from TMEM as its A operand
// (no shared-memory round trip).  The MMA issue order
//     PV_A(j), S_A(j+1), PV_B(j), S_B(j+1), PV_A(j+1), ...
// gives each softmax group the time of two MMAs to produce its next P.
// Because MMAs complete in issue order, "S_X(j) complete" also means
// "PV_X(j-1) complete", so a softmax group may rescale O_X as soon as it sees S_X(j).
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
// moved out of the inner loop, parallel over query tiles; FA3: warp
// specialisation with asynchronous TMA).
#include <cuda_bf16.h>
#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace kvattn {
namespace {

constexpr int kBM = 128;          // query rows per tile (two tiles per CTA)
constexpr int kBN = 128;          // keys per K/V tile
constexpr int kThreads = 320;     // 8 softmax warps + TMA warp + MMA warp
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;   // log2 of the largest allowed p

template <int D>
struct PrefillCfg {
  static constexpr int kHalves = D / 64;
  static constexpr int kTileBytes = kBN * D * 2;          // one Q, K or V tile
  static constexpr int kHalfBytes = kBN * 128;            // 128 rows x 128 B
  static constexpr int kQOff = 0;                         // Q_A, Q_B
  static constexpr int kKOff = kQOff + 2 * kTileBytes;    // K stages 0, 1
  static constexpr int kVOff = kKOff + 2 * kTileBytes;    // V stages 0, 1
  static constexpr int kBarOff = kVOff + 2 * kTileBytes;
  static constexpr int kUsed = kBarOff + 256;
  // one CTA per SM: it owns all 512 TMEM columns
  static constexpr int kSmemBytes = (kUsed + 1024) > 120 * 1024 ? (kUsed + 1024) : 120 * 1024;
  static constexpr int kTmemCols = 512;
  // TMEM columns: S of tile t at 128*t, O of tile t at 256 + D*t
  __host__ __device__ static constexpr int s_col(int t) { return 128 * t; }
  __host__ __device__ static constexpr int o_col(int t) { return 256 + D * t; }
};

enum Bar {
  B_Q = 0,
  B_KFULL = 1,    // +stage
  B_VFULL = 3,    // +stage
  B_KVEMPTY = 5,  // +stage
  B_SFULL = 7,    // +tile
  B_PFULL = 9,    // +tile
  B_ODONE = 11,   // +tile
  B_DRAIN = 13,   // only used when a bounded wait gave up
  B_COUNT = 14
};

struct PrefillParams {
  void* o;
  float* lse;
  unsigned* status;
  int N, Hq, Hkv, G, n_qblocks, n_ktiles;
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
__global__ void __launch_bounds__(kThreads, 1)
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
  const int qb = p.n_qblocks - 1 - blockIdx.z;      // heaviest causal blocks launch first
  const int kvh = h / p.G;
  // K/V tiles each query tile needs
  const int n_kv0 = p.causal ? min(2 * qb + 1, p.n_ktiles) : p.n_ktiles;
  const int n_load = p.causal ? min(2 * qb + 2, p.n_ktiles) : p.n_ktiles;   // = tile B's count, >= n_kv0

  if (threadIdx.x == 0) {
    mbar_init(&bars[B_Q], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[B_KFULL + s], 1);
      mbar_init(&bars[B_VFULL + s], 1);
      mbar_init(&bars[B_KVEMPTY + s], 1);
      mbar_init(&bars[B_SFULL + s], 1);
      mbar_init(&bars[B_PFULL + s], 4);
      mbar_init(&bars[B_ODONE + s], 1);
    }
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

  if (warp == 8) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      const uint64_t keep = policy_evict_last();    // K/V tiles are re-read by other query blocks and heads
      const uint64_t once = policy_evict_first();
      mbar_arrive_expect_tx(&bars[B_Q], 2 * C::kTileBytes);
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int hh = 0; hh < C::kHalves; ++hh)
          tma_load_4d(smem + C::kQOff + t * C::kTileBytes + hh * C::kHalfBytes, &tmQ, &bars[B_Q], hh * 64, h,
                      (2 * qb + t) * kBM, b, once);
      int last_t[2] = {-1, -1};
      for (int t = 0; t < n_load; ++t) {
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
  } else if (warp == 9) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(kBM, kBN, 0, 0);     // Q (K-major) x K^T (K-major)
      constexpr uint32_t idO = idesc_bf16(kBM, D, 0, 1);       // P (TMEM) x V (N-major)
      auto issue_s = [&](int t, int j) {      // S_t = Q_t K_j^T
        const uint32_t q_s = smem_u32(smem + C::kQOff + t * C::kTileBytes);
        const uint32_t k_s = smem_u32(smem + C::kKOff + (j & 1) * C::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kHalfBytes + (kk & 3) * 32;
          tc_mma_ss(tmem + C::s_col(t), smem_desc(q_s + off, 16, 1024), smem_desc(k_s + off, 16, 1024), idS, kk > 0);
        }
        tc_commit(&bars[B_SFULL + t]);
      };
      auto issue_pv = [&](int t, int j) {     // O_t += P_t V_j, P_t in the first 64 columns of S_t
        const uint32_t v_s = smem_u32(smem + C::kVOff + (j & 1) * C::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          tc_mma_ts(tmem + C::o_col(t), tmem + C::s_col(t) + kk * 8, smem_desc(v_s + kk * 16 * 128, C::kHalfBytes, 1024),
                    idO, (j > 0 || kk > 0) ? 1u : 0u);
      };
      bool ok = wait_or_abort(&bars[B_Q], 0, abort_flag, p.status) &&
                wait_or_abort(&bars[B_KFULL], 0, abort_flag, p.status);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(1, 0);
      }
      for (int j = 0; ok && j < n_load; ++j) {
        const int st = j & 1;
        const bool next_k = j + 1 < n_load;
        ok = wait_or_abort(&bars[B_VFULL + st], (j >> 1) & 1, abort_flag, p.status);
        if (!ok) break;
        if (j < n_kv0) {
          ok = wait_or_abort(&bars[B_PFULL + 0], j & 1, abort_flag, p.status);
          if (!ok) break;
          tc_fence_after();
          issue_pv(0, j);
          if (j == n_kv0 - 1) tc_commit(&bars[B_ODONE + 0]);
        }
        if (next_k) {
          ok = wait_or_abort(&bars[B_KFULL + ((j + 1) & 1)], ((j + 1) >> 1) & 1, abort_flag, p.status);
          if (!ok) break;
          tc_fence_after();
          if (j + 1 < n_kv0) issue_s(0, j + 1);
        }
        ok = wait_or_abort(&bars[B_PFULL + 1], j & 1, abort_flag, p.status);
        if (!ok) break;
        tc_fence_after();
        issue_pv(1, j);
        tc_commit(&bars[B_KVEMPTY + st]);       // K_j and V_j are no longer needed
        if (j == n_load - 1) tc_commit(&bars[B_ODONE + 1]);
        if (next_k) issue_s(1, j + 1);
      }
    }
  } else {
    // -------------------------------------------------- softmax warps 0-7
    const int t = warp >> 2;                            // query tile of this group
    const int row = (warp & 3) * 32 + lane;             // TMEM lane == query row in the tile
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t s_addr = lane_base + C::s_col(t);
    const uint32_t o_addr = lane_base + C::o_col(t);
    const int q_row = (2 * qb + t) * kBM + row;
    const int nkv = t ? n_load : n_kv0;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      if (!wait_or_abort(&bars[B_SFULL + t], j & 1, abort_flag, p.status)) { ok = false; break; }
      tc_fence_after();
      float s[kBN];
#pragma unroll
      for (int c = 0; c < kBN; c += 32) {
        uint32_t r[32];
        tmem_ld32(s_addr + c, r);
#pragma unroll
        for (int e = 0; e < 32; ++e) s[c + e] = __uint_as_float(r[e]);
      }
      tc_wait_ld();

      // mask (causal diagonal tile, or keys past N) and the row maximum of the raw scores
      const int key0 = j * kBN;
      const int lim = p.causal ? min(q_row - key0 + 1, p.N - key0) : (p.N - key0);   // visible keys: [0, lim)
      if (lim < kBN) {
#pragma unroll
        for (int c = 0; c < kBN; ++c) s[c] = (c < lim) ? s[c] : -INFINITY;
      }
      float mx8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx8[i] = max3f(s[i], s[i + 8], s[i + 16]);
#pragma unroll
      for (int c = 24; c + 8 < kBN; c += 16)
#pragma unroll
        for (int i = 0; i < 8; ++i) mx8[i] = max3f(mx8[i], s[c + i], s[c + 8 + i]);
#pragma unroll
      for (int i = 0; i < 8; ++i) mx8[i] = fmaxf(mx8[i], s[kBN - 8 + i]);
      float mx = max3f(max3f(mx8[0], mx8[1], mx8[2]), max3f(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
      mx *= p.scale_log2;                                      // scores in log2 units
      const bool raise = mx > m + kRescaleThreshold;          // also true on the first tile (m = -inf)
      const bool warp_raise = __any_sync(0xffffffffu, raise);
      float alpha = 1.f;
      if (warp_raise) {
        const float m_new = fmaxf(m, mx);
        alpha = ex2(m - m_new);                                 // 0 when m == -inf
        m = m_new;
      }
      const float neg_mu = (m == -INFINITY) ? 0.f : -m;
      float ls4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < kBN; c += 16) {
        uint32_t pk[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          const float p0 = ex2(fmaf(s[c + e], p.scale_log2, neg_mu));
          const float p1 = ex2(fmaf(s[c + e + 1], p.scale_log2, neg_mu));
          ls4[(e >> 1) & 3] += p0 + p1;
          pk[e / 2] = pack_bf16x2(p0, p1);
        }
        tmem_st8(s_addr + c / 2, pk);           // P row over the consumed S columns
      }
      const float ls = (ls4[0] + ls4[1]) + (ls4[2] + ls4[3]);
      l = l * alpha + ls;
      // O_t is stable here (PV_t(j-1) completed before S_t(j) did) and PV_t(j)
      // waits for this group's arrival below
      if (warp_raise && j > 0) {
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t r[32];
          tmem_ld32(o_addr + c, r);
          tc_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tmem_st32(o_addr + c, r);
        }
      }
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_PFULL + t]);
    }

    // ---------------------------------------------------------- epilogue
    if (ok && wait_or_abort(&bars[B_ODONE + t], 0, abort_flag, p.status)) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      const bool store = q_row < p.N;
      const size_t obase = (((size_t)b * p.N + q_row) * p.Hq + h) * D;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t r[32];
        tmem_ld32(o_addr + c, r);
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
  if (*abort_flag && warp == 9 && lane == 0) {
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
  p.n_qblocks = (a.N + 2 * kBM - 1) / (2 * kBM);
  p.n_ktiles = (a.N + kBN - 1) / kBN;
  p.scale_log2 = a.scale * kLog2e;
  p.causal = a.causal;
  p.o_bf16 = a.o_bf16;
  auto kern = prefill_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(a.Hq, a.B, p.n_qblocks);
  kern<<<grid, kThreads, C::kSmemBytes, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const PrefillLaunch& a, cudaStream_t stream) {
  return a.d == 128 ? run_prefill<128>(a, stream) : run_prefill<64>(a, stream);
}

}  // namespace kvattn
