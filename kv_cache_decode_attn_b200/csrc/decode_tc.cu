// Split-KV attention of T new tokens against a KV cache on the sm_100a tensor
// cores, for many query rows per KV head (R = (Hq/Hkv) * T above 16: grouped
// heads times several new tokens -- a speculative-verify step of 8 or 16
// tokens, or a whole prompt chunk appended to an existing cache, which is
// chunked prefill / prefill against a cached prefix).
//
// The rows of KV head g are numbered r = t * G + hh (token t, grouped head hh)
// and cut into row tiles of TT whole tokens (TT * G <= 128 rows, the tcgen05 M).
// One CTA owns one work item (row tile, key chunk c, KV head g, sequence b) and
// writes the same per-chunk partials (normalised O and log-sum-exp per row) that
// the combine kernel merges.  With the bottom-right mask a row tile only reads
// keys up to the last one its last token sees.  Warp roles:
//   warps 0..3  softmax: thread i owns row i (TMEM lane i); warps whose rows are
//               all >= R stay idle (FP8 with R <= 64: warps 3 and 2 help convert
//               the K and V tiles);
//   warps 4, 6  TMA producers: warp 4 loads Q once and the K tiles, warp 6 the V
//               tiles, each into its own 2-stage ring with the evict-first L2
//               policy (64-token tiles; contiguous: one 64-row box per 64
//               columns of d; paged: one 16-row box per physical block, its
//               page-table entry checked first).  K is released by S_j, V only by
//               PV_j, so separate producers let the K ring run ahead (FP8:
//               warps 7 and 6 copy and convert, see below);
//   warp 5      MMA issuer: S_j = Q K_j^T (SS) into one of two TMEM S buffers,
//               O += P_j V_j (P read from TMEM, where the softmax wrote it over
//               the consumed S columns).  S_{j+1} is issued before PV_j, so the
//               tensor core computes the next scores while the softmax runs.
// Online softmax with the lazy rescale of the prefill kernel: a row's reference
// maximum is raised only when a tile's maximum exceeds it by more than 8.
// 64-token tiles keep a CTA at 99.6 KB of shared memory and 256 TMEM columns, so
// two CTAs share an SM: one streams while the other starts up or writes its
// partials, and the grid's last wave is split over twice as many slots.
//
// Method: "[BEE-30062] FlashAttention 與高效注意力核心", "背景" and
// "為長上下文推論啟用 FlashDecoding" (split along the KV length, stable merge of
// partial softmax results); "Effizienz", "Der wichtige Maskenfehler beim Cache"
// (several new tokens need the positional offset in the mask); "大模型面試笔记"
// section 2 (online safe softmax).
#include <cuda_bf16.h>
#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace kvattn {
namespace {

constexpr int kRows = 128;   // MMA M (query rows per KV head, padded)
constexpr int kTok = kDecodeTcTile;   // keys per K/V tile (the host's tensor-map box)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

constexpr int kStages = 2;    // K/V ring stages (S is double-buffered in TMEM)
constexpr int kCtasPerSm = kDecodeTcCtasPerSm;   // shared memory and TMEM of one CTA
// FP8 adds warp 7: the K converter runs on warp 7 and the V converter on warp 6, so
// that neither shares an SM sub-partition (warp index mod 4) with softmax warps 0
// and 1, the only ones a tile of up to 64 rows uses.
template <bool FP8>
constexpr int tc_threads() { return FP8 ? 256 : 224; }

// FP8: the cache holds e4m3 codes.  The copies land in a ring of raw stages; the K
// (V) producer warp then converts each raw tile into one f16 K (V) tile in the
// operand layout the MMAs read (every e4m3 value is exact in f16), and the MMAs run
// on f16 operands: Q is converted to f16 in place once per CTA (exact for bf16
// magnitudes 2^-14 .. 65504) and P is stored as f16.
template <int D, bool FP8 = false>
struct TcCfg {
  static constexpr int kHalves = D / 64;
  static constexpr int kQHalfBytes = kRows * 128;            // Q: 128 rows x 128 B per 64 columns of d
  static constexpr int kHalfBytes = kTok * 128;              // K or V tile: kTok rows x 128 B
  static constexpr int kQBytes = kRows * D * 2;
  static constexpr int kTileBytes = kTok * D * 2;            // one 16-bit K or V tile
  static constexpr int kRawBytes = kTok * D;                 // one e4m3 K or V tile (FP8)
  static constexpr int kOperandStages = FP8 ? 1 : kStages;   // 16-bit tiles the MMAs read
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kQBytes;              // K stages (FP8: the converted K tile)
  static constexpr int kVOff = kKOff + kOperandStages * kTileBytes;   // V stages (FP8: the converted V tile)
  static constexpr int kRawKOff = kVOff + kOperandStages * kTileBytes;   // FP8: raw K stages
  static constexpr int kRawVOff = kRawKOff + (FP8 ? kStages * kRawBytes : 0);
  static constexpr int kBarOff = kRawVOff + (FP8 ? kStages * kRawBytes : 0);
  static constexpr int kPlanOff = kBarOff + 256;             // balanced split: the plan, built per CTA
  static constexpr int kPlanBytes = kBalancedMaxB * 4 * 4;   // length, base share, chunks, first chunk
  static constexpr int kSmemBytes = kPlanOff + kPlanBytes + 1024;
  static constexpr int kSCols = kTok;                        // one S buffer (fp32 scores of a tile)
  static constexpr int kOCol = 2 * kSCols;                   // S0 | S1 | O
  static constexpr int kTmemCols = kOCol + D <= 256 ? 256 : 512;
};

// K and V stages are released separately: K_j as soon as S_j is done, V_j once PV_j is done.
// P_FULL is one barrier per S buffer: S_{j+1} exists before PV_j is issued, so a
// fast softmax warp may finish tile j+1 while a slow one is still on tile j, and
// its arrival must not count towards tile j.
// O_DONE completes once per PV and is waited on only one tile behind (before a
// rescale, where PV_{j-2} is known to be done); the epilogue, which may be two
// PVs behind, waits on O_FINAL, committed once after the last PV.
// K/V barriers: one per ring stage; S_FULL / P_FULL: one per S buffer.
enum TcBar {
  T_Q = 0,
  T_KFULL = 1,
  T_VFULL = T_KFULL + kStages,
  T_KEMPTY = T_VFULL + kStages,
  T_VEMPTY = T_KEMPTY + kStages,
  T_SFULL = T_VEMPTY + kStages,
  T_PFULL = T_SFULL + 2,
  T_ODONE = T_PFULL + 2,
  T_OFINAL,
  T_DRAIN,
  T_QC,        // FP8: Q is converted to f16
  T_KCFULL,    // FP8: the converted K tile is ready
  T_VCFULL,
  T_KCEMPTY,   // FP8: the MMA reading the converted K tile is done
  T_VCEMPTY,
  T_KHDONE,    // FP8, R <= 64: the helper warp has converted its half of the K tile
  T_VHDONE,
  T_COUNT
};

struct TcParams {
  const float* k_scale;   // FP8: [Hkv]
  const float* v_scale;
  const int32_t* seqlens;
  const int32_t* page_table;
  float* part_o;
  float* part_lse;
  unsigned* status;
  int T, Hq, Hkv, G, R;   // R = G * T rows per KV head (the partials' row count)
  int TT;                 // tokens per row tile (TT * G <= 128)
  int chunk, max_chunks, capacity, max_blocks, num_blocks, max_seqlen;
  float scale_log2;
  int causal;
  int balanced, n_chunks, B;   // balanced split: n_chunks over the batch (per KV head)
  int* plan;                   // [B, 3] written by CTA 0 for the combine kernel
};

// Balanced split: the chunks of this launch and this CTA's (sequence, KV head, chunk),
// built identically by every CTA from the lengths (integer arithmetic only).  Sequence
// b gets 1 + floor(L_b (N - B) / sum L) chunks plus one more if its remainder is among
// the N - B - sum(floor) largest (ties by index), so exactly N chunks in all; its chunk
// length is ceil(L_b / n_b) rounded up to whole 64-token tiles.  Linear block index
// i = Hkv * first_b + g * n_b + c is the partial's index.  Lengths outside
// [1, max_seqlen] count as clamped (such a sequence's rows are reported invalid anyway).
struct BalancedItem {
  int b, g, c, chunk;
};
__device__ __forceinline__ BalancedItem balanced_item(const TcParams& p, int* plan_smem) {
  int* len = plan_smem;                                   // [B]
  int* base = plan_smem + kBalancedMaxB;                  // [B] floor share
  int* nb = plan_smem + 2 * kBalancedMaxB;                // [B] chunks
  int* first = plan_smem + 3 * kBalancedMaxB;             // [B] first chunk
  const int B = p.B, N = p.n_chunks;
  for (int i = threadIdx.x; i < B; i += blockDim.x) len[i] = min(max(p.seqlens[i], 1), p.max_seqlen);
  __syncthreads();
  long long tot = 0;
  for (int i = 0; i < B; ++i) tot += len[i];
  const long long spare = N - B;
  for (int i = threadIdx.x; i < B; i += blockDim.x) base[i] = (int)((long long)len[i] * spare / tot);
  __syncthreads();
  long long used = 0;
  for (int i = 0; i < B; ++i) used += base[i];
  const long long extra = spare - used;                   // 0 <= extra < B
  for (int i = threadIdx.x; i < B; i += blockDim.x) {
    const long long ri = (long long)len[i] * spare % tot;
    int rank = 0;
    for (int j = 0; j < B; ++j) {
      const long long rj = (long long)len[j] * spare % tot;
      rank += (rj > ri) || (rj == ri && j < i);
    }
    nb[i] = 1 + base[i] + (rank < extra ? 1 : 0);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int f = 0;
    for (int i = 0; i < B; ++i) {
      first[i] = f;
      f += nb[i];
    }
  }
  __syncthreads();
  BalancedItem it;
  const int id = blockIdx.x;
  int b = 0;
  while (b + 1 < B && p.Hkv * first[b + 1] <= id) ++b;
  const int rem = id - p.Hkv * first[b];
  it.b = b;
  it.g = rem / nb[b];
  it.c = rem - it.g * nb[b];
  const int per = (len[b] + nb[b] - 1) / nb[b];
  it.chunk = (per + kTok - 1) / kTok * kTok;
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < B; i += blockDim.x) {
      const int per_i = (len[i] + nb[i] - 1) / nb[i];
      p.plan[3 * i] = first[i];
      p.plan[3 * i + 1] = nb[i];
      p.plan[3 * i + 2] = (per_i + kTok - 1) / kTok * kTok;
    }
  return it;
}

__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                        unsigned* status) {
  if (*abort_flag) return false;
  if (mbar_wait(bar, parity)) return true;
  atomicOr(status, DEV_TIMEOUT);
  *abort_flag = 1;
  return false;
}

// Convert one raw e4m3 tile (kTok rows of D codes, 128-byte rows with the 128-byte
// swizzle the copy applies) into the f16 operand tile (two halves of D/2 columns,
// kTok rows of 128 bytes, same swizzle), one warp.  Called for d = 128 only: a raw
// row of D codes is one 128-byte swizzle span.
// 16-byte shared accesses are served per quarter-warp, one 128-byte wavefront for
// eight lanes that hit eight different 16-byte bank groups.  So each quarter-warp
// takes rows 2p and 2p+1 of a row pair, four chunks of each, from opposite halves of
// d: chunk c of row r sits in bank group c ^ (r & 7) of the raw tile and c' ^ (r & 7)
// (c' = 2 (c mod 4) or that + 1) of its half of the f16 tile, and the two rows'
// groups are then disjoint for the load and for both stores.  (Eight chunks of one
// row put chunks c and c + 4, which land in the two halves at the same offset, on
// one bank group: every store took two wavefronts.)  Pass k converts rows 4k .. 4k+3;
// the warp runs passes k0 .. k1 - 1 (all kTok / 4 of them, or half when two warps
// share the tile).
template <int D>
__device__ __forceinline__ void convert_tile_e4m3(const uint8_t* raw, uint8_t* conv, int lane, int k0, int k1) {
  const int hi = (lane >> 2) & 1, v = (lane >> 3) & 1;
#pragma unroll 4
  for (int k = k0; k < k1; ++k) {
    const int r = 2 * (2 * k + (lane >> 4)) + hi;             // row: rows 4k .. 4k+3 per pass
    const int c = ((hi ^ v) << 2) + (lane & 3);               // 16-code chunk (d = 16c .. 16c+15)
    const uint4 w = *reinterpret_cast<const uint4*>(raw + r * 128 + ((c ^ (r & 7)) << 4));
    uint32_t o[8];
    e4m3x4_to_f16x2x2(w.x, o[0], o[1]);
    e4m3x4_to_f16x2x2(w.y, o[2], o[3]);
    e4m3x4_to_f16x2x2(w.z, o[4], o[5]);
    e4m3x4_to_f16x2x2(w.w, o[6], o[7]);
    const int c0 = (c & 3) * 2;                           // first 16-byte chunk in the half's row
    uint8_t* rowp = conv + (c >> 2) * (kTok * 128) + r * 128;
    *reinterpret_cast<uint4*>(rowp + ((c0 ^ (r & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
    *reinterpret_cast<uint4*>(rowp + (((c0 + 1) ^ (r & 7)) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

// bf16 pair to f16 pair, round to nearest (exact for magnitudes 2^-14 .. 65504).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t x) {
  return pack_f16x2(__uint_as_float(x << 16), __uint_as_float(x & 0xFFFF0000u));
}

template <int D, bool PAGED, bool FP8>
__global__ void __launch_bounds__(tc_threads<FP8>(), kCtasPerSm)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const TcParams p) {
  using C = TcCfg<D, FP8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + T_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int c, rt, g, b, chunk;
  size_t item;
  if (p.balanced) {
    const BalancedItem bi = balanced_item(p, reinterpret_cast<int*>(smem + C::kPlanOff));
    c = bi.c;
    rt = 0;
    g = bi.g;
    b = bi.b;
    chunk = bi.chunk;
    item = blockIdx.x;
  } else {
    c = blockIdx.x % p.max_chunks;
    rt = blockIdx.x / p.max_chunks;
    g = blockIdx.y;
    b = blockIdx.z;
    chunk = p.chunk;
    item = ((size_t)b * p.Hkv + g) * p.max_chunks + c;
  }
  const int L = p.seqlens[b];
  // invalid lengths are reported (and their rows made NaN) by the combine kernel
  if (L < p.T || L > p.max_seqlen || (!PAGED && L > p.capacity) ||
      (PAGED && (L + kPageTokens - 1) / kPageTokens > p.max_blocks))
    return;
  const int tok_begin = c * chunk;
  if (tok_begin >= L) return;   // the combine reads only chunks that start before L
  const int t0 = rt * p.TT;                      // first token of this row tile
  const int tile_tokens = min(p.TT, p.T - t0);
  const int tile_rows = tile_tokens * p.G;       // live rows: 0 .. tile_rows - 1
  const size_t row0 = item * p.R + (size_t)t0 * p.G;   // partial row of tile row 0
  int tok_end = min(tok_begin + chunk, L);
  if (p.causal) tok_end = min(tok_end, L - p.T + t0 + tile_tokens);   // last token's first invisible key
  if (tok_end <= tok_begin) {
    // no key of this chunk is visible to any row of the tile: an empty partial
    for (int i = threadIdx.x; i < tile_rows * D; i += blockDim.x) p.part_o[row0 * D + i] = 0.f;
    for (int r = threadIdx.x; r < tile_rows; r += blockDim.x) p.part_lse[row0 + r] = -INFINITY;
    return;
  }
  const int n_tiles = (tok_end - tok_begin + kTok - 1) / kTok;
  const int active_warps = (tile_rows + 31) / 32;
  // FP8 with at most 64 rows: softmax warps 2 and 3 are free and convert the second half
  // of every K (warp 3) and V (warp 2) tile beside the producers
  const bool conv_split = FP8 && active_warps <= 2;
  float scale_log2 = p.scale_log2, v_mul = 1.f;   // FP8: K scale in the exponent, V scale on O
  if constexpr (FP8) {
    const float ks = __ldg(p.k_scale + g), vs = __ldg(p.v_scale + g);
    scale_log2 = p.scale_log2 * ks;
    v_mul = vs;
    if (!(ks > 0.f && ks <= 3.402823466e38f && vs > 0.f && vs <= 3.402823466e38f)) {
      // a scale that is not a positive finite number: the whole CTA leaves before any
      // barrier (the scales are uniform across it)
      if (threadIdx.x == 0 && c == 0 && rt == 0) atomicOr(p.status, DEV_SCALE);
      for (int r = threadIdx.x; r < tile_rows; r += blockDim.x) p.part_lse[row0 + r] = NAN;
      return;
    }
  }

  if (threadIdx.x == 0) {
    mbar_init(&bars[T_Q], 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars[T_KFULL + s], 1);
      mbar_init(&bars[T_VFULL + s], 1);
      mbar_init(&bars[T_KEMPTY + s], 1);
      mbar_init(&bars[T_VEMPTY + s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[T_SFULL + s], 1);
      mbar_init(&bars[T_PFULL + s], active_warps);
    }
    mbar_init(&bars[T_ODONE], 1);
    mbar_init(&bars[T_OFINAL], 1);
    mbar_init(&bars[T_DRAIN], 1);
    mbar_init(&bars[T_QC], 1);
    mbar_init(&bars[T_KCFULL], 1);
    mbar_init(&bars[T_VCFULL], 1);
    mbar_init(&bars[T_KCEMPTY], 1);
    mbar_init(&bars[T_VCEMPTY], 1);
    if (FP8) {
      mbar_init(&bars[T_KHDONE], 1);
      mbar_init(&bars[T_VHDONE], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  // rows TT*G..127 of the Q tile are never loaded: make them zero (whole 128-byte rows);
  // rows of tokens >= T inside the box are zero-filled by the copy
  {
    const int box_rows = p.TT * p.G;
    const int per_half = (kRows - box_rows) * 8;   // 16-byte chunks of rows box_rows..127 in one half of d
    for (int i = threadIdx.x; i < per_half * C::kHalves; i += blockDim.x) {
      const int half = i / per_half, rem = i - half * per_half;
      *reinterpret_cast<uint4*>(smem + C::kQOff + half * C::kQHalfBytes + box_rows * 128 + rem * 16) =
          make_uint4(0, 0, 0, 0);
    }
  }
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (FP8 && (warp == 7 || warp == 6)) {
    // ------------------------------------------------ FP8 producers and converters
    // Lane 0 copies raw e4m3 tiles into a 2-stage ring; the whole warp converts each
    // raw tile into the one f16 operand tile once the MMA has finished reading the
    // previous one, then refills the raw stage it has just read.  Warp 7 handles K
    // (and Q), warp 6 V; warp 4 has no work.  With conv_split the warp converts rows
    // 0 .. kTok/2 - 1 and its helper (below) the rest; the tile is published, and its raw
    // stage refilled, once the helper has arrived on its barrier for that tile.
    const bool is_k = warp == 7;
    const CUtensorMap* map = is_k ? &tmK : &tmV;
    uint8_t* raw_ring = smem + (is_k ? C::kRawKOff : C::kRawVOff);
    uint8_t* conv = smem + (is_k ? C::kKOff : C::kVOff);
    const int full0 = is_k ? T_KFULL : T_VFULL;
    uint64_t* cfull = &bars[is_k ? T_KCFULL : T_VCFULL];
    uint64_t* cempty = &bars[is_k ? T_KCEMPTY : T_VCEMPTY];
    const uint64_t pol = policy_evict_first();
    constexpr int kBlocks = kTok / kPageTokens;
    auto copy_tile = [&](int i) {      // lane 0 only
      uint8_t* base = raw_ring + (i % kStages) * C::kRawBytes;
      uint64_t* full = &bars[full0 + i % kStages];
      const int tt = tok_begin + i * kTok;
      if (!PAGED) {
        mbar_arrive_expect_tx(full, C::kRawBytes);
        tma_load_3d(base, map, full, 0, g, b * p.capacity + tt, pol);
      } else {
        const int nb = min(kBlocks, (tok_end - tt + kPageTokens - 1) / kPageTokens);
        const int32_t* tab = p.page_table + (size_t)b * p.max_blocks + tt / kPageTokens;
        int ids[kBlocks];
#pragma unroll
        for (int j = 0; j < kBlocks; ++j) ids[j] = j < nb ? __ldg(tab + j) : 0;
#pragma unroll
        for (int j = 0; j < kBlocks; ++j)
          if (j < nb && (ids[j] < 0 || ids[j] >= p.num_blocks)) {
            atomicOr(p.status, DEV_PAGE_ID);
            ids[j] = 0;   // keep the byte count; the result is flagged invalid
          }
        mbar_arrive_expect_tx(full, nb * kPageTokens * 128);
#pragma unroll
        for (int j = 0; j < kBlocks; ++j)
          if (j < nb) tma_load_3d(base + j * kPageTokens * 128, map, full, 0, g, ids[j] * kPageTokens, pol);
      }
    };
    int issued = 0;
    if (lane == 0) {
      prefetch_tmap(map);
      if (is_k) {
        mbar_arrive_expect_tx(&bars[T_Q], p.TT * p.G * D * 2);
#pragma unroll
        for (int hh = 0; hh < C::kHalves; ++hh)
          tma_load_4d(smem + C::kQOff + hh * C::kQHalfBytes, &tmQ, &bars[T_Q], hh * 64, g * p.G, t0, b, pol);
      }
      for (; issued < kStages && issued < n_tiles; ++issued) copy_tile(issued);
    }
    issued = __shfl_sync(0xffffffffu, issued, 0);
    bool ok = true;
    if (is_k) {
      // Q to f16 in place (same element size, same layout), then published to the MMA warp
      ok = tc_wait(&bars[T_Q], 0, abort_flag, p.status);
      if (ok) {
        for (int idx = lane; idx < C::kQBytes / 16; idx += 32) {
          uint4* q = reinterpret_cast<uint4*>(smem + C::kQOff) + idx;
          uint4 v = *q;
          v = make_uint4(bf16x2_to_f16x2(v.x), bf16x2_to_f16x2(v.y), bf16x2_to_f16x2(v.z), bf16x2_to_f16x2(v.w));
          *q = v;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[T_QC]);
      }
    }
    for (int i = 0; ok && i < n_tiles; ++i) {
      if (!tc_wait(&bars[full0 + i % kStages], (i / kStages) & 1, abort_flag, p.status)) break;
      if (i > 0 && !tc_wait(cempty, (i - 1) & 1, abort_flag, p.status)) break;
      convert_tile_e4m3<D>(raw_ring + (i % kStages) * C::kRawBytes, conv, lane, 0, conv_split ? kTok / 8 : kTok / 4);
      fence_proxy_async_smem();       // the converted tile is read by the MMAs (async proxy)
      __syncwarp();
      // the helper finishes tile i before the MMA of tile i can release the converted
      // tile, so its barrier is never more than one phase ahead of this wait
      if (conv_split && !tc_wait(&bars[is_k ? T_KHDONE : T_VHDONE], i & 1, abort_flag, p.status)) break;
      if (lane == 0) {
        mbar_arrive(cfull);
        if (i + kStages < n_tiles) {   // the raw stage just read takes the tile kStages ahead
          copy_tile(i + kStages);
          ++issued;
        }
      }
      issued = __shfl_sync(0xffffffffu, issued, 0);
    }
    // no copy may still be landing in shared memory when the CTA exits
    if (lane == 0) {
      if (is_k) mbar_wait(&bars[T_Q], 0);
      for (int i = max(0, issued - kStages); i < issued; ++i) mbar_wait(&bars[full0 + i % kStages], (i / kStages) & 1);
    }
  } else if (conv_split && (warp == 3 || warp == 2)) {
    // ------------------------------------------------ FP8 conversion helpers (R <= 64)
    // Rows kTok/2 .. kTok - 1 of every raw tile: the same waits as the producer's
    // conversion (raw tile landed, previous converted tile released by the MMA), then
    // one arrival per tile.  The producer refills the raw stage only after that arrival.
    const bool is_k = warp == 3;
    const uint8_t* raw_ring = smem + (is_k ? C::kRawKOff : C::kRawVOff);
    uint8_t* conv = smem + (is_k ? C::kKOff : C::kVOff);
    const int full0 = is_k ? T_KFULL : T_VFULL;
    uint64_t* cempty = &bars[is_k ? T_KCEMPTY : T_VCEMPTY];
    uint64_t* hdone = &bars[is_k ? T_KHDONE : T_VHDONE];
    for (int i = 0; i < n_tiles; ++i) {
      if (!tc_wait(&bars[full0 + i % kStages], (i / kStages) & 1, abort_flag, p.status)) break;
      if (i > 0 && !tc_wait(cempty, (i - 1) & 1, abort_flag, p.status)) break;
      convert_tile_e4m3<D>(raw_ring + (i % kStages) * C::kRawBytes, conv, lane, kTok / 8, kTok / 4);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(hdone);
    }
  } else if (!FP8 && (warp == 4 || warp == 6)) {
    // ------------------------------------------------------------- TMA producers
    if (lane == 0) {
      const bool is_k = warp == 4;
      const CUtensorMap* map = is_k ? &tmK : &tmV;
      prefetch_tmap(map);
      const uint64_t pol = policy_evict_first();
      if (is_k) {
        // Q rows (t, head g*G + hh) for t0 <= t < t0 + TT, hh < G: one box {64, G, TT, 1} per half
        // of d (the full box is counted, also where tokens >= T are zero-filled)
        mbar_arrive_expect_tx(&bars[T_Q], p.TT * p.G * D * 2);
#pragma unroll
        for (int hh = 0; hh < C::kHalves; ++hh)
          tma_load_4d(smem + C::kQOff + hh * C::kQHalfBytes, &tmQ, &bars[T_Q], hh * 64, g * p.G, t0, b, pol);
      }
      uint8_t* ring = smem + (is_k ? C::kKOff : C::kVOff);
      const int full0 = is_k ? T_KFULL : T_VFULL, empty0 = is_k ? T_KEMPTY : T_VEMPTY;
      int last[kStages];
#pragma unroll
      for (int s = 0; s < kStages; ++s) last[s] = -1;
      constexpr int kBlocks = kTok / kPageTokens;
      // physical blocks of one tile, read together (the copies' memory clobbers
      // would otherwise serialise one table read per block)
      auto read_ids = [&](int i, int (&ids)[kBlocks]) {
        const int tt = tok_begin + i * kTok;
        const int nb = min(kBlocks, (tok_end - tt + kPageTokens - 1) / kPageTokens);
        const int32_t* tab = p.page_table + (size_t)b * p.max_blocks + tt / kPageTokens;
#pragma unroll
        for (int j = 0; j < kBlocks; ++j) ids[j] = j < nb ? __ldg(tab + j) : 0;
#pragma unroll
        for (int j = 0; j < kBlocks; ++j)
          if (j < nb && (ids[j] < 0 || ids[j] >= p.num_blocks)) {
            atomicOr(p.status, DEV_PAGE_ID);
            ids[j] = 0;   // keep the byte count; the result is flagged invalid
          }
        return nb;
      };
      int ids[kBlocks] = {};
      int nb = PAGED ? read_ids(0, ids) : 0;
      for (int i = 0; i < n_tiles; ++i) {
        const int ks = i % kStages;
        if (i >= kStages && !tc_wait(&bars[empty0 + ks], ((i / kStages) - 1) & 1, abort_flag, p.status)) break;
        last[ks] = i;
        uint8_t* base = ring + ks * C::kTileBytes;
        uint64_t* full = &bars[full0 + ks];
        const int tt = tok_begin + i * kTok;
        if (!PAGED) {
          mbar_arrive_expect_tx(full, C::kTileBytes);
#pragma unroll
          for (int hh = 0; hh < C::kHalves; ++hh)
            tma_load_3d(base + hh * C::kHalfBytes, map, full, hh * 64, g, b * p.capacity + tt, pol);
        } else {
          mbar_arrive_expect_tx(full, nb * C::kHalves * kPageTokens * 128);
#pragma unroll
          for (int j = 0; j < kBlocks; ++j) {
            if (j >= nb) break;
#pragma unroll
            for (int hh = 0; hh < C::kHalves; ++hh)
              tma_load_3d(base + hh * C::kHalfBytes + j * kPageTokens * 128, map, full, hh * 64, g,
                          ids[j] * kPageTokens, pol);
          }
          if (i + 1 < n_tiles) nb = read_ids(i + 1, ids);
        }
      }
      // no copy may still be landing in shared memory when the CTA exits
      if (is_k) mbar_wait(&bars[T_Q], 0);
      for (int ks = 0; ks < kStages; ++ks)
        if (last[ks] >= 0) mbar_wait(&bars[full0 + ks], (last[ks] / kStages) & 1);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------- MMA issuer
    // The whole warp runs the loop (warp-uniform operands, descriptors as precomputed
    // low words plus compile-time offsets); one elected lane issues and commits.
    const uint32_t leader = elect_one();
    constexpr uint32_t idS = FP8 ? idesc_f16(kRows, kTok, 0, 0) : idesc_bf16(kRows, kTok, 0, 0);
    constexpr uint32_t idO = FP8 ? idesc_f16(kRows, D, 0, 1) : idesc_bf16(kRows, D, 0, 1);
    const uint32_t sbase = smem_u32(smem);
    const uint32_t q_lo = desc_lo(sbase + C::kQOff, 16);
    // the K / V operand tile of key tile i: ring stage i % kStages (bf16), the one converted tile (FP8)
    auto k_full = [&](int i) { return FP8 ? &bars[T_KCFULL] : &bars[T_KFULL + i % kStages]; };
    auto v_full = [&](int i) { return FP8 ? &bars[T_VCFULL] : &bars[T_VFULL + i % kStages]; };
    auto full_parity = [&](int i) -> uint32_t { return FP8 ? (i & 1) : ((i / kStages) & 1); };
    auto issue_s = [&](int i) {
      const int sb = i & 1, ks = FP8 ? 0 : i % kStages;   // S buffer, K operand stage
      const uint32_t k_lo = desc_lo(sbase + C::kKOff + ks * C::kTileBytes, 16);
      const uint32_t d = tmem + sb * C::kSCols;
      tc_mma_ss_lo<0>(leader, d, q_lo, k_lo, idS);
#pragma unroll
      for (int kk = 1; kk < D / 16; ++kk) {
        const uint32_t q_off = ((kk >> 2) * C::kQHalfBytes + (kk & 3) * 32) >> 4;
        const uint32_t k_off = ((kk >> 2) * C::kHalfBytes + (kk & 3) * 32) >> 4;
        tc_mma_ss_lo<1>(leader, d, q_lo + q_off, k_lo + k_off, idS);
      }
      tc_commit_if(leader, &bars[T_SFULL + sb]);
      tc_commit_if(leader, FP8 ? &bars[T_KCEMPTY] : &bars[T_KEMPTY + ks]);     // K_i is read only by S_i
    };
    bool ok = tc_wait(&bars[FP8 ? T_QC : T_Q], 0, abort_flag, p.status) &&
              tc_wait(k_full(0), 0, abort_flag, p.status);
    if (ok) {
      tc_fence_after();
      issue_s(0);
    }
    for (int i = 0; ok && i < n_tiles; ++i) {
      const int sb = i & 1, ks = i % kStages;
      if (i + 1 < n_tiles) {
        ok = tc_wait(k_full(i + 1), full_parity(i + 1), abort_flag, p.status);
        if (!ok) break;
        tc_fence_after();
        issue_s(i + 1);   // its S buffer last held P_{i-1}, whose PV was issued before
      }
      ok = tc_wait(&bars[T_PFULL + sb], (i >> 1) & 1, abort_flag, p.status) &&
           tc_wait(v_full(i), full_parity(i), abort_flag, p.status);
      if (!ok) break;
      // keys at or past this CTA's end may hold anything (past L: any bytes; past a row
      // tile's last visible key in a paged cache: blocks never loaded, stale shared
      // memory), even NaN: zero their V rows, which the PV MMA would otherwise multiply
      // by p = 0.  This warp consumes the V tiles' phases in order, so the wait above
      // is for exactly this tile's V (a softmax warp's parity wait could be satisfied
      // by the tile two phases back while this one is still being written).
      const int valid = tok_end - (tok_begin + i * kTok);
      if (valid < kTok) {
        uint8_t* vst = smem + C::kVOff + (FP8 ? 0 : ks) * C::kTileBytes;
        for (int idx = max(valid, 0) * 8 + lane; idx < kTok * 8; idx += 32)
#pragma unroll
          for (int hh = 0; hh < C::kHalves; ++hh)
            *reinterpret_cast<uint4*>(vst + hh * C::kHalfBytes + idx * 16) = make_uint4(0, 0, 0, 0);
        fence_proxy_async_smem();
        __syncwarp();
      }
      tc_fence_after();
      const uint32_t v_lo = desc_lo(sbase + C::kVOff + (FP8 ? 0 : ks) * C::kTileBytes, C::kHalfBytes);
      const uint32_t d = tmem + C::kOCol, pa = tmem + sb * C::kSCols;
      if (i == 0) tc_mma_ts_lo<0>(leader, d, pa, v_lo, idO);
      else tc_mma_ts_lo<1>(leader, d, pa, v_lo, idO);
#pragma unroll
      for (int kk = 1; kk < kTok / 16; ++kk)
        tc_mma_ts_lo<1>(leader, d, pa + kk * 8, v_lo + ((kk * 16 * 128) >> 4), idO);
      tc_commit_if(leader, &bars[T_ODONE]);
      tc_commit_if(leader, FP8 ? &bars[T_VCEMPTY] : &bars[T_VEMPTY + ks]);
    }
    // also on a failed wait, so that the epilogue does not wait in vain (abort_flag marks the result)
    tc_commit_if(leader, &bars[T_OFINAL]);
  } else if (warp < active_warps) {
    // ------------------------------------------------------------- softmax warps
    const int row = warp * 32 + lane;
    const bool live = row < tile_rows;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    const int t = live ? t0 + row / p.G : 0;
    const int end = p.causal ? L - p.T + t + 1 : L;       // first invisible key of this row
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int i = 0; i < n_tiles; ++i) {
      const int st = i & 1;
      if (!tc_wait(&bars[T_SFULL + st], (i >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
      tc_fence_after();
      const uint32_t s_addr = lane_base + st * C::kSCols;
      float s[kTok];
#pragma unroll
      for (int cc = 0; cc < kTok; cc += 32) {
        uint32_t r[32];
        tmem_ld32(s_addr + cc, r);
#pragma unroll
        for (int e = 0; e < 32; ++e) s[cc + e] = __uint_as_float(r[e]);
      }
      tc_wait_ld();
      const int key0 = tok_begin + i * kTok;
      const int lim = live ? end - key0 : 0;              // visible keys of this row in the tile: [0, lim)
      if (lim < kTok) {
#pragma unroll
        for (int cc = 0; cc < kTok; ++cc) s[cc] = (cc < lim) ? s[cc] : -INFINITY;
      }
      float mx8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx8[k] = max3f(s[k], s[k + 8], s[k + 16]);
#pragma unroll
      for (int cc = 24; cc + 8 < kTok; cc += 16)
#pragma unroll
        for (int k = 0; k < 8; ++k) mx8[k] = max3f(mx8[k], s[cc + k], s[cc + 8 + k]);
#pragma unroll
      for (int k = 0; k < 8; ++k) mx8[k] = fmaxf(mx8[k], s[kTok - 8 + k]);
      float mx = max3f(max3f(mx8[0], mx8[1], mx8[2]), max3f(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
      mx *= scale_log2;
      const bool warp_raise = __any_sync(0xffffffffu, mx > m + 8.f);
      float alpha = 1.f;
      if (warp_raise) {
        const float m_new = fmaxf(m, mx);
        alpha = ex2(m - ((m_new == -INFINITY) ? 0.f : m_new));   // 0 while m is -inf
        m = m_new;
      }
      const float neg_mu = (m == -INFINITY) ? 0.f : -m;
      float ls4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int cc = 0; cc < kTok; cc += 16) {
        uint32_t pk[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          const float p0 = ex2(fmaf(s[cc + e], scale_log2, neg_mu));
          const float p1 = ex2(fmaf(s[cc + e + 1], scale_log2, neg_mu));
          ls4[(e >> 1) & 3] += p0 + p1;
          pk[e / 2] = FP8 ? pack_f16x2(p0, p1) : pack_bf16x2(p0, p1);
        }
        tmem_st8(s_addr + cc / 2, pk);      // P row over the consumed S columns
      }
      l = l * alpha + ((ls4[0] + ls4[1]) + (ls4[2] + ls4[3]));
      if (warp_raise && i > 0) {
        // PV_{i-1} must be done before O is rescaled (S_i was issued before it)
        if (!tc_wait(&bars[T_ODONE], (i - 1) & 1, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < D; cc += 32) {
          uint32_t r[32];
          tmem_ld32(lane_base + C::kOCol + cc, r);
          tc_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tmem_st32(lane_base + C::kOCol + cc, r);
        }
      }
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[T_PFULL + st]);
    }

    // ---------------------------------------------------------- epilogue
    launch_dependents();   // the combine kernel may start launching (it waits for this grid)
    if (ok && tc_wait(&bars[T_OFINAL], 0, abort_flag, p.status) && !*abort_flag) {
      tc_fence_after();
      float* out = p.part_o + (row0 + row) * D;
      const float inv_l = l > 0.f ? v_mul / l : 0.f;
#pragma unroll
      for (int cc = 0; cc < D; cc += 32) {
        uint32_t r[32];
        tmem_ld32(lane_base + C::kOCol + cc, r);
        tc_wait_ld();
        if (live) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(out + cc + e) =
                make_float4(__uint_as_float(r[e]) * inv_l, __uint_as_float(r[e + 1]) * inv_l,
                            __uint_as_float(r[e + 2]) * inv_l, __uint_as_float(r[e + 3]) * inv_l);
        }
      }
      if (live) p.part_lse[row0 + row] = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
    } else if (live) {
      p.part_lse[row0 + row] = NAN;   // a wait gave up
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag && warp == 5) {
    // the lane that issued the MMAs commits, so the drain covers them
    const uint32_t leader = elect_one();
    tc_commit_if(leader, &bars[T_DRAIN]);
    mbar_wait(&bars[T_DRAIN], 0);
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int D, bool PAGED, bool FP8>
cudaError_t run_tc(const DecodeLaunch& a, const CUtensorMap& tk, const CUtensorMap& tv, cudaStream_t stream) {
  using C = TcCfg<D, FP8>;
  const int G = a.Hq / a.Hkv;
  const int TT = decode_tc_tile_tokens(a.T, G);
  const int row_tiles = (a.T + TT - 1) / TT;
  CUtensorMap tq;
  // q [B, T, Hq, d] as {d, Hq, T, B}; one box covers the G heads of a KV head for TT tokens
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)a.Hq, (cuuint64_t)a.T, (cuuint64_t)a.B};
  cuuint64_t str[3] = {(cuuint64_t)D * 2, (cuuint64_t)a.Hq * D * 2, (cuuint64_t)a.T * a.Hq * D * 2};
  cuuint32_t box[4] = {64, (cuuint32_t)G, (cuuint32_t)TT, 1};
  if (encode_tmap_nd(&tq, a.q, 4, dims, str, box)) return cudaErrorInvalidValue;
  TcParams p;
  p.k_scale = a.k_scale;
  p.v_scale = a.v_scale;
  p.seqlens = a.seqlens;
  p.page_table = a.page_table;
  p.part_o = a.part_o;
  p.part_lse = a.part_lse;
  p.status = a.status;
  p.T = a.T;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.G = G;
  p.R = G * a.T;
  p.TT = TT;
  p.chunk = a.chunk;
  p.max_chunks = a.max_chunks;
  p.capacity = a.capacity;
  p.max_blocks = a.max_blocks;
  p.num_blocks = a.num_blocks;
  p.max_seqlen = a.max_seqlen;
  p.scale_log2 = a.scale * kLog2e;
  p.causal = a.causal;
  p.balanced = a.balanced;
  p.n_chunks = a.n_chunks;
  p.B = a.B;
  p.plan = a.plan;
  if (a.balanced && (a.B > kBalancedMaxB || row_tiles != 1 || a.n_chunks < a.B)) return cudaErrorInvalidValue;
  auto kern = decode_tc_kernel<D, PAGED, FP8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  if ((long long)a.max_chunks * row_tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
  dim3 grid(a.max_chunks * row_tiles, a.Hkv, a.B);
  if (a.balanced) grid = dim3((unsigned)a.n_chunks * a.Hkv);
  kern<<<grid, tc_threads<FP8>(), C::kSmemBytes, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_tc(const DecodeLaunch& a, const CUtensorMap& tk, const CUtensorMap& tv,
                             cudaStream_t stream) {
  const bool paged = a.page_table != nullptr;
  if (a.fp8) {   // api.cu admits FP8 caches with d = 128 only
    if (a.d != 128) return cudaErrorInvalidValue;
    return paged ? run_tc<128, true, true>(a, tk, tv, stream) : run_tc<128, false, true>(a, tk, tv, stream);
  }
  if (a.d == 128)
    return paged ? run_tc<128, true, false>(a, tk, tv, stream) : run_tc<128, false, false>(a, tk, tv, stream);
  return paged ? run_tc<64, true, false>(a, tk, tv, stream) : run_tc<64, false, false>(a, tk, tv, stream);
}

}  // namespace kvattn
