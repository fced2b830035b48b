// Prefill attention on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Persistent: one CTA per SM takes work items from a queue, heaviest causal
// query blocks first (its first item is its block index; every further item is
// a ticket from a global counter, so a CTA that finishes early takes more
// work instead of waiting on a fixed share).  A work item is two 128-row query tiles (A: rows 256*qb .. +127,
// B: the next 128) of one (batch, query head); both tiles share every K/V tile
// loaded for the item.  Warp roles (12 warps, three warpgroups):
//   warps 0-3  softmax of tile A, warps 4-7 softmax of tile B: thread i of a
//              group owns query row i, which is TMEM lane i of its S and O;
//   warps 8,10 TMA producers: warp 8 loads Q_A and Q_B per item (the next
//              item's Q is prefetched into L2 early) and the K tiles, warp 10
//              the V tiles, each through its own ring (2 stages at d = 128, 4
//              at d = 64) that runs on across items; K is released after the
//              second S MMA reading it, V after the second PV;
//   warp 9     MMA issuer: the whole warp runs the loop, one elected lane
//              issues (operands stay warp-uniform, so each MMA costs the
//              issuing warp only a few instructions on a sub-partition it
//              shares with two busy softmax warps);
//   warp 11    completes the producer warpgroup for the register split.
// TMEM (512 columns): S_A | S_B | O_A | O_B.  Each softmax group reads its S row,
// turns it into bf16 probabilities P and writes P back over the first half of
// the same S columns, in two halves of 64 keys: the PV MMA of the first half
// (reading P straight from TMEM as its A operand) is issued while the group
// computes the second.
// The MMA issue order  PV_A(j), S_A(j+1), PV_B(j), S_B(j+1), PV_A(j+1), ...
// gives each softmax group the time of two MMAs to produce its next P.  Because
// MMAs complete in issue order, "S_X(j) complete" also means "PV_X(j-1)
// complete", so a softmax group may rescale O_X as soon as it sees S_X(j).  At
// an item boundary the next item's first S MMAs run while the softmax warps
// write out the previous item's O; the first PV of the new item waits until
// that O has been read (O_FREE).
//
// Prefill against an existing cache (KV = contiguous or paged cache): the Nq
// new queries of sequence b are its LAST Nq positions, so query row i sees keys
// j <= L_b - Nq + i, where L_b = seqlens[b] counts the cached prefix plus the
// Nq new keys (already appended).  Each item reads L_b, limits its K/V tiles to
// the last key its rows see, and the softmax group that consumes a tile zeroes
// the V rows at or past L_b in shared memory (cache rows there may hold any
// bytes; paged blocks there are never loaded).  Paged caches load each 128-key
// tile as eight 16-row boxes, one per physical block of the page table.
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
// specialisation with asynchronous TMA); "Effizienz", "Der wichtige Maskenfehler
// beim Cache" (queries aligned to the end of the key sequence) and the lesson's
// "用它" (prefix caching) for the cached form.
#include <cuda_bf16.h>
#include <math.h>

#include <atomic>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace kvattn {

// Work-queue counters of the prefill kernel: slot i holds (next ticket, CTAs
// done) of one launch; launches take slots in turn, and each launch's last CTA
// zeroes its slot, so launches in flight at the same time (up to kQueueSlots)
// never share counters.  Zero at load time.
constexpr int kQueueSlots = 1024;
__device__ unsigned g_prefill_queue[2 * kQueueSlots];

namespace {

constexpr int kBM = 128;          // query rows per tile (two tiles per CTA)
constexpr int kBN = 128;          // keys per K/V tile
constexpr int kThreads = 384;     // 8 softmax warps + 2 TMA warps + MMA warp + 1 idle warp (a full warpgroup)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;   // log2 of the largest allowed p
constexpr int kMaxStages = 4;     // K or V ring stages (barrier slots)
constexpr int kItemSlots = 4;     // work items published ahead (see item_slot)

// K/V ring depth.  d = 128: two stages (a third K stage measured no faster: the copies
// are issued about one KV step ahead of their use).  d = 64: the tiles are half the
// size and a KV step is shorter, and four stages measured about 3 % faster on the
// GPT-2-sized causal prefill with K/V resident in L2.
template <int D>
struct PrefillCfg {
  static constexpr int kHalves = D / 64;
  static constexpr int kKStages = D == 64 ? 4 : 2;
  static constexpr int kVStages = D == 64 ? 4 : 2;
  static_assert(kKStages <= kMaxStages && kVStages <= kMaxStages, "ring stages");
  static constexpr int kTileBytes = kBN * D * 2;          // one Q, K or V tile
  static constexpr int kHalfBytes = kBN * 128;            // 128 rows x 128 B
  static constexpr int kQOff = 0;                         // Q_A, Q_B
  static constexpr int kKOff = kQOff + 2 * kTileBytes;          // K stages 0..kKStages-1
  static constexpr int kVOff = kKOff + kKStages * kTileBytes;   // V stages 0..kVStages-1
  static constexpr int kBarOff = kVOff + kVStages * kTileBytes;
  static constexpr int kOrderOff = kBarOff + 256;        // cached forms: sequences by length, longest first
  static constexpr int kMaxOrdered = 256;
  static constexpr int kUsed = kOrderOff + kMaxOrdered * 4;
  // one CTA per SM: it owns all 512 TMEM columns
  static constexpr int kSmemBytes = (kUsed + 1024) > 120 * 1024 ? (kUsed + 1024) : 120 * 1024;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory of one CTA");
  static constexpr int kTmemCols = 512;
  // TMEM columns: S of tile t at 128*t, O of tile t at 256 + D*t
  __host__ __device__ static constexpr int s_col(int t) { return 128 * t; }
  __host__ __device__ static constexpr int o_col(int t) { return 256 + D * t; }
};

enum Bar {
  B_QFULL = 0,
  B_QEMPTY = 1,                     // all MMAs of an item done and every softmax warp and the V
                                    // producer have read the item (10 arrivals): its Q may be replaced
  B_KFULL = 2,                      // +K stage
  B_KEMPTY = B_KFULL + kMaxStages,  // +K stage: both S MMAs reading this K stage are done
  B_VFULL = B_KEMPTY + kMaxStages,  // +V stage
  B_VEMPTY = B_VFULL + kMaxStages,  // +V stage: both PV MMAs reading this V stage are done
  B_SFULL = B_VEMPTY + kMaxStages,  // +tile
  B_PHALF = B_SFULL + 2,            // +tile: P of the tile's first 64 keys is in TMEM (and O is rescaled)
  B_PFULL = B_PHALF + 2,            // +tile: P of all 128 keys is in TMEM
  B_ODONE = B_PFULL + 2,            // +tile: last PV of an item done
  B_OFREE = B_ODONE + 2,            // +tile: the softmax group has read O out
  B_DRAIN = B_OFREE + 2,            // only used when a bounded wait gave up
  B_COUNT = B_DRAIN + 1
};
static_assert(B_COUNT * 8 + 8 + 4 * kItemSlots <= 256, "barrier block");

// Where K and V come from.
// KV_DENSE_GROUPED: the dense form with its items in the cached forms' order.
enum KvSource { KV_DENSE = 0, KV_CACHE = 1, KV_PAGED = 2, KV_DENSE_GROUPED = 3 };

// Register split (setmaxnreg): 384 threads launch with 168 registers each; the producer
// warpgroup (two TMA warps, the MMA warp and one more) gives back down to regs_io() so
// each softmax thread can hold its 128 scores and the exponential temporaries.  Chosen
// per form by ptxas's spill report: the dense d = 128 softmax needs 216 registers, the
// other forms spill less with 208 and 88 for the producers (the cached forms' producers
// also track the sequence lengths and page-table entries).
template <int D, int KV>
constexpr int regs_softmax() { return D == 128 && KV == KV_DENSE ? 216 : 208; }
template <int D, int KV>
constexpr int regs_io() { return D == 128 && KV == KV_DENSE ? 72 : 88; }
static_assert(2 * 128 * regs_softmax<128, KV_DENSE>() + 128 * regs_io<128, KV_DENSE>() <= 168 * kThreads,
              "register split exceeds the launch");
static_assert(2 * 128 * regs_softmax<64, KV_PAGED>() + 128 * regs_io<64, KV_PAGED>() <= 168 * kThreads,
              "register split exceeds the launch");
template <int KV>
constexpr bool kDenseKv = KV == KV_DENSE || KV == KV_DENSE_GROUPED;

// K+V bytes of one (sequence, K/V head) of a dense prefill from which its items are
// grouped by K/V head.  Measured on B200 (4 x 32 x 8 heads, d = 128): grouped is
// 9 % slower at 4096 causal keys (16 x 4096 too, by 1 %), where the heaviest-first
// order balances the short items best, and 1-3 % faster from 8192 keys on (causal
// 16384 and 32768, non-causal 8192), where all heads' K/V no longer stay in L2.
constexpr double kDenseKvHeadBytes = 4.0 * 1024 * 1024;

struct PrefillParams {
  void* o;
  float* lse;
  unsigned* status;
  unsigned* next_item;   // work queue: tickets handed out after the first gridDim.x items
  unsigned* done_ctas;   // the last CTA to finish resets both counters for the next launch
  int B, N, Hq, Hkv, G, n_qblocks, n_ktiles, n_items;   // N: queries per sequence (Nq)
  float scale_log2;
  int causal, o_bf16;
  // cached forms only
  const int32_t* seqlens;      // [B] keys per sequence, including the N new ones
  const int32_t* page_table;   // [B, max_blocks] (paged)
  int max_keys;                // cache capacity in tokens (contiguous) or max_blocks * 16 (paged)
  int max_blocks, num_blocks;
};

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                              unsigned* status) {
  if (*abort_flag) return false;
  if (mbar_wait(bar, parity)) return true;
  atomicOr(status, DEV_TIMEOUT);
  *abort_flag = 1;
  return false;
}

struct Item {
  int qb, h, b, n_kv0, n_load;   // n_kv0: K/V tiles of query tile A; n_load: of tile B (>= n_kv0)
  int L, off;                    // keys of the sequence; query row i sees keys j <= off + i (causal)
  bool bad;                      // invalid length (cached forms): the rows are written as NaN
};

// Work item w.  Dense with short sequences: heaviest causal query blocks first, then
// consecutive heads (the query heads of one K/V head are adjacent, so its K/V tiles
// are reused from L2).  Cached forms, where sequences differ in length, and dense
// long sequences (KV_DENSE_GROUPED): sequences longest
// first (`order`, or index order when the batch is too large to rank), then K/V
// head, then query blocks heaviest first, then the heads of that K/V head --
// roughly longest-processing-time first, and every reader of one K/V range runs
// at about the same time, so that range is read from L2.
template <int KV>
__device__ __forceinline__ Item item_of(int w, const PrefillParams& p, const int* order) {
  Item it;
  if constexpr (KV == KV_DENSE) {
    const int per = p.Hq * p.B;
    it.qb = p.n_qblocks - 1 - w / per;
    const int r = w - (w / per) * per;
    it.h = r % p.Hq;
    it.b = r / p.Hq;
  } else {
    const int per_g = p.n_qblocks * p.G;        // items of one (sequence, K/V head)
    const int per_b = p.Hkv * per_g;
    const int r = w / per_b, rem = w - r * per_b;
    it.b = order ? order[r] : r;
    const int kvh = rem / per_g, rem2 = rem - kvh * per_g;
    it.qb = p.n_qblocks - 1 - rem2 / p.G;
    it.h = kvh * p.G + rem2 % p.G;
  }
  if constexpr (kDenseKv<KV>) {
    it.L = p.N;
    it.off = 0;
    it.bad = false;
    it.n_kv0 = p.causal ? min(2 * it.qb + 1, p.n_ktiles) : p.n_ktiles;
    it.n_load = p.causal ? min(2 * it.qb + 2, p.n_ktiles) : p.n_ktiles;
  } else {
    int L = __ldg(p.seqlens + it.b);
    it.bad = L < p.N || L > p.max_keys;
    if (it.bad) L = p.N;               // a safe stand-in; the host checked p.N <= p.max_keys
    it.L = L;
    it.off = L - p.N;
    const int nt = (L + kBN - 1) / kBN;
    it.n_kv0 = p.causal ? min((it.off + 2 * it.qb * kBM + kBM + kBN - 1) / kBN, nt) : nt;
    it.n_load = p.causal ? min((it.off + 2 * it.qb * kBM + 2 * kBM + kBN - 1) / kBN, nt) : nt;
  }
  return it;
}

// 2^x for two values on the FMA pipe (no SFU): x = n + f with n = round(x) (the
// "magic number" 1.5 * 2^23 rounds to the nearest integer), 2^f on [-1/2, 1/2] by a
// cubic fitted for minimax relative error (7.5e-5, far below the 2^-9 of the bf16 P it
// feeds), and 2^n added to the exponent field.  x is clamped to [-126, +inf): scores
// reach here relative to the running maximum (x <= 8), and below -126 the true value
// (< 1.2e-38) is replaced by a denormal of about that size.
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
  constexpr float kMagic = 12582912.f;
  constexpr float kC0 = 0.99992807f, kC1 = 0.69326097f, kC2 = 0.24261113f, kC3 = 0.055171669f;
  x.x = fmaxf(x.x, -126.f);
  x.y = fmaxf(x.y, -126.f);
  const float2 t = __fadd2_rn(x, make_float2(kMagic, kMagic));            // low bits hold n
  const float2 n = __fadd2_rn(t, make_float2(-kMagic, -kMagic));
  const float2 f = __ffma2_rn(n, make_float2(-1.f, -1.f), x);             // x - n, exact
  float2 q = __ffma2_rn(f, make_float2(kC3, kC3), make_float2(kC2, kC2));
  q = __ffma2_rn(q, f, make_float2(kC1, kC1));
  q = __ffma2_rn(q, f, make_float2(kC0, kC0));
  return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(t.y) << 23)));
}

// Which pairs of each 16-key group take the FMA-pipe exponential (bit i: keys 2i, 2i+1).
// The SFU issues 16 exponentials per clock per SM, so a 128 x 128 score tile alone costs
// as much SFU time as its two MMAs at d = 128, and twice as much at d = 64.  Measured on
// B200: at d = 128 the extra FMA-pipe instructions cost more than the SFU time they
// save (the softmax warps share their sub-partitions' issue slots with the MMA warp),
// so every exponential stays on the SFU; at d = 64, three pairs in eight (37.5 %) on the
// FMA pipe gained 3-4 % on the GPT-2-sized prefill.
template <int D>
constexpr unsigned exp_fma_pairs() { return D == 64 ? 0x92u : 0u; }

// Exponentials of keys 64*HALF .. 64*HALF+63 of one row: p = 2^(s*sc - m) (nm = -m), the
// pair sums added to sum2, and bf16 P stored to TMEM at taddr (two keys per column).
// FMA: use the FMA-pipe exponential on the pairs kExpFmaPairs selects (rows without
// masked keys only; no pair when it is 0).
template <int HALF, bool FMA, unsigned kExpFmaPairs>
__device__ __forceinline__ void exp_store_half(const float (&s)[kBN], float2 sc, float2 nm, float2 (&sum2)[4],
                                               uint32_t taddr) {
  // one TMEM store per 16 keys (measured faster than stores of 32 or 64 keys)
#pragma unroll
  for (int c = HALF * (kBN / 2); c < (HALF + 1) * (kBN / 2); c += 16) {
    uint32_t pk[8];
#pragma unroll
    for (int e = 0; e < 16; e += 2) {
      const float2 x = __ffma2_rn(make_float2(s[c + e], s[c + e + 1]), sc, nm);
      float2 pr;
      if (FMA && ((kExpFmaPairs >> (e / 2)) & 1u)) pr = exp2_fma2(x);
      else pr = make_float2(ex2(x.x), ex2(x.y));
      sum2[(e >> 1) & 3] = __fadd2_rn(sum2[(e >> 1) & 3], pr);
      pk[e / 2] = pack_bf16x2(pr.x, pr.y);
    }
    tmem_st8(taddr + c / 2, pk);
  }
}

template <int D, int KV>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  using C = PrefillCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // work item of the CTA's it-th item in slot it % kItemSlots, published by the producer
  // before that item's Q copies complete B_QFULL phase it; -1 = no more work.  The slot
  // is written again for item it + kItemSlots only after B_QEMPTY of item
  // it + kItemSlots - 1, which every softmax warp and the V producer reach after
  // reading item it.
  volatile int* item_slot = reinterpret_cast<volatile int*>(tmem_slot + 2);
  int* order_smem = reinterpret_cast<int*>(smem + C::kOrderOff);
  const int* order = (!kDenseKv<KV> && p.B <= C::kMaxOrdered) ? order_smem : nullptr;
  if (order) {
    // rank of each sequence by length, longest first (ties by index)
    for (int bb = threadIdx.x; bb < p.B; bb += blockDim.x) {
      const int lb = __ldg(p.seqlens + bb);
      int rank = 0;
      for (int o = 0; o < p.B; ++o) {
        const int lo = __ldg(p.seqlens + o);
        rank += (lo > lb) || (lo == lb && o < bb);
      }
      order_smem[rank] = bb;
    }
  }

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&bars[B_QFULL], 1);
    // the MMA warp's commit and one arrival per softmax warp and from the V producer:
    // B_QFULL then never runs two phases ahead of a warp that reads the item (a parity
    // wait would miss the phase it wants)
    mbar_init(&bars[B_QEMPTY], 1 + 8 + 1);
    for (int s = 0; s < C::kKStages; ++s) {
      mbar_init(&bars[B_KFULL + s], 1);
      mbar_init(&bars[B_KEMPTY + s], 1);
    }
    for (int s = 0; s < C::kVStages; ++s) {
      mbar_init(&bars[B_VFULL + s], 1);
      mbar_init(&bars[B_VEMPTY + s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[B_SFULL + s], 1);
      mbar_init(&bars[B_PHALF + s], 4);
      mbar_init(&bars[B_PFULL + s], 4);
      mbar_init(&bars[B_ODONE + s], 1);
      mbar_init(&bars[B_OFREE + s], 4);
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
  if (warp >= 8) {
  reg_dealloc<regs_io<D, KV>()>();
  if (warp == 8 || warp == 10) {
    // ------------------------------------------------------------- TMA producers
    // Warp 8 loads Q per item and the K ring, warp 10 the V ring.  Each ring runs on
    // across items, so a K copy never waits for a V stage that the PV MMAs still read.
    // Paged caches: lane jb < 8 of the warp reads page-table entry jb of a tile (one tile
    // ahead) and copies that physical block, so the eight blocks of a tile are handled in
    // parallel instead of one after another by a single thread.
    const bool is_k = warp == 8;
    const CUtensorMap* map = is_k ? &tmK : &tmV;
    const int stages = is_k ? C::kKStages : C::kVStages;
    const int full0 = is_k ? B_KFULL : B_VFULL, empty0 = is_k ? B_KEMPTY : B_VEMPTY;
    uint8_t* const ring = smem + (is_k ? C::kKOff : C::kVOff);
    if (lane == 0) {
      prefetch_tmap(map);
      if (is_k) prefetch_tmap(&tmQ);
    }
    const uint64_t keep = policy_evict_last();    // K/V tiles are re-read by other query blocks and heads
    const uint64_t once = policy_evict_first();
    constexpr int kBlocks = kBN / kPageTokens;
    int g = 0, it = 0, q_loaded = 0;              // tiles loaded, items started, Q loads issued
    int last[kMaxStages];                         // last tile whose copy was issued per stage
#pragma unroll
    for (int i = 0; i < kMaxStages; ++i) last[i] = -1;
    bool ok = true, clean_end = false;
    for (int w = blockIdx.x;; ++it) {
      Item itm;
      int w_next = 0;
      if (is_k) {
        // Q of the previous item no longer read (this also means its copy landed), and
        // that item read by every softmax warp and by the V producer
        if (it > 0 && !wait_or_abort(&bars[B_QEMPTY], (it - 1) & 1, abort_flag, p.status)) break;
        if (w >= p.n_items) {
          // no more work: complete B_QFULL phase `it` without a copy
          if (lane == 0) {
            item_slot[it % kItemSlots] = -1;
            mbar_arrive(&bars[B_QFULL]);
          }
          clean_end = true;
          break;
        }
        if (lane == 0) item_slot[it % kItemSlots] = w;
        itm = item_of<KV>(w, p, order);
        if (lane == 0) w_next = (int)gridDim.x + (int)atomicAdd(p.next_item, 1u);
        w_next = __shfl_sync(0xffffffffu, w_next, 0);
        ++q_loaded;
        if (lane == 0) {
          mbar_arrive_expect_tx(&bars[B_QFULL], 2 * C::kTileBytes);
#pragma unroll
          for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int hh = 0; hh < C::kHalves; ++hh)
              tma_load_4d(smem + C::kQOff + t * C::kTileBytes + hh * C::kHalfBytes, &tmQ, &bars[B_QFULL], hh * 64,
                          itm.h, (2 * itm.qb + t) * kBM, itm.b, once);
          if (w_next < p.n_items) {                 // warm L2 with the next item's Q
            const Item nx = item_of<KV>(w_next, p, order);
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
              for (int hh = 0; hh < C::kHalves; ++hh)
                tma_prefetch_4d(&tmQ, hh * 64, nx.h, (2 * nx.qb + t) * kBM, nx.b);
          }
        }
      } else {
        // the item the K producer published (the V copies of an item follow its Q copies)
        if (!wait_or_abort(&bars[B_QFULL], it & 1, abort_flag, p.status)) break;
        const int wi = item_slot[it % kItemSlots];
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[B_QEMPTY]);
        if (wi < 0) {
          clean_end = true;
          break;
        }
        itm = item_of<KV>(wi, p, order);
      }
      const int kvh = itm.h / p.G;
      // paged: this lane's physical block of tile t (lanes >= 8 and blocks past L: none)
      auto read_id = [&](int t) -> int {
        const int nb = min(kBlocks, (itm.L - t * kBN + kPageTokens - 1) / kPageTokens);
        return lane < nb ? __ldg(p.page_table + (size_t)itm.b * p.max_blocks + t * kBlocks + lane) : -1;
      };
      int id = 0;
      if constexpr (KV == KV_PAGED) id = read_id(0);
      for (int t = 0; t < itm.n_load; ++t, ++g) {
        const int s = g % stages;
        if (g >= stages && !wait_or_abort(&bars[empty0 + s], ((g / stages) - 1) & 1, abort_flag, p.status)) {
          ok = false;
          break;
        }
        last[s] = g;
        uint8_t* const dst = ring + s * C::kTileBytes;
        if constexpr (KV != KV_PAGED) {
          if (lane == 0) {
            mbar_arrive_expect_tx(&bars[full0 + s], C::kTileBytes);
#pragma unroll
            for (int hh = 0; hh < C::kHalves; ++hh)
              tma_load_4d(dst + hh * C::kHalfBytes, map, &bars[full0 + s], hh * 64, kvh, t * kBN, itm.b, keep);
          }
        } else {
          // one 16-row box per 64 columns of d and physical block holding keys of this tile below L
          const int nb = min(kBlocks, (itm.L - t * kBN + kPageTokens - 1) / kPageTokens);
          int blk = id;
          if (lane < nb && (blk < 0 || blk >= p.num_blocks)) {
            atomicOr(p.status, DEV_PAGE_ID);
            blk = 0;   // keep the byte count; the result is flagged invalid
          }
          if (lane == 0) mbar_arrive_expect_tx(&bars[full0 + s], nb * C::kHalves * kPageTokens * 128);
          __syncwarp();
          if (lane < nb) {
#pragma unroll
            for (int hh = 0; hh < C::kHalves; ++hh)
              tma_load_3d(dst + hh * C::kHalfBytes + lane * kPageTokens * 128, map, &bars[full0 + s], hh * 64, kvh,
                          blk * kPageTokens, keep);
          }
          if (t + 1 < itm.n_load) id = read_id(t + 1);
        }
      }
      if (!ok) break;
      w = w_next;
    }
    // no copy may still be landing in shared memory when the CTA exits (after a clean
    // end, the wait on B_QEMPTY above already covered the last Q copy)
    if (lane == 0) {
      if (is_k && !clean_end && q_loaded > 0) mbar_wait(&bars[B_QFULL], (q_loaded - 1) & 1);
      for (int i = 0; i < stages; ++i)
        if (last[i] >= 0) mbar_wait(&bars[full0 + i], (last[i] / stages) & 1);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------- MMA issuer
    // The whole warp runs this loop and its waits, so that every operand (descriptors,
    // stages, item sizes) is warp-uniform; one elected lane issues the MMAs and commits.
    // Issued from a single divergent lane, each MMA cost about 110 clock cycles of
    // issue on a sub-partition shared with two softmax warps -- more than its 64 cycles
    // of tensor-core time.
    const uint32_t leader = elect_one();
    constexpr int kKStages = C::kKStages, kVStages = C::kVStages;
    constexpr uint32_t idS = idesc_bf16(kBM, kBN, 0, 0);     // Q (K-major) x K^T (K-major)
    constexpr uint32_t idO = idesc_bf16(kBM, D, 0, 1);       // P (TMEM) x V (N-major)
    // shared-memory descriptors (128-byte swizzle, 1024-byte row-group stride): only the
    // low word varies -- the start address in 16-byte units -- so every operand is a
    // precomputed base (Q tile, K or V ring stage) plus a compile-time K-step offset
    const uint32_t sbase = smem_u32(smem);
    const uint32_t q_lo0 = desc_lo(sbase + C::kQOff, 16), q_lo1 = desc_lo(sbase + C::kQOff + C::kTileBytes, 16);
    const uint32_t k_lo0 = desc_lo(sbase + C::kKOff, 16);
    const uint32_t v_lo0 = desc_lo(sbase + C::kVOff, C::kHalfBytes);
    constexpr uint32_t kStageLo = C::kTileBytes >> 4;     // one ring stage in descriptor units
    auto issue_s = [&](int t, int ks) {     // S_t = Q_t K^T, K in ring stage ks
      const uint32_t qa = t ? q_lo1 : q_lo0, kb = k_lo0 + ks * kStageLo;
      const uint32_t d = tmem + C::s_col(t);
      tc_mma_ss_lo<0>(leader, d, qa, kb, idS);
#pragma unroll
      for (int kk = 1; kk < D / 16; ++kk) {
        const uint32_t off = ((kk >> 2) * C::kHalfBytes + (kk & 3) * 32) >> 4;
        tc_mma_ss_lo<1>(leader, d, qa + off, kb + off, idS);
      }
      tc_commit_if(leader, &bars[B_SFULL + t]);
    };
    // O_t (+)= P_t V over keys 64*half .. 64*half+63; P_t sits in the first 64 columns of S_t
    auto issue_pv = [&](int t, int vs, bool first, int half) {
      const uint32_t vb = v_lo0 + vs * kStageLo;
      const uint32_t d = tmem + C::o_col(t), pa = tmem + C::s_col(t);
#pragma unroll
      for (int k4 = 0; k4 < kBN / 32; ++k4) {
        const int kk = half * (kBN / 32) + k4;
        if (kk == 0 && first) tc_mma_ts_lo<0>(leader, d, pa, vb, idO);
        else tc_mma_ts_lo<1>(leader, d, pa + kk * 8, vb + ((kk * 16 * 128) >> 4), idO);
      }
    };
    int pcnt[2] = {0, 0};                  // P phases consumed per tile
    // both halves of PV_t(j): the first as soon as the softmax group has published P of
    // the first 64 keys (the second half's exponentials overlap it)
    auto pv_tile = [&](int t, int st, int j, int it) -> bool {
      const uint32_t par = (pcnt[t]++) & 1;
      if (!wait_or_abort(&bars[B_PHALF + t], par, abort_flag, p.status)) return false;
      if (j == 0 && it > 0 && !wait_or_abort(&bars[B_OFREE + t], (it - 1) & 1, abort_flag, p.status)) return false;
      tc_fence_after();
      issue_pv(t, st, j == 0, 0);
      if (!wait_or_abort(&bars[B_PFULL + t], par, abort_flag, p.status)) return false;
      tc_fence_after();
      issue_pv(t, st, j == 0, 1);
      return true;
    };
    int g = 0, it = 0;                     // K/V tiles consumed, items done
    bool ok = true;
    for (;; ++it) {
      if (!wait_or_abort(&bars[B_QFULL], it & 1, abort_flag, p.status)) break;
      const int w = __shfl_sync(0xffffffffu, item_slot[it % kItemSlots], 0);
      if (w < 0) break;                    // no more work
      const Item itm = item_of<KV>(w, p, order);
      const int n_load = __shfl_sync(0xffffffffu, itm.n_load, 0);
      const int n_kv0 = __shfl_sync(0xffffffffu, itm.n_kv0, 0);
      const int g0 = g;
      const int ks0 = g0 % kKStages;
      ok = wait_or_abort(&bars[B_KFULL + ks0], (g0 / kKStages) & 1, abort_flag, p.status);
      if (!ok) break;
      tc_fence_after();
      issue_s(0, ks0);
      issue_s(1, ks0);
      tc_commit_if(leader, &bars[B_KEMPTY + ks0]);
      for (int j = 0; j < n_load; ++j) {
        const int gj = g0 + j, st = gj % kVStages;
        const int ksn = (gj + 1) % kKStages;     // K stage of the next tile
        const bool next_k = j + 1 < n_load;
        ok = wait_or_abort(&bars[B_VFULL + st], (gj / kVStages) & 1, abort_flag, p.status);
        if (!ok) break;
        if constexpr (!kDenseKv<KV>) {
          // V rows of keys >= L: any bytes (cache) or never loaded (paged); the PV MMAs
          // would multiply them by p = 0.  Zeroed here, by the warp that consumes the V
          // phases in order, before either PV of the tile is issued.
          const int valid = __shfl_sync(0xffffffffu, itm.L, 0) - j * kBN;
          if (valid < kBN) {
            uint8_t* vst = smem + C::kVOff + st * C::kTileBytes;
            for (int idx = max(valid, 0) * 8 + lane; idx < kBN * 8; idx += 32)
#pragma unroll
              for (int hh = 0; hh < C::kHalves; ++hh)
                *reinterpret_cast<uint4*>(vst + hh * C::kHalfBytes + idx * 16) = make_uint4(0, 0, 0, 0);
            fence_proxy_async_smem();
            __syncwarp();
          }
        }
        if (j < n_kv0) {
          ok = pv_tile(0, st, j, it);
          if (!ok) break;
          if (j == n_kv0 - 1) tc_commit_if(leader, &bars[B_ODONE + 0]);
        }
        if (next_k) {
          ok = wait_or_abort(&bars[B_KFULL + ksn], ((gj + 1) / kKStages) & 1, abort_flag, p.status);
          if (!ok) break;
          tc_fence_after();
          if (j + 1 < n_kv0) issue_s(0, ksn);
        }
        ok = pv_tile(1, st, j, it);
        if (!ok) break;
        tc_commit_if(leader, &bars[B_VEMPTY + st]);        // V of this stage is no longer needed
        if (j == n_load - 1) tc_commit_if(leader, &bars[B_ODONE + 1]);
        if (next_k) {
          issue_s(1, ksn);
          tc_commit_if(leader, &bars[B_KEMPTY + ksn]);
          // that was the item's last MMA reading Q: the next item's Q may land once it is done
          if (j + 2 == n_load) tc_commit_if(leader, &bars[B_QEMPTY]);
        }
      }
      if (!ok) break;
      if (n_load == 1) tc_commit_if(leader, &bars[B_QEMPTY]);
      g = g0 + n_load;
    }
  }
  } else {
    reg_alloc<regs_softmax<D, KV>()>();
    // -------------------------------------------------- softmax warps 0-7
    const int t = warp >> 2;                            // query tile of this group
    const int row = (warp & 3) * 32 + lane;             // TMEM lane == query row in the tile
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t s_addr = lane_base + C::s_col(t);
    const uint32_t o_addr = lane_base + C::o_col(t);
    int scnt = 0, it = 0;                               // S_FULL phases consumed, items done
    bool ok = true;
    for (;; ++it) {
    if (!wait_or_abort(&bars[B_QFULL], it & 1, abort_flag, p.status)) { ok = false; break; }
    const int w = item_slot[it % kItemSlots];
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars[B_QEMPTY]);        // this warp has read the item
    if (w < 0) break;                                   // no more work
    const Item itm = item_of<KV>(w, p, order);
    const int q_row = (2 * itm.qb + t) * kBM + row;
    const int nkv = t ? itm.n_load : itm.n_kv0;
    float m = -INFINITY, l = 0.f;
    for (int j = 0; j < nkv; ++j) {
      if (!wait_or_abort(&bars[B_SFULL + t], (scnt++) & 1, abort_flag, p.status)) { ok = false; break; }
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
      const int lim = p.causal ? min(itm.off + q_row - key0 + 1, itm.L - key0) : (itm.L - key0);   // visible: [0, lim)
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
      // O_t is stable here (PV_t(j-1) completed before S_t(j) did) and PV_t(j)
      // waits for this group's first arrival below
      // (16 columns at a time: the scores still occupy 128 registers)
      if (warp_raise && j > 0) {
#pragma unroll 1
        for (int c = 0; c < D; c += 16) {
          uint32_t r[16];
          tmem_ld16(o_addr + c, r);
          tc_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tmem_st16(o_addr + c, r);
        }
      }
      // p = 2^(s*scale_log2 - m), bf16 P over the consumed S columns, in two halves of 64
      // keys: the first half is published (with the rescaled O) before the second is computed
      const float2 sc2 = make_float2(p.scale_log2, p.scale_log2), nm2 = make_float2(neg_mu, neg_mu);
      float2 sum2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      // rows with masked keys (-inf scores) take every exponential on the SFU
      constexpr unsigned kFma = exp_fma_pairs<D>();
      const bool soft = kFma != 0 && !__any_sync(0xffffffffu, lim < kBN);
      if (soft) exp_store_half<0, true, kFma>(s, sc2, nm2, sum2, s_addr);
      else exp_store_half<0, false, kFma>(s, sc2, nm2, sum2, s_addr);
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_PHALF + t]);
      if (soft) exp_store_half<1, true, kFma>(s, sc2, nm2, sum2, s_addr);
      else exp_store_half<1, false, kFma>(s, sc2, nm2, sum2, s_addr);
      const float2 sa = __fadd2_rn(sum2[0], sum2[1]), sb = __fadd2_rn(sum2[2], sum2[3]);
      const float2 sab = __fadd2_rn(sa, sb);
      l = l * alpha + (sab.x + sab.y);
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_PFULL + t]);
    }

    // ---------------------------------------------------------- epilogue
    if (!ok || !wait_or_abort(&bars[B_ODONE + t], it & 1, abort_flag, p.status)) {
      ok = false;
      break;
    }
    {
      tc_fence_after();
      const float inv_l = itm.bad ? __int_as_float(0x7fc00000) : 1.f / l;   // NaN rows for a bad length
      if (itm.bad && t == 0 && row == 0) atomicOr(p.status, DEV_SEQLEN);
      const bool store = q_row < p.N;
      const size_t obase = (((size_t)itm.b * p.N + q_row) * p.Hq + itm.h) * D;
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
      if (store && p.lse)
        p.lse[((size_t)itm.b * p.Hq + itm.h) * p.N + q_row] = itm.bad ? __int_as_float(0x7fc00000) : (m + log2f(l)) * kLn2;
      // O_t has been read: the next item's first PV may overwrite it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_OFREE + t]);
    }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag && warp == 9) {
    // a wait gave up: let every tensor-core op this CTA issued drain before TMEM is released
    // (the commit comes from the lane that issued the MMAs)
    const uint32_t leader = elect_one();
    tc_commit_if(leader, &bars[B_DRAIN]);
    mbar_wait(&bars[B_DRAIN], 0);
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
  if (threadIdx.x == 0 && atomicAdd(p.done_ctas, 1u) == gridDim.x - 1) {
    // every CTA has taken its last ticket: leave the queue at zero for the next launch
    atomicExch(p.next_item, 0u);
    atomicExch(p.done_ctas, 0u);
  }
}

// This launch's pair of queue counters on the current device.
cudaError_t queue_slot(unsigned** next, unsigned** done) {
  constexpr int kMaxDevices = 64;
  static void* base[kMaxDevices] = {};
  static std::atomic<unsigned> launches[kMaxDevices];
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> g(mu);
    if (!base[dev] && (e = cudaGetSymbolAddress(&base[dev], g_prefill_queue)) != cudaSuccess) return e;
  }
  const unsigned slot = launches[dev].fetch_add(1u) % kQueueSlots;
  *next = static_cast<unsigned*>(base[dev]) + slot;
  *done = static_cast<unsigned*>(base[dev]) + kQueueSlots + slot;
  return cudaSuccess;
}

template <int D, int KV>
cudaError_t run_prefill(const PrefillLaunch& a, cudaStream_t stream) {
  using C = PrefillCfg<D>;
  CUtensorMap tq, tk, tv;
  // 4-D views {d, heads, rows, B}; box {64, 1, 128, 1} with the 128-byte swizzle
  auto enc = [&](CUtensorMap* m, const void* base, int heads, int rows) {
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)rows, (cuuint64_t)a.B};
    cuuint64_t str[3] = {(cuuint64_t)D * 2, (cuuint64_t)heads * D * 2, (cuuint64_t)rows * heads * D * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)kBN, 1};
    return encode_tmap_nd(m, base, 4, dims, str, box);
  };
  if (enc(&tq, a.q, a.Hq, a.N)) return cudaErrorInvalidValue;
  if constexpr (kDenseKv<KV>) {
    if (enc(&tk, a.k, a.Hkv, a.N) || enc(&tv, a.v, a.Hkv, a.N)) return cudaErrorInvalidValue;
  } else if constexpr (KV == KV_CACHE) {
    if (enc(&tk, a.k, a.Hkv, a.capacity) || enc(&tv, a.v, a.Hkv, a.capacity)) return cudaErrorInvalidValue;
  } else {
    // pools [num_blocks, 16, Hkv, d] as {d, Hkv, num_blocks * 16}; one 16-row box per block
    const uint64_t rows = (uint64_t)a.num_blocks * kPageTokens;
    const uint64_t s1 = (uint64_t)D * 2, s2 = (uint64_t)a.Hkv * D * 2;
    if (encode_tmap_3d(&tk, a.k, D, a.Hkv, rows, s1, s2, 64, 1, kPageTokens) ||
        encode_tmap_3d(&tv, a.v, D, a.Hkv, rows, s1, s2, 64, 1, kPageTokens))
      return cudaErrorInvalidValue;
  }
  PrefillParams p;
  p.o = a.o;
  p.lse = a.lse;
  p.status = a.status;
  p.N = a.N;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.G = a.Hq / a.Hkv;
  p.B = a.B;
  p.n_qblocks = (a.N + 2 * kBM - 1) / (2 * kBM);
  p.n_ktiles = (a.N + kBN - 1) / kBN;
  const long long items = (long long)p.n_qblocks * a.Hq * a.B;
  if (items > INT32_MAX) return cudaErrorInvalidValue;
  p.n_items = (int)items;
  p.scale_log2 = a.scale * kLog2e;
  p.causal = a.causal;
  p.o_bf16 = a.o_bf16;
  p.seqlens = a.seqlens;
  p.page_table = a.page_table;
  p.max_blocks = a.max_blocks;
  p.num_blocks = a.num_blocks;
  p.max_keys = KV == KV_PAGED ? a.max_blocks * kPageTokens : (KV == KV_CACHE ? a.capacity : a.N);
  if (!kDenseKv<KV> && a.max_seqlen > 0 && a.max_seqlen < p.max_keys) p.max_keys = a.max_seqlen;
  cudaError_t qe = queue_slot(&p.next_item, &p.done_ctas);
  if (qe != cudaSuccess) return qe;
  auto kern = prefill_kernel<D, KV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  // the softmax warpgroups' register increase waits until the producer warpgroup's
  // decrease has made room, out of what the block was launched with: refuse a build
  // whose launch register count could not cover the split
  cudaFuncAttributes fa;
  if ((e = cudaFuncGetAttributes(&fa, kern)) != cudaSuccess) return e;
  if (fa.numRegs * kThreads < 2 * 128 * regs_softmax<D, KV>() + 128 * regs_io<D, KV>())
    return cudaErrorInvalidConfiguration;
  // persistent: one CTA per SM (each owns all 512 TMEM columns)
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int grid = p.n_items < sms ? p.n_items : sms;
  kern<<<grid, kThreads, C::kSmemBytes, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const PrefillLaunch& a, cudaStream_t stream) {
  if (!a.seqlens) {
    const bool grouped = 4.0 * a.N * a.d >= kDenseKvHeadBytes;
    if (a.d == 128) return grouped ? run_prefill<128, KV_DENSE_GROUPED>(a, stream) : run_prefill<128, KV_DENSE>(a, stream);
    return grouped ? run_prefill<64, KV_DENSE_GROUPED>(a, stream) : run_prefill<64, KV_DENSE>(a, stream);
  }
  if (!a.page_table)
    return a.d == 128 ? run_prefill<128, KV_CACHE>(a, stream) : run_prefill<64, KV_CACHE>(a, stream);
  return a.d == 128 ? run_prefill<128, KV_PAGED>(a, stream) : run_prefill<64, KV_PAGED>(a, stream);
}

}  // namespace kvattn
