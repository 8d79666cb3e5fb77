// BigBird block-sparse attention forward for B200 (sm_100a).
//
// Computes, per (batch b, head h, query token t),
//   O = softmax over the attended keys of (q_t . k_p * scale) times V,  lse = ln sum exp(...)
// i.e. Softmax(Q K^T / sqrt(d_k) restricted to M) V ("Adapt or Perish ... Adaptive Sparse
// Transformer", sparse-attention formula; "BigBird 稀疏注意力机制解析", 核心实现: one
// softmax over global + window + random key blocks), with the block mask kept as a
// per-tile list of 64-key blocks ("SQA 稀疏注意力机制详解" 3.1: block-sparse mask,
// attention only on non-zero blocks).
//
// Kernel design (head dim 64; FwdCfg below has what changes at 128): one persistent
// CTA per SM (512 threads, four warpgroups) running two independent pipelines
// ("slots"), each with its own work items, shared-memory rings, barriers and 256 TMEM
// columns: O (64), S (128) and P (64, bf16 pairs).  A tile is two
// 64-row query blocks of the same (b, h) over the union of their key-block lists; a
// chunk is two consecutive union entries (128 keys).
//   warps 0-3 / 4-7  softmax of slot 0 / 1 (thread r of the slot owns tile row r =
//               TMEM lane r).  Per chunk: load all of S(g) into registers and hand the
//               S columns back at once (S(g + 1) is computed during this chunk's
//               exponentials); the chunk max; p = 2^(s * scale * log2 e - m) on the ex2
//               unit; P (bf16) into the P columns once PV(g - 1) has read them.  m is
//               raised only when a chunk's max exceeds it by more than 8 (log2 units;
//               then l and O are rescaled), so p <= 2^8.  A finished tile's epilogue runs
//               in the next tile's first chunk.
//   warp 8 + s  K producer of slot s: stages the slot's work items; TMA loads of the Q tile
//               and of K, the chunk's two 64-key blocks per 16 KB stage, 2 stages.
//   warp 14 + s V producer of slot s: TMA loads of V into 2 stages of 16 KB.
//   warp 10 + s tcgen05 S issuer: S(g) = Q K_g^T (M=128, N=128, or 64 for a lone entry).
//   warp 12 + s tcgen05 PV issuer: O (+)= P(g) V_g (A = P from TMEM, 16 keys per MMA).
// A tcgen05.mma holds its issuing warp for ~120 cycles, and a TMA load's issue waits on
// its stage; a role per warp keeps these latencies off each other's paths.  Every
// per-chunk hand-off costs the softmax warps a few hundred cycles of latency, so a chunk
// spans 128 keys to spread that cost over 128 exponentials per thread.
// Entries carry per-block membership bits so each half of the tile sees exactly its own
// row (a softmax warp keeps an item's bits as two ballots); a warp whose half does not
// attend a block gives it zero P without exponentials, and entries whose 64 keys are all
// padded are dropped when the item is staged.
// Long unions (global rows) are cut into chunks run as separate work items; each stores
// a partial (O, m, l) record, and bsa_merge_kernel, launched after the forward, merges a
// split tile's records into its output rows.
// Token-level layouts (window and global tokens not aligned to blocks) run their own
// instantiation (kTok): flagged entries get a per-row mask of their 64 keys.
// Every wait is bounded (globaltimer); on expiry the CTA records BSA_ERR_DEVICE_TIMEOUT,
// drains its own copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <mutex>
#include <type_traits>

#include "bsa_internal.h"
#include "sm100_ptx.cuh"
#include "bsa_wait.cuh"
#include "bsa_host_cuda.h"

namespace bsa {

constexpr int kItemRing = 4;  // work items a slot's K producer may publish ahead
constexpr int kChunkEnt = 2;  // union entries (64-key blocks) per chunk
constexpr int kKStages = 2;
constexpr int kVStages = 2;
constexpr uint32_t kBoxBytes = 64 * 128;  // one TMA box: 64 rows x 64 bf16 columns
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;  // m is raised when a chunk's max exceeds it by more
constexpr uint32_t kOStageBytes = 32 * 128;  // one warp's 32 O rows of one 64-column half

enum : int {
  kBarQFull = 0,                     // [Q stage] the tile's Q landed (TMA)
  kBarQEmpty = kBarQFull + 2,        // [Q stage] 4 softmax warps: the tile's S MMAs and its
                                     // O staging are done with the buffer
  kBarKFull = kBarQEmpty + 2,        // [K stage] K of the chunk landed (TMA)
  kBarKFree = kBarKFull + kKStages,  // [K stage] MMA commit after the chunk's S
  kBarVFull = kBarKFree + kKStages,  // [V stage] V of the chunk landed (TMA)
  kBarVFree = kBarVFull + kVStages,  // [V stage] MMA commits after the chunk's PV (one per
                                     // PV issuer): the V stage and the P columns are
                                     // reusable, O holds chunk g
  kBarSFull = kBarVFree + kVStages,  // MMA commit after S: the S columns are readable
  kBarSFree = kBarSFull + 1,         // the 128 softmax threads are done with S
  kBarPFull = kBarSFree + 1,         // the 128 softmax threads have stored P
  kBarMmaFinal = kBarPFull + 1,      // [S issuer, PV issuers]
  kBarItemFull = kBarMmaFinal + 3,   // [item ring] the K producer published a work item
  kBarItemEmpty = kBarItemFull + kItemRing,  // [item ring] one arrival from every reader:
                                             // V producer, the issuers, the softmax warps
  kNumBars = kBarItemEmpty + kItemRing
};
constexpr uint32_t kWarpArrivals = 4;     // Q release: one arrival per softmax warp
constexpr uint32_t kThreadArrivals = 128;  // S free, P full: every softmax thread arrives

// One published work item in shared memory: its index, its fields, its query-block
// pair and, per union entry, the entry and the key-padding bits of its key block.
constexpr int kMaxItemEntries = 64;
static_assert(kSplitThreshold <= kMaxItemEntries && kSplitChunk <= kMaxItemEntries,
              "an item's entries must fit its stage");
static_assert(kMaxItemEntries <= 64, "a softmax warp keeps an item's entry bits in two 32-lane ballots");
struct ItemStage {
  int t;  // work item index, or kItemNone
  int qa, qb;
  int b;
  int pad[4];
  WorkItem w;
  uint32_t ent[kMaxItemEntries];
  unsigned long long kb[kMaxItemEntries];  // all ones without a key mask
};
static_assert(sizeof(ItemStage) % 16 == 0, "stage alignment");

// What depends on the head dim d (64 or 128).  Operands in shared memory are kept as
// d / 64 column halves of 64 bf16 (one 128-byte swizzle atom wide), each half laid
// out as at d = 64: a Q buffer is [half][128 rows][64], a K or V stage
// [half][entry][64 keys][64].  TMEM of a slot: O (d columns), S (128), P (64, bf16
// pairs).
//   d = 64:  two slots per CTA, 512 threads: softmax warps 0-7 (slot = warp / 4),
//            K producer 8 + s, S issuer 10 + s, PV issuer 12 + s, V producer 14 + s.
//   d = 128: one slot (a second would need 256 KB of shared memory), 384 threads:
//            softmax warps 0-3, K producer 4, S issuer 5, PV issuers 6 and 7 (one per
//            column half of O, so that each issues eight N = 64 MMAs a chunk), V
//            producer 8; warps 9-11 only take part in the register split.
template <int kD>
struct FwdCfg {
  static_assert(kD == 64 || kD == 128, "head dim");
  static constexpr int kHalves = kD / 64;
  static constexpr int kSlots = kD == 64 ? 2 : 1;
  static constexpr int kThreads = kD == 64 ? 512 : 384;
  static constexpr int kPvIssuers = kHalves;  // per slot
  static constexpr int kKProdWarp = 4 * kSlots;  // + slot
  static constexpr int kSWarp = kKProdWarp + kSlots;  // + slot; the first allocates and frees TMEM
  static constexpr int kPvWarp = kSWarp + kSlots;     // + slot * kPvIssuers + half
  static constexpr int kVProdWarp = kPvWarp + kSlots * kPvIssuers;  // + slot
  static_assert(kVProdWarp + kSlots <= kThreads / 32, "role warps");
  // Register split: the softmax warpgroups take kSoftmaxRegs, the other warpgroups
  // kOtherRegs; the sum stays within the launch's pool (threads x registers a thread).
  static constexpr uint32_t kSoftmaxRegs = kD == 64 ? 200 : 232;
  static constexpr uint32_t kOtherRegs = 56;
  static constexpr uint32_t kLaunchRegs = (65536 / kThreads) & ~7u;
  static_assert(kSlots * 128 * kSoftmaxRegs + (kThreads - kSlots * 128) * kOtherRegs <= kThreads * kLaunchRegs,
                "register split exceeds the launch budget");
  // the noinline wait paths of the two register budgets (one instantiation per budget)
  static constexpr int kSoftRegion = kD == 64 ? 1 : 3;
  static constexpr int kRoleRegion = kD == 64 ? 2 : 4;
  static constexpr uint32_t kItemReaders = 4 + 2 + kPvIssuers;  // softmax warps, V producer, S issuer, PV
  static constexpr uint32_t kQHalfBytes = 2 * kBoxBytes;          // one column half of the 128-row tile
  static constexpr uint32_t kQBytes = kHalves * kQHalfBytes;
  static constexpr uint32_t kStageHalfBytes = kChunkEnt * kBoxBytes;  // one column half of a chunk
  static constexpr uint32_t kStageBytes = kHalves * kStageHalfBytes;
  static constexpr uint32_t kTmemO = 0;
  static constexpr uint32_t kTmemS = kD;
  static constexpr uint32_t kTmemP = kD + 128;
  static constexpr uint32_t kSlotCols = 256;  // slot s owns columns from 256 s
  static_assert(kTmemP + 64 <= (kSlots == 2 ? kSlotCols : kTmemCols), "TMEM map");
  static constexpr int kRecFloats = rec_floats(kD);
  // shared memory map of one slot (offsets from its 1024-aligned base)
  static constexpr uint32_t kSmemQ = 0;  // 2 Q tiles; a finished tile's buffer also stages its O
  static constexpr uint32_t kSmemK = kSmemQ + 2 * kQBytes;
  static constexpr uint32_t kSmemV = kSmemK + kKStages * kStageBytes;
  static constexpr uint32_t kSmemBar = kSmemV + kVStages * kStageBytes;
  static constexpr uint32_t kSmemItems = (kSmemBar + 8 * kNumBars + 15) & ~15u;  // ItemStage[kItemRing]
  static constexpr uint32_t kSlotBytes = (kSmemItems + sizeof(ItemStage) * kItemRing + 1023) & ~1023u;
  static constexpr uint32_t kSmemMisc = kSlots * kSlotBytes;  // u32 TMEM base, int abort flag
  static constexpr uint32_t kSmemAlloc = kSmemMisc + 16 + 1024;  // + slack for 1024-byte alignment
  static_assert(kSmemAlloc <= 227 * 1024, "shared memory budget");
  static_assert(kQHalfBytes == 4 * kOStageBytes, "a Q buffer half stages the four warps' O rows");
};

// Where one slot's roles find their resources.  Work items are handed out
// dynamically: the slot's K producer takes the next index from a global counter and
// publishes it to the slot's other roles through a small ring in shared memory.
struct Slot {
  uint32_t sQ, sK, sV, bars;
  uint8_t* q_generic;  // generic pointer to the Q buffers (O staging)
  ItemStage* items;    // the item ring
  uint32_t tmem;       // TMEM address of the slot's column 0
};

struct FwdParams {
  CUtensorMap tm_q, tm_k, tm_v;
  CUtensorMap tm_o;  // O as [B*H*L, 64] bf16, 32-row boxes (epilogue stores)
  __nv_bfloat16* out;
  float* lse;
  const WorkItem* items;
  const int32_t* pair_q;
  const uint32_t* pair_ent;
  const unsigned long long* keybits;  // [B, nb] or null
  float* partials;
  int* sched;  // [0] next work item, [1] slots finished; cleared before each launch
  int B, H, L, nb, items_per_batch, n_split, n_records;
  int split_items;  // the first split_items items of a batch element are split-tile chunks
  int split_lead;   // split chunks are handed out this many batch elements early
  const int32_t* item_order;  // null, or the items of one batch element head by head
  // token-level layouts (else null): bit c of word j set when token 64 j + c is global;
  // the window in tokens.  Entries flagged at kEntMaskShift + half get per-row masks.
  const unsigned long long* tok_gbits;
  long long tok_window;
  float scale_log2;
  unsigned long long timeout_ns;
};

constexpr int kItemNone = -1;   // no work left
constexpr int kItemAbort = -2;  // a wait gave up

__device__ __forceinline__ uint32_t bar_at(uint32_t bars, int i) { return bars + 8u * static_cast<uint32_t>(i); }

// The slot's k-th work item for an issuer (one thread): its index and entry count.
// The stage is released at once.
template <int kRegion>
__device__ __forceinline__ int take_item_one(const Slot& sl, uint32_t k, int* count, volatile int* abort_flag,
                                             uint64_t timeout_ns) {
  const uint32_t i = k % kItemRing;
  if (!wait_one<kRegion>(bar_at(sl.bars, kBarItemFull + i), (k / kItemRing) & 1u, abort_flag, timeout_ns))
    return kItemAbort;
  const ItemStage& st = sl.items[i];
  const int t = st.t;
  *count = st.w.count;
  ptx::mbar_arrive(bar_at(sl.bars, kBarItemEmpty + i));
  return t;
}

// The slot's k-th work item for a warp that keeps reading its stage (the V producer
// until its last load, a softmax warp until the item's epilogue); released with
// release_item_warp.
template <int kRegion>
__device__ __forceinline__ int take_item_warp(const Slot& sl, uint32_t k, volatile int* abort_flag,
                                              uint64_t timeout_ns) {
  const uint32_t i = k % kItemRing;
  if (!wait_warp<kRegion>(bar_at(sl.bars, kBarItemFull + i), (k / kItemRing) & 1u, abort_flag, timeout_ns))
    return kItemAbort;
  return sl.items[i].t;
}

__device__ __forceinline__ void release_item_warp(const Slot& sl, uint32_t k, int lane) {
  __syncwarp();
  if (lane == 0) ptx::mbar_arrive(bar_at(sl.bars, kBarItemEmpty + k % kItemRing));
}

// Lets every copy a producer thread issued land before the CTA exits (after an abort):
// the last issue into ring slot s of n issues had index s + R * floor((n - 1 - s) / R).
template <int kRegion>
__device__ __forceinline__ void drain_ring(uint32_t bars, int first_bar, uint32_t n, uint32_t ring,
                                           volatile int* abort_flag, uint64_t timeout_ns) {
  for (uint32_t s = 0; s < ring; ++s) {
    if (n > s) {
      const uint32_t last = s + ring * ((n - 1u - s) / ring);
      wait_force<kRegion>(bar_at(bars, first_bar + static_cast<int>(s)), (last / ring) & 1u, abort_flag, timeout_ns);
    }
  }
}

// The order in which work items are handed out: t -> (batch element, item).  A batch
// element's items are its ns split-tile chunks (the longest items: each reads every key
// block of its head), then its nn other tiles.  Elements follow one another, so that one
// element's K/V stay in L2 while its items run, except that the split chunks of element
// b are handed out d elements early, at the start of element b - d's items (elements
// 0..d's at the very start), so that no long item starts near the end of the run.  The
// host picks d from the item lengths; d = 0 is the plain element-after-element order.
__host__ __device__ __forceinline__ int2 item_of(int t, int B, int ns, int nn, int d) {
  const int per = ns + nn;
  if (d == 0 || ns == 0) return make_int2(t / per, t - (t / per) * per);
  if (t < (d + 1) * ns) return make_int2(t / ns, t - (t / ns) * ns);  // chunks of elements 0..d
  t -= (d + 1) * ns;
  if (t < nn) return make_int2(0, ns + t);  // element 0's other tiles
  t -= nn;
  const int full = B - 1 - d;  // elements 1..B-1-d: chunks of element j + d, tiles of j
  if (t < full * per) {
    const int j = 1 + t / per, u = t - (j - 1) * per;
    return u < ns ? make_int2(j + d, u) : make_int2(j, u);
  }
  t -= full * per;  // elements B-d..B-1: tiles only
  const int j = B - d + t / nn;
  return make_int2(j, ns + (t - (j - (B - d)) * nn));
}

// K producer, one warp.  Per work item the warp stages the item, its union entries and
// their key-padding bits in the slot's item ring; then lane 0 issues the loads: the Q
// tile into Q buffer (tile % 2) once the tile two back has released it, and for each
// chunk g its K blocks into K stage g % 2 once S(g - 2) is done.  Each 64-row block
// goes in d / 64 boxes, one per column half.
template <int kD>
__device__ __forceinline__ void k_producer(const FwdParams& p, const Slot& sl, int lane, volatile int* abort_flag) {
  using C = FwdCfg<kD>;
  constexpr int R = C::kRoleRegion;
  const uint32_t sQ = sl.sQ, sK = sl.sK, bars = sl.bars;
  auto bar = [&](int i) { return bar_at(bars, i); };
  const uint64_t pol_q = ptx::policy_evict_first();
  const uint64_t pol_kv = ptx::policy_evict_last();
  const int total = p.B * p.items_per_batch;
  uint32_t nq = 0, nk = 0;  // Q tiles and K blocks issued (lane 0)
  bool alive = true;
  int t_next = lane == 0 ? atomicAdd(p.sched, 1) : 0;
  for (uint32_t k = 0;; ++k) {
    t_next = __shfl_sync(0xffffffffu, t_next, 0);
    const int t = t_next < total ? t_next : kItemNone;
    const uint32_t ii = k % kItemRing;
    bool ok = true;
    if (lane == 0)
      ok = wait_one<R>(bar(kBarItemEmpty + static_cast<int>(ii)), ((k / kItemRing) & 1u) ^ 1u, abort_flag,
                          p.timeout_ns);
    if (!__shfl_sync(0xffffffffu, ok, 0)) {
      alive = false;
      break;
    }
    // stage the item for the slot's other roles
    ItemStage& st = sl.items[ii];
    if (t >= 0) {
      const int2 bi = item_of(t, p.B, p.split_items, p.items_per_batch - p.split_items, p.split_lead);
      const int b = bi.x, i = p.item_order != nullptr ? p.item_order[bi.y] : bi.y;
      const WorkItem w = p.items[i];
      int kept = w.count;
      if (p.keybits == nullptr) {
        for (int e = lane; e < w.count; e += 32) {
          st.ent[e] = p.pair_ent[w.start + e];
          st.kb[e] = ~0ull;
        }
      } else {
        // Entries whose 64 keys are all padded are dropped here, so that no load or MMA
        // is issued for them.  Lane x looks at entries x and x + 32 (at most 64); the
        // kept ones are packed in order.  If none is kept, entry 0 stays with no
        // membership bits: its P is zero and the tile's rows are still written.
        const bool h0 = lane < w.count, h1 = lane + 32 < w.count;
        const uint32_t en0 = h0 ? p.pair_ent[w.start + lane] : 0u;
        const uint32_t en1 = h1 ? p.pair_ent[w.start + lane + 32] : 0u;
        const unsigned long long* kbb = p.keybits + static_cast<size_t>(b) * p.nb;
        const unsigned long long kb0 = h0 ? kbb[en0 & kEntColMask] : 0ull;
        const unsigned long long kb1 = h1 ? kbb[en1 & kEntColMask] : 0ull;
        const uint32_t keep0 = __ballot_sync(0xffffffffu, kb0 != 0ull);
        const uint32_t keep1 = __ballot_sync(0xffffffffu, kb1 != 0ull);
        const uint32_t below = (1u << lane) - 1u;
        const int n0 = __popc(keep0);
        kept = n0 + __popc(keep1);
        if (kb0 != 0ull) {
          st.ent[__popc(keep0 & below)] = en0;
          st.kb[__popc(keep0 & below)] = kb0;
        }
        if (kb1 != 0ull) {
          st.ent[n0 + __popc(keep1 & below)] = en1;
          st.kb[n0 + __popc(keep1 & below)] = kb1;
        }
        if (kept == 0) {
          if (lane == 0) {
            st.ent[0] = en0 & kEntColMask;
            st.kb[0] = 0ull;
          }
          kept = 1;
        }
      }
      if (lane == 0) {
        st.w = w;
        st.w.count = kept;
        st.b = b;
        st.qa = p.pair_q[2 * w.pair];
        st.qb = p.pair_q[2 * w.pair + 1];
      }
    }
    if (lane == 0) st.t = t;
    __threadfence_block();
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(bar(kBarItemFull + static_cast<int>(ii)));
    if (t < 0) break;
    if (lane == 0) {
      t_next = atomicAdd(p.sched, 1);  // the next item's index arrives while this tile loads
      const WorkItem& w = st.w;
      const int row0 = (st.b * p.H + w.h) * p.L;
      const int qa = st.qa, qb = st.qb;
      const uint32_t qs = nq & 1u;
      if (!wait_one<R>(bar(kBarQEmpty + qs), ((nq >> 1) & 1u) ^ 1u, abort_flag, p.timeout_ns)) {
        alive = false;
      } else {
        ptx::mbar_arrive_expect_tx(bar(kBarQFull + qs), C::kQBytes);
#pragma unroll
        for (int hf = 0; hf < C::kHalves; ++hf) {
          const uint32_t dst = sQ + qs * C::kQBytes + hf * C::kQHalfBytes;
          ptx::tma_load_2d(dst, &p.tm_q, bar(kBarQFull + qs), 64 * hf, row0 + qa * 64, pol_q);
          ptx::tma_load_2d(dst + kBoxBytes, &p.tm_q, bar(kBarQFull + qs), 64 * hf,
                           row0 + (qb >= 0 ? qb : qa) * 64, pol_q);
        }
        ++nq;
        for (int e0 = 0; e0 < w.count; e0 += kChunkEnt) {
          const int ne = min(kChunkEnt, w.count - e0);
          const uint32_t ks = nk % kKStages;
          if (!wait_one<R>(bar(kBarKFree + ks), ((nk / kKStages) & 1u) ^ 1u, abort_flag, p.timeout_ns)) {
            alive = false;
            break;
          }
          ptx::mbar_arrive_expect_tx(bar(kBarKFull + ks), kBoxBytes * C::kHalves * ne);
          for (int x = 0; x < ne; ++x) {
            const int krow = row0 + static_cast<int>(st.ent[e0 + x] & kEntColMask) * 64;
#pragma unroll
            for (int hf = 0; hf < C::kHalves; ++hf)
              ptx::tma_load_2d(sK + ks * C::kStageBytes + hf * C::kStageHalfBytes + x * kBoxBytes, &p.tm_k,
                               bar(kBarKFull + ks), 64 * hf, krow, pol_kv);
          }
          ++nk;
        }
      }
    }
    if (!__shfl_sync(0xffffffffu, alive, 0)) {
      alive = false;
      break;
    }
  }
  if (lane != 0) return;
  if (alive) {
    // Every slot's K producer counts itself out once it has drawn its last index; the
    // last one resets both counters, so the workspace is left as the call found it.
    __threadfence();
    if (atomicAdd(p.sched + 1, 1) == C::kSlots * static_cast<int>(gridDim.x) - 1) {
      p.sched[0] = 0;
      p.sched[1] = 0;
    }
  } else {
    drain_ring<R>(bars, kBarQFull, nq, 2u, abort_flag, p.timeout_ns);
    drain_ring<R>(bars, kBarKFull, nk, static_cast<uint32_t>(kKStages), abort_flag, p.timeout_ns);
  }
}

// V producer, one warp: follows the item ring and loads V of chunk g into V stage
// g % 2 once PV(g - 2) is done, releasing each item after its last load.
template <int kD>
__device__ __forceinline__ void v_producer(const FwdParams& p, const Slot& sl, int lane, volatile int* abort_flag) {
  using C = FwdCfg<kD>;
  constexpr int R = C::kRoleRegion;
  const uint32_t sV = sl.sV, bars = sl.bars;
  auto bar = [&](int i) { return bar_at(bars, i); };
  const uint64_t pol_kv = ptx::policy_evict_last();
  uint32_t nv = 0;
  bool alive = true;
  for (uint32_t k = 0; alive; ++k) {
    const int t = take_item_warp<R>(sl, k, abort_flag, p.timeout_ns);
    if (t < 0) {
      if (t == kItemAbort) alive = false;
      break;
    }
    const ItemStage& st = sl.items[k % kItemRing];
    if (lane == 0) {
      const int row0 = (st.b * p.H + st.w.h) * p.L;
      for (int e0 = 0; e0 < st.w.count; e0 += kChunkEnt) {
        const int ne = min(kChunkEnt, st.w.count - e0);
        const uint32_t vs = nv % kVStages;
        if (!wait_one<R>(bar(kBarVFree + vs), ((nv / kVStages) & 1u) ^ 1u, abort_flag, p.timeout_ns)) {
          alive = false;
          break;
        }
        ptx::mbar_arrive_expect_tx(bar(kBarVFull + vs), kBoxBytes * C::kHalves * ne);
        for (int x = 0; x < ne; ++x) {
          const int vrow = row0 + static_cast<int>(st.ent[e0 + x] & kEntColMask) * 64;
#pragma unroll
          for (int hf = 0; hf < C::kHalves; ++hf)
            ptx::tma_load_2d(sV + vs * C::kStageBytes + hf * C::kStageHalfBytes + x * kBoxBytes, &p.tm_v,
                             bar(kBarVFull + vs), 64 * hf, vrow, pol_kv);
        }
        ++nv;
      }
    }
    alive = __shfl_sync(0xffffffffu, alive, 0);
    release_item_warp(sl, k, lane);
  }
  if (lane == 0 && !alive) drain_ring<R>(bars, kBarVFull, nv, static_cast<uint32_t>(kVStages), abort_flag, p.timeout_ns);
}

// tcgen05 S issuer, one thread.  S(g) = Q K_g^T (N = 64 per key block of the chunk) into
// the S columns once K(g) has landed and the softmax has loaded S(g - 1).  Its commits
// signal S full and release K stage g % 2.  The head dim runs in steps of 16: four per
// 64-column half of Q and K.
template <int kD>
__device__ __forceinline__ void s_issuer(const FwdParams& p, const Slot& sl, volatile int* abort_flag) {
  using C = FwdCfg<kD>;
  constexpr int R = C::kRoleRegion;
  const uint32_t sQ = sl.sQ, sK = sl.sK, bars = sl.bars, tmem = sl.tmem;
  auto bar = [&](int i) { return bar_at(bars, i); };
  constexpr uint32_t kIdescS2 = ptx::idesc_bf16_f32(128, 128, false);
  constexpr uint32_t kIdescS1 = ptx::idesc_bf16_f32(128, 64, false);
  // descriptor start-address fields count 16-byte units
  const uint64_t dq0 = ptx::smem_desc_sw128(sQ, 16);
  const uint64_t dk0 = ptx::smem_desc_sw128(sK, 16);
  uint32_t g = 0;
  bool alive = true;
  for (uint32_t nq = 0; alive; ++nq) {
    int count = 0;
    if (take_item_one<R>(sl, nq, &count, abort_flag, p.timeout_ns) < 0) break;
    const uint32_t qs = nq & 1u;
    if (!wait_one<R>(bar(kBarQFull + qs), (nq >> 1) & 1u, abort_flag, p.timeout_ns)) break;
    const uint64_t dq = dq0 + qs * (C::kQBytes >> 4);
    for (int e0 = 0; e0 < count; e0 += kChunkEnt, ++g) {
      const uint32_t ks = g % kKStages;
      if (!wait_one<R>(bar(kBarKFull + ks), (g / kKStages) & 1u, abort_flag, p.timeout_ns) ||
          (g > 0 && !wait_one<R>(bar(kBarSFree), (g - 1u) & 1u, abort_flag, p.timeout_ns))) {
        alive = false;
        break;
      }
      ptx::tc_fence_after();
      const uint64_t dk = dk0 + ks * (C::kStageBytes >> 4);
      const uint32_t d = tmem + C::kTmemS;
      const uint32_t idesc = count - e0 >= 2 ? kIdescS2 : kIdescS1;
#pragma unroll
      for (int hf = 0; hf < C::kHalves; ++hf) {  // 64 columns = 4 steps of 16: +32 bytes a step
        const uint64_t dqh = dq + hf * (C::kQHalfBytes >> 4), dkh = dk + hf * (C::kStageHalfBytes >> 4);
        ptx::mma_ss(d, dqh, dkh, idesc, hf > 0 ? 1u : 0u);
        ptx::mma_ss(d, dqh + 2, dkh + 2, idesc, 1u);
        ptx::mma_ss(d, dqh + 4, dkh + 4, idesc, 1u);
        ptx::mma_ss(d, dqh + 6, dkh + 6, idesc, 1u);
      }
      ptx::mma_commit(bar(kBarSFull));
      ptx::mma_commit(bar(kBarKFree + static_cast<int>(ks)));
    }
  }
  // Every MMA this thread issued must finish before TMEM is released.
  ptx::mma_commit(bar(kBarMmaFinal));
  wait_force<R>(bar(kBarMmaFinal), 0, abort_flag, p.timeout_ns);
}

// tcgen05 PV issuer, one thread, for the 64 columns of O from 64 hf.  Chunk g: once
// V(g) has landed and the softmax has written P(g), O (+)= P(g) V_g, 16 keys per MMA
// (the first MMA of a tile overwrites O), then one commit that (with the other
// column half's, at d = 128) frees V stage g % 2 and the P columns and tells the
// softmax warps that O holds chunk g.
template <int kD>
__device__ __forceinline__ void pv_issuer(const FwdParams& p, const Slot& sl, int hf, volatile int* abort_flag) {
  using C = FwdCfg<kD>;
  constexpr int R = C::kRoleRegion;
  const uint32_t sV = sl.sV + static_cast<uint32_t>(hf) * C::kStageHalfBytes, bars = sl.bars, tmem = sl.tmem;
  auto bar = [&](int i) { return bar_at(bars, i); };
  constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(128, 64, true);
  const uint64_t dv0 = ptx::smem_desc_sw128(sV, 0);
  const uint32_t d = tmem + C::kTmemO + 64u * static_cast<uint32_t>(hf);
  uint32_t g = 0;
  bool alive = true;
  for (uint32_t nq = 0; alive; ++nq) {
    int count = 0;
    if (take_item_one<R>(sl, nq, &count, abort_flag, p.timeout_ns) < 0) break;
    for (int e0 = 0; e0 < count; e0 += kChunkEnt, ++g) {
      const uint32_t vs = g % kVStages;
      if (!wait_one<R>(bar(kBarVFull + vs), (g / kVStages) & 1u, abort_flag, p.timeout_ns) ||
          !wait_one<R>(bar(kBarPFull), g & 1u, abort_flag, p.timeout_ns)) {
        alive = false;
        break;
      }
      ptx::tc_fence_after();
      const uint64_t dv = dv0 + vs * (C::kStageBytes >> 4);
      const uint32_t a = tmem + C::kTmemP;
      ptx::mma_ts(d, a, dv, kIdescPV, e0 == 0 ? 0u : 1u);  // 16 keys per MMA
      ptx::mma_ts(d, a + 8u, dv + (2048u >> 4), kIdescPV, 1u);
      ptx::mma_ts(d, a + 16u, dv + (4096u >> 4), kIdescPV, 1u);
      ptx::mma_ts(d, a + 24u, dv + (6144u >> 4), kIdescPV, 1u);
      if (count - e0 >= 2) {
        ptx::mma_ts(d, a + 32u, dv + (8192u >> 4), kIdescPV, 1u);
        ptx::mma_ts(d, a + 40u, dv + (10240u >> 4), kIdescPV, 1u);
        ptx::mma_ts(d, a + 48u, dv + (12288u >> 4), kIdescPV, 1u);
        ptx::mma_ts(d, a + 56u, dv + (14336u >> 4), kIdescPV, 1u);
      }
      ptx::mma_commit(bar(kBarVFree + static_cast<int>(vs)));
    }
  }
  ptx::mma_commit(bar(kBarMmaFinal + 1 + hf));
  wait_force<R>(bar(kBarMmaFinal + 1 + hf), 0, abort_flag, p.timeout_ns);
}

// What the epilogue of a finished tile needs; it runs in the first chunk of the next
// tile, after that chunk's wait for the tile's last PV.
struct TileDone {
  uint32_t k;  // the item's position in the slot's item sequence (its stage: k % ring)
  float m, l;  // the row's running max (log2 units) and sum
};

// Epilogue of a finished tile (its last PV is done): normalise O and store it with
// lse, or, for a chunk of a split tile, its partial record.  O rows go through the
// tile's own Q buffer (its S MMAs are complete) and one TMA store per warp and column
// half.  Out of line: it runs once per tile and would otherwise crowd the chunk loop's
// code and registers (only the softmax warps call it, so it is compiled to their
// budget).
template <int kD>
__device__ __noinline__ void tile_epilogue(const FwdParams& p, const TileDone& td, const ItemStage& st,
                                              const Slot& sl, uint32_t obase, int warp, int lane) {
  using C = FwdCfg<kD>;
  const int r = (warp & 3) * 32 + lane;
  const int half = r >> 6;
  const int tb = st.b;
  const WorkItem& tw = st.w;
  const int tqa = st.qa, tqb = st.qb;
  const int tbh = tb * p.H + tw.h;
  const float m = td.m, l = td.l;
  const bool row_active = half == 0 || tqb >= 0;
  const int qblk = half ? tqb : tqa;
  const size_t row = static_cast<size_t>(tbh) * p.L + static_cast<size_t>(qblk) * 64 + (r & 63);
  if (tw.split < 0) {
    if (row_active) {  // warp-uniform: a warp's 32 rows lie in one half
      // O rows through this warp's quarter of each column half of the tile's Q buffer
      // (128-byte swizzle: 16-byte chunk j of row r at r * 128 + ((j ^ (r % 8)) * 16)),
      // then one TMA store of the warp's 32 x 64 box per column half.
      const float inv = l > 0.f ? ptx::rcp_approx(l) : 0.f;
      const uint64_t inv2 = ptx::pack2(inv, inv);
      const uint32_t qs = td.k & 1u;
#pragma unroll
      for (int hf = 0; hf < C::kHalves; ++hf) {
        float o[64];
        {
          uint32_t raw[2][32];
          ptx::tmem_ld32(obase + 64u * hf, raw[0]);
          ptx::tmem_ld32(obase + 64u * hf + 32u, raw[1]);
          ptx::tmem_wait_ld();
          ptx::reg_fence(raw[0]);
          ptx::reg_fence(raw[1]);
#pragma unroll
          for (int c = 0; c < 64; ++c) o[c] = __uint_as_float(raw[c >> 5][c & 31]);
        }
        const uint32_t off = qs * C::kQBytes + hf * C::kQHalfBytes + (warp & 3) * kOStageBytes;
        uint8_t* stg = sl.q_generic + off;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          uint32_t w4[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float y0, y1;
            ptx::unpack2(ptx::fmul2(ptx::pack2(o[8 * j + 2 * q], o[8 * j + 2 * q + 1]), inv2), y0, y1);
            w4[q] = pack_bf16x2(y0, y1);
          }
          const uint4 u = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          *reinterpret_cast<uint4*>(stg + lane * 128 + ((j ^ (lane & 7)) << 4)) = u;
        }
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0)
          ptx::tma_store_2d(&p.tm_o, sl.sQ + off, 64 * hf, static_cast<int>(row - static_cast<size_t>(r & 31)));
      }
      if (lane == 0) ptx::bulk_commit_group();
      p.lse[row] = l > 0.f ? (m + ptx::lg2_approx(l)) * kLn2 : -INFINITY;
    }
    return;
  }
  // ---- split chunk: its partial record (unnormalised O, m, l)
  float* rec = p.partials + (static_cast<size_t>(tb) * p.n_records + tw.rec) * C::kRecFloats;
  float4* orow = reinterpret_cast<float4*>(rec + r * kD);
#pragma unroll
  for (int hf = 0; hf < C::kHalves; ++hf) {
    uint32_t raw[2][32];
    ptx::tmem_ld32(obase + 64u * hf, raw[0]);
    ptx::tmem_ld32(obase + 64u * hf + 32u, raw[1]);
    ptx::tmem_wait_ld();
    ptx::reg_fence(raw[0]);
    ptx::reg_fence(raw[1]);
#pragma unroll
    for (int v4 = 0; v4 < 16; ++v4) {
      const int c = v4 * 4;
      orow[hf * 16 + v4] = make_float4(__uint_as_float(raw[c >> 5][c & 31]), __uint_as_float(raw[c >> 5][(c & 31) + 1]),
                                       __uint_as_float(raw[c >> 5][(c & 31) + 2]),
                                       __uint_as_float(raw[c >> 5][(c & 31) + 3]));
    }
  }
  rec[kTileRows * kD + r] = l > 0.f ? m : -INFINITY;
  rec[kTileRows * kD + kTileRows + r] = l;
}

// Releases the Q buffer of the tile whose epilogue ran last: its O store (if any)
// has finished reading the staged rows.
__device__ __forceinline__ void release_q(const Slot& sl, uint32_t k, int lane) {
  if (lane == 0) ptx::bulk_wait_read_all();
  __syncwarp();
  if (lane == 0) ptx::mbar_arrive(bar_at(sl.bars, kBarQEmpty + static_cast<int>(k & 1u)));
}

// Masks the scores of padded keys (keys 0-31 in a, 32-63 in b).
__device__ __forceinline__ void mask_group(uint32_t (&a)[32], uint32_t (&b)[32], unsigned long long mk) {
  if (mk == ~0ull) return;
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    if (!((mk >> c) & 1ull)) a[c] = __float_as_uint(-INFINITY);
    if (!((mk >> (c + 32)) & 1ull)) b[c] = __float_as_uint(-INFINITY);
  }
}

// Rare paths, out of line so that the chunk loop's code stays small (softmax warps
// only; one instantiation per head dim, as the softmax register budget differs).
// Scores of padded keys of one 64-key group of this warp's rows set to -inf in TMEM.
template <int kD>
__device__ __noinline__ void mask_scores(uint32_t taddr, unsigned long long mk) {
  uint32_t a[32], b[32];
  ptx::tmem_ld32(taddr, a);
  ptx::tmem_ld32(taddr + 32u, b);
  ptx::tmem_wait_ld();
  ptx::reg_fence(a);
  ptx::reg_fence(b);
  mask_group(a, b, mk);
  ptx::tmem_st32(taddr, a);
  ptx::tmem_st32(taddr + 32u, b);
  ptx::tmem_wait_st();
}

// O (d columns of this warp's rows) scaled by alpha in TMEM; the caller's next
// tcgen05.wait::st covers the stores.
template <int kD>
__device__ __noinline__ void rescale_o(uint32_t obase, float alpha) {
#pragma unroll
  for (int hlf = 0; hlf < kD / 32; ++hlf) {
    uint32_t o[32];
    ptx::tmem_ld32(obase + 32u * hlf, o);
    ptx::tmem_wait_ld();
    ptx::reg_fence(o);
#pragma unroll
    for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
    ptx::tmem_st32(obase + 32u * hlf, o);
  }
}

// Zeros 32 TMEM columns of this warp's rows (the P of a group this half does not
// attend): eight four-column stores from one zero register, instead of 32 registers
// set to zero for one wide store.
__device__ __forceinline__ void tmem_zero32(uint32_t taddr) {
  const uint32_t z = 0u;
#pragma unroll
  for (int i = 0; i < 32; i += 4)
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %1, %1, %1};" ::"r"(taddr + i), "r"(z) : "memory");
}

__device__ __forceinline__ float group_max(const uint32_t (&a)[32], const uint32_t (&b)[32]) {
  auto f = [](uint32_t x) { return __uint_as_float(x); };
  // four independent chains of three-input maxima
  float mx[4] = {fmaxf(f(a[0]), f(a[1])), fmaxf(f(a[2]), f(a[3])), fmaxf(f(b[0]), f(b[1])),
                 fmaxf(f(b[2]), f(b[3]))};
#pragma unroll
  for (int c = 4; c < 32; c += 4) {
    mx[0] = ptx::fmax3(mx[0], f(a[c]), f(a[c + 1]));
    mx[1] = ptx::fmax3(mx[1], f(a[c + 2]), f(a[c + 3]));
    mx[2] = ptx::fmax3(mx[2], f(b[c]), f(b[c + 1]));
    mx[3] = ptx::fmax3(mx[3], f(b[c + 2]), f(b[c + 3]));
  }
  return fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
}

// p = 2^(s * scale_log2 - m) for the 64 scores of one group (keys 0-31 in a, 32-63 in
// b), packed to bf16 pairs in key order; returns the fp32 sum of p.  The scaling and
// the sums run on packed fp32 pairs (two lanes per instruction).
__device__ __forceinline__ float group_exp(uint32_t (&a)[32], const uint32_t (&b)[32], uint64_t sc2,
                                           uint64_t nm2) {
  uint64_t acc0 = 0ull, acc1 = 0ull;
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    const uint32_t* src = c < 16 ? a : b;
    const int cc = (c & 15) * 2;
    float x0, x1;
    ptx::unpack2(ptx::ffma2(ptx::pack2(__uint_as_float(src[cc]), __uint_as_float(src[cc + 1])), sc2, nm2), x0, x1);
    const float p0 = ptx::ex2_approx(x0), p1 = ptx::ex2_approx(x1);
    if (c & 1)
      acc1 = ptx::fadd2(acc1, ptx::pack2(p0, p1));
    else
      acc0 = ptx::fadd2(acc0, ptx::pack2(p0, p1));
    a[c] = pack_bf16x2(p0, p1);  // in place: a[c] was read at step c / 2
  }
  float s0, s1;
  ptx::unpack2(ptx::fadd2(acc0, acc1), s0, s1);
  return s0 + s1;
}

// The membership-and-padding mask of union entry e for this half of the tile: 0 when
// the half does not attend the key block, else the block's kept-key bits.
__device__ __forceinline__ unsigned long long entry_mask(const ItemStage& st, int e, int half) {
  return ((st.ent[e] >> (kEntBitsShift + half)) & 1u) ? st.kb[e] : 0ull;
}

// Token-level layouts: the keys of key block jb that query token i attends by the
// token rule (i global: all; else the band |i - j| <= w and the global keys).  The
// random blocks never get here (their entries need no mask).
__device__ __forceinline__ unsigned long long token_row_mask(const FwdParams& p, long long i, bool row_global,
                                                             int jb) {
  if (row_global) return ~0ull;
  const long long lo = i - p.tok_window - 64ll * jb, hi = i + p.tok_window - 64ll * jb;
  unsigned long long band = 0ull;
  if (hi >= 0 && lo <= 63) {
    const int l = lo < 0 ? 0 : static_cast<int>(lo), h = hi > 63 ? 63 : static_cast<int>(hi);
    band = (h == 63 ? ~0ull : ((1ull << (h + 1)) - 1ull)) & ~((1ull << l) - 1ull);
  }
  return band | p.tok_gbits[jb];
}

// The -inf mask of one attended 64-key group of this warp's rows (rare path, out of
// line): the key-padding bits, and at a token-level layout the row's token mask when
// the entry is flagged for this half.
template <int kD>
__device__ __noinline__ void mask_entry(const FwdParams& p, const ItemStage& st, uint32_t taddr, int e, int half,
                                       long long itok, bool row_global) {
  unsigned long long mk = entry_mask(st, e, half);
  if (p.tok_gbits != nullptr && ((st.ent[e] >> (kEntMaskShift + half)) & 1u))
    mk &= token_row_mask(p, itok, row_global, static_cast<int>(st.ent[e] & kEntColMask));
  mask_scores<kD>(taddr, mk);
}

// kTok: the layout is token-level (per-row masks in flagged entries; rows may then see
// chunks with no allowed key).
template <int kD, bool kTok>
__device__ __forceinline__ void softmax_role(const FwdParams& p, const Slot& sl, int warp, int lane,
                                             volatile int* abort_flag) {
  using C = FwdCfg<kD>;
  constexpr int R = C::kSoftRegion;
  const uint32_t bars = sl.bars, tmem = sl.tmem;
  auto bar = [&](int i) { return bar_at(bars, i); };
  const int r = (warp & 3) * 32 + lane;  // tile row == TMEM lane (warp w reaches lanes 32 (w % 4)..)
  const int half = r >> 6;               // warp-uniform: a warp's 32 rows lie in one half
  const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
  const uint32_t obase = tmem + lane_addr + C::kTmemO;
  const float sl2 = p.scale_log2;
  uint32_t g = 0;
  bool alive = true;
  // waits for PV(x): its commit freed V stage x % 2
  auto wait_pv = [&](uint32_t x) {
    return wait_warp<R>(bar(kBarVFree + static_cast<int>(x % kVStages)), (x / kVStages) & 1u, abort_flag,
                           p.timeout_ns);
  };

  TileDone pend{};
  bool have_pend = false;  // a finished tile waits for its epilogue
  bool q_pending = false;  // the tile of the last epilogue still holds its Q buffer
  uint32_t q_k = 0;
  for (uint32_t k = 0; alive; ++k) {
    const int t = take_item_warp<R>(sl, k, abort_flag, p.timeout_ns);
    if (t < 0) {
      if (t == kItemAbort) alive = false;
      break;
    }
    // the tile's union entries and their key-padding bits, staged by the K producer
    const ItemStage& st = sl.items[k % kItemRing];
    const int count = st.w.count;
    float m_run = -INFINITY, l_run = 0.f;
    // Per union entry, one bit each: this half attends the entry's key block and not all
    // of its keys are padded (att), and some of them are (part).  Lane x looks at entries
    // x and x + 32 (an item has at most 64), and the warp's ballots hold the bits.
    uint64_t att_bits, part_bits;
    {
      const unsigned long long k0 = lane < count ? entry_mask(st, lane, half) : 0ull;
      const unsigned long long k1 = lane + 32 < count ? entry_mask(st, lane + 32, half) : 0ull;
      att_bits = static_cast<uint64_t>(__ballot_sync(0xffffffffu, k0 != 0ull)) |
                 (static_cast<uint64_t>(__ballot_sync(0xffffffffu, k1 != 0ull)) << 32);
      part_bits = static_cast<uint64_t>(__ballot_sync(0xffffffffu, k0 + 1ull > 1ull)) |
                  (static_cast<uint64_t>(__ballot_sync(0xffffffffu, k1 + 1ull > 1ull)) << 32);
    }
    // token-level layouts: entries whose pairs this half's rows mask row by row
    long long itok = 0;
    bool row_global = false;
    if constexpr (kTok) {
      const uint32_t sh = kEntMaskShift + half;
      const bool t0 = lane < count && ((st.ent[lane] >> sh) & 1u);
      const bool t1 = lane + 32 < count && ((st.ent[lane + 32] >> sh) & 1u);
      part_bits |= static_cast<uint64_t>(__ballot_sync(0xffffffffu, t0)) |
                   (static_cast<uint64_t>(__ballot_sync(0xffffffffu, t1)) << 32);
      const int qblk = half ? st.qb : st.qa;
      if (qblk >= 0) {
        itok = 64ll * qblk + (r & 63);
        row_global = (p.tok_gbits[qblk] >> (r & 63)) & 1ull;
      }
    }
    for (int e0 = 0; e0 < count; e0 += kChunkEnt, ++g) {
      if (q_pending && e0 > 0) {  // one chunk after the epilogue: its O store has had time
        q_pending = false;
        release_q(sl, q_k, lane);
      }
      const bool two = count - e0 >= 2;
      if (!wait_warp<R>(bar(kBarSFull), g & 1u, abort_flag, p.timeout_ns)) {
        alive = false;
        break;
      }
      ptx::tc_fence_after();
      // All of S(g) into registers (loaded whatever the membership: a load under a
      // condition makes the compiler keep both versions of the registers alive), then
      // the S columns go straight back to the S issuer, so that S(g + 1) is computed
      // while this chunk's exponentials run.
      //
      // The running max m follows one rule: it is raised to the chunk max cm when cm
      // exceeds it by more than kRescaleLog2, so every p = 2^(s - m) stays at or below
      // 2^kRescaleLog2 and O is rescaled only when m moves that far.  A warp's rows
      // share membership and key bits, so the branches are warp-uniform.
      const uint32_t sbase = tmem + lane_addr + C::kTmemS;
      const bool att0 = (att_bits >> e0) & 1ull, att1 = (att_bits >> (e0 + 1)) & 1ull;
      const bool part = ((part_bits >> e0) & 3ull) != 0ull;
      if (part) {  // some keys of an attended block are padded or masked (rare): -inf in TMEM
        if constexpr (kTok) {
          if (att0) mask_entry<kD>(p, st, sbase, e0, half, itok, row_global);
          if (att1) mask_entry<kD>(p, st, sbase + 64u, e0 + 1, half, itok, row_global);
        } else {
          if (att0) mask_scores<kD>(sbase, entry_mask(st, e0, half));
          if (att1) mask_scores<kD>(sbase + 64u, entry_mask(st, e0 + 1, half));
        }
      }
      // P is written over the scores it came from (a0 and a1 hold P after the
      // exponentials), so that the TMEM stores read the registers the loads wrote
      uint32_t a0[32], b0[32], a1[32], b1[32];
      ptx::tmem_ld32(sbase, a0);
      ptx::tmem_ld32(sbase + 32u, b0);
      ptx::tmem_ld32(sbase + 64u, a1);
      ptx::tmem_ld32(sbase + 96u, b1);
      ptx::tmem_wait_ld();
      ptx::reg_fence(a0);
      ptx::reg_fence(b0);
      ptx::reg_fence(a1);
      ptx::reg_fence(b1);
      ptx::tc_fence_before();
      ptx::mbar_arrive(bar(kBarSFree));  // every thread
      // the chunk max over the keys this row attends (a padded key holds -inf; an
      // attended block keeps at least one key)
      float cm = -INFINITY;
      if (att0) cm = group_max(a0, b0);
      if (att1) cm = fmaxf(cm, group_max(a1, b1));
      const float cm2 = cm * sl2;  // scale > 0: the max of the scaled scores
      const float m_new = cm2 > m_run + kRescaleLog2 ? cm2 : m_run;
      // token level: a row with no allowed key so far (every score -inf) takes
      // p = 2^-inf = 0 (at block level an attended block keeps a key)
      const float m_off = (kTok && m_new == -INFINITY) ? 0.f : m_new;
      const uint64_t sc2 = ptx::pack2(sl2, sl2), nm2 = ptx::pack2(-m_off, -m_off);
      float psum = 0.f;
      if (att0) psum += group_exp(a0, b0, sc2, nm2);
      if (att1) psum += group_exp(a1, b1, sc2, nm2);
      const bool grew = m_new != m_run;
      const float alpha = grew ? ptx::ex2_approx(m_run - m_new) : 1.f;  // 2^-inf = 0
      const bool rescale = grew && l_run > 0.f;  // O holds this tile's earlier chunks
      // PV(g - 1) done: the P columns are free, and O holds the previous chunk (the
      // previous tile's last, at e0 == 0) for the epilogue or a rescale
      if (g > 0 && !wait_pv(g - 1)) {
        alive = false;
        break;
      }
      ptx::tc_fence_after();
      if (e0 == 0 && have_pend) {  // the previous tile's epilogue
        have_pend = false;
        tile_epilogue<kD>(p, pend, sl.items[pend.k % kItemRing], sl, obase, warp, lane);
        release_item_warp(sl, pend.k, lane);
        q_pending = true;
        q_k = pend.k;
      }
      if (__any_sync(0xffffffffu, rescale)) rescale_o<kD>(obase, alpha);
      const uint32_t pbase = tmem + lane_addr + C::kTmemP;
      if (att0) ptx::tmem_st32(pbase, a0); else tmem_zero32(pbase);
      if (two) {
        if (att1) ptx::tmem_st32(pbase + 32u, a1); else tmem_zero32(pbase + 32u);
      }
      l_run = l_run * alpha + psum;
      m_run = m_new;
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(bar(kBarPFull));  // every thread
    }
    if (!alive) break;
    if (q_pending) {  // a one-chunk tile: release before the next item's loads need the buffer
      q_pending = false;
      release_q(sl, q_k, lane);
    }
    pend = TileDone{k, m_run, l_run};
    have_pend = true;
  }
  if (alive && have_pend && wait_pv(g - 1)) {
    // the last tile: its last PV is done
    ptx::tc_fence_after();
    tile_epilogue<kD>(p, pend, sl.items[pend.k % kItemRing], sl, obase, warp, lane);
    release_item_warp(sl, pend.k, lane);
  }
  if (lane == 0) ptx::bulk_wait_all();  // O stores complete before the CTA exits
}

template <int kD, bool kTok>
__global__ void __launch_bounds__(FwdCfg<kD>::kThreads, 1) bsa_fwd_kernel(const __grid_constant__ FwdParams p) {
  using C = FwdCfg<kD>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + C::kSmemMisc);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kSlots; ++s) {
      const uint32_t bars = base + s * C::kSlotBytes + C::kSmemBar;
      for (int i = 0; i < kNumBars; ++i) {
        uint32_t count = 1;
        if (i >= kBarQEmpty && i < kBarQEmpty + 2) count = kWarpArrivals;
        if (i >= kBarVFree && i < kBarVFree + kVStages) count = C::kPvIssuers;
        if (i == kBarSFree || i == kBarPFull) count = kThreadArrivals;
        if (i >= kBarItemEmpty && i < kBarItemEmpty + kItemRing) count = C::kItemReaders;
        ptx::mbar_init(bars + 8u * i, count);
      }
    }
    misc[1] = 0;
    ptx::fence_barrier_init();
  }
  if (warp == C::kKProdWarp && lane == 0) {
    ptx::prefetch_tensormap(&p.tm_q);
    ptx::prefetch_tensormap(&p.tm_k);
    ptx::prefetch_tensormap(&p.tm_v);
    ptx::prefetch_tensormap(&p.tm_o);
  }
  if (warp == C::kSWarp) {
    ptx::tmem_alloc(ptx::smem_addr(const_cast<uint32_t*>(&misc[0])), kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  volatile int* abort_flag = reinterpret_cast<volatile int*>(&misc[1]);

  // the warp's slot: softmax warps 4 s..4 s + 3, then each role's kSlots warps in turn
  int slot = 0, hf = 0;
  if constexpr (C::kSlots == 2 && C::kPvIssuers == 1) {
    static_assert(C::kKProdWarp == 8 && C::kVProdWarp == 14, "two-slot warp map");
    slot = warp < 8 ? (warp >> 2) : (warp & 1);  // roles alternate slots from warp 8
  } else if (warp < C::kKProdWarp) {
    slot = warp >> 2;
  } else if (warp < C::kPvWarp) {
    slot = (warp - C::kKProdWarp) % C::kSlots;
  } else if (warp < C::kVProdWarp) {
    slot = (warp - C::kPvWarp) / C::kPvIssuers;
    hf = (warp - C::kPvWarp) % C::kPvIssuers;
  } else {
    slot = (warp - C::kVProdWarp) % C::kSlots;
  }
  Slot sl;
  sl.sQ = base + slot * C::kSlotBytes + C::kSmemQ;
  sl.sK = base + slot * C::kSlotBytes + C::kSmemK;
  sl.sV = base + slot * C::kSlotBytes + C::kSmemV;
  sl.bars = base + slot * C::kSlotBytes + C::kSmemBar;
  sl.q_generic = smem + slot * C::kSlotBytes + C::kSmemQ;
  sl.items = reinterpret_cast<ItemStage*>(smem + slot * C::kSlotBytes + C::kSmemItems);
  sl.tmem = misc[0] + static_cast<uint32_t>(slot) * C::kSlotCols;

  if (warp < C::kKProdWarp) {
    ptx::setmaxnreg_inc<C::kSoftmaxRegs>();
    softmax_role<kD, kTok>(p, sl, warp, lane, abort_flag);
  } else {
    ptx::setmaxnreg_dec<C::kOtherRegs>();
    if (warp < C::kSWarp) {
      k_producer<kD>(p, sl, lane, abort_flag);
    } else if (warp < C::kPvWarp) {
      if (lane == 0) s_issuer<kD>(p, sl, abort_flag);
    } else if (warp < C::kVProdWarp) {
      if (lane == 0) {
        if constexpr (C::kPvIssuers == 1)
          pv_issuer<kD>(p, sl, 0, abort_flag);
        else
          pv_issuer<kD>(p, sl, hf, abort_flag);
      }
    } else if (warp < C::kVProdWarp + C::kSlots) {
      v_producer<kD>(p, sl, lane, abort_flag);
    }
    __syncwarp();
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == C::kSWarp) ptx::tmem_dealloc(misc[0], kTmemCols);
}

// Merge of split tiles: one warp per (batch element, split tile, tile row).  The
// row's records were written by the forward's chunks of that tile: unnormalised O
// relative to the chunk's max m (log2 units), m (-inf: the row attended nothing in
// the chunk) and l.  O = sum_c 2^(m_c - M) O_c / sum_c 2^(m_c - M) l_c with M the
// largest m_c; lse = (M + log2 of that sum) ln 2.  The records are read in groups
// of eight with every load of a group in flight at once, and folded into a running
// (M, sum, O) -- the same rescaling the forward applies between chunks.  Lane x
// owns output columns (d / 32) x .. (d / 32) x + d / 32 - 1, so each record row is
// one coalesced line.
struct MergeParams {
  const float* partials;
  const SplitTile* splits;
  __nv_bfloat16* out;
  float* lse;
  int B, H, L, n_split, n_records;
};

template <int kD>
__global__ void __launch_bounds__(128) bsa_merge_kernel(const __grid_constant__ MergeParams p) {
  // launched as the forward's programmatic dependent: its launch overlaps the
  // forward's end, and this wait returns once the forward has finished and its
  // records are visible
  asm volatile("griddepcontrol.wait;" ::: "memory");
  constexpr int kGroup = 8;
  constexpr int kCols = kD / 32;  // output columns per lane: kCols * lane ..
  constexpr int kRec = FwdCfg<kD>::kRecFloats;
  using Vec = typename std::conditional<kCols == 2, float2, float4>::type;
  const int lane = threadIdx.x & 31;
  const int task = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int per_b = p.n_split * kTileRows;
  if (task >= p.B * per_b) return;
  const int b = task / per_b, rem = task - b * per_b;
  const int s = rem / kTileRows, r = rem - s * kTileRows;
  const SplitTile st = p.splits[s];
  const int qblk = (r >> 6) ? st.qb : st.qa;
  if (qblk < 0) return;  // the unused half of a single-block tile
  const size_t row = static_cast<size_t>(b * p.H + st.h) * p.L + static_cast<size_t>(qblk) * 64 + (r & 63);
  const float* base = p.partials + (static_cast<size_t>(b) * p.n_records + st.rec_base) * kRec;
  constexpr int kM = kTileRows * kD, kL = kTileRows * kD + kTileRows;
  const int nc = st.nchunks;
  float M = -INFINITY, lsum = 0.f;
  float acc[kCols] = {};
  for (int x0 = 0; x0 < nc; x0 += kGroup) {
    float mg[kGroup], lg[kGroup];
    Vec og[kGroup];
#pragma unroll
    for (int j = 0; j < kGroup; ++j) {
      const int x = x0 + j < nc ? x0 + j : nc - 1;  // a repeated record gets weight 0 below
      const float* rc = base + static_cast<size_t>(x) * kRec;
      mg[j] = __ldcg(rc + kM + r);
      lg[j] = __ldcg(rc + kL + r);
      og[j] = __ldcg(reinterpret_cast<const Vec*>(rc + r * kD) + lane);
    }
    float gm = -INFINITY;
#pragma unroll
    for (int j = 0; j < kGroup; ++j)
      if (x0 + j < nc) gm = fmaxf(gm, mg[j]);
    if (gm == -INFINITY) continue;  // no record of the group attended anything
    const float Mn = fmaxf(M, gm);
    const float a = M == -INFINITY ? 0.f : ptx::ex2_approx(M - Mn);
    lsum *= a;
#pragma unroll
    for (int c = 0; c < kCols; ++c) acc[c] *= a;
#pragma unroll
    for (int j = 0; j < kGroup; ++j) {
      // a record whose row attended nothing has m = -inf and O = 0: weight 0
      const float f = (x0 + j < nc && mg[j] != -INFINITY) ? ptx::ex2_approx(mg[j] - Mn) : 0.f;
      lsum += f * lg[j];
      const float* ov = reinterpret_cast<const float*>(&og[j]);
#pragma unroll
      for (int c = 0; c < kCols; ++c) acc[c] += f * ov[c];
    }
    M = Mn;
  }
  const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
  uint32_t packed[kCols / 2];
#pragma unroll
  for (int c = 0; c < kCols / 2; ++c) packed[c] = pack_bf16x2(acc[2 * c] * inv, acc[2 * c + 1] * inv);
  if constexpr (kCols == 2) {
    reinterpret_cast<uint32_t*>(p.out + row * kD)[lane] = packed[0];
  } else {
    reinterpret_cast<uint2*>(p.out + row * kD)[lane] = make_uint2(packed[0], packed[1]);
  }
  if (lane == 0) p.lse[row] = lsum > 0.f ? (M + log2f(lsum)) * kLn2 : -INFINITY;
}

// Per (b, key block): bit c set when key 64*j + c is kept by the padding mask.
__global__ void bsa_keybits_kernel(const uint8_t* __restrict__ key_mask,
                                   unsigned long long* __restrict__ bits, int B, int L, int nb) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= B * nb) return;
  const int b = idx / nb, j = idx - b * nb;
  const uint8_t* m = key_mask + static_cast<size_t>(b) * L + static_cast<size_t>(j) * 64;
  unsigned long long out = 0;
#pragma unroll 8
  for (int c = 0; c < 64; ++c)
    if (m[c] != 0) out |= 1ull << c;
  bits[idx] = out;
}

// A barrier nothing arrives on: exercises the bounded-wait path.
__global__ void bsa_debug_wait_kernel(unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ptx::mbar_init(ptx::smem_addr(&bar), 1);
    abort_flag = 0;
    ptx::fence_barrier_init();
  }
  __syncthreads();
  wait_warp(ptx::smem_addr(&bar), 0, &abort_flag, timeout_ns);
  __syncthreads();
}

// ------------------------------------------------------------ host helpers
namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

}  // namespace

// [rows, d] bf16 row-major tensor (d a multiple of 64), boxes of 64 columns x box_rows
// rows, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* ptr, uint64_t rows, uint32_t box_rows, int d) {
  auto fn = get_encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), rows};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_keybits(const uint8_t* key_mask, unsigned long long* bits, int B, int L, int nb,
                           cudaStream_t s) {
  const int n = B * nb;
  bsa_keybits_kernel<<<(n + 255) / 256, 256, 0, s>>>(key_mask, bits, B, L, nb);
  return cudaGetLastError();
}

namespace {

struct DeviceInfo {
  int sms = 0;
  bool sm100 = false;
  bool configured = false;
};
constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

int device_setup(int dev, DeviceInfo* out) {
  if (dev < 0 || dev >= kMaxDevices) return BSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.configured) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return BSA_ERR_CUDA;
    d.sm100 = (major == 10 && minor == 0);
    d.sms = sms;
    if (d.sm100 &&
        (cudaFuncSetAttribute(bsa_fwd_kernel<64, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(FwdCfg<64>::kSmemAlloc)) != cudaSuccess ||
         cudaFuncSetAttribute(bsa_fwd_kernel<64, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(FwdCfg<64>::kSmemAlloc)) != cudaSuccess ||
         cudaFuncSetAttribute(bsa_fwd_kernel<128, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(FwdCfg<128>::kSmemAlloc)) != cudaSuccess ||
         cudaFuncSetAttribute(bsa_fwd_kernel<128, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(FwdCfg<128>::kSmemAlloc)) != cudaSuccess))
      return BSA_ERR_CUDA;
    d.configured = true;
  }
  *out = d;
  return d.sm100 ? BSA_OK : BSA_ERR_UNSUPPORTED;
}

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// A forward call whose arguments have been checked: its workspace plan and device.
struct ForwardCall {
  WorkspacePlan plan;
  int dev = -1;
  DeviceInfo info;
};

// The checks a forward entry point makes before it enqueues anything, so that a
// call that fails leaves the GPU untouched: first the arguments (no CUDA call;
// fills in the workspace plan), then -- after the entry point has checked its
// scratch against the plan -- the device.
int validate_forward_args(const void* q, const void* k, const void* v, int B, int H, int L, int d,
                          const bsa_layout* lay, const void* out, const float* lse, float scale, ForwardCall* c) {
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr || lse == nullptr || lay == nullptr ||
      B < 1 || H < 1 || L < 1)
    return BSA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return BSA_ERR_UNSUPPORTED;
  if (H != lay->H || L != lay->L) return BSA_ERR_LAYOUT_MISMATCH;
  if (static_cast<int64_t>(B) * H * L > INT32_MAX - 64) return BSA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(lse, 4))
    return BSA_ERR_INVALID_ARG;
  if (!(scale == scale) || std::isinf(scale)) return BSA_ERR_INVALID_ARG;
  c->plan = plan_workspace(*lay, B, d);
  return BSA_OK;
}

int validate_forward_device(const bsa_layout* lay, ForwardCall* c) {
  if (lay->device < 0) return BSA_ERR_LAYOUT_MISMATCH;
  if (cudaGetDevice(&c->dev) != cudaSuccess) return BSA_ERR_CUDA;
  if (c->dev != lay->device) return BSA_ERR_LAYOUT_MISMATCH;
  return device_setup(c->dev, &c->info);
}

// Enqueues a checked forward call on workspace ws (at least c.plan.total bytes):
// clears the schedule counters, then the key bits (with a mask), the forward and
// the split-row merge.
int enqueue_forward(const ForwardCall& c, const void* q, const void* k, const void* v, int B, int H, int L, int d,
                    const bsa_layout* lay, const uint8_t* key_mask, float scale, void* out, float* lse,
                    uint8_t* ws, cudaStream_t s) {
  const WorkspacePlan& plan = c.plan;
  FwdParams prm{};
  const uint64_t rows = static_cast<uint64_t>(B) * H * L;
  if (!make_map(&prm.tm_q, q, rows, 64, d) || !make_map(&prm.tm_k, k, rows, 64, d) ||
      !make_map(&prm.tm_v, v, rows, 64, d) || !make_map(&prm.tm_o, out, rows, 32, d))
    return BSA_ERR_CUDA;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  prm.items = lay->d_items;
  prm.pair_q = lay->d_pair_q;
  prm.pair_ent = lay->d_pair_ent;
  prm.keybits = key_mask ? reinterpret_cast<const unsigned long long*>(ws + plan.keybits_off) : nullptr;
  prm.partials = reinterpret_cast<float*>(ws + plan.partials_off);
  prm.sched = reinterpret_cast<int*>(ws + plan.sched_off);
  prm.B = B;
  prm.H = H;
  prm.L = L;
  prm.nb = lay->nb;
  prm.items_per_batch = static_cast<int>(lay->items.size());
  prm.split_items = static_cast<int>(std::count_if(lay->items.begin(), lay->items.end(),
                                                   [](const WorkItem& it) { return it.split >= 0; }));
  prm.n_split = lay->n_split;
  prm.n_records = lay->n_records;
  prm.tok_gbits = lay->token ? lay->d_tok_gbits : nullptr;
  prm.tok_window = lay->tok_window;
  const float sc = scale > 0.f ? scale : 1.f / std::sqrt(static_cast<float>(d));
  prm.scale_log2 = sc * kLog2e;
  prm.timeout_ns = kDefaultTimeoutNs;

  // the schedule counters start at zero whatever an earlier call (or a device
  // error) left in the workspace
  if (cudaMemsetAsync(ws + plan.sched_off, 0, plan.sched_bytes, s) != cudaSuccess) return BSA_ERR_CUDA;
  if (key_mask != nullptr &&
      launch_keybits(key_mask, reinterpret_cast<unsigned long long*>(ws + plan.keybits_off), B, L, lay->nb, s) !=
          cudaSuccess)
    return BSA_ERR_CUDA;
  const int64_t total = static_cast<int64_t>(B) * prm.items_per_batch;
  // two slots per CTA at d = 64, one at d = 128; items are drawn dynamically
  const int slots_per_cta = d == 64 ? FwdCfg<64>::kSlots : FwdCfg<128>::kSlots;
  const int grid = static_cast<int>(std::min<int64_t>((total + slots_per_cta - 1) / slots_per_cta, c.info.sms));
  if (grid < 1) return BSA_OK;
  // How many batch elements early the split chunks go out: the last element's must
  // start while each slot still has at least one such chunk's length of work ahead.
  prm.split_lead = 0;
  prm.item_order = nullptr;
  if (prm.split_items > 0) {
    int64_t work = 0;  // chunks of one batch element
    int longest = 0;
    for (const WorkItem& it : lay->items) {
      const int ch = (it.count + kChunkEnt - 1) / kChunkEnt;
      work += ch;
      if (it.split >= 0) longest = std::max(longest, ch);
    }
    const int64_t slots = static_cast<int64_t>(slots_per_cta) * grid;
    while (prm.split_lead < B - 1 && (prm.split_lead + 1) * work < longest * slots) ++prm.split_lead;
    // One head's items are enough work to hand out its split chunks just before its
    // other tiles (the last head's chunks still start early enough): head by head.
    if (prm.split_lead == 0 && work >= static_cast<int64_t>(longest) * slots * H)
      prm.item_order = lay->d_head_order;
  }
  const bool tok = prm.tok_gbits != nullptr;
  if (d == 64 && !tok)
    bsa_fwd_kernel<64, false><<<grid, FwdCfg<64>::kThreads, FwdCfg<64>::kSmemAlloc, s>>>(prm);
  else if (d == 64)
    bsa_fwd_kernel<64, true><<<grid, FwdCfg<64>::kThreads, FwdCfg<64>::kSmemAlloc, s>>>(prm);
  else if (!tok)
    bsa_fwd_kernel<128, false><<<grid, FwdCfg<128>::kThreads, FwdCfg<128>::kSmemAlloc, s>>>(prm);
  else
    bsa_fwd_kernel<128, true><<<grid, FwdCfg<128>::kThreads, FwdCfg<128>::kSmemAlloc, s>>>(prm);
  if (cudaGetLastError() != cudaSuccess) return BSA_ERR_CUDA;
  if (lay->n_split > 0) {
    MergeParams mp{};
    mp.partials = prm.partials;
    mp.splits = lay->d_splits;
    mp.out = prm.out;
    mp.lse = lse;
    mp.B = B;
    mp.H = H;
    mp.L = L;
    mp.n_split = lay->n_split;
    mp.n_records = lay->n_records;
    const int64_t tasks = static_cast<int64_t>(B) * lay->n_split * kTileRows;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((tasks + 3) / 4));
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = d == 64 ? cudaLaunchKernelEx(&cfg, bsa_merge_kernel<64>, mp)
                                  : cudaLaunchKernelEx(&cfg, bsa_merge_kernel<128>, mp);
    if (e != cudaSuccess) return BSA_ERR_CUDA;
  }
  return BSA_OK;
}

}  // namespace

void free_device(bsa_layout* lay) {
  if (lay->device < 0) return;
  int cur = -1;
  const bool have_cur = cudaGetDevice(&cur) == cudaSuccess;
  if (cudaSetDevice(lay->device) == cudaSuccess) {
    cudaFree(lay->d_pair_q);
    cudaFree(lay->d_pair_ent);
    cudaFree(lay->d_items);
    cudaFree(lay->d_head_order);
    cudaFree(lay->d_splits);
    cudaFree(lay->d_kpair_q);
    cudaFree(lay->d_kpair_ent);
    cudaFree(lay->d_dq_items);
    cudaFree(lay->d_dkv_items);
    cudaFree(lay->d_dq_splits);
    cudaFree(lay->d_dkv_splits);
    cudaFree(lay->d_tok_gbits);
  }
  if (have_cur) cudaSetDevice(cur);
  lay->d_pair_q = nullptr;
  lay->d_pair_ent = nullptr;
  lay->d_items = nullptr;
  lay->d_head_order = nullptr;
  lay->d_splits = nullptr;
  lay->d_kpair_q = nullptr;
  lay->d_kpair_ent = nullptr;
  lay->d_dq_items = nullptr;
  lay->d_dkv_items = nullptr;
  lay->d_dq_splits = nullptr;
  lay->d_dkv_splits = nullptr;
  lay->d_tok_gbits = nullptr;
  lay->device = -1;
}

}  // namespace bsa

using namespace bsa;

extern "C" {

int bsa_layout_upload(bsa_layout* lay, void* stream) {
  if (lay == nullptr) return BSA_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return BSA_ERR_CUDA;
  free_device(lay);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // (device pointer, host data, bytes) of every table the kernels read
  struct Table {
    void** dst;
    const void* src;
    size_t bytes;
  };
  const Table tables[] = {
      {reinterpret_cast<void**>(&lay->d_pair_q), lay->pair_q.data(), lay->pair_q.size() * sizeof(int32_t)},
      {reinterpret_cast<void**>(&lay->d_pair_ent), lay->pair_ent.data(), lay->pair_ent.size() * sizeof(uint32_t)},
      {reinterpret_cast<void**>(&lay->d_items), lay->items.data(), lay->items.size() * sizeof(WorkItem)},
      {reinterpret_cast<void**>(&lay->d_head_order), lay->head_order.data(),
       lay->head_order.size() * sizeof(int32_t)},
      {reinterpret_cast<void**>(&lay->d_splits), lay->splits.data(), lay->splits.size() * sizeof(SplitTile)},
      {reinterpret_cast<void**>(&lay->d_kpair_q), lay->ktiles.pair_q.data(),
       lay->ktiles.pair_q.size() * sizeof(int32_t)},
      {reinterpret_cast<void**>(&lay->d_kpair_ent), lay->ktiles.pair_ent.data(),
       lay->ktiles.pair_ent.size() * sizeof(uint32_t)},
      {reinterpret_cast<void**>(&lay->d_dq_items), lay->dq_plan.items.data(),
       lay->dq_plan.items.size() * sizeof(BwdItem)},
      {reinterpret_cast<void**>(&lay->d_dkv_items), lay->dkv_plan.items.data(),
       lay->dkv_plan.items.size() * sizeof(BwdItem)},
      {reinterpret_cast<void**>(&lay->d_dq_splits), lay->dq_plan.splits.data(),
       lay->dq_plan.splits.size() * sizeof(SplitTile)},
      {reinterpret_cast<void**>(&lay->d_dkv_splits), lay->dkv_plan.splits.data(),
       lay->dkv_plan.splits.size() * sizeof(SplitTile)},
      {reinterpret_cast<void**>(&lay->d_tok_gbits), lay->tok_gbits.data(),
       lay->tok_gbits.size() * sizeof(uint64_t)},
  };
  lay->device = dev;
  for (const Table& t : tables) {
    if (cudaMalloc(t.dst, std::max<size_t>(t.bytes, 32)) != cudaSuccess) {
      free_device(lay);
      return BSA_ERR_OOM;
    }
  }
  for (const Table& t : tables) {
    if (t.bytes > 0 && cudaMemcpyAsync(*t.dst, t.src, t.bytes, cudaMemcpyHostToDevice, s) != cudaSuccess) {
      free_device(lay);
      return BSA_ERR_CUDA;
    }
  }
  if (cudaStreamSynchronize(s) != cudaSuccess) {
    free_device(lay);
    return BSA_ERR_CUDA;
  }
  return BSA_OK;
}

int bsa_forward(const void* q, const void* k, const void* v, int B, int H, int L, int d,
                const bsa_layout* lay, const uint8_t* key_mask, float scale, void* out, float* lse,
                void* workspace, size_t workspace_bytes, void* stream) {
  ForwardCall c;
  int st = validate_forward_args(q, k, v, B, H, L, d, lay, out, lse, scale, &c);
  if (st != BSA_OK) return st;
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < c.plan.total) return BSA_ERR_WORKSPACE;
  st = validate_forward_device(lay, &c);
  if (st != BSA_OK) return st;
  return enqueue_forward(c, q, k, v, B, H, L, d, lay, key_mask, scale, out, lse,
                         static_cast<uint8_t*>(workspace), static_cast<cudaStream_t>(stream));
}

int bsa_sync_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return BSA_ERR_CUDA;
  int st = 0;
  if (cudaMemcpyFromSymbol(&st, g_bsa_status, sizeof(int)) != cudaSuccess) return BSA_ERR_CUDA;
  if (st != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_bsa_status, &zero, sizeof(int)) != cudaSuccess) return BSA_ERR_CUDA;
  }
  const int st_bwd = bwd_take_status();  // the backward kernels' status word
  const int st_proj = proj_take_status();  // the projection kernels' status word
  return st != 0 ? st : (st_bwd != 0 ? st_bwd : st_proj);
}

int bsa_debug_wait_timeout(uint64_t timeout_ns, void* stream) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return BSA_ERR_CUDA;
  DeviceInfo info;
  const int st = device_setup(dev, &info);
  if (st != BSA_OK) return st;
  const unsigned long long t =
      std::min<unsigned long long>(std::max<unsigned long long>(timeout_ns, 1000ull), 2000000000ull);
  bsa_debug_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(t);
  return cudaGetLastError() == cudaSuccess ? BSA_OK : BSA_ERR_CUDA;
}

}  // extern "C"

// ------------------------------------------------------------ allocation-free entry
// Scratch of bsa_forward_static_ws: a file-scope device array, so that callers who
// cannot allocate device memory can still run the forward.  In host code its name
// is only a stand-in; the device address is looked up per device below.
static __device__ __align__(256) unsigned char g_bsa_static_ws[BSA_STATIC_WORKSPACE_BYTES];

namespace {
// Per device, the array's device address once a lookup has succeeded (a failed
// lookup is retried on the next call).  Not refreshed after cudaDeviceReset.
void* g_static_ws_addr[kMaxDevices];
std::mutex g_static_ws_mu;
}  // namespace

extern "C" int bsa_forward_static_ws(const void* q, const void* k, const void* v, int B, int H, int L,
                                     int d, const bsa_layout* lay, const uint8_t* key_mask, float scale,
                                     void* out, float* lse, void* stream) {
  ForwardCall c;
  int st = validate_forward_args(q, k, v, B, H, L, d, lay, out, lse, scale, &c);
  if (st != BSA_OK) return st;
  if (c.plan.total > BSA_STATIC_WORKSPACE_BYTES) return BSA_ERR_STATIC_WORKSPACE;
  st = validate_forward_device(lay, &c);
  if (st != BSA_OK) return st;
  void* addr = nullptr;
  {
    // with this device current: the array's address on it
    std::lock_guard<std::mutex> lk(g_static_ws_mu);
    if (g_static_ws_addr[c.dev] == nullptr) {
      void* found = nullptr;
      if (cudaGetSymbolAddress(&found, g_bsa_static_ws) != cudaSuccess || found == nullptr) return BSA_ERR_CUDA;
      g_static_ws_addr[c.dev] = found;
    }
    addr = g_static_ws_addr[c.dev];
  }
  return enqueue_forward(c, q, k, v, B, H, L, d, lay, key_mask, scale, out, lse, static_cast<uint8_t*>(addr),
                         static_cast<cudaStream_t>(stream));
}
