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
// Kernel design (one persistent CTA per SM, 352 threads):
//   warp 8      TMA producer: Q tile (2 x 64 rows), then K and V of two key blocks per
//               chunk of the tile's key-block union into a K ring (released when the
//               chunk's S is done) and a deeper V ring (released after its PV).
//   warp 9      tcgen05 S issuer: S = Q K^T (M=128, N=64|128, K=64) into one of three
//               TMEM S buffers.
//   warp 10     tcgen05 PV issuer: per key block O_x += P_x V_x (A = P from TMEM, M=128,
//               N=64, K=64) into that block's own accumulator.  Two issuing threads
//               keep the tensor pipe fed: each tcgen05 instruction, barrier wait and
//               commit blocks its thread, and d = 64 makes every MMA short.
//   warps 0-7   softmax + epilogue, two warpgroups.  Warpgroup x (warps 4x..4x+3)
//               handles key block x of every chunk: thread (warp w, lane l) owns tile
//               row r = 32 (w % 4) + l = TMEM lane r.  Each warpgroup keeps its own
//               running max m_x and sum l_x (fp32) and its own O_x accumulator, writes
//               P_x (bf16) over its half of S, and rescales O_x when m_x grows by more
//               than kRescaleLog2.  The epilogue merges (m_A, l_A, O_A) and
//               (m_B, l_B, O_B); each warpgroup finishes 32 of the 64 output columns.
// A tile is two query blocks of the same (b, h) over the sorted union of their rows;
// entries carry per-block membership bits so each half of the tile sees exactly its
// own row, and a warp whose half does not attend a block skips its exponentials.
// Long unions (global rows) are cut into chunks processed by different CTAs; each
// chunk stores a partial (O, m, l) and the last one to arrive merges them.
// Every wait is bounded (globaltimer); on expiry the CTA records
// BSA_ERR_DEVICE_TIMEOUT, drains its own copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <mutex>

#include "bsa_internal.h"
#include "sm100_ptx.cuh"

namespace bsa {

constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;  // S issuer; also allocates and frees TMEM
constexpr int kPvWarp = 10;
constexpr int kThreads = 352;
constexpr int kKStages = 3;  // == kSBufs: K stage g % 3 is free once S(g) is done
constexpr int kVStages = 5;  // V stage g % 5 is free once PV(g) is done
constexpr uint32_t kBlkBytes = 64 * 128;         // one 64 x 64 bf16 block
constexpr uint32_t kQBytes = 2 * kBlkBytes;      // 128-row Q tile
constexpr uint32_t kStageBytes = 2 * kBlkBytes;  // two key blocks
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSBufs = 3;    // S buffers of 128 columns at [0,128), [128,256), [256,384)
constexpr uint32_t kTmemS = 0;
constexpr uint32_t kTmemO = 384;  // O_A [384,448), O_B [448,512)
constexpr float kRescaleLog2 = 8.0f;
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLog2e = 1.44269504088896340736f;
constexpr uint32_t kMaxSpin = 1u << 24;
constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;
constexpr uint32_t kWaitSleepNs = 20000;  // upper bound on one sleep inside a barrier wait

// shared memory map (offsets from a 1024-aligned base)
constexpr uint32_t kSmemQ = 0;
constexpr uint32_t kSmemK = kSmemQ + 2 * kQBytes;
constexpr uint32_t kSmemV = kSmemK + kKStages * kStageBytes;
constexpr uint32_t kSmemBar = kSmemV + kVStages * kStageBytes;
enum : int {
  kBarQFull = 0,
  kBarQEmpty = 2,
  kBarKFull = 4,                          // [K stage] K of the stage landed (TMA)
  kBarVFull = kBarKFull + kKStages,       // [V stage] V of the stage landed (TMA)
  kBarVFree = kBarVFull + kVStages,       // [V stage] MMA commit after the chunk's PV: the V
                                          // stage is reusable and both O_x hold that chunk
  kBarSFull = kBarVFree + kVStages,       // [S buffer] MMA commit after S: S readable, and
                                          // the K stage of the same index reusable
  kBarPFull = kBarSFull + kSBufs,         // [S buffer] both warpgroups' P written, 256 arrivals
  kBarOFree = kBarPFull + kSBufs,         // 256 arrivals once the epilogue has read O
  kBarMmaFinal = kBarOFree + 1,           // [2 issuers]
  kBarEpi = kBarMmaFinal + 2,        // 256 softmax threads, epilogue rendezvous
  kNumBars = kBarEpi + 1
};
constexpr uint32_t kSmemMisc = kSmemBar + 8 * kNumBars;
constexpr uint32_t kSmemXch = (kSmemMisc + 16 + 15) & ~15u;  // [2 tile parity][2 wg][2 (m,l)][128] fp32
constexpr uint32_t kSmemUsed = kSmemXch + 2 * 2 * 2 * kTileRows * 4;
constexpr uint32_t kSmemAlloc = kSmemUsed + 1024;  // slack for 1024-byte alignment
static_assert(kSmemAlloc <= 227 * 1024, "shared memory budget");

struct FwdParams {
  CUtensorMap tm_q, tm_k, tm_v;
  __nv_bfloat16* out;
  float* lse;
  const WorkItem* items;
  const int32_t* pair_q;
  const uint32_t* pair_ent;
  const unsigned long long* keybits;  // [B, nb] or null
  float* partials;
  int* tickets;
  int B, H, L, nb, items_per_batch, n_split, n_records;
  float scale_log2;
  unsigned long long timeout_ns;
};

__device__ int g_bsa_status;

// ------------------------------------------------------------ bounded waits
__device__ __noinline__ bool wait_slow(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                       uint64_t timeout_ns, bool honor_abort) {
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    // sleeping in the barrier instead of spinning leaves issue slots to the
    // warps that share this SM sub-partition
    if (ptx::mbar_try_wait_sleep(bar, parity, kWaitSleepNs)) return true;
    if ((it & 15u) == 0) {
      if (honor_abort && *abort_flag) return false;
      if (ptx::globaltimer_ns() - t0 > timeout_ns || it > kMaxSpin) {
        *abort_flag = 1;
        atomicCAS(&g_bsa_status, 0, static_cast<int>(BSA_ERR_DEVICE_TIMEOUT));
        return false;
      }
    }
  }
}

// Whole-warp wait; the result is warp-uniform.
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t timeout_ns) {
  bool ok = ptx::mbar_try_wait(bar, parity);
  if (__all_sync(0xffffffffu, ok)) return true;
  ok = wait_slow(bar, parity, abort_flag, timeout_ns, true);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void wait_force(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                           uint64_t timeout_ns) {
  if (!ptx::mbar_try_wait(bar, parity)) wait_slow(bar, parity, abort_flag, timeout_ns, false);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// ------------------------------------------------------------ roles
// Single-thread wait (the TMA and MMA roles run on one elected lane).
__device__ __forceinline__ bool wait_one(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         uint64_t timeout_ns) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  return wait_slow(bar, parity, abort_flag, timeout_ns, true);
}

// TMA producer, one thread: Q tile, then for each chunk c its K into K stage c % 3
// (once S(c - 3) is done) and its V into V stage c % 5 (once PV(c - 5) is done).
__device__ __forceinline__ void producer_role(const FwdParams& p, uint32_t sQ, uint32_t sK,
                                              uint32_t sV, uint32_t bars, volatile int* abort_flag) {
  static_assert(kKStages == static_cast<int>(kSBufs), "K stages are released by the S-full commits");
  auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
  const uint64_t pol_q = ptx::policy_evict_first();
  const uint64_t pol_kv = ptx::policy_evict_last();
  const int total = p.B * p.items_per_batch;
  uint32_t nq = 0, nk = 0, nv = 0;  // Q tiles, K chunks, V chunks issued
  bool alive = true;
  for (int t = blockIdx.x; alive && t < total; t += gridDim.x) {
    const int b = t / p.items_per_batch;
    const WorkItem w = p.items[t - b * p.items_per_batch];
    const int row0 = (b * p.H + w.h) * p.L;
    const int qa = p.pair_q[2 * w.pair], qb = p.pair_q[2 * w.pair + 1];
    const uint32_t qs = nq & 1u;
    if (!wait_one(bar(kBarQEmpty + qs), ((nq >> 1) & 1u) ^ 1u, abort_flag, p.timeout_ns)) {
      alive = false;
      break;
    }
    ptx::mbar_arrive_expect_tx(bar(kBarQFull + qs), kQBytes);
    ptx::tma_load_2d(sQ + qs * kQBytes, &p.tm_q, bar(kBarQFull + qs), 0, row0 + qa * 64, pol_q);
    ptx::tma_load_2d(sQ + qs * kQBytes + kBlkBytes, &p.tm_q, bar(kBarQFull + qs), 0,
                     row0 + (qb >= 0 ? qb : qa) * 64, pol_q);
    ++nq;
    const uint32_t* ent = p.pair_ent + w.start;
    for (int e = 0; e < w.count; e += 2) {
      const int j0 = static_cast<int>(ent[e] & kEntColMask);
      const bool two = e + 1 < w.count;
      const int j1 = two ? static_cast<int>(ent[e + 1] & kEntColMask) : 0;
      const uint32_t bytes = two ? 2 * kBlkBytes : kBlkBytes;
      const uint32_t ks = nk % kKStages;
      if (!wait_one(bar(kBarSFull + ks), ((nk / kKStages) & 1u) ^ 1u, abort_flag, p.timeout_ns)) {
        alive = false;
        break;
      }
      const uint32_t dk = sK + ks * kStageBytes;
      ptx::mbar_arrive_expect_tx(bar(kBarKFull + ks), bytes);
      ptx::tma_load_2d(dk, &p.tm_k, bar(kBarKFull + ks), 0, row0 + j0 * 64, pol_kv);
      if (two) ptx::tma_load_2d(dk + kBlkBytes, &p.tm_k, bar(kBarKFull + ks), 0, row0 + j1 * 64, pol_kv);
      ++nk;
      const uint32_t vs = nv % kVStages;
      if (!wait_one(bar(kBarVFree + vs), ((nv / kVStages) & 1u) ^ 1u, abort_flag, p.timeout_ns)) {
        alive = false;
        break;
      }
      const uint32_t dv = sV + vs * kStageBytes;
      ptx::mbar_arrive_expect_tx(bar(kBarVFull + vs), bytes);
      ptx::tma_load_2d(dv, &p.tm_v, bar(kBarVFull + vs), 0, row0 + j0 * 64, pol_kv);
      if (two) ptx::tma_load_2d(dv + kBlkBytes, &p.tm_v, bar(kBarVFull + vs), 0, row0 + j1 * 64, pol_kv);
      ++nv;
    }
  }
  if (!alive) {
    // Aborted: let every copy this thread issued land before the CTA exits.  The
    // last issue into ring slot s had index s + R * floor((n - 1 - s) / R).
    auto drain = [&](int first_bar, uint32_t n, uint32_t ring) {
      for (uint32_t s = 0; s < ring; ++s) {
        if (n > s) {
          const uint32_t last = s + ring * ((n - 1u - s) / ring);
          wait_force(bar(first_bar + static_cast<int>(s)), (last / ring) & 1u, abort_flag, p.timeout_ns);
        }
      }
    };
    drain(kBarQFull, nq, 2u);
    drain(kBarKFull, nk, static_cast<uint32_t>(kKStages));
    drain(kBarVFull, nv, static_cast<uint32_t>(kVStages));
  }
}

// tcgen05 S issuer, one thread.  S(g) = Q K_g^T into S buffer g % 3 once K(g) has
// landed and PV(g - 3), the previous reader of that buffer, is done.  Its commit
// also releases K stage g % 3 to the producer.
__device__ __forceinline__ void s_issuer(const FwdParams& p, uint32_t sQ, uint32_t sK, uint32_t bars,
                                         uint32_t tmem, volatile int* abort_flag) {
  auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
  constexpr uint32_t kIdescS128 = ptx::idesc_bf16_f32(128, 128, false);
  constexpr uint32_t kIdescS64 = ptx::idesc_bf16_f32(128, 64, false);
  // descriptor start-address fields count 16-byte units
  const uint64_t dq0 = ptx::smem_desc_sw128(sQ, 16);
  const uint64_t dk0 = ptx::smem_desc_sw128(sK, 16);
  const int total = p.B * p.items_per_batch;
  uint32_t g = 0, nq = 0;
  bool alive = true;
  for (int t = blockIdx.x; alive && t < total; t += gridDim.x, ++nq) {
    const int b = t / p.items_per_batch;
    const WorkItem w = p.items[t - b * p.items_per_batch];
    const uint32_t qs = nq & 1u;
    if (!wait_one(bar(kBarQFull + qs), (nq >> 1) & 1u, abort_flag, p.timeout_ns)) break;
    const uint64_t dq = dq0 + qs * (kQBytes >> 4);
    const int nch = (w.count + 1) >> 1;
    for (int n = 0; n < nch; ++n, ++g) {
      const uint32_t ks = g % kKStages;
      if (!wait_one(bar(kBarKFull + ks), (g / kKStages) & 1u, abort_flag, p.timeout_ns)) {
        alive = false;
        break;
      }
      if (g >= kSBufs) {
        const uint32_t gp = g - kSBufs;
        if (!wait_one(bar(kBarVFree + gp % kVStages), (gp / kVStages) & 1u, abort_flag, p.timeout_ns)) {
          alive = false;
          break;
        }
      }
      ptx::tc_fence_after();
      const bool two = 2 * n + 1 < w.count;
      const uint64_t dk = dk0 + ks * (kStageBytes >> 4);
      const uint32_t d = tmem + kTmemS + (g % kSBufs) * 128u;
      const uint32_t id = two ? kIdescS128 : kIdescS64;
      ptx::mma_ss(d, dq, dk, id, 0u);  // head dim 64 = 4 x 16: +32 bytes per step
      ptx::mma_ss(d, dq + 2, dk + 2, id, 1u);
      ptx::mma_ss(d, dq + 4, dk + 4, id, 1u);
      ptx::mma_ss(d, dq + 6, dk + 6, id, 1u);
      ptx::mma_commit(bar(kBarSFull + g % kSBufs));
      if (n == nch - 1) ptx::mma_commit(bar(kBarQEmpty + qs));
    }
  }
  // Every MMA this thread issued must finish before TMEM is released.
  ptx::mma_commit(bar(kBarMmaFinal));
  wait_force(bar(kBarMmaFinal), 0, abort_flag, p.timeout_ns);
}

// tcgen05 PV issuer, one thread.  Chunk g: once V(g) has landed and both warpgroups
// have written P(g), O_x (+)= P_x V_x for the chunk's key blocks, then one commit
// that frees V stage g % 5, tells the S issuer S buffer g % 3 is free, and tells the
// softmax warps that O holds chunk g.  A tile's first PV waits until the previous
// tile's epilogue has read O.
__device__ __forceinline__ void pv_issuer(const FwdParams& p, uint32_t sV, uint32_t bars, uint32_t tmem,
                                          volatile int* abort_flag) {
  auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
  constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(128, 64, true);
  const uint64_t dv0 = ptx::smem_desc_sw128(sV, 0);
  const int total = p.B * p.items_per_batch;
  uint32_t g = 0, nq = 0;
  bool alive = true;
  for (int t = blockIdx.x; alive && t < total; t += gridDim.x, ++nq) {
    const int b = t / p.items_per_batch;
    const WorkItem w = p.items[t - b * p.items_per_batch];
    const int nch = (w.count + 1) >> 1;
    for (int n = 0; n < nch; ++n, ++g) {
      if (n == 0 && !wait_one(bar(kBarOFree), (nq & 1u) ^ 1u, abort_flag, p.timeout_ns)) {
        alive = false;
        break;
      }
      const uint32_t vs = g % kVStages, sb = g % kSBufs;
      if (!wait_one(bar(kBarVFull + vs), (g / kVStages) & 1u, abort_flag, p.timeout_ns) ||
          !wait_one(bar(kBarPFull + sb), (g / kSBufs) & 1u, abort_flag, p.timeout_ns)) {
        alive = false;
        break;
      }
      ptx::tc_fence_after();
      const bool two = 2 * n + 1 < w.count;
      const uint32_t acc0 = n == 0 ? 0u : 1u;
      const uint64_t dv = dv0 + vs * (kStageBytes >> 4);
      for (uint32_t x = 0; x < (two ? 2u : 1u); ++x) {
        const uint32_t d = tmem + kTmemO + x * 64u;
        const uint32_t a = tmem + kTmemS + sb * 128u + x * 64u;
        const uint64_t bx = dv + x * (kBlkBytes >> 4);
        ptx::mma_ts(d, a, bx, kIdescPV, acc0);  // 16 keys per MMA
        ptx::mma_ts(d, a + 8u, bx + (2048u >> 4), kIdescPV, 1u);
        ptx::mma_ts(d, a + 16u, bx + (4096u >> 4), kIdescPV, 1u);
        ptx::mma_ts(d, a + 24u, bx + (6144u >> 4), kIdescPV, 1u);
      }
      ptx::mma_commit(bar(kBarVFree + vs));
    }
  }
  ptx::mma_commit(bar(kBarMmaFinal + 1));
  wait_force(bar(kBarMmaFinal + 1), 0, abort_flag, p.timeout_ns);
}

__device__ __forceinline__ void mask_cols(float (&s)[64], unsigned long long mk) {
  if (mk == ~0ull) return;
#pragma unroll
  for (int c = 0; c < 64; ++c)
    if (!((mk >> c) & 1ull)) s[c] = -INFINITY;
}

// What the epilogue of a finished tile needs; it runs one chunk later (after the
// first chunk of the next tile) so the wait for the tile's last PV is hidden.  The
// epilogue's 256-thread rendezvous is an mbarrier with a bounded wait (a plain
// bar.sync could not give up if another softmax warp had already aborted).
struct TileDone {
  int t;            // work item index (its fields are reloaded by the epilogue)
  uint32_t g_last;  // global index of the tile's last chunk
  uint32_t nt;      // tile count of this CTA when the tile started
  float m, l;       // this warpgroup's running max (log2 units) and sum for the row
};

// Epilogue of a finished tile: merge (m_A, l_A, O_A) with (m_B, l_B, O_B), store O
// and lse (or the split chunk's partial record, merging when last).  Kept out of
// line: it runs once per tile and would otherwise crowd the chunk loop's registers.
__device__ __noinline__ bool tile_epilogue(const FwdParams& p, const TileDone& td, uint32_t bars,
                                           uint32_t obase, int warp, int lane, volatile int* abort_flag,
                                           volatile uint32_t* last_flag, float* xch, uint32_t* n_epi) {
  auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
  const int wg = warp >> 2;
  const int r = (warp & 3) * 32 + lane;
  const int half = r >> 6;
  auto epi_sync = [&]() -> bool {
    ptx::mbar_arrive(bar(kBarEpi));
    const bool ok = wait_warp(bar(kBarEpi), *n_epi & 1u, abort_flag, p.timeout_ns);
    ++*n_epi;
    return ok;
  };
  {
    const int tb = td.t / p.items_per_batch;
    const WorkItem tw = p.items[td.t - tb * p.items_per_batch];
    const int tqa = p.pair_q[2 * tw.pair], tqb = p.pair_q[2 * tw.pair + 1];
    const int tbh = tb * p.H + tw.h;
    // PV of the tile's last chunk.  Unambiguous phase: S(g_last) was seen, and it
    // was issued after PV(g_last - 3) was done; PV(g_last + kVStages) needs P this
    // warpgroup has not produced.
    if (!wait_warp(bar(kBarVFree + static_cast<int>(td.g_last % kVStages)), (td.g_last / kVStages) & 1u,
                   abort_flag, p.timeout_ns))
      return false;
    // (m, l) exchange, double-buffered by tile parity: a warpgroup that runs ahead
    // into the next tile cannot overwrite values the other has not read yet.
    float* xt = xch + (td.nt & 1u) * (2 * 2 * kTileRows);
    xt[(wg * 2 + 0) * kTileRows + r] = td.m;
    xt[(wg * 2 + 1) * kTileRows + r] = td.l;
    if (!epi_sync()) return false;
    ptx::tc_fence_after();
    const float m_o = xt[((1 - wg) * 2 + 0) * kTileRows + r];
    const float l_o = xt[((1 - wg) * 2 + 1) * kTileRows + r];
    const float mA = wg == 0 ? td.m : m_o, lA = wg == 0 ? td.l : l_o;
    const float mB = wg == 0 ? m_o : td.m, lB = wg == 0 ? l_o : td.l;
    const float m = fmaxf(mA, mB);
    const bool useA = lA > 0.f, useB = lB > 0.f;  // an unused O_x may hold stale values
    const float fA = useA ? ptx::ex2_approx(mA - m) : 0.f;
    const float fB = useB ? ptx::ex2_approx(mB - m) : 0.f;
    const float l = lA * fA + lB * fB;
    // this warpgroup finishes output columns [32 wg, 32 wg + 32)
    uint32_t oa[32], ob[32];
    ptx::tmem_ld32(obase + static_cast<uint32_t>(wg) * 32u, oa);
    ptx::tmem_ld32(obase + 64u + static_cast<uint32_t>(wg) * 32u, ob);
    ptx::tmem_wait_ld();
    ptx::reg_fence(oa);
    ptx::reg_fence(ob);
    ptx::tc_fence_before();
    ptx::mbar_arrive(bar(kBarOFree));  // O may now be overwritten by the next tile
    float o[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      const float a = useA ? __uint_as_float(oa[c]) * fA : 0.f;
      const float bb = useB ? __uint_as_float(ob[c]) * fB : 0.f;
      o[c] = a + bb;
    }
    const bool row_active = half == 0 || tqb >= 0;
    const int qblk = half ? tqb : tqa;
    const size_t row = static_cast<size_t>(tbh) * p.L + static_cast<size_t>(qblk) * 64 + (r & 63);
    if (tw.split < 0) {
      if (row_active) {
        const float inv = l > 0.f ? 1.f / l : 0.f;
        uint4* dst = reinterpret_cast<uint4*>(p.out + row * 64 + wg * 32);
#pragma unroll
        for (int v8 = 0; v8 < 4; ++v8) {
          uint4 u;
          u.x = pack_bf16x2(o[v8 * 8 + 0] * inv, o[v8 * 8 + 1] * inv);
          u.y = pack_bf16x2(o[v8 * 8 + 2] * inv, o[v8 * 8 + 3] * inv);
          u.z = pack_bf16x2(o[v8 * 8 + 4] * inv, o[v8 * 8 + 5] * inv);
          u.w = pack_bf16x2(o[v8 * 8 + 6] * inv, o[v8 * 8 + 7] * inv);
          dst[v8] = u;
        }
        if (wg == 0) p.lse[row] = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
      }
      return true;
    }
    // ---- split chunk: store the partial record, then the last arriver merges
    float* rec = p.partials + (static_cast<size_t>(tb) * p.n_records + tw.rec) * kRecFloats;
    float4* orow = reinterpret_cast<float4*>(rec + r * 64 + wg * 32);
#pragma unroll
    for (int v4 = 0; v4 < 8; ++v4)
      orow[v4] = make_float4(o[v4 * 4 + 0], o[v4 * 4 + 1], o[v4 * 4 + 2], o[v4 * 4 + 3]);
    if (wg == 0) {
      rec[kTileRows * 64 + r] = l > 0.f ? m : -INFINITY;
      rec[kTileRows * 64 + kTileRows + r] = l;
    }
    __threadfence();
    if (!epi_sync()) return false;
    int* ticket = p.tickets + static_cast<size_t>(tb) * p.n_split + tw.split;
    if (warp == 0 && lane == 0) *last_flag = (atomicAdd(ticket, 1) == tw.nchunks - 1) ? 1u : 0u;
    if (!epi_sync()) return false;
    if (!*last_flag) return true;
    __threadfence();
    if (row_active) {
      const float* base = p.partials + (static_cast<size_t>(tb) * p.n_records + tw.rec_base) * kRecFloats;
      float ms = -INFINITY;
      for (int c = 0; c < tw.nchunks; ++c)
        ms = fmaxf(ms, __ldcg(base + static_cast<size_t>(c) * kRecFloats + kTileRows * 64 + r));
      float acc[32];
#pragma unroll
      for (int x = 0; x < 32; ++x) acc[x] = 0.f;
      float lsum = 0.f;
      if (ms != -INFINITY) {
        for (int c = 0; c < tw.nchunks; ++c) {
          const float* rc = base + static_cast<size_t>(c) * kRecFloats;
          const float mc = __ldcg(rc + kTileRows * 64 + r);
          const float lc = __ldcg(rc + kTileRows * 64 + kTileRows + r);
          if (mc == -INFINITY) continue;
          const float f = ptx::ex2_approx(mc - ms);
          lsum += lc * f;
          const float4* oc = reinterpret_cast<const float4*>(rc + r * 64 + wg * 32);
#pragma unroll
          for (int v4 = 0; v4 < 8; ++v4) {
            const float4 x = __ldcg(oc + v4);
            acc[v4 * 4 + 0] += f * x.x;
            acc[v4 * 4 + 1] += f * x.y;
            acc[v4 * 4 + 2] += f * x.z;
            acc[v4 * 4 + 3] += f * x.w;
          }
        }
      }
      const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
      uint4* dst = reinterpret_cast<uint4*>(p.out + row * 64 + wg * 32);
#pragma unroll
      for (int v8 = 0; v8 < 4; ++v8) {
        uint4 u;
        u.x = pack_bf16x2(acc[v8 * 8 + 0] * inv, acc[v8 * 8 + 1] * inv);
        u.y = pack_bf16x2(acc[v8 * 8 + 2] * inv, acc[v8 * 8 + 3] * inv);
        u.z = pack_bf16x2(acc[v8 * 8 + 4] * inv, acc[v8 * 8 + 5] * inv);
        u.w = pack_bf16x2(acc[v8 * 8 + 6] * inv, acc[v8 * 8 + 7] * inv);
        dst[v8] = u;
      }
      if (wg == 0) p.lse[row] = lsum > 0.f ? (ms + log2f(lsum)) * kLn2 : -INFINITY;
    }
    if (warp == 0 && lane == 0) *ticket = 0;  // leave the workspace clean for the next call
    return true;
  }
}


__device__ __forceinline__ void softmax_role(const FwdParams& p, uint32_t bars, uint32_t tmem,
                                             int warp, int lane, volatile int* abort_flag,
                                             volatile uint32_t* last_flag, float* xch) {
  auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
  const int wg = warp >> 2;              // key block of each chunk handled here
  const int r = (warp & 3) * 32 + lane;  // tile row == TMEM lane
  const int half = r >> 6;
  const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
  const uint32_t obase = tmem + lane_addr + kTmemO;
  const int total = p.B * p.items_per_batch;
  const float sl2 = p.scale_log2;
  uint32_t g = 0;
  uint32_t n_epi = 0;  // uses of the epilogue barrier
  uint32_t nt = 0;     // tiles started
  bool alive = true;

  TileDone pend{};
  bool have_pend = false;
  for (int t = blockIdx.x; alive && t < total; t += gridDim.x, ++nt) {
    const int b = t / p.items_per_batch;
    const WorkItem w = p.items[t - b * p.items_per_batch];
    // The tile's union entries (at most 64) and their key-padding bits, one or two
    // per lane; each chunk picks its entry with a shuffle.
    const uint32_t ent_lo = lane < w.count ? p.pair_ent[w.start + lane] : 0u;
    const uint32_t ent_hi = lane + 32 < w.count ? p.pair_ent[w.start + 32 + lane] : 0u;
    unsigned long long kb_lo = ~0ull, kb_hi = ~0ull;
    if (p.keybits != nullptr) {
      const size_t kb0 = static_cast<size_t>(b) * p.nb;
      if (lane < w.count) kb_lo = p.keybits[kb0 + (ent_lo & kEntColMask)];
      if (lane + 32 < w.count) kb_hi = p.keybits[kb0 + (ent_hi & kEntColMask)];
    }
    float m_run = -INFINITY, l_run = 0.f;
    const int nch = (w.count + 1) >> 1;
    for (int n = 0; n < nch; ++n, ++g) {
      const int idx = 2 * n + wg;  // warp-uniform
      const bool has = idx < w.count;
      const uint32_t e = __shfl_sync(0xffffffffu, idx < 32 ? ent_lo : ent_hi, idx & 31);
      const unsigned long long kb = __shfl_sync(0xffffffffu, idx < 32 ? kb_lo : kb_hi, idx & 31);
      // warp-uniform: a warp's 32 rows lie in one half of the tile
      const unsigned long long mk = (has && ((e >> (kEntBitsShift + half)) & 1u)) ? kb : 0ull;
      const uint32_t sb = g % kSBufs;
      if (!wait_warp(bar(kBarSFull + static_cast<int>(sb)), (g / kSBufs) & 1u, abort_flag, p.timeout_ns)) {
        alive = false;
        break;
      }
      ptx::tc_fence_after();
      const uint32_t sbase = tmem + lane_addr + kTmemS + sb * 128u + static_cast<uint32_t>(wg) * 64u;
      // Pass 1: the row maximum of this warpgroup's 64 scores.
      float mxs = -INFINITY;
      if (mk != 0ull) {
        uint32_t raw[2][32];
        ptx::tmem_ld32(sbase + 0, raw[0]);
        ptx::tmem_ld32(sbase + 32, raw[1]);
        ptx::tmem_wait_ld();
        ptx::reg_fence(raw[0]);
        ptx::reg_fence(raw[1]);
        float s[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) s[c] = __uint_as_float(raw[c >> 5][c & 31]);
        mask_cols(s, mk);
        float mx4[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
        for (int c = 4; c < 64; c += 2) mx4[(c >> 1) & 3] = ptx::fmax3(mx4[(c >> 1) & 3], s[c], s[c + 1]);
        const float mx = fmaxf(ptx::fmax3(mx4[0], mx4[1], mx4[2]), mx4[3]);
        mxs = mx * sl2;  // scale > 0: -inf stays -inf
      }
      float m_new = m_run;
      bool rescale = false;
      if (n == 0) {
        m_new = mxs;
      } else if (__any_sync(0xffffffffu, mxs > m_run + kRescaleLog2)) {
        rescale = true;
        m_new = fmaxf(m_run, mxs);
      }
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      // Pass 2: p = 2^(s * scale * log2 e - m) 32 columns at a time, reloaded from TMEM
      // to keep few registers live; P_x (bf16, two keys per column) goes over S
      // columns already read.  The buffer's previous reader, PV of chunk g - 3,
      // completed before S(g) was issued.
      float psum = 0.f;
      if (mk != 0ull) {
        const uint64_t sc2 = ptx::pack2(sl2, sl2), nm2 = ptx::pack2(-m_use, -m_use);
        uint64_t acc0 = 0ull, acc1 = 0ull;  // packed partial row sums
#pragma unroll
        for (int hb = 0; hb < 2; ++hb) {
          uint32_t raw[32];
          ptx::tmem_ld32(sbase + 32u * hb, raw);
          ptx::tmem_wait_ld();
          ptx::reg_fence(raw);
          float s[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) s[c] = __uint_as_float(raw[c]);
          const uint32_t mh = static_cast<uint32_t>(mk >> (32 * hb));
          if (mh != 0xffffffffu) {
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (!((mh >> c) & 1u)) s[c] = -INFINITY;
          }
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            float x0, x1;
            ptx::unpack2(ptx::ffma2(ptx::pack2(s[2 * c], s[2 * c + 1]), sc2, nm2), x0, x1);
            const float p0 = ptx::ex2_approx(x0), p1 = ptx::ex2_approx(x1);
            if (c & 1)
              acc1 = ptx::fadd2(acc1, ptx::pack2(p0, p1));
            else
              acc0 = ptx::fadd2(acc0, ptx::pack2(p0, p1));
            pk[c] = pack_bf16x2(p0, p1);
          }
          ptx::tmem_st16(sbase + 16u * hb, pk);
        }
        float a0, a1;
        ptx::unpack2(ptx::fadd2(acc0, acc1), a0, a1);
        psum = a0 + a1;
      } else if (has) {
        // this half of the tile does not attend the block: its P rows are zero
        uint32_t zero[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) zero[c] = 0u;
        ptx::tmem_st32(sbase, zero);
      }
      if (n == 0) {
        l_run = psum;
      } else {
        const float alpha = (m_new == m_run) ? 1.f : ptx::ex2_approx(m_run - m_new);
        l_run = l_run * alpha + psum;
        if (rescale) {  // warp-uniform
          // O_x must hold PV of chunk g - 1 before it is rescaled: wait for its
          // V-free phase.  Unambiguous: S(g) was issued after PV(g - 3) was done, and
          // PV(g - 1 + kVStages) needs this warpgroup's P first.
          const uint32_t gp = g - 1u;
          if (!wait_warp(bar(kBarVFree + static_cast<int>(gp % kVStages)), (gp / kVStages) & 1u,
                         abort_flag, p.timeout_ns)) {
            alive = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t ox = obase + static_cast<uint32_t>(wg) * 64u;
#pragma unroll
          for (int hlf = 0; hlf < 2; ++hlf) {
            uint32_t o[32];
            ptx::tmem_ld32(ox + 32u * hlf, o);
            ptx::tmem_wait_ld();
            ptx::reg_fence(o);
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            ptx::tmem_st32(ox + 32u * hlf, o);
          }
        }
      }
      m_run = m_new;
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(bar(kBarPFull + static_cast<int>(sb)));
      if (n == 0 && have_pend) {  // the previous tile's epilogue, one chunk late
        have_pend = false;
        if (!tile_epilogue(p, pend, bars, obase, warp, lane, abort_flag, last_flag, xch, &n_epi)) {
          alive = false;
          break;
        }
      }
    }
    if (!alive) break;
    pend = TileDone{t, g - 1u, nt, m_run, l_run};
    have_pend = true;
  }
  if (alive && have_pend) tile_epilogue(p, pend, bars, obase, warp, lane, abort_flag, last_flag, xch, &n_epi);
}

__global__ void __launch_bounds__(kThreads, 1) bsa_fwd_kernel(const __grid_constant__ FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t sQ = base + kSmemQ, sK = base + kSmemK, sV = base + kSmemV, bars = base + kSmemBar;
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + kSmemMisc);
  float* xch = reinterpret_cast<float*>(smem + kSmemXch);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      uint32_t count = 1;
      if ((i >= kBarPFull && i < kBarPFull + static_cast<int>(kSBufs)) || i == kBarOFree || i == kBarEpi)
        count = 256;
      ptx::mbar_init(bars + 8u * i, count);
    }
    misc[1] = 0;
    misc[2] = 0;
    ptx::fence_barrier_init();
  }
  if (warp == kProducerWarp && lane == 0) {
    ptx::prefetch_tensormap(&p.tm_q);
    ptx::prefetch_tensormap(&p.tm_k);
    ptx::prefetch_tensormap(&p.tm_v);
  }
  if (warp == kMmaWarp) {
    ptx::tmem_alloc(ptx::smem_addr(const_cast<uint32_t*>(&misc[0])), kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = misc[0];
  volatile int* abort_flag = reinterpret_cast<volatile int*>(&misc[1]);

  if (warp == kProducerWarp) {
    if (lane == 0) producer_role(p, sQ, sK, sV, bars, abort_flag);
    __syncwarp();
  } else if (warp == kMmaWarp) {
    if (lane == 0) s_issuer(p, sQ, sK, bars, tmem, abort_flag);
    __syncwarp();
  } else if (warp == kPvWarp) {
    if (lane == 0) pv_issuer(p, sV, bars, tmem, abort_flag);
    __syncwarp();
  } else {
    softmax_role(p, bars, tmem, warp, lane, abort_flag, &misc[2], xch);
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == kMmaWarp) ptx::tmem_dealloc(tmem, kTmemCols);
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

bool make_map(CUtensorMap* m, const void* ptr, uint64_t rows) {
  auto fn = get_encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {64, rows};
  cuuint64_t strides[1] = {128};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

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
        cudaFuncSetAttribute(bsa_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemAlloc)) != cudaSuccess)
      return BSA_ERR_CUDA;
    d.configured = true;
  }
  *out = d;
  return d.sm100 ? BSA_OK : BSA_ERR_UNSUPPORTED;
}

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

void free_device(bsa_layout* lay) {
  if (lay->device < 0) return;
  int cur = -1;
  const bool have_cur = cudaGetDevice(&cur) == cudaSuccess;
  if (cudaSetDevice(lay->device) == cudaSuccess) {
    cudaFree(lay->d_pair_q);
    cudaFree(lay->d_pair_ent);
    cudaFree(lay->d_items);
  }
  if (have_cur) cudaSetDevice(cur);
  lay->d_pair_q = nullptr;
  lay->d_pair_ent = nullptr;
  lay->d_items = nullptr;
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
  const size_t bq = lay->pair_q.size() * sizeof(int32_t);
  const size_t be = lay->pair_ent.size() * sizeof(uint32_t);
  const size_t bi = lay->items.size() * sizeof(WorkItem);
  if (cudaMalloc(&lay->d_pair_q, std::max<size_t>(bq, 16)) != cudaSuccess ||
      cudaMalloc(&lay->d_pair_ent, std::max<size_t>(be, 16)) != cudaSuccess ||
      cudaMalloc(&lay->d_items, std::max<size_t>(bi, 32)) != cudaSuccess) {
    lay->device = dev;
    free_device(lay);
    return BSA_ERR_OOM;
  }
  lay->device = dev;
  if (cudaMemcpyAsync(lay->d_pair_q, lay->pair_q.data(), bq, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(lay->d_pair_ent, lay->pair_ent.data(), be, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(lay->d_items, lay->items.data(), bi, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess) {
    free_device(lay);
    return BSA_ERR_CUDA;
  }
  return BSA_OK;
}

int bsa_forward(const void* q, const void* k, const void* v, int B, int H, int L, int d,
                const bsa_layout* lay, const uint8_t* key_mask, float scale, void* out, float* lse,
                void* workspace, size_t workspace_bytes, void* stream) {
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr || lse == nullptr ||
      lay == nullptr || B < 1 || H < 1 || L < 1)
    return BSA_ERR_INVALID_ARG;
  if (d != kHeadDim) return BSA_ERR_UNSUPPORTED;
  if (H != lay->H || L != lay->L) return BSA_ERR_LAYOUT_MISMATCH;
  if (static_cast<int64_t>(B) * H * L > INT32_MAX - 64) return BSA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(lse, 4))
    return BSA_ERR_INVALID_ARG;
  if (!(scale == scale) || std::isinf(scale)) return BSA_ERR_INVALID_ARG;
  const WorkspacePlan plan = plan_workspace(*lay, B);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < plan.total)
    return BSA_ERR_WORKSPACE;
  if (lay->device < 0) return BSA_ERR_LAYOUT_MISMATCH;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return BSA_ERR_CUDA;
  if (dev != lay->device) return BSA_ERR_LAYOUT_MISMATCH;
  DeviceInfo info;
  const int st = device_setup(dev, &info);
  if (st != BSA_OK) return st;

  FwdParams prm{};
  const uint64_t rows = static_cast<uint64_t>(B) * H * L;
  if (!make_map(&prm.tm_q, q, rows) || !make_map(&prm.tm_k, k, rows) || !make_map(&prm.tm_v, v, rows))
    return BSA_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  prm.items = lay->d_items;
  prm.pair_q = lay->d_pair_q;
  prm.pair_ent = lay->d_pair_ent;
  prm.keybits = key_mask ? reinterpret_cast<const unsigned long long*>(ws + plan.keybits_off) : nullptr;
  prm.partials = reinterpret_cast<float*>(ws + plan.partials_off);
  prm.tickets = reinterpret_cast<int*>(ws + plan.tickets_off);
  prm.B = B;
  prm.H = H;
  prm.L = L;
  prm.nb = lay->nb;
  prm.items_per_batch = static_cast<int>(lay->items.size());
  prm.n_split = lay->n_split;
  prm.n_records = lay->n_records;
  const float sc = scale > 0.f ? scale : 1.f / std::sqrt(static_cast<float>(d));
  prm.scale_log2 = sc * kLog2e;
  prm.timeout_ns = kDefaultTimeoutNs;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (key_mask != nullptr) {
    const int n = B * lay->nb;
    bsa_keybits_kernel<<<(n + 255) / 256, 256, 0, s>>>(
        key_mask, reinterpret_cast<unsigned long long*>(ws + plan.keybits_off), B, L, lay->nb);
    if (cudaGetLastError() != cudaSuccess) return BSA_ERR_CUDA;
  }
  const int64_t total = static_cast<int64_t>(B) * prm.items_per_batch;
  const int grid = static_cast<int>(std::min<int64_t>(total, info.sms));
  if (grid < 1) return BSA_OK;
  bsa_fwd_kernel<<<grid, kThreads, kSmemAlloc, s>>>(prm);
  if (cudaGetLastError() != cudaSuccess) return BSA_ERR_CUDA;
  return BSA_OK;
}

int bsa_sync_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return BSA_ERR_CUDA;
  int st = 0;
  if (cudaMemcpyFromSymbol(&st, g_bsa_status, sizeof(int)) != cudaSuccess) return BSA_ERR_CUDA;
  if (st != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_bsa_status, &zero, sizeof(int)) != cudaSuccess) return BSA_ERR_CUDA;
  }
  return st;
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
void* g_static_ws_addr[kMaxDevices];
cudaError_t g_static_ws_err[kMaxDevices];
std::once_flag g_static_ws_once[kMaxDevices];
}  // namespace

extern "C" int bsa_forward_static_ws(const void* q, const void* k, const void* v, int B, int H, int L,
                                     int d, const bsa_layout* lay, const uint8_t* key_mask, float scale,
                                     void* out, float* lse, void* stream) {
  // The checks bsa_forward makes before touching the GPU, repeated so that a bad
  // call enqueues nothing (not even the ticket clear below).
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr || lse == nullptr ||
      lay == nullptr || B < 1 || H < 1 || L < 1)
    return BSA_ERR_INVALID_ARG;
  if (d != kHeadDim) return BSA_ERR_UNSUPPORTED;
  if (H != lay->H || L != lay->L) return BSA_ERR_LAYOUT_MISMATCH;
  if (static_cast<int64_t>(B) * H * L > INT32_MAX - 64) return BSA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(lse, 4))
    return BSA_ERR_INVALID_ARG;
  if (!(scale == scale) || std::isinf(scale)) return BSA_ERR_INVALID_ARG;
  const WorkspacePlan plan = plan_workspace(*lay, B);
  if (plan.total > BSA_STATIC_WORKSPACE_BYTES) return BSA_ERR_STATIC_WORKSPACE;
  if (lay->device < 0) return BSA_ERR_LAYOUT_MISMATCH;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return BSA_ERR_CUDA;
  if (dev != lay->device) return BSA_ERR_LAYOUT_MISMATCH;
  if (dev < 0 || dev >= kMaxDevices) return BSA_ERR_UNSUPPORTED;
  DeviceInfo info;
  const int st = device_setup(dev, &info);
  if (st != BSA_OK) return st;
  // once per device, with that device current: the array's address on it
  std::call_once(g_static_ws_once[dev], [dev] {
    g_static_ws_err[dev] = cudaGetSymbolAddress(&g_static_ws_addr[dev], g_bsa_static_ws);
  });
  if (g_static_ws_err[dev] != cudaSuccess || g_static_ws_addr[dev] == nullptr) return BSA_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(g_static_ws_addr[dev]);
  // the arrival tickets must start at zero; the other regions are written before read
  if (cudaMemsetAsync(ws + plan.tickets_off, 0, plan.tickets_bytes, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return BSA_ERR_CUDA;
  return bsa_forward(q, k, v, B, H, L, d, lay, key_mask, scale, out, lse, ws, BSA_STATIC_WORKSPACE_BYTES,
                     stream);
}
