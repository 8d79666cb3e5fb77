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
// Kernel design (one persistent CTA per SM, 192 threads):
//   warp 4      TMA producer: Q tile (2 x 64 rows), then K and V blocks of the tile's
//               key-block union into a kStages-deep shared-memory ring.
//   warp 5      tcgen05 issuer: S = Q K^T (M=128, N=64|128, K=64) into one of two TMEM
//               S buffers, then O += P V (A = P read from TMEM, M=128, N=64).
//   warps 0-3   softmax + epilogue: thread r owns tile row r = TMEM lane r.  Reads S,
//               applies the tile's membership bits and key padding, keeps the running
//               max / sum in fp32, writes P (bf16) over S in TMEM, rescales O when the
//               max grows by more than kRescaleLog2, and finally normalises O.
// A tile is two query blocks of the same (b, h) over the sorted union of their rows;
// entries carry per-block membership bits so each half sees exactly its own row.
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

constexpr int kThreads = 192;
constexpr int kStages = 4;
constexpr uint32_t kBlkBytes = 64 * 128;         // one 64 x 64 bf16 block
constexpr uint32_t kQBytes = 2 * kBlkBytes;      // 128-row Q tile
constexpr uint32_t kStageBytes = 2 * kBlkBytes;  // two key blocks
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemS = 0;      // S buffers at columns [0,128) and [128,256)
constexpr uint32_t kTmemO = 256;    // O accumulator at [256, 320)
constexpr float kRescaleLog2 = 8.0f;
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLog2e = 1.44269504088896340736f;
constexpr uint32_t kMaxSpin = 1u << 24;
constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;

// shared memory map (offsets from a 1024-aligned base)
constexpr uint32_t kSmemQ = 0;
constexpr uint32_t kSmemK = kSmemQ + 2 * kQBytes;
constexpr uint32_t kSmemV = kSmemK + kStages * kStageBytes;
constexpr uint32_t kSmemBar = kSmemV + kStages * kStageBytes;
enum : int {
  kBarQFull = 0,
  kBarQEmpty = 2,
  kBarKFull = 4,
  kBarKEmpty = kBarKFull + kStages,
  kBarVFull = kBarKEmpty + kStages,
  kBarVEmpty = kBarVFull + kStages,
  kBarSFull = kBarVEmpty + kStages,
  kBarPFull = kBarSFull + 2,
  kBarODone = kBarPFull + 2,
  kBarMmaFinal = kBarODone + 1,
  kBarEpi = kBarMmaFinal + 1,  // 128 softmax threads, split-chunk epilogue
  kNumBars = kBarEpi + 1
};
constexpr uint32_t kSmemMisc = kSmemBar + 8 * kNumBars;
constexpr uint32_t kSmemUsed = kSmemMisc + 16;
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
    if (ptx::mbar_try_wait(bar, parity)) return true;
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
__device__ __forceinline__ void producer_role(const FwdParams& p, uint32_t sQ, uint32_t sK,
                                              uint32_t sV, uint32_t bars, int lane,
                                              volatile int* abort_flag) {
  auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
  const uint64_t pol_q = ptx::policy_evict_first();
  const uint64_t pol_kv = ptx::policy_evict_last();
  const int total = p.B * p.items_per_batch;
  uint32_t nq = 0, nq_issued = 0, nk = 0, nv = 0;  // tiles visited; loads issued per ring
  bool alive = true;
  for (int t = blockIdx.x; alive && t < total; t += gridDim.x, ++nq) {
    const int b = t / p.items_per_batch;
    const WorkItem w = p.items[t - b * p.items_per_batch];
    const int row0 = (b * p.H + w.h) * p.L;
    const int qa = p.pair_q[2 * w.pair], qb = p.pair_q[2 * w.pair + 1];
    const uint32_t qs = nq & 1u;
    if (!wait_warp(bar(kBarQEmpty + qs), ((nq >> 1) & 1u) ^ 1u, abort_flag, p.timeout_ns)) {
      alive = false;
      break;
    }
    if (lane == 0) {
      ptx::mbar_arrive_expect_tx(bar(kBarQFull + qs), kQBytes);
      ptx::tma_load_2d(sQ + qs * kQBytes, &p.tm_q, bar(kBarQFull + qs), 0, row0 + qa * 64, pol_q);
      ptx::tma_load_2d(sQ + qs * kQBytes + kBlkBytes, &p.tm_q, bar(kBarQFull + qs), 0,
                       row0 + (qb >= 0 ? qb : qa) * 64, pol_q);
    }
    __syncwarp();
    ++nq_issued;
    const int nch = (w.count + 1) >> 1;
    for (int n = 0; n < nch; ++n) {
      const int e = w.start + 2 * n;
      const int j0 = static_cast<int>(p.pair_ent[e] & kEntColMask);
      const bool two = 2 * n + 1 < w.count;
      const int j1 = two ? static_cast<int>(p.pair_ent[e + 1] & kEntColMask) : 0;
      const uint32_t bytes = two ? 2 * kBlkBytes : kBlkBytes;
      const uint32_t st = nk % kStages;
      if (!wait_warp(bar(kBarKEmpty + st), ((nk / kStages) & 1u) ^ 1u, abort_flag, p.timeout_ns)) {
        alive = false;
        break;
      }
      if (lane == 0) {
        ptx::mbar_arrive_expect_tx(bar(kBarKFull + st), bytes);
        ptx::tma_load_2d(sK + st * kStageBytes, &p.tm_k, bar(kBarKFull + st), 0, row0 + j0 * 64, pol_kv);
        if (two)
          ptx::tma_load_2d(sK + st * kStageBytes + kBlkBytes, &p.tm_k, bar(kBarKFull + st), 0,
                           row0 + j1 * 64, pol_kv);
      }
      __syncwarp();
      ++nk;
      if (!wait_warp(bar(kBarVEmpty + st), ((nv / kStages) & 1u) ^ 1u, abort_flag, p.timeout_ns)) {
        alive = false;
        break;
      }
      if (lane == 0) {
        ptx::mbar_arrive_expect_tx(bar(kBarVFull + st), bytes);
        ptx::tma_load_2d(sV + st * kStageBytes, &p.tm_v, bar(kBarVFull + st), 0, row0 + j0 * 64, pol_kv);
        if (two)
          ptx::tma_load_2d(sV + st * kStageBytes + kBlkBytes, &p.tm_v, bar(kBarVFull + st), 0,
                           row0 + j1 * 64, pol_kv);
      }
      __syncwarp();
      ++nv;
    }
  }
  if (!alive) {
    // Aborted: let every copy this warp issued land before the CTA exits.  The
    // last issue into ring slot s had index s + R * floor((n - 1 - s) / R).
    auto drain = [&](int first_bar, uint32_t n, uint32_t ring) {
      for (uint32_t s = 0; s < ring; ++s) {
        if (n > s) {
          const uint32_t last = s + ring * ((n - 1u - s) / ring);
          wait_force(bar(first_bar + static_cast<int>(s)), (last / ring) & 1u, abort_flag, p.timeout_ns);
        }
      }
    };
    drain(kBarQFull, nq_issued, 2u);
    drain(kBarKFull, nk, static_cast<uint32_t>(kStages));
    drain(kBarVFull, nv, static_cast<uint32_t>(kStages));
  }
}

__device__ __forceinline__ void mma_role(const FwdParams& p, uint32_t sQ, uint32_t sK, uint32_t sV,
                                         uint32_t bars, uint32_t tmem, int lane,
                                         volatile int* abort_flag) {
  auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
  constexpr uint32_t kIdescS128 = ptx::idesc_bf16_f32(128, 128, false);
  constexpr uint32_t kIdescS64 = ptx::idesc_bf16_f32(128, 64, false);
  constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(128, 64, true);
  const int total = p.B * p.items_per_batch;
  uint32_t g = 0;   // global chunk counter (== K/V ring position)
  uint32_t nq = 0;  // tiles started
  bool alive = true;
  bool have_prev = false;
  uint32_t prev_g = 0, prev_two = 0, prev_first = 0;

  auto issue_pv = [&](uint32_t pg, uint32_t two, uint32_t first) -> bool {
    const uint32_t sb = pg & 1u;
    if (!wait_warp(bar(kBarPFull + sb), (pg >> 1) & 1u, abort_flag, p.timeout_ns)) return false;
    const uint32_t st = pg % kStages;
    if (!wait_warp(bar(kBarVFull + st), (pg / kStages) & 1u, abort_flag, p.timeout_ns)) return false;
    ptx::tc_fence_after();
    if (lane == 0) {
      const uint32_t vbase = sV + st * kStageBytes;
      const int ksteps = two ? 8 : 4;  // 16 keys per MMA
      for (int k = 0; k < ksteps; ++k) {
        const uint64_t bdesc = ptx::smem_desc_sw128(vbase + static_cast<uint32_t>(k) * 2048u, 0);
        ptx::mma_ts(tmem + kTmemO, tmem + kTmemS + sb * 128u + static_cast<uint32_t>(k) * 8u, bdesc,
                    kIdescPV, (k > 0 || !first) ? 1u : 0u);
      }
      ptx::mma_commit(bar(kBarODone));
      ptx::mma_commit(bar(kBarVEmpty + st));
    }
    __syncwarp();
    return true;
  };

  for (int t = blockIdx.x; alive && t < total; t += gridDim.x, ++nq) {
    const int b = t / p.items_per_batch;
    const WorkItem w = p.items[t - b * p.items_per_batch];
    const uint32_t qs = nq & 1u;
    if (!wait_warp(bar(kBarQFull + qs), (nq >> 1) & 1u, abort_flag, p.timeout_ns)) {
      alive = false;
      break;
    }
    const int nch = (w.count + 1) >> 1;
    for (int n = 0; n < nch; ++n, ++g) {
      const uint32_t st = g % kStages;
      if (!wait_warp(bar(kBarKFull + st), (g / kStages) & 1u, abort_flag, p.timeout_ns)) {
        alive = false;
        break;
      }
      ptx::tc_fence_after();
      const bool two = 2 * n + 1 < w.count;
      if (lane == 0) {
        const uint32_t qbase = sQ + qs * kQBytes;
        const uint32_t kbase = sK + st * kStageBytes;
        for (int k = 0; k < 4; ++k) {  // head dim 64 = 4 x 16, +32 bytes per step
          const uint64_t adesc = ptx::smem_desc_sw128(qbase + static_cast<uint32_t>(k) * 32u, 16);
          const uint64_t bdesc = ptx::smem_desc_sw128(kbase + static_cast<uint32_t>(k) * 32u, 16);
          ptx::mma_ss(tmem + kTmemS + (g & 1u) * 128u, adesc, bdesc, two ? kIdescS128 : kIdescS64,
                      k > 0 ? 1u : 0u);
        }
        ptx::mma_commit(bar(kBarSFull + (g & 1u)));
        ptx::mma_commit(bar(kBarKEmpty + st));
        if (n == nch - 1) ptx::mma_commit(bar(kBarQEmpty + qs));
      }
      __syncwarp();
      if (have_prev && !issue_pv(prev_g, prev_two, prev_first)) {
        alive = false;
        break;
      }
      have_prev = true;
      prev_g = g;
      prev_two = two ? 1u : 0u;
      prev_first = n == 0 ? 1u : 0u;
    }
  }
  if (alive && have_prev) issue_pv(prev_g, prev_two, prev_first);
  // Every MMA this thread issued must finish before TMEM is released.
  if (lane == 0) ptx::mma_commit(bar(kBarMmaFinal));
  __syncwarp();
  wait_force(bar(kBarMmaFinal), 0, abort_flag, p.timeout_ns);
}

__device__ __forceinline__ void mask_block(float (&s)[128], int off, unsigned long long mk) {
  if (mk == ~0ull) return;
  if (mk == 0ull) {
#pragma unroll
    for (int c = 0; c < 64; ++c) s[off + c] = -INFINITY;
    return;
  }
#pragma unroll
  for (int c = 0; c < 64; ++c)
    if (!((mk >> c) & 1ull)) s[off + c] = -INFINITY;
}

__device__ __forceinline__ void softmax_role(const FwdParams& p, uint32_t bars, uint32_t tmem,
                                             int warp, volatile int* abort_flag,
                                             volatile uint32_t* last_flag) {
  auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
  const int r = threadIdx.x;  // tile row == TMEM lane
  const int half = r >> 6;
  const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
  const int total = p.B * p.items_per_batch;
  const float sl2 = p.scale_log2;
  uint32_t g = 0;
  uint32_t n_epi = 0;  // uses of the epilogue barrier
  bool alive = true;
  // Bounded 128-thread rendezvous (a plain bar.sync could not give up if another
  // softmax warp had already aborted).
  auto epi_sync = [&]() -> bool {
    ptx::mbar_arrive(bar(kBarEpi));
    const bool ok = wait_warp(bar(kBarEpi), n_epi & 1u, abort_flag, p.timeout_ns);
    ++n_epi;
    return ok;
  };
  for (int t = blockIdx.x; alive && t < total; t += gridDim.x) {
    const int b = t / p.items_per_batch;
    const WorkItem w = p.items[t - b * p.items_per_batch];
    const int bh = b * p.H + w.h;
    const int qa = p.pair_q[2 * w.pair], qb = p.pair_q[2 * w.pair + 1];
    const bool row_active = half == 0 || qb >= 0;
    float m_run = -INFINITY, l_run = 0.f;
    const int nch = (w.count + 1) >> 1;
    for (int n = 0; n < nch; ++n, ++g) {
      const int e = w.start + 2 * n;
      const uint32_t e0 = p.pair_ent[e];
      const bool two = 2 * n + 1 < w.count;
      const uint32_t e1 = two ? p.pair_ent[e + 1] : 0u;
      unsigned long long mk0 = ((e0 >> (kEntBitsShift + half)) & 1u) ? ~0ull : 0ull;
      unsigned long long mk1 = ((e1 >> (kEntBitsShift + half)) & 1u) ? ~0ull : 0ull;
      if (p.keybits != nullptr) {
        mk0 &= p.keybits[static_cast<size_t>(b) * p.nb + (e0 & kEntColMask)];
        if (two) mk1 &= p.keybits[static_cast<size_t>(b) * p.nb + (e1 & kEntColMask)];
      }
      const uint32_t sb = g & 1u;
      if (!wait_warp(bar(kBarSFull + sb), (g >> 1) & 1u, abort_flag, p.timeout_ns)) {
        alive = false;
        break;
      }
      ptx::tc_fence_after();
      uint32_t raw[4][32];
      const uint32_t sbase = tmem + lane_addr + kTmemS + sb * 128u;
      ptx::tmem_ld32(sbase + 0, raw[0]);
      ptx::tmem_ld32(sbase + 32, raw[1]);
      ptx::tmem_ld32(sbase + 64, raw[2]);
      ptx::tmem_ld32(sbase + 96, raw[3]);
      ptx::tmem_wait_ld();
      ptx::reg_fence(raw[0]);
      ptx::reg_fence(raw[1]);
      ptx::reg_fence(raw[2]);
      ptx::reg_fence(raw[3]);
      float s[128];
#pragma unroll
      for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(raw[c >> 5][c & 31]);
      mask_block(s, 0, mk0);
      mask_block(s, 64, mk1);
      float mx8[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) mx8[c] = s[c];
#pragma unroll
      for (int c = 8; c < 128; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], s[c]);
      float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                       fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      const float mxs = mx * sl2;  // scale > 0: -inf stays -inf
      float m_new = m_run;
      bool rescale = false;
      if (n == 0) {
        m_new = mxs;
      } else if (__any_sync(0xffffffffu, mxs > m_run + kRescaleLog2)) {
        rescale = true;
        m_new = fmaxf(m_run, mxs);
      }
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      uint32_t pk[2][32];
      float sum4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float p0 = ptx::ex2_approx(fmaf(s[2 * c], sl2, -m_use));
        const float p1 = ptx::ex2_approx(fmaf(s[2 * c + 1], sl2, -m_use));
        sum4[c & 3] += p0 + p1;
        pk[c >> 5][c & 31] = pack_bf16x2(p0, p1);
      }
      const float psum = (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]);
      // PV of the previous chunk must be done before O is touched (and this keeps
      // the O-done phase tracking exact: one wait per completed PV).
      if (g > 0) {
        if (!wait_warp(bar(kBarODone), (g - 1u) & 1u, abort_flag, p.timeout_ns)) {
          alive = false;
          break;
        }
        ptx::tc_fence_after();
      }
      if (n == 0) {
        l_run = psum;
      } else {
        const float alpha = (m_new == m_run) ? 1.f : ptx::ex2_approx(m_run - m_new);
        l_run = l_run * alpha + psum;
        if (rescale) {  // warp-uniform
          uint32_t o[2][32];
          const uint32_t obase = tmem + lane_addr + kTmemO;
          ptx::tmem_ld32(obase + 0, o[0]);
          ptx::tmem_ld32(obase + 32, o[1]);
          ptx::tmem_wait_ld();
          ptx::reg_fence(o[0]);
          ptx::reg_fence(o[1]);
#pragma unroll
          for (int c = 0; c < 64; ++c)
            o[c >> 5][c & 31] = __float_as_uint(__uint_as_float(o[c >> 5][c & 31]) * alpha);
          ptx::tmem_st32(obase + 0, o[0]);
          ptx::tmem_st32(obase + 32, o[1]);
        }
      }
      m_run = m_new;
      ptx::tmem_st32(sbase + 0, pk[0]);
      ptx::tmem_st32(sbase + 32, pk[1]);
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(bar(kBarPFull + sb));
    }
    if (!alive || nch == 0) break;
    // ---- epilogue: wait for the tile's last PV, then read O
    if (!wait_warp(bar(kBarODone), (g - 1u) & 1u, abort_flag, p.timeout_ns)) {
      alive = false;
      break;
    }
    ptx::tc_fence_after();
    uint32_t o[2][32];
    const uint32_t obase = tmem + lane_addr + kTmemO;
    ptx::tmem_ld32(obase + 0, o[0]);
    ptx::tmem_ld32(obase + 32, o[1]);
    ptx::tmem_wait_ld();
    ptx::reg_fence(o[0]);
    ptx::reg_fence(o[1]);
    const int qblk = half ? qb : qa;
    if (w.split < 0) {
      if (row_active) {
        const size_t row = static_cast<size_t>(bh) * p.L + static_cast<size_t>(qblk) * 64 + (r & 63);
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
        uint4* dst = reinterpret_cast<uint4*>(p.out + row * 64);
#pragma unroll
        for (int v8 = 0; v8 < 8; ++v8) {
          uint4 u;
          u.x = pack_bf16x2(__uint_as_float(o[v8 >> 2][(v8 & 3) * 8 + 0]) * inv,
                            __uint_as_float(o[v8 >> 2][(v8 & 3) * 8 + 1]) * inv);
          u.y = pack_bf16x2(__uint_as_float(o[v8 >> 2][(v8 & 3) * 8 + 2]) * inv,
                            __uint_as_float(o[v8 >> 2][(v8 & 3) * 8 + 3]) * inv);
          u.z = pack_bf16x2(__uint_as_float(o[v8 >> 2][(v8 & 3) * 8 + 4]) * inv,
                            __uint_as_float(o[v8 >> 2][(v8 & 3) * 8 + 5]) * inv);
          u.w = pack_bf16x2(__uint_as_float(o[v8 >> 2][(v8 & 3) * 8 + 6]) * inv,
                            __uint_as_float(o[v8 >> 2][(v8 & 3) * 8 + 7]) * inv);
          dst[v8] = u;
        }
        p.lse[row] = l_run > 0.f ? (m_run + log2f(l_run)) * kLn2 : -INFINITY;
      }
    } else {
      // ---- split chunk: store the partial record, then the last arriver merges
      float* rec = p.partials + (static_cast<size_t>(b) * p.n_records + w.rec) * kRecFloats;
      float4* orow = reinterpret_cast<float4*>(rec + r * 64);
#pragma unroll
      for (int v4 = 0; v4 < 16; ++v4)
        orow[v4] = make_float4(__uint_as_float(o[v4 >> 3][(v4 & 7) * 4 + 0]),
                               __uint_as_float(o[v4 >> 3][(v4 & 7) * 4 + 1]),
                               __uint_as_float(o[v4 >> 3][(v4 & 7) * 4 + 2]),
                               __uint_as_float(o[v4 >> 3][(v4 & 7) * 4 + 3]));
      rec[kTileRows * 64 + r] = m_run;
      rec[kTileRows * 64 + kTileRows + r] = l_run;
      __threadfence();
      if (!epi_sync()) {
        alive = false;
        break;
      }
      int* ticket = p.tickets + static_cast<size_t>(b) * p.n_split + w.split;
      if (r == 0) *last_flag = (atomicAdd(ticket, 1) == w.nchunks - 1) ? 1u : 0u;
      if (!epi_sync()) {
        alive = false;
        break;
      }
      if (*last_flag) {
        __threadfence();
        if (row_active) {
          const float* base = p.partials + (static_cast<size_t>(b) * p.n_records + w.rec_base) * kRecFloats;
          float ms = -INFINITY;
          for (int c = 0; c < w.nchunks; ++c)
            ms = fmaxf(ms, __ldcg(base + static_cast<size_t>(c) * kRecFloats + kTileRows * 64 + r));
          const size_t row = static_cast<size_t>(bh) * p.L + static_cast<size_t>(qblk) * 64 + (r & 63);
          float acc[64];
#pragma unroll
          for (int x = 0; x < 64; ++x) acc[x] = 0.f;
          float lsum = 0.f;
          if (ms != -INFINITY) {
            for (int c = 0; c < w.nchunks; ++c) {
              const float* rc = base + static_cast<size_t>(c) * kRecFloats;
              const float mc = __ldcg(rc + kTileRows * 64 + r);
              const float lc = __ldcg(rc + kTileRows * 64 + kTileRows + r);
              if (mc == -INFINITY) continue;
              const float f = ptx::ex2_approx(mc - ms);
              lsum += lc * f;
              const float4* oc = reinterpret_cast<const float4*>(rc + r * 64);
#pragma unroll
              for (int v4 = 0; v4 < 16; ++v4) {
                const float4 x = __ldcg(oc + v4);
                acc[v4 * 4 + 0] += f * x.x;
                acc[v4 * 4 + 1] += f * x.y;
                acc[v4 * 4 + 2] += f * x.z;
                acc[v4 * 4 + 3] += f * x.w;
              }
            }
          }
          const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
          uint4* dst = reinterpret_cast<uint4*>(p.out + row * 64);
#pragma unroll
          for (int v8 = 0; v8 < 8; ++v8) {
            uint4 u;
            u.x = pack_bf16x2(acc[v8 * 8 + 0] * inv, acc[v8 * 8 + 1] * inv);
            u.y = pack_bf16x2(acc[v8 * 8 + 2] * inv, acc[v8 * 8 + 3] * inv);
            u.z = pack_bf16x2(acc[v8 * 8 + 4] * inv, acc[v8 * 8 + 5] * inv);
            u.w = pack_bf16x2(acc[v8 * 8 + 6] * inv, acc[v8 * 8 + 7] * inv);
            dst[v8] = u;
          }
          p.lse[row] = lsum > 0.f ? (ms + log2f(lsum)) * kLn2 : -INFINITY;
        }
        if (r == 0) *ticket = 0;  // leave the workspace clean for the next call
      }
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1) bsa_fwd_kernel(const __grid_constant__ FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t sQ = base + kSmemQ, sK = base + kSmemK, sV = base + kSmemV, bars = base + kSmemBar;
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + kSmemMisc);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i)
      ptx::mbar_init(bars + 8u * i, (i == kBarPFull || i == kBarPFull + 1 || i == kBarEpi) ? 128u : 1u);
    misc[1] = 0;
    misc[2] = 0;
    ptx::fence_barrier_init();
  }
  if (warp == 4 && lane == 0) {
    ptx::prefetch_tensormap(&p.tm_q);
    ptx::prefetch_tensormap(&p.tm_k);
    ptx::prefetch_tensormap(&p.tm_v);
  }
  if (warp == 5) {
    ptx::tmem_alloc(ptx::smem_addr(const_cast<uint32_t*>(&misc[0])), kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = misc[0];
  volatile int* abort_flag = reinterpret_cast<volatile int*>(&misc[1]);

  if (warp == 4) {
    producer_role(p, sQ, sK, sV, bars, lane, abort_flag);
  } else if (warp == 5) {
    mma_role(p, sQ, sK, sV, bars, tmem, lane, abort_flag);
  } else {
    softmax_role(p, bars, tmem, warp, abort_flag, &misc[2]);
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 5) ptx::tmem_dealloc(tmem, kTmemCols);
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
