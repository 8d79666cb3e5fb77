// BigBird block-sparse attention backward for B200 (sm_100a).
//
// Gradients of O = softmax(Q K^T * scale restricted to the layout) V ("Adapt or
// Perish ... Adaptive Sparse Transformer", sparse-attention formula; one softmax
// over the union of the BigBird patterns, "BigBird 稀疏注意力机制解析", 核心实现)
// for a loss gradient dO, given the forward's O and lse.  The pages train such
// models ("BERT 稀疏注意力机制入门指南", 生产环境部署建议; "BigBird 稀疏注意力机制解析",
// 避坑指南) without printing the gradient; it is the plain derivative:
//   D  = rowsum(dO * O)                               bsa_bwd_prep_kernel
//   P  = 2^(S * scale * log2 e - lse * log2 e),  S = Q K^T on the attended keys
//   dP = dO V^T,  dS = P * (dP - D)
//   dQ = scale * dS K                                 bsa_bwd_dq_kernel
//   dK = scale * dS^T Q,  dV = P^T dO                 bsa_bwd_dkv_kernel
// P is rebuilt from lse, so no softmax statistics are recomputed.
//
// Both main kernels run one 128-row tile per CTA (128 threads; thread r owns tile
// row r = TMEM lane r) and walk the tile's entries one 64-block at a time:
//   dQ kernel   tile = two query blocks (the forward's tiles), entries = key blocks.
//               S = Q K_j^T and dP = dO V_j^T (tcgen05, A and B from shared
//               memory), dS (bf16) written over the S columns, dQ += dS K_j
//               (A = dS from TMEM).
//   dKV kernel  tile = two key blocks (tiles of the transposed layout), entries =
//               the query blocks that attend them.  S^T = K Q_i^T, dP^T = V dO_i^T,
//               P^T and dS^T (bf16) over their columns, dV += P^T dO_i and
//               dK += dS^T Q_i (A from TMEM).
// One thread issues the TMA loads and the MMAs; the next entry's blocks load
// while the current one is processed.  Tiles with long unions are cut into chunks
// whose partial sums (fp32) bsa_bwd_merge_kernel adds up.  Every wait is bounded;
// on expiry the CTA records BSA_ERR_DEVICE_TIMEOUT, lets its copies and MMAs
// finish, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <mutex>

#include "bsa_host_cuda.h"
#include "bsa_internal.h"
#include "bsa_wait.cuh"
#include "sm100_ptx.cuh"

namespace bsa {
namespace {

constexpr int kThreads = 128;
constexpr uint32_t kBlkBytes = 64 * 128;  // one 64 x 64 bf16 block
constexpr uint32_t kTmemCols = 256;
// TMEM columns: two 64-column score buffers, two 64-column accumulators
constexpr uint32_t kTmemA = 0;    // S (dQ) or S^T (dKV); bf16 dS / P^T over its first 32
constexpr uint32_t kTmemB = 64;   // dP (dQ) or dP^T (dKV); bf16 dS^T over its first 32 (dKV)
constexpr uint32_t kTmemC = 128;  // dQ accumulator (dQ) or dV (dKV)
constexpr uint32_t kTmemD = 192;  // dK accumulator (dKV)

// shared memory (offsets from the 1024-aligned base).  The tile's own two 64-row
// blocks of two operands (Q and dO, or K and V) stay resident; the entry's two
// blocks (K_j and V_j, or Q_i and dO_i) cycle through two stages.
constexpr uint32_t kSmemTileA = 0;                       // 2 blocks
constexpr uint32_t kSmemTileB = kSmemTileA + 2 * kBlkBytes;  // 2 blocks
constexpr uint32_t kSmemEntA = kSmemTileB + 2 * kBlkBytes;   // 2 stages
constexpr uint32_t kSmemEntB = kSmemEntA + 2 * kBlkBytes;    // 2 stages
constexpr uint32_t kSmemVec = kSmemEntB + 2 * kBlkBytes;     // dKV: lse2 and D of the entry, 2 stages
constexpr uint32_t kVecBytes = 64 * 4;
constexpr uint32_t kSmemBar = kSmemVec + 4 * kVecBytes;
enum : int {
  kBarTile = 0,      // the tile's resident blocks landed
  kBarEnt = 1,       // [2 stages] the entry's blocks landed
  kBarSdp = 3,       // MMA commit: S and dP (or S^T and dP^T) are in TMEM
  kBarDs = 4,        // 128 arrivals: dS (and P^T) written to TMEM
  kBarAcc = 5,       // MMA commit: the accumulating MMAs of the entry are done
  kBarFinal = 6,     // MMA commit of an aborting CTA
  kNumBars = 7
};
constexpr uint32_t kSmemMisc = kSmemBar + 8 * kNumBars;  // u32 TMEM base, int abort flag
constexpr uint32_t kSmemUsed = kSmemMisc + 16;
// Requested dynamic shared memory: the used part plus alignment slack, rounded up
// so that at most two CTAs share an SM -- two fill its 512 TMEM columns.
constexpr uint32_t kSmemAlloc = 96 * 1024;
static_assert(kSmemUsed + 1024 <= kSmemAlloc, "shared memory budget");
static_assert(3 * (kSmemAlloc + 1024) > 228 * 1024, "at most two CTAs per SM");

struct BwdParams {
  CUtensorMap tm_q, tm_k, tm_v, tm_do;
  const float* dsum;  // D per row, [B*H*L]
  const float* lse2;  // lse * log2 e per row, +inf where lse = -inf (P = 0)
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  const BwdItem* items;
  const int32_t* pair;       // tile blocks, 2 per tile (second -1: single block)
  const uint32_t* pair_ent;  // entries: block | membership << 24
  const unsigned long long* keybits;  // [B, nb] or null
  float* records;  // partial sums of split tiles, per batch element n_records of them
  int B, H, L, nb, n_records;
  float scale, scale_log2;
  unsigned long long timeout_ns;
};

constexpr uint32_t kIdescQK = ptx::idesc_bf16_f32(128, 64, false);  // B K-major
constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(128, 64, true);   // B MN-major

// Issues A (128 rows, K-major, at smem a) times B^T (64 rows, K-major, at smem b)
// into TMEM column d: head dim 64 = 4 steps of K = 16, +32 bytes each.
__device__ __forceinline__ void mma_rows_x_rows(uint32_t d, uint32_t a, uint32_t b) {
  const uint64_t da = ptx::smem_desc_sw128(a, 16), db = ptx::smem_desc_sw128(b, 16);
#pragma unroll
  for (uint32_t kk = 0; kk < 4; ++kk) ptx::mma_ss(d, da + 2 * kk, db + 2 * kk, kIdescQK, kk > 0 ? 1u : 0u);
}

// Issues D (+)= A (128 x 64, bf16 in TMEM column a) times B (a 64 x 64 row-major
// block at smem b, read MN-major): 4 steps of K = 16 rows of B, +2048 bytes each.
__device__ __forceinline__ void mma_tmem_x_block(uint32_t d, uint32_t a, uint32_t b, bool accumulate) {
  const uint64_t db = ptx::smem_desc_sw128(b, 0);
#pragma unroll
  for (uint32_t kk = 0; kk < 4; ++kk)
    ptx::mma_ts(d, a + 8u * kk, db + kk * (2048u >> 4), kIdescPV, (accumulate || kk > 0) ? 1u : 0u);
}

// Bookkeeping of the issuing thread, for draining after an abort.
struct IssueState {
  uint32_t ent_issued = 0, ent_waited = 0;  // entry loads
  bool tile_issued = false, tile_waited = false;
  bool mma_issued = false;
};

// After an abort: wait (bounded) for this thread's copies and MMAs so that nothing
// lands in shared memory or TMEM after the CTA has left.
__device__ void drain(const IssueState& is, uint32_t bars, volatile int* abort_flag, uint64_t timeout_ns) {
  auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
  if (is.tile_issued && !is.tile_waited) wait_force(bar(kBarTile), 0, abort_flag, timeout_ns);
  for (uint32_t x = is.ent_waited; x < is.ent_issued; ++x)
    wait_force(bar(kBarEnt + static_cast<int>(x & 1u)), (x >> 1) & 1u, abort_flag, timeout_ns);
  if (is.mma_issued) {
    ptx::mma_commit(bar(kBarFinal));
    wait_force(bar(kBarFinal), 0, abort_flag, timeout_ns);
  }
}

// Common prologue: barriers, TMEM.  Returns the TMEM base.
__device__ __forceinline__ uint32_t cta_setup(uint8_t* smem, uint32_t base) {
  const uint32_t bars = base + kSmemBar;
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + kSmemMisc);
  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i)
      ptx::mbar_init(bars + 8u * static_cast<uint32_t>(i), i == kBarDs ? static_cast<uint32_t>(kThreads) : 1u);
    misc[1] = 0;
    ptx::fence_barrier_init();
  }
  if ((threadIdx.x >> 5) == 0) {
    ptx::tmem_alloc(ptx::smem_addr(const_cast<uint32_t*>(&misc[0])), kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  return misc[0];
}

__device__ __forceinline__ void cta_teardown(uint32_t tmem) {
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if ((threadIdx.x >> 5) == 0) ptx::tmem_dealloc(tmem, kTmemCols);
}

// 64 fp32 values of this thread's row from TMEM column `col` (lane offset included).
__device__ __forceinline__ void load_row64(uint32_t taddr, float (&v)[64]) {
  uint32_t raw[2][32];
  ptx::tmem_ld32(taddr, raw[0]);
  ptx::tmem_ld32(taddr + 32u, raw[1]);
  ptx::tmem_wait_ld();
  ptx::reg_fence(raw[0]);
  ptx::reg_fence(raw[1]);
#pragma unroll
  for (int c = 0; c < 64; ++c) v[c] = __uint_as_float(raw[c >> 5][c & 31]);
}

// Stores a row of 64 values times f: bf16 to `out` (a whole tile) or fp32 to `rec`
// (a chunk of a split tile).
__device__ __forceinline__ void store_row64(const float (&v)[64], float f, __nv_bfloat16* out, float* rec) {
  if (rec != nullptr) {
    float4* o = reinterpret_cast<float4*>(rec);
#pragma unroll
    for (int x = 0; x < 16; ++x) o[x] = make_float4(v[4 * x] * f, v[4 * x + 1] * f, v[4 * x + 2] * f, v[4 * x + 3] * f);
  } else {
    uint4* o = reinterpret_cast<uint4*>(out);
#pragma unroll
    for (int x = 0; x < 8; ++x) {
      uint4 u;
      u.x = pack_bf16x2(v[8 * x + 0] * f, v[8 * x + 1] * f);
      u.y = pack_bf16x2(v[8 * x + 2] * f, v[8 * x + 3] * f);
      u.z = pack_bf16x2(v[8 * x + 4] * f, v[8 * x + 5] * f);
      u.w = pack_bf16x2(v[8 * x + 6] * f, v[8 * x + 7] * f);
      o[x] = u;
    }
  }
}

// ------------------------------------------------------------------ dQ
__global__ void __launch_bounds__(kThreads, 1) bsa_bwd_dq_kernel(const __grid_constant__ BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t bars = base + kSmemBar;
  auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
  const uint32_t tmem = cta_setup(smem, base);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kSmemMisc + 4);
  const int tid = threadIdx.x, warp = tid >> 5;
  const bool leader = tid == 0;

  const int it = blockIdx.x / p.B, b = blockIdx.x - it * p.B;
  const BwdItem w = p.items[it];
  const int qa = p.pair[2 * w.pair], qb = p.pair[2 * w.pair + 1];
  const int row0 = (b * p.H + w.h) * p.L;
  const int half = tid >> 6;
  const bool row_active = half == 0 || qb >= 0;
  const size_t grow = static_cast<size_t>(row0) + static_cast<size_t>(half ? qb : qa) * 64 + (tid & 63);
  const float lse2 = row_active ? p.lse2[grow] : INFINITY;
  const float drow = row_active ? p.dsum[grow] : 0.f;
  const float sl2 = p.scale_log2;
  const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t sQ = base + kSmemTileA, sDO = base + kSmemTileB, sK = base + kSmemEntA, sV = base + kSmemEntB;

  IssueState is;
  bool ok = true;
  const uint64_t pol = ptx::policy_evict_last();
  auto issue_entry = [&](int n) {  // K_j and V_j of entry n into stage n % 2
    const int j = static_cast<int>(p.pair_ent[w.start + n] & kEntColMask);
    const uint32_t st = static_cast<uint32_t>(n) & 1u;
    ptx::mbar_arrive_expect_tx(bar(kBarEnt + static_cast<int>(st)), 2 * kBlkBytes);
    ptx::tma_load_2d(sK + st * kBlkBytes, &p.tm_k, bar(kBarEnt + static_cast<int>(st)), 0, row0 + j * 64, pol);
    ptx::tma_load_2d(sV + st * kBlkBytes, &p.tm_v, bar(kBarEnt + static_cast<int>(st)), 0, row0 + j * 64, pol);
    ++is.ent_issued;
  };
  if (leader) {
    const int qb_ld = qb >= 0 ? qb : qa;  // a single-block tile loads its block twice
    ptx::mbar_arrive_expect_tx(bar(kBarTile), 4 * kBlkBytes);
    ptx::tma_load_2d(sQ, &p.tm_q, bar(kBarTile), 0, row0 + qa * 64, pol);
    ptx::tma_load_2d(sQ + kBlkBytes, &p.tm_q, bar(kBarTile), 0, row0 + qb_ld * 64, pol);
    ptx::tma_load_2d(sDO, &p.tm_do, bar(kBarTile), 0, row0 + qa * 64, pol);
    ptx::tma_load_2d(sDO + kBlkBytes, &p.tm_do, bar(kBarTile), 0, row0 + qb_ld * 64, pol);
    is.tile_issued = true;
    issue_entry(0);
  }

  for (int n = 0; n < w.count && ok; ++n) {
    const uint32_t e = p.pair_ent[w.start + n];
    const uint32_t st = static_cast<uint32_t>(n) & 1u;
    const uint32_t ph = static_cast<uint32_t>(n) & 1u;  // phase of the once-per-entry barriers
    if (leader) {
      // stage st ^ 1 last served entry n - 1, whose MMAs are done (waited below)
      if (n + 1 < w.count) issue_entry(n + 1);
      if (n == 0) {
        ok = wait_one(bar(kBarTile), 0, abort_flag, p.timeout_ns);
        is.tile_waited = ok;
      }
      ok = ok && wait_one(bar(kBarEnt + static_cast<int>(st)), (static_cast<uint32_t>(n) >> 1) & 1u, abort_flag,
                          p.timeout_ns);
      if (ok) {
        ++is.ent_waited;
        ptx::tc_fence_after();
        mma_rows_x_rows(tmem + kTmemA, sQ, sK + st * kBlkBytes);    // S = Q K_j^T
        mma_rows_x_rows(tmem + kTmemB, sDO, sV + st * kBlkBytes);   // dP = dO V_j^T
        ptx::mma_commit(bar(kBarSdp));
        is.mma_issued = true;
      }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok) break;
    if (!wait_warp(bar(kBarSdp), ph, abort_flag, p.timeout_ns)) {
      ok = false;
      break;
    }
    ptx::tc_fence_after();
    // this half's keys of block j: membership bit, then key padding
    unsigned long long mk = 0ull;
    if (row_active && ((e >> (kEntBitsShift + half)) & 1u))
      mk = p.keybits != nullptr ? p.keybits[static_cast<size_t>(b) * p.nb + (e & kEntColMask)] : ~0ull;
    uint32_t pk[32];
    if (mk != 0ull) {  // warp-uniform
#pragma unroll
      for (int hc = 0; hc < 2; ++hc) {
        uint32_t s_raw[32], dp_raw[32];
        ptx::tmem_ld32(tmem + lane_addr + kTmemA + 32u * hc, s_raw);
        ptx::tmem_ld32(tmem + lane_addr + kTmemB + 32u * hc, dp_raw);
        ptx::tmem_wait_ld();
        ptx::reg_fence(s_raw);
        ptx::reg_fence(dp_raw);
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int c0 = 32 * hc + 2 * c;
          const float p0 = ((mk >> c0) & 1ull) ? ptx::ex2_approx(__uint_as_float(s_raw[2 * c]) * sl2 - lse2) : 0.f;
          const float p1 =
              ((mk >> (c0 + 1)) & 1ull) ? ptx::ex2_approx(__uint_as_float(s_raw[2 * c + 1]) * sl2 - lse2) : 0.f;
          pk[16 * hc + c] = pack_bf16x2(p0 * (__uint_as_float(dp_raw[2 * c]) - drow),
                                        p1 * (__uint_as_float(dp_raw[2 * c + 1]) - drow));
        }
      }
    } else {
#pragma unroll
      for (int c = 0; c < 32; ++c) pk[c] = 0u;
    }
    ptx::tmem_st32(tmem + lane_addr + kTmemA, pk);  // dS over S columns already read
    ptx::tmem_wait_st();
    ptx::tc_fence_before();
    ptx::mbar_arrive(bar(kBarDs));
    if (leader) {
      ok = wait_one(bar(kBarDs), ph, abort_flag, p.timeout_ns);
      if (ok) {
        ptx::tc_fence_after();
        mma_tmem_x_block(tmem + kTmemC, tmem + kTmemA, sK + st * kBlkBytes, n > 0);  // dQ += dS K_j
        ptx::mma_commit(bar(kBarAcc));
        ok = wait_one(bar(kBarAcc), ph, abort_flag, p.timeout_ns);
      }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);  // keep the loop warp-uniform
  }
  ok = __syncthreads_and(ok ? 1 : 0) != 0;
  if (ok && w.count > 0) {
    if (!wait_warp(bar(kBarAcc), static_cast<uint32_t>(w.count - 1) & 1u, abort_flag, p.timeout_ns)) ok = false;
  }
  if (ok) {
    ptx::tc_fence_after();
    float v[64];
    load_row64(tmem + lane_addr + kTmemC, v);
    if (row_active) {
      float* rec = w.rec >= 0 ? p.records + (static_cast<size_t>(b) * p.n_records + w.rec) * kBwdDqRecFloats +
                                    static_cast<size_t>(tid) * 64
                              : nullptr;
      store_row64(v, p.scale, p.dq + grow * 64, rec);
    }
  } else if (leader) {
    drain(is, bars, abort_flag, p.timeout_ns);
  }
  cta_teardown(tmem);
}

// ------------------------------------------------------------------ dK, dV
__global__ void __launch_bounds__(kThreads, 1) bsa_bwd_dkv_kernel(const __grid_constant__ BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t bars = base + kSmemBar;
  auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
  const uint32_t tmem = cta_setup(smem, base);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kSmemMisc + 4);
  const int tid = threadIdx.x, warp = tid >> 5;
  const bool leader = tid == 0;

  const int it = blockIdx.x / p.B, b = blockIdx.x - it * p.B;
  const BwdItem w = p.items[it];
  const int ka = p.pair[2 * w.pair], kb = p.pair[2 * w.pair + 1];
  const int row0 = (b * p.H + w.h) * p.L;
  const int half = tid >> 6;
  const bool row_active = half == 0 || kb >= 0;
  const int kblk = half ? kb : ka;
  const size_t grow = static_cast<size_t>(row0) + static_cast<size_t>(kblk) * 64 + (tid & 63);
  // this key row takes part at all: its key is not dropped by the padding mask
  const bool key_kept =
      row_active && (p.keybits == nullptr || ((p.keybits[static_cast<size_t>(b) * p.nb + kblk] >> (tid & 63)) & 1ull));
  const float sl2 = p.scale_log2;
  const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t sK = base + kSmemTileA, sV = base + kSmemTileB, sQ = base + kSmemEntA, sDO = base + kSmemEntB;
  const float* vec = reinterpret_cast<const float*>(smem + kSmemVec);  // [stage][lse2 64, D 64]

  IssueState is;
  bool ok = true;
  const uint64_t pol = ptx::policy_evict_last();
  auto issue_entry = [&](int n) {  // Q_i, dO_i, lse2 and D of query block i into stage n % 2
    const int i = static_cast<int>(p.pair_ent[w.start + n] & kEntColMask);
    const uint32_t st = static_cast<uint32_t>(n) & 1u;
    const uint32_t eb = bar(kBarEnt + static_cast<int>(st));
    ptx::mbar_arrive_expect_tx(eb, 2 * kBlkBytes + 2 * kVecBytes);
    ptx::tma_load_2d(sQ + st * kBlkBytes, &p.tm_q, eb, 0, row0 + i * 64, pol);
    ptx::tma_load_2d(sDO + st * kBlkBytes, &p.tm_do, eb, 0, row0 + i * 64, pol);
    const uint32_t sv = base + kSmemVec + st * 2 * kVecBytes;
    ptx::bulk_load(sv, p.lse2 + static_cast<size_t>(row0) + static_cast<size_t>(i) * 64, kVecBytes, eb);
    ptx::bulk_load(sv + kVecBytes, p.dsum + static_cast<size_t>(row0) + static_cast<size_t>(i) * 64, kVecBytes, eb);
    ++is.ent_issued;
  };
  if (leader) {
    const int kb_ld = kb >= 0 ? kb : ka;
    ptx::mbar_arrive_expect_tx(bar(kBarTile), 4 * kBlkBytes);
    ptx::tma_load_2d(sK, &p.tm_k, bar(kBarTile), 0, row0 + ka * 64, pol);
    ptx::tma_load_2d(sK + kBlkBytes, &p.tm_k, bar(kBarTile), 0, row0 + kb_ld * 64, pol);
    ptx::tma_load_2d(sV, &p.tm_v, bar(kBarTile), 0, row0 + ka * 64, pol);
    ptx::tma_load_2d(sV + kBlkBytes, &p.tm_v, bar(kBarTile), 0, row0 + kb_ld * 64, pol);
    is.tile_issued = true;
    issue_entry(0);
  }

  for (int n = 0; n < w.count && ok; ++n) {
    const uint32_t e = p.pair_ent[w.start + n];
    const uint32_t st = static_cast<uint32_t>(n) & 1u;
    const uint32_t ph = static_cast<uint32_t>(n) & 1u;
    if (leader) {
      if (n + 1 < w.count) issue_entry(n + 1);
      if (n == 0) {
        ok = wait_one(bar(kBarTile), 0, abort_flag, p.timeout_ns);
        is.tile_waited = ok;
      }
    }
    // every thread: the entry's stage landed (the threads read lse2 and D from it)
    if (!wait_warp(bar(kBarEnt + static_cast<int>(st)), (static_cast<uint32_t>(n) >> 1) & 1u, abort_flag,
                   p.timeout_ns)) {
      ok = false;
      break;
    }
    if (leader) {
      ++is.ent_waited;
      ok = ok && !*abort_flag;
      if (ok) {
        ptx::tc_fence_after();
        mma_rows_x_rows(tmem + kTmemA, sK, sQ + st * kBlkBytes);    // S^T = K Q_i^T
        mma_rows_x_rows(tmem + kTmemB, sV, sDO + st * kBlkBytes);   // dP^T = V dO_i^T
        ptx::mma_commit(bar(kBarSdp));
        is.mma_issued = true;
      }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok) break;
    if (!wait_warp(bar(kBarSdp), ph, abort_flag, p.timeout_ns)) {
      ok = false;
      break;
    }
    ptx::tc_fence_after();
    const bool take = key_kept && ((e >> (kEntBitsShift + half)) & 1u);  // warp-uniform membership
    uint32_t ppk[32], dpk[32];
    if (__any_sync(0xffffffffu, take)) {
      const float* l2 = vec + st * 128;
      const float* dd = l2 + 64;
#pragma unroll
      for (int hc = 0; hc < 2; ++hc) {
        uint32_t s_raw[32], dp_raw[32];
        ptx::tmem_ld32(tmem + lane_addr + kTmemA + 32u * hc, s_raw);
        ptx::tmem_ld32(tmem + lane_addr + kTmemB + 32u * hc, dp_raw);
        ptx::tmem_wait_ld();
        ptx::reg_fence(s_raw);
        ptx::reg_fence(dp_raw);
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int c0 = 32 * hc + 2 * c;
          const float2 lv = *reinterpret_cast<const float2*>(l2 + c0);
          const float2 dv2 = *reinterpret_cast<const float2*>(dd + c0);
          const float p0 = take ? ptx::ex2_approx(__uint_as_float(s_raw[2 * c]) * sl2 - lv.x) : 0.f;
          const float p1 = take ? ptx::ex2_approx(__uint_as_float(s_raw[2 * c + 1]) * sl2 - lv.y) : 0.f;
          ppk[16 * hc + c] = pack_bf16x2(p0, p1);
          dpk[16 * hc + c] = pack_bf16x2(p0 * (__uint_as_float(dp_raw[2 * c]) - dv2.x),
                                         p1 * (__uint_as_float(dp_raw[2 * c + 1]) - dv2.y));
        }
      }
    } else {
#pragma unroll
      for (int c = 0; c < 32; ++c) ppk[c] = dpk[c] = 0u;
    }
    ptx::tmem_st32(tmem + lane_addr + kTmemA, ppk);  // P^T over S^T columns already read
    ptx::tmem_st32(tmem + lane_addr + kTmemB, dpk);  // dS^T over dP^T columns already read
    ptx::tmem_wait_st();
    ptx::tc_fence_before();
    ptx::mbar_arrive(bar(kBarDs));
    if (leader) {
      ok = wait_one(bar(kBarDs), ph, abort_flag, p.timeout_ns);
      if (ok) {
        ptx::tc_fence_after();
        mma_tmem_x_block(tmem + kTmemC, tmem + kTmemA, sDO + st * kBlkBytes, n > 0);  // dV += P^T dO_i
        mma_tmem_x_block(tmem + kTmemD, tmem + kTmemB, sQ + st * kBlkBytes, n > 0);   // dK += dS^T Q_i
        ptx::mma_commit(bar(kBarAcc));
        ok = wait_one(bar(kBarAcc), ph, abort_flag, p.timeout_ns);
      }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);  // keep the loop warp-uniform
  }
  ok = __syncthreads_and(ok ? 1 : 0) != 0;
  if (ok && w.count > 0) {
    if (!wait_warp(bar(kBarAcc), static_cast<uint32_t>(w.count - 1) & 1u, abort_flag, p.timeout_ns)) ok = false;
  }
  if (ok) {
    ptx::tc_fence_after();
    float* rec = w.rec >= 0 ? p.records + (static_cast<size_t>(b) * p.n_records + w.rec) * kBwdDkvRecFloats +
                                  static_cast<size_t>(tid) * 64
                            : nullptr;
    float v[64];
    load_row64(tmem + lane_addr + kTmemD, v);
    if (row_active) store_row64(v, p.scale, p.dk + grow * 64, rec);
    load_row64(tmem + lane_addr + kTmemC, v);
    if (row_active) store_row64(v, 1.f, p.dv + grow * 64, rec != nullptr ? rec + kTileRows * 64 : nullptr);
  } else if (leader) {
    drain(is, bars, abort_flag, p.timeout_ns);
  }
  cta_teardown(tmem);
}

// ------------------------------------------------------------------ D, lse2
// One row per 8 threads: D = sum_c dO[c] O[c] in fp32 (O as the forward stored it),
// lse2 = lse * log2 e, with lse = -inf (a row with no attended key) mapped to +inf
// so that 2^(s - lse2) = 0 there.
__global__ void __launch_bounds__(256) bsa_bwd_prep_kernel(const __nv_bfloat16* __restrict__ out,
                                                           const __nv_bfloat16* __restrict__ dout,
                                                           const float* __restrict__ lse, float* __restrict__ dsum,
                                                           float* __restrict__ lse2, int64_t rows) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t row = t >> 3;
  const int part = static_cast<int>(t & 7);
  float acc = 0.f;
  if (row < rows) {
    const uint4 a = *reinterpret_cast<const uint4*>(out + row * 64 + part * 8);
    const uint4 g = *reinterpret_cast<const uint4*>(dout + row * 64 + part * 8);
    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&g);
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const float2 af = __bfloat1622float2(a2[x]), gf = __bfloat1622float2(g2[x]);
      acc = fmaf(af.x, gf.x, acc);
      acc = fmaf(af.y, gf.y, acc);
    }
  }
  acc += __shfl_xor_sync(0xffffffffu, acc, 4);
  acc += __shfl_xor_sync(0xffffffffu, acc, 2);
  acc += __shfl_xor_sync(0xffffffffu, acc, 1);
  if (row < rows && part == 0) {
    dsum[row] = acc;
    const float l = lse[row];
    lse2[row] = l == -INFINITY ? INFINITY : l * kLog2e;
  }
}

// ------------------------------------------------------------------ merge
// Sum of a split tile's partial records (already scaled), one warp per (batch
// element, split tile, tile row); lane x owns columns 2x, 2x + 1.
struct BwdMergeParams {
  const float* records;
  const SplitTile* splits;
  __nv_bfloat16* out;
  int rec_floats, plane;  // floats per record; offset of this output's plane in it
  int B, H, L, n_split, n_records;
};

__global__ void __launch_bounds__(128) bsa_bwd_merge_kernel(const __grid_constant__ BwdMergeParams p) {
  const int lane = threadIdx.x & 31;
  const int task = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int per_b = p.n_split * kTileRows;
  if (task >= p.B * per_b) return;
  const int b = task / per_b, rem = task - b * per_b;
  const int s = rem / kTileRows, r = rem - s * kTileRows;
  const SplitTile st = p.splits[s];
  const int blk = (r >> 6) ? st.qb : st.qa;
  if (blk < 0) return;
  const size_t row = static_cast<size_t>(b * p.H + st.h) * p.L + static_cast<size_t>(blk) * 64 + (r & 63);
  const float* src = p.records + (static_cast<size_t>(b) * p.n_records + st.rec_base) * p.rec_floats + p.plane +
                     static_cast<size_t>(r) * 64;
  float2 acc = make_float2(0.f, 0.f);
  for (int x = 0; x < st.nchunks; ++x) {
    const float2 v = __ldcg(reinterpret_cast<const float2*>(src + static_cast<size_t>(x) * p.rec_floats) + lane);
    acc.x += v.x;
    acc.y += v.y;
  }
  reinterpret_cast<uint32_t*>(p.out + row * 64)[lane] = pack_bf16x2(acc.x, acc.y);
}

// ------------------------------------------------------------------ host
constexpr int kMaxDevices = 64;
std::once_flag g_setup_once[kMaxDevices];
int g_setup_status[kMaxDevices];

int bwd_device_setup(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return BSA_ERR_UNSUPPORTED;
  std::call_once(g_setup_once[dev], [dev] {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
      g_setup_status[dev] = BSA_ERR_CUDA;
      return;
    }
    if (major != 10 || minor != 0) {
      g_setup_status[dev] = BSA_ERR_UNSUPPORTED;
      return;
    }
    if (cudaFuncSetAttribute(bsa_bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemAlloc)) != cudaSuccess ||
        cudaFuncSetAttribute(bsa_bwd_dkv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemAlloc)) != cudaSuccess) {
      g_setup_status[dev] = BSA_ERR_CUDA;
      return;
    }
    g_setup_status[dev] = BSA_OK;
  });
  return g_setup_status[dev];
}

inline bool aligned(const void* ptr, size_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

int launch_merge(const float* records, const SplitTile* splits, __nv_bfloat16* out, int rec_floats, int plane,
                 int B, int H, int L, int n_split, int n_records, cudaStream_t s) {
  if (n_split == 0) return BSA_OK;
  BwdMergeParams mp{records, splits, out, rec_floats, plane, B, H, L, n_split, n_records};
  const int64_t tasks = static_cast<int64_t>(B) * n_split * kTileRows;
  bsa_bwd_merge_kernel<<<static_cast<int>((tasks + 3) / 4), 128, 0, s>>>(mp);
  return cudaGetLastError() == cudaSuccess ? BSA_OK : BSA_ERR_CUDA;
}

}  // namespace

int bwd_take_status() {
  int st = 0;
  if (cudaMemcpyFromSymbol(&st, g_bsa_status, sizeof(int)) != cudaSuccess) return BSA_ERR_CUDA;
  if (st != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_bsa_status, &zero, sizeof(int)) != cudaSuccess) return BSA_ERR_CUDA;
  }
  return st;
}

}  // namespace bsa

using namespace bsa;

extern "C" int bsa_backward(const void* q, const void* k, const void* v, const void* out, const void* dout,
                            const float* lse, int B, int H, int L, int d, const bsa_layout* lay,
                            const uint8_t* key_mask, float scale, void* dq, void* dk, void* dv, void* workspace,
                            size_t workspace_bytes, void* stream) {
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr || dout == nullptr || lse == nullptr ||
      dq == nullptr || dk == nullptr || dv == nullptr || lay == nullptr || B < 1 || H < 1 || L < 1)
    return BSA_ERR_INVALID_ARG;
  if (d != kHeadDim) return BSA_ERR_UNSUPPORTED;
  if (H != lay->H || L != lay->L) return BSA_ERR_LAYOUT_MISMATCH;
  if (static_cast<int64_t>(B) * H * L > INT32_MAX - 64) return BSA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(dout, 16) ||
      !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(lse, 4))
    return BSA_ERR_INVALID_ARG;
  if (!(scale == scale) || std::isinf(scale)) return BSA_ERR_INVALID_ARG;
  const BwdWorkspacePlan plan = plan_bwd_workspace(*lay, B);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < plan.total) return BSA_ERR_WORKSPACE;
  if (lay->device < 0) return BSA_ERR_LAYOUT_MISMATCH;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return BSA_ERR_CUDA;
  if (dev != lay->device) return BSA_ERR_LAYOUT_MISMATCH;
  const int su = bwd_device_setup(dev);
  if (su != BSA_OK) return su;

  BwdParams prm{};
  const uint64_t rows = static_cast<uint64_t>(B) * H * L;
  if (!make_map(&prm.tm_q, q, rows, 64) || !make_map(&prm.tm_k, k, rows, 64) || !make_map(&prm.tm_v, v, rows, 64) ||
      !make_map(&prm.tm_do, dout, rows, 64))
    return BSA_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  auto* keybits = reinterpret_cast<unsigned long long*>(ws + plan.keybits_off);
  if (key_mask != nullptr && launch_keybits(key_mask, keybits, B, L, lay->nb, s) != cudaSuccess) return BSA_ERR_CUDA;
  prm.dsum = reinterpret_cast<float*>(ws + plan.dsum_off);
  prm.lse2 = reinterpret_cast<float*>(ws + plan.lse2_off);
  {
    const int64_t threads = static_cast<int64_t>(rows) * 8;
    bsa_bwd_prep_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(out), static_cast<const __nv_bfloat16*>(dout), lse,
        const_cast<float*>(prm.dsum), const_cast<float*>(prm.lse2), static_cast<int64_t>(rows));
    if (cudaGetLastError() != cudaSuccess) return BSA_ERR_CUDA;
  }
  prm.dq = static_cast<__nv_bfloat16*>(dq);
  prm.dk = static_cast<__nv_bfloat16*>(dk);
  prm.dv = static_cast<__nv_bfloat16*>(dv);
  prm.keybits = key_mask != nullptr ? keybits : nullptr;
  prm.B = B;
  prm.H = H;
  prm.L = L;
  prm.nb = lay->nb;
  const float sc = scale > 0.f ? scale : 1.f / std::sqrt(static_cast<float>(d));
  prm.scale = sc;
  prm.scale_log2 = sc * kLog2e;
  prm.timeout_ns = kDefaultTimeoutNs;

  // dQ over the query tiles
  BwdParams pq = prm;
  pq.items = lay->d_dq_items;
  pq.pair = lay->d_pair_q;
  pq.pair_ent = lay->d_pair_ent;
  pq.records = reinterpret_cast<float*>(ws + plan.dq_rec_off);
  pq.n_records = lay->dq_plan.n_records;
  const int64_t gq = static_cast<int64_t>(B) * static_cast<int64_t>(lay->dq_plan.items.size());
  if (gq > 0) {
    bsa_bwd_dq_kernel<<<static_cast<unsigned>(gq), kThreads, kSmemAlloc, s>>>(pq);
    if (cudaGetLastError() != cudaSuccess) return BSA_ERR_CUDA;
  }
  // dK and dV over the key tiles
  BwdParams pk = prm;
  pk.items = lay->d_dkv_items;
  pk.pair = lay->d_kpair_q;
  pk.pair_ent = lay->d_kpair_ent;
  pk.records = reinterpret_cast<float*>(ws + plan.dkv_rec_off);
  pk.n_records = lay->dkv_plan.n_records;
  const int64_t gk = static_cast<int64_t>(B) * static_cast<int64_t>(lay->dkv_plan.items.size());
  if (gk > 0) {
    bsa_bwd_dkv_kernel<<<static_cast<unsigned>(gk), kThreads, kSmemAlloc, s>>>(pk);
    if (cudaGetLastError() != cudaSuccess) return BSA_ERR_CUDA;
  }
  const int n_dq_split = static_cast<int>(lay->dq_plan.splits.size());
  const int n_kv_split = static_cast<int>(lay->dkv_plan.splits.size());
  int st = launch_merge(pq.records, lay->d_dq_splits, prm.dq, kBwdDqRecFloats, 0, B, H, L, n_dq_split,
                        pq.n_records, s);
  if (st == BSA_OK)
    st = launch_merge(pk.records, lay->d_dkv_splits, prm.dk, kBwdDkvRecFloats, 0, B, H, L, n_kv_split,
                      pk.n_records, s);
  if (st == BSA_OK)
    st = launch_merge(pk.records, lay->d_dkv_splits, prm.dv, kBwdDkvRecFloats, kTileRows * 64, B, H, L, n_kv_split,
                      pk.n_records, s);
  return st;
}
