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
//   dQ = scale * dS K                                 bsa_bwd_kernel<false, .>
//   dK = scale * dS^T Q,  dV = P^T dO                 bsa_bwd_kernel<true, .>
// P is rebuilt from lse, so no softmax statistics are recomputed.
//
// bsa_bwd_kernel runs persistent CTAs (one per SM, 352 threads) over a list of
// 128-row tiles, each CTA taking items blockIdx.x, blockIdx.x + gridDim.x, ...
// of a list sorted longest first.  A tile walks its entries one 64-block at a time:
//   dQ   tile = two query blocks (the forward's tiles), entries = key blocks j.
//        S = Q K_j^T, dP = dO V_j^T; dS (bf16) over S; dQ += dS K_j.
//   dKV  tile = two key blocks (tiles of the transposed layout), entries = the
//        query blocks i attending them.  S^T = K Q_i^T, dP^T = V dO_i^T; P^T and
//        dS^T (bf16) over them; dV += P^T dO_i, dK += dS^T Q_i.
// Roles:
//   warps 0-7  compute: warp w owns TMEM lanes 32 (w % 4) .. + 31 (tile rows) and
//              score columns 32 (w / 4) .. + 31; it writes its 32 bf16 results
//              packed into the first 16 of those columns (columns it has read).
//              They also run each tile's epilogue, one entry into the next tile.
//   warp 8     TMA producer: the tile's two resident operands (2 stages, so the
//              next tile loads during this one) and each entry's two blocks (and,
//              for dKV, the entry's 64 values of lse * log2 e and D) into a
//              4-stage ring.
//   warp 9     score issuer: S and dP of entry g into TMEM score stage g % 2 --
//              one entry ahead of the compute warps.  Allocates TMEM.
//   warp 10    accumulate issuer: once dS of entry g is written, the accumulating
//              MMAs of entry g into TMEM accumulator stage (tile % 2), so the
//              epilogue of a tile overlaps the next one.
// Tiles with long unions are cut into chunks whose partial sums (fp32)
// bsa_bwd_merge_kernel adds up.  Every wait is bounded; on expiry the CTA records
// BSA_ERR_DEVICE_TIMEOUT, lets its copies and MMAs finish, frees TMEM and returns.
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

static_assert(kSplitThreshold <= 64 && kSplitChunk <= 64, "a backward item has at most 64 entries");
constexpr int kComputeWarps = 8;
constexpr int kComputeThreads = 32 * kComputeWarps;
constexpr int kProducerWarp = 8;
constexpr int kScoreWarp = 9;
constexpr int kAccWarp = 10;
constexpr int kThreads = 352;
constexpr int kEStages = 4;                   // entry ring
constexpr uint32_t kBlkBytes = 64 * 128;      // one 64 x 64 bf16 block
constexpr uint32_t kOpBytes = 2 * kBlkBytes;  // a 128-row tile operand
constexpr uint32_t kVecBytes = 64 * 4;
constexpr uint32_t kTmemCols = 512;
// TMEM: score stage s at 128 s (S or S^T at +0, dP or dP^T at +64); accumulator
// stage a after the score stages, kAccCols apart (dQ; or dV at +0 and dK at +64)
constexpr uint32_t kTmemScore = 0;

// shared memory (offsets from the 1024-aligned base)
constexpr uint32_t kSmemTile = 0;                                // [2 stages][operand A | operand B]
constexpr uint32_t kSmemEnt = kSmemTile + 2 * 2 * kOpBytes;      // [4 stages][block A | block B]
constexpr uint32_t kSmemVec = kSmemEnt + kEStages * 2 * kBlkBytes;  // [4 stages][lse2 | D] (dKV)
constexpr uint32_t kSmemBar = kSmemVec + kEStages * 2 * kVecBytes;
enum : int {
  kBarTileFull = 0,                      // [2] the tile's operands landed
  kBarTileEmpty = 2,                     // [2] the tile's last score MMAs are done
  kBarEntFull = 4,                       // [4] the entry's blocks (and vectors) landed
  kBarEntEmpty = kBarEntFull + kEStages,      // [4] the entry's accumulating MMAs are done
  kBarScoreFull = kBarEntEmpty + kEStages,    // [3] S and dP of the entry are in TMEM
  kBarScoreFree = kBarScoreFull + 3,          // [3] the entry's accumulating MMAs read its dS
  kBarDsFull = kBarScoreFree + 3,             // [3] 256 arrivals: dS (and P^T) written
  kBarAccFull = kBarDsFull + 3,               // [2] the tile's last accumulating MMAs are done (dK/dV uses one)
  kBarAccEmpty = kBarAccFull + 2,             // [2] 256 arrivals: the epilogue read the accumulators
  kBarFinal = kBarAccEmpty + 2,               // [2] the issuers' last commits
  kNumBars = kBarFinal + 2
};
constexpr uint32_t kSmemMisc = kSmemBar + 8 * kNumBars;  // u32 TMEM base, int abort flag
constexpr uint32_t kSmemAlloc = kSmemMisc + 16 + 1024;   // + slack for 1024-byte alignment
static_assert(kSmemAlloc <= 227 * 1024, "shared memory budget");

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
  // token-level layouts (else null): bit c of word j set when token 64 j + c is global,
  // and the window in tokens; entries flagged at kEntMaskShift + half get a mask of
  // the other block's 64 tokens per row
  const unsigned long long* tok_gbits;
  long long tok_window;
  float* records;  // partial sums of split tiles, per batch element n_records of them
  int B, H, L, nb, n_items, n_records;
  float scale, scale_log2;
  unsigned long long timeout_ns;
};

// The tokens of block `blk` within [c - w, c + w]: the token-level band of token c
// (its keys for a query, its queries for a key), one bit per token of the block.
__device__ __forceinline__ unsigned long long band_bits(long long c, long long w, int blk) {
  const long long lo = c - w - 64ll * blk, hi = c + w - 64ll * blk;
  if (hi < 0 || lo > 63) return 0ull;
  const int l = lo < 0 ? 0 : static_cast<int>(lo), h = hi > 63 ? 63 : static_cast<int>(hi);
  return (h == 63 ? ~0ull : ((1ull << (h + 1)) - 1ull)) & ~((1ull << l) - 1ull);
}

constexpr uint32_t kIdescQK = ptx::idesc_bf16_f32(128, 64, false);  // B K-major
constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(128, 64, true);   // B MN-major

// A (128 rows, K-major, at smem a) times B^T (64 rows, K-major, at smem b) into
// TMEM column d: head dim 64 = 4 steps of K = 16, +32 bytes each.
__device__ __forceinline__ void mma_rows_x_rows(uint32_t d, uint32_t a, uint32_t b) {
  const uint64_t da = ptx::smem_desc_sw128(a, 16), db = ptx::smem_desc_sw128(b, 16);
#pragma unroll
  for (uint32_t kk = 0; kk < 4; ++kk) ptx::mma_ss(d, da + 2 * kk, db + 2 * kk, kIdescQK, kk > 0 ? 1u : 0u);
}

// D (+)= A times B: A is 128 x 64 bf16 in TMEM starting at column a, packed two
// per column, keys 0-31 in columns a .. a + 15 and keys 32-63 in a + 32 .. a + 47
// (each compute warp packs its 32 columns into the first half of them); B is a
// 64 x 64 row-major block at smem b, read MN-major, 16 rows (2048 bytes) per step.
__device__ __forceinline__ void mma_tmem_x_block(uint32_t d, uint32_t a, uint32_t b, bool accumulate) {
  const uint64_t db = ptx::smem_desc_sw128(b, 0);
#pragma unroll
  for (uint32_t kk = 0; kk < 4; ++kk)
    ptx::mma_ts(d, a + 8u * kk + (kk >= 2 ? 16u : 0u), db + kk * (2048u >> 4), kIdescPV,
                (accumulate || kk > 0) ? 1u : 0u);
}

struct ItemRef {
  BwdItem w;
  int b, ta, tb, row0;
};

__device__ __forceinline__ ItemRef item_at(const BwdParams& p, int it) {
  ItemRef r;
  const int i = it / p.B;
  r.b = it - i * p.B;
  r.w = p.items[i];
  r.ta = p.pair[2 * r.w.pair];
  r.tb = p.pair[2 * r.w.pair + 1];
  r.row0 = (r.b * p.H + r.w.h) * p.L;
  return r;
}

// 32 fp32 values of this thread's lane from TMEM column taddr.
__device__ __forceinline__ void load32(uint32_t taddr, float (&v)[32]) {
  uint32_t raw[32];
  ptx::tmem_ld32(taddr, raw);
  ptx::tmem_wait_ld();
  ptx::reg_fence(raw);
#pragma unroll
  for (int c = 0; c < 32; ++c) v[c] = __uint_as_float(raw[c]);
}

// Stores 32 values times f: bf16 to `out` or fp32 to `rec` (a chunk of a split tile).
__device__ __forceinline__ void store32(const float (&v)[32], float f, __nv_bfloat16* out, float* rec) {
  if (rec != nullptr) {
    float4* o = reinterpret_cast<float4*>(rec);
#pragma unroll
    for (int x = 0; x < 8; ++x) o[x] = make_float4(v[4 * x] * f, v[4 * x + 1] * f, v[4 * x + 2] * f, v[4 * x + 3] * f);
  } else {
    uint4* o = reinterpret_cast<uint4*>(out);
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      uint4 u;
      u.x = pack_bf16x2(v[8 * x + 0] * f, v[8 * x + 1] * f);
      u.y = pack_bf16x2(v[8 * x + 2] * f, v[8 * x + 3] * f);
      u.z = pack_bf16x2(v[8 * x + 4] * f, v[8 * x + 5] * f);
      u.w = pack_bf16x2(v[8 * x + 6] * f, v[8 * x + 7] * f);
      o[x] = u;
    }
  }
}

// kTok: the layout is token-level (flagged entries get per-row masks); block layouts
// run the instantiation without that code.
template <bool kDkv, bool kTok>
__global__ void __launch_bounds__(kThreads, 1) bsa_bwd_kernel(const __grid_constant__ BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t bars = base + kSmemBar;
  auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + kSmemMisc);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      const bool many = (i >= kBarDsFull && i < kBarDsFull + 3) || (i >= kBarAccEmpty && i < kBarAccEmpty + 2);
      ptx::mbar_init(bar(i), many ? static_cast<uint32_t>(kComputeThreads) : 1u);
    }
    misc[1] = 0;
    ptx::fence_barrier_init();
  }
  if (warp == kScoreWarp) {
    ptx::tmem_alloc(ptx::smem_addr(const_cast<uint32_t*>(&misc[0])), kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = misc[0];
  volatile int* abort_flag = reinterpret_cast<volatile int*>(&misc[1]);
  const int total = p.B * p.n_items;
  constexpr uint32_t kAccCols = kDkv ? 128u : 64u;
  // three score stages; accumulators: two stages of 64 columns (dQ), one of 128 (dK/dV)
  constexpr uint32_t kSStages = 3u;
  constexpr uint32_t kAccStages = kDkv ? 1u : 2u;
  constexpr uint32_t kAccBase = 384u;
  static_assert(128u * kSStages <= kAccBase && kAccBase + kAccStages * kAccCols <= kTmemCols, "TMEM map");
  auto tile_op = [&](uint32_t ts, int op) { return base + kSmemTile + ts * 2 * kOpBytes + op * kOpBytes; };
  auto ent_op = [&](uint32_t es, int op) { return base + kSmemEnt + es * 2 * kBlkBytes + op * kBlkBytes; };

  if (warp == kProducerWarp) {
    if (lane == 0) {
      // ---------------- TMA producer
      const uint64_t pol = ptx::policy_evict_last();
      const CUtensorMap* tmA = kDkv ? &p.tm_k : &p.tm_q;   // tile operands
      const CUtensorMap* tmB = kDkv ? &p.tm_v : &p.tm_do;
      const CUtensorMap* emA = kDkv ? &p.tm_q : &p.tm_k;   // entry operands
      const CUtensorMap* emB = kDkv ? &p.tm_do : &p.tm_v;
      const uint32_t ent_tx = 2 * kBlkBytes + (kDkv ? 2 * kVecBytes : 0u);
      uint32_t k = 0, g = 0, tiles = 0;  // tiles: tile loads issued; g: entry loads issued
      bool ok = true;
      for (int it = blockIdx.x; it < total && ok; it += gridDim.x, ++k) {
        const ItemRef r = item_at(p, it);
        const uint32_t ts = k & 1u;
        if (!wait_one(bar(kBarTileEmpty + static_cast<int>(ts)), ((k >> 1) & 1u) ^ 1u, abort_flag, p.timeout_ns)) {
          ok = false;
          break;
        }
        ++tiles;
        const int tb = r.tb >= 0 ? r.tb : r.ta;  // a single-block tile loads its block twice
        ptx::mbar_arrive_expect_tx(bar(kBarTileFull + static_cast<int>(ts)), 2 * kOpBytes);
        ptx::tma_load_2d(tile_op(ts, 0), tmA, bar(kBarTileFull + ts), 0, r.row0 + r.ta * 64, pol);
        ptx::tma_load_2d(tile_op(ts, 0) + kBlkBytes, tmA, bar(kBarTileFull + ts), 0, r.row0 + tb * 64, pol);
        ptx::tma_load_2d(tile_op(ts, 1), tmB, bar(kBarTileFull + ts), 0, r.row0 + r.ta * 64, pol);
        ptx::tma_load_2d(tile_op(ts, 1) + kBlkBytes, tmB, bar(kBarTileFull + ts), 0, r.row0 + tb * 64, pol);
        for (int n = 0; n < r.w.count; ++n) {
          const int blk = static_cast<int>(p.pair_ent[r.w.start + n] & kEntColMask);
          const uint32_t es = g % kEStages;
          if (!wait_one(bar(kBarEntEmpty + static_cast<int>(es)), ((g / kEStages) & 1u) ^ 1u, abort_flag,
                        p.timeout_ns)) {
            ok = false;
            break;
          }
          ++g;
          const uint32_t eb = bar(kBarEntFull + static_cast<int>(es));
          ptx::mbar_arrive_expect_tx(eb, ent_tx);
          ptx::tma_load_2d(ent_op(es, 0), emA, eb, 0, r.row0 + blk * 64, pol);
          ptx::tma_load_2d(ent_op(es, 1), emB, eb, 0, r.row0 + blk * 64, pol);
          if constexpr (kDkv) {
            const uint32_t sv = base + kSmemVec + es * 2 * kVecBytes;
            const size_t off = static_cast<size_t>(r.row0) + static_cast<size_t>(blk) * 64;
            ptx::bulk_load(sv, p.lse2 + off, kVecBytes, eb);
            ptx::bulk_load(sv + kVecBytes, p.dsum + off, kVecBytes, eb);
          }
        }
      }
      if (!ok) {
        // let every copy this thread issued land before the CTA exits: the last
        // issue into ring slot s of a ring of R had index s + R floor((n - 1 - s) / R)
        auto drain = [&](int first_bar, uint32_t n, uint32_t ring) {
          for (uint32_t s = 0; s < ring; ++s)
            if (n > s) {
              const uint32_t last = s + ring * ((n - 1u - s) / ring);
              wait_force(bar(first_bar + static_cast<int>(s)), (last / ring) & 1u, abort_flag, p.timeout_ns);
            }
        };
        drain(kBarTileFull, tiles, 2u);
        drain(kBarEntFull, g, static_cast<uint32_t>(kEStages));
      }
    }
  } else if (warp == kScoreWarp) {
    if (lane == 0) {
      // ---------------- score issuer: S and dP of entry g into score stage g % 2
      uint32_t k = 0, g = 0;
      bool ok = true, issued = false;
      for (int it = blockIdx.x; it < total && ok; it += gridDim.x, ++k) {
        const ItemRef r = item_at(p, it);
        const uint32_t ts = k & 1u;
        if (!wait_one(bar(kBarTileFull + static_cast<int>(ts)), (k >> 1) & 1u, abort_flag, p.timeout_ns)) {
          ok = false;
          break;
        }
        for (int n = 0; n < r.w.count; ++n, ++g) {
          const uint32_t es = g % kEStages, ss = g % kSStages;
          if (!wait_one(bar(kBarEntFull + static_cast<int>(es)), (g / kEStages) & 1u, abort_flag, p.timeout_ns) ||
              !wait_one(bar(kBarScoreFree + static_cast<int>(ss)), ((g / kSStages) & 1u) ^ 1u, abort_flag,
                        p.timeout_ns)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t d = tmem + kTmemScore + 128u * ss;
          mma_rows_x_rows(d, tile_op(ts, 0), ent_op(es, 0));        // S  (or S^T)
          mma_rows_x_rows(d + 64u, tile_op(ts, 1), ent_op(es, 1));  // dP (or dP^T)
          ptx::mma_commit(bar(kBarScoreFull + static_cast<int>(ss)));
          issued = true;
        }
        if (ok) ptx::mma_commit(bar(kBarTileEmpty + static_cast<int>(ts)));
      }
      if (issued) {  // every MMA of this thread done before TMEM is released
        ptx::mma_commit(bar(kBarFinal));
        wait_force(bar(kBarFinal), 0, abort_flag, p.timeout_ns);
      }
    }
  } else if (warp == kAccWarp) {
    if (lane == 0) {
      // ---------------- accumulate issuer
      uint32_t k = 0, g = 0;
      bool ok = true, issued = false;
      for (int it = blockIdx.x; it < total && ok; it += gridDim.x, ++k) {
        const ItemRef r = item_at(p, it);
        const uint32_t as = k % kAccStages;
        if (!wait_one(bar(kBarAccEmpty + static_cast<int>(as)), ((k / kAccStages) & 1u) ^ 1u, abort_flag,
                      p.timeout_ns)) {
          ok = false;
          break;
        }
        const uint32_t acc = tmem + kAccBase + kAccCols * as;
        for (int n = 0; n < r.w.count; ++n, ++g) {
          const uint32_t es = g % kEStages, ss = g % kSStages;
          if (!wait_one(bar(kBarDsFull + static_cast<int>(ss)), (g / kSStages) & 1u, abort_flag, p.timeout_ns)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t sc = tmem + kTmemScore + 128u * ss;
          if constexpr (kDkv) {
            mma_tmem_x_block(acc, sc, ent_op(es, 1), n > 0);              // dV += P^T dO_i
            mma_tmem_x_block(acc + 64u, sc + 64u, ent_op(es, 0), n > 0);  // dK += dS^T Q_i
          } else {
            mma_tmem_x_block(acc, sc, ent_op(es, 0), n > 0);  // dQ += dS K_j
          }
          ptx::mma_commit(bar(kBarScoreFree + static_cast<int>(ss)));
          ptx::mma_commit(bar(kBarEntEmpty + static_cast<int>(es)));
          issued = true;
        }
        if (ok) ptx::mma_commit(bar(kBarAccFull + static_cast<int>(as)));
      }
      if (issued) {
        ptx::mma_commit(bar(kBarFinal + 1));
        wait_force(bar(kBarFinal + 1), 0, abort_flag, p.timeout_ns);
      }
    }
  } else {
    // ---------------- compute warps (the single-lane roles above rejoin their
    // warps below)
    const int quad = warp & 3, ch = warp >> 2;  // TMEM lane quadrant, column half
    const int r = quad * 32 + lane;               // tile row
    const int half = r >> 6;                      // which block of the tile
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    const float sl2 = p.scale_log2;
    uint32_t k = 0, g = 0;
    bool ok = true;
    // the previous tile, whose epilogue runs after this tile's first entry
    bool have_pend = false;
    uint32_t pend_k = 0;
    ItemRef pend{};
    auto epilogue = [&](uint32_t kt, const ItemRef& t) -> bool {
      const uint32_t as = kt % kAccStages;
      if (!wait_warp(bar(kBarAccFull + static_cast<int>(as)), (kt / kAccStages) & 1u, abort_flag, p.timeout_ns))
        return false;
      ptx::tc_fence_after();
      const bool active = half == 0 || t.tb >= 0;
      const size_t grow =
          static_cast<size_t>(t.row0) + static_cast<size_t>(half ? t.tb : t.ta) * 64 + static_cast<size_t>(r & 63);
      const uint32_t acc = tmem + lane_addr + kAccBase + kAccCols * as + 32u * ch;
      float* rec = nullptr;
      if (t.w.rec >= 0)
        rec = p.records + (static_cast<size_t>(t.b) * p.n_records + t.w.rec) * (kDkv ? kBwdDkvRecFloats : kBwdDqRecFloats) +
              static_cast<size_t>(r) * 64 + 32 * ch;
      float v[32];
      if constexpr (kDkv) {
        load32(acc + 64u, v);  // dK
        if (active) store32(v, p.scale, p.dk + grow * 64 + 32 * ch, rec);
        load32(acc, v);  // dV
        if (active) store32(v, 1.f, p.dv + grow * 64 + 32 * ch, rec != nullptr ? rec + kTileRows * 64 : nullptr);
      } else {
        load32(acc, v);
        if (active) store32(v, p.scale, p.dq + grow * 64 + 32 * ch, rec);
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(bar(kBarAccEmpty + static_cast<int>(as)));
      return true;
    };
    for (int it = blockIdx.x; it < total && ok; it += gridDim.x, ++k) {
      const ItemRef t = item_at(p, it);
      const bool active = half == 0 || t.tb >= 0;
      const int blk = half ? t.tb : t.ta;
      // token-level layouts: this row's token (a query for dQ, a key for dK/dV) and
      // whether it is global (it then pairs with every token)
      long long tok_self = 0;
      bool tok_self_global = false;
      if (kTok && active) {
        tok_self = 64ll * blk + (r & 63);
        tok_self_global = (p.tok_gbits[blk] >> (r & 63)) & 1ull;
      }
      // dQ: this row's lse (log2) and D; dKV: whether this key is kept by the padding mask
      float lse2 = INFINITY, drow = 0.f;
      bool key_kept = false;
      if constexpr (kDkv) {
        key_kept = active && (p.keybits == nullptr ||
                              ((p.keybits[static_cast<size_t>(t.b) * p.nb + blk] >> (r & 63)) & 1ull));
      } else if (active) {
        const size_t grow = static_cast<size_t>(t.row0) + static_cast<size_t>(blk) * 64 + (r & 63);
        lse2 = p.lse2[grow];
        drow = p.dsum[grow];
      }
      // the item's union entries, lane x holding entries x and x + 32 (an item has at
      // most 64), handed round by shuffles instead of a global load per entry
      const uint32_t ent_lo = lane < t.w.count ? p.pair_ent[t.w.start + lane] : 0u;
      const uint32_t ent_hi = lane + 32 < t.w.count ? p.pair_ent[t.w.start + lane + 32] : 0u;
      for (int n = 0; n < t.w.count; ++n, ++g) {
        const uint32_t e = __shfl_sync(0xffffffffu, n < 32 ? ent_lo : ent_hi, n & 31);
        const uint32_t ss = g % kSStages, es = g % kEStages;
        if (!wait_warp(bar(kBarScoreFull + static_cast<int>(ss)), (g / kSStages) & 1u, abort_flag, p.timeout_ns)) {
          ok = false;
          break;
        }
        if constexpr (kDkv) {  // the entry's lse2 and D vectors are read from its stage
          if (!wait_warp(bar(kBarEntFull + static_cast<int>(es)), (g / kEStages) & 1u, abort_flag, p.timeout_ns)) {
            ok = false;
            break;
          }
        }
        ptx::tc_fence_after();
        const uint32_t sc = tmem + lane_addr + kTmemScore + 128u * ss + 32u * ch;
        uint32_t s_raw[32], dp_raw[32];
        ptx::tmem_ld32(sc, s_raw);
        ptx::tmem_ld32(sc + 64u, dp_raw);
        ptx::tmem_wait_ld();
        ptx::reg_fence(s_raw);
        ptx::reg_fence(dp_raw);
        const bool member = active && ((e >> (kEntBitsShift + half)) & 1u);
        // the other block's tokens this row pairs with: all, unless the entry is
        // flagged (token level: global tokens, and the band around this row's token)
        unsigned long long pair_mask = ~0ull;
        if (kTok && ((e >> (kEntMaskShift + half)) & 1u) && !tok_self_global) {
          const int ob = static_cast<int>(e & kEntColMask);
          pair_mask = band_bits(tok_self, p.tok_window, ob) | p.tok_gbits[ob];
        }
        if constexpr (kDkv) {
          const bool take = member && key_kept;
          // this warp's 32 queries of the entry's block that this key pairs with (all
          // of them or none at block level)
          const uint32_t qh = take ? static_cast<uint32_t>(pair_mask >> (32 * ch)) : 0u;
          const float* vec = reinterpret_cast<const float*>(smem + kSmemVec + es * 2 * kVecBytes) + 32 * ch;
          uint32_t ppk[16], dpk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float2 l2 = *reinterpret_cast<const float2*>(vec + 2 * c);
            const float2 dd = *reinterpret_cast<const float2*>(vec + 64 + 2 * c);
            const bool t0 = kTok ? ((qh >> (2 * c)) & 1u) != 0u : take;
            const bool t1 = kTok ? ((qh >> (2 * c + 1)) & 1u) != 0u : take;
            const float p0 = t0 ? ptx::ex2_approx(__uint_as_float(s_raw[2 * c]) * sl2 - l2.x) : 0.f;
            const float p1 = t1 ? ptx::ex2_approx(__uint_as_float(s_raw[2 * c + 1]) * sl2 - l2.y) : 0.f;
            ppk[c] = pack_bf16x2(p0, p1);
            dpk[c] = pack_bf16x2(p0 * (__uint_as_float(dp_raw[2 * c]) - dd.x),
                                 p1 * (__uint_as_float(dp_raw[2 * c + 1]) - dd.y));
          }
          ptx::tmem_st16(sc, ppk);         // P^T over S^T columns this warp has read
          ptx::tmem_st16(sc + 64u, dpk);   // dS^T over dP^T columns this warp has read
        } else {
          unsigned long long mk = 0ull;
          if (member)
            mk = (p.keybits != nullptr ? p.keybits[static_cast<size_t>(t.b) * p.nb + (e & kEntColMask)] : ~0ull) &
                 pair_mask;
          const uint32_t mh = static_cast<uint32_t>(mk >> (32 * ch));  // this warp's 32 keys
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float p0 = ((mh >> (2 * c)) & 1u) ? ptx::ex2_approx(__uint_as_float(s_raw[2 * c]) * sl2 - lse2) : 0.f;
            const float p1 =
                ((mh >> (2 * c + 1)) & 1u) ? ptx::ex2_approx(__uint_as_float(s_raw[2 * c + 1]) * sl2 - lse2) : 0.f;
            pk[c] = pack_bf16x2(p0 * (__uint_as_float(dp_raw[2 * c]) - drow),
                                p1 * (__uint_as_float(dp_raw[2 * c + 1]) - drow));
          }
          ptx::tmem_st16(sc, pk);  // dS over S columns this warp has read
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar(kBarDsFull + static_cast<int>(ss)));
        if (n == 0 && have_pend) {
          have_pend = false;
          if (!epilogue(pend_k, pend)) {
            ok = false;
            break;
          }
        }
      }
      ok = ok && !*abort_flag;
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      have_pend = true;
      pend_k = k;
      pend = t;
    }
    if (ok && have_pend) epilogue(pend_k, pend);
  }

  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == kScoreWarp) ptx::tmem_dealloc(tmem, kTmemCols);
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
int g_sms[kMaxDevices];

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
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaFuncSetAttribute(bsa_bwd_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemAlloc)) != cudaSuccess ||
        cudaFuncSetAttribute(bsa_bwd_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemAlloc)) != cudaSuccess ||
        cudaFuncSetAttribute(bsa_bwd_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemAlloc)) != cudaSuccess ||
        cudaFuncSetAttribute(bsa_bwd_kernel<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemAlloc)) != cudaSuccess) {
      g_setup_status[dev] = BSA_ERR_CUDA;
      return;
    }
    g_sms[dev] = sms;
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
  prm.tok_gbits = lay->token ? lay->d_tok_gbits : nullptr;
  prm.tok_window = lay->tok_window;
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
  pq.n_items = static_cast<int>(lay->dq_plan.items.size());
  const int64_t gq = std::min<int64_t>(static_cast<int64_t>(B) * pq.n_items, g_sms[dev]);
  if (gq > 0) {
    if (lay->token)
      bsa_bwd_kernel<false, true><<<static_cast<unsigned>(gq), kThreads, kSmemAlloc, s>>>(pq);
    else
      bsa_bwd_kernel<false, false><<<static_cast<unsigned>(gq), kThreads, kSmemAlloc, s>>>(pq);
    if (cudaGetLastError() != cudaSuccess) return BSA_ERR_CUDA;
  }
  // dK and dV over the key tiles
  BwdParams pk = prm;
  pk.items = lay->d_dkv_items;
  pk.pair = lay->d_kpair_q;
  pk.pair_ent = lay->d_kpair_ent;
  pk.records = reinterpret_cast<float*>(ws + plan.dkv_rec_off);
  pk.n_records = lay->dkv_plan.n_records;
  pk.n_items = static_cast<int>(lay->dkv_plan.items.size());
  const int64_t gk = std::min<int64_t>(static_cast<int64_t>(B) * pk.n_items, g_sms[dev]);
  if (gk > 0) {
    if (lay->token)
      bsa_bwd_kernel<true, true><<<static_cast<unsigned>(gk), kThreads, kSmemAlloc, s>>>(pk);
    else
      bsa_bwd_kernel<true, false><<<static_cast<unsigned>(gk), kThreads, kSmemAlloc, s>>>(pk);
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
