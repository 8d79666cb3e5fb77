// Internal structures shared by the host library (bsa_host.cpp) and the CUDA
// forward (bsa_fwd_sm100.cu) and backward (bsa_bwd_sm100.cu).  Not part of the
// public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <vector>

#include "../../include/bsa.h"

namespace bsa {

// Tile geometry.  A tile is 128 query rows = two 64-row query blocks that run
// over the sorted union of their key-block lists (tcgen05's M = 128 datapath).
constexpr int kBlock = 64;
constexpr int kHeadDim = 64;
constexpr int kTileRows = 128;

// A tile whose key-block union is longer than kSplitThreshold is cut into
// chunks of kSplitChunk union entries, each run as its own work item.  Each chunk
// writes a partial (O, m, l) record; a second kernel merges a split tile's records
// into its output rows.
constexpr int kSplitThreshold = BSA_SPLIT_THRESHOLD;
constexpr int kSplitChunk = BSA_SPLIT_CHUNK;

// Partial record of one split chunk: O[128][d] fp32 (unnormalised, relative to
// the chunk's running max), then m[128] (log2 units, scaled) and l[128].
constexpr int rec_floats(int d) { return kTileRows * d + 2 * kTileRows; }
constexpr int kRecFloats = rec_floats(kHeadDim);

// One unit of the static schedule (32 bytes, read with two 16-byte loads).
struct WorkItem {
  int32_t h;         // head
  int32_t pair;      // tile (query-block pair) index within the head
  int32_t start;     // first entry in pair_ent (absolute index)
  int32_t count;     // number of union entries processed by this item (>= 1)
  int32_t split;     // -1: whole tile; otherwise split-tile index within a batch element
  int32_t rec;       // partial record index within a batch element (split only)
  int32_t nchunks;   // number of chunks of the split tile
  int32_t rec_base;  // first record of the split tile within a batch element
};
static_assert(sizeof(WorkItem) == 32, "WorkItem must stay 32 bytes");

// A split tile, for the merge: its head, query blocks (qb = -1: single block) and
// its records [rec_base, rec_base + nchunks) within a batch element.
struct SplitTile {
  int32_t h, qa, qb, rec_base, nchunks;
  int32_t pad[3];
};
static_assert(sizeof(SplitTile) == 32, "SplitTile must stay 32 bytes");

// One work item of the backward kernels: a whole tile, or one chunk of a split
// tile (rec >= 0: its partial record index within a batch element).
struct BwdItem {
  int32_t h, pair, start, count, rec;
  int32_t pad[3];
};
static_assert(sizeof(BwdItem) == 32, "BwdItem must stay 32 bytes");

// Tiles of 128 rows over a block CSR: pair_q (2 per tile), pair_ptr (H*n_pairs+1),
// pair_ent (key block | membership << 24).
struct TileSet {
  std::vector<int32_t> pair_q;
  int n_pairs = 0;
  std::vector<int32_t> pair_ptr;
  std::vector<uint32_t> pair_ent;
};

// Work list of a backward kernel over a TileSet: split-tile chunks first, then
// whole tiles, longest first; the split tiles for the merge.
struct BwdPlan {
  std::vector<BwdItem> items;
  std::vector<SplitTile> splits;
  int n_records = 0;
};

constexpr uint32_t kEntColMask = 0x00FFFFFFu;
constexpr int kEntBitsShift = 24;
// Token-level layouts: bit kEntMaskShift + half set when that half's rows need a
// per-row mask in the entry (not every pair of the two blocks is allowed).
constexpr int kEntMaskShift = 26;

}  // namespace bsa

struct bsa_layout {
  // block: the caller's block size (a multiple of 64); nb: 64-key blocks, L / 64,
  // the granularity every table below and every kernel works at
  int H = 0, L = 0, block = 0, nb = 0;
  int window = 0, n_global = 0, n_random = 0;
  uint64_t seed = 0;
  std::vector<int32_t> globals;     // sorted, distinct, in the caller's block units
  std::vector<int32_t> row_ptr;     // H*nb + 1 (64-key blocks)
  std::vector<int32_t> col_idx;     // nnz (64-key blocks)
  // the layout in the caller's block units when block > 64 (H*(L/block) + 1 and
  // its columns); row (h, I) at block 64 m is rows (h, m I .. m I + m - 1) of
  // the tables above, each listing blocks m J .. m J + m - 1 for J in row (h, I)
  std::vector<int32_t> user_row_ptr, user_col_idx;
  // token-level layouts (bsa_layout_build_tokens): the window in tokens, one bit per
  // global token (word j: the tokens of block j), and per CSR entry whether the
  // block pair needs a per-row mask (not every pair of tokens allowed)
  bool token = false;
  int64_t tok_window = 0;
  std::vector<uint64_t> tok_gbits;
  std::vector<uint8_t> tok_masked;
  std::vector<int32_t> pair_q;      // 2 * n_pairs
  int n_pairs = 0;
  std::vector<int32_t> pair_ptr;    // H*n_pairs + 1
  std::vector<uint32_t> pair_ent;   // union entries
  std::vector<bsa::WorkItem> items; // schedule for ONE batch element (head-major)
  // the same items head by head, each head's split chunks first: item indices, for the
  // forward's order when one head's work is long enough to hand out its split chunks
  // just before its other tiles (its K/V then stay in L2)
  std::vector<int32_t> head_order;
  std::vector<bsa::SplitTile> splits;  // the split tiles of one batch element
  int n_split = 0;                  // split tiles per batch element
  int n_records = 0;                // partial records per batch element
  // backward: key-major tiles (pairs of key blocks over the union of the query
  // blocks that attend them) and the work lists of its two kernels
  bsa::TileSet ktiles;
  bsa::BwdPlan dq_plan, dkv_plan;
  // device copies (bsa_layout_upload)
  int device = -1;
  int32_t* d_pair_q = nullptr;
  uint32_t* d_pair_ent = nullptr;
  bsa::WorkItem* d_items = nullptr;
  int32_t* d_head_order = nullptr;
  bsa::SplitTile* d_splits = nullptr;
  int32_t* d_kpair_q = nullptr;
  uint32_t* d_kpair_ent = nullptr;
  bsa::BwdItem* d_dq_items = nullptr;
  bsa::BwdItem* d_dkv_items = nullptr;
  bsa::SplitTile* d_dq_splits = nullptr;
  unsigned long long* d_tok_gbits = nullptr;
  bsa::SplitTile* d_dkv_splits = nullptr;
};

namespace bsa {
// Workspace carve-up for batch size B (all offsets 256-byte aligned).
struct WorkspacePlan {
  // [sched_off, +sched_bytes): the area that must be zero before a call and is
  // zero again after one: the work-item counter and finished-slot counter of the
  // dynamic schedule.
  size_t sched_off, sched_bytes;
  size_t keybits_off, keybits_bytes;
  size_t partials_off, partials_bytes;
  size_t total;
};
WorkspacePlan plan_workspace(const bsa_layout& lay, int B, int d = kHeadDim);
// Backward workspace for batch size B: key-padding bits, D = rowsum(dO * O) and
// lse in log2 units per row, and the partial records of split tiles (dQ: 128 x 64
// floats each; dK and dV: 2 x 128 x 64 floats each).
struct BwdWorkspacePlan {
  size_t keybits_off, dsum_off, lse2_off, dq_rec_off, dkv_rec_off, total;
};
BwdWorkspacePlan plan_bwd_workspace(const bsa_layout& lay, int B);
constexpr int kBwdDqRecFloats = kTileRows * kHeadDim;
constexpr int kBwdDkvRecFloats = 2 * kTileRows * kHeadDim;
void free_device(bsa_layout* lay);
}  // namespace bsa
