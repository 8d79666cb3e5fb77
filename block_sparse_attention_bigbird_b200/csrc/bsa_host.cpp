// Host side of the BigBird block-sparse attention library: the seeded layout
// builder, layouts from a caller's block CSR, the 128-row tile decomposition
// (query-major for the forward and dQ, key-major over the transposed layout for
// dK and dV) and the work lists.  Pure C++, no GPU needed.  Every entry point
// validates its arguments and returns a bsa_status; no exception crosses the C
// ABI.
#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <new>

#include "bsa_internal.h"

namespace {

// ---------------------------------------------------------------------------
// Philox4x64-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy
// as 1, 2, 3", SC'11): a counter-based generator.  Each of the ten rounds
// multiplies counter words 0 and 2 by two fixed 64-bit constants, swaps the
// halves across the words and xors in the round key; the key is bumped by two
// Weyl constants (golden ratio and sqrt(3)-1 in 64-bit fixed point) between
// rounds.  The stream here follows the convention of numpy's Philox bit
// generator: the 256-bit counter is incremented BEFORE each 4-word block is
// produced and the words of a block are handed out in order 0..3.
// ---------------------------------------------------------------------------
constexpr uint64_t kPhiloxM0 = 0xD2E7470EE14C6C93ull;
constexpr uint64_t kPhiloxM1 = 0xCA5A826395121157ull;
constexpr uint64_t kPhiloxW0 = 0x9E3779B97F4A7C15ull;
constexpr uint64_t kPhiloxW1 = 0xBB67AE8584CAA73Bull;

inline void mulhilo64(uint64_t a, uint64_t b, uint64_t* hi, uint64_t* lo) {
  unsigned __int128 p = static_cast<unsigned __int128>(a) * b;
  *hi = static_cast<uint64_t>(p >> 64);
  *lo = static_cast<uint64_t>(p);
}

void philox4x64_10(const uint64_t in[4], const uint64_t key_in[2], uint64_t out[4]) {
  uint64_t c0 = in[0], c1 = in[1], c2 = in[2], c3 = in[3];
  uint64_t k0 = key_in[0], k1 = key_in[1];
  for (int round = 0; round < 10; ++round) {
    if (round > 0) {
      k0 += kPhiloxW0;
      k1 += kPhiloxW1;
    }
    uint64_t hi0, lo0, hi1, lo1;
    mulhilo64(kPhiloxM0, c0, &hi0, &lo0);
    mulhilo64(kPhiloxM1, c2, &hi1, &lo1);
    const uint64_t n0 = hi1 ^ c1 ^ k0;
    const uint64_t n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
  out[0] = c0;
  out[1] = c1;
  out[2] = c2;
  out[3] = c3;
}

class PhiloxStream {
 public:
  PhiloxStream(uint64_t seed, uint64_t i, uint64_t h) {
    ctr_[0] = 0;
    ctr_[1] = i;
    ctr_[2] = h;
    ctr_[3] = 0;
    key_[0] = seed;
    key_[1] = 0;
  }
  uint64_t next() {
    if (pos_ == 4) {
      for (int w = 0; w < 4; ++w) {  // 256-bit little-endian increment
        if (++ctr_[w] != 0) break;
      }
      philox4x64_10(ctr_, key_, buf_);
      pos_ = 0;
    }
    return buf_[pos_++];
  }

 private:
  uint64_t ctr_[4];
  uint64_t key_[2];
  uint64_t buf_[4] = {0, 0, 0, 0};
  int pos_ = 4;
};

// k-th (0-based) block of [0, nb) that is not in the sorted list `excl`.
inline int kth_free(int k, const std::vector<int>& excl) {
  int v = k;
  for (int e : excl) {
    if (e <= v)
      ++v;
    else
      break;
  }
  return v;
}

// One row of the layout (BigBird: window + globals + random, see bsa.h).
void build_row(int h, int i, int nb, int window, const std::vector<int32_t>& globals,
               const std::vector<uint8_t>& is_global, int n_random, uint64_t seed,
               std::vector<int32_t>* row) {
  row->clear();
  if (is_global[i]) {
    for (int j = 0; j < nb; ++j) row->push_back(j);
    return;
  }
  const int lo = std::max(0, i - window);
  const int hi = std::min(nb - 1, i + window);
  // excluded = window U globals, sorted and distinct
  std::vector<int> excl;
  excl.reserve(static_cast<size_t>(hi - lo + 1) + globals.size());
  for (int j = lo; j <= hi; ++j) excl.push_back(j);
  for (int g : globals)
    if (g < lo || g > hi) excl.push_back(g);
  std::sort(excl.begin(), excl.end());
  const int m = nb - static_cast<int>(excl.size());
  const int take = std::min(n_random, m);
  // Partial Fisher-Yates over the ascending candidate list C (implicit: C[k] =
  // kth_free(k)), touching only the positions the shuffle swaps.
  std::vector<std::pair<int, int>> swapped;  // position -> candidate index
  auto get = [&](int pos) {
    for (const auto& s : swapped)
      if (s.first == pos) return s.second;
    return pos;
  };
  auto set = [&](int pos, int val) {
    for (auto& s : swapped)
      if (s.first == pos) {
        s.second = val;
        return;
      }
    swapped.emplace_back(pos, val);
  };
  std::vector<int> rnd;
  rnd.reserve(static_cast<size_t>(take));
  PhiloxStream rng(seed, static_cast<uint64_t>(i), static_cast<uint64_t>(h));
  for (int t = 0; t < take; ++t) {
    const uint64_t u = rng.next();
    const int j = t + static_cast<int>(u % static_cast<uint64_t>(m - t));
    const int ct = get(t), cj = get(j);
    set(t, cj);
    set(j, ct);
    rnd.push_back(kth_free(cj, excl));
  }
  row->insert(row->end(), excl.begin(), excl.end());
  row->insert(row->end(), rnd.begin(), rnd.end());
  std::sort(row->begin(), row->end());
}

}  // namespace

namespace bsa {

WorkspacePlan plan_workspace(const bsa_layout& lay, int B, int d) {
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  WorkspacePlan p{};
  p.sched_off = 0;
  p.sched_bytes = up(2 * sizeof(int32_t));
  p.keybits_off = p.sched_off + p.sched_bytes;
  p.keybits_bytes = up(sizeof(uint64_t) * static_cast<size_t>(B) * lay.nb);
  p.partials_off = p.keybits_off + p.keybits_bytes;
  p.partials_bytes =
      up(sizeof(float) * static_cast<size_t>(rec_floats(d)) * static_cast<size_t>(B) * lay.n_records);
  p.total = p.partials_off + p.partials_bytes;
  return p;
}

BwdWorkspacePlan plan_bwd_workspace(const bsa_layout& lay, int B) {
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  const size_t rows = static_cast<size_t>(B) * lay.H * lay.L;
  BwdWorkspacePlan p{};
  p.keybits_off = 0;
  p.dsum_off = up(sizeof(uint64_t) * static_cast<size_t>(B) * lay.nb);
  p.lse2_off = p.dsum_off + up(sizeof(float) * rows);
  p.dq_rec_off = p.lse2_off + up(sizeof(float) * rows);
  p.dkv_rec_off = p.dq_rec_off + up(sizeof(float) * kBwdDqRecFloats * static_cast<size_t>(B) * lay.dq_plan.n_records);
  p.total = p.dkv_rec_off + up(sizeof(float) * kBwdDkvRecFloats * static_cast<size_t>(B) * lay.dkv_plan.n_records);
  return p;
}

}  // namespace bsa

namespace {

// Tiles of 128 rows over a block CSR (H x nb rows, head-major): rows paired in
// ascending order, the dense ones (flagged) with each other and the others with
// each other; an odd one out forms a single-row tile.  Per tile and head the
// entries are the union of the two rows with membership bits: the blocks in both
// rows, then the blocks in one row only, alternating first/second, each group
// ascending.  The order is free (one softmax over the union), and this one keeps
// the two halves of the tile -- whose warps skip the work of a block their half
// does not take part in -- doing equal work chunk by chunk.  `masked` (optional, one
// flag per CSR entry) marks block pairs that need a per-row mask; an entry carries the
// flag of each row it comes from at bit kEntMaskShift + half.
void make_tiles(int H, int nb, const std::vector<int32_t>& row_ptr, const std::vector<int32_t>& col_idx,
                const std::vector<uint8_t>& dense, std::vector<int32_t>* pair_q, int* n_pairs,
                std::vector<int32_t>* pair_ptr, std::vector<uint32_t>* pair_ent,
                const std::vector<uint8_t>* masked = nullptr) {
  std::vector<int32_t> gl, ng;
  for (int i = 0; i < nb; ++i) (dense[static_cast<size_t>(i)] ? gl : ng).push_back(i);
  pair_q->clear();
  for (const auto* lst : {&gl, &ng}) {
    for (size_t x = 0; x < lst->size(); x += 2) {
      pair_q->push_back((*lst)[x]);
      pair_q->push_back(x + 1 < lst->size() ? (*lst)[x + 1] : -1);
    }
  }
  *n_pairs = static_cast<int>(pair_q->size() / 2);
  const int P = *n_pairs;
  pair_ptr->assign(1, 0);
  pair_ent->clear();
  std::vector<uint32_t> both, only_a, only_b;
  for (int h = 0; h < H; ++h) {
    for (int p = 0; p < P; ++p) {
      const int qa = (*pair_q)[2 * p], qb = (*pair_q)[2 * p + 1];
      const int32_t* ra = col_idx.data() + row_ptr[static_cast<size_t>(h) * nb + qa];
      const int32_t* ra_end = col_idx.data() + row_ptr[static_cast<size_t>(h) * nb + qa + 1];
      const int32_t* rb = ra_end;
      const int32_t* rb_end = ra_end;
      if (qb >= 0) {
        rb = col_idx.data() + row_ptr[static_cast<size_t>(h) * nb + qb];
        rb_end = col_idx.data() + row_ptr[static_cast<size_t>(h) * nb + qb + 1];
      }
      both.clear();
      only_a.clear();
      only_b.clear();
      // the masked bits of the entry at CSR position x, for half hf
      auto mbit = [&](const int32_t* x, int hf) -> uint32_t {
        return (masked != nullptr && (*masked)[static_cast<size_t>(x - col_idx.data())])
                   ? (1u << (bsa::kEntMaskShift + hf))
                   : 0u;
      };
      while (ra != ra_end || rb != rb_end) {
        if (rb == rb_end || (ra != ra_end && *ra < *rb)) {
          only_a.push_back(static_cast<uint32_t>(*ra) | (1u << bsa::kEntBitsShift) | mbit(ra, 0));
          ++ra;
        } else if (ra == ra_end || *rb < *ra) {
          only_b.push_back(static_cast<uint32_t>(*rb) | (2u << bsa::kEntBitsShift) | mbit(rb, 1));
          ++rb;
        } else {
          both.push_back(static_cast<uint32_t>(*ra) | (3u << bsa::kEntBitsShift) | mbit(ra, 0) | mbit(rb, 1));
          ++ra;
          ++rb;
        }
      }
      pair_ent->insert(pair_ent->end(), both.begin(), both.end());
      for (size_t x = 0; x < std::max(only_a.size(), only_b.size()); ++x) {
        if (x < only_a.size()) pair_ent->push_back(only_a[x]);
        if (x < only_b.size()) pair_ent->push_back(only_b[x]);
      }
      // A tile whose rows are all empty (possible in a caller's CSR) still runs one
      // entry so that its output rows get written (zeros): block 0 with no
      // membership bit, which neither half takes part in.
      if (both.empty() && only_a.empty() && only_b.empty()) pair_ent->push_back(0u);
      pair_ptr->push_back(static_cast<int32_t>(pair_ent->size()));
    }
  }
}

// Work list of a backward kernel: first the chunks of the tiles whose union is
// longer than kSplitThreshold (kSplitChunk entries each, every one writing a
// partial record), then the other tiles, longest first.
void make_bwd_plan(int H, const std::vector<int32_t>& pair_q, int P, const std::vector<int32_t>& pair_ptr,
                   bsa::BwdPlan* plan) {
  plan->items.clear();
  plan->splits.clear();
  plan->n_records = 0;
  std::vector<bsa::BwdItem> whole;
  for (int h = 0; h < H; ++h) {
    for (int p = 0; p < P; ++p) {
      const int32_t s = pair_ptr[static_cast<size_t>(h) * P + p];
      const int32_t U = pair_ptr[static_cast<size_t>(h) * P + p + 1] - s;
      if (U <= bsa::kSplitThreshold) {
        whole.push_back(bsa::BwdItem{h, p, s, U, -1, {0, 0, 0}});
        continue;
      }
      const int nch = (U + bsa::kSplitChunk - 1) / bsa::kSplitChunk;
      const int base = plan->n_records;
      plan->n_records += nch;
      plan->splits.push_back(bsa::SplitTile{h, pair_q[2 * p], pair_q[2 * p + 1], base, nch, {0, 0, 0}});
      for (int c = 0; c < nch; ++c) {
        const int cs = c * bsa::kSplitChunk;
        plan->items.push_back(bsa::BwdItem{h, p, s + cs, std::min(bsa::kSplitChunk, U - cs), base + c, {0, 0, 0}});
      }
    }
  }
  std::stable_sort(whole.begin(), whole.end(),
                   [](const bsa::BwdItem& a, const bsa::BwdItem& b) { return a.count > b.count; });
  plan->items.insert(plan->items.end(), whole.begin(), whole.end());
}

// dense[i]: 64-key query block i lists every key block in every head (it pairs
// with other such blocks).
void build_tiles(bsa_layout* lay, const std::vector<uint8_t>& dense) {
  const int nb = lay->nb, H = lay->H;
  make_tiles(H, nb, lay->row_ptr, lay->col_idx, dense, &lay->pair_q, &lay->n_pairs, &lay->pair_ptr,
             &lay->pair_ent, lay->token ? &lay->tok_masked : nullptr);
  const int P = lay->n_pairs;
  // Work items of one batch element: first the chunks of split tiles (the longest
  // items, kept away from the end of the element's run), then the other tiles,
  // head-major so that items running at the same time share the head's K/V in L2.
  // The forward hands out every item of one batch element before the next one's.
  lay->items.clear();
  lay->splits.clear();
  lay->n_split = 0;
  lay->n_records = 0;
  for (const bool split_pass : {true, false}) {
    for (int h = 0; h < H; ++h) {
      for (int p = 0; p < P; ++p) {
        const int32_t s = lay->pair_ptr[static_cast<size_t>(h) * P + p];
        const int32_t U = lay->pair_ptr[static_cast<size_t>(h) * P + p + 1] - s;
        const bool split = U > bsa::kSplitThreshold;
        if (split != split_pass) continue;
        if (!split) {
          lay->items.push_back(bsa::WorkItem{h, p, s, U, -1, 0, 1, 0});
          continue;
        }
        const int nch = (U + bsa::kSplitChunk - 1) / bsa::kSplitChunk;
        const int slot = lay->n_split++;
        const int base = lay->n_records;
        lay->n_records += nch;
        lay->splits.push_back(bsa::SplitTile{h, lay->pair_q[2 * p], lay->pair_q[2 * p + 1], base, nch, {0, 0, 0}});
        for (int c = 0; c < nch; ++c) {
          const int cs = c * bsa::kSplitChunk;
          lay->items.push_back(bsa::WorkItem{h, p, s + cs, std::min(bsa::kSplitChunk, U - cs),
                                             slot, base + c, nch, base});
        }
      }
    }
  }
  lay->head_order.clear();
  for (int h = 0; h < H; ++h)
    for (const bool split_pass : {true, false})
      for (size_t x = 0; x < lay->items.size(); ++x)
        if (lay->items[x].h == h && (lay->items[x].split >= 0) == split_pass)
          lay->head_order.push_back(static_cast<int32_t>(x));
  // Backward.  dQ runs over the same query tiles.  dK and dV run over key tiles:
  // the transposed CSR (row (h, j) = the query blocks whose row holds key block j,
  // ascending) cut into tiles the same way, the key blocks every query block
  // attends in every head (BigBird's globals) paired with each other.
  make_bwd_plan(H, lay->pair_q, P, lay->pair_ptr, &lay->dq_plan);
  std::vector<int32_t> t_ptr(static_cast<size_t>(H) * nb + 1, 0), t_col(lay->col_idx.size());
  for (int h = 0; h < H; ++h)
    for (int i = 0; i < nb; ++i)
      for (int32_t x = lay->row_ptr[static_cast<size_t>(h) * nb + i];
           x < lay->row_ptr[static_cast<size_t>(h) * nb + i + 1]; ++x)
        ++t_ptr[static_cast<size_t>(h) * nb + lay->col_idx[static_cast<size_t>(x)] + 1];
  for (size_t x = 0; x + 1 < t_ptr.size(); ++x) t_ptr[x + 1] += t_ptr[x];
  std::vector<int32_t> fill(t_ptr.begin(), t_ptr.end() - 1);
  // a token-level layout's per-pair mask flags follow their entries into the transpose
  std::vector<uint8_t> t_masked(lay->token ? lay->col_idx.size() : 0);
  for (int h = 0; h < H; ++h)
    for (int i = 0; i < nb; ++i)
      for (int32_t x = lay->row_ptr[static_cast<size_t>(h) * nb + i];
           x < lay->row_ptr[static_cast<size_t>(h) * nb + i + 1]; ++x) {
        const size_t dst =
            static_cast<size_t>(fill[static_cast<size_t>(h) * nb + lay->col_idx[static_cast<size_t>(x)]]++);
        t_col[dst] = i;
        if (lay->token) t_masked[dst] = lay->tok_masked[static_cast<size_t>(x)];
      }
  std::vector<uint8_t> kdense(static_cast<size_t>(nb), 1);
  for (int h = 0; h < H; ++h)
    for (int j = 0; j < nb; ++j)
      if (t_ptr[static_cast<size_t>(h) * nb + j + 1] - t_ptr[static_cast<size_t>(h) * nb + j] != nb)
        kdense[static_cast<size_t>(j)] = 0;
  make_tiles(H, nb, t_ptr, t_col, kdense, &lay->ktiles.pair_q, &lay->ktiles.n_pairs, &lay->ktiles.pair_ptr,
             &lay->ktiles.pair_ent, lay->token ? &t_masked : nullptr);
  make_bwd_plan(H, lay->ktiles.pair_q, lay->ktiles.n_pairs, lay->ktiles.pair_ptr, &lay->dkv_plan);
}

// Expands a CSR over blocks of 64 m keys (H x nbu rows, head-major, rows
// ascending) to 64-key blocks: row (h, m I + t) lists m J + u, u = 0 .. m - 1, for
// every J in row (h, I).  Attention restricted to (64 m)-blocks is exactly
// attention restricted to these 64-blocks.  False if the result would not fit
// int32 offsets.
bool expand_csr(int H, int nbu, int m, const std::vector<int32_t>& rp, const std::vector<int32_t>& ci,
                std::vector<int32_t>* rp64, std::vector<int32_t>* ci64) {
  if (static_cast<int64_t>(ci.size()) * m * m > INT32_MAX) return false;
  rp64->assign(1, 0);
  ci64->clear();
  ci64->reserve(ci.size() * static_cast<size_t>(m) * m);
  for (int h = 0; h < H; ++h)
    for (int I = 0; I < nbu; ++I) {
      const size_t r = static_cast<size_t>(h) * nbu + I;
      for (int t = 0; t < m; ++t) {
        for (int32_t x = rp[r]; x < rp[r + 1]; ++x)
          for (int u = 0; u < m; ++u) ci64->push_back(ci[static_cast<size_t>(x)] * m + u);
        rp64->push_back(static_cast<int32_t>(ci64->size()));
      }
    }
  return true;
}

// Stores a layout given in the caller's block units (rows ascending and
// duplicate-free) at 64-key granularity, and builds its tiles.  dense_user[I]:
// block I's row lists every block in every head.  False on int32 overflow.
bool set_rows(bsa_layout* lay, std::vector<int32_t> urp, std::vector<int32_t> uci,
              const std::vector<uint8_t>& dense_user) {
  const int m = lay->block / bsa::kBlock, nbu = lay->L / lay->block;
  std::vector<uint8_t> dense(static_cast<size_t>(lay->nb), 0);
  for (int I = 0; I < nbu; ++I)
    for (int u = 0; u < m; ++u) dense[static_cast<size_t>(I) * m + u] = dense_user[static_cast<size_t>(I)];
  if (m == 1) {
    lay->row_ptr = std::move(urp);
    lay->col_idx = std::move(uci);
  } else {
    if (!expand_csr(lay->H, nbu, m, urp, uci, &lay->row_ptr, &lay->col_idx)) return false;
    lay->user_row_ptr = std::move(urp);
    lay->user_col_idx = std::move(uci);
  }
  build_tiles(lay, dense);
  return lay->pair_ent.size() <= static_cast<size_t>(INT32_MAX) &&
         lay->ktiles.pair_ent.size() <= static_cast<size_t>(INT32_MAX);
}

}  // namespace

extern "C" {

int bsa_layout_build(int H, int L, int block, int window, int n_global, int n_random,
                     uint64_t seed, const int32_t* globals, bsa_layout** out) {
  if (out == nullptr) return BSA_ERR_INVALID_ARG;
  *out = nullptr;
  if (block < bsa::kBlock || block % bsa::kBlock != 0) return BSA_ERR_UNSUPPORTED;
  if (H < 1 || L < 1 || L % block != 0 || window < 0 || n_global < 0 || n_random < 0)
    return BSA_ERR_INVALID_ARG;
  const int nb = L / block;  // the caller's blocks; the kernels run L / 64 blocks of 64
  if (L / bsa::kBlock > static_cast<int>(bsa::kEntColMask) || static_cast<int64_t>(H) * (L / bsa::kBlock) > (1 << 30))
    return BSA_ERR_INVALID_ARG;
  bsa_layout* lay = new (std::nothrow) bsa_layout();
  if (lay == nullptr) return BSA_ERR_OOM;
  try {
    lay->H = H;
    lay->L = L;
    lay->block = block;
    lay->nb = L / bsa::kBlock;
    lay->window = window;
    lay->n_global = n_global;
    lay->n_random = n_random;
    lay->seed = seed;
    // globals
    std::vector<int32_t> g;
    if (globals != nullptr) {
      for (int x = 0; x < n_global; ++x) {
        if (globals[x] < 0 || globals[x] >= nb) {
          delete lay;
          return BSA_ERR_INVALID_ARG;
        }
        g.push_back(globals[x]);
      }
    } else if (n_global == 1) {
      g.push_back(0);
    } else if (n_global >= 2) {
      for (int k = 0; k < n_global; ++k)
        g.push_back(static_cast<int32_t>((static_cast<int64_t>(k) * (nb - 1)) / (n_global - 1)));
    }
    std::sort(g.begin(), g.end());
    g.erase(std::unique(g.begin(), g.end()), g.end());
    lay->globals = g;
    std::vector<uint8_t> is_global(static_cast<size_t>(nb), 0);
    for (int x : g) is_global[static_cast<size_t>(x)] = 1;
    // CSR rows in the caller's block units, head-major
    std::vector<int32_t> urp, uci, row;
    urp.reserve(static_cast<size_t>(H) * nb + 1);
    urp.push_back(0);
    for (int h = 0; h < H; ++h) {
      for (int i = 0; i < nb; ++i) {
        build_row(h, i, nb, window, g, is_global, n_random, seed, &row);
        uci.insert(uci.end(), row.begin(), row.end());
        if (uci.size() > static_cast<size_t>(INT32_MAX)) {
          delete lay;
          return BSA_ERR_INVALID_ARG;
        }
        urp.push_back(static_cast<int32_t>(uci.size()));
      }
    }
    if (!set_rows(lay, std::move(urp), std::move(uci), is_global)) {
      delete lay;
      return BSA_ERR_INVALID_ARG;
    }
  } catch (const std::bad_alloc&) {
    delete lay;
    return BSA_ERR_OOM;
  } catch (...) {
    delete lay;
    return BSA_ERR_INVALID_ARG;
  }
  *out = lay;
  return BSA_OK;
}

int bsa_layout_build_tokens(int H, int L, int window, int n_global, int n_random, uint64_t seed,
                            const int32_t* global_tokens, bsa_layout** out) {
  if (out == nullptr) return BSA_ERR_INVALID_ARG;
  *out = nullptr;
  if (H < 1 || L < bsa::kBlock || L % bsa::kBlock != 0 || window < 0 || n_global < 0 || n_random < 0)
    return BSA_ERR_INVALID_ARG;
  const int nb = L / bsa::kBlock;
  if (nb > static_cast<int>(bsa::kEntColMask) || static_cast<int64_t>(H) * nb > (1 << 30)) return BSA_ERR_INVALID_ARG;
  bsa_layout* lay = new (std::nothrow) bsa_layout();
  if (lay == nullptr) return BSA_ERR_OOM;
  try {
    lay->H = H;
    lay->L = L;
    lay->block = bsa::kBlock;
    lay->nb = nb;
    lay->n_random = n_random;
    lay->seed = seed;
    // global tokens: the caller's, or the linspace rule over tokens
    std::vector<int64_t> g;
    if (global_tokens != nullptr) {
      for (int x = 0; x < n_global; ++x) {
        if (global_tokens[x] < 0 || global_tokens[x] >= L) {
          delete lay;
          return BSA_ERR_INVALID_ARG;
        }
        g.push_back(global_tokens[x]);
      }
    } else if (n_global == 1) {
      g.push_back(0);
    } else if (n_global >= 2) {
      for (int k = 0; k < n_global; ++k) g.push_back((static_cast<int64_t>(k) * (L - 1)) / (n_global - 1));
    }
    lay->tok_gbits.assign(static_cast<size_t>(nb), 0ull);
    for (int64_t t : g) lay->tok_gbits[static_cast<size_t>(t / 64)] |= 1ull << (t % 64);
    // the blocks holding a global token play the part of global blocks at block level
    std::vector<int32_t> gblocks;
    std::vector<uint8_t> is_gb(static_cast<size_t>(nb), 0);
    for (int j = 0; j < nb; ++j)
      if (lay->tok_gbits[static_cast<size_t>(j)] != 0) {
        gblocks.push_back(j);
        is_gb[static_cast<size_t>(j)] = 1;
      }
    lay->globals = gblocks;
    lay->n_global = static_cast<int>(gblocks.size());
    // the band's blocks: |I - J| <= floor((w + 63) / 64)
    const int64_t wb64 = (static_cast<int64_t>(window) + 63) / 64;
    const int wb = static_cast<int>(std::min<int64_t>(wb64, nb));
    lay->window = wb;
    lay->token = true;
    lay->tok_window = window;
    std::vector<int32_t> urp, uci, row;
    urp.reserve(static_cast<size_t>(H) * nb + 1);
    urp.push_back(0);
    lay->tok_masked.clear();
    for (int h = 0; h < H; ++h) {
      for (int I = 0; I < nb; ++I) {
        build_row(h, I, nb, wb, gblocks, is_gb, n_random, seed, &row);
        for (int32_t J : row) {
          // every pair of the two blocks is allowed: a random block (drawn only for a
          // block without a global token, outside the band's and the global blocks),
          // the band covering the whole pair, or a block of global tokens only
          const int64_t dist = std::abs(static_cast<int64_t>(I) - J);
          const bool random = !is_gb[static_cast<size_t>(I)] && dist > wb && !is_gb[static_cast<size_t>(J)];
          const bool full = random || 64 * dist + 63 <= static_cast<int64_t>(window) ||
                            lay->tok_gbits[static_cast<size_t>(I)] == ~0ull ||
                            lay->tok_gbits[static_cast<size_t>(J)] == ~0ull;
          lay->tok_masked.push_back(full ? 0 : 1);
        }
        uci.insert(uci.end(), row.begin(), row.end());
        if (uci.size() > static_cast<size_t>(INT32_MAX)) {
          delete lay;
          return BSA_ERR_INVALID_ARG;
        }
        urp.push_back(static_cast<int32_t>(uci.size()));
      }
    }
    if (!set_rows(lay, std::move(urp), std::move(uci), is_gb)) {
      delete lay;
      return BSA_ERR_INVALID_ARG;
    }
  } catch (const std::bad_alloc&) {
    delete lay;
    return BSA_ERR_OOM;
  } catch (...) {
    delete lay;
    return BSA_ERR_INVALID_ARG;
  }
  *out = lay;
  return BSA_OK;
}

int bsa_layout_token_masks(const bsa_layout* lay, int* window, const uint64_t** global_bits) {
  if (lay == nullptr) return BSA_ERR_INVALID_ARG;
  if (!lay->token) return BSA_ERR_UNSUPPORTED;
  if (window != nullptr) *window = static_cast<int>(lay->tok_window);
  if (global_bits != nullptr) *global_bits = lay->tok_gbits.data();
  return BSA_OK;
}

int bsa_layout_from_csr(int H, int L, int block, const int32_t* row_ptr, const int32_t* col_idx,
                        bsa_layout** out) {
  if (out == nullptr) return BSA_ERR_INVALID_ARG;
  *out = nullptr;
  if (block < bsa::kBlock || block % bsa::kBlock != 0) return BSA_ERR_UNSUPPORTED;
  if (H < 1 || L < 1 || L % block != 0 || row_ptr == nullptr) return BSA_ERR_INVALID_ARG;
  const int nb = L / block;  // the caller's blocks
  if (L / bsa::kBlock > static_cast<int>(bsa::kEntColMask) || static_cast<int64_t>(H) * (L / bsa::kBlock) > (1 << 30))
    return BSA_ERR_INVALID_ARG;
  const size_t n_rows = static_cast<size_t>(H) * nb;
  // row_ptr: starts at 0, never decreases; col_idx may be NULL only if it is empty
  if (row_ptr[0] != 0) return BSA_ERR_INVALID_ARG;
  for (size_t x = 0; x < n_rows; ++x)
    if (row_ptr[x + 1] < row_ptr[x]) return BSA_ERR_INVALID_ARG;
  const int64_t nnz_in = row_ptr[n_rows];
  if (nnz_in > 0 && col_idx == nullptr) return BSA_ERR_INVALID_ARG;
  for (int64_t x = 0; x < nnz_in; ++x)
    if (col_idx[x] < 0 || col_idx[x] >= nb) return BSA_ERR_INVALID_ARG;
  bsa_layout* lay = new (std::nothrow) bsa_layout();
  if (lay == nullptr) return BSA_ERR_OOM;
  try {
    lay->H = H;
    lay->L = L;
    lay->block = block;
    lay->nb = L / bsa::kBlock;
    lay->window = -1;  // not a generated layout
    lay->n_random = -1;
    // rows sorted ascending and deduplicated
    std::vector<int32_t> urp, uci, row;
    urp.reserve(n_rows + 1);
    urp.push_back(0);
    uci.reserve(static_cast<size_t>(nnz_in));
    // dense[i]: block i lists every block in every head
    std::vector<uint8_t> dense(static_cast<size_t>(nb), 1);
    for (size_t x = 0; x < n_rows; ++x) {
      row.assign(col_idx + row_ptr[x], col_idx + row_ptr[x + 1]);
      std::sort(row.begin(), row.end());
      row.erase(std::unique(row.begin(), row.end()), row.end());
      if (static_cast<int>(row.size()) != nb) dense[x % static_cast<size_t>(nb)] = 0;
      uci.insert(uci.end(), row.begin(), row.end());
      urp.push_back(static_cast<int32_t>(uci.size()));
    }
    // The dense query blocks play the part of BigBird's global blocks in the
    // pairing: they pair with each other, so that no sparse row is paired with a
    // full one.
    for (int i = 0; i < nb; ++i)
      if (dense[static_cast<size_t>(i)]) lay->globals.push_back(i);
    lay->n_global = static_cast<int>(lay->globals.size());
    if (!set_rows(lay, std::move(urp), std::move(uci), dense)) {
      delete lay;
      return BSA_ERR_INVALID_ARG;
    }
  } catch (const std::bad_alloc&) {
    delete lay;
    return BSA_ERR_OOM;
  } catch (...) {
    delete lay;
    return BSA_ERR_INVALID_ARG;
  }
  *out = lay;
  return BSA_OK;
}

int bsa_layout_csr(const bsa_layout* lay, const int32_t** row_ptr, const int32_t** col_idx,
                   int64_t* nnz, int* nb, int* H) {
  if (lay == nullptr) return BSA_ERR_INVALID_ARG;
  const bool user = lay->block != bsa::kBlock;  // the caller's block units
  const std::vector<int32_t>& rp = user ? lay->user_row_ptr : lay->row_ptr;
  const std::vector<int32_t>& ci = user ? lay->user_col_idx : lay->col_idx;
  if (row_ptr) *row_ptr = rp.data();
  if (col_idx) *col_idx = ci.data();
  if (nnz) *nnz = static_cast<int64_t>(ci.size());
  if (nb) *nb = lay->L / lay->block;
  if (H) *H = lay->H;
  return BSA_OK;
}

int bsa_layout_globals(const bsa_layout* lay, const int32_t** globals, int* n_global) {
  if (lay == nullptr) return BSA_ERR_INVALID_ARG;
  if (globals) *globals = lay->globals.data();
  if (n_global) *n_global = static_cast<int>(lay->globals.size());
  return BSA_OK;
}

int bsa_layout_tiles(const bsa_layout* lay, const int32_t** pair_q, int* n_pairs,
                     const int32_t** pair_ptr, const uint32_t** pair_ent, int64_t* n_ent) {
  if (lay == nullptr) return BSA_ERR_INVALID_ARG;
  if (pair_q) *pair_q = lay->pair_q.data();
  if (n_pairs) *n_pairs = lay->n_pairs;
  if (pair_ptr) *pair_ptr = lay->pair_ptr.data();
  if (pair_ent) *pair_ent = lay->pair_ent.data();
  if (n_ent) *n_ent = static_cast<int64_t>(lay->pair_ent.size());
  return BSA_OK;
}

int bsa_layout_key_tiles(const bsa_layout* lay, const int32_t** pair_k, int* n_pairs,
                         const int32_t** pair_ptr, const uint32_t** pair_ent, int64_t* n_ent) {
  if (lay == nullptr) return BSA_ERR_INVALID_ARG;
  if (pair_k) *pair_k = lay->ktiles.pair_q.data();
  if (n_pairs) *n_pairs = lay->ktiles.n_pairs;
  if (pair_ptr) *pair_ptr = lay->ktiles.pair_ptr.data();
  if (pair_ent) *pair_ent = lay->ktiles.pair_ent.data();
  if (n_ent) *n_ent = static_cast<int64_t>(lay->ktiles.pair_ent.size());
  return BSA_OK;
}

int bsa_backward_workspace_bytes(const bsa_layout* lay, int B, size_t* bytes) {
  if (lay == nullptr || bytes == nullptr || B < 1) return BSA_ERR_INVALID_ARG;
  *bytes = bsa::plan_bwd_workspace(*lay, B).total;
  return BSA_OK;
}

void bsa_layout_free(bsa_layout* lay) {
  if (lay == nullptr) return;
  bsa::free_device(lay);
  delete lay;
}

int bsa_workspace_bytes(const bsa_layout* lay, int B, size_t* bytes) {
  return bsa_forward_workspace_bytes(lay, B, bsa::kHeadDim, bytes);
}

int bsa_forward_workspace_bytes(const bsa_layout* lay, int B, int d, size_t* bytes) {
  if (lay == nullptr || bytes == nullptr || B < 1) return BSA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return BSA_ERR_UNSUPPORTED;
  *bytes = bsa::plan_workspace(*lay, B, d).total;
  return BSA_OK;
}

const char* bsa_strerror(int status) {
  switch (status) {
    case BSA_OK: return "success";
    case BSA_ERR_INVALID_ARG: return "invalid argument";
    case BSA_ERR_UNSUPPORTED: return "unsupported configuration (block must be a multiple of 64, head dim 64, device sm_100)";
    case BSA_ERR_CUDA: return "CUDA call failed";
    case BSA_ERR_LAYOUT_MISMATCH: return "layout does not match H/L or is not uploaded to the current device";
    case BSA_ERR_DEVICE_TIMEOUT: return "a bounded wait inside a kernel timed out";
    case BSA_ERR_OOM: return "out of memory";
    case BSA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case BSA_ERR_STATIC_WORKSPACE: return "problem needs more scratch than the built-in static workspace holds";
    default: return "unknown status";
  }
}

}  // extern "C"
