// Host planner: cu_seqlens + chunk partition -> non-empty tile items and the
// forward / backward work schedules.
//
// This is the single-GPU counterpart of the schedule that the HSAP paper
// generates ahead of time for the irregular attention of packed sequences
// (HSAP / Sequence-Aware Parallelism page, abstract and method details: the
// JIT-generated instruction sequences, and the load-balancing scheduler).
// Here the schedule is a compact list of tiles that the kernels walk, with
// cross-document tiles skipped entirely.
//
// Cost is O(items + N): for a q-tile whose first row starts document-wise at
// token s, the kv tiles that hold an unmasked pair are exactly
// floor(s / BN) .. floor((last row) / BN), because the key ranges of the rows
// of one q-tile are contiguous and together cover [s, last row].  Tags need
// O(1) work per item because the first key of a row is non-decreasing in the
// row.
//
// Chunks are contiguous token ranges: P equal ones, or explicit tile-aligned
// bounds (for example the balanced cut below).  A rank plan keeps the items of
// one q chunk -- the work of one device under sequence parallelism -- and the
// window of tokens that device holds: its own chunk for the queries, and for
// keys and values the span from the start of the document that reaches into
// the chunk (the only earlier tokens any of its queries may see).
#include <algorithm>
#include <numeric>

#include "plan.hpp"

// Forward schedule.  Default: one unit per (q-tile, kv-chunk) run of items, a
// partial slot for each unit of a q-tile that sees several kv chunks, and a
// merge entry per such q-tile.  Fused: one unit per q-tile over all its items
// (every kv chunk), written directly, so there are no partials and no merges.
void sap_plan_build_fwd_schedule(sap_plan_s* p, bool fused) {
  p->fused_merge = fused;
  p->fwd_units.clear();
  p->merges.clear();
  p->n_slots = 0;
  {
    size_t a = 0;
    const size_t ni = p->items.size();
    while (a < ni) {
      size_t e = a;
      while (e < ni && p->items[e].q_tile == p->items[a].q_tile) ++e;  // items of this q-tile: [a, e)
      std::vector<std::pair<size_t, size_t>> runs;
      size_t r = a;
      while (r < e) {
        size_t s = r;
        while (s < e && (fused || p->items[s].kv_chunk == p->items[r].kv_chunk)) ++s;
        runs.push_back({r, s - r});
        r = s;
      }
      const bool partial = runs.size() > 1;
      if (partial)
        p->merges.insert(p->merges.end(),
                         {p->items[a].q_tile, (int32_t)p->n_slots, (int32_t)runs.size()});
      for (auto& run : runs) {
        int32_t slot = partial ? (int32_t)(p->n_slots++) : -1;
        p->fwd_units.insert(p->fwd_units.end(),
                            {p->items[a].q_tile, (int32_t)run.first, (int32_t)run.second, slot});
      }
      a = e;
    }
  }
  const size_t nu = p->fwd_units.size() / 4;
  p->fwd_order.resize(nu);
  std::iota(p->fwd_order.begin(), p->fwd_order.end(), 0);
  // heavy-first; among units of equal size, kv chunk first, so that the CTAs running at the same
  // time stream the K/V tiles of one kv chunk (which then stay in L2) rather than of several
  auto chunk_of = [&](int32_t u) { return p->items[p->fwd_units[4 * u + 1]].kv_chunk; };
  std::stable_sort(p->fwd_order.begin(), p->fwd_order.end(), [&](int32_t x, int32_t y) {
    const int32_t cx = p->fwd_units[4 * x + 2], cy = p->fwd_units[4 * y + 2];
    return cx != cy ? cx > cy : chunk_of(x) < chunk_of(y);
  });
  // A rank plan runs its own-chunk units first (each part keeps the heavy-first order), so that
  // they can run while the keys of earlier chunks are still arriving.
  p->n_local_units = (int64_t)nu;
  if (p->rank_chunk >= 0) {
    auto local = [&](int32_t u) {
      const int32_t b = p->fwd_units[4 * u + 1], c = p->fwd_units[4 * u + 2];
      for (int32_t e = b; e < b + c; ++e)
        if (p->items[e].kv_chunk != p->rank_chunk) return false;
      return true;
    };
    auto mid = std::stable_partition(p->fwd_order.begin(), p->fwd_order.end(), local);
    p->n_local_units = mid - p->fwd_order.begin();
  }
}

namespace {

int check_cu(const int32_t* cu, int32_t num_docs, int64_t n) {
  if (!cu || num_docs < 0 || n < 0) return SAP_ERR_INVALID_ARG;
  if (n > INT32_MAX - 256) return SAP_ERR_INVALID_ARG;
  if (cu[0] != 0) return SAP_ERR_BAD_SEQLENS;
  for (int32_t k = 0; k < num_docs; ++k)
    if (cu[k + 1] < cu[k]) return SAP_ERR_BAD_SEQLENS;
  if ((int64_t)cu[num_docs] != n) return SAP_ERR_BAD_SEQLENS;
  return SAP_OK;
}

// Backward: items grouped by kv tile, q-tile descending within a kv tile.  A kv tile whose list
// has at most kBwdBandTiles q tiles is one unit; a longer list is cut into bands of kBwdBandTiles
// q tiles, one unit per (kv tile, band) piece.  Units are ordered band-major from the top band
// down (a unit's band is that of its top q tile), heavy-first within a band.  The persistent CTAs
// take units in this order, so at any time they all work on Q, dO and dQ rows of about one band
// (a few tens of MB at 32 heads) and those rows stay in L2; the price is one fp32 dK/dV reduction
// per unit of a cut list instead of one bf16 store per kv tile.  A kv tile with a single unit
// stores its dK/dV directly (full plans; see kv_direct).
void build_bwd_schedule(sap_plan_s* p) {
  const int64_t ntk = (p->n + p->block_n - 1) / p->block_n;
  std::vector<int64_t> cnt((size_t)ntk + 1, 0);
  for (const auto& it : p->items) cnt[(size_t)it.kv_tile + 1]++;
  for (int64_t t = 0; t < ntk; ++t) cnt[t + 1] += cnt[t];
  p->kv_entries.assign(p->items.size() * 2, 0);
  {
    std::vector<int64_t> pos(cnt.begin() + 1, cnt.end());  // fill each group from its end
    for (const auto& it : p->items) {
      int64_t w = --pos[it.kv_tile];
      p->kv_entries[2 * w] = it.q_tile;
      p->kv_entries[2 * w + 1] = it.tag;
    }
  }
  struct Unit {
    int32_t band, kv_tile, first, count;
  };
  std::vector<Unit> units;
  std::vector<int32_t> units_of_tile((size_t)ntk, 0);
  for (int64_t t = 0; t < ntk; ++t) {
    int64_t e = cnt[t];
    const bool whole = cnt[t + 1] - cnt[t] <= kBwdBandTiles;
    while (e < cnt[t + 1]) {
      const int32_t band = p->kv_entries[2 * e] / kBwdBandTiles;
      int64_t f = whole ? cnt[t + 1] : e + 1;
      while (f < cnt[t + 1] && p->kv_entries[2 * f] / kBwdBandTiles == band) ++f;
      units.push_back(Unit{band, (int32_t)t, (int32_t)e, (int32_t)(f - e)});
      units_of_tile[t]++;
      e = f;
    }
  }
  // direct bf16 stores: full plans, kv tiles of a single unit (tile index local to the window)
  const int64_t kt0 = p->kv_begin / p->block_n;
  const int64_t ntl = (p->kv_rows() + p->block_n - 1) / p->block_n;
  p->kv_direct.assign((size_t)ntl, 0);
  p->kv_acc_tiles.clear();
  for (int64_t l = 0; l < ntl; ++l) {
    const int64_t t = kt0 + l;
    if (p->rank_chunk < 0 && t < ntk && units_of_tile[t] == 1) p->kv_direct[l] = 1;
    else p->kv_acc_tiles.push_back((int32_t)l);
  }
  std::stable_sort(units.begin(), units.end(), [](const Unit& a, const Unit& b) {
    return a.band != b.band ? a.band > b.band : a.count > b.count;
  });
  p->kv_units.clear();
  p->kv_units.reserve(units.size() * 3);
  for (const Unit& u : units) p->kv_units.insert(p->kv_units.end(), {u.kv_tile, u.first, u.count});
}

void count_chunk_pairs(sap_plan_s* p) {
  std::vector<char> seen((size_t)p->num_chunks * p->num_chunks, 0);
  p->n_chunk_pairs = 0;
  for (const auto& it : p->items) {
    char& s = seen[(size_t)it.q_chunk * p->num_chunks + it.kv_chunk];
    if (!s) s = 1, ++p->n_chunk_pairs;
  }
}

// Number of kv tiles a q tile touches: floor(first key / bn) .. floor(last row / bn).
int64_t tile_cost(const std::vector<int32_t>& tok_lo, int64_t n, int64_t qt, int32_t bm, int32_t bn) {
  const int64_t i0 = qt * bm, ilast = std::min<int64_t>(i0 + bm, n) - 1;
  return ilast / bn - tok_lo[i0] / bn + 1;
}

}  // namespace

int sap_plan_build(const int32_t* cu, int32_t num_docs, int64_t n, int32_t num_chunks, const int64_t* bounds,
                   int32_t block_m, int32_t block_n, sap_plan_s* p) {
  if (!p || block_m <= 0 || block_n <= 0) return SAP_ERR_INVALID_ARG;
  int rc = check_cu(cu, num_docs, n);
  if (rc) return rc;
  if (num_chunks < 1) return SAP_ERR_BAD_CHUNKS;
  std::vector<int64_t> b((size_t)num_chunks + 1);
  if (bounds) {
    // explicit contiguous chunks: non-empty, interior bounds on tile boundaries of both tile sizes
    if (bounds[0] != 0 || bounds[num_chunks] != n) return SAP_ERR_BAD_CHUNKS;
    for (int32_t c = 0; c < num_chunks; ++c) {
      if (bounds[c + 1] <= bounds[c] && !(num_chunks == 1 && n == 0)) return SAP_ERR_BAD_CHUNKS;
      if (c > 0 && (bounds[c] % block_m || bounds[c] % block_n)) return SAP_ERR_BAD_CHUNKS;
    }
    b.assign(bounds, bounds + num_chunks + 1);
  } else if (num_chunks == 1) {
    b = {0, n};
  } else {
    if (n % num_chunks) return SAP_ERR_BAD_CHUNKS;
    const int64_t chunk = n / num_chunks;
    if (chunk % block_m || chunk % block_n) return SAP_ERR_BAD_CHUNKS;
    for (int32_t c = 0; c <= num_chunks; ++c) b[c] = c * chunk;
  }
  p->n = n;
  p->num_docs = num_docs;
  p->num_chunks = num_chunks;
  p->block_m = block_m;
  p->block_n = block_n;
  p->bounds = b;
  p->cu.assign(cu, cu + num_docs + 1);
  p->rank_chunk = -1;
  p->q_begin = 0, p->q_end = n, p->kv_begin = 0, p->span_begin = 0;

  // per-token document bounds
  p->tok_lo.assign((size_t)n, 0);
  p->tok_hi.assign((size_t)n, 0);
  p->unmasked_pairs = 0;
  std::vector<int32_t> doc_of((size_t)n);
  for (int32_t k = 0; k < num_docs; ++k) {
    int64_t L = (int64_t)cu[k + 1] - cu[k];
    p->unmasked_pairs += L * (L + 1) / 2;
    for (int64_t i = cu[k]; i < cu[k + 1]; ++i) {
      p->tok_lo[i] = cu[k];
      p->tok_hi[i] = cu[k + 1] - 1;
      doc_of[i] = k;
    }
  }
  auto chunk_of = [&](int64_t tok) {
    return (int32_t)(std::upper_bound(p->bounds.begin(), p->bounds.end(), tok) - p->bounds.begin() - 1);
  };

  // items, canonical order
  p->items.clear();
  const int64_t ntq = (n + block_m - 1) / block_m;
  const int64_t ntk = (n + block_n - 1) / block_n;
  std::vector<int32_t> kv_chunk((size_t)ntk);  // chunk of each kv tile's first key (bounds ascend)
  for (int64_t kt = 0; kt < ntk; ++kt) kv_chunk[(size_t)kt] = chunk_of(kt * block_n);
  int64_t n_items = 0;
  for (int64_t qt = 0; qt < ntq; ++qt)
    n_items += (std::min<int64_t>(qt * block_m + block_m, n) - 1) / block_n - p->tok_lo[qt * block_m] / block_n + 1;
  p->items.reserve((size_t)n_items);
  for (int64_t qt = 0; qt < ntq; ++qt) {
    const int64_t i0 = qt * block_m;
    const int64_t ilast = std::min<int64_t>(i0 + block_m, n) - 1;  // last real row
    const bool tile_complete = (i0 + block_m) <= n;
    const int64_t kt_first = p->tok_lo[i0] / block_n, kt_last = ilast / block_n;
    const int32_t qc = chunk_of(i0);
    for (int64_t kt = kt_first; kt <= kt_last; ++kt) {
      const int64_t j0 = kt * block_n, j1 = j0 + block_n - 1;
      int32_t tag;
      // every nominal row exists, the latest-starting row starts at or before j0,
      // and the earliest row ends at or after j1
      if (tile_complete && p->tok_lo[ilast] <= j0 && j1 <= i0)
        tag = SAP_TAG_FULL;
      else if (block_m == block_n && kt == qt && doc_of[i0] == doc_of[ilast])
        tag = SAP_TAG_CAUSAL;
      else
        tag = SAP_TAG_MASKED;
      p->items.push_back(sap_item_t{(int32_t)qt, (int32_t)kt, qc, kv_chunk[(size_t)kt], tag});
    }
  }
  count_chunk_pairs(p);
  sap_plan_build_fwd_schedule(p, false);
  build_bwd_schedule(p);
  return SAP_OK;
}

int sap_plan_build_rank(const sap_plan_s* f, int32_t chunk, sap_plan_s* r) {
  if (!f || !r || f->rank_chunk >= 0 || chunk < 0 || chunk >= f->num_chunks) return SAP_ERR_INVALID_ARG;
  r->n = f->n;
  r->num_docs = f->num_docs;
  r->num_chunks = f->num_chunks;
  r->block_m = f->block_m;
  r->block_n = f->block_n;
  r->bounds = f->bounds;
  r->cu = f->cu;
  r->tok_lo = f->tok_lo;
  r->tok_hi = f->tok_hi;
  r->rank_chunk = chunk;
  r->q_begin = f->bounds[chunk];
  r->q_end = f->bounds[chunk + 1];
  r->span_begin = r->q_begin < f->n ? f->tok_lo[r->q_begin] : r->q_begin;
  r->kv_begin = r->span_begin / f->block_n * f->block_n;
  r->items.clear();
  for (const auto& it : f->items)
    if (it.q_chunk == chunk) r->items.push_back(it);
  r->unmasked_pairs = 0;
  for (int64_t i = r->q_begin; i < r->q_end; ++i) r->unmasked_pairs += i - f->tok_lo[i] + 1;
  count_chunk_pairs(r);
  sap_plan_build_fwd_schedule(r, f->fused_merge);
  build_bwd_schedule(r);
  return SAP_OK;
}

// Balanced cut.  The cost of a q tile is the number of kv tiles it touches (one 128 x 128 tile of
// both passes' GEMMs each, masked or not).  M* = the smallest possible maximum over chunks of the
// summed cost, found by bisection with a greedy feasibility test (pack tiles left to right into
// chunks of cost <= M; feasible iff at most num_chunks chunks are needed).  Among the cuts that
// reach M*, the bounds are the lexicographically largest: each chunk takes as many tiles as fit
// while leaving at least one tile for every later chunk.
int sap_balanced_bounds(const int32_t* cu, int32_t num_docs, int64_t n, int32_t num_chunks, int32_t block,
                        int64_t* bounds) {
  if (!bounds || block <= 0) return SAP_ERR_INVALID_ARG;
  int rc = check_cu(cu, num_docs, n);
  if (rc) return rc;
  if (num_chunks < 1) return SAP_ERR_BAD_CHUNKS;
  const int64_t T = (n + block - 1) / block;
  if (n == 0) {
    if (num_chunks != 1) return SAP_ERR_BAD_CHUNKS;
    bounds[0] = bounds[1] = 0;
    return SAP_OK;
  }
  if (num_chunks > T) return SAP_ERR_BAD_CHUNKS;
  std::vector<int32_t> tok_lo((size_t)n, 0);
  for (int32_t k = 0; k < num_docs; ++k)
    for (int64_t i = cu[k]; i < cu[k + 1]; ++i) tok_lo[i] = cu[k];
  std::vector<int64_t> cost((size_t)T);
  int64_t total = 0, top = 0;
  for (int64_t t = 0; t < T; ++t) {
    cost[t] = tile_cost(tok_lo, n, t, block, block);
    total += cost[t];
    top = std::max(top, cost[t]);
  }
  auto chunks_needed = [&](int64_t cap) {
    int64_t used = 1, acc = 0;
    for (int64_t t = 0; t < T; ++t) {
      if (acc + cost[t] > cap) ++used, acc = 0;
      acc += cost[t];
    }
    return used;
  };
  int64_t lo = top, hi = total;  // chunks_needed(hi) == 1
  while (lo < hi) {
    const int64_t mid = lo + (hi - lo) / 2;
    if (chunks_needed(mid) <= num_chunks)
      hi = mid;
    else
      lo = mid + 1;
  }
  const int64_t cap = lo;
  int64_t pos = 0;
  bounds[0] = 0;
  for (int32_t k = 0; k + 1 < num_chunks; ++k) {
    const int64_t later = num_chunks - k - 1;  // chunks still to fill after this one
    int64_t e = pos, acc = 0;
    while (e < T - later && acc + cost[e] <= cap) acc += cost[e++];
    bounds[k + 1] = e * block;
    pos = e;
  }
  bounds[num_chunks] = n;
  return SAP_OK;
}
