// Internal plan layout shared by the host planner (plan.cpp) and the device
// entry points (api.cu).  Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <vector>

#include "sap.h"

// Backward units: a kv tile's list of at most kBwdBandTiles q tiles is one unit; a longer list
// is cut into the pieces that fall in one band of kBwdBandTiles q tiles each.
constexpr int32_t kBwdBandTiles = 16;

struct sap_plan_s {
  // inputs
  int64_t n = 0;
  int32_t num_docs = 0;
  int32_t num_chunks = 1;
  int32_t block_m = 128, block_n = 128;
  std::vector<int64_t> bounds;  // chunk c is tokens [bounds[c], bounds[c+1]); bounds[0] = 0, bounds[P] = n
  std::vector<int32_t> cu;

  // Window of the buffers the device calls take.  A full plan covers every token (q rows
  // [0, n), kv rows [0, n)).  A rank plan (sap_plan_rank) holds the items of one q chunk:
  // its query-side buffers (Q, O, dO, dQ, LSE) are rows [q_begin, q_end) and its key/value-side
  // buffers (K, V, dK, dV) rows [kv_begin, q_end); kv_begin is span_begin rounded down to a
  // kv tile, span_begin the first token of the document that holds token q_begin.
  int32_t rank_chunk = -1;  // -1: full plan
  int64_t q_begin = 0, q_end = 0, kv_begin = 0, span_begin = 0;

  // canonical items
  std::vector<sap_item_t> items;

  // forward schedule
  std::vector<int32_t> fwd_units;   // [U][4] (q_tile, item_begin, item_count, slot)
  std::vector<int32_t> fwd_order;   // [U]
  std::vector<int32_t> merges;      // [M][3] (q_tile, first_slot, n_slots)
  int64_t n_slots = 0;
  bool fused_merge = false;  // forward units span all kv chunks of a q-tile (no partials)
  // Rank plans list first (in fwd_order) the units whose kv tiles all lie in the device's own
  // chunk: they read no received keys.  n_local_units of them; full plans count every unit.
  int64_t n_local_units = 0;

  // backward schedule
  std::vector<int32_t> kv_units;    // [V][3] (kv_tile, first_entry, n_entries): band-major, heavy-first in a band
  std::vector<int32_t> kv_entries;  // [items][2] (q_tile, tag)
  // Per kv tile of the window (local index = (kv_tile * block_n - kv_begin) / block_n): 1 when the
  // tile has a single backward unit in a full plan, which then stores the tile's dK/dV as bf16
  // directly (in a rank plan, dK/dV rows may still receive other devices' partials, so every tile
  // goes through the fp32 accumulators).  kv_acc_tiles lists the local indices of the other tiles.
  std::vector<int32_t> kv_direct, kv_acc_tiles;

  // per-token document bounds (global token index): first token of the document, last token of the document
  std::vector<int32_t> tok_lo, tok_hi;

  // stats
  int64_t unmasked_pairs = 0;  // over the plan's query rows
  int32_t n_chunk_pairs = 0;

  // device copy (one allocation; offsets in int32 elements)
  void* dev = nullptr;
  int dev_id = -1;
  size_t off_items = 0, off_units = 0, off_order = 0, off_merges = 0, off_kv_units = 0, off_kv_entries = 0,
         off_kv_direct = 0, off_kv_acc_tiles = 0, off_tok_lo = 0, off_tok_hi = 0, dev_words = 0;

  int64_t q_rows() const { return q_end - q_begin; }
  int64_t kv_rows() const { return q_end - kv_begin; }
};

void sap_plan_build_fwd_schedule(sap_plan_s* p, bool fused);

// Equal chunks (num_chunks) or explicit bounds (bounds != nullptr, num_chunks + 1 entries).
int sap_plan_build(const int32_t* cu, int32_t num_docs, int64_t n, int32_t num_chunks, const int64_t* bounds,
                   int32_t block_m, int32_t block_n, sap_plan_s* p);

// The rank plan of q chunk `chunk` of a full plan.
int sap_plan_build_rank(const sap_plan_s* full, int32_t chunk, sap_plan_s* r);

// Balanced contiguous cut of the q tiles into num_chunks chunks (bounds: num_chunks + 1 entries).
int sap_balanced_bounds(const int32_t* cu, int32_t num_docs, int64_t n, int32_t num_chunks, int32_t block,
                        int64_t* bounds);
