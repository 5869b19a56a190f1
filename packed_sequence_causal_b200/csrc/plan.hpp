// Internal plan layout shared by the host planner (plan.cpp) and the device
// entry points (api.cu).  Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <vector>

#include "sap.h"

// Backward units cover at most this many q tiles of one kv tile's list (one "band").
constexpr int32_t kBwdBandTiles = 16;

struct sap_plan_s {
  // inputs
  int64_t n = 0;
  int32_t num_docs = 0;
  int32_t num_chunks = 1;
  int32_t block_m = 128, block_n = 128;
  int64_t chunk = 0;  // tokens per chunk (N when P = 1)
  std::vector<int32_t> cu;

  // canonical items
  std::vector<sap_item_t> items;

  // forward schedule
  std::vector<int32_t> fwd_units;   // [U][4] (q_tile, item_begin, item_count, slot)
  std::vector<int32_t> fwd_order;   // [U]
  std::vector<int32_t> merges;      // [M][3] (q_tile, first_slot, n_slots)
  int64_t n_slots = 0;
  bool fused_merge = false;  // forward units span all kv chunks of a q-tile (no partials)

  // backward schedule
  std::vector<int32_t> kv_units;    // [V][3] (kv_tile, first_entry, n_entries): band-major, heavy-first in a band
  std::vector<int32_t> kv_entries;  // [items][2] (q_tile, tag)

  // per-token document bounds: first token of the document, last token of the document
  std::vector<int32_t> tok_lo, tok_hi;

  // stats
  int64_t unmasked_pairs = 0;
  int32_t n_chunk_pairs = 0;

  // device copy (one allocation; offsets in int32 elements)
  void* dev = nullptr;
  int dev_id = -1;
  size_t off_items = 0, off_units = 0, off_order = 0, off_merges = 0, off_kv_units = 0, off_kv_entries = 0,
         off_tok_lo = 0, off_tok_hi = 0, dev_words = 0;
};

void sap_plan_build_fwd_schedule(sap_plan_s* p, bool fused);

int sap_plan_build(const int32_t* cu, int32_t num_docs, int64_t n, int32_t num_chunks, int32_t block_m,
                   int32_t block_n, sap_plan_s* p);
