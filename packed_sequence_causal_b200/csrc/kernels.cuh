// Kernel parameter blocks and launchers (internal to the library).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace sap {

struct FwdParams {
  const int32_t* items;   // [n_items][5] (q_tile, kv_tile, q_chunk, kv_chunk, tag)
  const int32_t* units;   // [n_units][4] (q_tile, item_begin, item_count, slot)
  const int32_t* order;   // [n_units] heavy-first permutation of the units
  const int32_t* tok_lo;  // [N] first token of each token's document
  int32_t n_units;
  int32_t hq, group;      // query heads, hq / hkv
  // Buffer windows (global token indices): Q, O and LSE hold rows [q0, q_end), K and V rows
  // [kv0, q_end); tiles, items and the per-token arrays stay in global coordinates.
  int64_t q0, kv0, q_end;
  int64_t lse_ld;         // row stride of LSE (q_end - q0)
  float scale_log2;       // softmax_scale * log2(e)
  __nv_bfloat16* o;       // [q rows][hq][D]
  float* lse;             // [hq][lse_ld]
  float* o_part;          // [slots][hq][128][D]
  float* lse_part;        // [slots][hq][128]
  int* err;               // device error word
  uint64_t wait_ns;       // pipeline wait limit of this launch
  int32_t skip_v_load;    // test hook: CTA 0 leaves its first V load out, so a wait runs out
  int* work_next;         // two-tile kernel, one-CTA form: work items handed out beyond the first
                          // gridDim.x (zero at launch); nullptr: static round-robin order
};

struct BwdParams {
  const int32_t* kv_units;    // [n_kv_units][3] (kv_tile, first_entry, n_entries), band-major
  const int32_t* entries;     // [n_items][2] (q_tile, tag)
  const int32_t* tok_hi;      // [N] last token of each token's document
  int32_t n_kv_units;
  int32_t hq, hkv, group;
  // Buffer windows as in FwdParams: query-side rows [q0, q_end), key/value-side rows [kv0, q_end).
  int64_t q0, kv0, q_end;
  int64_t n_pad, n_pad_kv;    // query / key-value window rows rounded up to 128
  float scale_log2;           // softmax_scale * log2(e)
  float scale;                // softmax_scale
  const float* lse2;          // [hq][n_pad] LSE * log2(e) (+inf past the window)
  const float* dvec;          // [hq][n_pad] D_i = <dO_i, O_i> (0 past the window)
  float* dq_acc;              // [n_pad][hq][D] fp32 dQ accumulator (reduced into through the tdq map)
  const int32_t* kv_direct;   // per 128-row kv tile of the window: 1 = store dK/dV as bf16 directly
  int* work_next;             // work items handed out beyond the first gridDim.x (zero at launch)
  int* err;
  uint64_t wait_ns;           // pipeline wait limit of this launch
};

// two_cta (D = 128, hq / hkv a multiple of 4): the two-CTA cluster variant; tk must then be a map
// with 64-row boxes (each CTA of a pair loads half of every K tile).  grid: CTAs (SMs) to use.
template <int D>
cudaError_t launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p,
                       int grid, cudaStream_t stream, bool two_cta = false);

// tdkv: the fp32 dK/dV accumulators; tdk, tdv: the bf16 dK, dV outputs (tiles with kv_direct set).
template <int D>
cudaError_t launch_bwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tdo,
                       const CUtensorMap& tdq, const CUtensorMap& tdkv, const CUtensorMap& tdk,
                       const CUtensorMap& tdv, const BwdParams& p, int grid, cudaStream_t stream);

// Merge into O rows [q0, q_end) (O and LSE hold the window's rows; LSE row stride q_end - q0).
template <int D>
cudaError_t launch_merge(const int32_t* merges, int64_t n_merges, int32_t hq, int64_t q0, int64_t q_end,
                         const float* o_part, const float* lse_part, __nv_bfloat16* o, float* lse,
                         cudaStream_t stream);

// n rows of O, dO and LSE (padded to n_pad); n_pad_kv rows of each dK/dV accumulator, except the
// 128-row tiles t with kv_direct[t] != 0 (their dK/dV are stored directly by the backward kernel);
// work_next (the backward's work counter) set to zero.
template <int D>
cudaError_t launch_bwd_pre(const __nv_bfloat16* o, const __nv_bfloat16* dout, const float* lse, int64_t n,
                           int64_t n_pad, int64_t n_pad_kv, int32_t hq, int32_t hkv, float* dvec, float* lse2,
                           float* dq_acc, float* dkv_acc, const int32_t* kv_direct, int* work_next,
                           cudaStream_t stream);

// dkv_acc rows [row0, row0 + rows) += the fp32 partials dk_part, dv_part ([rows][hkv][D] each), then
// those rows of dk and dv (same row numbering as the accumulator) are rewritten as bf16.
cudaError_t launch_kv_add(float* dkv_acc, int64_t dv_offset, const float* dk_part, const float* dv_part,
                          int64_t row0, int64_t rows, int64_t row_elems, __nv_bfloat16* dk, __nv_bfloat16* dv,
                          cudaStream_t stream);

// fp32 accumulators -> bf16: dq (count_q values); dk and dv (count_kv values each; the dV
// accumulator starts dv_offset values after the dK one) on the n_acc_tiles 128-row tiles listed in
// acc_tiles (row_elems values per row).
cudaError_t launch_bwd_post(const float* dq_acc, __nv_bfloat16* dq, int64_t count_q, const float* dkv_acc,
                            __nv_bfloat16* dk, __nv_bfloat16* dv, int64_t count_kv, int64_t dv_offset,
                            const int32_t* acc_tiles, int64_t n_acc_tiles, int64_t row_elems, cudaStream_t stream);

}  // namespace sap
