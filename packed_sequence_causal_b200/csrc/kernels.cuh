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
  int64_t n;              // packed tokens
  float scale_log2;       // softmax_scale * log2(e)
  __nv_bfloat16* o;       // [N][hq][D]
  float* lse;             // [hq][N]
  float* o_part;          // [slots][hq][128][D]
  float* lse_part;        // [slots][hq][128]
  int* err;               // device error word
};

struct BwdParams {
  const int32_t* kv_units;    // [n_kv_units][3] (kv_tile, first_entry, n_entries), band-major
  const int32_t* entries;     // [n_items][2] (q_tile, tag)
  const int32_t* tok_hi;      // [N] last token of each token's document
  int32_t n_kv_units;
  int32_t hq, hkv, group;
  int64_t n, n_pad;           // tokens, tokens rounded up to 128
  float scale_log2;           // softmax_scale * log2(e)
  float scale;                // softmax_scale
  const float* lse2;          // [hq][n_pad] LSE * log2(e) (+inf past N)
  const float* dvec;          // [hq][n_pad] D_i = <dO_i, O_i> (0 past N)
  float* dq_acc;              // [n_pad][hq][D] fp32 dQ accumulator (reduced into through the tdq map)
  int* err;
};

template <int D>
cudaError_t launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p,
                       int grid, cudaStream_t stream);

template <int D>
cudaError_t launch_bwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tdo,
                       const CUtensorMap& tdq, const CUtensorMap& tdkv, const BwdParams& p, int grid,
                       cudaStream_t stream);

template <int D>
cudaError_t launch_merge(const int32_t* merges, int64_t n_merges, int32_t hq, int64_t n, const float* o_part,
                         const float* lse_part, __nv_bfloat16* o, float* lse, cudaStream_t stream);

template <int D>
cudaError_t launch_bwd_pre(const __nv_bfloat16* o, const __nv_bfloat16* dout, const float* lse, int64_t n,
                           int64_t n_pad, int32_t hq, int32_t hkv, float* dvec, float* lse2, float* dq_acc,
                           float* dkv_acc, cudaStream_t stream);

// fp32 accumulators -> bf16: dq (count_q values), dk and dv (count_kv values each; the dV
// accumulator starts dv_offset values after the dK one).
cudaError_t launch_bwd_post(const float* dq_acc, __nv_bfloat16* dq, int64_t count_q, const float* dkv_acc,
                            __nv_bfloat16* dk, __nv_bfloat16* dv, int64_t count_kv, int64_t dv_offset,
                            cudaStream_t stream);

}  // namespace sap
