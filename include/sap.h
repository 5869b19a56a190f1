/*
 * sap.h -- C ABI of the B200 (sm_100a) packed causal attention library.
 *
 * The operation (HSAP / Sequence-Aware Parallelism paper page, abstract):
 * causal attention over a *packed* sequence -- many documents laid end to end
 * -- in which a token attends only to earlier (and its own) tokens of its own
 * document, so that packing causes no cross-contamination.  The sequence is
 * cut into P equal chunks as sequence parallelism would cut it; every
 * (query-chunk, key/value-chunk) pair yields a partial output and its
 * log-sum-exp ("partial attention computation", same abstract), and the
 * partials are merged exactly, which by the equivalence stated in the
 * sequence-parallelism explainer page (FAQ on equivalence with one device)
 * gives the single-device result.  On one GPU the P chunks are simulated in
 * place.
 *
 * Conventions used by every call
 *   N      packed tokens;  cu_seqlens: int32[num_docs+1], cu[0] = 0,
 *          non-decreasing, cu[num_docs] = N; document k is [cu[k], cu[k+1]).
 *          Zero-length documents are allowed.
 *   Q, O, dO, dQ : bf16, [N][hq][head_dim], contiguous (row = token).
 *   K, V, dK, dV : bf16, [N][hkv][head_dim], contiguous.
 *   LSE          : fp32, [hq][N], natural-log log-sum-exp of the scaled scores.
 *   GQA          : query head h reads key/value head h / (hq / hkv).
 *   Scores       : S_ij = softmax_scale * <q_i, k_j>, kept for doc(j) == doc(i)
 *                  and j <= i (the diagonal is included).
 *   Kernels support head_dim in {64, 128} and 128 x 128 tiles.
 *
 * Ownership: the caller owns every device buffer (inputs, outputs and the
 * workspace).  The library owns only a plan: its host arrays and their device
 * copy, released by sap_plan_destroy.  One exception: the library keeps a
 * 16 MiB device array of its own on every device that loads it, the scratch
 * of sap_attn_fwd_static_scratch (see that declaration).  Device pointers,
 * workspaces included, must be 16-byte aligned.
 *
 * Streams: every device call is asynchronous on the given cudaStream_t
 * (passed as void*, NULL = the legacy default stream).
 *
 * Errors: every int-returning call returns SAP_OK (0) or a negative SAP_ERR_*
 * code; nothing is printed and no exception crosses the ABI.  A CUDA failure
 * returns SAP_ERR_CUDA and the CUDA status is kept for sap_last_cuda_error().
 * The kernels never trap: a pipeline wait that runs past its time limit sets a
 * device error word, read (with a device synchronisation) by
 * sap_device_status().
 */
#ifndef SAP_H_
#define SAP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  SAP_OK = 0,
  SAP_ERR_INVALID_ARG = -1,  /* null pointer, bad head counts, hq % hkv != 0, bad sizes        */
  SAP_ERR_BAD_SEQLENS = -2,  /* cu[0] != 0, decreasing, or cu[num_docs] != N                   */
  SAP_ERR_BAD_CHUNKS = -3,   /* P < 1, or P > 1 with N % P != 0 or (N/P) % block != 0          */
  SAP_ERR_WORKSPACE = -4,    /* workspace missing or smaller than sap_workspace_size           */
  SAP_ERR_CUDA = -5,         /* a CUDA runtime call failed (see sap_last_cuda_error)           */
  SAP_ERR_DEVICE = -6,       /* the device error word is set (a kernel wait timed out)         */
  SAP_ERR_UNSUPPORTED = -7,  /* head_dim not in {64,128}, or plan tiles other than 128 x 128   */
  SAP_ERR_NOMEM = -8         /* host allocation failed                                         */
};

enum { SAP_TAG_FULL = 0, SAP_TAG_CAUSAL = 1, SAP_TAG_MASKED = 2 };
enum { SAP_WS_FWD = 0, SAP_WS_BWD = 1 };

typedef struct sap_plan_s* sap_plan_t;

/* One non-empty (q-tile, kv-tile) pair of the packed causal mask.
 *   tag FULL   : no pair of the block_m x block_n box is masked (never a partial
 *                last tile: its missing rows count as masked);
 *   tag CAUSAL : a diagonal box (same token range) whose real rows all lie in one
 *                document, a partial last tile included; inside it the mask is
 *                exactly j <= i;
 *   tag MASKED : anything else (a document boundary inside the box, or an
 *                off-diagonal box of a partial last tile).
 * q_chunk = q_tile*block_m / C and kv_chunk = kv_tile*block_n / C, C = N / P. */
typedef struct {
  int32_t q_tile, kv_tile, q_chunk, kv_chunk, tag;
} sap_item_t;

/* Build a plan on the host (no device work) -- the ahead-of-time schedule of the irregular,
 * document-bounded attention of a packed batch (HSAP page, method details: the SAP schedule is
 * generated before the run for the hybrid-context attention pattern; abstract: no attention
 * across documents).  Validates cu_seqlens and the
 * chunking, lists the non-empty tiles in canonical order (q-tile ascending,
 * then kv-tile ascending; bit-exact with the tile-list definition above), and
 * derives the work schedule: forward units = (q-tile, kv-chunk) groups of
 * items, partial slots for q-tiles that see more than one kv-chunk and a
 * heavy-first launch order; backward units = per-kv-tile q lists cut into bands
 * of 16 q tiles, in band-major order (sap_plan_bwd_schedule).
 * P = num_chunks; with P = 1 any N >= 0 is accepted (a partial last tile is
 * masked).  On success *out owns the plan. */
int sap_plan(const int32_t* cu_seqlens_host, int32_t num_docs, int64_t total_tokens, int32_t num_chunks,
             int32_t block_m, int32_t block_n, sap_plan_t* out);

/* Plan over explicit contiguous chunks: chunk c is tokens [chunk_bounds[c], chunk_bounds[c+1]),
 * with chunk_bounds[0] = 0, chunk_bounds[num_chunks] = N, strictly increasing, and every
 * interior bound a multiple of block_m and block_n (otherwise SAP_ERR_BAD_CHUNKS).  Equal chunks
 * (sap_plan) are the special case chunk_bounds[c] = c N / P.  The items, tags and schedules are
 * those of sap_plan with q_chunk / kv_chunk the chunk that holds the tile's first token.
 * (HSAP page, method details: the sequence is cut into parts per device; the load-balancing
 * scheduler chooses the cut -- see sap_balanced_chunks.)  chunk_bounds is read, not kept. */
int sap_plan_chunks(const int32_t* cu_seqlens_host, int32_t num_docs, int64_t total_tokens,
                    const int64_t* chunk_bounds, int32_t num_chunks, int32_t block_m, int32_t block_n,
                    sap_plan_t* out);

/* Balanced chunk bounds (HSAP page, method details: the load-balancing scheduler; explainer page,
 * challenges: uneven document lengths leave devices idle).  The cost of a q tile of `block`
 * tokens is the number of kv tiles it touches (its items: one block x block tile of work per
 * head in each pass).  Writes num_chunks + 1 bounds into chunk_bounds (caller-owned): contiguous,
 * interior bounds multiples of block, every chunk non-empty, minimising the largest summed cost
 * of a chunk; among the cuts that reach that minimum, the lexicographically largest bounds (each
 * chunk takes as many tiles as fit, leaving at least one tile per later chunk).  Errors:
 * SAP_ERR_BAD_SEQLENS, SAP_ERR_BAD_CHUNKS (num_chunks < 1 or more chunks than tiles). */
int sap_balanced_chunks(const int32_t* cu_seqlens_host, int32_t num_docs, int64_t total_tokens, int32_t num_chunks,
                        int32_t block, int64_t* chunk_bounds);

/* The chunk bounds of a plan (num_chunks + 1 entries; host memory owned by the plan). */
int sap_plan_chunk_bounds(sap_plan_t plan, const int64_t** bounds, int32_t* num_chunks);

/* Per q chunk c (caller-owned arrays of num_chunks entries, either may be NULL): the plan's items
 * whose q tile lies in chunk c, and the unmasked (i, j) pairs of its query rows (per head).  The
 * work of device c under sequence parallelism; a rank plan reports its own chunk only. */
int sap_plan_chunk_stats(sap_plan_t plan, int64_t* items_per_chunk, int64_t* pairs_per_chunk);

/* Rank plan for sequence parallelism (HSAP page, abstract and method details: each device computes
 * the partial attention of its own part of the sequence, and only the key/value data of documents
 * that reach into that part crosses devices).  From a full plan, the plan of the device that owns
 * q chunk `chunk`: the items whose q tile lies in the chunk, with the same tags and global tile
 * indices, and their forward / backward schedules.  Its device calls take WINDOWED buffers:
 *   query side  Q, O, dO, dQ : rows [q_begin, q_end) = the chunk;  LSE [hq][q_end - q_begin];
 *   key side    K, V, dK, dV : rows [kv_begin, q_end),
 * where span_begin = first token of the document holding token q_begin (the earliest key any
 * query of the chunk may see) and kv_begin = span_begin rounded down to a kv tile
 * (sap_plan_window).  K/V rows [kv_begin, span_begin) are never attended to but are read as whole
 * tiles: they must hold finite values (zeros will do).  Rows [span_begin, q_begin) are the other
 * devices' keys and values (sap_plan_rank_spans lists who sends which).  dK/dV rows below q_begin
 * are this device's partial sums for other devices' tokens (see sap_attn_bwd_kv_add).  The rank
 * plan is independent of the full plan (destroy both). */
int sap_plan_rank(sap_plan_t plan, int32_t chunk, sap_plan_t* out);

/* Buffer window of a plan: [q_begin, q_end) query rows, [kv_begin, q_end) key/value rows, and
 * span_begin (see sap_plan_rank).  A full plan reports 0, N, 0, 0. */
int sap_plan_window(sap_plan_t plan, int64_t* q_begin, int64_t* q_end, int64_t* kv_begin, int64_t* span_begin);

/* Exchange list of the device owning q chunk `chunk` (full plans only): for every earlier chunk b
 * that holds keys of a document reaching into `chunk`, one entry (b, lo, hi) = the token range
 * [lo, hi) of chunk b that this device needs; *n_spans entries are written into spans (caller-owned,
 * 3 * num_chunks int64).  These are exactly the chunk pairs of the plan's chunk-pair table with
 * q_chunk = chunk and kv_chunk < chunk, cut to the document-spanning part -- the sequence-aware
 * transfer of the HSAP abstract, instead of a ring that passes every chunk. */
int sap_plan_rank_spans(sap_plan_t plan, int32_t chunk, int64_t* spans, int32_t* n_spans);

/* Canonical item list (see sap_item_t and sap_plan); host memory owned by the plan. */
int sap_plan_items(sap_plan_t plan, const sap_item_t** items, int64_t* n_items);

/* Plan statistics.  unmasked_pairs = sum over documents of L(L+1)/2 (per head) -- the pairs the
 * packed causal mask keeps (HSAP abstract: attention only inside each document), the unit of the
 * FLOP count;
 * n_partial_slots = forward units that write a partial (q-tiles with > 1 unit);
 * n_chunk_pairs = distinct (q_chunk, kv_chunk) pairs that hold an item. */
int sap_plan_stats(sap_plan_t plan, int64_t* unmasked_pairs, int64_t* n_partial_slots, int32_t* n_chunk_pairs);

/* Forward schedule (the work order of sap_attn_fwd: one unit per partial of the HSAP abstract's
 * partial attention computation), host memory owned by the plan:
 *   units: int32[n_units][4] = (q_tile, item_begin, item_count, slot), slot = -1
 *          when the unit writes O/LSE directly, else its partial slot;
 *   order: int32[n_units], heavy-first (item_count descending; ties by the kv chunk
 *          of the unit's items, then by index, so that concurrent units share K/V tiles);
 *   merges: int32[n_merges][3] = (q_tile, first_slot, n_slots). */
int sap_plan_fwd_schedule(sap_plan_t plan, const int32_t** units, int64_t* n_units, const int32_t** order,
                          const int32_t** merges, int64_t* n_merges);

/* Backward schedule (the work order of sap_attn_bwd), host memory owned by the plan:
 *   entries:  int32[n_items][2] = (q_tile, tag), grouped by kv tile, q-tile descending;
 *   kv_units: int32[n_kv_units][3] = (kv_tile, first_entry, n_entries).  A kv tile whose entries
 *             number at most 16 is one unit; a longer list is cut into the parts whose q tiles fall
 *             in one band of 16 q tiles (q_tile / 16 equal), so such a kv tile has several units.
 *             Units are ordered band-major (top band first; a unit's band is that of its first,
 *             highest q tile) and heavy-first (n_entries descending, ties by kv tile) within a band. */
int sap_plan_bwd_schedule(sap_plan_t plan, const int32_t** kv_units, int64_t* n_kv_units, const int32_t** entries);

/* Direct dK/dV stores of sap_attn_bwd, host memory owned by the plan: int32[n_tiles] over the kv
 * tiles of the plan's key/value window (tile l = rows [kv_begin + l * block_n, ...)), 1 where the
 * tile has exactly one backward unit in a full plan.  That unit writes the tile's dK and dV as
 * bf16 directly; every other tile (all tiles of a rank plan, whose dK/dV rows may still receive
 * other devices' partials) is accumulated in fp32 in the workspace and converted at the end. */
int sap_plan_bwd_direct(sap_plan_t plan, const int32_t** flags, int64_t* n_tiles);

/* Fused-merge mode (enable != 0; the pages have no such mode: it computes the merged result of
 * the partials of sap_attn_fwd + sap_merge in one pass, which the exactness of the merge --
 * explainer page, FAQ on equivalence with one device -- allows): the forward schedule gets one unit per
 * q-tile spanning all of its kv chunks, so sap_attn_fwd carries the online
 * softmax across chunk boundaries and writes O and LSE directly -- no fp32
 * partials (the forward workspace holds only the work counter and may be NULL),
 * and sap_merge has nothing to do.  The result
 * is the merged result of the chunked path (the merge is exact), computed in
 * one pass; the per-(q-chunk, kv-chunk) partials are not produced.  enable = 0
 * restores the chunked schedule.  Host-side only: the device copy of the plan
 * is released (the device is synchronised) and uploaded again by the next
 * device call. */
int sap_plan_set_fused_merge(sap_plan_t plan, int enable);

/* Copy the plan's device arrays to the current device on `stream` (plumbing; no counterpart in
 * the pages).  Called
 * implicitly by the first device call that needs them; calling it first keeps
 * the one host-to-device transfer out of later timed calls. */
int sap_plan_upload(sap_plan_t plan, void* stream);

void sap_plan_destroy(sap_plan_t plan);

/* Workspace bytes (plumbing; no counterpart in the pages) for a call with these head counts
 * (which = SAP_WS_FWD for
 * sap_attn_fwd + sap_merge, SAP_WS_BWD for sap_attn_bwd).  The forward
 * workspace holds the fp32 partial outputs and LSEs of the partial slots and
 * the forward's work counter; the backward one holds the fp32 dQ, dK and dV
 * accumulators, the per-row D and LSE*log2(e) and the backward's work counter.
 * Calls that share a workspace must not run at the same time. */
int sap_workspace_size(sap_plan_t plan, int32_t hq, int32_t hkv, int32_t head_dim, int32_t which, size_t* bytes);

/* Forward (HSAP page, abstract: the partial attention computation of each part of the sequence
 * against each part of its keys; method details: the attention pattern of hybrid-context
 * sequences): for every forward unit (q-tile, kv-chunk) and head, the partial
 * attention of the q-tile's rows over that chunk's kv tiles (masked per tag),
 * with online softmax in fp32 on tcgen05 tensor cores.  A q-tile with one unit
 * writes bf16 O and fp32 LSE directly; the others leave fp32 partials (O, LSE)
 * in the workspace for sap_merge.  Rows of a partial that see no key have
 * LSE = -inf and O = 0.  The workspace may be NULL when the plan has no partial slots; with a
 * workspace of the full size the persistent CTAs take their work items in schedule order from a
 * counter in it (reset on `stream` first), without one in a fixed round-robin order (same
 * results: every work item is computed the same way whichever CTA takes it). */
int sap_attn_fwd(sap_plan_t plan, const void* q, const void* k, const void* v, int32_t hq, int32_t hkv,
                 int32_t head_dim, float softmax_scale, void* o, float* lse, void* workspace, size_t ws_bytes,
                 void* stream);

/* One part of the forward, so that the key/value exchange of sequence parallelism can overlap
 * the device's own work (explainer page, compute-communication overlap bullet: compute the current
 * block while the next one arrives).  In a rank plan the forward order lists first the units whose
 * kv tiles all lie in the device's own chunk (sap_plan_fwd_local_units): part 1 runs those -- they
 * read no received keys --, part 2 the others, part 0 all (= sap_attn_fwd).  max_ctas > 0 caps the
 * persistent grid, leaving SMs to a transfer kernel running at the same time (0 = every SM).  The
 * parts write disjoint outputs and partial slots of the same workspace; run parts 1 and 2 before
 * sap_merge.  For a full plan part 1 is every unit and part 2 none.  Other arguments, layouts and
 * errors as sap_attn_fwd (part or max_ctas out of range: SAP_ERR_INVALID_ARG). */
int sap_attn_fwd_part(sap_plan_t plan, int32_t part, int32_t max_ctas, const void* q, const void* k, const void* v,
                      int32_t hq, int32_t hkv, int32_t head_dim, float softmax_scale, void* o, float* lse,
                      void* workspace, size_t ws_bytes, void* stream);

/* Forward units of a plan, and how many of them (listed first in the forward order) lie entirely
 * in a rank plan's own chunk; for a full plan both are the number of units. */
int sap_plan_fwd_local_units(sap_plan_t plan, int64_t* n_local, int64_t* n_units);

/* Merge (HSAP abstract: partial attention results combined into the attention of the whole
 * sequence; explainer page, FAQ: the split computation equals the single-device one -- exact
 * here up to rounding): for every q-tile with several partials, per (row, head)
 *   LSE = M + log sum_b exp(LSE_b - M), M = max_b LSE_b;  O = sum_b exp(LSE_b - LSE) O_b,
 * written as bf16 O and fp32 LSE.  Must follow sap_attn_fwd with the same
 * workspace; a no-op when no q-tile has more than one partial. */
int sap_merge(sap_plan_t plan, const void* workspace, size_t ws_bytes, int32_t hq, int32_t head_dim, void* o,
              float* lse, void* stream);

/* Backward (HSAP page, abstract: training of packed sequences; the gradient is the exact
 * derivative of <dO, O> of the forward above) with the merged O and LSE:
 * D_i = <dO_i, O_i>, P_ij = exp(S_ij - LSE_i),
 * dV_j = sum P_ij dO_i, dS_ij = P_ij (<dO_i, V_j> - D_i), dQ_i = scale sum_j dS_ij K_j,
 * dK_j = scale sum_i dS_ij Q_i, with dK/dV summed over the q heads of each kv
 * head.  Chunk pairs need no merge here: the final LSE normalises every pair
 * and their gradients add.  dQ, dK and dV are accumulated in fp32 in the
 * workspace (dQ once per (q tile, kv tile, head), dK/dV once per backward unit)
 * and converted to bf16 at the end, except the dK/dV of kv tiles with a single unit in a full
 * plan (sap_plan_bwd_direct), which that unit stores as bf16 directly. */
int sap_attn_bwd(sap_plan_t plan, const void* q, const void* k, const void* v, const void* o, const float* lse,
                 const void* dout, int32_t hq, int32_t hkv, int32_t head_dim, float softmax_scale, void* dq,
                 void* dk, void* dv, void* workspace, size_t ws_bytes, void* stream);

/* Byte offsets, inside the backward workspace, of the fp32 dK and dV accumulators that
 * sap_attn_bwd leaves behind: [rows][hkv][head_dim] each, row r = token kv_begin + r of the plan's
 * window (row stride hkv * head_dim floats).  Under sequence parallelism (rank plans) the rows
 * below q_begin hold this device's partial dK/dV for other devices' tokens: sent to their owners
 * and added there with sap_attn_bwd_kv_add.  In a full plan the rows of directly stored tiles
 * (sap_plan_bwd_direct) are not written. */
int sap_workspace_kv_offsets(sap_plan_t plan, int32_t hq, int32_t hkv, int32_t head_dim, size_t* dk_offset,
                             size_t* dv_offset);

/* Adds received fp32 partial gradients into the dK/dV accumulators that the last sap_attn_bwd with
 * this rank plan and workspace left behind, and rewrites the bf16 dK/dV of those rows:
 *   acc[t] += part[t - row_begin]; dk[t] = bf16(acc_dK[t]); dv[t] = bf16(acc_dV[t])
 * for tokens t in [row_begin, row_begin + rows), which must lie in the plan's key/value window
 * (SAP_ERR_INVALID_ARG otherwise, and for a full plan, whose accumulators skip direct tiles).  dk_part, dv_part: fp32 [rows][hkv][head_dim], 16-byte
 * aligned; dk, dv: the bf16 window buffers sap_attn_bwd wrote.  Several calls add up (the chunk
 * pair gradients of the backward add, as on one device); calls on one stream are ordered. */
int sap_attn_bwd_kv_add(sap_plan_t plan, void* workspace, size_t ws_bytes, int32_t hq, int32_t hkv, int32_t head_dim,
                        const float* dk_part, const float* dv_part, int64_t row_begin, int64_t rows, void* dk,
                        void* dv, void* stream);

/* Forward + merge (the same kernels as sap_attn_fwd followed by sap_merge)
 * without any device allocation: the partial outputs and LSEs live in a
 * 16 MiB array compiled into the library instead of a caller-owned workspace.
 * The paper has no counterpart; this call exists for callers that cannot call
 * cudaMalloc -- for example code whose framework owns all device memory
 * through its own pool, or a plugin that is handed only its input and output
 * pointers.
 *   - The plan must already be uploaded to the current device
 *     (sap_plan_upload, or any earlier device call with it), because uploading
 *     allocates; otherwise SAP_ERR_INVALID_ARG.
 *   - Plans whose forward workspace (sap_workspace_size with SAP_WS_FWD)
 *     exceeds 16 MiB are rejected with SAP_ERR_WORKSPACE.
 *   - The first call on a device looks up the array's device address (and the
 *     library's other per-device handles); make that first call before any
 *     stream capture begins.
 *   - All calls on a device share that device's one array, which keeps the
 *     last call's contents.  Calls that may run at the same time on one GPU
 *     (for example on two streams) race on it: serialise them.
 *   - Every device on which the library's kernels are loaded holds the 16 MiB
 *     until the process exits.
 * Arguments, layouts and errors are otherwise those of sap_attn_fwd. */
int sap_attn_fwd_static_scratch(sap_plan_t plan, const void* q, const void* k, const void* v, int32_t hq,
                                int32_t hkv, int32_t head_dim, float softmax_scale, void* o, float* lse,
                                void* stream);

/* Failure detection (no counterpart in the pages).  Synchronise the current device and return
 * SAP_OK, or SAP_ERR_DEVICE if a
 * kernel set the device error word (its code is stored in *code, then the word
 * is cleared). */
int sap_device_status(int32_t* code);

/* Text for a status code (no counterpart in the pages). */
const char* sap_error_string(int status);

/* The last cudaError_t seen by a call that returned SAP_ERR_CUDA (no counterpart in the pages). */
int sap_last_cuda_error(void);

/* Pipeline wait limit of every later kernel launch, in nanoseconds (0 restores the default of
 * 4 s; accepted range 1 ms .. 600 s, else SAP_ERR_INVALID_ARG).  A wait that runs past it sets
 * the device error word (read by sap_device_status) and winds its CTA down: copies and MMAs in
 * flight are waited for, again within the limit, before shared memory and tensor memory are
 * released; that CTA's remaining outputs are left unwritten.  A limit shorter than the longest
 * legitimate wait (a forward unit's whole pass over its kv tiles: milliseconds for long
 * documents) reports false timeouts.  Process-wide; no counterpart in the pages. */
int sap_set_wait_limit_ns(uint64_t limit_ns);

/* Forward kernel variant for later sap_attn_fwd / sap_attn_fwd_part calls (process-wide; the
 * pages have no counterpart -- a B200 form of the same computation):
 *   0 (default)  one CTA per work item of two query heads: two heads of a kv group share each
 *                K/V tile load (even hq / hkv); with an odd group (MHA included) and an even hq,
 *                two adjacent heads each load their own K/V tiles; an odd hq runs one head per
 *                work item;
 *   1            two-CTA clusters (tcgen05 cta_group::2) where head_dim = 128 and hq / hkv is a
 *                multiple of 4: a pair of SMs runs every MMA of four query heads of a kv group as
 *                one M = 256 MMA, each SM loading half of every K and V tile; other shapes keep
 *                variant 0.
 * Both compute the same partials (within rounding: the MMAs' summation order may differ).
 * SAP_ERR_INVALID_ARG for other values. */
int sap_set_forward_variant(int32_t variant);

/* Failure-detection test hook (no counterpart in the pages): arms the next sap_attn_fwd call
 * so that its launch uses wait_limit_ns (100 us .. 10 s, else SAP_ERR_INVALID_ARG) and its first
 * CTA leaves its first V tile out -- no copy is issued, so nothing is in flight --: the MMA
 * issuer's wait for that tile, or the producer's wait for its ring stage to be released,
 * whichever started first, runs out.  The call returns SAP_OK; sap_device_status() then reports
 * SAP_ERR_DEVICE with that wait's timeout bit, and the outputs of that launch are incomplete.
 * The hook disarms itself at that launch; later calls are normal. */
int sap_test_arm_wait_timeout(uint64_t wait_limit_ns);

#ifdef __cplusplus
}
#endif

#endif /* SAP_H_ */
