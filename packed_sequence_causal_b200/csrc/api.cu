// extern "C" entry points of libsap.so (declared in include/sap.h): argument
// checks, plan upload, TMA tensor maps and kernel launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cstring>
#include <mutex>
#include <new>

#include "kernels.cuh"
#include "plan.hpp"
#include "sap.h"

namespace {

thread_local int g_last_cuda_error = 0;

// Pipeline wait limit given to every kernel launch (sap_set_wait_limit_ns), and the armed
// wait-timeout test hook (sap_test_arm_wait_timeout): its limit, 0 when disarmed.
std::atomic<uint64_t> g_wait_limit_ns{4000000000ull};
std::atomic<uint64_t> g_test_timeout_ns{0};

// Forward kernel variant (sap_set_forward_variant): 0 one CTA per work item, 1 two-CTA clusters.
std::atomic<int> g_fwd_variant{0};

// Device error word (bitwise OR of sap::kErr* codes), one per device.
__device__ int g_device_err;

int cuda_fail(cudaError_t e) {
  g_last_cuda_error = (int)e;
  return SAP_ERR_CUDA;
}

#define SAP_CUDA(call)                           \
  do {                                           \
    cudaError_t e_ = (call);                     \
    if (e_ != cudaSuccess) return cuda_fail(e_); \
  } while (0)

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int sms = 0;
  int* err = nullptr;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int device_info(DeviceInfo** out) {
  int dev = 0;
  SAP_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return SAP_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    SAP_CUDA(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev));
    void* p = nullptr;
    SAP_CUDA(cudaGetSymbolAddress(&p, g_device_err));
    d.err = static_cast<int*>(p);
    if (!g_encode) {
      cudaDriverEntryPointQueryResult q;
      void* fn = nullptr;
      SAP_CUDA(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q));
      if (q != cudaDriverEntryPointSuccess || !fn) return cuda_fail(cudaErrorSymbolNotFound);
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    d.ready = true;
  }
  *out = &d;
  return SAP_OK;
}

// [rows][heads][hd] bf16 -> 3-D map with box_rows-row x 64-column boxes, 128-byte swizzle.
int make_map(CUtensorMap* map, const void* base, int64_t rows, int32_t heads, int32_t hd, uint32_t box_rows = 128) {
  cuuint64_t dims[3] = {(cuuint64_t)hd, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)hd * 2, (cuuint64_t)heads * hd * 2};
  cuuint32_t box[3] = {64, 1, box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
  return SAP_OK;
}

// fp32 dQ accumulator [rows][heads][hd] -> 3-D map whose box is a quarter q tile of one head
// (32 rows x hd features, no swizzle): the target of the backward's bulk reductions.
int make_map_f32_tile(CUtensorMap* map, void* base, int64_t rows, int32_t heads, int32_t hd) {
  cuuint64_t dims[3] = {(cuuint64_t)hd, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)hd * 4, (cuuint64_t)heads * hd * 4};
  cuuint32_t box[3] = {(cuuint32_t)hd, 1, 32};  // a quarter of a q tile: the kernel stages and reduces 32 rows at a time
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
  return SAP_OK;
}

// fp32 [rows][heads][hd] accumulator (dK then dV, rows = 2 * n_pad), reduced into in boxes of
// 32 features x 128 rows with 128-byte swizzle (the staging layout the drain warps write).
int make_map_f32_sw128(CUtensorMap* map, void* base, int64_t rows, int32_t heads, int32_t hd) {
  cuuint64_t dims[3] = {(cuuint64_t)hd, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)hd * 4, (cuuint64_t)heads * hd * 4};
  cuuint32_t box[3] = {32, 1, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
  return SAP_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

int check_heads(int32_t hq, int32_t hkv, int32_t hd) {
  if (hq <= 0 || hkv <= 0 || hq % hkv) return SAP_ERR_INVALID_ARG;
  if (hd != 64 && hd != 128) return SAP_ERR_UNSUPPORTED;
  return SAP_OK;
}

int check_kernel_plan(const sap_plan_s* p) {
  if (!p) return SAP_ERR_INVALID_ARG;
  if (p->block_m != 128 || p->block_n != 128) return SAP_ERR_UNSUPPORTED;
  return SAP_OK;
}

// Workspace layouts (256-byte aligned pieces).
struct FwdWs {
  size_t o_part = 0, lse_part = 0, work_next = 0, total = 0;
};
FwdWs fwd_ws(const sap_plan_s* p, int32_t hq, int32_t hd) {
  FwdWs w;
  const size_t slots = (size_t)p->n_slots;
  w.o_part = 0;                                                           // [slots][hq][128][hd] fp32
  w.lse_part = round_up((int64_t)(slots * hq * 128 * hd * 4), 256);      // [slots][hq][128] fp32
  w.work_next = w.lse_part + round_up((int64_t)(slots * hq * 128 * 4), 256);  // int: work counter
  w.total = w.work_next + 256;
  return w;
}
struct BwdWs {
  size_t dq_acc = 0, dkv_acc = 0, dvec = 0, lse2 = 0, work_next = 0, total = 0;
  int64_t n_pad = 0, n_pad_kv = 0;  // query-side and key/value-side window rows, rounded up to 128
};
BwdWs bwd_ws(const sap_plan_s* p, int32_t hq, int32_t hkv, int32_t hd) {
  BwdWs w;
  w.n_pad = round_up(p->q_rows(), 128);
  w.n_pad_kv = round_up(p->kv_rows(), 128);
  w.dq_acc = 0;                                                             // [n_pad][hq][hd] fp32
  w.dkv_acc = round_up(w.n_pad * hq * hd * 4, 1024);                        // [2][n_pad_kv][hkv][hd] fp32
  w.dvec = w.dkv_acc + round_up(2 * w.n_pad_kv * hkv * hd * 4, 256);        // [hq][n_pad]
  w.lse2 = w.dvec + round_up(w.n_pad * hq * 4, 256);                        // [hq][n_pad]
  w.work_next = w.lse2 + round_up(w.n_pad * hq * 4, 256);                   // int: work counter
  w.total = w.work_next + 256;
  return w;
}

// Forward parameters of a plan's window (everything but the buffers and the error word).
sap::FwdParams fwd_params(const sap_plan_s* p, int32_t hq, int32_t hkv, float softmax_scale) {
  const int32_t* base = static_cast<const int32_t*>(p->dev);
  sap::FwdParams fp{};
  fp.items = base + p->off_items;
  fp.units = base + p->off_units;
  fp.order = base + p->off_order;
  fp.tok_lo = base + p->off_tok_lo;
  fp.n_units = (int32_t)(p->fwd_units.size() / 4);
  fp.hq = hq;
  fp.group = hq / hkv;
  fp.q0 = p->q_begin;
  fp.kv0 = p->kv_begin;
  fp.q_end = p->q_end;
  fp.lse_ld = p->q_rows();
  fp.scale_log2 = softmax_scale * 1.4426950408889634f;
  fp.wait_ns = g_wait_limit_ns.load();
  fp.skip_v_load = 0;
  return fp;
}

// Scratch for sap_attn_fwd_static_scratch: the forward's partial outputs and
// LSEs live here instead of in a caller-allocated workspace.  Every GPU that
// loads the library holds these 16 MiB until the process exits.
constexpr size_t kStaticScratchBytes = size_t(16) << 20;
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch per device, looked up once with that
// device current (host code must not use the symbol itself as a pointer).
void* g_static_scratch_addr[kMaxDevices] = {};
std::mutex g_static_scratch_mu;

int static_scratch_address(void** out) {
  int dev = 0;
  SAP_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return SAP_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_static_scratch_mu);
  if (!g_static_scratch_addr[dev]) {
    void* ptr = nullptr;
    SAP_CUDA(cudaGetSymbolAddress(&ptr, g_static_scratch));
    g_static_scratch_addr[dev] = ptr;
  }
  *out = g_static_scratch_addr[dev];
  return SAP_OK;
}

}  // namespace

extern "C" {

int sap_plan(const int32_t* cu_seqlens_host, int32_t num_docs, int64_t total_tokens, int32_t num_chunks,
             int32_t block_m, int32_t block_n, sap_plan_t* out) {
  if (!out) return SAP_ERR_INVALID_ARG;
  *out = nullptr;
  sap_plan_s* p = new (std::nothrow) sap_plan_s();
  if (!p) return SAP_ERR_NOMEM;
  int rc;
  try {
    rc = sap_plan_build(cu_seqlens_host, num_docs, total_tokens, num_chunks, nullptr, block_m, block_n, p);
  } catch (const std::bad_alloc&) {
    rc = SAP_ERR_NOMEM;
  }
  if (rc != SAP_OK) {
    delete p;
    return rc;
  }
  *out = p;
  return SAP_OK;
}

int sap_plan_chunks(const int32_t* cu_seqlens_host, int32_t num_docs, int64_t total_tokens,
                    const int64_t* chunk_bounds, int32_t num_chunks, int32_t block_m, int32_t block_n,
                    sap_plan_t* out) {
  if (!out || !chunk_bounds) return SAP_ERR_INVALID_ARG;
  *out = nullptr;
  if (num_chunks < 1) return SAP_ERR_BAD_CHUNKS;
  sap_plan_s* p = new (std::nothrow) sap_plan_s();
  if (!p) return SAP_ERR_NOMEM;
  int rc;
  try {
    rc = sap_plan_build(cu_seqlens_host, num_docs, total_tokens, num_chunks, chunk_bounds, block_m, block_n, p);
  } catch (const std::bad_alloc&) {
    rc = SAP_ERR_NOMEM;
  }
  if (rc != SAP_OK) {
    delete p;
    return rc;
  }
  *out = p;
  return SAP_OK;
}

int sap_balanced_chunks(const int32_t* cu_seqlens_host, int32_t num_docs, int64_t total_tokens, int32_t num_chunks,
                        int32_t block, int64_t* chunk_bounds) {
  try {
    return sap_balanced_bounds(cu_seqlens_host, num_docs, total_tokens, num_chunks, block, chunk_bounds);
  } catch (const std::bad_alloc&) {
    return SAP_ERR_NOMEM;
  }
}

int sap_plan_rank(sap_plan_t plan, int32_t chunk, sap_plan_t* out) {
  if (!out) return SAP_ERR_INVALID_ARG;
  *out = nullptr;
  sap_plan_s* r = new (std::nothrow) sap_plan_s();
  if (!r) return SAP_ERR_NOMEM;
  int rc;
  try {
    rc = sap_plan_build_rank(plan, chunk, r);
  } catch (const std::bad_alloc&) {
    rc = SAP_ERR_NOMEM;
  }
  if (rc != SAP_OK) {
    delete r;
    return rc;
  }
  *out = r;
  return SAP_OK;
}

int sap_plan_window(sap_plan_t plan, int64_t* q_begin, int64_t* q_end, int64_t* kv_begin, int64_t* span_begin) {
  if (!plan) return SAP_ERR_INVALID_ARG;
  if (q_begin) *q_begin = plan->q_begin;
  if (q_end) *q_end = plan->q_end;
  if (kv_begin) *kv_begin = plan->kv_begin;
  if (span_begin) *span_begin = plan->span_begin;
  return SAP_OK;
}

int sap_plan_chunk_bounds(sap_plan_t plan, const int64_t** bounds, int32_t* num_chunks) {
  if (!plan) return SAP_ERR_INVALID_ARG;
  if (bounds) *bounds = plan->bounds.data();
  if (num_chunks) *num_chunks = plan->num_chunks;
  return SAP_OK;
}

int sap_plan_chunk_stats(sap_plan_t plan, int64_t* items_per_chunk, int64_t* pairs_per_chunk) {
  if (!plan) return SAP_ERR_INVALID_ARG;
  const int32_t P = plan->num_chunks;
  if (items_per_chunk) {
    for (int32_t c = 0; c < P; ++c) items_per_chunk[c] = 0;
    for (const auto& it : plan->items) items_per_chunk[it.q_chunk]++;
  }
  if (pairs_per_chunk) {
    for (int32_t c = 0; c < P; ++c) {
      pairs_per_chunk[c] = 0;
      const int64_t a = plan->bounds[c] > plan->q_begin ? plan->bounds[c] : plan->q_begin;
      const int64_t b = plan->bounds[c + 1] < plan->q_end ? plan->bounds[c + 1] : plan->q_end;
      for (int64_t i = a; i < b; ++i) pairs_per_chunk[c] += i - plan->tok_lo[i] + 1;
    }
  }
  return SAP_OK;
}

int sap_plan_rank_spans(sap_plan_t plan, int32_t chunk, int64_t* spans, int32_t* n_spans) {
  if (!plan || !spans || !n_spans || plan->rank_chunk >= 0 || chunk < 0 || chunk >= plan->num_chunks)
    return SAP_ERR_INVALID_ARG;
  const int64_t q0 = plan->bounds[chunk];
  const int64_t s0 = q0 < plan->n ? plan->tok_lo[q0] : q0;
  int32_t k = 0;
  for (int32_t b = 0; b < chunk; ++b) {
    const int64_t lo = s0 > plan->bounds[b] ? s0 : plan->bounds[b];
    const int64_t hi = q0 < plan->bounds[b + 1] ? q0 : plan->bounds[b + 1];
    if (lo < hi) {
      spans[3 * k] = b, spans[3 * k + 1] = lo, spans[3 * k + 2] = hi;
      ++k;
    }
  }
  *n_spans = k;
  return SAP_OK;
}

int sap_plan_items(sap_plan_t plan, const sap_item_t** items, int64_t* n_items) {
  if (!plan || !items || !n_items) return SAP_ERR_INVALID_ARG;
  *items = plan->items.data();
  *n_items = (int64_t)plan->items.size();
  return SAP_OK;
}

int sap_plan_stats(sap_plan_t plan, int64_t* unmasked_pairs, int64_t* n_partial_slots, int32_t* n_chunk_pairs) {
  if (!plan) return SAP_ERR_INVALID_ARG;
  if (unmasked_pairs) *unmasked_pairs = plan->unmasked_pairs;
  if (n_partial_slots) *n_partial_slots = plan->n_slots;
  if (n_chunk_pairs) *n_chunk_pairs = plan->n_chunk_pairs;
  return SAP_OK;
}

int sap_plan_fwd_schedule(sap_plan_t plan, const int32_t** units, int64_t* n_units, const int32_t** order,
                          const int32_t** merges, int64_t* n_merges) {
  if (!plan) return SAP_ERR_INVALID_ARG;
  if (units) *units = plan->fwd_units.data();
  if (n_units) *n_units = (int64_t)plan->fwd_units.size() / 4;
  if (order) *order = plan->fwd_order.data();
  if (merges) *merges = plan->merges.data();
  if (n_merges) *n_merges = (int64_t)plan->merges.size() / 3;
  return SAP_OK;
}

int sap_plan_bwd_schedule(sap_plan_t plan, const int32_t** kv_units, int64_t* n_kv_units, const int32_t** entries) {
  if (!plan) return SAP_ERR_INVALID_ARG;
  if (kv_units) *kv_units = plan->kv_units.data();
  if (n_kv_units) *n_kv_units = (int64_t)plan->kv_units.size() / 3;
  if (entries) *entries = plan->kv_entries.data();
  return SAP_OK;
}

int sap_plan_bwd_direct(sap_plan_t plan, const int32_t** flags, int64_t* n_tiles) {
  if (!plan) return SAP_ERR_INVALID_ARG;
  if (flags) *flags = plan->kv_direct.data();
  if (n_tiles) *n_tiles = (int64_t)plan->kv_direct.size();
  return SAP_OK;
}

int sap_plan_upload(sap_plan_t p, void* stream) {
  if (!p) return SAP_ERR_INVALID_ARG;
  int dev = 0;
  SAP_CUDA(cudaGetDevice(&dev));
  if (p->dev && p->dev_id == dev) return SAP_OK;
  if (p->dev) {
    cudaFree(p->dev);
    p->dev = nullptr;
  }
  // One int32 buffer; every piece starts on a 64-element (256-byte) boundary.
  size_t off = 0;
  auto place = [&](size_t words) {
    size_t o = off;
    off += (size_t)round_up((int64_t)words, 64);
    return o;
  };
  p->off_items = place(p->items.size() * 5);
  p->off_units = place(p->fwd_units.size());
  p->off_order = place(p->fwd_order.size());
  p->off_merges = place(p->merges.size());
  p->off_kv_units = place(p->kv_units.size());
  p->off_kv_entries = place(p->kv_entries.size());
  p->off_kv_direct = place(p->kv_direct.size());
  p->off_kv_acc_tiles = place(p->kv_acc_tiles.size());
  p->off_tok_lo = place(p->tok_lo.size());
  p->off_tok_hi = place(p->tok_hi.size());
  p->dev_words = off > 0 ? off : 64;
  void* d = nullptr;
  SAP_CUDA(cudaMalloc(&d, p->dev_words * 4));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* base = static_cast<int32_t*>(d);
  auto put = [&](size_t o, const void* src, size_t words) -> cudaError_t {
    if (!words) return cudaSuccess;
    return cudaMemcpyAsync(base + o, src, words * 4, cudaMemcpyHostToDevice, s);
  };
  cudaError_t e = cudaSuccess;
  if (e == cudaSuccess) e = put(p->off_items, p->items.data(), p->items.size() * 5);
  if (e == cudaSuccess) e = put(p->off_units, p->fwd_units.data(), p->fwd_units.size());
  if (e == cudaSuccess) e = put(p->off_order, p->fwd_order.data(), p->fwd_order.size());
  if (e == cudaSuccess) e = put(p->off_merges, p->merges.data(), p->merges.size());
  if (e == cudaSuccess) e = put(p->off_kv_units, p->kv_units.data(), p->kv_units.size());
  if (e == cudaSuccess) e = put(p->off_kv_entries, p->kv_entries.data(), p->kv_entries.size());
  if (e == cudaSuccess) e = put(p->off_kv_direct, p->kv_direct.data(), p->kv_direct.size());
  if (e == cudaSuccess) e = put(p->off_kv_acc_tiles, p->kv_acc_tiles.data(), p->kv_acc_tiles.size());
  if (e == cudaSuccess) e = put(p->off_tok_lo, p->tok_lo.data(), p->tok_lo.size());
  if (e == cudaSuccess) e = put(p->off_tok_hi, p->tok_hi.data(), p->tok_hi.size());
  // The host arrays stay alive with the plan, but copies from pageable memory
  // may still be staged: finish them before returning.
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    cudaFree(d);
    return cuda_fail(e);
  }
  p->dev = d;
  p->dev_id = dev;
  return SAP_OK;
}

int sap_plan_set_fused_merge(sap_plan_t plan, int enable) {
  if (!plan) return SAP_ERR_INVALID_ARG;
  if (plan->fused_merge == (enable != 0)) return SAP_OK;
  try {
    sap_plan_build_fwd_schedule(plan, enable != 0);
  } catch (const std::bad_alloc&) {
    return SAP_ERR_NOMEM;
  }
  if (plan->dev) {  // the device copy no longer matches: drop it, the next device call uploads again
    cudaError_t e = cudaFree(plan->dev);
    plan->dev = nullptr;
    plan->dev_id = -1;
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return SAP_OK;
}

void sap_plan_destroy(sap_plan_t plan) {
  if (!plan) return;
  if (plan->dev) cudaFree(plan->dev);
  delete plan;
}

int sap_workspace_kv_offsets(sap_plan_t plan, int32_t hq, int32_t hkv, int32_t head_dim, size_t* dk_offset,
                             size_t* dv_offset) {
  if (!plan) return SAP_ERR_INVALID_ARG;
  int rc = check_heads(hq, hkv, head_dim);
  if (rc) return rc;
  const BwdWs ws = bwd_ws(plan, hq, hkv, head_dim);
  if (dk_offset) *dk_offset = ws.dkv_acc;
  if (dv_offset) *dv_offset = ws.dkv_acc + (size_t)ws.n_pad_kv * hkv * head_dim * 4;
  return SAP_OK;
}

int sap_workspace_size(sap_plan_t plan, int32_t hq, int32_t hkv, int32_t head_dim, int32_t which, size_t* bytes) {
  if (!plan || !bytes) return SAP_ERR_INVALID_ARG;
  int rc = check_heads(hq, hkv, head_dim);
  if (rc) return rc;
  if (which == SAP_WS_FWD)
    *bytes = fwd_ws(plan, hq, head_dim).total;
  else if (which == SAP_WS_BWD)
    *bytes = bwd_ws(plan, hq, hkv, head_dim).total;
  else
    return SAP_ERR_INVALID_ARG;
  return SAP_OK;
}

int sap_attn_fwd(sap_plan_t p, const void* q, const void* k, const void* v, int32_t hq, int32_t hkv,
                 int32_t head_dim, float softmax_scale, void* o, float* lse, void* workspace, size_t ws_bytes,
                 void* stream) {
  return sap_attn_fwd_part(p, 0, 0, q, k, v, hq, hkv, head_dim, softmax_scale, o, lse, workspace, ws_bytes, stream);
}

int sap_plan_fwd_local_units(sap_plan_t plan, int64_t* n_local, int64_t* n_units) {
  if (!plan) return SAP_ERR_INVALID_ARG;
  if (n_local) *n_local = plan->n_local_units;
  if (n_units) *n_units = (int64_t)plan->fwd_units.size() / 4;
  return SAP_OK;
}

int sap_attn_fwd_part(sap_plan_t p, int32_t part, int32_t max_ctas, const void* q, const void* k, const void* v,
                      int32_t hq, int32_t hkv, int32_t head_dim, float softmax_scale, void* o, float* lse,
                      void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_kernel_plan(p);
  if (rc) return rc;
  if (part < 0 || part > 2 || max_ctas < 0) return SAP_ERR_INVALID_ARG;
  if ((rc = check_heads(hq, hkv, head_dim))) return rc;
  if (p->q_rows() == 0) return SAP_OK;
  if (!q || !k || !v || !o || !lse) return SAP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return SAP_ERR_INVALID_ARG;
  const FwdWs ws = fwd_ws(p, hq, head_dim);
  if (ws.total > 0 && p->n_slots > 0 && (!workspace || ws_bytes < ws.total || !aligned16(workspace)))
    return SAP_ERR_WORKSPACE;
  DeviceInfo* di = nullptr;
  if ((rc = device_info(&di))) return rc;
  if ((rc = sap_plan_upload(p, stream))) return rc;
  // the two-CTA variant where it applies (head_dim 128, GQA group a multiple of 4); each CTA of a
  // pair loads 64-row halves of the K tiles
  const bool two_cta = g_fwd_variant.load() == 1 && head_dim == 128 && (hq / hkv) % 4 == 0;
  CUtensorMap tq, tk, tv;
  if ((rc = make_map(&tq, q, p->q_rows(), hq, head_dim))) return rc;
  if ((rc = make_map(&tk, k, p->kv_rows(), hkv, head_dim, two_cta ? 64 : 128))) return rc;
  if ((rc = make_map(&tv, v, p->kv_rows(), hkv, head_dim))) return rc;
  sap::FwdParams fp = fwd_params(p, hq, hkv, softmax_scale);
  // part 1: the first n_local_units of the order; part 2: the rest; part 0: all
  const int64_t n_all = (int64_t)(p->fwd_units.size() / 4);
  const int64_t first = part == 2 ? p->n_local_units : 0;
  const int64_t count = part == 0 ? n_all : part == 1 ? p->n_local_units : n_all - p->n_local_units;
  fp.order += first;
  fp.n_units = (int32_t)count;
  if (const uint64_t t = g_test_timeout_ns.exchange(0)) {  // armed test hook: this launch only
    fp.skip_v_load = 1;
    fp.wait_ns = t;
  }
  fp.o = static_cast<__nv_bfloat16*>(o);
  fp.lse = lse;
  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  fp.o_part = p->n_slots ? reinterpret_cast<float*>(wsb + ws.o_part) : nullptr;
  fp.lse_part = p->n_slots ? reinterpret_cast<float*>(wsb + ws.lse_part) : nullptr;
  fp.err = di->err;
  const int64_t work = (int64_t)fp.n_units * hq;
  if (work == 0) return SAP_OK;
  if (work > INT32_MAX) return SAP_ERR_INVALID_ARG;
  // A full workspace carries the work counter of the dynamic work order (reset on this stream
  // before the launch); without one (allowed when there are no partial slots) the order is static.
  if (workspace && ws_bytes >= ws.total && aligned16(workspace)) {
    fp.work_next = reinterpret_cast<int*>(wsb + ws.work_next);
    const cudaError_t ez = cudaMemsetAsync(fp.work_next, 0, sizeof(int), static_cast<cudaStream_t>(stream));
    if (ez != cudaSuccess) return cuda_fail(ez);
  }
  const int sms = max_ctas > 0 && max_ctas < di->sms ? max_ctas : di->sms;
  const int grid = (int)(work < sms ? work : sms);
  cudaError_t e = head_dim == 64
                      ? sap::launch_fwd<64>(tq, tk, tv, fp, grid, static_cast<cudaStream_t>(stream))
                      : sap::launch_fwd<128>(tq, tk, tv, fp, grid, static_cast<cudaStream_t>(stream), two_cta);
  if (e != cudaSuccess) return cuda_fail(e);
  return SAP_OK;
}

int sap_merge(sap_plan_t p, const void* workspace, size_t ws_bytes, int32_t hq, int32_t head_dim, void* o,
              float* lse, void* stream) {
  int rc = check_kernel_plan(p);
  if (rc) return rc;
  if (hq <= 0) return SAP_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return SAP_ERR_UNSUPPORTED;
  const int64_t n_merges = (int64_t)p->merges.size() / 3;
  if (p->q_rows() == 0 || n_merges == 0) return SAP_OK;
  if (!o || !lse || !aligned16(o)) return SAP_ERR_INVALID_ARG;
  const FwdWs ws = fwd_ws(p, hq, head_dim);
  if (!workspace || ws_bytes < ws.total || !aligned16(workspace)) return SAP_ERR_WORKSPACE;
  if ((rc = sap_plan_upload(p, stream))) return rc;
  const int32_t* base = static_cast<const int32_t*>(p->dev);
  const uint8_t* wsb = static_cast<const uint8_t*>(workspace);
  const float* op = reinterpret_cast<const float*>(wsb + ws.o_part);
  const float* lp = reinterpret_cast<const float*>(wsb + ws.lse_part);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e =
      head_dim == 64 ? sap::launch_merge<64>(base + p->off_merges, n_merges, hq, p->q_begin, p->q_end, op, lp,
                                             static_cast<__nv_bfloat16*>(o), lse, s)
                     : sap::launch_merge<128>(base + p->off_merges, n_merges, hq, p->q_begin, p->q_end, op, lp,
                                              static_cast<__nv_bfloat16*>(o), lse, s);
  if (e != cudaSuccess) return cuda_fail(e);
  return SAP_OK;
}

int sap_attn_bwd(sap_plan_t p, const void* q, const void* k, const void* v, const void* o, const float* lse,
                 const void* dout, int32_t hq, int32_t hkv, int32_t head_dim, float softmax_scale, void* dq,
                 void* dk, void* dv, void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_kernel_plan(p);
  if (rc) return rc;
  if ((rc = check_heads(hq, hkv, head_dim))) return rc;
  if (p->q_rows() == 0) return SAP_OK;
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return SAP_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, o, lse, dout, dq, dk, dv};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return SAP_ERR_INVALID_ARG;
  const BwdWs ws = bwd_ws(p, hq, hkv, head_dim);
  if (!workspace || ws_bytes < ws.total || !aligned16(workspace)) return SAP_ERR_WORKSPACE;
  DeviceInfo* di = nullptr;
  if ((rc = device_info(&di))) return rc;
  if ((rc = sap_plan_upload(p, stream))) return rc;
  CUtensorMap tq, tk, tv, tdo;
  if ((rc = make_map(&tq, q, p->q_rows(), hq, head_dim))) return rc;
  if ((rc = make_map(&tk, k, p->kv_rows(), hkv, head_dim))) return rc;
  if ((rc = make_map(&tv, v, p->kv_rows(), hkv, head_dim))) return rc;
  if ((rc = make_map(&tdo, dout, p->q_rows(), hq, head_dim))) return rc;
  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  float* dq_acc = reinterpret_cast<float*>(wsb + ws.dq_acc);
  float* dkv_acc = reinterpret_cast<float*>(wsb + ws.dkv_acc);
  CUtensorMap tdq, tdkv;
  // d = 128 stages dQ^T as 64-row [q][d] tiles; d = 64 stages dQ rows as 128-byte-swizzled boxes
  if ((rc = head_dim == 128 ? make_map_f32_tile(&tdq, dq_acc, ws.n_pad, hq, head_dim)
                            : make_map_f32_sw128(&tdq, dq_acc, ws.n_pad, hq, head_dim)))
    return rc;
  if ((rc = make_map_f32_sw128(&tdkv, dkv_acc, 2 * ws.n_pad_kv, hkv, head_dim))) return rc;
  float* dvec = reinterpret_cast<float*>(wsb + ws.dvec);
  float* lse2 = reinterpret_cast<float*>(wsb + ws.lse2);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const __nv_bfloat16* ob = static_cast<const __nv_bfloat16*>(o);
  const __nv_bfloat16* dob = static_cast<const __nv_bfloat16*>(dout);
  // bf16 dK / dV outputs, stored directly by the units of kv tiles that have no other unit
  CUtensorMap tdk, tdv;
  if ((rc = make_map(&tdk, dk, p->kv_rows(), hkv, head_dim))) return rc;
  if ((rc = make_map(&tdv, dv, p->kv_rows(), hkv, head_dim))) return rc;
  const int32_t* base = static_cast<const int32_t*>(p->dev);
  const int32_t* kv_direct = base + p->off_kv_direct;
  cudaError_t e = head_dim == 64 ? sap::launch_bwd_pre<64>(ob, dob, lse, p->q_rows(), ws.n_pad, ws.n_pad_kv, hq, hkv,
                                                           dvec, lse2, dq_acc, dkv_acc, kv_direct,
                                                           reinterpret_cast<int*>(wsb + ws.work_next), s)
                                 : sap::launch_bwd_pre<128>(ob, dob, lse, p->q_rows(), ws.n_pad, ws.n_pad_kv, hq, hkv,
                                                            dvec, lse2, dq_acc, dkv_acc, kv_direct,
                                                            reinterpret_cast<int*>(wsb + ws.work_next), s);
  if (e != cudaSuccess) return cuda_fail(e);
  sap::BwdParams bp;
  bp.kv_units = base + p->off_kv_units;
  bp.entries = base + p->off_kv_entries;
  bp.tok_hi = base + p->off_tok_hi;
  bp.n_kv_units = (int32_t)(p->kv_units.size() / 3);
  bp.hq = hq;
  bp.hkv = hkv;
  bp.group = hq / hkv;
  bp.q0 = p->q_begin;
  bp.kv0 = p->kv_begin;
  bp.q_end = p->q_end;
  bp.n_pad = ws.n_pad;
  bp.n_pad_kv = ws.n_pad_kv;
  bp.scale_log2 = softmax_scale * 1.4426950408889634f;
  bp.scale = softmax_scale;
  bp.lse2 = lse2;
  bp.dvec = dvec;
  bp.dq_acc = dq_acc;
  bp.kv_direct = kv_direct;
  bp.work_next = reinterpret_cast<int*>(wsb + ws.work_next);  // zeroed by the pre-pass
  bp.err = di->err;
  bp.wait_ns = g_wait_limit_ns.load();
  const int64_t work = (int64_t)bp.n_kv_units * hkv;
  if (work > 0) {
    const int grid = (int)(work < di->sms ? work : di->sms);
    e = head_dim == 64 ? sap::launch_bwd<64>(tq, tk, tv, tdo, tdq, tdkv, tdk, tdv, bp, grid, s)
                       : sap::launch_bwd<128>(tq, tk, tv, tdo, tdq, tdkv, tdk, tdv, bp, grid, s);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  e = sap::launch_bwd_post(dq_acc, static_cast<__nv_bfloat16*>(dq), p->q_rows() * hq * head_dim, dkv_acc,
                           static_cast<__nv_bfloat16*>(dk), static_cast<__nv_bfloat16*>(dv),
                           p->kv_rows() * hkv * head_dim, ws.n_pad_kv * hkv * head_dim, base + p->off_kv_acc_tiles,
                           (int64_t)p->kv_acc_tiles.size(), (int64_t)hkv * head_dim, s);
  if (e != cudaSuccess) return cuda_fail(e);
  return SAP_OK;
}

int sap_attn_bwd_kv_add(sap_plan_t p, void* workspace, size_t ws_bytes, int32_t hq, int32_t hkv, int32_t head_dim,
                        const float* dk_part, const float* dv_part, int64_t row_begin, int64_t rows, void* dk,
                        void* dv, void* stream) {
  if (!p) return SAP_ERR_INVALID_ARG;
  int rc = check_heads(hq, hkv, head_dim);
  if (rc) return rc;
  if (p->rank_chunk < 0) return SAP_ERR_INVALID_ARG;  // a full plan's accumulators may skip direct tiles
  if (rows == 0) return SAP_OK;
  if (rows < 0 || row_begin < p->kv_begin || row_begin + rows > p->q_end) return SAP_ERR_INVALID_ARG;
  if (!dk_part || !dv_part || !dk || !dv || !aligned16(dk_part) || !aligned16(dv_part) || !aligned16(dk) ||
      !aligned16(dv))
    return SAP_ERR_INVALID_ARG;
  const BwdWs ws = bwd_ws(p, hq, hkv, head_dim);
  if (!workspace || ws_bytes < ws.total || !aligned16(workspace)) return SAP_ERR_WORKSPACE;
  float* dkv_acc = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + ws.dkv_acc);
  const int64_t row_elems = (int64_t)hkv * head_dim;
  cudaError_t e = sap::launch_kv_add(dkv_acc, ws.n_pad_kv * row_elems, dk_part, dv_part, row_begin - p->kv_begin,
                                     rows, row_elems, static_cast<__nv_bfloat16*>(dk),
                                     static_cast<__nv_bfloat16*>(dv), static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return SAP_OK;
}

int sap_device_status(int32_t* code) {
  DeviceInfo* di = nullptr;
  int rc = device_info(&di);
  if (rc) return rc;
  SAP_CUDA(cudaDeviceSynchronize());
  int v = 0;
  SAP_CUDA(cudaMemcpyFromSymbol(&v, g_device_err, sizeof(int)));
  if (code) *code = v;
  if (v) {
    const int zero = 0;
    SAP_CUDA(cudaMemcpyToSymbol(g_device_err, &zero, sizeof(int)));
    return SAP_ERR_DEVICE;
  }
  return SAP_OK;
}

const char* sap_error_string(int status) {
  switch (status) {
    case SAP_OK: return "ok";
    case SAP_ERR_INVALID_ARG: return "invalid argument";
    case SAP_ERR_BAD_SEQLENS: return "invalid cu_seqlens";
    case SAP_ERR_BAD_CHUNKS: return "invalid chunk partition";
    case SAP_ERR_WORKSPACE: return "workspace missing or too small";
    case SAP_ERR_CUDA: return "CUDA runtime error";
    case SAP_ERR_DEVICE: return "device error word set (a kernel wait timed out)";
    case SAP_ERR_UNSUPPORTED: return "unsupported head_dim or tile size";
    case SAP_ERR_NOMEM: return "host allocation failed";
    default: return "unknown status";
  }
}

int sap_last_cuda_error(void) { return g_last_cuda_error; }

int sap_set_wait_limit_ns(uint64_t limit_ns) {
  if (limit_ns == 0) limit_ns = 4000000000ull;
  if (limit_ns < 1000000ull || limit_ns > 600000000000ull) return SAP_ERR_INVALID_ARG;
  g_wait_limit_ns.store(limit_ns);
  return SAP_OK;
}

int sap_set_forward_variant(int32_t variant) {
  if (variant != 0 && variant != 1) return SAP_ERR_INVALID_ARG;
  g_fwd_variant.store(variant);
  return SAP_OK;
}

int sap_test_arm_wait_timeout(uint64_t wait_limit_ns) {
  if (wait_limit_ns < 100000ull || wait_limit_ns > 10000000000ull) return SAP_ERR_INVALID_ARG;
  g_test_timeout_ns.store(wait_limit_ns);
  return SAP_OK;
}

int sap_attn_fwd_static_scratch(sap_plan_t p, const void* q, const void* k, const void* v, int32_t hq, int32_t hkv,
                                int32_t head_dim, float softmax_scale, void* o, float* lse, void* stream) {
  int rc = check_kernel_plan(p);
  if (rc) return rc;
  if ((rc = check_heads(hq, hkv, head_dim))) return rc;
  if (p->q_rows() == 0) return SAP_OK;
  if (!q || !k || !v || !o || !lse) return SAP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return SAP_ERR_INVALID_ARG;
  // Uploading a plan allocates device memory, so this call only accepts a plan
  // already uploaded to the current device.
  int dev = 0;
  SAP_CUDA(cudaGetDevice(&dev));
  if (!p->dev || p->dev_id != dev) return SAP_ERR_INVALID_ARG;
  const FwdWs ws = fwd_ws(p, hq, head_dim);
  if (ws.total > kStaticScratchBytes) return SAP_ERR_WORKSPACE;
  DeviceInfo* di = nullptr;
  if ((rc = device_info(&di))) return rc;
  void* scratch = nullptr;
  if ((rc = static_scratch_address(&scratch))) return rc;
  CUtensorMap tq, tk, tv;
  if ((rc = make_map(&tq, q, p->q_rows(), hq, head_dim))) return rc;
  if ((rc = make_map(&tk, k, p->kv_rows(), hkv, head_dim))) return rc;
  if ((rc = make_map(&tv, v, p->kv_rows(), hkv, head_dim))) return rc;
  const int32_t* base = static_cast<const int32_t*>(p->dev);
  uint8_t* wsb = static_cast<uint8_t*>(scratch);
  sap::FwdParams fp = fwd_params(p, hq, hkv, softmax_scale);
  fp.o = static_cast<__nv_bfloat16*>(o);
  fp.lse = lse;
  // Every (slot, head, row) partial that the merge reads is written by this
  // call's forward kernel first, so nothing in the scratch needs clearing.
  fp.o_part = reinterpret_cast<float*>(wsb + ws.o_part);
  fp.lse_part = reinterpret_cast<float*>(wsb + ws.lse_part);
  fp.err = di->err;
  const int64_t work = (int64_t)fp.n_units * hq;
  if (work == 0) return SAP_OK;
  if (work > INT32_MAX) return SAP_ERR_INVALID_ARG;
  const int grid = (int)(work < di->sms ? work : di->sms);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = head_dim == 64 ? sap::launch_fwd<64>(tq, tk, tv, fp, grid, s)
                                 : sap::launch_fwd<128>(tq, tk, tv, fp, grid, s);
  if (e != cudaSuccess) return cuda_fail(e);
  const int64_t n_merges = (int64_t)p->merges.size() / 3;
  if (n_merges > 0) {
    e = head_dim == 64 ? sap::launch_merge<64>(base + p->off_merges, n_merges, hq, p->q_begin, p->q_end, fp.o_part,
                                               fp.lse_part, fp.o, lse, s)
                       : sap::launch_merge<128>(base + p->off_merges, n_merges, hq, p->q_begin, p->q_end,
                                                fp.o_part, fp.lse_part, fp.o, lse, s);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return SAP_OK;
}

}  // extern "C"
