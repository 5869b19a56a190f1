// Memory-bound kernels of the path: the exact LSE merge of partial outputs,
// the backward pre-pass (D_i and LSE in the log2 domain, zeroed dQ, dK and dV
// accumulators) and the fp32 -> bf16 conversion of the dQ, dK and dV
// accumulators.  One warp per (row, head) keeps every global access coalesced
// along the head dimension.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.cuh"

namespace sap {

namespace {

constexpr int kWarpsPerBlock = 8;

template <int E>
struct Vec;
template <>
struct Vec<2> {
  static __device__ __forceinline__ void load(const float* p, float* v) {
    float2 t = *reinterpret_cast<const float2*>(p);
    v[0] = t.x, v[1] = t.y;
  }
  static __device__ __forceinline__ void load_bf16(const __nv_bfloat16* p, float* v) {
    __nv_bfloat162 t = *reinterpret_cast<const __nv_bfloat162*>(p);
    v[0] = __bfloat162float(t.x), v[1] = __bfloat162float(t.y);
  }
  static __device__ __forceinline__ void store_bf16(__nv_bfloat16* p, const float* v) {
    *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(v[0], v[1]);
  }
  static __device__ __forceinline__ void store_zero(float* p) { *reinterpret_cast<float2*>(p) = make_float2(0.f, 0.f); }
};
template <>
struct Vec<4> {
  static __device__ __forceinline__ void load(const float* p, float* v) {
    float4 t = *reinterpret_cast<const float4*>(p);
    v[0] = t.x, v[1] = t.y, v[2] = t.z, v[3] = t.w;
  }
  static __device__ __forceinline__ void load_bf16(const __nv_bfloat16* p, float* v) {
    uint2 t = *reinterpret_cast<const uint2*>(p);
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&t.x), b = *reinterpret_cast<__nv_bfloat162*>(&t.y);
    v[0] = __bfloat162float(a.x), v[1] = __bfloat162float(a.y), v[2] = __bfloat162float(b.x),
    v[3] = __bfloat162float(b.y);
  }
  static __device__ __forceinline__ void store_bf16(__nv_bfloat16* p, const float* v) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]), b = __floats2bfloat162_rn(v[2], v[3]);
    uint2 t;
    t.x = *reinterpret_cast<uint32_t*>(&a);
    t.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = t;
  }
  static __device__ __forceinline__ void store_zero(float* p) {
    *reinterpret_cast<float4*>(p) = make_float4(0.f, 0.f, 0.f, 0.f);
  }
};

// Merge of the partials of one q-tile: warp = (merge entry, head, row).  O and LSE hold the
// query rows [q0, q_end) (global token indices); LSE's row stride is q_end - q0.
template <int D>
__global__ void __launch_bounds__(kWarpsPerBlock * 32, 8)  // 8 resident blocks: more rows' loads in flight
    merge_kernel(const int32_t* merges, int64_t n_merges, int32_t hq, int64_t q0, int64_t q_end,
                 const float* o_part, const float* lse_part, __nv_bfloat16* o, float* lse) {
  constexpr int E = D / 32;
  const int64_t wid = (int64_t)blockIdx.x * kWarpsPerBlock + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (wid >= n_merges * hq * 128) return;
  const int64_t mi = wid / (hq * 128);
  const int h = (int)((wid / 128) % hq), r = (int)(wid % 128);
  const int qt = merges[3 * mi], s0 = merges[3 * mi + 1], ns = merges[3 * mi + 2];
  const int64_t gi = (int64_t)qt * 128 + r;
  if (gi >= q_end) return;
  const int64_t i = gi - q0, n = q_end - q0;  // row in the window, window rows
  float mx = -INFINITY;
  for (int b = 0; b < ns; ++b) mx = fmaxf(mx, lse_part[((size_t)(s0 + b) * hq + h) * 128 + r]);
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  float lse_all = -INFINITY;
  if (mx != -INFINITY) {
    float sum = 0.f;
    for (int b = 0; b < ns; ++b) sum += __expf(lse_part[((size_t)(s0 + b) * hq + h) * 128 + r] - mx);
    lse_all = mx + __logf(sum);
    // two partials' rows are loaded before they are accumulated (in order): with eight resident
    // blocks (32 registers) more warps' loads are in flight than four rows per round would allow
    for (int b0 = 0; b0 < ns; b0 += 2) {
      float v[2][E], wgt[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (b0 + u < ns) {
          const size_t row = ((size_t)(s0 + b0 + u) * hq + h) * 128 + r;
          wgt[u] = lse_part[row];
          Vec<E>::load(o_part + row * D + lane * E, v[u]);
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (b0 + u < ns) {
          const float w = __expf(wgt[u] - lse_all);
#pragma unroll
          for (int e = 0; e < E; ++e) acc[e] = fmaf(w, v[u][e], acc[e]);
        }
      }
    }
  }
  Vec<E>::store_bf16(o + ((size_t)i * hq + h) * D + lane * E, acc);
  if (lane == 0) lse[(size_t)h * n + i] = lse_all;
}

// D_i = <dO_i, O_i>, LSE_i * log2(e), and zeroed accumulator rows (dQ for every head of the n_pad
// query rows, dK and dV for the kv heads of the n_pad_kv key/value rows): warp = (row, head), over
// max(n_pad, n_pad_kv) rows.
template <int D>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    bwd_pre_kernel(const __nv_bfloat16* o, const __nv_bfloat16* dout, const float* lse, int64_t n, int64_t n_pad,
                   int64_t n_pad_kv, int32_t hq, int32_t hkv, float* dvec, float* lse2, float* dq_acc,
                   float* dkv_acc, const int32_t* kv_direct, int* work_next) {
  constexpr int E = D / 32;
  const int64_t wid = (int64_t)blockIdx.x * kWarpsPerBlock + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (wid == 0 && lane == 0) *work_next = 0;
  const int64_t i = wid / hq;
  const int h = (int)(wid % hq);
  if (i < n_pad_kv && h < hkv && !kv_direct[i >> 7]) {  // tiles stored directly need no accumulator
    const size_t kv_row = ((size_t)i * hkv + h) * D + lane * E;
    Vec<E>::store_zero(dkv_acc + kv_row);
    Vec<E>::store_zero(dkv_acc + (size_t)n_pad_kv * hkv * D + kv_row);
  }
  if (i >= n_pad) return;
  Vec<E>::store_zero(dq_acc + (size_t)wid * D + lane * E);
  float dsum = 0.f;
  if (i < n) {
    float a[E], b[E];
    Vec<E>::load_bf16(o + (size_t)wid * D + lane * E, a);
    Vec<E>::load_bf16(dout + (size_t)wid * D + lane * E, b);
#pragma unroll
    for (int e = 0; e < E; ++e) dsum = fmaf(a[e], b[e], dsum);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, off);
  }
  if (lane == 0) {
    dvec[(size_t)h * n_pad + i] = dsum;
    lse2[(size_t)h * n_pad + i] = i < n ? lse[(size_t)h * n + i] * 1.4426950408889634f : INFINITY;
  }
}

// fp32 accumulator -> bf16, four values per thread (dQ).
__global__ void bwd_post_q_kernel(const float* dq_acc, __nv_bfloat16* dq, int64_t q4) {
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= q4) return;
  float v[4];
  Vec<4>::load(dq_acc + 4 * t, v);
  Vec<4>::store_bf16(dq + 4 * t, v);
}

// fp32 dK (blockIdx.z = 0) / dV (1) accumulators -> bf16 on the 128-row kv tiles listed in
// acc_tiles (blockIdx.y = list position; the other tiles were stored directly by the backward
// kernel), four values per thread; tile4 = 4-value groups per tile, values past kv_count skipped.
__global__ void bwd_post_kv_kernel(const float* dkv_acc, __nv_bfloat16* dk, __nv_bfloat16* dv, int64_t dv_offset,
                                   const int32_t* acc_tiles, int32_t tile4, int64_t kv_count) {
  const int32_t t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= tile4) return;
  const int64_t e = (int64_t)acc_tiles[blockIdx.y] * (4 * (int64_t)tile4) + 4 * (int64_t)t;
  if (e >= kv_count) return;
  const bool is_v = blockIdx.z != 0;
  float v[4];
  Vec<4>::load(dkv_acc + (is_v ? dv_offset : 0) + e, v);
  Vec<4>::store_bf16((is_v ? dv : dk) + e, v);
}

// Received fp32 dK/dV partials added into rows of the fp32 accumulators, and those rows
// rewritten as bf16: four values per thread, dK then dV.
__global__ void kv_add_kernel(float* dkv_acc, int64_t dv_offset, const float* dk_part, const float* dv_part,
                              int64_t base, int64_t count4, __nv_bfloat16* dk, __nv_bfloat16* dv) {
  int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  float* acc;
  const float* part;
  __nv_bfloat16* dst;
  if (t < count4) {
    acc = dkv_acc + base + 4 * t, part = dk_part + 4 * t, dst = dk + base + 4 * t;
  } else if ((t -= count4) < count4) {
    acc = dkv_acc + dv_offset + base + 4 * t, part = dv_part + 4 * t, dst = dv + base + 4 * t;
  } else {
    return;
  }
  float a[4], b[4];
  Vec<4>::load(acc, a);
  Vec<4>::load(part, b);
#pragma unroll
  for (int e = 0; e < 4; ++e) a[e] += b[e];
  *reinterpret_cast<float4*>(acc) = make_float4(a[0], a[1], a[2], a[3]);
  Vec<4>::store_bf16(dst, a);
}

}  // namespace

template <int D>
cudaError_t launch_merge(const int32_t* merges, int64_t n_merges, int32_t hq, int64_t q0, int64_t q_end,
                         const float* o_part, const float* lse_part, __nv_bfloat16* o, float* lse,
                         cudaStream_t stream) {
  const int64_t warps = n_merges * hq * 128;
  if (warps == 0) return cudaSuccess;
  const int64_t blocks = (warps + kWarpsPerBlock - 1) / kWarpsPerBlock;
  merge_kernel<D><<<(unsigned)blocks, kWarpsPerBlock * 32, 0, stream>>>(merges, n_merges, hq, q0, q_end, o_part,
                                                                        lse_part, o, lse);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_bwd_pre(const __nv_bfloat16* o, const __nv_bfloat16* dout, const float* lse, int64_t n,
                           int64_t n_pad, int64_t n_pad_kv, int32_t hq, int32_t hkv, float* dvec, float* lse2,
                           float* dq_acc, float* dkv_acc, const int32_t* kv_direct, int* work_next,
                           cudaStream_t stream) {
  const int64_t warps = (n_pad > n_pad_kv ? n_pad : n_pad_kv) * hq;
  if (warps == 0) return cudaSuccess;
  const int64_t blocks = (warps + kWarpsPerBlock - 1) / kWarpsPerBlock;
  bwd_pre_kernel<D><<<(unsigned)blocks, kWarpsPerBlock * 32, 0, stream>>>(o, dout, lse, n, n_pad, n_pad_kv, hq, hkv,
                                                                          dvec, lse2, dq_acc, dkv_acc, kv_direct,
                                                                          work_next);
  return cudaGetLastError();
}

cudaError_t launch_kv_add(float* dkv_acc, int64_t dv_offset, const float* dk_part, const float* dv_part,
                          int64_t row0, int64_t rows, int64_t row_elems, __nv_bfloat16* dk, __nv_bfloat16* dv,
                          cudaStream_t stream) {
  const int64_t count4 = rows * row_elems / 4;
  if (count4 == 0) return cudaSuccess;
  kv_add_kernel<<<(unsigned)((2 * count4 + 255) / 256), 256, 0, stream>>>(dkv_acc, dv_offset, dk_part, dv_part,
                                                                          row0 * row_elems, count4, dk, dv);
  return cudaGetLastError();
}

cudaError_t launch_bwd_post(const float* dq_acc, __nv_bfloat16* dq, int64_t count_q, const float* dkv_acc,
                            __nv_bfloat16* dk, __nv_bfloat16* dv, int64_t count_kv, int64_t dv_offset,
                            const int32_t* acc_tiles, int64_t n_acc_tiles, int64_t row_elems, cudaStream_t stream) {
  const int64_t q4 = count_q / 4;
  if (q4 > 0) {
    bwd_post_q_kernel<<<(unsigned)((q4 + 255) / 256), 256, 0, stream>>>(dq_acc, dq, q4);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const int32_t tile4 = (int32_t)(128 * row_elems / 4);
  // grid.y is limited to 65535 tiles per launch: larger lists go in several launches
  for (int64_t first = 0; first < n_acc_tiles; first += 65535) {
    const int64_t nt = n_acc_tiles - first < 65535 ? n_acc_tiles - first : 65535;
    dim3 grid((unsigned)((tile4 + 255) / 256), (unsigned)nt, 2);
    bwd_post_kv_kernel<<<grid, 256, 0, stream>>>(dkv_acc, dk, dv, dv_offset, acc_tiles + first, tile4, count_kv);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template cudaError_t launch_merge<64>(const int32_t*, int64_t, int32_t, int64_t, int64_t, const float*,
                                      const float*, __nv_bfloat16*, float*, cudaStream_t);
template cudaError_t launch_merge<128>(const int32_t*, int64_t, int32_t, int64_t, int64_t, const float*,
                                       const float*, __nv_bfloat16*, float*, cudaStream_t);
template cudaError_t launch_bwd_pre<64>(const __nv_bfloat16*, const __nv_bfloat16*, const float*, int64_t, int64_t,
                                        int64_t, int32_t, int32_t, float*, float*, float*, float*, const int32_t*,
                                        int*, cudaStream_t);
template cudaError_t launch_bwd_pre<128>(const __nv_bfloat16*, const __nv_bfloat16*, const float*, int64_t, int64_t,
                                         int64_t, int32_t, int32_t, float*, float*, float*, float*, const int32_t*,
                                         int*, cudaStream_t);

}  // namespace sap
