// Backward kernel: dK, dV (and dQ by fp32 reduction) for one kv tile and one
// kv head per work item, looping over the q heads of its GQA group and the
// q tiles that attend to the kv tile (the per-kv-tile lists of the planner).
// With the final, merged LSE every (q-tile, kv-tile) pair is normalised
// already, so the pairs of different chunks are independent and their
// gradients simply add.
//
// Persistent CTA, warp-specialised (320 threads), everything transposed so
// that a TMEM lane is a key/value row:
//   warp 0      TMA producer: K, V tile per work item; per iteration the Q and
//               dO tiles plus the 128 LSE*log2(e) and D values of the q tile.
//   warp 1      TMEM owner and tcgen05.mma issuer (one thread), per iteration
//                 S^T  = K Q^T        (M=128 kv, N=128 q, K=D)   -> TMEM S
//                 dP^T = V dO^T       (M=128 kv, N=128 q, K=D)   -> TMEM dP
//                 dV  += P^T dO       (M=128 kv, N=D, K=128 q)   -> TMEM dV
//                 dK  += dS^T Q       (M=128 kv, N=D, K=128 q)   -> TMEM dK
//                 dQ   = dS K         (M=128 q,  N=D, K=128 kv)  -> TMEM dQ
//               (dS^T is read as a K-major operand for dK and as an M-major
//               operand for dQ from the same shared tile).
//   warps 2..5  thread t owns kv row j = kt*128 + t: P^T_ji = exp2(S*c - LSE2_i)
//               on the pairs of its document with i >= j (all pairs for FULL
//               tiles), dS^T = P^T (dP^T - D_i) * scale; both go to 128-byte
//               swizzled shared tiles as bf16.
//   warps 6..9  drain dQ from TMEM into the fp32 accumulator with vector
//               reductions, and write dK, dV (bf16) at the end of a work item.
//
// TMEM columns: dK [0,D), dV [D,2D), S [2D,2D+128), dP [2D+128,2D+256),
// dQ at 384 for D = 64, aliased onto S for D = 128 (S is consumed before dQ
// is produced; the next S waits until dQ has been drained).
#include <cuda.h>
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace sap {

template <int D>
struct BwdCfg {
  static constexpr int NSQ = (D == 64) ? 2 : 1;  // Q/dO ring depth
  static constexpr int BOX = 128 * 128;
  static constexpr int TILE = D * 128 * 2;       // bytes of one 128-row bf16 tile of width D
  static constexpr int VEC = 128 * 4;            // 128 fp32 values
  static constexpr int STAGE = 2 * TILE + 2 * VEC;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_P = OFF_V + TILE;
  static constexpr int OFF_DS = OFF_P + 128 * 128 * 2;
  static constexpr int OFF_ST = OFF_DS + 128 * 128 * 2;  // stages: Q, dO, lse2, dvec
  static constexpr int OFF_BAR = OFF_ST + NSQ * STAGE;
  static constexpr int NBAR = 2 + 2 * NSQ + 10;
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;
  static constexpr int THREADS = 320;
  static constexpr uint32_t COL_DK = 0, COL_DV = D, COL_S = 2 * D, COL_DP = 2 * D + 128;
  static constexpr bool ALIAS_DQ = (D == 128);
  static constexpr uint32_t COL_DQ = ALIAS_DQ ? COL_S : 384;
};

template <int D>
__global__ void __launch_bounds__(320, 1)
    sap_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                   const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* kv_full = bars + 0;
  uint64_t* kv_empty = bars + 1;
  uint64_t* q_full = bars + 2;           // [NSQ]
  uint64_t* q_empty = q_full + C::NSQ;   // [NSQ]
  uint64_t* s_full = q_empty + C::NSQ;
  uint64_t* dp_full = s_full + 1;
  uint64_t* pds_ready = dp_full + 1;
  uint64_t* pds_free = pds_ready + 1;
  uint64_t* dq_full = pds_free + 1;
  uint64_t* dq_free = dq_full + 1;
  uint64_t* dkdv_full = dq_free + 1;
  uint64_t* dkdv_free = dkdv_full + 1;
  uint64_t* mma_drain = dkdv_free + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const Guard guard{abort_flag, p.err};

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int s = 0; s < C::NSQ; ++s) {
      mbar_init(q_full + s, 1);
      mbar_init(q_empty + s, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(pds_ready, 128);
    mbar_init(pds_free, 1);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 128);
    mbar_init(dkdv_full, 1);
    mbar_init(dkdv_free, 128);
    mbar_init(mma_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int total = p.n_kv_units * p.hkv;
  const int G = p.group;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmDO);
      uint32_t unit_iter = 0, q_iter = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
        const int u = w / p.hkv, g = w % p.hkv;
        const int kt = p.kv_units[3 * u], e0 = p.kv_units[3 * u + 1], ne = p.kv_units[3 * u + 2];
        if (!mbar_wait(kv_empty, (unit_iter & 1) ^ 1, guard, kErrTimeoutLoad)) break;
        mbar_arrive_expect_tx(kv_full, 2 * C::TILE);
        for (int b = 0; b < D / 64; ++b) {
          tma_load_3d(smem + C::OFF_K + b * C::BOX, &tmK, kv_full, 64 * b, g, kt * 128);
          tma_load_3d(smem + C::OFF_V + b * C::BOX, &tmV, kv_full, 64 * b, g, kt * 128);
        }
        for (int hh = 0; hh < G && ok; ++hh) {
          const int h = g * G + hh;
          for (int e = 0; e < ne; ++e) {
            const int qt = p.entries[2 * (e0 + e)];
            const int s = q_iter % C::NSQ;
            const uint32_t ph = (q_iter / C::NSQ) & 1;
            if (!mbar_wait(q_empty + s, ph ^ 1, guard, kErrTimeoutLoad)) { ok = false; break; }
            uint8_t* st = smem + C::OFF_ST + s * C::STAGE;
            mbar_arrive_expect_tx(q_full + s, C::STAGE);
            for (int b = 0; b < D / 64; ++b) {
              tma_load_3d(st + b * C::BOX, &tmQ, q_full + s, 64 * b, h, qt * 128);
              tma_load_3d(st + C::TILE + b * C::BOX, &tmDO, q_full + s, 64 * b, h, qt * 128);
            }
            bulk_load(st + 2 * C::TILE, p.lse2 + (size_t)h * p.n_pad + (size_t)qt * 128, C::VEC, q_full + s);
            bulk_load(st + 2 * C::TILE + C::VEC, p.dvec + (size_t)h * p.n_pad + (size_t)qt * 128, C::VEC,
                      q_full + s);
            ++q_iter;
          }
        }
        ++unit_iter;
      }
      if (unit_iter > 0) drain_wait(kv_full, (unit_iter - 1) & 1);
      for (uint32_t t = (q_iter > (uint32_t)C::NSQ ? q_iter - C::NSQ : 0); t < q_iter; ++t)
        drain_wait(q_full + t % C::NSQ, (t / C::NSQ) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ----------------------------------------------------------------- MMA
      constexpr uint32_t id_sq = idesc_bf16(128, 128, false, false);  // S^T, dP^T
      constexpr uint32_t id_kv = idesc_bf16(128, D, false, true);     // dV, dK
      constexpr uint32_t id_dq = idesc_bf16(128, D, true, true);      // dQ
      const uint32_t sK = smem_u32(smem + C::OFF_K), sV = smem_u32(smem + C::OFF_V);
      const uint32_t sP = smem_u32(smem + C::OFF_P), sDS = smem_u32(smem + C::OFF_DS);
      const uint32_t sST = smem_u32(smem + C::OFF_ST);
      uint32_t unit_iter = 0, it = 0;  // it: global iteration counter
      bool ok = true;
      for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
        const int u = w / p.hkv;
        const int ne = p.kv_units[3 * u + 2];
        const int n_it = ne * G;
        if (!mbar_wait(kv_full, unit_iter & 1, guard, kErrTimeoutMma)) break;
        for (int j = 0; j < n_it; ++j, ++it) {
          const int s = it % C::NSQ;
          const uint32_t ph = (it / C::NSQ) & 1;
          const uint32_t sQ = sST + s * C::STAGE, sDO = sQ + C::TILE;
          if (!mbar_wait(q_full + s, ph, guard, kErrTimeoutMma)) { ok = false; break; }
          // S^T may overwrite the dQ of the previous iteration when they share columns.
          if (C::ALIAS_DQ && it > 0 && !mbar_wait(dq_free, (it - 1) & 1, guard, kErrTimeoutMma)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t ko = (kk / 4) * C::BOX + (kk % 4) * 32;
            mma_bf16(tmem + C::COL_S, sdesc_sw128(sK + ko, 16, 1024), sdesc_sw128(sQ + ko, 16, 1024), id_sq,
                     kk > 0);
          }
          tc_commit(s_full);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t ko = (kk / 4) * C::BOX + (kk % 4) * 32;
            mma_bf16(tmem + C::COL_DP, sdesc_sw128(sV + ko, 16, 1024), sdesc_sw128(sDO + ko, 16, 1024), id_sq,
                     kk > 0);
          }
          tc_commit(dp_full);
          // P^T and dS^T of this iteration are in shared memory.
          if (!mbar_wait(pds_ready, it & 1, guard, kErrTimeoutMma)) { ok = false; break; }
          // dK/dV of the previous work item must have been read out before they restart.
          if (j == 0 && unit_iter > 0 && !mbar_wait(dkdv_free, (unit_iter - 1) & 1, guard, kErrTimeoutMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 128 / 16; ++kk) {  // dV += P^T dO
            const uint64_t a = sdesc_sw128(sP + (kk / 4) * C::BOX + (kk % 4) * 32, 16, 1024);
            const uint64_t b = sdesc_sw128(sDO + kk * 2048, C::BOX, 1024);
            mma_bf16(tmem + C::COL_DV, a, b, id_kv, (j > 0 || kk > 0) ? 1u : 0u);
          }
#pragma unroll
          for (int kk = 0; kk < 128 / 16; ++kk) {  // dK += dS^T Q
            const uint64_t a = sdesc_sw128(sDS + (kk / 4) * C::BOX + (kk % 4) * 32, 16, 1024);
            const uint64_t b = sdesc_sw128(sQ + kk * 2048, C::BOX, 1024);
            mma_bf16(tmem + C::COL_DK, a, b, id_kv, (j > 0 || kk > 0) ? 1u : 0u);
          }
          if (!C::ALIAS_DQ && it > 0 && !mbar_wait(dq_free, (it - 1) & 1, guard, kErrTimeoutMma)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 128 / 16; ++kk) {  // dQ = dS K
            const uint64_t a = sdesc_sw128(sDS + kk * 2048, C::BOX, 1024);
            const uint64_t b = sdesc_sw128(sK + kk * 2048, C::BOX, 1024);
            mma_bf16(tmem + C::COL_DQ, a, b, id_dq, kk > 0);
          }
          tc_commit(dq_full);
          tc_commit(pds_free);
          tc_commit(q_empty + s);
        }
        if (!ok) break;
        tc_commit(dkdv_full);
        tc_commit(kv_empty);
        ++unit_iter;
      }
      tc_commit(mma_drain);
      drain_wait(mma_drain, 0);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------- P^T and dS^T
    const int quad = warp & 3;
    const int t = quad * 32 + lane;  // kv row within the tile
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    uint8_t* sPt = smem + C::OFF_P;
    uint8_t* sDSt = smem + C::OFF_DS;
    const float sl2 = p.scale_log2, scale = p.scale;
    uint32_t it = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
      const int u = w / p.hkv;
      const int kt = p.kv_units[3 * u], e0 = p.kv_units[3 * u + 1], ne = p.kv_units[3 * u + 2];
      const int64_t jrow = (int64_t)kt * 128 + t;
      const bool real_row = jrow < p.n;
      const int j_lo = real_row ? (int)jrow : 1;              // queries i with j <= i <= last token of the doc
      const int j_hi = real_row ? p.tok_hi[jrow] : 0;
      for (int hh = 0; hh < G && ok; ++hh) {
        for (int e = 0; e < ne; ++e, ++it) {
          const int qt = p.entries[2 * (e0 + e)], tag = p.entries[2 * (e0 + e) + 1];
          const int s = it % C::NSQ;
          const uint32_t ph = (it / C::NSQ) & 1;
          const float* lse2 = reinterpret_cast<const float*>(smem + C::OFF_ST + s * C::STAGE + 2 * C::TILE);
          const float* dvec = lse2 + 128;
          if (!mbar_wait_warp(q_full + s, ph, guard, kErrTimeoutSoftmax)) { ok = false; break; }
          if (!mbar_wait_warp(s_full, it & 1, guard, kErrTimeoutSoftmax)) { ok = false; break; }
          if (!mbar_wait_warp(dp_full, it & 1, guard, kErrTimeoutSoftmax)) { ok = false; break; }
          if (it > 0 && !mbar_wait_warp(pds_free, (it - 1) & 1, guard, kErrTimeoutSoftmax)) { ok = false; break; }
          tc_fence_after();
          const int c_lo = j_lo - qt * 128, c_hi = j_hi - qt * 128;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            float sv[32], dpv[32];
            tmem_ld32(lane_base + C::COL_S + 32 * c, sv);
            tmem_ld32(lane_base + C::COL_DP + 32 * c, dpv);
            uint32_t pw[16], dw[16];
#pragma unroll
            for (int e2 = 0; e2 < 32; e2 += 2) {
              float pp[2], dd[2];
#pragma unroll
              for (int q = 0; q < 2; ++q) {
                const int col = 32 * c + e2 + q;
                const bool valid = (tag == 0) || (col >= c_lo && col <= c_hi);
                const float pr = valid ? ex2(fmaf(sv[e2 + q], sl2, -lse2[col])) : 0.f;
                pp[q] = pr;
                dd[q] = pr * (dpv[e2 + q] - dvec[col]) * scale;
              }
              pw[e2 / 2] = pack_bf16x2(pp[0], pp[1]);
              dw[e2 / 2] = pack_bf16x2(dd[0], dd[1]);
            }
            // columns 32c .. 32c+31 = 16-byte chunks 4c .. 4c+3 of the 128-column row
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              const int cc = 4 * c + q4;
              const uint32_t off = (cc / 8) * C::BOX + sw128_offset(t, cc % 8);
              st_shared_v4(smem_u32(sPt + off), pw[4 * q4], pw[4 * q4 + 1], pw[4 * q4 + 2], pw[4 * q4 + 3]);
              st_shared_v4(smem_u32(sDSt + off), dw[4 * q4], dw[4 * q4 + 1], dw[4 * q4 + 2], dw[4 * q4 + 3]);
            }
          }
          fence_async_smem();
          tc_fence_before();
          mbar_arrive(pds_ready);
        }
      }
    }
  } else {
    // ------------------------------------------------ dQ drain, dK/dV epilogue
    const int quad = warp & 3;
    const int t = quad * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    uint32_t it = 0, unit_iter = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
      const int u = w / p.hkv, g = w % p.hkv;
      const int kt = p.kv_units[3 * u], e0 = p.kv_units[3 * u + 1], ne = p.kv_units[3 * u + 2];
      for (int hh = 0; hh < G && ok; ++hh) {
        const int h = g * G + hh;
        for (int e = 0; e < ne; ++e, ++it) {
          const int qt = p.entries[2 * (e0 + e)];
          if (!mbar_wait_warp(dq_full, it & 1, guard, kErrTimeoutEpilogue)) { ok = false; break; }
          tc_fence_after();
          float* dst = p.dq_acc + (((size_t)qt * 128 + t) * p.hq + h) * D;
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            float v[32];
            tmem_ld32(lane_base + C::COL_DQ + 32 * c, v);
#pragma unroll
            for (int e4 = 0; e4 < 32; e4 += 4)
              atomicAdd(reinterpret_cast<float4*>(dst + 32 * c + e4), make_float4(v[e4], v[e4 + 1], v[e4 + 2], v[e4 + 3]));
          }
          tc_fence_before();
          mbar_arrive(dq_free);
        }
      }
      if (!ok) break;
      if (!mbar_wait_warp(dkdv_full, unit_iter & 1, guard, kErrTimeoutEpilogue)) break;
      tc_fence_after();
      const int64_t jrow = (int64_t)kt * 128 + t;
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        __nv_bfloat16* out = (which == 0 ? p.dk : p.dv) + ((size_t)jrow * p.hkv + g) * D;
        const uint32_t col = which == 0 ? C::COL_DK : C::COL_DV;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          float v[32];
          tmem_ld32(lane_base + col + 32 * c, v);
          if (jrow < p.n) {
#pragma unroll
            for (int e8 = 0; e8 < 32; e8 += 8) {
              uint4 pk;
              pk.x = pack_bf16x2(v[e8], v[e8 + 1]);
              pk.y = pack_bf16x2(v[e8 + 2], v[e8 + 3]);
              pk.z = pack_bf16x2(v[e8 + 4], v[e8 + 5]);
              pk.w = pack_bf16x2(v[e8 + 6], v[e8 + 7]);
              *reinterpret_cast<uint4*>(out + 32 * c + e8) = pk;
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(dkdv_free);
      ++unit_iter;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

template <int D>
cudaError_t launch_bwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tdo,
                       const BwdParams& p, int grid, cudaStream_t stream) {
  auto kern = sap_bwd_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, BwdCfg<D>::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<grid, BwdCfg<D>::THREADS, BwdCfg<D>::SMEM, stream>>>(tq, tk, tv, tdo, p);
  return cudaGetLastError();
}

template cudaError_t launch_bwd<64>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                    const BwdParams&, int, cudaStream_t);
template cudaError_t launch_bwd<128>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                     const BwdParams&, int, cudaStream_t);

}  // namespace sap
