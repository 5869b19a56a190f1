// Backward kernel: dK, dV (and dQ by fp32 reduction) for one backward unit and one
// kv head per work item.  A unit is the part of one kv tile's q-tile list (the
// planner's per-kv-tile lists) that falls in one band of 16 q tiles; the work
// item loops over those q tiles and the q heads of the kv head's GQA group.
// With the final, merged LSE every (q-tile, kv-tile) pair is normalised
// already, so the pairs of different chunks (and of different bands) are
// independent and their gradients simply add.
//
// Persistent CTA, warp-specialised (448 threads), transposed so that a TMEM
// lane is a key/value row:
//   warp 0       work index of each item (dynamic: the next free item in
//                schedule order, shared with the other roles through a ring);
//                TMA producer: K, V per work item; per iteration Q, dO and the
//                128 LSE*log2(e) and D values of the q tile, through an
//                NSQ-stage ring.
//   warp 1       TMEM owner and tcgen05.mma issuer (one thread); S^T_j = K Q_j^T
//                (M=128 kv, N=128 q, K=D) -> R1 is issued one iteration ahead, then
//                per iteration j
//                  dV    += P^T_j dO_j  (A = P^T from TMEM R1)         -> dV
//                  dP^T_j = V dO_j^T  (M=128 kv, N=128 q, K=D)        -> R2
//                  S^T_{j+1}          (R1 is free once dV_j has read P^T_j)
//                  dQ_j               (D=128: dQ^T = K^T dS^T -> R2; D=64: dQ = dS K -> DQ)
//                  dK    += dS^T_j Q_j  (A = dS^T from shared memory) -> dK
//                At D = 128 dV goes first because P^T_j is ready long before the
//                previous dQ^T has left R2 (which dP^T_j needs); at D = 64 dP^T_j has
//                R2 to itself and is issued first, right after dK_{j-1}, so that it is
//                ready when the softmax has written P^T_j.  dQ goes before dK so that
//                its drain overlaps dK; the Q/dO ring slot is released once dK_j and
//                dQ_j have read it.
//   warps 2..9   two warpgroups, one per half of the 128 q columns; thread t
//                owns kv row j = kt*128 + t.  P^T = exp2(S^T c - LSE2_i) on the
//                pairs of its document with i >= j (all pairs for FULL tiles),
//                written back to TMEM as packed bf16 over its own S columns;
//                dS^T = P^T (dP^T - D_i) (the softmax scale is applied to dK and dQ
//                as they are drained) written to a 128-byte swizzled shared tile
//                as bf16 (read as a K-major operand by dK and as an MN-major
//                operand by dQ): for D = 128 over the ring slot's dO tile once dV_j
//                has read it, for D = 64 into a buffer of its own.
//   warps 10..13 drain dQ from TMEM into the fp32 accumulator by TMA bulk
//                reductions (D = 128: dQ^T staged 32 q rows at a time; D = 64: dQ
//                staged as two 128-byte-swizzled boxes of 32 features) through a
//                staging buffer of two 16 KB slots, so that two reductions are in
//                flight, and at the end of a work item add its dK and dV into fp32
//                accumulators the same way (the conversion to bf16 is a separate
//                elementwise kernel), or, when the kv tile has no other unit, store
//                them as bf16 directly.
//
// TMEM columns: dK [0,D), dV [D,2D), R1 = S^T/P^T [2D, 2D+128),
// R2 = dP^T [2D+128, 2D+256); dQ shares R2 for D = 128 (dP^T is consumed
// before dQ is produced, and the next dP^T waits for the drain) and has its
// own columns [384, 448) for D = 64.
#include <cuda.h>
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace sap {

// Each unit walks its q tiles starting at entry kt mod (entries), wrapping around, so that the units
// of one band that run at the same time reduce into different q tiles' dQ rows rather than all into
// the band's first tile.
__device__ __forceinline__ int entry_rotation(int kt, int ne) { return ne > 1 ? kt % ne : 0; }
__device__ __forceinline__ int rotated(int e, int rot, int ne) { return e + rot >= ne ? e + rot - ne : e + rot; }

template <int D>
struct BwdCfg {
  static constexpr int NSQ = (D == 64) ? 3 : 2;  // Q/dO ring depth
  static constexpr int BOX = 128 * 128;          // one 128-row x 64-column bf16 box
  static constexpr int TILE = D * 128 * 2;       // one 128-row bf16 tile of width D
  static constexpr int VEC = 128 * 4;            // 128 fp32 values
  static constexpr int STAGE = 2 * TILE + 2 * VEC;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE;
  // d = 64: dS^T (128 x 128 bf16).  d = 128: dS^T lives in the dO half of its iteration's stage and this
  // region is the staging buffer (two slots of 32 q rows x 128 fp32 of dQ, or of one dK/dV box).
  static constexpr int OFF_DS = OFF_V + TILE;
  static constexpr int OFF_ST = OFF_DS + 128 * 128 * 2;  // stages: Q, dO, lse2, dvec
  // dK/dV epilogue staging (128 rows x 64 fp32 as two 128-byte-swizzled boxes of 32 features):
  // d = 128 shares the dQ staging buffer; d = 64 has its own, which also stages dQ (d = 64 dQ is
  // [q][d] in TMEM, the same row-per-lane shape).  Same warps and barriers in both cases.
  static constexpr int EPI_BYTES = 128 * 64 * 4;
  // The staging buffer is used as two 16 KB slots at d = 128 (two TMA operations in flight) and as
  // one 32 KB slot at d = 64, where a dQ tile is two 16 KB boxes that leave together.
  static constexpr int NSLOT = (D == 128) ? 2 : 1;
  static constexpr int SLOT = EPI_BYTES / NSLOT;
  static constexpr int OFF_EPI = (D == 128) ? OFF_DS : OFF_ST + NSQ * STAGE;
  static constexpr int OFF_BAR = (D == 128) ? OFF_ST + NSQ * STAGE : OFF_EPI + EPI_BYTES;
  static constexpr int NW = 4;  // work-index ring depth
  static constexpr int NBAR = 2 + 2 * NSQ + 13 + 2 * NW;
  // The dynamic shared window starts 1024-byte aligned (checked at run time),
  // so no alignment slack is reserved: the D = 128 layout needs 231,672 bytes.
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 4 * NW;
  static_assert(SMEM <= 232448, "shared memory per block");
  static_assert(OFF_EPI % 1024 == 0 && OFF_ST % 1024 == 0 && STAGE % 1024 == 0, "128-byte swizzle alignment");
  static constexpr int THREADS = 448;
  static constexpr uint32_t COL_DK = 0, COL_DV = D, COL_R1 = 2 * D, COL_R2 = 2 * D + 128;
  static constexpr bool DQ_T = (D == 128);  // dQ^T in R2 (coalesced drain) vs dQ in its own columns
  static constexpr uint32_t COL_DQ = DQ_T ? COL_R2 : 384;
};

// 448 threads are granted registers as 16 warps, so 128 registers per thread is the ceiling
// (the compiler spills a few bytes at d = 128 and d = 64 to stay under it).
template <int D>
__global__ void __launch_bounds__(448, 1)
    sap_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                   const __grid_constant__ CUtensorMap tmDQ, const __grid_constant__ CUtensorMap tmDKV,
                   const __grid_constant__ CUtensorMap tmDK, const __grid_constant__ CUtensorMap tmDV,
                   const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {  // TMA 128-byte swizzle and the descriptors need 1024-byte alignment
    if (threadIdx.x == 0) atomicOr(p.err, kErrSmemAlign);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* kv_full = bars + 0;
  uint64_t* kv_empty = bars + 1;
  uint64_t* q_full = bars + 2;          // [NSQ]
  uint64_t* q_empty = q_full + C::NSQ;  // [NSQ]
  uint64_t* s_full = q_empty + C::NSQ;
  uint64_t* dp_full = s_full + 1;
  uint64_t* p_ready = dp_full + 1;
  uint64_t* ds_ready = p_ready + 1;
  uint64_t* dq_full = ds_ready + 1;
  uint64_t* dq_free = dq_full + 1;
  uint64_t* dkdv_full = dq_free + 1;
  uint64_t* dkdv_free = dkdv_full + 1;
  uint64_t* mma_drain = dkdv_free + 1;
  uint64_t* stg_ready = mma_drain + 1;  // [2] a staging slot holds a dQ or dK/dV box
  uint64_t* stg_free = stg_ready + 2;   // [2] the slot's TMA operation has read it
  uint64_t* sched_full = stg_free + 2;  // [NW] the producer wrote the next work index
  uint64_t* sched_empty = sched_full + C::NW;  // [NW] every other role has read it
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* sched_w = reinterpret_cast<volatile int*>(smem + C::OFF_BAR + C::NBAR * 8 + 16);  // [NW]

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const Guard guard{abort_flag, p.err, p.wait_ns};

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int s = 0; s < C::NSQ; ++s) {
      mbar_init(q_full + s, 1);
      mbar_init(q_empty + s, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_ready, 8);    // one arrival per softmax warp
    mbar_init(ds_ready, 8);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 4);    // one arrival per drain warp
    mbar_init(dkdv_full, 1);
    mbar_init(dkdv_free, 4);
    mbar_init(mma_drain, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(stg_ready + s, 4);  // one arrival per drain warp
      mbar_init(stg_free + s, 1);
    }
    for (int s = 0; s < C::NW; ++s) {
      mbar_init(sched_full + s, 1);
      mbar_init(sched_empty + s, 1 + 8 + 4);  // the MMA thread, the 8 softmax and 4 drain warps
    }
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
  // Work items are handed out dynamically in schedule order: the first one of a CTA is blockIdx.x,
  // the next ones come from a global counter, so a CTA that finishes early takes the next item
  // (list scheduling of the heavy-first order).  The producer fetches each index and publishes it
  // through a ring of NW slots; every other role reads the indices in the same order.  -1 ends the
  // sequence; -2 marks a wait that ran out.
  auto take_work = [&](uint32_t i, int code) -> int {  // warp-wide (softmax and drain warps)
    const int s = i % C::NW;
    if (!mbar_wait_warp(sched_full + s, (i / C::NW) & 1, guard, code)) return -2;
    const int w = sched_w[s];
    __syncwarp();
    if (lane == 0) mbar_arrive(sched_empty + s);
    return w;
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmDO);
      uint32_t unit_iter = 0, q_iter = 0;
      bool ok = true;
      for (uint32_t wi = 0; ok; ++wi) {
        const int ws = wi % C::NW;
        if (!mbar_wait(sched_empty + ws, ((wi / C::NW) & 1) ^ 1, guard, kErrTimeoutLoad)) break;
        int w = wi == 0 ? (int)blockIdx.x : (int)gridDim.x + atomicAdd(p.work_next, 1);
        if (w >= total) w = -1;
        sched_w[ws] = w;
        mbar_arrive(sched_full + ws);
        if (w < 0) break;
        const int u = w / p.hkv, g = w % p.hkv;
        const int kt = p.kv_units[3 * u], e0 = p.kv_units[3 * u + 1], ne = p.kv_units[3 * u + 2];
        if (!mbar_wait(kv_empty, (unit_iter & 1) ^ 1, guard, kErrTimeoutLoad)) break;
        mbar_arrive_expect_tx(kv_full, 2 * C::TILE);
        for (int b = 0; b < D / 64; ++b) {
          tma_load_3d(smem + C::OFF_K + b * C::BOX, &tmK, kv_full, 64 * b, g, kt * 128 - (int)p.kv0);
          tma_load_3d(smem + C::OFF_V + b * C::BOX, &tmV, kv_full, 64 * b, g, kt * 128 - (int)p.kv0);
        }
        // entries are walked q-tile outer, head inner; the next q tile is fetched one entry ahead
        const int rot = entry_rotation(kt, ne);
        int qt_next = p.entries[2 * (e0 + rot)];
        for (int e = 0; e < ne && ok; ++e) {
          const int qt = qt_next;
          const int qrow = qt * 128 - (int)p.q0;  // first row of the q tile in the query-side buffers
          if (e + 1 < ne) qt_next = p.entries[2 * (e0 + rotated(e + 1, rot, ne))];
          for (int hh = 0; hh < G; ++hh) {
            const int h = g * G + hh;
            const int s = q_iter % C::NSQ;
            const uint32_t ph = (q_iter / C::NSQ) & 1;
            if (!mbar_wait(q_empty + s, ph ^ 1, guard, kErrTimeoutLoad)) { ok = false; break; }
            uint8_t* st = smem + C::OFF_ST + s * C::STAGE;
            mbar_arrive_expect_tx(q_full + s, C::STAGE);
            for (int b = 0; b < D / 64; ++b) {
              tma_load_3d(st + b * C::BOX, &tmQ, q_full + s, 64 * b, h, qrow);
              tma_load_3d(st + C::TILE + b * C::BOX, &tmDO, q_full + s, 64 * b, h, qrow);
            }
            bulk_load(st + 2 * C::TILE, p.lse2 + (size_t)h * p.n_pad + (size_t)qrow, C::VEC, q_full + s);
            bulk_load(st + 2 * C::TILE + C::VEC, p.dvec + (size_t)h * p.n_pad + (size_t)qrow, C::VEC,
                      q_full + s);
            ++q_iter;
          }
        }
        ++unit_iter;
      }
      if (unit_iter > 0) drain_wait(kv_full, (unit_iter - 1) & 1, p.wait_ns);
      for (uint32_t t = (q_iter > (uint32_t)C::NSQ ? q_iter - C::NSQ : 0); t < q_iter; ++t)
        drain_wait(q_full + t % C::NSQ, (t / C::NSQ) & 1, p.wait_ns);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ----------------------------------------------------------------- MMA
      constexpr uint32_t id_sq = idesc_bf16(128, 128, false, false);  // S^T, dP^T
      constexpr uint32_t id_kv = idesc_bf16(128, D, false, true);     // dV (A in TMEM), dK
      constexpr uint32_t id_dq = C::DQ_T ? idesc_bf16(128, 128, true, true) : idesc_bf16(128, D, true, true);
      const uint32_t sK = smem_u32(smem + C::OFF_K), sV = smem_u32(smem + C::OFF_V);
      const uint32_t sDS = smem_u32(smem + C::OFF_DS);
      const uint32_t sST = smem_u32(smem + C::OFF_ST);
      const uint32_t R1 = tmem + C::COL_R1, R2 = tmem + C::COL_R2;
      // Shared-memory descriptors, computed once per operand base; per k-slice only an offset is
      // added (K-major: 16-byte leading offset; MN-major: one box apart).
      const uint64_t dK_k = sdesc_sw128(sK, 16, 1024), dV_k = sdesc_sw128(sV, 16, 1024);
      const uint64_t dK_mn = sdesc_sw128(sK, C::BOX, 1024);
      uint32_t unit_iter = 0, it = 0;  // it: global iteration counter (all barriers below count per iteration)
      bool ok = true;
      auto stage_q = [&](uint32_t i) { return sST + (i % C::NSQ) * C::STAGE; };
      auto issue_s = [&](uint32_t i) -> bool {  // S^T_i = K Q_i^T -> R1
        if (!mbar_wait(q_full + i % C::NSQ, (i / C::NSQ) & 1, guard, kErrTimeoutMma)) return false;
        tc_fence_after();
        const uint64_t dQ_k = sdesc_sw128(stage_q(i), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ko = (kk / 4) * C::BOX + (kk % 4) * 32;
          mma_bf16(R1, sdesc_off(dK_k, ko), sdesc_off(dQ_k, ko), id_sq, kk > 0);
        }
        tc_commit(s_full);
        return true;
      };
      for (uint32_t wi = 0; ok; ++wi) {
        const int ws = wi % C::NW;
        if (!mbar_wait(sched_full + ws, (wi / C::NW) & 1, guard, kErrTimeoutMma)) break;
        const int w = sched_w[ws];
        mbar_arrive(sched_empty + ws);
        if (w < 0) break;
        const int u = w / p.hkv;
        const int n_it = p.kv_units[3 * u + 2] * G;
        if (!mbar_wait(kv_full, unit_iter & 1, guard, kErrTimeoutMma)) break;
        tc_fence_after();
        if (!issue_s(it)) break;
        for (int j = 0; j < n_it; ++j, ++it) {
          const uint32_t sQ = stage_q(it), sDO = sQ + C::TILE;
          const uint64_t dQ_mn = sdesc_sw128(sQ, C::BOX, 1024);
          const uint64_t dDO_k = sdesc_sw128(sDO, 16, 1024), dDO_mn = sdesc_sw128(sDO, C::BOX, 1024);
          auto issue_dp = [&]() {  // dP^T_j = V dO_j^T -> R2
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t ko = (kk / 4) * C::BOX + (kk % 4) * 32;
              mma_bf16(R2, sdesc_off(dV_k, ko), sdesc_off(dDO_k, ko), id_sq, kk > 0);
            }
            tc_commit(dp_full);
          };
          // D = 64: dP^T_j needs only V and dO_j, and R2 is free once the softmax has read dP^T_{j-1}
          // (before it signalled dS^T_{j-1}), so it is issued before P^T_j is waited for and is ready
          // when the softmax has written P^T_j.
          if (!C::DQ_T) issue_dp();
          // dV += P^T_j dO_j (P^T in TMEM, packed bf16 over the S^T columns of each half); at D = 128
          // it goes first because P^T_j is usually ready well before the previous dQ has been drained.
          if (!mbar_wait(p_ready, it & 1, guard, kErrTimeoutMma)) { ok = false; break; }
          if (j == 0 && unit_iter > 0 && !mbar_wait(dkdv_free, (unit_iter - 1) & 1, guard, kErrTimeoutMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 128 / 16; ++kk)
            mma_bf16_tmem_a(tmem + C::COL_DV, R1 + (kk / 4) * 64 + (kk % 4) * 8,
                            sdesc_off(dDO_mn, kk * 2048), id_kv, (j > 0 || kk > 0) ? 1u : 0u);
          // D = 128: dP^T_j -> R2 once the previous dQ^T (same columns) has been drained
          if (C::DQ_T) {
            if (it > 0 && !mbar_wait(dq_free, (it - 1) & 1, guard, kErrTimeoutMma)) { ok = false; break; }
            tc_fence_after();
            issue_dp();
          }
          const uint32_t sDSj = C::DQ_T ? sDO : sDS;  // d = 128: dS^T_j over dO_j
          const uint64_t dDS_k = sdesc_sw128(sDSj, 16, 1024), dDS_mn = sdesc_sw128(sDSj, C::BOX, 1024);
          // S^T_{j+1}: R1 is rewritten only after dV_j (issued above) has read P^T_j
          if (j + 1 < n_it && !issue_s(it + 1)) { ok = false; break; }
          // dQ_j and dK += dS^T_j Q_j
          if (!mbar_wait(ds_ready, it & 1, guard, kErrTimeoutMma)) { ok = false; break; }
          tc_fence_after();
          if (!C::DQ_T && it > 0 && !mbar_wait(dq_free, (it - 1) & 1, guard, kErrTimeoutMma)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 128 / 16; ++kk) {
            // D=128: dQ^T[d][q] = sum_kv K[kv][d] dS^T[kv][q]  (A = K, B = dS^T, both MN-major)
            // D=64 : dQ[q][d]   = sum_kv dS^T[kv][q] K[kv][d]  (A = dS^T, B = K, both MN-major)
            const uint64_t kd = sdesc_off(dK_mn, kk * 2048);
            const uint64_t sd = sdesc_off(dDS_mn, kk * 2048);
            mma_bf16(tmem + C::COL_DQ, C::DQ_T ? kd : sd, C::DQ_T ? sd : kd, id_dq, kk > 0);
          }
          tc_commit(dq_full);
#pragma unroll
          for (int kk = 0; kk < 128 / 16; ++kk) {
            const uint64_t a = sdesc_off(dDS_k, (kk / 4) * C::BOX + (kk % 4) * 32);
            mma_bf16(tmem + C::COL_DK, a, sdesc_off(dQ_mn, kk * 2048), id_kv,
                     (j > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(q_empty + it % C::NSQ);
        }
        if (!ok) break;
        tc_commit(dkdv_full);
        tc_commit(kv_empty);
        ++unit_iter;
      }
      tc_commit(mma_drain);
      drain_wait(mma_drain, 0, p.wait_ns);
    }
  } else if (warp < 10) {
    // ----------------------------------------------------- P^T and dS^T
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;  // q columns [64*half, 64*half + 64)
    const int t = quad * 32 + lane;    // kv row within the tile
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    const uint32_t R1 = lane_base + C::COL_R1 + 64 * half, R2 = lane_base + C::COL_R2 + 64 * half;
    const float sl2 = p.scale_log2;
    uint32_t it = 0;
    bool ok = true;
    for (uint32_t wi = 0; ok; ++wi) {
      const int w = take_work(wi, kErrTimeoutSoftmax);
      if (w < 0) {
        ok = w == -1;
        break;
      }
      const int u = w / p.hkv;
      const int kt = p.kv_units[3 * u], e0 = p.kv_units[3 * u + 1], ne = p.kv_units[3 * u + 2];
      const int64_t jrow = (int64_t)kt * 128 + t;
      const bool real_row = jrow < p.q_end;
      const int j_lo = real_row ? (int)jrow : 1;  // queries i with j <= i <= last token of the document
      const int j_hi = real_row ? p.tok_hi[jrow] : 0;
      const int rot = entry_rotation(kt, ne);
      int qt_next = p.entries[2 * (e0 + rot)], tag_next = p.entries[2 * (e0 + rot) + 1];
      for (int e = 0; e < ne && ok; ++e) {
        const int qt = qt_next, tag = tag_next;
        if (e + 1 < ne) {
          const int en = e0 + rotated(e + 1, rot, ne);
          qt_next = p.entries[2 * en], tag_next = p.entries[2 * en + 1];
        }
        for (int hh = 0; hh < G; ++hh, ++it) {
          const float* lse2 =
              reinterpret_cast<const float*>(smem + C::OFF_ST + (it % C::NSQ) * C::STAGE + 2 * C::TILE) + 64 * half;
          const float* dvec = lse2 + 128;
          const int c_lo = j_lo - qt * 128 - 64 * half, c_hi = j_hi - qt * 128 - 64 * half;
          // S^T_j is issued only after the MMA thread has seen the stage's loads (Q, dO, LSE, D) land,
          // so its completion also means that this stage's vectors are in shared memory.
          if (!mbar_wait_warp(s_full, it & 1, guard, kErrTimeoutSoftmax)) { ok = false; break; }
          tc_fence_after();
          float pr[64];
          {
            const float4* l4 = reinterpret_cast<const float4*>(lse2);
            float sv[32];
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              tmem_ld32(R1 + 32 * c, sv);
              if (tag == 0) {  // FULL tile: no pair is masked
#pragma unroll
                for (int e4 = 0; e4 < 32; e4 += 4) {
                  const float4 l = l4[(32 * c + e4) / 4];
                  pr[32 * c + e4] = ex2(fmaf(sv[e4], sl2, -l.x));
                  pr[32 * c + e4 + 1] = ex2(fmaf(sv[e4 + 1], sl2, -l.y));
                  pr[32 * c + e4 + 2] = ex2(fmaf(sv[e4 + 2], sl2, -l.z));
                  pr[32 * c + e4 + 3] = ex2(fmaf(sv[e4 + 3], sl2, -l.w));
                }
              } else {
#pragma unroll
                for (int e2 = 0; e2 < 32; ++e2) {
                  const int col = 32 * c + e2;
                  const bool valid = col >= c_lo && col <= c_hi;
                  pr[col] = valid ? ex2(fmaf(sv[e2], sl2, -lse2[col])) : 0.f;
                }
              }
            }
            uint32_t pk[32];
#pragma unroll
            for (int e2 = 0; e2 < 32; ++e2) pk[e2] = pack_bf16x2(pr[2 * e2], pr[2 * e2 + 1]);
            tmem_st32_u(R1, pk);  // P^T over this half's first 32 S^T columns (already read)
          }
          tc_fence_before();
          mbar_arrive_warp(p_ready);
          // dp_full tracks every MMA the MMA thread issued before dP^T_j: dV_j (d = 128: dS^T_j goes
          // over dO_j, which dV_j was the last to read) and the previous iteration's dQ and dK (d = 64:
          // the dS^T buffer they read is free again).
          if (!mbar_wait_warp(dp_full, it & 1, guard, kErrTimeoutSoftmax)) { ok = false; break; }
          tc_fence_after();
          uint8_t* sDSt = (C::DQ_T ? smem + C::OFF_ST + (it % C::NSQ) * C::STAGE + C::TILE : smem + C::OFF_DS) +
                          half * C::BOX;
          const float4* d4 = reinterpret_cast<const float4*>(dvec);
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            float dpv[32];
            tmem_ld32(R2 + 32 * c, dpv);
            uint32_t dw[16];
            // dS^T without the softmax scale; the scale is applied to dK and dQ when they are drained
#pragma unroll
            for (int e4 = 0; e4 < 32; e4 += 4) {
              const int col = 32 * c + e4;
              const float4 dd = d4[col / 4];
              dw[e4 / 2] = pack_bf16x2(pr[col] * (dpv[e4] - dd.x), pr[col + 1] * (dpv[e4 + 1] - dd.y));
              dw[e4 / 2 + 1] = pack_bf16x2(pr[col + 2] * (dpv[e4 + 2] - dd.z), pr[col + 3] * (dpv[e4 + 3] - dd.w));
            }
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {  // 16-byte chunks 4c .. 4c+3 of this half's 64 columns
              const uint32_t off = sw128_offset(t, 4 * c + q4);
              st_shared_v4(smem_u32(sDSt + off), dw[4 * q4], dw[4 * q4 + 1], dw[4 * q4 + 2], dw[4 * q4 + 3]);
            }
          }
          fence_async_smem();
          tc_fence_before();
          mbar_arrive_warp(ds_ready);
        }
      }
    }
  } else {
    // ------------------------------------------------ dQ drain, dK/dV epilogue
    const int quad = warp & 3;
    const int t = quad * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    // Staging: each use of a slot stages one piece and thread 0 issues its TMA operations.  With two
    // 16 KB slots (d = 128: a quarter of a dQ^T tile, one [128 rows][32 fp32] box of dK/dV, or one
    // bf16 [128 rows][64] box of a directly stored dK/dV) the slots are used in turn and two
    // operations are in flight: after issuing use n, thread 0 waits only until use n - 1 has read
    // its slot and then frees that slot.  With one 32 KB slot (d = 64: a dQ tile or 64 dK/dV features
    // as two [128 rows][32 fp32] boxes) thread 0 waits until the use has read the slot.  stg_ready[s]
    // needs all four drain warps and stg_free[s] completes only after the use (two slots: the next
    // use) has been issued, so neither parity wait can skip a phase.
    uint32_t it = 0, unit_iter = 0, n_stg = 0;  // n_stg: uses of the staging slots
    uint8_t* const stg_base = smem + (C::DQ_T ? C::OFF_DS : C::OFF_EPI);
    auto stg_acquire = [&]() -> uint8_t* {  // warp-wide: the slot of use n_stg, once it is free
      const uint32_t s = C::NSLOT == 2 ? n_stg & 1 : 0;
      const uint32_t k = C::NSLOT == 2 ? n_stg >> 1 : n_stg;  // earlier uses of this slot
      if (k >= 1 && !mbar_wait_warp(stg_free + s, (k - 1) & 1, guard, kErrTimeoutEpilogue)) return nullptr;
      return stg_base + s * C::SLOT;
    };
    auto stg_ready_sync = [&]() -> bool {  // warp-wide, after this warp has written its rows
      const uint32_t s = C::NSLOT == 2 ? n_stg & 1 : 0;
      fence_async_smem();
      mbar_arrive_warp(stg_ready + s);
      return mbar_wait_warp(stg_ready + s, (C::NSLOT == 2 ? n_stg >> 1 : n_stg) & 1, guard, kErrTimeoutEpilogue);
    };
    auto stg_done = [&]() {  // warp-wide, after thread 0 has issued the use's TMA operations
      if (t == 0) {
        bulk_commit_group();
        if (C::NSLOT == 1) {
          bulk_wait_group_read0();
          mbar_arrive(stg_free);
        } else if (n_stg >= 1) {
          bulk_wait_group_read1();
          mbar_arrive(stg_free + ((n_stg & 1) ^ 1));
        }
      }
      __syncwarp();  // the warp is converged again before its next warp-collective TMEM load
      ++n_stg;
    };
    bool ok = true;
    for (uint32_t wi = 0; ok; ++wi) {
      const int w = take_work(wi, kErrTimeoutEpilogue);
      if (w < 0) {
        ok = w == -1;
        break;
      }
      const int u = w / p.hkv, g = w % p.hkv;
      const int kt = p.kv_units[3 * u], e0 = p.kv_units[3 * u + 1], ne = p.kv_units[3 * u + 2];
      const int rot = entry_rotation(kt, ne);
      int qt_next = p.entries[2 * (e0 + rot)];
      for (int e = 0; e < ne && ok; ++e) {
        const int qt = qt_next;
        if (e + 1 < ne) qt_next = p.entries[2 * (e0 + rotated(e + 1, rot, ne))];
        const int qrow = qt * 128 - (int)p.q0;  // first row of the q tile in the query-side buffers
        for (int hh = 0; hh < G; ++hh, ++it) {
          const int h = g * G + hh;
          if (!mbar_wait_warp(dq_full, it & 1, guard, kErrTimeoutEpilogue)) { ok = false; break; }
          tc_fence_after();
          if (C::DQ_T) {
            // Lane t holds feature t of dQ^T (one column per q row).  Each quarter of the tile (32 q
            // rows) is staged row-major [q][d] in one slot and added to the accumulator by one TMA
            // bulk reduction.  The first two quarters go through the slots, the last two are held in
            // registers, so R2 is released once the first two are staged.
#pragma unroll 1
            for (int c = 0; c < 2 && ok; ++c) {
              float v[32];
              tmem_ld32(lane_base + C::COL_DQ + 32 * c, v);
              float* stg = reinterpret_cast<float*>(stg_acquire());
              if (!stg) { ok = false; break; }
#pragma unroll
              for (int e2 = 0; e2 < 32; ++e2) stg[e2 * 128 + t] = v[e2] * p.scale;
              if (!stg_ready_sync()) { ok = false; break; }
              if (t == 0) tma_reduce_add_3d(&tmDQ, stg, 0, h, qrow + 32 * c);
              stg_done();
            }
            if (!ok) break;
            float v2[32], v3[32];
            tmem_ld32(lane_base + C::COL_DQ + 64, v2);
            tmem_ld32(lane_base + C::COL_DQ + 96, v3);
            tc_fence_before();
            mbar_arrive_warp(dq_free);  // all of dQ^T is in registers or staged: R2 may take the next dP^T
            float* stg = reinterpret_cast<float*>(stg_acquire());
            if (!stg) { ok = false; break; }
#pragma unroll
            for (int e2 = 0; e2 < 32; ++e2) stg[e2 * 128 + t] = v2[e2] * p.scale;
            if (!stg_ready_sync()) { ok = false; break; }
            if (t == 0) tma_reduce_add_3d(&tmDQ, stg, 0, h, qrow + 64);
            stg_done();
            stg = reinterpret_cast<float*>(stg_acquire());
            if (!stg) { ok = false; break; }
#pragma unroll
            for (int e2 = 0; e2 < 32; ++e2) stg[e2 * 128 + t] = v3[e2] * p.scale;
            if (!stg_ready_sync()) { ok = false; break; }
            if (t == 0) tma_reduce_add_3d(&tmDQ, stg, 0, h, qrow + 96);
            stg_done();
          } else {
            // Lane t holds q row t of dQ (D = 64 features).  The tile is staged, times the softmax
            // scale, as two 128-byte-swizzled boxes [128 rows][32 fp32] (the same layout as the
            // dK/dV epilogue) in the one slot and added by two TMA bulk reductions.
            static_assert(C::DQ_T || C::NSLOT == 1, "d = 64 stages a dQ tile in one 32 KB slot");
            uint8_t* b = stg_acquire();
            if (!b) { ok = false; break; }
            float v0[32], v1[32];
            tmem_ld32(lane_base + C::COL_DQ, v0);
            tmem_ld32(lane_base + C::COL_DQ + 32, v1);
            tc_fence_before();
            mbar_arrive_warp(dq_free);  // all of dQ is in registers: the next dQ may overwrite its columns
#pragma unroll
            for (int c16 = 0; c16 < 8; ++c16) {
              const uint32_t off = sw128_offset(t, c16);
              st_shared_v4(smem_u32(b + off), __float_as_uint(v0[4 * c16] * p.scale),
                           __float_as_uint(v0[4 * c16 + 1] * p.scale), __float_as_uint(v0[4 * c16 + 2] * p.scale),
                           __float_as_uint(v0[4 * c16 + 3] * p.scale));
              st_shared_v4(smem_u32(b + C::EPI_BYTES / 2 + off), __float_as_uint(v1[4 * c16] * p.scale),
                           __float_as_uint(v1[4 * c16 + 1] * p.scale), __float_as_uint(v1[4 * c16 + 2] * p.scale),
                           __float_as_uint(v1[4 * c16 + 3] * p.scale));
            }
            if (!stg_ready_sync()) { ok = false; break; }
            if (t == 0) {
              tma_reduce_add_3d(&tmDQ, b, 0, h, qrow);
              tma_reduce_add_3d(&tmDQ, b + C::EPI_BYTES / 2, 32, h, qrow);
            }
            stg_done();
          }
        }
      }
      if (!ok) break;
      if (!mbar_wait_warp(dkdv_full, unit_iter & 1, guard, kErrTimeoutEpilogue)) break;
      tc_fence_after();
      // This unit's dK (times the softmax scale left out of dS) and dV leave TMEM 64 features at a
      // time: lane t holds row t and stages it, and thread 0 issues the TMA.  A kv tile with other
      // units adds its partial to the fp32 accumulators: two 128-byte-swizzled boxes [128 rows][32
      // fp32] reduced into them (rows past N hold zeros: their keys and values were loaded as zeros
      // and all their pairs are masked).  A kv tile with no other unit (direct) is final: one
      // 128-byte-swizzled box [128 rows][64 bf16] stored to the bf16 output.
      const bool direct = p.kv_direct[(kt * 128 - (int)p.kv0) >> 7] != 0;
      const int row = kt * 128 - (int)p.kv0;  // first row of the kv tile in the key/value-side buffers
      constexpr int NCH = 2 * (D / 64);
#pragma unroll 1
      for (int m = 0; m < NCH && ok; ++m) {
        const int which = m / (D / 64), cb = m % (D / 64);
        const uint32_t col = (which == 0 ? C::COL_DK : C::COL_DV) + 64 * cb;
        const float f = which == 0 ? p.scale : 1.f;
        float v0[32], v1[32];
        tmem_ld32(lane_base + col, v0);
        tmem_ld32(lane_base + col + 32, v1);
        if (m == NCH - 1) {  // all of dK/dV has been read: the next unit may accumulate over it
          tc_fence_before();
          mbar_arrive_warp(dkdv_free);
        }
        if (direct) {
          uint8_t* b = stg_acquire();
          if (!b) { ok = false; break; }
#pragma unroll
          for (int c16 = 0; c16 < 8; ++c16) {
            const float* v = c16 < 4 ? v0 + 8 * c16 : v1 + 8 * (c16 - 4);
            st_shared_v4(smem_u32(b + sw128_offset(t, c16)), pack_bf16x2(v[0] * f, v[1] * f),
                         pack_bf16x2(v[2] * f, v[3] * f), pack_bf16x2(v[4] * f, v[5] * f),
                         pack_bf16x2(v[6] * f, v[7] * f));
          }
          if (!stg_ready_sync()) { ok = false; break; }
          if (t == 0) tma_store_3d(which == 0 ? &tmDK : &tmDV, b, 64 * cb, g, row);
          stg_done();
        } else {
          const int row0 = (which == 0 ? 0 : (int)p.n_pad_kv) + row;
          // two slots: one box per use; one slot: both boxes in one use
          constexpr int PER_USE = C::NSLOT == 2 ? 1 : 2;
#pragma unroll 1
          for (int c = 0; c < 2 && ok; c += PER_USE) {
            uint8_t* b = stg_acquire();
            if (!b) { ok = false; break; }
#pragma unroll
            for (int k = 0; k < PER_USE; ++k) {
              const float* v = c + k == 0 ? v0 : v1;
#pragma unroll
              for (int c16 = 0; c16 < 8; ++c16)
                st_shared_v4(smem_u32(b + k * (C::EPI_BYTES / 2) + sw128_offset(t, c16)),
                             __float_as_uint(v[4 * c16] * f), __float_as_uint(v[4 * c16 + 1] * f),
                             __float_as_uint(v[4 * c16 + 2] * f), __float_as_uint(v[4 * c16 + 3] * f));
            }
            if (!stg_ready_sync()) { ok = false; break; }
            if (t == 0)
              for (int k = 0; k < PER_USE; ++k)
                tma_reduce_add_3d(&tmDKV, b + k * (C::EPI_BYTES / 2), 64 * cb + 32 * (c + k), g, row0);
            stg_done();
          }
        }
      }
      if (!ok) break;
      ++unit_iter;
    }
  }

  if (warp >= 10) bulk_wait_group0();  // the dQ reductions issued by this thread have completed
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
                       const CUtensorMap& tdq, const CUtensorMap& tdkv, const CUtensorMap& tdk,
                       const CUtensorMap& tdv, const BwdParams& p, int grid, cudaStream_t stream) {
  auto kern = sap_bwd_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, BwdCfg<D>::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<grid, BwdCfg<D>::THREADS, BwdCfg<D>::SMEM, stream>>>(tq, tk, tv, tdo, tdq, tdkv, tdk, tdv, p);
  return cudaGetLastError();
}

template cudaError_t launch_bwd<64>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                    const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                    const BwdParams&, int, cudaStream_t);
template cudaError_t launch_bwd<128>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                     const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                     const BwdParams&, int, cudaStream_t);

}  // namespace sap
