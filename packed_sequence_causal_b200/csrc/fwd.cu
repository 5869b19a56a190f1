// Forward kernel: partial attention of one q-tile over the kv tiles of one kv
// chunk ("partial attention computation" of the HSAP / Sequence-Aware
// Parallelism abstract), for every (forward unit, query head) work item.
//
// Persistent CTA, warp-specialised (192 threads):
//   warp 0      TMA producer: Q tile per work item, K/V tiles through an
//               NS-stage ring (128-byte swizzled boxes of 64 columns).
//   warp 1      TMEM owner and tcgen05.mma issuer (one thread):
//                 S_b = Q K^T   (M=128, N=128, K=D)   into TMEM buffer b = j % 2
//                 O  += P V     (M=128, N=D,   K=128) into the TMEM O accumulator
//               S_{j+1} is issued before P_j V_j so QK^T overlaps the softmax.
//   warps 2..5  softmax warpgroup: thread t owns TMEM lane t = query row t of
//               the tile.  Per kv tile it reads its S row, masks it (tag != FULL:
//               keys outside [first token of its document, its own token]),
//               runs the online softmax in the log2 domain, writes P (bf16)
//               into a 128-byte swizzled shared tile for the PV MMA, and
//               rescales O in TMEM when its running max grows by more than
//               2^8 (lazy rescaling; exact, because the final division uses
//               the same running max).  The epilogue normalises O and writes
//               either bf16 O + LSE (single-chunk q-tiles) or an fp32 partial.
//
// TMEM columns: S0 [0,128), S1 [128,256), O [256, 256+D).
#include <cuda.h>
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace sap {

template <int D>
struct FwdCfg {
  static constexpr int BM = 128, BN = 128;
  static constexpr int NS = (D == 64) ? 3 : 2;          // K/V ring depth
  static constexpr int BOX = 128 * 128;                 // bytes of one 128-row x 64-col bf16 box
  static constexpr int QBYTES = D * BM * 2;
  static constexpr int KVBYTES = D * BN * 2;
  static constexpr int PBYTES = BM * BN * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QBYTES;
  static constexpr int OFF_V = OFF_K + NS * KVBYTES;
  static constexpr int OFF_P = OFF_V + NS * KVBYTES;
  static constexpr int OFF_BAR = OFF_P + PBYTES;
  static constexpr int NBAR = 2 + 4 * NS + 4 + 2 + 1;
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;  // + tmem slot/abort flag + alignment slack
  static constexpr int THREADS = 192;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_O = 256;
};

template <int D>
__global__ void __launch_bounds__(192, 1)
    sap_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;
  uint64_t* k_empty = k_full + C::NS;
  uint64_t* v_full = k_empty + C::NS;
  uint64_t* v_empty = v_full + C::NS;
  uint64_t* s_full = v_empty + C::NS;  // [2]
  uint64_t* s_empty = s_full + 2;      // [2]
  uint64_t* p_full = s_empty + 2;
  uint64_t* pv_done = p_full + 1;
  uint64_t* mma_drain = pv_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const Guard guard{abort_flag, p.err, p.wait_ns};
  // Softmax-to-MMA handoffs: one arrival per warp at d = 64, one per thread at d = 128 (measured:
  // per-warp arrivals made the d = 64 forward 1.3% faster and the d = 128 forward 0.8% slower).
  constexpr bool kPWarp = D == 64;
  auto softmax_arrive = [](uint64_t* bar) {
    if constexpr (kPWarp)
      mbar_arrive_warp(bar);
    else
      mbar_arrive(bar);
  };

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(k_empty + s, 1);
      mbar_init(v_full + s, 1);
      mbar_init(v_empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full + b, 1);
      mbar_init(s_empty + b, kPWarp ? 4 : 128);  // per softmax warp (d = 64) or thread
    }
    mbar_init(p_full, kPWarp ? 4 : 128);
    mbar_init(pv_done, 1);
    mbar_init(mma_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int total = p.n_units * p.hq;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      uint32_t kv_iter = 0, unit_iter = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
        const int u = p.order[w / p.hq], h = w % p.hq, g = h / p.group;
        const int qt = p.units[4 * u], ib = p.units[4 * u + 1], ic = p.units[4 * u + 2];
        if (!mbar_wait(q_empty, (unit_iter & 1) ^ 1, guard, kErrTimeoutLoad)) break;
        mbar_arrive_expect_tx(q_full, C::QBYTES);
        for (int b = 0; b < D / 64; ++b)
          tma_load_3d(smem + C::OFF_Q + b * C::BOX, &tmQ, q_full, 64 * b, h, qt * 128 - (int)p.q0);
        for (int t = 0; t < ic; ++t) {
          const int kt = p.items[5 * (ib + t) + 1];
          const int s = kv_iter % C::NS;
          const uint32_t ph = (kv_iter / C::NS) & 1;
          if (!mbar_wait(k_empty + s, ph ^ 1, guard, kErrTimeoutLoad)) { ok = false; break; }
          mbar_arrive_expect_tx(k_full + s, C::KVBYTES);
          for (int b = 0; b < D / 64; ++b)
            tma_load_3d(smem + C::OFF_K + s * C::KVBYTES + b * C::BOX, &tmK, k_full + s, 64 * b, g,
                        kt * 128 - (int)p.kv0);
          if (!mbar_wait(v_empty + s, ph ^ 1, guard, kErrTimeoutLoad)) { ok = false; break; }
          // test hook: CTA 0 leaves its first V tile out (nothing is issued), so the MMA wait on it runs out
          if (!(p.skip_v_load && blockIdx.x == 0 && kv_iter == 0)) {
            mbar_arrive_expect_tx(v_full + s, C::KVBYTES);
            for (int b = 0; b < D / 64; ++b)
              tma_load_3d(smem + C::OFF_V + s * C::KVBYTES + b * C::BOX, &tmV, v_full + s, 64 * b, g,
                          kt * 128 - (int)p.kv0);
          }
          ++kv_iter;
        }
        ++unit_iter;
      }
      // Let every copy this thread started land before the CTA can exit.
      if (unit_iter > 0) drain_wait(q_full, (unit_iter - 1) & 1, p.wait_ns);
      for (uint32_t t = (kv_iter > (uint32_t)C::NS ? kv_iter - C::NS : 0); t < kv_iter; ++t) {
        const int s = t % C::NS;
        const uint32_t ph = (t / C::NS) & 1;
        drain_wait(k_full + s, ph, p.wait_ns);
        drain_wait(v_full + s, ph, p.wait_ns);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ----------------------------------------------------------------- MMA
      constexpr uint32_t idesc_qk = idesc_bf16(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16(128, D, false, true);
      const uint32_t sQ = smem_u32(smem + C::OFF_Q), sK = smem_u32(smem + C::OFF_K),
                     sV = smem_u32(smem + C::OFF_V), sP = smem_u32(smem + C::OFF_P);
      // descriptors computed once per operand base; per k-slice and stage only an offset is added
      const uint64_t dQ = sdesc_sw128(sQ, 16, 1024), dK = sdesc_sw128(sK, 16, 1024);
      const uint64_t dV = sdesc_sw128(sV, C::BOX, 1024), dP = sdesc_sw128(sP, 16, 1024);
      uint32_t kv_iter = 0, unit_iter = 0, s_iter = 0, pv_iter = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
        const int u = p.order[w / p.hq];
        const int ic = p.units[4 * u + 2];
        if (!mbar_wait(q_full, unit_iter & 1, guard, kErrTimeoutMma)) break;
        tc_fence_after();
        auto issue_pv = [&](uint32_t it) -> bool {  // it = kv_iter index of the tile
          const int s = it % C::NS;
          const uint32_t ph = (it / C::NS) & 1;
          if (!mbar_wait(p_full, pv_iter & 1, guard, kErrTimeoutMma)) return false;
          if (!mbar_wait(v_full + s, ph, guard, kErrTimeoutMma)) return false;
          tc_fence_after();
          const bool first = (it == kv_iter);  // first tile of this unit
#pragma unroll
          for (int kk = 0; kk < 128 / 16; ++kk) {
            const uint64_t a = sdesc_off(dP, (kk / 4) * C::BOX + (kk % 4) * 32);
            const uint64_t b = sdesc_off(dV, s * C::KVBYTES + kk * 2048);
            mma_bf16(tmem + C::COL_O, a, b, idesc_pv, (first && kk == 0) ? 0u : 1u);
          }
          tc_commit(pv_done);
          tc_commit(v_empty + s);
          ++pv_iter;
          return true;
        };
        for (int j = 0; j < ic; ++j) {
          const uint32_t it = kv_iter + j;
          const int s = it % C::NS;
          const uint32_t ph = (it / C::NS) & 1;
          const int b = s_iter & 1;
          if (!mbar_wait(k_full + s, ph, guard, kErrTimeoutMma)) { ok = false; break; }
          if (!mbar_wait(s_empty + b, ((s_iter >> 1) & 1) ^ 1, guard, kErrTimeoutMma)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t a = sdesc_off(dQ, (kk / 4) * C::BOX + (kk % 4) * 32);
            const uint64_t bd = sdesc_off(dK, s * C::KVBYTES + (kk / 4) * C::BOX + (kk % 4) * 32);
            mma_bf16(tmem + 128 * b, a, bd, idesc_qk, kk > 0 ? 1u : 0u);
          }
          tc_commit(s_full + b);
          tc_commit(k_empty + s);
          ++s_iter;
          if (j >= 1 && !issue_pv(it - 1)) { ok = false; break; }
        }
        if (ok && !issue_pv(kv_iter + ic - 1)) ok = false;
        tc_commit(q_empty);
        kv_iter += ic;
        ++unit_iter;
      }
      // Wait for every MMA this thread issued before TMEM is released.
      tc_commit(mma_drain);
      drain_wait(mma_drain, 0, p.wait_ns);
    }
  } else {
    // ------------------------------------------------------------- softmax
    const int quad = warp & 3;            // TMEM lane quadrant this warp may access
    const int r = quad * 32 + lane;       // query row within the tile
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    uint8_t* sP = smem + C::OFF_P;
    uint32_t s_iter = 0, pv_iter = 0;
    const float sl2 = p.scale_log2;
    for (int w = blockIdx.x; w < total; w += gridDim.x) {
      const int u = p.order[w / p.hq], h = w % p.hq;
      const int qt = p.units[4 * u], ib = p.units[4 * u + 1], ic = p.units[4 * u + 2], slot = p.units[4 * u + 3];
      const int64_t i = (int64_t)qt * 128 + r;
      const bool real_row = i < p.q_end;
      const int row_lo = real_row ? p.tok_lo[i] : 1;  // empty key range for rows past the window
      const int row_hi = real_row ? (int)i : 0;
      float m = -INFINITY, l = 0.f;
      bool ok = true;
      for (int j = 0; j < ic; ++j) {
        const int kt = p.items[5 * (ib + j) + 1], tag = p.items[5 * (ib + j) + 4];
        const int b = s_iter & 1;
        if (!mbar_wait_warp(s_full + b, (s_iter >> 1) & 1, guard, kErrTimeoutSoftmax)) { ok = false; break; }
        tc_fence_after();
        float sv[128];
        tmem_ld128(lane_base + 128 * b, sv);
        tc_fence_before();
        softmax_arrive(s_empty + b);
        ++s_iter;
        if (tag != 0) {
          const int c_lo = row_lo - kt * 128, c_hi = row_hi - kt * 128;
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c < c_lo || c > c_hi) sv[c] = -INFINITY;
        }
        // row max as 8 independent chains (a single 128-long chain is latency-bound)
        float mx8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mx8[e] = sv[e];
#pragma unroll
        for (int c = 8; c < 128; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], sv[c]);
#pragma unroll
        for (int e = 0; e < 4; ++e) mx8[e] = fmaxf(mx8[e], mx8[e + 4]);
        const float mx = fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3]));
        const float m_tile = mx * sl2;
        // P_{j-1} V_{j-1} must be complete before O is rescaled or P is overwritten.
        if (j > 0) {
          if (!mbar_wait_warp(pv_done, pv_iter & 1, guard, kErrTimeoutSoftmax)) { ok = false; break; }
          ++pv_iter;
          tc_fence_after();
        }
        // Rows decide independently whether their max moved; the TMEM
        // load/store of O is warp-collective, so the warp rescales together
        // when any of its rows needs it (alpha = 1 for the others).
        const bool grow = m_tile > m + 8.0f;
        const float alpha = grow ? ex2(m - m_tile) : 1.f;  // 0 when m = -inf
        if (j > 0 && __any_sync(0xffffffffu, grow && l > 0.f)) {
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            float ov[32];
            tmem_ld32(lane_base + C::COL_O + 32 * c, ov);
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] *= alpha;
            tmem_st32(lane_base + C::COL_O + 32 * c, ov);
          }
        }
        if (grow) {
          l *= alpha;
          m = m_tile;
        }
        const float base = (m == -INFINITY) ? 0.f : m;
        float rs4[4] = {0.f, 0.f, 0.f, 0.f};  // row sum as 4 independent chains
#pragma unroll
        for (int cc = 0; cc < 16; ++cc) {
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float p0 = ex2(fmaf(sv[cc * 8 + 2 * e], sl2, -base));
            const float p1 = ex2(fmaf(sv[cc * 8 + 2 * e + 1], sl2, -base));
            rs4[e] += p0 + p1;
            w4[e] = pack_bf16x2(p0, p1);
          }
          const uint32_t addr = smem_u32(sP + (cc / 8) * C::BOX + sw128_offset(r, cc % 8));
          st_shared_v4(addr, w4[0], w4[1], w4[2], w4[3]);
        }
        l += (rs4[0] + rs4[1]) + (rs4[2] + rs4[3]);
        fence_async_smem();
        tc_fence_before();
        softmax_arrive(p_full);
      }
      if (!ok) break;
      // ------------------------------------------------------------ epilogue
      if (!mbar_wait_warp(pv_done, pv_iter & 1, guard, kErrTimeoutEpilogue)) break;
      ++pv_iter;
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      const float lse_val = l > 0.f ? (m + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
      if (slot < 0) {
        __nv_bfloat16* orow = p.o + ((size_t)(i - p.q0) * p.hq + h) * D;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          float ov[32];
          tmem_ld32(lane_base + C::COL_O + 32 * c, ov);
          if (real_row) {
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              uint4 pk;
              pk.x = pack_bf16x2(ov[e] * inv_l, ov[e + 1] * inv_l);
              pk.y = pack_bf16x2(ov[e + 2] * inv_l, ov[e + 3] * inv_l);
              pk.z = pack_bf16x2(ov[e + 4] * inv_l, ov[e + 5] * inv_l);
              pk.w = pack_bf16x2(ov[e + 6] * inv_l, ov[e + 7] * inv_l);
              *reinterpret_cast<uint4*>(orow + 32 * c + e) = pk;
            }
          }
        }
        if (real_row) p.lse[(size_t)h * p.lse_ld + (i - p.q0)] = lse_val;
      } else {
        float* orow = p.o_part + (((size_t)slot * p.hq + h) * 128 + r) * D;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          float ov[32];
          tmem_ld32(lane_base + C::COL_O + 32 * c, ov);
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(orow + 32 * c + e) =
                make_float4(ov[e] * inv_l, ov[e + 1] * inv_l, ov[e + 2] * inv_l, ov[e + 3] * inv_l);
        }
        p.lse_part[((size_t)slot * p.hq + h) * 128 + r] = lse_val;
      }
      // The next unit's first PV overwrites O only after p_full, which these
      // threads signal after this point, so the TMEM reads above are ordered
      // before it by the fence below.
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Two-tile variant for an even GQA group: one CTA computes the same q tile for
// two query heads of one kv group, so both tiles walk the same kv tiles and
// share every K/V load.  P is written back into TMEM (packed bf16 over the S
// columns) and read from there by the PV MMA, and the MMA thread interleaves
// the tiles -- S0, S1, PV0, S0', PV1, S1', ... -- so that while one softmax
// warpgroup exponentiates its tile the tensor core works on the other.  Each PV
// is issued in two halves (kv rows 0..63, then 64..127): the softmax signals
// p_half once the first half of P is in TMEM, so the first half of PV runs while
// the second half of P is being computed.
//
// KVS = true (odd GQA group, MHA included): the two heads 2p and 2p+1 may belong to different kv
// heads, so each tile gets its own K and V tiles: the rings hold K_A(t), K_B(t), ... and
// V_A(t), V_B(t), ... in order of use, and each stage is released as soon as its one tile has read
// it.  The kv tile sequence is the same for both tiles (one q tile, one unit).
//
// Threads: warp 0 TMA, warp 1 MMA, warps 2..5 softmax of tile 0 (head 2p),
// warps 6..9 softmax of tile 1 (head 2p+1).
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [256+D,256+2D); at D = 64 also
// P0 [384,448) and P1 [448,512) (P has columns of its own there; at D = 128 it goes over S).
//
// CTA2 = true (D = 128, GQA group a multiple of 4): a cluster of two CTAs takes one q tile of
// four query heads of a kv group, two per CTA, and runs every MMA as one two-CTA tcgen05.mma
// (cta_group::2, M = 256) issued by the leader (cluster rank 0): rows 0..127 of the product are
// the leader's tile, rows 128..255 the other CTA's.  The B operand is split between the pair:
// each CTA loads only its half of every K tile (64 of the 128 kv rows) and of every V tile (64 of
// the D columns), so a kv tile is read once per four heads and each SM's shared-memory operand
// traffic for B halves.  Both CTAs' copies complete on the leader's barriers; the leader's
// commits arrive on both CTAs' barriers; the other CTA's softmax threads arrive on the leader's
// P barriers (remote arrivals; the tensor-memory fences order their P writes before the MMAs).
// Softmax and epilogue are unchanged: each CTA owns the TMEM rows of its tiles.
template <int D, bool CTA2>
struct Fwd2Cfg {
  static_assert(!CTA2 || D == 128, "the two-CTA variant is built for head_dim 128");
  static constexpr int NS = CTA2 ? 4 : (D == 64) ? 3 : 2;
  static constexpr int BOX = 128 * 128;
  static constexpr int QBYTES = D * 128 * 2;
  // one stage: this CTA's K tile and V tile (CTA2: its 64 kv rows of K, its 64 columns of V)
  static constexpr int KBYTES = CTA2 ? D * 64 * 2 : D * 128 * 2;
  static constexpr int VBYTES = CTA2 ? 64 * 128 * 2 : D * 128 * 2;
  static constexpr int KSLAB = CTA2 ? 64 * 128 : BOX;  // bytes between the 64-column slabs of a K tile
  static constexpr int OFF_Q0 = 0;
  static constexpr int OFF_Q1 = QBYTES;
  static constexpr int OFF_K = 2 * QBYTES;
  static constexpr int OFF_V = OFF_K + NS * KBYTES;
  static constexpr int OFF_BAR = OFF_V + NS * VBYTES;
  static constexpr int NW = 4;  // work-index ring depth (dynamic order)
  static constexpr int NBAR = 2 + 4 * NS + 2 + 2 + 2 + 2 + 2 * NW + 4;
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 4 * NW;
  static constexpr int THREADS = 320;
  static constexpr uint32_t COL_O = 256;
};

template <int D, bool CTA2, bool KVS>
__global__ void __launch_bounds__(320, 1)
    sap_fwd_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  static_assert(!(CTA2 && KVS), "the two-CTA variant shares K/V between the heads of a kv group");
  using C = Fwd2Cfg<D, CTA2>;
  constexpr int LPS = KVS ? 2 : 1;  // K (and V) tiles loaded per kv step: one per tile with KVS
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) atomicOr(p.err, kErrSmemAlign);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;
  uint64_t* k_empty = k_full + C::NS;
  uint64_t* v_full = k_empty + C::NS;
  uint64_t* v_empty = v_full + C::NS;
  uint64_t* s_full = v_empty + C::NS;  // [2], one per tile
  uint64_t* p_full = s_full + 2;       // [2]
  uint64_t* p_half = p_full + 2;       // [2] first half of P (kv rows 0..63) is in TMEM
  uint64_t* o_done = p_half + 2;
  uint64_t* mma_drain = o_done + 1;
  uint64_t* sched_full = mma_drain + 1;        // [NW] the producer wrote the next work index
  uint64_t* sched_empty = sched_full + C::NW;  // [NW] the MMA thread and the 8 softmax warps read it
  uint64_t* s_loaded = sched_empty + C::NW;    // [2] d = 64: the softmax has read all of S
  uint64_t* pv_done = s_loaded + 2;            // [2] d = 64: the tile's PV has completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* sched_w = reinterpret_cast<volatile int*>(smem + C::OFF_BAR + C::NBAR * 8 + 16);  // [NW]

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const Guard guard{abort_flag, p.err, p.wait_ns};
  // Softmax-to-MMA handoffs: one arrival per warp at d = 64, one per thread at d = 128 (measured:
  // per-warp arrivals made the d = 64 forward 1.3% faster and the d = 128 forward 0.8% slower).
  constexpr bool kPWarp = D == 64;
  // Early S (d = 64): TMEM has 128 columns beyond S0, S1, O0 and O1, so each tile's P (packed bf16,
  // 64 columns) gets a region of its own, [384 + 64 * tile, +64), instead of going over S.  The next S
  // then needs neither P's columns nor the PV: it is issued as soon as the softmax has read all of S,
  // and the softmax finds it ready instead of waiting for the PV and the next S to run.  The softmax
  // writes the next P once the PV that read the previous one has completed.
  constexpr bool kEarlyS = D == 64 && !CTA2;
  auto softmax_arrive = [](uint64_t* bar) {
    if constexpr (kPWarp)
      mbar_arrive_warp(bar);
    else
      mbar_arrive(bar);
  };
  const uint32_t rank = CTA2 ? cluster_ctarank() : 0u;  // CTA2: 0 = leader of the pair
  const bool leader = rank == 0;
  // CTA2: the leader's barrier at the same offset (shared::cluster address); where the loads of
  // both CTAs complete and the P arrivals of both CTAs land
  auto at_leader = [&](uint64_t* bar) { return mapa_shared(smem_u32(bar), 0); };
  auto commit = [&](uint64_t* bar) {  // arrives on this barrier in both CTAs (CTA2) or in this CTA
    if constexpr (CTA2)
      tc_commit_pair(bar, 0x3);
    else
      tc_commit(bar);
  };

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(k_empty + s, 1);
      mbar_init(v_full + s, 1);
      mbar_init(v_empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full + b, 1);
      mbar_init(p_full + b, CTA2 ? 256 : kPWarp ? 4 : 128);  // per softmax warp (d = 64) or thread
      mbar_init(p_half + b, CTA2 ? 256 : kPWarp ? 4 : 128);
      mbar_init(s_loaded + b, kPWarp ? 4 : 128);
      mbar_init(pv_done + b, 1);
    }
    mbar_init(o_done, 1);
    mbar_init(mma_drain, 1);
    for (int s = 0; s < C::NW; ++s) {
      mbar_init(sched_full + s, 1);
      mbar_init(sched_empty + s, 1 + 8);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    if constexpr (CTA2) {
      tmem_alloc_pair(tmem_slot, 512);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, 512);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (CTA2) cluster_sync();  // both CTAs' barriers are initialised before any remote use
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  constexpr int HEADS = CTA2 ? 4 : 2;  // query heads per work item (two per CTA)
  const int pairs = p.hq / HEADS;
  const int total = p.n_units * pairs;
  const int w0 = CTA2 ? (int)(blockIdx.x / 2) : (int)blockIdx.x;  // work items are per cluster
  const int wstep = CTA2 ? (int)(gridDim.x / 2) : (int)gridDim.x;
  // Work order.  Static: item w0 + i * wstep for the i-th item of this CTA (CTA2 always).  Dynamic
  // (p.work_next set): the first item is w0, the next ones come from a global counter, so a CTA that
  // finishes early takes the next item in schedule order; the producer fetches each index and
  // publishes it through a ring of NW slots, and the MMA thread and the softmax warps read them in
  // the same order.  -1 ends the sequence; -2 marks a wait that ran out.
  const bool dynamic = !CTA2 && p.work_next != nullptr;
  auto publish_work = [&](uint32_t i) -> int {  // producer thread
    if (!dynamic) return (int)(w0 + i * wstep) < total ? (int)(w0 + i * wstep) : -1;
    const int ws = i % C::NW;
    if (!mbar_wait(sched_empty + ws, ((i / C::NW) & 1) ^ 1, guard, kErrTimeoutLoad)) return -2;
    int w = i == 0 ? w0 : wstep + atomicAdd(p.work_next, 1);
    if (w >= total) w = -1;
    sched_w[ws] = w;
    mbar_arrive(sched_full + ws);
    return w;
  };
  auto read_work = [&](uint32_t i, int code, bool warp_wide) -> int {  // MMA thread, softmax warps
    if (!dynamic) return (int)(w0 + i * wstep) < total ? (int)(w0 + i * wstep) : -1;
    const int ws = i % C::NW;
    const bool got = warp_wide ? mbar_wait_warp(sched_full + ws, (i / C::NW) & 1, guard, code)
                               : mbar_wait(sched_full + ws, (i / C::NW) & 1, guard, code);
    if (!got) return -2;
    const int w = sched_w[ws];
    if (warp_wide) {
      __syncwarp();
      if (lane == 0) mbar_arrive(sched_empty + ws);
    } else {
      mbar_arrive(sched_empty + ws);
    }
    return w;
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      uint32_t kq = 0, vq = 0, unit_iter = 0;  // K / V loads issued (ring positions)
      bool ok = true;
      // K, V tile of kv tile kt for kv head g into the next ring stage
      auto load_k = [&](int g, int kt) -> bool {
        const int s = kq % C::NS;
        if (!mbar_wait(k_empty + s, ((kq / C::NS) & 1) ^ 1, guard, kErrTimeoutLoad)) return false;
        if (leader) mbar_arrive_expect_tx(k_full + s, (CTA2 ? 2 : 1) * C::KBYTES);
        for (int b = 0; b < D / 64; ++b) {
          if constexpr (CTA2)  // this CTA's 64 kv rows of the tile (the K map has 64-row boxes)
            tma_load_3d_pair(smem + C::OFF_K + s * C::KBYTES + b * C::KSLAB, &tmK, at_leader(k_full + s), 64 * b,
                             g, kt * 128 - (int)p.kv0 + 64 * (int)rank);
          else
            tma_load_3d(smem + C::OFF_K + s * C::KBYTES + b * C::BOX, &tmK, k_full + s, 64 * b, g,
                        kt * 128 - (int)p.kv0);
        }
        ++kq;
        return true;
      };
      auto load_v = [&](int g, int kt) -> bool {
        const int s = vq % C::NS;
        if (!mbar_wait(v_empty + s, ((vq / C::NS) & 1) ^ 1, guard, kErrTimeoutLoad)) return false;
        // test hook: CTA 0 leaves its first V tile out (nothing is issued), so the MMA wait on it runs out
        if (!(p.skip_v_load && blockIdx.x == 0 && vq == 0)) {
          if (leader) mbar_arrive_expect_tx(v_full + s, (CTA2 ? 2 : 1) * C::VBYTES);
          if constexpr (CTA2)  // this CTA's 64 of the D columns, all 128 kv rows
            tma_load_3d_pair(smem + C::OFF_V + s * C::VBYTES, &tmV, at_leader(v_full + s), 64 * (int)rank, g,
                             kt * 128 - (int)p.kv0);
          else
            for (int b = 0; b < D / 64; ++b)
              tma_load_3d(smem + C::OFF_V + s * C::VBYTES + b * C::BOX, &tmV, v_full + s, 64 * b, g,
                          kt * 128 - (int)p.kv0);
        }
        ++vq;
        return true;
      };
      for (uint32_t wi = 0; ok; ++wi) {
        const int w = publish_work(wi);
        if (w < 0) break;
        const int u = p.order[w / pairs], h0 = HEADS * (w % pairs) + 2 * (int)rank;
        const int gA = h0 / p.group, gB = KVS ? (h0 + 1) / p.group : gA;  // kv heads of the two tiles
        const int qt = p.units[4 * u], ib = p.units[4 * u + 1], ic = p.units[4 * u + 2];
        if (!mbar_wait(q_empty, (unit_iter & 1) ^ 1, guard, kErrTimeoutLoad)) break;
        if (leader) mbar_arrive_expect_tx(q_full, (CTA2 ? 4 : 2) * C::QBYTES);
        for (int b = 0; b < D / 64; ++b) {
          if constexpr (CTA2) {
            tma_load_3d_pair(smem + C::OFF_Q0 + b * C::BOX, &tmQ, at_leader(q_full), 64 * b, h0,
                             qt * 128 - (int)p.q0);
            tma_load_3d_pair(smem + C::OFF_Q1 + b * C::BOX, &tmQ, at_leader(q_full), 64 * b, h0 + 1,
                             qt * 128 - (int)p.q0);
          } else {
            tma_load_3d(smem + C::OFF_Q0 + b * C::BOX, &tmQ, q_full, 64 * b, h0, qt * 128 - (int)p.q0);
            tma_load_3d(smem + C::OFF_Q1 + b * C::BOX, &tmQ, q_full, 64 * b, h0 + 1, qt * 128 - (int)p.q0);
          }
        }
        // Order of the loads = order of their use: K of step 0 (per tile with KVS), then per step t
        // V(t) and K(t + 1), tile A before tile B.
        int kt = p.items[5 * ib + 1];
        if (!load_k(gA, kt) || (KVS && !load_k(gB, kt))) break;
        for (int t = 0; t < ic; ++t) {
          const int kt_next = t + 1 < ic ? p.items[5 * (ib + t + 1) + 1] : -1;
          if (!load_v(gA, kt) || (kt_next >= 0 && !load_k(gA, kt_next))) { ok = false; break; }
          if (KVS && (!load_v(gB, kt) || (kt_next >= 0 && !load_k(gB, kt_next)))) { ok = false; break; }
          kt = kt_next;
        }
        ++unit_iter;
      }
      // Let every copy land before the CTA can exit.  CTA2: the full barriers live in the leader and
      // count both CTAs' copies; the other CTA is held at the final cluster barrier until then.
      if (leader) {
        if (unit_iter > 0) drain_wait(q_full, (unit_iter - 1) & 1, p.wait_ns);
        for (uint32_t t = (kq > (uint32_t)C::NS ? kq - C::NS : 0); t < kq; ++t)
          drain_wait(k_full + t % C::NS, (t / C::NS) & 1, p.wait_ns);
        for (uint32_t t = (vq > (uint32_t)C::NS ? vq - C::NS : 0); t < vq; ++t)
          drain_wait(v_full + t % C::NS, (t / C::NS) & 1, p.wait_ns);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {  // CTA2: only the leader issues the pair's MMAs
      // ----------------------------------------------------------------- MMA
      constexpr uint32_t idesc_qk = idesc_bf16(CTA2 ? 256 : 128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16(CTA2 ? 256 : 128, D, false, true);
      // P arrivals (CTA2: from both CTAs' softmax threads)
      auto wait_p = [&](uint64_t* bar, uint32_t parity) { return mbar_wait(bar, parity, guard, kErrTimeoutMma); };
      const uint32_t sQ0 = smem_u32(smem + C::OFF_Q0), sQ1 = smem_u32(smem + C::OFF_Q1);
      const uint32_t sK = smem_u32(smem + C::OFF_K), sV = smem_u32(smem + C::OFF_V);
      uint32_t unit_iter = 0, tile_iter = 0;  // tile_iter counts kv tiles (per tile barrier phases)
      bool ok = true;
      // descriptors computed once per operand base; per k-slice only an offset is added
      const uint64_t dQ0 = sdesc_sw128(sQ0, 16, 1024), dQ1 = sdesc_sw128(sQ1, 16, 1024);
      const uint64_t dK = sdesc_sw128(sK, 16, 1024), dV = sdesc_sw128(sV, C::BOX, 1024);
      auto issue_s = [&](int tile, uint32_t it) {  // S_tile = Q_tile K_it^T
        const uint64_t dQ = tile ? dQ1 : dQ0;
        const uint64_t dKs = sdesc_off(dK, (it % C::NS) * C::KBYTES);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t a = sdesc_off(dQ, (kk / 4) * C::BOX + (kk % 4) * 32);
          const uint64_t bd = sdesc_off(dKs, (kk / 4) * C::KSLAB + (kk % 4) * 32);
          if constexpr (CTA2)
            mma_bf16_pair(tmem + 128 * tile, a, bd, idesc_qk, kk > 0);
          else
            mma_bf16(tmem + 128 * tile, a, bd, idesc_qk, kk > 0);
        }
        commit(s_full + tile);
      };
      auto issue_pv = [&](int tile, uint32_t it, bool first, int part) {  // O_tile += P_tile V_it (half), P from TMEM
        const uint64_t dVs = sdesc_off(dV, (it % C::NS) * C::VBYTES);
        const uint32_t colP = kEarlyS ? 384u + 64u * tile : 128u * tile;
#pragma unroll
        for (int kk = 4 * part; kk < 4 * part + 4; ++kk) {
          const uint64_t bd = sdesc_off(dVs, kk * 2048);
          if constexpr (CTA2)
            mma_bf16_tmem_a_pair(tmem + C::COL_O + D * tile, tmem + colP + kk * 8, bd, idesc_pv,
                                 (first && kk == 0) ? 0u : 1u);
          else
            mma_bf16_tmem_a(tmem + C::COL_O + D * tile, tmem + colP + kk * 8, bd, idesc_pv,
                            (first && kk == 0) ? 0u : 1u);
        }
      };
      auto wait_k = [&](uint32_t i) { return mbar_wait(k_full + i % C::NS, (i / C::NS) & 1, guard, kErrTimeoutMma); };
      auto wait_v = [&](uint32_t i) { return mbar_wait(v_full + i % C::NS, (i / C::NS) & 1, guard, kErrTimeoutMma); };
      uint32_t kc = 0, vc = 0;  // K / V ring positions consumed (LPS per kv step)
      for (uint32_t wi = 0; ok; ++wi) {
        const int w = read_work(wi, kErrTimeoutMma, false);
        if (w < 0) break;
        const int u = p.order[w / pairs];
        const int ic = p.units[4 * u + 2];
        if (!mbar_wait(q_full, unit_iter & 1, guard, kErrTimeoutMma)) break;
        if (!wait_k(kc)) break;
        tc_fence_after();
        issue_s(0, kc);
        if (KVS) {
          commit(k_empty + kc % C::NS);
          if (!wait_k(kc + 1)) break;
          tc_fence_after();
        }
        issue_s(1, kc + LPS - 1);
        commit(k_empty + (kc + LPS - 1) % C::NS);
        kc += LPS;
        for (int j = 0; j < ic; ++j, ++tile_iter, vc += LPS) {
          if constexpr (kEarlyS) {
            // Per tile: the first PV half, the next S once the softmax has read all of S (it signals
            // p_half, then s_loaded, then p_full), the second PV half.
            const bool more = j + 1 < ic;
            const uint32_t g = tile_iter;
            if (!wait_v(vc) || !wait_p(p_half + 0, g & 1)) { ok = false; break; }
            tc_fence_after();
            issue_pv(0, vc, j == 0, 0);
            if (more) {
              if (!mbar_wait(s_loaded + 0, g & 1, guard, kErrTimeoutMma) || !wait_k(kc)) { ok = false; break; }
              tc_fence_after();
              issue_s(0, kc);
              if (KVS) commit(k_empty + kc % C::NS);
            }
            if (!wait_p(p_full + 0, g & 1)) { ok = false; break; }
            tc_fence_after();
            issue_pv(0, vc, j == 0, 1);
            commit(pv_done + 0);
            if (KVS) commit(v_empty + vc % C::NS);
            if ((KVS && !wait_v(vc + 1)) || !wait_p(p_half + 1, g & 1)) { ok = false; break; }
            tc_fence_after();
            issue_pv(1, vc + LPS - 1, j == 0, 0);
            if (more) {
              if (!mbar_wait(s_loaded + 1, g & 1, guard, kErrTimeoutMma)) { ok = false; break; }
              if (KVS && !wait_k(kc + 1)) { ok = false; break; }
              tc_fence_after();
              issue_s(1, kc + LPS - 1);
              commit(k_empty + (kc + LPS - 1) % C::NS);
              kc += LPS;
            }
            if (!wait_p(p_full + 1, g & 1)) { ok = false; break; }
            tc_fence_after();
            issue_pv(1, vc + LPS - 1, j == 0, 1);
            commit(pv_done + 1);
            commit(v_empty + (vc + LPS - 1) % C::NS);
            continue;
          }
          if (!wait_v(vc)) { ok = false; break; }
          if (!wait_p(p_half + 0, tile_iter & 1)) { ok = false; break; }
          tc_fence_after();
          issue_pv(0, vc, j == 0, 0);
          if (!wait_p(p_full + 0, tile_iter & 1)) { ok = false; break; }
          tc_fence_after();
          issue_pv(0, vc, j == 0, 1);
          if (KVS) commit(v_empty + vc % C::NS);
          const bool more = j + 1 < ic;
          if (more) {
            if (!wait_k(kc)) { ok = false; break; }
            tc_fence_after();
            issue_s(0, kc);  // rewrites S0/P0 only after PV0 (issued above) has read P0
            if (KVS) commit(k_empty + kc % C::NS);
          }
          if (KVS && !wait_v(vc + 1)) { ok = false; break; }
          if (!wait_p(p_half + 1, tile_iter & 1)) { ok = false; break; }
          tc_fence_after();
          issue_pv(1, vc + LPS - 1, j == 0, 0);
          if (!wait_p(p_full + 1, tile_iter & 1)) { ok = false; break; }
          tc_fence_after();
          issue_pv(1, vc + LPS - 1, j == 0, 1);
          commit(v_empty + (vc + LPS - 1) % C::NS);
          if (more) {
            if (KVS) {
              if (!wait_k(kc + 1)) { ok = false; break; }
              tc_fence_after();
            }
            issue_s(1, kc + LPS - 1);
            commit(k_empty + (kc + LPS - 1) % C::NS);
            kc += LPS;
          }
        }
        if (!ok) break;
        commit(o_done);
        commit(q_empty);
        ++unit_iter;
      }
      // Wait for every MMA this thread issued before TMEM is released (CTA2: the leader's own barrier).
      if constexpr (CTA2)
        tc_commit_pair(mma_drain, 0x1);
      else
        tc_commit(mma_drain);
      drain_wait(mma_drain, 0, p.wait_ns);
    }
  } else {
    // ------------------------------------------------------------- softmax
    const int tile = (warp - 2) >> 2;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    const uint32_t colS = 128 * tile, colO = C::COL_O + D * tile;
    const uint32_t colP = kEarlyS ? 384u + 64u * tile : colS;  // P: own region (early S) or over S
    uint32_t tile_iter = 0, unit_iter = 0;
    const float sl2 = p.scale_log2;
    bool ok = true;
    for (uint32_t wi = 0; ok; ++wi) {
      const int w = read_work(wi, kErrTimeoutSoftmax, true);
      if (w < 0) break;
      const int u = p.order[w / pairs], h = HEADS * (w % pairs) + 2 * (int)rank + tile;
      const int qt = p.units[4 * u], ib = p.units[4 * u + 1], ic = p.units[4 * u + 2], slot = p.units[4 * u + 3];
      const int64_t i = (int64_t)qt * 128 + r;
      const bool real_row = i < p.q_end;
      const int row_lo = real_row ? p.tok_lo[i] : 1;
      const int row_hi = real_row ? (int)i : 0;
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < ic; ++j, ++tile_iter) {
        const int kt = p.items[5 * (ib + j) + 1], tag = p.items[5 * (ib + j) + 4];
        if (!mbar_wait_warp(s_full + tile, tile_iter & 1, guard, kErrTimeoutSoftmax)) { ok = false; break; }
        tc_fence_after();
        float sv[128];
        tmem_ld128(lane_base + colS, sv);
        if (tag != 0) {
          const int c_lo = row_lo - kt * 128, c_hi = row_hi - kt * 128;
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c < c_lo || c > c_hi) sv[c] = -INFINITY;
        }
        // row max as 8 independent chains (a single 128-long chain is latency-bound)
        float mx8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mx8[e] = sv[e];
#pragma unroll
        for (int c = 8; c < 128; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], sv[c]);
#pragma unroll
        for (int e = 0; e < 4; ++e) mx8[e] = fmaxf(mx8[e], mx8[e + 4]);
        const float mx = fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3]));
        const float m_tile = mx * sl2;
        // s_full of this tile also means the previous PV into O has completed -- except with early S,
        // where S_g is issued before the second half of PV_{g-1}: there the previous PV is waited for
        // here, before O is rescaled or P_g written over P_{g-1} (S_g was issued after PV_{g-2}, so
        // the parity wait cannot be a phase behind).
        if (kEarlyS && j > 0) {
          if (!mbar_wait_warp(pv_done + tile, (tile_iter - 1) & 1, guard, kErrTimeoutSoftmax)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        const bool grow = m_tile > m + 8.0f;
        const float alpha = grow ? ex2(m - m_tile) : 1.f;
        if (j > 0 && __any_sync(0xffffffffu, grow && l > 0.f)) {
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            float ov[32];
            tmem_ld32(lane_base + colO + 32 * c, ov);
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] *= alpha;
            tmem_st32(lane_base + colO + 32 * c, ov);
          }
        }
        if (grow) {
          l *= alpha;
          m = m_tile;
        }
        const float base = (m == -INFINITY) ? 0.f : m;
        float rs4[4] = {0.f, 0.f, 0.f, 0.f};  // row sum as 4 independent chains
        // The exponentials re-read S from TMEM 64 columns at a time: sv is dead after the row max,
        // which keeps the softmax warps inside the 168 registers that 10 warps per CTA allow.
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t pk[32];
          float sh[64];
          tmem_ld32(lane_base + colS + 64 * half, sh);
          tmem_ld32(lane_base + colS + 64 * half + 32, sh + 32);
          if (kEarlyS && half == 1) {  // all of S has been read: the next S may be written
            tc_fence_before();
            softmax_arrive(s_loaded + tile);
          }
          if (tag != 0) {
            const int c_lo = row_lo - kt * 128 - 64 * half, c_hi = row_hi - kt * 128 - 64 * half;
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (c < c_lo || c > c_hi) sh[c] = -INFINITY;
          }
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float p0 = ex2(fmaf(sh[2 * e], sl2, -base));
            const float p1 = ex2(fmaf(sh[2 * e + 1], sl2, -base));
            rs4[e & 3] += p0 + p1;
            pk[e] = pack_bf16x2(p0, p1);
          }
          tmem_st32_u(lane_base + colP + 32 * half, pk);  // P: over the S columns already read, or its own region
          if (half == 0) {  // PV over kv rows 0..63 may start while the second half is computed
            tc_fence_before();
            if constexpr (CTA2)
              mbar_arrive_remote(at_leader(p_half + tile));
            else
              softmax_arrive(p_half + tile);
          }
        }
        l += (rs4[0] + rs4[1]) + (rs4[2] + rs4[3]);
        tc_fence_before();
        if constexpr (CTA2)
          mbar_arrive_remote(at_leader(p_full + tile));
        else
          softmax_arrive(p_full + tile);
      }
      if (!ok) break;
      // ------------------------------------------------------------ epilogue
      if (!mbar_wait_warp(o_done, unit_iter & 1, guard, kErrTimeoutEpilogue)) break;
      ++unit_iter;
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      const float lse_val = l > 0.f ? (m + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
      if (slot < 0) {
        __nv_bfloat16* orow = p.o + ((size_t)(i - p.q0) * p.hq + h) * D;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          float ov[32];
          tmem_ld32(lane_base + colO + 32 * c, ov);
          if (real_row) {
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              uint4 pk;
              pk.x = pack_bf16x2(ov[e] * inv_l, ov[e + 1] * inv_l);
              pk.y = pack_bf16x2(ov[e + 2] * inv_l, ov[e + 3] * inv_l);
              pk.z = pack_bf16x2(ov[e + 4] * inv_l, ov[e + 5] * inv_l);
              pk.w = pack_bf16x2(ov[e + 6] * inv_l, ov[e + 7] * inv_l);
              *reinterpret_cast<uint4*>(orow + 32 * c + e) = pk;
            }
          }
        }
        if (real_row) p.lse[(size_t)h * p.lse_ld + (i - p.q0)] = lse_val;
      } else {
        float* orow = p.o_part + (((size_t)slot * p.hq + h) * 128 + r) * D;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          float ov[32];
          tmem_ld32(lane_base + colO + 32 * c, ov);
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(orow + 32 * c + e) =
                make_float4(ov[e] * inv_l, ov[e + 1] * inv_l, ov[e + 2] * inv_l, ov[e + 3] * inv_l);
        }
        p.lse_part[((size_t)slot * p.hq + h) * 128 + r] = lse_val;
      }
      // The next unit's first PV into O waits for this warpgroup's next p_half and p_full.
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  // CTA2: the leader's MMAs read this CTA's shared and tensor memory, and this CTA's copies
  // complete on the leader's barriers; neither CTA leaves before the leader has drained both.
  if constexpr (CTA2) cluster_sync();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    if constexpr (CTA2)
      tmem_dealloc_pair(tmem, 512);
    else
      tmem_dealloc(tmem, 512);
  }
}

template <int D>
int fwd_smem_bytes() {
  return FwdCfg<D>::SMEM;
}

template <int D>
cudaError_t launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p,
                       int grid, cudaStream_t stream, bool two_cta) {
  if constexpr (D == 128) {
    if (two_cta) {  // clusters of two CTAs, four heads of a kv group per cluster (group % 4 == 0)
      if (p.group % 4 != 0) return cudaErrorInvalidValue;
      auto kern = sap_fwd_pair_kernel<128, true, false>;
      using C2 = Fwd2Cfg<128, true>;
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C2::SMEM);
      if (e != cudaSuccess) return e;
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.blockDim = dim3(C2::THREADS);
      cfg.dynamicSmemBytes = C2::SMEM;
      cfg.stream = stream;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      // persistent clusters: no more than can be resident at once, nor than there is work
      int max_clusters = 0;
      cfg.gridDim = dim3(2 * (grid / 2 > 0 ? grid / 2 : 1));
      e = cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg);
      if (e != cudaSuccess) return e;
      const int64_t work = (int64_t)p.n_units * (p.hq / 4);
      int64_t clusters = grid / 2;
      if (max_clusters > 0 && clusters > max_clusters) clusters = max_clusters;
      if (clusters > work) clusters = work;
      if (clusters <= 0) return cudaSuccess;
      cfg.gridDim = dim3((unsigned)(2 * clusters));
      e = cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, p);
      if (e != cudaSuccess) return e;
      return cudaGetLastError();
    }
  }
  // Two query heads per CTA: of one kv group (even group: shared K/V loads), or any two adjacent
  // heads with their own K/V loads (odd group, even number of query heads).
  if (p.group % 2 == 0 || p.hq % 2 == 0) {
    const int64_t work = (int64_t)p.n_units * (p.hq / 2);
    const int g2 = (int)(work < grid ? work : grid);
    auto kern2 = p.group % 2 == 0 ? sap_fwd_pair_kernel<D, false, false> : sap_fwd_pair_kernel<D, false, true>;
    cudaError_t e =
        cudaFuncSetAttribute(kern2, cudaFuncAttributeMaxDynamicSharedMemorySize, Fwd2Cfg<D, false>::SMEM);
    if (e != cudaSuccess) return e;
    if (g2 > 0) kern2<<<g2, Fwd2Cfg<D, false>::THREADS, Fwd2Cfg<D, false>::SMEM, stream>>>(tq, tk, tv, p);
    return cudaGetLastError();
  }
  auto kern = sap_fwd_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, FwdCfg<D>::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<grid, FwdCfg<D>::THREADS, FwdCfg<D>::SMEM, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

template cudaError_t launch_fwd<64>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const FwdParams&,
                                    int, cudaStream_t, bool);
template cudaError_t launch_fwd<128>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const FwdParams&,
                                     int, cudaStream_t, bool);

}  // namespace sap
