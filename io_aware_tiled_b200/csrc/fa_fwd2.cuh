// fa_fwd2.cuh -- forward kernel on CTA pairs (2-SM tensor-core MMAs), d = 128.
//
// Same computation as fa_fwd.cuh (tiled attention with an online softmax:
// "FlashAttention分块计算优化Transformer显存效率", sections 1.1, 2.2, 3.2), laid
// out for the paired form of tcgen05.mma (cta_group::2):
//   * A cluster of two CTAs on two SMs works on 2 adjacent query tiles of one
//     head, one per CTA; one MMA instruction (M = 256) covers both.
//   * S_j = Q K_j^T: B = the key tile, split by keys: each CTA loads 64 of the
//     128 keys (all 128 columns).  O += P_j V_j: B = V_j, split by columns:
//     each CTA loads the 64 columns it contributes, for all 128 keys.  So every
//     CTA streams half of each K/V tile (16 KB + 16 KB per step).
//   * Tensor memory per CTA: three S buffers [0,128), [128,256), [256,384) and
//     O [384,512).  The leader CTA (rank 0) issues every MMA: S for two tiles
//     ahead of the softmax, then PV_j as soon as both CTAs have written P_j
//     (bf16, over S_j's columns).  So the softmax warpgroup of each CTA never
//     waits for its next S, and the tensor core runs PV_j and S_{j+3} while
//     the exponentials of S_{j+1} run.
//   * The leader commits to the barriers of both CTAs (multicast commit); each
//     CTA's loads complete on the leader's full barriers, which the leader
//     arms for both CTAs' bytes.  The softmax threads
//     of each CTA arrive on their own CTA's P and O-empty barriers (a remote
//     arrival costs hundreds of nanoseconds, too much for 128 threads on the
//     critical path); in CTA 1 a relay warp forwards each completed phase to
//     the leader with a single remote arrival.
//   * Softmax: two warpgroups per CTA split every row's 128 scores (64 each);
//     they exchange partial row maxima through shared memory once per step and
//     combine row sums only at the end.  Base 2; O (each warpgroup its half of
//     the columns) is rescaled only when a row max grows by more than a factor
//     2^rescale_log2 (8 by default), after waiting for the previous PV (an "O
//     done" barrier committed after every PV).  One exponential in 8 runs on
//     the FMA pipe (exp2_poly3).  The exponent arguments, the row sums and the
//     O rescale use the paired fp32 instructions (two values per instruction).
//   * A unit's Q tiles are released after its last S product, so the next
//     unit's Q loads while its last PVs run; the leader waits for the last
//     PV's V_EMPTY arrival before the teardown.
#pragma once

#include "fa_device.cuh"

namespace fa {

struct Fwd2Cfg {
  static constexpr int D = 128;
  static constexpr int BM = 128;                 // query rows per CTA
  static constexpr int BN = 128;                 // keys per K/V step
  static constexpr int CHUNK = 128 * 128;        // one 64-column chunk of a 128-row tile
  static constexpr int HCHUNK = 64 * 128;        // one 64-column chunk of a 64-row tile
  static constexpr int Q_TILE = BM * D * 2;      // 32 KB
  static constexpr int K_HALF = 64 * D * 2;      // 64 keys x 128 columns = 16 KB
  static constexpr int V_HALF = BN * 64 * 2;     // 128 keys x 64 columns = 16 KB
  static constexpr int ST = 5;                   // K and V ring depth
  static constexpr int NS = 3;                   // S buffers in tensor memory
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_TILE;
  static constexpr int OFF_V = OFF_K + ST * K_HALF;
  static constexpr int OFF_BAR = OFF_V + ST * V_HALF;
  static constexpr int B_Q_FULL = 0, B_Q_EMPTY = 1;
  static constexpr int B_K_FULL = 2, B_K_EMPTY = 2 + ST, B_V_FULL = 2 + 2 * ST, B_V_EMPTY = 2 + 3 * ST;
  static constexpr int B_S_FULL = 2 + 4 * ST, B_P_FULL = B_S_FULL + NS, B_O_DONE = B_P_FULL + NS,
                       B_O_EMPTY = B_O_DONE + 2;  // O_DONE[2]: PV of tile g commits to O_DONE[g % 2]
  static constexpr int NUM_BARS = B_O_EMPTY + 1;
  static constexpr int OFF_TMEM_SLOT = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_XCH = OFF_TMEM_SLOT + 16;  // max exchange [2 steps][2 halves][128] + sums [2][128]
  static constexpr int SMEM_BYTES = OFF_XCH + 6 * 128 * 4 + 1024;
  static constexpr uint32_t TM_O = 384;          // S buffer b at column 128 * b
  static constexpr uint32_t TMEM_COLS = 512;
  // warp 0 loads, warp 1 MMA (leader) or relay (peer), warps 4-7 and 8-11: the
  // softmax warpgroups of the low and the high 64 columns
  static constexpr int THREADS = 384;
  static constexpr int EXP_EMUL_EVERY = 5;  // 1/5 of the exponentials on the FMA pipe (exp2_poly3)
  static constexpr uint16_t BOTH = 0x3;          // multicast mask: both CTAs of the pair
};

enum Fwd2WaitSite : unsigned int {
  F2_PROD_Q = 80, F2_PROD_K, F2_PROD_V, F2_MMA_Q, F2_MMA_K, F2_MMA_V, F2_MMA_P, F2_MMA_OE, F2_SM_S, F2_SM_O
};

// Pair unit u covers query tiles 2*qp (rank 0) and 2*qp+1 (rank 1) of head bh.
// Non-causal: head-major (concurrent pairs share a few heads' K/V in L2),
// dealt in serpentine order.  Causal: numbered longest first across all
// heads; the host's per-pair lists (the one-SM kernel's unit lists, one
// worker per CTA pair: heads in L2-sized groups, longest first inside a
// group, longest-processing-time assignment) say which pair runs which.
__device__ __forceinline__ void fwd2_decode_unit(int u, int BH, int NQP, bool causal, int& bh, int& qp) {
  if (causal) {
    const int r = u / BH;
    bh = u - r * BH;
    qp = NQP - 1 - r;
  } else {
    bh = u / NQP;
    qp = u - bh * NQP;
  }
}

template <bool CAUSAL>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Fwd2Cfg::THREADS, 1)
    fa_fwd_2sm_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKh,
                      const __grid_constant__ CUtensorMap tmV, __nv_bfloat16* __restrict__ O,
                      float* __restrict__ LSE, int BH, int N, float scale_log2, float rescale_log2,
                      const __grid_constant__ typename UnitListOf<CAUSAL>::type list) {
  using C = Fwd2Cfg;
  constexpr int D = C::D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::OFF_Q, sK = sbase + C::OFF_K, sV = sbase + C::OFF_V;
  const uint32_t bars = sbase + C::OFF_BAR;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM_SLOT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  auto bar = [&](int i) { return bars + 8u * i; };                          // this CTA's barrier
  auto lead = [&](int i) { return map_shared_to_rank(bars + 8u * i, 0); };  // the leader's barrier

  if (threadIdx.x == 0) {
    // Full barriers (used on the leader): one local expect_tx arrival by the
    // leader for the bytes of BOTH CTAs; the peer's loads only complete bytes
    // on them (a remote arrival would cost the peer's producer ~1 us per tile).
    mbar_init(bar(C::B_Q_FULL), 1);
    mbar_init(bar(C::B_Q_EMPTY), 1);
    for (int s = 0; s < C::ST; ++s) {
      mbar_init(bar(C::B_K_FULL + s), 1);
      mbar_init(bar(C::B_K_EMPTY + s), 1);
      mbar_init(bar(C::B_V_FULL + s), 1);
      mbar_init(bar(C::B_V_EMPTY + s), 1);
    }
    // P and O-empty: the 256 local softmax threads, plus on the leader the
    // relay's one arrival for CTA 1
    const uint32_t cnt = rank == 0 ? 257u : 256u;
    for (int b = 0; b < C::NS; ++b) {
      mbar_init(bar(C::B_S_FULL + b), 1);
      mbar_init(bar(C::B_P_FULL + b), cnt);
    }
    mbar_init(bar(C::B_O_DONE + 0), 1);
    mbar_init(bar(C::B_O_DONE + 1), 1);
    mbar_init(bar(C::B_O_EMPTY), cnt);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmKh);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers and tensor memory exist before any cross-CTA use
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int NKT = (N + C::BN - 1) / C::BN;
  const int NQT = (N + C::BM - 1) / C::BM;
  const int NQP = (NQT + 1) / 2;
  const int units = BH * NQP;

  if (warp == 0) {
    // ------------------------------------------------------------ loads (both CTAs)
    if (lane == 0) {
      uint32_t kv_it = 0, q_it = 0;
      for (int k = 0, u = worker_unit(list, 0, units, pair, npairs); u < units; u = worker_unit(list, ++k, units, pair, npairs)) {
        int bh, qp;
        fwd2_decode_unit(u, BH, NQP, CAUSAL, bh, qp);
        const int nk = CAUSAL ? min(2 * qp + 2, NKT) : NKT;
        if (!mbar_wait_cluster(bar(C::B_Q_EMPTY), (q_it & 1) ^ 1, F2_PROD_Q)) break;
        ++q_it;
        if (rank == 0) mbar_arrive_expect_tx(bar(C::B_Q_FULL), 2 * C::Q_TILE);
        for (int c = 0; c < 2; ++c)
          tma_load_3d_pair(sQ + c * C::CHUNK, &tmQ, lead(C::B_Q_FULL), c * 64, (2 * qp + rank) * C::BM, bh);
        bool ok = true;
        for (int j = 0; j < nk; ++j, ++kv_it) {
          const int s = kv_it % C::ST;
          const uint32_t ph = (kv_it / C::ST) & 1;
          if (!mbar_wait_cluster(bar(C::B_K_EMPTY + s), ph ^ 1, F2_PROD_K)) { ok = false; break; }
          if (rank == 0) mbar_arrive_expect_tx(bar(C::B_K_FULL + s), 2 * C::K_HALF);
          for (int c = 0; c < 2; ++c)  // keys j*128 + 64*rank .. +63, both column chunks
            tma_load_3d_pair(sK + s * C::K_HALF + c * C::HCHUNK, &tmKh, lead(C::B_K_FULL + s), c * 64,
                             j * C::BN + 64 * rank, bh);
          if (!mbar_wait_cluster(bar(C::B_V_EMPTY + s), ph ^ 1, F2_PROD_V)) { ok = false; break; }
          if (rank == 0) mbar_arrive_expect_tx(bar(C::B_V_FULL + s), 2 * C::V_HALF);
          // columns 64*rank .. +63 of keys j*128 .. +127
          tma_load_3d_pair(sV + s * C::V_HALF, &tmV, lead(C::B_V_FULL + s), 64 * rank, j * C::BN, bh);
        }
        if (!ok) break;
      }
    }
  } else if (warp == 1 && rank == 0) {
    // ------------------------------------------------------------ MMA issuer (leader CTA only)
    constexpr uint32_t IDESC_S = idesc_bf16(256, 128, false, false);
    constexpr uint32_t IDESC_PV = idesc_bf16(256, D, false, true);
    const uint32_t hi = sdesc_hi(1024);
    // s_it counts this CTA pair's S tiles; tile g lives in buffer g % NS, and
    // each buffer's barriers complete once per use, in order, so the phase of
    // tile g's wait is (g / NS) & 1.
    uint32_t kv_it = 0, q_it = 0, unit_it = 0, s_it = 0;
    bool ok = true;
    // S for the key tile of global step `it` into buffer `b`.
    auto issue_s = [&](uint32_t it, int b) -> bool {
      const int s = it % C::ST;
      if (!__all_sync(0xffffffffu, mbar_wait_cluster(bar(C::B_K_FULL + s), (it / C::ST) & 1, F2_MMA_K))) return false;
      tc_fence_after();
      const uint32_t b_smem = sK + s * C::K_HALF;
      mma2_ss_k128(tmem + 128 * b, sdesc_make(sdesc_lo(sQ, 16), hi), sdesc_make(sdesc_lo(sQ + C::CHUNK, 16), hi),
                   sdesc_make(sdesc_lo(b_smem, 16), hi), sdesc_make(sdesc_lo(b_smem + C::HCHUNK, 16), hi), IDESC_S,
                   0u);
      tc_commit_pair_warp(bar(C::B_S_FULL + b), C::BOTH);
      tc_commit_pair_warp(bar(C::B_K_EMPTY + s), C::BOTH);
      return true;
    };
    for (int k = 0, u = worker_unit(list, 0, units, pair, npairs); u < units && ok; u = worker_unit(list, ++k, units, pair, npairs), ++unit_it) {
      int bh, qp;
      fwd2_decode_unit(u, BH, NQP, CAUSAL, bh, qp);
      (void)bh;
      const int nk = CAUSAL ? min(2 * qp + 2, NKT) : NKT;
      if (!(ok = __all_sync(0xffffffffu, mbar_wait_cluster(bar(C::B_Q_FULL), q_it & 1, F2_MMA_Q)))) break;
      ++q_it;
      tc_fence_after();
      const uint32_t s_base = s_it;  // buffer of this unit's tile j is (s_base + j) % NS
      // after the unit's last S its Q half is free for the next unit's loads
      // (the PVs still to come do not read Q)
      for (int j = 0; j < nk && j < C::NS && ok; ++j) {
        ok = issue_s(kv_it + j, (s_base + j) % C::NS);
        if (ok && j == nk - 1) tc_commit_pair_warp(bar(C::B_Q_EMPTY), C::BOTH);
      }
      for (int j = 0; j < nk && ok; ++j) {
        const uint32_t it = kv_it + j;
        const int s = it % C::ST, b = (s_base + j) % C::NS;
        if (!(ok = __all_sync(0xffffffffu,
                                 mbar_wait_cluster(bar(C::B_P_FULL + b), ((s_base + j) / C::NS) & 1, F2_MMA_P))))
          break;
        if (j == 0 && !(ok = __all_sync(0xffffffffu, mbar_wait_cluster(bar(C::B_O_EMPTY), (unit_it & 1) ^ 1,
                                                                         F2_MMA_OE))))
          break;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait_cluster(bar(C::B_V_FULL + s), (it / C::ST) & 1, F2_MMA_V))))
          break;
        tc_fence_after();
        mma2_ts_k128(tmem + C::TM_O, tmem + 128 * b, sdesc_make(sdesc_lo(sV + s * C::V_HALF, C::CHUNK), hi),
                     IDESC_PV, j > 0 ? 1u : 0u);
        tc_commit_pair_warp(bar(C::B_O_DONE + ((s_base + j) & 1)), C::BOTH);
        tc_commit_pair_warp(bar(C::B_V_EMPTY + s), C::BOTH);
        if (j + C::NS < nk) {
          ok = issue_s(it + C::NS, b);  // buffer b is free once PV_j has read P_j
          if (ok && j + C::NS == nk - 1) tc_commit_pair_warp(bar(C::B_Q_EMPTY), C::BOTH);
        }
      }
      if (!ok) break;
      kv_it += nk;
      s_it += nk;
    }
    // The last PV's V_EMPTY arrival is the last one the commits make (the
    // unit's Q_EMPTY went out after its last S); wait for it here, so none
    // lands after the teardown.
    if (ok && kv_it > 0)
      (void)__all_sync(0xffffffffu, mbar_wait_cluster(bar(C::B_V_EMPTY + (kv_it - 1) % C::ST),
                                                     ((kv_it - 1) / C::ST) & 1, F2_MMA_V));
  } else if (warp == 1) {
    // ------------------------------------------------------------ relay (CTA 1)
    // Forwards each completed phase of CTA 1's P and O-empty barriers to the
    // leader's, one remote arrival per phase.
    if (lane == 0) {
      uint32_t g = 0, unit_it = 0;
      for (int k = 0, u = worker_unit(list, 0, units, pair, npairs); u < units; u = worker_unit(list, ++k, units, pair, npairs), ++unit_it) {
        int bh, qp;
        fwd2_decode_unit(u, BH, NQP, CAUSAL, bh, qp);
        (void)bh;
        const int nk = CAUSAL ? min(2 * qp + 2, NKT) : NKT;
        bool ok = true;
        for (int j = 0; j < nk; ++j, ++g) {
          const int b = g % C::NS;
          if (!(ok = mbar_wait_cluster(bar(C::B_P_FULL + b), (g / C::NS) & 1, F2_MMA_P))) break;
          // carry the softmax threads' tensor-memory stores across this thread
          tc_fence_after();
          tc_fence_before();
          mbar_arrive_cluster(lead(C::B_P_FULL + b));
        }
        if (!ok || !mbar_wait_cluster(bar(C::B_O_EMPTY), unit_it & 1, F2_MMA_OE)) break;
        tc_fence_after();
        tc_fence_before();
        mbar_arrive_cluster(lead(C::B_O_EMPTY));
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax warpgroups (both CTAs)
    const int h = (warp - 4) >> 2;           // which 64 of the 128 columns
    const int sp = warp & 3;
    const int r = sp * 32 + lane;            // the row (TMEM lane) this thread shares with its partner
    const uint32_t lane_off = static_cast<uint32_t>(sp * 32) << 16;
    const uint32_t tO = tmem + lane_off + C::TM_O + 64 * h;  // this warpgroup's half of O
    float* xch = reinterpret_cast<float*>(smem + C::OFF_XCH);
    float* xmax = xch;                        // [step & 1][half][row]
    float* xsum = xch + 4 * 128;              // [half][row]
    uint32_t s_it = 0;
    bool ok = true;
    for (int k = 0, u = worker_unit(list, 0, units, pair, npairs); u < units && ok; u = worker_unit(list, ++k, units, pair, npairs)) {
      int bh, qp;
      fwd2_decode_unit(u, BH, NQP, CAUSAL, bh, qp);
      const int qt = 2 * qp + static_cast<int>(rank);
      const int nk = CAUSAL ? min(2 * qp + 2, NKT) : NKT;
      const int row = qt * C::BM + r;
      float m_ref = -INFINITY, l = 0.f;  // l: this thread's partial row sum
      for (int j = 0; j < nk; ++j) {
        const uint32_t g = s_it;  // global tile index of this CTA pair
        const int b = g % C::NS;
        const uint32_t sph = (g / C::NS) & 1;
        ++s_it;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait_cluster(bar(C::B_S_FULL + b), sph, F2_SM_S)))) break;
        tc_fence_after();
        const uint32_t tS = tmem + lane_off + 128 * b;
        uint32_t sr[64];
        tmem_ld32(tS + 64 * h, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(tS + 64 * h + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_ld_wait();
        reg_fence(*reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        reg_fence(*reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        float s[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) s[c] = __uint_as_float(sr[c]);
        const int kbase = j * C::BN + 64 * h;
        if ((CAUSAL && j * C::BN + C::BN - 1 > qt * C::BM) || j * C::BN + C::BN > N) {
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const int key = kbase + c;
            if (key >= N || (CAUSAL && key > row)) s[c] = -INFINITY;
          }
        }
        const float pmax = row_max<64>(s);
        // Row max across the two halves.  The exchange slot alternates with the
        // step, so a slot is rewritten only after the partner has passed the
        // next barrier, i.e. after it read this step's value.  Both halves
        // then hold the same max, hence the same m and rescale decisions.
        float* slot = xmax + (j & 1) * 256;
        slot[h * 128 + r] = pmax;
        named_bar_sync(1, 256);
        const float mx = fmaxf(pmax, slot[(1 - h) * 128 + r]);
        // Both halves have loaded their S before that barrier, so from here on
        // P may be written over S's columns.
        const float m_new = fmaxf(m_ref, mx * scale_log2);
        const bool need = m_new > m_ref + rescale_log2;
        const bool warp_rescale = __any_sync(0xffffffffu, need);
        const float alpha = need ? ex2(m_ref - m_new) : 1.f;  // ex2(-inf) = 0 on the first tile
        if (need) {
          l *= alpha;
          m_ref = m_new;
        }
        // a row whose keys so far are all masked keeps m = -inf and P = 0
        const float neg = (m_ref == -INFINITY) ? 0.f : -m_ref;
        // pairs of scores through the paired fp32 instructions (one FMA and one
        // add for two elements); 4 x 2 independent partial row sums
        const uint64_t sc2 = f2_make(scale_log2, scale_log2), ng2 = f2_make(neg, neg);
        uint64_t ps2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t p[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            float t0, t1;
            f2_split(f2_fma(f2_make(s[32 * ch + 2 * c], s[32 * ch + 2 * c + 1]), sc2, ng2), t0, t1);
            const bool emul = c % C::EXP_EMUL_EVERY == C::EXP_EMUL_EVERY - 1;  // resolved at compile time
            const float p0 = emul ? exp2_poly3(t0) : ex2(t0);
            const float p1 = emul ? exp2_poly3(t1) : ex2(t1);
            ps2[c & 3] = f2_add(ps2[c & 3], f2_make(p0, p1));
            p[c] = pack_bf16(p0, p1);
          }
          tmem_st16(tS + 32 * h + ch * 16, p);  // keys 64h.. -> packed columns 32h..
        }
        float ps[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) f2_split(ps2[e], ps[2 * e], ps[2 * e + 1]);
#pragma unroll
        for (int w = 4; w > 0; w >>= 1)
#pragma unroll
          for (int e = 0; e < w; ++e) ps[e] += ps[e + w];
        // Tile g's PV commits to O_DONE[g % 2], whose phase for it is (g / 2) & 1.
        // Only a rescale (and the epilogue) needs a PV to be complete; step j
        // (global tile g) then waits for the PV of tile g-1.  A parity test of
        // phase k is exact while its barrier has completed k or k+1 phases: the
        // PV two tiles back on that barrier (tile g-3) is complete because S of
        // tile g, already seen complete, was issued after it, and the next PV
        // on that barrier needs tile g+1's P, which this CTA has not produced.
        if (j >= 1 && warp_rescale) {
          const uint32_t gp = g - 1;
          ok = __all_sync(0xffffffffu, mbar_wait_cluster(bar(C::B_O_DONE + (gp & 1)), (gp >> 1) & 1, F2_SM_O));
        }
        if (!ok) break;
        if (j > 0 && warp_rescale) {
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + c * 32, o);
            tmem_ld_wait();
            reg_fence(o);
            scale32(o, alpha);
            tmem_st32(tO + c * 32, o);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar(C::B_P_FULL + b));
        l += ps[0];
      }
      if (!ok) break;
      // epilogue: the unit's last PV.  A parity test of phase k is exact only
      // while its barrier has completed k or k+1 phases.  The PV before the
      // previous one (tile g-3) is complete since S of tile g was issued after
      // it, so first wait for tile g-1's PV (the other barrier), which makes
      // tile g-2's PV complete too, then for tile g's.
      {
        const uint32_t gl = s_it - 1;
        ok = __all_sync(0xffffffffu, mbar_wait_cluster(bar(C::B_O_DONE + ((gl - 1) & 1)), ((gl - 1) >> 1) & 1, F2_SM_O));
        ok = ok && __all_sync(0xffffffffu, mbar_wait_cluster(bar(C::B_O_DONE + (gl & 1)), (gl >> 1) & 1, F2_SM_O));
        if (!ok) break;
      }
      tc_fence_after();
      xsum[h * 128 + r] = l;
      named_bar_sync(1, 256);
      const float l_row = l + xsum[(1 - h) * 128 + r];
      const float inv_l = 1.f / l_row;
      __nv_bfloat16* orow = O + (static_cast<size_t>(bh) * N + row) * D + 64 * h;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + c * 32, o);
        tmem_ld_wait();
        reg_fence(o);
        if (row < N) store_bf16x32(orow + c * 32, o, inv_l);
      }
      if (h == 0 && row < N) LSE[static_cast<size_t>(bh) * N + row] = (m_ref + __log2f(l_row)) * kLn2;
      tc_fence_before();
      mbar_arrive(bar(C::B_O_EMPTY));
    }
  }

  // teardown: every thread of both CTAs
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the leader's MMAs into this CTA's tensor memory are complete
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, C::TMEM_COLS);
  }
}

}  // namespace fa
