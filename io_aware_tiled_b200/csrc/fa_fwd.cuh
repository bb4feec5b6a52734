// fa_fwd.cuh -- forward kernel of tiled, IO-aware exact attention for sm_100a.
//
// What it computes (per head, per query row i):
//   S_ij = scale * q_i . k_j, masked (causal: j > i; ragged tail: j >= N),
//   O_i  = sum_j softmax(S_i)_j v_j,   LSE_i = ln sum_j exp(S_ij),
// tile by tile, so the N x N S and P never leave the SM
// ("FlashAttention分块计算优化Transformer显存效率", section 1.1 tiled loop;
// section 3.2 online softmax: running max m, running sum l, the partial O
// rescaled by exp(m_old - m_new); section 2.2 causal block skipping with
// masking only on the diagonal blocks).  The final O = O_partial / l and the
// stored statistic LSE = m + ln l are the completion of section 3.2 that makes
// the result equal the global softmax ("图解Flash Attention运算原理", 分块 Softmax).
//
// B200 design (what differs from the pages' A100-era sizing):
//   * One persistent CTA per SM; a work unit is a PAIR of 128-row Q tiles of
//     one (batch, head).  Two softmax warpgroups (one per Q tile) alternate, so
//     the tensor core computes one tile's S or PV while the other tile's
//     exponentials run.
//   * Three warpgroups: the control warpgroup gives registers back
//     (setmaxnreg) to the two softmax warpgroups, which hold a full S row each.
//   * Warp 0 issues TMA loads: Q pair once per unit, K_j and V_j through
//     separate rings of ST stages (128 keys x d, 128-byte swizzle).  At
//     d = 64 shared memory holds two Q pairs, so the next unit's Q arrives
//     while the current unit still runs (NQB buffers).
//   * Warp 1 issues tcgen05.mma from one thread: S_t = Q_t K_j^T (M=128,
//     N=128, K=d, both operands K-major in shared memory) into tensor memory,
//     and O_t += P_t V_j (M=128, N=d, K=128) with P_t read from TENSOR MEMORY
//     (bf16, written over S_t's columns) and V_j MN-major from shared memory.
//   * Tensor memory (512 columns x 128 lanes x 32 bit): S0 [0,128), S1
//     [128,256), O0 [256, 256+d), O1 [256+d, 256+2d).  At d = 128 S_t is Q
//     tile t's buffer: a tile's next S waits until its PV has read P.  At
//     d = 64 the free columns [384,512) hold a third buffer S2 and the three
//     form a ring over the unit's tiles in issue order, so a Q tile's next S
//     is computed while its softmax still runs; before rescaling O the
//     softmax then waits for its previous PV (an O_DONE barrier per Q tile
//     and PV-count parity).
//   * Softmax: each thread owns one full row of S (tcgen05.ld 32x32b), so the
//     row max and row sum are register reductions.  Work is in base 2 with
//     scale*log2(e) folded into one FMA, issued for two scores at a time
//     (fma.rn.f32x2; the row sum and the O rescale use the paired add and
//     multiply too).  O is rescaled only when a row's max grows by more than
//     a factor 2^rescale_log2 (8 by default; exact: the final division uses
//     the same max).  A fixed share of the exponentials runs on the FMA pipe
//     (exp2_poly3_x2, two at a time), the rest on the MUFU.
//   * Epilogue: O / l as bf16 and LSE as fp32, stored once per row (32-byte
//     stores where the rows are 32-byte aligned).
//   * With one Q buffer (d = 128) a unit's Q pair is released after its last
//     S product, so the next unit's Q loads while its last PVs run.
#pragma once

#include "fa_device.cuh"

namespace fa {

template <int D, int BN_ = 128>
struct FwdCfg {
  static constexpr int BM = 128;                 // query rows per Q tile
  static constexpr int BN = BN_;                 // keys per K/V tile: 128, or 64 (tile-size comparisons)
  static constexpr int R = BM / BN;              // key tiles per query tile's width
  static constexpr int CH = D / 64;              // 128-byte column chunks per row
  static constexpr int CHUNK = 128 * 128;        // bytes of one 64-column chunk of a 128-row Q tile
  static constexpr int KV_CHUNK = BN * 128;      // bytes of one 64-column chunk of a K or V tile
  static constexpr int Q_TILE = BM * D * 2;
  static constexpr int KV_TILE = BN * D * 2;
  static constexpr int ST = ((D == 128) ? 2 : 4) * R;  // K and V ring depth (same bytes for either BN)
  static constexpr int NQB = (D == 64) ? 2 : 1;  // Q-pair buffers (the next unit's Q loads early)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + NQB * 2 * Q_TILE;
  static constexpr int OFF_V = OFF_K + ST * KV_TILE;
  static constexpr int OFF_BAR = OFF_V + ST * KV_TILE;
  // barrier indices
  static constexpr int B_Q_FULL = 0, B_Q_EMPTY = NQB;
  static constexpr int B_K_FULL = 2 * NQB, B_K_EMPTY = 2 * NQB + ST, B_V_FULL = 2 * NQB + 2 * ST,
                       B_V_EMPTY = 2 * NQB + 3 * ST;
  // S buffers: two (one per Q tile) at d = 128; at d = 64 with 128-key tiles
  // a ring of three over the unit's tiles in issue order (the spare tensor
  // memory after O0 and O1 holds the third)
  static constexpr int NS = (D == 64 && BN == 128) ? 3 : 2;
  static constexpr int B_S_FULL = 2 * NQB + 4 * ST, B_P_FULL = B_S_FULL + NS, B_O_FULL = B_P_FULL + NS,
                       B_O_EMPTY = B_O_FULL + 2, B_O_DONE = B_O_EMPTY + 2;  // O_DONE: [Q tile][PV count & 1]
  static constexpr int NUM_BARS = B_O_DONE + 4;
  static constexpr int OFF_TMEM_SLOT = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_TMEM_SLOT + 16 + 1024;  // + room to align the base to 1024
  static constexpr uint32_t TM_S0 = 0, TM_S1 = BN, TM_O0 = 256, TM_O1 = 256 + D, TM_S2 = 384;
  static_assert(NS == 2 || TM_O1 + D <= TM_S2, "third S buffer overlaps O");
  __host__ __device__ static constexpr uint32_t tm_s(int b) { return b == 0 ? TM_S0 : (b == 1 ? TM_S1 : TM_S2); }
  static constexpr uint32_t TMEM_COLS = 512;
  // warpgroup 0: warp 0 TMA, warp 1 MMA, warps 2-3 idle; warpgroups 1 and 2: softmax of Q tile 0 and 1
  static constexpr int THREADS = 384;
  // register split (launch: 384 threads x 168 = 64512): control warpgroup 64,
  // softmax warpgroups 208 each (128 x 64 + 256 x 208 = 61440)
  static constexpr uint32_t REGS_CONTROL = 64, REGS_SOFTMAX = 208;
  // one exponential pair in EXP_EMUL_EVERY goes to exp2_poly3 (FMA pipe)
  // instead of the MUFU: 1/16 of them at d = 64 (with the S ring the
  // softmax's issue slots, not the MUFU, bound it), 1/4 at d = 128 (measured
  // best under sustained load at the power limit, and no worse in isolated calls)
  static constexpr int EXP_EMUL_EVERY = (D == 64) ? 16 : 4;
};

// wait-site identifiers recorded in the error word
enum FwdWaitSite : unsigned int {
  FW_PROD_Q = 1, FW_PROD_K, FW_PROD_V, FW_MMA_Q, FW_MMA_K, FW_MMA_V, FW_MMA_P, FW_MMA_OE, FW_SM_S, FW_SM_O
};

// Unit order.  Non-causal: head-major, so the CTAs running at the same time
// share a few heads' K and V in L2, dealt in serpentine order.  Causal: unit u
// is rank u / BH (0 = the longest, the last query pair) of head u % BH; the
// host gives each CTA its list of units (FwdUnitList): heads in groups whose K
// and V fit in L2, longest units first inside a group, each unit assigned to
// the CTA with the least work so far.  A static deal of that grouped order
// would leave some CTAs with far more work; the assignment keeps both the
// balance of a global longest-first deal and the L2 locality of the groups.
// Without a list (more units or CTAs than it holds) the causal units are
// dealt longest first, in serpentine order.
__device__ __forceinline__ void fwd_decode_unit(int u, int BH, int NP, bool causal, int& bh, int& qp) {
  if (causal) {
    const int r = u / BH;
    bh = u - r * BH;
    qp = NP - 1 - r;
  } else {
    bh = u / NP;
    qp = u - bh * NP;
  }
}

// Order of a unit's tiles in the S-buffer ring (three buffers, d = 64): key
// tile j of Q tile 0, then key tile j of Q tile 1, for j < nk0; then Q tile 1
// alone for its last nk1 - nk0 key tiles (causal).  Tile i of a CTA's whole
// sequence uses buffer i % 3.
__device__ __forceinline__ int ring_pos(int j, int t, int nk0) { return j < nk0 ? 2 * j + t : nk0 + j; }
__device__ __forceinline__ void ring_tile(int i, int nk0, int& j, int& t) {
  if (i < 2 * nk0) {
    j = i >> 1;
    t = i & 1;
  } else {
    j = i - nk0;
    t = 1;
  }
}

// Per-CTA unit lists of the causal forward (UnitList): unit indices as
// fwd_decode_unit reads them; none without the mask.
using FwdUnitList = UnitList;
using FwdNoList = NoUnitList;
template <bool CAUSAL>
using FwdListOf = UnitListOf<CAUSAL>;

// The k-th unit of this CTA (>= units when it has no more).
template <typename L>
__device__ __forceinline__ int fwd_unit(const L& list, int k, int units) {
  return list_unit(list, k, units);
}

template <int D, bool CAUSAL, int BN_ = 128>
__global__ void __launch_bounds__(FwdCfg<D, BN_>::THREADS, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, __nv_bfloat16* __restrict__ O,
                  float* __restrict__ LSE, int BH, int N, float scale_log2,
                  float rescale_log2, const __grid_constant__ typename FwdListOf<CAUSAL>::type list) {
  using C = FwdCfg<D, BN_>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::OFF_Q, sK = sbase + C::OFF_K, sV = sbase + C::OFF_V;
  const uint32_t bars = sbase + C::OFF_BAR;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM_SLOT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int qb = 0; qb < C::NQB; ++qb) {
      mbar_init(bars + 8 * (C::B_Q_FULL + qb), 1);
      mbar_init(bars + 8 * (C::B_Q_EMPTY + qb), 1);
    }
    for (int s = 0; s < C::ST; ++s) {
      mbar_init(bars + 8 * (C::B_K_FULL + s), 1);
      mbar_init(bars + 8 * (C::B_K_EMPTY + s), 1);
      mbar_init(bars + 8 * (C::B_V_FULL + s), 1);
      mbar_init(bars + 8 * (C::B_V_EMPTY + s), 1);
    }
    for (int b = 0; b < C::NS; ++b) {
      mbar_init(bars + 8 * (C::B_S_FULL + b), 1);
      mbar_init(bars + 8 * (C::B_P_FULL + b), 128);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bars + 8 * (C::B_O_FULL + t), 1);
      mbar_init(bars + 8 * (C::B_O_EMPTY + t), 128);
      mbar_init(bars + 8 * (C::B_O_DONE + 2 * t), 1);
      mbar_init(bars + 8 * (C::B_O_DONE + 2 * t + 1), 1);
    }
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int NKT = (N + C::BN - 1) / C::BN;  // key tiles
  const int NQT = (N + C::BM - 1) / C::BM;  // query tiles
  const int NP = (NQT + 1) / 2;             // query tile pairs
  const int units = BH * NP;

  // Each role's setmaxnreg dominates that role's code, and the paths join only
  // at the teardown, so the compiler gives each region its own register limit.
  if (warp < 4) {
    regs_dec<C::REGS_CONTROL>();
    if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t kv_it = 0, q_it = 0;
      for (int k = 0, u = fwd_unit(list, 0, units); u < units; u = fwd_unit(list, ++k, units)) {
        int bh, qp;
        fwd_decode_unit(u, BH, NP, CAUSAL, bh, qp);
        const int nk1 = CAUSAL ? min((2 * qp + 2) * C::R, NKT) : NKT;
        const int qb = q_it % C::NQB;
        if (!mbar_wait(bars + 8 * (C::B_Q_EMPTY + qb), ((q_it / C::NQB) & 1) ^ 1, FW_PROD_Q)) break;
        ++q_it;
        mbar_arrive_expect_tx(bars + 8 * (C::B_Q_FULL + qb), 2 * C::Q_TILE);
        for (int t = 0; t < 2; ++t)
          for (int c = 0; c < C::CH; ++c)
            tma_load_3d(sQ + (qb * 2 + t) * C::Q_TILE + c * C::CHUNK, &tmQ, bars + 8 * (C::B_Q_FULL + qb), c * 64,
                        (2 * qp + t) * C::BM, bh);
        bool ok = true;
        for (int j = 0; j < nk1; ++j, ++kv_it) {
          const int s = kv_it % C::ST;
          const uint32_t ph = (kv_it / C::ST) & 1;
          if (!mbar_wait(bars + 8 * (C::B_K_EMPTY + s), ph ^ 1, FW_PROD_K)) { ok = false; break; }
          mbar_arrive_expect_tx(bars + 8 * (C::B_K_FULL + s), C::KV_TILE);
          for (int c = 0; c < C::CH; ++c)
            tma_load_3d(sK + s * C::KV_TILE + c * C::KV_CHUNK, &tmK, bars + 8 * (C::B_K_FULL + s), c * 64,
                        j * C::BN, bh);
          if (!mbar_wait(bars + 8 * (C::B_V_EMPTY + s), ph ^ 1, FW_PROD_V)) { ok = false; break; }
          mbar_arrive_expect_tx(bars + 8 * (C::B_V_FULL + s), C::KV_TILE);
          for (int c = 0; c < C::CH; ++c)
            tma_load_3d(sV + s * C::KV_TILE + c * C::KV_CHUNK, &tmV, bars + 8 * (C::B_V_FULL + s), c * 64,
                        j * C::BN, bh);
        }
        if (!ok) break;
      }
    }
    } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop with warp-uniform values; one elected lane
    // issues each tcgen05.mma / commit.
    {
      constexpr uint32_t IDESC_S = idesc_bf16(128, C::BN, false, false);
      constexpr uint32_t IDESC_PV = idesc_bf16(128, D, false, true);
      // S = Q_t K_j^T: K = d in steps of 16 (one 8- or 4-MMA group).
      auto issue_s = [&](uint32_t d_tmem, uint32_t a_smem, uint32_t b_smem) {
        const uint32_t hi = sdesc_hi(1024);
        const uint64_t a0 = sdesc_make(sdesc_lo(a_smem, 16), hi), b0 = sdesc_make(sdesc_lo(b_smem, 16), hi);
        if (D == 128)
          mma_ss_k128(d_tmem, a0, sdesc_make(sdesc_lo(a_smem + C::CHUNK, 16), hi), b0,
                      sdesc_make(sdesc_lo(b_smem + C::KV_CHUNK, 16), hi), IDESC_S, 0u);
        else
          mma_ss_k64(d_tmem, a0, b0, IDESC_S, 0u);
      };
      // O_t += P_t V_j: BN/16 steps of 16 keys; P_t from tensor memory, V_j MN-major.
      auto issue_pv = [&](uint32_t d_tmem, uint32_t p_tmem, uint32_t v_smem, bool acc) {
        const uint64_t vd = sdesc_make(sdesc_lo(v_smem, C::KV_CHUNK), sdesc_hi(1024));
        if (C::BN == 128)
          mma_ts_k128(d_tmem, p_tmem, vd, IDESC_PV, acc ? 1u : 0u);
        else
          mma_ts_k64(d_tmem, p_tmem, vd, IDESC_PV, acc ? 1u : 0u);
      };
      uint32_t kv_it = 0, q_it = 0, unit_it = 0;
      if constexpr (C::NS == 3) {
        // Ring of three S buffers: after PV of tile i the MMA of tile i + 3
        // goes into the buffer P_i occupied, so each Q tile's next S is ready
        // while its softmax still runs.
        uint32_t g0 = 0, pv0 = 0, pv1 = 0;  // ring tiles before this unit; PVs issued per Q tile
        for (int k = 0, u = fwd_unit(list, 0, units); u < units; u = fwd_unit(list, ++k, units), ++unit_it) {
          int bh, qp;
          fwd_decode_unit(u, BH, NP, CAUSAL, bh, qp);
          (void)bh;
          const int nk0 = CAUSAL ? min((2 * qp + 1) * C::R, NKT) : NKT;
          const int nk1 = CAUSAL ? min((2 * qp + 2) * C::R, NKT) : NKT;
          const int n = nk0 + nk1;
          const int qb = q_it % C::NQB;
          const uint32_t sQb = sQ + qb * 2 * C::Q_TILE;
          bool ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * (C::B_Q_FULL + qb), (q_it / C::NQB) & 1, FW_MMA_Q));
          ++q_it;
          if (!ok) break;
          tc_fence_after();
          // S of the unit's ring tile i into its buffer; K_j is free after Q tile 1's S
          auto s_of = [&](int i) -> bool {
            int j, t;
            ring_tile(i, nk0, j, t);
            const uint32_t it = kv_it + j;
            const int s = it % C::ST;
            if (!__all_sync(0xffffffffu, mbar_wait(bars + 8 * (C::B_K_FULL + s), (it / C::ST) & 1, FW_MMA_K)))
              return false;
            tc_fence_after();
            const int b = (g0 + i) % C::NS;
            issue_s(tmem + C::tm_s(b), sQb + t * C::Q_TILE, sK + s * C::KV_TILE);
            tc_commit_warp(bars + 8 * (C::B_S_FULL + b));
            if (t == 1) tc_commit_warp(bars + 8 * (C::B_K_EMPTY + s));
            return true;
          };
          for (int i = 0; i < n && i < C::NS && ok; ++i) ok = s_of(i);
          for (int i = 0; i < n && ok; ++i) {
            int j, t;
            ring_tile(i, nk0, j, t);
            const uint32_t it = kv_it + j, g = g0 + i;
            const int s = it % C::ST, b = g % C::NS;
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * (C::B_V_FULL + s), (it / C::ST) & 1, FW_MMA_V))))
              break;
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * (C::B_P_FULL + b), (g / C::NS) & 1, FW_MMA_P))))
              break;
            if (j == 0 && !(ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * (C::B_O_EMPTY + t), (unit_it & 1) ^ 1,
                                                                     FW_MMA_OE))))
              break;
            tc_fence_after();
            issue_pv(tmem + (t ? C::TM_O1 : C::TM_O0), tmem + C::tm_s(b), sV + s * C::KV_TILE, j > 0);
            const uint32_t pc = t ? pv1 : pv0;
            tc_commit_warp(bars + 8 * (C::B_O_DONE + 2 * t + (pc & 1)));
            if (t) ++pv1; else ++pv0;
            if (t == 1) tc_commit_warp(bars + 8 * (C::B_V_EMPTY + s));
            if (j == (t ? nk1 : nk0) - 1) tc_commit_warp(bars + 8 * (C::B_O_FULL + t));
            if (i + C::NS < n) ok = s_of(i + C::NS);
          }
          if (!ok) break;
          // (two Q pairs: the next unit's is already loaded, so the release
          // can wait for the unit's end)
          tc_commit_warp(bars + 8 * (C::B_Q_EMPTY + qb));
          kv_it += nk1;
          g0 += n;
        }
      } else {
      uint32_t p_ph0 = 0, p_ph1 = 0;
      for (int k = 0, u = fwd_unit(list, 0, units); u < units; u = fwd_unit(list, ++k, units), ++unit_it) {
        int bh, qp;
        fwd_decode_unit(u, BH, NP, CAUSAL, bh, qp);
        (void)bh;
        const int nk0 = CAUSAL ? min((2 * qp + 1) * C::R, NKT) : NKT;
        const int nk1 = CAUSAL ? min((2 * qp + 2) * C::R, NKT) : NKT;
        const int qb = q_it % C::NQB;
        const uint32_t sQb = sQ + qb * 2 * C::Q_TILE;
        bool ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * (C::B_Q_FULL + qb), (q_it / C::NQB) & 1, FW_MMA_Q));
        ++q_it;
        if (!ok) break;
        tc_fence_after();
        {
          const int s = kv_it % C::ST;
          if (!__all_sync(0xffffffffu, mbar_wait(bars + 8 * (C::B_K_FULL + s), (kv_it / C::ST) & 1, FW_MMA_K))) break;
          tc_fence_after();
          issue_s(tmem + C::TM_S0, sQb, sK + s * C::KV_TILE);
          tc_commit_warp(bars + 8 * (C::B_S_FULL + 0));
          issue_s(tmem + C::TM_S1, sQb + C::Q_TILE, sK + s * C::KV_TILE);
          tc_commit_warp(bars + 8 * (C::B_S_FULL + 1));
          tc_commit_warp(bars + 8 * (C::B_K_EMPTY + s));
          if (nk1 == 1) tc_commit_warp(bars + 8 * (C::B_Q_EMPTY + qb));  // no further S reads the Q pair
        }
        for (int j = 0; j < nk1 && ok; ++j) {
          const uint32_t it = kv_it + j;
          const int s = it % C::ST;
          const bool more = j + 1 < nk1;
          const int sn = (it + 1) % C::ST;
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * (C::B_V_FULL + s), (it / C::ST) & 1, FW_MMA_V)))) break;
          if (more && !(ok = __all_sync(0xffffffffu,
                                        mbar_wait(bars + 8 * (C::B_K_FULL + sn), ((it + 1) / C::ST) & 1, FW_MMA_K))))
            break;
          tc_fence_after();
          if (j < nk0) {
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * (C::B_P_FULL + 0), p_ph0, FW_MMA_P)))) break;
            p_ph0 ^= 1;
            if (j == 0 && !(ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * (C::B_O_EMPTY + 0), (unit_it & 1) ^ 1, FW_MMA_OE)))) break;
            tc_fence_after();
            issue_pv(tmem + C::TM_O0, tmem + C::TM_S0, sV + s * C::KV_TILE, j > 0);
            if (j == nk0 - 1) tc_commit_warp(bars + 8 * (C::B_O_FULL + 0));
          }
          if (more) {
            if (j + 1 < nk0) {
              issue_s(tmem + C::TM_S0, sQb, sK + sn * C::KV_TILE);
              tc_commit_warp(bars + 8 * (C::B_S_FULL + 0));
            }
          }
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * (C::B_P_FULL + 1), p_ph1, FW_MMA_P)))) break;
          p_ph1 ^= 1;
          if (j == 0 && !(ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * (C::B_O_EMPTY + 1), (unit_it & 1) ^ 1, FW_MMA_OE)))) break;
          tc_fence_after();
          issue_pv(tmem + C::TM_O1, tmem + C::TM_S1, sV + s * C::KV_TILE, j > 0);
          tc_commit_warp(bars + 8 * (C::B_V_EMPTY + s));
          if (j == nk1 - 1) tc_commit_warp(bars + 8 * (C::B_O_FULL + 1));
          if (more) {
            issue_s(tmem + C::TM_S1, sQb + C::Q_TILE, sK + sn * C::KV_TILE);
            tc_commit_warp(bars + 8 * (C::B_S_FULL + 1));
            tc_commit_warp(bars + 8 * (C::B_K_EMPTY + sn));
            // the unit's last S: its Q pair is free for the next unit's loads
            // (the PVs still to come do not read Q)
            if (j + 2 == nk1) tc_commit_warp(bars + 8 * (C::B_Q_EMPTY + qb));
          }
        }
        if (!ok) break;
        kv_it += nk1;
      }
      }
      // Wait for the last unit's Q_EMPTY arrival, so none lands after the CTA
      // has exited: with the S ring it is this thread's last commit; with two
      // S buffers it precedes the last PV's commits, whose final O_FULL
      // arrival the softmax warpgroups wait for before the teardown.
      if (q_it > 0)
        (void)__all_sync(0xffffffffu, mbar_wait(bars + 8 * (C::B_Q_EMPTY + (q_it - 1) % C::NQB),
                                                ((q_it - 1) / C::NQB) & 1, FW_MMA_Q));
    }
    }
    // teardown (each branch has its own, so the register regions never merge)
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc(tmem, C::TMEM_COLS);
    }
  } else {
    regs_inc<C::REGS_SOFTMAX>();
    // ------------------------------------------------------------ softmax warpgroups
    const int wg = (warp - 4) >> 2;          // which Q tile of the pair
    const int sp = warp & 3;                 // TMEM lane window of this warp
    const int r = sp * 32 + lane;            // row inside the tile
    const uint32_t lane_off = static_cast<uint32_t>(sp * 32) << 16;
    const uint32_t tS = tmem + lane_off + (wg ? C::TM_S1 : C::TM_S0);
    const uint32_t tO = tmem + lane_off + (wg ? C::TM_O1 : C::TM_O0);
    const uint32_t bar_s = bars + 8 * (C::B_S_FULL + wg), bar_p = bars + 8 * (C::B_P_FULL + wg);
    const uint32_t bar_o = bars + 8 * (C::B_O_FULL + wg), bar_oe = bars + 8 * (C::B_O_EMPTY + wg);
    uint32_t s_it = 0, o_it = 0;
    uint32_t g0 = 0, pv_c = 0;  // three-buffer ring: ring tiles before this unit; this Q tile's tiles so far
    bool ok = true;
    for (int k = 0, u = fwd_unit(list, 0, units); u < units && ok; u = fwd_unit(list, ++k, units)) {
      int bh, qp;
      fwd_decode_unit(u, BH, NP, CAUSAL, bh, qp);
      const int qt = 2 * qp + wg;
      const int nk = CAUSAL ? min((qt + 1) * C::R, NKT) : NKT;
      const int nk0 = CAUSAL ? min((2 * qp + 1) * C::R, NKT) : NKT;  // Q tile 0's key tiles
      const int row = qt * C::BM + r;
      float m_ref = -INFINITY, l = 0.f;
      for (int j = 0; j < nk; ++j, ++pv_c) {
        // this tile's S buffer and barriers
        uint32_t tS_j = tS, bar_s_j = bar_s, bar_p_j = bar_p, s_ph = s_it & 1;
        if constexpr (C::NS == 3) {
          const uint32_t g = g0 + ring_pos(j, wg, nk0);
          const int b = g % C::NS;
          tS_j = tmem + lane_off + C::tm_s(b);
          bar_s_j = bars + 8 * (C::B_S_FULL + b);
          bar_p_j = bars + 8 * (C::B_P_FULL + b);
          s_ph = (g / C::NS) & 1;
        }
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(bar_s_j, s_ph, FW_SM_S)))) break;
        ++s_it;
        tc_fence_after();
        constexpr int NC = C::BN;  // score columns per row
        uint32_t sr[NC];
#pragma unroll
        for (int c = 0; c < NC / 32; ++c) tmem_ld32(tS_j + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < NC / 32; ++c) reg_fence(*reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
        float s[NC];
#pragma unroll
        for (int c = 0; c < NC; ++c) s[c] = __uint_as_float(sr[c]);
        const int kbase = j * C::BN;
        // the diagonal tiles: some key of the tile lies past some row of the Q tile
        // (with 128-key tiles exactly the tile j == qt)
        const bool diag = C::BN == C::BM ? j == qt : kbase + C::BN - 1 > qt * C::BM;
        if ((CAUSAL && diag) || kbase + C::BN > N) {
#pragma unroll
          for (int c = 0; c < NC; ++c) {
            const int key = kbase + c;
            if (key >= N || (CAUSAL && key > row)) s[c] = -INFINITY;
          }
        }
        const float mx = row_max<NC>(s);  // 8 independent chains of 3-input maxima
        const float m_new = fmaxf(m_ref, mx * scale_log2);
        const bool need = m_new > m_ref + rescale_log2;
        const bool warp_rescale = __any_sync(0xffffffffu, need);
        const float alpha = need ? ex2(m_ref - m_new) : 1.f;  // ex2(-inf) = 0 on the first tile
        if (need) {
          l *= alpha;
          m_ref = m_new;
        }
        const float neg = -m_ref;
        // pairs of scores through the paired fp32 instructions: one FMA and
        // one add for two elements; 4 x 2 independent partial row sums
        const uint64_t sc2 = f2_make(scale_log2, scale_log2), ng2 = f2_make(neg, neg);
        uint64_t ps2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int ch = 0; ch < NC / 32; ++ch) {  // 32 scores -> 16 packed bf16 pairs -> 16 TMEM columns
          uint32_t p[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const uint64_t t2 = f2_fma(f2_make(s[32 * ch + 2 * c], s[32 * ch + 2 * c + 1]), sc2, ng2);
            float p0, p1;
            if (c % C::EXP_EMUL_EVERY == C::EXP_EMUL_EVERY - 1) {  // resolved at compile time
              exp2_poly3_x2(t2, p0, p1);
            } else {
              float t0, t1;
              f2_split(t2, t0, t1);
              p0 = ex2(t0);
              p1 = ex2(t1);
            }
            ps2[c & 3] = f2_add(ps2[c & 3], f2_make(p0, p1));
            p[c] = pack_bf16(p0, p1);
          }
          tmem_st16(tS_j + ch * 16, p);
        }
        float ps[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) f2_split(ps2[e], ps[2 * e], ps[2 * e + 1]);
#pragma unroll
        for (int w = 4; w > 0; w >>= 1)
#pragma unroll
          for (int e = 0; e < w; ++e) ps[e] += ps[e + w];
        const float lsum = ps[0];
        // Rescale O before this tile's PV is issued.  With two S buffers O holds
        // PV of tiles 0..j-1 already (the S MMA that signalled s_full was issued
        // after them); with the ring, wait for the PV of tile j-1 first.
        if (warp_rescale && j > 0) {
          if constexpr (C::NS == 3) {
            const uint32_t pc = pv_c - 1;
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * (C::B_O_DONE + 2 * wg + (pc & 1)),
                                                         (pc >> 1) & 1, FW_SM_O))))
              break;
            tc_fence_after();
          }
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
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
        mbar_arrive(bar_p_j);
        l += lsum;
      }
      if (!ok) break;
      g0 += nk0 + (CAUSAL ? min((2 * qp + 2) * C::R, NKT) : NKT);
      // epilogue: O / l (bf16) and LSE (fp32, natural log of the scaled logits)
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(bar_o, o_it & 1, FW_SM_O)))) break;
      ++o_it;
      tc_fence_after();
      const float inv_l = 1.f / l;
      __nv_bfloat16* orow = O + (static_cast<size_t>(bh) * N + row) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + c * 32, o);
        tmem_ld_wait();
        reg_fence(o);
        if (row < N) store_bf16x32(orow + c * 32, o, inv_l);
      }
      if (row < N) LSE[static_cast<size_t>(bh) * N + row] = (m_ref + __log2f(l)) * kLn2;
      tc_fence_before();
      mbar_arrive(bar_oe);
    }
    tc_fence_before();
    __syncthreads();
  }
}

}  // namespace fa
