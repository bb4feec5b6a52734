// fa_bwd2.cuh -- dK, dV on CTA pairs (tcgen05 cta_group::2), d = 128.
//
// The same computation as fa_bwd_dkdv_kernel ("图解Flash Attention运算原理",
// 总结: the backward recomputes P from the kept statistic; the gradients are
// the analytic ones of the definition), with the MMAs of two SMs joined:
//
//   * A CTA pair owns 256 consecutive keys of one head, 128 per CTA (each
//     CTA's K and V rows, and its rows of the S^T, dP^T, dV, dK accumulators).
//   * Per tile of 64 queries the leader CTA issues S^T = K Q^T and
//     dP^T = V dO^T as M = 256 (keys), N = 64 (queries), K = 128 MMAs.  B is
//     split by N between the CTAs: each loads 32 of the 64 query rows of Q and
//     dO ("row slices").
//   * dV += P^T dO and dK += dS^T Q are M = 256, N = 128 (= d), K = 64 MMAs
//     with A (P^T, dS^T) read from each CTA's tensor memory; B is split by
//     N again: each CTA loads the 64 columns 64*rank.. of the tile's 64 rows of
//     dO and Q ("column slices").
//   * Loads use .cta_group::2 TMA (no multicast) and complete on the leader's
//     barriers, which the leader arms for both CTAs' bytes.  Each CTA stages
//     its own copy of the tile's LSE and D (its softmax threads read them).
//     MMA completions are committed to both CTAs; the peer's softmax threads
//     arrive on their own CTA's barrier and one relay thread forwards one
//     arrival per phase to the leader.
//   * Per SM this halves the L2 reads of Q and dO per key and runs the tensor
//     core at the pair rates (M=256: ~84 cycles per N=64 step of K=16, ~69 per
//     N=128 TMEM-operand step, against ~96 and ~83 on one SM).
#pragma once

#include "fa_device.cuh"

namespace fa {

struct Dkdv2Cfg {
  static constexpr int D = 128;
  static constexpr int BK = 128;                 // keys per CTA (256 per pair)
  static constexpr int BQ = 64;                  // queries per tile
  static constexpr int KCHUNK = BK * 128;        // one 64-column chunk of the 128-key tile (16 KB)
  static constexpr int K_TILE = BK * D * 2;      // 32 KB
  static constexpr int R_CHUNK = 32 * 128;       // one 64-column chunk of a 32-row slice (4 KB)
  static constexpr int ROWS = 32 * D * 2;        // row slice: 32 queries x 128 columns (8 KB)
  static constexpr int COLS = BQ * 64 * 2;       // column slice: 64 queries x 64 columns (8 KB)
  static constexpr int STAGE = 2 * ROWS + 2 * COLS;  // Q rows, dO rows, Q columns, dO columns
  static constexpr int Q_ROWS = 0, DO_ROWS = ROWS, Q_COLS = 2 * ROWS, DO_COLS = 2 * ROWS + COLS;
  static constexpr int ST = 4;                   // stages of query tiles
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = K_TILE;
  static constexpr int OFF_STAGE = 2 * K_TILE;
  static constexpr int OFF_LSE = OFF_STAGE + ST * STAGE;  // ST x BQ floats (LSE * log2 e)
  static constexpr int OFF_DD = OFF_LSE + ST * BQ * 4;    // ST x BQ floats (D)
  static constexpr int OFF_BAR = OFF_DD + ST * BQ * 4;
  static constexpr int B_KV_FULL = 0, B_Q_FULL = 1, B_Q_EMPTY = 1 + ST, B_LD_FULL = 1 + 2 * ST,
                       B_S_FULL = 1 + 3 * ST, B_P_FULL = B_S_FULL + 2, B_DKV_FULL = B_P_FULL + 2;
  static constexpr int NUM_BARS = B_DKV_FULL + 1;
  static constexpr int OFF_TMEM_SLOT = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_TMEM_SLOT + 16 + 1024;
  static constexpr uint32_t TM_S = 0, TM_DP = 128, TM_DV = 256, TM_DK = 384;  // S^T / dP^T: two 64-col buffers
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int THREADS = 192;  // warp 0 loads, warp 1 MMA (leader) or relay (peer), warps 2-5 gradients
  static constexpr uint16_t BOTH = 0x3;
};

enum Bwd2WaitSite : unsigned int {
  B2_PROD_QE = 96, B2_MMA_KV, B2_MMA_Q, B2_MMA_P, B2_RELAY, B2_SM_S, B2_SM_LD, B2_SM_DKV
};

template <bool CAUSAL>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Dkdv2Cfg::THREADS, 1)
    fa_bwd_dkdv_2sm_kernel(const __grid_constant__ CUtensorMap tmQr, const __grid_constant__ CUtensorMap tmdOr,
                           const __grid_constant__ CUtensorMap tmQc, const __grid_constant__ CUtensorMap tmdOc,
                           const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                           const float* __restrict__ LSE, const float* __restrict__ Dvec,
                           __nv_bfloat16* __restrict__ dK, __nv_bfloat16* __restrict__ dV, int N, float scale,
                           float scale_log2) {
  using C = Dkdv2Cfg;
  constexpr int D = C::D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sK = sbase + C::OFF_K, sV = sbase + C::OFF_V, sStage = sbase + C::OFF_STAGE;
  float* sLSE = reinterpret_cast<float*>(smem + C::OFF_LSE);
  float* sDD = reinterpret_cast<float*>(smem + C::OFF_DD);
  const uint32_t bars = sbase + C::OFF_BAR;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM_SLOT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  auto bar = [&](int i) { return bars + 8u * i; };
  auto lead = [&](int i) { return map_shared_to_rank(bars + 8u * i, 0); };

  // Pair order as in the one-SM kernel: head-major without a mask; with it,
  // the longest key tiles (the first ones) of every head first.
  const int pair = blockIdx.x >> 1;
  const int NKP = (N + 2 * C::BK - 1) / (2 * C::BK);
  const int BHg = (gridDim.x >> 1) / NKP;
  int bh, kp;
  if (CAUSAL) {
    causal_grouped_unit(pair, BHg, NKP, causal_head_group(BHg, N, D), bh, kp);
  } else {
    bh = pair / NKP;
    kp = pair - bh * NKP;
  }
  const int key0 = kp * 2 * C::BK + static_cast<int>(rank) * C::BK;  // this CTA's first key
  const int NQT = (N + C::BQ - 1) / C::BQ;
  const int i0 = CAUSAL ? (kp * 2 * C::BK) / C::BQ : 0;  // first query tile that sees the pair's keys
  const int nt = NQT - i0;                                // the same for both CTAs

  if (threadIdx.x == 0) {
    mbar_init(bar(C::B_KV_FULL), 1);
    for (int s = 0; s < C::ST; ++s) {
      mbar_init(bar(C::B_Q_FULL + s), 1);    // the leader's expect_tx arrival (both CTAs' bytes)
      mbar_init(bar(C::B_Q_EMPTY + s), 1);   // one commit from the leader
      mbar_init(bar(C::B_LD_FULL + s), 32);  // this CTA's 32 load lanes (LSE and D staged)
    }
    const uint32_t cnt = rank == 0 ? 129u : 128u;  // + the relay's arrival on the leader
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(C::B_S_FULL + b), 1);
      mbar_init(bar(C::B_P_FULL + b), cnt);
    }
    mbar_init(bar(C::B_DKV_FULL), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ loads (both CTAs, whole warp)
    if (lane == 0) {
      tma_prefetch_desc(&tmQr);
      tma_prefetch_desc(&tmdOr);
      tma_prefetch_desc(&tmQc);
      tma_prefetch_desc(&tmdOc);
      if (rank == 0) mbar_arrive_expect_tx(bar(C::B_KV_FULL), 2 * 2 * C::K_TILE);
      for (int c = 0; c < 2; ++c) {
        tma_load_3d_pair(sK + c * C::KCHUNK, &tmK, lead(C::B_KV_FULL), c * 64, key0, bh);
        tma_load_3d_pair(sV + c * C::KCHUNK, &tmV, lead(C::B_KV_FULL), c * 64, key0, bh);
      }
    }
    for (int it = 0; it < nt; ++it) {
      const int st = it % C::ST;
      const int qi = i0 + it;
      const bool ok = mbar_wait_cluster(bar(C::B_Q_EMPTY + st), ((it / C::ST) & 1) ^ 1, B2_PROD_QE);
      if (!__all_sync(0xffffffffu, ok)) break;
      if (lane == 0) {
        const uint32_t base = sStage + st * C::STAGE;
        const uint32_t full = lead(C::B_Q_FULL + st);
        if (rank == 0) mbar_arrive_expect_tx(bar(C::B_Q_FULL + st), 2 * C::STAGE);
        const int r0 = qi * C::BQ + 32 * static_cast<int>(rank);  // this CTA's 32 query rows
        for (int c = 0; c < 2; ++c) {
          tma_load_3d_pair(base + C::Q_ROWS + c * C::R_CHUNK, &tmQr, full, c * 64, r0, bh);
          tma_load_3d_pair(base + C::DO_ROWS + c * C::R_CHUNK, &tmdOr, full, c * 64, r0, bh);
        }
        // columns 64*rank .. +63 of the tile's 64 query rows
        tma_load_3d_pair(base + C::Q_COLS, &tmQc, full, 64 * static_cast<int>(rank), qi * C::BQ, bh);
        tma_load_3d_pair(base + C::DO_COLS, &tmdOc, full, 64 * static_cast<int>(rank), qi * C::BQ, bh);
      }
#pragma unroll
      for (int e = lane; e < C::BQ; e += 32) {
        const int q = qi * C::BQ + e;
        const bool valid = q < N;
        sLSE[st * C::BQ + e] = valid ? LSE[static_cast<size_t>(bh) * N + q] * kLog2e : INFINITY;
        sDD[st * C::BQ + e] = valid ? Dvec[static_cast<size_t>(bh) * N + q] : 0.f;
      }
      mbar_arrive(bar(C::B_LD_FULL + st));
    }
  } else if (warp == 1 && rank == 0) {
    // ------------------------------------------------------------ MMA issuer (leader CTA only)
    constexpr uint32_t IDESC_T = idesc_bf16(256, C::BQ, false, false);  // S^T, dP^T: M=256 keys, N=64 queries
    constexpr uint32_t IDESC_G = idesc_bf16(256, D, false, true);       // dV, dK: B (column slices) MN-major
    const uint32_t hi = sdesc_hi(1024);
    const uint64_t ka0 = sdesc_make(sdesc_lo(sK, 16), hi), ka1 = sdesc_make(sdesc_lo(sK + C::KCHUNK, 16), hi);
    const uint64_t va0 = sdesc_make(sdesc_lo(sV, 16), hi), va1 = sdesc_make(sdesc_lo(sV + C::KCHUNK, 16), hi);
    bool ok = __all_sync(0xffffffffu, mbar_wait_cluster(bar(C::B_KV_FULL), 0, B2_MMA_KV));
    tc_fence_after();
    for (int it = 0; it <= nt && ok; ++it) {
      if (it < nt) {
        const int st = it % C::ST, b = it & 1;
        if (!(ok = __all_sync(0xffffffffu,
                                 mbar_wait_cluster(bar(C::B_Q_FULL + st), (it / C::ST) & 1, B2_MMA_Q))))
          break;
        tc_fence_after();
        const uint32_t base = sStage + st * C::STAGE;
        mma2_ss_k128(tmem + C::TM_S + b * 64, ka0, ka1, sdesc_make(sdesc_lo(base + C::Q_ROWS, 16), hi),
                     sdesc_make(sdesc_lo(base + C::Q_ROWS + C::R_CHUNK, 16), hi), IDESC_T, 0u);
        mma2_ss_k128(tmem + C::TM_DP + b * 64, va0, va1, sdesc_make(sdesc_lo(base + C::DO_ROWS, 16), hi),
                     sdesc_make(sdesc_lo(base + C::DO_ROWS + C::R_CHUNK, 16), hi), IDESC_T, 0u);
        tc_commit_pair_warp(bar(C::B_S_FULL + b), C::BOTH);
      }
      if (it > 0) {
        const int pit = it - 1, pst = pit % C::ST, pb = pit & 1;
        if (!(ok = __all_sync(0xffffffffu,
                                 mbar_wait_cluster(bar(C::B_P_FULL + pb), (pit >> 1) & 1, B2_MMA_P))))
          break;
        tc_fence_after();
        const uint32_t pbase = sStage + pst * C::STAGE;
        mma2_ts_k64(tmem + C::TM_DV, tmem + C::TM_S + pb * 64,
                    sdesc_make(sdesc_lo(pbase + C::DO_COLS, C::COLS), hi), IDESC_G, pit > 0 ? 1u : 0u);
        mma2_ts_k64(tmem + C::TM_DK, tmem + C::TM_DP + pb * 64,
                    sdesc_make(sdesc_lo(pbase + C::Q_COLS, C::COLS), hi), IDESC_G, pit > 0 ? 1u : 0u);
        // Stages are reused only for tile pit + ST; skipping the commit for
        // the last ST tiles leaves DKV_FULL as the last arrival the commits
        // make, and every thread of both CTAs waits for it.
        if (pit + C::ST < nt) tc_commit_pair_warp(bar(C::B_Q_EMPTY + pst), C::BOTH);
      }
    }
    if (ok) tc_commit_pair_warp(bar(C::B_DKV_FULL), C::BOTH);
  } else if (warp == 1) {
    // ------------------------------------------------------------ relay (CTA 1)
    if (lane == 0) {
      for (int it = 0; it < nt; ++it) {
        const int b = it & 1;
        if (!mbar_wait_cluster(bar(C::B_P_FULL + b), (it >> 1) & 1, B2_RELAY)) break;
        tc_fence_after();  // carry the gradient threads' tensor-memory stores across this thread
        tc_fence_before();
        mbar_arrive_cluster(lead(C::B_P_FULL + b));
      }
    }
  } else {
    // ------------------------------------------------------------ gradient warpgroup (both CTAs)
    const int sp = warp & 3;
    const int r = sp * 32 + lane;
    const int key = key0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(sp * 32) << 16;
    bool ok = true;
    for (int it = 0; it < nt; ++it) {
      const int st = it % C::ST, b = it & 1;
      const int qi = i0 + it;
      bool w = mbar_wait_cluster(bar(C::B_S_FULL + b), (it >> 1) & 1, B2_SM_S);
      w = w && mbar_wait(bar(C::B_LD_FULL + st), (it / C::ST) & 1, B2_SM_LD);
      if (!(ok = __all_sync(0xffffffffu, w))) break;
      tc_fence_after();
      const uint32_t tS = tmem + lane_off + C::TM_S + b * 64;
      const uint32_t tP = tmem + lane_off + C::TM_DP + b * 64;
      const float* lse2 = sLSE + st * C::BQ;
      const float* dd = sDD + st * C::BQ;
      const bool diag = CAUSAL && (qi * C::BQ < key0 + C::BK);  // some query of the tile precedes some key here
      // two halves of 32 queries: load S^T and dP^T columns 32*ch.., write the
      // 16 packed columns of P^T and dS^T at 16*ch (below the next half's loads)
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        uint32_t sr[32], dr[32];
        tmem_ld32(tS + 32 * ch, sr);
        tmem_ld32(tP + 32 * ch, dr);
        tmem_ld_wait();
        reg_fence(sr);
        reg_fence(dr);
        uint32_t pp[16], dsp[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int e = 32 * ch + 2 * c;
          float p0 = ex2(fmaf(__uint_as_float(sr[2 * c]), scale_log2, -lse2[e]));
          float p1 = ex2(fmaf(__uint_as_float(sr[2 * c + 1]), scale_log2, -lse2[e + 1]));
          if (diag) {
            const int q0 = qi * C::BQ + e;
            if (q0 < key) p0 = 0.f;
            if (q0 + 1 < key) p1 = 0.f;
          }
          const float ds0 = p0 * (__uint_as_float(dr[2 * c]) - dd[e]);
          const float ds1 = p1 * (__uint_as_float(dr[2 * c + 1]) - dd[e + 1]);
          pp[c] = pack_bf16(p0, p1);
          dsp[c] = pack_bf16(ds0, ds1);
        }
        tmem_st16(tS + ch * 16, pp);
        tmem_st16(tP + ch * 16, dsp);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(C::B_P_FULL + b));
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait_cluster(bar(C::B_DKV_FULL), 0, B2_SM_DKV))) {
      tc_fence_after();
      const size_t base = (static_cast<size_t>(bh) * N + key) * D;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t tA = tmem + lane_off + (which ? C::TM_DK : C::TM_DV);
        __nv_bfloat16* dst_row = (which ? dK : dV) + base;
        const float mul = which ? scale : 1.f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t a[32];
          tmem_ld32(tA + c * 32, a);
          tmem_ld_wait();
          reg_fence(a);
          if (key < N) {
            uint4* dst = reinterpret_cast<uint4*>(dst_row + c * 32);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 wv;
              wv.x = pack_bf16(__uint_as_float(a[8 * v + 0]) * mul, __uint_as_float(a[8 * v + 1]) * mul);
              wv.y = pack_bf16(__uint_as_float(a[8 * v + 2]) * mul, __uint_as_float(a[8 * v + 3]) * mul);
              wv.z = pack_bf16(__uint_as_float(a[8 * v + 4]) * mul, __uint_as_float(a[8 * v + 5]) * mul);
              wv.w = pack_bf16(__uint_as_float(a[8 * v + 6]) * mul, __uint_as_float(a[8 * v + 7]) * mul);
              dst[v] = wv;
            }
          }
        }
      }
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
