// fa_bwd_fused.cuh -- the backward of tiled, IO-aware exact attention as five
// tensor-core products per tile (sm_100a).
//
// The backward keeps only O and the per-row statistic and recomputes the
// attention weights tile by tile ("图解Flash Attention运算原理", 总结:
// Recomputation keeps the softmax statistics and recomputes P when needed):
// P_ij = exp(S_ij - LSE_i).  The gradients of the loss sum(dO * O) (the
// analytic gradient of the definition; the pages do not print it):
//   D_i = sum_c dO_ic O_ic                 (over the bf16 O given)
//   dV_j = sum_i P_ij dO_i,  dP_ij = dO_i . V_j,  dS_ij = P_ij (dP_ij - D_i)
//   dK_j = scale sum_i dS_ij Q_i,  dQ_i = scale sum_j dS_ij K_j
//
// A unit is one (head, 128-key tile); for every 64-row query tile that can
// see its keys it takes all five products: S^T = K Q^T and dP^T = V dO^T into
// tensor memory, P^T and dS^T from them, dV += P^T dO and dK += dS^T Q with
// dV, dK accumulating in tensor memory over the whole loop, and the tile's
// contribution to dQ, dQ_t^T = K^T dS_t^T (d x 64, fp32).  Every key tile of
// a head adds into the same rows of dQ, so that partial goes to an fp32
// accumulator in global memory through the bulk-copy engine's reduce-add
// (element-wise fp32 adds performed in L2, from a shared-memory staging
// tile).  Three launches in all:
//   1. fa_bwd_preprocess_kernel<D, true>: D, and zeros into the accumulator;
//   2. fa_bwd_fused_kernel: dK, dV (bf16, written once) and the dQ partials;
//   3. fa_bwd_dq_convert_kernel: dQ = bf16(scale * accumulator).
// The order in which key tiles' partials reach a row of the accumulator is
// not fixed, so dQ can differ in the last bits from run to run; dK and dV
// are accumulated in a fixed order.  (fa_bwd.cuh holds the deterministic
// form: a separate dQ kernel that recomputes S and dP, seven products.)
//
// The kernel is persistent: one CTA per SM walks its units in order (with
// the mask, per-CTA lists computed on the host, longest first; otherwise a
// serpentine deal), so one unit's fixed work overlaps the next one's: its
// first query tiles load while the previous unit still runs, and its dK and
// dV are stored while the next unit's K and V load and its first products
// run.  Every role counts the query tiles of all its units, so the per-tile
// barriers keep their phases across units.
// Warp roles (384 threads, three warpgroups):
//   warp 0       TMA: per unit the first ST query tiles (Q and dO, through ST
//                stages), then K and V once the previous unit's products are
//                done reading them, then the remaining query tiles;
//                -LSE*log2(e) and D of each query tile into shared memory.
//   warp 1       tcgen05.mma issue (one elected lane), commits; a unit's
//                first dV and dK wait until the previous unit's are stored.
//   warps 4-7    softmax gradient: thread = key row.  Reads S^T and dP^T
//                from tensor memory, writes P^T and dS^T (bf16) back over
//                S^T's columns (the A operands of dV and dK) and dS^T also to
//                shared memory (the B operand of dQ^T).
//   warps 8-11   dQ drain: thread = column c of d.  Reads dQ_t^T from tensor
//                memory, stores it as a [64 queries][d] fp32 tile in shared
//                memory and issues the bulk reduce-add of that tile into the
//                accumulator rows of the query tile.  It reads all 64
//                columns into registers before staging, so the tensor-memory
//                buffer returns to the next dP^T product sooner.  After
//                a unit's last tile: its dK and dV (thread = key row) from
//                tensor memory to global memory.
// Tensor memory (512 columns): S^T/P^T/dS^T double buffer [0, 128) (64 each:
// S^T fp32, then P^T in its first 32 and dS^T in its next 32 columns as packed
// bf16); dP^T double buffer [128, 256), reused for dQ_t^T once the softmax
// gradient has read dP^T; dV [256, 256+d); dK [256+d, 256+2d).  At d = 64
// the dQ^T product runs with M = 128 over the adjacent K and V tiles (rows
// 64..127 of its result, V^T dS^T, are never read), which keeps every MMA in
// the M = 128 form.
#pragma once

#include "fa_device.cuh"

namespace fa {

template <int D, int ST_ = ((D == 128) ? 3 : 4), int NDQ_ = ((D == 128) ? 1 : 2)>
struct FusedCfg {
  static constexpr int BK = 128;                      // keys per CTA (MMA M of S^T, dP^T, dV, dK)
  static constexpr int BQ = 64;                       // queries per tile
  static constexpr int CH = D / 64;
  static constexpr int KCHUNK = BK * 128;             // one 64-column chunk of the key tile
  static constexpr int QCHUNK = BQ * 128;             // one 64-column chunk of a query tile
  static constexpr int K_TILE = BK * D * 2;
  static constexpr int Q_TILE = BQ * D * 2;
  static constexpr int DS_TILE = BK * BQ * 2;         // dS^T: 128 key rows of 64 bf16 (one swizzled chunk)
  static constexpr int DQ_TILE = BQ * D * 4;          // dQ partial staging: [64 queries][d] fp32
  static constexpr int ST = ST_;                      // Q / dO stages
  static constexpr int NDQ = NDQ_;                    // dQ staging buffers
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + K_TILE;        // adjacent to K: the d = 64 dQ^T product reads both
  static constexpr int OFF_Q = OFF_V + K_TILE;
  static constexpr int OFF_DO = OFF_Q + ST * Q_TILE;
  static constexpr int OFF_DS = OFF_DO + ST * Q_TILE;
  static constexpr int OFF_DQ = OFF_DS + 2 * DS_TILE;
  static constexpr int OFF_LSE = OFF_DQ + NDQ * DQ_TILE;  // ST x BQ floats (-LSE * log2 e)
  static constexpr int OFF_DD = OFF_LSE + ST * BQ * 4;    // ST x BQ floats (D)
  static constexpr int OFF_BAR = OFF_DD + ST * BQ * 4;
  static constexpr int B_KV_FULL = 0, B_Q_FULL = 1, B_Q_EMPTY = 1 + ST, B_S_FULL = 1 + 2 * ST,
                       B_P_FULL = B_S_FULL + 2, B_DQ_FULL = B_P_FULL + 2, B_DQ_EMPTY = B_DQ_FULL + 2,
                       B_STG_FREE = B_DQ_EMPTY + 2, B_STG_FULL = B_STG_FREE + NDQ, B_DKV_FULL = B_STG_FULL + NDQ,
                       B_KV_EMPTY = B_DKV_FULL + 1, B_ACC_EMPTY = B_KV_EMPTY + 1;
  static constexpr int NUM_BARS = B_ACC_EMPTY + 1;
  static constexpr int OFF_TMEM_SLOT = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_TMEM_SLOT + 16 + 1024;  // + room to align the base to 1024
  static_assert(SMEM_BYTES <= 232448, "shared memory of the fused backward exceeds 227 KB");
  static constexpr uint32_t TM_S = 0, TM_DP = 128, TM_DV = 256, TM_DK = 256 + D;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int THREADS = 384;
  // register split (launch: 384 x 168 = 64512): control 112 and dQ drain 136
  // (both decrease: never above the 168 of the launch), softmax gradient 256
  // (128 x 504 = 64512)
  static constexpr uint32_t REGS_CONTROL = 112, REGS_GRAD = 256, REGS_DRAIN = 136;
  static_assert(REGS_CONTROL <= 168 && REGS_DRAIN <= 168 && 128 * (REGS_CONTROL + REGS_GRAD + REGS_DRAIN) <= 64512,
                "register split must fit the registers of the launch");
};

enum FusedWaitSite : unsigned int {
  BF_PROD_QE = 64, BF_MMA_KV, BF_MMA_Q, BF_MMA_DQE, BF_MMA_P, BF_SM_S, BF_SM_Q, BF_SM_DKV, BF_DR_DQ, BF_DR_FREE,
  BF_DR_FULL, BF_PROD_KVE, BF_MMA_ACC
};

// Unit u of the persistent kernel: key tile kt of head bh.  Without the mask
// head-major (the CTAs running at the same time share a few heads' Q and dO
// in L2); with it, the longest key tiles (the first ones) of every head of an
// L2-sized group first (the host's lists assign them longest first).
template <bool CAUSAL>
__device__ __forceinline__ void fused_unit(int u, int BH, int NKT, int N, int D, int& bh, int& kt) {
  if (CAUSAL) {
    causal_grouped_unit(u, BH, NKT, causal_head_group(BH, N, D), bh, kt);
  } else {
    bh = u / NKT;
    kt = u - bh * NKT;
  }
}

// Query tile of the it-th step of key tile kt.  With the mask the steps start
// at the first query tile that sees the keys (i0) and walk up.  Without it
// every key tile of a head sees all nt query tiles; key tile kt starts at query
// tile 2kt (mod nt), so the CTAs of a head that run at the same time add their
// dQ partials into different rows of the accumulator.
template <bool CAUSAL>
__device__ __forceinline__ int fused_query_tile(int it, int i0, int nt, int kt) {
  if (CAUSAL) return i0 + it;
  int q = it + 2 * kt;
  q %= nt;
  return q;
}

// One row of an accumulator (dK or dV: this thread's tensor-memory lane) to
// global memory as bf16, times `mul`: D/32 loads of 32 columns, 16-byte stores.
template <int D>
__device__ __forceinline__ void store_accumulator_row(uint32_t t_row, __nv_bfloat16* dst_row, float mul, bool valid) {
#pragma unroll 1
  for (int cc = 0; cc < D / 32; ++cc) {
    uint32_t a[32];
    tmem_ld32(t_row + cc * 32, a);
    tmem_ld_wait();
    reg_fence(a);
    if (valid) store_bf16x32(dst_row + cc * 32, a, mul);
  }
}

template <int D, bool CAUSAL, int ST_ = ((D == 128) ? 3 : 4), int NDQ_ = ((D == 128) ? 1 : 2)>
__global__ void __launch_bounds__(FusedCfg<D, ST_, NDQ_>::THREADS, 1)
    fa_bwd_fused_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                        const float* __restrict__ LSE, const float* __restrict__ Dvec,
                        __nv_bfloat16* __restrict__ dK, __nv_bfloat16* __restrict__ dV,
                        float* __restrict__ dQacc, int BH, int N, float scale, float scale_log2,
                        const __grid_constant__ typename UnitListOf<CAUSAL>::type list) {
  using C = FusedCfg<D, ST_, NDQ_>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sK = sbase + C::OFF_K, sV = sbase + C::OFF_V, sQ = sbase + C::OFF_Q, sdO = sbase + C::OFF_DO;
  const uint32_t sDS = sbase + C::OFF_DS, sDQ = sbase + C::OFF_DQ;
  float* sLSE = reinterpret_cast<float*>(smem + C::OFF_LSE);
  float* sDD = reinterpret_cast<float*>(smem + C::OFF_DD);
  const uint32_t bars = sbase + C::OFF_BAR;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM_SLOT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Persistent: this CTA walks its units (key tiles of heads) in order; every
  // role counts the query tiles of the units before the current one (tb), so
  // the per-tile barriers keep their phases across units.
  const int NKT = (N + C::BK - 1) / C::BK;
  const int NQT = (N + C::BQ - 1) / C::BQ;
  const int units = BH * NKT;
  auto unit_tiles = [&](int kt, int& i0, int& nt) {
    i0 = CAUSAL ? (kt * C::BK) / C::BQ : 0;
    nt = NQT - i0;  // >= 1
  };

  if (threadIdx.x == 0) {
    mbar_init(bars + 8 * C::B_KV_FULL, 1);
    for (int s = 0; s < C::ST; ++s) {
      mbar_init(bars + 8 * (C::B_Q_FULL + s), 33);  // expect_tx arrive + 32 lanes writing LSE and D
      mbar_init(bars + 8 * (C::B_Q_EMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bars + 8 * (C::B_S_FULL + b), 1);
      mbar_init(bars + 8 * (C::B_P_FULL + b), 128);
      mbar_init(bars + 8 * (C::B_DQ_FULL + b), 1);
      mbar_init(bars + 8 * (C::B_DQ_EMPTY + b), 128);
    }
    for (int b = 0; b < C::NDQ; ++b) {
      mbar_init(bars + 8 * (C::B_STG_FREE + b), 1);    // the issuing thread: the buffer's last reduce has read it
      mbar_init(bars + 8 * (C::B_STG_FULL + b), 128);  // every drain thread: its column is stored
    }
    mbar_init(bars + 8 * C::B_DKV_FULL, 1);
    mbar_init(bars + 8 * C::B_KV_EMPTY, 1);    // the unit's last product that reads K and V is done
    mbar_init(bars + 8 * C::B_ACC_EMPTY, 128);  // the drain warps have stored the unit's dK and dV
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    regs_dec<C::REGS_CONTROL>();
    if (warp == 0) {
      // ---------------------------------------------------------- loads (whole warp)
      if (lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmdO);
      }
      int tb = 0;
      bool ok = true;
      for (int k = 0, u = list_unit(list, 0, units); u < units && ok; u = list_unit(list, ++k, units)) {
        int bh, kt, i0, nt;
        fused_unit<CAUSAL>(u, BH, NKT, N, D, bh, kt);
        unit_tiles(kt, i0, nt);
        // query tile it of this unit into its stage (once the tile that used the
        // stage before has had its dV and dK products)
        auto load_q = [&](int it) -> bool {
          const int g = tb + it, st = g % C::ST;
          const int qi = fused_query_tile<CAUSAL>(it, i0, nt, kt);
          if (!__all_sync(0xffffffffu, mbar_wait(bars + 8 * (C::B_Q_EMPTY + st), ((g / C::ST) & 1) ^ 1, BF_PROD_QE)))
            return false;
          if (lane == 0) {
            mbar_arrive_expect_tx(bars + 8 * (C::B_Q_FULL + st), 2 * C::Q_TILE);
            for (int c = 0; c < C::CH; ++c) {
              tma_load_3d(sQ + st * C::Q_TILE + c * C::QCHUNK, &tmQ, bars + 8 * (C::B_Q_FULL + st), c * 64,
                          qi * C::BQ, bh);
              tma_load_3d(sdO + st * C::Q_TILE + c * C::QCHUNK, &tmdO, bars + 8 * (C::B_Q_FULL + st), c * 64,
                          qi * C::BQ, bh);
            }
          }
#pragma unroll
          for (int e = lane; e < C::BQ; e += 32) {
            const int q = qi * C::BQ + e;
            const bool valid = q < N;
            sLSE[st * C::BQ + e] = valid ? -(LSE[static_cast<size_t>(bh) * N + q] * kLog2e) : -INFINITY;
            sDD[st * C::BQ + e] = valid ? Dvec[static_cast<size_t>(bh) * N + q] : 0.f;
          }
          mbar_arrive(bars + 8 * (C::B_Q_FULL + st));
          return true;
        };
        // the unit's first query tiles go while the previous unit still runs;
        // K and V once the previous unit's products are done reading them
        const int early = nt < C::ST ? nt : C::ST;
        for (int it = 0; it < early && ok; ++it) ok = load_q(it);
        if (!ok) break;
        if (k > 0 && !(ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * C::B_KV_EMPTY, (k - 1) & 1, BF_PROD_KVE))))
          break;
        if (lane == 0) {
          mbar_arrive_expect_tx(bars + 8 * C::B_KV_FULL, 2 * C::K_TILE);
          for (int c = 0; c < C::CH; ++c) {
            tma_load_3d(sK + c * C::KCHUNK, &tmK, bars + 8 * C::B_KV_FULL, c * 64, kt * C::BK, bh);
            tma_load_3d(sV + c * C::KCHUNK, &tmV, bars + 8 * C::B_KV_FULL, c * 64, kt * C::BK, bh);
          }
        }
        for (int it = early; it < nt && ok; ++it) ok = load_q(it);
        if (!ok) break;
        tb += nt;
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------- MMA issue (whole warp, one elected lane)
      constexpr uint32_t IDESC_T = idesc_bf16(128, C::BQ, false, false);  // S^T, dP^T: M=128 keys, N=64
      constexpr uint32_t IDESC_G = idesc_bf16(128, D, false, true);        // dV, dK: B MN-major
      constexpr uint32_t IDESC_DQ = idesc_bf16(128, C::BQ, true, true);    // dQ^T: A and B MN-major
      auto issue_t = [&](uint32_t d_tmem, uint32_t a_smem, uint32_t b_smem) {
        const uint32_t hi = sdesc_hi(1024);
        const uint64_t a0 = sdesc_make(sdesc_lo(a_smem, 16), hi), b0 = sdesc_make(sdesc_lo(b_smem, 16), hi);
        if (D == 128)
          mma_ss_k128(d_tmem, a0, sdesc_make(sdesc_lo(a_smem + C::KCHUNK, 16), hi), b0,
                      sdesc_make(sdesc_lo(b_smem + C::QCHUNK, 16), hi), IDESC_T, 0u);
        else
          mma_ss_k64(d_tmem, a0, b0, IDESC_T, 0u);
      };
      auto issue_g = [&](uint32_t d_tmem, uint32_t a_tmem, uint32_t b_smem, bool acc) {
        mma_ts_k64(d_tmem, a_tmem, sdesc_make(sdesc_lo(b_smem, C::QCHUNK), sdesc_hi(1024)), IDESC_G,
                   acc ? 1u : 0u);
      };
      // dQ^T = K^T dS^T: A = the key tile read MN-major (M = d columns, two
      // 64-column chunks KCHUNK apart; at d = 64 the second chunk is the V
      // tile), B = dS^T read MN-major (N = 64 queries, one chunk); K = 128 keys.
      const uint64_t dq_a = sdesc_make(sdesc_lo(sK, C::KCHUNK), sdesc_hi(1024));
      int tb = 0;
      bool ok = true;
      for (int k = 0, u = list_unit(list, 0, units); u < units && ok; u = list_unit(list, ++k, units)) {
        int bh, kt, i0, nt;
        fused_unit<CAUSAL>(u, BH, NKT, N, D, bh, kt);
        unit_tiles(kt, i0, nt);
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * C::B_KV_FULL, k & 1, BF_MMA_KV)))) break;
        tc_fence_after();
        for (int it = 0; it <= nt && ok; ++it) {
          if (it < nt) {
            const int g = tb + it, st = g % C::ST, b = g & 1;
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * (C::B_Q_FULL + st), (g / C::ST) & 1, BF_MMA_Q))))
              break;
            tc_fence_after();
            issue_t(tmem + C::TM_S + b * 64, sK, sQ + st * C::Q_TILE);
            if (g >= 2) {  // dP^T's buffer holds dQ^T of tile g-2 until the drain has read it
              if (!(ok = __all_sync(0xffffffffu,
                                    mbar_wait(bars + 8 * (C::B_DQ_EMPTY + b), ((g >> 1) & 1) ^ 1, BF_MMA_DQE))))
                break;
              tc_fence_after();
            }
            issue_t(tmem + C::TM_DP + b * 64, sV, sdO + st * C::Q_TILE);
            tc_commit_warp(bars + 8 * (C::B_S_FULL + b));
          }
          if (it > 0) {
            const int pit = it - 1, pg = tb + pit, pst = pg % C::ST, pb = pg & 1;
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * (C::B_P_FULL + pb), (pg >> 1) & 1, BF_MMA_P))))
              break;
            // the unit's first dV and dK overwrite the accumulators: the drain
            // warps must have read the previous unit's
            if (pit == 0 && k > 0 &&
                !(ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * C::B_ACC_EMPTY, (k - 1) & 1, BF_MMA_ACC))))
              break;
            tc_fence_after();
            issue_g(tmem + C::TM_DV, tmem + C::TM_S + pb * 64, sdO + pst * C::Q_TILE, pit > 0);
            issue_g(tmem + C::TM_DK, tmem + C::TM_S + pb * 64 + 32, sQ + pst * C::Q_TILE, pit > 0);
            tc_commit_warp(bars + 8 * (C::B_Q_EMPTY + pst));
            mma_ss_k128_mnmn(tmem + C::TM_DP + pb * 64, dq_a,
                             sdesc_make(sdesc_lo(sDS + pb * C::DS_TILE, C::DS_TILE), sdesc_hi(1024)), IDESC_DQ, 0u);
            tc_commit_warp(bars + 8 * (C::B_DQ_FULL + pb));
          }
        }
        if (!ok) break;
        tc_commit_warp(bars + 8 * C::B_KV_EMPTY);  // K and V free for the next unit's loads
        tc_commit_warp(bars + 8 * C::B_DKV_FULL);  // dK and dV complete
        tb += nt;
      }
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax gradient (thread = key row)
    regs_inc<C::REGS_GRAD>();
    const int sp = warp & 3;
    const int r = sp * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(sp * 32) << 16;
    int tb = 0;
    bool ok = true;
    for (int k = 0, u = list_unit(list, 0, units); u < units && ok; u = list_unit(list, ++k, units)) {
    int bh, kt, i0, nt;
    fused_unit<CAUSAL>(u, BH, NKT, N, D, bh, kt);
    unit_tiles(kt, i0, nt);
    const int key = kt * C::BK + r;
    const bool key_valid = key < N;
    int qi = fused_query_tile<CAUSAL>(0, i0, nt, kt);  // advanced by one (mod NQT) per tile
    for (int it = 0; it < nt; ++it, qi = qi + 1 == NQT ? 0 : qi + 1) {
      const int g = tb + it, st = g % C::ST, b = g & 1;
      bool w = mbar_wait(bars + 8 * (C::B_S_FULL + b), (g >> 1) & 1, BF_SM_S);
      w = w && mbar_wait(bars + 8 * (C::B_Q_FULL + st), (g / C::ST) & 1, BF_SM_Q);
      if (!(ok = __all_sync(0xffffffffu, w))) break;
      tc_fence_after();
      const uint32_t tS = tmem + lane_off + C::TM_S + b * 64;
      const uint32_t tP = tmem + lane_off + C::TM_DP + b * 64;
      uint32_t sr[64], dr[64];
      tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_ld32(tP, *reinterpret_cast<uint32_t(*)[32]>(&dr[0]));
      tmem_ld32(tP + 32, *reinterpret_cast<uint32_t(*)[32]>(&dr[32]));
      tmem_ld_wait();
      reg_fence(*reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      reg_fence(*reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      reg_fence(*reinterpret_cast<uint32_t(*)[32]>(&dr[0]));
      reg_fence(*reinterpret_cast<uint32_t(*)[32]>(&dr[32]));
      const float* nlse2 = sLSE + st * C::BQ;  // -LSE * log2(e) of the tile's queries
      [[maybe_unused]] const uint64_t sc2 = f2_make(scale_log2, scale_log2);
      const float* dd = sDD + st * C::BQ;
      // masking: queries e < lim of this tile get P = 0 in this key row -- the
      // causal mask (query q sees key j iff j <= q) and key rows past N
      // (zero-filled K and V) -- so lim <= 0 means no masking
      const int lim = !key_valid ? C::BQ : (CAUSAL ? key - qi * C::BQ : 0);
      const bool mask = lim > 0;
      uint8_t* ds_row = smem + C::OFF_DS + b * C::DS_TILE + r * 128;
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {  // 32 queries -> 16 packed columns of P^T and of dS^T
        uint32_t pp[16], dsp[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int e = 32 * ch + 2 * c;
          // the same operations either way (one rounding per fma, sub, mul);
          // at d = 64 on paired fp32 instructions, which measured faster there
          // (at d = 128 the scalar form measured as fast or faster)
          float p0, p1, ds0, ds1;
          if constexpr (D == 64) {
            f2_split(f2_fma(f2_make(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1])), sc2,
                            f2_make(nlse2[e], nlse2[e + 1])),
                     p0, p1);
          } else {
            p0 = fmaf(__uint_as_float(sr[e]), scale_log2, nlse2[e]);
            p1 = fmaf(__uint_as_float(sr[e + 1]), scale_log2, nlse2[e + 1]);
          }
          p0 = ex2(p0);
          p1 = ex2(p1);
          if (mask) {
            if (e < lim) p0 = 0.f;
            if (e + 1 < lim) p1 = 0.f;
          }
          if constexpr (D == 64) {
            f2_split(f2_mul(f2_make(p0, p1), f2_sub(f2_make(__uint_as_float(dr[e]), __uint_as_float(dr[e + 1])),
                                                    f2_make(dd[e], dd[e + 1]))),
                     ds0, ds1);
          } else {
            ds0 = p0 * (__uint_as_float(dr[e]) - dd[e]);
            ds1 = p1 * (__uint_as_float(dr[e + 1]) - dd[e + 1]);
          }
          pp[c] = pack_bf16(p0, p1);
          dsp[c] = pack_bf16(ds0, ds1);
        }
        tmem_st16(tS + ch * 16, pp);
        tmem_st16(tS + 32 + ch * 16, dsp);
        // dS^T row r of the 128-byte-swizzled tile: 16-byte chunk j (queries
        // 8j .. 8j+7) sits at chunk position j ^ (r % 8)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int j = 4 * ch + jj;
          uint4 v;
          v.x = dsp[4 * jj];
          v.y = dsp[4 * jj + 1];
          v.z = dsp[4 * jj + 2];
          v.w = dsp[4 * jj + 3];
          *reinterpret_cast<uint4*>(ds_row + ((j ^ (r & 7)) << 4)) = v;
        }
      }
      tmem_st_wait();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bars + 8 * (C::B_P_FULL + b));
    }
    tb += nt;
    }
  } else {
    // ------------------------------------------------------------ dQ drain (thread = column c of d)
    regs_dec<C::REGS_DRAIN>();
    const int sp = warp & 3;
    const int c = sp * 32 + lane;
    const bool active = c < D;  // d = 64: rows 64..127 of the product are V^T dS^T, not read
    const uint32_t lane_off = static_cast<uint32_t>(sp * 32) << 16;
    const bool issuer = threadIdx.x == 256;
    float* stg = reinterpret_cast<float*>(smem + C::OFF_DQ);
    int tb = 0;
    bool ok = true;
    for (int k = 0, u = list_unit(list, 0, units); u < units && ok; u = list_unit(list, ++k, units)) {
    int bh, kt, i0, nt;
    fused_unit<CAUSAL>(u, BH, NKT, N, D, bh, kt);
    unit_tiles(kt, i0, nt);
    for (int it = 0; it < nt; ++it) {
      const int g = tb + it, b = g & 1, sb = g % C::NDQ;
      const int qi = fused_query_tile<CAUSAL>(it, i0, nt, kt);
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * (C::B_DQ_FULL + b), (g >> 1) & 1, BF_DR_DQ)))) break;
      tc_fence_after();
      // all 64 columns into registers, release the tensor-memory buffer at
      // once (the next dP^T product may go ahead), then stage
      uint32_t v[64];
      if (active) {
        tmem_ld32(tmem + lane_off + C::TM_DP + b * 64, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        tmem_ld32(tmem + lane_off + C::TM_DP + b * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        tmem_ld_wait();
        reg_fence(*reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        reg_fence(*reinterpret_cast<uint32_t(*)[32]>(&v[32]));
      }
      tc_fence_before();
      mbar_arrive(bars + 8 * (C::B_DQ_EMPTY + b));
      // the staging buffer sb is free once the reduce issued NDQ tiles ago has read it
      if (issuer) {
        bulk_wait_read<C::NDQ - 1>();
        mbar_arrive(bars + 8 * (C::B_STG_FREE + sb));
      }
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * (C::B_STG_FREE + sb), (g / C::NDQ) & 1, BF_DR_FREE))))
        break;
      if (active) {
        float* t = stg + sb * (C::DQ_TILE / 4) + c;
#pragma unroll
        for (int q = 0; q < C::BQ; ++q) t[q * D] = __uint_as_float(v[q]);
      }
      fence_proxy_async_smem();
      mbar_arrive(bars + 8 * (C::B_STG_FULL + sb));
      bool stored = true;
      if (issuer) {
        stored = mbar_wait(bars + 8 * (C::B_STG_FULL + sb), (g / C::NDQ) & 1, BF_DR_FULL);
        if (stored) {
          const int rows = min(C::BQ, N - qi * C::BQ);
          bulk_reduce_add_f32(dQacc + (static_cast<size_t>(bh) * N + static_cast<size_t>(qi) * C::BQ) * D,
                              sDQ + sb * C::DQ_TILE, static_cast<uint32_t>(rows * D * 4));
          bulk_commit();
        }
      }
      if (!(ok = __all_sync(0xffffffffu, stored))) break;
    }
    if (!ok) break;
    // the unit's dK and dV (thread = key row of the warp's lane window), while
    // the next unit's K and V load and the softmax warps start on its tiles
    if (!(ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * C::B_DKV_FULL, k & 1, BF_SM_DKV)))) break;
    tc_fence_after();
    {
      const int key = kt * C::BK + sp * 32 + lane;
      const size_t row = (static_cast<size_t>(bh) * N + key) * D;
      store_accumulator_row<D>(tmem + lane_off + C::TM_DV, dV + row, 1.f, key < N);
      store_accumulator_row<D>(tmem + lane_off + C::TM_DK, dK + row, scale, key < N);
    }
    tc_fence_before();
    mbar_arrive(bars + 8 * C::B_ACC_EMPTY);
    tb += nt;
    }
    if (issuer) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}


// ---------------------------------------------------------------------------
// dQ = bf16(scale * accumulator): eight elements per thread, 16-byte stores
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) fa_bwd_dq_convert_kernel(const float* __restrict__ acc,
                                                                 __nv_bfloat16* __restrict__ dQ, long long n8,
                                                                 float scale) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const float4 a = reinterpret_cast<const float4*>(acc)[2 * i];
  const float4 b = reinterpret_cast<const float4*>(acc)[2 * i + 1];
  uint4 w;
  w.x = pack_bf16(a.x * scale, a.y * scale);
  w.y = pack_bf16(a.z * scale, a.w * scale);
  w.z = pack_bf16(b.x * scale, b.y * scale);
  w.w = pack_bf16(b.z * scale, b.w * scale);
  reinterpret_cast<uint4*>(dQ)[i] = w;
}

}  // namespace fa
