// fa_bwd3.cuh -- dK, dV with persistent CTAs (opt-in: FA_BWD_PERSIST=1; it
// measured no faster than one CTA per 128-key tile, 2-6% slower without the
// mask at B=2, H=16, N=4096 and 0.6% faster with it at B=4, H=32, N=2048).
//
// The same computation as fa_bwd_dkdv_kernel ("图解Flash Attention运算原理",
// 总结: P recomputed from the kept statistic; the gradients are the analytic
// ones of the definition), but one CTA per SM walks a list of (head, 128-key
// tile) units, so the fixed costs of a unit overlap the work of its
// neighbours instead of idling the tensor core:
//   * K and V are double-buffered: the next unit's tiles load while this
//     unit's query tiles run.
//   * The dK / dV epilogue (tensor memory -> bf16 rows in HBM) belongs to its
//     own warpgroup, which frees the accumulators through a barrier; the
//     gradient warpgroup goes straight on to the next unit, whose first S^T
//     and dP^T MMAs run during the epilogue.  Only the next unit's first dV /
//     dK MMA waits for the epilogue.
//   * Query stages, S^T / dP^T buffers and their barriers run on counters
//     that continue across units.
// Units are ordered as the one-SM-per-tile kernel's blocks (head-major without
// the mask; longest first within head groups with it) and dealt to the CTAs
// in serpentine order.
#pragma once

#include "fa_device.cuh"

namespace fa {

template <int D>
struct Dkdv3Cfg {
  static constexpr int BK = 128;                     // keys per unit (MMA M)
  static constexpr int BQ = 64;                      // queries per tile (MMA N of S^T)
  static constexpr int CH = D / 64;
  static constexpr int KCHUNK = BK * 128;            // one 64-column chunk of the key tile
  static constexpr int QCHUNK = BQ * 128;            // one 64-column chunk of a query tile
  static constexpr int K_TILE = BK * D * 2;
  static constexpr int KV_BUF = 2 * K_TILE;          // K then V of one unit
  static constexpr int Q_TILE = BQ * D * 2;
  static constexpr int ST = (D == 128) ? 3 : 4;
  static constexpr int OFF_KV = 0;                   // two K/V buffers
  static constexpr int OFF_Q = OFF_KV + 2 * KV_BUF;  // ST stages of Q tiles
  static constexpr int OFF_DO = OFF_Q + ST * Q_TILE; // ST stages of dO tiles
  static constexpr int OFF_LSE = OFF_DO + ST * Q_TILE;  // ST x BQ floats (LSE * log2 e)
  static constexpr int OFF_DD = OFF_LSE + ST * BQ * 4;  // ST x BQ floats (D)
  static constexpr int OFF_BAR = OFF_DD + ST * BQ * 4;
  static constexpr int B_KV_FULL = 0, B_KV_EMPTY = 2, B_Q_FULL = 4, B_Q_EMPTY = 4 + ST, B_S_FULL = 4 + 2 * ST,
                       B_P_FULL = B_S_FULL + 2, B_DKV_FULL = B_P_FULL + 2, B_DKV_EMPTY = B_DKV_FULL + 1;
  static constexpr int NUM_BARS = B_DKV_EMPTY + 1;
  static constexpr int OFF_TMEM_SLOT = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_TMEM_SLOT + 16 + 1024;
  static constexpr uint32_t TM_S = 0, TM_DP = 128, TM_DV = 256, TM_DK = 256 + D;  // S/dP: two 64-col buffers
  static constexpr uint32_t TMEM_COLS = 512;
  // warpgroup 0: warp 0 loads, warp 1 MMA; warpgroup 1: dK/dV epilogue;
  // warpgroup 2: gradients (thread = key)
  static constexpr int THREADS = 384;
  // register split (launch: 384 x 168 = 64512): 56 + 96 + 256 per thread (52224)
  static constexpr uint32_t REGS_CONTROL = 56, REGS_EPILOGUE = 96, REGS_GRAD = 256;
};

enum Bwd3WaitSite : unsigned int {
  B3_PROD_KVE = 112 + 16, B3_PROD_QE, B3_MMA_KV, B3_MMA_Q, B3_MMA_P, B3_MMA_DE, B3_SM_S, B3_SM_Q, B3_EP_DKV
};

// Unit u: head bh, key tile kt.
__device__ __forceinline__ void dkdv3_decode_unit(int u, int BH, int NKT, int G, bool causal, int& bh, int& kt) {
  if (causal) {
    causal_grouped_unit(u, BH, NKT, G, bh, kt);
  } else {
    bh = u / NKT;
    kt = u - bh * NKT;
  }
}

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(Dkdv3Cfg<D>::THREADS, 1)
    fa_bwd_dkdv_persistent_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                                  const float* __restrict__ LSE, const float* __restrict__ Dvec,
                                  __nv_bfloat16* __restrict__ dK, __nv_bfloat16* __restrict__ dV, int BH, int N,
                                  float scale, float scale_log2) {
  using C = Dkdv3Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sKV = sbase + C::OFF_KV, sQ = sbase + C::OFF_Q, sdO = sbase + C::OFF_DO;
  float* sLSE = reinterpret_cast<float*>(smem + C::OFF_LSE);
  float* sDD = reinterpret_cast<float*>(smem + C::OFF_DD);
  const uint32_t bars = sbase + C::OFF_BAR;
  auto bar = [&](int i) { return bars + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM_SLOT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int NKT = (N + C::BK - 1) / C::BK;
  const int NQT = (N + C::BQ - 1) / C::BQ;
  const int units = BH * NKT;
  const int G = CAUSAL ? causal_head_group(BH, N, D) : BH;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(C::B_KV_FULL + s), 1);
      mbar_init(bar(C::B_KV_EMPTY + s), 1);
      mbar_init(bar(C::B_S_FULL + s), 1);
      mbar_init(bar(C::B_P_FULL + s), 128);
    }
    for (int s = 0; s < C::ST; ++s) {
      mbar_init(bar(C::B_Q_FULL + s), 33);  // expect_tx arrive + 32 lanes writing LSE and D
      mbar_init(bar(C::B_Q_EMPTY + s), 1);
    }
    mbar_init(bar(C::B_DKV_FULL), 1);
    mbar_init(bar(C::B_DKV_EMPTY), 128);
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

  // Each role's setmaxnreg dominates its code; the paths join only at the teardown.
  if (warp < 4) {
    regs_dec<C::REGS_CONTROL>();
    if (warp == 0) {
      // ------------------------------------------------------------ loads (whole warp)
      if (lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmdO);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
      }
      uint32_t gq = 0;
      int unit_it = 0;
      bool ok = true;
      for (int k = 0, u = blockIdx.x; u < units && ok; u = serpentine_unit(++k, blockIdx.x, gridDim.x), ++unit_it) {
        int bh, kt;
        dkdv3_decode_unit(u, BH, NKT, G, CAUSAL, bh, kt);
        const int i0 = CAUSAL ? (kt * C::BK) / C::BQ : 0;
        const int nt = NQT - i0;
        const int slot = unit_it & 1;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(bar(C::B_KV_EMPTY + slot), ((unit_it >> 1) & 1) ^ 1,
                                                      B3_PROD_KVE))))
          break;
        if (lane == 0) {
          const uint32_t kvb = sKV + slot * C::KV_BUF;
          mbar_arrive_expect_tx(bar(C::B_KV_FULL + slot), 2 * C::K_TILE);
          for (int c = 0; c < C::CH; ++c) {
            tma_load_3d(kvb + c * C::KCHUNK, &tmK, bar(C::B_KV_FULL + slot), c * 64, kt * C::BK, bh);
            tma_load_3d(kvb + C::K_TILE + c * C::KCHUNK, &tmV, bar(C::B_KV_FULL + slot), c * 64, kt * C::BK, bh);
          }
        }
        for (int it = 0; it < nt; ++it, ++gq) {
          const int st = gq % C::ST;
          const int qi = i0 + it;
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(bar(C::B_Q_EMPTY + st), ((gq / C::ST) & 1) ^ 1,
                                                        B3_PROD_QE))))
            break;
          if (lane == 0) {
            mbar_arrive_expect_tx(bar(C::B_Q_FULL + st), 2 * C::Q_TILE);
            for (int c = 0; c < C::CH; ++c) {
              tma_load_3d(sQ + st * C::Q_TILE + c * C::QCHUNK, &tmQ, bar(C::B_Q_FULL + st), c * 64, qi * C::BQ, bh);
              tma_load_3d(sdO + st * C::Q_TILE + c * C::QCHUNK, &tmdO, bar(C::B_Q_FULL + st), c * 64, qi * C::BQ,
                          bh);
            }
          }
#pragma unroll
          for (int e = lane; e < C::BQ; e += 32) {
            const int q = qi * C::BQ + e;
            const bool valid = q < N;
            sLSE[st * C::BQ + e] = valid ? LSE[static_cast<size_t>(bh) * N + q] * kLog2e : INFINITY;
            sDD[st * C::BQ + e] = valid ? Dvec[static_cast<size_t>(bh) * N + q] : 0.f;
          }
          mbar_arrive(bar(C::B_Q_FULL + st));
        }
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer (whole warp, uniform values)
      constexpr uint32_t IDESC_T = idesc_bf16(128, C::BQ, false, false);  // S^T, dP^T: M=128 keys, N=64 queries
      constexpr uint32_t IDESC_G = idesc_bf16(128, D, false, true);        // dV, dK: B operand MN-major
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
        mma_ts_k64(d_tmem, a_tmem, sdesc_make(sdesc_lo(b_smem, C::QCHUNK), sdesc_hi(1024)), IDESC_G, acc ? 1u : 0u);
      };
      uint32_t g = 0;
      int unit_it = 0;
      bool ok = true;
      for (int k = 0, u = blockIdx.x; u < units && ok; u = serpentine_unit(++k, blockIdx.x, gridDim.x), ++unit_it) {
        int bh, kt;
        dkdv3_decode_unit(u, BH, NKT, G, CAUSAL, bh, kt);
        const int i0 = CAUSAL ? (kt * C::BK) / C::BQ : 0;
        const int nt = NQT - i0;
        const int slot = unit_it & 1;
        const uint32_t sK = sKV + slot * C::KV_BUF, sV = sK + C::K_TILE;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(bar(C::B_KV_FULL + slot), (unit_it >> 1) & 1, B3_MMA_KV))))
          break;
        tc_fence_after();
        for (int it = 0; it <= nt && ok; ++it) {
          if (it < nt) {
            const uint32_t gi = g + it;
            const int st = gi % C::ST, b = gi & 1;
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(bar(C::B_Q_FULL + st), (gi / C::ST) & 1, B3_MMA_Q))))
              break;
            tc_fence_after();
            issue_t(tmem + C::TM_S + b * 64, sK, sQ + st * C::Q_TILE);
            issue_t(tmem + C::TM_DP + b * 64, sV, sdO + st * C::Q_TILE);
            tc_commit_warp(bar(C::B_S_FULL + b));
          }
          if (it > 0) {
            const uint32_t pgi = g + it - 1;
            const int pst = pgi % C::ST, pb = pgi & 1;
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(bar(C::B_P_FULL + pb), (pgi >> 1) & 1, B3_MMA_P)))) break;
            // the unit's first dV/dK MMA overwrites the accumulators: the
            // previous unit's epilogue must have read them
            if (it == 1 && unit_it > 0 &&
                !(ok = __all_sync(0xffffffffu, mbar_wait(bar(C::B_DKV_EMPTY), (unit_it - 1) & 1, B3_MMA_DE))))
              break;
            tc_fence_after();
            issue_g(tmem + C::TM_DV, tmem + C::TM_S + pb * 64, sdO + pst * C::Q_TILE, it > 1);
            issue_g(tmem + C::TM_DK, tmem + C::TM_DP + pb * 64, sQ + pst * C::Q_TILE, it > 1);
            tc_commit_warp(bar(C::B_Q_EMPTY + pst));
          }
        }
        if (!ok) break;
        tc_commit_warp(bar(C::B_DKV_FULL));
        tc_commit_warp(bar(C::B_KV_EMPTY + slot));
        g += nt;
      }
      // The last unit's K/V-empty arrival is the last one this thread's
      // commits make; wait for it so no arrival lands after the CTA has exited.
      if (ok && unit_it > 0)
        (void)__all_sync(0xffffffffu, mbar_wait(bar(C::B_KV_EMPTY + ((unit_it - 1) & 1)), ((unit_it - 1) >> 1) & 1,
                                                 B3_MMA_KV));
    }
    // teardown (each branch has its own, so the register regions never merge)
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc(tmem, C::TMEM_COLS);
    }
  } else if (warp < 8) {
    regs_dec<C::REGS_EPILOGUE>();
    // ------------------------------------------------------------ dK/dV epilogue warpgroup
    const int sp = warp & 3;
    const int r = sp * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(sp * 32) << 16;
    int unit_it = 0;
    for (int k = 0, u = blockIdx.x; u < units; u = serpentine_unit(++k, blockIdx.x, gridDim.x), ++unit_it) {
      int bh, kt;
      dkdv3_decode_unit(u, BH, NKT, G, CAUSAL, bh, kt);
      const int key = kt * C::BK + r;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(C::B_DKV_FULL), unit_it & 1, B3_EP_DKV))) break;
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
          if (which == 1 && c == D / 32 - 1) {  // the accumulators are read: the next unit may overwrite them
            tc_fence_before();
            mbar_arrive(bar(C::B_DKV_EMPTY));
          }
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
    tc_fence_before();
    __syncthreads();
  } else {
    regs_inc<C::REGS_GRAD>();
    // ------------------------------------------------------------ gradient warpgroup
    const int sp = warp & 3;
    const int r = sp * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(sp * 32) << 16;
    uint32_t g = 0;
    bool ok = true;
    for (int k = 0, u = blockIdx.x; u < units && ok; u = serpentine_unit(++k, blockIdx.x, gridDim.x)) {
      int bh, kt;
      dkdv3_decode_unit(u, BH, NKT, G, CAUSAL, bh, kt);
      const int i0 = CAUSAL ? (kt * C::BK) / C::BQ : 0;
      const int nt = NQT - i0;
      const int key = kt * C::BK + r;
      for (int it = 0; it < nt; ++it) {
        const uint32_t gi = g + it;
        const int st = gi % C::ST, b = gi & 1;
        const int qi = i0 + it;
        bool w = mbar_wait(bar(C::B_S_FULL + b), (gi >> 1) & 1, B3_SM_S);
        w = w && mbar_wait(bar(C::B_Q_FULL + st), (gi / C::ST) & 1, B3_SM_Q);
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
        const float* lse2 = sLSE + st * C::BQ;
        const float* dd = sDD + st * C::BQ;
        const bool diag = CAUSAL && (qi * C::BQ < kt * C::BK + C::BK);
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {  // 32 queries -> 16 packed columns of P^T and of dS^T
          uint32_t pp[16], dsp[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int e = 32 * ch + 2 * c;
            float p0 = ex2(fmaf(__uint_as_float(sr[e]), scale_log2, -lse2[e]));
            float p1 = ex2(fmaf(__uint_as_float(sr[e + 1]), scale_log2, -lse2[e + 1]));
            if (diag) {
              const int q0 = qi * C::BQ + e;
              if (q0 < key) p0 = 0.f;
              if (q0 + 1 < key) p1 = 0.f;
            }
            const float ds0 = p0 * (__uint_as_float(dr[e]) - dd[e]);
            const float ds1 = p1 * (__uint_as_float(dr[e + 1]) - dd[e + 1]);
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
      g += nt;
    }
    tc_fence_before();
    __syncthreads();
  }
}

}  // namespace fa
