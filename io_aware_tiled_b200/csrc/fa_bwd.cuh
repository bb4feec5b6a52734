// fa_bwd.cuh -- backward kernels of tiled, IO-aware exact attention for sm_100a.
//
// The backward keeps only O and the per-row statistic and recomputes the
// attention weights tile by tile ("图解Flash Attention运算原理", 总结:
// Recomputation keeps the softmax statistics and recomputes P when needed).
// With LSE_i = ln sum_j exp(S_ij) stored by the forward, P_ij = exp(S_ij -
// LSE_i) exactly.  The gradients are the analytic gradient of the definition
// for the loss sum(dO * O) (not printed on the pages):
//   D_i = sum_c dO_ic O_ic               (preprocess, over the bf16 O given)
//   dV_j = sum_i P_ij dO_i,   dP_ij = dO_i . V_j,   dS_ij = P_ij (dP_ij - D_i)
//   dK_j = scale sum_i dS_ij Q_i,   dQ_i = scale sum_j dS_ij K_j
//
// Kernels (all on the caller's stream):
//   1. fa_bwd_preprocess_kernel: D into the workspace (memory-bound pass).
//   2. fa_bwd_dkdv_kernel: one CTA per (head, 128-key tile).  Loops over the
//      64-row query tiles that can see the keys; per tile it computes
//      S^T = K Q^T and dP^T = V dO^T (tcgen05, M = 128 keys) into tensor
//      memory, then P^T and dS^T (bf16, written back over S^T and dP^T), then
//      dV += P^T dO and dK += dS^T Q with the A operand read from tensor
//      memory.  S^T/dP^T are double-buffered so the next tile's two GEMMs run
//      while this tile's exponentials run.
//   3. fa_bwd_dq_kernel: one CTA per (head, 128-row query tile); loops over
//      64-key tiles: S = Q K^T, dP = dO V^T, dS, dQ += dS K.  Keeping dQ in its
//      own kernel costs two extra GEMMs per tile but needs no atomics, so dQ
//      is deterministic and written once as bf16.
#pragma once

#include "fa_device.cuh"

namespace fa {

// ---------------------------------------------------------------------------
// D_i = sum_c dO_ic * O_ic  (fp32), one group of D/8 threads per row.  With
// ZERO the same pass also clears the row of the fp32 dQ accumulator that the
// fused backward adds into (8 floats per thread).
// ---------------------------------------------------------------------------
template <int D, bool ZERO = false>
__global__ void __launch_bounds__(256) fa_bwd_preprocess_kernel(const __nv_bfloat16* __restrict__ O,
                                                                 const __nv_bfloat16* __restrict__ dO,
                                                                 float* __restrict__ Dout, long long rows,
                                                                 float* __restrict__ dQacc = nullptr) {
  constexpr int G = D / 8;  // threads per row; each reads 16 bytes of O and of dO
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long row = gid / G;
  const int part = static_cast<int>(gid % G);
  float acc = 0.f;
  if (ZERO && row < rows) {
    float4* z = reinterpret_cast<float4*>(dQacc + row * D + part * 8);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  if (row < rows) {
    const uint4 a = *reinterpret_cast<const uint4*>(O + row * D + part * 8);
    const uint4 b = *reinterpret_cast<const uint4*>(dO + row * D + part * 8);
    const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 fa2 = __bfloat1622float2(pa[e]);
      const float2 fb2 = __bfloat1622float2(pb[e]);
      acc = fmaf(fa2.x, fb2.x, acc);
      acc = fmaf(fa2.y, fb2.y, acc);
    }
  }
#pragma unroll
  for (int off = G / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (part == 0 && row < rows) Dout[row] = acc;
}

// ---------------------------------------------------------------------------
// dK, dV
// ---------------------------------------------------------------------------
template <int D>
struct DkdvCfg {
  static constexpr int BK = 128;                     // keys per CTA (MMA M)
  static constexpr int BQ = 64;                      // queries per tile (MMA N of S^T)
  static constexpr int CH = D / 64;
  static constexpr int KCHUNK = BK * 128;            // one 64-column chunk of the key tile
  static constexpr int QCHUNK = BQ * 128;            // one 64-column chunk of a query tile
  static constexpr int K_TILE = BK * D * 2;
  static constexpr int Q_TILE = BQ * D * 2;
  static constexpr int ST = (D == 128) ? 3 : 4;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + K_TILE;
  static constexpr int OFF_Q = OFF_V + K_TILE;       // ST stages of Q tiles
  static constexpr int OFF_DO = OFF_Q + ST * Q_TILE; // ST stages of dO tiles
  static constexpr int OFF_LSE = OFF_DO + ST * Q_TILE;  // ST x BQ floats (LSE * log2 e)
  static constexpr int OFF_DD = OFF_LSE + ST * BQ * 4;  // ST x BQ floats (D)
  static constexpr int OFF_BAR = OFF_DD + ST * BQ * 4;
  static constexpr int B_KV_FULL = 0, B_Q_FULL = 1, B_Q_EMPTY = 1 + ST, B_S_FULL = 1 + 2 * ST,
                       B_P_FULL = B_S_FULL + 2, B_DKV_FULL = B_P_FULL + 2;
  static constexpr int NUM_BARS = B_DKV_FULL + 1;
  static constexpr int OFF_TMEM_SLOT = OFF_BAR + NUM_BARS * 8;
  static constexpr int USED = OFF_TMEM_SLOT + 16 + 1024;
  // at least 120 KB so that one CTA (and one tensor-memory allocation) sits on an SM
  static constexpr int SMEM_BYTES = USED > 120 * 1024 ? USED : 120 * 1024;
  static constexpr uint32_t TM_S = 0, TM_DP = 128, TM_DV = 256, TM_DK = 256 + D;  // S/dP: two 64-col buffers
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int THREADS = 192;  // warp 0 loads, warp 1 MMA, warps 2-5 one warpgroup (thread = key)
};

enum BwdWaitSite : unsigned int {
  BW_PROD_QE = 32, BW_MMA_KV, BW_MMA_Q, BW_MMA_P, BW_SM_S, BW_SM_Q, BW_SM_DKV,
  BQ_PROD_KVE, BQ_MMA_Q, BQ_MMA_KV, BQ_MMA_P, BQ_SM_S, BQ_SM_DQ
};

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(DkdvCfg<D>::THREADS, 1)
    fa_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                       const float* __restrict__ LSE, const float* __restrict__ Dvec,
                       __nv_bfloat16* __restrict__ dK, __nv_bfloat16* __restrict__ dV, int N, float scale,
                       float scale_log2) {
  using C = DkdvCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sK = sbase + C::OFF_K, sV = sbase + C::OFF_V, sQ = sbase + C::OFF_Q, sdO = sbase + C::OFF_DO;
  float* sLSE = reinterpret_cast<float*>(smem + C::OFF_LSE);
  float* sDD = reinterpret_cast<float*>(smem + C::OFF_DD);
  const uint32_t bars = sbase + C::OFF_BAR;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM_SLOT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Block order: head-major without a mask (the blocks resident together
  // share one head's Q and dO in L2); with the causal mask, the longest key
  // tiles (the first ones) of every head of a group (causal_head_group) come
  // first, so the last wave is short.
  const int NKT = (N + C::BK - 1) / C::BK;
  const int BHg = gridDim.x / NKT;
  int bh, kt;
  if (CAUSAL) {
    causal_grouped_unit(blockIdx.x, BHg, NKT, causal_head_group(BHg, N, D), bh, kt);
  } else {
    bh = blockIdx.x / NKT;
    kt = blockIdx.x - bh * NKT;
  }
  const int NQT = (N + C::BQ - 1) / C::BQ;
  const int i0 = CAUSAL ? (kt * C::BK) / C::BQ : 0;  // first query tile that sees these keys
  const int nt = NQT - i0;                           // >= 1: the tile holding query kt*BK exists

  if (threadIdx.x == 0) {
    mbar_init(bars + 8 * C::B_KV_FULL, 1);
    for (int s = 0; s < C::ST; ++s) {
      mbar_init(bars + 8 * (C::B_Q_FULL + s), 33);  // expect_tx arrive + 32 lanes writing LSE and D
      mbar_init(bars + 8 * (C::B_Q_EMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bars + 8 * (C::B_S_FULL + b), 1);
      mbar_init(bars + 8 * (C::B_P_FULL + b), 128);
    }
    mbar_init(bars + 8 * C::B_DKV_FULL, 1);
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

  if (warp == 0) {
    // ------------------------------------------------------------ loads (whole warp)
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmdO);
      mbar_arrive_expect_tx(bars + 8 * C::B_KV_FULL, 2 * C::K_TILE);
      for (int c = 0; c < C::CH; ++c) {
        tma_load_3d(sK + c * C::KCHUNK, &tmK, bars + 8 * C::B_KV_FULL, c * 64, kt * C::BK, bh);
        tma_load_3d(sV + c * C::KCHUNK, &tmV, bars + 8 * C::B_KV_FULL, c * 64, kt * C::BK, bh);
      }
    }
    for (int it = 0; it < nt; ++it) {
      const int st = it % C::ST;
      const int qi = i0 + it;
      const bool ok = mbar_wait(bars + 8 * (C::B_Q_EMPTY + st), ((it / C::ST) & 1) ^ 1, BW_PROD_QE);
      if (!__all_sync(0xffffffffu, ok)) break;
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
        sLSE[st * C::BQ + e] = valid ? LSE[static_cast<size_t>(bh) * N + q] * kLog2e : INFINITY;
        sDD[st * C::BQ + e] = valid ? Dvec[static_cast<size_t>(bh) * N + q] : 0.f;
      }
      mbar_arrive(bars + 8 * (C::B_Q_FULL + st));
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    {  // whole warp, warp-uniform values; one elected lane issues each MMA / commit
      constexpr uint32_t IDESC_T = idesc_bf16(128, C::BQ, false, false);  // S^T, dP^T: M=128 keys, N=64 queries
      constexpr uint32_t IDESC_G = idesc_bf16(128, D, false, true);        // dV, dK: B operand MN-major
      // S^T / dP^T: K = d; A (keys) and B (queries) K-major in shared memory.
      auto issue_t = [&](uint32_t d_tmem, uint32_t a_smem, uint32_t b_smem) {
        const uint32_t hi = sdesc_hi(1024);
        const uint64_t a0 = sdesc_make(sdesc_lo(a_smem, 16), hi), b0 = sdesc_make(sdesc_lo(b_smem, 16), hi);
        if (D == 128)
          mma_ss_k128(d_tmem, a0, sdesc_make(sdesc_lo(a_smem + C::KCHUNK, 16), hi), b0,
                      sdesc_make(sdesc_lo(b_smem + C::QCHUNK, 16), hi), IDESC_T, 0u);
        else
          mma_ss_k64(d_tmem, a0, b0, IDESC_T, 0u);
      };
      // dV / dK: K = 64 queries; A (P^T or dS^T) from tensor memory, B MN-major.
      auto issue_g = [&](uint32_t d_tmem, uint32_t a_tmem, uint32_t b_smem, bool acc) {
        mma_ts_k64(d_tmem, a_tmem, sdesc_make(sdesc_lo(b_smem, C::QCHUNK), sdesc_hi(1024)), IDESC_G, acc ? 1u : 0u);
      };
      bool ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * C::B_KV_FULL, 0, BW_MMA_KV));
      tc_fence_after();
      for (int it = 0; it <= nt && ok; ++it) {
        if (it < nt) {
          const int st = it % C::ST, b = it & 1;
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * (C::B_Q_FULL + st), (it / C::ST) & 1, BW_MMA_Q)))) break;
          tc_fence_after();
          issue_t(tmem + C::TM_S + b * 64, sK, sQ + st * C::Q_TILE);
          issue_t(tmem + C::TM_DP + b * 64, sV, sdO + st * C::Q_TILE);
          tc_commit_warp(bars + 8 * (C::B_S_FULL + b));
        }
        if (it > 0) {
          const int pit = it - 1, pst = pit % C::ST, pb = pit & 1;
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * (C::B_P_FULL + pb), (pit >> 1) & 1, BW_MMA_P)))) break;
          tc_fence_after();
          issue_g(tmem + C::TM_DV, tmem + C::TM_S + pb * 64, sdO + pst * C::Q_TILE, pit > 0);
          issue_g(tmem + C::TM_DK, tmem + C::TM_DP + pb * 64, sQ + pst * C::Q_TILE, pit > 0);
          tc_commit_warp(bars + 8 * (C::B_Q_EMPTY + pst));
        }
      }
      if (ok) tc_commit_warp(bars + 8 * C::B_DKV_FULL);
    }
  } else {
    // ------------------------------------------------------------ softmax-gradient warpgroup
    const int sp = warp & 3;
    const int r = sp * 32 + lane;
    const int key = kt * C::BK + r;
    const uint32_t lane_off = static_cast<uint32_t>(sp * 32) << 16;
    bool ok = true;
    for (int it = 0; it < nt; ++it) {
      const int st = it % C::ST, b = it & 1;
      const int qi = i0 + it;
      bool w = mbar_wait(bars + 8 * (C::B_S_FULL + b), (it >> 1) & 1, BW_SM_S);
      w = w && mbar_wait(bars + 8 * (C::B_Q_FULL + st), (it / C::ST) & 1, BW_SM_Q);
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
      mbar_arrive(bars + 8 * (C::B_P_FULL + b));
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(bars + 8 * C::B_DKV_FULL, 0, BW_SM_DKV))) {
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

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// dQ
// ---------------------------------------------------------------------------
template <int D>
struct DqCfg {
  static constexpr int BQ = 128;                     // query rows per CTA (MMA M)
  static constexpr int BK = 64;                      // keys per tile
  static constexpr int CH = D / 64;
  static constexpr int QCHUNK = BQ * 128;
  static constexpr int KCHUNK = BK * 128;
  static constexpr int Q_TILE = BQ * D * 2;
  static constexpr int K_TILE = BK * D * 2;
  static constexpr int ST = (D == 128) ? 3 : 4;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = OFF_Q + Q_TILE;
  static constexpr int OFF_K = OFF_DO + Q_TILE;      // ST stages
  static constexpr int OFF_V = OFF_K + ST * K_TILE;  // ST stages
  static constexpr int OFF_BAR = OFF_V + ST * K_TILE;
  static constexpr int B_Q_FULL = 0, B_KV_FULL = 1, B_KV_EMPTY = 1 + ST, B_S_FULL = 1 + 2 * ST,
                       B_P_FULL = B_S_FULL + 2, B_DQ_FULL = B_P_FULL + 2;
  static constexpr int NUM_BARS = B_DQ_FULL + 1;
  static constexpr int OFF_TMEM_SLOT = OFF_BAR + NUM_BARS * 8;
  static constexpr int USED = OFF_TMEM_SLOT + 16 + 1024;
  static constexpr int SMEM_BYTES = USED > 120 * 1024 ? USED : 120 * 1024;
  static constexpr uint32_t TM_S = 0, TM_DP = 128, TM_DQ = 256;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int THREADS = 192;
};

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(DqCfg<D>::THREADS, 1)
    fa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                     const float* __restrict__ LSE, const float* __restrict__ Dvec, __nv_bfloat16* __restrict__ dQ,
                     int N, float scale, float scale_log2) {
  using C = DqCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::OFF_Q, sdO = sbase + C::OFF_DO, sK = sbase + C::OFF_K, sV = sbase + C::OFF_V;
  const uint32_t bars = sbase + C::OFF_BAR;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM_SLOT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Block order as in the dK/dV kernel: head-major without a mask, longest
  // query tiles (the last ones) of every head of a group first with it.
  const int NQT = (N + C::BQ - 1) / C::BQ;
  const int BHg = gridDim.x / NQT;
  int bh, qt;
  if (CAUSAL) {
    int r;
    causal_grouped_unit(blockIdx.x, BHg, NQT, causal_head_group(BHg, N, D), bh, r);
    qt = NQT - 1 - r;
  } else {
    bh = blockIdx.x / NQT;
    qt = blockIdx.x - bh * NQT;
  }
  const int NKT = (N + C::BK - 1) / C::BK;
  const int nt = CAUSAL ? min(NKT, (qt * C::BQ + C::BQ - 1) / C::BK + 1) : NKT;

  if (threadIdx.x == 0) {
    mbar_init(bars + 8 * C::B_Q_FULL, 1);
    for (int s = 0; s < C::ST; ++s) {
      mbar_init(bars + 8 * (C::B_KV_FULL + s), 1);
      mbar_init(bars + 8 * (C::B_KV_EMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bars + 8 * (C::B_S_FULL + b), 1);
      mbar_init(bars + 8 * (C::B_P_FULL + b), 128);
    }
    mbar_init(bars + 8 * C::B_DQ_FULL, 1);
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

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(bars + 8 * C::B_Q_FULL, 2 * C::Q_TILE);
      for (int c = 0; c < C::CH; ++c) {
        tma_load_3d(sQ + c * C::QCHUNK, &tmQ, bars + 8 * C::B_Q_FULL, c * 64, qt * C::BQ, bh);
        tma_load_3d(sdO + c * C::QCHUNK, &tmdO, bars + 8 * C::B_Q_FULL, c * 64, qt * C::BQ, bh);
      }
      for (int it = 0; it < nt; ++it) {
        const int st = it % C::ST;
        if (!mbar_wait(bars + 8 * (C::B_KV_EMPTY + st), ((it / C::ST) & 1) ^ 1, BQ_PROD_KVE)) break;
        mbar_arrive_expect_tx(bars + 8 * (C::B_KV_FULL + st), 2 * C::K_TILE);
        for (int c = 0; c < C::CH; ++c) {
          tma_load_3d(sK + st * C::K_TILE + c * C::KCHUNK, &tmK, bars + 8 * (C::B_KV_FULL + st), c * 64,
                      it * C::BK, bh);
          tma_load_3d(sV + st * C::K_TILE + c * C::KCHUNK, &tmV, bars + 8 * (C::B_KV_FULL + st), c * 64,
                      it * C::BK, bh);
        }
      }
    }
  } else if (warp == 1) {
    {  // whole warp, warp-uniform values; one elected lane issues each MMA / commit
      constexpr uint32_t IDESC_S = idesc_bf16(128, C::BK, false, false);  // S, dP: M=128 queries, N=64 keys
      constexpr uint32_t IDESC_Q = idesc_bf16(128, D, false, true);       // dQ: B (K tile) MN-major
      // S / dP: K = d; A (queries) and B (keys) K-major in shared memory.
      auto issue_s = [&](uint32_t d_tmem, uint32_t a_smem, uint32_t b_smem) {
        const uint32_t hi = sdesc_hi(1024);
        const uint64_t a0 = sdesc_make(sdesc_lo(a_smem, 16), hi), b0 = sdesc_make(sdesc_lo(b_smem, 16), hi);
        if (D == 128)
          mma_ss_k128(d_tmem, a0, sdesc_make(sdesc_lo(a_smem + C::QCHUNK, 16), hi), b0,
                      sdesc_make(sdesc_lo(b_smem + C::KCHUNK, 16), hi), IDESC_S, 0u);
        else
          mma_ss_k64(d_tmem, a0, b0, IDESC_S, 0u);
      };
      bool ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * C::B_Q_FULL, 0, BQ_MMA_Q));
      tc_fence_after();
      for (int it = 0; it <= nt && ok; ++it) {
        if (it < nt) {
          const int st = it % C::ST, b = it & 1;
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * (C::B_KV_FULL + st), (it / C::ST) & 1, BQ_MMA_KV)))) break;
          tc_fence_after();
          issue_s(tmem + C::TM_S + b * 64, sQ, sK + st * C::K_TILE);
          issue_s(tmem + C::TM_DP + b * 64, sdO, sV + st * C::K_TILE);
          tc_commit_warp(bars + 8 * (C::B_S_FULL + b));
        }
        if (it > 0) {
          const int pit = it - 1, pst = pit % C::ST, pb = pit & 1;
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * (C::B_P_FULL + pb), (pit >> 1) & 1, BQ_MMA_P)))) break;
          tc_fence_after();
          // dQ += dS K: K = 64 keys; dS from tensor memory, K tile MN-major.
          mma_ts_k64(tmem + C::TM_DQ, tmem + C::TM_DP + pb * 64,
                     sdesc_make(sdesc_lo(sK + pst * C::K_TILE, C::KCHUNK), sdesc_hi(1024)), IDESC_Q,
                     pit > 0 ? 1u : 0u);
          tc_commit_warp(bars + 8 * (C::B_KV_EMPTY + pst));
        }
      }
      if (ok) tc_commit_warp(bars + 8 * C::B_DQ_FULL);
    }
  } else {
    const int sp = warp & 3;
    const int r = sp * 32 + lane;
    const int q = qt * C::BQ + r;
    const uint32_t lane_off = static_cast<uint32_t>(sp * 32) << 16;
    const bool qvalid = q < N;
    const float lse2 = qvalid ? LSE[static_cast<size_t>(bh) * N + q] * kLog2e : 0.f;
    const float dd = qvalid ? Dvec[static_cast<size_t>(bh) * N + q] : 0.f;
    bool ok = true;
    for (int it = 0; it < nt; ++it) {
      const int b = it & 1;
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * (C::B_S_FULL + b), (it >> 1) & 1, BQ_SM_S))))
        break;
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
      const int kbase = it * C::BK;
      const bool need_mask = (kbase + C::BK > N) || (CAUSAL && kbase + C::BK - 1 > qt * C::BQ);
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {  // 32 keys -> 16 packed columns of dS
        uint32_t dsp[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int e = 32 * ch + 2 * c;
          float p0 = ex2(fmaf(__uint_as_float(sr[e]), scale_log2, -lse2));
          float p1 = ex2(fmaf(__uint_as_float(sr[e + 1]), scale_log2, -lse2));
          if (need_mask) {
            const int k0 = kbase + e;
            if (k0 >= N || (CAUSAL && k0 > q)) p0 = 0.f;
            if (k0 + 1 >= N || (CAUSAL && k0 + 1 > q)) p1 = 0.f;
          }
          dsp[c] = pack_bf16(p0 * (__uint_as_float(dr[e]) - dd), p1 * (__uint_as_float(dr[e + 1]) - dd));
        }
        tmem_st16(tP + ch * 16, dsp);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bars + 8 * (C::B_P_FULL + b));
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(bars + 8 * C::B_DQ_FULL, 0, BQ_SM_DQ))) {
      tc_fence_after();
      __nv_bfloat16* dst_row = dQ + (static_cast<size_t>(bh) * N + q) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t a[32];
        tmem_ld32(tmem + lane_off + C::TM_DQ + c * 32, a);
        tmem_ld_wait();
        reg_fence(a);
        if (qvalid) {
          uint4* dst = reinterpret_cast<uint4*>(dst_row + c * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 wv;
            wv.x = pack_bf16(__uint_as_float(a[8 * v + 0]) * scale, __uint_as_float(a[8 * v + 1]) * scale);
            wv.y = pack_bf16(__uint_as_float(a[8 * v + 2]) * scale, __uint_as_float(a[8 * v + 3]) * scale);
            wv.z = pack_bf16(__uint_as_float(a[8 * v + 4]) * scale, __uint_as_float(a[8 * v + 5]) * scale);
            wv.w = pack_bf16(__uint_as_float(a[8 * v + 6]) * scale, __uint_as_float(a[8 * v + 7]) * scale);
            dst[v] = wv;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fa
