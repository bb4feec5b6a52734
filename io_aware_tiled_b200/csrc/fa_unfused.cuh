// fa_unfused.cuh -- standard (unfused) attention forward for sm_100a: the
// comparison column of the memory-access table in "FlashAttention分块计算优化
// Transformer显存效率" (section 2.1, 内存访问模式对比).  The N x N score and
// probability matrices go through HBM, in 16-bit elements as in that table:
//
//   1. fa_unf_scores_kernel   S = scale * Q K^T    (fp16, written to HBM)
//   2. fa_unf_softmax_kernel  P = softmax_rows(S)  (bf16, written over S) and
//                             LSE = m + ln(sum)    (fp32)
//   3. fa_unf_pv_kernel       O = P V              (bf16)
//
// It exists to measure the HBM traffic the tiled kernels avoid; it computes the
// same O and LSE.  Causal masking is applied in step 2 only (the standard
// method computes every score).  S and P are stored [B*H][Nr][Nr] with
// Nr = N rounded up to 128, so every 128 x 128 tile is whole: rows >= N hold
// values no output reads, and columns >= N of P are written as zero.
//
// S is fp16 rather than bf16 because the softmax reads it back: fp16 keeps 3
// more mantissa bits for scores of moderate size.  P is bf16, the type of V,
// because one tcgen05.mma takes A and B of the same type.
#pragma once

#include <cuda_fp16.h>

#include "fa_device.cuh"

namespace fa {

enum UnfWaitSite : unsigned int { UW_S_TMA = 112, UW_S_MMA, UW_PV_FULL, UW_PV_EMPTY, UW_PV_DONE };

// ---------------------------------------------------------------------------
// 1. scores: one CTA per 128 x 128 tile of S, 4 warps
// ---------------------------------------------------------------------------
template <int D>
struct UnfScoresCfg {
  static constexpr int T = 128;
  static constexpr int CH = D / 64;           // 64-column chunks per row
  static constexpr int CHUNK = T * 128;       // bytes of one chunk of a 128-row tile
  static constexpr int TILE = T * D * 2;
  static constexpr int OFF_Q = 0, OFF_K = TILE, OFF_BAR = 2 * TILE;
  static constexpr int OFF_SLOT = OFF_BAR + 16;
  // at least 60 KB, so at most 3 blocks share an SM and their tensor memory
  // (3 x 128 of 512 columns) never runs out
  static constexpr int SMEM_USED = OFF_SLOT + 16 + 1024;
  static constexpr int SMEM_BYTES = SMEM_USED > 60 * 1024 ? SMEM_USED : 60 * 1024;
  static constexpr uint32_t TMEM_COLS = 128;
};

template <int D>
__global__ void __launch_bounds__(128)
    fa_unf_scores_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         __half* __restrict__ S, int NT, int Nr, float scale) {
  using C = UnfScoresCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::OFF_Q, sK = sbase + C::OFF_K;
  const uint32_t bar_full = sbase + C::OFF_BAR, bar_done = bar_full + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_SLOT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // block -> (head, query tile, key tile), key tiles fastest
  const long long t = blockIdx.x;
  const int kt = static_cast<int>(t % NT);
  const int qt = static_cast<int>((t / NT) % NT);
  const int bh = static_cast<int>(t / (static_cast<long long>(NT) * NT));

  if (threadIdx.x == 0) {
    mbar_init(bar_full, 1);
    mbar_init(bar_done, 1);
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

  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(bar_full, 2 * C::TILE);
    for (int c = 0; c < C::CH; ++c) {
      tma_load_3d(sQ + c * C::CHUNK, &tmQ, bar_full, c * 64, qt * C::T, bh);
      tma_load_3d(sK + c * C::CHUNK, &tmK, bar_full, c * 64, kt * C::T, bh);
    }
  }
  if (warp == 1) {
    if (__all_sync(0xffffffffu, mbar_wait(bar_full, 0, UW_S_TMA))) {
      tc_fence_after();
      constexpr uint32_t IDESC = idesc_bf16(128, 128, false, false);
      const uint32_t hi = sdesc_hi(1024);
      const uint64_t a0 = sdesc_make(sdesc_lo(sQ, 16), hi), b0 = sdesc_make(sdesc_lo(sK, 16), hi);
      if (D == 128)
        mma_ss_k128(tmem, a0, sdesc_make(sdesc_lo(sQ + C::CHUNK, 16), hi), b0,
                    sdesc_make(sdesc_lo(sK + C::CHUNK, 16), hi), IDESC, 0u);
      else
        mma_ss_k64(tmem, a0, b0, IDESC, 0u);
      tc_commit_warp(bar_done);
    }
  }
  // epilogue: each thread converts one row of the tile (128 fp32 -> fp16)
  if (mbar_wait(bar_done, 0, UW_S_MMA)) {
    tc_fence_after();
    const int row = qt * C::T + warp * 32 + lane;
    uint4* dst = reinterpret_cast<uint4*>(S + (static_cast<size_t>(bh) * Nr + row) * Nr + kt * C::T);
    const uint32_t taddr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t r[32];
      tmem_ld32(taddr + c * 32, r);
      tmem_ld_wait();
      reg_fence(r);
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __half2 h = __floats2half2_rn(__uint_as_float(r[8 * v + 2 * e]) * scale,
                                              __uint_as_float(r[8 * v + 2 * e + 1]) * scale);
          w[e] = *reinterpret_cast<const uint32_t*>(&h);
        }
        dst[c * 4 + v] = make_uint4(w[0], w[1], w[2], w[3]);
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
// 2. row softmax: one warp per row, 8 rows per block.  Pass 1 reads the row
// (16-byte loads, coalesced across the warp) and keeps a running max and sum
// per lane in base 2; a butterfly merges the lanes.  Pass 2 reads the row
// again (from L2) and writes P in place.
// ---------------------------------------------------------------------------
constexpr int kUnfSoftmaxRows = 8;

__global__ void __launch_bounds__(256)
    fa_unf_softmax_kernel(__half* __restrict__ S, float* __restrict__ LSE, long long rows, int N, int Nr,
                          int causal) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long gr = static_cast<long long>(blockIdx.x) * kUnfSoftmaxRows + warp;
  if (gr >= rows) return;
  const int bh = static_cast<int>(gr / N), i = static_cast<int>(gr % N);
  uint4* rowp = reinterpret_cast<uint4*>(S + (static_cast<size_t>(bh) * Nr + i) * Nr);
  const int nvis = causal ? i + 1 : N;  // keys this row sees: 0 .. nvis-1
  const int cvis = (nvis + 7) >> 3;     // 8-element chunks holding them
  const int nchunks = Nr >> 3;

  float m = -INFINITY, l = 0.f;
  for (int c = lane; c < cvis; c += 32) {
    const uint4 w = rowp[c];
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
    float t[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&ww[e]));
      t[2 * e] = (c * 8 + 2 * e < nvis) ? f.x * kLog2e : -INFINITY;
      t[2 * e + 1] = (c * 8 + 2 * e + 1 < nvis) ? f.y * kLog2e : -INFINITY;
    }
    float cm = t[0];
#pragma unroll
    for (int e = 1; e < 8; ++e) cm = fmaxf(cm, t[e]);
    if (cm > m) {  // m = -inf before the first chunk: ex2(-inf) = 0 and l is 0
      l *= ex2(m - cm);
      m = cm;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) l += ex2(t[e] - m);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float om = __shfl_xor_sync(0xffffffffu, m, off), ol = __shfl_xor_sync(0xffffffffu, l, off);
    const float nm = fmaxf(m, om);
    const float a = (m == -INFINITY) ? 0.f : ex2(m - nm);
    const float b = (om == -INFINITY) ? 0.f : ex2(om - nm);
    l = l * a + ol * b;
    m = nm;
  }
  // every row sees key 0, so m is finite and l >= 1 here
  if (lane == 0) LSE[gr] = (m + __log2f(l)) * kLn2;
  const float inv_l = 1.f / l;
  for (int c = lane; c < nchunks; c += 32) {
    uint4 out = make_uint4(0u, 0u, 0u, 0u);
    if (c < cvis) {
      const uint4 w = rowp[c];
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
      uint32_t p[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&ww[e]));
        const float p0 = (c * 8 + 2 * e < nvis) ? ex2(fmaf(f.x, kLog2e, -m)) * inv_l : 0.f;
        const float p1 = (c * 8 + 2 * e + 1 < nvis) ? ex2(fmaf(f.y, kLog2e, -m)) * inv_l : 0.f;
        p[e] = pack_bf16(p0, p1);
      }
      out = make_uint4(p[0], p[1], p[2], p[3]);
    }
    rowp[c] = out;
  }
}

// ---------------------------------------------------------------------------
// 3. O = P V: one CTA per (head, 128-row query tile), K loop over the keys in
// steps of 64 through a 4-stage ring.  Warp 0 loads (TMA), warp 1 issues the
// MMAs (A = P tile K-major, B = V tile MN-major, both in shared memory), all
// four warps convert the fp32 accumulator to bf16 rows of O.
// ---------------------------------------------------------------------------
template <int D>
struct UnfPvCfg {
  static constexpr int BK = 64;                  // keys per stage
  static constexpr int ST = 4;                   // ring depth
  static constexpr int A_STAGE = 128 * BK * 2;   // P tile: 128 rows x 64 keys
  static constexpr int B_CHUNK = BK * 64 * 2;    // V tile: 64 keys x 64 columns
  static constexpr int B_STAGE = (D / 64) * B_CHUNK;
  static constexpr int OFF_A = 0, OFF_B = ST * A_STAGE, OFF_BAR = OFF_B + ST * B_STAGE;
  static constexpr int B_FULL = 0, B_EMPTY = ST, B_DONE = 2 * ST, NUM_BARS = 2 * ST + 1;
  static constexpr int OFF_SLOT = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_SLOT + 16 + 1024;  // 1 block per SM at d=128, 2 at d=64
  static constexpr uint32_t TMEM_COLS = D;
};

template <int D>
__global__ void __launch_bounds__(128)
    fa_unf_pv_kernel(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmV,
                     __nv_bfloat16* __restrict__ O, int N, int Nr) {
  using C = UnfPvCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sA = sbase + C::OFF_A, sB = sbase + C::OFF_B, bars = sbase + C::OFF_BAR;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_SLOT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NT = Nr / 128;
  const int qt = blockIdx.x % NT, bh = blockIdx.x / NT;
  const int nk = Nr / C::BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::ST; ++s) {
      mbar_init(bars + 8 * (C::B_FULL + s), 1);
      mbar_init(bars + 8 * (C::B_EMPTY + s), 1);
    }
    mbar_init(bars + 8 * C::B_DONE, 1);
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
      for (int it = 0; it < nk; ++it) {
        const int s = it % C::ST;
        const uint32_t ph = (it / C::ST) & 1;
        if (!mbar_wait(bars + 8 * (C::B_EMPTY + s), ph ^ 1, UW_PV_EMPTY)) break;
        mbar_arrive_expect_tx(bars + 8 * (C::B_FULL + s), C::A_STAGE + C::B_STAGE);
        tma_load_3d(sA + s * C::A_STAGE, &tmP, bars + 8 * (C::B_FULL + s), it * C::BK, qt * 128, bh);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(sB + s * C::B_STAGE + c * C::B_CHUNK, &tmV, bars + 8 * (C::B_FULL + s), c * 64, it * C::BK,
                      bh);
      }
    }
  } else if (warp == 1) {
    constexpr uint32_t IDESC = idesc_bf16(128, D, false, true);
    const uint32_t hi = sdesc_hi(1024);
    bool ok = true;
    for (int it = 0; it < nk; ++it) {
      const int s = it % C::ST;
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * (C::B_FULL + s), (it / C::ST) & 1, UW_PV_FULL))))
        break;
      tc_fence_after();
      mma_ss_k64_bmn(tmem, sdesc_make(sdesc_lo(sA + s * C::A_STAGE, 16), hi),
                     sdesc_make(sdesc_lo(sB + s * C::B_STAGE, C::B_CHUNK), hi), IDESC, it > 0 ? 1u : 0u);
      // The producer reuses a stage only for iteration it + ST; the last
      // stages get no EMPTY commit, so the DONE commit below is this thread's
      // last arrival and none lands after the block has exited.
      if (it + C::ST < nk) tc_commit_warp(bars + 8 * (C::B_EMPTY + s));
    }
    if (ok) tc_commit_warp(bars + 8 * C::B_DONE);
  }
  __syncwarp();
  if (mbar_wait(bars + 8 * C::B_DONE, 0, UW_PV_DONE)) {
    tc_fence_after();
    const int row = qt * 128 + warp * 32 + lane;
    const uint32_t taddr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    __nv_bfloat16* orow = O + (static_cast<size_t>(bh) * N + row) * D;
#pragma unroll 1
    for (int c = 0; c < D / 32; ++c) {
      uint32_t r[32];
      tmem_ld32(taddr + c * 32, r);
      tmem_ld_wait();
      reg_fence(r);
      if (row < N) {
        uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
        for (int v = 0; v < 4; ++v)
          dst[v] = make_uint4(pack_bf16(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1])),
                              pack_bf16(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3])),
                              pack_bf16(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5])),
                              pack_bf16(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7])));
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
