// sm_100a GEMMs of the blockwise feed-forward network (page
// "RingAttention核心功能全解析", 核心API调用: ``blockwise_feedforward`` is
// exported next to ``ringattention``; the model configuration the page shards
// is LLaMA's, whose feed-forward network is a SwiGLU without biases):
//
//   gated:  H = silu(X W1^T) * (X W3^T)      (one kernel, two accumulators)
//   plain:  Y = H W2^T
//
// over one chunk of tokens at a time (the caller, ra_feedforward, loops over
// the chunks, so only a chunk's H is ever held).  Every operand is K-major
// (rows of the reduction dimension contiguous: X [T, d_model], H [chunk,
// d_ff], weights output-major [out, in]), read by TMA in 64-element (128-byte)
// k-blocks with the 128-byte swizzle, multiplied by tcgen05.mma (bf16 in,
// fp32 accumulate in TMEM).
//
// Persistent kernel, one CTA per SM, warp-specialized (192 threads):
//   warp 0      TMA producer: per output tile and k-block, A [128 x 64] and
//               B [256 x 64] (plain) or B1, B3 [128 x 64] each (gated) into
//               one of STAGES shared-memory stages.
//   warp 1      TMEM owner and MMA issuer (converged warp, elected lane):
//               per k-block 4 K-steps of M = 128, N = 256 (plain) or two
//               N = 128 products sharing A (gated), into one of two
//               256-column accumulator buffers.
//   warps 2-5   epilogue: thread = output row; TMEM -> registers (32 columns
//               at a time) -> silu gate (gated) -> bf16 -> global.  Two
//               accumulator buffers let the epilogue of tile i run while the
//               MMAs of tile i+1 do.
// Tiles are visited n-block-major within a band of m-blocks so the CTAs
// running at once share their A rows and B columns in L2.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "ra_common.cuh"

namespace ra {

struct FfnLayout {
  static constexpr int BM = 128, BK = 64;
  static constexpr int BN = 256;                        // accumulator columns per tile (plain: N; gated: 2 x 128)
  static constexpr int STAGES = 4;
  static constexpr int A_BYTES = BM * BK * 2;           // 16 KB
  static constexpr int B_BYTES = BN * BK * 2;           // 32 KB (gated: B1 rows 0-127, B3 rows 128-255)
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int OFF_BAR = STAGES * STAGE_BYTES;
  static constexpr int B_FULL = 0;                      // [STAGES]
  static constexpr int B_EMPTY = B_FULL + STAGES;       // [STAGES]
  static constexpr int B_ACCFULL = B_EMPTY + STAGES;    // [2]
  static constexpr int B_ACCEMPTY = B_ACCFULL + 2;      // [2] 4 arrivals: epilogue warps
  static constexpr int B_DRAIN = B_ACCEMPTY + 2;
  static constexpr int NBAR = B_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_ALLOC = OFF_MISC + 16 + 1024;
  static constexpr uint32_t TMEM_COLS = 512;            // two 256-column accumulator buffers
  static constexpr int THREADS = 192;
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

struct FfnParams {
  int32_t M;                 // rows of this chunk
  int32_t a_row0;            // first row of the chunk in A's tensor map
  int64_t c_row0;            // first row of the chunk in C
  int32_t N, K;              // output columns (multiple of 32); reduction length (multiple of 8)
  int32_t n_tiles, m_tiles;  // N / (gated ? 128 : 256), ceil(M / 128)
  __nv_bfloat16* c;          // output [rows, N] row-major (row stride ldc elements)
  int64_t ldc;
};

__device__ __forceinline__ float silu_f(float a) { return a / (1.f + __expf(-a)); }

template <bool GATED>
__global__ void __launch_bounds__(192, 1)
    ra_ffn_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                       const __grid_constant__ CUtensorMap tm_b3, const __grid_constant__ FfnParams p) {
  using L = FfnLayout;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto bar = [&](int i) -> uint32_t { return sbase + L::OFF_BAR + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::OFF_MISC + 4);

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::STAGES; ++i) { mbar_init(bar(L::B_FULL + i), 1); mbar_init(bar(L::B_EMPTY + i), 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(bar(L::B_ACCFULL + i), 1); mbar_init(bar(L::B_ACCEMPTY + i), 4); }
    mbar_init(bar(L::B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int n_tiles = p.n_tiles, total = p.m_tiles * p.n_tiles;
  const int kblocks = (p.K + L::BK - 1) / L::BK;   // a ragged last k-block reads TMA's zero fill
  constexpr int BAND = 8;                     // m-blocks per band of the tile order
  // tile index -> (m block, n block): bands of BAND m-blocks, n-block-major inside a band
  auto tile_mn = [&](int t, int& mb, int& nb) {
    const int band = t / (BAND * n_tiles);
    const int in = t % (BAND * n_tiles);
    const int rows = min(BAND, p.m_tiles - band * BAND);
    nb = in / rows;
    mb = band * BAND + in % rows;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    const uint64_t pol_a = l2_policy_evict_first(), pol_b = l2_policy_evict_last();
    int it = 0;   // k-blocks issued
    bool ok = true;
    for (int t = blockIdx.x; ok && t < total; t += gridDim.x) {
      int mb, nb;
      tile_mn(t, mb, nb);
      for (int kb = 0; kb < kblocks; ++kb, ++it) {
        const int st = it % L::STAGES;
        if (it >= L::STAGES && !(ok = ra_wait_warp(bar(L::B_EMPTY + st), ((it / L::STAGES) & 1) ^ 1, abort_flag)))
          break;
        if (elect_one()) {
          const uint32_t sa = sbase + st * L::STAGE_BYTES, sb = sa + L::A_BYTES;
          mbar_arrive_expect_tx(bar(L::B_FULL + st), L::STAGE_BYTES);
          tma_load_2d_hint(sa, &tm_a, bar(L::B_FULL + st), kb * L::BK, p.a_row0 + mb * L::BM, pol_a);
          if constexpr (GATED) {
            tma_load_2d_hint(sb, &tm_b, bar(L::B_FULL + st), kb * L::BK, nb * 128, pol_b);
            tma_load_2d_hint(sb + L::B_BYTES / 2, &tm_b3, bar(L::B_FULL + st), kb * L::BK, nb * 128, pol_b);
          } else {
            tma_load_2d_hint(sb, &tm_b, bar(L::B_FULL + st), kb * L::BK, nb * L::BN, pol_b);
          }
        }
        __syncwarp();
      }
    }
    for (int i = it - L::STAGES; i < it; ++i)
      if (i >= 0) ra_wait_drain(bar(L::B_FULL + i % L::STAGES), (i / L::STAGES) & 1);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t IDESC = GATED ? idesc_bf16_f32(128, 128, false, false) : idesc_bf16_f32(128, 256, false, false);
    int it = 0, local = 0;   // k-blocks consumed, tiles done by this CTA
    bool ok = true;
    for (int t = blockIdx.x; ok && t < total; t += gridDim.x, ++local) {
      const int buf = local & 1;
      const uint32_t acc = tmem + buf * 256;
      // the epilogue must have emptied this accumulator buffer (two tiles ago)
      if (local >= 2 && !(ok = ra_wait_warp(bar(L::B_ACCEMPTY + buf), ((local >> 1) - 1) & 1, abort_flag))) break;
      tc_fence_after();
      for (int kb = 0; kb < kblocks; ++kb, ++it) {
        const int st = it % L::STAGES;
        if (!(ok = ra_wait_warp(bar(L::B_FULL + st), (it / L::STAGES) & 1, abort_flag))) break;
        tc_fence_after();
        const uint32_t sa = sbase + st * L::STAGE_BYTES, sb = sa + L::A_BYTES;
        const uint64_t ad = smem_desc_sw128(sa, 16, 1024);
        const uint64_t bd = smem_desc_sw128(sb, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < L::BK / 16; ++kk) {
          const uint32_t o = (kk * 32) >> 4;     // 16 elements = 32 bytes along the swizzled row
          const uint32_t accum = (kb > 0 || kk > 0) ? 1u : 0u;
          if constexpr (GATED) {
            mma_ss_w(acc, ad + o, bd + o, IDESC, accum);
            mma_ss_w(acc + 128, ad + o, bd + ((L::B_BYTES / 2) >> 4) + o, IDESC, accum);
          } else {
            mma_ss_w(acc, ad + o, bd + o, IDESC, accum);
          }
        }
        mma_commit_w(bar(L::B_EMPTY + st));
      }
      if (!ok) break;
      mma_commit_w(bar(L::B_ACCFULL + buf));
    }
    mma_commit_w(bar(L::B_DRAIN));
    ra_wait_drain(bar(L::B_DRAIN), 0);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue: thread = output row
    const int quarter = warp & 3;                // TMEM lanes 32*quarter .. +31 (warps 2..5)
    const int r = quarter * 32 + lane;
    const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
    int local = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++local) {
      int mb, nb;
      tile_mn(t, mb, nb);
      const int buf = local & 1;
      if (!(ok = ra_wait_warp(bar(L::B_ACCFULL + buf), (local >> 1) & 1, abort_flag))) break;
      tc_fence_after();
      const int row = mb * L::BM + r;                 // row within the chunk
      const bool valid = row < p.M;
      __nv_bfloat16* dst = p.c + (p.c_row0 + (valid ? row : 0)) * p.ldc;
      constexpr int OUT_COLS = GATED ? 128 : 256;
      const int n0 = nb * OUT_COLS;
#pragma unroll 1
      for (int c = 0; c < OUT_COLS; c += 32) {
        uint32_t v[32];
        tmem_ld32(trow + buf * 256 + c, v);
        uint32_t g[32];
        if constexpr (GATED) tmem_ld32(trow + buf * 256 + 128 + c, g);
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          reg_fence(v[e]);
          reg_fence(v[e + 1]);
          float a0 = __uint_as_float(v[e]), a1 = __uint_as_float(v[e + 1]);
          if constexpr (GATED) {
            reg_fence(g[e]);
            reg_fence(g[e + 1]);
            a0 = silu_f(a0) * __uint_as_float(g[e]);
            a1 = silu_f(a1) * __uint_as_float(g[e + 1]);
          }
          pk[e >> 1] = pack_bf16x2(a0, a1);
        }
        if (valid && n0 + c < p.N && RA_IN_RANGE(n0 + c + 31, p.N, kSiteFfnOut)) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + n0 + c);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) d4[q4] = make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
        }
      }
      // this warp's TMEM reads of the buffer are complete: the MMAs may reuse it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::B_ACCEMPTY + buf));
    }
    (void)ok;
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

}  // namespace ra
