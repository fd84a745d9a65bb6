// sm_100a backward (bf16 in, fp32 accumulate, head_dim 64 or 128): gradients of
// blockwise exact attention, recomputing probabilities from the saved
// log-sum-exp (the recompute policy "nothing_saveable" of page
// "RingAttention核心功能全解析", 核心API调用).
//
// Work unit = one (batch, head, 128-key tile).  The key/value tile stays
// resident while 128-row query tiles stream past in ring order: in the ring,
// a key/value block of ring block src meets query block (src + t) mod P at
// step t (page "Ring Attention技术解析" §2.2), so dK and dV accumulate as the
// block travels.  Per query tile i (all products on the tensor cores, fp32
// accumulators in TMEM, M = N = 128 everywhere):
//   S^T  = K Q_i^T              (SS, K-major)                 -> TMEM [128 x 128]
//   dP^T = V dO_i^T             (SS, K-major)                 -> TMEM [128 x 128]
//   P^T  = exp2(S^T log2e/sqrt(D) - lse_i log2e) (masked), dS^T = P^T (dP^T - Delta_i)
//   dV  += P^T dO_i             (TS: P^T bf16 in TMEM, dO MN-major)
//   dK  += dS^T Q_i             (TS: dS^T bf16 in TMEM, Q MN-major)
//   dQ^T = K^T dS^T             (SS: K and dS^T both MN-major) -> TMEM [128 x 128]
// dQ^T is read back by a dedicated warpgroup and added straight from
// registers into the fp32 dQ workspace with coalesced global reductions (dQ
// gathers contributions from every key tile); shared memory, whose
// bandwidth the tensor cores' operand reads mostly use, is not involved.
//
// Why 128 x 128: every product then has N = 128, where a shared-memory
// operand read (A 4 KB + B 4 KB per K-step) keeps pace with the tensor core
// (64 cycles each); with 64-query tiles the three SS products ran at N = 64
// and were bound by shared-memory bandwidth, and the stationary K and V were
// re-read twice as often per query.
//
// Roles (512 threads): warp 0 TMA producer, warp 1 TMEM owner + MMA issuer,
// warps 4-7 and 12-15 "softmax" (thread = key row; warpgroup w takes query
// columns [64w, 64w + 64) of each tile, in two chunks of 32: P^T, dS^T, then
// dK (w = 0) or dV (w = 1) in the epilogue), warps 8-11 dQ readout (thread =
// head-dim lane d of dQ^T).  setmaxnreg moves registers from warpgroup 0 and
// the readout group to the two softmax groups.
//
// TMEM (512 columns), a single slot:
//   [0, 128)    S^T; query chunk c (queries 32c .. 32c+31) is overwritten by
//               its own P^T (bf16 pairs) in [32c, 32c+16) and dS^T in
//               [32c+16, 32c+32): each softmax thread writes only the
//               columns of its own row it has already read;
//   [128, 256)  dP^T, then dQ^T once the softmax has read dP^T;
//   [256, 256+D) dK, [256+D, 256+2D) dV, accumulated over all query tiles.
// MMA issue order (tile n):  dV(n)  dK(n)  S^T(n+1)  dQ^T(n)  | dP^T(n+1).
// The tensor pipe runs one thread's MMAs in issue order: S^T(n+1) overwrites
// P^T / dS^T(n) only after dV / dK(n) read them; dP^T(n+1) waits for the
// readout of dQ^T(n).  The softmax exponentials of tile n+1 (P^T, signalled
// separately) overlap dQ^T(n), the readout and dP^T(n+1); its dS^T work
// overlaps dV(n+1).  dS^T also goes to shared memory (one buffer: softmax
// n+1 writes it only after dP^T(n+1), which follows dQ^T(n)) as the B
// operand of dQ^T.  At D = 64, dQ^T keeps M = 128 by reading a zero block as
// the upper half of K^T, so only its first 64 rows are read out.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "ra_common.cuh"
#include "ra_simt.cuh"

namespace ra {

template <int D_>
struct BwdLayout {
  static constexpr int D = D_;                    // 64 or 128
  static constexpr int KCH = D / 64;              // 128-byte swizzle chunks along D
  static constexpr int QT = kQTileBwd;            // 128 query rows per tile
  static constexpr int KV_BYTES = kTile * D * 2;  // 32 KB at D = 128
  static constexpr int CHUNK = kTile * 128;       // 16 KB box: 128 rows x 128 B
  static constexpr int Q_BYTES = QT * D * 2;      // 32 KB at D = 128
  static constexpr int DS_HALF = kTile * 64 * 2;  // 16 KB: 128 keys x 64 queries bf16
  static constexpr int DS_BYTES = 2 * DS_HALF;    // 128 keys x 128 queries
  static constexpr int NS = 2;                    // query-side stages (the next tile loads while one computes)
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KV_BYTES;
  static constexpr int OFF_Q = OFF_V + KV_BYTES;
  static constexpr int OFF_DO = OFF_Q + NS * Q_BYTES;
  static constexpr int OFF_DS = OFF_DO + NS * Q_BYTES;
  // dQ^T = K^T dS^T is an M = 128 product along D.  At D = 64 its second
  // 64-row half of A reads this zero block, so rows 64..127 of dQ^T are 0.
  static constexpr int OFF_ZERO = OFF_DS + DS_BYTES;
  static constexpr int ZERO_BYTES = D == 64 ? CHUNK : 0;
  static constexpr uint32_t LBO_DQ = D == 128 ? CHUNK : OFF_ZERO - OFF_K;   // distance between the D halves
  static constexpr int OFF_BAR = OFF_ZERO + ZERO_BYTES;
  static constexpr int B_KV = 0;
  static constexpr int B_QF = 1;                  // [NS] query stage loaded
  static constexpr int B_QE = B_QF + NS;          // [NS] query stage free
  static constexpr int B_SFULL = B_QE + NS;       // S^T computed
  static constexpr int B_DPFULL = B_SFULL + 1;    // dP^T computed
  static constexpr int B_PREADY = B_DPFULL + 1;   // P^T written (8 arrivals: softmax warps)
  static constexpr int B_DSREADY = B_PREADY + 1;  // dS^T written to TMEM and shared memory (8 arrivals)
  static constexpr int B_DQFULL = B_DSREADY + 1;  // dQ^T computed
  static constexpr int B_SLOTFREE = B_DQFULL + 1; // dQ^T read out (4 arrivals: readout warps)
  static constexpr int B_FINAL = B_SLOTFREE + 1;
  static constexpr int NBAR = B_FINAL + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int SMEM_ALLOC = BYTES + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S = 0, COL_DP = 128;
  static constexpr uint32_t COL_DK = 256, COL_DV = 256 + D;
  static constexpr int THREADS = 512;
  // Register split (setmaxnreg), per thread: warpgroup 0 (producer, issuer),
  // the two softmax warpgroups and the readout warpgroup.  The host checks
  // 128 * (REGS_WG0 + 2 * REGS_SOFTMAX + REGS_READOUT) <= 512 * (registers
  // per thread at launch) before launching, so every increase can be met.
  static constexpr int REGS_WG0 = 96, REGS_SOFTMAX = 160, REGS_READOUT = 96;
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
  static_assert(OFF_ZERO % 1024 == 0 && LBO_DQ % 16 == 0 && (LBO_DQ >> 4) < (1u << 14), "dQ^T operand layout");
  static_assert(D == 64 || D == 128, "head dim");
};

struct BwdParams {
  RingDesc rd;
  int32_t B, H;
  float scale_log2;          // log2(e) / sqrt(D)
  float scale;               // 1 / sqrt(D)
  const float* lse2;         // [B*H][s_pad]: -lse * log2(e), -inf for rows with no visible key
  const float* delta;        // [B*H][s_pad]: -<dO_i, O_i>
  int64_t s_pad;
  float* dqacc;              // [B*H][S][D] fp32, pre-zeroed
  void* dk;
  int64_t dk_sb, dk_ss, dk_sh;
  void* dv;
  int64_t dv_sb, dv_ss, dv_sh;
  int32_t grad_bf16;         // dK / dV element type: 1 bf16, 0 fp32
  const int32_t* seg;
  int64_t seg_sb, seg_ss;
  const float* bias;
  int64_t bias_sb, bias_ss;
  const int4* meta;
  int32_t* dbg_count;        // RA_DEBUG_COUNT builds: visible queries per key, [B, H, S], pre-zeroed
};

// fp32 add into global memory without a return value (a reduction at L2).
__device__ __forceinline__ void red_add_f32(float* addr, float v) {
  asm volatile("red.relaxed.gpu.global.add.f32 [%0], %1;" ::"l"(addr), "f"(v) : "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

template <int D>
__global__ void __launch_bounds__(512, 1)
    ra_bwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                        const __grid_constant__ BwdParams p) {
  using L = BwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Head-major order: the resident CTAs work on the key tiles of one or two
  // heads at a time, so that head's Q / dO stream stays in L2; within a head
  // the first key tiles (most query tiles under causal masking) go first.
  const int bh = blockIdx.x / p.rd.ntiles;
  const int kt = blockIdx.x % p.rd.ntiles;
  const int b = bh / p.H, h = bh % p.H;
  const int64_t k0 = (int64_t)kt * kTile;
  const int64_t S = p.rd.S;

  auto bar = [&](int i) -> uint32_t { return sbase + L::OFF_BAR + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::OFF_MISC + 4);

  if (threadIdx.x == 0) {
    mbar_init(bar(L::B_KV), 1);
    for (int i = 0; i < L::NS; ++i) { mbar_init(bar(L::B_QF + i), 1); mbar_init(bar(L::B_QE + i), 1); }
    mbar_init(bar(L::B_SFULL), 1);
    mbar_init(bar(L::B_DPFULL), 1);
    mbar_init(bar(L::B_PREADY), 8);      // one arrive per softmax warp
    mbar_init(bar(L::B_DSREADY), 8);
    mbar_init(bar(L::B_DQFULL), 1);
    mbar_init(bar(L::B_SLOTFREE), 4);    // one arrive per readout warp
    mbar_init(bar(L::B_FINAL), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), L::TMEM_COLS);
    tmem_relinquish();
  }
  if constexpr (L::ZERO_BYTES > 0) {
    for (int i = threadIdx.x; i < L::ZERO_BYTES / 16; i += L::THREADS)
      reinterpret_cast<uint4*>(gbase + L::OFF_ZERO)[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();   // the tensor cores read it through the async proxy
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const bool use_seg = p.seg != nullptr, use_bias = p.bias != nullptr;
  const int4* meta_b = p.meta ? p.meta + (int64_t)b * p.rd.ntiles : nullptr;
  const int4 km = meta_b ? load_meta(meta_b + kt) : make_int4(0, 0, 3, 0);
  // A key tile whose every bias is -inf is invisible to all queries.
  const bool dead = use_bias && !(km.z & kMetaAnyFinite);

  if (warp < 4) {
  regs_dec<L::REGS_WG0>();
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // The whole warp runs the loop (its lanes scan 32 query tiles per
    // metadata round trip, q_iter_next_warp); one elected lane issues copies.
    if (elect_one()) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      prefetch_tmap(&tm_do);
      mbar_arrive_expect_tx(bar(L::B_KV), 2 * L::KV_BYTES);
      for (int c = 0; c < L::KCH; ++c) {
        tma_load_4d(sbase + L::OFF_K + c * L::CHUNK, &tm_k, bar(L::B_KV), c * 64, h, (int)k0, b);
        tma_load_4d(sbase + L::OFF_V + c * L::CHUNK, &tm_v, bar(L::B_KV), c * 64, h, (int)k0, b);
      }
    }
    __syncwarp();
    int n = 0;
    if (!dead) {
      QIter it;
      q_iter_init(it, p.rd, k0, meta_b, use_seg);
      for (int32_t q = q_iter_next_warp(it, p.rd); q >= 0; q = q_iter_next_warp(it, p.rd), ++n) {
        const int st = n % L::NS;
        if (n >= L::NS && !ra_wait_warp(bar(L::B_QE + st), ((n / L::NS) & 1) ^ 1, abort_flag)) break;
        const int q0 = q * L::QT;
        if (elect_one()) {
          mbar_arrive_expect_tx(bar(L::B_QF + st), 2 * L::Q_BYTES);
          for (int c = 0; c < L::KCH; ++c) {
            tma_load_4d(sbase + L::OFF_Q + st * L::Q_BYTES + c * L::CHUNK, &tm_q, bar(L::B_QF + st), c * 64, h, q0, b);
            tma_load_4d(sbase + L::OFF_DO + st * L::Q_BYTES + c * L::CHUNK, &tm_do, bar(L::B_QF + st), c * 64, h, q0,
                        b);
          }
        }
        __syncwarp();
      }
    }
    ra_wait_drain(bar(L::B_KV), 0);
    for (int i = n - L::NS; i < n; ++i)
      if (i >= 0) ra_wait_drain(bar(L::B_QF + i % L::NS), (i / L::NS) & 1);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the issuer; one elected lane issues (ptx.cuh).
    constexpr uint32_t IDESC_SD = idesc_bf16_f32(128, L::QT, false, false);
    constexpr uint32_t IDESC_KV = idesc_bf16_f32(128, D, false, true);
    constexpr uint32_t IDESC_DQ = idesc_bf16_f32(128, L::QT, true, true);
    const uint32_t ka = sbase + L::OFF_K, va = sbase + L::OFF_V;
    // Descriptors are built once per operand tile; the K-step offsets are
    // added to the start-address field (address >> 4, no carry: shared
    // memory ends below 2^18 bytes), keeping the issue loop short.
    const uint64_t ka_k = smem_desc_sw128(ka, 16, 1024), va_k = smem_desc_sw128(va, 16, 1024);
    const uint64_t ka_mn = smem_desc_sw128(ka, L::LBO_DQ, 1024);
    const uint64_t ds_mn = smem_desc_sw128(sbase + L::OFF_DS, L::DS_HALF, 1024);
    auto issue_sd = [&](uint32_t d_tmem, uint64_t a_desc, uint32_t b_base) {   // S^T or dP^T
      const uint64_t b_desc = smem_desc_sw128(b_base, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t o = ((kk / 4) * L::CHUNK + (kk % 4) * 32) >> 4;
        mma_ss_w(d_tmem, a_desc + o, b_desc + o, IDESC_SD, kk > 0);
      }
    };
    // dV += P^T dO or dK += dS^T Q over the tile's 128 queries: K-step kk
    // covers queries 16kk .. 16kk+15, held (bf16 pairs) in columns
    // 32 (kk/2) + 8 (kk%2) + a_off of the S^T region (a_off 0: P^T, 16: dS^T).
    auto issue_kv = [&](uint32_t d_tmem, uint32_t a_off, uint32_t b_base, bool acc) {
      const uint64_t b_desc = smem_desc_sw128(b_base, L::CHUNK, 1024);
#pragma unroll
      for (int kk = 0; kk < L::QT / 16; ++kk)
        mma_ts_w(d_tmem, tmem + L::COL_S + 32 * (kk / 2) + 8 * (kk % 2) + a_off, b_desc + kk * (2048 >> 4), IDESC_KV,
                 (acc || kk > 0) ? 1u : 0u);
    };
    auto issue_dq = [&]() {   // dQ^T = K^T dS^T over the 128 keys
#pragma unroll
      for (int kk = 0; kk < kTile / 16; ++kk)
        mma_ss_w(tmem + L::COL_DP, ka_mn + kk * (2048 >> 4), ds_mn + kk * (2048 >> 4), IDESC_DQ, kk > 0);
    };
    // number of query tiles this key tile visits
    int N = 0;
    if (!dead) {
      QIter it;
      q_iter_init(it, p.rd, k0, meta_b, use_seg);
      while (q_iter_next_warp(it, p.rd) >= 0) ++N;
    }
    bool ok = ra_wait_warp(bar(L::B_KV), 0, abort_flag);
    if (ok && N > 0) {
      ok = ra_wait_warp(bar(L::B_QF + 0), 0, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_sd(tmem + L::COL_S, ka_k, sbase + L::OFF_Q);
        mma_commit_w(bar(L::B_SFULL));
        issue_sd(tmem + L::COL_DP, va_k, sbase + L::OFF_DO);
        mma_commit_w(bar(L::B_DPFULL));
      }
    }
    for (int n = 0; ok && n < N; ++n) {
      const int st = n % L::NS;
      const uint32_t ph = n & 1;
      if (!(ok = ra_wait_warp(bar(L::B_PREADY), ph, abort_flag))) break;
      tc_fence_after();
      issue_kv(tmem + L::COL_DV, 0, sbase + L::OFF_DO + st * L::Q_BYTES, n > 0);
      if (!(ok = ra_wait_warp(bar(L::B_DSREADY), ph, abort_flag))) break;
      tc_fence_after();
      issue_kv(tmem + L::COL_DK, 16, sbase + L::OFF_Q + st * L::Q_BYTES, n > 0);
      mma_commit_w(bar(L::B_QE + st));
      const bool more = n + 1 < N;
      if (more) {
        const int st1 = (n + 1) % L::NS;
        if (!(ok = ra_wait_warp(bar(L::B_QF + st1), ((n + 1) / L::NS) & 1, abort_flag))) break;
        issue_sd(tmem + L::COL_S, ka_k, sbase + L::OFF_Q + st1 * L::Q_BYTES);
        mma_commit_w(bar(L::B_SFULL));
      }
      issue_dq();
      mma_commit_w(bar(L::B_DQFULL));
      if (more) {
        if (!(ok = ra_wait_warp(bar(L::B_SLOTFREE), ph, abort_flag))) break;
        tc_fence_after();
        issue_sd(tmem + L::COL_DP, va_k, sbase + L::OFF_DO + ((n + 1) % L::NS) * L::Q_BYTES);
        mma_commit_w(bar(L::B_DPFULL));
      }
    }
    mma_commit_w(bar(L::B_FINAL));
    ra_wait_drain(bar(L::B_FINAL), 0);
    __syncwarp();
  }
  } else if ((warp >= 4 && warp < 8) || warp >= 12) {
    // ------------------------------------------------------------ softmax groups: one key row per thread
    regs_inc<L::REGS_SOFTMAX>();
    const int wg = warp >= 12;                       // query columns [64 wg, 64 wg + 64) of each tile
    const int sub = warp & 3;
    const int row = sub * 32 + lane;
    const int64_t j = k0 + row;                      // this thread's key
    const bool row_valid = j < S;
    const int64_t jc = row_valid ? j : S - 1;
    const uint32_t trow = tmem + ((uint32_t)(sub * 32) << 16);
    const int my_seg = use_seg ? p.seg[b * p.seg_sb + jc * p.seg_ss] : 0;
    float brow = 0.f;                                // bias of this key, log2 units
    if (use_bias) brow = p.bias[b * p.bias_sb + jc * p.bias_ss] * kLog2e;
    const int32_t cbs = p.rd.cbs;
    const int64_t i_first = cbs > 0 ? (j / cbs) * (int64_t)cbs : 0;   // first query that can see key j
    // A query tile starting at q0 needs the causal mask iff q0 is before the
    // causal block of the tile's last key (no per-tile division).
    const int64_t k_last_blk = cbs > 0 ? ((k0 + kTile - 1) / cbs) * (int64_t)cbs : 0;
    const float sc = p.scale_log2;
    const float* lse2_bh = p.lse2 + (int64_t)bh * p.s_pad;
    const float* delta_bh = p.delta + (int64_t)bh * p.s_pad;
#ifdef RA_DEBUG_COUNT
    int dbg_vis = 0;
#endif
    int n = 0;
    bool ok = true;
    if (!dead) {
      QIter it;
      q_iter_init(it, p.rd, k0, meta_b, use_seg);
      for (int32_t q = q_iter_next_warp(it, p.rd); q >= 0; q = q_iter_next_warp(it, p.rd), ++n) {
        const uint32_t ph = n & 1;
        const int64_t q0 = (int64_t)q * L::QT;
        // the query tile's metadata load is issued before the wait, so it lands meanwhile
        const int4 qm = meta_b ? load_meta(meta_b + q) : make_int4(0, 0, 3, 0);
        const bool need_causal = cbs > 0 && q0 < k_last_blk;
        const bool need_ragged = (q0 + L::QT > S) || (k0 + kTile > S);
        const bool need_seg = use_seg && !(qm.x == qm.y && km.x == km.y && qm.x == km.x);
        const bool need_mask = need_causal || need_ragged || need_seg || !row_valid;
        if (!(ok = ra_wait_warp(bar(L::B_SFULL), ph, abort_flag))) break;
        tc_fence_after();
        // ---- P^T for the group's two chunks of 32 queries
        float pr[2][32];
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int c = 2 * wg + jj;                 // chunk: queries 32c .. 32c+31 of the tile
          uint32_t sr[32];
          tmem_ld32(trow + L::COL_S + 32 * c, sr);
          tmem_ld_wait();
          float* x = pr[jj];
          const float4* nl4 = reinterpret_cast<const float4*>(lse2_bh + q0 + 32 * c);   // -lse*log2e, broadcast
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            float4 nl = __ldg(nl4 + e / 4);
            if (use_bias) {
              nl.x += brow; nl.y += brow; nl.z += brow; nl.w += brow;
            }
            reg_fence(sr[e]); reg_fence(sr[e + 1]); reg_fence(sr[e + 2]); reg_fence(sr[e + 3]);
            ffma2(x[e], x[e + 1], __uint_as_float(sr[e]), __uint_as_float(sr[e + 1]), sc, sc, nl.x, nl.y);
            ffma2(x[e + 2], x[e + 3], __uint_as_float(sr[e + 2]), __uint_as_float(sr[e + 3]), sc, sc, nl.z, nl.w);
          }
          if (need_mask) {
            const int64_t qc0 = q0 + 32 * c;
            const int64_t cmin64 = i_first - qc0;                  // visible iff e >= cmin
            const int cmin = cmin64 < 0 ? 0 : (cmin64 > 32 ? 32 : (int)cmin64);
            const int64_t cmax64 = S - qc0;                        // valid iff e < cmax
            const int cmax = row_valid ? (cmax64 > 32 ? 32 : (cmax64 < 0 ? 0 : (int)cmax64)) : 0;
            uint32_t vb = ~0u;
            if (need_seg) {
              const int32_t* sp = p.seg + b * p.seg_sb;
              vb = 0;
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                const int64_t i = qc0 + e < S ? qc0 + e : S - 1;
                vb |= (uint32_t)(__ldg(sp + i * p.seg_ss) == my_seg) << e;
              }
            }
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const bool vis = e >= cmin && e < cmax && ((vb >> e) & 1u);
              x[e] = vis ? x[e] : -INFINITY;
            }
          }
#ifdef RA_DEBUG_COUNT
          // visible pairs as decided by this kernel's own tile skipping and masking
#pragma unroll
          for (int e = 0; e < 32; ++e) dbg_vis += x[e] != -INFINITY;
#endif
          uint32_t pp[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            x[e] = ex2_approx(x[e]);
            x[e + 1] = ex2_approx(x[e + 1]);
            pp[e >> 1] = pack_bf16x2(x[e], x[e + 1]);
          }
          tmem_st16(trow + L::COL_S + 32 * c, pp);    // over this row's own, already read, S^T columns
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::B_PREADY));
        // ---- dS^T = P^T (dP^T - Delta) for the same chunks
        if (!(ok = ra_wait_warp(bar(L::B_DPFULL), ph, abort_flag))) break;
        tc_fence_after();
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int c = 2 * wg + jj;
          uint32_t dr[32];
          tmem_ld32(trow + L::COL_DP + 32 * c, dr);
          tmem_ld_wait();
          const float4* nd4 = reinterpret_cast<const float4*>(delta_bh + q0 + 32 * c);   // -Delta, broadcast
          uint32_t dd[16];
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const float4 nd = __ldg(nd4 + e / 4);
            reg_fence(dr[e]); reg_fence(dr[e + 1]); reg_fence(dr[e + 2]); reg_fence(dr[e + 3]);
            float t0, t1, t2, t3, s0, s1, s2, s3;
            fadd2(t0, t1, __uint_as_float(dr[e]), __uint_as_float(dr[e + 1]), nd.x, nd.y);
            fadd2(t2, t3, __uint_as_float(dr[e + 2]), __uint_as_float(dr[e + 3]), nd.z, nd.w);
            fmul2(s0, s1, pr[jj][e], pr[jj][e + 1], t0, t1);
            fmul2(s2, s3, pr[jj][e + 2], pr[jj][e + 3], t2, t3);
            dd[e >> 1] = pack_bf16x2(s0, s1);
            dd[(e >> 1) + 1] = pack_bf16x2(s2, s3);
          }
          tmem_st16(trow + L::COL_S + 32 * c + 16, dd);
          // dS^T into shared memory for dQ^T = K^T dS^T (MN-major, 128-byte
          // swizzle): queries 64h .. 64h+63 form half h; key row `row` is one
          // 128-byte line of it, and 16-byte chunk u lands at u ^ (row % 8).
          const uint32_t line = sbase + L::OFF_DS + (c / 2) * L::DS_HALF + row * 128;
#pragma unroll
          for (int u4 = 0; u4 < 4; ++u4) {
            const int u = (c % 2) * 4 + u4;
            st_shared_v4(line + ((u ^ (row & 7)) << 4), dd[4 * u4], dd[4 * u4 + 1], dd[4 * u4 + 2], dd[4 * u4 + 3]);
          }
        }
        fence_proxy_async_smem();
        tmem_st_wait();
        tc_fence_before();
        // one arrive per warp: per-lane arrives on one barrier serialise in the
        // shared-memory pipe, which the tensor cores' operand reads also use
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::B_DSREADY));
      }
    }
#ifdef RA_DEBUG_COUNT
    // the two query halves of a key row add their counts
    if (row_valid && ok && p.dbg_count) atomicAdd(p.dbg_count + ((int64_t)b * p.H + h) * S + j, dbg_vis);
#endif
    // ---------------------------------------------------------- epilogue: dK (group 0) or dV (group 1)
    bool have = n > 0 && ok;
    if (have) have = ra_wait(bar(L::B_FINAL), 0, abort_flag);
    have = __all_sync(0xffffffffu, have);
    n = __shfl_sync(0xffffffffu, n, 0);
    tc_fence_after();
    {
      const uint32_t col = wg == 0 ? L::COL_DK : L::COL_DV;
      const float mul = wg == 0 ? p.scale : 1.f;
      char* base = static_cast<char*>(wg == 0 ? p.dk : p.dv);
      const int64_t sb = wg == 0 ? p.dk_sb : p.dv_sb, ss = wg == 0 ? p.dk_ss : p.dv_ss,
                    sh = wg == 0 ? p.dk_sh : p.dv_sh;
      const int64_t off = b * sb + jc * ss + h * sh;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t r[32];
        if (have) {
          tmem_ld32(trow + col + c, r);
          tmem_ld_wait();
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          if (have) reg_fence(r[e]);
          else r[e] = 0u;
        }
        if (row_valid && (have || n == 0)) {
          if (p.grad_bf16) {
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(base) + off + c);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e)
                w[e] = pack_bf16x2(__uint_as_float(r[8 * v4 + 2 * e]) * mul, __uint_as_float(r[8 * v4 + 2 * e + 1]) * mul);
              dst[v4] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          } else {
            float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(base) + off + c);
#pragma unroll
            for (int v4 = 0; v4 < 8; ++v4)
              dst[v4] = make_float4(__uint_as_float(r[4 * v4]) * mul, __uint_as_float(r[4 * v4 + 1]) * mul,
                                    __uint_as_float(r[4 * v4 + 2]) * mul, __uint_as_float(r[4 * v4 + 3]) * mul);
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ dQ readout: thread = head-dim lane d
    // Each thread takes its row d of dQ^T (128 queries, in two halves) out of
    // TMEM and adds the values straight into the fp32 accumulator
    // dqacc[bh][q][d]: a warp's 32 lanes cover 32 consecutive d of one query
    // row, so every reduction is one coalesced 128-byte request.  The slot
    // is released as soon as the second half is in registers.
    regs_dec<L::REGS_READOUT>();
    const int sub = warp & 3;
    const int d = sub * 32 + lane;
    const uint32_t trow = tmem + ((uint32_t)(sub * 32) << 16);
    if (!dead) {
      QIter it;
      q_iter_init(it, p.rd, k0, meta_b, use_seg);
      int n = 0;
      for (int32_t q = q_iter_next_warp(it, p.rd); q >= 0; q = q_iter_next_warp(it, p.rd), ++n) {
        if (!ra_wait_warp(bar(L::B_DQFULL), n & 1, abort_flag)) break;
        tc_fence_after();
        const int64_t q0 = (int64_t)q * L::QT;
        const int64_t rows = S - q0 < L::QT ? S - q0 : L::QT;   // the last query tile may be ragged
        float* dst = p.dqacc + ((int64_t)bh * S + q0) * D + d;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t r[64];
          tmem_ld32(trow + L::COL_DP + 64 * half, r);
          tmem_ld32(trow + L::COL_DP + 64 * half + 32, r + 32);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 64; ++c) reg_fence(r[c]);
          if (half == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(L::B_SLOTFREE));
          }
          if (d < D) {   // at D = 64 the upper half of dQ^T is the zero padding
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (64 * half + c < rows) red_add_f32(dst + (int64_t)(64 * half + c) * D, __uint_as_float(r[c]) * p.scale);
          }
        }
      }
    }
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
