// sm_100a backward (bf16 in, fp32 accumulate, head_dim 64 or 128): gradients of
// blockwise exact attention, recomputing probabilities from the saved
// log-sum-exp (the recompute policy "nothing_saveable" of page
// "RingAttention核心功能全解析", 核心API调用).
//
// Work unit = one (batch, head, 128-key tile).  The key/value tile stays
// resident while 64-row query tiles stream past in ring order: in the ring,
// a key/value block of ring block src meets query block (src + t) mod P at
// step t (page "Ring Attention技术解析" §2.2), so dK and dV accumulate as the
// block travels.  Per query tile i (all products on the tensor cores, fp32
// accumulators in TMEM, M = 128 everywhere):
//   S^T  = K Q_i^T              (SS, K-major)            -> TMEM [128 x 64]
//   dP^T = V dO_i^T             (SS, K-major)            -> TMEM [128 x 64]
//   P^T  = exp2(S^T log2e/sqrt(D) - lse_i log2e) (masked), dS^T = P^T (dP^T - Delta_i)
//   dV  += P^T dO_i             (TS: P^T bf16 in TMEM, dO MN-major)
//   dK  += dS^T Q_i             (TS: dS^T bf16 in TMEM, Q MN-major)
//   dQ^T = K^T dS^T             (SS: K and dS^T both MN-major) -> TMEM [128 x 64]
// dQ^T is read back by a dedicated warpgroup, staged in shared memory as a
// [64 queries x D] fp32 tile and added into the fp32 dQ workspace with one
// TMA bulk reduce-add per tile (dQ gathers contributions from every key tile).
//
// Roles (512 threads): warp 0 TMA producer, warp 1 TMEM owner + MMA issuer,
// warps 4-7 and 12-15 "softmax" (thread = key row; the two warpgroups take
// query columns 0-31 and 32-63 of each tile: P^T, dS^T, then dK resp. dV in
// the epilogue), warps 8-11 dQ readout (thread = head-dim lane d of dQ^T).
// TMEM (512 columns): two 128-column slots, then dK [256,256+D), dV [256+D,256+2D).
// Query tile n uses slot n % 2: S^T -> [0,64), dP^T -> [64,128); softmax
// group h overwrites its own S^T columns [32h, 32h+32) with P^T ([32h,
// 32h+16)) and dS^T ([32h+16, 32h+32), bf16 pairs), so no group writes a
// column the other still has to read, and dQ^T(n) lands in [64,128) once
// dP^T has been read.  A slot is reused two tiles later, after the readout
// group has taken dQ^T out of it.
//
// Overlap: with two slots the "head" products of tile n+1 (S^T, dP^T) are
// computed while the softmax groups work on tile n; the issue order is given
// at the MMA issuer below.  At D = 64, dQ^T keeps M = 128 by reading a zero
// block as the upper half of K^T, so only its first 64 rows are read out.
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
  static constexpr int QT = kQTileBwd;            // 64 query rows per tile
  static constexpr int KV_BYTES = kTile * D * 2;  // 32 KB at D = 128
  static constexpr int KV_CHUNK = kTile * 128;    // 16 KB box: 128 rows x 128 B
  static constexpr int Q_BYTES = QT * D * 2;      // 16 KB at D = 128
  static constexpr int Q_CHUNK = QT * 128;        // 8 KB box: 64 rows x 128 B
  static constexpr int DS_BYTES = kTile * QT * 2; // 16 KB: 128 keys x 64 queries bf16
  static constexpr int NS = 3;                    // query-side stages (two tiles in flight + one loading)
  static constexpr int NSLOT = 2;                 // TMEM slots
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KV_BYTES;
  static constexpr int OFF_Q = OFF_V + KV_BYTES;
  static constexpr int OFF_DO = OFF_Q + NS * Q_BYTES;
  static constexpr int OFF_DS = OFF_DO + NS * Q_BYTES;
  // dQ^T = K^T dS^T is an M = 128 product along D.  At D = 64 its second
  // 64-row half of A reads this zero block, so rows 64..127 of dQ^T are 0.
  static constexpr int OFF_ZERO = OFF_DS + NSLOT * DS_BYTES;
  static constexpr int ZERO_BYTES = D == 64 ? KV_CHUNK : 0;
  static constexpr uint32_t LBO_DQ = D == 128 ? KV_CHUNK : OFF_ZERO - OFF_K;   // distance between the D halves
  static constexpr int OFF_LD = OFF_ZERO + ZERO_BYTES;       // per stage: lse2[64], delta[64]
  static constexpr int LD_BYTES = 2 * QT * 4;
  static constexpr int OFF_DQS = OFF_LD + NS * LD_BYTES;    // dQ staging [64][D] fp32
  static constexpr int DQS_BYTES = QT * D * 4;               // 32 KB at D = 128
  static constexpr int OFF_BAR = OFF_DQS + DQS_BYTES;
  static constexpr int B_KV = 0;
  static constexpr int B_QF = 1;                  // [NS] query stage loaded
  static constexpr int B_QE = B_QF + NS;          // [NS] query stage free
  static constexpr int B_SFULL = B_QE + NS;       // [NSLOT] S^T computed
  static constexpr int B_DPFULL = B_SFULL + NSLOT;   // [NSLOT] dP^T computed
  static constexpr int B_DSREADY = B_DPFULL + NSLOT; // [NSLOT] P^T, dS^T written (8 arrivals: softmax warps)
  static constexpr int B_DQFULL = B_DSREADY + NSLOT; // [NSLOT] dQ^T computed
  static constexpr int B_SLOTFREE = B_DQFULL + NSLOT;  // [NSLOT] dQ^T read out (4 arrivals: readout warps)
  static constexpr int B_FINAL = B_SLOTFREE + NSLOT;
  static constexpr int B_DQSFULL = B_FINAL + 1;      // staging written (4 arrivals)
  static constexpr int B_DQSFREE = B_DQSFULL + 1;    // staging read by the bulk reduce
  static constexpr int NBAR = B_DQSFREE + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int SMEM_ALLOC = BYTES + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t SLOT_COLS = 128;
  // Softmax group h (query columns [32h, 32h+32)) writes its P^T into S^T
  // columns [32h, 32h+16) and its dS^T into [32h+16, 32h+32): only columns of
  // its own rows and queries that it has already read.
  static constexpr uint32_t SLOT_ST = 0, SLOT_DPT = 64, SLOT_PT = 0, SLOT_DST = 16, SLOT_DQT = 64;
  static constexpr uint32_t COL_DK = 256, COL_DV = 256 + D;
  static constexpr int THREADS = 512;
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
  static_assert(OFF_DQS % 128 == 0, "bulk reduce source alignment");
  static_assert(OFF_LD % 16 == 0 && LD_BYTES % 16 == 0, "16-byte loads of the LSE / Delta rows");
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

// Tensor bulk reduce-add shared -> global (3-D tile, fp32 add), tracked by a bulk group.
__device__ __forceinline__ void tma_reduce_add_3d(const void* tmap, uint32_t src, int c0, int c1, int c2) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
          reinterpret_cast<uint64_t>(tmap)),
      "r"(c0), "r"(c1), "r"(c2), "r"(src)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_group_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_group0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void st_shared_f32(uint32_t addr, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

// 1-D bulk copy global -> shared (16-byte aligned, size multiple of 16).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// Four floats from shared memory in one access (a warp reading one address
// gets them as a broadcast: one wavefront for 16 bytes).
__device__ __forceinline__ float4 ld_shared_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

template <int D>
__global__ void __launch_bounds__(512, 1)
    ra_bwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                        const __grid_constant__ CUtensorMap tm_dq, const __grid_constant__ BwdParams p) {
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
  if (!(RA_IN_RANGE(b, p.B, kSiteBwdUnit) && RA_IN_RANGE(h, p.H, kSiteBwdUnit))) return;   // debug build only

  auto bar = [&](int i) -> uint32_t { return sbase + L::OFF_BAR + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::OFF_MISC + 4);

  if (threadIdx.x == 0) {
    mbar_init(bar(L::B_KV), 1);
    for (int i = 0; i < L::NS; ++i) { mbar_init(bar(L::B_QF + i), 1); mbar_init(bar(L::B_QE + i), 1); }
    for (int i = 0; i < L::NSLOT; ++i) {
      mbar_init(bar(L::B_SFULL + i), 1);
      mbar_init(bar(L::B_DPFULL + i), 1);
      mbar_init(bar(L::B_DSREADY + i), 8);     // one arrive per softmax warp
      mbar_init(bar(L::B_DQFULL + i), 1);
      mbar_init(bar(L::B_SLOTFREE + i), 4);    // one arrive per readout warp
    }
    mbar_init(bar(L::B_FINAL), 1);
    mbar_init(bar(L::B_DQSFULL), 4);
    mbar_init(bar(L::B_DQSFREE), 1);
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

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // The whole warp runs the loop (its lanes scan 32 query tiles per
    // metadata round trip, q_iter_next_warp); one elected lane issues copies.
    {
      if (elect_one()) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_do);
        mbar_arrive_expect_tx(bar(L::B_KV), 2 * L::KV_BYTES);
        for (int c = 0; c < L::KCH; ++c) {
          tma_load_4d(sbase + L::OFF_K + c * L::KV_CHUNK, &tm_k, bar(L::B_KV), c * 64, h, (int)k0, b);
          tma_load_4d(sbase + L::OFF_V + c * L::KV_CHUNK, &tm_v, bar(L::B_KV), c * 64, h, (int)k0, b);
        }
      }
      __syncwarp();
      int n = 0;
      if (!dead) {
        QIter it;
        q_iter_init(it, p.rd, k0, meta_b, use_seg);
        const float* lse_row = p.lse2 + (int64_t)bh * p.s_pad;
        const float* dl_row = p.delta + (int64_t)bh * p.s_pad;
        for (int32_t q = q_iter_next_warp(it, p.rd); q >= 0; q = q_iter_next_warp(it, p.rd), ++n) {
          const int st = n % L::NS;
          if (n >= L::NS && !ra_wait_warp(bar(L::B_QE + st), ((n / L::NS) & 1) ^ 1, abort_flag)) break;
          const int q0 = q * L::QT;
          if (elect_one()) {
            mbar_arrive_expect_tx(bar(L::B_QF + st), 2 * L::Q_BYTES + L::LD_BYTES);
            for (int c = 0; c < L::KCH; ++c) {
              tma_load_4d(sbase + L::OFF_Q + st * L::Q_BYTES + c * L::Q_CHUNK, &tm_q, bar(L::B_QF + st), c * 64, h,
                          q0, b);
              tma_load_4d(sbase + L::OFF_DO + st * L::Q_BYTES + c * L::Q_CHUNK, &tm_do, bar(L::B_QF + st), c * 64,
                          h, q0, b);
            }
            // (an out-of-range row in the debug build skips the copies; the
            // stage then never completes and its consumers' bounded waits give up)
            if (RA_IN_RANGE(q0 + L::QT - 1, p.s_pad, kSiteBwdLseDelta)) {
              bulk_load(sbase + L::OFF_LD + st * L::LD_BYTES, lse_row + q0, L::QT * 4, bar(L::B_QF + st));
              bulk_load(sbase + L::OFF_LD + st * L::LD_BYTES + L::QT * 4, dl_row + q0, L::QT * 4, bar(L::B_QF + st));
            }
          }
          __syncwarp();
        }
      }
      ra_wait_drain(bar(L::B_KV), 0);
      for (int i = n - L::NS; i < n; ++i)
        if (i >= 0) ra_wait_drain(bar(L::B_QF + i % L::NS), (i / L::NS) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    {   // the whole warp runs the issuer; one elected lane issues (ptx.cuh)
      constexpr uint32_t IDESC_SD = idesc_bf16_f32(128, L::QT, false, false);
      constexpr uint32_t IDESC_KV = idesc_bf16_f32(128, D, false, true);
      constexpr uint32_t IDESC_DQ = idesc_bf16_f32(128, L::QT, true, true);
      const uint32_t ka = sbase + L::OFF_K, va = sbase + L::OFF_V;
      // Descriptors are built once per operand tile; the K-step offsets are
      // added to the start-address field (address >> 4, no carry: shared
      // memory ends below 2^18 bytes), keeping the issue loop short.
      const uint64_t ka_k = smem_desc_sw128(ka, 16, 1024), va_k = smem_desc_sw128(va, 16, 1024);
      const uint64_t ka_mn = smem_desc_sw128(ka, L::LBO_DQ, 1024);
      auto issue_sd = [&](uint32_t d_tmem, uint64_t a_desc, uint32_t b_base) {   // S^T or dP^T
        const uint64_t b_desc = smem_desc_sw128(b_base, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t oa = ((kk / 4) * L::KV_CHUNK + (kk % 4) * 32) >> 4;
          const uint32_t ob = ((kk / 4) * L::Q_CHUNK + (kk % 4) * 32) >> 4;
          mma_ss_w(d_tmem, a_desc + oa, b_desc + ob, IDESC_SD, kk > 0);
        }
      };
      auto issue_kv = [&](uint32_t d_tmem, uint32_t a_tmem, uint32_t b_base, bool acc) {   // dV or dK
        const uint64_t b_desc = smem_desc_sw128(b_base, L::Q_CHUNK, 1024);
#pragma unroll
        for (int kk = 0; kk < L::QT / 16; ++kk)
          mma_ts_w(d_tmem, a_tmem + 32 * (kk / 2) + 8 * (kk % 2), b_desc + kk * (2048 >> 4), IDESC_KV,
                   (acc || kk > 0) ? 1u : 0u);
      };
      auto issue_dq = [&](uint32_t d_tmem, uint32_t ds_base) {
        const uint64_t b_desc = smem_desc_sw128(ds_base, L::DS_BYTES, 1024);
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          mma_ss_w(d_tmem, ka_mn + kk * (2048 >> 4), b_desc + kk * (2048 >> 4), IDESC_DQ, kk > 0);
      };
      // number of query tiles this key tile visits
      int N = 0;
      if (!dead) {
        QIter it;
        q_iter_init(it, p.rd, k0, meta_b, use_seg);
        while (q_iter_next_warp(it, p.rd) >= 0) ++N;
      }
      // Issue order (two TMEM slots, tile n in slot n % 2):
      //   S^T(0) dP^T(0) S^T(1) dP^T(1) | tail(0) S^T(2) dP^T(2) | tail(1) S^T(3) dP^T(3) | ...
      // with tail(n) = dQ^T(n), then dV(n), dK(n).  The tensor pipe runs one
      // thread's MMAs in issue order, so S^T(n+2) may follow tail(n) at once
      // (it overwrites P^T / dS^T(n) only after dV / dK(n) have read them);
      // dP^T(n+2) overwrites dQ^T(n) and waits for its readout, which runs
      // while dV, dK(n) and S^T(n+2) execute.  The softmax of tile n+1 has
      // tail(n), S^T(n+2) and dP^T(n+2) of tensor work to hide behind.
      bool ok = ra_wait_warp(bar(L::B_KV), 0, abort_flag);
      auto head_s = [&](int m) -> bool {
        const int st = m % L::NS;
        if (!ra_wait_warp(bar(L::B_QF + st), (m / L::NS) & 1, abort_flag)) return false;
        tc_fence_after();
        issue_sd(tmem + (m & 1) * L::SLOT_COLS + L::SLOT_ST, ka_k, sbase + L::OFF_Q + st * L::Q_BYTES);
        mma_commit_w(bar(L::B_SFULL + (m & 1)));
        return true;
      };
      auto head_dp = [&](int m) -> bool {
        const int s = m & 1, st = m % L::NS;
        if (m >= L::NSLOT && !ra_wait_warp(bar(L::B_SLOTFREE + s), ((m >> 1) - 1) & 1, abort_flag)) return false;
        tc_fence_after();
        issue_sd(tmem + s * L::SLOT_COLS + L::SLOT_DPT, va_k, sbase + L::OFF_DO + st * L::Q_BYTES);
        mma_commit_w(bar(L::B_DPFULL + s));
        return true;
      };
      for (int m = 0; ok && m < N && m < L::NSLOT; ++m) ok = head_s(m) && head_dp(m);
      for (int t = 0; ok && t < N; ++t) {
        const int s = t & 1, st = t % L::NS;
        if (!(ok = ra_wait_warp(bar(L::B_DSREADY + s), (t >> 1) & 1, abort_flag))) break;
        tc_fence_after();
        const uint32_t slot = tmem + s * L::SLOT_COLS;
        issue_dq(slot + L::SLOT_DQT, sbase + L::OFF_DS + s * L::DS_BYTES);
        mma_commit_w(bar(L::B_DQFULL + s));
        issue_kv(tmem + L::COL_DV, slot + L::SLOT_PT, sbase + L::OFF_DO + st * L::Q_BYTES, t > 0);
        issue_kv(tmem + L::COL_DK, slot + L::SLOT_DST, sbase + L::OFF_Q + st * L::Q_BYTES, t > 0);
        mma_commit_w(bar(L::B_QE + st));
        if (t + L::NSLOT < N) ok = head_s(t + L::NSLOT) && head_dp(t + L::NSLOT);
      }
      mma_commit_w(bar(L::B_FINAL));
      ra_wait_drain(bar(L::B_FINAL), 0);
    }
    __syncwarp();
  } else if ((warp >= 4 && warp < 8) || warp >= 12) {
    // ------------------------------------------------------------ softmax groups: one key row per thread
    const int half = warp >= 12;                     // query columns [32*half, 32*half + 32) of each tile
    const int c0 = half * 32;
    const int sub = warp & 3;
    const int row = sub * 32 + lane;
    const int64_t j = k0 + row;                      // this thread's key
    const bool row_valid = j < S;
    const int64_t jc = row_valid ? j : S - 1;
    const uint32_t lane_off = (uint32_t)(sub * 32) << 16;
    const uint32_t trow = tmem + lane_off;
    const bool key_in = RA_IN_RANGE(jc, S, kSiteBwdKeyRow);
    const int my_seg = use_seg && key_in ? p.seg[b * p.seg_sb + jc * p.seg_ss] : 0;
    float brow = 0.f;                                // bias of this key, log2 units
    if (use_bias && key_in) brow = p.bias[b * p.bias_sb + jc * p.bias_ss] * kLog2e;
    const int32_t cbs = p.rd.cbs;
    const int64_t i_first = cbs > 0 ? (j / cbs) * (int64_t)cbs : 0;   // first query that can see key j
    // A query tile starting at q0 needs the causal mask iff q0 is before the
    // causal block of the tile's last key (no per-tile division).
    const int64_t k_last_blk = cbs > 0 ? ((k0 + kTile - 1) / cbs) * (int64_t)cbs : 0;
    const float sc = p.scale_log2;
#ifdef RA_DEBUG_COUNT
    int dbg_vis = 0;
#endif
    int n = 0;
    bool ok = true;
    if (!dead) {
      QIter it;
      q_iter_init(it, p.rd, k0, meta_b, use_seg);
      for (int32_t q = q_iter_next_warp(it, p.rd); q >= 0; q = q_iter_next_warp(it, p.rd), ++n) {
        const int st = n % L::NS, s = n & 1;
        const uint32_t slot = trow + s * L::SLOT_COLS;
        const int64_t q0 = (int64_t)q * L::QT;
        // the query tile's metadata load is issued before the waits, so it lands meanwhile
        const int4 qm = meta_b && RA_IN_RANGE(q0 / kTile, p.rd.ntiles, kSiteBwdQueryMeta) ? load_meta(meta_b + q0 / kTile)
                                                                                      : make_int4(0, 0, 3, 0);
        if (!(ok = ra_wait_warp(bar(L::B_QF + st), (n / L::NS) & 1, abort_flag))) break;
        if (!(ok = ra_wait_warp(bar(L::B_SFULL + s), (n >> 1) & 1, abort_flag))) break;
        tc_fence_after();
        uint32_t sr[32];
        tmem_ld32(slot + L::SLOT_ST + c0, sr);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 32; ++c) reg_fence(sr[c]);
        float* x = reinterpret_cast<float*>(sr);
        // this group's 32 queries of the stage's -lse*log2e and -Delta rows, read
        // four at a time (every lane reads the same address)
        const uint32_t nl = sbase + L::OFF_LD + st * L::LD_BYTES + c0 * 4;
        const uint32_t nd = nl + L::QT * 4;
        // x = S * log2(e)/sqrt(D) + bias(key) - lse(query) * log2(e), two columns per instruction
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          const float4 bl = ld_shared_f4(nl + c * 4);
          float b0 = bl.x, b1 = bl.y, b2 = bl.z, b3 = bl.w;
          if (use_bias) {
            fadd2(b0, b1, b0, b1, brow, brow);
            fadd2(b2, b3, b2, b3, brow, brow);
          }
          ffma2(x[c], x[c + 1], x[c], x[c + 1], sc, sc, b0, b1);
          ffma2(x[c + 2], x[c + 3], x[c + 2], x[c + 3], sc, sc, b2, b3);
        }
        // per-element mask on causal-diagonal / ragged / mixed-segment tiles
        const bool need_causal = cbs > 0 && q0 < k_last_blk;
        const bool need_ragged = (q0 + L::QT > S) || (k0 + kTile > S);
        const bool need_seg = use_seg && !(qm.x == qm.y && km.x == km.y && qm.x == km.x);
        if (need_causal || need_ragged || need_seg || !row_valid) {
          const int64_t cmin64 = i_first - (q0 + c0);              // visible iff c >= cmin
          const int cmin = cmin64 < 0 ? 0 : (cmin64 > 32 ? 32 : (int)cmin64);
          const int64_t cmax64 = S - (q0 + c0);                    // valid iff c < cmax
          const int cmax = row_valid ? (cmax64 > 32 ? 32 : (cmax64 < 0 ? 0 : (int)cmax64)) : 0;
          uint32_t vb = ~0u;
          if (need_seg && qm.x == qm.y) {
            vb = my_seg == qm.x ? ~0u : 0u;   // every query of the tile is in segment qm.x
          } else if (need_seg) {
            const int32_t* sp = p.seg + b * p.seg_sb;
            vb = 0;
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              const int64_t i = q0 + c0 + c < S ? q0 + c0 + c : S - 1;
              vb |= (uint32_t)(RA_IN_RANGE(i, S, kSiteBwdQuerySeg) && __ldg(sp + i * p.seg_ss) == my_seg) << c;
            }
          }
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const bool vis = c >= cmin && c < cmax && ((vb >> c) & 1u);
            x[c] = vis ? x[c] : -INFINITY;
          }
        }
#ifdef RA_DEBUG_COUNT
        // visible pairs as decided by this kernel's own tile skipping and masking
#pragma unroll
        for (int c = 0; c < 32; ++c) dbg_vis += x[c] != -INFINITY;
#endif
        float pr[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) pr[c] = ex2_approx(x[c]);
        if (!(ok = ra_wait_warp(bar(L::B_DPFULL + s), (n >> 1) & 1, abort_flag))) break;
        tc_fence_after();
        uint32_t dr[32];
        tmem_ld32(slot + L::SLOT_DPT + c0, dr);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 32; ++c) reg_fence(dr[c]);
        uint32_t pp[16], dd[16];
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          const float4 dl = ld_shared_f4(nd + c * 4);
          float t0, t1, t2, t3, ds0, ds1, ds2, ds3;
          fadd2(t0, t1, __uint_as_float(dr[c]), __uint_as_float(dr[c + 1]), dl.x, dl.y);   // dP - Delta
          fadd2(t2, t3, __uint_as_float(dr[c + 2]), __uint_as_float(dr[c + 3]), dl.z, dl.w);
          fmul2(ds0, ds1, pr[c], pr[c + 1], t0, t1);
          fmul2(ds2, ds3, pr[c + 2], pr[c + 3], t2, t3);
          pp[c >> 1] = pack_bf16x2(pr[c], pr[c + 1]);
          pp[(c >> 1) + 1] = pack_bf16x2(pr[c + 2], pr[c + 3]);
          dd[c >> 1] = pack_bf16x2(ds0, ds1);
          dd[(c >> 1) + 1] = pack_bf16x2(ds2, ds3);
        }
        // P^T and dS^T (bf16, two per column) into this slot's first half.
        tmem_st16(slot + L::SLOT_PT + c0, pp);
        tmem_st16(slot + L::SLOT_DST + c0, dd);
        // dS^T into shared memory for dQ^T = K^T dS^T (MN-major, 128-byte swizzle):
        // key row `row` is one 128-byte line; 16-byte chunk c lands at c ^ (row % 8).
        const uint32_t line = sbase + L::OFF_DS + s * L::DS_BYTES + row * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int chunk = half * 4 + c;
          const uint32_t off = (uint32_t)row * 128 + ((chunk ^ (row & 7)) << 4);   // within this slot's dS^T buffer
          if (RA_IN_RANGE(off + 15, L::DS_BYTES, kSiteBwdDsSmem))
            st_shared_v4(line - (uint32_t)row * 128 + off, dd[4 * c], dd[4 * c + 1], dd[4 * c + 2], dd[4 * c + 3]);
        }
        fence_proxy_async_smem();
        tmem_st_wait();
        tc_fence_before();
        // one arrive per warp: per-lane arrives on one barrier serialise in the
        // shared-memory pipe, which the tensor cores' operand reads also use
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::B_DSREADY + s));
      }
    }
#ifdef RA_DEBUG_COUNT
    // the two column halves of a key row add their counts
    if (row_valid && ok && p.dbg_count) atomicAdd(p.dbg_count + ((int64_t)b * p.H + h) * S + j, dbg_vis);
#endif
    // ---------------------------------------------------------- epilogue: dK (columns group 0) or dV (group 1)
    bool have = n > 0 && ok;
    if (have) have = ra_wait(bar(L::B_FINAL), 0, abort_flag);
    have = __all_sync(0xffffffffu, have);
    n = __shfl_sync(0xffffffffu, n, 0);
    tc_fence_after();
    {
      const int which = half;
      const uint32_t col = which == 0 ? L::COL_DK : L::COL_DV;
      const float mul = which == 0 ? p.scale : 1.f;
      char* base = static_cast<char*>(which == 0 ? p.dk : p.dv);
      const int64_t sb = which == 0 ? p.dk_sb : p.dv_sb, ss = which == 0 ? p.dk_ss : p.dv_ss,
                    sh = which == 0 ? p.dk_sh : p.dv_sh;
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
        if (row_valid && (have || n == 0) && key_in) {
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
  } else if (warp >= 8 && warp < 12) {
    // ------------------------------------------------------------ dQ readout: thread = head-dim lane d
    const int sub = warp & 3;
    const int d = sub * 32 + lane;
    const bool leader = threadIdx.x == 256;
    const uint32_t trow = tmem + ((uint32_t)(sub * 32) << 16);
    const uint32_t dqs = sbase + L::OFF_DQS;
    bool pending = false;   // leader: a bulk reduce may still be reading the staging tile
    if (!dead) {
      if (leader) prefetch_tmap(&tm_dq);
      QIter it;
      q_iter_init(it, p.rd, k0, meta_b, use_seg);
      int n = 0;
      for (int32_t q = q_iter_next_warp(it, p.rd); q >= 0; q = q_iter_next_warp(it, p.rd), ++n) {
        const int s = n & 1;
        if (!ra_wait_warp(bar(L::B_DQFULL + s), (n >> 1) & 1, abort_flag)) break;
        tc_fence_after();
        uint32_t r[64];
        tmem_ld32(trow + s * L::SLOT_COLS + L::SLOT_DQT, r);
        tmem_ld32(trow + s * L::SLOT_COLS + L::SLOT_DQT + 32, r + 32);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 64; ++c) reg_fence(r[c]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::B_SLOTFREE + s));
        // The previous tile's bulk reduce must have read the staging tile before
        // it is rewritten; that wait comes only now, after the TMEM slot was
        // released, so the next S^T / dP^T never waits on the reduction.
        if (leader && pending) {
          bulk_wait_group_read0();
          mbar_arrive(bar(L::B_DQSFREE));
          pending = false;
        }
        // staging tile [query c][d]: a warp writes 32 consecutive floats per row
        if (n > 0 && !ra_wait_warp(bar(L::B_DQSFREE), (n - 1) & 1, abort_flag)) break;
        if (d < D) {   // at D = 64 the upper half of dQ^T is the zero padding
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (RA_IN_RANGE(c * (D * 4) + d * 4 + 3, L::DQS_BYTES, kSiteBwdDqStaging))
              st_shared_f32(dqs + c * (D * 4) + d * 4, __uint_as_float(r[c]) * p.scale);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::B_DQSFULL));
        if (leader) {
          if (!ra_wait(bar(L::B_DQSFULL), n & 1, abort_flag)) break;
          // rows past S fall outside the tensor map and are not written
          tma_reduce_add_3d(&tm_dq, dqs, 0, q * L::QT, bh);
          bulk_commit_group();
          pending = true;
        }
      }
    }
    if (leader && pending) bulk_wait_group0();
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
