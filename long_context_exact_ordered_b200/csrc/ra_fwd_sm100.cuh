// sm_100a forward: blockwise exact attention over the virtual ring, bf16 in,
// fp32 accumulate, tcgen05 MMAs into TMEM.
//
// Work unit = one (batch, head, pair of 128-row query tiles).  The pair
// stays resident (the pages' "each device keeps its query block", page
// "手把手拆解RingAttention" §1) while 128-key K/V tiles stream through
// double-buffered shared-memory stages in ring order (page "Ring
// Attention技术解析" §2.2: a device holds the current block and the incoming
// one), loaded by TMA.
//
// Roles (384 threads):
//   warp 0      TMA producer (the whole warp walks the schedule, one elected
//               lane issues copies): Q pair once, then K_t, V_t per tile.
//   warp 1      TMEM owner; the whole warp runs the issue loop and one
//               elected lane issues every tcgen05.mma:
//                 S_q = Q_q K_t^T  (SS form, both K-major, M=N=128, fp32 in TMEM)
//                 O_q += P_q V_t   (TS form: P from TMEM, V MN-major from SMEM)
//   warps 4-7   softmax for query tile 0, warps 8-11 for query tile 1: thread
//               r owns row r of S (TMEM lane r), so row max and row sum are
//               thread-local.  Masks, scale and bias are applied, the exp2
//               online softmax runs with a lazily updated reference max, P is
//               written back into the S columns of TMEM as bf16.
//   warps 2-3   idle.
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+D), O1 after it.
//
// Exactness of the lazy max: O and l are both kept relative to the same
// reference m_ref; m_ref only moves when a tile's max exceeds it by more than
// 8 (log2 units), so unnormalised probabilities stay <= 2^8 and the final
// O / l is unchanged.
//
// Pipeline: order per key tile PV0(t), S0(t+1), PV1(t), S1(t+1): while
// softmax 1 works on S1(t) the tensor core runs PV0/S0, and vice versa.
// S_q(t+1) reuses the TMEM columns holding P_q(t); it is issued by the same
// thread right behind PV_q(t) and the tensor pipe executes a thread's MMAs
// in issue order.  P_q(t) is signalled per half of the keys and PV_q(t) is
// issued in two halves, so the first half runs while the softmax still
// computes P for the second.
//
// Ring-step mode (STEP = true, the per-step entry ra_step): the same kernel
// runs one iteration of the ring loop on its own.  The query block (Sq
// tokens starting at global token q_off) meets one visiting key/value block
// (Sk tokens starting at k_off); masks use global positions; the block's
// tiles are visited in order (StepKvIter); and the epilogue merges the
// block's partial (reference max, sum, unnormalised O) into the caller's
// running fp32 state (m, l, o_acc) instead of writing O and LSE.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "ra_common.cuh"

namespace ra {

template <int D>
struct FwdLayout {
  static_assert(D == 64 || D == 128, "head_dim must be 64 or 128");
  static constexpr int KCH = D / 64;                 // 128-byte swizzle chunks along D
  static constexpr int TILE_BYTES = kTile * D * 2;   // one 128 x D bf16 tile
  static constexpr int CHUNK_BYTES = kTile * 128;    // one 128-row x 128-byte TMA box
  static constexpr int KS = D == 128 ? 2 : 3;        // K stages
  static constexpr int VS = D == 128 ? 2 : 3;        // V stages
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * TILE_BYTES;
  static constexpr int OFF_V = OFF_K + KS * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_V + VS * TILE_BYTES;
  // barriers
  static constexpr int B_Q = 0;
  static constexpr int B_KFULL = 1;
  static constexpr int B_KEMPTY = B_KFULL + KS;
  static constexpr int B_VFULL = B_KEMPTY + KS;
  static constexpr int B_VEMPTY = B_VFULL + VS;
  static constexpr int B_SFULL = B_VEMPTY + VS;      // [2]
  static constexpr int B_PFULL = B_SFULL + 2;        // [2][2]: P of keys 0-63 / 64-127 written, per query tile
  static constexpr int B_PVDONE = B_PFULL + 4;       // [2]
  static constexpr int B_DRAIN = B_PVDONE + 2;       // issuer's final commit
  static constexpr int NBAR = B_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;   // tmem slot, abort flag
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int SMEM_ALLOC = BYTES + 1024;       // slack for 1024-byte alignment
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O0 = 256, COL_O1 = 256 + D;
  // Register split (setmaxnreg): warpgroup 0 (producer, MMA issuer) gives up
  // registers to the two softmax warpgroups.  The host checks
  // 128*REGS_LOW + 256*REGS_HIGH <= 384 * (registers per thread at launch)
  // before launching, so the increase can always be satisfied.
  static constexpr int REGS_LOW = 88, REGS_HIGH = 200;
  static constexpr int THREADS = 384;
};

struct FwdParams {
  RingDesc rd;
  int32_t B, H;
  int32_t npairs;          // ceil(ntiles / 2)
  float scale_log2;        // log2(e) / sqrt(D)
  __nv_bfloat16* o;        // [B, S, H, D]
  int64_t o_sb, o_ss, o_sh;
  float* lse;              // [B, H, S], natural log
  int64_t lse_sb, lse_sh, lse_ss;
  const int32_t* seg;      // [B, S] or null
  int64_t seg_sb, seg_ss;
  const float* bias;       // [B, S] or null
  int64_t bias_sb, bias_ss;
  const int4* meta;        // [B, ntiles] or null
  int32_t* dbg_count;      // RA_DEBUG_COUNT builds: visible keys per query row, [B, H, S]
  // Ring-step mode only (rd.S is then Sq, `seg` the query block's ids and
  // `bias` the visiting keys' bias [B, Sk]).
  int64_t Sk, q_off, k_off;
  const int32_t* seg_k;    // [B, Sk] visiting keys' segment ids, or null
  int64_t segk_sb, segk_ss;
  float* acc;              // [B, Sq, H, D] fp32 running unnormalised output
  int64_t acc_sb, acc_ss, acc_sh;
  float* m_state;          // [B, H, Sq] running max (natural-log units)
  float* l_state;          // [B, H, Sq] running sum
  int64_t ml_sb, ml_sh, ml_ss;
  int32_t kv_bcast;        // 1: the key/value block (and its bias / segment ids) has batch 1, shared by every query row b
};

// The key/value tiles a pair of query tiles visits: the whole ring
// (KvIter, tile metadata precomputed) or, in ring-step mode, the visiting
// block (StepKvIter, metadata computed on the fly).  Every lane of a warp
// calls these.
template <bool STEP>
struct FwdTiles;

template <>
struct FwdTiles<false> {
  KvIter it;
  const int4* meta_b;
  int32_t ntiles;
  __device__ __forceinline__ void init(const FwdParams& p, int, int64_t q0, const int4* mb, bool use_seg,
                                       bool use_bias) {
    meta_b = mb;
    ntiles = p.rd.ntiles;
    kv_iter_init(it, p.rd, q0, q0 + 2 * kTile - 1, mb, use_seg, use_bias);
  }
  __device__ __forceinline__ int32_t next(const FwdParams& p) { return kv_iter_next_warp(it, p.rd); }
  __device__ __forceinline__ int4 meta(int32_t t) const {
    return meta_b && RA_IN_RANGE(t, ntiles, kSiteFwdTileMeta) ? load_meta(meta_b + t)
                                                              : make_int4(0, 0, kMetaAnyFinite | kMetaAllZero, 0);
  }
};

template <>
struct FwdTiles<true> {
  StepKvIter it;
  int4 km;
  __device__ __forceinline__ void init(const FwdParams& p, int b, int64_t q0, const int4*, bool use_seg,
                                       bool use_bias) {
    step_iter_init_warp(it, q0, q0 + 2 * kTile - 1, p.rd.S, p.Sk, p.q_off, p.k_off, p.rd.cbs,
                        use_seg ? p.seg + b * p.seg_sb : nullptr, p.seg_ss,
                        use_seg ? p.seg_k + (p.kv_bcast ? 0 : b) * p.segk_sb : nullptr, p.segk_ss,
                        use_bias ? p.bias + (p.kv_bcast ? 0 : b) * p.bias_sb : nullptr, p.bias_ss);
  }
  __device__ __forceinline__ int32_t next(const FwdParams&) { return step_iter_next_warp(it, km); }
  __device__ __forceinline__ int4 meta(int32_t) const { return km; }
};

constexpr float kRescaleThreshold = 8.0f;   // log2 units

template <int D, bool STEP>
__global__ void __launch_bounds__(384, 1)
    ra_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ FwdParams p) {
  using L = FwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Head-major order (resident CTAs share one head's K / V in L2); within a
  // head the longest causal units (last query pairs) launch first.
  const int unit = blockIdx.x;
  const int pair = p.npairs - 1 - unit % p.npairs;
  const int bh = unit / p.npairs;
  const int b = bh / p.H, h = bh % p.H;
  const int bk = (STEP && p.kv_bcast) ? 0 : b;   // batch row of the key/value side
  const int64_t q0 = (int64_t)pair * 2 * kTile;
  const int64_t S = p.rd.S;                   // query rows (Sq in ring-step mode)
  const int64_t Sk = STEP ? p.Sk : S;         // key rows
  if (!(RA_IN_RANGE(b, p.B, kSiteFwdUnit) && RA_IN_RANGE(h, p.H, kSiteFwdUnit))) return;   // debug build only

  auto bar = [&](int i) -> uint32_t { return sbase + L::OFF_BAR + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::OFF_MISC + 4);

  if (threadIdx.x == 0) {
    mbar_init(bar(L::B_Q), 1);
    for (int i = 0; i < L::KS; ++i) { mbar_init(bar(L::B_KFULL + i), 1); mbar_init(bar(L::B_KEMPTY + i), 1); }
    for (int i = 0; i < L::VS; ++i) { mbar_init(bar(L::B_VFULL + i), 1); mbar_init(bar(L::B_VEMPTY + i), 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(L::B_SFULL + i), 1);
      mbar_init(bar(L::B_PFULL + 2 * i), 4);       // one arrive per softmax warp
      mbar_init(bar(L::B_PFULL + 2 * i + 1), 4);
      mbar_init(bar(L::B_PVDONE + i), 1);
    }
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

  const bool use_seg = p.seg != nullptr, use_bias = p.bias != nullptr;
  const int4* meta_b = p.meta ? p.meta + (int64_t)b * p.rd.ntiles : nullptr;

  if (warp < 4) {
  regs_dec<L::REGS_LOW>();
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // The whole warp runs the loop (its lanes scan 32 KV tiles per metadata
    // round trip, kv_iter_next_warp); one elected lane issues the copies.
    {
      if (elect_one()) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        mbar_arrive_expect_tx(bar(L::B_Q), 2 * L::TILE_BYTES);
        for (int qt = 0; qt < 2; ++qt)
          for (int c = 0; c < L::KCH; ++c)
            tma_load_4d(sbase + L::OFF_Q + qt * L::TILE_BYTES + c * L::CHUNK_BYTES, &tm_q, bar(L::B_Q), c * 64, h,
                        (int)(q0 + qt * kTile), b);
      }
      __syncwarp();
      FwdTiles<STEP> tiles;
      tiles.init(p, b, q0, meta_b, use_seg, use_bias);
      const uint64_t pol = l2_policy_evict_last();   // K/V tiles are re-read by every query pair of the head
      int nk = 0, nv = 0;   // K / V tiles issued
      for (int32_t t = tiles.next(p); t >= 0; t = tiles.next(p)) {
        const int ks = nk % L::KS, vs = nv % L::VS;
        if (nk >= L::KS && !ra_wait_warp(bar(L::B_KEMPTY + ks), ((nk / L::KS) & 1) ^ 1, abort_flag)) break;
        if (elect_one()) {
          mbar_arrive_expect_tx(bar(L::B_KFULL + ks), L::TILE_BYTES);
          for (int c = 0; c < L::KCH; ++c)
            tma_load_4d_hint(sbase + L::OFF_K + ks * L::TILE_BYTES + c * L::CHUNK_BYTES, &tm_k, bar(L::B_KFULL + ks),
                             c * 64, h, t * kTile, bk, pol);
        }
        __syncwarp();
        ++nk;
        if (nv >= L::VS && !ra_wait_warp(bar(L::B_VEMPTY + vs), ((nv / L::VS) & 1) ^ 1, abort_flag)) break;
        if (elect_one()) {
          mbar_arrive_expect_tx(bar(L::B_VFULL + vs), L::TILE_BYTES);
          for (int c = 0; c < L::KCH; ++c)
            tma_load_4d_hint(sbase + L::OFF_V + vs * L::TILE_BYTES + c * L::CHUNK_BYTES, &tm_v, bar(L::B_VFULL + vs),
                             c * 64, h, t * kTile, bk, pol);
        }
        __syncwarp();
        ++nv;
      }
      // Drain: every load issued must land before the block may exit.
      ra_wait_drain(bar(L::B_Q), 0);
      for (int i = nk - L::KS; i < nk; ++i)
        if (i >= 0) ra_wait_drain(bar(L::B_KFULL + i % L::KS), (i / L::KS) & 1);
      for (int i = nv - L::VS; i < nv; ++i)
        if (i >= 0) ra_wait_drain(bar(L::B_VFULL + i % L::VS), (i / L::VS) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    {   // the whole warp runs the issuer; one elected lane issues (ptx.cuh)
      constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, false, true);
      const uint32_t tS[2] = {tmem + L::COL_S0, tmem + L::COL_S1};
      const uint32_t tO[2] = {tmem + L::COL_O0, tmem + L::COL_O1};
      auto issue_s = [&](int qt, int ks) {
        const uint32_t qa = sbase + L::OFF_Q + qt * L::TILE_BYTES;
        const uint32_t ka = sbase + L::OFF_K + ks * L::TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * L::CHUNK_BYTES + (kk % 4) * 32;
          mma_ss_w(tS[qt], smem_desc_sw128(qa + off, 16, 1024), smem_desc_sw128(ka + off, 16, 1024), IDESC_S,
                 kk > 0);
        }
      };
      auto issue_pv = [&](int qt, int vs, int key_half, bool acc) {   // keys 64*key_half .. +63
        const uint32_t va = sbase + L::OFF_V + vs * L::TILE_BYTES;
#pragma unroll
        for (int k = 0; k < kTile / 32; ++k) {
          const int kk = key_half * (kTile / 32) + k;
          mma_ts_w(tO[qt], tS[qt] + kk * 8, smem_desc_sw128(va + kk * 2048, L::CHUNK_BYTES, 1024), IDESC_PV,
                   (acc || k > 0) ? 1u : 0u);
        }
      };
      FwdTiles<STEP> tiles;
      tiles.init(p, b, q0, meta_b, use_seg, use_bias);
      int32_t t = tiles.next(p);
      bool ok = ra_wait_warp(bar(L::B_Q), 0, abort_flag);
      if (ok && t >= 0) {
        ok = ra_wait_warp(bar(L::B_KFULL + 0), 0, abort_flag);
        if (ok) {
          tc_fence_after();
          issue_s(0, 0);
          mma_commit_w(bar(L::B_SFULL + 0));
          issue_s(1, 0);
          mma_commit_w(bar(L::B_SFULL + 1));
          mma_commit_w(bar(L::B_KEMPTY + 0));
        }
        for (int n = 0; ok; ++n) {
          const int32_t tn = tiles.next(p);
          const bool last = tn < 0;
          const int vs = n % L::VS, ks1 = (n + 1) % L::KS;
          const uint32_t ph = n & 1;
          if (!(ok = ra_wait_warp(bar(L::B_VFULL + vs), (n / L::VS) & 1, abort_flag))) break;
          // query tile 0
          // PV in two halves of the keys: the first runs while the softmax
          // still computes P for the second
          if (!(ok = ra_wait_warp(bar(L::B_PFULL + 0), ph, abort_flag))) break;
          tc_fence_after();
          issue_pv(0, vs, 0, n > 0);
          if (!(ok = ra_wait_warp(bar(L::B_PFULL + 1), ph, abort_flag))) break;
          tc_fence_after();
          issue_pv(0, vs, 1, true);
          mma_commit_w(bar(L::B_PVDONE + 0));
          if (!last) {
            // S0(n+1) overwrites the TMEM columns PV0(n) reads P0 from; the
            // tensor pipe executes this thread's MMAs in issue order, so it is
            // issued right behind PV0(n) without waiting for its completion.
            if (!(ok = ra_wait_warp(bar(L::B_KFULL + ks1), ((n + 1) / L::KS) & 1, abort_flag))) break;
            issue_s(0, ks1);
            mma_commit_w(bar(L::B_SFULL + 0));
          }
          // query tile 1
          if (!(ok = ra_wait_warp(bar(L::B_PFULL + 2), ph, abort_flag))) break;
          tc_fence_after();
          issue_pv(1, vs, 0, n > 0);
          if (!(ok = ra_wait_warp(bar(L::B_PFULL + 3), ph, abort_flag))) break;
          tc_fence_after();
          issue_pv(1, vs, 1, true);
          mma_commit_w(bar(L::B_PVDONE + 1));
          mma_commit_w(bar(L::B_VEMPTY + vs));
          if (!last) {
            issue_s(1, ks1);
            mma_commit_w(bar(L::B_SFULL + 1));
            mma_commit_w(bar(L::B_KEMPTY + ks1));
          }
          if (last) break;
        }
      }
      // Every MMA and commit issued above must complete before TMEM is freed
      // and before the block's shared memory (barriers included) is released.
      mma_commit_w(bar(L::B_DRAIN));
      ra_wait_drain(bar(L::B_DRAIN), 0);
    }
    __syncwarp();
  }
  } else {
    // ------------------------------------------------------------ softmax
    regs_inc<L::REGS_HIGH>();
    const int qt = (warp - 4) >> 2;
    const int sub = warp & 3;
    const int row = sub * 32 + lane;
    const int64_t q_first = q0 + qt * kTile;
    const int64_t qrow = q_first + row;
    const uint32_t lane_off = (uint32_t)(sub * 32) << 16;
    const uint32_t tS_row = tmem + lane_off + (qt ? L::COL_S1 : L::COL_S0);
    const uint32_t tO_row = tmem + lane_off + (qt ? L::COL_O1 : L::COL_O0);
    const int64_t qrow_c = qrow < S ? qrow : S - 1;
    const int my_seg = use_seg && RA_IN_RANGE(qrow_c, S, kSiteFwdQuerySeg) ? p.seg[b * p.seg_sb + qrow_c * p.seg_ss] : 0;
    // key-side segment ids (the visiting block's in ring-step mode)
    const int32_t* segk = STEP ? p.seg_k : p.seg;
    const int64_t segk_sb = STEP ? p.segk_sb : p.seg_sb, segk_ss = STEP ? p.segk_ss : p.seg_ss;
    int4 qm = make_int4(0, 0, kMetaAnyFinite | kMetaAllZero, 0);
    if constexpr (STEP) {
      if (use_seg) {
        const int2 r = step_q_seg_range_warp(p.seg + b * p.seg_sb, p.seg_ss, q_first, q_first + kTile - 1, S);
        qm.x = r.x;
        qm.y = r.y;
      }
    } else {
      const int q_tile_idx = (int)(q_first / kTile);
      if (meta_b && q_tile_idx < p.rd.ntiles) qm = load_meta(meta_b + q_tile_idx);
    }
    const int32_t cbs = p.rd.cbs;
    // Masks compare global positions; keys are indexed locally from k_base.
    const int64_t q_base = STEP ? p.q_off : 0, k_base = STEP ? p.k_off : 0;
    const int64_t causal_jmax = cbs > 0 ? ((q_base + qrow) / cbs + 1) * (int64_t)cbs - 1 - k_base : Sk - 1;
    // Per-tile mask test without divisions: a KV tile needs the per-element
    // mask iff it reaches past the causal block of the tile's first query
    // (k_last > q_blk_end), runs past the last key, or mixes segment ids.
    const int64_t q_blk_end = cbs > 0 ? ((q_base + q_first) / cbs + 1) * (int64_t)cbs - 1 - k_base : INT64_MAX;
    const bool q_seg_uniform = qm.x == qm.y;

    FwdTiles<STEP> tiles;
    tiles.init(p, b, q0, meta_b, use_seg, use_bias);
    float m_ref = -INFINITY, l = 0.f;
#ifdef RA_DEBUG_COUNT
    int dbg_vis = 0;
#endif
    int n = 0;
    bool ok = true;
    for (int32_t t = tiles.next(p); t >= 0; t = tiles.next(p), ++n) {
      // the tile's metadata load is issued before the wait, so it lands while S is computed
      const int4 km = tiles.meta(t);
      if (!(ok = ra_wait_warp(bar(L::B_SFULL + qt), n & 1, abort_flag))) break;
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld32(tS_row + 0, sr);
      tmem_ld32(tS_row + 32, sr + 32);
      tmem_ld32(tS_row + 64, sr + 64);
      tmem_ld32(tS_row + 96, sr + 96);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 128; ++c) reg_fence(sr[c]);
      float* x = reinterpret_cast<float*>(sr);

      const int64_t k0 = (int64_t)t * kTile;
      // Scores stay raw (the scale is folded into the exponent's FMA) unless a
      // non-zero bias must be added first; loads are issued 32 keys at a time
      // (the empty asm keeps the compiler from hoisting all 128 and spilling).
      const bool has_bias = use_bias && !(km.z & kMetaAllZero);
      if (has_bias) {
        const float* bp = p.bias + bk * p.bias_sb;
#pragma unroll
        for (int c0 = 0; c0 < 128; c0 += 32) {
#pragma unroll
          for (int c = c0; c < c0 + 32; ++c) {
            const int64_t j = k0 + c < Sk ? k0 + c : Sk - 1;
            const float bj = RA_IN_RANGE(j, Sk, kSiteFwdKeyBias) ? __ldg(bp + j * p.bias_ss) : 0.f;
            x[c] = fmaf(x[c], p.scale_log2, bj * kLog2e);
          }
          asm volatile("" ::: "memory");
        }
      }
      // per-element mask on diagonal / ragged / mixed-segment tiles
      const int64_t k_last = k0 + kTile - 1;
      const bool need_mask = k_last > Sk - 1 || k_last > q_blk_end ||
                             (use_seg && !(q_seg_uniform && km.x == km.y && qm.x == km.x));
      if (need_mask) {
        int64_t jmax = causal_jmax < Sk - 1 ? causal_jmax : Sk - 1;
        const int64_t lim64 = jmax - k0;
        const int lim = lim64 < -1 ? -1 : (lim64 > 127 ? 127 : (int)lim64);
        uint32_t vb[4] = {~0u, ~0u, ~0u, ~0u};   // segment match bits, 32 keys per word
        if (use_seg && km.x == km.y) {
          // every key of the tile is in segment km.x: the row sees all or none
          const uint32_t all = my_seg == km.x ? ~0u : 0u;
          vb[0] = vb[1] = vb[2] = vb[3] = all;
        } else if (use_seg) {
          const int32_t* sp = segk + bk * segk_sb;
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            uint32_t bits = 0;
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              const int64_t j = k0 + 32 * w + c < Sk ? k0 + 32 * w + c : Sk - 1;
              bits |= (uint32_t)(RA_IN_RANGE(j, Sk, kSiteFwdKeySeg) && __ldg(sp + j * segk_ss) == my_seg) << c;
            }
            vb[w] = bits;
            asm volatile("" ::: "memory");
          }
        }
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          const bool vis = (c <= lim) && ((vb[c >> 5] >> (c & 31)) & 1u);
          x[c] = vis ? x[c] : -INFINITY;
        }
      }
#ifdef RA_DEBUG_COUNT
      // visible pairs as decided by this kernel's own tile skipping and
      // masking: every score still finite here enters the softmax
#pragma unroll
      for (int c = 0; c < 128; ++c) dbg_vis += x[c] != -INFINITY;
#endif
      // tile max (three-input max, two independent chains)
      float mx0 = fmaxf(x[0], x[1]), mx1 = fmaxf(x[2], x[3]);
#pragma unroll
      for (int c = 4; c < 128; c += 4) {
        mx0 = fmax3(mx0, x[c], x[c + 1]);
        mx1 = fmax3(mx1, x[c + 2], x[c + 3]);
      }
      const float sc = has_bias ? 1.f : p.scale_log2;   // x * sc is the score in log2 units
      const float mx = fmaxf(mx0, mx1) * sc;
      const bool need = mx > m_ref + kRescaleThreshold;
      float alpha = 1.f;
      if (need) {
        alpha = (m_ref == -INFINITY) ? 0.f : ex2_approx(m_ref - mx);
        m_ref = mx;
        l *= alpha;
      }
      if (n > 0 && __any_sync(0xffffffffu, need)) {
        // rescale this warp's O rows in TMEM (PV of the previous tile has completed:
        // the commit that released S_q(n) covers it)
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t orow[32];
          tmem_ld32(tO_row + c, orow);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            reg_fence(orow[e]);
            orow[e] = __float_as_uint(__uint_as_float(orow[e]) * alpha);
          }
          tmem_st32(tO_row + c, orow);
        }
      }
      const float nref = (m_ref == -INFINITY) ? 0.f : -m_ref;
      float l0 = 0.f, l1 = 0.f, l2 = 0.f, l3 = 0.f;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 64; c += 4) {
          const int i = half * 64 + c;
          float a0, a1, a2, a3;
          ffma2(a0, a1, x[i], x[i + 1], sc, sc, nref, nref);
          ffma2(a2, a3, x[i + 2], x[i + 3], sc, sc, nref, nref);
          const float e0 = ex2_approx(a0), e1 = ex2_approx(a1), e2 = ex2_approx(a2), e3 = ex2_approx(a3);
          fadd2(l0, l1, l0, l1, e0, e1);
          fadd2(l2, l3, l2, l3, e2, e3);
          pk[c >> 1] = pack_bf16x2(e0, e1);
          pk[(c >> 1) + 1] = pack_bf16x2(e2, e3);
        }
        tmem_st32(tS_row + half * 32, pk);
        // P of this half of the keys is in TMEM: the MMA warp may start its half of PV
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::B_PFULL + 2 * qt + half));
      }
      l += (l0 + l1) + (l2 + l3);
    }
    // ---------------------------------------------------------- epilogue
    if (ok && n > 0) ok = ra_wait_warp(bar(L::B_PVDONE + qt), (n - 1) & 1, abort_flag);
    n = __shfl_sync(0xffffffffu, n, 0);   // warp-uniform (lanes agree unless a wait gave up)
    tc_fence_after();
    if constexpr (STEP) {
      // Merge this block's partial (reference max m_ref in log2 units, sum l,
      // O in TMEM, both relative to 2^m_ref) into the caller's running state
      // (m in natural-log units, l, o_acc relative to e^m):
      //   m' = max(m, m_blk), o_acc' = e^(m - m') o_acc + e^(m_blk - m') O, l' likewise.
      const int64_t mi = b * p.ml_sb + h * p.ml_sh + qrow_c * p.ml_ss;
      const bool row_in = RA_IN_RANGE(qrow_c, S, kSiteFwdStepState);
      const float m_in = row_in ? p.m_state[mi] : -INFINITY, l_in = row_in ? p.l_state[mi] : 0.f;
      const float m_blk = (n > 0 && m_ref != -INFINITY) ? m_ref * kLn2 : -INFINITY;
      const float m_new = fmaxf(m_in, m_blk);
      // a block with no visible tile for this CTA leaves the state as it is
      // (the merge would be the identity), so its rows are not rewritten
      const bool write = qrow < S && ok && m_new != -INFINITY && row_in && n > 0;
      const float a_in = m_in == -INFINITY ? 0.f : expf(m_in - m_new);
      const float a_blk = m_blk == -INFINITY ? 0.f : expf(m_blk - m_new);
      float* ap = p.acc + b * p.acc_sb + qrow_c * p.acc_ss + h * p.acc_sh;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t orow[32];
        if (n > 0) {
          tmem_ld32(tO_row + c, orow);
          tmem_ld_wait();
        }
        if (write) {
          float4* a4 = reinterpret_cast<float4*>(ap + c);
#pragma unroll
          for (int v4 = 0; v4 < 8; ++v4) {
            float o4[4] = {0.f, 0.f, 0.f, 0.f};
            if (n > 0) {
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                reg_fence(orow[4 * v4 + e]);
                o4[e] = __uint_as_float(orow[4 * v4 + e]);
              }
            }
            float4 x = a4[v4];
            x.x = fmaf(a_in, x.x, a_blk * o4[0]);
            x.y = fmaf(a_in, x.y, a_blk * o4[1]);
            x.z = fmaf(a_in, x.z, a_blk * o4[2]);
            x.w = fmaf(a_in, x.w, a_blk * o4[3]);
            a4[v4] = x;
          }
        }
      }
      if (write) {
        p.m_state[mi] = m_new;
        p.l_state[mi] = fmaf(a_in, l_in, a_blk * l);
      }
    } else {
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* op = p.o + b * p.o_sb + qrow_c * p.o_ss + h * p.o_sh;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t orow[32];
        if (n > 0) {
          tmem_ld32(tO_row + c, orow);
          tmem_ld_wait();
        }
        uint32_t pkd[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float a0 = 0.f, a1 = 0.f;
          if (n > 0) {
            reg_fence(orow[e]);
            reg_fence(orow[e + 1]);
            a0 = __uint_as_float(orow[e]) * inv;
            a1 = __uint_as_float(orow[e + 1]) * inv;
          }
          pkd[e >> 1] = pack_bf16x2(a0, a1);
        }
        if (qrow < S && ok && RA_IN_RANGE(qrow, S, kSiteFwdOut)) {
          uint4* dst = reinterpret_cast<uint4*>(op + c);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            dst[v4] = make_uint4(pkd[4 * v4], pkd[4 * v4 + 1], pkd[4 * v4 + 2], pkd[4 * v4 + 3]);
        }
      }
      if (qrow < S && ok)
        p.lse[b * p.lse_sb + h * p.lse_sh + qrow * p.lse_ss] = l > 0.f ? (m_ref + log2f(l)) * kLn2 : -INFINITY;
#ifdef RA_DEBUG_COUNT
      if (qrow < S && ok && p.dbg_count) p.dbg_count[((int64_t)b * p.H + h) * S + qrow] = dbg_vis;
#endif
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
