// Problem description, ring-ordered KV-tile schedule and tile metadata,
// shared by the sm_100a kernels, the CUDA-core kernels and the host.
//
// The ring (page "Ring Attention技术解析", §2.2): the sequence of S tokens is
// cut into P contiguous blocks; virtual rank r owns query block r; at step t
// it holds the key/value block that started t ranks behind it, i.e. block
// (r - t) mod P (each rank sends its block to the next rank and receives the
// previous rank's).  On one GPU the ranks are virtual: the ring becomes the
// order in which a query tile visits key/value tiles.  `order` lets a caller
// permute the steps (the result does not depend on it).
//
// Hardware tiles are 128 tokens.  Tile t belongs to ring block
// floor(128 t / (S/P)) (the block of its first token), so the tiles of block
// `src` are [ceil(src*blk/128), ceil((src+1)*blk/128)) and every tile is
// visited exactly once.
#pragma once

#include <cstdint>

#if defined(__CUDACC__)
#define RA_HD __host__ __device__ __forceinline__
#else
#define RA_HD inline
#endif

namespace ra {

constexpr int kTile = 128;           // tokens per hardware tile
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kMaxRing = 64;         // largest supported ring size P

struct RingDesc {
  int64_t S;                 // sequence length (tokens)
  int64_t blk;               // tokens per ring block, S / P
  int32_t P;                 // ring size (virtual ranks)
  int32_t ntiles;            // ceil(S / 128)
  int32_t cbs;               // causal_block_size; 0 = non-causal
  int32_t order[kMaxRing];   // step offsets t, a permutation of 0..P-1
};

// Per 128-token tile of one batch row: x = min segment id, y = max segment
// id, z = flags (bit 0: some key has a finite bias, bit 1: every bias is 0).
// Without segment ids x = y = 0; without a bias z = 3.
enum : int32_t { kMetaAnyFinite = 1, kMetaAllZero = 2 };

RA_HD int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Index checks of the debug build (-DRA_DEBUG_COUNT, libringattn_count.so).
// Before each global or shared-memory access whose address a kernel computes
// from indices (TMA copies excepted: the tensor maps bound those), the debug
// build tests every index against its extent.  An index out of range skips the
// access and records the first such event device-wide in g_ra_bounds_hit:
// the site id (RaSite) in bits 48-63 and the index's low 48 bits below;
// ra_debug_bounds() reads and clears it.  In the release build the test is
// the constant true, and the indices are not even evaluated.
enum RaSite : int {
  kSiteFwdTileMeta = 1,   // forward: key-tile metadata (tile < ntiles)
  kSiteFwdUnit,           // forward: batch row / head of the CTA's unit (b < B, h < H)
  kSiteFwdQuerySeg,       // forward: query row's segment id (row < S)
  kSiteFwdKeyBias,        // forward: key bias (key < Sk)
  kSiteFwdKeySeg,         // forward: key segment id (key < Sk)
  kSiteFwdStepState,      // ring step: running m, l and accumulator row (row < Sq)
  kSiteFwdOut,            // forward: O row, LSE and visible-count stores (row < S)
  kSiteBwdUnit,           // backward: batch row / head / key tile of the CTA (b < B, h < H)
  kSiteBwdKeyRow,         // backward: key row's segment id, bias, dK / dV row (key < S)
  kSiteBwdQueryMeta,      // backward: query tile's metadata (tile < ntiles)
  kSiteBwdQuerySeg,       // backward: query segment ids (query < S)
  kSiteBwdDsSmem,         // backward: dS^T shared-memory stores (byte offset < buffer)
  kSiteBwdDqStaging,      // backward: dQ staging stores (byte offset < buffer)
  kSiteBwdLseDelta,       // backward: LSE / Delta rows of a query tile (row + 64 <= padded rows)
  kSiteIterMeta,          // tile iterators: key- and query-tile metadata (tile < ntiles)
  kSiteStepKeys,          // ring-step iterator: visiting keys' segment ids / bias (key < Sk)
  kSiteStepQueries,       // ring-step iterator: query segment ids (row < Sq)
  kSiteTileMeta,          // tile metadata kernel: key reads and metadata write
  kSiteBwdPre,            // backward preprocess: O, dO, LSE reads, Delta / LSE2 / dQ-accumulator writes
  kSiteDqConvert,         // dQ conversion: accumulator read, dQ write
  kSiteFinalize,          // finalize and LSE merge rows (row < B*S*H)
  kSiteFfnOut,            // feed-forward GEMMs: output tile rows and columns
};
#if defined(RA_DEBUG_COUNT) && defined(__CUDACC__)
__device__ unsigned long long g_ra_bounds_hit;
#endif
#if defined(RA_DEBUG_COUNT) && defined(__CUDA_ARCH__)
__device__ __forceinline__ bool ra_in_range(long long i, long long n, int site) {
  if (i >= 0 && i < n) return true;
  atomicCAS(&g_ra_bounds_hit, 0ull, ((unsigned long long)site << 48) | ((unsigned long long)i & 0xFFFFFFFFFFFFull));
  return false;
}
#define RA_IN_RANGE(i, n, site) ::ra::ra_in_range((long long)(i), (long long)(n), (site))
#else
#define RA_IN_RANGE(i, n, site) true
#endif

#if defined(__CUDA_ARCH__)
RA_HD int4 load_meta(const int4* p) { return __ldg(p); }
#else
RA_HD int4 load_meta(const int4* p) { return *p; }
#endif

// Last key visible to any query <= q_last under causal_block_size c
// (key j visible to query i iff floor(i/c) >= floor(j/c)).
RA_HD int64_t causal_last_key(int64_t q_last, int32_t c, int64_t S) {
  if (c <= 0) return S - 1;
  int64_t j = (q_last / c + 1) * (int64_t)c - 1;
  return j < S - 1 ? j : S - 1;
}

// Iterator over the KV tiles a query range [q_first, q_last] must visit, in
// ring order, skipping tiles that causal masking, disjoint segment ranges or
// an all -inf bias make invisible to every query of the range.
struct KvIter {
  int32_t r;          // ring block of q_first
  int32_t step;       // current ring step
  int32_t tile;       // next tile to consider within the step
  int32_t tile_end;   // end of the step's tile range
  int32_t t_cap;      // last tile not fully hidden by causal masking
  int32_t q_seg_min, q_seg_max;
  int32_t use_seg, use_bias;
  const int4* meta;   // this batch row's tile metadata, or null
  uint32_t win;       // warp iterator: visible tiles of the window at win_base not yet returned
  int32_t win_base;
};

RA_HD void kv_iter_init(KvIter& it, const RingDesc& rd, int64_t q_first, int64_t q_last, const int4* meta_b,
                        bool use_seg, bool use_bias) {
  if (q_last > rd.S - 1) q_last = rd.S - 1;
  it.r = (int32_t)(q_first / rd.blk);
  it.step = -1;
  it.tile = 0;
  it.tile_end = 0;
  it.t_cap = (int32_t)(causal_last_key(q_last, rd.cbs, rd.S) / kTile);
  it.meta = (use_seg || use_bias) ? meta_b : nullptr;
  it.use_seg = use_seg;
  it.use_bias = use_bias;
  it.win = 0;
  it.win_base = 0;
  it.q_seg_min = 0x7fffffff;
  it.q_seg_max = -0x7fffffff - 1;
  if (use_seg) {
    for (int64_t qt = q_first / kTile; qt <= q_last / kTile; ++qt) {
      if (!RA_IN_RANGE(qt, rd.ntiles, kSiteIterMeta)) break;
      int4 m = load_meta(meta_b + qt);
      it.q_seg_min = m.x < it.q_seg_min ? m.x : it.q_seg_min;
      it.q_seg_max = m.y > it.q_seg_max ? m.y : it.q_seg_max;
    }
  }
}

// Whether KV tile metadata m can hold a pair visible to the iterator's query rows.
RA_HD bool kv_tile_visible(const KvIter& it, int4 m) {
  if (it.use_seg && (m.y < it.q_seg_min || m.x > it.q_seg_max)) return false;
  if (it.use_bias && !(m.z & kMetaAnyFinite)) return false;
  return true;
}

// Move to the next ring step's tile range; false once the ring is closed.
RA_HD bool kv_iter_step(KvIter& it, const RingDesc& rd) {
  if (++it.step >= rd.P) return false;
  int32_t src = it.r - rd.order[it.step];
  src %= rd.P;
  if (src < 0) src += rd.P;
  int64_t a = (int64_t)src * rd.blk, b = (int64_t)(src + 1) * rd.blk;
  it.tile = (int32_t)ceil_div64(a, kTile);
  int64_t e = ceil_div64(b, kTile);
  if (e > it.t_cap + 1) e = it.t_cap + 1;
  it.tile_end = (int32_t)e;
  return true;
}

// Next KV tile index in ring order, or -1 when the ring is closed.
RA_HD int32_t kv_iter_next(KvIter& it, const RingDesc& rd) {
  while (true) {
    while (it.tile < it.tile_end) {
      int32_t t = it.tile++;
      if (it.meta && !kv_tile_visible(it, load_meta(it.meta + t))) continue;
      return t;
    }
    if (!kv_iter_step(it, rd)) return -1;
  }
}

#ifdef __CUDACC__
// kv_iter_next for a converged warp whose lanes all hold the same iterator:
// the lanes test 32 candidate tiles at once and the warp keeps the ballot, so
// both skipped and visible tiles cost one metadata round trip per 32 tiles
// instead of one per tile.  Returns the same sequence as kv_iter_next.
__device__ __forceinline__ int32_t kv_iter_next_warp(KvIter& it, const RingDesc& rd) {
  const int lane = threadIdx.x & 31;
  while (true) {
    if (!it.meta) {
      if (it.tile < it.tile_end) return it.tile++;
    } else {
      while (true) {
        if (it.win) {   // the window's visibility is known: no round trip
          const int32_t first = it.win_base + __ffs(it.win) - 1;
          it.win &= it.win - 1;
          return first;
        }
        if (it.tile >= it.tile_end) break;
        const int32_t t = it.tile + lane;
        const bool vis = t < it.tile_end && RA_IN_RANGE(t, rd.ntiles, kSiteIterMeta) &&
                         kv_tile_visible(it, load_meta(it.meta + t));
        it.win = __ballot_sync(0xffffffffu, vis);
        it.win_base = it.tile;
        it.tile += 32;
      }
    }
    if (!kv_iter_step(it, rd)) return -1;
  }
}
#endif

#ifdef __CUDACC__
// One ring step on its own ("Ring Attention技术解析" §2.2, one iteration of the
// loop): a query block meets one visiting key/value block of Sk tokens that
// starts at global token k_off.  StepKvIter walks that block's 128-key tiles
// in order for the query rows [q_first, q_last] (local to the query block,
// which starts at global token q_off), skipping tiles that causal masking
// (global positions), disjoint segment ids or an all -inf bias hide from
// every row.  No precomputed metadata exists for a visiting block, so a
// converged warp computes each candidate tile's segment range and bias flags
// itself (four keys per lane).  All functions must be called by every lane.
struct StepKvIter {
  int32_t tile, tile_end;
  int32_t q_seg_min, q_seg_max;
  const int32_t* seg_k;   // this batch row's key segment ids, or null
  int64_t segk_ss;
  const float* bias;      // this batch row's key bias, or null
  int64_t bias_ss;
  int64_t Sk;
};

// Metadata (as tile_meta_kernel writes it) of key tile t of the visiting block.
__device__ __forceinline__ int4 step_tile_meta_warp(const StepKvIter& it, int32_t t) {
  const int lane = threadIdx.x & 31;
  int smin = 0x7fffffff, smax = -0x7fffffff - 1;
  unsigned any = 0u, zero = 1u;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t j = (int64_t)t * kTile + lane * 4 + i;
    if (j < it.Sk && RA_IN_RANGE(j, it.Sk, kSiteStepKeys)) {
      const int s = it.seg_k ? __ldg(it.seg_k + j * it.segk_ss) : 0;
      smin = s < smin ? s : smin;
      smax = s > smax ? s : smax;
      if (it.bias) {
        const float x = __ldg(it.bias + j * it.bias_ss);
        any |= (unsigned)(x > -INFINITY);
        zero &= (unsigned)(x == 0.0f);
      } else {
        any = 1u;
      }
    }
  }
  smin = __reduce_min_sync(0xffffffffu, smin);
  smax = __reduce_max_sync(0xffffffffu, smax);
  any = __reduce_or_sync(0xffffffffu, any);
  zero = __reduce_and_sync(0xffffffffu, zero);
  return make_int4(smin, smax, (any ? kMetaAnyFinite : 0) | (zero ? kMetaAllZero : 0), 0);
}

// Segment id range of the query rows [q_first, q_last] (local, clamped to Sq).
__device__ __forceinline__ int2 step_q_seg_range_warp(const int32_t* seg_q, int64_t segq_ss, int64_t q_first,
                                                      int64_t q_last, int64_t Sq) {
  const int lane = threadIdx.x & 31;
  int smin = 0x7fffffff, smax = -0x7fffffff - 1;
  if (q_last > Sq - 1) q_last = Sq - 1;
  for (int64_t i = q_first + lane; i <= q_last; i += 32) {
    if (!RA_IN_RANGE(i, Sq, kSiteStepQueries)) break;
    const int s = __ldg(seg_q + i * segq_ss);
    smin = s < smin ? s : smin;
    smax = s > smax ? s : smax;
  }
  return make_int2(__reduce_min_sync(0xffffffffu, smin), __reduce_max_sync(0xffffffffu, smax));
}

// cbs: causal_block_size (0 = non-causal).  seg_q_b / seg_k_b: this batch
// row's segment ids (both null without segments); bias_b: its key bias or null.
__device__ __forceinline__ void step_iter_init_warp(StepKvIter& it, int64_t q_first, int64_t q_last, int64_t Sq,
                                                    int64_t Sk, int64_t q_off, int64_t k_off, int32_t cbs,
                                                    const int32_t* seg_q_b, int64_t segq_ss, const int32_t* seg_k_b,
                                                    int64_t segk_ss, const float* bias_b, int64_t bias_ss) {
  if (q_last > Sq - 1) q_last = Sq - 1;
  const int32_t ntk = (int32_t)ceil_div64(Sk, kTile);
  it.tile = 0;
  it.tile_end = ntk;
  if (cbs > 0) {
    // last visible key (global) of the last query row, in this block's local terms
    const int64_t last = ((q_off + q_last) / cbs + 1) * (int64_t)cbs - 1 - k_off;
    const int64_t e = last < 0 ? 0 : last / kTile + 1;
    if (e < it.tile_end) it.tile_end = (int32_t)e;
  }
  it.seg_k = seg_k_b;
  it.segk_ss = segk_ss;
  it.bias = bias_b;
  it.bias_ss = bias_ss;
  it.Sk = Sk;
  it.q_seg_min = 0;
  it.q_seg_max = 0;
  if (seg_k_b) {
    const int2 r = step_q_seg_range_warp(seg_q_b, segq_ss, q_first, q_last, Sq);
    it.q_seg_min = r.x;
    it.q_seg_max = r.y;
  }
}

// Next visible key tile (local index) and its metadata, or -1 at the end of the block.
__device__ __forceinline__ int32_t step_iter_next_warp(StepKvIter& it, int4& km) {
  while (it.tile < it.tile_end) {
    const int32_t t = it.tile++;
    if (!it.seg_k && !it.bias) {
      km = make_int4(0, 0, kMetaAnyFinite | kMetaAllZero, 0);
      return t;
    }
    km = step_tile_meta_warp(it, t);
    const bool seg_ok = !it.seg_k || !(km.y < it.q_seg_min || km.x > it.q_seg_max);
    const bool bias_ok = !it.bias || (km.z & kMetaAnyFinite);
    if (seg_ok && bias_ok) return t;
  }
  return -1;
}
#endif

// Backward direction of the same ring: a key/value tile of ring block src
// meets the query blocks (src + order[t]) mod P at steps t = 0, 1, ...
// (rank r holds block (r - order[t]) mod P at step t).  QIter walks the
// 64-row query tiles a key tile [k_first, k_last] must visit in that order,
// skipping tiles hidden from it by causal masking or disjoint segments.
constexpr int kQTileBwd = 64;

struct QIter {
  int32_t src;        // ring block of the key tile
  int32_t step;
  int32_t tile, tile_end;
  int32_t q_min;      // first query tile not fully hidden by causal masking
  int32_t nqt;        // number of 64-row query tiles
  int32_t k_seg_min, k_seg_max;
  int32_t use_seg;
  const int4* meta;   // 128-token tile metadata of this batch row, or null
  uint32_t win;       // warp iterator: visible tiles of the window at win_base not yet returned
  int32_t win_base;
};

RA_HD void q_iter_init(QIter& it, const RingDesc& rd, int64_t k_first, const int4* meta_b, bool use_seg) {
  it.src = (int32_t)(k_first / rd.blk);
  it.step = -1;
  it.tile = it.tile_end = 0;
  it.nqt = (int32_t)ceil_div64(rd.S, kQTileBwd);
  const int64_t i_min = rd.cbs > 0 ? (k_first / rd.cbs) * (int64_t)rd.cbs : 0;   // first query that can see k_first's block
  it.q_min = (int32_t)(i_min / kQTileBwd);
  it.use_seg = use_seg;
  it.meta = use_seg ? meta_b : nullptr;
  it.win = 0;
  it.win_base = 0;
  it.k_seg_min = 0;
  it.k_seg_max = 0;
  if (use_seg && RA_IN_RANGE(k_first / kTile, rd.ntiles, kSiteIterMeta)) {
    int4 m = load_meta(meta_b + k_first / kTile);
    it.k_seg_min = m.x;
    it.k_seg_max = m.y;
  }
}

RA_HD bool q_tile_visible(const QIter& it, int32_t q) {
  if (!RA_IN_RANGE(q, it.nqt, kSiteIterMeta)) return false;
  const int4 m = load_meta(it.meta + (int64_t)q * kQTileBwd / kTile);
  return !(m.y < it.k_seg_min || m.x > it.k_seg_max);
}

RA_HD bool q_iter_step(QIter& it, const RingDesc& rd) {
  if (++it.step >= rd.P) return false;
  int32_t r = (it.src + rd.order[it.step]) % rd.P;
  int64_t a = (int64_t)r * rd.blk, b = (int64_t)(r + 1) * rd.blk;
  int64_t lo = ceil_div64(a, kQTileBwd), hi = ceil_div64(b, kQTileBwd);
  if (hi > it.nqt) hi = it.nqt;
  if (lo < it.q_min) lo = it.q_min;
  it.tile = (int32_t)lo;
  it.tile_end = (int32_t)(hi > lo ? hi : lo);
  return true;
}

RA_HD int32_t q_iter_next(QIter& it, const RingDesc& rd) {
  while (true) {
    while (it.tile < it.tile_end) {
      int32_t q = it.tile++;
      if (it.meta && !q_tile_visible(it, q)) continue;
      return q;
    }
    if (!q_iter_step(it, rd)) return -1;
  }
}

#ifdef __CUDACC__
// q_iter_next for a converged warp (same contract as kv_iter_next_warp).
__device__ __forceinline__ int32_t q_iter_next_warp(QIter& it, const RingDesc& rd) {
  const int lane = threadIdx.x & 31;
  while (true) {
    if (!it.meta) {
      if (it.tile < it.tile_end) return it.tile++;
    } else {
      while (true) {
        if (it.win) {
          const int32_t first = it.win_base + __ffs(it.win) - 1;
          it.win &= it.win - 1;
          return first;
        }
        if (it.tile >= it.tile_end) break;
        const int32_t q = it.tile + lane;
        const bool vis = q < it.tile_end && q_tile_visible(it, q);
        it.win = __ballot_sync(0xffffffffu, vis);
        it.win_base = it.tile;
        it.tile += 32;
      }
    }
    if (!q_iter_step(it, rd)) return -1;
  }
}
#endif

// Whether a (query tile, KV tile) pair needs the per-element mask: a causal
// diagonal, a partly-out-of-range KV tile, or mixed segment ids.
RA_HD bool tile_needs_mask(const RingDesc& rd, int64_t q_first, int32_t t, bool use_seg, int4 qm, int4 km) {
  int64_t k_first = (int64_t)t * kTile;
  int64_t k_last = k_first + kTile - 1;
  if (k_last > rd.S - 1) return true;
  if (rd.cbs > 0 && (q_first / rd.cbs) < (k_last / rd.cbs)) return true;
  if (use_seg && !(qm.x == qm.y && km.x == km.y && qm.x == km.x)) return true;
  return false;
}

}  // namespace ra
