// CUDA-core kernels (fp32 arithmetic): tile metadata, the fp32 forward, the
// single ring step, finalize, log-sum-exp merge, the backward preprocess and
// a direct fp32 backward for fp32 inputs.
//
// Online softmax (the exact merge behind "全局注意力 完整保留" in page
// "手把手拆解RingAttention" §1): per query row keep a running max m, a running
// sum l and an unnormalised output acc; a new key tile with scores s updates
//   m' = max(m, max s),  acc = e^(m-m') acc + sum_j e^(s_j-m') v_j,
//   l  = e^(m-m') l + sum_j e^(s_j-m').
// Here m and s are in natural-log units and the exponentials are expf.
#pragma once

#include <cuda_bf16.h>
#include <math_constants.h>

#include "ptx.cuh"
#include "ra_common.cuh"

namespace ra {

__device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

struct MaskArgs {
  const int32_t* seg;   // [B, S] segment ids or null
  int64_t seg_sb, seg_ss;
  const float* bias;    // [B, S] additive key bias or null
  int64_t bias_sb, bias_ss;
};

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// ---------------------------------------------------------------- tile metadata

// grid (ntiles, B), block 128: one thread per token of the tile.
__global__ void __launch_bounds__(128) tile_meta_kernel(MaskArgs mk, int64_t S, int32_t ntiles, int4* meta) {
  const int t = blockIdx.x, b = blockIdx.y;
  const int64_t j = (int64_t)t * kTile + threadIdx.x;
  const bool valid = j < S;
  int smin = 0x7fffffff, smax = -0x7fffffff - 1;
  int any_finite = 0, all_zero = 1;
  if (valid) {
    if (mk.seg) {
      int s = mk.seg[b * mk.seg_sb + j * mk.seg_ss];
      smin = smax = s;
    } else {
      smin = smax = 0;
    }
    if (mk.bias) {
      float x = mk.bias[b * mk.bias_sb + j * mk.bias_ss];
      any_finite = x > -CUDART_INF_F;
      all_zero = x == 0.0f;
    } else {
      any_finite = 1;
    }
  }
  __shared__ int red[4][4];
  for (int o = 16; o > 0; o >>= 1) {
    smin = min(smin, __shfl_xor_sync(0xffffffffu, smin, o));
    smax = max(smax, __shfl_xor_sync(0xffffffffu, smax, o));
    any_finite |= __shfl_xor_sync(0xffffffffu, any_finite, o);
    all_zero &= __shfl_xor_sync(0xffffffffu, all_zero, o);
  }
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    red[w][0] = smin; red[w][1] = smax; red[w][2] = any_finite; red[w][3] = all_zero;
  }
  __syncthreads();
  if (threadIdx.x == 0 && RA_IN_RANGE(t, ntiles, kSiteTileMeta)) {
    for (int i = 1; i < 4; ++i) {
      red[0][0] = min(red[0][0], red[i][0]);
      red[0][1] = max(red[0][1], red[i][1]);
      red[0][2] |= red[i][2];
      red[0][3] &= red[i][3];
    }
    meta[(int64_t)b * ntiles + t] =
        make_int4(red[0][0], red[0][1], (red[0][2] ? kMetaAnyFinite : 0) | (red[0][3] ? kMetaAllZero : 0), 0);
  }
}

// ---------------------------------------------------------------- forward / step (SIMT)

// Tensor view: element strides of a [B, S, H, D] tensor.
struct View4 {
  const void* p;
  int64_t sb, ss, sh;
};
struct OutView4 {
  void* p;
  int64_t sb, ss, sh;
};

constexpr int kSimtRows = 64;   // query rows per block (one thread each)
constexpr int kSimtKeys = 64;   // keys staged per pass

template <int D>
struct SimtSmem {
  static constexpr int QS = D + 1;   // padded row stride (floats) against bank conflicts
  static constexpr int BYTES = (kSimtRows * QS + 2 * kSimtKeys * D) * 4;
};

// One pass of the online softmax over up to kSimtKeys keys held in shared
// memory.  `kpos0` is the global position of key 0; invisible keys are
// skipped through `vis`.
template <int D>
__device__ __forceinline__ void simt_update(const float* qrow, const float* ks, const float* vs, int nk,
                                            const bool* vis, const float* kbias, float scale, float& m, float& l,
                                            float* acc) {
  float s[kSimtKeys];
  float mx = -CUDART_INF_F;
#pragma unroll 4
  for (int j = 0; j < kSimtKeys; ++j) {
    float d = 0.f;
    if (j < nk && vis[j]) {
#pragma unroll 16
      for (int e = 0; e < D; ++e) d = fmaf(qrow[e], ks[j * D + e], d);
      d = d * scale + kbias[j];
    } else {
      d = -CUDART_INF_F;
    }
    s[j] = d;
    mx = fmaxf(mx, d);
  }
  const float m_new = fmaxf(m, mx);
  if (m_new == -CUDART_INF_F) return;               // nothing visible yet
  const float alpha = (m == -CUDART_INF_F) ? 0.f : expf(m - m_new);
  l *= alpha;
#pragma unroll
  for (int e = 0; e < D; ++e) acc[e] *= alpha;
  for (int j = 0; j < kSimtKeys; ++j) {
    if (s[j] == -CUDART_INF_F) continue;
    const float pj = expf(s[j] - m_new);
    l += pj;
#pragma unroll
    for (int e = 0; e < D; ++e) acc[e] = fmaf(pj, vs[j * D + e], acc[e]);
  }
  m = m_new;
}

// Stage keys [k0, k0+n) of (b, h) into shared memory as fp32.
template <int D, typename T>
__device__ __forceinline__ void simt_stage_kv(const View4& K, const View4& V, int b, int h, int64_t k0, int n,
                                              float* ks, float* vs) {
  const T* kp = static_cast<const T*>(K.p);
  const T* vp = static_cast<const T*>(V.p);
  for (int idx = threadIdx.x; idx < kSimtKeys * D; idx += blockDim.x) {
    const int j = idx / D, e = idx % D;
    float kv = 0.f, vv = 0.f;
    if (j < n) {
      kv = to_f<T>(kp[b * K.sb + (k0 + j) * K.ss + h * K.sh + e]);
      vv = to_f<T>(vp[b * V.sb + (k0 + j) * V.ss + h * V.sh + e]);
    }
    ks[idx] = kv;
    vs[idx] = vv;
  }
}

struct SimtFwdArgs {
  RingDesc rd;
  int B, H;
  float scale;
  MaskArgs mk;
  const int4* meta;
  View4 q, k, v;
  OutView4 o;
  float* lse;           // [B, H, S]
  int64_t lse_sb, lse_sh, lse_ss;
};

// Full forward on CUDA cores: grid (ceil(S/64), B*H), block 64.  Each query
// tile visits the KV tiles in ring order (KvIter) and runs the online
// softmax; the finalize divides by l and writes O and the natural-log LSE.
template <int D, typename T>
__global__ void __launch_bounds__(kSimtRows) simt_fwd_kernel(const SimtFwdArgs a) {
  extern __shared__ float sm[];
  float* qs = sm;
  float* ks = qs + kSimtRows * SimtSmem<D>::QS;
  float* vs = ks + kSimtKeys * D;
  const int b = blockIdx.y / a.H, h = blockIdx.y % a.H;
  const int64_t q0 = (int64_t)blockIdx.x * kSimtRows;
  const int64_t S = a.rd.S;
  const int64_t qi = q0 + threadIdx.x;
  const T* qp = static_cast<const T*>(a.q.p);
  for (int idx = threadIdx.x; idx < kSimtRows * D; idx += blockDim.x) {
    const int r = idx / D, e = idx % D;
    const int64_t i = q0 + r;
    qs[r * SimtSmem<D>::QS + e] = i < S ? to_f<T>(qp[b * a.q.sb + i * a.q.ss + h * a.q.sh + e]) : 0.f;
  }
  const int my_seg = (a.mk.seg && qi < S) ? a.mk.seg[b * a.mk.seg_sb + qi * a.mk.seg_ss] : 0;
  float acc[D];
#pragma unroll
  for (int e = 0; e < D; ++e) acc[e] = 0.f;
  float m = -CUDART_INF_F, l = 0.f;
  KvIter it;
  const int4* meta_b = a.meta ? a.meta + (int64_t)b * a.rd.ntiles : nullptr;
  kv_iter_init(it, a.rd, q0, q0 + kSimtRows - 1, meta_b, a.mk.seg != nullptr, a.mk.bias != nullptr);
  __syncthreads();
  for (int32_t t = kv_iter_next(it, a.rd); t >= 0; t = kv_iter_next(it, a.rd)) {
    for (int half = 0; half < kTile / kSimtKeys; ++half) {
      const int64_t k0 = (int64_t)t * kTile + half * kSimtKeys;
      if (k0 >= S) break;
      const int n = (int)min64(kSimtKeys, S - k0);
      __syncthreads();
      simt_stage_kv<D, T>(a.k, a.v, b, h, k0, n, ks, vs);
      __syncthreads();
      bool vis[kSimtKeys];
      float kb[kSimtKeys];
      for (int j = 0; j < kSimtKeys; ++j) {
        const int64_t kj = k0 + j;
        bool ok = j < n && qi < S;
        if (ok && a.rd.cbs > 0) ok = (qi / a.rd.cbs) >= (kj / a.rd.cbs);
        if (ok && a.mk.seg) ok = a.mk.seg[b * a.mk.seg_sb + kj * a.mk.seg_ss] == my_seg;
        float bj = 0.f;
        if (ok && a.mk.bias) {
          bj = a.mk.bias[b * a.mk.bias_sb + kj * a.mk.bias_ss];
          ok = bj > -CUDART_INF_F;
        }
        vis[j] = ok;
        kb[j] = ok ? bj : 0.f;
      }
      simt_update<D>(qs + threadIdx.x * SimtSmem<D>::QS, ks, vs, n, vis, kb, a.scale, m, l, acc);
    }
  }
  if (qi < S) {
    T* op = static_cast<T*>(a.o.p) + b * a.o.sb + qi * a.o.ss + h * a.o.sh;
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int e = 0; e < D; ++e) op[e] = from_f<T>(acc[e] * inv);
    a.lse[b * a.lse_sb + h * a.lse_sh + qi * a.lse_ss] = l > 0.f ? m + logf(l) : -CUDART_INF_F;
  }
}

struct SimtStepArgs {
  int B, H, D;
  int64_t Sq, Sk, q_off, k_off;
  int32_t cbs;
  float scale;
  View4 q, k, v;
  const int32_t* seg_q; int64_t segq_sb, segq_ss;
  const int32_t* seg_k; int64_t segk_sb, segk_ss;
  const float* bias; int64_t bias_sb, bias_ss;
  float* acc; int64_t acc_sb, acc_ss, acc_sh;     // [B, Sq, H, D] fp32, unnormalised
  float* m; float* l; int64_t ml_sb, ml_sh, ml_ss; // [B, H, Sq] fp32 (natural-log units)
};

// One ring step: the query block (global offset q_off) against one visiting
// key/value block (global offset k_off), updating the caller's running
// (acc, m, l).  grid (ceil(Sq/64), B*H), block 64.
template <int D, typename T>
__global__ void __launch_bounds__(kSimtRows) simt_step_kernel(const SimtStepArgs a) {
  extern __shared__ float sm[];
  float* qs = sm;
  float* ks = qs + kSimtRows * SimtSmem<D>::QS;
  float* vs = ks + kSimtKeys * D;
  const int b = blockIdx.y / a.H, h = blockIdx.y % a.H;
  const int64_t r0 = (int64_t)blockIdx.x * kSimtRows;
  const int64_t r = r0 + threadIdx.x;
  const T* qp = static_cast<const T*>(a.q.p);
  for (int idx = threadIdx.x; idx < kSimtRows * D; idx += blockDim.x) {
    const int rr = idx / D, e = idx % D;
    const int64_t i = r0 + rr;
    qs[rr * SimtSmem<D>::QS + e] = i < a.Sq ? to_f<T>(qp[b * a.q.sb + i * a.q.ss + h * a.q.sh + e]) : 0.f;
  }
  float acc[D];
  float m = -CUDART_INF_F, l = 0.f;
  const int64_t mi = b * a.ml_sb + h * a.ml_sh + r * a.ml_ss;
  float* accp = a.acc + b * a.acc_sb + r * a.acc_ss + h * a.acc_sh;
  if (r < a.Sq) {
    m = a.m[mi];
    l = a.l[mi];
#pragma unroll
    for (int e = 0; e < D; ++e) acc[e] = accp[e];
  } else {
#pragma unroll
    for (int e = 0; e < D; ++e) acc[e] = 0.f;
  }
  const int my_seg = (a.seg_q && r < a.Sq) ? a.seg_q[b * a.segq_sb + r * a.segq_ss] : 0;
  const int64_t qpos = a.q_off + r;
  for (int64_t k0 = 0; k0 < a.Sk; k0 += kSimtKeys) {
    const int n = (int)min64(kSimtKeys, a.Sk - k0);
    __syncthreads();
    simt_stage_kv<D, T>(a.k, a.v, b, h, k0, n, ks, vs);
    __syncthreads();
    bool vis[kSimtKeys];
    float kb[kSimtKeys];
    for (int j = 0; j < kSimtKeys; ++j) {
      const int64_t kj = k0 + j;
      const int64_t kpos = a.k_off + kj;
      bool ok = j < n && r < a.Sq;
      if (ok && a.cbs > 0) ok = (qpos / a.cbs) >= (kpos / a.cbs);
      if (ok && a.seg_q) ok = a.seg_k[b * a.segk_sb + kj * a.segk_ss] == my_seg;
      float bj = 0.f;
      if (ok && a.bias) {
        bj = a.bias[b * a.bias_sb + kj * a.bias_ss];
        ok = bj > -CUDART_INF_F;
      }
      vis[j] = ok;
      kb[j] = ok ? bj : 0.f;
    }
    simt_update<D>(qs + threadIdx.x * SimtSmem<D>::QS, ks, vs, n, vis, kb, a.scale, m, l, acc);
  }
  if (r < a.Sq) {
    a.m[mi] = m;
    a.l[mi] = l;
#pragma unroll
    for (int e = 0; e < D; ++e) accp[e] = acc[e];
  }
}

// ---------------------------------------------------------------- finalize / merge

struct FinalizeArgs {
  int B, S, H, D;
  const float* acc; int64_t acc_sb, acc_ss, acc_sh;
  const float* m; const float* l; int64_t ml_sb, ml_sh, ml_ss;
  void* o; int64_t o_sb, o_ss, o_sh; int o_bf16;
  float* lse; int64_t lse_sb, lse_sh, lse_ss;
};

// o = acc / l, lse = m + log l (rows with l == 0: o = 0, lse = -inf).
// One thread per (b, i, h) row.
__global__ void finalize_kernel(const FinalizeArgs a) {
  const int64_t row = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t n = (int64_t)a.B * a.S * a.H;
  if (row >= n) return;
  const int h = (int)(row % a.H);
  const int64_t i = (row / a.H) % a.S;
  const int b = (int)(row / ((int64_t)a.H * a.S));
  if (!RA_IN_RANGE(b, a.B, kSiteFinalize)) return;
  const int64_t mi = b * a.ml_sb + h * a.ml_sh + i * a.ml_ss;
  const float l = a.l[mi];
  const float inv = l > 0.f ? 1.f / l : 0.f;
  const float* accp = a.acc + b * a.acc_sb + i * a.acc_ss + h * a.acc_sh;
  const int64_t oo = b * a.o_sb + i * a.o_ss + h * a.o_sh;
  for (int e = 0; e < a.D; ++e) {
    const float x = accp[e] * inv;
    if (a.o_bf16) static_cast<__nv_bfloat16*>(a.o)[oo + e] = __float2bfloat16_rn(x);
    else static_cast<float*>(a.o)[oo + e] = x;
  }
  a.lse[b * a.lse_sb + h * a.lse_sh + i * a.lse_ss] = l > 0.f ? a.m[mi] + logf(l) : -CUDART_INF_F;
}

struct MergeArgs {
  int B, S, H, D;
  const void* oa; int64_t oa_sb, oa_ss, oa_sh;
  const float* la; int64_t la_sb, la_sh, la_ss;
  const void* ob; int64_t ob_sb, ob_ss, ob_sh;
  const float* lb; int64_t lb_sb, lb_sh, lb_ss;
  void* oo; int64_t oo_sb, oo_ss, oo_sh;
  float* lo; int64_t lo_sb, lo_sh, lo_ss;
  int bf16;   // o tensors are bf16 (else fp32)
};

// Merge of two normalised partials over disjoint key sets:
// lse = max + log1p(exp(-|lse_a - lse_b|)), o = o_a e^(lse_a-lse) + o_b e^(lse_b-lse).
// Outputs may alias input a.
__global__ void lse_merge_kernel(const MergeArgs a) {
  const int64_t row = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t n = (int64_t)a.B * a.S * a.H;
  if (row >= n) return;
  const int h = (int)(row % a.H);
  const int64_t i = (row / a.H) % a.S;
  const int b = (int)(row / ((int64_t)a.H * a.S));
  if (!RA_IN_RANGE(b, a.B, kSiteFinalize)) return;
  const float xa = a.la[b * a.la_sb + h * a.la_sh + i * a.la_ss];
  const float xb = a.lb[b * a.lb_sb + h * a.lb_sh + i * a.lb_ss];
  const float hi = fmaxf(xa, xb), lo = fminf(xa, xb);
  float lse, wa, wb;
  if (hi == -CUDART_INF_F) {
    lse = -CUDART_INF_F; wa = 0.f; wb = 0.f;
  } else {
    lse = hi + log1pf(expf(lo - hi));
    wa = xa == -CUDART_INF_F ? 0.f : expf(xa - lse);
    wb = xb == -CUDART_INF_F ? 0.f : expf(xb - lse);
  }
  const int64_t ia = b * a.oa_sb + i * a.oa_ss + h * a.oa_sh;
  const int64_t ib = b * a.ob_sb + i * a.ob_ss + h * a.ob_sh;
  const int64_t io = b * a.oo_sb + i * a.oo_ss + h * a.oo_sh;
  for (int e = 0; e < a.D; ++e) {
    float va, vb;
    if (a.bf16) {
      va = __bfloat162float(static_cast<const __nv_bfloat16*>(a.oa)[ia + e]);
      vb = __bfloat162float(static_cast<const __nv_bfloat16*>(a.ob)[ib + e]);
    } else {
      va = static_cast<const float*>(a.oa)[ia + e];
      vb = static_cast<const float*>(a.ob)[ib + e];
    }
    const float x = wa * va + wb * vb;
    if (a.bf16) static_cast<__nv_bfloat16*>(a.oo)[io + e] = __float2bfloat16_rn(x);
    else static_cast<float*>(a.oo)[io + e] = x;
  }
  a.lo[b * a.lo_sb + h * a.lo_sh + i * a.lo_ss] = lse;
}

// ---------------------------------------------------------------- failure-path self-test

// One warp waits, through the same bounded wait the attention kernels use, on
// an mbarrier phase that nothing ever completes.  The wait must give up after
// `budget` cycles, record RA_ERR_DEVICE_TIMEOUT in the status word, raise the
// block's abort flag (checked by the remaining lanes) and return.
__global__ void selftest_timeout_kernel(long long budget, int* gave_up) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const bool ok = ra_wait_budget(smem_u32(&bar), 0, &abort_flag, budget);
  if (threadIdx.x == 0) *gave_up = ok ? 0 : 1;
}

// ---------------------------------------------------------------- backward

struct BwdPreArgs {
  int B, S, H, D;
  const void* o; int64_t o_sb, o_ss, o_sh;
  const void* dO; int64_t do_sb, do_ss, do_sh;
  const float* lse; int64_t lse_sb, lse_sh, lse_ss;
  int bf16;
  int64_t s_pad;
  float* delta;          // [B*H][s_pad]
  float* lse2;           // [B*H][s_pad]
  float* dqacc;          // [B*H][S][D] or null
};

// Backward preprocess, one warp per (b, h, i) row of the padded [B*H][s_pad]
// layout, written negated for the backward kernels' fused multiply-adds:
// delta = -<dO_i, O_i> (fp32) and lse2 = -lse_i * log2(e) (-inf for a row
// with no visible key, so its probabilities come out as 0); the row of the
// fp32 dQ accumulator is set to zero.  Padding rows get delta = 0 and
// lse2 = -inf.
__global__ void bwd_pre_kernel(const BwdPreArgs a) {
  const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t n = (int64_t)a.B * a.H * a.s_pad;
  if (row >= n) return;
  const int64_t i = row % a.s_pad;
  const int64_t bh = row / a.s_pad;
  const int h = (int)(bh % a.H), b = (int)(bh / a.H);
  if (i >= a.S) {
    if (lane == 0) {
      a.delta[row] = 0.f;
      a.lse2[row] = -CUDART_INF_F;
    }
    return;
  }
  float s = 0.f;
  const int64_t io = b * a.o_sb + i * a.o_ss + h * a.o_sh;
  const int64_t id = b * a.do_sb + i * a.do_ss + h * a.do_sh;
  for (int e = lane; e < a.D; e += 32) {
    if (a.bf16) {
      s += __bfloat162float(static_cast<const __nv_bfloat16*>(a.o)[io + e]) *
           __bfloat162float(static_cast<const __nv_bfloat16*>(a.dO)[id + e]);
    } else {
      s += static_cast<const float*>(a.o)[io + e] * static_cast<const float*>(a.dO)[id + e];
    }
    if (a.dqacc && RA_IN_RANGE(bh, (int64_t)a.B * a.H, kSiteBwdPre)) a.dqacc[(bh * a.S + i) * a.D + e] = 0.f;
  }
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) {
    a.delta[row] = -s;
    const float l = a.lse[b * a.lse_sb + h * a.lse_sh + i * a.lse_ss];
    a.lse2[row] = l == -CUDART_INF_F ? -CUDART_INF_F : -l * 1.4426950408889634f;
  }
}

struct DqConvertArgs {
  int B, S, H, D;
  const float* dqacc;    // [B*H][S][D]
  void* dq; int64_t dq_sb, dq_ss, dq_sh;
  int bf16;
};

// dQ accumulator (fp32, [B*H][S][D]) -> dq [B, S, H, D] in bf16 or fp32.
__global__ void dq_convert_kernel(const DqConvertArgs a) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t n = (int64_t)a.B * a.S * a.H * a.D;
  if (idx >= n) return;
  const int e = (int)(idx % a.D);
  const int64_t i = (idx / a.D) % a.S;
  const int64_t bh = idx / ((int64_t)a.D * a.S);
  const int h = (int)(bh % a.H), b = (int)(bh / a.H);
  if (!RA_IN_RANGE(b, a.B, kSiteDqConvert)) return;
  const float x = a.dqacc[idx];
  const int64_t o = b * a.dq_sb + i * a.dq_ss + h * a.dq_sh + e;
  if (a.bf16) static_cast<__nv_bfloat16*>(a.dq)[o] = __float2bfloat16_rn(x);
  else static_cast<float*>(a.dq)[o] = x;
}

struct SimtBwdArgs {
  RingDesc rd;
  int B, H;
  float scale;
  MaskArgs mk;
  View4 q, k, v, dO;
  const float* lse; int64_t lse_sb, lse_sh, lse_ss;
  const float* delta;    // [B*H][s_pad], negated: -<dO_i, O_i>
  int64_t s_pad;
  OutView4 dq, dk, dv;
  int out_bf16;          // gradient element type: 1 bf16, 0 fp32
};

__device__ __forceinline__ bool simt_visible(const SimtBwdArgs& a, int b, int64_t i, int64_t j, float& bias_j) {
  bias_j = 0.f;
  if (a.rd.cbs > 0 && (i / a.rd.cbs) < (j / a.rd.cbs)) return false;
  if (a.mk.seg && a.mk.seg[b * a.mk.seg_sb + i * a.mk.seg_ss] != a.mk.seg[b * a.mk.seg_sb + j * a.mk.seg_ss])
    return false;
  if (a.mk.bias) {
    bias_j = a.mk.bias[b * a.mk.bias_sb + j * a.mk.bias_ss];
    if (!(bias_j > -CUDART_INF_F)) return false;
  }
  return true;
}

__device__ __forceinline__ void simt_store_row(const OutView4& o, int b, int64_t i, int h, const float* x, int D,
                                               int bf16) {
  const int64_t off = b * o.sb + i * o.ss + h * o.sh;
  for (int e = 0; e < D; ++e) {
    if (bf16) static_cast<__nv_bfloat16*>(o.p)[off + e] = __float2bfloat16_rn(x[e]);
    else static_cast<float*>(o.p)[off + e] = x[e];
  }
}

// dQ on CUDA cores: one thread per query row, keys visited in ring order.
// grid (ceil(S/64), B*H), block 64.
template <int D, typename T>
__global__ void __launch_bounds__(64) simt_bwd_dq_kernel(const SimtBwdArgs a) {
  const int b = blockIdx.y / a.H, h = blockIdx.y % a.H;
  const int64_t i = (int64_t)blockIdx.x * 64 + threadIdx.x;
  if (i >= a.rd.S) return;
  const T* q = static_cast<const T*>(a.q.p) + b * a.q.sb + i * a.q.ss + h * a.q.sh;
  const T* dO = static_cast<const T*>(a.dO.p) + b * a.dO.sb + i * a.dO.ss + h * a.dO.sh;
  const float lse = a.lse[b * a.lse_sb + h * a.lse_sh + i * a.lse_ss];
  const float dl = -a.delta[(int64_t)blockIdx.y * a.s_pad + i];
  float acc[D];
#pragma unroll
  for (int e = 0; e < D; ++e) acc[e] = 0.f;
  if (lse > -CUDART_INF_F) {
    KvIter it;
    kv_iter_init(it, a.rd, i, i, nullptr, false, false);
    for (int32_t t = kv_iter_next(it, a.rd); t >= 0; t = kv_iter_next(it, a.rd)) {
      for (int64_t j = (int64_t)t * kTile; j < min64(a.rd.S, (int64_t)t * kTile + kTile); ++j) {
        float bj;
        if (!simt_visible(a, b, i, j, bj)) continue;
        const T* k = static_cast<const T*>(a.k.p) + b * a.k.sb + j * a.k.ss + h * a.k.sh;
        const T* v = static_cast<const T*>(a.v.p) + b * a.v.sb + j * a.v.ss + h * a.v.sh;
        float s = 0.f, dp = 0.f;
        for (int e = 0; e < D; ++e) {
          s = fmaf(to_f<T>(q[e]), to_f<T>(k[e]), s);
          dp = fmaf(to_f<T>(dO[e]), to_f<T>(v[e]), dp);
        }
        const float p = expf(s * a.scale + bj - lse);
        const float ds = p * (dp - dl) * a.scale;
#pragma unroll
        for (int e = 0; e < D; ++e) acc[e] = fmaf(ds, to_f<T>(k[e]), acc[e]);
      }
    }
  }
  simt_store_row(a.dq, b, i, h, acc, D, a.out_bf16);
}

// dK, dV on CUDA cores: one thread per key row, all query rows visited.
template <int D, typename T>
__global__ void __launch_bounds__(64) simt_bwd_dkdv_kernel(const SimtBwdArgs a) {
  const int b = blockIdx.y / a.H, h = blockIdx.y % a.H;
  const int64_t j = (int64_t)blockIdx.x * 64 + threadIdx.x;
  if (j >= a.rd.S) return;
  const T* k = static_cast<const T*>(a.k.p) + b * a.k.sb + j * a.k.ss + h * a.k.sh;
  const T* v = static_cast<const T*>(a.v.p) + b * a.v.sb + j * a.v.ss + h * a.v.sh;
  float dk[D], dv[D];
#pragma unroll
  for (int e = 0; e < D; ++e) { dk[e] = 0.f; dv[e] = 0.f; }
  for (int64_t i = 0; i < a.rd.S; ++i) {
    float bj;
    if (!simt_visible(a, b, i, j, bj)) continue;
    const float lse = a.lse[b * a.lse_sb + h * a.lse_sh + i * a.lse_ss];
    if (!(lse > -CUDART_INF_F)) continue;
    const T* q = static_cast<const T*>(a.q.p) + b * a.q.sb + i * a.q.ss + h * a.q.sh;
    const T* dO = static_cast<const T*>(a.dO.p) + b * a.dO.sb + i * a.dO.ss + h * a.dO.sh;
    float s = 0.f, dp = 0.f;
    for (int e = 0; e < D; ++e) {
      s = fmaf(to_f<T>(q[e]), to_f<T>(k[e]), s);
      dp = fmaf(to_f<T>(dO[e]), to_f<T>(v[e]), dp);
    }
    const float p = expf(s * a.scale + bj - lse);
    const float ds = p * (dp + a.delta[(int64_t)blockIdx.y * a.s_pad + i]) * a.scale;
#pragma unroll
    for (int e = 0; e < D; ++e) {
      dv[e] = fmaf(p, to_f<T>(dO[e]), dv[e]);
      dk[e] = fmaf(ds, to_f<T>(q[e]), dk[e]);
    }
  }
  simt_store_row(a.dk, b, j, h, dk, D, a.out_bf16);
  simt_store_row(a.dv, b, j, h, dv, D, a.out_bf16);
}

}  // namespace ra
