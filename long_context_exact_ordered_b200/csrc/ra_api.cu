// C ABI of the library (declared in include/ringattn.h): argument checks,
// workspace layout, TMA tensor maps, kernel launches, and the host-only
// schedule / visible-pair introspection.  Single translation unit: every
// kernel header is included here.
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>   // header-only; a no-op unless a profiler injects itself

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <unordered_map>
#include <vector>

#include "../../include/ringattn.h"
#include "ra_common.cuh"
#include "ra_fwd_sm100.cuh"
#include "ra_bwd_sm100.cuh"
#include "ra_ffn_sm100.cuh"
#include "ra_simt.cuh"

using namespace ra;

// Fixed scratch for ra_forward_static (tile metadata), one copy per device.
// Host code must not pass this symbol to a kernel directly: on the host it is
// only a stand-in, so its device address is looked up with
// cudaGetSymbolAddress in the current context, on every call.
static __device__ __align__(256) unsigned char g_ra_static_scratch[RA_STATIC_SCRATCH_BYTES];
// Written only by the failure-path self-test kernel (1 = its wait gave up).
static __device__ int g_ra_selftest_result;

#ifdef RA_DEBUG_COUNT
#include "../../include/ringattn_debug.h"
// Count buffers of the debug build (set by ra_debug_set_counts; null = off).
static int32_t* g_dbg_fwd_rows = nullptr;
static int32_t* g_dbg_bwd_cols = nullptr;
#endif

namespace {

// ---------------------------------------------------------------- CUDA failures

// What stood behind the last RA_ERR_CUDA returned to this thread (read by
// ra_last_error_message).
thread_local char t_last_error[192] = "";

int cuda_fail(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return RA_OK;
  std::snprintf(t_last_error, sizeof(t_last_error), "%s: %s (%s, %d)", what, cudaGetErrorString(e),
                cudaGetErrorName(e), (int)e);
  return RA_ERR_CUDA;
}

int cu_fail(CUresult r, const char* what) {
  if (r == CUDA_SUCCESS) return RA_OK;
  std::snprintf(t_last_error, sizeof(t_last_error), "%s: CUresult %d", what, (int)r);
  return RA_ERR_CUDA;
}

// ---------------------------------------------------------------- validation

bool is_dtype(const ra_tensor* t, int dt) { return t && t->dtype == dt; }

// [B, S, H, D] with contiguous last dim.
int check_bshd(const ra_tensor* t, int64_t B, int64_t S, int64_t H, int64_t D) {
  if (!t) return RA_ERR_NULL;
  if (t->ndim != 4) return RA_ERR_SHAPE;
  if (t->shape[0] != B || t->shape[1] != S || t->shape[2] != H || t->shape[3] != D) return RA_ERR_SHAPE;
  if (t->stride[3] != 1) return RA_ERR_STRIDE;
  if (!t->data && B * S * H * D > 0) return RA_ERR_NULL;
  return RA_OK;
}

// bf16 operand read by TMA / written with 16-byte vector stores.
int check_tma_bf16(const ra_tensor* t) {
  if (reinterpret_cast<uintptr_t>(t->data) % 16) return RA_ERR_STRIDE;
  for (int i = 0; i < 3; ++i) {
    if ((t->stride[i] * 2) % 16) return RA_ERR_STRIDE;
    if (t->stride[i] < 0 || t->stride[i] * 2 >= (int64_t(1) << 40)) return RA_ERR_STRIDE;
  }
  return RA_OK;
}

// Output written with 16-byte vector stores (bf16 or fp32 elements).
int check_vec16(const ra_tensor* t) {
  const int64_t es = t->dtype == RA_BF16 ? 2 : 4;
  if (reinterpret_cast<uintptr_t>(t->data) % 16) return RA_ERR_STRIDE;
  for (int i = 0; i < 3; ++i)
    if ((t->stride[i] * es) % 16) return RA_ERR_STRIDE;
  return RA_OK;
}

// [B, H, S] fp32 (lse, m, l).
int check_bhs(const ra_tensor* t, int64_t B, int64_t H, int64_t S) {
  if (!t) return RA_ERR_NULL;
  if (t->ndim != 3) return RA_ERR_SHAPE;
  if (t->shape[0] != B || t->shape[1] != H || t->shape[2] != S) return RA_ERR_SHAPE;
  if (t->dtype != RA_F32) return RA_ERR_DTYPE;
  if (!t->data && B * H * S > 0) return RA_ERR_NULL;
  return RA_OK;
}

// [B, S] (bias fp32 / segment ids int32), optional.
int check_bs(const ra_tensor* t, int64_t B, int64_t S, int dtype) {
  if (!t) return RA_OK;
  if (t->ndim != 2) return RA_ERR_SHAPE;
  if (t->shape[0] != B || t->shape[1] != S) return RA_ERR_SHAPE;
  if (t->dtype != dtype) return RA_ERR_DTYPE;
  if (!t->data && B * S > 0) return RA_ERR_NULL;
  return RA_OK;
}

#define RA_TRY(x)               \
  do {                          \
    int _e = (x);               \
    if (_e != RA_OK) return _e; \
  } while (0)

int make_ring(const ra_params* p, int64_t S, RingDesc* rd) {
  if (!p) return RA_ERR_NULL;
  if (p->reserved != 0) return RA_ERR_UNSUPPORTED;
  if (p->ring_size < 1) return RA_ERR_DIVISIBILITY;
  if (p->ring_size > kMaxRing) return RA_ERR_UNSUPPORTED;
  if (p->causal_block_size < 0) return RA_ERR_DIVISIBILITY;
  if (S % p->ring_size) return RA_ERR_DIVISIBILITY;
  const int64_t blk = S / p->ring_size;
  if (p->query_chunk_size < 1 || p->key_chunk_size < 1) return RA_ERR_DIVISIBILITY;
  if (blk > 0 && (blk % p->query_chunk_size || blk % p->key_chunk_size)) return RA_ERR_DIVISIBILITY;
  if (p->causal_block_size > INT32_MAX || S > (int64_t(1) << 31) - kTile) return RA_ERR_UNSUPPORTED;
  std::memset(rd, 0, sizeof(*rd));
  rd->S = S;
  rd->blk = blk > 0 ? blk : 1;
  rd->P = (int32_t)p->ring_size;
  rd->ntiles = (int32_t)ceil_div64(S, kTile);
  rd->cbs = (int32_t)p->causal_block_size;
  bool seen[kMaxRing] = {false};
  for (int t = 0; t < rd->P; ++t) {
    int32_t o = p->use_ring_order ? p->ring_order[t] : t;
    if (o < 0 || o >= rd->P || seen[o]) return RA_ERR_ORDER;
    seen[o] = true;
    rd->order[t] = o;
  }
  return RA_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace layout.  Forward: tile metadata (only with bias or segment ids).
// Backward: metadata, Delta and lse*log2(e) rows padded to a multiple of 64
// ([B*H][s_pad] each), and the fp32 dQ accumulator [B*H][S][D].
struct WsLayout {
  size_t meta = 0, delta = 0, lse2 = 0, dqacc = 0, total = 0;
  int64_t s_pad = 0;
};

WsLayout ws_layout(int which, int64_t B, int64_t S, int64_t H, int64_t D, bool need_meta) {
  WsLayout w;
  size_t off = 0;
  if (need_meta) {
    w.meta = off;
    off += align256((size_t)B * ceil_div64(S, kTile) * sizeof(int4));
  }
  if (which == 1) {
    w.s_pad = ceil_div64(S, kQTileBwd) * kQTileBwd;
    w.delta = off;
    off += align256((size_t)B * H * w.s_pad * sizeof(float));
    w.lse2 = off;
    off += align256((size_t)B * H * w.s_pad * sizeof(float));
    w.dqacc = off;
    off += align256((size_t)B * H * S * D * sizeof(float));
  }
  w.total = off;
  return w;
}

// ---------------------------------------------------------------- device facts

// Makes the device that holds `data` current for this thread and its primary
// context current (the tensor-map encoder is a driver call and needs one: a
// thread that has made no runtime call yet, such as an autograd worker, may
// have none), then returns that device's compute-capability major, or -1
// (the cause recorded) on failure.
int bind_device(const void* data) {
  cudaPointerAttributes a;
  if (cuda_fail(cudaPointerGetAttributes(&a, data), "cudaPointerGetAttributes") != RA_OK) return -1;
  int dev = a.device;
  if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged) {
    if (cuda_fail(cudaGetDevice(&dev), "cudaGetDevice") != RA_OK) return -1;
  }
  if (cuda_fail(cudaSetDevice(dev), "cudaSetDevice") != RA_OK) return -1;
  int major = 0;
  if (cuda_fail(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev), "cudaDeviceGetAttribute") !=
      RA_OK)
    return -1;
  return major;
}

// ---------------------------------------------------------------- TMA maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// bf16 [B, S, H, D] -> 4-D map (D, H, S, B), box 64 x 1 x rows x 1, 128-byte swizzle.
int make_tmap_bshd(CUtensorMap* m, const ra_tensor* t, int rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cu_fail(CUDA_ERROR_NOT_FOUND, "cuTensorMapEncodeTiled entry point");
  cuuint64_t dims[4] = {(cuuint64_t)t->shape[3], (cuuint64_t)t->shape[2], (cuuint64_t)t->shape[1],
                        (cuuint64_t)t->shape[0]};
  cuuint64_t strides[3] = {(cuuint64_t)t->stride[2] * 2, (cuuint64_t)t->stride[1] * 2, (cuuint64_t)t->stride[0] * 2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, t->data, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return cu_fail(r, "cuTensorMapEncodeTiled (bf16 [B,S,H,D])");
}

// bf16 row-major matrix [rows, cols] (row stride in elements) -> 2-D map
// (cols, rows), box 64 x box_rows, 128-byte swizzle.
int make_tmap_rows(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t row_stride, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cu_fail(CUDA_ERROR_NOT_FOUND, "cuTensorMapEncodeTiled entry point");
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_stride * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return cu_fail(r, "cuTensorMapEncodeTiled (bf16 matrix)");
}

int last_cuda(const char* what = "kernel launch") { return cuda_fail(cudaGetLastError(), what); }

// fp32 [BH][S][D] workspace -> 3-D map (D, S, BH), box D x rows x 1, no swizzle.
int make_tmap_dqacc(CUtensorMap* m, float* base, int64_t BH, int64_t S, int64_t D, int rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cu_fail(CUDA_ERROR_NOT_FOUND, "cuTensorMapEncodeTiled entry point");
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)S, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)D * 4, (cuuint64_t)S * D * 4};
  cuuint32_t box[3] = {(cuuint32_t)D, (cuuint32_t)rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return cu_fail(r, "cuTensorMapEncodeTiled (fp32 dQ accumulator)");
}

// NVTX range around one entry point's host work (its launches show under it
// in an nsys / ncu timeline).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Profiling hooks of ra_params: events recorded around the main kernel.
struct ProfScope {
  cudaEvent_t b = nullptr, e = nullptr;
  cudaStream_t st;
  ProfScope(const ra_params* p, cudaStream_t s) : st(s) {
    if (p && p->prof_event_begin && p->prof_event_end) {
      b = static_cast<cudaEvent_t>(p->prof_event_begin);
      e = static_cast<cudaEvent_t>(p->prof_event_end);
    }
  }
  void begin() const { if (b) cudaEventRecord(b, st); }
  void end() const { if (e) cudaEventRecord(e, st); }
};

MaskArgs mask_args(const ra_tensor* bias, const ra_tensor* seg) {
  MaskArgs mk{};
  if (seg) {
    mk.seg = static_cast<const int32_t*>(seg->data);
    mk.seg_sb = seg->stride[0];
    mk.seg_ss = seg->stride[1];
  }
  if (bias) {
    mk.bias = static_cast<const float*>(bias->data);
    mk.bias_sb = bias->stride[0];
    mk.bias_ss = bias->stride[1];
  }
  return mk;
}

int launch_meta(const MaskArgs& mk, int64_t B, const RingDesc& rd, int4* meta, cudaStream_t st) {
  dim3 grid(rd.ntiles, (unsigned)B);
  tile_meta_kernel<<<grid, 128, 0, st>>>(mk, rd.S, rd.ntiles, meta);
  return last_cuda();
}

// Shared-memory size attribute of the forward kernel, and the check that its
// register split (setmaxnreg) fits in the registers the block launches with.
template <int D, bool STEP>
int fwd_kernel_attrs() {
  using L = FwdLayout<D>;
  RA_TRY(cuda_fail(cudaFuncSetAttribute(ra_fwd_sm100_kernel<D, STEP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        L::SMEM_ALLOC),
                   "cudaFuncSetAttribute (forward kernel)"));
  cudaFuncAttributes fa;
  RA_TRY(cuda_fail(cudaFuncGetAttributes(&fa, ra_fwd_sm100_kernel<D, STEP>), "cudaFuncGetAttributes (forward kernel)"));
  if (128 * L::REGS_LOW + 256 * L::REGS_HIGH > L::THREADS * fa.numRegs) return RA_ERR_UNSUPPORTED;
  return RA_OK;
}

// A kernel launch whose set-up (tensor maps, kernel attributes, register
// split check) is done by prepare(), before any launch of the entry point,
// so that every set-up error is returned with nothing queued on the stream.
template <int D, bool STEP = false>
struct FwdSm100Launch {
  using L = FwdLayout<D>;
  CUtensorMap tq, tk, tv;
  FwdParams prm;
  int64_t grid = 0;

  int prepare(const ra_tensor* q, const ra_tensor* k, const ra_tensor* v, const MaskArgs& mk, const RingDesc& rd,
              const int4* meta, ra_tensor* o, ra_tensor* lse) {
    RA_TRY(make_tmap_bshd(&tq, q, kTile));
    RA_TRY(make_tmap_bshd(&tk, k, kTile));
    RA_TRY(make_tmap_bshd(&tv, v, kTile));
    std::memset(&prm, 0, sizeof(prm));
    prm.rd = rd;
    prm.B = (int32_t)q->shape[0];
    prm.H = (int32_t)q->shape[2];
    prm.npairs = (rd.ntiles + 1) / 2;
    prm.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
    prm.o = static_cast<__nv_bfloat16*>(o->data);
    prm.o_sb = o->stride[0];
    prm.o_ss = o->stride[1];
    prm.o_sh = o->stride[2];
    prm.lse = static_cast<float*>(lse->data);
    prm.lse_sb = lse->stride[0];
    prm.lse_sh = lse->stride[1];
    prm.lse_ss = lse->stride[2];
    prm.seg = mk.seg;
    prm.seg_sb = mk.seg_sb;
    prm.seg_ss = mk.seg_ss;
    prm.bias = mk.bias;
    prm.bias_sb = mk.bias_sb;
    prm.bias_ss = mk.bias_ss;
    prm.meta = meta;
#ifdef RA_DEBUG_COUNT
    prm.dbg_count = g_dbg_fwd_rows;
#endif
    grid = (int64_t)prm.npairs * prm.B * prm.H;
    if (grid > INT32_MAX) return RA_ERR_UNSUPPORTED;
    return fwd_kernel_attrs<D, STEP>();
  }
  // Ring-step mode: q_blk [B,Sq,H,D] at global token q_off against one
  // visiting block k_blk, v_blk [B,Sk,H,D] at k_off, merged into (acc, m, l).
  int prepare_step(const ra_tensor* q, const ra_tensor* k, const ra_tensor* v, int64_t q_off, int64_t k_off,
                   int32_t cbs, const ra_tensor* bias, const ra_tensor* seg_q, const ra_tensor* seg_k,
                   ra_tensor* acc, ra_tensor* m, ra_tensor* l) {
    RA_TRY(make_tmap_bshd(&tq, q, kTile));
    RA_TRY(make_tmap_bshd(&tk, k, kTile));
    RA_TRY(make_tmap_bshd(&tv, v, kTile));
    std::memset(&prm, 0, sizeof(prm));
    const int64_t Sq = q->shape[1];
    prm.rd.S = Sq;
    prm.rd.blk = Sq;
    prm.rd.P = 1;
    prm.rd.ntiles = (int32_t)ceil_div64(Sq, kTile);
    prm.rd.cbs = cbs;
    prm.B = (int32_t)q->shape[0];
    prm.H = (int32_t)q->shape[2];
    prm.npairs = (prm.rd.ntiles + 1) / 2;
    prm.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
    if (seg_q) {
      prm.seg = static_cast<const int32_t*>(seg_q->data);
      prm.seg_sb = seg_q->stride[0];
      prm.seg_ss = seg_q->stride[1];
      prm.seg_k = static_cast<const int32_t*>(seg_k->data);
      prm.segk_sb = seg_k->stride[0];
      prm.segk_ss = seg_k->stride[1];
    }
    if (bias) {
      prm.bias = static_cast<const float*>(bias->data);
      prm.bias_sb = bias->stride[0];
      prm.bias_ss = bias->stride[1];
    }
    prm.Sk = k->shape[1];
    prm.q_off = q_off;
    prm.k_off = k_off;
    prm.acc = static_cast<float*>(acc->data);
    prm.acc_sb = acc->stride[0];
    prm.acc_ss = acc->stride[1];
    prm.acc_sh = acc->stride[2];
    prm.m_state = static_cast<float*>(m->data);
    prm.l_state = static_cast<float*>(l->data);
    prm.ml_sb = m->stride[0];
    prm.ml_sh = m->stride[1];
    prm.ml_ss = m->stride[2];
    grid = (int64_t)prm.npairs * prm.B * prm.H;
    if (grid > INT32_MAX) return RA_ERR_UNSUPPORTED;
    return fwd_kernel_attrs<D, STEP>();
  }
  int launch(cudaStream_t st) const {
    ra_fwd_sm100_kernel<D, STEP><<<(unsigned)grid, L::THREADS, L::SMEM_ALLOC, st>>>(tq, tk, tv, prm);
    return last_cuda();
  }
};

View4 view4(const ra_tensor* t) { return View4{t->data, t->stride[0], t->stride[1], t->stride[2]}; }
OutView4 oview4(ra_tensor* t) { return OutView4{t->data, t->stride[0], t->stride[1], t->stride[2]}; }

template <int D, typename T>
struct FwdSimtLaunch {
  SimtFwdArgs a;
  dim3 grid;
  static constexpr int kSmem = SimtSmem<D>::BYTES;

  int prepare(const ra_tensor* q, const ra_tensor* k, const ra_tensor* v, const MaskArgs& mk, const RingDesc& rd,
              const int4* meta, ra_tensor* o, ra_tensor* lse) {
    std::memset(&a, 0, sizeof(a));
    a.rd = rd;
    a.B = (int)q->shape[0];
    a.H = (int)q->shape[2];
    a.scale = (float)(1.0 / std::sqrt((double)D));
    a.mk = mk;
    a.meta = meta;
    a.q = view4(q);
    a.k = view4(k);
    a.v = view4(v);
    a.o = oview4(o);
    a.lse = static_cast<float*>(lse->data);
    a.lse_sb = lse->stride[0];
    a.lse_sh = lse->stride[1];
    a.lse_ss = lse->stride[2];
    grid = dim3((unsigned)ceil_div64(rd.S, kSimtRows), (unsigned)(a.B * a.H));
    return cuda_fail(cudaFuncSetAttribute(simt_fwd_kernel<D, T>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem),
                     "cudaFuncSetAttribute (fp32 forward kernel)");
  }
  int launch(cudaStream_t st) const {
    simt_fwd_kernel<D, T><<<grid, kSimtRows, kSmem, st>>>(a);
    return last_cuda();
  }
};

template <int D>
struct BwdSm100Launch {
  using L = BwdLayout<D>;
  CUtensorMap tq, tk, tv, tdo, tdq;
  BwdParams prm;
  int64_t grid = 0;

  int prepare(const ra_tensor* q, const ra_tensor* k, const ra_tensor* v, const ra_tensor* d_o, const MaskArgs& mk,
              const RingDesc& rd, const int4* meta, const WsLayout& w, char* ws, ra_tensor* dk, ra_tensor* dv) {
    RA_TRY(make_tmap_bshd(&tq, q, L::QT));
    RA_TRY(make_tmap_bshd(&tk, k, kTile));
    RA_TRY(make_tmap_bshd(&tv, v, kTile));
    RA_TRY(make_tmap_bshd(&tdo, d_o, L::QT));
    RA_TRY(make_tmap_dqacc(&tdq, reinterpret_cast<float*>(ws + w.dqacc), q->shape[0] * q->shape[2], q->shape[1],
                           L::D, L::QT));
    std::memset(&prm, 0, sizeof(prm));
    prm.rd = rd;
    prm.B = (int32_t)q->shape[0];
    prm.H = (int32_t)q->shape[2];
    prm.scale = (float)(1.0 / std::sqrt((double)L::D));
    prm.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)L::D));
    prm.lse2 = reinterpret_cast<const float*>(ws + w.lse2);
    prm.delta = reinterpret_cast<const float*>(ws + w.delta);
    prm.s_pad = w.s_pad;
    prm.dqacc = reinterpret_cast<float*>(ws + w.dqacc);
    prm.dk = dk->data;
    prm.dk_sb = dk->stride[0];
    prm.dk_ss = dk->stride[1];
    prm.dk_sh = dk->stride[2];
    prm.dv = dv->data;
    prm.dv_sb = dv->stride[0];
    prm.dv_ss = dv->stride[1];
    prm.dv_sh = dv->stride[2];
    prm.grad_bf16 = dk->dtype == RA_BF16;
    prm.seg = mk.seg;
    prm.seg_sb = mk.seg_sb;
    prm.seg_ss = mk.seg_ss;
    prm.bias = mk.bias;
    prm.bias_sb = mk.bias_sb;
    prm.bias_ss = mk.bias_ss;
    prm.meta = meta;
#ifdef RA_DEBUG_COUNT
    prm.dbg_count = g_dbg_bwd_cols;
#endif
    grid = (int64_t)rd.ntiles * prm.B * prm.H;
    if (grid > INT32_MAX) return RA_ERR_UNSUPPORTED;
    return cuda_fail(
        cudaFuncSetAttribute(ra_bwd_sm100_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM_ALLOC),
        "cudaFuncSetAttribute (backward kernel)");
  }
  int launch(cudaStream_t st) const {
    ra_bwd_sm100_kernel<D><<<(unsigned)grid, L::THREADS, L::SMEM_ALLOC, st>>>(tq, tk, tv, tdo, tdq, prm);
    return last_cuda();
  }
};

template <int D, typename T>
int launch_bwd_simt(const SimtBwdArgs& a, int64_t S, cudaStream_t st) {
  dim3 grid((unsigned)ceil_div64(S, 64), (unsigned)(a.B * a.H));
  simt_bwd_dq_kernel<D, T><<<grid, 64, 0, st>>>(a);
  simt_bwd_dkdv_kernel<D, T><<<grid, 64, 0, st>>>(a);
  return last_cuda();
}

}  // namespace

// ====================================================================== C ABI

extern "C" {

const char* ra_strerror(int code) {
  switch (code) {
    case RA_OK: return "ok";
    case RA_ERR_NULL: return "a required pointer is NULL";
    case RA_ERR_DTYPE: return "unsupported or mismatched dtype";
    case RA_ERR_SHAPE: return "rank or shape mismatch";
    case RA_ERR_STRIDE: return "head dim not contiguous or TMA alignment violated (16-byte base and strides)";
    case RA_ERR_DIVISIBILITY: return "S must be divisible by ring_size, and S/ring_size by both chunk sizes";
    case RA_ERR_UNSUPPORTED: return "unsupported configuration (head_dim, ring_size, device or size limits)";
    case RA_ERR_WORKSPACE: return "workspace missing or too small";
    case RA_ERR_CUDA: return "CUDA runtime error";
    case RA_ERR_DEVICE_TIMEOUT: return "a device-side bounded wait ran out";
    case RA_ERR_ORDER: return "ring_order is not a permutation of 0..ring_size-1";
    case RA_ERR_STATIC_LIMIT:
      return "problem needs more scratch than ra_forward_static provides (B * ceil(S/128) must be <= 65536)";
    default: return "unknown error";
  }
}

size_t ra_workspace_size(int which, const ra_tensor* q, const ra_params* p, int has_bias, int has_segments) {
  if (!q || !p || q->ndim != 4 || (which != 0 && which != 1)) return (size_t)-1;
  return ws_layout(which, q->shape[0], q->shape[1], q->shape[2], q->shape[3], has_bias || has_segments).total;
}

int ra_forward(const ra_tensor* q, const ra_tensor* k, const ra_tensor* v, const ra_tensor* attention_bias,
               const ra_tensor* segment_ids, const ra_params* p, ra_tensor* o, ra_tensor* lse, void* workspace,
               size_t workspace_bytes, void* stream) {
  const NvtxRange nvtx_range("ra_forward");
  if (!q || !k || !v || !o || !lse || !p) return RA_ERR_NULL;
  if (q->ndim != 4) return RA_ERR_SHAPE;
  const int64_t B = q->shape[0], S = q->shape[1], H = q->shape[2], D = q->shape[3];
  if (B < 0 || S < 0 || H < 0) return RA_ERR_SHAPE;
  RA_TRY(check_bshd(q, B, S, H, D));
  RA_TRY(check_bshd(k, B, S, H, D));
  RA_TRY(check_bshd(v, B, S, H, D));
  RA_TRY(check_bshd(o, B, S, H, D));
  RA_TRY(check_bhs(lse, B, H, S));
  RA_TRY(check_bs(attention_bias, B, S, RA_F32));
  RA_TRY(check_bs(segment_ids, B, S, RA_I32));
  if (D != 64 && D != 128) return RA_ERR_UNSUPPORTED;
  const int dt = q->dtype;
  if (dt != RA_BF16 && dt != RA_F32) return RA_ERR_DTYPE;
  if (!is_dtype(k, dt) || !is_dtype(v, dt) || !is_dtype(o, dt)) return RA_ERR_DTYPE;
  if (B * S * H == 0) {
    RingDesc rd;
    return make_ring(p, S, &rd) == RA_ERR_ORDER ? RA_ERR_ORDER : RA_OK;
  }
  RingDesc rd;
  RA_TRY(make_ring(p, S, &rd));
  if (dt == RA_BF16) {
    RA_TRY(check_tma_bf16(q));
    RA_TRY(check_tma_bf16(k));
    RA_TRY(check_tma_bf16(v));
    RA_TRY(check_tma_bf16(o));
  }
  const bool need_meta = attention_bias || segment_ids;
  const WsLayout w = ws_layout(0, B, S, H, D, need_meta);
  if (w.total > 0 && (!workspace || workspace_bytes < w.total)) return RA_ERR_WORKSPACE;
  if (w.total > 0 && reinterpret_cast<uintptr_t>(workspace) % 256) return RA_ERR_WORKSPACE;
  {
    const int major = bind_device(q->data);
    if (major < 0) return RA_ERR_CUDA;   // cause recorded by bind_device
    if (dt == RA_BF16 && major != 10) return RA_ERR_UNSUPPORTED;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const MaskArgs mk = mask_args(attention_bias, segment_ids);
  int4* meta = need_meta ? reinterpret_cast<int4*>(static_cast<char*>(workspace) + w.meta) : nullptr;
  const ProfScope prof(p, st);
  // Set-up first (tensor maps, attributes), then the launches: a set-up
  // error returns with nothing queued.
  auto run = [&](auto& lc) -> int {
    RA_TRY(lc.prepare(q, k, v, mk, rd, meta, o, lse));
    if (meta) RA_TRY(launch_meta(mk, B, rd, meta, st));
    prof.begin();
    const int rc = lc.launch(st);
    prof.end();
    return rc;
  };
  if (dt == RA_BF16) {
    if (D == 64) {
      FwdSm100Launch<64> lc;
      return run(lc);
    }
    FwdSm100Launch<128> lc;
    return run(lc);
  }
  if (D == 64) {
    FwdSimtLaunch<64, float> lc;
    return run(lc);
  }
  FwdSimtLaunch<128, float> lc;
  return run(lc);
}

int ra_backward(const ra_tensor* q, const ra_tensor* k, const ra_tensor* v, const ra_tensor* o,
                const ra_tensor* d_o, const ra_tensor* lse, const ra_tensor* attention_bias,
                const ra_tensor* segment_ids, const ra_params* p, ra_tensor* dq, ra_tensor* dk, ra_tensor* dv,
                void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !o || !d_o || !lse || !p || !dq || !dk || !dv) return RA_ERR_NULL;
  const NvtxRange nvtx_range("ra_backward");
  if (q->ndim != 4) return RA_ERR_SHAPE;
  const int64_t B = q->shape[0], S = q->shape[1], H = q->shape[2], D = q->shape[3];
  if (B < 0 || S < 0 || H < 0) return RA_ERR_SHAPE;
  for (const ra_tensor* t : {q, k, v, o, d_o, (const ra_tensor*)dq, (const ra_tensor*)dk, (const ra_tensor*)dv})
    RA_TRY(check_bshd(t, B, S, H, D));
  RA_TRY(check_bhs(lse, B, H, S));
  RA_TRY(check_bs(attention_bias, B, S, RA_F32));
  RA_TRY(check_bs(segment_ids, B, S, RA_I32));
  if (D != 64 && D != 128) return RA_ERR_UNSUPPORTED;
  const int dt = q->dtype;
  if (dt != RA_BF16 && dt != RA_F32) return RA_ERR_DTYPE;
  for (const ra_tensor* t : {k, v, o, d_o})
    if (!is_dtype(t, dt)) return RA_ERR_DTYPE;
  for (const ra_tensor* t : {(const ra_tensor*)dq, (const ra_tensor*)dk, (const ra_tensor*)dv}) {
    if (t->dtype != RA_BF16 && t->dtype != RA_F32) return RA_ERR_DTYPE;
    if (dt == RA_F32 && t->dtype != RA_F32) return RA_ERR_DTYPE;
  }
  RingDesc rd;
  if (B * S * H == 0) return make_ring(p, S, &rd) == RA_ERR_ORDER ? RA_ERR_ORDER : RA_OK;
  RA_TRY(make_ring(p, S, &rd));
  if (dt == RA_BF16) {
    for (const ra_tensor* t : {q, k, v, o, d_o}) RA_TRY(check_tma_bf16(t));
    if (D == 128) {
      RA_TRY(check_vec16(dk));
      RA_TRY(check_vec16(dv));
    }
  }
  const bool need_meta = attention_bias || segment_ids;
  const WsLayout w = ws_layout(1, B, S, H, D, need_meta);
  if (!workspace || workspace_bytes < w.total || reinterpret_cast<uintptr_t>(workspace) % 256)
    return RA_ERR_WORKSPACE;
  {
    const int major = bind_device(q->data);
    if (major < 0) return RA_ERR_CUDA;   // cause recorded by bind_device
    if (dt == RA_BF16 && major != 10) return RA_ERR_UNSUPPORTED;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const MaskArgs mk = mask_args(attention_bias, segment_ids);
  char* ws = static_cast<char*>(workspace);
  int4* meta = need_meta ? reinterpret_cast<int4*>(ws + w.meta) : nullptr;
  const bool tc_path = dt == RA_BF16;   // tensor-core backward (D = 64 or 128); fp32 inputs on CUDA cores
  if (!tc_path && (dk->dtype != dq->dtype || dv->dtype != dq->dtype)) return RA_ERR_DTYPE;
  // Set-up of the main kernel first: a set-up error returns with nothing queued.
  BwdSm100Launch<64> lc64;
  BwdSm100Launch<128> lc128;
  if (tc_path) {
    if (D == 64) RA_TRY(lc64.prepare(q, k, v, d_o, mk, rd, meta, w, ws, dk, dv));
    else RA_TRY(lc128.prepare(q, k, v, d_o, mk, rd, meta, w, ws, dk, dv));
  }
  if (meta) RA_TRY(launch_meta(mk, B, rd, meta, st));
  {
    BwdPreArgs pa;
    std::memset(&pa, 0, sizeof(pa));
    pa.B = (int)B; pa.S = (int)S; pa.H = (int)H; pa.D = (int)D;
    pa.o = o->data; pa.o_sb = o->stride[0]; pa.o_ss = o->stride[1]; pa.o_sh = o->stride[2];
    pa.dO = d_o->data; pa.do_sb = d_o->stride[0]; pa.do_ss = d_o->stride[1]; pa.do_sh = d_o->stride[2];
    pa.lse = static_cast<const float*>(lse->data);
    pa.lse_sb = lse->stride[0]; pa.lse_sh = lse->stride[1]; pa.lse_ss = lse->stride[2];
    pa.bf16 = dt == RA_BF16;
    pa.s_pad = w.s_pad;
    pa.delta = reinterpret_cast<float*>(ws + w.delta);
    pa.lse2 = reinterpret_cast<float*>(ws + w.lse2);
    pa.dqacc = tc_path ? reinterpret_cast<float*>(ws + w.dqacc) : nullptr;
    const int64_t threads = B * H * w.s_pad * 32;
    bwd_pre_kernel<<<(unsigned)ceil_div64(threads, 256), 256, 0, st>>>(pa);
    RA_TRY(last_cuda());
  }
  const ProfScope prof(p, st);
  if (tc_path) {
    prof.begin();
    const int rc = D == 64 ? lc64.launch(st) : lc128.launch(st);
    prof.end();
    RA_TRY(rc);
    DqConvertArgs ca{(int)B, (int)S, (int)H, (int)D, reinterpret_cast<const float*>(ws + w.dqacc),
                     dq->data, dq->stride[0], dq->stride[1], dq->stride[2], dq->dtype == RA_BF16};
    const int64_t n = B * S * H * D;
    dq_convert_kernel<<<(unsigned)ceil_div64(n, 256), 256, 0, st>>>(ca);
    return last_cuda();
  }
  SimtBwdArgs a;
  std::memset(&a, 0, sizeof(a));
  a.rd = rd;
  a.B = (int)B;
  a.H = (int)H;
  a.scale = (float)(1.0 / std::sqrt((double)D));
  a.mk = mk;
  a.q = view4(q);
  a.k = view4(k);
  a.v = view4(v);
  a.dO = view4(d_o);
  a.lse = static_cast<const float*>(lse->data);
  a.lse_sb = lse->stride[0];
  a.lse_sh = lse->stride[1];
  a.lse_ss = lse->stride[2];
  a.delta = reinterpret_cast<const float*>(ws + w.delta);
  a.s_pad = w.s_pad;
  a.dq = oview4(dq);
  a.dk = oview4(dk);
  a.dv = oview4(dv);
  a.out_bf16 = dq->dtype == RA_BF16;
  prof.begin();
  int rc;
  rc = D == 64 ? launch_bwd_simt<64, float>(a, S, st) : launch_bwd_simt<128, float>(a, S, st);   // fp32 inputs
  prof.end();
  return rc;
}

int ra_step(const ra_tensor* q_blk, const ra_tensor* k_blk, const ra_tensor* v_blk, int64_t q_off, int64_t k_off,
            const ra_tensor* bias_blk, const ra_tensor* seg_q, const ra_tensor* seg_k, const ra_params* p,
            ra_tensor* o_acc, ra_tensor* m, ra_tensor* l, void* stream) {
  if (!q_blk || !k_blk || !v_blk || !p || !o_acc || !m || !l) return RA_ERR_NULL;
  if (q_blk->ndim != 4 || k_blk->ndim != 4) return RA_ERR_SHAPE;
  const int64_t B = q_blk->shape[0], Sq = q_blk->shape[1], H = q_blk->shape[2], D = q_blk->shape[3];
  const int64_t Sk = k_blk->shape[1];
  // A key/value block of batch 1 is shared by every query batch row (one
  // cached prefix serving several requests); otherwise batches match.
  const int64_t Bk = k_blk->shape[0];
  if (B < 0 || Sq < 0 || Sk < 0 || H < 0) return RA_ERR_SHAPE;
  if (Bk != B && Bk != 1) return RA_ERR_SHAPE;
  const bool kv_bcast = Bk == 1 && B != 1;
  RA_TRY(check_bshd(q_blk, B, Sq, H, D));
  RA_TRY(check_bshd(k_blk, Bk, Sk, H, D));
  RA_TRY(check_bshd(v_blk, Bk, Sk, H, D));
  RA_TRY(check_bshd(o_acc, B, Sq, H, D));
  RA_TRY(check_bhs(m, B, H, Sq));
  RA_TRY(check_bhs(l, B, H, Sq));
  RA_TRY(check_bs(bias_blk, Bk, Sk, RA_F32));
  if ((seg_q == nullptr) != (seg_k == nullptr)) return RA_ERR_NULL;
  RA_TRY(check_bs(seg_q, B, Sq, RA_I32));
  RA_TRY(check_bs(seg_k, Bk, Sk, RA_I32));
  if (D != 64 && D != 128) return RA_ERR_UNSUPPORTED;
  const int dt = q_blk->dtype;
  if (dt != RA_BF16 && dt != RA_F32) return RA_ERR_DTYPE;
  if (!is_dtype(k_blk, dt) || !is_dtype(v_blk, dt) || o_acc->dtype != RA_F32) return RA_ERR_DTYPE;
  if (p->causal_block_size < 0 || q_off < 0 || k_off < 0) return RA_ERR_DIVISIBILITY;
  if (m->stride[0] != l->stride[0] || m->stride[1] != l->stride[1] || m->stride[2] != l->stride[2])
    return RA_ERR_STRIDE;
  if (B * Sq * H == 0 || Sk == 0) return RA_OK;
  if (Sq > (int64_t(1) << 31) - kTile || Sk > (int64_t(1) << 31) - kTile) return RA_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int major = bind_device(q_blk->data);
  if (major < 0) return RA_ERR_CUDA;   // cause recorded by bind_device
  if (dt == RA_BF16) {
    // tensor-core step: the forward kernel in ring-step mode
    for (const ra_tensor* t : {q_blk, k_blk, v_blk}) RA_TRY(check_tma_bf16(t));
    RA_TRY(check_vec16(o_acc));   // the state is read and written with 16-byte vectors
    if (major != 10) return RA_ERR_UNSUPPORTED;
    const int32_t cbs = (int32_t)(p->causal_block_size > INT32_MAX ? INT32_MAX : p->causal_block_size);
    auto run = [&](auto& lc) -> int {
      RA_TRY(lc.prepare_step(q_blk, k_blk, v_blk, q_off, k_off, cbs, bias_blk, seg_q, seg_k, o_acc, m, l));
      lc.prm.kv_bcast = kv_bcast ? 1 : 0;
      return lc.launch(st);
    };
    if (D == 64) {
      FwdSm100Launch<64, true> lc;
      return run(lc);
    }
    FwdSm100Launch<128, true> lc;
    return run(lc);
  }
  SimtStepArgs a;
  std::memset(&a, 0, sizeof(a));
  a.B = (int)B;
  a.H = (int)H;
  a.D = (int)D;
  a.Sq = Sq;
  a.Sk = Sk;
  a.q_off = q_off;
  a.k_off = k_off;
  a.cbs = (int32_t)p->causal_block_size;
  a.scale = (float)(1.0 / std::sqrt((double)D));
  a.q = view4(q_blk);
  a.k = view4(k_blk);
  a.v = view4(v_blk);
  if (kv_bcast) a.k.sb = a.v.sb = 0;   // every query batch row reads key/value batch row 0
  if (seg_q) {
    a.seg_q = static_cast<const int32_t*>(seg_q->data);
    a.segq_sb = seg_q->stride[0];
    a.segq_ss = seg_q->stride[1];
    a.seg_k = static_cast<const int32_t*>(seg_k->data);
    a.segk_sb = kv_bcast ? 0 : seg_k->stride[0];
    a.segk_ss = seg_k->stride[1];
  }
  if (bias_blk) {
    a.bias = static_cast<const float*>(bias_blk->data);
    a.bias_sb = kv_bcast ? 0 : bias_blk->stride[0];
    a.bias_ss = bias_blk->stride[1];
  }
  a.acc = static_cast<float*>(o_acc->data);
  a.acc_sb = o_acc->stride[0];
  a.acc_ss = o_acc->stride[1];
  a.acc_sh = o_acc->stride[2];
  a.m = static_cast<float*>(m->data);
  a.l = static_cast<float*>(l->data);
  a.ml_sb = m->stride[0];
  a.ml_sh = m->stride[1];
  a.ml_ss = m->stride[2];
  dim3 grid((unsigned)ceil_div64(Sq, kSimtRows), (unsigned)(B * H));
  // fp32 inputs: CUDA-core step
  if (D == 64) {
    const int smem = SimtSmem<64>::BYTES;
    RA_TRY(cuda_fail(cudaFuncSetAttribute(simt_step_kernel<64, float>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem),
                     "cudaFuncSetAttribute (fp32 step kernel)"));
    simt_step_kernel<64, float><<<grid, kSimtRows, smem, st>>>(a);
  } else {
    const int smem = SimtSmem<128>::BYTES;
    RA_TRY(cuda_fail(cudaFuncSetAttribute(simt_step_kernel<128, float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          smem),
                     "cudaFuncSetAttribute (fp32 step kernel)"));
    simt_step_kernel<128, float><<<grid, kSimtRows, smem, st>>>(a);
  }
  return last_cuda();
}

int ra_finalize(const ra_tensor* o_acc, const ra_tensor* m, const ra_tensor* l, ra_tensor* o, ra_tensor* lse,
                void* stream) {
  if (!o_acc || !m || !l || !o || !lse) return RA_ERR_NULL;
  if (o_acc->ndim != 4) return RA_ERR_SHAPE;
  const int64_t B = o_acc->shape[0], S = o_acc->shape[1], H = o_acc->shape[2], D = o_acc->shape[3];
  RA_TRY(check_bshd(o_acc, B, S, H, D));
  RA_TRY(check_bshd(o, B, S, H, D));
  RA_TRY(check_bhs(m, B, H, S));
  RA_TRY(check_bhs(l, B, H, S));
  RA_TRY(check_bhs(lse, B, H, S));
  if (o_acc->dtype != RA_F32) return RA_ERR_DTYPE;
  if (o->dtype != RA_F32 && o->dtype != RA_BF16) return RA_ERR_DTYPE;
  if (m->stride[0] != l->stride[0] || m->stride[1] != l->stride[1] || m->stride[2] != l->stride[2])
    return RA_ERR_STRIDE;
  const int64_t n = B * S * H;
  if (n == 0) return RA_OK;
  FinalizeArgs a{(int)B, (int)S, (int)H, (int)D,
                 static_cast<const float*>(o_acc->data), o_acc->stride[0], o_acc->stride[1], o_acc->stride[2],
                 static_cast<const float*>(m->data), static_cast<const float*>(l->data),
                 m->stride[0], m->stride[1], m->stride[2],
                 o->data, o->stride[0], o->stride[1], o->stride[2], o->dtype == RA_BF16,
                 static_cast<float*>(lse->data), lse->stride[0], lse->stride[1], lse->stride[2]};
  if (bind_device(o_acc->data) < 0) return RA_ERR_CUDA;
  finalize_kernel<<<(unsigned)ceil_div64(n, 128), 128, 0, static_cast<cudaStream_t>(stream)>>>(a);
  return last_cuda();
}

int ra_lse_merge(const ra_tensor* o_a, const ra_tensor* lse_a, const ra_tensor* o_b, const ra_tensor* lse_b,
                 ra_tensor* o_out, ra_tensor* lse_out, void* stream) {
  if (!o_a || !lse_a || !o_b || !lse_b || !o_out || !lse_out) return RA_ERR_NULL;
  if (o_a->ndim != 4) return RA_ERR_SHAPE;
  const int64_t B = o_a->shape[0], S = o_a->shape[1], H = o_a->shape[2], D = o_a->shape[3];
  RA_TRY(check_bshd(o_a, B, S, H, D));
  RA_TRY(check_bshd(o_b, B, S, H, D));
  RA_TRY(check_bshd(o_out, B, S, H, D));
  RA_TRY(check_bhs(lse_a, B, H, S));
  RA_TRY(check_bhs(lse_b, B, H, S));
  RA_TRY(check_bhs(lse_out, B, H, S));
  const int dt = o_a->dtype;
  if (dt != RA_F32 && dt != RA_BF16) return RA_ERR_DTYPE;
  if (o_b->dtype != dt || o_out->dtype != dt) return RA_ERR_DTYPE;
  const int64_t n = B * S * H;
  if (n == 0) return RA_OK;
  MergeArgs a{(int)B, (int)S, (int)H, (int)D,
              o_a->data, o_a->stride[0], o_a->stride[1], o_a->stride[2],
              static_cast<const float*>(lse_a->data), lse_a->stride[0], lse_a->stride[1], lse_a->stride[2],
              o_b->data, o_b->stride[0], o_b->stride[1], o_b->stride[2],
              static_cast<const float*>(lse_b->data), lse_b->stride[0], lse_b->stride[1], lse_b->stride[2],
              o_out->data, o_out->stride[0], o_out->stride[1], o_out->stride[2],
              static_cast<float*>(lse_out->data), lse_out->stride[0], lse_out->stride[1], lse_out->stride[2],
              dt == RA_BF16};
  if (bind_device(o_a->data) < 0) return RA_ERR_CUDA;
  lse_merge_kernel<<<(unsigned)ceil_div64(n, 128), 128, 0, static_cast<cudaStream_t>(stream)>>>(a);
  return last_cuda();
}

size_t ra_feedforward_workspace_size(int64_t chunk_size, int64_t d_ff) {
  if (chunk_size < 1 || d_ff < 1) return (size_t)-1;
  return align256((size_t)chunk_size * (size_t)d_ff * 2);
}

int ra_feedforward(const ra_tensor* x, const ra_tensor* w1, const ra_tensor* w3, const ra_tensor* w2, ra_tensor* y,
                   int64_t chunk_size, void* workspace, size_t workspace_bytes, void* stream) {
  const NvtxRange nvtx_range("ra_feedforward");
  if (!x || !w1 || !w3 || !w2 || !y) return RA_ERR_NULL;
  for (const ra_tensor* t : {x, w1, w3, w2, (const ra_tensor*)y}) {
    if (t->ndim != 2) return RA_ERR_SHAPE;
    if (t->dtype != RA_BF16) return RA_ERR_DTYPE;
  }
  const int64_t T = x->shape[0], dm = x->shape[1], dff = w1->shape[0];
  if (T < 0 || dm < 1 || dff < 1) return RA_ERR_SHAPE;
  if (w1->shape[1] != dm || w3->shape[0] != dff || w3->shape[1] != dm || w2->shape[0] != dm || w2->shape[1] != dff ||
      y->shape[0] != T || y->shape[1] != dm)
    return RA_ERR_SHAPE;
  for (const ra_tensor* t : {x, w1, w3, w2, (const ra_tensor*)y}) {
    if (t->stride[1] != 1) return RA_ERR_STRIDE;
    if (reinterpret_cast<uintptr_t>(t->data) % 16 || (t->stride[0] * 2) % 16 || t->stride[0] < t->shape[1])
      return RA_ERR_STRIDE;
    if (!t->data && t->shape[0] * t->shape[1] > 0) return RA_ERR_NULL;
  }
  // output columns are written 32 at a time; rows of the reduction are read by TMA
  if (dm % 32 || dff % 32) return RA_ERR_UNSUPPORTED;
  if (chunk_size < 1) return RA_ERR_DIVISIBILITY;
  if (T == 0) return RA_OK;
  const int64_t chunk = chunk_size < T ? chunk_size : T;
  if (chunk > INT32_MAX / 2 || T > INT32_MAX / 2 || dff > INT32_MAX / 2 || dm > INT32_MAX / 2) return RA_ERR_UNSUPPORTED;
  const size_t need = ra_feedforward_workspace_size(chunk, dff);
  if (!workspace || workspace_bytes < need || reinterpret_cast<uintptr_t>(workspace) % 256) return RA_ERR_WORKSPACE;
  const int major = bind_device(x->data);
  if (major < 0) return RA_ERR_CUDA;
  if (major != 10) return RA_ERR_UNSUPPORTED;
  int dev = 0, sms = 0;
  RA_TRY(cuda_fail(cudaGetDevice(&dev), "cudaGetDevice"));
  RA_TRY(cuda_fail(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev), "cudaDeviceGetAttribute"));
  // set-up first: every tensor map and attribute, then the launches
  __nv_bfloat16* hbuf = static_cast<__nv_bfloat16*>(workspace);
  CUtensorMap tx, tw1, tw3, tw2, th;
  RA_TRY(make_tmap_rows(&tx, x->data, T, dm, x->stride[0], FfnLayout::BM));
  RA_TRY(make_tmap_rows(&tw1, w1->data, dff, dm, w1->stride[0], 128));
  RA_TRY(make_tmap_rows(&tw3, w3->data, dff, dm, w3->stride[0], 128));
  RA_TRY(make_tmap_rows(&tw2, w2->data, dm, dff, w2->stride[0], FfnLayout::BN));
  RA_TRY(make_tmap_rows(&th, hbuf, chunk, dff, dff, FfnLayout::BM));
  RA_TRY(cuda_fail(cudaFuncSetAttribute(ra_ffn_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        FfnLayout::SMEM_ALLOC),
                   "cudaFuncSetAttribute (feed-forward gated GEMM)"));
  RA_TRY(cuda_fail(cudaFuncSetAttribute(ra_ffn_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        FfnLayout::SMEM_ALLOC),
                   "cudaFuncSetAttribute (feed-forward GEMM)"));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  __nv_bfloat16* yp = static_cast<__nv_bfloat16*>(y->data);
  for (int64_t m0 = 0; m0 < T; m0 += chunk) {
    const int64_t M = T - m0 < chunk ? T - m0 : chunk;
    FfnParams g{};
    g.M = (int32_t)M;
    g.a_row0 = (int32_t)m0;
    g.c_row0 = 0;
    g.N = (int32_t)dff;
    g.K = (int32_t)dm;
    g.n_tiles = (int32_t)((dff + 127) / 128);
    g.m_tiles = (int32_t)((M + FfnLayout::BM - 1) / FfnLayout::BM);
    g.c = hbuf;
    g.ldc = dff;
    const int grid1 = (int)std::min<int64_t>((int64_t)g.n_tiles * g.m_tiles, sms);
    ra_ffn_gemm_kernel<true><<<grid1, FfnLayout::THREADS, FfnLayout::SMEM_ALLOC, st>>>(tx, tw1, tw3, g);
    RA_TRY(last_cuda("feed-forward gated GEMM launch"));
    FfnParams o{};
    o.M = (int32_t)M;
    o.a_row0 = 0;
    o.c_row0 = m0;
    o.N = (int32_t)dm;
    o.K = (int32_t)dff;
    o.n_tiles = (int32_t)((dm + FfnLayout::BN - 1) / FfnLayout::BN);
    o.m_tiles = g.m_tiles;
    o.c = yp;
    o.ldc = y->stride[0];
    const int grid2 = (int)std::min<int64_t>((int64_t)o.n_tiles * o.m_tiles, sms);
    ra_ffn_gemm_kernel<false><<<grid2, FfnLayout::THREADS, FfnLayout::SMEM_ALLOC, st>>>(th, tw2, tw2, o);
    RA_TRY(last_cuda("feed-forward GEMM launch"));
  }
  return RA_OK;
}

int ra_forward_static(const ra_tensor* q, const ra_tensor* k, const ra_tensor* v, const ra_tensor* attention_bias,
                      const ra_tensor* segment_ids, const ra_params* p, ra_tensor* o, ra_tensor* lse, void* stream) {
  if (!q || q->ndim != 4) return q ? RA_ERR_SHAPE : RA_ERR_NULL;
  if (q->shape[0] < 0 || q->shape[1] < 0 || q->shape[2] < 0 || q->shape[3] < 0) return RA_ERR_SHAPE;
  const bool need_meta = attention_bias || segment_ids;
  const WsLayout w = ws_layout(0, q->shape[0], q->shape[1], q->shape[2], q->shape[3], need_meta);
  if (w.total > RA_STATIC_SCRATCH_BYTES) return RA_ERR_STATIC_LIMIT;
  void* scratch = nullptr;
  if (w.total > 0) {
    // The array's device address belongs to the module loaded in the current
    // context; it is looked up on every call (a host-side table lookup once
    // the module is loaded), so a context that was destroyed and created
    // again, or another context on the same device, gets its own address.
    RA_TRY(cuda_fail(cudaGetSymbolAddress(&scratch, g_ra_static_scratch), "cudaGetSymbolAddress (static scratch)"));
    if (!scratch) return cuda_fail(cudaErrorInvalidSymbol, "cudaGetSymbolAddress (static scratch)");
  }
  return ra_forward(q, k, v, attention_bias, segment_ids, p, o, lse, scratch, RA_STATIC_SCRATCH_BYTES, stream);
}

namespace {

bool contiguous_bshd(const ra_tensor* t) {
  return t && t->ndim == 4 && t->stride[3] == 1 && t->stride[2] == t->shape[3] &&
         t->stride[1] == t->shape[2] * t->shape[3] && t->stride[0] == t->shape[1] * t->stride[1];
}
bool contiguous_bhs(const ra_tensor* t) {
  return t && t->ndim == 3 && t->stride[2] == 1 && t->stride[1] == t->shape[2] &&
         t->stride[0] == t->shape[1] * t->shape[2];
}
bool same_shape(const ra_tensor* a, const ra_tensor* b) {
  if (a->ndim != b->ndim || a->dtype != b->dtype) return false;
  for (int i = 0; i < a->ndim; ++i)
    if (a->shape[i] != b->shape[i]) return false;
  return true;
}
size_t elem_bytes(int dt) { return dt == RA_BF16 ? 2 : 4; }

// The heads [h0, h0 + hg) of a contiguous [B,S,H,D] tensor, as a strided view.
ra_tensor head_view(const ra_tensor& t, int64_t h0, int64_t hg) {
  ra_tensor v = t;
  v.data = static_cast<char*>(t.data) + h0 * t.shape[3] * elem_bytes(t.dtype);
  v.shape[2] = hg;
  return v;
}
// The heads [h0, h0 + hg) of a contiguous [B,H,S] tensor.
ra_tensor head_view_bhs(const ra_tensor& t, int64_t h0, int64_t hg) {
  ra_tensor v = t;
  v.data = static_cast<char*>(t.data) + h0 * t.shape[2] * 4;
  v.shape[1] = hg;
  return v;
}
// Copy heads [h0, h0 + hg) of a contiguous [B,S,H,D] tensor: B*S rows of
// hg*D elements, pitch H*D elements.
cudaError_t copy_heads(const ra_tensor& dst, const ra_tensor& src, int64_t h0, int64_t hg, cudaMemcpyKind kind,
                       cudaStream_t st) {
  const size_t e = elem_bytes(src.dtype), D = (size_t)src.shape[3], H = (size_t)src.shape[2];
  const size_t off = (size_t)h0 * D * e, pitch = H * D * e;
  return cudaMemcpy2DAsync(static_cast<char*>(dst.data) + off, pitch, static_cast<const char*>(src.data) + off,
                           pitch, (size_t)hg * D * e, (size_t)(src.shape[0] * src.shape[1]), kind, st);
}
// Heads [h0, h0 + hg) of a contiguous fp32 [B,H,S] tensor: B rows of hg*S floats.
cudaError_t copy_heads_bhs(const ra_tensor& dst, const ra_tensor& src, int64_t h0, int64_t hg, cudaMemcpyKind kind,
                           cudaStream_t st) {
  const size_t S = (size_t)src.shape[2], H = (size_t)src.shape[1];
  const size_t off = (size_t)h0 * S * 4, pitch = H * S * 4;
  return cudaMemcpy2DAsync(static_cast<char*>(dst.data) + off, pitch, static_cast<const char*>(src.data) + off,
                           pitch, (size_t)hg * S * 4, (size_t)src.shape[0], kind, st);
}

struct EventPool {   // events of one call, released on every return path
  std::vector<cudaEvent_t> ev;
  ~EventPool() {
    for (cudaEvent_t e : ev) cudaEventDestroy(e);   // pending events are released once they complete
  }
  cudaEvent_t make() {
    cudaEvent_t e = nullptr;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return nullptr;
    ev.push_back(e);
    return e;
  }
};

}  // namespace

int ra_train_step_host(const ra_host_step* t, const ra_tensor* attention_bias, const ra_tensor* segment_ids,
                       const ra_params* p, int64_t heads_per_group, void* workspace, size_t workspace_bytes,
                       void* compute_stream, void* h2d_stream, void* d2h_stream) {
  if (!t || !p) return RA_ERR_NULL;
  const NvtxRange nvtx_range("ra_train_step_host");
  const ra_tensor* bshd[] = {&t->q, &t->k, &t->v, &t->d_o, &t->o, &t->dq, &t->dk, &t->dv,
                             &t->dev_q, &t->dev_k, &t->dev_v, &t->dev_do, &t->dev_o, &t->dev_dq, &t->dev_dk,
                             &t->dev_dv};
  for (const ra_tensor* x : bshd)
    if (x->ndim != 4) return RA_ERR_SHAPE;
  for (const ra_tensor* x : bshd)
    if (!same_shape(x, &t->q)) return x->dtype != t->q.dtype ? RA_ERR_DTYPE : RA_ERR_SHAPE;
  for (const ra_tensor* x : bshd)
    if (!contiguous_bshd(x)) return RA_ERR_STRIDE;
  const int64_t B = t->q.shape[0], S = t->q.shape[1], H = t->q.shape[2];
  for (const ra_tensor* x : {&t->lse, &t->dev_lse}) {
    if (x->ndim != 3 || x->dtype != RA_F32) return x->ndim != 3 ? RA_ERR_SHAPE : RA_ERR_DTYPE;
    if (x->shape[0] != B || x->shape[1] != H || x->shape[2] != S) return RA_ERR_SHAPE;
    if (!contiguous_bhs(x)) return RA_ERR_STRIDE;
  }
  if (heads_per_group < 1 || H % heads_per_group) return RA_ERR_DIVISIBILITY;
  if (B * S * H == 0) return RA_OK;   // nothing to move or compute
  for (const ra_tensor* x : bshd)
    if (!x->data) return RA_ERR_NULL;
  if (!t->lse.data || !t->dev_lse.data) return RA_ERR_NULL;
  cudaStream_t sc = static_cast<cudaStream_t>(compute_stream), si = static_cast<cudaStream_t>(h2d_stream),
               so = static_cast<cudaStream_t>(d2h_stream);
  EventPool pool;
  // The copies of this step start after everything queued before it on compute_stream.
  cudaEvent_t start = pool.make();
  if (!start) return cuda_fail(cudaGetLastError(), "cudaEventCreateWithFlags");
  RA_TRY(cuda_fail(cudaEventRecord(start, sc), "cudaEventRecord"));
  RA_TRY(cuda_fail(cudaStreamWaitEvent(si, start, 0), "cudaStreamWaitEvent (h2d stream)"));
  RA_TRY(cuda_fail(cudaStreamWaitEvent(so, start, 0), "cudaStreamWaitEvent (d2h stream)"));
  const int64_t hg = heads_per_group;
  for (int64_t h0 = 0; h0 < H; h0 += hg) {
    const ra_tensor* in_h[] = {&t->q, &t->k, &t->v, &t->d_o};
    const ra_tensor* in_d[] = {&t->dev_q, &t->dev_k, &t->dev_v, &t->dev_do};
    for (int i = 0; i < 4; ++i)
      RA_TRY(cuda_fail(copy_heads(*in_d[i], *in_h[i], h0, hg, cudaMemcpyHostToDevice, si), "cudaMemcpy2DAsync (h2d)"));
    cudaEvent_t landed = pool.make(), done = pool.make();
    if (!landed || !done) return cuda_fail(cudaGetLastError(), "cudaEventCreateWithFlags");
    RA_TRY(cuda_fail(cudaEventRecord(landed, si), "cudaEventRecord"));
    RA_TRY(cuda_fail(cudaStreamWaitEvent(sc, landed, 0), "cudaStreamWaitEvent (compute stream)"));
    ra_tensor q = head_view(t->dev_q, h0, hg), k = head_view(t->dev_k, h0, hg), v = head_view(t->dev_v, h0, hg),
              d_o = head_view(t->dev_do, h0, hg), o = head_view(t->dev_o, h0, hg),
              dq = head_view(t->dev_dq, h0, hg), dk = head_view(t->dev_dk, h0, hg),
              dv = head_view(t->dev_dv, h0, hg), lse = head_view_bhs(t->dev_lse, h0, hg);
    RA_TRY(ra_forward(&q, &k, &v, attention_bias, segment_ids, p, &o, &lse, workspace, workspace_bytes, sc));
    RA_TRY(ra_backward(&q, &k, &v, &o, &d_o, &lse, attention_bias, segment_ids, p, &dq, &dk, &dv, workspace,
                       workspace_bytes, sc));
    RA_TRY(cuda_fail(cudaEventRecord(done, sc), "cudaEventRecord"));
    RA_TRY(cuda_fail(cudaStreamWaitEvent(so, done, 0), "cudaStreamWaitEvent (d2h stream)"));
    const ra_tensor* out_d[] = {&t->dev_o, &t->dev_dq, &t->dev_dk, &t->dev_dv};
    const ra_tensor* out_h[] = {&t->o, &t->dq, &t->dk, &t->dv};
    for (int i = 0; i < 4; ++i)
      RA_TRY(cuda_fail(copy_heads(*out_h[i], *out_d[i], h0, hg, cudaMemcpyDeviceToHost, so), "cudaMemcpy2DAsync (d2h)"));
    RA_TRY(cuda_fail(copy_heads_bhs(t->lse, t->dev_lse, h0, hg, cudaMemcpyDeviceToHost, so), "cudaMemcpy2DAsync (d2h)"));
  }
  cudaEvent_t fin = pool.make();
  if (!fin) return cuda_fail(cudaGetLastError(), "cudaEventCreateWithFlags");
  RA_TRY(cuda_fail(cudaEventRecord(fin, so), "cudaEventRecord"));
  RA_TRY(cuda_fail(cudaStreamWaitEvent(sc, fin, 0), "cudaStreamWaitEvent (compute stream)"));
  return RA_OK;
}

int ra_selftest_timeout(int64_t budget_cycles, void* stream) {
  if (budget_cycles < 1000 || budget_cycles > 1000000000ll) return RA_ERR_UNSUPPORTED;
  int* ptr = nullptr;
  RA_TRY(cuda_fail(cudaGetSymbolAddress(reinterpret_cast<void**>(&ptr), g_ra_selftest_result),
                   "cudaGetSymbolAddress (self-test word)"));
  selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(budget_cycles, ptr);
  return last_cuda();
}

#ifdef RA_DEBUG_COUNT
namespace {
// MUFU ex2 throughput: 8 independent ex2 chains per thread (an FADD keeps
// each chain bounded near -1); one CTA per SM records its cycle count.
__global__ void __launch_bounds__(512, 1) debug_ex2_rate_kernel(int iters, long long* cycles, float* sink) {
  float x[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) x[j] = -0.125f * (float)(j + 1) - 1e-3f * (float)threadIdx.x;
  __syncthreads();
  const long long t0 = clock64();
  for (int i = 0; i < iters; ++i) {
#pragma unroll
    for (int j = 0; j < 8; ++j) x[j] = ex2_approx(x[j]) - 1.5f;
  }
  __syncthreads();
  const long long t1 = clock64();
  float acc = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) acc += x[j];
  if (acc == 12345.f) sink[threadIdx.x] = acc;   // keeps the chains live
  if (threadIdx.x == 0) cycles[blockIdx.x] = t1 - t0;
}
}  // namespace

int ra_debug_ex2_rate(int32_t iters, int32_t blocks, long long* cycles, float* sink, void* stream) {
  if (!cycles || !sink) return RA_ERR_NULL;
  if (iters < 1 || blocks < 1) return RA_ERR_SHAPE;
  debug_ex2_rate_kernel<<<(unsigned)blocks, 512, 0, static_cast<cudaStream_t>(stream)>>>(iters, cycles, sink);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

int ra_debug_bounds(uint64_t* first_hit) {
  if (!first_hit) return RA_ERR_NULL;
  unsigned long long v = 0;
  RA_TRY(cuda_fail(cudaMemcpyFromSymbol(&v, ra::g_ra_bounds_hit, sizeof(v)), "cudaMemcpyFromSymbol (index-check word)"));
  const unsigned long long zero = 0;
  RA_TRY(cuda_fail(cudaMemcpyToSymbol(ra::g_ra_bounds_hit, &zero, sizeof(zero)), "cudaMemcpyToSymbol (index-check word)"));
  *first_hit = v;
  return RA_OK;
}

int ra_debug_set_counts(int32_t* fwd_row_counts, int32_t* bwd_col_counts) {
  g_dbg_fwd_rows = fwd_row_counts;
  g_dbg_bwd_cols = bwd_col_counts;
  return RA_OK;
}
#endif

int ra_get_device_status(void* stream) {
  RA_TRY(cuda_fail(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)), "cudaStreamSynchronize"));
  int v = 0;
  RA_TRY(cuda_fail(cudaMemcpyFromSymbol(&v, ra::g_ra_status, sizeof(int)), "cudaMemcpyFromSymbol (status word)"));
  const int zero = 0;
  RA_TRY(cuda_fail(cudaMemcpyToSymbol(ra::g_ra_status, &zero, sizeof(int)), "cudaMemcpyToSymbol (status word)"));
  return v;
}

const char* ra_last_error_message(void) { return t_last_error; }

int64_t ra_count_visible_pairs(int64_t B, int64_t S, int64_t H, int64_t causal_block_size, const int32_t* seg_host,
                               const float* bias_host) {
  if (B < 0 || S < 0 || H < 0 || causal_block_size < 0) return -1;
  int64_t total = 0;
  for (int64_t b = 0; b < B; ++b) {
    const int32_t* sg = seg_host ? seg_host + b * S : nullptr;
    const float* bs = bias_host ? bias_host + b * S : nullptr;
    std::unordered_map<int32_t, int64_t> cnt;   // visible-key count per segment id so far
    auto key_ok = [&](int64_t j) { return !bs || bs[j] > -INFINITY; };
    const int64_t c = causal_block_size > 0 ? causal_block_size : S;
    for (int64_t a = 0; a < S; a += c) {
      const int64_t e = a + c < S ? a + c : S;
      for (int64_t j = a; j < e; ++j)        // keys of this causal block become visible
        if (key_ok(j)) ++cnt[sg ? sg[j] : 0];
      for (int64_t i = a; i < e; ++i) {      // queries of the block see every key so far
        auto f = cnt.find(sg ? sg[i] : 0);
        if (f != cnt.end()) total += f->second;
      }
    }
  }
  return total * H;
}

int64_t ra_ring_schedule(int64_t S, const ra_params* p, int64_t q_first, int64_t q_last, const int32_t* seg_host,
                         const float* bias_host, int32_t* out_host, int64_t cap) {
  RingDesc rd;
  if (S < 1 || make_ring(p, S, &rd) != RA_OK) return -1;
  if (q_first < 0 || q_last < q_first || q_first >= S) return -1;
  std::vector<int4> meta;
  if (seg_host || bias_host) {
    meta.resize(rd.ntiles);
    for (int32_t t = 0; t < rd.ntiles; ++t) {
      int smin = INT32_MAX, smax = INT32_MIN, any = 0, zero = 1;
      for (int64_t j = (int64_t)t * kTile; j < S && j < (int64_t)(t + 1) * kTile; ++j) {
        const int s = seg_host ? seg_host[j] : 0;
        smin = s < smin ? s : smin;
        smax = s > smax ? s : smax;
        if (bias_host) {
          any |= bias_host[j] > -INFINITY;
          zero &= bias_host[j] == 0.0f;
        } else {
          any = 1;
        }
      }
      meta[t] = make_int4(smin, smax, (any ? kMetaAnyFinite : 0) | (zero ? kMetaAllZero : 0), 0);
    }
  }
  KvIter it;
  kv_iter_init(it, rd, q_first, q_last, meta.empty() ? nullptr : meta.data(), seg_host != nullptr,
               bias_host != nullptr);
  int64_t n = 0;
  for (int32_t t = kv_iter_next(it, rd); t >= 0; t = kv_iter_next(it, rd)) {
    if (out_host && n < cap) out_host[n] = t;
    ++n;
  }
  return n;
}

}  // extern "C"
