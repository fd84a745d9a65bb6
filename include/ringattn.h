/*
 * ringattn.h — C ABI of a B200 (sm_100a) implementation of Ring Attention's
 * blockwise *exact* attention, with the P ring ranks virtual on one GPU.
 *
 * Method (pages describing Ring Attention, cited by title and section):
 *  - "Ring Attention技术解析：突破大模型长上下文训练瓶颈" §2.2: the sequence is
 *    cut into P blocks; devices form a ring; each device sends its key/value
 *    block to the next device and receives the previous one's.
 *  - "手把手拆解RingAttention：如何用分布式计算突破百万token长视频处理瓶颈" §1:
 *    queries stay, keys/values travel, and global attention is kept complete
 *    (complexity table, row "RingAttention").  So the result is exactly
 *    full softmax attention; partials are combined by an online softmax
 *    (running max, running sum, rescale) / log-sum-exp merge.
 *  - "RingAttention核心功能全解析", 核心API调用 and 核心技术原理 1: the call
 *    ringattention(xq, xk, xv, attention_bias, segment_ids, blockwise_kwargs=
 *    {query_chunk_size, key_chunk_size, causal_block_size, policy}); the
 *    policy "nothing_saveable" means the backward recomputes attention from
 *    the inputs (here: from the saved log-sum-exp).
 *
 * Conventions for every entry point
 *  - Tensors are described by ra_tensor: a pointer plus dtype, rank, shape
 *    and strides in ELEMENTS.  Data pointers are DEVICE pointers unless a
 *    parameter says "host".  The caller owns every buffer; the library never
 *    allocates device memory.  Its device-side state is one status word per
 *    device, one word written by ra_selftest_timeout, and the fixed scratch
 *    array of ra_forward_static (see there for how calls share it).
 *  - q, k, v, o, dO, dq, dk, dv are [B, S, H, D] (batch, token, head, head
 *    dim); the head dim must be contiguous (stride 1) and D in {64, 128}.
 *    bf16 tensors additionally need 16-byte aligned base pointers and
 *    strides whose byte size is a multiple of 16 (they are read by TMA).
 *  - lse, m, l are fp32 [B, H, S] (any strides).  LSE is in natural-log
 *    units; a query row with no visible key has o = 0 and lse = -inf.
 *  - attention_bias: NULL or fp32 [B, S]: additive bias per KEY, broadcast
 *    over heads and queries; -inf masks the key.
 *  - segment_ids: NULL or int32 [B, S]: a key is visible only to queries
 *    with the same id.
 *  - Masking uses global token positions: with causal_block_size c >= 1,
 *    key j is visible to query i iff floor(i/c) >= floor(j/c); c = 0 means
 *    non-causal.  Softmax scale is 1/sqrt(D).
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream).  Arguments, tensor maps and kernel attributes are
 *    checked and prepared before the first launch, so an error found there
 *    returns with nothing queued; only RA_ERR_CUDA from a failed launch can
 *    follow launches already queued.  After a non-zero return the outputs
 *    are unspecified.  No exception or exit crosses the ABI.
 *  - Errors detected on the device (a bounded wait that ran out) are
 *    recorded in the device status word; ra_get_device_status() reads it.
 *  - Every call that launches work makes the device that holds its tensors
 *    current for the calling thread (cudaSetDevice), which also makes that
 *    device's primary context current: the calls work from threads that have
 *    made no CUDA call yet (for example an autograd worker thread).
 */
#ifndef RINGATTN_H_
#define RINGATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { RA_F32 = 0, RA_BF16 = 1, RA_I32 = 2 } ra_dtype;

enum {
  RA_OK = 0,
  RA_ERR_NULL = 1,           /* a required pointer is NULL */
  RA_ERR_DTYPE = 2,          /* dtype not allowed for this argument, or inputs disagree */
  RA_ERR_SHAPE = 3,          /* rank or shape mismatch between arguments */
  RA_ERR_STRIDE = 4,         /* head dim not contiguous, or TMA alignment rules violated */
  RA_ERR_DIVISIBILITY = 5,   /* S % ring_size, (S/ring_size) % chunk, or a size < 1 */
  RA_ERR_UNSUPPORTED = 6,    /* D not in {64,128}, ring_size > 64, or bf16 path on a non-sm_100 device */
  RA_ERR_WORKSPACE = 7,      /* workspace NULL or smaller than ra_workspace_size() */
  RA_ERR_CUDA = 8,           /* a CUDA runtime call failed (launch, attribute, tensor map) */
  RA_ERR_DEVICE_TIMEOUT = 9, /* device-side bounded wait ran out (reported by ra_get_device_status) */
  RA_ERR_ORDER = 10,         /* ring_order is not a permutation of 0..ring_size-1 */
  RA_ERR_STATIC_LIMIT = 11   /* problem needs more scratch than ra_forward_static's fixed array */
};

typedef struct {
  void* data;         /* device pointer (see each entry point) */
  int32_t dtype;      /* ra_dtype */
  int32_t ndim;       /* number of valid entries in shape / stride */
  int64_t shape[4];
  int64_t stride[4];  /* in elements */
} ra_tensor;

#define RA_MAX_RING 64

typedef struct {
  /* blockwise_kwargs of "RingAttention核心功能全解析" 核心技术原理 1: chunk sizes
   * group the hardware's 128-token tiles; each must be >= 1 and divide S /
   * ring_size.  They do not change the (exact) result. */
  int64_t query_chunk_size;
  int64_t key_chunk_size;
  /* 0 = non-causal; c >= 1: block-causal with block c (1 = ordinary causal). */
  int64_t causal_block_size;
  /* P, the number of virtual ring ranks; 1 <= P <= 64 and S % P == 0. */
  int64_t ring_size;
  /* If use_ring_order != 0, step t visits key/value block
   * (r - ring_order[t]) mod P instead of (r - t) mod P; ring_order must be a
   * permutation of 0..P-1 (RA_ERR_ORDER otherwise). */
  int32_t ring_order[RA_MAX_RING];
  int32_t use_ring_order;
  int32_t reserved;   /* must be 0 */
  /* Optional profiling hooks: two cudaEvent_t handles (or NULL).  When both
   * are set, ra_forward / ra_backward record them on `stream` immediately
   * before and after their main attention kernel, so a caller can time that
   * kernel alone (preprocessing and conversion launches excluded). */
  void* prof_event_begin;
  void* prof_event_end;
} ra_params;

/* Workspace bytes (device memory, caller-allocated, 256-byte aligned base)
 * needed by ra_forward (which = 0) or ra_backward (which = 1) for a problem
 * shaped like q.  has_bias / has_segments say whether attention_bias /
 * segment_ids will be passed.  Returns 0 when none is needed, or
 * (size_t)-1 for invalid arguments. */
size_t ra_workspace_size(int which, const ra_tensor* q, const ra_params* p, int has_bias, int has_segments);

/* Forward: o = softmax(q k^T / sqrt(D) + bias, masked) v and its
 * log-sum-exp, every query tile visiting the key/value tiles in ring order
 * ("Ring Attention技术解析" §2.2) with the exact online-softmax merge.
 *  q, k, v: [B,S,H,D], all bf16 (sm_100a tensor-core path) or all fp32
 *           (CUDA-core fp32 path).
 *  attention_bias, segment_ids: may be NULL (see conventions).
 *  o: [B,S,H,D], dtype of q (bf16 rounded to nearest even).  lse: fp32 [B,H,S].
 *  workspace: device buffer of at least ra_workspace_size(0, ...) bytes
 *  (may be NULL when that size is 0).  Contents are scratch. */
int ra_forward(const ra_tensor* q, const ra_tensor* k, const ra_tensor* v, const ra_tensor* attention_bias,
               const ra_tensor* segment_ids, const ra_params* p, ra_tensor* o, ra_tensor* lse, void* workspace,
               size_t workspace_bytes, void* stream);

/* Backward of ra_forward given the upstream gradient dO, recomputing the
 * attention probabilities from q, k and the saved lse (the recompute policy
 * "nothing_saveable" of "RingAttention核心功能全解析" 核心API调用):
 *   Delta_i = <dO_i, o_i>, P_ij = exp(s_ij - lse_i), dP_ij = <dO_i, v_j>,
 *   dS_ij = P_ij (dP_ij - Delta_i), dq = dS k / sqrt(D), dk = dS^T q / sqrt(D),
 *   dv = P^T dO.
 *  q, k, v, o, d_o: same dtype (bf16 or fp32), [B,S,H,D]; lse fp32 [B,H,S]
 *  as written by ra_forward.  dq, dk, dv: [B,S,H,D] (bf16 or fp32; with
 *  fp32 inputs they must be fp32).  workspace: at least
 *  ra_workspace_size(1, ...) bytes (holds Delta and an fp32 dq accumulator). */
int ra_backward(const ra_tensor* q, const ra_tensor* k, const ra_tensor* v, const ra_tensor* o,
                const ra_tensor* d_o, const ra_tensor* lse, const ra_tensor* attention_bias,
                const ra_tensor* segment_ids, const ra_params* p, ra_tensor* dq, ra_tensor* dk, ra_tensor* dv,
                void* workspace, size_t workspace_bytes, void* stream);

/* One ring step ("Ring Attention技术解析" §2.2, one iteration of the loop):
 * the local query block q_blk [B,Sq,H,D] (tokens q_off .. q_off+Sq-1 of the
 * sequence) attends to one visiting key/value block k_blk, v_blk [B,Sk,H,D]
 * (tokens k_off ..), updating the caller-held running state in place:
 *   o_acc fp32 [B,Sq,H,D] (unnormalised output), m, l fp32 [B,H,Sq]
 *   (reference max in natural-log units, running sum), with
 *   o_acc = sum_j e^(s_j - m) v_j and l = sum_j e^(s_j - m) over the keys
 *   seen so far.
 * Initialise m = -inf, l = 0, o_acc = 0 before the first step; any step
 * order gives the same finalized result (ra_finalize).  bias_blk: NULL or
 * fp32 [B,Sk] for the visiting keys; seg_q / seg_k: both NULL or int32
 * [B,Sq] / [B,Sk].  Only p->causal_block_size is used from p; masks compare
 * global positions.  m and l must have identical strides.
 *  - The key/value side (k_blk, v_blk, bias_blk, seg_k) may have batch 1
 *    while q_blk has batch B: that one block is then shared by every query
 *    batch row, e.g. a cached prefix common to B requests ("Ring
 *    Attention技术解析" §7: requests with the same prefix share its cache). 
 *  - bf16 q/k/v: tensor cores (the forward kernel in ring-step mode: TMA
 *    K/V stages, tcgen05 S = Q K^T and O += P V, exp2 online softmax), the
 *    block's partial merged into the state in the kernel's epilogue.  o_acc
 *    needs a 16-byte aligned base and 16-byte multiple strides.  m may sit
 *    up to 8 ln 2 below the true running max (the kernel moves its
 *    reference max lazily); l and o_acc are scaled to match, so the state
 *    finalizes to the same result.
 *  - fp32 q/k/v: CUDA cores in fp32 with accurate expf; m is the true max. */
int ra_step(const ra_tensor* q_blk, const ra_tensor* k_blk, const ra_tensor* v_blk, int64_t q_off, int64_t k_off,
            const ra_tensor* bias_blk, const ra_tensor* seg_q, const ra_tensor* seg_k, const ra_params* p,
            ra_tensor* o_acc, ra_tensor* m, ra_tensor* l, void* stream);

/* Finalize a running state: o = o_acc / l (bf16 or fp32 output), lse = m +
 * log(l); rows with l == 0 give o = 0 and lse = -inf. */
int ra_finalize(const ra_tensor* o_acc, const ra_tensor* m, const ra_tensor* l, ra_tensor* o, ra_tensor* lse,
                void* stream);

/* Merge two normalised partial results computed over disjoint key sets:
 *   lse = max(a,b) + log1p(exp(-|lse_a - lse_b|)),
 *   o   = o_a exp(lse_a - lse) + o_b exp(lse_b - lse).
 * o_* [B,S,H,D] (all bf16 or all fp32), lse_* fp32 [B,H,S].  o_out / lse_out
 * may alias o_a / lse_a (element-wise in place). */
int ra_lse_merge(const ra_tensor* o_a, const ra_tensor* lse_a, const ra_tensor* o_b, const ra_tensor* lse_b,
                 ra_tensor* o_out, ra_tensor* lse_out, void* stream);

/* Blockwise feed-forward network, exported next to ringattention
 * ("RingAttention核心功能全解析" 核心API调用: from ringattention import
 * ringattention, blockwise_feedforward).  The page prints no formula; the
 * reading taken is the position-wise feed-forward network of the LLaMA
 * configuration the page shards, a SwiGLU without biases:
 *   h_t = silu(x_t W1^T) * (x_t W3^T),  y_t = h_t W2^T,  silu(a) = a / (1 + e^-a),
 * evaluated chunk_size tokens at a time, so only one chunk's h [chunk, d_ff]
 * (bf16, in `workspace`) is ever held: memory linear in the sequence length.
 * Both products run on the tensor cores (bf16 in, fp32 accumulate); h is
 * rounded to bf16 between them, y to bf16 at the end.
 *  x: bf16 [T, d_model]; w1, w3: bf16 [d_ff, d_model]; w2: bf16 [d_model, d_ff]
 *  (weights output-major, like a linear layer's); y: bf16 [T, d_model].  Rows
 *  contiguous (stride[1] = 1), 16-byte aligned bases and row strides;
 *  d_model and d_ff multiples of 32.
 *  workspace: device, at least ra_feedforward_workspace_size(chunk_size, d_ff)
 *  bytes, 256-byte aligned. */
size_t ra_feedforward_workspace_size(int64_t chunk_size, int64_t d_ff);
int ra_feedforward(const ra_tensor* x, const ra_tensor* w1, const ra_tensor* w3, const ra_tensor* w2, ra_tensor* y,
                   int64_t chunk_size, void* workspace, size_t workspace_bytes, void* stream);

/* Forward that allocates nothing, for callers that cannot allocate device
 * memory: a host program that links only this library and owns no device
 * allocator, or code running under a fixed, pre-planned memory budget where a
 * cudaMalloc could fail or implicitly synchronize the device.  The paper has
 * no counterpart for this entry point: it is an addition of this library.
 * Same arguments, semantics and results as ra_forward minus the workspace:
 * the scratch ra_forward would take from `workspace` (per-128-token tile
 * metadata, used only when attention_bias or segment_ids is given) lives in
 * one file-scope device array of RA_STATIC_SCRATCH_BYTES (1 MiB), enough for
 * B * ceil(S / 128) <= 65536 (for example B = 8 at 1M tokens).  Larger
 * problems return RA_ERR_STATIC_LIMIT and launch nothing.
 *  - The array is held by every GPU that loads the library until the process
 *    exits.  Each call looks up the array's device address in the current
 *    context (cudaGetSymbolAddress), so the address stays right after a
 *    context is destroyed and created again.  The first call on a device may
 *    load the library's device code; make that first call before any stream
 *    capture.
 *  - Every call shares the array and it keeps the last call's contents.  All
 *    of it that a call reads is rewritten by that call first, so nothing has
 *    to be cleared, but calls that overlap on the GPU (concurrent streams)
 *    race on it: serialize them. */
#define RA_STATIC_SCRATCH_BYTES (1u << 20)
int ra_forward_static(const ra_tensor* q, const ra_tensor* k, const ra_tensor* v, const ra_tensor* attention_bias,
                      const ra_tensor* segment_ids, const ra_params* p, ra_tensor* o, ra_tensor* lse, void* stream);

/* Tensors of one training step whose inputs and outputs live in HOST memory
 * (ra_train_step_host).  Host tensors should be page-locked (cudaHostAlloc /
 * pinned torch tensors) for the copies to overlap with the kernels.  Every
 * tensor here must be contiguous: [B,S,H,D] row-major for q .. dv and their
 * device twins, [B,H,S] for lse. */
typedef struct {
  ra_tensor q, k, v, d_o;                 /* HOST inputs, [B,S,H,D], bf16 or fp32 */
  ra_tensor o, lse, dq, dk, dv;           /* HOST outputs: o, dq, dk, dv like q; lse fp32 [B,H,S] */
  ra_tensor dev_q, dev_k, dev_v, dev_do;  /* DEVICE staging, same shapes and dtypes as the host twins */
  ra_tensor dev_o, dev_lse, dev_dq, dev_dk, dev_dv;
} ra_host_step;

/* Forward and backward of one training step with every input and output in
 * host memory: the end-to-end call of a training loop that keeps its
 * tensors on the host.  The definition computes every (batch, head) pair
 * independently, so the step is cut into groups of heads_per_group heads
 * and pipelined over
 * three streams: the host->device copy of group g+1 (h2d_stream) runs while
 * the kernels of group g run (compute_stream), and the device->host copy of
 * group g-1's results (d2h_stream) runs beside both.  Per group the work is
 * exactly ra_forward followed by ra_backward on that group's heads, so the
 * results equal those two calls on the whole tensors.
 *  t: the tensors (see ra_host_step); dq, dk, dv take the dtype of q.
 *  attention_bias / segment_ids: NULL or DEVICE tensors as in ra_forward.
 *  heads_per_group: >= 1 and divides H.
 *  workspace: DEVICE, at least ra_workspace_size(1, q', p, ...) bytes for q'
 *  = q with H replaced by heads_per_group (reused by every group).
 *  Streams may coincide (then nothing overlaps).  The call is asynchronous;
 *  compute_stream is made to wait for the last device->host copy, so
 *  synchronizing compute_stream covers the whole step.  Calls using the
 *  same buffers are serialized through compute_stream.  The library creates
 *  and releases CUDA events inside the call and allocates no memory.
 *  Returns the first error of any part; outputs are then unspecified, and
 *  part of the step may already have been queued. */
int ra_train_step_host(const ra_host_step* t, const ra_tensor* attention_bias, const ra_tensor* segment_ids,
                       const ra_params* p, int64_t heads_per_group, void* workspace, size_t workspace_bytes,
                       void* compute_stream, void* h2d_stream, void* d2h_stream);

/* Synchronizes `stream`, returns the device status word of the current
 * device (RA_OK or RA_ERR_DEVICE_TIMEOUT) and clears it.  RA_ERR_CUDA if
 * the synchronization itself failed. */
int ra_get_device_status(void* stream);

/* Failure-path self-test: launches one warp that waits, through the same
 * bounded mbarrier wait the attention kernels use, on a barrier phase that
 * nothing ever completes.  After budget_cycles clock cycles (1e3 .. 1e9) the
 * wait gives up, records RA_ERR_DEVICE_TIMEOUT in the device status word and
 * the kernel returns normally; read the result with ra_get_device_status().
 * No fault, trap or hang is involved: the device context stays usable.
 * Returns RA_ERR_UNSUPPORTED for a budget outside the range. */
int ra_selftest_timeout(int64_t budget_cycles, void* stream);

/* Static description of an error code (never NULL). */
const char* ra_strerror(int code);

/* The CUDA call and error behind the most recent RA_ERR_CUDA returned to
 * the calling thread, as text (for example "kernel launch: invalid argument
 * (cudaErrorInvalidValue, 1)"); an empty string if there was none.  The
 * pointer is to thread-local storage, valid until the thread's next call
 * into the library. */
const char* ra_last_error_message(void);

/* Host-only introspection (no device work).
 * Exact number of visible (query, key) pairs summed over batch and heads,
 * from the same mask rules the kernels use.  seg_host: NULL or int32 [B*S]
 * row-major (host memory); bias_host: NULL or fp32 [B*S] (host).  Returns
 * -1 on invalid arguments. */
int64_t ra_count_visible_pairs(int64_t B, int64_t S, int64_t H, int64_t causal_block_size,
                               const int32_t* seg_host, const float* bias_host);

/* Host-only introspection: the key/value tile indices (128-token tiles),
 * in visiting order, that the query rows [q_first, q_last] of batch row 0
 * visit on the ring: step t covers the tiles of block (r - order[t]) mod P,
 * r = q_first's ring block; tiles that masking hides from every row of the
 * range are skipped.  seg_host / bias_host as in ra_count_visible_pairs
 * (batch row 0 only).  Writes at most `cap` indices to out_host and returns
 * the full count, or -1 on invalid arguments. */
int64_t ra_ring_schedule(int64_t S, const ra_params* p, int64_t q_first, int64_t q_last, const int32_t* seg_host,
                         const float* bias_host, int32_t* out_host, int64_t cap);

#ifdef __cplusplus
}
#endif

#endif /* RINGATTN_H_ */
