/*
 * ringattn_debug.h — extra entry point of the debug build of the library
 * (compiled with -DRA_DEBUG_COUNT into libringattn_count.so; the release
 * libringattn.so neither declares nor exports it).
 *
 * Purpose: the masks must be exact, integer decisions.  The pages fix which
 * pairs take part ("RingAttention核心功能全解析", 核心API调用: causal_block_size
 * and segment_ids; 核心技术原理 1: attention_bias), and the attention is
 * complete over those pairs ("手把手拆解RingAttention…", §1, complexity table,
 * row "RingAttention").  In the debug build the tensor-core kernels count,
 * for every row they own, the pairs their own tile skipping and per-element
 * masking let into the softmax (a score that is still finite there), so a
 * test can compare those counts bit for bit with an integer reference.
 * It also carries a MUFU exp2 throughput microbenchmark, and index checks:
 * in this build every kernel tests each index it computes for a global or
 * shared-memory access against its extent before the access (TMA copies
 * excepted: their tensor maps bound them).  An index out of range skips the
 * access and is recorded; see ra_debug_bounds.  (The sanitizer tools are not
 * available where this library is tested; these checks stand in for their
 * out-of-bounds detection on the paths the tests drive.)
 */
#ifndef RINGATTN_DEBUG_H
#define RINGATTN_DEBUG_H

#include <stdint.h>

#include "ringattn.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Sets (or, with NULL, clears) the count buffers used by every later
 * ra_forward / ra_backward call of this process that takes the tensor-core
 * path (bf16 q/k/v, D = 64 or 128).
 *  - fwd_row_counts: DEVICE int32 [B, H, S], contiguous: for each query row,
 *    the number of keys the forward kernel let into its softmax.  Every row
 *    below S is overwritten by each forward call.
 *  - bwd_col_counts: DEVICE int32 [B, H, S], contiguous: for each key, the
 *    number of query rows the backward kernel paired it with.  The kernel
 *    ADDS to it, so the caller zeroes it before each backward call.
 * The caller owns both buffers and keeps them alive while calls that use
 * them run; the shapes must match those calls' B, H and S (not checked).
 * A process-wide setting: not for concurrent use from several threads.
 * Always returns RA_OK. */
int ra_debug_set_counts(int32_t* fwd_row_counts, int32_t* bwd_col_counts);

/* MUFU exp2 throughput microbenchmark (the forward's co-bound: one ex2 per
 * visible pair).  Launches `blocks` CTAs of 512 threads (one per SM when
 * blocks equals the SM count); each thread runs `iters` rounds of 8
 * independent ex2.approx operations, and CTA i writes its elapsed SM clock
 * cycles to cycles[i] (DEVICE, `blocks` entries).  sink: DEVICE float[512],
 * never read (keeps the work live).  ex2 per clock per SM =
 * 512 * 8 * iters / cycles[i].  RA_ERR_NULL / RA_ERR_SHAPE on bad arguments. */
int ra_debug_ex2_rate(int32_t iters, int32_t blocks, long long* cycles, float* sink, void* stream);

/* Index checks of this build.  Reads the record of the first out-of-range
 * index any kernel of this library met since the previous call (device-wide,
 * first one wins) and clears it.  *first_hit (HOST) = 0 when none was met;
 * otherwise bits 48-63 hold the site and bits 0-47 the index's low 48 bits.
 * Sites:
 *   1 forward: key-tile metadata             2 forward: batch row / head of a CTA
 *   3 forward: query row's segment id         4 forward: key bias
 *   5 forward: key segment id                 6 ring step: running m, l, accumulator row
 *   7 forward: O, LSE and count stores        8 backward: batch row / head of a CTA
 *   9 backward: key row (segment, bias, dK/dV) 10 backward: query-tile metadata
 *  11 backward: query segment ids             12 backward: dS^T shared-memory stores
 *  13 backward: dQ staging stores             14 backward: LSE / Delta rows
 *  15 tile iterators: tile metadata           16 ring-step iterator: visiting keys
 *  17 ring-step iterator: query segment ids   18 tile metadata kernel
 *  19 backward preprocess                     20 dQ conversion
 *  21 finalize and LSE merge                  22 feed-forward output tiles
 * Synchronous with respect to the device (a CUDA memcpy of 8 bytes each way).
 * RA_ERR_NULL for a NULL pointer; RA_ERR_CUDA if a copy fails. */
int ra_debug_bounds(uint64_t* first_hit);

#ifdef __cplusplus
}
#endif

#endif /* RINGATTN_DEBUG_H */
