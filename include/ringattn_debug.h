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

#ifdef __cplusplus
}
#endif

#endif /* RINGATTN_DEBUG_H */
