/*
 * bd_attn_debug.h -- test hooks of libbdattn.so (no counterpart on the
 * source pages): the failure-detection path, the grid size of the
 * persistent kernels, the forward kernel selected, and the work counters.
 *
 * Every wait inside the tensor-core kernels is bounded: when one runs out,
 * the kernel records BD_ERR_DEVICE_TIMEOUT in the device status word (read
 * by bd_attn_get_device_status), the affected CTA leaves its loops, waits
 * (bounded) for its own copies and tensor-core operations in flight, frees
 * its tensor memory and exits; nothing faults, traps or hangs.  This hook
 * makes that path run on purpose.
 */
#ifndef BD_ATTN_DEBUG_H
#define BD_ATTN_DEBUG_H

#include "bd_attn.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Arms a one-shot fault on the current device: in the next launch of the
 * tcgen05 kernel (bd_attn_fwd or bd_attn_decode with d = 128 or 64), CTA 0
 * skips the copy of its first K tile, so the wait for that tile runs out
 * after about two seconds and the launch reports BD_ERR_DEVICE_TIMEOUT.
 * The outputs of that launch are undefined; later launches are unaffected.
 * kind: 0 disarms, 1 arms.  Returns BD_OK, BD_ERR_INVALID_ARG for another
 * kind, or BD_ERR_CUDA.
 */
BD_API bd_status bd_attn_debug_inject_fault(int kind);

/*
 * Caps the grid of the persistent tcgen05 kernels (bd_attn_fwd and
 * bd_attn_decode with d = 128 or 64) at `ctas` CTAs for every later launch from
 * any thread, so tests can run the forward's dynamic hand-out and the
 * decode's stream-K split and combine at grid sizes other than one CTA per
 * SM.  ctas = 0 restores the default (one CTA per SM, at most 148).
 * Results are the same at any grid size up to rounding order.  Returns
 * BD_OK, or BD_ERR_INVALID_ARG for ctas < 0 or ctas > 148.
 */
BD_API bd_status bd_attn_debug_set_grid(int ctas);

/*
 * Fixes the chunk size of the persistent kernels' work lists for every later
 * launch from any thread: `groups` heads (head pairs in the paired forward
 * kernel) per chunk of the forward and dQ lists, and `groups` (batch,
 * kv-head) groups per chunk of the clean key tiles in the dK/dV list.  Each
 * list runs chunk by chunk, heaviest item first inside a chunk, so tests can
 * run several chunks and a ragged last one on small sizes.  groups = 0
 * restores the default (forward and dQ: as many as keep the chunk's K/V
 * within 64 MB; dK/dV: 8).  Results are the same for any chunk size up to
 * rounding order.  Returns BD_OK, or BD_ERR_INVALID_ARG for groups < 0.
 */
BD_API bd_status bd_attn_debug_set_chunk(int groups);

/*
 * Which kernel bd_attn_fwd runs for these sizes on the current device:
 * 2 = tcgen05 kernel with two query heads of a GQA group per CTA (even group
 * size), 1 = tcgen05 kernel with one query tile per CTA (odd group size, or
 * the paired kernel's register split unavailable), -1 = sizes bd_attn_fwd
 * rejects.  (0, an mma.sync kernel, is no longer returned: every head dim
 * runs on the tcgen05 kernels.)
 * Needs the CUDA runtime (it reads the compiled kernel's attributes).
 */
BD_API int bd_attn_debug_fwd_kernel(int Hq, int Hkv, int d);

/*
 * Synchronises the current device, then zeroes every work-counter pair of
 * the persistent kernels (item counter, finished-CTA counter, claim
 * counter).  For tests that run overlapping launches on one pair on
 * purpose: the pair's counts are then mixed, and its next user would take
 * wrong items.  Returns BD_OK or BD_ERR_CUDA.
 */
BD_API bd_status bd_attn_debug_reset_sched(void);

#ifdef __cplusplus
}
#endif

#endif /* BD_ATTN_DEBUG_H */
