/*
 * bd_attn_debug.h -- test hook of libbdattn.so for the failure-detection
 * path (no counterpart on the source pages).
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
 * head-dim-128 kernel (bd_attn_fwd or bd_attn_decode with d = 128), CTA 0
 * skips the copy of its first K tile, so the wait for that tile runs out
 * after about two seconds and the launch reports BD_ERR_DEVICE_TIMEOUT.
 * The outputs of that launch are undefined; later launches are unaffected.
 * kind: 0 disarms, 1 arms.  Returns BD_OK, BD_ERR_INVALID_ARG for another
 * kind, or BD_ERR_CUDA.
 */
BD_API bd_status bd_attn_debug_inject_fault(int kind);

#ifdef __cplusplus
}
#endif

#endif /* BD_ATTN_DEBUG_H */
