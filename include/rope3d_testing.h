/*
 * rope3d_testing.h -- test hooks of librope3d.so.  Not for production use: they change
 * process-wide settings of the library for every later launch on every thread.
 */
#ifndef ROPE3D_TESTING_H
#define ROPE3D_TESTING_H

#include <stdint.h>

#include "rope3d.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Kernel path of rope3d_qk_norm_rope_append. */
#define ROPE3D_PATH_AUTO 0       /* the path measured faster for the shape (see rope3d.cu)     */
#define ROPE3D_PATH_REGISTERS 1  /* rows loaded straight into registers                        */
#define ROPE3D_PATH_TMA 2        /* rows streamed through shared memory (EINVAL if it does not fit) */

/*
 * Bounded-wait settings of the bulk-copy ring kernel for later launches:
 * wait_limit_ns replaces the 2 s limit (0 restores it); tx_extra_bytes makes every
 * stage wait for that many bytes more than its copies deliver, so its wait runs out
 * and the kernel reports ROPE3D_ETIMEOUT through rope3d_check_device_status (0 is the
 * normal setting).  No fault is involved: the copies land, the wait simply expires.
 */
ROPE3D_API void rope3d_testing_set_waits(uint64_t wait_limit_ns, uint32_t tx_extra_bytes);

/* Choose the kernel path for later launches (ROPE3D_PATH_*).  EINVAL for other values. */
ROPE3D_API int rope3d_testing_force_path(int path);

/* Form of the QKV projection kernel for later launches: 1 = one CTA per 128x256 tile
 * (tcgen05 cta_group::1), 2 = a pair of CTAs in a cluster per 256x256 tile (cta_group::2,
 * each CTA loading half of the weight rows), 0 = the default (2).  EINVAL otherwise. */
ROPE3D_API int rope3d_testing_gemm_cta_group(int group);

/*
 * Checked build only (librope3d_checked.so; a no-op in librope3d.so): for later launches
 * of the step kernels, the device-side check of a cache row accepts rows below
 * cache_tokens - shrink_rows instead of below cache_tokens.  Rows at or above that bound
 * are then treated as out of extent: the kernel skips all of that token row's stores
 * (q_out, K and V) and records ROPE3D_EINDEX in the status word.  The skipped rows lie
 * inside the caller's buffers, so the check's firing path is exercised without any access
 * outside them.  0 (the default) restores the plain check; negative values are EINVAL.
 */
ROPE3D_API int rope3d_testing_shrink_checked_cache(int64_t shrink_rows);

/*
 * The kernels' 32-bit position decode divides by the token count, H * W, W and the cache
 * length with a multiply-and-shift instead of a divide instruction.  This runs the same
 * arithmetic on the host: floor(n / d) for n < 2^31 and 1 <= d < 2^31, or 0xFFFFFFFF for
 * arguments outside that range.
 */
ROPE3D_API uint32_t rope3d_testing_fast_divide(uint32_t n, uint32_t d);

/* The path (ROPE3D_PATH_REGISTERS or ROPE3D_PATH_TMA) of the calling thread's most recent
 * successful rope3d_qk_norm_rope_append launch; ROPE3D_PATH_AUTO before the first. */
ROPE3D_API int rope3d_testing_last_path(void);

#ifdef __cplusplus
}
#endif

#endif /* ROPE3D_TESTING_H */
