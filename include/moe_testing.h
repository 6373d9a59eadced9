/*
 * moe_testing.h - test-only control of the library's failure paths.
 *
 * The page articles have no counterpart to this: it exists so that a test can
 * make one of the kernels' bounded waits run out on a GPU without faulting,
 * trapping or hanging it, and check that the call reports MOE_ERR_TIMEOUT and
 * that the device stays usable.
 */
#ifndef MOE_TESTING_H
#define MOE_TESTING_H

#include "moe.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Arm (cta >= 0) or clear (cta < 0) a stall for the next launches of the
 * mat-vec kernel (moe_ffn / moe_mul_mat_id at decode sizes, and
 * moe_ffn_decode_noalloc) on this process: the weight producer of CTA `cta`
 * does not issue its ring stage number `stage` (counted from 0 across its work
 * items) - no copy is started for it, so none is in flight when the CTA leaves
 * - and every bounded wait of those launches gives up after `wait_us`
 * microseconds instead of about two seconds.  A consumer of that CTA then
 * waits for data that never comes; its wait expires, the status word gets
 * MOE_ERR_TIMEOUT and header word 3 the expired wait's site (1<<30 | warp<<20
 * | shared-memory offset of its barrier); every role of the CTA leaves its loop
 * and the launch ends.
 *
 * The same stall applies to the grouped GEMM (moe_ffn / moe_mul_mat_id above
 * the mat-vec threshold): the activation producer of CTA `cta` does not issue
 * the copy of its k-step number `stage` (counted from 0 across its tiles), and
 * every bounded wait of those launches gives up after `wait_us` microseconds.
 * The warp that waits for the MMA warp's operands then gives up, hands the
 * failure to the MMA warp through their named barrier, and the launch ends the
 * same way (status MOE_ERR_TIMEOUT, the site in header word 3).  Not
 * thread-safe; not for production use.
 */
MOE_API void moe_testing_stall(int cta, int stage, int wait_us);

#ifdef __cplusplus
}
#endif
#endif /* MOE_TESTING_H */
