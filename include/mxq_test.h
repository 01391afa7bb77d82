/* mxq_test.h -- test-only hooks of libmxq.so.  Not part of the conversion
 * API (include/mxq.h); they exist so that tests can show, without faulting
 * or hanging the GPU, that the library's failure paths answer as specified.
 */
#ifndef MXQ_TEST_H
#define MXQ_TEST_H

#include "mxq.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Make the next single-pass NVFP4 launch stall on purpose.  On several
 * groups (mxq_quantize_nvfp4 where the single-pass kernel holds the shape)
 * its per-SM publisher never releases a group; on one group read once by a
 * grid of CTAs (a tile too large for one cluster that fits the SMs' shared
 * memory) the first CTA never reports its amax.  Either way every inter-CTA
 * wait of that launch runs into its iteration limit.  The launch then ORs
 * MXQ_DEV_WAIT_TIMEOUT into *status, lets its copies in flight land and
 * returns, well under a second; the outputs of that call are undefined and
 * the device stays usable.  `on` = 0 withdraws a pending request.  The
 * request is taken by exactly one launch (the next one of any thread of the
 * process); it is ignored by the other kernels. */
MXQ_API void mxq_test_stall_next_single_pass(int on);

#ifdef __cplusplus
}
#endif

#endif /* MXQ_TEST_H */
