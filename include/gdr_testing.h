/*
 * gdr_testing.h -- test-only entry points of the gated delta-rule library.
 *
 * These exist so that tests can exercise the library's failure reporting on
 * a GPU without faulting, trapping or hanging it.  The method described by
 * the pages has no counterpart.  Not for production use.
 */
#ifndef GDR_TESTING_H_
#define GDR_TESTING_H_

#include "gdr.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Makes the NEXT gdr_chunk_fwd call on this host thread that runs on the
 * tensor-core path (bf16, scalar gate, d_k = d_v = 128) skip issuing the input
 * load of chunk `chunk`.  The waits for that chunk's data give up after their
 * bound (about 2 s), every CTA unwinds (in-flight copies and MMAs drained,
 * TMEM freed) and the device status word reports GDR_ERR_TIMEOUT, which
 * gdr_get_device_status() returns.  The outputs of that call are undefined;
 * the CUDA context stays usable.  Only the next call is affected.
 * Returns GDR_ERR_INVALID_ARG for chunk < 0, else GDR_OK.
 */
gdr_status gdr_testing_skip_stage_load(int chunk);

#ifdef __cplusplus
}
#endif

#endif /* GDR_TESTING_H_ */
