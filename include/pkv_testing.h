/*
 * pkv_testing.h -- test hooks of libpkv.so.  Not part of the decode path and
 * not for production use; the pages have no counterpart.  They let a test
 * drive a kernel's failure handling without faulting the GPU.
 */
#ifndef PKV_TESTING_H_
#define PKV_TESTING_H_

#include <stdint.h>

#include "pkv.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * pkv_testing_prefill_timeout -- arm a timeout for the NEXT pkv_paged_prefill
 * call made by the calling thread (that call disarms it, whatever it returns).
 * In that call the copy lane of every CTA copies the q rows and only the
 * K/V tiles before `stop_tile` (>= 0), then stops; the other roles wait for the
 * missing tiles, their bounded waits (limit `wait_ns` nanoseconds instead of
 * the normal 0.2 s) run out, every role leaves its loop, the copies and
 * tensor-core products already issued are drained, the CTA frees its tensor
 * memory, and PKV_DEVERR_TIMEOUT is set in the device error word.  The rows
 * of the affected units are not written.
 * Returns PKV_EINVAL (nothing armed) for stop_tile < 0 or wait_ns outside
 * [1e5, 2e8].
 */
pkv_status pkv_testing_prefill_timeout(int stop_tile, uint64_t wait_ns);

#ifdef __cplusplus
}
#endif

#endif /* PKV_TESTING_H_ */
