/*
 * ivit_selftest.h -- diagnostic entry points of the integer-only ViT library.
 *
 * These exercise the library's failure path without a GPU fault.  Every wait
 * inside the library's kernels (an mbarrier spin) is bounded by a budget of
 * one second of %globaltimer; a wait that runs out records IVIT_ERR_TIMEOUT
 * in the per-device status word, and the kernel returns instead of hanging.
 * The conventions of ivit.h apply.
 */
#ifndef IVIT_SELFTEST_H_
#define IVIT_SELFTEST_H_

#include "ivit.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Enqueues one kernel on `stream` whose single waiting thread waits, through
 * the same bounded wait as every kernel of the library, on an mbarrier that
 * nothing ever arrives at.  After the wait budget (one second) it records
 * IVIT_ERR_TIMEOUT in the device status word and returns, so the context
 * stays usable: ivit_stream_status() then returns IVIT_ERR_TIMEOUT once and
 * clears the word.  Returns IVIT_OK when the kernel was enqueued,
 * IVIT_ERR_UNSUPPORTED without an sm_100 device, IVIT_ERR_CUDA if the launch
 * failed.  Takes about one second of GPU time.                               */
ivit_status ivit_selftest_wait_timeout(ivit_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* IVIT_SELFTEST_H_ */
