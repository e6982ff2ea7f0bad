/*
 * ivit_selftest.h -- diagnostic entry points of the integer-only ViT library.
 *
 * They exercise the library's failure paths without a GPU fault (a wait that
 * nothing completes; a producer told to stop early) and measure the integer
 * throughput that bounds the attention kernels.  Every wait
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

/* Integer throughput probe: the roof of the attention kernels' Shiftmax
 * passes ("I-ViT", section 3.3), whose per-score work runs on the CUDA cores.
 * Enqueues one kernel of 4 x (SM count) blocks of 256 threads; every thread
 * runs `iters` iterations over 8 independent chains of the per-score integer
 * mix (requant mul.hi, two clamps, offset from the row maximum, table index,
 * ShiftExp table load from shared memory, row-sum add, a shift and two adds
 * that feed the next step: 10 operations).  *ops receives the operations one
 * launch executes (blocks x 256 x iters x 8 x 10); the caller times the
 * launch (CUDA events on `stream`) and divides.  sink: device int32 array of
 * at least sink_len >= 4 x (SM count) elements, owned by the caller, which
 * receives one checksum per block (read-modify-write: its contents are not
 * meaningful).  Returns IVIT_ERR_INVALID_ARG for iters < 1, a NULL pointer or
 * a short sink, IVIT_ERR_UNSUPPORTED without an sm_100 device, IVIT_ERR_CUDA
 * if the launch failed.                                                      */
ivit_status ivit_selftest_int_rate(int32_t iters, int32_t *sink, int32_t sink_len, int64_t *ops,
                                   ivit_stream_t stream);

/* Failure path of the production kernels, without a fault.  After this call
 * the next launch of the named kernel -- 1: the INT8 GEMM of every linear
 * layer (ivit_linear_requant, ivit_linear_shiftgelu and the linear layers of
 * ivit_block_forward); 2: the short-sequence attention kernel (ivit_attention
 * with N <= 256) -- has the TMA producer of its first CTA stop before its
 * `index`-th load (a k-slice of the GEMM, an item of the attention), so the
 * tensor-core issuer's bounded wait for that load runs out after one second.
 * The kernel then records IVIT_ERR_TIMEOUT in the device status word, every
 * role gives up its waits, the issued MMAs and copies drain, the tensor
 * memory is released and the kernel returns; its output is incomplete.
 * ivit_stream_status() then returns IVIT_ERR_TIMEOUT once.  The request is
 * taken by that one launch (a later call replaces a pending one).  index
 * beyond the CTA's loads leaves that launch untouched.  Returns
 * IVIT_ERR_INVALID_ARG for another kernel number or a negative index.      */
ivit_status ivit_selftest_withhold(int32_t kernel, int32_t index);

#ifdef __cplusplus
}
#endif

#endif /* IVIT_SELFTEST_H_ */
