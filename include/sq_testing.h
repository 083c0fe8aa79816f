/*
 * sq_testing.h -- failure injection for the tests of libsq.  Not part of the
 * decode path; the pages have no counterpart to it.
 *
 * The prefill kernels -- sq_linear on many tokens (SQ_LAYOUT_ROWS, group size
 * 128) and sq_nvfp4_linear -- bound every wait on their pipeline barriers.  When a wait runs out, the
 * kernel records SQ_ERR_TIMEOUT in the caller's status word and winds down:
 * it first waits (again bounded) for the operand copies it has requested and
 * for the tensor-core MMAs it has issued, then frees its tensor memory and
 * returns, so the context stays usable.  This entry point makes that happen
 * on purpose, without any fault: the operands of one channel group (stage)
 * are simply never requested, and every wait is limited to wait_ns.
 */
#ifndef SQ_TESTING_H
#define SQ_TESTING_H

#include "sq.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * sq_linear on the prefill kernel with its waits limited to wait_ns
 * (1 .. 10^9 nanoseconds) and the operands of channel group skip_group
 * (0 <= skip_group < ceil(K/128)) never requested; skip_group = -1 requests
 * everything and gives the result of sq_linear.  Arguments are those of
 * sq_linear; the weight must be in SQ_LAYOUT_ROWS with group size 128, M at
 * least 64 (else SQ_ERR_SHAPE).  With a group skipped, dev_status ends up
 * SQ_ERR_TIMEOUT and y is unspecified.
 */
sq_status sq_testing_prefill_stalled(const sq_packed_weight *w, const int8_t *xq, const float *sx,
                                     const float *x_out, const int32_t *idx, int32_t n_out,
                                     int32_t M, float *y, int32_t skip_group, uint64_t wait_ns,
                                     int32_t *dev_status, void *stream);

/*
 * sq_nvfp4_linear with its waits limited to wait_ns (1 .. 10^9 nanoseconds)
 * and the operands of channel stage skip_stage (256 channels each,
 * 0 <= skip_stage < roundup(K,256)/256) never requested for any tile;
 * skip_stage = -1 requests everything and gives the result of
 * sq_nvfp4_linear.  Arguments are those of sq_nvfp4_linear.  With a stage
 * skipped, dev_status ends up SQ_ERR_TIMEOUT and y is unspecified.
 */
sq_status sq_testing_nvfp4_stalled(const sq_nvfp4_matrix *w, const sq_nvfp4_matrix *x, float *y,
                                   int32_t skip_stage, uint64_t wait_ns, int32_t *dev_status,
                                   void *stream);

/*
 * Dense tensor-core throughput probe, the peak the prefill kernels are
 * reported against: every SM issues `iters` x 4 back-to-back tcgen05.mma of
 * one kind on operands resident in its shared memory (a fixed pseudo-random
 * pattern; scales 1.0), accumulating in tensor memory.
 *   kind 0: kind::i8, 128 x 256 x 32;  kind 1: kind::mxf4nvf4 (block 16),
 *   128 x 256 x 64
 *   ops_per_s  host: 2 x multiply-adds per second of device time (CUDA
 *              events around one launch, after a warm-up launch)
 * 1 <= iters <= 100000.  Synchronous on `stream`.
 */
sq_status sq_testing_mma_peak(int32_t kind, int32_t iters, double *ops_per_s, int32_t *dev_status,
                              void *stream);

/*
 * Pure-read HBM probe, the second denominator of the decode kernels (which
 * read weights and write almost nothing; a device copy also writes): `iters`
 * back-to-back read-only sweeps of a caller's buffer, 16-byte coalesced
 * loads, eight in flight per thread, four 512-thread CTAs per SM.
 *   buf          device, 16-byte aligned, `bytes` readable bytes (contents
 *                irrelevant); choose bytes well above the L2 size (126 MB)
 *   bytes        a multiple of 16, >= 16
 *   bytes_per_s  host: bytes x iters / device time (CUDA events around the
 *                sweeps, after a warm-up sweep)
 * 1 <= iters <= 1000.  Synchronous on `stream`.
 */
sq_status sq_testing_read_peak(const void *buf, uint64_t bytes, int32_t iters, double *bytes_per_s,
                               void *stream);

#ifdef __cplusplus
}
#endif
#endif /* SQ_TESTING_H */
