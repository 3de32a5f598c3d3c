/*
 * tq_testing.h — test hooks of the tq library. Not for production use.
 *
 * The tensor-core path of tq_linear bounds every in-kernel wait: a wait that
 * does not complete within the limit (2 s) makes the kernel stop, write NaN
 * to the outputs it owns, let its issued tensor-core operations finish, free
 * its tensor memory and return, so that a broken pipeline can never hang the
 * GPU. This hook lets a test take that path without any fault: it shortens
 * the limit and makes the kernel's decoder warps withhold their first
 * "operand stage ready" signal, so that the MMA issuer's wait runs out.
 */
#ifndef TQ_TESTING_H
#define TQ_TESTING_H

#include <stdint.h>

#include "tq.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Applies to the tensor-core tq_linear launches issued after the call, in
 * every thread of the process, until it is called again with (0, 0).
 *   withhold_first_arrive  non-zero: decoders skip their first "A stage
 *                          ready" arrive (the MMA issuer then times out).
 *   wait_limit_ns          limit of every in-kernel wait; 0 = the default.
 * Not thread-safe with respect to concurrent tq_linear calls. Returns TQ_OK. */
tq_status tq_testing_linear_wait_fault(int32_t withhold_first_arrive,
                                       uint64_t wait_limit_ns);

/* Route the tq_linear calls issued after this call, in every thread of the
 * process, to one family of kernels, so that tests and measurements can
 * compare them at the same shape:
 *   0  automatic (the default dispatch by format and batch);
 *   1  the CUDA-core kernels (GEMV where it takes the batch, else the
 *      one-warp-per-row kernel);
 *   2  the tensor-core kernel;
 *   3  the tensor-core kernel with every Format B code-book entry split
 *      into a bf16 hi + lo operand pair, even where the code book allows
 *      the single-operand path (integer multiples of one unit).
 * A family that cannot take the call falls back to the automatic choice.
 * Returns TQ_ERR_INVALID_ARG for other values. */
tq_status tq_testing_force_linear_path(int32_t path);

/* Plan the tensor-core tq_linear launches issued after this call, in every
 * thread of the process, with a split of K over clusters of `ks` CTAs
 * (1..8; 0 = the planner's choice) and at most `max_clusters` clusters
 * (0 = as many as are resident or as there are row tiles), so that tests
 * can make each cluster walk several tiles on a small shape. A split the
 * shape or the device cannot take makes those calls fail
 * (TQ_ERR_CUDA). Returns TQ_ERR_INVALID_ARG for values out of range. */
tq_status tq_testing_tc_split(int32_t ks, int32_t max_clusters);

/* Select the self-checking build of the tensor-core kernel for the tq_linear
 * calls issued after this call (enable != 0), or the ordinary one. The
 * self-checking kernel verifies every shared-memory, tensor-memory,
 * distributed-shared-memory and output address it computes against the
 * region it must lie in; a violation is recorded (never performed) and the
 * access goes to a safe address instead; waits that give up are recorded too.
 * If record_out is not NULL, the record is copied there (synchronously):
 * [0] the first violation (site << 48 | warp << 40 | block index), [1] its
 * value, [2] the number of violations; reset != 0 then clears it. */
tq_status tq_testing_tc_self_check(int32_t enable, uint64_t record_out[4],
                                   int32_t reset);

/* Progress trace of the self-checking tensor-core kernel: while set, every
 * role of every CTA writes the last step it reached to
 * mapped_host_buffer[block * 8 + role] (page-locked host memory the device
 * can address; it stays readable after a device fault). NULL stops it. */
tq_status tq_testing_tc_trace(uint64_t *mapped_host_buffer);

#ifdef __cplusplus
}
#endif
#endif /* TQ_TESTING_H */
