/*
 * dg_test.h -- failure-detection test hooks of libdg.so (sm_100a).
 *
 * These entry points are exported by the same library as the ones in dg.h but are not part of the
 * sampler's interface: they exist so that tests can make every bounded device-side wait of the
 * library run out on purpose, without any fault, trap or endless loop, and check that the kernel
 * gives up, reports through dg_device_error() and leaves the device usable.  Conventions (status
 * codes, dg_last_error, streams, workspaces) are those of dg.h.
 */
#ifndef DG_TEST_H_
#define DG_TEST_H_

#include "dg.h"

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------------------ */
/* Failure-detection test hooks (the pages have no counterpart).  Every wait */
/* inside the library's kernels is bounded; these entry points make a wait  */
/* run out on purpose -- without any fault, trap or endless loop -- so that */
/* tests can check that the kernel gives up, reports through                */
/* dg_device_error() (code 1) and leaves the device usable.                 */
/* dg_test_bounded_wait: one thread waits on a barrier nothing arrives on;  */
/*   the wait gives up after limit_cycles (> 0) SM clock cycles.             */
/* dg_test_selfcond_stall: dg_selfcond with the copy of one 64-id block of  */
/*   E never issued (stalled_block >= 0, in [0, ceil(V/64)) to take effect) */
/*   and every wait limited to limit_cycles: the CTAs that need the block   */
/*   abort, drain their in-flight copies, free their tensor memory and      */
/*   return.  z is then incomplete.  Same arguments as dg_selfcond otherwise.*/
/* ------------------------------------------------------------------------ */
int dg_test_bounded_wait(uint32_t limit_cycles, dg_stream_t stream);

/* dg_test_merge_stall: the logits pass's per-row merge kernel alone (the   */
/*   statistics epilogue), with no streaming kernel writing this call's     */
/*   records: every row's wait gives up after limit_cycles (> 0), records   */
/*   device error 1, and the merge finishes on whatever the workspace holds */
/*   (lse is then meaningless).  logits as dg_sampler_step with B = 1,      */
/*   C = rows; lse: device float [rows]; workspace:                         */
/*   dg_sampler_step_workspace_size(rows, V) bytes, zeroed.                 */
int dg_test_merge_stall(const void* logits, int logits_dtype, int64_t ld, int32_t rows, int32_t V,
                        float* lse, void* workspace, size_t workspace_bytes, uint32_t limit_cycles,
                        dg_stream_t stream);

int dg_test_selfcond_stall(const void* logits, int logits_dtype, int64_t ld, int32_t B, int32_t C,
                           int32_t V, const float* inv_tau, const float* lse, const void* E,
                           int embed_dtype, int32_t d, void* z, void* workspace,
                           size_t workspace_bytes, dg_stream_t stream, int32_t stalled_block,
                           uint32_t limit_cycles);

#ifdef __cplusplus
}
#endif

#endif /* DG_TEST_H_ */
