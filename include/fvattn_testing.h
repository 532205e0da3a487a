/*
 * fvattn test hooks: entry points that exist only so that tests can drive the library's
 * error paths on a real GPU without faulting it.  Not part of the method (the FVAttn
 * explainer has no counterpart); applications have no use for them.
 */
#ifndef FVATTN_TESTING_H_
#define FVATTN_TESTING_H_

#include "fvattn.h"

#ifdef __cplusplus
extern "C" {
#endif

/* fvattn_block_sparse_attn (same arguments, minus sm_busy_ns) in which every CTA of the
 * attention kernel, at its first tile, waits on a barrier that nothing ever completes,
 * bounded by about stall_ns nanoseconds (0 < stall_ns <= 1e8, else
 * FVATTN_ERR_INVALID_ARG).  The wait gives up, as any stuck wait of the kernel would:
 * the CTA raises its abort flag and the workspace's error word, every role leaves its
 * loop, armed copies and issued MMAs are drained, tensor memory is released and the
 * kernel returns.  Afterwards fvattn_device_status(workspace) reports
 * FVATTN_ERR_DEVICE_TIMEOUT; out and lse are unspecified; the CUDA context stays usable
 * and the next call on the same workspace starts clean. */
FVATTN_API fvattn_status_t fvattn_testing_attn_stall(const fvattn_geom_t* g, const void* q, const void* k,
                                                     const void* v, const uint32_t* mask, float scale,
                                                     void* out, float* lse, void* workspace, size_t ws_bytes,
                                                     unsigned long long stall_ns, fvattn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FVATTN_TESTING_H_ */
