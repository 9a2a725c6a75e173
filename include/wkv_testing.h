/*
 * wkv_testing.h — test hooks of libwkv.so. Not part of the operator: these entry points
 * exist so that the library's failure handling can be exercised without faulting a GPU.
 */
#ifndef WKV_TESTING_H_
#define WKV_TESTING_H_

#include <stdint.h>

#include "wkv.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Runs the chunked forward on a small internal problem (B = 1, C = 32, three time
 * segments; every input zero) in which segment 0 withholds its published aggregate, so
 * the later segments wait for a flag that nothing sets and give up
 * after `wait_ns` nanoseconds (bounded wait; no trap, no hang). The kernel still ends and
 * the next wkv_stream_status(stream) returns WKV_ERR_TIMEOUT, after which the error word
 * is clear again. Allocates its buffers with cudaMallocAsync on `stream` and frees them in
 * stream order. Returns the launch status.
 */
WKV_API int wkv_testing_lookback_timeout(uint64_t wait_ns, cudaStream_t stream);

/*
 * Forces the plain (non-TMA) forward kernel for one fp32 / bf16 forward; otherwise as
 * wkv_forward / wkv_forward_bf16. Lets tests compare the two kernels on the same inputs.
 */
WKV_API int wkv_testing_forward_plain(int64_t B, int64_t T, int64_t C, const float* w,
                                      const float* u, const void* k, const void* v,
                                      const void* r, void* y, int bf16, cudaStream_t stream);

/*
 * Runs the backward on a small internal problem (B = 1, T = 192, C = 32: three segments
 * of the time-parallel reverse pass; every input zero) in which the last segment
 * withholds its published map, so the earlier segments wait for a flag that nothing sets
 * and give up after `wait_ns` nanoseconds (bounded wait; no trap, no hang). The kernels
 * still end and the next wkv_stream_status(stream) returns WKV_ERR_TIMEOUT, after which
 * the error word is clear again. Allocates its buffers with cudaMallocAsync on `stream`
 * and frees them in stream order. Returns the launch status.
 */
WKV_API int wkv_testing_backward_timeout(uint64_t wait_ns, cudaStream_t stream);

/*
 * Chooses the reverse pass of the backward's TMA path for every later call in this process
 * (wkv_backward, wkv_backward_state, wkv_backward_checkpointed): 0 automatic (one CTA per
 * channel group when there are at least twice as many groups (batch row x 32 channels) as
 * SMs, else time-parallel segments), 1 always time-parallel segments, 2 always one CTA per
 * channel group. Lets tests run both on the same inputs. Other values: WKV_ERR_INVALID_ARG.
 */
WKV_API int wkv_testing_set_backward_path(int path);

/*
 * Forces the backward's plain (non-TMA) tile movement; otherwise as wkv_backward.
 */
WKV_API int wkv_testing_backward_plain(int64_t B, int64_t T, int64_t C, const float* w,
                                       const float* u, const float* k, const float* v,
                                       const float* r, const float* dy, float* dk, float* dv,
                                       float* dw, float* du, float* dr, void* workspace,
                                       size_t workspace_bytes, cudaStream_t stream);

/*
 * Forces the plain (non-TMA) tile movement of wkv_backward_state; otherwise as it.
 */
WKV_API int wkv_testing_backward_state_plain(
    int64_t B, int64_t T, int64_t C, const float* w, const float* u, const float* k,
    const float* v, const float* r, const float* dy, const float* a0, const float* b0,
    const float* p0, const float* ga1, const float* gb1, const float* p1, float* dk, float* dv,
    float* dw, float* du, float* dr, float* da0, float* db0, float* dp0, void* workspace,
    size_t workspace_bytes, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* WKV_TESTING_H_ */
