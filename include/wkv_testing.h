/*
 * wkv_testing.h — test hooks of libwkv.so. Not part of the operator: these entry points
 * exist so that the library's failure handling can be exercised without faulting a GPU,
 * so that tests can force one path or another, and so that the rooflines' compute
 * denominators can be measured on the GPU at hand.
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
 * channel group (of five warps while the groups number at most three times the SMs, else
 * four), 3 always one CTA of four warps per channel group. Lets tests run every form on the
 * same inputs. Other values: WKV_ERR_INVALID_ARG.
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

/* Pipes wkv_testing_pipe_rate can measure. */
#define WKV_PIPE_EX2 0   /* ex2.approx.ftz.f32 instructions per second (MUFU) */
#define WKV_PIPE_FFMA2 1 /* fp32 flops per second through packed fp32x2 FMA (4 per instruction) */

/*
 * Measures one pipe's throughput on the current device: a grid of 8 CTAs x 256 threads per
 * SM, each thread running 8 independent chains of `iters` instructions (1 <= iters <=
 * 2^30), timed with CUDA events on `stream` (the call synchronises on its end event).
 * Writes the rate to *per_second (host pointer): the denominators of the exponential
 * (SFU) roofline term of the forward and of the RWKV-7 recurrence's FP32 roofline, as this
 * GPU sustains them (nominal figures, unit counts x the maximum clock, assume a clock the
 * power cap does not always allow). Compute only, apart from a one-float buffer it
 * allocates and frees on `stream` (nothing is ever stored to it).
 * Returns WKV_ERR_INVALID_ARG for an unknown pipe, out-of-range iters or a null pointer.
 */
WKV_API int wkv_testing_pipe_rate(int pipe, int64_t iters, double* per_second,
                                  cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* WKV_TESTING_H_ */
