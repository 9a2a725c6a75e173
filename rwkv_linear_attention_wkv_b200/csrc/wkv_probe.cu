// Pipe-throughput probes (sm_100a): the denominators of two rooflines, measured on the GPU
// the library runs on rather than derived from unit counts and a clock.
//   WKV_PIPE_EX2:   ex2.approx.ftz.f32 per second (the MUFU pipe; the forward's SFU term:
//                   every exponential of the operator is one ex2 after a base-2 pre-scale);
//   WKV_PIPE_FFMA2: fp32 flops per second through packed fp32x2 fused multiply-adds (the
//                   FMA pipe; the RWKV-7 recurrence's bound), 4 flops per instruction.
// Every thread of a full-occupancy grid (8 CTAs of 256 threads per SM) runs 8 independent
// chains, so that issue, not latency, limits the rate. The chains stay bounded: x -> 2^-x
// maps [0.5, 1) into (0.5, 0.71], and acc -> acc a + b with a < 1 converges. The sum of a
// thread's chains is stored to a one-float device buffer (allocated on the stream) only if
// it equals -1, which it never does, but which the compiler cannot rule out: the work is
// kept, and a store, were it ever made, would land in that buffer.
#include <algorithm>

#include "wkv_device.cuh"
#include "wkv_internal.h"
#include "wkv_testing.h"

namespace wkv {

namespace {

constexpr int kProbeThreads = 256;
constexpr int kProbeCtasPerSm = 8;
constexpr int kChains = 8;

__global__ void __launch_bounds__(kProbeThreads) ex2_probe_kernel(int iters, float* sink) {
  float x[kChains];
#pragma unroll
  for (int j = 0; j < kChains; ++j) x[j] = 0.5f + 0.01f * float((threadIdx.x + j) & 31);
  for (int i = 0; i < iters; ++i) {
#pragma unroll
    for (int j = 0; j < kChains; ++j) x[j] = ex2(-x[j]);
  }
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < kChains; ++j) s += x[j];
  if (s == -1.f) *sink = s;
}

__global__ void __launch_bounds__(kProbeThreads) ffma2_probe_kernel(int iters, float* sink) {
  float2 acc[kChains];
#pragma unroll
  for (int j = 0; j < kChains; ++j) acc[j] = make_float2(float(j), float(threadIdx.x & 7));
  const float2 a = make_float2(0.999f, 0.998f), c = make_float2(1e-3f, 2e-3f);
  for (int i = 0; i < iters; ++i) {
#pragma unroll
    for (int j = 0; j < kChains; ++j) acc[j] = __ffma2_rn(acc[j], a, c);
  }
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < kChains; ++j) s += acc[j].x + acc[j].y;
  if (s == -1.f) *sink = s;
}

}  // namespace

}  // namespace wkv

WKV_API int wkv_testing_pipe_rate(int pipe, int64_t iters, double* per_second,
                                  cudaStream_t stream) {
  using namespace wkv;
  if (per_second == nullptr || iters < 1 || iters > (int64_t(1) << 30) ||
      (pipe != WKV_PIPE_EX2 && pipe != WKV_PIPE_FFMA2))
    return WKV_ERR_INVALID_ARG;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return WKV_ERR_CUDA;
  const int grid = sms * kProbeCtasPerSm;
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  if (cudaEventCreate(&e0) != cudaSuccess || cudaEventCreate(&e1) != cudaSuccess) {
    if (e0) cudaEventDestroy(e0);
    return WKV_ERR_CUDA;
  }
  int rc = WKV_OK;
  float ms = 0.f;
  float* sink = nullptr;
  if (cudaMallocAsync(reinterpret_cast<void**>(&sink), sizeof(float), stream) != cudaSuccess)
    rc = WKV_ERR_CUDA;
  if (rc == WKV_OK && cudaEventRecord(e0, stream) != cudaSuccess) rc = WKV_ERR_CUDA;
  if (rc == WKV_OK) {
    if (pipe == WKV_PIPE_EX2)
      ex2_probe_kernel<<<grid, kProbeThreads, 0, stream>>>(int(iters), sink);
    else
      ffma2_probe_kernel<<<grid, kProbeThreads, 0, stream>>>(int(iters), sink);
    if (cudaPeekAtLastError() != cudaSuccess || cudaEventRecord(e1, stream) != cudaSuccess ||
        cudaEventSynchronize(e1) != cudaSuccess || cudaEventElapsedTime(&ms, e0, e1) != cudaSuccess ||
        ms <= 0.f)
      rc = WKV_ERR_CUDA;
  }
  if (sink != nullptr) cudaFreeAsync(sink, stream);
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  if (rc != WKV_OK) return rc;
  const double per_instr = pipe == WKV_PIPE_EX2 ? 1.0 : 4.0;  // ex2, or 2 lanes x (mul + add)
  *per_second = double(grid) * kProbeThreads * kChains * double(iters) * per_instr /
                (double(ms) * 1e-3);
  return WKV_OK;
}
