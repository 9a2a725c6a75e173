// C-ABI entry points of libwkv.so: argument checks, plan selection, launches.
// Declarations and their documentation: include/wkv.h.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdint>
#include <mutex>

#include "wkv_device.cuh"
#include "wkv_internal.h"
#include "wkv_testing.h"

namespace wkv {

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Device error word (one per device context): bit kErrTimeout is set by a kernel that
// gave up a bounded wait. Read and cleared by wkv_stream_status().
__device__ unsigned g_error_word;

namespace {

constexpr int kMaxDevices = 64;

// The per-device cache is filled under a lock: host threads may make their first calls
// on the same device at the same time.
unsigned* error_word() {
  static unsigned* cached[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (cached[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
    cached[dev] = static_cast<unsigned*>(p);
  }
  return cached[dev];
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool aligned(const void* p, size_t a) {
  return p == nullptr || (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

// All three state pointers given, or none.
bool state_triplet_ok(const void* a, const void* b, const void* p) {
  return (a == nullptr) == (b == nullptr) && (a == nullptr) == (p == nullptr);
}

int check_fwd(int64_t B, int64_t T, int64_t C, const void* w, const void* u, const void* k,
              const void* v, const void* r, const void* y, size_t esz) {
  if (B < 0 || T < 0 || C < 0) return WKV_ERR_INVALID_ARG;
  if (B == 0 || C == 0) return WKV_OK;
  if (!w || !u) return WKV_ERR_INVALID_ARG;
  if (T > 0 && (!k || !v || !y)) return WKV_ERR_INVALID_ARG;
  if (!aligned(w, 4) || !aligned(u, 4) || !aligned(k, esz) || !aligned(v, esz) ||
      !aligned(r, esz) || !aligned(y, esz))
    return WKV_ERR_ALIGNMENT;
  // Kernel indexing: T and C fit in int32 for tile coordinates; B*T*C in int64.
  if (T >= (int64_t(1) << 31) || C >= (int64_t(1) << 31) || B >= (int64_t(1) << 31))
    return WKV_ERR_UNSUPPORTED;
  if (T > 0 && B > INT64_MAX / T / C) return WKV_ERR_UNSUPPORTED;
  return WKV_OK;
}

}  // namespace

unsigned* device_error_word() { return error_word(); }

int encode_btc_map(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                   int elem_bytes, int64_t B, int64_t T, int64_t C, int box_c, int box_t) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return WKV_ERR_CUDA;
  cuuint64_t dims[3] = {cuuint64_t(C), cuuint64_t(T), cuuint64_t(B)};
  cuuint64_t strides[2] = {cuuint64_t(C) * elem_bytes, cuuint64_t(T) * C * elem_bytes};
  cuuint32_t box[3] = {cuuint32_t(box_c), cuuint32_t(box_t), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult rc = enc(map, dtype, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return rc == CUDA_SUCCESS ? WKV_OK : WKV_ERR_CUDA;
}

// Shared by the three forward entry points.
static int forward_impl(int64_t B, int64_t T, int64_t C, const float* w, const float* u,
                        const void* k, const void* v, const void* r, void* y, const float* a0,
                        const float* b0, const float* p0, float* a1, float* b1, float* p1,
                        bool bf16, cudaStream_t stream) {
  int rc = check_fwd(B, T, C, w, u, k, v, r, y, bf16 ? 2 : 4);
  if (rc != WKV_OK) return rc;
  if (!state_triplet_ok(a0, b0, p0) || !state_triplet_ok(a1, b1, p1)) return WKV_ERR_INVALID_ARG;
  if (!aligned(a0, 4) || !aligned(b0, 4) || !aligned(p0, 4) || !aligned(a1, 4) ||
      !aligned(b1, 4) || !aligned(p1, 4))
    return WKV_ERR_ALIGNMENT;
  if (B == 0 || C == 0) return WKV_OK;
  if (T == 0 && a1 == nullptr) return WKV_OK;
  unsigned* err = error_word();
  if (err == nullptr) return WKV_ERR_CUDA;
  FwdArgs a{B, T, C, w, u, k, v, r, y, a0, b0, p0, a1, b1, p1, err};
  if (!bf16 && T > 0) {
    int64_t flag_bytes = 0;
    int nseg = 1;
    const size_t scratch = chunked_scratch_bytes(B, T, C, &flag_bytes, &nseg);
    if (nseg > 1) {
      void* ws = nullptr;
      if (cudaMallocAsync(&ws, scratch, stream) != cudaSuccess) return WKV_ERR_CUDA;
      if (cudaMemsetAsync(ws, 0, size_t(flag_bytes), stream) != cudaSuccess) {
        cudaFreeAsync(ws, stream);
        return WKV_ERR_CUDA;
      }
      rc = launch_fwd_chunked(a, ws, nseg, stream);
      cudaFreeAsync(ws, stream);
      return rc;
    }
  }
  return launch_fwd_stream(a, bf16, /*force_plain=*/T == 0, stream);
}

// The state arguments of wkv_backward_state (all NULL for wkv_backward).
struct StateArgs {
  const float* a0 = nullptr;
  const float* b0 = nullptr;
  const float* p0 = nullptr;
  const float* ga1 = nullptr;
  const float* gb1 = nullptr;
  const float* p1 = nullptr;
  float* da0 = nullptr;
  float* db0 = nullptr;
  float* dp0 = nullptr;
};

static bool all_or_none(const void* x, const void* y, const void* z) {
  return (x == nullptr) == (y == nullptr) && (x == nullptr) == (z == nullptr);
}

static int backward_impl(int64_t B, int64_t T, int64_t C, const float* w, const float* u,
                         const float* k, const float* v, const float* r, const float* dy,
                         float* dk, float* dv, float* dw, float* du, float* dr, void* workspace,
                         size_t workspace_bytes, bool force_plain, cudaStream_t stream,
                         const StateArgs& st = StateArgs(), bool have_ckpt = false) {
  if (B < 0 || T < 0 || C < 0) return WKV_ERR_INVALID_ARG;
  if (!all_or_none(st.a0, st.b0, st.p0) || !all_or_none(st.ga1, st.gb1, st.p1) ||
      !all_or_none(st.da0, st.db0, st.dp0))
    return WKV_ERR_INVALID_ARG;
  if (C == 0) return WKV_OK;
  if (!w || !u || !dw || !du) return WKV_ERR_INVALID_ARG;
  if (r == nullptr && dr != nullptr) return WKV_ERR_INVALID_ARG;
  const void* ptrs[] = {w,     u,     k,     v,      r,      dy,     dk,     dv,     dw, du,
                        dr,    st.a0, st.b0, st.p0,  st.ga1, st.gb1, st.p1,  st.da0, st.db0,
                        st.dp0};
  for (const void* q : ptrs)
    if (!aligned(q, 4)) return WKV_ERR_ALIGNMENT;
  if (B == 0) return WKV_OK;
  if (T == 0) {  // no tokens: zero gradients for the parameters; the state passes through
    if (cudaMemsetAsync(dw, 0, size_t(C) * sizeof(float), stream) != cudaSuccess ||
        cudaMemsetAsync(du, 0, size_t(C) * sizeof(float), stream) != cudaSuccess)
      return WKV_ERR_CUDA;
    if (st.da0 == nullptr) return WKV_OK;
    if (B > INT64_MAX / C) return WKV_ERR_UNSUPPORTED;
    BwdArgs a{B, T, C, w, u, k, v, r, dy, dk, dv, dw, du, dr, nullptr, nullptr};
    a.a0 = st.a0; a.b0 = st.b0; a.p0 = st.p0;
    a.ga1 = st.ga1; a.gb1 = st.gb1; a.p1 = st.p1;
    a.da0 = st.da0; a.db0 = st.db0; a.dp0 = st.dp0;
    return launch_backward_no_tokens(a, stream);
  }
  if (!k || !v || !dy || !dk || !dv) return WKV_ERR_INVALID_ARG;
  if (T >= (int64_t(1) << 31) || C >= (int64_t(1) << 31) || B >= (int64_t(1) << 31) ||
      B > INT64_MAX / T / C || B * ((C + 31) / 32) >= (int64_t(1) << 31))
    return WKV_ERR_UNSUPPORTED;
  if (workspace == nullptr || !aligned(workspace, 256) ||
      workspace_bytes < backward_workspace_bytes(B, T, C))
    return WKV_ERR_INVALID_ARG;
  unsigned* err = error_word();
  if (err == nullptr) return WKV_ERR_CUDA;
  BwdArgs a{B, T, C, w, u, k, v, r, dy, dk, dv, dw, du, dr, workspace, err};
  a.a0 = st.a0; a.b0 = st.b0; a.p0 = st.p0;
  a.ga1 = st.ga1; a.gb1 = st.gb1; a.p1 = st.p1;
  a.da0 = st.da0; a.db0 = st.db0; a.dp0 = st.dp0;
  a.have_ckpt = have_ckpt ? 1 : 0;
  return launch_backward(a, force_plain, stream);
}

// wkv_forward_checkpointed: the forward of wkv_forward_state (without the final state) that
// also writes the backward's checkpoints into `workspace`.
static int forward_ckpt_impl(int64_t B, int64_t T, int64_t C, const float* w, const float* u,
                             const float* k, const float* v, const float* r, float* y,
                             const float* a0, const float* b0, const float* p0, void* workspace,
                             size_t workspace_bytes, cudaStream_t stream) {
  int rc = check_fwd(B, T, C, w, u, k, v, r, y, 4);
  if (rc != WKV_OK) return rc;
  if (!state_triplet_ok(a0, b0, p0)) return WKV_ERR_INVALID_ARG;
  if (!aligned(a0, 4) || !aligned(b0, 4) || !aligned(p0, 4)) return WKV_ERR_ALIGNMENT;
  if (B == 0 || C == 0 || T == 0) return WKV_OK;
  if (B * ((C + 31) / 32) >= (int64_t(1) << 31)) return WKV_ERR_UNSUPPORTED;
  if (workspace == nullptr || !aligned(workspace, 256) ||
      workspace_bytes < backward_workspace_bytes(B, T, C))
    return WKV_ERR_INVALID_ARG;
  unsigned* err = error_word();
  if (err == nullptr) return WKV_ERR_CUDA;
  FwdArgs a{B, T, C, w, u, k, v, r, y, a0, b0, p0, nullptr, nullptr, nullptr, err};
  return launch_fwd_ckpt(a, workspace, stream);
}

}  // namespace wkv

using namespace wkv;

extern "C" {

WKV_API const char* wkv_status_string(int status) {
  switch (status) {
    case WKV_OK: return "WKV_OK";
    case WKV_ERR_INVALID_ARG: return "WKV_ERR_INVALID_ARG";
    case WKV_ERR_ALIGNMENT: return "WKV_ERR_ALIGNMENT";
    case WKV_ERR_CUDA: return "WKV_ERR_CUDA";
    case WKV_ERR_TIMEOUT: return "WKV_ERR_TIMEOUT";
    case WKV_ERR_UNSUPPORTED: return "WKV_ERR_UNSUPPORTED";
    case WKV_ERR_SCRATCH_LIMIT: return "WKV_ERR_SCRATCH_LIMIT";
    case WKV_ERR_RANGE: return "WKV_ERR_RANGE";
    default: return "WKV_ERR_UNKNOWN";
  }
}

WKV_API int wkv_version(void) { return 10100; }

WKV_API int wkv_forward(int64_t B, int64_t T, int64_t C, const float* w, const float* u,
                        const float* k, const float* v, const float* r, float* y,
                        cudaStream_t stream) {
  return forward_impl(B, T, C, w, u, k, v, r, y, nullptr, nullptr, nullptr, nullptr, nullptr,
                      nullptr, false, stream);
}

WKV_API int wkv_forward_bf16(int64_t B, int64_t T, int64_t C, const float* w, const float* u,
                             const void* k, const void* v, const void* r, void* y,
                             cudaStream_t stream) {
  return forward_impl(B, T, C, w, u, k, v, r, y, nullptr, nullptr, nullptr, nullptr, nullptr,
                      nullptr, true, stream);
}

WKV_API int wkv_forward_state(int64_t B, int64_t T, int64_t C, const float* w, const float* u,
                              const float* k, const float* v, const float* r, float* y,
                              const float* a0, const float* b0, const float* p0, float* a1,
                              float* b1, float* p1, cudaStream_t stream) {
  return forward_impl(B, T, C, w, u, k, v, r, y, a0, b0, p0, a1, b1, p1, false, stream);
}

WKV_API int wkv_decode_step(int64_t N, int64_t L, int64_t C, const float* w, const float* u,
                            const float* k, const float* v, const float* r, float* y, float* a,
                            float* b, float* p, cudaStream_t stream) {
  if (N < 0 || L < 0 || C < 0) return WKV_ERR_INVALID_ARG;
  if (N == 0 || L == 0 || C == 0) return WKV_OK;
  if (!w || !u || !k || !v || !y || !a || !b || !p) return WKV_ERR_INVALID_ARG;
  const void* ptrs[] = {w, u, k, v, r, y, a, b, p};
  for (const void* q : ptrs)
    if (!aligned(q, 4)) return WKV_ERR_ALIGNMENT;
  if (L > INT64_MAX / C || N > INT64_MAX / (L * C)) return WKV_ERR_UNSUPPORTED;
  DecodeArgs d{N, L, C, w, u, k, v, r, y, a, b, p};
  return launch_decode(d, stream);
}

WKV_API int wkv_decode_steps(int64_t N, int64_t L, int64_t C, int64_t S, const float* w,
                             const float* u, const float* k, const float* v, const float* r,
                             float* y, float* a, float* b, float* p, cudaStream_t stream) {
  if (N < 0 || L < 0 || C < 0 || S < 0) return WKV_ERR_INVALID_ARG;
  if (N == 0 || L == 0 || C == 0 || S == 0) return WKV_OK;
  if (!w || !u || !k || !v || !y || !a || !b || !p) return WKV_ERR_INVALID_ARG;
  const void* ptrs[] = {w, u, k, v, r, y, a, b, p};
  for (const void* q : ptrs)
    if (!aligned(q, 4)) return WKV_ERR_ALIGNMENT;
  if (L > INT64_MAX / C || N > INT64_MAX / (L * C) || S >= (int64_t(1) << 31) ||
      S > INT64_MAX / (N * L * C))
    return WKV_ERR_UNSUPPORTED;
  DecodeArgs d{N, L, C, w, u, k, v, r, y, a, b, p};
  return launch_decode_steps(d, S, stream);
}

WKV_API size_t wkv_backward_workspace_bytes(int64_t B, int64_t T, int64_t C) {
  if (B <= 0 || T <= 0 || C <= 0) return 256;
  return backward_workspace_bytes(B, T, C);
}

WKV_API int wkv_backward(int64_t B, int64_t T, int64_t C, const float* w, const float* u,
                         const float* k, const float* v, const float* r, const float* dy,
                         float* dk, float* dv, float* dw, float* du, float* dr, void* workspace,
                         size_t workspace_bytes, cudaStream_t stream) {
  return backward_impl(B, T, C, w, u, k, v, r, dy, dk, dv, dw, du, dr, workspace,
                       workspace_bytes, false, stream);
}

WKV_API int wkv_backward_state(int64_t B, int64_t T, int64_t C, const float* w, const float* u,
                               const float* k, const float* v, const float* r, const float* dy,
                               const float* a0, const float* b0, const float* p0,
                               const float* ga1, const float* gb1, const float* p1, float* dk,
                               float* dv, float* dw, float* du, float* dr, float* da0,
                               float* db0, float* dp0, void* workspace, size_t workspace_bytes,
                               cudaStream_t stream) {
  StateArgs st;
  st.a0 = a0; st.b0 = b0; st.p0 = p0;
  st.ga1 = ga1; st.gb1 = gb1; st.p1 = p1;
  st.da0 = da0; st.db0 = db0; st.dp0 = dp0;
  return backward_impl(B, T, C, w, u, k, v, r, dy, dk, dv, dw, du, dr, workspace,
                       workspace_bytes, false, stream, st);
}

WKV_API int wkv_forward_checkpointed(int64_t B, int64_t T, int64_t C, const float* w,
                                     const float* u, const float* k, const float* v,
                                     const float* r, float* y, const float* a0, const float* b0,
                                     const float* p0, void* workspace, size_t workspace_bytes,
                                     cudaStream_t stream) {
  return forward_ckpt_impl(B, T, C, w, u, k, v, r, y, a0, b0, p0, workspace, workspace_bytes,
                           stream);
}

WKV_API int wkv_backward_checkpointed(
    int64_t B, int64_t T, int64_t C, const float* w, const float* u, const float* k,
    const float* v, const float* r, const float* dy, const float* a0, const float* b0,
    const float* p0, const float* ga1, const float* gb1, const float* p1, float* dk, float* dv,
    float* dw, float* du, float* dr, float* da0, float* db0, float* dp0, void* workspace,
    size_t workspace_bytes, cudaStream_t stream) {
  StateArgs st;
  st.a0 = a0; st.b0 = b0; st.p0 = p0;
  st.ga1 = ga1; st.gb1 = gb1; st.p1 = p1;
  st.da0 = da0; st.db0 = db0; st.dp0 = dp0;
  return backward_impl(B, T, C, w, u, k, v, r, dy, dk, dv, dw, du, dr, workspace,
                       workspace_bytes, false, stream, st, /*have_ckpt=*/true);
}

WKV_API int wkv7_forward(int64_t B, int64_t T, int64_t H, int64_t N, const float* r,
                         const float* w, const float* k, const float* v, const float* a,
                         const float* b, float* y, const float* s0, float* s1,
                         cudaStream_t stream) {
  if (B < 0 || T < 0 || H < 0 || N < 0) return WKV_ERR_INVALID_ARG;
  if (B == 0 || H == 0) return WKV_OK;
  if (N != 64) return WKV_ERR_UNSUPPORTED;
  if (T > 0 && (!r || !w || !k || !v || !a || !b || !y)) return WKV_ERR_INVALID_ARG;
  const void* ptrs[] = {r, w, k, v, a, b, y, s0, s1};
  for (const void* q : ptrs)
    if (!aligned(q, 16)) return WKV_ERR_ALIGNMENT;
  if (T >= (int64_t(1) << 31) || B * H >= (int64_t(1) << 31) || H >= (int64_t(1) << 24) ||
      B > INT64_MAX / T / (H * N))
    return WKV_ERR_UNSUPPORTED;
  const size_t sbytes = size_t(B) * H * N * N * sizeof(float);
  if (T == 0) {  // no tokens: the state passes through
    if (s1 == nullptr || s1 == s0) return WKV_OK;
    const cudaError_t e = s0 ? cudaMemcpyAsync(s1, s0, sbytes, cudaMemcpyDeviceToDevice, stream)
                             : cudaMemsetAsync(s1, 0, sbytes, stream);
    return e == cudaSuccess ? WKV_OK : WKV_ERR_CUDA;
  }
  unsigned* err = error_word();
  if (err == nullptr) return WKV_ERR_CUDA;
  return launch_wkv7(B, T, H, r, w, k, v, a, b, y, s0, s1, err, stream);
}

WKV_API int wkv_mstate_forward(int64_t B, int64_t T, int64_t H, int64_t N, const float* r,
                               const float* w, const float* k, const float* v, float* y,
                               const float* s0, float* s1, cudaStream_t stream) {
  if (B < 0 || T < 0 || H < 0 || N < 0) return WKV_ERR_INVALID_ARG;
  if (B == 0 || H == 0) return WKV_OK;
  if (N != 64) return WKV_ERR_UNSUPPORTED;
  if (T > 0 && (!r || !w || !k || !v || !y)) return WKV_ERR_INVALID_ARG;
  const void* ptrs[] = {r, w, k, v, y, s0, s1};
  for (const void* q : ptrs)
    if (!aligned(q, 16)) return WKV_ERR_ALIGNMENT;
  if (T >= (int64_t(1) << 31) || B * H >= (int64_t(1) << 24) ||
      (T > 0 && B > INT64_MAX / T / (H * N)) || B * H * ((T + 63) / 64) >= (int64_t(1) << 31))
    return WKV_ERR_UNSUPPORTED;
  const size_t sbytes = size_t(B) * H * N * N * sizeof(float);
  if (T == 0) {  // no tokens: the state passes through
    if (s1 == nullptr || s1 == s0) return WKV_OK;
    const cudaError_t e = s0 ? cudaMemcpyAsync(s1, s0, sbytes, cudaMemcpyDeviceToDevice, stream)
                             : cudaMemsetAsync(s1, 0, sbytes, stream);
    return e == cudaSuccess ? WKV_OK : WKV_ERR_CUDA;
  }
  unsigned* err = error_word();
  if (err == nullptr) return WKV_ERR_CUDA;
  void* ws = nullptr;
  if (cudaMallocAsync(&ws, mstate_scratch_bytes(B, H), stream) != cudaSuccess)
    return WKV_ERR_CUDA;
  const int rc = launch_mstate(B, T, H, r, w, k, v, y, s0, s1, ws, err, stream);
  cudaFreeAsync(ws, stream);
  return rc;
}

WKV_API int wkv_stream_status(cudaStream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return WKV_ERR_CUDA;
  unsigned* err = error_word();
  if (err == nullptr) return WKV_ERR_CUDA;
  unsigned h = 0;
  if (cudaMemcpy(&h, err, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return WKV_ERR_CUDA;
  if (h != 0) {
    if (cudaMemset(err, 0, sizeof(unsigned)) != cudaSuccess) return WKV_ERR_CUDA;
    return (h & kErrTimeout) ? WKV_ERR_TIMEOUT : WKV_ERR_RANGE;
  }
  return WKV_OK;
}

WKV_API int wkv_testing_lookback_timeout(uint64_t wait_ns, cudaStream_t stream) {
  const int64_t B = 1, T = 768, C = 32;
  int64_t flag_bytes = 0;
  int nseg = 1;
  const size_t scratch = chunked_scratch_bytes(B, T, C, &flag_bytes, &nseg);
  if (nseg < 2) return WKV_ERR_UNSUPPORTED;
  const size_t n = size_t(B * T * C) * sizeof(float);
  const size_t total = 4 * n + 2 * C * sizeof(float) + scratch + 256;
  char* buf = nullptr;
  if (cudaMallocAsync(reinterpret_cast<void**>(&buf), total, stream) != cudaSuccess)
    return WKV_ERR_CUDA;
  if (cudaMemsetAsync(buf, 0, total, stream) != cudaSuccess) {
    cudaFreeAsync(buf, stream);
    return WKV_ERR_CUDA;
  }
  float* k = reinterpret_cast<float*>(buf);
  float* v = k + B * T * C;
  float* r = v + B * T * C;
  float* y = r + B * T * C;
  float* w = y + B * T * C;
  float* u = w + C;
  void* ws = reinterpret_cast<void*>((reinterpret_cast<uintptr_t>(u + C) + 255) & ~uintptr_t(255));
  unsigned* err = error_word();
  int rc = err ? WKV_OK : WKV_ERR_CUDA;
  if (rc == WKV_OK) {
    FwdArgs a{B, T, C, w, u, k, v, r, y, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, err};
    rc = launch_fwd_chunked_ex(a, ws, nseg, (unsigned long long)wait_ns, 1, stream);
  }
  cudaFreeAsync(buf, stream);
  return rc;
}

WKV_API int wkv_testing_backward_timeout(uint64_t wait_ns, cudaStream_t stream) {
  const int64_t B = 1, T = 192, C = 32;  // 12 chunks of 16 tokens: 3 reverse segments
  const size_t n = align_up(size_t(B * T * C) * sizeof(float), 256);
  const size_t c4 = align_up(size_t(C) * sizeof(float), 256);
  const size_t wsb = backward_workspace_bytes(B, T, C);
  const size_t total = 7 * n + 4 * c4 + wsb + 256;
  char* buf = nullptr;
  if (cudaMallocAsync(reinterpret_cast<void**>(&buf), total, stream) != cudaSuccess)
    return WKV_ERR_CUDA;
  if (cudaMemsetAsync(buf, 0, total, stream) != cudaSuccess) {
    cudaFreeAsync(buf, stream);
    return WKV_ERR_CUDA;
  }
  char* p = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(buf) + 255) & ~uintptr_t(255));
  auto take = [&](size_t bytes) {
    float* q = reinterpret_cast<float*>(p);
    p += bytes;
    return q;
  };
  float *k = take(n), *v = take(n), *r = take(n), *dy = take(n), *dk = take(n), *dv = take(n),
        *dr = take(n), *w = take(c4), *u = take(c4), *dw = take(c4), *du = take(c4);
  void* ws = p;
  unsigned* err = error_word();
  int rc = err ? WKV_OK : WKV_ERR_CUDA;
  if (rc == WKV_OK) {
    BwdArgs a{B, T, C, w, u, k, v, r, dy, dk, dv, dw, du, dr, ws, err};
    a.wait_ns = (unsigned long long)wait_ns;
    a.withhold_last_map = 1;
    rc = launch_backward(a, false, stream);
  }
  cudaFreeAsync(buf, stream);
  return rc;
}

WKV_API int wkv_testing_forward_plain(int64_t B, int64_t T, int64_t C, const float* w,
                                      const float* u, const void* k, const void* v,
                                      const void* r, void* y, int bf16, cudaStream_t stream) {
  int rc = check_fwd(B, T, C, w, u, k, v, r, y, bf16 ? 2 : 4);
  if (rc != WKV_OK || B == 0 || C == 0 || T == 0) return rc;
  unsigned* err = error_word();
  if (err == nullptr) return WKV_ERR_CUDA;
  FwdArgs a{B, T, C, w, u, k, v, r, y, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, err};
  return launch_fwd_stream(a, bf16 != 0, /*force_plain=*/true, stream);
}

WKV_API int wkv_testing_set_backward_path(int path) {
  if (path < 0 || path > 3) return WKV_ERR_INVALID_ARG;
  set_backward_path(path);
  return WKV_OK;
}

WKV_API int wkv_testing_backward_plain(int64_t B, int64_t T, int64_t C, const float* w,
                                       const float* u, const float* k, const float* v,
                                       const float* r, const float* dy, float* dk, float* dv,
                                       float* dw, float* du, float* dr, void* workspace,
                                       size_t workspace_bytes, cudaStream_t stream) {
  return backward_impl(B, T, C, w, u, k, v, r, dy, dk, dv, dw, du, dr, workspace,
                       workspace_bytes, true, stream);
}

WKV_API int wkv_testing_backward_state_plain(
    int64_t B, int64_t T, int64_t C, const float* w, const float* u, const float* k,
    const float* v, const float* r, const float* dy, const float* a0, const float* b0,
    const float* p0, const float* ga1, const float* gb1, const float* p1, float* dk, float* dv,
    float* dw, float* du, float* dr, float* da0, float* db0, float* dp0, void* workspace,
    size_t workspace_bytes, cudaStream_t stream) {
  StateArgs st;
  st.a0 = a0; st.b0 = b0; st.p0 = p0;
  st.ga1 = ga1; st.gb1 = gb1; st.p1 = p1;
  st.da0 = da0; st.db0 = db0; st.dp0 = dp0;
  return backward_impl(B, T, C, w, u, k, v, r, dy, dk, dv, dw, du, dr, workspace,
                       workspace_bytes, true, stream, st);
}

}  // extern "C"
