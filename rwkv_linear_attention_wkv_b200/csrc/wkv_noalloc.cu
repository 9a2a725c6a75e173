// wkv_forward_state_static: the stateful forward without any device allocation.
//
// Who needs it: callers that cannot call cudaMalloc / cudaMallocAsync at the point where
// they run the operator, e.g. a serving loop that must not risk the implicit device
// synchronisation an allocation can cause, an application whose memory manager owns all
// device memory and forbids raw allocations, or a deployment that permits no dynamic
// allocation once it has started. wkv_forward_state allocates the scratch of its
// chunked path with cudaMallocAsync; this variant takes that scratch from a fixed array in
// the library's own device memory instead.
//
// The array below is a file-scope __device__ object: every GPU that loads the library
// holds its kStaticScratchBytes until the process exits. In host code its name is only a
// host-side stand-in, never a device address, so the device address is looked up with
// cudaGetSymbolAddress once per device (on the first call made with that device current)
// and cached.
#include <mutex>

#include "wkv_internal.h"

namespace wkv {

namespace {

// 8 MiB + 64 KiB. The chunked path needs 1 KiB of carries per item (batch row x
// 32-channel group x 256-token segment) plus a 4-byte flag per item and a 16-byte ticket
// header, so this holds up to 8223 items: e.g. one sequence of 32768 tokens x 2048
// channels (8192 items, 8,421,392 bytes); one more segment (33024 tokens, 8256 items) is
// over the limit.
constexpr size_t kStaticScratchBytes = (size_t(8) << 20) + (size_t(64) << 10);

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;

// Device address of g_static_scratch on the current device; nullptr (and *rc set) on error.
void* static_scratch(int* rc) {
  static void* addr[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *rc = WKV_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) {
      *rc = WKV_ERR_CUDA;
      return nullptr;
    }
    addr[dev] = p;
  }
  return addr[dev];
}

bool al(const void* p, size_t a) { return p == nullptr || reinterpret_cast<uintptr_t>(p) % a == 0; }

}  // namespace

}  // namespace wkv

using namespace wkv;

extern "C" WKV_API int wkv_forward_state_static(int64_t B, int64_t T, int64_t C, const float* w,
                                                const float* u, const float* k, const float* v,
                                                const float* r, float* y, const float* a0,
                                                const float* b0, const float* p0, float* a1,
                                                float* b1, float* p1, cudaStream_t stream) {
  if (B < 0 || T < 0 || C < 0) return WKV_ERR_INVALID_ARG;
  if ((a0 == nullptr) != (b0 == nullptr) || (a0 == nullptr) != (p0 == nullptr) ||
      (a1 == nullptr) != (b1 == nullptr) || (a1 == nullptr) != (p1 == nullptr))
    return WKV_ERR_INVALID_ARG;
  if (B == 0 || C == 0) return WKV_OK;
  if (!w || !u || (T > 0 && (!k || !v || !y))) return WKV_ERR_INVALID_ARG;
  const void* ptrs[] = {w, u, k, v, r, y, a0, b0, p0, a1, b1, p1};
  for (const void* q : ptrs)
    if (!al(q, 4)) return WKV_ERR_ALIGNMENT;
  if (T >= (int64_t(1) << 31) || C >= (int64_t(1) << 31) || B >= (int64_t(1) << 31) ||
      (T > 0 && B > INT64_MAX / T / C))
    return WKV_ERR_UNSUPPORTED;
  if (T == 0 && a1 == nullptr) return WKV_OK;
  unsigned* err = device_error_word();
  if (err == nullptr) return WKV_ERR_CUDA;
  FwdArgs a{B, T, C, w, u, k, v, r, y, a0, b0, p0, a1, b1, p1, err};
  int64_t flag_bytes = 0;
  int nseg = 1;
  const size_t need = T > 0 ? chunked_scratch_bytes(B, T, C, &flag_bytes, &nseg) : 0;
  if (nseg <= 1) return launch_fwd_stream(a, false, /*force_plain=*/T == 0, stream);
  if (need > kStaticScratchBytes) return WKV_ERR_SCRATCH_LIMIT;
  int rc = WKV_OK;
  void* scratch = static_scratch(&rc);
  if (scratch == nullptr) return rc;
  // The flags and the segment ticket must start at zero; the rest of the
  // scratch is written before it is read.
  if (cudaMemsetAsync(scratch, 0, size_t(flag_bytes), stream) != cudaSuccess) return WKV_ERR_CUDA;
  return launch_fwd_chunked(a, scratch, nseg, stream);
}
