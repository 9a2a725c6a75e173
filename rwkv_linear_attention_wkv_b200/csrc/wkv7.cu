// RWKV-7 generalised-delta-rule recurrence per head (sm_100a).
//
// The research report "RWKV模型深度研究报告（截至2026年初）", section 1.3.3 "RWKV-7 (Goose)",
// gives the state update with a matrix state S per head, input-dependent decay w_t and
// in-context-learning vectors a_t, b_t:
//   S_t = S_{t-1} (diag(w_t) + a_t^T b_t) + v_t^T k_t,
// i.e. for row i (value channel) and column j (key channel)
//   S_t[i][j] = S_{t-1}[i][j] w_t[j] + sa_i b_t[j] + v_t[i] k_t[j],  sa_i = sum_l S_{t-1}[i][l] a_t[l].
// The report gives no read-out; this library reads the state with the receptance as the
// query, y_t = S_t r_t^T.
//
// One CTA per (batch row, head) of head size N = 64, 128 threads: thread pair (2i, 2i+1)
// holds row i of S in registers, 32 columns each. The per-token vectors r, w, k, v, a, b
// ([64] fp32 each) come in TMA tiles of kT7 tokens through a kS7-stage mbarrier pipeline;
// y is staged in shared memory and TMA-stored a tile at a time. Per token and thread:
// sa (32 FMA + one shuffle), the update (3 operations per element), y (32 FMA + one
// shuffle). Bound: the FP32 pipe (about 5 N^2 operations per token per head).
#include "wkv_device.cuh"
#include "wkv_internal.h"

namespace wkv {

namespace {

constexpr int kN7 = 64;        // head size
constexpr int kT7 = 8;         // tokens per tile
constexpr int kS7 = 4;         // pipeline stages
constexpr int kHalf = kN7 / 2; // columns per thread
constexpr int kTile7 = kT7 * kN7;  // floats per tensor tile

struct Wkv7Maps {
  CUtensorMap r, w, k, v, a, b, y;
};

__global__ void __launch_bounds__(2 * kN7) wkv7_fwd_kernel(const __grid_constant__ Wkv7Maps maps,
                                                          int B, int T, int H,
                                                          const float* __restrict__ s0,
                                                          float* __restrict__ s1,
                                                          unsigned* err) {
  // stage st: tiles r, w, k, v, a, b at smem + (6 st + slot) kTile7; y tiles after them
  extern __shared__ __align__(128) float smem7[];
  float* ybuf = smem7 + 6 * kS7 * kTile7;  // [2][kT7][64]
  __shared__ uint64_t bars[kS7];
  const int tid = threadIdx.x;
  const int i = tid >> 1;            // row of S
  const int c0 = (tid & 1) * kHalf;  // first column of this thread
  const int bh = blockIdx.x;
  const int b = bh / H, h = bh - b * H;
  const int ntile = (T + kT7 - 1) / kT7;

  auto issue = [&](int st, int tile) {
    uint64_t* bar = &bars[st];
    mbar_arrive_expect_tx(bar, 6u * kTile7 * sizeof(float));
    float* dst = smem7 + 6 * st * kTile7;
    const int x = h * kN7, t0 = tile * kT7;
    tma_load_3d(dst + 0 * kTile7, &maps.r, bar, x, t0, b);
    tma_load_3d(dst + 1 * kTile7, &maps.w, bar, x, t0, b);
    tma_load_3d(dst + 2 * kTile7, &maps.k, bar, x, t0, b);
    tma_load_3d(dst + 3 * kTile7, &maps.v, bar, x, t0, b);
    tma_load_3d(dst + 4 * kTile7, &maps.a, bar, x, t0, b);
    tma_load_3d(dst + 5 * kTile7, &maps.b, bar, x, t0, b);
  };
  if (tid == 0) {
    for (int st = 0; st < kS7; ++st) mbar_init(&bars[st], 1);
    mbar_fence_init();
    for (int st = 0; st < kS7 && st < ntile; ++st) issue(st, st);
  }
  __syncthreads();

  float S[kHalf];
  {
    const float* src = s0 ? s0 + (size_t(bh) * kN7 + i) * kN7 + c0 : nullptr;
#pragma unroll
    for (int j = 0; j < kHalf; j += 4) {
      const float4 q = src ? *reinterpret_cast<const float4*>(src + j) : make_float4(0, 0, 0, 0);
      S[j] = q.x;
      S[j + 1] = q.y;
      S[j + 2] = q.z;
      S[j + 3] = q.w;
    }
  }

  for (int tile = 0; tile < ntile; ++tile) {
    const int st = tile % kS7;
    mbar_wait(&bars[st], (tile / kS7) & 1, err);
    const float* base = smem7 + 6 * st * kTile7;
    float* yt = ybuf + (tile & 1) * kTile7;
    if (tile >= 2 && tid == 0) tma_store_wait_read<1>();  // this y buffer's last store has read it
    __syncthreads();
    const int n = min(kT7, T - tile * kT7);
    for (int t = 0; t < n; ++t) {
      const float* R = base + 0 * kTile7 + t * kN7 + c0;
      const float* W = base + 1 * kTile7 + t * kN7 + c0;
      const float* K = base + 2 * kTile7 + t * kN7 + c0;
      const float vi = base[3 * kTile7 + t * kN7 + i];
      const float* A = base + 4 * kTile7 + t * kN7 + c0;
      const float* Bv = base + 5 * kTile7 + t * kN7 + c0;
      // sa_i = S_{t-1}[i] . a_t, four partial sums for instruction-level parallelism
      float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
#pragma unroll
      for (int j = 0; j < kHalf; j += 4) {
        const float4 q = *reinterpret_cast<const float4*>(A + j);
        p0 = fmaf(S[j], q.x, p0);
        p1 = fmaf(S[j + 1], q.y, p1);
        p2 = fmaf(S[j + 2], q.z, p2);
        p3 = fmaf(S[j + 3], q.w, p3);
      }
      float sa = (p0 + p1) + (p2 + p3);
      sa += __shfl_xor_sync(0xffffffffu, sa, 1);
      // S_t[i][j] = S[i][j] w_j + sa_i b_j + v_i k_j;  y_i = S_t[i] . r_t
      float y0 = 0.f, y1 = 0.f, y2 = 0.f, y3 = 0.f;
#pragma unroll
      for (int j = 0; j < kHalf; j += 4) {
        const float4 wq = *reinterpret_cast<const float4*>(W + j);
        const float4 kq = *reinterpret_cast<const float4*>(K + j);
        const float4 bq = *reinterpret_cast<const float4*>(Bv + j);
        const float4 rq = *reinterpret_cast<const float4*>(R + j);
        S[j] = fmaf(S[j], wq.x, fmaf(sa, bq.x, vi * kq.x));
        S[j + 1] = fmaf(S[j + 1], wq.y, fmaf(sa, bq.y, vi * kq.y));
        S[j + 2] = fmaf(S[j + 2], wq.z, fmaf(sa, bq.z, vi * kq.z));
        S[j + 3] = fmaf(S[j + 3], wq.w, fmaf(sa, bq.w, vi * kq.w));
        y0 = fmaf(S[j], rq.x, y0);
        y1 = fmaf(S[j + 1], rq.y, y1);
        y2 = fmaf(S[j + 2], rq.z, y2);
        y3 = fmaf(S[j + 3], rq.w, y3);
      }
      float yv = (y0 + y1) + (y2 + y3);
      yv += __shfl_xor_sync(0xffffffffu, yv, 1);
      if ((tid & 1) == 0) yt[t * kN7 + i] = yv;
    }
    fence_proxy_async_smem();  // the y tile's writes, visible to the TMA store
    __syncthreads();           // the stage is consumed and the y tile complete
    if (tid == 0) {
      tma_store_3d(&maps.y, yt, h * kN7, tile * kT7, b);
      tma_store_commit();
      if (tile + kS7 < ntile) issue(st, tile + kS7);
    }
  }
  if (s1 != nullptr) {
    float* dst = s1 + (size_t(bh) * kN7 + i) * kN7 + c0;
#pragma unroll
    for (int j = 0; j < kHalf; j += 4)
      *reinterpret_cast<float4*>(dst + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
  }
  if (tid == 0) tma_store_wait_all();
}

}  // namespace

int launch_wkv7(int64_t B, int64_t T, int64_t H, const float* r, const float* w, const float* k,
                const float* v, const float* a, const float* b, float* y, const float* s0,
                float* s1, unsigned* err, cudaStream_t stream) {
  const int64_t C = H * kN7;
  Wkv7Maps m;
  const auto dt = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const struct {
    CUtensorMap* map;
    const void* p;
  } tabs[7] = {{&m.r, r}, {&m.w, w}, {&m.k, k}, {&m.v, v}, {&m.a, a}, {&m.b, b}, {&m.y, y}};
  for (const auto& e : tabs)
    if (int rc = encode_btc_map(e.map, e.p, dt, 4, B, T, C, kN7, kT7)) return rc;
  const size_t smem = (6 * kS7 + 2) * size_t(kTile7) * sizeof(float);
  if (cudaFuncSetAttribute(wkv7_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           int(smem)) != cudaSuccess)
    return WKV_ERR_CUDA;
  wkv7_fwd_kernel<<<unsigned(B * H), 2 * kN7, smem, stream>>>(m, int(B), int(T), int(H), s0, s1,
                                                              err);
  return cudaPeekAtLastError() == cudaSuccess ? WKV_OK : WKV_ERR_CUDA;
}

}  // namespace wkv
