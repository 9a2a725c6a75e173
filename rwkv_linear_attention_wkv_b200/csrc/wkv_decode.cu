// One recurrent-inference token for N sequences x L layers x C channels (sm_100a).
//
// Single-token step of the paper notes "RWKV - 把 RNN 重新带回 Transformer 时代的线性大模型",
// "关键设计 4" (only the state is kept between tokens) with the output and update rules of
// "一句话总结". Purely elementwise and bound by HBM traffic (read k, v, r, a, b, p; write
// y, a, b, p: 40 bytes per state), so each thread handles four adjacent channels with
// 16-byte loads and stores when C and the pointers allow it; w and u ([L, C], shared by
// all N sequences) come from L2.
//
// State (a, b, p): numerator a e^p, denominator b e^p, p natural-log. Output against the
// state before the token, each side stabilised by its own maximum:
//   dO = (u + k) - p:   wkv = (o1 a + o2 v) / (o1 b + o2),  {o1, o2} = {2^{-|dO| log2 e}, 1}
//   d  = k - (p - w):   a' = e1 a + e2 v, b' = e1 b + e2, p' = max(p - w, k).
//
// Several chained tokens per launch (wkv_decode_steps): the news page "RWKV CUDA linear
// attention GPU" (技术深度解析, 持久化内核设计) describes a kernel that stays resident
// across token generations instead of being relaunched per token. Here each thread keeps
// its four channels' (a, b, p) in registers over the S tokens it is given, reading each
// token's k, v, r and writing its y, so the state crosses HBM once per launch rather than
// once per token: 16 + 24/S bytes per state and token instead of 40. The arithmetic per
// token is decode_one, so S tokens in one launch give bit for bit what S single-token
// launches give.
#include <algorithm>

#include "wkv_internal.h"
#include "wkv_step.cuh"

namespace wkv {

template <bool GATE>
__device__ __forceinline__ void decode_one(float w, float u, float k, float v, float r, float& y,
                                           float& a, float& b, float& p) {
  const float dO = (u + k) - p;
  const float o = ex2(-fabsf(dO) * kLog2e);
  const bool co = dO > 0.f;
  const float o1 = co ? o : 1.f;
  const float o2 = co ? 1.f : o;
  const float num = fmaf(o1, a, o2 * v);
  float den = fmaf(o1, b, o2);
  if (GATE) {
    const float er = ex2(r * -kLog2e);
    den = fmaf(den, er, den);
  }
  y = num * rcp(den);
  const float pw = p - w;
  const float d = k - pw;
  const float e = ex2(-fabsf(d) * kLog2e);
  const bool c = d > 0.f;
  const float e1 = c ? e : 1.f;
  const float e2 = c ? 1.f : e;
  a = fmaf(e1, a, e2 * v);
  b = fmaf(e1, b, e2);
  p = fmaxf(pw, k);
}

// Four channels per thread; requires C % 4 == 0 and 16-byte aligned pointers.
template <bool GATE>
__global__ void __launch_bounds__(256) wkv_decode_vec4_kernel(
    int64_t n4, int64_t LC4, int64_t C4, const float4* __restrict__ w, const float4* __restrict__ u,
    const float4* __restrict__ k, const float4* __restrict__ v, const float4* __restrict__ r,
    float4* __restrict__ y, float4* a, float4* b, float4* p) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t lc = i % LC4;  // (layer, channel/4) index into w, u
    const float4 ww = __ldg(&w[lc]), uu = __ldg(&u[lc]);
    const float4 kk = __ldcs(&k[i]), vv = __ldcs(&v[i]);
    const float4 rr = GATE ? __ldcs(&r[i]) : make_float4(0.f, 0.f, 0.f, 0.f);
    float4 aa = a[i], bb = b[i], pp = p[i], yy;
    decode_one<GATE>(ww.x, uu.x, kk.x, vv.x, rr.x, yy.x, aa.x, bb.x, pp.x);
    decode_one<GATE>(ww.y, uu.y, kk.y, vv.y, rr.y, yy.y, aa.y, bb.y, pp.y);
    decode_one<GATE>(ww.z, uu.z, kk.z, vv.z, rr.z, yy.z, aa.z, bb.z, pp.z);
    decode_one<GATE>(ww.w, uu.w, kk.w, vv.w, rr.w, yy.w, aa.w, bb.w, pp.w);
    __stcs(&y[i], yy);
    a[i] = aa;
    b[i] = bb;
    p[i] = pp;
  }
  (void)C4;
}

template <bool GATE>
__global__ void __launch_bounds__(256) wkv_decode_scalar_kernel(
    int64_t n, int64_t LC, const float* __restrict__ w, const float* __restrict__ u,
    const float* __restrict__ k, const float* __restrict__ v, const float* __restrict__ r,
    float* __restrict__ y, float* a, float* b, float* p) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t lc = i % LC;
    float aa = a[i], bb = b[i], pp = p[i], yy;
    decode_one<GATE>(w[lc], u[lc], k[i], v[i], GATE ? r[i] : 0.f, yy, aa, bb, pp);
    y[i] = yy;
    a[i] = aa;
    b[i] = bb;
    p[i] = pp;
  }
}

// S chained tokens, four channels per thread; k, v, r, y are [S, N, L, C] (a token plane
// of n4 float4 per step); requires C % 4 == 0 and 16-byte aligned pointers. The next
// token's k, v, r are loaded before this token is computed, so each thread keeps one
// token of loads in flight behind its serial chain through the state.
template <bool GATE>
__global__ void __launch_bounds__(256) wkv_decode_steps_vec4_kernel(
    int64_t n4, int64_t LC4, int S, const float4* __restrict__ w, const float4* __restrict__ u,
    const float4* __restrict__ k, const float4* __restrict__ v, const float4* __restrict__ r,
    float4* __restrict__ y, float4* __restrict__ a, float4* __restrict__ b,
    float4* __restrict__ p) {
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  const int64_t lc = i % LC4;
  const float4 ww = __ldg(&w[lc]), uu = __ldg(&u[lc]);
  float4 aa = a[i], bb = b[i], pp = p[i];
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
  float4 kk = __ldcs(&k[i]), vv = __ldcs(&v[i]);
  float4 rr = GATE ? __ldcs(&r[i]) : zero;
  for (int s = 0; s < S; ++s) {
    const int64_t cur = int64_t(s) * n4 + i;
    float4 kn = zero, vn = zero, rn = zero;
    if (s + 1 < S) {
      const int64_t nxt = cur + n4;
      kn = __ldcs(&k[nxt]);
      vn = __ldcs(&v[nxt]);
      if (GATE) rn = __ldcs(&r[nxt]);
    }
    float4 yy;
    decode_one<GATE>(ww.x, uu.x, kk.x, vv.x, rr.x, yy.x, aa.x, bb.x, pp.x);
    decode_one<GATE>(ww.y, uu.y, kk.y, vv.y, rr.y, yy.y, aa.y, bb.y, pp.y);
    decode_one<GATE>(ww.z, uu.z, kk.z, vv.z, rr.z, yy.z, aa.z, bb.z, pp.z);
    decode_one<GATE>(ww.w, uu.w, kk.w, vv.w, rr.w, yy.w, aa.w, bb.w, pp.w);
    __stcs(&y[cur], yy);
    kk = kn;
    vv = vn;
    rr = rn;
  }
  a[i] = aa;
  b[i] = bb;
  p[i] = pp;
}

// The same, one channel per thread, for any C and 4-byte aligned pointers.
template <bool GATE>
__global__ void __launch_bounds__(256) wkv_decode_steps_scalar_kernel(
    int64_t n, int64_t LC, int S, const float* __restrict__ w, const float* __restrict__ u,
    const float* __restrict__ k, const float* __restrict__ v, const float* __restrict__ r,
    float* __restrict__ y, float* __restrict__ a, float* __restrict__ b,
    float* __restrict__ p) {
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int64_t lc = i % LC;
  const float ww = w[lc], uu = u[lc];
  float aa = a[i], bb = b[i], pp = p[i];
  for (int s = 0; s < S; ++s) {
    const int64_t cur = int64_t(s) * n + i;
    float yy;
    decode_one<GATE>(ww, uu, k[cur], v[cur], GATE ? r[cur] : 0.f, yy, aa, bb, pp);
    y[cur] = yy;
  }
  a[i] = aa;
  b[i] = bb;
  p[i] = pp;
}

int launch_decode_steps(const DecodeArgs& d, int64_t S, cudaStream_t stream) {
  const int64_t n = d.N * d.L * d.C;
  if (n == 0 || S == 0) return WKV_OK;
  auto al16 = [](const void* q) {
    return q == nullptr || (reinterpret_cast<uintptr_t>(q) & 15) == 0;
  };
  const bool vec = d.C % 4 == 0 && al16(d.w) && al16(d.u) && al16(d.k) && al16(d.v) &&
                   al16(d.r) && al16(d.y) && al16(d.a) && al16(d.b) && al16(d.p);
  const int block = 256;
  const int64_t items = vec ? n / 4 : n;
  const int64_t grid = (items + block - 1) / block;
  if (grid >= (int64_t(1) << 31)) return WKV_ERR_UNSUPPORTED;
  const bool gate = d.r != nullptr;
  const int s32 = int(S);
  if (vec) {
    auto f4 = [](const float* q) { return reinterpret_cast<const float4*>(q); };
    auto m4 = [](float* q) { return reinterpret_cast<float4*>(q); };
    const int64_t LC4 = d.L * d.C / 4;
    if (gate)
      wkv_decode_steps_vec4_kernel<true><<<unsigned(grid), block, 0, stream>>>(
          items, LC4, s32, f4(d.w), f4(d.u), f4(d.k), f4(d.v), f4(d.r), m4(d.y), m4(d.a),
          m4(d.b), m4(d.p));
    else
      wkv_decode_steps_vec4_kernel<false><<<unsigned(grid), block, 0, stream>>>(
          items, LC4, s32, f4(d.w), f4(d.u), f4(d.k), f4(d.v), nullptr, m4(d.y), m4(d.a),
          m4(d.b), m4(d.p));
  } else {
    const int64_t LC = d.L * d.C;
    if (gate)
      wkv_decode_steps_scalar_kernel<true><<<unsigned(grid), block, 0, stream>>>(
          items, LC, s32, d.w, d.u, d.k, d.v, d.r, d.y, d.a, d.b, d.p);
    else
      wkv_decode_steps_scalar_kernel<false><<<unsigned(grid), block, 0, stream>>>(
          items, LC, s32, d.w, d.u, d.k, d.v, nullptr, d.y, d.a, d.b, d.p);
  }
  return cudaPeekAtLastError() == cudaSuccess ? WKV_OK : WKV_ERR_CUDA;
}

int launch_decode(const DecodeArgs& d, cudaStream_t stream) {
  const int64_t n = d.N * d.L * d.C;
  if (n == 0) return WKV_OK;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  auto al16 = [](const void* q) {
    return q == nullptr || (reinterpret_cast<uintptr_t>(q) & 15) == 0;
  };
  const bool vec = d.C % 4 == 0 && al16(d.w) && al16(d.u) && al16(d.k) && al16(d.v) &&
                   al16(d.r) && al16(d.y) && al16(d.a) && al16(d.b) && al16(d.p);
  const int block = 256;
  const int64_t items = vec ? n / 4 : n;
  // Enough resident blocks to cover the SMs several times; grid-stride beyond that.
  const int64_t grid = std::min<int64_t>((items + block - 1) / block, int64_t(sms) * 16);
  const bool gate = d.r != nullptr;
  if (vec) {
    auto f4 = [](const float* q) { return reinterpret_cast<const float4*>(q); };
    auto m4 = [](float* q) { return reinterpret_cast<float4*>(q); };
    const int64_t LC4 = d.L * d.C / 4;
    if (gate)
      wkv_decode_vec4_kernel<true><<<unsigned(grid), block, 0, stream>>>(
          items, LC4, d.C / 4, f4(d.w), f4(d.u), f4(d.k), f4(d.v), f4(d.r), m4(d.y), m4(d.a),
          m4(d.b), m4(d.p));
    else
      wkv_decode_vec4_kernel<false><<<unsigned(grid), block, 0, stream>>>(
          items, LC4, d.C / 4, f4(d.w), f4(d.u), f4(d.k), f4(d.v), nullptr, m4(d.y), m4(d.a),
          m4(d.b), m4(d.p));
  } else {
    const int64_t LC = d.L * d.C;
    if (gate)
      wkv_decode_scalar_kernel<true><<<unsigned(grid), block, 0, stream>>>(
          items, LC, d.w, d.u, d.k, d.v, d.r, d.y, d.a, d.b, d.p);
    else
      wkv_decode_scalar_kernel<false><<<unsigned(grid), block, 0, stream>>>(
          items, LC, d.w, d.u, d.k, d.v, nullptr, d.y, d.a, d.b, d.p);
  }
  return cudaPeekAtLastError() == cudaSuccess ? WKV_OK : WKV_ERR_CUDA;
}

}  // namespace wkv
