// WKV backward: dk, dv (and dr), dw, du for L = sum_t dy_t . y_t (sm_100a).
//
// The pages state only that the operator trains with ordinary backpropagation (news page
// "RWKV CUDA linear attention GPU": fused forward/backward kernels and an autograd
// function). Gradients follow from the parallel form (concept page, section 3.2) by the
// chain rule. With h_t = dy_t sigmoid(r_t) / D_t (D_t the output denominator) and sums
// over t > i:
//   beta_i  = sum h_t e^{-(t-1-i)w},   gamma_i  = sum h_t wkv_t e^{-(t-1-i)w},
//   betad_i = sum (t-1-i) h_t e^{..},  gammad_i = sum (t-1-i) h_t wkv_t e^{..},
//   dv_i = e^{k_i} (h_i e^u + beta_i),
//   dk_i = e^{k_i} (h_i e^u (v_i - wkv_i) + v_i beta_i - gamma_i),
//   dw   = -sum e^{k_i} (v_i betad_i - gammad_i),   du = sum h_t e^{u+k_t} (v_t - wkv_t),
//   dr_t = dy_t wkv_t sigmoid(r_t) (1 - sigmoid(r_t)),
// with beta_{i-1} = h_i + e^{-w} beta_i and betad_{i-1} = e^{-w} (betad_i + beta_i).
//
// Stabilisation without a reverse scale of its own: the accumulators are carried scaled
// by the forward state's scale at the same token, X~_i = X_i 2^{P_i}. Since
// P_i = max(P_{i-1} - w2, k_i log2 e), the factor 2^{P_{i-1} - w2 - P_i} is exactly the
// forward update's e1_i and 2^{k_i log2 e - P_i} its e2_i, so
//   beta~_{i-1}  = inj_i + e1_i beta~_i,      gamma~_{i-1}  = inj_i wkv_i + e1_i gamma~_i,
//   betad~_{i-1} = e1_i (betad~_i + beta~_i), gammad~_{i-1} = e1_i (gammad~_i + gamma~_i),
//   dv_i = cur_i + e2_i beta~_i,  dk_i = cur_i (v_i - wkv_i) + e2_i (v_i beta~_i - gamma~_i),
// where inj_i = h_i 2^{P_{i-1}} and cur_i = h_i e^{u+k_i} are dy_i times per-token factors
// of the forward recomputation. Every factor is <= 1 and the accumulators stay bounded by
// sums of |dy sigmoid(r) / den|: no exponential in the reverse pass, nothing to overflow,
// and the scale is the forward's exact windowed one, so nothing drifts.
//
// Two kernels plus a reduction:
//   1. checkpoint: one warp per 32 channels streams k, v forward (TMA) and stores the
//      state entering every chunk of TT tokens;
//   2. reverse: one warp per 32 channels walks the chunks from last to first; for each it
//      loads k, v, r, dy, recomputes the forward factors from the chunk's checkpoint into
//      shared memory, then runs the reverse recurrences and writes dk, dv (dr) in place of
//      k, v (r) in shared memory for TMA stores; per-(b, c) partial sums of dw, du go to
//      the workspace;
//   3. reduce: dw[c], du[c] = sums over b in a fixed order (deterministic).
#include <algorithm>

#include "wkv_internal.h"
#include "wkv_step.cuh"

namespace wkv {

namespace {

constexpr int kTT = 32;  // tokens per chunk

struct BwdLayout {
  float4* ckpt;  // [B, nchunks, C] state entering each chunk: (a, b, Q, pl)
  float* pdw;    // [B, C]
  float* pdu;    // [B, C]
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

__host__ __device__ inline BwdLayout bwd_layout(void* ws, int64_t B, int64_t T, int64_t C) {
  const int64_t nch = (T + kTT - 1) / kTT;
  char* p = static_cast<char*>(ws);
  BwdLayout L;
  L.ckpt = reinterpret_cast<float4*>(p);
  p += align256(size_t(B) * nch * C * sizeof(float4));
  L.pdw = reinterpret_cast<float*>(p);
  p += align256(size_t(B) * C * sizeof(float));
  L.pdu = reinterpret_cast<float*>(p);
  return L;
}

__host__ __device__ inline size_t bwd_bytes(int64_t B, int64_t T, int64_t C) {
  const int64_t nch = (T + kTT - 1) / kTT;
  return align256(size_t(B) * nch * C * sizeof(float4)) + 2 * align256(size_t(B) * C * sizeof(float));
}

// ---- tile movement: TMA, or plain per-lane loads/stores for unaligned shapes ----------
// Up to four global tensors addressed by slot (no pointer arrays: they would live in local
// memory).
struct Ptr4 {
  const float* p0;
  const float* p1;
  const float* p2;
  const float* p3;
  __device__ __forceinline__ const float* operator[](int i) const {
    return i == 0 ? p0 : (i == 1 ? p1 : (i == 2 ? p2 : p3));
  }
};
struct MPtr3 {
  float* p0;
  float* p1;
  float* p2;
  __device__ __forceinline__ float* operator[](int i) const {
    return i == 0 ? p0 : (i == 1 ? p1 : p2);
  }
};

// Tiles of [kTT tokens x 32 channels] fp32; the nt tiles of one transfer are consecutive in
// shared memory (kTT * 32 floats apart), tensor i paired with map i / pointer slot i.
template <bool TMA>
struct Tiles {
  static __device__ __forceinline__ void load(const CUtensorMap* maps, const Ptr4& ptrs, int nt,
                                              float* dst, uint64_t* bar, int b, int g, int t0,
                                              int T, int C, int lane) {
    if (TMA) {
      if (lane == 0) {
        mbar_arrive_expect_tx(bar, uint32_t(nt) * kTT * 32 * sizeof(float));
        for (int i = 0; i < nt; ++i)
          tma_load_3d(dst + i * kTT * 32, &maps[i], bar, g << 5, t0, b);
      }
    } else {
      const int c = (g << 5) + lane;
      for (int i = 0; i < nt; ++i) {
        const float* src = ptrs[i];
        for (int t = 0; t < kTT; ++t) {
          const int tt = t0 + t;
          dst[i * kTT * 32 + t * 32 + lane] =
              (c < C && tt < T) ? src[(int64_t(b) * T + tt) * C + c] : 0.f;
        }
      }
    }
  }
  static __device__ __forceinline__ void wait(uint64_t* bar, uint32_t parity, unsigned* err) {
    if (TMA) mbar_wait(bar, parity, err);
    __syncwarp();
  }
  static __device__ __forceinline__ void store(const CUtensorMap* maps, const MPtr3& ptrs, int nt,
                                               const float* src, int b, int g, int t0, int T,
                                               int C, int lane) {
    if (TMA) {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        for (int i = 0; i < nt; ++i) tma_store_3d(&maps[i], src + i * kTT * 32, g << 5, t0, b);
        tma_store_commit();
      }
    } else {
      __syncwarp();
      const int c = (g << 5) + lane;
      if (c < C)
        for (int i = 0; i < nt; ++i) {
          float* dst = ptrs[i];
          for (int t = 0; t < kTT && t0 + t < T; ++t)
            dst[(int64_t(b) * T + t0 + t) * C + c] = src[i * kTT * 32 + t * 32 + lane];
        }
    }
  }
  static __device__ __forceinline__ void store_drain(int lane) {
    if (TMA && lane == 0) tma_store_wait_all();
    __syncwarp();
  }
};

struct TensorMaps4 {
  CUtensorMap m[4];
};

// ---- 1. checkpoints --------------------------------------------------------------------
template <bool TMA>
__global__ void __launch_bounds__(32) wkv_bwd_ckpt_kernel(const __grid_constant__ TensorMaps4 maps,
                                                          const float* __restrict__ k,
                                                          const float* __restrict__ v,
                                                          int B, int T, int C,
                                                          const float* __restrict__ w,
                                                          void* ws, unsigned* err) {
  constexpr int S = 3;
  constexpr int kTile = kTT * 32;
  __shared__ __align__(128) float tiles[S][2][kTile];  // per stage: k, v
  __shared__ uint64_t bars[S];
  const int lane = threadIdx.x;
  const int G = (C + 31) >> 5;
  const int b = blockIdx.x / G, g = blockIdx.x % G;
  const int c = (g << 5) + lane;
  const bool valid = c < C;
  const int nch = (T + kTT - 1) / kTT;
  const BwdLayout lay = bwd_layout(ws, B, T, C);
  const Ptr4 ptrs{k, v, nullptr, nullptr};

  auto issue = [&](int st, int ch) {
    Tiles<TMA>::load(maps.m, ptrs, 2, &tiles[st][0][0], &bars[st], b, g, ch * kTT, T, C, lane);
  };
  if (lane == 0) {
    for (int st = 0; st < S; ++st) mbar_init(&bars[st], 1);
    mbar_fence_init();
  }
  __syncwarp();
  for (int st = 0; st < S && st < nch; ++st) issue(st, st);

  ChanParams cp = chan_params(valid ? w[c] : 1.f, 0.f);
  const int rb = window_tokens(cp.w2, 128.f);
  ChanState s = empty_state();
  for (int ch = 0; ch < nch; ++ch) {
    const int st = ch % S;
    if (valid) lay.ckpt[(int64_t(b) * nch + ch) * C + c] = make_float4(s.a, s.b, s.Q, s.pl);
    Tiles<TMA>::wait(&bars[st], (ch / S) & 1, err);
    const int n = min(kTT, T - ch * kTT);
    int j = 0;
    for (int t = 0; t < n; ++t) {
      wkv_absorb(s, cp, float(j + 1), tiles[st][0][t * 32 + lane], tiles[st][1][t * 32 + lane]);
      if (++j == rb) {
        wkv_rebase(s, float(rb) * cp.w2);
        j = 0;
      }
    }
    if (j) wkv_rebase_partial(s, j, cp.w2);
    __syncwarp();
    if (ch + S < nch) issue(st, ch + S);
  }
}

// ---- 2. reverse pass ---------------------------------------------------------------------
// Shared memory per CTA (floats): 2 stages x 4 tiles (k, v, r, dy; dk, dv, dr written in
// place of k, v, r) + 6 factor tiles (e1, e2, f_inj, f_cur, wkv, sigma).
template <bool TMA, bool GATE, bool DR>
__global__ void __launch_bounds__(32) wkv_bwd_main_kernel(
    const __grid_constant__ TensorMaps4 in_maps, const __grid_constant__ TensorMaps4 out_maps,
    const float* __restrict__ k, const float* __restrict__ v, const float* __restrict__ r,
    const float* __restrict__ dy, float* dk, float* dv, float* dr, int B, int T, int C,
    const float* __restrict__ w, const float* __restrict__ u, void* ws, unsigned* err) {
  constexpr int kTile = kTT * 32;
  extern __shared__ __align__(128) float smem[];
  // stage s2 holds tiles k, v, r (or dy), dy at smem + (4 s2 + slot) kTile
  float* fe1 = smem + 8 * kTile;
  float* fe2 = fe1 + kTile;
  float* finj = fe2 + kTile;
  float* fcur = finj + kTile;
  float* fwkv = fcur + kTile;
  float* fsig = fwkv + kTile;
  uint64_t* bars = reinterpret_cast<uint64_t*>(fsig + kTile);

  const int lane = threadIdx.x;
  const int G = (C + 31) >> 5;
  const int b = blockIdx.x / G, g = blockIdx.x % G;
  const int c = (g << 5) + lane;
  const bool valid = c < C;
  const int nch = (T + kTT - 1) / kTT;
  const BwdLayout lay = bwd_layout(ws, B, T, C);
  // Tensors loaded per chunk: k, v, dy, and r when gated (r sits in slot 2, dy in slot 3).
  const Ptr4 ptrs{k, v, GATE ? r : dy, dy};
  const int nload = GATE ? 4 : 3;
  const MPtr3 outp{dk, dv, dr};
  const int nstore = DR ? 3 : 2;

  auto issue = [&](int s2, int ch) {
    Tiles<TMA>::load(in_maps.m, ptrs, nload, smem + 4 * s2 * kTile, &bars[s2], b, g, ch * kTT,
                     T, C, lane);
  };
  if (lane == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    mbar_fence_init();
  }
  __syncwarp();

  const ChanParams cp = chan_params(valid ? w[c] : 1.f, valid ? u[c] : 0.f);
  const bool fast = __all_sync(0xffffffffu, fabsf(cp.uw2) <= kFastOutBound);
  const int rb = window_tokens(cp.w2, 128.f);

  float beta = 0.f, gamma = 0.f, betad = 0.f, gammad = 0.f;  // scaled suffix sums
  float dw_acc = 0.f, du_acc = 0.f;

  issue(0, nch - 1);
  if (nch > 1) issue(1, nch - 2);
  for (int it = 0; it < nch; ++it) {
    const int ch = nch - 1 - it;
    const int s2 = it & 1;
    Tiles<TMA>::wait(&bars[s2], (it >> 1) & 1, err);
    float* K = smem + (4 * s2 + 0) * kTile;
    float* V = smem + (4 * s2 + 1) * kTile;
    float* R = smem + (4 * s2 + 2) * kTile;
    float* DY = smem + (4 * s2 + (GATE ? 3 : 2)) * kTile;
    const int n = min(kTT, T - ch * kTT);

    // Forward recomputation of the chunk from its checkpoint: per-token factors.
    float4 ck = valid ? lay.ckpt[(int64_t(b) * nch + ch) * C + c]
                      : make_float4(0.f, 0.f, kEmptyLogScale, 0.f);
    ChanState s;
    s.a = ck.x;
    s.b = ck.y;
    s.Q = ck.z;
    s.pl = ck.w;
    int j = 0;
    for (int t = 0; t < n; ++t) {
      const int o = t * 32 + lane;
      const float kk = K[o], vv = V[o];
      const float m = fmaf(float(j + 1), cp.w2, fmaf(kk, kLog2e, -s.pl));
      const float d = m - s.Q;
      const float e = ex2(-fabsf(d));
      const bool cnd = d > 0.f;
      const float e1 = cnd ? e : 1.f;
      const float e2 = cnd ? 1.f : e;
      s.Q = fmaxf(s.Q, m);
      float num, den, ki, kc;
      if (fast) {
        const float he = cp.H * e2;
        num = fmaf(e1, s.a, he * vv);
        den = fmaf(e1, s.b, he);
        ki = e1;
        kc = he;
      } else {
        const float dO = d + cp.uw2;
        const float oo = ex2(-fabsf(dO));
        const bool co = dO > 0.f;
        const float o1 = co ? oo : 1.f;
        const float o2 = co ? 1.f : oo;
        num = fmaf(o1, s.a, o2 * vv);
        den = fmaf(o1, s.b, o2);
        ki = o1;
        kc = o2;
      }
      const float rden = rcp(den);
      float sig = 1.f;
      if (GATE) sig = rcp(1.f + ex2(R[o] * -kLog2e));
      const float rc = sig * rden;  // sigmoid(r) / den
      fe1[o] = e1;
      fe2[o] = e2;
      finj[o] = rc * ki;
      fcur[o] = rc * kc;
      fwkv[o] = num * rden;
      if (DR) fsig[o] = sig;
      s.a = fmaf(e1, s.a, e2 * vv);
      s.b = fmaf(e1, s.b, e2);
      if (++j == rb) {
        wkv_rebase(s, float(rb) * cp.w2);
        j = 0;
      }
    }
    // Reverse over the chunk; dk, dv (dr) replace k, v (r) in shared memory.
    for (int t = n - 1; t >= 0; --t) {
      const int o = t * 32 + lane;
      const float gy = DY[o], vv = V[o];
      const float e1 = fe1[o], e2 = fe2[o], wk = fwkv[o];
      const float inj = gy * finj[o];
      const float cur = gy * fcur[o];
      const float vm = vv - wk;
      V[o] = fmaf(e2, beta, cur);                               // dv
      K[o] = fmaf(cur, vm, e2 * fmaf(vv, beta, -gamma));        // dk
      dw_acc = fmaf(e2, fmaf(vv, betad, -gammad), dw_acc);
      du_acc = fmaf(cur, vm, du_acc);
      if (DR) {
        const float sg = fsig[o];
        R[o] = gy * wk * sg * (1.f - sg);
      }
      betad = e1 * (betad + beta);
      gammad = e1 * (gammad + gamma);
      beta = fmaf(e1, beta, inj);
      gamma = fmaf(e1, gamma, inj * wk);
    }
    Tiles<TMA>::store(out_maps.m, outp, nstore, K, b, g, ch * kTT, T, C, lane);
    if (it + 2 < nch) {
      // The stores read this stage's tiles: drain them before the refill overwrites.
      Tiles<TMA>::store_drain(lane);
      issue(s2, ch - 2);
    }
  }
  Tiles<TMA>::store_drain(lane);
  if (valid) {
    lay.pdw[int64_t(b) * C + c] = -dw_acc;
    lay.pdu[int64_t(b) * C + c] = du_acc;
  }
}

// ---- 3. reduction over the batch, fixed order ----------------------------------------------
__global__ void wkv_bwd_reduce_kernel(int B, int C, const void* ws, int T, float* dw, float* du) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= C) return;
  const BwdLayout lay = bwd_layout(const_cast<void*>(ws), B, T, C);
  float sw = 0.f, su = 0.f;
  for (int b = 0; b < B; ++b) {
    sw += lay.pdw[int64_t(b) * C + c];
    su += lay.pdu[int64_t(b) * C + c];
  }
  dw[c] = sw;
  du[c] = su;
}

size_t bwd_main_smem() { return (8 + 6) * kTT * 32 * sizeof(float) + 2 * sizeof(uint64_t); }

template <bool TMA, bool GATE, bool DR>
int launch_main(const BwdArgs& a, const TensorMaps4& in, const TensorMaps4& out,
                cudaStream_t stream) {
  auto kern = wkv_bwd_main_kernel<TMA, GATE, DR>;
  const size_t smem = bwd_main_smem();
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
      cudaSuccess)
    return WKV_ERR_CUDA;
  const int64_t grid = a.B * ((a.C + 31) / 32);
  kern<<<unsigned(grid), 32, smem, stream>>>(in, out, a.k, a.v, a.r, a.dy, a.dk, a.dv, a.dr,
                                             int(a.B), int(a.T), int(a.C), a.w, a.u, a.ws, a.err);
  return cudaPeekAtLastError() == cudaSuccess ? WKV_OK : WKV_ERR_CUDA;
}

template <bool TMA>
int launch_all(const BwdArgs& a, cudaStream_t stream) {
  TensorMaps4 ck{}, in{}, out{};
  const int64_t grid = a.B * ((a.C + 31) / 32);
  if (TMA) {
    const auto dt = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    const void* ins[4] = {a.k, a.v, a.r ? a.r : a.dy, a.dy};
    void* outs[3] = {a.dk, a.dv, a.dr ? a.dr : a.dk};
    for (int i = 0; i < 4; ++i)
      if (int rc = encode_btc_map(&in.m[i], ins[i], dt, 4, a.B, a.T, a.C, 32, kTT)) return rc;
    for (int i = 0; i < 3; ++i)
      if (int rc = encode_btc_map(&out.m[i], outs[i], dt, 4, a.B, a.T, a.C, 32, kTT)) return rc;
    ck.m[0] = in.m[0];
    ck.m[1] = in.m[1];
  }
  wkv_bwd_ckpt_kernel<TMA><<<unsigned(grid), 32, 0, stream>>>(ck, a.k, a.v, int(a.B), int(a.T),
                                                              int(a.C), a.w, a.ws, a.err);
  if (cudaPeekAtLastError() != cudaSuccess) return WKV_ERR_CUDA;
  int rc;
  if (a.r)
    rc = a.dr ? launch_main<TMA, true, true>(a, in, out, stream)
              : launch_main<TMA, true, false>(a, in, out, stream);
  else
    rc = launch_main<TMA, false, false>(a, in, out, stream);
  if (rc) return rc;
  wkv_bwd_reduce_kernel<<<unsigned((a.C + 127) / 128), 128, 0, stream>>>(int(a.B), int(a.C), a.ws,
                                                                        int(a.T), a.dw, a.du);
  return cudaPeekAtLastError() == cudaSuccess ? WKV_OK : WKV_ERR_CUDA;
}

}  // namespace

size_t backward_workspace_bytes(int64_t B, int64_t T, int64_t C) { return bwd_bytes(B, T, C); }

int launch_backward(const BwdArgs& a, bool force_plain, cudaStream_t stream) {
  auto al16 = [](const void* p) {
    return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15) == 0;
  };
  const bool tma = !force_plain && a.C % 4 == 0 && al16(a.k) && al16(a.v) && al16(a.r) &&
                   al16(a.dy) && al16(a.dk) && al16(a.dv) && al16(a.dr);
  return tma ? launch_all<true>(a, stream) : launch_all<false>(a, stream);
}

}  // namespace wkv
