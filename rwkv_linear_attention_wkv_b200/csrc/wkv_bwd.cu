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
// Two passes plus a reduction:
//   1. checkpoints: the state entering every chunk of kTT tokens. On TMA shapes either
//      time-parallel (wkv_bwd_ckpt_seg_kernel: chunk aggregates folded across segments, in
//      the state-independent token weights of wkv_indep.cuh) or, when the channel groups
//      (batch row x 32 channels) number at least twice the SMs, one persistent CTA per
//      group walking its segments in order (wkv_bwd_ckpt_group_kernel); serially on other
//      shapes (wkv_bwd_ckpt_kernel: one warp per 32 channels walks the sequence in the
//      streaming forward's arithmetic). In the checkpointed training pair the forward has
//      written them already (the streaming kernel's checkpointing mode) and this pass is
//      skipped;
//   2. reverse (TMA shapes): one warp per chunk recomputes the chunk's forward from its
//      checkpoint (in the arithmetic that made the checkpoint: the template flag FWD) and
//      then runs the reverse over its chunk. The carry at each segment's end (kSW chunks)
//      is either chained across CTAs through published maps (wkv_bwd_seg_kernel,
//      time-parallel) or, with as many groups as above, kept on chip by one persistent CTA
//      per group walking its segments from the last (wkv_bwd_group_kernel). Shapes TMA
//      cannot address take the serial form: one warp per 32 channels walks the chunks from
//      last to first, recomputing each chunk's factors into shared memory before its
//      reverse;
//   both write dk, dv (dr) in place of k, v (r) in shared memory for the stores, and
//   partial sums of dw, du to the workspace;
//   3. reduce: dw[c], du[c] = sums of the partials over b and t in a fixed order
//      (deterministic): a kernel of its own (wkv_bwd_reduce_kernel), or, on the per-group
//      path, the last reverse-pass CTA of each channel group.
#include <algorithm>
#include <atomic>

#include "wkv_internal.h"
#include "wkv_async.cuh"
#include "wkv_indep.cuh"
#include "wkv_step.cuh"

namespace wkv {

namespace {

constexpr int kTT = 16;   // tokens per chunk (checkpoint interval; one warp's unit of work)
constexpr int kSW = 4;    // chunks (warps) per segment of the time-parallel passes
// Segments whose results a segment folds in directly before taking a carry from further
// away (which makes one link of a serial chain per kFoldF / kFoldR + 1 segments): in the
// checkpoint pass (forward) and the reverse pass.
constexpr int kFoldF = 8;
constexpr int kFoldR = 5;

struct BwdLayout {
  float4* ckpt;      // [B, nch, C] forward state entering each chunk: (a, b, Q, pl)
  float4* ckend;     // [B, C] forward state after the last token
  float* pdw;        // [B, nseg, C] per-segment partial sums of dw
  float* pdu;        // [B, nseg, C] per-segment partial sums of du
  unsigned* fticket;  // segment tickets of the checkpoint pass (forward chain)
  unsigned* rticket;  // segment tickets of the reverse pass (reverse chain)
  unsigned* fflags;   // [nbg * nseg']: 1 once the checkpoint segment's aggregate is published,
                      // 2 once the state entering it (its first checkpoint) is written
                      // (nseg' <= nseg checkpoint segments of kSW kCK chunks); on the
                      // per-group path its first G words count the batch rows done per
                      // channel group instead
  unsigned* rflags;   // [nbg * nseg]: 1 once the segment's reverse map is published, 2 its carry
  float4* fagg;      // [nbg * nseg', 32]: the checkpoint segment's aggregate (a, b, ph, pl)
  float4* rmap;      // [nbg * nseg, 32, 2]: the segment's reverse map (see RevAgg)
  float4* carry;     // [nbg * nseg, 32]: (beta, gamma, betad, gammad) at the segment start
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

__host__ __device__ inline int64_t bwd_nseg(int64_t T) {
  const int64_t nch = (T + kTT - 1) / kTT;
  return (nch + kSW - 1) / kSW;
}

// Bytes of the chain flags (with the tickets) that must be zero at the start of a call.
__host__ __device__ inline size_t bwd_flag_bytes(int64_t B, int64_t T, int64_t C) {
  const int64_t nitems = B * ((C + 31) / 32) * bwd_nseg(T);
  return align256(size_t(16 + 8 * nitems));
}

__host__ __device__ inline BwdLayout bwd_layout(void* ws, int64_t B, int64_t T, int64_t C) {
  const int64_t nch = (T + kTT - 1) / kTT;
  const int64_t nitems = B * ((C + 31) / 32) * bwd_nseg(T);
  char* p = static_cast<char*>(ws);
  BwdLayout L;
  L.fticket = reinterpret_cast<unsigned*>(p);
  L.rticket = reinterpret_cast<unsigned*>(p + 4);
  L.fflags = reinterpret_cast<unsigned*>(p + 16);
  L.rflags = L.fflags + nitems;
  p += bwd_flag_bytes(B, T, C);
  L.ckpt = reinterpret_cast<float4*>(p);
  p += align256(size_t(B) * nch * C * sizeof(float4));
  L.ckend = reinterpret_cast<float4*>(p);
  p += align256(size_t(B) * C * sizeof(float4));
  L.pdw = reinterpret_cast<float*>(p);
  p += align256(size_t(B) * bwd_nseg(T) * C * sizeof(float));
  L.pdu = reinterpret_cast<float*>(p);
  p += align256(size_t(B) * bwd_nseg(T) * C * sizeof(float));
  L.fagg = reinterpret_cast<float4*>(p);
  p += align256(size_t(nitems) * 32 * sizeof(float4));
  L.rmap = reinterpret_cast<float4*>(p);
  p += align256(size_t(nitems) * 32 * 2 * sizeof(float4));
  L.carry = reinterpret_cast<float4*>(p);
  return L;
}

__host__ __device__ inline size_t bwd_bytes(int64_t B, int64_t T, int64_t C) {
  const int64_t nch = (T + kTT - 1) / kTT;
  const int64_t nitems = B * ((C + 31) / 32) * bwd_nseg(T);
  return bwd_flag_bytes(B, T, C) + align256(size_t(B) * nch * C * sizeof(float4)) +
         align256(size_t(B) * C * sizeof(float4)) +
         2 * align256(size_t(B) * bwd_nseg(T) * C * sizeof(float)) +
         align256(size_t(nitems) * 32 * sizeof(float4)) +
         align256(size_t(nitems) * 32 * 2 * sizeof(float4)) +
         align256(size_t(nitems) * 32 * sizeof(float4));
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
  // Only until the stores have read their shared-memory sources (enough to refill them).
  static __device__ __forceinline__ void store_read_drain(int lane) {
    if (TMA && lane == 0) tma_store_wait_read<0>();
    __syncwarp();
  }
};

struct TensorMaps4 {
  CUtensorMap m[4];
};

// Backward through a state (see BwdArgs): all NULL for the plain backward.
struct StateIO {
  const float* a0;
  const float* b0;
  const float* p0;
  const float* ga1;
  const float* gb1;
  const float* p1;
  float* da0;
  float* db0;
  float* dp0;
};

// The state entering the sequence: the given initial state, or the empty one.
__device__ __forceinline__ ChanState initial_state(const StateIO& io, int64_t sidx, bool valid) {
  return (io.a0 != nullptr && valid) ? load_state(io.a0[sidx], io.b0[sidx], io.p0[sidx])
                                     : empty_state();
}

// The scaled reverse carry at the end of the sequence, from the gradients (ga1, gb1) of a
// later loss with respect to the final state's a1, b1 (log-scale p1): beta = dL/dA_T =
// ga1 e^{-p1}, gamma = -dL/dB_T = -gb1 e^{-p1}, both scaled by 2^P for the log2-scale P
// = (Ph, Pl) of the state after the last token as this pass represents it.
__device__ __forceinline__ float2 end_carry(const StateIO& io, int64_t sidx, bool valid,
                                            float Ph, float Pl) {
  if (io.ga1 == nullptr || !valid) return make_float2(0.f, 0.f);
  const float p1 = io.p1[sidx];
  const float qh = p1 * kLog2e;
  const float ql = fmaf(p1, kLog2e, -qh);  // exact low part of the product
  const float f = ex2(fminf((Ph - qh) + (Pl - ql), 126.f));
  return make_float2(io.ga1[sidx] * f, -io.gb1[sidx] * f);
}

// ---- 1. checkpoints --------------------------------------------------------------------
template <bool TMA>
__global__ void __launch_bounds__(32, 8) wkv_bwd_ckpt_kernel(const __grid_constant__ TensorMaps4 maps,
                                                          const float* __restrict__ k,
                                                          const float* __restrict__ v,
                                                          int B, int T, int C,
                                                          const float* __restrict__ w,
                                                          const StateIO io, void* ws,
                                                          unsigned* err) {
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
  ChanState s = initial_state(io, int64_t(b) * C + c, valid);
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
  if (valid) lay.ckend[int64_t(b) * C + c] = make_float4(s.a, s.b, s.Q, s.pl);
}

// Token weights and the scale step of the time-parallel checkpoints and of the
// recomputation that starts from them: wkv_indep.cuh.
__device__ __forceinline__ void absorb_indep(ChanState& s, const ChanParams& cp, float fj, float k,
                                             float v) {
  const ScaleStep st = indep_step(tok_log2w(fj, cp.w2, k), s.Q, s.pl);
  s.a = fmaf(st.e1, s.a, st.e2 * v);
  s.b = fmaf(st.e1, s.b, st.e2);
}

// Time-parallel form (TMA shapes). One CTA per (checkpoint segment of kSW x kCK chunks,
// batch row, 32-channel group), warp i on chunks kCK i .. kCK i + kCK - 1 of the segment;
// CTAs take segments in ticket order from the first on, so every segment a CTA waits for
// belongs to a CTA that started earlier. Each warp folds its chunks' k, v into each chunk's
// aggregate from the empty state. Warp 0 publishes the segment's aggregate; the last warp
// forms the state entering the segment in a fixed order (bitwise reproducible): the state
// entering segment j0 = max(0, seg - kFoldF) (its first checkpoint), then the published
// aggregates of segments j0 .. seg-1, so one link of a serial chain spans kFoldF segments.
// After a barrier each warp combines that state with the aggregates of the chunks before
// its own and writes its chunks' checkpoints. One pass, 8 bytes of HBM reads per element.
constexpr int kCK = 2;  // chunks per warp in the checkpoint pass

// Aggregate of one chunk of n tokens from the empty state (windows of RB tokens).
template <int RB>
__device__ __forceinline__ Agg chunk_aggregate(const float* K, const float* V, int n,
                                               const ChanParams& cp) {
  ChanState s = empty_state();
  if (n == kTT) {
    // absorb_indep token by token, with the log-weights and the products e2 v two tokens
    // to an fp32x2 instruction (each lane rounded as the scalar form)
#pragma unroll
    for (int t = 0; t < kTT; t += 2) {
      const float2 kk = make_float2(K[t * 32], K[(t + 1) * 32]);
      const float2 vv = make_float2(V[t * 32], V[(t + 1) * 32]);
      const float2 m =
          tok_log2w2(make_float2(float(t % RB + 1), float((t + 1) % RB + 1)), cp.w2, kk);
      float e1s[2], e2s[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const ScaleStep st = indep_step(h ? m.y : m.x, s.Q, s.pl);
        e1s[h] = st.e1;
        e2s[h] = st.e2;
        if ((t + h + 1) % RB == 0) wkv_rebase(s, float(RB) * cp.w2);
      }
      const float2 ev = __fmul2_rn(make_float2(e2s[0], e2s[1]), vv);
      s.a = fmaf(e1s[0], s.a, ev.x);
      s.b = fmaf(e1s[0], s.b, e2s[0]);
      s.a = fmaf(e1s[1], s.a, ev.y);
      s.b = fmaf(e1s[1], s.b, e2s[1]);
    }
  } else {
    int j = 0;
    for (int t = 0; t < n; ++t) {
      absorb_indep(s, cp, float(j + 1), K[t * 32], V[t * 32]);
      if (++j == RB) {
        wkv_rebase(s, float(RB) * cp.w2);
        j = 0;
      }
    }
    if (j) wkv_rebase_partial(s, j, cp.w2);
  }
  return to_agg(s);
}

__global__ void __launch_bounds__(kSW * 32, 6) wkv_bwd_ckpt_seg_kernel(
    const __grid_constant__ TensorMaps4 maps, int B, int T, int C, const float* __restrict__ w,
    const StateIO io, void* ws, unsigned* err, unsigned long long wait_ns) {
  constexpr int kTile = kTT * 32;
  constexpr int kSegC = kSW * kCK;  // chunks per checkpoint segment
  __shared__ __align__(128) float tiles[kSW][kCK][2][kTile];  // k, v of each warp's chunks
  __shared__ float4 sagg[kSegC][32];
  __shared__ float4 sfold[kFoldF][32];  // earlier segments' aggregates
  __shared__ float4 sin_[32];           // the state entering the segment
  __shared__ uint64_t bars[kSW];
  __shared__ unsigned s_ticket[3];

  const int G = (C + 31) >> 5;
  const int64_t nbg = int64_t(B) * G;
  const int nch = (T + kTT - 1) / kTT;
  const int nseg = (nch + kSegC - 1) / kSegC;
  const BwdLayout lay = bwd_layout(ws, B, T, C);
  if (threadIdx.x == 0) {  // ticket -> (segment, batch row, channel group), decoded once
    const unsigned ticket = atomicAdd(lay.fticket, 1u);  // < 2^31 (host check)
    const unsigned sg = ticket / unsigned(nbg);
    const unsigned r = ticket - sg * unsigned(nbg);
    const unsigned bb = r / unsigned(G);
    s_ticket[0] = sg;
    s_ticket[1] = bb;
    s_ticket[2] = r - bb * unsigned(G);
  }
  __syncthreads();
  const int seg = int(s_ticket[0]);
  const int b = int(s_ticket[1]);
  const int g = int(s_ticket[2]);
  const int64_t bg = int64_t(b) * G + g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = (g << 5) + lane;
  const bool valid = c < C;
  const int ch0 = seg * kSegC + warp * kCK;  // this warp's first chunk
  const int64_t item0 = bg * nseg;
  const int64_t item = item0 + seg;
  float4* ck = lay.ckpt + int64_t(b) * nch * C + c;  // checkpoint of chunk i at ck[i * C]

  uint64_t* bar = &bars[warp];
  if (lane == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
    const int nc = max(0, min(kCK, nch - ch0));  // chunks of this warp
    if (nc > 0) {
      mbar_arrive_expect_tx(bar, uint32_t(nc) * 2u * kTile * sizeof(float));
      for (int q = 0; q < nc; ++q) {
        tma_load_3d(&tiles[warp][q][0][0], &maps.m[0], bar, g << 5, (ch0 + q) * kTT, b);
        tma_load_3d(&tiles[warp][q][1][0], &maps.m[1], bar, g << 5, (ch0 + q) * kTT, b);
      }
    }
  }
  __syncwarp();
  const ChanParams cp = chan_params(valid ? w[c] : 1.f, 0.f);
  const int rb = window_tokens(cp.w2, 128.f);

  // The fold's inputs (below) are usually published before this segment starts: the last
  // warp checks their flags now (one acquire load per lane, while the tiles load) and, if
  // all are set, copies them into shared memory (cp.async) while the aggregates are
  // formed; otherwise it waits for them after that.
  const int j0 = max(0, seg - kFoldF);
  const int mfold = seg - j0;  // aggregates to fold
  const unsigned fwant = lane < mfold ? 1u : ((lane == 31 && j0 > 0) ? 2u : 0u);
  bool fold_early = false;
  if (warp == kSW - 1) {
    const unsigned* flag = lane < mfold ? &lay.fflags[item0 + j0 + lane] : &lay.fflags[item0 + j0];
    const unsigned fl = fwant != 0 ? ld_acquire(flag) : 0u;
    fold_early = __all_sync(0xffffffffu, fl >= fwant);
    __syncwarp();  // orders every lane's acquire before every lane's copies below
    if (fold_early) {
      for (int l = 0; l < mfold; ++l) cp_async_16(&sfold[l][lane], &lay.fagg[(item0 + j0 + l) * 32 + lane]);
      if (j0 > 0 && valid) cp_async_16(&sin_[lane], &ck[int64_t(j0) * kSegC * C]);
      cp_async_commit();
    }
  }

  // ---- the chunks' aggregates from the empty state ----
  if (ch0 < nch) mbar_wait_suspend(bar, 0, err);
  __syncwarp();
#pragma unroll
  for (int q = 0; q < kCK; ++q) {
    const int n = max(0, min(kTT, T - (ch0 + q) * kTT));  // tokens of the chunk
    Agg A = agg_empty();
    if (n > 0) {
      const float* K = &tiles[warp][q][0][lane];
      const float* V = &tiles[warp][q][1][lane];
      A = rb == 16 ? chunk_aggregate<16>(K, V, n, cp)
                   : (rb == 4 ? chunk_aggregate<4>(K, V, n, cp) : chunk_aggregate<1>(K, V, n, cp));
    }
    sagg[warp * kCK + q][lane] = make_float4(A.a, A.b, A.ph, A.pl);
  }
  __syncthreads();

  // ---- the segment's aggregate, for the segments after it ----
  const bool first = seg > 0 && seg + kFoldF < nseg;  // segment seg + kFoldF starts here
  if (warp == 0 && seg + 1 < nseg) {
    Agg S = agg_empty();
#pragma unroll
    for (int i = 0; i < kSegC; ++i) {
      const float4 q = sagg[i][lane];
      S = combine(S, Agg{q.x, q.y, q.z, q.w}, float(kTT), cp.w2);  // all chunks full
    }
    lay.fagg[item * 32 + lane] = make_float4(S.a, S.b, S.ph, S.pl);
    warp_publish(&lay.fflags[item], 1u);
  }
  // ---- the state entering the segment (last warp; the aggregate above does not wait) ----
  if (warp == kSW - 1) {
    const int m = mfold;
    bool ok = true;
    if (fold_early) {
      cp_async_wait_all();
    } else {  // wait for the flags not yet set, then fetch (L2 loads: L1 may be stale)
      const unsigned* flag = lane < m ? &lay.fflags[item0 + j0 + lane] : &lay.fflags[item0 + j0];
      const unsigned fl = fwant != 0 ? wait_flag(flag, fwant, wait_ns, err) : 1u;
      ok = __all_sync(0xffffffffu, fl != 0);
      __syncwarp();  // orders every lane's acquire before every lane's fetch below
      if (ok) {  // (a wait that gave up flagged the error word: continue from the empty state)
        for (int l = 0; l < m; ++l) sfold[l][lane] = __ldcg(&lay.fagg[(item0 + j0 + l) * 32 + lane]);
        if (j0 > 0 && valid) sin_[lane] = __ldcg(&ck[int64_t(j0) * kSegC * C]);
      }
    }
    __syncwarp();
    Agg X = to_agg(initial_state(io, int64_t(b) * C + c, valid));
    if (j0 > 0) {
      const float4 q = sin_[lane];
      X = (ok && valid) ? Agg{q.x, q.y, q.z, q.w} : agg_empty();
    }
    if (ok)
      for (int l = 0; l < m; ++l) {
        const float4 a = sfold[l][lane];
        X = combine(X, Agg{a.x, a.y, a.z, a.w}, float(kSegC * kTT), cp.w2);
      }
    __syncwarp();
    sin_[lane] = make_float4(X.a, X.b, X.ph, X.pl);
  }
  __syncthreads();

  // ---- checkpoints ----
  {
    const float4 q = sin_[lane];
    Agg X{q.x, q.y, q.z, q.w};
    for (int i = 0; i < warp * kCK; ++i) {  // chunks before this warp's (full)
      const float4 a = sagg[i][lane];
      X = combine(X, Agg{a.x, a.y, a.z, a.w}, float(kTT), cp.w2);
    }
#pragma unroll
    for (int q2 = 0; q2 < kCK; ++q2) {
      const int chq = ch0 + q2;
      if (chq < nch) {
        if (valid) ck[int64_t(chq) * C] = make_float4(X.a, X.b, X.ph, X.pl);
        if (q2 + 1 < kCK || chq + 1 == nch) {
          const float4 a = sagg[warp * kCK + q2][lane];
          X = combine(X, Agg{a.x, a.y, a.z, a.w}, float(min(kTT, T - chq * kTT)), cp.w2);
          // after the last chunk: the state after the last token
          if (chq + 1 == nch && valid) lay.ckend[int64_t(b) * C + c] = make_float4(X.a, X.b, X.ph, X.pl);
        }
      }
    }
  }
  if (warp == 0 && first) warp_publish(&lay.fflags[item], 2u);  // the first checkpoint is written
}

// ---- 1'. checkpoints, one persistent CTA per channel group --------------------------------
// The counterpart of wkv_bwd_group_kernel for the checkpoint pass: one CTA per channel
// group walks the group's checkpoint segments (kSW warps x kCK chunks) in order; the warps
// form their chunks' aggregates from the empty state in parallel, then write the
// checkpoints from the state entering the segment, which comes from the previous iteration
// in shared memory (the initial state for the first). No tickets, flags or waits on other
// CTAs.
__global__ void __launch_bounds__(kSW * 32, 4) wkv_bwd_ckpt_group_kernel(
    const __grid_constant__ TensorMaps4 maps, int B, int T, int C, const float* __restrict__ w,
    const StateIO io, void* ws, unsigned* err, const Ptr4 pre) {
  constexpr int kTile = kTT * 32;
  constexpr int kSegC = kSW * kCK;  // chunks per checkpoint segment
  __shared__ __align__(128) float tiles[kSW][kCK][2][kTile];  // k, v of each warp's chunks
  __shared__ float4 sagg[kSegC][32];
  __shared__ float4 sin_[2][32];  // the state entering the segment (double-buffered)
  __shared__ uint64_t bars[kSW];

  const int G = (C + 31) >> 5;
  const int nch = (T + kTT - 1) / kTT;
  const int nseg = (nch + kSegC - 1) / kSegC;
  const BwdLayout lay = bwd_layout(ws, B, T, C);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = int(blockIdx.x) / G, g = int(blockIdx.x) % G;
  const int c = (g << 5) + lane;
  const bool valid = c < C;
  float4* ck = lay.ckpt + int64_t(b) * nch * C + c;  // checkpoint of chunk i at ck[i * C]
  const ChanParams cp = chan_params(valid ? w[c] : 1.f, 0.f);
  const int rb = window_tokens(cp.w2, 128.f);
  uint64_t* bar = &bars[warp];
  if (lane == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
  }
  if (warp == 0) {
    const Agg X = to_agg(initial_state(io, int64_t(b) * C + c, valid));
    sin_[0][lane] = make_float4(X.a, X.b, X.ph, X.pl);
  }
  // the reverse pass that follows counts the batch rows done per channel group from zero
  if (b == 0 && threadIdx.x == 0) lay.fflags[g] = 0u;
  __syncthreads();

  uint32_t phase = 0;
  for (int seg = 0; seg < nseg; ++seg) {
    const int ch0 = seg * kSegC + warp * kCK;  // this warp's first chunk
    const int nc = max(0, min(kCK, nch - ch0));
    if (lane == 0 && nc > 0) {
      fence_proxy_async_smem();  // the previous segment's reads of these tiles come first
      mbar_arrive_expect_tx(bar, uint32_t(nc) * 2u * kTile * sizeof(float));
      for (int q = 0; q < nc; ++q) {
        tma_load_3d(&tiles[warp][q][0][0], &maps.m[0], bar, g << 5, (ch0 + q) * kTT, b);
        tma_load_3d(&tiles[warp][q][1][0], &maps.m[1], bar, g << 5, (ch0 + q) * kTT, b);
      }
    }
    // the next segment's rows of this warp's chunks into L2 meanwhile
    if (seg + 1 < nseg) {
      const int tn = (seg + 1) * kSegC * kTT + warp * kCK * kTT + lane;
      if (tn < T) {
        const int64_t off = (int64_t(b) * T + tn) * C + (int64_t(g) << 5);
        prefetch_l2(pre[0] + off);
        prefetch_l2(pre[1] + off);
      }
    }
    __syncwarp();
    if (nc > 0) {
      mbar_wait_suspend(bar, phase, err);
      phase ^= 1u;
    }
    __syncwarp();
#pragma unroll
    for (int q = 0; q < kCK; ++q) {
      const int n = max(0, min(kTT, T - (ch0 + q) * kTT));  // tokens of the chunk
      Agg A = agg_empty();
      if (n > 0) {
        const float* K = &tiles[warp][q][0][lane];
        const float* V = &tiles[warp][q][1][lane];
        A = rb == 16 ? chunk_aggregate<16>(K, V, n, cp)
                     : (rb == 4 ? chunk_aggregate<4>(K, V, n, cp) : chunk_aggregate<1>(K, V, n, cp));
      }
      sagg[warp * kCK + q][lane] = make_float4(A.a, A.b, A.ph, A.pl);
    }
    __syncthreads();

    // ---- checkpoints; the last warp hands the state after the segment on ----
    const float4 q = sin_[seg & 1][lane];
    Agg X{q.x, q.y, q.z, q.w};
    for (int i = 0; i < warp * kCK; ++i) {  // chunks before this warp's (full)
      const float4 a = sagg[i][lane];
      X = combine(X, Agg{a.x, a.y, a.z, a.w}, float(kTT), cp.w2);
    }
#pragma unroll
    for (int q2 = 0; q2 < kCK; ++q2) {
      const int chq = ch0 + q2;
      if (chq < nch) {
        if (valid) ck[int64_t(chq) * C] = make_float4(X.a, X.b, X.ph, X.pl);
        const float4 a = sagg[warp * kCK + q2][lane];
        X = combine(X, Agg{a.x, a.y, a.z, a.w}, float(min(kTT, T - chq * kTT)), cp.w2);
        // after the last chunk: the state after the last token
        if (chq + 1 == nch && valid) lay.ckend[int64_t(b) * C + c] = make_float4(X.a, X.b, X.ph, X.pl);
      }
    }
    if (warp == kSW - 1) sin_[(seg + 1) & 1][lane] = make_float4(X.a, X.b, X.ph, X.pl);
    __syncthreads();
  }
}

// ---- 2. reverse pass ---------------------------------------------------------------------
// Shared memory per CTA (floats): kMS stages x 4 tiles (k, v, r, dy; dk, dv, dr written in
// place of k, v, r) + 6 factor tiles (e1, e2, f_inj, f_cur, wkv, sigma).
constexpr int kMS = 3;
// Launch bounds with a minimum of 3 resident CTAs (all that shared memory allows): without
// one, ptxas budgets registers for 32 CTAs per SM (64 per thread).
template <bool TMA, bool GATE, bool DR>
__global__ void __launch_bounds__(32, 3) wkv_bwd_main_kernel(
    const __grid_constant__ TensorMaps4 in_maps, const __grid_constant__ TensorMaps4 out_maps,
    const float* __restrict__ k, const float* __restrict__ v, const float* __restrict__ r,
    const float* __restrict__ dy, float* dk, float* dv, float* dr, int B, int T, int C,
    const float* __restrict__ w, const float* __restrict__ u, const StateIO io, void* ws,
    unsigned* err) {
  constexpr int kTile = kTT * 32;
  extern __shared__ __align__(128) float smem[];
  // stage s2 holds tiles k, v, r (or dy), dy at smem + (4 s2 + slot) kTile
  float* fe1 = smem + 4 * kMS * kTile;
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
    for (int st = 0; st < kMS; ++st) mbar_init(&bars[st], 1);
    mbar_fence_init();
  }
  __syncwarp();

  const ChanParams cp = chan_params(valid ? w[c] : 1.f, valid ? u[c] : 0.f);
  const bool fast = __all_sync(0xffffffffu, fabsf(cp.uw2) <= kFastOutBound);
  const int rb = window_tokens(cp.w2, 128.f);

  float beta = 0.f, gamma = 0.f, betad = 0.f, gammad = 0.f;  // scaled suffix sums
  float dw_acc = 0.f, du_acc = 0.f;

  for (int st = 0; st < kMS && st < nch; ++st) issue(st, nch - 1 - st);
  auto ckpt_of = [&](int ch) {
    return valid ? lay.ckpt[(int64_t(b) * nch + ch) * C + c]
                 : make_float4(0.f, 0.f, kEmptyLogScale, 0.f);
  };
  float4 ck_next = ckpt_of(nch - 1);  // checkpoints are read one chunk ahead
  for (int it = 0; it < nch; ++it) {
    const int ch = nch - 1 - it;
    const int s2 = it % kMS;
    const float4 ck = ck_next;
    if (ch > 0) ck_next = ckpt_of(ch - 1);
    Tiles<TMA>::wait(&bars[s2], (it / kMS) & 1, err);
    float* K = smem + (4 * s2 + 0) * kTile;
    float* V = smem + (4 * s2 + 1) * kTile;
    float* R = smem + (4 * s2 + 2) * kTile;
    float* DY = smem + (4 * s2 + (GATE ? 3 : 2)) * kTile;
    const int n = min(kTT, T - ch * kTT);

    // Forward recomputation of the chunk from its checkpoint: per-token factors.
    ChanState s;
    s.a = ck.x;
    s.b = ck.y;
    s.Q = ck.z;
    s.pl = ck.w;
    int j = 0;
#pragma unroll 8
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
    if (it == 0) {  // the last chunk: the carry after the last token, from a later loss
      float Ph = s.Q, Pl = s.pl;
      if (j) decay_pair(s.Q, s.pl, float(j), cp.w2, Ph, Pl);  // mid-window: P after token T-1
      const float2 e = end_carry(io, int64_t(b) * C + c, valid, Ph, Pl);
      beta = e.x;
      gamma = e.y;
    }
    // Reverse over the chunk; dk, dv (dr) replace k, v (r) in shared memory.
#pragma unroll 8
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
    if (ch == 0) {  // the start of the sequence: the initial state's gradients
      const float a0 = valid ? ck.x : 0.f, b0 = valid ? ck.y : 0.f;  // ck: the initial state
      if (io.da0 != nullptr && valid) {
        const int64_t sidx = int64_t(b) * C + c;
        io.da0[sidx] = beta;
        io.db0[sidx] = -gamma;
        io.dp0[sidx] = fmaf(a0, beta, -b0 * gamma);
      }
      dw_acc = fmaf(a0, betad, fmaf(-b0, gammad, dw_acc));  // -dw_acc is stored below
    }
    if (ch % kSW == 0) {  // the segment's first chunk: its partial sums are complete
      if (valid) {
        const int64_t nseg = bwd_nseg(T);
        lay.pdw[(int64_t(b) * nseg + ch / kSW) * C + c] = -dw_acc;
        lay.pdu[(int64_t(b) * nseg + ch / kSW) * C + c] = du_acc;
      }
      dw_acc = 0.f;
      du_acc = 0.f;
    }
    Tiles<TMA>::store(out_maps.m, outp, nstore, K, b, g, ch * kTT, T, C, lane);
    if (it + kMS < nch) {
      // The stores read this stage's tiles: let them finish reading before the refill.
      Tiles<TMA>::store_read_drain(lane);
      issue(s2, ch - kMS);
    }
  }
  Tiles<TMA>::store_drain(lane);
}

// ---- 2'. time-parallel reverse pass ------------------------------------------------------
// The reverse recurrences are linear in the carried sums, so a span of L tokens acts on the
// carry X = (beta~, gamma~, betad~, gammad~) at its end as an affine map: with E the product
// of the forward factors e1 over the span and (lb, lg, lbd, lgd) the span's own sums from a
// zero carry,
//   beta' = E beta + lb,  gamma' = E gamma + lg,
//   betad' = E (betad + L beta) + lbd,  gammad' = E (gammad + L gamma) + lgd
// (unrolling betad_{i-1} = e1_i (betad_i + beta_i) over the span). The maps of the chunks
// come out of the parallel forward recomputation; only the cheap application of a
// segment's maps to its carry is serial, chained from the last segment to the first.
struct RevAgg {
  float E, L, lb, lg, lbd, lgd;
};
struct RevCarry {
  float b, g, bd, gd;
};

__device__ __forceinline__ RevAgg rev_identity() { return RevAgg{1.f, 0.f, 0.f, 0.f, 0.f, 0.f}; }

// The carry at the start of span A, given the carry X at its end.
__device__ __forceinline__ RevCarry rev_apply(const RevAgg& A, const RevCarry& X) {
  RevCarry r;
  r.b = fmaf(A.E, X.b, A.lb);
  r.g = fmaf(A.E, X.g, A.lg);
  r.bd = fmaf(A.E, fmaf(A.L, X.b, X.bd), A.lbd);
  r.gd = fmaf(A.E, fmaf(A.L, X.g, X.gd), A.lgd);
  return r;
}

// A1 directly before A2 in time: rev_apply(rev_compose(A1, A2), X) = rev_apply(A1, rev_apply(A2, X)).
__device__ __forceinline__ RevAgg rev_compose(const RevAgg& A1, const RevAgg& A2) {
  RevAgg r;
  r.E = A1.E * A2.E;
  r.L = A1.L + A2.L;
  r.lb = fmaf(A1.E, A2.lb, A1.lb);
  r.lg = fmaf(A1.E, A2.lg, A1.lg);
  r.lbd = fmaf(A1.E, fmaf(A1.L, A2.lb, A2.lbd), A1.lbd);
  r.lgd = fmaf(A1.E, fmaf(A1.L, A2.lg, A2.lgd), A1.lgd);
  return r;
}

__device__ __forceinline__ void put_agg(float4* p, const RevAgg& A) {
  p[0] = make_float4(A.E, A.lb, A.lg, A.lbd);
  p[1] = make_float4(A.lgd, A.L, 0.f, 0.f);
}
__device__ __forceinline__ RevAgg get_agg(float4 x, float4 y) {
  return RevAgg{x.x, y.y, x.y, x.z, x.w, y.x};
}

// Per-token factors of one chunk from the forward recomputation. e1/e2: one of them is 1,
// the other is fe[t]; bit t of `tok` says which (set: the token's own term dominated,
// e1 = fe[t], e2 = 1). inj carries the token's dy. fe and inj stay in registers (every
// index is a compile-time constant after unrolling); wkv and cur (h e^{u+k}, with dy) go to
// shared memory in place of k and dy, which the reverse no longer needs.
struct ChunkFactors {
  float fe[kTT], inj[kTT];
  unsigned tok;
};

// Forward recomputation of one chunk of kTT tokens from its entering state s (left holding
// the state after the chunk): fills the per-token factors (wkv into K, cur into DY), writes
// dr in place of r (DR), and returns the chunk's reverse map (its sums from a zero carry,
// composed token by token in time order). Token by token, in either output form; the
// single-exponential form goes through chunk_forward_pairs below.
template <bool GATE, bool DR, bool FASTOUT, int RB, bool FWD>
__device__ __forceinline__ RevAgg chunk_forward(ChanState& s, const ChanParams& cp, float* K,
                                                const float* V, float* R, float* DY,
                                                ChunkFactors& f) {
  static_assert(kTT % RB == 0, "windows must tile the chunk");
  RevAgg A = rev_identity();
  f.tok = 0u;
#pragma unroll
  for (int t = 0; t < kTT; ++t) {
    const float kk = K[t * 32], vv = V[t * 32], gy = DY[t * 32];
    float m, d;
    if (FWD) {  // the streaming forward's scale: m against the window start, running maximum
      m = fmaf(float(t % RB + 1), cp.w2, fmaf(kk, kLog2e, -s.pl));
      d = m - s.Q;
    } else {  // as indep_step
      m = tok_log2w(float(t % RB + 1), cp.w2, kk);
      d = (m - s.Q) - s.pl;
    }
    const float e = ex2(-fabsf(d));
    const bool cnd = d > 0.f;
    const float e1 = cnd ? e : 1.f;
    const float e2 = cnd ? 1.f : e;
    if (FWD) {
      s.Q = fmaxf(s.Q, m);
    } else {
      s.Q = cnd ? m : s.Q;
      s.pl = cnd ? 0.f : s.pl;
    }
    float num, den, ki, kc;
    if (FASTOUT) {
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
    if (GATE) sig = rcp(1.f + ex2(R[t * 32] * -kLog2e));
    const float h = gy * sig * rden;  // dy sigmoid(r) / den
    const float wk = num * rden;
    const float inj = h * ki;
    f.fe[t] = e;
    f.tok |= cnd ? (1u << t) : 0u;
    f.inj[t] = inj;
    K[t * 32] = wk;
    DY[t * 32] = h * kc;
    if (DR) R[t * 32] = gy * wk * sig * (1.f - sig);  // dr in place of r
    // Compose the single-token map (E = e1, L = 1, l_beta = inj, l_gamma = inj wkv) after A.
    const float ej = A.E * inj;
    A.lbd = fmaf(ej, float(t), A.lbd);
    A.lgd = fmaf(ej * wk, float(t), A.lgd);
    A.lb += ej;
    A.lg = fmaf(ej, wk, A.lg);
    A.E *= e1;
    s.a = fmaf(e1, s.a, e2 * vv);
    s.b = fmaf(e1, s.b, e2);
    if ((t + 1) % RB == 0) wkv_rebase(s, float(RB) * cp.w2);
  }
  A.L = float(kTT);
  return A;
}

// chunk_forward in the single-exponential output form with the work off the serial chains
// two tokens to an fp32x2 instruction. The chains stay scalar, token by token, in the same
// operations as absorb_indep (so the state after the chunk is bit for bit the checkpoint
// pass's): the scale (d, the takeover selects, the window rebase), a and b, and the
// running product E of the map. Each token's a, b and E before it land in its half of a
// register pair for the packed output, gate, factor and dr arithmetic, whose lanes round
// as the scalar forms. The map's sums (lb, lg, lbd, lgd) are kept as even- and odd-token
// partial sums, added at the end.
template <bool GATE, bool DR, int RB, bool FWD>
__device__ __forceinline__ RevAgg chunk_forward_pairs(ChanState& s, const ChanParams& cp, float* K,
                                                      const float* V, float* R, float* DY,
                                                      ChunkFactors& f) {
  static_assert(kTT % RB == 0 && kTT % 2 == 0, "windows and pairs must tile the chunk");
  static_assert(!FWD || RB >= 2, "a pair must not straddle two windows of the forward's form");
  const float2 l2e = make_float2(kLog2e, kLog2e);
  const float2 w2 = make_float2(cp.w2, cp.w2);
  const float2 H = make_float2(cp.H, cp.H);
  float E = 1.f, a = s.a, b = s.b, Q = s.Q, pl = s.pl;
  float2 lb = make_float2(0.f, 0.f), lg = lb, lbd = lb, lgd = lb;
  f.tok = 0u;
#pragma unroll
  for (int t = 0; t < kTT; t += 2) {
    const float2 kk = make_float2(K[t * 32], K[(t + 1) * 32]);
    const float2 vv = make_float2(V[t * 32], V[(t + 1) * 32]);
    const float2 gy = make_float2(DY[t * 32], DY[(t + 1) * 32]);
    // FWD: the streaming forward's token weights, against the window start (RB >= 2: both
    // tokens of a pair share it); else tok_log2w of both tokens: the product rounded on its
    // own, then the fma
    float2 m;
    if (FWD)
      m = __ffma2_rn(make_float2(float(t % RB + 1), float((t + 1) % RB + 1)), w2,
                     __ffma2_rn(kk, l2e, make_float2(-pl, -pl)));
    else
      m = __ffma2_rn(make_float2(float(t % RB + 1), float((t + 1) % RB + 1)), w2,
                     __fmul2_rn(kk, l2e));
    float2 sig = make_float2(1.f, 1.f);
    if (GATE) {
      const float2 x = __fmul2_rn(make_float2(R[t * 32], R[(t + 1) * 32]),
                                  make_float2(-kLog2e, -kLog2e));
      const float2 q = __fadd2_rn(make_float2(ex2(x.x), ex2(x.y)), make_float2(1.f, 1.f));
      sig = make_float2(rcp(q.x), rcp(q.y));
    }
    // the scale chain, token t then t + 1 (as absorb_indep)
    float ee[2], e1s[2], e2s[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float mh = h ? m.y : m.x;
      const float d = FWD ? mh - Q : (mh - Q) - pl;
      ee[h] = ex2(-fabsf(d));
      const bool cnd = d > 0.f;
      e1s[h] = cnd ? ee[h] : 1.f;
      e2s[h] = cnd ? 1.f : ee[h];
      if (FWD) {
        Q = fmaxf(Q, mh);
      } else {
        Q = cnd ? mh : Q;
        pl = cnd ? 0.f : pl;
      }
      f.tok |= cnd ? (1u << (t + h)) : 0u;
      if ((t + h + 1) % RB == 0) indep_rebase(Q, pl, float(RB) * cp.w2);
    }
    f.fe[t] = ee[0];
    f.fe[t + 1] = ee[1];
    const float2 e1 = make_float2(e1s[0], e1s[1]);
    const float2 e2 = make_float2(e2s[0], e2s[1]);
    // the a, b and E chains; each value before its token kept for the pair
    const float2 ev = __fmul2_rn(e2, vv);
    float2 ap, bp, Ep;
    ap.x = a;
    bp.x = b;
    Ep.x = E;
    a = fmaf(e1.x, a, ev.x);
    b = fmaf(e1.x, b, e2.x);
    E *= e1.x;
    ap.y = a;
    bp.y = b;
    Ep.y = E;
    a = fmaf(e1.y, a, ev.y);
    b = fmaf(e1.y, b, e2.y);
    E *= e1.y;
    // output, factors, dr, and the map's sums
    const float2 he = __fmul2_rn(H, e2);
    const float2 num = __ffma2_rn(e1, ap, __fmul2_rn(he, vv));
    const float2 den = __ffma2_rn(e1, bp, he);
    const float2 rden = make_float2(rcp(den.x), rcp(den.y));
    const float2 hh = __fmul2_rn(__fmul2_rn(gy, sig), rden);  // dy sigmoid(r) / den
    const float2 wk = __fmul2_rn(num, rden);
    const float2 inj = __fmul2_rn(hh, e1);
    f.inj[t] = inj.x;
    f.inj[t + 1] = inj.y;
    K[t * 32] = wk.x;
    K[(t + 1) * 32] = wk.y;
    const float2 cur = __fmul2_rn(hh, he);
    DY[t * 32] = cur.x;
    DY[(t + 1) * 32] = cur.y;
    if (DR) {
      const float2 dr = __fmul2_rn(__fmul2_rn(__fmul2_rn(gy, wk), sig),
                                   __ffma2_rn(sig, make_float2(-1.f, -1.f), make_float2(1.f, 1.f)));
      R[t * 32] = dr.x;
      R[(t + 1) * 32] = dr.y;
    }
    const float2 ej = __fmul2_rn(Ep, inj);
    const float2 tt = make_float2(float(t), float(t + 1));
    lbd = __ffma2_rn(ej, tt, lbd);
    lgd = __ffma2_rn(__fmul2_rn(ej, wk), tt, lgd);
    lb = __fadd2_rn(lb, ej);
    lg = __ffma2_rn(ej, wk, lg);
  }
  s.a = a;
  s.b = b;
  s.Q = Q;
  s.pl = pl;
  RevAgg A;
  A.E = E;
  A.L = float(kTT);
  A.lb = lb.x + lb.y;
  A.lg = lg.x + lg.y;
  A.lbd = lbd.x + lbd.y;
  A.lgd = lgd.x + lgd.y;
  return A;
}

template <bool GATE, bool DR, bool FASTOUT, bool FWD>
__device__ __forceinline__ RevAgg chunk_forward_rb(ChanState& s, const ChanParams& cp, int rb,
                                                   float* K, const float* V, float* R, float* DY,
                                                   ChunkFactors& f) {
  if constexpr (FASTOUT) {
    if (rb == 16) return chunk_forward_pairs<GATE, DR, 16, FWD>(s, cp, K, V, R, DY, f);
    if (rb == 4) return chunk_forward_pairs<GATE, DR, 4, FWD>(s, cp, K, V, R, DY, f);
    if constexpr (FWD)  // windows of one token: each its own window start
      return chunk_forward<GATE, DR, true, 1, FWD>(s, cp, K, V, R, DY, f);
    else
      return chunk_forward_pairs<GATE, DR, 1, FWD>(s, cp, K, V, R, DY, f);
  } else {
    if (rb == 16) return chunk_forward<GATE, DR, false, 16, FWD>(s, cp, K, V, R, DY, f);
    if (rb == 4) return chunk_forward<GATE, DR, false, 4, FWD>(s, cp, K, V, R, DY, f);
    return chunk_forward<GATE, DR, false, 1, FWD>(s, cp, K, V, R, DY, f);
  }
}

// Reverse over one chunk from the carry X after its last real token (position nvalid - 1;
// TAIL: nvalid < kTT, the positions after it are skipped): dk, dv replace wkv (in K), v in
// shared memory; returns the chunk's partial sums of -dw (.x) and du (.y).
template <bool TAIL>
__device__ __forceinline__ float2 chunk_reverse(const ChunkFactors& f, RevCarry X, float* K,
                                                float* V, const float* CUR, int nvalid) {
  float dw_acc = 0.f, du_acc = 0.f;
#pragma unroll
  for (int t = kTT - 1; t >= 0; --t) {
    if (TAIL && t >= nvalid) continue;
    const float vv = V[t * 32], wk = K[t * 32], cur = CUR[t * 32];
    const bool dom = (f.tok >> t) & 1u;
    const float e1 = dom ? f.fe[t] : 1.f;
    const float e2 = dom ? 1.f : f.fe[t];
    const float inj = f.inj[t];
    const float vm = vv - wk;
    V[t * 32] = fmaf(e2, X.b, cur);                            // dv
    K[t * 32] = fmaf(cur, vm, e2 * fmaf(vv, X.b, -X.g));       // dk
    dw_acc = fmaf(e2, fmaf(vv, X.bd, -X.gd), dw_acc);
    du_acc = fmaf(cur, vm, du_acc);
    X.bd = e1 * (X.bd + X.b);
    X.gd = e1 * (X.gd + X.g);
    X.b = fmaf(e1, X.b, inj);
    X.g = fmaf(e1, X.g, inj * wk);
  }
  return make_float2(-dw_acc, du_acc);
}

// chunk_reverse over a whole chunk with the work off the carry's chains two tokens (t and
// t - 1) to an fp32x2 instruction. The chains stay scalar, token by token, and carry -gamma
// and -gammad in place of gamma and gammad (negation is exact, so every value is the
// scalar form's, with the subtractions dk and dw need turned into the fma's own add). The
// carry before each token lands in its half of a register pair for dv, dk and the dw, du
// terms; dw and du are kept as partial sums by token parity.
__device__ __forceinline__ float2 chunk_reverse_pairs(const ChunkFactors& f, RevCarry X, float* K,
                                                      float* V, const float* CUR) {
  static_assert(kTT % 2 == 0, "pairs must tile the chunk");
  float xb = X.b, ng = -X.g, xbd = X.bd, ngd = -X.gd;
  float2 dw = make_float2(0.f, 0.f), du = dw;
#pragma unroll
  for (int t = kTT - 1; t > 0; t -= 2) {
    const float2 vv = make_float2(V[t * 32], V[(t - 1) * 32]);
    const float2 wk = make_float2(K[t * 32], K[(t - 1) * 32]);
    const float2 cur = make_float2(CUR[t * 32], CUR[(t - 1) * 32]);
    const float2 inj = make_float2(f.inj[t], f.inj[t - 1]);
    const bool d0 = (f.tok >> t) & 1u, d1 = (f.tok >> (t - 1)) & 1u;
    const float2 e1 = make_float2(d0 ? f.fe[t] : 1.f, d1 ? f.fe[t - 1] : 1.f);
    const float2 e2 = make_float2(d0 ? 1.f : f.fe[t], d1 ? 1.f : f.fe[t - 1]);
    const float2 iw = __fmul2_rn(inj, wk);
    float2 pb, png, pbd, pngd;  // the carry before each token of the pair
    pb.x = xb;
    png.x = ng;
    pbd.x = xbd;
    pngd.x = ngd;
    xbd = e1.x * (xbd + xb);
    ngd = e1.x * (ngd + ng);
    xb = fmaf(e1.x, xb, inj.x);
    ng = fmaf(e1.x, ng, -iw.x);
    pb.y = xb;
    png.y = ng;
    pbd.y = xbd;
    pngd.y = ngd;
    xbd = e1.y * (xbd + xb);
    ngd = e1.y * (ngd + ng);
    xb = fmaf(e1.y, xb, inj.y);
    ng = fmaf(e1.y, ng, -iw.y);
    const float2 vm = __ffma2_rn(wk, make_float2(-1.f, -1.f), vv);  // v - wkv
    const float2 dv = __ffma2_rn(e2, pb, cur);
    const float2 dk = __ffma2_rn(cur, vm, __fmul2_rn(e2, __ffma2_rn(vv, pb, png)));
    dw = __ffma2_rn(e2, __ffma2_rn(vv, pbd, pngd), dw);
    du = __ffma2_rn(cur, vm, du);
    V[t * 32] = dv.x;
    V[(t - 1) * 32] = dv.y;
    K[t * 32] = dk.x;
    K[(t - 1) * 32] = dk.y;
  }
  return make_float2(-(dw.x + dw.y), du.x + du.y);
}

// One CTA per (segment of kSW chunks, batch row, 32-channel group); warp i owns chunk
// kSW seg + i. CTAs take segments in ticket order from the LAST segment backward, so every
// segment a CTA waits for belongs to a CTA that started earlier: the waits always end.
//   1. every warp TMA-loads its chunk's k, v, (r,) dy tiles and recomputes the forward from
//      the chunk's checkpoint: factors, dr in place of r, and the chunk's reverse map;
//   2. warp 0 publishes the segment's map; the last warp forms the carry at the segment's
//      end in a fixed order (bitwise reproducible): the carry published at the start of
//      segment jc = seg + kFoldR + 1 (zero past the end), then the maps of segments
//      jc-1 .. seg+1, so one link of a serial chain spans kFoldR + 1 segments;
//   3. each warp applies the maps of the chunks after it to that carry and runs the reverse
//      over its chunk: dk, dv in place of wkv, v, TMA-stored with dr; warp 0 publishes the
//      carry at the segment's start where a segment further back starts from it; the
//      chunks' partial sums of dw, du are added in a fixed order into per-segment partials.
template <bool GATE, bool DR, bool FWD>
__global__ void __launch_bounds__(kSW * 32, 5)
    wkv_bwd_seg_kernel(const __grid_constant__ TensorMaps4 in_maps,
                       const __grid_constant__ TensorMaps4 out_maps, int B, int T, int C,
                       const float* __restrict__ w, const float* __restrict__ u,
                       const StateIO io, void* ws, unsigned* err, unsigned long long wait_ns,
                       int withhold_last_map) {
  constexpr int kTile = kTT * 32;
  constexpr int kNL = GATE ? 4 : 3;  // tiles per chunk: k, v, (r,) dy
  // Dynamic: [kSW warps][kNL tiles][kTile] floats.
  extern __shared__ __align__(128) float dyn_tiles[];
  __shared__ float4 sagg[kSW][32][2];           // the chunks' reverse maps
  __shared__ float4 sfold[2 * kFoldR + 1][32];  // later segments' maps and carry
  __shared__ float4 sxe[32];                    // the carry at the segment's end
  __shared__ uint64_t bars[kSW];
  __shared__ unsigned s_tk[3];
  // The chunks' partial sums (-dw, du), in sfold's space (used at other times).
  static_assert(2 * kFoldR + 1 >= kSW / 2, "spart must fit in sfold");
  auto spart = reinterpret_cast<float2(*)[32]>(&sfold[0][0]);

  const int G = (C + 31) >> 5;
  const int64_t nbg = int64_t(B) * G;
  const int nch = (T + kTT - 1) / kTT;
  const int nseg = (nch + kSW - 1) / kSW;
  const BwdLayout lay = bwd_layout(ws, B, T, C);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {  // ticket -> (segments from the end, batch row, channel group)
    const unsigned tk = atomicAdd(lay.rticket, 1u);  // < 2^31 (host check)
    const unsigned bk = tk / unsigned(nbg);
    const unsigned r = tk - bk * unsigned(nbg);
    const unsigned bb = r / unsigned(G);
    s_tk[0] = bk;
    s_tk[1] = bb;
    s_tk[2] = r - bb * unsigned(G);
  }
  __syncthreads();
  const int seg = nseg - 1 - int(s_tk[0]);
  const int b = int(s_tk[1]);
  const int g = int(s_tk[2]);
  const int64_t bg = int64_t(b) * G + g;
  const int c = (g << 5) + lane;
  const bool valid = c < C;
  const int ch = seg * kSW + warp;
  const bool live = ch < nch;
  const int t0 = ch * kTT;
  const int64_t item0 = bg * nseg;
  const int64_t item = item0 + seg;
  float* tiles = dyn_tiles + warp * kNL * kTile;
  float* K = tiles + lane;
  float* V = tiles + kTile + lane;
  float* R = tiles + 2 * kTile + lane;
  float* DY = tiles + (kNL - 1) * kTile + lane;
  uint64_t* bar = &bars[warp];
  if (lane == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
    if (live) {
      mbar_arrive_expect_tx(bar, uint32_t(kNL) * kTile * sizeof(float));
      for (int i = 0; i < kNL; ++i) tma_load_3d(tiles + i * kTile, &in_maps.m[i], bar, g << 5, t0, b);
    }
  }
  __syncwarp();
  const float4 ck = (live && valid) ? lay.ckpt[(int64_t(b) * nch + ch) * C + c]
                                    : make_float4(0.f, 0.f, kEmptyLogScale, 0.f);
  // The log2-scale of the state entering the next chunk (its checkpoint; after the last
  // chunk, the state after the last token), see below.
  const int64_t sidx = int64_t(b) * C + c;
  const float2 nsc = (ch < nch && valid)
                         ? *reinterpret_cast<const float2*>(
                               ch + 1 < nch ? &lay.ckpt[(int64_t(b) * nch + ch + 1) * C + c].z
                                            : &lay.ckend[sidx].z)
                         : make_float2(0.f, 0.f);
  const int nvalid = min(kTT, T - t0);  // real tokens of this chunk
  const ChanParams cp = chan_params(valid ? w[c] : 1.f, valid ? u[c] : 0.f);
  const bool fast = __all_sync(0xffffffffu, fabsf(cp.uw2) <= kFastOutBound);
  const int rb = window_tokens(cp.w2, 128.f);
  // The fold's inputs (step 2) are usually published before this segment starts: the last
  // warp checks their flags now (one acquire load per lane, while the tiles load) and, if
  // all are set, copies them into shared memory (cp.async) during the forward
  // recomputation; otherwise it waits for them after that.
  const int jc = min(nseg, seg + kFoldR + 1);
  const int mfold = jc - 1 - seg;  // maps to apply
  const unsigned fwant = lane < mfold ? 1u : ((lane == 31 && jc < nseg) ? 2u : 0u);
  bool fold_early = false;
  if (warp == kSW - 1) {
    const unsigned* flag = lane < mfold ? &lay.rflags[item0 + seg + 1 + lane] : &lay.rflags[item0 + jc];
    const unsigned fl = fwant != 0 ? ld_acquire(flag) : 0u;
    fold_early = __all_sync(0xffffffffu, fl >= fwant);
    __syncwarp();  // orders every lane's acquire before every lane's copies below
    if (fold_early) {
      for (int l = 0; l < 2 * mfold; ++l)  // map of segment seg + 1 + l / 2, half l % 2
        cp_async_16(&sfold[l][lane], &lay.rmap[((item0 + seg + 1 + (l >> 1)) * 32 + lane) * 2 + (l & 1)]);
      if (jc < nseg) cp_async_16(&sfold[2 * mfold][lane], &lay.carry[(item0 + jc) * 32 + lane]);
      cp_async_commit();
    }
  }

  // ---- 1. forward recomputation and the chunk's reverse map ----
  ChunkFactors f;
  RevAgg A = rev_identity();
  ChanState s;
  s.a = ck.x;
  s.b = ck.y;
  s.Q = ck.z;
  s.pl = ck.w;
  if (live) {
    mbar_wait_suspend(bar, 0, err);
    __syncwarp();
    // Past the last token (zero-filled tiles): a weight of 2^{-huge} makes the positions
    // inert (e1 = 1, e2 = 0: the state and the reverse sums pass through unchanged).
    for (int t = nvalid; t < kTT; ++t) K[t * 32] = -1.0e30f;
    A = fast ? chunk_forward_rb<GATE, DR, true, FWD>(s, cp, rb, K, V, R, DY, f)
             : chunk_forward_rb<GATE, DR, false, FWD>(s, cp, rb, K, V, R, DY, f);
    A.L = float(nvalid);  // the inert positions add no distance
  }
  // The carry at this chunk's end comes scaled by the state entering the next chunk (its
  // checkpoint, or the state after the last token); this chunk's own sums are scaled by
  // its recomputed state after its last real token. Both are the same state reached by
  // different orders of rounding: rescale by the exact ratio of the two scales
  // (beta~ = beta 2^P) so the reverse sums stay consistent. The factor is folded into the
  // chunk's map (E) for the chunks before it. (Inert positions after the last token moved
  // the frame on by (kTT - nvalid) w2: undone here.)
  float Ph = s.Q, Pl = s.pl;
  if (nvalid < kTT) decay_pair(s.Q, s.pl, float(nvalid - kTT), cp.w2, Ph, Pl);
  const float rme = (live && valid) ? ex2(fminf((Ph - nsc.x) + (Pl - nsc.y), 64.f)) : 1.f;
  A.E *= rme;
  put_agg(&sagg[warp][lane][0], A);
  __syncthreads();

  // ---- 2. the segment's map; the carry at its end ----
  if (warp == 0 && seg > 0 && !(withhold_last_map && seg == nseg - 1)) {
    // the segment's map, for the segments before it
    RevAgg M = get_agg(sagg[kSW - 1][lane][0], sagg[kSW - 1][lane][1]);
#pragma unroll
    for (int i = kSW - 2; i >= 0; --i) M = rev_compose(get_agg(sagg[i][lane][0], sagg[i][lane][1]), M);
    put_agg(&lay.rmap[(item * 32 + lane) * 2], M);
    warp_publish(&lay.rflags[item], 1u);
  }
  if (warp == kSW - 1) {
    const int m = mfold;
    bool ok = true;
    if (fold_early) {
      cp_async_wait_all();
    } else {  // wait for the flags not yet set, then fetch (L2 loads: L1 may be stale)
      const unsigned* flag = lane < m ? &lay.rflags[item0 + seg + 1 + lane] : &lay.rflags[item0 + jc];
      const unsigned fl = fwant != 0 ? wait_flag(flag, fwant, wait_ns, err) : 1u;
      ok = __all_sync(0xffffffffu, fl != 0);
      __syncwarp();  // orders every lane's acquire before every lane's fetch below
      if (ok) {  // (a wait that gave up flagged the error word: continue from a zero carry)
        for (int l = 0; l < 2 * m; ++l)
          sfold[l][lane] = __ldcg(&lay.rmap[((item0 + seg + 1 + (l >> 1)) * 32 + lane) * 2 + (l & 1)]);
        if (jc < nseg) sfold[2 * m][lane] = __ldcg(&lay.carry[(item0 + jc) * 32 + lane]);
      }
    }
    __syncwarp();
    RevCarry X{0.f, 0.f, 0.f, 0.f};
    if (jc == nseg) {  // the carry at the end of the sequence (a later loss's gradient)
      if (io.ga1 != nullptr && valid) {
        const float4 q = lay.ckend[sidx];
        const float2 e = end_carry(io, sidx, valid, q.z, q.w);
        X = RevCarry{e.x, e.y, 0.f, 0.f};
      }
    } else if (ok) {
      const float4 q = sfold[2 * m][lane];
      X = RevCarry{q.x, q.y, q.z, q.w};
    }
    if (ok)
      for (int l = m - 1; l >= 0; --l)
        X = rev_apply(get_agg(sfold[2 * l][lane], sfold[2 * l + 1][lane]), X);
    sxe[lane] = make_float4(X.b, X.g, X.bd, X.gd);
  }
  __syncthreads();

  // ---- 3. carries, reverse over the chunks ----
  const float4 xe = sxe[lane];
  RevCarry X{xe.x, xe.y, xe.z, xe.w};
  for (int i = kSW - 1; i > warp; --i) X = rev_apply(get_agg(sagg[i][lane][0], sagg[i][lane][1]), X);
  if (warp == 0 && seg > kFoldR) {  // segment seg - kFoldR - 1 starts from this carry
    const RevCarry X0 = rev_apply(A, X);
    lay.carry[item * 32 + lane] = make_float4(X0.b, X0.g, X0.bd, X0.gd);
    warp_publish(&lay.rflags[item], 2u);
  }
  float dw_init = 0.f;  // the initial state's part of dw (first segment)
  if (warp == 0 && seg == 0) {
    // The carry at the start of the sequence is scaled by the initial state's own scale
    // (the first checkpoint is that state as given): beta~ = e^{p0} dL/dA0 = dL/da0.
    const RevCarry X0 = rev_apply(A, X);
    const float a0 = ck.x, b0 = ck.y;
    if (io.da0 != nullptr && valid) {
      io.da0[sidx] = X0.b;
      io.db0[sidx] = -X0.g;
      io.dp0[sidx] = fmaf(a0, X0.b, -b0 * X0.g);
    }
    dw_init = -fmaf(a0, X0.bd, -b0 * X0.gd);
  }
  float2 part = make_float2(0.f, 0.f);
  if (live) {
    const RevCarry Xc{X.b * rme, X.g * rme, X.bd * rme, X.gd * rme};
    part = nvalid == kTT ? chunk_reverse_pairs(f, Xc, K, V, DY)
                         : chunk_reverse<true>(f, Xc, K, V, DY, nvalid);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      for (int i = 0; i < (DR ? 3 : 2); ++i) tma_store_3d(&out_maps.m[i], tiles + i * kTile, g << 5, t0, b);
      tma_store_commit();
    }
    __syncwarp();
  }
  spart[warp][lane] = part;  // (sfold's last reader, the fold, ended before the barrier above)
  __syncthreads();
  if (warp == 0 && valid) {  // the segment's partial sums, chunks in a fixed order
    float sw = dw_init, su = 0.f;
#pragma unroll
    for (int i = 0; i < kSW; ++i) {
      sw += spart[i][lane].x;
      su += spart[i][lane].y;
    }
    lay.pdw[(int64_t(b) * nseg + seg) * C + c] = sw;
    lay.pdu[(int64_t(b) * nseg + seg) * C + c] = su;
  }
  if (live && lane == 0) tma_store_wait_read<0>();  // the tiles stay until the stores read them
  __syncwarp();
}

// ---- 2'. reverse pass, one persistent CTA per channel group -----------------------------
// When there are more channel groups (batch row x 32 channels) than a wave of the
// time-parallel pass needs to fill the GPU, one CTA per group walks the group's segments
// from the last to the first: NW warps recompute and reverse the segment's NW chunks in
// parallel, as in wkv_bwd_seg_kernel, but the carry at the segment's end comes from the
// previous iteration in shared memory. No tickets, no published maps, no waits on other
// CTAs. The next segment's tiles are brought into L2 while this one is worked on. The CTA
// adds its segments' partial sums of dw, du in a fixed order (last segment first) into one
// row per batch row; the last CTA of a channel group to finish (a counter per group, zero
// on entry) adds the group's rows in batch order and writes dw, du: no reduction kernel.
template <bool GATE, bool DR, bool FWD, int NW>
__global__ void __launch_bounds__(NW * 32, NW <= 4 ? 4 : 3)
    wkv_bwd_group_kernel(const __grid_constant__ TensorMaps4 in_maps,
                         const __grid_constant__ TensorMaps4 out_maps, int B, int T, int C,
                         const float* __restrict__ w, const float* __restrict__ u,
                         const StateIO io, void* ws, unsigned* err, const Ptr4 pre,
                         float* __restrict__ dw, float* __restrict__ du) {
  constexpr int kTile = kTT * 32;
  constexpr int kNL = GATE ? 4 : 3;  // tiles per chunk: k, v, (r,) dy
  extern __shared__ __align__(128) float dyn_tiles[];
  __shared__ float4 sagg[NW][32][2];  // the chunks' reverse maps
  __shared__ float4 sxe[2][32];        // the carry at the segment's end (double-buffered)
  __shared__ float2 spart[NW][32];    // the chunks' partial sums (-dw, du)
  __shared__ uint64_t bars[NW];

  const int G = (C + 31) >> 5;
  const int nch = (T + kTT - 1) / kTT;
  const int nseg = (nch + NW - 1) / NW;  // this kernel's segments of NW chunks
  const BwdLayout lay = bwd_layout(ws, B, T, C);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = int(blockIdx.x) / G, g = int(blockIdx.x) % G;
  const int c = (g << 5) + lane;
  const bool valid = c < C;
  const int64_t sidx = int64_t(b) * C + c;
  const ChanParams cp = chan_params(valid ? w[c] : 1.f, valid ? u[c] : 0.f);
  const bool fast = __all_sync(0xffffffffu, fabsf(cp.uw2) <= kFastOutBound);
  const int rb = window_tokens(cp.w2, 128.f);
  float* tiles = dyn_tiles + warp * kNL * kTile;
  float* K = tiles + lane;
  float* V = tiles + kTile + lane;
  float* R = tiles + 2 * kTile + lane;
  float* DY = tiles + (kNL - 1) * kTile + lane;
  uint64_t* bar = &bars[warp];
  if (lane == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
  }
  // The carry at the end of the sequence (a later loss's gradient, else zero).
  if (warp == 0) {
    float2 e = make_float2(0.f, 0.f);
    if (io.ga1 != nullptr && valid) {
      const float4 q = lay.ckend[sidx];
      e = end_carry(io, sidx, valid, q.z, q.w);
    }
    sxe[0][lane] = make_float4(e.x, e.y, 0.f, 0.f);
  }
  __syncthreads();

  uint32_t phase = 0;
  float tw = 0.f, tu = 0.f;  // warp 0: this batch row's sums of -dw, du so far
  for (int seg = nseg - 1, it = 0; seg >= 0; --seg, ++it) {
    const int ch = seg * NW + warp;
    const bool live = ch < nch;
    const int t0 = ch * kTT;
    if (lane == 0 && live) {
      mbar_arrive_expect_tx(bar, uint32_t(kNL) * kTile * sizeof(float));
      for (int i = 0; i < kNL; ++i) tma_load_3d(tiles + i * kTile, &in_maps.m[i], bar, g << 5, t0, b);
    }
    // the next (earlier) segment's rows of this warp's chunk into L2 meanwhile
    if (seg > 0) {
      const int tn = (seg - 1) * NW * kTT + warp * kTT + (lane & 15);
      const int64_t off = (int64_t(b) * T + tn) * C + (int64_t(g) << 5);
#pragma unroll
      for (int i = 0; i < 2; ++i) prefetch_l2(pre[2 * (lane >> 4) + i] + off);
    }
    __syncwarp();
    const float4 ck = (live && valid) ? lay.ckpt[(int64_t(b) * nch + ch) * C + c]
                                      : make_float4(0.f, 0.f, kEmptyLogScale, 0.f);
    const float2 nsc = (live && valid)
                           ? *reinterpret_cast<const float2*>(
                                 ch + 1 < nch ? &lay.ckpt[(int64_t(b) * nch + ch + 1) * C + c].z
                                              : &lay.ckend[sidx].z)
                           : make_float2(0.f, 0.f);
    const int nvalid = min(kTT, T - t0);

    // ---- forward recomputation and the chunk's reverse map ----
    ChunkFactors f;
    RevAgg A = rev_identity();
    ChanState s;
    s.a = ck.x;
    s.b = ck.y;
    s.Q = ck.z;
    s.pl = ck.w;
    if (live) {
      mbar_wait_suspend(bar, phase, err);
      phase ^= 1u;
      __syncwarp();
      for (int t = nvalid; t < kTT; ++t) K[t * 32] = -1.0e30f;  // inert positions
      A = fast ? chunk_forward_rb<GATE, DR, true, FWD>(s, cp, rb, K, V, R, DY, f)
               : chunk_forward_rb<GATE, DR, false, FWD>(s, cp, rb, K, V, R, DY, f);
      A.L = float(nvalid);
    }
    // the exact ratio between this chunk's recomputed end scale and the next checkpoint's
    float Ph = s.Q, Pl = s.pl;
    if (nvalid < kTT) decay_pair(s.Q, s.pl, float(nvalid - kTT), cp.w2, Ph, Pl);
    const float rme = (live && valid) ? ex2(fminf((Ph - nsc.x) + (Pl - nsc.y), 64.f)) : 1.f;
    A.E *= rme;
    put_agg(&sagg[warp][lane][0], A);
    __syncthreads();

    // ---- the carry at this chunk's end; the carry at the segment's start for the next ----
    const float4 xe = sxe[it & 1][lane];
    RevCarry X{xe.x, xe.y, xe.z, xe.w};
    for (int i = NW - 1; i > warp; --i) X = rev_apply(get_agg(sagg[i][lane][0], sagg[i][lane][1]), X);
    float dw_init = 0.f;  // the initial state's part of dw (first segment)
    if (warp == 0) {
      const RevCarry X0 = rev_apply(A, X);
      sxe[(it + 1) & 1][lane] = make_float4(X0.b, X0.g, X0.bd, X0.gd);
      if (seg == 0) {
        // The carry at the start of the sequence is scaled by the initial state's own
        // scale (the first checkpoint is that state as given): beta~ = dL/da0.
        const float a0 = ck.x, b0 = ck.y;
        if (io.da0 != nullptr && valid) {
          io.da0[sidx] = X0.b;
          io.db0[sidx] = -X0.g;
          io.dp0[sidx] = fmaf(a0, X0.b, -b0 * X0.g);
        }
        dw_init = -fmaf(a0, X0.bd, -b0 * X0.gd);
      }
    }
    float2 part = make_float2(0.f, 0.f);
    if (live) {
      const RevCarry Xc{X.b * rme, X.g * rme, X.bd * rme, X.gd * rme};
      part = nvalid == kTT ? chunk_reverse_pairs(f, Xc, K, V, DY)
                           : chunk_reverse<true>(f, Xc, K, V, DY, nvalid);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        for (int i = 0; i < (DR ? 3 : 2); ++i) tma_store_3d(&out_maps.m[i], tiles + i * kTile, g << 5, t0, b);
        tma_store_commit();
      }
      __syncwarp();
    }
    spart[warp][lane] = part;
    __syncthreads();
    if (warp == 0) {  // the segment's partial sums, chunks in a fixed order
      float sw = dw_init, su = 0.f;
#pragma unroll
      for (int i = 0; i < NW; ++i) {
        sw += spart[i][lane].x;
        su += spart[i][lane].y;
      }
      tw += sw;
      tu += su;
    }
    if (live && lane == 0) tma_store_wait_read<0>();  // the tiles are reloaded next
    __syncwarp();
  }
  // ---- this batch row's sums; the group's last CTA adds the rows and writes dw, du ----
  if (warp == 0) {
    if (valid) {
      __stcg(&lay.pdw[int64_t(b) * bwd_nseg(T) * C + c], tw);
      __stcg(&lay.pdu[int64_t(b) * bwd_nseg(T) * C + c], tu);
    }
    __threadfence();  // the row is visible before the count says so
    __syncwarp();
    unsigned done = 0;
    if (lane == 0) done = atomicAdd(&lay.fflags[g], 1u);
    done = __shfl_sync(0xffffffffu, done, 0);
    if (done == unsigned(B) - 1u) {
      __threadfence();  // every other row is visible after the count that said so
      float sw = 0.f, su = 0.f;
      if (valid)
        for (int bb = 0; bb < B; ++bb) {
          sw += __ldcg(&lay.pdw[int64_t(bb) * bwd_nseg(T) * C + c]);
          su += __ldcg(&lay.pdu[int64_t(bb) * bwd_nseg(T) * C + c]);
        }
      if (valid) {
        dw[c] = sw;
        du[c] = su;
      }
    }
  }
}

// ---- 3. reduction over batch rows and segments, fixed order -------------------------------
// Block (32, kRS): lane x owns a channel; slice y sums the rows y, y + kRS, ... in order,
// then slice 0 adds the slices' sums in order. Same order on every call: deterministic.
constexpr int kRS = 32;
__global__ void __launch_bounds__(32 * kRS) wkv_bwd_reduce_kernel(int B, int C, const void* ws,
                                                                 int T, float* dw, float* du) {
  __shared__ float2 sp[kRS][33];
  const int c = blockIdx.x * 32 + threadIdx.x;
  const BwdLayout lay = bwd_layout(const_cast<void*>(ws), B, T, C);
  const int64_t rows = int64_t(B) * bwd_nseg(T);
  float sw = 0.f, su = 0.f;
  if (c < C) {
#pragma unroll 8
    for (int64_t i = threadIdx.y; i < rows; i += kRS) {
      sw += lay.pdw[i * C + c];
      su += lay.pdu[i * C + c];
    }
  }
  sp[threadIdx.y][threadIdx.x] = make_float2(sw, su);
  __syncthreads();
  if (threadIdx.y == 0 && c < C) {
    float tw = 0.f, tu = 0.f;
    for (int y = 0; y < kRS; ++y) {
      tw += sp[y][threadIdx.x].x;
      tu += sp[y][threadIdx.x].y;
    }
    dw[c] = tw;
    du[c] = tu;
  }
}

StateIO state_io(const BwdArgs& a) {
  return StateIO{a.a0, a.b0, a.p0, a.ga1, a.gb1, a.p1, a.da0, a.db0, a.dp0};
}

size_t bwd_main_smem() {
  return (4 * kMS + 6) * kTT * 32 * sizeof(float) + kMS * sizeof(uint64_t);
}

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
                                             int(a.B), int(a.T), int(a.C), a.w, a.u,
                                             state_io(a), a.ws, a.err);
  return cudaPeekAtLastError() == cudaSuccess ? WKV_OK : WKV_ERR_CUDA;
}

template <bool GATE, bool DR>
int launch_seg(const BwdArgs& a, const TensorMaps4& in, const TensorMaps4& out, int64_t nitems,
               cudaStream_t stream) {
  // Checkpoints made by the streaming forward: recompute in its arithmetic.
  auto kern = a.have_ckpt ? wkv_bwd_seg_kernel<GATE, DR, true> : wkv_bwd_seg_kernel<GATE, DR, false>;
  const size_t smem = size_t(kSW) * (GATE ? 4 : 3) * kTT * 32 * sizeof(float);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
      cudaSuccess)
    return WKV_ERR_CUDA;
  kern<<<unsigned(nitems), kSW * 32, smem, stream>>>(in, out, int(a.B), int(a.T), int(a.C), a.w,
                                                      a.u, state_io(a), a.ws, a.err, a.wait_ns,
                                                      a.withhold_last_map);
  return cudaPeekAtLastError() == cudaSuccess ? WKV_OK : WKV_ERR_CUDA;
}

// Reverse pass with one CTA per channel group: taken when there are enough groups to fill
// the GPU (one wave of CTAs at least as wide as the SMs), or when a test forces it.
// 0 automatic, 1 time-parallel segments, 2 per group (warps per CTA automatic), 3 per group
// with 4 warps per CTA.
std::atomic<int> g_bwd_path{0};

int sm_count() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

bool use_group_path(const BwdArgs& a) {
  const int forced = g_bwd_path.load();
  if (forced != 0) return forced >= 2;
  return a.B * ((a.C + 31) / 32) >= 2 * int64_t(sm_count());
}

template <bool GATE, bool DR, int NW>
int launch_group_nw(const BwdArgs& a, const TensorMaps4& in, const TensorMaps4& out,
                    cudaStream_t stream) {
  auto kern = a.have_ckpt ? wkv_bwd_group_kernel<GATE, DR, true, NW>
                          : wkv_bwd_group_kernel<GATE, DR, false, NW>;
  const size_t smem = size_t(NW) * (GATE ? 4 : 3) * kTT * 32 * sizeof(float);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
      cudaSuccess)
    return WKV_ERR_CUDA;
  const Ptr4 pre{a.k, a.v, a.r ? a.r : a.dy, a.dy};
  kern<<<unsigned(a.B * ((a.C + 31) / 32)), NW * 32, smem, stream>>>(
      in, out, int(a.B), int(a.T), int(a.C), a.w, a.u, state_io(a), a.ws, a.err, pre, a.dw,
      a.du);
  return cudaPeekAtLastError() == cudaSuccess ? WKV_OK : WKV_ERR_CUDA;
}

// Five warps (five chunks an iteration, 3 CTAs per SM at 128 registers) while every group's
// CTA fits in one wave at 3 per SM, else four (4 per SM): measured 76.6 against 79.8 us at
// 384 groups, 198.7 against 194.8 at 1024.
template <bool GATE, bool DR>
int launch_group(const BwdArgs& a, const TensorMaps4& in, const TensorMaps4& out,
                 cudaStream_t stream) {
  const bool five = g_bwd_path.load() != 3 &&
                    a.B * ((a.C + 31) / 32) <= 3 * int64_t(sm_count());
  return five ? launch_group_nw<GATE, DR, 5>(a, in, out, stream)
              : launch_group_nw<GATE, DR, 4>(a, in, out, stream);
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
  int rc;
  const bool group = TMA && use_group_path(a) && a.withhold_last_map == 0;
  if (TMA) {
    // Time-parallel checkpoints and reverse: the chain flags and the tickets start at zero.
    // Per-group path: only the counters of batch rows done per channel group, which the
    // per-group checkpoint pass clears when it runs.
    const int64_t nitems = grid * bwd_nseg(a.T);
    if (nitems >= (int64_t(1) << 31)) return WKV_ERR_UNSUPPORTED;
    if (!group) {
      if (cudaMemsetAsync(a.ws, 0, bwd_flag_bytes(a.B, a.T, a.C), stream) != cudaSuccess)
        return WKV_ERR_CUDA;
    } else if (a.have_ckpt) {
      const BwdLayout lay = bwd_layout(a.ws, a.B, a.T, a.C);
      if (cudaMemsetAsync(lay.fflags, 0, size_t((a.C + 31) / 32) * sizeof(unsigned), stream) !=
          cudaSuccess)
        return WKV_ERR_CUDA;
    }
    if (!a.have_ckpt) {
      const int64_t nch = (a.T + kTT - 1) / kTT;
      const int64_t citems = grid * ((nch + kSW * kCK - 1) / (kSW * kCK));
      if (group) {
        const Ptr4 pre{a.k, a.v, a.k, a.v};
        wkv_bwd_ckpt_group_kernel<<<unsigned(grid), kSW * 32, 0, stream>>>(
            ck, int(a.B), int(a.T), int(a.C), a.w, state_io(a), a.ws, a.err, pre);
      } else {
        wkv_bwd_ckpt_seg_kernel<<<unsigned(citems), kSW * 32, 0, stream>>>(
            ck, int(a.B), int(a.T), int(a.C), a.w, state_io(a), a.ws, a.err, a.wait_ns);
      }
      if (cudaPeekAtLastError() != cudaSuccess) return WKV_ERR_CUDA;
    }
    if (group) {
      if (a.r)
        rc = a.dr ? launch_group<true, true>(a, in, out, stream)
                  : launch_group<true, false>(a, in, out, stream);
      else
        rc = launch_group<false, false>(a, in, out, stream);
    } else if (a.r) {
      rc = a.dr ? launch_seg<true, true>(a, in, out, nitems, stream)
                : launch_seg<true, false>(a, in, out, nitems, stream);
    } else {
      rc = launch_seg<false, false>(a, in, out, nitems, stream);
    }
  } else {
    wkv_bwd_ckpt_kernel<TMA><<<unsigned(grid), 32, 0, stream>>>(ck, a.k, a.v, int(a.B), int(a.T),
                                                                int(a.C), a.w, state_io(a), a.ws,
                                                                a.err);
    if (cudaPeekAtLastError() != cudaSuccess) return WKV_ERR_CUDA;
    if (a.r)
      rc = a.dr ? launch_main<TMA, true, true>(a, in, out, stream)
                : launch_main<TMA, true, false>(a, in, out, stream);
    else
      rc = launch_main<TMA, false, false>(a, in, out, stream);
  }
  if (rc || group) return rc;  // (the per-group reverse pass writes dw, du itself)
  wkv_bwd_reduce_kernel<<<unsigned((a.C + 31) / 32), dim3(32, kRS), 0, stream>>>(
      int(a.B), int(a.C), a.ws, int(a.T), a.dw, a.du);
  return cudaPeekAtLastError() == cudaSuccess ? WKV_OK : WKV_ERR_CUDA;
}

}  // namespace

size_t backward_workspace_bytes(int64_t B, int64_t T, int64_t C) { return bwd_bytes(B, T, C); }

void backward_checkpoint_ptrs(void* ws, int64_t B, int64_t T, int64_t C, float4** ckpt,
                              float4** ckend) {
  const BwdLayout lay = bwd_layout(ws, B, T, C);
  *ckpt = lay.ckpt;
  *ckend = lay.ckend;
}

namespace {
// No tokens: the final state is the initial one, so dL/dA0 = dL/dA_T = ga1 e^{-p1} and
// da0 = e^{p0} dL/dA0 (the same for b); dp0 = a0 da0 + b0 db0.
__global__ void wkv_bwd_no_tokens_kernel(int64_t n, const StateIO io) {
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float a0 = io.a0 ? io.a0[i] : 0.f, b0 = io.a0 ? io.b0[i] : 0.f;
  float da = 0.f, db = 0.f;
  if (io.ga1 != nullptr && io.a0 != nullptr) {
    const float f = ex2(fminf((io.p0[i] - io.p1[i]) * kLog2e, 126.f));
    da = io.ga1[i] * f;
    db = io.gb1[i] * f;
  }
  io.da0[i] = da;
  io.db0[i] = db;
  io.dp0[i] = fmaf(a0, da, b0 * db);
}
}  // namespace

int launch_backward_no_tokens(const BwdArgs& a, cudaStream_t stream) {
  const int64_t n = a.B * a.C;
  wkv_bwd_no_tokens_kernel<<<unsigned((n + 255) / 256), 256, 0, stream>>>(n, state_io(a));
  return cudaPeekAtLastError() == cudaSuccess ? WKV_OK : WKV_ERR_CUDA;
}

bool backward_time_parallel_ok(const BwdArgs& a) {
  auto al16 = [](const void* p) {
    return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15) == 0;
  };
  return a.C % 4 == 0 && al16(a.k) && al16(a.v) && al16(a.r) && al16(a.dy) && al16(a.dk) &&
         al16(a.dv) && al16(a.dr);
}

void set_backward_path(int path) { g_bwd_path.store(path); }

int launch_backward(const BwdArgs& a, bool force_plain, cudaStream_t stream) {
  const bool tma = !force_plain && backward_time_parallel_ok(a);
  if (a.have_ckpt && !tma) return WKV_ERR_UNSUPPORTED;
  return tma ? launch_all<true>(a, stream) : launch_all<false>(a, stream);
}

}  // namespace wkv
