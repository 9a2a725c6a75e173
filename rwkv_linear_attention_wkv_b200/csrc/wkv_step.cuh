// The per-channel WKV recurrence in log-max-stabilised, base-2 form (sm_100a).
//
// Definition (concept page "RWKV（Receptance Weighted Key Value）概念", section 3.2, and the
// paper notes "RWKV - 把 RNN 重新带回 Transformer 时代的线性大模型", "一句话总结"):
//   wkv_t = (A_{t-1} + e^{u+k_t} v_t) / (B_{t-1} + e^{u+k_t}),   y_t = sigmoid(r_t) wkv_t
//   A_t = e^{-w} A_{t-1} + e^{k_t} v_t,   B_t = e^{-w} B_{t-1} + e^{k_t}.
// The notes name a stabilising exponent p in the inference state but give no formula; the
// reading used here is A = a 2^P, B = b 2^P with P the running maximum of the (decayed)
// log2-weights, so that one of the two factors of every update is exactly 1.
//
// Representation per channel: (a, b) scaled numerator and denominator, and the log2-scale
// P_t kept as an exact pair of floats across "windows" of consecutive tokens:
//   * at the start of a window, P = Q + pl with Q, pl floats (|pl| <= ulp(Q)/2);
//   * token j = 1..n of the window has the log2-weight m_j = k_j log2(e) + j w2 - pl,
//     measured against the window start (w2 = w log2(e)); Q tracks max(Q, m_j);
//   * at the end of the window P = Q + pl - n w2 is re-split exactly (TwoSum).
// Decaying the scale by w2 once per token in float would round the same way every step
// (the low bits of w2 below ulp(P) are constant) and drift by up to ulp(P)/2 per token;
// the window form rounds each m_j once and never accumulates. The price is that m_j and Q
// grow to about n w2 within a window, and their difference d is rounded at that magnitude;
// so the window length n is chosen per warp from the largest w2 of its channels
// (window_tokens below): long windows for slowly decaying channels, where drift matters,
// short ones for fast decay, where only the last few tokens carry weight.
//
// Per token (d = m_j - Q; one of e1, e2 is 1, the other 2^{-|d|}):
//   state update   a' = e1 a + e2 v,  b' = e1 b + e2,  Q' = max(Q, m_j)
//   output         with H = 2^{u2 - w2} = e^{u-w}:
//                  wkv = (e1 a + H e2 v) / (e1 b + H e2)
// i.e. numerator and denominator of the output scaled by e^{-w} 2^{-P_t}, which is the
// scale of the updated state, so the output costs no exponential of its own. This needs
// H to be a normal float; for |u - w| beyond ~69 (nats) the generic form below takes
// over, which stabilises the output with its own exponential.
#pragma once

#include "wkv_device.cuh"

namespace wkv {

struct ChanState {
  float a, b;   // scaled numerator / denominator
  float Q, pl;  // log2-scale of the state: Q + pl (see above)
};

struct ChanParams {
  float w2;   // w log2(e)
  float uw2;  // (u - w) log2(e)
  float H;    // 2^{uw2}
};

// |u - w| log2(e) bound for the single-exponential output form.
constexpr float kFastOutBound = 100.0f;

__device__ __forceinline__ ChanParams chan_params(float w, float u) {
  ChanParams p;
  p.w2 = w * kLog2e;
  p.uw2 = fmaf(u, kLog2e, -p.w2);
  p.H = ex2(p.uw2);
  return p;
}

__device__ __forceinline__ ChanState empty_state() {
  ChanState s;
  s.a = 0.f;
  s.b = 0.f;
  s.Q = kEmptyLogScale;
  s.pl = 0.f;
  return s;
}

// State given as (a, b, p) with A = a e^p, B = b e^p (p in natural log).
__device__ __forceinline__ ChanState load_state(float a, float b, float p) {
  ChanState s;
  s.a = a;
  s.b = b;
  s.Q = p * kLog2e;
  s.pl = fmaf(p, kLog2e, -s.Q);  // exact low part of the product
  return s;
}

// Natural-log scale of the state (one rounding).
__device__ __forceinline__ float state_log_scale(const ChanState& s) {
  return fmaf(s.Q, kLn2, s.pl * kLn2);
}

// One token given d = m_j - Q (its log2-weight against the state's running scale, with
// Q already advanced by the caller): output and state update.
template <bool GATE, bool FASTOUT>
__device__ __forceinline__ float wkv_token_d(ChanState& s, const ChanParams& cp, float d, float v,
                                             float r) {
  const float e = ex2(-fabsf(d));
  const bool c = d > 0.f;
  const float e1 = c ? e : 1.f;
  const float e2 = c ? 1.f : e;
  float num, den;
  if (FASTOUT) {
    const float he = cp.H * e2;
    num = fmaf(e1, s.a, he * v);
    den = fmaf(e1, s.b, he);
  } else {
    // Output stabilised on its own: exponent of the current token against the state
    // before it is d + (u - w) log2(e).
    const float dO = d + cp.uw2;
    const float o = ex2(-fabsf(dO));
    const bool co = dO > 0.f;
    const float o1 = co ? o : 1.f;
    const float o2 = co ? 1.f : o;
    num = fmaf(o1, s.a, o2 * v);
    den = fmaf(o1, s.b, o2);
  }
  if (GATE) {
    // sigmoid(r) folded into the division: y = num / (den (1 + e^{-r})).
    const float er = ex2(r * -kLog2e);
    den = fmaf(den, er, den);
  }
  s.a = fmaf(e1, s.a, e2 * v);
  s.b = fmaf(e1, s.b, e2);
  return num * rcp(den);
}

// One token; fj = j as float (1-based position within the window).
template <bool GATE, bool FASTOUT>
__device__ __forceinline__ float wkv_token(ChanState& s, const ChanParams& cp, float fj, float k,
                                           float v, float r) {
  const float m = fmaf(fj, cp.w2, fmaf(k, kLog2e, -s.pl));
  const float d = m - s.Q;
  s.Q = fmaxf(s.Q, m);
  return wkv_token_d<GATE, FASTOUT>(s, cp, d, v, r);
}

// State update only (no output): used for chunk aggregates and recomputation.
__device__ __forceinline__ void wkv_absorb(ChanState& s, const ChanParams& cp, float fj, float k,
                                           float v) {
  const float m = fmaf(fj, cp.w2, fmaf(k, kLog2e, -s.pl));
  const float d = m - s.Q;
  const float e = ex2(-fabsf(d));
  const bool c = d > 0.f;
  const float e1 = c ? e : 1.f;
  const float e2 = c ? 1.f : e;
  s.Q = fmaxf(s.Q, m);
  s.a = fmaf(e1, s.a, e2 * v);
  s.b = fmaf(e1, s.b, e2);
}

// End of a window of n tokens: P = Q + pl - n w2, re-split exactly. For n a power of two
// n w2 is exact; the one rounding of pl - n w2 is 2^-24 of the window's decay, the same
// relative size as the rounding of w2 itself, and does not grow with the window count.
__device__ __forceinline__ void wkv_rebase(ChanState& s, float nw2) {
  const float c2 = s.pl - nw2;
  float hi, lo;
  two_sum(s.Q, c2, hi, lo);
  s.Q = hi;
  s.pl = lo;
}

// (h, l) = ph + pl - n w2 as an unevaluated pair, with the product n w2 taken exactly
// (its rounding error recovered by an fma) and the large subtraction done by TwoSum.
// For spans that are not a power of two (partial windows, carries across chunks).
__device__ __forceinline__ void decay_pair(float ph, float pl, float n, float w2, float& h,
                                           float& l) {
  const float prod = n * w2;
  const float perr = fmaf(n, w2, -prod);  // n w2 = prod + perr exactly
  float h1, l1;
  two_sum(ph, -prod, h1, l1);
  two_sum(h1, l1 + (pl - perr), h, l);
}

__device__ __forceinline__ void wkv_rebase_partial(ChanState& s, int n, float w2) {
  decay_pair(s.Q, s.pl, float(n), w2, s.Q, s.pl);
}

// Window length for a warp: the largest of 16, 4, 1 tokens for which n w2 stays within
// `limit` (log2 units) for every channel of the warp. fp32 outputs use limit 128 (m_j
// rounded at ~2^-17 absolute), bf16 outputs 512 (bf16 resolution is 2^-8 relative).
__device__ __forceinline__ int window_tokens(float w2, float limit) {
  float m = w2;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  return (16.f * m <= limit) ? 16 : ((4.f * m <= limit) ? 4 : 1);
}

// ---- span aggregates ------------------------------------------------------------------
// Because the decay e^{-w} does not depend on time, the state after two adjacent spans is an
// associative combination of the first span's state and the second span's own aggregate
// (its state from the empty state):
//   X (+) Y over a span Y of L tokens:  scale_X' = scale_X - L w2 (log2),
//   (a, b) = (a_X 2^{scale_X' - s} + a_Y 2^{scale_Y - s}, same for b),  s = max(scale_X', scale_Y)
// (one exponential: one of the two factors is 1). Scales are exact float pairs (hi, lo) so
// that a long chain of combinations does not drift.
struct Agg {  // scaled numerator, denominator, log2-scale as an exact pair
  float a, b, ph, pl;
};

__device__ __forceinline__ Agg agg_empty() { return Agg{0.f, 0.f, kEmptyLogScale, 0.f}; }

// X (+) Y where Y spans `len` tokens after X.
__device__ __forceinline__ Agg combine(const Agg& X, const Agg& Y, float len, float w2) {
  float xh, xl;
  decay_pair(X.ph, X.pl, len, w2, xh, xl);
  const float d = (xh - Y.ph) + (xl - Y.pl);
  const float f = ex2(-fabsf(d));
  Agg r;
  if (d > 0.f) {
    r.a = fmaf(f, Y.a, X.a);
    r.b = fmaf(f, Y.b, X.b);
    r.ph = xh;
    r.pl = xl;
  } else {
    r.a = fmaf(f, X.a, Y.a);
    r.b = fmaf(f, X.b, Y.b);
    r.ph = Y.ph;
    r.pl = Y.pl;
  }
  return r;
}

__device__ __forceinline__ Agg to_agg(const ChanState& s) { return Agg{s.a, s.b, s.Q, s.pl}; }
__device__ __forceinline__ ChanState to_state(const Agg& g) {
  ChanState s;
  s.a = g.a;
  s.b = g.b;
  s.Q = g.ph;
  s.pl = g.pl;
  return s;
}

}  // namespace wkv
