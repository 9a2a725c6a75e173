// Window-at-a-time forms of the per-channel recurrence of wkv_step.cuh over tiles in
// shared memory, shared by the streaming forward (wkv_fwd.cu) and the chunked forward
// (wkv_scan.cu): one thread per channel, tokens in rows of RS elements.
#pragma once

#include "wkv_step.cuh"

namespace wkv {

// One full window of RB tokens from shared memory (row stride RS elements, this thread's
// column), written in phases so that the only serial chains are the ones the recurrence
// has (a running max for the scale, one fma per token for a and b): every load of the
// window first, then the log-weights and their running max, then the per-token
// arithmetic, then every store. (Token by token, each token's loads would wait for the
// previous token's store, which the compiler must assume may alias them.) Every token in
// scalar instructions; see window_smem for the form that is used.
template <typename Tin, bool GATE, bool FASTOUT, int RB, int RS>
__device__ __forceinline__ void window_scalar(ChanState& s, const ChanParams& cp, const Tin* K,
                                              const Tin* V, const Tin* R, Tin* Y) {
  float kk[RB], vv[RB], m[RB], d[RB], den[RB], num[RB];
  float rr[GATE ? RB : 1];
#pragma unroll
  for (int j = 0; j < RB; ++j) {
    kk[j] = Elem<Tin>::to_f(K[j * RS]);
    vv[j] = Elem<Tin>::to_f(V[j * RS]);
    if (GATE) rr[j] = Elem<Tin>::to_f(R[j * RS]);
  }
#pragma unroll
  for (int j = 0; j < RB; ++j) m[j] = fmaf(float(j + 1), cp.w2, fmaf(kk[j], kLog2e, -s.pl));
  float Q = s.Q;
#pragma unroll
  for (int j = 0; j < RB; ++j) {
    d[j] = m[j] - Q;
    Q = fmaxf(Q, m[j]);
  }
  s.Q = Q;
  if (FASTOUT) {
    // Exponentials of the window first (they depend on the scale chain only), then the
    // fma chains of a and b, then the reciprocals: the MUFU pipe is never waiting on the
    // chains, and the chains never wait on a MUFU result issued late.
    float e[RB];
#pragma unroll
    for (int j = 0; j < RB; ++j) e[j] = ex2(-fabsf(d[j]));
    float er[GATE ? RB : 1];
    if (GATE) {
#pragma unroll
      for (int j = 0; j < RB; ++j) er[j] = ex2(rr[j] * -kLog2e);
    }
    float a = s.a, b = s.b;
#pragma unroll
    for (int j = 0; j < RB; ++j) {
      const bool c = d[j] > 0.f;
      const float e1 = c ? e[j] : 1.f;
      const float e2 = c ? 1.f : e[j];
      const float he = cp.H * e2;
      num[j] = fmaf(e1, a, he * vv[j]);
      den[j] = fmaf(e1, b, he);
      if (GATE) den[j] = fmaf(den[j], er[j], den[j]);
      a = fmaf(e1, a, e2 * vv[j]);
      b = fmaf(e1, b, e2);
    }
    s.a = a;
    s.b = b;
  } else {
#pragma unroll
    for (int j = 0; j < RB; ++j) {
      // generic output form, token by token; the returned value is num/den, folded below
      const float y = wkv_token_d<GATE, false>(s, cp, d[j], vv[j], GATE ? rr[j] : 0.f);
      num[j] = y;
      den[j] = 1.f;
    }
  }
#pragma unroll
  for (int j = 0; j < RB; ++j)
    Y[j * RS] = Elem<Tin>::from_f(FASTOUT ? num[j] * rcp(den[j]) : num[j]);
  wkv_rebase(s, float(RB) * cp.w2);
}

// Tokens 2i and 2i+1 of the window share an fp32x2 register pair for every quantity that is
// not on a serial chain: log-weights, their differences from the running maximum, the
// selected factors, products with v and H, numerator, denominator, output. The chains
// themselves (running maximum Q, a, b) stay scalar, token by token, and the value of a (b)
// before each token lands in its half of a pair for the output's fma. Each packed
// instruction rounds its lanes as the scalar form would, so the results are those of the
// scalar code bit for bit.
template <typename Tin, bool GATE, int RB, int RS>
__device__ __forceinline__ void window_fast_pairs(ChanState& s, const ChanParams& cp,
                                                  const Tin* K, const Tin* V, const Tin* R,
                                                  Tin* Y) {
  static_assert(RB % 2 == 0, "token pairs");
  constexpr int NP = RB / 2;
  float2 kk[NP], vv[NP], rr[GATE ? NP : 1];
#pragma unroll
  for (int i = 0; i < NP; ++i) {
    kk[i] = make_float2(Elem<Tin>::to_f(K[2 * i * RS]), Elem<Tin>::to_f(K[(2 * i + 1) * RS]));
    vv[i] = make_float2(Elem<Tin>::to_f(V[2 * i * RS]), Elem<Tin>::to_f(V[(2 * i + 1) * RS]));
    if (GATE)
      rr[i] = make_float2(Elem<Tin>::to_f(R[2 * i * RS]), Elem<Tin>::to_f(R[(2 * i + 1) * RS]));
  }
  const float2 l2e = make_float2(kLog2e, kLog2e);
  const float2 w2 = make_float2(cp.w2, cp.w2);
  const float2 npl = make_float2(-s.pl, -s.pl);
  float2 m[NP], d[NP];
#pragma unroll
  for (int i = 0; i < NP; ++i)
    m[i] = __ffma2_rn(make_float2(float(2 * i + 1), float(2 * i + 2)), w2,
                      __ffma2_rn(kk[i], l2e, npl));
  float Q = s.Q;
#pragma unroll
  for (int i = 0; i < NP; ++i) {
    float2 qp;  // the running maximum before each token of the pair
    qp.x = Q;
    Q = fmaxf(Q, m[i].x);
    qp.y = Q;
    Q = fmaxf(Q, m[i].y);
    d[i] = __ffma2_rn(qp, make_float2(-1.f, -1.f), m[i]);  // m - Q, one rounding
  }
  s.Q = Q;
  float2 e1[NP], e2[NP];
#pragma unroll
  for (int i = 0; i < NP; ++i) {
    const float ex = ex2(-fabsf(d[i].x)), ey = ex2(-fabsf(d[i].y));
    const bool cx = d[i].x > 0.f, cy = d[i].y > 0.f;
    e1[i] = make_float2(cx ? ex : 1.f, cy ? ey : 1.f);
    e2[i] = make_float2(cx ? 1.f : ex, cy ? 1.f : ey);
  }
  float2 er[GATE ? NP : 1];
  if (GATE) {
    const float2 nl2e = make_float2(-kLog2e, -kLog2e);
#pragma unroll
    for (int i = 0; i < NP; ++i) {
      const float2 x = __fmul2_rn(rr[i], nl2e);
      er[i] = make_float2(ex2(x.x), ex2(x.y));
    }
  }
  const float2 H = make_float2(cp.H, cp.H);
  float a = s.a, b = s.b;
  float2 num[NP], den[NP];
#pragma unroll
  for (int i = 0; i < NP; ++i) {
    const float2 ev = __fmul2_rn(e2[i], vv[i]);
    const float2 he = __fmul2_rn(H, e2[i]);
    float2 ap, bp;  // a and b before each token of the pair
    ap.x = a;
    bp.x = b;
    a = fmaf(e1[i].x, a, ev.x);
    b = fmaf(e1[i].x, b, e2[i].x);
    ap.y = a;
    bp.y = b;
    a = fmaf(e1[i].y, a, ev.y);
    b = fmaf(e1[i].y, b, e2[i].y);
    num[i] = __ffma2_rn(e1[i], ap, __fmul2_rn(he, vv[i]));
    den[i] = __ffma2_rn(e1[i], bp, he);
    if (GATE) den[i] = __ffma2_rn(den[i], er[i], den[i]);
  }
  s.a = a;
  s.b = b;
#pragma unroll
  for (int i = 0; i < NP; ++i) {
    const float2 y = __fmul2_rn(num[i], make_float2(rcp(den[i].x), rcp(den[i].y)));
    Y[2 * i * RS] = Elem<Tin>::from_f(y.x);
    Y[(2 * i + 1) * RS] = Elem<Tin>::from_f(y.y);
  }
  wkv_rebase(s, float(RB) * cp.w2);
}

// One full window of RB tokens: in the single-exponential output form, windows of two or
// more tokens go through window_fast_pairs (the operations off the recurrence's serial
// chains packed two tokens to an fp32x2 instruction, same results); otherwise
// window_scalar.
template <typename Tin, bool GATE, bool FASTOUT, int RB, int RS>
__device__ __forceinline__ void window_smem(ChanState& s, const ChanParams& cp, const Tin* K,
                                            const Tin* V, const Tin* R, Tin* Y) {
  if constexpr (FASTOUT && RB >= 2)
    window_fast_pairs<Tin, GATE, RB, RS>(s, cp, K, V, R, Y);
  else
    window_scalar<Tin, GATE, FASTOUT, RB, RS>(s, cp, K, V, R, Y);
}

// Process n tokens of a tile in shared memory (row stride RS, this thread's column).
// FULL: n == TT, in unrolled windows of RB tokens; otherwise token by token with the
// runtime window length rb (the last, partial tile of a sequence).
template <typename Tin, bool GATE, bool FASTOUT, int TT, int RB, int RS, bool FULL>
__device__ __forceinline__ void tile_tokens(ChanState& s, const ChanParams& cp, const Tin* K,
                                            const Tin* V, const Tin* R, Tin* Y, int n, int rb) {
  if (FULL) {
#pragma unroll
    for (int w0 = 0; w0 < TT; w0 += RB)
      window_smem<Tin, GATE, FASTOUT, RB, RS>(s, cp, K + w0 * RS, V + w0 * RS, R + w0 * RS,
                                              Y + w0 * RS);
  } else {
    int j = 0;
    for (int t = 0; t < n; ++t) {
      const int row = t * RS;
      const float k = Elem<Tin>::to_f(K[row]);
      const float v = Elem<Tin>::to_f(V[row]);
      const float r = GATE ? Elem<Tin>::to_f(R[row]) : 0.f;
      Y[row] = Elem<Tin>::from_f(wkv_token<GATE, FASTOUT>(s, cp, float(j + 1), k, v, r));
      if (++j == rb) {
        wkv_rebase(s, float(rb) * cp.w2);
        j = 0;
      }
    }
    if (j) wkv_rebase_partial(s, j, cp.w2);
  }
}

template <typename Tin, bool GATE, bool FASTOUT, int TT, int RS>
__device__ __forceinline__ void full_tile(ChanState& s, const ChanParams& cp, const Tin* K,
                                          const Tin* V, const Tin* R, Tin* Y, int rb) {
  if (rb == 16)
    tile_tokens<Tin, GATE, FASTOUT, TT, 16, RS, true>(s, cp, K, V, R, Y, TT, rb);
  else if (rb == 4)
    tile_tokens<Tin, GATE, FASTOUT, TT, 4, RS, true>(s, cp, K, V, R, Y, TT, rb);
  else
    tile_tokens<Tin, GATE, FASTOUT, TT, 1, RS, true>(s, cp, K, V, R, Y, TT, rb);
}

// Largest window allowed for the output precision (see window_tokens).
template <typename Tin>
__host__ __device__ constexpr float window_limit() {
  return sizeof(Tin) == 2 ? 512.f : 128.f;
}

// State update only (chunk aggregates) over a full window of RB tokens of fp32 in shared
// memory (row stride RS, this thread's column): wkv_absorb's operations token by token,
// with the ones off the serial chains two tokens to an fp32x2 instruction (bit for bit
// the same results), then the window's rebase.
template <int RB, int RS>
__device__ __forceinline__ void window_absorb(ChanState& s, const ChanParams& cp, const float* K,
                                              const float* V) {
  if constexpr (RB == 1) {
    wkv_absorb(s, cp, 1.f, K[0], V[0]);
  } else {
    constexpr int NP = RB / 2;
    float2 kk[NP], vv[NP], m[NP], d[NP];
#pragma unroll
    for (int i = 0; i < NP; ++i) {
      kk[i] = make_float2(K[2 * i * RS], K[(2 * i + 1) * RS]);
      vv[i] = make_float2(V[2 * i * RS], V[(2 * i + 1) * RS]);
    }
    const float2 l2e = make_float2(kLog2e, kLog2e);
    const float2 w2 = make_float2(cp.w2, cp.w2);
    const float2 npl = make_float2(-s.pl, -s.pl);
#pragma unroll
    for (int i = 0; i < NP; ++i)
      m[i] = __ffma2_rn(make_float2(float(2 * i + 1), float(2 * i + 2)), w2,
                        __ffma2_rn(kk[i], l2e, npl));
    float Q = s.Q;
#pragma unroll
    for (int i = 0; i < NP; ++i) {
      float2 qp;
      qp.x = Q;
      Q = fmaxf(Q, m[i].x);
      qp.y = Q;
      Q = fmaxf(Q, m[i].y);
      d[i] = __ffma2_rn(qp, make_float2(-1.f, -1.f), m[i]);
    }
    s.Q = Q;
    float a = s.a, b = s.b;
#pragma unroll
    for (int i = 0; i < NP; ++i) {
      const float ex = ex2(-fabsf(d[i].x)), ey = ex2(-fabsf(d[i].y));
      const bool cx = d[i].x > 0.f, cy = d[i].y > 0.f;
      const float2 e1 = make_float2(cx ? ex : 1.f, cy ? ey : 1.f);
      const float2 e2 = make_float2(cx ? 1.f : ex, cy ? 1.f : ey);
      const float2 ev = __fmul2_rn(e2, vv[i]);
      a = fmaf(e1.x, a, ev.x);
      b = fmaf(e1.x, b, e2.x);
      a = fmaf(e1.y, a, ev.y);
      b = fmaf(e1.y, b, e2.y);
    }
    s.a = a;
    s.b = b;
  }
  wkv_rebase(s, float(RB) * cp.w2);
}

// A full tile of TT tokens (a multiple of 16) absorbed in windows of rb in {16, 4, 1}.
template <int TT, int RS>
__device__ __forceinline__ void absorb_full_tile(ChanState& s, const ChanParams& cp,
                                                 const float* K, const float* V, int rb) {
  if (rb == 16) {
#pragma unroll
    for (int w0 = 0; w0 < TT; w0 += 16) window_absorb<16, RS>(s, cp, K + w0 * RS, V + w0 * RS);
  } else if (rb == 4) {
#pragma unroll
    for (int w0 = 0; w0 < TT; w0 += 4) window_absorb<4, RS>(s, cp, K + w0 * RS, V + w0 * RS);
  } else {
#pragma unroll 4
    for (int w0 = 0; w0 < TT; ++w0) window_absorb<1, RS>(s, cp, K + w0 * RS, V + w0 * RS);
  }
}

}  // namespace wkv
