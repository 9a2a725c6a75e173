// The per-token scale step with a state-independent token weight, used by the backward's
// checkpoint pass and by its reverse pass when it recomputes from that pass's checkpoints
// (wkv_bwd.cu).
//
// Those checkpoints are formed by combining chunk aggregates (not by walking the tokens),
// and the reverse pass recomputes each chunk from one. Both sides must weigh every token
// identically, or a dominant token (a spike in k) would carry two different roundings of
// its weight into the two sides and the reverse sums would be inconsistent at the level of
// ulp(k log2 e). So the token's log2-weight in the window, m = k log2(e) + j w2, is rounded
// independently of the state, and the state's low part enters only the comparison
// d = (m - Q) - pl; a token that takes over the scale sets it to (m, 0). (The streaming
// forward of wkv_step.cuh folds pl into m instead and keeps Q as a running maximum: the
// same quantity, rounded differently. Checkpoints that the streaming forward writes are
// recomputed in that form.)
#pragma once

#include "wkv_step.cuh"

namespace wkv {

// m = j w2 + k log2(e). The product is rounded on its own (__fmul_rn): with fj a
// compile-time 1 the compiler could otherwise fuse it into the fma, and two kernels would
// round differently.
__device__ __forceinline__ float tok_log2w(float fj, float w2, float k) {
  return fmaf(fj, w2, __fmul_rn(k, kLog2e));
}

// The same for two tokens in one fp32x2 multiply and one fp32x2 fma (each lane rounded as
// the scalar form).
__device__ __forceinline__ float2 tok_log2w2(float2 fj, float w2, float2 k) {
  return __ffma2_rn(fj, make_float2(w2, w2), __fmul2_rn(k, make_float2(kLog2e, kLog2e)));
}

// One token's scale step: d = (m - Q) - pl against the state's scale; e = 2^{-|d|}; the
// factors (e1 on the state, e2 on the token; one of them is 1); a token with d > 0 takes
// over the scale.
struct ScaleStep {
  float d, e, e1, e2;
  bool dom;  // the token dominated (e1 = e, e2 = 1)
};

__device__ __forceinline__ ScaleStep indep_step(float m, float& Q, float& pl) {
  ScaleStep r;
  r.d = (m - Q) - pl;
  r.e = ex2(-fabsf(r.d));
  r.dom = r.d > 0.f;
  r.e1 = r.dom ? r.e : 1.f;
  r.e2 = r.dom ? 1.f : r.e;
  Q = r.dom ? m : Q;
  pl = r.dom ? 0.f : pl;
  return r;
}

// The scale's rebase at the end of a window of n tokens (wkv_rebase on (Q, pl) alone).
__device__ __forceinline__ void indep_rebase(float& Q, float& pl, float nw2) {
  ChanState r;
  r.Q = Q;
  r.pl = pl;
  wkv_rebase(r, nw2);
  Q = r.Q;
  pl = r.pl;
}

}  // namespace wkv
