// Training forward that also writes the backward's checkpoints (sm_100a).
//
// The backward (wkv_bwd.cu) recomputes each chunk of 16 tokens from the state entering it
// (a checkpoint) and otherwise spends a whole pass over k and v forming those states. A
// training step runs the forward over the same k and v just before, so this kernel writes
// the checkpoints on its way: one float4 (a, b, Q, pl) per channel every 16 tokens (1 byte
// per element) into the backward's workspace, and the state after the last token.
//
// The states must be the ones the backward's recomputation produces, bit for bit: the
// scale follows the backward's per-token step (wkv_indep.cuh: state-independent token
// weight, takeover selects, rebase at the end of every window of 16/4/1 tokens, windows
// aligned with the chunks), and a and b take the same fma's. Then the recomputation of a
// chunk from its checkpoint ends exactly on the next checkpoint. The output y is formed as
// in the streaming forward (numerator and denominator against the state before the token,
// sigma(r) folded into the division); it rounds differently from wkv_forward's, within the
// same tolerance of the exact result.
//
// Streaming structure as wkv_fwd_tma_kernel (fp32): one warp per 32 channels of a batch
// row walks the whole sequence; TMA tiles of 32 tokens (two chunks), 3 stages; y staged in
// shared memory and TMA-stored. Within a full chunk, the work off the serial chains runs
// two tokens to an fp32x2 instruction.
#include <cuda.h>

#include "wkv_indep.cuh"
#include "wkv_internal.h"

namespace wkv {

namespace {

constexpr int kCT = 16;  // tokens per checkpoint interval (the backward's chunk)
constexpr int kTTc = 32; // tokens per tile: two chunks
constexpr int kSc = 3;   // pipeline stages

// Outputs of a pair of tokens against the state before each, (ap, bp), given the tokens'
// scale steps; FASTOUT: the single-exponential form (H = e^{u-w}); otherwise the current
// token's weight against that state is stabilised on its own (d + (u - w) log2 e).
template <bool FASTOUT>
__device__ __forceinline__ void pair_output(const ScaleStep& s0, const ScaleStep& s1,
                                            const ChanParams& cp, float2 ap, float2 bp,
                                            float2 vv, float2& num, float2& den) {
  const float2 e1 = make_float2(s0.e1, s1.e1);
  const float2 e2 = make_float2(s0.e2, s1.e2);
  if (FASTOUT) {
    const float2 he = __fmul2_rn(make_float2(cp.H, cp.H), e2);
    num = __ffma2_rn(e1, ap, __fmul2_rn(he, vv));
    den = __ffma2_rn(e1, bp, he);
  } else {
    float o1[2], o2[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float dO = (h ? s1.d : s0.d) + cp.uw2;
      const float oo = ex2(-fabsf(dO));
      const bool co = dO > 0.f;
      o1[h] = co ? oo : 1.f;
      o2[h] = co ? 1.f : oo;
    }
    const float2 f1 = make_float2(o1[0], o1[1]), f2 = make_float2(o2[0], o2[1]);
    num = __ffma2_rn(f1, ap, __fmul2_rn(f2, vv));
    den = __ffma2_rn(f1, bp, f2);
  }
}

// One full chunk of kCT tokens in windows of RB (tiles in shared memory, row stride 32,
// this thread's column): y for every token, the state left after the chunk.
template <bool GATE, bool FASTOUT, int RB>
__device__ __forceinline__ void ckpt_chunk(ChanState& s, const ChanParams& cp, const float* K,
                                           const float* V, const float* R, float* Y) {
  static_assert(kCT % RB == 0, "windows must tile the chunk");
  float a = s.a, b = s.b, Q = s.Q, pl = s.pl;
#pragma unroll
  for (int t = 0; t < kCT; t += 2) {
    const float2 kk = make_float2(K[t * 32], K[(t + 1) * 32]);
    const float2 vv = make_float2(V[t * 32], V[(t + 1) * 32]);
    const float2 m =
        tok_log2w2(make_float2(float(t % RB + 1), float((t + 1) % RB + 1)), cp.w2, kk);
    float2 er = make_float2(0.f, 0.f);
    if (GATE) {
      const float2 x = __fmul2_rn(make_float2(R[t * 32], R[(t + 1) * 32]),
                                  make_float2(-kLog2e, -kLog2e));
      er = make_float2(ex2(x.x), ex2(x.y));
    }
    const ScaleStep s0 = indep_step(m.x, Q, pl);
    if ((t + 1) % RB == 0) indep_rebase(Q, pl, float(RB) * cp.w2);
    const ScaleStep s1 = indep_step(m.y, Q, pl);
    if ((t + 2) % RB == 0) indep_rebase(Q, pl, float(RB) * cp.w2);
    const float2 ev = __fmul2_rn(make_float2(s0.e2, s1.e2), vv);
    float2 ap, bp;  // a and b before each token of the pair
    ap.x = a;
    bp.x = b;
    a = fmaf(s0.e1, a, ev.x);
    b = fmaf(s0.e1, b, s0.e2);
    ap.y = a;
    bp.y = b;
    a = fmaf(s1.e1, a, ev.y);
    b = fmaf(s1.e1, b, s1.e2);
    float2 num, den;
    pair_output<FASTOUT>(s0, s1, cp, ap, bp, vv, num, den);
    if (GATE) den = __ffma2_rn(den, er, den);  // sigma(r) folded into the division
    const float2 y = __fmul2_rn(num, make_float2(rcp(den.x), rcp(den.y)));
    Y[t * 32] = y.x;
    Y[(t + 1) * 32] = y.y;
  }
  s.a = a;
  s.b = b;
  s.Q = Q;
  s.pl = pl;
}

template <bool GATE, bool FASTOUT>
__device__ __forceinline__ void ckpt_chunk_rb(ChanState& s, const ChanParams& cp, int rb,
                                              const float* K, const float* V, const float* R,
                                              float* Y) {
  if (rb == 16)
    ckpt_chunk<GATE, FASTOUT, 16>(s, cp, K, V, R, Y);
  else if (rb == 4)
    ckpt_chunk<GATE, FASTOUT, 4>(s, cp, K, V, R, Y);
  else
    ckpt_chunk<GATE, FASTOUT, 1>(s, cp, K, V, R, Y);
}

// The last, partial chunk of a sequence (n < kCT tokens), token by token; the scale is
// left at the position after the last token.
template <bool GATE, bool FASTOUT>
__device__ __forceinline__ void ckpt_tail(ChanState& s, const ChanParams& cp, int rb,
                                          const float* K, const float* V, const float* R,
                                          float* Y, int n) {
  int j = 0;
  for (int t = 0; t < n; ++t) {
    const float kk = K[t * 32], vv = V[t * 32];
    const ScaleStep st = indep_step(tok_log2w(float(j + 1), cp.w2, kk), s.Q, s.pl);
    float2 num, den;
    pair_output<FASTOUT>(st, st, cp, make_float2(s.a, s.a), make_float2(s.b, s.b),
                         make_float2(vv, vv), num, den);
    float dn = den.x;
    if (GATE) {
      const float er = ex2(R[t * 32] * -kLog2e);
      dn = fmaf(dn, er, dn);
    }
    Y[t * 32] = num.x * rcp(dn);
    s.a = fmaf(st.e1, s.a, st.e2 * vv);
    s.b = fmaf(st.e1, s.b, st.e2);
    if (++j == rb) {
      wkv_rebase(s, float(rb) * cp.w2);
      j = 0;
    }
  }
  if (j) wkv_rebase_partial(s, j, cp.w2);
}

template <bool GATE>
__global__ void __launch_bounds__(32, 4) wkv_fwd_ckpt_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
    const __grid_constant__ CUtensorMap tm_r, const __grid_constant__ CUtensorMap tm_y, int T,
    int C, const float* __restrict__ w, const float* __restrict__ u, const float* a0,
    const float* b0, const float* p0, float4* ckpt, float4* ckend, unsigned* err) {
  constexpr int kTile = kTTc * 32;
  constexpr uint32_t kStageBytes = (GATE ? 3u : 2u) * kTile * sizeof(float);
  extern __shared__ __align__(128) unsigned char smem_raw[];
  float* sk = reinterpret_cast<float*>(smem_raw);
  float* sv = sk + kSc * kTile;
  float* sr = sv + kSc * kTile;  // unused without the gate
  float* sy = sr + (GATE ? kSc * kTile : 0);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sy + kSc * kTile);

  const int tid = threadIdx.x;
  const int G = (C + 31) >> 5;
  const int b = blockIdx.x / G;
  const int g = blockIdx.x - b * G;
  const int c = (g << 5) + tid;
  const bool valid = c < C;
  const int ntiles = (T + kTTc - 1) / kTTc;
  const int nch = (T + kCT - 1) / kCT;

  auto issue = [&](int stage, int tile) {
    uint64_t* bar = &bars[stage];
    mbar_arrive_expect_tx(bar, kStageBytes);
    tma_load_3d(sk + stage * kTile, &tm_k, bar, g << 5, tile * kTTc, b);
    tma_load_3d(sv + stage * kTile, &tm_v, bar, g << 5, tile * kTTc, b);
    if (GATE) tma_load_3d(sr + stage * kTile, &tm_r, bar, g << 5, tile * kTTc, b);
  };

  if (tid == 0) {
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    if (GATE) prefetch_tmap(&tm_r);
    prefetch_tmap(&tm_y);
#pragma unroll
    for (int st = 0; st < kSc; ++st) mbar_init(&bars[st], 1);
    mbar_fence_init();
    for (int st = 0; st < kSc && st < ntiles; ++st) issue(st, st);
  }
  __syncwarp();

  const ChanParams cp = chan_params(valid ? w[c] : 1.f, valid ? u[c] : 0.f);
  const size_t sidx = size_t(b) * C + c;
  ChanState s = (a0 != nullptr && valid) ? load_state(a0[sidx], b0[sidx], p0[sidx])
                                         : empty_state();
  // The backward's per-warp choices, made the same way over the same 32 channels.
  const bool fast = __all_sync(0xffffffffu, fabsf(cp.uw2) <= kFastOutBound);
  const int rb = window_tokens(cp.w2, 128.f);
  float4* ck = ckpt + int64_t(b) * nch * C + c;  // the state entering chunk i at ck[i * C]

  for (int i = 0; i < ntiles; ++i) {
    const int st = i % kSc;
    mbar_wait(&bars[st], (i / kSc) & 1, err);
    const int n = min(kTTc, T - i * kTTc);
#pragma unroll
    for (int q = 0; q < kTTc / kCT; ++q) {
      const int t0 = q * kCT;
      if (t0 < n) {
        if (valid) ck[int64_t(i * (kTTc / kCT) + q) * C] = make_float4(s.a, s.b, s.Q, s.pl);
        const int off = st * kTile + t0 * 32 + tid;
        const float* K = sk + off;
        const float* V = sv + off;
        const float* R = sr + off;
        float* Y = sy + off;
        const int nq = min(kCT, n - t0);
        if (nq == kCT) {
          if (fast)
            ckpt_chunk_rb<GATE, true>(s, cp, rb, K, V, R, Y);
          else
            ckpt_chunk_rb<GATE, false>(s, cp, rb, K, V, R, Y);
        } else if (fast) {
          ckpt_tail<GATE, true>(s, cp, rb, K, V, R, Y, nq);
        } else {
          ckpt_tail<GATE, false>(s, cp, rb, K, V, R, Y, nq);
        }
      }
    }
    // The y stage written next (tile i+1) was last stored as group i+1-S: let at most S-2
    // of the groups committed so far (through i-1) still be reading shared memory.
    if (tid == 0) tma_store_wait_read<kSc - 2>();
    fence_proxy_async_smem();
    __syncwarp();  // all of tile i read and all of its y written
    if (tid == 0) {
      tma_store_3d(&tm_y, sy + st * kTile, g << 5, i * kTTc, b);
      tma_store_commit();
      if (i + kSc < ntiles) issue(st, i + kSc);
    }
  }
  if (tid == 0) tma_store_wait_all();
  if (valid) ckend[sidx] = make_float4(s.a, s.b, s.Q, s.pl);
}

}  // namespace

int launch_fwd_ckpt(const FwdArgs& a, void* ws, cudaStream_t stream) {
  if (!fwd_tma_ok(a, 4)) return WKV_ERR_UNSUPPORTED;
  CUtensorMap tk, tv, tr, ty;
  const auto dt = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  int rc = encode_btc_map(&tk, a.k, dt, 4, a.B, a.T, a.C, 32, kTTc);
  if (!rc) rc = encode_btc_map(&tv, a.v, dt, 4, a.B, a.T, a.C, 32, kTTc);
  if (!rc) rc = encode_btc_map(&tr, a.r ? a.r : a.k, dt, 4, a.B, a.T, a.C, 32, kTTc);
  if (!rc) rc = encode_btc_map(&ty, a.y, dt, 4, a.B, a.T, a.C, 32, kTTc);
  if (rc) return rc;
  float4 *ckpt = nullptr, *ckend = nullptr;
  backward_checkpoint_ptrs(ws, a.B, a.T, a.C, &ckpt, &ckend);
  const bool gate = a.r != nullptr;
  const size_t smem =
      size_t(kSc) * ((gate ? 3 : 2) + 1) * kTTc * 32 * sizeof(float) + kSc * sizeof(uint64_t);
  auto kern = gate ? wkv_fwd_ckpt_kernel<true> : wkv_fwd_ckpt_kernel<false>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
      cudaSuccess)
    return WKV_ERR_CUDA;
  const int64_t grid = a.B * ((a.C + 31) / 32);
  kern<<<unsigned(grid), 32, smem, stream>>>(tk, tv, tr, ty, int(a.T), int(a.C), a.w, a.u, a.a0,
                                             a.b0, a.p0, ckpt, ckend, a.err);
  return cudaPeekAtLastError() == cudaSuccess ? WKV_OK : WKV_ERR_CUDA;
}

}  // namespace wkv
