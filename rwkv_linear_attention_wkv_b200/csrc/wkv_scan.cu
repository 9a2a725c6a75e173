// Chunked (time-parallel) WKV forward for long sequences with few channels (sm_100a).
//
// The research report "RWKV模型深度研究报告", section 1.4.1, trains with the sequence cut
// into blocks that hand their state on, and the concept page "RWKV（Receptance Weighted Key
// Value）概念", section 3.4, computes the whole sequence with a parallel prefix scan. Because
// the decay e^{-w} does not depend on time, the state after a block is an associative
// combination of the state before it and the block's own aggregate:
//   X (+) Y over a block Y of L tokens:  scale_X' = scale_X - L w2 (log2),
//   (a, b) = (a_X 2^{scale_X' - s} + a_Y 2^{scale_Y - s}, same for b),  s = max(scale_X', scale_Y)
// (one exponential: one of the two factors is 1). Scales are kept as exact float pairs
// (hi, lo) so that a long chain of combinations does not drift.
//
// One CTA = W warps x 32 channels of one batch row, covering one segment of W x LS tokens;
// warp w owns sub-chunk w (LS tokens). CTAs take segments in ticket order, so every segment
// a CTA waits for belongs to a CTA that started earlier. Single pass, 16 bytes of HBM
// traffic per element:
//   1. every warp TMA-loads its k, v, r sub-tile into shared memory (kept resident) and
//      folds k, v into the sub-chunk aggregate from the empty state (whole sub-chunks in
//      windows, as the streaming kernel runs them);
//   2. warp 0 combines the W aggregates and publishes the segment's aggregate; the last
//      warp forms the state entering the segment in a fixed order from the published
//      aggregates of up to kFold earlier segments and the state entering the first of
//      them (so the result is bitwise reproducible, unlike a look-back that takes whichever
//      earlier result happens to be ready);
//   3. every warp combines that state with the aggregates of the sub-chunks before its own,
//      re-runs its sub-chunk from there out of shared memory, writes y in place of k and
//      TMA-stores it. The warp holding the last token writes the final state.
// Every wait is bounded in wall time; a wait that gives up flags the error word and
// carries on with an empty carry (the result is then wrong, but the kernel ends).
#include "wkv_internal.h"
#include "wkv_async.cuh"
#include "wkv_step.cuh"
#include "wkv_window.cuh"

namespace wkv {

namespace {

// Segment shape (the macros exist for sweeps): kW warps per CTA, each owning a sub-chunk
// of kLS tokens; and the channel count below which the time-parallel path is used. The
// streaming kernel runs each channel's tokens at its per-warp latency (about 29 ns a token
// on B200: one warp walks 4096 tokens in 119 us), this kernel at about 3.4 ps an element
// over the whole GPU (1 x 32768 x 4096 in 0.45 ms, against 0.94 ms streaming): the two
// cross near 29 ns / 3.4 ps = 8500 channels, so below 8192 channels (256 warps, 1.7 per
// SM) the time-parallel path is taken.
#ifndef WKV_SCAN_W
#define WKV_SCAN_W 8
#endif
#ifndef WKV_SCAN_LS
#define WKV_SCAN_LS 32
#endif
#ifndef WKV_SCAN_MIN_CH
#define WKV_SCAN_MIN_CH 8192
#endif
constexpr int kW = WKV_SCAN_W;     // warps per CTA (sub-chunks per segment)
constexpr int kLS = WKV_SCAN_LS;   // tokens per sub-chunk
constexpr int kFold = 16;          // earlier segments folded in directly (see the kernel)
constexpr int kSeg = kW * kLS;
constexpr int64_t kChunkBelowChannels = WKV_SCAN_MIN_CH;

struct ScanLayout {
  unsigned* ticket;
  unsigned* flags;  // [nbg * nseg]: 0 none, 1 aggregate, 2 entering state published
  float4* agg;      // [nbg * nseg * 32]: the segment's aggregate from the empty state
  float4* incl;     // [nbg * nseg * 32]: the state entering the segment (fold starts only)
};

__host__ __device__ inline int64_t scan_flag_bytes(int64_t nitems) {
  return (16 + nitems * 4 + 15) / 16 * 16;
}

__host__ __device__ inline ScanLayout scan_layout(void* base, int64_t nitems) {
  ScanLayout L;
  char* p = static_cast<char*>(base);
  L.ticket = reinterpret_cast<unsigned*>(p);
  L.flags = reinterpret_cast<unsigned*>(p + 16);
  char* q = p + scan_flag_bytes(nitems);
  L.agg = reinterpret_cast<float4*>(q);
  L.incl = reinterpret_cast<float4*>(q + nitems * 32 * sizeof(float4));
  return L;
}

template <bool GATE>
__global__ void __launch_bounds__(kW * 32) wkv_fwd_chunked_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
    const __grid_constant__ CUtensorMap tm_r, const __grid_constant__ CUtensorMap tm_y, int B,
    int T, int C, int nseg, const float* __restrict__ w, const float* __restrict__ u,
    const float* a0, const float* b0, const float* p0, float* a1, float* b1, float* p1,
    void* scratch, unsigned* err, unsigned long long wait_ns, int withhold_seg0) {
  constexpr int kTile = kLS * 32;
  constexpr uint32_t kTileBytes = kTile * sizeof(float);
  extern __shared__ __align__(128) unsigned char smem_raw[];
  float* sk = reinterpret_cast<float*>(smem_raw);        // [W][LS][32], y written in place
  float* sv = sk + kW * kTile;
  float* sr = sv + kW * kTile;
  float4* sagg = reinterpret_cast<float4*>(sr + (GATE ? kW * kTile : 0));  // [W][32]
  float4* sin = sagg + kW * 32;                                            // [32]
  float4* sfold = sin + 32;                                                // [kFold][32]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sfold + kFold * 32);         // [W]
  __shared__ unsigned s_ticket[3];

  const int G = (C + 31) >> 5;
  const int64_t nbg = int64_t(B) * G;
  const ScanLayout lay = scan_layout(scratch, nbg * nseg);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {  // ticket -> (segment, batch row, channel group), decoded once
    const unsigned ticket = atomicAdd(lay.ticket, 1u);  // < 2^31 (host check)
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
  const int c = (g << 5) + lane;
  const bool valid = c < C;
  const int64_t item0 = bg * nseg;
  const int64_t item = item0 + seg;
  const size_t sidx = size_t(b) * C + c;

  const int t0 = seg * kSeg + warp * kLS;           // first token of this warp
  const int n = max(0, min(kLS, T - t0));           // tokens of this warp
  uint64_t* bar = &bars[warp];
  if (lane == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
    if (n > 0) {
      mbar_arrive_expect_tx(bar, (GATE ? 3u : 2u) * kTileBytes);
      tma_load_3d(sk + warp * kTile, &tm_k, bar, g << 5, t0, b);
      tma_load_3d(sv + warp * kTile, &tm_v, bar, g << 5, t0, b);
      if (GATE) tma_load_3d(sr + warp * kTile, &tm_r, bar, g << 5, t0, b);
    }
  }
  __syncwarp();

  const ChanParams cp = chan_params(valid ? w[c] : 1.f, valid ? u[c] : 0.f);
  const float* K = sk + warp * kTile + lane;
  const float* V = sv + warp * kTile + lane;
  const float* R = sr + warp * kTile + lane;
  float* Y = sk + warp * kTile + lane;
  const int rb = window_tokens(cp.w2, 128.f);

  // The state entering the segment is formed in a fixed order (bitwise reproducible):
  // the state entering segment j0 = max(0, seg - kFold) (published by that segment; the
  // initial state for j0 = 0), then the published aggregates of segments j0 .. seg-1. Only
  // j0 > 0 waits for another segment's fold, so one link of a serial chain spans kFold
  // segments. The last warp checks the flags now (one acquire load per lane, while the
  // tiles load) and, if all are set, copies the inputs into shared memory (cp.async)
  // while the aggregates are formed; otherwise it waits for them after that.
  const int j0 = max(0, seg - kFold);
  const int mfold = seg - j0;  // aggregates to fold
  const unsigned fwant = lane < mfold ? 1u : ((lane == 31 && j0 > 0) ? 2u : 0u);
  const unsigned* fflag = lane < mfold ? &lay.flags[item0 + j0 + lane] : &lay.flags[item0 + j0];
  bool fold_early = false;
  if (warp == kW - 1) {
    const unsigned fl = fwant != 0 ? ld_acquire(fflag) : 0u;
    fold_early = __all_sync(0xffffffffu, fl >= fwant);
    __syncwarp();  // orders every lane's acquire before every lane's copies below
    if (fold_early) {
      for (int l = 0; l < mfold; ++l) cp_async_16(&sfold[l * 32 + lane], &lay.agg[(item0 + j0 + l) * 32 + lane]);
      if (j0 > 0) cp_async_16(&sin[lane], &lay.incl[(item0 + j0) * 32 + lane]);
      cp_async_commit();
    }
  }

  // ---- 1. sub-chunk aggregate from the empty state ----
  if (n > 0) mbar_wait_suspend(bar, 0, err);
  __syncwarp();
  ChanState s = empty_state();
  if (n == kLS) {
    absorb_full_tile<kLS, 32>(s, cp, K, V, rb);
  } else {
    int j = 0;
    for (int t = 0; t < n; ++t) {
      wkv_absorb(s, cp, float(j + 1), K[t * 32], V[t * 32]);
      if (++j == rb) {
        wkv_rebase(s, float(rb) * cp.w2);
        j = 0;
      }
    }
    if (j) wkv_rebase_partial(s, j, cp.w2);
  }
  const Agg mine = to_agg(s);
  sagg[warp * 32 + lane] = make_float4(mine.a, mine.b, mine.ph, mine.pl);
  __syncthreads();

  // ---- 2. the segment's aggregate; the state entering the segment ----
  if (warp == 0 && seg + 1 < nseg && !(withhold_seg0 && seg == 0)) {
    Agg A = agg_empty();
    for (int i = 0; i < kW; ++i) {
      const float4 q = sagg[i * 32 + lane];
      A = combine(A, Agg{q.x, q.y, q.z, q.w}, float(kLS), cp.w2);  // all sub-chunks full
    }
    lay.agg[item * 32 + lane] = make_float4(A.a, A.b, A.ph, A.pl);
    warp_publish(&lay.flags[item], 1u);
  }
  if (warp == kW - 1) {
    bool ok = true;
    if (fold_early) {
      cp_async_wait_all();
    } else {  // wait for the flags not yet set, then fetch (L2 loads: L1 may be stale)
      const unsigned fl = fwant != 0 ? wait_flag(fflag, fwant, wait_ns, err) : 1u;
      ok = __all_sync(0xffffffffu, fl != 0);
      __syncwarp();  // orders every lane's acquire before every lane's fetch below
      if (ok) {  // (a wait that gave up flagged the error word: continue from the empty state)
        for (int l = 0; l < mfold; ++l) sfold[l * 32 + lane] = __ldcg(&lay.agg[(item0 + j0 + l) * 32 + lane]);
        if (j0 > 0) sin[lane] = __ldcg(&lay.incl[(item0 + j0) * 32 + lane]);
      }
    }
    __syncwarp();
    Agg X = agg_empty();
    if (j0 == 0) {
      if (a0 != nullptr && valid) X = to_agg(load_state(a0[sidx], b0[sidx], p0[sidx]));
    } else if (ok) {
      const float4 q = sin[lane];
      X = Agg{q.x, q.y, q.z, q.w};
    }
    if (ok)
      for (int l = 0; l < mfold; ++l) {
        const float4 a = sfold[l * 32 + lane];
        X = combine(X, Agg{a.x, a.y, a.z, a.w}, float(kSeg), cp.w2);
      }
    __syncwarp();
    sin[lane] = make_float4(X.a, X.b, X.ph, X.pl);
  }
  __syncthreads();

  // ---- 3. each warp's carry-in; re-run the sub-chunk from it, write y ----
  Agg cin;
  {
    const float4 q = sin[lane];
    cin = Agg{q.x, q.y, q.z, q.w};
  }
  if (warp == 0 && seg > 0 && seg + kFold < nseg) {  // segment seg + kFold starts here
    lay.incl[item * 32 + lane] = make_float4(cin.a, cin.b, cin.ph, cin.pl);
    warp_publish(&lay.flags[item], 2u);
  }
  for (int i = 0; i < warp; ++i) {
    const float4 q = sagg[i * 32 + lane];
    cin = combine(cin, Agg{q.x, q.y, q.z, q.w}, float(kLS), cp.w2);
  }
  s = to_state(cin);
  if (n > 0) {
    const bool fast = __all_sync(0xffffffffu, fabsf(cp.uw2) <= kFastOutBound);
    if (n == kLS) {  // whole windows (y overwrites k only after the window has read it)
      if (fast)
        full_tile<float, GATE, true, kLS, 32>(s, cp, K, V, R, Y, rb);
      else
        full_tile<float, GATE, false, kLS, 32>(s, cp, K, V, R, Y, rb);
    } else {
      int j = 0;
      for (int t = 0; t < n; ++t) {
        const float kk = K[t * 32], vv = V[t * 32], rr = GATE ? R[t * 32] : 0.f;
        Y[t * 32] = fast ? wkv_token<GATE, true>(s, cp, float(j + 1), kk, vv, rr)
                         : wkv_token<GATE, false>(s, cp, float(j + 1), kk, vv, rr);
        if (++j == rb) {
          wkv_rebase(s, float(rb) * cp.w2);
          j = 0;
        }
      }
      if (j) wkv_rebase_partial(s, j, cp.w2);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_3d(&tm_y, sk + warp * kTile, g << 5, t0, b);
      tma_store_commit();
      tma_store_wait_read<0>();  // the tile stays until the store has read it
    }
    __syncwarp();
    if (a1 != nullptr && valid && t0 + n == T) {
      a1[sidx] = s.a;
      b1[sidx] = s.b;
      p1[sidx] = state_log_scale(s);
    }
  }
}

}  // namespace

size_t chunked_scratch_bytes(int64_t B, int64_t T, int64_t C, int64_t* flag_bytes,
                             int* n_segments) {
  const int64_t nseg = (T + kSeg - 1) / kSeg;
  if (B * C >= kChunkBelowChannels || nseg <= 1 || T >= (int64_t(1) << 31) ||
      C >= (int64_t(1) << 31) || B * ((C + 31) / 32) * nseg >= (int64_t(1) << 31)) {
    *n_segments = 1;
    *flag_bytes = 0;
    return 0;
  }
  const int64_t nitems = B * ((C + 31) / 32) * nseg;
  *n_segments = int(nseg);
  *flag_bytes = scan_flag_bytes(nitems);
  return size_t(scan_flag_bytes(nitems) + 2 * nitems * 32 * int64_t(sizeof(float4)));
}

static size_t chunked_smem_bytes(bool gate) {
  return size_t(gate ? 3 : 2) * kW * kLS * 32 * sizeof(float) +
         (kW * 32 + 32 + kFold * 32) * sizeof(float4) + kW * sizeof(uint64_t);
}

int launch_fwd_chunked_ex(const FwdArgs& a, void* scratch, int nseg, unsigned long long wait_ns,
                          int withhold_seg0, cudaStream_t stream) {
  auto al16 = [](const void* p) {
    return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15) == 0;
  };
  if (a.C % 4 != 0 || !al16(a.k) || !al16(a.v) || !al16(a.r) || !al16(a.y))
    return launch_fwd_stream(a, false, false, stream);
  CUtensorMap tk, tv, tr, ty;
  const auto dt = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  int rc = encode_btc_map(&tk, a.k, dt, 4, a.B, a.T, a.C, 32, kLS);
  if (!rc) rc = encode_btc_map(&tv, a.v, dt, 4, a.B, a.T, a.C, 32, kLS);
  if (!rc) rc = encode_btc_map(&tr, a.r ? a.r : a.k, dt, 4, a.B, a.T, a.C, 32, kLS);
  if (!rc) rc = encode_btc_map(&ty, a.y, dt, 4, a.B, a.T, a.C, 32, kLS);
  if (rc) return rc;
  const bool gate = a.r != nullptr;
  const size_t smem = chunked_smem_bytes(gate);
  auto kern = gate ? wkv_fwd_chunked_kernel<true> : wkv_fwd_chunked_kernel<false>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
      cudaSuccess)
    return WKV_ERR_CUDA;
  const int64_t grid = a.B * ((a.C + 31) / 32) * nseg;
  kern<<<unsigned(grid), kW * 32, smem, stream>>>(tk, tv, tr, ty, int(a.B), int(a.T), int(a.C),
                                                  nseg, a.w, a.u, a.a0, a.b0, a.p0, a.a1, a.b1,
                                                  a.p1, scratch, a.err, wait_ns, withhold_seg0);
  return cudaPeekAtLastError() == cudaSuccess ? WKV_OK : WKV_ERR_CUDA;
}

int launch_fwd_chunked(const FwdArgs& a, void* scratch, int nseg, cudaStream_t stream) {
  return launch_fwd_chunked_ex(a, scratch, nseg, kWaitLimitNs, 0, stream);
}

}  // namespace wkv
