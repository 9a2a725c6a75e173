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
// warp w owns sub-chunk w (LS tokens). Single pass, 16 bytes of HBM traffic per element:
//   1. every warp TMA-loads its k, v, r sub-tile into shared memory (kept resident) and
//      folds k, v into the sub-chunk aggregate from the empty state;
//   2. warp 0 combines the W aggregates, publishes the segment aggregate, walks back over
//      the predecessors' published aggregates / inclusive prefixes (decoupled look-back;
//      CTAs take segments in ticket order, so every predecessor is already resident or
//      done) and publishes the inclusive prefix; each warp then forms its own carry-in;
//   3. every warp re-runs its sub-chunk from the carry-in out of shared memory, writes y
//      in place of k and TMA-stores it. The warp holding the last token writes the final
//      state.
// Every wait is bounded in wall time; a wait that gives up flags the error word and
// carries on with an empty carry (the result is then wrong, but the kernel ends).
#include "wkv_internal.h"
#include "wkv_step.cuh"

namespace wkv {

namespace {

// Segment shape (the macros exist for sweeps): kW warps per CTA, each owning a sub-chunk
// of kLS tokens; and the channel count below which the time-parallel path is used. The
// streaming kernel runs each channel's tokens at its per-warp latency (about 30 ns a token
// on B200), this kernel at about 4.5 ps an element over the whole GPU: below ~8192
// channels (256 warps, 1.7 per SM) the time-parallel path is faster (measured: 16 x 1024 x
// 768 streams in 37 us against 80 us chunked; 1 x 32768 x 4096 chunked in 0.60 ms against
// 0.94 ms streaming).
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
constexpr int kSeg = kW * kLS;
constexpr int64_t kChunkBelowChannels = WKV_SCAN_MIN_CH;

struct ScanLayout {
  unsigned* ticket;
  unsigned* flags;  // [nbg * nseg]: 0 none, 1 aggregate, 2 inclusive prefix
  float4* agg;      // [nbg * nseg * 32]
  float4* incl;     // [nbg * nseg * 32]
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
  float4* scarry = sagg + kW * 32;                                         // [32]
  uint64_t* bars = reinterpret_cast<uint64_t*>(scarry + 32);                // [W]
  __shared__ unsigned s_ticket;

  const int G = (C + 31) >> 5;
  const int64_t nbg = int64_t(B) * G;
  const ScanLayout lay = scan_layout(scratch, nbg * nseg);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) s_ticket = atomicAdd(lay.ticket, 1u);
  __syncthreads();
  const int64_t ticket = s_ticket;
  const int seg = int(ticket / nbg);
  const int64_t bg = ticket - int64_t(seg) * nbg;
  const int b = int(bg / G);
  const int g = int(bg - int64_t(b) * G);
  const int c = (g << 5) + lane;
  const bool valid = c < C;

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

  // ---- 1. sub-chunk aggregate from the empty state ----
  const int rb = window_tokens(cp.w2, 128.f);
  if (n > 0) mbar_wait(bar, 0, err);
  ChanState s = empty_state();
  {
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

  // ---- 2. segment aggregate, look-back, carries ----
  if (warp == 0) {
    auto ld = [&](const float4& q) { return Agg{q.x, q.y, q.z, q.w}; };
    Agg A = ld(sagg[lane]);
    for (int i = 1; i < kW; ++i) {
      const int ni = max(0, min(kLS, T - (seg * kSeg + i * kLS)));
      A = combine(A, ld(sagg[i * 32 + lane]), float(ni), cp.w2);
    }
    const int seg_len = min(kSeg, T - seg * kSeg);
    const int64_t item = bg * nseg + seg;
    Agg carry;
    if (seg == 0) {
      const size_t sidx = size_t(b) * C + c;
      carry = (a0 != nullptr && valid) ? to_agg(load_state(a0[sidx], b0[sidx], p0[sidx]))
                                       : agg_empty();
    } else {
      lay.agg[item * 32 + lane] = make_float4(A.a, A.b, A.ph, A.pl);
      warp_publish(&lay.flags[item], 1u);
      // Walk back: acc covers the segments between j and seg (exclusive), all full.
      Agg acc = agg_empty();
      int covered = 0;
      carry = agg_empty();
      for (int j = seg - 1; j >= 0; --j) {
        const int64_t pj = bg * nseg + j;
        unsigned f = 0;
        if (lane == 0) {
          f = ld_acquire(&lay.flags[pj]);
          if (f == 0) {
            const uint64_t start = global_ns();
            while ((f = ld_acquire(&lay.flags[pj])) == 0) {
              if (global_ns() - start > wait_ns) break;
              __nanosleep(64);
            }
            if (f == 0) atomicOr(err, kErrTimeout);
          }
        }
        f = __shfl_sync(0xffffffffu, f, 0);
        __syncwarp();
        if (f == 0) {  // gave up: continue from an empty carry
          carry = acc;
          break;
        }
        // L2 loads (.cg): the line may sit stale in this SM's L1 from an earlier read.
        const float4 q = (f == 2) ? __ldcg(&lay.incl[pj * 32 + lane]) : __ldcg(&lay.agg[pj * 32 + lane]);
        acc = combine(ld(q), acc, float(covered), cp.w2);
        covered += kSeg;
        if (f == 2) {
          carry = acc;
          break;
        }
        if (j == 0) carry = acc;  // unreachable: segment 0 publishes only inclusive
      }
    }
    const Agg incl = combine(carry, A, float(seg_len), cp.w2);
    if (!(withhold_seg0 && seg == 0)) {
      lay.incl[item * 32 + lane] = make_float4(incl.a, incl.b, incl.ph, incl.pl);
      warp_publish(&lay.flags[item], 2u);
    }
    scarry[lane] = make_float4(carry.a, carry.b, carry.ph, carry.pl);
  }
  __syncthreads();

  // ---- 3. re-run the sub-chunk from its carry-in, write y ----
  {
    auto ld = [&](const float4& q) { return Agg{q.x, q.y, q.z, q.w}; };
    Agg cin = ld(scarry[lane]);
    for (int i = 0; i < warp; ++i) cin = combine(cin, ld(sagg[i * 32 + lane]), float(kLS), cp.w2);
    s = to_state(cin);
  }
  if (n > 0) {
    const bool fast = __all_sync(0xffffffffu, fabsf(cp.uw2) <= kFastOutBound);
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
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_3d(&tm_y, sk + warp * kTile, g << 5, t0, b);
      tma_store_commit();
      tma_store_wait_all();
    }
    if (a1 != nullptr && valid && t0 + n == T) {
      const size_t sidx = size_t(b) * C + c;
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
  return size_t(gate ? 3 : 2) * kW * kLS * 32 * sizeof(float) + (kW * 32 + 32) * sizeof(float4) +
         kW * sizeof(uint64_t);
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
