// WKV forward over full sequences, one thread per (b, c) channel (sm_100a).
//
// Streaming kernel: a CTA of NW warps owns 32*NW adjacent channels of one batch row and
// walks the whole sequence; each thread carries one channel's state (a, b, P) in registers.
// Tiles of [TT tokens x 32*NW channels] of k, v, r are brought into shared memory by TMA
// (3-D tensor maps over (C, T, B), so ragged T and C edges are zero-filled on load and
// clipped on store), S stages deep, each stage on its own mbarrier; y is staged in shared
// memory and written back by TMA store. A CTA is one warp by default: with two warps the
// bf16 boxes get 128-byte rows, which a compute-free probe of this access pattern streams
// about 15% faster on B200, but the kernel as a whole measured no faster (it is bound by
// per-warp issue of the recurrence, not by DRAM efficiency), and one-warp CTAs balance
// better over 148 SMs (1024 CTAs at the 8 x 4096 x 4096 shape: 6.9 per SM).
//
// A plain kernel (direct coalesced global loads, same arithmetic) serves shapes the TMA
// path cannot describe: C not a multiple of 4 (fp32) / 8 (bf16), or base pointers that
// are not 16-byte aligned.
#include <cuda.h>

#include "wkv_internal.h"
#include "wkv_step.cuh"
#include "wkv_window.cuh"

namespace wkv {

// A full tile of TT tokens for the checkpointing forward: windows of RB tokens, and before
// each chunk of 16 the state entering it stored at ck[h * stride] (explicitly global, so
// the store does not order the shared-memory traffic around it).
template <typename Tin, bool GATE, bool FASTOUT, int TT, int RS, int RB>
__device__ __forceinline__ void ckpt_tile(ChanState& s, const ChanParams& cp, const Tin* K,
                                          const Tin* V, const Tin* R, Tin* Y, float4* ck,
                                          size_t stride, bool valid) {
#pragma unroll
  for (int h = 0; h < TT / 16; ++h) {
    if (valid) __stcg(ck + h * stride, make_float4(s.a, s.b, s.Q, s.pl));
#pragma unroll
    for (int w0 = h * 16; w0 < h * 16 + 16; w0 += RB)
      window_smem<Tin, GATE, FASTOUT, RB, RS>(s, cp, K + w0 * RS, V + w0 * RS, R + w0 * RS,
                                              Y + w0 * RS);
  }
}

template <typename Tin, bool GATE, bool FASTOUT, int TT, int RS>
__device__ __forceinline__ void ckpt_tile_rb(ChanState& s, const ChanParams& cp, const Tin* K,
                                             const Tin* V, const Tin* R, Tin* Y, int rb,
                                             float4* ck, size_t stride, bool valid) {
  if (rb == 16)
    ckpt_tile<Tin, GATE, FASTOUT, TT, RS, 16>(s, cp, K, V, R, Y, ck, stride, valid);
  else if (rb == 4)
    ckpt_tile<Tin, GATE, FASTOUT, TT, RS, 4>(s, cp, K, V, R, Y, ck, stride, valid);
  else
    ckpt_tile<Tin, GATE, FASTOUT, TT, RS, 1>(s, cp, K, V, R, Y, ck, stride, valid);
}

__device__ __forceinline__ void cta_sync(int nw) {
  if (nw == 1)
    __syncwarp();
  else
    __syncthreads();
}

// Launch bounds: with no minimum, ptxas sizes registers for the 32-CTA residency limit
// (32 registers at NW = 2), which serialises the windows; residency is bounded by shared
// memory to a few CTAs per SM anyway, so ask for 4.
// CKPT (fp32 training forward): also write the state entering every chunk of 16 tokens to
// ckpt ([B, ceil(T/16), C] float4 (a, b, Q, pl)) and the state after the last token to
// ckend ([B, C]): the checkpoints of the backward's reverse pass, which recomputes each chunk
// from them in these same operations. The chunks are processed as separate pieces of 16
// tokens, which changes nothing: windows never cross a multiple of 16.
template <typename Tin, bool GATE, int TT, int S, int NW, bool CKPT = false>
__global__ void __launch_bounds__(NW * 32, 4) wkv_fwd_tma_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
    const __grid_constant__ CUtensorMap tm_r, const __grid_constant__ CUtensorMap tm_y, int T,
    int C, const float* __restrict__ w, const float* __restrict__ u, const float* a0,
    const float* b0, const float* p0, float* a1, float* b1, float* p1, unsigned* err,
    float4* ckpt, float4* ckend) {
  // Full tiles are processed in whole windows of up to 16 tokens.
  static_assert(TT % 16 == 0, "tile length must be a multiple of the longest window");
  static_assert(S >= 2, "the y staging wait below assumes two or more stages");
  constexpr int CW = NW * 32;  // channels per CTA = elements per tile row
  constexpr int kTile = TT * CW;
  constexpr uint32_t kTileBytes = kTile * sizeof(Tin);
  constexpr uint32_t kStageBytes = (GATE ? 3u : 2u) * kTileBytes;

  extern __shared__ __align__(128) unsigned char smem_raw[];
  Tin* sk = reinterpret_cast<Tin*>(smem_raw);
  Tin* sv = sk + S * kTile;
  Tin* sr = sv + S * kTile;                      // unused without the gate
  Tin* sy = sr + (GATE ? S * kTile : 0);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sy + S * kTile);

  const int tid = threadIdx.x;
  const int G = (C + CW - 1) / CW;
  const int b = blockIdx.x / G;
  const int g = blockIdx.x - b * G;
  const int c = g * CW + tid;
  const bool valid = c < C;
  const int ntiles = (T + TT - 1) / TT;

  auto issue = [&](int stage, int tile) {
    uint64_t* bar = &bars[stage];
    mbar_arrive_expect_tx(bar, kStageBytes);
    tma_load_3d(sk + stage * kTile, &tm_k, bar, g * CW, tile * TT, b);
    tma_load_3d(sv + stage * kTile, &tm_v, bar, g * CW, tile * TT, b);
    if (GATE) tma_load_3d(sr + stage * kTile, &tm_r, bar, g * CW, tile * TT, b);
  };

  if (tid == 0) {
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    if (GATE) prefetch_tmap(&tm_r);
    prefetch_tmap(&tm_y);
#pragma unroll
    for (int st = 0; st < S; ++st) mbar_init(&bars[st], 1);
    mbar_fence_init();
    for (int st = 0; st < S && st < ntiles; ++st) issue(st, st);
  }
  cta_sync(NW);

  const ChanParams cp = chan_params(valid ? w[c] : 1.f, valid ? u[c] : 0.f);
  const size_t sidx = size_t(b) * C + c;
  const bool has_state = a0 != nullptr;
  ChanState s = (has_state && valid) ? load_state(a0[sidx], b0[sidx], p0[sidx]) : empty_state();
  // Per-warp choices (window length, output form): warps of a CTA may differ.
  const bool fast = __all_sync(0xffffffffu, fabsf(cp.uw2) <= kFastOutBound);
  const int rb = window_tokens(cp.w2, window_limit<Tin>());

  for (int i = 0; i < ntiles; ++i) {
    const int st = i % S;
    mbar_wait(&bars[st], (i / S) & 1, err);
    const Tin* K = sk + st * kTile + tid;
    const Tin* V = sv + st * kTile + tid;
    const Tin* R = sr + st * kTile + tid;
    Tin* Y = sy + st * kTile + tid;
    const int n = min(TT, T - i * TT);
    if (CKPT && n == TT) {
      float4* ck = ckpt + (size_t(b) * ((T + 15) / 16) + size_t(i) * (TT / 16)) * C + c;
      if (fast)
        ckpt_tile_rb<Tin, GATE, true, TT, CW>(s, cp, K, V, R, Y, rb, ck, size_t(C), valid);
      else
        ckpt_tile_rb<Tin, GATE, false, TT, CW>(s, cp, K, V, R, Y, rb, ck, size_t(C), valid);
    } else if (CKPT) {  // the last, partial tile: chunk by chunk
      const int nch = (T + 15) / 16;
#pragma unroll
      for (int h = 0; h < TT / 16; ++h) {
        if (h * 16 < n) {
          if (valid)
            ckpt[(size_t(b) * nch + size_t(i) * (TT / 16) + h) * C + c] =
                make_float4(s.a, s.b, s.Q, s.pl);
          const int o = h * 16 * CW;
          const int nq = min(16, n - h * 16);
          if (nq == 16) {
            if (fast)
              full_tile<Tin, GATE, true, 16, CW>(s, cp, K + o, V + o, R + o, Y + o, rb);
            else
              full_tile<Tin, GATE, false, 16, CW>(s, cp, K + o, V + o, R + o, Y + o, rb);
          } else if (fast) {
            tile_tokens<Tin, GATE, true, 16, 1, CW, false>(s, cp, K + o, V + o, R + o, Y + o,
                                                          nq, rb);
          } else {
            tile_tokens<Tin, GATE, false, 16, 1, CW, false>(s, cp, K + o, V + o, R + o, Y + o,
                                                           nq, rb);
          }
        }
      }
    } else if (n == TT) {
      if (fast)
        full_tile<Tin, GATE, true, TT, CW>(s, cp, K, V, R, Y, rb);
      else
        full_tile<Tin, GATE, false, TT, CW>(s, cp, K, V, R, Y, rb);
    } else {
      if (fast)
        tile_tokens<Tin, GATE, true, TT, 1, CW, false>(s, cp, K, V, R, Y, n, rb);
      else
        tile_tokens<Tin, GATE, false, TT, 1, CW, false>(s, cp, K, V, R, Y, n, rb);
    }
    // The y stage written next (tile i+1) was last stored as group i+1-S: let at most S-2
    // of the groups committed so far (through i-1) still be reading shared memory.
    if (tid == 0) tma_store_wait_read<S - 2>();
    fence_proxy_async_smem();
    cta_sync(NW);  // all of tile i read and all of its y written
    if (tid == 0) {
      tma_store_3d(&tm_y, sy + st * kTile, g * CW, i * TT, b);
      tma_store_commit();
      if (i + S < ntiles) issue(st, i + S);
    }
  }
  if (tid == 0) tma_store_wait_all();
  if (CKPT && valid) ckend[sidx] = make_float4(s.a, s.b, s.Q, s.pl);

  if (a1 != nullptr && valid) {
    a1[sidx] = s.a;
    b1[sidx] = s.b;
    p1[sidx] = (T == 0 && has_state) ? p0[sidx] : state_log_scale(s);
  }
}

// Plain kernel: one thread per (b, c), coalesced across threads, no shared memory.
template <typename Tin, bool GATE>
__global__ void __launch_bounds__(128) wkv_fwd_plain_kernel(
    int64_t B, int64_t T, int64_t C, const float* __restrict__ w, const float* __restrict__ u,
    const Tin* __restrict__ k, const Tin* __restrict__ v, const Tin* __restrict__ r,
    Tin* __restrict__ y, const float* a0, const float* b0, const float* p0, float* a1, float* b1,
    float* p1) {
  const int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const bool valid = idx < B * C;
  const int64_t bb = valid ? idx / C : 0;
  const int64_t c = valid ? idx - bb * C : 0;
  const ChanParams cp = chan_params(valid ? w[c] : 1.f, valid ? u[c] : 0.f);
  const bool has_state = a0 != nullptr;
  ChanState s = (has_state && valid) ? load_state(a0[idx], b0[idx], p0[idx]) : empty_state();
  const bool fast = __all_sync(0xffffffffu, fabsf(cp.uw2) <= kFastOutBound);
  const int rb = window_tokens(cp.w2, window_limit<Tin>());
  if (!valid) return;
  const int64_t base = bb * T * C + c;
  int j = 0;
  for (int64_t t = 0; t < T; ++t) {
    const int64_t e = base + t * C;
    const float kk = Elem<Tin>::to_f(k[e]);
    const float vv = Elem<Tin>::to_f(v[e]);
    const float rr = GATE ? Elem<Tin>::to_f(r[e]) : 0.f;
    const float out = fast ? wkv_token<GATE, true>(s, cp, float(j + 1), kk, vv, rr)
                           : wkv_token<GATE, false>(s, cp, float(j + 1), kk, vv, rr);
    y[e] = Elem<Tin>::from_f(out);
    if (++j == rb) {
      wkv_rebase(s, float(rb) * cp.w2);
      j = 0;
    }
  }
  if (j) wkv_rebase_partial(s, j, cp.w2);
  if (a1 != nullptr) {
    a1[idx] = s.a;
    b1[idx] = s.b;
    p1[idx] = (T == 0 && has_state) ? p0[idx] : state_log_scale(s);
  }
}

// ---------------------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------------------
namespace {

// Tile shape of the streaming kernel per element type: TT tokens per tile, S stages,
// NW warps per CTA (32*NW channels, TMA box rows of 32*NW elements). The defaults come
// from sweeps on B200; the macros exist for such sweeps.
#ifndef WKV_FWD_TT_BF16
#define WKV_FWD_TT_BF16 32
#endif
#ifndef WKV_FWD_S_BF16
#define WKV_FWD_S_BF16 3
#endif
#ifndef WKV_FWD_NW_BF16
#define WKV_FWD_NW_BF16 1
#endif
#ifndef WKV_FWD_TT_F32
#define WKV_FWD_TT_F32 32
#endif
#ifndef WKV_FWD_S_F32
#define WKV_FWD_S_F32 3
#endif
#ifndef WKV_FWD_NW_F32
#define WKV_FWD_NW_F32 1
#endif

template <typename Tin> struct FwdCfg;
template <> struct FwdCfg<__nv_bfloat16> {
  static constexpr int TT = WKV_FWD_TT_BF16, S = WKV_FWD_S_BF16, NW = WKV_FWD_NW_BF16;
};
template <> struct FwdCfg<float> {
  static constexpr int TT = WKV_FWD_TT_F32, S = WKV_FWD_S_F32, NW = WKV_FWD_NW_F32;
};

template <typename Tin, bool GATE>
size_t tma_smem_bytes() {
  using F = FwdCfg<Tin>;
  return size_t(F::S) * ((GATE ? 3 : 2) + 1) * F::TT * F::NW * 32 * sizeof(Tin) +
         F::S * sizeof(uint64_t);
}

template <typename Tin, bool GATE, bool CKPT = false>
int launch_tma(const FwdArgs& a, cudaStream_t stream, float4* ckpt = nullptr,
               float4* ckend = nullptr) {
  using F = FwdCfg<Tin>;
  constexpr int CW = F::NW * 32;
  CUtensorMap tk, tv, tr, ty;
  const CUtensorMapDataType dt =
      sizeof(Tin) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  int rc = encode_btc_map(&tk, a.k, dt, sizeof(Tin), a.B, a.T, a.C, CW, F::TT);
  if (!rc) rc = encode_btc_map(&tv, a.v, dt, sizeof(Tin), a.B, a.T, a.C, CW, F::TT);
  if (!rc) rc = encode_btc_map(&tr, GATE ? a.r : a.k, dt, sizeof(Tin), a.B, a.T, a.C, CW, F::TT);
  if (!rc) rc = encode_btc_map(&ty, a.y, dt, sizeof(Tin), a.B, a.T, a.C, CW, F::TT);
  if (rc) return rc;
  auto kern = wkv_fwd_tma_kernel<Tin, GATE, F::TT, F::S, F::NW, CKPT>;
  const size_t smem = tma_smem_bytes<Tin, GATE>();
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
      cudaSuccess)
    return WKV_ERR_CUDA;
  const int64_t G = (a.C + CW - 1) / CW;
  const int64_t grid = a.B * G;
  kern<<<unsigned(grid), CW, smem, stream>>>(tk, tv, tr, ty, int(a.T), int(a.C), a.w, a.u, a.a0,
                                             a.b0, a.p0, a.a1, a.b1, a.p1, a.err, ckpt, ckend);
  return cudaPeekAtLastError() == cudaSuccess ? WKV_OK : WKV_ERR_CUDA;
}

template <typename Tin, bool GATE>
int launch_plain(const FwdArgs& a, cudaStream_t stream) {
  const int64_t n = a.B * a.C;
  const int block = 128;
  const int64_t grid = (n + block - 1) / block;
  wkv_fwd_plain_kernel<Tin, GATE><<<unsigned(grid), block, 0, stream>>>(
      a.B, a.T, a.C, a.w, a.u, static_cast<const Tin*>(a.k), static_cast<const Tin*>(a.v),
      static_cast<const Tin*>(a.r), static_cast<Tin*>(a.y), a.a0, a.b0, a.p0, a.a1, a.b1, a.p1);
  return cudaPeekAtLastError() == cudaSuccess ? WKV_OK : WKV_ERR_CUDA;
}

template <typename Tin>
int dispatch(const FwdArgs& a, bool use_tma, cudaStream_t stream) {
  const bool gate = a.r != nullptr;
  if (use_tma) return gate ? launch_tma<Tin, true>(a, stream) : launch_tma<Tin, false>(a, stream);
  return gate ? launch_plain<Tin, true>(a, stream) : launch_plain<Tin, false>(a, stream);
}

}  // namespace

bool fwd_tma_ok(const FwdArgs& a, int elem_bytes) {
  auto al16 = [](const void* p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  return (a.C * elem_bytes) % 16 == 0 && al16(a.k) && al16(a.v) && al16(a.r) && al16(a.y) &&
         a.T < (int64_t(1) << 31) && a.C < (int64_t(1) << 31) && a.B < (int64_t(1) << 31) &&
         a.B * ((a.C + 31) / 32) < (int64_t(1) << 31);
}

int launch_fwd_ckpt(const FwdArgs& a, void* ws, cudaStream_t stream) {
  static_assert(FwdCfg<float>::NW == 1, "checkpoints are made per warp of 32 channels");
  if (!fwd_tma_ok(a, 4)) return WKV_ERR_UNSUPPORTED;
  float4 *ckpt = nullptr, *ckend = nullptr;
  backward_checkpoint_ptrs(ws, a.B, a.T, a.C, &ckpt, &ckend);
  return a.r != nullptr ? launch_tma<float, true, true>(a, stream, ckpt, ckend)
                        : launch_tma<float, false, true>(a, stream, ckpt, ckend);
}

int launch_fwd_stream(const FwdArgs& a, bool bf16, bool force_plain, cudaStream_t stream) {
  const bool tma = !force_plain && fwd_tma_ok(a, bf16 ? 2 : 4);
  return bf16 ? dispatch<__nv_bfloat16>(a, tma, stream) : dispatch<float>(a, tma, stream);
}

}  // namespace wkv
