// RWKV-7 generalised-delta-rule recurrence per head (sm_100a).
//
// The research report "RWKV模型深度研究报告（截至2026年初）", section 1.3.3 "RWKV-7 (Goose)",
// gives the state update with a matrix state S per head, input-dependent decay w_t and
// in-context-learning vectors a_t, b_t:
//   S_t = S_{t-1} (diag(w_t) + a_t^T b_t) + v_t^T k_t,
// i.e. for row i (value channel) and column j (key channel)
//   S_t[i][j] = S_{t-1}[i][j] w_t[j] + sa_i b_t[j] + v_t[i] k_t[j],  sa_i = sum_l S_{t-1}[i][l] a_t[l].
// The report gives no read-out; this library reads the state with the receptance as the
// query, y_t = S_t r_t^T.
//
// One CTA per (batch row, head) of head size N = 64, 64 threads: thread t holds the 4 x 16
// block of S at rows 4 (t / 4) .., columns {8 m + 2 (t mod 4), 8 m + 2 (t mod 4) + 1 : m < 8}
// in registers, as pairs for packed fp32x2 arithmetic. A token's vectors are read from
// shared memory once per thread (conflict-free 8-byte reads, 32 contiguous bytes per
// instruction, shared by broadcast between row blocks) instead of once per row. Row sums
// (sa_i = S[i] . a and y_i = S[i] . r) reduce over the 4 threads of a row block by
// recursive halving (3 shuffles for 4 rows; 8 x 8 blocks over 8 threads took 7 for 8 rows
// and measured 5% slower), and sa is gathered back the same way. r, w, k, v, a, b ([64] fp32 each per token) come in TMA tiles of kT7 tokens through
// a kS7-stage mbarrier pipeline; y is staged in shared memory and TMA-stored a tile at a
// time. Bound: the FP32 pipe (about 5 N^2 operations per token per head).
#include "wkv_device.cuh"
#include "wkv_internal.h"

namespace wkv {

namespace {

constexpr int kN7 = 64;        // head size
constexpr int kT7 = 8;         // tokens per tile
constexpr int kS7 = 4;         // pipeline stages
constexpr int kBR = 4;         // rows of S per thread
constexpr int kBC = 16;        // columns of S per thread (kPr pairs, 2 kLB columns apart)
constexpr int kPr = kBC / 2;   // column pairs per thread
constexpr int kLB = kN7 / kBC; // lanes of a row block (threads sharing its rows)
constexpr int kThr7 = (kN7 / kBR) * kLB;  // threads per head (64)
static_assert(kBR == kLB, "the row reductions halve rows and lanes together");
constexpr int kTile7 = kT7 * kN7;  // floats per tensor tile

struct Wkv7Maps {
  CUtensorMap r, w, k, v, a, b, y;
};

// Sum over the kLB lanes of a row block of x[r] for each of its kBR (= kLB) rows: recursive
// halving (exchange half the rows with the lane differing in the highest bit of the block,
// then the next, ...). Lane l ends with the full sum for row l mod kLB of the block.
__device__ __forceinline__ float rowblock_reduce(float (&x)[kBR], int lc) {
  int half = kBR / 2;
#pragma unroll
  for (int bit = kLB / 2; bit >= 1; bit >>= 1) {
    const bool up = lc & bit;
#pragma unroll
    for (int r = 0; r < kBR / 2; ++r) {
      if (r < half) {
        const float send = up ? x[r] : x[r + half];
        const float got = __shfl_xor_sync(0xffffffffu, send, bit);
        x[r] = (up ? x[r + half] : x[r]) + got;
      }
    }
    half >>= 1;
  }
  return x[0];
}

// Two row reductions at once (independent shuffles interleave).
__device__ __forceinline__ void rowblock_reduce2(float (&x)[kBR], float (&z)[kBR], int lc,
                                                 float& xs, float& zs) {
  int half = kBR / 2;
#pragma unroll
  for (int bit = kLB / 2; bit >= 1; bit >>= 1) {
    const bool up = lc & bit;
#pragma unroll
    for (int r = 0; r < kBR / 2; ++r) {
      if (r < half) {
        const float sx = up ? x[r] : x[r + half];
        const float sz = up ? z[r] : z[r + half];
        const float gx = __shfl_xor_sync(0xffffffffu, sx, bit);
        const float gz = __shfl_xor_sync(0xffffffffu, sz, bit);
        x[r] = (up ? x[r + half] : x[r]) + gx;
        z[r] = (up ? z[r + half] : z[r]) + gz;
      }
    }
    half >>= 1;
  }
  xs = x[0];
  zs = z[0];
}

__global__ void __launch_bounds__(kThr7) wkv7_fwd_kernel(const __grid_constant__ Wkv7Maps maps,
                                                        int B, int T, int H,
                                                        const float* __restrict__ s0,
                                                        float* __restrict__ s1,
                                                        unsigned* err) {
  // stage st: tiles r, w, k, v, a, b at smem + (6 st + slot) kTile7; y tiles after them
  extern __shared__ __align__(128) float smem7[];
  float* ybuf = smem7 + 6 * kS7 * kTile7;  // [2][kT7][64]
  __shared__ uint64_t bars[kS7];
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int lc = tid & (kLB - 1);    // column block (and, after a row reduction, the row)
  const int r0 = (tid / kLB) * kBR;  // first row of this thread's block
  const int bh = blockIdx.x;
  const int b = bh / H, h = bh - b * H;
  const int ntile = (T + kT7 - 1) / kT7;
  // column of pair m (0 .. kPr-1), element e (0..1) of this thread
  auto col = [&](int m, int e) { return 2 * kLB * m + 2 * lc + e; };

  auto issue = [&](int st, int tile) {
    uint64_t* bar = &bars[st];
    mbar_arrive_expect_tx(bar, 6u * kTile7 * sizeof(float));
    float* dst = smem7 + 6 * st * kTile7;
    const int x = h * kN7, t0 = tile * kT7;
    tma_load_3d(dst + 0 * kTile7, &maps.r, bar, x, t0, b);
    tma_load_3d(dst + 1 * kTile7, &maps.w, bar, x, t0, b);
    tma_load_3d(dst + 2 * kTile7, &maps.k, bar, x, t0, b);
    tma_load_3d(dst + 3 * kTile7, &maps.v, bar, x, t0, b);
    tma_load_3d(dst + 4 * kTile7, &maps.a, bar, x, t0, b);
    tma_load_3d(dst + 5 * kTile7, &maps.b, bar, x, t0, b);
  };
  if (tid == 0) {
    for (int st = 0; st < kS7; ++st) mbar_init(&bars[st], 1);
    mbar_fence_init();
    for (int st = 0; st < kS7 && st < ntile; ++st) issue(st, st);
  }
  __syncthreads();

  float2 S[kBR][kPr];  // S[r][m] = state[r0 + r][col(m, 0 .. 1)]
  {
    const float* src = s0 ? s0 + (size_t(bh) * kN7 + r0) * kN7 : nullptr;
#pragma unroll
    for (int r = 0; r < kBR; ++r)
#pragma unroll
      for (int m = 0; m < kPr; ++m)
        S[r][m] = src ? *reinterpret_cast<const float2*>(src + r * kN7 + col(m, 0))
                      : make_float2(0.f, 0.f);
  }

  for (int tile = 0; tile < ntile; ++tile) {
    const int st = tile % kS7;
    mbar_wait(&bars[st], (tile / kS7) & 1, err);
    const float* base = smem7 + 6 * st * kTile7;
    float* yt = ybuf + (tile & 1) * kTile7;
    if (tile >= 2 && tid == 0) tma_store_wait_read<1>();  // this y buffer's last store has read it
    __syncthreads();
    const int n = min(kT7, T - tile * kT7);
    // sa for the tile's first token: S_{t-1} . a_t summed over this thread's columns, then
    // over the row block. Within the tile the next token's sa is computed together with
    // this token's y (both read the updated state), so their two row reductions run
    // side by side.
    float part[kBR], part2[kBR];
    {
      const float* tok = base;
#pragma unroll
      for (int r = 0; r < kBR; ++r) {
        float2 p = make_float2(0.f, 0.f);
#pragma unroll
        for (int m = 0; m < kPr; ++m)
          p = __ffma2_rn(S[r][m], *reinterpret_cast<const float2*>(tok + 4 * kTile7 + col(m, 0)), p);
        part[r] = p.x + p.y;
      }
    }
    float sa_mine = rowblock_reduce(part, lc);  // sa for row r0 + lc
#pragma unroll 1
    for (int t = 0; t < n; ++t) {
      const float* tok = base + t * kN7;
      const bool next = t + 1 < n;
      // the token's vectors at this thread's columns (pairs), and v at its rows
      float2 rv[kPr], wv[kPr], kv[kPr], bv[kPr], an[kPr];
#pragma unroll
      for (int m = 0; m < kPr; ++m) {
        rv[m] = *reinterpret_cast<const float2*>(tok + 0 * kTile7 + col(m, 0));
        wv[m] = *reinterpret_cast<const float2*>(tok + 1 * kTile7 + col(m, 0));
        kv[m] = *reinterpret_cast<const float2*>(tok + 2 * kTile7 + col(m, 0));
        bv[m] = *reinterpret_cast<const float2*>(tok + 5 * kTile7 + col(m, 0));
        an[m] = next ? *reinterpret_cast<const float2*>(tok + kN7 + 4 * kTile7 + col(m, 0))
                     : make_float2(0.f, 0.f);  // a of the next token
      }
      float vv[kBR];
#pragma unroll
      for (int r = 0; r < kBR; r += 4) {
        const float4 x = *reinterpret_cast<const float4*>(tok + 3 * kTile7 + r0 + r);
        vv[r] = x.x; vv[r + 1] = x.y; vv[r + 2] = x.z; vv[r + 3] = x.w;
      }
      // S_t[i][j] = S[i][j] w_j + sa_i b_j + v_i k_j; then y_i = S_t[i] . r_t and the next
      // token's sa_i = S_t[i] . a_{t+1}
#pragma unroll
      for (int r = 0; r < kBR; ++r) {
        const float sr = __shfl_sync(0xffffffffu, sa_mine, (lane & ~(kLB - 1)) | r);
        const float2 sa2 = make_float2(sr, sr);
        const float2 v2 = make_float2(vv[r], vv[r]);
        float2 p = make_float2(0.f, 0.f), q = make_float2(0.f, 0.f);
#pragma unroll
        for (int m = 0; m < kPr; ++m) {
          S[r][m] = __ffma2_rn(S[r][m], wv[m], __ffma2_rn(sa2, bv[m], __fmul2_rn(v2, kv[m])));
          p = __ffma2_rn(S[r][m], rv[m], p);
          q = __ffma2_rn(S[r][m], an[m], q);
        }
        part[r] = p.x + p.y;
        part2[r] = q.x + q.y;
      }
      float y_mine;
      if (next) {
        rowblock_reduce2(part, part2, lc, y_mine, sa_mine);
      } else {
        y_mine = rowblock_reduce(part, lc);
      }
      yt[t * kN7 + r0 + lc] = y_mine;
    }
    fence_proxy_async_smem();  // the y tile's writes, visible to the TMA store
    __syncthreads();           // the stage is consumed and the y tile complete
    if (tid == 0) {
      tma_store_3d(&maps.y, yt, h * kN7, tile * kT7, b);
      tma_store_commit();
      if (tile + kS7 < ntile) issue(st, tile + kS7);
    }
  }
  if (s1 != nullptr) {
    float* dst = s1 + (size_t(bh) * kN7 + r0) * kN7;
#pragma unroll
    for (int r = 0; r < kBR; ++r)
#pragma unroll
      for (int m = 0; m < kPr; ++m) *reinterpret_cast<float2*>(dst + r * kN7 + col(m, 0)) = S[r][m];
  }
  if (tid == 0) tma_store_wait_all();
}

}  // namespace

int launch_wkv7(int64_t B, int64_t T, int64_t H, const float* r, const float* w, const float* k,
                const float* v, const float* a, const float* b, float* y, const float* s0,
                float* s1, unsigned* err, cudaStream_t stream) {
  const int64_t C = H * kN7;
  Wkv7Maps m;
  const auto dt = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const struct {
    CUtensorMap* map;
    const void* p;
  } tabs[7] = {{&m.r, r}, {&m.w, w}, {&m.k, k}, {&m.v, v}, {&m.a, a}, {&m.b, b}, {&m.y, y}};
  for (const auto& e : tabs)
    if (int rc = encode_btc_map(e.map, e.p, dt, 4, B, T, C, kN7, kT7)) return rc;
  const size_t smem = (6 * kS7 + 2) * size_t(kTile7) * sizeof(float);
  if (cudaFuncSetAttribute(wkv7_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           int(smem)) != cudaSuccess)
    return WKV_ERR_CUDA;
  wkv7_fwd_kernel<<<unsigned(B * H), kThr7, smem, stream>>>(m, int(B), int(T), int(H), s0, s1,
                                                            err);
  return cudaPeekAtLastError() == cudaSuccess ? WKV_OK : WKV_ERR_CUDA;
}

}  // namespace wkv
