// Matrix-valued-state WKV with a per-key-channel, data-dependent decay (the RWKV-5/6
// form), chunked, with the products inside a chunk on the tcgen05 tensor cores (sm_100a).
//
// Sources: research report "RWKV模型深度研究报告", section 1.3.2 (RWKV-5/6 carry a
// matrix-valued state, and every feature channel decays at its own rate) and section 1.4.1
// (chunkwise-parallel training: matrix products inside a chunk, the state handed from
// chunk to chunk). The update is the a = b = 0 case of section 1.3.3's
// S_t = S_{t-1} (diag(w_t) + a_t^T b_t) + v_t^T k_t, read out with the receptance as the
// query: per head of N = 64 channels,
//   S_t[i][j] = S_{t-1}[i][j] w_t[j] + v_t[i] k_t[j],    y_t[i] = sum_j S_t[i][j] r_t[j].
//
// A chunk of L = 64 tokens entered with the state S_0. With gamma_t = prod_{u<=t} w_u
// (per key channel, from the chunk's first token), a reference token m = 31 and
// G_t = gamma_t / gamma_m, every decay between two tokens factors as
// gamma_t / gamma_s = G_t / G_s, with G bounded by the decay over half a chunk. Writing
// R~ for the rows G_t o r_t and K~ for the rows k_s / G_s:
//   A   = tril(R~ K~^T)                                   (token t x token s, s <= t)
//   Y   = R~ (S_0 o gamma_m)^T + A V                       (token t x value channel i)
//   S_L = S_0 o gamma_L + (V^T K~) o G_{L-1}               (o: scaling of column j)
// Four 64 x 64 x 64 products. Each operand is split into three bf16 parts (x = hi + mid +
// lo, 24 significant bits) and each product runs as six bf16 tensor-core products (hi.hi,
// then hi.mid, mid.hi, hi.lo, lo.hi, mid.mid), which leaves about 2^-24 relative error, the
// rounding of an fp32 product. hi.hi accumulates in one tensor-memory accumulator and the
// five small products in a second; the epilogue adds the two in fp32, so the small terms
// are not rounded into the large sum one product at a time. (A two-part tf32 split leaves
// 2^-22; measured, its error on the output was twice the token-by-token fp32 recurrence's.)
//
// One CTA per (chunk, batch row, head), taken in ticket order chunk-major, so the CTA of
// chunk c starts after the CTA of chunk c - 1 of the same head. The state crosses chunks
// through a two-slot ring per head in global memory (L2-resident): chunk c waits (bounded)
// for chunk c - 1's state, forms its own state right after its first products and
// publishes it at once, so the serial part of the chain is one 64 x 64 multiply-add per
// chunk; everything else of every chunk runs in parallel.
//
// Shared memory: bf16 tiles of 64 x 64 without swizzle, in interleaved core matrices of
// 8 rows x 16 bytes: element (row, col) at (row % 8) * 16 + (col / 8) * 128 + (row / 8) *
// 1024 + (col % 8) * 2, read as K-major operands (rows = M or N, cols = K; LBO 128, SBO
// 1024). An operand is three such tiles (hi, mid, lo: 24 KiB). Every operand is K-major
// (in this layout MN-major tf32 operands read as zeros, measured): R~ and K~ token-major,
// K~ also transposed (rows = key channel j), V transposed (rows = value channel i). After
// the first products (D_A, D_U) the K~ tiles take (S_0 o gamma_m) and the K~^T tiles take A,
// so that the inter-chunk term and A V run together as the second and last MMA phase.
// Tensor memory: 256 columns, each result a (main, correction) pair of 64-column
// accumulators (M = 64 layout): D_A at 0/64, D_U (= V^T K~) at 128/192, and D_Y at 128/192
// once D_U has been read.
#include <algorithm>

#include "wkv_internal.h"
#include "wkv_tc.cuh"

namespace wkv {

namespace {

constexpr int kCL = 64;                 // tokens per chunk
constexpr int kHN = 64;                 // head size
constexpr uint32_t kTile = 8192;        // bytes of a 64 x 64 bf16 tile
constexpr uint32_t kOp = 3 * kTile;     // an operand: hi, mid, lo tiles
constexpr int kGP = 68;                 // row pitch (floats) of the decay table
constexpr uint32_t kOffR = 0, kOffK = kOp, kOffKt = 2 * kOp, kOffV = 3 * kOp;  // G in V's space
constexpr uint32_t kOffVec = 4 * kOp;  // gref, g63 [64] each, quarter totals [4][64]
constexpr uint32_t kSmemBytes = kOffVec + 6 * kHN * 4;
constexpr uint32_t kTmemCols = 256;
static_assert(kCL * kGP * 4 <= kOp, "the decay table must fit in V's space");

// Byte offset of element (row, col) in a tile.
__device__ __forceinline__ uint32_t el_off(int row, int col) {
  return uint32_t((row & 7) * 16 + (col >> 3) * 128 + (row >> 3) * 1024 + (col & 7) * 2);
}

// Four values split into three bf16 quadruples (hi, mid, lo), 8 bytes each.
struct Split4 {
  uint2 p[3];
};

__device__ __forceinline__ uint32_t bits2(__nv_bfloat162 v) {
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ Split4 split4(float4 x) {
  __nv_bfloat162 h0, m0, l0, h1, m1, l1;
  bf16_split3x2(make_float2(x.x, x.y), h0, m0, l0);
  bf16_split3x2(make_float2(x.z, x.w), h1, m1, l1);
  Split4 s;
  s.p[0] = make_uint2(bits2(h0), bits2(h1));
  s.p[1] = make_uint2(bits2(m0), bits2(m1));
  s.p[2] = make_uint2(bits2(l0), bits2(l1));
  return s;
}

// Elements (row, col .. col + 3), col % 4 == 0, of an operand's three tiles.
__device__ __forceinline__ void st_row4(unsigned char* op, int row, int col, const Split4& s) {
  const uint32_t off = el_off(row, col);
#pragma unroll
  for (int t = 0; t < 3; ++t) *reinterpret_cast<uint2*>(op + t * kTile + off) = s.p[t];
}

// Elements (row .. row + 3, col), row % 4 == 0, of an operand's three tiles: the transpose
// of st_row4. The four rows share a core matrix, 16 bytes apart.
__device__ __forceinline__ void st_col4(unsigned char* op, int row, int col, const Split4& s) {
  unsigned char* const at = op + el_off(row, col);
#pragma unroll
  for (int t = 0; t < 3; ++t) {
    const uint32_t lo = s.p[t].x, hi = s.p[t].y;
    *reinterpret_cast<uint16_t*>(at + t * kTile + 0) = uint16_t(lo);
    *reinterpret_cast<uint16_t*>(at + t * kTile + 16) = uint16_t(lo >> 16);
    *reinterpret_cast<uint16_t*>(at + t * kTile + 32) = uint16_t(hi);
    *reinterpret_cast<uint16_t*>(at + t * kTile + 48) = uint16_t(hi >> 16);
  }
}

// The 64 x 64 x 64 product of two split operands (A: rows M, cols K; B: rows N, cols K),
// given the descriptors of their hi tiles (an operand's tiles and K steps differ only in
// the start-address field, so each MMA's descriptor is the base plus a constant):
// hi.hi into d, the five correction products into d + 64. accumulate: add to d, d + 64.
__device__ __forceinline__ void mma_split(uint32_t d, uint64_t a, uint64_t b, bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16(64, 64);
  // (a part, b part) in tiles: hi = 0, mid = 1, lo = 2
  constexpr int pa[6] = {0, 0, 1, 0, 2, 1}, pb[6] = {0, 1, 0, 2, 0, 1};
#pragma unroll
  for (int p = 0; p < 6; ++p)
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
      mma_bf16(p == 0 ? d : d + 64, a + uint64_t((pa[p] * kTile + ks * 256) >> 4),
               b + uint64_t((pb[p] * kTile + ks * 256) >> 4), idesc,
               (accumulate || ks > 0 || p > 1) ? 1u : 0u);
}

// 16 columns of a (main, correction) accumulator pair, summed.
__device__ __forceinline__ void tmem_ld16_pair(uint32_t taddr, float (&v)[16]) {
  float c[16];
  tmem_ld16(taddr, v);
  tmem_ld16(taddr + 64, c);
  tmem_wait_ld();
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __fadd_rn(v[i], c[i]);
}

// An M = 64 result fills lanes 0-15 of each sub-partition, so after a 16-column load only
// lanes 0-15 hold data. Hand the upper 8 of those 16 columns to lanes 16-31 (lane l + 16
// takes lane l's), so that each lane works on 8 columns of row (lane % 16): columns
// 0-7 of the 16 in lanes 0-15, 8-15 in lanes 16-31.
__device__ __forceinline__ void half_row(const float (&v)[16], float (&x)[8], int lane) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float up = __shfl_sync(0xffffffffu, v[8 + i], lane & 15);
    x[i] = lane < 16 ? v[i] : up;
  }
}

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads, 2) wkv_mstate_kernel(
    const float* __restrict__ r, const float* __restrict__ w, const float* __restrict__ k,
    const float* __restrict__ v, float* __restrict__ y, const float* s0, float* s1, int B,
    int T, int H, int nch, float* ring, unsigned* flags, unsigned* ticket, unsigned* err,
    unsigned long long wait_ns) {
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_slot;
  __shared__ unsigned s_item;
  unsigned char* const sR = smem + kOffR;
  unsigned char* const sK = smem + kOffK;
  unsigned char* const sKt = smem + kOffKt;
  unsigned char* const sV = smem + kOffV;
  float* const G = reinterpret_cast<float*>(smem + kOffV);  // [64][kGP], until V is split
  float* const gref = reinterpret_cast<float*>(smem + kOffVec);
  float* const g63 = gref + kHN;
  float* const qtot = g63 + kHN;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int BH = B * H;
  const unsigned nitems = unsigned(BH) * unsigned(nch);
  const int64_t rs = int64_t(H) * kHN;  // floats between consecutive tokens
  if (tid == 0) {
    s_item = atomicAdd(ticket, 1u);
    mbar_init(&bar, 1);
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = tmem_slot;
  const uint32_t sb = smem_u32(smem);
  const uint64_t aR = smem_desc(sb + kOffR, 128, 1024), aK = smem_desc(sb + kOffK, 128, 1024),
                 aKt = smem_desc(sb + kOffKt, 128, 1024), aV = smem_desc(sb + kOffV, 128, 1024);
  unsigned item = s_item;
  uint32_t phase = 0;  // parity of the next completion of the MMA barrier

  // Persistent: each CTA takes chunks in ticket order (chunk-major over all heads), and
  // takes its next ticket while it works on the current one, so that the next chunk's
  // inputs can be prefetched into L2 meanwhile. A CTA holds at most one future ticket and
  // works on its tickets in order, so the chunk every wait is for has been taken by a CTA
  // that works on it first.
  while (item < nitems) {
  __syncthreads();  // every thread has read s_item
  if (tid == 0) s_item = atomicAdd(ticket, 1u);
  const int c = int(item / unsigned(BH)), bh = int(item % unsigned(BH));
  const int b = bh / H, h = bh % H;
  const int t0 = c * kCL, nvalid = min(kCL, T - t0);
  const int64_t base = (int64_t(b) * T + t0) * rs + int64_t(h) * kHN;

  // Raw w, r, k, v in registers, all loads in flight at once: unit (row, 4 columns) with
  // the row group and column quad from (it, warp) and (row % 8, column group in the quad)
  // from the lane, so that a warp's loads cover 8 rows x 64 bytes and its 8-byte tile
  // stores are conflict-free. Tokens past the end: r, k, v zero, w one.
  float4 ww[4], rr[4], kk[4], vv[4];
  const float4 zero4 = make_float4(0.f, 0.f, 0.f, 0.f);
  const float4 one4 = make_float4(1.f, 1.f, 1.f, 1.f);
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int combo = it * 8 + warp;
    const int row = (combo >> 2) * 8 + (lane & 7), cg = (combo & 3) * 4 + (lane >> 3);
    const int64_t g = base + row * rs + cg * 4;
    const bool ok = row < nvalid;
    ww[it] = ok ? __ldcs(reinterpret_cast<const float4*>(w + g)) : one4;
    rr[it] = ok ? __ldcs(reinterpret_cast<const float4*>(r + g)) : zero4;
    kk[it] = ok ? __ldcs(reinterpret_cast<const float4*>(k + g)) : zero4;
    vv[it] = ok ? __ldcs(reinterpret_cast<const float4*>(v + g)) : zero4;
  }
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int combo = it * 8 + warp;
    const int row = (combo >> 2) * 8 + (lane & 7), cg = (combo & 3) * 4 + (lane >> 3);
    *reinterpret_cast<float4*>(G + row * kGP + cg * 4) = ww[it];
  }
  __syncthreads();

  // The next chunk's inputs into L2 while this one is worked on.
  const unsigned next = s_item;
  if (next < nitems) {
    const int nc = int(next / unsigned(BH)), nbh = int(next % unsigned(BH));
    const int nt0 = nc * kCL, nvalid2 = min(kCL, T - nt0);
    const int64_t nbase = (int64_t(nbh / H) * T + nt0) * rs + int64_t(nbh % H) * kHN;
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int combo = it * 8 + warp;
      const int row = (combo >> 2) * 8 + (lane & 7), cg = (combo & 3) * 4 + (lane >> 3);
      if (row < nvalid2 && (lane >> 3) % 2 == 0) {  // one lane per 128-byte line
        const int64_t g = nbase + row * rs + cg * 4;
        prefetch_l2(w + g);
        prefetch_l2(r + g);
        prefetch_l2(k + g);
        prefetch_l2(v + g);
      }
    }
  }

  // Decays of the chunk, per key channel j, in quarters of 16 tokens (thread (j, q)): a
  // running product p_t within each quarter and the quarter totals Q_0..Q_3; then
  // gamma_t = Q_0 p_t (second quarter), gamma_m = Q_0 Q_1 (m = 31), and G_t = gamma_t /
  // gamma_m in the first half, G_t = p_t (third quarter) or Q_2 p_t (fourth) in the second.
  {
    const int j = tid & 63, qtr = tid >> 6;
    float p[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) p[t] = G[(16 * qtr + t) * kGP + j];
#pragma unroll
    for (int t = 1; t < 16; ++t) p[t] = __fmul_rn(p[t - 1], p[t]);
    qtot[qtr * kHN + j] = p[15];
    __syncthreads();
    const float q0 = qtot[j], q1 = qtot[kHN + j], q2 = qtot[2 * kHN + j];
    if (qtr < 2) {
      const float gm = __fmul_rn(q0, q1);
      const float f = __fmul_rn(qtr == 1 ? q0 : 1.f, __frcp_rn(gm));
#pragma unroll
      for (int t = 0; t < 16; ++t) G[(16 * qtr + t) * kGP + j] = __fmul_rn(f, p[t]);
      if (qtr == 0) {
        gref[j] = gm;
        // The factorisation needs the decay over each half of the chunk to stay above
        // 2^-60 (G_0 = 1 / (w_1 ... w_31), G_63 = w_32 ... w_63); beyond that R~ or K~
        // could leave the float range. Flag it rather than return infinities silently.
        if (!(G[j] <= 0x1p60f)) atomicOr(err, kErrRange);
      }
    } else {
      const float f = qtr == 3 ? q2 : 1.f;
#pragma unroll
      for (int t = 0; t < 16; ++t) G[(16 * qtr + t) * kGP + j] = __fmul_rn(f, p[t]);
      if (qtr == 3) {
        const float g = __fmul_rn(q2, p[15]);
        g63[j] = g;
        if (!(g >= 0x1p-60f)) atomicOr(err, kErrRange);
      }
    }
  }
  __syncthreads();

  // R~ = G o r and K~ = k / G: split, token-major, and K~ also transposed.
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int combo = it * 8 + warp;
    const int row = (combo >> 2) * 8 + (lane & 7), col = ((combo & 3) * 4 + (lane >> 3)) * 4;
    const float4 gg = *reinterpret_cast<const float4*>(G + row * kGP + col);
    const Split4 rs4 = split4(make_float4(__fmul_rn(rr[it].x, gg.x), __fmul_rn(rr[it].y, gg.y),
                                          __fmul_rn(rr[it].z, gg.z), __fmul_rn(rr[it].w, gg.w)));
    const Split4 ks4 = split4(make_float4(__fmul_rn(kk[it].x, __frcp_rn(gg.x)),
                                          __fmul_rn(kk[it].y, __frcp_rn(gg.y)),
                                          __fmul_rn(kk[it].z, __frcp_rn(gg.z)),
                                          __fmul_rn(kk[it].w, __frcp_rn(gg.w))));
    st_row4(sR, row, col, rs4);
    st_row4(sK, row, col, ks4);
    st_col4(sKt, col, row, ks4);
  }
  __syncthreads();  // G is read no more: its space takes V^T
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int combo = it * 8 + warp;
    const int row = (combo >> 2) * 8 + (lane & 7), col = ((combo & 3) * 4 + (lane >> 3)) * 4;
    st_col4(sV, col, row, split4(vv[it]));
  }
  fence_proxy_async_smem();
  __syncthreads();

  if (tid == 0) {
    tc_fence_after();
    mma_split(tm + 0, aR, aK, false);     // D_A = R~ K~^T
    mma_split(tm + 128, aV, aKt, false);  // D_U = V^T K~
    mma_commit(&bar);
  }

  // Epilogue roles: warp w reads tensor-memory sub-partition w % 4 (rows 16 (w % 4) ..
  // + 15 of an M = 64 result in its lanes 0-15) and the column half w / 4.
  const int sub = warp & 3, ch = warp >> 2;
  const int ri = 16 * sub + (lane & 15);
  const int c8 = (lane >> 4) * 8;  // this lane's 8 of each 16 columns (half_row)
  const uint32_t trow = tm + (uint32_t(32 * sub) << 16);
  const float* sprev = c == 0 ? (s0 ? s0 + int64_t(bh) * kHN * kHN : nullptr)
                              : ring + (int64_t(bh) * 2 + ((c - 1) & 1)) * kHN * kHN;
  float* snext = c == nch - 1 ? (s1 ? s1 + int64_t(bh) * kHN * kHN : nullptr)
                              : ring + (int64_t(bh) * 2 + (c & 1)) * kHN * kHN;

  // The state entering this chunk: published by chunk c - 1 of this head (ticket order
  // guarantees that CTA has started), or the caller's initial state.
  if (c > 0 && tid == 0) wait_flag(flags + bh, unsigned(c), wait_ns, err);
  __syncthreads();
  float4 sp[4];  // this lane's 8 columns of each 16 (half_row) of its row of S_{c-1}
#pragma unroll
  for (int e = 0; e < 4; ++e)
    sp[e] = sprev ? __ldcg(reinterpret_cast<const float4*>(
                        sprev + ri * kHN + 32 * ch + 16 * (e >> 1) + c8 + 4 * (e & 1)))
                  : zero4;
  if (warp == 0) mbar_wait(&bar, phase, err);  // the others sleep at the barrier
  phase ^= 1u;
  __syncthreads();
  tc_fence_after();

  // S_c = S_{c-1} o gamma_L + D_U o G_63 (gamma_L = gamma_m G_63), stored and published;
  // (S_{c-1} o gamma_m) split into the K~ tiles (read no more) for the inter-chunk term.
#pragma unroll
  for (int qq = 0; qq < 2; ++qq) {
    const int q = 2 * ch + qq;
    float v16[16], du[8];
    tmem_ld16_pair(trow + 128 + 16 * q, v16);
    half_row(v16, du, lane);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int j = 16 * q + c8 + 4 * e;
      const float4 x = sp[2 * qq + e];
      const float4 g = *reinterpret_cast<const float4*>(g63 + j);
      const float4 m = *reinterpret_cast<const float4*>(gref + j);
      if (snext) {
        const float4 sn = make_float4(
            fmaf(x.x, __fmul_rn(m.x, g.x), __fmul_rn(du[4 * e + 0], g.x)),
            fmaf(x.y, __fmul_rn(m.y, g.y), __fmul_rn(du[4 * e + 1], g.y)),
            fmaf(x.z, __fmul_rn(m.z, g.z), __fmul_rn(du[4 * e + 2], g.z)),
            fmaf(x.w, __fmul_rn(m.w, g.w), __fmul_rn(du[4 * e + 3], g.w)));
        __stcg(reinterpret_cast<float4*>(snext + ri * kHN + j), sn);
      }
      st_row4(sK, ri, j, split4(make_float4(__fmul_rn(x.x, m.x), __fmul_rn(x.y, m.y),
                                            __fmul_rn(x.z, m.z), __fmul_rn(x.w, m.w))));
    }
  }
  // A = tril(D_A), split into the K~^T tiles (read no more).
  const int t_row = ri;
#pragma unroll
  for (int qq = 0; qq < 2; ++qq) {
    const int q = 2 * ch + qq;
    float v16[16], a[8];
    tmem_ld16_pair(trow + 0 + 16 * q, v16);
    half_row(v16, a, lane);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int s = 16 * q + c8 + 4 * e;
      st_row4(sKt, t_row, s,
              split4(make_float4(s + 0 <= t_row ? a[4 * e + 0] : 0.f,
                                 s + 1 <= t_row ? a[4 * e + 1] : 0.f,
                                 s + 2 <= t_row ? a[4 * e + 2] : 0.f,
                                 s + 3 <= t_row ? a[4 * e + 3] : 0.f)));
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    st_release(flags + bh, unsigned(c + 1));
    tc_fence_after();
    mma_split(tm + 128, aR, aK, false);   // D_Y = R~ (S_0 o gamma_m)^T
    mma_split(tm + 128, aKt, aV, true);   //     + A V
    mma_commit(&bar);
  }
  if (warp == 0) mbar_wait(&bar, phase, err);  // the others sleep at the barrier
  phase ^= 1u;
  __syncthreads();
  tc_fence_after();

  // y rows of this chunk.
  float* const yrow = y + base + int64_t(t_row) * rs;
#pragma unroll
  for (int qq = 0; qq < 2; ++qq) {
    const int q = 2 * ch + qq;
    float v16[16], o[8];
    tmem_ld16_pair(trow + 128 + 16 * q, v16);
    half_row(v16, o, lane);
    if (t_row < nvalid) {
#pragma unroll
      for (int e = 0; e < 2; ++e)
        __stcs(reinterpret_cast<float4*>(yrow + 16 * q + c8 + 4 * e),
               make_float4(o[4 * e + 0], o[4 * e + 1], o[4 * e + 2], o[4 * e + 3]));
    }
  }
  tc_fence_before();
  item = next;
  }  // while
  __syncthreads();
  if (warp == 0) tmem_dealloc(tm, kTmemCols);
}

}  // namespace

size_t mstate_scratch_bytes(int64_t B, int64_t H) {
  const int64_t BH = B * H;
  return size_t((16 + 4 * BH + 255) / 256 * 256) + size_t(BH) * 2 * kHN * kHN * sizeof(float);
}

int launch_mstate(int64_t B, int64_t T, int64_t H, const float* r, const float* w,
                  const float* k, const float* v, float* y, const float* s0, float* s1,
                  void* scratch, unsigned* err, cudaStream_t stream) {
  const int64_t BH = B * H, nch = (T + kCL - 1) / kCL;
  if (BH * nch >= (int64_t(1) << 31)) return WKV_ERR_UNSUPPORTED;
  const size_t head = size_t((16 + 4 * BH + 255) / 256 * 256);
  if (cudaMemsetAsync(scratch, 0, head, stream) != cudaSuccess) return WKV_ERR_CUDA;
  unsigned* ticket = static_cast<unsigned*>(scratch);
  unsigned* flags = ticket + 4;
  float* ring = reinterpret_cast<float*>(static_cast<char*>(scratch) + head);
  // Two CTAs per SM (shared memory and the 2 x 256 tensor-memory columns allow exactly
  // that): ask for the whole shared-memory carveout.
  if (cudaFuncSetAttribute(wkv_mstate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           int(kSmemBytes)) != cudaSuccess ||
      cudaFuncSetAttribute(wkv_mstate_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                           100) != cudaSuccess)
    return WKV_ERR_CUDA;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t grid = std::min<int64_t>(BH * nch, int64_t(2) * sms);  // persistent, 2 per SM
  wkv_mstate_kernel<<<unsigned(grid), kThreads, kSmemBytes, stream>>>(
      r, w, k, v, y, s0, s1, int(B), int(T), int(H), int(nch), ring, flags, ticket, err,
      kWaitLimitNs);
  return cudaPeekAtLastError() == cudaSuccess ? WKV_OK : WKV_ERR_CUDA;
}

}  // namespace wkv
