// Internal interfaces between the C-ABI layer (wkv_api.cu) and the kernel files.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "wkv.h"

namespace wkv {

// Arguments of one forward pass over (B, T, C). k, v, r, y are fp32 or bf16 according to
// the entry point; r may be null (no gate); a0/b0/p0 null = empty initial state; a1/b1/p1
// null = final state not wanted.
struct FwdArgs {
  int64_t B, T, C;
  const float* w;
  const float* u;
  const void* k;
  const void* v;
  const void* r;
  void* y;
  const float* a0;
  const float* b0;
  const float* p0;
  float* a1;
  float* b1;
  float* p1;
  unsigned* err;  // device error word
};

// Device address of this library's error word on the current device (nullptr on error).
unsigned* device_error_word();

// 3-D tiled tensor map over a (B, T, C) tensor (C fastest) with a box of
// [box_c channels x box_t tokens x 1 batch row]. Returns a wkv_status.
int encode_btc_map(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                   int elem_bytes, int64_t B, int64_t T, int64_t C, int box_c, int box_t);

// Whether the TMA streaming kernel can describe this problem (alignment, extents).
bool fwd_tma_ok(const FwdArgs& a, int elem_bytes);

// Whole-sequence forward, one thread per channel (streaming TMA kernel, or the plain
// kernel when the TMA kernel cannot be used or force_plain is set).
int launch_fwd_stream(const FwdArgs& a, bool bf16, bool force_plain, cudaStream_t stream);

// Chunked (time-parallel) forward for problems with few channels; fp32 only.
// scratch: device memory of chunked_scratch_bytes(); its first flag_bytes must be
// zero on entry (the caller clears them).
size_t chunked_scratch_bytes(int64_t B, int64_t T, int64_t C, int64_t* flag_bytes,
                             int* n_segments);
int launch_fwd_chunked(const FwdArgs& a, void* scratch, int n_segments, cudaStream_t stream);
// Same, with the wait limit (ns) given and, for tests of the bounded wait, segment 0
// optionally withholding its published aggregate so that its successors give up.
int launch_fwd_chunked_ex(const FwdArgs& a, void* scratch, int n_segments,
                          unsigned long long wait_ns, int withhold_seg0, cudaStream_t stream);

// One decode step over N x L x C states.
struct DecodeArgs {
  int64_t N, L, C;
  const float* w;
  const float* u;
  const float* k;
  const float* v;
  const float* r;
  float* y;
  float* a;
  float* b;
  float* p;
};
int launch_decode(const DecodeArgs& a, cudaStream_t stream);
// S chained tokens: k, v, r, y are [S, N, L, C]; the state stays on chip between tokens.
int launch_decode_steps(const DecodeArgs& a, int64_t S, cudaStream_t stream);

// Matrix-valued-state forward (heads of 64), chunked on the tensor cores. scratch: device
// memory of mstate_scratch_bytes(B, H) bytes (cleared in part by the launcher).
size_t mstate_scratch_bytes(int64_t B, int64_t H);
int launch_mstate(int64_t B, int64_t T, int64_t H, const float* r, const float* w,
                  const float* k, const float* v, float* y, const float* s0, float* s1,
                  void* scratch, unsigned* err, cudaStream_t stream);

// Backward over (B, T, C), fp32. r null: no gate (dr must be null). ws: device workspace of
// backward_workspace_bytes(B, T, C) bytes, 256-byte aligned; no part needs clearing.
struct BwdArgs {
  int64_t B, T, C;
  const float* w;
  const float* u;
  const float* k;
  const float* v;
  const float* r;
  const float* dy;
  float* dk;
  float* dv;
  float* dw;
  float* du;
  float* dr;
  void* ws;
  unsigned* err;
  // Backward through a state (all may be NULL): the initial state (a0, b0, p0) [B, C];
  // the gradients (ga1, gb1) of a later loss with respect to the final state's a1, b1,
  // whose log-scale is p1 [B, C]; and the outputs (da0, db0, dp0) [B, C].
  const float* a0 = nullptr;
  const float* b0 = nullptr;
  const float* p0 = nullptr;
  const float* ga1 = nullptr;
  const float* gb1 = nullptr;
  const float* p1 = nullptr;
  float* da0 = nullptr;
  float* db0 = nullptr;
  float* dp0 = nullptr;
  // Chain waits of the time-parallel passes: their limit (ns) and, for tests of the
  // bounded wait only, the last segment of the reverse pass withholding its published map.
  unsigned long long wait_ns = 2000000000ull;
  int withhold_last_map = 0;
  // The workspace already holds the checkpoints (written by launch_fwd_ckpt over the same
  // w, k, v and initial state): the checkpoint pass is skipped and the reverse pass
  // recomputes in the streaming forward's arithmetic. Time-parallel path only.
  int have_ckpt = 0;
};
size_t backward_workspace_bytes(int64_t B, int64_t T, int64_t C);
// Where the backward's workspace keeps the checkpoints ([B, ceil(T/16), C] float4: the state
// (a, b, Q, pl) entering every chunk of 16 tokens) and the state after the last token
// ([B, C] float4).
void backward_checkpoint_ptrs(void* ws, int64_t B, int64_t T, int64_t C, float4** ckpt,
                              float4** ckend);
// Whether the backward takes its time-parallel (checkpointed) path for these arguments.
bool backward_time_parallel_ok(const BwdArgs& a);
// Forward (fp32, TMA shapes only: else WKV_ERR_UNSUPPORTED) that also writes the backward's
// checkpoints into its workspace ws: the streaming kernel in its checkpointing mode
// (wkv_fwd.cu); a backward with have_ckpt set recomputes in the same arithmetic.
int launch_fwd_ckpt(const FwdArgs& a, void* ws, cudaStream_t stream);
int launch_backward(const BwdArgs& a, bool force_plain, cudaStream_t stream);
// Which reverse pass the TMA path takes: 0 automatic, 1 time-parallel segments, 2 one CTA
// per channel group, 3 one CTA of four warps per channel group (a test hook; process-wide).
void set_backward_path(int path);
// T == 0 with the state's gradients wanted: they pass straight through.
int launch_backward_no_tokens(const BwdArgs& a, cudaStream_t stream);

// RWKV-7 recurrence (wkv7.cu), head size 64, all pointers 16-byte aligned.
int launch_wkv7(int64_t B, int64_t T, int64_t H, const float* r, const float* w, const float* k,
                const float* v, const float* a, const float* b, float* y, const float* s0,
                float* s1, unsigned* err, cudaStream_t stream);

}  // namespace wkv
