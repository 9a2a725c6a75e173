/*
 * wkv.h — C ABI of the B200 (sm_100a) WKV library (libwkv.so).
 *
 * The operator is RWKV's WKV time mixing. For every channel (b, c) of a (B, T, C)
 * sequence batch, with 1-based token index t:
 *
 *   wkv_t = ( sum_{i<t} e^{-(t-1-i) w + k_i} v_i + e^{u + k_t} v_t )
 *         / ( sum_{i<t} e^{-(t-1-i) w + k_i}     + e^{u + k_t} )
 *   y_t   = sigmoid(r_t) * wkv_t
 *
 * (concept page "RWKV（Receptance Weighted Key Value）概念", section 3.2 "时间混合
 * （Time-mixing）与 WKV 算子": the wkv_t equation and out_t = sigmoid(Receptance_t) wkv_t).
 * Equivalently (paper notes "RWKV - 把 RNN 重新带回 Transformer 时代的线性大模型",
 * "一句话总结"), with a_0 = b_0 = 0,
 *   a_t = e^{-w} a_{t-1} + e^{k_t} v_t,   b_t = e^{-w} b_{t-1} + e^{k_t},
 *   wkv_t = (a_{t-1} + e^{u+k_t} v_t) / (b_{t-1} + e^{u+k_t}).
 * w > 0 is the per-channel decay rate (the value itself, not its logarithm) and u the
 * per-channel bonus of the current token (same section 3.2).
 *
 * Conventions shared by every entry point:
 *  - Pointers are DEVICE pointers owned by the caller; the library keeps none after the
 *    call returns and allocates nothing it does not free again within the call's stream
 *    order.
 *  - Tensors of shape (B, T, C) are dense row-major, C fastest. w and u are fp32 [C]
 *    (decode: [L, C]). "bf16" buffers hold IEEE bfloat16 values (passed as void*).
 *  - Sizes are int64. B, T or C == 0 is a valid empty problem (nothing is launched; a
 *    requested final state is set to the initial state). Negative sizes, null required
 *    pointers and pointers not aligned to their element size return
 *    WKV_ERR_INVALID_ARG / WKV_ERR_ALIGNMENT before anything is enqueued.
 *  - Every call is asynchronous on `stream` (0 = legacy default stream). The return value
 *    covers argument checks and launch errors only. Errors raised on the device (a
 *    bounded wait that gave up) are reported by wkv_stream_status().
 *  - Preconditions that are documented, not checked on the device: inputs finite, w > 0,
 *    state denominators b > 0. The empty state is (a, b, p) = (0, 0, -1e38) (or NULL);
 *    never pass -inf.
 *  - Numerics: fp32 accumulation in a log-max-stabilised base-2 form; no exponential
 *    overflows for any finite input. bf16 outputs are rounded to nearest even.
 *  - The library uses one GPU: the device current on the calling thread.
 */
#ifndef WKV_H_
#define WKV_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define WKV_API __attribute__((visibility("default")))
#else
#define WKV_API
#endif

typedef enum wkv_status {
  WKV_OK = 0,
  WKV_ERR_INVALID_ARG = 1, /* negative size, null required pointer, bad workspace size */
  WKV_ERR_ALIGNMENT = 2,   /* a pointer not aligned to its element size                */
  WKV_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed              */
  WKV_ERR_TIMEOUT = 4,     /* a bounded device-side wait gave up (wkv_stream_status)   */
  WKV_ERR_UNSUPPORTED = 5, /* a size beyond what the kernels index (e.g. T >= 2^31), or
                              a shape an entry point's kernels cannot take (documented
                              with the entry point)                                       */
  WKV_ERR_SCRATCH_LIMIT = 6, /* wkv_forward_state_static: the problem needs more scratch
                                than the library's fixed array holds                      */
  WKV_ERR_RANGE = 7          /* reported by wkv_stream_status: an input lay outside the
                                range a kernel handles (wkv_mstate_forward: a decay too
                                strong within a chunk); the outputs are then undefined     */
} wkv_status;

/* Human-readable name of a status code. Never NULL. */
WKV_API const char* wkv_status_string(int status);

/* Library ABI version (major * 10000 + minor * 100 + patch). 1.1: the checkpointed
 * training pair (wkv_forward_checkpointed, wkv_backward_checkpointed). */
WKV_API int wkv_version(void);

/*
 * Forward, fp32. k, v, r, y: fp32 (B, T, C). w, u: fp32 [C].
 * r == NULL: no receptance gate (y = wkv). y must not alias k, v or r.
 * Definition: concept page section 3.2 (see the top of this file).
 */
WKV_API int wkv_forward(int64_t B, int64_t T, int64_t C, const float* w, const float* u,
                        const float* k, const float* v, const float* r, float* y,
                        cudaStream_t stream);

/*
 * Forward, bf16 in and out (k, v, r, y bf16 (B, T, C)); w, u and all arithmetic fp32.
 * Otherwise as wkv_forward.
 */
WKV_API int wkv_forward_bf16(int64_t B, int64_t T, int64_t C, const float* w, const float* u,
                             const void* k, const void* v, const void* r, void* y,
                             cudaStream_t stream);

/*
 * Forward with state in and out, fp32, for streaming and segment-wise encoding (the
 * research report "RWKV模型深度研究报告", section 4.4.2: encode a long input segment by
 * segment and carry the state across; the paper notes' "关键设计 4": the inference state
 * holds numerator, denominator and a stabilising exponent).
 *
 * State layout: three fp32 [B, C] arrays (a, b, p) meaning numerator A = a e^p and
 * denominator B = b e^p of the past (p in natural log). The representation is not unique:
 * (a e^s, b e^s, p - s) is the same state; compare states by a/b and p + ln b.
 * a0/b0/p0: initial state, all three NULL = empty state. a1/b1/p1: final state after the
 * last token, all three NULL = not wanted; they may alias a0/b0/p0.
 * Running the two halves of a sequence through this call with the state handed over gives
 * the result of one call over the whole sequence.
 *
 * Long sequences with few channels (B*C small) are split into time segments processed in
 * parallel; each segment folds the results that earlier segments publish, in a fixed order
 * (bitwise reproducible), with bounded waits. This path allocates its scratch with
 * cudaMallocAsync on `stream` and frees it again in stream order.
 */
WKV_API int wkv_forward_state(int64_t B, int64_t T, int64_t C, const float* w, const float* u,
                              const float* k, const float* v, const float* r, float* y,
                              const float* a0, const float* b0, const float* p0, float* a1,
                              float* b1, float* p1, cudaStream_t stream);

/*
 * wkv_forward_state without any device allocation. No counterpart in the pages: this is a
 * deployment variant of the entry point above, for callers that cannot allocate device
 * memory when they run the operator (a serving loop that must not risk the implicit
 * device synchronisation an allocation can bring, a memory manager that owns all device
 * memory, a deployment that forbids dynamic allocation after start-up).
 *
 * Same arguments, layout, semantics and results as wkv_forward_state; the caller passes
 * all inputs and outputs. The scratch of the chunked path (a 4-byte flag and 1 KiB of
 * published carries per item, an item being one batch row x 32-channel group x 256-token
 * segment, plus a 16-byte header) comes from a fixed array of 8 MiB + 64 KiB in the
 * library's device memory, which every GPU that loads the library holds until the process
 * exits: up to 8223 items, e.g. one sequence of 32768 tokens x 2048 channels (8192
 * items). The chunked path is taken below 8192 channels B*C. Problems whose chunked
 * plan needs more return WKV_ERR_SCRATCH_LIMIT before anything is enqueued; problems that
 * take the streaming path need no scratch and have no limit. Nothing is allocated: no
 * cudaMalloc, cudaMallocAsync or cudaFree (the flags are cleared with cudaMemsetAsync).
 *
 * The first call made with a given device current looks up the array's device address
 * (cudaGetSymbolAddress) and caches it; make that first call before any stream capture.
 * Every call shares the one array and leaves its contents behind: calls whose work
 * overlaps on the GPU (different streams, or host threads not ordered with each other)
 * race on it and give undefined results; order such calls, e.g. on one stream.
 */
WKV_API int wkv_forward_state_static(int64_t B, int64_t T, int64_t C, const float* w,
                                     const float* u, const float* k, const float* v,
                                     const float* r, float* y, const float* a0,
                                     const float* b0, const float* p0, float* a1, float* b1,
                                     float* p1, cudaStream_t stream);

/*
 * One token for N sequences x L layers (recurrent inference; paper notes "关键设计 4",
 * the single-token step keeps only the state). k, v, r, y: fp32 [N, L, C]; w, u: fp32
 * [L, C] (layer l of every sequence uses row l); a, b, p: fp32 [N, L, C] state in the
 * representation of wkv_forward_state, read and updated in place. r == NULL: no gate.
 * The output uses the state before the token; the state is then advanced by the token.
 */
WKV_API int wkv_decode_step(int64_t N, int64_t L, int64_t C, const float* w, const float* u,
                            const float* k, const float* v, const float* r, float* y, float* a,
                            float* b, float* p, cudaStream_t stream);

/*
 * S chained tokens for N sequences x L layers in one call, the state kept on chip between
 * them (the news page "RWKV CUDA linear attention GPU", 技术深度解析, 持久化内核设计: a
 * kernel that stays resident across token generations rather than one launch per token).
 * Token s of every sequence and layer is the single-token step of wkv_decode_step applied
 * to the state that token s - 1 left; the state is read once at the start and written
 * once at the end, so a token moves 16 bytes per state (k, v, r in, y out) plus 24/S for
 * the state, against 40 for separate wkv_decode_step calls. Results are bit for bit those
 * of S wkv_decode_step calls.
 *   k, v, r, y: fp32 [S, N, L, C] (token-major: token s is the [N, L, C] block at
 *     s N L C); w, u: fp32 [L, C]; a, b, p: fp32 [N, L, C] state, read and updated in
 *     place. r == NULL: no gate. y must not overlap k, v, r, a, b or p, and a, b, p must
 *     not overlap each other or the inputs.
 *   The tokens must be known in advance (as in prefill through a decode-shaped state
 *   batch, or in checking several drafted tokens at once); a model whose next token
 *   depends on this token's output calls wkv_decode_step per token.
 * S == 0 or an empty batch: nothing is done. S >= 2^31: WKV_ERR_UNSUPPORTED.
 */
WKV_API int wkv_decode_steps(int64_t N, int64_t L, int64_t C, int64_t S, const float* w,
                             const float* u, const float* k, const float* v, const float* r,
                             float* y, float* a, float* b, float* p, cudaStream_t stream);

/*
 * Backward of the forward (wkv_forward with the same w, u, k, v, r), fp32: gradients of
 * L = sum dy . y. The pages say only that the operator trains by ordinary backpropagation
 * (news page "RWKV CUDA linear attention GPU": fused forward and backward kernels); the
 * formulas are the chain rule applied to the wkv_t equation of the concept page, section
 * 3.2, with w the positive decay rate itself:
 *   dk, dv, dr: fp32 (B, T, C), overwritten; dr = dL/dr, may be NULL (then not computed);
 *   dw, du:     fp32 [C], overwritten with the sums over b and t.
 * r == NULL: the ungated forward (y = wkv); dr must then be NULL.
 * workspace: caller-owned device memory of at least wkv_backward_workspace_bytes(B, T, C)
 * bytes, 256-byte aligned; its contents need no initialisation and are scratch after the
 * call. Too small a workspace returns WKV_ERR_INVALID_ARG. Deterministic: dw and du are
 * reduced over b in a fixed order.
 */
WKV_API size_t wkv_backward_workspace_bytes(int64_t B, int64_t T, int64_t C);
WKV_API int wkv_backward(int64_t B, int64_t T, int64_t C, const float* w, const float* u,
                         const float* k, const float* v, const float* r, const float* dy,
                         float* dk, float* dv, float* dw, float* du, float* dr, void* workspace,
                         size_t workspace_bytes, cudaStream_t stream);

/*
 * Backward of the stateful forward (wkv_forward_state with the same w, u, k, v, r and
 * initial state), fp32: gradients of L = sum dy . y + L', where L' is a later loss that
 * depends on the final state, as when a long sequence is trained in consecutive pieces.
 * Defined, like wkv_backward, by the chain rule through the recurrence of the paper notes
 * "RWKV - 把 RNN 重新带回 Transformer 时代的线性大模型", "一句话总结" (numerator and
 * denominator decayed by e^{-w} and advanced by e^{k} v and e^{k}).
 *   a0, b0, p0: the initial state given to the forward (fp32 [B, C], the representation of
 *     wkv_forward_state: numerator a0 e^{p0}, denominator b0 e^{p0}); all NULL = the empty
 *     state.
 *   ga1, gb1:   dL'/da1 and dL'/db1 for the final state (a1, b1, p1) that the forward
 *     returned, p1 its log-scale (fp32 [B, C]); all three NULL = no later loss. L' is
 *     taken to depend on the state through its numerator a1 e^{p1} and denominator
 *     b1 e^{p1} only (p is a scale, not information), so no gradient for p1 is needed.
 *   da0, db0, dp0: dL/da0, dL/db0, dL/dp0 (fp32 [B, C], overwritten; dp0 = a0 da0 +
 *     b0 db0); all NULL = not wanted. Passing one piece's (da0, db0, p0) as the previous
 *     piece's (ga1, gb1, p1) chains the backward over consecutive pieces.
 *   dk, dv, dr, dw, du, r, workspace (wkv_backward_workspace_bytes(B, T, C)): as
 *     wkv_backward; dw includes the decay of the initial state and of the final state's
 *     gradient.
 * T == 0: dw, du are zeroed and the state's gradients pass through (the final state is
 * the initial one). Each triple must be all NULL or all non-NULL (else
 * WKV_ERR_INVALID_ARG). Deterministic, like wkv_backward.
 */
WKV_API int wkv_backward_state(int64_t B, int64_t T, int64_t C, const float* w, const float* u,
                               const float* k, const float* v, const float* r, const float* dy,
                               const float* a0, const float* b0, const float* p0,
                               const float* ga1, const float* gb1, const float* p1, float* dk,
                               float* dv, float* dw, float* du, float* dr, float* da0,
                               float* db0, float* dp0, void* workspace, size_t workspace_bytes,
                               cudaStream_t stream);

/*
 * Training step with the checkpoints made by the forward. The backward (wkv_backward,
 * wkv_backward_state) spends about a quarter of its time on a pass over k and v that forms
 * the state entering every chunk of 16 tokens; in training the forward has just walked the
 * same tokens, so wkv_forward_checkpointed writes those states (1 byte per element) into the
 * backward's workspace as it goes, and wkv_backward_checkpointed, given that workspace,
 * skips the pass.
 *
 * wkv_forward_checkpointed: y as wkv_forward_state (initial state a0, b0, p0 or all NULL;
 *   no final state), fp32, and the checkpoints into `workspace` (device, 256-byte aligned,
 *   at least wkv_backward_workspace_bytes(B, T, C) bytes, owned by the caller and kept
 *   unchanged until the backward). y is bit for bit what wkv_forward's streaming kernel
 *   computes (wkv_forward takes a chunked form instead below 8192 channels B*C, which
 *   rounds differently); the backward then recomputes in that kernel's arithmetic.
 *   Needs the shapes of the streaming kernel: C a multiple of 4 and k, v, r, y 16-byte
 *   aligned, else WKV_ERR_UNSUPPORTED. Errors as wkv_forward_state; a missing or short
 *   workspace is WKV_ERR_INVALID_ARG. T == 0: nothing is written.
 * wkv_backward_checkpointed: arguments and results as wkv_backward_state; `workspace` must
 *   be the one the forward filled, with the same B, T, C, w, u, k, v and initial state
 *   (nothing checks this: other inputs give wrong gradients). Needs C a multiple of 4 and
 *   k, v, r, dy, dk, dv, dr 16-byte aligned, else WKV_ERR_UNSUPPORTED. The checkpoints are
 *   read, not changed: one forward can serve several backward calls. Deterministic.
 */
WKV_API int wkv_forward_checkpointed(int64_t B, int64_t T, int64_t C, const float* w,
                                     const float* u, const float* k, const float* v,
                                     const float* r, float* y, const float* a0, const float* b0,
                                     const float* p0, void* workspace, size_t workspace_bytes,
                                     cudaStream_t stream);
WKV_API int wkv_backward_checkpointed(
    int64_t B, int64_t T, int64_t C, const float* w, const float* u, const float* k,
    const float* v, const float* r, const float* dy, const float* a0, const float* b0,
    const float* p0, const float* ga1, const float* gb1, const float* p1, float* dk, float* dv,
    float* dw, float* du, float* dr, float* da0, float* db0, float* dp0, void* workspace,
    size_t workspace_bytes, cudaStream_t stream);

/*
 * RWKV-7 recurrence per head, fp32 (research report "RWKV模型深度研究报告（截至2026年初）",
 * section 1.3.3 "RWKV-7 (Goose)": the generalised-delta-rule state update
 *   S_t = S_{t-1} (diag(w_t) + a_t^T b_t) + v_t^T k_t
 * with an N x N state per head, row i = value channel, column j = key channel). The
 * report gives no read-out; the output is y_t = S_t r_t^T (the receptance as the query).
 *   r, w, k, v, a, b, y: fp32 (B, T, H, N) row-major (C = H N channels, head h holding
 *     channels h N .. h N + N - 1); w is the decay factor itself (typically in (0, 1)).
 *   s0: the initial state, fp32 (B, H, N, N) with S[i][j] at i N + j; NULL = zero.
 *   s1: the final state, same layout; NULL = not wanted; may alias s0.
 * N must be 64 (else WKV_ERR_UNSUPPORTED); every pointer must be 16-byte aligned (else
 * WKV_ERR_ALIGNMENT). T == 0: s1 = s0 (zero if s0 is NULL). Asynchronous on `stream`.
 */
WKV_API int wkv7_forward(int64_t B, int64_t T, int64_t H, int64_t N, const float* r,
                         const float* w, const float* k, const float* v, const float* a,
                         const float* b, float* y, const float* s0, float* s1,
                         cudaStream_t stream);

/*
 * Matrix-valued-state WKV with a per-key-channel, data-dependent decay, fp32: the RWKV-5/6
 * form (research report "RWKV模型深度研究报告", section 1.3.2: a matrix-valued state per
 * head, each feature channel with its own time decay), computed chunkwise with matrix
 * products inside each chunk of 64 tokens and the state carried between chunks (section
 * 1.4.1), the products on the tensor cores. Per head of N channels:
 *   S_t[i][j] = S_{t-1}[i][j] w_t[j] + v_t[i] k_t[j],    y_t[i] = sum_j S_t[i][j] r_t[j]
 * i.e. wkv7_forward with a = b = 0 (section 1.3.3's update without the delta term), and
 * the same read-out and layouts:
 *   r, w, k, v, y: fp32 (B, T, H, N) row-major; w the decay factor itself (in (0, 1]).
 *   s0: initial state (B, H, N, N), S[i][j] at i N + j; NULL = zero. s1: final state, same
 *     layout; NULL = not wanted; may alias s0.
 * Numerics: the products run as three tf32 tensor-core products of operands split into
 * tf32 high and low parts, accumulated in fp32 (about 2^-22 relative error per product).
 * Range: the decay over any 31 or 32 consecutive tokens aligned to half a chunk must stay
 * above 2^-60 per channel (e.g. w >= 0.27 on every token); otherwise wkv_stream_status()
 * reports WKV_ERR_RANGE and y, s1 are undefined (wkv7_forward with a = b = 0 handles any
 * decay, token by token).
 * N must be 64 (else WKV_ERR_UNSUPPORTED); every pointer 16-byte aligned (else
 * WKV_ERR_ALIGNMENT); y must not overlap the inputs or the states. T == 0: s1 = s0 (zero
 * if s0 is NULL). Scratch (a two-slot state ring per head, 32 KiB per (batch row, head))
 * is allocated with cudaMallocAsync on `stream` and freed in stream order. Chunks of one
 * head wait for one another on the device, with bounded waits (WKV_ERR_TIMEOUT).
 */
WKV_API int wkv_mstate_forward(int64_t B, int64_t T, int64_t H, int64_t N, const float* r,
                               const float* w, const float* k, const float* v, float* y,
                               const float* s0, float* s1, cudaStream_t stream);

/*
 * Query and clear device-side errors. Synchronises `stream`, then returns WKV_ERR_TIMEOUT
 * if any kernel of this library on the current device gave up a bounded wait since the
 * last query, else WKV_ERR_RANGE if a kernel met an input outside its range (the outputs
 * of that call are undefined in both cases), WKV_ERR_CUDA if the stream reports a CUDA
 * error, else WKV_OK.
 */
WKV_API int wkv_stream_status(cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* WKV_H_ */
