/*
 * qlora.h — C ABI of the frozen-GGUF-base + LoRA layer library for NVIDIA B200 (sm_100a).
 *
 * The layer is the one the LoRA-over-GGUF training recipe runs in every projection: a frozen,
 * block-quantized base weight (GGUF Q8_0, Q4_0 or Q4_K) plus a trainable rank-r adapter, dense and
 * as routed per-expert SwiGLU MoE ("Things involved in the training" of Show HN: LoRA over GGUF:
 * MMQ and grouped MMQ, the fast LoRA backward formula for linear and MoE layers, MoE routing, the
 * GGUF dequant function). With s = alpha / r:
 *
 *   forward   Y  = X deq(W)^T + s (X A^T) B^T             H = X A^T is returned for the backward
 *   backward  dX = dY deq(W) + s (dY B) A,  dA = s (dY B)^T X,  dB = s dY^T H;  W is never updated
 *
 * Conventions for every entry point
 *   - All tensor arguments are DEVICE pointers to row-major, contiguous buffers that the caller
 *     allocated and owns; the library never allocates, frees or synchronises. Work is enqueued on
 *     `stream` (a cudaStream_t passed as void*, NULL = legacy default stream) and is asynchronous:
 *     results are valid after the caller synchronises that stream.
 *   - bf16 tensors are IEEE bfloat16 (uint16 storage). Packed weights are GGUF blocks in file
 *     order: a weight [rows x cols] is `rows` packed rows of cols/QK blocks each (QK = 32 for
 *     Q4_0/Q8_0, 256 for the K-quants; 18, 34 bytes per Q4_0 / Q8_0 block, 144, 176, 210 per
 *     Q4_K / Q5_K / Q6_K superblock). Expert stacks are [E][rows][...].
 *   - Every pointer must be 16-byte aligned; the packed weight rows, X, dY, A and B rows must make
 *     every row start 16-byte aligned (guaranteed by the shape rules below).
 *   - Return value: a ql_status. Argument errors are detected on the host before anything is
 *     launched. Launch failures return QL_ERR_CUDA. Faults inside kernels surface at the caller's
 *     synchronisation as CUDA errors; a device-side wait that exceeds its bound (about one second)
 *     sets a device status word, read with qlora_device_status().
 *   - Workspace: entry points that need scratch take (ws, ws_bytes); the required size comes from
 *     the matching *_workspace_bytes() query. The caller owns it; its contents on entry do not
 *     matter.
 */
#ifndef QLORA_H
#define QLORA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif
#if defined(__GNUC__)
#pragma GCC visibility push(default)
#endif

/* GGML type ids of the supported block formats. Q2_K (84-byte superblocks) and Q6_K (210 bytes),
 * whose superblocks are not a multiple of 16 bytes and so are not copied by TMA, are supported by
 * gguf_dequant only; the layer entry points return QL_ERR_UNSUPPORTED for them. */
typedef enum { QL_Q4_0 = 2, QL_Q8_0 = 8, QL_Q2_K = 10, QL_Q4_K = 12, QL_Q5_K = 13, QL_Q6_K = 14 } ql_qtype;

/* Element type of an output tensor. */
typedef enum { QL_F32 = 0, QL_BF16 = 1 } ql_dtype;

typedef enum {
  QL_OK = 0,
  QL_ERR_INVALID_ARG = 1, /* null pointer, bad enum, non-positive size */
  QL_ERR_UNSUPPORTED = 2, /* a qtype / rank / expert count the library does not handle */
  QL_ERR_SHAPE = 3,       /* a size rule is broken (e.g. K % 256 != 0) */
  QL_ERR_ALIGNMENT = 4,   /* a pointer is not 16-byte aligned */
  QL_ERR_WORKSPACE = 5,   /* ws is NULL or smaller than the query says */
  QL_ERR_CUDA = 6,        /* a CUDA runtime / driver call failed */
  QL_ERR_TIMEOUT = 7      /* a device-side bounded wait gave up (device status word) */
} ql_status;

/* Human-readable name of a status code. Never NULL. */
const char* qlora_status_string(int status);

/* Number of the library's own kernel launches since load (all entry points, all streams). */
uint64_t qlora_launch_count(void);

/* Timing hook: when set, the library records `start` / `stop` (cudaEvent_t, as void*) on the
 * launch stream right before / after every launch of the tensor-core GEMM kernel of a slot:
 * 0 = dense forward GEMM, 1 = dense input-gradient GEMM, 2 = MoE gate/up GEMM, 3 = MoE down GEMM,
 * 4 = MoE down input-gradient GEMM, 5 = MoE gate/up input-gradient GEMM. Both NULL clears the slot.
 * The caller owns the events; they must outlive every launch made while they are set. Not
 * thread-safe with concurrent calls that launch into the same slot. */
int qlora_set_kernel_events(int slot, void* start, void* stop);

/* Which of the dense linear's pair GEMMs may compute the adapter row products (H = X A^T in the
 * forward, G = s dY B in the input gradient, and the operands built from them) inside their own
 * launch, on the SM pairs their tiles leave idle, instead of in a separate launch before them: bit 0
 * the forward GEMM, bit 1 the input-gradient GEMM (default 1). Either way the results obey the same
 * bounds. Process-wide; returns the previous mask. */
int qlora_set_rows_fusion(int mask);

/* Reads the device status word of the current device (synchronises the device first). Returns
 * QL_OK or the first recorded device-side error (QL_ERR_TIMEOUT); *site (nullable) receives the
 * code of the wait that gave up. reset != 0 clears the word afterwards. */
int qlora_device_status(int* site, int reset);

/* Self-check of the bounded-wait path: launches one block that waits on a barrier nothing ever
 * arrives at, with a limit of `limit_us` microseconds (1..2000000). The wait gives up, records
 * QL_ERR_TIMEOUT in the device status word and the kernel returns normally. */
int qlora_selftest_wait_timeout(int64_t limit_us, void* stream);

/* ---------------------------------------------------------------------------------------------
 * gguf_dequant — expand packed GGUF rows to fp32 or bf16.
 * The pages' recipe runs a standalone GGUF dequant function (Show HN: LoRA over GGUF, "Other
 * notes"); the layer's own kernels never call this: they expand blocks in shared memory.
 *   qtype     QL_Q4_0 | QL_Q8_0 | QL_Q2_K | QL_Q4_K | QL_Q5_K | QL_Q6_K
 *   wq        [rows][cols/QK blocks] packed bytes
 *   rows      > 0
 *   cols      > 0, multiple of 256
 *   out       [rows x cols] of out_dtype. fp32 output is the exact decode rounded once to fp32;
 *             bf16 output is that fp32 value rounded to nearest-even bf16.
 * ------------------------------------------------------------------------------------------- */
int gguf_dequant(int qtype, const void* wq, int64_t rows, int64_t cols, void* out, int out_dtype,
                 void* stream);

/* ---------------------------------------------------------------------------------------------
 * Dense layer (one projection). Shapes: X [M x K] bf16, W packed [N rows x K], A [r x K] bf16,
 * B [N x r] bf16, dY [M x N] bf16. Rules: M >= 1; K % 256 == 0; N % 64 == 0; 1 <= r <= 64.
 * ------------------------------------------------------------------------------------------- */

/* Scratch bytes needed by qlora_linear_fwd / qlora_linear_bwd for these sizes. */
size_t qlora_linear_workspace_bytes(int64_t M, int64_t N, int64_t K, int r);

/* Forward: Y = X deq(W)^T + scale (X A^T) B^T.
 *   Y      [M x N] of y_dtype (QL_F32 or QL_BF16; bf16 is the fp32 result rounded once)
 *   H      [M x r] fp32, receives X A^T (without scale) for the backward; required
 *   Computes deq(W) tile by tile in shared memory; no full-precision weight is written to HBM. */
int qlora_linear_fwd(int qtype, const void* wq, int64_t N, int64_t K, const void* X, int64_t M,
                     const void* A, const void* B, int r, float scale, void* Y, int y_dtype, float* H,
                     void* ws, size_t ws_bytes, void* stream);

/* Backward:
 *   dX  [M x K] of dx_dtype, = dY deq(W) + G A with G = scale dY B; nullable (skips dX)
 *   dA  [r x K] fp32, = G^T X (overwritten)
 *   dB  [N x r] fp32, = scale dY^T H (overwritten)
 *   H   [M x r] fp32 from the forward. */
int qlora_linear_bwd(int qtype, const void* wq, int64_t N, int64_t K, const void* X, const void* dY,
                     int64_t M, const void* A, const void* B, int r, float scale, const float* H,
                     void* dX, int dx_dtype, float* dA, float* dB, void* ws, size_t ws_bytes,
                     void* stream);

/* ---------------------------------------------------------------------------------------------
 * Routed MoE layer with SwiGLU experts (the recipe's MoE routing, grouped quantized matmul and fast
 * LoRA backward for the MoE layer: Show HN: LoRA over GGUF, "Things involved in the training").
 * Expert e: gate/up weight Wgu_e [2I x H] (rows [0, I) gate, [I, 2I) up), down weight Wd_e [H x I],
 * packed and stacked [E][rows][...]; adapters A_gu [E][r][H], B_gu [E][2I][r], A_d [E][r][I],
 * B_d [E][H][r] (bf16); s = scale.
 *   gu = x Wgu^T + s (x A_gu^T) B_gu^T;  h = silu(gu[:I]) * gu[I:];  o = h Wd^T + s (h A_d^T) B_d^T
 *   Y[t] = sum over the k selected slots (slot order) of w_tj * o_tj.
 * Rules: 1 <= k <= min(E, 16); E <= 256; H % 256 == 0; I % 256 == 0; 1 <= r <= 64; T >= 1.
 * P = T * k routed pairs.
 * ------------------------------------------------------------------------------------------- */

/* Scratch bytes for qlora_moe_route: ceil(T / 32) x E int32 (the expert histograms of 32-token rows). */
size_t qlora_moe_route_workspace_bytes(int64_t T, int E, int k);

/* Routing. logits [T x E] bf16. Writes (device buffers of the caller):
 *   topk_idx [T x k] int32   selected experts, descending logit, equal logits -> lower index
 *   topk_w   [T x k] fp32    softmax over the k selected logits
 *   counts   [E] int32, offsets [E+1] int32 (exclusive scan; offsets[E] = P)
 *   perm     [P] int32       pairs t*k+j sorted by (expert, token, slot); inv_perm [P] its inverse
 *   mblk     [E+1] int32     sum over earlier experts of ceil(counts/128): the grouped GEMMs' block list
 * Indices, counts, offsets, perm, inv_perm and mblk are exact (no floating point decides them
 * beyond comparisons of the bf16 logits). Three launches: per row of 32 tokens, the top-k (a warp
 * per token) and the row's expert histogram by warp match (no global atomics); one scan over rows
 * and experts; per row, each pair's position from the scanned counts and the row's lane masks.
 * ws (ws_bytes >= qlora_moe_route_workspace_bytes) holds the histograms; its contents on entry do
 * not matter. */
int qlora_moe_route(const void* logits, int64_t T, int E, int k, int32_t* topk_idx, float* topk_w,
                    int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv_perm, int32_t* mblk,
                    void* ws, size_t ws_bytes, void* stream);

/* Bytes of the activations the forward saves for the backward (caller-owned buffer `saved`):
 * g, u [P x I] fp32, h [P x I] bf16, the bf16 residual h - bf16(h) [P x I] and X A_gu^T, h A_d^T
 * [P x r] fp32, in pair order. */
size_t qlora_moe_saved_bytes(int64_t T, int k, int64_t H, int64_t I, int r);

/* Scratch bytes for qlora_moe_fwd / qlora_moe_bwd with these sizes. */
size_t qlora_moe_workspace_bytes(int64_t T, int k, int E, int64_t H, int64_t I, int r);

/* Forward. X [T x H] bf16; the routing buffers as written by qlora_moe_route; Y [T x H] of y_dtype.
 * The weighted per-pair outputs stay fp32 up to the slot-ordered fp32 sum; g and u are saved in
 * fp32 (the backward's SwiGLU derivative takes them unrounded), h in bf16 (from the fp32 g, u) with
 * its bf16 residual. */
int qlora_moe_fwd(int qtype, const void* w_gu, const void* w_d, int E, int64_t H, int64_t I,
                  const void* X, int64_t T, int k, const int32_t* topk_idx, const float* topk_w,
                  const int32_t* offsets, const int32_t* perm, const int32_t* inv_perm,
                  const int32_t* mblk, const void* A_gu, const void* B_gu, const void* A_d,
                  const void* B_d, int r, float scale, void* Y, int y_dtype, void* saved,
                  size_t saved_bytes, void* ws, size_t ws_bytes, void* stream);

/* Backward. dY [T x H] bf16; saved from the forward. Writes dX [T x H] of dx_dtype (per-pair input
 * gradients stay fp32 up to the slot-ordered sum; d[g|u] enters the gate/up input-gradient GEMM in
 * bf16 and the adapter gradients as an fp32-accurate bf16 pair, like h), dA_gu [E][r][H], dB_gu [E][2I][r],
 * dA_d [E][r][I], dB_d [E][H][r] (fp32, overwritten; experts without tokens get zeros) and, if
 * d_logits is not NULL, the router-logit gradient [T x E] fp32 (zero off the selected experts). */
int qlora_moe_bwd(int qtype, const void* w_gu, const void* w_d, int E, int64_t H, int64_t I,
                  const void* X, const void* dY, int64_t T, int k, const int32_t* topk_idx,
                  const float* topk_w, const int32_t* offsets, const int32_t* perm,
                  const int32_t* inv_perm, const int32_t* mblk, const void* A_gu, const void* B_gu,
                  const void* A_d, const void* B_d, int r, float scale, const void* saved,
                  size_t saved_bytes, void* dX, int dx_dtype, float* dA_gu, float* dB_gu,
                  float* dA_d, float* dB_d, float* d_logits, void* ws, size_t ws_bytes,
                  void* stream);

/* ---------------------------------------------------------------------------------------------
 * Quantized lm_head with chunked cross-entropy ("Chunked cross entropy loss like Liger Kernel, which
 * works with MMQ", Show HN: LoRA over GGUF, "Things involved in the training"). W packed [V rows x K]
 * (a type the layer's GEMMs take), X [M x K] bf16 (the final hidden states), labels [M] int32 in
 * [0, V) or negative (ignored token). Rules: K % 256 == 0, V % 64 == 0.
 * Per chunk of `chunk` token rows: fp32 logits = X_c deq(W)^T in the workspace (the dequant GEMM,
 * no adapter); per row lse = log sum exp(logits), loss[m] = lse - logits[label] (0 if ignored); if
 * dX is not NULL, D = (softmax - onehot(label)) grad_scale in bf16 (zero rows for ignored tokens) and
 * dX_c = D deq(W) (dx_dtype): the gradient of grad_scale times the summed loss. The full [M x V]
 * logits never exist: the workspace holds one chunk's fp32 logits and bf16 D. */
size_t qlora_lm_head_ce_workspace_bytes(int64_t M, int64_t V, int64_t K, int64_t chunk);
int qlora_lm_head_ce(int qtype, const void* wq, int64_t V, int64_t K, const void* X, int64_t M,
                     const int32_t* labels, int64_t chunk, float grad_scale, float* loss, void* dX, int dx_dtype,
                     void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------------------
 * RMSNorm in front of the first projection (the recipe's Liger RMSNorm, Show HN: LoRA over GGUF,
 * "Things involved in the training"). X [M x K] bf16, gamma [K] bf16 (frozen), K % 8 == 0.
 * Forward: rstd[m] = 1 / sqrt(mean_k X[m][k]^2 + eps) (fp32), Xn = bf16(X rstd gamma) [M x K]: the
 * bf16 input of qlora_linear_fwd / qlora_linear_bwd. One pass per row (a warp per row).
 * Backward: dX = rstd gamma d - (rstd^3 X / K) sum_k X gamma d, d = dXn [M x K] (dxn_dtype, e.g. the
 * dX of qlora_linear_bwd) -> dX of dx_dtype. gamma is not trained (no gradient for it). */
int qlora_rmsnorm_fwd(const void* X, const void* gamma, int64_t M, int64_t K, float eps, void* Xn, float* rstd,
                      void* stream);
int qlora_rmsnorm_bwd(const void* X, const void* gamma, const float* rstd, const void* dXn, int dxn_dtype,
                      int64_t M, int64_t K, void* dX, int dx_dtype, void* stream);

/* ---------------------------------------------------------------------------------------------
 * 8-bit AdamW step on the adapter parameters (the recipe's bitsandbytes 8-bit AdamW optimizer,
 * Show HN: LoRA over GGUF, "Things involved in the training"): AdamW with decoupled weight decay
 * whose moments are kept in 8 bits, block-wise.
 *   p        [n] fp32 master parameters, updated in place
 *   grad     [n] fp32 gradient (e.g. dA or dB of this layer)
 *   m_q, v_q [n] uint8 codes of the first and second moment; m_absmax, v_absmax [ceil(n / 256)] fp32
 *            scales, one per block of 256 values; all four updated in place. Zeros everywhere is the
 *            state before the first step.
 *   step     t >= 1 (the bias corrections use 1 - beta^t)
 *   p_bf16   [n] bf16 (nullable): receives the updated parameters rounded to bf16 (the layer's A, B)
 * Update, in fp32: m = b1 m + (1 - b1) g; v = b2 v + (1 - b2) g^2;
 *   p = p - lr (m / c1 / (sqrt(v / c2) + eps) + weight_decay p), c1 = 1 - b1^t, c2 = 1 - b2^t.
 * A code q of a block with scale a stands for a * T[q]. T is the dynamic tree table: after the sign
 * bit (m only), E zero bits give the decade 10^-E, then an indicator bit, then B bits F of linear
 * fraction: |T| = (0.1 + 0.9 (F + 1/2) / 2^B) / 10^E; no indicator codes 0. After the update each
 * block's scale is max |value| over the block and each value takes the code of the nearest entry to
 * value / scale (equal distances: the smaller entry). No workspace; one launch. */
int qlora_adamw8_step(float* p, const float* grad, uint8_t* m_q, float* m_absmax, uint8_t* v_q, float* v_absmax,
                      int64_t n, float lr, float beta1, float beta2, float eps, float weight_decay, int64_t step,
                      void* p_bf16, void* stream);

/* Forward without allocation (no counterpart in the method's sources; a convenience of this
 * library). Same arguments, results and rules as qlora_linear_fwd, minus (ws, ws_bytes).
 *
 * For callers that cannot allocate device memory: code running where every byte of the device
 * pool is already owned by a caching allocator, or where a cudaMalloc (which can synchronise the
 * whole device) is not acceptable, and that therefore cannot hand this library a workspace.
 * Instead of a workspace it uses one static device array of 4 MiB that the library image itself
 * reserves on every device that loads it (held until the process exits). It holds the two adapter
 * operands, roundup256(2*KL*M) + roundup256(2*KL*N) bytes with KL = 64 for r <= 32 and 128 for
 * r <= 64 (about M + N <= 32768 at r <= 32, M + N <= 16384 at r <= 64); sizes that do not fit
 * return QL_ERR_WORKSPACE before any launch.
 * It calls no allocation routine of any kind.
 *
 * The first call in each context (per device) looks up the array's device address
 * (cudaGetSymbolAddress) while that device is current, and looks it up again when a call finds
 * another context current (after a device reset the library image is loaded anew and the array
 * may move); make the first call in a context before any stream capture. All calls on a device
 * share the one array and leave their operands in it: two calls whose kernels overlap on the GPU
 * (different streams, no ordering between them) race on it and may produce wrong results; calls
 * on one stream, or otherwise ordered, are fine. Each call rewrites everything it reads.
 * It always runs the tensor-core GEMM without a K split (the split's fp32 partials would not fit
 * the array), also where qlora_linear_fwd would take the small-M weight stream or a K split, so
 * decode-shaped calls (a few tokens) are slower here than through qlora_linear_fwd. */
int qlora_linear_fwd_noalloc(int qtype, const void* wq, int64_t N, int64_t K, const void* X, int64_t M,
                             const void* A, const void* B, int r, float scale, void* Y, int y_dtype,
                             float* H, void* stream);

#if defined(__GNUC__)
#pragma GCC visibility pop
#endif
#ifdef __cplusplus
}
#endif
#endif /* QLORA_H */
