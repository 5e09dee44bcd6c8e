/*
 * rz.h -- C ABI of librz: batch-invariant token logprobs and the REINFORCE Zero
 * loss / gradient on one NVIDIA B200 (sm_100a).
 *
 * What the library computes is defined on the page "vLLM says aligned kernels make
 * asynchronous RL stable at lag 64" (ainewsbites.com), section "REINFORCE Zero removes
 * the mismatch first", and the batch-invariance contract on "vLLM Train-Inference
 * Consistency Release Notes" (agentlenshq.com), section "Achieving Bitwise Consistency":
 *
 *   z[t,v]  = sum_k H[t,k] W[v,k]                      (LM head, no bias, temperature 1)
 *   lse[t]  = log sum_v exp z[t,v];   lp[t] = z[t, y_t] - lse[t]
 *   w_t     = exp(lp[t] - lp_rollout[t])               (unclipped importance ratio)
 *   A_i     = r_i - mean_{j in group(i)} r_j           (group-mean advantage)
 *   loss    = -(1/N) sum_i (A_i / L_i) sum_{t in i} w_t (token mean per response, N responses)
 *   kappa_t = -A_i w_t / (N L_i) = d loss / d lp_t
 *   dZ[t,v] = kappa_t ([v == y_t] - exp(z[t,v] - lse[t]))
 *   dH      = dZ W,   dW = dZ^T H
 *
 * Batch invariance: the bits of lp[t] and lse[t] depend only on (H[t,:], y_t, W), never
 * on n_tok, on the row's position, on the other rows of the call, or on how a sequence
 * is split into calls (prefill chunks vs one-token decode calls).  rz_loss_fwd_bwd's
 * lp_out is bitwise equal to rz_token_logprobs' lp_out for the same rows.  All outputs
 * are deterministic: the same call on the same inputs gives the same bits.
 *
 * Conventions for every entry point:
 *   - Array pointers are DEVICE pointers owned by the caller, dense row-major, and must
 *     not alias one another (outputs never alias inputs).
 *   - bf16 arrays are passed as their 16-bit patterns (rz_bf16 = uint16_t).
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls enqueue work
 *     on it and return without synchronising; argument checks happen on the host first
 *     and, on error, nothing is enqueued.
 *   - `workspace` is caller-allocated device memory of at least the size the matching
 *     rz_workspace_bytes_* query returns, 256-byte aligned.  Its first word is the
 *     device status of the most recent call that used it (read with
 *     rz_read_device_status).  A workspace must not be shared by calls that may run
 *     concurrently.  The library allocates no memory.
 *   - Shapes: d % 64 == 0 (64 <= d <= 32768); 1 <= V <= 2^31 - 1; 0 <= n_tok < 2^31.
 *     H, W, dH, dW must be 16-byte aligned; other arrays 4-byte aligned (8 for int64).
 *   - Device-checked inputs (a violation sets a bit of the device status and never
 *     traps): 0 <= token_ids[t] < V (the row's lp becomes NaN); seg_offsets[0] = 0,
 *     seg_offsets strictly increasing, seg_offsets[n_resp] = n_tok; 0 <= group_ids < n_groups.
 *     After a failed device check the loss path's outputs carry no meaning: a NaN logprob
 *     or coefficient spreads into its response's kappa, the loss, its dH rows and all of
 *     dW.  Read the status (rz_read_device_status) before using them.
 */
#ifndef RZ_H_
#define RZ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t rz_bf16; /* bit pattern of a bfloat16 value */

typedef enum {
  RZ_OK = 0,
  RZ_ERR_INVALID_ARG = 1,         /* null pointer, bad size, misaligned pointer            */
  RZ_ERR_UNSUPPORTED_SHAPE = 2,   /* d not a multiple of 64, or a size beyond the limits  */
  RZ_ERR_WORKSPACE_TOO_SMALL = 3, /* ws_bytes below the rz_workspace_bytes_* query         */
  RZ_ERR_CUDA = 4,                /* a CUDA runtime/driver call failed (launch, memset…)   */
  RZ_ERR_DEVICE_CHECK = 5,        /* device-side input check failed (ids, segments, groups)*/
  RZ_ERR_DEVICE_TIMEOUT = 6       /* a kernel wait gave up (bounded wait limit reached)    */
} rz_status;

/* Device status bits (the first int32 of a workspace). */
#define RZ_DEV_BAD_TOKEN_ID 1
#define RZ_DEV_BAD_SEGMENTS 2
#define RZ_DEV_BAD_GROUP_ID 4
#define RZ_DEV_WAIT_TIMEOUT 8

/* Human-readable name of a status code (static storage, never NULL). */
const char* rz_status_string(rz_status s);

/* Workspace bytes for rz_token_logprobs(n_tok, d, V); 0 if the shape is unsupported. */
size_t rz_workspace_bytes_logprobs(int64_t n_tok, int32_t d, int32_t V);

/* Workspace bytes for rz_loss_fwd_bwd; 0 if the shape is unsupported. */
size_t rz_workspace_bytes_loss(int64_t n_tok, int32_t n_resp, int32_t n_groups, int32_t d, int32_t V);

/* Workspace bytes for rz_segment_loss; 0 if the sizes are unsupported. */
size_t rz_workspace_bytes_segment_loss(int64_t n_tok, int32_t n_resp, int32_t n_groups);

/*
 * Token logprobs (the learner's own probability of each sampled token; page
 * "vLLM says aligned kernels…", section "REINFORCE Zero removes the mismatch first").
 *
 *   H          [n_tok, d] bf16   final hidden states
 *   W_head     [V, d]     bf16   LM head (nn.Linear weight layout, no bias)
 *   token_ids  [n_tok]    int32  sampled tokens
 *   lp_out     [n_tok]    fp32   out: lp[t] = z[t,y_t] - lse[t]
 *   lse_out    [n_tok]    fp32   out, nullable: log-sum-exp of row t's logits
 *
 * Logits are never written to memory: a fused tensor-core kernel computes H W^T tile by
 * tile and keeps an online log-sum-exp per row over fixed vocabulary segments, then a
 * second kernel merges the segments in fixed order.  A call of few rows (too few row blocks
 * to occupy the GPU with one unit per segment) runs one unit per 256-column tile and the
 * merge replays the same per-tile folds: the bits are the same either way.  n_tok == 0 is
 * a no-op.
 */
rz_status rz_token_logprobs(const rz_bf16* H, const rz_bf16* W_head, const int32_t* token_ids, int64_t n_tok,
                            int32_t d, int32_t V, float* lp_out, float* lse_out, void* workspace,
                            size_t ws_bytes, void* stream);

/*
 * Forward, REINFORCE Zero loss and backward in one call.
 *
 *   H, W_head, token_ids  as in rz_token_logprobs
 *   lp_rollout [n_tok]      fp32   logprobs the rollout recorded for the same tokens
 *   rewards    [n_resp]     fp32   one reward per response
 *   seg_offsets[n_resp+1]   int64  response i owns tokens seg_offsets[i] .. seg_offsets[i+1]-1
 *   group_ids  [n_resp]     int32  group of each response, in [0, n_groups)
 *   loss       [1]          fp32   out: the scalar loss (to be minimised)
 *   dH         [n_tok, d]   bf16   out: d loss / d H
 *   dW         [V, d]       fp32   out: d loss / d W_head (overwritten, not accumulated)
 *   lp_out     [n_tok]      fp32   out, nullable: token logprobs (bitwise equal to
 *                                   rz_token_logprobs on the same rows)
 *   kappa_out  [n_tok]      fp32   out, nullable: kappa_t = d loss / d lp_t
 *
 * The gradient of the ratio surrogate is exact; it equals the REINFORCE gradient with
 * the ratio w_t held constant.  No clipping, no value model, no rejection gates.
 * Requires n_tok >= 1, n_resp >= 1, n_groups >= 1.
 */
rz_status rz_loss_fwd_bwd(const rz_bf16* H, const rz_bf16* W_head, const int32_t* token_ids,
                          const float* lp_rollout, const float* rewards, const int64_t* seg_offsets,
                          const int32_t* group_ids, int64_t n_tok, int32_t n_resp, int32_t n_groups, int32_t d,
                          int32_t V, float* loss, rz_bf16* dH, float* dW, float* lp_out, float* kappa_out,
                          void* workspace, size_t ws_bytes, void* stream);

/*
 * The loss stage alone, from logprobs the caller already has (same definitions and the
 * same kernels rz_loss_fwd_bwd uses after its forward).
 *
 *   lp, lp_rollout [n_tok] fp32;  rewards, seg_offsets, group_ids as above
 *   loss       [1]     fp32  out
 *   kappa_out  [n_tok] fp32  out: -A_i w_t / (N L_i)
 *   w_out      [n_tok] fp32  out, nullable: unclipped ratio exp(lp - lp_rollout)
 */
rz_status rz_segment_loss(const float* lp, const float* lp_rollout, const float* rewards,
                          const int64_t* seg_offsets, const int32_t* group_ids, int64_t n_tok, int32_t n_resp,
                          int32_t n_groups, float* loss, float* kappa_out, float* w_out, void* workspace,
                          size_t ws_bytes, void* stream);

/*
 * Variants of the loss stage: the baselines the pages contrast REINFORCE Zero with
 * ("vLLM says aligned kernels…", sections "REINFORCE Zero removes the mismatch first" and
 * "Zero mismatch expands to newer models"), plus a global response count for
 * data-parallel shards.  A NULL options pointer, or flags == 0 with n_resp_total == 0,
 * gives exactly (bit for bit) rz_loss_fwd_bwd / rz_segment_loss.
 *
 *   kappa_t = -A_i * s_i * m_t * g(w_t) / (N * L_i),   loss = sum_t kappa_t
 *
 *   RZ_LOSS_CLIP_IS    g(w) = min(w, clip_max) (clip_max > 0): truncated importance
 *                      weights, used as a constant coefficient of the token's gradient
 *                      (the reported loss is the same sum with the capped weights).
 *   RZ_LOSS_SEQ_GATE   s_i = 1 iff gate_lo <= exp(mean over the counted tokens of response i
 *                      of (lp - lp_rollout)) <= gate_hi, else 0; a rejected response keeps
 *                      its reward in its group's mean and stays counted in N.
 *                      rz_loss_fwd_bwd_ex then runs the forward twice (the gate needs every
 *                      logprob before any kappa).
 *   RZ_LOSS_TOKEN_MASK m_t = token_mask[t] != 0 (device [n_tok] bytes, 4-byte aligned);
 *                      L_i counts only the tokens with m_t = 1 (a response with none
 *                      contributes nothing).
 *   n_resp_total > 0   N = n_resp_total instead of n_resp.
 * Invalid options (unknown flag bits, clip_max <= 0, gate_lo > gate_hi, a missing mask,
 * n_resp_total < 0) return RZ_ERR_INVALID_ARG.
 */
#define RZ_LOSS_CLIP_IS 1
#define RZ_LOSS_SEQ_GATE 2
#define RZ_LOSS_TOKEN_MASK 4

typedef struct {
  int32_t flags;
  float clip_max;
  double gate_lo, gate_hi;
  const uint8_t* token_mask;
  int32_t n_resp_total;
} rz_loss_options;

/* rz_loss_fwd_bwd with loss-stage options (same workspace size). */
rz_status rz_loss_fwd_bwd_ex(const rz_bf16* H, const rz_bf16* W_head, const int32_t* token_ids,
                             const float* lp_rollout, const float* rewards, const int64_t* seg_offsets,
                             const int32_t* group_ids, int64_t n_tok, int32_t n_resp, int32_t n_groups, int32_t d,
                             int32_t V, const rz_loss_options* options, float* loss, rz_bf16* dH, float* dW,
                             float* lp_out, float* kappa_out, void* workspace, size_t ws_bytes, void* stream);

/*
 * rz_loss_fwd_bwd_ex with the hidden states read from HOST memory, the copy overlapped with
 * the compute.  The call enqueues on a copy stream of its own (one per device, created on
 * first use) one cudaMemcpyAsync per 16384-token chunk of H_host into H_dev, and each
 * chunk's kernels on `stream` wait for that chunk's copy only, so the copy of chunk c + 1
 * runs while chunk c computes.  The copies begin after all work already enqueued on
 * `stream` (which may still be reading H_dev).  With RZ_LOSS_SEQ_GATE the first forward
 * pass waits for every chunk.
 *
 *   H_host  host, [n_tok, d] bf16 row-major; pinned (cudaHostAlloc / cudaHostRegister) for
 *           the copies to overlap (pageable memory works, without overlap).  Must stay
 *           unchanged until the call's work on `stream` has finished.
 *   H_dev   device, [n_tok, d] bf16, 16-byte aligned, caller-owned; on return of the work
 *           it holds a copy of H_host.
 *   every other argument as rz_loss_fwd_bwd_ex (device pointers, same workspace size).
 * Errors: as rz_loss_fwd_bwd_ex, plus RZ_ERR_INVALID_ARG for a null H_host and RZ_ERR_CUDA
 * when the copy stream, its event or a copy cannot be created or enqueued (nothing of the
 * compute is enqueued past that point).
 */
rz_status rz_loss_fwd_bwd_streamed(const rz_bf16* H_host, rz_bf16* H_dev, const rz_bf16* W_head,
                                   const int32_t* token_ids, const float* lp_rollout, const float* rewards,
                                   const int64_t* seg_offsets, const int32_t* group_ids, int64_t n_tok,
                                   int32_t n_resp, int32_t n_groups, int32_t d, int32_t V,
                                   const rz_loss_options* options, float* loss, rz_bf16* dH, float* dW,
                                   float* lp_out, float* kappa_out, void* workspace, size_t ws_bytes, void* stream);

/*
 * rz_loss_fwd_bwd_streamed with the gradients also delivered to HOST memory: the whole step
 * from host inputs to host results, for a trainer that keeps activations and gradients in
 * host memory.  On top of the streamed call, each 16384-token chunk's rows of dH are copied
 * to dH_host right after that chunk's dH contraction (on a device-to-host stream of its own,
 * one per device, created on first use, so the copy of chunk c overlaps the compute of
 * chunk c + 1 and the host-to-device copy of the next chunk's H), and dW to dW_host after
 * the last chunk's dW contraction.  Every copy is finished before any work enqueued on
 * `stream` after this call starts, so a stream synchronisation after the call means the
 * host buffers hold the results.
 *
 *   dH_host  host, [n_tok, d] bf16, nullable (no dH copy); pinned for the copies to overlap
 *   dW_host  host, [V, d] fp32, nullable (no dW copy); pinned for the copy to run asynchronously
 *   every other argument as rz_loss_fwd_bwd_streamed (dH and dW still receive the device copies).
 * Errors: as rz_loss_fwd_bwd_streamed, plus RZ_ERR_CUDA when the device-to-host stream, its
 * event or a copy cannot be created or enqueued.
 */
rz_status rz_loss_fwd_bwd_host_io(const rz_bf16* H_host, rz_bf16* H_dev, const rz_bf16* W_head,
                                  const int32_t* token_ids, const float* lp_rollout, const float* rewards,
                                  const int64_t* seg_offsets, const int32_t* group_ids, int64_t n_tok, int32_t n_resp,
                                  int32_t n_groups, int32_t d, int32_t V, const rz_loss_options* options,
                                  float* loss, rz_bf16* dH, float* dW, float* lp_out, float* kappa_out,
                                  rz_bf16* dH_host, float* dW_host, void* workspace, size_t ws_bytes, void* stream);

/* rz_segment_loss with loss-stage options (same workspace size). */
rz_status rz_segment_loss_ex(const float* lp, const float* lp_rollout, const float* rewards,
                             const int64_t* seg_offsets, const int32_t* group_ids, int64_t n_tok, int32_t n_resp,
                             int32_t n_groups, const rz_loss_options* options, float* loss, float* kappa_out,
                             float* w_out, void* workspace, size_t ws_bytes, void* stream);

/*
 * Diagnostics of the ratio w_t = exp(lp_t - lp_rollout_t) over the counted tokens
 * (token_mask nullable) — the pages' observables: the importance-weight deviation peak
 * against its median ("vLLM says aligned kernels…", section "Asynchronous training has two
 * different gaps") and the rollout-to-learner KL (section "Reported results include 2.40
 * times higher throughput").
 *
 *   stats_out [9] fp64, device: k1 = mean(lp_rollout - lp), k2 = mean((lp - lp_rollout)^2/2),
 *             k3 = mean(w - 1 - (lp - lp_rollout)), min w, max w, max |w - 1|, the exact
 *             lower median of |w - 1| (rank floor((m-1)/2) of the m counted tokens), their
 *             ratio (peak / median), m
 *   resp_mean_ratio_out [n_resp] fp32, device, nullable: mean w over each response's counted
 *             tokens (0 if none)
 * Deterministic; w is computed exactly as the loss stage computes it.
 */
size_t rz_workspace_bytes_ratio_stats(int64_t n_tok, int32_t n_resp);
rz_status rz_ratio_stats(const float* lp, const float* lp_rollout, const int64_t* seg_offsets, int64_t n_tok,
                         int32_t n_resp, const uint8_t* token_mask, double* stats_out, float* resp_mean_ratio_out,
                         void* workspace, size_t ws_bytes, void* stream);

/*
 * Frobenius norms of the gradients: norms_out[0] = ||dH|| (bf16 [n_tok, d]),
 * norms_out[1] = ||dW|| (fp32 [V, d]), fp64, device; fixed-order reductions (deterministic).
 * The pages report the peak pre-clipping gradient norm ("vLLM says aligned
 * kernels…", section "Reported results include 2.40 times higher throughput").
 */
size_t rz_workspace_bytes_grad_norms(void);
rz_status rz_grad_norms(const rz_bf16* dH, const float* dW, int64_t n_tok, int32_t d, int32_t V, double* norms_out,
                        void* workspace, size_t ws_bytes, void* stream);

/*
 * Low-precision forward: token logprobs from e4m3 (fp8) operands with per-row scales, the
 * pages' reduced-precision arithmetic on the rollout side ("vLLM Train-Inference Consistency
 * Release Notes", section "The Technical Challenge"; "vLLM says aligned kernels…", section
 * "Zero mismatch expands to newer models": FP8 weights), under the same batch-invariance
 * contract as rz_token_logprobs.
 *
 *   rz_quantize_rows_e4m3: X [rows, d] bf16 -> X8 [rows, d] e4m3 bytes and scale [rows] fp32,
 *     scale = max|x| / 448 (1 for an all-zero row), X8 = e4m3(x / scale), round to nearest
 *     even, saturating (both divisions IEEE fp32).
 *   rz_token_logprobs_fp8: z[t,v] = h_scale[t] * y[t,v], y[t,v] = (sum_k H8[t,k] W8[v,k]) *
 *     w_scale[v] (e4m3 x e4m3 products accumulated in fp32 on the tensor cores, then the
 *     column scale, one fp32 rounding); the row scale (positive) enters the log-sum-exp as
 *     exp(z - max z) = 2^((y - max y) * h_scale[t] * log2 e), and lp = h_scale[t] * y[t,y_t] - lse;
 *     lse as rz_token_logprobs.  d must be a multiple of 128; w_scale needs 4-byte
 *     alignment (16 bytes for the fastest loads); workspace size =
 *     rz_workspace_bytes_logprobs(n_tok, d, V).
 */
rz_status rz_quantize_rows_e4m3(const rz_bf16* X, int64_t rows, int32_t d, uint8_t* X8, float* scale, void* stream);
rz_status rz_token_logprobs_fp8(const uint8_t* H8, const float* h_scale, const uint8_t* W8, const float* w_scale,
                                const int32_t* token_ids, int64_t n_tok, int32_t d, int32_t V, float* lp_out,
                                float* lse_out, void* workspace, size_t ws_bytes, void* stream);

/*
 * MXFP4 forward: token logprobs from OCP Microscaling MXFP4 operands (the FP4 weights with
 * block scales of "vLLM says aligned kernels…", section "Zero mismatch expands to newer
 * models"), the block-scaled products on the tensor cores, under the same batch-invariance
 * contract as rz_token_logprobs (same vocabulary segments and per-row log-sum-exp).
 *
 *   Format: each row is cut into 32-element blocks along d; a block's scale is 2^X stored as
 *   the byte X + 127 (UE8M0), X = floor(log2 max|x|) - 2 clamped to [-127, 127] (-127 for an
 *   all-zero block); each element is the E2M1 value (0, 0.5, 1, 1.5, 2, 3, 4, 6 with a sign)
 *   nearest to x / 2^X, ties to the even code, saturating at 6.
 *   codes  [rows, d/2] bytes: element 2j in the low nibble of byte j, element 2j+1 in the high one.
 *   scales rz_mxfp4_scale_bytes(rows, d) bytes, tiled: the scale of row r, block k (columns
 *          32k .. 32k+31) is byte ((r/128)*(d/128) + k/4)*512 + (r%32)*16 + ((r%128)/32)*4 + k%4;
 *          rows are padded with zero bytes to a multiple of 256.
 *   d must be a multiple of 256 (256 <= d <= 32768).
 *
 *   rz_mxfp4_scale_bytes: size of the tiled scale array of `rows` rows (0 for an unsupported d).
 *   rz_quantize_rows_mxfp4: X [rows, d] bf16 -> codes X4 and tiled scales (16-byte aligned X, X4).
 *   rz_token_logprobs_mxfp4: z[t,v] = sum_k decode(H4)[t,k] decode(W4)[v,k] (exact products,
 *     fp32 accumulation on the tensor cores), lp and lse as rz_token_logprobs; scale arrays
 *     16-byte aligned; workspace size = rz_workspace_bytes_logprobs(n_tok, d, V).
 */
size_t rz_mxfp4_scale_bytes(int64_t rows, int32_t d);
rz_status rz_quantize_rows_mxfp4(const rz_bf16* X, int64_t rows, int32_t d, uint8_t* X4, uint8_t* scales,
                                 void* stream);
rz_status rz_token_logprobs_mxfp4(const uint8_t* H4, const uint8_t* h_scales, const uint8_t* W4,
                                  const uint8_t* w_scales, const int32_t* token_ids, int64_t n_tok, int32_t d,
                                  int32_t V, float* lp_out, float* lse_out, void* workspace, size_t ws_bytes,
                                  void* stream);

/*
 * Cross-GPU consistency ("vLLM Train-Inference Consistency Release Notes", section
 * "Achieving Bitwise Consistency": communication reductions that do not vary with timing
 * or scheduling).  The reduction step of a data-parallel all-reduce of dW:
 *   out[i] = sum_{r = 0 .. nshards-1} stacked[r * count + i]
 * in rank order, accumulated in fp64 and rounded once, so the result is the same bits on
 * every rank whatever collective moved the shards.  stacked [nshards, count] fp32 and out
 * [count] fp32 are device arrays; used after an all-to-all that gives each rank its slice
 * from every rank, before an all-gather (invariant_logprobs_reinforce_b200.dp).
 */
rz_status rz_sum_shards_f32(const float* stacked, int32_t nshards, int64_t count, float* out, void* stream);

/*
 * Self-test of the bounded waits: every mbarrier wait in this library gives up after a time
 * limit (4 s in the kernels) instead of spinning forever, sets RZ_DEV_WAIT_TIMEOUT in the
 * status word and lets the kernel exit normally.  This launches one thread that waits, with
 * limit_ns (at most 10 s), on a barrier nothing arrives on.  Afterwards
 * rz_read_device_status(workspace) reports RZ_ERR_DEVICE_TIMEOUT; waited_ns_out (host,
 * nullable; when given the call synchronises the stream) receives the time waited.
 * workspace: at least 256 bytes, 256-byte aligned.
 */
rz_status rz_selftest_wait_timeout(uint64_t limit_ns, void* workspace, size_t ws_bytes, uint64_t* waited_ns_out,
                                   void* stream);

/* Kernel kinds reported per launch by rz_loss_fwd_bwd_timed. */
#define RZ_KERNEL_LMHEAD_LSE 0    /* fused LM head + online log-sum-exp + gather (tensor cores) */
#define RZ_KERNEL_MERGE_LSE 1     /* fixed-order merge of the vocabulary-segment partials       */
#define RZ_KERNEL_RESPONSE_COEF 2 /* loss setup: checks, group means, -A_i / (N L_i), block starts */
#define RZ_KERNEL_TOKEN_KAPPA 3   /* ratio and kappa per token, loss partials; the call's last
                                     block also sums the partials into the loss                 */
#define RZ_KERNEL_LOSS_FINAL 4    /* not reported: the loss is summed inside RZ_KERNEL_TOKEN_KAPPA */
#define RZ_KERNEL_DZ 5            /* kept exponentials -> dZ chunk in place (HBM pass)           */
#define RZ_KERNEL_DH 6            /* dH chunk = dZ W (tensor cores)                              */
#define RZ_KERNEL_DW 7            /* dW (+)= dZ^T H (tensor cores)                               */
#define RZ_KERNEL_BLOCK_FIRST 8   /* not reported: the block starts come from RZ_KERNEL_RESPONSE_COEF */

/* Number of launches rz_loss_fwd_bwd_timed records for n_tok tokens (0 if n_tok < 1): the
 * loss setup, then six per 16384-token chunk (forward, merge, kappa, dZ, dH, dW). */
int32_t rz_num_launches_loss(int64_t n_tok);

/*
 * rz_loss_fwd_bwd with per-launch timing: identical arguments and results, plus
 *   launch_events [2*capacity] cudaEvent_t created by the caller (timing enabled); the
 *                  library records events[2i] before and events[2i+1] after launch i
 *                  on `stream`
 *   launch_kinds  [capacity] host int32, out: RZ_KERNEL_* kind of launch i
 *   n_launches    host int32, out: launches recorded (at most capacity)
 * Launches past `capacity` still run but are not recorded.
 */
rz_status rz_loss_fwd_bwd_timed(const rz_bf16* H, const rz_bf16* W_head, const int32_t* token_ids,
                                const float* lp_rollout, const float* rewards, const int64_t* seg_offsets,
                                const int32_t* group_ids, int64_t n_tok, int32_t n_resp, int32_t n_groups,
                                int32_t d, int32_t V, float* loss, rz_bf16* dH, float* dW, float* lp_out,
                                float* kappa_out, void* workspace, size_t ws_bytes, void* stream,
                                void* const* launch_events, int32_t* launch_kinds, int32_t capacity,
                                int32_t* n_launches);

/* Size of the library-owned scratch array used by rz_token_logprobs_noalloc (32 MiB). */
#define RZ_NOALLOC_SCRATCH_BYTES (32u << 20)

/*
 * rz_token_logprobs without a caller workspace and without any allocation.
 *
 * The pages have no counterpart to this call; it exists for callers that cannot
 * allocate device memory: a rollout or serving engine that reserved nearly all of HBM
 * for its KV cache at start-up and hands out only fixed buffers, a latency-critical
 * loop where cudaMalloc/cudaFree could synchronise the device, or a plugin that receives
 * device pointers from a host framework but has no access to its allocator.
 *
 * Arguments and results are those of rz_token_logprobs (same kernels, same bits), minus
 * the workspace.  The scratch is a fixed array of RZ_NOALLOC_SCRATCH_BYTES inside the
 * library, held by every GPU that loads the library until the process exits.  A call
 * needs 256 + 4*n_tok*(2*C + 1) bytes of it (rounded up to 256-byte pieces), C =
 * ceil(V/2048), or C = ceil(V/256) for a call of few rows (ceil(n_tok/128)*ceil(V/2048) <
 * 296): at V = 151936 that is about 55,000 tokens per call.  Larger calls return
 * RZ_ERR_WORKSPACE_TOO_SMALL and enqueue nothing; split them into several calls.
 *
 * The first call on each device looks up the scratch address (cudaGetSymbolAddress)
 * and caches it with the device's CUDA context; make that first call before any stream
 * capture begins.  If the context is destroyed and recreated (cudaDeviceReset, or a
 * released primary context), the next call sees the new context and looks the address
 * up again, so make that call outside a capture as well.  The device that is current when
 * the call is made must be the one that holds H, W_head, token_ids and the outputs, and
 * `stream` must belong to it.  All calls share the one array: calls whose GPU work can
 * overlap (different streams, or different host threads) race on it and must be
 * serialised by the caller.  Each call clears the scratch's status word.  The status word
 * is internal (rz_read_device_status does not apply), so problems show in the outputs:
 * an out-of-range token id gives that row a NaN logprob, and a kernel wait that gave up
 * gives NaN in every lp and lse of the call.  Nothing here calls cudaMalloc, cudaFree or
 * any allocating routine.
 */
rz_status rz_token_logprobs_noalloc(const rz_bf16* H, const rz_bf16* W_head, const int32_t* token_ids,
                                    int64_t n_tok, int32_t d, int32_t V, float* lp_out, float* lse_out,
                                    void* stream);

/*
 * Self-test of what a forward call returns after one of its waits gave up.  Runs
 * rz_token_logprobs on `workspace` (use_noalloc_scratch == 0) or rz_token_logprobs_noalloc
 * (use_noalloc_scratch != 0; workspace and ws_bytes are ignored) with one extra bounded
 * wait, on a barrier nothing arrives on and with a 1 ms limit, enqueued right after the
 * call clears its status word.  That wait gives up and sets RZ_DEV_WAIT_TIMEOUT exactly as
 * a wait inside the forward's kernels would; the forward then runs normally and its merge,
 * seeing the bit, writes NaN to every lp_out and lse_out (nullable) element.  With a
 * workspace, rz_read_device_status then returns RZ_ERR_DEVICE_TIMEOUT.  Arguments, checks
 * and errors otherwise as the call it runs.  No GPU fault or hang is involved.
 */
rz_status rz_selftest_forward_after_timeout(int32_t use_noalloc_scratch, const rz_bf16* H, const rz_bf16* W_head,
                                            const int32_t* token_ids, int64_t n_tok, int32_t d, int32_t V,
                                            float* lp_out, float* lse_out, void* workspace, size_t ws_bytes,
                                            void* stream);

/*
 * Synchronises `stream`, then reads the device status word of `workspace`.
 * Returns RZ_OK, RZ_ERR_DEVICE_CHECK (bad ids / segments / groups),
 * RZ_ERR_DEVICE_TIMEOUT (a bounded wait gave up) or RZ_ERR_CUDA.
 * bits_out (nullable) receives the raw RZ_DEV_* bits.
 */
rz_status rz_read_device_status(const void* workspace, void* stream, int32_t* bits_out);

#ifdef __cplusplus
}
#endif

#endif /* RZ_H_ */
