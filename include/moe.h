/*
 * moe.h -- C ABI of the B200 (sm_100a) fused MoE expert layer.
 *
 * The layer replaces the for-loop over experts of Hugging Face MoE blocks
 * ("Integration of fused moe kernel (e.g., megablocks) for efficient moe
 * training", axolotl issue #3155, Feature description) with routed grouped
 * GEMMs:
 *
 *   logits [T,E] --moe_route--> top-k ids/weights --moe_permute--> counts,
 *   offsets, expert-sorted pair order, gathered rows Xp --moe_experts_fwd-->
 *   SwiGLU(gate/up) and down per expert segment, routing weight applied -->
 *   moe_combine --> Y [T,H];  moe_layer_bwd gives dX, dW_gate/up/down and
 *   d router logits.
 *
 * Notation: T tokens, H hidden size, E experts, k experts per token, I expert
 * intermediate size, P = T*k (token, expert) pairs. Pair id q = t*k + j where
 * j is the rank of the expert in token t's top-k (descending score). Row r of
 * every permuted buffer holds pair sorted_pair[r]; the rows of expert e are
 * [offsets[e], offsets[e+1]).
 *
 * Conventions shared by every call:
 *  - Memory: every pointer is a DEVICE pointer owned by the caller, row-major
 *    and contiguous, 16-byte aligned. The library allocates no device memory
 *    and keeps no pointer after a call returns; scratch space is the caller's
 *    `ws` buffer, sized by the matching *_workspace_bytes query.
 *  - Types: bf16 tensors are passed as moe_bf16 (the raw 16-bit pattern);
 *    index tensors are int32; weights/logits/gradients of the router are fp32.
 *  - Streams: each call only enqueues work on `stream` (NULL = legacy default
 *    stream) and returns without synchronising. Nothing is read back to the
 *    host; the per-expert counts never leave the device.
 *  - Errors: arguments are checked before anything is launched. A bad shape,
 *    a NULL required pointer or a pointer that is not 16-byte aligned returns
 *    MOE_ERR_INVALID_ARG, a workspace that is too small MOE_ERR_WORKSPACE, a
 *    device that is not sm_100 MOE_ERR_UNSUPPORTED, a failed launch
 *    MOE_ERR_CUDA. Problems found on the device (an expert id outside [0,E),
 *    segment bounds `offsets` given to a GEMM call that are not
 *    0 <= offsets[0] <= ... <= offsets[E] <= T*k, a pipeline wait that
 *    exceeded its time limit) are recorded in a device status word that
 *    moe_last_device_status reads; kernels never trap. A GEMM given such
 *    offsets computes no tile (a weight gradient is written as zeros).
 *  - Limits: 1 <= k <= E <= 1024, T >= 0 (T == 0 is a valid empty batch),
 *    T*k < 2^31, H and I positive multiples of 8 (16-byte rows).
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t moe_bf16;                 /* bfloat16 bit pattern */
typedef struct CUstream_st* moe_stream_t;  /* identical to cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,
  MOE_ERR_UNSUPPORTED = 2,
  MOE_ERR_WORKSPACE = 3,
  MOE_ERR_CUDA = 4,
  MOE_ERR_TIMEOUT = 5,
  MOE_ERR_DEVICE_CHECK = 6
} moe_status;

/* Number of kernels this library has launched (enqueued) in this process so
 * far, on every stream and device; a launch recorded into a CUDA graph counts
 * once, when it is captured. */
unsigned long long moe_launch_count(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* moe_status_str(int status);

/* Synchronises `stream`, then returns and clears the device status word of
 * the current device: MOE_OK, MOE_ERR_TIMEOUT (a kernel wait ran out and the
 * kernel unwound) or MOE_ERR_DEVICE_CHECK (an expert id outside [0,E) was
 * skipped, or a GEMM refused its segment bounds). MOE_ERR_CUDA if the
 * synchronisation itself failed. */
int moe_last_device_status(moe_stream_t stream);

/*
 * moe_route -- router softmax, top-k, renormalisation.
 * Source: fused-MoE Triton project summary (sourcepulse), Highlighted
 * Details ("fused softmax-topk"); "[WIP] Qwen3 MoE support" (torchtune PR
 * #2820), review comment: the top-k scores are divided by their sum + 1e-20.
 *
 *   p[t,:]       = softmax(logits[t,:])             (fp32)
 *   topk_idx[t,:] = the k experts with the largest logits, ordered by logit
 *                   descending, ties to the lower expert index (the set is
 *                   the top-k of p because softmax is increasing)
 *   topk_w[t,j]  = p[t,idx_j] / (sum_j' p[t,idx_j'] + 1e-20)
 *
 * logits   [T,E] fp32 in.      topk_idx [T,k] int32 out.
 * topk_w   [T,k] fp32 out.     probs    [T,E] fp32 out, or NULL to skip
 *                              (moe_layer_bwd needs it).
 */
int moe_route(const float* logits, int T, int E, int k, int32_t* topk_idx, float* topk_w, float* probs,
              moe_stream_t stream);

/* Bytes of workspace moe_permute needs for this problem size. */
size_t moe_permute_workspace_bytes(int T, int E, int k);

/*
 * moe_permute -- per-expert histogram, prefix sum and stable scatter that
 * sorts the P pairs by expert, plus the row gather Xp[r] = X[sorted_pair[r]/k].
 * Source: "[MoE] Improve moe kernels for unsloth fine tuning #3812", review
 * of the token-routing logic: counts = bincount(flat expert ids, minlength=E)
 * (one value per expert) and gather indices = stable argsort of the flat ids;
 * fused-MoE summary, How It Works: inputs sorted by expert.
 *
 * topk_idx    [T,k] int32 in (values in [0,E); others are skipped and flagged
 *             as MOE_ERR_DEVICE_CHECK in the device status word).
 * counts      [E] int32 out;  offsets [E+1] int32 out (exclusive prefix sum).
 * sorted_pair [P] int32 out: pair ids in expert order, ascending pair id
 *             within an expert (bit-identical to a stable argsort).
 * pair_pos    [P] int32 out: inverse permutation, pair_pos[sorted_pair[r]] = r.
 * X [T,H] bf16 in and Xp [P,H] bf16 out: the gather; both NULL to skip it
 *             (H is then ignored).
 * ws          >= moe_permute_workspace_bytes(T,E,k) bytes of device scratch.
 */
int moe_permute(const int32_t* topk_idx, int T, int E, int k, int32_t* counts, int32_t* offsets,
                int32_t* sorted_pair, int32_t* pair_pos, const moe_bf16* X, int H, moe_bf16* Xp, void* ws,
                size_t ws_bytes, moe_stream_t stream);

/* Bytes of workspace moe_route_permute needs for this problem size. */
size_t moe_route_permute_workspace_bytes(int T, int E, int k);

/*
 * moe_route_permute -- moe_route followed by moe_permute in two kernels
 * instead of five (plus the gather): the routing kernel also counts, per
 * chunk of 32 tokens, how many of the chunk's pairs chose each expert, and
 * one kernel turns those counts into counts/offsets and scatters the pairs.
 * Source: fused-MoE Triton project summary (sourcepulse), Highlighted
 * Details: softmax-topk fused with the expert indexing; the results are
 * defined by moe_route and moe_permute above and are bit-identical to
 * calling them in turn (topk_idx, topk_w, probs, counts, offsets,
 * sorted_pair, pair_pos, Xp).
 *
 * Arguments as in moe_route and moe_permute (probs may be NULL; X and Xp
 * both NULL skip the gather). ws >= moe_route_permute_workspace_bytes(T,E,k)
 * bytes of device scratch (one byte per expert, rounded up to 16, per chunk
 * of 32 tokens); MOE_ERR_WORKSPACE if smaller. Errors otherwise as the two
 * calls; nothing is launched when an argument is rejected.
 */
int moe_route_permute(const float* logits, int T, int E, int k, int32_t* topk_idx, float* topk_w, float* probs,
                      int32_t* counts, int32_t* offsets, int32_t* sorted_pair, int32_t* pair_pos,
                      const moe_bf16* X, int H, moe_bf16* Xp, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_permute_noalloc -- moe_permute without a workspace argument, for
 * callers that cannot allocate device memory: a host program or plug-in that
 * links only this library and has no device allocator of its own, or code
 * that must not call cudaMalloc (it synchronises the device). The pages have
 * no counterpart; this is a calling convenience of this library.
 *
 * Arguments and results are exactly those of moe_permute (same kernels).
 * The scratch comes from one fixed 1 MiB device array inside the library
 * (held on every GPU that loads the library until the process exits), so the
 * problem must satisfy ceil(T*k / 2048) * E <= 262144 (for E = 128: up to
 * 4,194,304 pairs); larger problems return MOE_ERR_WORKSPACE and launch
 * nothing. The first call on a device looks up that array's device address
 * (cudaGetSymbolAddress) with the device current. The address is kept for the
 * life of the process: after
 * cudaDeviceReset (or anything else that destroys and re-creates the device's
 * context) it is stale, so do not call this entry point again in that
 * process. All calls share the array: calls whose executions
 * overlap on the GPU (other streams or host threads on the same device) race
 * on it. Leftover contents from earlier calls are harmless: every value read
 * is written earlier in the same call.
 */
int moe_permute_noalloc(const int32_t* topk_idx, int T, int E, int k, int32_t* counts, int32_t* offsets,
                        int32_t* sorted_pair, int32_t* pair_pos, const moe_bf16* X, int H, moe_bf16* Xp,
                        moe_stream_t stream);

/*
 * moe_experts_fwd -- the two persistent grouped GEMMs over the expert
 * segments (tcgen05 tensor cores, TMEM accumulators, TMA-fed tiles; experts
 * with no rows cost nothing).
 * Source: fused-MoE summary, How It Works (grouped GEMM with persistent
 * workers over expert-sorted rows); unsloth PR #3812, stacked weight shapes
 * and the fused post-multiply by the routing weight ("fuse_mul_post").
 *
 *   gate/up:  g = Xp[r] W_gu[e,0:I]^T,  u = Xp[r] W_gu[e,I:2I]^T  (fp32 acc)
 *             h[r] = silu(g) * u  -> bf16          (SwiGLU in the epilogue)
 *   down:     O[r] = w_q * (h[r] W_d[e]^T)  -> bf16 (weight in the epilogue)
 *   with q = sorted_pair[r], w_q = topk_w[q] (topk_w NULL: w_q = 1).
 *
 * Xp [P,H] bf16 in; offsets [E+1], sorted_pair [P] int32 in (moe_permute).
 * W_gu [E,2I,H] bf16: rows 0..I-1 gate, I..2I-1 up (Linear [out,in] layout).
 * W_d  [E,H,I]  bf16.
 * h [P,I] bf16 out; gu_save [P,2I] bf16 out (g then u per row) or NULL;
 * O [P,H] bf16 out. Rows of Xp/h/O past P are never touched.
 */
int moe_experts_fwd(const moe_bf16* Xp, const int32_t* offsets, const int32_t* sorted_pair, const float* topk_w,
                    int T, int E, int k, int H, int I, const moe_bf16* W_gu, const moe_bf16* W_d, moe_bf16* h,
                    moe_bf16* gu_save, moe_bf16* O, moe_stream_t stream);

/*
 * moe_combine -- un-permute and sum each token's k results:
 *   Y[t] = sum_{j=0..k-1} O[pair_pos[t*k+j]], summed in fp32 in j order,
 *   rounded once to bf16.
 * Source: modelopt moe helpers, a2a_moe Flow (weight by the routing weights
 * and sum each token's top-k results; results return in the hidden dtype).
 * O [P,H] bf16 in; pair_pos [P] int32 in; Y [T,H] bf16 out.
 */
int moe_combine(const moe_bf16* O, const int32_t* pair_pos, int T, int k, int H, moe_bf16* Y,
                moe_stream_t stream);

/* Bytes of workspace moe_layer_bwd needs; recompute_gu != 0 adds room to
 * recompute the gate/up activations when gu_save is not available. */
size_t moe_layer_bwd_workspace_bytes(int T, int E, int k, int H, int I, int recompute_gu);

/*
 * moe_layer_bwd -- backward of route -> experts -> combine for upstream
 * gradient dY, with the top-k selection held constant. The pages give no
 * backward formulas; these are the derivatives of the forward above:
 *   dw_q      = <dY[t], h[r] W_d[e]^T>                  (d routing weight)
 *   dh[r]     = w_q * dY[t] W_d[e]
 *   du, dg    = dh*silu(g),  dh*u*s*(1+g*(1-s)), s = sigmoid(g)
 *   dW_d[e]   = sum_r (w_q dY[t])^T h[r];  dW_gu[e] = sum_r [dg;du]^T Xp[r]
 *   dX[t]     = sum_j [dg;du][pair_pos[t*k+j]] W_gu[e]
 *   dlogits   = softmax Jacobian of (renormalisation Jacobian of dw)
 * Experts with no rows get exactly zero dW.
 *
 * dY [T,H] bf16 in. Xp, offsets, sorted_pair, pair_pos, topk_idx, topk_w
 * and probs as produced by the forward calls. gu_save [P,2I] from
 * moe_experts_fwd, or NULL to recompute it (needs recompute_gu workspace).
 * h is not read (h = silu(g)*u is recomputed from g|u in the dgrad epilogue,
 * which saves its DRAM traffic); it may be NULL.
 * Outputs: dX [T,H] bf16, dW_gu [E,2I,H] bf16, dW_d [E,H,I] bf16,
 * dlogits [T,E] fp32. ws >= moe_layer_bwd_workspace_bytes(...).
 */
int moe_layer_bwd(const moe_bf16* dY, const moe_bf16* Xp, const moe_bf16* gu_save, const moe_bf16* h,
                  const float* probs, const int32_t* topk_idx, const float* topk_w, const int32_t* offsets,
                  const int32_t* sorted_pair, const int32_t* pair_pos, int T, int E, int k, int H, int I,
                  const moe_bf16* W_gu, const moe_bf16* W_d, moe_bf16* dX, moe_bf16* dW_gu, moe_bf16* dW_d,
                  float* dlogits, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Expert parallelism: the experts are split over ranks in contiguous blocks of
 * experts_per_rank; each (token, expert) pair's row travels to the expert's
 * owner, is computed there with moe_permute / moe_experts_fwd /
 * moe_layer_bwd_pair_dw and comes back. The transport between ranks is the
 * caller's (all-to-all); these calls prepare and finish the rows around it.
 * Source: modelopt `moe` helpers, a2a_moe Flow: the pairs are expanded and
 * sent to the experts, and the results come back to be weighted by the
 * routing weights and summed per token.
 *
 * moe_ep_pack_rows -- for every expert-sorted row r (the rows of expert e are
 * [offsets[e], offsets[e+1]) of a permutation made by moe_permute):
 *   local_expert[r] = e % experts_per_rank  (its expert's index on the owner)
 *   row_w[r]        = topk_w[sorted_pair[r]] (its routing weight)
 * offsets [E+1], sorted_pair [T*k] int32 in; topk_w [T*k] fp32 in;
 * local_expert [T*k] int32 out; row_w [T*k] fp32 out. E must be a multiple of
 * experts_per_rank (else MOE_ERR_INVALID_ARG). Nothing is launched for T*k = 0.
 */
int moe_ep_pack_rows(const int32_t* offsets, const int32_t* sorted_pair, const float* topk_w, int T, int E, int k,
                     int experts_per_rank, int32_t* local_expert, float* row_w, moe_stream_t stream);

/*
 * moe_layer_bwd_pair_dw -- moe_layer_bwd without the router backward: in
 * place of d logits it returns every pair's routing-weight gradient
 *   dw[q] = <dY[q / k], o_q>,  o_q = the pair's unweighted expert output,
 * summed in a fixed order. On an expert's owner rank it runs with k = 1 over
 * the received rows (each row its own "token"; dY = the received dY rows), so
 * dX and dw come back in the order the rows arrived.
 * Arguments as moe_layer_bwd (probs, topk_idx and dlogits are not taken);
 * dw [T*k] fp32 out; ws >= moe_layer_bwd_workspace_bytes(...).
 */
int moe_layer_bwd_pair_dw(const moe_bf16* dY, const moe_bf16* Xp, const moe_bf16* gu_save, const moe_bf16* h,
                          const float* topk_w, const int32_t* offsets, const int32_t* sorted_pair,
                          const int32_t* pair_pos, int T, int E, int k, int H, int I, const moe_bf16* W_gu,
                          const moe_bf16* W_d, moe_bf16* dX, moe_bf16* dW_gu, moe_bf16* dW_d, float* dw, void* ws,
                          size_t ws_bytes, moe_stream_t stream);

/*
 * moe_router_bwd_from_dw -- the router backward of moe_layer_bwd from
 * routing-weight gradients given per expert-sorted row (dw_rows[r], r the
 * row of pair q = pair_pos[q]), e.g. those returned by the experts' owners.
 * Same formulas as moe_layer_bwd's d logits ("[WIP] Qwen3 MoE support",
 * torchtune PR #2820, review comment: renormalisation by the top-k sum +
 * 1e-20; then the softmax Jacobian). dw_rows [T*k], pair_pos [T*k], probs
 * [T,E], topk_idx / topk_w [T,k] in; dlogits [T,E] fp32 out.
 */
int moe_router_bwd_from_dw(const float* dw_rows, const int32_t* pair_pos, const float* probs,
                           const int32_t* topk_idx, const float* topk_w, int T, int E, int k, float* dlogits,
                           moe_stream_t stream);

/*
 * moe_layer_bwd with fp32 weight gradients: dW_gu [E,2I,H] and dW_d [E,H,I]
 * are fp32, the wgrad GEMMs' fp32 accumulators stored without rounding
 * (moe_layer_bwd rounds the same accumulators to bf16, so rounding this
 * output to bf16 gives moe_layer_bwd's dW bit for bit).
 * accumulate != 0: dW_gu += gradient and dW_d += gradient (one fp32 add per
 * element, each element written by one thread; experts with no rows leave
 * their dW unchanged) -- a gradient summed over micro-batches in fp32.
 * accumulate == 0: dW = gradient, zeros for experts with no rows.
 * dW_gu / dW_d 16-byte aligned, contiguous. Every other argument, the
 * workspace (moe_layer_bwd_workspace_bytes) and the error codes are those
 * of moe_layer_bwd.
 * Source: "[MoE] Improve moe kernels for unsloth fine tuning #3812", the
 * stacked expert weights [num_experts, 2*intermediate_dim, hidden_dim] and
 * [num_experts, hidden_dim, intermediate_dim]; the pages train in bf16 and
 * leave the gradient's precision open.
 */
int moe_layer_bwd_dw_f32(const moe_bf16* dY, const moe_bf16* Xp, const moe_bf16* gu_save, const moe_bf16* h,
                         const float* probs, const int32_t* topk_idx, const float* topk_w, const int32_t* offsets,
                         const int32_t* sorted_pair, const int32_t* pair_pos, int T, int E, int k, int H, int I,
                         const moe_bf16* W_gu, const moe_bf16* W_d, moe_bf16* dX, float* dW_gu, float* dW_d,
                         int accumulate, float* dlogits, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * LoRA adapters on the stacked expert weights.
 * Source: fused-MoE Triton project summary (sourcepulse), Highlighted
 * Details: LoRA on the fused expert weights. The pages give no formulas; the
 * update is the published LoRA form (Hu et al., 2021): a frozen W [out, in]
 * is used as W + scale * B A. Here one adapter per expert on each stacked
 * weight, gate|up fused:
 *   A_gu [E,r,H], B_gu [E,2I,r] on W_gu;  A_d [E,r,I], B_d [E,H,r] on W_d,
 * all bf16, row-major; r a multiple of 8 in [8, 512]; one scale.
 * moe_experts_fwd_lora -- moe_experts_fwd with the adapted weights. The low-
 * rank term is not formed as a matrix: each expert GEMM runs over [act | Z]
 * and [W | B] along K (its accumulator takes both), where
 *   Z_gu = scale * Xp A_gu^T  and  Z_d = scale * h A_d^T      [P, r] bf16
 * are written to the caller's Z_gu / Z_d (outputs, kept for the backward).
 * Errors: as moe_experts_fwd; r out of range -> MOE_ERR_INVALID_ARG.
 */
int moe_experts_fwd_lora(const moe_bf16* Xp, const int32_t* offsets, const int32_t* sorted_pair, const float* topk_w,
                         int T, int E, int k, int H, int I, const moe_bf16* W_gu, const moe_bf16* W_d, int r,
                         float scale, const moe_bf16* A_gu, const moe_bf16* B_gu, const moe_bf16* A_d,
                         const moe_bf16* B_d, moe_bf16* h, moe_bf16* gu_save, moe_bf16* O, moe_bf16* Z_gu,
                         moe_bf16* Z_d, moe_stream_t stream);

/* Bytes of workspace moe_layer_bwd_lora needs (0 for invalid sizes). */
size_t moe_layer_bwd_lora_workspace_bytes(int T, int E, int k, int H, int I, int r, int recompute_gu);

/*
 * moe_layer_bwd_lora -- backward of the adapted layer. With G the gradient
 * reaching a stacked weight (that of W, equal to that of W + scale B A):
 *   dA = scale B^T G,  dB = scale G A^T      per expert (chain rule),
 * computed without forming G: dA_gu = V_gu^T Xp, dB_gu = dGU^T Z_gu,
 * dA_d = V_d^T (w h), dB_d = dYp^T (w Z_d) over each expert's rows, with
 * V_d = scale dYp B_d and V_gu = scale dGU B_gu (which also extend the dgrad
 * GEMMs along K, as in the forward).
 * dA_gu [E,r,H], dB_gu [E,2I,r], dA_d [E,r,I], dB_d [E,H,r]: fp32 outputs;
 * accumulate != 0 adds to them (experts without rows add nothing), else
 * they are overwritten (zeros for such experts).
 * dW_gu / dW_d: bf16 gradients of the base weights, or NULL to skip them
 * (frozen base weights: their two GEMMs are not run).
 * Z_gu, Z_d: the forward's. Every other argument and error as moe_layer_bwd;
 * ws >= moe_layer_bwd_lora_workspace_bytes(...).
 */
int moe_layer_bwd_lora(const moe_bf16* dY, const moe_bf16* Xp, const moe_bf16* gu_save, const moe_bf16* h,
                       const float* probs, const int32_t* topk_idx, const float* topk_w, const int32_t* offsets,
                       const int32_t* sorted_pair, const int32_t* pair_pos, int T, int E, int k, int H, int I,
                       const moe_bf16* W_gu, const moe_bf16* W_d, int r, float scale, const moe_bf16* A_gu,
                       const moe_bf16* B_gu, const moe_bf16* A_d, const moe_bf16* B_d, const moe_bf16* Z_gu,
                       const moe_bf16* Z_d, moe_bf16* dX, float* dA_gu, float* dB_gu, float* dA_d, float* dB_d,
                       int accumulate, moe_bf16* dW_gu, moe_bf16* dW_d, float* dlogits, void* ws, size_t ws_bytes,
                       moe_stream_t stream);

/*
 * Gather-fused variants -- the same results as moe_experts_fwd and
 * moe_layer_bwd, reading the activations in token order: the GEMMs load the
 * rows of X [T,H] (and of dY [T,H]) by token index t = sorted_pair[r] / k
 * with row-gather TMA loads (tile::gather4, four 128-byte row pieces per
 * load) issued by the GEMM itself, so no permuted copies Xp / dYp are made
 * or read.
 * Source: fused-MoE Triton project summary (sourcepulse), How It Works:
 * inputs are sorted by expert for coalesced grouped-GEMM reads; here the
 * sort is applied inside the GEMM's operand loads. moe_permute may then be
 * called with X = Xp = NULL.
 */
int moe_experts_fwd_x(const moe_bf16* X, const int32_t* offsets, const int32_t* sorted_pair, const float* topk_w,
                      int T, int E, int k, int H, int I, const moe_bf16* W_gu, const moe_bf16* W_d, moe_bf16* h,
                      moe_bf16* gu_save, moe_bf16* O, moe_stream_t stream);

/* Scratch bytes of moe_layer_bwd_x (smaller than moe_layer_bwd's: no dYp). */
size_t moe_layer_bwd_x_workspace_bytes(int T, int E, int k, int H, int I, int recompute_gu);

/* moe_layer_bwd with X [T,H] in token order in place of Xp;
 * ws >= moe_layer_bwd_x_workspace_bytes(...). */
int moe_layer_bwd_x(const moe_bf16* dY, const moe_bf16* X, const moe_bf16* gu_save, const moe_bf16* h,
                    const float* probs, const int32_t* topk_idx, const float* topk_w, const int32_t* offsets,
                    const int32_t* sorted_pair, const int32_t* pair_pos, int T, int E, int k, int H, int I,
                    const moe_bf16* W_gu, const moe_bf16* W_d, moe_bf16* dX, moe_bf16* dW_gu, moe_bf16* dW_d,
                    float* dlogits, void* ws, size_t ws_bytes, moe_stream_t stream);

/* moe_layer_bwd_dw_f32 with X [T,H] in token order in place of Xp;
 * ws >= moe_layer_bwd_x_workspace_bytes(...). */
int moe_layer_bwd_x_dw_f32(const moe_bf16* dY, const moe_bf16* X, const moe_bf16* gu_save, const moe_bf16* h,
                           const float* probs, const int32_t* topk_idx, const float* topk_w, const int32_t* offsets,
                           const int32_t* sorted_pair, const int32_t* pair_pos, int T, int E, int k, int H, int I,
                           const moe_bf16* W_gu, const moe_bf16* W_d, moe_bf16* dX, float* dW_gu, float* dW_d,
                           int accumulate, float* dlogits, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Router Linear -- logits = X W_r^T and its backward, on the tensor cores.
 * Source: "Integration of fused moe kernel (e.g., megablocks) for efficient
 * moe training" (axolotl issue #3155), discussion of the router's weight
 * shape: the router is a Linear(hidden -> experts) whose weight is
 * [num_experts, hidden]; the router runs in fp32.
 *
 * X [T,H] is bf16, W_r [E,H] fp32. Every fp32 operand is split exactly into
 * three bf16 terms on the device, so the logits are the exact products of X
 * and W_r summed in fp32 (tensor-core accumulation order; split-K partial
 * sums added in a fixed order, so results are deterministic).
 * Limits: T >= 0, 3*T < 2^31, 1 <= E <= 1024, H a positive multiple of 8.
 */

/* Scratch bytes for moe_router_fwd and moe_router_bwd (the same buffer
 * serves both); 0 for invalid shapes. */
size_t moe_router_workspace_bytes(int T, int H, int E);

/*
 * moe_router_fwd -- logits = X W_r^T, then what moe_route computes from them.
 *   logits [T,E] fp32 (optional output, may be NULL), topk_idx [T,k] int32,
 *   topk_w [T,k] fp32, probs [T,E] fp32 (optional, may be NULL): the same
 *   outputs, with the same rules, as moe_route applied to these logits.
 *   ws >= moe_router_workspace_bytes(T, H, E).
 */
int moe_router_fwd(const moe_bf16* X, const float* W_r, int T, int H, int E, int k, float* logits,
                   int32_t* topk_idx, float* topk_w, float* probs, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_router_bwd -- gradients of logits = X W_r^T for upstream dlogits [T,E]
 * fp32 (for instance moe_layer_bwd's output).
 *   dW_r [E,H] fp32 (output, may be NULL): dlogits^T X, exact products of the
 *     fp32 dlogits and bf16 X summed in fp32.
 *   dX [T,H] bf16 (in/out, may be NULL): on entry the rest of the layer's
 *     input gradient (moe_layer_bwd's dX); on return bf16(dX + dlogits W_r),
 *     the product carried to about 2^-16 relative (the two leading bf16
 *     terms of each operand), far below the bf16 rounding of the result.
 *   X is read only for dW_r, W_r only for dX. With T == 0, dW_r is zeroed.
 *   ws >= moe_router_workspace_bytes(T, H, E).
 */
int moe_router_bwd(const float* dlogits, const moe_bf16* X, const float* W_r, int T, int H, int E, float* dW_r,
                   moe_bf16* dX, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_selftest_wait_timeout -- diagnostics: enqueues one kernel that waits on
 * a barrier nothing signals, using the same bounded wait as the pipeline
 * kernels but with a limit of limit_ms (1..2000) milliseconds. When the limit
 * passes the kernel records MOE_ERR_TIMEOUT in the device status word and
 * exits, so moe_last_device_status(stream) then returns MOE_ERR_TIMEOUT and
 * the context stays usable. No counterpart on the pages.
 */
int moe_selftest_wait_timeout(int limit_ms, moe_stream_t stream);

/*
 * Per-kernel timing with CUDA events recorded on the launching stream around
 * every kernel launch (off by default; measurement only, no effect on results).
 * moe_profile_enable(1) starts recording and clears earlier records.
 * moe_profile_read synchronises on the recorded events and returns the total
 * device milliseconds and launch count of kernel `name` (see
 * moe_profile_kernel_name); MOE_ERR_INVALID_ARG for an unknown name.
 */
int moe_profile_enable(int on);
/* Restricts recording to kernel `name` until the next moe_profile_enable
 * (NULL: every kernel), so that one kernel can be timed with the least
 * disturbance of the launch stream. MOE_ERR_INVALID_ARG for an unknown name. */
int moe_profile_only(const char* name);
int moe_profile_read(const char* name, double* total_ms, int* launches);
/* Effective SM clock (MHz) of grouped-GEMM kernel `name` over the launches
 * recorded since moe_profile_enable(1): SM cycles counted by each CTA's MMA
 * issuer over its main loop, divided by the global nanoseconds of the same
 * interval. It shows the clock the kernel really ran at (the power limit
 * lowers it). 0 when nothing was recorded or `name` is not a GEMM.
 * Synchronises the device. MOE_ERR_INVALID_ARG for an unknown name. */
int moe_profile_read_clock(const char* name, double* sm_mhz);
/* Name of kernel slot i (0-based), NULL past the last one. */
const char* moe_profile_kernel_name(int i);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
