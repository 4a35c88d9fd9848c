/*
 * moe.h -- C ABI of the B200 (sm_100a) token-choice mixture-of-experts layer.
 *
 * One layer, forward and backward, on one GPU:
 *   route      logits = x W_gate (+bias); top-k per token; softmax over the k
 *   permute    histogram of expert choices, prefix sum, stable scatter into
 *              expert-contiguous rows (optionally token-rounded)
 *   ffn_fwd    grouped GEMM [x W1 | x W3] with fused SwiGLU, grouped GEMM A W2
 *   combine    O_t = sum over the rows of token t of weight * Y(row)
 *   layer_bwd  dS = <dA', A>, SwiGLU backward, dX / dW grouped GEMMs, router
 *              gradient
 *
 * Sources, cited by page title and section:
 *   [Beam]     "From 501B to 23B: what is Beam doing", sec. 2.2 (MoE layer:
 *              router W_gate [d_model, N], top-k, weighted sum of experts),
 *              sec. 5.3 (MoELayer: topk, softmax of the k values, per-expert
 *              loop that grouped GEMM replaces), sec. 5.4 (expert counts).
 *   [Trinity]  "Trinity Large: open 400B sparse MoE" commentary, examples 1-3
 *              (top-k + softmax gating, bincount, dispatch / combine).
 *   [SonicMoE] techwalker summary of SonicMoE, sec. 1 (dS = <dA', A>, Y not
 *              stored) and sec. 3 (token rounding to multiples of the tile).
 *   [Olmo]     Olmo-core 3 news piece (rows placed straight into expert input
 *              buffers; GPU-resident routing; grouped GEMM).
 *
 * Conventions for every call:
 *   - Tensor arguments are DEVICE pointers on the current CUDA device,
 *     allocated and owned by the caller, row-major and contiguous.  The
 *     library allocates no device memory; scratch comes from a caller
 *     workspace whose size the matching *_workspace_size() call returns.
 *     The one exception is moe_permute_noalloc, whose scratch is a static
 *     512 KiB device array that every device loading the library keeps.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls only
 *     enqueue kernels on it; none synchronises or copies routing metadata to
 *     the host, so the row count R lives on the device only (offsets[E]).
 *   - dtype MOE_BF16: bf16 activations/weights, fp32 accumulation,
 *     tcgen05 tensor cores.  MOE_F32: fp32 everywhere, CUDA-core path.
 *   - Return value: MOE_OK or a negative MOE_ERR_* code; moe_last_error()
 *     gives a message.  Arguments are checked on the host before any launch;
 *     a failed check launches nothing.  Device-side waits are bounded: if one
 *     expires the kernel records a code in a device status word and returns,
 *     and moe_check_status() reports it as MOE_ERR_DEVICE_TIMEOUT.  Device-side
 *     data checks (an expert id out of range) skip the bad item and record a
 *     code that moe_check_status() reports as MOE_ERR_DEVICE_CHECK.
 *   - Shapes: 1 <= k <= 8, k <= E <= 256, T >= 0.  The bf16 path needs
 *     d % 128 == 0 and f % 128 == 0; the f32 path d % 64 == 0 and f % 64 == 0.
 *   - Row space: expert e owns rows [offsets[e], offsets[e+1]); each segment
 *     starts at a multiple of `tile` (128) and padding rows are empty (token
 *     -1, weight 0).  Row buffers hold cap = moe_row_capacity(T,E,k,tile)
 *     rows; only rows < offsets[E] are touched.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_OK 0
#define MOE_ERR_INVALID_ARG (-1)
#define MOE_ERR_UNSUPPORTED (-2)
#define MOE_ERR_CUDA (-3)
#define MOE_ERR_DEVICE_TIMEOUT (-4)
#define MOE_ERR_WORKSPACE (-5)
#define MOE_ERR_DEVICE_CHECK (-6)

#define MOE_F32 0
#define MOE_BF16 1

#define MOE_ROUND_NONE 0
#define MOE_ROUND_NEAREST 1
#define MOE_ROUND_CAPACITY 2

#define MOE_GATE_TOPK_SOFTMAX 0
#define MOE_GATE_SOFTMAX_TOPK 1

/* Library version (major*10000 + minor*100 + patch). */
int moe_version(void);

/* Message describing the last error returned on the calling host thread. */
const char* moe_last_error(void);

/* Number of rows a plan may occupy: T*k + E*tile. */
size_t moe_row_capacity(int T, int E, int k, int tile);

/*
 * moe_route -- router logits, top-k and the gates of the k chosen experts.
 * [Beam] sec. 2.2 and 5.3; [Trinity] example 1.
 *   x [T,d] (dtype), w_gate [d,E] (dtype).
 *   gate_mode MOE_GATE_TOPK_SOFTMAX: gates = softmax of the k chosen logits
 *     ([Beam] sec. 5.3, [Trinity] example 1).  MOE_GATE_SOFTMAX_TOPK: gates =
 *     softmax over all E logits, the k largest kept without renormalising
 *     ([Beam] sec. 2.2 formula, [Trinity] challenge 1).  The choice of
 *     experts is the same in both modes.
 *   logits_override [T,E] fp32 or NULL: when given, x and w_gate are not read
 *     and these values replace x W_gate (random-routing workloads).
 *   logit_bias [E] fp32 or NULL: added to every token's logits.
 *   logit_noise [T,E] fp32 or NULL: noisy top-k gating ([Beam] sec. 3.3,
 *     noise on the routing scores in training): added after the bias
 *     (fp32 adds in that order); the caller draws it.  Choice, gates and the
 *     returned logits are those of the noisy scores; the gradient
 *     moe_layer_bwd returns for the logits is also that of the clean ones.
 *   logits [T,E] fp32 out; idx [T,k] int32 out: the k largest logits in
 *   descending order, ties to the lowest expert id; gate [T,k] fp32 out:
 *   the gates of those k experts (per gate_mode).
 */
int moe_route(const void* x, const void* w_gate, int T, int d, int E, int k, int dtype,
              int gate_mode, const float* logits_override, const float* logit_bias,
              const float* logit_noise, float* logits, int32_t* idx, float* gate,
              void* stream);

/*
 * moe_permute -- expert histogram, prefix sum and stable permutation into
 * expert-contiguous rows.  [Trinity] examples 2-3; [Olmo] (expert input
 * buffers, GPU-resident routing); [Beam] sec. 5.4 (counts).
 * round_mode MOE_ROUND_NEAREST applies token rounding ([SonicMoE] sec. 3):
 * each expert's count becomes the nearest multiple of `tile` (halves up,
 * capped at tile*floor(T/tile)); drops remove the pairs with the smallest
 * score exp(l - LSE), larger token first on ties; additions take the
 * unassigned tokens with the largest score, smaller token first on ties;
 * row weights are those scores (kept pairs: their gate).  LSE is the
 * log-sum-exp of the token's k chosen logits (gate_mode
 * MOE_GATE_TOPK_SOFTMAX) or of all its E logits (MOE_GATE_SOFTMAX_TOPK), so
 * the score is the gate the pair has or would have.
 * round_mode MOE_ROUND_CAPACITY applies a capacity factor ([Beam] sec. 2.3):
 * an expert chosen by more than `capacity` tokens keeps the `capacity` pairs
 * with the largest score (the same score and tie rule as rounding drops) and
 * drops the rest; no pair is added, segments are padded to the tile with
 * empty rows.  A dropped slot contributes nothing to its token's output.
 *   idx [T,k], gate [T,k]: from moe_route.  logits [T,E]: read only when
 *     rounding or dropping (round_mode != MOE_ROUND_NONE).
 *   gate_mode: the mode moe_route used (read only when round_mode !=
 *     MOE_ROUND_NONE).
 *   capacity: tokens per expert for MOE_ROUND_CAPACITY (>= 0; e.g.
 *     ceil(capacity_factor * T * k / E)); ignored otherwise.
 *   tile: must be 128 (the grouped-GEMM M tile, also the rounding unit).
 *   counts [E] out: token count per expert before rounding.
 *   offsets [E+1] out: segment starts (multiples of tile); offsets[E] = R.
 *   row_token [cap], row_gate [cap] fp32, row_slot [cap] out: token, weight
 *     and slot (t*k+j, or -1 for a row added by rounding) of each row;
 *     padding rows get -1, 0, -1.
 *   slot_row [T*k] out: row of slot (t,j), or -1 if rounding or the
 *     capacity dropped it.
 *   extra_row [T,E] out (required with MOE_ROUND_NEAREST, else may be NULL
 *     and is not written): row of the pair (t,e) added by rounding, or -1.
 *   ws: workspace of at least moe_permute_workspace_size() bytes.
 */
size_t moe_permute_workspace_size(int T, int E, int k, int round_mode);
int moe_permute(const int32_t* idx, const float* gate, const float* logits,
                int T, int E, int k, int round_mode, int tile, int gate_mode, int capacity,
                int32_t* counts, int32_t* offsets, int32_t* row_token, float* row_gate,
                int32_t* row_slot, int32_t* slot_row, int32_t* extra_row,
                void* ws, size_t ws_bytes, void* stream);

/*
 * moe_permute_noalloc -- moe_permute without rounding, for callers that
 * cannot allocate device memory at call time: plugin hosts that pass a
 * kernel nothing but its input and output buffers and own every allocation,
 * and step loops that must not call cudaMalloc between launches because it
 * can synchronise the whole device.  The pages have no counterpart of this
 * entry point; it computes exactly what moe_permute (round_mode
 * MOE_ROUND_NONE) computes, with the same arguments minus logits, extra_row
 * and the workspace.
 *   Scratch: a static device array of 512 KiB (per-block expert counts and
 *   bases) that every device which loads the library keeps until exit.
 *   Limit: T <= 65536 (and E <= 256); larger T returns MOE_ERR_UNSUPPORTED.
 *   The first call on a device looks up the array's device address (a
 *   one-time set-up with that device current); make that first call before
 *   any stream capture.  Calls share the array, so calls whose kernels
 *   overlap on the GPU (different streams or host threads) race and must be
 *   ordered by the caller.  Nothing in it needs clearing between calls.
 *   Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 */
int moe_permute_noalloc(const int32_t* idx, const float* gate, int T, int E, int k, int tile,
                        int32_t* counts, int32_t* offsets, int32_t* row_token, float* row_gate,
                        int32_t* row_slot, int32_t* slot_row, void* stream);

/*
 * moe_expert_ffn_fwd -- per-expert SwiGLU FFN on the permuted rows.
 * [Beam] sec. 2.2/5.3 (expert FFN, grouped instead of looped); [Olmo]
 * (grouped GEMM; rows placed straight into expert input buffers).  Experts
 * are SwiGLU:
 *   H = [x W1_e | x W3_e]  (saved for backward, dtype)
 *   A = silu(H1) * H3      (transient)
 *   Y_perm = A W2_e        (transient, dtype)
 *   x [T,d]; w1, w3 [E,d,f]; w2 [E,f,d]; row_token [cap], offsets [E+1],
 *   slot_row [T*k] and extra_row [T,E] (NULL without rounding) from
 *   moe_permute with tile 128.  H [cap,2f] out; Y_perm [cap,d] out.
 */
size_t moe_ffn_fwd_workspace_size(int T, int d, int f, int E, int k, int dtype);
int moe_expert_ffn_fwd(const void* x, const void* w1, const void* w3, const void* w2,
                       const int32_t* row_token, const int32_t* offsets,
                       const int32_t* slot_row, const int32_t* extra_row,
                       int T, int d, int f, int E, int k, int dtype,
                       void* H, void* Y_perm, void* ws, size_t ws_bytes, void* stream);

/*
 * MXFP8 expert FFN forward (the "MXFP8 low-precision switch" of the Olmo-core
 * 3 news piece; FP8/MXFP8 support is the SonicMoE summary's future work).
 * Format: OCP Microscaling (MX) v1.0 with E4M3 elements -- blocks of 32
 * consecutive elements along each GEMM's contraction dimension share one E8M0
 * scale 2^(code-127); shared exponent floor(log2 max|v|) - 8 (clamped to
 * [-127, 127]), elements rounded to nearest-even and saturated to +-448.
 * Scale arrays are 512-byte blocks [rows/128][K/128]; the scale of row r and
 * 32-element K-block j is byte (r%32)*16 + ((r/32)%4)*4 + (j%4) of its block.
 * The GEMMs run on the tcgen05 block-scaled tensor cores (kind::mxf8f6f4)
 * with fp32 accumulation; H and Y are bf16 as in moe_expert_ffn_fwd.  The
 * backward is moe_layer_bwd (all bf16) or moe_layer_bwd_mxfp8, whose dX GEMM
 * takes MXFP8 dH and W1/W3 (blocks along f), and optionally its weight-
 * gradient GEMMs MXFP8 operands along tokens; either way the quantisers pass
 * gradients straight through.
 *
 * moe_mxfp8_weight_sizes: sizes[8] out = bytes of W13q, W13s, W2q, W2s,
 *   W1r, W1r scales, W3r, W3r scales for E experts (d and f multiples of 128,
 *   else MOE_ERR_UNSUPPORTED).
 * moe_mxfp8_quantize_weights: w1, w3 [E,d,f] and w2 [E,f,d] bf16 ->
 *   W13q [E, 2f, d] E4M3 (K = d contiguous; rows 256b..256b+127 are columns
 *   128b..128b+127 of W1 and rows 256b+128..256b+255 the same columns of W3),
 *   W13s its scales, W2q [E, d, f] E4M3 (K = f contiguous), W2s its scales,
 *   and, when w1rq.. are not NULL (all four or none), W1r / W3r [E, d, f]
 *   E4M3 in the weights' own layout with blocks along f, for
 *   moe_layer_bwd_mxfp8.  Run it once per weight update; caller-owned device
 *   buffers of the sizes above, 16-byte aligned.
 * moe_expert_ffn_fwd_mxfp8: as moe_expert_ffn_fwd (bf16 x, same plan
 *   arguments, H [cap,2f] and Y_perm [cap,d] bf16 out) with the quantised
 *   weights; x rows are quantised while they are scattered and A in the
 *   up-projection's epilogue.  ws: at least
 *   moe_ffn_fwd_mxfp8_workspace_size() bytes; after the call it holds, each
 *   piece starting at the next multiple of 256 bytes: Xq [capr, d] E4M3, its
 *   scales, Aq [capr, f] E4M3, its scales (capr = cap rounded up to 128).
 *   Needs an sm_100 device.
 */
int moe_mxfp8_weight_sizes(int E, int d, int f, size_t* sizes);
int moe_mxfp8_quantize_weights(const void* w1, const void* w3, const void* w2, int E, int d,
                               int f, uint8_t* w13q, uint8_t* w13s, uint8_t* w2q, uint8_t* w2s,
                               uint8_t* w1rq, uint8_t* w1rs, uint8_t* w3rq, uint8_t* w3rs,
                               void* stream);
size_t moe_ffn_fwd_mxfp8_workspace_size(int T, int d, int f, int E, int k);
/*
 * moe_mxfp8_quantize_tokens -- a row-space matrix quantised along its rows
 * (the token axis), as the MXFP8 weight-gradient GEMMs of
 * moe_layer_bwd_mxfp8 take it.  Row r is src row r of a bf16 [rows, n]
 * matrix, or, when gather_row is not NULL, token row gather_row[r] of a
 * token-major bf16 [T, n] matrix (-1: a zero row).  Rows below offsets[E]
 * (the plan's rows; segments are multiples of 128) are quantised in blocks
 * of 32 consecutive rows: q [n, capr] E4M3 (column c of the source is row c
 * of q, rows contiguous) and sf its E8M0 scales in the layout above with n
 * as the row (MN) dimension and capr / 128 K chunks.  Bytes of q and sf for
 * rows at or above offsets[E] are left untouched.  n and capr: multiples of
 * 128 (capr >= offsets[E]); src has src_rows rows; src and q 16-byte
 * aligned; device buffers owned by the caller.  A plan past capr, or a
 * source row at or past src_rows, is a device data check (code 0x140 from
 * moe_check_status; the plan is skipped, the row read as zeros).
 */
int moe_mxfp8_quantize_tokens(const void* src, int src_rows, const int32_t* gather_row,
                              const int32_t* offsets, int E, int n, int capr, uint8_t* q,
                              uint8_t* sf, void* stream);
/*
 * moe_layer_bwd_mxfp8 -- moe_layer_bwd (bf16 only) whose dX_perm GEMM runs
 * on MXFP8 operands: the dA' epilogue also writes dH in E4M3 with blocks
 * along 2f, and W1r/W3r come from moe_mxfp8_quantize_weights.
 * wgrad_mxfp8 = 1 also runs the weight-gradient GEMMs (dW2 = (s*A)^T dO,
 * [dW1 | dW3] = x^T dH per expert) on MXFP8 operands: x, dO, s*A and dH are
 * quantised along the tokens -- the contraction dimension of these GEMMs --
 * in blocks of 32 consecutive rows of each expert's segment of the row space
 * (padding rows count as zero rows); d and 2f must then be multiples of 256
 * (else MOE_ERR_UNSUPPORTED).  wgrad_mxfp8 = 0 keeps them bf16.  dA' and the
 * router gradient are as in moe_layer_bwd; the quantisers pass gradients
 * straight through.  ws: at least
 * moe_layer_bwd_mxfp8_workspace_size(..., wgrad_mxfp8) bytes.
 */
size_t moe_layer_bwd_mxfp8_workspace_size(int T, int d, int f, int E, int k, int wgrad_mxfp8);
int moe_layer_bwd_mxfp8(const void* dout, const void* x, const void* w_gate,
                        const void* w1, const void* w3, const void* w2,
                        const uint8_t* w1rq, const uint8_t* w1rs,
                        const uint8_t* w3rq, const uint8_t* w3rs,
                        const int32_t* idx, const float* gate, const float* gate_grad,
                        const float* logits, int gate_mode, const int32_t* offsets,
                        const int32_t* row_token, const float* row_gate,
                        const int32_t* slot_row, const int32_t* extra_row, const void* H,
                        int T, int d, int f, int E, int k, int router_grad, int wgrad_mxfp8,
                        void* dx, float* dw_gate, void* dw1, void* dw3, void* dw2,
                        float* dS, float* dlogits, void* ws, size_t ws_bytes, void* stream);

int moe_expert_ffn_fwd_mxfp8(const void* x, const uint8_t* w13q, const uint8_t* w13s,
                             const uint8_t* w2q, const uint8_t* w2s,
                             const int32_t* row_token, const int32_t* offsets,
                             const int32_t* slot_row, const int32_t* extra_row,
                             int T, int d, int f, int E, int k,
                             void* H, void* Y_perm, void* ws, size_t ws_bytes, void* stream);

/*
 * moe_combine -- routing-weighted unpermute: O_t = sum over token t's rows of
 * row_gate[row] * Y_perm[row], summed in fp32 in a fixed order (kept slots in
 * slot order, then rows added by rounding in ascending expert id).
 * [Beam] sec. 2.2 (weighted sum); [Trinity] example 3 (add back per token).
 *   Y_perm [cap,d]; row_gate [cap]; slot_row [T*k]; extra_row [T,E] or NULL.
 *   out [T,d] (dtype).
 */
int moe_combine(const void* Y_perm, const float* row_gate, const int32_t* slot_row,
                const int32_t* extra_row, int T, int d, int E, int k, int dtype,
                void* out, void* stream);

/*
 * moe_layer_bwd -- backward of the whole layer from the saved set
 * {x, idx, gate, plan, H}.  Y is never stored: the router-score gradient is
 * dS = <dA', A> with dA' = dO W2^T and A recomputed from H ([SonicMoE] sec. 1).
 *   dA = s dA'; SwiGLU backward gives dH = [dA*H3*silu'(H1) | dA*silu(H1)];
 *   dW2_e = sum (s A)^T dO;  [dW1|dW3]_e = sum x^T dH;
 *   dX_perm = dH [W1|W3]^T;  dx_t = sum over t's rows of dX_perm + dlogits_t W_gate^T;
 *   dlogits_te = [e in F_t] s_te dS_te - [e in K_t] g_te sum_{F_t} s dS
 *   (F_t: token t's final rows with weights s; K_t: its top-k) with
 *   gate_mode MOE_GATE_TOPK_SOFTMAX; with MOE_GATE_SOFTMAX_TOPK the gates
 *   are p = softmax over all E logits and every expert gets the second term:
 *   dlogits_te = [e in F_t] p_te dS_te - p_te sum_{F_t} p dS;
 *   dW_gate = x^T dlogits.
 *   logits [T,E] fp32 (from moe_route): read only with MOE_GATE_SOFTMAX_TOPK
 *   (may be NULL otherwise).  gate_mode: the mode moe_route used.
 *   router_grad = 0 when the logits did not come from x W_gate (override):
 *   dW_gate is then zero and dx gets no router term.
 *   gate_grad [T,k] fp32 or NULL: gradient of auxiliary losses with respect
 *   to the gates (e.g. from moe_balance_loss); it enters dlogits through the
 *   softmax over the k logits: dl_t,idx_j += g_j (a_j - sum_i g_i a_i)
 *   (MOE_GATE_SOFTMAX_TOPK: dl_te += [e in K_t] p_e a_e - p_e sum_i g_i a_i).
 *   Outputs: dx [T,d] (dtype), dw_gate [d,E] fp32, dw1, dw3 [E,d,f] (dtype),
 *   dw2 [E,f,d] (dtype), dS [cap] fp32 (may be NULL), dlogits [T,E] fp32
 *   (may be NULL).  Every output element is written (no accumulation).
 */
size_t moe_layer_bwd_workspace_size(int T, int d, int f, int E, int k, int dtype);
int moe_layer_bwd(const void* dout, const void* x, const void* w_gate,
                  const void* w1, const void* w3, const void* w2,
                  const int32_t* idx, const float* gate, const float* gate_grad,
                  const float* logits, int gate_mode, const int32_t* offsets,
                  const int32_t* row_token, const float* row_gate,
                  const int32_t* slot_row, const int32_t* extra_row, const void* H,
                  int T, int d, int f, int E, int k, int dtype, int router_grad,
                  void* dx, float* dw_gate, void* dw1, void* dw3, void* dw2,
                  float* dS, float* dlogits, void* ws, size_t ws_bytes, void* stream);

/*
 * Expert parallelism across G ranks (one GPU each): rank g owns experts
 * g*El .. g*El+El-1 (El = E/G) and keeps their weights resident; the
 * permuted rows travel to the experts instead ("Olmo-core 3" news piece:
 * experts stay on their GPU and data is routed to them, row-wise expert
 * parallelism places rows straight into the experts' input buffers; "From
 * 501B to 23B: what is Beam doing", sec. 4.2: tokens reach the GPU holding
 * their expert through an all-to-all exchange).  The token side (route,
 * permute, combine, router gradient, dx) runs where the tokens are; the
 * expert side (grouped GEMMs, dS, expert weight gradients) where the
 * experts are.  The calls below are those pieces; the exchange itself is
 * the caller's (NCCL send/recv of whole 128-aligned segments).
 *
 * moe_gather_rows -- dst[r] = src[row_token[r]] for every row r < offsets[E]
 *   of a plan from moe_permute (padding rows zero): the row gather that
 *   moe_expert_ffn_fwd and moe_layer_bwd run internally.  src [T,width],
 *   dst [cap,width] (dtype); width a multiple of 8.  The segments of rank
 *   g's experts, rows offsets[g*El] .. offsets[g*El+El], are what this rank
 *   sends to rank g.
 */
int moe_gather_rows(const void* src, const int32_t* row_token, const int32_t* offsets,
                    const int32_t* slot_row, const int32_t* extra_row, int T, int width, int E,
                    int k, int dtype, void* dst, void* stream);

/*
 * moe_ep_dispatch_counts -- seg_rows[e] = offsets[e+1] - offsets[e] [E]: the
 *   rows this rank sends for expert e (to the rank owning e), a multiple of
 *   128.  Exchanged between ranks, they become the receivers' recv_rows.
 * moe_ep_receive_plan -- placement of received segments on a rank owning El
 *   experts.  recv_rows [G, El]: rows source s sends for local expert j.
 *   local_offsets [El+1] out: local expert j owns rows local_offsets[j] ..
 *   local_offsets[j+1] (sources in rank order; local_offsets[El] = rows
 *   received).  recv_row [G, El] out: first local row of the segment from
 *   (s, j).  A count that is negative or not a multiple of 128 is treated as
 *   0 and recorded as a device data check (code 0x130, MOE_ERR_DEVICE_CHECK
 *   from moe_check_status).  El <= 256.
 */
int moe_ep_dispatch_counts(const int32_t* offsets, int E, int32_t* seg_rows, void* stream);
int moe_ep_receive_plan(const int32_t* recv_rows, int G, int El, int32_t* local_offsets,
                        int32_t* recv_row, void* stream);

/*
 * moe_expert_rows_fwd -- the expert side of moe_expert_ffn_fwd on rows that
 *   are already in expert-contiguous order: H = [xg W1_e | xg W3_e], A =
 *   silu(H1) * H3, Y = A W2_e for the rows of each expert e < E, segments
 *   offsets[e] .. offsets[e+1] (multiples of 128; offsets[E] <= rows; rows
 *   of zeros give zeros).  xg [rows,d], w1, w3 [E,d,f], w2 [E,f,d], H
 *   [rows,2f] out, Y [rows,d] out; bf16 only (sm_100 tensor cores); rows a
 *   positive multiple of 128.  ws: at least
 *   moe_expert_rows_fwd_workspace_size() bytes.
 */
size_t moe_expert_rows_fwd_workspace_size(int rows, int f, int dtype);
int moe_expert_rows_fwd(const void* xg, const void* w1, const void* w3, const void* w2,
                        const int32_t* offsets, int rows, int d, int f, int E, int dtype, void* H,
                        void* Y, void* ws, size_t ws_bytes, void* stream);

/*
 * moe_expert_rows_bwd -- the expert side of moe_layer_bwd on the same rows:
 *   dA' = dog W2_e^T, dS = <dA', A> (A recomputed from H; "SonicMoE"
 *   summary, sec. 1), dA = row_gate * dA', SwiGLU backward -> dH,
 *   dX_rows = dH [W1_e | W3_e]^T, dW2_e = (row_gate A)^T dog,
 *   [dW1_e | dW3_e] = xg^T dH, every output written (experts without rows
 *   get zero gradients).  dog [rows,d] (gathered dO rows), xg [rows,d], H
 *   [rows,2f] (from moe_expert_rows_fwd), row_gate [rows] fp32 (the rows'
 *   weights, moe_permute's row_gate carried with the rows); dX_rows
 *   [rows,d] out; dS [rows] fp32 out (rows below offsets[E]); dw1, dw3
 *   [E,d,f], dw2 [E,f,d] out.  bf16 only; ws: at least
 *   moe_expert_rows_bwd_workspace_size() bytes.
 */
size_t moe_expert_rows_bwd_workspace_size(int rows, int d, int f, int dtype);
int moe_expert_rows_bwd(const void* dog, const void* xg, const float* row_gate, const void* H,
                        const void* w1, const void* w3, const void* w2, const int32_t* offsets,
                        int rows, int d, int f, int E, int dtype, void* dX_rows, float* dS,
                        void* dw1, void* dw3, void* dw2, void* ws, size_t ws_bytes,
                        void* stream);

/*
 * moe_token_bwd -- the token side of moe_layer_bwd: from each row's dX_rows
 *   and dS in this rank's own row space (returned by the experts' ranks),
 *   dlogits (as in moe_layer_bwd), dW_gate = x^T dlogits over this rank's
 *   tokens (data-parallel ranks add theirs), dx = unpermute-sum of dX_rows +
 *   dlogits W_gate^T.  Arguments as in moe_layer_bwd; dX_rows [cap,d]
 *   (dtype), dS [cap] fp32.  ws: at least moe_token_bwd_workspace_size().
 */
size_t moe_token_bwd_workspace_size(int T, int d, int E, int k, int dtype);
int moe_token_bwd(const void* dX_rows, const float* dS, const void* x, const void* w_gate,
                  const int32_t* idx, const float* gate, const float* gate_grad,
                  const float* logits, int gate_mode, const float* row_gate,
                  const int32_t* slot_row, const int32_t* extra_row, int T, int d, int E, int k,
                  int dtype, int router_grad, void* dx, float* dw_gate, float* dlogits, void* ws,
                  size_t ws_bytes, void* stream);

/*
 * moe_balance_loss -- load-balance loss and routing statistics.
 * ["Breaking the hundred-billion-parameter barrier: how MoE reshapes
 * distributed training", challenge 1, solution 1]: L = lambda * CV(m)^2 with
 * m_e = (1/T) sum_t G_te the mean routing distribution (G_t: token t's top-k
 * gates, zero elsewhere) and CV the population coefficient of variation over
 * the E experts.  Statistics of the expert token counts: [Trinity] example 2
 * (bincount, squared deviation from the mean), [Beam] sec. 5.4 (share of the
 * busiest expert).
 *   idx [T,k], gate [T,k] from moe_route (T >= 1).
 *   stats [4] fp32 out: loss, max share of assignments, CV^2 of the counts,
 *     mean squared deviation of the counts from their mean.
 *   importance [E] fp32 out: m.
 *   dgate [T,k] fp32 out or NULL: dL/dgate, to pass to moe_layer_bwd.
 *   All sums run in a fixed order (deterministic).
 */
size_t moe_balance_loss_workspace_size(int T, int E, int k);
int moe_balance_loss(const int32_t* idx, const float* gate, int T, int E, int k, float lambda,
                     float* stats, float* importance, float* dgate, void* ws, size_t ws_bytes,
                     void* stream);

/*
 * moe_check_status -- synchronises `stream`, then reads and clears the
 * device status word of the current device.  Returns MOE_OK, MOE_ERR_CUDA
 * (a CUDA error), MOE_ERR_DEVICE_TIMEOUT if a bounded device wait expired
 * since the last check (codes 0x2nn: the kernel gave up, drained its copies,
 * freed its TMEM and returned; its outputs are undefined), or
 * MOE_ERR_DEVICE_CHECK if a kernel met invalid data and skipped it (0x120:
 * an expert id outside [0, E); 0x130: an expert-parallel row count that is
 * not a 128-multiple; 0x140: a row-space plan or source row outside the
 * token-axis quantiser's buffers; 0x1ff: shared memory not 1 KB aligned).  The
 * code is in moe_last_error()'s message.
 */
int moe_check_status(void* stream);

/*
 * moe_debug_expire_next_wait -- test hook for the bounded device waits (the
 * pages have no counterpart).  The next tensor-core GEMM launch of the
 * library (on any stream of this process) runs with its TMA producer issuing
 * no copies and every bounded wait limited to wait_ns nanoseconds, so that
 * the MMA issuer's wait for a full stage expires with nothing in flight; the
 * hook then resets itself.  That launch's outputs are undefined and
 * moe_check_status() afterwards returns MOE_ERR_DEVICE_TIMEOUT.  wait_ns <= 0
 * cancels a pending request.  Returns MOE_OK.
 */
int moe_debug_expire_next_wait(long long wait_ns);

/*
 * Measurement hook (the pages have no counterpart; it serves the benchmark).
 * moe_profile_enable(1): from now on every kernel the library launches is
 * bracketed by two CUDA events recorded on the kernel's own stream.
 * moe_profile_enable(0) stops recording.
 * moe_profile_report: waits for the recorded events, then writes one line
 * "<kernel> <launches> <total_ms> <median_ms>" per kernel name into buf
 * (NUL-terminated; median_ms is the median single-launch time) and forgets
 * the records.  Returns MOE_ERR_INVALID_ARG if buf is too small.
 */
int moe_profile_enable(int on);
int moe_profile_report(char* buf, size_t buf_len);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
