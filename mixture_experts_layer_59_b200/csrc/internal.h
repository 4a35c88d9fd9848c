// Host-side launchers shared between the translation units of the library.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// ---------------------------------------------------------------- routing
int launch_router_logits_simt(const void* x, const void* wg, int T, int d, int E, int dtype,
                              const float* bias, float* logits, cudaStream_t s);
int launch_topk_softmax(const float* logits_in, const float* bias, const float* noise,
                        float* logits_out, int T, int E, int k, int gate_mode, int32_t* idx,
                        float* gate, cudaStream_t s);

// ---------------------------------------------------------------- permutation
struct PermuteWs {
  int32_t* blockcnt;   // [nb, E]
  int32_t* blockbase;  // [nb, E]
  // exact plan (used as input of the rounding pass)
  int32_t* ex_counts;
  int32_t* ex_offsets;
  int32_t* ex_row_token;
  float* ex_row_gate;
  int32_t* ex_row_slot;
  double* lse;         // [T]
};
size_t permute_ws_bytes(int T, int E, int k, int round_mode, int tile);
int carve_permute_ws(void* ws, size_t bytes, int T, int E, int k, int round_mode, int tile,
                     PermuteWs* out);
int launch_permute_exact(const int32_t* idx, const float* gate, int T, int E, int k, int tile,
                         int32_t* counts, int32_t* offsets, int32_t* row_token, float* row_gate,
                         int32_t* row_slot, int32_t* slot_row, const PermuteWs& w, cudaStream_t s);
// Token rounding (capacity < 0) or capacity-factor dropping (capacity >= 0).
int launch_permute_round(const int32_t* idx, const float* gate, const float* logits, int T, int E,
                         int k, int tile, int gate_mode, int capacity, int32_t* counts,
                         int32_t* offsets, int32_t* row_token, float* row_gate, int32_t* row_slot,
                         int32_t* slot_row, int32_t* extra_row, const PermuteWs& w,
                         cudaStream_t s);

// ---------------------------------------------------------------- row ops
// dst[row] = src[token of row] for every row (token-order scatter: each source
// row read once); padding rows (token -1) zeroed.
int launch_scatter_rows(const void* src, const int32_t* slot_row, const int32_t* extra_row,
                        const int32_t* row_token, const int32_t* offsets, int T, int width, int E,
                        int k, int dtype, void* dst, cudaStream_t s);
// dx = bf16(sum of the token's dX_perm rows + dl W_gate^T), W_gate staged in smem.
bool dx_fused_ok(int d, int E);
int launch_dx_fused(const void* dxp, const int32_t* slot_row, const int32_t* extra_row,
                    const float* dl, const void* wg, int T, int d, int E, int k, void* dx,
                    cudaStream_t s);
// out[t] = sum over token t's rows (kept slots in order, then added rows by
// ascending expert) of (weighted ? row_gate[r] : 1) * src[r]; out fp32 or dtype.
int launch_token_reduce(const void* src, const float* row_gate, const int32_t* slot_row,
                        const int32_t* extra_row, int T, int width, int E, int k, int dtype,
                        bool weighted, bool out_f32, void* out, cudaStream_t s);
// dlogits and (optionally) the final dS rows from dS partials [cap, nparts].
// Optionally also writes dlogits split as bf16 hi + bf16 lo (tensor-core router GEMMs).
int launch_router_bwd(const float* ds_part, int nparts, const int32_t* idx, const float* gate,
                      const float* row_gate, const int32_t* slot_row, const int32_t* extra_row,
                      const float* gate_grad, const float* logits, int gate_mode, int T, int E,
                      int k, float* dlogits, float* dS_out, void* dl_hi, void* dl_lo,
                      cudaStream_t s);
// Load-balance loss lambda*CV^2, routing statistics and dL/dgate.
size_t balance_ws_bytes(int T, int E);
int launch_balance_loss(const int32_t* idx, const float* gate, int T, int E, int k, float lam,
                        float* stats, float* importance, float* dgate, void* ws, size_t ws_bytes,
                        cudaStream_t s);

// ---------------------------------------------------------------- CUDA-core GEMM path
struct FfnPtrs {
  const void *x, *w1, *w3, *w2;
  const int32_t *row_token, *offsets;
  int T, d, f, E, cap, dtype;
};
int simt_ffn_fwd(const FfnPtrs& p, void* H, void* act, void* Y, cudaStream_t s);
int simt_ffn_bwd(const FfnPtrs& p, const void* dout, const float* row_gate, const void* H,
                 float* dap, void* dH, void* gact, float* ds, void* dXp, void* dw1, void* dw3,
                 void* dw2, cudaStream_t s);
int simt_router_bwd_gemms(const void* x, const void* wg, const float* dl, const float* dx_acc,
                          int T, int d, int E, int dtype, float* dw_gate, void* dx, cudaStream_t s);

// ---------------------------------------------------------------- tensor-core path
bool tc_available();
int tc_ffn_fwd(const FfnPtrs& p, const void* xg, void* H, void* act, void* Y, int num_sms,
               cudaStream_t s);
int tc_ffn_fwd_mx(const FfnPtrs& p, const uint8_t* xq, const uint8_t* xs, const uint8_t* w13q,
                  const uint8_t* w13s, const uint8_t* w2q, const uint8_t* w2s, void* H,
                  uint8_t* actq, uint8_t* acts, void* Y, int num_sms, cudaStream_t s);
// MXFP8 operands of the backward dX GEMM (null: bf16 dX GEMM).
struct MxBwd {
  const uint8_t *w1rq, *w1rs, *w3rq, *w3rs;   // W1, W3 [E, d, f] quantised along f
  uint8_t *dhq, *dhs;                          // dH [cap, 2f] quantised along 2f (DAP writes it)
  // weight gradients on MXFP8 operands (wgrad = 1): x, dO, s*A and dH
  // quantised along the rows, [n, capr] E4M3 + scales; x is gathered from
  // the token rows through row_token
  int wgrad, capr, T;
  const void* x;
  const int32_t* row_token;
  uint8_t *xq, *xs, *oq, *os, *aq, *as, *hq, *hs;
};
int tc_ffn_bwd(const FfnPtrs& p, const void* dog, const void* xg, const float* row_gate,
               const void* H, void* dH, void* gact, float* ds_part, void* dXp, void* dw1,
               void* dw3, void* dw2, int num_sms, cudaStream_t s, const MxBwd* mx = nullptr);
int tc_num_dS_parts(int f);
bool tc_router_ok(int E);
int tc_dwg_splits(int T, int d, int* chunk);
int tc_router_fwd(const void* x, const void* wg, const float* bias, const float* noise, int T,
                  int d, int E, int k, int gate_mode, float* logits, int32_t* idx, float* gate,
                  int num_sms, cudaStream_t s);
int tc_router_bwd(const void* x, const void* wg, const void* dl_hi, const void* dl_lo, int T,
                  int d, int E, int k, float* dwg_part, float* dw_gate, const float* dx_acc,
                  void* dx, int num_sms, cudaStream_t s);

int device_sm_count();

// ---------------------------------------------------------------- expert parallelism (ep.cu)
int launch_ep_dispatch_counts(const int32_t* offsets, int E, int32_t* seg_rows, cudaStream_t s);
int launch_ep_receive_plan(const int32_t* recv_rows, int G, int El, int32_t* local_offsets,
                           int32_t* recv_row, cudaStream_t s);
// dS[r] = sum over p of ds_part[r, p] (fixed order) for r < offsets[E].
int launch_ds_rows(const float* ds_part, int nparts, const int32_t* offsets, int E, int rows,
                   float* dS, cudaStream_t s);

// Test hook of the bounded device waits: the wait limit (ns) requested for
// the next tensor-core GEMM launch, or 0; taking it clears the request.
long long take_debug_expire();

// ---------------------------------------------------------------- MXFP8 (mx.cu, tc_gemm.cu)
int launch_mx_quant_weights(const void* w1, const void* w3, const void* w2, int E, int d, int f,
                            uint8_t* w13q, uint8_t* w13s, uint8_t* w2q, uint8_t* w2s,
                            uint8_t* w1rq, uint8_t* w1rs, uint8_t* w3rq, uint8_t* w3rs,
                            cudaStream_t s);
int launch_mx_quant_cols(const void* src, int src_rows, const int32_t* gather_row,
                         const int32_t* offsets, int E, int n, int capr, uint8_t* q, uint8_t* sf,
                         cudaStream_t s);
int launch_mx_scatter_rows(const void* x, const int32_t* slot_row, const int32_t* extra_row,
                           const int32_t* row_token, const int32_t* offsets, int T, int d, int E,
                           int k, uint8_t* q, uint8_t* sf, cudaStream_t s);

}  // namespace moe
