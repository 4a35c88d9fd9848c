// extern "C" entry points: argument checks, workspace layout, kernel order.
#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace moe {

static thread_local std::string g_err = "";

void set_error(const std::string& msg) { g_err = msg; }
int fail(int code, const std::string& msg) {
  g_err = msg;
  return code;
}
int cuda_fail(cudaError_t e, const char* what) {
  g_err = std::string(what) + ": " + cudaGetErrorString(e);
  return MOE_ERR_CUDA;
}

__device__ int g_moe_status = 0;

// The host-side name of a __device__ variable is only a stand-in: its device
// address is looked up once per device (with that device current) and kept
// in an atomic slot, so concurrent host threads may race to fill it safely.
int* status_ptr() {
  static std::atomic<int*> cache[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  int* p = cache[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    void* q = nullptr;
    if (cudaGetSymbolAddress(&q, g_moe_status) == cudaSuccess) {
      p = static_cast<int*>(q);
      cache[dev].store(p, std::memory_order_release);
    }
  }
  return p;
}

static std::atomic<long long> g_debug_expire{0};

long long take_debug_expire() {
  if (g_debug_expire.load(std::memory_order_relaxed) == 0) return 0;
  return g_debug_expire.exchange(0);
}

// ------------------------------------------------------------ profiling hook
namespace {
std::mutex g_prof_mu;
bool g_prof_on = false;
struct ProfRec {
  std::string name;
  cudaEvent_t a, b;
};
std::vector<ProfRec> g_recs;
std::vector<cudaEvent_t> g_pool;

cudaEvent_t prof_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}
}  // namespace

ProfScope::ProfScope(const char* n, cudaStream_t s) : name(n), stream(s) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (!g_prof_on) return;
  start = prof_event();
  cudaEventRecord(start, stream);
}

ProfScope::~ProfScope() {
  if (start == nullptr) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  cudaEvent_t stop = prof_event();
  cudaEventRecord(stop, stream);
  g_recs.push_back(ProfRec{name, start, stop});
}

int device_sm_count() {
  static std::atomic<int> cache[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    n = n > 0 ? n : 1;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// ------------------------------------------------------------ checks
static int check_common(int T, int E, int k, int dtype) {
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T must be >= 0");
  if (k < 1 || k > 8) return fail(MOE_ERR_UNSUPPORTED, "k must be in [1, 8]");
  if (E < k || E > 256) return fail(MOE_ERR_UNSUPPORTED, "E must be in [k, 256]");
  if (dtype != MOE_F32 && dtype != MOE_BF16) return fail(MOE_ERR_UNSUPPORTED, "dtype must be MOE_F32 or MOE_BF16");
  return MOE_OK;
}

static int check_dims(int d, int f, int dtype) {
  const int q = dtype == MOE_BF16 ? 128 : 64;
  if (d <= 0 || d % q) return fail(MOE_ERR_UNSUPPORTED, "d must be a positive multiple of " + std::to_string(q));
  if (f < 0 || f % q || f == 0) return fail(MOE_ERR_UNSUPPORTED, "f must be a positive multiple of " + std::to_string(q));
  return MOE_OK;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define REQUIRE_PTR(p)                                                              \
  do {                                                                              \
    if ((p) == nullptr) return fail(MOE_ERR_INVALID_ARG, #p " must not be NULL");   \
  } while (0)
#define REQUIRE_ALIGNED(p)                                                                 \
  do {                                                                                     \
    if (!aligned16(p)) return fail(MOE_ERR_INVALID_ARG, #p " must be 16-byte aligned");     \
  } while (0)

static size_t esize(int dtype) { return dtype == MOE_BF16 ? 2 : 4; }

// ------------------------------------------------------------ workspace layouts
template <class A>
struct FwdWs {
  void* xg = nullptr;
  void* act = nullptr;
  void carve(A& a, int T, int d, int f, int E, int k, int dtype) {
    const size_t cap = (size_t)T * k + (size_t)E * 128;
    if (dtype == MOE_BF16 && tc_available()) xg = a.template take<uint16_t>(cap * d);
    act = a.template take<char>(cap * f * esize(dtype));
  }
};

template <class A>
struct FwdMxWs {
  uint8_t *xq = nullptr, *xs = nullptr, *actq = nullptr, *acts = nullptr;
  void carve(A& a, int T, int d, int f, int E, int k) {
    const size_t cap = (size_t)T * k + (size_t)E * 128;
    const size_t capr = (cap + 127) / 128 * 128;   // scale blocks cover 128 rows
    xq = a.template take<uint8_t>(capr * d);
    xs = a.template take<uint8_t>(capr * d / 32);
    actq = a.template take<uint8_t>(capr * f);
    acts = a.template take<uint8_t>(capr * f / 32);
  }
};

template <class A>
struct BwdWs {
  void *dog = nullptr, *xg = nullptr, *dH = nullptr, *gact = nullptr, *dxp = nullptr;
  float *dap = nullptr, *ds = nullptr, *dl = nullptr, *dx_acc = nullptr, *dwg_part = nullptr;
  void *dl_hi = nullptr, *dl_lo = nullptr;
  int nparts = 1;
  void carve(A& a, int T, int d, int f, int E, int k, int dtype) {
    const size_t cap = (size_t)T * k + (size_t)E * 128;
    const size_t es = esize(dtype);
    const bool tc = dtype == MOE_BF16 && tc_available();
    nparts = tc ? tc_num_dS_parts(f) : 1;
    if (tc) {
      dog = a.template take<char>(cap * d * es);
      xg = a.template take<char>(cap * d * es);
    } else {
      dap = a.template take<float>(cap * f);
    }
    dH = a.template take<char>(cap * 2 * f * es);
    gact = a.template take<char>(cap * f * es);
    dxp = a.template take<char>(cap * d * es);
    ds = a.template take<float>(cap * nparts);
    dl = a.template take<float>((size_t)T * E + 1);
    dx_acc = a.template take<float>((size_t)T * d + 1);
    if (tc && tc_router_ok(E)) {
      int chunk = 0;
      const int splits = tc_dwg_splits(T, d, &chunk);
      dl_hi = a.template take<uint16_t>((size_t)T * E + 8);
      dl_lo = a.template take<uint16_t>((size_t)T * E + 8);
      dwg_part = a.template take<float>((size_t)splits * d * E);
    }
  }
};

// Workspace of the token side of the backward (router gradient and dx).
struct TokenWs {
  float *dl, *dx_acc;
  void *dl_hi, *dl_lo;
  float* dwg_part;
};

template <class A>
struct TokenBwdWs {
  TokenWs w{};
  void carve(A& a, int T, int d, int E, int dtype) {
    const bool tc = dtype == MOE_BF16 && tc_available();
    w.dl = a.template take<float>((size_t)T * E + 1);
    w.dx_acc = a.template take<float>((size_t)T * d + 1);
    if (tc && tc_router_ok(E)) {
      int chunk = 0;
      const int splits = tc_dwg_splits(T, d, &chunk);
      w.dl_hi = a.template take<uint16_t>((size_t)T * E + 8);
      w.dl_lo = a.template take<uint16_t>((size_t)T * E + 8);
      w.dwg_part = a.template take<float>((size_t)splits * d * E);
    }
  }
};

}  // namespace moe

using namespace moe;

extern "C" {

int moe_version(void) { return 10000; }

const char* moe_last_error(void) { return g_err.c_str(); }

size_t moe_row_capacity(int T, int E, int k, int tile) {
  if (T < 0 || E < 0 || k < 0 || tile < 0) return 0;
  return (size_t)T * k + (size_t)E * tile;
}

int moe_route(const void* x, const void* w_gate, int T, int d, int E, int k, int dtype,
              int gate_mode, const float* logits_override, const float* logit_bias,
              const float* logit_noise, float* logits, int32_t* idx, float* gate,
              void* stream) {
  if (int rc = check_common(T, E, k, dtype)) return rc;
  if (gate_mode != MOE_GATE_TOPK_SOFTMAX && gate_mode != MOE_GATE_SOFTMAX_TOPK)
    return fail(MOE_ERR_INVALID_ARG, "gate_mode must be MOE_GATE_TOPK_SOFTMAX or MOE_GATE_SOFTMAX_TOPK");
  if (T == 0) return MOE_OK;
  REQUIRE_PTR(logits);
  REQUIRE_PTR(idx);
  REQUIRE_PTR(gate);
  cudaStream_t s = (cudaStream_t)stream;
  const float* src = logits_override;
  if (src == nullptr) {
    REQUIRE_PTR(x);
    REQUIRE_PTR(w_gate);
    if (d <= 0) return fail(MOE_ERR_INVALID_ARG, "d must be > 0");
    if (dtype == MOE_BF16 && d % 64 == 0 && tc_router_ok(E)) {
      // tensor-core router GEMM with the bias, top-k and softmax in its epilogue
      REQUIRE_ALIGNED(x);
      REQUIRE_ALIGNED(w_gate);
      return tc_router_fwd(x, w_gate, logit_bias, logit_noise, T, d, E, k, gate_mode, logits,
                           idx, gate, device_sm_count(), s);
    }
    if (int rc = launch_router_logits_simt(x, w_gate, T, d, E, dtype, nullptr, logits, s)) return rc;
    src = logits;
  }
  return launch_topk_softmax(src, logit_bias, logit_noise, logits, T, E, k, gate_mode, idx, gate,
                             s);
}

size_t moe_permute_workspace_size(int T, int E, int k, int round_mode) {
  if (T < 0 || E <= 0 || k <= 0) return 0;
  return permute_ws_bytes(T, E, k, round_mode, 128);
}

int moe_permute(const int32_t* idx, const float* gate, const float* logits, int T, int E, int k,
                int round_mode, int tile, int gate_mode, int capacity, int32_t* counts,
                int32_t* offsets, int32_t* row_token, float* row_gate, int32_t* row_slot,
                int32_t* slot_row, int32_t* extra_row, void* ws, size_t ws_bytes, void* stream) {
  if (int rc = check_common(T, E, k, MOE_F32)) return rc;
  if (tile != 128)
    return fail(MOE_ERR_UNSUPPORTED, "tile must be 128 (the grouped-GEMM M tile)");
  if (round_mode != MOE_ROUND_NONE && round_mode != MOE_ROUND_NEAREST &&
      round_mode != MOE_ROUND_CAPACITY)
    return fail(MOE_ERR_INVALID_ARG,
                "round_mode must be MOE_ROUND_NONE, MOE_ROUND_NEAREST or MOE_ROUND_CAPACITY");
  if (gate_mode != MOE_GATE_TOPK_SOFTMAX && gate_mode != MOE_GATE_SOFTMAX_TOPK)
    return fail(MOE_ERR_INVALID_ARG, "gate_mode must be MOE_GATE_TOPK_SOFTMAX or MOE_GATE_SOFTMAX_TOPK");
  if (round_mode == MOE_ROUND_CAPACITY && capacity < 0)
    return fail(MOE_ERR_INVALID_ARG, "capacity must be >= 0 with MOE_ROUND_CAPACITY");
  REQUIRE_PTR(counts);
  REQUIRE_PTR(offsets);
  if (T > 0) {
    REQUIRE_PTR(idx);
    REQUIRE_PTR(gate);
    REQUIRE_PTR(row_token);
    REQUIRE_PTR(row_gate);
    REQUIRE_PTR(row_slot);
    REQUIRE_PTR(slot_row);
  }
  if (round_mode != MOE_ROUND_NONE) REQUIRE_PTR(logits);
  if (round_mode == MOE_ROUND_NEAREST) REQUIRE_PTR(extra_row);
  if (ws_bytes < permute_ws_bytes(T, E, k, round_mode, tile))
    return fail(MOE_ERR_WORKSPACE, "permute workspace smaller than moe_permute_workspace_size()");
  PermuteWs w;
  if (int rc = carve_permute_ws(ws, ws_bytes, T, E, k, round_mode, tile, &w)) return rc;
  cudaStream_t s = (cudaStream_t)stream;
  if (round_mode == MOE_ROUND_NONE)
    return launch_permute_exact(idx, gate, T, E, k, tile, counts, offsets, row_token, row_gate,
                                row_slot, slot_row, w, s);
  // capacity mode adds no pairs, so it never writes extra_row
  return launch_permute_round(idx, gate, logits, T, E, k, tile, gate_mode,
                              round_mode == MOE_ROUND_CAPACITY ? capacity : -1, counts, offsets,
                              row_token, row_gate, row_slot, slot_row,
                              round_mode == MOE_ROUND_CAPACITY ? nullptr : extra_row, w, s);
}

size_t moe_ffn_fwd_workspace_size(int T, int d, int f, int E, int k, int dtype) {
  if (T < 0 || d <= 0 || f <= 0 || E <= 0 || k <= 0) return 0;
  Sizer z;
  FwdWs<Sizer> w;
  w.carve(z, T, d, f, E, k, dtype);
  return z.used;
}

int moe_expert_ffn_fwd(const void* x, const void* w1, const void* w3, const void* w2,
                       const int32_t* row_token, const int32_t* offsets, const int32_t* slot_row,
                       const int32_t* extra_row, int T, int d, int f, int E, int k, int dtype,
                       void* H, void* Y_perm, void* ws, size_t ws_bytes, void* stream) {
  if (int rc = check_common(T, E, k, dtype)) return rc;
  if (int rc = check_dims(d, f, dtype)) return rc;
  REQUIRE_PTR(x); REQUIRE_PTR(w1); REQUIRE_PTR(w3); REQUIRE_PTR(w2);
  REQUIRE_PTR(row_token); REQUIRE_PTR(offsets); REQUIRE_PTR(H); REQUIRE_PTR(Y_perm);
  if (T > 0) REQUIRE_PTR(slot_row);
  REQUIRE_ALIGNED(x); REQUIRE_ALIGNED(w1); REQUIRE_ALIGNED(w3); REQUIRE_ALIGNED(w2);
  REQUIRE_ALIGNED(H); REQUIRE_ALIGNED(Y_perm); REQUIRE_ALIGNED(ws);
  if (ws_bytes < moe_ffn_fwd_workspace_size(T, d, f, E, k, dtype))
    return fail(MOE_ERR_WORKSPACE, "ffn workspace smaller than moe_ffn_fwd_workspace_size()");
  Carve c(ws, ws_bytes);
  FwdWs<Carve> w;
  w.carve(c, T, d, f, E, k, dtype);
  if (!c.ok) return fail(MOE_ERR_WORKSPACE, "ffn workspace too small");
  cudaStream_t s = (cudaStream_t)stream;
  FfnPtrs p{x, w1, w3, w2, row_token, offsets, T, d, f, E, (int)((size_t)T * k + (size_t)E * 128), dtype};
  if (dtype == MOE_BF16 && tc_available()) {
    if (int rc = launch_scatter_rows(x, slot_row, extra_row, row_token, offsets, T, d, E, k, dtype,
                                     w.xg, s))
      return rc;
    return tc_ffn_fwd(p, w.xg, H, w.act, Y_perm, device_sm_count(), s);
  }
  return simt_ffn_fwd(p, H, w.act, Y_perm, s);
}

int moe_mxfp8_weight_sizes(int E, int d, int f, size_t* sizes) {
  REQUIRE_PTR(sizes);
  if (E < 0 || d <= 0 || f <= 0 || d % 128 || f % 128)
    return fail(MOE_ERR_UNSUPPORTED, "MXFP8 needs d and f positive multiples of 128");
  const size_t n = (size_t)E * d * f;
  sizes[0] = 2 * n;        // W13q
  sizes[1] = 2 * n / 32;   // W13s
  sizes[2] = n;            // W2q
  sizes[3] = n / 32;       // W2s
  sizes[4] = n;            // W1r (backward dX GEMM)
  sizes[5] = n / 32;
  sizes[6] = n;            // W3r
  sizes[7] = n / 32;
  return MOE_OK;
}

int moe_mxfp8_quantize_tokens(const void* src, int src_rows, const int32_t* gather_row,
                              const int32_t* offsets, int E, int n, int capr, uint8_t* q,
                              uint8_t* sf, void* stream) {
  if (E < 1 || E > 256) return fail(MOE_ERR_UNSUPPORTED, "E must be in [1, 256]");
  if (src_rows < 0) return fail(MOE_ERR_INVALID_ARG, "src_rows must be >= 0");
  if (n <= 0 || n % 128 || capr <= 0 || capr % 128)
    return fail(MOE_ERR_UNSUPPORTED, "n and capr must be positive multiples of 128");
  REQUIRE_PTR(src); REQUIRE_PTR(offsets); REQUIRE_PTR(q); REQUIRE_PTR(sf);
  REQUIRE_ALIGNED(src); REQUIRE_ALIGNED(q);
  return launch_mx_quant_cols(src, src_rows, gather_row, offsets, E, n, capr, q, sf,
                              (cudaStream_t)stream);
}

int moe_mxfp8_quantize_weights(const void* w1, const void* w3, const void* w2, int E, int d,
                               int f, uint8_t* w13q, uint8_t* w13s, uint8_t* w2q, uint8_t* w2s,
                               uint8_t* w1rq, uint8_t* w1rs, uint8_t* w3rq, uint8_t* w3rs,
                               void* stream) {
  size_t sz[8];
  if (int rc = moe_mxfp8_weight_sizes(E, d, f, sz)) return rc;
  if (E < 1 || E > 256) return fail(MOE_ERR_UNSUPPORTED, "E must be in [1, 256]");
  REQUIRE_PTR(w1); REQUIRE_PTR(w3); REQUIRE_PTR(w2);
  REQUIRE_PTR(w13q); REQUIRE_PTR(w13s); REQUIRE_PTR(w2q); REQUIRE_PTR(w2s);
  REQUIRE_ALIGNED(w1); REQUIRE_ALIGNED(w3); REQUIRE_ALIGNED(w2);
  REQUIRE_ALIGNED(w13q); REQUIRE_ALIGNED(w13s); REQUIRE_ALIGNED(w2q); REQUIRE_ALIGNED(w2s);
  const bool bwd = w1rq != nullptr;
  if (bwd != (w1rs != nullptr) || bwd != (w3rq != nullptr) || bwd != (w3rs != nullptr))
    return fail(MOE_ERR_INVALID_ARG, "w1rq, w1rs, w3rq, w3rs must be all set or all NULL");
  if (bwd) {
    REQUIRE_ALIGNED(w1rq); REQUIRE_ALIGNED(w1rs); REQUIRE_ALIGNED(w3rq); REQUIRE_ALIGNED(w3rs);
  }
  return launch_mx_quant_weights(w1, w3, w2, E, d, f, w13q, w13s, w2q, w2s, w1rq, w1rs, w3rq,
                                 w3rs, (cudaStream_t)stream);
}

size_t moe_ffn_fwd_mxfp8_workspace_size(int T, int d, int f, int E, int k) {
  if (T < 0 || d <= 0 || f <= 0 || E <= 0 || k <= 0) return 0;
  Sizer z;
  FwdMxWs<Sizer> w;
  w.carve(z, T, d, f, E, k);
  return z.used;
}

int moe_expert_ffn_fwd_mxfp8(const void* x, const uint8_t* w13q, const uint8_t* w13s,
                             const uint8_t* w2q, const uint8_t* w2s, const int32_t* row_token,
                             const int32_t* offsets, const int32_t* slot_row,
                             const int32_t* extra_row, int T, int d, int f, int E, int k, void* H,
                             void* Y_perm, void* ws, size_t ws_bytes, void* stream) {
  if (int rc = check_common(T, E, k, MOE_BF16)) return rc;
  if (int rc = check_dims(d, f, MOE_BF16)) return rc;
  if (!tc_available()) return fail(MOE_ERR_UNSUPPORTED, "MXFP8 GEMMs need an sm_100 device");
  REQUIRE_PTR(x); REQUIRE_PTR(w13q); REQUIRE_PTR(w13s); REQUIRE_PTR(w2q); REQUIRE_PTR(w2s);
  REQUIRE_PTR(row_token); REQUIRE_PTR(offsets); REQUIRE_PTR(H); REQUIRE_PTR(Y_perm);
  if (T > 0) REQUIRE_PTR(slot_row);
  REQUIRE_ALIGNED(x); REQUIRE_ALIGNED(w13q); REQUIRE_ALIGNED(w13s); REQUIRE_ALIGNED(w2q);
  REQUIRE_ALIGNED(w2s); REQUIRE_ALIGNED(H); REQUIRE_ALIGNED(Y_perm); REQUIRE_ALIGNED(ws);
  if (ws_bytes < moe_ffn_fwd_mxfp8_workspace_size(T, d, f, E, k))
    return fail(MOE_ERR_WORKSPACE, "workspace smaller than moe_ffn_fwd_mxfp8_workspace_size()");
  Carve c(ws, ws_bytes);
  FwdMxWs<Carve> w;
  w.carve(c, T, d, f, E, k);
  if (!c.ok) return fail(MOE_ERR_WORKSPACE, "mxfp8 workspace too small");
  cudaStream_t s = (cudaStream_t)stream;
  FfnPtrs p{x, nullptr, nullptr, nullptr, row_token, offsets, T, d, f, E,
            (int)((size_t)T * k + (size_t)E * 128), MOE_BF16};
  if (int rc = launch_mx_scatter_rows(x, slot_row, extra_row, row_token, offsets, T, d, E, k,
                                      w.xq, w.xs, s))
    return rc;
  return tc_ffn_fwd_mx(p, w.xq, w.xs, w13q, w13s, w2q, w2s, H, w.actq, w.acts, Y_perm,
                       device_sm_count(), s);
}

int moe_combine(const void* Y_perm, const float* row_gate, const int32_t* slot_row,
                const int32_t* extra_row, int T, int d, int E, int k, int dtype, void* out,
                void* stream) {
  if (int rc = check_common(T, E, k, dtype)) return rc;
  if (d <= 0 || d % 8) return fail(MOE_ERR_UNSUPPORTED, "d must be a positive multiple of 8");
  if (T == 0) return MOE_OK;
  REQUIRE_PTR(Y_perm); REQUIRE_PTR(row_gate); REQUIRE_PTR(slot_row); REQUIRE_PTR(out);
  REQUIRE_ALIGNED(Y_perm); REQUIRE_ALIGNED(out);
  return launch_token_reduce(Y_perm, row_gate, slot_row, extra_row, T, d, E, k, dtype, true,
                             false, out, (cudaStream_t)stream);
}

size_t moe_layer_bwd_workspace_size(int T, int d, int f, int E, int k, int dtype) {
  if (T < 0 || d <= 0 || f <= 0 || E <= 0 || k <= 0) return 0;
  Sizer z;
  BwdWs<Sizer> w;
  w.carve(z, T, d, f, E, k, dtype);
  return z.used;
}

// Token side of the backward, from the expert side's per-row results:
// dlogits from dS (partials summed in a fixed order), dW_gate = x^T dlogits,
// dx = unpermute-sum of dX_perm + dlogits W_gate^T.
static int token_bwd_impl(const void* dxp, const float* ds_part, int nparts, const void* x,
                          const void* w_gate, const int32_t* idx, const float* gate,
                          const float* gate_grad, const float* logits, int gate_mode,
                          const float* row_gate, const int32_t* slot_row,
                          const int32_t* extra_row, int T, int d, int E, int k, int dtype,
                          int router_grad, void* dx, float* dw_gate, float* dS, float* dlogits,
                          const TokenWs& w, cudaStream_t s) {
  int rc;
  float* dl = dlogits ? dlogits : w.dl;
  const bool tc_router = router_grad && w.dl_hi != nullptr;
  if ((rc = launch_router_bwd(ds_part, nparts, idx, gate, row_gate, slot_row, extra_row,
                              gate_grad, logits, gate_mode, T, E, k, dl, dS,
                              tc_router ? w.dl_hi : nullptr,
                              tc_router ? w.dl_lo : nullptr, s)))
    return rc;
  if (tc_router) {
    // dW_gate on the tensor cores (split-K, hi/lo dlogits); dx = unpermute-sum
    // of dX_perm + dl W_gate^T: one CUDA-core pass when W_gate fits in shared
    // memory, otherwise fp32 row sums + the tensor-core router term
    if (dx_fused_ok(d, E)) {
      if ((rc = tc_router_bwd(x, w_gate, w.dl_hi, w.dl_lo, T, d, E, k, w.dwg_part, dw_gate,
                              nullptr, nullptr, device_sm_count(), s)))
        return rc;
      return launch_dx_fused(dxp, slot_row, extra_row, dl, w_gate, T, d, E, k, dx, s);
    }
    if ((rc = launch_token_reduce(dxp, row_gate, slot_row, extra_row, T, d, E, k, dtype, false,
                                  true, w.dx_acc, s)))
      return rc;
    return tc_router_bwd(x, w_gate, w.dl_hi, w.dl_lo, T, d, E, k, w.dwg_part, dw_gate, w.dx_acc,
                         dx, device_sm_count(), s);
  }
  if (router_grad) {
    if ((rc = launch_token_reduce(dxp, row_gate, slot_row, extra_row, T, d, E, k, dtype, false,
                                  true, w.dx_acc, s)))
      return rc;
    return simt_router_bwd_gemms(x, w_gate, dl, w.dx_acc, T, d, E, dtype, dw_gate, dx, s);
  }
  cudaError_t e = cudaMemsetAsync(dw_gate, 0, (size_t)d * E * sizeof(float), s);
  if (e != cudaSuccess) return cuda_fail(e, "memset dw_gate");
  return launch_token_reduce(dxp, row_gate, slot_row, extra_row, T, d, E, k, dtype, false, false,
                             dx, s);
}

static int layer_bwd_impl(const void* dout, const void* x, const void* w_gate, const void* w1,
                  const void* w3, const void* w2, const int32_t* idx, const float* gate,
                  const float* gate_grad, const float* logits, int gate_mode,
                  const int32_t* offsets, const int32_t* row_token, const float* row_gate,
                  const int32_t* slot_row, const int32_t* extra_row, const void* H, int T, int d,
                  int f, int E, int k, int dtype, int router_grad, void* dx, float* dw_gate,
                  void* dw1, void* dw3, void* dw2, float* dS, float* dlogits, void* ws,
                  size_t ws_bytes, void* stream, const uint8_t* const* mxw, int mx_wgrad = 0) {
  if (int rc = check_common(T, E, k, dtype)) return rc;
  if (int rc = check_dims(d, f, dtype)) return rc;
  REQUIRE_PTR(dout); REQUIRE_PTR(x); REQUIRE_PTR(w1); REQUIRE_PTR(w3); REQUIRE_PTR(w2);
  REQUIRE_PTR(idx); REQUIRE_PTR(gate); REQUIRE_PTR(offsets); REQUIRE_PTR(row_token);
  REQUIRE_PTR(row_gate); REQUIRE_PTR(slot_row); REQUIRE_PTR(H); REQUIRE_PTR(dx);
  REQUIRE_PTR(dw_gate); REQUIRE_PTR(dw1); REQUIRE_PTR(dw3); REQUIRE_PTR(dw2);
  if (router_grad) REQUIRE_PTR(w_gate);
  if (gate_mode != MOE_GATE_TOPK_SOFTMAX && gate_mode != MOE_GATE_SOFTMAX_TOPK)
    return fail(MOE_ERR_INVALID_ARG, "gate_mode must be MOE_GATE_TOPK_SOFTMAX or MOE_GATE_SOFTMAX_TOPK");
  if (gate_mode == MOE_GATE_SOFTMAX_TOPK) REQUIRE_PTR(logits);
  REQUIRE_ALIGNED(dout); REQUIRE_ALIGNED(x); REQUIRE_ALIGNED(w1); REQUIRE_ALIGNED(w3);
  REQUIRE_ALIGNED(w2); REQUIRE_ALIGNED(H); REQUIRE_ALIGNED(dx); REQUIRE_ALIGNED(dw1);
  REQUIRE_ALIGNED(dw3); REQUIRE_ALIGNED(dw2); REQUIRE_ALIGNED(ws);
  const size_t need = mxw ? moe_layer_bwd_mxfp8_workspace_size(T, d, f, E, k, mx_wgrad)
                         : moe_layer_bwd_workspace_size(T, d, f, E, k, dtype);
  if (ws_bytes < need)
    return fail(MOE_ERR_WORKSPACE, "bwd workspace smaller than the matching *_workspace_size()");
  Carve c(ws, ws_bytes);
  BwdWs<Carve> w;
  w.carve(c, T, d, f, E, k, dtype);
  MxBwd mx{};
  if (mxw) {  // dH in MXFP8 for the dX GEMM, after the bf16 workspace
    const size_t capr = ((size_t)T * k + (size_t)E * 128 + 127) / 128 * 128;
    mx = MxBwd{mxw[0], mxw[1], mxw[2], mxw[3], c.take<uint8_t>(capr * 2 * f),
               c.take<uint8_t>(capr * 2 * f / 32)};
    if (mx_wgrad) {   // x, dO, s*A, dH quantised along the rows for the dW GEMMs
      mx.wgrad = 1;
      mx.capr = (int)capr;
      mx.T = T;
      mx.x = x;
      mx.row_token = row_token;
      mx.xq = c.take<uint8_t>(capr * d);
      mx.xs = c.take<uint8_t>(capr * d / 32);
      mx.oq = c.take<uint8_t>(capr * d);
      mx.os = c.take<uint8_t>(capr * d / 32);
      mx.aq = c.take<uint8_t>(capr * f);
      mx.as = c.take<uint8_t>(capr * f / 32);
      mx.hq = c.take<uint8_t>(capr * 2 * f);
      mx.hs = c.take<uint8_t>(capr * 2 * f / 32);
    }
  }
  if (!c.ok) return fail(MOE_ERR_WORKSPACE, "bwd workspace too small");
  cudaStream_t s = (cudaStream_t)stream;
  FfnPtrs p{x, w1, w3, w2, row_token, offsets, T, d, f, E, (int)((size_t)T * k + (size_t)E * 128), dtype};
  int rc;
  if (dtype == MOE_BF16 && tc_available()) {
    if ((rc = launch_scatter_rows(dout, slot_row, extra_row, row_token, offsets, T, d, E, k, dtype,
                                  w.dog, s)))
      return rc;
    if (!mx.wgrad &&   // (MXFP8 weight gradients quantise x straight from the token rows)
        (rc = launch_scatter_rows(x, slot_row, extra_row, row_token, offsets, T, d, E, k, dtype,
                                  w.xg, s)))
      return rc;
    if ((rc = tc_ffn_bwd(p, w.dog, w.xg, row_gate, H, w.dH, w.gact, w.ds, w.dxp, dw1, dw3, dw2,
                         device_sm_count(), s, mxw ? &mx : nullptr)))
      return rc;
  } else {
    if ((rc = simt_ffn_bwd(p, dout, row_gate, H, w.dap, w.dH, w.gact, w.ds, w.dxp, dw1, dw3, dw2, s)))
      return rc;
  }
  return token_bwd_impl(w.dxp, w.ds, w.nparts, x, w_gate, idx, gate, gate_grad, logits, gate_mode,
                        row_gate, slot_row, extra_row, T, d, E, k, dtype, router_grad, dx, dw_gate,
                        dS, dlogits, TokenWs{w.dl, w.dx_acc, w.dl_hi, w.dl_lo, w.dwg_part}, s);
}

int moe_layer_bwd(const void* dout, const void* x, const void* w_gate, const void* w1,
                  const void* w3, const void* w2, const int32_t* idx, const float* gate,
                  const float* gate_grad, const float* logits, int gate_mode,
                  const int32_t* offsets, const int32_t* row_token, const float* row_gate,
                  const int32_t* slot_row, const int32_t* extra_row, const void* H, int T, int d,
                  int f, int E, int k, int dtype, int router_grad, void* dx, float* dw_gate,
                  void* dw1, void* dw3, void* dw2, float* dS, float* dlogits, void* ws,
                  size_t ws_bytes, void* stream) {
  return layer_bwd_impl(dout, x, w_gate, w1, w3, w2, idx, gate, gate_grad, logits, gate_mode,
                        offsets, row_token, row_gate, slot_row, extra_row, H, T, d, f, E, k, dtype,
                        router_grad, dx, dw_gate, dw1, dw3, dw2, dS, dlogits, ws, ws_bytes, stream,
                        nullptr);
}

size_t moe_layer_bwd_mxfp8_workspace_size(int T, int d, int f, int E, int k, int wgrad_mxfp8) {
  if (T < 0 || d <= 0 || f <= 0 || E <= 0 || k <= 0) return 0;
  Sizer z;
  BwdWs<Sizer> w;
  w.carve(z, T, d, f, E, k, MOE_BF16);
  const size_t capr = ((size_t)T * k + (size_t)E * 128 + 127) / 128 * 128;
  z.take<uint8_t>(capr * 2 * f);
  z.take<uint8_t>(capr * 2 * f / 32);
  if (wgrad_mxfp8) {
    for (size_t n : {(size_t)d, (size_t)d, (size_t)f, (size_t)2 * f}) {
      z.take<uint8_t>(capr * n);
      z.take<uint8_t>(capr * n / 32);
    }
  }
  return z.used;
}

int moe_layer_bwd_mxfp8(const void* dout, const void* x, const void* w_gate, const void* w1,
                        const void* w3, const void* w2, const uint8_t* w1rq, const uint8_t* w1rs,
                        const uint8_t* w3rq, const uint8_t* w3rs, const int32_t* idx,
                        const float* gate, const float* gate_grad, const float* logits,
                        int gate_mode, const int32_t* offsets, const int32_t* row_token,
                        const float* row_gate, const int32_t* slot_row, const int32_t* extra_row,
                        const void* H, int T, int d, int f, int E, int k, int router_grad,
                        int wgrad_mxfp8, void* dx, float* dw_gate, void* dw1, void* dw3,
                        void* dw2, float* dS, float* dlogits, void* ws, size_t ws_bytes,
                        void* stream) {
  REQUIRE_PTR(w1rq); REQUIRE_PTR(w1rs); REQUIRE_PTR(w3rq); REQUIRE_PTR(w3rs);
  if (wgrad_mxfp8 != 0 && wgrad_mxfp8 != 1) return fail(MOE_ERR_INVALID_ARG, "wgrad_mxfp8 must be 0 or 1");
  if (wgrad_mxfp8 && (d % 256 || (2 * f) % 256))
    return fail(MOE_ERR_UNSUPPORTED, "MXFP8 weight gradients need d and 2f multiples of 256");
  REQUIRE_ALIGNED(w1rq); REQUIRE_ALIGNED(w1rs); REQUIRE_ALIGNED(w3rq); REQUIRE_ALIGNED(w3rs);
  if (!tc_available()) return fail(MOE_ERR_UNSUPPORTED, "MXFP8 GEMMs need an sm_100 device");
  const uint8_t* mxw[4] = {w1rq, w1rs, w3rq, w3rs};
  return layer_bwd_impl(dout, x, w_gate, w1, w3, w2, idx, gate, gate_grad, logits, gate_mode,
                        offsets, row_token, row_gate, slot_row, extra_row, H, T, d, f, E, k,
                        MOE_BF16, router_grad, dx, dw_gate, dw1, dw3, dw2, dS, dlogits, ws,
                        ws_bytes, stream, mxw, wgrad_mxfp8);
}

// ------------------------------------------------------------ row-space pieces
// (expert parallelism: the token side and the expert side of the layer run on
// different ranks, with the permuted rows exchanged in between)

int moe_gather_rows(const void* src, const int32_t* row_token, const int32_t* offsets,
                    const int32_t* slot_row, const int32_t* extra_row, int T, int width, int E,
                    int k, int dtype, void* dst, void* stream) {
  if (int rc = check_common(T, E, k, dtype)) return rc;
  if (width <= 0 || width % 8) return fail(MOE_ERR_UNSUPPORTED, "width must be a positive multiple of 8");
  REQUIRE_PTR(row_token); REQUIRE_PTR(offsets); REQUIRE_PTR(dst);
  if (T > 0) { REQUIRE_PTR(src); REQUIRE_PTR(slot_row); }
  REQUIRE_ALIGNED(src); REQUIRE_ALIGNED(dst);
  return launch_scatter_rows(src, slot_row, extra_row, row_token, offsets, T, width, E, k, dtype,
                             dst, (cudaStream_t)stream);
}

static int check_rows_args(int rows, int d, int f, int E, int dtype) {
  if (dtype != MOE_BF16) return fail(MOE_ERR_UNSUPPORTED, "the row-space entry points take bf16");
  if (!tc_available()) return fail(MOE_ERR_UNSUPPORTED, "the row-space entry points need an sm_100 device");
  if (E < 1 || E > 256) return fail(MOE_ERR_UNSUPPORTED, "E must be in [1, 256]");
  if (rows < 128 || rows % 128) return fail(MOE_ERR_UNSUPPORTED, "rows must be a positive multiple of 128");
  return check_dims(d, f, dtype);
}

size_t moe_expert_rows_fwd_workspace_size(int rows, int f, int dtype) {
  if (rows < 0 || f <= 0) return 0;
  Sizer z;
  z.take<char>((size_t)rows * f * esize(dtype));
  return z.used;
}

int moe_expert_rows_fwd(const void* xg, const void* w1, const void* w3, const void* w2,
                        const int32_t* offsets, int rows, int d, int f, int E, int dtype, void* H,
                        void* Y, void* ws, size_t ws_bytes, void* stream) {
  if (int rc = check_rows_args(rows, d, f, E, dtype)) return rc;
  REQUIRE_PTR(xg); REQUIRE_PTR(w1); REQUIRE_PTR(w3); REQUIRE_PTR(w2); REQUIRE_PTR(offsets);
  REQUIRE_PTR(H); REQUIRE_PTR(Y);
  REQUIRE_ALIGNED(xg); REQUIRE_ALIGNED(w1); REQUIRE_ALIGNED(w3); REQUIRE_ALIGNED(w2);
  REQUIRE_ALIGNED(H); REQUIRE_ALIGNED(Y); REQUIRE_ALIGNED(ws);
  if (ws_bytes < moe_expert_rows_fwd_workspace_size(rows, f, dtype))
    return fail(MOE_ERR_WORKSPACE, "workspace smaller than moe_expert_rows_fwd_workspace_size()");
  Carve c(ws, ws_bytes);
  void* act = c.take<char>((size_t)rows * f * esize(dtype));
  if (!c.ok) return fail(MOE_ERR_WORKSPACE, "workspace too small");
  FfnPtrs p{nullptr, w1, w3, w2, nullptr, offsets, 0, d, f, E, rows, dtype};
  return tc_ffn_fwd(p, xg, H, act, Y, device_sm_count(), (cudaStream_t)stream);
}

size_t moe_expert_rows_bwd_workspace_size(int rows, int d, int f, int dtype) {
  if (rows < 0 || d <= 0 || f <= 0) return 0;
  const size_t es = esize(dtype);
  Sizer z;
  z.take<char>((size_t)rows * 2 * f * es);                  // dH
  z.take<char>((size_t)rows * f * es);                      // s * A
  z.take<float>((size_t)rows * tc_num_dS_parts(f));         // dS partials
  return z.used;
}

int moe_expert_rows_bwd(const void* dog, const void* xg, const float* row_gate, const void* H,
                        const void* w1, const void* w3, const void* w2, const int32_t* offsets,
                        int rows, int d, int f, int E, int dtype, void* dX_rows, float* dS,
                        void* dw1, void* dw3, void* dw2, void* ws, size_t ws_bytes,
                        void* stream) {
  if (int rc = check_rows_args(rows, d, f, E, dtype)) return rc;
  REQUIRE_PTR(dog); REQUIRE_PTR(xg); REQUIRE_PTR(row_gate); REQUIRE_PTR(H); REQUIRE_PTR(w1);
  REQUIRE_PTR(w3); REQUIRE_PTR(w2); REQUIRE_PTR(offsets); REQUIRE_PTR(dX_rows); REQUIRE_PTR(dS);
  REQUIRE_PTR(dw1); REQUIRE_PTR(dw3); REQUIRE_PTR(dw2);
  REQUIRE_ALIGNED(dog); REQUIRE_ALIGNED(xg); REQUIRE_ALIGNED(H); REQUIRE_ALIGNED(w1);
  REQUIRE_ALIGNED(w3); REQUIRE_ALIGNED(w2); REQUIRE_ALIGNED(dX_rows); REQUIRE_ALIGNED(dw1);
  REQUIRE_ALIGNED(dw3); REQUIRE_ALIGNED(dw2); REQUIRE_ALIGNED(ws);
  if (ws_bytes < moe_expert_rows_bwd_workspace_size(rows, d, f, dtype))
    return fail(MOE_ERR_WORKSPACE, "workspace smaller than moe_expert_rows_bwd_workspace_size()");
  const size_t es = esize(dtype);
  const int nparts = tc_num_dS_parts(f);
  Carve c(ws, ws_bytes);
  void* dH = c.take<char>((size_t)rows * 2 * f * es);
  void* gact = c.take<char>((size_t)rows * f * es);
  float* ds_part = c.take<float>((size_t)rows * nparts);
  if (!c.ok) return fail(MOE_ERR_WORKSPACE, "workspace too small");
  cudaStream_t s = (cudaStream_t)stream;
  FfnPtrs p{nullptr, w1, w3, w2, nullptr, offsets, 0, d, f, E, rows, dtype};
  if (int rc = tc_ffn_bwd(p, dog, xg, row_gate, H, dH, gact, ds_part, dX_rows, dw1, dw3, dw2,
                          device_sm_count(), s))
    return rc;
  return launch_ds_rows(ds_part, nparts, offsets, E, rows, dS, s);
}

size_t moe_token_bwd_workspace_size(int T, int d, int E, int k, int dtype) {
  (void)k;
  if (T < 0 || d <= 0 || E <= 0) return 0;
  Sizer z;
  TokenBwdWs<Sizer> w;
  w.carve(z, T, d, E, dtype);
  return z.used;
}

int moe_token_bwd(const void* dX_rows, const float* dS, const void* x, const void* w_gate,
                  const int32_t* idx, const float* gate, const float* gate_grad,
                  const float* logits, int gate_mode, const float* row_gate,
                  const int32_t* slot_row, const int32_t* extra_row, int T, int d, int E, int k,
                  int dtype, int router_grad, void* dx, float* dw_gate, float* dlogits, void* ws,
                  size_t ws_bytes, void* stream) {
  if (int rc = check_common(T, E, k, dtype)) return rc;
  if (d <= 0 || d % 8) return fail(MOE_ERR_UNSUPPORTED, "d must be a positive multiple of 8");
  if (gate_mode != MOE_GATE_TOPK_SOFTMAX && gate_mode != MOE_GATE_SOFTMAX_TOPK)
    return fail(MOE_ERR_INVALID_ARG, "gate_mode must be MOE_GATE_TOPK_SOFTMAX or MOE_GATE_SOFTMAX_TOPK");
  REQUIRE_PTR(dX_rows); REQUIRE_PTR(dS); REQUIRE_PTR(x); REQUIRE_PTR(idx); REQUIRE_PTR(gate);
  REQUIRE_PTR(row_gate); REQUIRE_PTR(slot_row); REQUIRE_PTR(dx); REQUIRE_PTR(dw_gate);
  if (router_grad) REQUIRE_PTR(w_gate);
  if (gate_mode == MOE_GATE_SOFTMAX_TOPK) REQUIRE_PTR(logits);
  REQUIRE_ALIGNED(dX_rows); REQUIRE_ALIGNED(x); REQUIRE_ALIGNED(w_gate); REQUIRE_ALIGNED(dx);
  REQUIRE_ALIGNED(ws);
  if (ws_bytes < moe_token_bwd_workspace_size(T, d, E, k, dtype))
    return fail(MOE_ERR_WORKSPACE, "workspace smaller than moe_token_bwd_workspace_size()");
  if (T == 0) return MOE_OK;
  Carve c(ws, ws_bytes);
  TokenBwdWs<Carve> w;
  w.carve(c, T, d, E, dtype);
  if (!c.ok) return fail(MOE_ERR_WORKSPACE, "workspace too small");
  return token_bwd_impl(dX_rows, dS, 1, x, w_gate, idx, gate, gate_grad, logits, gate_mode,
                        row_gate, slot_row, extra_row, T, d, E, k, dtype, router_grad, dx, dw_gate,
                        nullptr, dlogits, w.w, (cudaStream_t)stream);
}

int moe_ep_dispatch_counts(const int32_t* offsets, int E, int32_t* seg_rows, void* stream) {
  if (E < 1 || E > 256) return fail(MOE_ERR_UNSUPPORTED, "E must be in [1, 256]");
  REQUIRE_PTR(offsets); REQUIRE_PTR(seg_rows);
  return launch_ep_dispatch_counts(offsets, E, seg_rows, (cudaStream_t)stream);
}

int moe_ep_receive_plan(const int32_t* recv_rows, int G, int El, int32_t* local_offsets,
                        int32_t* recv_row, void* stream) {
  if (G < 1) return fail(MOE_ERR_INVALID_ARG, "G must be >= 1");
  if (El < 1 || El > 256) return fail(MOE_ERR_UNSUPPORTED, "El must be in [1, 256]");
  REQUIRE_PTR(recv_rows); REQUIRE_PTR(local_offsets); REQUIRE_PTR(recv_row);
  return launch_ep_receive_plan(recv_rows, G, El, local_offsets, recv_row, (cudaStream_t)stream);
}

int moe_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = on != 0;
  return MOE_OK;
}

int moe_profile_report(char* buf, size_t buf_len) {
  if (buf == nullptr || buf_len == 0) return fail(MOE_ERR_INVALID_ARG, "buf must not be NULL");
  std::lock_guard<std::mutex> lk(g_prof_mu);
  std::map<std::string, std::vector<float>> agg;   // launch times per kernel name
  int rc = MOE_OK;
  for (auto& r : g_recs) {
    float ms = 0.f;
    cudaError_t e = cudaEventSynchronize(r.b);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, r.a, r.b);
    if (e != cudaSuccess) rc = cuda_fail(e, "profile event");
    agg[r.name].push_back(ms);
    g_pool.push_back(r.a);
    g_pool.push_back(r.b);
  }
  g_recs.clear();
  std::string out;
  char line[192];
  for (auto& kv : agg) {
    std::vector<float>& v = kv.second;
    double total = 0.0;
    for (float ms : v) total += ms;
    std::sort(v.begin(), v.end());
    const size_t n = v.size();
    const double median = n % 2 ? v[n / 2] : 0.5 * ((double)v[n / 2 - 1] + v[n / 2]);
    snprintf(line, sizeof(line), "%s %d %.6f %.6f\n", kv.first.c_str(), (int)n, total, median);
    out += line;
  }
  if (out.size() + 1 > buf_len) return fail(MOE_ERR_INVALID_ARG, "report buffer too small");
  memcpy(buf, out.c_str(), out.size() + 1);
  return rc;
}

size_t moe_balance_loss_workspace_size(int T, int E, int k) {
  (void)k;
  if (T < 0 || E <= 0) return 0;
  return balance_ws_bytes(T, E);
}

int moe_balance_loss(const int32_t* idx, const float* gate, int T, int E, int k, float lambda,
                     float* stats, float* importance, float* dgate, void* ws, size_t ws_bytes,
                     void* stream) {
  if (int rc = check_common(T, E, k, MOE_F32)) return rc;
  if (T == 0) return fail(MOE_ERR_INVALID_ARG, "the balance loss needs T >= 1");
  REQUIRE_PTR(idx); REQUIRE_PTR(gate); REQUIRE_PTR(stats); REQUIRE_PTR(importance);
  if (ws_bytes < balance_ws_bytes(T, E))
    return fail(MOE_ERR_WORKSPACE, "balance workspace smaller than moe_balance_loss_workspace_size()");
  return launch_balance_loss(idx, gate, T, E, k, lambda, stats, importance, dgate, ws, ws_bytes,
                             (cudaStream_t)stream);
}

int moe_check_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  int flag = 0;
  e = cudaMemcpyFromSymbol(&flag, g_moe_status, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "read status flag");
  if (flag != 0) {
    int zero = 0;
    e = cudaMemcpyToSymbol(g_moe_status, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "clear status flag");
    char buf[96];
    if (flag & 0x200) {
      snprintf(buf, sizeof(buf), "a bounded device wait expired (code 0x%x)", flag);
      return fail(MOE_ERR_DEVICE_TIMEOUT, buf);
    }
    snprintf(buf, sizeof(buf), "device-side data check failed (code 0x%x)", flag);
    return fail(MOE_ERR_DEVICE_CHECK, buf);
  }
  return MOE_OK;
}

int moe_debug_expire_next_wait(long long wait_ns) {
  g_debug_expire.store(wait_ns > 0 ? wait_ns : 0);
  return MOE_OK;
}

}  // extern "C"
