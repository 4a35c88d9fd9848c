// CUDA-core (SIMT) grouped GEMMs: the fp32 path of the layer, and the small
// router GEMMs (logits = x W_gate, dW_gate = x^T dlogits, dlogits W_gate^T).
//
// Each kernel computes one 64x64 output tile per 256-thread block with a
// 16-deep k loop through shared memory; each thread owns a 4x4 sub-tile.
// Operands are read through small accessor functors, which also perform the
// row gathers (x[row_token[r]]) and the expert selection of a row tile.
#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int SB = 64;   // tile edge
constexpr int SK = 16;   // k step

template <class LA, class LB>
__device__ __forceinline__ void simt_tile(const LA& la, const LB& lb, int K, float (&acc)[4][4]) {
  __shared__ float As[SK][SB + 4];
  __shared__ float Bs[SK][SB + 4];
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int k0 = 0; k0 < K; k0 += SK) {
    for (int i = tid; i < SB * SK; i += 256) {
      const int m = i / SK, kk = i % SK;
      As[kk][m] = (k0 + kk < K) ? la(m, k0 + kk) : 0.f;
    }
    for (int i = tid; i < SB * SK; i += 256) {
      const int kk = i / SB, n = i % SB;
      Bs[kk][n] = (k0 + kk < K) ? lb(k0 + kk, n) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
}

#define SIMT_EPILOGUE(BODY)                                   \
  {                                                           \
    const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;   \
    _Pragma("unroll") for (int i = 0; i < 4; ++i)             \
      _Pragma("unroll") for (int j = 0; j < 4; ++j) {         \
        const int m = ty * 4 + i, n = tx * 4 + j;             \
        const float v = acc[i][j];                            \
        BODY                                                  \
      }                                                       \
  }

// ------------------------------------------------------------ router logits
template <class T>
__global__ void k_router_logits(const T* __restrict__ x, const T* __restrict__ wg, int T_, int d,
                                int E, float* __restrict__ logits) {
  const int m0 = blockIdx.x * SB, n0 = blockIdx.y * SB;
  auto la = [&](int m, int k) { return m0 + m < T_ ? to_f(x[(size_t)(m0 + m) * d + k]) : 0.f; };
  auto lb = [&](int k, int n) { return n0 + n < E ? to_f(wg[(size_t)k * E + n0 + n]) : 0.f; };
  float acc[4][4];
  simt_tile(la, lb, d, acc);
  SIMT_EPILOGUE(if (m0 + m < T_ && n0 + n < E) logits[(size_t)(m0 + m) * E + n0 + n] = v;)
}

int launch_router_logits_simt(const void* x, const void* wg, int T, int d, int E, int dtype,
                              const float* bias, float* logits, cudaStream_t s) {
  (void)bias;
  if (T == 0) return MOE_OK;
  dim3 grid((T + SB - 1) / SB, (E + SB - 1) / SB);
  if (dtype == MOE_BF16) {
    ProfScope _ps("router_logits", s);
    k_router_logits<__nv_bfloat16><<<grid, 256, 0, s>>>((const __nv_bfloat16*)x,
                                                        (const __nv_bfloat16*)wg, T, d, E, logits);
  } else {
    ProfScope _ps("router_logits", s);
    k_router_logits<float><<<grid, 256, 0, s>>>((const float*)x, (const float*)wg, T, d, E, logits);
  }
  MOE_CHECK_LAUNCH("router_logits");
  return MOE_OK;
}

// ------------------------------------------------------------ varlen-M tiles
// Row tile m0 of the padded row space belongs to one expert (segments start
// at multiples of 128).  Returns -1 when the tile lies beyond R.
__device__ __forceinline__ int tile_expert(const int32_t* offsets, int E, int m0) {
  if (m0 >= offsets[E]) return -1;
  return row_expert(offsets, E, m0);
}

// H[r, :] = [x W1_e | x W3_e](row_token[r]); padding rows give 0.
template <class T>
__global__ void k_simt_up(FfnPtrs p, T* __restrict__ H) {
  const int m0 = blockIdx.x * SB, n0 = blockIdx.y * SB;
  const int e = tile_expert(p.offsets, p.E, m0);
  if (e < 0) return;
  const int d = p.d, f = p.f;
  const T* x = (const T*)p.x;
  const T* w1 = (const T*)p.w1 + (size_t)e * d * f;
  const T* w3 = (const T*)p.w3 + (size_t)e * d * f;
  auto la = [&](int m, int k) {
    const int t = p.row_token[m0 + m];
    return t >= 0 ? to_f(x[(size_t)t * d + k]) : 0.f;
  };
  auto lb = [&](int k, int n) {
    const int c = n0 + n;
    return c < f ? to_f(w1[(size_t)k * f + c]) : to_f(w3[(size_t)k * f + c - f]);
  };
  float acc[4][4];
  simt_tile(la, lb, d, acc);
  SIMT_EPILOGUE(H[(size_t)(m0 + m) * 2 * f + n0 + n] = from_f<T>(v);)
}

// A[r, j] = silu(H1) * H3 (rounded to the storage type).
template <class T>
__global__ void k_simt_swiglu(const T* __restrict__ H, const int32_t* __restrict__ offsets, int E,
                              int f, T* __restrict__ act) {
  const int R = offsets[E];
  const size_t total = (size_t)R * f;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    const size_t r = i / f, j = i % f;
    const float h1 = to_f(H[r * 2 * f + j]), h3 = to_f(H[r * 2 * f + f + j]);
    act[i] = from_f<T>(silu_f(h1) * h3);
  }
}

// Y[r, :] = A[r, :] W2_e
template <class T>
__global__ void k_simt_down(FfnPtrs p, const T* __restrict__ act, T* __restrict__ Y) {
  const int m0 = blockIdx.x * SB, n0 = blockIdx.y * SB;
  const int e = tile_expert(p.offsets, p.E, m0);
  if (e < 0) return;
  const int d = p.d, f = p.f;
  const T* w2 = (const T*)p.w2 + (size_t)e * f * d;
  auto la = [&](int m, int k) { return to_f(act[(size_t)(m0 + m) * f + k]); };
  auto lb = [&](int k, int n) { return to_f(w2[(size_t)k * d + n0 + n]); };
  float acc[4][4];
  simt_tile(la, lb, f, acc);
  SIMT_EPILOGUE(Y[(size_t)(m0 + m) * d + n0 + n] = from_f<T>(v);)
}

// dA'[r, :] = dO[row_token[r], :] W2_e^T  (fp32)
template <class T>
__global__ void k_simt_dap(FfnPtrs p, const T* __restrict__ dout, float* __restrict__ dap) {
  const int m0 = blockIdx.x * SB, n0 = blockIdx.y * SB;
  const int e = tile_expert(p.offsets, p.E, m0);
  if (e < 0) return;
  const int d = p.d, f = p.f;
  const T* w2 = (const T*)p.w2 + (size_t)e * f * d;
  auto la = [&](int m, int k) {
    const int t = p.row_token[m0 + m];
    return t >= 0 ? to_f(dout[(size_t)t * d + k]) : 0.f;
  };
  auto lb = [&](int k, int n) { return to_f(w2[(size_t)(n0 + n) * d + k]); };
  float acc[4][4];
  simt_tile(la, lb, d, acc);
  SIMT_EPILOGUE(dap[(size_t)(m0 + m) * f + n0 + n] = v;)
}

// Per row (one warp): A = silu(H1)*H3 recomputed; dS = <dA', A>; dA = s dA';
// dH = [dA H3 silu'(H1) | dA silu(H1)]; gA = s A.
template <class T>
__global__ void k_simt_dap_epi(const float* __restrict__ dap, const T* __restrict__ H,
                               const float* __restrict__ row_gate, const int32_t* __restrict__ offsets,
                               int E, int f, T* __restrict__ dH, T* __restrict__ gact,
                               float* __restrict__ ds) {
  const int R = offsets[E];
  const int lane = threadIdx.x & 31, warps = blockDim.x >> 5;
  for (int r = blockIdx.x * warps + (threadIdx.x >> 5); r < R; r += gridDim.x * warps) {
    const float g = row_gate[r];
    float acc = 0.f;
    for (int j = lane; j < f; j += 32) {
      const float h1 = to_f(H[(size_t)r * 2 * f + j]), h3 = to_f(H[(size_t)r * 2 * f + f + j]);
      const float sl = silu_f(h1);
      const float a = to_f(from_f<T>(sl * h3));
      const float dp = dap[(size_t)r * f + j];
      acc = fmaf(dp, a, acc);
      const float da = g * dp;
      dH[(size_t)r * 2 * f + j] = from_f<T>(da * h3 * silu_grad_f(h1));
      dH[(size_t)r * 2 * f + f + j] = from_f<T>(da * sl);
      gact[(size_t)r * f + j] = from_f<T>(g * a);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) ds[r] = acc;
  }
}

// dX_perm[r, :] = dH[r, :] [W1_e | W3_e]^T
template <class T>
__global__ void k_simt_dx(FfnPtrs p, const T* __restrict__ dH, T* __restrict__ dxp) {
  const int m0 = blockIdx.x * SB, n0 = blockIdx.y * SB;
  const int e = tile_expert(p.offsets, p.E, m0);
  if (e < 0) return;
  const int d = p.d, f = p.f;
  const T* w1 = (const T*)p.w1 + (size_t)e * d * f;
  const T* w3 = (const T*)p.w3 + (size_t)e * d * f;
  auto la = [&](int m, int k) { return to_f(dH[(size_t)(m0 + m) * 2 * f + k]); };
  auto lb = [&](int k, int n) {
    return k < f ? to_f(w1[(size_t)(n0 + n) * f + k]) : to_f(w3[(size_t)(n0 + n) * f + k - f]);
  };
  float acc[4][4];
  simt_tile(la, lb, 2 * f, acc);
  SIMT_EPILOGUE(dxp[(size_t)(m0 + m) * d + n0 + n] = from_f<T>(v);)
}

// dW2_e[m, n] = sum over rows of e of gA[row, m] dO[row_token[row], n]
template <class T>
__global__ void k_simt_dw2(FfnPtrs p, const T* __restrict__ dout, const T* __restrict__ gact,
                           T* __restrict__ dw2) {
  const int m0 = blockIdx.x * SB, n0 = blockIdx.y * SB, e = blockIdx.z;
  const int d = p.d, f = p.f;
  const int r0 = p.offsets[e], nr = p.offsets[e + 1] - r0;
  auto la = [&](int m, int k) { return to_f(gact[(size_t)(r0 + k) * f + m0 + m]); };
  auto lb = [&](int k, int n) {
    const int t = p.row_token[r0 + k];
    return t >= 0 ? to_f(dout[(size_t)t * d + n0 + n]) : 0.f;
  };
  float acc[4][4];
  simt_tile(la, lb, nr, acc);
  SIMT_EPILOGUE(dw2[(size_t)e * f * d + (size_t)(m0 + m) * d + n0 + n] = from_f<T>(v);)
}

// [dW1_e | dW3_e][m, n] = sum over rows of e of x[row_token[row], m] dH[row, n]
template <class T>
__global__ void k_simt_dw13(FfnPtrs p, const T* __restrict__ dH, T* __restrict__ dw1,
                            T* __restrict__ dw3) {
  const int m0 = blockIdx.x * SB, n0 = blockIdx.y * SB, e = blockIdx.z;
  const int d = p.d, f = p.f;
  const T* x = (const T*)p.x;
  const int r0 = p.offsets[e], nr = p.offsets[e + 1] - r0;
  auto la = [&](int m, int k) {
    const int t = p.row_token[r0 + k];
    return t >= 0 ? to_f(x[(size_t)t * d + m0 + m]) : 0.f;
  };
  auto lb = [&](int k, int n) { return to_f(dH[(size_t)(r0 + k) * 2 * f + n0 + n]); };
  float acc[4][4];
  simt_tile(la, lb, nr, acc);
  SIMT_EPILOGUE({
    const int c = n0 + n;
    if (c < f) dw1[(size_t)e * d * f + (size_t)(m0 + m) * f + c] = from_f<T>(v);
    else dw3[(size_t)e * d * f + (size_t)(m0 + m) * f + c - f] = from_f<T>(v);
  })
}

// dW_gate[m, n] = sum_t x[t, m] dlogits[t, n]
template <class T>
__global__ void k_simt_dwg(const T* __restrict__ x, const float* __restrict__ dl, int T_, int d,
                           int E, float* __restrict__ dwg) {
  const int m0 = blockIdx.x * SB, n0 = blockIdx.y * SB;
  auto la = [&](int m, int k) { return to_f(x[(size_t)k * d + m0 + m]); };
  auto lb = [&](int k, int n) { return n0 + n < E ? dl[(size_t)k * E + n0 + n] : 0.f; };
  float acc[4][4];
  simt_tile(la, lb, T_, acc);
  SIMT_EPILOGUE(if (n0 + n < E) dwg[(size_t)(m0 + m) * E + n0 + n] = v;)
}

// dx[t, c] = dx_acc[t, c] + sum_e dlogits[t, e] W_gate[c, e]
template <class T>
__global__ void k_simt_dx_router(const float* __restrict__ dl, const T* __restrict__ wg,
                                 const float* __restrict__ dx_acc, int T_, int d, int E,
                                 T* __restrict__ dx) {
  const int m0 = blockIdx.x * SB, n0 = blockIdx.y * SB;
  auto la = [&](int m, int k) { return m0 + m < T_ ? dl[(size_t)(m0 + m) * E + k] : 0.f; };
  auto lb = [&](int k, int n) { return to_f(wg[(size_t)(n0 + n) * E + k]); };
  float acc[4][4];
  simt_tile(la, lb, E, acc);
  SIMT_EPILOGUE(if (m0 + m < T_) {
    const size_t o = (size_t)(m0 + m) * d + n0 + n;
    dx[o] = from_f<T>(v + dx_acc[o]);
  })
}

// ------------------------------------------------------------ launchers
static dim3 rows_grid(int cap, int ncols) { return dim3((cap + SB - 1) / SB, ncols / SB); }

template <class T>
static int ffn_fwd_t(const FfnPtrs& p, T* H, T* act, T* Y, cudaStream_t s) {
  {
    ProfScope _ps("simt_up", s);
    k_simt_up<T><<<rows_grid(p.cap, 2 * p.f), 256, 0, s>>>(p, H);
  }
  MOE_CHECK_LAUNCH("simt_up");
  {
    ProfScope _ps("simt_swiglu", s);
    k_simt_swiglu<T><<<device_sm_count() * 8, 256, 0, s>>>(H, p.offsets, p.E, p.f, act);
  }
  MOE_CHECK_LAUNCH("simt_swiglu");
  {
    ProfScope _ps("simt_down", s);
    k_simt_down<T><<<rows_grid(p.cap, p.d), 256, 0, s>>>(p, act, Y);
  }
  MOE_CHECK_LAUNCH("simt_down");
  return MOE_OK;
}

int simt_ffn_fwd(const FfnPtrs& p, void* H, void* act, void* Y, cudaStream_t s) {
  if (p.dtype == MOE_BF16)
    return ffn_fwd_t<__nv_bfloat16>(p, (__nv_bfloat16*)H, (__nv_bfloat16*)act, (__nv_bfloat16*)Y, s);
  return ffn_fwd_t<float>(p, (float*)H, (float*)act, (float*)Y, s);
}

template <class T>
static int ffn_bwd_t(const FfnPtrs& p, const T* dout, const float* row_gate, const T* H,
                     float* dap, T* dH, T* gact, float* ds, T* dxp, T* dw1, T* dw3, T* dw2,
                     cudaStream_t s) {
  {
    ProfScope _ps("simt_dap", s);
    k_simt_dap<T><<<rows_grid(p.cap, p.f), 256, 0, s>>>(p, dout, dap);
  }
  MOE_CHECK_LAUNCH("simt_dap");
  {
    ProfScope _ps("simt_dap_epi", s);
    k_simt_dap_epi<T><<<device_sm_count() * 8, 256, 0, s>>>(dap, H, row_gate, p.offsets, p.E, p.f,
                                                            dH, gact, ds);
  }
  MOE_CHECK_LAUNCH("simt_dap_epi");
  {
    ProfScope _ps("simt_dx", s);
    k_simt_dx<T><<<rows_grid(p.cap, p.d), 256, 0, s>>>(p, dH, dxp);
  }
  MOE_CHECK_LAUNCH("simt_dx");
  {
    ProfScope _ps("simt_dw2", s);
    k_simt_dw2<T><<<dim3(p.f / SB, p.d / SB, p.E), 256, 0, s>>>(p, dout, gact, dw2);
  }
  MOE_CHECK_LAUNCH("simt_dw2");
  {
    ProfScope _ps("simt_dw13", s);
    k_simt_dw13<T><<<dim3(p.d / SB, 2 * p.f / SB, p.E), 256, 0, s>>>(p, dH, dw1, dw3);
  }
  MOE_CHECK_LAUNCH("simt_dw13");
  return MOE_OK;
}

int simt_ffn_bwd(const FfnPtrs& p, const void* dout, const float* row_gate, const void* H,
                 float* dap, void* dH, void* gact, float* ds, void* dXp, void* dw1, void* dw3,
                 void* dw2, cudaStream_t s) {
  if (p.dtype == MOE_BF16)
    return ffn_bwd_t<__nv_bfloat16>(p, (const __nv_bfloat16*)dout, row_gate,
                                    (const __nv_bfloat16*)H, dap, (__nv_bfloat16*)dH,
                                    (__nv_bfloat16*)gact, ds, (__nv_bfloat16*)dXp,
                                    (__nv_bfloat16*)dw1, (__nv_bfloat16*)dw3, (__nv_bfloat16*)dw2, s);
  return ffn_bwd_t<float>(p, (const float*)dout, row_gate, (const float*)H, dap, (float*)dH,
                          (float*)gact, ds, (float*)dXp, (float*)dw1, (float*)dw3, (float*)dw2, s);
}

template <class T>
static int router_bwd_t(const T* x, const T* wg, const float* dl, const float* dx_acc, int T_,
                        int d, int E, float* dwg, T* dx, cudaStream_t s) {
  {
    ProfScope _ps("simt_dwg", s);
    k_simt_dwg<T><<<dim3(d / SB, (E + SB - 1) / SB), 256, 0, s>>>(x, dl, T_, d, E, dwg);
  }
  MOE_CHECK_LAUNCH("simt_dwg");
  if (T_ > 0) {
    {
      ProfScope _ps("simt_dx_router", s);
      k_simt_dx_router<T><<<dim3((T_ + SB - 1) / SB, d / SB), 256, 0, s>>>(dl, wg, dx_acc, T_, d, E, dx);
    }
    MOE_CHECK_LAUNCH("simt_dx_router");
  }
  return MOE_OK;
}

int simt_router_bwd_gemms(const void* x, const void* wg, const float* dl, const float* dx_acc,
                          int T, int d, int E, int dtype, float* dw_gate, void* dx, cudaStream_t s) {
  if (dtype == MOE_BF16)
    return router_bwd_t<__nv_bfloat16>((const __nv_bfloat16*)x, (const __nv_bfloat16*)wg, dl,
                                       dx_acc, T, d, E, dw_gate, (__nv_bfloat16*)dx, s);
  return router_bwd_t<float>((const float*)x, (const float*)wg, dl, dx_acc, T, d, E, dw_gate,
                             (float*)dx, s);
}

}  // namespace moe
