// Row gather, per-token reductions (combine / dx unpermute-sum) and the
// router backward.  HBM-bound SIMT kernels with 16-byte vector accesses.
//
// Combine: O_t = sum_j g_tj Y(row of slot (t,j)) -- Beam article sec. 2.2,
// Trinity Large commentary example 3.  Router backward from the per-row
// router-score gradients dS = <dA', A> -- SonicMoE summary sec. 1.
#include "common.cuh"
#include "internal.h"

namespace moe {

// 16-byte vector of 8 bf16 or 4 fp32.
template <class T> struct Vec;
template <> struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  uint4 v;
  __device__ __forceinline__ float get(int i) const {
    const __nv_bfloat16* p = reinterpret_cast<const __nv_bfloat16*>(&v);
    return __bfloat162float(p[i]);
  }
  __device__ __forceinline__ void set(int i, float f) {
    __nv_bfloat16* p = reinterpret_cast<__nv_bfloat16*>(&v);
    p[i] = __float2bfloat16_rn(f);
  }
};
template <> struct Vec<float> {
  static constexpr int N = 4;
  uint4 v;
  __device__ __forceinline__ float get(int i) const { return reinterpret_cast<const float*>(&v)[i]; }
  __device__ __forceinline__ void set(int i, float f) { reinterpret_cast<float*>(&v)[i] = f; }
};

// ============================================================== scatter rows
// dst[row, :] = src[t, :] for every row of token t (its kept slots, then the
// rows added by token rounding); rows that hold no pair (padding, token -1)
// are zeroed.  The last nbt blocks own tokens, one warp per token, so each
// source row is read once and written to its k rows with coalesced 16-byte
// stores; the first blocks of the grid zero the padding rows (first, so that
// this runs beside the token blocks instead of after them).
template <class T>
__global__ void __launch_bounds__(256)
k_scatter_rows(const T* __restrict__ src, const int32_t* __restrict__ slot_row,
               const int32_t* __restrict__ extra_row, const int32_t* __restrict__ row_token,
               const int32_t* __restrict__ offsets, int T_, int width, int E, int k, int nbt,
               T* __restrict__ dst) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int nvec = width / Vec<T>::N;
  const int nzb = gridDim.x - nbt;        // the first nzb blocks zero the padding rows
  if ((int)blockIdx.x >= nzb) {
    const int t = (blockIdx.x - nzb) * 8 + w;
    if (t >= T_) return;
    const int mine = lane < k ? slot_row[(size_t)t * k + lane] : -1;
    int rk[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) rk[j] = __shfl_sync(0xffffffffu, mine, j);
    const uint4* s4 = reinterpret_cast<const uint4*>(src + (size_t)t * width);
    for (int i = lane; i < nvec; i += 32) {
      const uint4 v = __ldg(s4 + i);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (rk[j] >= 0) reinterpret_cast<uint4*>(dst + (size_t)rk[j] * width)[i] = v;
    }
    if (extra_row != nullptr) {
      for (int e0 = 0; e0 < E; e0 += 32) {
        const int re = e0 + lane < E ? extra_row[(size_t)t * E + e0 + lane] : -1;
        unsigned bal = __ballot_sync(0xffffffffu, re >= 0);
        while (bal) {
          const int b = __ffs(bal) - 1;
          bal &= bal - 1;
          const int r = __shfl_sync(0xffffffffu, re, b);
          uint4* d4 = reinterpret_cast<uint4*>(dst + (size_t)r * width);
          for (int i = lane; i < nvec; i += 32) d4[i] = __ldg(s4 + i);
        }
      }
    }
  } else {
    // a warp tests 32 rows at once and zeroes the padding rows among them
    const int R = offsets[E];
    for (int r0 = (blockIdx.x * 8 + w) * 32; r0 < R; r0 += nzb * 8 * 32) {
      const int r = r0 + lane;
      unsigned bal = __ballot_sync(0xffffffffu, r < R && row_token[r] < 0);
      while (bal) {
        const int b = __ffs(bal) - 1;
        bal &= bal - 1;
        uint4* d4 = reinterpret_cast<uint4*>(dst + (size_t)(r0 + b) * width);
        for (int i = lane; i < nvec; i += 32) d4[i] = make_uint4(0, 0, 0, 0);
      }
    }
  }
}

// 32-byte global accesses (sm_100 256-bit loads and stores).
__device__ __forceinline__ void ld_nc_v8(const void* p, uint4& a, uint4& b) {
  asm volatile("ld.global.nc.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
               : "l"(p));
}
__device__ __forceinline__ void st_v8(void* p, const uint4& a, const uint4& b) {
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(a.x), "r"(a.y),
               "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
               : "memory");
}

// The same scatter for rows of a multiple of 32 bytes (32-byte aligned): a
// warp loads a whole 32 * SR_UNITS-unit slice of its token's row (SR_UNITS
// 32-byte loads per lane in flight) and then writes that slice to each of
// the token's rows in turn, so each destination row is written as one
// contiguous burst.  Rows of up to 32 * SR_UNITS * 32 bytes take one pass.
// The padding rows are zeroed by the first blocks of the grid, so that this
// work runs beside the token blocks instead of after them.
constexpr int SR_UNITS = 4;

__global__ void __launch_bounds__(256)
k_scatter_rows_wide(const uint8_t* __restrict__ src, const int32_t* __restrict__ slot_row,
                    const int32_t* __restrict__ extra_row, const int32_t* __restrict__ row_token,
                    const int32_t* __restrict__ offsets, int T_, int nunit, int E, int k, int nbt,
                    uint8_t* __restrict__ dst) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const size_t rb = (size_t)nunit * 32;   // bytes per row
  const int nzb = gridDim.x - nbt;        // the first nzb blocks zero the padding rows
  if ((int)blockIdx.x >= nzb) {
    const int t = (blockIdx.x - nzb) * 8 + w;
    if (t >= T_) return;
    const int mine = lane < k ? slot_row[(size_t)t * k + lane] : -1;
    int rk[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) rk[j] = __shfl_sync(0xffffffffu, mine, j);
    const uint8_t* s = src + (size_t)t * rb;
    for (int u0 = 0; u0 < nunit; u0 += 32 * SR_UNITS) {
      uint4 va[SR_UNITS], vb[SR_UNITS];
#pragma unroll
      for (int q = 0; q < SR_UNITS; ++q) {
        const int u = u0 + q * 32 + lane;
        if (u < nunit) ld_nc_v8(s + (size_t)u * 32, va[q], vb[q]);
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (rk[j] < 0) continue;
        uint8_t* d = dst + (size_t)rk[j] * rb;
#pragma unroll
        for (int q = 0; q < SR_UNITS; ++q) {
          const int u = u0 + q * 32 + lane;
          if (u < nunit) st_v8(d + (size_t)u * 32, va[q], vb[q]);
        }
      }
      if (extra_row != nullptr) {
        for (int e0 = 0; e0 < E; e0 += 32) {
          const int re = e0 + lane < E ? extra_row[(size_t)t * E + e0 + lane] : -1;
          unsigned bal = __ballot_sync(0xffffffffu, re >= 0);
          while (bal) {
            const int b = __ffs(bal) - 1;
            bal &= bal - 1;
            uint8_t* d = dst + (size_t)__shfl_sync(0xffffffffu, re, b) * rb;
#pragma unroll
            for (int q = 0; q < SR_UNITS; ++q) {
              const int u = u0 + q * 32 + lane;
              if (u < nunit) st_v8(d + (size_t)u * 32, va[q], vb[q]);
            }
          }
        }
      }
    }
  } else {
    // a warp tests 32 rows at once and zeroes the padding rows among them
    const int R = offsets[E];
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int r0 = (blockIdx.x * 8 + w) * 32; r0 < R; r0 += nzb * 8 * 32) {
      const int r = r0 + lane;
      unsigned bal = __ballot_sync(0xffffffffu, r < R && row_token[r] < 0);
      while (bal) {
        const int b = __ffs(bal) - 1;
        bal &= bal - 1;
        uint8_t* d = dst + (size_t)(r0 + b) * rb;
        for (int u = lane; u < nunit; u += 32) st_v8(d + (size_t)u * 32, z, z);
      }
    }
  }
}

int launch_scatter_rows(const void* src, const int32_t* slot_row, const int32_t* extra_row,
                        const int32_t* row_token, const int32_t* offsets, int T, int width, int E,
                        int k, int dtype, void* dst, cudaStream_t s) {
  const int nbt = (T + 7) / 8;
  const int blocks = nbt + device_sm_count() * 2;
  const size_t row_bytes = (size_t)width * (dtype == MOE_BF16 ? 2 : 4);
  if (row_bytes % 32 == 0 && (uintptr_t)src % 32 == 0 && (uintptr_t)dst % 32 == 0) {
    ProfScope _ps("scatter_rows", s);
    k_scatter_rows_wide<<<blocks, 256, 0, s>>>((const uint8_t*)src, slot_row, extra_row, row_token,
                                               offsets, T, (int)(row_bytes / 32), E, k, nbt,
                                               (uint8_t*)dst);
  } else if (dtype == MOE_BF16) {
    ProfScope _ps("scatter_rows", s);
    k_scatter_rows<__nv_bfloat16><<<blocks, 256, 0, s>>>(
        (const __nv_bfloat16*)src, slot_row, extra_row, row_token, offsets, T, width, E, k, nbt,
        (__nv_bfloat16*)dst);
  } else {
    ProfScope _ps("scatter_rows", s);
    k_scatter_rows<float><<<blocks, 256, 0, s>>>((const float*)src, slot_row, extra_row, row_token,
                                                 offsets, T, width, E, k, nbt, (float*)dst);
  }
  MOE_CHECK_LAUNCH("scatter_rows");
  return MOE_OK;
}

// ============================================================== fused dx (small router)
// dx[t, :] = bf16( sum over t's rows of dX_perm[row, :] + sum_e dl[t, e] W_gate[:, e] )
// for routers whose W_gate fits in shared memory (E <= 32, d*E*2 <= 48 KB).
// One warp per token; a lane owns 8 consecutive columns per step and loads the
// next step's rows before summing the current ones.
// dx_t = sum over token t's rows of dX_perm + dl_t W_gate^T, for small
// routers (E <= 32): one warp per token; each lane owns 8 consecutive columns
// per vector and handles two vectors per pass, issuing the loads of all the
// token's rows for both before any arithmetic.  The row sum runs in fp32 in
// slot order, then the rows added by rounding in ascending expert id, then the
// router term in ascending expert id.
template <int MAXE, int MAXK> struct DxfTraits {
  // vectors per lane per pass (loads in flight) and resident blocks per SM,
  // chosen so that the registers fit without spilling
  static constexpr int V = MAXK <= 4 ? 2 : 1;
  static constexpr int MINB = (MAXE * MAXK <= 32 || (MAXE <= 16 && MAXK <= 2)) ? 4 : 2;
};

template <int MAXE, int MAXK>
__global__ void __launch_bounds__(256, (DxfTraits<MAXE, MAXK>::MINB))
k_dx_fused(const __nv_bfloat16* __restrict__ dxp, const int32_t* __restrict__ slot_row,
           const int32_t* __restrict__ extra_row, const float* __restrict__ dl,
           const __nv_bfloat16* __restrict__ wg, int T_, int d, int E, int k,
           __nv_bfloat16* __restrict__ dx) {
  extern __shared__ __align__(16) uint8_t smem_wg[];
  // W_gate transposed to [E][d] (bf16): a lane's 8 consecutive columns of one
  // expert are one conflict-free 16-byte shared load.  Staged once per block
  // (persistent grid).
  __nv_bfloat16* w_t = reinterpret_cast<__nv_bfloat16*>(smem_wg);
  __shared__ int s_extra[8][32];  // rows added by rounding, per warp (E <= 32)
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    for (int e0 = 0; e0 < E; e0 += 8) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(wg + (size_t)c * E + e0));
      const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&u);
#pragma unroll
      for (int q = 0; q < 8; ++q) w_t[(size_t)(e0 + q) * d + c] = h[q];
    }
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int nvec = d / 8;
  for (int t = blockIdx.x * 8 + w; t < T_; t += gridDim.x * 8) {
    // the token's added rows, in ascending expert id (whole warp)
    int n_extra = 0;
    if (extra_row != nullptr) {
      const int re = lane < E ? extra_row[(size_t)t * E + lane] : -1;
      const unsigned bal = __ballot_sync(0xffffffffu, re >= 0);
      if (re >= 0) s_extra[w][__popc(bal & ((1u << lane) - 1u))] = re;
      n_extra = __popc(bal);
      __syncwarp();
    }
    float dlr[MAXE];
#pragma unroll
    for (int e = 0; e < MAXE; ++e) dlr[e] = e < E ? dl[(size_t)t * E + e] : 0.f;
    const int mine = lane < k ? slot_row[(size_t)t * k + lane] : -1;
    int rk[MAXK];
#pragma unroll
    for (int j = 0; j < MAXK; ++j) rk[j] = __shfl_sync(0xffffffffu, mine, j);
    constexpr int V = DxfTraits<MAXE, MAXK>::V;
    for (int i0 = lane; i0 < nvec; i0 += 32 * V) {
      uint4 raw[V][MAXK];
#pragma unroll
      for (int v = 0; v < V; ++v) {
        const int i = i0 + 32 * v;
#pragma unroll
        for (int j = 0; j < MAXK; ++j)
          raw[v][j] = (i < nvec && rk[j] >= 0)
                          ? __ldg(reinterpret_cast<const uint4*>(dxp + (size_t)rk[j] * d) + i)
                          : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int v = 0; v < V; ++v) {
        const int i = i0 + 32 * v;
        if (i >= nvec) break;
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.f;
#pragma unroll
        for (int j = 0; j < MAXK; ++j) {
          if (rk[j] >= 0) {
            Vec<__nv_bfloat16> u;
            u.v = raw[v][j];
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[q] += u.get(q);
          }
        }
        for (int j = 0; j < n_extra; ++j) {
          Vec<__nv_bfloat16> u;
          u.v = __ldg(reinterpret_cast<const uint4*>(dxp + (size_t)s_extra[w][j] * d) + i);
#pragma unroll
          for (int q = 0; q < 8; ++q) acc[q] += u.get(q);
        }
        // router term: columns 8i..8i+7 of every expert column of W_gate
#pragma unroll
        for (int e = 0; e < MAXE; ++e) {
          if (e < E) {
            Vec<__nv_bfloat16> wv;
            wv.v = reinterpret_cast<const uint4*>(w_t + (size_t)e * d)[i];
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[q] = fmaf(dlr[e], wv.get(q), acc[q]);
          }
        }
        Vec<__nv_bfloat16> o;
#pragma unroll
        for (int q = 0; q < 8; ++q) o.set(q, acc[q]);
        reinterpret_cast<uint4*>(dx + (size_t)t * d)[i] = o.v;
      }
    }
    __syncwarp();
  }
}

bool dx_fused_ok(int d, int E) { return E <= 32 && E % 8 == 0 && (size_t)d * E * 2 <= 48 * 1024; }

template <int MAXE, int MAXK>
static void dx_fused_go(int blocks, size_t smem, cudaStream_t s, const void* dxp,
                        const int32_t* slot_row, const int32_t* extra_row, const float* dl,
                        const void* wg, int T, int d, int E, int k, void* dx) {
  k_dx_fused<MAXE, MAXK><<<blocks, 256, smem, s>>>((const __nv_bfloat16*)dxp, slot_row, extra_row,
                                                   dl, (const __nv_bfloat16*)wg, T, d, E, k,
                                                   (__nv_bfloat16*)dx);
}

template <int MAXE>
static int dx_fused_k(int blocks, size_t smem, cudaStream_t s, const void* dxp,
                      const int32_t* slot_row, const int32_t* extra_row, const float* dl,
                      const void* wg, int T, int d, int E, int k, void* dx) {
  if (smem > 48 * 1024) {
    cudaError_t e;
    if (k <= 2) e = cudaFuncSetAttribute(k_dx_fused<MAXE, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    else if (k <= 4) e = cudaFuncSetAttribute(k_dx_fused<MAXE, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    else e = cudaFuncSetAttribute(k_dx_fused<MAXE, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "dx_fused smem attribute");
  }
  if (k <= 2) dx_fused_go<MAXE, 2>(blocks, smem, s, dxp, slot_row, extra_row, dl, wg, T, d, E, k, dx);
  else if (k <= 4) dx_fused_go<MAXE, 4>(blocks, smem, s, dxp, slot_row, extra_row, dl, wg, T, d, E, k, dx);
  else dx_fused_go<MAXE, 8>(blocks, smem, s, dxp, slot_row, extra_row, dl, wg, T, d, E, k, dx);
  return MOE_OK;
}

int launch_dx_fused(const void* dxp, const int32_t* slot_row, const int32_t* extra_row,
                    const float* dl, const void* wg, int T, int d, int E, int k, void* dx,
                    cudaStream_t s) {
  if (T == 0) return MOE_OK;
  const size_t smem = (size_t)d * E * 2;
  int blocks = (T + 7) / 8;
  const int fit = (int)(220 * 1024 / (smem + 2048));
  const int per_sm = fit < 4 ? (fit > 0 ? fit : 1) : 4;
  if (blocks > device_sm_count() * per_sm) blocks = device_sm_count() * per_sm;
  int rc;
  {
    ProfScope _ps("dx_fused", s);
    if (E <= 8) rc = dx_fused_k<8>(blocks, smem, s, dxp, slot_row, extra_row, dl, wg, T, d, E, k, dx);
    else if (E <= 16) rc = dx_fused_k<16>(blocks, smem, s, dxp, slot_row, extra_row, dl, wg, T, d, E, k, dx);
    else rc = dx_fused_k<32>(blocks, smem, s, dxp, slot_row, extra_row, dl, wg, T, d, E, k, dx);
  }
  if (rc) return rc;
  MOE_CHECK_LAUNCH("dx_fused");
  return MOE_OK;
}

// out[t, :] = sum_rows (weighted ? row_gate[r] : 1) * src[r, :].
// One warp per token: the warp first lists the token's rows in shared memory
// (kept slots in slot order, then added rows by ascending expert), then each
// lane sums 16-byte vectors of up to 8 rows at a time, issuing the loads of
// all those rows before accumulating, in fixed row order.
constexpr int TR_WARPS = 8;

template <class T, class OutT>
__global__ void __launch_bounds__(TR_WARPS * 32)
k_token_reduce(const T* __restrict__ src, const float* __restrict__ row_gate,
               const int32_t* __restrict__ slot_row, const int32_t* __restrict__ extra_row,
               int T_, int width, int E, int k, bool weighted, OutT* __restrict__ out) {
  __shared__ int s_rows[TR_WARPS][8 + 256];
  __shared__ float s_wts[TR_WARPS][8 + 256];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int* rows = s_rows[w];
  float* wts = s_wts[w];
  const int nvec = width / Vec<T>::N;
  for (int t = blockIdx.x * TR_WARPS + w; t < T_; t += gridDim.x * TR_WARPS) {
    // kept slots: ordered compaction of slot_row[t, 0..k)
    const int rs = lane < k ? slot_row[(size_t)t * k + lane] : -1;
    unsigned bal = __ballot_sync(0xffffffffu, rs >= 0);
    int n = __popc(bal);
    if (rs >= 0) rows[__popc(bal & ((1u << lane) - 1u))] = rs;
    if (extra_row != nullptr) {
      for (int e0 = 0; e0 < E; e0 += 32) {
        const int re = (e0 + lane < E) ? extra_row[(size_t)t * E + e0 + lane] : -1;
        bal = __ballot_sync(0xffffffffu, re >= 0);
        if (re >= 0) rows[n + __popc(bal & ((1u << lane) - 1u))] = re;
        n += __popc(bal);
      }
    }
    __syncwarp();
    if (weighted)
      for (int j = lane; j < n; j += 32) wts[j] = row_gate[rows[j]];
    __syncwarp();
    for (int i = lane; i < nvec; i += 32) {
      float acc[Vec<T>::N];
#pragma unroll
      for (int q = 0; q < Vec<T>::N; ++q) acc[q] = 0.f;
      for (int j0 = 0; j0 < n; j0 += 8) {
        Vec<T> v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (j0 + j < n)
            v[j].v = __ldg(reinterpret_cast<const uint4*>(src + (size_t)rows[j0 + j] * width) + i);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (j0 + j < n) {
            const float wt = weighted ? wts[j0 + j] : 1.0f;
#pragma unroll
            for (int q = 0; q < Vec<T>::N; ++q) acc[q] = fmaf(wt, v[j].get(q), acc[q]);
          }
        }
      }
      OutT* o = out + (size_t)t * width + (size_t)i * Vec<T>::N;
      if constexpr (sizeof(OutT) == 2) {
        Vec<T> r;
#pragma unroll
        for (int q = 0; q < Vec<T>::N; ++q) r.set(q, acc[q]);
        *reinterpret_cast<uint4*>(o) = r.v;
      } else {
#pragma unroll
        for (int q = 0; q < Vec<T>::N; q += 4)
          *reinterpret_cast<float4*>(o + q) = make_float4(acc[q], acc[q + 1], acc[q + 2], acc[q + 3]);
      }
    }
    __syncwarp();
  }
}

// The same reduction for bf16 rows of a multiple of 16 elements (32-byte
// aligned) when a token has at most 4 kept slots: a lane owns 16 consecutive
// columns per pass and loads them from each row with one 32-byte load, so a
// 4 KB row takes half the passes (each a round trip to memory) of 16-byte
// loads.  Rows are summed in the same order as above (bit-identical).
template <class OutT>
__global__ void __launch_bounds__(TR_WARPS * 32)
k_token_reduce_w32(const __nv_bfloat16* __restrict__ src, const float* __restrict__ row_gate,
                   const int32_t* __restrict__ slot_row, const int32_t* __restrict__ extra_row,
                   int T_, int width, int E, int k, bool weighted, OutT* __restrict__ out) {
  constexpr int RB = 4;   // rows whose loads are in flight together
  __shared__ int s_rows[TR_WARPS][8 + 256];
  __shared__ float s_wts[TR_WARPS][8 + 256];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int* rows = s_rows[w];
  float* wts = s_wts[w];
  const int nu = width / 16;   // 32-byte units per row
  for (int t = blockIdx.x * TR_WARPS + w; t < T_; t += gridDim.x * TR_WARPS) {
    const int rs = lane < k ? slot_row[(size_t)t * k + lane] : -1;
    unsigned bal = __ballot_sync(0xffffffffu, rs >= 0);
    int n = __popc(bal);
    if (rs >= 0) rows[__popc(bal & ((1u << lane) - 1u))] = rs;
    if (extra_row != nullptr) {
      for (int e0 = 0; e0 < E; e0 += 32) {
        const int re = (e0 + lane < E) ? extra_row[(size_t)t * E + e0 + lane] : -1;
        bal = __ballot_sync(0xffffffffu, re >= 0);
        if (re >= 0) rows[n + __popc(bal & ((1u << lane) - 1u))] = re;
        n += __popc(bal);
      }
    }
    __syncwarp();
    if (weighted)
      for (int j = lane; j < n; j += 32) wts[j] = row_gate[rows[j]];
    __syncwarp();
    for (int u = lane; u < nu; u += 32) {
      float acc[16];
#pragma unroll
      for (int q = 0; q < 16; ++q) acc[q] = 0.f;
      for (int j0 = 0; j0 < n; j0 += RB) {
        Vec<__nv_bfloat16> va[RB], vb[RB];
#pragma unroll
        for (int j = 0; j < RB; ++j)
          if (j0 + j < n) ld_nc_v8(src + (size_t)rows[j0 + j] * width + 16 * u, va[j].v, vb[j].v);
#pragma unroll
        for (int j = 0; j < RB; ++j) {
          if (j0 + j < n) {
            const float wt = weighted ? wts[j0 + j] : 1.0f;
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[q] = fmaf(wt, va[j].get(q), acc[q]);
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[8 + q] = fmaf(wt, vb[j].get(q), acc[8 + q]);
          }
        }
      }
      OutT* o = out + (size_t)t * width + 16 * u;
      if constexpr (sizeof(OutT) == 2) {
        Vec<__nv_bfloat16> ra, rb;
#pragma unroll
        for (int q = 0; q < 8; ++q) { ra.set(q, acc[q]); rb.set(q, acc[8 + q]); }
        st_v8(o, ra.v, rb.v);
      } else {
#pragma unroll
        for (int q = 0; q < 16; q += 8)
          st_v8(o + q, make_uint4(__float_as_uint(acc[q]), __float_as_uint(acc[q + 1]),
                                  __float_as_uint(acc[q + 2]), __float_as_uint(acc[q + 3])),
                make_uint4(__float_as_uint(acc[q + 4]), __float_as_uint(acc[q + 5]),
                           __float_as_uint(acc[q + 6]), __float_as_uint(acc[q + 7])));
      }
    }
    __syncwarp();
  }
}

int launch_token_reduce(const void* src, const float* row_gate, const int32_t* slot_row,
                        const int32_t* extra_row, int T, int width, int E, int k, int dtype,
                        bool weighted, bool out_f32, void* out, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  int blocks = (T + TR_WARPS - 1) / TR_WARPS;
  if (blocks > device_sm_count() * 32) blocks = device_sm_count() * 32;
  if (dtype == MOE_BF16 && k <= 4 && width % 16 == 0 && (uintptr_t)src % 32 == 0 &&
      (uintptr_t)out % 32 == 0) {
    ProfScope _ps("token_reduce", s);
    if (out_f32)
      k_token_reduce_w32<float><<<blocks, TR_WARPS * 32, 0, s>>>(
          (const __nv_bfloat16*)src, row_gate, slot_row, extra_row, T, width, E, k, weighted,
          (float*)out);
    else
      k_token_reduce_w32<__nv_bfloat16><<<blocks, TR_WARPS * 32, 0, s>>>(
          (const __nv_bfloat16*)src, row_gate, slot_row, extra_row, T, width, E, k, weighted,
          (__nv_bfloat16*)out);
  } else if (dtype == MOE_BF16) {
    if (out_f32) {
      ProfScope _ps("token_reduce", s);
      k_token_reduce<__nv_bfloat16, float><<<blocks, TR_WARPS * 32, 0, s>>>(
          (const __nv_bfloat16*)src, row_gate, slot_row, extra_row, T, width, E, k, weighted,
          (float*)out);
    } else {
      ProfScope _ps("token_reduce", s);
      k_token_reduce<__nv_bfloat16, __nv_bfloat16><<<blocks, TR_WARPS * 32, 0, s>>>(
          (const __nv_bfloat16*)src, row_gate, slot_row, extra_row, T, width, E, k, weighted,
          (__nv_bfloat16*)out);
    }
  } else {
    {
      ProfScope _ps("token_reduce", s);
      k_token_reduce<float, float><<<blocks, TR_WARPS * 32, 0, s>>>((const float*)src, row_gate, slot_row,
                                                          extra_row, T, width, E, k, weighted,
                                                          (float*)out);
    }
  }
  MOE_CHECK_LAUNCH("token_reduce");
  return MOE_OK;
}

// ============================================================== load-balance loss
// importance_e = (1/T) sum_t G_te, G_t = token t's top-k gates (zero elsewhere);
// L = lambda * CV(importance)^2 with the population CV over the E experts
// ("Breaking the hundred-billion-parameter barrier" article, challenge 1);
// token counts per expert give the routing statistics (Trinity commentary
// example 2, Beam article sec. 5.4).  All sums run in a fixed order.
constexpr int BAL_TOK = 256;

__global__ void __launch_bounds__(256)
k_balance_partial(const int32_t* __restrict__ idx, const float* __restrict__ gate, int T, int E,
                  int k, float* __restrict__ psum, int32_t* __restrict__ pcnt) {
  __shared__ int s_key[BAL_TOK * 8];
  __shared__ float s_val[BAL_TOK * 8];
  const int t0 = blockIdx.x * BAL_TOK;
  const int n = min(BAL_TOK, T - t0) * k;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    s_key[i] = idx[(size_t)t0 * k + i];
    s_val[i] = gate[(size_t)t0 * k + i];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    float acc = 0.f;
    int c = 0;
    for (int i = 0; i < n; ++i) {
      if (s_key[i] == e) { acc += s_val[i]; ++c; }
    }
    psum[(size_t)blockIdx.x * E + e] = acc;
    pcnt[(size_t)blockIdx.x * E + e] = c;
  }
}

// One block: reduce the partials, then loss, statistics and dL/dimportance.
__global__ void __launch_bounds__(256)
k_balance_final(const float* __restrict__ psum, const int32_t* __restrict__ pcnt, int nb, int T,
                int E, float lam, float* __restrict__ stats, float* __restrict__ importance,
                float* __restrict__ dimp) {
  __shared__ float s_imp[256];
  __shared__ float s_cnt[256];
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    float acc = 0.f;
    int c = 0;
    for (int b = 0; b < nb; ++b) {
      acc += psum[(size_t)b * E + e];
      c += pcnt[(size_t)b * E + e];
    }
    s_imp[e] = acc / (float)T;
    s_cnt[e] = (float)c;
    importance[e] = acc / (float)T;
  }
  __syncthreads();
  __shared__ float s_m, s_var, s_cm, s_cvar, s_cmax, s_ctot;
  if (threadIdx.x == 0) {
    double m = 0, cm = 0, cmax = 0, ctot = 0;
    for (int e = 0; e < E; ++e) {
      m += s_imp[e];
      cm += s_cnt[e];
      cmax = fmax(cmax, (double)s_cnt[e]);
    }
    ctot = cm;
    m /= E;
    cm /= E;
    double var = 0, cvar = 0;
    for (int e = 0; e < E; ++e) {
      var += (s_imp[e] - m) * (s_imp[e] - m);
      cvar += (s_cnt[e] - cm) * (s_cnt[e] - cm);
    }
    var /= E;
    cvar /= E;
    s_m = (float)m;
    s_var = (float)var;
    stats[0] = (float)(lam * var / (m * m));
    stats[1] = ctot > 0 ? (float)(cmax / ctot) : 0.f;
    stats[2] = cm > 0 ? (float)(cvar / (cm * cm)) : 0.f;
    stats[3] = (float)cvar;
  }
  __syncthreads();
  // d(var/m^2)/d imp_e = (2/E)(imp_e - m)/m^2 - 2 var/(E m^3)
  const float m = s_m, var = s_var;
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    dimp[e] = lam * (2.0f / E * (s_imp[e] - m) / (m * m) - 2.0f * var / (E * m * m * m));
}

__global__ void k_balance_dgate(const int32_t* __restrict__ idx, const float* __restrict__ dimp,
                                int n, float inv_T, float* __restrict__ dgate) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
    dgate[i] = dimp[idx[i]] * inv_T;
}

size_t balance_ws_bytes(int T, int E) {
  Sizer z;
  const int nb = (T + BAL_TOK - 1) / BAL_TOK;
  z.take<float>((size_t)nb * E);
  z.take<int32_t>((size_t)nb * E);
  z.take<float>(E);
  return z.used;
}

int launch_balance_loss(const int32_t* idx, const float* gate, int T, int E, int k, float lam,
                        float* stats, float* importance, float* dgate, void* ws, size_t ws_bytes,
                        cudaStream_t s) {
  Carve c(ws, ws_bytes);
  const int nb = (T + BAL_TOK - 1) / BAL_TOK;
  float* psum = c.take<float>((size_t)nb * E);
  int32_t* pcnt = c.take<int32_t>((size_t)nb * E);
  float* dimp = c.take<float>(E);
  if (!c.ok) return fail(MOE_ERR_WORKSPACE, "balance-loss workspace too small");
  {
    ProfScope _ps("balance_partial", s);
    k_balance_partial<<<nb, 256, 0, s>>>(idx, gate, T, E, k, psum, pcnt);
  }
  MOE_CHECK_LAUNCH("balance_partial");
  {
    ProfScope _ps("balance_final", s);
    k_balance_final<<<1, 256, 0, s>>>(psum, pcnt, nb, T, E, lam, stats, importance, dimp);
  }
  MOE_CHECK_LAUNCH("balance_final");
  if (dgate != nullptr) {
    const int n = T * k;
    int blocks = (n + 255) / 256;
    if (blocks > device_sm_count() * 4) blocks = device_sm_count() * 4;
    {
      ProfScope _ps("balance_dgate", s);
      k_balance_dgate<<<blocks, 256, 0, s>>>(idx, dimp, n, 1.0f / (float)T, dgate);
    }
    MOE_CHECK_LAUNCH("balance_dgate");
  }
  return MOE_OK;
}

// ============================================================== router backward
// One warp per token.  dS of a row = sum of its partials (fixed order).
//   v_r = row_gate[r] * dS[r] for every row r of token t (expert e_r)
//   dl[t, e_r] += v_r;  dl[t, idx[t,j]] -= gate[t,j] * sum_r v_r
__global__ void k_router_bwd(const float* __restrict__ ds_part, int nparts,
                             const int32_t* __restrict__ idx, const float* __restrict__ gate,
                             const float* __restrict__ row_gate, const int32_t* __restrict__ slot_row,
                             const int32_t* __restrict__ extra_row, const float* __restrict__ gate_grad,
                             const float* __restrict__ logits, int gate_mode,
                             int T, int E, int k, float* __restrict__ dlogits,
                             float* __restrict__ dS_out, __nv_bfloat16* __restrict__ dl_hi,
                             __nv_bfloat16* __restrict__ dl_lo) {
  __shared__ float s_dl[8][256];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  float* dl = s_dl[w];
  for (int t = blockIdx.x * 8 + w; t < T; t += gridDim.x * 8) {
    for (int e = lane; e < E; e += 32) dl[e] = 0.f;
    __syncwarp();
    float part = 0.f;
    // kept slots (lanes 0..k-1): experts are distinct, plain stores
    if (lane < k) {
      const int r = slot_row[(size_t)t * k + lane];
      if (r >= 0) {
        float ds = 0.f;
#pragma unroll 4
        for (int p = 0; p < nparts; ++p) ds += ds_part[(size_t)r * nparts + p];
        if (dS_out) dS_out[r] = ds;
        const float v = row_gate[r] * ds;
        dl[idx[(size_t)t * k + lane]] = v;
        part = v;
      }
    }
    if (extra_row != nullptr) {
      for (int e = lane; e < E; e += 32) {
        const int r = extra_row[(size_t)t * E + e];
        if (r >= 0) {
          float ds = 0.f;
#pragma unroll 4
          for (int p = 0; p < nparts; ++p) ds += ds_part[(size_t)r * nparts + p];
          if (dS_out) dS_out[r] = ds;
          const float v = row_gate[r] * ds;
          dl[e] = v;
          part += v;
        }
      }
    }
    // fixed-order warp sum
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    __syncwarp();
    // gradient of auxiliary router losses on the gates, through the
    // softmax over the k logits: g_j (a_j - sum_i g_i a_i)
    float ga = 0.f, aj = 0.f;
    if (gate_grad != nullptr && lane < k) {
      aj = gate_grad[(size_t)t * k + lane];
      ga = gate[(size_t)t * k + lane] * aj;
    }
    if (gate_grad != nullptr) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ga += __shfl_xor_sync(0xffffffffu, ga, o);
    }
    if (gate_mode == 0) {
      if (lane < k) {
        const int e = idx[(size_t)t * k + lane];
        const float gj = gate[(size_t)t * k + lane];
        dl[e] -= gj * part;
        if (gate_grad != nullptr) dl[e] += gj * (aj - ga);
      }
    } else {
      // gates are softmax probabilities over all E logits: every expert gets
      // -p_e * (sum of s dS over the rows + sum of g a over the slots)
      float mx = -INFINITY;
      for (int e = lane; e < E; e += 32) mx = fmaxf(mx, logits[(size_t)t * E + e]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      float z = 0.f;
      for (int e = lane; e < E; e += 32) z += expf(logits[(size_t)t * E + e] - mx);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
      const float inv = 1.0f / z;
      __syncwarp();
      if (gate_grad != nullptr && lane < k) {
        const int e = idx[(size_t)t * k + lane];
        dl[e] += gate[(size_t)t * k + lane] * aj;
      }
      __syncwarp();
      for (int e = lane; e < E; e += 32)
        dl[e] -= expf(logits[(size_t)t * E + e] - mx) * inv * (part + ga);
    }
    __syncwarp();
    for (int e = lane; e < E; e += 32) {
      const float v = dl[e];
      dlogits[(size_t)t * E + e] = v;
      if (dl_hi != nullptr) {
        // v = hi + lo with hi = bf16(v), lo = bf16(v - hi): ~16 significant bits
        const __nv_bfloat16 h = __float2bfloat16_rn(v);
        dl_hi[(size_t)t * E + e] = h;
        dl_lo[(size_t)t * E + e] = __float2bfloat16_rn(v - __bfloat162float(h));
      }
    }
    __syncwarp();
  }
}

int launch_router_bwd(const float* ds_part, int nparts, const int32_t* idx, const float* gate,
                      const float* row_gate, const int32_t* slot_row, const int32_t* extra_row,
                      const float* gate_grad, const float* logits, int gate_mode, int T, int E,
                      int k, float* dlogits, float* dS_out, void* dl_hi, void* dl_lo,
                      cudaStream_t s) {
  if (T == 0) return MOE_OK;
  int blocks = (T + 7) / 8;
  if (blocks > device_sm_count() * 16) blocks = device_sm_count() * 16;
  {
    ProfScope _ps("router_bwd", s);
    k_router_bwd<<<blocks, 256, 0, s>>>(ds_part, nparts, idx, gate, row_gate, slot_row, extra_row,
                                        gate_grad, logits, gate_mode, T, E, k, dlogits, dS_out,
                                        (__nv_bfloat16*)dl_hi,
                                        (__nv_bfloat16*)dl_lo);
  }
  MOE_CHECK_LAUNCH("router_bwd");
  return MOE_OK;
}

}  // namespace moe
