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

// ============================================================== gather rows
// dst[r, :] = src[row_token[r], :] for live rows, 0 for padding rows; r < R.
template <class T>
__global__ void k_gather_rows(const T* __restrict__ src, const int32_t* __restrict__ row_token,
                              const int32_t* __restrict__ offsets, int E, int width,
                              T* __restrict__ dst) {
  const int R = offsets[E];
  const int nvec = width / Vec<T>::N;
  const int warps = blockDim.x >> 5, lane = threadIdx.x & 31;
  for (int r = blockIdx.x * warps + (threadIdx.x >> 5); r < R; r += gridDim.x * warps) {
    const int t = row_token[r];
    const uint4* s = reinterpret_cast<const uint4*>(src + (size_t)(t < 0 ? 0 : t) * width);
    uint4* o = reinterpret_cast<uint4*>(dst + (size_t)r * width);
    for (int i = lane; i < nvec; i += 32) o[i] = t >= 0 ? __ldg(s + i) : make_uint4(0, 0, 0, 0);
  }
}

int launch_gather_rows(const void* src, const int32_t* row_token, const int32_t* offsets, int E,
                       int width, int dtype, void* dst, cudaStream_t s) {
  const int blocks = device_sm_count() * 8;
  if (dtype == MOE_BF16) {
    ProfScope _ps("gather_rows", s);
    k_gather_rows<__nv_bfloat16><<<blocks, 256, 0, s>>>(
        (const __nv_bfloat16*)src, row_token, offsets, E, width, (__nv_bfloat16*)dst);
  } else {
    ProfScope _ps("gather_rows", s);
    k_gather_rows<float><<<blocks, 256, 0, s>>>((const float*)src, row_token, offsets, E, width,
                                                (float*)dst);
  }
  MOE_CHECK_LAUNCH("gather_rows");
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

int launch_token_reduce(const void* src, const float* row_gate, const int32_t* slot_row,
                        const int32_t* extra_row, int T, int width, int E, int k, int dtype,
                        bool weighted, bool out_f32, void* out, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  int blocks = (T + TR_WARPS - 1) / TR_WARPS;
  if (blocks > device_sm_count() * 32) blocks = device_sm_count() * 32;
  if (dtype == MOE_BF16) {
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

// ============================================================== router backward
// One warp per token.  dS of a row = sum of its partials (fixed order).
//   v_r = row_gate[r] * dS[r] for every row r of token t (expert e_r)
//   dl[t, e_r] += v_r;  dl[t, idx[t,j]] -= gate[t,j] * sum_r v_r
__global__ void k_router_bwd(const float* __restrict__ ds_part, int nparts,
                             const int32_t* __restrict__ idx, const float* __restrict__ gate,
                             const float* __restrict__ row_gate, const int32_t* __restrict__ slot_row,
                             const int32_t* __restrict__ extra_row, int T, int E, int k,
                             float* __restrict__ dlogits, float* __restrict__ dS_out,
                             __nv_bfloat16* __restrict__ dl_hi, __nv_bfloat16* __restrict__ dl_lo) {
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
    if (lane < k) {
      const int e = idx[(size_t)t * k + lane];
      dl[e] -= gate[(size_t)t * k + lane] * part;
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
                      int T, int E, int k, float* dlogits, float* dS_out, void* dl_hi,
                      void* dl_lo, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  int blocks = (T + 7) / 8;
  if (blocks > device_sm_count() * 16) blocks = device_sm_count() * 16;
  {
    ProfScope _ps("router_bwd", s);
    k_router_bwd<<<blocks, 256, 0, s>>>(ds_part, nparts, idx, gate, row_gate, slot_row, extra_row, T,
                                        E, k, dlogits, dS_out, (__nv_bfloat16*)dl_hi,
                                        (__nv_bfloat16*)dl_lo);
  }
  MOE_CHECK_LAUNCH("router_bwd");
  return MOE_OK;
}

}  // namespace moe
