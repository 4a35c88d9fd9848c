// MXFP8 operand preparation for the block-scaled expert GEMMs (format and
// scale layout: mx.cuh).
//   weights  W1, W3 [E, d, f] -> W13q [E, 2f, d] (K = d contiguous; rows
//            256b..256b+127 are columns 128b.. of W1, rows 256b+128..256b+255
//            the same columns of W3, so one 256-row GEMM tile yields
//            matching H1 / H3 columns) and W2 [E, f, d] ->
//            W2q [E, d, f] (K = f contiguous), blocks of 32 along K; for the
//            backward dX GEMM also W1r, W3r [E, d, f] (the weights' own
//            layout, blocks of 32 along f), from the same loaded tiles.
//   rows     x [T, d] -> Xq [cap, d]: each token row quantised once (blocks
//            of 32 along d) and written to all of its rows in the row space;
//            padding rows get zero elements and zero scales.
#include "common.cuh"
#include "internal.h"
#include "mx.cuh"

namespace moe {

// ============================================================== weights
// One block per (128 K, 128 output rows, expert): the bf16 source tile goes
// to shared memory as [k][n] (all of the block's loads in flight before the
// first store); then thread (p, j) quantises the two adjacent output rows
// 2p, 2p+1 over the 32 K-values 32j..32j+31, reading both with one 32-bit
// shared load per K-value, and writes 32 contiguous bytes of each row.
// 256-thread blocks of at most 80 registers keep three blocks (96 KB of
// loads) in flight per SM.
constexpr int WQ_THREADS = 256;

// Quantise 32 bf16 values held as the low (hi = false) or high halves of
// packed pairs as one MXFP8 block (same arithmetic as mx_store_block, whose
// bf16 rounding is exact here).
__device__ __forceinline__ void mx_store_block_packed(const uint32_t* pk, bool hi, uint8_t* dst,
                                                      uint8_t* sf) {
  auto val = [&](int i) -> float {
    return __uint_as_float(hi ? (pk[i] & 0xffff0000u) : (pk[i] << 16));
  };
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(val(i)));
  const uint32_t code = mx_scale_code(amax);
  const float inv = mx_inv_scale(code);
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    w[i] = cvt_e4m3x2(val(4 * i) * inv, val(4 * i + 1) * inv) |
           (cvt_e4m3x2(val(4 * i + 2) * inv, val(4 * i + 3) * inv) << 16);
  reinterpret_cast<uint4*>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
  reinterpret_cast<uint4*>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
  *sf = (uint8_t)code;
}

template <bool W13>
__global__ void __launch_bounds__(WQ_THREADS, 3)
k_mx_quant_weights(const __nv_bfloat16* __restrict__ wa, const __nv_bfloat16* __restrict__ wb,
                   int K, int N, int Nout, uint8_t* __restrict__ q, uint8_t* __restrict__ sf,
                   uint8_t* __restrict__ qa_r, uint8_t* __restrict__ sfa_r,
                   uint8_t* __restrict__ qb_r, uint8_t* __restrict__ sfb_r) {
  // rows padded by 16 bytes: the row-wise pass reads 16-byte vectors of
  // consecutive rows without bank conflicts
  __shared__ __align__(16) __nv_bfloat16 tile[128][136];
  const int k0 = blockIdx.x * 128, t = blockIdx.y, e = blockIdx.z;
  const int kchunks = K / 128;
  // source tile: 128 K-rows x 128 output rows (16-byte vectors of 8 bf16);
  // output tile t of W13q is W1 (t even) or W3 (t odd), columns 128 (t/2)..
  const __nv_bfloat16* base = W13 ? ((t & 1) ? wb : wa) + (size_t)(t >> 1) * 128
                                  : wa + (size_t)t * 128;
  constexpr int PER = 128 * 16 / WQ_THREADS;
  uint4 u[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {   // all loads in flight before the shared stores
    const int v = threadIdx.x + i * WQ_THREADS;
    u[i] = __ldg(reinterpret_cast<const uint4*>(base + ((size_t)e * K + k0 + (v >> 4)) * N +
                                                (v & 15) * 8));
  }
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int v = threadIdx.x + i * WQ_THREADS;
    *reinterpret_cast<uint4*>(&tile[v >> 4][(v & 15) * 8]) = u[i];
  }
  __syncthreads();
  {
    const int p = threadIdx.x & 63, j = threadIdx.x >> 6;
    uint32_t pk[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) pk[i] = *reinterpret_cast<const uint32_t*>(&tile[32 * j + i][2 * p]);
    const int row = e * Nout + t * 128 + 2 * p;   // output row across experts (Nout % 128 == 0)
#pragma unroll
    for (int h = 0; h < 2; ++h)
      mx_store_block_packed(pk, h == 1, q + (size_t)(row + h) * K + k0 + 32 * j,
                            sf + mx_sf_offset(row + h, (k0 >> 5) + j, kchunks));
  }
  if (W13 && qa_r != nullptr) {
    // row-wise: source row k0 + kk of W1 (t even) or W3 (t odd), 32 columns
    // starting at 128 (t/2) + 32 jb, in the weight's own [E, d, f] layout
    uint8_t* qr = (t & 1) ? qb_r : qa_r;
    uint8_t* sr = (t & 1) ? sfb_r : sfa_r;
#pragma unroll
    for (int it = 0; it < 512 / WQ_THREADS; ++it) {
      const int item = threadIdx.x + it * WQ_THREADS;
      const int kk = item & 127, jb = item >> 7;
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 w4 = *reinterpret_cast<const uint4*>(&tile[kk][32 * jb + 8 * i]);
        pk[4 * i] = w4.x; pk[4 * i + 1] = w4.y; pk[4 * i + 2] = w4.z; pk[4 * i + 3] = w4.w;
      }
      float v[32];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        v[2 * i] = __uint_as_float(pk[i] << 16);
        v[2 * i + 1] = __uint_as_float(pk[i] & 0xffff0000u);
      }
      const int srow = e * K + k0 + kk;         // row of [E*d, f]
      const int col = (t >> 1) * 128 + 32 * jb;
      mx_store_block(v, qr + (size_t)srow * N + col, sr + mx_sf_offset(srow, col >> 5, N / 128));
    }
  }
}

int launch_mx_quant_weights(const void* w1, const void* w3, const void* w2, int E, int d, int f,
                            uint8_t* w13q, uint8_t* w13s, uint8_t* w2q, uint8_t* w2s,
                            uint8_t* w1rq, uint8_t* w1rs, uint8_t* w3rq, uint8_t* w3rs,
                            cudaStream_t s) {
  if (E == 0) return MOE_OK;
  {
    ProfScope _ps("mx_quant_weights", s);
    k_mx_quant_weights<true><<<dim3(d / 128, (2 * f) / 128, E), WQ_THREADS, 0, s>>>(
        (const __nv_bfloat16*)w1, (const __nv_bfloat16*)w3, d, f, 2 * f, w13q, w13s, w1rq, w1rs,
        w3rq, w3rs);
    k_mx_quant_weights<false><<<dim3(f / 128, d / 128, E), WQ_THREADS, 0, s>>>(
        (const __nv_bfloat16*)w2, nullptr, f, d, d, w2q, w2s, nullptr, nullptr, nullptr, nullptr);
  }
  MOE_CHECK_LAUNCH("mx_quant_weights");
  return MOE_OK;
}

// ============================================================== rows
// Blocks [0, nbt) own tokens (one warp per token): lanes 4g..4g+3 hold the 32
// elements of one block as four 16-byte vectors, share its maximum by
// shuffles, and write 8 E4M3 bytes each to every row of the token; the first
// lane of the group writes the scale.  The remaining blocks zero the padding
// rows (elements and scales).
__global__ void __launch_bounds__(256)
k_mx_scatter_rows(const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ slot_row,
                  const int32_t* __restrict__ extra_row, const int32_t* __restrict__ row_token,
                  const int32_t* __restrict__ offsets, int T_, int d, int E, int k, int nbt,
                  uint8_t* __restrict__ q, uint8_t* __restrict__ sf) {
  __shared__ int s_extra[8][256];   // rows added by rounding, per warp (E <= 256)
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int nvec = d / 8, kchunks = d / 128;
  if ((int)blockIdx.x < nbt) {
    const int t = blockIdx.x * 8 + w;
    if (t >= T_) return;  // whole warp
    const int mine = lane < k ? slot_row[(size_t)t * k + lane] : -1;
    int rk[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) rk[j] = __shfl_sync(0xffffffffu, mine, j);
    int n_extra = 0;
    if (extra_row != nullptr) {
      for (int e0 = 0; e0 < E; e0 += 32) {
        const int re = e0 + lane < E ? extra_row[(size_t)t * E + e0 + lane] : -1;
        const unsigned bal = __ballot_sync(0xffffffffu, re >= 0);
        if (re >= 0) s_extra[w][n_extra + __popc(bal & ((1u << lane) - 1u))] = re;
        n_extra += __popc(bal);
      }
      __syncwarp();
    }
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * d);
    for (int i0 = 0; i0 < nvec; i0 += 32) {
      const int i = i0 + lane;
      const bool valid = i < nvec;
      float b[8];
      float amax = 0.f;
      if (valid) {
        const uint4 u = __ldg(src + i);
        const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&u);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          b[e] = __bfloat162float(h[e]);
          amax = fmaxf(amax, fabsf(b[e]));
        }
      }
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      if (!valid) continue;
      const uint32_t code = mx_scale_code(amax);
      const float inv = mx_inv_scale(code);
      uint2 pk;
      pk.x = cvt_e4m3x2(b[0] * inv, b[1] * inv) | (cvt_e4m3x2(b[2] * inv, b[3] * inv) << 16);
      pk.y = cvt_e4m3x2(b[4] * inv, b[5] * inv) | (cvt_e4m3x2(b[6] * inv, b[7] * inv) << 16);
      const bool first = (lane & 3) == 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int r = rk[j];
        if (r >= 0) {
          *reinterpret_cast<uint2*>(q + (size_t)r * d + 8 * i) = pk;
          if (first) sf[mx_sf_offset(r, i >> 2, kchunks)] = (uint8_t)code;
        }
      }
      for (int j = 0; j < n_extra; ++j) {
        const int r = s_extra[w][j];
        *reinterpret_cast<uint2*>(q + (size_t)r * d + 8 * i) = pk;
        if (first) sf[mx_sf_offset(r, i >> 2, kchunks)] = (uint8_t)code;
      }
    }
  } else {
    const int R = offsets[E];
    const int nb = gridDim.x - nbt;
    for (int r = (blockIdx.x - nbt) * 8 + w; r < R; r += nb * 8) {
      if (row_token[r] >= 0) continue;
      uint4* d4 = reinterpret_cast<uint4*>(q + (size_t)r * d);
      for (int i = lane; i < d / 16; i += 32) d4[i] = make_uint4(0, 0, 0, 0);
      for (int kb = lane; kb < d / 32; kb += 32) sf[mx_sf_offset(r, kb, kchunks)] = 0;
    }
  }
}

int launch_mx_scatter_rows(const void* x, const int32_t* slot_row, const int32_t* extra_row,
                           const int32_t* row_token, const int32_t* offsets, int T, int d, int E,
                           int k, uint8_t* q, uint8_t* sf, cudaStream_t s) {
  const int nbt = (T + 7) / 8;
  const int blocks = nbt + device_sm_count() * 2;
  {
    ProfScope _ps("mx_scatter_rows", s);
    k_mx_scatter_rows<<<blocks, 256, 0, s>>>((const __nv_bfloat16*)x, slot_row, extra_row,
                                             row_token, offsets, T, d, E, k, nbt, q, sf);
  }
  MOE_CHECK_LAUNCH("mx_scatter_rows");
  return MOE_OK;
}

}  // namespace moe
