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
// One block per (32 K-rows, up to 512 columns, source matrix, expert) of a
// weight [E, K, N] (N contiguous): the 32 rows' 1 KB runs arrive with all of
// the block's loads in flight (8 per thread), so DRAM sees long contiguous
// runs.  Thread p then quantises the two columns 2p, 2p+1 over these 32
// K-values -- one MXFP8 block each, both read with one 32-bit shared load per
// K-value -- and writes the 32 bytes into each column's output row (blocks
// along K).  For the backward copies (blocks along N) the same tile gives
// each of its 32 rows ncols / 32 blocks.
constexpr int WQ_THREADS = 256;
constexpr int WQ_ROWS = 32;          // one MXFP8 block along K
constexpr int WQ_COLS = 512;
constexpr int WQ_LD = WQ_COLS + 8;   // shared row stride (bf16): 16 bytes of padding

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

// W13 = true: sources W1 (blockIdx.z even) and W3 (odd) [E, d, f] -> W13q
// [E, 2f, d] (column n of W1 is row 256 (n/128) + n%128, of W3 that row +
// 128) and, when qa_r is set, W1r / W3r [E, d, f] with blocks along f.
// W13 = false: source W2 [E, f, d] -> W2q [E, d, f] (column n is row n).
template <bool W13>
__global__ void __launch_bounds__(WQ_THREADS, 3)
k_mx_quant_weights(const __nv_bfloat16* __restrict__ wa, const __nv_bfloat16* __restrict__ wb,
                   int K, int N, uint8_t* __restrict__ q, uint8_t* __restrict__ sf,
                   uint8_t* __restrict__ qa_r, uint8_t* __restrict__ sfa_r,
                   uint8_t* __restrict__ qb_r, uint8_t* __restrict__ sfb_r) {
  __shared__ __align__(16) __nv_bfloat16 tile[WQ_ROWS][WQ_LD];
  const int k0 = blockIdx.x * WQ_ROWS, c0 = blockIdx.y * WQ_COLS;
  const int which = W13 ? (blockIdx.z & 1) : 0;
  const int e = W13 ? (blockIdx.z >> 1) : blockIdx.z;
  const int ncols = min(WQ_COLS, N - c0);             // a multiple of 128
  const __nv_bfloat16* src = (which ? wb : wa) + ((size_t)e * K + k0) * N + c0;
  constexpr int VPR = WQ_COLS / 8;                     // 16-byte vectors per tile row
  constexpr int PER = WQ_ROWS * VPR / WQ_THREADS;
  uint4 u[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {   // all loads in flight before the shared stores
    const int v = threadIdx.x + i * WQ_THREADS;
    const int r = v / VPR, c = (v % VPR) * 8;
    if (c < ncols) u[i] = __ldg(reinterpret_cast<const uint4*>(src + (size_t)r * N + c));
  }
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int v = threadIdx.x + i * WQ_THREADS;
    const int r = v / VPR, c = (v % VPR) * 8;
    if (c < ncols) *reinterpret_cast<uint4*>(&tile[r][c]) = u[i];
  }
  __syncthreads();
  const int kchunks = K / 128;
  if (2 * (int)threadIdx.x < ncols) {
    const int p = threadIdx.x;
    uint32_t pk[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) pk[i] = *reinterpret_cast<const uint32_t*>(&tile[i][2 * p]);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int n = c0 + 2 * p + h;                    // source column
      const int row = W13 ? e * 2 * N + 256 * (n >> 7) + 128 * which + (n & 127) : e * N + n;
      mx_store_block_packed(pk, h == 1, q + (size_t)row * K + k0,
                            sf + mx_sf_offset(row, k0 >> 5, kchunks));
    }
  }
  if (W13 && qa_r != nullptr) {
    uint8_t* qr = which ? qb_r : qa_r;
    uint8_t* sr = which ? sfb_r : sfa_r;
    const int nb = ncols / 32;                         // blocks along N per tile row
    for (int item = threadIdx.x; item < WQ_ROWS * nb; item += WQ_THREADS) {
      const int i = item / nb, b = item % nb;
      uint32_t pk[16];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 w4 = *reinterpret_cast<const uint4*>(&tile[i][32 * b + 8 * j]);
        pk[4 * j] = w4.x; pk[4 * j + 1] = w4.y; pk[4 * j + 2] = w4.z; pk[4 * j + 3] = w4.w;
      }
      float v[32];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        v[2 * j] = __uint_as_float(pk[j] << 16);
        v[2 * j + 1] = __uint_as_float(pk[j] & 0xffff0000u);
      }
      const int srow = e * K + k0 + i;                 // row of [E*d, f]
      const int col = c0 + 32 * b;
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
    k_mx_quant_weights<true><<<dim3(d / WQ_ROWS, (f + WQ_COLS - 1) / WQ_COLS, 2 * E), WQ_THREADS,
                               0, s>>>((const __nv_bfloat16*)w1, (const __nv_bfloat16*)w3, d, f,
                                       w13q, w13s, w1rq, w1rs, w3rq, w3rs);
    k_mx_quant_weights<false><<<dim3(f / WQ_ROWS, (d + WQ_COLS - 1) / WQ_COLS, E), WQ_THREADS,
                                0, s>>>((const __nv_bfloat16*)w2, nullptr, f, d, w2q, w2s, nullptr,
                                        nullptr, nullptr, nullptr);
  }
  MOE_CHECK_LAUNCH("mx_quant_weights");
  return MOE_OK;
}

// ============================================================== along tokens
// Row-space matrix [rows, n] bf16 -> Q [n, capr] E4M3 with blocks of 32
// along the rows (the contraction dimension of the weight-gradient GEMMs),
// scales in the layout of mx.cuh with n as the MN dimension and the rows as
// K (capr / 128 K chunks).  Row r of the source is src row r, or, with
// gather_row, token row gather_row[r] of a token-major source (-1: a zero
// row).  Each block owns a 256-column strip and walks its 64-row tiles
// (grid-stride), double-buffered: the next tile's 16-byte cp.async copies
// are in flight while thread p quantises column pair p' = p mod 128 over the
// 32 rows 32 (p / 128).. of the current one (two MXFP8 blocks, each value
// pair one 32-bit shared load) and writes 32 bytes of each column's output
// row.  Only rows below offsets[E] are read or written.  A plan larger than
// capr, or a source row at or past src_rows, is recorded as device data
// check 0x140 (the plan is skipped, the row read as zeros).
constexpr int QC_ROWS = 64, QC_COLS = 256, QC_LD = QC_COLS + 8;
constexpr int QC_TILE = QC_ROWS * QC_LD;               // bf16 elements per buffer

__device__ __forceinline__ void qc_load_tile(__nv_bfloat16* buf, const __nv_bfloat16* src,
                                             const int32_t* gather_row, int src_rows, int n,
                                             int r0, int c0, int ncols, int* status) {
  constexpr int VPR = QC_COLS / 8;
#pragma unroll
  for (int i = 0; i < QC_ROWS * VPR / WQ_THREADS; ++i) {
    const int v = threadIdx.x + i * WQ_THREADS;
    const int r = v / VPR, c = (v % VPR) * 8;
    if (c >= ncols) continue;
    int sr = gather_row != nullptr ? gather_row[r0 + r] : r0 + r;
    if (sr >= src_rows) {   // a row the source does not have: flag it, read a zero row
      record_status(status, 0x140);
      sr = -1;
    }
    const __nv_bfloat16* g = src + (size_t)(sr >= 0 ? sr : 0) * n + c0 + c;
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(buf + r * QC_LD + c);
    const int bytes = sr >= 0 ? 16 : 0;                // 0: zero fill
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(g), "r"(bytes)
                 : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

__global__ void __launch_bounds__(WQ_THREADS, 3)
k_mx_quant_cols(const __nv_bfloat16* __restrict__ src, int src_rows,
                const int32_t* __restrict__ gather_row, const int32_t* __restrict__ offsets, int E,
                int n, int capr, uint8_t* __restrict__ q, uint8_t* __restrict__ sf, int* status) {
  extern __shared__ __align__(16) uint8_t qc_smem[];
  __nv_bfloat16* bufs = reinterpret_cast<__nv_bfloat16*>(qc_smem);
  int R = offsets[E];
  if (R > capr || R < 0 || R % 128) {   // a plan that does not fit the output: flag it, do nothing
    if (threadIdx.x == 0) record_status(status, 0x140);
    return;
  }
  const int c0 = blockIdx.y * QC_COLS;
  const int ncols = min(QC_COLS, n - c0);             // a multiple of 128
  const int ntiles = R / QC_ROWS;                      // R is a multiple of 128
  const int p = threadIdx.x & (QC_COLS / 2 - 1);       // column pair
  const int rb = 32 * (threadIdx.x / (QC_COLS / 2));   // this thread's 32 rows of a tile
  const int kchunks = capr / 128;
  int t = blockIdx.x;
  if (t < ntiles) qc_load_tile(bufs, src, gather_row, src_rows, n, t * QC_ROWS, c0, ncols, status);
  for (int it = 0; t < ntiles; ++it, t += gridDim.x) {
    const int tn = t + gridDim.x;
    __nv_bfloat16* cur = bufs + (it & 1) * QC_TILE;
    if (tn < ntiles) {
      qc_load_tile(bufs + ((it + 1) & 1) * QC_TILE, src, gather_row, src_rows, n, tn * QC_ROWS,
                   c0, ncols, status);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    if (2 * p < ncols) {
      const int r0 = t * QC_ROWS + rb;
      uint32_t pk[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) pk[i] = *reinterpret_cast<const uint32_t*>(cur + (rb + i) * QC_LD + 2 * p);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int col = c0 + 2 * p + h;
        mx_store_block_packed(pk, h == 1, q + (size_t)col * capr + r0,
                              sf + mx_sf_offset(col, r0 >> 5, kchunks));
      }
    }
    __syncthreads();                                   // the buffer is refilled next iteration
  }
}

int launch_mx_quant_cols(const void* src, int src_rows, const int32_t* gather_row,
                         const int32_t* offsets, int E, int n, int capr, uint8_t* q, uint8_t* sf,
                         cudaStream_t s) {
  if (n % 128 || capr % 128) return fail(MOE_ERR_UNSUPPORTED, "token-axis MXFP8 needs n and rows in multiples of 128");
  const int strips = (n + QC_COLS - 1) / QC_COLS;
  int per = device_sm_count() * 3 / strips;            // resident blocks over the column strips
  if (per < 1) per = 1;
  if (per > capr / QC_ROWS) per = capr / QC_ROWS;
  dim3 grid(per, strips);
  const int smem = 2 * QC_TILE * 2;
  cudaError_t e = cudaFuncSetAttribute(k_mx_quant_cols, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return cuda_fail(e, "mx_quant_cols smem attribute");
  {
    ProfScope _ps("mx_quant_cols", s);
    k_mx_quant_cols<<<grid, WQ_THREADS, smem, s>>>((const __nv_bfloat16*)src, src_rows, gather_row,
                                                   offsets, E, n, capr, q, sf, status_ptr());
  }
  MOE_CHECK_LAUNCH("mx_quant_cols");
  return MOE_OK;
}

// ============================================================== rows
// The last nbt blocks own tokens (one warp per token): lanes 4g..4g+3 hold
// the 32 elements of one block as four 16-byte vectors, share its maximum by
// shuffles, and write 8 E4M3 bytes each to every row of the token; the first
// lane of the group writes the scale.  The first blocks of the grid zero the
// padding rows (elements and scales) beside them.
__global__ void __launch_bounds__(256)
k_mx_scatter_rows(const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ slot_row,
                  const int32_t* __restrict__ extra_row, const int32_t* __restrict__ row_token,
                  const int32_t* __restrict__ offsets, int T_, int d, int E, int k, int nbt,
                  uint8_t* __restrict__ q, uint8_t* __restrict__ sf) {
  __shared__ int s_extra[8][256];   // rows added by rounding, per warp (E <= 256)
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int nvec = d / 8, kchunks = d / 128;
  const int nzb = gridDim.x - nbt;        // the first nzb blocks zero the padding rows
  if ((int)blockIdx.x >= nzb) {
    const int t = (blockIdx.x - nzb) * 8 + w;
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
    // a warp tests 32 rows at once and zeroes the padding rows among them
    const int R = offsets[E];
    for (int r0 = (blockIdx.x * 8 + w) * 32; r0 < R; r0 += nzb * 8 * 32) {
      unsigned bal = __ballot_sync(0xffffffffu, r0 + lane < R && row_token[r0 + lane] < 0);
      while (bal) {
        const int r = r0 + __ffs(bal) - 1;
        bal &= bal - 1;
        uint4* d4 = reinterpret_cast<uint4*>(q + (size_t)r * d);
        for (int i = lane; i < d / 16; i += 32) d4[i] = make_uint4(0, 0, 0, 0);
        for (int kb = lane; kb < d / 32; kb += 32) sf[mx_sf_offset(r, kb, kchunks)] = 0;
      }
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
