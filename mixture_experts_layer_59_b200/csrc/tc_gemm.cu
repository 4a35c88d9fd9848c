// Tensor-core (tcgen05 + TMEM + TMA) grouped GEMMs of the expert FFN,
// forward and backward.
//
// One persistent kernel template serves six GEMMs ("kinds").  Per expert e,
// rows [offsets[e], offsets[e+1]) of the permuted row space (segments start at
// multiples of 128, padding rows are zero):
//   UP    H  = Xg [W1_e | W3_e]      varlen-M, K = d,  epilogue: H and
//                                    A = silu(H1) * H3 (fused SwiGLU)
//   DOWN  Y  = A W2_e                varlen-M, K = f
//   DAP   dA' = dOg W2_e^T           varlen-M, K = d,  epilogue: recompute A
//                                    from H, dS partial = <dA', A>, dA = s dA',
//                                    SwiGLU backward -> dH, and s*A
//   DX    dXp = dH [W1_e | W3_e]^T   varlen-M, K = 2f
//   DW2   dW2_e = (sA)^T dOg         varlen-K (K = rows of e)
//   DW13  [dW1_e | dW3_e] = Xg^T dH  varlen-K
//   RT    logits = x W_gate (+bias)  one group, N = E padded to 64; epilogue:
//                                    top-k (ties: lowest id) and softmax over
//                                    the k logits (Beam sec. 5.3 / Trinity ex. 1)
//   DWG   dW_gate = x^T dlogits      split-K over tokens; dlogits enters as a
//                                    bf16 hi part plus a bf16 lo remainder,
//                                    accumulated in the same fp32 accumulator
//   DXR   dx = (fp32 sum of the token's dX_perm rows) + dlogits W_gate^T
//   UPQ   UP with MXFP8 operands (E4M3, one E8M0 scale per 32 along K):
//         Xq [W13q], epilogue as UP but A leaves as MXFP8 (blocks along f);
//         256-column tiles (128 W1 + 128 W3 columns), one accumulator
//   DOWNQ DOWN with MXFP8 operands: Aq W2q
//   DXQ   DX with MXFP8 operands: dHq [W1r | W3r]^T (dH quantised along 2f by
//         DAPQ, the weights along f in their own layout)
//   DAPQ  DAP whose epilogue also writes dH as MXFP8 for DXQ
//         (kind::mxf8f6f4 block-scaled MMAs, K = 32 per instruction; the two
//         512-byte scale blocks of each stage go shared -> TMEM by tcgen05.cp)
// The grouped GEMM replaces the per-expert loop of the Beam article's
// MoELayer (sec. 5.3); Olmo-core 3 names grouped GEMM for the same purpose;
// dS = <dA', A> without a stored Y is the SonicMoE summary's sec. 1.
//
// CTA layout (320 threads, one CTA per SM):
//   warp 0      TMA producer (one lane): A and B tiles into a ring of stages
//   warp 1      TMEM allocator + MMA issuer (one lane): 128 x BN x 16 UMMAs
//   warps 2..9  epilogue: tcgen05.ld of the fp32 accumulator, fused math,
//               16-byte global stores.  Warp w reads TMEM lanes 32*(w%4)..+31
//               (the rows it may access); warps w and w+4 split the columns.
// The accumulator is double-buffered in TMEM (2 x BN columns) so that the
// epilogue of tile i overlaps the main loop of tile i+1.  Tiles are assigned
// round-robin to the CTAs; the row count R and the per-expert segments are
// read on the device, so no host synchronisation is needed.
#include <dlfcn.h>

#include <cstring>

#include "common.cuh"
#include "internal.h"
#include "mx.cuh"
#include "tcgen05.cuh"

namespace moe {

using namespace tc;

enum Kind : int {
  K_UP = 0, K_DOWN = 1, K_DAP = 2, K_DX = 3, K_DW2 = 4, K_DW13 = 5, K_RT = 6, K_DWG = 7, K_DXR = 8,
  K_UPQ = 9, K_DOWNQ = 10, K_DXQ = 11, K_DAPQ = 12, K_DW2Q = 13, K_DW13Q = 14, K_DAPQW = 15
};
constexpr int NUM_KINDS = 16;
constexpr int MX_SF_COL = 256;         // TMEM column of the scale blocks (after the accumulators)

constexpr int BM = 128;
constexpr int BK = 64;                 // 64 bf16 = 128 bytes = one swizzle row
constexpr int ATOM = 8192;             // one 64 x 64 bf16 TMA box
constexpr int A_BYTES = BM * BK * 2;   // 16 KB
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;
constexpr int THREADS = 320;           // 2 control warps + 8 epilogue warps
constexpr int EPI_THREADS = 256;

// Sigmoid for the tensor-core epilogues (fast exponential and division; the
// results are rounded to bf16 afterwards).
__device__ __forceinline__ float sigmoid_fast(float z) {
  return __fdividef(1.0f, 1.0f + __expf(-z));
}

struct TcArgs {
  CUtensorMap mA;    // A operand
  CUtensorMap mA1;   // second A source (DXR: dlogits lo part)
  CUtensorMap mB0;   // B operand (W1 / W2 / activation / W_gate / dlogits hi)
  CUtensorMap mB1;   // second B source (W3, dlogits lo) where the kind has one
  CUtensorMap sO0;   // bf16 outputs written by TMA stores (32 x 32 boxes, 64-byte swizzle)
  CUtensorMap sO1;
  CUtensorMap sO2;
  const int32_t* offsets;
  int E, d, f;
  int M, N, K;       // varlen-M: N, K fixed; varlen-K: M, N fixed
  // epilogue operands (bf16 outputs go through the sO* store maps)
  const __nv_bfloat16* hin;  // H (DAP)
  const float* row_gate;     // DAP
  float* ds_part;            // DAP: [cap, nparts]
  int nparts;
  int* status;
  // router kinds
  int T, k, splits, chunk;
  int gate_mode;             // RT: 0 softmax over the top-k, 1 softmax over all E
  const float* bias;         // RT: [E] or null
  const float* noise;        // RT: [T, E] routing noise or null
  float* logits;             // RT: [T, E]
  int32_t* idx;              // RT: [T, k]
  float* gate;               // RT: [T, k]
  float* dwg_part;           // DWG: [splits, d, E]
  const float* dx_acc;       // DXR: [T, d] fp32 sums of each token's dX_perm rows
  // MXFP8 kinds: 512-byte scale blocks [rows/128][K/128] of A and [E][N/128][K/128] of B
  const uint8_t* sfa;
  const uint8_t* sfb;
  int kchunks;               // K / 128
  uint8_t* act_q;            // UPQ: A as E4M3 [cap, f]
  uint8_t* act_s;            // UPQ: its scale blocks [cap/128][f/128]
  uint8_t* dh_q;             // DAP (MXFP8 backward): dH as E4M3 [cap, 2f], or null
  uint8_t* dh_s;             // its scale blocks [cap/128][2f/128]
  // DAPQ with MXFP8 weight gradients: dH and s*A quantised along the rows
  // ([2f, capr] and [f, capr] E4M3 + scales) instead of written in bf16
  uint8_t* dht_q;
  uint8_t* dht_s;
  uint8_t* gat_q;
  uint8_t* gat_s;
  int capr;
  const uint8_t* sfb1;       // DXQ: scale blocks of W3r (sfb: of W1r)
  int kh;                    // DXQ: K chunks per weight half (f / 128)
  // bounded waits give up after wait_ns; dbg_no_load (test hook) makes the
  // producer issue no copies so that the consumers' waits expire
  uint64_t wait_ns;
  int dbg_no_load;
};

template <int KIND> struct KT {
  static constexpr bool VARLEN_K = (KIND == K_DW2 || KIND == K_DW13 || KIND == K_DW2Q ||
                                    KIND == K_DW13Q);
  static constexpr bool A_MN = VARLEN_K || KIND == K_DWG;
  static constexpr bool B_MN = (KIND == K_UP || KIND == K_DOWN || VARLEN_K || KIND == K_RT ||
                                KIND == K_DWG);
  static constexpr bool ROUTER = (KIND == K_RT || KIND == K_DWG || KIND == K_DXR);
  static constexpr bool MX = (KIND == K_UPQ || KIND == K_DOWNQ || KIND == K_DXQ ||
                              KIND == K_DW2Q || KIND == K_DW13Q);
};

// A stage holds a 128 x 128-byte A tile and a BN x 128-byte B tile (64 bf16
// or 128 E4M3 elements of K), plus, for the MXFP8 kinds, one 512-byte scale
// block of A and BN/128 of B (the stage is padded to a 1 KB multiple).
// Accumulators are double-buffered in TMEM except for 256-column MXFP8 tiles,
// whose scale blocks need the columns of the second buffer; those also keep
// one 2 KB staging tile per epilogue warp instead of two, to fit 4 stages.
template <int BN, bool MX = false> struct Cfg {
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int SF_TX = MX ? 512 * (1 + BN / 128) : 0;   // scale bytes copied per stage
  static constexpr int SF_BYTES = (SF_TX + 1023) / 1024 * 1024;
  static constexpr int STAGE = A_BYTES + B_BYTES + SF_BYTES;
  static constexpr int TX = A_BYTES + B_BYTES + SF_TX;           // bytes a stage's copies deliver
  static constexpr int STAGES = MX ? (BN == 256 ? 4 : 5) : ((BN == 256) ? 4 : (BN == 128 ? 6 : 8));
  static constexpr int NACC = (MX && BN == 256) ? 1 : 2;
  static constexpr int OUT_TILES = (MX && BN == 256) ? 1 : 2;    // 32 x 32 bf16 staging tiles per epilogue warp
  static constexpr int OUT_BYTES = 8 * OUT_TILES * 2048;
  static constexpr int SMEM = STAGES * STAGE + OUT_BYTES;
  static constexpr int TMEM_COLS = MX ? 512 : 2 * BN;
  static_assert(!MX || NACC * BN == MX_SF_COL, "scale blocks follow the accumulators");
  static_assert(STAGE % 1024 == 0, "stages must keep 1 KB alignment");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

struct TileInfo {
  int e, m0, n0, kb_count, krow0, ntile;
  int rev;   // weight gradients: walk this tile's K rows backwards
};

template <int KIND, int BN>
__device__ __forceinline__ bool tile_info(int t, const TcArgs& a, const int* s_off, int total,
                                          TileInfo& ti) {
  if (t >= total) return false;
  const int ntiles = a.N / BN;
  if constexpr (KIND == K_RT) {
    ti.e = 0;
    ti.m0 = t * BM;
    ti.ntile = 0;
    ti.n0 = 0;
    ti.krow0 = 0;
    ti.kb_count = a.K / BK;
  } else if constexpr (KIND == K_DWG) {
    const int mtiles = a.M / BM;
    const int sp = t / mtiles;          // split of the token range
    ti.e = sp;
    ti.m0 = (t - sp * mtiles) * BM;
    ti.ntile = 0;
    ti.n0 = 0;
    ti.krow0 = sp * a.chunk;
    const int rows = min(a.chunk, a.T - ti.krow0);
    ti.kb_count = 2 * ((rows + BK - 1) / BK);   // hi pass, then lo pass
  } else if constexpr (KIND == K_DXR) {
    const int mt = t / ntiles;
    ti.e = 0;
    ti.ntile = t - mt * ntiles;
    ti.m0 = mt * BM;
    ti.n0 = ti.ntile * BN;
    ti.krow0 = 0;
    ti.kb_count = 2 * ((a.E + BK - 1) / BK);    // hi pass, then lo pass
  } else if constexpr (KT<KIND>::VARLEN_K) {
    const int per = (a.M / BM) * ntiles;
    ti.e = t / per;
    const int rem = t - ti.e * per;
    ti.m0 = (rem / ntiles) * BM;
    ti.ntile = rem % ntiles;
    ti.n0 = ti.ntile * BN;
    ti.krow0 = s_off[ti.e];
    // Tiles of odd waves walk their rows backwards: an expert whose tiles
    // straddle two waves then starts its second wave on the rows the first
    // read last, which are still in L2 (about 1 % faster, fewer DRAM re-reads).
    ti.rev = (t / (int)gridDim.x) & 1;
    // k-blocks of BK bf16 rows, or 128-row K chunks of E4M3
    ti.kb_count = (s_off[ti.e + 1] - s_off[ti.e]) / (KT<KIND>::MX ? 128 : BK);
  } else {
    const int mt = t / ntiles;
    ti.ntile = t - mt * ntiles;
    ti.m0 = mt * BM;
    ti.n0 = ti.ntile * BN;
    int lo = 0, hi = a.E - 1;  // expert owning row m0
    while (lo < hi) {
      int mid = (lo + hi + 1) >> 1;
      if (s_off[mid] <= ti.m0) lo = mid; else hi = mid - 1;
    }
    ti.e = lo;
    ti.krow0 = 0;
    ti.kb_count = KT<KIND>::MX ? a.kchunks : a.K / BK;
  }
  return true;
}

__device__ __forceinline__ bool bounded_wait(uint64_t* bar, uint32_t parity, volatile int* s_abort,
                                             int* status, int code, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63) == 0) {
      if (*s_abort) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        *s_abort = 1;
        record_status(status, 0x200 | code);
        return false;
      }
    }
  }
}

// Element i of 32 bf16 values packed in four uint4, as fp32.
__device__ __forceinline__ float bf16_lane(const uint4 (&p)[4], int i) {
  const uint32_t w = reinterpret_cast<const uint32_t*>(&p[i >> 3])[(i >> 1) & 3];
  return __uint_as_float((i & 1) ? (w & 0xffff0000u) : (w << 16));
}

__device__ __forceinline__ void ld_bf16x32(const __nv_bfloat16* src, float* v) {
  const uint4* p = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 u = p[q];
    __nv_bfloat162 h[4];
    memcpy(h, &u, 16);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f2 = __bfloat1622float2(h[i]);
      v[q * 8 + 2 * i] = f2.x;
      v[q * 8 + 2 * i + 1] = f2.y;
    }
  }
}

// Stage one warp's 32 rows x 32 columns (row = lane) in one of its two 2 KB
// shared tiles (64-byte swizzle: 16-byte chunk c of row r sits at chunk
// c ^ ((r >> 1) & 3)) and store it with one TMA tile store at (col, row0).
// The tiles alternate; before a tile is rewritten, the store issued from it
// two calls ago must have finished reading it.
template <int NT = 2>
__device__ __forceinline__ void stage_store(uint8_t* tiles, int& which, const float* v,
                                            const CUtensorMap* map, int col, int row0, int lane) {
  uint8_t* tile = tiles + which * 2048;
  if (NT == 2) which ^= 1;
  if (lane == 0) {
    if (NT == 2) bulk_wait_read_1();
    else bulk_wait_read_all();
  }
  __syncwarp();
  uint8_t* rowp = tile + lane * 64;
  const int sw = (lane >> 1) & 3;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    __nv_bfloat162 h[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[q * 8 + 2 * i], v[q * 8 + 2 * i + 1]);
    uint4 u;
    memcpy(&u, h, 16);
    *reinterpret_cast<uint4*>(rowp + ((q ^ sw) << 4)) = u;
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(map, tile, col, row0);
    bulk_commit();
  }
}

// A warp's 32 x 32 chunk (lane = row row0 + lane, v = its 32 columns col0..)
// quantised along the rows: each column is one MXFP8 block of 32 rows (the
// bf16 values, as stored).  The chunk goes through shared memory as bf16
// pairs (lane l writes its row, 16 words; lane c then reads column c, one
// 16-bit value per row, once for the maximum and once for the codes; rows
// 17 words apart, so neither side collides in a bank).  Lane c owns its
// column: the block maximum, scale and the 32 codes, written to row col0 + c
// of q [n, capr] and sf.
__device__ __forceinline__ void colq_store(const float* v, uint32_t* tbuf, uint8_t* q, uint8_t* sf,
                                           int col0, int row0, int capr, int lane) {
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
    uint32_t u;
    memcpy(&u, &h, 4);
    tbuf[lane * 17 + j] = u;
  }
  __syncwarp();
  // column values read twice (maximum, then codes) rather than held in registers
  auto val = [&](int i) {
    const uint32_t u = tbuf[i * 17 + (lane >> 1)];
    return __uint_as_float((lane & 1) ? (u & 0xffff0000u) : (u << 16));
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
  __syncwarp();
  uint4* dst = reinterpret_cast<uint4*>(q + (size_t)(col0 + lane) * capr + row0);
  dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
  dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
  sf[mx_sf_offset(col0 + lane, row0 >> 5, capr / 128)] = (uint8_t)code;
}

template <int KIND, int BN>
__global__ void __launch_bounds__(THREADS, 1) k_tc_gemm(const __grid_constant__ TcArgs a) {
  using C = Cfg<BN, KT<KIND>::MX>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[C::STAGES];
  __shared__ __align__(8) uint64_t empty_bar[C::STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ uint32_t s_tmem;
  __shared__ int s_off[257];
  __shared__ volatile int s_abort;

  uint8_t* smem = smem_raw;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // 128-byte swizzled tiles need a 1024-byte aligned base: refuse to run otherwise
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) record_status(a.status, 0x1ff);
    return;
  }

  if (a.offsets != nullptr)
    for (int i = threadIdx.x; i <= a.E; i += blockDim.x) s_off[i] = a.offsets[i];
  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&tfull_bar[s], 1);
      mbar_init(&tempty_bar[s], EPI_THREADS);
    }
    fence_mbar_init();
    prefetch_tmap(&a.mA);
    prefetch_tmap(&a.mB0);
    if (KIND == K_UP || KIND == K_DX || KIND == K_DWG || KIND == K_DXQ) prefetch_tmap(&a.mB1);
    if (KIND == K_DXR) prefetch_tmap(&a.mA1);
  }
  if (warp == 1) {
    tmem_alloc(&s_tmem, C::TMEM_COLS);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem_base = s_tmem;

  int total;
  if constexpr (KIND == K_RT) total = (a.T + BM - 1) / BM;
  else if constexpr (KIND == K_DWG) total = (a.M / BM) * a.splits;
  else if constexpr (KIND == K_DXR) total = ((a.T + BM - 1) / BM) * (a.N / BN);
  else if constexpr (KT<KIND>::VARLEN_K) total = a.E * (a.M / BM) * (a.N / BN);
  else total = (s_off[a.E] / BM) * (a.N / BN);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && !a.dbg_no_load) {
      int stage = 0;
      uint32_t phase = 0;
      TileInfo ti;
      for (int t = blockIdx.x; tile_info<KIND, BN>(t, a, s_off, total, ti); t += gridDim.x) {
        for (int kb = 0; kb < ti.kb_count; ++kb) {
          if (!bounded_wait(&empty_bar[stage], phase ^ 1, &s_abort, a.status, 1, a.wait_ns)) goto producer_done;
          uint8_t* sA = smem + stage * C::STAGE;
          uint8_t* sB = sA + A_BYTES;
          mbar_arrive_expect_tx(&full_bar[stage], C::TX);
          const int k0 = kb * BK;
          if constexpr (KIND == K_UP) {
            tma_load_2d(sA, &a.mA, &full_bar[stage], k0, ti.m0);
            const int nf = ti.ntile * (BN / 2);   // BN / 128 atoms of W1, then of W3
            tma_load_4d(sB, &a.mB0, &full_bar[stage], 0, k0, nf / 64, ti.e);
            tma_load_4d(sB + (BN / 128) * ATOM, &a.mB1, &full_bar[stage], 0, k0, nf / 64, ti.e);
          } else if constexpr (KIND == K_DOWN) {
            tma_load_2d(sA, &a.mA, &full_bar[stage], k0, ti.m0);
            tma_load_4d(sB, &a.mB0, &full_bar[stage], 0, k0, ti.n0 / 64, ti.e);   // BN / 64 atoms
          } else if constexpr (KIND == K_DAP || KIND == K_DAPQ || KIND == K_DAPQW) {
            tma_load_2d(sA, &a.mA, &full_bar[stage], k0, ti.m0);
            tma_load_3d(sB, &a.mB0, &full_bar[stage], k0, ti.n0, ti.e);
          } else if constexpr (KIND == K_DX) {
            tma_load_2d(sA, &a.mA, &full_bar[stage], k0, ti.m0);
            if (k0 < a.f) tma_load_3d(sB, &a.mB0, &full_bar[stage], k0, ti.n0, ti.e);
            else tma_load_3d(sB, &a.mB1, &full_bar[stage], k0 - a.f, ti.n0, ti.e);
          } else if constexpr (KIND == K_RT) {
            // CTAs start their K loop at different k-blocks so that concurrent
            // tile loads spread over more DRAM pages (measured: -18 % time at
            // 16 K tokens); the sum order of each row's logits is still fixed
            const int kr = ((kb + (int)blockIdx.x * 5) % ti.kb_count) * BK;
            tma_load_2d(sA, &a.mA, &full_bar[stage], kr, ti.m0);
#pragma unroll
            for (int h = 0; h < BN / 64; ++h)
              tma_load_2d(sB + h * ATOM, &a.mB0, &full_bar[stage], 64 * h, kr);
          } else if constexpr (KIND == K_DWG) {
            const int nkb = ti.kb_count / 2;
            const int pass = kb >= nkb;
            const int r = ti.krow0 + (kb - pass * nkb) * BK;
            tma_load_2d(sA, &a.mA, &full_bar[stage], ti.m0, r);
            tma_load_2d(sA + ATOM, &a.mA, &full_bar[stage], ti.m0 + 64, r);
            const CUtensorMap* mb = pass ? &a.mB1 : &a.mB0;
#pragma unroll
            for (int h = 0; h < BN / 64; ++h)
              tma_load_2d(sB + h * ATOM, mb, &full_bar[stage], 64 * h, r);
          } else if constexpr (KT<KIND>::MX && KT<KIND>::VARLEN_K) {
            // weight gradients on MXFP8 operands: A [M, capr] and B [N, capr]
            // E4M3 with blocks along the rows of the row space (K); this
            // expert's K chunks start at row krow0 (a multiple of 128)
            const int kc = ti.krow0 / 128 + kb;
            tma_load_3d(sA, &a.mA, &full_bar[stage], kc * 128, ti.m0, 0);
            tma_load_3d(sB, &a.mB0, &full_bar[stage], kc * 128, ti.n0, 0);
            uint8_t* sSF = sB + C::B_BYTES;
            bulk_load(sSF, a.sfa + ((size_t)(ti.m0 / BM) * a.kchunks + kc) * 512, 512,
                      &full_bar[stage]);
#pragma unroll
            for (int b = 0; b < BN / 128; ++b)
              bulk_load(sSF + 512 * (1 + b), a.sfb + ((size_t)(ti.n0 / 128 + b) * a.kchunks + kc) * 512,
                        512, &full_bar[stage]);
          } else if constexpr (KT<KIND>::MX) {
            // E4M3 tiles: 128 elements of K = 128 bytes; then the A and B
            // scale blocks of this K chunk
            // DXQ: K chunks [0, kh) come from W1r, [kh, 2kh) from W3r
            const bool hi = KIND == K_DXQ && kb >= a.kh;
            const int kk = hi ? kb - a.kh : kb;
            const int kcs = KIND == K_DXQ ? a.kh : a.kchunks;
            tma_load_3d(sA, &a.mA, &full_bar[stage], kb * 128, ti.m0, 0);
            tma_load_3d(sB, hi ? &a.mB1 : &a.mB0, &full_bar[stage], kk * 128, ti.n0, ti.e);
            uint8_t* sSF = sB + C::B_BYTES;
            bulk_load(sSF, a.sfa + ((size_t)(ti.m0 / BM) * a.kchunks + kb) * 512, 512,
                      &full_bar[stage]);
            const uint8_t* sfb = hi ? a.sfb1 : a.sfb;
#pragma unroll
            for (int b = 0; b < BN / 128; ++b)
              bulk_load(sSF + 512 * (1 + b),
                        sfb + ((size_t)(ti.e * (a.N / 128) + ti.n0 / 128 + b) * kcs + kk) * 512,
                        512, &full_bar[stage]);
          } else if constexpr (KIND == K_DXR) {
            const int nkb = ti.kb_count / 2;
            const int pass = kb >= nkb;
            const int kk = (kb - pass * nkb) * BK;
            tma_load_2d(sA, pass ? &a.mA1 : &a.mA, &full_bar[stage], kk, ti.m0);
            tma_load_2d(sB, &a.mB0, &full_bar[stage], kk, ti.n0);
          } else {  // varlen-K: A and B are row-space activations, MN-major
            const int r = ti.krow0 + (ti.rev ? (ti.kb_count - 1 - kb) * BK : k0);
            tma_load_4d(sA, &a.mA, &full_bar[stage], 0, r, ti.m0 / 64, 0);    // 2 atoms
            tma_load_4d(sB, &a.mB0, &full_bar[stage], 0, r, ti.n0 / 64, 0);   // BN / 64 atoms
          }
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
      }
    producer_done:;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16(BM, BN, KT<KIND>::A_MN, KT<KIND>::B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      TileInfo ti;
      for (int t = blockIdx.x; tile_info<KIND, BN>(t, a, s_off, total, ti); t += gridDim.x, ++it) {
        const int acc = C::NACC == 1 ? 0 : (it & 1);
        const uint32_t acc_phase = C::NACC == 1 ? (it & 1) : ((it >> 1) & 1);
        if (!bounded_wait(&tempty_bar[acc], acc_phase ^ 1, &s_abort, a.status, 2, a.wait_ns)) break;
        fence_after_sync();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < ti.kb_count; ++kb) {
          if (!bounded_wait(&full_bar[stage], phase, &s_abort, a.status, 3, a.wait_ns)) goto mma_done;
          fence_after_sync();
          const uint32_t sA = smem_u32(smem + stage * C::STAGE);
          const uint32_t sB = sA + A_BYTES;
          if constexpr (KT<KIND>::MX) {
            // scale blocks -> TMEM (in order with the MMAs below and with the
            // previous stage's MMAs, which have read the old blocks)
            const uint32_t sSF = sB + C::B_BYTES;
            const uint32_t sfa = tmem_base + MX_SF_COL, sfb = tmem_base + MX_SF_COL + 4;
            tmem_cp_32x128b_x4(sfa, sdesc_noswz(sSF, 16, 128));
#pragma unroll
            for (int b = 0; b < BN / 128; ++b)      // B rows 128b.. -> columns sfb + 4b..
              tmem_cp_32x128b_x4(sfb + 4 * b, sdesc_noswz(sSF + 512 * (1 + b), 16, 128));
#pragma unroll
            for (uint32_t ks = 0; ks < 4; ++ks) {   // K = 32 E4M3 (32 bytes) per MMA
              umma_mxf8(d_tmem, sdesc_sw128(sA + ks * 32, 16, 1024),
                        sdesc_sw128(sB + ks * 32, 16, 1024), idesc_mxf8(BM, BN, ks),
                        sfa | (ks << 30), sfb | (ks << 30), (kb | ks) != 0);
            }
          } else {
#pragma unroll
          for (int ks = 0; ks < BK / 16; ++ks) {
            const uint64_t ad = KT<KIND>::A_MN ? sdesc_sw128(sA + ks * 2048, ATOM, 1024)
                                               : sdesc_sw128(sA + ks * 32, 16, 1024);
            const uint64_t bd = KT<KIND>::B_MN ? sdesc_sw128(sB + ks * 2048, ATOM, 1024)
                                               : sdesc_sw128(sB + ks * 32, 16, 1024);
            umma_bf16(d_tmem, ad, bd, IDESC, (kb | ks) != 0);
          }
          }
          umma_commit(&empty_bar[stage]);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
        if (ti.kb_count > 0) umma_commit(&tfull_bar[acc]);
        else mbar_arrive(&tfull_bar[acc]);
      }
    mma_done:;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                      // TMEM lane quarter of this warp
    const int half = (warp - 2) >> 2;            // which half of the tile's columns
    const int rloc = q * 32 + lane;              // row of the tile owned by this thread
    int obuf = 0;                                // staging tile used by the next store
    int it = 0;
    TileInfo ti;
    for (int t = blockIdx.x; tile_info<KIND, BN>(t, a, s_off, total, ti); t += gridDim.x, ++it) {
      const int acc = C::NACC == 1 ? 0 : (it & 1);
      const uint32_t acc_phase = C::NACC == 1 ? (it & 1) : ((it >> 1) & 1);
      // DAP: the first chunk of H does not depend on the accumulator, so its
      // loads are issued before waiting for the main loop
      uint4 hn1[4], hn3[4];
      const __nv_bfloat16* hrow = nullptr;
      if constexpr (KIND == K_DAP || KIND == K_DAPQ || KIND == K_DAPQW) {
        hrow = a.hin + (size_t)(ti.m0 + rloc) * 2 * a.f;
        const uint4* s1 = reinterpret_cast<const uint4*>(hrow + ti.n0 + half * (BN / 2));
        const uint4* s3 = reinterpret_cast<const uint4*>(hrow + a.f + ti.n0 + half * (BN / 2));
#pragma unroll
        for (int q = 0; q < 4; ++q) { hn1[q] = s1[q]; hn3[q] = s3[q]; }
      }
      if (!bounded_wait(&tfull_bar[acc], acc_phase, &s_abort, a.status, 4, a.wait_ns)) break;
      fence_after_sync();
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN;
      const int row = ti.m0 + rloc;
      float v[32];
      uint32_t r[32];
      uint8_t* otile = smem + C::STAGES * C::STAGE + (warp - 2) * (C::OUT_TILES * 2048);
      const int row0 = ti.m0 + q * 32;           // first row of this warp's 32-row slab
      bool released = false;  // accumulator handed back before the end of the epilogue
      if constexpr (KT<KIND>::MX && C::NACC == 1) {
        // one accumulator: copy this thread's 4 x 32 columns to registers and
        // release it at once, so that the next tile's MMAs overlap the math
        // and stores below
        uint32_t ra[32], rb[32], rc[32], rd[32];
        int col[4];
        if constexpr (KIND == K_UPQ) {   // H1 cols half*64.., H3 cols 128 + half*64..
          col[0] = half * 64; col[1] = half * 64 + 32; col[2] = 128 + half * 64; col[3] = 160 + half * 64;
        } else {
          col[0] = half * 128; col[1] = col[0] + 32; col[2] = col[0] + 64; col[3] = col[0] + 96;
        }
        tmem_ld32(tbase + col[0], ra);
        tmem_ld32(tbase + col[1], rb);
        tmem_ld32(tbase + col[2], rc);
        tmem_ld32(tbase + col[3], rd);
        tmem_ld_wait();
        fence_before_sync();
        mbar_arrive(&tempty_bar[acc]);
        released = true;
        if constexpr (KIND == K_UPQ) {
          const int f = a.f, nf = ti.ntile * (BN / 2);
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const uint32_t* r1 = j ? rb : ra;
            const uint32_t* r3 = j ? rd : rc;
            const int c = half * 64 + 32 * j;
            float h3[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) { v[i] = __uint_as_float(r1[i]); h3[i] = __uint_as_float(r3[i]); }
            stage_store<C::OUT_TILES>(otile, obuf, v, &a.sO0, nf + c, row0, lane);        // H1
            stage_store<C::OUT_TILES>(otile, obuf, h3, &a.sO0, f + nf + c, row0, lane);   // H3
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float h1 = bf16_round(v[i]);
              v[i] = h1 * sigmoid_fast(h1) * bf16_round(h3[i]);
            }
            mx_store_block(v, a.act_q + (size_t)row * f + nf + c,
                           a.act_s + mx_sf_offset(row, (nf + c) / 32, f / 128));
          }
        } else if constexpr (KT<KIND>::VARLEN_K) {
          // dW rows e*M + m; an expert without rows ran no MMA: zeros
          const int orow0 = ti.e * a.M + row0;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t* rr = j == 0 ? ra : (j == 1 ? rb : (j == 2 ? rc : rd));
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = ti.kb_count > 0 ? __uint_as_float(rr[i]) : 0.f;
            const int cc = ti.n0 + col[j];
            if constexpr (KIND == K_DW2Q) {
              stage_store<C::OUT_TILES>(otile, obuf, v, &a.sO0, cc, orow0, lane);
            } else {
              if (cc < a.f) stage_store<C::OUT_TILES>(otile, obuf, v, &a.sO0, cc, orow0, lane);
              else stage_store<C::OUT_TILES>(otile, obuf, v, &a.sO1, cc - a.f, orow0, lane);
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t* rr = j == 0 ? ra : (j == 1 ? rb : (j == 2 ? rc : rd));
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(rr[i]);
            stage_store<C::OUT_TILES>(otile, obuf, v, &a.sO0, ti.n0 + col[j], row0, lane);
          }
        }
      } else if constexpr (KIND == K_UP || KIND == K_UPQ) {
        const int f = a.f, nf = ti.ntile * (BN / 2);
        float h3[32];
        for (int c = half * (BN / 4); c < (half + 1) * (BN / 4); c += 32) {
          tmem_ld32(tbase + c, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
          tmem_ld32(tbase + BN / 2 + c, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) h3[i] = __uint_as_float(r[i]);
          stage_store<C::OUT_TILES>(otile, obuf, v, &a.sO0, nf + c, row0, lane);        // H1
          stage_store<C::OUT_TILES>(otile, obuf, h3, &a.sO0, f + nf + c, row0, lane);   // H3
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float h1 = bf16_round(v[i]);
            v[i] = h1 * sigmoid_fast(h1) * bf16_round(h3[i]);
          }
          if constexpr (KIND == K_UPQ) {
            // A (bf16-rounded) as one MXFP8 block: this thread's 32 columns
            mx_store_block(v, a.act_q + (size_t)row * f + nf + c,
                           a.act_s + mx_sf_offset(row, (nf + c) / 32, f / 128));
          } else {
            stage_store<C::OUT_TILES>(otile, obuf, v, &a.sO1, nf + c, row0, lane);      // A
          }
        }
      } else if constexpr (KIND == K_DOWN || KIND == K_DX || KIND == K_DOWNQ || KIND == K_DXQ) {
        for (int c = half * (BN / 2); c < (half + 1) * (BN / 2); c += 32) {
          tmem_ld32(tbase + c, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
          stage_store<C::OUT_TILES>(otile, obuf, v, &a.sO0, ti.n0 + c, row0, lane);
        }
      } else if constexpr (KIND == K_DAP || KIND == K_DAPQ || KIND == K_DAPQW) {
        const int f = a.f;
        const float g = a.row_gate[row];
        float ds = 0.f;
        const int c_end = (half + 1) * (BN / 2);
        for (int c = half * (BN / 2); c < c_end; c += 32) {
          tmem_ld32(tbase + c, r);
          // this chunk's H (prefetched), then the next chunk's loads in flight
          uint4 p1[4], p3[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) { p1[q] = hn1[q]; p3[q] = hn3[q]; }
          if (c + 32 < c_end) {
            const uint4* s1 = reinterpret_cast<const uint4*>(hrow + ti.n0 + c + 32);
            const uint4* s3 = reinterpret_cast<const uint4*>(hrow + f + ti.n0 + c + 32);
#pragma unroll
            for (int q = 0; q < 4; ++q) { hn1[q] = s1[q]; hn3[q] = s3[q]; }
          }
          tmem_ld_wait();
          float da3[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float h1 = bf16_lane(p1, i), h3 = bf16_lane(p3, i);
            const float dap = __uint_as_float(r[i]);
            const float sg = sigmoid_fast(h1);
            const float sl = h1 * sg;
            const float av = bf16_round(sl * h3);
            ds = fmaf(dap, av, ds);
            const float da = g * dap;
            v[i] = da * h3 * (sg * (1.0f + h1 * (1.0f - sg)));
            da3[i] = da * sl;
            r[i] = __float_as_uint(g * av);                           // s * A
          }
          // MXFP8 weight gradients: dH and s*A leave quantised along the rows
          // instead of in bf16 (the staging tiles hold the transposes)
          constexpr bool colq = KIND == K_DAPQW;
          uint32_t* tbuf = reinterpret_cast<uint32_t*>(otile);
          if constexpr (!colq) {
            stage_store<C::OUT_TILES>(otile, obuf, v, &a.sO0, ti.n0 + c, row0, lane);       // dH1
            stage_store<C::OUT_TILES>(otile, obuf, da3, &a.sO0, f + ti.n0 + c, row0, lane); // dH3
          }
          if constexpr (KIND == K_DAPQ || KIND == K_DAPQW) {  // MXFP8 backward: dH blocks along 2f for the dX GEMM
            const int kc = (2 * f) / 128;
            mx_store_block(v, a.dh_q + (size_t)row * 2 * f + ti.n0 + c,
                           a.dh_s + mx_sf_offset(row, (ti.n0 + c) / 32, kc));
            mx_store_block(da3, a.dh_q + (size_t)row * 2 * f + f + ti.n0 + c,
                           a.dh_s + mx_sf_offset(row, (f + ti.n0 + c) / 32, kc));
            if constexpr (colq) {
              colq_store(v, tbuf, a.dht_q, a.dht_s, ti.n0 + c, row0, a.capr, lane);
              colq_store(da3, tbuf, a.dht_q, a.dht_s, f + ti.n0 + c, row0, a.capr, lane);
            }
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
          if constexpr (colq) colq_store(v, tbuf, a.gat_q, a.gat_s, ti.n0 + c, row0, a.capr, lane);   // s * A
          else stage_store<C::OUT_TILES>(otile, obuf, v, &a.sO1, ti.n0 + c, row0, lane);   // s * A
        }
        a.ds_part[(size_t)row * a.nparts + 2 * ti.ntile + half] = ds;
      } else if constexpr (KIND == K_RT) {
        // logits (+bias) and a running top-8 list kept sorted in registers;
        // equal values keep the lower expert id first (ids arrive ascending)
        if (half == 0) {
          const int t = row;
          const bool valid = t < a.T;
          float tv[8];
          int tix[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) { tv[j] = -INFINITY; tix[j] = 0x7fffffff; }
          for (int c = 0; c < a.E; c += 32) {
            tmem_ld32(tbase + c, r);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              v[i] = __uint_as_float(r[i]);
              if (a.bias && c + i < a.E) v[i] += a.bias[c + i];
              if (a.noise && valid && c + i < a.E) v[i] += a.noise[(size_t)t * a.E + c + i];
            }
            if (valid) {
              float4* dst = reinterpret_cast<float4*>(a.logits + (size_t)t * a.E + c);
#pragma unroll
              for (int q = 0; q < 8; ++q)
                if (c + 4 * q < a.E) dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              if (c + i < a.E && v[i] > tv[7]) {
                tv[7] = v[i];
                tix[7] = c + i;
#pragma unroll
                for (int j = 7; j > 0; --j) {
                  if (tv[j] > tv[j - 1]) {
                    const float fv = tv[j]; tv[j] = tv[j - 1]; tv[j - 1] = fv;
                    const int iv = tix[j]; tix[j] = tix[j - 1]; tix[j - 1] = iv;
                  }
                }
              }
            }
          }
          // gate_mode 1: normaliser over all E logits, from a second pass over
          // the accumulator (every lane of the warp takes part in the loads)
          float zall = 0.f;
          if (a.gate_mode == 1) {
            for (int c = 0; c < a.E; c += 32) {
              tmem_ld32(tbase + c, r);
              tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (c + i < a.E) {
                  float l = __uint_as_float(r[i]);
                  if (a.bias) l += a.bias[c + i];
                  if (a.noise && valid) l += a.noise[(size_t)t * a.E + c + i];
                  zall += expf(l - tv[0]);
                }
            }
          }
          if (valid) {
            const float m = tv[0];
            float z = 0.f, ex[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              ex[j] = j < a.k ? expf(tv[j] - m) : 0.f;
              z += ex[j];
            }
            if (a.gate_mode == 1) z = zall;
            const float inv = 1.0f / z;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              if (j < a.k) {
                a.idx[(size_t)t * a.k + j] = tix[j];
                a.gate[(size_t)t * a.k + j] = ex[j] * inv;
              }
            }
          }
        }
      } else if constexpr (KIND == K_DWG) {
        // row = d index; partial sums of split ti.e
        float* dst = a.dwg_part + ((size_t)ti.e * a.M + row) * a.E;
        for (int c = half * (BN / 2); c < a.E && c < (half + 1) * (BN / 2); c += 32) {
          tmem_ld32(tbase + c, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c + i < a.E) dst[c + i] = __uint_as_float(r[i]);
        }
      } else if constexpr (KIND == K_DXR) {
        const int t = row;
        const bool valid = t < a.T;
        for (int c = half * (BN / 2); c < (half + 1) * (BN / 2); c += 32) {
          tmem_ld32(tbase + c, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
          const int col = ti.n0 + c;
          if (valid) {
            const float4* s4 = reinterpret_cast<const float4*>(a.dx_acc + (size_t)t * a.N + col);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 u = s4[q];
              v[4 * q] += u.x; v[4 * q + 1] += u.y; v[4 * q + 2] += u.z; v[4 * q + 3] += u.w;
            }
          }
          // rows at or beyond T are clipped by the tensor map
          stage_store<C::OUT_TILES>(otile, obuf, v, &a.sO0, col, row0, lane);
        }
      } else {  // DW2 / DW13: output row m = row of dW_e (maps view dW as [E*M, N])
        const int orow0 = ti.e * a.M + row0;
        for (int c = half * (BN / 2); c < (half + 1) * (BN / 2); c += 32) {
          if (ti.kb_count > 0) {
            tmem_ld32(tbase + c, r);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0.f;
          }
          const int col = ti.n0 + c;
          if constexpr (KIND == K_DW2) {
            stage_store<C::OUT_TILES>(otile, obuf, v, &a.sO0, col, orow0, lane);
          } else {
            if (col < a.f) stage_store<C::OUT_TILES>(otile, obuf, v, &a.sO0, col, orow0, lane);
            else stage_store<C::OUT_TILES>(otile, obuf, v, &a.sO1, col - a.f, orow0, lane);
          }
        }
      }
      if (!released) {
        fence_before_sync();
        mbar_arrive(&tempty_bar[acc]);
      }
    }
  }

  // the epilogue's bulk stores must finish before the CTA exits
  if (warp >= 2 && lane == 0) bulk_wait_all();

  // on an aborted run give in-flight TMA copies and MMAs time to land
  if (s_abort) {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 2000000ull) __nanosleep(1000);
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    fence_after_sync();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ============================================================== host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Looked up once; the initialisation of a function-local static is
// thread-safe, so host threads may make their first calls concurrently.
static EncodeTiledFn encode_fn() {
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* h = dlopen("libcuda.so.1", RTLD_NOW | RTLD_GLOBAL);
    return h ? reinterpret_cast<EncodeTiledFn>(dlsym(h, "cuTensorMapEncodeTiled")) : nullptr;
  }();
  return fn;
}

bool tc_available() {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return true;  // sizing on a host without a GPU
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  (void)minor;
  return major == 10;
}

// dS partial sums per row: one per N tile of the DAP GEMM and column half.
int tc_num_dS_parts(int f) { return 2 * ((f % 256 == 0) ? f / 256 : f / 128); }

// bf16 row-major [outer, inner] viewed in boxes of box_outer x box_inner.
static int make_map_2d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer,
                       uint32_t box_inner, uint32_t box_outer,
                       CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled (2d) failed: " + std::to_string((int)r));
  return MOE_OK;
}

// 8-bit [d2, d1, d0] (d0 innermost; d2 = 1 for a matrix) in boxes of box1 x
// box0 bytes, 128-byte swizzle (E4M3 operand tiles).
static int make_map_u8(CUtensorMap* m, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2,
                       uint32_t box0, uint32_t box1) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0, d0 * d1};
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box,
                  es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled (u8) failed: " + std::to_string((int)r));
  return MOE_OK;
}

// Output map of the epilogue's TMA stores: 32 x 32 boxes, 64-byte swizzle.
static int make_store_map(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer) {
  return make_map_2d(m, ptr, inner, outer, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
}

// bf16 [batch, outer, inner] (inner contiguous, a multiple of 64) as the
// 4-d view [batch][inner / 64][outer][64]: one box brings `atoms` adjacent
// 64-column blocks of BK rows, stored block after block (BK x 128 bytes
// each, 128-byte swizzle) -- the shared-memory layout of an MN-major
// operand -- so a stage's operand takes one copy instead of one per block.
static int make_map_atoms(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer,
                          uint64_t batch, uint32_t atoms) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  if (inner % 64 != 0) return fail(MOE_ERR_INVALID_ARG, "operand width not a multiple of 64");
  cuuint64_t dims[4] = {64, outer, inner / 64, batch};
  cuuint64_t strides[3] = {inner * 2, 128, inner * outer * 2};
  cuuint32_t box[4] = {64, (cuuint32_t)BK, atoms, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled (atoms) failed: " + std::to_string((int)r));
  return MOE_OK;
}

// bf16 [d2, d1, d0] (d0 innermost) viewed in boxes of box1 x box0.
static int make_map_3d(CUtensorMap* m, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2,
                       uint32_t box0, uint32_t box1) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled (3d) failed: " + std::to_string((int)r));
  return MOE_OK;
}

template <int KIND, int BN>
static int launch(const TcArgs& args, int grid, cudaStream_t s) {
  using C = Cfg<BN, KT<KIND>::MX>;
  TcArgs a = args;
  a.wait_ns = WAIT_LIMIT_NS;
  a.dbg_no_load = 0;
  if (const long long dbg = take_debug_expire(); dbg > 0) {
    a.wait_ns = (uint64_t)dbg;
    a.dbg_no_load = 1;
  }
  cudaError_t e = cudaFuncSetAttribute(k_tc_gemm<KIND, BN>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return cuda_fail(e, "tc gemm smem attribute");
  static const char* kNames[NUM_KINDS] = {
      "tc_up",   "tc_down",   "tc_dap",       "tc_dx",        "tc_dw2",   "tc_dw13",
      "tc_router", "tc_router_dw", "tc_dx_router", "tc_up_mxfp8", "tc_down_mxfp8", "tc_dx_mxfp8",
      "tc_dap", "tc_dw2_mxfp8", "tc_dw13_mxfp8", "tc_dap"};
  static_assert(KIND >= 0 && KIND < NUM_KINDS, "kind out of range");
  {
    ProfScope _ps(kNames[KIND], s);
    k_tc_gemm<KIND, BN><<<grid, THREADS, C::SMEM, s>>>(a);
  }
  MOE_CHECK_LAUNCH("tc_gemm");
  return MOE_OK;
}

template <int KIND>
static int launch_bn(const TcArgs& a, int bn, int grid, cudaStream_t s) {
  if (bn == 256) return launch<KIND, 256>(a, grid, s);
  if (bn == 64) return launch<KIND, 64>(a, grid, s);
  return launch<KIND, 128>(a, grid, s);
}

// N tile covering E router columns: 64, 128 or 256.
static int router_bn(int E) { return E <= 64 ? 64 : (E <= 128 ? 128 : 256); }

static int pick_bn(int n) { return n % 256 == 0 ? 256 : 128; }

static TcArgs base_args(const FfnPtrs& p) {
  TcArgs a;
  memset(&a, 0, sizeof(a));
  a.offsets = p.offsets;
  a.E = p.E;
  a.d = p.d;
  a.f = p.f;
  a.status = status_ptr();
  return a;
}

// ------------------------------------------------------------ router
bool tc_router_ok(int E) { return E % 8 == 0 && E <= 256 && tc_available(); }

int tc_dwg_splits(int T, int d, int* chunk) {
  // as many token splits as keep every (split, d-tile) pair in one wave on the
  // 148 SMs: a second partial wave would double the kernel time
  const int mtiles = d / BM;
  int splits = 148 / mtiles;
  const int max_splits = (T + BK - 1) / BK;
  if (splits > max_splits) splits = max_splits;
  if (splits < 1) splits = 1;
  int c = (T + splits - 1) / splits;
  c = (c + BK - 1) / BK * BK;
  if (c < BK) c = BK;
  *chunk = c;
  return (T + c - 1) / c > 0 ? (T + c - 1) / c : 1;
}

int tc_router_fwd(const void* x, const void* wg, const float* bias, const float* noise, int T,
                  int d, int E, int k, int gate_mode, float* logits, int32_t* idx, float* gate,
                  int num_sms, cudaStream_t s) {
  TcArgs a;
  memset(&a, 0, sizeof(a));
  a.gate_mode = gate_mode;
  a.E = E;
  a.d = d;
  a.K = d;
  a.N = router_bn(E);
  a.T = T;
  a.k = k;
  a.bias = bias;
  a.noise = noise;
  a.logits = logits;
  a.idx = idx;
  a.gate = gate;
  a.status = status_ptr();
  int rc;
  if ((rc = make_map_2d(&a.mA, x, d, T, 64, BM))) return rc;
  if ((rc = make_map_2d(&a.mB0, wg, E, d, 64, 64))) return rc;
  const int tiles = (T + BM - 1) / BM;
  return launch_bn<K_RT>(a, a.N, tiles < num_sms ? tiles : num_sms, s);
}

__global__ void k_dwg_reduce(const float* __restrict__ part, int splits, int n,
                             float* __restrict__ out) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    float acc = 0.f;
    for (int sp = 0; sp < splits; ++sp) acc += part[(size_t)sp * n + i];
    out[i] = acc;
  }
}

int tc_router_bwd(const void* x, const void* wg, const void* dl_hi, const void* dl_lo, int T,
                  int d, int E, int k, float* dwg_part, float* dw_gate, const float* dx_acc,
                  void* dx, int num_sms, cudaStream_t s) {
  int rc;
  {  // dW_gate = x^T (dl_hi + dl_lo), split over tokens, then a fixed-order sum
    TcArgs a;
    memset(&a, 0, sizeof(a));
    a.E = E;
    a.d = d;
    a.M = d;
    a.N = router_bn(E);
    a.T = T;
    a.status = status_ptr();
    a.splits = tc_dwg_splits(T, d, &a.chunk);
    a.dwg_part = dwg_part;
    if ((rc = make_map_2d(&a.mA, x, d, T, 64, 64))) return rc;
    if ((rc = make_map_2d(&a.mB0, dl_hi, E, T, 64, 64))) return rc;
    if ((rc = make_map_2d(&a.mB1, dl_lo, E, T, 64, 64))) return rc;
    const int tiles = (d / BM) * a.splits;
    if ((rc = launch_bn<K_DWG>(a, a.N, tiles < num_sms ? tiles : num_sms, s))) return rc;
    {
      ProfScope _ps("dwg_reduce", s);
      k_dwg_reduce<<<num_sms * 4, 256, 0, s>>>(dwg_part, a.splits, d * E, dw_gate);
    }
    MOE_CHECK_LAUNCH("dwg_reduce");
  }
  if (dx != nullptr) {  // dx = fp32 unpermute-sum of dX_perm + dl W_gate^T
    TcArgs a;
    memset(&a, 0, sizeof(a));
    a.E = E;
    a.d = d;
    a.N = d;
    a.T = T;
    a.k = k;
    a.status = status_ptr();
    a.dx_acc = dx_acc;
    const int bn = pick_bn(d);
    if ((rc = make_store_map(&a.sO0, dx, d, T))) return rc;
    if ((rc = make_map_2d(&a.mA, dl_hi, E, T, 64, BM))) return rc;
    if ((rc = make_map_2d(&a.mA1, dl_lo, E, T, 64, BM))) return rc;
    if ((rc = make_map_2d(&a.mB0, wg, E, d, 64, bn))) return rc;
    if ((rc = launch_bn<K_DXR>(a, bn, num_sms, s))) return rc;
  }
  return MOE_OK;
}

int tc_ffn_fwd(const FfnPtrs& p, const void* xg, void* H, void* act, void* Y, int num_sms,
               cudaStream_t s) {
  const int d = p.d, f = p.f, E = p.E, cap = p.cap;
  int rc;
  {  // UP: H = Xg [W1 | W3], A = silu(H1) H3
    TcArgs a = base_args(p);
    a.N = 2 * f;
    a.K = d;
    if ((rc = make_map_2d(&a.mA, xg, d, cap, 64, BM))) return rc;
    if ((rc = make_map_atoms(&a.mB0, p.w1, f, d, E, 256 / 128))) return rc;
    if ((rc = make_map_atoms(&a.mB1, p.w3, f, d, E, 256 / 128))) return rc;
    if ((rc = make_store_map(&a.sO0, H, 2 * f, cap))) return rc;
    if ((rc = make_store_map(&a.sO1, act, f, cap))) return rc;
    if ((rc = launch<K_UP, 256>(a, num_sms, s))) return rc;
  }
  {  // DOWN: Y = A W2
    TcArgs a = base_args(p);
    a.N = d;
    a.K = f;
    const int bn = pick_bn(d);
    if ((rc = make_map_2d(&a.mA, act, f, cap, 64, BM))) return rc;
    if ((rc = make_map_atoms(&a.mB0, p.w2, d, f, E, bn / 64))) return rc;
    if ((rc = make_store_map(&a.sO0, Y, d, cap))) return rc;
    if ((rc = launch_bn<K_DOWN>(a, bn, num_sms, s))) return rc;
  }
  return MOE_OK;
}

// MXFP8 forward: H = Xq [W1q | W3q] (bf16 out), A -> E4M3 blocks along f in
// the epilogue, Y = Aq W2q (bf16 out).  xq/xs: quantised rows; w13q/w13s and
// w2q/w2s: quantised weights (layouts in mx.cu); actq/acts: A's workspace.
int tc_ffn_fwd_mx(const FfnPtrs& p, const uint8_t* xq, const uint8_t* xs, const uint8_t* w13q,
                  const uint8_t* w13s, const uint8_t* w2q, const uint8_t* w2s, void* H,
                  uint8_t* actq, uint8_t* acts, void* Y, int num_sms, cudaStream_t s) {
  const int d = p.d, f = p.f, E = p.E, cap = p.cap;
  int rc;
  {  // UPQ
    TcArgs a = base_args(p);
    a.N = 2 * f;
    a.K = d;
    a.kchunks = d / 128;
    a.sfa = xs;
    a.sfb = w13s;
    a.act_q = actq;
    a.act_s = acts;
    if ((rc = make_map_u8(&a.mA, xq, d, cap, 1, 128, BM))) return rc;
    if ((rc = make_map_u8(&a.mB0, w13q, d, 2 * f, E, 128, 256))) return rc;
    if ((rc = make_store_map(&a.sO0, H, 2 * f, cap))) return rc;
    if ((rc = launch<K_UPQ, 256>(a, num_sms, s))) return rc;
  }
  {  // DOWNQ
    TcArgs a = base_args(p);
    a.N = d;
    a.K = f;
    a.kchunks = f / 128;
    a.sfa = acts;
    a.sfb = w2s;
    if ((rc = make_map_u8(&a.mA, actq, f, cap, 1, 128, BM))) return rc;
    const int bn = pick_bn(d);
    if ((rc = make_map_u8(&a.mB0, w2q, f, d, E, 128, bn))) return rc;
    if ((rc = make_store_map(&a.sO0, Y, d, cap))) return rc;
    if (bn == 256) {
      if ((rc = launch<K_DOWNQ, 256>(a, num_sms, s))) return rc;
    } else if ((rc = launch<K_DOWNQ, 128>(a, num_sms, s))) {
      return rc;
    }
  }
  return MOE_OK;
}

int tc_ffn_bwd(const FfnPtrs& p, const void* dog, const void* xg, const float* row_gate,
               const void* H, void* dH, void* gact, float* ds_part, void* dXp, void* dw1,
               void* dw3, void* dw2, int num_sms, cudaStream_t s, const MxBwd* mx) {
  const int d = p.d, f = p.f, E = p.E, cap = p.cap;
  int rc;
  {  // DAP: dA' = dOg W2^T with the SwiGLU-backward epilogue
    TcArgs a = base_args(p);
    a.N = f;
    a.K = d;
    const int bn = pick_bn(f);
    if ((rc = make_map_2d(&a.mA, dog, d, cap, 64, BM))) return rc;
    if ((rc = make_map_3d(&a.mB0, p.w2, d, f, E, 64, bn))) return rc;
    a.hin = (const __nv_bfloat16*)H;
    a.row_gate = row_gate;
    if ((rc = make_store_map(&a.sO0, dH, 2 * f, cap))) return rc;
    if ((rc = make_store_map(&a.sO1, gact, f, cap))) return rc;
    a.ds_part = ds_part;
    if (mx != nullptr) {
      a.dh_q = mx->dhq;
      a.dh_s = mx->dhs;
      if (mx->wgrad) {   // dH and s*A straight to the rows-quantised operands of the dW GEMMs
        a.dht_q = mx->hq;
        a.dht_s = mx->hs;
        a.gat_q = mx->aq;
        a.gat_s = mx->as;
        a.capr = mx->capr;
      }
    }
    a.nparts = 2 * (f / bn);
    if (a.nparts != tc_num_dS_parts(f)) return fail(MOE_ERR_UNSUPPORTED, "dS partition mismatch");
    if (mx != nullptr) {
      if (mx->wgrad) {
        if ((rc = launch_bn<K_DAPQW>(a, bn, num_sms, s))) return rc;
      } else if ((rc = launch_bn<K_DAPQ>(a, bn, num_sms, s))) {
        return rc;
      }
    } else if ((rc = launch_bn<K_DAP>(a, bn, num_sms, s))) {
      return rc;
    }
  }
  if (mx != nullptr) {  // DXQ: dXp = dHq [W1r | W3r]^T on the block-scaled tensor cores
    TcArgs a = base_args(p);
    a.N = d;
    a.K = 2 * f;
    a.kchunks = (2 * f) / 128;
    a.kh = f / 128;
    a.sfa = mx->dhs;
    a.sfb = mx->w1rs;
    a.sfb1 = mx->w3rs;
    const int bn = pick_bn(d);
    if ((rc = make_map_u8(&a.mA, mx->dhq, 2 * f, cap, 1, 128, BM))) return rc;
    if ((rc = make_map_u8(&a.mB0, mx->w1rq, f, d, E, 128, bn))) return rc;
    if ((rc = make_map_u8(&a.mB1, mx->w3rq, f, d, E, 128, bn))) return rc;
    if ((rc = make_store_map(&a.sO0, dXp, d, cap))) return rc;
    if (bn == 256) {
      if ((rc = launch<K_DXQ, 256>(a, num_sms, s))) return rc;
    } else if ((rc = launch<K_DXQ, 128>(a, num_sms, s))) {
      return rc;
    }
  } else {  // DX: dXp = dH [W1 | W3]^T
    TcArgs a = base_args(p);
    a.N = d;
    a.K = 2 * f;
    const int bn = pick_bn(d);
    if ((rc = make_map_2d(&a.mA, dH, 2 * f, cap, 64, BM))) return rc;
    if ((rc = make_map_3d(&a.mB0, p.w1, f, d, E, 64, bn))) return rc;
    if ((rc = make_map_3d(&a.mB1, p.w3, f, d, E, 64, bn))) return rc;
    if ((rc = make_store_map(&a.sO0, dXp, d, cap))) return rc;
    if ((rc = launch_bn<K_DX>(a, bn, num_sms, s))) return rc;
  }
  if (mx != nullptr && mx->wgrad) {
    // dW2_e = (sA)^T dOg and [dW1 | dW3]_e = Xg^T dH on MXFP8 operands
    // quantised along the rows of each expert's segment
    const int capr = mx->capr;
    if (d % 256 || (2 * f) % 256)
      return fail(MOE_ERR_UNSUPPORTED, "MXFP8 weight gradients need d and 2f multiples of 256");
    if ((rc = launch_mx_quant_cols(mx->x, mx->T, mx->row_token, p.offsets, E, d, capr, mx->xq, mx->xs, s)))
      return rc;
    if ((rc = launch_mx_quant_cols(dog, cap, nullptr, p.offsets, E, d, capr, mx->oq, mx->os, s))) return rc;
    // (dH and s*A: quantised along the rows by the dA' epilogue)
    {
      TcArgs a = base_args(p);
      a.M = f;
      a.N = d;
      a.kchunks = capr / 128;
      a.sfa = mx->as;
      a.sfb = mx->os;
      if ((rc = make_map_u8(&a.mA, mx->aq, capr, f, 1, 128, BM))) return rc;
      if ((rc = make_map_u8(&a.mB0, mx->oq, capr, d, 1, 128, 256))) return rc;
      if ((rc = make_store_map(&a.sO0, dw2, d, (uint64_t)E * f))) return rc;
      if ((rc = launch<K_DW2Q, 256>(a, num_sms, s))) return rc;
    }
    {
      TcArgs a = base_args(p);
      a.M = d;
      a.N = 2 * f;
      a.kchunks = capr / 128;
      a.sfa = mx->xs;
      a.sfb = mx->hs;
      if ((rc = make_map_u8(&a.mA, mx->xq, capr, d, 1, 128, BM))) return rc;
      if ((rc = make_map_u8(&a.mB0, mx->hq, capr, 2 * f, 1, 128, 256))) return rc;
      if ((rc = make_store_map(&a.sO0, dw1, f, (uint64_t)E * d))) return rc;
      if ((rc = make_store_map(&a.sO1, dw3, f, (uint64_t)E * d))) return rc;
      if ((rc = launch<K_DW13Q, 256>(a, num_sms, s))) return rc;
    }
    return MOE_OK;
  }
  {  // DW2: dW2_e = (sA)^T dOg
    TcArgs a = base_args(p);
    a.M = f;
    a.N = d;
    const int bn = pick_bn(d);
    if ((rc = make_map_atoms(&a.mA, gact, f, cap, 1, BM / 64))) return rc;
    if ((rc = make_map_atoms(&a.mB0, dog, d, cap, 1, bn / 64))) return rc;
    if ((rc = make_store_map(&a.sO0, dw2, d, (uint64_t)E * f))) return rc;
    if ((rc = launch_bn<K_DW2>(a, bn, num_sms, s))) return rc;
  }
  {  // DW13: [dW1 | dW3]_e = Xg^T dH
    TcArgs a = base_args(p);
    a.M = d;
    a.N = 2 * f;
    const int bn = pick_bn(2 * f);
    if ((rc = make_map_atoms(&a.mA, xg, d, cap, 1, BM / 64))) return rc;
    if ((rc = make_map_atoms(&a.mB0, dH, 2 * f, cap, 1, bn / 64))) return rc;
    if ((rc = make_store_map(&a.sO0, dw1, f, (uint64_t)E * d))) return rc;
    if ((rc = make_store_map(&a.sO1, dw3, f, (uint64_t)E * d))) return rc;
    if ((rc = launch_bn<K_DW13>(a, bn, num_sms, s))) return rc;
  }
  return MOE_OK;
}

}  // namespace moe
