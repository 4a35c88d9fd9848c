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
// The grouped GEMM replaces the per-expert loop of the Beam article's
// MoELayer (sec. 5.3); Olmo-core 3 names grouped GEMM for the same purpose;
// dS = <dA', A> without a stored Y is the SonicMoE summary's sec. 1.
//
// CTA layout (192 threads, one CTA per SM):
//   warp 0      TMA producer (one lane): A and B tiles into a ring of stages
//   warp 1      TMEM allocator + MMA issuer (one lane): 128 x BN x 16 UMMAs
//   warps 2..5  epilogue: tcgen05.ld of the fp32 accumulator, fused math,
//               16-byte global stores
// The accumulator is double-buffered in TMEM (2 x BN columns) so that the
// epilogue of tile i overlaps the main loop of tile i+1.  Tiles are assigned
// round-robin to the CTAs; the row count R and the per-expert segments are
// read on the device, so no host synchronisation is needed.
#include <dlfcn.h>

#include <cstring>

#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace moe {

using namespace tc;

enum Kind : int { K_UP = 0, K_DOWN = 1, K_DAP = 2, K_DX = 3, K_DW2 = 4, K_DW13 = 5 };

constexpr int BM = 128;
constexpr int BK = 64;                 // 64 bf16 = 128 bytes = one swizzle row
constexpr int ATOM = 8192;             // one 64 x 64 bf16 TMA box
constexpr int A_BYTES = BM * BK * 2;   // 16 KB
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;

struct TcArgs {
  CUtensorMap mA;    // A operand
  CUtensorMap mB0;   // B operand (W1 / W2 / activation)
  CUtensorMap mB1;   // second B source (W3) where the kind has one
  const int32_t* offsets;
  int E, d, f;
  int M, N, K;       // varlen-M: N, K fixed; varlen-K: M, N fixed
  // epilogue operands
  __nv_bfloat16* out0;   // H / Y / dXp / dW2 / dW1
  __nv_bfloat16* out1;   // A (UP) / dH (DAP) / dW3 (DW13)
  __nv_bfloat16* out2;   // s*A (DAP)
  const __nv_bfloat16* hin;  // H (DAP)
  const float* row_gate;     // DAP
  float* ds_part;            // DAP: [cap, nparts]
  int nparts;
  int* status;
};

template <int KIND> struct KT {
  static constexpr bool VARLEN_K = (KIND == K_DW2 || KIND == K_DW13);
  static constexpr bool A_MN = VARLEN_K;
  static constexpr bool B_MN = (KIND == K_UP || KIND == K_DOWN || VARLEN_K);
};

template <int BN> struct Cfg {
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int STAGES = (BN == 256) ? 4 : 6;
  static constexpr int SMEM = STAGES * STAGE + 1024;
  static constexpr int TMEM_COLS = 2 * BN;
};

struct TileInfo {
  int e, m0, n0, kb_count, krow0, ntile;
};

template <int KIND, int BN>
__device__ __forceinline__ bool tile_info(int t, const TcArgs& a, const int* s_off, int total,
                                          TileInfo& ti) {
  if (t >= total) return false;
  const int ntiles = a.N / BN;
  if constexpr (KT<KIND>::VARLEN_K) {
    const int per = (a.M / BM) * ntiles;
    ti.e = t / per;
    const int rem = t - ti.e * per;
    ti.m0 = (rem / ntiles) * BM;
    ti.ntile = rem % ntiles;
    ti.n0 = ti.ntile * BN;
    ti.krow0 = s_off[ti.e];
    ti.kb_count = (s_off[ti.e + 1] - s_off[ti.e]) / BK;
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
    ti.kb_count = a.K / BK;
  }
  return true;
}

__device__ __forceinline__ bool bounded_wait(uint64_t* bar, uint32_t parity, volatile int* s_abort,
                                             int* status, int code) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63) == 0) {
      if (*s_abort) return false;
      if (globaltimer_ns() - t0 > WAIT_LIMIT_NS) {
        *s_abort = 1;
        record_status(status, 0x200 | code);
        return false;
      }
    }
  }
}

__device__ __forceinline__ void st_bf16x32(__nv_bfloat16* dst, const float* v) {
  uint4* p = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 u;
    __nv_bfloat162 h[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[q * 8 + 2 * i], v[q * 8 + 2 * i + 1]);
    memcpy(&u, h, 16);
    p[q] = u;
  }
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

template <int KIND, int BN>
__global__ void __launch_bounds__(192, 1) k_tc_gemm(const __grid_constant__ TcArgs a) {
  using C = Cfg<BN>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[C::STAGES];
  __shared__ __align__(8) uint64_t empty_bar[C::STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ uint32_t s_tmem;
  __shared__ int s_off[257];
  __shared__ volatile int s_abort;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  for (int i = threadIdx.x; i <= a.E; i += blockDim.x) s_off[i] = a.offsets[i];
  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&tfull_bar[s], 1);
      mbar_init(&tempty_bar[s], 128);
    }
    fence_mbar_init();
    prefetch_tmap(&a.mA);
    prefetch_tmap(&a.mB0);
    if (KIND == K_UP || KIND == K_DX) prefetch_tmap(&a.mB1);
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
  if constexpr (KT<KIND>::VARLEN_K) total = a.E * (a.M / BM) * (a.N / BN);
  else total = (s_off[a.E] / BM) * (a.N / BN);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      TileInfo ti;
      for (int t = blockIdx.x; tile_info<KIND, BN>(t, a, s_off, total, ti); t += gridDim.x) {
        for (int kb = 0; kb < ti.kb_count; ++kb) {
          if (!bounded_wait(&empty_bar[stage], phase ^ 1, &s_abort, a.status, 1)) goto producer_done;
          uint8_t* sA = smem + stage * C::STAGE;
          uint8_t* sB = sA + A_BYTES;
          mbar_arrive_expect_tx(&full_bar[stage], C::STAGE);
          const int k0 = kb * BK;
          if constexpr (KIND == K_UP) {
            tma_load_2d(sA, &a.mA, &full_bar[stage], k0, ti.m0);
            const int nf = ti.ntile * (BN / 2);
#pragma unroll
            for (int h = 0; h < BN / 128; ++h) {
              tma_load_3d(sB + h * ATOM, &a.mB0, &full_bar[stage], nf + 64 * h, k0, ti.e);
              tma_load_3d(sB + (BN / 128 + h) * ATOM, &a.mB1, &full_bar[stage], nf + 64 * h, k0, ti.e);
            }
          } else if constexpr (KIND == K_DOWN) {
            tma_load_2d(sA, &a.mA, &full_bar[stage], k0, ti.m0);
#pragma unroll
            for (int h = 0; h < BN / 64; ++h)
              tma_load_3d(sB + h * ATOM, &a.mB0, &full_bar[stage], ti.n0 + 64 * h, k0, ti.e);
          } else if constexpr (KIND == K_DAP) {
            tma_load_2d(sA, &a.mA, &full_bar[stage], k0, ti.m0);
            tma_load_3d(sB, &a.mB0, &full_bar[stage], k0, ti.n0, ti.e);
          } else if constexpr (KIND == K_DX) {
            tma_load_2d(sA, &a.mA, &full_bar[stage], k0, ti.m0);
            if (k0 < a.f) tma_load_3d(sB, &a.mB0, &full_bar[stage], k0, ti.n0, ti.e);
            else tma_load_3d(sB, &a.mB1, &full_bar[stage], k0 - a.f, ti.n0, ti.e);
          } else {  // varlen-K: A and B are row-space activations, MN-major
            const int r = ti.krow0 + k0;
            tma_load_2d(sA, &a.mA, &full_bar[stage], ti.m0, r);
            tma_load_2d(sA + ATOM, &a.mA, &full_bar[stage], ti.m0 + 64, r);
#pragma unroll
            for (int h = 0; h < BN / 64; ++h)
              tma_load_2d(sB + h * ATOM, &a.mB0, &full_bar[stage], ti.n0 + 64 * h, r);
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
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!bounded_wait(&tempty_bar[acc], acc_phase ^ 1, &s_abort, a.status, 2)) break;
        fence_after_sync();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < ti.kb_count; ++kb) {
          if (!bounded_wait(&full_bar[stage], phase, &s_abort, a.status, 3)) goto mma_done;
          fence_after_sync();
          const uint32_t sA = smem_u32(smem + stage * C::STAGE);
          const uint32_t sB = sA + A_BYTES;
#pragma unroll
          for (int ks = 0; ks < BK / 16; ++ks) {
            const uint64_t ad = KT<KIND>::A_MN ? sdesc_sw128(sA + ks * 2048, ATOM, 1024)
                                               : sdesc_sw128(sA + ks * 32, 16, 1024);
            const uint64_t bd = KT<KIND>::B_MN ? sdesc_sw128(sB + ks * 2048, ATOM, 1024)
                                               : sdesc_sw128(sB + ks * 32, 16, 1024);
            umma_bf16(d_tmem, ad, bd, IDESC, (kb | ks) != 0);
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
    const int rloc = q * 32 + lane;              // row of the tile owned by this thread
    int it = 0;
    TileInfo ti;
    for (int t = blockIdx.x; tile_info<KIND, BN>(t, a, s_off, total, ti); t += gridDim.x, ++it) {
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      if (!bounded_wait(&tfull_bar[acc], acc_phase, &s_abort, a.status, 4)) break;
      fence_after_sync();
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN;
      const int row = ti.m0 + rloc;
      float v[32];
      uint32_t r[32];
      if constexpr (KIND == K_UP) {
        const int f = a.f, nf = ti.ntile * (BN / 2);
        float h3[32];
        for (int c = 0; c < BN / 2; c += 32) {
          tmem_ld32(tbase + c, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
          tmem_ld32(tbase + BN / 2 + c, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) h3[i] = __uint_as_float(r[i]);
          __nv_bfloat16* hrow = a.out0 + (size_t)row * 2 * f;
          st_bf16x32(hrow + nf + c, v);
          st_bf16x32(hrow + f + nf + c, h3);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = silu_f(bf16_round(v[i])) * bf16_round(h3[i]);
          st_bf16x32(a.out1 + (size_t)row * f + nf + c, v);
        }
      } else if constexpr (KIND == K_DOWN || KIND == K_DX) {
        for (int c = 0; c < BN; c += 32) {
          tmem_ld32(tbase + c, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
          st_bf16x32(a.out0 + (size_t)row * a.N + ti.n0 + c, v);
        }
      } else if constexpr (KIND == K_DAP) {
        const int f = a.f;
        const float g = a.row_gate[row];
        float ds = 0.f;
        float h1[32], h3[32];
        for (int c = 0; c < BN; c += 32) {
          tmem_ld32(tbase + c, r);
          const __nv_bfloat16* hrow = a.hin + (size_t)row * 2 * f;
          ld_bf16x32(hrow + ti.n0 + c, h1);
          ld_bf16x32(hrow + f + ti.n0 + c, h3);
          tmem_ld_wait();
          float da3[32], ga[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float dap = __uint_as_float(r[i]);
            const float sg = sigmoid_f(h1[i]);
            const float sl = h1[i] * sg;
            const float av = bf16_round(sl * h3[i]);
            ds = fmaf(dap, av, ds);
            const float da = g * dap;
            v[i] = da * h3[i] * (sg * (1.0f + h1[i] * (1.0f - sg)));
            da3[i] = da * sl;
            ga[i] = g * av;
          }
          __nv_bfloat16* drow = a.out1 + (size_t)row * 2 * f;
          st_bf16x32(drow + ti.n0 + c, v);
          st_bf16x32(drow + f + ti.n0 + c, da3);
          st_bf16x32(a.out2 + (size_t)row * f + ti.n0 + c, ga);
        }
        a.ds_part[(size_t)row * a.nparts + ti.ntile] = ds;
      } else {  // DW2 / DW13: output row m = row of dW_e
        const size_t ebase = (size_t)ti.e * a.M * (KIND == K_DW2 ? a.N : a.f);
        for (int c = 0; c < BN; c += 32) {
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
            st_bf16x32(a.out0 + ebase + (size_t)row * a.N + col, v);
          } else {
            if (col < a.f) st_bf16x32(a.out0 + ebase + (size_t)row * a.f + col, v);
            else st_bf16x32(a.out1 + ebase + (size_t)row * a.f + col - a.f, v);
          }
        }
      }
      fence_before_sync();
      mbar_arrive(&tempty_bar[acc]);
    }
  }

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

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* h = dlopen("libcuda.so.1", RTLD_NOW | RTLD_GLOBAL);
    if (h) fn = reinterpret_cast<EncodeTiledFn>(dlsym(h, "cuTensorMapEncodeTiled"));
  }
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

int tc_num_dS_parts(int f) { return (f % 256 == 0) ? f / 256 : f / 128; }

// bf16 row-major [outer, inner] viewed in boxes of box_outer x box_inner.
static int make_map_2d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer,
                       uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled (2d) failed: " + std::to_string((int)r));
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
static int launch(const TcArgs& a, int grid, cudaStream_t s) {
  using C = Cfg<BN>;
  cudaError_t e = cudaFuncSetAttribute(k_tc_gemm<KIND, BN>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return cuda_fail(e, "tc gemm smem attribute");
  static const char* kNames[6] = {"tc_up", "tc_down", "tc_dap", "tc_dx", "tc_dw2", "tc_dw13"};
  {
    ProfScope _ps(kNames[KIND], s);
    k_tc_gemm<KIND, BN><<<grid, 192, C::SMEM, s>>>(a);
  }
  MOE_CHECK_LAUNCH("tc_gemm");
  return MOE_OK;
}

template <int KIND>
static int launch_bn(const TcArgs& a, int bn, int grid, cudaStream_t s) {
  if (bn == 256) return launch<KIND, 256>(a, grid, s);
  return launch<KIND, 128>(a, grid, s);
}

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

int tc_ffn_fwd(const FfnPtrs& p, const void* xg, void* H, void* act, void* Y, int num_sms,
               cudaStream_t s) {
  const int d = p.d, f = p.f, E = p.E, cap = p.cap;
  int rc;
  {  // UP: H = Xg [W1 | W3], A = silu(H1) H3
    TcArgs a = base_args(p);
    a.N = 2 * f;
    a.K = d;
    if ((rc = make_map_2d(&a.mA, xg, d, cap, 64, BM))) return rc;
    if ((rc = make_map_3d(&a.mB0, p.w1, f, d, E, 64, 64))) return rc;
    if ((rc = make_map_3d(&a.mB1, p.w3, f, d, E, 64, 64))) return rc;
    a.out0 = (__nv_bfloat16*)H;
    a.out1 = (__nv_bfloat16*)act;
    if ((rc = launch<K_UP, 256>(a, num_sms, s))) return rc;
  }
  {  // DOWN: Y = A W2
    TcArgs a = base_args(p);
    a.N = d;
    a.K = f;
    const int bn = pick_bn(d);
    if ((rc = make_map_2d(&a.mA, act, f, cap, 64, BM))) return rc;
    if ((rc = make_map_3d(&a.mB0, p.w2, d, f, E, 64, 64))) return rc;
    a.out0 = (__nv_bfloat16*)Y;
    if ((rc = launch_bn<K_DOWN>(a, bn, num_sms, s))) return rc;
  }
  return MOE_OK;
}

int tc_ffn_bwd(const FfnPtrs& p, const void* dog, const void* xg, const float* row_gate,
               const void* H, void* dH, void* gact, float* ds_part, void* dXp, void* dw1,
               void* dw3, void* dw2, int num_sms, cudaStream_t s) {
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
    a.out1 = (__nv_bfloat16*)dH;
    a.out2 = (__nv_bfloat16*)gact;
    a.ds_part = ds_part;
    a.nparts = f / bn;
    if (a.nparts != tc_num_dS_parts(f)) return fail(MOE_ERR_UNSUPPORTED, "dS partition mismatch");
    if ((rc = launch_bn<K_DAP>(a, bn, num_sms, s))) return rc;
  }
  {  // DX: dXp = dH [W1 | W3]^T
    TcArgs a = base_args(p);
    a.N = d;
    a.K = 2 * f;
    const int bn = pick_bn(d);
    if ((rc = make_map_2d(&a.mA, dH, 2 * f, cap, 64, BM))) return rc;
    if ((rc = make_map_3d(&a.mB0, p.w1, f, d, E, 64, bn))) return rc;
    if ((rc = make_map_3d(&a.mB1, p.w3, f, d, E, 64, bn))) return rc;
    a.out0 = (__nv_bfloat16*)dXp;
    if ((rc = launch_bn<K_DX>(a, bn, num_sms, s))) return rc;
  }
  {  // DW2: dW2_e = (sA)^T dOg
    TcArgs a = base_args(p);
    a.M = f;
    a.N = d;
    const int bn = pick_bn(d);
    if ((rc = make_map_2d(&a.mA, gact, f, cap, 64, 64))) return rc;
    if ((rc = make_map_2d(&a.mB0, dog, d, cap, 64, 64))) return rc;
    a.out0 = (__nv_bfloat16*)dw2;
    if ((rc = launch_bn<K_DW2>(a, bn, num_sms, s))) return rc;
  }
  {  // DW13: [dW1 | dW3]_e = Xg^T dH
    TcArgs a = base_args(p);
    a.M = d;
    a.N = 2 * f;
    const int bn = pick_bn(2 * f);
    if ((rc = make_map_2d(&a.mA, xg, d, cap, 64, 64))) return rc;
    if ((rc = make_map_2d(&a.mB0, dH, 2 * f, cap, 64, 64))) return rc;
    a.out0 = (__nv_bfloat16*)dw1;
    a.out1 = (__nv_bfloat16*)dw3;
    if ((rc = launch_bn<K_DW13>(a, bn, num_sms, s))) return rc;
  }
  return MOE_OK;
}

}  // namespace moe
