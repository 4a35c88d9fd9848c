// Router top-k/softmax and the expert permutation (exact and token-rounded).
//
// Top-k then softmax over the k logits: Beam article sec. 5.3 / Trinity Large
// commentary example 1.  Histogram + prefix sum + stable scatter into
// expert-contiguous rows: Trinity example 2-3, Olmo-core 3 ("row-wise EP puts
// data straight into expert input buffers", routing kept on the GPU).
// Token rounding: SonicMoE summary sec. 3.
#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace moe {

// ============================================================== top-k + softmax
// One warp per token.  Each lane holds up to 8 of the E <= 256 logits
// (expert e = lane + 32*i).  k rounds of a warp arg-max (ties: lowest id).
__global__ void k_topk_softmax(const float* __restrict__ logits_in, const float* __restrict__ bias,
                               const float* __restrict__ noise, float* __restrict__ logits_out,
                               int T, int E, int k, int gate_mode, int32_t* __restrict__ idx,
                               float* __restrict__ gate) {
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  for (int t = blockIdx.x * warps + (threadIdx.x >> 5); t < T; t += gridDim.x * warps) {
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      int e = lane + 32 * i;
      float l = -INFINITY;
      if (e < E) {
        l = logits_in[(size_t)t * E + e];
        if (bias) l += bias[e];
        if (noise) l += noise[(size_t)t * E + e];
        if (logits_out != logits_in || bias || noise) logits_out[(size_t)t * E + e] = l;
      }
      v[i] = l;
    }
    unsigned taken = 0;  // bit i: my element i already selected
    float top[8];
    int topi[8];
    for (int j = 0; j < k; ++j) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        int e = lane + 32 * i;
        if (e < E && !(taken >> i & 1u)) {
          if (v[i] > bv || (v[i] == bv && e < bi)) { bv = v[i]; bi = e; }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
      }
      if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
      top[j] = bv;
      topi[j] = bi;
    }
    // gate_mode 1: normaliser over all E logits (max = top[0])
    float zall = 0.f;
    if (gate_mode == 1) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (lane + 32 * i < E) zall += expf(v[i] - top[0]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) zall += __shfl_xor_sync(0xffffffffu, zall, o);
    }
    if (lane == 0) {
      float m = top[0], z = 0.f;
      float ex[8];
      for (int j = 0; j < k; ++j) { ex[j] = expf(top[j] - m); z += ex[j]; }
      float inv = 1.0f / (gate_mode == 1 ? zall : z);
      for (int j = 0; j < k; ++j) {
        idx[(size_t)t * k + j] = topi[j];
        gate[(size_t)t * k + j] = ex[j] * inv;
      }
    }
  }
}

int launch_topk_softmax(const float* logits_in, const float* bias, const float* noise,
                        float* logits_out, int T, int E, int k, int gate_mode, int32_t* idx,
                        float* gate, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  int blocks = (T + 7) / 8;
  if (blocks > 148 * 16) blocks = 148 * 16;
  {
    ProfScope _ps("topk_softmax", s);
    k_topk_softmax<<<blocks, 256, 0, s>>>(logits_in, bias, noise, logits_out, T, E, k, gate_mode,
                                          idx, gate);
  }
  MOE_CHECK_LAUNCH("topk_softmax");
  return MOE_OK;
}

// ============================================================== exact permutation
// Block b owns tokens [256 b, 256 b + 256); warp w of it owns 32 of them.
// bits[w][e] has bit `lane` set when token (w, lane) chose expert e, so the
// rank of a token among the block's tokens of expert e (ascending token id)
// is sum over earlier warps of popc(bits[w'][e]) + popc(bits[w][e] & lanes below).
constexpr int PERM_TOK = 256;

__device__ __forceinline__ void build_bits(const int32_t* __restrict__ idx, int T, int E, int k,
                                           uint32_t* bits, int* status) {
  for (int i = threadIdx.x; i < 8 * E; i += blockDim.x) bits[i] = 0;
  __syncthreads();
  const int t = blockIdx.x * PERM_TOK + threadIdx.x;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (t < T) {
    for (int j = 0; j < k; ++j) {
      int e = idx[(size_t)t * k + j];
      if (e >= 0 && e < E) atomicOr(&bits[w * E + e], 1u << lane);
      else record_status(status, 0x120);  // invalid expert id: flag it, skip the slot
    }
  }
  __syncthreads();
}

__global__ void k_perm_count(const int32_t* __restrict__ idx, int T, int E, int k,
                             int32_t* __restrict__ blockcnt, int* status) {
  extern __shared__ uint32_t sm[];
  uint32_t* bits = sm;
  build_bits(idx, T, E, k, bits, status);
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) c += __popc(bits[w * E + e]);
    blockcnt[(size_t)blockIdx.x * E + e] = c;
  }
}

// Single block: per-expert running sums over blocks, padded exclusive scan
// over experts, padding rows.  With few experts warp w scans the block
// counts of experts w, w + 32, ... (lanes over blocks, shuffle scans); with
// many, a thread per expert walks the blocks (reads coalesced over experts).
// Warp 0 then scans the tile-padded totals over experts.
__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

__global__ void __launch_bounds__(512)
k_perm_scan(const int32_t* __restrict__ blockcnt, int nb, int E, int tile,
            int32_t* __restrict__ blockbase, int32_t* __restrict__ counts,
            int32_t* __restrict__ offsets, int32_t* __restrict__ row_token,
            float* __restrict__ row_gate, int32_t* __restrict__ row_slot) {
  __shared__ int s_cnt[256];
  __shared__ int s_off[257];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  // blockbase = running count within the expert (the segment offset is added below)
  if (E <= 16) {   // few experts: lanes over blocks, shuffle scans
    for (int e = warp; e < E; e += nw) {
      int base = 0;
      for (int b0 = 0; b0 < nb; b0 += 32) {
        const int b = b0 + lane;
        const int c = b < nb ? blockcnt[(size_t)b * E + e] : 0;
        const int incl = warp_incl_scan(c, lane);
        if (b < nb) blockbase[(size_t)b * E + e] = base + incl - c;
        base += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) {
        s_cnt[e] = base;
        counts[e] = base;
      }
    }
  } else {         // many experts: a thread per expert, coalesced over experts
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      int run = 0, b = 0;
      for (; b + 8 <= nb; b += 8) {
        int c[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) c[j] = blockcnt[(size_t)(b + j) * E + e];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          blockbase[(size_t)(b + j) * E + e] = run;
          run += c[j];
        }
      }
      for (; b < nb; ++b) {
        const int c = blockcnt[(size_t)b * E + e];
        blockbase[(size_t)b * E + e] = run;
        run += c;
      }
      s_cnt[e] = run;
      counts[e] = run;
    }
  }
  __syncthreads();
  if (warp == 0) {
    int run = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      const int p = e < E ? (s_cnt[e] + tile - 1) / tile * tile : 0;
      const int incl = warp_incl_scan(p, lane);
      if (e < E) s_off[e] = run + incl - p;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) s_off[E] = run;
  }
  __syncthreads();
  for (int e = threadIdx.x; e <= E; e += blockDim.x) offsets[e] = s_off[e];
  if (E <= 16) {
    for (int e = warp; e < E; e += nw) {
      const int o = s_off[e];
      for (int b = lane; b < nb; b += 32) blockbase[(size_t)b * E + e] += o;
    }
  } else {
    for (int i = threadIdx.x; i < nb * E; i += blockDim.x) blockbase[i] += s_off[i % E];
  }
  // padding rows of every segment (fewer than `tile` per expert): a warp per expert
  for (int e = warp; e < E; e += nw) {
    const int lo = s_off[e] + s_cnt[e], hi = s_off[e + 1];
    for (int r = lo + lane; r < hi; r += 32) {
      row_token[r] = -1;
      row_gate[r] = 0.f;
      row_slot[r] = -1;
    }
  }
}

__global__ void k_perm_scatter(const int32_t* __restrict__ idx, const float* __restrict__ gate,
                               int T, int E, int k, const int32_t* __restrict__ blockbase,
                               int32_t* __restrict__ row_token, float* __restrict__ row_gate,
                               int32_t* __restrict__ row_slot, int32_t* __restrict__ slot_row,
                               int* status) {
  extern __shared__ uint32_t sm[];
  uint32_t* bits = sm;
  int* wpre = reinterpret_cast<int*>(sm + 8 * E);
  build_bits(idx, T, E, k, bits, status);
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = blockbase[(size_t)blockIdx.x * E + e];
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      wpre[w * E + e] = run;
      run += __popc(bits[w * E + e]);
    }
  }
  __syncthreads();
  const int t = blockIdx.x * PERM_TOK + threadIdx.x;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (t >= T) return;
  const uint32_t below = (1u << lane) - 1u;
  for (int j = 0; j < k; ++j) {
    const int s = t * k + j;
    int e = idx[s];
    if (e < 0 || e >= E) { slot_row[s] = -1; continue; }
    int row = wpre[w * E + e] + __popc(bits[w * E + e] & below);
    row_token[row] = t;
    row_gate[row] = gate[s];
    row_slot[row] = s;
    slot_row[s] = row;
  }
}

static int perm_blocks(int T) { return (T + PERM_TOK - 1) / PERM_TOK; }

size_t permute_ws_bytes(int T, int E, int k, int round_mode, int tile) {
  Sizer z;
  int nb = perm_blocks(T) > 0 ? perm_blocks(T) : 1;
  z.take<int32_t>((size_t)nb * E);
  z.take<int32_t>((size_t)nb * E);
  if (round_mode) {
    size_t cap = (size_t)T * k + (size_t)E * tile;
    z.take<int32_t>(E);
    z.take<int32_t>(E + 1);
    z.take<int32_t>(cap);
    z.take<float>(cap);
    z.take<int32_t>(cap);
    z.take<double>(T > 0 ? T : 1);
  }
  return z.used;
}

int carve_permute_ws(void* ws, size_t bytes, int T, int E, int k, int round_mode, int tile,
                     PermuteWs* o) {
  Carve c(ws, bytes);
  int nb = perm_blocks(T) > 0 ? perm_blocks(T) : 1;
  *o = PermuteWs{};
  o->blockcnt = c.take<int32_t>((size_t)nb * E);
  o->blockbase = c.take<int32_t>((size_t)nb * E);
  if (round_mode) {
    size_t cap = (size_t)T * k + (size_t)E * tile;
    o->ex_counts = c.take<int32_t>(E);
    o->ex_offsets = c.take<int32_t>(E + 1);
    o->ex_row_token = c.take<int32_t>(cap);
    o->ex_row_gate = c.take<float>(cap);
    o->ex_row_slot = c.take<int32_t>(cap);
    o->lse = c.take<double>(T > 0 ? T : 1);
  }
  if (!c.ok) return fail(MOE_ERR_WORKSPACE, "permute workspace too small");
  return MOE_OK;
}

int launch_permute_exact(const int32_t* idx, const float* gate, int T, int E, int k, int tile,
                         int32_t* counts, int32_t* offsets, int32_t* row_token, float* row_gate,
                         int32_t* row_slot, int32_t* slot_row, const PermuteWs& w,
                         cudaStream_t s) {
  const int nb = perm_blocks(T);
  const size_t smem_count = (size_t)8 * E * sizeof(uint32_t);
  if (nb > 0) {
    {
      ProfScope _ps("perm_count", s);
      k_perm_count<<<nb, PERM_TOK, smem_count, s>>>(idx, T, E, k, w.blockcnt, status_ptr());
    }
    MOE_CHECK_LAUNCH("perm_count");
  }
  {
    ProfScope _ps("perm_scan", s);
    k_perm_scan<<<1, 512, 0, s>>>(w.blockcnt, nb, E, tile, w.blockbase, counts, offsets,
                                   row_token, row_gate, row_slot);
  }
  MOE_CHECK_LAUNCH("perm_scan");
  if (nb > 0) {
    {
      ProfScope _ps("perm_scatter", s);
      k_perm_scatter<<<nb, PERM_TOK, 2 * smem_count, s>>>(idx, gate, T, E, k, w.blockbase,
                                                          row_token, row_gate, row_slot, slot_row,
                                                          status_ptr());
    }
    MOE_CHECK_LAUNCH("perm_scatter");
  }
  return MOE_OK;
}

// ============================================================== token rounding
// Log-sum-exp of each token's top-k logits, in fp64 so that the ranking key
// l_te - LSE_t orders pairs the same way on any correctly rounding host.
// gate_mode 0: over the token's top-k logits; gate_mode 1: over all E logits.
__global__ void k_round_lse(const float* __restrict__ logits, const int32_t* __restrict__ idx,
                            int T, int E, int k, int gate_mode, double* __restrict__ lse) {
  int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  const int n = gate_mode == 1 ? E : k;
  auto lg = [&](int j) -> double {
    return (double)logits[(size_t)t * E + (gate_mode == 1 ? j : idx[(size_t)t * k + j])];
  };
  double m = -INFINITY;
  for (int j = 0; j < n; ++j) m = fmax(m, lg(j));
  double z = 0.0;
  for (int j = 0; j < n; ++j) z += exp(lg(j) - m);
  lse[t] = m + log(z);
}

__device__ __forceinline__ uint64_t order_key(double v) {
  if (v == 0.0) v = 0.0;  // fold -0 into +0
  uint64_t u = (uint64_t)__double_as_longlong(v);
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

constexpr int RS_THREADS = 1024;

// Block-wide exclusive scan of one int per thread (1024 threads).
__device__ __forceinline__ int block_excl_scan(int v, int* s_warp, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[w] = x;
  __syncthreads();
  if (w == 0) {
    int y = s_warp[lane];
    int z = y;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int q = __shfl_up_sync(0xffffffffu, z, o);
      if (lane >= o) z += q;
    }
    s_warp[lane] = z - y;  // exclusive prefix of warp totals
    if (lane == 31) s_warp[32] = z;
  }
  __syncthreads();
  int r = s_warp[w] + x - v;
  *total = s_warp[32];
  __syncthreads();
  return r;
}

// One block per expert.  Chooses the final members of expert e's segment and
// writes the final rows.  `cand` is either the assigned tokens (drop case,
// candidates = rows of the exact segment) or the unassigned ones (add case).
__global__ void __launch_bounds__(RS_THREADS)
k_round_select(const float* __restrict__ logits, const double* __restrict__ lse,
               const int32_t* __restrict__ ex_counts, const int32_t* __restrict__ ex_offsets,
               const int32_t* __restrict__ ex_row_token, const float* __restrict__ ex_row_gate,
               const int32_t* __restrict__ ex_row_slot, int T, int E, int tile, int capacity,
               int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
               int32_t* __restrict__ row_token, float* __restrict__ row_gate,
               int32_t* __restrict__ row_slot, int32_t* __restrict__ slot_row,
               int32_t* __restrict__ extra_row, int key_cache) {
  // dynamic shared memory: membership bitmap of the assigned tokens (T bits),
  // then, when key_cache != 0, every candidate's 64-bit key (computed once
  // instead of once per radix pass)
  extern __shared__ uint32_t bm[];
  __shared__ int s_off[257];
  __shared__ int s_hist[256];
  __shared__ int s_warp[33];
  __shared__ int s_sel, s_rem, s_r;
  const int e = blockIdx.x;
  if (threadIdx.x == 0) {
    // target rows per expert: nearest multiple of the tile (capacity < 0), or
    // at most `capacity` (capacity factor); segments start at tile multiples
    int acc = 0;
    const int cap_rows = tile * (T / tile);
    for (int i = 0; i < E; ++i) {
      s_off[i] = acc;
      const int c = ex_counts[i];
      int r;
      if (capacity < 0) {
        r = tile * ((c + tile / 2) / tile);
        r = r < cap_rows ? r : cap_rows;
      } else {
        r = c < capacity ? c : capacity;
      }
      if (i == e) s_r = r;
      acc += (r + tile - 1) / tile * tile;
    }
    s_off[E] = acc;
  }
  __syncthreads();
  if (e == 0) {
    for (int i = threadIdx.x; i <= E; i += blockDim.x) offsets[i] = s_off[i];
    for (int i = threadIdx.x; i < E; i += blockDim.x) counts[i] = ex_counts[i];
  }
  const int c = ex_counts[e];
  const int r = s_r;
  const int in0 = ex_offsets[e];
  const int out0 = s_off[e];
  // padding rows after the r members (capacity mode; none with rounding)
  for (int i = out0 + r + threadIdx.x; i < s_off[e + 1]; i += blockDim.x) {
    row_token[i] = -1;
    row_gate[i] = 0.f;
    row_slot[i] = -1;
  }

  if (r == c) {  // nothing to drop or add: copy the segment
    for (int i = threadIdx.x; i < c; i += blockDim.x) {
      int s = ex_row_slot[in0 + i];
      row_token[out0 + i] = ex_row_token[in0 + i];
      row_gate[out0 + i] = ex_row_gate[in0 + i];
      row_slot[out0 + i] = s;
      slot_row[s] = out0 + i;
    }
    return;
  }
  const bool drop = r < c;
  const int m = drop ? r : r - c;  // how many candidates to select (largest first)
  const int ncand = drop ? c : T;
  const int nwords = (T + 31) / 32;
  if (!drop) {
    for (int i = threadIdx.x; i < nwords; i += blockDim.x) bm[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < c; i += blockDim.x) {
      int t = ex_row_token[in0 + i];
      atomicOr(&bm[t >> 5], 1u << (t & 31));
    }
    __syncthreads();
  }
  auto cand_token = [&](int i) -> int { return drop ? ex_row_token[in0 + i] : i; };
  auto is_cand = [&](int i) -> bool { return drop || !((bm[i >> 5] >> (i & 31)) & 1u); };
  auto cand_key = [&](int t) -> uint64_t {
    return order_key((double)logits[(size_t)t * E + e] - lse[t]);
  };
  uint64_t* kc = key_cache ? reinterpret_cast<uint64_t*>(bm + ((nwords + 1) & ~1)) : nullptr;
  if (kc != nullptr && m > 0) {
    for (int i = threadIdx.x; i < ncand; i += blockDim.x)
      kc[i] = is_cand(i) ? cand_key(cand_token(i)) : 0;
    __syncthreads();
  }
  auto key_of = [&](int i) -> uint64_t { return kc ? kc[i] : cand_key(cand_token(i)); };

  // radix select of the m-th largest key among the candidates
  uint64_t prefix = 0, pmask = 0;
  int rem = m;
  if (m > 0) {
    for (int shift = 56; shift >= 0; shift -= 8) {
      for (int i = threadIdx.x; i < 256; i += blockDim.x) s_hist[i] = 0;
      __syncthreads();
      // histogram of the current digit: keys share few digits in the high
      // passes, so lanes with equal digits add once per warp
      for (int i0 = 0; i0 < ncand; i0 += blockDim.x) {
        const int i = i0 + threadIdx.x;
        int bin = -1;
        if (i < ncand && is_cand(i)) {
          const uint64_t u = key_of(i);
          if ((u & pmask) == prefix) bin = (int)((u >> shift) & 255);
        }
        const unsigned grp = __match_any_sync(0xffffffffu, bin);
        if (bin >= 0 && (int)(threadIdx.x & 31) == __ffs(grp) - 1)
          atomicAdd(&s_hist[bin], __popc(grp));
      }
      __syncthreads();
      // digit of the rem-th largest key: lane l holds digits 255-8l .. 248-8l
      if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        int loc[8], sum = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) { loc[j] = s_hist[255 - (8 * lane + j)]; sum += loc[j]; }
        int inc = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, inc, o);
          if (lane >= o) inc += y;
        }
        int cum = inc - sum;   // keys with a larger digit than this lane's range
        if (cum < rem && inc >= rem) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (cum + loc[j] >= rem) {
              s_sel = 255 - (8 * lane + j);
              s_rem = rem - cum;
              break;
            }
            cum += loc[j];
          }
        }
      }
      __syncthreads();
      prefix |= (uint64_t)s_sel << shift;
      pmask |= (uint64_t)255 << shift;
      rem = s_rem;
      __syncthreads();
    }
  }
  const uint64_t thr = prefix;  // value of the m-th largest key
  const int need_eq = rem;      // how many keys equal to thr are selected

  // ordered pass: ties broken by ascending position (= ascending token id)
  int eq_base = 0, out_base = 0, asg_base = 0;
  for (int i0 = 0; i0 < ncand; i0 += blockDim.x) {
    const int i = i0 + threadIdx.x;
    int t = -1, assigned = 0, cand = 0, eq = 0, gt = 0;
    uint64_t u = 0;
    if (i < ncand) {
      t = cand_token(i);
      cand = is_cand(i);
      assigned = drop ? 1 : !cand;
      if (cand && m > 0) {
        u = key_of(i);
        eq = (u == thr);
        gt = (u > thr);
      }
    }
    int tot;
    const int eq_rank = eq_base + block_excl_scan(eq, s_warp, &tot);
    eq_base += tot;
    const int selected = cand && m > 0 && (gt || (eq && eq_rank < need_eq));
    // drop case: members are the selected (kept) candidates;
    // add case: members are the assigned tokens plus the selected ones
    const int member = drop ? selected : (assigned || selected);
    const int pos = out_base + block_excl_scan(member, s_warp, &tot);
    out_base += tot;
    const int asg_rank = asg_base + block_excl_scan(assigned, s_warp, &tot);
    asg_base += tot;
    if (i < ncand) {
      const int row = out0 + pos;
      if (assigned) {
        const int src = drop ? in0 + i : in0 + asg_rank;
        const int s = ex_row_slot[src];
        if (member) {
          row_token[row] = t;
          row_gate[row] = ex_row_gate[src];
          row_slot[row] = s;
          slot_row[s] = row;
        } else {
          slot_row[s] = -1;
        }
      } else if (member) {
        row_token[row] = t;
        row_gate[row] = (float)exp((double)logits[(size_t)t * E + e] - lse[t]);
        row_slot[row] = -1;
        extra_row[(size_t)t * E + e] = row;
      }
    }
  }
}

int launch_permute_round(const int32_t* idx, const float* gate, const float* logits, int T, int E,
                         int k, int tile, int gate_mode, int capacity, int32_t* counts,
                         int32_t* offsets, int32_t* row_token, float* row_gate, int32_t* row_slot,
                         int32_t* slot_row, int32_t* extra_row, const PermuteWs& w,
                         cudaStream_t s) {
  // 1. exact plan into the workspace (its slot_row is scratch: the final
  //    slot_row is fully rewritten by the selection below)
  int rc = launch_permute_exact(idx, gate, T, E, k, tile, w.ex_counts, w.ex_offsets,
                                w.ex_row_token, w.ex_row_gate, w.ex_row_slot, slot_row, w, s);
  if (rc) return rc;
  if (T > 0) {
    {
      ProfScope _ps("round_lse", s);
      k_round_lse<<<(T + 255) / 256, 256, 0, s>>>(logits, idx, T, E, k, gate_mode, w.lse);
    }
    MOE_CHECK_LAUNCH("round_lse");
    if (extra_row != nullptr) {
      cudaError_t e = cudaMemsetAsync(extra_row, 0xff, (size_t)T * E * sizeof(int32_t), s);
      if (e != cudaSuccess) return cuda_fail(e, "memset extra_row");
    }
  }
  size_t smem = (size_t)((T + 31) / 32 + 1) * sizeof(uint32_t);
  if (smem > 200 * 1024) return fail(MOE_ERR_UNSUPPORTED, "token rounding supports T <= 1.6M");
  // candidate keys in shared memory when all T of them fit next to the bitmap
  const size_t words = (size_t)(((T + 31) / 32 + 1) & ~1);
  const size_t with_keys = words * sizeof(uint32_t) + (size_t)T * sizeof(uint64_t);
  const int key_cache = with_keys <= 200 * 1024 ? 1 : 0;
  if (key_cache) smem = with_keys;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k_round_select, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "round_select smem attribute");
  }
  {
    ProfScope _ps("round_select", s);
    k_round_select<<<E, RS_THREADS, smem, s>>>(logits, w.lse, w.ex_counts, w.ex_offsets,
                                               w.ex_row_token, w.ex_row_gate, w.ex_row_slot, T, E,
                                               tile, capacity, counts, offsets, row_token, row_gate,
                                               row_slot, slot_row, extra_row, key_cache);
  }
  MOE_CHECK_LAUNCH("round_select");
  return MOE_OK;
}

}  // namespace moe

// ============================================================== allocation-free permute
// Some callers cannot allocate device memory at call time: plugin hosts that
// hand a kernel only its input and output buffers and own every allocation,
// and step loops that must not call cudaMalloc between launches (it can
// synchronise the whole device).  moe_permute_noalloc serves them: the exact
// permutation with its per-block scratch (expert counts and bases of each
// 256-token block) kept in the static array below instead of a workspace.
//
// Limits: T <= 65536 and E <= 256, i.e. 2 * 256 blocks * 256 experts * 4 B
// = 512 KiB, held by every device that loads the library until exit.
// Every call shares this array and overwrites each word it later reads, so
// nothing needs clearing between calls; calls whose kernels overlap on the
// GPU (other streams, other host threads) race on it and must be ordered by
// the caller.
namespace moe {
namespace {
constexpr int NOALLOC_MAX_T = 65536;
constexpr int NOALLOC_MAX_E = 256;
constexpr int NOALLOC_BLOCKS = NOALLOC_MAX_T / PERM_TOK;
constexpr size_t NOALLOC_WORDS = (size_t)2 * NOALLOC_BLOCKS * NOALLOC_MAX_E;
}  // namespace

static __device__ __align__(256) int32_t g_permute_scratch[NOALLOC_WORDS];

// Device address of g_permute_scratch on the current device.  The host-side
// name of a __device__ array is only a stand-in, so the address is looked up
// once per device (with that device current) and cached.
// The cache slots are atomic, so host threads that make their first calls
// at the same time may both look the address up; they store the same value.
static int permute_scratch_address(int32_t** out) {
  static std::atomic<int32_t*> cache[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(MOE_ERR_UNSUPPORTED, "device ordinal >= 64");
  int32_t* p = cache[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    void* q = nullptr;
    e = cudaGetSymbolAddress(&q, g_permute_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(permute scratch)");
    p = static_cast<int32_t*>(q);
    cache[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return MOE_OK;
}

}  // namespace moe

extern "C" int moe_permute_noalloc(const int32_t* idx, const float* gate, int T, int E, int k,
                                   int tile, int32_t* counts, int32_t* offsets,
                                   int32_t* row_token, float* row_gate, int32_t* row_slot,
                                   int32_t* slot_row, void* stream) {
  using namespace moe;
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T must be >= 0");
  if (k < 1 || k > 8) return fail(MOE_ERR_UNSUPPORTED, "k must be in [1, 8]");
  if (E < k || E > 256) return fail(MOE_ERR_UNSUPPORTED, "E must be in [k, 256]");
  if (tile != 128) return fail(MOE_ERR_UNSUPPORTED, "tile must be 128 (the grouped-GEMM M tile)");
  if (T > NOALLOC_MAX_T)
    return fail(MOE_ERR_UNSUPPORTED,
                "moe_permute_noalloc: T = " + std::to_string(T) +
                    " exceeds the static scratch limit of 65536 tokens; use moe_permute");
  if (counts == nullptr || offsets == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "counts and offsets must not be NULL");
  if (T > 0 && (idx == nullptr || gate == nullptr || row_token == nullptr ||
                row_gate == nullptr || row_slot == nullptr || slot_row == nullptr))
    return fail(MOE_ERR_INVALID_ARG, "idx, gate and the row maps must not be NULL");
  int32_t* scratch = nullptr;
  if (int rc = permute_scratch_address(&scratch)) return rc;
  const int nb = perm_blocks(T) > 0 ? perm_blocks(T) : 1;
  PermuteWs w{};
  w.blockcnt = scratch;
  w.blockbase = scratch + (size_t)nb * E;
  return launch_permute_exact(idx, gate, T, E, k, tile, counts, offsets, row_token, row_gate,
                              row_slot, slot_row, w, (cudaStream_t)stream);
}
