// Expert-parallel exchange plan and the row-space pieces of the backward.
//
// With G ranks each owning El = E / G consecutive experts (rank g owns
// experts g*El .. g*El+El-1), a rank's permuted row space is already a send
// buffer: the rows for rank g are the segments of its experts, contiguous
// and 128-aligned (the Olmo-core 3 piece: row-wise expert parallelism puts
// the data straight into the experts' input buffers).  A receiving rank
// places the segment that source s sends for local expert j at
//   recv_row[s][j] = local_offsets[j] + sum over s' < s of recv_rows[s'][j],
//   local_offsets[j] = sum over j' < j, all s of recv_rows[s][j'],
// so every local expert's rows are contiguous (sources in rank order) and
// every segment stays a multiple of 128 rows: the grouped GEMMs run on the
// received rows exactly as on a local plan.
#include "common.cuh"
#include "internal.h"

namespace moe {

__global__ void k_ep_dispatch_counts(const int32_t* __restrict__ offsets, int E,
                                     int32_t* __restrict__ seg_rows) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) seg_rows[e] = offsets[e + 1] - offsets[e];
}

// One block; thread j owns local expert j (El <= 256).  A segment length that
// is negative or not a multiple of 128 cannot come from a plan: it is flagged
// (code 0x130) and counted as empty.
__global__ void k_ep_receive_plan(const int32_t* __restrict__ recv_rows, int G, int El,
                                  int32_t* __restrict__ local_offsets,
                                  int32_t* __restrict__ recv_row, int* status) {
  __shared__ int32_t tot[256];
  __shared__ int32_t base[257];
  const int j = threadIdx.x;
  auto rows_of = [&](int s) -> int32_t {
    const int32_t c = recv_rows[(size_t)s * El + j];
    if (c < 0 || (c & 127)) {
      record_status(status, 0x130);
      return 0;
    }
    return c;
  };
  if (j < El) {
    int32_t t = 0;
    for (int s = 0; s < G; ++s) t += rows_of(s);
    tot[j] = t;
  }
  __syncthreads();
  if (j == 0) {
    base[0] = 0;
    for (int i = 0; i < El; ++i) base[i + 1] = base[i] + tot[i];
  }
  __syncthreads();
  for (int i = j; i <= El; i += blockDim.x) local_offsets[i] = base[i];
  if (j < El) {
    int32_t pos = base[j];
    for (int s = 0; s < G; ++s) {
      recv_row[(size_t)s * El + j] = pos;
      pos += rows_of(s);
    }
  }
}

// dS of each row below offsets[E]: its partial sums added in a fixed order
// (the order in which the router backward adds them), so that the router
// gradient computed from these rows matches the one-GPU layer bit for bit.
__global__ void k_ds_rows(const float* __restrict__ ds_part, int nparts,
                          const int32_t* __restrict__ offsets, int E, float* __restrict__ dS) {
  const int R = offsets[E];
  for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < R; r += gridDim.x * blockDim.x) {
    float ds = 0.f;
    for (int p = 0; p < nparts; ++p) ds += ds_part[(size_t)r * nparts + p];
    dS[r] = ds;
  }
}

int launch_ep_dispatch_counts(const int32_t* offsets, int E, int32_t* seg_rows, cudaStream_t s) {
  {
    ProfScope _ps("ep_dispatch_counts", s);
    k_ep_dispatch_counts<<<1, 256, 0, s>>>(offsets, E, seg_rows);
  }
  MOE_CHECK_LAUNCH("ep_dispatch_counts");
  return MOE_OK;
}

int launch_ep_receive_plan(const int32_t* recv_rows, int G, int El, int32_t* local_offsets,
                           int32_t* recv_row, cudaStream_t s) {
  {
    ProfScope _ps("ep_receive_plan", s);
    k_ep_receive_plan<<<1, 256, 0, s>>>(recv_rows, G, El, local_offsets, recv_row, status_ptr());
  }
  MOE_CHECK_LAUNCH("ep_receive_plan");
  return MOE_OK;
}

int launch_ds_rows(const float* ds_part, int nparts, const int32_t* offsets, int E, int rows,
                   float* dS, cudaStream_t s) {
  int blocks = (rows + 255) / 256;
  if (blocks < 1) blocks = 1;
  if (blocks > device_sm_count() * 8) blocks = device_sm_count() * 8;
  {
    ProfScope _ps("ds_rows", s);
    k_ds_rows<<<blocks, 256, 0, s>>>(ds_part, nparts, offsets, E, dS);
  }
  MOE_CHECK_LAUNCH("ds_rows");
  return MOE_OK;
}

}  // namespace moe
