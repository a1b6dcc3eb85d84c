// Expert parallelism: the row lists around the two all-to-alls.
//
// With the routed experts spread over P ranks (mlxcel issue #838, sections
// "Shared experts are one wide MLP, not N separate experts" and "Touchpoints &
// acceptance criteria": a distributed entry), a rank sends its permuted rows
// (grouped by expert, hence by owner) to the experts' owners and gets the
// weighted results back. These kernels build what the exchange needs on the
// device: the per-expert counts and the routing weight of every permuted row
// (send side), the local expert of every received row (receive side), and the
// results' scatter back to slot order. Each is a small bandwidth-bound pass.
#include "common.cuh"

namespace moe {

namespace {

// counts[e] = offsets[e+1] - offsets[e] (int64, the count exchange's payload);
// row_w[r] = topk_w[tok_of[r]] for r < offsets[E] (0 for an invalid slot).
__global__ void __launch_bounds__(256) ep_send_kernel(const int32_t* __restrict__ offsets, int E,
                                                      const int32_t* __restrict__ tok_of,
                                                      const float* __restrict__ topk_w, int64_t R_max,
                                                      int64_t* __restrict__ counts, float* __restrict__ row_w) {
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t e = tid; e < E; e += stride) counts[e] = (int64_t)offsets[e + 1] - offsets[e];
  int64_t R = offsets[E];
  if (R < 0) R = 0;
  if (R > R_max) R = R_max;
  for (int64_t r = tid; r < R; r += stride) {
    const int64_t sl = tok_of[r];
    row_w[r] = (sl >= 0 && sl < R_max) ? topk_w[sl] : 0.0f;
  }
}

// local_expert[r] = (segment of r) % n_local, where the received rows come
// source by source and, within a source, expert by expert: segment s holds
// recv_counts[s] rows. Every block scans the (at most 1024) counts itself,
// then places its share of the rows by binary search.
__global__ void __launch_bounds__(1024) ep_recv_kernel(const int64_t* __restrict__ recv_counts, int nseg,
                                                       int n_local, int64_t R, int32_t* __restrict__ local_expert) {
  __shared__ int64_t start[1025];
  __shared__ int64_t warp_sums[32];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  int64_t v = tid < nseg ? recv_counts[tid] : 0;
  if (v < 0) v = 0;
  int64_t incl = v;
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sums[w] = incl;
  __syncthreads();
  if (w == 0) {
    int64_t s = warp_sums[lane];
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    warp_sums[lane] = s;  // inclusive sums of the warps
  }
  __syncthreads();
  const int64_t excl = incl - v + (w > 0 ? warp_sums[w - 1] : 0);
  if (tid < nseg) start[tid] = excl;
  if (tid == 0) start[nseg] = warp_sums[31];
  __syncthreads();
  for (int64_t r = (int64_t)blockIdx.x * blockDim.x + tid; r < R; r += (int64_t)gridDim.x * blockDim.x) {
    int lo = 0, hi = nseg - 1;  // the last segment whose start <= r
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (start[mid] <= r) lo = mid;
      else hi = mid - 1;
    }
    local_expert[r] = r < start[nseg] ? lo % n_local : -1;
  }
}

// y_slots[tok_of[r]] = y_perm[r] for r < R (slots < n_slots), one thread per 16 bytes.
__global__ void __launch_bounds__(256) ep_scatter_back_kernel(const float* __restrict__ y_perm,
                                                              const int32_t* __restrict__ tok_of, int64_t R,
                                                              int64_t n_slots, int H, float* __restrict__ y_slots) {
  const int nv = H / 4;
  const int64_t n = R * nv;
  const float4* src = reinterpret_cast<const float4*>(y_perm);
  float4* dst = reinterpret_cast<float4*>(y_slots);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / nv;
    const int v = (int)(i - r * nv);
    const int64_t sl = tok_of[r];
    if (sl >= 0 && sl < n_slots) dst[sl * nv + v] = __ldg(src + i);
  }
}

int64_t grid_for(int64_t n, int per_block) {
  int64_t b = (n + per_block - 1) / per_block;
  const int64_t cap = (int64_t)sm_count() * 8;
  if (b > cap) b = cap;
  return b < 1 ? 1 : b;
}

}  // namespace

cudaError_t launch_ep_send(const int32_t* offsets, int E, const int32_t* tok_of, const float* topk_w, int64_t R_max,
                           int64_t* counts, float* row_w, cudaStream_t s) {
  ep_send_kernel<<<(unsigned)grid_for(R_max > E ? R_max : E, 256), 256, 0, s>>>(offsets, E, tok_of, topk_w, R_max,
                                                                                counts, row_w);
  after_launch(MOE_KERNEL_COUNT, s);  // no timer selects this id: only counts the launch
  return cudaGetLastError();
}

cudaError_t launch_ep_recv(const int64_t* recv_counts, int nseg, int n_local, int64_t R, int32_t* local_expert,
                           cudaStream_t s) {
  if (R == 0) return cudaSuccess;
  ep_recv_kernel<<<(unsigned)grid_for(R, 1024), 1024, 0, s>>>(recv_counts, nseg, n_local, R, local_expert);
  after_launch(MOE_KERNEL_COUNT, s);
  return cudaGetLastError();
}

cudaError_t launch_ep_scatter_back(const float* y_perm, const int32_t* tok_of, int64_t R, int64_t n_slots, int H,
                                   float* y_slots, cudaStream_t s) {
  if (R == 0) return cudaSuccess;
  ep_scatter_back_kernel<<<(unsigned)grid_for(R * (H / 4), 256), 256, 0, s>>>(y_perm, tok_of, R, n_slots, H,
                                                                              y_slots);
  after_launch(MOE_KERNEL_COUNT, s);
  return cudaGetLastError();
}

}  // namespace moe
