// Token-to-expert permutation: histogram -> exclusive scan -> stable scatter.
//
// The pages name no permutation: the gather-matmul over stacked experts
// (mlxcel issue #838, section "Weight remap": experts stacked into
// switch_mlp tensors) implies one. This one orders the T*k assignments by
// (expert, token). The rank of assignment (t, e) inside its expert is the
// number of earlier tokens that also chose e, computed deterministically from
// per-tile bitmasks: mask[e] has bit t set when token t of the tile chose e,
// and the rank inside the tile is popcount(mask[e] & (bits below t)).
//
// Kernels (tile = 128 tokens):
//   count   : per tile, popcount of each expert's mask -> tile_cnt[tile][e]
//   scan    : one block: expert totals, exclusive scan -> offsets, per-tile
//             bases tile_base[tile][e], compacted list of experts with rows
//   scatter : per tile, rebuild masks, row = base + rank; write row_of/tok_of
//   rows    : when asked, x rows into x_perm in token order (each row of x
//             read once and written to the rows of its k slots)
// A single tile (T <= 128) runs all three steps in one block.
#include "common.cuh"

namespace moe {

namespace {

constexpr int kTile = 128;            // tokens per tile (one thread per token)
constexpr int kWords = kTile / 32;    // mask words per expert

// Builds the tile's masks in shared memory. Out-of-range or repeated ids are
// skipped and recorded. Called by all kTile threads; ends with __syncthreads.
__device__ void build_masks(uint32_t* masks, const int32_t* __restrict__ idx, int64_t t0, int64_t T, int k, int E,
                            WsHeader* hdr, bool record) {
  for (int i = threadIdx.x; i < E * kWords; i += blockDim.x) masks[i] = 0u;
  __syncthreads();
  const int tl = threadIdx.x;
  const int64_t t = t0 + tl;
  if (t < T) {
    for (int j = 0; j < k; ++j) {
      const int e = idx[t * k + j];
      if (e < 0 || e >= E) {
        if (record) record_error(hdr, MOE_ERR_DEVICE_CHECK, (int)(t * k + j));
        continue;
      }
      const uint32_t bit = 1u << (tl & 31);
      const uint32_t old = atomicOr(&masks[e * kWords + (tl >> 5)], bit);
      if ((old & bit) && record) record_error(hdr, MOE_ERR_DEVICE_CHECK, (int)(t * k + j));
    }
  }
  __syncthreads();
}

__device__ __forceinline__ int tile_count(const uint32_t* masks, int e) {
  int c = 0;
#pragma unroll
  for (int w = 0; w < kWords; ++w) c += __popc(masks[e * kWords + w]);
  return c;
}

// Rank of token tl among the tile's tokens that chose e.
__device__ __forceinline__ int tile_rank(const uint32_t* masks, int e, int tl) {
  int r = 0;
  const int wl = tl >> 5;
#pragma unroll
  for (int w = 0; w < kWords; ++w)
    if (w < wl) r += __popc(masks[e * kWords + w]);
  r += __popc(masks[e * kWords + wl] & ((1u << (tl & 31)) - 1u));
  return r;
}

// Writes row_of / tok_of for the tile's assignments, given each expert's base.
// Repeated ids were dropped from the masks: the first slot holding e keeps it,
// later ones get row -1.
__device__ void scatter_tile(const uint32_t* masks, const int* base_of_e, const int32_t* __restrict__ idx,
                             int64_t t0, int64_t T, int k, int E, int32_t* __restrict__ row_of,
                             int32_t* __restrict__ tok_of) {
  const int tl = threadIdx.x;
  const int64_t t = t0 + tl;
  if (t >= T) return;
  for (int j = 0; j < k; ++j) {
    const int e = idx[t * k + j];
    int32_t r = -1;
    if (e >= 0 && e < E) {
      bool dup = false;
      for (int jj = 0; jj < j; ++jj) dup |= (idx[t * k + jj] == e);
      if (!dup) r = base_of_e[e] + tile_rank(masks, e, tl);
    }
    row_of[t * k + j] = r;
    if (r >= 0) tok_of[r] = (int32_t)(t * k + j);
  }
}

// x_perm[r] = x[tok_of[r] / k] for the rows [0, offsets[E]); one thread per
// 16-byte chunk, grid-stride, so the copy keeps many loads in flight.
__global__ void __launch_bounds__(256) gather_rows_kernel(const int32_t* __restrict__ offsets, int E,
                                                          const int32_t* __restrict__ tok_of, int k, int64_t T,
                                                          const uint16_t* __restrict__ x, int H,
                                                          uint16_t* __restrict__ x_perm) {
  pdl_launch_dependents();
  pdl_wait();
  int64_t R = offsets[E];
  if (R < 0) R = 0;
  if (R > T * k) R = T * k;
  const int nv = H / 8;
  const int64_t n = R * nv;
  const uint4* src = reinterpret_cast<const uint4*>(x);
  uint4* dst = reinterpret_cast<uint4*>(x_perm);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / nv;
    const int v = (int)(i - r * nv);
    const int64_t slot = tok_of[r];
    if (slot < 0 || slot >= T * k) continue;
    dst[i] = __ldg(src + (slot / k) * nv + v);
  }
}

// The same copy in token order, when row_of is known: each 16-byte chunk of
// x[t] is read once and written to the k rows row_of[t*k + j] (x read once
// instead of k times).
__global__ void __launch_bounds__(256) scatter_rows_kernel(const int32_t* __restrict__ row_of, int k, int64_t T,
                                                           const uint16_t* __restrict__ x, int H,
                                                           uint16_t* __restrict__ x_perm) {
  pdl_launch_dependents();
  pdl_wait();
  const int nv = H / 8;
  const int64_t n = T * nv, R = T * k;
  const uint4* src = reinterpret_cast<const uint4*>(x);
  uint4* dst = reinterpret_cast<uint4*>(x_perm);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / nv;
    const int v = (int)(i - t * nv);
    const uint4 val = __ldg(src + i);
    for (int j = 0; j < k; ++j) {
      const int64_t r = row_of[t * k + j];
      if (r >= 0 && r < R) dst[r * nv + v] = val;
    }
  }
}

__global__ void __launch_bounds__(kTile) permute_count_kernel(const int32_t* __restrict__ idx, int64_t T, int k, int E,
                                                              int32_t* __restrict__ tile_cnt, WsHeader* hdr) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ uint32_t masks[];
  const int64_t t0 = (int64_t)blockIdx.x * kTile;
  build_masks(masks, idx, t0, T, k, E, hdr, true);
  for (int e = threadIdx.x; e < E; e += blockDim.x) tile_cnt[(int64_t)blockIdx.x * E + e] = tile_count(masks, e);
}

// Block-wide exclusive scan of one value per thread (blockDim.x == 1024).
__device__ int block_excl_scan(int v, int* total) {
  __shared__ int warp_sums[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_sums[lane] = w;
  }
  __syncthreads();
  const int prefix = (warp > 0 ? warp_sums[warp - 1] : 0) + x - v;
  *total = warp_sums[31];
  __syncthreads();
  return prefix;
}

__global__ void __launch_bounds__(1024) permute_scan_kernel(const int32_t* __restrict__ tile_cnt, int n_tiles, int E,
                                                            int32_t* __restrict__ offsets,
                                                            int32_t* __restrict__ tile_base,
                                                            int32_t* __restrict__ active, WsHeader* hdr) {
  pdl_launch_dependents();
  pdl_wait();
  const int e = threadIdx.x;
  int total = 0;
  if (e < E)
    for (int tile = 0; tile < n_tiles; ++tile) total += tile_cnt[(int64_t)tile * E + e];
  int all = 0;
  const int off = block_excl_scan(e < E ? total : 0, &all);
  int n_active = 0;
  const int aoff = block_excl_scan((e < E && total > 0) ? 1 : 0, &n_active);
  if (e < E) {
    offsets[e] = off;
    if (total > 0) active[aoff] = e;
    int run = off;
    for (int tile = 0; tile < n_tiles; ++tile) {
      tile_base[(int64_t)tile * E + e] = run;
      run += tile_cnt[(int64_t)tile * E + e];
    }
  }
  if (e == 0) {
    offsets[E] = all;
    hdr->num_active = n_active;
  }
}

__global__ void __launch_bounds__(kTile) permute_scatter_kernel(const int32_t* __restrict__ idx, int64_t T, int k, int E,
                                                                const int32_t* __restrict__ tile_base,
                                                                int32_t* __restrict__ row_of,
                                                                int32_t* __restrict__ tok_of) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ uint32_t masks[];
  const int64_t t0 = (int64_t)blockIdx.x * kTile;
  build_masks(masks, idx, t0, T, k, E, nullptr, false);
  scatter_tile(masks, tile_base + (int64_t)blockIdx.x * E, idx, t0, T, k, E, row_of, tok_of);
}

// T <= kTile: count, scan and scatter in one block of 1024 threads (the first
// kTile threads own the tokens).
__global__ void __launch_bounds__(1024) permute_small_kernel(const int32_t* __restrict__ idx, int64_t T, int k, int E,
                                                             int32_t* __restrict__ offsets, int32_t* __restrict__ row_of,
                                                             int32_t* __restrict__ tok_of, int32_t* __restrict__ active,
                                                             WsHeader* hdr) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ uint32_t masks[];
  int* base = reinterpret_cast<int*>(masks + E * kWords);
  for (int i = threadIdx.x; i < E * kWords; i += blockDim.x) masks[i] = 0u;
  __syncthreads();
  const int tl = threadIdx.x;
  if (tl < kTile && tl < T) {
    for (int j = 0; j < k; ++j) {
      const int e = idx[(int64_t)tl * k + j];
      if (e < 0 || e >= E) {
        record_error(hdr, MOE_ERR_DEVICE_CHECK, tl * k + j);
        continue;
      }
      const uint32_t bit = 1u << (tl & 31);
      const uint32_t old = atomicOr(&masks[e * kWords + (tl >> 5)], bit);
      if (old & bit) record_error(hdr, MOE_ERR_DEVICE_CHECK, tl * k + j);
    }
  }
  __syncthreads();
  const int cnt = (tl < E) ? tile_count(masks, tl) : 0;
  int all = 0;
  const int off = block_excl_scan(cnt, &all);
  int n_active = 0;
  const int aoff = block_excl_scan(cnt > 0 ? 1 : 0, &n_active);
  if (tl < E) {
    offsets[tl] = off;
    base[tl] = off;
    if (cnt > 0) active[aoff] = tl;
  }
  if (tl == 0) {
    offsets[E] = all;
    hdr->num_active = n_active;
  }
  __syncthreads();
  if (tl < kTile) scatter_tile(masks, base, idx, 0, T, k, E, row_of, tok_of);
}

}  // namespace

size_t permute_scratch_ints(int E, int64_t T) {
  const int64_t n_tiles = (T + kTile - 1) / kTile;
  return (size_t)(n_tiles > 0 ? n_tiles : 1) * E;
}

cudaError_t launch_permute(const moe_config& c, const int32_t* idx, int64_t T, const uint16_t* x, int32_t* offsets,
                           int32_t* row_of, int32_t* tok_of, uint16_t* x_perm, int32_t* active, int32_t* tile_cnt,
                           int32_t* tile_base, WsHeader* hdr, cudaStream_t s) {
  const int E = c.num_experts, k = c.num_experts_per_tok, H = c.hidden_size;
  const size_t mask_bytes = (size_t)E * kWords * sizeof(uint32_t);
  int nk = 0;
  before_launch(MOE_KERNEL_PERMUTE, s);
  if (T <= kTile) {
    const size_t smem = mask_bytes + (size_t)E * sizeof(int);
    nk = 1;
    launch_pdl(permute_small_kernel, dim3(1), dim3(1024), smem, s, idx, T, k, E, offsets, row_of, tok_of, active, hdr);
  } else {
    const int n_tiles = (int)((T + kTile - 1) / kTile);
    nk = 3;
    launch_pdl(permute_count_kernel, dim3(n_tiles), dim3(kTile), mask_bytes, s, idx, T, k, E, tile_cnt, hdr);
    launch_pdl(permute_scan_kernel, dim3(1), dim3(1024), 0, s, tile_cnt, n_tiles, E, offsets, tile_base, active, hdr);
    launch_pdl(permute_scatter_kernel, dim3(n_tiles), dim3(kTile), mask_bytes, s, idx, T, k, E, tile_base, row_of, tok_of);
  }
  if (x_perm != nullptr) {  // row_of is known here: copy in token order, each x row read once
    const int64_t chunks = T * (H / 8);
    int64_t blocks = (chunks + 255) / 256;
    const int64_t cap = (int64_t)sm_count() * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    launch_pdl(scatter_rows_kernel, dim3((unsigned)blocks), dim3(256), 0, s, row_of, k, T, x, H, x_perm);
    ++nk;
  }
  after_launch(MOE_KERNEL_PERMUTE, s, nk);
  return cudaGetLastError();
}

cudaError_t launch_gather_rows(const int32_t* offsets, int E, const int32_t* tok_of, int k, int64_t T,
                               const uint16_t* x, int H, uint16_t* x_perm, cudaStream_t s) {
  const int64_t chunks = T * k * (H / 8);
  int64_t blocks = (chunks + 255) / 256;
  const int64_t cap = (int64_t)sm_count() * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  before_launch(MOE_KERNEL_PERMUTE, s);
  launch_pdl(gather_rows_kernel, dim3((unsigned)blocks), dim3(256), 0, s, offsets, E, tok_of, k, T, x, H, x_perm);
  after_launch(MOE_KERNEL_PERMUTE, s);
  return cudaGetLastError();
}

// Rebuilds the compacted list of experts with rows from expert_offsets (used
// when moe_expert_ffn is called on its own).
__global__ void __launch_bounds__(1024) active_from_offsets_kernel(const int32_t* __restrict__ offsets, int E,
                                                                   int32_t* __restrict__ active, WsHeader* hdr) {
  pdl_launch_dependents();
  pdl_wait();
  const int e = threadIdx.x;
  const int has = (e < E && offsets[e + 1] > offsets[e]) ? 1 : 0;
  int n = 0;
  const int pos = block_excl_scan(has, &n);
  if (has) active[pos] = e;
  if (e == 0) hdr->num_active = n;
}

cudaError_t launch_active_from_offsets(const int32_t* offsets, int E, int32_t* active, WsHeader* hdr,
                                       cudaStream_t s) {
  before_launch(MOE_KERNEL_PERMUTE, s);
  launch_pdl(active_from_offsets_kernel, dim3(1), dim3(1024), 0, s, offsets, E, active, hdr);
  after_launch(MOE_KERNEL_PERMUTE, s);
  return cudaGetLastError();
}

// The routing of a dense MLP seen as a block of one expert with one slot per
// token and weight 1.0: offsets {0, T}, row r holds slot r, every weight 1.
__global__ void __launch_bounds__(256) identity_route_kernel(int64_t T, int32_t* __restrict__ offsets,
                                                             int32_t* __restrict__ tok_of, float* __restrict__ w) {
  pdl_launch_dependents();
  pdl_wait();
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < T; i += stride) {
    tok_of[i] = (int32_t)i;
    w[i] = 1.0f;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    offsets[0] = 0;
    offsets[1] = (int32_t)T;
  }
}

cudaError_t launch_identity_route(int64_t T, int32_t* offsets, int32_t* tok_of, float* w, cudaStream_t s) {
  int64_t blocks = (T + 255) / 256;
  const int64_t cap = (int64_t)sm_count() * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  before_launch(MOE_KERNEL_PERMUTE, s);
  launch_pdl(identity_route_kernel, dim3((unsigned)blocks), dim3(256), 0, s, T, offsets, tok_of, w);
  after_launch(MOE_KERNEL_PERMUTE, s);
  return cudaGetLastError();
}

}  // namespace moe
