// Fused decode: the whole MoE block for 1-2 tokens in one launch.
//
// At decode the block is bound by HBM bandwidth: it must stream the router
// weight and the weights of the few selected experts ("only the selected
// experts are read", page "Ling-3.0-flash-GGUF", section "Measured
// performance") plus the shared MLP. As separate kernels the chain of six
// launches, each a few microseconds of latency, dominates the ~20 us of
// streaming. Here one cooperative grid (every CTA resident) runs the steps as
// phases separated by grid barriers:
//
//   A  router logits (one warp per router row, fp32 FMA) and the shared MLP's
//      gate/up rows (they do not depend on the routing)            -> barrier
//   B  every CTA routes the 1-2 tokens itself (route_one_token, the router
//      kernel's own code) and lists the selected experts in shared memory:
//      no barrier needed, each CTA already holds the routing
//   C  gate/up rows of the selected experts, SwiGLU in fp32         -> barrier
//   D  down rows of the selected experts (weighted by the routing) and of the
//      shared MLP, fp32 per slot                                    -> barrier
//   E  combine: y = bf16(sum of the k slot rows + the shared row), slot order
//
// Data written in one phase and read in a later one by other CTAs is read
// with ld.global.cg (L2), never through the read-only path. Each grid barrier
// is bounded (globaltimer, ~2 s): a barrier that runs out records
// MOE_ERR_TIMEOUT in the workspace and the CTA returns.
#include "common.cuh"
#include "route.cuh"

namespace moe {

struct DecodeArgs {
  const uint16_t* x;  // [T, H]
  int T, H, E, k, I, Is, n_group, topk_group, score_fn, norm;
  float scale;
  const float* router_w;         // [E, H] or null when logits are given
  const float* expert_bias;      // [E] or null
  const float* logits_override;  // [T, E] or null
  const uint16_t* w_gate_up;     // [E, 2I, H]
  const uint16_t* w_down;        // [E, H, I]
  const uint16_t* ws_gate_up;    // [2Is, H] or null
  const uint16_t* ws_down;       // [H, Is]
  float* logits;                 // [T, E] workspace
  int32_t* topk_idx_out;         // [T, k] or null
  float* topk_w_out;             // [T, k] or null
  float* h;                      // [T*k, I] workspace
  float* h_shared;               // [T, Is] workspace
  float* y_slots;                // [T*k, H] workspace
  float* shared_out;             // [T, H] workspace
  uint16_t* y;                   // [T, H] output
  WsHeader* hdr;
};

namespace {

constexpr int kFusedThreads = 256;
constexpr int kFusedMaxT = 2;
constexpr int kDownRows = 8;
constexpr uint64_t kBarrierTimeoutNs = 2000000000ull;

__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Grid-wide barrier over gridDim.x CTAs (sense by generation). Returns false
// if it timed out. Writes before it are visible to ld.global.cg after it.
__device__ bool grid_barrier(WsHeader* hdr, int site, int* s_flag) {
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    volatile uint32_t* gen = &hdr->bar_gen;
    const uint32_t g = *gen;
    __threadfence();
    const uint32_t arrived = atomicAdd(&hdr->bar_count, 1u);
    if (arrived == gridDim.x - 1) {
      hdr->bar_count = 0u;
      __threadfence();
      atomicAdd(&hdr->bar_gen, 1u);
    } else {
      const uint64_t t0 = gtimer();
      while (*gen == g) {
        if (gtimer() - t0 > kBarrierTimeoutNs) {
          record_error(hdr, MOE_ERR_TIMEOUT, 100 + site);
          ok = 0;
          break;
        }
      }
    }
    __threadfence();
    *s_flag = ok;
  }
  __syncthreads();
  return *s_flag != 0;
}

__device__ __forceinline__ float4 ldcg4(const float* p) { return __ldcg(reinterpret_cast<const float4*>(p)); }

// silu(gate . x_t) * (up . x_t) for up to two token rows against one pair of
// gate/up weight rows (H bf16 each), fp32. One warp; every lane gets the sums.
__device__ __forceinline__ void gate_up_dot(const uint16_t* __restrict__ gate, const uint16_t* __restrict__ up,
                                            const uint16_t* x0, const uint16_t* x1, int H, float* h0, float* h1) {
  const int lane = threadIdx.x & 31;
  const int nv = H / 8;
  float g0 = 0.f, u0 = 0.f, g1 = 0.f, u1 = 0.f;
  for (int v0 = lane; v0 < nv; v0 += 32 * 8) {
    uint4 gv[8], uv[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int v = v0 + 32 * u;
      if (v < nv) {
        gv[u] = ld_stream_u4(gate + v * 8);
        uv[u] = ld_stream_u4(up + v * 8);
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int v = v0 + 32 * u;
      if (v < nv) {
        float xf[8];
        unpack8_bf16(ld_nc_u4(x0 + v * 8), xf);
        g0 = dot8_bf16(gv[u], xf, g0);
        u0 = dot8_bf16(uv[u], xf, u0);
        if (x1 != nullptr) {
          unpack8_bf16(ld_nc_u4(x1 + v * 8), xf);
          g1 = dot8_bf16(gv[u], xf, g1);
          u1 = dot8_bf16(uv[u], xf, u1);
        }
      }
    }
  }
  g0 = warp_sum(g0);
  u0 = warp_sum(u0);
  *h0 = silu_f32(g0) * u0;
  if (x1 != nullptr) {
    g1 = warp_sum(g1);
    u1 = warp_sum(u1);
    *h1 = silu_f32(g1) * u1;
  }
}

// kDownRows rows (K bf16 each) of a down projection against up to two fp32
// h rows (written earlier in this launch: read through L2). Lane r*2 + t ends
// up holding the dot of row r with h row t.
__device__ __forceinline__ float down_dot(const uint16_t* __restrict__ w0, int nrows, int K, const float* hr0,
                                          const float* hr1) {
  const int lane = threadIdx.x & 31;
  const int nvk = K / 8;
  float acc[kDownRows][2];
#pragma unroll
  for (int r = 0; r < kDownRows; ++r) acc[r][0] = acc[r][1] = 0.f;
  for (int v = lane; v < nvk; v += 32) {
    uint4 wv[kDownRows];
#pragma unroll
    for (int r = 0; r < kDownRows; ++r)
      if (r < nrows) wv[r] = ld_stream_u4(w0 + (int64_t)r * K + v * 8);
    const float4 a0 = ldcg4(hr0 + v * 8), a1 = ldcg4(hr0 + v * 8 + 4);
    const float f0[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
    for (int r = 0; r < kDownRows; ++r)
      if (r < nrows) acc[r][0] = dot8_bf16(wv[r], f0, acc[r][0]);
    if (hr1 != nullptr) {
      const float4 b0 = ldcg4(hr1 + v * 8), b1 = ldcg4(hr1 + v * 8 + 4);
      const float f1[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int r = 0; r < kDownRows; ++r)
        if (r < nrows) acc[r][1] = dot8_bf16(wv[r], f1, acc[r][1]);
    }
  }
  float mine = 0.f;
#pragma unroll
  for (int r = 0; r < kDownRows; ++r)
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      if (r < nrows && (t == 0 || hr1 != nullptr)) {
        const float s = warp_sum(acc[r][t]);
        if (lane == r * 2 + t) mine = s;
      }
    }
  return mine;
}

template <int P>
__global__ void __launch_bounds__(kFusedThreads) decode_fused_kernel(const DecodeArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int T = a.T, E = a.E, k = a.k, H = a.H, I = a.I, Is = a.Is;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gw = blockIdx.x * (kFusedThreads / 32) + warp;
  const int nw = gridDim.x * (kFusedThreads / 32);
  // shared memory: per-token route scratch, routing, slot table, active list
  float* rbuf = reinterpret_cast<float*>(smem_raw);                       // [kFusedMaxT][32*P]
  int32_t* s_idx = reinterpret_cast<int32_t*>(rbuf + kFusedMaxT * 32 * P);  // [T*k]
  float* s_w = reinterpret_cast<float*>(s_idx + kFusedMaxT * E);          // [T*k]
  int32_t* s_slot = reinterpret_cast<int32_t*>(s_w + kFusedMaxT * E);     // [T][E]: slot of expert e, or -1
  int32_t* s_active = s_slot + kFusedMaxT * E;                            // [E]
  int* s_misc = s_active + E;                                             // [0] n_active, [1] barrier flag, [2..] scan

  // ---- A: router logits and the shared MLP's gate/up rows ----
  const int n_router = a.logits_override == nullptr ? E : 0;
  const int n_shared = a.ws_gate_up != nullptr ? Is : 0;
  const float* logits = a.logits_override != nullptr ? a.logits_override : a.logits;
  for (int item = gw; item < n_router + n_shared; item += nw) {
    if (item < n_router) {
      const float* wr = a.router_w + (int64_t)item * H;
      float acc0 = 0.f, acc1 = 0.f;
      for (int h4 = lane; h4 < H / 4; h4 += 32) {
        const float4 w4 = __ldg(reinterpret_cast<const float4*>(wr) + h4);
        const uint2 xa = __ldg(reinterpret_cast<const uint2*>(a.x) + h4);
        acc0 = fmaf(bf16_lo(xa.x), w4.x, acc0);
        acc0 = fmaf(bf16_hi(xa.x), w4.y, acc0);
        acc0 = fmaf(bf16_lo(xa.y), w4.z, acc0);
        acc0 = fmaf(bf16_hi(xa.y), w4.w, acc0);
        if (T > 1) {
          const uint2 xb = __ldg(reinterpret_cast<const uint2*>(a.x + H) + h4);
          acc1 = fmaf(bf16_lo(xb.x), w4.x, acc1);
          acc1 = fmaf(bf16_hi(xb.x), w4.y, acc1);
          acc1 = fmaf(bf16_lo(xb.y), w4.z, acc1);
          acc1 = fmaf(bf16_hi(xb.y), w4.w, acc1);
        }
      }
      acc0 = warp_sum(acc0);
      if (T > 1) acc1 = warp_sum(acc1);
      if (lane == 0) {
        a.logits[item] = acc0;
        if (T > 1) a.logits[E + item] = acc1;
      }
    } else {
      const int j = item - n_router;
      const uint16_t* gate = a.ws_gate_up + (int64_t)j * H;
      float h0, h1;
      gate_up_dot(gate, gate + (int64_t)Is * H, a.x, T > 1 ? a.x + H : nullptr, H, &h0, &h1);
      if (lane == 0) {
        a.h_shared[j] = h0;
        if (T > 1) a.h_shared[Is + j] = h1;
      }
    }
  }
  if (!grid_barrier(a.hdr, 1, s_misc + 1)) return;

  // ---- B: every CTA routes the tokens and lists the selected experts ----
  for (int i = threadIdx.x; i < kFusedMaxT * E; i += blockDim.x) s_slot[i] = -1;
  if (warp < T)
    route_one_token<P, true>(logits + (int64_t)warp * E, a.expert_bias, E, k, a.n_group, a.topk_group, a.score_fn,
                             a.norm, a.scale, rbuf + warp * 32 * P, s_idx + warp * k, s_w + warp * k);
  __syncthreads();
  for (int i = threadIdx.x; i < T * k; i += blockDim.x) {
    const int t = i / k, e = s_idx[i];
    s_slot[t * E + e] = i;  // ids are valid and distinct per token
    if (blockIdx.x == 0) {
      if (a.topk_idx_out != nullptr) a.topk_idx_out[i] = e;
      if (a.topk_w_out != nullptr) a.topk_w_out[i] = s_w[i];
    }
  }
  __syncthreads();
  {  // compact the selected experts in ascending id order (4 ids per thread)
    int cnt = 0;
    int flags[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e = threadIdx.x * 4 + q;
      flags[q] = (e < E) && (s_slot[e] >= 0 || (T > 1 && s_slot[E + e] >= 0));
      cnt += flags[q];
    }
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int* wsum = s_misc + 2;
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += wsum[w];
    int pos = base + incl - cnt;
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (flags[q]) s_active[pos++] = threadIdx.x * 4 + q;
    if (threadIdx.x == blockDim.x - 1) s_misc[0] = base + incl;
  }
  __syncthreads();
  const int n_act = s_misc[0];

  // ---- C: gate/up rows of the selected experts ----
  for (int item = gw; item < n_act * I; item += nw) {
    const int ai = item / I, j = item - ai * I;
    const int e = s_active[ai];
    const int sl0 = s_slot[e], sl1 = T > 1 ? s_slot[E + e] : -1;
    const int slA = sl0 >= 0 ? sl0 : sl1;  // first slot holding e
    const int slB = sl0 >= 0 ? sl1 : -1;   // second (token 1), if both tokens chose e
    const uint16_t* gate = a.w_gate_up + ((int64_t)e * 2 * I + j) * H;
    float hA, hB;
    gate_up_dot(gate, gate + (int64_t)I * H, a.x + (int64_t)(slA / k) * H,
                slB >= 0 ? a.x + (int64_t)(slB / k) * H : nullptr, H, &hA, &hB);
    if (lane == 0) {
      a.h[(int64_t)slA * I + j] = hA;
      if (slB >= 0) a.h[(int64_t)slB * I + j] = hB;
    }
  }
  if (!grid_barrier(a.hdr, 2, s_misc + 1)) return;

  // ---- D: down rows, routed (weighted, per slot) and shared ----
  const int nrb = (H + kDownRows - 1) / kDownRows;
  const int routed_items = n_act * nrb;
  const int total = routed_items + (a.ws_down != nullptr ? nrb : 0);
  for (int item = gw; item < total; item += nw) {
    const bool shared = item >= routed_items;
    const int ai = shared ? 0 : item / nrb;
    const int n0 = (shared ? item - routed_items : item - ai * nrb) * kDownRows;
    const int nrows = min(kDownRows, H - n0);
    if (shared) {
      const float mine = down_dot(a.ws_down + (int64_t)n0 * Is, nrows, Is, a.h_shared, T > 1 ? a.h_shared + Is : nullptr);
      const int r = lane >> 1, t = lane & 1;
      if (r < nrows && t < T) a.shared_out[(int64_t)t * H + n0 + r] = mine;
    } else {
      const int e = s_active[ai];
      const int sl0 = s_slot[e], sl1 = T > 1 ? s_slot[E + e] : -1;
      const int slA = sl0 >= 0 ? sl0 : sl1;
      const int slB = sl0 >= 0 ? sl1 : -1;
      const float mine = down_dot(a.w_down + ((int64_t)e * H + n0) * I, nrows, I, a.h + (int64_t)slA * I,
                                  slB >= 0 ? a.h + (int64_t)slB * I : nullptr);
      const int r = lane >> 1, t = lane & 1;
      const int sl = t == 0 ? slA : slB;
      if (r < nrows && sl >= 0) a.y_slots[(int64_t)sl * H + n0 + r] = s_w[sl] * mine;
    }
  }
  if (!grid_barrier(a.hdr, 3, s_misc + 1)) return;

  // ---- E: y[t] = bf16( sum_j y_slots[t*k + j] + shared_out[t] ), slot order ----
  const int nv = H / 4;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < T * nv; i += gridDim.x * blockDim.x) {
    const int t = i / nv, v = i - t * nv;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      const float4 f = ldcg4(a.y_slots + ((int64_t)(t * k + j) * H) + v * 4);
      acc.x += f.x;
      acc.y += f.y;
      acc.z += f.z;
      acc.w += f.w;
    }
    if (a.ws_down != nullptr) {
      const float4 f = ldcg4(a.shared_out + (int64_t)t * H + v * 4);
      acc.x += f.x;
      acc.y += f.y;
      acc.z += f.z;
      acc.w += f.w;
    }
    reinterpret_cast<uint2*>(a.y)[i] = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
  }
}

template <int P>
size_t fused_smem(int E) {
  return (size_t)kFusedMaxT * 32 * P * 4 + (size_t)kFusedMaxT * E * 4 * 3 + (size_t)E * 4 + 64;
}

template <int P>
cudaError_t launch_fused_p(const DecodeArgs& a, cudaStream_t s) {
  const size_t smem = fused_smem<P>(a.E);
  cudaError_t e = cudaFuncSetAttribute(decode_fused_kernel<P>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_fused_kernel<P>, kFusedThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const int blocks = sm_count() * per_sm;  // every CTA resident: the grid barriers rely on it
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(kFusedThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  before_launch(MOE_KERNEL_DECODE_FUSED, s);
  e = cudaLaunchKernelEx(&cfg, decode_fused_kernel<P>, a);
  after_launch(MOE_KERNEL_DECODE_FUSED, s);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

bool decode_fused_supported(int64_t T, int k, int E) {
  // k <= E and the token count: the slot table holds two tokens
  return T >= 1 && T <= kFusedMaxT && k <= E && E <= 1024;
}

cudaError_t launch_decode_fused(const DecodeArgs& a, cudaStream_t s) {
  const int per = (a.E + 31) / 32;
  if (per <= 1) return launch_fused_p<1>(a, s);
  if (per <= 2) return launch_fused_p<2>(a, s);
  if (per <= 4) return launch_fused_p<4>(a, s);
  if (per <= 8) return launch_fused_p<8>(a, s);
  if (per <= 16) return launch_fused_p<16>(a, s);
  return launch_fused_p<32>(a, s);
}

}  // namespace moe
