// Router projection: logits[t, e] = sum_h x[t, h] * router_w[e, h], fp32 FMA
// accumulation (mlxcel issue #838, section "Router: selection uses biased
// scores, weights come from unbiased scores": gates are float32 before the
// score function; section "Validation checkpoint": router weight mlp.gate
// is [E, H]).
//
// Small T: a weight-streaming GEMV (one warp per expert row, 16-byte loads,
// every token of the batch against each row). Larger T: a shared-memory tiled
// SIMT GEMM, 64 tokens x 64 experts per block.
#include "common.cuh"

namespace moe {

namespace {

constexpr int kGemvMaxT = 16;

// One warp per expert row; each lane covers 8 consecutive h per step
// (two float4 of router_w, one 16-byte bf16 chunk of x per token).
__global__ void __launch_bounds__(256) logits_gemv_kernel(const uint16_t* __restrict__ x, const float* __restrict__ w,
                                                          float* __restrict__ out, int T, int H, int E) {
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int nv = H / 8;
  for (int e = gw; e < E; e += nw) {
    const float* wr = w + (size_t)e * H;
    float acc[kGemvMaxT];
#pragma unroll
    for (int t = 0; t < kGemvMaxT; ++t) acc[t] = 0.0f;
    for (int v = lane; v < nv; v += 32) {
      const uint4 a = ld_stream_u4(wr + v * 8);
      const uint4 b = ld_stream_u4(wr + v * 8 + 4);
      float wf[8] = {__uint_as_float(a.x), __uint_as_float(a.y), __uint_as_float(a.z), __uint_as_float(a.w),
                     __uint_as_float(b.x), __uint_as_float(b.y), __uint_as_float(b.z), __uint_as_float(b.w)};
#pragma unroll
      for (int t = 0; t < kGemvMaxT; ++t) {
        if (t < T) {
          const uint4 xv = ld_nc_u4(x + (size_t)t * H + v * 8);
          float xf[8];
          unpack8_bf16(xv, xf);
          float s = acc[t];
#pragma unroll
          for (int i = 0; i < 8; ++i) s = fmaf(xf[i], wf[i], s);
          acc[t] = s;
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kGemvMaxT; ++t) {
      if (t < T) {
        const float s = warp_sum(acc[t]);
        if (lane == 0) out[(size_t)t * E + e] = s;
      }
    }
  }
}

// Tiled SIMT GEMM: block = 256 threads computes a 64 (tokens) x 64 (experts)
// tile, each thread 4 x 4 outputs; K staged through shared memory 32 at a time.
constexpr int TM = 64, TN = 64, TK = 32;

__global__ void __launch_bounds__(256) logits_tiled_kernel(const uint16_t* __restrict__ x, const float* __restrict__ w,
                                                           float* __restrict__ out, int T, int H, int E) {
  __shared__ float xs[TK][TM + 4];
  __shared__ float ws[TK][TN + 4];
  const int tid = threadIdx.x;
  const int t0 = blockIdx.y * TM, e0 = blockIdx.x * TN;
  const int ty = tid / 16, tx = tid % 16;  // 16 x 16 threads, 4 x 4 outputs each
  float acc[4][4] = {};
  for (int k0 = 0; k0 < H; k0 += TK) {
    // x tile: 64 rows x 32 cols bf16 -> 256 threads x 8 elements (one 16-byte load)
    {
      const int r = tid / 4, c = (tid % 4) * 8;
      const int t = t0 + r;
      float f[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      if (t < T && k0 + c < H) unpack8_bf16(ld_nc_u4(x + (size_t)t * H + k0 + c), f);
#pragma unroll
      for (int i = 0; i < 8; ++i) xs[c + i][r] = f[i];
    }
    // w tile: 64 rows x 32 cols fp32 -> 256 threads x 8 elements (two 16-byte loads)
    {
      const int r = tid / 4, c = (tid % 4) * 8;
      const int e = e0 + r;
      float f[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      if (e < E && k0 + c < H) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(w + (size_t)e * H + k0 + c));
        const float4 b = __ldg(reinterpret_cast<const float4*>(w + (size_t)e * H + k0 + c + 4));
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) ws[c + i][r] = f[i];
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < TK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = xs[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = ws[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + ty * 4 + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = e0 + tx * 4 + j;
      if (e < E) out[(size_t)t * E + e] = acc[i][j];
    }
  }
}

}  // namespace

cudaError_t launch_router_logits(const moe_config& c, const uint16_t* x, int64_t T, const float* w, float* out,
                                 cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int H = c.hidden_size, E = c.num_experts;
  before_launch(MOE_KERNEL_ROUTER_LOGITS, s);
  if (T <= kGemvMaxT) {
    int blocks = (E * 32 + 255) / 256;
    logits_gemv_kernel<<<blocks, 256, 0, s>>>(x, w, out, (int)T, H, E);
  } else {
    dim3 grid((E + TN - 1) / TN, (unsigned)((T + TM - 1) / TM));
    logits_tiled_kernel<<<grid, 256, 0, s>>>(x, w, out, (int)T, H, E);
  }
  after_launch(MOE_KERNEL_ROUTER_LOGITS, s);
  return cudaGetLastError();
}

}  // namespace moe
