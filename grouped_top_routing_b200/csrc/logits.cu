// Router projection: logits[t, e] = sum_h x[t, h] * router_w[e, h], fp32 FMA
// accumulation (mlxcel issue #838, section "Router: selection uses biased
// scores, weights come from unbiased scores": gates are float32 before the
// score function; section "Validation checkpoint": router weight mlp.gate
// is [E, H]).
//
// This file holds the small-batch form (T <= 16): a weight-streaming GEMV, one
// warp per expert row, 16-byte loads, every token of the batch against each
// row, fp32 FMA. Larger batches run on the tensor cores (umma_ffn.cu).
#include "common.cuh"

namespace moe {

namespace {

constexpr int kGemvMaxT = 16;  // largest batch this kernel takes

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

}  // namespace

cudaError_t launch_router_logits_gemv(const moe_config& c, const uint16_t* x, int64_t T, const float* w, float* out,
                                      cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  if (T > kGemvMaxT) return cudaErrorInvalidValue;
  const int H = c.hidden_size, E = c.num_experts;
  before_launch(MOE_KERNEL_ROUTER_LOGITS, s);
  const int blocks = (E * 32 + 255) / 256;
  logits_gemv_kernel<<<blocks, 256, 0, s>>>(x, w, out, (int)T, H, E);
  after_launch(MOE_KERNEL_ROUTER_LOGITS, s);
  return cudaGetLastError();
}

}  // namespace moe
