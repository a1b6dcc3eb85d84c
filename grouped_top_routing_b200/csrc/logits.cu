// Router projection: logits[t, e] = sum_h x[t, h] * router_w[e, h], fp32 FMA
// accumulation (mlxcel issue #838, section "Router: selection uses biased
// scores, weights come from unbiased scores": gates are float32 before the
// score function; section "Validation checkpoint": router weight mlp.gate
// is [E, H]).
//
// This file holds the small-batch form (T <= 16): a weight-streaming GEMV, one
// block per expert row, 16-byte loads, every token of the batch against each
// row, fp32 FMA. Larger batches run on the tensor cores (umma_ffn.cu).
#include "common.cuh"

namespace moe {

namespace {

constexpr int kGemvMaxT = 16;  // largest batch this kernel takes

// One block of 128 threads per expert row: thread i covers h in
// [32 i, 32 i + 32) (eight float4 of router_w, issued together), against every
// token of the batch; a block reduction then gives the T logits of the row.
// With one block per row, the whole router weight is in flight at once.
template <int MT>
__global__ void __launch_bounds__(128) logits_gemv_kernel(const uint16_t* __restrict__ x, const float* __restrict__ w,
                                                          float* __restrict__ out, int T, int H, int E) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ float red[4][MT];
  const int e = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* wr = w + (size_t)e * H;
  float acc[MT];
#pragma unroll
  for (int t = 0; t < MT; ++t) acc[t] = 0.0f;
  for (int h0 = tid * 32; h0 < H; h0 += 128 * 32) {
    float4 wv[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      wv[u] = (h0 + 4 * u < H) ? __ldg(reinterpret_cast<const float4*>(wr + h0) + u) : make_float4(0, 0, 0, 0);
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      if (t < T) {
        float s = acc[t];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (h0 + 8 * u < H) {
            float xf[8];
            unpack8_bf16(ld_nc_u4(x + (size_t)t * H + h0 + 8 * u), xf);
            const float4 a = wv[2 * u], b = wv[2 * u + 1];
            s = fmaf(xf[0], a.x, s);
            s = fmaf(xf[1], a.y, s);
            s = fmaf(xf[2], a.z, s);
            s = fmaf(xf[3], a.w, s);
            s = fmaf(xf[4], b.x, s);
            s = fmaf(xf[5], b.y, s);
            s = fmaf(xf[6], b.z, s);
            s = fmaf(xf[7], b.w, s);
          }
        }
        acc[t] = s;
      }
    }
  }
#pragma unroll
  for (int t = 0; t < MT; ++t) {
    const float v = warp_sum(acc[t]);
    if (lane == 0) red[warp][t] = v;
  }
  __syncthreads();
  if (tid < MT && tid < T) out[(size_t)tid * E + e] = (red[0][tid] + red[1][tid]) + (red[2][tid] + red[3][tid]);
}

}  // namespace

cudaError_t launch_router_logits_gemv(const moe_config& c, const uint16_t* x, int64_t T, const float* w, float* out,
                                      cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  if (T > kGemvMaxT) return cudaErrorInvalidValue;
  const int H = c.hidden_size, E = c.num_experts;
  before_launch(MOE_KERNEL_ROUTER_LOGITS, s);
  if (T <= 1) launch_pdl(logits_gemv_kernel<1>, dim3(E), dim3(128), 0, s, x, w, out, (int)T, H, E);
  else if (T <= 4) launch_pdl(logits_gemv_kernel<4>, dim3(E), dim3(128), 0, s, x, w, out, (int)T, H, E);
  else launch_pdl(logits_gemv_kernel<16>, dim3(E), dim3(128), 0, s, x, w, out, (int)T, H, E);
  after_launch(MOE_KERNEL_ROUTER_LOGITS, s);
  return cudaGetLastError();
}

}  // namespace moe
