// Router kernel: one warp per token, running route_one_token (route.cuh).
#include "common.cuh"
#include "route.cuh"

namespace moe {

namespace {

template <int P>
__global__ void __launch_bounds__(256) route_kernel(
    const float* __restrict__ logits, const float* __restrict__ bias, int T, int E, int k, int n_group,
    int topk_group, int score_fn, int norm, float scale, int32_t* __restrict__ idx_out,
    float* __restrict__ w_out) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ float smem[];
  const int warp = threadIdx.x >> 5;
  const int wpb = blockDim.x >> 5;
  float* buf = smem + warp * (32 * P);  // per-warp scratch: biased scores, then raw weights
  for (int t = blockIdx.x * wpb + warp; t < T; t += gridDim.x * wpb)
    route_one_token<P>(logits + (size_t)t * E, bias, E, k, n_group, topk_group, score_fn, norm, scale, buf,
                       idx_out + (size_t)t * k, w_out + (size_t)t * k);
}

template <int P>
cudaError_t launch_route_p(const moe_config& c, const float* logits, const float* bias, int T,
                           int32_t* idx, float* w, cudaStream_t s) {
  const int wpb = 8;
  int blocks = (T + wpb - 1) / wpb;
  const int cap = sm_count() * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  const size_t smem = (size_t)wpb * 32 * P * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(route_kernel<P>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  before_launch(MOE_KERNEL_ROUTE, s);
  launch_pdl(route_kernel<P>, dim3(blocks), dim3(wpb * 32), smem, s, logits, bias, T, c.num_experts, c.num_experts_per_tok,
                                                 c.n_group, c.topk_group, c.score_function, c.norm_topk_prob,
                                                 c.routed_scaling_factor, idx, w);
  after_launch(MOE_KERNEL_ROUTE, s);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route(const moe_config& c, const float* logits, const float* bias, int64_t T, int32_t* idx,
                         float* w, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int E = c.num_experts;
  const int per = (E + 31) / 32;
  const int t = (int)T;
  if (per <= 1) return launch_route_p<1>(c, logits, bias, t, idx, w, s);
  if (per <= 2) return launch_route_p<2>(c, logits, bias, t, idx, w, s);
  if (per <= 4) return launch_route_p<4>(c, logits, bias, t, idx, w, s);
  if (per <= 8) return launch_route_p<8>(c, logits, bias, t, idx, w, s);
  if (per <= 16) return launch_route_p<16>(c, logits, bias, t, idx, w, s);
  return launch_route_p<32>(c, logits, bias, t, idx, w, s);
}

}  // namespace moe
