// bf16 -> fp16 conversion of down-projection weights, once, for the
// tensor-core down pass on fp16 operands (moe_options.w_down_f16). A
// bandwidth-bound elementwise pass: 16-byte loads and stores, a grid of a few
// CTAs per SM striding over the array, one atomic per warp for the count of
// values fp16 cannot hold.
#include "common.cuh"

namespace moe {

namespace {

__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v, int* bad) {
  const uint16_t a = f32_to_f16(__uint_as_float(v << 16));
  const uint16_t b = f32_to_f16(__uint_as_float(v & 0xFFFF0000u));
  *bad += (f16_finite(a) ? 0 : 1) + (f16_finite(b) ? 0 : 1);
  return (uint32_t)a | ((uint32_t)b << 16);
}

__global__ void __launch_bounds__(256) convert_bf16_to_f16_kernel(const uint16_t* __restrict__ src,
                                                                  uint16_t* __restrict__ dst, int64_t n,
                                                                  int32_t* __restrict__ bad_count) {
  int bad = 0;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t n8 = n / 8;
  const uint4* s8 = reinterpret_cast<const uint4*>(src);
  uint4* d8 = reinterpret_cast<uint4*>(dst);
  for (int64_t i = tid; i < n8; i += stride) {
    const uint4 v = __ldg(s8 + i);
    d8[i] = make_uint4(bf16x2_to_f16x2(v.x, &bad), bf16x2_to_f16x2(v.y, &bad), bf16x2_to_f16x2(v.z, &bad),
                       bf16x2_to_f16x2(v.w, &bad));
  }
  for (int64_t i = n8 * 8 + tid; i < n; i += stride) {  // the last n % 8 values
    const uint16_t h = f32_to_f16(__uint_as_float((uint32_t)src[i] << 16));
    bad += f16_finite(h) ? 0 : 1;
    dst[i] = h;
  }
  for (int o = 16; o > 0; o >>= 1) bad += __shfl_xor_sync(0xffffffffu, bad, o);
  if ((threadIdx.x & 31) == 0 && bad != 0) atomicAdd(bad_count, bad);
}

}  // namespace

cudaError_t launch_convert_bf16_to_f16(const uint16_t* src, uint16_t* dst, int64_t n, int32_t* bad_count,
                                       cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(bad_count, 0, sizeof(int32_t), s);
  if (e != cudaSuccess || n == 0) return e;
  int64_t blocks = (n / 8 + 255) / 256;
  if (blocks < 1) blocks = 1;
  if (blocks > (int64_t)sm_count() * 4) blocks = (int64_t)sm_count() * 4;
  convert_bf16_to_f16_kernel<<<(unsigned)blocks, 256, 0, s>>>(src, dst, n, bad_count);
  after_launch(MOE_KERNEL_COUNT, s);  // no timer selects this id: only counts the launch
  return cudaGetLastError();
}

}  // namespace moe
