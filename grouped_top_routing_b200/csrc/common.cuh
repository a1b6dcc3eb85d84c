// Shared device/host helpers of libmoe.so (sm_100a only).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "moe.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libmoe targets sm_100a only"
#endif

namespace moe {

// ---------------------------------------------------------------------------
// Workspace header: the first 256 bytes of every workspace.
// ---------------------------------------------------------------------------
struct WsHeader {
  int32_t error;        // first moe_status recorded on the device (0 = none)
  int32_t error_info;   // kernel-specific detail (offending index, wait site)
  int32_t num_active;   // number of experts with rows (written by permute)
  int32_t pad0[3];
  uint64_t bar_arrivals;  // grid barrier of the fused decode kernels: arrivals, only ever growing
  int32_t pad[56];
};
static_assert(sizeof(WsHeader) == 256, "header is 256 bytes");

__device__ __forceinline__ void record_error(WsHeader* h, int status, int info) {
  if (h == nullptr) return;
  if (atomicCAS(&h->error, 0, status) == 0) h->error_info = info;
}

// ---------------------------------------------------------------------------
// bf16 helpers (raw uint16 bits)
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// fp32 -> bf16, round to nearest even (NaN kept quiet).
__device__ __forceinline__ uint16_t f32_to_bf16(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u);
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return (uint32_t)f32_to_bf16(lo) | ((uint32_t)f32_to_bf16(hi) << 16);
}

// 16-byte streaming load that bypasses L1 allocation (weights are read once).
__device__ __forceinline__ uint4 ld_stream_u4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}
__device__ __forceinline__ uint4 ld_nc_u4(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

// fp32 -> fp16 bits, round to nearest even; and whether fp16 bits are finite.
__device__ __forceinline__ uint16_t f32_to_f16(float f) {
  uint16_t h;
  asm("cvt.rn.f16.f32 %0, %1;" : "=h"(h) : "f"(f));
  return h;
}
__device__ __forceinline__ bool f16_finite(uint16_t h) { return (h & 0x7C00u) != 0x7C00u; }

__device__ __forceinline__ float silu_f32(float z) { return z / (1.0f + expf(-z)); }

// Sum of the 8 products of one 16-byte bf16 weight chunk with 8 fp32 values.
__device__ __forceinline__ float dot8_bf16(uint4 w, const float* v, float acc) {
  acc = fmaf(bf16_lo(w.x), v[0], acc);
  acc = fmaf(bf16_hi(w.x), v[1], acc);
  acc = fmaf(bf16_lo(w.y), v[2], acc);
  acc = fmaf(bf16_hi(w.y), v[3], acc);
  acc = fmaf(bf16_lo(w.z), v[4], acc);
  acc = fmaf(bf16_hi(w.z), v[5], acc);
  acc = fmaf(bf16_lo(w.w), v[6], acc);
  acc = fmaf(bf16_hi(w.w), v[7], acc);
  return acc;
}
__device__ __forceinline__ void unpack8_bf16(uint4 v, float* o) {
  o[0] = bf16_lo(v.x); o[1] = bf16_hi(v.x); o[2] = bf16_lo(v.y); o[3] = bf16_hi(v.y);
  o[4] = bf16_lo(v.z); o[5] = bf16_hi(v.z); o[6] = bf16_lo(v.w); o[7] = bf16_hi(v.w);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch. Every kernel of this library is launched with
// programmatic stream serialization (launch_pdl), lets its successor be
// scheduled as soon as it starts (pdl_launch_dependents), and waits for its
// predecessor to complete, memory included (pdl_wait), before it reads
// anything an earlier launch wrote. Since every kernel waits, completion is
// transitive along the stream. Launch latency and prologues (barrier set-up,
// TMEM allocation) overlap the previous kernel's tail.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------------------
// Host-side launch bookkeeping (defined in moe_api.cu)
// ---------------------------------------------------------------------------
void before_launch(int kernel_id, cudaStream_t s);
void after_launch(int kernel_id, cudaStream_t s, int nkernels = 1);
int sm_count();
// Options of the entry point running on this thread (moe_options; defaults
// outside a call): the bound on device waits and the test aid.
uint64_t opt_wait_ns();
int opt_withhold();

}  // namespace moe
