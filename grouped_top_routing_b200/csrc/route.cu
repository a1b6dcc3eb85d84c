// Router: scores, selection-only bias, grouped top-k, expert top-k, weights.
//
// Follows mlxcel issue #838 "add Ant Group Ling / Bailing MoE", section
// "Router: selection uses biased scores, weights come from unbiased scores"
// (score in fp32, bias on a copy used only for selection, weights gathered
// from the unbiased scores, renormalisation only when k > 1 with a 1e-20
// epsilon), section "moe_router_enable_routed_scaling is dead code upstream"
// (scaling always applied) and the model card "Ling-2.6-flash-JANGTQ",
// paragraph "MoE routing" (8 groups, top-4 groups, top-8 experts).
//
// One warp per token. Lane l holds experts l*P .. l*P+P-1 in registers
// (P = experts per lane, a power of two), so E <= 32*P. Every decision is a
// comparison of fp32 values through a total order key (value descending,
// expert id ascending), reduced across the warp with shuffles.
#include <math.h>

#include "common.cuh"

namespace moe {

namespace {

constexpr uint32_t kKeyNegInf = 0x007fffffu;  // order key of -inf (and NaN)

// Monotone map of fp32 to uint32: larger float -> larger key. -0 == +0;
// NaN ranks with -inf. Key 0 is below every float (used for padding lanes).
__device__ __forceinline__ uint32_t order_key(float f) {
  if (f != f) return kKeyNegInf;
  if (f == 0.0f) f = 0.0f;
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Warp-wide arg-max of (key, ~id): every lane gets the winning pair.
__device__ __forceinline__ void warp_argmax(uint32_t& key, uint32_t& nid) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    uint32_t ok = __shfl_xor_sync(0xffffffffu, key, o);
    uint32_t on = __shfl_xor_sync(0xffffffffu, nid, o);
    if (ok > key || (ok == key && on > nid)) { key = ok; nid = on; }
  }
}

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max_f32(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

template <int P>
__global__ void __launch_bounds__(256) route_kernel(
    const float* __restrict__ logits, const float* __restrict__ bias, int T, int E, int k, int n_group,
    int topk_group, int score_fn, int norm, float scale, int32_t* __restrict__ idx_out,
    float* __restrict__ w_out) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ float smem[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int wpb = blockDim.x >> 5;
  float* buf = smem + warp * (32 * P);  // per-warp scratch: biased scores, then raw weights
  const bool grouped = n_group > 1 && topk_group < n_group;
  const int gsz = E / n_group;

  for (int t = blockIdx.x * wpb + warp; t < T; t += gridDim.x * wpb) {
    const float* Lrow = logits + (size_t)t * E;
    float L[P], orig[P], sel[P];
#pragma unroll
    for (int i = 0; i < P; ++i) {
      const int e = lane * P + i;
      L[i] = (e < E) ? __ldg(Lrow + e) : -INFINITY;
    }

    // ---- score function: fp64 evaluation, one rounding to fp32 ----
    if (score_fn == MOE_SCORE_SOFTMAX) {
      float m = -INFINITY;
#pragma unroll
      for (int i = 0; i < P; ++i) m = fmaxf(m, L[i]);
      m = warp_max_f32(m);
      const double md = (double)m;
      double sum = 0.0;
#pragma unroll
      for (int i = 0; i < P; ++i)
        if (lane * P + i < E) sum += exp((double)L[i] - md);
      sum = warp_sum_f64(sum);
#pragma unroll
      for (int i = 0; i < P; ++i) orig[i] = __double2float_rn(exp((double)L[i] - md) / sum);
    } else {
#pragma unroll
      for (int i = 0; i < P; ++i) orig[i] = __double2float_rn(1.0 / (1.0 + exp(-(double)L[i])));
    }

    // ---- selection copy with the bias (fp32 add) ----
#pragma unroll
    for (int i = 0; i < P; ++i) {
      const int e = lane * P + i;
      float s = orig[i];
      if (bias != nullptr && e < E) s = __fadd_rn(s, __ldg(bias + e));
      sel[i] = s;
    }

    // ---- grouped top-k: group score = top1 + top2, keep topk_group groups ----
    if (grouped) {
#pragma unroll
      for (int i = 0; i < P; ++i)
        if (lane * P + i < E) buf[lane * P + i] = sel[i];
      __syncwarp();
      uint32_t gkey = 0, gnid = 0;
      if (lane < n_group) {
        float top1 = -INFINITY, top2 = -INFINITY;
        const float* g = buf + lane * gsz;
        for (int i = 0; i < gsz; ++i) {
          const float v = g[i];
          if (v > top1) { top2 = top1; top1 = v; }
          else if (v > top2) { top2 = v; }
        }
        const float gs = (gsz == 1) ? top1 : __fadd_rn(top1, top2);
        gkey = order_key(gs);
        gnid = ~(uint32_t)lane;
      }
      uint32_t kept = 0;
      for (int r = 0; r < topk_group; ++r) {
        uint32_t key = (kept >> lane) & 1u ? 0u : gkey;
        uint32_t nid = gnid;
        warp_argmax(key, nid);
        kept |= 1u << (~nid);
      }
#pragma unroll
      for (int i = 0; i < P; ++i) {
        const int e = lane * P + i;
        if (e < E && !((kept >> (e / gsz)) & 1u)) sel[i] = -INFINITY;
      }
      __syncwarp();
    }

    // ---- expert top-k: k rounds of warp arg-max on (sel desc, id asc) ----
    uint32_t skey[P];
#pragma unroll
    for (int i = 0; i < P; ++i) skey[i] = (lane * P + i < E) ? order_key(sel[i]) : 0u;
    uint32_t taken = 0;
    for (int j = 0; j < k; ++j) {
      uint32_t key = 0, nid = 0;
      float my_orig = 0.0f;
#pragma unroll
      for (int i = 0; i < P; ++i) {
        const int e = lane * P + i;
        if (e < E && !((taken >> i) & 1u)) {
          const uint32_t kk = skey[i];
          const uint32_t nn = ~(uint32_t)e;
          if (kk > key || (kk == key && nn > nid)) { key = kk; nid = nn; my_orig = orig[i]; }
        }
      }
      const float mine = my_orig;
      warp_argmax(key, nid);
      const int e = (int)(~nid);
      const int owner = e / P;
      const float w_raw = __shfl_sync(0xffffffffu, mine, owner);
      if (lane == owner) taken |= 1u << (e - owner * P);
      if (lane == 0) {
        idx_out[(size_t)t * k + j] = e;
        buf[j] = w_raw;
      }
    }
    __syncwarp();

    // ---- weights: renormalise (k > 1), then scale; fp32, slot order ----
    float den = 0.0f;
    const bool do_norm = norm && k > 1;
    if (do_norm) {
      if (lane == 0) {
        den = buf[0];
        for (int j = 1; j < k; ++j) den = __fadd_rn(den, buf[j]);
        den = __fadd_rn(den, 1e-20f);
      }
      den = __shfl_sync(0xffffffffu, den, 0);
    }
    for (int j = lane; j < k; j += 32) {
      float w = buf[j];
      if (do_norm) w = __fdiv_rn(w, den);
      w_out[(size_t)t * k + j] = __fmul_rn(w, scale);
    }
    __syncwarp();
  }
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
