// Router for one token, executed by one warp, and the helpers the fused
// decode kernel's block-wide router shares with it.
//
// Follows mlxcel issue #838 "add Ant Group Ling / Bailing MoE", section
// "Router: selection uses biased scores, weights come from unbiased scores"
// (score in fp32, bias on a copy used only for selection, weights gathered
// from the unbiased scores, renormalisation only when k > 1 with a 1e-20
// epsilon), section "moe_router_enable_routed_scaling is dead code upstream"
// (scaling always applied) and the model card "Ling-2.6-flash-JANGTQ",
// paragraph "MoE routing" (8 groups, top-4 groups, top-8 experts).
//
// Lane l holds experts l*P .. l*P+P-1 in registers (P = experts per lane, a
// power of two), so E <= 32*P. Every decision is a comparison of fp32 values
// through a total order key (value descending, expert id ascending), reduced
// across the warp with shuffles.
#pragma once

#include <math.h>

#include "common.cuh"

namespace moe {
namespace route_detail {

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

}  // namespace route_detail

// Routes the token whose fp32 gates are Lrow[0..E): writes idx_out[0..k) (expert
// ids, ordered by biased score descending then id ascending) and w_out[0..k)
// (routing weights). buf: this warp's 32*P floats of shared memory.
template <int P>
__device__ __forceinline__ void route_one_token(const float* __restrict__ Lrow, const float* __restrict__ bias, int E,
                                                int k, int n_group, int topk_group, int score_fn, int norm,
                                                float scale, float* buf, int32_t* idx_out, float* w_out) {
  using namespace route_detail;
  const int lane = threadIdx.x & 31;
  const bool grouped = n_group > 1 && topk_group < n_group;
  const int gsz = E / n_group;
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
      idx_out[j] = e;
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
    w_out[j] = __fmul_rn(w, scale);
  }
  __syncwarp();
}

}  // namespace moe
