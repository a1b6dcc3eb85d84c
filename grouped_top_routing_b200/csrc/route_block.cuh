// Routing of 1-2 tokens by a whole thread block, for the fused decode kernels.
//
// Takes the same decisions as the per-token router kernel (route.cuh): the
// same fp64 score evaluation rounded once to fp32, the same softmax sum
// association, group scores from the multiset top-2 of each group, and the
// top-k by (biased score descending, expert id ascending), taken by one warp
// per token in k rounds of warp arg-max over unique 64-bit keys (order key of
// the biased score above the complemented id), which is exact for a total
// order. The block's warps share the per-expert passes (scores, groups, keys);
// the selection itself needs no block barrier. Pages: mlxcel issue
// #838 "add Ant Group Ling / Bailing MoE", section "Router: selection uses
// biased scores, weights come from unbiased scores", and the model card
// "Ling-2.6-flash-JANGTQ", paragraph "MoE routing".
#pragma once

#include "decode_fused.cuh"
#include "route.cuh"

namespace moe {
namespace block_route {

constexpr int kMaxT = 2;      // tokens
constexpr int kMaxSlots = 32;  // T * k: one warp lane per slot

// Shared-memory state of the routing of a block of W warps (the routing runs
// on the W warps that share named barrier 1); the results are idx .. n_act.
template <int W>
struct Smem {
  uint32_t gkey[kMaxT][32];             // group score keys
  uint32_t kept[kMaxT];                 // kept-group masks
  float red[kMaxT][W];
  double sum[kMaxT];
  int32_t idx[kMaxSlots];  // slot -> expert
  float w_raw[kMaxSlots];  // unbiased score of the slot's expert
  float w[kMaxSlots];      // routing weight
  int32_t act_e[kMaxSlots], act_a[kMaxSlots], act_b[kMaxSlots];  // distinct expert, first slot, second slot or -1
  int n_act;
};

// Dynamic shared memory the routing needs: [T*E] fp32 scores, [T*E] fp32
// biased scores, [T*E] 64-bit keys.
__host__ __device__ __forceinline__ size_t scratch_bytes(int T, int E) { return (size_t)T * E * 16; }

// Unique selection key: the order key of the biased score above the
// complemented expert id, so that a larger key is a higher score or, on a tie,
// a lower id. Real keys are > 0 (the order key of -inf is 0x007fffff).
__device__ __forceinline__ uint64_t sel_key(float s, int e) {
  return ((uint64_t)route_detail::order_key(s) << 32) | (uint64_t)(~(uint32_t)e);
}

// The k best of one token's E experts by one warp: lane l holds the keys of
// experts l + 32 r, with their unbiased scores; each of k rounds takes the
// warp's largest key (the high words first, then the low words among the lanes
// holding the largest high word: keys are unique, so the pair is the maximum)
// and its owner drops it. Round j yields slot j: biased score descending,
// expert id ascending. Lane 0 writes the slot's expert and unbiased score.
// kGlobal: key and orig were written in this launch by other CTAs (read
// through L2); else they are in shared memory.
template <int R, bool kGlobal>
__device__ __forceinline__ void topk_warp(const uint64_t* key, const float* orig, int E, int k, int32_t* idx,
                                          float* w_raw) {
  const int lane = threadIdx.x & 31;
  uint64_t mine[R];
  float mo[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int e = lane + 32 * r;
    mine[r] = 0ull;  // below every real key
    mo[r] = 0.f;
    if (e < E) {
      mine[r] = kGlobal ? __ldcg(reinterpret_cast<const unsigned long long*>(key) + e) : key[e];
      mo[r] = kGlobal ? __ldcg(orig + e) : orig[e];
    }
  }
  for (int j = 0; j < k; ++j) {
    uint64_t best = mine[0];
#pragma unroll
    for (int r = 1; r < R; ++r) best = mine[r] > best ? mine[r] : best;
    const uint32_t hi = (uint32_t)(best >> 32);
    const uint32_t mh = __reduce_max_sync(0xffffffffu, hi);
    const uint32_t ml = __reduce_max_sync(0xffffffffu, hi == mh ? (uint32_t)best : 0u);
    const uint64_t win = ((uint64_t)mh << 32) | ml;
    float wo = 0.f;
#pragma unroll
    for (int r = 0; r < R; ++r)
      if (mine[r] == win) {
        wo = mo[r];
        mine[r] = 0ull;
      }
    const int owner = __ffs(__ballot_sync(0xffffffffu, best == win)) - 1;
    wo = __shfl_sync(0xffffffffu, wo, owner);
    if (lane == 0) {
      idx[j] = (int)(~ml);
      w_raw[j] = wo;
    }
  }
}

// Whether the fused kernel stores each router logit's sigmoid score and
// selection key as it produces the logit (then the routing starts from them):
// sigmoid scores, no group selection, logits computed in this launch.
__device__ __forceinline__ bool scores_with_logits(const DecodeArgs& a) {
  return a.pre_key != nullptr && a.score_fn == MOE_SCORE_SIGMOID && !(a.n_group > 1 && a.topk_group < a.n_group) &&
         a.logits_override == nullptr;
}

// The unbiased score of logit L (fp64 evaluation rounded once to fp32, as the
// per-token router computes it) and the selection key of expert e of token t,
// stored for the routing. bias: the expert bias (any memory) or null.
__device__ __forceinline__ void store_score(const DecodeArgs& a, int t, int e, float L, const float* bias) {
  const float o = __double2float_rn(1.0 / (1.0 + exp(-(double)L)));
  a.pre_orig[t * a.E + e] = o;
  a.pre_key[t * a.E + e] = sel_key(bias != nullptr ? __fadd_rn(o, bias[e]) : o, e);
}

template <int W>
__device__ void route_block(const DecodeArgs& a, const float* logits, const float* bias, unsigned char* scratch,
                            Smem<W>& sm) {
  static_assert(W >= kMaxT, "route_block needs a warp per token");
  constexpr int kConsumerWarps = W, kConsumers = W * 32;
  auto consumer_sync = [] { asm volatile("bar.sync 1, %0;" ::"n"(kConsumers) : "memory"); };
  using namespace route_detail;
  const int T = a.T, E = a.E, k = a.k;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float* s_orig = reinterpret_cast<float*>(scratch);
  float* s_sel = s_orig + T * E;
  uint64_t* s_key = reinterpret_cast<uint64_t*>(s_sel + T * E);
  double* s_ex = reinterpret_cast<double*>(s_key);

  // With scores and keys stored along with the logits (scores_with_logits),
  // the selection starts from them; otherwise the block computes them here.
  const bool pre = scores_with_logits(a);
  if (!pre) {
    // ---- scores: fp64 evaluation, one rounding to fp32; selection copy with the bias ----
    if (a.score_fn != MOE_SCORE_SOFTMAX) {
      for (int t = 0; t < T; ++t)
        for (int e = threadIdx.x; e < E; e += kConsumers) {
          const float L = __ldcg(logits + (int64_t)t * E + e);
          const float o = __double2float_rn(1.0 / (1.0 + exp(-(double)L)));
          s_orig[t * E + e] = o;
          s_sel[t * E + e] = bias != nullptr ? __fadd_rn(o, bias[e]) : o;
        }
    } else {
      float m[kMaxT] = {-INFINITY, -INFINITY};
  #pragma unroll
      for (int t = 0; t < kMaxT; ++t)
        if (t < T)
          for (int e = threadIdx.x; e < E; e += kConsumers) {
            const float L = __ldcg(logits + (int64_t)t * E + e);
            s_orig[t * E + e] = L;
            m[t] = fmaxf(m[t], L);
          }
  #pragma unroll
      for (int t = 0; t < kMaxT; ++t) {
        const float mt = warp_max_f32(m[t]);
        if (lane == 0 && t < T) sm.red[t][warp] = mt;
      }
      consumer_sync();
      for (int t = 0; t < T; ++t) {
        float mt = sm.red[t][0];
        for (int w = 1; w < kConsumerWarps; ++w) mt = fmaxf(mt, sm.red[t][w]);
        const double md = (double)mt;
        for (int e = threadIdx.x; e < E; e += kConsumers) s_ex[t * E + e] = exp((double)s_orig[t * E + e] - md);
      }
      consumer_sync();
      if (warp < T) {
        // the per-token router's association: lane l sums experts l*P .. l*P+P-1
        int P = 1;
        while (P * 32 < E) P <<= 1;
        double sum = 0.0;
        for (int i = 0; i < P; ++i) {
          const int e = lane * P + i;
          if (e < E) sum += s_ex[warp * E + e];
        }
        sum = warp_sum_f64(sum);
        if (lane == 0) sm.sum[warp] = sum;
      }
      consumer_sync();
      for (int t = 0; t < T; ++t)
        for (int e = threadIdx.x; e < E; e += kConsumers) {
          const float o = __double2float_rn(s_ex[t * E + e] / sm.sum[t]);
          s_orig[t * E + e] = o;
          s_sel[t * E + e] = bias != nullptr ? __fadd_rn(o, bias[e]) : o;
        }
    }
    consumer_sync();

    // ---- groups: score = top1 + top2 of the group's biased scores; keep topk_group ----
    const bool grouped = a.n_group > 1 && a.topk_group < a.n_group;
    const int gsz = E / a.n_group;
    if (grouped) {
      for (int p = warp; p < T * a.n_group; p += kConsumerWarps) {
        const int t = p / a.n_group, g = p - t * a.n_group;
        const float* gv = s_sel + t * E + g * gsz;
        float top1 = -INFINITY, top2 = -INFINITY;  // NaN never enters: it fails both comparisons
        for (int i = lane; i < gsz; i += 32) {
          const float v = gv[i];
          if (v > top1) {
            top2 = top1;
            top1 = v;
          } else if (v > top2) {
            top2 = v;
          }
        }
  #pragma unroll
        for (int o = 16; o > 0; o >>= 1) {  // multiset top-2 of two lanes' pairs
          const float b1 = __shfl_xor_sync(0xffffffffu, top1, o), b2 = __shfl_xor_sync(0xffffffffu, top2, o);
          if (b1 > top1) {
            top2 = fmaxf(top1, b2);
            top1 = b1;
          } else {
            top2 = fmaxf(top2, b1);
          }
        }
        if (lane == 0) sm.gkey[t][g] = order_key(gsz == 1 ? top1 : __fadd_rn(top1, top2));
      }
      consumer_sync();
      if (warp < T) {
        const uint32_t gk = lane < a.n_group ? sm.gkey[warp][lane] : 0u;
        uint32_t kept = 0;
        for (int r = 0; r < a.topk_group; ++r) {
          const uint32_t key = ((kept >> lane) & 1u) ? 0u : gk;
          const uint32_t mx = __reduce_max_sync(0xffffffffu, key);
          const uint32_t win = __reduce_min_sync(0xffffffffu, key == mx ? (uint32_t)lane : 0xffffffffu);
          kept |= 1u << win;
        }
        if (lane == 0) sm.kept[warp] = kept;
      }
      consumer_sync();
    }

    // ---- selection keys (experts of dropped groups select as -inf) ----
    for (int t = 0; t < T; ++t) {
      const uint32_t kept = grouped ? sm.kept[t] : 0xffffffffu;
      for (int e = threadIdx.x; e < E; e += kConsumers) {
        const bool live = !grouped || ((kept >> (e / gsz)) & 1u);
        s_key[t * E + e] = sel_key(live ? s_sel[t * E + e] : -INFINITY, e);
      }
    }
    consumer_sync();
  }

  // ---- top-k of token t by warp t (E <= 1024: at most 32 keys per lane) ----
  if (warp < T) {
    const int t = warp;
    const int R = (E + 31) / 32;
    int32_t* idx = sm.idx + t * k;
    float* w_raw = sm.w_raw + t * k;
    if (pre) {
      const uint64_t* key = reinterpret_cast<const uint64_t*>(a.pre_key) + t * E;
      const float* orig = a.pre_orig + t * E;
      if (R <= 2) topk_warp<2, true>(key, orig, E, k, idx, w_raw);
      else if (R <= 4) topk_warp<4, true>(key, orig, E, k, idx, w_raw);
      else if (R <= 8) topk_warp<8, true>(key, orig, E, k, idx, w_raw);
      else if (R <= 16) topk_warp<16, true>(key, orig, E, k, idx, w_raw);
      else topk_warp<32, true>(key, orig, E, k, idx, w_raw);
    } else {
      const uint64_t* key = s_key + t * E;
      const float* orig = s_orig + t * E;
      if (R <= 2) topk_warp<2, false>(key, orig, E, k, idx, w_raw);
      else if (R <= 4) topk_warp<4, false>(key, orig, E, k, idx, w_raw);
      else if (R <= 8) topk_warp<8, false>(key, orig, E, k, idx, w_raw);
      else if (R <= 16) topk_warp<16, false>(key, orig, E, k, idx, w_raw);
      else topk_warp<32, false>(key, orig, E, k, idx, w_raw);
    }
    __syncwarp();
  }

  // ---- weights: renormalise (k > 1) with the 1e-20 epsilon, then scale; fp32, slot order ----
  if (warp < T) {
    const int t = warp;
    const bool do_norm = a.norm && k > 1;
    float den = 0.f;
    if (do_norm) {
      if (lane == 0) {
        den = sm.w_raw[t * k];
        for (int j = 1; j < k; ++j) den = __fadd_rn(den, sm.w_raw[t * k + j]);
        den = __fadd_rn(den, 1e-20f);
      }
      den = __shfl_sync(0xffffffffu, den, 0);
    }
    for (int j = lane; j < k; j += 32) {
      float w = sm.w_raw[t * k + j];
      if (do_norm) w = __fdiv_rn(w, den);
      sm.w[t * k + j] = __fmul_rn(w, a.scale);
    }
  }
  consumer_sync();

  // ---- distinct experts, in order of first slot, with the slot(s) holding each ----
  if (warp == 0) {
    const int ns = T * k;
    const int e = lane < ns ? sm.idx[lane] : (int)(0x40000000u | (uint32_t)lane);  // unique dummies
    const uint32_t same = __match_any_sync(0xffffffffu, e);
    const bool first = lane < ns && (__ffs(same) - 1) == lane;
    const uint32_t firsts = __ballot_sync(0xffffffffu, first);
    if (first) {
      const int pos = __popc(firsts & ((1u << lane) - 1u));
      const uint32_t other = same & ~(1u << lane);  // the other token's slot (ids are distinct per token)
      sm.act_e[pos] = e;
      sm.act_a[pos] = lane;
      sm.act_b[pos] = other != 0u ? __ffs(other) - 1 : -1;
    }
    if (lane == 0) sm.n_act = __popc(firsts);
    if (blockIdx.x == 0 && lane < ns) {
      if (a.topk_idx_out != nullptr) a.topk_idx_out[lane] = e;
      if (a.topk_w_out != nullptr) a.topk_w_out[lane] = sm.w[lane];
    }
  }
  consumer_sync();
}

}  // namespace block_route
}  // namespace moe
