// Fused decode: the whole MoE block for up to 8 tokens in one persistent launch.
//
// At decode the block is bound by reading weights: the router projection, the
// shared MLP and only the experts the router picked (page "Ling-3.0-flash-GGUF",
// section "Measured performance": a decode step reads just the chosen
// experts). The kernel is a weight-streaming engine over all SMs: one CTA per
// SM, fifteen worker warps that stream weights with 16-byte loads straight
// into registers and multiply them on the tensor cores (mma.sync m16n8k16,
// bf16 in, fp32 sums; the n = 8 columns are the tokens), and one scheduler
// warp that hands the CTA its next unit of work from a queue shared by all
// CTAs.
//
// Units, in queue order (a CTA draws them in increasing order):
//   router  : rpu rows of the fp32 router projection, split over the warps by
//             columns; the reduction writes logits[t][e] (CUDA-core FMAs).
//   shared gate/up, then the routing unit, then shared down: the shared MLP
//             does not depend on the routing (mlxcel issue #838, section
//             "Shared experts are one wide MLP, not N separate experts"), so it
//             streams while the router rows finish and the routing runs.
//   route   : one CTA routes every token (the router of route.cuh, one warp per
//             token, bit-identical to moe_route) once all logits are written,
//             and publishes the distinct experts and their per-token weights.
//   routed gate/up: 8 gate rows + the matching 8 up rows of one expert over the
//             whole hidden size, split over the worker warps by columns; the
//             reduction applies SwiGLU, multiplies by each token's routing
//             weight and stores w*h as two bf16 planes (hi, lo).
//   routed down: 16*rgd output rows of one expert, each row group's columns
//             split over ksd warps; the reduction writes the expert's weighted
//             fp32 output rows. The last of a 16-row block's contributions sums
//             them in a fixed order (routed experts by id, then the shared
//             MLP) and writes y once, rounded to bf16.
//
// Per unit, each warp: consume its registers (loaded during the previous
// unit), write its partial sums to shared memory, then load the next unit's
// weights before the CTA-wide hand-over, so the loads are in flight while the
// rotating reducer warp folds the partials. Dependencies between CTAs are
// counters (release/acquire) polled by the scheduler warp, which holds back a
// unit's descriptor until what it reads is complete; nothing waits on a grid
// barrier.
//
// Every wait is bounded (moe_options.wait_limit_ns). One that runs out records
// MOE_ERR_TIMEOUT, raises an abort word that every scheduler checks, and the
// kernel winds down: schedulers hand out no more units, workers finish the
// unit in hand. The last CTA to leave restores the counters to zero.
#include "common.cuh"
#include "decode.cuh"
#include "mbarrier.cuh"
#include "route.cuh"

namespace moe {

namespace {

constexpr int kWorkers = 15;  // + 1 scheduler warp: 16 warps, 128 registers a thread
constexpr int kThreads = (kWorkers + 1) * 32;
constexpr int kMaxT = kDecodeMaxT;
constexpr int kMaxSlots = kDecodeMaxSlots;
constexpr int kStageChunks = 9;    // 32-column chunks per warp per register stage (gate/up, down)
constexpr int kStagePieces = 16;   // 128-float pieces per warp per register stage (router)
constexpr int kRedFloats = kWorkers * 32 * 4;  // one partial buffer: a warp's 32 lanes x 4 sums

enum : int { kDone = 0, kRouter = 1, kGateUp = 2, kDown = 3, kRoute = 4 };

// sync words (int32), zero at launch
enum : int { kHead = 0, kRouterDone = 1, kRouteFlag = 2, kExit = 3, kAbort = 4, kGuDone = 8,
             kRowBlocks = 8 + kMaxSlots };

struct Desc {
  int kind, slot, block, pad;
};

struct Geo {
  int xs_stride, hs_stride;         // bytes per smem row of x / of staged w*h
  int rpu, ks_r, np_r, nr;          // router: rows per unit, warps per row, pieces per warp, units
  int gu_cpw, gu_units_r, gu_units_s;
  int dn_ksd_r, dn_rgd_r, dn_cpw_r, dn_units_r;
  int dn_ksd_s, dn_rgd_s, dn_cpw_s, dn_units_s;
  int P;                            // experts per lane in the router (power of two)
  int off_hb, off_red, off_misc;    // smem offsets
  int smem;
};

// smem misc block
struct Misc {
  uint64_t desc_full[2], desc_empty[2], bar_e[2], bar_a, pad_bar;
  Desc desc[2];
  int32_t U, have_route, last, pad;
  int32_t expert[kMaxSlots];
  float wt[kMaxSlots][kMaxT];
  int32_t r_idx[kMaxT][64];
  float r_w[kMaxT][64];
  uint32_t mask[32];
  int32_t base[32];
};

// ---------------------------------------------------------------------------
// device helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ int ld_acquire(const int32_t* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release(int32_t* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ int ld_volatile(const int32_t* p) { return *reinterpret_cast<const volatile int32_t*>(p); }

// Records a timeout and raises the abort word that every scheduler reads.
__device__ __forceinline__ void fail_timeout(const DecodeArgs& a, int site) {
  record_error(a.hdr, MOE_ERR_TIMEOUT, site);
  atomicExch(a.sync + kAbort, 1);
}

// Bounded wait of one thread for an mbarrier phase.
__device__ __forceinline__ bool wait_phase(uint64_t* bar, uint32_t parity, uint64_t limit) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer() - t0 > limit) return false;
  return true;
}

// Bounded wait of one thread until *p >= target (acquire). False on timeout
// or when the launch is aborting.
__device__ __forceinline__ bool wait_count(const DecodeArgs& a, const int32_t* p, int target, int site) {
  if (ld_acquire(p) >= target) return true;
  const uint64_t t0 = globaltimer();
  for (;;) {
    __nanosleep(64);
    if (ld_acquire(p) >= target) return true;
    if (ld_volatile(a.sync + kAbort)) return false;
    if (globaltimer() - t0 > a.wait_ns) {
      fail_timeout(a, site);
      return false;
    }
  }
}

__device__ __forceinline__ void mma16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 lds128(const uint8_t* p) { return *reinterpret_cast<const uint4*>(p); }

// Unit decoding shared by the scheduler and the workers: the row set of a
// gate/up or down unit.
struct UnitRows {
  const uint16_t* w;  // weight matrix base
  int64_t row0;       // first row of the unit's first row group (gate rows for gate/up)
  int64_t row_up;     // gate/up: first up row
  int K;              // row length
};

__device__ __forceinline__ UnitRows gu_rows(const DecodeArgs& a, const Misc& ms, const Desc& d) {
  UnitRows r;
  r.K = a.H;
  if (d.slot == 0) {
    r.w = a.ws_gate_up;
    r.row0 = (int64_t)d.block * 8;
    r.row_up = a.Is + (int64_t)d.block * 8;
  } else {
    const int64_t e = ms.expert[d.slot];
    r.w = a.w_gate_up;
    r.row0 = e * 2 * a.I + (int64_t)d.block * 8;
    r.row_up = r.row0 + a.I;
  }
  return r;
}

// ---------------------------------------------------------------------------
// worker stages: issue the loads of a unit, consume them
// ---------------------------------------------------------------------------
struct Regs {
  uint4 v[2 * kStageChunks > kStagePieces ? 2 * kStageChunks : kStagePieces];
};

// Loads of stage `st` of the warp's share of unit d into r.
__device__ __forceinline__ void issue(const DecodeArgs& a, const Geo& g, const Misc& ms, const Desc& d, int warp,
                                      int lane, int st, Regs& r) {
  const int gq = lane >> 2, tig = lane & 3;
  if (d.kind == kRouter) {
    const int row = d.block * g.rpu + warp / g.ks_r;
    const int ks = warp % g.ks_r;
    if (warp / g.ks_r >= g.rpu || row >= a.E) return;
    const float* base = a.router_w + (int64_t)row * a.H + lane * 4;
    const int npieces = a.H / 128;
#pragma unroll
    for (int j = 0; j < kStagePieces; ++j) {
      const int p = ks + g.ks_r * (st * kStagePieces + j);
      if (st * kStagePieces + j < g.np_r && p < npieces) r.v[j] = ld_stream_u4(base + (int64_t)p * 128);
    }
  } else if (d.kind == kGateUp) {
    const UnitRows ur = gu_rows(a, ms, d);
    const int nch = a.H / 32;
    const uint16_t* pg = ur.w + (ur.row0 + gq) * ur.K + tig * 8;
    const uint16_t* pu = ur.w + (ur.row_up + gq) * ur.K + tig * 8;
#pragma unroll
    for (int j = 0; j < kStageChunks; ++j) {
      const int c = warp + kWorkers * (st * kStageChunks + j);  // chunks dealt round-robin over the warps
      if (c < nch && st * kStageChunks + j < g.gu_cpw) {
        r.v[2 * j] = ld_stream_u4(pg + c * 32);
        r.v[2 * j + 1] = ld_stream_u4(pu + c * 32);
      }
    }
  } else if (d.kind == kDown) {
    const bool sh = d.slot == 0;
    const int K = sh ? a.Is : a.I;
    const int ksd = sh ? g.dn_ksd_s : g.dn_ksd_r, rgd = sh ? g.dn_rgd_s : g.dn_rgd_r;
    const int cpw = sh ? g.dn_cpw_s : g.dn_cpw_r;
    const int rg = warp / ksd, ks = warp % ksd;
    const int n0 = (d.block * rgd + rg) * 16;
    if (rg >= rgd || n0 >= a.H) return;
    const uint16_t* w = sh ? a.ws_down : a.w_down + (int64_t)ms.expert[d.slot] * a.H * a.I;
    const uint16_t* p0 = w + (int64_t)(n0 + gq) * K + tig * 8;
    const uint16_t* p1 = p0 + (int64_t)8 * K;
    const int nch = K / 32;
#pragma unroll
    for (int j = 0; j < kStageChunks; ++j) {
      const int c = ks + ksd * (st * kStageChunks + j);  // chunks dealt round-robin over the row group's warps
      if (c < nch && st * kStageChunks + j < cpw) {
        r.v[2 * j] = ld_stream_u4(p0 + c * 32);
        r.v[2 * j + 1] = ld_stream_u4(p1 + c * 32);
      }
    }
  }
}

__device__ __forceinline__ int stages_of(const DecodeArgs& a, const Geo& g, const Desc& d) {
  if (d.kind == kRouter) return (g.np_r + kStagePieces - 1) / kStagePieces;
  if (d.kind == kGateUp) return (g.gu_cpw + kStageChunks - 1) / kStageChunks;
  if (d.kind == kDown) {
    const int cpw = d.slot == 0 ? g.dn_cpw_s : g.dn_cpw_r;
    return (cpw + kStageChunks - 1) / kStageChunks;
  }
  return 0;
}

// Consumes stage st of unit d from r into the running sums.
__device__ __forceinline__ void consume(const DecodeArgs& a, const Geo& g, const Desc& d, int warp, int lane, int st,
                                        const Regs& r, const uint8_t* xs, const uint8_t* hb, float* acc) {
  const int gq = lane >> 2, tig = lane & 3;
  if (d.kind == kRouter) {
    const int row = d.block * g.rpu + warp / g.ks_r;
    const int ks = warp % g.ks_r;
    if (warp / g.ks_r >= g.rpu || row >= a.E) return;
    const int npieces = a.H / 128;
#pragma unroll
    for (int j = 0; j < kStagePieces; ++j) {
      const int p = ks + g.ks_r * (st * kStagePieces + j);
      if (st * kStagePieces + j < g.np_r && p < npieces) {
        const float4 w4 = *reinterpret_cast<const float4*>(&r.v[j]);
        const int col = p * 128 + lane * 4;
#pragma unroll
        for (int t = 0; t < kMaxT; ++t) {
          const uint2 xv = *reinterpret_cast<const uint2*>(xs + t * g.xs_stride + col * 2);
          float s = acc[t];
          s = fmaf(w4.x, bf16_lo(xv.x), s);
          s = fmaf(w4.y, bf16_hi(xv.x), s);
          s = fmaf(w4.z, bf16_lo(xv.y), s);
          s = fmaf(w4.w, bf16_hi(xv.y), s);
          acc[t] = s;
        }
      }
    }
  } else if (d.kind == kGateUp) {
    const int nch = a.H / 32;
    const uint8_t* xrow = xs + gq * g.xs_stride + tig * 16;
#pragma unroll
    for (int j = 0; j < kStageChunks; ++j) {
      const int c = warp + kWorkers * (st * kStageChunks + j);
      if (c < nch && st * kStageChunks + j < g.gu_cpw) {
        const uint4 wg = r.v[2 * j], wu = r.v[2 * j + 1];
        const uint4 b = lds128(xrow + c * 64);
        mma16816(acc, wg.x, wu.x, wg.y, wu.y, b.x, b.y);
        mma16816(acc, wg.z, wu.z, wg.w, wu.w, b.z, b.w);
      }
    }
  } else if (d.kind == kDown) {
    const bool sh = d.slot == 0;
    const int K = sh ? a.Is : a.I;
    const int ksd = sh ? g.dn_ksd_s : g.dn_ksd_r, rgd = sh ? g.dn_rgd_s : g.dn_rgd_r;
    const int cpw = sh ? g.dn_cpw_s : g.dn_cpw_r;
    const int rg = warp / ksd, ks = warp % ksd;
    if (rg >= rgd || (d.block * rgd + rg) * 16 >= a.H) return;
    const int nch = K / 32;
    const uint8_t* hrow = hb + gq * g.hs_stride + tig * 16;
    const uint8_t* lrow = hrow + 8 * g.hs_stride;
#pragma unroll
    for (int j = 0; j < kStageChunks; ++j) {
      const int c = ks + ksd * (st * kStageChunks + j);
      if (c < nch && st * kStageChunks + j < cpw) {
        const uint4 w0 = r.v[2 * j], w1 = r.v[2 * j + 1];
        const uint4 bh = lds128(hrow + c * 64);
        const uint4 bl = lds128(lrow + c * 64);
        mma16816(acc, w0.x, w1.x, w0.y, w1.y, bh.x, bh.y);
        mma16816(acc, w0.x, w1.x, w0.y, w1.y, bl.x, bl.y);
        mma16816(acc, w0.z, w1.z, w0.w, w1.w, bh.z, bh.w);
        mma16816(acc, w0.z, w1.z, w0.w, w1.w, bl.z, bl.w);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// reductions (by the unit's reducer warp)
// ---------------------------------------------------------------------------
template <int P>
__device__ __noinline__ void route_token(const DecodeArgs& a, float* scratch, int t, Misc& ms) {
  const int lane = threadIdx.x & 31;
  float* lrow = scratch;           // 32 * P gates
  float* buf = scratch + 32 * P;   // route_one_token's own scratch
  for (int e = lane; e < 32 * P; e += 32) {
    float v = -INFINITY;
    if (e < a.E)
      v = a.logits_override != nullptr ? __ldg(a.logits_override + (int64_t)t * a.E + e)
                                       : __ldcg(a.logits + (int64_t)t * a.E + e);
    lrow[e] = v;
  }
  __syncwarp();
  route_one_token<P, false>(lrow, a.expert_bias, a.E, a.k, a.n_group, a.topk_group, a.score_fn, a.norm, a.scale, buf,
                            ms.r_idx[t], ms.r_w[t]);
  __syncwarp();
  for (int j = lane; j < a.k; j += 32) {
    if (a.topk_idx_out != nullptr) a.topk_idx_out[(int64_t)t * a.k + j] = ms.r_idx[t][j];
    if (a.topk_w_out != nullptr) a.topk_w_out[(int64_t)t * a.k + j] = ms.r_w[t][j];
  }
}

__device__ void route_unit(const DecodeArgs& a, const Geo& g, float* scratch, int warp, Misc& ms) {
  if (warp >= a.T) return;
  float* s = scratch + warp * 64 * g.P;
  switch (g.P) {
    case 1: route_token<1>(a, s, warp, ms); break;
    case 2: route_token<2>(a, s, warp, ms); break;
    case 4: route_token<4>(a, s, warp, ms); break;
    case 8: route_token<8>(a, s, warp, ms); break;
    default: route_token<16>(a, s, warp, ms); break;
  }
}

// The distinct experts of all tokens (slots 1..U, ascending id) and each
// token's weight per slot; published for every CTA with a release store.
__device__ void publish_route(const DecodeArgs& a, Misc& ms) {
  const int lane = threadIdx.x & 31;
  ms.mask[lane] = 0u;
  __syncwarp();
  const int n = a.T * a.k;
  for (int i = lane; i < n; i += 32) {
    const int e = ms.r_idx[i / a.k][i % a.k];
    atomicOr(&ms.mask[e >> 5], 1u << (e & 31));
  }
  __syncwarp();
  const uint32_t word = ms.mask[lane];
  const int cnt = __popc(word);
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const int U = __shfl_sync(0xffffffffu, incl, 31);
  ms.base[lane] = incl - cnt;
  DecodeRoute* rt = a.route;
  {
    uint32_t wv = word;
    int r = 0;
    while (wv) {
      const int b = __ffs(wv) - 1;
      wv &= wv - 1;
      rt->expert[1 + incl - cnt + r] = lane * 32 + b;
      ++r;
    }
  }
  for (int i = lane; i < (U + 1) * kMaxT; i += 32) rt->wt[i / kMaxT][i % kMaxT] = i < kMaxT ? 1.0f : 0.0f;
  __syncwarp();
  for (int i = lane; i < n; i += 32) {
    const int t = i / a.k, j = i % a.k;
    const int e = ms.r_idx[t][j];
    const uint32_t wrd = ms.mask[e >> 5];
    const int slot = 1 + ms.base[e >> 5] + __popc(wrd & ((1u << (e & 31)) - 1u));
    rt->wt[slot][t] = ms.r_w[t][j];
  }
  if (lane == 0) rt->U = U;
  __threadfence();
  __syncwarp();
  if (lane == 0 && !a.withhold) st_release(a.sync + kRouteFlag, 1);
}

// Sum of the slots' weighted rows for one 16-row block: routed experts in
// ascending id, then the shared MLP; one bf16 rounding.
__device__ void combine_block(const DecodeArgs& a, int blk, int U) {
  const int lane = threadIdx.x & 31;
  for (int i = lane; i < 16 * kMaxT; i += 32) {
    const int r = i / kMaxT, t = i % kMaxT;
    const int n = blk * 16 + r;
    if (t >= a.T || n >= a.H) continue;
    float acc = 0.0f;
    for (int s = 1; s <= U; ++s) acc += __ldcg(a.part + ((int64_t)s * a.H + n) * kMaxT + t);
    if (a.ws_down != nullptr) acc += __ldcg(a.part + (int64_t)n * kMaxT + t);
    a.y[(int64_t)t * a.H + n] = f32_to_bf16(acc);
  }
}

__device__ void reduce_unit(const DecodeArgs& a, const Geo& g, const Desc& d, const float* red, Misc& ms) {
  const int lane = threadIdx.x & 31;
  const int gq = lane >> 2, tig = lane & 3;
  if (d.kind == kRouter) {
    for (int i = lane; i < g.rpu * kMaxT; i += 32) {
      const int rr = i / kMaxT, t = i % kMaxT;
      const int row = d.block * g.rpu + rr;
      if (row >= a.E || t >= a.T) continue;
      float v = 0.0f;
      for (int ks = 0; ks < g.ks_r; ++ks) v += red[(rr * g.ks_r + ks) * 128 + t];
      a.logits[(int64_t)t * a.E + row] = v;
    }
    __threadfence();
    __syncwarp();
    if (lane == 0) atomicAdd(a.sync + kRouterDone, 1);
  } else if (d.kind == kGateUp) {
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    for (int w = 0; w < kWorkers; ++w) {
      const float4 p = *reinterpret_cast<const float4*>(red + w * 128 + lane * 4);
      v[0] += p.x;
      v[1] += p.y;
      v[2] += p.z;
      v[3] += p.w;
    }
    // v[0..1]: gate row i, tokens 2tig, 2tig+1; v[2..3]: the matching up row
    const int Kmax = a.I > a.Is ? a.I : a.Is;
    uint16_t* hb = a.hbuf + (int64_t)d.slot * 16 * Kmax;
    const int i = d.block * 8 + gq;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int t = 2 * tig + c;
      const float h = silu_f32(v[c]) * v[2 + c];
      const float p = ms.wt[d.slot][t] * h;
      const uint16_t hi = f32_to_bf16(p);
      const uint16_t lo = f32_to_bf16(p - __uint_as_float((uint32_t)hi << 16));
      hb[(int64_t)t * Kmax + i] = hi;
      hb[(int64_t)(8 + t) * Kmax + i] = lo;
    }
    __threadfence();
    __syncwarp();
    if (lane == 0) atomicAdd(a.sync + kGuDone + d.slot, 1);
  } else if (d.kind == kDown) {
    const bool sh = d.slot == 0;
    const int ksd = sh ? g.dn_ksd_s : g.dn_ksd_r, rgd = sh ? g.dn_rgd_s : g.dn_rgd_r;
    // the number of contributions per row block: routed experts (+ shared)
    int nslots;
    if (!sh) {
      nslots = ms.U + (a.ws_down != nullptr ? 1 : 0);
    } else {
      const int flag = ld_acquire(a.sync + kRouteFlag);
      nslots = flag ? __ldcg(&a.route->U) + 1 : 1 << 30;  // routing unknown: no routed row has arrived
    }
    for (int rg = 0; rg < rgd; ++rg) {
      const int n0 = (d.block * rgd + rg) * 16;
      if (n0 >= a.H) break;
      float v[4] = {0.f, 0.f, 0.f, 0.f};
      for (int ks = 0; ks < ksd; ++ks) {
        const float4 p = *reinterpret_cast<const float4*>(red + (rg * ksd + ks) * 128 + lane * 4);
        v[0] += p.x;
        v[1] += p.y;
        v[2] += p.z;
        v[3] += p.w;
      }
      float* prow = a.part + ((int64_t)d.slot * a.H + n0) * kMaxT;
      // rows gq and gq + 8, tokens 2tig and 2tig + 1
      *reinterpret_cast<float2*>(prow + gq * kMaxT + 2 * tig) = make_float2(v[0], v[1]);
      *reinterpret_cast<float2*>(prow + (gq + 8) * kMaxT + 2 * tig) = make_float2(v[2], v[3]);
      __threadfence();
      __syncwarp();
      int last = 0;
      if (lane == 0) last = atomicAdd(a.sync + kRowBlocks + n0 / 16, 1) + 1 == nslots;
      last = __shfl_sync(0xffffffffu, last, 0);
      if (last) {
        __threadfence();
        const int U = nslots - (a.ws_down != nullptr ? 1 : 0);
        combine_block(a, n0 / 16, U);
      }
    }
  } else if (d.kind == kRoute) {
    publish_route(a, ms);
  }
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1) decode_stream_kernel(const DecodeArgs a, const Geo g) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* xs = smem;
  uint8_t* hb = smem + g.off_hb;
  float* red = reinterpret_cast<float*>(smem + g.off_red);
  Misc& ms = *reinterpret_cast<Misc*>(smem + g.off_misc);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t worker_limit = 4 * a.wait_ns + 1000000ull;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ms.desc_full[i], 1);
      mbar_init(&ms.desc_empty[i], kWorkers);
      mbar_init(&ms.bar_e[i], kWorkers);
    }
    mbar_init(&ms.bar_a, kWorkers);
    ms.last = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kWorkers) {
    // shared MLP slot: weight 1 for every token
    for (int t = lane; t < kMaxT; t += 32) ms.wt[0][t] = 1.0f;
    if (lane == 0) {
      ms.expert[0] = -1;
      ms.have_route = 0;
      ms.U = 0;
    }
  } else {
    // x into shared memory as bf16 rows (rows T..7 zero: the mma's unused columns)
    const int per_row = a.H / 8;
    for (int i = threadIdx.x; i < kMaxT * per_row; i += kWorkers * 32) {
      const int t = i / per_row, c8 = i - t * per_row;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (t < a.T) v = __ldg(reinterpret_cast<const uint4*>(a.x + (int64_t)t * a.H) + c8);
      *reinterpret_cast<uint4*>(xs + t * g.xs_stride + c8 * 16) = v;
    }
  }
  __syncthreads();

  const int NR = a.logits_override != nullptr ? 0 : g.nr;
  const bool has_shared = a.ws_gate_up != nullptr;
  const int SGU = has_shared ? g.gu_units_s : 0;
  const int SDN = has_shared ? g.dn_units_s : 0;
  const int pre = NR + SGU + 1 + SDN;

  if (warp == kWorkers) {
    // ============================ scheduler ============================
    for (int m = 0;; ++m) {
      const int s = m & 1;
      Desc d{kDone, 0, 0, 0};
      bool ok = true;
      if (lane == 0) {
        if (!wait_phase(&ms.desc_empty[s], (uint32_t)((m >> 1) & 1) ^ 1u, worker_limit)) {
          fail_timeout(a, 40);
          ok = false;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      int j = 0;
      if (lane == 0 && ok && !ld_volatile(a.sync + kAbort)) j = atomicAdd(a.sync + kHead, 1);
      else if (lane == 0) j = -1;
      j = __shfl_sync(0xffffffffu, j, 0);
      if (j >= 0) {
        if (j < NR) {
          d = Desc{kRouter, 0, j, 0};
        } else if (j < NR + SGU) {
          d = Desc{kGateUp, 0, j - NR, 0};
        } else if (j == NR + SGU) {
          int r = 1;
          if (lane == 0) r = wait_count(a, a.sync + kRouterDone, NR, 41) ? 1 : 0;
          r = __shfl_sync(0xffffffffu, r, 0);
          d = r ? Desc{kRoute, 0, 0, 0} : Desc{kDone, 0, 0, 0};
        } else if (j < pre) {
          int r = 1;
          if (lane == 0) r = wait_count(a, a.sync + kGuDone, SGU, 42) ? 1 : 0;
          r = __shfl_sync(0xffffffffu, r, 0);
          d = r ? Desc{kDown, 0, j - (NR + SGU + 1), 0} : Desc{kDone, 0, 0, 0};
        } else {
          int r = 1;
          if (!ms.have_route) {
            if (lane == 0) r = wait_count(a, a.sync + kRouteFlag, 1, 43) ? 1 : 0;
            r = __shfl_sync(0xffffffffu, r, 0);
            if (r) {
              const int U = __ldcg(&a.route->U);
              for (int i = 1 + lane; i <= U; i += 32) ms.expert[i] = __ldcg(&a.route->expert[i]);
              for (int i = kMaxT + lane; i < (U + 1) * kMaxT; i += 32)
                ms.wt[i / kMaxT][i % kMaxT] = __ldcg(&a.route->wt[i / kMaxT][i % kMaxT]);
              if (lane == 0) {
                ms.U = U;
                ms.have_route = 1;
              }
              __syncwarp();
            }
          }
          if (r) {
            const int U = ms.U;
            const int jj = j - pre;
            if (jj < U * g.gu_units_r) {
              d = Desc{kGateUp, 1 + jj / g.gu_units_r, jj % g.gu_units_r, 0};
            } else if (jj < U * (g.gu_units_r + g.dn_units_r)) {
              const int q = jj - U * g.gu_units_r;
              const int slot = 1 + q / g.dn_units_r;
              if (lane == 0) r = wait_count(a, a.sync + kGuDone + slot, g.gu_units_r, 44) ? 1 : 0;
              r = __shfl_sync(0xffffffffu, r, 0);
              if (r) d = Desc{kDown, slot, q % g.dn_units_r, 0};
            }
          }
        }
      }
      if (lane == 0) {
        ms.desc[s] = d;
        mbar_arrive(&ms.desc_full[s]);
      }
      if (d.kind == kDone) break;
    }
  } else {
    // ============================= workers =============================
    Regs r;
    Desc cur, prev{kDone, 0, 0, 0};
    bool ok = true;
    // the first unit's descriptor and loads
    {
      int got = 1;
      if (lane == 0) got = wait_phase(&ms.desc_full[0], 0u, worker_limit) ? 1 : 0;
      got = __shfl_sync(0xffffffffu, got, 0);
      __syncwarp();
      if (!got) {
        if (lane == 0) fail_timeout(a, 50);
        cur = Desc{kDone, 0, 0, 0};
      } else {
        cur = ms.desc[0];
      }
    }
    bool issued = false;
    if (cur.kind != kDone) {
      issue(a, g, ms, cur, warp, lane, 0, r);
      issued = true;
    }
    int n_down = 0;  // down units seen (phase of bar_a)
    for (int m = 0;; ++m) {
      const int s = m & 1;
      // (1) the previous unit's reduction, by its reducer
      if (m > 0 && prev.kind != kDone && warp == (m - 1) % kWorkers)
        reduce_unit(a, g, prev, red + ((m - 1) & 1) * kRedFloats, ms);
      if (cur.kind == kDone) break;
      // (2) loads of this unit, if the descriptor was not ready earlier
      if (!issued) {
        int got = 1;
        if (lane == 0) got = wait_phase(&ms.desc_full[s], (uint32_t)((m >> 1) & 1), worker_limit) ? 1 : 0;
        got = __shfl_sync(0xffffffffu, got, 0);
        __syncwarp();
        if (!got) {
          if (lane == 0) fail_timeout(a, 51);
          break;
        }
        cur = ms.desc[s];
        if (cur.kind == kDone) break;
        issue(a, g, ms, cur, warp, lane, 0, r);
      }
      // (3) a down unit: stage its 16 rows of w*h in shared memory
      if (cur.kind == kDown) {
        const int K = cur.slot == 0 ? a.Is : a.I;
        const int Kmax = a.I > a.Is ? a.I : a.Is;
        for (int row = warp; row < 16; row += kWorkers) {
          const uint16_t* src = a.hbuf + ((int64_t)cur.slot * 16 + row) * Kmax;
          uint8_t* dst = hb + row * g.hs_stride;
          for (int c = lane; c < K / 8; c += 32)
            *reinterpret_cast<uint4*>(dst + c * 16) = __ldcg(reinterpret_cast<const uint4*>(src) + c);
        }
        if (lane == 0) {
          mbar_arrive(&ms.bar_a);
          if (!wait_phase(&ms.bar_a, (uint32_t)(n_down & 1), worker_limit)) fail_timeout(a, 52);
        }
        __syncwarp();
        ++n_down;
      }
      // (4) consume
      float acc[kMaxT];
#pragma unroll
      for (int t = 0; t < kMaxT; ++t) acc[t] = 0.0f;
      if (cur.kind == kRoute) {
        route_unit(a, g, reinterpret_cast<float*>(hb), warp, ms);
      } else {
        const int nst = stages_of(a, g, cur);
        consume(a, g, cur, warp, lane, 0, r, xs, hb, acc);
        for (int st = 1; st < nst; ++st) {
          issue(a, g, ms, cur, warp, lane, st, r);
          consume(a, g, cur, warp, lane, st, r, xs, hb, acc);
        }
      }
      float* my = red + s * kRedFloats + warp * 128;
      if (cur.kind == kRouter) {
#pragma unroll
        for (int t = 0; t < kMaxT; ++t) {
          const float v = warp_sum(acc[t]);
          if (lane == 0) my[t] = v;
        }
      } else if (cur.kind == kGateUp || cur.kind == kDown) {
        *reinterpret_cast<float4*>(my + lane * 4) = make_float4(acc[0], acc[1], acc[2], acc[3]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms.desc_empty[s]);
      // (5) the next unit's loads, when its descriptor is already there
      const int s1 = (m + 1) & 1;
      int ready = 0;
      if (lane == 0) ready = mbar_test_wait(&ms.desc_full[s1], (uint32_t)(((m + 1) >> 1) & 1)) ? 1 : 0;
      ready = __shfl_sync(0xffffffffu, ready, 0);
      __syncwarp();
      prev = cur;
      issued = false;
      if (ready) {
        cur = ms.desc[s1];
        if (cur.kind != kDone) issue(a, g, ms, cur, warp, lane, 0, r);
        issued = true;
      }
      // (6) hand-over: every warp's partial sums of unit m are in `red`
      if (lane == 0) {
        mbar_arrive(&ms.bar_e[s]);
        if (!wait_phase(&ms.bar_e[s], (uint32_t)((m >> 1) & 1), worker_limit)) fail_timeout(a, 53);
      }
      __syncwarp();
      ok = ok && true;
    }
    (void)ok;
  }

  // ---- leave: the last CTA out restores the counters to zero ----
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    ms.last = atomicAdd(a.sync + kExit, 1) == (int)gridDim.x - 1 ? 1 : 0;
  }
  __syncthreads();
  if (ms.last) {
    __threadfence();
    const int nwords = kRowBlocks + (a.H + 15) / 16;
    for (int i = threadIdx.x; i < nwords; i += blockDim.x) a.sync[i] = 0;
    __threadfence();
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
int pow2_at_least(int v) {
  int p = 1;
  while (p < v) p <<= 1;
  return p;
}

// Split of a down unit over the worker warps: ksd warps share a 16-row group
// (chunks dealt round-robin), rgd = kWorkers / ksd row groups per unit. Picks
// the split that keeps the most warps busy, then the fewest register stages,
// then the fewest partial sums.
void down_split(int K, int* ksd, int* rgd, int* cpw) {
  const int nch = K / 32;
  int best = 1, best_active = -1, best_stages = 1 << 30;
  for (int k = 1; k <= kWorkers; ++k) {
    const int active = (kWorkers / k) * k;
    const int stages = ((nch + k - 1) / k + kStageChunks - 1) / kStageChunks;
    if (active > best_active || (active == best_active && stages < best_stages)) {
      best = k;
      best_active = active;
      best_stages = stages;
    }
  }
  *ksd = best;
  *rgd = kWorkers / best;
  *cpw = (nch + best - 1) / best;
}

int row_stride(int K) { return ((2 * K + 127) / 128) * 128 + 64; }

Geo make_geo(const DecodeArgs& a) {
  Geo g{};
  g.xs_stride = row_stride(a.H);
  const int Kmax = a.I > a.Is ? a.I : a.Is;
  g.hs_stride = row_stride(Kmax);
  // router: the most rows per unit that still gives enough units to spread
  // over the SMs (128, or one per row), then every warp on those rows, each
  // a slice of 128-float pieces
  const int npieces = a.H / 128;
  const int want = a.E < 128 ? a.E : 128;
  int rpu = kWorkers;
  while (rpu > 1 && (a.E + rpu - 1) / rpu < want) --rpu;
  int ks = kWorkers / rpu;
  if (ks > npieces) ks = npieces;
  g.ks_r = ks;
  g.rpu = rpu;
  g.np_r = (npieces + ks - 1) / ks;
  g.nr = (a.E + g.rpu - 1) / g.rpu;
  g.gu_cpw = (a.H / 32 + kWorkers - 1) / kWorkers;
  g.gu_units_r = a.I / 8;
  g.gu_units_s = a.Is / 8;
  down_split(a.I, &g.dn_ksd_r, &g.dn_rgd_r, &g.dn_cpw_r);
  g.dn_units_r = (a.H + 16 * g.dn_rgd_r - 1) / (16 * g.dn_rgd_r);
  if (a.Is > 0) {
    down_split(a.Is, &g.dn_ksd_s, &g.dn_rgd_s, &g.dn_cpw_s);
    g.dn_units_s = (a.H + 16 * g.dn_rgd_s - 1) / (16 * g.dn_rgd_s);
  } else {
    g.dn_ksd_s = g.dn_rgd_s = g.dn_cpw_s = 1;
    g.dn_units_s = 0;
  }
  g.P = pow2_at_least((a.E + 31) / 32);
  const int xs_bytes = kMaxT * g.xs_stride;
  const int hb_bytes = 16 * g.hs_stride;
  const int route_bytes = kMaxT * 64 * g.P * 4;  // per routing warp: 32P gates + 32P scratch
  g.off_hb = (xs_bytes + 127) / 128 * 128;
  const int hb_or_route = hb_bytes > route_bytes ? hb_bytes : route_bytes;
  g.off_red = g.off_hb + (hb_or_route + 127) / 128 * 128;
  g.off_misc = g.off_red + 2 * kRedFloats * 4;
  g.smem = g.off_misc + (int)((sizeof(Misc) + 127) / 128 * 128);
  return g;
}

}  // namespace

size_t decode_hbuf_bytes(int I, int Is) {
  const int Kmax = I > Is ? I : Is;
  return (size_t)kDecodeMaxSlots * 16 * Kmax * 2;
}

size_t decode_part_bytes(int H) { return (size_t)kDecodeMaxSlots * H * kDecodeMaxT * 4; }

bool decode_supported(int64_t T, int k, int E, int H, int I, int Is) {
  if (T < 1 || T > kDecodeMaxT || T * k > 64 || E > kDecodeMaxE || k > E) return false;
  if (H % 128 != 0 || H > 8192 || I % 32 != 0 || Is % 32 != 0) return false;
  if ((int64_t)(kRowBlocks + H / 16) * 4 > (int64_t)kWsSyncBytes) return false;
  DecodeArgs a{};
  a.T = (int)T;
  a.E = E;
  a.H = H;
  a.I = I;
  a.Is = Is;
  return make_geo(a).smem <= 227 * 1024;
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s) {
  const Geo g = make_geo(a);
  cudaError_t e = cudaFuncSetAttribute(decode_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, g.smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sm_count());  // one CTA per SM, all resident: CTAs wait on each other's counters
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = (size_t)g.smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  before_launch(MOE_KERNEL_DECODE_FUSED, s);
  e = cudaLaunchKernelEx(&cfg, decode_stream_kernel, a, g);
  after_launch(MOE_KERNEL_DECODE_FUSED, s);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace moe
