// Fused decode: the whole MoE block for 1-2 tokens in one launch.
//
// At decode the block is bound by HBM bandwidth: it streams the router weight,
// the shared MLP and, of the routed experts, only the few that were selected
// (page "Ling-3.0-flash-GGUF", section "Measured performance"): ~120 MB for
// Ling-3.0-flash against a few microseconds of arithmetic. The kernel is
// therefore a weight-streaming engine: one CTA per SM, a producer thread that
// keeps a ring of shared-memory stages filled with untiled bulk copies
// (cp.async.bulk, mbarrier completion), and twelve consumer warps that each
// take whole stages and reduce them with the token rows on the CUDA cores. A stage holds 4H bytes: one fp32 router row, or one bf16
// gate row plus the matching up row, or a block of down-projection rows.
//
// Every phase's rows are split evenly into one contiguous range per CTA, and
// each CTA streams its ranges in this order:
//
//   A  router rows (logits, fp32 FMA) and the shared MLP's gate/up rows
//                                                            -> grid barrier
//   S  the shared MLP's down rows: their copies start during the barrier and
//      the routing, since they do not depend on it
//   (every CTA routes the 1-2 tokens itself with all consumer warps: no
//    second barrier; the producer then learns the selected experts)
//   C  gate/up rows of the selected experts, SwiGLU in fp32; each warp adds
//      its rows to a per-expert completion counter
//   D  down rows of the selected experts, weighted by the routing; a block
//      starts once its expert's counter shows all of h
//
// Each output row y[t, n] counts its k + 1 contributions (k slot rows and the
// shared row); the lane that brings the last one sums them in slot order and
// rounds once to bf16. Counters are released with a fence after the rows they
// cover; data written in this launch is read through L2 (ld.global.cg). Every
// wait is bounded (globaltimer, DecodeArgs::wait_ns): one that runs out records
// MOE_ERR_TIMEOUT in the workspace and returns; the producer first waits
// (bounded) for its copies in flight, so no copy lands after its CTA exits.
//
// The routing (route_block.cuh) takes the same decisions as the per-token
// router kernel, bit for bit.
#include "decode_fused.cuh"
#include "mbarrier.cuh"
#include "fused_common.cuh"
#include "route_block.cuh"

namespace moe {

namespace {

using namespace fused;

constexpr int kConsumerWarps = 12;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kFusedThreads = kConsumers + 32;  // + the producer warp
constexpr int kFusedMaxT = 2;
constexpr int kMaxStages = 16;
constexpr int kMinStages = 4;
constexpr int kMaxDownRows = 16;   // rows per down block: lane t*16 + r holds (slot or token t, row r)
constexpr int kMaxHidden = 8192;   // a stage (4H bytes) must leave room for kMinStages
constexpr int kSmemBudget = 227 * 1024;
constexpr int kMaxPend = 4;   // uncounted output rows per lane

// Stream geometry, the same on host and device.
struct Geo {
  int stage_bytes;  // 4H
  int depth;        // ring stages
  int rd, rs;       // rows per routed / shared down block
  int nblk, nsblk;  // down blocks per expert / of the shared MLP
};

struct FusedSmem {
  uint64_t full[kMaxStages], empty[kMaxStages], route_ready;
  // Stage tags: the stream index a slot was last filled with. Consumer warps
  // run ahead of one another, so a warp can reach a slot while the slot's
  // previous fill is still in flight, when its parity would read as the phase
  // the warp waits for; the tag shows which fill is pending.
  volatile uint32_t tag[kMaxStages];
  block_route::Smem<kConsumerWarps> rt;  // routing state and results
  int flag;
  volatile int abort;  // a consumer warp stopped before the grid barrier
  unsigned int next_unit;  // the next stream unit a consumer warp may claim
};


// Dynamic shared memory after the ring: routing scratch ([T*E] fp32 scores,
// [T*E] fp32 biased scores, [T*E] 64-bit keys), then the token rows (fp32,
// converted once) and the expert bias (fp32).
__host__ __device__ __forceinline__ size_t route_scratch_bytes(int T, int E) { return block_route::scratch_bytes(T, E); }
__host__ __device__ __forceinline__ size_t scratch_bytes(int T, int E, int H) {
  return route_scratch_bytes(T, E) + (size_t)T * H * 4 + (size_t)E * 4;
}


__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kConsumers) : "memory"); }

constexpr int ilog2(int n) { return n <= 1 ? 0 : 1 + ilog2(n / 2); }

// Warp reduce-scatter of N (a power of two <= 32) values per lane: returns the
// warp total of value `which`, with which = lane >> (5 - log2 N) (the lane's
// top log2 N bits). log2 N halving steps, then a butterfly over the rest:
// N - 1 + 5 - log2 N shuffles instead of 5 N.
template <int N>
__device__ __forceinline__ float reduce_scatter(float (&v)[N]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int step = 0; step < ilog2(N); ++step) {
    const int o = 16 >> step, n = N >> step;
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < n / 2; ++i) {
      const float keep = up ? v[i + n / 2] : v[i];
      const float give = up ? v[i] : v[i + n / 2];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, give, o);
    }
  }
#pragma unroll
  for (int o = 16 >> ilog2(N); o > 0; o >>= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
  return v[0];
}

// Frees a stage once every lane of the warp has read it.
__device__ __forceinline__ void release_stage(uint64_t* empty) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(empty);
}

// Products of one 16-byte bf16 weight chunk with 8 fp32 values, added to two
// accumulators (even and odd elements): each dependent chain is half as long.
__device__ __forceinline__ void dot8x2(uint4 w, const float* v, float& e, float& o) {
  e = fmaf(bf16_lo(w.x), v[0], e);
  o = fmaf(bf16_hi(w.x), v[1], o);
  e = fmaf(bf16_lo(w.y), v[2], e);
  o = fmaf(bf16_hi(w.y), v[3], o);
  e = fmaf(bf16_lo(w.z), v[4], e);
  o = fmaf(bf16_hi(w.z), v[5], o);
  e = fmaf(bf16_lo(w.w), v[6], e);
  o = fmaf(bf16_hi(w.w), v[7], o);
}

// ---------------------------------------------------------------------------
// Stage consumers (one warp each). Lane l takes the 16-byte columns l, l + 32,
// ... of a row: contiguous across the warp, so shared-memory reads are free of
// bank conflicts. Token rows x come from the shared-memory copy made at
// kernel start; h rows (written in this launch) through L2.
// ---------------------------------------------------------------------------

// One fp32 router row (H) against up to two bf16 token rows. Returns the logit
// of token 0 in lane 0 and of token 1 in lane 16.
__device__ __forceinline__ float router_unit(const float* w, int H, const float* xs, int T, uint64_t* empty) {
  const int lane = threadIdx.x & 31;
  const float4* x0 = reinterpret_cast<const float4*>(xs);
  const float4* x1 = reinterpret_cast<const float4*>(xs + H);
  float e0 = 0.f, o0 = 0.f, e1 = 0.f, o1 = 0.f;
#pragma unroll 2
  for (int c = lane; c < H / 4; c += 32) {
    const float4 w4 = reinterpret_cast<const float4*>(w)[c];
    const float4 xa = x0[c];
    e0 = fmaf(xa.x, w4.x, e0);
    o0 = fmaf(xa.y, w4.y, o0);
    e0 = fmaf(xa.z, w4.z, e0);
    o0 = fmaf(xa.w, w4.w, o0);
    if (T > 1) {
      const float4 xb = x1[c];
      e1 = fmaf(xb.x, w4.x, e1);
      o1 = fmaf(xb.y, w4.y, o1);
      e1 = fmaf(xb.z, w4.z, e1);
      o1 = fmaf(xb.w, w4.w, o1);
    }
  }
  release_stage(empty);
  float v[2] = {e0 + o0, e1 + o1};
  return reduce_scatter<2>(v);
}

// One gate row and one up row (H bf16 each) against up to two token rows:
// returns silu(gate . x_t) * (up . x_t) for token row 0 in lane 0 and for
// token row 1 in lane 16, fp32.
__device__ __forceinline__ float gate_up_unit(const uint16_t* gate, const uint16_t* up, int H, const float* x0,
                                              const float* x1, uint64_t* empty) {
  const int lane = threadIdx.x & 31;
  float ve[4] = {0.f, 0.f, 0.f, 0.f}, vo[4] = {0.f, 0.f, 0.f, 0.f};  // gate . x0, up . x0, gate . x1, up . x1
#pragma unroll 2
  for (int c = lane; c < H / 8; c += 32) {
    const uint4 gv = reinterpret_cast<const uint4*>(gate)[c];
    const uint4 uv = reinterpret_cast<const uint4*>(up)[c];
    const float4 a0 = reinterpret_cast<const float4*>(x0)[2 * c], a1 = reinterpret_cast<const float4*>(x0)[2 * c + 1];
    const float xf[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    dot8x2(gv, xf, ve[0], vo[0]);
    dot8x2(uv, xf, ve[1], vo[1]);
    if (x1 != nullptr) {
      const float4 b0 = reinterpret_cast<const float4*>(x1)[2 * c], b1 = reinterpret_cast<const float4*>(x1)[2 * c + 1];
      const float xg[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
      dot8x2(gv, xg, ve[2], vo[2]);
      dot8x2(uv, xg, ve[3], vo[3]);
    }
  }
  release_stage(empty);
  float v[4] = {ve[0] + vo[0], ve[1] + vo[1], ve[2] + vo[2], ve[3] + vo[3]};
  const float s = reduce_scatter<4>(v);                     // lane >> 3 = 2 t + (0 gate, 1 up)
  const float up_sum = __shfl_xor_sync(0xffffffffu, s, 8);  // the up sum sits 8 lanes above the gate sum
  return silu_f32(s) * up_sum;
}

// One 8-column chunk of up to two fp32 h rows (h1 null: the h0 values again).
struct HChunk {
  float4 a0, a1, b0, b1;
};

__device__ __forceinline__ HChunk load_h(const float* h0, const float* h1, int c, int nc) {
  HChunk p;
  if (c < nc) {
    p.a0 = ldcg4(h0 + c * 8);
    p.a1 = ldcg4(h0 + c * 8 + 4);
    p.b0 = p.a0;
    p.b1 = p.a1;
    if (h1 != nullptr) {
      p.b0 = ldcg4(h1 + c * 8);
      p.b1 = ldcg4(h1 + c * 8 + 4);
    }
  } else {
    p.a0 = p.a1 = p.b0 = p.b1 = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  return p;
}

// nrows (<= 16) rows of K bf16 against up to two fp32 h rows. `first` holds
// this lane's first h chunk, loaded before the stage was waited on; each later
// chunk is loaded one step ahead. Returns the dot of row r with h row t in
// lane t*16 + r.
__device__ __forceinline__ float down_unit(const uint16_t* w, int nrows, int K, const float* h0, const float* h1,
                                           HChunk first, uint64_t* empty) {
  const int lane = threadIdx.x & 31;
  const int nc = K / 8;
  const bool two = h1 != nullptr;
  float acc[2 * kMaxDownRows];
#pragma unroll
  for (int i = 0; i < 2 * kMaxDownRows; ++i) acc[i] = 0.f;
  HChunk cur = first;
#pragma unroll 1
  for (int c = lane; c < nc; c += 32) {
    const HChunk nxt = load_h(h0, h1, c + 32, nc);
    const float f0[8] = {cur.a0.x, cur.a0.y, cur.a0.z, cur.a0.w, cur.a1.x, cur.a1.y, cur.a1.z, cur.a1.w};
    const float f1[8] = {cur.b0.x, cur.b0.y, cur.b0.z, cur.b0.w, cur.b1.x, cur.b1.y, cur.b1.z, cur.b1.w};
#pragma unroll
    for (int r = 0; r < kMaxDownRows; ++r) {
      if (r < nrows) {
        const uint4 wv = reinterpret_cast<const uint4*>(w + (size_t)r * K)[c];
        acc[r] = dot8_bf16(wv, f0, acc[r]);
        if (two) acc[kMaxDownRows + r] = dot8_bf16(wv, f1, acc[kMaxDownRows + r]);
      }
    }
    cur = nxt;
  }
  release_stage(empty);
  return reduce_scatter<2 * kMaxDownRows>(acc);
}


// ---------------------------------------------------------------------------
// The stream of one CTA: a sequence of segments, each a contiguous share of
// one kind of rows. A (router rows, then shared gate/up pairs) and S (shared
// down blocks) are split evenly over the CTAs. Then every CTA takes a share
// of each distinct expert's gate/up pairs (C0 .. C(n-1)) and then of each
// one's down blocks (D0 .. D(n-1)): expert i's h is complete once every CTA
// has passed its C share of it, long before the CTAs reach Di, so the down
// blocks rarely wait. The shares of expert i are rotated by i*G/n CTAs so
// that the rounding of the even split does not favour the same CTAs for every
// expert.
// ---------------------------------------------------------------------------
enum SegKind { kSegA, kSegS, kSegC, kSegD };

struct Seg {
  int kind, ai;  // kind, distinct expert (C and D)
  Range r;       // the share: rows (C), blocks (D), items (A, S)
};

__device__ __forceinline__ int num_segments(int n_act) { return 2 + 2 * n_act; }

__device__ __forceinline__ Seg segment(const DecodeArgs& a, const Geo& g, int n_act, int i) {
  const int G = gridDim.x, b = blockIdx.x;
  Seg sg{};
  if (i == 0) {
    sg.kind = kSegA;
    sg.r = split((a.logits_override == nullptr ? a.E : 0) + (a.ws_gate_up != nullptr ? a.Is : 0), b, G);
    return sg;
  }
  if (i == 1) {
    sg.kind = kSegS;
    sg.r = split(a.ws_down != nullptr ? g.nsblk : 0, b, G);
    return sg;
  }
  const int j = i - 2;
  sg.kind = j < n_act ? kSegC : kSegD;
  sg.ai = j < n_act ? j : j - n_act;
  const int rb = (b + (int)((int64_t)sg.ai * G / n_act)) % G;
  sg.r = split(sg.kind == kSegC ? a.I : g.nblk, rb, G);
  return sg;
}

// The global rows of one stream unit: up to two contiguous pieces.
struct UnitSrc {
  const void* p0;
  const void* p1;
  uint32_t n0, n1;
};

__device__ __forceinline__ UnitSrc unit_src(const DecodeArgs& a, const Geo& g, const FusedSmem& sm, const Seg& sg,
                                           int i) {
  const int H = a.H, I = a.I, Is = a.Is;
  const int n_router = a.logits_override == nullptr ? a.E : 0;
  UnitSrc u{nullptr, nullptr, 0u, 0u};
  if (sg.kind == kSegA) {
    if (i < n_router) {
      u.p0 = a.router_w + (int64_t)i * H;
      u.n0 = 4u * H;
    } else {
      const int j = i - n_router;
      u.p0 = a.ws_gate_up + (int64_t)j * H;
      u.p1 = a.ws_gate_up + (int64_t)(Is + j) * H;
      u.n0 = u.n1 = 2u * H;
    }
  } else if (sg.kind == kSegS) {
    const int n0 = i * g.rs, rows = min(g.rs, H - n0);
    u.p0 = a.ws_down + (int64_t)n0 * Is;
    u.n0 = 2u * rows * Is;
  } else if (sg.kind == kSegC) {
    const uint16_t* gate = a.w_gate_up + ((int64_t)sm.rt.act_e[sg.ai] * 2 * I + i) * H;
    u.p0 = gate;
    u.p1 = gate + (int64_t)I * H;
    u.n0 = u.n1 = 2u * H;
  } else {
    const int n0 = i * g.rd, rows = min(g.rd, H - n0);
    u.p0 = a.w_down + ((int64_t)sm.rt.act_e[sg.ai] * H + n0) * I;
    u.n0 = 2u * rows * I;
  }
  return u;
}

// A position in the CTA's stream: segment si, item i of its share.
struct Cursor {
  int si, i;
  Seg sg;
};

// Moves c past finished segments to its next unit; false when none is left in
// the first nseg segments (c then stays on its last segment, so that it can
// resume once nseg grows).
__device__ __forceinline__ bool cursor_valid(const DecodeArgs& a, const Geo& g, int n_act, int nseg, Cursor& c) {
  while (c.i >= c.sg.r.lo + c.sg.r.n) {
    if (c.si + 1 >= nseg) return false;
    ++c.si;
    c.sg = segment(a, g, n_act, c.si);
    c.i = c.sg.r.lo;
  }
  return true;
}

// The producer thread: issues the CTA's stream in order, unit u into ring slot
// u % depth once the consumer of the slot's previous unit freed it. (Bulk L2
// prefetches of the units ahead of the ring were measured here and made the
// step 1.5x slower.)
__device__ void producer(const DecodeArgs& a, const Geo& g, unsigned char* ring, FusedSmem& sm) {
  uint32_t u = 0;
  bool ok = true;
  int nseg = 2, n_act = 0;  // the segments after S need this CTA's routing
  Cursor c{0, 0, segment(a, g, 0, 0)};
  c.i = c.sg.r.lo;
  for (;;) {
    if (!cursor_valid(a, g, n_act, nseg, c)) {
      if (nseg > 2) break;
      // end of S: wait for the routing, then continue with the selected experts
      ok = thread_wait_phase(&sm.route_ready, 0, a.hdr, 500, a.wait_ns);
      if (!ok) break;
      n_act = sm.rt.n_act;
      nseg = num_segments(n_act);
      continue;
    }
    const int s = (int)(u % (uint32_t)g.depth);
    const uint32_t n = u / (uint32_t)g.depth;
    if (n > 0 && !thread_wait_phase(&sm.empty[s], (n - 1) & 1u, a.hdr, 400 + s, a.wait_ns)) {
      ok = false;
      break;
    }
    const UnitSrc q = unit_src(a, g, sm, c.sg, c.i);
    sm.tag[s] = u;  // the slot's previous fill is consumed: its phase is complete
    mbar_expect_tx(&sm.full[s], q.n0 + q.n1);
    unsigned char* dst = ring + (size_t)s * g.stage_bytes;
    bulk_load(dst, q.p0, q.n0, &sm.full[s]);
    if (q.n1 != 0) bulk_load(dst + q.n0, q.p1, q.n1, &sm.full[s]);
    ++c.i;
    ++u;
  }
  if (!ok) {
    // the consumers stopped: wait (bounded) for the copies still in flight
    const uint32_t first = u > (uint32_t)g.depth ? u - g.depth : 0u;
    for (uint32_t v = first; v < u; ++v)
      thread_wait_phase(&sm.full[v % g.depth], (v / g.depth) & 1u, nullptr, 0, a.wait_ns);
  }
}

// The next unclaimed stream unit of the CTA, for the whole warp. Warps claim
// units in stream order as they become free, so a warp that drew short units
// takes more of them: no warp is left with a static share that outlasts the
// others.
__device__ __forceinline__ uint32_t claim_unit(FusedSmem& sm) {
  uint32_t u = 0;
  if ((threadIdx.x & 31) == 0) u = atomicAdd(&sm.next_unit, 1u);
  return __shfl_sync(0xffffffffu, u, 0);
}

// A consumer warp: claims its CTA's stream units in order (claim_unit).
__device__ void consumer(const DecodeArgs& a, const Geo& g, unsigned char* ring, unsigned char* scratch,
                         FusedSmem& sm) {
  const int T = a.T, k = a.k, H = a.H, I = a.I, Is = a.Is, E = a.E;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int32_t* done = a.sync;  // [kMaxSlots]: gate/up rows finished per distinct expert

  // counters: each CTA zeroes its share; the grid barrier orders it before use
  const Range z = split(kMaxSlots + kFusedMaxT * H, blockIdx.x, gridDim.x);
  for (int i = threadIdx.x; i < z.n; i += kConsumers) a.sync[z.lo + i] = 0;

  // token rows (as fp32) and expert bias into shared memory (one coalesced pass)
  float* xs = reinterpret_cast<float*>(scratch + route_scratch_bytes(T, E));
  float* bias_s = a.expert_bias != nullptr ? xs + (size_t)T * H : nullptr;
  for (int i = threadIdx.x; i < T * H / 8; i += kConsumers) {
    float f[8];
    unpack8_bf16(ld_nc_u4(a.x + (size_t)i * 8), f);
    reinterpret_cast<float4*>(xs)[2 * i] = make_float4(f[0], f[1], f[2], f[3]);
    reinterpret_cast<float4*>(xs)[2 * i + 1] = make_float4(f[4], f[5], f[6], f[7]);
  }
  if (bias_s != nullptr)
    for (int e = threadIdx.x; e < E; e += kConsumers) bias_s[e] = __ldg(a.expert_bias + e);
  consumer_sync();

  const int n_router = a.logits_override == nullptr ? E : 0;
  const float* logits = a.logits_override != nullptr ? a.logits_override : a.logits;
  const bool pre_scores = block_route::scores_with_logits(a);
  const int target = k + (a.ws_down != nullptr ? 1 : 0);
  Pending<kMaxPend> q;
  q.np = 0;
  auto flush_if_pending = [&]() {
    if (q.np > 0) publish(a, q, target);
  };
  // Waits for stream unit v; publishes the pending work first if it would block.
  auto stage = [&](uint32_t v, const unsigned char** p, uint64_t** empty) {
    const int s = (int)(v % (uint32_t)g.depth);
    const uint32_t parity = (v / g.depth) & 1u;
    *p = ring + (size_t)s * g.stage_bytes;
    *empty = &sm.empty[s];
    if (__all_sync(0xffffffffu, sm.tag[s] == v && mbar_try_wait(&sm.full[s], parity))) return true;
    flush_if_pending();
    return warp_wait_tag(&sm.tag[s], v, a.hdr, 300 + s, a.wait_ns) &&
           warp_wait_phase(&sm.full[s], parity, a.hdr, 300 + s, a.wait_ns);
  };

  // ---- A: router rows and shared gate/up pairs ----
  // A warp whose wait runs out must still reach the named barriers below (they
  // have no timeout): it flags the CTA, and the consumers leave together after
  // the grid barrier.
  uint32_t carried;  // a unit claimed past phase A, processed after the routing
  {
    const Seg sg = segment(a, g, 0, 0);
    for (;;) {
      const uint32_t u = claim_unit(sm);
      if (u >= (uint32_t)sg.r.n) {
        carried = u;
        break;
      }
      const unsigned char* st;
      uint64_t* empty;
      if (!stage(u, &st, &empty)) {
        sm.abort = 1;
        carried = 0xffffffffu;
        break;
      }
      const int i = sg.r.lo + (int)u;
      if (i < n_router) {
        const float v = router_unit(reinterpret_cast<const float*>(st), H, xs, T, empty);
        if (lane == 0 || (lane == 16 && T > 1)) {
          const int t = lane >> 4;
          a.logits[t * E + i] = v;
          if (pre_scores) block_route::store_score(a, t, i, v, bias_s);
        }
      } else {
        const int j = i - n_router;
        const uint16_t* gate = reinterpret_cast<const uint16_t*>(st);
        const float v = gate_up_unit(gate, gate + H, H, xs, T > 1 ? xs + H : nullptr, empty);
        if (lane == 0) a.h_shared[j] = v;
        if (lane == 16 && T > 1) a.h_shared[Is + j] = v;
      }
    }
  }
  if (!grid_barrier<kConsumers>(a.hdr, 1, &sm.flag, a.wait_ns, a.withhold != 0 && blockIdx.x == 0) || sm.abort != 0) return;

  // ---- routing; then the producer may issue the selected experts' rows ----
  block_route::route_block(a, logits, bias_s, scratch, sm.rt);
  if (threadIdx.x == 0) mbar_arrive(&sm.route_ready);
  const int n_act = sm.rt.n_act;
  const int tq = lane >> 4, rr = lane & 15;  // down blocks: lane t*16 + r holds (slot or token t, row r)

  const int nseg = num_segments(n_act);
  int si = 0;        // segment of the last claimed unit
  uint32_t base = 0;  // its first stream index
  Seg sg = segment(a, g, n_act, 0);
  for (uint32_t u = carried;; u = claim_unit(sm)) {
    while (si < nseg && u >= base + (uint32_t)sg.r.n) {  // segments are visited in order
      base += sg.r.n;
      if (++si < nseg) sg = segment(a, g, n_act, si);
    }
    if (si >= nseg) break;
    {
      const int i = sg.r.lo + (int)(u - base);
      const unsigned char* st;
      uint64_t* empty;
      if (sg.kind == kSegS) {  // ---- shared down block ----
        const int n0 = i * g.rs, rows = min(g.rs, H - n0);
        const float* h1 = T > 1 ? a.h_shared + Is : nullptr;
        const HChunk p = load_h(a.h_shared, h1, lane, Is / 8);
        if (!stage(u, &st, &empty)) return;
        const float v = down_unit(reinterpret_cast<const uint16_t*>(st), rows, Is, a.h_shared, h1, p, empty);
        int idx = -1;
        if (rr < rows && tq < T) {
          a.shared_out[(int64_t)tq * H + n0 + rr] = v;
          idx = tq * H + n0 + rr;
        }
        add_pending(q, idx);
      } else if (sg.kind == kSegC) {  // ---- gate/up pair of a selected expert ----
        const int slA = sm.rt.act_a[sg.ai], slB = sm.rt.act_b[sg.ai];
        if (!stage(u, &st, &empty)) return;
        const uint16_t* w = reinterpret_cast<const uint16_t*>(st);
        const float v = gate_up_unit(w, w + H, H, xs + (slA / k) * H, slB >= 0 ? xs + (slB / k) * H : nullptr, empty);
        // each writer lane releases its own row: the down blocks of this expert
        // wait for I rows per slot holding it
        if (lane == 0 || (lane == 16 && slB >= 0)) {
          a.h[(int64_t)(lane == 0 ? slA : slB) * I + i] = v;
          red_release_add(done + sg.ai, 1);
        }
      } else {  // ---- down block of a selected expert ----
        const int ai = sg.ai, slA = sm.rt.act_a[ai], slB = sm.rt.act_b[ai];
        const int n0 = i * g.rd, rows = min(g.rd, H - n0);
        const int need = slB >= 0 ? 2 * I : I;
        int complete = lane == 0 ? ld_acquire(done + ai) >= need : 0;
        if (!__shfl_sync(0xffffffffu, complete, 0)) {
          flush_if_pending();
          if (!warp_wait_count(done + ai, need, a.hdr, 200 + ai, a.wait_ns)) return;
        }
        __syncwarp();
        const float* h0 = a.h + (int64_t)slA * I;
        const float* h1 = slB >= 0 ? a.h + (int64_t)slB * I : nullptr;
        const HChunk p = load_h(h0, h1, lane, I / 8);
        if (!stage(u, &st, &empty)) return;
        const float v = down_unit(reinterpret_cast<const uint16_t*>(st), rows, I, h0, h1, p, empty);
        const int sl = tq == 0 ? slA : slB;
        int idx = -1;
        if (rr < rows && sl >= 0) {
          a.y_slots[(int64_t)sl * H + n0 + rr] = sm.rt.w[sl] * v;
          idx = (sl / k) * H + n0 + rr;
        }
        add_pending(q, idx);
      }
      if (q.np == kMaxPend) publish(a, q, target);
    }
  }
  publish(a, q, target);
}

__global__ void __launch_bounds__(kFusedThreads, 1) decode_fused_kernel(const DecodeArgs a, const Geo g) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  __shared__ FusedSmem sm;
  unsigned char* ring = smem_raw;
  unsigned char* scratch = smem_raw + (size_t)g.depth * g.stage_bytes;
  if (threadIdx.x == 0) {
    for (int s = 0; s < g.depth; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
      sm.tag[s] = 0xffffffffu;
    }
    mbar_init(&sm.route_ready, 1);
    sm.abort = 0;
    sm.next_unit = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x >= kConsumers) {
    if (threadIdx.x == kConsumers) producer(a, g, ring, sm);
    return;
  }
  consumer(a, g, ring, scratch, sm);
}


// Stream geometry for a launch; depth 0 when the shapes do not fit.
Geo make_geo(int T, int E, int H, int I, int Is) {
  Geo g{};
  if (H > kMaxHidden || I > 2 * H || Is > 2 * H) return g;
  g.stage_bytes = 4 * H;
  const int rd = g.stage_bytes / (2 * I), rs = Is > 0 ? g.stage_bytes / (2 * Is) : 1;
  g.rd = rd < kMaxDownRows ? rd : kMaxDownRows;
  g.rs = rs < kMaxDownRows ? rs : kMaxDownRows;
  g.nblk = (H + g.rd - 1) / g.rd;
  g.nsblk = Is > 0 ? (H + g.rs - 1) / g.rs : 0;
  const int avail = kSmemBudget - (int)sizeof(FusedSmem) - (int)scratch_bytes(T, E, H);
  g.depth = avail / g.stage_bytes < kMaxStages ? avail / g.stage_bytes : kMaxStages;
  if (g.depth < kMinStages) g.depth = 0;
  return g;
}

}  // namespace

size_t decode_fused_sync_ints(int H) { return (size_t)kMaxSlots + (size_t)kFusedMaxT * H + 1; }

bool decode_fused_supported(int64_t T, int k, int E, int H, int I, int Is) {
  // at most two tokens and one warp lane per slot; a stage must hold a router row
  return T >= 1 && T <= kFusedMaxT && k <= E && E <= 1024 && T * k <= kMaxSlots &&
         make_geo((int)T, E, H, I, Is).depth > 0;
}

cudaError_t launch_decode_fused(const DecodeArgs& a, cudaStream_t s) {
  const Geo g = make_geo(a.T, a.E, a.H, a.I, a.Is);
  if (g.depth == 0) return cudaErrorInvalidValue;
  const size_t smem = (size_t)g.depth * g.stage_bytes + scratch_bytes(a.T, a.E, a.H);
  cudaError_t e = cudaFuncSetAttribute(decode_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_fused_kernel, kFusedThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sm_count());  // one CTA per SM, all resident: the grid barrier and the waits rely on it
  cfg.blockDim = dim3(kFusedThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  before_launch(MOE_KERNEL_DECODE_FUSED, s);
  e = cudaLaunchKernelEx(&cfg, decode_fused_kernel, a, g);
  after_launch(MOE_KERNEL_DECODE_FUSED, s);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace moe
