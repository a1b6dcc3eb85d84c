// Fused decode on the tensor cores: the whole MoE block for 1-2 tokens in one
// launch, for hidden sizes that are a multiple of 512 (up to 4096) and expert
// and shared widths that are multiples of 64 up to 512 (Ling-3.0-flash: H =
// 4096, I = Is = 512). moe_forward runs it when moe_set_decode_kernel(2)
// selects it; at these shapes it measures within a microsecond of the CUDA-core
// kernel (decode_fused.cu), both bound by the grid barrier, the routing and the
// counters between phases rather than by bytes or arithmetic.
//
// Decode streams the router weight, the shared MLP and just the experts the
// router chose (page "Ling-3.0-flash-GGUF", section "Measured performance"),
// so it is bound by HBM bandwidth, and the arithmetic must cost little per
// byte.
// On the CUDA cores a bf16 weight costs about two instructions (unpack and
// FMA); here the consumers multiply with mma.sync (m16n8k16, bf16 inputs, fp32
// accumulation), one ldmatrix, one 8-byte shared load and one mma per 512
// bytes of weights. The token (or slot) dimension is the n = 8 side of the
// mma, of which 1-2 columns are real: the tensor cores idle, the instruction
// stream is short.
//
// Structure (as in decode_fused.cu): one CTA per SM, a producer warp that
// keeps a ring of 16 KB shared-memory stages filled, and consumer warps that
// claim the CTA's stream units in order. Weight tiles arrive by TMA
// (cp.async.bulk.tensor, mbarrier completion) through a 3-D view of each
// weight matrix: 64 columns, then rows, then blocks of 64 columns. A box
// lands as [column block][row][64 columns] with the 128-byte swizzle, which
// XORs the 16-byte chunk index with the row, so the 8 row addresses of an
// ldmatrix fall in distinct banks; one copy moves 8 KB (8 gate or 8 up rows
// x 512 columns) or 16 KB (16 down rows x the expert width). Router rows are
// one untiled bulk copy each.
//
//   router row  one fp32 router row (4H bytes, no padding), on the CUDA cores
//   chunk       gate rows p..p+7 and up rows p..p+7 over 512 columns; a chunk
//               unit is the H/512 such stages, all taken by one warp, whose
//               accumulators then hold gate.x and up.x of 8 rows: SwiGLU
//               happens in the lane, no cross-warp sum is needed
//   tile        16 down rows over the whole expert width (<= 512), against
//               the expert's h rows, which each warp copies into its own
//               area of shared memory when it moves to another expert
//
// Each CTA streams contiguous shares of, in order:
//
//   A   router rows                                           -> grid barrier
//   Cs  the shared MLP's gate/up chunks: they need no routing, so their
//       copies fill the ring during the barrier and the routing (which every
//       CTA does itself, as in decode_fused.cu)
//   C   the selected experts' gate/up chunks
//   Ds  the shared MLP's down tiles
//   D   the selected experts' down tiles, weighted by the routing
//
// Each h row is released to a counter (one per selected expert, one for the
// shared MLP) by the lane that wrote it; a down tile starts once its counter
// shows all of h. Only the router rows precede the barrier, so every CTA
// reaches it after the same amount of streaming.
//
// h is kept as two bf16 planes, h_hi = bf16(h) and h_lo = bf16(h - h_hi)
// (about 16 significant bits, as on the tensor-core expert path), and a down
// tile adds W.h_hi and W.h_lo in fp32: with h rounded once to bf16, outputs
// near |y| = 6 miss a 2e-2 max-abs bar. Logits, gate/up and down sums are
// fp32. Output rows are counted and combined as in fused_common.cuh. Every
// wait is bounded.
#include <cudaTypedefs.h>

#include "fused_common.cuh"
#include "route_block.cuh"

namespace moe {

namespace {

using namespace fused;

constexpr int kWarps = 8;
constexpr int kConsumers = kWarps * 32;
constexpr int kThreads = kConsumers + 32;  // + the producer warp
constexpr int kMaxT = 2;
constexpr int kSlice = 512;             // columns of a chunk stage; the largest expert width
constexpr int kKSteps = kSlice / 16;    // mma k-steps per stage
constexpr int kPitch = kSlice * 2 + 16;  // bytes between the rows of a warp's h area
constexpr int kStageBytes = 16384;       // 16 rows x 512 columns bf16, or one fp32 router row
constexpr int kMaxStages = 16;
constexpr int kMinStages = 4;
constexpr int kMaxPend = 8;   // uncounted output rows per lane (4 per tile)
constexpr int kSmemBudget = 227 * 1024;

// The kinds of stream units, in stream order.
enum Kind { kRouter, kSharedChunk, kChunk, kSharedTile, kTile, kNumKinds };

// Dynamic shared memory after the ring: each warp's h area (2 planes x T rows,
// kPitch apart), routing scratch, the token rows (bf16, for the router rows),
// the token rows as mma B fragments, the expert bias.
__host__ __device__ __forceinline__ size_t harea_bytes(int T) { return (size_t)2 * T * kPitch; }
__host__ __device__ __forceinline__ size_t xfrag_bytes(int T, int H) { return (size_t)(H / 16) * T * 4 * 8; }
__host__ __device__ __forceinline__ size_t extra_bytes(int T, int E, int H) {
  return kWarps * harea_bytes(T) + block_route::scratch_bytes(T, E) + (size_t)T * H * 2 + xfrag_bytes(T, H) +
         (size_t)E * 4;
}

// Units of each kind in the whole grid and stages per unit.
__device__ __forceinline__ int kind_units(const DecodeArgs& a, int n_act, int kind) {
  switch (kind) {
    case kRouter: return a.logits_override == nullptr ? a.E : 0;
    case kSharedChunk: return a.ws_gate_up != nullptr ? a.Is / 8 : 0;
    case kSharedTile: return a.ws_down != nullptr ? a.H / 16 : 0;
    case kChunk: return n_act * (a.I / 8);
    default: return n_act * (a.H / 16);
  }
}
__device__ __forceinline__ int kind_stages(const DecodeArgs& a, int kind) {
  return kind == kSharedChunk || kind == kChunk ? a.H / kSlice : 1;
}

// This CTA's stream: per kind, its share of the units and the stream index of
// its first unit and first stage. kChunk and kTile need the routing.
struct Stream {
  Range r[kNumKinds];
  uint32_t unit0[kNumKinds + 1], stage0[kNumKinds + 1];
};

// Chunks are the coarse units (H/512 stages each), so their split decides the
// balance: when there are no more shared chunks than CTAs, CTA b < ns takes
// shared chunk b (known before the routing, so it can be prefetched), and the
// routed chunks fill every CTA up to an even share of all chunks: CTA b takes
// routed chunks [R(b), R(b+1)), R(b) = floor(W b / G) - min(b, ns), W = ns +
// nr, which is nondecreasing once W >= G (each CTA's share is then >= 1).
// Otherwise both kinds are split evenly on their own, as the other kinds are.
__device__ __forceinline__ Stream make_stream(const DecodeArgs& a, int n_act) {
  const int G = gridDim.x, b = blockIdx.x;
  Stream m;
  for (int k = 0; k < kNumKinds; ++k) m.r[k] = split(kind_units(a, n_act, k), b, G);
  const int ns = kind_units(a, n_act, kSharedChunk), nr = kind_units(a, n_act, kChunk), W = ns + nr;
  if (ns <= G) {
    m.r[kSharedChunk] = b < ns ? Range{b, 1} : Range{0, 0};
    if (W >= G) {
      const int lo = (int)((int64_t)W * b / G) - min(b, ns), hi = (int)((int64_t)W * (b + 1) / G) - min(b + 1, ns);
      m.r[kChunk] = Range{lo, hi - lo};
    }
  }
  m.unit0[0] = m.stage0[0] = 0;
  for (int k = 0; k < kNumKinds; ++k) {
    m.unit0[k + 1] = m.unit0[k] + m.r[k].n;
    m.stage0[k + 1] = m.stage0[k] + (uint32_t)m.r[k].n * kind_stages(a, k);
  }
  return m;
}

struct TcSmem {
  uint64_t full[kMaxStages], empty[kMaxStages], route_ready;
  // The stream index each slot was last filled with: a warp can reach a slot
  // while the slot's previous fill is still in flight, when its parity would
  // read as the phase it waits for.
  volatile uint32_t tag[kMaxStages];
  uint4 zero16;                  // B rows of absent slots read these 16 bytes
  block_route::Smem<kWarps> rt;  // routing state and results
  Stream m;                      // this CTA's stream (the routed kinds once routed)
  int flag;
  volatile int abort;      // a consumer warp stopped before the grid barrier
  unsigned int next_unit;  // the next stream unit a consumer warp may claim
};

// ---------------------------------------------------------------------------
// Tensor-core primitives (sm_80+ warp-level mma, valid on sm_100a)
// ---------------------------------------------------------------------------

// Four 8x8 bf16 matrices from shared memory: lanes 8m..8m+7 give the row
// addresses of matrix m; lane l receives row l/4, columns 2(l%4), +1 of each.
// (The memory clobber keeps it between the stage's wait and its release.)
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}

// d += A (16x16, row-major bf16) * B (16x8, column-major bf16), fp32.
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// h as its two bf16 planes: hi at p, lo (the rounding residual) at p + lo_off.
__device__ __forceinline__ void store_h2(uint16_t* p, int64_t lo_off, float h) {
  const uint16_t hi = f32_to_bf16(h);
  p[0] = hi;
  p[lo_off] = f32_to_bf16(h - __uint_as_float((uint32_t)hi << 16));
}

// One box of a 3-D tensor map into shared memory, completing on bar.
__device__ __forceinline__ void tma_load_3d(const CUtensorMap* map, uint64_t* bar, void* dst, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
      "[%2];" ::"r"(smem_addr(dst)),
      "l"(map), "r"(smem_addr(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Byte offsets of this lane's ldmatrix row in a swizzled box: box row `row`,
// 16-byte chunk 2(4j + c) + lane / 16 of 64-column block j (k-step 4j + c).
// base + c[c] is the offset in block 0; block j adds j * (box rows) * 128.
struct SwzRow {
  uint32_t base;  // row offset
  uint32_t c[4];  // swizzled chunk offsets
};
__device__ __forceinline__ SwzRow swz_row(int row, int lane) {
  SwzRow r;
  r.base = row * 128;
  const int hi = lane >> 4;
#pragma unroll
  for (int c = 0; c < 4; ++c) r.c[c] = (uint32_t)((((c << 1) | hi) ^ (row & 7)) << 4);
  return r;
}

// Frees a stage once every lane of the warp has read it.
__device__ __forceinline__ void release_stage(uint64_t* empty) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(empty);
}

// The next unclaimed stream unit of the CTA, for the whole warp.
__device__ __forceinline__ uint32_t claim_unit(TcSmem& sm) {
  uint32_t u = 0;
  if ((threadIdx.x & 31) == 0) u = atomicAdd(&sm.next_unit, 1u);
  return __shfl_sync(0xffffffffu, u, 0);
}

// ---------------------------------------------------------------------------
// Stage consumers
// ---------------------------------------------------------------------------

// One fp32 router row (H) against the bf16 token rows xs ([T, H]); the logit of
// token t in every lane (T = 1: token 1's is 0).
__device__ __forceinline__ float2 router_row(const unsigned char* st, int H, const uint16_t* xs, int T,
                                             uint64_t* empty) {
  const int lane = threadIdx.x & 31;
  const float4* w = reinterpret_cast<const float4*>(st);
  const uint2* x0 = reinterpret_cast<const uint2*>(xs);
  const uint2* x1 = reinterpret_cast<const uint2*>(xs + H);
  float e0 = 0.f, o0 = 0.f, e1 = 0.f, o1 = 0.f;
#pragma unroll 4
  for (int c = lane; c < H / 4; c += 32) {
    const float4 w4 = w[c];
    const uint2 xa = x0[c];
    e0 = fmaf(w4.x, bf16_lo(xa.x), e0);
    o0 = fmaf(w4.y, bf16_hi(xa.x), o0);
    e0 = fmaf(w4.z, bf16_lo(xa.y), e0);
    o0 = fmaf(w4.w, bf16_hi(xa.y), o0);
    if (T > 1) {
      const uint2 xb = x1[c];
      e1 = fmaf(w4.x, bf16_lo(xb.x), e1);
      o1 = fmaf(w4.y, bf16_hi(xb.x), o1);
      e1 = fmaf(w4.z, bf16_lo(xb.y), e1);
      o1 = fmaf(w4.w, bf16_hi(xb.y), o1);
    }
  }
  release_stage(empty);
  return make_float2(warp_sum(e0 + o0), warp_sum(e1 + o1));
}

// Independent accumulator chains of the mma loops (k-step i adds into chain
// i % kChains): a chain is a dependent sequence of mmas, so more chains mean
// a shorter stage for the warp that holds it.
constexpr int kChains = 4;

// Sum of the chains, in a fixed order.
__device__ __forceinline__ float chain_sum(const float (&acc)[kChains][4], int i) {
  return (acc[0][i] + acc[1][i]) + (acc[2][i] + acc[3][i]);
}

// The k-steps of one chunk stage: 16 rows (8 gate, 8 up) x 512 columns against
// the token rows' B fragments xf (this stage's 32 k-steps, T per k-step).
// The stage holds the gate box (8 rows) at 0 and the up box at 8 KB, each
// [8 column blocks][8 rows][64 columns] swizzled: tile row m is box row m % 8
// of box m / 8.
__device__ __forceinline__ void chunk_stage(const unsigned char* st, const uint2* xf, int T,
                                            float (&acc)[kChains][4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3, m = lane & 15;
  const SwzRow w = swz_row(m & 7, lane);
  const uint32_t base = smem_addr(st) + (m >> 3) * 8192 + w.base;
  const bool has_b = g < T;
  static_assert(kChains == 4, "one 64-column block per group of kChains k-steps");
#pragma unroll 2
  for (int ks = 0; ks < kKSteps; ks += kChains) {
#pragma unroll
    for (int c = 0; c < kChains; ++c) {
      uint32_t a[4];
      ldsm_x4(base + (ks >> 2) * 1024 + w.c[c], a);
      const uint2 b = has_b ? xf[((ks + c) * T + g) * 4 + t] : make_uint2(0u, 0u);
      mma_bf16(acc[c], a, b.x, b.y);
    }
  }
}

// Chunks are streamed in groups of up to kGroup, their stages interleaved
// (stage sj of every chunk of the group, then stage sj + 1, ...), so the warps
// that hold a group's chunks all have a stage in the ring at once.
constexpr int kGroup = kWarps;

// Stream index of stage 0 of chunk uu (of n in this CTA's share of a chunk
// kind whose first stage is v0), and the distance between its stages.
__device__ __forceinline__ uint32_t chunk_first(uint32_t v0, uint32_t uu, int n, int nk, int* stride) {
  const uint32_t g = uu / kGroup, pos = uu - g * kGroup;
  *stride = min(kGroup, n - (int)(g * kGroup));
  return v0 + g * kGroup * nk + pos;
}

// One chunk: stages v0, v0 + stride, ... (nk of them, waited for with stage),
// summed in acc; false on a timeout.
template <class StageFn>
__device__ __forceinline__ bool run_chunk(StageFn& stage, uint32_t v0, int stride, int nk, const uint2* xf, int T,
                                          float (&acc)[kChains][4]) {
#pragma unroll
  for (int c = 0; c < kChains; ++c)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[c][i] = 0.f;
  for (int sj = 0; sj < nk; ++sj) {
    const unsigned char* st;
    uint64_t* empty;
    if (!stage(v0 + (uint32_t)(sj * stride), &st, &empty)) return false;
    chunk_stage(st, xf + (size_t)sj * kKSteps * T * 4, T, acc);
    release_stage(empty);
  }
  return true;
}

// One tile: 16 down rows x K (<= 512, a multiple of 64; the stage holds the
// box [K/64 column blocks][16 rows][64 columns] swizzled) against the h rows in
// the warp's area (plane p, row n at p*T + n rows of kPitch bytes; rows n >=
// nt read the zero block). Chains 0 and 2 get W.h_hi, 1 and 3 W.h_lo (even and
// odd k-steps). The B fragments
// come from one ldmatrix.x4 per k-step: matrices (h_hi, k0), (h_hi, k0 + 8),
// (h_lo, k0), (h_lo, k0 + 8), whose 8 rows are the 8 columns n of B.
__device__ __forceinline__ void tile_stage(const unsigned char* st, int K, const unsigned char* harea, int T, int nt,
                                           const uint4* zero16, float (&acc)[kChains][4]) {
  const int lane = threadIdx.x & 31, mat = lane >> 3, n = lane & 7;
  const SwzRow w = swz_row(lane & 15, lane);
  const uint32_t a_base = smem_addr(st) + w.base;
  const bool real = n < nt;
  const uint32_t b_base =
      real ? smem_addr(harea) + ((mat >> 1) * T + n) * kPitch + (mat & 1) * 16 : smem_addr(zero16);
  const uint32_t b_step = real ? 32u : 0u;
  const int nks = K / 16;
  auto step = [&](int ks, uint32_t chunk, float (&hi)[4], float (&lo)[4]) {
    uint32_t wa[4], h[4];
    ldsm_x4(a_base + (ks >> 2) * 2048 + chunk, wa);
    ldsm_x4(b_base + ks * b_step, h);
    mma_bf16(hi, wa, h[0], h[1]);
    mma_bf16(lo, wa, h[2], h[3]);
  };
  // nks is a multiple of 4 (K % 64 == 0)
#pragma unroll 2
  for (int ks = 0; ks < nks; ks += 4) {
    step(ks, w.c[0], acc[0], acc[1]);
    step(ks + 1, w.c[1], acc[2], acc[3]);
    step(ks + 2, w.c[2], acc[0], acc[1]);
    step(ks + 3, w.c[3], acc[2], acc[3]);
  }
}

// Copies up to two h rows of length K (both planes: hi at r, lo at r + lo_off
// elements) into the warp's area; r1 null: one row.
__device__ __forceinline__ void stage_h(unsigned char* harea, int T, const uint16_t* r0, const uint16_t* r1, int K,
                                        int64_t lo_off) {
  const int lane = threadIdx.x & 31;
  const int nt = r1 != nullptr ? 2 : 1, nc = K / 8;
  for (int i = lane; i < 2 * nt * nc; i += 32) {
    const int c = i % nc, n = (i / nc) % nt, pl = i / (nc * nt);
    const uint16_t* src = (n == 0 ? r0 : r1) + (pl ? lo_off : 0) + c * 8;
    *reinterpret_cast<uint4*>(harea + (pl * T + n) * kPitch + c * 16) = __ldcg(reinterpret_cast<const uint4*>(src));
  }
  __syncwarp();
}

// ---------------------------------------------------------------------------
// The producer warp: issues the CTA's stream in order, stage v into ring slot
// v % depth once the consumers freed the slot's previous stage. Every lane
// waits; lane 0 arms the stage's barrier; lane r issues the copy of tile row
// r, so the 16 row copies of a stage cost one pass of the warp.
// ---------------------------------------------------------------------------
// The weight views the producer copies from (3-D tensor maps, see the top).
struct TcMaps {
  CUtensorMap gu, sgu;  // [E*2I, H], [2Is, H]: boxes of 8 rows x 512 columns
  CUtensorMap dn, sdn;  // [E*H, I], [H, Is]: boxes of 16 rows x the whole row
};

__device__ void producer(const DecodeArgs& a, const TcMaps& maps, unsigned char* ring, int depth, TcSmem& sm) {
  const int H = a.H, I = a.I;
  const int lane = threadIdx.x & 31;
  Stream m = make_stream(a, 0);
  uint32_t v = 0;
  bool ok = true;
  for (int kind = 0; kind < kNumKinds && ok; ++kind) {
    if (kind == kChunk) {  // the rest needs this CTA's routing
      ok = __all_sync(0xffffffffu, thread_wait_phase(&sm.route_ready, 0, a.hdr, 500));
      if (!ok) break;
      m = make_stream(a, sm.rt.n_act);
    }
    // stages in stream order: chunks in groups with interleaved stages (see
    // chunk_first), every other unit one stage
    const int spu = kind_stages(a, kind), lo = m.r[kind].lo, n_units = m.r[kind].n;
    const int gsz = spu > 1 ? kGroup : 1;
    for (int g0 = 0; g0 < n_units && ok; g0 += gsz) {
      const int gs = min(gsz, n_units - g0);
      for (int sj = 0; sj < spu && ok; ++sj)
        for (int pos = 0; pos < gs; ++pos, ++v) {
          const int q = lo + g0 + pos;
          const int s = (int)(v % (uint32_t)depth);
          const uint32_t n = v / (uint32_t)depth;
          if (!__all_sync(0xffffffffu, n == 0 || thread_wait_phase(&sm.empty[s], (n - 1) & 1u, a.hdr, 400 + s))) {
            ok = false;
            break;
          }
          if (lane == 0) {
            unsigned char* dst = ring + (size_t)s * kStageBytes;
            uint64_t* full = &sm.full[s];
            sm.tag[s] = v;  // the slot's previous fill is consumed: its phase is complete
            if (kind == kRouter) {
              mbar_expect_tx(full, 4u * H);
              bulk_load(dst, a.router_w + (int64_t)q * H, 4u * H, full);
            } else if (kind == kSharedChunk || kind == kChunk) {
              // gate rows p..p+7 and up rows p..p+7, columns 512 sj .. 512 sj + 511
              const CUtensorMap* map = kind == kSharedChunk ? &maps.sgu : &maps.gu;
              int gate_row, up_row;
              if (kind == kSharedChunk) {
                gate_row = q * 8;
                up_row = a.Is + q * 8;
              } else {
                const int per = I / 8, ai = q / per, p = (q - ai * per) * 8;
                gate_row = sm.rt.act_e[ai] * 2 * I + p;
                up_row = gate_row + I;
              }
              mbar_expect_tx(full, kStageBytes);
              tma_load_3d(map, full, dst, 0, gate_row, sj * (kSlice / 64));
              tma_load_3d(map, full, dst + kStageBytes / 2, 0, up_row, sj * (kSlice / 64));
            } else {
              // down rows n0..n0+15, all columns, of the shared MLP or of a selected expert
              int row, K;
              const CUtensorMap* map;
              if (kind == kSharedTile) {
                row = q * 16;
                K = a.Is;
                map = &maps.sdn;
              } else {
                const int per = H / 16, ai = q / per;
                row = sm.rt.act_e[ai] * H + (q - ai * per) * 16;
                K = I;
                map = &maps.dn;
              }
              mbar_expect_tx(full, 32u * K);
              tma_load_3d(map, full, dst, 0, row, 0);
            }
          }
          __syncwarp();
        }
    }
  }
  if (!ok && lane == 0) {
    // the consumers stopped: wait (bounded) for the copies still in flight
    const uint32_t first = v > (uint32_t)depth ? v - depth : 0u;
    for (uint32_t w = first; w < v; ++w) thread_wait_phase(&sm.full[w % depth], (w / depth) & 1u, nullptr, 0);
  }
}

// ---------------------------------------------------------------------------
// A consumer warp: claims its CTA's stream units in order.
// ---------------------------------------------------------------------------
__device__ void consumer(const DecodeArgs& a, const unsigned char* ring, int depth, unsigned char* scratch,
                         TcSmem& sm) {
  const int T = a.T, k = a.k, H = a.H, I = a.I, Is = a.Is, E = a.E;
  const int lane = threadIdx.x & 31, g = lane >> 2, t4 = lane & 3;
  const int nk = H / kSlice;  // stages per chunk
  int32_t* done = a.sync;     // [kMaxSlots]: h rows finished per distinct expert
  int32_t* done_shared = a.sync + kMaxSlots + kMaxT * H;  // and of the shared MLP, after the row counters
  // h as two bf16 planes: hi [T*k, I] then lo [T*k, I]; the shared MLP's hi
  // [T, Is] then lo [T, Is]
  uint16_t* h16 = reinterpret_cast<uint16_t*>(a.h);
  uint16_t* hs16 = reinterpret_cast<uint16_t*>(a.h_shared);
  const int64_t h_lo = (int64_t)T * k * I, hs_lo = (int64_t)T * Is;
  auto consumer_sync = [] { asm volatile("bar.sync 1, %0;" ::"n"(kConsumers) : "memory"); };

  // counters: each CTA zeroes its share; the grid barrier orders it before use
  const Range z = split(kMaxSlots + kMaxT * H + 1, blockIdx.x, gridDim.x);
  for (int i = threadIdx.x; i < z.n; i += kConsumers) a.sync[z.lo + i] = 0;

  // the token rows (bf16, for the router rows) and their mma B fragments
  // (k-step ks, token g, lane t: columns 16ks + 2t, +1 and 16ks + 8 + 2t, +1)
  unsigned char* harea = scratch + (size_t)(threadIdx.x >> 5) * harea_bytes(T);  // this warp's h rows
  unsigned char* rscratch = scratch + kWarps * harea_bytes(T);                   // routing scratch
  unsigned char* p = rscratch + block_route::scratch_bytes(T, E);
  uint16_t* xs = reinterpret_cast<uint16_t*>(p);
  p += (size_t)T * H * 2;
  uint2* xf = reinterpret_cast<uint2*>(p);
  p += xfrag_bytes(T, H);
  float* bias_s = a.expert_bias != nullptr ? reinterpret_cast<float*>(p) : nullptr;
  for (int i = threadIdx.x; i < T * H / 8; i += kConsumers)
    reinterpret_cast<uint4*>(xs)[i] = ld_nc_u4(a.x + (size_t)i * 8);
  for (int i = threadIdx.x; i < (H / 16) * T * 4; i += kConsumers) {
    const int t = i & 3, tok = (i >> 2) % T, ks = (i >> 2) / T;
    const unsigned int* row = reinterpret_cast<const unsigned int*>(a.x + (size_t)tok * H + ks * 16 + 2 * t);
    xf[i] = make_uint2(__ldg(row), __ldg(row + 4));
  }
  if (bias_s != nullptr)
    for (int e = threadIdx.x; e < E; e += kConsumers) bias_s[e] = __ldg(a.expert_bias + e);
  if (threadIdx.x == 0) sm.m = make_stream(a, 0);
  consumer_sync();

  const float* logits = a.logits_override != nullptr ? a.logits_override : a.logits;
  const bool pre_scores = block_route::scores_with_logits(a);
  const int target = k + (a.ws_down != nullptr ? 1 : 0);
  Pending<kMaxPend> q;
  q.np = 0;
  // Waits for stream stage v; counts the pending rows first if it would block.
  auto stage = [&](uint32_t v, const unsigned char** st, uint64_t** empty) {
    const int s = (int)(v % (uint32_t)depth);
    const uint32_t parity = (v / (uint32_t)depth) & 1u;
    *st = ring + (size_t)s * kStageBytes;
    *empty = &sm.empty[s];
    if (__all_sync(0xffffffffu, sm.tag[s] == v && mbar_try_wait(&sm.full[s], parity))) return true;
    if (q.np > 0) publish(a, q, target);
    return warp_wait_tag(&sm.tag[s], v, a.hdr, 300 + s) && warp_wait_phase(&sm.full[s], parity, a.hdr, 300 + s);
  };

  // ---- A: router rows ----
  // A warp whose wait runs out must still reach the named barriers below (they
  // have no timeout): it flags the CTA, and the consumers leave together after
  // the grid barrier.
  const Stream& m = sm.m;
  uint32_t carried;  // a unit claimed past phase A, processed after the routing
  for (;;) {
    const uint32_t u = claim_unit(sm);
    if (u >= m.unit0[kSharedChunk]) {
      carried = u;
      break;
    }
    const int i = m.r[kRouter].lo + (int)u;
    const unsigned char* st;
    uint64_t* empty;
    if (!stage(m.stage0[kRouter] + u, &st, &empty)) {
      sm.abort = 1;
      carried = 0xffffffffu;
      break;
    }
    const float2 lg = router_row(st, H, xs, T, empty);
    if (lane < T) {  // lane t: token t
      const float v = lane == 0 ? lg.x : lg.y;
      a.logits[lane * E + i] = v;
      if (pre_scores) block_route::store_score(a, lane, i, v, bias_s);
    }
  }
  if (!grid_barrier<kConsumers>(a.hdr, 1, &sm.flag) || sm.abort != 0) return;

  // ---- routing; then the producer may issue the selected experts' rows ----
  block_route::route_block<kWarps>(a, logits, bias_s, rscratch, sm.rt);
  if (threadIdx.x == 0) {
    sm.m = make_stream(a, sm.rt.n_act);
    mbar_arrive(&sm.route_ready);
  }
  consumer_sync();

  int hb_key = -1;  // whose h rows the warp's area holds: -2 the shared MLP, e >= 0 distinct expert e
  int nt = 0;       // and how many
  for (uint32_t u = carried;; u = claim_unit(sm)) {
    if (u >= m.unit0[kNumKinds]) break;
    int kind = kSharedChunk;
    while (u >= m.unit0[kind + 1]) ++kind;
    const uint32_t uu = u - m.unit0[kind];
    const int qi = m.r[kind].lo + (int)uu;
    if (kind == kSharedChunk) {  // ---- 8 gate/up pairs of the shared MLP ----
      float acc[kChains][4];
      int stride;
      const uint32_t v0 = chunk_first(m.stage0[kSharedChunk], uu, m.r[kSharedChunk].n, nk, &stride);
      if (!run_chunk(stage, v0, stride, nk, xf, T, acc)) return;
      if (t4 == 0) {  // lane 4g: gate . x_t in d[t], up . x_t in d[2 + t] of pair 8qi + g
#pragma unroll
        for (int t = 0; t < kMaxT; ++t)
          if (t < T) store_h2(hs16 + t * Is + 8 * qi + g, hs_lo, silu_f32(chain_sum(acc, t)) * chain_sum(acc, 2 + t));
        red_release_add(done_shared, T);
      }
      continue;
    }
    if (kind == kChunk) {  // ---- 8 gate/up pairs of a selected expert ----
      const int per = I / 8, ai = qi / per, p8 = (qi - ai * per) * 8;
      const int slA = sm.rt.act_a[ai], slB = sm.rt.act_b[ai];
      float acc[kChains][4];
      int stride;
      const uint32_t v0 = chunk_first(m.stage0[kChunk], uu, m.r[kChunk].n, nk, &stride);
      if (!run_chunk(stage, v0, stride, nk, xf, T, acc)) return;
      if (t4 == 0) {
        const float h0 = silu_f32(chain_sum(acc, 0)) * chain_sum(acc, 2);  // token 0
        const float h1 = silu_f32(chain_sum(acc, 1)) * chain_sum(acc, 3);  // token 1
        store_h2(h16 + (int64_t)slA * I + p8 + g, h_lo, slA / k == 0 ? h0 : h1);
        if (slB >= 0) store_h2(h16 + (int64_t)slB * I + p8 + g, h_lo, slB / k == 0 ? h0 : h1);
        // the down tiles of this expert wait for I rows per slot holding it
        red_release_add(done + ai, slB >= 0 ? 2 : 1);
      }
      continue;
    }
    // ---- a tile of 16 down rows: the shared MLP's (S) or a selected expert's (D) ----
    int K, n0, ai = -1, slA = 0, slB = -1;
    if (kind == kSharedTile) {
      K = Is;
      n0 = qi * 16;
    } else {
      const int per = H / 16;
      ai = qi / per;
      n0 = (qi - ai * per) * 16;
      K = I;
      slA = sm.rt.act_a[ai];
      slB = sm.rt.act_b[ai];
    }
    const int key = kind == kSharedTile ? -2 : ai;
    if (key != hb_key) {
      if (kind == kTile) {
        const int need = slB >= 0 ? 2 * I : I;
        const int complete = lane == 0 ? ld_acquire(done + ai) >= need : 0;
        if (!__shfl_sync(0xffffffffu, complete, 0)) {
          if (q.np > 0) publish(a, q, target);
          if (!warp_wait_count(done + ai, need, a.hdr, 200 + ai)) return;
        }
        __syncwarp();
        stage_h(harea, T, h16 + (int64_t)slA * I, slB >= 0 ? h16 + (int64_t)slB * I : nullptr, I, h_lo);
        nt = slB >= 0 ? 2 : 1;
      } else {
        // all of the shared MLP's h: Is rows per token
        const int complete = lane == 0 ? ld_acquire(done_shared) >= Is * T : 0;
        if (!__shfl_sync(0xffffffffu, complete, 0)) {
          if (q.np > 0) publish(a, q, target);
          if (!warp_wait_count(done_shared, Is * T, a.hdr, 250)) return;
        }
        __syncwarp();
        stage_h(harea, T, hs16, T > 1 ? hs16 + Is : nullptr, Is, hs_lo);
        nt = T;
      }
      hb_key = key;
    }
    const unsigned char* st;
    uint64_t* empty;
    if (!stage(m.stage0[kind] + uu, &st, &empty)) return;
    float acc[kChains][4];
#pragma unroll
    for (int c = 0; c < kChains; ++c)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[c][i] = 0.f;
    tile_stage(st, K, harea, T, nt, &sm.zero16, acc);
    release_stage(empty);
    // lane 4g holds rows n0 + g (d0: column 0, d1: column 1) and n0 + g + 8 (d2, d3)
    int idx[4] = {-1, -1, -1, -1};
    if (t4 == 0) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int row = n0 + g + 8 * (j >> 1), c = j & 1;
        const float val = chain_sum(acc, j);
        if (kind == kSharedTile) {
          if (c < T) {
            a.shared_out[(int64_t)c * H + row] = val;
            idx[j] = c * H + row;
          }
        } else {
          const int sl = c == 0 ? slA : slB;
          if (sl >= 0) {
            a.y_slots[(int64_t)sl * H + row] = sm.rt.w[sl] * val;
            idx[j] = (sl / k) * H + row;
          }
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) add_pending(q, idx[j]);
    if (q.np > kMaxPend - 4) publish(a, q, target);
  }
  publish(a, q, target);
}

__global__ void __launch_bounds__(kThreads, 1)
    decode_tc_kernel(const DecodeArgs a, const __grid_constant__ TcMaps maps, const int depth) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  __shared__ TcSmem sm;
  // swizzled boxes need 1024-byte aligned destinations
  unsigned char* ring = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  unsigned char* scratch = ring + (size_t)depth * kStageBytes;
  if (threadIdx.x == 0) {
    for (int s = 0; s < depth; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
      sm.tag[s] = 0xffffffffu;
    }
    mbar_init(&sm.route_ready, 1);
    sm.abort = 0;
    sm.next_unit = 0;
    sm.zero16 = make_uint4(0u, 0u, 0u, 0u);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x >= kConsumers) {
    producer(a, maps, ring, depth, sm);
    return;
  }
  consumer(a, ring, depth, scratch, sm);
}

// Ring stages that fit next to the rest of shared memory (the static TcSmem,
// counted in whole KB since the compiler may pad it, and the 1 KB that
// aligning the ring may cost); 0 when too few.
int tc_depth(int T, int E, int H) {
  const int64_t static_bytes = ((int64_t)sizeof(TcSmem) + 1023) / 1024 * 1024;
  const int64_t avail = (int64_t)kSmemBudget - static_bytes - (int64_t)extra_bytes(T, E, H) - 1024;
  int64_t d = avail / kStageBytes;
  if (d > kMaxStages) d = kMaxStages;
  return d >= kMinStages ? (int)d : 0;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// The 3-D view of a row-major bf16 matrix [rows, cols] (cols a multiple of
// 64): {64 columns, rows, cols / 64 column blocks}, strides {2 cols, 128}
// bytes, boxes of {64, box_rows, box_blocks} with the 128-byte swizzle.
bool make_map3(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows, int box_blocks) {
  EncodeTiledFn fn = encode_tiled();
  if (fn == nullptr || cols % 64 != 0 || rows < 1) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)rows, (cuuint64_t)(cols / 64)};
  cuuint64_t strides[2] = {(cuuint64_t)cols * 2, 128};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, (cuuint32_t)box_blocks};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool decode_tc_supported(int64_t T, int k, int E, int H, int I, int Is) {
  return T >= 1 && T <= kMaxT && k >= 1 && k <= E && E <= 1024 && T * k <= kMaxSlots &&  // routing
         H >= kSlice && H % kSlice == 0 && 4 * H <= kStageBytes &&                      // a router row per stage
         I >= 64 && I % 64 == 0 && I <= kSlice && (Is == 0 || (Is % 64 == 0 && Is <= kSlice)) &&
         tc_depth((int)T, E, H) > 0;
}

cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t s) {
  if (!decode_tc_supported(a.T, a.k, a.E, a.H, a.I, a.ws_down != nullptr ? a.Is : 0)) return cudaErrorNotSupported;
  const int depth = tc_depth(a.T, a.E, a.H);
  const size_t smem = (size_t)depth * kStageBytes + extra_bytes(a.T, a.E, a.H) + 1024;
  TcMaps maps;
  const bool shared = a.ws_down != nullptr && a.Is > 0;
  // a weight view the driver refuses: no launch (reported as an invalid resource)
  if (!make_map3(&maps.gu, a.w_gate_up, (int64_t)a.E * 2 * a.I, a.H, 8, kSlice / 64) ||
      !make_map3(&maps.dn, a.w_down, (int64_t)a.E * a.H, a.I, 16, a.I / 64))
    return cudaErrorInvalidResourceHandle;
  if (shared) {
    if (!make_map3(&maps.sgu, a.ws_gate_up, 2 * (int64_t)a.Is, a.H, 8, kSlice / 64) ||
        !make_map3(&maps.sdn, a.ws_down, a.H, a.Is, 16, a.Is / 64))
      return cudaErrorInvalidResourceHandle;
  } else {
    maps.sgu = maps.gu;  // never read
    maps.sdn = maps.dn;
  }
  cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_tc_kernel, kThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sm_count());  // one CTA per SM, all resident: the grid barrier and the waits rely on it
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  before_launch(MOE_KERNEL_DECODE_FUSED, s);
  e = cudaLaunchKernelEx(&cfg, decode_tc_kernel, a, maps, depth);
  after_launch(MOE_KERNEL_DECODE_FUSED, s);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace moe
