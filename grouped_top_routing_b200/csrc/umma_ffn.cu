// Expert FFN on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// Each routed expert (and the shared MLP) is a dense contraction over the
// tokens routed to it: the gather-matmul of mlxcel issue #838 (section
// "Weight remap": experts stacked into switch_mlp tensors; section
// "Architecture notes": SwiGLU experts plus one always-on shared MLP).
//
// Orientation: the weight rows are the MMA's M side (128 rows per operand) and
// the expert's tokens its N side (BN columns), so an expert that received only
// a handful of tokens still fills the 128-row tensor-core tile, and every
// weight tile is read from HBM once per BN tokens.
//
//   pass GATE_UP: D0 = W_gate[n0:n0+128] . X^T, D1 = W_up[n0:n0+128] . X^T,
//                 h[token, n0+i] = silu(D0[i]) * D1[i]  -> (h_hi, h_lo)
//   pass DOWN   : D = W_down[n0:n0+128] . [H_hi | H_lo]^T   (one MMA of N = 2 BN),
//                 y_slots[slot(token), n] = w_slot * (D_hi[n] + D_lo[n])
//                 (fp32; shared MLP: weight 1)
//
// With bf16 down weights, h is written as two bf16 planes, h_hi = bf16(h) and
// h_lo = bf16(h - h_hi). The DOWN stage holds the token tile of each plane back
// to back, so the pair is a single B operand of 2 BN rows: one MMA per weight
// tile yields both W.h_hi and W.h_lo, which the epilogue adds. The SwiGLU
// product thus carries ~16 significant bits into the down projection, at twice
// the down pass's tensor work.
//
// With an fp16 copy of the down weights (exact for bf16 values of magnitude
// 2^-14 or more), h is written as one fp16 plane (11 significant bits) and the
// down pass runs kind::f16 MMAs on fp16 operands: one MMA per k-step and half
// the h bytes. A SwiGLU product beyond fp16's range is recorded as
// MOE_ERR_RANGE.
//
// Persistent, warp-specialised CTA (one per SM, 192 threads):
//   warp 0      : TMA producer (one lane), STAGES-deep ring of weight and token tiles
//   warp 1      : TMEM allocator; one lane issues tcgen05.mma, commits to barriers
//   warps 2..5  : epilogue; TMEM -> registers (tcgen05.ld), SwiGLU / weighting, stores
// The two TMEM accumulator pairs are double-buffered so the epilogue of one tile
// overlaps the main loop of the next. Tiles run (group, n-block, m-block) with
// the m-block fastest, so CTAs that share a weight block run side by side and
// its re-reads hit L2; token-major groups with many m-blocks and weights that
// fit in L2 run (group, m-block, n-block) instead, so the tiles sharing a token
// tile do (see decode_tile).
//
// Every mbarrier wait is bounded (globaltimer; the call's moe_options.wait_limit_ns,
// 2 s by default). A wait that runs out sets
// MOE_ERR_TIMEOUT in the workspace, raises a CTA-wide abort flag, and all roles
// wind down: the producer waits (bounded) for its copies in flight, the MMA lane
// waits (bounded) for its MMAs, and TMEM is freed before the CTA exits.
#include <cuda.h>

#include "common.cuh"
#include "ffn.cuh"
#include "mbarrier.cuh"

namespace moe {

namespace {

constexpr int BM = 128;         // weight rows per A operand (MMA M)
constexpr int BK = 64;          // K per stage: 64 bf16 = 128 bytes = one swizzle span
constexpr int kThreads = 192;
constexpr int kMaxGroups = 1025;  // routed experts (<= 1024) + the shared MLP

// Modes. kGateUp / kDown: weight rows are the MMA's M side, the expert's
// tokens its N side (skinny experts). kGateUpTM / kDownTM ("token-major", for
// experts with many rows): 128 token rows are M and 256 weight rows N, one
// 128 x 256 MMA per k-step, which reads less shared memory per flop.
enum : int { kGateUp = 0, kDown = 1, kLogits = 2, kGateUpTM = 3, kDownTM = 4 };
constexpr bool token_major(int mode) { return mode == kGateUpTM || mode == kDownTM; }
constexpr int kLogitsBN = 64;  // token columns per logits tile; chunk sums live in registers
// The router-logits GEMM accumulates at most this many k-blocks (32 MMAs of
// K = 16) in one TMEM accumulator; the epilogue adds the chunk sums in fp32
// registers. Long tensor-core accumulation chains drift (measured: error
// grows with the chain length), short ones stay within a few fp32 ulps.
constexpr int kLogitsChunk = 8;

struct UmmaParams {
  int64_t T;
  int H, I, Is, k, E;
  int has_shared;
  const int32_t* offsets;
  const int32_t* tok_of;
  const int32_t* active;
  WsHeader* hdr;
  const float* topk_w;
  uint16_t* h_perm;    // hi plane [T*k, I], lo plane follows
  uint16_t* h_shared;  // hi plane [T, Is], lo plane follows
  float* y_slots;
  float* shared_out;
  // router-logits mode: A = the three bf16 planes of the router weight [3E, H]
  float* logits_out;  // [ksplit, T, E] partial sums (ksplit == 1: the logits)
  int ksplit, kper, kbH;
  uint64_t wait_ns;  // bound on every mbarrier wait
  int withhold;      // test aid: 1 = never hand the first accumulator to the epilogue
  int slots16;       // H16 DOWN: routed slot rows are fp16 (y_slots holds uint16_t), the shared rows fp32
};

// ----------------------------------------------------------------------------
// PTX wrappers
// ----------------------------------------------------------------------------
// Bounded wait for the phase of `bar` with the given parity. Returns false when
// the CTA is aborting or the wait ran out (which raises the abort).
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag, WsHeader* hdr,
                                         int site, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t n = 1;; ++n) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((n & 255u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > limit_ns) {
        *abort_flag = 1;
        record_error(hdr, MOE_ERR_TIMEOUT, site);
        return false;
      }
    }
  }
}

// Bounded wait that ignores the abort flag (used to drain in-flight work).
__device__ __forceinline__ void drain_bar(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer() - t0 > limit_ns) return;
}

__device__ __forceinline__ void tma_load_2d(const CUtensorMap* map, uint64_t* bar, void* dst, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::
          "r"(smem_addr(dst)),
      "l"(map), "r"(smem_addr(bar)), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(slot)), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

// D[tmem] (+)= A[smem] . B[smem]^T, 16-bit inputs (bf16 or fp16, per the
// instruction descriptor), fp32 accumulate, 128 x N x 16.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  const uint32_t z = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(z), "r"(z), "r"(z), "r"(z)
      : "memory");
}

// 32 lanes x 16 consecutive fp32 columns of TMEM into registers.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor: K-major tile, 128-byte swizzle, rows of
// 128 bytes, 8-row groups 1024 bytes apart (the layout a TMA box {64, rows}
// with CU_TENSOR_MAP_SWIZZLE_128B writes).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor, kind::f16: D fp32, A and B both bf16 (format 1) or
// both fp16 (format 0), both K-major.
template <int N>
__device__ __forceinline__ constexpr uint32_t idesc_bf16() {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}
template <int N>
__device__ __forceinline__ constexpr uint32_t idesc_fp16() {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

// ----------------------------------------------------------------------------
// tile schedule
// ----------------------------------------------------------------------------
// Stage = NA weight tiles (128 x 64) then NB token tiles (BN x 64), all
// 1024-byte aligned. GATE_UP / LOGITS: NA = 2, NB = 1 (gate and up rows, or
// two blocks of router rows, share the token tile). DOWN with two h planes:
// NB = 2 (the h_hi and h_lo token tiles, one B operand of 2 BN rows) and
// NA = 2 while the TMEM budget allows (BN <= 64), else 1; with one fp16 plane
// (H16): NB = 1, NA = 2. Each accumulator is NCOL columns.
//
// Token-major modes (BN = 128 token rows): NA = token tiles per stage (1; the
// h_hi and h_lo planes for kDownTM on bf16 weights), NB = 2 weight boxes of
// 128 rows forming one B operand of 256 rows, one accumulator of NCOL = 256.
template <int BN, int MODE, bool H16>
struct Shape {
  static constexpr bool TM = token_major(MODE);
  static constexpr bool kTwoPlanes = (MODE == kDown || MODE == kDownTM) && !H16;  // h_hi and h_lo tiles
  static constexpr int NA = TM ? (MODE == kDownTM && kTwoPlanes ? 2 : 1)
                               : ((MODE == kLogits || (MODE == kDown && kTwoPlanes && BN > 64)) ? 1 : 2);
  static constexpr int NB = TM ? 2 : (MODE == kDown && kTwoPlanes ? 2 : 1);
  static constexpr int NCOL = TM ? 256 : (MODE == kDown && kTwoPlanes ? 2 * BN : BN);
  static constexpr int NACC = TM ? 1 : NA;                         // accumulators per buffer
  static constexpr int ROWS = TM ? (MODE == kDownTM ? 256 : BM) : NA * BM;  // weight rows per tile
  static constexpr uint32_t kTmemCols = 2 * NACC * NCOL;           // two buffers
  static_assert(kTmemCols == 128 || kTmemCols == 256 || kTmemCols == 512, "TMEM allocation");
};

struct TileInfo {
  bool shared;
  int e, m, nb, mb, ks;
  int64_t r0;
  int a0_row, a1_row, b_row, kb0, kblocks, nchunks;
};

template <int BN, int MODE, bool H16>
__device__ __forceinline__ TileInfo decode_tile(int tile, int n_groups, const int* pre, const int16_t* s_e, const int* s_m,
                                                const int* s_r0, const UmmaParams& p) {
  int lo = 0, hi = n_groups - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pre[mid] <= tile) lo = mid;
    else hi = mid - 1;
  }
  TileInfo t;
  t.e = s_e[lo];
  t.shared = t.e < 0;
  t.m = s_m[lo];
  t.r0 = s_r0[lo];
  const int mblocks = (t.m + BN - 1) / BN;
  const int local = tile - pre[lo];
  t.kb0 = 0;
  t.ks = 0;
  if (MODE == kLogits) {  // one group (all tokens); split-K index fastest
    t.ks = local % p.ksplit;
    const int rest = local / p.ksplit;
    t.nb = rest / mblocks;
    t.mb = rest - t.nb * mblocks;
    t.a0_row = t.nb * BM;  // one 128-row block of router rows per tile
    t.a1_row = t.a0_row;
    t.b_row = t.mb * BN;
    t.kb0 = t.ks * p.kper;
    t.kblocks = min(p.kper, 3 * p.kbH - t.kb0);
    t.nchunks = (t.kblocks + kLogitsChunk - 1) / kLogitsChunk;
    return t;
  }
  const int nbl = (pre[lo + 1] - pre[lo]) / mblocks;  // weight blocks of the group in this pass
  // Token-major groups of at least 4 m-blocks whose weights for this pass fit
  // well inside L2 (<= 32 MB) run their weight blocks fastest: the tiles that
  // share a token tile run side by side and read it from L2, and the group's
  // weights stay in L2 across its m-blocks (with m-blocks fastest, about 1.4
  // of each token tile's 8 reads missed L2 at 32768 tokens: 1.43x the gate/up
  // pass's operand bytes from DRAM, against 1.05x). Other groups (few
  // m-blocks, or weights like the 151 MB dense MLP's) keep the m-block
  // fastest, so each weight block is re-read only by concurrent tiles.
  const int Kp = MODE == kGateUpTM ? p.H : (t.shared ? p.Is : p.I);
  if (token_major(MODE) && mblocks >= 4 && (int64_t)nbl * 256 * Kp * 2 <= (int64_t(32) << 20)) {
    t.mb = local / nbl;
    t.nb = local - t.mb * nbl;
  } else {
    t.nb = local / mblocks;
    t.mb = local - t.nb * mblocks;
  }
  int K;
  if (token_major(MODE)) {  // a0/a1 rows: the two 128-row weight boxes; b_row: the token rows
    if (MODE == kGateUpTM) {
      K = p.H;
      t.a0_row = t.shared ? t.nb * BM : t.e * 2 * p.I + t.nb * BM;
      t.a1_row = t.shared ? p.Is + t.nb * BM : t.a0_row + p.I;
    } else {
      K = t.shared ? p.Is : p.I;
      t.a0_row = (t.shared ? 0 : t.e * p.H) + t.nb * 2 * BM;
      t.a1_row = t.a0_row + BM;
    }
  } else if (MODE == kGateUp) {
    K = p.H;
    if (t.shared) {
      t.a0_row = t.nb * BM;
      t.a1_row = p.Is + t.nb * BM;
    } else {
      t.a0_row = t.e * 2 * p.I + t.nb * BM;
      t.a1_row = t.a0_row + p.I;
    }
  } else {
    K = t.shared ? p.Is : p.I;
    t.a0_row = (t.shared ? 0 : t.e * p.H) + t.nb * Shape<BN, MODE, H16>::ROWS;
    t.a1_row = t.a0_row + BM;  // used when the stage holds two weight tiles
  }
  t.b_row = (int)t.r0 + t.mb * BN;
  t.kblocks = (K + BK - 1) / BK;
  t.nchunks = 1;
  return t;
}

// Shared-memory carve-up of one CTA.
template <int BN, int STAGES, int MODE, bool H16>
struct Smem {
  static constexpr int NA = Shape<BN, MODE, H16>::NA;
  static constexpr int NB = Shape<BN, MODE, H16>::NB;
  static constexpr int kA = BM * BK * 2;
  static constexpr int kB = BN * BK * 2;
  static constexpr int kStage = NA * kA + NB * kB;
  static constexpr int kBarriers = (2 * STAGES + 5) * 8;
  static constexpr int kTables = 3 * (kMaxGroups + 1) * 4 + ((kMaxGroups + 1) * 2 + 15) / 16 * 16;
  static constexpr size_t kBase = 1024 + (size_t)STAGES * kStage + kBarriers + 16 + kTables;
  // Token-major DOWN epilogue: per epilogue warp, one tile of 32 rows x kCW
  // fp32 columns, rows padded by 16 bytes so that both the row-per-thread
  // writes and the row-per-lane-group reads are free of bank conflicts. The
  // widest chunk that fits beside the ring.
  static constexpr size_t kLimit = 232448;
  static constexpr size_t stg_bytes(int cw) { return (size_t)4 * 32 * (cw * 4 + 16); }
  static constexpr bool kStg = MODE == kDownTM;
  static constexpr int kCW = (!kStg || kBase + stg_bytes(32) <= kLimit) ? 32 : 16;  // (unused without kStg)
  static constexpr int kStgRow = kCW * 4 + 16;
  static constexpr size_t kStaging = kStg ? stg_bytes(kCW) : 0;
  static constexpr size_t kTotal = kBase + kStaging;
};

template <int BN, int STAGES, int MODE, bool H16>
__global__ void __launch_bounds__(kThreads, 1)
    umma_ffn_kernel(const __grid_constant__ CUtensorMap mapA_r, const __grid_constant__ CUtensorMap mapB_r,
                    const __grid_constant__ CUtensorMap mapB2_r, const __grid_constant__ CUtensorMap mapA_s,
                    const __grid_constant__ CUtensorMap mapB_s, const __grid_constant__ CUtensorMap mapB2_s,
                    const UmmaParams p) {
  pdl_launch_dependents();
  using L = Smem<BN, STAGES, MODE, H16>;
  using SH = Shape<BN, MODE, H16>;
  constexpr uint32_t kTmemCols = SH::kTmemCols;
  constexpr bool kDownF16 = H16 && (MODE == kDown || MODE == kDownTM);  // fp16 operands
  constexpr uint32_t kIdesc = idesc_bf16<BN>();
  constexpr uint32_t kIdescDown = kDownF16 ? idesc_fp16<BN>() : idesc_bf16<(2 * BN <= 256 ? 2 * BN : 256)>();
  constexpr uint32_t kIdescTM = kDownF16 ? idesc_fp16<256>() : idesc_bf16<256>();
  static_assert(MODE != kDown || !SH::kTwoPlanes || 2 * BN <= 256, "DOWN issues N = 2 BN <= 256");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  uint8_t* staging = smem + (size_t)STAGES * L::kStage;  // L::kStaging bytes (token-major DOWN only)
  uint64_t* full = reinterpret_cast<uint64_t*>(staging + L::kStaging);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* pre = reinterpret_cast<int*>(tmem_slot + 4);
  int* s_m = pre + (kMaxGroups + 1);
  int* s_r0 = s_m + (kMaxGroups + 1);
  int16_t* s_e = reinterpret_cast<int16_t*>(s_r0 + (kMaxGroups + 1));  // expert ids < 1024 (-1: shared MLP)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  pdl_wait();  // everything below may read what earlier launches wrote

  // ---- group table: active experts (+ shared MLP), tiles per group ----
  const int n_act = MODE == kLogits ? 0 : min(max(*(volatile int*)&p.hdr->num_active, 0), p.E);
  const int n_groups = MODE == kLogits ? 1 : n_act + (p.has_shared ? 1 : 0);
  const int64_t R = p.T * p.k;
  constexpr bool kGU = MODE == kGateUp || MODE == kGateUpTM;
  const int nb_routed = kGU ? (p.I + BM - 1) / BM : (p.H + SH::ROWS - 1) / SH::ROWS;
  const int nb_shared = kGU ? (p.Is + BM - 1) / BM : (p.H + SH::ROWS - 1) / SH::ROWS;
  for (int g = threadIdx.x; g < n_groups; g += blockDim.x) {
    int e = -1, m = 0, tiles = 0;
    int64_t r0 = 0;
    if (g < n_act) {
      e = p.active[g];
      if (e >= 0 && e < p.E) {
        const int64_t lo = p.offsets[e], hi = p.offsets[e + 1];
        if (lo >= 0 && hi <= R && hi >= lo) {
          r0 = lo;
          m = (int)(hi - lo);
          tiles = nb_routed * ((m + BN - 1) / BN);
        } else if (blockIdx.x == 0) {
          record_error(p.hdr, MOE_ERR_DEVICE_CHECK, e);
        }
      } else if (blockIdx.x == 0) {
        record_error(p.hdr, MOE_ERR_DEVICE_CHECK, g);
      }
      if (e < 0 || e >= p.E) e = 0;  // zero tiles; keep the id in range
    } else if (MODE == kLogits) {
      m = (int)p.T;
      tiles = ((p.E + BM - 1) / BM) * ((m + BN - 1) / BN) * p.ksplit;
    } else {
      m = (int)p.T;
      tiles = nb_shared * ((m + BN - 1) / BN);
    }
    s_e[g] = (int16_t)e;
    s_m[g] = m;
    s_r0[g] = (int)r0;
    pre[g + 1] = tiles;
  }
  __syncthreads();
  if (warp == 0) {  // inclusive scan of pre[1..n_groups] by one warp, in chunks
    const int per = (n_groups + 31) / 32;
    const int beg = 1 + lane * per;
    const int end = min(beg + per, n_groups + 1);
    int sum = 0;
    for (int i = beg; i < end; ++i) sum += pre[i];
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int run = incl - sum;
    for (int i = beg; i < end; ++i) {
      run += pre[i];
      pre[i] = run;
    }
    if (lane == 0) pre[0] = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int total_tiles = n_groups > 0 ? pre[n_groups] : 0;
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ======================= TMA producer =======================
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
        const TileInfo t = decode_tile<BN, MODE, H16>(tile, n_groups, pre, s_e, s_m, s_r0, p);
        const CUtensorMap* mA = t.shared ? &mapA_s : &mapA_r;
        const CUtensorMap* mB = t.shared ? &mapB_s : &mapB_r;
        const CUtensorMap* mB2 = t.shared ? &mapB2_s : &mapB2_r;
        for (int kb = 0; kb < t.kblocks; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!wait_bar(&empty[s], ph ^ 1u, abort_flag, p.hdr, 1, p.wait_ns)) {
            ok = false;
            break;
          }
          uint8_t* st = stages + (size_t)s * L::kStage;
          const int gkb = t.kb0 + kb;
          int kx = gkb * BK, a0y = t.a0_row, a1y = t.a1_row;
          if (MODE == kLogits) {  // k-block gkb lies in weight plane gkb / kbH
            const int piece = gkb / p.kbH;
            kx = (gkb - piece * p.kbH) * BK;
            a0y += piece * p.E;
            a1y += piece * p.E;
          }
          mbar_expect_tx(&full[s], L::kStage);
          uint8_t* sb = st + L::NA * L::kA;
          if (SH::TM) {  // A: token tile(s); B: the two weight boxes, back to back
            tma_load_2d(mB, &full[s], st, kx, t.b_row);
            if (L::NA == 2) tma_load_2d(mB2, &full[s], st + L::kA, kx, t.b_row);
            tma_load_2d(mA, &full[s], sb, kx, a0y);
            tma_load_2d(mA, &full[s], sb + L::kB, kx, a1y);
          } else {
            tma_load_2d(mA, &full[s], st, kx, a0y);
            if (L::NA == 2) tma_load_2d(mA, &full[s], st + L::kA, kx, a1y);
            tma_load_2d(mB, &full[s], sb, kx, t.b_row);
            if (L::NB == 2) tma_load_2d(mB2, &full[s], sb + L::kB, kx, t.b_row);
          }
        }
      }
      // drain: the copies of the last STAGES iterations must have landed
      for (int j = max(0, it - STAGES); j < it; ++j) drain_bar(&full[j % STAGES], (uint32_t)(j / STAGES) & 1u, p.wait_ns);
    }
  } else if (warp == 1) {
    // ======================= MMA issuer =======================
    if (lane == 0) {
      int it = 0, tcount = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
        const TileInfo t = decode_tile<BN, MODE, H16>(tile, n_groups, pre, s_e, s_m, s_r0, p);
        for (int ch = 0; ok && ch < t.nchunks; ++ch, ++tcount) {
          const int a = tcount & 1;
          const uint32_t tph = (uint32_t)(tcount >> 1) & 1u;
          if (!wait_bar(&tempty[a], tph ^ 1u, abort_flag, p.hdr, 2, p.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d0 = tmem_base + (uint32_t)(a * SH::NACC * SH::NCOL);
          const uint32_t d1 = d0 + SH::NCOL;
          const int kb_begin = t.nchunks == 1 ? 0 : ch * kLogitsChunk;
          const int kb_end = t.nchunks == 1 ? t.kblocks : min(kb_begin + kLogitsChunk, t.kblocks);
          for (int kb = kb_begin; kb < kb_end; ++kb, ++it) {
            const int s = it % STAGES;
            const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
            if (!wait_bar(&full[s], ph, abort_flag, p.hdr, 3, p.wait_ns)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sa0 = smem_addr(stages + (size_t)s * L::kStage);
            const uint32_t sb = sa0 + L::NA * L::kA;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              const uint32_t acc = (kb > kb_begin || kk > 0) ? 1u : 0u;
              const uint64_t bdesc = sw128_desc(sb + kk * 32);
              if (SH::TM) {  // D (128 tokens x 256 weight rows) += A_token . B_weights
                umma_bf16(d0, sw128_desc(sa0 + kk * 32), bdesc, kIdescTM, acc);
                if (MODE == kDownTM && SH::kTwoPlanes)
                  umma_bf16(d0, sw128_desc(sa0 + L::kA + kk * 32), bdesc, kIdescTM, 1u);  // h_lo
              } else if (MODE == kDown) {  // B = [h_hi tile; h_lo tile] (2 BN rows, D spans 2 BN columns) or the fp16 h tile
                umma_bf16(d0, sw128_desc(sa0 + kk * 32), bdesc, kIdescDown, acc);
                if (SH::NA == 2) umma_bf16(d1, sw128_desc(sa0 + L::kA + kk * 32), bdesc, kIdescDown, acc);
              } else {
                umma_bf16(d0, sw128_desc(sa0 + kk * 32), bdesc, kIdesc, acc);
                if (SH::NA == 2) umma_bf16(d1, sw128_desc(sa0 + L::kA + kk * 32), bdesc, kIdesc, acc);
              }
            }
            tc_commit(&empty[s]);  // frees the stage once these MMAs have read it
          }
          if (!ok) break;
          if (!(p.withhold && tcount == 0)) tc_commit(&tfull[a]);  // accumulators ready for the epilogue
        }
      }
      tc_commit(done);
      drain_bar(done, 0, p.wait_ns);
    }
  } else {
    // ======================= epilogue (warps 2..5) =======================
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;
    constexpr int kColRegs = (BN + 31) / 32;                // token columns per lane (DOWN)
    constexpr int kSumCols = MODE == kLogits ? BN : 1;      // running chunk sums (LOGITS)
    int tcount = 0;
    bool alive = true;
    for (int tile = blockIdx.x; alive && tile < total_tiles; tile += gridDim.x) {
      const TileInfo t = decode_tile<BN, MODE, H16>(tile, n_groups, pre, s_e, s_m, s_r0, p);
      const int mvalid = min(BN, t.m - t.mb * BN);
      // DOWN: every token column's destination slot and routing weight, fetched
      // once per tile (column lane + 32 r in register r) before the accumulator
      // is ready, so the stores below need no memory round trip
      long long col_slot[kColRegs];
      float col_w[kColRegs];
      if (MODE == kDown) {
#pragma unroll
        for (int r = 0; r < kColRegs; ++r) {
          const int c = lane + 32 * r;
          col_slot[r] = -1;
          col_w[r] = 1.0f;
          if (c < mvalid) {
            const int64_t tok_row = (int64_t)t.mb * BN + c;
            if (t.shared) {
              col_slot[r] = tok_row;
            } else {
              const long long sl = p.tok_of[t.r0 + tok_row];
              if (sl < 0 || sl >= R) record_error(p.hdr, MOE_ERR_DEVICE_CHECK, (int)(t.r0 + tok_row));
              else col_slot[r] = sl;
            }
          }
        }
        if (!t.shared && p.topk_w != nullptr) {
#pragma unroll
          for (int r = 0; r < kColRegs; ++r)
            if (col_slot[r] >= 0) col_w[r] = p.topk_w[col_slot[r]];
        }
      }
      // token-major: this thread owns token row `row` of the tile; DOWN needs
      // its destination slot and routing weight, fetched before the wait
      const bool tm_valid = SH::TM && row < mvalid;
      const int64_t tm_tok = (int64_t)t.mb * BN + row;
      long long tm_slot = -1;
      float tm_w = 1.0f;
      if (MODE == kDownTM && tm_valid) {
        if (t.shared) {
          tm_slot = tm_tok;
        } else {
          const long long sl = p.tok_of[t.r0 + tm_tok];
          if (sl < 0 || sl >= R) {
            record_error(p.hdr, MOE_ERR_DEVICE_CHECK, (int)(t.r0 + tm_tok));
          } else {
            tm_slot = sl;
            if (p.topk_w != nullptr) tm_w = p.topk_w[sl];
          }
        }
      }
      float sum0[kSumCols];
      for (int ch = 0; ch < t.nchunks; ++ch, ++tcount) {
        const int a = tcount & 1;
        const uint32_t tph = (uint32_t)(tcount >> 1) & 1u;
        // one lane waits, the warp follows its verdict: the TMEM loads below are
        // .sync.aligned and need the whole warp converged
        int ok = 1;
        if (lane == 0) ok = wait_bar(&tfull[a], tph, abort_flag, p.hdr, 4, p.wait_ns) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        __syncwarp();
        if (!ok) {
          alive = false;
          break;
        }
        tc_fence_after();
        const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(a * SH::NACC * SH::NCOL);
        if (MODE == kGateUpTM) {
          // columns [0,128): gate rows nb*128 + c, [128,256): the matching up rows
          const int width = t.shared ? p.Is : p.I;
          uint16_t* hrow = t.shared ? p.h_shared + tm_tok * p.Is : p.h_perm + (t.r0 + tm_tok) * p.I;
          const int64_t plane = t.shared ? p.T * p.Is : p.T * p.k * p.I;
#pragma unroll 1
          for (int c0 = 0; c0 < BM; c0 += 16) {
            float g[16], u[16];
            tmem_ld16(taddr + c0, g);
            tmem_ld16(taddr + BM + c0, u);
            const int j0 = t.nb * BM + c0;
            if (H16 && tm_valid && j0 < width) {
              uint32_t h2[8];
              bool fin = true;
#pragma unroll
              for (int i = 0; i < 16; i += 2) {
                const uint16_t a0 = f32_to_f16(silu_f32(g[i]) * u[i]), a1 = f32_to_f16(silu_f32(g[i + 1]) * u[i + 1]);
                fin = fin && f16_finite(a0) && f16_finite(a1);
                h2[i / 2] = (uint32_t)a0 | ((uint32_t)a1 << 16);
              }
              if (!fin) record_error(p.hdr, MOE_ERR_RANGE, (int)(t.r0 + tm_tok));
              if (j0 + 16 <= width) {
                uint4* dh = reinterpret_cast<uint4*>(hrow + j0);
                dh[0] = make_uint4(h2[0], h2[1], h2[2], h2[3]);
                dh[1] = make_uint4(h2[4], h2[5], h2[6], h2[7]);
              } else {
#pragma unroll
                for (int i = 0; i < 16; ++i)
                  if (j0 + i < width) hrow[j0 + i] = (uint16_t)(h2[i / 2] >> (16 * (i & 1)));
              }
            } else if (tm_valid && j0 < width) {
              uint32_t hi2[8], lo2[8];
#pragma unroll
              for (int i = 0; i < 16; i += 2) {
                const float h0 = silu_f32(g[i]) * u[i], h1 = silu_f32(g[i + 1]) * u[i + 1];
                const uint16_t a0 = f32_to_bf16(h0), a1 = f32_to_bf16(h1);
                hi2[i / 2] = (uint32_t)a0 | ((uint32_t)a1 << 16);
                lo2[i / 2] = (uint32_t)f32_to_bf16(h0 - __uint_as_float((uint32_t)a0 << 16)) |
                             ((uint32_t)f32_to_bf16(h1 - __uint_as_float((uint32_t)a1 << 16)) << 16);
              }
              if (j0 + 16 <= width) {
                uint4* dh = reinterpret_cast<uint4*>(hrow + j0);
                uint4* dl = reinterpret_cast<uint4*>(hrow + plane + j0);
                dh[0] = make_uint4(hi2[0], hi2[1], hi2[2], hi2[3]);
                dh[1] = make_uint4(hi2[4], hi2[5], hi2[6], hi2[7]);
                dl[0] = make_uint4(lo2[0], lo2[1], lo2[2], lo2[3]);
                dl[1] = make_uint4(lo2[4], lo2[5], lo2[6], lo2[7]);
              } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                  if (j0 + i < width) {
                    hrow[j0 + i] = (uint16_t)(hi2[i / 2] >> (16 * (i & 1)));
                    hrow[plane + j0 + i] = (uint16_t)(lo2[i / 2] >> (16 * (i & 1)));
                  }
                }
              }
            }
          }
        } else if (MODE == kDownTM) {
          // columns: 256 weight rows n0 .. n0+255 (with two h planes, h_hi and h_lo
          // are already summed by the MMA). Thread `lane` holds output row
          // `lane` of the warp's 32; each chunk of kCW columns is turned around
          // in shared memory so that every store instruction writes whole
          // row segments: lane l stores 16 bytes of row (l / G) of a group of
          // 32 / G rows, G = kCW / 4 lanes per row (row-per-thread 16-byte
          // stores touched 32 lines per instruction and left the pass
          // store-bound at twice its MMA time).
          constexpr int kCW = L::kCW, G = kCW / 4, RPI = 32 / G;  // lanes per row, rows per instruction
          static_assert(!H16 || L::kStgRow >= 144, "fp16 slot rows stage 64 columns (128 bytes) per row");
          const int n0 = t.nb * 2 * BM;
          if (H16 && p.slots16 && !t.shared) {
            // fp16 slot rows: 64 columns (128 bytes) per row and chunk, 8 lanes per row
            const long long dst16 = (tm_valid && tm_slot >= 0) ? tm_slot * (long long)p.H : -1ll;
            uint16_t* o16 = reinterpret_cast<uint16_t*>(p.y_slots);
            uint8_t* stg16 = staging + (size_t)q * 32 * L::kStgRow;
            const int sub8 = lane >> 3, part8 = lane & 7;
            bool fin = true;
#pragma unroll 1
            for (int c0 = 0; c0 < 2 * BM; c0 += 64) {
              float v[64];
#pragma unroll
              for (int j = 0; j < 64; j += 16) tmem_ld16(taddr + c0 + j, v + j);
              const int n = n0 + c0;
              if (n >= p.H) continue;  // warp-uniform
              uint32_t h2[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const uint16_t lo = f32_to_f16(tm_w * v[2 * i]), hi = f32_to_f16(tm_w * v[2 * i + 1]);
                fin = fin && f16_finite(lo) && f16_finite(hi);
                h2[i] = (uint32_t)lo | ((uint32_t)hi << 16);
              }
              if (n + 64 <= p.H) {
                __syncwarp();  // the previous chunk's reads of the tile are done
                uint4* d = reinterpret_cast<uint4*>(stg16 + lane * L::kStgRow);
#pragma unroll
                for (int i = 0; i < 8; ++i) d[i] = make_uint4(h2[4 * i], h2[4 * i + 1], h2[4 * i + 2], h2[4 * i + 3]);
                __syncwarp();
#pragma unroll
                for (int r0 = 0; r0 < 32; r0 += 4) {
                  const int r = r0 + sub8;
                  const long long dst = __shfl_sync(0xffffffffu, dst16, r);
                  const uint4 val = *reinterpret_cast<const uint4*>(stg16 + r * L::kStgRow + part8 * 16);
                  if (dst >= 0) *reinterpret_cast<uint4*>(o16 + dst + n + part8 * 8) = val;
                }
              } else if (dst16 >= 0) {  // ragged last chunk of the hidden size: per element
#pragma unroll
                for (int i = 0; i < 64; ++i)
                  if (n + i < p.H) o16[dst16 + n + i] = (uint16_t)(h2[i / 2] >> (16 * (i & 1)));
              }
            }
            if (!fin && dst16 >= 0) record_error(p.hdr, MOE_ERR_RANGE, (int)(t.r0 + tm_tok));
          } else {
          // the destination row offset of this lane's row, or -1 when the row is absent
          const long long my_dst = !(tm_valid && tm_slot >= 0)
                                       ? -1ll
                                       : (t.shared ? (long long)tm_tok : tm_slot) * (long long)p.H;
          float* obase = t.shared ? p.shared_out : p.y_slots;
          uint8_t* stg = staging + (size_t)q * 32 * L::kStgRow;
          const int sub = lane / G, part = lane % G;  // this lane's row within a group, its 16-byte column part
#pragma unroll 1
          for (int c0 = 0; c0 < 2 * BM; c0 += kCW) {
            float v[kCW];
#pragma unroll
            for (int j = 0; j < kCW; j += 16) tmem_ld16(taddr + c0 + j, v + j);
            const int n = n0 + c0;
            if (n >= p.H) continue;  // warp-uniform
            if (n + kCW <= p.H) {
              __syncwarp();  // the previous chunk's reads of the tile are done
              float4* d = reinterpret_cast<float4*>(stg + lane * L::kStgRow);
#pragma unroll
              for (int i = 0; i < G; ++i)
                d[i] = make_float4(tm_w * v[4 * i], tm_w * v[4 * i + 1], tm_w * v[4 * i + 2], tm_w * v[4 * i + 3]);
              __syncwarp();
#pragma unroll
              for (int r0 = 0; r0 < 32; r0 += RPI) {
                const int r = r0 + sub;
                const long long dst = __shfl_sync(0xffffffffu, my_dst, r);
                const float4 val = *reinterpret_cast<const float4*>(stg + r * L::kStgRow + part * 16);
                if (dst >= 0) *reinterpret_cast<float4*>(obase + dst + n + part * 4) = val;
              }
            } else if (my_dst >= 0) {  // ragged last chunk of the hidden size: per element
#pragma unroll
              for (int i = 0; i < kCW; ++i)
                if (n + i < p.H) obase[my_dst + n + i] = tm_w * v[i];
            }
          }
          }
        }
#pragma unroll
        for (int c0 = 0; c0 < BN; c0 += 16) {
          if (SH::TM || c0 >= mvalid) break;  // warp-uniform
          float v0[16], v1[16];
          if (MODE == kLogits) {
            // chunk sums stay in registers; one fp32 add per chunk per element
            tmem_ld16(taddr + c0, v0);
#pragma unroll
            for (int i = 0; i < 16; ++i)
              sum0[(c0 + i) % kSumCols] = ch == 0 ? v0[i] : sum0[(c0 + i) % kSumCols] + v0[i];
          } else if (MODE == kGateUp) {
            tmem_ld16(taddr + c0, v0);
            tmem_ld16(taddr + SH::NCOL + c0, v1);
            const int j = t.nb * BM + row;
            const int width = t.shared ? p.Is : p.I;
            if (j < width) {
              uint16_t* hi = t.shared ? p.h_shared : p.h_perm + t.r0 * p.I;
              const int64_t plane = t.shared ? p.T * p.Is : p.T * p.k * p.I;
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const int c = c0 + i;
                if (c < mvalid) {
                  const float h = silu_f32(v0[i]) * v1[i];
                  const int64_t at = ((int64_t)t.mb * BN + c) * width + j;
                  if (H16) {
                    const uint16_t hh = f32_to_f16(h);
                    if (!f16_finite(hh)) record_error(p.hdr, MOE_ERR_RANGE, (int)(t.r0 + t.mb * BN + c));
                    hi[at] = hh;
                  } else {
                    const uint16_t h_hi = f32_to_bf16(h);
                    const uint16_t h_lo = f32_to_bf16(h - __uint_as_float((uint32_t)h_hi << 16));
                    hi[at] = h_hi;
                    hi[plane + at] = h_lo;
                  }
                }
              }
            }
          } else {
            const int n = t.nb * SH::ROWS + row;
            float* base = t.shared ? p.shared_out : p.y_slots;
#pragma unroll
            for (int acc_i = 0; acc_i < SH::NA; ++acc_i) {  // accumulator acc_i: weight rows n + acc_i * 128
              const uint32_t ta = taddr + (uint32_t)(acc_i * SH::NCOL);
              tmem_ld16(ta + c0, v0);  // W . h_hi (or W . h, one fp16 plane)
              if (SH::kTwoPlanes) tmem_ld16(ta + BN + c0, v1);  // W . h_lo
              const int nn = n + acc_i * BM;
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const int c = c0 + i;  // compile-time after unrolling
                const long long slot = __shfl_sync(0xffffffffu, col_slot[c / 32], c % 32);
                const float w = __shfl_sync(0xffffffffu, col_w[c / 32], c % 32);
                const float d = SH::kTwoPlanes ? v0[i] + v1[i] : v0[i];
                if (slot >= 0 && nn < p.H) {
                  if (H16 && p.slots16 && !t.shared) {
                    const uint16_t hv = f32_to_f16(w * d);
                    if (!f16_finite(hv)) record_error(p.hdr, MOE_ERR_RANGE, (int)slot);
                    reinterpret_cast<uint16_t*>(p.y_slots)[slot * p.H + nn] = hv;
                  } else {
                    base[slot * p.H + nn] = w * d;
                  }
                }
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[a]);
      }
      if (MODE == kLogits && alive) {  // the tile's logits, written once
        const int e0 = t.nb * BM + row;
        float* out = p.logits_out + (int64_t)t.ks * p.T * p.E;
#pragma unroll
        for (int c = 0; c < kSumCols; ++c) {
          if (c < mvalid && e0 < p.E) out[((int64_t)t.mb * BN + c) * p.E + e0] = sum0[c];
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ----------------------------------------------------------------------------
// host side
// ----------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

// 2-D 16-bit tensor [rows, cols] (cols contiguous; bf16, or fp16 when f16),
// box {64 cols, box_rows}, 128B swizzle.
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows, bool f16 = false) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)(rows > 0 ? rows : 1)};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
            dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, int STAGES, int MODE, bool H16>
cudaError_t launch_pass(const CUtensorMap* maps, const UmmaParams& p, int kernel_id, cudaStream_t s) {
  const size_t smem = Smem<BN, STAGES, MODE, H16>::kTotal;
  static_assert(Smem<BN, STAGES, MODE, H16>::kTotal <= 232448, "shared memory over the 227 KB limit");
  cudaError_t e = cudaFuncSetAttribute(umma_ffn_kernel<BN, STAGES, MODE, H16>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  before_launch(kernel_id, s);
  launch_pdl(umma_ffn_kernel<BN, STAGES, MODE, H16>, dim3(sm_count()), dim3(kThreads), smem, s, maps[0], maps[1],
             maps[2], maps[3], maps[4], maps[5], p);
  after_launch(kernel_id, s);
  return cudaGetLastError();
}

// Stage counts: gate/up stages hold two weight tiles and one token tile; down
// stages the weight tile(s) and the token tiles of both h planes, or of the
// one fp16 plane (H16: the down weights' fp16 copy, a.w_down_f16).
template <int BN, int ST_GU, int ST_DN, bool TM, bool H16>
cudaError_t run_bn(const FfnArgs& a, const uint16_t* x_perm, cudaStream_t s) {
  static_assert(!TM || BN == BM, "token-major tiles hold 128 token rows");
  const int64_t R = a.T * a.k;
  const bool shared = a.ws_gate_up != nullptr;
  UmmaParams p{};
  p.T = a.T;
  p.H = a.H;
  p.I = a.I;
  p.Is = a.Is;
  p.k = a.k;
  p.E = a.E;
  p.has_shared = shared ? 1 : 0;
  p.offsets = a.offsets;
  p.tok_of = a.tok_of;
  p.active = a.active;
  p.hdr = a.hdr;
  p.topk_w = a.topk_w;
  p.h_perm = static_cast<uint16_t*>(a.h_perm);
  p.h_shared = static_cast<uint16_t*>(a.h_shared);
  p.y_slots = a.y_slots;
  p.shared_out = a.shared_out;
  p.wait_ns = opt_wait_ns();
  p.withhold = opt_withhold() == 2 ? 1 : 0;
  p.slots16 = (H16 && a.slots_f16) ? 1 : 0;
  // maps: A routed, B routed, B2 routed, A shared, B shared, B2 shared
  CUtensorMap m[6];

  // pass 1: gate/up with SwiGLU
  bool ok = make_map(&m[0], a.w_gate_up, (int64_t)a.E * 2 * a.I, a.H, BM) && make_map(&m[1], x_perm, R, a.H, BN);
  m[2] = m[1];
  if (shared) ok = ok && make_map(&m[3], a.ws_gate_up, 2 * (int64_t)a.Is, a.H, BM) && make_map(&m[4], a.x, a.T, a.H, BN);
  else {
    m[3] = m[0];
    m[4] = m[1];
  }
  m[5] = m[4];
  if (!ok) return cudaErrorInvalidValue;
  cudaError_t e = launch_pass<BN, ST_GU, TM ? kGateUpTM : kGateUp, H16>(m, p, MOE_KERNEL_EXPERT_GATE_UP, s);
  if (e != cudaSuccess) return e;

  // pass 2: down projection of h (h_hi + h_lo, or the fp16 plane), weighted
  // scatter into slot order
  if (H16) {
    ok = make_map(&m[0], a.w_down_f16, (int64_t)a.E * a.H, a.I, BM, true) &&
         make_map(&m[1], p.h_perm, R, a.I, BN, true);
    m[2] = m[1];
    if (shared) {
      ok = ok && make_map(&m[3], a.ws_down_f16, a.H, a.Is, BM, true) &&
           make_map(&m[4], p.h_shared, a.T, a.Is, BN, true);
      m[5] = m[4];
    }
  } else {
    ok = make_map(&m[0], a.w_down, (int64_t)a.E * a.H, a.I, BM) && make_map(&m[1], p.h_perm, R, a.I, BN) &&
         make_map(&m[2], p.h_perm + R * a.I, R, a.I, BN);
    if (shared)
      ok = ok && make_map(&m[3], a.ws_down, a.H, a.Is, BM) && make_map(&m[4], p.h_shared, a.T, a.Is, BN) &&
           make_map(&m[5], p.h_shared + a.T * a.Is, a.T, a.Is, BN);
  }
  if (!shared) {
    m[3] = m[0];
    m[4] = m[1];
    m[5] = m[2];
  }
  if (!ok) return cudaErrorInvalidValue;
  return launch_pass<BN, ST_DN, TM ? kDownTM : kDown, H16>(m, p, MOE_KERNEL_EXPERT_DOWN, s);
}

// Splits the fp32 router weight into three bf16 planes whose sum is the weight
// (to within one fp32 ulp): hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid).
// x is bf16, so every product x * plane is exact in fp32 and the tensor cores
// accumulate sum_h x[t,h] * w[e,h] over K = 3H in fp32.
__global__ void __launch_bounds__(256) split_router_weight_kernel(const float* __restrict__ w, int64_t n,
                                                                  uint16_t* __restrict__ planes) {
  pdl_launch_dependents();
  pdl_wait();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const float v = __ldg(w + i);
    const uint16_t hi = f32_to_bf16(v);
    const float r1 = v - __uint_as_float((uint32_t)hi << 16);
    const uint16_t mid = f32_to_bf16(r1);
    const float r2 = r1 - __uint_as_float((uint32_t)mid << 16);
    planes[i] = hi;
    planes[n + i] = mid;
    planes[2 * n + i] = f32_to_bf16(r2);
  }
}

// logits[t, e] = sum_s part[s, t, e], s ascending.
__global__ void __launch_bounds__(256) reduce_splits_kernel(const float* __restrict__ part, int ksplit, int64_t n,
                                                            float* __restrict__ out) {
  pdl_launch_dependents();
  pdl_wait();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    float acc = part[i];
    for (int s = 1; s < ksplit; ++s) acc += part[(int64_t)s * n + i];
    out[i] = acc;
  }
}

}  // namespace

// Split-K factor of the router-logits GEMM: enough tiles to cover the SMs when
// the token count alone does not; every split gets at least one k-block.
void logits_split(int64_t T, int E, int H, int* ksplit, int* kper) {
  const int kbH = (H + BK - 1) / BK;
  const int total = 3 * kbH;
  const int64_t tiles = (int64_t)((E + BM - 1) / BM) * ((T + kLogitsBN - 1) / kLogitsBN);
  int want = (int)((128 + tiles - 1) / tiles);
  want = want < 1 ? 1 : (want > 24 ? 24 : want);
  if (want > total) want = total;
  const int per = (total + want - 1) / want;
  *kper = per;
  *ksplit = (total + per - 1) / per;
}

cudaError_t launch_router_logits_tc(const moe_config& c, const uint16_t* x, int64_t T, const float* w,
                                    float* logits, uint16_t* planes, float* partials, cudaStream_t s) {
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  const int E = c.num_experts, H = c.hidden_size;
  const int64_t n = (int64_t)E * H;
  int ksplit, kper;
  logits_split(T, E, H, &ksplit, &kper);
  int64_t blocks = (n + 255) / 256;
  if (blocks > (int64_t)sm_count() * 8) blocks = (int64_t)sm_count() * 8;
  before_launch(MOE_KERNEL_ROUTER_LOGITS, s);
  launch_pdl(split_router_weight_kernel, dim3((unsigned)blocks), dim3(256), 0, s, w, n, planes);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  UmmaParams p{};
  p.T = T;
  p.H = H;
  p.E = E;
  p.k = 1;
  p.logits_out = ksplit > 1 ? partials : logits;
  p.ksplit = ksplit;
  p.kper = kper;
  p.kbH = (H + BK - 1) / BK;
  p.wait_ns = opt_wait_ns();
  CUtensorMap m[6];
  if (!make_map(&m[0], planes, 3 * (int64_t)E, H, BM) || !make_map(&m[1], x, T, H, kLogitsBN))
    return cudaErrorInvalidValue;
  m[2] = m[1];
  m[3] = m[0];
  m[4] = m[1];
  m[5] = m[1];
  constexpr int kStages = 8;
  const size_t smem = Smem<kLogitsBN, kStages, kLogits, false>::kTotal;
  e = cudaFuncSetAttribute(umma_ffn_kernel<kLogitsBN, kStages, kLogits, false>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  launch_pdl(umma_ffn_kernel<kLogitsBN, kStages, kLogits, false>, dim3(sm_count()), dim3(kThreads), smem, s, m[0], m[1], m[2], m[3], m[4], m[5], p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  int nk = 2;
  if (ksplit > 1) {
    const int64_t nl = T * E;
    int64_t rb = (nl + 255) / 256;
    if (rb > (int64_t)sm_count() * 8) rb = (int64_t)sm_count() * 8;
    launch_pdl(reduce_splits_kernel, dim3((unsigned)rb), dim3(256), 0, s, partials, ksplit, nl, logits);
    nk = 3;
  }
  after_launch(MOE_KERNEL_ROUTER_LOGITS, s, nk);
  return cudaGetLastError();
}

// Tile shape from the mean rows per expert (R / min(R, E)): weight-major
// tiles of BN = 32 / 64 / 128 token columns for skinny experts, token-major
// 128 x 256 tiles (returned as 256) once experts average 96 rows or more.
int umma_pick_bn(int64_t T, int k, int E) {
  const int64_t R = T * k;
  const int64_t groups = R < E ? R : E;
  const int64_t avg = groups > 0 ? (R + groups - 1) / groups : 1;
  if (avg <= 24) return 32;
  if (avg <= 64) return 64;
  if (avg < 96) return 128;
  return 256;
}

cudaError_t launch_umma_ffn(const FfnArgs& a, const uint16_t* x_perm, int bn, cudaStream_t s) {
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  if (a.w_down_f16 != nullptr) {  // one fp16 h plane: smaller down stages, one more of them where it fits
    switch (bn) {
      case 32: return run_bn<32, 5, 5, false, true>(a, x_perm, s);
      case 64: return run_bn<64, 5, 5, false, true>(a, x_perm, s);
      case 128: return run_bn<128, 4, 4, false, true>(a, x_perm, s);
      default: return run_bn<128, 4, 4, true, true>(a, x_perm, s);  // token-major
    }
  }
  switch (bn) {
    case 32: return run_bn<32, 5, 5, false, false>(a, x_perm, s);
    case 64: return run_bn<64, 5, 4, false, false>(a, x_perm, s);
    case 128: return run_bn<128, 4, 4, false, false>(a, x_perm, s);
    default: return run_bn<128, 4, 3, true, false>(a, x_perm, s);  // token-major
  }
}

}  // namespace moe
