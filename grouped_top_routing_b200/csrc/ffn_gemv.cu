// Decode expert FFN: weight-streaming GEMV over the selected experts only.
//
// The page "Ling-3.0-flash-GGUF" (section "Measured performance") bounds
// decode by memory bandwidth, since a decode step touches just the weights of
// the experts the router chose.
// The expert is the SwiGLU MLP of mlxcel issue #838 ("Architecture notes";
// "Shared experts are one wide MLP, not N separate experts"):
//   h = silu(gate x) * (up x),  y = down h.
//
// Work items are single weight rows (gate/up pass) or blocks of ROWS rows
// (down pass) of the experts in the compacted active list written by the
// permutation, plus the shared MLP's rows. Weights are bf16, or 8-bit affine
// (w = scale * q + bias per group of inputs, scale and bias bf16: the 8-bit
// recipes of the pages "Ling-3.0-tiny-8bit-XL-mlx", section "XL Quantization
// Recipe", and "Ling-2.6-flash-JANGTQ", quantization summary), dequantised in
// the stream. One warp per item: lanes stride the
// row in 16-byte chunks (ld.global.nc, no L1 allocation), every token routed
// to that expert is multiplied against the chunk, and the warp reduces with
// shuffles. Tokens are taken MT at a time (MT follows the batch, up to 8); an
// expert with more rows streams its weights again per group of MT (those
// re-reads hit L2), which is why larger batches take the tensor-core path.
#include <cuda_fp16.h>

#include "common.cuh"
#include "ffn.cuh"

namespace moe {

namespace {

constexpr int kUnroll = 8;  // 16-byte chunks in flight per lane per weight row (gate/up pass)
// The same for the bf16 shared MLP inside the 8-bit kernels: a short stream
// there keeps the kernels' register need, hence their resident warps, set by
// the 8-bit rows.
constexpr int kUnrollBf16InQ8 = 2;

// Resolves the rows [r0, r0 + m) of one active expert, clamped to [0, T*k).
__device__ __forceinline__ bool expert_rows(const FfnArgs& a, int aidx, int& e, int64_t& r0, int64_t& m) {
  e = a.active[aidx];
  if (e < 0 || e >= a.E) {
    record_error(a.hdr, MOE_ERR_DEVICE_CHECK, aidx);
    return false;
  }
  const int64_t R = a.T * a.k;
  int64_t lo = a.offsets[e], hi = a.offsets[e + 1];
  if (lo < 0 || hi > R || hi < lo) {
    record_error(a.hdr, MOE_ERR_DEVICE_CHECK, e);
    return false;
  }
  r0 = lo;
  m = hi - lo;
  return true;
}

__device__ __forceinline__ int64_t slot_token(const FfnArgs& a, int64_t row, int64_t& slot) {
  slot = a.tok_of[row];
  if (slot < 0 || slot >= a.T * a.k) {
    record_error(a.hdr, MOE_ERR_DEVICE_CHECK, (int)row);
    return -1;
  }
  return slot / a.k;
}

// Per-block copy of what every item looks up: each active expert's id and
// rows [r0, r0 + m) (by index in the compacted list), and, when the batch has
// at most kStagedSlots permuted rows, each row's slot id. Read once per block
// after the permutation has finished, so an item's weight and activation
// loads no longer wait behind a chain of dependent lookups (active list ->
// offsets -> slot -> token row).
constexpr int kStagedExperts = 1024;  // the largest num_experts the boundary accepts
constexpr int kStagedSlots = 2048;

struct StagedRows {
  int32_t e[kStagedExperts];
  int32_t r0[kStagedExperts];
  int32_t m[kStagedExperts];   // 0: the expert is skipped (bad id or offsets, recorded)
  int32_t slot[kStagedSlots];  // tok_of[r] as read (checked where used)
};

// Fills `st` for the n_act active experts (n_act <= E <= kStagedExperts) and
// returns whether the slot ids were staged too. Every thread of the block
// calls it: it ends with a block barrier.
__device__ __forceinline__ bool stage_rows(const FfnArgs& a, int n_act, StagedRows& st) {
  for (int i = threadIdx.x; i < n_act; i += blockDim.x) {
    int e;
    int64_t r0, m;
    if (!expert_rows(a, i, e, r0, m)) e = 0, r0 = 0, m = 0;
    st.e[i] = e;
    st.r0[i] = (int32_t)r0;
    st.m[i] = (int32_t)m;
  }
  const int64_t R = a.T * a.k;
  const bool slots = R <= kStagedSlots;
  if (slots)
    for (int r = threadIdx.x; r < R; r += blockDim.x) st.slot[r] = a.tok_of[r];
  __syncthreads();
  return slots;
}

// slot_token on the staged slot ids when `staged` (row < T*k <= kStagedSlots)
__device__ __forceinline__ int64_t staged_slot_token(const FfnArgs& a, const StagedRows& st, bool staged,
                                                     int64_t row, int64_t& slot) {
  if (!staged) return slot_token(a, row, slot);
  slot = st.slot[row];
  if (slot < 0 || slot >= a.T * a.k) {
    record_error(a.hdr, MOE_ERR_DEVICE_CHECK, (int)row);
    return -1;
  }
  return slot / a.k;
}

constexpr int kUnrollQ = 4;  // 16-byte chunks in flight per lane per 8-bit weight row

__device__ __forceinline__ float bf16_word(uint16_t v) { return __uint_as_float((uint32_t)v << 16); }

// 8-bit affine weights, w = s * q + b over a group of inputs, enter a dot
// product with activations v as s * sum(q v) + b * sum(v), so the per-weight
// work is the code's product alone. Codes become floats without a conversion
// instruction: q (0..255) placed in bits 16..23 of a zero word reads as the
// fp32 value q * 2^-133. Below 128 that word is subnormal (q * 2^16 units of
// 2^-149); from 128 up q's top bit is the exponent's low bit and the word
// reads 2^-126 * (1 + (q - 128) / 128), again q * 2^-133. Against activations
// scaled by 2^33 the products are q * v * 2^-100, exact inside one fma, and a
// chunk's sum is scaled back by 2^100 (exact). The scaling keeps v * 2^33
// finite for |v| < 2^95; a product under 2^-126 (|q v| < 2^-26) is rounded
// in the subnormal range, an absolute error of at most 2^-50 once scaled back.
constexpr float kQ8VScale = 0x1p33f;
constexpr float kQ8Unscale = 0x1p100f;

// byte i of w as q * 2^-133 (see above): the byte moved to bits 16..23, the
// other bytes zero
template <int I>
__device__ __forceinline__ float code_f(uint32_t w) {
  return __uint_as_float(__byte_perm(w, 0u, 0x4044u | (I << 8)));
}

// a * b + c with subnormal operands kept (the code floats are subnormal below
// 128), whatever flush-to-zero setting the file is compiled with
__device__ __forceinline__ float fma_sub(float a, float b, float c) {
  float d;
  asm("fma.rn.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// sum_i q_i * vs_i over the 16 codes of one chunk, in units of 2^-100 when
// vs = v * 2^33
__device__ __forceinline__ float qdot16(uint4 q, const float (&vs)[16]) {
  float d = 0.0f;
  d = fma_sub(code_f<0>(q.x), vs[0], d);
  d = fma_sub(code_f<1>(q.x), vs[1], d);
  d = fma_sub(code_f<2>(q.x), vs[2], d);
  d = fma_sub(code_f<3>(q.x), vs[3], d);
  d = fma_sub(code_f<0>(q.y), vs[4], d);
  d = fma_sub(code_f<1>(q.y), vs[5], d);
  d = fma_sub(code_f<2>(q.y), vs[6], d);
  d = fma_sub(code_f<3>(q.y), vs[7], d);
  d = fma_sub(code_f<0>(q.z), vs[8], d);
  d = fma_sub(code_f<1>(q.z), vs[9], d);
  d = fma_sub(code_f<2>(q.z), vs[10], d);
  d = fma_sub(code_f<3>(q.z), vs[11], d);
  d = fma_sub(code_f<0>(q.w), vs[12], d);
  d = fma_sub(code_f<1>(q.w), vs[13], d);
  d = fma_sub(code_f<2>(q.w), vs[14], d);
  d = fma_sub(code_f<3>(q.w), vs[15], d);
  return d;
}

// One chunk's share of a row's dot product: s * sum(q v) + b * sum(v), with
// d = sum(q v) in units of 2^-100 and sv = sum(v).
__device__ __forceinline__ float q8_chunk(float acc, uint16_t s, uint16_t b, float d, float sv) {
  return fmaf(bf16_word(s), d * kQ8Unscale, fmaf(bf16_word(b), sv, acc));
}

// The 16 activations of one chunk, vs = v * 2^33, and their plain sum.
__device__ __forceinline__ float prep16(const float (&v)[16], float (&vs)[16]) {
  float sv = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    sv += v[i];
    vs[i] = v[i] * kQ8VScale;
  }
  return sv;
}

// Gate and up dot products of one bf16 row pair (H each) against up to MT
// token rows (xr[t]; null: no token), U 16-byte chunks in flight per lane
// per row.
template <int MT, int U>
__device__ __forceinline__ void rowpair_bf16(const uint16_t* gate, const uint16_t* up, int H,
                                             const uint16_t* const (&xr)[MT], float (&ag)[MT], float (&au)[MT]) {
  const int lane = threadIdx.x & 31, nv = H / 8;
  for (int v0 = lane; v0 < nv; v0 += 32 * U) {
    uint4 gv[U], uv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + 32 * u;
      if (v < nv) {
        gv[u] = ld_stream_u4(gate + v * 8);
        uv[u] = ld_stream_u4(up + v * 8);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + 32 * u;
      if (v < nv) {
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          if (xr[t] != nullptr) {
            float xf[8];
            unpack8_bf16(ld_nc_u4(xr[t] + v * 8), xf);
            ag[t] = dot8_bf16(gv[u], xf, ag[t]);
            au[t] = dot8_bf16(uv[u], xf, au[t]);
          }
        }
      }
    }
  }
}

// The same for rows rg (gate) and ru (up) of an 8-bit affine matrix.
template <int MT>
__device__ __forceinline__ void rowpair_q8(const Q8Mat& m, int64_t rg, int64_t ru, int H, int group,
                                           const uint16_t* const (&xr)[MT], float (&ag)[MT], float (&au)[MT]) {
  const int lane = threadIdx.x & 31, nv = H / 16, ng = H / group;
  const uint8_t* gq = m.q + rg * H;
  const uint8_t* uq = m.q + ru * H;
  const uint16_t* gs = m.scale + rg * ng;
  const uint16_t* gb = m.bias + rg * ng;
  const uint16_t* us = m.scale + ru * ng;
  const uint16_t* ub = m.bias + ru * ng;
#pragma unroll 1
  for (int v0 = lane; v0 < nv; v0 += 32 * kUnrollQ) {
    uint4 gv[kUnrollQ], uv[kUnrollQ];
    uint16_t sg[kUnrollQ], bg[kUnrollQ], su[kUnrollQ], bu[kUnrollQ];
#pragma unroll
    for (int u = 0; u < kUnrollQ; ++u) {
      const int v = v0 + 32 * u;
      if (v < nv) {
        const int g = v * 16 / group;  // a 16-element chunk lies in one group
        gv[u] = ld_stream_u4(gq + v * 16);
        uv[u] = ld_stream_u4(uq + v * 16);
        sg[u] = __ldg(gs + g);
        bg[u] = __ldg(gb + g);
        su[u] = __ldg(us + g);
        bu[u] = __ldg(ub + g);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnrollQ; ++u) {
      const int v = v0 + 32 * u;
      if (v < nv) {
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          if (xr[t] != nullptr) {
            float xf[16], vs[16];
            unpack8_bf16(ld_nc_u4(xr[t] + v * 16), xf);
            unpack8_bf16(ld_nc_u4(xr[t] + v * 16 + 8), xf + 8);
            const float sv = prep16(xf, vs);
            ag[t] = q8_chunk(ag[t], sg[u], bg[u], qdot16(gv[u], vs), sv);
            au[t] = q8_chunk(au[t], su[u], bu[u], qdot16(uv[u], vs), sv);
          }
        }
      }
    }
  }
}

// Asks L2 for [p, p + bytes) ahead of its use: a hint, with nothing to wait
// for. Skipped unless the address and size are multiples of 16 bytes (the
// bulk-copy unit's rule).
__device__ __forceinline__ void prefetch_l2(const void* p, int64_t bytes) {
  if (p == nullptr || bytes <= 0 || bytes > (int64_t(1) << 30) || ((reinterpret_cast<uintptr_t>(p) | bytes) & 15))
    return;
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"((uint32_t)bytes) : "memory");
}

// Lanes 0..2 of the warp ask L2 for `rows` consecutive rows of K inputs from
// row r0 of an 8-bit matrix: codes, scales, biases.
__device__ __forceinline__ void prefetch_q8_rows(const Q8Mat& m, int64_t r0, int rows, int K, int group) {
  const int lane = threadIdx.x & 31, ng = K / group;
  if (lane == 0) prefetch_l2(m.q + r0 * K, (int64_t)rows * K);
  if (lane == 1) prefetch_l2(m.scale + r0 * ng, (int64_t)rows * ng * 2);
  if (lane == 2) prefetch_l2(m.bias + r0 * ng, (int64_t)rows * ng * 2);
}

// 8-bit streaming: a warp asks L2 for the weight rows of the item that lies
// kAheadGateUp (kAheadDown) grid strides ahead while the current one streams,
// so later items' loads find their lines cached or already requested, with no
// registers held for them.
constexpr int kAheadGateUp = 2;  // items of the gate/up pass (2 rows of H each)
constexpr int kAheadDown = 4;    // items of the down pass (ROWS rows of I each)

__device__ __forceinline__ void prefetch_gate_up_item(const FfnArgs& a, const StagedRows& st, int64_t item,
                                                      int64_t routed_items, int64_t total, int nsp) {
  if (item >= total) return;
  if (item < routed_items) {
    const int aidx = (int)(item / a.I), j = (int)(item - (int64_t)aidx * a.I);
    if (st.m[aidx] == 0) return;
    const int e = st.e[aidx];
    const int64_t rg = (int64_t)e * 2 * a.I + j;
    prefetch_q8_rows(a.q_gate_up, rg, 1, a.H, a.group);
    prefetch_q8_rows(a.q_gate_up, rg + a.I, 1, a.H, a.group);
  } else {
    const int64_t j = (item - routed_items) / nsp;
    if (a.qs_gate_up.q != nullptr) {
      prefetch_q8_rows(a.qs_gate_up, j, 1, a.H, a.group);
      prefetch_q8_rows(a.qs_gate_up, a.Is + j, 1, a.H, a.group);
    } else if ((threadIdx.x & 31) == 3) {
      prefetch_l2(a.ws_gate_up + j * a.H, (int64_t)a.H * 2);
      prefetch_l2(a.ws_gate_up + (a.Is + j) * a.H, (int64_t)a.H * 2);
    }
  }
}

template <int ROWS>
__device__ __forceinline__ void prefetch_down_item(const FfnArgs& a, const StagedRows& st, int64_t item,
                                                   int64_t routed_items, int64_t total, int nrb, int nsp) {
  if (item >= total) return;
  if (item < routed_items) {
    const int aidx = (int)(item / nrb);
    const int n0 = (int)(item - (int64_t)aidx * nrb) * ROWS;
    if (st.m[aidx] == 0) return;
    const int e = st.e[aidx];
    prefetch_q8_rows(a.q_down, (int64_t)e * a.H + n0, min(ROWS, a.H - n0), a.I, a.group);
  } else {
    const int n0 = (int)((item - routed_items) / nsp) * ROWS, rows = min(ROWS, a.H - n0);
    if (a.qs_down.q != nullptr) prefetch_q8_rows(a.qs_down, n0, rows, a.Is, a.group);
    else if ((threadIdx.x & 31) == 3) prefetch_l2(a.ws_down + (int64_t)n0 * a.Is, (int64_t)rows * a.Is * 2);
  }
}

// Gate/up pass: one warp per intermediate index j of one expert, streaming its
// gate row and up row (bf16, or 8-bit affine when Q8) against up to MT tokens
// per pass. The shared MLP, which sees every token, has one item per (j,
// block of MT tokens), so its passes spread over warps like the experts'.
// Launch bounds: the 8-bit kernels ask for two resident 256-thread blocks per
// SM (at most 128 registers a thread); a minimum of 0 leaves the bf16
// kernels' register use to the compiler, as with no minimum at all.
template <int MT, bool Q8>
__global__ void __launch_bounds__(256, Q8 ? 2 : 0) gemv_gate_up_kernel(FfnArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int n_act = min(max(*(volatile int*)&a.hdr->num_active, 0), a.E);
  const int64_t routed_items = (int64_t)n_act * a.I;
  const bool has_shared = a.ws_gate_up != nullptr || (Q8 && a.qs_gate_up.q != nullptr);
  const int nsp = (int)((a.T + MT - 1) / MT);  // token blocks of the shared MLP
  const int64_t total = routed_items + (has_shared ? (int64_t)a.Is * nsp : 0);
  const int H = a.H;
  __shared__ StagedRows st;
  const bool staged = stage_rows(a, n_act, st);
  if (Q8)
    for (int d = 0; d < kAheadGateUp; ++d)
      prefetch_gate_up_item(a, st, gw + (int64_t)d * nw, routed_items, total, nsp);

  for (int64_t item = gw; item < total; item += nw) {
    if (Q8) prefetch_gate_up_item(a, st, item + (int64_t)kAheadGateUp * nw, routed_items, total, nsp);
    const bool shared = item >= routed_items;
    int j, e = 0;
    int64_t r0 = 0, m = 0, tb = 0;  // tb: first token of a shared item
    if (!shared) {
      const int aidx = (int)(item / a.I);
      j = (int)(item - (int64_t)aidx * a.I);
      e = st.e[aidx];
      r0 = st.r0[aidx];
      m = st.m[aidx];
    } else {
      const int64_t sidx = item - routed_items;
      j = (int)(sidx / nsp);
      tb = (sidx - (int64_t)j * nsp) * MT;
      m = min((int64_t)MT, a.T - tb);
    }
    for (int64_t c0 = 0; c0 < m; c0 += MT) {
      const int mc = (int)min((int64_t)MT, m - c0);
      const uint16_t* xr[MT];
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        xr[t] = nullptr;
        if (t < mc) {
          int64_t tok = tb + c0 + t, slot;
          if (!shared) tok = staged_slot_token(a, st, staged, r0 + c0 + t, slot);
          if (tok >= 0) xr[t] = a.x + tok * H;
        }
      }
      float ag[MT], au[MT];
#pragma unroll
      for (int t = 0; t < MT; ++t) ag[t] = au[t] = 0.0f;
      // the row pair: 8-bit (routed rows when Q8; shared rows when 8-bit too) or bf16
      const Q8Mat* qm = nullptr;
      int64_t rg, ru;
      const uint16_t* wbase;
      if (!shared) {
        rg = (int64_t)e * 2 * a.I + j;
        ru = rg + a.I;
        wbase = a.w_gate_up;
        if (Q8) qm = &a.q_gate_up;
      } else {
        rg = j;
        ru = (int64_t)a.Is + j;
        wbase = a.ws_gate_up;
        if (Q8 && a.qs_gate_up.q != nullptr) qm = &a.qs_gate_up;
      }
      if (Q8 && qm != nullptr) rowpair_q8<MT>(*qm, rg, ru, H, a.group, xr, ag, au);
      else rowpair_bf16<MT, Q8 ? kUnrollBf16InQ8 : kUnroll>(wbase + rg * H, wbase + ru * H, H, xr, ag, au);
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        if (t < mc) {
          const float g = warp_sum(ag[t]);
          const float u = warp_sum(au[t]);
          if (lane == t && xr[t] != nullptr) {
            const float h = silu_f32(g) * u;  // kept in fp32 on this path
            if (!shared) static_cast<float*>(a.h_perm)[(r0 + c0 + t) * a.I + j] = h;
            else static_cast<float*>(a.h_shared)[(tb + c0 + t) * a.Is + j] = h;
          }
        }
      }
    }
  }
}

// ROWS bf16 rows (K each, row r at w0 + r*K) against up to MT fp32 h rows
// (hin + (hrow0 + t) * K); the chunk loop unrolled U times.
template <int MT, int ROWS, int U>
__device__ __forceinline__ void rows_bf16(const uint16_t* w0, int nrows, int K, const float* hin, int64_t hrow0,
                                          int mc, float (&acc)[ROWS][MT]) {
  const int lane = threadIdx.x & 31, nvk = K / 8;
#pragma unroll U
  for (int v = lane; v < nvk; v += 32) {
    uint4 wv[ROWS];
#pragma unroll
    for (int r = 0; r < ROWS; ++r)
      if (r < nrows) wv[r] = ld_stream_u4(w0 + (int64_t)r * K + v * 8);
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      if (t < mc) {
        const float4* hp = reinterpret_cast<const float4*>(hin + (hrow0 + t) * K + v * 8);
        const float4 h0 = __ldg(hp), h1 = __ldg(hp + 1);
        const float hf[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
#pragma unroll
        for (int r = 0; r < ROWS; ++r)
          if (r < nrows) acc[r][t] = dot8_bf16(wv[r], hf, acc[r][t]);
      }
    }
  }
}

// The same for rows row0 .. row0 + nrows of an 8-bit affine matrix.
template <int MT, int ROWS>
__device__ __forceinline__ void rows_q8(const Q8Mat& m, int64_t row0, int nrows, int K, int group, const float* hin,
                                        int64_t hrow0, int mc, float (&acc)[ROWS][MT]) {
  const int lane = threadIdx.x & 31, nv = K / 16, ng = K / group;
  const uint8_t* qb = m.q + row0 * K;
  const uint16_t* sb = m.scale + row0 * ng;
  const uint16_t* bb = m.bias + row0 * ng;
  const float* hb = hin + hrow0 * K;
#pragma unroll 1
  for (int v = lane; v < nv; v += 32) {
    const int g = v * 16 / group;
    uint4 wv[ROWS];
    uint16_t sc[ROWS], bi[ROWS];
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
      if (r < nrows) {
        wv[r] = ld_stream_u4(qb + (r * K + v * 16));
        sc[r] = __ldg(sb + (r * ng + g));
        bi[r] = __ldg(bb + (r * ng + g));
      }
    }
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      if (t < mc) {
        const float4* hp = reinterpret_cast<const float4*>(hb + (t * K + v * 16));
        float hf[16], hs[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 h4 = __ldg(hp + i);
          hf[4 * i] = h4.x, hf[4 * i + 1] = h4.y, hf[4 * i + 2] = h4.z, hf[4 * i + 3] = h4.w;
        }
        const float sv = prep16(hf, hs);
#pragma unroll
        for (int r = 0; r < ROWS; ++r)
          if (r < nrows) acc[r][t] = q8_chunk(acc[r][t], sc[r], bi[r], qdot16(wv[r], hs), sv);
      }
    }
  }
}

// Down pass: one warp per block of ROWS output rows of one expert; the rows
// (I each, bf16 or 8-bit affine when Q8) are streamed together against up to
// MT tokens' h per pass. The shared MLP has one item per (row block, block of
// MT tokens).
template <int MT, int ROWS, bool Q8>
__global__ void __launch_bounds__(256, Q8 ? 2 : 0) gemv_down_kernel(FfnArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  static_assert(ROWS * MT <= 32, "one lane per (row, token) output");
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int n_act = min(max(*(volatile int*)&a.hdr->num_active, 0), a.E);
  const int H = a.H;
  const int nrb = (H + ROWS - 1) / ROWS;
  const int64_t routed_items = (int64_t)n_act * nrb;
  const bool has_shared = a.ws_down != nullptr || (Q8 && a.qs_down.q != nullptr);
  const int nsp = (int)((a.T + MT - 1) / MT);  // token blocks of the shared MLP
  const int64_t total = routed_items + (has_shared ? (int64_t)nrb * nsp : 0);
  __shared__ StagedRows st;
  const bool staged = stage_rows(a, n_act, st);
  if (Q8)
    for (int d = 0; d < kAheadDown; ++d)
      prefetch_down_item<ROWS>(a, st, gw + (int64_t)d * nw, routed_items, total, nrb, nsp);

  for (int64_t item = gw; item < total; item += nw) {
    if (Q8) prefetch_down_item<ROWS>(a, st, item + (int64_t)kAheadDown * nw, routed_items, total, nrb, nsp);
    const bool shared = item >= routed_items;
    int n0, K, e = 0;
    const float* hin;
    int64_t r0 = 0, m = 0, tb = 0;  // tb: first token of a shared item
    if (!shared) {
      const int aidx = (int)(item / nrb);
      n0 = (int)(item - (int64_t)aidx * nrb) * ROWS;
      e = st.e[aidx];
      r0 = st.r0[aidx];
      m = st.m[aidx];
      K = a.I;
      hin = static_cast<const float*>(a.h_perm);
    } else {
      const int64_t sidx = item - routed_items;
      const int blk = (int)(sidx / nsp);
      n0 = blk * ROWS;
      tb = (sidx - (int64_t)blk * nsp) * MT;
      K = a.Is;
      hin = static_cast<const float*>(a.h_shared);
      m = min((int64_t)MT, a.T - tb);
    }
    const int nrows = min(ROWS, H - n0);
    for (int64_t c0 = 0; c0 < m; c0 += MT) {
      const int mc = (int)min((int64_t)MT, m - c0);
      float acc[ROWS][MT];
#pragma unroll
      for (int r = 0; r < ROWS; ++r)
#pragma unroll
        for (int t = 0; t < MT; ++t) acc[r][t] = 0.0f;
      const Q8Mat* qm = nullptr;
      const int64_t row0 = shared ? n0 : (int64_t)e * H + n0, hrow0 = shared ? tb + c0 : r0 + c0;
      if (Q8) qm = shared ? (a.qs_down.q != nullptr ? &a.qs_down : nullptr) : &a.q_down;
      if (Q8 && qm != nullptr) rows_q8<MT, ROWS>(*qm, row0, nrows, K, a.group, hin, hrow0, mc, acc);
      else rows_bf16<MT, ROWS, Q8 ? 1 : 2>((shared ? a.ws_down : a.w_down) + row0 * K, nrows, K, hin, hrow0, mc, acc);
      float mine = 0.0f;
#pragma unroll
      for (int r = 0; r < ROWS; ++r)
#pragma unroll
        for (int t = 0; t < MT; ++t)
          if (t < mc && r < nrows) {
            const float s = warp_sum(acc[r][t]);
            if (lane == r * MT + t) mine = s;
          }
      const int r = lane / MT, t = lane % MT;
      if (r < nrows && t < mc) {
        if (!shared) {
          int64_t slot;
          if (staged_slot_token(a, st, staged, r0 + c0 + t, slot) >= 0) {
            const float w = a.topk_w != nullptr ? a.topk_w[slot] : 1.0f;
            a.y_slots[slot * H + n0 + r] = w * mine;
          }
        } else {
          a.shared_out[(tb + c0 + t) * H + n0 + r] = mine;
        }
      }
    }
  }
}

// y[t] = bf16( sum_j y_slots[t*k + j] + shared_out[t] ), fp32 in slot order
// then the shared row, one rounding; one thread per 4 outputs.
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ y_slots,
                                                      const float* __restrict__ shared_out, int64_t T, int k, int H,
                                                      uint16_t* __restrict__ y) {
  pdl_launch_dependents();
  pdl_wait();
  const int nv = H / 4;
  const int64_t n = T * nv;
  const float4* ys = reinterpret_cast<const float4*>(y_slots);
  const float4* sh = reinterpret_cast<const float4*>(shared_out);
  uint2* out = reinterpret_cast<uint2*>(y);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / nv;
    const int v = (int)(i - t * nv);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      const float4 f = __ldg(ys + (t * k + j) * nv + v);
      acc.x += f.x;
      acc.y += f.y;
      acc.z += f.z;
      acc.w += f.w;
    }
    if (sh != nullptr) {
      const float4 f = __ldg(sh + i);
      acc.x += f.x;
      acc.y += f.y;
      acc.z += f.z;
      acc.w += f.w;
    }
    out[i] = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
  }
}

// The same with fp16 slot rows (the tensor-core path on fp16 down weights):
// y[t] = bf16( sum_j float(y16[t*k + j]) + shared_out[t] ); one thread per 8
// outputs (16-byte slot loads).
__global__ void __launch_bounds__(256) combine16_kernel(const uint16_t* __restrict__ y16,
                                                        const float* __restrict__ shared_out, int64_t T, int k, int H,
                                                        uint16_t* __restrict__ y) {
  pdl_launch_dependents();
  pdl_wait();
  const int nv = H / 8;
  const int64_t n = T * nv;
  const uint4* ys = reinterpret_cast<const uint4*>(y16);
  const float4* sh = reinterpret_cast<const float4*>(shared_out);
  uint4* out = reinterpret_cast<uint4*>(y);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / nv;
    const int v = (int)(i - t * nv);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < k; ++j) {
      const uint4 f = __ldg(ys + (t * k + j) * nv + v);
      const uint32_t w4[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        acc[2 * q] += __half2float(__ushort_as_half((unsigned short)(w4[q] & 0xFFFFu)));
        acc[2 * q + 1] += __half2float(__ushort_as_half((unsigned short)(w4[q] >> 16)));
      }
    }
    if (sh != nullptr) {
      const float4 a = __ldg(sh + 2 * i), b = __ldg(sh + 2 * i + 1);
      acc[0] += a.x;
      acc[1] += a.y;
      acc[2] += a.z;
      acc[3] += a.w;
      acc[4] += b.x;
      acc[5] += b.y;
      acc[6] += b.z;
      acc[7] += b.w;
    }
    out[i] = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                        pack_bf16x2(acc[6], acc[7]));
  }
}

}  // namespace

// One resident wave: as many 256-thread blocks as the kernel's register use
// lets every SM hold at once (a second wave would double the latency chain).
template <typename K>
int resident_blocks(K kernel) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, 256, 0) != cudaSuccess || per_sm < 1) per_sm = 1;
  return sm_count() * per_sm;
}

template <int MT, int ROWS, bool Q8>
cudaError_t launch_gemv_mt(const FfnArgs& a, cudaStream_t s) {
  before_launch(MOE_KERNEL_EXPERT_GATE_UP, s);
  launch_pdl(gemv_gate_up_kernel<MT, Q8>, dim3(resident_blocks(gemv_gate_up_kernel<MT, Q8>)), dim3(256), 0, s, a);
  after_launch(MOE_KERNEL_EXPERT_GATE_UP, s);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  before_launch(MOE_KERNEL_EXPERT_DOWN, s);
  launch_pdl(gemv_down_kernel<MT, ROWS, Q8>, dim3(resident_blocks(gemv_down_kernel<MT, ROWS, Q8>)), dim3(256), 0, s,
             a);
  after_launch(MOE_KERNEL_EXPERT_DOWN, s);
  return cudaGetLastError();
}

template <bool Q8>
cudaError_t launch_gemv_fmt(const FfnArgs& a, cudaStream_t s) {
  // 8-bit: 4 down rows per warp and at most 4 tokens per pass, within the
  // 128 registers a thread that two resident 256-thread blocks per SM allow
  if (a.T <= 1) return launch_gemv_mt<1, Q8 ? 4 : 8, Q8>(a, s);
  if (a.T <= 2) return launch_gemv_mt<2, Q8 ? 4 : 8, Q8>(a, s);
  if constexpr (Q8) {
    return launch_gemv_mt<4, 4, Q8>(a, s);
  } else {
    if (a.T <= 4) return launch_gemv_mt<4, 4, Q8>(a, s);
    return launch_gemv_mt<8, 4, Q8>(a, s);
  }
}

// Tokens per pass follow the batch (an expert has at most T rows), so the
// single-token decode step carries one accumulator per row.
cudaError_t launch_gemv_ffn(const FfnArgs& a, cudaStream_t s) {
  return a.group > 0 ? launch_gemv_fmt<true>(a, s) : launch_gemv_fmt<false>(a, s);
}

cudaError_t launch_combine(const float* y_slots, const float* shared_out, int64_t T, int k, int H, uint16_t* y,
                           cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int64_t n = T * (H / 4);
  int64_t blocks = (n + 255) / 256;
  const int64_t cap = (int64_t)sm_count() * 8;
  if (blocks > cap) blocks = cap;
  before_launch(MOE_KERNEL_COMBINE, s);
  launch_pdl(combine_kernel, dim3((unsigned)blocks), dim3(256), 0, s, y_slots, shared_out, T, k, H, y);
  after_launch(MOE_KERNEL_COMBINE, s);
  return cudaGetLastError();
}

cudaError_t launch_combine16(const uint16_t* y16, const float* shared_out, int64_t T, int k, int H, uint16_t* y,
                             cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int64_t n = T * (H / 8);
  int64_t blocks = (n + 255) / 256;
  const int64_t cap = (int64_t)sm_count() * 8;
  if (blocks > cap) blocks = cap;
  before_launch(MOE_KERNEL_COMBINE, s);
  launch_pdl(combine16_kernel, dim3((unsigned)blocks), dim3(256), 0, s, y16, shared_out, T, k, H, y);
  after_launch(MOE_KERNEL_COMBINE, s);
  return cudaGetLastError();
}

}  // namespace moe
