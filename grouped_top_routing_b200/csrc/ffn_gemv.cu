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

constexpr int kUnrollQ = 4;  // 16-byte chunks in flight per lane per 8-bit weight row

__device__ __forceinline__ float bf16_word(uint16_t v) { return __uint_as_float((uint32_t)v << 16); }

// Sum of the 16 products of one 16-byte chunk of 8-bit affine weights
// (w = s * q + b, one fp32 rounding) with 16 fp32 values.
__device__ __forceinline__ float dot16_q8(uint4 q, float s, float b, const float* v, float acc) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float qi = (float)((w[i >> 2] >> (8 * (i & 3))) & 0xffu);
    acc = fmaf(fmaf(s, qi, b), v[i], acc);
  }
  return acc;
}

// Gate and up dot products of one bf16 row pair (H each) against up to MT
// token rows (xr[t]; null: no token).
template <int MT>
__device__ __forceinline__ void rowpair_bf16(const uint16_t* gate, const uint16_t* up, int H,
                                             const uint16_t* const (&xr)[MT], float (&ag)[MT], float (&au)[MT]) {
  const int lane = threadIdx.x & 31, nv = H / 8;
  for (int v0 = lane; v0 < nv; v0 += 32 * kUnroll) {
    uint4 gv[kUnroll], uv[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int v = v0 + 32 * u;
      if (v < nv) {
        gv[u] = ld_stream_u4(gate + v * 8);
        uv[u] = ld_stream_u4(up + v * 8);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
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
  for (int v0 = lane; v0 < nv; v0 += 32 * kUnrollQ) {
    uint4 gv[kUnrollQ], uv[kUnrollQ];
#pragma unroll
    for (int u = 0; u < kUnrollQ; ++u) {
      const int v = v0 + 32 * u;
      if (v < nv) {
        gv[u] = ld_stream_u4(gq + v * 16);
        uv[u] = ld_stream_u4(uq + v * 16);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnrollQ; ++u) {
      const int v = v0 + 32 * u;
      if (v < nv) {
        const int g = v * 16 / group;  // a 16-element chunk lies in one group
        const float sg = bf16_word(__ldg(m.scale + rg * ng + g)), bg = bf16_word(__ldg(m.bias + rg * ng + g));
        const float su = bf16_word(__ldg(m.scale + ru * ng + g)), bu = bf16_word(__ldg(m.bias + ru * ng + g));
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          if (xr[t] != nullptr) {
            float xf[16];
            unpack8_bf16(ld_nc_u4(xr[t] + v * 16), xf);
            unpack8_bf16(ld_nc_u4(xr[t] + v * 16 + 8), xf + 8);
            ag[t] = dot16_q8(gv[u], sg, bg, xf, ag[t]);
            au[t] = dot16_q8(uv[u], su, bu, xf, au[t]);
          }
        }
      }
    }
  }
}

// Gate/up pass: one warp per intermediate index j of one expert, streaming its
// gate row and up row (bf16, or 8-bit affine when Q8) against up to MT tokens
// per pass.
template <int MT, bool Q8>
__global__ void __launch_bounds__(256) gemv_gate_up_kernel(FfnArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int n_act = min(max(*(volatile int*)&a.hdr->num_active, 0), a.E);
  const int64_t routed_items = (int64_t)n_act * a.I;
  const bool has_shared = a.ws_gate_up != nullptr || (Q8 && a.qs_gate_up.q != nullptr);
  const int64_t total = routed_items + (has_shared ? a.Is : 0);
  const int H = a.H;

  for (int64_t item = gw; item < total; item += nw) {
    const bool shared = item >= routed_items;
    int j, e = 0;
    int64_t r0 = 0, m = 0;
    if (!shared) {
      const int aidx = (int)(item / a.I);
      j = (int)(item - (int64_t)aidx * a.I);
      if (!expert_rows(a, aidx, e, r0, m)) continue;
    } else {
      j = (int)(item - routed_items);
      m = a.T;
    }
    for (int64_t c0 = 0; c0 < m; c0 += MT) {
      const int mc = (int)min((int64_t)MT, m - c0);
      const uint16_t* xr[MT];
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        xr[t] = nullptr;
        if (t < mc) {
          int64_t tok = c0 + t, slot;
          if (!shared) tok = slot_token(a, r0 + c0 + t, slot);
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
      else rowpair_bf16<MT>(wbase + rg * H, wbase + ru * H, H, xr, ag, au);
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        if (t < mc) {
          const float g = warp_sum(ag[t]);
          const float u = warp_sum(au[t]);
          if (lane == t && xr[t] != nullptr) {
            const float h = silu_f32(g) * u;  // kept in fp32 on this path
            if (!shared) static_cast<float*>(a.h_perm)[(r0 + c0 + t) * a.I + j] = h;
            else static_cast<float*>(a.h_shared)[(c0 + t) * a.Is + j] = h;
          }
        }
      }
    }
  }
}

// ROWS bf16 rows (K each, row r at w0 + r*K) against up to MT fp32 h rows
// (hin + (hrow0 + t) * K).
template <int MT, int ROWS>
__device__ __forceinline__ void rows_bf16(const uint16_t* w0, int nrows, int K, const float* hin, int64_t hrow0,
                                          int mc, float (&acc)[ROWS][MT]) {
  const int lane = threadIdx.x & 31, nvk = K / 8;
#pragma unroll 2
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
  for (int v = lane; v < nv; v += 32) {
    const int g = v * 16 / group;
    uint4 wv[ROWS];
    float sc[ROWS], bi[ROWS];
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
      if (r < nrows) {
        wv[r] = ld_stream_u4(m.q + (row0 + r) * K + v * 16);
        sc[r] = bf16_word(__ldg(m.scale + (row0 + r) * ng + g));
        bi[r] = bf16_word(__ldg(m.bias + (row0 + r) * ng + g));
      }
    }
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      if (t < mc) {
        const float4* hp = reinterpret_cast<const float4*>(hin + (hrow0 + t) * K + v * 16);
        float hf[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 h4 = __ldg(hp + i);
          hf[4 * i] = h4.x, hf[4 * i + 1] = h4.y, hf[4 * i + 2] = h4.z, hf[4 * i + 3] = h4.w;
        }
#pragma unroll
        for (int r = 0; r < ROWS; ++r)
          if (r < nrows) acc[r][t] = dot16_q8(wv[r], sc[r], bi[r], hf, acc[r][t]);
      }
    }
  }
}

// Down pass: one warp per block of ROWS output rows of one expert; the rows
// (I each, bf16 or 8-bit affine when Q8) are streamed together against up to
// MT tokens' h per pass.
template <int MT, int ROWS, bool Q8>
__global__ void __launch_bounds__(256) gemv_down_kernel(FfnArgs a) {
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
  const int64_t total = routed_items + (has_shared ? nrb : 0);

  for (int64_t item = gw; item < total; item += nw) {
    const bool shared = item >= routed_items;
    int n0, K, e = 0;
    const float* hin;
    int64_t r0 = 0, m = 0;
    if (!shared) {
      const int aidx = (int)(item / nrb);
      n0 = (int)(item - (int64_t)aidx * nrb) * ROWS;
      if (!expert_rows(a, aidx, e, r0, m)) continue;
      K = a.I;
      hin = static_cast<const float*>(a.h_perm);
    } else {
      n0 = (int)(item - routed_items) * ROWS;
      K = a.Is;
      hin = static_cast<const float*>(a.h_shared);
      m = a.T;
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
      const int64_t row0 = shared ? n0 : (int64_t)e * H + n0, hrow0 = shared ? c0 : r0 + c0;
      if (Q8) qm = shared ? (a.qs_down.q != nullptr ? &a.qs_down : nullptr) : &a.q_down;
      if (Q8 && qm != nullptr) rows_q8<MT, ROWS>(*qm, row0, nrows, K, a.group, hin, hrow0, mc, acc);
      else rows_bf16<MT, ROWS>((shared ? a.ws_down : a.w_down) + row0 * K, nrows, K, hin, hrow0, mc, acc);
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
          if (slot_token(a, r0 + c0 + t, slot) >= 0) {
            const float w = a.topk_w != nullptr ? a.topk_w[slot] : 1.0f;
            a.y_slots[slot * H + n0 + r] = w * mine;
          }
        } else {
          a.shared_out[(c0 + t) * H + n0 + r] = mine;
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
  if (a.T <= 1) return launch_gemv_mt<1, 8, Q8>(a, s);
  if (a.T <= 2) return launch_gemv_mt<2, 8, Q8>(a, s);
  if (a.T <= 4) return launch_gemv_mt<4, 4, Q8>(a, s);
  return launch_gemv_mt<8, 4, Q8>(a, s);
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
