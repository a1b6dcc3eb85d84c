// Arguments of the expert FFN kernels (routed experts + shared MLP).
#pragma once

#include "common.cuh"

namespace moe {

// 8-bit affine weight matrix: for each row and each group of `group`
// consecutive inputs, w = scale * q + bias (q uint8, scale and bias bf16).
struct Q8Mat {
  const uint8_t* q;       // [rows, K]
  const uint16_t* scale;  // [rows, K / group]
  const uint16_t* bias;   // [rows, K / group]
};

struct FfnArgs {
  const uint16_t* x;          // [T, H]
  int64_t T;
  int H, I, Is, k, E;
  const int32_t* offsets;     // [E+1]
  const int32_t* tok_of;      // [T*k]
  const int32_t* active;      // [num_active]
  WsHeader* hdr;              // num_active, error word
  const float* topk_w;        // [T*k] or null
  const uint16_t* w_gate_up;  // [E, 2I, H]
  const uint16_t* w_down;     // [E, H, I]
  const uint16_t* ws_gate_up; // [2Is, H] or null
  const uint16_t* ws_down;    // [H, Is]
  // fp16 copies of the down weights, or null: the tensor-core path then keeps
  // h as one fp16 plane and multiplies fp16 operands in the down pass
  const uint16_t* w_down_f16;   // [E, H, I]
  const uint16_t* ws_down_f16;  // [H, Is]; set whenever ws_gate_up is
  // with the fp16 down weights: write the routed slot rows as fp16 (y_slots
  // then holds [T*k, H] uint16_t; shared_out stays fp32)
  bool slots_f16;
  void* h_perm;               // [T*k, I]: fp32 (streaming path), two bf16 planes or one fp16 plane (tensor cores)
  void* h_shared;             // [T, Is]: same element type as h_perm
  float* y_slots;             // [T*k, H]
  float* shared_out;          // [T, H]
  // 8-bit affine weights (streaming path only): group > 0 selects them for the
  // routed experts; the shared MLP is 8-bit when qs_gate_up.q is set, else bf16.
  int group;
  Q8Mat q_gate_up, q_down;    // [E*2I, H], [E*H, I]
  Q8Mat qs_gate_up, qs_down;  // [2Is, H], [H, Is]
};

cudaError_t launch_gemv_ffn(const FfnArgs& a, cudaStream_t s);
// y[t] = bf16( sum_j y16[t*k + j] + shared_out[t] ) for fp16 slot rows
cudaError_t launch_combine16(const uint16_t* y16, const float* shared_out, int64_t T, int k, int H, uint16_t* y,
                             cudaStream_t s);
int umma_pick_bn(int64_t T, int k, int E);
cudaError_t launch_umma_ffn(const FfnArgs& a, const uint16_t* x_perm, int bn, cudaStream_t s);

}  // namespace moe
