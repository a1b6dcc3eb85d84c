// Arguments and host entry points of the fused decode kernel (decode_fused.cu).
#pragma once

#include "common.cuh"

namespace moe {

struct DecodeArgs {
  const uint16_t* x;  // [T, H]
  int T, H, E, k, I, Is, n_group, topk_group, score_fn, norm;
  float scale;
  const float* router_w;         // [E, H] or null when logits are given
  const float* expert_bias;      // [E] or null
  const float* logits_override;  // [T, E] or null
  const uint16_t* w_gate_up;     // [E, 2I, H]
  const uint16_t* w_down;        // [E, H, I]
  const uint16_t* ws_gate_up;    // [2Is, H] or null
  const uint16_t* ws_down;       // [H, Is]
  float* logits;                 // [T, E] workspace
  int32_t* topk_idx_out;         // [T, k] or null
  float* topk_w_out;             // [T, k] or null
  float* h;                      // [T*k, I] workspace
  float* h_shared;               // [T, Is] workspace
  float* y_slots;                // [T*k, H] workspace
  float* shared_out;             // [T, H] workspace
  int32_t* sync;                 // decode_fused_sync_ints(H) counters, workspace
  // Sigmoid scores and selection keys computed with each router logit (null:
  // the routing computes them from the logits): [T, E] fp32 unbiased scores and
  // [T, E] 64-bit keys, workspace.
  float* pre_orig;
  unsigned long long* pre_key;
  uint16_t* y;                   // [T, H] output
  WsHeader* hdr;
  uint64_t wait_ns;  // bound on every device-side wait
  int withhold;      // test aid: CTA 0 never arrives at the grid barrier after the router rows
};

// Completion counters the kernels need in the workspace (zeroed by the kernels):
// kMaxSlots per-expert counters, 2H per-row counters, one shared-MLP counter.
size_t decode_fused_sync_ints(int H);
// Whether the fused kernel handles this batch and shape (1-2 tokens, at most 32
// slots, hidden size up to 8192, expert widths up to twice the hidden size).
bool decode_fused_supported(int64_t T, int k, int E, int H, int I, int Is);
cudaError_t launch_decode_fused(const DecodeArgs& a, cudaStream_t s);

}  // namespace moe
