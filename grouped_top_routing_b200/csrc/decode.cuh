// Arguments and host entry points of the fused decode kernel (decode_stream.cu):
// the whole block for up to kDecodeMaxT tokens in one persistent launch.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kDecodeMaxT = 8;        // tokens per launch (the mma's n = 8 columns)
constexpr int kDecodeMaxSlots = 65;   // the shared MLP + up to 64 distinct routed experts
constexpr int kDecodeMaxE = 512;      // experts the in-kernel router handles (16 per lane)

// Routing of one launch as the kernel publishes it: slot 0 is the shared MLP,
// slots 1..U the distinct routed experts in ascending id; wt[slot][t] is token
// t's routing weight for that slot (0 when t did not select it; 1 for slot 0).
struct DecodeRoute {
  int32_t U;
  int32_t pad[3];
  int32_t expert[kDecodeMaxSlots];
  float wt[kDecodeMaxSlots][kDecodeMaxT];
};

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
  uint16_t* y;                   // [T, H] out
  int32_t* topk_idx_out;         // [T, k] or null
  float* topk_w_out;             // [T, k] or null
  // workspace
  float* logits;                 // [T, E]
  uint16_t* hbuf;                // [kDecodeMaxSlots][16][max(I, Is)] bf16: w*h split hi (rows 0-7) / lo (8-15)
  float* part;                   // [kDecodeMaxSlots][H][8] fp32: each slot's weighted output rows
  DecodeRoute* route;            // published routing
  int32_t* sync;                 // counters, zero at launch (kWsSyncBytes after the header)
  WsHeader* hdr;
  uint64_t wait_ns;              // bound on every device-side wait
  int withhold;                  // test aid: never release the routing
};

// Whether one launch handles this batch and shape.
bool decode_supported(int64_t T, int k, int E, int H, int I, int Is);
// Workspace bytes of the kernel's own buffers (hbuf, part, route) for this shape.
size_t decode_hbuf_bytes(int I, int Is);
size_t decode_part_bytes(int H);
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s);

}  // namespace moe
