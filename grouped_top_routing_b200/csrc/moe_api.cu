// C ABI of libmoe.so: argument validation, workspace layout, launch sequence.
//
// Validation follows mlxcel issue #838, section "Defensive requirements":
// magnitude ceilings on every architecture scalar, zero checks before any
// divisibility check, 1 <= k <= E, E divisible by n_group, topk_group in
// [1, n_group], reject rather than terminate. Every rule here runs on the host
// before the first launch and returns a status with a message naming the field.
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "common.cuh"
#include "decode_fused.cuh"
#include "ffn.cuh"

namespace moe {

cudaError_t launch_router_logits_gemv(const moe_config& c, const uint16_t* x, int64_t T, const float* w, float* out,
                                      cudaStream_t s);
void logits_split(int64_t T, int E, int H, int* ksplit, int* kper);
cudaError_t launch_router_logits_tc(const moe_config& c, const uint16_t* x, int64_t T, const float* w,
                                    float* logits, uint16_t* planes, float* partials, cudaStream_t s);
cudaError_t launch_route(const moe_config& c, const float* logits, const float* bias, int64_t T, int32_t* idx,
                         float* w, cudaStream_t s);
size_t permute_scratch_ints(int E, int64_t T);
cudaError_t launch_permute(const moe_config& c, const int32_t* idx, int64_t T, const uint16_t* x, int32_t* offsets,
                           int32_t* row_of, int32_t* tok_of, uint16_t* x_perm, int32_t* active, int32_t* tile_cnt,
                           int32_t* tile_base, WsHeader* hdr, cudaStream_t s);
cudaError_t launch_active_from_offsets(const int32_t* offsets, int E, int32_t* active, WsHeader* hdr,
                                       cudaStream_t s);
cudaError_t launch_identity_route(int64_t T, int32_t* offsets, int32_t* tok_of, float* w, cudaStream_t s);
cudaError_t launch_combine(const float* y_slots, const float* shared_out, int64_t T, int k, int H, uint16_t* y,
                           cudaStream_t s);
cudaError_t launch_ep_send(const int32_t* offsets, int E, const int32_t* tok_of, const float* topk_w, int64_t R_max,
                           int64_t* counts, float* row_w, cudaStream_t s);
cudaError_t launch_ep_recv(const int64_t* recv_counts, int nseg, int n_local, int64_t R, int32_t* local_expert,
                           cudaStream_t s);
cudaError_t launch_ep_scatter_back(const float* y_perm, const int32_t* tok_of, int64_t R, int64_t n_slots, int H,
                                   float* y_slots, cudaStream_t s);
cudaError_t launch_convert_bf16_to_f16(const uint16_t* src, uint16_t* dst, int64_t n, int32_t* bad_count,
                                       cudaStream_t s);
cudaError_t launch_gather_rows(const int32_t* offsets, int E, const int32_t* tok_of, int k, int64_t T,
                               const uint16_t* x, int H, uint16_t* x_perm, cudaStream_t s);

// ---------------------------------------------------------------------------
// errors, hooks, device cache
// ---------------------------------------------------------------------------
namespace {

thread_local char g_err[512] = "";
thread_local uint64_t t_launches = 0;
// The options of the entry point running on this thread (set for the
// duration of one call by CallScope, null otherwise): kernel choices, the
// wait limit and the timing hook. Nothing outlives the call.
thread_local const moe_options* t_opts = nullptr;
int g_sm_count[64] = {};

moe_status fail(moe_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

moe_status cuda_fail(cudaError_t e, const char* where) {
  return fail(MOE_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

constexpr uint64_t kDefaultWaitNs = 2000000000ull;

// Installs a call's options on this thread for the duration of the call.
struct CallScope {
  explicit CallScope(const moe_options* o) { t_opts = o; }
  ~CallScope() { t_opts = nullptr; }
  CallScope(const CallScope&) = delete;
  CallScope& operator=(const CallScope&) = delete;
};

moe_status validate_options(const moe_options* o) {
  if (o == nullptr) return MOE_OK;
  if (o->ffn_path < 0 || o->ffn_path > 2)
    return fail(MOE_ERR_INVALID_ARG, "opts->ffn_path = %d is not 0 (auto), 1 (streaming) or 2 (tensor cores)",
                o->ffn_path);
  if (o->decode_kernel < 0 || o->decode_kernel > 1)
    return fail(MOE_ERR_INVALID_ARG, "opts->decode_kernel = %d is not 0 (auto) or 1 (never fused)", o->decode_kernel);
  if (o->timer_kernel < -1 || o->timer_kernel >= MOE_KERNEL_COUNT)
    return fail(MOE_ERR_INVALID_ARG, "opts->timer_kernel = %d is not a kernel id or -1", o->timer_kernel);
  if (o->timer_kernel >= 0 && (o->timer_start == nullptr || o->timer_stop == nullptr))
    return fail(MOE_ERR_INVALID_ARG, "opts->timer_kernel = %d needs both timer events", o->timer_kernel);
  if (o->test_withhold < 0 || o->test_withhold > 2)
    return fail(MOE_ERR_INVALID_ARG, "opts->test_withhold = %d is not 0, 1 or 2", o->test_withhold);
  return MOE_OK;
}

}  // namespace

int opt_ffn_path() { return t_opts != nullptr ? t_opts->ffn_path : 0; }
int opt_decode_kernel() { return t_opts != nullptr ? t_opts->decode_kernel : 0; }
int opt_withhold() { return t_opts != nullptr ? t_opts->test_withhold : 0; }
uint64_t opt_wait_ns() {
  return (t_opts != nullptr && t_opts->wait_limit_ns != 0) ? t_opts->wait_limit_ns : kDefaultWaitNs;
}

void before_launch(int id, cudaStream_t s) {
  if (t_opts != nullptr && t_opts->timer_kernel == id && t_opts->timer_start != nullptr)
    cudaEventRecord(static_cast<cudaEvent_t>(t_opts->timer_start), s);
}

void after_launch(int id, cudaStream_t s, int nkernels) {
  t_launches += (uint64_t)nkernels;
  if (t_opts != nullptr && t_opts->timer_kernel == id && t_opts->timer_stop != nullptr)
    cudaEventRecord(static_cast<cudaEvent_t>(t_opts->timer_stop), s);
}

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (g_sm_count[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    g_sm_count[dev] = n;
  }
  return g_sm_count[dev];
}

// ---------------------------------------------------------------------------
// validation
// ---------------------------------------------------------------------------
namespace {

constexpr int32_t kMaxHidden = 32768;
constexpr int32_t kMaxExperts = 1024;
constexpr int32_t kMaxGroups = 32;
constexpr int32_t kMaxIntermediate = 32768;
constexpr int32_t kMaxShared = 64;
constexpr int64_t kMaxTokens = int64_t(1) << 22;

int32_t shared_width(const moe_config& c) {
  if (c.num_shared_experts <= 0) return 0;
  const int32_t per = c.moe_shared_expert_intermediate_size > 0 ? c.moe_shared_expert_intermediate_size
                                                                : c.moe_intermediate_size;
  return per * c.num_shared_experts;
}

moe_status check_range(const char* name, int64_t v, int64_t lo, int64_t hi) {
  if (v < lo || v > hi) return fail(MOE_ERR_INVALID_ARG, "%s = %lld outside [%lld, %lld]", name, (long long)v,
                                    (long long)lo, (long long)hi);
  return MOE_OK;
}

#define MOE_TRY(expr)              \
  do {                             \
    moe_status _st = (expr);       \
    if (_st != MOE_OK) return _st; \
  } while (0)

moe_status validate_config(const moe_config* c) {
  if (c == nullptr) return fail(MOE_ERR_INVALID_ARG, "cfg is NULL");
  MOE_TRY(check_range("hidden_size", c->hidden_size, 1, kMaxHidden));
  MOE_TRY(check_range("num_experts", c->num_experts, 1, kMaxExperts));
  MOE_TRY(check_range("num_experts_per_tok", c->num_experts_per_tok, 1, c->num_experts));
  MOE_TRY(check_range("n_group", c->n_group, 1, kMaxGroups));
  MOE_TRY(check_range("topk_group", c->topk_group, 1, c->n_group));  // zero rejected before any division
  if (c->n_group > 1) {
    if (c->num_experts % c->n_group != 0)
      return fail(MOE_ERR_INVALID_ARG, "num_experts = %d not divisible by n_group = %d", c->num_experts, c->n_group);
    const int gsz = c->num_experts / c->n_group;
    if ((int64_t)c->topk_group * gsz < c->num_experts_per_tok)
      return fail(MOE_ERR_INVALID_ARG, "topk_group * (num_experts / n_group) = %d < num_experts_per_tok = %d",
                  c->topk_group * gsz, c->num_experts_per_tok);
  }
  if (c->score_function != MOE_SCORE_SOFTMAX && c->score_function != MOE_SCORE_SIGMOID)
    return fail(MOE_ERR_INVALID_ARG, "score_function = %d is neither softmax (0) nor sigmoid (1)", c->score_function);
  MOE_TRY(check_range("norm_topk_prob", c->norm_topk_prob, 0, 1));
  if (!std::isfinite(c->routed_scaling_factor))
    return fail(MOE_ERR_INVALID_ARG, "routed_scaling_factor is not finite");
  MOE_TRY(check_range("moe_intermediate_size", c->moe_intermediate_size, 1, kMaxIntermediate));
  MOE_TRY(check_range("num_shared_experts", c->num_shared_experts, 0, kMaxShared));
  MOE_TRY(check_range("moe_shared_expert_intermediate_size", c->moe_shared_expert_intermediate_size, 0,
                      kMaxIntermediate));
  if (c->hidden_size % 8 != 0)
    return fail(MOE_ERR_UNSUPPORTED, "hidden_size = %d is not a multiple of 8 (16-byte rows)", c->hidden_size);
  if (c->moe_intermediate_size % 8 != 0)
    return fail(MOE_ERR_UNSUPPORTED, "moe_intermediate_size = %d is not a multiple of 8 (16-byte rows)",
                c->moe_intermediate_size);
  if (c->moe_shared_expert_intermediate_size % 8 != 0)
    return fail(MOE_ERR_UNSUPPORTED, "moe_shared_expert_intermediate_size = %d is not a multiple of 8",
                c->moe_shared_expert_intermediate_size);
  if (shared_width(*c) > kMaxIntermediate * 4)
    return fail(MOE_ERR_UNSUPPORTED, "shared MLP width %d exceeds %d", shared_width(*c), kMaxIntermediate * 4);
  return MOE_OK;
}

moe_status check_tokens(const moe_config& c, int64_t T) {
  if (T < 0 || T > kMaxTokens) return fail(MOE_ERR_INVALID_ARG, "T = %lld outside [0, %lld]", (long long)T,
                                           (long long)kMaxTokens);
  if (T * c.num_experts_per_tok > INT32_MAX)
    return fail(MOE_ERR_UNSUPPORTED, "T * num_experts_per_tok = %lld exceeds int32 row indices",
                (long long)(T * c.num_experts_per_tok));
  return MOE_OK;
}

moe_status check_ptr(const char* name, const void* p, size_t align, bool required) {
  if (p == nullptr) {
    if (required) return fail(MOE_ERR_INVALID_ARG, "%s is NULL", name);
    return MOE_OK;
  }
  if (reinterpret_cast<uintptr_t>(p) % align != 0)
    return fail(MOE_ERR_INVALID_ARG, "%s is not %zu-byte aligned", name, align);
  return MOE_OK;
}

// opts->w_down_f16 / ws_down_f16 against the call: aligned, and the shared
// MLP's copy present whenever the call runs a shared MLP.
moe_status check_down_f16(bool shared_used) {
  if (t_opts == nullptr) return MOE_OK;
  if (t_opts->w_down_f16 == nullptr) {
    if (t_opts->ws_down_f16 != nullptr)
      return fail(MOE_ERR_INVALID_ARG, "opts->ws_down_f16 is set but opts->w_down_f16 is NULL");
    return MOE_OK;
  }
  MOE_TRY(check_ptr("opts->w_down_f16", t_opts->w_down_f16, 16, true));
  MOE_TRY(check_ptr("opts->ws_down_f16", t_opts->ws_down_f16, 16, shared_used));
  return MOE_OK;
}

// ---------------------------------------------------------------------------
// workspace layout
// ---------------------------------------------------------------------------
constexpr int64_t kLogitsGemvMaxT = 16;  // larger batches: router logits on the tensor cores

struct Layout {
  size_t hdr, logits, wr_planes, logit_parts, topk_idx, topk_w, offsets, row_of, tok_of, active, tile_cnt, tile_base;
  size_t x_perm, h_perm, h_shared, y_slots, shared_out, decode_sync, decode_pre, total;
};

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Split-K partial sums of the router logits: the largest need of any token
// count up to T (a smaller batch can split K more ways), so that a workspace
// sized for T serves every smaller call.
size_t logit_partial_bytes(const moe_config& c, int64_t T) {
  size_t best = 0;
  auto need = [&](int64_t t) {
    if (t <= kLogitsGemvMaxT) return;
    int ksplit = 1, kper = 1;
    logits_split(t, c.num_experts, c.hidden_size, &ksplit, &kper);
    if (ksplit > 1) {
      const size_t b = (size_t)ksplit * t * c.num_experts * 4;
      if (b > best) best = b;
    }
  };
  need(T);
  for (int64_t t = 128; t <= T && t <= 128 * 256; t += 128) need(t);  // splits change only at 128-token steps
  need(kLogitsGemvMaxT + 1 <= T ? kLogitsGemvMaxT + 1 : 0);
  return best;
}

Layout layout(const moe_config& c, int64_t max_tokens) {
  const int64_t T = max_tokens > 0 ? max_tokens : 1;
  const int64_t E = c.num_experts, k = c.num_experts_per_tok, H = c.hidden_size, I = c.moe_intermediate_size;
  const int64_t Is = shared_width(c);
  const int64_t R = T * k;
  Layout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  L.hdr = take(sizeof(WsHeader));
  L.logits = take((size_t)T * E * 4);
  L.wr_planes = take(T > kLogitsGemvMaxT ? (size_t)3 * E * H * 2 : 0);
  L.logit_parts = take(logit_partial_bytes(c, T));
  L.topk_idx = take((size_t)R * 4);
  L.topk_w = take((size_t)R * 4);
  L.offsets = take((size_t)(E + 1) * 4);
  L.row_of = take((size_t)R * 4);
  L.tok_of = take((size_t)R * 4);
  L.active = take((size_t)E * 4);
  L.tile_cnt = take(permute_scratch_ints((int)E, T) * 4);
  L.tile_base = take(permute_scratch_ints((int)E, T) * 4);
  L.x_perm = take((size_t)R * H * 2);
  L.h_perm = take((size_t)R * I * 4);                  // fp32 (streaming) or bf16 (tensor cores)
  L.h_shared = take((size_t)T * (Is > 0 ? Is : 8) * 4);
  L.y_slots = take((size_t)R * H * 4);
  L.shared_out = take((size_t)T * H * 4);
  const bool fused = decode_fused_supported(1, (int)k, (int)E, (int)H, (int)I, (int)Is);
  L.decode_sync = take(fused ? decode_fused_sync_ints((int)H) * 4 : 0);
  L.decode_pre = take(fused ? (size_t)2 * E * 12 : 0);  // up to 2 tokens: scores then keys
  L.total = off;
  return L;
}

template <class P>
P* at(void* ws, size_t off) {
  return reinterpret_cast<P*>(static_cast<char*>(ws) + off);
}

moe_status check_ws(const moe_config& c, int64_t T, void* ws, size_t ws_bytes) {
  if (ws == nullptr) return fail(MOE_ERR_WORKSPACE, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return fail(MOE_ERR_WORKSPACE, "workspace is not 256-byte aligned");
  const size_t need = layout(c, T).total;
  if (ws_bytes < need)
    return fail(MOE_ERR_WORKSPACE, "workspace of %zu bytes < %zu needed for T = %lld", ws_bytes, need, (long long)T);
  return MOE_OK;
}

cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

moe_status run_logits(const moe_config& c, const uint16_t* x, int64_t T, const float* w, float* out, void* ws,
                      cudaStream_t s) {
  cudaError_t e;
  if (T <= kLogitsGemvMaxT) {
    e = launch_router_logits_gemv(c, x, T, w, out, s);
  } else {
    const Layout L = layout(c, T);
    e = launch_router_logits_tc(c, x, T, w, out, at<uint16_t>(ws, L.wr_planes), at<float>(ws, L.logit_parts), s);
  }
  if (e != cudaSuccess) return cuda_fail(e, "router logits");
  return MOE_OK;
}

// The streaming GEMV serves batches of up to kStreamMaxT tokens (measured on
// B200: faster than the tensor cores at 1-2 tokens, slower from 4): every expert
// then has at most that many rows, all taken in one pass over its weights, and
// the weight rows spread over every SM. Larger batches take the tensor cores.
constexpr int64_t kStreamMaxT = 2;

bool use_tensor_cores(const moe_config& c, int64_t T) {
  (void)c;
  if (opt_ffn_path() == 1) return false;
  if (opt_ffn_path() == 2) return true;
  return T > kStreamMaxT;
}

Q8Mat q8mat(const moe_q8_matrix& m) { return Q8Mat{m.q, m.scale, m.bias}; }

// q8: 8-bit affine expert weights (dequantised by the streaming kernels), or
// null for bf16 weights. slots16: when given, the caller takes fp16 slot rows
// (y_slots as [T*k, H] uint16_t) where the fp16 down path runs, and learns
// here whether it did.
moe_status run_ffn(const moe_config& c, int64_t T, const uint16_t* x, const uint16_t* x_perm,
                   const int32_t* offsets, const int32_t* tok_of, const float* topk_w, const uint16_t* wgu,
                   const uint16_t* wd, const uint16_t* swgu, const uint16_t* swd, float* y_slots, float* shared_out,
                   void* ws, bool active_ready, cudaStream_t s, const moe_q8_weights* q8 = nullptr,
                   bool* slots16 = nullptr) {
  const Layout L = layout(c, T);
  WsHeader* hdr = at<WsHeader>(ws, L.hdr);
  int32_t* active = at<int32_t>(ws, L.active);
  cudaError_t e;
  if (!active_ready) {
    e = launch_active_from_offsets(offsets, c.num_experts, active, hdr, s);
    if (e != cudaSuccess) return cuda_fail(e, "active list");
  }
  FfnArgs a{};
  a.x = x;
  a.T = T;
  a.H = c.hidden_size;
  a.I = c.moe_intermediate_size;
  a.Is = shared_width(c);
  a.k = c.num_experts_per_tok;
  a.E = c.num_experts;
  a.offsets = offsets;
  a.tok_of = tok_of;
  a.active = active;
  a.hdr = hdr;
  a.topk_w = topk_w;
  a.w_gate_up = wgu;
  a.w_down = wd;
  a.ws_gate_up = (swgu != nullptr && a.Is > 0) ? swgu : nullptr;
  a.ws_down = a.ws_gate_up != nullptr ? swd : nullptr;
  a.h_perm = at<void>(ws, L.h_perm);
  a.h_shared = at<void>(ws, L.h_shared);
  a.y_slots = y_slots;
  a.shared_out = shared_out;
  if (q8 != nullptr) {
    a.group = q8->group_size;
    a.q_gate_up = q8mat(q8->gate_up);
    a.q_down = q8mat(q8->down);
    if (q8->shared_gate_up.q != nullptr && a.Is > 0) {
      a.qs_gate_up = q8mat(q8->shared_gate_up);
      a.qs_down = q8mat(q8->shared_down);
      a.ws_gate_up = nullptr;
      a.ws_down = nullptr;
    }
    e = launch_gemv_ffn(a, s);
    if (e != cudaSuccess) return cuda_fail(e, "expert ffn (8-bit)");
    return MOE_OK;
  }
  if (use_tensor_cores(c, T)) {
    if (t_opts != nullptr && t_opts->w_down_f16 != nullptr) {
      a.w_down_f16 = t_opts->w_down_f16;
      a.ws_down_f16 = a.ws_gate_up != nullptr ? t_opts->ws_down_f16 : nullptr;
      a.slots_f16 = slots16 != nullptr;
      if (slots16 != nullptr) *slots16 = true;
    }
    if (x_perm == nullptr) {  // the tensor-core path reads expert rows contiguously
      uint16_t* xp = at<uint16_t>(ws, L.x_perm);
      e = launch_gather_rows(offsets, c.num_experts, tok_of, c.num_experts_per_tok, T, x, c.hidden_size, xp, s);
      if (e != cudaSuccess) return cuda_fail(e, "gather rows");
      x_perm = xp;
    }
    e = launch_umma_ffn(a, x_perm, umma_pick_bn(T, a.k, a.E), s);
    if (e != cudaSuccess) return cuda_fail(e, "expert ffn (tensor cores)");
    return MOE_OK;
  }
  e = launch_gemv_ffn(a, s);
  if (e != cudaSuccess) return cuda_fail(e, "expert ffn");
  return MOE_OK;
}

// The dense-prefix MLP as a block of one expert, one slot per token, weight 1
// and no shared MLP: the expert kernels then compute exactly the dense MLP.
moe_config dense_config(int32_t hidden_size, int32_t intermediate_size) {
  moe_config c{};
  c.hidden_size = hidden_size;
  c.num_experts = 1;
  c.num_experts_per_tok = 1;
  c.n_group = 1;
  c.topk_group = 1;
  c.score_function = MOE_SCORE_SOFTMAX;
  c.norm_topk_prob = 0;
  c.routed_scaling_factor = 1.0f;
  c.moe_intermediate_size = intermediate_size;
  c.num_shared_experts = 0;
  c.moe_shared_expert_intermediate_size = 0;
  return c;
}

moe_status check_q8_matrix(const char* name, const moe_q8_matrix& m) {
  char field[64];
  std::snprintf(field, sizeof field, "%s.q", name);
  MOE_TRY(check_ptr(field, m.q, 16, true));
  std::snprintf(field, sizeof field, "%s.scale", name);
  MOE_TRY(check_ptr(field, m.scale, 16, true));
  std::snprintf(field, sizeof field, "%s.bias", name);
  MOE_TRY(check_ptr(field, m.bias, 16, true));
  return MOE_OK;
}

// 8-bit weights: group size, divisibility of every row length by it, and the
// pointers (the shared MLP either 8-bit or bf16, as the config requires).
moe_status validate_q8(const moe_config& c, const moe_q8_weights* w, const uint16_t* ws_gate_up,
                       const uint16_t* ws_down) {
  if (w == nullptr) return fail(MOE_ERR_INVALID_ARG, "8-bit weights (w) is NULL");
  const int g = w->group_size;
  if (g != 32 && g != 64 && g != 128)
    return fail(MOE_ERR_UNSUPPORTED, "group_size = %d is not 32, 64 or 128", g);
  const int Is = shared_width(c);
  if (c.hidden_size % g != 0) return fail(MOE_ERR_UNSUPPORTED, "hidden_size = %d not divisible by group_size = %d", c.hidden_size, g);
  if (c.moe_intermediate_size % g != 0)
    return fail(MOE_ERR_UNSUPPORTED, "moe_intermediate_size = %d not divisible by group_size = %d",
                c.moe_intermediate_size, g);
  MOE_TRY(check_q8_matrix("gate_up", w->gate_up));
  MOE_TRY(check_q8_matrix("down", w->down));
  const bool shared_q8 = w->shared_gate_up.q != nullptr;
  if (Is == 0) {
    if (shared_q8 || ws_gate_up != nullptr)
      return fail(MOE_ERR_INVALID_ARG, "shared MLP weights given but the config has no shared MLP");
    return MOE_OK;
  }
  if (shared_q8) {
    if (Is % g != 0) return fail(MOE_ERR_UNSUPPORTED, "shared MLP width %d not divisible by group_size = %d", Is, g);
    if (ws_gate_up != nullptr) return fail(MOE_ERR_INVALID_ARG, "shared MLP given both as 8-bit and as bf16 (ws_gate_up)");
    MOE_TRY(check_q8_matrix("shared_gate_up", w->shared_gate_up));
    MOE_TRY(check_q8_matrix("shared_down", w->shared_down));
    return MOE_OK;
  }
  MOE_TRY(check_ptr("ws_gate_up", ws_gate_up, 16, true));
  MOE_TRY(check_ptr("ws_down", ws_down, 16, true));
  return MOE_OK;
}

moe_status validate_dense(int32_t hidden_size, int32_t intermediate_size) {
  MOE_TRY(check_range("hidden_size", hidden_size, 1, kMaxHidden));
  MOE_TRY(check_range("intermediate_size", intermediate_size, 1, kMaxIntermediate));
  if (hidden_size % 8 != 0)
    return fail(MOE_ERR_UNSUPPORTED, "hidden_size = %d is not a multiple of 8 (16-byte rows)", hidden_size);
  if (intermediate_size % 8 != 0)
    return fail(MOE_ERR_UNSUPPORTED, "intermediate_size = %d is not a multiple of 8 (16-byte rows)",
                intermediate_size);
  return MOE_OK;
}

}  // namespace
}  // namespace moe

// ---------------------------------------------------------------------------
// extern "C" entry points
// ---------------------------------------------------------------------------
using namespace moe;

extern "C" {

size_t moe_workspace_size(const moe_config* cfg, int64_t max_tokens) {
  if (validate_config(cfg) != MOE_OK) return 0;
  if (check_tokens(*cfg, max_tokens) != MOE_OK) return 0;
  g_err[0] = '\0';
  return layout(*cfg, max_tokens).total;
}

moe_status moe_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (ws == nullptr || ws_bytes < sizeof(WsHeader)) return fail(MOE_ERR_WORKSPACE, "workspace is NULL or too small");
  if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return fail(MOE_ERR_WORKSPACE, "workspace is not 256-byte aligned");
  cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(WsHeader), as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "workspace init");
  return MOE_OK;
}

moe_status moe_router_logits(const moe_config* cfg, const uint16_t* x, int64_t T, const float* router_w,
                             float* logits, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(validate_config(cfg));
  MOE_TRY(check_tokens(*cfg, T));
  MOE_TRY(check_ws(*cfg, T, ws, ws_bytes));
  if (T == 0) return MOE_OK;
  MOE_TRY(check_ptr("x", x, 16, true));
  MOE_TRY(check_ptr("router_w", router_w, 16, true));
  MOE_TRY(check_ptr("logits", logits, 16, true));
  return run_logits(*cfg, x, T, router_w, logits, ws, as_stream(stream));
}

moe_status moe_route(const moe_config* cfg, const float* logits, const float* expert_bias, int64_t T,
                     int32_t* topk_idx, float* topk_w, void* stream) {
  MOE_TRY(validate_config(cfg));
  MOE_TRY(check_tokens(*cfg, T));
  if (T == 0) return MOE_OK;
  MOE_TRY(check_ptr("logits", logits, 4, true));
  MOE_TRY(check_ptr("expert_bias", expert_bias, 4, false));
  MOE_TRY(check_ptr("topk_idx", topk_idx, 4, true));
  MOE_TRY(check_ptr("topk_w", topk_w, 4, true));
  cudaError_t e = launch_route(*cfg, logits, expert_bias, T, topk_idx, topk_w, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "route");
  return MOE_OK;
}

moe_status moe_permute(const moe_config* cfg, const int32_t* topk_idx, int64_t T, const uint16_t* x,
                       int32_t* expert_offsets, int32_t* row_of, int32_t* tok_of, uint16_t* x_perm, void* ws,
                       size_t ws_bytes, void* stream) {
  MOE_TRY(validate_config(cfg));
  MOE_TRY(check_tokens(*cfg, T));
  MOE_TRY(check_ws(*cfg, T, ws, ws_bytes));
  MOE_TRY(check_ptr("expert_offsets", expert_offsets, 4, true));
  if (T > 0) {
    MOE_TRY(check_ptr("topk_idx", topk_idx, 4, true));
    MOE_TRY(check_ptr("row_of", row_of, 4, true));
    MOE_TRY(check_ptr("tok_of", tok_of, 4, true));
    MOE_TRY(check_ptr("x_perm", x_perm, 16, false));
    MOE_TRY(check_ptr("x", x, 16, x_perm != nullptr));
  }
  const Layout L = layout(*cfg, T);
  cudaStream_t s = as_stream(stream);
  if (T == 0) {
    cudaError_t e = cudaMemsetAsync(expert_offsets, 0, (size_t)(cfg->num_experts + 1) * 4, s);
    if (e != cudaSuccess) return cuda_fail(e, "permute");
    return MOE_OK;
  }
  cudaError_t e = launch_permute(*cfg, topk_idx, T, x, expert_offsets, row_of, tok_of, x_perm,
                                 at<int32_t>(ws, L.active), at<int32_t>(ws, L.tile_cnt), at<int32_t>(ws, L.tile_base),
                                 at<WsHeader>(ws, L.hdr), s);
  if (e != cudaSuccess) return cuda_fail(e, "permute");
  return MOE_OK;
}

moe_status moe_expert_ffn(const moe_config* cfg, int64_t T, const uint16_t* x, const uint16_t* x_perm,
                          const int32_t* expert_offsets, const int32_t* tok_of, const float* topk_w,
                          const uint16_t* w_gate_up, const uint16_t* w_down, const uint16_t* ws_gate_up,
                          const uint16_t* ws_down, float* y_slots, float* shared_out, void* ws,
                          size_t ws_bytes, void* stream, const moe_options* opts) {
  MOE_TRY(validate_options(opts));
  CallScope scope(opts);
  MOE_TRY(validate_config(cfg));
  MOE_TRY(check_tokens(*cfg, T));
  MOE_TRY(check_ws(*cfg, T, ws, ws_bytes));
  if (T == 0) return MOE_OK;
  const bool has_shared = shared_width(*cfg) > 0;
  MOE_TRY(check_ptr("x", x, 16, true));
  MOE_TRY(check_ptr("x_perm", x_perm, 16, false));
  MOE_TRY(check_ptr("expert_offsets", expert_offsets, 4, true));
  MOE_TRY(check_ptr("tok_of", tok_of, 4, true));
  MOE_TRY(check_ptr("topk_w", topk_w, 4, false));
  MOE_TRY(check_ptr("w_gate_up", w_gate_up, 16, true));
  MOE_TRY(check_ptr("w_down", w_down, 16, true));
  MOE_TRY(check_ptr("y_slots", y_slots, 16, true));
  MOE_TRY(check_ptr("ws_gate_up", ws_gate_up, 16, false));
  MOE_TRY(check_ptr("ws_down", ws_down, 16, ws_gate_up != nullptr));
  MOE_TRY(check_ptr("shared_out", shared_out, 16, ws_gate_up != nullptr));
  if (ws_gate_up != nullptr && !has_shared)
    return fail(MOE_ERR_INVALID_ARG, "ws_gate_up given but the config has no shared MLP");
  MOE_TRY(check_down_f16(ws_gate_up != nullptr));
  if (ws_gate_up == nullptr) shared_out = nullptr;
  return run_ffn(*cfg, T, x, x_perm, expert_offsets, tok_of, topk_w, w_gate_up, w_down, ws_gate_up, ws_down, y_slots,
                 shared_out, ws, false, as_stream(stream));
}

moe_status moe_combine(const moe_config* cfg, int64_t T, const float* y_slots, const float* shared_out,
                       uint16_t* y, void* stream) {
  MOE_TRY(validate_config(cfg));
  MOE_TRY(check_tokens(*cfg, T));
  if (T == 0) return MOE_OK;
  MOE_TRY(check_ptr("y_slots", y_slots, 16, true));
  MOE_TRY(check_ptr("shared_out", shared_out, 16, false));
  MOE_TRY(check_ptr("y", y, 16, true));
  cudaError_t e =
      launch_combine(y_slots, shared_out, T, cfg->num_experts_per_tok, cfg->hidden_size, y, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "combine");
  return MOE_OK;
}

moe_status moe_forward(const moe_config* cfg, const uint16_t* x, int64_t T, const float* router_w,
                       const float* expert_bias, const float* logits_override, const uint16_t* w_gate_up,
                       const uint16_t* w_down, const uint16_t* ws_gate_up, const uint16_t* ws_down, uint16_t* y,
                       int32_t* topk_idx_out, float* topk_w_out, void* ws, size_t ws_bytes, void* stream,
                       const moe_options* opts) {
  MOE_TRY(validate_options(opts));
  CallScope scope(opts);
  MOE_TRY(validate_config(cfg));
  MOE_TRY(check_tokens(*cfg, T));
  MOE_TRY(check_ws(*cfg, T, ws, ws_bytes));
  if (T == 0) return MOE_OK;
  const moe_config& c = *cfg;
  const bool has_shared = shared_width(c) > 0;
  MOE_TRY(check_ptr("x", x, 16, true));
  MOE_TRY(check_ptr("logits_override", logits_override, 4, false));
  MOE_TRY(check_ptr("router_w", router_w, 16, logits_override == nullptr));
  MOE_TRY(check_ptr("expert_bias", expert_bias, 4, false));
  MOE_TRY(check_ptr("w_gate_up", w_gate_up, 16, true));
  MOE_TRY(check_ptr("w_down", w_down, 16, true));
  MOE_TRY(check_down_f16(has_shared));
  MOE_TRY(check_ptr("ws_gate_up", ws_gate_up, 16, has_shared));
  MOE_TRY(check_ptr("ws_down", ws_down, 16, has_shared));
  MOE_TRY(check_ptr("y", y, 16, true));
  MOE_TRY(check_ptr("topk_idx_out", topk_idx_out, 4, false));
  MOE_TRY(check_ptr("topk_w_out", topk_w_out, 4, false));
  if (!has_shared && ws_gate_up != nullptr)
    return fail(MOE_ERR_INVALID_ARG, "ws_gate_up given but the config has no shared MLP");

  const Layout L = layout(c, T);
  cudaStream_t s = as_stream(stream);
  WsHeader* hdr = at<WsHeader>(ws, L.hdr);
  if (opt_decode_kernel() == 0 && decode_fused_supported(T, c.num_experts_per_tok, c.num_experts, c.hidden_size,
                                                         c.moe_intermediate_size, shared_width(c))) {
    DecodeArgs d{};
    d.x = x;
    d.T = (int)T;
    d.H = c.hidden_size;
    d.E = c.num_experts;
    d.k = c.num_experts_per_tok;
    d.I = c.moe_intermediate_size;
    d.Is = shared_width(c);
    d.n_group = c.n_group;
    d.topk_group = c.topk_group;
    d.score_fn = c.score_function;
    d.norm = c.norm_topk_prob;
    d.scale = c.routed_scaling_factor;
    d.router_w = router_w;
    d.expert_bias = expert_bias;
    d.logits_override = logits_override;
    d.w_gate_up = w_gate_up;
    d.w_down = w_down;
    d.ws_gate_up = has_shared ? ws_gate_up : nullptr;
    d.ws_down = has_shared ? ws_down : nullptr;
    d.logits = at<float>(ws, L.logits);
    d.topk_idx_out = topk_idx_out;
    d.topk_w_out = topk_w_out;
    d.h = at<float>(ws, L.h_perm);
    d.h_shared = at<float>(ws, L.h_shared);
    d.y_slots = at<float>(ws, L.y_slots);
    d.shared_out = at<float>(ws, L.shared_out);
    d.sync = at<int32_t>(ws, L.decode_sync);
    d.pre_orig = at<float>(ws, L.decode_pre);
    d.pre_key = reinterpret_cast<unsigned long long*>(at<char>(ws, L.decode_pre) + (size_t)2 * c.num_experts * 4);
    d.y = y;
    d.hdr = hdr;
    d.wait_ns = opt_wait_ns();
    d.withhold = opt_withhold() == 1 ? 1 : 0;
    cudaError_t e = launch_decode_fused(d, s);
    if (e != cudaSuccess) return cuda_fail(e, "fused decode");
    return MOE_OK;
  }
  const float* logits = logits_override;
  cudaError_t e;
  if (logits == nullptr) {
    float* lg = at<float>(ws, L.logits);
    MOE_TRY(run_logits(c, x, T, router_w, lg, ws, s));
    logits = lg;
  }
  int32_t* idx = topk_idx_out != nullptr ? topk_idx_out : at<int32_t>(ws, L.topk_idx);
  float* w = topk_w_out != nullptr ? topk_w_out : at<float>(ws, L.topk_w);
  e = launch_route(c, logits, expert_bias, T, idx, w, s);
  if (e != cudaSuccess) return cuda_fail(e, "route");
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* tok_of = at<int32_t>(ws, L.tok_of);
  uint16_t* x_perm = use_tensor_cores(c, T) ? at<uint16_t>(ws, L.x_perm) : nullptr;
  e = launch_permute(c, idx, T, x, offsets, at<int32_t>(ws, L.row_of), tok_of, x_perm, at<int32_t>(ws, L.active),
                     at<int32_t>(ws, L.tile_cnt), at<int32_t>(ws, L.tile_base), hdr, s);
  if (e != cudaSuccess) return cuda_fail(e, "permute");
  float* y_slots = at<float>(ws, L.y_slots);
  float* shared_out = has_shared ? at<float>(ws, L.shared_out) : nullptr;
  // on the fp16 down path the routed slot rows are fp16 (half the bytes
  // written by the down pass and read by the combine)
  bool slots16 = false;
  MOE_TRY(run_ffn(c, T, x, x_perm, offsets, tok_of, w, w_gate_up, w_down, has_shared ? ws_gate_up : nullptr,
                  has_shared ? ws_down : nullptr, y_slots, shared_out, ws, true, s, nullptr, &slots16));
  e = slots16 ? launch_combine16(reinterpret_cast<const uint16_t*>(y_slots), shared_out, T, c.num_experts_per_tok,
                                 c.hidden_size, y, s)
              : launch_combine(y_slots, shared_out, T, c.num_experts_per_tok, c.hidden_size, y, s);
  if (e != cudaSuccess) return cuda_fail(e, "combine");
  return MOE_OK;
}

moe_status moe_check_device(void* ws, size_t ws_bytes, void* stream) {
  if (ws == nullptr || ws_bytes < sizeof(WsHeader)) return fail(MOE_ERR_WORKSPACE, "workspace is NULL or too small");
  cudaStream_t s = as_stream(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "stream");
  int32_t word[2] = {0, 0};
  e = cudaMemcpy(word, ws, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read error word");
  if (word[0] == 0) return MOE_OK;
  e = cudaMemsetAsync(ws, 0, sizeof(WsHeader), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "clear error word");
  if (word[0] == MOE_ERR_TIMEOUT) return fail(MOE_ERR_TIMEOUT, "device wait timed out (site %d)", word[1]);
  if (word[0] == MOE_ERR_RANGE)
    return fail(MOE_ERR_RANGE, "a SwiGLU product left fp16's range (expert row %d); use the bf16 down weights",
                word[1]);
  return fail(MOE_ERR_DEVICE_CHECK, "device index check failed (index %d)", word[1]);
}

moe_status moe_ep_send(const moe_config* cfg, int64_t T, const int32_t* expert_offsets, const int32_t* tok_of,
                       const float* topk_w, int64_t* counts, float* row_w, void* stream) {
  MOE_TRY(validate_config(cfg));
  MOE_TRY(check_tokens(*cfg, T));
  MOE_TRY(check_ptr("expert_offsets", expert_offsets, 4, true));
  MOE_TRY(check_ptr("counts", counts, 8, true));
  MOE_TRY(check_ptr("tok_of", tok_of, 4, T > 0));
  MOE_TRY(check_ptr("topk_w", topk_w, 4, T > 0));
  MOE_TRY(check_ptr("row_w", row_w, 4, T > 0));
  cudaError_t e = launch_ep_send(expert_offsets, cfg->num_experts, tok_of, topk_w, T * cfg->num_experts_per_tok,
                                 counts, row_w, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "expert-parallel send lists");
  return MOE_OK;
}

moe_status moe_ep_recv(const int64_t* recv_counts, int32_t P, int32_t n_local, int64_t R_recv, int32_t* local_expert,
                       void* stream) {
  if (P < 1 || n_local < 1 || (int64_t)P * n_local > 1024)
    return fail(MOE_ERR_INVALID_ARG, "P = %d, n_local = %d: need P, n_local >= 1 and P * n_local <= 1024", P,
                n_local);
  if (R_recv < 0) return fail(MOE_ERR_INVALID_ARG, "R_recv = %lld is negative", (long long)R_recv);
  MOE_TRY(check_ptr("recv_counts", recv_counts, 8, true));
  MOE_TRY(check_ptr("local_expert", local_expert, 4, R_recv > 0));
  cudaError_t e = launch_ep_recv(recv_counts, P * n_local, n_local, R_recv, local_expert, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "expert-parallel receive list");
  return MOE_OK;
}

moe_status moe_ep_scatter_back(const float* y_perm, const int32_t* tok_of, int64_t R, int64_t n_slots, int32_t H,
                               float* y_slots, void* stream) {
  if (R < 0 || n_slots < 0) return fail(MOE_ERR_INVALID_ARG, "R = %lld, n_slots = %lld", (long long)R,
                                        (long long)n_slots);
  if (H < 4 || H % 4 != 0 || H > kMaxHidden)
    return fail(MOE_ERR_INVALID_ARG, "H = %d is not a multiple of 4 in [4, %d]", H, kMaxHidden);
  MOE_TRY(check_ptr("y_perm", y_perm, 16, R > 0));
  MOE_TRY(check_ptr("tok_of", tok_of, 4, R > 0));
  MOE_TRY(check_ptr("y_slots", y_slots, 16, R > 0));
  cudaError_t e = launch_ep_scatter_back(y_perm, tok_of, R, n_slots, H, y_slots, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "expert-parallel scatter back");
  return MOE_OK;
}

moe_status moe_convert_bf16_to_f16(const uint16_t* src, uint16_t* dst, int64_t n, int32_t* out_of_range,
                                   void* stream) {
  if (n < 0) return fail(MOE_ERR_INVALID_ARG, "n = %lld is negative", (long long)n);
  MOE_TRY(check_ptr("src", src, 16, n > 0));
  MOE_TRY(check_ptr("dst", dst, 16, n > 0));
  MOE_TRY(check_ptr("out_of_range", out_of_range, 4, true));
  if (n > 0) {
    const uintptr_t s0 = reinterpret_cast<uintptr_t>(src), d0 = reinterpret_cast<uintptr_t>(dst);
    const uintptr_t bytes = (uintptr_t)n * 2;
    if (s0 < d0 + bytes && d0 < s0 + bytes) return fail(MOE_ERR_INVALID_ARG, "src and dst overlap");
  }
  cudaError_t e = launch_convert_bf16_to_f16(src, dst, n, out_of_range, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "bf16 -> fp16 conversion");
  return MOE_OK;
}

uint64_t moe_launch_count(void) { return t_launches; }

const char* moe_last_error(void) { return g_err; }

size_t moe_dense_mlp_workspace_size(int32_t hidden_size, int32_t intermediate_size, int64_t max_tokens) {
  if (validate_dense(hidden_size, intermediate_size) != MOE_OK) return 0;
  const moe_config c = dense_config(hidden_size, intermediate_size);
  if (check_tokens(c, max_tokens) != MOE_OK) return 0;
  g_err[0] = '\0';
  return layout(c, max_tokens).total;
}

moe_status moe_dense_mlp(int32_t hidden_size, int32_t intermediate_size, const uint16_t* x, int64_t T,
                         const uint16_t* w_gate_up, const uint16_t* w_down, uint16_t* y, void* ws, size_t ws_bytes,
                         void* stream, const moe_options* opts) {
  MOE_TRY(validate_options(opts));
  CallScope scope(opts);
  MOE_TRY(validate_dense(hidden_size, intermediate_size));
  const moe_config c = dense_config(hidden_size, intermediate_size);
  MOE_TRY(check_tokens(c, T));
  MOE_TRY(check_ws(c, T, ws, ws_bytes));
  if (T == 0) return MOE_OK;
  MOE_TRY(check_ptr("x", x, 16, true));
  MOE_TRY(check_ptr("w_gate_up", w_gate_up, 16, true));
  MOE_TRY(check_ptr("w_down", w_down, 16, true));
  MOE_TRY(check_ptr("y", y, 16, true));
  MOE_TRY(check_down_f16(false));
  const Layout L = layout(c, T);
  cudaStream_t s = as_stream(stream);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* tok_of = at<int32_t>(ws, L.tok_of);
  float* w = at<float>(ws, L.topk_w);
  float* y_slots = at<float>(ws, L.y_slots);
  cudaError_t e = launch_identity_route(T, offsets, tok_of, w, s);
  if (e != cudaSuccess) return cuda_fail(e, "dense routing");
  // one expert and one slot per token: the permuted rows are the token rows
  MOE_TRY(run_ffn(c, T, x, x, offsets, tok_of, w, w_gate_up, w_down, nullptr, nullptr, y_slots, nullptr, ws, false, s));
  e = launch_combine(y_slots, nullptr, T, 1, hidden_size, y, s);
  if (e != cudaSuccess) return cuda_fail(e, "dense output");
  return MOE_OK;
}

moe_status moe_forward_q8(const moe_config* cfg, const uint16_t* x, int64_t T, const float* router_w,
                          const float* expert_bias, const float* logits_override, const moe_q8_weights* w,
                          const uint16_t* ws_gate_up, const uint16_t* ws_down, uint16_t* y, int32_t* topk_idx_out,
                          float* topk_w_out, void* ws, size_t ws_bytes, void* stream, const moe_options* opts) {
  MOE_TRY(validate_options(opts));
  CallScope scope(opts);
  MOE_TRY(validate_config(cfg));
  MOE_TRY(check_tokens(*cfg, T));
  MOE_TRY(check_ws(*cfg, T, ws, ws_bytes));
  const moe_config& c = *cfg;
  MOE_TRY(validate_q8(c, w, ws_gate_up, ws_down));
  if (opts != nullptr && (opts->w_down_f16 != nullptr || opts->ws_down_f16 != nullptr))
    return fail(MOE_ERR_INVALID_ARG, "opts->w_down_f16 applies to bf16 weights, not to moe_forward_q8");
  if (T == 0) return MOE_OK;
  const bool has_shared = shared_width(c) > 0;
  MOE_TRY(check_ptr("x", x, 16, true));
  MOE_TRY(check_ptr("logits_override", logits_override, 4, false));
  MOE_TRY(check_ptr("router_w", router_w, 16, logits_override == nullptr));
  MOE_TRY(check_ptr("expert_bias", expert_bias, 4, false));
  MOE_TRY(check_ptr("y", y, 16, true));
  MOE_TRY(check_ptr("topk_idx_out", topk_idx_out, 4, false));
  MOE_TRY(check_ptr("topk_w_out", topk_w_out, 4, false));
  const Layout L = layout(c, T);
  cudaStream_t s = as_stream(stream);
  WsHeader* hdr = at<WsHeader>(ws, L.hdr);
  const float* logits = logits_override;
  cudaError_t e;
  if (logits == nullptr) {
    float* lg = at<float>(ws, L.logits);
    MOE_TRY(run_logits(c, x, T, router_w, lg, ws, s));
    logits = lg;
  }
  int32_t* idx = topk_idx_out != nullptr ? topk_idx_out : at<int32_t>(ws, L.topk_idx);
  float* tw = topk_w_out != nullptr ? topk_w_out : at<float>(ws, L.topk_w);
  e = launch_route(c, logits, expert_bias, T, idx, tw, s);
  if (e != cudaSuccess) return cuda_fail(e, "route");
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* tok_of = at<int32_t>(ws, L.tok_of);
  e = launch_permute(c, idx, T, x, offsets, at<int32_t>(ws, L.row_of), tok_of, nullptr, at<int32_t>(ws, L.active),
                     at<int32_t>(ws, L.tile_cnt), at<int32_t>(ws, L.tile_base), hdr, s);
  if (e != cudaSuccess) return cuda_fail(e, "permute");
  float* y_slots = at<float>(ws, L.y_slots);
  float* shared_out = has_shared ? at<float>(ws, L.shared_out) : nullptr;
  MOE_TRY(run_ffn(c, T, x, nullptr, offsets, tok_of, tw, nullptr, nullptr, has_shared ? ws_gate_up : nullptr,
                  has_shared ? ws_down : nullptr, y_slots, shared_out, ws, true, s, w));
  e = launch_combine(y_slots, shared_out, T, c.num_experts_per_tok, c.hidden_size, y, s);
  if (e != cudaSuccess) return cuda_fail(e, "combine");
  return MOE_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// moe_permute_static: the permutation without a caller-provided workspace.
//
// For callers that cannot allocate device memory: code running under a host
// framework that owns every device allocation, plugins whose host forbids
// them, or latency-critical loops where cudaMalloc's implicit device-wide
// synchronisation is not acceptable. Its scratch lives in one file-scope
// device array; every GPU that loads this library holds it until exit.
// ---------------------------------------------------------------------------
namespace moe {
namespace {

constexpr size_t kStaticScratchBytes = size_t(1) << 20;  // 1 MiB
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];
std::atomic<void*> g_static_scratch_addr[64];  // device address of g_static_scratch, per device

// Scratch bytes the permutation needs for T tokens: the 256-byte header (error
// word, active-expert count), the active-expert list, and for T > 128 the
// per-tile counts and bases.
size_t static_scratch_need(const moe_config& c, int64_t T) {
  const size_t tiles = T > 128 ? permute_scratch_ints(c.num_experts, T) * 4 : 0;
  return align256(sizeof(WsHeader)) + align256((size_t)c.num_experts * 4) + 2 * align256(tiles);
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_permute_static(const moe_config* cfg, const int32_t* topk_idx, int64_t T,
                                         const uint16_t* x, int32_t* expert_offsets, int32_t* row_of,
                                         int32_t* tok_of, uint16_t* x_perm, void* stream) {
  MOE_TRY(validate_config(cfg));
  MOE_TRY(check_tokens(*cfg, T));
  MOE_TRY(check_ptr("expert_offsets", expert_offsets, 4, true));
  if (T > 0) {
    MOE_TRY(check_ptr("topk_idx", topk_idx, 4, true));
    MOE_TRY(check_ptr("row_of", row_of, 4, true));
    MOE_TRY(check_ptr("tok_of", tok_of, 4, true));
    MOE_TRY(check_ptr("x_perm", x_perm, 16, false));
    MOE_TRY(check_ptr("x", x, 16, x_perm != nullptr));
  }
  const size_t need = static_scratch_need(*cfg, T);
  if (need > kStaticScratchBytes)
    return fail(MOE_ERR_UNSUPPORTED,
                "T = %lld tokens over num_experts = %d needs %zu bytes of scratch; the static scratch of "
                "moe_permute_static holds %zu bytes (use moe_permute with a workspace)",
                (long long)T, cfg->num_experts, need, kStaticScratchBytes);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "moe_permute_static: current device");
  if (dev < 0 || dev >= 64) return fail(MOE_ERR_UNSUPPORTED, "device ordinal %d above 63", dev);
  // Set-up, once per device, with that device current: the host-side name of a
  // __device__ array is not its device address; ask the runtime for it.
  void* base = g_static_scratch_addr[dev].load(std::memory_order_acquire);
  if (base == nullptr) {
    e = cudaGetSymbolAddress(&base, g_static_scratch);
    if (e != cudaSuccess || base == nullptr) return cuda_fail(e, "moe_permute_static: cudaGetSymbolAddress");
    g_static_scratch_addr[dev].store(base, std::memory_order_release);
  }
  cudaStream_t s = as_stream(stream);
  char* p = static_cast<char*>(base);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(p);
  int32_t* active = reinterpret_cast<int32_t*>(p + align256(sizeof(WsHeader)));
  const size_t tiles = T > 128 ? permute_scratch_ints(cfg->num_experts, T) * 4 : 0;
  int32_t* tile_cnt = reinterpret_cast<int32_t*>(p + align256(sizeof(WsHeader)) + align256((size_t)cfg->num_experts * 4));
  int32_t* tile_base = reinterpret_cast<int32_t*>(reinterpret_cast<char*>(tile_cnt) + align256(tiles));
  // The array keeps the previous call's contents: the header (error word and
  // active count) must start at zero; the other regions are fully rewritten.
  e = cudaMemsetAsync(hdr, 0, sizeof(WsHeader), s);
  if (e != cudaSuccess) return cuda_fail(e, "moe_permute_static: clear scratch header");
  if (T == 0) {
    e = cudaMemsetAsync(expert_offsets, 0, (size_t)(cfg->num_experts + 1) * 4, s);
    if (e != cudaSuccess) return cuda_fail(e, "moe_permute_static");
    return MOE_OK;
  }
  e = launch_permute(*cfg, topk_idx, T, x, expert_offsets, row_of, tok_of, x_perm, active, tile_cnt, tile_base, hdr,
                     s);
  if (e != cudaSuccess) return cuda_fail(e, "moe_permute_static");
  return MOE_OK;
}
