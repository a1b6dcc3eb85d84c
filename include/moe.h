/*
 * moe.h -- C ABI of libmoe.so, the B200 (sm_100a) grouped top-k MoE block.
 *
 * The block is the Bailing/Ling mixture-of-experts feed-forward layer:
 *   router (softmax or sigmoid scores, selection-only expert bias, optional
 *   grouped top-k, renormalisation, routed scaling) -> token-to-expert
 *   permutation -> SwiGLU routed experts + one always-on shared MLP ->
 *   weighted combine.
 *
 * Sources (page title, section):
 *   [ROUTER]  mlxcel issue #838 "add Ant Group Ling / Bailing MoE (bailing_moe)",
 *             section "Router: selection uses biased scores, weights come from
 *             unbiased scores".
 *   [SCALE]   same issue, "moe_router_enable_routed_scaling is dead code
 *             upstream" (the scaling factor is applied unconditionally).
 *   [SHARED]  same issue, "Shared experts are one wide MLP, not N separate
 *             experts".
 *   [FIELDS]  same issue, "Config fields the checkpoint does not contain".
 *   [ARCH]    same issue, "Architecture notes".
 *   [DEFENSE] same issue, "Defensive requirements" (validate before use, reject
 *             instead of terminating, take gather bounds from real shapes).
 *   [LING26]  model card "Ling-2.6-flash-JANGTQ", "Architecture
 *             (bailing_hybrid)", paragraph "MoE routing".
 *   [GGUF]    page "Ling-3.0-flash-GGUF", "Measured performance": a decode
 *             step touches just the chosen experts' weights.
 *   [Q8]      model card "Ling-3.0-tiny-8bit-XL-mlx", "XL Quantization Recipe"
 *             (routed experts and the dense MLP 8-bit; router and shared
 *             experts bf16); model card "Ling-2.6-flash-JANGTQ", quantization
 *             summary (8-bit affine on the shared experts and the layer-0
 *             dense MLP); mlxcel issue #838, "Upstream sanitize" (quantized
 *             expert tensors carry weight, scales and biases; group size 64).
 *   [DENSE]   mlxcel issue #838, "Architecture notes": the first
 *             first_k_dense_replace layers use a plain MLP at
 *             intermediate_size instead of the MoE block; model card
 *             "Ling-2.6-flash-JANGTQ", "Architecture (bailing_hybrid)", layer
 *             table: layer 0 is a dense MLP of intermediate size 9216.
 *
 * Conventions for every entry point:
 *   - Pointers are DEVICE pointers unless stated otherwise. bf16 tensors are
 *     passed as uint16_t (raw bf16 bits), row-major, densely packed.
 *   - Every matrix and vector pointer must be 16-byte aligned (vector and TMA
 *     loads); the workspace 256-byte aligned.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL
 *     is the legacy default stream). They return once the work is enqueued.
 *   - The caller owns every buffer. The library allocates no device memory and
 *     keeps no state between calls beyond a per-device attribute cache (SM
 *     count, the address of moe_permute_static's scratch array) and per-thread
 *     error text and launch count. Kernel choices, wait limits and timing hooks
 *     travel with each call in a moe_options struct (NULL: the defaults).
 *   - All arguments are validated on the host BEFORE any launch. A rejected call
 *     launches nothing and returns a status; the library never aborts or throws
 *     across this ABI ([DEFENSE]). moe_last_error() names the offending field.
 *   - Index-driven reads on the device are bounds-checked against the sizes
 *     passed in; an out-of-range id is skipped and recorded in the workspace
 *     error word, which moe_check_device() reports as MOE_ERR_DEVICE_CHECK.
 *   - Device-side waits are bounded; a wait that runs out records
 *     MOE_ERR_TIMEOUT in the same word and the kernel returns. After a
 *     timeout, call moe_check_device (which reports it and zeroes the
 *     header) or moe_workspace_init before the workspace's next use: the
 *     fused decode kernel's grid barrier counts arrivals in the header, and
 *     an interrupted count would make every later barrier wait out its limit.
 *     For the same reason a workspace belongs to one device (the barrier's
 *     generation size is that device's SM count).
 *
 * Shapes (T tokens, H hidden_size, E num_experts, k num_experts_per_tok,
 * I moe_intermediate_size, Is the shared MLP width):
 *   x          [T, H]      bf16
 *   router_w   [E, H]      fp32          (router projection, mlp.gate)
 *   expert_bias[E]         fp32 or NULL  (e_score_correction_bias)
 *   w_gate_up  [E, 2I, H]  bf16          rows [0,I) gate_proj, rows [I,2I) up_proj
 *   w_down     [E, H, I]   bf16          down_proj
 *   ws_gate_up [2Is, H]    bf16          shared MLP, same row split
 *   ws_down    [H, Is]     bf16
 *   Is = (moe_shared_expert_intermediate_size ? that : I) * num_shared_experts
 *   ([SHARED]: one wide MLP, added at weight 1.0, never routed).
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* a config field, size or pointer is invalid */
  MOE_ERR_UNSUPPORTED = 2,  /* valid for the method, outside this build's limits */
  MOE_ERR_WORKSPACE = 3,    /* workspace missing or smaller than moe_workspace_size */
  MOE_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
  MOE_ERR_DEVICE_CHECK = 5, /* a device-side index check failed (see moe_check_device) */
  MOE_ERR_TIMEOUT = 6,      /* a bounded device-side wait ran out */
  MOE_ERR_RANGE = 7         /* a value left the range of an fp16 intermediate (see moe_options.w_down_f16) */
} moe_status;

typedef enum { MOE_SCORE_SOFTMAX = 0, MOE_SCORE_SIGMOID = 1 } moe_score_function;

/* Block configuration. Field names follow the Bailing config ([FIELDS]). */
typedef struct {
  int32_t hidden_size;          /* H: multiple of 8, <= 32768 */
  int32_t num_experts;          /* E: 1..1024 */
  int32_t num_experts_per_tok;  /* k: 1..E */
  int32_t n_group;              /* >= 1; E % n_group == 0 when > 1; <= 32 */
  int32_t topk_group;           /* 1..n_group; == n_group keeps every group */
  int32_t score_function;       /* moe_score_function; anything else is rejected ([FIELDS]) */
  int32_t norm_topk_prob;       /* 0/1: renormalise, only when k > 1, eps 1e-20 ([ROUTER]) */
  float routed_scaling_factor;  /* finite; always applied ([SCALE]) */
  int32_t moe_intermediate_size;               /* I: multiple of 8, <= 32768 */
  int32_t num_shared_experts;                  /* 0..64; 0 = no shared MLP */
  int32_t moe_shared_expert_intermediate_size; /* 0 = use I ([SHARED]) */
} moe_config;

/* Kernels that moe_options.timer_kernel can bracket. */
typedef enum {
  MOE_KERNEL_ROUTER_LOGITS = 0,
  MOE_KERNEL_ROUTE = 1,
  MOE_KERNEL_PERMUTE = 2,
  MOE_KERNEL_EXPERT_GATE_UP = 3, /* routed + shared gate/up projections with SwiGLU */
  MOE_KERNEL_EXPERT_DOWN = 4,    /* routed + shared down projections, weighted */
  MOE_KERNEL_COMBINE = 5,
  MOE_KERNEL_DECODE_FUSED = 6,   /* the whole block for a few tokens in one launch (moe_forward) */
  MOE_KERNEL_COUNT = 7
} moe_kernel_id;

/* Per-call options of moe_expert_ffn, moe_forward, moe_forward_q8 and
 * moe_dense_mlp. Pass NULL for the defaults; a zero-initialised struct with
 * timer_kernel = -1 is the same. The library reads the struct during the call
 * only and keeps no pointer to it. */
typedef struct {
  int32_t ffn_path;       /* expert kernels: 0 automatic (the streaming GEMV for
                             T <= 2 tokens when the block is not fused, the
                             tensor-core grouped GEMM above), 1 always the
                             streaming GEMV, 2 always the tensor-core GEMM */
  int32_t decode_kernel;  /* moe_forward on a few tokens: 0 automatic (one fused
                             launch where the shapes allow it), 1 never fused
                             (the separate kernels of the larger batches) */
  uint64_t wait_limit_ns; /* bound on every device-side wait of the call's
                             kernels; 0 = the default of 2 s. A wait that runs
                             out records MOE_ERR_TIMEOUT and the kernel returns. */
  int32_t timer_kernel;   /* moe_kernel_id whose launches in this call are
                             bracketed by the two events, or -1 for none */
  void* timer_start;      /* cudaEvent_t recorded just before each such launch */
  void* timer_stop;       /* cudaEvent_t recorded just after it */
  int32_t test_withhold;  /* test aid, 0 in normal use. 1: CTA 0 of the fused
                             decode kernel never arrives at its grid barrier,
                             so every other CTA's wait runs out; 2: the tensor-core
                             expert kernel withholds its first accumulator
                             hand-over, so the epilogue's wait runs out. Both
                             end in MOE_ERR_TIMEOUT after wait_limit_ns and
                             leave the workspace usable once moe_check_device
                             has reported. Any other value is rejected. */
  /* Optional fp16 copies of the call's down-projection weights (layouts of
   * w_down [E,H,I] and ws_down [H,Is], e.g. from moe_convert_bf16_to_f16),
   * read by the tensor-core expert path only; NULL: bf16 throughout. With
   * them, the SwiGLU product h is rounded to fp16 (11 significant bits)
   * rather than split into two bf16 planes (about 16), and the down pass
   * runs one fp16 MMA per k-step instead of two bf16 ones, with half the h
   * bytes. An h beyond fp16's range (|h| >= 65520, or not finite) is
   * recorded as MOE_ERR_RANGE in the workspace error word. ws_down_f16 is
   * required when the block has a shared MLP. The bf16 weights stay
   * required: the streaming kernels read them. */
  const uint16_t* w_down_f16;
  const uint16_t* ws_down_f16;
} moe_options;

/* Workspace bytes moe_permute, moe_expert_ffn and moe_forward need for up to
 * max_tokens tokens. Returns 0 (and sets moe_last_error) on an invalid config.
 * The workspace holds the device error word, routing and permutation scratch
 * and the intermediate activations. Only its header must be zeroed, once, by
 * moe_workspace_init; the rest needs no initialisation. */
size_t moe_workspace_size(const moe_config* cfg, int64_t max_tokens);

/* Zeroes the workspace's 256-byte header (its device error word). Call once
 * after allocating a workspace and before its first use; moe_check_device
 * clears the word again after reporting. Asynchronous on `stream`. */
moe_status moe_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Router projection ([ROUTER]; router weight mlp.gate [E, H]):
 *   logits[t, e] = sum_h float(x[t, h]) * router_w[e, h]   (fp32 accumulate)
 * x [T,H] bf16, router_w [E,H] fp32, logits [T,E] fp32 out. T may be 0.
 * T <= 16: an fp32 streaming GEMV over router_w. Larger T: the tensor cores,
 * with router_w split exactly into three bf16 planes (hi + mid + lo, to one
 * fp32 ulp) in the workspace, so every product is exact and the sum is
 * accumulated in fp32 over K = 3H. ws / ws_bytes >= moe_workspace_size(cfg, T). */
moe_status moe_router_logits(const moe_config* cfg, const uint16_t* x, int64_t T,
                             const float* router_w, float* logits, void* ws, size_t ws_bytes, void* stream);

/* Router on fp32 gates ([ROUTER], [ARCH], [LING26]). Per token:
 *   s    = softmax(logits) or sigmoid(logits), each score the fp32 rounding of
 *          the value evaluated in fp64;
 *   sel  = s + expert_bias (fp32; selection only; skipped when bias is NULL);
 *   if n_group > 1 and topk_group < n_group: group score = top-1 + top-2 of sel
 *          in each contiguous group of E/n_group experts; keep the topk_group
 *          best groups (ties: lower group id), sel = -inf elsewhere;
 *   topk_idx[t, 0..k) = the k largest sel, ordered (sel desc, id asc);
 *   w_j  = s[idx_j] (UNBIASED); if norm_topk_prob and k > 1:
 *          w_j /= (((w_0 + w_1) + ...) + 1e-20f); then w_j *= routed_scaling_factor.
 * logits [T,E] fp32; expert_bias [E] fp32 or NULL; topk_idx [T,k] int32 out;
 * topk_w [T,k] fp32 out. Indices are always valid and distinct, even for
 * non-finite logits (whose selection is then unspecified). */
moe_status moe_route(const moe_config* cfg, const float* logits, const float* expert_bias, int64_t T,
                     int32_t* topk_idx, float* topk_w, void* stream);

/* Token-to-expert permutation (histogram -> exclusive scan -> stable scatter).
 * The T*k assignments are ordered by (expert, token):
 *   expert_offsets [E+1] int32 out: rows of expert e are [off[e], off[e+1]);
 *   row_of [T*k] int32 out: permuted row of assignment (t, j), index t*k + j;
 *   tok_of [T*k] int32 out: the slot t*k + j that permuted row r holds;
 *   x_perm [T*k, H] bf16 out (optional): x_perm[r] = x[tok_of[r] / k];
 *   x may be NULL when x_perm is NULL.
 * topk_idx entries outside [0, E) or repeated within a token are skipped and
 * recorded as MOE_ERR_DEVICE_CHECK in the workspace error word. */
moe_status moe_permute(const moe_config* cfg, const int32_t* topk_idx, int64_t T, const uint16_t* x,
                       int32_t* expert_offsets, int32_t* row_of, int32_t* tok_of, uint16_t* x_perm,
                       void* ws, size_t ws_bytes, void* stream);

/* Routed SwiGLU experts and the shared MLP ([ARCH], [SHARED], [GGUF]):
 *   F_e(v) = down_e( silu(gate_e v) * up_e v ),   silu(z) = z / (1 + exp(-z)),
 * fp32 accumulation. The SwiGLU product stays fp32 on the streaming (decode)
 * path. The tensor-core path's MMA operands are 16-bit: it keeps h as two bf16
 * planes (h_hi = bf16(h), h_lo = bf16(h - h_hi)) whose products the down pass
 * adds, or, given opts->w_down_f16, as one fp16 plane. Only experts with rows
 * in expert_offsets are read.
 *   y_slots[t*k + j] = topk_w[t*k + j] * F_{e}(x_t)  (fp32) for the expert e
 *                      holding that slot (topk_w NULL: weight 1);
 *   shared_out[t]    = F_shared(x_t)  (fp32; when ws_gate_up is not NULL).
 * x [T,H]; x_perm [T*k,H] from moe_permute, or NULL (rows are then gathered
 * from x through tok_of); expert_offsets [E+1], tok_of [T*k] from moe_permute;
 * y_slots [T*k,H] fp32 out; shared_out [T,H] fp32 out or NULL. */
moe_status moe_expert_ffn(const moe_config* cfg, int64_t T, const uint16_t* x, const uint16_t* x_perm,
                          const int32_t* expert_offsets, const int32_t* tok_of, const float* topk_w,
                          const uint16_t* w_gate_up, const uint16_t* w_down,
                          const uint16_t* ws_gate_up, const uint16_t* ws_down,
                          float* y_slots, float* shared_out,
                          void* ws, size_t ws_bytes, void* stream, const moe_options* opts);

/* Weighted combine ([ROUTER], [SHARED]: out = routed mixture + shared(x)):
 *   y[t] = bf16( sum_{j<k} y_slots[t*k + j] + shared_out[t] ),
 * summed in fp32 in slot order then the shared row, rounded once: deterministic.
 * y_slots [T*k,H] fp32 (already weighted); shared_out [T,H] fp32 or NULL;
 * y [T,H] bf16 out. */
moe_status moe_combine(const moe_config* cfg, int64_t T, const float* y_slots, const float* shared_out,
                       uint16_t* y, void* stream);

/* The whole block: router logits -> route -> permute -> experts -> combine.
 * With opts->decode_kernel = 0 (the default), T <= 2 tokens, at most 32 slots
 * (T*k), E <= 1024 and H <= 8192, the block runs as one cooperative launch
 * (MOE_KERNEL_DECODE_FUSED): a weight-streaming kernel, one CTA per SM, with
 * one bounded grid barrier and bounded per-expert and per-row counters, that
 * multiplies on the CUDA cores (fp32 sums throughout).
 * Its routing (indices and weights) is bit-identical to moe_route on the same
 * logits; its logits and output equal those of the separate kernels up to the
 * fp32 summation order of the dot products. Larger batches run the separate
 * kernels; on the tensor-core path with opts->w_down_f16, h and the routed
 * slot rows handed from the down pass to the combine are fp16 (the shared
 * MLP's rows stay fp32), half the bytes of the fp32 rows of moe_expert_ffn.
 *   logits_override [T,E] fp32 or NULL: when given, replaces the router
 *   projection (router_w may then be NULL).
 *   topk_idx_out [T,k] int32 / topk_w_out [T,k] fp32: optional copies of the
 *   routing. y [T,H] bf16 out. ws / ws_bytes >= moe_workspace_size(cfg, T).
 *   opts: per-call options or NULL. */
moe_status moe_forward(const moe_config* cfg, const uint16_t* x, int64_t T, const float* router_w,
                       const float* expert_bias, const float* logits_override,
                       const uint16_t* w_gate_up, const uint16_t* w_down,
                       const uint16_t* ws_gate_up, const uint16_t* ws_down,
                       uint16_t* y, int32_t* topk_idx_out, float* topk_w_out,
                       void* ws, size_t ws_bytes, void* stream, const moe_options* opts);

/* The dense-prefix MLP ([DENSE]): y = W_down (silu(W_gate x) * (W_up x)), bf16
 * in and out, fp32 accumulation, on the expert kernels of moe_expert_ffn (the
 * MLP is run as a block of one expert, one slot per token, weight 1.0).
 *   w_gate_up [2*intermediate_size, hidden_size] bf16: rows [0, Id) gate_proj,
 *   rows [Id, 2Id) up_proj. w_down [hidden_size, intermediate_size] bf16.
 *   x, y [T, hidden_size] bf16. hidden_size and intermediate_size must be
 *   multiples of 8. ws / ws_bytes >= moe_dense_mlp_workspace_size(.., T). */
size_t moe_dense_mlp_workspace_size(int32_t hidden_size, int32_t intermediate_size, int64_t max_tokens);
moe_status moe_dense_mlp(int32_t hidden_size, int32_t intermediate_size, const uint16_t* x, int64_t T,
                         const uint16_t* w_gate_up, const uint16_t* w_down, uint16_t* y,
                         void* ws, size_t ws_bytes, void* stream, const moe_options* opts);

/* 8-bit affine weights ([Q8]): for each row and each group of `group_size`
 * consecutive inputs, w = scale * q + bias, with q uint8 and scale, bias bf16
 * (raw bits). A matrix of R rows and K inputs: q [R, K], scale and bias
 * [R, K / group_size], all row-major, 16-byte aligned. */
typedef struct {
  const uint8_t*  q;
  const uint16_t* scale;
  const uint16_t* bias;
} moe_q8_matrix;

typedef struct {
  int32_t group_size;           /* 32, 64 or 128; divides H, I and Is */
  moe_q8_matrix gate_up;        /* routed experts: R = E*2I, K = H (rows as w_gate_up) */
  moe_q8_matrix down;           /* routed experts: R = E*H,  K = I (rows as w_down) */
  moe_q8_matrix shared_gate_up; /* R = 2Is, K = H; q NULL: the shared MLP is bf16 (ws_* of moe_forward_q8) */
  moe_q8_matrix shared_down;    /* R = H, K = Is */
} moe_q8_weights;

/* The whole block with 8-bit affine expert weights, dequantised in the
 * streaming expert kernels (every T; the router projection stays fp32). The
 * shared MLP is 8-bit when w->shared_gate_up.q is set, else bf16 from
 * ws_gate_up / ws_down (the XL recipe keeps it bf16). Routing, permutation and
 * combine are those of moe_forward. H, I and Is must be multiples of 16 (one
 * 16-byte chunk of codes per lane step). ws / ws_bytes >= moe_workspace_size.
 * Arithmetic: per 16 inputs of one group, scale * sum(q * v) + bias * sum(v)
 * in fp32, the products q * v formed exactly on activations scaled by 2^33;
 * activations x and the fp32 SwiGLU products h must stay below 2^95 in
 * magnitude (larger ones give non-finite outputs). */
moe_status moe_forward_q8(const moe_config* cfg, const uint16_t* x, int64_t T, const float* router_w,
                          const float* expert_bias, const float* logits_override, const moe_q8_weights* w,
                          const uint16_t* ws_gate_up, const uint16_t* ws_down, uint16_t* y,
                          int32_t* topk_idx_out, float* topk_w_out, void* ws, size_t ws_bytes, void* stream,
                          const moe_options* opts);

/* Synchronises `stream`, reads and clears the workspace error word (after an
 * error the whole 256-byte header is cleared, barrier state included). Returns
 * MOE_OK, MOE_ERR_DEVICE_CHECK, MOE_ERR_TIMEOUT or MOE_ERR_RANGE (the first
 * error recorded), or MOE_ERR_CUDA if the stream itself reports an error.
 * Blocking. */
moe_status moe_check_device(void* ws, size_t ws_bytes, void* stream);

/* Expert parallelism ([ARCH]: a distributed entry; [SHARED]: the shared MLP
 * is never routed, so every rank keeps it). The routed experts are placed
 * contiguously, E/P per rank. A rank routes and permutes its own T tokens; its
 * permuted rows are then grouped by expert, hence by owner. The caller moves
 * rows with two variable-size all-to-alls; these three calls build what the
 * exchange needs, on the device, in the call's stream:
 *
 * moe_ep_send: counts[e] = expert_offsets[e+1] - expert_offsets[e] (int64
 *   [E], the payload of the count exchange, [P, E/P] by owner) and
 *   row_w[r] = topk_w[tok_of[r]] (fp32 [T*k]) for the rows r < expert_offsets[E]
 *   (the routing weight travels with its row). expert_offsets [E+1], tok_of
 *   [T*k] from moe_permute; topk_w [T*k] fp32.
 * moe_ep_recv: the local expert id (0 .. n_local-1, int32) of every received
 *   row. recv_counts [P * n_local] int64 is what the count exchange delivered:
 *   rows arrive source by source, each source's grouped by local expert in
 *   ascending order. R_recv = sum(recv_counts); rows past it get -1.
 *   n_local = E/P; P * n_local <= 1024.
 * moe_ep_scatter_back: y_slots[tok_of[r]] = y_perm[r] for r < R (the rows
 *   this rank sent, returned in the order sent), fp32 [., H], H a multiple of
 *   4; a slot outside [0, n_slots) is skipped. */
moe_status moe_ep_send(const moe_config* cfg, int64_t T, const int32_t* expert_offsets, const int32_t* tok_of,
                       const float* topk_w, int64_t* counts, float* row_w, void* stream);
moe_status moe_ep_recv(const int64_t* recv_counts, int32_t P, int32_t n_local, int64_t R_recv, int32_t* local_expert,
                       void* stream);
moe_status moe_ep_scatter_back(const float* y_perm, const int32_t* tok_of, int64_t R, int64_t n_slots,
                               int32_t H, float* y_slots, void* stream);

/* dst[i] = fp16(src[i]) for n bf16 values, round to nearest even: a one-time
 * conversion of down-projection weights for moe_options.w_down_f16. Every
 * bf16 value of magnitude 2^-14 .. 65504 is exact in fp16; smaller ones keep
 * fp16's subnormal spacing of 2^-24 (an absolute error of at most 2^-25).
 * *out_of_range (device int32, zeroed by the call) counts the values that
 * become infinite or are not finite (|v| >= 65520, inf, NaN); weights with a
 * nonzero count cannot use the fp16 path. src and dst may not overlap. */
moe_status moe_convert_bf16_to_f16(const uint16_t* src, uint16_t* dst, int64_t n, int32_t* out_of_range,
                                   void* stream);

/* Number of this library's kernel launches made by the calling thread since
 * the library was loaded (a host-side counter). */
uint64_t moe_launch_count(void);

/* moe_permute without a workspace, for callers that cannot allocate device
 * memory (a host framework that owns every device allocation, a plugin host
 * that forbids them, or a latency-critical loop where cudaMalloc's implicit
 * device synchronisation is unacceptable). The pages have no counterpart: it
 * is a packaging of the permutation above, with the same outputs bit for bit.
 *   Scratch: one file-scope 1 MiB device array, held by every GPU that loads
 *   this library until exit. T beyond what 1 MiB holds is rejected with
 *   MOE_ERR_UNSUPPORTED (about 65k tokens at E = 256, 16k at E = 1024; any T
 *   <= 128). The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture. The address is then cached for the life of
 *   the process: it does not survive cudaDeviceReset (or the destruction of
 *   the device's primary context), after which this function must not be
 *   called on that device again.
 *   Calls on one device share that device's array: two of them whose work
 *   overlaps on the GPU (issued on different streams, or from different
 *   threads) race and corrupt each other's results; calls in one stream, and
 *   calls on different devices, are safe. Each call clears what must start
 *   at zero.
 *   Invalid or repeated ids are skipped as in moe_permute; with no workspace
 *   error word to read, a caller detects them by expert_offsets[E] < T*k.
 * Arguments, layouts and ownership otherwise as moe_permute. Allocates nothing. */
moe_status moe_permute_static(const moe_config* cfg, const int32_t* topk_idx, int64_t T, const uint16_t* x,
                              int32_t* expert_offsets, int32_t* row_of, int32_t* tok_of, uint16_t* x_perm,
                              void* stream);

/* Per-thread text of the last rejected call ("" when none). Never NULL. */
const char* moe_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
