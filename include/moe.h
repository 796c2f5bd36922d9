/*
 * moe.h: C ABI of the sparse Mixture-of-Experts layer on NVIDIA B200 (sm_100a): the forward
 * pass, its router statistics, expert weights in MX formats, the redirect overflow policy and
 * the backward pass.
 *
 * The layer (page «Sparse Mixture-of-Experts», bigdataschool wiki):
 *   1. router logits      L = x W_r^T (+ b), a linear layer without bias term
 *                         (section «Роутер и top-k gating»; b is an optional per-expert
 *                         additive logit bias used to skew loads);
 *   2. softmax over the N experts, top-k experts per token, and the k probabilities
 *      renormalised to sum to one (same section);
 *   3. capacity: ceil(capacity_factor * T / N) slots per expert; a (token, choice) pair that
 *      arrives at a full expert is dropped and contributes nothing, so a token whose every
 *      choice is dropped leaves the layer unchanged through the residual
 *      (section «Expert capacity и capacity factor»); arrival order is every token's first
 *      choice in token order, then every token's second choice, and so on;
 *   4. the kept pairs are sorted by expert id into expert-contiguous rows and every expert's
 *      FFN runs as one grouped GEMM over packed expert weights (page «Что такое Mixture of
 *      Experts (MoE) в трансформерах», aglamov.biz, sections «Бэкенд для экспертов»,
 *      grouped_mm, and «Динамическая загрузка весов с WeightConverter», packed layouts);
 *   5. the output is residual + the sum of the kept experts' outputs weighted by the
 *      renormalised router probabilities (section «Роутер и top-k gating»).
 * moe_backward differentiates these steps (the choice of experts and the slots pass no
 * gradient); moe_redirect_overflow replaces step 3's dropping by redirection.
 *
 * Conventions for every call:
 *   - Every pointer is a DEVICE pointer, allocated and owned by the caller, 16-byte aligned.
 *     The library allocates nothing and frees nothing. Its process-wide state is: a cached
 *     driver entry point; per-device kernel attributes and device properties, set or read
 *     once per device; the wait limit of moe_debug_set_wait_timeout_ns; and, for
 *     moe_route_noalloc only, static scratch arrays in device memory with their cached
 *     device addresses.
 *   - "bf16" buffers hold bfloat16 bit patterns (uint16_t). All tensors are row-major and
 *     contiguous.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*; NULL = legacy
 *     default stream). No call synchronises with the host. The number of kept rows R lives
 *     only on the device. Row buffers are sized for R_max = moe_max_rows().
 *   - Host-side validation runs before any launch:
 *       MOE_ERR_INVALID      null pointer where one is required, negative size, k > N, k < 1
 *       MOE_ERR_UNSUPPORTED  d_model or d_ff not a multiple of 64, N > 256, k > 8, a pointer
 *                            that is not 16-byte aligned, a device that is not sm_100, or a
 *                            grid whose CTAs wait on one another (the grouped FFN) that the
 *                            device cannot hold resident at once
 *       MOE_ERR_WORKSPACE    ws_bytes below what moe_workspace_bytes() reports
 *       MOE_ERR_CUDA         a CUDA runtime or driver call failed while launching
 *     Nothing is launched when validation fails. T == 0 is valid and launches nothing.
 *   - Faults found on the device are written into the workspace's status word, not trapped:
 *       MOE_ERR_TIMEOUT      a bounded wait inside a kernel ran out (the kernel then stops)
 *       MOE_ERR_BOUNDS       a row index computed from device data fell outside its buffer
 *                            (the access is skipped)
 *     moe_read_device_error() reads and clears that word.
 *   - Inputs must be finite; results for NaN or Inf inputs are unspecified.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID = -1,
  MOE_ERR_UNSUPPORTED = -2,
  MOE_ERR_CUDA = -3,
  MOE_ERR_WORKSPACE = -4,
  MOE_ERR_TIMEOUT = -5,
  MOE_ERR_BOUNDS = -6
} moe_status;

typedef enum { MOE_ACT_SWIGLU = 0, MOE_ACT_GELU = 1 } moe_act;

/* Storage of the expert weights. MX formats follow the OCP Microscaling (MX) Specification
 * v1.0: every block of 32 consecutive elements along the reduction axis K shares one E8M0
 * scale X = 2^(s - 127) (s = 255: NaN), and an element's value is X times its own value.
 *   MOE_WFMT_MXFP8  elements FP8 E4M3 (bias 7, subnormals, max 448, S.1111.111 NaN), 1 byte
 *   MOE_WFMT_MXFP4  elements FP4 E2M1 (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), 2 per byte,
 *                   element 2i in the low nibble of byte i */
/*   MOE_WFMT_MXFP8_BS, MOE_WFMT_MXFP4_BS  the same MXFP8 / MXFP4 weights read by the
 *                   block-scaled tensor-core MMA (tcgen05 kind::mxf8f6f4): the token rows and h
 *                   are quantised to MXFP8 (E4M3 elements, per 32 along K one E8M0 scale
 *                   X = 2^(floor(log2 amax) - 8), nearest-even rounding, saturation at 448, as
 *                   the OCP MX v1.0 conversion reads). MXFP4_BS needs d_model and d_ff to be
 *                   multiples of 128. See moe_mx_act_workspace_bytes. */
typedef enum {
  MOE_WFMT_BF16 = 0,
  MOE_WFMT_MXFP8 = 1,
  MOE_WFMT_MXFP4 = 2,
  MOE_WFMT_MXFP8_BS = 3,
  MOE_WFMT_MXFP4_BS = 4
} moe_wfmt;

/* Shape of one layer invocation. */
typedef struct {
  int32_t T;          /* tokens in the batch, >= 0 */
  int32_t d_model;    /* hidden size d, multiple of 64 */
  int32_t n_experts;  /* N, 1..256 */
  int32_t top_k;      /* k, 1..min(8, N) */
  int32_t d_ff;       /* expert FFN width F, multiple of 64 */
  int32_t act;        /* moe_act: SwiGLU (gate/up/down) or GELU (up/down) */
  int32_t capacity;   /* slots per expert, >= 0; a value >= T means no limit */
} moe_dims;

/* Slots per expert: ceil(capacity_factor * T / n_experts), computed as
 * ceil((capacity_factor * T) / n_experts) in IEEE double.
 * capacity_factor <= 0, NaN or infinite means no limit and returns T.
 * Source: page «Sparse Mixture-of-Experts», section «Expert capacity и capacity factor».
 * Returns -1 if T < 0 or n_experts < 1. Host-only; touches no device. */
int32_t moe_capacity(double capacity_factor, int32_t T, int32_t n_experts);

/* Upper bound on kept rows: R_max = min(T * k, N * min(capacity, T)).
 * Row buffers (pair_of_row, x_perm, h, y_perm) must hold R_max rows. Returns -1 on bad dims. Host-only. */
int64_t moe_max_rows(const moe_dims* dims);

/* Bytes of the per-stage workspace `ws` taken by moe_route, moe_route_from_logits,
 * moe_permute, moe_grouped_ffn and moe_unpermute_combine. Host-only. Its regions:
 *   - the device status word (first 256 bytes);
 *   - the grouped FFN's per-tile arrival counters for its stream-K schedule. They must be
 *     zero between calls (each call leaves them zero);
 *   - one region shared by the stages, which run one after another on the stream:
 *       - the capacity scan's chunk totals;
 *       - the router's bf16 three-term split of W_r, on the tensor-core path;
 *       - the grouped FFN's stream-K partial tiles (two per CTA);
 *       - moe_router_stats's partial sums;
 *       - moe_redirect_overflow's per-token lists of next experts.
 * Zero a workspace once before its first use, with moe_workspace_init or any memset to 0.
 * Zero it again after a device error. */
moe_status moe_workspace_bytes(const moe_dims* dims, size_t* bytes);

/* Zero a workspace (an async memset of ws_bytes on `stream`). */
moe_status moe_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Route: steps 1-3 above. Decode-sized batches (1 <= T <= 16, with ceil(d_model / 128) * T * N
 * fp32 partial sums of at most 1 MiB) route in one launch: CTA c takes d columns
 * [128 c, 128 c + 128) of every dot product; the last CTA to finish adds the partials in
 * order of c, then takes top-k and the slots. Larger batches run the router, then the slot
 * pass(es). The results follow the same rules either way; the logits' rounding follows the
 * path's summation order.
 *   x            [T, d_model] bf16            hidden states
 *   w_router     [N, d_model] fp32            router weight (linear, no bias term)
 *   logit_bias   [N] fp32 or NULL             optional additive per-expert logit bias
 *   logits       [T, N] fp32 (out)            x W_r^T (+ b), fp32 accumulation
 *   topk_idx     [T, k] int32 (out)           chosen experts, best first; equal logits go
 *                                             to the lower expert index
 *   topk_w       [T, k] fp32 (out)            renormalised weights, sum to 1 per token:
 *                                             exp(L_j - L_0) / sum_i exp(L_i - L_0)
 *   slot         [T, k] int32 (out)           slot of each pair in its expert's buffer, -1 = dropped
 *   expert_count [N] int32 (out)              kept pairs per expert = min(picks, capacity)
 *   ws, ws_bytes                              per-stage workspace (moe_workspace_bytes)
 */
moe_status moe_route(const moe_dims* dims, const uint16_t* x, const float* w_router,
                     const float* logit_bias, float* logits, int32_t* topk_idx, float* topk_w,
                     int32_t* slot, int32_t* expert_count, void* ws, size_t ws_bytes, void* stream);

/* Route from given logits [T, N] fp32 (steps 2-3 only). Same outputs as moe_route.
 * Lets a caller supply crafted logits (exact ties) or re-route stored logits. */
moe_status moe_route_from_logits(const moe_dims* dims, const float* logits, int32_t* topk_idx,
                                 float* topk_w, int32_t* slot, int32_t* expert_count, void* ws,
                                 size_t ws_bytes, void* stream);

/* moe_route_with_stats: moe_route that also emits the router statistics of moe_router_stats
 * from the routing launches themselves (page «Sparse Mixture-of-Experts», section «Маршрутизация
 * токена и auxiliary loss»): the router writes per-tile sums of its softmax probabilities while
 * the logits are still on chip, and the capacity pass, which counts each expert's picks, adds
 * them in a fixed order. Decode-sized batches form the statistics in the one routing launch.
 * Inputs and routing outputs are those of moe_route; the statistics are those of
 * moe_router_stats:
 *   picks      [N] int32    (token, choice) pairs that chose expert e, before the capacity
 *   prob_mean  [N] fp32     P_e, the batch mean of the router's softmax probability of e
 *   aux_loss   [1] fp32     alpha * N * sum_e (picks_e / T) * P_e (alpha = 1e-2 on the page)
 *   dropped    [1] int32    pairs over the capacity
 * The sums are deterministic; their order differs from moe_router_stats', so the fp32 results
 * may differ from it in the last bits. Uses the per-stage workspace (moe_workspace_bytes). */
moe_status moe_route_with_stats(const moe_dims* dims, const uint16_t* x, const float* w_router,
                                const float* logit_bias, float* logits, int32_t* topk_idx,
                                float* topk_w, int32_t* slot, int32_t* expert_count, float alpha,
                                int32_t* picks, float* prob_mean, float* aux_loss,
                                int32_t* dropped, void* ws, size_t ws_bytes, void* stream);

/* Overflow policy "redirect": a pair that arrives at a full expert goes to the next most
 * suitable expert instead of being dropped (page «Архитектура MoE в больших языковых моделях —
 * кто такие «эксперты»?», section «Как работает MoE: принцип маршрутизации», which names
 * dropping and redirecting as the two ways to handle an expert over capacity).
 * Call after moe_route or moe_route_from_logits; it replaces their drop-policy slots. Pairs
 * arrive in the same (choice, token) order. A pair whose expert is full goes to the token's
 * expert with the largest logit (equal logits: lower index; NaN counts as -inf) that has a
 * free slot and that the token does not already use (another of its top-k choices or an
 * earlier redirect); with none, it is dropped (slot -1, topk_idx unchanged). A redirected
 * pair keeps its router weight topk_w.
 *   logits       [T, N] fp32            the router logits (from moe_route)
 *   topk_idx     [T, k] int32 (in/out)  the router's choices in; the expert serving each pair out
 *   slot         [T, k] int32 (out)     slot in the serving expert's buffer, -1 = dropped
 *   expert_count [N] int32 (out)        kept pairs per expert, <= capacity
 * topk_idx must be the top-k of these logits as moe_route writes them: a list of each token's
 * next 16 experts after its top-k (written into the workspace by a first launch over all SMs)
 * stands in for a scan of its logits, which only runs when all 16 fail. The decisions depend
 * on each other in arrival order, so one warp then takes them in sequence (second launch);
 * it stops once no expert has a free slot, and every later pair stays dropped.
 * An expert id in topk_idx outside [0, N) is reported as MOE_ERR_BOUNDS in the workspace's
 * status word; such a pair holds no expert and may be redirected like an overflowing one.
 * MOE_ERR_UNSUPPORTED when T * k > 163840 (every pair's serving expert is held as a byte in
 * shared memory). Uses the per-stage workspace: T * 16 bytes of lists, T * k bytes of experts
 * and T * k / 8 bytes of flags. */
moe_status moe_redirect_overflow(const moe_dims* dims, const float* logits, int32_t* topk_idx,
                                 int32_t* slot, int32_t* expert_count, void* ws, size_t ws_bytes,
                                 void* stream);

/* Permute: step 4, sort by expert id.
 *   expert_offset [N+1] int32 (out)  exclusive prefix sum of expert_count; expert e owns rows
 *                                    [expert_offset[e], expert_offset[e+1]); R = expert_offset[N]
 *   row_of_pair   [T, k] int32 (out) row of pair (t, j) = expert_offset[e] + slot, -1 if dropped
 *   pair_of_row   [R_max] int32 (out) t * k + j for rows < R; rows >= R are not written
 *   x_perm        [R_max, d_model] bf16 (out) x_perm[row_of_pair[t, j]] = x[t]; rows >= R not written
 */
moe_status moe_permute(const moe_dims* dims, const uint16_t* x, const int32_t* topk_idx,
                       const int32_t* slot, const int32_t* expert_count, int32_t* expert_offset,
                       int32_t* row_of_pair, int32_t* pair_of_row, uint16_t* x_perm, void* ws,
                       size_t ws_bytes, void* stream);

/* Grouped expert FFN over the expert-contiguous rows (step 4), on tcgen05 tensor cores.
 *   w_gate_up  SwiGLU: [N, 2F, d_model] bf16, rows 0..F-1 of expert e are the gate projection
 *              and rows F..2F-1 the up projection (the packed gate_up_proj layout);
 *              GELU:   [N, F, d_model] bf16
 *   w_down     [N, d_model, F] bf16 (the packed down_proj layout)
 *   h          [R_max, F] bf16 (out)   act(x_perm W_gu^T) in fp32, rounded once to bf16
 *   y_perm     [R_max, d_model] fp32 (out)  h W_d^T with fp32 accumulation
 * Rows >= R of h and y_perm are not written. Experts with no kept rows cost nothing.
 * When the tiles do not fill the SMs evenly (decode-sized and mid-sized batches), a GEMM runs
 * stream-K: its tiles' K blocks, end to end, are cut into one equal range per CTA. A tile
 * cut by a range boundary gets fp32 partial tiles in the workspace, and the last CTA to finish
 * it adds them in order of CTA index, so results are deterministic for a given device.
 * ws_bytes must be at least moe_workspace_bytes(). */
moe_status moe_grouped_ffn(const moe_dims* dims, const uint16_t* x_perm,
                           const int32_t* expert_offset, const uint16_t* w_gate_up,
                           const uint16_t* w_down, uint16_t* h, float* y_perm, void* ws,
                           size_t ws_bytes, void* stream);

/* Combine: step 5, back to token order.
 *   out[t] = residual[t] + sum over kept j (ascending) of topk_w[t, j] * y_perm[row_of_pair[t, j]]
 * summed in fp32 and rounded once. A token with no kept pair gets residual[t]'s bits
 * unchanged (zeros if residual is NULL). out_f32 = 0: out is [T, d_model] bf16;
 * out_f32 = 1: out is [T, d_model] fp32. `out` may alias `residual` (same dtype).
 * ws may be NULL; if given, bounds faults are recorded in its status word. */
moe_status moe_unpermute_combine(const moe_dims* dims, const float* y_perm,
                                 const int32_t* row_of_pair, const float* topk_w,
                                 const uint16_t* residual, void* out, int32_t out_f32, void* ws,
                                 size_t ws_bytes, void* stream);

/* Router statistics and the auxiliary load-balancing loss (page «Sparse Mixture-of-Experts»,
 * section «Маршрутизация токена и auxiliary loss»; the loss is alpha * N * sum_i f_i * P_i).
 *   logits    [T, N] fp32            the router logits (from moe_route)
 *   topk_idx  [T, k] int32, slot [T, k] int32   the routing (from moe_route)
 *   alpha                             loss coefficient (the page reports 1e-2 as best)
 *   picks     [N] int32 (out)         pairs that chose expert e, before the capacity limit
 *   prob_mean [N] fp32 (out)          P_e: the mean over the batch of softmax(logits)_e
 *   aux_loss  [1] fp32 (out)          alpha * N * sum_e (picks_e / T) * P_e; f_e counts a token
 *                                     once for each of its chosen experts (sum_e f_e = k)
 *   dropped   [1] int32 (out)         pairs with slot -1
 * Deterministic: partial sums are added in a fixed order. Uses the per-stage workspace. */
moe_status moe_router_stats(const moe_dims* dims, const float* logits, const int32_t* topk_idx,
                            const int32_t* slot, float alpha, int32_t* picks, float* prob_mean,
                            float* aux_loss, int32_t* dropped, void* ws, size_t ws_bytes,
                            void* stream);

/* Pointers into a moe_forward workspace (all device pointers; sizes as in the calls above). */
typedef struct {
  float* logits;
  int32_t* topk_idx;
  float* topk_w;
  int32_t* slot;
  int32_t* expert_count;
  int32_t* expert_offset;
  int32_t* row_of_pair;
  int32_t* pair_of_row;
  uint16_t* x_perm;
  uint16_t* h;
  float* y_perm;
  void* stage_ws;
  size_t stage_ws_bytes;
} moe_forward_buffers;

/* Bytes of workspace moe_forward needs: every intermediate plus the per-stage workspace. */
moe_status moe_forward_workspace_bytes(const moe_dims* dims, size_t* bytes);

/* Carve a moe_forward workspace into its intermediates (host arithmetic only). */
moe_status moe_forward_layout(const moe_dims* dims, void* ws, size_t ws_bytes,
                              moe_forward_buffers* bufs);

/* The whole layer on one stream: route, permute, grouped FFN, combine.
 *   out [T, d_model] bf16 (out). `residual` may be NULL (out = MoE part only) and may alias x;
 *   out may alias residual. Intermediates stay in `ws` (see moe_forward_layout). */
moe_status moe_forward(const moe_dims* dims, const uint16_t* x, const float* w_router,
                       const float* logit_bias, const uint16_t* w_gate_up, const uint16_t* w_down,
                       const uint16_t* residual, uint16_t* out, void* ws, size_t ws_bytes,
                       void* stream);

/* Backward pass of the layer (bf16 expert weights), after moe_forward on the same inputs.
 * The pages discuss training MoE layers (page «Что такое Mixture of Experts (MoE) в
 * трансформерах», section «Обучение MoE с помощью Transformers») without formulas; this is
 * the chain rule of the forward pass. The choice of experts and the capacity slots pass no
 * gradient; a dropped pair's weight gets none, but it still takes part in the softmax over
 * the chosen logits.
 *   x, w_router, w_gate_up, w_down   the forward's inputs (residual excluded)
 *   fwd_ws, fwd_ws_bytes   the moe_forward workspace holding that forward's intermediates
 *                          (routing, x_perm, y_perm; see moe_forward_layout), read only
 *   d_out        [T, d_model] bf16      gradient of the layer output
 *   d_x          [T, d_model] fp32 (out) gradient through the router and the experts; the
 *                                       residual's own gradient is d_out and is not added
 *   d_w_router   [N, d_model] fp32 (out)  dL^T x, dL the logits' gradient
 *   d_logit_bias [N] fp32 (out) or NULL   sum over tokens of dL
 *   d_w_gate_up  [N, 2F, d_model] (SwiGLU) or [N, F, d_model] (GELU) fp32 (out)
 *   d_w_down     [N, d_model, d_ff] fp32 (out); experts with no kept rows get zeros
 *   ws, ws_bytes  backward workspace (moe_backward_workspace_bytes), no zeroing needed
 * Precision: the expert GEMMs take bf16 operands (d_out * w and the activation's gradient
 * are rounded once to bf16) with fp32 accumulation on tensor cores; the router's gradients
 * are fp32 throughout. Deterministic for a given device. The status word of the backward
 * workspace (its first int32) records MOE_ERR_TIMEOUT or MOE_ERR_BOUNDS like the forward's;
 * read it with moe_read_device_error(ws). */
moe_status moe_backward_workspace_bytes(const moe_dims* dims, size_t* bytes);
moe_status moe_backward(const moe_dims* dims, const uint16_t* x, const float* w_router,
                        const uint16_t* w_gate_up, const uint16_t* w_down, const void* fwd_ws,
                        size_t fwd_ws_bytes, const uint16_t* d_out, float* d_x, float* d_w_router,
                        float* d_logit_bias, float* d_w_gate_up, float* d_w_down, void* ws,
                        size_t ws_bytes, void* stream);

/* Expert weights in an MX format (device pointers, 16-byte aligned):
 *   fmt             MOE_WFMT_MXFP8 or MOE_WFMT_MXFP4
 *   gate_up         elements of the packed gate_up rows, [N, 2F, d_model] (SwiGLU: gate rows
 *                   then up rows) or [N, F, d_model] (GELU): d_model bytes a row (MXFP8) or
 *                   d_model / 2 (MXFP4)
 *   gate_up_scales  [N, d_model / 32, 2F (or F)] uint8 E8M0: block b of row r at [e][b][r]
 *   down            elements of [N, d_model, d_ff]: d_ff (MXFP8) or d_ff / 2 (MXFP4) bytes a row
 *   down_scales     [N, d_ff / 32, d_model] uint8 E8M0
 * The scale axis order (K blocks outer, rows inner) lets one TMA box carry a tile's scales. */
typedef struct {
  int32_t fmt;
  const void* gate_up;
  const uint8_t* gate_up_scales;
  const void* down;
  const uint8_t* down_scales;
} moe_mx_weights;

/* moe_grouped_ffn with MX weights. The weights stream from HBM in their packed form (1/2 or
 * 1/4 of the bf16 bytes) and are decoded in shared memory, exactly, into bf16 (a power-of-two
 * scale times an FP8/FP4 value is a bf16 value while it stays in bf16's normal range); the
 * tensor-core arithmetic, h, y_perm and their rounding rules are those of moe_grouped_ffn on
 * the decoded weights. Same workspace. MOE_ERR_INVALID for a bad fmt or a NULL pointer. */
moe_status moe_grouped_ffn_mx(const moe_dims* dims, const uint16_t* x_perm,
                              const int32_t* expert_offset, const moe_mx_weights* w, uint16_t* h,
                              float* y_perm, void* ws, size_t ws_bytes, void* stream);

/* Extra workspace of the block-scaled formats (MOE_WFMT_MXFP8_BS, MOE_WFMT_MXFP4_BS): the
 * quantised token rows ([R_max, d_model] E4M3 codes) and the E8M0 scales of the rows and of h
 * in the tensor-memory copy layout. moe_grouped_ffn_mx then needs ws_bytes >=
 * round_up(moe_workspace_bytes, 256) + this, moe_forward_mx a forward workspace of
 * round_up(moe_forward_workspace_bytes, 256) + this; the extra bytes follow the usual regions.
 * With these formats h (the buffer passed in, or the forward layout's) receives h's E4M3 codes,
 * [R_max, d_ff] bytes. Host-only. */
moe_status moe_mx_act_workspace_bytes(const moe_dims* dims, size_t* bytes);

/* moe_forward with MX expert weights (same workspace, layout and routing). */
moe_status moe_forward_mx(const moe_dims* dims, const uint16_t* x, const float* w_router,
                          const float* logit_bias, const moe_mx_weights* w,
                          const uint16_t* residual, uint16_t* out, void* ws, size_t ws_bytes,
                          void* stream);

/* Size of the scratch array built into the library for moe_route_noalloc. */
#define MOE_ROUTE_NOALLOC_SCRATCH_BYTES 65536

/* moe_route_noalloc: moe_route without a caller-provided workspace. The pages have no
 * counterpart to this call; it exists for callers that cannot allocate device memory.
 * Examples: an engine that hands out all device memory from its own arena up front; code on
 * a real-time path where an allocation could synchronise the device or fail mid-run; a plugin
 * whose host framework owns every allocation.
 *
 * Inputs, outputs, results and validation are those of moe_route. The capacity scan's scratch
 * comes from a static array of MOE_ROUTE_NOALLOC_SCRATCH_BYTES in the library's own device
 * memory. Every GPU that loads the library holds that array until the process exits.
 *   - Limit: when T * k spans more than one capacity chunk (4096 pairs), the scan needs
 *     ceil(T * k / 4096) * N int32 of scratch. A shape that needs more than the array holds
 *     is rejected with MOE_ERR_WORKSPACE before anything is launched. With N = 256 the limit
 *     is T * k <= 262144 pairs (64 chunks).
 *   - The call allocates nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 *   - The first call on each device looks up the array's device address (cudaGetSymbolAddress,
 *     with that device current) and caches it. Make that first call before any stream capture.
 *   - Decode-sized batches (the one-launch routing of moe_route, below) take their partial
 *     dot products from a second static array of 1 MiB and their arrival counter from a
 *     third; the counter is zero when the library loads and every call leaves it zero.
 *   - All calls share the arrays, and they keep the last call's contents. Each call writes
 *     every scratch entry before reading it, so nothing has to start at zero. Calls that
 *     overlap on the GPU (on concurrent streams) race on the arrays and must be serialised
 *     by the caller.
 *   - Device-side faults are not reported. moe_route keeps its status word in the caller's
 *     workspace; this call has none. Its kernels bound their waits as moe_route's do. A wait
 *     that runs out (which only a limit far below the default 2 s makes happen, see
 *     moe_debug_set_wait_timeout_ns) stops the kernel early: the outputs of that call are
 *     then undefined and the call has still returned MOE_OK. Expert ids outside [0, N) that
 *     such a call may leave behind are never given a slot. The next call is unaffected. */
moe_status moe_route_noalloc(const moe_dims* dims, const uint16_t* x, const float* w_router,
                             const float* logit_bias, float* logits, int32_t* topk_idx,
                             float* topk_w, int32_t* slot, int32_t* expert_count, void* stream);

/* Synchronise `stream`, read the status word of a per-stage workspace into *err and clear it.
 * (For a moe_forward workspace pass moe_forward_buffers.stage_ws.) */
moe_status moe_read_device_error(void* ws, void* stream, moe_status* err);

/* Diagnostics: set the limit, in nanoseconds, of every bounded wait inside the library's
 * tensor-core kernels, for calls made afterwards in this process; 0 restores the default of
 * 2 s. Returns the previous limit. A limit too short for the work makes the kernels stop
 * early and record MOE_ERR_TIMEOUT in the workspace status word. Their outputs are then
 * undefined, and the workspace must be zeroed again (moe_workspace_init). Copies and MMAs
 * already in flight are still waited for, under a separate 1 s limit, before a CTA exits.
 * Meant for testing the error path. */
uint64_t moe_debug_set_wait_timeout_ns(uint64_t ns);

/* Static description of a status code. */
const char* moe_status_string(moe_status s);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H_ */
