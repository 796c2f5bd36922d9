// C ABI of the MoE layer forward pass: host-side validation, workspace layout and the
// launch sequence of each stage. The meaning of every call is documented in include/moe.h.
#include <math.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "launch.h"
#include "common.cuh"

namespace moe {

std::atomic<uint64_t> g_wait_timeout_ns{kDefaultWaitTimeoutNs};

namespace {
constexpr int kMaxDevices = 64;
DeviceInfo g_info[kMaxDevices];
std::once_flag g_info_once[kMaxDevices];
cudaError_t g_info_err[kMaxDevices];


}  // namespace

uint64_t wait_timeout_ns() { return g_wait_timeout_ns.load(std::memory_order_relaxed); }

cudaError_t device_info(DeviceInfo* out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::call_once(g_info_once[dev], [dev] {
    DeviceInfo di{};
    cudaError_t e = cudaDeviceGetAttribute(&di.sm_count, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&di.cc_major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&di.cc_minor, cudaDevAttrComputeCapabilityMinor, dev);
    g_info[dev] = di;
    g_info_err[dev] = e;
  });
  *out = g_info[dev];
  return g_info_err[dev];
}

}  // namespace moe

using moe::DeviceInfo;

namespace {

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

moe_status check_dims(const moe_dims* d) {
  if (d == nullptr) return MOE_ERR_INVALID;
  if (d->T < 0 || d->d_model <= 0 || d->n_experts <= 0 || d->top_k <= 0 || d->d_ff <= 0 ||
      d->capacity < 0)
    return MOE_ERR_INVALID;
  if (d->top_k > d->n_experts) return MOE_ERR_INVALID;
  if (d->act != MOE_ACT_SWIGLU && d->act != MOE_ACT_GELU) return MOE_ERR_INVALID;
  if (d->n_experts > 256 || d->top_k > 8) return MOE_ERR_UNSUPPORTED;
  if (d->d_model % 64 != 0 || d->d_ff % 64 != 0) return MOE_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(d->T) * d->top_k > INT32_MAX) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status check_device() {
  DeviceInfo di;
  if (moe::device_info(&di) != cudaSuccess) return MOE_ERR_CUDA;
  if (di.cc_major != 10 || di.cc_minor != 0) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

int64_t max_rows(const moe_dims* d) {
  const int64_t cap = std::min<int64_t>(d->capacity, d->T);
  return std::min<int64_t>(static_cast<int64_t>(d->T) * d->top_k,
                           static_cast<int64_t>(d->n_experts) * cap);
}

// Per-stage workspace: [status word, 256 B][capacity-scan chunk totals][router weight split].
size_t slot_scratch_bytes(const moe_dims* d) {
  const int64_t chunks = moe::slot_chunks(static_cast<int64_t>(d->T) * d->top_k);
  return chunks > 1 ? round_up(static_cast<size_t>(chunks) * d->n_experts * sizeof(int32_t), 256) : 0;
}

size_t split_scratch_bytes(const moe_dims* d) {
  return moe::router_uses_tensor_cores(d->T, d->n_experts, d->d_model)
             ? round_up(moe::router_split_bytes(d->n_experts, d->d_model), 256)
             : 0;
}

// Partial dot products of the one-launch router of decode-sized batches.
size_t decode_scratch_bytes(const moe_dims* d) {
  return moe::use_decode_route(d->T, d->n_experts, d->d_model)
             ? round_up(moe::decode_route_scratch_bytes(d->T, d->n_experts, d->d_model), 256)
             : 0;
}

moe::FfnScratchPlan ffn_plan(const moe_dims* d) {
  return moe::ffn_scratch_plan(d->n_experts, d->d_model, d->d_ff, d->act, max_rows(d),
                               std::min(d->capacity, d->T));
}

// Per-stage workspace:
//   [status word, 256 B][grouped-FFN counters, zero between calls]
//   [shared region: routing scratch (capacity-scan chunk totals, router weight split, the
//    decode router's partial dot products) or,
//    later on the stream, the grouped FFN's stream-K partial tiles]
size_t counters_bytes(const moe_dims* d) { return round_up(ffn_plan(d).counter_bytes, 256); }

// Router statistics emitted by the routing launches: the router's per-tile probability sums,
// after the routing scratch (both are live during the same call).
size_t route_stats_bytes(const moe_dims* d) {
  if (d->T == 0 || moe::use_decode_route(d->T, d->n_experts, d->d_model)) return 0;
  return round_up(static_cast<size_t>(moe::route_stats_parts(d->T, d->n_experts, d->d_model)) *
                      d->n_experts * sizeof(float),
                  256);
}

size_t shared_region_bytes(const moe_dims* d) {
  const size_t routing = slot_scratch_bytes(d) + split_scratch_bytes(d) + decode_scratch_bytes(d) +
                         route_stats_bytes(d);
  const size_t ffn = round_up(ffn_plan(d).part_bytes, 256);
  const size_t stats = round_up(moe::router_stats_scratch_bytes(d->T, d->n_experts), 256);
  const size_t redirect = round_up(moe::redirect_scratch_bytes(d->T, d->top_k), 256);
  return std::max(std::max(std::max(routing, ffn), stats), redirect);
}

size_t stage_ws_bytes(const moe_dims* d) {
  return moe::kStatusBytes + counters_bytes(d) + shared_region_bytes(d);
}

char* shared_region_of(const moe_dims* d, void* ws) {
  return static_cast<char*>(ws) + moe::kStatusBytes + counters_bytes(d);
}

uint16_t* split_scratch_of(const moe_dims* d, void* ws) {
  if (split_scratch_bytes(d) == 0) return nullptr;
  return reinterpret_cast<uint16_t*>(shared_region_of(d, ws) + slot_scratch_bytes(d));
}

int* status_of(void* ws) { return static_cast<int*>(ws); }

// One-launch routing of a decode-sized batch (moe::use_decode_route); the four permute
// outputs are null unless the same launch also sorts by expert.
moe::DecodeRouteArgs decode_route_args(const moe_dims* d, const uint16_t* x, const float* w_router,
                                       const float* bias, float* logits, int32_t* topk_idx,
                                       float* topk_w, int32_t* slot, int32_t* expert_count,
                                       void* ws) {
  moe::DecodeRouteArgs a{};
  a.x = x;
  a.w_router = w_router;
  a.bias = bias;
  a.logits = logits;
  a.topk_idx = topk_idx;
  a.topk_w = topk_w;
  a.slot = slot;
  a.expert_count = expert_count;
  a.part = reinterpret_cast<float*>(shared_region_of(d, ws) + slot_scratch_bytes(d) +
                                    split_scratch_bytes(d));
  a.counter = reinterpret_cast<int*>(static_cast<char*>(ws) + moe::kDecodeCounterOffset);
  a.T = d->T;
  a.d = d->d_model;
  a.N = d->n_experts;
  a.k = d->top_k;
  a.cap = std::min(d->capacity, d->T);
  return a;
}

// A grid that cannot be resident at once (the kernels whose CTAs wait on one another check
// this before launching) is an unsupported configuration; any other launch error is a CUDA one.
moe_status launch_status(cudaError_t e) {
  if (e == cudaSuccess) return MOE_OK;
  return e == cudaErrorInvalidConfiguration ? MOE_ERR_UNSUPPORTED : MOE_ERR_CUDA;
}

// Shared by moe_route and moe_route_from_logits once top-k is written.
moe_status route_slots(const moe_dims* d, int32_t* topk_idx, int32_t* slot, int32_t* expert_count,
                       void* ws, cudaStream_t s) {
  int32_t* scratch = reinterpret_cast<int32_t*>(shared_region_of(d, ws));
  const int cap = std::min(d->capacity, d->T);
  return launch_status(moe::launch_capacity_slots(topk_idx, slot, expert_count, scratch, d->T,
                                                  d->n_experts, d->top_k, cap, s));
}

}  // namespace

extern "C" {

int32_t moe_capacity(double capacity_factor, int32_t T, int32_t n_experts) {
  if (T < 0 || n_experts < 1) return -1;
  if (!(capacity_factor > 0.0) || isinf(capacity_factor)) return T;  // <= 0, NaN, inf: no limit
  const double c = ceil((capacity_factor * static_cast<double>(T)) / static_cast<double>(n_experts));
  return c >= static_cast<double>(INT32_MAX) ? INT32_MAX : static_cast<int32_t>(c);
}

int64_t moe_max_rows(const moe_dims* dims) {
  if (check_dims(dims) != MOE_OK) return -1;
  return max_rows(dims);
}

moe_status moe_workspace_bytes(const moe_dims* dims, size_t* bytes) {
  const moe_status st = check_dims(dims);
  if (st != MOE_OK) return st;
  if (bytes == nullptr) return MOE_ERR_INVALID;
  *bytes = stage_ws_bytes(dims);
  return MOE_OK;
}

moe_status moe_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (ws == nullptr || ws_bytes < moe::kStatusBytes) return MOE_ERR_INVALID;
  return launch_status(cudaMemsetAsync(ws, 0, ws_bytes, as_stream(stream)));
}

moe_status moe_route(const moe_dims* dims, const uint16_t* x, const float* w_router,
                     const float* logit_bias, float* logits, int32_t* topk_idx, float* topk_w,
                     int32_t* slot, int32_t* expert_count, void* ws, size_t ws_bytes,
                     void* stream) {
  moe_status st = check_dims(dims);
  if (st != MOE_OK) return st;
  if (dims->T == 0) return MOE_OK;
  if (!x || !w_router || !logits || !topk_idx || !topk_w || !slot || !expert_count || !ws)
    return MOE_ERR_INVALID;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(logits) || !aligned16(topk_idx) ||
      !aligned16(topk_w) || !aligned16(slot) || !aligned16(expert_count) || !aligned16(ws) ||
      (logit_bias && !aligned16(logit_bias)))
    return MOE_ERR_UNSUPPORTED;
  if (ws_bytes < stage_ws_bytes(dims)) return MOE_ERR_WORKSPACE;
  if ((st = check_device()) != MOE_OK) return st;
  const cudaStream_t s = as_stream(stream);
  if (moe::use_decode_route(dims->T, dims->n_experts, dims->d_model))
    return launch_status(moe::launch_decode_route(
        decode_route_args(dims, x, w_router, logit_bias, logits, topk_idx, topk_w, slot,
                          expert_count, ws),
        s));
  st = launch_status(moe::launch_router_topk(x, w_router, logit_bias, logits, topk_idx, topk_w,
                                             dims->T, dims->d_model, dims->n_experts,
                                             dims->top_k, split_scratch_of(dims, ws), status_of(ws),
                                             moe::wait_timeout_ns(), s));
  if (st != MOE_OK) return st;
  return route_slots(dims, topk_idx, slot, expert_count, ws, s);
}

moe_status moe_route_with_stats(const moe_dims* dims, const uint16_t* x, const float* w_router,
                                const float* logit_bias, float* logits, int32_t* topk_idx,
                                float* topk_w, int32_t* slot, int32_t* expert_count, float alpha,
                                int32_t* picks, float* prob_mean, float* aux_loss,
                                int32_t* dropped, void* ws, size_t ws_bytes, void* stream) {
  moe_status st = check_dims(dims);
  if (st != MOE_OK) return st;
  if (dims->T == 0) return MOE_OK;
  if (!x || !w_router || !logits || !topk_idx || !topk_w || !slot || !expert_count || !ws ||
      !picks || !prob_mean || !aux_loss || !dropped)
    return MOE_ERR_INVALID;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(logits) || !aligned16(topk_idx) ||
      !aligned16(topk_w) || !aligned16(slot) || !aligned16(expert_count) || !aligned16(ws) ||
      !aligned16(picks) || !aligned16(prob_mean) || (logit_bias && !aligned16(logit_bias)))
    return MOE_ERR_UNSUPPORTED;
  if (ws_bytes < stage_ws_bytes(dims)) return MOE_ERR_WORKSPACE;
  if ((st = check_device()) != MOE_OK) return st;
  const cudaStream_t s = as_stream(stream);
  if (moe::use_decode_route(dims->T, dims->n_experts, dims->d_model)) {
    moe::DecodeRouteArgs a = decode_route_args(dims, x, w_router, logit_bias, logits, topk_idx,
                                               topk_w, slot, expert_count, ws);
    a.st_picks = picks;
    a.st_prob_mean = prob_mean;
    a.st_aux_loss = aux_loss;
    a.st_dropped = dropped;
    a.st_alpha = alpha;
    return launch_status(moe::launch_decode_route(a, s));
  }
  moe::RouteStats rs{};
  rs.prob_part = reinterpret_cast<float*>(shared_region_of(dims, ws) + slot_scratch_bytes(dims) +
                                          split_scratch_bytes(dims) + decode_scratch_bytes(dims));
  rs.n_parts = moe::route_stats_parts(dims->T, dims->n_experts, dims->d_model);
  rs.alpha = alpha;
  rs.picks = picks;
  rs.prob_mean = prob_mean;
  rs.aux_loss = aux_loss;
  rs.dropped = dropped;
  st = launch_status(moe::launch_router_topk(x, w_router, logit_bias, logits, topk_idx, topk_w,
                                             dims->T, dims->d_model, dims->n_experts,
                                             dims->top_k, split_scratch_of(dims, ws), status_of(ws),
                                             moe::wait_timeout_ns(), s, rs.prob_part));
  if (st != MOE_OK) return st;
  int32_t* scratch = reinterpret_cast<int32_t*>(shared_region_of(dims, ws));
  return launch_status(moe::launch_capacity_slots(topk_idx, slot, expert_count, scratch, dims->T,
                                                  dims->n_experts, dims->top_k,
                                                  std::min(dims->capacity, dims->T), s, &rs));
}

moe_status moe_route_from_logits(const moe_dims* dims, const float* logits, int32_t* topk_idx,
                                 float* topk_w, int32_t* slot, int32_t* expert_count, void* ws,
                                 size_t ws_bytes, void* stream) {
  moe_status st = check_dims(dims);
  if (st != MOE_OK) return st;
  if (dims->T == 0) return MOE_OK;
  if (!logits || !topk_idx || !topk_w || !slot || !expert_count || !ws) return MOE_ERR_INVALID;
  if (!aligned16(logits) || !aligned16(topk_idx) || !aligned16(topk_w) || !aligned16(slot) ||
      !aligned16(expert_count) || !aligned16(ws))
    return MOE_ERR_UNSUPPORTED;
  if (ws_bytes < stage_ws_bytes(dims)) return MOE_ERR_WORKSPACE;
  if ((st = check_device()) != MOE_OK) return st;
  const cudaStream_t s = as_stream(stream);
  st = launch_status(moe::launch_topk_from_logits(logits, topk_idx, topk_w, dims->T,
                                                  dims->n_experts, dims->top_k, s));
  if (st != MOE_OK) return st;
  return route_slots(dims, topk_idx, slot, expert_count, ws, s);
}

moe_status moe_redirect_overflow(const moe_dims* dims, const float* logits, int32_t* topk_idx,
                                 int32_t* slot, int32_t* expert_count, void* ws, size_t ws_bytes,
                                 void* stream) {
  moe_status st = check_dims(dims);
  if (st != MOE_OK) return st;
  if (dims->T == 0) return MOE_OK;
  if (!logits || !topk_idx || !slot || !expert_count || !ws) return MOE_ERR_INVALID;
  if (static_cast<int64_t>(dims->T) * dims->top_k > moe::kRerouteMaxPairs)
    return MOE_ERR_UNSUPPORTED;
  if (!aligned16(logits) || !aligned16(topk_idx) || !aligned16(slot) || !aligned16(expert_count) ||
      !aligned16(ws))
    return MOE_ERR_UNSUPPORTED;
  if (ws_bytes < stage_ws_bytes(dims)) return MOE_ERR_WORKSPACE;
  if ((st = check_device()) != MOE_OK) return st;
  uint8_t* scratch = reinterpret_cast<uint8_t*>(shared_region_of(dims, ws));
  return launch_status(moe::launch_reroute_slots(logits, scratch, topk_idx, slot, expert_count,
                                                 dims->T, dims->n_experts, dims->top_k,
                                                 std::min(dims->capacity, dims->T),
                                                 status_of(ws), as_stream(stream)));
}

moe_status moe_permute(const moe_dims* dims, const uint16_t* x, const int32_t* topk_idx,
                       const int32_t* slot, const int32_t* expert_count, int32_t* expert_offset,
                       int32_t* row_of_pair, int32_t* pair_of_row, uint16_t* x_perm, void* ws,
                       size_t ws_bytes, void* stream) {
  moe_status st = check_dims(dims);
  if (st != MOE_OK) return st;
  if (dims->T == 0) return MOE_OK;
  const int64_t rmax = max_rows(dims);
  if (!x || !topk_idx || !slot || !expert_count || !expert_offset || !row_of_pair || !ws ||
      (rmax > 0 && (!pair_of_row || !x_perm)))
    return MOE_ERR_INVALID;
  if (!aligned16(x) || !aligned16(topk_idx) || !aligned16(slot) || !aligned16(expert_count) ||
      !aligned16(expert_offset) || !aligned16(row_of_pair) || !aligned16(ws) ||
      (pair_of_row && !aligned16(pair_of_row)) || (x_perm && !aligned16(x_perm)))
    return MOE_ERR_UNSUPPORTED;
  if (ws_bytes < moe::kStatusBytes) return MOE_ERR_WORKSPACE;
  if ((st = check_device()) != MOE_OK) return st;
  return launch_status(moe::launch_permute(x, topk_idx, slot, expert_count, expert_offset,
                                           row_of_pair, pair_of_row, x_perm, dims->T,
                                           dims->d_model, dims->n_experts, dims->top_k, rmax,
                                           status_of(ws), as_stream(stream)));
}

namespace {
// Expert weights of either storage: bf16 (scales null) or an MX format.
struct Weights {
  int fmt;
  const void* gate_up;
  const uint8_t* gate_up_scales;
  const void* down;
  const uint8_t* down_scales;
};

bool block_scaled(int fmt) { return fmt == MOE_WFMT_MXFP8_BS || fmt == MOE_WFMT_MXFP4_BS; }

moe_status check_weights(const Weights& w) {
  if (w.fmt != MOE_WFMT_BF16 && w.fmt != MOE_WFMT_MXFP8 && w.fmt != MOE_WFMT_MXFP4 &&
      !block_scaled(w.fmt))
    return MOE_ERR_INVALID;
  if (!w.gate_up || !w.down) return MOE_ERR_INVALID;
  if (w.fmt != MOE_WFMT_BF16 && (!w.gate_up_scales || !w.down_scales)) return MOE_ERR_INVALID;
  if (!aligned16(w.gate_up) || !aligned16(w.down) ||
      (w.gate_up_scales && !aligned16(w.gate_up_scales)) ||
      (w.down_scales && !aligned16(w.down_scales)))
    return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

Weights weights_of(const moe_mx_weights* w) {
  return Weights{w->fmt, w->gate_up, w->gate_up_scales, w->down, w->down_scales};
}

// act_ws: the block-scaled formats' activation region (moe_mx_act_workspace_bytes), or null.
moe_status grouped_ffn_impl(const moe_dims* dims, const uint16_t* x_perm,
                            const int32_t* expert_offset, const Weights& w, uint16_t* h,
                            float* y_perm, void* ws, size_t ws_bytes, void* stream,
                            void* act_ws = nullptr) {
  moe_status st = check_dims(dims);
  if (st != MOE_OK) return st;
  const int64_t rmax = max_rows(dims);
  if (dims->T == 0 || rmax == 0) return MOE_OK;
  if ((st = check_weights(w)) != MOE_OK) return st;
  if (block_scaled(w.fmt)) {
    if (act_ws == nullptr || !aligned16(act_ws)) return MOE_ERR_WORKSPACE;
    if (w.fmt == MOE_WFMT_MXFP4_BS && (dims->d_model % 128 != 0 || dims->d_ff % 128 != 0))
      return MOE_ERR_UNSUPPORTED;
  }
  if (!x_perm || !expert_offset || !h || !y_perm || !ws) return MOE_ERR_INVALID;
  if (!aligned16(x_perm) || !aligned16(expert_offset) || !aligned16(h) || !aligned16(y_perm) ||
      !aligned16(ws))
    return MOE_ERR_UNSUPPORTED;
  if (ws_bytes < stage_ws_bytes(dims)) return MOE_ERR_WORKSPACE;
  if ((st = check_device()) != MOE_OK) return st;
  moe::GroupedFfnArgs a{};
  a.x_perm = x_perm;
  a.expert_offset = expert_offset;
  a.wfmt = w.fmt;
  a.w_gate_up = w.gate_up;
  a.w_down = w.down;
  a.w_gate_up_scales = w.gate_up_scales;
  a.w_down_scales = w.down_scales;
  a.h = h;
  a.y_perm = y_perm;
  a.N = dims->n_experts;
  a.d = dims->d_model;
  a.F = dims->d_ff;
  a.act = dims->act;
  a.r_max = rmax;
  a.status = status_of(ws);
  a.timeout_ns = moe::wait_timeout_ns();
  a.rows_per_expert = std::min(dims->capacity, dims->T);
  const moe::FfnScratchPlan plan = ffn_plan(dims);
  a.counters = reinterpret_cast<int*>(static_cast<char*>(ws) + moe::kStatusBytes);
  if (plan.part_bytes > 0) a.part = reinterpret_cast<float*>(shared_region_of(dims, ws));
  a.act_ws = act_ws;
  return launch_status(moe::launch_grouped_ffn(a, as_stream(stream)));
}
}  // namespace

moe_status moe_grouped_ffn(const moe_dims* dims, const uint16_t* x_perm,
                           const int32_t* expert_offset, const uint16_t* w_gate_up,
                           const uint16_t* w_down, uint16_t* h, float* y_perm, void* ws,
                           size_t ws_bytes, void* stream) {
  return grouped_ffn_impl(dims, x_perm, expert_offset,
                          Weights{MOE_WFMT_BF16, w_gate_up, nullptr, w_down, nullptr}, h, y_perm,
                          ws, ws_bytes, stream);
}

moe_status moe_mx_act_workspace_bytes(const moe_dims* dims, size_t* bytes) {
  const moe_status st = check_dims(dims);
  if (st != MOE_OK) return st;
  if (bytes == nullptr) return MOE_ERR_INVALID;
  *bytes = moe::mx_act_layout(dims->n_experts, dims->d_model, dims->d_ff, max_rows(dims)).total;
  return MOE_OK;
}

moe_status moe_grouped_ffn_mx(const moe_dims* dims, const uint16_t* x_perm,
                              const int32_t* expert_offset, const moe_mx_weights* w, uint16_t* h,
                              float* y_perm, void* ws, size_t ws_bytes, void* stream) {
  if (w == nullptr || w->fmt == MOE_WFMT_BF16) return MOE_ERR_INVALID;
  void* act_ws = nullptr;
  if (block_scaled(w->fmt) && check_dims(dims) == MOE_OK && ws != nullptr) {
    const size_t base = round_up(stage_ws_bytes(dims), 256);
    size_t extra = 0;
    moe_mx_act_workspace_bytes(dims, &extra);
    if (ws_bytes < base + extra) return MOE_ERR_WORKSPACE;
    act_ws = static_cast<char*>(ws) + base;
  }
  return grouped_ffn_impl(dims, x_perm, expert_offset, weights_of(w), h, y_perm, ws, ws_bytes,
                          stream, act_ws);
}

moe_status moe_unpermute_combine(const moe_dims* dims, const float* y_perm,
                                 const int32_t* row_of_pair, const float* topk_w,
                                 const uint16_t* residual, void* out, int32_t out_f32, void* ws,
                                 size_t ws_bytes, void* stream) {
  moe_status st = check_dims(dims);
  if (st != MOE_OK) return st;
  if (dims->T == 0) return MOE_OK;
  const int64_t rmax = max_rows(dims);
  if (!row_of_pair || !topk_w || !out || (rmax > 0 && !y_perm)) return MOE_ERR_INVALID;
  if (out_f32 != 0 && out_f32 != 1) return MOE_ERR_INVALID;
  if ((y_perm && !aligned16(y_perm)) || !aligned16(row_of_pair) || !aligned16(topk_w) ||
      !aligned16(out) || (residual && !aligned16(residual)) || (ws && !aligned16(ws)))
    return MOE_ERR_UNSUPPORTED;
  if (ws && ws_bytes < moe::kStatusBytes) return MOE_ERR_WORKSPACE;
  if ((st = check_device()) != MOE_OK) return st;
  return launch_status(moe::launch_combine(y_perm, row_of_pair, topk_w, residual, out, out_f32,
                                           dims->T, dims->d_model, dims->top_k, rmax,
                                           ws ? status_of(ws) : nullptr, as_stream(stream)));
}

moe_status moe_router_stats(const moe_dims* dims, const float* logits, const int32_t* topk_idx,
                            const int32_t* slot, float alpha, int32_t* picks, float* prob_mean,
                            float* aux_loss, int32_t* dropped, void* ws, size_t ws_bytes,
                            void* stream) {
  moe_status st = check_dims(dims);
  if (st != MOE_OK) return st;
  if (dims->T == 0) return MOE_OK;
  if (!logits || !topk_idx || !slot || !picks || !prob_mean || !aux_loss || !dropped || !ws)
    return MOE_ERR_INVALID;
  if (!aligned16(logits) || !aligned16(topk_idx) || !aligned16(slot) || !aligned16(picks) ||
      !aligned16(prob_mean) || !aligned16(ws))
    return MOE_ERR_UNSUPPORTED;
  if (ws_bytes < stage_ws_bytes(dims)) return MOE_ERR_WORKSPACE;
  if ((st = check_device()) != MOE_OK) return st;
  return launch_status(moe::launch_router_stats(logits, topk_idx, slot, alpha, picks, prob_mean,
                                                aux_loss, dropped, shared_region_of(dims, ws),
                                                dims->T, dims->n_experts, dims->top_k,
                                                as_stream(stream)));
}

moe_status moe_forward_workspace_bytes(const moe_dims* dims, size_t* bytes) {
  const moe_status st = check_dims(dims);
  if (st != MOE_OK) return st;
  if (bytes == nullptr) return MOE_ERR_INVALID;
  // lay the buffers out from address 0 to measure the total
  size_t off = 0;
  const int64_t T = dims->T, N = dims->n_experts, k = dims->top_k, d = dims->d_model,
                F = dims->d_ff, R = max_rows(dims);
  const size_t sizes[] = {size_t(T * N * 4), size_t(T * k * 4), size_t(T * k * 4), size_t(T * k * 4),
                          size_t(N * 4),     size_t((N + 1) * 4), size_t(T * k * 4), size_t(R * 4),
                          size_t(R * d * 2), size_t(R * F * 2),  size_t(R * d * 4),
                          stage_ws_bytes(dims)};
  for (size_t s : sizes) off += round_up(s, 256);
  *bytes = off;
  return MOE_OK;
}

moe_status moe_forward_layout(const moe_dims* dims, void* ws, size_t ws_bytes,
                              moe_forward_buffers* bufs) {
  moe_status st = check_dims(dims);
  if (st != MOE_OK) return st;
  if (ws == nullptr || bufs == nullptr) return MOE_ERR_INVALID;
  if (!aligned16(ws)) return MOE_ERR_UNSUPPORTED;
  size_t need = 0;
  moe_forward_workspace_bytes(dims, &need);
  if (ws_bytes < need) return MOE_ERR_WORKSPACE;
  const int64_t T = dims->T, N = dims->n_experts, k = dims->top_k, d = dims->d_model,
                F = dims->d_ff, R = max_rows(dims);
  char* p = static_cast<char*>(ws);
  auto take = [&p](size_t bytes) {
    char* q = p;
    p += round_up(bytes, 256);
    return q;
  };
  bufs->logits = reinterpret_cast<float*>(take(T * N * 4));
  bufs->topk_idx = reinterpret_cast<int32_t*>(take(T * k * 4));
  bufs->topk_w = reinterpret_cast<float*>(take(T * k * 4));
  bufs->slot = reinterpret_cast<int32_t*>(take(T * k * 4));
  bufs->expert_count = reinterpret_cast<int32_t*>(take(N * 4));
  bufs->expert_offset = reinterpret_cast<int32_t*>(take((N + 1) * 4));
  bufs->row_of_pair = reinterpret_cast<int32_t*>(take(T * k * 4));
  bufs->pair_of_row = reinterpret_cast<int32_t*>(take(R * 4));
  bufs->x_perm = reinterpret_cast<uint16_t*>(take(R * d * 2));
  bufs->h = reinterpret_cast<uint16_t*>(take(R * F * 2));
  bufs->y_perm = reinterpret_cast<float*>(take(R * d * 4));
  bufs->stage_ws_bytes = stage_ws_bytes(dims);
  bufs->stage_ws = take(bufs->stage_ws_bytes);
  return MOE_OK;
}

namespace {
// Regions of a backward workspace, in order (each rounded up to 256 bytes).
struct BackwardLayout {
  size_t sizes[9];
};
BackwardLayout backward_layout(const moe_dims* dims) {
  const int64_t T = dims->T, N = dims->n_experts, d = dims->d_model, F = dims->d_ff,
                R = max_rows(dims);
  const int64_t n_gu = dims->act == MOE_ACT_SWIGLU ? 2 * F : F;
  const int64_t chunk = static_cast<int64_t>(moe::backward_router_chunk(static_cast<int>(T)));
  const int64_t chunks = T > 0 ? (T + chunk - 1) / chunk : 0;
  BackwardLayout l{{moe::kStatusBytes, size_t(T * N * 4), size_t(R * d * 2), size_t(R * n_gu * 4),
                    size_t(R * F * 4), size_t(R * n_gu * 2), size_t(R * F * 2), size_t(R * d * 4),
                    size_t(chunks * N * d * 4)}};
  return l;
}
}  // namespace

moe_status moe_backward_workspace_bytes(const moe_dims* dims, size_t* bytes) {
  const moe_status st = check_dims(dims);
  if (st != MOE_OK) return st;
  if (bytes == nullptr) return MOE_ERR_INVALID;
  size_t off = 0;
  for (size_t s : backward_layout(dims).sizes) off += round_up(s, 256);
  *bytes = off;
  return MOE_OK;
}

moe_status moe_backward(const moe_dims* dims, const uint16_t* x, const float* w_router,
                        const uint16_t* w_gate_up, const uint16_t* w_down, const void* fwd_ws,
                        size_t fwd_ws_bytes, const uint16_t* d_out, float* d_x, float* d_w_router,
                        float* d_logit_bias, float* d_w_gate_up, float* d_w_down, void* ws,
                        size_t ws_bytes, void* stream) {
  moe_status st = check_dims(dims);
  if (st != MOE_OK) return st;
  if (dims->T == 0) return MOE_OK;
  if (!x || !w_router || !w_gate_up || !w_down || !fwd_ws || !d_out || !d_x || !d_w_router ||
      !d_w_gate_up || !d_w_down || !ws)
    return MOE_ERR_INVALID;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(w_gate_up) || !aligned16(w_down) ||
      !aligned16(d_out) || !aligned16(d_x) || !aligned16(d_w_router) || !aligned16(d_w_gate_up) ||
      !aligned16(d_w_down) || !aligned16(ws) || (d_logit_bias && !aligned16(d_logit_bias)))
    return MOE_ERR_UNSUPPORTED;
  size_t need = 0;
  moe_backward_workspace_bytes(dims, &need);
  if (ws_bytes < need) return MOE_ERR_WORKSPACE;
  moe_forward_buffers fb;
  if ((st = moe_forward_layout(dims, const_cast<void*>(fwd_ws), fwd_ws_bytes, &fb)) != MOE_OK)
    return st;
  if ((st = check_device()) != MOE_OK) return st;
  const BackwardLayout l = backward_layout(dims);
  char* regions[9];
  char* p = static_cast<char*>(ws);
  for (int i = 0; i < 9; ++i) {
    regions[i] = p;
    p += round_up(l.sizes[i], 256);
  }
  moe::BackwardArgs a{};
  a.d_out = d_out;
  a.x = x;
  a.w_router = w_router;
  a.w_gate_up = w_gate_up;
  a.w_down = w_down;
  a.topk_w = fb.topk_w;
  a.topk_idx = fb.topk_idx;
  a.row_of_pair = fb.row_of_pair;
  a.expert_offset = fb.expert_offset;
  a.x_perm = fb.x_perm;
  a.y_perm = fb.y_perm;
  a.status = reinterpret_cast<int*>(regions[0]);
  a.d_logits = reinterpret_cast<float*>(regions[1]);
  a.dy_perm = reinterpret_cast<uint16_t*>(regions[2]);
  a.pre = reinterpret_cast<float*>(regions[3]);
  a.dh = reinterpret_cast<float*>(regions[4]);
  a.d_pre = reinterpret_cast<uint16_t*>(regions[5]);
  a.h = reinterpret_cast<uint16_t*>(regions[6]);
  a.dx_rows = reinterpret_cast<float*>(regions[7]);
  a.router_part = reinterpret_cast<float*>(regions[8]);
  a.d_x = d_x;
  a.d_w_router = d_w_router;
  a.d_logit_bias = d_logit_bias;
  a.d_w_gate_up = d_w_gate_up;
  a.d_w_down = d_w_down;
  a.T = dims->T;
  a.d = dims->d_model;
  a.N = dims->n_experts;
  a.k = dims->top_k;
  a.F = dims->d_ff;
  a.act = dims->act;
  a.r_max = max_rows(dims);
  a.timeout_ns = moe::wait_timeout_ns();
  return launch_status(moe::launch_backward(a, as_stream(stream)));
}

namespace {
moe_status forward_impl(const moe_dims* dims, const uint16_t* x, const float* w_router,
                        const float* logit_bias, const Weights& w, const uint16_t* residual,
                        uint16_t* out, void* ws, size_t ws_bytes, void* stream) {
  moe_forward_buffers b;
  moe_status st = moe_forward_layout(dims, ws, ws_bytes, &b);
  if (st != MOE_OK) return st;
  void* act_ws = nullptr;
  if (block_scaled(w.fmt)) {  // the activation region follows the forward layout
    size_t base = 0, extra = 0;
    moe_forward_workspace_bytes(dims, &base);
    moe_mx_act_workspace_bytes(dims, &extra);
    base = round_up(base, 256);
    if (ws_bytes < base + extra) return MOE_ERR_WORKSPACE;
    act_ws = static_cast<char*>(ws) + base;
  }
  if (dims->T == 0) return MOE_OK;
  if (!x || !w_router || !out) return MOE_ERR_INVALID;
  if ((st = check_weights(w)) != MOE_OK) return st;
  const int64_t rmax = max_rows(dims);
  const bool route_sorts = moe::use_decode_route(dims->T, dims->n_experts, dims->d_model) &&
                           rmax * dims->d_model * 2 <= moe::kDecodePermuteMaxBytes;
  if (route_sorts) {
    // decode-sized batch: routing and the sort by expert in one launch
    if (!aligned16(x) || !aligned16(w_router) || (logit_bias && !aligned16(logit_bias)))
      return MOE_ERR_UNSUPPORTED;
    if ((st = check_device()) != MOE_OK) return st;
    moe::DecodeRouteArgs a = decode_route_args(dims, x, w_router, logit_bias, b.logits,
                                               b.topk_idx, b.topk_w, b.slot, b.expert_count,
                                               b.stage_ws);
    a.expert_offset = b.expert_offset;
    a.row_of_pair = b.row_of_pair;
    a.pair_of_row = b.pair_of_row;
    a.x_perm = b.x_perm;
    st = launch_status(moe::launch_decode_route(a, as_stream(stream)));
  } else {
    st = moe_route(dims, x, w_router, logit_bias, b.logits, b.topk_idx, b.topk_w, b.slot,
                   b.expert_count, b.stage_ws, b.stage_ws_bytes, stream);
    if (st != MOE_OK) return st;
    st = moe_permute(dims, x, b.topk_idx, b.slot, b.expert_count, b.expert_offset, b.row_of_pair,
                     b.pair_of_row, b.x_perm, b.stage_ws, b.stage_ws_bytes, stream);
  }
  if (st != MOE_OK) return st;
  st = grouped_ffn_impl(dims, b.x_perm, b.expert_offset, w, b.h, b.y_perm, b.stage_ws,
                        b.stage_ws_bytes, stream, act_ws);
  if (st != MOE_OK) return st;
  return moe_unpermute_combine(dims, b.y_perm, b.row_of_pair, b.topk_w, residual, out, 0,
                               b.stage_ws, b.stage_ws_bytes, stream);
}
}  // namespace

moe_status moe_forward(const moe_dims* dims, const uint16_t* x, const float* w_router,
                       const float* logit_bias, const uint16_t* w_gate_up, const uint16_t* w_down,
                       const uint16_t* residual, uint16_t* out, void* ws, size_t ws_bytes,
                       void* stream) {
  return forward_impl(dims, x, w_router, logit_bias,
                      Weights{MOE_WFMT_BF16, w_gate_up, nullptr, w_down, nullptr}, residual, out,
                      ws, ws_bytes, stream);
}

moe_status moe_forward_mx(const moe_dims* dims, const uint16_t* x, const float* w_router,
                          const float* logit_bias, const moe_mx_weights* w,
                          const uint16_t* residual, uint16_t* out, void* ws, size_t ws_bytes,
                          void* stream) {
  if (w == nullptr || w->fmt == MOE_WFMT_BF16) return MOE_ERR_INVALID;
  return forward_impl(dims, x, w_router, logit_bias, weights_of(w), residual, out, ws, ws_bytes,
                      stream);
}

moe_status moe_read_device_error(void* ws, void* stream, moe_status* err) {
  if (ws == nullptr || err == nullptr) return MOE_ERR_INVALID;
  const cudaStream_t s = as_stream(stream);
  int v = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemcpy(&v, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemset(ws, 0, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  *err = static_cast<moe_status>(v);
  return MOE_OK;
}

uint64_t moe_debug_set_wait_timeout_ns(uint64_t ns) {
  return moe::g_wait_timeout_ns.exchange(ns == 0 ? moe::kDefaultWaitTimeoutNs : ns);
}

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape, alignment or device";
    case MOE_ERR_CUDA: return "CUDA launch error";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_TIMEOUT: return "device wait timed out";
    case MOE_ERR_BOUNDS: return "device index out of bounds";
  }
  return "unknown status";
}

}  // extern "C"
