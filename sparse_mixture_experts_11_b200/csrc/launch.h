// Host-side launchers of the MoE kernels (internal to the library; the C ABI is in moe.h).
// Each launcher only enqueues work on `stream` and returns the launch error, if any.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "moe.h"

namespace moe {

// Launch a library kernel with programmatic stream serialisation (see pdl_wait/pdl_trigger).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// The same, in thread-block clusters of `cluster_x` CTAs along x (grid.x a multiple of it).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block,
                                      size_t smem, cudaStream_t s, unsigned cluster_x,
                                      Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster_x;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Runs a set-up step (a kernel attribute such as the dynamic shared-memory limit, which the
// runtime keeps per device) once on each device it is called on, the current device at the
// time of the call, and returns that device's cached result afterwards.
class PerDeviceOnce {
 public:
  static constexpr int kDevices = 64;
  template <typename Fn>
  cudaError_t run(Fn fn) {
    int dev = 0;
    const cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kDevices) return cudaErrorInvalidDevice;
    std::call_once(flag_[dev], [&] { err_[dev] = fn(); });
    return err_[dev];
  }

 private:
  std::once_flag flag_[kDevices];
  cudaError_t err_[kDevices] = {};
};

// Per-stage workspace layout: [0, 256) status word (+ padding); [256, ...) capacity-scan scratch.
constexpr size_t kStatusBytes = 256;
constexpr int kSlotChunk = 4096;  // (token, choice) pairs ranked per block in the slot pass
constexpr uint64_t kDefaultWaitTimeoutNs = 2000000000ull;  // limit of one mbarrier wait (2 s)
// Limit of the waits a CTA makes, after giving up, for its own TMA copies and MMAs still in
// flight (independent of the wait limit above, so a short limit never cuts the drain short).
constexpr uint64_t kDrainTimeoutNs = 1000000000ull;
// The wait limit the entry points pass to the kernels (moe_debug_set_wait_timeout_ns).
uint64_t wait_timeout_ns();

inline int64_t slot_chunks(int64_t pairs) { return (pairs + kSlotChunk - 1) / kSlotChunk; }

struct DeviceInfo {
  int sm_count;
  int cc_major;
  int cc_minor;
};
cudaError_t device_info(DeviceInfo* out);

// Router path choice. One block per token re-reads W_r from L2 for every token; once that
// traffic (T * N * d * 4 bytes) passes 256 MiB the tensor-core router, which reads W_r once
// per 128 tokens, is used instead.
inline bool router_uses_tensor_cores(int64_t T, int64_t N, int64_t d) {
  return static_cast<double>(T) * N * d * 4.0 > 268435456.0;
}
// Bytes of the [3][N][d] bf16 split of W_r the tensor-core router reads when given scratch.
size_t router_split_bytes(int N, int d);

// Router statistics emitted by the routing launches (moe_route_with_stats). The router writes
// per-tile sums of its softmax probabilities, prob_part [n_parts][N] (the tensor-core router:
// one row per 128-token tile, or per CTA of a tile split over a cluster; the per-token router:
// one row per token); the capacity pass, which counts each expert's picks before the
// capacity, adds the rows in order and forms the outputs. prob_part null: no statistics.
struct RouteStats {
  float* prob_part;
  int n_parts;
  float alpha;
  int32_t* picks;     // [N] pairs that chose each expert
  float* prob_mean;   // [N] mean router probability
  float* aux_loss;    // alpha * N * sum_e (picks_e / T) * prob_mean_e
  int32_t* dropped;   // pairs over the capacity
};
// partial rows the router writes: the tensor-core router's (tiles x cluster size) or T
int router_tc_parts(int T, int d);
inline int route_stats_parts(int64_t T, int64_t N, int64_t d) {
  return router_uses_tensor_cores(T, N, d) ? router_tc_parts(static_cast<int>(T), static_cast<int>(d))
                                           : static_cast<int>(T);
}

// router: logits = x W_r^T (+ b), then top-k and renormalised weights. status may be null.
// split_scratch: router_split_bytes() of device memory for the tensor-core path, or null to
// split W_r inside the router kernel (same results, slower). prob_part: see RouteStats.
cudaError_t launch_router_topk(const uint16_t* x, const float* w_router, const float* bias,
                               float* logits, int32_t* topk_idx, float* topk_w, int T, int d,
                               int N, int k, uint16_t* split_scratch, int* status,
                               uint64_t timeout_ns, cudaStream_t s, float* prob_part = nullptr);
cudaError_t launch_router_tc(const uint16_t* x, const float* w_router, const float* bias,
                             float* logits, int32_t* topk_idx, float* topk_w, int T, int d, int N,
                             int k, uint16_t* split_scratch, int* status, uint64_t timeout_ns,
                             float* prob_part, cudaStream_t s);
// Decode-sized batches (T <= kDecodeRouteMaxT) route in one launch: CTA c takes columns
// [128 c, 128 c + 128) of d for every token and expert and stores partial dot products; the
// last CTA to finish (arrival counter, zero between calls) adds them in order of c, then takes
// top-k, the capacity slots and, when given the permute outputs, the sort by expert and the
// x_perm copy. Scratch: decode_route_scratch_bytes(); the counter lives in the status region.
constexpr int kDecodeRouteMaxT = 16;
constexpr int kDecodeSlice = 128;
constexpr size_t kDecodeCounterOffset = 128;  // bytes into the workspace's status region
constexpr size_t kDecodeMaxScratch = size_t(1) << 20;  // partial dot products, at most
// the last CTA copies x_perm only while it is this small
constexpr int64_t kDecodePermuteMaxBytes = 512 * 1024;
inline size_t decode_route_scratch_bytes(int64_t T, int64_t N, int64_t d) {
  return static_cast<size_t>((d + kDecodeSlice - 1) / kDecodeSlice) * T * N * sizeof(float);
}
// moe_route, moe_forward and moe_route_noalloc all take this path under the same rule, so
// their routing agrees bit for bit.
inline bool use_decode_route(int64_t T, int64_t N, int64_t d) {
  return T >= 1 && T <= kDecodeRouteMaxT && decode_route_scratch_bytes(T, N, d) <= kDecodeMaxScratch;
}
struct DecodeRouteArgs {
  const uint16_t* x;
  const float* w_router;
  const float* bias;
  float* logits;
  int32_t* topk_idx;
  float* topk_w;
  int32_t* slot;
  int32_t* expert_count;
  int32_t* expert_offset;  // these four null: no permutation
  int32_t* row_of_pair;
  int32_t* pair_of_row;
  uint16_t* x_perm;
  float* part;    // decode_route_scratch_bytes()
  int* counter;   // zero between calls
  int T, d, N, k, cap;
  // router statistics (moe_route_with_stats), formed by the CTA that finishes the routing;
  // picks null: none
  int32_t* st_picks;
  float* st_prob_mean;
  float* st_aux_loss;
  int32_t* st_dropped;
  float st_alpha;
};
cudaError_t launch_decode_route(const DecodeRouteArgs& a, cudaStream_t s);
// Overflow policy "redirect to the next most suitable expert" (see route.cu): slots and the
// serving experts from the router's top-k and logits, for at most kRerouteMaxPairs pairs (the
// sequential pass holds every pair's expert as a byte in shared memory).
// Scratch (16-byte aligned pieces): the preference lists, T * kRedirectPrefs bytes; the pairs'
// experts as bytes, P rounded up to 32; a bit per pair marking an expert id outside [0, N).
constexpr int64_t kRerouteMaxPairs = 163840;
constexpr int kRedirectPrefs = 16;
inline size_t redirect_round16(int64_t b) { return static_cast<size_t>((b + 15) / 16 * 16); }
inline size_t redirect_scratch_bytes(int64_t T, int k) {
  const int64_t P = T * k;
  if (P > kRerouteMaxPairs) return 0;
  return redirect_round16(T * kRedirectPrefs) + static_cast<size_t>((P + 31) / 32 * 32) +
         redirect_round16((P + 31) / 32 * 4);
}
cudaError_t launch_reroute_slots(const float* logits, uint8_t* scratch, int32_t* topk_idx,
                                int32_t* slot, int32_t* expert_count, int T, int N, int k,
                                int capacity, int* status, cudaStream_t s);
// top-k and renormalised weights from given logits
cudaError_t launch_topk_from_logits(const float* logits, int32_t* topk_idx, float* topk_w, int T,
                                    int N, int k, cudaStream_t s);
// capacity slots in (choice, token) arrival order
cudaError_t launch_capacity_slots(const int32_t* topk_idx, int32_t* slot, int32_t* expert_count,
                                  int32_t* chunk_scratch, int T, int N, int k, int capacity,
                                  cudaStream_t s, const RouteStats* stats = nullptr);
// sort kept pairs into expert-contiguous rows
cudaError_t launch_permute(const uint16_t* x, const int32_t* topk_idx, const int32_t* slot,
                           const int32_t* expert_count, int32_t* expert_offset,
                           int32_t* row_of_pair, int32_t* pair_of_row, uint16_t* x_perm, int T,
                           int d, int N, int k, int64_t r_max, int* status, cudaStream_t s);
// weighted sum back in token order
cudaError_t launch_combine(const float* y_perm, const int32_t* row_of_pair, const float* topk_w,
                           const uint16_t* residual, void* out, int out_f32, int T, int d, int k,
                           int64_t r_max, int* status, cudaStream_t s);

// router statistics and the auxiliary loss (two deterministic passes)
size_t router_stats_scratch_bytes(int T, int N);
cudaError_t launch_router_stats(const float* logits, const int32_t* topk_idx, const int32_t* slot,
                                float alpha, int32_t* picks, float* prob_mean, float* aux_loss,
                                int32_t* dropped, void* scratch, int T, int N, int k,
                                cudaStream_t s);

// grouped expert GEMMs on tcgen05
//
// Scratch of the grouped FFN (one launch for both GEMMs). Counters, zero between calls (each
// call leaves them zero), as ints: [per m-tile: finished gate/up tiles][CTAs done][stream-K
// arrival counters of the gate/up tiles][... of the down tiles]. Partial slots, as floats:
// [gate/up: sk_ctas1 x 2 x slot_rows x 256][down: sk_ctas2 x 2 x slot_rows x 256].
struct FfnScratchPlan {
  int bm;                  // rows per tile: 64 when no expert can hold more, else 128
  int slot_rows;           // rows of a partial slot: min(bm, rows_per_expert)
  int sk_ctas1, sk_ctas2;  // CTAs with stream-K partial slots per GEMM (0: whole tiles only)
  int64_t m_tiles_ub, tiles1_ub, tiles2_ub;
  size_t counter_bytes;
  size_t part_bytes;       // shares the workspace region with the routing scratch
};
// rows_per_expert: the most rows any one expert can receive, min(capacity, T). block_scaled:
// the plan of the block-scaled formats (128-row tiles, k blocks of 128); it never needs more
// counter or partial bytes than the default plan of the same shape.
FfnScratchPlan ffn_scratch_plan(int N, int d, int F, int act, int64_t r_max,
                                int64_t rows_per_expert, bool block_scaled = false);
// Bytes the block-scaled formats need besides the per-stage workspace: the quantised token
// rows [r_max, d] (1 byte each) and the scale atoms of the rows and of h (512 bytes per m-tile
// and k block of 128), each region rounded up to 256 bytes.
struct MxActLayout {
  size_t xq_bytes, x_atom_bytes, h_atom_bytes, total;
};
MxActLayout mx_act_layout(int N, int d, int F, int64_t r_max);

struct GroupedFfnArgs {
  const uint16_t* x_perm;
  const int32_t* expert_offset;
  int wfmt;                    // moe_wfmt: bf16 or an MX format
  const void* w_gate_up;       // bf16 weights, or MX packed elements
  const void* w_down;
  const uint8_t* w_gate_up_scales;  // MX only: E8M0 scales [N][K/32][rows]
  const uint8_t* w_down_scales;
  uint16_t* h;
  float* y_perm;
  int N, d, F, act;
  int64_t r_max;
  int* status;
  uint64_t timeout_ns;
  int* counters;            // ffn_scratch_plan().counter_bytes, zero between calls
  float* part;              // ffn_scratch_plan().part_bytes, or null: whole tiles only
  int64_t rows_per_expert;  // min(capacity, T)
  void* act_ws;             // block-scaled formats: mx_act_layout().total bytes; else unused
};
cudaError_t launch_grouped_ffn(const GroupedFfnArgs& a, cudaStream_t s);

// Backward pass (backward.cu). Saved from the forward: the routing, x_perm and y_perm.
struct BackwardArgs {
  const uint16_t* d_out;          // [T, d] bf16
  const uint16_t* x;              // [T, d] bf16
  const float* w_router;          // [N, d]
  const uint16_t* w_gate_up;      // [N, n_gu, d]
  const uint16_t* w_down;         // [N, d, F]
  const float* topk_w;            // [T, k]
  const int32_t* topk_idx;        // [T, k]
  const int32_t* row_of_pair;     // [T, k]
  const int32_t* expert_offset;   // [N + 1]
  const uint16_t* x_perm;         // [r_max, d]
  const float* y_perm;            // [r_max, d]
  // workspace
  float* d_logits;                // [T, N]
  uint16_t* dy_perm;              // [r_max, d]
  float* pre;                     // [r_max, n_gu]
  float* dh;                      // [r_max, F]
  uint16_t* d_pre;                // [r_max, n_gu]
  uint16_t* h;                    // [r_max, F]
  float* dx_rows;                 // [r_max, d]
  float* router_part;             // [chunks, N, d], chunks = ceil(T / backward_router_chunk(T))
  // outputs
  float* d_x;                     // [T, d]
  float* d_w_router;              // [N, d]
  float* d_logit_bias;            // [N] or null
  float* d_w_gate_up;             // [N, n_gu, d]
  float* d_w_down;                // [N, d, F]
  int T, d, N, k, F, act;
  int64_t r_max;
  int* status;
  uint64_t timeout_ns;
};
size_t backward_router_chunk(int T);
cudaError_t launch_backward(const BackwardArgs& a, cudaStream_t s);

}  // namespace moe
