// moe_route_noalloc: moe_route for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc, or have no allocator to ask. Examples: an inference
// engine that hands out all device memory up front from its own arena; code on a real-time
// path where an allocation could synchronise the device or fail mid-run; a plugin whose host
// framework owns every allocation. moe_route needs a caller-provided workspace for its
// capacity scan (and, for large batches, for a bf16 split of the router weight; for
// decode-sized batches, for the one-launch router's partial dot products and its arrival
// counter). This variant takes that scratch from fixed arrays in the library's own device
// memory and splits the router weight inside the router kernel instead, so its caller passes
// only inputs and outputs. Its results are identical to moe_route's.
//
// The scratch lives in a file-scope __device__ array. Every GPU that loads the library holds
// it until the process exits. In host code, the array's name is only a host-side stand-in
// for the symbol: it is not a device address. A kernel given it would fault, or on a system
// where the GPU can reach host memory, silently use the wrong memory. The device address is
// therefore looked up once per device with cudaGetSymbolAddress (with that device current)
// and then passed to the kernels.
#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace {

constexpr int kScratchInts = MOE_ROUTE_NOALLOC_SCRATCH_BYTES / 4;
static_assert(MOE_ROUTE_NOALLOC_SCRATCH_BYTES % 256 == 0, "scratch size");

// Per-chunk expert histograms of the capacity scan: [n_chunks, N] int32. Each call writes
// every entry it later reads, so nothing in it has to start at zero.
static __device__ __align__(256) int32_t g_route_scratch[kScratchInts];
// The one-launch decode router's partial dot products (written before they are read) and its
// arrival counter (zero at load; every call leaves it zero).
static __device__ __align__(256) float g_decode_part[moe::kDecodeMaxScratch / sizeof(float)];
static __device__ __align__(256) int g_decode_counter[64];

constexpr int kMaxDevices = 64;
std::once_flag g_once[kMaxDevices];
struct Scratch {
  int32_t* slots;
  float* decode_part;
  int* decode_counter;
};
Scratch g_scratch[kMaxDevices];
cudaError_t g_scratch_err[kMaxDevices];

// Device addresses of the scratch arrays on the current device; looked up on the first call
// per device (with that device current) and cached.
cudaError_t scratch_on_current_device(Scratch* out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::call_once(g_once[dev], [dev] {
    void* a = nullptr;
    void* b = nullptr;
    void* c = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&a, g_route_scratch);
    if (e == cudaSuccess) e = cudaGetSymbolAddress(&b, g_decode_part);
    if (e == cudaSuccess) e = cudaGetSymbolAddress(&c, g_decode_counter);
    g_scratch_err[dev] = e;
    g_scratch[dev] = Scratch{static_cast<int32_t*>(a), static_cast<float*>(b), static_cast<int*>(c)};
  });
  *out = g_scratch[dev];
  return g_scratch_err[dev];
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" moe_status moe_route_noalloc(const moe_dims* dims, const uint16_t* x,
                                        const float* w_router, const float* logit_bias,
                                        float* logits, int32_t* topk_idx, float* topk_w,
                                        int32_t* slot, int32_t* expert_count, void* stream) {
  if (dims == nullptr) return MOE_ERR_INVALID;
  // Same shape rules as moe_route (moe_workspace_bytes validates and sizes).
  size_t ws_bytes = 0;
  const moe_status st = moe_workspace_bytes(dims, &ws_bytes);
  if (st != MOE_OK) return st;
  if (dims->T == 0) return MOE_OK;
  const int64_t pairs = static_cast<int64_t>(dims->T) * dims->top_k;
  const int64_t chunks = moe::slot_chunks(pairs);
  const int64_t scratch_ints = chunks > 1 ? chunks * dims->n_experts : 0;
  if (scratch_ints > kScratchInts) return MOE_ERR_WORKSPACE;  // beyond the built-in scratch
  if (!x || !w_router || !logits || !topk_idx || !topk_w || !slot || !expert_count)
    return MOE_ERR_INVALID;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(logits) || !aligned16(topk_idx) ||
      !aligned16(topk_w) || !aligned16(slot) || !aligned16(expert_count) ||
      (logit_bias && !aligned16(logit_bias)))
    return MOE_ERR_UNSUPPORTED;
  moe::DeviceInfo di;
  if (moe::device_info(&di) != cudaSuccess) return MOE_ERR_CUDA;
  if (di.cc_major != 10 || di.cc_minor != 0) return MOE_ERR_UNSUPPORTED;
  Scratch scratch{};
  if (scratch_on_current_device(&scratch) != cudaSuccess || scratch.slots == nullptr ||
      scratch.decode_part == nullptr || scratch.decode_counter == nullptr)
    return MOE_ERR_CUDA;

  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int cap = dims->capacity < dims->T ? dims->capacity : dims->T;
  if (moe::use_decode_route(dims->T, dims->n_experts, dims->d_model)) {
    moe::DecodeRouteArgs a{};
    a.x = x;
    a.w_router = w_router;
    a.bias = logit_bias;
    a.logits = logits;
    a.topk_idx = topk_idx;
    a.topk_w = topk_w;
    a.slot = slot;
    a.expert_count = expert_count;
    a.part = scratch.decode_part;
    a.counter = scratch.decode_counter;
    a.T = dims->T;
    a.d = dims->d_model;
    a.N = dims->n_experts;
    a.k = dims->top_k;
    a.cap = cap;
    return moe::launch_decode_route(a, s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  }
  if (moe::launch_router_topk(x, w_router, logit_bias, logits, topk_idx, topk_w, dims->T,
                              dims->d_model, dims->n_experts, dims->top_k, nullptr, nullptr,
                              moe::wait_timeout_ns(), s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (moe::launch_capacity_slots(topk_idx, slot, expert_count, scratch.slots, dims->T, dims->n_experts,
                                 dims->top_k, cap, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}
