// Routing kernels: router logits, top-k with renormalised weights, capacity slots.
//
// Page «Sparse Mixture-of-Experts» (bigdataschool wiki):
//   «Роутер и top-k gating»: logits from a linear layer without bias term, softmax over the
//     experts, the k most probable experts per token, their probabilities renormalised to one;
//   «Expert capacity и capacity factor»: ceil(capacity_factor * T / N) slots per expert, and a
//     pair that arrives at a full expert is dropped (first come, first served in batch order).
//
// Selection is made on the fp32 logits (softmax is strictly increasing, so the chosen experts
// are the same); equal logits go to the lower expert index. The renormalised weight of choice j
// is exp(L_j - L_0) / sum_i exp(L_i - L_0) over the chosen logits, which equals p_j / sum p_i.
// Arrival order for the capacity is (choice, token): all first choices in token order, then
// all second choices, and so on.
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "decode_route.cuh"
#include "launch.h"

namespace moe {
namespace {

using dr::better;
using dr::kFull;
using dr::warp_best;
using dr::warp_topk_write;

// ------------------------------------------------------------------ router (SIMT fp32)
// One block of 1024 threads per token for small batches. g warps share each expert's dot
// product (g = the largest power of two with g * N <= 32, at least 1), each taking every g-th
// 128-element slice of d with
// float4 loads of W_r and 4-bf16 loads of x; experts beyond 32 / g take further passes. Warp
// partial sums meet in shared memory and are added in a fixed order, then warp 0 takes the
// token's top-k.
constexpr int kTokThreads = 1024;
constexpr int kTokWarps = kTokThreads / 32;

template <int EPT>
__global__ void __launch_bounds__(kTokThreads) router_token_kernel(
    const uint16_t* __restrict__ x, const float* __restrict__ w, const float* __restrict__ bias,
    float* __restrict__ logits, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w, int T,
    int d, int N, int k, float* __restrict__ prob_part) {
  __shared__ float s_part[kTokWarps][EPT];  // [warp][pass]: at most EPT passes of 32 experts
  __shared__ float s_logit[EPT * 32];
  pdl_trigger();
  pdl_wait();
  const int t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint16_t* xr = x + static_cast<int64_t>(t) * d;
  int g = 1;  // warps per expert
  while (g * 2 * N <= kTokWarps) g *= 2;
  const int experts_per_pass = kTokWarps / g;
  const int part = warp % g;
  int pass = 0;
  for (int e0 = 0; e0 < N; e0 += experts_per_pass, ++pass) {
    const int e = e0 + warp / g;
    float acc = 0.f;
    if (e < N) {
      const float* wr = w + static_cast<int64_t>(e) * d;
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 8
      for (int i = (part * 32 + lane) * 4; i < d; i += 128 * g) {
        const float4 wv = __ldg(reinterpret_cast<const float4*>(wr + i));
        const uint2 xv = __ldg(reinterpret_cast<const uint2*>(xr + i));
        a0 = fmaf(__uint_as_float(xv.x << 16), wv.x, a0);
        a1 = fmaf(__uint_as_float(xv.x & 0xffff0000u), wv.y, a1);
        a2 = fmaf(__uint_as_float(xv.y << 16), wv.z, a2);
        a3 = fmaf(__uint_as_float(xv.y & 0xffff0000u), wv.w, a3);
      }
      acc = (a0 + a1) + (a2 + a3);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
    }
    if (lane == 0) s_part[warp][pass] = acc;
  }
  __syncthreads();
  // the g partial sums of each expert, added in order of part
  for (int e = threadIdx.x; e < N; e += kTokThreads) {
    const int p = e / experts_per_pass, wbase = (e % experts_per_pass) * g;
    float L = 0.f;
    for (int q = 0; q < g; ++q) L += s_part[wbase + q][p];
    if (bias != nullptr) L += bias[e];
    s_logit[e] = L;
    logits[static_cast<int64_t>(t) * N + e] = L;
  }
  __syncthreads();
  if (warp == 0) {
    float val[EPT];
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
      const int e = lane + 32 * j;
      val[j] = (e < N) ? s_logit[e] : -INFINITY;
    }
    warp_topk_write<EPT>(val, N, k, t, topk_idx, topk_w);
  } else if (warp == 1 && prob_part != nullptr) {
    // router statistics: this token's softmax over the experts, one row per token
    float v[EPT];
    float m = -INFINITY;
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
      const int e = lane + 32 * j;
      v[j] = e < N ? s_logit[e] : -INFINITY;
      m = fmaxf(m, v[j]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
      v[j] = (lane + 32 * j) < N ? expf(v[j] - m) : 0.f;
      sum += v[j];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(kFull, sum, o);
    const float inv = 1.0f / sum;
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
      const int e = lane + 32 * j;
      if (e < N) prob_part[static_cast<int64_t>(t) * N + e] = v[j] * inv;
    }
  }
}

template <int EPT>
__global__ void __launch_bounds__(256) topk_from_logits_kernel(const float* __restrict__ logits,
                                                               int32_t* __restrict__ topk_idx,
                                                               float* __restrict__ topk_w, int T,
                                                               int N, int k) {
  pdl_trigger();
  pdl_wait();
  const int warps = blockDim.x >> 5;
  for (int t = blockIdx.x * warps + (threadIdx.x >> 5); t < T; t += gridDim.x * warps) {
    float val[EPT];
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
      const int e = static_cast<int>(lane_id()) + 32 * j;
      val[j] = (e < N) ? logits[static_cast<int64_t>(t) * N + e] : -INFINITY;
    }
    warp_topk_write<EPT>(val, N, k, t, topk_idx, topk_w);
  }
}

// ------------------------------------------------------------------ capacity slots
// Pair p = j * T + t (choice-major) is the p-th arrival. Its slot is the number of earlier
// arrivals with the same expert; it is kept iff that number is below the capacity.
//
// Pass 1 (one block per chunk of kSlotChunk arrivals): warp w ranks its 512 consecutive
// arrivals 32 at a time (lanes with the same expert found by bit ballots), keeping per-warp
// running counts per expert in
// shared memory; then the block turns the per-warp counts into exclusive offsets and either
//   - (one chunk) writes final slots and kept counts directly, or
//   - (several chunks) writes chunk-local ranks into `slot` and chunk totals into scratch.
// Pass 2 (one block): per expert, exclusive scan of the chunk totals; kept counts.
// Pass 3: slot = chunk-local rank + chunk base, or -1 when it reaches the capacity.
// Lanes of the warp whose key equals this lane's key (0 <= key < 512): the AND over the 9 key
// bits of the ballot of lanes agreeing on that bit. Nine ballots, independent of how many
// distinct keys the warp holds.
__device__ __forceinline__ unsigned peers_with_same_key(int key) {
  unsigned peers = kFull;
#pragma unroll
  for (int b = 0; b < 9; ++b) {
    const bool bit = (key >> b) & 1;
    const unsigned bal = __ballot_sync(kFull, bit);
    peers &= bit ? bal : ~bal;
  }
  return peers;
}

constexpr int kSlThreads = 256;
constexpr int kSlWarps = kSlThreads / 32;
constexpr int kSlIters = kSlotChunk / kSlThreads;  // arrivals per lane

// Router statistics from the picks each expert got before the capacity (run, shared memory) and
// the router's partial rows of probability sums, added in row order (page «Sparse
// Mixture-of-Experts», «Маршрутизация токена и auxiliary loss»: alpha * N * sum_i f_i * P_i with
// f_i = picks_i / T and P_i the batch mean of the router's probability for expert i). One block;
// s_term holds 256 floats of shared memory.
__device__ __forceinline__ void route_stats_finish(const RouteStats& st, const int* run, int T,
                                                   int N, int cap, float* s_term) {
  for (int e = threadIdx.x; e < 256; e += blockDim.x) s_term[e] = 0.f;
  for (int e = threadIdx.x; e < N; e += blockDim.x) {
    float sum = 0.f;
    int b = 0;
    for (; b + 8 <= st.n_parts; b += 8) {  // eight independent loads in flight per step
      float v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = __ldcg(st.prob_part + static_cast<int64_t>(b + i) * N + e);
#pragma unroll
      for (int i = 0; i < 8; ++i) sum += v[i];
    }
    for (; b < st.n_parts; ++b) sum += __ldcg(st.prob_part + static_cast<int64_t>(b) * N + e);
    const float P = sum / static_cast<float>(T);
    st.prob_mean[e] = P;
    st.picks[e] = run[e];
    s_term[e] = (static_cast<float>(run[e]) / static_cast<float>(T)) * P;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float total = 0.f;
    int dropped = 0;
    for (int e = 0; e < N; ++e) {
      total += s_term[e];
      dropped += max(0, run[e] - cap);
    }
    *st.aux_loss = st.alpha * static_cast<float>(N) * total;
    *st.dropped = dropped;
  }
}

__global__ void __launch_bounds__(kSlThreads) slot_rank_kernel(
    const int32_t* __restrict__ topk_idx, int32_t* __restrict__ slot,
    int32_t* __restrict__ chunk_hist, int32_t* __restrict__ expert_count, int T, int N, int k,
    int cap, int single_chunk, const RouteStats st) {
  __shared__ int s_cnt[kSlWarps][256];
  __shared__ int s_run[256];
  __shared__ float s_term[256];
  pdl_trigger();
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int P = T * k;  // < 2^31, checked on the host
  for (int i = tid; i < kSlWarps * 256; i += kSlThreads) (&s_cnt[0][0])[i] = 0;
  pdl_wait();

  const int p_base = blockIdx.x * kSlotChunk + w * (kSlotChunk / kSlWarps);
  int ex[kSlIters];
  int q_of[kSlIters];  // storage index t * k + j of each arrival
  // every load is issued before any is used, so their latencies overlap
#pragma unroll
  for (int it = 0; it < kSlIters; ++it) {
    const int p = p_base + it * 32 + lane;
    int q = -1;
    if (p < P) {
      const int j = p / T;
      q = (p - j * T) * k + j;
    }
    q_of[it] = q;
  }
#pragma unroll
  for (int it = 0; it < kSlIters; ++it) ex[it] = q_of[it] >= 0 ? __ldg(topk_idx + q_of[it]) : -1;
#pragma unroll
  for (int it = 0; it < kSlIters; ++it)
    if (q_of[it] >= 0 && (ex[it] < 0 || ex[it] >= N)) ex[it] = -2;  // invalid id: never kept
  __syncthreads();
  int local[kSlIters];
#pragma unroll
  for (int it = 0; it < kSlIters; ++it) {
    const int e = ex[it];
    const unsigned peers = peers_with_same_key(e + 2);  // e + 2 in [0, 257]
    const int rank = __popc(peers & lanemask_lt());
    const int cnt = (e >= 0) ? s_cnt[w][e] : 0;
    __syncwarp();
    if (e >= 0 && rank == 0) s_cnt[w][e] = cnt + __popc(peers);
    __syncwarp();
    local[it] = cnt + rank;
  }
  __syncthreads();
  for (int e = tid; e < N; e += kSlThreads) {
    int run = 0;
#pragma unroll
    for (int w2 = 0; w2 < kSlWarps; ++w2) {
      const int v = s_cnt[w2][e];
      s_cnt[w2][e] = run;
      run += v;
    }
    if (single_chunk)
      expert_count[e] = min(run, cap);
    else
      chunk_hist[static_cast<int64_t>(blockIdx.x) * N + e] = run;
    s_run[e] = run;
  }
  __syncthreads();
#pragma unroll
  for (int it = 0; it < kSlIters; ++it) {
    if (q_of[it] < 0) continue;
    const int e = ex[it];
    int out = -1;
    if (e >= 0) {
      const int r = local[it] + s_cnt[w][e];
      out = single_chunk ? (r < cap ? r : -1) : r;
    }
    slot[q_of[it]] = out;
  }
  if (single_chunk && st.prob_part != nullptr) route_stats_finish(st, s_run, T, N, cap, s_term);
}

__global__ void __launch_bounds__(256) slot_scan_kernel(int32_t* __restrict__ chunk_hist,
                                                        int32_t* __restrict__ expert_count,
                                                        int n_chunks, int T, int N, int cap,
                                                        const RouteStats st) {
  __shared__ int s_run[256];
  __shared__ float s_term[256];
  pdl_trigger();
  pdl_wait();
  for (int e = threadIdx.x; e < N; e += blockDim.x) {
    int run = 0;
    for (int c = 0; c < n_chunks; ++c) {
      const int v = chunk_hist[static_cast<int64_t>(c) * N + e];
      chunk_hist[static_cast<int64_t>(c) * N + e] = run;
      run += v;
    }
    expert_count[e] = min(run, cap);
    s_run[e] = run;
  }
  __syncthreads();
  if (st.prob_part != nullptr) route_stats_finish(st, s_run, T, N, cap, s_term);
}

__global__ void __launch_bounds__(256) slot_finalize_kernel(const int32_t* __restrict__ topk_idx,
                                                            int32_t* __restrict__ slot,
                                                            const int32_t* __restrict__ chunk_hist,
                                                            int T, int N, int k, int cap) {
  pdl_trigger();
  pdl_wait();
  const int P = T * k;
  for (int p = blockIdx.x * blockDim.x + threadIdx.x; p < P; p += gridDim.x * blockDim.x) {
    const int j = p / T;
    const int t = p - j * T;
    const int q = t * k + j;
    const int e = topk_idx[q];
    const int local = slot[q];
    if (e < 0 || e >= N || local < 0) {
      slot[q] = -1;
      continue;
    }
    const int r = local + chunk_hist[static_cast<int64_t>(p / kSlotChunk) * N + e];
    slot[q] = r < cap ? r : -1;
  }
}

// ------------------------------------------------------------------ overflow: redirect
// Page «Архитектура MoE в больших языковых моделях — кто такие «эксперты»?», section «Как
// работает MoE: принцип маршрутизации»: a pair over its expert's capacity may be dropped or
// redirected to the next most suitable expert. Reading: arrivals in (choice, token) order; a
// pair whose expert is full goes to the token's best expert (largest logit, equal logits to
// the lower index) that has a free slot and that the token does not use yet; with none, it is
// dropped. topk_idx is rewritten with the serving expert; the router weights stay.
//
// Two launches. redirect_prefs_kernel (one warp per token, all SMs) writes each token's next
// kRedirectPrefs experts after its top-k, best first, as bytes (255 = none). The experts of
// the top-k never qualify later: each is either still the token's or was full when its pair
// arrived, and counts only grow. So the best qualifying expert is the first qualifying entry
// of the list, unless every entry fails and the list does not cover all the token's other
// experts; only then are the token's logits scanned.
//
// reroute_slots_kernel: each decision depends on all earlier ones, so one warp walks the
// arrivals in order, 32 at a time (lane l takes arrival a0 + l), and decides every pair of the
// window from the counts at its start: a pair whose expert has room targets it; otherwise
// the pair targets the first qualifying entry of its token's list (or is dropped). Lanes that
// target the same expert take consecutive slots in lane order. A lane's decision is the one
// the sequential rule makes as long as its target still has room after the earlier lanes'
// slots: experts that were full stay full, and a token's other pairs only change in the same
// window when T < 32, which also ends the window. So the window commits every lane before the
// first one whose slot is past the capacity (or that needs the full scan, or whose token is
// already in the window), and the next window starts there. A window's first lane always
// commits; when it needs the scan, the warp scans the token's logits for it alone. Once no
// expert has a free slot, the rest are dropped. The pairs come into shared memory with
// cp.async, and the lists stream through a ring of kRedirectRing rows refilled half a ring
// ahead of the walk, so the sequential path does not wait on global memory.
constexpr int kRedirectRing = 2048;

// Shared memory of the sequential pass: the list ring, the per-expert counts, every pair's
// serving expert as a byte (padded to 32) and a bit per pair for ids outside [0, N).
struct RerouteSmem {
  static __host__ __device__ size_t ex_bytes(int P) { return static_cast<size_t>((P + 31) / 32) * 32; }
  static __host__ __device__ size_t inv_bytes(int P) {
    return (static_cast<size_t>((P + 31) / 32) * 4 + 15) / 16 * 16;
  }
  static __host__ __device__ size_t bytes(int P) {
    return static_cast<size_t>(kRedirectRing) * kRedirectPrefs + 256 * 4 + ex_bytes(P) + inv_bytes(P);
  }
};

__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_newest_pending() {
  asm volatile("cp.async.wait_group 1;" ::: "memory");
}

// Lanes holding the same value v (0 <= v < 256) among the lanes where `on` holds.
__device__ __forceinline__ unsigned lanes_with_same(int v, bool on) {
  unsigned same = __ballot_sync(kFull, on);
#pragma unroll
  for (int b = 0; b < 8; ++b) {
    const bool bit = (v >> b) & 1;
    const unsigned m = __ballot_sync(kFull, bit);
    same &= bit ? m : ~m;
  }
  return same;
}

// Experts ranked k .. k + kRedirectPrefs - 1 in the token's order (logit descending, equal
// logits to the lower index, NaN as -inf), as bytes; 255 past the last expert.
// Also, for the sequential pass: every pair's expert as a byte (ex8) with a bit per pair for
// ids outside [0, N) (inv; such a pair is reported as MOE_ERR_BOUNDS and holds no expert), and
// every slot set to -1, so that the pass writes only the pairs it decides.
__global__ void __launch_bounds__(256) redirect_prefs_kernel(const float* __restrict__ logits,
                                                             uint8_t* __restrict__ prefs,
                                                             const int32_t* __restrict__ topk_idx,
                                                             uint8_t* __restrict__ ex8,
                                                             uint32_t* __restrict__ inv,
                                                             int32_t* __restrict__ slot, int T,
                                                             int N, int k, int* status) {
  pdl_wait();
  pdl_trigger();
  const int lane = static_cast<int>(lane_id());
  const int warps = gridDim.x * (blockDim.x / 32);
  {
    const int P = T * k;
    const int words = (P + 31) / 32;
    bool bad = false;
    for (int w = blockIdx.x * blockDim.x + threadIdx.x; w < words; w += gridDim.x * blockDim.x) {
      uint32_t bits = 0;
      uint32_t packed[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) packed[i] = 0;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int q = w * 32 + i;
        if (q >= P) break;
        const int e = topk_idx[q];
        const bool ok = e >= 0 && e < N;
        bad |= !ok;
        if (!ok) bits |= 1u << i;
        packed[i >> 2] |= static_cast<uint32_t>(ok ? e : 0) << (8 * (i & 3));
        slot[q] = -1;
      }
      uint4* dst = reinterpret_cast<uint4*>(ex8 + static_cast<int64_t>(w) * 32);
      dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
      inv[w] = bits;
    }
    if (bad) report_error(status, MOE_ERR_BOUNDS);
  }
  const int rounds = min(N, k + kRedirectPrefs);
  for (int t = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32; t < T; t += warps) {
    float val[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      const float v = e < N ? logits[static_cast<int64_t>(t) * N + e] : -INFINITY;
      val[i] = isnan(v) ? -INFINITY : v;
    }
    uint32_t taken = 0;
    int mine = 255;  // lane r < kRedirectPrefs keeps the expert of rank k + r
    for (int r = 0; r < rounds; ++r) {
      float bv = -INFINITY;
      int be = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        if (e < N && !((taken >> i) & 1u) && better(val[i], e, bv, be)) {
          bv = val[i];
          be = e;
        }
      }
      warp_best(bv, be);
      if ((be & 31) == lane) taken |= 1u << (be >> 5);
      if (r >= k && lane == r - k) mine = be;
    }
    if (lane < kRedirectPrefs)
      prefs[static_cast<int64_t>(t) * kRedirectPrefs + lane] = static_cast<uint8_t>(mine);
  }
}

// Lists of stream positions [from, to) (position a is token a mod T) into ring rows a mod
// kRedirectRing, one cp.async group.
__device__ __forceinline__ void stage_prefs(const uint8_t* prefs, uint8_t* ring, int from, int to,
                                            int T, int lane) {
  for (int a = from + lane; a < to; a += 32)
    cp_async_16(smem_u32(ring + (a % kRedirectRing) * kRedirectPrefs),
                prefs + static_cast<int64_t>(a % T) * kRedirectPrefs);
  cp_async_commit();
}

__global__ void __launch_bounds__(32) reroute_slots_kernel(const float* __restrict__ logits,
                                                           const uint8_t* __restrict__ prefs,
                                                           const uint8_t* __restrict__ ex8_g,
                                                           const uint32_t* __restrict__ inv_g,
                                                           int32_t* __restrict__ topk_idx,
                                                           int32_t* __restrict__ slot,
                                                           int32_t* __restrict__ expert_count,
                                                           int T, int N, int k, int cap) {
  extern __shared__ __align__(16) int r_sm[];
  const int P = T * k;
  uint8_t* ring = reinterpret_cast<uint8_t*>(r_sm);      // [ring][prefs]
  int* cnt = r_sm + kRedirectRing * kRedirectPrefs / 4;  // [256] filled slots
  uint8_t* ex8 = reinterpret_cast<uint8_t*>(cnt + 256);  // [P] serving experts, as bytes
  uint32_t* inv = reinterpret_cast<uint32_t*>(ex8 + RerouteSmem::ex_bytes(P));  // id outside [0, N)
  pdl_trigger();
  pdl_wait();
  const int lane = static_cast<int>(lane_id());
  {  // the pairs' experts and invalid bits (16-byte pieces, padded in global memory alike)
    const int n16 = static_cast<int>(RerouteSmem::ex_bytes(P) / 16);
    for (int i = lane; i < n16; i += 32) cp_async_16(smem_u32(ex8 + 16 * i), ex8_g + 16 * i);
    const int m16 = static_cast<int>(RerouteSmem::inv_bytes(P) / 16);
    const uint8_t* inv_src = reinterpret_cast<const uint8_t*>(inv_g);
    for (int i = lane; i < m16; i += 32) cp_async_16(smem_u32(inv) + 16 * i, inv_src + 16 * i);
    cp_async_commit();
  }
  // expert serving pair q, or -1 for an id outside [0, N)
  auto expert_of = [&](int q) -> int {
    return ((inv[q >> 5] >> (q & 31)) & 1u) ? -1 : static_cast<int>(ex8[q]);
  };
  constexpr int kHalf = kRedirectRing / 2;
  int filled = min(P, kHalf);  // lists of positions below `filled` are requested
  stage_prefs(prefs, ring, 0, filled, T, lane);
  int newest = 0;  // first position of the newest group
  if (filled < P) {
    newest = filled;
    stage_prefs(prefs, ring, filled, min(P, 2 * kHalf), T, lane);
    filled = min(P, 2 * kHalf);
  }
  for (int e = lane; e < 256; e += 32) cnt[e] = 0;
  const bool whole_list = N - k <= kRedirectPrefs;  // the list holds every other expert
  int room = cap > 0 ? N : 0;                       // experts with a free slot
  cp_async_wait_all();
  __syncwarp();
  int waited = filled;  // lists of positions below `waited` have landed
  int t = lane % T;     // token and choice of arrival a0 + lane
  int j = lane / T;
  int a0 = 0;           // first arrival not decided yet
  while (a0 < P) {
    if (room == 0) break;  // no free slot anywhere: the rest stay dropped (slot -1)
    if (filled < P && a0 >= filled - kHalf) {
      // the walk is past the older half: refill it with the next positions
      cp_async_wait_newest_pending();  // the group that last wrote those rows has landed
      waited = max(waited, newest);
      __syncwarp();
      newest = filled;
      stage_prefs(prefs, ring, filled, min(P, filled + kHalf), T, lane);
      filled = min(P, filled + kHalf);
    }
    const int n_act = min(32, P - a0);
    const bool act = lane < n_act;
    const int q = t * k + j;
    const int e = act ? expert_of(q) : -1;
    const bool valid = act && e >= 0 && e < N;
    const bool need = act && (!valid || cnt[e] >= cap);  // own expert full: search the list
    if (__any_sync(kFull, need) && a0 + n_act - 1 >= waited) {
      if (a0 + n_act - 1 >= newest) {
        cp_async_wait_all();
        waited = filled;
      } else {
        cp_async_wait_newest_pending();
        waited = newest;
      }
      __syncwarp();
    }
    int target = (act && !need) ? e : -1;
    bool scan = false;
    if (need && room > 0) {
      const uint4 row =
          *reinterpret_cast<const uint4*>(ring + ((a0 + lane) % kRedirectRing) * kRedirectPrefs);
      int own[8];  // the token's current experts
#pragma unroll
      for (int j2 = 0; j2 < 8; ++j2) own[j2] = j2 < k ? expert_of(t * k + j2) : -1;
      const uint32_t w4[4] = {row.x, row.y, row.z, row.w};
#pragma unroll
      for (int r = 0; r < kRedirectPrefs; ++r) {
        const int cand = (w4[r >> 2] >> (8 * (r & 3))) & 0xff;
        bool ok = cand < N && cnt[cand] < cap;
#pragma unroll
        for (int j2 = 0; j2 < 8; ++j2) ok &= own[j2] != cand;
        if (ok && target < 0) target = cand;
      }
      scan = target < 0 && !whole_list;
    }
    const unsigned same = lanes_with_same(target, target >= 0);
    const int c = target >= 0 ? cnt[target] + __popc(same & lanemask_lt()) : -1;
    bool dup = false;  // the token already has an earlier lane in this window
    if (T < 32) {
      const unsigned st = lanes_with_same(t, act);
      dup = (st & lanemask_lt()) != 0;
    }
    const unsigned bad = __ballot_sync(kFull, act && ((target >= 0 && c >= cap) || scan || dup));
    const int first = bad ? __ffs(bad) - 1 : n_act;
    __syncwarp();  // every lane has read cnt and ex before they change
    if (first == 0) {
      // the window's first pair needs a scan of its token's logits
      const int t0 = __shfl_sync(kFull, t, 0);
      const int q0 = __shfl_sync(kFull, q, 0);
      const float* lrow = logits + static_cast<int64_t>(t0) * N;
      float v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = (lane + 32 * i < N) ? lrow[lane + 32 * i] : -INFINITY;
      int used = 0;  // bit i: expert lane + 32 i is already one of the token's
      for (int j2 = 0; j2 < k; ++j2) {
        const int e2 = expert_of(t0 * k + j2);
        if (e2 >= 0 && e2 < N && (e2 & 31) == lane) used |= 1 << (e2 >> 5);
      }
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int c2 = lane + 32 * i;
        if (c2 < N && !((used >> i) & 1) && cnt[c2] < cap) {
          const float vi = isnan(v[i]) ? -INFINITY : v[i];
          if (better(vi, c2, bv, bi)) {
            bv = vi;
            bi = c2;
          }
        }
      }
      warp_best(bv, bi);
      const int out = bi != 0x7fffffff ? cnt[bi] : -1;
      if (out >= 0 && out + 1 == cap) --room;
      __syncwarp();
      if (lane == 0) {
        slot[q0] = out;
        if (out >= 0) {
          cnt[bi] = out + 1;
          ex8[q0] = static_cast<uint8_t>(bi);
          inv[q0 >> 5] &= ~(1u << (q0 & 31));
          topk_idx[q0] = bi;
        }
      }
      __syncwarp();
      a0 += 1;
      t += 1;
      while (t >= T) {
        t -= T;
        ++j;
      }
      continue;
    }
    const unsigned commit = first >= 32 ? kFull : ((1u << first) - 1);
    const bool mine = lane < first;
    const bool last = target >= 0 && ((same & commit) >> lane) == 1u;  // last lane on target
    if (mine) {
      slot[q] = target >= 0 ? c : -1;
      if (target >= 0 && target != e) {  // redirected: the serving expert changes
        ex8[q] = static_cast<uint8_t>(target);
        if (e < 0) atomicAnd(&inv[q >> 5], ~(1u << (q & 31)));
        topk_idx[q] = target;
      }
      if (last) cnt[target] = c + 1;
    }
    room -= __popc(__ballot_sync(kFull, mine && last && c + 1 == cap));
    __syncwarp();
    a0 += first;
    t += first;
    while (t >= T) {
      t -= T;
      ++j;
    }
  }
  cp_async_wait_all();
  __syncwarp();
  for (int e = lane; e < N; e += 32) expert_count[e] = cnt[e];
}

// ------------------------------------------------------------------ decode-sized batches
// One launch for T <= kDecodeRouteMaxT tokens (see dr::decode_route_body).
template <int TMAX, int EPT>
__global__ void __launch_bounds__(dr::kDrThreads) decode_route_kernel(const DecodeRouteArgs a) {
  __shared__ dr::DecodeRouteSmem<TMAX, EPT> sm;
  pdl_trigger();
  pdl_wait();
  const int ctas = static_cast<int>(gridDim.x);
  if (!dr::decode_route_partials<TMAX, EPT>(a, static_cast<int>(blockIdx.x), ctas, sm)) return;
  __threadfence();
  dr::decode_route_finish<TMAX, EPT>(a, ctas, sm, true);  // the last CTA to arrive
  if (threadIdx.x == 0) *a.counter = 0;  // every CTA has arrived
}

}  // namespace

// ------------------------------------------------------------------ launchers
cudaError_t launch_router_topk(const uint16_t* x, const float* w_router, const float* bias,
                               float* logits, int32_t* topk_idx, float* topk_w, int T, int d,
                               int N, int k, uint16_t* split_scratch, int* status,
                               uint64_t timeout_ns, cudaStream_t s, float* prob_part) {
  if (router_uses_tensor_cores(T, N, d))
    return launch_router_tc(x, w_router, bias, logits, topk_idx, topk_w, T, d, N, k,
                            split_scratch, status, timeout_ns, prob_part, s);
  auto kern = N <= 32 ? router_token_kernel<1> : N <= 64 ? router_token_kernel<2>
             : N <= 128 ? router_token_kernel<4> : router_token_kernel<8>;
  return launch_pdl(kern, dim3(T), dim3(kTokThreads), 0, s, x, w_router, bias, logits, topk_idx,
                    topk_w, T, d, N, k, prob_part);
}

cudaError_t launch_decode_route(const DecodeRouteArgs& a, cudaStream_t s) {
  if (!use_decode_route(a.T, a.N, a.d) || a.N > 256 || a.k > 8) return cudaErrorInvalidValue;
  const int ctas = (a.d + kDecodeSlice - 1) / kDecodeSlice;
  const int ept = a.N <= 32 ? 1 : a.N <= 64 ? 2 : a.N <= 128 ? 4 : 8;
  auto pick = [&](auto k1, auto k2, auto k4, auto k8) {
    return ept == 1 ? k1 : ept == 2 ? k2 : ept == 4 ? k4 : k8;
  };
  if (a.T <= 4)
    return launch_pdl(pick(decode_route_kernel<4, 1>, decode_route_kernel<4, 2>,
                           decode_route_kernel<4, 4>, decode_route_kernel<4, 8>),
                      dim3(ctas), dim3(dr::kDrThreads), 0, s, a);
  return launch_pdl(pick(decode_route_kernel<16, 1>, decode_route_kernel<16, 2>,
                         decode_route_kernel<16, 4>, decode_route_kernel<16, 8>),
                    dim3(ctas), dim3(dr::kDrThreads), 0, s, a);
}

cudaError_t launch_reroute_slots(const float* logits, uint8_t* scratch, int32_t* topk_idx,
                                int32_t* slot, int32_t* expert_count, int T, int N, int k,
                                int capacity, int* status, cudaStream_t s) {
  if (static_cast<int64_t>(T) * k > kRerouteMaxPairs || N > 256) return cudaErrorInvalidValue;
  static PerDeviceOnce once;
  const cudaError_t attr = once.run([] {
    return cudaFuncSetAttribute(
        reroute_slots_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
        static_cast<int>(RerouteSmem::bytes(static_cast<int>(kRerouteMaxPairs))));
  });
  if (attr != cudaSuccess) return attr;
  const int P = T * k;
  uint8_t* prefs = scratch;
  uint8_t* ex8 = prefs + redirect_round16(static_cast<int64_t>(T) * kRedirectPrefs);
  uint32_t* inv = reinterpret_cast<uint32_t*>(ex8 + RerouteSmem::ex_bytes(P));
  const int blocks = std::max(1, std::min((T + 7) / 8, 4 * 148));
  cudaError_t e = launch_pdl(redirect_prefs_kernel, dim3(blocks), dim3(256), 0, s, logits, prefs,
                             static_cast<const int32_t*>(topk_idx), ex8, inv, slot, T, N, k, status);
  if (e != cudaSuccess) return e;
  return launch_pdl(reroute_slots_kernel, dim3(1), dim3(32), RerouteSmem::bytes(P), s, logits,
                    static_cast<const uint8_t*>(prefs), static_cast<const uint8_t*>(ex8),
                    static_cast<const uint32_t*>(inv), topk_idx, slot, expert_count, T, N, k,
                    capacity);
}

cudaError_t launch_topk_from_logits(const float* logits, int32_t* topk_idx, float* topk_w, int T,
                                    int N, int k, cudaStream_t s) {
  const int blocks = (T + 7) / 8;
  auto kern = N <= 32 ? topk_from_logits_kernel<1> : N <= 64 ? topk_from_logits_kernel<2>
             : N <= 128 ? topk_from_logits_kernel<4> : topk_from_logits_kernel<8>;
  return launch_pdl(kern, dim3(blocks), dim3(256), 0, s, logits, topk_idx, topk_w, T, N, k);
}

cudaError_t launch_capacity_slots(const int32_t* topk_idx, int32_t* slot, int32_t* expert_count,
                                  int32_t* chunk_scratch, int T, int N, int k, int capacity,
                                  cudaStream_t s, const RouteStats* stats) {
  RouteStats st{};
  if (stats != nullptr) st = *stats;
  const int64_t P = static_cast<int64_t>(T) * k;
  const int n_chunks = static_cast<int>(slot_chunks(P));
  const int single = n_chunks == 1 ? 1 : 0;
  cudaError_t e = launch_pdl(slot_rank_kernel, dim3(n_chunks), dim3(kSlThreads), 0, s, topk_idx,
                             slot, chunk_scratch, expert_count, T, N, k, capacity, single, st);
  if (e != cudaSuccess || single) return e;
  e = launch_pdl(slot_scan_kernel, dim3(1), dim3(256), 0, s, chunk_scratch, expert_count, n_chunks,
                 T, N, capacity, st);
  if (e != cudaSuccess) return e;
  const int blocks = static_cast<int>(std::min<int64_t>((P + 255) / 256, 148 * 8));
  return launch_pdl(slot_finalize_kernel, dim3(blocks), dim3(256), 0, s, topk_idx, slot,
                    chunk_scratch, T, N, k, capacity);
}

}  // namespace moe
