// Router statistics and the auxiliary load-balancing loss.
//
// Page «Sparse Mixture-of-Experts», section «Маршрутизация токена и auxiliary loss»: the loss
// is alpha * N * sum_i f_i * P_i, where f_i is the fraction of the batch's tokens sent to
// expert i and P_i the router's mean probability for expert i over the batch (alpha = 1e-2
// is the value the page reports as best). f_i counts a token once for each of its chosen
// experts (picks_i / T), before the capacity limit; P_i averages the full softmax over N.
//
// Two deterministic passes (no floating-point atomics):
//   1. one block per 64 tokens: warp per token computes the softmax (max, exp, sum by warp
//      shuffles) and adds the probabilities into per-warp registers; the block adds the warps'
//      sums in warp order and writes a partial row; picks and drops are integer counts;
//   2. one block adds the partial rows in block order and forms the loss.
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace moe {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kStatTok = 64;  // tokens per block in pass 1
constexpr int kStatThreads = 256;
constexpr int kStatWarps = kStatThreads / 32;

template <int EPT>
__global__ void __launch_bounds__(kStatThreads) stats_partial_kernel(
    const float* __restrict__ logits, const int32_t* __restrict__ topk_idx,
    const int32_t* __restrict__ slot, float* __restrict__ part_prob, int* __restrict__ part_picks,
    int* __restrict__ part_dropped, int T, int N, int k) {
  __shared__ float s_acc[kStatWarps][EPT * 32];
  __shared__ int s_picks[EPT * 32];
  __shared__ int s_dropped;
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = threadIdx.x; e < EPT * 32; e += kStatThreads) s_picks[e] = 0;
  if (threadIdx.x == 0) s_dropped = 0;
  pdl_wait();
  __syncthreads();
  float acc[EPT];
#pragma unroll
  for (int j = 0; j < EPT; ++j) acc[j] = 0.f;
  const int t_begin = blockIdx.x * kStatTok;
  const int t_end = min(T, t_begin + kStatTok);
  int dropped = 0;
  for (int t = t_begin + warp; t < t_end; t += kStatWarps) {
    float v[EPT];
    float m = -INFINITY;
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
      const int e = lane + 32 * j;
      v[j] = e < N ? logits[static_cast<int64_t>(t) * N + e] : -INFINITY;
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
    for (int j = 0; j < EPT; ++j) acc[j] += v[j] * inv;
    if (lane < k) {
      const int64_t q = static_cast<int64_t>(t) * k + lane;
      const int e = topk_idx[q];
      if (e >= 0 && e < N) atomicAdd(&s_picks[e], 1);
      if (slot[q] < 0) ++dropped;
    }
  }
#pragma unroll
  for (int j = 0; j < EPT; ++j) s_acc[warp][lane + 32 * j] = acc[j];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) dropped += __shfl_xor_sync(kFull, dropped, o);
  if (lane == 0) atomicAdd(&s_dropped, dropped);
  __syncthreads();
  for (int e = threadIdx.x; e < N; e += kStatThreads) {
    float s = 0.f;
    for (int w = 0; w < kStatWarps; ++w) s += s_acc[w][e];  // warp order: deterministic
    part_prob[static_cast<int64_t>(blockIdx.x) * N + e] = s;
    part_picks[static_cast<int64_t>(blockIdx.x) * N + e] = s_picks[e];
  }
  if (threadIdx.x == 0) part_dropped[blockIdx.x] = s_dropped;
}

__global__ void __launch_bounds__(256) stats_final_kernel(
    const float* __restrict__ part_prob, const int* __restrict__ part_picks,
    const int* __restrict__ part_dropped, int n_parts, int T, int N, float alpha,
    int32_t* __restrict__ picks, float* __restrict__ prob_mean, float* __restrict__ aux_loss,
    int32_t* __restrict__ dropped) {
  __shared__ float s_term[256];
  pdl_trigger();
  pdl_wait();
  for (int e = threadIdx.x; e < 256; e += blockDim.x) s_term[e] = 0.f;
  for (int e = threadIdx.x; e < N; e += blockDim.x) {
    float s = 0.f;
    int c = 0;
    // block order (deterministic); eight independent loads in flight per step
    int b = 0;
    for (; b + 8 <= n_parts; b += 8) {
      float v[8];
      int u[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        v[i] = part_prob[static_cast<int64_t>(b + i) * N + e];
        u[i] = part_picks[static_cast<int64_t>(b + i) * N + e];
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        s += v[i];
        c += u[i];
      }
    }
    for (; b < n_parts; ++b) {
      s += part_prob[static_cast<int64_t>(b) * N + e];
      c += part_picks[static_cast<int64_t>(b) * N + e];
    }
    const float P = s / static_cast<float>(T);
    prob_mean[e] = P;
    picks[e] = c;
    s_term[e] = (static_cast<float>(c) / static_cast<float>(T)) * P;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float total = 0.f;
    for (int e = 0; e < N; ++e) total += s_term[e];
    int d = 0;
    for (int b2 = 0; b2 < n_parts; ++b2) d += part_dropped[b2];
    *aux_loss = alpha * static_cast<float>(N) * total;
    *dropped = d;
  }
}

}  // namespace

size_t router_stats_scratch_bytes(int T, int N) {
  const int64_t parts = (T + kStatTok - 1) / kStatTok;
  return static_cast<size_t>(parts) * (2 * N + 1) * 4;
}

cudaError_t launch_router_stats(const float* logits, const int32_t* topk_idx, const int32_t* slot,
                                float alpha, int32_t* picks, float* prob_mean, float* aux_loss,
                                int32_t* dropped, void* scratch, int T, int N, int k,
                                cudaStream_t s) {
  const int parts = (T + kStatTok - 1) / kStatTok;
  float* part_prob = static_cast<float*>(scratch);
  int* part_picks = reinterpret_cast<int*>(part_prob + static_cast<int64_t>(parts) * N);
  int* part_dropped = part_picks + static_cast<int64_t>(parts) * N;
  auto kern = N <= 32 ? stats_partial_kernel<1> : N <= 64 ? stats_partial_kernel<2>
            : N <= 128 ? stats_partial_kernel<4> : stats_partial_kernel<8>;
  cudaError_t e = launch_pdl(kern, dim3(parts), dim3(kStatThreads), 0, s, logits, topk_idx, slot,
                             part_prob, part_picks, part_dropped, T, N, k);
  if (e != cudaSuccess) return e;
  return launch_pdl(stats_final_kernel, dim3(1), dim3(256), 0, s, part_prob, part_picks,
                    part_dropped, parts, T, N, alpha, picks, prob_mean, aux_loss, dropped);
}

}  // namespace moe
