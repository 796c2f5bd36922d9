// Routing of decode-sized batches in one pass over a few CTAs, and the warp-level top-k it
// shares with the other routing kernels. Used by the decode router kernel (moe_route,
// moe_forward, moe_route_noalloc).
//
// Page «Sparse Mixture-of-Experts» (bigdataschool wiki), «Роутер и top-k gating» (linear router,
// softmax, top-k, renormalisation) and «Expert capacity и capacity factor» (capacity slots,
// first come first served).
#pragma once

#include <math.h>

#include "common.cuh"
#include "launch.h"

namespace moe {
namespace dr {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ bool better(float av, int ae, float bv, int be) {
  return av > bv || (av == bv && ae < be);
}

// Best (value, expert) over the warp; every lane ends with the same pair.
__device__ __forceinline__ void warp_best(float& v, int& e) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(kFull, v, o);
    const int oe = __shfl_xor_sync(kFull, e, o);
    if (better(ov, oe, v, e)) {
      v = ov;
      e = oe;
    }
  }
}

// Top-k of one token whose N logits are spread over the warp: lane l holds experts l + 32 j.
// Lanes r < k write choice r. NaN logits are never preferred (unspecified input, but never
// an out-of-range expert index).
template <int EPT>
__device__ __forceinline__ void warp_topk_write(const float (&val)[EPT], int N, int k, int t,
                                                int32_t* topk_idx, float* topk_w) {
  const int lane = static_cast<int>(lane_id());
  uint32_t taken = 0;
  float sel_v[8];
  int sel_e[8];
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    sel_v[r] = 0.f;
    sel_e[r] = 0;
    if (r < k) {
      float bv = -INFINITY;
      int be = 0x7fffffff;
#pragma unroll
      for (int j = 0; j < EPT; ++j) {
        const int e = lane + 32 * j;
        const float v = isnan(val[j]) ? -INFINITY : val[j];
        if (e < N && !((taken >> j) & 1u) && better(v, e, bv, be)) {
          bv = v;
          be = e;
        }
      }
      warp_best(bv, be);
      if ((be & 31) == lane) taken |= 1u << (be >> 5);
      sel_v[r] = bv;
      sel_e[r] = be;
    }
  }
  // renormalised weights: softmax over the chosen logits (the largest is sel_v[0])
  float den = 0.f;
  float num[8];
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    num[r] = (r < k) ? expf(sel_v[r] - sel_v[0]) : 0.f;
    den += num[r];
  }
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    if (r < k && lane == r) {
      topk_idx[static_cast<int64_t>(t) * k + r] = sel_e[r];
      topk_w[static_cast<int64_t>(t) * k + r] = num[r] / den;
    }
  }
}

// Decode-sized batches (T <= kDecodeRouteMaxT). CTA c owns d columns [128 c, 128 c + 128): lane
// l holds 4 of them of every token's x, and warp w takes experts w, w + 8, ... one float4 of
// W_r per lane, so W_r is read once over all CTAs. Per (token, expert) the warp adds its
// lanes' products by a butterfly and stores the slice's partial dot product. The last CTA to
// arrive adds the partials in order of slice (deterministic), then runs top-k per token, the
// capacity slots in (choice, token) order and, if asked, the permutation.
constexpr int kDrThreads = 256;
constexpr int kDrWarps = kDrThreads / 32;

template <int TMAX, int EPT>
struct DecodeRouteSmem {
  float logit[TMAX][EPT * 32];
  int tidx[TMAX * 8];  // top-k, storage order t * k + j
  float tw[TMAX * 8];
  int pe[TMAX * 8];    // expert of arrival p = j * T + t
  int row[TMAX * 8];   // row of arrival p, -1 if dropped
  int cnt[256];
  int off[257];
  int warp[kDrWarps];
  int last;
  float term[256];  // router statistics: (picks_e / T) * P_e
};

// Phase 1: CTA `cta` of the `ctas` CTAs that split d stores its slice's partial dot products
// and counts its arrival (all kDrThreads threads of the CTA take part). Returns true in the CTA
// that arrived last.
template <int TMAX, int EPT>
__device__ __forceinline__ bool decode_route_partials(const DecodeRouteArgs& a, int cta, int ctas,
                                                      DecodeRouteSmem<TMAX, EPT>& sm) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int T = a.T, N = a.N, d = a.d;
  const int c0 = cta * kDecodeSlice + lane * 4;
  const bool col_ok = c0 < d;

  float xv[TMAX][4];
#pragma unroll
  for (int t = 0; t < TMAX; ++t) {
    uint2 u = make_uint2(0u, 0u);
    if (t < T && col_ok) u = __ldg(reinterpret_cast<const uint2*>(a.x + static_cast<int64_t>(t) * d + c0));
    xv[t][0] = __uint_as_float(u.x << 16);
    xv[t][1] = __uint_as_float(u.x & 0xffff0000u);
    xv[t][2] = __uint_as_float(u.y << 16);
    xv[t][3] = __uint_as_float(u.y & 0xffff0000u);
  }
  float* part = a.part + static_cast<int64_t>(cta) * T * N;
  for (int e0 = warp; e0 < N; e0 += 4 * kDrWarps) {
    float4 w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {  // four experts' loads in flight before any is used
      const int e = e0 + i * kDrWarps;
      w[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (e < N && col_ok) w[i] = __ldg(reinterpret_cast<const float4*>(a.w_router + static_cast<int64_t>(e) * d + c0));
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = e0 + i * kDrWarps;
      if (e >= N) break;  // warp-uniform
#pragma unroll
      for (int t = 0; t < TMAX; ++t) {
        if (t >= T) break;  // warp-uniform
        float acc = xv[t][0] * w[i].x;
        acc = fmaf(xv[t][1], w[i].y, acc);
        acc = fmaf(xv[t][2], w[i].z, acc);
        acc = fmaf(xv[t][3], w[i].w, acc);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
        if (lane == 0) part[t * N + e] = acc;
      }
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) sm.last = atomicAdd(a.counter, 1) == ctas - 1;
  __syncthreads();
  return sm.last != 0;
}

// Phase 2, once every slice's partial dot products are stored: the logits (slices added in
// order), top-k with the renormalised weights, the capacity slots in (choice, token) order, the
// kept counts, the expert offsets and the rows of the kept pairs; all of it in shared memory
// (sm). With `write` the CTA also stores the routing's outputs to global memory, and when the
// permute outputs are given the offsets, the row maps and the x_perm copy as well.
template <int TMAX, int EPT>
__device__ __forceinline__ void decode_route_finish(const DecodeRouteArgs& a, int ctas,
                                                    DecodeRouteSmem<TMAX, EPT>& sm, bool write) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int T = a.T, N = a.N, d = a.d, k = a.k;
  const int S = ctas;
  for (int i = tid; i < T * N; i += kDrThreads) {
    const int t = i / N, e = i - t * N;
    const float* src = a.part + static_cast<int64_t>(t) * N + e;
    const int64_t stride = static_cast<int64_t>(T) * N;
    // slices added in order of c; each group's 16 loads are issued before any is used, so the
    // L2 round trips overlap instead of following one another
    float L = 0.f;
    int c = 0;
    for (; c + 16 <= S; c += 16) {
      float v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) v[u] = __ldcg(src + (c + u) * stride);
#pragma unroll
      for (int u = 0; u < 16; ++u) L += v[u];
    }
    if (c < S) {
      float v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) v[u] = c + u < S ? __ldcg(src + (c + u) * stride) : 0.f;
#pragma unroll
      for (int u = 0; u < 16; ++u)
        if (c + u < S) L += v[u];
    }
    if (a.bias != nullptr) L += a.bias[e];
    sm.logit[t][e] = L;
    if (write) a.logits[static_cast<int64_t>(t) * N + e] = L;
  }
  __syncthreads();
  for (int t = warp; t < T; t += kDrWarps) {
    float val[EPT];
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
      const int e = lane + 32 * j;
      val[j] = (e < N) ? sm.logit[t][e] : -INFINITY;
    }
    warp_topk_write<EPT>(val, N, k, t, sm.tidx, sm.tw);
  }
  __syncthreads();

  const int P = T * k;  // <= 8 * TMAX arrivals
  if (tid < P) {
    const int j = tid / T, t = tid - j * T;
    sm.pe[tid] = sm.tidx[t * k + j];
    if (write) {
      a.topk_idx[t * k + j] = sm.tidx[t * k + j];
      a.topk_w[t * k + j] = sm.tw[t * k + j];
    }
  }
  __syncthreads();
  int my_slot = -1, my_e = -1, my_q = 0;
  if (tid < P) {
    const int j = tid / T, t = tid - j * T;
    my_q = t * k + j;
    my_e = sm.pe[tid];
    int r = 0;
    for (int p2 = 0; p2 < tid; ++p2) r += sm.pe[p2] == my_e;
    my_slot = r < a.cap ? r : -1;
    if (write) a.slot[my_q] = my_slot;
  }
  const bool stats = write && a.st_picks != nullptr;
  if (stats) {
    // router statistics: each token's softmax over the experts, in place of its logits (they
    // are stored and no longer needed), warp per token
    for (int t = warp; t < T; t += kDrWarps) {
      float v[EPT];
      float m = -INFINITY;
#pragma unroll
      for (int j = 0; j < EPT; ++j) {
        const int e = lane + 32 * j;
        v[j] = e < N ? sm.logit[t][e] : -INFINITY;
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
      for (int j = 0; j < EPT; ++j)
        if (lane + 32 * j < N) sm.logit[t][lane + 32 * j] = v[j] * inv;
    }
    __syncthreads();
  }
  for (int e = tid; e < N; e += kDrThreads) {
    int c = 0;
    for (int p2 = 0; p2 < P; ++p2) c += sm.pe[p2] == e;
    if (stats) {  // picks before the capacity; P_e, the batch mean of the probability
      float sum = 0.f;
      for (int t = 0; t < T; ++t) sum += sm.logit[t][e];
      const float Pe = sum / static_cast<float>(T);
      a.st_picks[e] = c;
      a.st_prob_mean[e] = Pe;
      sm.term[e] = (static_cast<float>(c) / static_cast<float>(T)) * Pe;
    }
    c = min(c, a.cap);
    sm.cnt[e] = c;
    if (write) a.expert_count[e] = c;
  }
  __syncthreads();
  if (stats && tid == 0) {
    float total = 0.f;
    int kept = 0;
    for (int e = 0; e < N; ++e) {
      total += sm.term[e];
      kept += sm.cnt[e];
    }
    *a.st_aux_loss = a.st_alpha * static_cast<float>(N) * total;
    *a.st_dropped = P - kept;
  }
  // exclusive prefix of the kept counts (N <= 256 = blockDim.x)
  const int v = tid < N ? sm.cnt[tid] : 0;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) sm.warp[warp] = incl;
  __syncthreads();
  int base = 0;
  for (int i = 0; i < warp; ++i) base += sm.warp[i];
  sm.off[tid + 1] = base + incl;
  if (tid == 0) sm.off[0] = 0;
  __syncthreads();
  const bool permute = write && a.x_perm != nullptr;
  if (permute)
    for (int i = tid; i <= N; i += kDrThreads) a.expert_offset[i] = sm.off[i];
  if (tid < P) {
    const int row = my_slot >= 0 ? sm.off[my_e] + my_slot : -1;
    if (permute) {
      a.row_of_pair[my_q] = row;
      if (row >= 0) a.pair_of_row[row] = my_q;
    }
    sm.row[tid] = row;
  }
  __syncthreads();
  if (permute) {
    const int nv = d / 8;  // 16-byte vectors per row
    for (int i = tid; i < P * nv; i += kDrThreads) {
      const int p2 = i / nv, vv = i - p2 * nv;
      const int row = sm.row[p2];
      if (row < 0) continue;
      const int t = p2 % T;
      const uint4 val = reinterpret_cast<const uint4*>(a.x + static_cast<int64_t>(t) * d)[vv];
      reinterpret_cast<uint4*>(a.x_perm + static_cast<int64_t>(row) * d)[vv] = val;
    }
  }
}

}  // namespace dr
}  // namespace moe
