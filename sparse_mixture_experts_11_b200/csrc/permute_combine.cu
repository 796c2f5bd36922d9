// Sort-by-expert permutation and the weighted combine back to token order.
//
// Permute (page «Что такое Mixture of Experts (MoE) в трансформерах», section «Бэкенд для
// экспертов», grouped_mm): tokens are sorted by expert id and grouped so that one grouped GEMM
// covers every expert. Expert e owns rows [offset[e], offset[e+1]) with offset the exclusive
// prefix sum of the kept counts; a kept pair (t, j) with slot s sits in row offset[e] + s, so
// rows inside an expert follow arrival order.
//
// Combine (page «Sparse Mixture-of-Experts», sections «Роутер и top-k gating» and «Expert
// capacity и capacity factor»): out[t] = residual[t] + sum_j w[t, j] * y[row(t, j)] over the
// kept choices j in ascending order, accumulated in fp32 and rounded once; dropped pairs add
// nothing and a token with no kept pair passes the residual through bit for bit.
#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace moe {
namespace {

constexpr unsigned kFull = 0xffffffffu;

// Exclusive prefix sum of count[0..N) into s_off[0..N] (N <= 256, blockDim.x == 256).
__device__ __forceinline__ void block_offsets_256(const int32_t* __restrict__ count, int N,
                                                  int* s_off, int* s_warp) {
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  int v = (tid < N) ? count[tid] : 0;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) s_warp[w] = incl;
  __syncthreads();
  int base = 0;
  for (int i = 0; i < w; ++i) base += s_warp[i];
  s_off[tid + 1] = base + incl;
  if (tid == 0) s_off[0] = 0;
  __syncthreads();
}

__global__ void __launch_bounds__(256) permute_kernel(
    const uint16_t* __restrict__ x, const int32_t* __restrict__ topk_idx,
    const int32_t* __restrict__ slot, const int32_t* __restrict__ expert_count,
    int32_t* __restrict__ expert_offset, int32_t* __restrict__ row_of_pair,
    int32_t* __restrict__ pair_of_row, uint16_t* __restrict__ x_perm, int T, int d, int N, int k,
    int64_t r_max, int* status) {
  __shared__ int s_off[257];
  __shared__ int s_warp[8];
  block_offsets_256(expert_count, N, s_off, s_warp);
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i <= N; i += blockDim.x) expert_offset[i] = s_off[i];

  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const int nv = d / 8;  // 16-byte vectors per row
  for (int t = blockIdx.x * warps + (threadIdx.x >> 5); t < T; t += gridDim.x * warps) {
    int row = -1;
    if (lane < k) {
      const int64_t q = static_cast<int64_t>(t) * k + lane;
      const int s = slot[q];
      const int e = topk_idx[q];
      if (s >= 0 && e >= 0 && e < N) {
        row = s_off[e] + s;
        if (row >= s_off[e + 1] || row >= r_max) {
          report_error(status, MOE_ERR_BOUNDS);
          row = -1;
        }
      }
      row_of_pair[q] = row;
      if (row >= 0) pair_of_row[row] = static_cast<int32_t>(q);
    }
    int rows[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) rows[j] = __shfl_sync(kFull, row, j);
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(t) * d);
    for (int c = lane; c < nv; c += 32) {
      const uint4 v = src[c];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < k && rows[j] >= 0)
          reinterpret_cast<uint4*>(x_perm + static_cast<int64_t>(rows[j]) * d)[c] = v;
      }
    }
  }
}

__global__ void __launch_bounds__(256) combine_kernel(
    const float* __restrict__ y, const int32_t* __restrict__ row_of_pair,
    const float* __restrict__ topk_w, const uint16_t* residual, void* out, int out_f32, int T,
    int d, int k, int64_t r_max, int* status) {
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const int nq = d / 4;  // groups of 4 columns
  for (int t = blockIdx.x * warps + (threadIdx.x >> 5); t < T; t += gridDim.x * warps) {
    int row = -1;
    float w = 0.f;
    if (lane < k) {
      const int64_t q = static_cast<int64_t>(t) * k + lane;
      row = row_of_pair[q];
      w = topk_w[q];
      if (row >= r_max) {
        report_error(status, MOE_ERR_BOUNDS);
        row = -1;
      }
    }
    const bool any_kept = __ballot_sync(kFull, row >= 0) != 0;
    int rows[8];
    float ws[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      rows[j] = __shfl_sync(kFull, row, j);
      ws[j] = __shfl_sync(kFull, w, j);
    }
    const uint2* res = residual ? reinterpret_cast<const uint2*>(residual + static_cast<int64_t>(t) * d) : nullptr;
    for (int c = lane; c < nq; c += 32) {
      uint2 rbits = make_uint2(0u, 0u);
      if (res) rbits = res[c];
      if (!any_kept) {  // residual passes through unchanged
        if (out_f32) {
          float4 o;
          o.x = __uint_as_float(rbits.x << 16);
          o.y = __uint_as_float(rbits.x & 0xffff0000u);
          o.z = __uint_as_float(rbits.y << 16);
          o.w = __uint_as_float(rbits.y & 0xffff0000u);
          reinterpret_cast<float4*>(static_cast<float*>(out) + static_cast<int64_t>(t) * d)[c] = o;
        } else {
          reinterpret_cast<uint2*>(static_cast<uint16_t*>(out) + static_cast<int64_t>(t) * d)[c] = rbits;
        }
        continue;
      }
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < k && rows[j] >= 0) {
          const float4 v = reinterpret_cast<const float4*>(y + static_cast<int64_t>(rows[j]) * d)[c];
          a0 = fmaf(ws[j], v.x, a0);
          a1 = fmaf(ws[j], v.y, a1);
          a2 = fmaf(ws[j], v.z, a2);
          a3 = fmaf(ws[j], v.w, a3);
        }
      }
      const float o0 = __uint_as_float(rbits.x << 16) + a0;
      const float o1 = __uint_as_float(rbits.x & 0xffff0000u) + a1;
      const float o2 = __uint_as_float(rbits.y << 16) + a2;
      const float o3 = __uint_as_float(rbits.y & 0xffff0000u) + a3;
      if (out_f32) {
        reinterpret_cast<float4*>(static_cast<float*>(out) + static_cast<int64_t>(t) * d)[c] =
            make_float4(o0, o1, o2, o3);
      } else {
        reinterpret_cast<uint2*>(static_cast<uint16_t*>(out) + static_cast<int64_t>(t) * d)[c] =
            make_uint2(pack_bf16x2(o0, o1), pack_bf16x2(o2, o3));
      }
    }
  }
}

}  // namespace

cudaError_t launch_permute(const uint16_t* x, const int32_t* topk_idx, const int32_t* slot,
                           const int32_t* expert_count, int32_t* expert_offset,
                           int32_t* row_of_pair, int32_t* pair_of_row, uint16_t* x_perm, int T,
                           int d, int N, int k, int64_t r_max, int* status, cudaStream_t s) {
  DeviceInfo di;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  const int blocks = std::max(1, std::min((T + 7) / 8, di.sm_count * 8));
  permute_kernel<<<blocks, 256, 0, s>>>(x, topk_idx, slot, expert_count, expert_offset,
                                        row_of_pair, pair_of_row, x_perm, T, d, N, k, r_max, status);
  return cudaGetLastError();
}

cudaError_t launch_combine(const float* y_perm, const int32_t* row_of_pair, const float* topk_w,
                           const uint16_t* residual, void* out, int out_f32, int T, int d, int k,
                           int64_t r_max, int* status, cudaStream_t s) {
  DeviceInfo di;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  const int blocks = std::max(1, std::min((T + 7) / 8, di.sm_count * 8));
  combine_kernel<<<blocks, 256, 0, s>>>(y_perm, row_of_pair, topk_w, residual, out, out_f32, T, d,
                                        k, r_max, status);
  return cudaGetLastError();
}

}  // namespace moe
