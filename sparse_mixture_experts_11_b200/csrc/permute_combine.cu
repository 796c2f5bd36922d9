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

// Both kernels give one warp a token and a range of its 256-column groups (the token split
// into `parts` ranges so that small batches still occupy every SM). Lanes j < k read the
// token's pair j once and share it by shuffles; a lane then handles 8 columns of each group,
// with the loads of four groups (permute) or two (combine) issued before any of them is used.
constexpr int kGroupCols = 256;  // columns per warp step: 8 per lane
constexpr int kGroupsInFlight = 4;  // permute
constexpr int kCombInFlight = 2;    // combine: its fp32 sums take the registers
constexpr int kCopyInFlight = 6;    // combine of a token with no kept pair: a plain copy

__device__ __forceinline__ void token_part(int64_t item, int parts, int groups, int& t, int& g0,
                                           int& g1) {
  t = static_cast<int>(item / parts);
  const int p = static_cast<int>(item - static_cast<int64_t>(t) * parts);
  g0 = p * groups / parts;
  g1 = (p + 1) * groups / parts;
}

// Permute: the warp turns token t's k (expert, slot) pairs into rows (the first part also
// records row_of_pair / pair_of_row) and copies its columns of x[t] into every kept row.
// Expert offsets are rebuilt per block from the N <= 256 kept counts.
__global__ void __launch_bounds__(256) permute_kernel(
    const uint16_t* __restrict__ x, const int32_t* __restrict__ topk_idx,
    const int32_t* __restrict__ slot, const int32_t* __restrict__ expert_count,
    int32_t* __restrict__ expert_offset, int32_t* __restrict__ row_of_pair,
    int32_t* __restrict__ pair_of_row, uint16_t* __restrict__ x_perm, int T, int d, int N, int k,
    int parts, int64_t r_max, int* status) {
  __shared__ int s_off[257];
  __shared__ int s_warp[8];
  pdl_trigger();
  pdl_wait();
  block_offsets_256(expert_count, N, s_off, s_warp);
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i <= N; i += blockDim.x) expert_offset[i] = s_off[i];

  const int lane = threadIdx.x & 31;
  const int groups = (d + kGroupCols - 1) / kGroupCols;
  const int64_t items = static_cast<int64_t>(T) * parts;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t item = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       item < items; item += nwarps) {
    int t, g0, g1;
    token_part(item, parts, groups, t, g0, g1);
    int row = -1;
    if (lane < k) {
      const int64_t q = static_cast<int64_t>(t) * k + lane;
      const int sl = slot[q];
      const int e = topk_idx[q];
      if (sl >= 0 && e >= 0 && e < N) {
        row = s_off[e] + sl;
        if (row >= s_off[e + 1] || row >= r_max) {
          report_error(status, MOE_ERR_BOUNDS);
          row = -1;
        }
      }
      if (g0 == 0) {
        row_of_pair[q] = row;
        if (row >= 0) pair_of_row[row] = static_cast<int32_t>(q);
      }
    }
    int rows[8];
    bool any = false;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      rows[j] = __shfl_sync(kFull, row, j);
      if (j >= k) rows[j] = -1;
      any |= rows[j] >= 0;
    }
    if (!any) continue;  // a token whose every pair was dropped has nothing to copy
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(t) * d);
    for (int g = g0; g < g1; g += kGroupsInFlight) {
      uint4 v[kGroupsInFlight];
#pragma unroll
      for (int i = 0; i < kGroupsInFlight; ++i) {
        const int col = (g + i) * kGroupCols + lane * 8;
        if (g + i < g1 && col < d) v[i] = src[col / 8];
      }
#pragma unroll
      for (int i = 0; i < kGroupsInFlight; ++i) {
        const int col = (g + i) * kGroupCols + lane * 8;
        if (g + i >= g1 || col >= d) continue;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (rows[j] >= 0) reinterpret_cast<uint4*>(x_perm + static_cast<int64_t>(rows[j]) * d)[col / 8] = v[i];
      }
    }
  }
}

// Combine: per column the sum is the kept choices' w_j * y in ascending j (fp32 fma from zero),
// then plus the residual, rounded once; a row at or past R_max is skipped and reported; a token
// with no kept pair passes the residual's bits through.
constexpr int kCombBlocksPerSm = 4;

__global__ void __launch_bounds__(256, kCombBlocksPerSm) combine_kernel(
    const float* __restrict__ y, const int32_t* __restrict__ row_of_pair,
    const float* __restrict__ topk_w, const uint16_t* residual, void* out, int out_f32, int T,
    int d, int k, int parts, int64_t r_max, int* status) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int groups = (d + kGroupCols - 1) / kGroupCols;
  const int64_t items = static_cast<int64_t>(T) * parts;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t item = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       item < items; item += nwarps) {
    int t, g0, g1;
    token_part(item, parts, groups, t, g0, g1);
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
    const int nkept = __popc(__ballot_sync(kFull, lane < k && row >= 0));
    const uint4* res = reinterpret_cast<const uint4*>(residual + static_cast<int64_t>(t) * d);
    if (nkept == 0) {
      // every choice dropped: the residual passes through unchanged, six groups in flight
      for (int g = g0; g < g1; g += kCopyInFlight) {
        uint4 rb[kCopyInFlight];
#pragma unroll
        for (int i = 0; i < kCopyInFlight; ++i) {
          const int col = (g + i) * kGroupCols + lane * 8;
          rb[i] = make_uint4(0u, 0u, 0u, 0u);
          if (residual != nullptr && g + i < g1 && col < d) rb[i] = res[col / 8];
        }
#pragma unroll
        for (int i = 0; i < kCopyInFlight; ++i) {
          const int col = (g + i) * kGroupCols + lane * 8;
          if (g + i >= g1 || col >= d) continue;
          const int64_t o = static_cast<int64_t>(t) * d + col;
          if (out_f32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out) + o);
            dst[0] = make_float4(__uint_as_float(rb[i].x << 16), __uint_as_float(rb[i].x & 0xffff0000u),
                                 __uint_as_float(rb[i].y << 16), __uint_as_float(rb[i].y & 0xffff0000u));
            dst[1] = make_float4(__uint_as_float(rb[i].z << 16), __uint_as_float(rb[i].z & 0xffff0000u),
                                 __uint_as_float(rb[i].w << 16), __uint_as_float(rb[i].w & 0xffff0000u));
          } else {
            *reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + o) = rb[i];
          }
        }
      }
      continue;
    }
    for (int g = g0; g < g1; g += kCombInFlight) {
      uint4 rb[kCombInFlight];
#pragma unroll
      for (int i = 0; i < kCombInFlight; ++i) {
        const int col = (g + i) * kGroupCols + lane * 8;
        rb[i] = make_uint4(0u, 0u, 0u, 0u);
        if (residual != nullptr && g + i < g1 && col < d) rb[i] = res[col / 8];
      }
      float acc[kCombInFlight][8];
#pragma unroll
      for (int i = 0; i < kCombInFlight; ++i)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[i][c] = 0.f;
      if (nkept > 0) {
        for (int j = 0; j < k; ++j) {  // ascending choice order
          const int rj = __shfl_sync(kFull, row, j);
          const float wj = __shfl_sync(kFull, w, j);
          if (rj < 0) continue;
          const float* yr = y + static_cast<int64_t>(rj) * d;
          float4 a[kCombInFlight], b[kCombInFlight];
#pragma unroll
          for (int i = 0; i < kCombInFlight; ++i) {
            const int col = (g + i) * kGroupCols + lane * 8;
            if (g + i < g1 && col < d) {
              a[i] = *reinterpret_cast<const float4*>(yr + col);
              b[i] = *reinterpret_cast<const float4*>(yr + col + 4);
            }
          }
#pragma unroll
          for (int i = 0; i < kCombInFlight; ++i) {
            acc[i][0] = fmaf(wj, a[i].x, acc[i][0]);
            acc[i][1] = fmaf(wj, a[i].y, acc[i][1]);
            acc[i][2] = fmaf(wj, a[i].z, acc[i][2]);
            acc[i][3] = fmaf(wj, a[i].w, acc[i][3]);
            acc[i][4] = fmaf(wj, b[i].x, acc[i][4]);
            acc[i][5] = fmaf(wj, b[i].y, acc[i][5]);
            acc[i][6] = fmaf(wj, b[i].z, acc[i][6]);
            acc[i][7] = fmaf(wj, b[i].w, acc[i][7]);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < kCombInFlight; ++i) {
        const int col = (g + i) * kGroupCols + lane * 8;
        if (g + i >= g1 || col >= d) continue;
        const uint32_t rw[4] = {rb[i].x, rb[i].y, rb[i].z, rb[i].w};
        float r[8];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          r[2 * c] = __uint_as_float(rw[c] << 16);
          r[2 * c + 1] = __uint_as_float(rw[c] & 0xffff0000u);
        }
        const int64_t o = static_cast<int64_t>(t) * d + col;
        if (out_f32) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out) + o);
          if (nkept == 0) {  // every choice dropped: the residual passes through unchanged
            dst[0] = make_float4(r[0], r[1], r[2], r[3]);
            dst[1] = make_float4(r[4], r[5], r[6], r[7]);
          } else {
            dst[0] = make_float4(r[0] + acc[i][0], r[1] + acc[i][1], r[2] + acc[i][2], r[3] + acc[i][3]);
            dst[1] = make_float4(r[4] + acc[i][4], r[5] + acc[i][5], r[6] + acc[i][6], r[7] + acc[i][7]);
          }
        } else {
          uint4 ov = rb[i];
          if (nkept > 0)
            ov = make_uint4(pack_bf16x2(r[0] + acc[i][0], r[1] + acc[i][1]), pack_bf16x2(r[2] + acc[i][2], r[3] + acc[i][3]),
                            pack_bf16x2(r[4] + acc[i][4], r[5] + acc[i][5]), pack_bf16x2(r[6] + acc[i][6], r[7] + acc[i][7]));
          *reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + o) = ov;
        }
      }
    }
  }
}

// Token parts: enough warps for every SM (about 32 warps of work each), at most one part per
// 256-column group.
int parts_for(int64_t T, int d, int sm_count) {
  const int groups = (d + kGroupCols - 1) / kGroupCols;
  const int64_t target = static_cast<int64_t>(sm_count) * 32;
  int64_t parts = T > 0 ? (target + T - 1) / T : 1;
  if (parts > groups) parts = groups;
  return parts < 1 ? 1 : static_cast<int>(parts);
}

}  // namespace

cudaError_t launch_permute(const uint16_t* x, const int32_t* topk_idx, const int32_t* slot,
                           const int32_t* expert_count, int32_t* expert_offset,
                           int32_t* row_of_pair, int32_t* pair_of_row, uint16_t* x_perm, int T,
                           int d, int N, int k, int64_t r_max, int* status, cudaStream_t s) {
  DeviceInfo di;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  const int parts = parts_for(T, d, di.sm_count);
  const int64_t warps = static_cast<int64_t>(T) * parts;
  const int blocks = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((warps + 7) / 8, di.sm_count * 8)));
  return launch_pdl(permute_kernel, dim3(blocks), dim3(256), 0, s, x, topk_idx, slot, expert_count,
                    expert_offset, row_of_pair, pair_of_row, x_perm, T, d, N, k, parts, r_max, status);
}

cudaError_t launch_combine(const float* y_perm, const int32_t* row_of_pair, const float* topk_w,
                           const uint16_t* residual, void* out, int out_f32, int T, int d, int k,
                           int64_t r_max, int* status, cudaStream_t s) {
  DeviceInfo di;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  const int parts = parts_for(T, d, di.sm_count);
  const int64_t warps = static_cast<int64_t>(T) * parts;
  const int blocks = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((warps + 7) / 8, di.sm_count * kCombBlocksPerSm)));
  return launch_pdl(combine_kernel, dim3(blocks), dim3(256), 0, s, y_perm, row_of_pair, topk_w,
                    residual, out, out_f32, T, d, k, parts, r_max, status);
}

}  // namespace moe
