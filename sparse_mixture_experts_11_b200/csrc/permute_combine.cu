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

// Block (token t, chunk c): the block's first warp turns token t's k (expert, slot) pairs
// into rows; the token's chunk-0 block also records row_of_pair / pair_of_row. Then each
// thread copies one 16-byte vector of x[t] (chunk c) into every kept row. Many blocks per
// token keep small batches from being latency-bound; expert offsets are rebuilt per block
// from the N <= 256 kept counts.
constexpr int kVecPerBlock = 256;  // 16-byte vectors per block (4 KB of a bf16 row)

__global__ void __launch_bounds__(256) permute_kernel(
    const uint16_t* __restrict__ x, const int32_t* __restrict__ topk_idx,
    const int32_t* __restrict__ slot, const int32_t* __restrict__ expert_count,
    int32_t* __restrict__ expert_offset, int32_t* __restrict__ row_of_pair,
    int32_t* __restrict__ pair_of_row, uint16_t* __restrict__ x_perm, int T, int d, int N, int k,
    int64_t r_max, int* status) {
  __shared__ int s_off[257];
  __shared__ int s_warp[8];
  __shared__ int s_rows[8];
  pdl_trigger();
  pdl_wait();
  block_offsets_256(expert_count, N, s_off, s_warp);
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i <= N; i += blockDim.x) expert_offset[i] = s_off[i];

  const int nv = d / 8;  // 16-byte vectors per row
  const int chunks = (nv + kVecPerBlock - 1) / kVecPerBlock;
  const int64_t items = static_cast<int64_t>(T) * chunks;
  for (int64_t item = blockIdx.x; item < items; item += gridDim.x) {
    const int t = static_cast<int>(item / chunks);
    const int c = static_cast<int>(item - static_cast<int64_t>(t) * chunks);
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
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
        if (c == 0) {
          row_of_pair[q] = row;
          if (row >= 0) pair_of_row[row] = static_cast<int32_t>(q);
        }
        s_rows[lane] = row;
      }
    }
    __syncthreads();
    bool any = false;  // a token whose every pair was dropped has nothing to copy
    for (int j = 0; j < k; ++j) any |= s_rows[j] >= 0;
    const int v = c * kVecPerBlock + threadIdx.x;
    if (any && v < nv) {
      const uint4 val = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(t) * d)[v];
      for (int j = 0; j < k; ++j) {
        const int row = s_rows[j];
        if (row >= 0) reinterpret_cast<uint4*>(x_perm + static_cast<int64_t>(row) * d)[v] = val;
      }
    }
    __syncthreads();
  }
}

// Warp per item (token t, group g of 512 columns), grid-stride: lanes j < k read the token's
// pair j (its y_perm row and router weight; a row at or past R_max is skipped and reported),
// shared with the warp by shuffles, and each lane then handles 16 columns, one float4 of each
// kept row of y_perm and 4 bf16 of the residual for each of four 128-column steps (coalesced
// across the warp). The next item's pairs are read before this item's rows, so the dependent
// loads of consecutive items overlap; warps need no block-wide barrier. Per column the sum is
// the kept choices' w_j * y in ascending j (fp32 fma from zero), then plus the residual, rounded
// once; a token with no kept pair passes the residual's bits through.
constexpr int kCombCols = 512;

__device__ __forceinline__ void combine_pair(const int32_t* __restrict__ row_of_pair,
                                             const float* __restrict__ topk_w, int64_t t, int k,
                                             int64_t r_max, int lane, int* status, int& row,
                                             float& w) {
  row = -1;
  w = 0.f;
  if (lane < k) {
    const int64_t q = t * k + lane;
    row = row_of_pair[q];
    w = topk_w[q];
    if (row >= r_max) {
      report_error(status, MOE_ERR_BOUNDS);
      row = -1;
    }
  }
}

constexpr int kCombBlocksPerSm = 4;

__global__ void __launch_bounds__(256, kCombBlocksPerSm) combine_kernel(
    const float* __restrict__ y, const int32_t* __restrict__ row_of_pair,
    const float* __restrict__ topk_w, const uint16_t* residual, void* out, int out_f32, int T,
    int d, int k, int64_t r_max, int* status) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int groups = (d + kCombCols - 1) / kCombCols;
  const int64_t items = static_cast<int64_t>(T) * groups;
  int64_t item = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  int row_n = -1;
  float w_n = 0.f;
  if (item < items) combine_pair(row_of_pair, topk_w, item / groups, k, r_max, lane, status, row_n, w_n);
  for (; item < items; item += nwarps) {
    const int row = row_n;
    const float w = w_n;
    const int64_t next = item + nwarps;
    if (next < items) combine_pair(row_of_pair, topk_w, next / groups, k, r_max, lane, status, row_n, w_n);
    const int64_t t = item / groups;
    const int g = static_cast<int>(item - t * groups);
    int rows[8];
    float ws[8];
    bool any = false;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      rows[j] = __shfl_sync(kFull, row, j);
      ws[j] = __shfl_sync(kFull, w, j);
      if (j >= k) rows[j] = -1;
      any |= rows[j] >= 0;
    }
#pragma unroll 2
    for (int i = 0; i < kCombCols / 128; ++i) {
      const int col = g * kCombCols + i * 128 + lane * 4;
      if (col >= d) continue;
      uint2 rbits = make_uint2(0u, 0u);
      if (residual != nullptr) rbits = *reinterpret_cast<const uint2*>(residual + t * d + col);
      const float r0 = __uint_as_float(rbits.x << 16), r1 = __uint_as_float(rbits.x & 0xffff0000u);
      const float r2 = __uint_as_float(rbits.y << 16), r3 = __uint_as_float(rbits.y & 0xffff0000u);
      if (!any) {  // every choice dropped: the residual passes through unchanged
        if (out_f32)
          *reinterpret_cast<float4*>(static_cast<float*>(out) + t * d + col) = make_float4(r0, r1, r2, r3);
        else
          *reinterpret_cast<uint2*>(static_cast<uint16_t*>(out) + t * d + col) = rbits;
        continue;
      }
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {  // ascending choice order
        if (rows[j] < 0) continue;
        const float4 v = *reinterpret_cast<const float4*>(y + static_cast<int64_t>(rows[j]) * d + col);
        a0 = fmaf(ws[j], v.x, a0);
        a1 = fmaf(ws[j], v.y, a1);
        a2 = fmaf(ws[j], v.z, a2);
        a3 = fmaf(ws[j], v.w, a3);
      }
      const float o0 = r0 + a0, o1 = r1 + a1, o2 = r2 + a2, o3 = r3 + a3;
      if (out_f32)
        *reinterpret_cast<float4*>(static_cast<float*>(out) + t * d + col) = make_float4(o0, o1, o2, o3);
      else
        *reinterpret_cast<uint2*>(static_cast<uint16_t*>(out) + t * d + col) =
            make_uint2(pack_bf16x2(o0, o1), pack_bf16x2(o2, o3));
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
  const int64_t items = static_cast<int64_t>(T) * ((d / 8 + kVecPerBlock - 1) / kVecPerBlock);
  const int blocks = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(items, di.sm_count * 16)));
  return launch_pdl(permute_kernel, dim3(blocks), dim3(256), 0, s, x, topk_idx, slot, expert_count,
                    expert_offset, row_of_pair, pair_of_row, x_perm, T, d, N, k, r_max, status);
}

cudaError_t launch_combine(const float* y_perm, const int32_t* row_of_pair, const float* topk_w,
                           const uint16_t* residual, void* out, int out_f32, int T, int d, int k,
                           int64_t r_max, int* status, cudaStream_t s) {
  DeviceInfo di;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  const int64_t warps = static_cast<int64_t>(T) * ((d + kCombCols - 1) / kCombCols);
  const int blocks = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((warps + 7) / 8, di.sm_count * kCombBlocksPerSm)));
  return launch_pdl(combine_kernel, dim3(blocks), dim3(256), 0, s, y_perm, row_of_pair, topk_w,
                    residual, out, out_f32, T, d, k, r_max, status);
}

}  // namespace moe
