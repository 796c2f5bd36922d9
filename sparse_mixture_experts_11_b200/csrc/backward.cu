// Backward pass of the sparse MoE layer on sm_100a.
//
// The pages discuss training MoE layers with grouped-GEMM kernels (page «Что такое Mixture of
// Experts (MoE) в трансформерах», section «Обучение MoE с помощью Transformers») and print no
// gradient formulas; these kernels compute the chain rule of the forward pass:
//   out[t] = residual[t] + sum over kept j of w[t, j] y[row(t, j)],   y = h W_d^T,
//   h = silu(x W_g^T) (x W_u^T) (SwiGLU) or gelu(x W_1^T) (GELU),
//   w[t] = softmax of the chosen logits, L = x W_r^T (+ b).
// The choice of experts and the capacity slots pass no gradient. Steps, on one stream:
//   1 bwd_pairs_kernel      dy[row] = w[t, j] d_out[t] (bf16), dw[t, j] = <d_out[t], y[row]>,
//                           dL[t, i] = w_i (dw_i - sum_j w_j dw_j) on the chosen experts
//   2 bwd_gemm (rows)       pre = x_perm W_gu^T                (fp32, recomputed)
//   3 bwd_gemm (rows)       dh = dy W_d                        (W_d read MN-major)
//   4 act_bwd_kernel        d_pre = dh * act'(pre) (bf16), h = act(pre) (bf16)
//   5 bwd_gemm (rows)       dx_rows = d_pre W_gu               (W_gu read MN-major)
//   6 bwd_gemm (wgrad)      dW_d[e] = dy_e^T h_e               (both operands MN-major)
//   7 bwd_gemm (wgrad)      dW_gu[e] = d_pre_e^T x_e           (both operands MN-major)
//   8 router_wgrad kernels  dW_r = dL^T x, db = sum_t dL[t]    (fp32, fixed summation order)
//   9 bwd_dx_kernel         dx[t] = sum over kept j of dx_rows[row] + sum_j dL[t, idx_j] W_r[idx_j]
//
// bwd_gemm_kernel is persistent, one CTA per SM striding through 128 x 256 output tiles on
// tcgen05 (192 threads: TMA producer, MMA issuer, four epilogue warps; four 48 KB stages;
// two fp32 accumulators in TMEM, so one tile's epilogue overlaps the next one's loads and
// MMAs). Each operand is K-major (the contiguous axis is the reduction axis) or MN-major (the
// contiguous axis is the output's row or column axis), so the transposed products read the
// weights and the activations where they lie: an MN-major operand comes as 64 x 64 TMA boxes
// (128 bytes of the MN axis by 64 k rows, 128B-swizzled) and the MMA reads it through an
// MN-major shared-memory descriptor with the instruction's transpose bit set. Rows mode: the
// tile's rows are an expert's rows of the permuted batch and K is fixed. Weight-gradient mode:
// the tile is a block of an expert's [M, n_out] gradient and K runs over the expert's rows;
// the last k block is cut at the expert's end by zeroing the rows past it in shared memory.
// The epilogue sends each warp's 32 x 32 fp32 block out as one TMA store. Every wait is
// bounded; on timeout the CTA records MOE_ERR_TIMEOUT and drains what it issued.
#include <math.h>
#include <string.h>

#include <algorithm>

#include "common.cuh"
#include "launch.h"
#include "tma_host.h"

namespace moe {
namespace {

constexpr int kBM = 128;  // UMMA M
constexpr int kBN = 256;  // UMMA N
constexpr int kBK = 64;   // k per stage: 64 bf16, one 128-byte swizzle row
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK * 2;
constexpr int kBBytes = kBN * kBK * 2;
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kGemmThreads = 192;
constexpr int kStoreStage = 32 * 32 * 4;  // one epilogue warp's 32 x 32 fp32 block
constexpr int kGemmSmem = kStages * kStageBytes + 4 * kStoreStage + 1024;
constexpr int kBox = 64 * 64 * 2;  // one MN-major TMA box: 64 MN x 64 k rows, 8 KB

enum { GEMM_ROWS = 0, GEMM_WGRAD = 1 };

struct BwdGemmParams {
  const int32_t* expert_offset;  // [N + 1]
  int n_experts;
  int M;          // weight-gradient mode: rows of each expert's output block
  int n_out;      // output columns (a multiple of 16)
  int num_kb;     // rows mode: K / 64
  int r_max;      // rows of the permuted batch's buffers
  float* out;     // rows mode: [r_max, n_out]; weight-gradient mode: [N, M, n_out]
  int* status;
  uint64_t timeout_ns;
};

// Shared-memory descriptor of a 128B-swizzled MN-major operand: 8 k rows of 128 bytes (64 MN
// elements) form a 1024-byte group (stride-dimension offset); successive 64-element MN blocks
// are one TMA box (8 KB) apart (leading-dimension offset).
__device__ __forceinline__ uint64_t smem_desc_mn_sw128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(kBox >> 4) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

struct GemmTile {
  int e;     // expert
  int m0;    // rows mode: first row of the permuted batch; weight-gradient mode: first output row
  int rows;  // rows mode: valid rows of the tile; weight-gradient mode: the expert's rows (K)
  int k0;    // weight-gradient mode: the expert's first row (start of K)
  int n0;    // first output column
  int nkb;   // k blocks
};

// Tile t of the CTA-strided list. Rows mode: t = m-tile * n_tiles_n + n-tile, m-tiles numbered
// expert by expert (s_mt: each expert's first m-tile, s_off: its first row). Weight-gradient
// mode: t = (expert * m_tiles + m-tile) * n_tiles_n + n-tile.
template <int MODE>
__device__ __forceinline__ GemmTile decode_gemm_tile(int t, const BwdGemmParams& p, int n_tiles_n,
                                                     int m_tiles, const int* s_mt,
                                                     const int* s_off) {
  GemmTile c;
  const int nt = t % n_tiles_n;
  c.n0 = nt * kBN;
  if (MODE == GEMM_ROWS) {
    const int gm = t / n_tiles_n;
    int lo = 0, hi = p.n_experts;  // last e with s_mt[e] <= gm
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s_mt[mid] <= gm) lo = mid;
      else hi = mid;
    }
    c.e = lo;
    c.m0 = s_off[lo] + (gm - s_mt[lo]) * kBM;
    c.rows = min(kBM, s_off[lo + 1] - c.m0);
    c.k0 = 0;
    c.nkb = p.num_kb;
  } else {
    const int em = t / n_tiles_n;
    c.e = em / m_tiles;
    c.m0 = (em - c.e * m_tiles) * kBM;
    c.k0 = s_off[c.e];
    c.rows = s_off[c.e + 1] - c.k0;
    c.nkb = (c.rows + kBK - 1) / kBK;
  }
  return c;
}

template <bool A_MN, bool B_MN, int MODE>
__global__ void __launch_bounds__(kGemmThreads, 1)
    bwd_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmC, const BwdGemmParams p) {
  extern __shared__ __align__(1024) uint8_t dyn_smem[];
  __shared__ __align__(8) uint64_t full_bar[kStages];
  __shared__ __align__(8) uint64_t empty_bar[kStages];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t done_bar;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  __shared__ int s_mt[257];  // rows mode: first m-tile of each expert; s_mt[N] = all m-tiles
  __shared__ int s_off[257];
  __shared__ int s_tiles;

  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t tiles = (smem_u32(dyn_smem) + 1023u) & ~1023u;
  const int N = p.n_experts;
  if (threadIdx.x == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    prefetch_tensormap(&tmC);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&tfull_bar[b]), 1);
      mbar_init(smem_u32(&tempty_bar[b]), kGemmThreads - 64);
    }
    mbar_init(smem_u32(&done_bar), 1);
    s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&s_tmem), 2 * kBN);
    tmem_relinquish();
  }
  pdl_wait();
  const int n_tiles_n = (p.n_out + kBN - 1) / kBN;
  const int m_tiles = (p.M + kBM - 1) / kBM;  // weight-gradient mode
  if (warp == 0) {
    // per-expert offsets (and, rows mode, m-tile counts and their prefix); experts
    // lane * per .. lane * per + per - 1 on this lane
    const int per = (N + 31) / 32;
    int cnt[8];
    int sum = 0;
    bool bad = false;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      cnt[i] = 0;
      const int e = lane * per + i;
      if (i < per && e < N) {
        const int a = p.expert_offset[e], b = p.expert_offset[e + 1];
        s_off[e] = a;
        if (a < 0 || b < a || b > p.r_max) bad = true;
        else cnt[i] = (b - a + kBM - 1) / kBM;
        sum += cnt[i];
      }
    }
    if (lane == 31) s_off[N] = p.expert_offset[N];
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    int run = incl - sum;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane * per + i;
      if (i < per && e < N) {
        s_mt[e] = run;
        run += cnt[i];
      }
    }
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 31) {
      s_mt[N] = incl;
      s_tiles = bad ? 0 : (MODE == GEMM_ROWS ? incl * n_tiles_n : N * m_tiles * n_tiles_n);
      if (bad) report_error(p.status, MOE_ERR_BOUNDS);
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const int total = s_tiles;
  const uint32_t tmem = s_tmem;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_last();
      bool ok = true;
      int it = 0;
      for (int t = blockIdx.x; ok && t < total; t += gridDim.x) {
        const GemmTile c = decode_gemm_tile<MODE>(t, p, n_tiles_n, m_tiles, s_mt, s_off);
        for (int kb = 0; kb < c.nkb; ++kb, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(smem_u32(&empty_bar[s]), ((it / kStages) & 1) ^ 1u, p.timeout_ns, &s_abort)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&full_bar[s]);
          const uint32_t a_dst = tiles + s * kStageBytes, b_dst = a_dst + kABytes;
          mbar_arrive_expect_tx(fb, kStageBytes);
          if (!A_MN) {
            tma_load_2d(a_dst, &tmA, fb, kb * kBK, c.m0, pol);
          } else {
#pragma unroll
            for (int i = 0; i < kBM / 64; ++i)
              tma_load_2d(a_dst + i * kBox, &tmA, fb, c.m0 + 64 * i, c.k0 + kb * kBK, pol);
          }
          if (!B_MN) {
            tma_load_3d(b_dst, &tmB, fb, kb * kBK, c.n0, c.e, pol);
          } else if (MODE == GEMM_ROWS) {
#pragma unroll
            for (int i = 0; i < kBN / 64; ++i)
              tma_load_3d(b_dst + i * kBox, &tmB, fb, c.n0 + 64 * i, kb * kBK, c.e, pol);
          } else {
#pragma unroll
            for (int i = 0; i < kBN / 64; ++i)
              tma_load_2d(b_dst + i * kBox, &tmB, fb, c.n0 + 64 * i, c.k0 + kb * kBK, pol);
          }
        }
      }
      if (!ok) {
        s_abort = 1;
        report_error(p.status, MOE_ERR_TIMEOUT);
      }
      // no TMA write may still be landing in shared memory when the CTA exits
      for (int i = max(0, it - kStages); i < it; ++i)
        mbar_wait(smem_u32(&full_bar[i % kStages]), (i / kStages) & 1, kDrainTimeoutNs, nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN) | (A_MN ? (1u << 15) : 0u) |
                               (B_MN ? (1u << 16) : 0u);
    bool ok = true;
    bool issued = false;
    int it = 0, uc = 0;
    for (int t = blockIdx.x; ok && t < total; t += gridDim.x) {
      const GemmTile c = decode_gemm_tile<MODE>(t, p, n_tiles_n, m_tiles, s_mt, s_off);
      if (c.nkb == 0) continue;  // no rows: the epilogue writes zeros
      const int buf = uc & 1;
      const bool free_buf = mbar_wait(smem_u32(&tempty_bar[buf]), ((uc >> 1) & 1) ^ 1u, p.timeout_ns, &s_abort);
      if (!__all_sync(0xffffffffu, free_buf)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const uint32_t d_tmem = tmem + static_cast<uint32_t>(buf * kBN);
      for (int kb = 0; kb < c.nkb; ++kb, ++it) {
        const int s = it % kStages;
        const bool got = mbar_wait(smem_u32(&full_bar[s]), (it / kStages) & 1, p.timeout_ns, &s_abort);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        const uint32_t a_base = tiles + s * kStageBytes, b_base = a_base + kABytes;
        const int valid = c.rows - kb * kBK;
        if (MODE == GEMM_WGRAD && valid < kBK) {
          // the expert's rows end inside this k block: zero k rows [valid, 64) of every box
          uint8_t* st = dyn_smem + (a_base - smem_u32(dyn_smem));
          const int lines = kBK - valid;
          const int boxes = kBM / 64 + kBN / 64;
          for (int i = lane; i < boxes * lines * 8; i += 32) {
            const int box = i / (lines * 8), rem = i - box * lines * 8;
            const int line = valid + rem / 8, chunk = rem & 7;
            const uint32_t off = (box < kBM / 64 ? box * kBox : kABytes + (box - kBM / 64) * kBox) +
                                 line * 128 + chunk * 16;
            *reinterpret_cast<uint4*>(st + off) = make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();  // generic stores -> visible to the tensor core
          __syncwarp();
        }
        tc_fence_after_sync();
        if (lane == 0) {
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t da = A_MN ? smem_desc_mn_sw128(a_base + kk * 2048)
                                     : smem_desc_k_sw128(a_base + kk * 32);
            const uint64_t db = B_MN ? smem_desc_mn_sw128(b_base + kk * 2048)
                                     : smem_desc_k_sw128(b_base + kk * 32);
            tc_mma_f16(d_tmem, da, db, idesc, (kb != 0 || kk != 0) ? 1u : 0u);
          }
          tc_commit(smem_u32(&empty_bar[s]));
        }
        issued = true;
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) tc_commit(smem_u32(&tfull_bar[buf]));
      ++uc;
    }
    if (!ok && lane == 0) {
      s_abort = 1;
      report_error(p.status, MOE_ERR_TIMEOUT);
    }
    // every issued MMA has finished before TMEM is freed, also when the epilogue gave up on
    // a tile whose MMAs this warp had already issued
    if (issued && lane == 0) {
      tc_commit(smem_u32(&done_bar));
      mbar_wait(smem_u32(&done_bar), 0, kDrainTimeoutNs, nullptr);
    }
  } else {
    // ------------------------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;  // TMEM lane quadrant of this warp
    const uint32_t stg_addr = tiles + kStages * kStageBytes + (warp - 2) * kStoreStage;
    uint8_t* const stg = dyn_smem + (stg_addr - smem_u32(dyn_smem));
    int uc = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      const GemmTile c = decode_gemm_tile<MODE>(t, p, n_tiles_n, m_tiles, s_mt, s_off);
      const bool have = c.nkb > 0;
      const int buf = uc & 1;
      if (have) {
        const bool got = mbar_wait(smem_u32(&tfull_bar[buf]), (uc >> 1) & 1, p.timeout_ns, &s_abort);
        if (!__all_sync(0xffffffffu, got)) {
          s_abort = 1;
          report_error(p.status, MOE_ERR_TIMEOUT);
          break;
        }
        tc_fence_after_sync();
      }
      // rows q*32 .. q*32+31 of the tile, 32 columns at a time through this warp's block of
      // shared memory. A block whose 32 rows all exist leaves as one TMA store (128B-swizzled:
      // row r's 16-byte chunk j sits at chunk j ^ (r & 7)); the rows of an expert's last, partial
      // m-tile go out as plain stores, each instruction one row's 128 bytes.
      int row_lim;  // rows of this warp's 32 that exist
      float* base;  // row q*32 of the tile
      if (MODE == GEMM_ROWS) {
        row_lim = min(32, c.rows - q * 32);
        base = p.out + (static_cast<int64_t>(c.m0) + q * 32) * p.n_out;
      } else {
        row_lim = min(32, p.M - c.m0 - q * 32);
        base = p.out + (static_cast<int64_t>(c.e) * p.M + c.m0 + q * 32) * p.n_out;
      }
      const uint32_t t_row = tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(buf * kBN);
#pragma unroll 1
      for (int cc = 0; cc < kBN; cc += 32) {
        if (c.n0 + cc >= p.n_out) break;  // warp-uniform: ragged last n-tile
        uint32_t v[32];
        if (have) {
          tmem_ld_32x32b_x32(t_row + cc, v);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0u;  // an expert with no rows: zero gradient
        }
        if (lane == 0) tma_store_wait_read();  // the last store has read this warp's block
        __syncwarp();
        if (row_lim >= 32) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint4*>(stg + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
          fence_proxy_async_smem();  // generic stores -> visible to the TMA engine
          __syncwarp();
          if (lane == 0) {
            if (MODE == GEMM_ROWS) tma_store_2d(&tmC, stg_addr, c.n0 + cc, c.m0 + q * 32);
            else tma_store_3d(&tmC, stg_addr, c.n0 + cc, c.m0 + q * 32, c.e);
            tma_store_commit();
          }
        } else if (row_lim > 0) {
          // element i of row r at r * 32 + (i ^ r): conflict-free both ways
          float* f = reinterpret_cast<float*>(stg);
#pragma unroll
          for (int i = 0; i < 32; ++i) f[lane * 32 + (i ^ lane)] = __uint_as_float(v[i]);
          __syncwarp();
          const int col = c.n0 + cc + lane;
          if (col < p.n_out)
            for (int r = 0; r < row_lim; ++r) base[static_cast<int64_t>(r) * p.n_out + col] = f[r * 32 + (lane ^ r)];
          __syncwarp();
        }
      }
      if (have) {
        tc_fence_before_sync();
        mbar_arrive(smem_u32(&tempty_bar[buf]));  // TMEM buffer free for the tile after next
        ++uc;
      }
    }
    if (lane == 0) tma_store_wait_all();  // every store of this warp has landed
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, 2 * kBN);
  }
}

// ------------------------------------------------------------------ combine and router step
// Warp per token. For each kept choice j: dy[row] = bf16(w_j d_out[t]) and
// dw_j = <d_out[t], y[row]> (fp32); dropped choices have dw_j = 0. Then the renormalised
// softmax's gradient on the chosen logits, dL_i = w_i (dw_i - sum_j w_j dw_j); the row of dL
// is written whole (zeros on the other experts).
__global__ void __launch_bounds__(256) bwd_pairs_kernel(
    const uint16_t* __restrict__ d_out, const float* __restrict__ y_perm,
    const float* __restrict__ topk_w, const int32_t* __restrict__ topk_idx,
    const int32_t* __restrict__ row_of_pair, uint16_t* __restrict__ dy_perm,
    float* __restrict__ d_logits, int T, int d, int N, int k, int r_max, int* status) {
  pdl_wait();
  pdl_trigger();
  const int lane = static_cast<int>(lane_id());
  const int warps = gridDim.x * (blockDim.x / 32);
  for (int t = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32; t < T; t += warps) {
    int row[8], idx[8];
    float w[8], acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      row[j] = -1;
      idx[j] = -1;
      w[j] = 0.f;
      acc[j] = 0.f;
      if (j < k) {
        row[j] = row_of_pair[t * k + j];
        idx[j] = topk_idx[t * k + j];
        w[j] = topk_w[t * k + j];
        if (row[j] >= r_max) {
          if (lane == 0) report_error(status, MOE_ERR_BOUNDS);
          row[j] = -1;
        }
      }
    }
    for (int c = lane * 8; c < d; c += 256) {
      const uint4 g4 = *reinterpret_cast<const uint4*>(d_out + static_cast<int64_t>(t) * d + c);
      const uint32_t gw[4] = {g4.x, g4.y, g4.z, g4.w};
      float g[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        g[2 * i] = __uint_as_float(gw[i] << 16);
        g[2 * i + 1] = __uint_as_float(gw[i] & 0xffff0000u);
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (row[j] < 0) continue;
        const float4* yr = reinterpret_cast<const float4*>(y_perm + static_cast<int64_t>(row[j]) * d + c);
        const float4 y0 = yr[0], y1 = yr[1];
        acc[j] += g[0] * y0.x + g[1] * y0.y + g[2] * y0.z + g[3] * y0.w + g[4] * y1.x +
                  g[5] * y1.y + g[6] * y1.z + g[7] * y1.w;
        uint4 o;
        o.x = pack_bf16x2(w[j] * g[0], w[j] * g[1]);
        o.y = pack_bf16x2(w[j] * g[2], w[j] * g[3]);
        o.z = pack_bf16x2(w[j] * g[4], w[j] * g[5]);
        o.w = pack_bf16x2(w[j] * g[6], w[j] * g[7]);
        *reinterpret_cast<uint4*>(dy_perm + static_cast<int64_t>(row[j]) * d + c) = o;
      }
    }
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
      s += w[j] * acc[j];  // w[j] = 0 past k
    }
    for (int n = lane; n < N; n += 32) {
      float v = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (idx[j] == n) v = w[j] * (acc[j] - s);
      d_logits[static_cast<int64_t>(t) * N + n] = v;
    }
  }
}

// ------------------------------------------------------------------ activation backward
// Row r of the permuted batch (r < R = expert_offset[N]), 4 columns per thread:
//   SwiGLU  pre = [g | u]: h = silu(g) u, d_pre = [dh u silu'(g) | dh silu(g)],
//           silu'(g) = s (1 + g (1 - s)), s = 1 / (1 + exp(-g));
//   GELU    h = z Phi(z), d_pre = dh (Phi(z) + z phi(z)) (exact erf form).
// h and d_pre are rounded once to bf16 (operands of the weight-gradient GEMMs).
__global__ void __launch_bounds__(256) act_bwd_kernel(const float* __restrict__ pre,
                                                      const float* __restrict__ dh,
                                                      const int32_t* __restrict__ expert_offset,
                                                      uint16_t* __restrict__ d_pre,
                                                      uint16_t* __restrict__ h, int N, int F,
                                                      int swiglu) {
  pdl_wait();
  pdl_trigger();
  const int R = expert_offset[N];
  const int n_gu = swiglu ? 2 * F : F;
  const int64_t items = static_cast<int64_t>(R) * (F / 4);
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < items;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / (F / 4);
    const int c = static_cast<int>(i - r * (F / 4)) * 4;
    const float4 d4 = *reinterpret_cast<const float4*>(dh + r * F + c);
    const float4 z4 = *reinterpret_cast<const float4*>(pre + r * n_gu + c);
    const float dv[4] = {d4.x, d4.y, d4.z, d4.w};
    const float zv[4] = {z4.x, z4.y, z4.z, z4.w};
    float hv[4], da[4], du[4];
    if (swiglu) {
      const float4 u4 = *reinterpret_cast<const float4*>(pre + r * n_gu + F + c);
      const float uv[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float sg = 1.0f / (1.0f + expf(-zv[q]));
        const float sl = zv[q] * sg;
        hv[q] = sl * uv[q];
        da[q] = dv[q] * uv[q] * (sg * (1.0f + zv[q] * (1.0f - sg)));
        du[q] = dv[q] * sl;
      }
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float Phi = 0.5f * (1.0f + erff(zv[q] * 0.7071067811865476f));
        const float phi = expf(-0.5f * zv[q] * zv[q]) * 0.3989422804014327f;
        hv[q] = zv[q] * Phi;
        da[q] = dv[q] * (Phi + zv[q] * phi);
        du[q] = 0.f;
      }
    }
    *reinterpret_cast<uint2*>(h + r * F + c) = make_uint2(pack_bf16x2(hv[0], hv[1]), pack_bf16x2(hv[2], hv[3]));
    *reinterpret_cast<uint2*>(d_pre + r * n_gu + c) =
        make_uint2(pack_bf16x2(da[0], da[1]), pack_bf16x2(da[2], da[3]));
    if (swiglu)
      *reinterpret_cast<uint2*>(d_pre + r * n_gu + F + c) =
          make_uint2(pack_bf16x2(du[0], du[1]), pack_bf16x2(du[2], du[3]));
  }
}

// ------------------------------------------------------------------ router weight gradient
// dW_r = dL^T x in fp32, in two passes with a fixed summation order: chunk c of the tokens
// adds its tokens in order into part[c][n][col] (thread = column, 16 experts a block), then
// the chunks are added in order. dL is zero except on each token's k chosen experts (the
// renormalised weights depend on those logits only), so a block adds only the tokens with a
// chosen expert among its 16: the same sums in the same order, without the terms that are
// exactly zero. db[n] = sum_t dL[t, n]: warp w of a block adds tokens
// t = w mod 32 in order for 32 experts, and the 32 warp sums are added in warp order.
constexpr int kRwExperts = 16;
constexpr int kRwTokens = 64;

__global__ void __launch_bounds__(256) router_wgrad_partial_kernel(
    const float* __restrict__ d_logits, const uint16_t* __restrict__ x, float* __restrict__ part,
    int T, int d, int N, int chunk) {
  __shared__ float s_dl[kRwTokens][kRwExperts];
  __shared__ int s_list[kRwTokens];  // the staged tokens with a nonzero dL here, in order
  __shared__ int s_nz;
  pdl_wait();
  pdl_trigger();
  const int col = blockIdx.x * 256 + threadIdx.x;
  const int n0 = blockIdx.y * kRwExperts;
  const int t0 = blockIdx.z * chunk, t1 = min(T, t0 + chunk);
  float acc[kRwExperts];
#pragma unroll
  for (int i = 0; i < kRwExperts; ++i) acc[i] = 0.f;
  for (int tb = t0; tb < t1; tb += kRwTokens) {
    __syncthreads();
    for (int i = threadIdx.x; i < kRwTokens * kRwExperts; i += 256) {
      const int tt = tb + i / kRwExperts, n = n0 + i % kRwExperts;
      s_dl[i / kRwExperts][i % kRwExperts] =
          (tt < t1 && n < N) ? d_logits[static_cast<int64_t>(tt) * N + n] : 0.f;
    }
    __syncthreads();
    if (threadIdx.x < 32) {  // staged dL rows past the chunk's end are zero: never listed
      const int lane = threadIdx.x;
      int base = 0;
      for (int h = 0; h < kRwTokens; h += 32) {
        bool nz = false;
#pragma unroll
        for (int i = 0; i < kRwExperts; ++i) nz |= s_dl[h + lane][i] != 0.f;
        const unsigned m = __ballot_sync(0xffffffffu, nz);
        if (nz) s_list[base + __popc(m & ((1u << lane) - 1u))] = h + lane;
        base += __popc(m);
      }
      if (lane == 0) s_nz = base;
    }
    __syncthreads();
    if (col < d) {
      const int nz = s_nz;
      // eight listed tokens' loads in flight at once; the additions keep token order
      for (int u0 = 0; u0 < nz; u0 += 8) {
        int tl[8];
        float xv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          tl[u] = u0 + u < nz ? s_list[u0 + u] : -1;
          xv[u] = tl[u] >= 0 ? bf16_bits_to_float(x[static_cast<int64_t>(tb + tl[u]) * d + col]) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (tl[u] >= 0)
#pragma unroll
            for (int i = 0; i < kRwExperts; ++i) acc[i] += s_dl[tl[u]][i] * xv[u];
      }
    }
  }
  if (col < d) {
#pragma unroll
    for (int i = 0; i < kRwExperts; ++i)
      if (n0 + i < N)
        part[(static_cast<int64_t>(blockIdx.z) * N + n0 + i) * d + col] = acc[i];
  }
}

__global__ void __launch_bounds__(256) router_wgrad_final_kernel(const float* __restrict__ part,
                                                                 float* __restrict__ d_w_router,
                                                                 int d, int N, int chunks) {
  pdl_wait();
  pdl_trigger();
  const int64_t items = static_cast<int64_t>(N) * d;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < items;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float s = 0.f;
    for (int c = 0; c < chunks; ++c) s += part[c * items + i];
    d_w_router[i] = s;
  }
}

__global__ void __launch_bounds__(1024) router_bias_grad_kernel(const float* __restrict__ d_logits,
                                                                float* __restrict__ d_bias, int T,
                                                                int N) {
  __shared__ float s_sum[32][33];
  pdl_wait();
  pdl_trigger();
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = blockIdx.x * 32 + lane;
  float acc = 0.f;
  if (n < N)
    for (int t = w; t < T; t += 32) acc += d_logits[static_cast<int64_t>(t) * N + n];
  s_sum[w][lane] = acc;
  __syncthreads();
  if (w == 0 && n < N) {
    float s = 0.f;
    for (int i = 0; i < 32; ++i) s += s_sum[i][lane];
    d_bias[n] = s;
  }
}

// ------------------------------------------------------------------ back to token order
// dx[t] = sum over kept j (in choice order) of dx_rows[row(t, j)] + sum over j of
// dL[t, idx_j] W_r[idx_j] (dL is zero on the experts not chosen). Block per (token, 1024
// columns; tokens strided over grid.y), 4 columns a thread.
__global__ void __launch_bounds__(256) bwd_dx_kernel(
    const float* __restrict__ dx_rows, const int32_t* __restrict__ row_of_pair,
    const int32_t* __restrict__ topk_idx, const float* __restrict__ d_logits,
    const float* __restrict__ w_router, float* __restrict__ dx, int T, int d, int N, int k,
    int r_max) {
  pdl_wait();
  pdl_trigger();
  const int c = (blockIdx.x * 256 + threadIdx.x) * 4;
  if (c >= d) return;
  for (int t = blockIdx.y; t < T; t += gridDim.y) {
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = 0; j < k; ++j) {
    const int r = row_of_pair[t * k + j];
    if (r < 0 || r >= r_max) continue;
    const float4 v = *reinterpret_cast<const float4*>(dx_rows + static_cast<int64_t>(r) * d + c);
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  }
  for (int j = 0; j < k; ++j) {
    const int e = topk_idx[t * k + j];
    if (e < 0 || e >= N) continue;
    const float g = d_logits[static_cast<int64_t>(t) * N + e];
    const float4 wr = *reinterpret_cast<const float4*>(w_router + static_cast<int64_t>(e) * d + c);
    acc.x += g * wr.x;
    acc.y += g * wr.y;
    acc.z += g * wr.z;
    acc.w += g * wr.w;
  }
  *reinterpret_cast<float4*>(dx + static_cast<int64_t>(t) * d + c) = acc;
  }
}

// ------------------------------------------------------------------ host side
template <bool A_MN, bool B_MN, int MODE>
cudaError_t launch_gemm(const CUtensorMap& a, const CUtensorMap& b, const BwdGemmParams& p,
                        dim3 grid, cudaStream_t s) {
  // the output as fp32 32 x 32 store boxes: [r_max, n_out] (rows mode) or [N, M, n_out]
  CUtensorMap c;
  if (MODE == GEMM_ROWS) {
    const uint64_t dims[2] = {static_cast<uint64_t>(p.n_out), static_cast<uint64_t>(p.r_max)};
    const uint64_t str[1] = {static_cast<uint64_t>(p.n_out) * 4};
    const uint32_t box[2] = {32, 32};
    if (!make_map_f32(&c, p.out, 2, dims, str, box)) return cudaErrorInvalidValue;
  } else {
    const uint64_t dims[3] = {static_cast<uint64_t>(p.n_out), static_cast<uint64_t>(p.M),
                              static_cast<uint64_t>(p.n_experts)};
    const uint64_t str[2] = {static_cast<uint64_t>(p.n_out) * 4,
                             static_cast<uint64_t>(p.M) * p.n_out * 4};
    const uint32_t box[3] = {32, 32, 1};
    if (!make_map_f32(&c, p.out, 3, dims, str, box)) return cudaErrorInvalidValue;
  }
  auto kern = bwd_gemm_kernel<A_MN, B_MN, MODE>;
  static PerDeviceOnce once;
  const cudaError_t attr = once.run([] {
    return cudaFuncSetAttribute(bwd_gemm_kernel<A_MN, B_MN, MODE>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem);
  });
  if (attr != cudaSuccess) return attr;
  return launch_pdl(kern, grid, dim3(kGemmThreads), kGemmSmem, s, a, b, c, p);
}

// K-major operand [outer][K] bf16: boxes of 64 k x `rows`.
bool map_k_major_2d(CUtensorMap* m, const void* base, uint64_t K, uint64_t outer, uint32_t rows) {
  const uint64_t dims[2] = {K, outer};
  const uint64_t str[1] = {K * 2};
  const uint32_t box[2] = {static_cast<uint32_t>(kBK), rows};
  return make_map(m, base, 2, dims, str, box);
}
// MN-major operand [K rows][MN] bf16 (2-D): boxes of 64 MN x 64 k.
bool map_mn_major_2d(CUtensorMap* m, const void* base, uint64_t MN, uint64_t krows) {
  const uint64_t dims[2] = {MN, krows};
  const uint64_t str[1] = {MN * 2};
  const uint32_t box[2] = {64, static_cast<uint32_t>(kBK)};
  return make_map(m, base, 2, dims, str, box);
}

}  // namespace

size_t backward_router_chunk(int T) { return static_cast<size_t>(std::max(256, (T + 15) / 16)); }

cudaError_t launch_backward(const BackwardArgs& a, cudaStream_t s) {
  const int T = a.T, d = a.d, N = a.N, k = a.k, F = a.F;
  const bool swiglu = a.act == MOE_ACT_SWIGLU;
  const int n_gu = swiglu ? 2 * F : F;
  const uint64_t R = static_cast<uint64_t>(a.r_max);
  cudaError_t e;
  // 1: dy, dL
  {
    const int blocks = std::max(1, std::min((T + 7) / 8, 8 * 148));
    e = launch_pdl(bwd_pairs_kernel, dim3(blocks), dim3(256), 0, s, a.d_out, a.y_perm, a.topk_w,
                   a.topk_idx, a.row_of_pair, a.dy_perm, a.d_logits, T, d, N, k,
                   static_cast<int>(a.r_max), a.status);
    if (e != cudaSuccess) return e;
  }
  if (R > 0) {
    BwdGemmParams p{};
    p.expert_offset = a.expert_offset;
    p.n_experts = N;
    p.r_max = static_cast<int>(a.r_max);
    p.status = a.status;
    p.timeout_ns = a.timeout_ns;
    int sms = 148;
    {
      int dev = 0;
      if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    }
    // rows mode: the tile count depends on expert_offset, so every SM gets a CTA
    const dim3 rows_grid(static_cast<unsigned>(sms));
    auto wgrad_grid = [&](int M, int n_out) {
      const int64_t t = static_cast<int64_t>(N) * ((M + kBM - 1) / kBM) * ((n_out + kBN - 1) / kBN);
      return dim3(static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(t, sms))));
    };
    CUtensorMap mA, mB;
    // 2: pre = x_perm W_gu^T
    if (!map_k_major_2d(&mA, a.x_perm, d, R, kBM)) return cudaErrorInvalidValue;
    {
      const uint64_t dims[3] = {static_cast<uint64_t>(d), static_cast<uint64_t>(n_gu), static_cast<uint64_t>(N)};
      const uint64_t str[2] = {static_cast<uint64_t>(d) * 2, static_cast<uint64_t>(n_gu) * d * 2};
      const uint32_t box[3] = {static_cast<uint32_t>(kBK), static_cast<uint32_t>(kBN), 1};
      if (!make_map(&mB, a.w_gate_up, 3, dims, str, box)) return cudaErrorInvalidValue;
    }
    p.n_out = n_gu;
    p.num_kb = d / kBK;
    p.out = a.pre;
    e = launch_gemm<false, false, GEMM_ROWS>(mA, mB, p, rows_grid, s);
    if (e != cudaSuccess) return e;
    // 3: dh = dy W_d (W_d [N][d][F] read MN-major: F is the output axis)
    if (!map_k_major_2d(&mA, a.dy_perm, d, R, kBM)) return cudaErrorInvalidValue;
    {
      const uint64_t dims[3] = {static_cast<uint64_t>(F), static_cast<uint64_t>(d), static_cast<uint64_t>(N)};
      const uint64_t str[2] = {static_cast<uint64_t>(F) * 2, static_cast<uint64_t>(d) * F * 2};
      const uint32_t box[3] = {64, static_cast<uint32_t>(kBK), 1};
      if (!make_map(&mB, a.w_down, 3, dims, str, box)) return cudaErrorInvalidValue;
    }
    p.n_out = F;
    p.num_kb = d / kBK;
    p.out = a.dh;
    e = launch_gemm<false, true, GEMM_ROWS>(mA, mB, p, rows_grid, s);
    if (e != cudaSuccess) return e;
    // 4: d_pre, h
    {
      const int64_t items = static_cast<int64_t>(R) * (F / 4);
      const int blocks = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((items + 255) / 256, 16 * 148)));
      e = launch_pdl(act_bwd_kernel, dim3(blocks), dim3(256), 0, s, static_cast<const float*>(a.pre),
                     static_cast<const float*>(a.dh), a.expert_offset, a.d_pre, a.h, N, F,
                     swiglu ? 1 : 0);
      if (e != cudaSuccess) return e;
    }
    // 5: dx_rows = d_pre W_gu (W_gu [N][n_gu][d] read MN-major: d is the output axis)
    if (!map_k_major_2d(&mA, a.d_pre, n_gu, R, kBM)) return cudaErrorInvalidValue;
    {
      const uint64_t dims[3] = {static_cast<uint64_t>(d), static_cast<uint64_t>(n_gu), static_cast<uint64_t>(N)};
      const uint64_t str[2] = {static_cast<uint64_t>(d) * 2, static_cast<uint64_t>(n_gu) * d * 2};
      const uint32_t box[3] = {64, static_cast<uint32_t>(kBK), 1};
      if (!make_map(&mB, a.w_gate_up, 3, dims, str, box)) return cudaErrorInvalidValue;
    }
    p.n_out = d;
    p.num_kb = n_gu / kBK;
    p.out = a.dx_rows;
    e = launch_gemm<false, true, GEMM_ROWS>(mA, mB, p, rows_grid, s);
    if (e != cudaSuccess) return e;
    // 6: dW_d[e] = dy_e^T h_e  ([d, F] per expert)
    if (!map_mn_major_2d(&mA, a.dy_perm, d, R)) return cudaErrorInvalidValue;
    if (!map_mn_major_2d(&mB, a.h, F, R)) return cudaErrorInvalidValue;
    p.M = d;
    p.n_out = F;
    p.out = a.d_w_down;
    e = launch_gemm<true, true, GEMM_WGRAD>(mA, mB, p, wgrad_grid(d, F), s);
    if (e != cudaSuccess) return e;
    // 7: dW_gu[e] = d_pre_e^T x_e  ([n_gu, d] per expert)
    if (!map_mn_major_2d(&mA, a.d_pre, n_gu, R)) return cudaErrorInvalidValue;
    if (!map_mn_major_2d(&mB, a.x_perm, d, R)) return cudaErrorInvalidValue;
    p.M = n_gu;
    p.n_out = d;
    p.out = a.d_w_gate_up;
    e = launch_gemm<true, true, GEMM_WGRAD>(mA, mB, p, wgrad_grid(n_gu, d), s);
    if (e != cudaSuccess) return e;
  } else {
    // no kept rows: the experts' gradients are zero
    e = cudaMemsetAsync(a.d_w_gate_up, 0, static_cast<size_t>(N) * n_gu * d * 4, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(a.d_w_down, 0, static_cast<size_t>(N) * d * F * 4, s);
    if (e != cudaSuccess) return e;
  }
  // 8: router weight (and bias) gradient
  {
    const int chunk = static_cast<int>(backward_router_chunk(T));
    const int chunks = (T + chunk - 1) / chunk;
    e = launch_pdl(router_wgrad_partial_kernel,
                   dim3((d + 255) / 256, (N + kRwExperts - 1) / kRwExperts, chunks), dim3(256), 0, s,
                   static_cast<const float*>(a.d_logits), a.x, a.router_part, T, d, N, chunk);
    if (e != cudaSuccess) return e;
    const int64_t items = static_cast<int64_t>(N) * d;
    const int blocks = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((items + 255) / 256, 8 * 148)));
    e = launch_pdl(router_wgrad_final_kernel, dim3(blocks), dim3(256), 0, s,
                   static_cast<const float*>(a.router_part), a.d_w_router, d, N, chunks);
    if (e != cudaSuccess) return e;
    if (a.d_logit_bias != nullptr) {
      e = launch_pdl(router_bias_grad_kernel, dim3((N + 31) / 32), dim3(1024), 0, s,
                     static_cast<const float*>(a.d_logits), a.d_logit_bias, T, N);
      if (e != cudaSuccess) return e;
    }
  }
  // 9: dx
  return launch_pdl(bwd_dx_kernel, dim3((d + 1023) / 1024, std::min(T, 65535)), dim3(256), 0, s,
                    static_cast<const float*>(a.dx_rows), a.row_of_pair, a.topk_idx,
                    static_cast<const float*>(a.d_logits), a.w_router, a.d_x, T, d, N, k,
                    static_cast<int>(a.r_max));
}

}  // namespace moe
