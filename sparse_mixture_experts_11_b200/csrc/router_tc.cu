// Router logits on tcgen05 tensor cores, with top-k and renormalised weights in the epilogue.
//
// Page «Sparse Mixture-of-Experts», section «Роутер и top-k gating»: logits from a linear
// layer without bias term, softmax over the experts, the k most probable experts, their
// probabilities renormalised to one. Selection is made on the fp32 logits (the same experts as
// on the probabilities); equal logits go to the lower expert index.
//
// x is exactly bf16. The fp32 router weight is split, inside the kernel, into three bf16 terms
// hi + mid + lo (each the bf16 rounding of what the previous terms left over). Together they
// carry the fp32 significand, so x·hi + x·mid + x·lo accumulated in fp32 reproduces the fp32
// dot product to within fp32 accumulation error. Every product of two bf16 values is exact
// in fp32.
//
// Two ways to get the split terms, with identical results (same bf16 terms, same MMA order):
//   PRESPLIT  a small kernel writes [3][N][d] bf16 into the caller's workspace once per call
//             and the router kernel TMA-loads the three term tiles with each x tile;
//   in-kernel for callers without a workspace: warps 4-7 read W_r[:, k block] in fp32 and
//             write the three terms as K-major 128B-swizzled tiles into shared memory
//             (double buffered), every CTA repeating the conversion.
//
// One CTA per 128-token tile, 256 threads. When the tiles leave SMs idle, a cluster of 2 or 4
// CTAs shares a tile, each taking an equal range of the k blocks into its own TMEM
// accumulator; the non-leaders stage their partial logits in shared memory and the leader
// adds them through distributed shared memory in rank order (deterministic), then runs the
// epilogue below. Per CTA:
//   warp 0      TMA producer of the x tile [128 tokens x 64 k] (128B swizzle) into a ring
//               (and of the three weight term tiles when PRESPLIT);
//   warp 1      TMEM owner and MMA issuer: per k block 3 x 4 MMAs (M=128, N=NP, K=16) into one
//               fp32 accumulator of NP columns;
//   warps 4-7   (in-kernel split only) the converters, then the epilogue: thread i owns token
//               i's row of logits in TMEM, adds the bias, keeps a running sorted top-KMAX
//               (KMAX = k rounded up to 1, 2, 4 or 8) and writes the first k indices and
//               weights; the [128][N] logits tile is staged in the idle
//               pipeline shared memory and written out as one coalesced block.
// All mbarrier waits are bounded. A timeout records MOE_ERR_TIMEOUT, stops the CTA's work,
// drains its own copies and MMAs, and frees TMEM.
#include <math.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "launch.h"
#include "tma_host.h"

namespace moe {
namespace {

constexpr int kTok = 128;  // tokens per CTA (UMMA M)
constexpr int kBK = 64;    // k per block (one 128-byte swizzle row of bf16)
constexpr int kThreads = 256;
constexpr int kConvThreads = 128;
constexpr int kSmemLimit = 225 * 1024;
constexpr uint64_t kPairDrainNs = 1000000;  // 1 ms
constexpr int kCand = 96;  // listed top-k candidates per token in the epilogue

template <int NP, bool PRESPLIT, bool PAIR = false>
struct RCfg {
  static_assert(!PAIR || PRESPLIT, "CTA pairs load the split terms by TMA");
  static constexpr int A_BYTES = kTok * kBK * 2;           // 16 KB per x tile
  static constexpr int WROWS = PAIR ? NP / 2 : NP;         // term rows held by this CTA
  static constexpr int WT_BYTES = WROWS * kBK * 2;         // one split term tile
  static constexpr int WBUF_BYTES = 3 * WT_BYTES;          // hi, mid, lo
  // PRESPLIT: each ring stage holds the x tile and the three term tiles.
  // in-kernel: a ring of x tiles plus two converter-written term buffers.
  static constexpr int STAGE_BYTES = PRESPLIT ? A_BYTES + WBUF_BYTES : A_BYTES;
  static constexpr int FIXED_BYTES = PRESPLIT ? 0 : 2 * WBUF_BYTES;
  static constexpr int STAGES_FIT = (kSmemLimit - 1024 - FIXED_BYTES) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  static constexpr int TMEM_COLS = NP < 32 ? 32 : NP;
  static constexpr int SMEM_BYTES = FIXED_BYTES + STAGES * STAGE_BYTES + 1024;
  static_assert(STAGES >= 2, "router pipeline depth");
  static_assert(NP % 16 == 0 && NP >= 16 && NP <= 256, "UMMA N for M = 128");
  static_assert(!PAIR || NP % 32 == 0, "UMMA N for a CTA pair (M = 256)");
  static_assert(kTok * (NP + 4) * 4 <= SMEM_BYTES - 1024, "logits staging fits the pipeline smem");
  static_assert(kTok * (NP + 1) * 4 + kCand * kTok <= SMEM_BYTES - 1024,
                "logits staging and the top-k candidate lists fit the pipeline smem");
  // with a k split (never with a CTA pair): the staged partials plus the final rows of this CTA
  // (at most 64)
  static_assert(PAIR || (kTok + kTok / 2) * (NP + 4) * 4 <= SMEM_BYTES - 1024,
                "k-split staging (partials + final rows) fits the pipeline smem");
};

__device__ __forceinline__ bool better(float av, int ae, float bv, int be) {
  return av > bv || (av == bv && ae < be);
}

// The 128-byte swizzle: 16-byte chunk c of row n sits at chunk position c ^ (n & 7).
__device__ __forceinline__ uint32_t sw128_offset(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// Split 8 consecutive fp32 weights into three bf16 terms each (hi, mid, lo), packed in pairs.
__device__ __forceinline__ void split3(const float4& v0, const float4& v1, uint4& hi, uint4& mid,
                                       uint4& lo) {
  const float f[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
  uint32_t h[4], m[4], l[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float r0 = f[2 * q], r1 = f[2 * q + 1];
    const __nv_bfloat162 bh = __floats2bfloat162_rn(r0, r1);
    r0 -= __low2float(bh);
    r1 -= __high2float(bh);
    const __nv_bfloat162 bm = __floats2bfloat162_rn(r0, r1);
    r0 -= __low2float(bm);
    r1 -= __high2float(bm);
    const __nv_bfloat162 bl = __floats2bfloat162_rn(r0, r1);
    h[q] = *reinterpret_cast<const uint32_t*>(&bh);
    m[q] = *reinterpret_cast<const uint32_t*>(&bm);
    l[q] = *reinterpret_cast<const uint32_t*>(&bl);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  mid = make_uint4(m[0], m[1], m[2], m[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// W_r [N, d] fp32 -> [3][N][d] bf16 terms (row-major per term).
__global__ void __launch_bounds__(256) split_router_weights_kernel(const float* __restrict__ w,
                                                                   uint16_t* __restrict__ out,
                                                                   int64_t n_elems) {
  pdl_trigger();
  pdl_wait();
  const int64_t n8 = n_elems / 8;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4* src = reinterpret_cast<const float4*>(w) + 2 * i;
    uint4 hi, mid, lo;
    split3(__ldg(src), __ldg(src + 1), hi, mid, lo);
    reinterpret_cast<uint4*>(out)[i] = hi;
    reinterpret_cast<uint4*>(out + n_elems)[i] = mid;
    reinterpret_cast<uint4*>(out + 2 * n_elems)[i] = lo;
  }
}

// A sorted list of the best KMAX (>= k) (logit, expert) entries; entry KMAX-1 is the
// admission threshold. NaN logits rank below every number; equal logits go to the lower index.
template <int KMAX>
struct TopK {
  float v[KMAX];
  int e[KMAX];
  __device__ __forceinline__ TopK() {
#pragma unroll
    for (int r = 0; r < KMAX; ++r) {
      v[r] = -INFINITY;
      e[r] = 0x7fffffff;
    }
  }
  // add a candidate without branches: it takes the first slot whose entry it beats, and each
  // entry it displaces moves down by one slot (the last one drops out)
  __device__ __forceinline__ void insert(float key, int ex) {
#pragma unroll
    for (int r = 0; r < KMAX; ++r) {
      const bool b = better(key, ex, v[r], e[r]);
      const float tv = v[r];
      const int te = e[r];
      v[r] = b ? key : tv;
      e[r] = b ? ex : te;
      key = b ? tv : key;
      ex = b ? te : ex;
    }
  }
  // drop the best entry (the list moves up by one; the last slot empties)
  __device__ __forceinline__ void pop() {
#pragma unroll
    for (int r = 0; r + 1 < KMAX; ++r) {
      v[r] = v[r + 1];
      e[r] = e[r + 1];
    }
    v[KMAX - 1] = -INFINITY;
    e[KMAX - 1] = 0x7fffffff;
  }
  __device__ __forceinline__ void offer(float L, int ex) {
    const float key = isnan(L) ? -INFINITY : L;
    if (!better(key, ex, v[KMAX - 1], e[KMAX - 1])) return;
    // shift the entries the candidate beats down by one and drop it into place; every
    // slot's update reads only the old list, so the slots update in parallel
#pragma unroll
    for (int r = KMAX - 1; r >= 0; --r) {
      if (better(key, ex, v[r], e[r])) {
        const int u = r > 0 ? r - 1 : 0;
        const bool beats_prev = (r > 0) && better(key, ex, v[u], e[u]);
        v[r] = beats_prev ? v[u] : key;
        e[r] = beats_prev ? e[u] : ex;
      }
    }
  }
};

// Token t0 + ct's top-k indices and renormalised weights, then (after a barrier of the 128
// epilogue threads) the tile's logits out of the staging rows as one coalesced block.
template <int KMAX>
__device__ __forceinline__ bool finish_tile(const TopK<KMAX>& best, const float* stage, int t0,
                                            int ct, int T, int N, int NS, int k, float* logits,
                                            int32_t* topk_idx, float* topk_w, uint32_t epi_bar,
                                            uint64_t timeout_ns, const volatile int* abort) {
  const int t = t0 + ct;
  if (t < T) {
    float num[KMAX], den = 0.f;
#pragma unroll
    for (int r = 0; r < KMAX; ++r) {
      num[r] = (r < k) ? expf(best.v[r] - best.v[0]) : 0.f;
      den += num[r];
    }
#pragma unroll
    for (int r = 0; r < KMAX; ++r)
      if (r < k) {
        topk_idx[static_cast<int64_t>(t) * k + r] = best.e[r];
        topk_w[static_cast<int64_t>(t) * k + r] = num[r] / den;
      }
  }
  mbar_arrive(epi_bar);
  const bool synced = mbar_wait(epi_bar, 0, timeout_ns, abort);
  if (!__all_sync(0xffffffffu, synced)) return false;
  const int rows = min(kTok, T - t0);
  float* dst = logits + static_cast<int64_t>(t0) * N;
  if (N <= kConvThreads) {
    // thread ct copies column ct mod N of rows ct / N, ct / N + 128 / N, ...
    const int rstep = kConvThreads / N, r0 = ct / N, c = ct - r0 * N;
    if (r0 < rstep) {
      int r = r0;
      for (; r + 3 * rstep < rows; r += 4 * rstep) {
        float q[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) q[u] = stage[(r + u * rstep) * NS + c];
#pragma unroll
        for (int u = 0; u < 4; ++u) dst[(r + u * rstep) * N + c] = q[u];
      }
      for (; r < rows; r += rstep) dst[r * N + c] = stage[r * NS + c];
    }
  } else {
    // thread ct copies columns ct and ct + 128 of every row
    for (int c = ct; c < N; c += kConvThreads) {
      int r = 0;
      for (; r + 7 < rows; r += 8) {
        float q[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) q[u] = stage[(r + u) * NS + c];
#pragma unroll
        for (int u = 0; u < 8; ++u) dst[(r + u) * N + c] = q[u];
      }
      for (; r < rows; ++r) dst[r * N + c] = stage[r * NS + c];
    }
  }
  return true;
}

// For the router statistics: the tile's router probabilities summed per expert over its
// tokens. The staged rows of logits (rows valid ones of the buffer's, stride NS; ks threads per
// row, neighbouring lanes, ks = 1, 2 or 4) become their softmax in place, using m, the row's
// largest logit; after a barrier thread ct adds columns ct, ct + 128, ... over the rows in row
// order. Each barrier is a phase of the epilogue threads' mbarrier, starting at `parity`.
__device__ __forceinline__ bool tile_prob_sums(float m, float* buf, int rows, int NS, int N, int ks,
                                               int ct, float* out_row, uint32_t epi_bar,
                                               uint32_t parity, uint64_t timeout_ns,
                                               const volatile int* abort) {
  mbar_arrive(epi_bar);  // every thread has finished reading the staged logits
  bool ok = mbar_wait(epi_bar, parity, timeout_ns, abort);
  if (!__all_sync(0xffffffffu, ok)) return false;
  const int lr = ct / ks, part = ct - lr * ks;
  float sum = 0.f;
  if (lr < rows) {
    float* row = buf + lr * NS;
    for (int e = part; e < N; e += ks) {
      const float v = expf(row[e] - m);
      row[e] = v;
      sum += v;
    }
  }
  for (int o = 1; o < ks; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lr < rows) {
    const float inv = 1.0f / sum;
    float* row = buf + lr * NS;
    for (int e = part; e < N; e += ks) row[e] *= inv;
  }
  mbar_arrive(epi_bar);
  ok = mbar_wait(epi_bar, parity ^ 1u, timeout_ns, abort);
  if (!__all_sync(0xffffffffu, ok)) return false;
  for (int e = ct; e < N; e += kConvThreads) {
    float acc = 0.f;
    for (int r = 0; r < rows; ++r) acc += buf[r * NS + e];
    out_row[e] = acc;
  }
  return true;
}

template <int NP, bool PRESPLIT, int KMAX, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                     const float* __restrict__ w, const float* __restrict__ bias,
                     float* __restrict__ logits, int32_t* __restrict__ topk_idx,
                     float* __restrict__ topk_w, int T, int d, int N, int k, int* status,
                     uint64_t timeout_ns, float* __restrict__ prob_part, int ksplit) {
  using C = RCfg<NP, PRESPLIT, PAIR>;
  extern __shared__ __align__(1024) uint8_t dyn_smem[];
  __shared__ __align__(8) uint64_t a_full[C::STAGES];
  __shared__ __align__(8) uint64_t a_empty[C::STAGES];
  __shared__ __align__(8) uint64_t w_full[2];
  __shared__ __align__(8) uint64_t w_empty[2];
  __shared__ __align__(8) uint64_t acc_full;
  __shared__ __align__(8) uint64_t done_bar;
  __shared__ __align__(8) uint64_t epi_bar;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;

  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t base = (smem_u32(dyn_smem) + 1023u) & ~1023u;
  uint8_t* gbase = dyn_smem + (base - smem_u32(dyn_smem));  // generic pointer of `base`
  const uint32_t wbuf0 = base;                               // in-kernel: 2 x [3][NP][64] bf16
  const uint32_t ring0 = base + C::FIXED_BYTES;              // ring of stages
  // ksplit > 1: a cluster of ksplit CTAs shares one token tile, CTA `rank` taking k blocks
  // [kb_lo, kb_hi); the leader (rank 0) adds the partial logits in rank order
  const int rank = ksplit > 1 ? static_cast<int>(cluster_ctarank()) : 0;
  // PAIR: the cluster's two CTAs take neighbouring token tiles, and the even CTA issues M = 256
  // MMAs over both (its peer holds the other 128 tokens and the upper NP / 2 rows of each term)
  const int prank = PAIR ? static_cast<int>(cluster_ctarank()) : 0;
  const bool mma_cta = prank == 0;
  const int t0 = (blockIdx.x / ksplit) * kTok;
  const int num_kb = d / kBK;
  const int kb_lo = rank * num_kb / ksplit, kb_hi = (rank + 1) * num_kb / ksplit;
  const int n_it = kb_hi - kb_lo;
  // staged logits rows: N4 = N rounded up to 4 columns, stride NS (16-byte aligned rows)
  const int N4 = (N + 3) & ~3;
  const int NS = ksplit > 1 ? N4 + 4 : N + 1;  // N + 1: no bank conflicts in the 1-CTA path
  bool epi_ok = false;

  if (threadIdx.x == 0) {
    prefetch_tensormap(&tmX);
    if (PRESPLIT) prefetch_tensormap(&tmW);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_u32(&a_full[s]), 1);
      mbar_init(smem_u32(&a_empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&w_full[b]), kConvThreads);
      mbar_init(smem_u32(&w_empty[b]), 1);
    }
    mbar_init(smem_u32(&acc_full), 1);
    mbar_init(smem_u32(&done_bar), 1);
    mbar_init(smem_u32(&epi_bar), kConvThreads);
    s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    __syncwarp();
    if constexpr (PAIR) {
      tmem_alloc_pair(smem_u32(&s_tmem), C::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(&s_tmem), C::TMEM_COLS);
      tmem_relinquish();
    }
  }
  if (!PRESPLIT && warp >= 4 && NP > N) {
    // rows N..NP-1 of both term buffers stay zero for the whole kernel
    const int ct = threadIdx.x - 128;
    for (int b = 0; b < 2; ++b)
      for (int term = 0; term < 3; ++term)
        for (int i = ct; i < (NP - N) * 8; i += kConvThreads) {
          const int row = N + i / 8, chunk = i % 8;
          *reinterpret_cast<uint4*>(gbase + b * C::WBUF_BYTES + term * C::WT_BYTES +
                                    sw128_offset(row, chunk)) = make_uint4(0, 0, 0, 0);
        }
    fence_proxy_async_smem();
  }
  pdl_wait();  // everything below reads the previous kernels' outputs or writes global memory
  tc_fence_before_sync();
  if constexpr (PAIR)
    cluster_sync_all();  // both CTAs' barriers and TMEM exist before either CTA uses the other's
  else
    __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = s_tmem;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_x = l2_policy_evict_first();
      const uint64_t pol_w = l2_policy_evict_last();
      int i = 0;
      bool ok = true;
      for (; i < n_it; ++i) {
        const int kb = kb_lo + i;
        const int s = i % C::STAGES;
        if (!mbar_wait(smem_u32(&a_empty[s]), ((i / C::STAGES) & 1) ^ 1u, timeout_ns, &s_abort)) {
          ok = false;
          break;
        }
        const uint32_t st = ring0 + s * C::STAGE_BYTES;
        const uint32_t fb = smem_u32(&a_full[s]);
        if constexpr (PAIR) {
          // both CTAs' bytes complete on the even CTA's barrier, which the even CTA arms
          const uint32_t fb0 = map_smem_to_rank(fb, 0);
          if (mma_cta) mbar_arrive_expect_tx(fb, 2 * C::STAGE_BYTES);
          tma_load_2d_pair(st, &tmX, fb0, kb * kBK, t0, pol_x);
#pragma unroll
          for (int term = 0; term < 3; ++term)
            tma_load_3d_pair(st + C::A_BYTES + term * C::WT_BYTES, &tmW, fb0, kb * kBK,
                             prank * C::WROWS, term, pol_w);
        } else {
          mbar_arrive_expect_tx(fb, C::STAGE_BYTES);
          tma_load_2d(st, &tmX, fb, kb * kBK, t0, pol_x);
          if (PRESPLIT) {
#pragma unroll
            for (int term = 0; term < 3; ++term)
              tma_load_3d(st + C::A_BYTES + term * C::WT_BYTES, &tmW, fb, kb * kBK, 0, term, pol_w);
          }
        }
      }
      if (!ok) {
        s_abort = 1;
        report_error(status, MOE_ERR_TIMEOUT);
      }
      if (!PAIR || mma_cta) {
        for (int j = max(0, i - C::STAGES); j < i; ++j)
          mbar_wait(smem_u32(&a_full[j % C::STAGES]), (j / C::STAGES) & 1, kDrainTimeoutNs, nullptr);
      } else {
        // the odd CTA's copies complete on the even CTA's barriers: it waits until the MMAs have
        // released its last stages (so they landed), within one overall limit that leaves any
        // copy still in flight after a timeout ample time to land
        const uint64_t t_end = globaltimer_ns() + kPairDrainNs;
        for (int j = max(0, i - C::STAGES); j < i; ++j) {
          const uint64_t now = globaltimer_ns();
          mbar_wait(smem_u32(&a_empty[j % C::STAGES]), (j / C::STAGES) & 1,
                    now < t_end ? t_end - now : 1, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && PAIR && !mma_cta) {
      // the odd CTA of a pair issues nothing; its TMEM and shared memory stay in use until
      // the even CTA's MMAs are done (the even CTA always signals this barrier at the end)
      mbar_wait(smem_u32(&done_bar), 0, kDrainTimeoutNs, nullptr);
    } else if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(PAIR ? 2 * kTok : kTok, NP);
      bool ok = true, issued = false;
      for (int i = 0; i < n_it; ++i) {
        const int s = i % C::STAGES, b = i & 1;
        if (!mbar_wait(smem_u32(&a_full[s]), (i / C::STAGES) & 1, timeout_ns, &s_abort) ||
            (!PRESPLIT && !mbar_wait(smem_u32(&w_full[b]), (i >> 1) & 1, timeout_ns, &s_abort))) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t a = ring0 + s * C::STAGE_BYTES;
        const uint32_t wt0 = PRESPLIT ? a + C::A_BYTES : wbuf0 + b * C::WBUF_BYTES;
#pragma unroll
        for (int term = 0; term < 3; ++term) {
          const uint32_t bt = wt0 + term * C::WT_BYTES;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t ad = smem_desc_k_sw128(a + kk * 32), bd = smem_desc_k_sw128(bt + kk * 32);
            const uint32_t acc = (i | term | kk) != 0 ? 1u : 0u;
            if constexpr (PAIR)
              tc_mma_f16_pair(tmem, ad, bd, idesc, acc);
            else
              tc_mma_f16(tmem, ad, bd, idesc, acc);
          }
        }
        issued = true;
        if constexpr (PAIR) {
          tc_commit_pair(smem_u32(&a_empty[s]), 0x3);  // the stage is free in both CTAs
        } else {
          tc_commit(smem_u32(&a_empty[s]));
          if (!PRESPLIT) tc_commit(smem_u32(&w_empty[b]));
        }
      }
      if (ok) {
        if constexpr (PAIR)
          tc_commit_pair(smem_u32(&acc_full), 0x3);
        else
          tc_commit(smem_u32(&acc_full));
      } else {
        s_abort = 1;
        report_error(status, MOE_ERR_TIMEOUT);
      }
      // every issued MMA has finished before TMEM is freed, also when the epilogue gave up
      // waiting for the accumulator
      if constexpr (PAIR) {
        tc_commit_pair(smem_u32(&done_bar), 0x3);
        mbar_wait(smem_u32(&done_bar), 0, kDrainTimeoutNs, nullptr);
      } else if (issued) {
        tc_commit(smem_u32(&done_bar));
        mbar_wait(smem_u32(&done_bar), 0, kDrainTimeoutNs, nullptr);
      }
    }
  } else if (warp >= 4) {
    const int ct = threadIdx.x - 128;  // 0..127
    bool ok = true;
    if (!PRESPLIT) {
      // -------------------------------------------------------- in-kernel split of W_r
      constexpr int kTasks = (NP * 8 + kConvThreads - 1) / kConvThreads;  // <= 16
      for (int i = 0; i < n_it; ++i) {
        const int kb = kb_lo + i;
        const int b = i & 1;
        // issue every load of this k block before waiting, so their latencies overlap
        float4 v[kTasks][2];
#pragma unroll
        for (int u = 0; u < kTasks; ++u) {
          const int task = ct + u * kConvThreads;
          if (task < N * 8) {
            const float4* src = reinterpret_cast<const float4*>(
                w + static_cast<int64_t>(task >> 3) * d + kb * kBK + (task & 7) * 8);
            v[u][0] = __ldg(src);
            v[u][1] = __ldg(src + 1);
          }
        }
        const bool got = mbar_wait(smem_u32(&w_empty[b]), ((i >> 1) & 1) ^ 1u, timeout_ns, &s_abort);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        uint8_t* buf = gbase + b * C::WBUF_BYTES;
#pragma unroll
        for (int u = 0; u < kTasks; ++u) {
          const int task = ct + u * kConvThreads;
          if (task < N * 8) {
            uint4 hi, mid, lo;
            split3(v[u][0], v[u][1], hi, mid, lo);
            const uint32_t off = sw128_offset(task >> 3, task & 7);
            *reinterpret_cast<uint4*>(buf + off) = hi;
            *reinterpret_cast<uint4*>(buf + C::WT_BYTES + off) = mid;
            *reinterpret_cast<uint4*>(buf + 2 * C::WT_BYTES + off) = lo;
          }
        }
        fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core
        mbar_arrive(smem_u32(&w_full[b]));
      }
    }
    // ---------------------------------------------------------- epilogue: token t0 + ct
    if (ok) {
      const bool got = mbar_wait(smem_u32(&acc_full), 0, timeout_ns, &s_abort);
      ok = __all_sync(0xffffffffu, got);
    }
    if (ok) {
      tc_fence_after_sync();
      const int q = warp & 3;
      const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16);
      // the pipeline's shared memory is idle now: it stages the [128][N] logits tile
      float* stage = reinterpret_cast<float*>(gbase);
      if (ksplit > 1) {
        // this CTA's partial sums (its k range), raw, for the leader to add up
        for (int c0 = 0; c0 < N; c0 += 32) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(trow + c0, v);  // columns past NP are never used (see below)
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c0 + i < N4) stage[ct * NS + c0 + i] = __uint_as_float(v[i]);
        }
      } else {
        // the token's logits into its staging row, and the largest key (NaN ranks as -inf) of
        // each column class e mod KMAX: the smallest of these KMAX maxima, thr, is at most the
        // KMAX-th largest key (each class holds a key >= thr), so every top-k column has a
        // key >= thr
        float gmax[KMAX];
#pragma unroll
        for (int r = 0; r < KMAX; ++r) gmax[r] = -INFINITY;
        float* row = stage + ct * NS;
        // 32 columns per TMEM load (columns past NP are never used: c0 + 32 <= NP or N <= 16);
        // the chunk's bias values are loaded while the TMEM load is in flight
        for (int c0 = 0; c0 < N; c0 += 32) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(trow + c0, v);
          float bv[32];
#pragma unroll
          for (int i = 0; i < 32; ++i)
            bv[i] = (bias != nullptr && c0 + i < N) ? __ldg(bias + c0 + i) : 0.f;
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int e = c0 + i;
            if (e >= N) continue;
            const float L = __uint_as_float(v[i]) + bv[i];
            row[e] = L;
            gmax[i % KMAX] = fmaxf(gmax[i % KMAX], isnan(L) ? -INFINITY : L);
          }
        }
        float thr = gmax[0];
#pragma unroll
        for (int r = 1; r < KMAX; ++r) thr = fminf(thr, gmax[r]);
        // the columns with key >= thr, in column order, as bytes after the staging rows
        // ([kCand][kTok]); then the top-k of just those, all lanes of the warp stepping through
        // the longest list together. A token with more than kCand such columns (many equal
        // keys) takes every column instead.
        uint8_t* cand = reinterpret_cast<uint8_t*>(stage + kTok * NS);
        int nc = 0;
        for (int e0 = 0; e0 < N; e0 += 8) {
          float q[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) q[u] = e0 + u < N ? row[e0 + u] : 0.f;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const bool c = e0 + u < N && (isnan(q[u]) ? -INFINITY : q[u]) >= thr;
            if (c && nc < kCand) cand[nc * kTok + ct] = static_cast<uint8_t>(e0 + u);
            nc += c ? 1 : 0;
          }
        }
        const bool listed = nc <= kCand;
        const int rounds = __reduce_max_sync(0xffffffffu, listed ? nc : 0);
        TopK<KMAX> best;
        for (int j = 0; j < rounds; ++j) {
          float key = -INFINITY;
          int ex = 0x7fffffff;
          if (listed && j < nc) {
            ex = cand[j * kTok + ct];
            const float L = row[ex];
            key = isnan(L) ? -INFINITY : L;
          }
          best.insert(key, ex);
        }
        if (__any_sync(0xffffffffu, !listed)) {
          for (int e = 0; e < N; ++e) {
            const float L = row[e];
            if (!listed) best.insert(isnan(L) ? -INFINITY : L, e);
          }
        }
        ok = finish_tile<KMAX>(best, stage, t0, ct, T, N, NS, k, logits, topk_idx, topk_w,
                               smem_u32(&epi_bar), timeout_ns, &s_abort);
        if (ok && prob_part != nullptr)
          ok = tile_prob_sums(best.v[0], stage, min(kTok, T - t0), NS, N, 1, ct,
                              prob_part + static_cast<int64_t>(blockIdx.x) * N, smem_u32(&epi_bar),
                              1u, timeout_ns, &s_abort);
      }
    }
    epi_ok = ok;
    if (!ok) {
      s_abort = 1;
      report_error(status, MOE_ERR_TIMEOUT);
    }
  }

  if (ksplit > 1) {
    __syncwarp();
    cluster_sync_all();  // every CTA's partial tile is in its shared memory
    if (warp >= 4 && epi_ok) {
      // CTA `rank` finishes rows [rank * R, rank * R + R) of the tile: ksplit threads per row,
      // each adding the partials of its float4 column groups in rank order (all loads in
      // flight at once), then the row's top-k is merged across the row's threads by shuffles
      const int ct = threadIdx.x - 128;
      const int R = kTok / ksplit;
      const int lr = ct / ksplit, part = ct - lr * ksplit;  // local row, thread within the row
      const int row = rank * R + lr;
      float* stage = reinterpret_cast<float*>(gbase);
      float* fin = stage + kTok * NS;  // [R][NS] final logits of this CTA's rows
      const uint32_t src = smem_u32(stage + row * NS);
      uint32_t base_r[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) base_r[r] = r < ksplit ? map_smem_to_rank(src, r) : 0u;
      TopK<KMAX> best;
      constexpr int kGroups = (NP / 4 + 1) / 2;  // column groups per thread (ksplit >= 2)
      for (int g0 = 0; g0 < kGroups; g0 += 4) {
        float4 v[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int g = (g0 + j) * ksplit + part;
#pragma unroll
          for (int r = 0; r < 4; ++r)
            if (r < ksplit && g * 4 < N4) v[j][r] = ld_dsmem_f32x4(base_r[r] + g * 16);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int g = (g0 + j) * ksplit + part;
          if (g * 4 >= N4) continue;
          float4 acc = v[j][0];
#pragma unroll
          for (int r = 1; r < 4; ++r) {
            if (r < ksplit) {
              acc.x += v[j][r].x;
              acc.y += v[j][r].y;
              acc.z += v[j][r].z;
              acc.w += v[j][r].w;
            }
          }
          const float a4[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int e = g * 4 + i;
            if (e >= N) continue;
            float L = a4[i];
            if (bias != nullptr) L += __ldg(bias + e);
            fin[lr * NS + e] = L;
            best.offer(L, e);
          }
        }
      }
      // merge the row's ksplit sorted lists (neighbouring lanes): KMAX rounds of "best head
      // wins and is popped"; equal logits go to the lower expert index as everywhere else
      float sel_v[KMAX];
      int sel_e[KMAX];
#pragma unroll
      for (int r = 0; r < KMAX; ++r) {
        float bv = best.v[0];
        int be = best.e[0];
#pragma unroll
        for (int o = 1; o < 4; o <<= 1) {
          if (o < ksplit) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            if (better(ov, oe, bv, be)) {
              bv = ov;
              be = oe;
            }
          }
        }
        sel_v[r] = bv;
        sel_e[r] = be;
        if (best.e[0] == be && best.v[0] == bv) best.pop();  // this lane's head won
      }
      const int t = t0 + row;
      if (part == 0 && t < T) {
        float num[KMAX], den = 0.f;
#pragma unroll
        for (int r = 0; r < KMAX; ++r) {
          num[r] = (r < k) ? expf(sel_v[r] - sel_v[0]) : 0.f;
          den += num[r];
        }
#pragma unroll
        for (int r = 0; r < KMAX; ++r)
          if (r < k) {
            topk_idx[static_cast<int64_t>(t) * k + r] = sel_e[r];
            topk_w[static_cast<int64_t>(t) * k + r] = num[r] / den;
          }
      }
      // this CTA's rows of logits leave shared memory as one coalesced block
      mbar_arrive(smem_u32(&epi_bar));
      const bool synced = mbar_wait(smem_u32(&epi_bar), 0, timeout_ns, &s_abort);
      if (__all_sync(0xffffffffu, synced)) {
        const int rows = max(0, min(R, T - (t0 + rank * R)));
        float* dst = logits + static_cast<int64_t>(t0 + rank * R) * N;
        for (int i = ct; i < rows * N; i += kConvThreads) {
          const int r = i / N;
          dst[i] = fin[r * NS + (i - r * N)];
        }
        if (prob_part != nullptr &&
            !tile_prob_sums(sel_v[0], fin, rows, NS, N, ksplit, ct,
                            prob_part + static_cast<int64_t>(blockIdx.x) * N, smem_u32(&epi_bar),
                            1u, timeout_ns, &s_abort)) {
          s_abort = 1;
          report_error(status, MOE_ERR_TIMEOUT);
        }
      } else {
        s_abort = 1;
        report_error(status, MOE_ERR_TIMEOUT);
      }
    }
    __syncwarp();
    cluster_sync_all();  // every CTA has read the others' shared memory; they may exit
  }

  tc_fence_before_sync();
  if constexpr (PAIR)
    cluster_sync_all();  // neither CTA of a pair frees TMEM or exits while the other works
  else
    __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    if constexpr (PAIR)
      tmem_dealloc_pair(tmem, C::TMEM_COLS);
    else
      tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// CTAs per 128-token tile: the k blocks are split over a cluster of 2 or 4 CTAs while the
// tiles leave SMs idle and every CTA keeps at least 2 k blocks. A function of the shape only
// (SM count of a B200), so the workspace and in-kernel-split variants cut K alike and give
// identical logits.
int router_ksplit(int tiles, int num_kb) {
  constexpr int kSms = 148;
  int ks = 1;
  while (ks < 4 && static_cast<int64_t>(tiles) * ks * 2 <= kSms && num_kb >= ks * 4) ks *= 2;
  return ks;
}

// CTA pairs for the pre-split path when every tile has a CTA of its own and the tiles pair up:
// the even CTA's M = 256 MMAs take half of each term tile from each CTA's shared memory, so a
// CTA loads and its tensor core reads half the weight bytes per MMA (shared-memory bandwidth,
// not the MMA rate, bounds the unpaired kernel at N = 256).
bool router_pairs(int tiles, int num_kb, int np, bool presplit) {
  return presplit && np >= 128 && tiles % 2 == 0 && router_ksplit(tiles, num_kb) == 1;
}

template <int NP, bool PRESPLIT, int KMAX, bool PAIR>
cudaError_t launch_npk(const CUtensorMap& mx, const CUtensorMap& mw, const float* w,
                       const float* bias, float* logits, int32_t* topk_idx, float* topk_w, int T,
                       int d, int N, int k, int* status, uint64_t timeout_ns, float* prob_part, cudaStream_t s) {
  using C = RCfg<NP, PRESPLIT, PAIR>;
  auto kernel = router_tc_kernel<NP, PRESPLIT, KMAX, PAIR>;
  static PerDeviceOnce once;
  const cudaError_t attr = once.run([kernel] {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  });
  if (attr != cudaSuccess) return attr;
  const int tiles = (T + kTok - 1) / kTok;
  if constexpr (PAIR)
    return launch_pdl_cluster(kernel, dim3(tiles), dim3(kThreads), C::SMEM_BYTES, s, 2u, mx, mw, w,
                              bias, logits, topk_idx, topk_w, T, d, N, k, status, timeout_ns,
                              prob_part, 1);
  const int ksplit = router_ksplit(tiles, d / kBK);
  if (ksplit == 1)
    return launch_pdl(kernel, dim3(tiles), dim3(kThreads), C::SMEM_BYTES, s, mx, mw, w, bias,
                      logits, topk_idx, topk_w, T, d, N, k, status, timeout_ns, prob_part, 1);
  return launch_pdl_cluster(kernel, dim3(tiles * ksplit), dim3(kThreads), C::SMEM_BYTES, s,
                            static_cast<unsigned>(ksplit), mx, mw, w, bias, logits, topk_idx,
                            topk_w, T, d, N, k, status, timeout_ns, prob_part, ksplit);
}

template <int NP, bool PRESPLIT, int KMAX>
cudaError_t launch_npkp(bool pair, const CUtensorMap& mx, const CUtensorMap& mw, const float* w,
                        const float* bias, float* logits, int32_t* topk_idx, float* topk_w, int T,
                        int d, int N, int k, int* status, uint64_t timeout_ns, float* prob_part,
                        cudaStream_t s) {
  if constexpr (PRESPLIT && NP >= 128) {
    if (pair)
      return launch_npk<NP, true, KMAX, true>(mx, mw, w, bias, logits, topk_idx, topk_w, T, d, N,
                                              k, status, timeout_ns, prob_part, s);
  }
  return launch_npk<NP, PRESPLIT, KMAX, false>(mx, mw, w, bias, logits, topk_idx, topk_w, T, d, N,
                                               k, status, timeout_ns, prob_part, s);
}

template <int NP, bool PRESPLIT>
cudaError_t launch_np(bool pair, const CUtensorMap& mx, const CUtensorMap& mw, const float* w,
                      const float* bias, float* logits, int32_t* topk_idx, float* topk_w, int T,
                      int d, int N, int k, int* status, uint64_t timeout_ns, float* prob_part, cudaStream_t s) {
  if (k <= 1)
    return launch_npkp<NP, PRESPLIT, 1>(pair, mx, mw, w, bias, logits, topk_idx, topk_w, T, d, N, k, status, timeout_ns, prob_part, s);
  if (k <= 2)
    return launch_npkp<NP, PRESPLIT, 2>(pair, mx, mw, w, bias, logits, topk_idx, topk_w, T, d, N, k, status, timeout_ns, prob_part, s);
  if (k <= 4)
    return launch_npkp<NP, PRESPLIT, 4>(pair, mx, mw, w, bias, logits, topk_idx, topk_w, T, d, N, k, status, timeout_ns, prob_part, s);
  return launch_npkp<NP, PRESPLIT, 8>(pair, mx, mw, w, bias, logits, topk_idx, topk_w, T, d, N, k, status, timeout_ns, prob_part, s);
}

template <bool PRESPLIT>
cudaError_t launch_tc(bool pair, const CUtensorMap& mx, const CUtensorMap& mw, const float* w,
                      const float* bias, float* logits, int32_t* topk_idx, float* topk_w, int T,
                      int d, int N, int k, int* status, uint64_t timeout_ns, float* prob_part, cudaStream_t s) {
  if (N <= 16)
    return launch_np<16, PRESPLIT>(pair, mx, mw, w, bias, logits, topk_idx, topk_w, T, d, N, k, status, timeout_ns, prob_part, s);
  if (N <= 32)
    return launch_np<32, PRESPLIT>(pair, mx, mw, w, bias, logits, topk_idx, topk_w, T, d, N, k, status, timeout_ns, prob_part, s);
  if (N <= 64)
    return launch_np<64, PRESPLIT>(pair, mx, mw, w, bias, logits, topk_idx, topk_w, T, d, N, k, status, timeout_ns, prob_part, s);
  if (N <= 128)
    return launch_np<128, PRESPLIT>(pair, mx, mw, w, bias, logits, topk_idx, topk_w, T, d, N, k, status, timeout_ns, prob_part, s);
  return launch_np<256, PRESPLIT>(pair, mx, mw, w, bias, logits, topk_idx, topk_w, T, d, N, k, status, timeout_ns, prob_part, s);
}

bool encode_bf16(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                 const cuuint64_t* strides_bytes, const cuuint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides_bytes,
            box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t router_split_bytes(int N, int d) { return static_cast<size_t>(3) * N * d * 2; }

int router_tc_parts(int T, int d) {
  const int tiles = (T + kTok - 1) / kTok;
  return tiles * router_ksplit(tiles, d / kBK);
}

cudaError_t launch_router_tc(const uint16_t* x, const float* w_router, const float* bias,
                             float* logits, int32_t* topk_idx, float* topk_w, int T, int d, int N,
                             int k, uint16_t* split_scratch, int* status, uint64_t timeout_ns, float* prob_part,
                             cudaStream_t s) {
  CUtensorMap mx, mw;
  {
    const cuuint64_t gd[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(T)};
    const cuuint64_t gs[1] = {static_cast<cuuint64_t>(d) * 2};
    const cuuint32_t box[2] = {kBK, kTok};
    if (!encode_bf16(&mx, x, 2, gd, gs, box)) return cudaErrorInvalidValue;
  }
  const int np = N <= 16 ? 16 : N <= 32 ? 32 : N <= 64 ? 64 : N <= 128 ? 128 : 256;
  if (split_scratch == nullptr) {
    memset(&mw, 0, sizeof(mw));  // unused by the in-kernel split
    return launch_tc<false>(false, mx, mw, w_router, bias, logits, topk_idx, topk_w, T, d, N, k,
                            status, timeout_ns, prob_part, s);
  }
  const bool pair = router_pairs((T + kTok - 1) / kTok, d / kBK, np, true);
  {
    // a CTA of a pair loads rows [rank * np / 2, rank * np / 2 + np / 2) of each term
    const cuuint64_t gd[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), 3};
    const cuuint64_t gs[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(N) * d * 2};
    const cuuint32_t box[3] = {kBK, static_cast<cuuint32_t>(pair ? np / 2 : np), 1};
    if (!encode_bf16(&mw, split_scratch, 3, gd, gs, box)) return cudaErrorInvalidValue;
  }
  const int64_t n = static_cast<int64_t>(N) * d;
  const int blocks = static_cast<int>(std::min<int64_t>((n / 8 + 255) / 256, 148 * 8));
  cudaError_t e = launch_pdl(split_router_weights_kernel, dim3(blocks), dim3(256), 0, s, w_router,
                             split_scratch, n);
  if (e != cudaSuccess) return e;
  return launch_tc<true>(pair, mx, mw, w_router, bias, logits, topk_idx, topk_w, T, d, N, k,
                         status, timeout_ns, prob_part, s);
}

}  // namespace moe
