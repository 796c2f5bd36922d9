// Expert FFN of decode-sized batches on 5th-generation tensor cores (tcgen05, sm_100a), cut
// along d_ff, with every SM streaming an equal share of the weights.
//
// Page «Что такое Mixture of Experts (MoE) в трансформерах» (aglamov.biz): «Бэкенд для
// экспертов» (tokens grouped by expert, one grouped GEMM) and «Динамическая загрузка весов с
// WeightConverter» (packed gate_up_proj [N, 2F, d], gate rows first, and down_proj [N, d, F]).
// Page «Sparse Mixture-of-Experts», «Роутер и top-k gating»: the layer's output is the residual
// plus the kept experts' outputs weighted by the renormalised router probabilities.
//
// With at most 8 tokens an expert holds at most 8 rows, so the layer is a stream of the active
// experts' weights with little arithmetic per byte, and an SM streams only its share of HBM:
// the weights must be spread evenly over all SMs. A slice is 64 columns of h of one expert:
//   h[:, f0:f0+64] = silu(x W_g[f0:f0+64]^T) * (x W_u[f0:f0+64]^T), rounded once to bf16 (as
//                    the grouped FFN rounds h),
//   P = h[:, f0:f0+64] W_d[:, f0:f0+64]^T, an fp32 partial of y,
// from the slice's 64 gate rows, 64 up rows and 64 columns of W_d, each read once. A slice is
// d/64 gate/up units (k blocks of 64 gate + 64 up rows) followed by ceil(d/128) down units
// (128 rows of W_d x the slice's 64 columns). With at least as many slices as CTAs, the units
// of all slices, laid end to end, are cut into one equal range per CTA (stream-K); with fewer
// slices, each CTA takes one whole slice. A range boundary can cut a slice's gate/up units (the
// CTA before its owner, the CTA holding its last gate/up unit, then passes it an fp32 partial
// of the 128 x 16 accumulator) or its down units (the owner then publishes h and the later CTA
// reads it). Every CTA walks its slices from last to first, so the CTA that passes a partial
// or h does so at the start of its work while the CTA that needs it reaches that slice at the
// end of its own. After a grid-wide barrier, y = sum of the expert's F/64 partials, added in a
// fixed order (32 groups of consecutive slices, each group in slice order, then the groups in
// order); a gate/up accumulator split over two CTAs is the owner's k blocks plus the other
// CTA's, in that order. The split depends only on the routing and the SM count, so results do
// not depend on timing.
//
// Both GEMMs put the weights in the M operand: A = 128 weight rows (64 gate + 64 up rows, or
// 128 rows of W_d) x 64 k, B = 16 token rows (the gate/up GEMM: the expert's rows of x_perm in
// moe_grouped_ffn, or in moe_forward the batch's tokens x[0..16), as every token fits; the down
// GEMM: the slice's h from shared memory). UMMA M=128, N=16, K=16; the accumulators are 16 TMEM
// columns wide. A token column that does not belong to the expert is computed and never stored.
//
// Kernel structure (one CTA per SM, 256 threads):
//   warp 0     TMA producer through a ring of 18 KB stages (128B swizzle);
//   warp 1     allocates TMEM and issues the MMAs from one thread;
//   warps 4-7  epilogue: thread i holds TMEM lane i. Gate/up: the up half (lanes 64-127) goes
//              through shared memory to the gate half, which forms h, writes it to the bf16 B
//              tile of the down GEMM and to h in global memory. Down: each 128-row block of y's
//              partial is stored for the slice's tokens.
// Then every CTA (all 256 threads) takes part in the reduction and, in moe_forward, the combine:
// out[t] = residual[t] + sum over kept choices j, in order, of w_j y[row(t, j)] in fp32, rounded
// once (moe_unpermute_combine's arithmetic); a token with no kept pair passes the residual's
// bits through.
//
// In moe_forward the same launch first routes the batch: the first ceil(d/128) CTAs store the
// decode router's partial dot products (dr::decode_route_partials, as moe_route), and then
// every CTA adds them up and takes top-k and the capacity slots in its own shared memory
// (dr::decode_route_finish), so the routing is identical to moe_route's and no second pass
// through global memory stands before the weights start streaming.
//
// Every wait is bounded. A CTA that gives up records MOE_ERR_TIMEOUT, stops issuing work, waits
// (bounded) for its own copies and MMAs, and still takes part in the grid barrier's arrival
// count, so the others do not wait the full limit a second time.
#include <string.h>

#include <type_traits>

#include "common.cuh"
#include "decode_route.cuh"
#include "launch.h"
#include "tma_host.h"

namespace moe {
namespace {

constexpr int kDfThreads = 256;
constexpr int kDfN = 16;                 // UMMA N: token columns
constexpr int kDfBK = 64;                // k per stage
constexpr int kDfA = 128 * kDfBK * 2;    // 16 KB: 128 weight rows x 64 k, bf16
constexpr int kDfB = kDfN * kDfBK * 2;   // 2 KB: 16 token rows x 64 k
constexpr int kDfStage = kDfA + kDfB;    // 18 KB (a multiple of 1024: stages stay swizzle-aligned)
constexpr int kDfStages = 10;
constexpr int kDfYSlots = 8;             // down-GEMM accumulators in flight
constexpr int kDfTmemCols = 256;         // 2 x 16 gate/up + 8 x 16 down = 160 used
constexpr int kDfXStride = 17;           // floats per row of the up-half exchange buffer
constexpr int kDfGroups = 32;            // slice groups of the final reduction
constexpr int kDfCols = 32;              // output columns per reduction tile (8 float4)
constexpr int kDfMaxRows = kDecodeFfnMaxRows;  // rows per expert, and tokens, at most
constexpr int kDfMaxActive = 64;         // experts with rows at most (T * k <= 64)
constexpr int kDfSmem = kDfStages * kDfStage + 2 * kDfB + 64 * kDfXStride * 4 + 1024;
static_assert(kDfStage % 1024 == 0, "stage alignment");
static_assert(kDfGroups * kDfMaxRows * (kDfCols / 4) * 16 <= kDfStages * kDfStage,
              "the reduction's group sums fit in the ring");
static_assert(kDfThreads == kDfGroups * (kDfCols / 4), "one thread per (group, float4)");
static_assert(kDecodeFfnMaxT <= kDfMaxRows && kDfMaxRows <= kDfN, "rows per expert");

constexpr unsigned kFullMask = 0xffffffffu;

struct DfParams {
  const int32_t* expert_offset;  // moe_grouped_ffn: the sort's offsets (moe_forward: routed here)
  uint16_t* h;
  float* y;
  float* part;     // [F/64][r_max][d] fp32 partials of y
  float* part_gu;  // [s_max][8][128] fp32 gate/up partial a slice's owner receives
  int* flags;      // [2][s_max]: partial ready, h ready (1); zero between calls
  int* sync;       // [0] grid-barrier arrivals, [1] departures; zero between calls
  const int32_t* row_of_pair;  // combine without routing in the launch
  const float* topk_w;
  const uint16_t* residual;
  void* out;  // null: no combine
  int out_f32;
  int T, k, N, d, F;
  int64_t r_max;
  int s_max;
  int route_ctas;
  int* status;
  uint64_t timeout_ns;
  DecodeRouteArgs route;
};

__device__ __forceinline__ float silu_df(float g) { return g / (1.0f + __expf(-g)); }

__device__ __forceinline__ uint16_t bf16_bits(float v) {
  __nv_bfloat16 b = __float2bfloat16_rn(v);
  return *reinterpret_cast<uint16_t*>(&b);
}

// Barrier of the 128 epilogue threads on a reusable mbarrier (count 128), bounded.
__device__ __forceinline__ bool epi_sync(uint32_t bar, uint32_t& phase, uint64_t timeout_ns,
                                         const volatile int* abort) {
  mbar_arrive(bar);
  const bool ok = mbar_wait(bar, phase, timeout_ns, abort);
  phase ^= 1u;
  return ok;
}

__device__ __forceinline__ void st_release_gpu(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Bounded wait until *flag == want (acquire); false on timeout or when *abort is set.
__device__ __forceinline__ bool wait_flag(const int* flag, int want, uint64_t timeout_ns,
                                          const volatile int* abort) {
  if (ld_acquire_gpu(flag) == want) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (ld_acquire_gpu(flag) == want) return true;
    if (abort != nullptr && *abort != 0) return false;
    if (globaltimer_ns() - t0 > timeout_ns) return false;
    __nanosleep(32);
  }
}

__device__ __forceinline__ float4 add4(float4 a, float4 b) {
  return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

// The schedule: slices of L = KB + DB units (KB gate/up units, then DB down units), laid end to
// end. Stream-K (sk): CTA b takes units [b U / G, (b + 1) U / G); else CTA b < S takes slice b.
struct DfSched {
  int64_t L, U;
  int KB, DB, G;
  bool sk;
};
__device__ __forceinline__ int64_t df_begin(const DfSched& s, int b) {
  if (s.sk) return static_cast<int64_t>(b) * s.U / s.G;
  return min(static_cast<int64_t>(b), s.U / s.L) * s.L;
}

// CTA b's part of slice X (b's range [beg, end) intersects it).
struct DfSeg {
  int kb0, kb1;  // gate/up units of this CTA (empty: kb0 >= kb1)
  int db0, db1;  // down units of this CTA
  bool owner;    // holds the slice's last gate/up unit: forms h
  bool need_gu;  // owner whose first gate/up units are the previous CTA's: adds its partial
  bool publish;  // owner whose slice has down units in a later CTA: publishes h
};
__device__ __forceinline__ DfSeg df_seg(const DfSched& s, int64_t beg, int64_t end, int64_t X) {
  const int64_t x0 = X * s.L, g1 = x0 + s.KB, x1 = x0 + s.L;
  DfSeg g;
  g.kb0 = static_cast<int>(max(beg, x0) - x0);
  g.kb1 = static_cast<int>(max(min(end, g1) - x0, static_cast<int64_t>(g.kb0)));
  g.db0 = static_cast<int>(max(beg, g1) - g1);
  g.db1 = static_cast<int>(max(min(end, x1) - g1, static_cast<int64_t>(g.db0)));
  const bool has_gu = g.kb0 < g.kb1;
  g.owner = has_gu && end >= g1;
  g.need_gu = g.owner && beg > x0;
  g.publish = g.owner && end < x1;
  return g;
}

template <bool ROUTE, int EPT>
__global__ void __launch_bounds__(kDfThreads, 1)
    decode_ffn_kernel(const __grid_constant__ CUtensorMap tmGU, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmWD, const DfParams p) {
  extern __shared__ __align__(1024) uint8_t dyn_smem[];
  __shared__ __align__(8) uint64_t full_bar[kDfStages];
  __shared__ __align__(8) uint64_t empty_bar[kDfStages];
  __shared__ __align__(8) uint64_t gfull[2], gempty[2], hfull[2], hempty[2];
  __shared__ __align__(8) uint64_t yfull[kDfYSlots], yempty[kDfYSlots];
  __shared__ __align__(8) uint64_t epi_bar, done_bar;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  __shared__ int s_ok;
  __shared__ int s_nact;
  __shared__ int s_off[257];
  __shared__ int s_act[kDfMaxActive];
  __shared__ short s_colrow[kDfMaxActive][kDfN];  // output row of each token column, -1 if none
  __shared__ typename std::conditional<ROUTE, dr::DecodeRouteSmem<kDfMaxRows, EPT>, int>::type s_route;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t base = (smem_u32(dyn_smem) + 1023u) & ~1023u;
  uint8_t* gbase = dyn_smem + (base - smem_u32(dyn_smem));  // generic pointer of `base`
  const uint32_t ring = base;
  const uint32_t hbuf = base + kDfStages * kDfStage;  // two 2 KB h tiles (1024-aligned)
  float* xchg = reinterpret_cast<float*>(gbase + kDfStages * kDfStage + 2 * kDfB);
  const int G = static_cast<int>(gridDim.x);
  const int b = static_cast<int>(blockIdx.x);

  if (tid == 0) {
    prefetch_tensormap(&tmGU);
    prefetch_tensormap(&tmB);
    prefetch_tensormap(&tmWD);
    for (int s = 0; s < kDfStages; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&gfull[i]), 1);
      mbar_init(smem_u32(&gempty[i]), 128);
      mbar_init(smem_u32(&hfull[i]), 1);
      mbar_init(smem_u32(&hempty[i]), 1);
    }
    for (int y = 0; y < kDfYSlots; ++y) {
      mbar_init(smem_u32(&yfull[y]), 1);
      mbar_init(smem_u32(&yempty[y]), 128);
    }
    mbar_init(smem_u32(&epi_bar), 128);
    mbar_init(smem_u32(&done_bar), 1);
    s_abort = 0;
    s_ok = 1;
    fence_barrier_init();
  }
  if (warp == 1) {
    __syncwarp();
    tmem_alloc(smem_u32(&s_tmem), kDfTmemCols);
    tmem_relinquish();
  }
  pdl_wait();  // everything below reads the previous kernels' outputs or writes global memory
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = s_tmem;
  const int N = p.N;

  // ---------------------------------------------------------------- routing / the slice list
  if constexpr (ROUTE) {
    if (b < p.route_ctas) dr::decode_route_partials<kDfMaxRows, EPT>(p.route, b, p.route_ctas, s_route);
    if (tid == 0) {
      if (!wait_counter_at_least(p.route.counter, p.route_ctas, p.timeout_ns, nullptr)) {
        s_ok = 0;
        s_abort = 1;
        report_error(p.status, MOE_ERR_TIMEOUT);
      }
    }
    __syncthreads();
    if (s_ok) {
      // every CTA routes in its own shared memory; the last CTA stores the routing outputs and
      // CTA i copies the token row of arrival i into x_perm
      dr::decode_route_finish<kDfMaxRows, EPT>(p.route, p.route_ctas, s_route, b == G - 1, false);
      const int P = p.T * p.k;
      if (b < P && s_route.row[b] >= 0) {
        const int t = b % p.T;
        const uint4* src = reinterpret_cast<const uint4*>(p.route.x + static_cast<int64_t>(t) * p.d);
        uint4* dst = reinterpret_cast<uint4*>(p.route.x_perm + static_cast<int64_t>(s_route.row[b]) * p.d);
        for (int i = tid; i < p.d / 8; i += kDfThreads) dst[i] = src[i];
      }
      for (int i = tid; i <= N; i += kDfThreads) s_off[i] = s_route.off[i];
    } else {
      for (int i = tid; i <= N; i += kDfThreads) s_off[i] = 0;
    }
  } else {
    for (int i = tid; i <= N; i += kDfThreads) s_off[i] = __ldcg(p.expert_offset + i);
  }
  __syncthreads();
  if (warp == 0) {
    // experts with rows, in expert order; an expert whose rows do not fit the buffers or the
    // kernel's limits is skipped and reported
    int n = 0;
    bool bad = false;
    for (int e0 = 0; e0 < N; e0 += 32) {
      const int e = e0 + lane;
      bool act = false;
      if (e < N) {
        const int lo = s_off[e], hi = s_off[e + 1];
        const bool ok_rows = lo >= 0 && hi >= lo && hi <= p.r_max && hi - lo <= kDfMaxRows;
        act = ok_rows && hi > lo;
        bad |= !ok_rows;
      }
      const unsigned m = __ballot_sync(kFullMask, act);
      const int slot = n + __popc(m & lanemask_lt());
      if (act && slot < kDfMaxActive) s_act[slot] = e;
      n += __popc(m);
    }
    if (n > kDfMaxActive) {
      bad = true;
      n = kDfMaxActive;
    }
    if (__any_sync(kFullMask, bad) && lane == 0) report_error(p.status, MOE_ERR_BOUNDS);
    if (lane == 0) s_nact = n;
  }
  for (int i = tid; i < kDfMaxActive * kDfN; i += kDfThreads) (&s_colrow[0][0])[i] = -1;
  __syncthreads();
  // output row of each token column of each active expert
  if constexpr (ROUTE) {
    if (s_ok && tid < p.T * p.k) {  // arrival tid = j * T + t: token t's pair j
      const int row = s_route.row[tid];
      if (row >= 0) {
        const int e = s_route.pe[tid];
        for (int a = 0; a < s_nact; ++a)
          if (s_act[a] == e) s_colrow[a][tid % p.T] = static_cast<short>(row);
      }
    }
  } else {
    for (int i = tid; i < s_nact * kDfN; i += kDfThreads) {
      const int a = i / kDfN, c = i - a * kDfN;
      const int e = s_act[a];
      if (c < s_off[e + 1] - s_off[e]) s_colrow[a][c] = static_cast<short>(s_off[e] + c);
    }
  }
  __syncthreads();
  const int Fs = p.F / kDecodeFfnSlice;
  DfSched sc;
  sc.KB = p.d / kDfBK;
  sc.DB = (p.d + 127) / 128;
  sc.L = sc.KB + sc.DB;
  sc.G = G;
  const int64_t S = static_cast<int64_t>(s_nact) * Fs;
  sc.U = S * sc.L;
  sc.sk = S >= G;
  const int64_t beg = df_begin(sc, b), end = df_begin(sc, b + 1);
  const int64_t X_hi = end > beg ? (end - 1) / sc.L : -1;
  const int64_t X_lo = end > beg ? beg / sc.L : 0;
  const int target = 1;
  const bool run = s_abort == 0 && S <= p.s_max;
  if (S > p.s_max && tid == 0) report_error(p.status, MOE_ERR_BOUNDS);
  int* gu_flag = p.flags;
  int* h_flag = p.flags + p.s_max;

  if (warp == 0 && run) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      const uint64_t pol_w = l2_policy_evict_first();  // weights: read once, streamed
      const uint64_t pol_x = l2_policy_evict_last();   // token rows: read by many CTAs
      int it = 0;
      bool ok = true;
      for (int64_t X = X_hi; X >= X_lo && ok; --X) {
        const DfSeg sg = df_seg(sc, beg, end, X);
        const int a = static_cast<int>(X / Fs), j = static_cast<int>(X - static_cast<int64_t>(a) * Fs);
        const int e = s_act[a];
        const int row0 = ROUTE ? 0 : s_off[e];
        for (int kb = sg.kb0; kb < sg.kb1; ++kb, ++it) {
          const int s = it % kDfStages;
          if (!mbar_wait(smem_u32(&empty_bar[s]), ((it / kDfStages) & 1) ^ 1u, p.timeout_ns, &s_abort)) {
            ok = false;
            break;
          }
          const uint32_t st = ring + s * kDfStage, fb = smem_u32(&full_bar[s]);
          mbar_arrive_expect_tx(fb, kDfStage);
          tma_load_4d(st, &tmGU, fb, kb * kDfBK, j * 64, 0, e, pol_w);             // gate rows
          tma_load_4d(st + kDfA / 2, &tmGU, fb, kb * kDfBK, j * 64, 1, e, pol_w);  // up rows
          tma_load_2d(st + kDfA, &tmB, fb, kb * kDfBK, row0, pol_x);               // token rows
        }
        for (int db = sg.db0; db < sg.db1 && ok; ++db, ++it) {
          const int s = it % kDfStages;
          if (!mbar_wait(smem_u32(&empty_bar[s]), ((it / kDfStages) & 1) ^ 1u, p.timeout_ns, &s_abort)) {
            ok = false;
            break;
          }
          const uint32_t st = ring + s * kDfStage, fb = smem_u32(&full_bar[s]);
          mbar_arrive_expect_tx(fb, kDfA);
          tma_load_3d(st, &tmWD, fb, j * 64, db * 128, e, pol_w);
        }
      }
      if (!ok) {
        s_abort = 1;
        report_error(p.status, MOE_ERR_TIMEOUT);
      }
      // this thread's copies still in flight land before the CTA moves on (bounded)
      for (int q = max(0, it - kDfStages); q < it; ++q)
        mbar_wait(smem_u32(&full_bar[q % kDfStages]), (q / kDfStages) & 1, kDrainTimeoutNs, nullptr);
    }
  } else if (warp == 1 && run) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, kDfN);
      int it = 0, gu = 0, hc = 0, yc = 0;
      bool ok = true, issued = false;
      for (int64_t X = X_hi; X >= X_lo && ok; --X) {
        const DfSeg sg = df_seg(sc, beg, end, X);
        if (sg.kb0 < sg.kb1) {
          const int gb = gu & 1;
          if (!mbar_wait(smem_u32(&gempty[gb]), ((gu >> 1) & 1) ^ 1u, p.timeout_ns, &s_abort)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t dg = tmem + static_cast<uint32_t>(gb * kDfN);
          for (int kb = sg.kb0; kb < sg.kb1; ++kb, ++it) {
            const int s = it % kDfStages;
            if (!mbar_wait(smem_u32(&full_bar[s]), (it / kDfStages) & 1, p.timeout_ns, &s_abort)) {
              ok = false;
              break;
            }
            tc_fence_after_sync();
            const uint32_t a0 = ring + s * kDfStage, b0 = a0 + kDfA;
#pragma unroll
            for (int kk = 0; kk < kDfBK / 16; ++kk)
              tc_mma_f16(dg, smem_desc_k_sw128(a0 + kk * 32), smem_desc_k_sw128(b0 + kk * 32), idesc,
                         (kb != sg.kb0 || kk != 0) ? 1u : 0u);
            issued = true;
            tc_commit(smem_u32(&empty_bar[s]));
          }
          if (!ok) break;
          tc_commit(smem_u32(&gfull[gb]));
          ++gu;
        }
        if (sg.db0 < sg.db1) {
          const int hb = hc & 1;
          if (!mbar_wait(smem_u32(&hfull[hb]), (hc >> 1) & 1, p.timeout_ns, &s_abort)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t hd = hbuf + static_cast<uint32_t>(hb * kDfB);
          for (int db = sg.db0; db < sg.db1; ++db, ++it) {
            const int s = it % kDfStages, ys = yc % kDfYSlots;
            if (!mbar_wait(smem_u32(&full_bar[s]), (it / kDfStages) & 1, p.timeout_ns, &s_abort) ||
                !mbar_wait(smem_u32(&yempty[ys]), ((yc / kDfYSlots) & 1) ^ 1u, p.timeout_ns, &s_abort)) {
              ok = false;
              break;
            }
            tc_fence_after_sync();
            const uint32_t a0 = ring + s * kDfStage;
            const uint32_t dy = tmem + static_cast<uint32_t>((2 + ys) * kDfN);
#pragma unroll
            for (int kk = 0; kk < kDfBK / 16; ++kk)
              tc_mma_f16(dy, smem_desc_k_sw128(a0 + kk * 32), smem_desc_k_sw128(hd + kk * 32), idesc,
                         kk != 0 ? 1u : 0u);
            issued = true;
            tc_commit(smem_u32(&empty_bar[s]));
            tc_commit(smem_u32(&yfull[ys]));
            ++yc;
          }
          if (!ok) break;
          tc_commit(smem_u32(&hempty[hb]));
          ++hc;
        }
      }
      if (!ok) {
        s_abort = 1;
        report_error(p.status, MOE_ERR_TIMEOUT);
      }
      if (issued) {  // every issued MMA has finished before TMEM or the ring is reused
        tc_commit(smem_u32(&done_bar));
        mbar_wait(smem_u32(&done_bar), 0, kDrainTimeoutNs, nullptr);
      }
    }
  } else if (warp >= 4 && run) {
    // ---------------------------------------------------------- epilogue (warps 4-7)
    const int et = tid - 128;  // TMEM lane of this thread
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    int gu = 0, hc = 0, yc = 0;
    uint32_t epi_phase = 0;
    bool ok = true;
    for (int64_t X = X_hi; X >= X_lo && ok; --X) {
      const DfSeg sg = df_seg(sc, beg, end, X);
      const int a = static_cast<int>(X / Fs), j = static_cast<int>(X - static_cast<int64_t>(a) * Fs);
      const bool has_d = sg.db0 < sg.db1;
      const int hb = hc & 1;
      const int f = j * 64 + et;  // the h column of gate-half thread et
      if (sg.kb0 < sg.kb1) {
        const int gb = gu & 1;
        bool got = mbar_wait(smem_u32(&gfull[gb]), (gu >> 1) & 1, p.timeout_ns, &s_abort);
        if (!__all_sync(kFullMask, got)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        uint32_t v[16];
        tmem_ld_32x32b_x16(tmem + lane_base + static_cast<uint32_t>(gb * kDfN), v);
        tmem_ld_wait();
        tc_fence_before_sync();
        mbar_arrive(smem_u32(&gempty[gb]));
        ++gu;
        float* pg = p.part_gu + X * (kDfMaxRows * 128) + et;
        if (!sg.owner) {
          // the slice's owner (the next CTA) finishes the accumulator: pass this partial on
#pragma unroll
          for (int c = 0; c < kDfMaxRows; ++c) pg[c * 128] = __uint_as_float(v[c]);
          __threadfence();
          if (!epi_sync(smem_u32(&epi_bar), epi_phase, p.timeout_ns, &s_abort)) {
            ok = false;
            break;
          }
          if (et == 0) st_release_gpu(gu_flag + X, target);
          continue;
        }
        if (sg.need_gu) {
          // the previous CTA's partial of this slice's first k blocks (it passed it at the
          // start of its work; this CTA reaches the slice at the end of its own)
          if (et == 0 && !wait_flag(gu_flag + X, target, p.timeout_ns, &s_abort)) s_abort = 1;
          if (!epi_sync(smem_u32(&epi_bar), epi_phase, p.timeout_ns, &s_abort) || s_abort) {
            ok = false;
            break;
          }
#pragma unroll
          for (int c = 0; c < kDfMaxRows; ++c)
            v[c] = __float_as_uint(__uint_as_float(v[c]) + __ldcg(pg + c * 128));
        }
        if (et >= 64) {
#pragma unroll
          for (int t = 0; t < kDfN; ++t) xchg[(et - 64) * kDfXStride + t] = __uint_as_float(v[t]);
        }
        if (!epi_sync(smem_u32(&epi_bar), epi_phase, p.timeout_ns, &s_abort)) {
          ok = false;
          break;
        }
        if (et < 64) {
          got = !has_d || mbar_wait(smem_u32(&hempty[hb]), ((hc >> 1) & 1) ^ 1u, p.timeout_ns, &s_abort);
          if (__all_sync(kFullMask, got)) {
            uint8_t* ht = gbase + (hbuf - base) + hb * kDfB;
#pragma unroll
            for (int t = 0; t < kDfN; ++t) {
              const uint16_t hv =
                  bf16_bits(silu_df(__uint_as_float(v[t])) * xchg[et * kDfXStride + t]);
              // K-major 128B-swizzled tile: row t (token column), chunk et/8 XOR (t mod 8)
              if (has_d)
                *reinterpret_cast<uint16_t*>(ht + t * 128 + ((((et >> 3) ^ (t & 7))) << 4) + (et & 7) * 2) = hv;
              const int row = s_colrow[a][t];
              if (row >= 0) p.h[static_cast<int64_t>(row) * p.F + f] = hv;
            }
            if (has_d) fence_proxy_async_smem();  // generic writes -> visible to the tensor core
            if (sg.publish) __threadfence();      // h rows before the flag below
          } else {
            s_abort = 1;
          }
        }
        if (!epi_sync(smem_u32(&epi_bar), epi_phase, p.timeout_ns, &s_abort) || s_abort) {
          ok = false;
          break;
        }
        if (et == 0 && sg.publish) st_release_gpu(h_flag + X, target);
      } else if (has_d) {
        // down units only: h of this slice from global memory, published by its owner
        if (et == 0 && !wait_flag(h_flag + X, target, p.timeout_ns, &s_abort)) s_abort = 1;
        if (!epi_sync(smem_u32(&epi_bar), epi_phase, p.timeout_ns, &s_abort) || s_abort) {
          ok = false;
          break;
        }
        if (et < 64) {
          const bool got = mbar_wait(smem_u32(&hempty[hb]), ((hc >> 1) & 1) ^ 1u, p.timeout_ns, &s_abort);
          if (__all_sync(kFullMask, got)) {
            uint8_t* ht = gbase + (hbuf - base) + hb * kDfB;
#pragma unroll
            for (int t = 0; t < kDfN; ++t) {
              const int row = s_colrow[a][t];
              const uint16_t hv = row >= 0 ? __ldcg(p.h + static_cast<int64_t>(row) * p.F + f) : uint16_t(0);
              *reinterpret_cast<uint16_t*>(ht + t * 128 + ((((et >> 3) ^ (t & 7))) << 4) + (et & 7) * 2) = hv;
            }
            fence_proxy_async_smem();
          } else {
            s_abort = 1;
          }
        }
        if (!epi_sync(smem_u32(&epi_bar), epi_phase, p.timeout_ns, &s_abort) || s_abort) {
          ok = false;
          break;
        }
      }
      if (has_d) {
        if (et == 0) mbar_arrive(smem_u32(&hfull[hb]));
        ++hc;
        for (int db = sg.db0; db < sg.db1; ++db) {
          const int ys = yc % kDfYSlots;
          const bool got = mbar_wait(smem_u32(&yfull[ys]), (yc / kDfYSlots) & 1, p.timeout_ns, &s_abort);
          if (!__all_sync(kFullMask, got)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          uint32_t v[16];
          tmem_ld_32x32b_x16(tmem + lane_base + static_cast<uint32_t>((2 + ys) * kDfN), v);
          tmem_ld_wait();
          tc_fence_before_sync();
          mbar_arrive(smem_u32(&yempty[ys]));
          ++yc;
          const int drow = db * 128 + et;
          if (drow < p.d) {
            float* dst = p.part + static_cast<int64_t>(j) * p.r_max * p.d + drow;
#pragma unroll
            for (int t = 0; t < kDfN; ++t) {
              const int row = s_colrow[a][t];
              if (row >= 0) dst[static_cast<int64_t>(row) * p.d] = __uint_as_float(v[t]);
            }
          }
        }
      }
    }
    if (!ok) {
      s_abort = 1;
      report_error(p.status, MOE_ERR_TIMEOUT);
    }
  }

  // ---------------------------------------------------------------- grid barrier
  // every CTA's partials are stored; every CTA is resident (one per SM, grid <= SMs), so the
  // arrival count reaches the grid size unless a CTA gave up, which the limit bounds
  __threadfence();
  tc_fence_before_sync();
  __syncthreads();
  pdl_trigger();  // all of this grid is resident: the next kernel may start its prologue
  if (tid == 0) {
    atomicAdd(p.sync + 0, 1);
    const bool all = s_abort == 0 && wait_counter_at_least(p.sync + 0, G, p.timeout_ns, &s_abort);
    s_ok = all ? 1 : 0;
    if (!all) report_error(p.status, MOE_ERR_TIMEOUT);
  }
  __syncthreads();

  // ---------------------------------------------------------------- reduction (and combine)
  if (s_ok) {
    const int d = p.d, k = p.k;
    const int nct = (d + kDfCols - 1) / kDfCols;
    const int g = tid >> 3, q = tid & 7;
    const int j0 = g * Fs / kDfGroups, j1 = (g + 1) * Fs / kDfGroups;
    float4* red = reinterpret_cast<float4*>(gbase);  // [group][row][q], the ring is idle now
    const bool combine = p.out != nullptr;
    const int R = s_off[N] < 0 ? 0 : (s_off[N] > p.r_max ? static_cast<int>(p.r_max) : s_off[N]);
    const int64_t tiles = static_cast<int64_t>(combine ? p.T : R) * nct;
    const int64_t stride = p.r_max * static_cast<int64_t>(d);
    for (int64_t tile = b; tile < tiles; tile += G) {
      const int u = static_cast<int>(tile / nct), ct = static_cast<int>(tile - static_cast<int64_t>(u) * nct);
      const int col = ct * kDfCols + q * 4;
      const bool cok = col < d;
      int rows[kDfMaxRows];
      float wts[kDfMaxRows];
      int nr = 1;
      rows[0] = u;
      wts[0] = 0.f;
      if (combine) {
        nr = k;
#pragma unroll
        for (int jj = 0; jj < kDfMaxRows; ++jj) {
          rows[jj] = -1;
          wts[jj] = 0.f;
          if (jj < k) {
            int row;
            if constexpr (ROUTE) {
              row = s_route.row[jj * p.T + u];
              wts[jj] = s_route.tw[u * k + jj];
            } else {
              const int64_t pq = static_cast<int64_t>(u) * k + jj;
              row = __ldcg(p.row_of_pair + pq);
              wts[jj] = __ldcg(p.topk_w + pq);
            }
            if (row >= p.r_max) {
              if (tid == 0) report_error(p.status, MOE_ERR_BOUNDS);
              row = -1;
            }
            rows[jj] = row;
          }
        }
      }
      // group g's sum of the slices [j0, j1) of each row, its loads in flight together
#pragma unroll
      for (int jj = 0; jj < kDfMaxRows; ++jj) {
        if (jj >= nr) break;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (rows[jj] >= 0 && cok) {
          const float* src = p.part + static_cast<int64_t>(rows[jj]) * d + col;
          for (int jb = j0; jb < j1; jb += 8) {
            float4 v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
              if (jb + i < j1) v[i] = __ldcg(reinterpret_cast<const float4*>(src + (jb + i) * stride));
#pragma unroll
            for (int i = 0; i < 8; ++i)
              if (jb + i < j1) acc = add4(acc, v[i]);
          }
        }
        red[(g * kDfMaxRows + jj) * 8 + q] = acc;
      }
      __syncthreads();
      if (g == 0 && cok) {
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
        bool any = false;
        for (int jj = 0; jj < nr; ++jj) {
          if (rows[jj] < 0) continue;
          float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int g2 = 0; g2 < kDfGroups; ++g2)
            if (g2 * Fs / kDfGroups < (g2 + 1) * Fs / kDfGroups) y = add4(y, red[(g2 * kDfMaxRows + jj) * 8 + q]);
          *reinterpret_cast<float4*>(p.y + static_cast<int64_t>(rows[jj]) * d + col) = y;
          if (combine) {  // choices in ascending order, as moe_unpermute_combine
            const float wj = wts[jj];
            a0 = fmaf(wj, y.x, a0);
            a1 = fmaf(wj, y.y, a1);
            a2 = fmaf(wj, y.z, a2);
            a3 = fmaf(wj, y.w, a3);
            any = true;
          }
        }
        if (combine) {
          uint2 rb = make_uint2(0u, 0u);
          if (p.residual != nullptr)
            rb = *reinterpret_cast<const uint2*>(p.residual + static_cast<int64_t>(u) * d + col);
          const float r0 = __uint_as_float(rb.x << 16), r1 = __uint_as_float(rb.x & 0xffff0000u);
          const float r2 = __uint_as_float(rb.y << 16), r3 = __uint_as_float(rb.y & 0xffff0000u);
          if (p.out_f32) {
            float4 o = any ? make_float4(r0 + a0, r1 + a1, r2 + a2, r3 + a3) : make_float4(r0, r1, r2, r3);
            *reinterpret_cast<float4*>(static_cast<float*>(p.out) + static_cast<int64_t>(u) * d + col) = o;
          } else {
            // a token with no kept pair passes the residual's bits through unchanged
            const uint2 o = any ? make_uint2(pack_bf16x2(r0 + a0, r1 + a1), pack_bf16x2(r2 + a2, r3 + a3)) : rb;
            *reinterpret_cast<uint2*>(static_cast<uint16_t*>(p.out) + static_cast<int64_t>(u) * d + col) = o;
          }
        }
      }
      __syncthreads();
    }
  }

  // ---------------------------------------------------------------- departure
  // every flag is read before the grid barrier: each CTA clears the ones it set, and the last
  // CTA out puts the counters back to zero, for the next call
  __syncthreads();
  if (tid == 0 && run) {
    for (int64_t X = X_hi; X >= X_lo; --X) {
      const DfSeg sg = df_seg(sc, beg, end, X);
      if (sg.kb0 < sg.kb1 && !sg.owner) gu_flag[X] = 0;
      if (sg.publish) h_flag[X] = 0;
    }
  }
  if (tid == 0) {
    __threadfence();
    if (atomicAdd(p.sync + 1, 1) == G - 1) {
      p.sync[0] = 0;
      p.sync[1] = 0;
      if constexpr (ROUTE) *p.route.counter = 0;
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kDfTmemCols);
  }
}

template <bool ROUTE, int EPT>
cudaError_t launch_variant(const CUtensorMap& gu, const CUtensorMap& x, const CUtensorMap& wd,
                           const DfParams& p, int grid, cudaStream_t s) {
  auto kern = decode_ffn_kernel<ROUTE, EPT>;
  static PerDeviceOnce once;
  const cudaError_t attr = once.run([] {
    return cudaFuncSetAttribute(decode_ffn_kernel<ROUTE, EPT>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, kDfSmem);
  });
  if (attr != cudaSuccess) return attr;
  // the grid barrier needs every CTA resident at once: one per SM must fit
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kDfThreads, kDfSmem);
  if (e != cudaSuccess) return e;
  DeviceInfo di;
  e = device_info(&di);
  if (e != cudaSuccess) return e;
  if (static_cast<int64_t>(per_sm) * di.sm_count < grid) return cudaErrorInvalidConfiguration;
  return launch_pdl(kern, dim3(grid), dim3(kDfThreads), kDfSmem, s, gu, x, wd, p);
}

}  // namespace

cudaError_t launch_decode_ffn(const DecodeFfnArgs& a, cudaStream_t s) {
  if (!use_decode_ffn(a.T, MOE_ACT_SWIGLU, a.r_max) || a.N > 256 || a.k > 8 || a.d % 64 != 0 ||
      a.F % 64 != 0 || a.part == nullptr || a.part_gu == nullptr || a.flags == nullptr ||
      a.sync == nullptr)
    return cudaErrorInvalidValue;
  DeviceInfo di;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  const uint64_t d = static_cast<uint64_t>(a.d), F = static_cast<uint64_t>(a.F);
  const uint64_t N = static_cast<uint64_t>(a.N);
  CUtensorMap mGU, mB, mWD;
  {  // gate and up rows of one expert: [N][2][F][d], boxes of 64 k x 64 rows
    const uint64_t dims[4] = {d, F, 2, N};
    const uint64_t str[3] = {d * 2, F * d * 2, 2 * F * d * 2};
    const uint32_t box[4] = {kDfBK, 64, 1, 1};
    if (!make_map(&mGU, a.w_gate_up, 4, dims, str, box)) return cudaErrorInvalidValue;
  }
  {  // token rows, boxes of 64 k x 16 rows (rows past the end read as zero): the expert's rows
     // of x_perm, or with the routing in the launch the batch's tokens x[0..T)
    const void* rows = a.route_in_kernel ? static_cast<const void*>(a.route.x) : a.x_perm;
    const uint64_t nrows = a.route_in_kernel ? static_cast<uint64_t>(a.T) : static_cast<uint64_t>(a.r_max);
    const uint64_t dims[2] = {d, nrows};
    const uint64_t str[1] = {d * 2};
    const uint32_t box[2] = {kDfBK, kDfN};
    if (!make_map(&mB, rows, 2, dims, str, box)) return cudaErrorInvalidValue;
  }
  {  // W_d [N][d][F], boxes of 64 columns of F x 128 rows of d (rows past d read as zero)
    const uint64_t dims[3] = {F, d, N};
    const uint64_t str[2] = {F * 2, d * F * 2};
    const uint32_t box[3] = {kDfBK, 128, 1};
    if (!make_map(&mWD, a.w_down, 3, dims, str, box)) return cudaErrorInvalidValue;
  }
  DfParams p{};
  p.expert_offset = a.expert_offset;
  p.h = a.h;
  p.y = a.y_perm;
  p.part = a.part;
  p.part_gu = a.part_gu;
  p.flags = a.flags;
  p.sync = a.sync;
  p.row_of_pair = a.row_of_pair;
  p.topk_w = a.topk_w;
  p.residual = a.residual;
  p.out = a.out;
  p.out_f32 = a.out_f32;
  p.T = a.T;
  p.k = a.k;
  p.N = a.N;
  p.d = a.d;
  p.F = a.F;
  p.r_max = a.r_max;
  p.s_max = static_cast<int>(decode_ffn_max_slices(a.N, a.T, a.k, a.F));
  p.status = a.status;
  p.timeout_ns = a.timeout_ns;
  const int grid = di.sm_count;
  if (!a.route_in_kernel)
    return launch_variant<false, 1>(mGU, mB, mWD, p, grid, s);
  p.route = a.route;
  p.route_ctas = static_cast<int>((a.d + kDecodeSlice - 1) / kDecodeSlice);
  if (p.route_ctas > grid || !use_decode_route(a.T, a.N, a.d) || a.route.x_perm == nullptr ||
      static_cast<int64_t>(a.T) * a.k > grid)
    return cudaErrorInvalidValue;
  const int ept = a.N <= 32 ? 1 : a.N <= 64 ? 2 : a.N <= 128 ? 4 : 8;
  if (ept == 1) return launch_variant<true, 1>(mGU, mB, mWD, p, grid, s);
  if (ept == 2) return launch_variant<true, 2>(mGU, mB, mWD, p, grid, s);
  if (ept == 4) return launch_variant<true, 4>(mGU, mB, mWD, p, grid, s);
  return launch_variant<true, 8>(mGU, mB, mWD, p, grid, s);
}

}  // namespace moe
