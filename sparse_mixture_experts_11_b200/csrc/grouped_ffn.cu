// Grouped expert FFN on 5th-generation tensor cores (tcgen05, sm_100a).
//
// Page «Что такое Mixture of Experts (MoE) в трансформерах» (aglamov.biz):
//   «Динамическая загрузка весов с WeightConverter»: the experts' weights are packed into one
//     contiguous tensor per projection: gate_up_proj = every expert's w1 (gate) rows followed by
//     its w3 (up) rows, [N, 2F, d]; down_proj = [N, d, F];
//   «Бэкенд для экспертов», grouped_mm: tokens sorted by expert id run as a single grouped GEMM.
// Page «Sparse Mixture-of-Experts», «Архитектура и ключевые особенности»: an expert is an
// ordinary transformer FFN.
//
// Two launches of one persistent kernel template:
//   1. h = act(x_perm W_gu^T) per expert: SwiGLU silu(x W_g^T) * (x W_u^T), or GELU (erf form);
//      bf16 inputs, fp32 accumulation in TMEM, activation in fp32, h rounded once to bf16.
//   2. y_perm = h W_d^T per expert, fp32 out.
//
// Kernel structure (one CTA per SM, 192 threads):
//   warp 0      TMA producer: A tile [128 rows x 64 k] of the expert's rows and the weight tile
//               [UMMA_N rows x 64 k] into a STAGES-deep ring of 128B-swizzled shared-memory
//               stages (mbarrier full/empty pairs). For SwiGLU one B tile is the gate rows
//               [f0, f0+BN) stacked on the up rows [f0, f0+BN) of the same expert, so one MMA
//               chain produces both halves of the activation's input side by side.
//   warp 1      allocates TMEM (two accumulator buffers) and issues tcgen05.mma (M=128,
//               N=UMMA_N, K=16, four per stage) from one thread; tcgen05.commit frees smem
//               stages and publishes finished accumulators.
//   warps 2-5   epilogue: tcgen05.ld of the accumulator (thread i owns row i of the tile),
//               activation, conversion and masked global stores; then hand the TMEM buffer
//               back, so the epilogue of tile i overlaps the mainloop of tile i+1.
// Tile scheduler: tiles are (expert, n-tile, m-tile) with m fastest, numbered expert by
// expert; the per-expert tile counts come from expert_offset on the device (no host sync),
// and CTAs stride through the tile list. Experts without rows produce no tiles.
// Every mbarrier wait is bounded; on timeout the CTA records MOE_ERR_TIMEOUT, stops issuing
// work, waits (bounded) for its own TMA copies and MMAs, frees TMEM and exits.
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace moe {
namespace {

// Rows per tile (UMMA M) is a template parameter BM: 128, or 64 when no expert can hold more
// than 64 rows. For M = 64 the accumulator's row 16q + i (i < 16) sits in TMEM lane 32q + i.
constexpr int BK = 64;        // k per stage: 64 bf16 = one 128-byte swizzle row
constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;
constexpr int kSmemBudget = 200 * 1024;

enum { EPI_SWIGLU = 0, EPI_GELU = 1, EPI_STORE_F32 = 2 };

struct GemmParams {
  const int32_t* expert_offset;  // [N+1]
  void* out;                     // h (bf16) or y_perm (fp32)
  int64_t ld_out;                // row stride of out, elements
  int64_t r_max;
  int n_experts;
  int n_out;       // valid output columns per expert (multiple of 16)
  int n_tiles_n;   // ceil(n_out / BN_OUT)
  int num_kb;      // K / BK
  int* status;
  uint64_t timeout_ns;
  int weight_policy;  // 0 evict_normal, 1 evict_first
  // split-K (decode-sized batches): up to max_splits units per tile, each over a slice of K.
  // Every unit stores its fp32 partial tile into part[split][row][col]; the CTA whose unit
  // completes a tile last (per-tile arrival counter) adds the partials in order of split and
  // writes the tile's output. The counters are zero between calls.
  int max_splits;
  float* part;
  int part_ld;          // columns of a partial row: 2F (gate | up), F, or d
  int* tile_counters;
};

constexpr int pow2_at_least(int v) {
  int p = 32;
  while (p < v) p <<= 1;
  return p;
}

template <int EPI, int BN_OUT, int BM>
struct Cfg {
  static constexpr int UMMA_N = (EPI == EPI_SWIGLU) ? 2 * BN_OUT : BN_OUT;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = UMMA_N * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = (kSmemBudget / STAGE_BYTES) > 8 ? 8 : (kSmemBudget / STAGE_BYTES);
  static constexpr int TMEM_COLS = pow2_at_least(2 * UMMA_N);
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024;  // + alignment slack
  static_assert(UMMA_N % 16 == 0 && UMMA_N >= 16 && UMMA_N <= 256, "UMMA N for M=128");
  static_assert(TMEM_COLS <= 512, "two accumulators must fit in TMEM");
  static_assert(BN_OUT % 16 == 0, "epilogue works in 16-column groups");
  static_assert(STAGES >= 2, "pipeline depth");
  static_assert(BM == 64 || BM == 128, "UMMA M");
};

__device__ __forceinline__ uint64_t make_policy(int which) {
  uint64_t p;
  if (which == 1)
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  else if (which == 2)
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  else
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
  return p;
}

struct TileCoord {
  int e;      // expert
  int m0;     // first row of the tile (global row in x_perm / h)
  int rows;   // valid rows in the tile (<= BM)
  int n0;     // first output column
};

template <int BM>
__device__ __forceinline__ TileCoord decode_tile(int tile, int N, int bn_out,
                                                 const int* s_tile_start, const int* s_off) {
  int lo = 0, hi = N - 1;  // largest e with s_tile_start[e] <= tile
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_tile_start[mid] <= tile)
      lo = mid;
    else
      hi = mid - 1;
  }
  TileCoord c;
  c.e = lo;
  const int local = tile - s_tile_start[lo];
  const int m_e = s_off[lo + 1] - s_off[lo];
  const int mt = (m_e + BM - 1) / BM;
  const int nt = local / mt;
  const int mi = local - nt * mt;
  c.m0 = s_off[lo] + mi * BM;
  c.rows = min(BM, s_off[lo + 1] - c.m0);
  c.n0 = nt * bn_out;
  return c;
}

// Number of K slices per tile. With equal units dealt out in turn to `grid` CTAs, the busiest
// CTA runs ceil(units / grid) units of (num_kb / splits + kUnitOverheadKb) k-block times; the
// count minimising that wins, a larger one only when it is at least 5 % faster. Units keep at
// least 2 k blocks. The same pure function of (tiles, grid) on every CTA, so all agree.
constexpr float kUnitOverheadKb = 2.0f;  // epilogue, partial round trip and pipeline refill

__device__ __forceinline__ int choose_splits(int tiles, int grid, int num_kb, int max_splits) {
  if (max_splits <= 1 || tiles <= 0) return 1;
  auto cost = [=](int sp) {
    const int waves = (tiles * sp + grid - 1) / grid;
    return static_cast<float>(waves) * (static_cast<float>(num_kb) / sp + kUnitOverheadKb);
  };
  int best = 1;
  float best_cost = cost(1);
  for (int sp = 2; sp <= max_splits && num_kb / sp >= 2; ++sp) {
    const float c = cost(sp);
    if (c < 0.95f * best_cost) {
      best = sp;
      best_cost = c;
    }
  }
  return best;
}

// Barrier of the 128 epilogue threads on a reusable mbarrier (count 128), bounded like every
// other wait so that no thread can be left waiting for a warp that gave up.
__device__ __forceinline__ bool epilogue_sync(uint32_t bar, uint32_t& phase, uint64_t timeout_ns,
                                              const volatile int* abort) {
  mbar_arrive(bar);
  const bool ok = mbar_wait(bar, phase, timeout_ns, abort);
  phase ^= 1u;
  return ok;
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + __expf(-g)); }
__device__ __forceinline__ float gelu_f(float z) {
  return 0.5f * z * (1.0f + erff(z * 0.7071067811865476f));
}

__device__ __forceinline__ void store_f32x16(float* dst, const float (&a)[16]) {
  float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) d4[i] = make_float4(a[4 * i], a[4 * i + 1], a[4 * i + 2], a[4 * i + 3]);
}

// Final values of 4 consecutive output columns of one row (same rules as store_final16).
template <int EPI>
__device__ __forceinline__ void store_final4(const GemmParams& p, int64_t row, int col,
                                             const float4& a, const float4& b) {
  if (EPI == EPI_STORE_F32) {
    *reinterpret_cast<float4*>(static_cast<float*>(p.out) + row * p.ld_out + col) = a;
  } else {
    uint2 packed;
    if (EPI == EPI_SWIGLU) {
      packed.x = pack_bf16x2(silu_f(a.x) * b.x, silu_f(a.y) * b.y);
      packed.y = pack_bf16x2(silu_f(a.z) * b.z, silu_f(a.w) * b.w);
    } else {
      packed.x = pack_bf16x2(gelu_f(a.x), gelu_f(a.y));
      packed.y = pack_bf16x2(gelu_f(a.z), gelu_f(a.w));
    }
    *reinterpret_cast<uint2*>(static_cast<uint16_t*>(p.out) + row * p.ld_out + col) = packed;
  }
}

// Final values of 16 consecutive output columns of one row: SwiGLU h = silu(g) * u and GELU
// h = gelu(z) rounded once to bf16; the down projection stored as fp32.
template <int EPI>
__device__ __forceinline__ void store_final16(const GemmParams& p, int64_t row, int col,
                                              const float (&a)[16], const float (&b)[16]) {
  if (EPI == EPI_STORE_F32) {
    store_f32x16(static_cast<float*>(p.out) + row * p.ld_out + col, a);
  } else {
    uint32_t packed[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (EPI == EPI_SWIGLU)
        packed[i] = pack_bf16x2(silu_f(a[2 * i]) * b[2 * i], silu_f(a[2 * i + 1]) * b[2 * i + 1]);
      else
        packed[i] = pack_bf16x2(gelu_f(a[2 * i]), gelu_f(a[2 * i + 1]));
    }
    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + row * p.ld_out + col);
    dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
  }
}

template <int EPI, int BN_OUT, int BM>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB, const GemmParams p) {
  using C = Cfg<EPI, BN_OUT, BM>;
  extern __shared__ __align__(1024) uint8_t dyn_smem[];
  __shared__ __align__(8) uint64_t full_bar[C::STAGES];
  __shared__ __align__(8) uint64_t empty_bar[C::STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t done_bar;
  __shared__ __align__(8) uint64_t epi_bar;
  __shared__ uint32_t s_tmem_base;
  __shared__ volatile int s_abort;
  __shared__ int s_tile_start[257];
  __shared__ int s_off[257];
  __shared__ int s_splits;
  __shared__ int s_fixup;

  pdl_trigger();
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int N = p.n_experts;
  const uint32_t tiles = (smem_u32(dyn_smem) + 1023u) & ~1023u;

  if (threadIdx.x == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&tfull_bar[b]), 1);
      mbar_init(smem_u32(&tempty_bar[b]), kEpiThreads);
    }
    mbar_init(smem_u32(&done_bar), 1);
    mbar_init(smem_u32(&epi_bar), kEpiThreads);
    s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    __syncwarp();
    tmem_alloc(smem_u32(&s_tmem_base), C::TMEM_COLS);
    tmem_relinquish();
  }
  pdl_wait();  // below: reads of the previous kernels' outputs and writes to global memory
  if (warp == 2) {
    // Per-expert tile counts and their exclusive prefix (experts lane*per .. lane*per+per-1).
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
        if (a < 0 || b < a || b > p.r_max) {
          bad = true;
        } else {
          cnt[i] = ((b - a + BM - 1) / BM) * p.n_tiles_n;
        }
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
        s_tile_start[e] = run;
        run += cnt[i];
      }
    }
    if (lane == 31) {
      s_tile_start[N] = incl;
      s_splits = choose_splits(incl, gridDim.x, p.num_kb, p.max_splits);
    }
    if (bad) report_error(p.status, MOE_ERR_BOUNDS);  // such an expert gets no tiles
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();

  const uint32_t tmem_base = s_tmem_base;
  const int total_tiles = s_tile_start[N];
  const int splits = s_splits;
  const int total_units = total_tiles * splits;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      const uint64_t pol_a = make_policy(2);
      const uint64_t pol_b = make_policy(p.weight_policy);
      int it = 0;
      bool ok = true;
      for (int unit = blockIdx.x; ok && unit < total_units; unit += gridDim.x) {
        const int tile = unit / splits, sp = unit - tile * splits;
        const TileCoord c = decode_tile<BM>(tile, N, BN_OUT, s_tile_start, s_off);
        const int kb0 = sp * p.num_kb / splits, kb1 = (sp + 1) * p.num_kb / splits;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % C::STAGES;
          const uint32_t ph = (it / C::STAGES) & 1;
          if (!mbar_wait(smem_u32(&empty_bar[s]), ph ^ 1u, p.timeout_ns, &s_abort)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&full_bar[s]);
          const uint32_t a_dst = tiles + s * C::STAGE_BYTES;
          const uint32_t b_dst = a_dst + C::A_BYTES;
          mbar_arrive_expect_tx(fb, C::STAGE_BYTES);
          tma_load_2d(a_dst, &tmA, fb, kb * BK, c.m0, pol_a);
          if (EPI == EPI_SWIGLU) {
            tma_load_4d(b_dst, &tmB, fb, kb * BK, c.n0, 0, c.e, pol_b);
            tma_load_4d(b_dst + BN_OUT * BK * 2, &tmB, fb, kb * BK, c.n0, 1, c.e, pol_b);
          } else {
            tma_load_3d(b_dst, &tmB, fb, kb * BK, c.n0, c.e, pol_b);
          }
        }
      }
      if (!ok) {
        s_abort = 1;
        report_error(p.status, MOE_ERR_TIMEOUT);
      }
      // No TMA write may still be landing in shared memory when the CTA exits.
      for (int i = max(0, it - C::STAGES); i < it; ++i)
        mbar_wait(smem_u32(&full_bar[i % C::STAGES]), (i / C::STAGES) & 1, kDrainTimeoutNs, nullptr);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, C::UMMA_N);
      int it = 0, tc = 0;
      bool ok = true;
      bool issued = false;
      for (int unit = blockIdx.x; ok && unit < total_units; unit += gridDim.x, ++tc) {
        const int sp = unit % splits;
        const int kb0 = sp * p.num_kb / splits, kb1 = (sp + 1) * p.num_kb / splits;
        const int buf = tc & 1;
        const uint32_t tph = (tc >> 1) & 1;
        if (!mbar_wait(smem_u32(&tempty_bar[buf]), tph ^ 1u, p.timeout_ns, &s_abort)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * C::UMMA_N);
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % C::STAGES;
          const uint32_t ph = (it / C::STAGES) & 1;
          if (!mbar_wait(smem_u32(&full_bar[s]), ph, p.timeout_ns, &s_abort)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_base = tiles + s * C::STAGE_BYTES;
          const uint32_t b_base = a_base + C::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            tc_mma_f16(d_tmem, smem_desc_k_sw128(a_base + kk * 32), smem_desc_k_sw128(b_base + kk * 32),
                       idesc, (kb != kb0 || kk != 0) ? 1u : 0u);
          }
          issued = true;
          tc_commit(smem_u32(&empty_bar[s]));
        }
        if (!ok) break;
        tc_commit(smem_u32(&tfull_bar[buf]));
      }
      if (!ok) {
        s_abort = 1;
        report_error(p.status, MOE_ERR_TIMEOUT);
        if (issued) {  // let every issued MMA finish before TMEM is freed
          tc_commit(smem_u32(&done_bar));
          mbar_wait(smem_u32(&done_bar), 0, kDrainTimeoutNs, nullptr);
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue (warps 2..5)
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    // tile row held by this thread's TMEM lane (M = 64 uses lanes 0-15 of each quadrant)
    const int r_local = BM == 128 ? q * 32 + lane : (lane < 16 ? q * 16 + lane : BM);
    int tc = 0;
    uint32_t epi_phase = 0;
    bool ok = true;
    for (int unit = blockIdx.x; unit < total_units; unit += gridDim.x, ++tc) {
      const int tile = unit / splits, sp = unit - tile * splits;
      const TileCoord c = decode_tile<BM>(tile, N, BN_OUT, s_tile_start, s_off);
      const int buf = tc & 1;
      const uint32_t tph = (tc >> 1) & 1;
      const bool got = mbar_wait(smem_u32(&tfull_bar[buf]), tph, p.timeout_ns, &s_abort);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(buf * C::UMMA_N);
      const bool row_ok = r_local < c.rows;
      const int64_t row = static_cast<int64_t>(c.m0) + r_local;
#pragma unroll 1
      for (int cc = 0; cc < BN_OUT; cc += 16) {
        if (c.n0 + cc >= p.n_out) break;  // warp-uniform: ragged last n-tile
        float a[16], b[16];
        uint32_t v[16];
        tmem_ld_32x32b_x16(t_row + cc, v);
        if (EPI == EPI_SWIGLU) {
          uint32_t u[16];
          tmem_ld_32x32b_x16(t_row + BN_OUT + cc, u);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) b[i] = __uint_as_float(u[i]);
        } else {
          tmem_ld_wait();
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) a[i] = __uint_as_float(v[i]);
        if (!row_ok) continue;
        if (splits == 1) {
          store_final16<EPI>(p, row, c.n0 + cc, a, b);
        } else {  // this unit's partial tile
          float* dst = p.part + (static_cast<int64_t>(sp) * p.r_max + row) * p.part_ld + c.n0 + cc;
          store_f32x16(dst, a);
          if (EPI == EPI_SWIGLU) store_f32x16(dst + p.n_out, b);
        }
      }
      tc_fence_before_sync();
      mbar_arrive(smem_u32(&tempty_bar[buf]));  // TMEM buffer free for the next unit

      if (splits > 1) {
        // publish this partial; the unit that completes the tile adds all partials in order
        __threadfence();
        if (!__all_sync(0xffffffffu, epilogue_sync(smem_u32(&epi_bar), epi_phase, p.timeout_ns, &s_abort))) {
          ok = false;
          break;
        }
        if (threadIdx.x == 64) {
          const int prev = atomicAdd(p.tile_counters + tile, 1);
          const int last = prev == splits - 1;
          if (last) p.tile_counters[tile] = 0;  // every unit of the tile has arrived
          s_fixup = last;
        }
        if (!__all_sync(0xffffffffu, epilogue_sync(smem_u32(&epi_bar), epi_phase, p.timeout_ns, &s_abort))) {
          ok = false;
          break;
        }
        if (s_fixup) {
          // All 128 epilogue threads share the reduction: item i is (tile row i / G, float4
          // column group i % G), so neighbouring threads touch neighbouring columns.
          __threadfence();
          constexpr int G = BN_OUT / 4;
          const int cols = min(BN_OUT, p.n_out - c.n0);
          const int et = threadIdx.x - 64;  // 0..127
          for (int i = et; i < c.rows * G; i += kEpiThreads) {
            const int r = i / G, c4 = (i - r * G) * 4;
            if (c4 >= cols) continue;
            const int64_t orow = static_cast<int64_t>(c.m0) + r;
            const float* src = p.part + orow * p.part_ld + c.n0 + c4;
            const int64_t sstride = p.r_max * p.part_ld;
            float4 ga = make_float4(0.f, 0.f, 0.f, 0.f), ub = ga;
#pragma unroll 4
            for (int s2 = 0; s2 < splits; ++s2) {  // fixed order: deterministic sums
              const float4 v = __ldcg(reinterpret_cast<const float4*>(src + s2 * sstride));
              ga.x += v.x; ga.y += v.y; ga.z += v.z; ga.w += v.w;
              if (EPI == EPI_SWIGLU) {
                const float4 u = __ldcg(reinterpret_cast<const float4*>(src + s2 * sstride + p.n_out));
                ub.x += u.x; ub.y += u.y; ub.z += u.z; ub.w += u.w;
              }
            }
            store_final4<EPI>(p, orow, c.n0 + c4, ga, ub);
          }
        }
      }
    }
    if (!ok) {
      s_abort = 1;
      report_error(p.status, MOE_ERR_TIMEOUT);
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// bf16 tensor map with 128-byte swizzle; dims[0] is the contiguous (K) axis.
bool make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
              const uint64_t* strides_bytes, const uint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t gd[5];
  cuuint64_t gs[4];
  cuuint32_t bx[5];
  cuuint32_t es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) gs[i] = strides_bytes[i];
  }
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank),
                        const_cast<void*>(base), gd, gs, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int EPI, int BN_OUT, int BM>
cudaError_t launch_one(const CUtensorMap& ma, const CUtensorMap& mb, const GemmParams& gp,
                       int grid, cudaStream_t s) {
  using C = Cfg<EPI, BN_OUT, BM>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(grouped_gemm_kernel<EPI, BN_OUT, BM>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  });
  if (attr_err != cudaSuccess) return attr_err;
  return launch_pdl(grouped_gemm_kernel<EPI, BN_OUT, BM>, dim3(grid), dim3(kThreads), C::SMEM_BYTES, s,
                    ma, mb, gp);
}

int64_t tiles_upper_bound(int64_t r_max, int N, int n_tiles_n, int bm) {
  // sum_e ceil(m_e / bm) <= ceil(R / bm) + (experts with rows)
  const int64_t m_tiles_ub = (r_max + bm - 1) / bm + std::min<int64_t>(N, r_max);
  return m_tiles_ub * n_tiles_n;
}

int grid_for(int64_t r_max, int N, int n_tiles_n, int sm_count, int max_splits, int bm) {
  const int64_t units_ub = tiles_upper_bound(r_max, N, n_tiles_n, bm) * max_splits;
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(units_ub, sm_count)));
}

constexpr int64_t kSplitRowsMax = 256;                 // split-K only for decode-sized batches
constexpr size_t kPartBudget = size_t(64) << 20;       // bytes of partial tiles per GEMM
constexpr int kMaxSplits = 16;

int max_splits_for(int64_t r_max, int num_kb, int part_ld) {
  if (r_max > kSplitRowsMax) return 1;
  int ms = std::min(kMaxSplits, num_kb / 2);
  while (ms > 1 && static_cast<size_t>(ms) * r_max * part_ld * 4 > kPartBudget) --ms;
  return std::max(1, ms);
}

constexpr int kGuBnSwiglu = 128;  // output columns per tile of the gate/up GEMM (UMMA N = 256)
constexpr int kGuBnGelu = 256;
constexpr int kDnBn = 256;        // output columns per tile of the down GEMM

}  // namespace

FfnScratchPlan ffn_scratch_plan(int N, int d, int F, int act, int64_t r_max,
                                int64_t rows_per_expert) {
  FfnScratchPlan pl{1, 1, 0, 0, 128};
  if (r_max <= 0) return pl;
  pl.bm = rows_per_expert <= 64 ? 64 : 128;
  const bool swiglu = act == MOE_ACT_SWIGLU;
  const int bn1 = swiglu ? kGuBnSwiglu : kGuBnGelu;
  const int ld1 = swiglu ? 2 * F : F;
  pl.max_splits1 = max_splits_for(r_max, d / BK, ld1);
  pl.max_splits2 = max_splits_for(r_max, F / BK, d);
  size_t part = 0;
  int64_t tiles = 0;
  if (pl.max_splits1 > 1) {
    part = std::max(part, static_cast<size_t>(pl.max_splits1) * r_max * ld1 * 4);
    tiles = std::max(tiles, tiles_upper_bound(r_max, N, (F + bn1 - 1) / bn1, pl.bm));
  }
  if (pl.max_splits2 > 1) {
    part = std::max(part, static_cast<size_t>(pl.max_splits2) * r_max * d * 4);
    tiles = std::max(tiles, tiles_upper_bound(r_max, N, (d + kDnBn - 1) / kDnBn, pl.bm));
  }
  pl.part_bytes = part;
  pl.counter_bytes = static_cast<size_t>(tiles) * sizeof(int);
  return pl;
}

cudaError_t launch_grouped_ffn(const GroupedFfnArgs& a, cudaStream_t s) {
  if (a.r_max <= 0) return cudaSuccess;
  DeviceInfo di;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;

  const uint64_t d = static_cast<uint64_t>(a.d), F = static_cast<uint64_t>(a.F);
  const uint64_t N = static_cast<uint64_t>(a.N), R = static_cast<uint64_t>(a.r_max);
  const bool swiglu = a.act == MOE_ACT_SWIGLU;
  const int bn_gu = swiglu ? kGuBnSwiglu : kGuBnGelu;
  // weights are read once per m-tile; when every expert has at most one m-tile (decode-sized
  // batches) they are pure streams and should not displace the activations in L2
  const FfnScratchPlan plan =
      ffn_scratch_plan(a.N, a.d, a.F, a.act, a.r_max, a.rows_per_expert);
  const int bm = plan.bm;
  const int wpol = (a.rows_per_expert <= bm) ? 1 : 0;

  CUtensorMap mA1, mB1, mA2, mB2;
  {
    const uint64_t dims[2] = {d, R};
    const uint64_t str[1] = {d * 2};
    const uint32_t box[2] = {BK, static_cast<uint32_t>(bm)};
    if (!make_map(&mA1, a.x_perm, 2, dims, str, box)) return cudaErrorInvalidValue;
  }
  if (swiglu) {
    const uint64_t dims[4] = {d, F, 2, N};
    const uint64_t str[3] = {d * 2, F * d * 2, 2 * F * d * 2};
    const uint32_t box[4] = {BK, static_cast<uint32_t>(bn_gu), 1, 1};
    if (!make_map(&mB1, a.w_gate_up, 4, dims, str, box)) return cudaErrorInvalidValue;
  } else {
    const uint64_t dims[3] = {d, F, N};
    const uint64_t str[2] = {d * 2, F * d * 2};
    const uint32_t box[3] = {BK, static_cast<uint32_t>(bn_gu), 1};
    if (!make_map(&mB1, a.w_gate_up, 3, dims, str, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {F, R};
    const uint64_t str[1] = {F * 2};
    const uint32_t box[2] = {BK, static_cast<uint32_t>(bm)};
    if (!make_map(&mA2, a.h, 2, dims, str, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[3] = {F, d, N};
    const uint64_t str[2] = {F * 2, d * F * 2};
    const uint32_t box[3] = {BK, static_cast<uint32_t>(kDnBn), 1};
    if (!make_map(&mB2, a.w_down, 3, dims, str, box)) return cudaErrorInvalidValue;
  }

  GemmParams g1{};
  g1.expert_offset = a.expert_offset;
  g1.out = a.h;
  g1.ld_out = a.F;
  g1.r_max = a.r_max;
  g1.n_experts = a.N;
  g1.n_out = a.F;
  g1.n_tiles_n = (a.F + bn_gu - 1) / bn_gu;
  g1.num_kb = a.d / BK;
  g1.status = a.status;
  g1.timeout_ns = a.timeout_ns;
  g1.weight_policy = wpol;
  const bool can_split = a.part != nullptr && a.tile_counters != nullptr;
  g1.max_splits = can_split ? plan.max_splits1 : 1;
  g1.part = a.part;
  g1.part_ld = swiglu ? 2 * a.F : a.F;
  g1.tile_counters = a.tile_counters;
  const int grid1 = grid_for(a.r_max, a.N, g1.n_tiles_n, di.sm_count, g1.max_splits, bm);
  if (bm == 64)
    err = swiglu ? launch_one<EPI_SWIGLU, kGuBnSwiglu, 64>(mA1, mB1, g1, grid1, s)
                 : launch_one<EPI_GELU, kGuBnGelu, 64>(mA1, mB1, g1, grid1, s);
  else
    err = swiglu ? launch_one<EPI_SWIGLU, kGuBnSwiglu, 128>(mA1, mB1, g1, grid1, s)
                 : launch_one<EPI_GELU, kGuBnGelu, 128>(mA1, mB1, g1, grid1, s);
  if (err != cudaSuccess) return err;

  GemmParams g2 = g1;
  g2.out = a.y_perm;
  g2.ld_out = a.d;
  g2.n_out = a.d;
  g2.n_tiles_n = (a.d + kDnBn - 1) / kDnBn;
  g2.num_kb = a.F / BK;
  g2.max_splits = can_split ? plan.max_splits2 : 1;
  g2.part_ld = a.d;
  const int grid2 = grid_for(a.r_max, a.N, g2.n_tiles_n, di.sm_count, g2.max_splits, bm);
  return bm == 64 ? launch_one<EPI_STORE_F32, kDnBn, 64>(mA2, mB2, g2, grid2, s)
                  : launch_one<EPI_STORE_F32, kDnBn, 128>(mA2, mB2, g2, grid2, s);
}

}  // namespace moe
