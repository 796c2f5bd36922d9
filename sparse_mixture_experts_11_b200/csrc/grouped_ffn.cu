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

constexpr int BM = 128;       // rows per tile (UMMA M)
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
};

constexpr int pow2_at_least(int v) {
  int p = 32;
  while (p < v) p <<= 1;
  return p;
}

template <int EPI, int BN_OUT>
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

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + __expf(-g)); }
__device__ __forceinline__ float gelu_f(float z) {
  return 0.5f * z * (1.0f + erff(z * 0.7071067811865476f));
}

template <int EPI, int BN_OUT>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB, const GemmParams p) {
  using C = Cfg<EPI, BN_OUT>;
  extern __shared__ __align__(1024) uint8_t dyn_smem[];
  __shared__ __align__(8) uint64_t full_bar[C::STAGES];
  __shared__ __align__(8) uint64_t empty_bar[C::STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t done_bar;
  __shared__ uint32_t s_tmem_base;
  __shared__ volatile int s_abort;
  __shared__ int s_tile_start[257];
  __shared__ int s_off[257];

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
    s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    __syncwarp();
    tmem_alloc(smem_u32(&s_tmem_base), C::TMEM_COLS);
    tmem_relinquish();
  }
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
    if (lane == 31) s_tile_start[N] = incl;
    if (bad) report_error(p.status, MOE_ERR_BOUNDS);  // such an expert gets no tiles
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();

  const uint32_t tmem_base = s_tmem_base;
  const int total_tiles = s_tile_start[N];

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      const uint64_t pol_a = make_policy(2);
      const uint64_t pol_b = make_policy(p.weight_policy);
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
        const TileCoord c = decode_tile(tile, N, BN_OUT, s_tile_start, s_off);
        for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
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
        mbar_wait(smem_u32(&full_bar[i % C::STAGES]), (i / C::STAGES) & 1, p.timeout_ns, nullptr);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, C::UMMA_N);
      int it = 0, tc = 0;
      bool ok = true;
      bool issued = false;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x, ++tc) {
        const int buf = tc & 1;
        const uint32_t tph = (tc >> 1) & 1;
        if (!mbar_wait(smem_u32(&tempty_bar[buf]), tph ^ 1u, p.timeout_ns, &s_abort)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * C::UMMA_N);
        for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
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
                       idesc, (kb | kk) != 0 ? 1u : 0u);
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
          mbar_wait(smem_u32(&done_bar), 0, p.timeout_ns, nullptr);
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue (warps 2..5)
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const int r_local = q * 32 + lane;
    int tc = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++tc) {
      const TileCoord c = decode_tile(tile, N, BN_OUT, s_tile_start, s_off);
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
        if (EPI == EPI_STORE_F32) {
          uint32_t v[16];
          tmem_ld_32x32b_x16(t_row + cc, v);
          tmem_ld_wait();
          if (row_ok) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + row * p.ld_out + c.n0 + cc);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                   __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
          }
        } else {
          uint32_t g[16];
          uint32_t packed[8];
          tmem_ld_32x32b_x16(t_row + cc, g);
          if (EPI == EPI_SWIGLU) {
            uint32_t u[16];
            tmem_ld_32x32b_x16(t_row + BN_OUT + cc, u);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float h0 = silu_f(__uint_as_float(g[2 * i])) * __uint_as_float(u[2 * i]);
              const float h1 = silu_f(__uint_as_float(g[2 * i + 1])) * __uint_as_float(u[2 * i + 1]);
              packed[i] = pack_bf16x2(h0, h1);
            }
          } else {
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 8; ++i)
              packed[i] = pack_bf16x2(gelu_f(__uint_as_float(g[2 * i])), gelu_f(__uint_as_float(g[2 * i + 1])));
          }
          if (row_ok) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + row * p.ld_out + c.n0 + cc);
            dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
            dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
          }
        }
      }
      tc_fence_before_sync();
      mbar_arrive(smem_u32(&tempty_bar[buf]));
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

template <int EPI, int BN_OUT>
cudaError_t launch_one(const CUtensorMap& ma, const CUtensorMap& mb, const GemmParams& gp,
                       int grid, cudaStream_t s) {
  using C = Cfg<EPI, BN_OUT>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(grouped_gemm_kernel<EPI, BN_OUT>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  });
  if (attr_err != cudaSuccess) return attr_err;
  grouped_gemm_kernel<EPI, BN_OUT><<<grid, kThreads, C::SMEM_BYTES, s>>>(ma, mb, gp);
  return cudaGetLastError();
}

int grid_for(int64_t r_max, int N, int n_tiles_n, int sm_count) {
  const int64_t m_tiles_ub = (r_max + BM - 1) / BM + std::min<int64_t>(N, r_max);
  const int64_t tiles_ub = m_tiles_ub * n_tiles_n;
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(tiles_ub, sm_count)));
}

constexpr int kGuBnSwiglu = 128;  // output columns per tile of the gate/up GEMM (UMMA N = 256)
constexpr int kGuBnGelu = 256;
constexpr int kDnBn = 256;        // output columns per tile of the down GEMM

}  // namespace

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
  const int wpol = (a.r_max <= BM) ? 1 : 0;

  CUtensorMap mA1, mB1, mA2, mB2;
  {
    const uint64_t dims[2] = {d, R};
    const uint64_t str[1] = {d * 2};
    const uint32_t box[2] = {BK, BM};
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
    const uint32_t box[2] = {BK, BM};
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
  const int grid1 = grid_for(a.r_max, a.N, g1.n_tiles_n, di.sm_count);
  err = swiglu ? launch_one<EPI_SWIGLU, kGuBnSwiglu>(mA1, mB1, g1, grid1, s)
               : launch_one<EPI_GELU, kGuBnGelu>(mA1, mB1, g1, grid1, s);
  if (err != cudaSuccess) return err;

  GemmParams g2 = g1;
  g2.out = a.y_perm;
  g2.ld_out = a.d;
  g2.n_out = a.d;
  g2.n_tiles_n = (a.d + kDnBn - 1) / kDnBn;
  g2.num_kb = a.F / BK;
  const int grid2 = grid_for(a.r_max, a.N, g2.n_tiles_n, di.sm_count);
  return launch_one<EPI_STORE_F32, kDnBn>(mA2, mB2, g2, grid2, s);
}

}  // namespace moe
