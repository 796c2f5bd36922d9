// Expert FFN of decode-sized batches on 5th-generation tensor cores (tcgen05, sm_100a), with
// every SM streaming weights until none are left.
//
// Page «Что такое Mixture of Experts (MoE) в трансформерах» (aglamov.biz): «Бэкенд для
// экспертов» (tokens grouped by expert, one grouped GEMM) and «Динамическая загрузка весов с
// WeightConverter» (packed gate_up_proj [N, 2F, d], gate rows first, and down_proj [N, d, F]).
// Page «Sparse Mixture-of-Experts», «Роутер и top-k gating»: the layer's output is the residual
// plus the kept experts' outputs weighted by the renormalised router probabilities.
//
// With at most 8 tokens an expert holds at most 8 rows, so the layer is a stream of the active
// experts' weights with little arithmetic per byte, and an SM streams only its share of HBM
// (and SMs stream at rates that differ by half or more): the weights must go to whichever SM
// is free. The work is two GEMMs of tiles of 256 weight rows, each cut into k blocks of 64
// (units of 32 KB of weights):
//   phase A (gate/up): tile (expert, j) = the 128 gate and 128 up rows of d_ff columns
//     [128j, 128j+128), K = d; it yields h[:, 128j:128j+128] = silu(x W_g^T) * (x W_u^T),
//     rounded once to bf16 (as the grouped FFN rounds h);
//   phase B (down): tile (expert, m) = rows [256m, 256m+256) of W_d, K = F; it yields those 256
//     columns of y.
// Rows past d_ff or d read as zero and their outputs are not stored. A tile's units are cut
// into a fixed number of chunks (from the shape, a few hundred KB each). CTAs take chunks from
// a global counter, all of phase A (by column block j, then expert) before any of phase B (by
// chunk of F, then expert and row block), so an SM that streams faster takes more. Each chunk's
// fp32 partial of the 8 x 256 accumulator goes to global memory; the CTA that finishes a tile's
// last chunk adds the tile's partials in chunk order, so the result does not depend on which
// CTA took which chunk, nor on timing.
//
// Phase B needs h: the CTA that finishes a phase-A tile stores its h columns and raises the
// tile's flag; a phase-B unit's 8 x 64 tile of h is copied into its stage after that flag (its
// weights do not depend on h and stream regardless). In moe_forward the CTA that finishes the
// last of an output block's tiles (one per active expert) also combines that block:
// out[t] = residual[t] + sum over kept choices j, in order, of w_j y[row(t, j)] in fp32, rounded
// once (moe_unpermute_combine's arithmetic); a token with no kept pair passes the residual's
// bits through.
//
// Both GEMMs put the weights in the N operand (N = 256 rows x 64 k per unit) and the token
// rows in M = 64 (the gate/up GEMM: the expert's rows of x_perm in moe_grouped_ffn, or in
// moe_forward the batch's tokens x[0..8), as every token fits; the down GEMM: the expert's rows
// of h). Only 8 of the 64 rows are live: a stage holds their 1 KB and then the 32 KB of
// weights, and the A operand's other 56 rows read the start of the weights, which only fills
// accumulator rows that are never read. UMMA M=64, N=256, K=16; accumulator row r is TMEM lane
// r (r < 16), so one warp reads every live row.
//
// Kernel structure (one CTA per SM, 256 threads):
//   warp 0     takes chunks and is the TMA producer through a ring of 33 KB stages (128B
//              swizzle): the weights, and in phase A the token tile;
//   warp 1     allocates TMEM and issues the MMAs from one thread (two 256-column accumulators);
//   warp 2     copies each phase-B unit's tile of h into its stage (cp.async), after its flag;
//   warps 4-7  epilogue: warp 4 stores each chunk's partial; the CTA that completes a tile adds
//              its partials (all 128 threads) and stores h or y's rows, and, last for an output
//              block, combines it.
//
// In moe_forward the same launch first routes the batch: the first ceil(d/128) CTAs store the
// decode router's partial dot products (dr::decode_route_partials, as moe_route), and then
// every CTA adds them up and takes top-k and the capacity slots in its own shared memory
// (dr::decode_route_finish), so the routing is identical to moe_route's and no second pass
// through global memory stands before the weights start streaming.
//
// Every wait is bounded. A CTA that gives up records MOE_ERR_TIMEOUT, stops issuing work and
// waits (bounded) for its own copies and MMAs. The last CTA to leave puts the counters and flags
// back to zero, for the next call.
#include <string.h>

#include <type_traits>

#include "common.cuh"
#include "decode_route.cuh"
#include "launch.h"
#include "tma_host.h"

namespace moe {
namespace {

constexpr int kDfThreads = 256;
constexpr int kDfM = 64;                  // UMMA M: token rows (kDfMaxRows live)
constexpr int kDfN = 256;                 // UMMA N: weight rows
constexpr int kDfBK = 64;                 // k per unit
constexpr int kDfTok = 8 * 128;           // 1 KB: the 8 live token rows x 64 k, bf16
constexpr int kDfW = kDfN * kDfBK * 2;    // 32 KB: 256 weight rows x 64 k
constexpr int kDfStage = kDfTok + kDfW;   // 33 KB (a multiple of 1024: stages stay swizzle-aligned)
constexpr int kDfStages = 6;
constexpr int kDfTmemCols = 2 * kDfN;     // two accumulators
constexpr int kDfGU = 128;                // d_ff columns per phase-A tile
constexpr int kDfDB = 256;                // d rows per phase-B tile
constexpr int kDfMaxRows = kDecodeFfnMaxRows;  // rows per expert, and tokens, at most
constexpr int kDfMaxActive = 64;          // experts with rows at most (T * k <= 64)
constexpr int kDfChunkRing = 16;          // chunks taken by the producer, not yet retired
constexpr int kDfRedQ = 16;               // completed tiles waiting for the reducers
constexpr int kDfAcc = kDfMaxRows * kDfN * 4;  // 8 KB: an owned tile's live rows, fp32
constexpr int kDfSmem = kDfStages * kDfStage + kDfAcc + 1024;
static_assert(kDfStage % 1024 == 0, "stage alignment");
static_assert(kDfM * 128 <= kDfStage, "the A operand's rows stay inside the stage");
static_assert(kDecodeFfnMaxT <= kDfMaxRows && kDfMaxRows == 8, "rows per expert");
static_assert(kDfGU == kDecodeFfnSlice, "gate/up tile width");

constexpr unsigned kFullMask = 0xffffffffu;

struct DfParams {
  const int32_t* expert_offset;  // moe_grouped_ffn: the sort's offsets (moe_forward: routed here)
  uint16_t* h;
  float* y;
  float* part;     // [chunks][8][256] fp32 partial of each chunk
  int* hflag;      // [s_max] h of the phase-A tile stored (1)
  int* tcnt;       // [s_max + b_max] chunks finished, per phase-A tile, then per phase-B tile
  int* mdone;      // [ceil(d/256)] phase-B tiles of the output block finished
  int* sync;       // [1] departures, [2] the chunk counter; zero between calls
  const int32_t* row_of_pair;  // combine without routing in the launch
  const float* topk_w;
  const uint16_t* residual;
  void* out;  // null: no combine
  int out_f32;
  int T, k, N, d, F;
  int64_t r_max;
  int s_max;       // phase-A tiles at most (the counters' and flags' size)
  int nca, ncb;    // chunks per phase-A tile and per phase-B tile
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

// 16-byte copy global -> shared through L2 (src_bytes 0: zero-fill, nothing read).
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Bounded wait until the shared counter *c exceeds i; false on timeout or abort.
__device__ __forceinline__ bool wait_smem_above(const volatile int* c, int i, uint64_t timeout_ns,
                                                const volatile int* abort) {
  if (*c > i) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (*c > i) return true;
    if (*abort != 0) return false;
    if (globaltimer_ns() - t0 > timeout_ns) return false;
    __nanosleep(20);
  }
}

// Bounded wait until the shared flag *f is set; false on timeout.
__device__ __forceinline__ bool wait_smem_set(const volatile int* f, uint64_t timeout_ns) {
  if (*f != 0) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (*f != 0) return true;
    if (globaltimer_ns() - t0 > timeout_ns) return false;
    __nanosleep(20);
  }
}

// The chunk grid: NA phase-A chunks (by column block j, then expert a, then chunk c of the
// tile's d/64 units), then the phase-B chunks (by chunk c of the tile's F/64 units, then expert
// a, then row block m).
struct DfGeo {
  int nact, Ft, KB, FB, DB, nca, ncb;
  int NA, NC;
};
struct DfChunk {
  int phase;   // 0: gate/up, 1: down
  int a, jm;   // active expert, column block j (phase A) or row block m (phase B)
  int c;       // chunk of the tile
  int u0, u1;  // its units: k blocks of d (phase A) or of F (phase B)
  int tile;    // counter index: a * Ft + j, or nact * Ft + a * DB + m
};
__device__ __forceinline__ DfChunk df_chunk(const DfGeo& g, int id) {
  DfChunk ch;
  if (id < g.NA) {
    ch.phase = 0;
    const int per = g.nact * g.nca;
    ch.jm = id / per;
    const int r = id - ch.jm * per;
    ch.a = r / g.nca;
    ch.c = r - ch.a * g.nca;
    ch.u0 = ch.c * g.KB / g.nca;
    ch.u1 = (ch.c + 1) * g.KB / g.nca;
    ch.tile = ch.a * g.Ft + ch.jm;
  } else {
    ch.phase = 1;
    const int q = id - g.NA, per = g.nact * g.DB;
    ch.c = q / per;
    const int r = q - ch.c * per;
    ch.a = r / g.DB;
    ch.jm = r - ch.a * g.DB;
    ch.u0 = ch.c * g.FB / g.ncb;
    ch.u1 = (ch.c + 1) * g.FB / g.ncb;
    ch.tile = g.nact * g.Ft + ch.a * g.DB + ch.jm;
  }
  return ch;
}
// id of chunk c of the tile of `ch`
__device__ __forceinline__ int df_chunk_id(const DfGeo& g, const DfChunk& ch, int c) {
  if (ch.phase == 0) return (ch.jm * g.nact + ch.a) * g.nca + c;
  return g.NA + (c * g.nact + ch.a) * g.DB + ch.jm;
}

// The next chunk this CTA's producer has taken (chunk number seq of the CTA): its id, -1 when
// there are no more, -2 on timeout or abort.
__device__ __forceinline__ int df_wait_chunk(int seq, const volatile int* nch, const volatile int* end,
                                             const volatile int* ring, uint64_t timeout_ns,
                                             const volatile int* abort) {
  uint64_t t0 = 0;
  for (int n = 0;; ++n) {
    if (*nch > seq) {
      __threadfence_block();
      return ring[seq % kDfChunkRing];
    }
    if (*end != 0) {
      __threadfence_block();
      if (*nch > seq) return ring[seq % kDfChunkRing];
      return -1;
    }
    if (*abort != 0) return -2;
    if (n == 0) t0 = globaltimer_ns();
    else if (globaltimer_ns() - t0 > timeout_ns) return -2;
    __nanosleep(20);
  }
}

__device__ __forceinline__ void store_f32x16(float* dst, const float* v) {
  float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) d4[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}

template <bool ROUTE, int EPT>
__global__ void __launch_bounds__(kDfThreads, 1)
    decode_ffn_kernel(const __grid_constant__ CUtensorMap tmGU, const __grid_constant__ CUtensorMap tmX,
                      const __grid_constant__ CUtensorMap tmWD, const DfParams p) {
  extern __shared__ __align__(1024) uint8_t dyn_smem[];
  __shared__ __align__(8) uint64_t full_bar[kDfStages];
  __shared__ __align__(8) uint64_t empty_bar[kDfStages];
  __shared__ __align__(8) uint64_t tfull[2], tempty[2];
  __shared__ __align__(8) uint64_t red_bar, done_bar;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  __shared__ volatile int s_hdone;    // phase-B units whose tile of h the loader has delivered
  __shared__ volatile int s_hfinal;   // the loader has stopped
  __shared__ volatile int s_armed;    // units whose stage the producer has found free
  __shared__ volatile int s_nchunks;  // chunks the producer has taken
  __shared__ volatile int s_end;      // the producer takes no more chunks
  __shared__ volatile int s_chunk[kDfChunkRing];
  __shared__ volatile int s_redq[kDfRedQ];  // completed tiles (their last chunk), for the reducers
  __shared__ volatile int s_redq_n;          // entries pushed
  __shared__ volatile int s_redq_done;       // entries retired
  __shared__ volatile int s_redq_end;        // no more entries
  __shared__ int s_comb;
  __shared__ int s_lastcta;
  __shared__ int s_ok;
  __shared__ int s_nact;
  __shared__ int s_off[257];
  __shared__ int s_act[kDfMaxActive];
  __shared__ short s_colrow[kDfMaxActive][kDfMaxRows];  // output row of each token column, -1 if none
  __shared__ typename std::conditional<ROUTE, dr::DecodeRouteSmem<kDfMaxRows, EPT>, int>::type s_route;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t ring = (smem_u32(dyn_smem) + 1023u) & ~1023u;
  float* s_acc = reinterpret_cast<float*>(dyn_smem + (ring - smem_u32(dyn_smem)) + kDfStages * kDfStage);
  const int G = static_cast<int>(gridDim.x);
  const int b = static_cast<int>(blockIdx.x);

  if (tid == 0) {
    prefetch_tensormap(&tmGU);
    prefetch_tensormap(&tmX);
    prefetch_tensormap(&tmWD);
    for (int s = 0; s < kDfStages; ++s) {
      // two arrivals: the producer's (with the copies' bytes) and the token tile's: the
      // producer again for phase A (its copy), the h loader for phase B
      mbar_init(smem_u32(&full_bar[s]), 2);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&tfull[i]), 1);
      mbar_init(smem_u32(&tempty[i]), 32);
    }
    mbar_init(smem_u32(&red_bar), 96);
    mbar_init(smem_u32(&done_bar), 1);
    s_abort = 0;
    s_hdone = 0;
    s_hfinal = 0;
    s_armed = 0;
    s_nchunks = 0;
    s_end = 0;
    s_redq_n = 0;
    s_redq_done = 0;
    s_redq_end = 0;
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

  // ---------------------------------------------------------------- routing / the tile lists
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
  for (int i = tid; i < kDfMaxActive * kDfMaxRows; i += kDfThreads) (&s_colrow[0][0])[i] = -1;
  __syncthreads();
  // output row of each token column of each active expert (the gate/up GEMM's rows)
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
    for (int i = tid; i < s_nact * kDfMaxRows; i += kDfThreads) {
      const int a = i / kDfMaxRows, c = i - a * kDfMaxRows;
      const int e = s_act[a];
      if (c < s_off[e + 1] - s_off[e]) s_colrow[a][c] = static_cast<short>(s_off[e] + c);
    }
  }
  __syncthreads();
  const int nact = s_nact;
  DfGeo g;
  g.nact = nact;
  g.Ft = (p.F + kDfGU - 1) / kDfGU;   // phase-A tiles per expert
  g.KB = p.d / kDfBK;                 // phase-A units per tile
  g.FB = p.F / kDfBK;                 // phase-B units per tile
  g.DB = (p.d + kDfDB - 1) / kDfDB;   // phase-B tiles per expert (output blocks)
  g.nca = p.nca;
  g.ncb = p.ncb;
  g.NA = nact * g.Ft * g.nca;
  g.NC = g.NA + nact * g.DB * g.ncb;
  const bool run = s_abort == 0 && nact * g.Ft <= p.s_max;
  if (nact * g.Ft > p.s_max && tid == 0) report_error(p.status, MOE_ERR_BOUNDS);
  const bool combine = p.out != nullptr;

  if (warp == 0 && run) {
    // ---------------------------------------------------------- chunks and the TMA producer
    if (lane == 0) {
      const uint64_t pol_w = l2_policy_evict_first();  // weights: read once, streamed
      const uint64_t pol_x = l2_policy_evict_last();   // token rows: read by many CTAs
      int it = 0, seq = 0, nA = 0;
      bool ok = true;
      int next = atomicAdd(p.sync + 2, 1);
      for (;;) {
        const int cur = next;
        if (cur >= g.NC) break;
        next = atomicAdd(p.sync + 2, 1);  // taken now, its latency hidden behind this chunk
        const DfChunk ch = df_chunk(g, cur);
        const int e = s_act[ch.a];
        s_chunk[seq % kDfChunkRing] = cur;
        __threadfence_block();
        s_nchunks = seq + 1;
        for (int u = ch.u0; u < ch.u1; ++u, ++it) {
          const int s = it % kDfStages;
          if (!mbar_wait(smem_u32(&empty_bar[s]), ((it / kDfStages) & 1) ^ 1u, p.timeout_ns, &s_abort)) {
            ok = false;
            break;
          }
          s_armed = it + 1;
          const uint32_t st = ring + s * kDfStage, fb = smem_u32(&full_bar[s]);
          if (ch.phase == 0) {
            mbar_arrive_expect_tx(fb, kDfStage);
            tma_load_4d(st + kDfTok, &tmGU, fb, u * kDfBK, ch.jm * kDfGU, 0, e, pol_w);           // gate rows
            tma_load_4d(st + kDfTok + kDfW / 2, &tmGU, fb, u * kDfBK, ch.jm * kDfGU, 1, e, pol_w);  // up rows
            tma_load_2d(st, &tmX, fb, u * kDfBK, ROUTE ? 0 : s_off[e], pol_x);                     // token rows
            mbar_arrive(fb);  // the token tile's arrival (the loader's, in phase B)
          } else {
            mbar_arrive_expect_tx(fb, kDfW);
            tma_load_3d(st + kDfTok, &tmWD, fb, u * kDfBK, ch.jm * kDfDB, e, pol_w);  // W_d rows
          }
        }
        if (ch.phase == 0) nA = it;
        ++seq;
        if (!ok) break;
      }
      __threadfence_block();
      s_end = 1;
      if (!ok) {
        s_abort = 1;
        report_error(p.status, MOE_ERR_TIMEOUT);
      }
      // this thread's copies still in flight land before the CTA moves on (bounded). A phase-B
      // stage whose tile of h the loader gave up on gets the loader's arrival from here.
      if (it > nA) {
        wait_smem_set(&s_hfinal, kDrainTimeoutNs);
        __threadfence_block();
        const int hd = s_hdone;
        for (int q = max(nA + hd, it - kDfStages); q < it; ++q) mbar_arrive(smem_u32(&full_bar[q % kDfStages]));
      }
      for (int q = max(0, it - kDfStages); q < it; ++q)
        mbar_wait(smem_u32(&full_bar[q % kDfStages]), (q / kDfStages) & 1, kDrainTimeoutNs, nullptr);
    }
  } else if (warp == 1 && run) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kDfM, kDfN);
      int it = 0, tc = 0;
      bool ok = true, issued = false;
      for (int seq = 0; ok; ++seq, ++tc) {
        const int cur = df_wait_chunk(seq, &s_nchunks, &s_end, s_chunk, p.timeout_ns, &s_abort);
        if (cur < 0) {
          ok = cur == -1;
          break;
        }
        const DfChunk ch = df_chunk(g, cur);
        const int buf = tc & 1;
        if (!mbar_wait(smem_u32(&tempty[buf]), ((tc >> 1) & 1) ^ 1u, p.timeout_ns, &s_abort)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t acc = tmem + static_cast<uint32_t>(buf * kDfN);
        for (int u = ch.u0; u < ch.u1; ++u, ++it) {
          const int s = it % kDfStages;
          if (!mbar_wait(smem_u32(&full_bar[s]), (it / kDfStages) & 1, p.timeout_ns, &s_abort)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a0 = ring + s * kDfStage, b0 = a0 + kDfTok;
#pragma unroll
          for (int kk = 0; kk < kDfBK / 16; ++kk)
            tc_mma_f16(acc, smem_desc_k_sw128(a0 + kk * 32), smem_desc_k_sw128(b0 + kk * 32), idesc,
                       (u != ch.u0 || kk != 0) ? 1u : 0u);
          issued = true;
          tc_commit(smem_u32(&empty_bar[s]));
        }
        if (!ok) break;
        tc_commit(smem_u32(&tfull[buf]));
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
  } else if (warp == 2 && run) {
    // ---------------------------------------------------------- tiles of h for phase B
    // Once its phase-A tile's flag is up, a phase-B unit's 8 rows x 64 columns of h go into its
    // stage's token slot by cp.async (lane l: row l / 4, 16-byte chunks 2 (l & 3) and +1, at
    // chunk XOR row: the 128B-swizzled K-major layout; rows past the expert's count are zero).
    // Up to four units are in flight; each lane fences its own completed copies for the tensor
    // core before the stage's arrival. A unit's slot is written only after the producer has
    // armed the unit's stage, so the loader is never more than one phase of a barrier ahead.
    // A CTA's phase-B units follow all of its phase-A units.
    const int r = lane >> 2, c0 = (lane & 3) * 2;
    int it = 0, nA = -1, ib = 0, ic = 0;  // unit index, phase-A units, B units issued, delivered
    int last = -1;
    bool ok = true;
    for (int seq = 0; ok; ++seq) {
      int cur = 0;
      if (lane == 0) cur = df_wait_chunk(seq, &s_nchunks, &s_end, s_chunk, p.timeout_ns, &s_abort);
      cur = __shfl_sync(kFullMask, cur, 0);
      if (cur < 0) {
        ok = cur == -1;
        break;
      }
      const DfChunk ch = df_chunk(g, cur);
      if (ch.phase == 0) {
        it += ch.u1 - ch.u0;
        continue;
      }
      if (nA < 0) nA = it;
      const int e = s_act[ch.a];
      const int row0 = s_off[e], cnt = s_off[e + 1] - s_off[e];
      for (int fb = ch.u0; fb < ch.u1; ++fb, ++it) {
        const int need = ch.a * g.Ft + fb / (kDfGU / kDfBK);
        if (need != last) {
          bool ready = lane == 0 && ld_acquire_gpu(p.hflag + need) == 1;
          ready = __shfl_sync(kFullMask, ready, 0);
          if (!ready) {
            // deliver what is in flight before blocking on the flag
            cp_async_wait<0>();
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              for (int q = ic; q < ib; ++q) mbar_arrive(smem_u32(&full_bar[(nA + q) % kDfStages]));
              s_hdone = ib;
            }
            ic = ib;
            if (lane == 0) ready = wait_flag(p.hflag + need, 1, p.timeout_ns, &s_abort);
            ready = __shfl_sync(kFullMask, ready, 0);
            if (!ready) {
              ok = false;
              break;
            }
          }
          last = need;
        }
        const int s = it % kDfStages;
        bool got = lane == 0 && wait_smem_above(&s_armed, it, p.timeout_ns, &s_abort) &&
                   mbar_wait(smem_u32(&empty_bar[s]), ((it / kDfStages) & 1) ^ 1u, p.timeout_ns, &s_abort);
        got = __shfl_sync(kFullMask, got, 0);
        if (!got) {
          ok = false;
          break;
        }
        const uint32_t dst = ring + s * kDfStage + r * 128;
        const uint16_t* src = p.h + static_cast<int64_t>(row0 + (r < cnt ? r : 0)) * p.F + fb * kDfBK;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int c = c0 + q;
          cp_async_16(dst + ((c ^ r) << 4), src + c * 8, r < cnt ? 16u : 0u);
        }
        cp_async_commit();
        ++ib;
        if (ib - ic > 3) {
          cp_async_wait<3>();
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(smem_u32(&full_bar[(nA + ic) % kDfStages]));
            s_hdone = ic + 1;
          }
          ++ic;
        }
      }
    }
    cp_async_wait<0>();
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      for (int q = ic; q < ib; ++q) mbar_arrive(smem_u32(&full_bar[(nA + q) % kDfStages]));
      s_hdone = ib;
      if (!ok) {
        s_abort = 1;
        report_error(p.status, MOE_ERR_TIMEOUT);
      }
      __threadfence_block();
      s_hfinal = 1;
    }
  } else if (warp == 4 && run) {
    // ---------------------------------------------------------- accumulator drain (warp 4)
    // Each chunk's partial (rows 0-7 are TMEM lanes 0-7 of this warp's quadrant) goes to global
    // memory and is counted on its tile; a chunk that completes its tile goes to the reducers.
    bool ok = true;
    int nq = 0;
    for (int seq = 0, tc = 0; ok; ++seq, ++tc) {
      int cur = 0;
      if (lane == 0) cur = df_wait_chunk(seq, &s_nchunks, &s_end, s_chunk, p.timeout_ns, &s_abort);
      cur = __shfl_sync(kFullMask, cur, 0);
      if (cur < 0) {
        ok = cur == -1;
        break;
      }
      const DfChunk ch = df_chunk(g, cur);
      const int buf = tc & 1;
      if (!__all_sync(kFullMask, mbar_wait(smem_u32(&tfull[buf]), (tc >> 1) & 1, p.timeout_ns, &s_abort))) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const uint32_t t0 = tmem + static_cast<uint32_t>(buf * kDfN);
      float* dst = p.part + (static_cast<int64_t>(cur) * kDfMaxRows + lane) * kDfN;
#pragma unroll 1
      for (int c = 0; c < kDfN; c += 64) {
        uint32_t u[4][16];
#pragma unroll
        for (int q = 0; q < 4; ++q) tmem_ld_32x32b_x16(t0 + c + q * 16, u[q]);
        tmem_ld_wait();
        if (lane < kDfMaxRows) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float v[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(u[q][i]);
            store_f32x16(dst + c + q * 16, v);
          }
        }
      }
      tc_fence_before_sync();
      mbar_arrive(smem_u32(&tempty[buf]));  // the accumulator is free for the MMA
      __threadfence();
      __syncwarp();
      if (lane == 0) {
        const int n = ch.phase == 0 ? g.nca : g.ncb;
        const int prev = atomicAdd(p.tcnt + ch.tile, 1);
        if (prev == n - 1) {
          __threadfence();
          // the queue holds every chunk this CTA drains, so it cannot overflow: a tile completes
          // once, and the reducers retire entries in order
          if (!wait_smem_above(&s_redq_done, nq - (kDfRedQ - 1), p.timeout_ns, &s_abort)) ok = false;
          s_redq[nq % kDfRedQ] = cur;
          __threadfence_block();
          s_redq_n = ++nq;
        }
      }
      ok = __shfl_sync(kFullMask, ok, 0);
    }
    if (lane == 0) {
      __threadfence_block();
      s_redq_end = 1;
      if (!ok) {
        s_abort = 1;
        report_error(p.status, MOE_ERR_TIMEOUT);
      }
    }
  } else if (warp >= 5 && run) {
    // ---------------------------------------------------------- reducers (warps 5-7)
    // A completed tile: its partials added in chunk order (segment q of the 8 x 256 sums: row
    // q / 16, columns (q mod 16) * 16 .. + 16; the loads of four chunks in flight at once), then
    // h or y's rows, and, last of an output block, the combine.
    const int rt = tid - 160;  // 0..95
    uint32_t red_phase = 0;
    bool ok = true;
    for (int ridx = 0; ok; ++ridx) {
      int cur = -1;
      {
        uint64_t t0 = 0;
        for (int n = 0;; ++n) {
          if (s_redq_n > ridx) {
            __threadfence_block();
            cur = s_redq[ridx % kDfRedQ];
            break;
          }
          if (s_redq_end != 0) {
            __threadfence_block();
            if (s_redq_n > ridx) {
              cur = s_redq[ridx % kDfRedQ];
            }
            break;
          }
          if (s_abort != 0) {
            ok = false;
            break;
          }
          if (n == 0) t0 = globaltimer_ns();
          else if (globaltimer_ns() - t0 > p.timeout_ns) {
            ok = false;
            break;
          }
          __nanosleep(32);
        }
      }
      if (!ok || cur < 0) break;
      const DfChunk ch = df_chunk(g, cur);
      const int n = ch.phase == 0 ? g.nca : g.ncb;
      for (int q = rt; q < kDfMaxRows * (kDfN / 16); q += 96) {
        const int er = q >> 4, ec = (q & 15) * 16;
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = 0.f;
        for (int c = 0; c < n; c += 4) {
          float4 w4[4][4];
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            if (c + w < n) {
              const float4* src = reinterpret_cast<const float4*>(
                  p.part + (static_cast<int64_t>(df_chunk_id(g, ch, c + w)) * kDfMaxRows + er) * kDfN + ec);
#pragma unroll
              for (int i = 0; i < 4; ++i) w4[w][i] = __ldcg(src + i);
            }
          }
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            if (c + w < n) {
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                v[4 * i] += w4[w][i].x;
                v[4 * i + 1] += w4[w][i].y;
                v[4 * i + 2] += w4[w][i].z;
                v[4 * i + 3] += w4[w][i].w;
              }
            }
          }
        }
        if (ch.phase == 0) {
          store_f32x16(s_acc + er * kDfN + ec, v);
        } else {
          const int e = s_act[ch.a];
          const int row0 = s_off[e], cnt = s_off[e + 1] - s_off[e];
          const int drow = ch.jm * kDfDB + ec;
          if (er < cnt && drow < p.d) store_f32x16(p.y + static_cast<int64_t>(row0 + er) * p.d + drow, v);
        }
      }
      if (ch.phase == 0) {
        if (!epi_sync(smem_u32(&red_bar), red_phase, p.timeout_ns, &s_abort)) {
          ok = false;
          break;
        }
        // h = silu(gate) * up: gate columns [0, 128), up columns [128, 256) of the same row;
        // item q: row q / 16, h columns (q mod 16) * 8 .. + 8
        for (int q = rt; q < kDfMaxRows * 16; q += 96) {
          const int hr = q >> 4, hc = (q & 15) * 8;
          const int row = s_colrow[ch.a][hr];
          const int f0 = ch.jm * kDfGU + hc;
          if (row >= 0 && f0 < p.F) {
            const float* gt = s_acc + hr * kDfN + hc;
            const float* up = gt + kDfGU;
            uint32_t hw[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
              hw[i] = static_cast<uint32_t>(bf16_bits(silu_df(gt[2 * i]) * up[2 * i])) |
                      (static_cast<uint32_t>(bf16_bits(silu_df(gt[2 * i + 1]) * up[2 * i + 1])) << 16);
            *reinterpret_cast<uint4*>(p.h + static_cast<int64_t>(row) * p.F + f0) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          }
        }
        __threadfence();  // h before the flag below
        if (!epi_sync(smem_u32(&red_bar), red_phase, p.timeout_ns, &s_abort)) {
          ok = false;
          break;
        }
        if (rt == 0) st_release_gpu(p.hflag + ch.tile, 1);
      } else {
        __threadfence();  // y's rows before the block's count below
        if (!epi_sync(smem_u32(&red_bar), red_phase, p.timeout_ns, &s_abort)) {
          ok = false;
          break;
        }
        if (rt == 0) {
          const int prev = atomicAdd(p.mdone + ch.jm, 1);
          __threadfence();
          s_comb = combine && prev == nact - 1;
        }
        if (!epi_sync(smem_u32(&red_bar), red_phase, p.timeout_ns, &s_abort)) {
          ok = false;
          break;
        }
        if (s_comb) {
          // last of the block's tiles: combine columns [256m, 256m + 256) of every token
          for (int col = rt; col < kDfDB; col += 96) {
            const int dcol = ch.jm * kDfDB + col;
            if (dcol >= p.d) continue;
            for (int t = 0; t < p.T; ++t) {
              float acc = 0.f;
              bool any = false;
              for (int jj = 0; jj < p.k; ++jj) {  // choices in ascending order, as moe_unpermute_combine
                int row;
                float wj;
                if constexpr (ROUTE) {
                  row = s_route.row[jj * p.T + t];
                  wj = s_route.tw[t * p.k + jj];
                } else {
                  const int64_t pq = static_cast<int64_t>(t) * p.k + jj;
                  row = __ldcg(p.row_of_pair + pq);
                  wj = __ldcg(p.topk_w + pq);
                }
                if (row >= p.r_max) {
                  report_error(p.status, MOE_ERR_BOUNDS);
                  row = -1;
                }
                if (row < 0) continue;
                acc = fmaf(wj, __ldcg(p.y + static_cast<int64_t>(row) * p.d + dcol), acc);
                any = true;
              }
              const uint16_t rb = p.residual != nullptr ? p.residual[static_cast<int64_t>(t) * p.d + dcol] : uint16_t(0);
              const float rv = __uint_as_float(static_cast<uint32_t>(rb) << 16);
              if (p.out_f32)
                static_cast<float*>(p.out)[static_cast<int64_t>(t) * p.d + dcol] = any ? rv + acc : rv;
              else  // a token with no kept pair passes the residual's bits through unchanged
                static_cast<uint16_t*>(p.out)[static_cast<int64_t>(t) * p.d + dcol] = any ? bf16_bits(rv + acc) : rb;
            }
          }
        }
        // every reducer has read s_comb before the next tile may set it
        if (!epi_sync(smem_u32(&red_bar), red_phase, p.timeout_ns, &s_abort)) {
          ok = false;
          break;
        }
      }
      if (rt == 0) {
        __threadfence_block();
        s_redq_done = ridx + 1;
      }
    }
    if (!ok && rt == 0) {
      s_abort = 1;
      report_error(p.status, MOE_ERR_TIMEOUT);
    }
  }
  if (warp >= 4 && combine && run && nact == 0) {
    // no expert has rows: every token passes its residual through; CTA b takes blocks b, b + G, ...
    const int et = tid - 128;
    for (int m = b; m < g.DB; m += G) {
      for (int half = 0; half < 2; ++half) {
        const int dcol = m * kDfDB + half * 128 + et;
        if (dcol >= p.d) continue;
        for (int t = 0; t < p.T; ++t) {
          const uint16_t rb = p.residual != nullptr ? p.residual[static_cast<int64_t>(t) * p.d + dcol] : uint16_t(0);
          if (p.out_f32)
            static_cast<float*>(p.out)[static_cast<int64_t>(t) * p.d + dcol] = __uint_as_float(static_cast<uint32_t>(rb) << 16);
          else
            static_cast<uint16_t*>(p.out)[static_cast<int64_t>(t) * p.d + dcol] = rb;
        }
      }
    }
  }

  // ---------------------------------------------------------------- departure
  // The last CTA to leave (every other CTA has finished all its reads) puts the counters and
  // flags back to zero, for the next call.
  __threadfence();
  tc_fence_before_sync();
  __syncthreads();
  pdl_trigger();
  if (tid == 0) s_lastcta = atomicAdd(p.sync + 1, 1) == G - 1;
  __syncthreads();
  if (s_lastcta) {
    __threadfence();
    const int ntile = nact * g.Ft + nact * g.DB;
    for (int i = tid; i < nact * g.Ft; i += kDfThreads) p.hflag[i] = 0;
    for (int i = tid; i < ntile; i += kDfThreads) p.tcnt[i] = 0;
    for (int i = tid; i < g.DB; i += kDfThreads) p.mdone[i] = 0;
    if (tid == 0) {
      p.sync[1] = 0;
      p.sync[2] = 0;
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
  // CTAs wait on one another's flags: every CTA must be resident at once, one per SM
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
      a.F % 64 != 0 || a.part == nullptr || a.flags == nullptr || a.sync == nullptr || a.h == nullptr)
    return cudaErrorInvalidValue;
  DeviceInfo di;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  const uint64_t d = static_cast<uint64_t>(a.d), F = static_cast<uint64_t>(a.F);
  const uint64_t N = static_cast<uint64_t>(a.N);
  CUtensorMap mGU, mX, mWD;
  {  // gate and up rows of one expert: [N][2][F][d], boxes of 64 k x 128 rows (rows past F
     // read as zero)
    const uint64_t dims[4] = {d, F, 2, N};
    const uint64_t str[3] = {d * 2, F * d * 2, 2 * F * d * 2};
    const uint32_t box[4] = {kDfBK, kDfGU, 1, 1};
    if (!make_map(&mGU, a.w_gate_up, 4, dims, str, box)) return cudaErrorInvalidValue;
  }
  {  // token rows, boxes of 64 k x 8 rows (rows past the end read as zero): the expert's rows
     // of x_perm, or with the routing in the launch the batch's tokens x[0..T)
    const void* rows = a.route_in_kernel ? static_cast<const void*>(a.route.x) : a.x_perm;
    const uint64_t nrows = a.route_in_kernel ? static_cast<uint64_t>(a.T) : static_cast<uint64_t>(a.r_max);
    const uint64_t dims[2] = {d, nrows};
    const uint64_t str[1] = {d * 2};
    const uint32_t box[2] = {kDfBK, kDfMaxRows};
    if (!make_map(&mX, rows, 2, dims, str, box)) return cudaErrorInvalidValue;
  }
  {  // W_d [N][d][F], boxes of 64 columns of F x 256 rows of d (rows past d read as zero)
    const uint64_t dims[3] = {F, d, N};
    const uint64_t str[2] = {F * 2, d * F * 2};
    const uint32_t box[3] = {kDfBK, kDfDB, 1};
    if (!make_map(&mWD, a.w_down, 3, dims, str, box)) return cudaErrorInvalidValue;
  }
  DfParams p{};
  p.expert_offset = a.expert_offset;
  p.h = a.h;
  p.y = a.y_perm;
  p.part = a.part;
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
  const DecodeFfnChunks ck = decode_ffn_chunks(a.N, a.T, a.k, a.d, a.F);
  p.nca = ck.nca;
  p.ncb = ck.ncb;
  p.hflag = a.flags;
  p.tcnt = a.flags + p.s_max;
  p.mdone = p.tcnt + p.s_max + decode_ffn_max_down_tiles(a.N, a.T, a.k, a.d);
  p.status = a.status;
  p.timeout_ns = a.timeout_ns;
  const int grid = di.sm_count;
  if (grid > kDecodeFfnMaxCtas) return cudaErrorInvalidConfiguration;
  if (!a.route_in_kernel)
    return launch_variant<false, 1>(mGU, mX, mWD, p, grid, s);
  p.route = a.route;
  p.route_ctas = static_cast<int>((a.d + kDecodeSlice - 1) / kDecodeSlice);
  if (p.route_ctas > grid || !use_decode_route(a.T, a.N, a.d) || a.route.x_perm == nullptr ||
      static_cast<int64_t>(a.T) * a.k > grid)
    return cudaErrorInvalidValue;
  const int ept = a.N <= 32 ? 1 : a.N <= 64 ? 2 : a.N <= 128 ? 4 : 8;
  if (ept == 1) return launch_variant<true, 1>(mGU, mX, mWD, p, grid, s);
  if (ept == 2) return launch_variant<true, 2>(mGU, mX, mWD, p, grid, s);
  if (ept == 4) return launch_variant<true, 4>(mGU, mX, mWD, p, grid, s);
  return launch_variant<true, 8>(mGU, mX, mWD, p, grid, s);
}

}  // namespace moe
