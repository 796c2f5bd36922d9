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
// One persistent launch runs both GEMMs, one phase after the other on every CTA:
//   phase 0  h = act(x_perm W_gu^T) per expert: SwiGLU silu(x W_g^T) * (x W_u^T), or GELU (erf
//            form); bf16 inputs, fp32 accumulation in TMEM, activation in fp32, h rounded once
//            to bf16;
//   phase 1  y_perm = h W_d^T per expert, fp32 out.
// A down-projection tile needs its rows of h complete, that is every phase-0 tile of the same
// expert and m-tile. Each finished phase-0 tile adds one to its m-tile's counter (after its h
// stores); the producer of a phase-1 tile streams the tile's W_d blocks into the shared-memory
// ring at once and issues the h loads when the counter is full. So the down projection's
// weight stream starts as soon as a CTA runs out of phase-0 work, instead of after the whole
// first GEMM, its kernel boundary and the second kernel's start. Every CTA must be resident at
// the same time (one CTA per SM, at most one per SM of the grid); each wait is bounded.
//
// Kernel structure (one CTA per SM, 192 threads):
//   warp 0      TMA producer: A tile [BM rows x 64 k] of the expert's rows and the weight tile
//               [256 rows x 64 k] into a STAGES-deep ring of 128B-swizzled shared-memory
//               stages (mbarrier full/empty pairs). For SwiGLU one B tile is the gate rows
//               [f0, f0+128) stacked on the up rows [f0, f0+128) of the same expert, so one MMA
//               chain produces both halves of the activation's input side by side.
//   warp 1      allocates TMEM (two accumulator buffers) and issues tcgen05.mma (M=BM, N=256,
//               K=16, four per stage) from one thread; tcgen05.commit frees smem stages and
//               publishes finished accumulators.
//   warps 2-5   epilogue: tcgen05.ld of the accumulator (thread i owns row i of the tile),
//               activation, conversion and masked global stores; then hand the TMEM buffer
//               back, so the epilogue of one tile overlaps the mainloop of the next.
// Tile scheduler: tiles are (expert, n-tile, m-tile) with m fastest, numbered expert by
// expert; the per-expert m-tile counts come from expert_offset on the device (no host sync).
// Experts without rows produce no tiles. Each phase has one of two schedules, chosen on the
// device from its tile count by a cost model that every CTA evaluates alike:
//   whole tiles   CTAs stride through the tile list;
//   stream-K      the tiles' k blocks, laid end to end, are cut into one equal contiguous range
//                 per CTA, so no CTA idles in a last, partly filled wave. A tile that a range
//                 boundary cuts gets fp32 partial sums from each CTA that covers part of it;
//                 its owner (the CTA holding its first k blocks, which it reaches last) waits
//                 for the others' arrival count and adds the partials in order of CTA index.
//                 Each CTA holds at most two such partial tiles per phase (its first and its
//                 last), so the partials take two slots.
// Every wait is bounded; on timeout the CTA records MOE_ERR_TIMEOUT, stops issuing work, waits
// (bounded) for its own TMA copies and MMAs, frees TMEM and exits.
#include <string.h>

#include <algorithm>
#include <mutex>

#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "launch.h"
#include "tma_host.h"

namespace moe {
namespace {

// Rows per tile (UMMA M) is a template parameter BM: 128, or 64 when no expert can hold more
// than 64 rows. For M = 64 the accumulator's row 16q + i (i < 16) sits in TMEM lane 32q + i.
constexpr int BK = 64;         // k per stage: 64 bf16 = one 128-byte swizzle row
constexpr int kUmmaN = 256;    // UMMA N of both phases (SwiGLU: 128 gate + 128 up columns)
constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;
constexpr int kSmemBudget = 200 * 1024;
constexpr int kDnBn = 256;     // output columns per tile of the down projection

enum { EPI_SWIGLU = 0, EPI_GELU = 1, EPI_STORE_F32 = 2 };

struct PhaseParams {
  void* out;        // h (bf16) or y_perm (fp32)
  int64_t ld_out;   // row stride of out, elements
  int n_out;        // valid output columns per expert (multiple of 16)
  int n_tiles_n;    // ceil(n_out / BN)
  int num_kb;       // K / BK
  // stream-K: 0 disables it; else at most this many CTAs take ranges, each with two partial
  // slots part[cta][slot][row][kUmmaN] of slot_rows rows. The counters are zero between calls.
  int sk_ctas;
  float* part;
  int* tile_counters;
};

struct FfnParams {
  const int32_t* expert_offset;  // [N+1]
  // block-scaled formats: E8M0 scales of the quantised token rows (x) and of h, one 512-byte
  // atom per (m-tile, k block) in the TMEM copy layout (row r, block q at 16 (r % 32) + 4 (r / 32) + q)
  const uint8_t* x_atoms;
  uint8_t* h_atoms;
  int64_t r_max;
  int64_t rows_per_expert;       // no expert may hold more rows (partial slots are this tall)
  int n_experts;
  int slot_rows;
  PhaseParams ph[2];
  int* h_ready;    // per m-tile: phase-0 tiles finished; zero between calls
  int m_tiles_cap; // entries of h_ready (tile counters hold m_tiles_cap * n_tiles_n)
  int* done_ctas;  // CTAs finished; the last one zeroes h_ready
  int* status;
  uint64_t timeout_ns;
  int weight_policy;  // 0 evict_normal, 1 evict_first
};

// Weight storage: bf16, or an MX format (blocks of 32 elements along K sharing one E8M0
// scale) with E4M3 or E2M1 elements, decoded exactly to bf16 in shared memory; or, block-scaled
// (BS8, BS4), the same MX weights read by the block-scaled MMA (kind::mxf8f6f4) against token
// rows and h quantised to MXFP8.
enum { WFMT_BF16 = 0, WFMT_MXFP8 = 1, WFMT_MXFP4 = 2, WFMT_BS8 = 3, WFMT_BS4 = 4 };
constexpr int kBsK = 128;        // block-scaled: k per stage (128 one-byte elements = 128 bytes)
constexpr int kBsSfB = 2048;      // per B stage: raw B scales 1 KB, their atoms 1 KB
constexpr int kBsBudget = 226 * 1024;
constexpr int kBsSmallRows = 32;  // BS tiles with at most this many rows load only those rows
constexpr int kConvThreads = 256;  // MX decoders (warps 7-14)
constexpr int kConvWarps = kConvThreads / 32;

template <int BM, int WFMT>
struct Cfg {
  static constexpr bool MX = WFMT == WFMT_MXFP8 || WFMT == WFMT_MXFP4;  // decoded in smem
  static constexpr bool BS = WFMT == WFMT_BS8 || WFMT == WFMT_BS4;      // block-scaled MMA
  // MX: + the packed-ring producer and 8 decoder warps; BS: + a warp that lays out the weight
  // scales of each stage for the TMEM copy (6) and the weight producer (7)
  static constexpr int THREADS = MX ? kThreads + 32 + kConvThreads : (BS ? kThreads + 64 : kThreads);
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = kUmmaN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  // MX: bf16 stages (decoded from shared memory, not waiting on HBM) and a ring of packed
  // stages, each 256 rows of one 128-byte segment (KG k blocks: 2 of E4M3, 4 of E2M1; one
  // TMA row request then carries 2x or 4x the elements of a bf16 one) plus 2 KG x 256 scales
  static constexpr int ROW_BYTES = WFMT == WFMT_MXFP8 ? BK : BK / 2;  // per row and k block
  static constexpr int KG = MX ? 128 / ROW_BYTES : 1;
  static constexpr int STG_BYTES = MX ? kUmmaN * 128 + 2 * KG * kUmmaN : 0;
  // BS: weight stages (B tile + raw and laid-out scales) beside a ring of SA token-row stages
  // (A tile + its scale atom): rows come from L2, weights from HBM, so the weights get the depth
  static constexpr int SA_BS = 3;
  static constexpr int STAGES_RAW = BS ? (kBsBudget - SA_BS * (A_BYTES + 512)) / (B_BYTES + kBsSfB)
                                       : kSmemBudget / STAGE_BYTES;
  static constexpr int STAGES_FIT = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  // MX: two bf16 B stages (decoded from shared memory; a third measured no faster), a
  // separate ring of SA A stages
  // (token rows, loaded ahead of the decoders: an A copy waits on L2 for about 1.7 us when
  // the weight streams load it), and the rest of 224 KB for packed stages
  static constexpr int kMxBudget = 224 * 1024;
  static constexpr int STAGES = MX ? 2 : STAGES_FIT;
  static constexpr int SA = MX ? (BM == 64 ? 6 : 3) : (BS ? SA_BS : 0);
  static constexpr int B_RING = (MX || BS) ? STAGES * B_BYTES : STAGES * STAGE_BYTES;  // bytes
  static constexpr int A_RING = SA * A_BYTES;
  static constexpr int SST_FIT = MX ? (kMxBudget - B_RING - A_RING) / STG_BYTES : 0;
  static constexpr int SST = SST_FIT > 16 ? 16 : SST_FIT;
  static constexpr int TMEM_COLS = 2 * kUmmaN;
  // accumulator buffers in TMEM: two (the epilogue of one tile overlaps the next tile's MMAs),
  // or one for BS, whose scale factors take TMEM columns 256 (A) and 264-271 (B)
  static constexpr int NACC = BS ? 1 : 2;
  static constexpr int SF_RING = BS ? STAGES * kBsSfB + SA * 512 : 0;
  static constexpr int SMEM_BYTES = B_RING + A_RING + SST * STG_BYTES + SF_RING + 1024;  // + alignment slack
  static_assert(!BS || BM == 128, "block-scaled MMA: M = 128");
  static_assert(TMEM_COLS <= 512, "two accumulators must fit in TMEM");
  static_assert(STAGES >= 2, "pipeline depth");
  static_assert(!MX || SST >= 2, "MX staging depth");
  static_assert(!MX || STG_BYTES % 1024 == 0, "packed stages stay 1024-byte aligned (swizzle)");
  static_assert(BM == 64 || BM == 128, "UMMA M");
};

// Decoders of one MX row segment: 8 elements and the block scale X = 2^(s - 127) -> 8 bf16
// (one 16-byte chunk). Elements convert exactly to fp16 (CUDA's FP8/FP4 conversions), then
// to fp32; the product with a power of two and the final bf16 rounding are exact while the
// result stays in bf16's normal range.
__device__ __forceinline__ float e8m0_to_f32(uint32_t s) {
  if (s == 255u) return __uint_as_float(0x7fc00000u);
  if (s == 0u) return __uint_as_float(0x00400000u);  // 2^-127
  return __uint_as_float(s << 23);
}

__device__ __forceinline__ uint32_t half2raw_to_bf16x2(__half2_raw h, float x) {
  __half_raw lo, hi;
  lo.x = h.x;
  hi.x = h.y;
  return pack_bf16x2(__half2float(__half(lo)) * x, __half2float(__half(hi)) * x);
}

__device__ __forceinline__ uint4 decode8_e4m3(uint2 w, float x) {
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t word = i < 2 ? w.x : w.y;
    const __nv_fp8x2_storage_t pair = static_cast<__nv_fp8x2_storage_t>(word >> (16 * (i & 1)));
    o[i] = half2raw_to_bf16x2(__nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3), x);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ uint4 decode8_e2m1(uint32_t w, float x) {
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {  // byte i holds elements 2i (low nibble) and 2i + 1
    const __nv_fp4x2_storage_t pair = static_cast<__nv_fp4x2_storage_t>(w >> (8 * i));
    o[i] = half2raw_to_bf16x2(__nv_cvt_fp4x2_to_halfraw2(pair, __NV_E2M1), x);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

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
  int gm;     // global m-tile index (counter of the rows' h)
};

// Tile `tile` of a phase with `ntn` n-tiles per m-tile; s_mt[e] = first m-tile of expert e.
template <int BM>
__device__ __forceinline__ TileCoord decode_tile(int tile, int N, int bn, int ntn,
                                                 const int* s_mt, const int* s_off) {
  int lo = 0, hi = N - 1;  // largest e with s_mt[e] * ntn <= tile
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_mt[mid] * ntn <= tile)
      lo = mid;
    else
      hi = mid - 1;
  }
  TileCoord c;
  c.e = lo;
  const int local = tile - s_mt[lo] * ntn;
  const int mt = s_mt[lo + 1] - s_mt[lo];
  const int nt = local / mt;
  const int mi = local - nt * mt;
  c.m0 = s_off[lo] + mi * BM;
  c.rows = min(BM, s_off[lo + 1] - c.m0);
  c.n0 = nt * bn;
  c.gm = s_mt[lo] + mi;
  return c;
}

// Schedule of one phase in units of kg k blocks (kg = 1 for bf16 weights; MX weights stream
// 128-byte row segments, 2 or 4 k blocks, per copy, so their units are those groups). Stream-K
// gives CTA b < g the units [b * total / g, (b + 1) * total / g) of the tiles laid end to end
// (upt = ceil(num_kb / kg) per tile); a tile's last unit may hold fewer than kg k blocks.
struct Sched {
  int sk;         // 1: stream-K, 0: whole tiles
  int g;          // CTAs with a stream-K range
  int tiles;
  int num_kb;     // k blocks per tile
  int kg;         // k blocks per unit
  int upt;        // units per tile
  int64_t total;  // tiles * upt
};

__device__ __forceinline__ int64_t sk_begin(const Sched& s, int b) {
  return static_cast<int64_t>(b) * s.total / s.g;
}
// The CTA whose range holds unit i: the largest b with sk_begin(b) <= i.
__device__ __forceinline__ int sk_cta_of(const Sched& s, int64_t i) {
  return static_cast<int>(((i + 1) * s.g + s.total - 1) / s.total) - 1;
}

// Cost, in k-block times, of the busiest CTA: whole tiles take ceil(tiles / grid) waves of
// num_kb; stream-K takes ceil(total / g) units plus the partial round trip of the tile
// finished last (latency, and a k block's worth of traffic per 32 partial rows). Stream-K is
// chosen when at least 5 % faster. Ranges keep at least kSkMinKb k blocks.
constexpr int kSkMinKb = 4;
constexpr float kTailKb = 2.0f;  // epilogue of the last tile and pipeline refill

__device__ __forceinline__ Sched choose_schedule(int tiles, int grid, int num_kb, int kg,
                                                 int sk_ctas, int slot_rows) {
  const int upt = (num_kb + kg - 1) / kg;
  Sched s{0, 0, tiles, num_kb, kg, upt, static_cast<int64_t>(tiles) * upt};
  if (sk_ctas <= 0 || tiles <= 0) return s;
  const int min_u = max(1, min(kSkMinKb, num_kb) / kg);
  const int64_t by_size = s.total / min_u;
  const int64_t g = by_size < min(grid, sk_ctas) ? by_size : min(grid, sk_ctas);
  if (g < 2) return s;
  const float dp = static_cast<float>((tiles + grid - 1) / grid) * num_kb + kTailKb;
  const float fixup = 2.0f + slot_rows / 32.0f;
  const float sk = static_cast<float>((s.total + g - 1) / g) * kg + kTailKb + fixup;
  if (sk < 0.95f * dp) {
    s.sk = 1;
    s.g = static_cast<int>(g);
  }
  return s;
}

struct Seg {
  int tile, kb0, kb1;  // k blocks [kb0, kb1) of tile; kb0 is a multiple of the unit size
};

// Walks this CTA's segments (a tile and a k-block range of it) of one phase in order; the
// producers, the MMA issuer, the decoders and the epilogue each run their own copy and see
// the same sequence.
struct SegCursor {
  int64_t it, end;
  __device__ __forceinline__ SegCursor(const Sched& s) {
    if (s.sk) {
      const int b = static_cast<int>(blockIdx.x);
      it = b < s.g ? sk_begin(s, b) : 0;
      end = b < s.g ? sk_begin(s, b + 1) : 0;
    } else {
      it = blockIdx.x;
      end = s.tiles;
    }
  }
  __device__ __forceinline__ bool next(const Sched& s, Seg& g) {
    if (it >= end) return false;
    if (s.sk) {
      g.tile = static_cast<int>(it / s.upt);
      const int u0 = static_cast<int>(it - static_cast<int64_t>(g.tile) * s.upt);
      const int64_t left = end - it;
      const int u1 = left < s.upt - u0 ? u0 + static_cast<int>(left) : s.upt;
      g.kb0 = u0 * s.kg;
      g.kb1 = min(u1 * s.kg, s.num_kb);
      it += u1 - u0;
    } else {
      g.tile = static_cast<int>(it);
      g.kb0 = 0;
      g.kb1 = s.num_kb;
      it += gridDim.x;
    }
    return true;
  }
};

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
__device__ __forceinline__ void store_final4(const PhaseParams& p, int64_t row, int col,
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
__device__ __forceinline__ void store_final16(const PhaseParams& p, int64_t row, int col,
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

// One MX block of 32 fp32 values -> E4M3 codes of v / X with X = 2^(floor(log2 amax) - 8),
// X clamped to [2^-127, 2^127] (OCP MX v1.0 conversion: 8 is the exponent of E4M3's largest
// power of two; the elements round to nearest even and saturate at 448). Returns X's E8M0
// code; the codes of elements 0-15 go to lo, 16-31 to hi (element i in byte i).
__device__ __forceinline__ uint32_t mxfp8_block(const float (&v)[32], uint4& lo, uint4& hi) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const int ebits = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu);  // 0: zero or subnormal
  const int e = max(ebits - 127 - 8, -127);
  const float inv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);  // 2^-e exactly
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t p0 = __nv_cvt_float2_to_fp8x2(make_float2(v[4 * i] * inv, v[4 * i + 1] * inv),
                                                 __NV_SATFINITE, __NV_E4M3);
    const uint32_t p1 = __nv_cvt_float2_to_fp8x2(make_float2(v[4 * i + 2] * inv, v[4 * i + 3] * inv),
                                                 __NV_SATFINITE, __NV_E4M3);
    w[i] = p0 | (p1 << 16);
  }
  lo = make_uint4(w[0], w[1], w[2], w[3]);
  hi = make_uint4(w[4], w[5], w[6], w[7]);
  return static_cast<uint32_t>(e + 127);
}

// Byte of the scale of row r (of a 128-row tile) and 32-column block q (of a 128-column k
// block) in a 512-byte scale atom.
__device__ __forceinline__ int sf_atom_byte(int r, int q) { return 16 * (r & 31) + 4 * (r >> 5) + q; }

// h of 32 columns of one row as MXFP8: codes to h (bytes, row stride ld) and the scale into
// the h atom of (m-tile gm, k block col / 128) for the down projection's MMA.
template <int EPI>
__device__ __forceinline__ void store_h_mx32(const FfnParams& fp, const PhaseParams& p,
                                             int64_t row, int col, int gm, int r_local,
                                             const float (&a)[32], const float (&b)[32]) {
  float hv[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) hv[i] = EPI == EPI_SWIGLU ? silu_f(a[i]) * b[i] : gelu_f(a[i]);
  uint4 lo, hi;
  const uint32_t sc = mxfp8_block(hv, lo, hi);
  uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.out) + row * p.ld_out + col);
  dst[0] = lo;
  dst[1] = hi;
  fp.h_atoms[(static_cast<int64_t>(gm) * fp.ph[1].num_kb + col / kBsK) * 512 +
             sf_atom_byte(r_local, (col >> 5) & 3)] = static_cast<uint8_t>(sc);
}

// Epilogue of one segment (all 128 epilogue threads): read the accumulator from TMEM, store
// the final tile or this segment's partial, hand the TMEM buffer back; for a partial, count the
// arrival and, if last, add the partials in order and store the tile. Returns whether this CTA
// wrote the tile's final values in *finished; false on a timed-out wait.
// NACC: TMEM accumulator buffers (segment tc uses buffer tc % NACC). QH: h is stored as MXFP8
// (codes and scale atoms) instead of bf16.
template <int EPI, int BN, int BM, int NACC, bool QH>
__device__ __forceinline__ bool epilogue_segment(const FfnParams& fp, const PhaseParams& p,
                                                 const Sched& sched, const Seg& sg,
                                                 const TileCoord& c, uint32_t tmem_base, int tc,
                                                 uint32_t tfull, uint32_t tempty, uint32_t ebar,
                                                 uint32_t& epi_phase, volatile int* s_abort,
                                                 int* s_fixup, bool* finished) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = warp & 3;  // TMEM lane quadrant this warp may access
  // tile row held by this thread's TMEM lane (M = 64 uses lanes 0-15 of each quadrant)
  const int r_local = BM == 128 ? q * 32 + lane : (lane < 16 ? q * 16 + lane : BM);
  const int buf = NACC == 2 ? tc & 1 : 0;
  const uint32_t tph = NACC == 2 ? (tc >> 1) & 1 : tc & 1;
  const bool got = mbar_wait(tfull, tph, fp.timeout_ns, s_abort);
  if (!__all_sync(0xffffffffu, got)) return false;
  tc_fence_after_sync();
  const bool whole = sg.kb0 == 0 && sg.kb1 == sched.num_kb;
  // partial slot of this segment: 0 when the CTA's range starts inside this tile
  const int64_t t_it0 = static_cast<int64_t>(sg.tile) * sched.upt;  // the tile's first unit
  const int slot = whole ? 0 : (sk_begin(sched, blockIdx.x) >= t_it0 ? 0 : 1);
  float* const my_part =
      p.part + (static_cast<int64_t>(blockIdx.x * 2 + slot) * fp.slot_rows) * kUmmaN;
  const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                         static_cast<uint32_t>(buf * kUmmaN);
  const bool row_ok = r_local < c.rows;
  const int64_t row = static_cast<int64_t>(c.m0) + r_local;
  if (QH && whole) {
#pragma unroll 1
    for (int cc = 0; cc < BN; cc += 32) {
      if (c.n0 + cc >= p.n_out) break;  // warp-uniform: ragged last n-tile (F % 32 == 0)
      float a[32], b[32];
      uint32_t v[32];
      tmem_ld_32x32b_x32(t_row + cc, v);
      if (EPI == EPI_SWIGLU) {
        uint32_t u[32];
        tmem_ld_32x32b_x32(t_row + BN + cc, u);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) b[i] = __uint_as_float(u[i]);
      } else {
        tmem_ld_wait();
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) a[i] = __uint_as_float(v[i]);
      if (row_ok) store_h_mx32<EPI>(fp, p, row, c.n0 + cc, c.gm, r_local, a, b);
    }
  }
#pragma unroll 1
  for (int cc = 0; cc < BN && !(QH && whole); cc += 16) {
    if (c.n0 + cc >= p.n_out) break;  // warp-uniform: ragged last n-tile
    float a[16], b[16];
    uint32_t v[16];
    tmem_ld_32x32b_x16(t_row + cc, v);
    if (EPI == EPI_SWIGLU) {
      uint32_t u[16];
      tmem_ld_32x32b_x16(t_row + BN + cc, u);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 16; ++i) b[i] = __uint_as_float(u[i]);
    } else {
      tmem_ld_wait();
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) a[i] = __uint_as_float(v[i]);
    if (!row_ok) continue;
    if (whole) {
      store_final16<EPI>(p, row, c.n0 + cc, a, b);
    } else {  // this segment's partial tile
      float* dst = my_part + static_cast<int64_t>(r_local) * kUmmaN + cc;
      store_f32x16(dst, a);
      if (EPI == EPI_SWIGLU) store_f32x16(dst + BN, b);
    }
  }
  tc_fence_before_sync();
  mbar_arrive(tempty);  // TMEM buffer free for the next segment
  *finished = whole;
  if (whole) return true;

  // A tile cut by range boundaries is finished by its owner: the first CTA of its range,
  // whose segment (the tile's first k blocks) ends its range, so it is done last. The others
  // publish their partials with one release increment of the tile's counter (after a barrier
  // of the 128 epilogue threads, one fenced thread releases them all); the owner waits for
  // that count, then adds every partial in order of CTA index.
  const int first_cta = sk_cta_of(sched, t_it0);
  const int n_seg = sk_cta_of(sched, t_it0 + sched.upt - 1) - first_cta + 1;
  const bool owner = static_cast<int>(blockIdx.x) == first_cta;
  if (!__all_sync(0xffffffffu, epilogue_sync(ebar, epi_phase, fp.timeout_ns, s_abort))) return false;
  if (!owner) {
    if (threadIdx.x == 64) {
      __threadfence();
      atomicAdd(p.tile_counters + sg.tile, 1);  // result unused: a fire-and-forget reduction
    }
    return true;
  }
  if (threadIdx.x == 64) {
    const bool arrived =
        wait_counter_at_least(p.tile_counters + sg.tile, n_seg - 1, fp.timeout_ns, s_abort);
    if (arrived) p.tile_counters[sg.tile] = 0;  // every other segment has arrived
    *s_fixup = arrived;
  }
  if (!__all_sync(0xffffffffu, epilogue_sync(ebar, epi_phase, fp.timeout_ns, s_abort))) return false;
  if (!*s_fixup) return false;
  const int cols = min(BN, p.n_out - c.n0);
  const int et = threadIdx.x - 64;  // 0..127
  if (QH) {
    // MXFP8 h: item i is (tile row i / G32, 32-column block i % G32), one MX block per item
    constexpr int G32 = BN / 32;
    for (int i = et; i < c.rows * G32; i += kEpiThreads) {
      const int r = i / G32, c32 = (i - r * G32) * 32;
      if (c32 >= cols) continue;
      float ga[32], ub[32];
#pragma unroll
      for (int q = 0; q < 32; ++q) {
        ga[q] = 0.f;
        ub[q] = 0.f;
      }
#pragma unroll 1
      for (int j = 0; j < n_seg; ++j) {  // fixed order (CTA index): deterministic sums
        const int b2 = first_cta + j;
        const int slot2 = sk_begin(sched, b2) >= t_it0 ? 0 : 1;
        const float* src =
            p.part + (static_cast<int64_t>(b2 * 2 + slot2) * fp.slot_rows + r) * kUmmaN + c32;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 v = __ldcg(reinterpret_cast<const float4*>(src) + q);
          ga[4 * q] += v.x; ga[4 * q + 1] += v.y; ga[4 * q + 2] += v.z; ga[4 * q + 3] += v.w;
          if (EPI == EPI_SWIGLU) {
            const float4 u = __ldcg(reinterpret_cast<const float4*>(src + BN) + q);
            ub[4 * q] += u.x; ub[4 * q + 1] += u.y; ub[4 * q + 2] += u.z; ub[4 * q + 3] += u.w;
          }
        }
      }
      store_h_mx32<EPI>(fp, p, static_cast<int64_t>(c.m0) + r, c.n0 + c32, c.gm, r, ga, ub);
    }
    *finished = true;
    return true;
  }
  // All 128 epilogue threads share the reduction: item i is (tile row i / G, float4 column
  // group i % G), so neighbouring threads touch neighbouring columns.
  constexpr int G = BN / 4;
  for (int i = et; i < c.rows * G; i += kEpiThreads) {
    const int r = i / G, c4 = (i - r * G) * 4;
    if (c4 >= cols) continue;
    const int64_t orow = static_cast<int64_t>(c.m0) + r;
    float4 ga = make_float4(0.f, 0.f, 0.f, 0.f), ub = ga;
#pragma unroll 2
    for (int j = 0; j < n_seg; ++j) {  // fixed order (CTA index): deterministic sums
      const int b2 = first_cta + j;
      const int slot2 = sk_begin(sched, b2) >= t_it0 ? 0 : 1;
      const float* src =
          p.part + (static_cast<int64_t>(b2 * 2 + slot2) * fp.slot_rows + r) * kUmmaN + c4;
      const float4 v = __ldcg(reinterpret_cast<const float4*>(src));
      ga.x += v.x; ga.y += v.y; ga.z += v.z; ga.w += v.w;
      if (EPI == EPI_SWIGLU) {
        const float4 u = __ldcg(reinterpret_cast<const float4*>(src + BN));
        ub.x += u.x; ub.y += u.y; ub.z += u.z; ub.w += u.w;
      }
    }
    store_final4<EPI>(p, orow, c.n0 + c4, ga, ub);
  }
  *finished = true;
  return true;
}

// MX weights (WFMT != 0): tmB1 / tmB2 map the packed elements (uint8) and tmS1 / tmS2 the
// scales; warp 6 streams both into the packed ring and warps 7-14 decode each stage into
// the B half of a bf16 stage, which the MMA then reads as for bf16 weights.
template <int EPI1, int BN1, int BM, int WFMT>
__global__ void __launch_bounds__(Cfg<BM, WFMT>::THREADS, 1)
    grouped_ffn_kernel(const __grid_constant__ CUtensorMap tmA1,
                       const __grid_constant__ CUtensorMap tmB1,
                       const __grid_constant__ CUtensorMap tmA2,
                       const __grid_constant__ CUtensorMap tmB2,
                       const __grid_constant__ CUtensorMap tmS1,
                       const __grid_constant__ CUtensorMap tmS2,
                       const __grid_constant__ CUtensorMap tmA1s,
                       const __grid_constant__ CUtensorMap tmA2s, const FfnParams p) {
  using C = Cfg<BM, WFMT>;
  static_assert(EPI1 != EPI_SWIGLU || 2 * BN1 == kUmmaN, "SwiGLU tile: gate | up halves");
  static_assert(EPI1 == EPI_SWIGLU || BN1 == kUmmaN, "GELU tile");
  extern __shared__ __align__(1024) uint8_t dyn_smem[];
  __shared__ __align__(8) uint64_t full_bar[C::STAGES];
  __shared__ __align__(8) uint64_t empty_bar[C::STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t done_bar;
  __shared__ __align__(8) uint64_t epi_bar;
  __shared__ uint32_t s_tmem_base;
  __shared__ volatile int s_abort;
  __shared__ int s_mt[257];   // first m-tile of each expert; s_mt[N] = m-tiles in all
  __shared__ int s_off[257];
  __shared__ Sched s_sched[2];
  __shared__ int s_fixup;
  __shared__ int s_last_cta;
  __shared__ __align__(8) uint64_t sfull_bar[C::MX ? C::SST : 1];
  __shared__ __align__(8) uint64_t sempty_bar[C::MX ? C::SST : 1];
  __shared__ __align__(8) uint64_t afull_bar[(C::MX || C::BS) ? C::SA : 1];
  __shared__ __align__(8) uint64_t aempty_bar[(C::MX || C::BS) ? C::SA : 1];
  __shared__ __align__(8) uint64_t sfready_bar[C::BS ? C::STAGES : 1];  // BS: stage's scale atoms laid out

  pdl_trigger();
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int N = p.n_experts;
  const uint32_t tiles = (smem_u32(dyn_smem) + 1023u) & ~1023u;
  // bf16: stage s = [A | B]; MX: B stages, then the A ring, then the packed ring
  const uint32_t stg0 = tiles + C::B_RING + C::A_RING;
  constexpr bool kSplitA = C::MX || C::BS;  // the A operand has its own ring
  auto a_addr = [&](int i) -> uint32_t {
    return kSplitA ? tiles + C::B_RING + i * C::A_BYTES : tiles + i * C::STAGE_BYTES;
  };
  auto b_addr = [&](int i) -> uint32_t {
    return kSplitA ? tiles + i * C::B_BYTES : tiles + i * C::STAGE_BYTES + C::A_BYTES;
  };
  constexpr int AST = kSplitA ? C::SA : C::STAGES;  // stages of the A operand's ring
  // BS: per weight stage [raw B scales [2][4][128] | B scale atoms [2][512]], then per A stage
  // the rows' scale atom (512 B)
  const uint32_t sf0 = stg0 + C::SST * C::STG_BYTES;
  auto sf_addr = [&](int i) -> uint32_t { return sf0 + i * kBsSfB; };
  auto sfa_addr = [&](int i) -> uint32_t { return sf0 + C::STAGES * kBsSfB + i * 512; };
  // BS: the A scale atom of (m-tile gm, k block kb) of phase ph
  auto a_atom = [&](int ph, int gm, int kb) -> const uint8_t* {
    return (ph == 0 ? p.x_atoms : p.h_atoms) + (static_cast<int64_t>(gm) * p.ph[ph].num_kb + kb) * 512;
  };
  constexpr int KX = C::BS ? kBsK : BK;  // A / B column coordinate step per k block
  uint64_t* const a_full = kSplitA ? afull_bar : full_bar;
  uint64_t* const a_empty = kSplitA ? aempty_bar : empty_bar;

  if (threadIdx.x == 0) {
    prefetch_tensormap(&tmA1);
    prefetch_tensormap(&tmB1);
    prefetch_tensormap(&tmA2);
    prefetch_tensormap(&tmB2);
    if (C::MX || C::BS) {
      prefetch_tensormap(&tmS1);
      prefetch_tensormap(&tmS2);
    }
    if (C::MX) {
      for (int s = 0; s < C::SST; ++s) {
        mbar_init(smem_u32(&sfull_bar[s]), 1);
        mbar_init(smem_u32(&sempty_bar[s]), kConvWarps);
      }
    }
    for (int s = 0; s < C::STAGES; ++s) {
      // MX: B stages filled by the decoders, one arrival per decoder warp
      mbar_init(smem_u32(&full_bar[s]), C::MX ? kConvWarps : 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int s = 0; s < C::SA; ++s) {
      mbar_init(smem_u32(&afull_bar[s]), 1);
      mbar_init(smem_u32(&aempty_bar[s]), 1);
    }
    if (C::BS)
      for (int s = 0; s < C::STAGES; ++s) mbar_init(smem_u32(&sfready_bar[s]), 1);
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
    // Per-expert m-tile counts and their exclusive prefix (experts lane*per .. lane*per+per-1).
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
        if (a < 0 || b < a || b > p.r_max || b - a > p.rows_per_expert)
          bad = true;
        else
          cnt[i] = (b - a + BM - 1) / BM;
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
    if (__shfl_sync(0xffffffffu, incl, 31) > p.m_tiles_cap) {  // overlapping offsets: no tiles
      bad = true;
      for (int i = 0; i < 8; ++i) {
        const int e = lane * per + i;
        if (i < per && e < N) s_mt[e] = 0;
      }
      incl = 0;
    }
    if (lane == 31) {
      s_mt[N] = incl;
      for (int ph = 0; ph < 2; ++ph)
        s_sched[ph] = choose_schedule(incl * p.ph[ph].n_tiles_n, gridDim.x, p.ph[ph].num_kb,
                                      C::KG, p.ph[ph].sk_ctas, p.slot_rows);
    }
    if (bad) report_error(p.status, MOE_ERR_BOUNDS);  // such an expert gets no tiles
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();

  const uint32_t tmem_base = s_tmem_base;
  const int h_target = p.ph[0].n_tiles_n;  // phase-0 tiles per m-tile

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      const uint64_t pol_a = make_policy(2);
      const uint64_t pol_b = make_policy(p.weight_policy);
      int it = 0;
      bool ok = true;
      for (int ph = 0; ph < 2 && ok; ++ph) {
        const Sched sc = s_sched[ph];
        const int bn = ph == 0 ? BN1 : kDnBn;
        SegCursor cur(sc);
        Seg sg;
        while (ok && cur.next(sc, sg)) {
          const TileCoord c = decode_tile<BM>(sg.tile, N, bn, p.ph[ph].n_tiles_n, s_mt, s_off);
          // BS: a tile of at most 32 rows loads just those (the MMA's other rows read stale
          // shared memory; their results are never stored)
          const bool small_a = C::BS && c.rows <= kBsSmallRows;
          const CUtensorMap* tA = small_a ? (ph == 0 ? &tmA1s : &tmA2s) : (ph == 0 ? &tmA1 : &tmA2);
          const uint32_t a_bytes = small_a ? kBsSmallRows * 128 : C::A_BYTES;
          // phase 1: the W_d blocks go out at once; the h blocks once the rows' h is complete
          // (one poll here: an acquire load stalls this thread for an L2 round trip)
          bool ready = ph == 0 || ld_acquire_gpu(p.h_ready + c.gm) >= h_target;
          int pend_from = -1;  // first iteration whose stage holds its B block but not its A
          const int seg_it0 = it;
          for (int kb = sg.kb0; kb < sg.kb1; ++kb) {
            const int s = it % AST;
            const uint32_t par = (it / AST) & 1;
            if (!mbar_wait(smem_u32(&a_empty[s]), par ^ 1u, p.timeout_ns, &s_abort)) {
              ok = false;
              break;
            }
            const uint32_t fb = smem_u32(&a_full[s]);
            const uint32_t a_dst = a_addr(s);
            const uint32_t b_dst = b_addr(s);
            mbar_arrive_expect_tx(fb, C::MX ? C::A_BYTES : (C::BS ? a_bytes + 512 : C::STAGE_BYTES));
            if (!C::MX && !C::BS) {  // MX: the decoders fill the B half; BS: warp 7 loads it
              if (ph == 0) {
                if (EPI1 == EPI_SWIGLU) {
                  tma_load_4d(b_dst, &tmB1, fb, kb * BK, c.n0, 0, c.e, pol_b);
                  tma_load_4d(b_dst + BN1 * BK * 2, &tmB1, fb, kb * BK, c.n0, 1, c.e, pol_b);
                } else {
                  tma_load_3d(b_dst, &tmB1, fb, kb * BK, c.n0, c.e, pol_b);
                }
              } else {
                tma_load_3d(b_dst, &tmB2, fb, kb * BK, c.n0, c.e, pol_b);
              }
            }
            if (ready) {
              tma_load_2d(a_dst, tA, fb, kb * KX, c.m0, pol_a);
              if (C::BS) bulk_load(sfa_addr(s), a_atom(ph, c.gm, kb), 512, fb);
              ++it;
              continue;
            }
            if (pend_from < 0) pend_from = it;
            if (it - pend_from + 1 == AST || kb + 1 == sg.kb1) {
              // every stage holds a W_d block (or the segment ends): wait for the rows' h
              if (!wait_counter_at_least(p.h_ready + c.gm, h_target, p.timeout_ns, &s_abort))
                ok = false;  // the h loads below still complete the armed stages
              fence_proxy_async_global();
              for (int j = pend_from; j <= it; ++j) {
                const int sj = j % AST;
                const int kbj = sg.kb0 + (j - seg_it0);
                tma_load_2d(a_addr(sj), tA, smem_u32(&a_full[sj]), kbj * KX, c.m0, pol_a);
                if (C::BS) bulk_load(sfa_addr(sj), a_atom(ph, c.gm, kbj), 512, smem_u32(&a_full[sj]));
              }
              pend_from = -1;
              ready = true;
            }
            ++it;
            if (!ok) break;
          }
        }
      }
      if (!ok) {
        s_abort = 1;
        report_error(p.status, MOE_ERR_TIMEOUT);
      }
      // No TMA write may still be landing in shared memory when the CTA exits.
      for (int i = max(0, it - AST); i < it; ++i)
        mbar_wait(smem_u32(&a_full[i % AST]), (i / AST) & 1, kDrainTimeoutNs, nullptr);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if constexpr (C::BS) {
      // Block-scaled: once warp 6 has laid out a stage's scale atoms (which implies the stage's
      // loads have landed), lane 0 copies the A and B atoms into TMEM (A at column 256, B at
      // 264-271) and issues the four K = 32 MMAs. TMEM copies and MMAs of one thread run in
      // issue order, so one scale area in TMEM serves every stage.
      if (lane == 0) {
        constexpr int kBFmt = WFMT == WFMT_BS4 ? 5 : 0;  // E2M1 or E4M3 weights; A is E4M3
        const uint32_t t_sfa = tmem_base + kUmmaN, t_sfb = tmem_base + kUmmaN + 8;
        int it = 0, tc = 0;
        bool ok = true;
        bool issued = false;
        for (int ph = 0; ph < 2 && ok; ++ph) {
          const Sched sc = s_sched[ph];
          SegCursor cur(sc);
          Seg sg;
          for (; ok && cur.next(sc, sg); ++tc) {
            // one accumulator: the epilogue has read the previous segment's
            if (!mbar_wait(smem_u32(&tempty_bar[0]), (tc & 1) ^ 1u, p.timeout_ns, &s_abort)) {
              ok = false;
              break;
            }
            tc_fence_after_sync();
            for (int kb = sg.kb0; kb < sg.kb1; ++kb, ++it) {
              const int s = it % C::STAGES, sa = it % C::SA;
              if (!mbar_wait(smem_u32(&sfready_bar[s]), (it / C::STAGES) & 1, p.timeout_ns, &s_abort) ||
                  !mbar_wait(smem_u32(&afull_bar[sa]), (it / C::SA) & 1, p.timeout_ns, &s_abort)) {
                ok = false;
                break;
              }
              tc_fence_after_sync();
              const uint32_t a_base = a_addr(sa), b_base = b_addr(s);
              tc_cp_32x128b_x4(t_sfa, smem_desc_plain(sfa_addr(sa)));
              tc_cp_32x128b_x4(t_sfb, smem_desc_plain(sf_addr(s) + 1024));
              tc_cp_32x128b_x4(t_sfb + 4, smem_desc_plain(sf_addr(s) + 1536));
#pragma unroll
              for (int kk = 0; kk < kBsK / 32; ++kk)
                tc_mma_mx(tmem_base, smem_desc_k_sw128(a_base + kk * 32),
                          smem_desc_k_sw128(b_base + kk * 32), idesc_mx(BM, kUmmaN, 0, kBFmt, kk),
                          t_sfa | (static_cast<uint32_t>(kk) << 30),
                          t_sfb | (static_cast<uint32_t>(kk) << 30),
                          (kb != sg.kb0 || kk != 0) ? 1u : 0u);
              tc_commit(smem_u32(&empty_bar[s]));
              tc_commit(smem_u32(&aempty_bar[sa]));
              issued = true;
            }
            if (!ok) break;
            tc_commit(smem_u32(&tfull_bar[0]));
          }
        }
        if (!ok) {
          s_abort = 1;
          report_error(p.status, MOE_ERR_TIMEOUT);
        }
        if (issued) {
          tc_commit(smem_u32(&done_bar));
          mbar_wait(smem_u32(&done_bar), 0, kDrainTimeoutNs, nullptr);
        }
      }
    } else if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, kUmmaN);
      int it = 0, tc = 0;
      bool ok = true;
      bool issued = false;
      for (int ph = 0; ph < 2 && ok; ++ph) {
        const Sched sc = s_sched[ph];
        SegCursor cur(sc);
        Seg sg;
        for (; ok && cur.next(sc, sg); ++tc) {
          const int buf = tc & 1;
          const uint32_t tph = (tc >> 1) & 1;
          if (!mbar_wait(smem_u32(&tempty_bar[buf]), tph ^ 1u, p.timeout_ns, &s_abort)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * kUmmaN);
          for (int kb = sg.kb0; kb < sg.kb1; ++kb, ++it) {
            const int s = it % C::STAGES, sa = it % AST;
            const uint32_t par = (it / C::STAGES) & 1;
            if (!mbar_wait(smem_u32(&full_bar[s]), par, p.timeout_ns, &s_abort) ||
                (C::MX && !mbar_wait(smem_u32(&afull_bar[sa]), (it / AST) & 1, p.timeout_ns, &s_abort))) {
              ok = false;
              break;
            }
            tc_fence_after_sync();
            const uint32_t a_base = a_addr(C::MX ? sa : s);
            const uint32_t b_base = b_addr(s);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              tc_mma_f16(d_tmem, smem_desc_k_sw128(a_base + kk * 32),
                         smem_desc_k_sw128(b_base + kk * 32), idesc,
                         (kb != sg.kb0 || kk != 0) ? 1u : 0u);
            }
            issued = true;
            tc_commit(smem_u32(&empty_bar[s]));
            if (C::MX) tc_commit(smem_u32(&aempty_bar[sa]));
          }
          if (!ok) break;
          tc_commit(smem_u32(&tfull_bar[buf]));
        }
      }
      if (!ok) {
        s_abort = 1;
        report_error(p.status, MOE_ERR_TIMEOUT);
      }
      // every issued MMA has finished before TMEM is freed, also when the epilogue gave up
      // on a tile whose MMAs this thread had already issued
      if (issued) {
        tc_commit(smem_u32(&done_bar));
        mbar_wait(smem_u32(&done_bar), 0, kDrainTimeoutNs, nullptr);
      }
    }
  } else if (warp < 6) {
    // ---------------------------------------------------------------- epilogue (warps 2..5)
    int tc = 0;
    uint32_t epi_phase = 0;
    bool ok = true;
    for (int ph = 0; ph < 2 && ok; ++ph) {
      const Sched sc = s_sched[ph];
      const int bn = ph == 0 ? BN1 : kDnBn;
      SegCursor cur(sc);
      Seg sg;
      for (; cur.next(sc, sg); ++tc) {
        const TileCoord c = decode_tile<BM>(sg.tile, N, bn, p.ph[ph].n_tiles_n, s_mt, s_off);
        const int bi = C::NACC == 2 ? (tc & 1) : 0;
        const uint32_t tf = smem_u32(&tfull_bar[bi]), te = smem_u32(&tempty_bar[bi]);
        bool finished = false;
        if (ph == 0)
          ok = epilogue_segment<EPI1, BN1, BM, C::NACC, C::BS>(p, p.ph[0], sc, sg, c, tmem_base, tc,
                                                               tf, te, smem_u32(&epi_bar), epi_phase,
                                                               &s_abort, &s_fixup, &finished);
        else
          ok = epilogue_segment<EPI_STORE_F32, kDnBn, BM, C::NACC, false>(
              p, p.ph[1], sc, sg, c, tmem_base, tc, tf, te, smem_u32(&epi_bar), epi_phase,
              &s_abort, &s_fixup, &finished);
        if (!ok) break;
        if (ph == 0 && finished) {
          // this CTA wrote the tile's h: order it before TMA loads, then count it (one fenced
          // thread after the barrier releases every epilogue thread's stores)
          fence_proxy_async_global();
          if (!__all_sync(0xffffffffu, epilogue_sync(smem_u32(&epi_bar), epi_phase, p.timeout_ns, &s_abort))) {
            ok = false;
            break;
          }
          if (threadIdx.x == 64) {
            __threadfence();
            atomicAdd(p.h_ready + c.gm, 1);
          }
        }
      }
    }
    if (!ok) {
      s_abort = 1;
      report_error(p.status, MOE_ERR_TIMEOUT);
    }
  } else if (C::BS && warp == 6) {
    // ---------------------------------------------------------------- BS scale layout (warp 6)
    // Each stage's raw weight scales ([half][4 blocks][128 rows] bytes, as TMA loaded them)
    // become the two 512-byte atoms of the TMEM copy layout: row r = r0 + 32 r1 of half j and
    // block q at byte 16 r0 + 4 r1 + q of atom j; lane r0 writes its 16 bytes of each atom.
    // The stage is written again only after its MMAs (and their TMEM copies) have finished.
    int it = 0;
    bool ok = true;
    for (int ph = 0; ph < 2 && ok; ++ph) {
      const Sched sc = s_sched[ph];
      SegCursor cur(sc);
      Seg sg;
      while (ok && cur.next(sc, sg)) {
        for (int kb = sg.kb0; kb < sg.kb1; ++kb, ++it) {
          const int s = it % C::STAGES;
          ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&full_bar[s]), (it / C::STAGES) & 1,
                                                  p.timeout_ns, &s_abort));
          if (!ok) break;
          const uint8_t* raw = dyn_smem + (sf_addr(s) - smem_u32(dyn_smem));
          uint8_t* atoms = dyn_smem + (sf_addr(s) + 1024 - smem_u32(dyn_smem));
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            uint32_t w[4];
#pragma unroll
            for (int r1 = 0; r1 < 4; ++r1) {
              const uint8_t* src = raw + j * 512 + r1 * 32 + lane;
              w[r1] = static_cast<uint32_t>(src[0]) | (static_cast<uint32_t>(src[128]) << 8) |
                      (static_cast<uint32_t>(src[256]) << 16) | (static_cast<uint32_t>(src[384]) << 24);
            }
            *reinterpret_cast<uint4*>(atoms + j * 512 + lane * 16) = make_uint4(w[0], w[1], w[2], w[3]);
          }
          fence_proxy_async_smem();  // generic stores -> visible to the tensor core's copy
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&sfready_bar[s]));
        }
      }
    }
    if (!ok && lane == 0) {
      s_abort = 1;
      report_error(p.status, MOE_ERR_TIMEOUT);
    }
  } else if (C::BS && warp == 7) {
    // ---------------------------------------------------------------- BS weight producer (warp 7)
    // Weight tiles and their raw scales ([half][4 blocks][128 rows] bytes) into the weight ring,
    // running ahead of the token rows (warp 0), which come from L2.
    if (lane == 0) {
      const uint64_t pol_b = make_policy(p.weight_policy);
      int it = 0;
      bool ok = true;
      for (int ph = 0; ph < 2 && ok; ++ph) {
        const Sched sc = s_sched[ph];
        const int bn = ph == 0 ? BN1 : kDnBn;
        SegCursor cur(sc);
        Seg sg;
        while (ok && cur.next(sc, sg)) {
          const TileCoord c = decode_tile<BM>(sg.tile, N, bn, p.ph[ph].n_tiles_n, s_mt, s_off);
          for (int kb = sg.kb0; kb < sg.kb1; ++kb, ++it) {
            const int s = it % C::STAGES;
            if (!mbar_wait(smem_u32(&empty_bar[s]), ((it / C::STAGES) & 1) ^ 1u, p.timeout_ns, &s_abort)) {
              ok = false;
              break;
            }
            const uint32_t fb = smem_u32(&full_bar[s]);
            const uint32_t b_dst = b_addr(s), sfr = sf_addr(s);
            // E2M1 through the padded 4-bit type counts its packed bytes, half the smem it fills
            mbar_arrive_expect_tx(fb, (WFMT == WFMT_BS4 ? C::B_BYTES / 2 : C::B_BYTES) + 1024);
            const int kx = kb * kBsK;
            if (ph == 0 && EPI1 == EPI_SWIGLU) {
              tma_load_4d(b_dst, &tmB1, fb, kx, c.n0, 0, c.e, pol_b);
              tma_load_4d(b_dst + BN1 * 128, &tmB1, fb, kx, c.n0, 1, c.e, pol_b);
              tma_load_4d(sfr, &tmS1, fb, c.n0, 0, 4 * kb, c.e, pol_b);
              tma_load_4d(sfr + 512, &tmS1, fb, c.n0, 1, 4 * kb, c.e, pol_b);
            } else {
              const CUtensorMap* tb = ph == 0 ? &tmB1 : &tmB2;
              const CUtensorMap* ts = ph == 0 ? &tmS1 : &tmS2;
              tma_load_3d(b_dst, tb, fb, kx, c.n0, c.e, pol_b);
              tma_load_3d(sfr, ts, fb, c.n0, 4 * kb, c.e, pol_b);
              tma_load_3d(sfr + 512, ts, fb, c.n0 + 128, 4 * kb, c.e, pol_b);
            }
          }
        }
      }
      if (!ok) {
        s_abort = 1;
        report_error(p.status, MOE_ERR_TIMEOUT);
      }
      for (int i = max(0, it - C::STAGES); i < it; ++i)
        mbar_wait(smem_u32(&full_bar[i % C::STAGES]), (i / C::STAGES) & 1, kDrainTimeoutNs, nullptr);
    }
  } else if (C::MX && warp == 6) {
    // ---------------------------------------------------------------- MX packed-ring producer
    // One packed stage per unit of KG k blocks: 256 rows x 128 bytes (128B-swizzled) and the
    // rows' 2 KG block scales.
    if (lane == 0) {
      const uint64_t pol_b = make_policy(p.weight_policy);
      int su = 0;
      bool ok = true;
      for (int ph = 0; ph < 2 && ok; ++ph) {
        const Sched sc = s_sched[ph];
        const int bn = ph == 0 ? BN1 : kDnBn;
        SegCursor cur(sc);
        Seg sg;
        while (ok && cur.next(sc, sg)) {
          const TileCoord c = decode_tile<BM>(sg.tile, N, bn, p.ph[ph].n_tiles_n, s_mt, s_off);
          for (int kb = sg.kb0; kb < sg.kb1; kb += C::KG, ++su) {
            const int s = su % C::SST;
            if (!mbar_wait(smem_u32(&sempty_bar[s]), ((su / C::SST) & 1) ^ 1u, p.timeout_ns, &s_abort)) {
              ok = false;
              break;
            }
            const uint32_t fb = smem_u32(&sfull_bar[s]);
            const uint32_t dst = stg0 + s * C::STG_BYTES;
            const uint32_t sc_dst = dst + kUmmaN * 128;  // scales after the 32 KB of elements
            mbar_arrive_expect_tx(fb, C::STG_BYTES);
            const int kx = kb * C::ROW_BYTES;  // byte column of the unit's first k block
            if (ph == 0 && EPI1 == EPI_SWIGLU) {
              tma_load_4d(dst, &tmB1, fb, kx, c.n0, 0, c.e, pol_b);              // gate rows
              tma_load_4d(dst + BN1 * 128, &tmB1, fb, kx, c.n0, 1, c.e, pol_b);  // up rows
              tma_load_4d(sc_dst, &tmS1, fb, c.n0, 0, 2 * kb, c.e, pol_b);       // [2KG][128] gate
              tma_load_4d(sc_dst + 2 * C::KG * BN1, &tmS1, fb, c.n0, 1, 2 * kb, c.e, pol_b);
            } else if (ph == 0) {
              tma_load_3d(dst, &tmB1, fb, kx, c.n0, c.e, pol_b);
              tma_load_3d(sc_dst, &tmS1, fb, c.n0, 2 * kb, c.e, pol_b);  // [2KG][256]
            } else {
              tma_load_3d(dst, &tmB2, fb, kx, c.n0, c.e, pol_b);
              tma_load_3d(sc_dst, &tmS2, fb, c.n0, 2 * kb, c.e, pol_b);
            }
          }
        }
      }
      if (!ok) {
        s_abort = 1;
        report_error(p.status, MOE_ERR_TIMEOUT);
      }
      for (int i = max(0, su - C::SST); i < su; ++i)
        mbar_wait(smem_u32(&sfull_bar[i % C::SST]), (i / C::SST) & 1, kDrainTimeoutNs, nullptr);
    }
  } else if (C::MX) {
    // ---------------------------------------------------------------- MX decoders (warps 7..14)
    // Thread r decodes row r of every k block: 64 elements (8 chunks of 8) from its 128-byte
    // packed row segment (128B-swizzled: 16-byte chunk q at 16 * (q ^ (r & 7))) with the
    // row's two block scales, into the 128B-swizzled K-major bf16 layout the MMA reads (chunk
    // c of row r at 16 * (c ^ (r & 7))). A packed stage is released after its last k block.
    const int r = threadIdx.x - (kThreads + 32);  // 0..255
    int it = 0, su = 0;
    bool ok = true;
    for (int ph = 0; ph < 2 && ok; ++ph) {
      const Sched sc = s_sched[ph];
      // scale layout of this phase's stages: SwiGLU gate/up halves, or one [2KG][256] block
      const bool halves = ph == 0 && EPI1 == EPI_SWIGLU;
      const int sc_base = halves ? (r >> 7) * (2 * C::KG * 128) + (r & 127) : r;
      const int sc_step = halves ? 128 : 256;
      SegCursor cur(sc);
      Seg sg;
      while (ok && cur.next(sc, sg)) {
        for (int kb = sg.kb0; kb < sg.kb1; ++kb, ++it) {
          const int j = (kb - sg.kb0) % C::KG;  // k block within the packed stage
          const int s2 = su % C::SST, s = it % C::STAGES;
          bool got = true;
          if (j == 0) got = mbar_wait(smem_u32(&sfull_bar[s2]), (su / C::SST) & 1, p.timeout_ns, &s_abort);
          got = got && mbar_wait(smem_u32(&empty_bar[s]), ((it / C::STAGES) & 1) ^ 1u, p.timeout_ns, &s_abort);
          if (!got) {
            ok = false;
            break;
          }
          const uint8_t* stg = dyn_smem + (stg0 - smem_u32(dyn_smem)) + s2 * C::STG_BYTES;
          const uint8_t* scl = stg + kUmmaN * 128;
          const float x0 = e8m0_to_f32(scl[sc_base + (2 * j) * sc_step]);
          const float x1 = e8m0_to_f32(scl[sc_base + (2 * j + 1) * sc_step]);
          // this k block's part of the packed row (64 or 32 bytes), then the eight chunks
          constexpr int kQ = C::ROW_BYTES / 16;
          uint4 raw[kQ];
#pragma unroll
          for (int q = 0; q < kQ; ++q)
            raw[q] = *reinterpret_cast<const uint4*>(stg + r * 128 + (((j * kQ + q) ^ (r & 7)) << 4));
          const uint32_t* wd = reinterpret_cast<const uint32_t*>(raw);
          uint8_t* bdst = dyn_smem + (b_addr(s) - smem_u32(dyn_smem)) + r * 128;
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const float x = ch < 4 ? x0 : x1;  // elements 0..31: block 0; 32..63: block 1
            uint4 v;
            if (WFMT == WFMT_MXFP8)
              v = decode8_e4m3(make_uint2(wd[2 * ch], wd[2 * ch + 1]), x);
            else
              v = decode8_e2m1(wd[ch], x);
            *reinterpret_cast<uint4*>(bdst + ((ch ^ (r & 7)) << 4)) = v;
          }
          fence_proxy_async_smem();  // generic stores -> visible to the tensor core
          __syncwarp();
          const bool last = j == C::KG - 1 || kb + 1 == sg.kb1;
          if (lane == 0) {  // one arrival per warp on each barrier
            mbar_arrive(smem_u32(&full_bar[s]));
            if (last) mbar_arrive(smem_u32(&sempty_bar[s2]));
          }
          if (last) ++su;
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
  // the last CTA to finish zeroes the m-tile counters for the next call
  if (threadIdx.x == 0) {
    __threadfence();
    s_last_cta = atomicAdd(p.done_ctas, 1) == static_cast<int>(gridDim.x) - 1;
  }
  __syncthreads();
  if (s_last_cta) {
    __threadfence();
    for (int i = threadIdx.x; i < s_mt[N]; i += C::THREADS) p.h_ready[i] = 0;
    if (threadIdx.x == 0) *p.done_ctas = 0;
  }
}

// ------------------------------------------------------------------ CTA-pair kernel
// bf16 weights in batches whose experts hold many 128-row m-tiles (the tensor-bound regime): a
// cluster of two CTAs takes two neighbouring m-tiles of one expert and the same output
// columns. The even CTA issues M = 256 MMAs (cta_group::2); each CTA holds its own 128 token
// rows and half of the 256 weight rows (SwiGLU: the gate rows in the even CTA, the up rows in
// the odd one). Each SM's tensor core then reads 8 KB of operands per MMA instead of 12 KB, so
// the TMA writes and MMA reads of shared memory stay within its bandwidth. Whole tiles only;
// the down projection waits on the same per-m-tile h counters as the one-CTA kernel. A pair
// whose odd m-tile lies past its expert's rows computes it (from whatever rows TMA returns)
// and stores nothing.
constexpr int kPairStageBytes = 128 * BK * 2 * 2;           // A 16 KB + half of B 16 KB
constexpr int kPairStages = kSmemBudget / kPairStageBytes;  // 6
constexpr int kPairSmemBytes = kPairStages * kPairStageBytes + 1024;

struct PairTile {
  int e, m0, rows, n0, gm;
  bool valid;  // this CTA's m-tile exists (else rows = 0)
};

// Pair tile `tile` of a phase with ntn n-tiles; s_mp[e] = first m-tile pair of expert e.
__device__ __forceinline__ PairTile decode_pair_tile(int tile, int N, int bn, int ntn, int rank,
                                                     const int* s_mp, const int* s_mt,
                                                     const int* s_off) {
  int lo = 0, hi = N - 1;  // largest e with s_mp[e] * ntn <= tile
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_mp[mid] * ntn <= tile)
      lo = mid;
    else
      hi = mid - 1;
  }
  PairTile c;
  c.e = lo;
  const int local = tile - s_mp[lo] * ntn;
  const int np = s_mp[lo + 1] - s_mp[lo];
  const int nt = local / np;
  const int mi = 2 * (local - nt * np) + rank;
  c.valid = mi < s_mt[lo + 1] - s_mt[lo];
  c.m0 = s_off[lo] + mi * 128;
  c.rows = c.valid ? min(128, s_off[lo + 1] - c.m0) : 0;
  c.n0 = nt * bn;
  c.gm = s_mt[lo] + mi;
  return c;
}

template <int EPI1, int BN1>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_ffn_pair_kernel(const __grid_constant__ CUtensorMap tmA1,
                            const __grid_constant__ CUtensorMap tmB1,
                            const __grid_constant__ CUtensorMap tmA2,
                            const __grid_constant__ CUtensorMap tmB2, const FfnParams p) {
  static_assert(EPI1 != EPI_SWIGLU || 2 * BN1 == kUmmaN, "SwiGLU tile: gate | up halves");
  static_assert(EPI1 == EPI_SWIGLU || BN1 == kUmmaN, "GELU tile");
  extern __shared__ __align__(1024) uint8_t dyn_smem[];
  __shared__ __align__(8) uint64_t full_bar[kPairStages];   // even CTA: both CTAs' bytes
  __shared__ __align__(8) uint64_t empty_bar[kPairStages];  // both CTAs (multicast commit)
  __shared__ __align__(8) uint64_t tfull_bar[2];            // both CTAs (multicast commit)
  __shared__ __align__(8) uint64_t tempty_bar[2];           // even CTA: both epilogues
  __shared__ __align__(8) uint64_t done_bar;
  __shared__ __align__(8) uint64_t epi_bar;
  __shared__ uint32_t s_tmem_base;
  __shared__ volatile int s_abort;
  __shared__ int s_mt[257], s_mp[257], s_off[257];
  __shared__ int s_tiles[2];
  __shared__ int s_last_cta;

  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = p.n_experts;
  const int rank = static_cast<int>(cluster_ctarank());
  const bool lead = rank == 0;
  const int cl = static_cast<int>(blockIdx.x) >> 1, ncl = static_cast<int>(gridDim.x) >> 1;
  const uint32_t tiles0 = (smem_u32(dyn_smem) + 1023u) & ~1023u;
  auto a_addr = [&](int s) -> uint32_t { return tiles0 + s * kPairStageBytes; };
  auto b_addr = [&](int s) -> uint32_t { return tiles0 + s * kPairStageBytes + 128 * BK * 2; };

  if (threadIdx.x == 0) {
    prefetch_tensormap(&tmA1);
    prefetch_tensormap(&tmB1);
    prefetch_tensormap(&tmA2);
    prefetch_tensormap(&tmB2);
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&tfull_bar[b]), 1);
      mbar_init(smem_u32(&tempty_bar[b]), 2 * kEpiThreads);
    }
    mbar_init(smem_u32(&done_bar), 1);
    mbar_init(smem_u32(&epi_bar), kEpiThreads);
    s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    __syncwarp();
    tmem_alloc_pair(smem_u32(&s_tmem_base), 2 * kUmmaN);
    tmem_relinquish_pair();
  }
  pdl_wait();  // below: reads of the previous kernels' outputs and writes to global memory
  if (warp == 2) {
    // per-expert m-tiles and m-tile pairs, and their exclusive prefixes (serial over experts
    // in steps of 32)
    int acc_t = 0, acc_p = 0;
    bool bad = false;
    for (int e0 = 0; e0 < N; e0 += 32) {
      const int e = e0 + lane;
      int ct = 0;
      if (e < N) {
        const int a = p.expert_offset[e], b = p.expert_offset[e + 1];
        s_off[e] = a;
        if (a < 0 || b < a || b > p.r_max || b - a > p.rows_per_expert)
          bad = true;
        else
          ct = (b - a + 127) / 128;
      }
      const int cp = (ct + 1) / 2;
      int it = ct, ip = cp;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int ut = __shfl_up_sync(0xffffffffu, it, o);
        const int up = __shfl_up_sync(0xffffffffu, ip, o);
        if (lane >= o) {
          it += ut;
          ip += up;
        }
      }
      if (e < N) {
        s_mt[e] = acc_t + it - ct;
        s_mp[e] = acc_p + ip - cp;
      }
      acc_t += __shfl_sync(0xffffffffu, it, 31);
      acc_p += __shfl_sync(0xffffffffu, ip, 31);
    }
    bad = __any_sync(0xffffffffu, bad) || acc_t > p.m_tiles_cap;
    if (lane == 0) {
      s_off[N] = p.expert_offset[N];
      s_mt[N] = acc_t;
      s_mp[N] = bad ? 0 : acc_p;  // bad offsets: no tiles
      for (int ph = 0; ph < 2; ++ph) s_tiles[ph] = s_mp[N] * p.ph[ph].n_tiles_n;
      if (bad) report_error(p.status, MOE_ERR_BOUNDS);
    }
  }
  tc_fence_before_sync();
  cluster_sync_all();  // both CTAs' barriers and TMEM exist before either uses the other's
  tc_fence_after_sync();
  const uint32_t tmem_base = s_tmem_base;
  const int h_target = p.ph[0].n_tiles_n;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer (each CTA)
    if (lane == 0) {
      const uint64_t pol_a = make_policy(2);
      const uint64_t pol_b = make_policy(p.weight_policy);
      int it = 0;
      bool ok = true;
      for (int ph = 0; ph < 2 && ok; ++ph) {
        const int bn = ph == 0 ? BN1 : kDnBn;
        const CUtensorMap* tA = ph == 0 ? &tmA1 : &tmA2;
        const int nkb = p.ph[ph].num_kb;
        for (int tile = cl; ok && tile < s_tiles[ph]; tile += ncl) {
          const PairTile c = decode_pair_tile(tile, N, bn, p.ph[ph].n_tiles_n, rank, s_mp, s_mt, s_off);
          bool ready = ph == 0 || !c.valid || ld_acquire_gpu(p.h_ready + c.gm) >= h_target;
          int pend_from = -1;
          const int it0 = it;
          for (int kb = 0; kb < nkb; ++kb) {
            const int s = it % kPairStages;
            if (!mbar_wait(smem_u32(&empty_bar[s]), ((it / kPairStages) & 1) ^ 1u, p.timeout_ns, &s_abort)) {
              ok = false;
              break;
            }
            const uint32_t fb = smem_u32(&full_bar[s]);
            const uint32_t fb0 = map_smem_to_rank(fb, 0);
            if (lead) mbar_arrive_expect_tx(fb, 2 * kPairStageBytes);
            // this CTA's half of the 256 weight rows
            if (ph == 0 && EPI1 == EPI_SWIGLU)
              tma_load_4d_pair(b_addr(s), &tmB1, fb0, kb * BK, c.n0, rank, c.e, pol_b);
            else
              tma_load_3d_pair(b_addr(s), ph == 0 ? &tmB1 : &tmB2, fb0, kb * BK, c.n0 + 128 * rank,
                               c.e, pol_b);
            if (ready) {
              tma_load_2d_pair(a_addr(s), tA, fb0, kb * BK, c.m0, pol_a);
              ++it;
              continue;
            }
            if (pend_from < 0) pend_from = it;
            if (it - pend_from + 1 == kPairStages || kb + 1 == nkb) {
              // every stage holds a W_d block (or the tile ends): wait for the rows' h
              if (!wait_counter_at_least(p.h_ready + c.gm, h_target, p.timeout_ns, &s_abort))
                ok = false;  // the h loads below still complete the armed stages
              fence_proxy_async_global();
              for (int j = pend_from; j <= it; ++j) {
                const int sj = j % kPairStages;
                tma_load_2d_pair(a_addr(sj), tA, map_smem_to_rank(smem_u32(&full_bar[sj]), 0),
                                 (j - it0) * BK, c.m0, pol_a);
              }
              pend_from = -1;
              ready = true;
            }
            ++it;
            if (!ok) break;
          }
        }
      }
      if (!ok) {
        s_abort = 1;
        report_error(p.status, MOE_ERR_TIMEOUT);
      }
      if (lead) {
        for (int i = max(0, it - kPairStages); i < it; ++i)
          mbar_wait(smem_u32(&full_bar[i % kPairStages]), (i / kPairStages) & 1, kDrainTimeoutNs, nullptr);
      } else {
        // the odd CTA's copies complete on the even CTA's barriers: wait until the MMAs have
        // released its last stages, within one overall limit
        const uint64_t t_end = globaltimer_ns() + 1000000ull;
        for (int i = max(0, it - kPairStages); i < it; ++i) {
          const uint64_t now = globaltimer_ns();
          mbar_wait(smem_u32(&empty_bar[i % kPairStages]), (i / kPairStages) & 1,
                    now < t_end ? t_end - now : 1, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (even CTA)
    if (lane == 0 && lead) {
      constexpr uint32_t idesc = idesc_bf16_f32(256, kUmmaN);
      int it = 0, tc = 0;
      bool ok = true;
      for (int ph = 0; ph < 2 && ok; ++ph) {
        const int nkb = p.ph[ph].num_kb;
        for (int tile = cl; ok && tile < s_tiles[ph]; tile += ncl, ++tc) {
          const int buf = tc & 1;
          if (!mbar_wait(smem_u32(&tempty_bar[buf]), ((tc >> 1) & 1) ^ 1u, p.timeout_ns, &s_abort)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * kUmmaN);
          for (int kb = 0; kb < nkb; ++kb, ++it) {
            const int s = it % kPairStages;
            if (!mbar_wait(smem_u32(&full_bar[s]), (it / kPairStages) & 1, p.timeout_ns, &s_abort)) {
              ok = false;
              break;
            }
            tc_fence_after_sync();
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              tc_mma_f16_pair(d_tmem, smem_desc_k_sw128(a_addr(s) + kk * 32),
                              smem_desc_k_sw128(b_addr(s) + kk * 32), idesc,
                              (kb | kk) != 0 ? 1u : 0u);
            tc_commit_pair(smem_u32(&empty_bar[s]), 0x3);
          }
          if (!ok) break;
          tc_commit_pair(smem_u32(&tfull_bar[buf]), 0x3);
        }
      }
      if (!ok) {
        s_abort = 1;
        report_error(p.status, MOE_ERR_TIMEOUT);
      }
      // always signalled, so the odd CTA's wait below ends with the MMAs
      tc_commit_pair(smem_u32(&done_bar), 0x3);
      mbar_wait(smem_u32(&done_bar), 0, kDrainTimeoutNs, nullptr);
    } else if (lane == 0) {
      mbar_wait(smem_u32(&done_bar), 0, kDrainTimeoutNs, nullptr);
    }
  } else if (warp < 6) {
    // ---------------------------------------------------------------- epilogue (warps 2..5)
    const int q = warp & 3;
    const int r_local = q * 32 + lane;
    int tc = 0;
    uint32_t epi_phase = 0;
    bool ok = true;
    for (int ph = 0; ph < 2 && ok; ++ph) {
      const int bn = ph == 0 ? BN1 : kDnBn;
      const PhaseParams& pp = p.ph[ph];
      for (int tile = cl; tile < s_tiles[ph]; tile += ncl, ++tc) {
        const PairTile c = decode_pair_tile(tile, N, bn, pp.n_tiles_n, rank, s_mp, s_mt, s_off);
        const int buf = tc & 1;
        const bool got = mbar_wait(smem_u32(&tfull_bar[buf]), (tc >> 1) & 1, p.timeout_ns, &s_abort);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                               static_cast<uint32_t>(buf * kUmmaN);
        const bool row_ok = r_local < c.rows;
        const int64_t row = static_cast<int64_t>(c.m0) + r_local;
#pragma unroll 1
        for (int cc = 0; cc < bn; cc += 16) {
          if (c.n0 + cc >= pp.n_out) break;  // warp-uniform: ragged last n-tile
          float a[16], b[16];
          uint32_t v[16];
          tmem_ld_32x32b_x16(t_row + cc, v);
          if (ph == 0 && EPI1 == EPI_SWIGLU) {
            uint32_t u[16];
            tmem_ld_32x32b_x16(t_row + BN1 + cc, u);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) b[i] = __uint_as_float(u[i]);
          } else {
            tmem_ld_wait();
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) a[i] = __uint_as_float(v[i]);
          if (!row_ok) continue;
          if (ph == 0)
            store_final16<EPI1>(pp, row, c.n0 + cc, a, b);
          else
            store_final16<EPI_STORE_F32>(pp, row, c.n0 + cc, a, b);
        }
        tc_fence_before_sync();
        // the accumulator buffer is free once both CTAs' epilogues have read it
        if (lead)
          mbar_arrive(smem_u32(&tempty_bar[buf]));
        else
          mbar_arrive_cluster(map_smem_to_rank(smem_u32(&tempty_bar[buf]), 0));
        if (ph == 0 && c.valid) {
          // this CTA wrote the tile's h: order it before TMA loads, then count it
          fence_proxy_async_global();
          if (!__all_sync(0xffffffffu, epilogue_sync(smem_u32(&epi_bar), epi_phase, p.timeout_ns, &s_abort))) {
            ok = false;
            break;
          }
          if (threadIdx.x == 64) {
            __threadfence();
            atomicAdd(p.h_ready + c.gm, 1);
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
  cluster_sync_all();  // neither CTA of a pair frees TMEM or exits while the other works
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc_pair(tmem_base, 2 * kUmmaN);
  }
  // the last CTA to finish zeroes the m-tile counters for the next call
  if (threadIdx.x == 0) {
    __threadfence();
    s_last_cta = atomicAdd(p.done_ctas, 1) == static_cast<int>(gridDim.x) - 1;
  }
  __syncthreads();
  if (s_last_cta) {
    __threadfence();
    for (int i = threadIdx.x; i < s_mt[N]; i += kThreads) p.h_ready[i] = 0;
    if (threadIdx.x == 0) *p.done_ctas = 0;
  }
}

// Block-scaled formats: the token rows x_perm as MXFP8 (the A operand of the gate/up GEMM).
// Slot (gm, r) is row r of m-tile gm (the tiles of the grouped FFN: experts in order, 128
// rows each, the last one of an expert partial). A valid row's 32-column blocks become E4M3
// codes in xq [r_max, d] (bytes) and their scales go to the tile's atoms; rows past the
// expert's end and blocks past d get scale code 0 (2^-127). The h atoms (filled by the
// gate/up epilogue for valid rows) are zeroed first.
__global__ void __launch_bounds__(256) quantize_rows_kernel(const uint16_t* __restrict__ x,
                                                            const int32_t* __restrict__ expert_offset,
                                                            int N, int d, int num_kb, int64_t r_max,
                                                            int m_tiles_cap, uint8_t* __restrict__ xq,
                                                            uint8_t* __restrict__ x_atoms,
                                                            uint8_t* __restrict__ h_atoms,
                                                            int64_t h_atom_bytes, int* status) {
  __shared__ int s_mt[257], s_off[257];
  pdl_trigger();
  pdl_wait();
  const int tid = threadIdx.x, lane = tid & 31;
  // zero the h atoms (16-byte stores; the region is a multiple of 512 bytes)
  for (int64_t i = blockIdx.x * 256ll + tid; i < h_atom_bytes / 16; i += static_cast<int64_t>(gridDim.x) * 256)
    reinterpret_cast<uint4*>(h_atoms)[i] = make_uint4(0u, 0u, 0u, 0u);
  // per-expert m-tiles (one warp, serial over the <= 256 experts: tiny)
  if (tid < 32) {
    int acc = 0;
    bool bad = false;
    for (int e0 = 0; e0 < N; e0 += 32) {
      const int e = e0 + lane;
      int cnt = 0;
      if (e < N) {
        const int a = expert_offset[e], b = expert_offset[e + 1];
        s_off[e] = a;
        if (a < 0 || b < a || b > r_max) bad = true;
        else cnt = (b - a + 127) / 128;
      }
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      if (e < N) s_mt[e] = acc + incl - cnt;
      acc += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      s_off[N] = expert_offset[N];
      s_mt[N] = acc;
    }
    if (__any_sync(0xffffffffu, bad) || acc > m_tiles_cap) {
      if (lane == 0) {
        s_mt[N] = 0;  // no tiles: the grouped FFN reports the same offsets
        if (blockIdx.x == 0) report_error(status, MOE_ERR_BOUNDS);
      }
    }
  }
  __syncthreads();
  const int warp_g = blockIdx.x * 8 + (tid >> 5), warps = gridDim.x * 8;
  const int64_t slots = static_cast<int64_t>(s_mt[N]) * 128;
  for (int64_t sl = warp_g; sl < slots; sl += warps) {
    const int gm = static_cast<int>(sl >> 7), r = static_cast<int>(sl & 127);
    int lo = 0, hi = N - 1;  // expert of m-tile gm: the largest e with s_mt[e] <= gm
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_mt[mid] <= gm) lo = mid; else hi = mid - 1;
    }
    const int64_t row = s_off[lo] + static_cast<int64_t>(gm - s_mt[lo]) * 128 + r;
    const bool valid = row < s_off[lo + 1] && row < r_max;
    for (int q = lane; q < num_kb * 4; q += 32) {
      uint32_t sc = 0;
      if (valid && q * 32 < d) {
        const uint4* src = reinterpret_cast<const uint4*>(x + row * d + q * 32);
        float v[32];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint4 w = __ldg(src + j);
          const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            v[8 * j + 2 * t] = __uint_as_float(ww[t] << 16);
            v[8 * j + 2 * t + 1] = __uint_as_float(ww[t] & 0xffff0000u);
          }
        }
        uint4 lo4, hi4;
        sc = mxfp8_block(v, lo4, hi4);
        uint4* dst = reinterpret_cast<uint4*>(xq + row * d + q * 32);
        dst[0] = lo4;
        dst[1] = hi4;
      }
      x_atoms[(static_cast<int64_t>(gm) * num_kb + q / 4) * 512 + sf_atom_byte(r, q & 3)] =
          static_cast<uint8_t>(sc);
    }
  }
}

// ------------------------------------------------------------------ host side
template <int EPI1, int BN1>
cudaError_t launch_pair(const CUtensorMap& a1, const CUtensorMap& b1, const CUtensorMap& a2,
                        const CUtensorMap& b2, const FfnParams& fp, int grid, cudaStream_t s) {
  static PerDeviceOnce once;
  const cudaError_t attr_err = once.run([] {
    return cudaFuncSetAttribute(grouped_ffn_pair_kernel<EPI1, BN1>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, kPairSmemBytes);
  });
  if (attr_err != cudaSuccess) return attr_err;
  return launch_pdl_cluster(grouped_ffn_pair_kernel<EPI1, BN1>, dim3(grid), dim3(kThreads),
                            kPairSmemBytes, s, 2u, a1, b1, a2, b2, fp);
}

template <int EPI1, int BN1, int BM, int WFMT>
cudaError_t launch_one(const CUtensorMap& a1, const CUtensorMap& b1, const CUtensorMap& a2,
                       const CUtensorMap& b2, const CUtensorMap& s1, const CUtensorMap& s2,
                       const CUtensorMap& a1s, const CUtensorMap& a2s,
                       const FfnParams& fp, int grid, cudaStream_t s) {
  using C = Cfg<BM, WFMT>;
  static PerDeviceOnce once;
  const cudaError_t attr_err = once.run([] {
    return cudaFuncSetAttribute(grouped_ffn_kernel<EPI1, BN1, BM, WFMT>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  });
  if (attr_err != cudaSuccess) return attr_err;
  // down tiles wait for other CTAs' h counters: every CTA of the grid must be resident at once
  int per_sm = 0;
  const cudaError_t occ = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
      &per_sm, grouped_ffn_kernel<EPI1, BN1, BM, WFMT>, C::THREADS, C::SMEM_BYTES);
  if (occ != cudaSuccess) return occ;
  DeviceInfo di;
  const cudaError_t de = device_info(&di);
  if (de != cudaSuccess) return de;
  if (static_cast<int64_t>(per_sm) * di.sm_count < grid) return cudaErrorInvalidConfiguration;
  return launch_pdl(grouped_ffn_kernel<EPI1, BN1, BM, WFMT>, dim3(grid), dim3(C::THREADS),
                    C::SMEM_BYTES, s, a1, b1, a2, b2, s1, s2, a1s, a2s, fp);
}

template <int WFMT>
cudaError_t launch_fmt(bool swiglu, int bm, const CUtensorMap& a1, const CUtensorMap& b1,
                       const CUtensorMap& a2, const CUtensorMap& b2, const CUtensorMap& s1,
                       const CUtensorMap& s2, const CUtensorMap& a1s, const CUtensorMap& a2s,
                       const FfnParams& fp, int grid, cudaStream_t s);

// sum_e ceil(m_e / bm) <= ceil(R / bm) + (experts with rows)
int64_t m_tiles_upper_bound(int64_t r_max, int N, int bm) {
  return (r_max + bm - 1) / bm + std::min<int64_t>(N, r_max);
}

constexpr int kSkMaxCtas = 148;  // CTAs that hold stream-K partial slots (one per B200 SM)
// Stream-K only while a partial tile is at most this many rows: the last CTA of a tile adds the
// partials through L2 at latency-bound speed, which costs more than a last, partly filled wave
// of whole tiles once partial tiles reach 64 rows (measured on B200).
constexpr int kSkMaxSlotRows = 32;

// CTAs that can have work: whole tiles, or stream-K ranges of at least kSkMinKb k blocks.
int64_t useful_ctas(int64_t tiles_ub, int num_kb, int sk_ctas) {
  const int64_t sk = tiles_ub * num_kb / std::min(kSkMinKb, num_kb);
  return std::max<int64_t>(tiles_ub, std::min<int64_t>(sk_ctas, sk));
}

constexpr int kGuBnSwiglu = 128;  // output columns per tile of the gate/up GEMM (UMMA N = 256)
constexpr int kGuBnGelu = 256;

}  // namespace

FfnScratchPlan ffn_scratch_plan(int N, int d, int F, int act, int64_t r_max,
                                int64_t rows_per_expert, bool block_scaled) {
  FfnScratchPlan pl{};
  pl.bm = 128;
  if (r_max <= 0) return pl;
  pl.bm = (rows_per_expert <= 64 && !block_scaled) ? 64 : 128;
  const int kbe = block_scaled ? kBsK : BK;  // k per block
  const int nkb1 = (d + kbe - 1) / kbe, nkb2 = (F + kbe - 1) / kbe;
  pl.slot_rows = static_cast<int>(std::min<int64_t>(pl.bm, std::max<int64_t>(1, rows_per_expert)));
  const int bn1 = act == MOE_ACT_SWIGLU ? kGuBnSwiglu : kGuBnGelu;
  pl.m_tiles_ub = m_tiles_upper_bound(r_max, N, pl.bm);
  pl.tiles1_ub = pl.m_tiles_ub * ((F + bn1 - 1) / bn1);
  pl.tiles2_ub = pl.m_tiles_ub * ((d + kDnBn - 1) / kDnBn);
  if (pl.slot_rows <= kSkMaxSlotRows) {
    const int64_t by1 = pl.tiles1_ub * nkb1 / std::min(kSkMinKb, nkb1);
    const int64_t by2 = pl.tiles2_ub * nkb2 / std::min(kSkMinKb, nkb2);
    pl.sk_ctas1 = static_cast<int>(std::min<int64_t>(kSkMaxCtas, by1));
    pl.sk_ctas2 = static_cast<int>(std::min<int64_t>(kSkMaxCtas, by2));
  }
  const int64_t ints = pl.m_tiles_ub + 1 + (pl.sk_ctas1 > 0 ? pl.tiles1_ub : 0) +
                       (pl.sk_ctas2 > 0 ? pl.tiles2_ub : 0);
  pl.counter_bytes = static_cast<size_t>(ints) * sizeof(int);
  pl.part_bytes = static_cast<size_t>(pl.sk_ctas1 + pl.sk_ctas2) * 2 * pl.slot_rows * kUmmaN *
                  sizeof(float);
  return pl;
}

MxActLayout mx_act_layout(int N, int d, int F, int64_t r_max) {
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  MxActLayout l{};
  const int64_t mt = r_max > 0 ? m_tiles_upper_bound(r_max, N, 128) : 0;
  l.xq_bytes = up(static_cast<size_t>(std::max<int64_t>(r_max, 0)) * d);
  l.x_atom_bytes = up(static_cast<size_t>(mt) * ((d + kBsK - 1) / kBsK) * 512);
  l.h_atom_bytes = up(static_cast<size_t>(mt) * ((F + kBsK - 1) / kBsK) * 512);
  l.total = l.xq_bytes + l.x_atom_bytes + l.h_atom_bytes;
  return l;
}

cudaError_t launch_grouped_ffn(const GroupedFfnArgs& a, cudaStream_t s) {
  if (a.r_max <= 0) return cudaSuccess;
  if (a.counters == nullptr) return cudaErrorInvalidValue;
  DeviceInfo di;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;

  const uint64_t d = static_cast<uint64_t>(a.d), F = static_cast<uint64_t>(a.F);
  const uint64_t N = static_cast<uint64_t>(a.N), R = static_cast<uint64_t>(a.r_max);
  const bool swiglu = a.act == MOE_ACT_SWIGLU;
  const int bn_gu = swiglu ? kGuBnSwiglu : kGuBnGelu;
  const bool bs = a.wfmt == MOE_WFMT_MXFP8_BS || a.wfmt == MOE_WFMT_MXFP4_BS;
  const FfnScratchPlan plan =
      ffn_scratch_plan(a.N, a.d, a.F, a.act, a.r_max, a.rows_per_expert, bs);
  if (bs) {  // the workspace regions were sized by the default plan
    const FfnScratchPlan std_plan = ffn_scratch_plan(a.N, a.d, a.F, a.act, a.r_max, a.rows_per_expert);
    if (plan.counter_bytes > std_plan.counter_bytes || plan.part_bytes > std_plan.part_bytes ||
        a.act_ws == nullptr)
      return cudaErrorInvalidValue;
  }
  const int bm = plan.bm;
  // weights are read once per m-tile; when every expert has at most one m-tile (decode-sized
  // batches) they are pure streams and should not displace the activations in L2
  const int wpol = (a.rows_per_expert <= bm) ? 1 : 0;

  CUtensorMap mA1, mB1, mA2, mB2, mS1, mS2, mA1s, mA2s;
  memset(&mS1, 0, sizeof(mS1));  // bf16 weights: the scale maps are not read
  memset(&mS2, 0, sizeof(mS2));
  memset(&mA1s, 0, sizeof(mA1s));  // only the block-scaled formats read the 32-row maps
  memset(&mA2s, 0, sizeof(mA2s));
  const MxActLayout al = mx_act_layout(a.N, a.d, a.F, a.r_max);
  uint8_t* const xq = static_cast<uint8_t*>(a.act_ws);
  uint8_t* const x_atoms = bs ? xq + al.xq_bytes : nullptr;
  uint8_t* const h_atoms = bs ? x_atoms + al.x_atom_bytes : nullptr;
  if (bs) {
    // A: the quantised rows and h as bytes [R][K], 128-byte boxes of 128 rows (128B swizzle)
    {
      const uint64_t dims[2] = {d, R};
      const uint64_t str[1] = {d};
      const uint32_t box[2] = {128, 128};
      if (!make_map_u8(&mA1, xq, 2, dims, str, box, true)) return cudaErrorInvalidValue;
      const uint32_t box_s[2] = {128, static_cast<uint32_t>(kBsSmallRows)};
      if (!make_map_u8(&mA1s, xq, 2, dims, str, box_s, true)) return cudaErrorInvalidValue;
    }
    {
      const uint64_t dims[2] = {F, R};
      const uint64_t str[1] = {F};
      const uint32_t box[2] = {128, 128};
      if (!make_map_u8(&mA2, a.h, 2, dims, str, box, true)) return cudaErrorInvalidValue;
      const uint32_t box_s[2] = {128, static_cast<uint32_t>(kBsSmallRows)};
      if (!make_map_u8(&mA2s, a.h, 2, dims, str, box_s, true)) return cudaErrorInvalidValue;
    }
    // B: the MX elements, one k block (128 elements) of 128 or 256 rows a box; E4M3 as bytes,
    // E2M1 through the padded 4-bit type (k a multiple of 128). Scales: boxes of 4 blocks x
    // 128 rows from [N][K/32][rows].
    const bool fp4 = a.wfmt == MOE_WFMT_MXFP4_BS;
    if (fp4 && (d % 128 != 0 || F % 128 != 0)) return cudaErrorInvalidValue;
    const uint64_t db = fp4 ? d / 2 : d, fb = fp4 ? F / 2 : F;  // bytes per row
    auto emap = [&](CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
                    const uint64_t* str, const uint32_t* box) {
      return fp4 ? make_map_fp4_padded(m, base, rank, dims, str, box)
                 : make_map_u8(m, base, rank, dims, str, box, true);
    };
    if (swiglu) {
      const uint64_t dims[4] = {d, F, 2, N};
      const uint64_t str[3] = {db, F * db, 2 * F * db};
      const uint32_t box[4] = {128, 128, 1, 1};
      if (!emap(&mB1, a.w_gate_up, 4, dims, str, box)) return cudaErrorInvalidValue;
      const uint64_t sd[4] = {F, 2, d / 32, N};
      const uint64_t ss[3] = {F, 2 * F, (d / 32) * 2 * F};
      const uint32_t sb[4] = {128, 1, 4, 1};
      if (!make_map_u8(&mS1, a.w_gate_up_scales, 4, sd, ss, sb, false)) return cudaErrorInvalidValue;
    } else {
      const uint64_t dims[3] = {d, F, N};
      const uint64_t str[2] = {db, F * db};
      const uint32_t box[3] = {128, 256, 1};
      if (!emap(&mB1, a.w_gate_up, 3, dims, str, box)) return cudaErrorInvalidValue;
      const uint64_t sd[3] = {F, d / 32, N};
      const uint64_t ss[2] = {F, (d / 32) * F};
      const uint32_t sb[3] = {128, 4, 1};
      if (!make_map_u8(&mS1, a.w_gate_up_scales, 3, sd, ss, sb, false)) return cudaErrorInvalidValue;
    }
    {
      const uint64_t dims[3] = {F, d, N};
      const uint64_t str[2] = {fb, d * fb};
      const uint32_t box[3] = {128, 256, 1};
      if (!emap(&mB2, a.w_down, 3, dims, str, box)) return cudaErrorInvalidValue;
      const uint64_t sd[3] = {d, F / 32, N};
      const uint64_t ss[2] = {d, (F / 32) * d};
      const uint32_t sb[3] = {128, 4, 1};
      if (!make_map_u8(&mS2, a.w_down_scales, 3, sd, ss, sb, false)) return cudaErrorInvalidValue;
    }
  } else {
  {
    const uint64_t dims[2] = {d, R};
    const uint64_t str[1] = {d * 2};
    const uint32_t box[2] = {BK, static_cast<uint32_t>(bm)};
    if (!make_map(&mA1, a.x_perm, 2, dims, str, box)) return cudaErrorInvalidValue;
  }
  if (a.wfmt != MOE_WFMT_BF16) {
    // packed elements: [N][rows][K * rb / 64] bytes, 128-byte boxes (2 or 4 k blocks) with
    // 128B swizzle; scales: [N][K/32][rows] bytes, boxes of 2 KG blocks
    const uint64_t rb = a.wfmt == MOE_WFMT_MXFP8 ? BK : BK / 2;  // bytes per row and k block
    const uint32_t kg2 = static_cast<uint32_t>(2 * (128 / rb));    // scale blocks per box
    const uint64_t db = d * rb / BK, fb = F * rb / BK;
    if (swiglu) {
      const uint64_t dims[4] = {db, F, 2, N};
      const uint64_t str[3] = {db, F * db, 2 * F * db};
      const uint32_t box[4] = {128, static_cast<uint32_t>(bn_gu), 1, 1};
      if (!make_map_u8(&mB1, a.w_gate_up, 4, dims, str, box, true)) return cudaErrorInvalidValue;
      const uint64_t sd[4] = {F, 2, d / 32, N};
      const uint64_t ss[3] = {F, 2 * F, (d / 32) * 2 * F};
      const uint32_t sb[4] = {static_cast<uint32_t>(bn_gu), 1, kg2, 1};
      if (!make_map_u8(&mS1, a.w_gate_up_scales, 4, sd, ss, sb, false)) return cudaErrorInvalidValue;
    } else {
      const uint64_t dims[3] = {db, F, N};
      const uint64_t str[2] = {db, F * db};
      const uint32_t box[3] = {128, static_cast<uint32_t>(bn_gu), 1};
      if (!make_map_u8(&mB1, a.w_gate_up, 3, dims, str, box, true)) return cudaErrorInvalidValue;
      const uint64_t sd[3] = {F, d / 32, N};
      const uint64_t ss[2] = {F, (d / 32) * F};
      const uint32_t sb[3] = {static_cast<uint32_t>(bn_gu), kg2, 1};
      if (!make_map_u8(&mS1, a.w_gate_up_scales, 3, sd, ss, sb, false)) return cudaErrorInvalidValue;
    }
    {
      const uint64_t dims[3] = {fb, d, N};
      const uint64_t str[2] = {fb, d * fb};
      const uint32_t box[3] = {128, static_cast<uint32_t>(kDnBn), 1};
      if (!make_map_u8(&mB2, a.w_down, 3, dims, str, box, true)) return cudaErrorInvalidValue;
      const uint64_t sd[3] = {d, F / 32, N};
      const uint64_t ss[2] = {d, (F / 32) * d};
      const uint32_t sb[3] = {static_cast<uint32_t>(kDnBn), kg2, 1};
      if (!make_map_u8(&mS2, a.w_down_scales, 3, sd, ss, sb, false)) return cudaErrorInvalidValue;
    }
  } else if (swiglu) {
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
  if (a.wfmt == MOE_WFMT_BF16) {
    const uint64_t dims[3] = {F, d, N};
    const uint64_t str[2] = {F * 2, d * F * 2};
    const uint32_t box[3] = {BK, static_cast<uint32_t>(kDnBn), 1};
    if (!make_map(&mB2, a.w_down, 3, dims, str, box)) return cudaErrorInvalidValue;
  }
  }  // not block-scaled

  // CTA pairs for bf16 weights when the experts average at least eight 128-row m-tiles (the
  // tensor-bound regime): whole tiles, weight boxes of 128 rows. An expert's odd last m-tile
  // costs a whole pair tile, which at four m-tiles per expert outweighs the gain.
  const bool pair = a.wfmt == MOE_WFMT_BF16 && bm == 128 && a.r_max >= 1024LL * a.N;
  if (pair) {
    if (!swiglu) {
      const uint64_t dims[3] = {d, F, N};
      const uint64_t str[2] = {d * 2, F * d * 2};
      const uint32_t box[3] = {BK, 128, 1};
      if (!make_map(&mB1, a.w_gate_up, 3, dims, str, box)) return cudaErrorInvalidValue;
    }
    const uint64_t dims[3] = {F, d, N};
    const uint64_t str[2] = {F * 2, d * F * 2};
    const uint32_t box[3] = {BK, 128, 1};
    if (!make_map(&mB2, a.w_down, 3, dims, str, box)) return cudaErrorInvalidValue;
  }
  const bool stream_k = a.part != nullptr && !pair;
  FfnParams fp{};
  fp.expert_offset = a.expert_offset;
  fp.r_max = a.r_max;
  fp.rows_per_expert = a.rows_per_expert;
  fp.n_experts = a.N;
  fp.slot_rows = plan.slot_rows;
  int* cnt = a.counters;
  fp.h_ready = cnt;
  fp.m_tiles_cap = static_cast<int>(plan.m_tiles_ub);
  cnt += plan.m_tiles_ub;
  fp.done_ctas = cnt;
  cnt += 1;
  fp.status = a.status;
  fp.timeout_ns = a.timeout_ns;
  fp.weight_policy = wpol;
  fp.x_atoms = x_atoms;
  fp.h_atoms = h_atoms;

  PhaseParams& p1 = fp.ph[0];
  p1.out = a.h;
  p1.ld_out = a.F;
  p1.n_out = a.F;
  p1.n_tiles_n = (a.F + bn_gu - 1) / bn_gu;
  p1.num_kb = bs ? (a.d + kBsK - 1) / kBsK : a.d / BK;
  p1.sk_ctas = stream_k ? plan.sk_ctas1 : 0;
  p1.part = a.part;
  p1.tile_counters = cnt;
  if (plan.sk_ctas1 > 0) cnt += plan.tiles1_ub;

  PhaseParams& p2 = fp.ph[1];
  p2.out = a.y_perm;
  p2.ld_out = a.d;
  p2.n_out = a.d;
  p2.n_tiles_n = (a.d + kDnBn - 1) / kDnBn;
  p2.num_kb = bs ? (a.F + kBsK - 1) / kBsK : a.F / BK;
  p2.sk_ctas = stream_k ? plan.sk_ctas2 : 0;
  p2.part = stream_k ? a.part + static_cast<size_t>(plan.sk_ctas1) * 2 * plan.slot_rows * kUmmaN
                     : nullptr;
  p2.tile_counters = cnt;

  const int64_t useful = std::max(useful_ctas(plan.tiles1_ub, p1.num_kb, p1.sk_ctas),
                                  useful_ctas(plan.tiles2_ub, p2.num_kb, p2.sk_ctas));
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(useful, di.sm_count)));
  if (pair) {
    const int pgrid = 2 * std::max(1, std::min(di.sm_count / 2, static_cast<int>((useful + 1) / 2)));
    return swiglu ? launch_pair<EPI_SWIGLU, kGuBnSwiglu>(mA1, mB1, mA2, mB2, fp, pgrid, s)
                  : launch_pair<EPI_GELU, kGuBnGelu>(mA1, mB1, mA2, mB2, fp, pgrid, s);
  }
  if (bs) {
    const int qgrid = static_cast<int>(std::min<int64_t>(
        std::max<int64_t>(1, (plan.m_tiles_ub * 128 + 7) / 8), static_cast<int64_t>(di.sm_count) * 8));
    cudaError_t qe = launch_pdl(quantize_rows_kernel, dim3(qgrid), dim3(256), 0, s, a.x_perm,
                                a.expert_offset, a.N, a.d, p1.num_kb, a.r_max,
                                static_cast<int>(plan.m_tiles_ub), xq, x_atoms, h_atoms,
                                static_cast<int64_t>(al.h_atom_bytes), a.status);
    if (qe != cudaSuccess) return qe;
    if (a.wfmt == MOE_WFMT_MXFP8_BS)
      return launch_fmt<WFMT_BS8>(swiglu, 128, mA1, mB1, mA2, mB2, mS1, mS2, mA1s, mA2s, fp, grid, s);
    return launch_fmt<WFMT_BS4>(swiglu, 128, mA1, mB1, mA2, mB2, mS1, mS2, mA1s, mA2s, fp, grid, s);
  }
  if (a.wfmt == MOE_WFMT_MXFP8)
    return launch_fmt<WFMT_MXFP8>(swiglu, bm, mA1, mB1, mA2, mB2, mS1, mS2, mA1s, mA2s, fp, grid, s);
  if (a.wfmt == MOE_WFMT_MXFP4)
    return launch_fmt<WFMT_MXFP4>(swiglu, bm, mA1, mB1, mA2, mB2, mS1, mS2, mA1s, mA2s, fp, grid, s);
  return launch_fmt<WFMT_BF16>(swiglu, bm, mA1, mB1, mA2, mB2, mS1, mS2, mA1s, mA2s, fp, grid, s);
}

namespace {
template <int WFMT>
cudaError_t launch_fmt(bool swiglu, int bm, const CUtensorMap& a1, const CUtensorMap& b1,
                       const CUtensorMap& a2, const CUtensorMap& b2, const CUtensorMap& s1,
                       const CUtensorMap& s2, const CUtensorMap& a1s, const CUtensorMap& a2s,
                       const FfnParams& fp, int grid, cudaStream_t s) {
  if constexpr (WFMT == WFMT_BS8 || WFMT == WFMT_BS4) {  // 128-row tiles only
    return swiglu ? launch_one<EPI_SWIGLU, kGuBnSwiglu, 128, WFMT>(a1, b1, a2, b2, s1, s2, a1s, a2s, fp, grid, s)
                  : launch_one<EPI_GELU, kGuBnGelu, 128, WFMT>(a1, b1, a2, b2, s1, s2, a1s, a2s, fp, grid, s);
  } else {
    if (bm == 64)
      return swiglu ? launch_one<EPI_SWIGLU, kGuBnSwiglu, 64, WFMT>(a1, b1, a2, b2, s1, s2, a1s, a2s, fp, grid, s)
                    : launch_one<EPI_GELU, kGuBnGelu, 64, WFMT>(a1, b1, a2, b2, s1, s2, a1s, a2s, fp, grid, s);
  }
  return swiglu ? launch_one<EPI_SWIGLU, kGuBnSwiglu, 128, WFMT>(a1, b1, a2, b2, s1, s2, a1s, a2s, fp, grid, s)
                : launch_one<EPI_GELU, kGuBnGelu, 128, WFMT>(a1, b1, a2, b2, s1, s2, a1s, a2s, fp, grid, s);
}
}  // namespace

}  // namespace moe
