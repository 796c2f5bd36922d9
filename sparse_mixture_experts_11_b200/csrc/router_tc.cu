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
// One CTA per 128-token tile, 256 threads:
//   warp 0      TMA producer of the x tile [128 tokens x 64 k] (128B swizzle) into a ring;
//   warp 1      TMEM owner and MMA issuer: per k block 3 x 4 MMAs (M=128, N=NP, K=16) into one
//               fp32 accumulator of NP columns;
//   warps 4-7   split converters during the main loop: read W_r[:, k block] in fp32, write
//               hi/mid/lo as K-major 128B-swizzled bf16 tiles (double buffered); then the
//               epilogue: thread i owns token i's row of logits in TMEM, adds the bias,
//               writes the logits, keeps a running top-k and writes indices and weights.
// All mbarrier waits are bounded. A timeout records MOE_ERR_TIMEOUT, stops the CTA's work,
// drains its own copies and MMAs, and frees TMEM.
#include <math.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace moe {
namespace {

constexpr int kTok = 128;  // tokens per CTA (UMMA M)
constexpr int kBK = 64;    // k per block (one 128-byte swizzle row of bf16)
constexpr int kThreads = 256;
constexpr int kConvThreads = 128;
constexpr int kSmemLimit = 225 * 1024;

template <int NP>
struct RCfg {
  static constexpr int A_BYTES = kTok * kBK * 2;           // 16 KB per x stage
  static constexpr int WT_BYTES = NP * kBK * 2;            // one split term tile
  static constexpr int WBUF_BYTES = 3 * WT_BYTES;          // hi, mid, lo
  static constexpr int A_STAGES_FIT = (kSmemLimit - 1024 - 2 * WBUF_BYTES) / A_BYTES;
  static constexpr int A_STAGES = A_STAGES_FIT > 8 ? 8 : A_STAGES_FIT;
  static constexpr int TMEM_COLS = NP < 32 ? 32 : NP;
  static constexpr int SMEM_BYTES = 2 * WBUF_BYTES + A_STAGES * A_BYTES + 1024;
  static_assert(A_STAGES >= 2, "router pipeline depth");
  static_assert(NP % 16 == 0 && NP >= 16 && NP <= 256, "UMMA N for M = 128");
};

__device__ __forceinline__ bool better(float av, int ae, float bv, int be) {
  return av > bv || (av == bv && ae < be);
}

// The 128-byte swizzle: 16-byte chunk c of row n sits at chunk position c ^ (n & 7).
__device__ __forceinline__ uint32_t sw128_offset(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

template <int NP>
__global__ void __launch_bounds__(kThreads, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const float* __restrict__ w,
                     const float* __restrict__ bias, float* __restrict__ logits,
                     int32_t* __restrict__ topk_idx, float* __restrict__ topk_w, int T, int d,
                     int N, int k, int* status, uint64_t timeout_ns) {
  using C = RCfg<NP>;
  extern __shared__ __align__(1024) uint8_t dyn_smem[];
  __shared__ __align__(8) uint64_t a_full[C::A_STAGES];
  __shared__ __align__(8) uint64_t a_empty[C::A_STAGES];
  __shared__ __align__(8) uint64_t w_full[2];
  __shared__ __align__(8) uint64_t w_empty[2];
  __shared__ __align__(8) uint64_t acc_full;
  __shared__ __align__(8) uint64_t done_bar;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t base = (smem_u32(dyn_smem) + 1023u) & ~1023u;
  uint8_t* gbase = dyn_smem + (base - smem_u32(dyn_smem));  // generic pointer of `base`
  const uint32_t wbuf0 = base;                               // 2 x [3][NP][64] bf16
  const uint32_t abuf0 = base + 2 * C::WBUF_BYTES;           // A_STAGES x [128][64] bf16
  const int t0 = blockIdx.x * kTok;
  const int num_kb = d / kBK;

  if (threadIdx.x == 0) {
    prefetch_tensormap(&tmX);
    for (int s = 0; s < C::A_STAGES; ++s) {
      mbar_init(smem_u32(&a_full[s]), 1);
      mbar_init(smem_u32(&a_empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&w_full[b]), kConvThreads);
      mbar_init(smem_u32(&w_empty[b]), 1);
    }
    mbar_init(smem_u32(&acc_full), 1);
    mbar_init(smem_u32(&done_bar), 1);
    s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    __syncwarp();
    tmem_alloc(smem_u32(&s_tmem), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp >= 4 && NP > N) {
    // rows N..NP-1 of both split buffers stay zero for the whole kernel
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
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = s_tmem;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      int kb = 0;
      bool ok = true;
      for (; kb < num_kb; ++kb) {
        const int s = kb % C::A_STAGES;
        if (!mbar_wait(smem_u32(&a_empty[s]), ((kb / C::A_STAGES) & 1) ^ 1u, timeout_ns, &s_abort)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(smem_u32(&a_full[s]), C::A_BYTES);
        tma_load_2d(abuf0 + s * C::A_BYTES, &tmX, smem_u32(&a_full[s]), kb * kBK, t0, pol);
      }
      if (!ok) {
        s_abort = 1;
        report_error(status, MOE_ERR_TIMEOUT);
      }
      for (int i = max(0, kb - C::A_STAGES); i < kb; ++i)
        mbar_wait(smem_u32(&a_full[i % C::A_STAGES]), (i / C::A_STAGES) & 1, timeout_ns, nullptr);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kTok, NP);
      bool ok = true, issued = false;
      for (int kb = 0; kb < num_kb; ++kb) {
        const int s = kb % C::A_STAGES, b = kb & 1;
        if (!mbar_wait(smem_u32(&a_full[s]), (kb / C::A_STAGES) & 1, timeout_ns, &s_abort) ||
            !mbar_wait(smem_u32(&w_full[b]), (kb >> 1) & 1, timeout_ns, &s_abort)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t a = abuf0 + s * C::A_BYTES;
#pragma unroll
        for (int term = 0; term < 3; ++term) {
          const uint32_t bt = wbuf0 + b * C::WBUF_BYTES + term * C::WT_BYTES;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            tc_mma_f16(tmem, smem_desc_k_sw128(a + kk * 32), smem_desc_k_sw128(bt + kk * 32), idesc,
                       (kb | term | kk) != 0 ? 1u : 0u);
        }
        issued = true;
        tc_commit(smem_u32(&a_empty[s]));
        tc_commit(smem_u32(&w_empty[b]));
      }
      if (ok) {
        tc_commit(smem_u32(&acc_full));
      } else {
        s_abort = 1;
        report_error(status, MOE_ERR_TIMEOUT);
        if (issued) {
          tc_commit(smem_u32(&done_bar));
          mbar_wait(smem_u32(&done_bar), 0, timeout_ns, nullptr);
        }
      }
    }
  } else if (warp >= 4) {
    const int ct = threadIdx.x - 128;  // 0..127
    bool ok = true;
    // ---- main loop: split W_r[:, k block] into three bf16 terms, K-major swizzled tiles
    for (int kb = 0; kb < num_kb; ++kb) {
      const int b = kb & 1;
      const bool got = mbar_wait(smem_u32(&w_empty[b]), ((kb >> 1) & 1) ^ 1u, timeout_ns, &s_abort);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      uint8_t* buf = gbase + b * C::WBUF_BYTES;
      for (int task = ct; task < N * 8; task += kConvThreads) {
        const int row = task >> 3, chunk = task & 7;
        const float4* src = reinterpret_cast<const float4*>(w + static_cast<int64_t>(row) * d + kb * kBK + chunk * 8);
        const float4 v0 = __ldg(src), v1 = __ldg(src + 1);
        const float f[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        uint32_t hi[4], mid[4], lo[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float r0 = f[2 * q], r1 = f[2 * q + 1];
          const __nv_bfloat162 h = __floats2bfloat162_rn(r0, r1);
          r0 -= __low2float(h);
          r1 -= __high2float(h);
          const __nv_bfloat162 m = __floats2bfloat162_rn(r0, r1);
          r0 -= __low2float(m);
          r1 -= __high2float(m);
          const __nv_bfloat162 l = __floats2bfloat162_rn(r0, r1);
          hi[q] = *reinterpret_cast<const uint32_t*>(&h);
          mid[q] = *reinterpret_cast<const uint32_t*>(&m);
          lo[q] = *reinterpret_cast<const uint32_t*>(&l);
        }
        const uint32_t off = sw128_offset(row, chunk);
        *reinterpret_cast<uint4*>(buf + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(buf + C::WT_BYTES + off) = make_uint4(mid[0], mid[1], mid[2], mid[3]);
        *reinterpret_cast<uint4*>(buf + 2 * C::WT_BYTES + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
      fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core
      mbar_arrive(smem_u32(&w_full[b]));
    }
    // ---- epilogue: thread ct owns token t0 + ct
    if (ok) {
      const bool got = mbar_wait(smem_u32(&acc_full), 0, timeout_ns, &s_abort);
      ok = __all_sync(0xffffffffu, got);
    }
    if (ok) {
      tc_fence_after_sync();
      const int q = warp & 3;
      const int t = t0 + ct;
      const bool valid = t < T;
      const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16);
      float best_v[8];
      int best_e[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        best_v[r] = -INFINITY;
        best_e[r] = 0x7fffffff;
      }
      // the best 8 are kept whatever k is (entry 7 is the admission threshold); the first k
      // are written
      float thr_v = -INFINITY;
      int thr_e = 0x7fffffff;
      for (int c0 = 0; c0 < N; c0 += 16) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(trow + c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int e = c0 + i;
          if (e >= N) continue;
          float L = __uint_as_float(v[i]);
          if (bias != nullptr) L += __ldg(bias + e);
          if (valid) logits[static_cast<int64_t>(t) * N + e] = L;
          const float key = isnan(L) ? -INFINITY : L;
          // insert (key, e) into the sorted list best[0..7]
          if (better(key, e, thr_v, thr_e)) {
            // shift the entries the candidate beats down by one and drop it into place;
            // from the last slot up, so best[r - 1] is still the old value when read
#pragma unroll
            for (int r = 7; r >= 0; --r) {
              if (better(key, e, best_v[r], best_e[r])) {
                const bool above = (r == 0) || better(key, e, best_v[r > 0 ? r - 1 : 0], best_e[r > 0 ? r - 1 : 0]);
                best_v[r] = above ? key : best_v[r > 0 ? r - 1 : 0];
                best_e[r] = above ? e : best_e[r > 0 ? r - 1 : 0];
              }
            }
            thr_v = best_v[7];
            thr_e = best_e[7];
          }
        }
      }
      if (valid) {
        float num[8], den = 0.f;
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          num[r] = (r < k) ? expf(best_v[r] - best_v[0]) : 0.f;
          den += num[r];
        }
#pragma unroll
        for (int r = 0; r < 8; ++r)
          if (r < k) {
            topk_idx[static_cast<int64_t>(t) * k + r] = best_e[r];
            topk_w[static_cast<int64_t>(t) * k + r] = num[r] / den;
          }
      }
    } else {
      s_abort = 1;
      report_error(status, MOE_ERR_TIMEOUT);
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

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

template <int NP>
cudaError_t launch_np(const CUtensorMap& mx, const float* w, const float* bias, float* logits,
                      int32_t* topk_idx, float* topk_w, int T, int d, int N, int k, int* status,
                      uint64_t timeout_ns, cudaStream_t s) {
  using C = RCfg<NP>;
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [] {
    attr = cudaFuncSetAttribute(router_tc_kernel<NP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                C::SMEM_BYTES);
  });
  if (attr != cudaSuccess) return attr;
  const int grid = (T + kTok - 1) / kTok;
  router_tc_kernel<NP><<<grid, kThreads, C::SMEM_BYTES, s>>>(mx, w, bias, logits, topk_idx, topk_w,
                                                             T, d, N, k, status, timeout_ns);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router_tc(const uint16_t* x, const float* w_router, const float* bias,
                             float* logits, int32_t* topk_idx, float* topk_w, int T, int d, int N,
                             int k, int* status, uint64_t timeout_ns, cudaStream_t s) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return cudaErrorInvalidValue;
  CUtensorMap mx;
  const cuuint64_t gd[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(T)};
  const cuuint64_t gs[1] = {static_cast<cuuint64_t>(d) * 2};
  const cuuint32_t box[2] = {kBK, kTok};
  const cuuint32_t es[2] = {1, 1};
  if (fn(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(x), gd, gs, box, es,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (N <= 16) return launch_np<16>(mx, w_router, bias, logits, topk_idx, topk_w, T, d, N, k, status, timeout_ns, s);
  if (N <= 32) return launch_np<32>(mx, w_router, bias, logits, topk_idx, topk_w, T, d, N, k, status, timeout_ns, s);
  if (N <= 64) return launch_np<64>(mx, w_router, bias, logits, topk_idx, topk_w, T, d, N, k, status, timeout_ns, s);
  if (N <= 128) return launch_np<128>(mx, w_router, bias, logits, topk_idx, topk_w, T, d, N, k, status, timeout_ns, s);
  return launch_np<256>(mx, w_router, bias, logits, topk_idx, topk_w, T, d, N, k, status, timeout_ns, s);
}

}  // namespace moe
