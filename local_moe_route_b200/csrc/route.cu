// route.cu -- router logits, top-k selection and softmax weights.
//
// The router of every MoE layer picks a few experts per token (penglei.dev
// "Strata local MoE" post, section "原理一：把显存作为专家缓存"; 512 experts,
// top-10: kongchang.com "两天移植，预填充提速8倍：Strata引擎实测", section
// "Strata快在哪").  Readings used (the pages give no formula): logits =
// x . W_r (+ bias), the k largest logits with exact ties going to the lower
// expert index, weights = softmax over the k selected logits.
//
// Logits come from one of two kernels:
//  * a tcgen05 GEMM for prefill batches (x tile K-major and W_r tile MN-major,
//    both brought in by TMA with 128-byte swizzle, fp32 accumulators in TMEM);
//  * a CUDA-core kernel that splits K for small batches (a GEMV that only
//    streams W_r) and for shapes the TMA path does not cover.
// The top-k kernel then sums the K-split partials in a fixed order, adds the
// bias, and selects with one warp per token.
#include "common.cuh"
#include "internal.h"

namespace strata {

// ===========================================================================
// tcgen05 router GEMM: logits[t][e] = sum_i x[t][i] * W_r[i][e]
namespace rt {
constexpr int BM = 128;                 // tokens per CTA (TMEM lanes)
constexpr int BN = 128;                 // experts per CTA (TMEM columns)
constexpr int BK = 64;                  // K per stage (one 128-byte swizzle row)
constexpr int STAGES = 3;                // 99 KB of shared memory: two CTAs per SM
constexpr int A_BYTES = BM * BK * 2;    // x tile       16 KB
constexpr int B_BYTES = BN * BK * 2;    // W_r tile     16 KB (two 64-expert boxes)
constexpr int SMEM = 1024 + STAGES * (A_BYTES + B_BYTES) + 256;
constexpr int THREADS = 192;            // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
}  // namespace rt

__global__ void __launch_bounds__(rt::THREADS, 2)
    router_logits_tc_kernel(const __grid_constant__ CUtensorMap map_x,
                            const __grid_constant__ CUtensorMap map_wr, int T, int d, int E,
                            float* __restrict__ logits, unsigned* err) {
  using namespace rt;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES * B_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* accf = empty + STAGES;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(accf + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * BM;
  const int n0 = blockIdx.y * BN;
  const int KB = d / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&map_x);
    prefetch_tmap(&map_wr);
  }
  if (warp == 1) tmem_alloc(tmem_holder, BN);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % STAGES;
        if (kb >= STAGES && !mbar_wait(&empty[s], ((kb / STAGES) - 1) & 1, abort_flag, err)) break;
        mbar_arrive_expect_tx(&full[s], A_BYTES + B_BYTES);
        tma_load_2d(sA + s * A_BYTES, &map_x, kb * BK, m0, &full[s]);
        tma_load_2d(sB + s * B_BYTES, &map_wr, n0, kb * BK, &full[s]);
        tma_load_2d(sB + s * B_BYTES + B_BYTES / 2, &map_wr, n0 + 64, kb * BK, &full[s]);
      }
    }
  } else if (warp == 1) {
    // the whole warp follows the ring; one lane, elected once, issues the
    // MMAs and commits
    const bool leader = elect_one();
    const uint32_t idesc = idesc_f32acc(BM, BN, kFmtBF16, 1);
    bool stop = false;
    for (int kb = 0; kb < KB; ++kb) {
      const int s = kb % STAGES;
      if (!mbar_wait_warp(&full[s], (kb / STAGES) & 1, abort_flag, err)) {
        stop = true;
        break;
      }
      tc_fence_after();
      if (leader) {
        const uint32_t a0 = smem_addr(sA + s * A_BYTES);
        const uint32_t b0 = smem_addr(sB + s * B_BYTES);
#pragma unroll
        for (int ks = 0; ks < BK / 16; ++ks) {
          const uint64_t ad = desc_kmajor_sw128(a0 + ks * 32);
          const uint64_t bd = desc_mnmajor_sw128(b0 + ks * 16 * 128, B_BYTES / 2);
          mma_f16kind_ss(tmem, ad, bd, idesc, (kb | ks) != 0);
        }
        mma_commit(&empty[s]);
      }
      __syncwarp();
    }
    if (!stop && leader) mma_commit(accf);
    __syncwarp();
  } else {
    const int q = warp & 3;          // TMEM lane quadrant this warp may read
    const int row = q * 32 + lane;
    const int t = m0 + row;
    const bool ok = mbar_wait_warp(accf, 0, abort_flag, err);
    tc_fence_after();
    if (ok) {
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        __syncwarp();   // converged before the .sync.aligned TMEM load
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem + ((uint32_t)(q * 32) << 16) + c * 32, r);
        tmem_ld_wait();
        if (t < T) {
          float4* dst = reinterpret_cast<float4*>(logits + (size_t)t * E + n0 + c * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                 __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, BN);
  }
}

bool router_uses_tc(int T, int d, int E) {
  return T >= 128 && E % rt::BN == 0 && d % rt::BK == 0;
}

cudaError_t launch_router_logits_tc(const uint16_t* x, const uint16_t* w_router, int T, int d,
                                    int E, float* logits, unsigned* err, cudaStream_t s) {
  CUtensorMap mx, mw;
  if (encode_tmap_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, d, T, (uint64_t)d * 2, rt::BK,
                     rt::BM, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (encode_tmap_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w_router, E, d, (uint64_t)E * 2, 64,
                     rt::BK, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  {
    cudaError_t e = cudaFuncSetAttribute(router_logits_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, rt::SMEM);
    if (e != cudaSuccess) return e;
  }
  dim3 grid((T + rt::BM - 1) / rt::BM, E / rt::BN);
  router_logits_tc_kernel<<<grid, rt::THREADS, rt::SMEM, s>>>(mx, mw, T, d, E, logits, err);
  return cudaGetLastError();
}

// ===========================================================================
// CUDA-core router logits with K split: partial[split][t][e].
// Each thread owns two adjacent experts; x rows of an 8-token tile are staged
// in shared memory 256 K values at a time.
namespace rs {
constexpr int THREADS = 128;
constexpr int EXPERTS = 2 * THREADS;  // experts per block
constexpr int TT = 8;                 // tokens per register tile
constexpr int KC = 256;               // K values staged per pass
}  // namespace rs

int router_ksplit(int T, int d, int E) {
  if (router_uses_tc(T, d, E) || T > 16) return 1;
  int ks = d / 32;
  if (ks > 128) ks = 128;
  return ks < 1 ? 1 : ks;
}

__global__ void __launch_bounds__(rs::THREADS)
    router_logits_simt_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ wr,
                              int T, int d, int E, int rows_per_split,
                              float* __restrict__ partial) {
  using namespace rs;
  __shared__ float xs[TT][KC];
  const int e0 = blockIdx.x * EXPERTS + 2 * threadIdx.x;
  const int split = blockIdx.y;
  const int k_begin = split * rows_per_split;
  const int k_end = min(d, k_begin + rows_per_split);
  const bool even_e = (E & 1) == 0;
  for (int t0 = blockIdx.z * TT; t0 < T; t0 += gridDim.z * TT) {
    float acc[TT][2];
#pragma unroll
    for (int j = 0; j < TT; ++j) acc[j][0] = acc[j][1] = 0.f;
    for (int kc = k_begin; kc < k_end; kc += KC) {
      const int len = min(KC, k_end - kc);
      __syncthreads();
      for (int idx = threadIdx.x; idx < TT * KC; idx += THREADS) {
        const int j = idx / KC, i = idx % KC;
        float v = 0.f;
        if (t0 + j < T && i < len) v = bf16_lo(x[(size_t)(t0 + j) * d + kc + i]);
        xs[j][i] = v;
      }
      __syncthreads();
      if (e0 < E) {
#pragma unroll 8
        for (int i = 0; i < len; ++i) {
          const size_t off = (size_t)(kc + i) * E + e0;
          float w0, w1;
          if (even_e) {
            const uint32_t pr = *reinterpret_cast<const uint32_t*>(wr + off);
            w0 = bf16_lo(pr);
            w1 = bf16_hi(pr);
          } else {
            w0 = bf16_lo(wr[off]);
            w1 = (e0 + 1 < E) ? bf16_lo(wr[off + 1]) : 0.f;
          }
#pragma unroll
          for (int j = 0; j < TT; ++j) {
            acc[j][0] = fmaf(xs[j][i], w0, acc[j][0]);
            acc[j][1] = fmaf(xs[j][i], w1, acc[j][1]);
          }
        }
      }
    }
    if (e0 < E) {
#pragma unroll
      for (int j = 0; j < TT; ++j) {
        if (t0 + j >= T) break;
        float* dst = partial + ((size_t)split * T + t0 + j) * E + e0;
        dst[0] = acc[j][0];
        if (e0 + 1 < E) dst[1] = acc[j][1];
      }
    }
  }
}

// Sums the K-split partial logits of (token blockIdx.y, experts blockIdx.x *
// 32 ..) into split 0: warp j adds splits j, j + 8, ... and the eight warp
// sums are added in warp order, so the result does not depend on timing.
__global__ void __launch_bounds__(256)
    router_split_reduce_kernel(float* __restrict__ partial, int ksplit, int T, int E) {
  __shared__ float red[8][33];
  const int el = threadIdx.x & 31, sg = threadIdx.x >> 5;
  const int e = blockIdx.x * 32 + el, t = blockIdx.y;
  float acc = 0.f;
  if (e < E) {
#pragma unroll 4
    for (int sp = sg; sp < ksplit; sp += 8) acc += partial[((size_t)sp * T + t) * E + e];
  }
  red[sg][el] = acc;
  __syncthreads();
  if (sg == 0 && e < E) {
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) sum += red[j][el];
    partial[(size_t)t * E + e] = sum;
  }
}

// Logits into split 0 of `partial` (the other splits are scratch).
cudaError_t launch_router_logits_simt(const uint16_t* x, const uint16_t* w_router, int T, int d,
                                      int E, int ksplit, float* partial, cudaStream_t s) {
  const int rows = (d + ksplit - 1) / ksplit;
  // token tiles spread over grid.z (each block loops if there are more)
  const int tiles = (T + rs::TT - 1) / rs::TT;
  dim3 grid((E + rs::EXPERTS - 1) / rs::EXPERTS, ksplit, tiles < 65535 ? tiles : 65535);
  router_logits_simt_kernel<<<grid, rs::THREADS, 0, s>>>(x, w_router, T, d, E, rows, partial);
  if (ksplit > 1) {
    dim3 rgrid((E + 31) / 32, T);
    router_split_reduce_kernel<<<rgrid, 256, 0, s>>>(partial, ksplit, T, E);
  }
  return cudaGetLastError();
}

// ===========================================================================
// Order-preserving 32-bit key of a logit: larger float, larger key; NaN maps
// to the key of -inf and -0 to that of +0, so keys compare as the selection
// treats the floats.  Key 0 lies below every key (absent / taken entries).
__device__ __forceinline__ uint32_t logit_key(float f) {
  if (f != f) f = -INFINITY;
  if (f == 0.f) f = 0.f;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_logit(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Top-k + softmax, one warp per token.  Lane l holds experts l, l+32, ... as
// keys.  Each of the k rounds: every lane offers its best entry (largest key,
// lowest index among equal keys), the warp takes the largest key and the
// lowest expert index offering it (two redux.sync reductions), and the owning
// lane marks that entry taken; lane j keeps the j-th pick.  Exact ties go to the
// lower expert index and NaN never wins.
template <int VPL>
__global__ void __launch_bounds__(128)
    topk_softmax_kernel(const float* __restrict__ partial, int ksplit,
                        const float* __restrict__ bias, int T, int E, int k,
                        int32_t* __restrict__ ids, float* __restrict__ w,
                        float* __restrict__ logits_out) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * 4 + (threadIdx.x >> 5);
  if (t >= T) return;
  uint32_t key[VPL];
  uint32_t taken = 0;                         // entries already picked
  // the lane's VPL logits of split sp are loaded together (one round trip
  // per split, not one per logit), and the splits added in order
  float acc[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) acc[i] = 0.f;
  for (int sp = 0; sp < ksplit; ++sp) {
    const float* src = partial + ((size_t)sp * T + t) * E + lane;
    float v[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) v[i] = lane + 32 * i < E ? src[32 * i] : 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) acc[i] += v[i];
  }
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = lane + 32 * i;
    key[i] = 0u;
    if (e < E) {
      float a = acc[i];
      if (bias) a += bias[e];
      if (logits_out) logits_out[(size_t)t * E + e] = a;
      key[i] = logit_key(a);
    }
  }
  uint32_t my_key = 0, top = 0;
  int my_i = 0;
  for (int j = 0; j < k; ++j) {
    // up to four independent chains over i mod 4, merged in index order
    uint32_t bk[4] = {0u, 0u, 0u, 0u};
    int bs[4] = {0, 0, 0, 0};
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int c = i & 3;
      if (!((taken >> i) & 1u) && key[i] > bk[c]) {                   // the first of equal keys stays (lower index)
        bk[c] = key[i];
        bs[c] = i;
      }
    }
#pragma unroll
    for (int c = 1; c < 4; ++c) {
      if (bk[c] > bk[0] || (bk[c] == bk[0] && bs[c] < bs[0])) {
        bk[0] = bk[c];
        bs[0] = bs[c];
      }
    }
    const uint32_t wk = __reduce_max_sync(0xffffffffu, bk[0]);
    const int wi = __reduce_min_sync(0xffffffffu, bk[0] == wk ? lane + 32 * bs[0] : 0x7fffffff);
    if ((wi & 31) == lane) taken |= 1u << (wi >> 5);
    if (j == 0) top = wk;
    if (lane == j) {
      my_key = wk;
      my_i = wi;
    }
  }
  const float ex = (lane < k) ? expf(key_logit(my_key) - key_logit(top)) : 0.f;
  float sum = ex;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  if (lane < k) {
    ids[(size_t)t * k + lane] = my_i;
    w[(size_t)t * k + lane] = ex / sum;
  }
}

cudaError_t launch_topk_softmax(const float* partial, int ksplit, const float* bias, int T,
                                int E, int k, int32_t* ids, float* w, float* logits_out,
                                cudaStream_t s) {
  const dim3 grid((T + 3) / 4);
#define STRATA_TOPK(V)                                                                     \
  topk_softmax_kernel<V><<<grid, 128, 0, s>>>(partial, ksplit, bias, T, E, k, ids, w, \
                                                logits_out)
  if (E <= 32) STRATA_TOPK(1);
  else if (E <= 64) STRATA_TOPK(2);
  else if (E <= 128) STRATA_TOPK(4);
  else if (E <= 256) STRATA_TOPK(8);
  else if (E <= 512) STRATA_TOPK(16);
  else STRATA_TOPK(32);
#undef STRATA_TOPK
  return cudaGetLastError();
}

}  // namespace strata
