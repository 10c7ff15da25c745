// sparse_attn.cu -- attention over the KV-cache rows an indexer selected.
//
// The pages' model uses sparse attention: an indexer picks about 2000
// positions for every query, and Strata's own kernel reads only the
// selected KV-cache rows where llama.cpp builds a full mask and runs dense
// flash attention (kongchang.com "两天移植，预填充提速8倍：Strata引擎实测",
// section "Strata快在哪", attention paragraph).  Per query token t and query
// head h (KV head hk = h / (Hq / Hkv)):
//   o[t][h] = softmax_p( scale * q[t][h] . K[p][hk] ) . V[p][hk],  p in idx[t]
// with idx slots of -1 unused.
//
// Small query batches (decode, speculative verify) are bound by the bytes of
// the selected rows, 2 * Hkv * D * 2 bytes per position per query.  Two
// kernels, split-K style:
//   1. one CTA per (query, KV head, slice of 64 index slots): the slice's
//      selected K and V rows are copied into shared memory (cp.async, all
//      issued before one wait); two threads take one slot, each forming the
//      scores of the G query heads that share the KV head over half of D,
//      and add them; the slice's softmax maximum and sum per head stay in
//      shared memory; thread d accumulates sum_p exp(s - m) V[p][d] over the
//      slice, fp32;
//   2. one CTA per (query, head) rescales and adds the slices' partial sums
//      (max-subtracted exponentials, fixed order) and rounds to bf16.
#include "common.cuh"
#include "internal.h"

namespace strata {

namespace sa {
constexpr int SLICE = 64;      // index slots per CTA (two threads per slot for the scores)
constexpr int THREADS = 128;
constexpr int MAXG = 16;       // query heads per KV head
constexpr int MAXSPLIT = 1024; // slices per query (P <= 65536)
}  // namespace sa

template <int D>
__global__ void __launch_bounds__(sa::THREADS)
    sparse_attn_split_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ kc,
                             const uint16_t* __restrict__ vc, const int32_t* __restrict__ idx,
                             int L, int Hq, int Hkv, int P, int nsplit, float scale,
                             float* __restrict__ part_o, float* __restrict__ part_ml,
                             unsigned* err) {
  using namespace sa;
  constexpr int RP = D + 8;                  // halves per staged row (16 bytes of padding)
  const int split = blockIdx.x, hk = blockIdx.y, t = blockIdx.z;
  const int G = Hq / Hkv;
  extern __shared__ __align__(16) uint8_t sa_smem[];
  uint16_t* ks = reinterpret_cast<uint16_t*>(sa_smem);            // [SLICE][RP]
  uint16_t* vs = ks + SLICE * RP;                                  // [SLICE][RP]
  float* qs = reinterpret_cast<float*>(vs + SLICE * RP);           // [MAXG][D]
  float* ws = qs + MAXG * D;                                       // [MAXG][SLICE]
  int* rows = reinterpret_cast<int*>(ws + MAXG * SLICE);           // [SLICE]
  float* mx = reinterpret_cast<float*>(rows + SLICE);              // [MAXG]
  float* sm = mx + MAXG;                                           // [MAXG]
  const int th = threadIdx.x;
  // the slice's index slots and the G query rows of this KV head: every load
  // issued before the first barrier (16-byte loads of q, at most two per
  // thread: G * D <= 16 * 128)
  int p = -1;
  const int slot = split * SLICE + th;
  if (th < SLICE && slot < P) p = idx[(size_t)t * P + slot];
  uint4 qv[2];
  const uint16_t* qrow = q + ((size_t)t * Hq + hk * G) * D;   // G rows of D, contiguous
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int i = (th + u * THREADS) * 8;
    if (i < G * D) qv[u] = *reinterpret_cast<const uint4*>(qrow + i);
  }
  if (th < SLICE) {
    if (p >= L) {
      atomicOr(err, kErrIndex);
      p = -1;
    }
    rows[th] = p;
  }
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int i = (th + u * THREADS) * 8;
    if (i < G * D) {
      const uint4 v = qv[u];
      float* dst = qs + i;                   // [g][dd] with g * D + dd = i
      dst[0] = bf16_lo(v.x) * scale; dst[1] = bf16_hi(v.x) * scale;
      dst[2] = bf16_lo(v.y) * scale; dst[3] = bf16_hi(v.y) * scale;
      dst[4] = bf16_lo(v.z) * scale; dst[5] = bf16_hi(v.z) * scale;
      dst[6] = bf16_lo(v.w) * scale; dst[7] = bf16_hi(v.w) * scale;
    }
  }
  __syncthreads();
  // the slice's K and V rows into shared memory: every copy issued before
  // the one wait (a chain of dependent loads would cost a DRAM round trip
  // per row)
  constexpr int CPR = D / 8;                 // 16-byte chunks per row
  for (int c = th; c < SLICE * CPR; c += THREADS) {
    const int i = c / CPR, j = c % CPR;
    const int pr = rows[i];
    if (pr < 0) continue;
    const size_t off = ((size_t)pr * Hkv + hk) * D + 8 * j;
    const uint32_t dk = smem_addr(ks + i * RP + 8 * j), dv = smem_addr(vs + i * RP + 8 * j);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dk), "l"(kc + off) : "memory");
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dv), "l"(vc + off) : "memory");
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();
  // scores of slot th / 2 for the G heads: the two threads of a slot take
  // one half of D each and add their sums (fixed order: lower half first)
  const int sl = th >> 1, hf = th & 1;
  const int pr_s = rows[sl];
  float s[MAXG];
#pragma unroll
  for (int g = 0; g < MAXG; ++g) s[g] = 0.f;
  if (pr_s >= 0) {
    const uint4* kr = reinterpret_cast<const uint4*>(ks + sl * RP) + hf * (CPR / 2);
#pragma unroll 4
    for (int c = 0; c < CPR / 2; ++c) {
      const uint4 v = kr[c];
      const float e[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                          bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
      const int d0 = (hf * (CPR / 2) + c) * 8;
#pragma unroll
      for (int g = 0; g < MAXG; ++g) {
        if (g < G) {
#pragma unroll
          for (int j = 0; j < 8; ++j) s[g] = fmaf(qs[g * D + d0 + j], e[j], s[g]);
        }
      }
    }
  }
#pragma unroll
  for (int g = 0; g < MAXG; ++g) {
    const float o = __shfl_xor_sync(0xffffffffu, s[g], 1);
    const float tot = hf == 0 ? s[g] + o : o + s[g];
    if (g < G && hf == 0) ws[g * SLICE + sl] = pr_s >= 0 ? tot : -INFINITY;
  }
  __syncthreads();
  // per head: maximum and sum of exp(s - m) over the slice
  const int warp = th >> 5, lane = th & 31;
  for (int g = warp; g < G; g += THREADS / 32) {
    float m = -INFINITY;
    for (int i = lane; i < SLICE; i += 32) m = fmaxf(m, ws[g * SLICE + i]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float l = 0.f;
    for (int i = lane; i < SLICE; i += 32) {
      const float x = ws[g * SLICE + i];
      const float e = x == -INFINITY ? 0.f : __expf(x - m);
      ws[g * SLICE + i] = e;
      l += e;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
    if (lane == 0) {
      mx[g] = m;
      sm[g] = l;
    }
  }
  __syncthreads();
  // o[g][d] = sum_p e[g][p] V[p][d]; thread = feature d
  if (th < D) {
    float o[MAXG];
#pragma unroll
    for (int g = 0; g < MAXG; ++g) o[g] = 0.f;
    for (int i = 0; i < SLICE; ++i) {
      if (rows[i] < 0) continue;
      const float v = __uint_as_float((uint32_t)vs[i * RP + th] << 16);
#pragma unroll
      for (int g = 0; g < MAXG; ++g)
        if (g < G) o[g] = fmaf(ws[g * SLICE + i], v, o[g]);
    }
#pragma unroll
    for (int g = 0; g < MAXG; ++g)
      if (g < G) part_o[(((size_t)t * Hq + hk * G + g) * nsplit + split) * D + th] = o[g];
  }
  if (th < G) {
    const size_t b = (((size_t)t * Hq + hk * G + th) * nsplit + split) * 2;
    part_ml[b] = mx[th];
    part_ml[b + 1] = sm[th];
  }
}

template <int D>
constexpr int sparse_attn_smem() {
  return 2 * sa::SLICE * (D + 8) * 2 + sa::MAXG * D * 4 + sa::MAXG * sa::SLICE * 4 +
         sa::SLICE * 4 + 2 * sa::MAXG * 4;
}

// The slices' maxima and sums of one (query, head) are staged in shared
// memory first (all loads issued before any is used), then every thread forms
// the weights exp(m_s - M) and adds its feature over the slices, eight
// loads in flight at a time.
template <int D>
__global__ void __launch_bounds__(D)
    sparse_attn_combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_ml,
                               int nsplit, uint16_t* __restrict__ out) {
  __shared__ float f_s[sa::MAXSPLIT], l_s[sa::MAXSPLIT];
  __shared__ float red[D / 32];
  const int th = threadIdx.x;
  const size_t th_h = blockIdx.x;            // t * Hq + h
  float m_loc = -INFINITY;
  for (int s = th; s < nsplit; s += D) {
    const float2 ml = *reinterpret_cast<const float2*>(part_ml + (th_h * nsplit + s) * 2);
    f_s[s] = ml.x;
    l_s[s] = ml.y;
    m_loc = fmaxf(m_loc, ml.x);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m_loc = fmaxf(m_loc, __shfl_xor_sync(0xffffffffu, m_loc, off));
  if ((th & 31) == 0) red[th >> 5] = m_loc;
  __syncthreads();
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < D / 32; ++w) M = fmaxf(M, red[w]);
  // weights of the slices (0 for a slice with no valid slot)
  for (int s = th; s < nsplit; s += D)
    f_s[s] = (M == -INFINITY || f_s[s] == -INFINITY) ? 0.f : __expf(f_s[s] - M);
  __syncthreads();
  float num = 0.f, den = 0.f;
  const float* po = part_o + th_h * nsplit * D + th;
  int s = 0;
  for (; s + 8 <= nsplit; s += 8) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = po[(size_t)(s + u) * D];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      den = fmaf(f_s[s + u], l_s[s + u], den);
      num = fmaf(f_s[s + u], v[u], num);
    }
  }
  for (; s < nsplit; ++s) {
    den = fmaf(f_s[s], l_s[s], den);
    num = fmaf(f_s[s], po[(size_t)s * D], num);
  }
  const float o = den > 0.f ? num / den : 0.f;
  out[th_h * D + th] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
}

size_t sparse_attn_scratch(int T, int Hq, int P, int D) {
  const int nsplit = (P + sa::SLICE - 1) / sa::SLICE;
  return ((size_t)T * Hq * nsplit * (D + 2) * 4 + 255) & ~size_t(255);
}

cudaError_t launch_sparse_attn(const uint16_t* q, const uint16_t* kc, const uint16_t* vc,
                               const int32_t* idx, int T, int L, int Hq, int Hkv, int D, int P,
                               float scale, uint16_t* out, void* ws, unsigned* err,
                               cudaStream_t s) {
  const int nsplit = (P + sa::SLICE - 1) / sa::SLICE;
  float* part_o = static_cast<float*>(ws);
  float* part_ml = part_o + (size_t)T * Hq * nsplit * D;
  const dim3 grid(nsplit, Hkv, T);
  if (D == 128) {
    constexpr int sm = sparse_attn_smem<128>();
    cudaError_t e = cudaFuncSetAttribute(sparse_attn_split_kernel<128>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
    if (e != cudaSuccess) return e;
    sparse_attn_split_kernel<128><<<grid, sa::THREADS, sm, s>>>(q, kc, vc, idx, L, Hq, Hkv, P,
                                                                nsplit, scale, part_o, part_ml, err);
    sparse_attn_combine_kernel<128><<<T * Hq, 128, 0, s>>>(part_o, part_ml, nsplit, out);
  } else {
    constexpr int sm = sparse_attn_smem<64>();
    cudaError_t e = cudaFuncSetAttribute(sparse_attn_split_kernel<64>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
    if (e != cudaSuccess) return e;
    sparse_attn_split_kernel<64><<<grid, sa::THREADS, sm, s>>>(q, kc, vc, idx, L, Hq, Hkv, P,
                                                               nsplit, scale, part_o, part_ml, err);
    sparse_attn_combine_kernel<64><<<T * Hq, 64, 0, s>>>(part_o, part_ml, nsplit, out);
  }
  return cudaGetLastError();
}

}  // namespace strata
