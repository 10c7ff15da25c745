// decode_fused.cu -- the whole MoE layer for a decode / speculative-verify
// batch of at most four tokens in one persistent launch.
//
// A decode step reads the packed weights of every expert its tokens chose
// and does little arithmetic on them (kongchang.com
// "两天移植，预填充提速8倍：Strata引擎实测", section "Strata快在哪", decode
// paragraph: one token plus up to three MTP draft tokens are verified
// together), so the step is bound by HBM bandwidth over those bytes plus the
// fixed cost between the weight streams.  Here that fixed cost is one
// launch: the CTAs stay resident (cooperative launch, two per SM) and pass
// through five phases separated by grid-wide barriers with bounded waits:
//
//   P0  router partial logits (items of 512 rows of W_r x 64 experts);
//       every CTA also converts x of all tokens to fp16 in shared memory;
//   --- grid barrier
//   P0b the logits, each summed once from the partials (spread over CTAs);
//   --- grid barrier
//   P1  every CTA sums the partials, picks each token's top k (exact ties to
//       the lower expert index), the softmax weights, and groups the T*k
//       slots by expert (counts, offsets, stable order) in its own shared
//       memory: same inputs, same code, same result in every CTA, so no
//       barrier follows;
//   P2  gate/up + SwiGLU: units of 16 weight rows of one expert, K split
//       over the 8 consumer warps, both matrices streamed by TMA through a
//       3-deep ring, B operand = x from shared memory; h to global (fp16);
//   --- grid barrier
//   P3  down: units of 64 rows of one expert (4 row groups x 2 K halves),
//       each stage carries the expert's h rows; output rows to global (fp32);
//   --- grid barrier
//   P4  combine: y_t = sum_j w_tj * row_(t,j), fp32 in slot order, bf16.
//
// Matrix products use mma.sync m16n8k16 with fp16 operands: the weights as
// exact integer codes (a nibble pair (i, i + 4) becomes an fp16 pair with one
// mask-and-xor and one fma), the tokens as fp16 (x converted once, h as
// written by P2), fp32 accumulation; each scale group's sum is multiplied by
// its fp16 scale once.  With at most four tokens per expert the MMAs are
// never the limit: instructions per weight and bytes in flight are.
#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace strata {

namespace df {
constexpr int MAXT = 4;                   // tokens per batch on this path
constexpr int CONS = 8;                   // consumer warps
constexpr int THREADS = (CONS + 1) * 32;  // + one producer warp
constexpr int ST = 3;                     // ring stages
// A ring stage: gate/up: 16 rows x 1024 K of both matrices (16 KB) and their
// scales (16 rows x 1024 / G groups each, at most 2 KB); down: 64 rows x
// 256 K (8 KB), the expert's h rows (2 KB) and the unit's scale rows
// (64 rows x n / G groups, at most 4 KB).
constexpr int SLOT = 18432;               // bytes per ring stage
constexpr int P2_SC = 16384;              // offset of the gate/up scales in a stage
constexpr int P3_H = 8192, P3_SC = 10240; // offsets of h and of the down scales
constexpr int PF = 6;                     // stages the producer prefetches into L2 ahead
constexpr int P2_ROWS = 16;               // gate/up unit: 16 rows, K split 8 ways
constexpr int P2_KST = 1024;              // gate/up K per stage
constexpr int P3_ROWS = 64;               // down unit: 4 row groups x 2 K halves
constexpr int P3_KST = 256;               // down K per stage
constexpr int P0_RS = 512;                // router rows per item
constexpr int P0_MAXKS = 8;               // router K slices (d <= 4096)
constexpr int XPT = 8;                    // 16-byte chunks of x per thread (T * d <= 8 * 8 * THREADS)
constexpr int MAXE = 1024, MAXK = 32;
constexpr int MAXS = MAXT * MAXK;

// Shared memory (offsets from a 1024-byte aligned base).  The x area holds
// x of all tokens in fp16 ([T][d + 8], 16 bytes of padding per row so that
// rows land on different banks).
struct Smem {
  int ring, x, red, bars, route, total;
  __host__ __device__ static Smem of(int T, int d) {
    Smem s;
    s.ring = 0;
    s.x = ST * SLOT;
    const int xb = ((T * (d + 8) * 2) + 1023) & ~1023;
    s.red = s.x + xb;                            // [8 warps][32 lanes][8] fp32
    s.bars = s.red + CONS * 32 * 8 * 4;
    s.route = s.bars + 128;
    // ids, w [MAXS]; counts, active [MAXE]; offsets [MAXE + 1]; rowtok,
    // slotrow [MAXS]; misc [64]  (the scan scratch `pos` lives in the ring)
    s.total = s.route + (2 * MAXS + 2 * MAXE + MAXE + 1 + 2 * MAXS + 64) * 4;
    return s;
  }
};
}  // namespace df

struct FusedArgs {
  const uint16_t* x;         // [T][d] bf16
  const uint16_t* w_router;  // [d][E] bf16
  const float* bias;         // [E] or null
  const uint16_t* s_gate;    // [E][n][d/G] fp16
  const uint16_t* s_up;
  const uint16_t* s_down;    // [E][d][n/G]
  uint16_t* y;               // [T][d] bf16
  int32_t* ids_out;          // [T][k] or null
  float* w_out;              // [T][k] or null
  float* partial;            // [d / 512][T][E]
  float* logits;             // [T][E]
  uint16_t* h;               // [T*k][n] fp16, features interleaved within 8
  float* rows;               // [T*k][d] fp32
  unsigned* sync;            // [4] zeroed before the launch
  unsigned* err;
  int T, d, E, k, n, G;
};

// ---------------------------------------------------------------------------
// All threads of the CTA: returns whether every CTA arrived in time.  A CTA
// whose own waits gave up (cta_abort) raises the grid-wide abort first.
__device__ __forceinline__ bool df_sync_grid(unsigned* sync, int b, unsigned* err,
                                             volatile int* flag, volatile int* cta_abort) {
  __syncthreads();
  if (threadIdx.x == 0) {
    if (*cta_abort) atomicExch(&sync[2], 1u);
    *flag = grid_barrier_wait(sync, b, err) ? 1 : 0;
  }
  __syncthreads();
  const bool ok = *flag != 0;
  // order this CTA's later accesses through the async proxy (TMA) after the
  // barrier and after its own earlier generic accesses of shared memory
  asm volatile("fence.proxy.async;" ::: "memory");
  return ok;
}

// Block-wide exclusive scan of v[0..n) in place (each thread takes a run of
// consecutive entries), returning the total.  Uses tmp[0..32]; blockDim.x is
// a multiple of 32 and at most 1024.
__device__ int df_block_scan(int* v, int n, int* tmp) {
  const int th = threadIdx.x, lane = th & 31, warp = th >> 5, nw = blockDim.x >> 5;
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int b0 = th * per;
  int s = 0;
  for (int i = 0; i < per; ++i)
    if (b0 + i < n) s += v[b0 + i];
  int incl = s;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) tmp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int wv = lane < nw ? tmp[lane] : 0;
    int wi = wv;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += o;
    }
    __syncwarp();
    tmp[lane] = wi - wv;                         // exclusive prefix of the warp totals
    if (lane == 31) tmp[32] = wi;                // grand total
  }
  __syncthreads();
  int run = tmp[warp] + incl - s;
  const int total = tmp[32];
  for (int i = 0; i < per; ++i)
    if (b0 + i < n) {
      const int x = v[b0 + i];
      v[b0 + i] = run;
      run += x;
    }
  __syncthreads();
  return total;
}

// ---------------------------------------------------------------------------
// P0: partial router logits.  Item = (512 rows of W_r, 64 experts): thread
// (row group rr = th / 8 of 32, 16-byte chunk c = th % 8 of 8 experts) loads
// the chunk of rows rr, rr + 32, ... (16 rows) all at once, multiplies them
// by x of those rows (staged per item in shared memory as fp32) and the 32
// row groups are added in a fixed order.  Uses threads 0..255.
//   scratch: >= 32 * MAXT * 64 + MAXT * 512 floats
__device__ void df_router_partials(const FusedArgs& a, float* scratch) {
  using namespace df;
  const int th = threadIdx.x;
  const int neb = (a.E + 63) / 64, nks = a.d / P0_RS;
  float* red = scratch;                                   // [32][MAXT][64]
  float* xr = scratch + 32 * MAXT * 64;                   // [MAXT][512]
  for (int item = blockIdx.x; item < neb * nks; item += gridDim.x) {
    const int eb = item % neb, ks = item / neb;
    const int r0 = ks * P0_RS;
    if (th < a.T * (P0_RS / 8)) {                         // one 16-byte chunk per thread
      const int t = th / (P0_RS / 8), j = th % (P0_RS / 8);
      const uint4 v = ld_nc_v4(a.x + (size_t)t * a.d + r0 + 8 * j);
      float* dst = xr + t * P0_RS + 8 * j;
      dst[0] = bf16_lo(v.x); dst[1] = bf16_hi(v.x); dst[2] = bf16_lo(v.y); dst[3] = bf16_hi(v.y);
      dst[4] = bf16_lo(v.z); dst[5] = bf16_hi(v.z); dst[6] = bf16_lo(v.w); dst[7] = bf16_hi(v.w);
    }
    __syncthreads();
    if (th < 256) {
      const int c = th & 7, rr = th >> 3;
      const int e0 = eb * 64 + c * 8;
      float acc[MAXT][8];
#pragma unroll
      for (int t = 0; t < MAXT; ++t)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[t][j] = 0.f;
      if (e0 < a.E) {                                     // E % 8 == 0 on this path
        uint4 w[P0_RS / 32];
#pragma unroll
        for (int i = 0; i < P0_RS / 32; ++i)
          w[i] = ld_nc_v4(a.w_router + (size_t)(r0 + rr + 32 * i) * a.E + e0);
#pragma unroll
        for (int i = 0; i < P0_RS / 32; ++i) {
          const float wv[8] = {bf16_lo(w[i].x), bf16_hi(w[i].x), bf16_lo(w[i].y), bf16_hi(w[i].y),
                               bf16_lo(w[i].z), bf16_hi(w[i].z), bf16_lo(w[i].w), bf16_hi(w[i].w)};
#pragma unroll
          for (int t = 0; t < MAXT; ++t) {
            if (t < a.T) {
              const float xv = xr[t * P0_RS + rr + 32 * i];
#pragma unroll
              for (int j = 0; j < 8; ++j) acc[t][j] = fmaf(xv, wv[j], acc[t][j]);
            }
          }
        }
      }
#pragma unroll
      for (int t = 0; t < MAXT; ++t)
#pragma unroll
        for (int j = 0; j < 8; ++j) red[(rr * MAXT + t) * 64 + c * 8 + j] = acc[t][j];
    }
    __syncthreads();
    if (th < a.T * 64) {
      const int t = th / 64, l = th % 64;
      float sum = 0.f;
      for (int g = 0; g < 32; ++g) sum += red[(g * MAXT + t) * 64 + l];
      const int ee = eb * 64 + l;
      if (ee < a.E) a.partial[((size_t)ks * a.T + t) * a.E + ee] = sum;
    }
    __syncthreads();
  }
}

// x of all tokens -> fp16 in shared memory, features interleaved within
// groups of 8 (0, 4, 1, 5, 2, 6, 3, 7) to match the weight fragments.
__device__ bool df_load_x(const FusedArgs& a, uint16_t* xs) {
  using namespace df;
  bool over = false;
  const int cpr = a.d / 8;
  // every load of this thread first (at most XPT), then the conversions
  uint4 vin[XPT];
#pragma unroll
  for (int i = 0; i < XPT; ++i) {
    const int c = threadIdx.x + i * blockDim.x;
    if (c < a.T * cpr) vin[i] = ld_nc_v4(a.x + (size_t)c * 8);
  }
#pragma unroll
  for (int i = 0; i < XPT; ++i) {
    const int c = threadIdx.x + i * blockDim.x;
    if (c >= a.T * cpr) break;
    const int t = c / cpr, j = c % cpr;
    const uint4 v = vin[i];
    float e[8];
    e[0] = bf16_lo(v.x); e[1] = bf16_hi(v.x); e[2] = bf16_lo(v.y); e[3] = bf16_hi(v.y);
    e[4] = bf16_lo(v.z); e[5] = bf16_hi(v.z); e[6] = bf16_lo(v.w); e[7] = bf16_hi(v.w);
#pragma unroll
    for (int i = 0; i < 8; ++i) over |= fabsf(e[i]) > 65504.f;
    uint4 o;
    o.x = pack_f16x2(e[0], e[4]);
    o.y = pack_f16x2(e[1], e[5]);
    o.z = pack_f16x2(e[2], e[6]);
    o.w = pack_f16x2(e[3], e[7]);
    *reinterpret_cast<uint4*>(xs + (size_t)t * (a.d + 8) + 8 * j) = o;
  }
  return over;
}

// P1: logits, top k and softmax of every token (warp t), then the grouping
// of the T*k slots by expert.  Every CTA computes it; CTA 0 writes the
// optional outputs.
struct Route {
  int32_t* ids;      // [T*k]
  float* w;          // [T*k]
  int32_t* counts;   // [E]
  int32_t* offsets;  // [E + 1]
  int32_t* active;   // [n_active]
  int32_t* pos;      // [E] scratch
  int32_t* rowtok;   // [S] grouped row -> token
  int32_t* slotrow;  // [S] slot -> grouped row
  int* misc;         // [0] n_active, [1..32] scan scratch
};

// P0b: the logits, each once: the K slices' partial sums in order, then the
// bias.  Spread over the CTAs (every CTA reading all partials would make 64
// KB of L2 the hot spot of every SM at once).
__device__ void df_logits(const FusedArgs& a) {
  using namespace df;
  const int nks = a.d / P0_RS;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < a.T * a.E;
       i += gridDim.x * blockDim.x) {
    const int t = i / a.E, e = i % a.E;
    float p[P0_MAXKS];
#pragma unroll
    for (int ks = 0; ks < P0_MAXKS; ++ks)
      p[ks] = ks < nks ? __ldcg(a.partial + ((size_t)ks * a.T + t) * a.E + e) : 0.f;
    float acc = 0.f;
#pragma unroll
    for (int ks = 0; ks < P0_MAXKS; ++ks)
      if (ks < nks) acc += p[ks];
    if (a.bias) acc += __ldg(a.bias + e);
    a.logits[i] = acc;
  }
}

__device__ void df_route(const FusedArgs& a, const Route& R, float* logit_s) {
  using namespace df;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nks = a.d / P0_RS, S = a.T * a.k;
  // logits of every token (summed once, by all CTAs together, in P0b)
  for (int i = threadIdx.x; i < a.T * a.E; i += blockDim.x) logit_s[i] = __ldcg(a.logits + i);
  __syncthreads();
  // top k of each token by two warps: warp 2t + hf selects the k best of its
  // half of the experts (exact ties to the lower index, NaN never wins), then
  // warp 2t merges the two lists of k with the same order.  Any of the
  // token's k best lies among its half's k best, so the merge is exact.
  float* cand_v = logit_s + MAXT * MAXE;                  // [MAXT][2][MAXK]
  int* cand_i = reinterpret_cast<int*>(cand_v + MAXT * 2 * MAXK);
  const int half = (a.E + 1) / 2;
  if (warp < 2 * a.T) {
    const int t = warp >> 1, hf = warp & 1;
    const int lo = hf * half, hi = min(a.E, lo + half);
    float v[MAXE / 64];
    uint32_t taken = 0;
#pragma unroll
    for (int i = 0; i < MAXE / 64; ++i) {
      const int e = lo + lane + 32 * i;
      v[i] = -INFINITY;
      if (e < hi) v[i] = logit_s[t * a.E + e];
      else taken |= 1u << i;
    }
    for (int j = 0; j < a.k; ++j) {
      float best = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < MAXE / 64; ++i) {
        if (!((taken >> i) & 1u)) {
          const float c = (v[i] != v[i]) ? -INFINITY : v[i];
          const int e = lo + lane + 32 * i;
          if (c > best || (c == best && e < bi)) {
            best = c;
            bi = e;
          }
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, best, off);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
        if (ob > best || (ob == best && oi < bi)) {
          best = ob;
          bi = oi;
        }
      }
      if (bi != 0x7fffffff && ((bi - lo) & 31) == lane) taken |= 1u << ((bi - lo) >> 5);
      if (lane == 0) {
        cand_v[(t * 2 + hf) * MAXK + j] = best;
        cand_i[(t * 2 + hf) * MAXK + j] = bi;
      }
    }
  }
  __syncthreads();
  if (warp < a.T) {
    const int t = warp;
    // the 2k candidates, lane l holding numbers l and l + 32 (candidate c is
    // number c of the first half's list for c < k, else c - k of the second)
    float cv[2];
    int ci[2];
    bool taken[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int c = lane + 32 * u;
      cv[u] = -INFINITY;
      ci[u] = 0x7fffffff;
      if (c < 2 * a.k) {
        const int hf = c < a.k ? 0 : 1, j = c < a.k ? c : c - a.k;
        cv[u] = cand_v[(t * 2 + hf) * MAXK + j];
        ci[u] = cand_i[(t * 2 + hf) * MAXK + j];
      }
      taken[u] = ci[u] == 0x7fffffff;
    }
    float my_v = 0.f, top = 0.f;
    int my_i = 0;
    for (int j = 0; j < a.k; ++j) {
      float best = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (!taken[u] && (cv[u] > best || (cv[u] == best && ci[u] < bi))) {
          best = cv[u];
          bi = ci[u];
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, best, off);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
        if (ob > best || (ob == best && oi < bi)) {
          best = ob;
          bi = oi;
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u)
        if (!taken[u] && ci[u] == bi) taken[u] = true;
      if (j == 0) top = best;
      if (lane == j) {
        my_v = best;
        my_i = bi;
      }
    }
    const float ex = (lane < a.k) ? expf(my_v - top) : 0.f;
    float sum = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (lane < a.k) {
      R.ids[t * a.k + lane] = my_i;
      R.w[t * a.k + lane] = ex / sum;
      if (blockIdx.x == 0) {
        if (a.ids_out) a.ids_out[t * a.k + lane] = my_i;
        if (a.w_out) a.w_out[t * a.k + lane] = ex / sum;
      }
    }
  }
  __syncthreads();
  // counts per expert and the rank of each slot among the slots of its expert
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
    int c = 0;
    for (int s = 0; s < S; ++s) c += R.ids[s] == e;
    R.counts[e] = c;
    R.offsets[e] = c;
  }
  __syncthreads();
  df_block_scan(R.offsets, a.E, R.misc + 1);
  if (threadIdx.x == 0) R.offsets[a.E] = S;
  // active experts in ascending order: scan of the flags, then scatter
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) R.pos[e] = R.counts[e] > 0;
  __syncthreads();
  const int na = df_block_scan(R.pos, a.E, R.misc + 1);
  for (int e = threadIdx.x; e < a.E; e += blockDim.x)
    if (R.counts[e] > 0) R.active[R.pos[e]] = e;
  if (threadIdx.x == 0) R.misc[0] = na;
  for (int s = threadIdx.x; s < S; s += blockDim.x) {
    const int e = R.ids[s];
    int rank = 0;
    for (int s2 = 0; s2 < s; ++s2) rank += R.ids[s2] == e;
    const int row = R.offsets[e] + rank;
    R.slotrow[s] = row;
    R.rowtok[row] = s / a.k;
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------
// GEMM building blocks (one warp, 16 weight rows g and g + 8, one block of
// KB = 64 or 32 K).  Lane (g, t) holds K [t KB / 4, (t + 1) KB / 4) of the
// block: KB / 32 packed words per row, and KB / 8 registers of the token
// operand (pairs (i, i + 4) within each group of 8, the interleaved order).

// Eight int4 codes (one packed word, K order 0..7) as four exact fp16 pairs
// (i, i + 4): the mask-and-xor sets the exponent of 1024 and flips the
// code's sign bit (1024 + q + 8), codes 1, 3, 5, 7 come from bits 4..7 at
// 16x (exact: 16 (q + 8) <= 240 fits the mantissa) and the fma scales them
// back; one fma per pair removes the offset.
__device__ __forceinline__ void df_word(uint32_t w, uint32_t (&p)[4]) {
  const uint32_t w8 = w >> 8;
  const uint32_t v0 = (w & 0x000F000Fu) ^ 0x64086408u;
  const uint32_t v1 = (w & 0x00F000F0u) ^ 0x64806480u;
  const uint32_t v2 = (w8 & 0x000F000Fu) ^ 0x64086408u;
  const uint32_t v3 = (w8 & 0x00F000F0u) ^ 0x64806480u;
  // 1.0, -1032 and 1/16, -72 (fp16 pairs)
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(p[0]) : "r"(v0), "r"(0x3C003C00u), "r"(0xE408E408u));
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(p[1]) : "r"(v1), "r"(0x2C002C00u), "r"(0xD480D480u));
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(p[2]) : "r"(v2), "r"(0x3C003C00u), "r"(0xE408E408u));
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(p[3]) : "r"(v3), "r"(0x2C002C00u), "r"(0xD480D480u));
}

__device__ __forceinline__ void df_mma(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                       uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Sums of one block: c[0..1] rows g, cols 2t, 2t + 1; c[2..3] row g + 8.
template <int KB>
__device__ __forceinline__ void df_block(const uint32_t* w0, const uint32_t* w8, const uint32_t* b,
                                         float (&c)[4]) {
  c[0] = c[1] = c[2] = c[3] = 0.f;
#pragma unroll
  for (int i = 0; i < KB / 32; ++i) {
    uint32_t p0[4], p8[4];
    df_word(w0[i], p0);
    df_word(w8[i], p8);
    df_mma(c, p0[0], p8[0], p0[1], p8[1], b[4 * i + 0], b[4 * i + 1]);
    df_mma(c, p0[2], p8[2], p0[3], p8[3], b[4 * i + 2], b[4 * i + 3]);
  }
}

// Packed words of rows g and g + 8 for lane t: the tile holds `rows` rows of
// 128 bytes (one TMA box, 128-byte swizzle); `o` is the lane's byte offset
// in the row (a multiple of 4, of 8 when KB = 64).
template <int KB>
__device__ __forceinline__ void df_words(const uint8_t* tile, int g, int o, uint32_t* w0,
                                         uint32_t* w8) {
  const int sw = (((o >> 4) ^ (g & 7)) << 4) | (o & 15);
  const uint8_t* r0 = tile + g * 128 + sw;
  const uint8_t* r8 = r0 + 8 * 128;
  if (KB == 64) {
    const uint2 u0 = *reinterpret_cast<const uint2*>(r0);
    const uint2 u8 = *reinterpret_cast<const uint2*>(r8);
    w0[0] = u0.x; w0[1] = u0.y;
    w8[0] = u8.x; w8[1] = u8.y;
  } else {
    w0[0] = *reinterpret_cast<const uint32_t*>(r0);
    w8[0] = *reinterpret_cast<const uint32_t*>(r8);
  }
}

// KB / 8 registers of the token operand from a row of fp16 values.
template <int KB>
__device__ __forceinline__ void df_bfrag(const uint16_t* p, uint32_t* b) {
  const uint4 v = *reinterpret_cast<const uint4*>(p);
  b[0] = v.x; b[1] = v.y; b[2] = v.z; b[3] = v.w;
  if (KB == 64) {
    const uint4 u = *reinterpret_cast<const uint4*>(p + 8);
    b[4] = u.x; b[5] = u.y; b[6] = u.z; b[7] = u.w;
  }
}

__device__ __forceinline__ float df_half(const uint16_t* p) {
  return __half2float(__ushort_as_half(*p));
}

// Feature f's position in a row whose features are interleaved within groups
// of 8 (0, 4, 1, 5, 2, 6, 3, 7).
__device__ __forceinline__ int df_ilv(int f) {
  const int i = f & 7;
  return (f & ~7) | (i < 4 ? 2 * i : 2 * (i - 4) + 1);
}

// ---------------------------------------------------------------------------
template <int G>
__global__ void __launch_bounds__(df::THREADS, 2)
    moe_decode_fused_kernel(const __grid_constant__ CUtensorMap map_wg,
                            const __grid_constant__ CUtensorMap map_wu,
                            const __grid_constant__ CUtensorMap map_wd,
                            const __grid_constant__ CUtensorMap map_h,
                            const __grid_constant__ CUtensorMap map_sg,
                            const __grid_constant__ CUtensorMap map_su,
                            const __grid_constant__ CUtensorMap map_sd, const FusedArgs a) {
  using namespace df;
  constexpr int KB = G < 64 ? G : 64;      // K per block: one block lies in one scale group
  extern __shared__ uint8_t df_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(df_smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const Smem L = Smem::of(a.T, a.d);
  uint8_t* ring = smem + L.ring;
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem + L.x);
  float* red = reinterpret_cast<float*>(smem + L.red);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + ST;
  volatile int* flag = reinterpret_cast<volatile int*>(empty + ST);      // grid barrier result
  volatile int* abort_flag = flag + 1;
  Route R;
  {
    int32_t* r = reinterpret_cast<int32_t*>(smem + L.route);
    R.ids = r;
    R.w = reinterpret_cast<float*>(r + MAXS);
    R.counts = r + 2 * MAXS;
    R.active = R.counts + MAXE;
    // after the P1 logits and the top-k candidates
    R.pos = reinterpret_cast<int32_t*>(ring) + MAXT * MAXE + 2 * MAXT * 2 * MAXK;
    R.offsets = R.active + MAXE;
    R.rowtok = R.offsets + MAXE + 1;
    R.slotrow = R.rowtok + MAXS;
    R.misc = R.slotrow + MAXS;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g8 = lane >> 2, t = lane & 3;
  const int XP = a.d + 8;                   // halves per x row in shared memory

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], CONS);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == CONS && lane == 0) {
    prefetch_tmap(&map_wg);
    prefetch_tmap(&map_wu);
    prefetch_tmap(&map_wd);
    prefetch_tmap(&map_h);
    prefetch_tmap(&map_sg);
    prefetch_tmap(&map_su);
    prefetch_tmap(&map_sd);
  }
  // ---- P0: x in fp16 (this CTA's copy), router partials (shared work)
  if (df_load_x(a, xs)) atomicOr(a.err, kErrRange);
  __syncthreads();
  df_router_partials(a, reinterpret_cast<float*>(ring));
  bool ok = df_sync_grid(a.sync, 0, a.err, flag, abort_flag);
  if (ok) df_logits(a);
  ok = df_sync_grid(a.sync, 1, a.err, flag, abort_flag) && ok;
  // ---- P1: routes and grouping, in every CTA
  if (ok) df_route(a, R, reinterpret_cast<float*>(ring));
  // the ring held generic-proxy data (P0, P1); the TMA writes into it next
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  const int n_active = ok ? R.misc[0] : 0;
  const int S = a.T * a.k;

  uint32_t g = 0;                           // ring stage counter (both phases)
  // ---- P2: gate/up + SwiGLU, units (expert, 16 rows)
  const int FB2 = a.n / P2_ROWS, KS2 = a.d / P2_KST;
  const int units2 = n_active * FB2;
  if (warp == CONS) {
    if (lane == 0) {
      bool stop = false;
      // stage q of this CTA's gate/up stream: unit blockIdx.x + (q / KS2) * gridDim.x, K block q % KS2
      auto prefetch2 = [&](int q) {
        const int u = blockIdx.x + (q / KS2) * (int)gridDim.x;
        if (u >= units2) return;
        const int kc = q % KS2;
        const int wrow = R.active[u / FB2] * a.n + (u % FB2) * P2_ROWS;
#pragma unroll
        for (int b = 0; b < P2_KST / 256; ++b) {
          tma_prefetch_2d(&map_wg, kc * (P2_KST / 2) + b * 128, wrow);
          tma_prefetch_2d(&map_wu, kc * (P2_KST / 2) + b * 128, wrow);
        }
        tma_prefetch_2d(&map_sg, kc * (P2_KST / G), wrow);
        tma_prefetch_2d(&map_su, kc * (P2_KST / G), wrow);
      };
      for (int q = 0; q < PF; ++q) prefetch2(q);
      int q2 = 0;
      for (int u = blockIdx.x; u < units2 && !stop; u += gridDim.x) {
        const int e = R.active[u / FB2];
        const int wrow = e * a.n + (u % FB2) * P2_ROWS;
        for (int kc = 0; kc < KS2; ++kc, ++g, ++q2) {
          prefetch2(q2 + PF);
          const int s = g % ST;
          if (g >= (uint32_t)ST &&
              !mbar_wait(&empty[s], ((g / ST) - 1) & 1, abort_flag, a.err)) {
            stop = true;
            break;
          }
          uint8_t* sl = ring + s * SLOT;
          constexpr int SG = P2_ROWS * (P2_KST / G) * 2;   // scale bytes per matrix
          mbar_arrive_expect_tx(&full[s], 2 * P2_ROWS * (P2_KST / 2) + 2 * SG);
#pragma unroll
          for (int b = 0; b < P2_KST / 256; ++b) {
            tma_load_2d(sl + b * 2048, &map_wg, kc * (P2_KST / 2) + b * 128, wrow, &full[s]);
            tma_load_2d(sl + 8192 + b * 2048, &map_wu, kc * (P2_KST / 2) + b * 128, wrow,
                        &full[s]);
          }
          tma_load_2d(sl + P2_SC, &map_sg, kc * (P2_KST / G), wrow, &full[s]);
          tma_load_2d(sl + P2_SC + SG, &map_su, kc * (P2_KST / G), wrow, &full[s]);
        }
      }
    }
  } else {
    const int ks = warp;                    // this warp's 128 K of each stage
    constexpr int SGR = P2_KST / G;         // scale groups per row in a stage
    for (int u = blockIdx.x; u < units2; u += gridDim.x) {
      const int e = R.active[u / FB2], fb = u % FB2;
      const int cnt = R.counts[e], prow = R.offsets[e];
      const int tok = R.rowtok[prow + min(g8, cnt - 1)];
      const uint16_t* xr = xs + (size_t)tok * XP;
      float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      bool failed = false;
      for (int kc = 0; kc < KS2; ++kc, ++g) {
        const int s = g % ST;
        if (!mbar_wait_warp(&full[s], (g / ST) & 1, abort_flag, a.err)) {
          failed = true;
          break;
        }
        const uint8_t* sl = ring + s * SLOT;
        const int k0 = kc * P2_KST + ks * 128;          // first K of this warp's range
#pragma unroll
        for (int bi = 0; bi < 128 / KB; ++bi) {
          const int kb = k0 + bi * KB;
          uint32_t b[KB / 8];
          df_bfrag<KB>(xr + kb + t * (KB / 4), b);
          const int grp = (ks * 128 + bi * KB) / G;       // scale group within the stage
          const int o = (ks & 1) * 64 + (bi * KB + t * (KB / 4)) / 2;   // byte in the box row
#pragma unroll
          for (int m = 0; m < 2; ++m) {
            const uint8_t* tile = sl + m * 8192 + (ks >> 1) * 2048;
            uint32_t w0[KB / 32], w8[KB / 32];
            df_words<KB>(tile, g8, o, w0, w8);
            float c[4];
            df_block<KB>(w0, w8, b, c);
            const uint16_t* sp = reinterpret_cast<const uint16_t*>(sl + P2_SC) +
                                 m * P2_ROWS * SGR + g8 * SGR + grp;
            const float s0 = df_half(sp);
            const float s8 = df_half(sp + 8 * SGR);
            acc[m][0] = fmaf(s0, c[0], acc[m][0]);
            acc[m][1] = fmaf(s0, c[1], acc[m][1]);
            acc[m][2] = fmaf(s8, c[2], acc[m][2]);
            acc[m][3] = fmaf(s8, c[3], acc[m][3]);
          }
        }
        fence_proxy_async_smem();           // this stage's loads before its next TMA write
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
      // the 8 warps' sums of the unit meet in shared memory (fixed order)
      float4* rp = reinterpret_cast<float4*>(red + (warp * 32 + lane) * 8);
      rp[0] = make_float4(acc[0][0], acc[0][1], acc[0][2], acc[0][3]);
      rp[1] = make_float4(acc[1][0], acc[1][1], acc[1][2], acc[1][3]);
      if (named_barrier_or(1, CONS * 32, failed || *abort_flag)) break;   // all warps alike
      if (threadIdx.x < P2_ROWS * 8) {
        const int r = threadIdx.x >> 3, col = threadIdx.x & 7;
        const int ln = (r & 7) * 4 + (col >> 1), reg = (r >> 3) * 2 + (col & 1);
        float gs = 0.f, us = 0.f;
        for (int w = 0; w < CONS; ++w) {
          gs += red[(w * 32 + ln) * 8 + reg];
          us += red[(w * 32 + ln) * 8 + 4 + reg];
        }
        if (col < cnt) {
          const float hv = gs / (1.0f + __expf(-gs)) * us;
          if (f16_overflows(hv)) atomicOr(a.err, kErrRange);
          a.h[(size_t)(prow + col) * a.n + df_ilv(fb * P2_ROWS + r)] = f16_bits(hv);
        }
      }
      named_barrier_sync(1, CONS * 32);     // red is reused by the next unit
    }
  }
  ok = df_sync_grid(a.sync, 2, a.err, flag, abort_flag) && ok;

  // ---- P3: down, units (expert, 64 rows): 4 row groups x 2 K halves
  const int FB3 = a.d / P3_ROWS, KS3 = a.n / P3_KST;
  const int units3 = ok ? n_active * FB3 : 0;
  if (warp == CONS) {
    if (lane == 0) {
      bool stop = false;
      auto prefetch3 = [&](int q) {
        const int u = blockIdx.x + (q / KS3) * (int)gridDim.x;
        if (u >= units3) return;
        const int kc = q % KS3;
        const int e = R.active[u / FB3];
        const int wrow = e * a.d + (u % FB3) * P3_ROWS;
        tma_prefetch_2d(&map_wd, kc * (P3_KST / 2), wrow);
        if (kc == 0) tma_prefetch_2d(&map_sd, 0, wrow);
      };
      for (int q = 0; q < PF; ++q) prefetch3(q);
      int q3 = 0;
      for (int u = blockIdx.x; u < units3 && !stop; u += gridDim.x) {
        const int e = R.active[u / FB3];
        const int wrow = e * a.d + (u % FB3) * P3_ROWS;
        const int prow = R.offsets[e];
        for (int kc = 0; kc < KS3; ++kc, ++g, ++q3) {
          prefetch3(q3 + PF);
          const int s = g % ST;
          if (g >= (uint32_t)ST &&
              !mbar_wait(&empty[s], ((g / ST) - 1) & 1, abort_flag, a.err)) {
            stop = true;
            break;
          }
          uint8_t* sl = ring + s * SLOT;
          mbar_arrive_expect_tx(&full[s], P3_ROWS * (P3_KST / 2) + MAXT * P3_KST * 2 +
                                              P3_ROWS * (a.n / G) * 2);
          tma_load_2d(sl, &map_wd, kc * (P3_KST / 2), wrow, &full[s]);
          tma_load_2d(sl + P3_H, &map_h, kc * P3_KST, prow, &full[s]);
          tma_load_2d(sl + P3_SC, &map_sd, 0, wrow, &full[s]);     // the unit's scale rows
        }
      }
    }
  } else {
    const int rg = warp & 3, kh = warp >> 2;
    const int NG = a.n / G;                 // scale groups per down row
    for (int u = blockIdx.x; u < units3; u += gridDim.x) {
      const int e = R.active[u / FB3], fb = u % FB3;
      const int cnt = R.counts[e], prow = R.offsets[e];
      const int hrow = g8 < cnt ? g8 : 0;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      bool failed = false;
      for (int kc = 0; kc < KS3; ++kc, ++g) {
        const int s = g % ST;
        if (!mbar_wait_warp(&full[s], (g / ST) & 1, abort_flag, a.err)) {
          failed = true;
          break;
        }
        const uint8_t* sl = ring + s * SLOT;
        const uint16_t* hr = reinterpret_cast<const uint16_t*>(sl + P3_H) + hrow * P3_KST;
        const uint16_t* sc = reinterpret_cast<const uint16_t*>(sl + P3_SC) + (rg * 16 + g8) * NG;
        const uint8_t* tile = sl + rg * 16 * 128;
#pragma unroll
        for (int bi = 0; bi < 128 / KB; ++bi) {
          const int kl = kh * 128 + bi * KB;               // K within the stage
          uint32_t b[KB / 8];
          df_bfrag<KB>(hr + kl + t * (KB / 4), b);
          uint32_t w0[KB / 32], w8[KB / 32];
          df_words<KB>(tile, g8, (kl + t * (KB / 4)) / 2, w0, w8);
          float c[4];
          df_block<KB>(w0, w8, b, c);
          const int grp = (kc * P3_KST + kl) / G;
          const float s0 = df_half(sc + grp);
          const float s8 = df_half(sc + 8 * NG + grp);
          acc[0] = fmaf(s0, c[0], acc[0]);
          acc[1] = fmaf(s0, c[1], acc[1]);
          acc[2] = fmaf(s8, c[2], acc[2]);
          acc[3] = fmaf(s8, c[3], acc[3]);
        }
        fence_proxy_async_smem();           // this stage's loads before its next TMA write
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
      // second K half hands its sums to the first (fixed order: first + second)
      float4* rp = reinterpret_cast<float4*>(red + (rg * 32 + lane) * 4);
      if (kh == 1) *rp = make_float4(acc[0], acc[1], acc[2], acc[3]);
      if (named_barrier_or(1, CONS * 32, failed || *abort_flag)) break;   // all warps alike
      if (kh == 0) {
        const float4 o = *rp;
        const float v[4] = {acc[0] + o.x, acc[1] + o.y, acc[2] + o.z, acc[3] + o.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int col = 2 * t + (q & 1);
          const int feat = fb * P3_ROWS + rg * 16 + g8 + (q >> 1) * 8;
          if (col < cnt) a.rows[(size_t)(prow + col) * a.d + feat] = v[q];
        }
      }
      named_barrier_sync(1, CONS * 32);
    }
  }
  ok = df_sync_grid(a.sync, 3, a.err, flag, abort_flag) && ok;

  // ---- P4: combine, fp32 in slot order j = 0 .. k-1, one rounding to bf16
  if (ok) {
    const int cpr = a.d / 8;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < a.T * cpr; i += gridDim.x * blockDim.x) {
      const int tk = i / cpr, f0 = (i % cpr) * 8;
      float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int j = 0; j < a.k; ++j) {
        const int sl = tk * a.k + j;
        const float w = R.w[sl];
        const float4* rp = reinterpret_cast<const float4*>(a.rows + (size_t)R.slotrow[sl] * a.d + f0);
        const float4 r0 = __ldcg(rp), r1 = __ldcg(rp + 1);
        v[0] = fmaf(w, r0.x, v[0]); v[1] = fmaf(w, r0.y, v[1]);
        v[2] = fmaf(w, r0.z, v[2]); v[3] = fmaf(w, r0.w, v[3]);
        v[4] = fmaf(w, r1.x, v[4]); v[5] = fmaf(w, r1.y, v[5]);
        v[6] = fmaf(w, r1.z, v[6]); v[7] = fmaf(w, r1.w, v[7]);
      }
      uint4 o;
      o.x = pack_bf16x2(v[0], v[1]);
      o.y = pack_bf16x2(v[2], v[3]);
      o.z = pack_bf16x2(v[4], v[5]);
      o.w = pack_bf16x2(v[6], v[7]);
      *reinterpret_cast<uint4*>(a.y + (size_t)tk * a.d + f0) = o;
    }
  }
  (void)S;
}

// ---------------------------------------------------------------------------
bool decode_fused_fits(int T, int d, int E, int k, int n, int G) {
  using namespace df;
  if (T < 1 || T > MAXT || k > MAXK || E > MAXE) return false;
  if (G != 32 && G != 64 && G != 128) return false;
  if (d % P2_KST || d % P0_RS || d / P0_RS > P0_MAXKS || n % P3_KST || n % P2_ROWS ||
      d % P3_ROWS || E % 8 || T * d > 8 * XPT * THREADS)
    return false;
  // scale tiles by TMA: rows of at least 16 bytes, at most 256 groups, fitting the stage
  if ((P2_KST / G) % 8 || (n / G) % 8 || n / G > 256 || P3_SC + P3_ROWS * (n / G) * 2 > SLOT)
    return false;
  return Smem::of(T, d).total + 1024 <= 113 * 1024;
}

size_t decode_fused_scratch(int T, int d, int E, int k, int n) {
  // partial logits, h, rows, sync words (each region 256-byte aligned)
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t S = (size_t)T * k;
  return up((size_t)(d / df::P0_RS) * T * E * 4) + up((size_t)T * E * 4) + up(S * n * 2) +
         up(S * d * 4) + 256;
}

template <int G>
static cudaError_t launch_fused_g(const CUtensorMap* maps, const FusedArgs& a, int smem,
                                  cudaStream_t s) {
  auto kern = moe_decode_fused_kernel<G>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, df::THREADS, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorNotSupported;
  if (per_sm > 2) per_sm = 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(per_sm * sm_count()));
  cfg.blockDim = dim3(df::THREADS);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, maps[0], maps[1], maps[2], maps[3], maps[4], maps[5],
                            maps[6], a);
}

cudaError_t launch_decode_fused(const uint16_t* x, const uint16_t* w_router, const float* bias,
                                const uint8_t* q_gate, const uint16_t* s_gate,
                                const uint8_t* q_up, const uint16_t* s_up,
                                const uint8_t* q_down, const uint16_t* s_down, int T, int d,
                                int E, int k, int n, int G, uint16_t* y, int32_t* ids_out,
                                float* w_out, void* scratch, unsigned* err, cudaStream_t s) {
  using namespace df;
  if (!decode_fused_fits(T, d, E, k, n, G)) return cudaErrorNotSupported;
  auto up = [](size_t v) { return (v + 255) & ~size_t(255); };
  const size_t S = (size_t)T * k;
  uint8_t* base = static_cast<uint8_t*>(scratch);
  FusedArgs a;
  a.x = x;
  a.w_router = w_router;
  a.bias = bias;
  a.s_gate = s_gate;
  a.s_up = s_up;
  a.s_down = s_down;
  a.y = y;
  a.ids_out = ids_out;
  a.w_out = w_out;
  a.partial = reinterpret_cast<float*>(base);
  base += up((size_t)(d / P0_RS) * T * E * 4);
  a.logits = reinterpret_cast<float*>(base);
  base += up((size_t)T * E * 4);
  a.h = reinterpret_cast<uint16_t*>(base);
  base += up(S * n * 2);
  a.rows = reinterpret_cast<float*>(base);
  base += up(S * d * 4);
  a.sync = reinterpret_cast<unsigned*>(base);
  a.err = err;
  a.T = T;
  a.d = d;
  a.E = E;
  a.k = k;
  a.n = n;
  a.G = G;
  CUtensorMap maps[7];
  if (encode_tmap_2d(&maps[0], CU_TENSOR_MAP_DATA_TYPE_UINT8, q_gate, d / 2, (uint64_t)E * n, d / 2,
                     128, P2_ROWS, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B) != CUDA_SUCCESS ||
      encode_tmap_2d(&maps[1], CU_TENSOR_MAP_DATA_TYPE_UINT8, q_up, d / 2, (uint64_t)E * n, d / 2,
                     128, P2_ROWS, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B) != CUDA_SUCCESS ||
      encode_tmap_2d(&maps[2], CU_TENSOR_MAP_DATA_TYPE_UINT8, q_down, n / 2, (uint64_t)E * d, n / 2,
                     128, P3_ROWS, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B) != CUDA_SUCCESS ||
      encode_tmap_2d(&maps[3], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a.h, n, S, (uint64_t)n * 2, P3_KST,
                     MAXT, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_128B) != CUDA_SUCCESS ||
      // scales: gate/up 1024 / G groups x 16 rows per stage, down n / G groups
      // x 64 rows (a unit's whole scale rows) per stage
      encode_tmap_2d(&maps[4], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, s_gate, d / G, (uint64_t)E * n,
                     (uint64_t)(d / G) * 2, P2_KST / G, P2_ROWS, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_128B) != CUDA_SUCCESS ||
      encode_tmap_2d(&maps[5], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, s_up, d / G, (uint64_t)E * n,
                     (uint64_t)(d / G) * 2, P2_KST / G, P2_ROWS, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_128B) != CUDA_SUCCESS ||
      encode_tmap_2d(&maps[6], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, s_down, n / G, (uint64_t)E * d,
                     (uint64_t)(n / G) * 2, n / G, P3_ROWS, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  cudaError_t e = cudaMemsetAsync(a.sync, 0, 16, s);
  if (e != cudaSuccess) return e;
  const int smem = Smem::of(T, d).total + 1024;
  if (G == 32) return launch_fused_g<32>(maps, a, smem, s);
  if (G == 64) return launch_fused_g<64>(maps, a, smem, s);
  return launch_fused_g<128>(maps, a, smem, s);
}

}  // namespace strata
