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
// through five phases, separated by grid-wide barriers or per-expert
// counters with bounded waits:
//
//   P0  router partial logits (items of 128 rows of W_r x 64 experts);
//       every CTA also converts x of all tokens to fp16 in shared memory;
//   --- grid barrier
//   P0b the logits, each summed once from the partials (spread over CTAs);
//   --- grid barrier
//   P1  every CTA reads the logits, picks each token's top k (exact ties to
//       the lower expert index), the softmax weights, and groups the T*k
//       slots by expert (active experts, counts, first rows, stable order)
//       in its own shared memory: same inputs, same code, same result in
//       every CTA, so no barrier follows;
//   P2  gate/up + SwiGLU: units of 16 weight rows of one expert, K split
//       over the 8 consumer warps, both matrices streamed by TMA through a
//       3-deep ring, B operand = x from shared memory; h to global (fp16);
//       each stored unit adds one to its expert's counter;
//   P3  down: units of 64 rows of one expert (4 row groups x 2 K halves),
//       each stage carries the expert's h rows, loaded once the expert's
//       counter shows all of its gate/up units (a CTA starts its down units
//       while others still finish gate/up ones); output rows to global
//       (fp32); each stored unit adds one to a count of finished units;
//   P4  combine: y_t = sum_j w_tj * row_(t,j), fp32 in slot order, bf16, in
//       the CTAs that have combine items, once the count shows every down
//       unit (the other CTAs end after P3).
//
// Warp roles in P2 and P3: one producer warp (TMA), eight consumer warps
// (matrix products) and one reducer warp.  The units are handed out
// dynamically (a grid-wide counter, fetched one unit ahead by the producer),
// so a CTA that streams faster takes more of them.  Consumer warps pass each
// unit's partial sums to the reducer through a double buffer and go on to
// the next unit at once; the reducer adds the warps' sums in a fixed order,
// applies SwiGLU (P2) and stores.  Results do not depend on which CTA took
// a unit.
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
constexpr int THREADS = (CONS + 2) * 32;  // + one producer warp + one reducer warp
constexpr int ST = 3;                     // ring stages
// A ring stage: gate/up: 16 rows x 1024 K of both matrices (16 KB) and their
// scales (16 rows x 1024 / G groups each, at most 2 KB); down: 64 rows x
// 256 K (8 KB), the expert's h rows (2 KB) and the unit's scale rows
// (64 rows x n / G groups, at most 4 KB).
constexpr int SLOT = 18432;               // bytes per ring stage
constexpr int P2_SC = 16384;              // offset of the gate/up scales in a stage
constexpr int P3_H = 8192, P3_SC = 10240; // offsets of h and of the down scales
constexpr int P2_ROWS = 16;               // gate/up unit: 16 rows, K split 8 ways
constexpr int P2_KST = 1024;              // gate/up K per stage
constexpr int P3_ROWS = 64;               // down unit: 4 row groups x 2 K halves
constexpr int P3_KST = 256;               // down K per stage
constexpr int P0_RS = 128;                // router rows per item
constexpr int P0_MAXKS = 32;              // router K slices (d <= 4096)
constexpr int XPT = 8;                    // 16-byte chunks of x per thread (T * d <= 8 * 8 * THREADS)
constexpr int LPT = 16;                   // logits per thread in P1 (T * E <= 16 * THREADS)
constexpr int MAXE = 1024, MAXK = 32;
constexpr int MAXS = MAXT * MAXK;
// A hand-off buffer to the reducer: [consumer warp][lane (g, t < 2)][8] fp32
// (gate/up: rows g, g + 8 of gate then up, tokens 2t, 2t + 1; down: the first
// four).  Lanes with t >= 2 hold tokens 4..7, which never exist here.
constexpr int RED_BUF = CONS * 16 * 8;

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
    s.red = s.x + xb;                            // two hand-off buffers
    s.bars = s.red + 2 * RED_BUF * 4;
    s.route = s.bars + 128;
    // ids, w, active, acnt, aoff, first, rowtok, slotrow [MAXS]; misc [64]
    s.total = s.route + (8 * MAXS + 64) * 4;
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
  unsigned* sync;            // zeroed before the launch: [0] barrier arrivals,
                             // [2] abort, [4] / [5] gate-up / down unit counters,
                             // [6] down units done,
                             // [64 + i] gate/up units of active expert i done
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

// ---------------------------------------------------------------------------
// P0: partial router logits.  Item = (128 rows of W_r, 64 experts): thread
// (row group rr = th / 8 of 32, 16-byte chunk c = th % 8 of 8 experts) loads
// the chunk of rows rr, rr + 32, rr + 64, rr + 96 at once, then x of the
// item's rows is staged in shared memory as fp32, and the 32 row groups'
// products are added in a fixed order.  Uses threads 0..255.
//   scratch: >= 32 * MAXT * 64 + MAXT * P0_RS floats
__device__ void df_router_partials(const FusedArgs& a, float* scratch) {
  using namespace df;
  constexpr int RPT = P0_RS / 32;                         // rows per thread
  const int th = threadIdx.x;
  const int neb = (a.E + 63) / 64, nks = a.d / P0_RS;
  float* red = scratch;                                   // [32][MAXT][64]
  float* xr = scratch + 32 * MAXT * 64;                   // [MAXT][P0_RS]
  const int c = th & 7, rr = th >> 3;
  for (int item = blockIdx.x; item < neb * nks; item += gridDim.x) {
    const int eb = item % neb, ks = item / neb;
    const int r0 = ks * P0_RS;
    const int e0 = eb * 64 + c * 8;
    const bool live = th < 256 && e0 < a.E;               // E % 8 == 0 on this path
    uint4 w[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i)
      if (live) w[i] = ld_nc_v4(a.w_router + (size_t)(r0 + rr + 32 * i) * a.E + e0);
    if (th < a.T * (P0_RS / 8)) {                         // one 16-byte chunk of x per thread
      const int t = th / (P0_RS / 8), j = th % (P0_RS / 8);
      const uint4 v = ld_nc_v4(a.x + (size_t)t * a.d + r0 + 8 * j);
      float* dst = xr + t * P0_RS + 8 * j;
      dst[0] = bf16_lo(v.x); dst[1] = bf16_hi(v.x); dst[2] = bf16_lo(v.y); dst[3] = bf16_hi(v.y);
      dst[4] = bf16_lo(v.z); dst[5] = bf16_hi(v.z); dst[6] = bf16_lo(v.w); dst[7] = bf16_hi(v.w);
    }
    __syncthreads();
    if (th < 256) {
      float acc[MAXT][8];
#pragma unroll
      for (int t = 0; t < MAXT; ++t)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[t][j] = 0.f;
      if (live) {
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
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
      for (int gi = 0; gi < 32; ++gi) sum += red[(gi * MAXT + t) * 64 + l];
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
  int32_t* ids;      // [S] expert of each slot
  float* w;          // [S] its softmax weight
  int32_t* active;   // [n_active] experts with at least one slot, ascending
  int32_t* acnt;     // [n_active] their slot counts
  int32_t* aoff;     // [n_active] their first grouped row
  int32_t* first;    // [S] scratch: slot is its expert's first
  int32_t* rowtok;   // [S] grouped row -> token
  int32_t* slotrow;  // [S] slot -> grouped row
  int* misc;         // [0] n_active
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

// Order-preserving 32-bit key of a logit: larger float, larger key; NaN maps
// to the key of -inf and -0 to that of +0 (so they compare as the float
// comparison treats them in the selection).
__device__ __forceinline__ uint32_t df_order_key(float f) {
  if (f != f) f = -INFINITY;
  if (f == 0.f) f = 0.f;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float df_key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Top k of token t by one warp: lane l holds experts l, l + 32, ... (NV per
// lane, E <= 32 NV) as order-preserving keys (NaN as -inf, -0 as +0; absent
// entries as 0, below every key).  Each round every lane offers
// its best entry (largest key, then lowest index), the warp takes the
// largest key and, among the lanes offering it, the lowest expert index (two
// warp reductions), and the owning lane marks that entry taken: exact ties go
// to the lower expert index and NaN never wins.  Then the softmax over the k.
template <int NV>
__device__ __forceinline__ void df_topk(const FusedArgs& a, const Route& R, const float* logit_s,
                                        int t, int lane) {
  uint32_t key[NV];
  uint32_t taken = 0;                         // entries already picked
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int e = lane + 32 * i;
    key[i] = e < a.E ? df_order_key(logit_s[t * a.E + e]) : 0u;
  }
  uint32_t my_key = 0, top = 0;
  int my_i = 0;
  for (int j = 0; j < a.k; ++j) {
    // four independent chains over i mod 4, merged in index order
    uint32_t bk[4] = {0u, 0u, 0u, 0u};
    int bs[4] = {0, 0, 0, 0};
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int c = i & 3;
      if (!((taken >> i) & 1u) && key[i] > bk[c]) {                 // the first of equal keys stays (lower index)
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
  const float my_v = df_key_value(my_key), top_v = df_key_value(top);
  const float ex = (lane < a.k) ? expf(my_v - top_v) : 0.f;
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

__device__ void df_route(const FusedArgs& a, const Route& R, float* logit_s) {
  using namespace df;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.T * a.k;
  // logits of every token (summed once, by all CTAs together, in P0b)
  {
    float v[LPT];                                      // every load first, then the stores
#pragma unroll
    for (int u = 0; u < LPT; ++u) {
      const int i = threadIdx.x + u * blockDim.x;
      v[u] = i < a.T * a.E ? __ldcg(a.logits + i) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < LPT; ++u) {
      const int i = threadIdx.x + u * blockDim.x;
      if (i < a.T * a.E) logit_s[i] = v[u];
    }
  }
  __syncthreads();
  // top k of each token by one warp (warp t)
  if (warp < a.T) {
    if (a.E <= 512) df_topk<16>(a, R, logit_s, warp, lane);
    else df_topk<MAXE / 32>(a, R, logit_s, warp, lane);
  }
  __syncthreads();
  // grouping of the S <= 128 slots by expert, slot order within an expert:
  // thread s scans the S ids once for its slot's rank among the slots of its
  // expert, the slots of lower experts (its expert's first row) and its
  // expert's count; the first slot of each expert then finds the expert's
  // place among the active experts.
  const int s = threadIdx.x;
  int e = 0, rank = 0, less = 0, cnt = 0;
  if (s < S) {
    e = R.ids[s];
    for (int s2 = 0; s2 < S; ++s2) {
      const int e2 = R.ids[s2];
      rank += (e2 == e) & (s2 < s);
      less += e2 < e;
      cnt += e2 == e;
    }
    R.slotrow[s] = less + rank;
    R.rowtok[less + rank] = s / a.k;
    R.first[s] = rank == 0;
  }
  __syncthreads();
  if (s < S && rank == 0) {
    int j = 0;
    for (int s2 = 0; s2 < S; ++s2) j += R.first[s2] & (R.ids[s2] < e);
    R.active[j] = e;
    R.acnt[j] = cnt;
    R.aoff[j] = less;
  }
  if (s == 0) {
    int na = 0;
    for (int s2 = 0; s2 < S; ++s2) na += R.first[s2];
    R.misc[0] = na;
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

// A consumer warp hands its sums of unit u (u = -1: the phase's end) to the
// reducer: hand-off number rc uses buffer rc % 2, free once the reducer has
// finished hand-off rc - 2.  Warp 0 names the unit.  Returns false if the
// wait gave up.
__device__ __forceinline__ bool df_post(float* red, uint64_t* red_full, uint64_t* red_empty,
                                        volatile int* red_unit, uint32_t& rc, int u,
                                        const float* v, volatile int* abort, unsigned* err) {
  using namespace df;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = rc & 1;
  if (rc >= 2 && !mbar_wait_warp(&red_empty[b], ((rc >> 1) - 1) & 1, abort, err)) return false;
  if (v != nullptr && (lane & 3) < 2) {
    float4* p = reinterpret_cast<float4*>(red + b * RED_BUF +
                                          (warp * 16 + (lane >> 2) * 2 + (lane & 3)) * 8);
    p[0] = make_float4(v[0], v[1], v[2], v[3]);
    p[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
  if (warp == 0 && lane == 0) red_unit[b] = u;
  __syncwarp();
  if (lane == 0) mbar_arrive(&red_full[b]);
  ++rc;
  return true;
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
  uint64_t* red_full = empty + ST;          // [2] consumer warps -> reducer
  uint64_t* red_empty = red_full + 2;       // [2] reducer -> consumer warps
  volatile int* flag = reinterpret_cast<volatile int*>(red_empty + 2);  // grid barrier result
  volatile int* abort_flag = flag + 1;
  volatile int* hdr = abort_flag + 1;       // [ST] unit of each ring stage
  volatile int* red_unit = hdr + ST;        // [2] unit of each hand-off buffer
  Route R;
  {
    int32_t* r = reinterpret_cast<int32_t*>(smem + L.route);
    R.ids = r;
    R.w = reinterpret_cast<float*>(r + MAXS);
    R.active = r + 2 * MAXS;
    R.acnt = R.active + MAXS;
    R.aoff = R.acnt + MAXS;
    R.first = R.aoff + MAXS;
    R.rowtok = R.first + MAXS;
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
    for (int b = 0; b < 2; ++b) {
      mbar_init(&red_full[b], CONS);
      mbar_init(&red_empty[b], 1);
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

  uint32_t g = 0;                           // ring stage counter (both phases)
  uint32_t rc = 0;                          // hand-off counter to the reducer (both phases)
  // Units are handed out dynamically: CTA b starts with unit b, its producer
  // then takes the next one from a grid-wide counter (fetched one unit
  // ahead) and writes each stage's unit into hdr[stage]; a stage with unit
  // -1 ends the phase.  Consumer warps hand each unit's partial sums to the
  // reducer warp through one of two buffers and go straight on to the next
  // unit; the reducer adds them in a fixed warp order and stores the results.

  // ---- P2: gate/up + SwiGLU, units (expert, 16 rows)
  const int FB2 = a.n / P2_ROWS, KS2 = a.d / P2_KST;
  const int units2 = n_active * FB2;
  if (warp == CONS) {
    if (lane == 0 && ok) {
      int u = blockIdx.x;
      for (;;) {
        const bool last = u >= units2;
        const int nx = last ? 0 : (int)gridDim.x + (int)atomicAdd(&a.sync[4], 1u);
        bool stop = false;
        const int e = last ? 0 : R.active[u / FB2];
        const int wrow = e * a.n + (u % FB2) * P2_ROWS;
        for (int kc = 0; kc < (last ? 1 : KS2); ++kc, ++g) {
          const int s = g % ST;
          if (g >= (uint32_t)ST &&
              !mbar_wait(&empty[s], ((g / ST) - 1) & 1, abort_flag, a.err)) {
            stop = true;
            break;
          }
          hdr[s] = last ? -1 : u;
          if (last) {
            mbar_arrive(&full[s]);
            continue;
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
        if (stop || last) break;
        u = nx;
      }
    }
  } else if (warp < CONS) {
    const int ks = warp;                    // this warp's 128 K of each stage
    constexpr int SGR = P2_KST / G;         // scale groups per row in a stage
    while (ok) {
      int s = g % ST;
      if (!mbar_wait_warp(&full[s], (g / ST) & 1, abort_flag, a.err)) break;
      const int u = hdr[s];
      if (u < 0) {                          // the phase's end: release the stage, tell the reducer
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        ++g;
        df_post(red, red_full, red_empty, red_unit, rc, -1, nullptr, abort_flag, a.err);
        break;
      }
      const int cnt = R.acnt[u / FB2], prow = R.aoff[u / FB2];
      const int tok = R.rowtok[prow + min(g8, cnt - 1)];
      const uint16_t* xr = xs + (size_t)tok * XP;
      float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      bool failed = false;
      for (int kc = 0; kc < KS2; ++kc, ++g) {
        s = g % ST;
        if (kc > 0 && !mbar_wait_warp(&full[s], (g / ST) & 1, abort_flag, a.err)) {
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
      if (failed) break;
      const float v[8] = {acc[0][0], acc[0][1], acc[0][2], acc[0][3],
                          acc[1][0], acc[1][1], acc[1][2], acc[1][3]};
      if (!df_post(red, red_full, red_empty, red_unit, rc, u, v, abort_flag, a.err)) break;
    }
  } else {
    // reducer: gate and up sums of 16 rows x cnt tokens; lane = (row r, token pair cp)
    const int r = lane & 15, cp = lane >> 4;
    uint32_t rr = rc;
    while (ok) {
      const int b = rr & 1;
      if (!mbar_wait_warp(&red_full[b], (rr >> 1) & 1, abort_flag, a.err)) break;
      const int u = red_unit[b];
      if (u >= 0) {
        const int fb = u % FB2;
        const int cnt = R.acnt[u / FB2], prow = R.aoff[u / FB2];
        const float* rb = red + b * RED_BUF + ((r & 7) * 2 + cp) * 8 + (r >> 3) * 2;
        float gs[2] = {0.f, 0.f}, us[2] = {0.f, 0.f};
#pragma unroll
        for (int w = 0; w < CONS; ++w) {
          const float2 gv = *reinterpret_cast<const float2*>(rb + w * 128);
          const float2 uv = *reinterpret_cast<const float2*>(rb + w * 128 + 4);
          gs[0] += gv.x; gs[1] += gv.y;
          us[0] += uv.x; us[1] += uv.y;
        }
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int col = 2 * cp + c;
          if (col < cnt) {
            const float hv = gs[c] / (1.0f + __expf(-gs[c])) * us[c];
            if (f16_overflows(hv)) atomicOr(a.err, kErrRange);
            a.h[(size_t)(prow + col) * a.n + df_ilv(fb * P2_ROWS + r)] = f16_bits(hv);
          }
        }
        // the unit's h values, then one more finished unit of the expert:
        // the down phase of any CTA may read the expert's h once all of its
        // gate/up units are counted
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(&a.sync[64 + u / FB2], 1u);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&red_empty[b]);
      ++rr;
      if (u < 0) break;
    }
    rc = rr;
  }
  // No grid barrier here: a CTA goes on to down units as soon as its own
  // gate/up work is done, and its producer waits, per unit, until every
  // gate/up unit of that unit's expert has stored its h (a counter per
  // active expert) before it loads h; the down weights of the stage are
  // already on their way by then.

  // ---- P3: down, units (expert, 64 rows): 4 row groups x 2 K halves
  const int FB3 = a.d / P3_ROWS, KS3 = a.n / P3_KST;
  const int units3 = n_active * FB3;
  if (warp == CONS) {
    if (lane == 0 && ok) {
      int u = blockIdx.x;
      for (;;) {
        const bool last = u >= units3;
        const int nx = last ? 0 : (int)gridDim.x + (int)atomicAdd(&a.sync[5], 1u);
        bool stop = false;
        const int e = last ? 0 : R.active[u / FB3];
        const int wrow = e * a.d + (u % FB3) * P3_ROWS;
        const int prow = last ? 0 : R.aoff[u / FB3];
        for (int kc = 0; kc < (last ? 1 : KS3); ++kc, ++g) {
          const int s = g % ST;
          if (g >= (uint32_t)ST &&
              !mbar_wait(&empty[s], ((g / ST) - 1) & 1, abort_flag, a.err)) {
            stop = true;
            break;
          }
          hdr[s] = last ? -1 : u;
          if (last) {
            mbar_arrive(&full[s]);
            continue;
          }
          uint8_t* sl = ring + s * SLOT;
          mbar_arrive_expect_tx(&full[s], P3_ROWS * (P3_KST / 2) + MAXT * P3_KST * 2 +
                                              P3_ROWS * (a.n / G) * 2);
          tma_load_2d(sl, &map_wd, kc * (P3_KST / 2), wrow, &full[s]);
          tma_load_2d(sl + P3_SC, &map_sd, 0, wrow, &full[s]);     // the unit's scale rows
          const bool ready =
              kc != 0 || counter_wait(&a.sync[64 + u / FB3], (unsigned)FB2, &a.sync[2], a.err,
                                      abort_flag);
          // loaded either way, so the stage's copies all complete; after a
          // wait that gave up the CTA's roles are already winding down
          tma_load_2d(sl + P3_H, &map_h, kc * P3_KST, prow, &full[s]);
          if (!ready) {
            stop = true;
            break;
          }
        }
        if (stop || last) break;
        u = nx;
      }
    }
  } else if (warp < CONS) {
    const int rg = warp & 3, kh = warp >> 2;
    const int NG = a.n / G;                 // scale groups per down row
    while (ok) {
      int s = g % ST;
      if (!mbar_wait_warp(&full[s], (g / ST) & 1, abort_flag, a.err)) break;
      const int u = hdr[s];
      if (u < 0) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        ++g;
        df_post(red, red_full, red_empty, red_unit, rc, -1, nullptr, abort_flag, a.err);
        break;
      }
      const int cnt = R.acnt[u / FB3];
      const int hrow = g8 < cnt ? g8 : 0;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      bool failed = false;
      for (int kc = 0; kc < KS3; ++kc, ++g) {
        s = g % ST;
        if (kc > 0 && !mbar_wait_warp(&full[s], (g / ST) & 1, abort_flag, a.err)) {
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
      if (failed) break;
      const float v[8] = {acc[0], acc[1], acc[2], acc[3], 0.f, 0.f, 0.f, 0.f};
      if (!df_post(red, red_full, red_empty, red_unit, rc, u, v, abort_flag, a.err)) break;
    }
  } else {
    // reducer: 64 rows x cnt tokens, first K half + second K half (warps rg, rg + 4)
    uint32_t rr = rc;
    while (ok) {
      const int b = rr & 1;
      if (!mbar_wait_warp(&red_full[b], (rr >> 1) & 1, abort_flag, a.err)) break;
      const int u = red_unit[b];
      if (u >= 0) {
        const int fb = u % FB3;
        const int cnt = R.acnt[u / FB3], prow = R.aoff[u / FB3];
        const float* rb = red + b * RED_BUF;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int col = i >> 1, row = (i & 1) * 32 + lane;    // row of the unit's 64
          if (col < cnt) {
            const int rg = row >> 4, r16 = row & 15;
            const int at = ((r16 & 7) * 2 + (col >> 1)) * 8 + (r16 >> 3) * 2 + (col & 1);
            const float v = rb[rg * 128 + at] + rb[(rg + 4) * 128 + at];
            a.rows[(size_t)(prow + col) * a.d + fb * P3_ROWS + row] = v;
          }
        }
        // the unit's rows, then one more finished down unit
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(&a.sync[6], 1u);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&red_empty[b]);
      ++rr;
      if (u < 0) break;
    }
  }
  // ---- P4: combine, fp32 in slot order j = 0 .. k-1, one rounding to bf16.
  // Only the CTAs with combine items take part; they wait for the count of
  // finished down units instead of a grid barrier, and the others are done.
  const int cpr = a.d / 8;
  if ((int)(blockIdx.x * blockDim.x) >= a.T * cpr) return;
  __syncthreads();
  if (threadIdx.x == 0)
    *flag = ok && counter_wait(&a.sync[6], (unsigned)units3, &a.sync[2], a.err, abort_flag) ? 1 : 0;
  __syncthreads();
  ok = *flag != 0;
  if (ok) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < a.T * cpr; i += gridDim.x * blockDim.x) {
      const int tk = i / cpr, f0 = (i % cpr) * 8;
      float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      // rows of 8 slots at a time: their loads are all issued before the sums
      for (int j0 = 0; j0 < a.k; j0 += 8) {
        float4 r[8][2];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (j0 + u < a.k) {
            const float4* rp = reinterpret_cast<const float4*>(
                a.rows + (size_t)R.slotrow[tk * a.k + j0 + u] * a.d + f0);
            r[u][0] = __ldcg(rp);
            r[u][1] = __ldcg(rp + 1);
          }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (j0 + u < a.k) {
            const float w = R.w[tk * a.k + j0 + u];
            v[0] = fmaf(w, r[u][0].x, v[0]); v[1] = fmaf(w, r[u][0].y, v[1]);
            v[2] = fmaf(w, r[u][0].z, v[2]); v[3] = fmaf(w, r[u][0].w, v[3]);
            v[4] = fmaf(w, r[u][1].x, v[4]); v[5] = fmaf(w, r[u][1].y, v[5]);
            v[6] = fmaf(w, r[u][1].z, v[6]); v[7] = fmaf(w, r[u][1].w, v[7]);
          }
        }
      }
      uint4 o;
      o.x = pack_bf16x2(v[0], v[1]);
      o.y = pack_bf16x2(v[2], v[3]);
      o.z = pack_bf16x2(v[4], v[5]);
      o.w = pack_bf16x2(v[6], v[7]);
      *reinterpret_cast<uint4*>(a.y + (size_t)tk * a.d + f0) = o;
    }
  }
}

// ---------------------------------------------------------------------------
bool decode_fused_fits(int T, int d, int E, int k, int n, int G) {
  using namespace df;
  if (T < 1 || T > MAXT || k > MAXK || E > MAXE) return false;
  if (G != 32 && G != 64 && G != 128) return false;
  if (d % P2_KST || d % P0_RS || d / P0_RS > P0_MAXKS || n % P3_KST || n % P2_ROWS ||
      d % P3_ROWS || E % 8 || T * d > 8 * XPT * THREADS || T * E > LPT * THREADS)
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
         up(S * d * 4) + 256 + 4 * df::MAXS;
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
  // barrier words, unit counters and the per-expert counts of finished units
  cudaError_t e = cudaMemsetAsync(a.sync, 0, 256 + 4 * (size_t)T * k, s);
  if (e != cudaSuccess) return e;
  const int smem = Smem::of(T, d).total + 1024;
  if (G == 32) return launch_fused_g<32>(maps, a, smem, s);
  if (G == 64) return launch_fused_g<64>(maps, a, smem, s);
  return launch_fused_g<128>(maps, a, smem, s);
}

}  // namespace strata
