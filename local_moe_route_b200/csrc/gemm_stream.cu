// gemm_stream.cu -- expert projections for decode / speculative-verify
// batches (T <= 8 tokens, so every expert sees at most a few rows).
// Gate/up multiplies bf16 x by the exact integer codes as bf16; down
// multiplies the fp16 h rows by the codes as fp16; outputs are fp16.
//
// Decoding gives no large batch to hide behind; every token needs its experts'
// weights read again (kongchang.com "两天移植，预填充提速8倍：Strata引擎实测",
// section "Strata快在哪", decode paragraph; 1 token + up to 3 MTP drafts are
// verified together).  The work is bound by HBM bandwidth over the packed
// weights of the touched experts, so this kernel streams them once, with no
// shared-memory staging:
//   * one warp = 16 output features of one expert, full K;
//   * each lane loads its packed words straight into registers, turns them
//     into bf16 integer fragments (q exact) and feeds mma.sync m16n8k16 with
//     the expert's token rows (<= 8 columns) as the B operand;
//   * the K order inside each 32-wide half-block is permuted identically for
//     A and B so that one LOP3 yields a ready (elem i, elem i+4) pair;
//   * each MMA covers one 32-wide half of a 64-K block, i.e. one scale group
//     (group sizes 32/64/128), so the fp16 group scale multiplies the fp32
//     partial sum instead of every weight.
#include "common.cuh"
#include "internal.h"

namespace strata {

namespace st {
constexpr int WARPS = 8;
constexpr int THREADS = WARPS * 32;
constexpr int UNROLL = 4;          // 64-K blocks whose loads are in flight together
}  // namespace st

// Exact integer pair (q_i, q_{i+4}) from nibbles i and i+4 of a word whose
// nibbles were XORed with 8 (wx = w ^ 0x88888888, so a nibble holds q + 8):
// the nibble goes into the low mantissa bits of 128.0 (bf16, F16 = false) or
// 1024.0 (fp16, F16 = true) and one exact fma subtracts 136 or 1032.
template <bool F16>
__device__ __forceinline__ uint32_t nib_pair(uint32_t wx, int i) {
  uint32_t q;
  if (F16) {
    const uint32_t v = ((wx >> (4 * i)) & 0x000F000Fu) | 0x64006400u;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(q) : "r"(v), "r"(0x3C003C00u), "r"(0xE408E408u));
  } else {
    const uint32_t v = ((wx >> (4 * i)) & 0x000F000Fu) | 0x43004300u;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(q) : "r"(v), "r"(0x3F803F80u), "r"(0xC308C308u));
  }
  return q;
}

template <bool F16>
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  if (F16)
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  else
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

struct StreamArgs {
  const uint16_t* a;            // B operand rows: x [T][K] or h [S][K]
  int a_rows;
  const int32_t* sorted_token;  // gate/up: row -> token
  const int32_t* offsets;
  const int32_t* active;
  const int32_t* n_active;
  const uint8_t* q0; const uint16_t* s0;
  const uint8_t* q1; const uint16_t* s1;
  const float* row_scale;
  uint16_t* out;
  int K, N, G;
  int kspl;                     // warps per unit (1, 2, 4 or 8), splitting K
  unsigned* err;
};

// One 32-wide half-block for one weight matrix: two MMAs on 8 nibbles per
// row (rows g and g+8), result scaled into acc.
template <bool F16>
__device__ __forceinline__ void half_block(float (&acc)[4], uint32_t wg, uint32_t wg8,
                                           float sg, float sg8, uint32_t b00, uint32_t b01,
                                           uint32_t b10, uint32_t b11) {
  float c[4] = {0.f, 0.f, 0.f, 0.f};
  wg ^= 0x88888888u;
  wg8 ^= 0x88888888u;
  mma16816<F16>(c, nib_pair<F16>(wg, 0), nib_pair<F16>(wg8, 0), nib_pair<F16>(wg, 1),
                nib_pair<F16>(wg8, 1), b00, b01);
  mma16816<F16>(c, nib_pair<F16>(wg, 2), nib_pair<F16>(wg8, 2), nib_pair<F16>(wg, 3),
                nib_pair<F16>(wg8, 3), b10, b11);
  acc[0] = fmaf(sg, c[0], acc[0]);
  acc[1] = fmaf(sg, c[1], acc[1]);
  acc[2] = fmaf(sg8, c[2], acc[2]);
  acc[3] = fmaf(sg8, c[3], acc[3]);
}

template <int NMAT>
__global__ void __launch_bounds__(st::THREADS, 2)
    moe_gemm_q4_stream_kernel(const StreamArgs args) {
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2;           // fragment row group / B column
  const int t = lane & 3;            // thread in group
  const int K = args.K, N = args.N, G = args.G;
  const int KB = K / 64;
  const int FG = N / 16;
  const int units = (*args.n_active) * FG;
  const int warp = threadIdx.x >> 5;
  // kspl warps share a unit, splitting K: the split sp covers 64-K blocks
  // [kb_lo, kb_hi).  A block holds WARPS / kspl units side by side; the warps
  // of one unit meet at their own named barrier.
  const int kspl = args.kspl;
  const int per_block = st::WARPS / kspl;
  const int slot = warp / kspl, sp = warp - slot * kspl;
  const int kb_lo = sp * KB / kspl, kb_hi = (sp + 1) * KB / kspl;
  __shared__ float red[st::WARPS][32][8];

  for (int ub = blockIdx.x * per_block; ub < units; ub += gridDim.x * per_block) {
    const int u = ub + slot;
    if (u >= units) continue;            // the unit's warps skip together
    const int e = args.active[u / FG];
    const int f0 = (u % FG) * 16;
    const int p_begin = args.offsets[e];
    const int cnt = args.offsets[e + 1] - p_begin;
    const size_t row_g = (size_t)e * N + f0 + g;
    const uint8_t* qg0 = args.q0 + row_g * (K / 2);
    const uint8_t* qg0b = qg0 + (size_t)8 * (K / 2);
    const uint16_t* sg0 = args.s0 + row_g * (K / G);
    const uint16_t* sg0b = sg0 + (size_t)8 * (K / G);
    const uint8_t* qg1 = NMAT == 2 ? args.q1 + row_g * (K / 2) : qg0;
    const uint8_t* qg1b = qg1 + (size_t)8 * (K / 2);
    const uint16_t* sg1 = NMAT == 2 ? args.s1 + row_g * (K / G) : sg0;
    const uint16_t* sg1b = sg1 + (size_t)8 * (K / G);

    for (int c0 = 0; c0 < cnt; c0 += 8) {
      // B column g of this tile: a row of the expert, or zeros
      const int pr = c0 + g;
      const bool col_ok = pr < cnt;
      int src_row = 0;
      if (col_ok) {
        src_row = NMAT == 2 ? args.sorted_token[p_begin + pr] : p_begin + pr;
        if ((unsigned)src_row >= (unsigned)args.a_rows) {
          atomicOr(args.err, kErrIndex);
          src_row = 0;
        }
      }
      const uint16_t* brow = args.a + (size_t)src_row * K;
      float acc0[4] = {0.f, 0.f, 0.f, 0.f};
      float acc1[4] = {0.f, 0.f, 0.f, 0.f};

      __syncwarp();   // mma.sync.aligned needs the warp converged
      for (int kb0 = kb_lo; kb0 < kb_hi; kb0 += st::UNROLL) {
        uint32_t wa[st::UNROLL][2][2], wb[st::UNROLL][2][2];   // [blk][half][row g / g+8]
        uint4 xa[st::UNROLL][2];
        // group scales of rows g, g + 8 (gate, up) for each half-block, loaded
        // with the weights so their latency overlaps the weight loads
        uint16_t sa[st::UNROLL][2][2], sb[st::UNROLL][2][2];
#pragma unroll
        for (int j = 0; j < st::UNROLL; ++j) {
          const int kb = kb0 + j;
          if (kb < kb_hi) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int byte = kb * 32 + h * 16 + t * 4;
              wa[j][h][0] = __ldg(reinterpret_cast<const uint32_t*>(qg0 + byte));
              wa[j][h][1] = __ldg(reinterpret_cast<const uint32_t*>(qg0b + byte));
              if (NMAT == 2) {
                wb[j][h][0] = __ldg(reinterpret_cast<const uint32_t*>(qg1 + byte));
                wb[j][h][1] = __ldg(reinterpret_cast<const uint32_t*>(qg1b + byte));
              }
              xa[j][h] = col_ok ? __ldg(reinterpret_cast<const uint4*>(brow + kb * 64 + h * 32 + t * 8))
                                : make_uint4(0, 0, 0, 0);
              const int grp = (kb * 64 + h * 32) / G;
              sa[j][h][0] = __ldg(sg0 + grp);
              sa[j][h][1] = __ldg(sg0b + grp);
              if (NMAT == 2) {
                sb[j][h][0] = __ldg(sg1 + grp);
                sb[j][h][1] = __ldg(sg1b + grp);
              }
            }
          }
        }
#pragma unroll
        for (int j = 0; j < st::UNROLL; ++j) {
          const int kb = kb0 + j;
          if (kb < kb_hi) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint4 x = xa[j][h];
              // B fragments: K slots (2t, 2t+1) <- elements (i, i+4), (2t+8, 2t+9) <- (i+1, i+5)
              const uint32_t b00 = __byte_perm(x.x, x.z, 0x5410);   // (0, 4)
              const uint32_t b01 = __byte_perm(x.x, x.z, 0x7632);   // (1, 5)
              const uint32_t b10 = __byte_perm(x.y, x.w, 0x5410);   // (2, 6)
              const uint32_t b11 = __byte_perm(x.y, x.w, 0x7632);   // (3, 7)
              half_block<NMAT == 1>(acc0, wa[j][h][0], wa[j][h][1],
                                    __half2float(__ushort_as_half(sa[j][h][0])),
                                    __half2float(__ushort_as_half(sa[j][h][1])), b00, b01, b10, b11);
              if (NMAT == 2)
                half_block<false>(acc1, wb[j][h][0], wb[j][h][1],
                                  __half2float(__ushort_as_half(sb[j][h][0])),
                                  __half2float(__ushort_as_half(sb[j][h][1])), b00, b01, b10, b11);
            }
          }
        }
      }
      // K-split partial sums: added in split order (the result does not
      // depend on timing), then the first warp of the unit finishes the tile.
      if (kspl > 1) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          red[warp][lane][i] = acc0[i];
          red[warp][lane][4 + i] = acc1[i];
        }
        named_barrier_sync(1 + slot, kspl * 32);
        if (sp == 0) {
          for (int w = 1; w < kspl; ++w) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              acc0[i] += red[warp + w][lane][i];
              acc1[i] += red[warp + w][lane][4 + i];
            }
          }
        }
      }
      if (sp == 0) {
        // C fragment: (row g, cols 2t, 2t+1), (row g+8, cols 2t, 2t+1)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int col = c0 + 2 * t + (i & 1);
          const int feat = f0 + g + (i >> 1) * 8;
          if (col < cnt) {
            float v;
            if (NMAT == 2) {
              const float gv = acc0[i], uv = acc1[i];
              v = gv / (1.0f + __expf(-gv)) * uv;
            } else {
              v = acc0[i];
              if (args.row_scale) v *= args.row_scale[p_begin + col];
            }
            if (f16_overflows(v)) atomicOr(args.err, kErrRange);
            args.out[(size_t)(p_begin + col) * N + feat] = f16_bits(v);
          }
        }
      }
      if (kspl > 1) named_barrier_sync(1 + slot, kspl * 32);   // red is reused next tile
    }
  }
}

cudaError_t launch_gemm_stream(const GemmProblem& p, const Schedule& sch, cudaStream_t s) {
  const int num_sms = sm_count();
  StreamArgs a;
  a.a = p.a;
  a.a_rows = p.op == 0 ? p.T : p.S;
  a.sorted_token = p.sorted_token;
  a.offsets = p.offsets;
  a.active = sch.active;
  a.n_active = sch.n_active;
  a.q0 = p.q0;
  a.s0 = p.s0;
  a.q1 = p.q1;
  a.s1 = p.s1;
  a.row_scale = p.row_scale;
  a.out = p.out;
  a.K = p.K;
  a.N = p.N;
  a.G = p.G;
  a.err = p.err;
  const int max_active = p.S < p.E ? p.S : p.E;
  const long units = (long)max_active * (p.N / 16);
  // Enough warps in flight to cover HBM latency: about two unit-warps per
  // resident warp slot (2 blocks of 8 warps per SM); fewer units -> more
  // warps per unit, each taking a slice of K.
  const int KB = p.K / 64;
  int kspl = 1;
  while (kspl < st::WARPS && kspl * 2 <= KB && units * kspl < 2L * num_sms * 16) kspl *= 2;
  a.kspl = kspl;
  const long per_block = st::WARPS / kspl;
  long blocks = (units + per_block - 1) / per_block;
  if (blocks > 2L * num_sms) blocks = 2L * num_sms;
  if (blocks < 1) blocks = 1;
  if (p.op == 0)
    moe_gemm_q4_stream_kernel<2><<<(int)blocks, st::THREADS, 0, s>>>(a);
  else
    moe_gemm_q4_stream_kernel<1><<<(int)blocks, st::THREADS, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace strata
