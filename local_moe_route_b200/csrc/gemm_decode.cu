// gemm_decode.cu -- expert projections for decode / speculative-verify
// batches (T <= 8 tokens), weights staged through shared memory by TMA.
//
// Decode gives no batch to amortise the weights over: every step reads the
// packed weights of the experts its tokens chose (kongchang.com
// "两天移植，预填充提速8倍：Strata引擎实测", section "Strata快在哪", decode
// paragraph), so the work is bound by HBM bandwidth over those bytes.  Here a
// producer warp keeps a ring of shared-memory stages full with bulk tensor
// copies -- the bytes in flight no longer depend on registers -- and eight
// consumer warps turn each stage into mma.sync fragments:
//   * a unit is 64 output features of one expert (gate and up both for
//     gate/up); a stage holds, per weight matrix, 64 rows x 256 K (128 bytes
//     of packed int4 per row, 128-byte swizzle) plus the unit's token rows
//     for the same 256 K (up to 8 rows);
//   * consumer warp w owns rows 16 (w % 4) .. + 15 and one half of each
//     stage's K (w / 4); the two halves' fp32 sums meet in shared memory at
//     the end of the unit and are added in a fixed order;
//   * nibble pairs (i, i + 4) become exact integer fragments with one
//     mask-and-xor and one fma each (plus one shift per packed word for fp16,
//     three for bf16); the K order inside each 32-wide half-block is
//     permuted identically for the token operand;
//   * the MMAs of one scale group (32, 64 or 128 K, a compile-time constant)
//     sum integer codes times token values in fp32, and the group's fp16
//     scale multiplies that sum once.
#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace strata {

namespace dk {
constexpr int ROWS = 64;             // output features per unit
constexpr int KC = 256;              // K per stage
constexpr int WBYTES = ROWS * KC / 2;   // 8 KB of packed weights per matrix and stage
constexpr int XROWS = 8;             // token rows per unit (T <= 8)
constexpr int XBYTES = XROWS * KC * 2;  // 4 KB
constexpr int CONSUMERS = 8;         // 4 row groups x 2 halves of each stage's K
constexpr int THREADS = (CONSUMERS + 1) * 32;
constexpr int ST = 5;                // ring depth
template <int NMAT>
struct Layout {
  static constexpr int STAGE = NMAT * WBYTES + XBYTES;   // multiple of 1024
  static constexpr int BAR_OFF = ST * STAGE;
  static constexpr int RED_OFF = BAR_OFF + 2 * ST * 8 + 16;          // [4][32][8] fp32
  static constexpr int SMEM = 1024 + RED_OFF + 4 * 32 * 8 * 4;
};
}  // namespace dk

struct DecodeArgs {
  const int32_t* sorted_token;  // gate/up: row -> token
  const int32_t* offsets;
  const int32_t* active;
  const int32_t* n_active;
  const uint16_t* s0;
  const uint16_t* s1;
  const float* row_scale;
  uint16_t* out;
  int T, K, N;
  unsigned* err;
};

// The eight int4 codes of one packed word (K order 0..7, low nibble first)
// as four exact integer pairs: pair i holds codes (i, i + 4), in the low and
// high half of the register.  The mask-and-xor flips each code's sign bit
// and sets the exponent in one logic op, giving 1024 + (q + 8) (fp16) or
// 128 + (q + 8) (bf16), and one fma removes the offset.  fp16 takes codes 1
// and 3 straight from bits 4..7 as 1024 + 16 (q + 8) -- exact, 16 (q + 8) <=
// 240 fits the 10-bit mantissa -- and the same fma scales them back by 1/16,
// which saves two shifts per word; bf16's 7-bit mantissa has no room for
// that.
template <bool F16>
__device__ __forceinline__ void dk_word(uint32_t w, uint32_t (&p)[4]) {
  if (F16) {
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
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t v = ((w >> (4 * i)) & 0x000F000Fu) ^ 0x43084308u;
      // 1.0, -136 (bf16 pairs)
      asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(p[i]) : "r"(v), "r"(0x3F803F80u), "r"(0xC308C308u));
    }
  }
}

template <bool F16>
__device__ __forceinline__ void dk_mma(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
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

// Group scales of one row for one consumer warp's half of a stage (128 K:
// 128 / G consecutive fp16 values), one aligned load.
template <int G>
__device__ __forceinline__ uint2 dk_scales(const uint16_t* p) {
  uint2 v = make_uint2(0, 0);
  if (G == 32)
    v = ld_nc_v2(p);
  else if (G == 64)
    v.x = ld_nc_u32(p);
  else
    v.x = ld_nc_u16(p);
  return v;
}

// Scale j of those (j is a constant once the caller's loop is unrolled).
__device__ __forceinline__ float dk_scale_at(const uint2& v, int j) {
  const uint32_t x = (j & 2) ? v.y : v.x;
  return __half2float(__ushort_as_half(static_cast<unsigned short>((j & 1) ? (x >> 16) : x)));
}

template <int NMAT, int G>
__global__ void __launch_bounds__(dk::THREADS, NMAT == 1 ? 3 : 2)
    moe_gemm_q4_decode_kernel(const __grid_constant__ CUtensorMap map_w0,
                              const __grid_constant__ CUtensorMap map_w1,
                              const __grid_constant__ CUtensorMap map_x, const DecodeArgs args) {
  using namespace dk;
  using Lay = Layout<NMAT>;
  constexpr bool F16 = NMAT == 1;            // down: fp16 h rows; gate/up: bf16 x rows
  extern __shared__ uint8_t dk_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dk_smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Lay::BAR_OFF);
  uint64_t* empty = full + ST;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + ST);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = args.K, N = args.N;
  const int NKC = K / KC;                    // stages per unit
  const int FBK = N / ROWS;                  // units per expert
  const int units = (*args.n_active) * FBK;
  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], CONSUMERS);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == CONSUMERS && lane == 0) {
    prefetch_tmap(&map_w0);
    if (NMAT == 2) prefetch_tmap(&map_w1);
    prefetch_tmap(&map_x);
  }
  __syncthreads();
  const int my_units =
      (int)blockIdx.x < units ? (units - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;

  if (warp == CONSUMERS) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t g = 0;
      bool stop = false;
      for (int i = 0; i < my_units && !stop; ++i) {
        const int u = blockIdx.x + i * gridDim.x;
        const int e = args.active[u / FBK];
        const int p_begin = args.offsets[e];
        const int cnt_all = args.offsets[e + 1] - p_begin;
        const int wrow = e * N + (u % FBK) * ROWS;
        // the unit's rows in tiles of 8 (one tile unless an expert has more
        // rows than a decode batch has tokens)
        for (int c0 = 0; c0 < cnt_all && !stop; c0 += XROWS) {
        const int cnt = min(XROWS, cnt_all - c0);
        int trow[XROWS];
#pragma unroll
        for (int j = 0; j < XROWS; ++j) {
          int tk = 0;
          if (NMAT == 2 && j < cnt) {
            tk = args.sorted_token[p_begin + c0 + j];
            if ((unsigned)tk >= (unsigned)args.T) {
              atomicOr(args.err, kErrIndex);
              tk = 0;
            }
          }
          trow[j] = tk;
        }
        for (int kc = 0; kc < NKC; ++kc, ++g) {
          const int s = g % ST;
          if (g >= (uint32_t)ST &&
              !mbar_wait(&empty[s], ((g / ST) - 1) & 1, abort_flag, args.err)) {
            stop = true;
            break;
          }
          uint8_t* st = smem + s * Lay::STAGE;
          uint8_t* xs = st + NMAT * WBYTES;
          const uint32_t xbytes = NMAT == 2 ? (uint32_t)cnt * KC * 2 : (uint32_t)XBYTES;
          mbar_arrive_expect_tx(&full[s], NMAT * WBYTES + xbytes);
          tma_load_2d(st, &map_w0, kc * (KC / 2), wrow, &full[s]);
          if (NMAT == 2) {
            tma_load_2d(st + WBYTES, &map_w1, kc * (KC / 2), wrow, &full[s]);
#pragma unroll
            for (int j = 0; j < XROWS; ++j)
              if (j < cnt) tma_load_2d(xs + j * KC * 2, &map_x, kc * KC, trow[j], &full[s]);
          } else {
            tma_load_2d(xs, &map_x, kc * KC, p_begin + c0, &full[s]);   // 8 rows from p_begin + c0
          }
        }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    constexpr int NG = 128 / G;              // scale groups in a warp's half of a stage
    constexpr int HPG = G / 32;              // 32-K half-blocks per group
    const int g8 = lane >> 2, t = lane & 3;
    const int rg = warp & 3, kh = warp >> 2;   // row group, half of the stage's K
    const int r0 = rg * 16 + g8;             // rows r0 and r0 + 8 of the unit
    float* red = reinterpret_cast<float*>(smem + Lay::RED_OFF) + (rg * 32 + lane) * 8;
    const int swz = (r0 & 7) << 4;           // 128-byte swizzle (row r0 + 8 alike)
    uint32_t gst = 0;
    bool failed = false;                     // uniform over the consumer warps
    for (int i = 0; i < my_units && !failed; ++i) {
      const int u = blockIdx.x + i * gridDim.x;
      const int e = args.active[u / FBK];
      const int fb = u % FBK;
      const int p_begin = args.offsets[e];
      const int cnt_all = args.offsets[e + 1] - p_begin;
      // this warp's first scale of row r0: group (kc 256 + kh 128) / G of the row
      const size_t srow = (size_t)(e * N + fb * ROWS + r0) * (K / G) + kh * NG;
      const size_t srow8 = srow + (size_t)8 * (K / G);
      for (int c0 = 0; c0 < cnt_all && !failed; c0 += XROWS) {
      const int cnt = min(XROWS, cnt_all - c0);
      float acc[NMAT][4];
      uint2 sc[NMAT][2];                     // [matrix][row r0 / r0 + 8], next stage
#pragma unroll
      for (int m = 0; m < NMAT; ++m) {
        const uint16_t* sp = m == 0 ? args.s0 : args.s1;
        sc[m][0] = dk_scales<G>(sp + srow);
        sc[m][1] = dk_scales<G>(sp + srow8);
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[m][q] = 0.f;
      }
      for (int kc = 0; kc < NKC; ++kc, ++gst) {
        uint2 cur[NMAT][2];
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
          cur[m][0] = sc[m][0];
          cur[m][1] = sc[m][1];
        }
        if (kc + 1 < NKC) {
#pragma unroll
          for (int m = 0; m < NMAT; ++m) {
            const uint16_t* sp = m == 0 ? args.s0 : args.s1;
            sc[m][0] = dk_scales<G>(sp + srow + (size_t)(kc + 1) * (2 * NG));
            sc[m][1] = dk_scales<G>(sp + srow8 + (size_t)(kc + 1) * (2 * NG));
          }
        }
        const int s = gst % ST;
        if (!mbar_wait_warp(&full[s], (gst / ST) & 1, abort_flag, args.err)) break;
        const uint8_t* st = smem + s * Lay::STAGE;
        const uint8_t* xs = st + NMAT * WBYTES + g8 * (KC * 2) + kh * 256;
        float c[NMAT][4];                    // one scale group's integer-code sums
#pragma unroll
        for (int hb = 0; hb < 4; ++hb) {     // 32-K half-blocks of this warp's 128 K
          const int chunk = kh * 4 + hb;     // 16-byte chunk of the 128-byte row
          const uint4 x = *reinterpret_cast<const uint4*>(xs + (hb * 32 + t * 8) * 2);
          // B fragments: K slots (2t, 2t+1) <- elements (i, i+4), (2t+8, 2t+9) <- (i+1, i+5)
          const uint32_t b00 = __byte_perm(x.x, x.z, 0x5410);
          const uint32_t b01 = __byte_perm(x.x, x.z, 0x7632);
          const uint32_t b10 = __byte_perm(x.y, x.w, 0x5410);
          const uint32_t b11 = __byte_perm(x.y, x.w, 0x7632);
          const int off = ((chunk << 4) ^ swz) + t * 4;
#pragma unroll
          for (int m = 0; m < NMAT; ++m) {
            const uint8_t* W = st + m * WBYTES;
            uint32_t p0[4], p1[4];
            dk_word<F16>(*reinterpret_cast<const uint32_t*>(W + r0 * 128 + off), p0);
            dk_word<F16>(*reinterpret_cast<const uint32_t*>(W + (r0 + 8) * 128 + off), p1);
            if (hb % HPG == 0) {
#pragma unroll
              for (int q = 0; q < 4; ++q) c[m][q] = 0.f;
            }
            dk_mma<F16>(c[m], p0[0], p1[0], p0[1], p1[1], b00, b01);
            dk_mma<F16>(c[m], p0[2], p1[2], p0[3], p1[3], b10, b11);
            if (hb % HPG == HPG - 1) {       // group complete: apply its fp16 scales
              const int j = hb / HPG;
              const float s0 = dk_scale_at(cur[m][0], j), s8 = dk_scale_at(cur[m][1], j);
              acc[m][0] = fmaf(s0, c[m][0], acc[m][0]);
              acc[m][1] = fmaf(s0, c[m][1], acc[m][1]);
              acc[m][2] = fmaf(s8, c[m][2], acc[m][2]);
              acc[m][3] = fmaf(s8, c[m][3], acc[m][3]);
            }
          }
        }
        // release the stage; the fence orders its loads before the next TMA write
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
      // Every consumer warp reaches the two barriers below, also after a
      // wait that ran out (which raised abort_flag first); the first one
      // reduces the flag over all consumer threads, so the decision to stop
      // is the same in every warp.
      // The second K half hands its sums to the first (fixed order: first + second).
      if (kh == 1) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          red[q] = acc[0][q];
          if (NMAT == 2) red[4 + q] = acc[NMAT - 1][q];
        }
      }
      failed = named_barrier_or(1, CONSUMERS * 32, *abort_flag != 0);   // all warps alike
      if (kh == 0) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc[0][q] += red[q];
          if (NMAT == 2) acc[NMAT - 1][q] += red[4 + q];
        }
      }
      named_barrier_sync(1, CONSUMERS * 32);   // red is reused by the next tile
      if (failed || kh == 1) continue;
      // C fragment: (row g8, cols 2t, 2t+1), (row g8 + 8, cols 2t, 2t+1); column
      // j is grouped row p_begin + c0 + j
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int col = 2 * t + (q & 1);
        const int feat = fb * ROWS + r0 + (q >> 1) * 8;
        if (col < cnt) {
          float v;
          if (NMAT == 2) {
            const float gv = acc[0][q], uv = acc[NMAT - 1][q];
            v = gv / (1.0f + __expf(-gv)) * uv;
          } else {
            v = acc[0][q];
            if (args.row_scale) v *= args.row_scale[p_begin + c0 + col];
          }
          if (f16_overflows(v)) atomicOr(args.err, kErrRange);
          args.out[(size_t)(p_begin + c0 + col) * N + feat] = f16_bits(v);
        }
      }
      }
    }
  }
}

// One CTA per unit up to as many as fit on the GPU at once (three per SM for
// down, two for gate/up, by shared memory and registers).
template <int NMAT, int G>
static cudaError_t launch_decode(const CUtensorMap& mw0, const CUtensorMap& mw1,
                                 const CUtensorMap& mx, const DecodeArgs& a, long units,
                                 int num_sms, cudaStream_t s) {
  using namespace dk;
  auto kern = moe_gemm_q4_decode_kernel<NMAT, G>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Layout<NMAT>::SMEM);
  if (e != cudaSuccess) return e;
  static std::atomic<int> per_sm_cache{0};   // the same on every B200
  int per_sm = per_sm_cache.load(std::memory_order_relaxed);
  if (per_sm == 0) {
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, THREADS, Layout<NMAT>::SMEM);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    per_sm_cache.store(per_sm, std::memory_order_relaxed);
  }
  long blocks = units;
  if (blocks > (long)per_sm * num_sms) blocks = (long)per_sm * num_sms;
  if (blocks < 1) blocks = 1;
  kern<<<(int)blocks, THREADS, Layout<NMAT>::SMEM, s>>>(mw0, mw1, mx, a);
  return cudaSuccess;
}

// Takes the problem if its shapes fit the staged kernel (K a multiple of 256,
// N of 64); otherwise returns cudaErrorNotSupported and the caller uses the
// register-streaming kernel.
cudaError_t launch_gemm_decode(const GemmProblem& p, const Schedule& sch, cudaStream_t s) {
  using namespace dk;
  if (p.K % KC != 0 || p.N % ROWS != 0 || p.T > XROWS ||
      (p.G != 32 && p.G != 64 && p.G != 128))
    return cudaErrorNotSupported;
  const int num_sms = sm_count();
  CUtensorMap mw0, mw1, mx;
  const uint64_t rows = (uint64_t)p.E * p.N;
  if (encode_tmap_2d(&mw0, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.q0, p.K / 2, rows, p.K / 2, KC / 2, ROWS,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  mw1 = mw0;
  if (p.op == 0 &&
      encode_tmap_2d(&mw1, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.q1, p.K / 2, rows, p.K / 2, KC / 2,
                     ROWS, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  // token rows: x [T][K] bf16 one row per copy (gate/up), h [S][K] fp16
  // eight rows per copy (down)
  const bool gu = p.op == 0;
  if (encode_tmap_2d(&mx, gu ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                     p.a, p.K, gu ? p.T : p.S, (uint64_t)p.K * 2, KC, gu ? 1 : XROWS,
                     CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  DecodeArgs a;
  a.sorted_token = p.sorted_token;
  a.offsets = p.offsets;
  a.active = sch.active;
  a.n_active = sch.n_active;
  a.s0 = p.s0;
  a.s1 = p.s1;
  a.row_scale = p.row_scale;
  a.out = p.out;
  a.T = p.T;
  a.K = p.K;
  a.N = p.N;
  a.err = p.err;
  const int max_active = p.S < p.E ? p.S : p.E;
  const long units = (long)max_active * (p.N / ROWS);
  cudaError_t e = cudaSuccess;
  if (gu) {
    if (p.G == 32) e = launch_decode<2, 32>(mw0, mw1, mx, a, units, num_sms, s);
    else if (p.G == 64) e = launch_decode<2, 64>(mw0, mw1, mx, a, units, num_sms, s);
    else e = launch_decode<2, 128>(mw0, mw1, mx, a, units, num_sms, s);
  } else {
    if (p.G == 32) e = launch_decode<1, 32>(mw0, mw1, mx, a, units, num_sms, s);
    else if (p.G == 64) e = launch_decode<1, 64>(mw0, mw1, mx, a, units, num_sms, s);
    else e = launch_decode<1, 128>(mw0, mw1, mx, a, units, num_sms, s);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace strata
