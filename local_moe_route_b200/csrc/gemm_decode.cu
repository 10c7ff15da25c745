// gemm_decode.cu -- expert projections for decode / speculative-verify
// batches (T <= 8 tokens), weights staged through shared memory by TMA.
//
// Decode gives no batch to amortise the weights over: every step reads the
// packed weights of the experts its tokens chose (kongchang.com
// "两天移植，预填充提速8倍：Strata引擎实测", section "Strata快在哪", decode
// paragraph), so the work is bound by HBM bandwidth over those bytes.  Here a
// producer warp keeps a ring of shared-memory stages full with bulk tensor
// copies -- the bytes in flight no longer depend on registers -- and four
// consumer warps turn each stage into mma.sync fragments:
//   * a unit is 64 output features of one expert (gate and up both for
//     gate/up); a stage holds, per weight matrix, 64 rows x 256 K (128 bytes
//     of packed int4 per row, 128-byte swizzle) plus the unit's token rows
//     for the same 256 K (up to 8 rows);
//   * consumer warp w owns rows 16 (w % 4) .. + 15 and one half of each
//     stage's K (w / 4); the two halves' fp32 sums meet in shared memory at
//     the end of the unit and are added in a fixed order;
//   * nibble pairs (i, i + 4) become exact integer fragments with one shift,
//     one mask-and-or and one fma each; the K order inside each 32-wide
//     half-block is permuted identically for the token operand; each MMA
//     covers one 32-wide half-block, i.e. one scale group, and the fp16 group
//     scale multiplies the fp32 partial sum.
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
  int T, K, N, G;
  unsigned* err;
};

template <bool F16>
__device__ __forceinline__ uint32_t dk_pair(uint32_t wx, int i) {
  uint32_t q;
  if (F16) {
    const uint32_t v = ((wx >> (4 * i)) & 0x000F000Fu) | 0x64006400u;   // 1024 + (q + 8)
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(q) : "r"(v), "r"(0x3C003C00u), "r"(0xE408E408u));
  } else {
    const uint32_t v = ((wx >> (4 * i)) & 0x000F000Fu) | 0x43004300u;   // 128 + (q + 8)
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(q) : "r"(v), "r"(0x3F803F80u), "r"(0xC308C308u));
  }
  return q;
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

// One 32-wide half-block of one matrix: packed words of rows g and g + 8
// (nibbles XORed with 8 inside), two MMAs, the group scales applied to the
// fp32 partial sums.
template <bool F16>
__device__ __forceinline__ void dk_half(float (&acc)[4], uint32_t wg, uint32_t wg8, float sg,
                                        float sg8, uint32_t b00, uint32_t b01, uint32_t b10,
                                        uint32_t b11) {
  float c[4] = {0.f, 0.f, 0.f, 0.f};
  wg ^= 0x88888888u;
  wg8 ^= 0x88888888u;
  dk_mma<F16>(c, dk_pair<F16>(wg, 0), dk_pair<F16>(wg8, 0), dk_pair<F16>(wg, 1),
              dk_pair<F16>(wg8, 1), b00, b01);
  dk_mma<F16>(c, dk_pair<F16>(wg, 2), dk_pair<F16>(wg8, 2), dk_pair<F16>(wg, 3),
              dk_pair<F16>(wg8, 3), b10, b11);
  acc[0] = fmaf(sg, c[0], acc[0]);
  acc[1] = fmaf(sg, c[1], acc[1]);
  acc[2] = fmaf(sg8, c[2], acc[2]);
  acc[3] = fmaf(sg8, c[3], acc[3]);
}

// Group scales of one row for one stage (KC / G consecutive groups: 8, 4 or
// 2 fp16 values), one aligned load.
__device__ __forceinline__ uint4 dk_scales(const uint16_t* p, int groups) {
  uint4 v = make_uint4(0, 0, 0, 0);
  if (groups == 8) {
    v = ld_nc_v4(p);
  } else if (groups == 4) {
    const uint2 t = ld_nc_v2(p);
    v.x = t.x;
    v.y = t.y;
  } else {
    v.x = ld_nc_u32(p);
  }
  return v;
}

__device__ __forceinline__ float dk_scale_at(const uint4& v, int idx) {
  const int w = idx >> 1;
  const uint32_t x = (w & 2) ? ((w & 1) ? v.w : v.z) : ((w & 1) ? v.y : v.x);
  return __half2float(__ushort_as_half(static_cast<unsigned short>((idx & 1) ? (x >> 16) : x)));
}

template <int NMAT>
__global__ void __launch_bounds__(dk::THREADS)
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
  const int K = args.K, N = args.N, G = args.G;
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
    const int g8 = lane >> 2, t = lane & 3;
    const int rg = warp & 3, kh = warp >> 2;   // row group, half of the stage's K
    const int r0 = rg * 16 + g8;             // rows r0 and r0 + 8 of the unit
    float* red = reinterpret_cast<float*>(smem + Lay::RED_OFF) + (rg * 32 + lane) * 8;
    const int GS = KC / G;                   // scale groups per stage
    const int swz = (r0 & 7) << 4;           // 128-byte swizzle (row r0 + 8 alike)
    uint32_t gst = 0;
    bool failed = false;                     // uniform over the consumer warps
    for (int i = 0; i < my_units && !failed; ++i) {
      const int u = blockIdx.x + i * gridDim.x;
      const int e = args.active[u / FBK];
      const int fb = u % FBK;
      const int p_begin = args.offsets[e];
      const int cnt_all = args.offsets[e + 1] - p_begin;
      const size_t srow = (size_t)(e * N + fb * ROWS + r0) * (K / G);
      const size_t srow8 = srow + (size_t)8 * (K / G);
      for (int c0 = 0; c0 < cnt_all && !failed; c0 += XROWS) {
      const int cnt = min(XROWS, cnt_all - c0);
      float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
      uint4 sc[2][2];                        // [matrix][row r0 / r0 + 8], next stage
#pragma unroll
      for (int m = 0; m < NMAT; ++m) {
        const uint16_t* sp = m == 0 ? args.s0 : args.s1;
        sc[m][0] = dk_scales(sp + srow, GS);
        sc[m][1] = dk_scales(sp + srow8, GS);
      }
      for (int kc = 0; kc < NKC; ++kc, ++gst) {
        uint4 cur[2][2];
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
          cur[m][0] = sc[m][0];
          cur[m][1] = sc[m][1];
        }
        if (kc + 1 < NKC) {
#pragma unroll
          for (int m = 0; m < NMAT; ++m) {
            const uint16_t* sp = m == 0 ? args.s0 : args.s1;
            sc[m][0] = dk_scales(sp + srow + (size_t)(kc + 1) * GS, GS);
            sc[m][1] = dk_scales(sp + srow8 + (size_t)(kc + 1) * GS, GS);
          }
        }
        const int s = gst % ST;
        if (!mbar_wait_warp(&full[s], (gst / ST) & 1, abort_flag, args.err)) break;
        const uint8_t* st = smem + s * Lay::STAGE;
        const uint8_t* xs = st + NMAT * WBYTES + g8 * (KC * 2);
#pragma unroll
        for (int kk = 0; kk < KC / 128; ++kk) {
          const int kb = kh * (KC / 128) + kk;   // this warp's 64-K blocks of the stage
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int c = kb * 2 + h;        // 16-byte chunk of the 128-byte row
            const uint4 x = *reinterpret_cast<const uint4*>(xs + (kb * 64 + h * 32 + t * 8) * 2);
            // B fragments: K slots (2t, 2t+1) <- elements (i, i+4), (2t+8, 2t+9) <- (i+1, i+5)
            const uint32_t b00 = __byte_perm(x.x, x.z, 0x5410);
            const uint32_t b01 = __byte_perm(x.x, x.z, 0x7632);
            const uint32_t b10 = __byte_perm(x.y, x.w, 0x5410);
            const uint32_t b11 = __byte_perm(x.y, x.w, 0x7632);
            const int gi = (kb * 64 + h * 32) / G;   // group within the stage
            const int off = ((c << 4) ^ swz) + t * 4;
#pragma unroll
            for (int m = 0; m < NMAT; ++m) {
              const uint8_t* W = st + m * WBYTES;
              const uint32_t w0 = *reinterpret_cast<const uint32_t*>(W + r0 * 128 + off);
              const uint32_t w1 = *reinterpret_cast<const uint32_t*>(W + (r0 + 8) * 128 + off);
              dk_half<F16>(m == 0 ? acc0 : acc1, w0, w1, dk_scale_at(cur[m][0], gi),
                           dk_scale_at(cur[m][1], gi), b00, b01, b10, b11);
            }
          }
        }
        // the stage's words were consumed by the MMAs above; release it
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
      // Every consumer warp reaches the two barriers below, also after a
      // wait that ran out (which raised abort_flag first): the flag read
      // between them makes the decision to stop the same in all warps.
      // The second K half hands its sums to the first (fixed order: first + second).
      if (kh == 1) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          red[q] = acc0[q];
          red[4 + q] = acc1[q];
        }
      }
      named_barrier_sync(1, CONSUMERS * 32);
      failed = *abort_flag != 0;
      if (kh == 0) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc0[q] += red[q];
          acc1[q] += red[4 + q];
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
            const float gv = acc0[q], uv = acc1[q];
            v = gv / (1.0f + __expf(-gv)) * uv;
          } else {
            v = acc0[q];
            if (args.row_scale) v *= args.row_scale[p_begin + c0 + col];
          }
          args.out[(size_t)(p_begin + c0 + col) * N + feat] = f16_bits(v);
        }
      }
      }
    }
  }
}

// Takes the problem if its shapes fit the staged kernel (K a multiple of 256,
// N of 64); otherwise returns cudaErrorNotSupported and the caller uses the
// register-streaming kernel.
cudaError_t launch_gemm_decode(const GemmProblem& p, const Schedule& sch, cudaStream_t s) {
  using namespace dk;
  if (p.K % KC != 0 || p.N % ROWS != 0 || p.T > XROWS) return cudaErrorNotSupported;
  static int num_sms = 0;
  if (num_sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (num_sms <= 0) num_sms = 148;
  }
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
  a.G = p.G;
  a.err = p.err;
  const int max_active = p.S < p.E ? p.S : p.E;
  long blocks = (long)max_active * (p.N / ROWS);
  if (blocks > 2L * num_sms) blocks = 2L * num_sms;
  if (blocks < 1) blocks = 1;
  if (gu) {
    cudaError_t e = cudaFuncSetAttribute(moe_gemm_q4_decode_kernel<2>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Layout<2>::SMEM);
    if (e != cudaSuccess) return e;
    moe_gemm_q4_decode_kernel<2><<<(int)blocks, THREADS, Layout<2>::SMEM, s>>>(mw0, mw1, mx, a);
  } else {
    cudaError_t e = cudaFuncSetAttribute(moe_gemm_q4_decode_kernel<1>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Layout<1>::SMEM);
    if (e != cudaSuccess) return e;
    moe_gemm_q4_decode_kernel<1><<<(int)blocks, THREADS, Layout<1>::SMEM, s>>>(mw0, mw1, mx, a);
  }
  return cudaGetLastError();
}

}  // namespace strata
