// gemm_tc.cu -- grouped expert GEMM on the 5th-generation tensor cores with
// the int4 dequantisation fused into the mainloop.
//
// The expert matmul is the heaviest compute of the layer and dequantisation
// must happen inside it, never as a separate pass that materialises bf16
// weights (kongchang.com "两天移植，预填充提速8倍：Strata引擎实测", section
// "Strata快在哪" and its MMQ note; lqnn.cn static review, sections 1.2 and
// 6.2).  The activation is fused with the projection (yfxerp.com review,
// section 5.1): the gate/up kernel's epilogue applies SwiGLU.
//
// Swap-AB formulation, one work unit = (expert e, 128 output features,
// up to 128 rows of that expert):
//   A (M = 128)  dequantised weight rows of the expert, K-major, bf16
//   B (N <= 128) the unit's token rows, K-major, bf16 (gathered x rows for
//                gate/up, contiguous h rows for down), N rounded up to 16
//   D (TMEM)     fp32 accumulators, lane = feature, column = row
// Warp roles (192 threads, persistent CTAs, one per SM):
//   warp 0     TMA of packed int4 weights (32 B per row per 64-K stage) and
//              cp.async gather of the B rows straight into the swizzled tile
//   warp 1     one thread issues tcgen05.mma (kind::f16, fp32 accumulate)
//   warps 2-5  dequantise packed -> bf16 into the 128-byte-swizzled A tile
//              (thread = weight row), then run the epilogue of the unit from
//              TMEM (SwiGLU for gate/up, row scale for down)
// Operands are fp16 (kind::f16 with f16 A and B): the gathered token rows are
// an fp16 copy of x (exact for |x| < 65504; made once per call), h is kept in
// fp16, and each dequantised weight is RNE_fp16(q * s) -- fp16 holds q * s to
// 2^-11, where bf16 weights (2^-8) would cost the layer most of its error
// budget.  Dequantisation: q in [-8, 7] becomes the fp16 value 1032 + q by
// placing the nibble (sign bit flipped) in the mantissa of 1024.0, one fma
// subtracts 1032 exactly, and one fp16 multiply by the fp16 group scale
// rounds once.
#include "common.cuh"
#include "internal.h"

namespace strata {

namespace tc {
constexpr int BM = 128;                   // output features per unit (A rows, TMEM lanes)
constexpr int NT = kTileRows;             // max token rows per unit (B rows, TMEM columns)
constexpr int BK = 64;                    // K per stage
constexpr int A_BYTES = BM * BK * 2;      // 16 KB bf16 tile
constexpr int B_BYTES = NT * BK * 2;      // 16 KB bf16 tile
constexpr int RAW_BYTES = BM * BK / 2;    //  4 KB packed int4 tile
constexpr int THREADS = 192;

template <int NMAT>
struct Cfg {
  static constexpr int STAGES = NMAT == 2 ? 3 : 4;
  static constexpr int TMEM_COLS = NMAT * NT;
  static constexpr int A_OFF = 0;
  static constexpr int B_OFF = A_OFF + STAGES * NMAT * A_BYTES;
  static constexpr int RAW_OFF = B_OFF + STAGES * B_BYTES;
  static constexpr int BAR_OFF = RAW_OFF + STAGES * NMAT * RAW_BYTES;
  static constexpr int NBARS = 4 * STAGES + 2;
  static constexpr int TOK_OFF = BAR_OFF + NBARS * 8;
  static constexpr int MISC_OFF = TOK_OFF + NT * 4;
  static constexpr int SMEM = 1024 + MISC_OFF + 64;
};
}  // namespace tc

struct TcArgs {
  const uint16_t* a;
  const int32_t* sorted_token;
  const int32_t* offsets;
  const int2* tile_table;
  const int32_t* tile_prefix;
  const uint16_t* s0;
  const uint16_t* s1;
  const float* row_scale;
  uint16_t* out;
  int K, N, G;
  int a_rows;          // rows of `a` (bounds for the gathered token indices)
  unsigned* err;
};

// 8 int4 (natural order: nibble i = element i) -> 8 fp16 = RNE(q_i * s).
__device__ __forceinline__ uint4 dequant8(uint32_t w, uint32_t sc2) {
  const uint32_t w4 = w >> 4;
  uint32_t r[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    // byte i of w (element 2i in its low nibble) to the low half, byte i of
    // w >> 4 (element 2i+1 in its low nibble) to the high half
    const uint32_t t = __byte_perm(w, w4, (uint32_t)i | ((uint32_t)(4 + i) << 8));
    // fp16 pair 1024 + (nibble ^ 8) = 1032 + q
    const uint32_t v = ((t ^ 0x64086408u) & 0x000F000Fu) | 0x64006400u;
    uint32_t qv, o;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(qv) : "r"(v), "r"(0x3C003C00u), "r"(0xE408E408u));
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(o) : "r"(qv), "r"(sc2));
    r[i] = o;
  }
  return make_uint4(r[0], r[1], r[2], r[3]);
}

__device__ __forceinline__ uint32_t scale_f16x2(uint16_t s_f16) {
  return (uint32_t)s_f16 | ((uint32_t)s_f16 << 16);
}

// fp16 copy of bf16 rows (the gathered B operand of the gate/up GEMM).
// Values beyond the fp16 range become +-inf and are reported as kErrRange.
__global__ void __launch_bounds__(256)
    bf16_to_f16_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, size_t n8,
                       unsigned* err) {
  bool over = false;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n8;
       i += (size_t)gridDim.x * blockDim.x) {
    const uint4 v = src[i];
    const uint32_t in[4] = {v.x, v.y, v.z, v.w};
    uint32_t out[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float lo = bf16_lo(in[j]), hi = bf16_hi(in[j]);
      over |= fabsf(lo) > 65504.f || fabsf(hi) > 65504.f;
      out[j] = (uint32_t)f16_bits(lo) | ((uint32_t)f16_bits(hi) << 16);
    }
    dst[i] = make_uint4(out[0], out[1], out[2], out[3]);
  }
  if (over) atomicOr(err, kErrRange);
}

template <int NMAT>
__global__ void __launch_bounds__(tc::THREADS, 1)
    moe_gemm_q4_tc_kernel(const __grid_constant__ CUtensorMap map_q0,
                          const __grid_constant__ CUtensorMap map_q1, const TcArgs args) {
  using namespace tc;
  using C = Cfg<NMAT>;
  constexpr int ST = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sA = smem + C::A_OFF;     // [ST][NMAT][A_BYTES]
  uint8_t* sB = smem + C::B_OFF;     // [ST][B_BYTES]
  uint8_t* sRaw = smem + C::RAW_OFF; // [ST][NMAT][RAW_BYTES]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* raw_full = bars;
  uint64_t* b_full = bars + ST;
  uint64_t* a_full = bars + 2 * ST;
  uint64_t* empty = bars + 3 * ST;
  uint64_t* acc_full = bars + 4 * ST;
  uint64_t* acc_empty = acc_full + 1;
  int32_t* tok = reinterpret_cast<int32_t*>(smem + C::TOK_OFF);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int K = args.K, N = args.N;
  const int KB = K / BK;
  const int FB = N / BM;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&raw_full[s], 1);
      mbar_init(&b_full[s], 32);
      mbar_init(&a_full[s], 128);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 128);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&map_q0);
    if (NMAT == 2) prefetch_tmap(&map_q1);
  }
  if (warp == 1) tmem_alloc(tmem_holder, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  // total work = tiles x feature blocks (args.tile_prefix points at the
  // total tile count, entry E of the per-expert prefix)
  const int units = (*args.tile_prefix) * FB;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    uint32_t g = 0;
    bool stop = false;
    for (int u = blockIdx.x; u < units && !stop; u += gridDim.x) {
      const int2 te = args.tile_table[u / FB];
      const int fb = u % FB;
      const int e = te.x;
      const int p0 = args.offsets[e] + te.y * NT;
      const int cnt = min(NT, args.offsets[e + 1] - p0);
      const int nrows = (cnt + 15) & ~15;
      __syncwarp();
      for (int r = lane; r < NT; r += 32) {
        int tr = (r < cnt) ? (NMAT == 2 ? args.sorted_token[p0 + r] : p0 + r) : 0;
        if ((unsigned)tr >= (unsigned)args.a_rows) {
          atomicOr(args.err, kErrIndex);
          tr = 0;
        }
        tok[r] = tr;
      }
      __syncwarp();
      const int wrow = e * N + fb * BM;
      for (int kb = 0; kb < KB; ++kb, ++g) {
        const int s = g % ST;
        const uint32_t ph = (g / ST) & 1u;
        if (g >= (uint32_t)ST && !mbar_wait(&empty[s], ph ^ 1u, abort_flag, args.err)) {
          stop = true;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&raw_full[s], NMAT * RAW_BYTES);
          tma_load_2d(sRaw + (s * NMAT + 0) * RAW_BYTES, &map_q0, kb * (BK / 2), wrow,
                      &raw_full[s]);
          if (NMAT == 2)
            tma_load_2d(sRaw + (s * NMAT + 1) * RAW_BYTES, &map_q1, kb * (BK / 2), wrow,
                        &raw_full[s]);
        }
        const uint32_t bbase = smem_addr(sB + s * B_BYTES);
        const uint16_t* abase = args.a + (size_t)kb * BK;
        for (int idx = lane; idx < nrows * 8; idx += 32) {
          const int r = idx >> 3, c = idx & 7;
          const uint16_t* src = abase + (size_t)tok[r] * K + c * 8;
          cp_async_16(bbase + sw128_offset(r, c), src, r < cnt ? 16u : 0u);
        }
        cp_async_arrive(&b_full[s]);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      uint32_t g = 0;
      int i = 0;
      bool stop = false;
      for (int u = blockIdx.x; u < units && !stop; u += gridDim.x, ++i) {
        const int2 te = args.tile_table[u / FB];
        const int e = te.x;
        const int p0 = args.offsets[e] + te.y * NT;
        const int cnt = min(NT, args.offsets[e + 1] - p0);
        const int nrows = (cnt + 15) & ~15;
        const uint32_t idesc = idesc_f32acc(BM, nrows, kFmtF16, 0);
        if (i > 0) {
          if (!mbar_wait(acc_empty, (i - 1) & 1, abort_flag, args.err)) break;
          tc_fence_after();
        }
        for (int kb = 0; kb < KB; ++kb, ++g) {
          const int s = g % ST;
          const uint32_t ph = (g / ST) & 1u;
          if (!mbar_wait(&a_full[s], ph, abort_flag, args.err) ||
              !mbar_wait(&b_full[s], ph, abort_flag, args.err)) {
            stop = true;
            break;
          }
          fence_proxy_async_smem();
          tc_fence_after();
          const uint32_t b0 = smem_addr(sB + s * B_BYTES);
#pragma unroll
          for (int ks = 0; ks < BK / 16; ++ks) {
            const uint64_t bd = desc_kmajor_sw128(b0 + ks * 32);
#pragma unroll
            for (int m = 0; m < NMAT; ++m) {
              const uint64_t ad =
                  desc_kmajor_sw128(smem_addr(sA + (s * NMAT + m) * A_BYTES) + ks * 32);
              mma_f16kind_ss(tmem + m * NT, ad, bd, idesc, (kb | ks) != 0);
            }
          }
          mma_commit(&empty[s]);
        }
        if (!stop) mma_commit(acc_full);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ dequant + epilogue
    const int q = warp & 3;                 // TMEM lane quadrant of this warp
    const int r = q * 32 + lane;            // weight row of this thread
    const int G = args.G;
    uint32_t g = 0;
    int i = 0;
    bool stop = false;
    for (int u = blockIdx.x; u < units && !stop; u += gridDim.x, ++i) {
      const int2 te = args.tile_table[u / FB];
      const int fb = u % FB;
      const int e = te.x;
      const int p0 = args.offsets[e] + te.y * NT;
      const int cnt = min(NT, args.offsets[e + 1] - p0);
      const size_t wrow = (size_t)e * N + fb * BM + r;
      const uint16_t* srow0 = args.s0 + wrow * (K / G);
      const uint16_t* srow1 = NMAT == 2 ? args.s1 + wrow * (K / G) : nullptr;
      for (int kb = 0; kb < KB; ++kb, ++g) {
        const int s = g % ST;
        const uint32_t ph = (g / ST) & 1u;
        // scales of the (at most two) groups this 64-wide stage touches
        const int g0 = (kb * BK) / G;
        const int g1 = (kb * BK + BK / 2) / G;
        uint32_t sc[NMAT][2];
        sc[0][0] = scale_f16x2(__ldg(srow0 + g0));
        sc[0][1] = scale_f16x2(__ldg(srow0 + g1));
        if (NMAT == 2) {
          sc[NMAT - 1][0] = scale_f16x2(__ldg(srow1 + g0));
          sc[NMAT - 1][1] = scale_f16x2(__ldg(srow1 + g1));
        }
        if (!mbar_wait(&raw_full[s], ph, abort_flag, args.err)) {
          stop = true;
          break;
        }
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
          const uint4* rp = reinterpret_cast<const uint4*>(sRaw + (s * NMAT + m) * RAW_BYTES + r * 32);
          const uint4 lo = rp[0], hi = rp[1];
          const uint32_t words[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
          uint8_t* tile = sA + (s * NMAT + m) * A_BYTES;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 o = dequant8(words[c], sc[m][c >> 2]);
            *reinterpret_cast<uint4*>(tile + sw128_offset(r, c)) = o;
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&a_full[s]);
      }
      if (stop) break;
      // ---- epilogue of this unit
      bool ok = mbar_wait(acc_full, i & 1, abort_flag, args.err);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int feat = fb * BM + r;
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16);
      const int nch = (cnt + 31) >> 5;
      for (int c = 0; c < nch; ++c) {
        uint32_t acc0[32];
        tmem_ld_32x32b_x32(tbase + c * 32, acc0);
        if (NMAT == 2) {
          uint32_t acc1[32];
          tmem_ld_32x32b_x32(tbase + NT + c * 32, acc1);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int p = c * 32 + j;
            if (p < cnt) {
              const float gv = __uint_as_float(acc0[j]);
              const float uv = __uint_as_float(acc1[j]);
              const float h = gv / (1.0f + __expf(-gv)) * uv;
              args.out[(size_t)(p0 + p) * N + feat] = f16_bits(h);
            }
          }
        } else {
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int p = c * 32 + j;
            if (p < cnt) {
              float v = __uint_as_float(acc0[j]);
              if (args.row_scale) v *= args.row_scale[p0 + p];
              args.out[(size_t)(p0 + p) * N + feat] = f16_bits(v);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(acc_empty);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

static int g_num_sms = 0;

template <int NMAT>
static cudaError_t launch_tc_impl(const GemmProblem& p, const Schedule& sch, cudaStream_t s) {
  using C = tc::Cfg<NMAT>;
  CUtensorMap m0, m1;
  const uint64_t rows = (uint64_t)p.E * p.N;
  if (encode_tmap_2d(&m0, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.q0, p.K / 2, rows, p.K / 2,
                     tc::BK / 2, tc::BM, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  m1 = m0;
  if (NMAT == 2 &&
      encode_tmap_2d(&m1, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.q1, p.K / 2, rows, p.K / 2,
                     tc::BK / 2, tc::BM, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  {
    cudaError_t e = cudaFuncSetAttribute(moe_gemm_q4_tc_kernel<NMAT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
  }
  if (g_num_sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (g_num_sms <= 0) g_num_sms = 148;
  }
  if (p.op == 0) {
    // the gate/up B operand is the fp16 copy of x
    const size_t n8 = (size_t)p.T * p.K / 8;
    int blocks = (int)((n8 + 255) / 256);
    if (blocks > 8 * g_num_sms) blocks = 8 * g_num_sms;
    bf16_to_f16_kernel<<<blocks, 256, 0, s>>>(reinterpret_cast<const uint4*>(p.a),
                                              reinterpret_cast<uint4*>(p.a16), n8, p.err);
  }
  TcArgs a;
  a.a = p.op == 0 ? p.a16 : p.a;
  a.sorted_token = p.sorted_token;
  a.offsets = p.offsets;
  a.tile_table = sch.tile_table;
  a.tile_prefix = sch.tile_prefix + p.E;     // -> total tile count
  a.s0 = p.s0;
  a.s1 = p.s1;
  a.row_scale = p.row_scale;
  a.out = p.out;
  a.K = p.K;
  a.N = p.N;
  a.G = p.G;
  a.a_rows = p.op == 0 ? p.T : p.S;
  a.err = p.err;
  const int max_units = max_tiles(p.S, p.E) * (p.N / tc::BM);
  const int grid = max_units < g_num_sms ? max_units : g_num_sms;
  moe_gemm_q4_tc_kernel<NMAT><<<grid, tc::THREADS, C::SMEM, s>>>(m0, m1, a);
  return cudaGetLastError();
}

cudaError_t launch_gemm_tc(const GemmProblem& p, const Schedule& sch, cudaStream_t s) {
  return p.op == 0 ? launch_tc_impl<2>(p, sch, s) : launch_tc_impl<1>(p, sch, s);
}

}  // namespace strata
