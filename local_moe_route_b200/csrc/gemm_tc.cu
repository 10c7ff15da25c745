// gemm_tc.cu -- grouped expert GEMM on the 5th-generation tensor cores with
// the int4 dequantisation fused into the mainloop.
//
// The expert matmul is the heaviest compute of the layer and dequantisation
// must happen inside it, never as a separate pass that materialises dense
// weights (kongchang.com "两天移植，预填充提速8倍：Strata引擎实测", section
// "Strata快在哪" and its MMQ note; lqnn.cn static review, sections 1.2 and
// 6.2).  The activation is fused with the projection (yfxerp.com review,
// section 5.1): the gate/up epilogue applies SwiGLU.
//
// Swap-AB formulation.  One work unit = (expert e, two 128-row weight slots,
// up to 160 token rows of e):
//   gate/up: slot 0 = 128 gate rows, slot 1 = the same 128 up rows
//   down:    slot 0, slot 1 = two consecutive 128-row blocks of W_down
//   A (M = 128) dequantised weights, fp16, written by threads straight into
//               tensor memory (tcgen05.st), read by tcgen05.mma from TMEM
//   B (N <= 160) the unit's token rows, fp16, K-major, 128-byte swizzled in
//               shared memory (one tile feeds both slots' MMAs)
//   D           fp32 accumulators in TMEM, lane = weight row, column = token
// Units of up to 160 token rows: with a top-10 of 512 experts over 6144
// tokens an expert gets 120 rows on average and rarely more than 160, so
// nearly every expert is one unit per weight-row block and its weights are
// dequantised once.  (With 128-row units one expert in four needed a second,
// nearly empty unit that dequantised all of its weights again: 630 tiles
// instead of 512, and the layer took 2.37 ms instead of 2.16.)
// Keeping A out of shared memory leaves shared-memory bandwidth to the B
// tiles and the packed weights; the MMAs' own reads of B need half of it.
//
// Warp roles (gate/up 640 threads, down 768; persistent, one CTA per SM):
//   warp 0       TMA of packed int4 rows into a ring of 8 (down: 6) K stages
//                of 64: one copy covers two K stages when K is a multiple of
//                128 (a 64-byte row segment per weight row, 64-byte swizzle;
//                otherwise 32 bytes, 32-byte swizzle), and of the group
//                scales: one block of 8 groups of both slots' rows (16 B per
//                row) every 8 G / 64 stages into a two-deep ring
//   warps 1, 3   tcgen05.mma issue, one thread per slot
//   warp 2       token rows into a 5-deep (down: 4-deep) ring, one TMA tile
//                of 160 rows per stage (128 for units of at most 128 rows):
//                the down projection reads h, whose rows are already
//                grouped by expert; for gate/up a pre-pass writes the fp16 rows
//                of x in grouped order (x[sorted_token[p]]), so both operands
//                of every stage arrive by TMA.  (Gathering the rows from a
//                token-order copy with tile::gather4 copies instead, 32 per
//                stage, left the MMA waiting on them 64% of the time and
//                doubled the kernel's time at T = 6144.)
//   warps 4-15   three dequantising warpgroups taking
//                the stages round-robin; thread = weight row; fp16 pairs go to
//                TMEM with tcgen05.st; at each scale block a thread copies its
//                rows' 8 scales into registers and frees the ring slot.  (When
//                K / G is not a multiple of 8 the rows' scales are loaded from
//                global memory one block ahead instead: a thread's next
//                release of a ring slot waits for such a load in flight.)
//   warps 16-19  epilogue (down: warps 16-23, four per 128-feature slice):
//                TMEM -> registers -> SwiGLU or row scale -> fp16,
//                transposed through shared memory into whole-row stores
// TMEM (512 columns): accumulators of slot 0/1 at columns 0/160, three A
// stages of 64 columns (32 per slot) at 320..511.
//
// Operands are fp16 (kind::f16): x rows are copied to fp16 in grouped order
// once per call (exact for |x| < 65504), h is kept in fp16, and each weight is RNE_fp16(q * s): fp16
// keeps q * s to 2^-11, where bf16 weights (2^-8) would use up most of the
// layer's error budget.  Dequantisation: the nibble with its sign bit flipped
// goes into the mantissa of 1024.0 (giving 1032 + q), one fma subtracts 1032
// exactly, one fp16 multiply by the fp16 group scale rounds once.
#include "common.cuh"
#include "dequant.cuh"
#include "internal.h"

namespace strata {

namespace tc {
constexpr int BM = 128;                    // weight rows per slot (TMEM lanes)
constexpr int NT = kTileRows;              // token rows per unit (max MMA N)
constexpr int BK = 64;                     // K per stage
constexpr int A_ST = 3;                    // TMEM A stages
constexpr int RAW_BYTES = BM * BK / 2;     // 4 KB per slot
constexpr int B_BYTES = NT * BK * 2;       // 16 KB
constexpr int STG_PITCH = NT + 8;          // halves per staging row (one output feature)
// Group scales by TMA (when K / G is a multiple of 8): blocks of 8 groups of
// both slots' 128 rows (16 bytes per row and slot) in a two-deep ring.
constexpr int SC_GROUPS = 8;
constexpr int SC_BYTES = 2 * BM * SC_GROUPS * 2;   // 4 KB per block

constexpr int W_TMA = 0, W_MMA = 1, W_BTMA = 2, W_MMA2 = 3, W_DQ = 4;
// Dequantising warpgroups take the stages round-robin, three of them: with
// the MMAs issued from two threads the MMA warps wait on dequantised A
// stages (measured at T = 6144: gate/up 1.18 -> 1.14 ms with three groups
// instead of two, down 0.73 -> 0.67 ms).  Registers bound the count: three
// groups fit at 96 registers per thread (gate/up) and four epilogue warps
// more at 80 (down).
template <int OP>
struct Roles {
  static constexpr int NWG = 3;
  static constexpr int W_EPI = W_DQ + 4 * NWG;
  // epilogue warps: down has two 128-feature slices per unit and gives each
  // its own four warps, so the accumulator is read out in half the time
  static constexpr int NEPI = OP == 0 ? 4 : 8;
  static constexpr int THREADS = (W_EPI + NEPI) * 32;
};

// Shared memory per operation: gate/up writes one 128-feature slice per unit
// (SwiGLU merges the two slots), so its staging tile is half the size of
// down's and the space goes to two more token-row stages.
// RK: K stages per packed-weight copy (2 when K is a multiple of 128: one
// 64-byte row segment per weight row and copy instead of two 32-byte ones).
template <int OP, int RK>
struct Lay {
  static constexpr int B_ST = OP == 0 ? 5 : 4;                      // token-row ring depth
  // packed-weight ring depth in copies (8 / 5 K stages of 64, rounded up)
  static constexpr int RAW_ST = OP == 0 ? 8 / RK : (RK == 1 ? 5 : 3);
  static constexpr int RAW_SLOT = RK * RAW_BYTES;                   // one slot of one copy
  static constexpr int RAW_OFF = 0;                                 // [RAW_ST][2][RAW_SLOT]
  static constexpr int B_OFF = RAW_OFF + RAW_ST * 2 * RAW_SLOT;     // [B_ST][B_BYTES]
  static constexpr int STG_OFF = B_OFF + B_ST * B_BYTES;            // [slices * BM][STG_PITCH]
  static constexpr int STG_BYTES = (OP == 0 ? 1 : 2) * BM * STG_PITCH * 2;
  static constexpr int SC_OFF = STG_OFF + STG_BYTES;                 // [2][2][BM][8] fp16
  static constexpr int BAR_OFF = SC_OFF + 2 * SC_BYTES;
  static constexpr int NBARS = 2 * RAW_ST + 2 * B_ST + A_ST + 2 + 4;
  static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
  static constexpr int SMEM = 1024 + MISC_OFF + 64;
  static_assert(SMEM <= 232448, "shared memory per CTA");
};

// Packed-weight copies of RK K stages when the group scales come by TMA
// (K / G a multiple of 8 implies K a multiple of 128 for G >= 16).
template <bool STMA>
__host__ __device__ constexpr int raw_k_stages() { return STMA ? 2 : 1; }

constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t A_COL = 2 * NT;
}  // namespace tc

struct TcArgs {
  const uint16_t* a;            // B operand rows (fp16): x16 [T][K] or h [S][K]
  const int32_t* sorted_token;  // gate/up: row -> token
  const int32_t* offsets;
  const int4* tile_table;        // (expert, first row, rows, 0) per tile
  const int32_t* total_tiles;   // -> tile_prefix[E]
  const uint16_t* s0;
  const uint16_t* s1;
  const float* row_scale;
  uint16_t* out;
  int K, N, G, E;
  int a_rows;
  unsigned* err;
};

// One work unit, decoded from its index.
struct Unit {
  int e, p0, cnt, nrows, nslots;
  int wrow[2];      // first weight row of each slot in the [E*N] row space
  int fout[2];      // first output feature of each slot
};

template <int OP>
__device__ __forceinline__ Unit decode_unit(const TcArgs& a, int u, int FB) {
  Unit U;
  const int4 te = a.tile_table[u / FB];
  const int fb = u % FB;
  U.e = te.x;
  U.p0 = te.y;
  U.cnt = te.z;
  U.nrows = (U.cnt + 15) & ~15;
  if (OP == 0) {
    U.nslots = 2;
    U.fout[0] = U.fout[1] = fb * tc::BM;
    U.wrow[0] = U.wrow[1] = U.e * a.N + fb * tc::BM;
  } else {
    U.fout[0] = fb * 2 * tc::BM;
    U.fout[1] = U.fout[0] + tc::BM;
    U.nslots = U.fout[1] < a.N ? 2 : 1;
    U.wrow[0] = U.e * a.N + U.fout[0];
    U.wrow[1] = U.wrow[0] + tc::BM;
  }
  return U;
}

// Gate/up B operand: xs[p] = fp16(x[sorted_token[p]]) for the S grouped rows,
// with K interleaved within each group of 8 (0, 4, 1, 5, 2, 6, 3, 7) to match
// dequant8_interleaved.  Out-of-range token indices are reported (kErrIndex)
// and read row 0; values beyond the fp16 range become +-inf and are reported
// as kErrRange.
__global__ void __launch_bounds__(256)
    gather_rows_f16_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ sorted_token,
                           int T, int d, int S, uint16_t* __restrict__ xs, unsigned* err) {
  // one warp per grouped row; lane l converts 16-byte chunks l, l + 32, ...
  const int lane = threadIdx.x & 31;
  const int cpr = d / 8;                      // 16-byte chunks per row
  bool over = false, bad = false;
  for (int p = blockIdx.x * 8 + (threadIdx.x >> 5); p < S; p += gridDim.x * 8) {
    int t = sorted_token[p];
    if ((unsigned)t >= (unsigned)T) {
      bad = true;
      t = 0;
    }
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * d);
    uint4* dst = reinterpret_cast<uint4*>(xs + (size_t)p * d);
    // four 16-byte loads of the row in flight per lane before any is used;
    // the copy is written once and read back once by the GEMM's TMA, so it
    // goes out with an evict-first hint
    for (int c0 = lane; c0 < cpr; c0 += 4 * 32) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (c0 + 32 * u < cpr) v[u] = __ldg(src + c0 + 32 * u);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (c0 + 32 * u >= cpr) break;
        float e[8];
        e[0] = bf16_lo(v[u].x); e[1] = bf16_hi(v[u].x); e[2] = bf16_lo(v[u].y); e[3] = bf16_hi(v[u].y);
        e[4] = bf16_lo(v[u].z); e[5] = bf16_hi(v[u].z); e[6] = bf16_lo(v[u].w); e[7] = bf16_hi(v[u].w);
#pragma unroll
        for (int j = 0; j < 8; ++j) over |= fabsf(e[j]) > 65504.f;
        // K order within the group of 8: 0, 4, 1, 5, 2, 6, 3, 7 (the order the
        // weight dequantisation produces)
        uint4 o;
        o.x = pack_f16x2(e[0], e[4]);
        o.y = pack_f16x2(e[1], e[5]);
        o.z = pack_f16x2(e[2], e[6]);
        o.w = pack_f16x2(e[3], e[7]);
        __stcs(dst + c0 + 32 * u, o);
      }
    }
  }
  if (over) atomicOr(err, kErrRange);
  if (bad) atomicOr(err, kErrIndex);
}

cudaError_t launch_gather_rows_f16(const uint16_t* x, const int32_t* sorted_token, int T, int d,
                                   int S, uint16_t* xs, unsigned* err, cudaStream_t s) {
  long blocks = (S + 7) / 8;                       // 8 rows (warps) per block
  if (blocks > 16L * sm_count()) blocks = 16L * sm_count();
  if (blocks < 1) return cudaSuccess;
  gather_rows_f16_kernel<<<(int)blocks, 256, 0, s>>>(x, sorted_token, T, d, S, xs, err);
  return cudaGetLastError();
}

template <int OP, bool ILV, bool STMA>
__global__ void __launch_bounds__(tc::Roles<OP>::THREADS, 1)
    moe_gemm_q4_tc_kernel(const __grid_constant__ CUtensorMap map_q0,
                          const __grid_constant__ CUtensorMap map_q1,
                          const __grid_constant__ CUtensorMap map_b,
                          const __grid_constant__ CUtensorMap map_b128,
                          const __grid_constant__ CUtensorMap map_s0,
                          const __grid_constant__ CUtensorMap map_s1, const TcArgs args) {
  using namespace tc;
  constexpr int RK = raw_k_stages<STMA>();
  using Ly = Lay<OP, RK>;
  constexpr int B_ST = Ly::B_ST;
  constexpr int RAW_ST = Ly::RAW_ST;
  constexpr int RAW_SLOT = Ly::RAW_SLOT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sRaw = smem + Ly::RAW_OFF;
  uint8_t* sB = smem + Ly::B_OFF;
  uint16_t* sStg = reinterpret_cast<uint16_t*>(smem + Ly::STG_OFF);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Ly::BAR_OFF);
  uint64_t* raw_full = bars;
  uint64_t* raw_empty = raw_full + RAW_ST;
  uint64_t* b_full = raw_empty + RAW_ST;
  uint64_t* b_empty = b_full + B_ST;
  uint64_t* a_full = b_empty + B_ST;
  // An A stage is free again when the MMAs of the stage that last used it
  // are done, and those MMAs' commit to the token-row ring says so: the
  // dequantising warps wait on b_empty of that stage, one commit per stage.
  uint64_t* acc_full = a_full + A_ST;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* sc_full = acc_empty + 1;           // [2] scale blocks
  uint64_t* sc_empty = sc_full + 2;            // [2]
  uint8_t* sSc = smem + Ly::SC_OFF;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Ly::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Ly::MISC_OFF + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int K = args.K, N = args.N, G = args.G;
  const int KB = K / BK;
  const int FB = OP == 0 ? N / BM : (N + 2 * BM - 1) / (2 * BM);

  if (threadIdx.x == 0) {
    for (int s = 0; s < RAW_ST; ++s) {
      mbar_init(&raw_full[s], 1);
      mbar_init(&raw_empty[s], RK * BM);   // every K stage of the copy, one warpgroup each
    }
    for (int s = 0; s < B_ST; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 2);          // one commit per MMA-issuing thread
    }
    for (int s = 0; s < A_ST; ++s) {
      mbar_init(&a_full[s], BM);
    }
    mbar_init(acc_full, 2);
    mbar_init(acc_empty, Roles<OP>::NEPI * 32);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sc_full[b], 1);
      mbar_init(&sc_empty[b], Roles<OP>::NWG * BM);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == W_TMA && lane == 0) {
    prefetch_tmap(&map_q0);
    if (OP == 0) prefetch_tmap(&map_q1);
    prefetch_tmap(&map_b);
    prefetch_tmap(&map_b128);
    if (STMA) {
      prefetch_tmap(&map_s0);
      if (OP == 0) prefetch_tmap(&map_s1);
    }
  }
  if (warp == W_MMA) tmem_alloc(tmem_holder, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  const int units = (*args.total_tiles) * FB;
  const int my_units =
      (int)blockIdx.x < units ? (units - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
  const int total_stages = my_units * KB;

  if (warp == W_TMA) {
    // -------------------------------------------------------------- TMA producer
    {
      const CUtensorMap* map_slot1 = OP == 0 ? &map_q1 : &map_q0;
      const CUtensorMap* smap_slot1 = OP == 0 ? &map_s1 : &map_s0;
      const int SPB = SC_GROUPS * G / BK;     // stages per scale block (4, 8 or 16)
      uint32_t g = 0, gs = 0;
      bool stop = false;
      for (int i = 0; i < my_units && !stop; ++i) {
        const Unit U = decode_unit<OP>(args, blockIdx.x + i * gridDim.x, FB);
        for (int kb = 0; kb < KB; ++kb, ++g) {
          if (STMA && kb % SPB == 0) {
            // the scale block of the next SPB stages: rows of both slots,
            // groups kb * BK / G .. + 8 (x coordinate a multiple of 8)
            const int ss = gs & 1;
            if (gs >= 2 &&
                !mbar_wait_warp(&sc_empty[ss], ((gs >> 1) - 1) & 1, abort_flag, args.err)) {
              stop = true;
              break;
            }
            if (lane == 0) {
            mbar_arrive_expect_tx(&sc_full[ss], SC_BYTES);
            tma_load_2d(sSc + ss * SC_BYTES, &map_s0, kb * BK / G, U.wrow[0], &sc_full[ss]);
            tma_load_2d(sSc + ss * SC_BYTES + SC_BYTES / 2, smap_slot1, kb * BK / G, U.wrow[1],
                        &sc_full[ss]);
            }
            __syncwarp();
            ++gs;
          }
          if (kb % RK != 0) continue;       // this copy holds RK K stages
          const uint32_t gr = g / RK;
          const int s = gr % RAW_ST;
          if (gr >= (uint32_t)RAW_ST &&
              !mbar_wait_warp(&raw_empty[s], ((gr / RAW_ST) - 1) & 1, abort_flag, args.err)) {
            stop = true;
            break;
          }
          if (lane == 0) {
          mbar_arrive_expect_tx(&raw_full[s], 2 * RAW_SLOT);
          tma_load_2d(sRaw + (s * 2 + 0) * RAW_SLOT, &map_q0, kb * (BK / 2), U.wrow[0],
                      &raw_full[s]);
          tma_load_2d(sRaw + (s * 2 + 1) * RAW_SLOT, map_slot1, kb * (BK / 2), U.wrow[1],
                      &raw_full[s]);
          }
          __syncwarp();
        }
      }
    }
  } else if (warp == W_BTMA) {
    // -------------------------------------------------------------- token rows (B)
    // one TMA tile of 128 grouped rows per stage (rows past the unit belong
    // to other units or lie beyond S; the MMA reads only nrows of them)
    {
      uint32_t g = 0;
      bool stop = false;
      for (int i = 0; i < my_units && !stop; ++i) {
        const Unit U = decode_unit<OP>(args, blockIdx.x + i * gridDim.x, FB);
        for (int kb = 0; kb < KB; ++kb, ++g) {
          const int s = g % B_ST;
          if (g >= (uint32_t)B_ST &&
              !mbar_wait_warp(&b_empty[s], ((g / B_ST) - 1) & 1, abort_flag, args.err)) {
            stop = true;
            break;
          }
          // a unit of at most 128 rows takes a 128-row tile
          if (lane == 0) {
            const bool small = U.nrows <= 128;
            mbar_arrive_expect_tx(&b_full[s], small ? 128 * BK * 2 : B_BYTES);
            tma_load_2d(sB + s * B_BYTES, small ? &map_b128 : &map_b, kb * BK, U.p0, &b_full[s]);
          }
          __syncwarp();
        }
      }
    }
  } else if (warp == W_MMA || warp == W_MMA2) {
    // -------------------------------------------------------------- MMA issue
    // Two warps issue the MMAs, one per slot: a thread issues one
    // tcgen05.mma per ~64 cycles at most, which is all the time an M = 128,
    // N = 128, K = 16 product takes, so one issuing thread alone leaves the
    // tensor pipe idle whenever it does anything else.  Each warp follows the
    // rings as a whole; one lane, elected once, issues its slot's MMAs and
    // one commit per stage (a commit covers the MMAs of the thread that
    // issues it; the rings' empty barriers count both threads' commits).
    const int m = warp == W_MMA ? 0 : 1;
    uint32_t g = 0;
    bool stop = false;
    const bool leader = elect_one();
    for (int i = 0; i < my_units && !stop; ++i) {
      const Unit U = decode_unit<OP>(args, blockIdx.x + i * gridDim.x, FB);
      const uint32_t idesc = idesc_f32acc(BM, U.nrows, kFmtF16, 0);
      const bool issue = leader && m < U.nslots;
      if (i > 0) {
        if (!mbar_wait_warp(acc_empty, (i - 1) & 1, abort_flag, args.err)) break;
        tc_fence_after();
      }
      for (int kb = 0; kb < KB; ++kb, ++g) {
        const int sa = g % A_ST, sb = g % B_ST;
        if (!mbar_wait_warp(&a_full[sa], (g / A_ST) & 1, abort_flag, args.err) ||
            !mbar_wait_warp(&b_full[sb], (g / B_ST) & 1, abort_flag, args.err)) {
          stop = true;
          break;
        }
        tc_fence_after();
        if (issue) {
          const uint32_t b0 = smem_addr(sB + sb * B_BYTES);
          const uint32_t a0 = tmem + A_COL + sa * 64 + m * 32;
#pragma unroll
          for (int ks = 0; ks < BK / 16; ++ks)
            mma_f16kind_ts(tmem + m * NT, a0 + ks * 8, desc_kmajor_sw128(b0 + ks * 32), idesc,
                           (kb | ks) != 0);
        }
        // frees token-row slot sb and A stage sa once both threads' MMAs are done
        if (leader) mma_commit(&b_empty[sb]);
        __syncwarp();
      }
      if (!stop && leader) mma_commit(acc_full);
      __syncwarp();
    }
  } else if (warp < Roles<OP>::W_EPI) {
    // -------------------------------------------------------------- dequantise
    constexpr int NWG = Roles<OP>::NWG;
    const int wg = (warp - W_DQ) >> 2;       // takes the stages g with g % NWG == wg
    const int q = warp & 3;                  // TMEM lane quadrant
    const int r = q * 32 + lane;             // weight row within the slot
    const uint32_t t_lane = tmem + ((uint32_t)(q * 32) << 16);
    const int g_shift = G == 32 ? 5 : (G == 64 ? 6 : 7);
    const int KG = K / G;                    // groups per weight row
    // Group scales are read in blocks of SB consecutive groups per row and
    // slot (SB = the largest of 8, 4, 2, 1 dividing K / G, so a block is one
    // aligned 16-, 8-, 4- or 2-byte load).  The block after the one in use
    // is always in flight: a load has the time of SB groups to arrive.
    const int SB = (KG & 7) == 0 ? 8 : (KG & 3) == 0 ? 4 : (KG & 1) == 0 ? 2 : 1;
    uint32_t gsr = 0;                        // scale blocks taken from the ring (STMA)
    int4 te_c = make_int4(0, 0, 0, 0), te_n = make_int4(0, 0, 0, 0);
    int unit_c = -1;
    auto tile_of = [&](int i) { return ld_nc_s4(args.tile_table + (blockIdx.x + i * gridDim.x) / FB); };
    // first scale of block b0, slot mm, of unit i (tile entry te)
    auto scale_ptr = [&](const int4& te, int i, int mm, int b0) {
      const int fb = (blockIdx.x + i * gridDim.x) % FB;
      int f0 = OP == 0 ? fb * BM : fb * 2 * BM + mm * BM;
      if (f0 >= N) f0 -= BM;                 // a down slot beyond N: its results are unused
      const uint16_t* sp = (OP == 0 && mm == 1) ? args.s1 : args.s0;
      return sp + (size_t)(te.x * N + f0 + r) * KG + b0;
    };
    auto load_block = [&](const uint16_t* p) -> uint4 {
      uint4 v = make_uint4(0, 0, 0, 0);
      if (SB == 8) {
        v = ld_nc_v4(p);
      } else if (SB == 4) {
        const uint2 t = ld_nc_v2(p);
        v.x = t.x;
        v.y = t.y;
      } else if (SB == 2) {
        v.x = ld_nc_u32(p);
      } else {
        v.x = ld_nc_u16(p);
      }
      return v;
    };
    // the 32-bit word of a block holding groups 2w and 2w + 1
    auto word_at = [&](const uint4& v, int w) -> uint32_t {
      return (w & 2) ? ((w & 1) ? v.w : v.z) : ((w & 1) ? v.y : v.x);
    };
    uint4 blk_c[2], blk_n[2];
    // A group scale above 65504 / 8 could give a dequantised weight q * s
    // beyond the fp16 range: such scales are reported, once per thread.
    uint32_t big_scale = 0;
    int key_c = -1, key_n = -1;              // unit * 65536 + first group of the block
    int iu = 0, kb = wg;                     // unit and K block of stage g
    while (kb >= KB) {
      kb -= KB;
      ++iu;
    }
    for (int g = wg; g < total_stages; g += NWG) {
      const int grp0 = (kb * BK) >> g_shift;
      const int key = (iu << 16) | (grp0 & ~(SB - 1));
      if (STMA && key != key_c) {
        // this block's scales of both slots from the TMA ring into
        // registers; the slot is released at once
        const int ss = gsr & 1;
        if (!mbar_wait(&sc_full[ss], (gsr >> 1) & 1, abort_flag, args.err)) break;
#pragma unroll
        for (int mm = 0; mm < 2; ++mm)
          blk_c[mm] = *reinterpret_cast<const uint4*>(sSc + ss * SC_BYTES + mm * (SC_BYTES / 2) +
                                                       r * 16);
        fence_proxy_async_smem();              // the loads before the next TMA write
        mbar_arrive(&sc_empty[ss]);
        ++gsr;
        key_c = key;
#pragma unroll
        for (int mm = 0; mm < 2; ++mm) {
          const uint4 b = blk_c[mm];
          big_scale |= __vcmpgtu2(b.x & 0x7FFF7FFFu, 0x6FFF6FFFu) |
                       __vcmpgtu2(b.y & 0x7FFF7FFFu, 0x6FFF6FFFu) |
                       __vcmpgtu2(b.z & 0x7FFF7FFFu, 0x6FFF6FFFu) |
                       __vcmpgtu2(b.w & 0x7FFF7FFFu, 0x6FFF6FFFu);
        }
      } else if (!STMA && key != key_c) {
        if (iu != unit_c) {
          te_c = (unit_c >= 0 && iu == unit_c + 1) ? te_n : tile_of(iu);
          unit_c = iu;
          if (iu + 1 < my_units) te_n = tile_of(iu + 1);
        }
        if (key == key_n) {
          blk_c[0] = blk_n[0];
          blk_c[1] = blk_n[1];
        } else {
#pragma unroll
          for (int mm = 0; mm < 2; ++mm)
            blk_c[mm] = load_block(scale_ptr(te_c, iu, mm, key & 0xFFFF));
        }
        key_c = key;
#pragma unroll
        for (int mm = 0; mm < 2; ++mm) {
          const uint4 b = blk_c[mm];
          big_scale |= __vcmpgtu2(b.x & 0x7FFF7FFFu, 0x6FFF6FFFu) |
                       __vcmpgtu2(b.y & 0x7FFF7FFFu, 0x6FFF6FFFu) |
                       __vcmpgtu2(b.z & 0x7FFF7FFFu, 0x6FFF6FFFu) |
                       __vcmpgtu2(b.w & 0x7FFF7FFFu, 0x6FFF6FFFu);
        }
        // the block after this one: the next groups of this unit, or the
        // first block of the next unit
        int ni = iu, nb = (key & 0xFFFF) + SB;
        if (nb >= KG) {
          nb = 0;
          ++ni;
        }
        key_n = -1;
        if (ni < my_units) {
          key_n = (ni << 16) | nb;
#pragma unroll
          for (int mm = 0; mm < 2; ++mm)
            blk_n[mm] = load_block(scale_ptr(ni == iu ? te_c : te_n, ni, mm, nb));
        }
      }
      // fp16 scale pairs (the scale in both halves) for the stage's group(s);
      // with 32-wide groups the stage's two groups share one 32-bit word
      const int idx = grp0 & (SB - 1);
      const uint32_t sel = (G != 32 && (idx & 1)) ? 0x3232u : 0x1010u;
      uint32_t sc2[2][2];
#pragma unroll
      for (int mm = 0; mm < 2; ++mm) {
        const uint32_t w = word_at(blk_c[mm], idx >> 1);
        sc2[mm][0] = __byte_perm(w, 0, sel);
        sc2[mm][1] = G == 32 ? __byte_perm(w, 0, 0x3232u) : sc2[mm][0];
      }
      kb += NWG;
      while (kb >= KB) {
        kb -= KB;
        ++iu;
      }
      const int sr = (g / RK) % RAW_ST, sa = g % A_ST;
      if (!mbar_wait(&raw_full[sr], ((g / RK) / RAW_ST) & 1, abort_flag, args.err)) break;
      // packed words of this row: 16-byte chunks 2j, 2j + 1 of the copy's row
      // segment (j = the K stage within the copy); the 32-byte swizzle puts
      // chunk c at c ^ ((r >> 2) & 1), the 64-byte one at c ^ ((r >> 1) & 3)
      uint4 raw[2][2];
      const int sw = RK == 1 ? (r >> 2) & 1 : (r >> 1) & 3;
      const int c0 = 2 * (g % RK);
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const uint8_t* rowp = sRaw + (sr * 2 + m) * RAW_SLOT + r * (RK * 32);
        raw[m][0] = *reinterpret_cast<const uint4*>(rowp + 16 * (c0 ^ sw));
        raw[m][1] = *reinterpret_cast<const uint4*>(rowp + 16 * ((c0 + 1) ^ sw));
      }
      // The slots are dequantised one after the other once the A stage is
      // free (dequantising both into registers first, then waiting, needs
      // more registers than three warpgroups have).
      auto dq_slot = [&](int m, uint32_t(&out)[32]) {
        const uint32_t sc_a = sc2[m][0], sc_b = sc2[m][1];
        const uint32_t words[8] = {raw[m][0].x, raw[m][0].y, raw[m][0].z, raw[m][0].w,
                                   raw[m][1].x, raw[m][1].y, raw[m][1].z, raw[m][1].w};
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          // gate/up: the grouped copy of x is interleaved; down: h is
          // interleaved when the fused forward produced it
          if (OP == 0 || ILV) dequant8_interleaved(words[c], c < 4 ? sc_a : sc_b, &out[4 * c]);
          else dequant8(words[c], c < 4 ? sc_a : sc_b, &out[4 * c]);
        }
      };
      if (g >= A_ST && !mbar_wait_warp(&b_empty[(g - A_ST) % B_ST], ((g - A_ST) / B_ST) & 1,
                                       abort_flag, args.err))
        break;
      __syncwarp();       // converged before the .sync.aligned TMEM stores
      tc_fence_after();   // order the TMEM stores after the MMAs that released this A stage
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        uint32_t out[32];
        dq_slot(m, out);
        tmem_st_32x32b_x32(t_lane + A_COL + sa * 64 + m * 32, out);
      }
      fence_proxy_async_smem();      // the words' loads before the next TMA write
      mbar_arrive(&raw_empty[sr]);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&a_full[sa]);
    }
    if (big_scale) atomicOr(args.err, kErrRange);
  } else {
    // -------------------------------------------------------------- epilogue
    // The accumulator is read out in the layout TMEM holds it, one output
    // feature per thread: its token values go as packed fp16 into a staging
    // tile [feature][token] in shared memory (four 16-byte stores per 32
    // tokens), and the accumulator is handed back to the MMA warp right
    // after.  The transposition to the row-major output happens on the way
    // out: thread t gathers 8 features of token t and stores 16 bytes, while
    // the next unit's MMAs already run.
    constexpr int ET = Roles<OP>::NEPI * 32;              // epilogue threads
    const int q = warp & 3;
    const int et = threadIdx.x - Roles<OP>::W_EPI * 32;   // 0 .. ET - 1
    const int esl = (warp - Roles<OP>::W_EPI) >> 2;       // the output slice this warp reads
    const uint32_t t_lane = tmem + ((uint32_t)(q * 32) << 16);
    bool ov = false;            // an output of this thread overflowed fp16
    __half2 omax = __float2half2_rn(0.f);   // largest |output| of the current unit
    for (int i = 0; i < my_units; ++i) {
      const Unit U = decode_unit<OP>(args, blockIdx.x + i * gridDim.x, FB);
      const bool got = mbar_wait_warp(acc_full, i & 1, abort_flag, args.err);
      tc_fence_after();
      const int nch = (U.cnt + 31) >> 5;
      const int nout = OP == 0 ? 1 : U.nslots;        // 128-feature slices of output
      // 16 token values of slice m, columns 16 c16 .. -> fp16 pairs in the
      // staging row of this thread's feature.  The pairs are checked for fp16
      // overflow (a running maximum of |h| that lets NaN through, tested per
      // unit); columns past the unit's rows hold no result of this unit, and
      // only the last chunk of a unit can have such columns.
      auto emit16 = [&](int m, int c16, const float* v) {
        uint16_t* frow = sStg + (m * BM + q * 32 + lane) * STG_PITCH;
        uint32_t o[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) o[u] = pack_f16x2(v[2 * u], v[2 * u + 1]);
        const int lim = U.cnt - c16 * 16;
        if (lim >= 16) {
#pragma unroll
          for (int u = 0; u < 8; ++u)
            omax = __hmax2_nan(omax, __habs2(*reinterpret_cast<const __half2*>(&o[u])));
        } else {
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int j = 2 * u;
            const uint32_t live = j + 1 < lim ? o[u] : (j < lim ? (o[u] & 0xFFFFu) : 0u);
            omax = __hmax2_nan(omax, __habs2(*reinterpret_cast<const __half2*>(&live)));
          }
        }
        *reinterpret_cast<uint4*>(frow + c16 * 16) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(frow + c16 * 16 + 8) = make_uint4(o[4], o[5], o[6], o[7]);
      };
      if constexpr (OP == 0) {
        for (int c = 0; c < nch && got; ++c) {
          __syncwarp();   // converged before the .sync.aligned TMEM loads
          uint32_t a0[32], a1[32];
          tmem_ld_32x32b_x32(t_lane + c * 32, a0);
          tmem_ld_32x32b_x32(t_lane + NT + c * 32, a1);
          tmem_ld_wait_regs(a0);
          tmem_ld_wait_regs(a1);
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float gv = __uint_as_float(a0[j]), uv = __uint_as_float(a1[j]);
            v[j] = __fdividef(gv, 1.0f + __expf(-gv)) * uv;
          }
          emit16(0, 2 * c, v);
          emit16(0, 2 * c + 1, v + 16);
        }
      } else {
        // the chunks of slice esl, one TMEM load and wait each (two loads
        // per wait, or 16-column loads with the next one in flight, held the
        // accumulator longer)
        const int nq = got && esl < nout ? nch : 0;
        auto taddr = [&](int c) { return t_lane + esl * NT + c * 32; };
        auto convert = [&](int c, const uint32_t (&r)[32]) {
          const int m = esl;
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
          if (args.row_scale) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int t = c * 32 + j;
              if (t < U.cnt) v[j] *= args.row_scale[U.p0 + t];
            }
          }
          emit16(m, 2 * c, v);
          emit16(m, 2 * c + 1, v + 16);
        };
        for (int qq = 0; qq < nq; ++qq) {
          __syncwarp();   // converged before the .sync.aligned TMEM loads
          uint32_t ra[32];
          tmem_ld_32x32b_x32(taddr(qq), ra);
          tmem_ld_wait_regs(ra);
          convert(qq, ra);
        }
      }
      tc_fence_before();
      if (got) mbar_arrive(acc_empty);
      {
        // an overflowed (or NaN) half has all exponent bits set
        const uint32_t mb = *reinterpret_cast<const uint32_t*>(&omax);
        ov |= (mb & 0x7C00u) == 0x7C00u || (mb & 0x7C000000u) == 0x7C000000u;
        omax = __float2half2_rn(0.f);
      }
      // staging tile complete; a wait that gave up in any epilogue warp ends
      // the loop in all of them alike
      if (named_barrier_or(1, ET, !got)) break;
      // copy-out: item = (4 consecutive tokens, 8 consecutive features);
      // eight 8-byte loads give the 4 x 8 block, four 16-byte stores write it
      const int ntg = (U.cnt + 3) >> 2;
      const int items = ntg * nout * (BM / 8);
      for (int it = et; it < items; it += ET) {
        const int tg = it % ntg, ch = it / ntg;
        const uint16_t* src = sStg + ch * 8 * STG_PITCH + 4 * tg;
        uint2 h[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) h[k] = *reinterpret_cast<const uint2*>(src + k * STG_PITCH);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int tt = 4 * tg + u;
          if (tt >= U.cnt) break;
          // token u's value of feature k: half (u & 1) of h[k].x (u < 2) or h[k].y
          uint32_t f[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) f[k] = u < 2 ? h[k].x : h[k].y;
          const uint32_t sel = (u & 1) ? 0x7632u : 0x5410u;
          uint4 o;
          if (OP == 0 && ILV) {      // features 0,4 | 1,5 | 2,6 | 3,7 (see GemmProblem)
            o.x = __byte_perm(f[0], f[4], sel);
            o.y = __byte_perm(f[1], f[5], sel);
            o.z = __byte_perm(f[2], f[6], sel);
            o.w = __byte_perm(f[3], f[7], sel);
          } else {
            o.x = __byte_perm(f[0], f[1], sel);
            o.y = __byte_perm(f[2], f[3], sel);
            o.z = __byte_perm(f[4], f[5], sel);
            o.w = __byte_perm(f[6], f[7], sel);
          }
          *reinterpret_cast<uint4*>(args.out + (size_t)(U.p0 + tt) * N + U.fout[0] + ch * 8) = o;
        }
      }
      named_barrier_sync(1, ET);                      // staging tile free again
    }
    if (ov) atomicOr(args.err, kErrRange);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == W_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <int OP, bool ILV, bool STMA>
static cudaError_t launch_tc_impl(const GemmProblem& p, const Schedule& sch, cudaStream_t s) {
  CUtensorMap m0, m1;
  const uint64_t rows = (uint64_t)p.E * p.N;
  constexpr int RK = tc::raw_k_stages<STMA>();
  const CUtensorMapSwizzle raw_sw = RK == 1 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_64B;
  if (encode_tmap_2d(&m0, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.q0, p.K / 2, rows, p.K / 2,
                     RK * tc::BK / 2, tc::BM, raw_sw,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  m1 = m0;
  // B rows: grouped fp16 rows [S][K] (the gathered copy of x, or h)
  CUtensorMap mb;
  const uint16_t* brows = OP == 0 ? p.a16 : p.a;
  CUtensorMap mb128;
  if (encode_tmap_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, brows, p.K, p.S, (uint64_t)p.K * 2,
                     tc::BK, tc::NT, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_128B) != CUDA_SUCCESS ||
      encode_tmap_2d(&mb128, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, brows, p.K, p.S, (uint64_t)p.K * 2,
                     tc::BK, 128, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (OP == 0 &&
      encode_tmap_2d(&m1, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.q1, p.K / 2, rows, p.K / 2,
                     RK * tc::BK / 2, tc::BM, raw_sw,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  // group scales [E * N][K / G] fp16, blocks of 8 groups x 128 rows
  CUtensorMap ms0 = m0, ms1 = m0;
  if (STMA) {
    const int KG = p.K / p.G;
    if (encode_tmap_2d(&ms0, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, p.s0, KG, rows, (uint64_t)KG * 2,
                       tc::SC_GROUPS, tc::BM, CU_TENSOR_MAP_SWIZZLE_NONE,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_128B) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    ms1 = ms0;
    if (OP == 0 &&
        encode_tmap_2d(&ms1, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, p.s1, KG, rows, (uint64_t)KG * 2,
                       tc::SC_GROUPS, tc::BM, CU_TENSOR_MAP_SWIZZLE_NONE,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_128B) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    cudaError_t e = cudaFuncSetAttribute(moe_gemm_q4_tc_kernel<OP, ILV, STMA>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         tc::Lay<OP, RK>::SMEM);
    if (e != cudaSuccess) return e;
  }
  const int num_sms = sm_count();
  if (OP == 0) {
    // the gate/up B operand: fp16 rows of x in grouped order
    long blocks = (p.S + 7) / 8;                     // 8 rows (warps) per block
    if (blocks > 16L * num_sms) blocks = 16L * num_sms;
    gather_rows_f16_kernel<<<(int)blocks, 256, 0, s>>>(p.a, p.sorted_token, p.T, p.K, p.S, p.a16,
                                                       p.err);
  }
  TcArgs a;
  a.a = brows;
  a.sorted_token = p.sorted_token;
  a.offsets = p.offsets;
  a.tile_table = sch.tile_table;
  a.total_tiles = sch.tile_prefix + p.E;
  a.s0 = p.s0;
  a.s1 = p.s1;
  a.row_scale = p.row_scale;
  a.out = p.out;
  a.K = p.K;
  a.N = p.N;
  a.G = p.G;
  a.E = p.E;
  a.a_rows = OP == 0 ? p.T : p.S;
  a.err = p.err;
  const int FB = OP == 0 ? p.N / tc::BM : (p.N + 2 * tc::BM - 1) / (2 * tc::BM);
  const long max_units = (long)max_tiles(p.S, p.E) * FB;
  const int grid = (int)(max_units < num_sms ? max_units : num_sms);
  moe_gemm_q4_tc_kernel<OP, ILV, STMA><<<grid, tc::Roles<OP>::THREADS, tc::Lay<OP, RK>::SMEM, s>>>(
      m0, m1, mb, mb128, ms0, ms1, a);
  return cudaGetLastError();
}

cudaError_t launch_gemm_tc(const GemmProblem& p, const Schedule& sch, cudaStream_t s) {
  // scales by TMA when a row's K / G groups make whole 16-byte blocks
  const bool st = (p.K / p.G) % tc::SC_GROUPS == 0;
  if (p.op == 0) {
    if (st)
      return p.h_interleaved ? launch_tc_impl<0, true, true>(p, sch, s)
                             : launch_tc_impl<0, false, true>(p, sch, s);
    return p.h_interleaved ? launch_tc_impl<0, true, false>(p, sch, s)
                           : launch_tc_impl<0, false, false>(p, sch, s);
  }
  if (st)
    return p.h_interleaved ? launch_tc_impl<1, true, true>(p, sch, s)
                           : launch_tc_impl<1, false, true>(p, sch, s);
  return p.h_interleaved ? launch_tc_impl<1, true, false>(p, sch, s)
                         : launch_tc_impl<1, false, false>(p, sch, s);
}

}  // namespace strata
