// permute.cu -- grouping of token slots by expert, and the per-expert work
// lists the expert GEMMs read.
//
// Tokens that chose the same expert are processed together, so each expert's
// weights are read once for all its tokens (kongchang.com "两天移植，预填充提速
// 8倍：Strata引擎实测", section "Strata快在哪": bigger batches mean more tokens
// reuse every expert).  The grouping is a stable counting sort of the T*k
// slots by expert id:
//   1. histogram per chunk of kPermChunk slots (shared-memory counters);
//   2. one block scans the chunk histograms per expert (column prefix) and
//      the expert totals (exclusive scan -> offsets);
//   3. one warp per chunk walks its slots in order; lanes that share an
//      expert are ranked with __match_any_sync, so each row is the slot's rank
//      among earlier slots of the same expert.
// Every step is integer-only and deterministic.
#include "common.cuh"
#include "internal.h"

namespace strata {

__global__ void permute_count_kernel(const int32_t* __restrict__ ids, int S, int E,
                                     int32_t* __restrict__ hist, unsigned* err) {
  extern __shared__ int32_t cnt[];
  for (int i = threadIdx.x; i < E; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  const int s0 = blockIdx.x * kPermChunk;
  const int s1 = min(S, s0 + kPermChunk);
  for (int s = s0 + threadIdx.x; s < s1; s += blockDim.x) {
    int e = ids[s];
    if ((unsigned)e >= (unsigned)E) {
      atomicOr(err, kErrIndex);
      e = e < 0 ? 0 : E - 1;
    }
    atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < E; i += blockDim.x) hist[(size_t)blockIdx.x * E + i] = cnt[i];
}

// Exclusive scan of one value per thread over a block of up to 1024 threads.
// Returns the exclusive prefix; *total receives the block sum.
__device__ int block_exclusive_scan(int v, int* total) {
  __shared__ int warp_sums[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int inc = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, inc, off);
    if (lane >= off) inc += o;
  }
  if (lane == 31) warp_sums[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const int nw = (blockDim.x + 31) >> 5;
    int ws = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, ws, off);
      if (lane >= off) ws += o;
    }
    if (lane < nw) warp_sums[lane] = ws;       // inclusive prefix of warp sums
  }
  __syncthreads();
  const int before = warp > 0 ? warp_sums[warp - 1] : 0;
  *total = warp_sums[((blockDim.x + 31) >> 5) - 1];
  __syncthreads();
  return before + inc - v;
}

// One block of 1024 threads; thread e owns expert e.
__global__ void __launch_bounds__(1024)
    permute_scan_kernel(int32_t* __restrict__ hist, int nchunks, int E,
                        int32_t* __restrict__ counts, int32_t* __restrict__ offsets) {
  const int e = threadIdx.x;
  int c = 0;
  if (e < E)
    for (int ch = 0; ch < nchunks; ++ch) c += hist[(size_t)ch * E + e];
  int total;
  const int excl = block_exclusive_scan(c, &total);
  if (e < E) {
    counts[e] = c;
    offsets[e] = excl;
    int run = excl;
    for (int ch = 0; ch < nchunks; ++ch) {
      const int h = hist[(size_t)ch * E + e];
      hist[(size_t)ch * E + e] = run;      // first row of this chunk's slots of e
      run += h;
    }
  }
  if (e == 0) offsets[E] = total;
}

// One warp per chunk.  hist holds, per chunk and expert, the first row.
__global__ void __launch_bounds__(32)
    permute_scatter_kernel(const int32_t* __restrict__ ids, int S, int k, int E,
                           const int32_t* __restrict__ hist, int32_t* __restrict__ sorted_token,
                           int32_t* __restrict__ slot_row) {
  extern __shared__ int32_t next_row[];
  const int lane = threadIdx.x;
  for (int i = lane; i < E; i += 32) next_row[i] = hist[(size_t)blockIdx.x * E + i];
  __syncwarp();
  const int s0 = blockIdx.x * kPermChunk;
  const int s1 = min(S, s0 + kPermChunk);
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int sb = s0; sb < s1; sb += 32) {
    const int s = sb + lane;
    const bool valid = s < s1;
    int e = valid ? ids[s] : -1 - lane;           // invalid lanes never match
    if (valid && (unsigned)e >= (unsigned)E) e = e < 0 ? 0 : E - 1;
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & lt_mask);
    const int base = valid ? next_row[e] : 0;
    __syncwarp();
    if (valid && rank == 0) next_row[e] = base + __popc(peers);
    __syncwarp();
    if (valid) {
      const int p = base + rank;
      sorted_token[p] = s / k;
      slot_row[s] = p;
    }
  }
}

cudaError_t launch_permute(const int32_t* ids, int T, int k, int E, int32_t* counts,
                           int32_t* offsets, int32_t* sorted_token, int32_t* slot_row,
                           int32_t* hist, unsigned* err, cudaStream_t s) {
  const int S = T * k;
  const int nchunks = (S + kPermChunk - 1) / kPermChunk;
  const size_t sh = (size_t)E * sizeof(int32_t);
  permute_count_kernel<<<nchunks, 256, sh, s>>>(ids, S, E, hist, err);
  permute_scan_kernel<<<1, 1024, 0, s>>>(hist, nchunks, E, counts, offsets);
  permute_scatter_kernel<<<nchunks, 32, sh, s>>>(ids, S, k, E, hist, sorted_token, slot_row);
  return cudaGetLastError();
}

// Work lists for the expert GEMMs: tiles of tile_rows rows per expert, the
// table that maps a global tile index to (expert, tile in expert), and the
// ascending list of experts that received rows.  One block of 1024 threads.
// Offsets that are not a non-decreasing sequence from 0 to S are reported
// through the check word and leave every work list empty.
__global__ void __launch_bounds__(1024)
    schedule_kernel(const int32_t* __restrict__ offsets, int E, int S, int tile_rows,
                    Schedule sch, unsigned* err) {
  const int e = threadIdx.x;
  bool bad = false;
  if (e < E) bad = offsets[e] < 0 || offsets[e + 1] < offsets[e] || offsets[e + 1] > S;
  if (e == 0) bad = bad || offsets[0] != 0 || offsets[E] != S;
  bad = __syncthreads_or(bad);
  if (bad && e == 0) atomicOr(err, kErrIndex);
  const int cnt = (e < E && !bad) ? offsets[e + 1] - offsets[e] : 0;
  const int tiles = (cnt + tile_rows - 1) / tile_rows;
  int total_tiles, total_active;
  const int tp = block_exclusive_scan(tiles, &total_tiles);
  const int ap = block_exclusive_scan(cnt > 0 ? 1 : 0, &total_active);
  if (e < E) {
    sch.tile_prefix[e] = tp;
    for (int j = 0; j < tiles; ++j) {
      const int p0 = offsets[e] + j * tile_rows;
      sch.tile_table[tp + j] = make_int4(e, p0, min(tile_rows, cnt - j * tile_rows), 0);
    }
    if (cnt > 0) sch.active[ap] = e;
  }
  if (e == 0) {
    sch.tile_prefix[E] = total_tiles;
    *sch.n_active = total_active;
  }
}

cudaError_t launch_schedule(const int32_t* offsets, int E, int S, int tile_rows, Schedule sch,
                            unsigned* err, cudaStream_t s) {
  schedule_kernel<<<1, 1024, 0, s>>>(offsets, E, S, tile_rows, sch, err);
  return cudaGetLastError();
}

}  // namespace strata
