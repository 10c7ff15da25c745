// combine.cu -- weighted scatter-combine of the per-row expert outputs back
// to token order:  y[t] = sum_{j<k} w[t][j] * rows[slot_row[t*k+j]].
//
// Memory bound (reads T*k fp16 rows of d values, writes T bf16 rows).  One CTA of 128
// threads per token row; each thread owns 8 consecutive features and reads
// them with 16-byte loads from all k rows before accumulating in fp32 in the
// fixed order j = 0..k-1 (deterministic, no atomics), then rounds once.
#include "common.cuh"
#include "internal.h"

namespace strata {

__global__ void __launch_bounds__(128)
    combine_kernel(const uint16_t* __restrict__ rows, const float* __restrict__ w,
                   const int32_t* __restrict__ slot_row, int T, int k, int d, int S,
                   uint16_t* __restrict__ y, unsigned* err) {
  const int t = blockIdx.x;
  __shared__ int32_t s_row[32];
  __shared__ float s_w[32];
  if (threadIdx.x < k) {
    int r = slot_row[(size_t)t * k + threadIdx.x];
    if ((unsigned)r >= (unsigned)S) {
      atomicOr(err, kErrIndex);
      r = 0;
    }
    s_row[threadIdx.x] = r;
    s_w[threadIdx.x] = w ? w[(size_t)t * k + threadIdx.x] : 1.0f;
  }
  __syncthreads();
  for (int f = threadIdx.x * 8; f < d; f += blockDim.x * 8) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    int j = 0;
    for (; j + 4 <= k; j += 4) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        v[u] = __ldg(reinterpret_cast<const uint4*>(rows + (size_t)s_row[j + u] * d + f));
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float wj = s_w[j + u];
        const uint32_t p[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[2 * i] = fmaf(wj, f16_lo(p[i]), acc[2 * i]);
          acc[2 * i + 1] = fmaf(wj, f16_hi(p[i]), acc[2 * i + 1]);
        }
      }
    }
    for (; j < k; ++j) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(rows + (size_t)s_row[j] * d + f));
      const float wj = s_w[j];
      const uint32_t p[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] = fmaf(wj, f16_lo(p[i]), acc[2 * i]);
        acc[2 * i + 1] = fmaf(wj, f16_hi(p[i]), acc[2 * i + 1]);
      }
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(y + (size_t)t * d + f) = o;
  }
}

cudaError_t launch_combine_checked(const uint16_t* rows, const float* w, const int32_t* slot_row,
                                   int T, int k, int d, uint16_t* y, unsigned* err,
                                   cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  combine_kernel<<<T, 128, 0, s>>>(rows, w, slot_row, T, k, d, T * k, y, err);
  return cudaGetLastError();
}

// dst[i] = src[index[i]] for rows of `width` 16-bit values (width % 8 == 0):
// one warp per row, 16-byte loads and stores.  Indices outside [0, src_rows)
// are reported (kErrIndex) and read row 0.
__global__ void __launch_bounds__(256)
    gather_rows_kernel(const uint16_t* __restrict__ src, const int32_t* __restrict__ index,
                       int src_rows, int rows, int width, uint16_t* __restrict__ dst,
                       unsigned* err) {
  const int lane = threadIdx.x & 31;
  const int cpr = width / 8;
  bool bad = false;
  for (int i = blockIdx.x * 8 + (threadIdx.x >> 5); i < rows; i += gridDim.x * 8) {
    int r = index[i];
    if ((unsigned)r >= (unsigned)src_rows) {
      bad = true;
      r = 0;
    }
    const uint4* s4 = reinterpret_cast<const uint4*>(src + (size_t)r * width);
    uint4* d4 = reinterpret_cast<uint4*>(dst + (size_t)i * width);
    for (int c = lane; c < cpr; c += 32) d4[c] = __ldg(s4 + c);
  }
  if (bad) atomicOr(err, kErrIndex);
}

cudaError_t launch_gather_rows(const uint16_t* src, const int32_t* index, int src_rows,
                               int rows, int width, uint16_t* dst, unsigned* err,
                               cudaStream_t s) {
  if (rows == 0) return cudaSuccess;
  long blocks = (rows + 7) / 8;
  if (blocks > 16L * sm_count()) blocks = 16L * sm_count();
  gather_rows_kernel<<<(int)blocks, 256, 0, s>>>(src, index, src_rows, rows, width, dst, err);
  return cudaGetLastError();
}

}  // namespace strata
