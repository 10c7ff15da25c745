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

}  // namespace strata
