// selftest.cu -- runs the library's bounded waits into their time limit on
// purpose, so that the give-up path (record kErrTimeout, raise the abort
// flag, release what the kernel holds, return) is exercised on the device.
// Each wait here is on a condition that nothing ever satisfies: an mbarrier
// that no thread or copy arrives on, a grid barrier that one CTA never
// reaches, and a counter of finished work that nothing raises.  Nothing
// traps and nothing waits without a limit.
#include "../../include/strata_moe.h"
#include "common.cuh"
#include "internal.h"

namespace strata {

// One CTA, four warps.  Warp 0 waits (one lane) on an mbarrier nobody
// arrives on; warps 1-3 wait (whole warp) on a second one.  Warp 1 holds
// 32 columns of tensor memory while it waits and frees them afterwards.
//   out[w]   1 if warp w's wait completed, 0 if it gave up
//   out[4]   nanoseconds warp 0 waited
//   out[5]   1 once warp 1 has released its tensor memory
__global__ void __launch_bounds__(128, 1) selftest_mbar_kernel(int32_t* out, unsigned* err) {
  __shared__ uint64_t bars[2];
  __shared__ uint32_t tmem_holder;
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&tmem_holder, 32);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  volatile int* ab = &abort_flag;
  if (warp == 0) {
    if (lane == 0) {
      const unsigned long long t0 = global_ns();
      const bool ok = mbar_wait(&bars[0], 0, ab, err);
      out[4] = (int32_t)min(global_ns() - t0, 2000000000ull);
      out[0] = ok ? 1 : 0;
    }
  } else {
    const bool ok = mbar_wait_warp(&bars[1], 0, ab, err);
    if (lane == 0) out[warp] = ok ? 1 : 0;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_holder, 32);
    if (lane == 0) out[5] = 1;
  }
}

// Two CTAs (cooperative launch); CTA 1 never arrives at the grid barrier
// (sync[0], abort word sync[2]).  Meanwhile CTA 1 waits for a counter that
// nothing raises (sync[4], abort word sync[6]).
//   out[6] 1 if CTA 0's barrier completed, 0 if it gave up
//   out[7] nanoseconds CTA 0 waited
//   out[8] 1 if CTA 1's counter wait completed, 0 if it gave up
//   out[9] nanoseconds CTA 1 waited
__global__ void selftest_grid_kernel(int32_t* out, unsigned* sync, unsigned* err) {
  __shared__ int cta_abort;
  if (threadIdx.x != 0) return;
  const unsigned long long t0 = global_ns();
  if (blockIdx.x == 0) {
    const bool ok = grid_barrier_wait(sync, 0, err);
    out[7] = (int32_t)min(global_ns() - t0, 2000000000ull);
    out[6] = ok ? 1 : 0;
  } else {
    cta_abort = 0;
    const bool ok = counter_wait(&sync[4], 1u, &sync[6], err, &cta_abort);
    out[9] = (int32_t)min(global_ns() - t0, 2000000000ull);
    out[8] = ok ? 1 : 0;
  }
}

unsigned* check_word();

}  // namespace strata

using namespace strata;

extern "C" strata_status_t strata_moe_selftest_wait(int32_t* out, void* sync_ws,
                                                    strata_stream_t stream) {
  if (out == nullptr || sync_ws == nullptr ||
      (reinterpret_cast<uintptr_t>(out) & 15u) != 0 ||
      (reinterpret_cast<uintptr_t>(sync_ws) & 15u) != 0)
    return STRATA_ERR_INVALID_ARG;
  unsigned* err = check_word();
  if (!err) return STRATA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned* sync = static_cast<unsigned*>(sync_ws);
  if (cudaMemsetAsync(out, 0, 10 * sizeof(int32_t), s) != cudaSuccess ||
      cudaMemsetAsync(sync, 0, 32, s) != cudaSuccess)
    return STRATA_ERR_CUDA;
  selftest_mbar_kernel<<<1, 128, 0, s>>>(out, err);
  if (cudaGetLastError() != cudaSuccess) return STRATA_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2);
  cfg.blockDim = dim3(32);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, selftest_grid_kernel, out, sync, err) != cudaSuccess)
    return STRATA_ERR_CUDA;
  return STRATA_OK;
}
