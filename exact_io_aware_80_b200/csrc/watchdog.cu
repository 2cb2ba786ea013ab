// watchdog.cu -- self-test of the kernels' bounded waits.
//
// Every mbarrier wait in the tensor-core kernels gives up after a limit,
// records FA_ERR_TIMEOUT in the device status word and lets the kernel
// return, so a lost arrival cannot hang the GPU.  This kernel exercises that
// path on purpose without any fault: it waits on a barrier that nothing ever
// arrives on, with a short limit, through the same routine the attention
// kernels use.
#include <cuda_runtime.h>

#include "fa.h"
#include "kernels.h"
#include "sm100.cuh"

namespace fa {
namespace {

__global__ void watchdog_selftest_kernel(int* status, long long limit_cycles) {
  __shared__ __align__(8) unsigned long long bar_word;
  __shared__ int abort_flag;
  const uint32_t bar = smem_u32(&bar_word);
  if (threadIdx.x == 0) {
    sm100::mbar_init(bar, 1);
    abort_flag = 0;
    sm100::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) sm100::mbar_wait(bar, 0, &abort_flag, status, limit_cycles);  // nothing arrives
  __syncthreads();
}

}  // namespace

cudaError_t launch_watchdog_selftest(int* status, int limit_us, cudaStream_t s) {
  int dev = 0, khz = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&khz, cudaDevAttrClockRate, dev) != cudaSuccess ||
      khz <= 0)
    khz = 2000000;
  const long long cycles = (long long)limit_us * (khz / 1000);
  watchdog_selftest_kernel<<<1, 32, 0, s>>>(status, cycles);
  return cudaGetLastError();
}

}  // namespace fa
