// Self-test of the bounded waits that every kernel of the library relies on.
//
// One thread waits on a fresh mbarrier that nothing ever arrives on; the wait
// must give up after its time limit, mark the device error word (timeout bit)
// and return, so the call's failure reaches the host through fa_device_status()
// and the context stays usable.  This exercises the same wait routine the
// forward, decode, FP8 and backward kernels use.
#include <cstdint>

#include "fa_internal.h"
#include "ptx_sm100.cuh"
#include "../../include/fa.h"

namespace fa {
namespace {

__global__ void fa_wait_selftest_kernel(int* err, uint64_t limit_ns, int* gave_up) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // parity 0 of a fresh barrier completes only after one arrival: none comes
    const bool ok = mbar_wait(smem_u32(&bar), 0, &abort_flag, err, limit_ns);
    if (gave_up) *gave_up = ok ? 0 : 1;
  }
}

}  // namespace

int launch_wait_selftest(unsigned limit_us, int* gave_up, cudaStream_t stream, int device) {
  int* err = device_error_word(device);
  if (!err) return set_error(FA_ERR_CUDA, "device error word unavailable");
  fa_wait_selftest_kernel<<<1, 32, 0, stream>>>(err, static_cast<uint64_t>(limit_us) * 1000ull,
                                                gave_up);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return set_error(FA_ERR_CUDA, "self-test launch: %s", cudaGetErrorString(e));
  return FA_OK;
}

}  // namespace fa
