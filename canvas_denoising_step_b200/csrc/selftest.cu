// dg_selftest_bounded_wait: a self-test of the bounded waits that every
// kernel of the library uses.  One CTA waits on an mbarrier that nothing
// arrives on; the wait gives up after its time limit, records DG_ERR_TIMEOUT
// in an error word and the kernel returns normally, so the device stays usable.
#include "dg.h"
#include "dg_kernels.h"

namespace dg {
namespace {

__global__ void selftest_wait_kernel(int* err) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // phase 0 never completes: nothing arrives on the barrier
    if (mbar_wait(smem_u32(&bar), 0, &abort_flag, err)) raise_error(err, kErrFault);
  }
  __syncthreads();
}

}  // namespace
}  // namespace dg

extern "C" int dg_selftest_bounded_wait(void* cuda_stream) {
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  int* err = nullptr;
  if (cudaMalloc(&err, sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    return DG_ERR_OOM;
  }
  int host = 0;
  cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int), s);
  if (e == cudaSuccess) {
    dg::selftest_wait_kernel<<<1, 32, 0, s>>>(err);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaMemcpyAsync(&host, err, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  cudaFree(err);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return DG_ERR_CUDA;
  }
  return host == 0 ? DG_OK : host;
}
