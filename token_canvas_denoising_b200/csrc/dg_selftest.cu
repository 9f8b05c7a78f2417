// Failure-detection self-test: a wait that nothing completes must give up,
// report a timeout through the device error word and let the kernel return.
#include "dg_internal.cuh"
#include "dg_ops.h"
#include "dg_sm100.cuh"

namespace dg {
namespace {

__global__ void selftest_wait_kernel(int* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    sm100::fence_barrier_init();
    // phase 0 never completes: nobody arrives on the barrier
    sm100::mbar_wait(&bar, 0, err, nullptr);
  }
}

}  // namespace
}  // namespace dg

extern "C" dg_status dg_selftest_wait_timeout(void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* err = nullptr;
  if (cudaMallocAsync(reinterpret_cast<void**>(&err), sizeof(int), s) != cudaSuccess) {
    cudaGetLastError();
    dg::set_last_error("cudaMallocAsync failed");
    return DG_ERR_CUDA;
  }
  int host = -1;
  cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int), s);
  if (e == cudaSuccess) {
    dg::selftest_wait_kernel<<<1, 32, 0, s>>>(err);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaMemcpyAsync(&host, err, sizeof(int), cudaMemcpyDeviceToHost, s);
  cudaFreeAsync(err, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    dg::set_last_error(std::string("self-test: ") + cudaGetErrorString(e));
    return DG_ERR_CUDA;
  }
  if (host == dg::kDevWaitTimeout) return DG_ERR_TIMEOUT;
  dg::set_last_error("self-test: the wait did not report a timeout (error word " + std::to_string(host) + ")");
  return host == 0 ? DG_OK : DG_ERR_DEVICE_CHECK;
}
