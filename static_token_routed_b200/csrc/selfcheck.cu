// Check of the bounded-wait machinery every kernel relies on: a CTA waits on
// an mbarrier that nothing will ever complete, with the same bounded wait
// the kernels use. The wait must give up after its time limit, raise the
// CTA's abort flag, report DEV_ERR_TIMEOUT in global memory and return, so
// that the launch ends normally and the context stays usable. No trap, no
// fault, no unbounded loop: the only way this kernel ends is the time limit.
#include "l3_internal.cuh"
#include "sm100.cuh"

namespace l3 {
namespace {

__global__ void k_wait_never_completes(int *err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);  // one arrival expected; nobody arrives
    abort_flag = 0;
    sm100::fence_mbar_init();
  }
  __syncthreads();
  const sm100::Abort ab{&abort_flag, err};
  if (threadIdx.x == 0 && sm100::mbar_wait(&bar, 0, ab)) atomicOr(err, 1 << 30);  // cannot happen
}

}  // namespace
}  // namespace l3

using namespace l3;

extern "C" l3_status l3_check_bounded_wait(void *stream) {
  set_error("");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int *err = nullptr;
  L3_CUDA_TRY(cudaMalloc(&err, sizeof(int)));
  l3_status st = L3_OK;
  int host = 0;
  cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int), s);
  if (e == cudaSuccess) {
    k_wait_never_completes<<<1, 32, 0, s>>>(err);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaMemcpyAsync(&host, err, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  cudaFree(err);
  if (e != cudaSuccess) return cuda_fail(e, "l3_check_bounded_wait");
  if (host == DEV_ERR_TIMEOUT) {
    set_error("the bounded wait gave up as it should");
    st = L3_ERR_TIMEOUT;
  } else {
    set_error("the bounded wait did not report its give-up");
    st = L3_ERR_CUDA;
  }
  return st;
}
