// Self-test of the bounded device waits every kernel of the library uses.
//
// One CTA initialises an mbarrier that expects one arrival, never arrives on
// it, and waits for it with the same bounded wait the kernels use. The wait
// must give up after `limit_cycles` SM clocks and report it in a device word
// that the host reads; nothing faults and nothing hangs.
#include "../../include/fg.h"
#include "fg_internal.h"
#include "sm100_ptx.cuh"

namespace {

__global__ void bounded_wait_probe(long long limit_cycles, int32_t* word) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    fg::ptx::mbar_init(&bar, 1);
    fg::ptx::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool done = fg::ptx::mbar_wait_bounded(&bar, 0, limit_cycles);
    *word = done ? 0 : fg::kErrTimeout;
  }
}

}  // namespace

fg_status fg_set_error(fg_status st, const char* msg);

extern "C" fg_status fg_selftest_bounded_wait(int64_t limit_cycles, void* stream) {
  if (limit_cycles < 0 || limit_cycles > (int64_t)1 << 32)
    return fg_set_error(FG_ERR_INVALID_ARG, "limit_cycles must be in [0, 2^32]");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* word = nullptr;
  cudaError_t e = cudaMallocAsync(&word, sizeof(int32_t), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(word, 0xFF, sizeof(int32_t), st);
  if (e == cudaSuccess) {
    bounded_wait_probe<<<1, 32, 0, st>>>(limit_cycles, word);
    e = cudaGetLastError();
  }
  int32_t host = -1;
  if (e == cudaSuccess) e = cudaMemcpyAsync(&host, word, sizeof(int32_t), cudaMemcpyDeviceToHost, st);
  if (word) cudaFreeAsync(word, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return fg_set_error(FG_ERR_CUDA, cudaGetErrorString(e));
  if (host == fg::kErrTimeout) return fg_set_error(FG_ERR_TIMEOUT, "the bounded wait gave up, as designed");
  if (host == 0) return fg_set_error(FG_ERR_DEVICE_CHECK, "a wait with no arrival reported completion");
  return fg_set_error(FG_ERR_DEVICE_CHECK, "the probe did not report");
}
