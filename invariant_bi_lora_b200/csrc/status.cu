// status.cu -- device status word, status strings, bounded-wait self-test.
//
// Kernels that wait (on an mbarrier, a flag, a peer) give up after a fixed
// number of polls; they then record BI_ERR_TIMEOUT here instead of trapping,
// and return, so the context stays usable and the host can report it.
#include "common.cuh"

#include <mutex>

namespace bi {

__device__ unsigned g_status_word;

static std::mutex g_status_mu;
static unsigned *g_status_ptr[64];

unsigned *status_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_status_mu);
  if (!g_status_ptr[dev]) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_status_word) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<unsigned *>(ptr);
  }
  return g_status_ptr[dev];
}

// One CTA polls a flag in shared memory that nothing sets, at most
// max_polls times, then records the timeout.  Exercises the same give-up
// path the pipelined kernels use, without hanging anything.
__global__ void bounded_wait_kernel(unsigned *status, int max_polls) {
  __shared__ volatile int flag;
  if (threadIdx.x == 0) flag = 0;
  __syncthreads();
  int polls = 0;
  while (flag == 0) {
    if (++polls >= max_polls) {
      if (threadIdx.x == 0) flag_error(status, BI_ERR_TIMEOUT);
      break;
    }
    __nanosleep(32);
  }
}

}  // namespace bi

extern "C" bi_status bi_get_device_status(bi_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned *ptr = bi::status_word();
  if (!ptr) return BI_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return BI_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpy(&v, ptr, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return BI_ERR_CUDA;
  const unsigned zero = 0;
  if (cudaMemcpy(ptr, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return BI_ERR_CUDA;
  return static_cast<bi_status>(v);
}

extern "C" const char *bi_status_string(int status) {
  switch (status) {
    case BI_OK: return "BI_OK";
    case BI_ERR_INVALID_ARG: return "BI_ERR_INVALID_ARG";
    case BI_ERR_UNSUPPORTED_SHAPE: return "BI_ERR_UNSUPPORTED_SHAPE";
    case BI_ERR_WORKSPACE: return "BI_ERR_WORKSPACE";
    case BI_ERR_CUDA: return "BI_ERR_CUDA";
    case BI_ERR_TIMEOUT: return "BI_ERR_TIMEOUT";
    case BI_ERR_NO_DEVICE: return "BI_ERR_NO_DEVICE";
    default: return "BI_ERR_UNKNOWN";
  }
}

extern "C" bi_status bi_selftest_bounded_wait(int max_polls, bi_stream_t stream) {
  if (max_polls < 1) return BI_ERR_INVALID_ARG;
  unsigned *ptr = bi::status_word();
  if (!ptr) return BI_ERR_CUDA;
  bi::bounded_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(ptr, max_polls);
  return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}
