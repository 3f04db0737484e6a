// noalloc.cu -- segmented LoRA shrink for callers that cannot allocate.
//
// The regular multi-adapter path needs a token plan (the tokens grouped by
// adapter) in device memory that the caller allocates.  Some callers cannot
// do that: a plugin running inside a host application that owns every byte
// of device memory through its own pool and does not let libraries allocate,
// or a latency-critical serving loop where a cudaMalloc -- which may
// synchronise the whole device -- is not acceptable.  This entry point takes
// the adapter ids directly and keeps the plan in a fixed array of this
// library's own device memory instead.
//
// The scratch is a file-scope __device__ array that holds the largest plan
// (BI_NOALLOC_MAX_TOKENS tokens, 256 adapters: 152,904 int32, about 598 KiB);
// every GPU that loads the library holds it until the process exits.  Host code cannot use the array's name as a device address
// (on the host it names a stand-in object), so the first call on each device
// looks the address up with cudaGetSymbolAddress, with that device current,
// and caches it; that first call should therefore come before any stream
// capture on the device.  All calls share the one array and the next call
// overwrites it: calls whose kernels overlap on the GPU (other streams, other
// threads) race on it, so serialise them.  Nothing in the array has to start
// at zero: the plan kernel rewrites every entry a call reads.
#include "common.cuh"

#include <mutex>

namespace bi {

constexpr int kNoAllocMaxTokens = BI_NOALLOC_MAX_TOKENS;
constexpr int kNoAllocMaxAdapters = kMaxAdapters;

// A plan as bi_lora_plan lays it out (perm, offsets, tile table), at the
// largest size this entry point accepts.
static __device__ __align__(256) int32_t g_noalloc_plan[plan_words(kNoAllocMaxTokens, kNoAllocMaxAdapters)];

static std::mutex g_noalloc_mu;
static int32_t *g_noalloc_ptr[64];

// Device address of the scratch array on the current device (set-up on the
// first call per device).
static bi_status noalloc_scratch(int32_t **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return BI_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_plan) != cudaSuccess || !ptr) return BI_ERR_CUDA;
    g_noalloc_ptr[dev] = static_cast<int32_t *>(ptr);
  }
  *out = g_noalloc_ptr[dev];
  return BI_OK;
}

}  // namespace bi

extern "C" bi_status bi_lora_shrink_segmented_noalloc(const void *x, const void *A, const int32_t *ids,
                                                      int n_adapters, float *y, int M, int K, int r,
                                                      int splits, int mode, bi_stream_t stream) {
  if (M < 0 || n_adapters < 1) return BI_ERR_INVALID_ARG;
  if (M > bi::kNoAllocMaxTokens || n_adapters > bi::kNoAllocMaxAdapters) return BI_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return BI_OK;
  if (!ids) return BI_ERR_INVALID_ARG;
  int32_t *plan = nullptr;
  bi_status st = bi::noalloc_scratch(&plan);
  if (st != BI_OK) return st;
  const size_t plan_bytes = sizeof(int32_t) * (size_t)bi::plan_words(M, n_adapters);
  st = bi_lora_plan(ids, M, n_adapters, plan, plan_bytes, stream);
  if (st != BI_OK) return st;
  return bi_lora_shrink_segmented(x, A, plan, n_adapters, y, M, K, r, splits, mode, stream);
}
