// plan.cu -- multi-adapter token plan: stable counting sort of the tokens
// by adapter id (histogram -> exclusive scan -> stable scatter), integer
// work, bit-exact by construction.  Each adapter's tokens then form a
// contiguous segment that the segmented shrink / expand cut into row tiles
// of one adapter each ("Reproducible LoRA Inference Through Deterministic
// Split-K Reduction", Q&A: the LoRA kernels of a serving engine, many
// adapters in one batch).
#include "common.cuh"

namespace bi {

constexpr int kPlanThreads = 1024;

// One CTA.  Classes 0..n_ad-1 are adapters, class n_ad collects tokens whose
// id is outside [0, n_ad).  Shared memory: counts / running bases
// [n_ad + 1] and per-warp class counts [32][n_ad + 1].
__global__ void __launch_bounds__(kPlanThreads)
plan_kernel(const int32_t *__restrict__ ids, int M, int n_ad, int32_t *__restrict__ perm,
            int32_t *__restrict__ offsets) {
  extern __shared__ int plan_smem[];
  const int ncls = n_ad + 1;
  int *base = plan_smem;              // [ncls]
  int *wc = plan_smem + ncls;         // [32][ncls]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  for (int i = tid; i < ncls; i += blockDim.x) base[i] = 0;
  __syncthreads();
  for (int t = tid; t < M; t += blockDim.x) {
    const int a = ids[t];
    atomicAdd(&base[(a >= 0 && a < n_ad) ? a : n_ad], 1);
  }
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int a = 0; a < ncls; a++) {
      const int cnt = base[a];
      offsets[a] = run;
      base[a] = run;
      run += cnt;
    }
    offsets[ncls] = run;
  }
  __syncthreads();

  const unsigned lt_mask = (1u << lane) - 1u;
  for (int chunk = 0; chunk < M; chunk += blockDim.x) {
    const int t = chunk + tid;
    const bool valid = t < M;
    int cls = -1;
    if (valid) {
      const int a = ids[t];
      cls = (a >= 0 && a < n_ad) ? a : n_ad;
    }
    for (int i = lane; i < ncls; i += 32) wc[warp * ncls + i] = 0;
    __syncwarp();
    const unsigned peers = __match_any_sync(0xffffffffu, cls);
    const int rank = __popc(peers & lt_mask);
    if (valid && rank == 0) wc[warp * ncls + cls] = __popc(peers);
    __syncthreads();
    if (valid) {
      int pos = base[cls] + rank;
      for (int w = 0; w < warp; w++) pos += wc[w * ncls + cls];
      perm[pos] = t;
    }
    __syncthreads();
    for (int i = tid; i < ncls; i += blockDim.x) {
      int add = 0;
      for (int w = 0; w < 32; w++) add += wc[w * ncls + i];
      base[i] += add;
    }
    __syncthreads();
  }
}

}  // namespace bi

extern "C" size_t bi_lora_plan_bytes(int M, int n_adapters) {
  if (M < 0 || n_adapters < 1) return 0;
  return sizeof(int32_t) * ((size_t)M + (size_t)n_adapters + 2);
}

extern "C" bi_status bi_lora_plan(const int32_t *ids, int M, int n_adapters, void *plan,
                                  size_t plan_bytes, bi_stream_t stream) {
  if (M < 0 || n_adapters < 1 || n_adapters > bi::kMaxAdapters) return BI_ERR_INVALID_ARG;
  if (!plan || (M > 0 && !ids)) return BI_ERR_INVALID_ARG;
  if (plan_bytes < bi_lora_plan_bytes(M, n_adapters)) return BI_ERR_WORKSPACE;
  if (((uintptr_t)plan & 3u) != 0) return BI_ERR_UNSUPPORTED_SHAPE;
  int32_t *perm = static_cast<int32_t *>(plan);
  const size_t smem = sizeof(int) * (size_t)(n_adapters + 1) * 33;
  bi::plan_kernel<<<1, bi::kPlanThreads, smem, reinterpret_cast<cudaStream_t>(stream)>>>(
      ids, M, n_adapters, perm, perm + M);
  return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}
