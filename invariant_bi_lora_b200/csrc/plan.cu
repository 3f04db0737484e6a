// plan.cu -- multi-adapter token plan: stable counting sort of the tokens
// by adapter id (histogram -> exclusive scan -> stable scatter), integer
// work, bit-exact by construction.  Each adapter's tokens then form a
// contiguous segment that the segmented shrink / expand cut into row tiles
// of one adapter each ("Reproducible LoRA Inference Through Deterministic
// Split-K Reduction", Q&A: the LoRA kernels of a serving engine, many
// adapters in one batch).  Besides perm and the segment offsets the plan
// holds a table of 64-row tiles (adapter, rows, token ids; layout in
// common.cuh), so that a shrink CTA learns its adapter and all its token
// rows from one read.
//
// One CTA of 1024 threads.  Tokens are taken in chunks of 4096: warp w owns
// tokens chunk + 128w .. + 127, lane l the four tokens chunk + 128w + 32j + l
// (j = 0..3), so every load is a coalesced 128-byte line and the warp sees
// its tokens in index order j by j.  Within a warp, __match_any_sync groups
// the lanes of one class: a token's rank is the number of same-class lanes
// below it plus the warp's running count of that class, and one lane per
// class adds the group's size (no per-token atomics).  A per-class scan
// over the 32 warps turns the per-warp counts into bases, which keeps the
// sort stable.  The class histogram of the whole input comes first (the
// same warp aggregation), so the segment offsets are known before the
// scatter.
#include "common.cuh"

namespace bi {

constexpr int kPlanThreads = 1024;
constexpr int kPlanWarps = kPlanThreads / 32;
constexpr int kPlanPer = 4;                           // tokens per thread per chunk
constexpr int kPlanChunk = kPlanThreads * kPlanPer;

BI_DEV int plan_class(int a, int n_ad) { return (a >= 0 && a < n_ad) ? a : n_ad; }

// Classes of this thread's four tokens of a chunk (j-major inside the warp),
// -1 past the end.
BI_DEV void plan_load(const int32_t *__restrict__ ids, int M, int n_ad, int chunk, int warp, int lane,
                      int (&cls)[kPlanPer]) {
  int v[kPlanPer];
#pragma unroll
  for (int j = 0; j < kPlanPer; j++) {
    const int t = chunk + warp * (32 * kPlanPer) + 32 * j + lane;
    v[j] = t < M ? ids[t] : 0;
  }
#pragma unroll
  for (int j = 0; j < kPlanPer; j++) {
    const int t = chunk + warp * (32 * kPlanPer) + 32 * j + lane;
    cls[j] = t < M ? plan_class(v[j], n_ad) : -1;
  }
}

// Stable rank of each of the thread's tokens among the warp's tokens of its
// class (j by j, lanes in order), and the warp's count of every class in
// mine[] (zeroed here).
BI_DEV void plan_rank(const int (&cls)[kPlanPer], int *mine, int ncls, int lane, unsigned lt_mask,
                      int (&rank)[kPlanPer]) {
  for (int i = lane; i < ncls; i += 32) mine[i] = 0;
  __syncwarp();
#pragma unroll
  for (int j = 0; j < kPlanPer; j++) {
    const unsigned peers = __match_any_sync(0xffffffffu, cls[j]);
    rank[j] = __popc(peers & lt_mask) + (cls[j] >= 0 ? mine[cls[j]] : 0);
    __syncwarp();
    if (cls[j] >= 0 && (peers & lt_mask) == 0) mine[cls[j]] += __popc(peers);
    __syncwarp();
  }
}

// At most 32 classes and at most one chunk (n_ad <= 31, M <= 4096), the
// common serving case: a single pass with two block barriers.  A warp
// ranks its tokens with one ballot per class and j (no shared-memory
// atomics, no match), lane c of the warp records the warp's count of class
// c, and warp 0 alone turns the 32 x ncls counts into warp bases, segment
// starts and table bases (ncls lanes, a shuffle scan).
__global__ void __launch_bounds__(kPlanThreads, 1)
plan_small_kernel(const int32_t *__restrict__ ids, int M, int n_ad, int32_t *__restrict__ plan) {
  __shared__ int wc[kPlanWarps][33];     // warp counts, then warp bases
  __shared__ int s_off[33], s_tbase[33], s_cnt[33];
  const int ncls = n_ad + 1;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned lt_mask = (1u << lane) - 1u;
  int32_t *perm = plan;
  int32_t *offsets = plan + M;
  int32_t *table = plan + plan_table_word(M, n_ad);
  const int ntiles = (int)plan_tiles(M, n_ad);

  int cls[kPlanPer];
  plan_load(ids, M, n_ad, 0, warp, lane, cls);
  int rank[kPlanPer] = {0, 0, 0, 0};
  int mycount = 0;                                    // lane c: the warp's tokens of class c
  for (int c = 0; c < ncls; c++) {
    int run = 0;
#pragma unroll
    for (int j = 0; j < kPlanPer; j++) {
      const unsigned m = __ballot_sync(0xffffffffu, cls[j] == c);
      if (cls[j] == c) rank[j] = run + __popc(m & lt_mask);
      run += __popc(m);
    }
    if (lane == c) mycount = run;
  }
  if (lane < ncls) wc[warp][lane] = mycount;
  __syncthreads();
  if (warp == 0) {
    // lane c: its class's warp bases (in place) and total
    int total = 0;
    if (lane < ncls) {
#pragma unroll 8
      for (int w = 0; w < kPlanWarps; w++) {
        const int n = wc[w][lane];
        wc[w][lane] = total;
        total += n;
      }
    }
    const int tv = (total + kPlanTile - 1) / kPlanTile;
    int vin = total, tin = tv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, vin, o), b = __shfl_up_sync(0xffffffffu, tin, o);
      if (lane >= o) vin += a, tin += b;
    }
    if (lane < ncls) {
      s_off[lane] = vin - total;
      s_tbase[lane] = tin - tv;
      s_cnt[lane] = total;
      offsets[lane] = vin - total;
    }
    if (lane == ncls - 1) {
      s_off[ncls] = vin;
      s_tbase[ncls] = tin;
      offsets[ncls] = vin;
    }
    if (lane < plan_table_word(M, n_ad) - (M + ncls + 1)) plan[M + ncls + 1 + lane] = 0;   // padding
  }
  __syncthreads();
  // table headers and the unused id slots, one warp per record
  const int used = s_tbase[ncls];
  for (int i = warp; i < ntiles; i += kPlanWarps) {
    int a = -1, rows = 0, first = 0;
    if (i < used) {
      int lo = 0;
      while (lo + 1 < ncls && s_tbase[lo + 1] <= i) lo++;
      const int j = i - s_tbase[lo];
      a = lo;
      rows = min(kPlanTile, s_cnt[lo] - kPlanTile * j);
      first = s_off[lo] + kPlanTile * j;
    }
    int32_t *rec = table + (size_t)i * kPlanRec;
    if (lane == 0) *reinterpret_cast<int4 *>(rec) = make_int4(a, rows, first, 0);
    for (int s = rows + lane; s < kPlanTile; s += 32) rec[4 + s] = -1;
  }
  // stable scatter
#pragma unroll
  for (int j = 0; j < kPlanPer; j++) {
    if (cls[j] < 0) continue;
    const int t = warp * (32 * kPlanPer) + 32 * j + lane;
    const int sp = wc[warp][cls[j]] + rank[j];          // position inside the segment
    perm[s_off[cls[j]] + sp] = t;
    table[(size_t)(s_tbase[cls[j]] + sp / kPlanTile) * kPlanRec + 4 + sp % kPlanTile] = t;
  }
}

// Shared memory (ints): hist[ncls], off[ncls + 1], tbase[ncls + 1],
// base[ncls], wsum[2][32], wc[32][ncls].
__global__ void __launch_bounds__(kPlanThreads, 1)
plan_kernel(const int32_t *__restrict__ ids, int M, int n_ad, int32_t *__restrict__ plan) {
  extern __shared__ int plan_smem[];
  const int ncls = n_ad + 1;
  int *hist = plan_smem;                 // tokens per class
  int *off = hist + ncls;                // segment starts (+ total)
  int *tbase = off + ncls + 1;           // first table record of each class (+ total)
  int *base = tbase + ncls + 1;          // next free perm position of each class
  int *wsum = base + ncls;               // scan carries [2][32]
  int *wc = wsum + 64;                   // [32 warps][ncls]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned lt_mask = (1u << lane) - 1u;
  int *mine = wc + warp * ncls;

  int32_t *perm = plan;
  int32_t *offsets = plan + M;
  int32_t *table = plan + plan_table_word(M, n_ad);
  const int ntiles = (int)plan_tiles(M, n_ad);
  const bool one_chunk = M <= kPlanChunk;

  // ---- class histogram.  One chunk: the rank pass counts it per warp and
  // its bases come straight from those counts.  More: a counting pass first.
  int cls[kPlanPer], rank[kPlanPer];
  plan_load(ids, M, n_ad, 0, warp, lane, cls);
  if (one_chunk) {
    plan_rank(cls, mine, ncls, lane, lt_mask, rank);
    __syncthreads();
    // per class: warp counts -> exclusive bases inside the class (in place)
    for (int c = tid; c < ncls; c += kPlanThreads) {
      int run = 0;
#pragma unroll 8
      for (int w = 0; w < kPlanWarps; w++) {
        const int n = wc[w * ncls + c];
        wc[w * ncls + c] = run;
        run += n;
      }
      hist[c] = run;
    }
  } else {
    for (int i = tid; i < ncls; i += kPlanThreads) hist[i] = 0;
    __syncthreads();
    for (int chunk = 0; chunk < M; chunk += kPlanChunk) {
      int cc[kPlanPer];
      if (chunk == 0) {
#pragma unroll
        for (int j = 0; j < kPlanPer; j++) cc[j] = cls[j];
      } else {
        plan_load(ids, M, n_ad, chunk, warp, lane, cc);
      }
#pragma unroll
      for (int j = 0; j < kPlanPer; j++) {
        const unsigned peers = __match_any_sync(0xffffffffu, cc[j]);
        if (cc[j] >= 0 && (peers & lt_mask) == 0) atomicAdd(&hist[cc[j]], __popc(peers));
      }
    }
  }
  __syncthreads();

  // ---- exclusive scans over the classes: segment starts and table bases
  const int cls_warps = (ncls + 31) / 32;          // <= 9
  int v = 0, tv = 0, vin = 0, tin = 0;
  if (warp < cls_warps) {
    const int c = tid;
    v = c < ncls ? hist[c] : 0;
    tv = (v + kPlanTile - 1) / kPlanTile;
    vin = v, tin = tv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, vin, o), b = __shfl_up_sync(0xffffffffu, tin, o);
      if (lane >= o) vin += a, tin += b;
    }
    if (lane == 31) wsum[warp] = vin, wsum[32 + warp] = tin;
  }
  __syncthreads();
  if (warp < cls_warps) {
    for (int w = 0; w < warp; w++) vin += wsum[w], tin += wsum[32 + w];
    const int c = tid;
    if (c < ncls) {
      off[c] = vin - v;
      base[c] = vin - v;
      tbase[c] = tin - tv;
      offsets[c] = vin - v;
      if (c == ncls - 1) {
        off[ncls] = vin;
        tbase[ncls] = tin;
        offsets[ncls] = vin;
        for (long w = (long)M + ncls + 1; w < plan_table_word(M, n_ad); w++) plan[w] = 0;   // padding
      }
    }
  }
  __syncthreads();

  // ---- one warp per table record: header, and -1 in the unused id slots
  const int used = tbase[ncls];
  for (int i = warp; i < ntiles; i += kPlanWarps) {
    int a = -1, rows = 0, first = 0;
    if (i < used) {
      int lo = 0, hi = ncls - 1;                     // largest c with tbase[c] <= i
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tbase[mid] <= i) lo = mid; else hi = mid - 1;
      }
      const int j = i - tbase[lo];
      a = lo;
      rows = min(kPlanTile, hist[lo] - kPlanTile * j);
      first = off[lo] + kPlanTile * j;
    }
    int32_t *rec = table + (size_t)i * kPlanRec;
    if (lane == 0) *reinterpret_cast<int4 *>(rec) = make_int4(a, rows, first, 0);
    for (int s = rows + lane; s < kPlanTile; s += 32) rec[4 + s] = -1;
  }

  // ---- stable scatter
  auto scatter = [&](int chunk, const int (&cc)[kPlanPer], const int (&rk)[kPlanPer]) {
#pragma unroll
    for (int j = 0; j < kPlanPer; j++) {
      if (cc[j] < 0) continue;
      const int t = chunk + warp * (32 * kPlanPer) + 32 * j + lane;
      const int pos = off[cc[j]] + mine[cc[j]] + rk[j];
      perm[pos] = t;
      const int sp = pos - off[cc[j]];
      table[(size_t)(tbase[cc[j]] + sp / kPlanTile) * kPlanRec + 4 + sp % kPlanTile] = t;
    }
  };
  if (one_chunk) {
    scatter(0, cls, rank);
    return;
  }
  // several chunks: bases run on from chunk to chunk (base[] = next free
  // position of each class, relative to its segment start)
  for (int c = tid; c < ncls; c += kPlanThreads) base[c] = 0;
  __syncthreads();
  for (int chunk = 0; chunk < M; chunk += kPlanChunk) {
    int cc[kPlanPer], rk[kPlanPer];
    if (chunk == 0) {
#pragma unroll
      for (int j = 0; j < kPlanPer; j++) cc[j] = cls[j];
    } else {
      plan_load(ids, M, n_ad, chunk, warp, lane, cc);
    }
    plan_rank(cc, mine, ncls, lane, lt_mask, rk);
    __syncthreads();
    for (int c = tid; c < ncls; c += kPlanThreads) {
      int run = base[c];
#pragma unroll 8
      for (int w = 0; w < kPlanWarps; w++) {
        const int n = wc[w * ncls + c];
        wc[w * ncls + c] = run;
        run += n;
      }
      base[c] = run;
    }
    __syncthreads();
    scatter(chunk, cc, rk);
    __syncthreads();                                 // wc is rewritten by the next chunk
  }
}

}  // namespace bi

extern "C" size_t bi_lora_plan_bytes(int M, int n_adapters) {
  if (M < 0 || n_adapters < 1) return 0;
  return sizeof(int32_t) * (size_t)bi::plan_words(M, n_adapters);
}

extern "C" bi_status bi_lora_plan(const int32_t *ids, int M, int n_adapters, void *plan,
                                  size_t plan_bytes, bi_stream_t stream) {
  if (M < 0 || n_adapters < 1 || n_adapters > bi::kMaxAdapters) return BI_ERR_INVALID_ARG;
  if (!plan || (M > 0 && !ids)) return BI_ERR_INVALID_ARG;
  if (plan_bytes < bi_lora_plan_bytes(M, n_adapters)) return BI_ERR_WORKSPACE;
  if (!bi_aligned16(plan)) return BI_ERR_UNSUPPORTED_SHAPE;
  const int ncls = n_adapters + 1;
  const size_t smem = sizeof(int) * ((size_t)ncls * 4 + 2 + 64 + (size_t)bi::kPlanWarps * ncls);
  if (n_adapters <= 31 && M <= bi::kPlanChunk)
    bi::plan_small_kernel<<<1, bi::kPlanThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        ids, M, n_adapters, static_cast<int32_t *>(plan));
  else
    bi::plan_kernel<<<1, bi::kPlanThreads, smem, reinterpret_cast<cudaStream_t>(stream)>>>(
        ids, M, n_adapters, static_cast<int32_t *>(plan));
  return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}
