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
#include "tc.cuh"

#include <algorithm>
#include <cooperative_groups.h>

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

// At most 32 classes and at most 4096 tokens (n_ad <= 31), the common
// serving case: one cluster of ceil(M / 512) CTAs of 4 warps, a warp per
// 128 tokens, so that the rank work of up to 32 warps runs on up to 8 SMs.
//  * Rank: a class fits in nb <= 5 bits, so one ballot per bit of the
//    j-th tokens gives every lane both the lanes whose token shares its
//    class (the AND of the bit masks, complemented where its bit is 0) and,
//    for lane c, the lanes whose token has class c.  Lane c keeps the
//    warp's running count of class c; a token's rank is that count (read
//    from lane cls by shuffle) plus its same-class lanes below it.
//  * Bases: every warp pushes its row of class counts into every CTA's
//    [warp][class] table (distributed shared memory), and after one
//    cluster barrier each warp scans the whole table itself (lane c: its
//    class's count in the warps before this one and in all warps; a
//    shuffle scan over the lanes gives the segment starts and table bases).
//  * Table: records are written as 17 16-byte quads (header, 16 quads of
//    token slots), spread over all threads; a slot quad is written only
//    where it holds unused (-1) slots, the scatter fills the rest.
constexpr int kPlanSmallWarps = 4;                  // per CTA
constexpr int kPlanSmallCtas = 8;                   // per cluster: 8 * 4 * 128 = 4096 tokens
constexpr int kPlanQuads = kPlanRec / 4;            // 17

__global__ void __launch_bounds__(32 * kPlanSmallWarps)
plan_small_kernel(const int32_t *__restrict__ ids, int M, int n_ad, int32_t *__restrict__ plan) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  __shared__ int wc[kPlanSmallCtas * kPlanSmallWarps][32];   // warp w's count of class c
  const int ncls = n_ad + 1, ncta = gridDim.x;       // the grid is one cluster
  const int lane = threadIdx.x & 31;
  const int warp = blockIdx.x * kPlanSmallWarps + (threadIdx.x >> 5), nw = ncta * kPlanSmallWarps;
  const unsigned lt_mask = (1u << lane) - 1u;
  int32_t *perm = plan;
  int32_t *offsets = plan + M;
  int32_t *table = plan + plan_table_word(M, n_ad);
  const int ntiles = (int)plan_tiles(M, n_ad);
  // every CTA has started once this arrive is matched; the wait comes
  // before the first write into a peer's shared memory
  cluster_arrive_relaxed();
  // start the output's address translation while the ids are in flight
  if (warp == 0 && lane == 0) asm volatile("prefetch.global.L2 [%0];" ::"l"(plan));
  if (warp == nw - 1 && lane == 0)
    asm volatile("prefetch.global.L2 [%0];" ::"l"(table + (size_t)ntiles * kPlanRec - 1));

  int cls[kPlanPer];
  plan_load(ids, M, n_ad, 0, warp, lane, cls);
  const int nb = 32 - __clz(ncls - 1);                // bits of the largest class, 1..5
  int rank[kPlanPer];
  int run = 0;                                        // lane c: the warp's tokens of class c so far
#pragma unroll
  for (int j = 0; j < kPlanPer; j++) {
    unsigned same = __ballot_sync(0xffffffffu, cls[j] >= 0), mine = same;
#pragma unroll
    for (int bit = 0; bit < 5; bit++) {
      if (bit < nb) {
        const unsigned m = __ballot_sync(0xffffffffu, (cls[j] >> bit) & 1);
        same &= ((cls[j] >> bit) & 1) ? m : ~m;
        mine &= ((lane >> bit) & 1) ? m : ~m;
      }
    }
    rank[j] = __shfl_sync(0xffffffffu, run, cls[j] & 31) + __popc(same & lt_mask);
    run += __popc(mine);
  }
  const int mycount = lane < ncls ? run : 0;
  cluster_wait();
  for (int r = 0; r < ncta; r++) *cluster.map_shared_rank(&wc[warp][lane], r) = mycount;
  cluster_arrive_release();
  cluster_wait_acquire();

  int before = 0, total = 0;                          // lane c: class c in warps < this one, in all
#pragma unroll 8
  for (int w = 0; w < nw; w++) {
    const int n = wc[w][lane];
    before += w < warp ? n : 0;
    total += n;
  }
  const int tv = (total + kPlanTile - 1) / kPlanTile;
  int vin = total, tin = tv;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, vin, o), y = __shfl_up_sync(0xffffffffu, tin, o);
    if (lane >= o) vin += x, tin += y;
  }
  // lane c: segment start and first record of class c (lanes >= ncls: the
  // totals, so the table bases stay non-decreasing over all 32 lanes)
  const int off = vin - total, tbase = tin - tv;
  const int used = __shfl_sync(0xffffffffu, tin, 31);
  if (warp == 0) {
    if (lane < ncls) offsets[lane] = off;
    if (lane == ncls - 1) offsets[ncls] = vin;
    if (lane < plan_table_word(M, n_ad) - (M + ncls + 1)) plan[M + ncls + 1 + lane] = 0;   // padding
  }

  // stable scatter
#pragma unroll
  for (int j = 0; j < kPlanPer; j++) {
    const int c = cls[j] & 31;
    const int sp = __shfl_sync(0xffffffffu, before, c) + rank[j];   // position inside the segment
    const int o = __shfl_sync(0xffffffffu, off, c), tb = __shfl_sync(0xffffffffu, tbase, c);
    if (cls[j] < 0) continue;
    const int t = warp * (32 * kPlanPer) + 32 * j + lane;
    perm[o + sp] = t;
    table[(size_t)(tb + sp / kPlanTile) * kPlanRec + 4 + sp % kPlanTile] = t;
  }
  // table records: quad q of record i is item 17 i + q
  const int items = ntiles * kPlanQuads;
  for (int base = 32 * warp; base < items; base += 32 * nw) {
    const int it = base + lane, i = it / kPlanQuads, q = it - kPlanQuads * i;
    int c = 0;                                        // largest class whose first record is <= i
#pragma unroll
    for (int step = 16; step; step >>= 1)
      if (__shfl_sync(0xffffffffu, tbase, c + step) <= i) c += step;
    const int tb = __shfl_sync(0xffffffffu, tbase, c), o = __shfl_sync(0xffffffffu, off, c);
    const int cnt = __shfl_sync(0xffffffffu, total, c);
    if (it >= items) continue;
    int a = -1, rows = 0, first = 0;
    if (i < used) {
      a = c;
      rows = min(kPlanTile, cnt - kPlanTile * (i - tb));
      first = o + kPlanTile * (i - tb);
    }
    int32_t *rec = table + (size_t)i * kPlanRec;
    if (q == 0) {
      *reinterpret_cast<int4 *>(rec) = make_int4(a, rows, first, 0);
    } else {
      const int s0 = 4 * (q - 1);
      if (s0 >= rows)
        *reinterpret_cast<int4 *>(rec + 4 + s0) = make_int4(-1, -1, -1, -1);
      else
        for (int sl = rows; sl < s0 + 4; sl++) rec[4 + sl] = -1;
    }
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
  if (n_adapters <= 31 && M <= bi::kPlanChunk) {
    cudaLaunchConfig_t cfg = {};
    const unsigned ncta = (unsigned)std::max(1, (M + 511) / 512);
    cfg.gridDim = dim3(ncta, 1, 1);
    cfg.blockDim = dim3(32 * bi::kPlanSmallWarps, 1, 1);
    cfg.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = ncta;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int32_t *out = static_cast<int32_t *>(plan);
    if (cudaLaunchKernelEx(&cfg, bi::plan_small_kernel, ids, M, n_adapters, out) != cudaSuccess) return BI_ERR_CUDA;
  } else
    bi::plan_kernel<<<1, bi::kPlanThreads, smem, reinterpret_cast<cudaStream_t>(stream)>>>(
        ids, M, n_adapters, static_cast<int32_t *>(plan));
  return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}
