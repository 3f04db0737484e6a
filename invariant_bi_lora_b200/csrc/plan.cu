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
// One cluster of up to 8 CTAs, so that the work of up to 128 warps runs on
// up to 8 SMs and their counts meet in distributed shared memory.  Tokens
// go in chunks of 128: warp w owns the contiguous chunks w * cpw ..
// (w + 1) * cpw - 1, lane l the four tokens 128 k + 32 j + l of chunk k
// (j = 0..3), so every load is a coalesced 128-byte line and the warp sees
// its tokens in index order.
//  * Rank: a class fits in nb bits, so one ballot per bit of the j-th
//    tokens gives every lane the lanes whose token shares its class (the
//    AND of the bit masks, complemented where its bit is 0); its rank in
//    the warp is the warp's running count of that class plus its
//    same-class lanes below it.  With at most 32 classes (narrow) lane c
//    keeps the running count of class c in a register, read by shuffle
//    (and, from the same ballots, the lanes holding class c); with more,
//    the counts sit in a per-warp shared-memory row that the first lane of
//    each class group advances.
//  * Bases: pass 1 counts; every warp pushes its row of class counts into
//    every CTA's [warp][class] table by st.async, counted on that CTA's
//    mbarrier, and once its own table is complete each warp scans it itself (its class bases in the warps before
//    it, the class totals; a shuffle scan over the classes gives the
//    segment starts and the table bases).  Pass 2 ranks again from those
//    bases and scatters (one chunk per warp, the common case, keeps pass 1's
//    ranks and skips the second look at the ids).
//  * Table: records are written as 17 16-byte quads (header, 16 quads of
//    token slots), spread over all threads; a slot quad is written only
//    where it holds unused (-1) slots, the scatter fills the rest.
#include "common.cuh"
#include "tc.cuh"

#include <algorithm>

namespace bi {

constexpr int kPlanPer = 4;                         // tokens per lane per chunk
constexpr int kPlanChunkTok = 32 * kPlanPer;        // 128 tokens per warp chunk
constexpr int kPlanMaxCtas = 8;                     // one portable cluster
constexpr int kPlanQuads = kPlanRec / 4;            // 17

BI_DEV int plan_class(int a, int n_ad) { return (a >= 0 && a < n_ad) ? a : n_ad; }

// Classes of the lane's four tokens of chunk k, -1 past the end.
BI_DEV void plan_load(const int32_t *__restrict__ ids, int M, int n_ad, long k, int lane, int (&cls)[kPlanPer]) {
  int v[kPlanPer];
#pragma unroll
  for (int j = 0; j < kPlanPer; j++) {
    const long t = k * kPlanChunkTok + 32 * j + lane;
    v[j] = t < M ? ids[t] : 0;
  }
#pragma unroll
  for (int j = 0; j < kPlanPer; j++) {
    const long t = k * kPlanChunkTok + 32 * j + lane;
    cls[j] = t < M ? plan_class(v[j], n_ad) : -1;
  }
}

// Lanes whose token has this lane's class (`same`) and, narrow, lanes whose
// token has class == lane (`mine`; meaningful for lanes < 2^nb).
template <bool WIDE>
BI_DEV void plan_masks(int cls, int nb, int lane, unsigned &same, unsigned &mine) {
  same = __ballot_sync(0xffffffffu, cls >= 0);
  mine = same;
#pragma unroll
  for (int bit = 0; bit < (WIDE ? 9 : 5); bit++) {
    if (bit < nb) {
      const unsigned m = __ballot_sync(0xffffffffu, (cls >> bit) & 1);
      same &= ((cls >> bit) & 1) ? m : ~m;
      if (!WIDE) mine &= ((lane >> bit) & 1) ? m : ~m;
    }
  }
}

// WIDE: the warp's running count of class `cls` (row `cnt`), advanced by the
// group's first lane; returns the count before this group.
BI_DEV int plan_bump(int *cnt, int cls, unsigned same, unsigned lt_mask) {
  const int base = cls >= 0 ? cnt[cls] : 0;
  __syncwarp();
  if (cls >= 0 && (same & lt_mask) == 0) cnt[cls] = base + __popc(same);
  __syncwarp();
  return base;
}

// Dynamic shared memory (ints): tbl[nw][ncp] (ncp = 32 narrow, ncls wide);
// wide adds cnt[W][ncls], s_off[ncls + 1], s_tb[ncls + 1].
template <bool WIDE>
__global__ void __launch_bounds__(512)
plan_kernel(const int32_t *__restrict__ ids, int M, int n_ad, int cpw, int32_t *__restrict__ plan, unsigned *status) {
  extern __shared__ int plan_smem[];
  const int ncls = n_ad + 1, ncta = gridDim.x, W = blockDim.x >> 5;   // the grid is one cluster
  const int lane = threadIdx.x & 31, lw = threadIdx.x >> 5;
  const int warp = blockIdx.x * W + lw, nw = ncta * W;
  const unsigned lt_mask = (1u << lane) - 1u;
  const int ncp = WIDE ? ncls : 32;
  int *tbl = plan_smem;                               // warp w's count of class c
  int *cnt = tbl + nw * ncp + lw * ncls;              // WIDE: this warp's running counts
  int *s_off = tbl + nw * ncp + W * ncls;             // WIDE: segment starts (+ M)
  int *s_tb = s_off + ncls + 1;                       // WIDE: first records (+ used)
  int32_t *perm = plan;
  int32_t *offsets = plan + M;
  int32_t *table = plan + plan_table_word(M, n_ad);
  const int ntiles = (int)plan_tiles(M, n_ad);
  // every CTA has started (and initialised its table barrier) once this
  // arrive is matched; the wait comes before the first push into a peer
  __shared__ __align__(8) uint64_t s_tbar;
  if (threadIdx.x == 0) {
    mbar_init(&s_tbar, 1);
    mbar_fence_init();
    mbar_arrive_expect_tx(&s_tbar, 4u * (uint32_t)nw * (uint32_t)ncp);
  }
  cluster_arrive_relaxed();
  // start the output's address translation while the ids are in flight
  if (warp == 0 && lane == 0) asm volatile("prefetch.global.L2 [%0];" ::"l"(plan));
  if (warp == nw - 1 && lane == 0)
    asm volatile("prefetch.global.L2 [%0];" ::"l"(table + (size_t)ntiles * kPlanRec - 1));

  const int nb = 32 - __clz(ncls - 1);                // bits of the largest class
  const long k0 = (long)warp * cpw;                   // this warp's first chunk
  int cls0[kPlanPer], rank0[kPlanPer], nxt[kPlanPer];
  plan_load(ids, M, n_ad, k0, lane, cls0);
  if (WIDE) {
    for (int c = lane; c < ncls; c += 32) cnt[c] = 0;
    __syncwarp();
  }

  // ---- pass 1: the warp's count of every class (narrow: lane c's `run`)
  int run = 0, run0 = 0;
  for (int k = 0; k < cpw; k++) {
    int cls[kPlanPer];
#pragma unroll
    for (int j = 0; j < kPlanPer; j++) cls[j] = k == 0 ? cls0[j] : nxt[j];
    if (k + 1 < cpw) plan_load(ids, M, n_ad, k0 + k + 1, lane, nxt);
#pragma unroll
    for (int j = 0; j < kPlanPer; j++) {
      unsigned same, mine;
      plan_masks<WIDE>(cls[j], nb, lane, same, mine);
      int r;
      if (WIDE) {
        r = plan_bump(cnt, cls[j], same, lt_mask);
      } else {
        r = __shfl_sync(0xffffffffu, run, cls[j] & 31);
        run += __popc(mine);
      }
      if (k == 0) rank0[j] = r + __popc(same & lt_mask);
    }
    if (k == 0) run0 = run;
  }

  // ---- counts into every CTA's table (nw * ncp words land in each)
  cluster_wait();
  if (WIDE) {
    for (int c = lane; c < ncls; c += 32) {
      const int v = cnt[c];
      for (int r = 0; r < ncta; r++) st_async_u32(&tbl[warp * ncp + c], &s_tbar, (uint32_t)r, (uint32_t)v);
    }
  } else {
    const int v = lane < ncls ? run : 0;
    for (int r = 0; r < ncta; r++) st_async_u32(&tbl[warp * ncp + lane], &s_tbar, (uint32_t)r, (uint32_t)v);
  }
  if (!mbar_wait_cluster(&s_tbar, 0)) flag_error(status, BI_ERR_TIMEOUT);

  // ---- bases: this warp's start inside each class, segment starts, table bases
  int before = 0, total = 0, off = 0, tbase = 0, used = 0;   // narrow: lane c's class
  if (WIDE) {
    int carry_v = 0, carry_t = 0;
    for (int kc = 0; 32 * kc < ncls; kc++) {
      const int c = 32 * kc + lane;
      int b = 0, t = 0;
      if (c < ncls) {
#pragma unroll 8
        for (int w = 0; w < nw; w++) {
          const int n = tbl[w * ncp + c];
          b += w < warp ? n : 0;
          t += n;
        }
      }
      const int tv = (t + kPlanTile - 1) / kPlanTile;
      int vin = t, tin = tv;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, vin, o), y = __shfl_up_sync(0xffffffffu, tin, o);
        if (lane >= o) vin += x, tin += y;
      }
      if (c < ncls) {
        cnt[c] = b;
        if (lw == 0) s_off[c] = carry_v + vin - t, s_tb[c] = carry_t + tin - tv;
        if (warp == 0) offsets[c] = carry_v + vin - t;
      }
      carry_v += __shfl_sync(0xffffffffu, vin, 31);
      carry_t += __shfl_sync(0xffffffffu, tin, 31);
    }
    if (lane == 0 && lw == 0) s_off[ncls] = carry_v, s_tb[ncls] = carry_t;
    if (lane == 0 && warp == 0) offsets[ncls] = carry_v;
    used = carry_t;
    __syncwarp();
    __syncthreads();                                  // s_off / s_tb from warp 0 of this CTA
  } else {
#pragma unroll 8
    for (int w = 0; w < nw; w++) {
      const int n = tbl[w * ncp + lane];
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
    // lanes >= ncls hold the totals, so the table bases stay non-decreasing
    off = vin - total, tbase = tin - tv;
    used = __shfl_sync(0xffffffffu, tin, 31);
    if (warp == 0) {
      if (lane < ncls) offsets[lane] = off;
      if (lane == ncls - 1) offsets[ncls] = vin;
    }
  }
  if (warp == 0 && lane < plan_table_word(M, n_ad) - (M + ncls + 1)) plan[M + ncls + 1 + lane] = 0;   // padding

  // ---- pass 2: stable scatter
  auto put = [&](int c, int sp, int o, int tb, long t) {
    perm[o + sp] = (int32_t)t;
    table[(size_t)(tb + sp / kPlanTile) * kPlanRec + 4 + sp % kPlanTile] = (int32_t)t;
  };
  int pos = before + run0;                            // narrow, lane c: next position after chunk 0
  for (int k = 0; k < cpw; k++) {
    int cls[kPlanPer];
#pragma unroll
    for (int j = 0; j < kPlanPer; j++) cls[j] = k == 0 ? cls0[j] : nxt[j];
    if (k + 1 < cpw) plan_load(ids, M, n_ad, k0 + k + 1, lane, nxt);
#pragma unroll
    for (int j = 0; j < kPlanPer; j++) {
      const long t = (k0 + k) * kPlanChunkTok + 32 * j + lane;
      if (WIDE) {
        unsigned same, mine;
        plan_masks<true>(cls[j], nb, lane, same, mine);
        const int sp = plan_bump(cnt, cls[j], same, lt_mask) + __popc(same & lt_mask);
        if (cls[j] >= 0) put(cls[j], sp, s_off[cls[j]], s_tb[cls[j]], t);
      } else {
        const int c = cls[j] & 31;
        int sp;
        if (k == 0) {
          sp = __shfl_sync(0xffffffffu, before, c) + rank0[j];
        } else {
          unsigned same, mine;
          plan_masks<false>(cls[j], nb, lane, same, mine);
          sp = __shfl_sync(0xffffffffu, pos, c) + __popc(same & lt_mask);
          pos += __popc(mine);
        }
        const int o = __shfl_sync(0xffffffffu, off, c), tb = __shfl_sync(0xffffffffu, tbase, c);
        if (cls[j] >= 0) put(c, sp, o, tb, t);
      }
    }
  }

  // ---- table records: quad q of record i is item 17 i + q
  const int items = ntiles * kPlanQuads;
  for (int base = 32 * warp; base < items; base += 32 * nw) {
    const int it = base + lane, i = it / kPlanQuads, q = it - kPlanQuads * i;
    int c = 0, tb, o, n;                              // c: largest class whose first record is <= i
    if (WIDE) {
      for (int step = 256; step; step >>= 1)
        if (c + step < ncls && s_tb[c + step] <= i) c += step;
      tb = s_tb[c], o = s_off[c], n = s_off[c + 1] - s_off[c];
    } else {
#pragma unroll
      for (int step = 16; step; step >>= 1)
        if (__shfl_sync(0xffffffffu, tbase, c + step) <= i) c += step;
      tb = __shfl_sync(0xffffffffu, tbase, c), o = __shfl_sync(0xffffffffu, off, c);
      n = __shfl_sync(0xffffffffu, total, c);
    }
    if (it >= items) continue;
    int a = -1, rows = 0, first = 0;
    if (i < used) {
      a = c;
      rows = min(kPlanTile, n - kPlanTile * (i - tb));
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
  const bool wide = n_adapters > 31;
  const int ncls = n_adapters + 1;
  const long chunks = ((long)M + bi::kPlanChunkTok - 1) / bi::kPlanChunkTok;
  const int ncta = (int)std::min<long>(bi::kPlanMaxCtas, std::max<long>(1, (M + 511) / 512));
  const int W = (wide || M <= 4096) ? 4 : 16;       // warps per CTA
  const int nw = ncta * W;
  const int cpw = (int)std::max<long>(1, (chunks + nw - 1) / nw);
  const size_t smem = sizeof(int) * (wide ? (size_t)nw * ncls + (size_t)W * ncls + 2 * (size_t)(ncls + 1)
                                          : (size_t)nw * 32);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)ncta, 1, 1);
  cfg.blockDim = dim3(32 * W, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)ncta;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int32_t *out = static_cast<int32_t *>(plan);
  unsigned *status = bi::status_word();
  const cudaError_t e = wide ? cudaLaunchKernelEx(&cfg, bi::plan_kernel<true>, ids, M, n_adapters, cpw, out, status)
                             : cudaLaunchKernelEx(&cfg, bi::plan_kernel<false>, ids, M, n_adapters, cpw, out, status);
  if (e != cudaSuccess) return BI_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}
