// shrink.cu -- LoRA shrink y = x . A with a fixed-order split-K reduction.
//
// "Reproducible LoRA Inference Through Deterministic Split-K Reduction"
// (Highlights, Q&A): the split-K shrink of vLLM adds its K-partials with fp32
// atomics, so identical inputs give different bits; a deterministic split-K
// keeps the parallelism and combines the partials in a fixed order.
// "Deterministic Inference across Tensor Parallel Sizes ..." (Abstract): one
// hierarchical binary tree orders every level of the reduction.
//
// Reduction order (the same for every M, split count, tile shape, replay):
//   leaf   = 64 consecutive k; its value is one chain of four m16n8k16
//            tensor-core MMAs started from zero (the order inside an MMA is
//            the hardware's, identical for every row and every call);
//   leaves = combined by the canonical halving tree in fp32 (__fadd_rn).
// A CTA owns a contiguous power-of-two block of leaves (one subtree).  Its
// warps split that block into G contiguous groups (subtrees again); a warp
// folds its group's leaves in post order in registers, the G group values
// meet in shared memory (perfect tree), and in mode TREE the `splits` CTAs
// of a row tile -- one thread-block cluster -- meet through distributed
// shared memory (a reduce-scatter of st.async pushes, each rank waiting on
// its own barrier for the shares it adds), perfect
// tree again.  Every level is a level
// of the one canonical tree over the K/64 leaves, so the bits cannot depend
// on how the work was cut.
//
// Data path: both operands are K-contiguous (x [M][K], A [r][K]), so a
// thread fetches the eight consecutive k of its fragment row with one
// 128-bit load, for x and for A alike.  Inside a 32-wide k chunk, thread
// (g, c) feeds k = 8c..8c+7 to MMA k-slots {2c, 2c+1, 2c+8, 2c+9} of two
// MMAs; the same permutation is applied to both operands, so the products
// summed are exactly x[m][k] * A[j][k].  A CTA learns its tile (adapter and
// token rows) from one read of the plan's tile table.  Two kernels, same
// leaves and same tree, chosen by the grid size:
//   ring: x goes straight to registers through a ring of PF leaves per
//         warp, so every warp keeps PF leaves of loads in flight while it
//         multiplies; the CTA's slice of A is staged once in shared memory
//         when it fits in 64 KB.  Used when the grid needs more than one wave.
//   bulk: the CTA's whole x and A slices are requested at once by the copy
//         engine (one contiguous copy per row) into shared memory.  Used
//         when every CTA of the grid is resident at once.
// Each warp issues the MMAs of several leaves step by step across all of
// their chains, so no MMA waits right behind the one it depends on.
#include "tc.cuh"

#include <cooperative_groups.h>
#include <algorithm>
#include <vector>

namespace cg = cooperative_groups;

namespace bi {

constexpr int kLeaf = 64;          // k per leaf
constexpr int kMaxGroupLeaves = 1024;
constexpr int kMaxSplits = 16;
constexpr int kMaxBM = 64;         // rows per CTA tile (4 MMA row tiles)

struct ShrinkParams {
  const uint16_t *x;        // [M][K] bf16
  const uint16_t *at;       // [n_ad][r][K] bf16
  const int32_t *perm;      // token order grouped by adapter (nullptr: identity)
  const int32_t *offsets;   // [n_ad + 2] segment starts in perm (nullptr: one segment)
  float *y;                 // [M][r] fp32
  unsigned *status;
  int M, K, r, n_ad;
  int splits;               // CTAs per row tile (cluster width in mode TREE)
  int lc;                   // leaves per CTA = K / 64 / splits
  int groups;               // G: leaf groups per CTA (power of two, divides lc)
  int lg;                   // leaves per group = lc / G
  int mtiles;               // MT: 16-row MMA tiles per CTA
  int ngroups;              // NG: rank groups of NGW columns
  int mode;
  int a_staged;             // 1: the CTA's A slice sits in shared memory
  int a_offset;             // bytes from the start of dynamic shared memory to the A slice
  int g_offset;             // bytes to the exchange slots (mode TREE)
  int gather0;              // mode TREE: 1 = all partials to rank 0, 0 = reduce-scatter over the ranks
  // bulk-copy kernel only
  const int32_t *table;     // plan tile table (nullptr: rows in index order, adapter 0)
  int sub;                  // CTA tiles per 64-row table record (64 / bm)
  int rowbytes;             // bytes of one row's K range in one split (lc * 128)
  int x_off, part_off;      // shared-memory offsets of the x rows and the group values
  // fused expand (register-ring kernel only)
  int fuse;                 // 1: after y, out (+)= bf16(y) . B^T for the tile
  const uint16_t *bt;       // [n_ad][N][r] bf16
  float *out;               // [M][N] fp32
  int N, accumulate;
  int yfull_rel, stage_rel; // bytes from `part` to the full y tile, and from it to the strip buffers
  uint8_t merges[kMaxGroupLeaves];   // post-order merges after each leaf
};

// A leaf's operand fragments: x rows g and g+8 and the NT A columns, for the
// two 32-wide k chunks of the leaf.
template <int NT>
struct LeafFrag {
  uint4 xa[2][2];     // [chunk][row g / row g+8]
  uint4 ab[2][NT];    // [chunk][n-tile]
};

// NL leaves at once: each leaf's value is, per n-tile, one chain of four
// MMAs from zero -- k chunk 0 step 0, chunk 0 step 1, chunk 1 step 0,
// chunk 1 step 1, always in that order.  The chains of different n-tiles
// and leaves are independent, so they are issued step by step across all
// of them: a chain's next MMA never waits right behind its previous one.
template <int NT, int NL>
BI_DEV void mma_leaves(float (&acc)[NL][NT][4], const LeafFrag<NT> (&f)[NL]) {
#pragma unroll
  for (int l = 0; l < NL; l++)
#pragma unroll
    for (int t = 0; t < NT; t++)
#pragma unroll
      for (int q = 0; q < 4; q++) acc[l][t][q] = 0.0f;
#pragma unroll
  for (int h = 0; h < 2; h++)
#pragma unroll
    for (int s = 0; s < 2; s++)
#pragma unroll
      for (int l = 0; l < NL; l++) {
        const uint4 r0 = f[l].xa[h][0], r1 = f[l].xa[h][1];
        const uint32_t a[4] = {s ? r0.z : r0.x, s ? r1.z : r1.x, s ? r0.w : r0.y, s ? r1.w : r1.y};
#pragma unroll
        for (int t = 0; t < NT; t++) {
          const uint4 b = f[l].ab[h][t];
          const uint32_t bb[2] = {s ? b.z : b.x, s ? b.w : b.y};
          mma_bf16_16816(acc[l][t], a, bb, acc[l][t]);
        }
      }
}

// One leaf: four MMAs per n-tile (two k chunks x two k16 steps), from zero.
template <int NT>
BI_DEV void mma_leaf(float acc[NT][4], const LeafFrag<NT> &f) {
  float a1[1][NT][4];
  const LeafFrag<NT> f1[1] = {f};
  mma_leaves<NT, 1>(a1, f1);
#pragma unroll
  for (int t = 0; t < NT; t++)
#pragma unroll
    for (int q = 0; q < 4; q++) acc[t][q] = a1[0][t][q];
}

// Binary-counter fold of leaf i (an index known at compile time) into the
// pending subtree values lv: leaf i closes the levels where its index has a
// 1 bit (left = the parked subtree, right = the one just finished) and parks
// the result at its lowest 0 bit.  After the last leaf of a power-of-two
// group, acc holds the group's subtree value.
template <int NT, int LOG2>
BI_DEV void fold_leaf(int i, float (&lv)[LOG2 > 0 ? LOG2 : 1][NT][4], float (&acc)[NT][4]) {
#pragma unroll
  for (int L = 0; L < LOG2; L++) {
    if ((i >> L) & 1) {
#pragma unroll
      for (int t = 0; t < NT; t++)
#pragma unroll
        for (int q = 0; q < 4; q++) acc[t][q] = __fadd_rn(lv[L][t][q], acc[t][q]);
    } else {
#pragma unroll
      for (int t = 0; t < NT; t++)
#pragma unroll
        for (int q = 0; q < 4; q++) lv[L][t][q] = acc[t][q];
      break;
    }
  }
}

// Warp 0 of a CTA: its row tile's adapter (-1: no tile, n_ad: tokens
// without an adapter), rows, and the token index of each row, into shared
// memory.  With a plan, one read of the tile's table record (the CTA tile
// is part q of record tile / sub); without one, rows in index order.
BI_DEV void tile_record(const ShrinkParams &p, int bm, int tile, int lane, int32_t *s_rows, int *s_info) {
  int adapter = -1, rows = 0;
  if (p.table) {
    const int rec = tile / p.sub, q = tile - rec * p.sub;
    const int32_t *R = p.table + (size_t)rec * kPlanRec;
    const int4 h = *reinterpret_cast<const int4 *>(R);
    int4 id4 = make_int4(0, 0, 0, 0);
    if (lane < kPlanTile / 4) id4 = *reinterpret_cast<const int4 *>(R + 4 + 4 * lane);
    rows = min(bm, h.y - q * bm);
    adapter = rows > 0 ? h.x : -1;
    const int idv[4] = {id4.x, id4.y, id4.z, id4.w};
#pragma unroll
    for (int e = 0; e < 4; e++) {
      const int s = 4 * lane + e - q * bm;
      if (lane < kPlanTile / 4 && s >= 0 && s < rows) s_rows[s] = idv[e];
    }
  } else {
    const int row0 = tile * bm;
    rows = min(bm, p.M - row0);
    adapter = rows > 0 ? 0 : -1;
    for (int i = lane; i < rows; i += 32) s_rows[i] = row0 + i;
  }
  if (lane == 0) {
    s_info[0] = adapter;
    s_info[1] = rows > 0 ? rows : 0;
  }
}

// Fused expand ("Reproducible LoRA Inference ...", Q&A: LoRA is a shrink
// followed by an expand; here y stays on chip).  yfull [bm][r] holds the
// tile's final y rows in this CTA's shared memory.  Rank q of the S CTAs of
// the tile computes the 64-column strips j = q, q + S, ... of
// out[row][n] (+)= sum_j bf16(y[row][j]) * B[adapter][n][j]: per 16-row
// m-tile and 8-column n-tile one chain of KS = ceil(r/16) MMAs from zero,
// the same fragments and order as the expand kernel, so the bits equal a
// separate shrink then expand.  Each warp stages its 16 x 64 strip in
// shared memory (stride 68 floats) and writes whole 256-byte row segments.
template <int KS>
BI_DEV void fused_expand_ks(const ShrinkParams &p, const float *yfull, const int32_t *s_rows, int rows, int adapter,
                            int q, int S) {
  float *stage = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(const_cast<float *>(yfull)) + p.stage_rel);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  const int g = lane >> 2, c = lane & 3;
  const int half = lane >> 4, q4 = (lane & 15) * 4;
  float(*so)[68] = reinterpret_cast<float(*)[68]>(stage + (size_t)warp * 16 * 68);
  const int mts = (rows + 15) >> 4;
  const int strips = (p.N + 63) >> 6;
  const int my_strips = strips > q ? (strips - q + S - 1) / S : 0;
  const uint16_t *bad = p.bt + (size_t)adapter * p.N * p.r;
  for (int combo = warp; combo < mts * my_strips; combo += nwarps) {
    const int mt = combo % mts, sj = q + S * (combo / mts);
    const int lr0 = mt * 16 + g, lr1 = lr0 + 8;
    uint32_t afr[KS][4];
#pragma unroll
    for (int st = 0; st < KS; st++) {
      const int k0 = 16 * st + 2 * c, k1 = k0 + 8;
      float2 a00 = make_float2(0.f, 0.f), a10 = a00, a01 = a00, a11 = a00;
      if (k0 < p.r) {
        a00 = *reinterpret_cast<const float2 *>(yfull + lr0 * p.r + k0);
        a10 = *reinterpret_cast<const float2 *>(yfull + lr1 * p.r + k0);
      }
      if (k1 < p.r) {
        a01 = *reinterpret_cast<const float2 *>(yfull + lr0 * p.r + k1);
        a11 = *reinterpret_cast<const float2 *>(yfull + lr1 * p.r + k1);
      }
      afr[st][0] = pack_bf16x2(a00.x, a00.y);
      afr[st][1] = pack_bf16x2(a10.x, a10.y);
      afr[st][2] = pack_bf16x2(a01.x, a01.y);
      afr[st][3] = pack_bf16x2(a11.x, a11.y);
    }
    const int nbase = sj * 64;
#pragma unroll
    for (int i = 0; i < 8; i++) {
      const int n0 = nbase + i * 8;
      const uint16_t *brow = bad + (size_t)(n0 + g) * p.r;
      const bool ok = n0 < p.N;
      uint32_t bfr[KS][2];
#pragma unroll
      for (int st = 0; st < KS; st++) {
        const int k0 = 16 * st + 2 * c, k1 = k0 + 8;
        bfr[st][0] = ok && k0 < p.r ? __ldg(reinterpret_cast<const unsigned int *>(brow + k0)) : 0u;
        bfr[st][1] = ok && k1 < p.r ? __ldg(reinterpret_cast<const unsigned int *>(brow + k1)) : 0u;
      }
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int st = 0; st < KS; st++) mma_bf16_16816(acc, afr[st], bfr[st], acc);
      *reinterpret_cast<float2 *>(&so[g][i * 8 + 2 * c]) = make_float2(acc[0], acc[1]);
      *reinterpret_cast<float2 *>(&so[g + 8][i * 8 + 2 * c]) = make_float2(acc[2], acc[3]);
    }
    __syncwarp();
    const int n = nbase + q4;
#pragma unroll 2
    for (int j = 0; j < 8; j++) {
      const int lr = 2 * j + half, tr = mt * 16 + lr;
      if (tr < rows && n < p.N) {
        float4 v = *reinterpret_cast<const float4 *>(&so[lr][q4]);
        float4 *o = reinterpret_cast<float4 *>(p.out + (size_t)s_rows[tr] * p.N + n);
        if (p.accumulate) {
          const float4 old = *o;
          v.x = __fadd_rn(old.x, v.x);
          v.y = __fadd_rn(old.y, v.y);
          v.z = __fadd_rn(old.z, v.z);
          v.w = __fadd_rn(old.w, v.w);
        }
        __stcs(o, v);
      }
    }
    __syncwarp();
  }
}

BI_DEV void fused_expand(const ShrinkParams &p, const float *yfull, const int32_t *s_rows, int rows, int adapter, int q,
                         int S) {
  switch ((p.r + 15) >> 4) {
    case 1: fused_expand_ks<1>(p, yfull, s_rows, rows, adapter, q, S); break;
    case 2: fused_expand_ks<2>(p, yfull, s_rows, rows, adapter, q, S); break;
    case 3: fused_expand_ks<3>(p, yfull, s_rows, rows, adapter, q, S); break;
    case 4: fused_expand_ks<4>(p, yfull, s_rows, rows, adapter, q, S); break;
    case 5: fused_expand_ks<5>(p, yfull, s_rows, rows, adapter, q, S); break;
    case 6: fused_expand_ks<6>(p, yfull, s_rows, rows, adapter, q, S); break;
    case 7: fused_expand_ks<7>(p, yfull, s_rows, rows, adapter, q, S); break;
    default: fused_expand_ks<8>(p, yfull, s_rows, rows, adapter, q, S); break;
  }
}

// Mode TREE: the exchange barrier of this CTA counts the bytes its peers
// push into its slots (st.async), so a rank waits for exactly the shares it
// adds and never for its peers' threads.  Initialised, with its expected
// bytes, by one thread before the cluster arrive that every CTA makes on
// entry (the fence makes the initialisation visible to the cluster).
BI_DEV void exchange_init(const ShrinkParams &p, int bm, int split, uint64_t *xbar) {
  const uint32_t E = (uint32_t)bm * p.r;
  const uint32_t S = p.splits;
  const uint32_t bytes = p.gather0 ? (split == 0 ? (S - 1) * E * 4 : 0u) : (S - 1) * (E / S) * 4;
  mbar_init(xbar, 1);
  mbar_fence_init();
  mbar_arrive_expect_tx(xbar, bytes);
}

// The G group values of a row tile (part [G][bm][r], in shared memory,
// written and visible to the CTA) -> the tile's y rows: the perfect tree over
// the groups, then the cross-split combine of the mode.  Every thread of the
// CTA calls it.  In mode TREE with splits > 1 each CTA has made a relaxed
// cluster arrive on entry; the matching wait comes before the first write
// into a peer's shared memory.  slots: the exchange slots (mode TREE).
// With p.fuse, the final y values also go to yfull in every CTA of the tile
// (all-gather through distributed shared memory), and the tile's expand
// follows; y itself is written only when p.y is set.
BI_DEV void finish_tile(const ShrinkParams &p, float *part, float *slots, uint64_t *xbar, const int32_t *s_rows,
                        int rows, int bm, int split, int adapter) {
  const int E = bm * p.r;
  const int r_sh = (p.r & (p.r - 1)) == 0 ? __ffs(p.r) - 1 : -1;
  auto e_row = [&](int e) { return r_sh >= 0 ? e >> r_sh : e / p.r; };
  auto e_col = [&](int e) { return r_sh >= 0 ? e & (p.r - 1) : e % p.r; };
  // perfect tree over the G groups, in place into group 0
  for (int s = 1; s < p.groups; s <<= 1) {
    for (int e = threadIdx.x; e < E; e += blockDim.x)
      for (int q = 0; q + s < p.groups; q += 2 * s)
        part[(size_t)q * E + e] = __fadd_rn(part[(size_t)q * E + e], part[(size_t)(q + s) * E + e]);
    __syncthreads();
  }

  auto out_index = [&](int e) -> size_t { return (size_t)s_rows[e_row(e)] * p.r + e_col(e); };
  const int valid_E = rows * p.r;
  float *yfull = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(part) + p.yfull_rel);

  if (p.mode == BI_SHRINK_ATOMIC) {
    for (int e = threadIdx.x; e < valid_E; e += blockDim.x) atomicAdd(p.y + out_index(e), part[e]);
    return;
  }
  if (p.splits == 1) {
    for (int e = threadIdx.x; e < valid_E; e += blockDim.x) {
      if (p.y) p.y[out_index(e)] = part[e];
      if (p.fuse) yfull[e] = part[e];
    }
    if (p.fuse) {
      __syncthreads();
      fused_expand(p, yfull, s_rows, rows, adapter, 0, 1);
    }
    return;
  }

  // ---- mode TREE: the splits CTAs of this tile form one cluster; rank q
  // holds the subtree of leaves [q*lc, (q+1)*lc).  The tile's E elements
  // are cut into S shares; rank q finishes share q.  Every rank stores share
  // t of its partial into rank t's slot [q] by st.async (a reduce-scatter by
  // pushes), counted on rank t's exchange barrier; once its own barrier has
  // seen all S-1 shares land, each rank adds the S values of its share by
  // the perfect tree over the ranks, from its own shared memory, and writes
  // y.  Nothing reads a peer's memory, and every SM receives only (S-1)/S of
  // one partial.  A rank cannot finish before every share pushed to it has
  // landed, so no rank waits for its peers before it exits.
  cg::cluster_group cluster = cg::this_cluster();
  const int S = p.splits;
  // the relaxed arrive each CTA made on entry: once this wait returns,
  // every CTA of the cluster is running, so its shared memory may be written
  cluster_wait();
  // a final y value: to global memory and, fused, to every rank's yfull
  auto emit = [&](int e, float v) {
    if (p.y) p.y[out_index(e)] = v;
    if (p.fuse)
      for (int t = 0; t < S; t++) cluster.map_shared_rank(yfull, t)[e] = v;
  };
  if (p.gather0) {
    // small tiles: ranks 1..S-1 push their whole partial into rank 0's
    // slots [S-1][E]; after the barrier rank 0 alone adds and writes y
    float *gslots = slots;
    if (split != 0) {
      const float4 *src = reinterpret_cast<const float4 *>(part);
      for (int e4 = threadIdx.x; e4 < E / 4; e4 += blockDim.x)
        st_async_v4(gslots + (size_t)(split - 1) * E + 4 * e4, xbar, 0u, src[e4]);
    }
    if (split == 0) {
      if (!mbar_wait_cluster(xbar, 0)) flag_error(p.status, BI_ERR_TIMEOUT);
      for (int e = threadIdx.x; e < valid_E; e += blockDim.x) {
        float v[kMaxSplits];
        v[0] = part[e];
#pragma unroll
        for (int q = 1; q < kMaxSplits; q++) v[q] = q < S ? gslots[(size_t)(q - 1) * E + e] : 0.0f;
#pragma unroll
        for (int st = 1; st < kMaxSplits; st <<= 1)
#pragma unroll
          for (int q = 0; q + st < kMaxSplits; q += 2 * st)
            if (q + st < S) v[q] = __fadd_rn(v[q], v[q + st]);
        emit(e, v[0]);
      }
    }
  } else {
    const int share = E / S;                         // E = 16 * mt * r, a multiple of 128
    for (int t = 0; t < S; t++) {
      if (t == split) continue;
      const float4 *src = reinterpret_cast<const float4 *>(part + (size_t)t * share);
      for (int i4 = threadIdx.x; i4 < share / 4; i4 += blockDim.x)
        st_async_v4(slots + (size_t)split * share + 4 * i4, xbar, (uint32_t)t, src[i4]);
    }
    if (!mbar_wait_cluster(xbar, 0)) flag_error(p.status, BI_ERR_TIMEOUT);
    for (int i = threadIdx.x; i < share; i += blockDim.x) {
      const int e = split * share + i;
      if (e >= valid_E) break;
      float v[kMaxSplits];
#pragma unroll
      for (int q = 0; q < kMaxSplits; q++)
        v[q] = q < S ? (q == split ? part[e] : slots[(size_t)q * share + i]) : 0.0f;
#pragma unroll
      for (int st = 1; st < kMaxSplits; st <<= 1)
#pragma unroll
        for (int q = 0; q + st < kMaxSplits; q += 2 * st)
          if (q + st < S) v[q] = __fadd_rn(v[q], v[q + st]);
      emit(e, v[0]);
    }
  }
  if (!p.fuse) return;
  // every rank's yfull is complete once all ranks have emitted their shares
  cluster_arrive_release();
  cluster_wait_acquire();
  fused_expand(p, yfull, s_rows, rows, adapter, split, S);
}

// PF: leaves of x in flight per thread, in a register ring.  LG: leaves per
// warp when that count is a power of two known at compile time (the walk is
// then a binary counter with fixed register slots and a fully unrolled
// loop); LG = 0 walks any count with the host's post-order schedule on a
// predicated register stack of MAXD slots.
template <int NGW, int MAXD, int PF, bool ASTAGED, int LG>
__global__ void __launch_bounds__(256)
shrink_kernel(const __grid_constant__ ShrinkParams p) {
  constexpr int NT = NGW / 8;
  extern __shared__ float4 smem_f4[];
  float *part = reinterpret_cast<float *>(smem_f4);     // [G][BM][r]
  __shared__ int32_t s_rows[kMaxBM];                    // token row of each tile row
  __shared__ int s_info[2];
  __shared__ __align__(8) uint64_t s_xbar;              // mode TREE exchange barrier

  const int bm = 16 * p.mtiles;
  const int split = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const bool clustered = p.mode == BI_SHRINK_TREE && p.splits > 1;

  if (warp == 0) tile_record(p, bm, blockIdx.y, lane, s_rows, s_info);
  if (clustered && threadIdx.x == 32 % blockDim.x) exchange_init(p, bm, split, &s_xbar);
  __syncthreads();
  struct { int adapter, rows; } ti = {s_info[0], s_info[1]};
  // mode TREE: say "started" to the cluster now; finish_tile waits for the
  // others before it writes into their shared memory.  The exits below are
  // uniform across the cluster (every split sees the same tile) and wait too.
  if (clustered) cluster_arrive_relaxed();
  if (ti.adapter < 0) {
    if (clustered) cluster_wait();
    return;
  }

  // e -> (local row, column) of the [bm][r] tile; r is a power of two in
  // every common configuration, so the split is a shift and a mask
  const int r_sh = (p.r & (p.r - 1)) == 0 ? __ffs(p.r) - 1 : -1;
  auto e_row = [&](int e) { return r_sh >= 0 ? e >> r_sh : e / p.r; };
  auto e_col = [&](int e) { return r_sh >= 0 ? e & (p.r - 1) : e % p.r; };

  if (ti.adapter == p.n_ad) {                       // tokens without an adapter
    if (p.mode != BI_SHRINK_ATOMIC && split == 0 && p.y)
      for (int e = threadIdx.x; e < ti.rows * p.r; e += blockDim.x)
        p.y[(size_t)s_rows[e_row(e)] * p.r + e_col(e)] = 0.0f;
    if (p.fuse && !p.accumulate) {
      // their expand rows are zero; the splits share the columns
      const int n4 = p.N >> 2;
      for (int i = threadIdx.x + split * blockDim.x; i < ti.rows * n4; i += blockDim.x * p.splits)
        __stcs(reinterpret_cast<float4 *>(p.out + (size_t)s_rows[i / n4] * p.N) + i % n4,
               make_float4(0.f, 0.f, 0.f, 0.f));
    }
    if (clustered) cluster_wait();
    return;
  }

  // ---- warp role: (leaf group, m-tile, rank group)
  const int per_lg = p.mtiles * p.ngroups;
  const int lgi = warp / per_lg;
  const int mt = (warp % per_lg) / p.ngroups;
  const int ng = warp % p.ngroups;

  // rows g and g+8 of this warp's m-tile
  const int lr0 = mt * 16 + g, lr1 = lr0 + 8;       // local rows in the tile
  const bool v0 = lr0 < ti.rows, v1 = lr1 < ti.rows;

  // token rows of this thread's fragment rows: their loads go out before
  // the A staging, since the x loads wait on them
  int row0 = 0, row1 = 0;
  if (v0) row0 = s_rows[lr0];
  if (v1) row1 = s_rows[lr1];

  // ---- shared memory holds the CTA's A slice (staged once, by every
  // thread with 16-byte cp.async, when it fits in 64 KB).  Rows are 128 bytes
  // per leaf; the 16-byte chunk index is XOR-ed with (row & 1) << 2 so that
  // the two rows a quarter-warp reads fall on disjoint bank halves.
  constexpr bool a_staged = ASTAGED;
  uint8_t *sa = reinterpret_cast<uint8_t *>(smem_f4) + p.a_offset;      // [r][lc * 128]
  const int a_stride = p.lc * 128;
  if (a_staged) {
    // A rows [adapter][j][split*lc*64 ...) -> sa[j][...], all threads
    const int w = p.lc * 8;                          // 16-byte chunks per row
    const int w_sh = (w & (w - 1)) == 0 ? __ffs(w) - 1 : -1;
    const int pieces = p.r * w;
    const uint16_t *a0 = p.at + (size_t)ti.adapter * p.r * p.K + (size_t)split * p.lc * kLeaf;
    for (int pc = threadIdx.x; pc < pieces; pc += blockDim.x) {
      const int j = w_sh >= 0 ? pc >> w_sh : pc / w;  // row
      const int ch = pc - j * w;                       // 16-byte chunk in the row
      const int sw = (ch & ~7) | ((ch & 7) ^ ((j & 1) << 2));
      cp_async16(sa + (size_t)j * a_stride + sw * 16, a0 + (size_t)j * p.K + ch * 8);
    }
  }
  cp_async_commit();

  // x fragment rows g and g+8 of this warp's m-tile, read straight from
  // global memory into a register ring of PF leaves; A fragments come from
  // the staged slice, or from global memory with the x ones when A is not
  // staged.
  const uint16_t *xr0 = p.x + (size_t)row0 * p.K + 8 * c;
  const uint16_t *xr1 = p.x + (size_t)row1 * p.K + 8 * c;
  const uint16_t *acol[NT];
#pragma unroll
  for (int t = 0; t < NT; t++)
    acol[t] = p.at + ((size_t)ti.adapter * p.r + ng * NGW + t * 8 + g) * p.K + 8 * c;
  auto load_leaf = [&](LeafFrag<NT> &f, int leaf) {
    const size_t k = (size_t)leaf * kLeaf;
#pragma unroll
    for (int h = 0; h < 2; h++) {
      f.xa[h][0] = v0 ? ldg128_stream(xr0 + k + 32 * h) : make_uint4(0, 0, 0, 0);
      f.xa[h][1] = v1 ? ldg128_stream(xr1 + k + 32 * h) : make_uint4(0, 0, 0, 0);
      if (!a_staged)
#pragma unroll
        for (int t = 0; t < NT; t++) f.ab[h][t] = ldg128(acol[t] + k + 32 * h);
    }
  };
  const int swz = (g & 1) << 2;
  // A fragments of leaf i (index inside the warp's group) from the slice
  auto a_frags = [&](LeafFrag<NT> &f, int i) {
    if (a_staged) {
      const int li = lgi * p.lg + i;               // leaf index inside the CTA's split
#pragma unroll
      for (int h = 0; h < 2; h++) {
        const int ch = ((h * 4 + c) ^ swz) << 4;
#pragma unroll
        for (int t = 0; t < NT; t++)
          f.ab[h][t] = *reinterpret_cast<const uint4 *>(sa + (size_t)(ng * NGW + t * 8 + g) * a_stride + li * 128 + ch);
      }
    }
  };

  // ---- this warp's leaves: [leaf0, leaf0 + lg), folded in post order
  const int leaf0 = split * p.lc + lgi * p.lg;
  float res[NT][4];                                // the group's subtree value
  LeafFrag<NT> ring[PF];
#pragma unroll
  for (int j = 0; j < PF; j++)
    if (j < p.lg) load_leaf(ring[j], leaf0 + j);
  if (a_staged) {
    cp_async_wait<0>();                              // this thread's A pieces
    __syncthreads();                                 // everyone's
  }

  if constexpr (LG > 0) {
    // binary counter over the group's leaves (every index a compile-time
    // constant), two leaves' MMAs interleaved when the ring allows it
    constexpr int LOG2 = LG >= 16 ? 4 : (LG >= 8 ? 3 : (LG >= 4 ? 2 : (LG >= 2 ? 1 : 0)));
    constexpr int NB = (LG >= 2 && PF % 2 == 0) ? 2 : 1;
    float lv[LOG2 > 0 ? LOG2 : 1][NT][4];
#pragma unroll
    for (int i0 = 0; i0 < LG; i0 += NB) {
      LeafFrag<NT> f[NB];
#pragma unroll
      for (int b = 0; b < NB; b++) {
        const int i = i0 + b;
        f[b] = ring[i % PF];
        if (i + PF < LG) load_leaf(ring[i % PF], leaf0 + i + PF);
        a_frags(f[b], i);
      }
      float acc[NB][NT][4];
      mma_leaves<NT, NB>(acc, f);
#pragma unroll
      for (int b = 0; b < NB; b++) {
        fold_leaf<NT, LOG2>(i0 + b, lv, acc[b]);
        if (i0 + b == LG - 1)
#pragma unroll
          for (int t = 0; t < NT; t++)
#pragma unroll
            for (int q = 0; q < 4; q++) res[t][q] = acc[b][t][q];
      }
    }
  } else {
    float st[MAXD][NT][4];
#pragma unroll
    for (int d = 0; d < MAXD; d++)
#pragma unroll
      for (int t = 0; t < NT; t++)
#pragma unroll
        for (int q = 0; q < 4; q++) st[d][t][q] = 0.0f;
    int depth = 0;
    for (int i0 = 0; i0 < p.lg; i0 += PF) {
#pragma unroll
      for (int j = 0; j < PF; j++) {
        const int i = i0 + j;
        if (i < p.lg) {
          LeafFrag<NT> f = ring[j];
          if (i + PF < p.lg) load_leaf(ring[j], leaf0 + i + PF);
          a_frags(f, i);
          float acc[NT][4];
          mma_leaf<NT>(acc, f);
          // push (every index is a compile-time constant, the slot is
          // chosen by predication)
#pragma unroll
          for (int d = 0; d < MAXD; d++) {
            const bool hit = d == depth;
#pragma unroll
            for (int t = 0; t < NT; t++)
#pragma unroll
              for (int q = 0; q < 4; q++) st[d][t][q] = hit ? acc[t][q] : st[d][t][q];
          }
          depth++;
          // merge the subtrees that end at this leaf: left = st[depth-2]
          const int nm = p.merges[i];
#pragma unroll 1
          for (int m = 0; m < nm; m++) {
#pragma unroll
            for (int d = 1; d < MAXD; d++) {
              const bool hit = d == depth - 1;
#pragma unroll
              for (int t = 0; t < NT; t++)
#pragma unroll
                for (int q = 0; q < 4; q++) {
                  const float sum = __fadd_rn(st[d - 1][t][q], st[d][t][q]);
                  st[d - 1][t][q] = hit ? sum : st[d - 1][t][q];
                }
            }
            depth--;
          }
        }
      }
    }
    if (depth != 1) flag_error(p.status, BI_ERR_INVALID_ARG);   // schedule inconsistent
#pragma unroll
    for (int t = 0; t < NT; t++)
#pragma unroll
      for (int q = 0; q < 4; q++) res[t][q] = st[0][t][q];
  }

  // ---- group values -> shared memory, element (local row, column)
  const int E = bm * p.r;
#pragma unroll
  for (int t = 0; t < NT; t++) {
    const int col = ng * NGW + t * 8 + 2 * c;
    float *dst = part + (size_t)lgi * E;
    *reinterpret_cast<float2 *>(dst + lr0 * p.r + col) = make_float2(res[t][0], res[t][1]);
    *reinterpret_cast<float2 *>(dst + lr1 * p.r + col) = make_float2(res[t][2], res[t][3]);
  }
  __syncthreads();
  float *slots = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(smem_f4) + p.g_offset);
  finish_tile(p, part, slots, &s_xbar, s_rows, ti.rows, bm, split, ti.adapter);
}

// ----------------------------------------------------------------------
// Bulk-copy kernel: the CTA's whole x slice (bm rows x lc leaves) and,
// when staged, its A slice (r rows x lc leaves) are requested from HBM by
// the copy engine as soon as the tile is known, one contiguous
// `cp.async.bulk` per row (rowbytes = lc * 128 bytes), so a CTA has every
// byte it needs in flight after two dependent reads (its table record,
// then x).  Each 16-row m-tile lands on its own mbarrier; its warps start
// multiplying as soon as their rows are in.  Used when the slice fits:
// lc <= 16 leaves per split (e.g. K = 4096 at splits >= 4).
//
// Shared memory: [0, 64) mbarriers (m-tiles 0..3, A = 4, TREE exchange = 5); [64, 320) token
// rows; [320, 328) adapter and rows; x rows at x_off (row stride rowbytes);
// A rows at a_offset; the group values at part_off (they may overlay the x
// rows, which are dead by then); the TREE exchange slots at g_offset.
//
// Fragment reads: threads (g, c) of an 8-lane phase read rows g = 2q and
// 2q + 1.  Rows are rowbytes apart (a multiple of 128), so the same 64-byte
// half of both rows would fall on the same banks; odd rows therefore read
// their two halves in the other order, which makes every phase
// conflict-free without padding.
// ----------------------------------------------------------------------
template <int NGW, int LG, bool ASTAGED>
__global__ void __launch_bounds__(256)
shrink_bulk_kernel(const __grid_constant__ ShrinkParams p) {
  constexpr int NT = NGW / 8;
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem);
  int32_t *s_rows = reinterpret_cast<int32_t *>(smem + 64);
  int *s_info = reinterpret_cast<int *>(smem + 320);
  constexpr int kABar = 4, kXBar = 5;           // A-slice barrier, TREE exchange barrier

  const int bm = 16 * p.mtiles;
  const int split = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const int g = lane >> 2, c = lane & 3;

  // ---- the tile: adapter, rows and their token indices (one read)
  if (warp == 0) tile_record(p, bm, blockIdx.y, lane, s_rows, s_info);
  if (warp == (nwarps > 1 ? 1 : 0) && lane == 0) {
#pragma unroll
    for (int i = 0; i <= kABar; i++) mbar_init(&bars[i], 1);
    mbar_fence_init();
    if (p.mode == BI_SHRINK_TREE && p.splits > 1) exchange_init(p, bm, split, &bars[kXBar]);
  }
  __syncthreads();
  const int adapter = s_info[0], rows = s_info[1];
  const bool clustered = p.mode == BI_SHRINK_TREE && p.splits > 1;
  if (clustered) cluster_arrive_relaxed();          // matched in finish_tile / below
  if (adapter < 0) {                                // uniform across the cluster
    if (clustered) cluster_wait();
    return;
  }
  if (adapter == p.n_ad) {                          // tokens without an adapter
    if (p.mode != BI_SHRINK_ATOMIC && split == 0)
      for (int e = threadIdx.x; e < rows * p.r; e += blockDim.x) p.y[(size_t)s_rows[e / p.r] * p.r + e % p.r] = 0.0f;
    if (clustered) cluster_wait();
    return;
  }

  // ---- every byte of the slice requested at once
  uint8_t *xs = smem + p.x_off;
  uint8_t *as = smem + p.a_offset;
  const uint32_t rb = (uint32_t)p.rowbytes;
  const size_t row_bytes = (size_t)p.K * 2;
  const size_t koff = (size_t)split * rb;           // this split's K range inside a row
  if (warp < p.mtiles) {
    const int nv = max(0, min(16, rows - 16 * warp));
    if (lane == 0) mbar_arrive_expect_tx(&bars[warp], (uint32_t)nv * rb);
    __syncwarp();
    if (lane < nv)
      bulk_load(xs + (size_t)(16 * warp + lane) * rb,
                reinterpret_cast<const uint8_t *>(p.x) + (size_t)s_rows[16 * warp + lane] * row_bytes + koff, rb,
                &bars[warp]);
  }
  if (ASTAGED && warp == (nwarps > p.mtiles ? p.mtiles : 0)) {
    if (lane == 0) mbar_arrive_expect_tx(&bars[kABar], (uint32_t)p.r * rb);
    __syncwarp();
    for (int j = lane; j < p.r; j += 32)
      bulk_load(as + (size_t)j * rb,
                reinterpret_cast<const uint8_t *>(p.at) + ((size_t)adapter * p.r + j) * row_bytes + koff, rb,
                &bars[kABar]);
  }

  // ---- warp role: (leaf group, m-tile, rank group)
  const int per_lg = p.mtiles * p.ngroups;
  const int lgi = warp / per_lg;
  const int mt = (warp % per_lg) / p.ngroups;
  const int ng = warp % p.ngroups;
  const int lr0 = mt * 16 + g, lr1 = lr0 + 8;

  // A fragments straight from global memory (L2) when A is not staged
  const uint16_t *acol[NT];
#pragma unroll
  for (int t = 0; t < NT; t++)
    acol[t] = p.at + ((size_t)adapter * p.r + ng * NGW + t * 8 + g) * p.K + (size_t)split * p.lc * kLeaf +
              (size_t)lgi * LG * kLeaf + 8 * c;
  LeafFrag<NT> agl[ASTAGED ? 1 : LG];
  if (!ASTAGED) {
#pragma unroll
    for (int i = 0; i < LG; i++)
#pragma unroll
      for (int h = 0; h < 2; h++)
#pragma unroll
        for (int t = 0; t < NT; t++) agl[ASTAGED ? 0 : i].ab[h][t] = ldg128(acol[t] + i * kLeaf + 32 * h);
  }

  bool ok = mbar_wait(&bars[mt], 0);
  if (ASTAGED) ok = mbar_wait(&bars[kABar], 0) && ok;
  if (!ok) flag_error(p.status, BI_ERR_TIMEOUT);

  const int odd = g & 1;
  const int hA = odd ? 64 : 0, hB = 64 - hA;
  const uint8_t *xr0 = xs + (size_t)lr0 * rb + c * 16;
  const uint8_t *xr1 = xr0 + (size_t)8 * rb;
  auto lds = [](const uint8_t *q) { return *reinterpret_cast<const uint4 *>(q); };

  float res[NT][4];
  {
    constexpr int LOG2 = LG >= 16 ? 4 : (LG >= 8 ? 3 : (LG >= 4 ? 2 : (LG >= 2 ? 1 : 0)));
    constexpr int NB = LG < 4 ? LG : 4;             // leaves whose MMAs are interleaved
    float lv[LOG2 > 0 ? LOG2 : 1][NT][4];
#pragma unroll
    for (int i0 = 0; i0 < LG; i0 += NB) {
      LeafFrag<NT> f[NB];
#pragma unroll
      for (int b = 0; b < NB; b++) {
        const int i = i0 + b;
        const int lb = (lgi * LG + i) * 128;
        const uint4 p0 = lds(xr0 + lb + hA), p1 = lds(xr0 + lb + hB);
        const uint4 q0 = lds(xr1 + lb + hA), q1 = lds(xr1 + lb + hB);
        f[b].xa[0][0] = odd ? p1 : p0;
        f[b].xa[1][0] = odd ? p0 : p1;
        f[b].xa[0][1] = odd ? q1 : q0;
        f[b].xa[1][1] = odd ? q0 : q1;
        if (ASTAGED) {
#pragma unroll
          for (int t = 0; t < NT; t++) {
            const uint8_t *ar = as + (size_t)(ng * NGW + t * 8 + g) * rb + c * 16 + lb;
            const uint4 a0 = lds(ar + hA), a1 = lds(ar + hB);
            f[b].ab[0][t] = odd ? a1 : a0;
            f[b].ab[1][t] = odd ? a0 : a1;
          }
        } else {
#pragma unroll
          for (int h = 0; h < 2; h++)
#pragma unroll
            for (int t = 0; t < NT; t++) f[b].ab[h][t] = agl[ASTAGED ? 0 : i].ab[h][t];
        }
      }
      float acc[NB][NT][4];
      mma_leaves<NT, NB>(acc, f);
#pragma unroll
      for (int b = 0; b < NB; b++) {
        fold_leaf<NT, LOG2>(i0 + b, lv, acc[b]);
        if (i0 + b == LG - 1)
#pragma unroll
          for (int t = 0; t < NT; t++)
#pragma unroll
            for (int q = 0; q < 4; q++) res[t][q] = acc[b][t][q];
      }
    }
  }
  if (!ok) {
    // a copy may still be landing: wait for it (bounded) before the rows'
    // space is reused or the CTA exits
    mbar_wait(&bars[mt], 0);
    if (ASTAGED) mbar_wait(&bars[kABar], 0);
  }
  __syncthreads();                                  // every warp is done with the x rows

  // ---- group values -> shared memory (over the x rows), then the combine
  float *part = reinterpret_cast<float *>(smem + p.part_off);
  const int E = bm * p.r;
#pragma unroll
  for (int t = 0; t < NT; t++) {
    const int col = ng * NGW + t * 8 + 2 * c;
    float *dst = part + (size_t)lgi * E;
    *reinterpret_cast<float2 *>(dst + lr0 * p.r + col) = make_float2(res[t][0], res[t][1]);
    *reinterpret_cast<float2 *>(dst + lr1 * p.r + col) = make_float2(res[t][2], res[t][3]);
  }
  __syncthreads();
  float *slots = reinterpret_cast<float *>(smem + p.g_offset);
  finish_tile(p, part, slots, &bars[kXBar], s_rows, rows, bm, split, adapter);
}

// ----------------------------------------------------------------------
// Host side
// ----------------------------------------------------------------------

// Post-order merge schedule of the canonical tree over n leaves: after leaf
// i is pushed, merges[i] internal nodes end there.  Returns the largest
// stack depth reached.
static int tree_merge_schedule(int n, uint8_t *merges) {
  std::fill(merges, merges + n, 0);
  struct Rec {
    static void go(int lo, int hi, uint8_t *m) {
      if (hi - lo <= 1) return;
      const int h = lo + (hi - lo + 1) / 2;
      go(lo, h, m);
      go(h, hi, m);
      m[hi - 1]++;
    }
  };
  Rec::go(0, n, merges);
  int depth = 0, maxd = 0;
  for (int i = 0; i < n; i++) {
    depth++;
    maxd = std::max(maxd, depth);
    depth -= merges[i];
  }
  return maxd;
}

template <int NGW, int MAXD, int PF, int LG>
static cudaError_t launch_shrink_t(const ShrinkParams &p, int tiles, int threads, size_t smem,
                                   cudaStream_t stream) {
  void (*kern)(ShrinkParams);
  if constexpr (PF == 4) kern = shrink_kernel<NGW, MAXD, PF, true, LG>;   // chosen only with A staged
  else kern = p.a_staged ? shrink_kernel<NGW, MAXD, PF, true, LG> : shrink_kernel<NGW, MAXD, PF, false, LG>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.splits, tiles, 1);
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  int na = 0;
  if (p.mode == BI_SHRINK_TREE && p.splits > 1) {
    if (p.splits > 8) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return e;
    }
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = p.splits;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    na = 1;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

static cudaError_t launch_bulk(void (*kern)(ShrinkParams), const ShrinkParams &p, int tiles, int threads, size_t smem,
                               cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.splits, tiles, 1);
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  int na = 0;
  if (p.mode == BI_SHRINK_TREE && p.splits > 1) {
    if (p.splits > 8) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return e;
    }
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = p.splits;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    na = 1;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

template <int NGW, bool ASTAGED>
static void (*bulk_kernel_for(int lg))(ShrinkParams) {
  switch (lg) {
    case 1: return shrink_bulk_kernel<NGW, 1, ASTAGED>;
    case 2: return shrink_bulk_kernel<NGW, 2, ASTAGED>;
    case 4: return shrink_bulk_kernel<NGW, 4, ASTAGED>;
    default:
      if constexpr (ASTAGED) {
        if (lg == 8) return shrink_bulk_kernel<NGW, 8, true>;
        if (lg == 16) return shrink_bulk_kernel<NGW, 16, true>;
      }
      return nullptr;
  }
}

static void (*bulk_kernel(int ngw, bool staged, int lg))(ShrinkParams) {
  if (ngw == 16) return staged ? bulk_kernel_for<16, true>(lg) : bulk_kernel_for<16, false>(lg);
  return staged ? bulk_kernel_for<8, true>(lg) : bulk_kernel_for<8, false>(lg);
}

// Tiling of the bulk-copy kernel (bit-neutral), or false when the slice does
// not fit it: up to four 16-row m-tiles (at most 64 KB of x rows), then
// leaf groups until the CTA has eight warps; A staged in shared memory when
// its slice is at most 64 KB, else read from L2 by the warps (then at most
// four leaves per warp, their A fragments held in registers).
static bool bulk_tiling(ShrinkParams &p, int M, bool segmented, int &threads, int &tiles, size_t &smem) {
  const int rb = p.lc * 128;
  if (16 * rb > 64 * 1024) return false;
  int mt = std::min(4, (M + 15) / 16);
  while (mt > 1 && (mt * p.ngroups > 8 || 16 * mt * rb > 64 * 1024)) mt >>= 1;
  int G = 1;
  while (p.lc % (2 * G) == 0 && 2 * G * mt * p.ngroups <= 8) G *= 2;
  const int lg = p.lc / G;
  if (lg != 1 && lg != 2 && lg != 4 && lg != 8 && lg != 16) return false;
  const size_t a_bytes = (size_t)p.r * rb;
  const bool staged = a_bytes <= 64 * 1024;
  if (!staged && lg > 4) return false;
  const int bm = 16 * mt;
  p.mtiles = mt;
  p.groups = G;
  p.lg = lg;
  p.a_staged = staged ? 1 : 0;
  p.rowbytes = rb;
  p.sub = kPlanTile / bm;
  p.x_off = 512;
  size_t off = (size_t)p.x_off + (size_t)bm * rb;
  p.a_offset = (int)off;
  if (staged) off += a_bytes;
  const size_t part_bytes = (size_t)G * bm * p.r * sizeof(float);
  if (part_bytes <= (size_t)bm * rb) {
    p.part_off = p.x_off;
  } else {
    p.part_off = (int)off;
    off += part_bytes;
  }
  const size_t part1 = (size_t)bm * p.r * sizeof(float);
  p.gather0 = p.mode == BI_SHRINK_TREE && p.splits > 1 && (size_t)(p.splits - 1) * part1 <= 8 * 1024 ? 1 : 0;
  off = (off + 127) & ~size_t(127);
  p.g_offset = (int)off;
  if (p.mode == BI_SHRINK_TREE && p.splits > 1) off += p.gather0 ? (size_t)(p.splits - 1) * part1 : part1;
  smem = off;
  threads = 32 * G * mt * p.ngroups;
  tiles = segmented ? (int)plan_tiles(M, p.n_ad) * p.sub : (M + bm - 1) / bm;
  return smem <= 200 * 1024;
}

// The expand half of a fused call.
struct FuseArgs {
  const void *B;            // [n_ad][N][r] bf16
  float *out;               // [M][N] fp32
  int N, accumulate;
};

// Validates, picks the kernel and its (bit-neutral) tiling and launches.
// perm / offsets / table are null for the single-adapter call; fuse is
// null except for bi_lora_fused.
bi_status shrink_launch(const void *x, const void *A, const int32_t *perm, const int32_t *offsets,
                        const int32_t *table, int n_ad, float *y, int M, int K, int r, int splits, int mode,
                        cudaStream_t stream, const FuseArgs *fuse = nullptr) {
  if (M < 0 || K <= 0 || r <= 0 || n_ad < 1) return BI_ERR_INVALID_ARG;
  if (mode != BI_SHRINK_UNSPLIT && mode != BI_SHRINK_ATOMIC && mode != BI_SHRINK_TREE)
    return BI_ERR_INVALID_ARG;
  if (M > 0 && (!x || !A || (!y && !fuse))) return BI_ERR_INVALID_ARG;
  if (K % kLeaf != 0 || r % 8 != 0 || r > 128) return BI_ERR_UNSUPPORTED_SHAPE;
  const int L = K / kLeaf;
  if (mode == BI_SHRINK_UNSPLIT && splits != 1) return BI_ERR_UNSUPPORTED_SHAPE;
  if (!bi_pow2(splits) || splits > kMaxSplits || L % splits != 0) return BI_ERR_UNSUPPORTED_SHAPE;
  if (!bi_aligned16(x) || !bi_aligned16(A)) return BI_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return BI_OK;

  ShrinkParams p{};
  p.x = static_cast<const uint16_t *>(x);
  p.at = static_cast<const uint16_t *>(A);
  p.perm = perm;
  p.offsets = offsets;
  p.table = table;
  p.y = y;
  p.status = status_word();
  p.M = M; p.K = K; p.r = r; p.n_ad = n_ad;
  p.splits = splits;
  p.mode = mode;
  p.lc = L / splits;

  const int ngw = (r % 16 == 0) ? 16 : 8;
  p.ngroups = r / ngw;
  if (p.ngroups > 8) return BI_ERR_UNSUPPORTED_SHAPE;

  if (fuse) {
    if (mode == BI_SHRINK_ATOMIC) return BI_ERR_UNSUPPORTED_SHAPE;
    if (fuse->N <= 0 || !fuse->B || !fuse->out) return BI_ERR_INVALID_ARG;
    if (fuse->N % 8 != 0 || !bi_aligned16(fuse->B) || !bi_aligned16(fuse->out)) return BI_ERR_UNSUPPORTED_SHAPE;
    p.fuse = 1;
    p.bt = static_cast<const uint16_t *>(fuse->B);
    p.out = fuse->out;
    p.N = fuse->N;
    p.accumulate = fuse->accumulate ? 1 : 0;
  }
  if (!fuse) {
    ShrinkParams q = p;
    int threads = 0, tiles = 0;
    size_t smem = 0;
    void (*kern)(ShrinkParams) = nullptr;
    if (bulk_tiling(q, M, table != nullptr, threads, tiles, smem)) kern = bulk_kernel(ngw, q.a_staged != 0, q.lg);
    // The bulk kernel has every CTA request its whole slice at once, which
    // wins while the grid is resident in one wave (measured: M = 1024 at
    // split-K 8 in 7.3 us against 9-10 us); beyond that its 64 KB of x per
    // CTA halves the CTAs per SM and the register-ring kernel streams faster.
    int per_sm = 0;
    if (kern && cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) == cudaSuccess &&
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem) == cudaSuccess &&
        (long)tiles * splits * (splits > 1 && mode == BI_SHRINK_TREE ? 8 : 7) <= 7L * per_sm * num_sms()) {
      if (mode == BI_SHRINK_ATOMIC) BI_CUDA_TRY(cudaMemsetAsync(y, 0, (size_t)M * r * sizeof(float), stream));
      return launch_bulk(kern, q, tiles, threads, smem, stream) == cudaSuccess ? BI_OK : BI_ERR_CUDA;
    }
  }
  // Tiling (bit-neutral).  Leaf groups first: enough warps per row tile
  // that each walks at most 8 leaves (a power of two dividing the split's
  // leaves); then up to 4 row tiles of 16, at most 8 warps per CTA.
  int G = 1;
  while (p.lc / G > 8 && p.lc % (G * 2) == 0 && G * 2 * p.ngroups <= 8) G *= 2;
  int mt = std::min(4, (M + 15) / 16);
  while (mt > 1 && mt * G * p.ngroups > 8) mt >>= 1;
  // one row tile of 16 (decode-sized M): spend the CTA's eight warps on
  // leaf groups instead, so that every leaf's loads leave at once
  if (mt == 1)
    while (p.lc % (G * 2) == 0 && G * 2 * p.ngroups <= 8) G *= 2;
  p.mtiles = mt;
  p.groups = G;
  p.lg = p.lc / G;
  if (p.lg > kMaxGroupLeaves) return BI_ERR_UNSUPPORTED_SHAPE;
  const int depth = tree_merge_schedule(p.lg, p.merges);
  const int warps = G * mt * p.ngroups;
  const int threads = 32 * warps;
  const int bm = 16 * mt;
  const size_t part_bytes = ((size_t)G * bm * r * sizeof(float) + 127) & ~size_t(127);
  const size_t a_bytes = (size_t)r * p.lc * 128;
  p.a_staged = a_bytes <= 64 * 1024 ? 1 : 0;
  // x leaves in flight per thread: four when A comes from shared memory
  // (100 registers, four CTAs per SM), else two (A rides in the ring too)
  const int pf = p.lg >= 4 && p.a_staged ? 4 : (p.lg >= 2 ? 2 : 1);
  p.a_offset = (int)part_bytes;
  // mode TREE exchange slots: one partial's worth (S shares of E/S) for the
  // reduce-scatter; S-1 partials in rank 0 for small tiles (<= 8 KB in all),
  // where one CTA adding everything beats spreading it (M = 16: 2.8 us
  // against 4.8 us; at 64-row tiles the rank-0 gather took 19 us)
  const size_t part1 = (size_t)bm * r * sizeof(float);
  p.gather0 = mode == BI_SHRINK_TREE && splits > 1 && (size_t)(splits - 1) * part1 <= 8 * 1024 ? 1 : 0;
  const size_t slot_bytes = mode == BI_SHRINK_TREE && splits > 1 ? (p.gather0 ? (size_t)(splits - 1) * part1 : part1) : 0;
  const size_t base_smem = part_bytes + (p.a_staged ? a_bytes : 0);
  p.g_offset = (int)base_smem;
  size_t smem = base_smem + slot_bytes;
  if (p.fuse) {
    // the tile's full y rows, then one 16 x 68 float strip buffer per warp
    smem = (smem + 15) & ~size_t(15);
    p.yfull_rel = (int)smem;                       // part sits at offset 0
    const size_t yfull_bytes = ((size_t)bm * r * sizeof(float) + 15) & ~size_t(15);
    p.stage_rel = (int)yfull_bytes;
    smem += yfull_bytes + (size_t)warps * 16 * 68 * sizeof(float);
  }
  p.sub = kPlanTile / bm;
  const int tiles = table ? (int)plan_tiles(M, n_ad) * p.sub : (M + bm - 1) / bm;

  if (mode == BI_SHRINK_ATOMIC) {
    BI_CUDA_TRY(cudaMemsetAsync(y, 0, (size_t)M * r * sizeof(float), stream));
  }
  cudaError_t e;
  // a power-of-two leaf count per warp up to 16 runs the unrolled counter
  const int lgc = (p.lg == 1 || p.lg == 2 || p.lg == 4 || p.lg == 8 || p.lg == 16) ? p.lg : 0;
#define BI_SHRINK_LG(NGW_, PF_)                                                   \
  (lgc == 1    ? launch_shrink_t<NGW_, 4, PF_, 1>(p, tiles, threads, smem, stream)  \
   : lgc == 2  ? launch_shrink_t<NGW_, 4, PF_, 2>(p, tiles, threads, smem, stream)  \
   : lgc == 4  ? launch_shrink_t<NGW_, 4, PF_, 4>(p, tiles, threads, smem, stream)  \
   : lgc == 8  ? launch_shrink_t<NGW_, 4, PF_, 8>(p, tiles, threads, smem, stream)  \
   : lgc == 16 ? launch_shrink_t<NGW_, 4, PF_, 16>(p, tiles, threads, smem, stream) \
   : depth <= 4 ? launch_shrink_t<NGW_, 4, PF_, 0>(p, tiles, threads, smem, stream) \
   : depth <= 8 ? launch_shrink_t<NGW_, 8, PF_, 0>(p, tiles, threads, smem, stream) \
                : launch_shrink_t<NGW_, 12, PF_, 0>(p, tiles, threads, smem, stream))
#define BI_SHRINK_PF(NGW_, MAXD_)                                     \
  (pf == 4 ? BI_SHRINK_LG(NGW_, 4) : pf == 2 ? BI_SHRINK_LG(NGW_, 2) : BI_SHRINK_LG(NGW_, 1))
  if (ngw == 16) e = BI_SHRINK_PF(16, 0);
  else e = BI_SHRINK_PF(8, 0);
#undef BI_SHRINK_LG
#undef BI_SHRINK_PF
  return e == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

}  // namespace bi

extern "C" bi_status bi_lora_shrink(const void *x, const void *A, float *y, int M, int K, int r,
                                    int splits, int mode, bi_stream_t stream) {
  return bi::shrink_launch(x, A, nullptr, nullptr, nullptr, 1, y, M, K, r, splits, mode,
                           reinterpret_cast<cudaStream_t>(stream));
}

extern "C" bi_status bi_lora_fused(const void *x, const void *A, const void *B, const void *plan, int n_adapters,
                                   float *y, float *out, int M, int K, int r, int N, int splits, int accumulate,
                                   bi_stream_t stream) {
  if (M > 0 && !plan) return BI_ERR_INVALID_ARG;
  if (n_adapters < 1 || n_adapters > bi::kMaxAdapters) return BI_ERR_INVALID_ARG;
  if (M > 0 && !bi_aligned16(plan)) return BI_ERR_UNSUPPORTED_SHAPE;
  if (y && !bi_aligned16(y)) return BI_ERR_UNSUPPORTED_SHAPE;
  const int32_t *perm = static_cast<const int32_t *>(plan);
  const int32_t *table = perm + bi::plan_table_word(M, n_adapters);
  bi::FuseArgs f{B, out, N, accumulate};
  return bi::shrink_launch(x, A, perm, perm + M, table, n_adapters, y, M, K, r, splits,
                           splits > 1 ? BI_SHRINK_TREE : BI_SHRINK_UNSPLIT, reinterpret_cast<cudaStream_t>(stream), &f);
}

extern "C" bi_status bi_lora_shrink_segmented(const void *x, const void *A, const void *plan,
                                              int n_adapters, float *y, int M, int K, int r,
                                              int splits, int mode, bi_stream_t stream) {
  if (M > 0 && !plan) return BI_ERR_INVALID_ARG;
  if (n_adapters < 1 || n_adapters > bi::kMaxAdapters) return BI_ERR_INVALID_ARG;
  if (M > 0 && !bi_aligned16(plan)) return BI_ERR_UNSUPPORTED_SHAPE;
  const int32_t *perm = static_cast<const int32_t *>(plan);
  const int32_t *offsets = perm + M;
  const int32_t *table = perm + bi::plan_table_word(M, n_adapters);
  return bi::shrink_launch(x, A, perm, offsets, table, n_adapters, y, M, K, r, splits, mode,
                           reinterpret_cast<cudaStream_t>(stream));
}
