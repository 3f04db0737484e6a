// gemm_tree.cu -- tensor-parallel-invariant GEMM: C = A . W^T with the K
// reduction ordered by one hierarchical binary tree.
//
// "Deterministic Inference across Tensor Parallel Sizes That Eliminates
// Training-Inference Mismatch" (Abstract): with intra- and inter-GPU
// reductions aligned on one hierarchical binary tree, the result is the
// same bits for every TP size.
//
// Order: K is cut into leaves of 256.  A leaf is one TMEM accumulation of
// sixteen tcgen05.mma (M=128, K=16), restarted from zero for every leaf.
// Leaves are combined in fp32 by the canonical tree.  A shard (an emulated
// TP rank) owns a contiguous block of L/shards leaves -- one subtree -- and
// writes its partial; bi_tree_combine adds the top levels.  The bits of an
// accumulator element depend on its row of A, its row of W and the K order
// only, not on the instruction's N, so the two tile widths below give the
// same leaves (a test checks this against the batch-invariant GEMM).
//
// Per CTA (persistent, 320 threads): warp 0 issues TMA loads into a stage
// ring, warp 1 issues the MMAs into one of two TMEM leaf buffers, warps
// 2..9 fold finished leaves into the pending stack of the post-order tree
// walk; each epilogue thread owns one row (its TMEM lane) and half of the
// tile's columns.  Two layouts:
//  * BN = 128, 1/2/4/8/16 leaves per shard (known at compile time): the walk
//    is a binary counter; level 0 of the pending stack sits in registers,
//    the higher levels in TMEM (2 x 128 leaf buffers + 2 x 128 stack, or for
//    16 leaves 1 x 128 buffer + 3 x 128 stack: 512 columns either way).
//    The wide tile halves the operand bytes per flop that L2 must deliver.
//  * BN = 64, any leaf count up to 64: the host-computed post-order schedule
//    (merges per leaf), stack of 6 slots in TMEM (2 x 64 + 6 x 64 columns).
#include "tc.cuh"

#include <algorithm>

namespace bi {

bi_status tree_combine_launch(const float *partials, float *out, int s, size_t count, cudaStream_t stream);

namespace tg {
constexpr int BM = 128, BK = 64, LEAF = 256;
constexpr int KB_PER_LEAF = LEAF / BK;                // 4
constexpr int A_BYTES = BM * BK * 2;                  // 16 KB
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 32 * (2 + EPI_WARPS);         // 320
constexpr uint32_t TMEM_COLS = 512;
constexpr int STACK_SLOTS = 6;                        // BN = 64 layout
constexpr int MAX_LEAVES = 64;                        // per shard
constexpr int MAX_STAGES = 8;
template <int BN>
struct Cfg {
  static constexpr int STAGES = BN == 64 ? 8 : 6;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr size_t SMEM = 1024 + STAGES * STAGE_BYTES + 256;
};
}  // namespace tg

struct TreeGemmParams {
  float *out;          // shards == 1: C [M][N]; else partials [shards][M][N]
  unsigned *status;
  int M, N, K, shards, leaves;   // leaves per shard
  uint8_t merges[tg::MAX_LEAVES];
};

struct TreeSmemTail {
  uint64_t full[tg::MAX_STAGES];
  uint64_t empty[tg::MAX_STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;            // the MMA issuer's last commit, before TMEM is freed
  uint32_t tmem_base;
  uint32_t bail;
};

template <int N>
BI_DEV void add_rn(float (&cur)[N], const float (&left)[N]) {
#pragma unroll
  for (int q = 0; q < N; q++) cur[q] = __fadd_rn(left[q], cur[q]);
}

// LPS = 0: BN = 64, any leaf count (p.merges).  LPS = 1, 2, 4, 8, 16: BN = 128.
template <int BN, int LPS>
__global__ void __launch_bounds__(tg::THREADS, 1)
gemm_tree_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW,
                 const __grid_constant__ TreeGemmParams p) {
  using namespace tg;
  using C = Cfg<BN>;
  constexpr int STAGES = C::STAGES;
  constexpr int B_BYTES = C::B_BYTES;
  constexpr int STAGE_BYTES = C::STAGE_BYTES;
  static_assert(LPS == 0 || BN == 128, "counter layout is the 128-wide tile");
  static_assert(LPS != 0 || BN == 64, "schedule layout is the 64-wide tile");
  constexpr int LOG2 = LPS >= 16 ? 4 : (LPS >= 8 ? 3 : (LPS >= 4 ? 2 : (LPS >= 2 ? 1 : 0)));
  // TMEM leaf buffers: two, except for 16 leaves, whose three TMEM levels
  // (128 columns each) leave room for one
  constexpr int NBUF = LPS == 16 ? 1 : 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sa = smem;
  uint8_t *sb = smem + STAGES * A_BYTES;
  TreeSmemTail *tail = reinterpret_cast<TreeSmemTail *>(smem + STAGES * STAGE_BYTES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_m = (p.M + BM - 1) / BM, tiles_n = p.N / BN;
  const int num_tiles = tiles_m * tiles_n * p.shards;
  const int L = LPS ? LPS : p.leaves;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; s++) {
      mbar_init(&tail->full[s], 1);
      mbar_init(&tail->empty[s], 1);
    }
    for (int b = 0; b < 2; b++) {
      mbar_init(&tail->tfull[b], 1);
      mbar_init(&tail->tempty[b], EPI_WARPS);
    }
    mbar_init(&tail->drain, 1);
    tail->bail = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(&tail->tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tail->tmem_base;
  volatile uint32_t *bail = &tail->bail;

  // tile -> (m block, n block, shard); m fastest so concurrent CTAs share W
  auto decode = [&](int t, int &mb, int &nb, int &sh) {
    mb = t % tiles_m;
    t /= tiles_m;
    nb = t % tiles_n;
    sh = t / tiles_n;
  };

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_par = 0;           // per stage: loads in flight, and their phase
      for (int tile = blockIdx.x; tile < num_tiles && !*bail; tile += gridDim.x) {
        int mb, nb, sh;
        decode(tile, mb, nb, sh);
        const int kb0 = sh * L * KB_PER_LEAF;
        for (int kb = 0; kb < L * KB_PER_LEAF; kb++) {
          if (!mbar_wait(&tail->empty[stage], phase ^ 1)) {
            flag_error(p.status, BI_ERR_TIMEOUT);
            *bail = 1;
            break;
          }
          mbar_arrive_expect_tx(&tail->full[stage], STAGE_BYTES);
          tma_load_2d(&tmA, &tail->full[stage], sa + stage * A_BYTES, (kb0 + kb) * BK, mb * BM);
          tma_load_2d(&tmW, &tail->full[stage], sb + stage * B_BYTES, (kb0 + kb) * BK, nb * BN);
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // every load issued has landed before the CTA's shared memory is
      // given up (a stage the MMAs consumed passes at once)
      for (int s = 0; s < STAGES; s++)
        if ((issued >> s) & 1u)
          if (!mbar_wait(&tail->full[s], (issued_par >> s) & 1u)) flag_error(p.status, BI_ERR_TIMEOUT);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      int buf = 0;
      uint32_t buf_phase = 0;
      for (int tile = blockIdx.x; tile < num_tiles && !*bail; tile += gridDim.x) {
        for (int leaf = 0; leaf < L && !*bail; leaf++) {
          if (!mbar_wait(&tail->tempty[buf], buf_phase ^ 1)) {
            flag_error(p.status, BI_ERR_TIMEOUT);
            *bail = 1;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem + (uint32_t)(buf * BN);
          for (int kb = 0; kb < KB_PER_LEAF; kb++) {
            if (!mbar_wait(&tail->full[stage], phase)) {
              flag_error(p.status, BI_ERR_TIMEOUT);
              *bail = 1;
              break;
            }
            tc_fence_after();
            const uint32_t a0 = smem_u32(sa + stage * A_BYTES);
            const uint32_t b0 = smem_u32(sb + stage * B_BYTES);
#pragma unroll
            for (int k = 0; k < BK / 16; k++)
              umma_bf16(d, umma_desc_kmajor_sw128(a0 + 32 * k), umma_desc_kmajor_sw128(b0 + 32 * k), idesc,
                        (kb | k) != 0);                     // every leaf restarts from zero
            umma_commit(&tail->empty[stage]);
            if (++stage == STAGES) { stage = 0; phase ^= 1; }
          }
          umma_commit(&tail->tfull[buf]);
          if (++buf == NBUF) { buf = 0; buf_phase ^= 1; }
        }
      }
      // every MMA issued has completed before TMEM is freed
      umma_commit(&tail->drain);
      if (!mbar_wait(&tail->drain, 0)) flag_error(p.status, BI_ERR_TIMEOUT);
    }
  } else if constexpr (LPS == 0) {
    // ---------------- epilogue: post-order fold of the leaves, stack in TMEM
    const int ew = warp - 2;
    const int quad = warp & 3;                  // TMEM lane quadrant of this warp
    const int half = ew >> 2;                   // which 32 of the 64 columns
    const uint32_t lane_off = (uint32_t)(32 * quad) << 16;
    const uint32_t col_off = (uint32_t)(32 * half);
    int buf = 0;
    uint32_t buf_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      if (*bail) break;
      int mb, nb, sh;
      decode(tile, mb, nb, sh);
      int top = 0;
      for (int leaf = 0; leaf < L; leaf++) {
        if (!__all_sync(0xffffffffu, mbar_wait(&tail->tfull[buf], buf_phase))) {   // warp-uniform exit
          flag_error(p.status, BI_ERR_TIMEOUT);
          *bail = 1;
          break;
        }
        tc_fence_after();
        uint32_t cur[32];
        tmem_ld32(tmem + lane_off + (uint32_t)(buf * BN) + col_off, cur);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tail->tempty[buf]);
        if (++buf == NBUF) { buf = 0; buf_phase ^= 1; }
        // subtrees that end at this leaf: cur = left + cur, left popped
        for (int m = p.merges[leaf]; m > 0; m--) {
          top--;
          uint32_t left[32];
          tmem_ld32(tmem + lane_off + (uint32_t)(2 * BN + top * BN) + col_off, left);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; i++)
            cur[i] = __float_as_uint(__fadd_rn(__uint_as_float(left[i]), __uint_as_float(cur[i])));
        }
        if (leaf + 1 < L) {
          tmem_st32(tmem + lane_off + (uint32_t)(2 * BN + top * BN) + col_off, cur);
          tmem_wait_st();
          top++;
        } else {
          const int row = mb * BM + 32 * quad + lane;
          if (row < p.M) {
            float *dst = p.out + ((size_t)sh * p.M + row) * p.N + nb * BN + 32 * half;
#pragma unroll
            for (int j = 0; j < 8; j++)
              *reinterpret_cast<uint4 *>(dst + 4 * j) = make_uint4(cur[4 * j], cur[4 * j + 1], cur[4 * j + 2], cur[4 * j + 3]);
          }
        }
      }
    }
  } else {
    // ---------------- epilogue: binary counter over LPS leaves.  Leaf i
    // closes the subtrees of the levels where its index has a 1 bit (left =
    // the waiting subtree, right = the one just finished); at its lowest 0
    // bit it parks the result.  Level 0 parks in registers, level L >= 1 in
    // TMEM columns from (NBUF + L - 1) * 128.
    const int ew = warp - 2;
    const int quad = warp & 3;                  // TMEM lane quadrant of this warp
    const int half = ew >> 2;                   // which 64 of the 128 columns
    const uint32_t lane_off = (uint32_t)(32 * quad) << 16;
    const uint32_t col_off = (uint32_t)(64 * half);
    int buf = 0;
    uint32_t buf_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      if (*bail) break;
      int mb, nb, sh;
      decode(tile, mb, nb, sh);
      float lvl0[64];
      float cur[64];
      bool ok = true;
#pragma unroll
      for (int i = 0; i < LPS; i++) {
        if (!__all_sync(0xffffffffu, mbar_wait(&tail->tfull[buf], buf_phase))) {   // warp-uniform exit
          flag_error(p.status, BI_ERR_TIMEOUT);
          *bail = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        {
          uint32_t v0[32], v1[32];
          const uint32_t src = tmem + lane_off + (uint32_t)(buf * BN) + col_off;
          tmem_ld32(src, v0);
          tmem_ld32(src + 32, v1);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tail->tempty[buf]);
#pragma unroll
          for (int q = 0; q < 32; q++) {
            cur[q] = __uint_as_float(v0[q]);
            cur[32 + q] = __uint_as_float(v1[q]);
          }
        }
        if (++buf == NBUF) { buf = 0; buf_phase ^= 1; }
        if constexpr (LOG2 >= 1) {
          if ((i & 1) == 0) {
#pragma unroll
            for (int q = 0; q < 64; q++) lvl0[q] = cur[q];
            continue;
          }
          add_rn(cur, lvl0);
#pragma unroll
          for (int lv = 1; lv < LOG2; lv++) {
            const uint32_t slot = tmem + lane_off + (uint32_t)(NBUF * BN + (lv - 1) * BN) + col_off;
            if (((i >> lv) & 1) == 0) {
              uint32_t w0[32], w1[32];
#pragma unroll
              for (int q = 0; q < 32; q++) {
                w0[q] = __float_as_uint(cur[q]);
                w1[q] = __float_as_uint(cur[32 + q]);
              }
              tmem_st32(slot, w0);
              tmem_st32(slot + 32, w1);
              break;
            }
            tmem_wait_st();                       // this thread's parked subtree has landed
            uint32_t l0[32], l1[32];
            tmem_ld32(slot, l0);
            tmem_ld32(slot + 32, l1);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 32; q++) {
              cur[q] = __fadd_rn(__uint_as_float(l0[q]), cur[q]);
              cur[32 + q] = __fadd_rn(__uint_as_float(l1[q]), cur[32 + q]);
            }
          }
        }
      }
      if (!ok) break;
      const int row = mb * BM + 32 * quad + lane;
      if (row < p.M) {
        float *dst = p.out + ((size_t)sh * p.M + row) * p.N + nb * BN + 64 * half;
#pragma unroll
        for (int j = 0; j < 16; j++)
          *reinterpret_cast<float4 *>(dst + 4 * j) = make_float4(cur[4 * j], cur[4 * j + 1], cur[4 * j + 2], cur[4 * j + 3]);
      }
    }
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host

void tree_schedule(int n, uint8_t *merges);

static int schedule_depth(int n, const uint8_t *merges) {
  int depth = 0, maxd = 0;
  for (int i = 0; i < n; i++) {
    depth++;
    maxd = std::max(maxd, depth);
    depth -= merges[i];
  }
  return maxd;
}

static bi_status tree_check(const void *A, const void *W, int M, int N, int K, int shards) {
  if (M < 0 || N <= 0 || K <= 0 || shards < 1) return BI_ERR_INVALID_ARG;
  if (M > 0 && (!A || !W)) return BI_ERR_INVALID_ARG;
  if (K % tg::LEAF != 0 || N % 64 != 0) return BI_ERR_UNSUPPORTED_SHAPE;
  const int L = K / tg::LEAF;
  if (!bi_pow2(shards) || L % shards != 0 || L / shards > tg::MAX_LEAVES) return BI_ERR_UNSUPPORTED_SHAPE;
  if (!bi_aligned16(A) || !bi_aligned16(W)) return BI_ERR_UNSUPPORTED_SHAPE;
  return BI_OK;
}

static bi_status tree_partials_launch(const void *A, const void *W, float *out, int M, int N, int K, int shards,
                                      cudaStream_t stream) {
  using namespace tg;
  TreeGemmParams p{};
  p.out = out;
  p.status = status_word();
  p.M = M; p.N = N; p.K = K; p.shards = shards;
  p.leaves = K / LEAF / shards;
  tree_schedule(p.leaves, p.merges);
  if (schedule_depth(p.leaves, p.merges) > STACK_SLOTS + 1) return BI_ERR_UNSUPPORTED_SHAPE;
  const int lps = p.leaves;
  const bool wide = N % 128 == 0 && (lps == 1 || lps == 2 || lps == 4 || lps == 8 || lps == 16);
  const int bn = wide ? 128 : 64;
  CUtensorMap tmA, tmW;
  if (!make_tma_2d_bf16(&tmA, A, (uint64_t)K, (uint64_t)M, BK, BM)) return BI_ERR_CUDA;
  if (!make_tma_2d_bf16(&tmW, W, (uint64_t)K, (uint64_t)N, BK, bn)) return BI_ERR_CUDA;
  const long tiles = (long)((M + BM - 1) / BM) * (N / bn) * shards;
  const int grid = (int)std::min<long>(tiles, num_sms());
  auto run = [&](auto kern, size_t smem) -> bool {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return false;
    kern<<<grid, THREADS, smem, stream>>>(tmA, tmW, p);
    return true;
  };
  bool ok;
  switch (wide ? lps : 0) {
    case 1: ok = run(gemm_tree_kernel<128, 1>, Cfg<128>::SMEM); break;
    case 2: ok = run(gemm_tree_kernel<128, 2>, Cfg<128>::SMEM); break;
    case 4: ok = run(gemm_tree_kernel<128, 4>, Cfg<128>::SMEM); break;
    case 8: ok = run(gemm_tree_kernel<128, 8>, Cfg<128>::SMEM); break;
    case 16: ok = run(gemm_tree_kernel<128, 16>, Cfg<128>::SMEM); break;
    default: ok = run(gemm_tree_kernel<64, 0>, Cfg<64>::SMEM); break;
  }
  if (!ok) return BI_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

}  // namespace bi

// Workspace of bi_gemm_tree: the partials of the schedule it runs.  Every
// power-of-two cut of the leaves that divides their count is a cut into
// subtrees of the canonical tree, so the final C is the same bits whether
// the tree over a shard's leaves is folded in one partial or in several that
// a combine then adds; with up to 16 leaves per partial the kernel folds on
// its fast layout.  The size returned covers four partials at least, enough
// for K <= 16384 (64 leaves) at any shard count; with less, the call folds
// each shard's leaves in one partial (slower for 32 or 64 leaves a shard).
extern "C" size_t bi_gemm_tree_ws_bytes(int M, int N, int shards) {
  if (M < 0 || N < 0 || shards < 1) return 0;
  return sizeof(float) * (size_t)std::max(shards, 4) * M * N;
}

extern "C" bi_status bi_gemm_tree_partials(const void *A, const void *W, float *partials, int M, int N, int K,
                                           int shards, bi_stream_t stream) {
  bi_status st = bi::tree_check(A, W, M, N, K, shards);
  if (st != BI_OK) return st;
  if (M > 0 && (!partials || !bi_aligned16(partials))) return partials ? BI_ERR_UNSUPPORTED_SHAPE : BI_ERR_INVALID_ARG;
  if (M == 0) return BI_OK;
  return bi::tree_partials_launch(A, W, partials, M, N, K, shards, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" bi_status bi_gemm_tree(const void *A, const void *W, float *C, int M, int N, int K, int shards,
                                  void *ws, size_t ws_bytes, bi_stream_t stream) {
  bi_status st = bi::tree_check(A, W, M, N, K, shards);
  if (st != BI_OK) return st;
  if (M > 0 && !C) return BI_ERR_INVALID_ARG;
  if (M > 0 && !bi_aligned16(C)) return BI_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return BI_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // partials: the shards, cut further (power-of-two subtrees) until each
  // holds at most 16 leaves, when the workspace allows it
  const int L = K / bi::tg::LEAF;
  int P = shards;
  while (L / P > 16 && L % (2 * P) == 0 && 2 * P <= bi::tg::MAX_LEAVES) P *= 2;
  const size_t fast = sizeof(float) * (size_t)P * M * N;
  if (P > shards && (!ws || ws_bytes < fast || !bi_aligned16(ws))) P = shards;
  if (P == 1) return bi::tree_partials_launch(A, W, C, M, N, K, 1, s);
  const size_t need = sizeof(float) * (size_t)P * M * N;
  if (!ws || ws_bytes < need) return BI_ERR_WORKSPACE;
  if (!bi_aligned16(ws)) return BI_ERR_UNSUPPORTED_SHAPE;
  float *parts = static_cast<float *>(ws);
  st = bi::tree_partials_launch(A, W, parts, M, N, K, P, s);
  if (st != BI_OK) return st;
  return bi::tree_combine_launch(parts, C, P, (size_t)M * N, s);
}
