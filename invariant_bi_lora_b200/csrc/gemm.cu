// gemm.cu -- batch-invariant bf16 GEMM on the 5th-generation tensor cores.
//
// "The biggest Mystery of LLMs have just been solved" (Batch-Variant vs.
// Batch-Invariant): a batch-invariant matmul uses a locked kernel policy
// instead of an auto-picker, so the reduction order never depends on the
// batch.  "Restoring AI Reproducibility" (3-2): matmul stays data-parallel,
// with one consistent reduction order.  "Batch Invariant Ops" (Highlighted
// Details): torch.mm.
//
// Locked policy: every call, whatever M is, steps K from 0 to K in 64-wide
// stages and accumulates each output element in one TMEM accumulator by
// tcgen05.mma (M=128, K=16, bf16 in, fp32 accumulate), never splitting K.
// The accumulation of one output element is the same whatever the MMA's N
// (tests compare N = 32, 64 and 256 bit for bit), so the output tile's
// width is free: 128 x 256 tiles from M = 513 on, and narrower 128 x 64 or
// 128 x 32 tiles below, so that a small-M call still spreads its weight read
// over the SMs (N = 4096: 128 or 256 CTAs instead of 16).  Row m of C is
// therefore the same bits for every M; rows past M are zero-filled by TMA
// and dropped.  addmm adds a bf16 bias to the fp32 accumulator after the
// last K stage: C = fl(acc + bias[n]), then the optional bf16 rounding.
//
// Pipeline (persistent, one CTA per SM, 192 threads):
//   warp 0      TMA producer: A and W tiles into a shared ring
//               (128-byte swizzle; 4 x 48 KB for 256-wide tiles, 8 stages
//               for the narrow ones)
//   warp 1      TMEM allocator and MMA issuer (one elected thread)
//   warps 2..5  epilogue: TMEM -> registers -> global (fp32 or bf16),
//               lane quadrant = warp % 4
// Two TMEM accumulators let the epilogue of tile i overlap the MMAs of
// tile i+1.  Every wait is bounded (tc.cuh).
#include "tc.cuh"

#include <cudaTypedefs.h>
#include <atomic>
#include <mutex>

namespace bi {

namespace gemm {
constexpr int BM = 128, BK = 64;
constexpr int THREADS = 192;
constexpr int A_BYTES = BM * BK * 2;                  // 16 KB
// Per output-tile width BN: the W stage, the ring depth, TMEM columns.
template <int BN>
struct Cfg {
  static constexpr int STAGES = BN >= 256 ? 4 : 8;   // with full 128-row A stages
  static constexpr int MAX_STAGES = BN == 32 ? 32 : STAGES;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr uint32_t TMEM_COLS = 2 * BN < 32 ? 32 : 2 * BN;   // two accumulators
};
// The ring of one launch.  At M <= 64 the A box holds only a_rows =
// round_up(M, 8) rows, so a stage is mostly W and the ring can be deep; the
// MMA still reads a 128-row A window from each stage's start, whose rows
// past a_rows fall on the next stages (or on the slack after the ring) and
// produce output rows that are never stored: a row of an MMA's result
// depends on that row of A only.
struct GemmRing {
  int stages;        // ring depth
  int a_rows;        // rows of the A box (128, or round_up(M, 8) at M <= 64)
  int a_stage;       // bytes between A stages (a_rows * 128)
  int b_off;         // bytes from the ring start to the W stages
  int tail_off;      // bytes from the ring start to the barriers
};
}  // namespace gemm

template <int STAGES>
struct GemmSmemTail {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;            // the MMA issuer's last commit, before TMEM is freed
  uint32_t tmem_base;
  uint32_t bail;
};

// Test-only fault (bi_debug_set_fault): the producer of CTA 0 leaves the
// first stage of its first tile unloaded, so the MMA issuer's wait on it
// runs out; waits then give up after wait_ns.
struct GemmDebug {
  int fault;
  unsigned long long wait_ns;
};

template <int BN>
__global__ void __launch_bounds__(gemm::THREADS, 1)
gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW,
                 void *__restrict__ C, const uint16_t *__restrict__ bias, int M, int N, int K, int c_bf16,
                 unsigned *status, GemmDebug dbg, gemm::GemmRing ring) {
  using namespace gemm;
  constexpr int MAXST = Cfg<BN>::MAX_STAGES, B_BYTES = Cfg<BN>::B_BYTES;
  constexpr uint32_t TMEM_COLS = Cfg<BN>::TMEM_COLS;
  const int STAGES = ring.stages;
  const int A_STAGE = ring.a_stage;
  const uint32_t STAGE_TX = (uint32_t)(ring.a_rows * BK * 2 + B_BYTES);
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sa = smem;                                 // [STAGES][A_STAGE] + slack
  uint8_t *sb = smem + ring.b_off;                    // [STAGES][B_BYTES]
  GemmSmemTail<MAXST> *tail = reinterpret_cast<GemmSmemTail<MAXST> *>(smem + ring.tail_off);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_m = (M + BM - 1) / BM, tiles_n = (N + BN - 1) / BN;
  const int num_tiles = tiles_m * tiles_n;
  const int kblocks = K / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; s++) {
      mbar_init(&tail->full[s], 1);
      mbar_init(&tail->empty[s], 1);
    }
    for (int b = 0; b < 2; b++) {
      mbar_init(&tail->tfull[b], 1);
      mbar_init(&tail->tempty[b], 4);
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

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_par = 0;             // per stage: loads in flight, and their phase
      for (int tile = blockIdx.x; tile < num_tiles && !*bail; tile += gridDim.x) {
        const int mb = tile % tiles_m, nb = tile / tiles_m;
        for (int kb = 0; kb < kblocks; kb++) {
          if (!mbar_wait_for(&tail->empty[stage], phase ^ 1, dbg.wait_ns)) {
            flag_error(status, BI_ERR_TIMEOUT);
            *bail = 1;
            break;
          }
          const bool skip = dbg.fault == BI_FAULT_SKIP_STAGE && blockIdx.x == 0 && tile == (int)blockIdx.x && kb == 0;
          if (!skip) {
            mbar_arrive_expect_tx(&tail->full[stage], STAGE_TX);
            tma_load_2d(&tmA, &tail->full[stage], sa + stage * A_STAGE, kb * BK, mb * BM);
            tma_load_2d(&tmW, &tail->full[stage], sb + stage * B_BYTES, kb * BK, nb * BN);
            issued |= 1u << stage;
            issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          } else {
            issued &= ~(1u << stage);
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // every load issued has landed before the CTA's shared memory is
      // given up (a stage the MMAs consumed passes at once)
      for (int s = 0; s < STAGES; s++)
        if ((issued >> s) & 1u)
          if (!mbar_wait_for(&tail->full[s], (issued_par >> s) & 1u, dbg.wait_ns)) flag_error(status, BI_ERR_TIMEOUT);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      constexpr uint32_t idesc = umma_idesc_bf16(BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int tile = blockIdx.x; tile < num_tiles && !*bail; tile += gridDim.x) {
        if (!mbar_wait_for(&tail->tempty[acc], acc_phase ^ 1, dbg.wait_ns)) {
          flag_error(status, BI_ERR_TIMEOUT);
          *bail = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(acc * BN);
        for (int kb = 0; kb < kblocks; kb++) {
          if (!mbar_wait_for(&tail->full[stage], phase, dbg.wait_ns)) {
            flag_error(status, BI_ERR_TIMEOUT);
            *bail = 1;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sa + stage * A_STAGE);
          const uint32_t b0 = smem_u32(sb + stage * B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; k++)
            umma_bf16(d, umma_desc_kmajor_sw128(a0 + 32 * k), umma_desc_kmajor_sw128(b0 + 32 * k), idesc,
                      (kb | k) != 0);
          umma_commit(&tail->empty[stage]);          // stage reusable once these MMAs finish
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        umma_commit(&tail->tfull[acc]);              // accumulator ready for the epilogue
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
      // every MMA issued has completed before TMEM is freed
      umma_commit(&tail->drain);
      if (!mbar_wait_for(&tail->drain, 0, dbg.wait_ns)) flag_error(status, BI_ERR_TIMEOUT);
    }
  } else {
    // ---------------- epilogue: 4 warps, one TMEM lane quadrant each
    const int quad = warp & 3;
    const int row_in_tile = 32 * quad + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      if (*bail) break;
      if (!mbar_wait_for(&tail->tfull[acc], acc_phase, dbg.wait_ns)) {
        flag_error(status, BI_ERR_TIMEOUT);
        *bail = 1;
        break;
      }
      tc_fence_after();
      const int mb = tile % tiles_m, nb = tile / tiles_m;
      const int row = mb * BM + row_in_tile;
      const uint32_t tbase = tmem + ((uint32_t)(32 * quad) << 16) + (uint32_t)(acc * BN);
#pragma unroll 1
      for (int ch = 0; ch < BN / 32; ch++) {
        uint32_t v[32];
        tmem_ld32(tbase + 32 * ch, v);
        tmem_wait_ld();
        const int col0 = nb * BN + 32 * ch;
        if (bias && row < M) {
          // addmm: one rounding, after the whole K reduction
#pragma unroll
          for (int j = 0; j < 4; j++) {
            const uint4 b = col0 + 8 * j < N ? __ldg(reinterpret_cast<const uint4 *>(bias + col0 + 8 * j))
                                             : make_uint4(0, 0, 0, 0);
            const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int e = 0; e < 4; e++) {
              v[8 * j + 2 * e] = __float_as_uint(__fadd_rn(__uint_as_float(v[8 * j + 2 * e]), bf16lo(bw[e])));
              v[8 * j + 2 * e + 1] = __float_as_uint(__fadd_rn(__uint_as_float(v[8 * j + 2 * e + 1]), bf16hi(bw[e])));
            }
          }
        }
        if (row < M) {
          if (!c_bf16) {
            float *dst = static_cast<float *>(C) + (size_t)row * N + col0;
#pragma unroll
            for (int j = 0; j < 8; j++)
              if (col0 + 4 * j < N)
                *reinterpret_cast<uint4 *>(dst + 4 * j) = make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
          } else {
            uint16_t *dst = static_cast<uint16_t *>(C) + (size_t)row * N + col0;
#pragma unroll
            for (int j = 0; j < 4; j++)
              if (col0 + 8 * j < N) {
                uint4 o;
                o.x = pack_bf16x2(__uint_as_float(v[8 * j + 0]), __uint_as_float(v[8 * j + 1]));
                o.y = pack_bf16x2(__uint_as_float(v[8 * j + 2]), __uint_as_float(v[8 * j + 3]));
                o.z = pack_bf16x2(__uint_as_float(v[8 * j + 4]), __uint_as_float(v[8 * j + 5]));
                o.w = pack_bf16x2(__uint_as_float(v[8 * j + 6]), __uint_as_float(v[8 * j + 7]));
                *reinterpret_cast<uint4 *>(dst + 8 * j) = o;
              }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tail->tempty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host

static std::mutex g_tma_mu;

bool make_tma_2d_bf16(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                      uint32_t box_outer) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_tma_mu);
    if (!encode) {
      void *fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn)
        return false;
      encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
  }
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

static std::atomic<int> g_fault{0};

template <int BN>
static bi_status gemm_run(const void *A, const void *W, void *C, const void *bias, int M, int N, int K, int c_bf16,
                          cudaStream_t stream) {
  using namespace gemm;
  GemmRing ring{};
  ring.a_rows = (BN == 32 && M <= 64) ? ((M + 7) & ~7) : BM;
  ring.a_stage = ring.a_rows * BK * 2;
  const int slack = (BM - ring.a_rows) * BK * 2;     // the last stage's 128-row window
  if (ring.a_rows < BM) {
    const int budget = 200 * 1024 - slack;
    ring.stages = std::min(Cfg<BN>::MAX_STAGES, budget / (ring.a_stage + Cfg<BN>::B_BYTES));
  } else {
    ring.stages = Cfg<BN>::STAGES;
  }
  ring.b_off = (ring.stages * ring.a_stage + slack + 1023) & ~1023;
  ring.tail_off = ring.b_off + ring.stages * Cfg<BN>::B_BYTES;
  const size_t SMEM = 1024 + (size_t)ring.tail_off + sizeof(GemmSmemTail<Cfg<BN>::MAX_STAGES>);
  CUtensorMap tmA, tmW;
  if (!make_tma_2d_bf16(&tmA, A, (uint64_t)K, (uint64_t)M, BK, (uint32_t)ring.a_rows)) return BI_ERR_CUDA;
  if (!make_tma_2d_bf16(&tmW, W, (uint64_t)K, (uint64_t)N, BK, BN)) return BI_ERR_CUDA;
  // per launch: the attribute belongs to the current device, and a process
  // may drive several
  if (cudaFuncSetAttribute(gemm_bf16_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM) !=
      cudaSuccess)
    return BI_ERR_CUDA;
  const long tiles = (long)((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  const int grid = (int)std::min<long>(tiles, num_sms());
  GemmDebug dbg{g_fault.load(), g_fault.load() ? 10000000ull : kWaitLimitNs};
  gemm_bf16_kernel<BN><<<grid, THREADS, SMEM, stream>>>(tmA, tmW, C, static_cast<const uint16_t *>(bias), M, N, K,
                                                       c_bf16 ? 1 : 0, status_word(), dbg, ring);
  return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

bi_status gemm_launch(const void *A, const void *W, void *C, const void *bias, int M, int N, int K, int c_bf16,
                      cudaStream_t stream) {
  using namespace gemm;
  if (M < 0 || N <= 0 || K <= 0) return BI_ERR_INVALID_ARG;
  if (M > 0 && (!A || !W || !C)) return BI_ERR_INVALID_ARG;
  if (K % BK != 0 || N % 16 != 0) return BI_ERR_UNSUPPORTED_SHAPE;
  if (!bi_aligned16(A) || !bi_aligned16(W) || !bi_aligned16(C) || !bi_aligned16(bias)) return BI_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return BI_OK;
  // the tile width only spreads the work (bit-neutral): narrow tiles when
  // few rows would leave most SMs idle
  if (M <= 128 && N % 32 == 0) return gemm_run<32>(A, W, C, bias, M, N, K, c_bf16, stream);
  if (M <= 512 && N % 64 == 0) return gemm_run<64>(A, W, C, bias, M, N, K, c_bf16, stream);
  return gemm_run<256>(A, W, C, bias, M, N, K, c_bf16, stream);
}

}  // namespace bi

extern "C" bi_status bi_gemm(const void *A, const void *W, void *C, int M, int N, int K, int c_bf16,
                             bi_stream_t stream) {
  return bi::gemm_launch(A, W, C, nullptr, M, N, K, c_bf16, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" bi_status bi_addmm(const void *bias, const void *A, const void *W, void *C, int M, int N, int K,
                              int c_bf16, bi_stream_t stream) {
  if (M > 0 && !bias) return BI_ERR_INVALID_ARG;
  return bi::gemm_launch(A, W, C, bias, M, N, K, c_bf16, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" void bi_debug_set_fault(int fault_code) { bi::g_fault.store(fault_code); }
