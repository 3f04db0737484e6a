// expand.cu -- LoRA expand out (+)= bf16(y) . B^T, single or multi-adapter.
//
// "Reproducible LoRA Inference Through Deterministic Split-K Reduction"
// (Q&A): LoRA is two low-rank multiplications; the shrink reduces over the
// hidden size, the expand reduces over the rank r only.  With K = r (8..128)
// there is nothing to split: each output element is one tensor-core MMA
// chain over r, computed the same way whatever M is, so the expand is
// batch-invariant as it stands.  It is bound by the fp32 write of `out`
// (M x N x 4 bytes), so the kernel is shaped for stores.  A CTA owns 64 rows
// (one record of the plan's tile table: adapter, rows and token ids in one
// read) and kExpCB column blocks of 128; each warp computes a 16 x 64 strip
// per block, stages it in shared memory (row stride 72 floats: the fragment
// writes are conflict-free per half-warp) and writes whole 256-byte row
// segments, two rows per store instruction.  B fragments, two ways (the
// same values, the same MMAs):
//   r <= 32: from L2 into registers, the y fragments and the first block's
//     B requested together and, at r <= 16, each block's stores going out
//     while the next block's B is in flight; four CTAs per SM, so a
//     4096 x 4096 call is one wave;
//   r > 32: the CTA's slice of B (512 columns x r) copied once into shared
//     memory by 16-byte cp.async, in parallel with the y loads, and read by
//     ldmatrix (rows padded by 16 bytes: the eight rows of a matrix fall in
//     different bank groups), instead of 8 * r / 4 scattered 4-byte L2 loads
//     per thread and block.
#include "common.cuh"
#include "tc.cuh"

namespace bi {

constexpr int kExpBM = 64;     // rows per CTA (4 MMA row tiles): one plan record
constexpr int kExpBN = 128;    // columns per block
constexpr int kExpCB = 4;      // column blocks per CTA
constexpr int kExpThreads = 256;

struct ExpandParams {
  const float *y;           // [M][r] fp32
  const uint16_t *bt;       // [n_ad][N][r] bf16
  const int32_t *table;     // plan tile table (nullptr: rows in index order, adapter 0)
  float *out;               // [M][N] fp32
  int M, r, N, n_ad, accumulate;
};

// B fragments of NBL of the warp's eight n-tiles (i0 .. i0+NBL-1) of the
// column block at nbase: for n-tile i, column n0 + g, k slots 2c, 2c+1 and
// 2c+8, 2c+9 of each k16 step (zero past r and past N).
template <int KS, int NBL>
BI_DEV void expand_load_b(const ExpandParams &p, const uint16_t *bad, int nbase, int i0, int g, int c,
                          uint32_t (&bfr)[NBL][KS][2]) {
#pragma unroll
  for (int i = 0; i < NBL; i++) {
    const int n0 = nbase + (i0 + i) * 8;
    const uint16_t *brow = bad + (size_t)(n0 + g) * p.r;
    const bool ok = n0 < p.N;
#pragma unroll
    for (int s = 0; s < KS; s++) {
      const int k0 = 16 * s + 2 * c, k1 = k0 + 8;
      bfr[i][s][0] = ok && k0 < p.r ? __ldg(reinterpret_cast<const unsigned int *>(brow + k0)) : 0u;
      bfr[i][s][1] = ok && k1 < p.r ? __ldg(reinterpret_cast<const unsigned int *>(brow + k1)) : 0u;
    }
  }
}

// Two n-tiles' B fragments for one k16 step from the staged slice: lane t
// points at row t % 8 of matrix t / 8 = (n-tile i + (t/8)/2, k half (t/8)%2).
BI_DEV void expand_ldsm_b(uint32_t base, int bstride, int n0, int kbyte, int lane, uint32_t (&b)[4]) {
  const int j = lane >> 3;
  const uint32_t addr = base + (uint32_t)((n0 + (j >> 1) * 8 + (lane & 7)) * bstride + kbyte + (j & 1) * 16);
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(b[0]), "=r"(b[1]), "=r"(b[2]), "=r"(b[3])
               : "r"(addr));
}

// KS = number of k16 steps (r rounded up to 16, / 16).  The register-B
// form (r <= 32): at r <= 16 the next block's B fragments are prefetched
// (PF); the minimum-blocks bound keeps four CTAs per SM.
template <int KS>
__global__ void __launch_bounds__(kExpThreads, KS == 1 ? 4 : (KS == 2 ? 4 : 3))
expand_kernel(const __grid_constant__ ExpandParams p) {
  __shared__ int32_t s_rows[kExpBM];
  __shared__ int s_info[2];
  __shared__ __align__(16) float s_out[kExpThreads / 32][16][72];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;

  // ---- the tile: one read of its table record
  if (warp == 0) {
    int adapter, rows;
    if (p.table) {
      const int32_t *R = p.table + (size_t)blockIdx.y * kPlanRec;
      const int4 h = *reinterpret_cast<const int4 *>(R);
      const int4 id4 = *reinterpret_cast<const int4 *>(R + 4 + 4 * (lane & 15));
      adapter = h.x;
      rows = h.y;
      if (lane < 16) {
        const int idv[4] = {id4.x, id4.y, id4.z, id4.w};
#pragma unroll
        for (int e = 0; e < 4; e++) s_rows[4 * lane + e] = idv[e];
      }
    } else {
      const int row0 = blockIdx.y * kExpBM;
      rows = min(kExpBM, p.M - row0);
      adapter = rows > 0 ? 0 : -1;
      for (int i = lane; i < kExpBM; i += 32) s_rows[i] = row0 + i;
    }
    if (lane == 0) s_info[0] = adapter, s_info[1] = max(rows, 0);
  }
  __syncthreads();
  const int adapter = s_info[0], rows = s_info[1];
  if (adapter < 0) return;

  const int mt = warp & 3;                       // row tile 0..3
  const int lr0 = mt * 16 + g, lr1 = lr0 + 8;
  const bool v0 = lr0 < rows, v1 = lr1 < rows;
  const int row0 = v0 ? s_rows[lr0] : 0;
  const int row1 = v1 ? s_rows[lr1] : 0;
  const int half = lane >> 4, q4 = (lane & 15) * 4;
  float (*so)[72] = s_out[warp];
  const int nfirst = blockIdx.x * kExpCB * kExpBN + (warp >> 2) * 64;

  if (adapter == p.n_ad) {                       // tokens without an adapter
    if (!p.accumulate) {
      for (int cb = 0; cb < kExpCB; cb++) {
        const int n = nfirst + cb * kExpBN + q4;
        if (n >= p.N) break;
#pragma unroll 2
        for (int j = 0; j < 8; j++) {
          const int tr = mt * 16 + 2 * j + half;
          if (tr < rows)
            __stcs(reinterpret_cast<float4 *>(p.out + (size_t)s_rows[tr] * p.N + n), make_float4(0.f, 0.f, 0.f, 0.f));
        }
      }
    }
    return;
  }

  // y fragments (bf16(y) rows g, g+8, k slots 2c, 2c+1, 2c+8, 2c+9 of each
  // k16 step, zero past r) and block 0's B fragments, requested together
  const uint16_t *bad = p.bt + (size_t)adapter * p.N * p.r;
  float2 yv[KS][4];
#pragma unroll
  for (int s = 0; s < KS; s++) {
    const int k0 = 16 * s + 2 * c, k1 = k0 + 8;
    const float2 z = make_float2(0.f, 0.f);
    yv[s][0] = v0 && k0 < p.r ? *reinterpret_cast<const float2 *>(p.y + (size_t)row0 * p.r + k0) : z;
    yv[s][1] = v1 && k0 < p.r ? *reinterpret_cast<const float2 *>(p.y + (size_t)row1 * p.r + k0) : z;
    yv[s][2] = v0 && k1 < p.r ? *reinterpret_cast<const float2 *>(p.y + (size_t)row0 * p.r + k1) : z;
    yv[s][3] = v1 && k1 < p.r ? *reinterpret_cast<const float2 *>(p.y + (size_t)row1 * p.r + k1) : z;
  }
  constexpr bool PF = KS == 1;
  constexpr int NB = PF ? 8 : (KS <= 2 ? 8 : (KS <= 4 ? 4 : 2));
  uint32_t bcur[NB][KS][2], bnext[PF ? 8 : 1][KS][2];
  if (PF && nfirst < p.N) expand_load_b<KS, NB>(p, bad, nfirst, 0, g, c, bcur);
  uint32_t afr[KS][4];
#pragma unroll
  for (int s = 0; s < KS; s++)
#pragma unroll
    for (int q = 0; q < 4; q++) afr[s][q] = pack_bf16x2(yv[s][q].x, yv[s][q].y);

#pragma unroll 1
  for (int cb = 0; cb < kExpCB; cb++) {
    const int nbase = nfirst + cb * kExpBN;
    if (nbase >= p.N) break;                     // uniform in the warp
    if (PF && cb + 1 < kExpCB && nbase + kExpBN < p.N)
      expand_load_b<KS, NB>(p, bad, nbase + kExpBN, 0, g, c,
                            reinterpret_cast<uint32_t (&)[NB][KS][2]>(bnext));
#pragma unroll 1
    for (int nb0 = 0; nb0 < 8; nb0 += NB) {
      if (!PF) expand_load_b<KS, NB>(p, bad, nbase, nb0, g, c, bcur);
#pragma unroll
      for (int i = 0; i < NB; i++) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int s = 0; s < KS; s++) mma_bf16_16816(acc, afr[s], bcur[i][s], acc);
        const int col = (nb0 + i) * 8 + 2 * c;
        *reinterpret_cast<float2 *>(&so[g][col]) = make_float2(acc[0], acc[1]);
        *reinterpret_cast<float2 *>(&so[g + 8][col]) = make_float2(acc[2], acc[3]);
      }
    }
    __syncwarp();
    // rows 2j and 2j+1 of the strip per step: lanes 0-15 one row, 16-31 the other
    const int n = nbase + q4;
#pragma unroll 2
    for (int j = 0; j < 8; j++) {
      const int lr = 2 * j + half;               // row inside the warp's strip
      const int tr = mt * 16 + lr;               // row inside the tile
      if (tr < rows && n < p.N) {
        float4 v = *reinterpret_cast<const float4 *>(&so[lr][q4]);
        float4 *o = reinterpret_cast<float4 *>(p.out + (size_t)s_rows[tr] * p.N + n);
        if (p.accumulate) {
          const float4 q = *o;
          v.x = __fadd_rn(q.x, v.x);
          v.y = __fadd_rn(q.y, v.y);
          v.z = __fadd_rn(q.z, v.z);
          v.w = __fadd_rn(q.w, v.w);
        }
        __stcs(o, v);
      }
    }
    __syncwarp();                                // the strip buffer is reused
    if (PF)
#pragma unroll
      for (int i = 0; i < NB; i++)
#pragma unroll
        for (int s = 0; s < KS; s++) bcur[i][s][0] = bnext[PF ? i : 0][s][0], bcur[i][s][1] = bnext[PF ? i : 0][s][1];
  }
}

// The staged-B form (r > 32).  Dynamic shared memory: the B slice,
// kExpCB * kExpBN rows of 2r + 16 bytes.
template <int KS>
__global__ void __launch_bounds__(kExpThreads)
expand_sb_kernel(const __grid_constant__ ExpandParams p) {
  extern __shared__ __align__(128) uint8_t exp_smem[];
  __shared__ int32_t s_rows[kExpBM];
  __shared__ int s_info[2];
  __shared__ __align__(16) float s_out[kExpThreads / 32][16][72];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;

  // ---- the tile: one read of its table record
  if (warp == 0) {
    int adapter, rows;
    if (p.table) {
      const int32_t *R = p.table + (size_t)blockIdx.y * kPlanRec;
      const int4 h = *reinterpret_cast<const int4 *>(R);
      const int4 id4 = *reinterpret_cast<const int4 *>(R + 4 + 4 * (lane & 15));
      adapter = h.x;
      rows = h.y;
      if (lane < 16) {
        const int idv[4] = {id4.x, id4.y, id4.z, id4.w};
#pragma unroll
        for (int e = 0; e < 4; e++) s_rows[4 * lane + e] = idv[e];
      }
    } else {
      const int row0 = blockIdx.y * kExpBM;
      rows = min(kExpBM, p.M - row0);
      adapter = rows > 0 ? 0 : -1;
      for (int i = lane; i < kExpBM; i += 32) s_rows[i] = row0 + i;
    }
    if (lane == 0) s_info[0] = adapter, s_info[1] = max(rows, 0);
  }
  __syncthreads();
  const int adapter = s_info[0], rows = s_info[1];
  if (adapter < 0) return;

  const int mt = warp & 3;                       // row tile 0..3
  const int lr0 = mt * 16 + g, lr1 = lr0 + 8;
  const bool v0 = lr0 < rows, v1 = lr1 < rows;
  const int row0 = v0 ? s_rows[lr0] : 0;
  const int row1 = v1 ? s_rows[lr1] : 0;
  const int half = lane >> 4, q4 = (lane & 15) * 4;
  float (*so)[72] = s_out[warp];
  const int ncol0 = blockIdx.x * kExpCB * kExpBN;

  if (adapter == p.n_ad) {                       // tokens without an adapter
    if (!p.accumulate) {
      for (int cb = 0; cb < kExpCB; cb++) {
        const int n = ncol0 + cb * kExpBN + (warp >> 2) * 64 + q4;
        if (n >= p.N) break;
#pragma unroll 2
        for (int j = 0; j < 8; j++) {
          const int tr = mt * 16 + 2 * j + half;
          if (tr < rows)
            __stcs(reinterpret_cast<float4 *>(p.out + (size_t)s_rows[tr] * p.N + n), make_float4(0.f, 0.f, 0.f, 0.f));
        }
      }
    }
    return;
  }

  // ---- B slice -> shared memory (16-byte pieces, all in flight), and the
  // y fragments: bf16(y) rows g, g+8, k slots 2c, 2c+1, 2c+8, 2c+9 of each
  // k16 step, zero past r
  const int bstride = 2 * p.r + 16;
  const int ncols = min(kExpCB * kExpBN, p.N - ncol0);
  const int cpr = p.r / 8;                       // 16-byte pieces per B row
  const uint8_t *bsrc = reinterpret_cast<const uint8_t *>(p.bt + ((size_t)adapter * p.N + ncol0) * p.r);
  for (int i = threadIdx.x; i < ncols * cpr; i += kExpThreads) {
    const int n = i / cpr, k = i - n * cpr;
    cp_async16(exp_smem + n * bstride + 16 * k, bsrc + (size_t)i * 16);
  }
  cp_async_commit();
  if (p.r % 16 != 0)                             // the last k16 step's upper half reads the pad: zeros
    for (int n = threadIdx.x; n < kExpCB * kExpBN; n += kExpThreads)
      *reinterpret_cast<uint4 *>(exp_smem + n * bstride + 2 * p.r) = make_uint4(0, 0, 0, 0);
  float2 yv[KS][4];
#pragma unroll
  for (int s = 0; s < KS; s++) {
    const int k0 = 16 * s + 2 * c, k1 = k0 + 8;
    const float2 z = make_float2(0.f, 0.f);
    yv[s][0] = v0 && k0 < p.r ? *reinterpret_cast<const float2 *>(p.y + (size_t)row0 * p.r + k0) : z;
    yv[s][1] = v1 && k0 < p.r ? *reinterpret_cast<const float2 *>(p.y + (size_t)row1 * p.r + k0) : z;
    yv[s][2] = v0 && k1 < p.r ? *reinterpret_cast<const float2 *>(p.y + (size_t)row0 * p.r + k1) : z;
    yv[s][3] = v1 && k1 < p.r ? *reinterpret_cast<const float2 *>(p.y + (size_t)row1 * p.r + k1) : z;
  }
  uint32_t afr[KS][4];
#pragma unroll
  for (int s = 0; s < KS; s++)
#pragma unroll
    for (int q = 0; q < 4; q++) afr[s][q] = pack_bf16x2(yv[s][q].x, yv[s][q].y);
  cp_async_wait<0>();
  __syncthreads();

  const uint32_t bbase = smem_u32(exp_smem);
#pragma unroll 1
  for (int cb = 0; cb < kExpCB; cb++) {
    const int nloc = cb * kExpBN + (warp >> 2) * 64;   // first column of the strip, in the slice
    if (ncol0 + nloc >= p.N) break;              // uniform in the warp
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      uint32_t bfr[KS][4];
#pragma unroll
      for (int s = 0; s < KS; s++) expand_ldsm_b(bbase, bstride, nloc + i * 8, 32 * s, lane, bfr[s]);
#pragma unroll
      for (int u = 0; u < 2; u++) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int s = 0; s < KS; s++) {
          const uint32_t bb[2] = {bfr[s][2 * u], bfr[s][2 * u + 1]};
          mma_bf16_16816(acc, afr[s], bb, acc);
        }
        const int col = (i + u) * 8 + 2 * c;
        *reinterpret_cast<float2 *>(&so[g][col]) = make_float2(acc[0], acc[1]);
        *reinterpret_cast<float2 *>(&so[g + 8][col]) = make_float2(acc[2], acc[3]);
      }
    }
    __syncwarp();
    // rows 2j and 2j+1 of the strip per step: lanes 0-15 one row, 16-31 the other
    const int n = ncol0 + nloc + q4;
#pragma unroll 2
    for (int j = 0; j < 8; j++) {
      const int lr = 2 * j + half;               // row inside the warp's strip
      const int tr = mt * 16 + lr;               // row inside the tile
      if (tr < rows && n < p.N) {
        float4 v = *reinterpret_cast<const float4 *>(&so[lr][q4]);
        float4 *o = reinterpret_cast<float4 *>(p.out + (size_t)s_rows[tr] * p.N + n);
        if (p.accumulate) {
          const float4 q = *o;
          v.x = __fadd_rn(q.x, v.x);
          v.y = __fadd_rn(q.y, v.y);
          v.z = __fadd_rn(q.z, v.z);
          v.w = __fadd_rn(q.w, v.w);
        }
        __stcs(o, v);
      }
    }
    __syncwarp();                                // the strip buffer is reused
  }
}

bi_status expand_launch(const float *y, const void *B, const int32_t *table, int n_ad, float *out, int M,
                        int r, int N, int accumulate, cudaStream_t stream) {
  if (M < 0 || r <= 0 || N <= 0 || n_ad < 1) return BI_ERR_INVALID_ARG;
  if (M > 0 && (!y || !B || !out)) return BI_ERR_INVALID_ARG;
  if (r % 8 != 0 || r > 128 || N % 8 != 0) return BI_ERR_UNSUPPORTED_SHAPE;
  if (!bi_aligned16(y) || !bi_aligned16(B) || !bi_aligned16(out)) return BI_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return BI_OK;
  ExpandParams p{y, static_cast<const uint16_t *>(B), table, out, M, r, N, n_ad, accumulate ? 1 : 0};
  const int tiles = table ? (int)plan_tiles(M, n_ad) : (M + kExpBM - 1) / kExpBM;
  dim3 grid((N + kExpBN * kExpCB - 1) / (kExpBN * kExpCB), tiles);
  const int ks = (r + 15) / 16;
  if (ks <= 2) {
    if (ks == 1) expand_kernel<1><<<grid, kExpThreads, 0, stream>>>(p);
    else expand_kernel<2><<<grid, kExpThreads, 0, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
  }
  const size_t smem = (size_t)kExpCB * kExpBN * (2 * r + 16);
  cudaError_t err = cudaSuccess;
  auto launch = [&](void (*kern)(ExpandParams)) {
    // the static strip buffers count against the default 48 KB as well
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return;
    kern<<<grid, kExpThreads, smem, stream>>>(p);
    err = cudaGetLastError();
  };
  switch (ks) {
    case 3: launch(expand_sb_kernel<3>); break;
    case 4: launch(expand_sb_kernel<4>); break;
    case 5: launch(expand_sb_kernel<5>); break;
    case 6: launch(expand_sb_kernel<6>); break;
    case 7: launch(expand_sb_kernel<7>); break;
    default: launch(expand_sb_kernel<8>); break;
  }
  return err == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

}  // namespace bi

extern "C" bi_status bi_lora_expand(const float *y, const void *B, float *out, int M, int r, int N,
                                    int accumulate, bi_stream_t stream) {
  return bi::expand_launch(y, B, nullptr, 1, out, M, r, N, accumulate, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" bi_status bi_lora_expand_segmented(const float *y, const void *B, const void *plan,
                                              int n_adapters, float *out, int M, int r, int N,
                                              int accumulate, bi_stream_t stream) {
  if (M > 0 && !plan) return BI_ERR_INVALID_ARG;
  if (n_adapters < 1 || n_adapters > bi::kMaxAdapters) return BI_ERR_INVALID_ARG;
  if (M > 0 && !bi_aligned16(plan)) return BI_ERR_UNSUPPORTED_SHAPE;
  const int32_t *table = static_cast<const int32_t *>(plan) + bi::plan_table_word(M, n_adapters);
  return bi::expand_launch(y, B, table, n_adapters, out, M, r, N, accumulate,
                           reinterpret_cast<cudaStream_t>(stream));
}
