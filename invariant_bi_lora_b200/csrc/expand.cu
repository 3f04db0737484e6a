// expand.cu -- LoRA expand out (+)= bf16(y) . B^T, single or multi-adapter.
//
// "Reproducible LoRA Inference Through Deterministic Split-K Reduction"
// (Q&A): LoRA is two low-rank multiplications; the shrink reduces over the
// hidden size, the expand reduces over the rank r only.  With K = r (8..128)
// there is nothing to split: each output element is one tensor-core MMA
// chain over r, computed the same way whatever M is, so the expand is
// batch-invariant as it stands.  It is bound by the fp32 write of `out`
// (M x N x 4 bytes), so the kernel is shaped for stores.  A CTA owns 64 rows
// (one row tile of a segment) and kExpCB column blocks of 128: the tile's
// resolution, its token rows and each warp's y fragments are fetched once
// and reused for every block.  Each warp computes a 16 x 64 strip per
// block, stages it in shared memory (row stride 72 floats: the fragment
// writes are conflict-free per half-warp) and writes whole 256-byte row
// segments, two rows per store instruction.
#include "common.cuh"

namespace bi {

constexpr int kExpBM = 64;     // rows per CTA (4 MMA row tiles)
constexpr int kExpBN = 128;    // columns per block
constexpr int kExpCB = 4;      // column blocks per CTA
constexpr int kExpThreads = 256;

struct ExpandParams {
  const float *y;           // [M][r] fp32
  const uint16_t *bt;       // [n_ad][N][r] bf16
  const int32_t *perm;      // nullptr: identity
  const int32_t *offsets;   // [n_ad + 2] or nullptr
  float *out;               // [M][N] fp32
  int M, r, N, n_ad, accumulate;
};

// KS = number of k16 steps (r rounded up to 16, / 16).  The minimum-blocks
// bound lets six CTAs share an SM at r <= 16.
template <int KS>
__global__ void __launch_bounds__(kExpThreads, KS == 1 ? 6 : (KS == 2 ? 4 : 3))
expand_kernel(const __grid_constant__ ExpandParams p) {
  __shared__ TileInfo s_tile;
  __shared__ int32_t s_off[kMaxAdapters + 2];
  __shared__ int32_t s_rows[kExpBM];
  __shared__ __align__(16) float s_out[kExpThreads / 32][16][72];
  resolve_tile_block(p.offsets, p.n_ad, p.M, blockIdx.y, kExpBM, s_off, &s_tile);
  const TileInfo ti = s_tile;
  if (ti.adapter < 0) return;
  if ((int)threadIdx.x < ti.rows) s_rows[threadIdx.x] = tile_row(p.perm, ti, threadIdx.x);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int mt = warp & 3;                       // row tile 0..3
  const int lr0 = mt * 16 + g, lr1 = lr0 + 8;
  const bool v0 = lr0 < ti.rows, v1 = lr1 < ti.rows;
  const int row0 = v0 ? tile_row(p.perm, ti, lr0) : 0;
  const int row1 = v1 ? tile_row(p.perm, ti, lr1) : 0;
  __syncthreads();                               // s_rows
  const int half = lane >> 4, q4 = (lane & 15) * 4;
  float (*so)[72] = s_out[warp];

  if (ti.adapter == p.n_ad) {                    // tokens without an adapter
    if (!p.accumulate) {
      for (int cb = 0; cb < kExpCB; cb++) {
        const int n = (blockIdx.x * kExpCB + cb) * kExpBN + (warp >> 2) * 64 + q4;
        if (n >= p.N) break;
#pragma unroll 2
        for (int j = 0; j < 8; j++) {
          const int tr = mt * 16 + 2 * j + half;
          if (tr < ti.rows)
            __stcs(reinterpret_cast<float4 *>(p.out + (size_t)s_rows[tr] * p.N + n), make_float4(0.f, 0.f, 0.f, 0.f));
        }
      }
    }
    return;
  }

  // A fragments: bf16(y) rows g, g+8, k slots 2c, 2c+1, 2c+8, 2c+9 of each
  // k16 step (zero past r)
  uint32_t afr[KS][4];
#pragma unroll
  for (int s = 0; s < KS; s++) {
    const int k0 = 16 * s + 2 * c, k1 = k0 + 8;
    float2 a00 = make_float2(0.f, 0.f), a10 = a00, a01 = a00, a11 = a00;
    if (v0 && k0 < p.r) a00 = *reinterpret_cast<const float2 *>(p.y + (size_t)row0 * p.r + k0);
    if (v1 && k0 < p.r) a10 = *reinterpret_cast<const float2 *>(p.y + (size_t)row1 * p.r + k0);
    if (v0 && k1 < p.r) a01 = *reinterpret_cast<const float2 *>(p.y + (size_t)row0 * p.r + k1);
    if (v1 && k1 < p.r) a11 = *reinterpret_cast<const float2 *>(p.y + (size_t)row1 * p.r + k1);
    afr[s][0] = pack_bf16x2(a00.x, a00.y);
    afr[s][1] = pack_bf16x2(a10.x, a10.y);
    afr[s][2] = pack_bf16x2(a01.x, a01.y);
    afr[s][3] = pack_bf16x2(a11.x, a11.y);
  }

  const uint16_t *bad = p.bt + (size_t)ti.adapter * p.N * p.r;
  constexpr int NB = KS <= 2 ? 8 : (KS <= 4 ? 4 : 2);
#pragma unroll 1
  for (int cb = 0; cb < kExpCB; cb++) {
    const int nbase = (blockIdx.x * kExpCB + cb) * kExpBN + (warp >> 2) * 64;
    if (nbase >= p.N) break;                     // uniform in the warp
    // B fragments of NB n-tiles at a time (independent L2 loads in flight
    // together), then their MMAs
#pragma unroll 1
    for (int nb0 = 0; nb0 < 8; nb0 += NB) {
      uint32_t bfr[NB][KS][2];
#pragma unroll
      for (int i = 0; i < NB; i++) {
        const int n0 = nbase + (nb0 + i) * 8;
        const uint16_t *brow = bad + (size_t)(n0 + g) * p.r;   // B[n0+g][.]
        const bool ok = n0 < p.N;
#pragma unroll
        for (int s = 0; s < KS; s++) {
          const int k0 = 16 * s + 2 * c, k1 = k0 + 8;
          bfr[i][s][0] = ok && k0 < p.r ? __ldg(reinterpret_cast<const unsigned int *>(brow + k0)) : 0u;
          bfr[i][s][1] = ok && k1 < p.r ? __ldg(reinterpret_cast<const unsigned int *>(brow + k1)) : 0u;
        }
      }
#pragma unroll
      for (int i = 0; i < NB; i++) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int s = 0; s < KS; s++) mma_bf16_16816(acc, afr[s], bfr[i][s], acc);
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
      if (tr < ti.rows && n < p.N) {
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

bi_status expand_launch(const float *y, const void *B, const int32_t *perm, const int32_t *offsets,
                        int n_ad, float *out, int M, int r, int N, int accumulate,
                        cudaStream_t stream) {
  if (M < 0 || r <= 0 || N <= 0 || n_ad < 1) return BI_ERR_INVALID_ARG;
  if (M > 0 && (!y || !B || !out)) return BI_ERR_INVALID_ARG;
  if (r % 8 != 0 || r > 128 || N % 8 != 0) return BI_ERR_UNSUPPORTED_SHAPE;
  if (!bi_aligned16(y) || !bi_aligned16(B) || !bi_aligned16(out)) return BI_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return BI_OK;
  ExpandParams p{y, static_cast<const uint16_t *>(B), perm, offsets, out, M, r, N, n_ad,
                 accumulate ? 1 : 0};
  const int tiles = offsets ? (M + kExpBM - 1) / kExpBM + n_ad + 1 : (M + kExpBM - 1) / kExpBM;
  dim3 grid((N + kExpBN * kExpCB - 1) / (kExpBN * kExpCB), tiles);
  const int ks = (r + 15) / 16;
  switch (ks) {
    case 1: expand_kernel<1><<<grid, kExpThreads, 0, stream>>>(p); break;
    case 2: expand_kernel<2><<<grid, kExpThreads, 0, stream>>>(p); break;
    case 3: expand_kernel<3><<<grid, kExpThreads, 0, stream>>>(p); break;
    case 4: expand_kernel<4><<<grid, kExpThreads, 0, stream>>>(p); break;
    case 5: expand_kernel<5><<<grid, kExpThreads, 0, stream>>>(p); break;
    case 6: expand_kernel<6><<<grid, kExpThreads, 0, stream>>>(p); break;
    case 7: expand_kernel<7><<<grid, kExpThreads, 0, stream>>>(p); break;
    default: expand_kernel<8><<<grid, kExpThreads, 0, stream>>>(p); break;
  }
  return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

}  // namespace bi

extern "C" bi_status bi_lora_expand(const float *y, const void *B, float *out, int M, int r, int N,
                                    int accumulate, bi_stream_t stream) {
  return bi::expand_launch(y, B, nullptr, nullptr, 1, out, M, r, N, accumulate,
                           reinterpret_cast<cudaStream_t>(stream));
}

extern "C" bi_status bi_lora_expand_segmented(const float *y, const void *B, const void *plan,
                                              int n_adapters, float *out, int M, int r, int N,
                                              int accumulate, bi_stream_t stream) {
  if (M > 0 && !plan) return BI_ERR_INVALID_ARG;
  if (n_adapters < 1 || n_adapters > bi::kMaxAdapters) return BI_ERR_INVALID_ARG;
  const int32_t *perm = static_cast<const int32_t *>(plan);
  return bi::expand_launch(y, B, perm, perm + M, n_adapters, out, M, r, N, accumulate,
                           reinterpret_cast<cudaStream_t>(stream));
}
