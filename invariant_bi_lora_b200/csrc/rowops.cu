// rowops.cu -- batch-invariant RMSNorm, log_softmax and mean.
//
// "Restoring AI Reproducibility" (2-3, 3-1): RMSNorm contains a reduction,
// and stays batch-invariant when each batch element is reduced by its own
// core in a consistent order.  "Batch Invariant Ops" (Highlighted Details):
// log_softmax and mean are among the ops made batch-invariant.
//
// One CTA (or one thread-block cluster) per row; the work of a row never
// depends on how many rows the launch has.  The row sum is the canonical
// lane sum: T logical lanes, lane t chains (from +0, in order) the V
// elements of vectors t, t+T, t+2T, ..., and the T lane values are combined
// by the canonical tree -- inside a warp by the xor butterfly 1,2,4,8,16
// (which is that tree), across warps and CTAs by perfect trees over
// power-of-two counts.  Vectors are 16 bytes: V = 8 for bf16, V = 4 for fp32.
#include "bimath.cuh"
#include "tc.cuh"

#include <cooperative_groups.h>
#include <algorithm>

namespace cg = cooperative_groups;

namespace bi {

// ======================================================================
// RMSNorm: T = 512 lanes of V = 8 bf16.  One CTA of THREADS threads per
// row; thread u owns the LPT = 512/THREADS lanes u + THREADS*s (slot s), so
// each load or store instruction of a warp covers 32 consecutive vectors
// (512 contiguous bytes).  Slot s of all threads is the lane block
// [THREADS*s, THREADS*(s+1)), a subtree of the lane tree: a warp's 32 lanes
// of a slot are added by the xor butterfly, and the 16 (slot, warp) values
// -- in lane order -- by a perfect tree that every warp evaluates itself.
// The row stays in registers (VPL vectors per lane) between the sum and the
// scaling, so x is read from HBM once.
// ======================================================================
constexpr int kNormT = 512;

template <int THREADS, int VPL>
__global__ void __launch_bounds__(THREADS)
rmsnorm_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ w,
               uint16_t *__restrict__ y, int n, float eps) {
  constexpr int LPT = kNormT / THREADS;
  constexpr int NW = THREADS / 32;
  static_assert(LPT * NW == kNormT / 32, "16 (slot, warp) groups");
  __shared__ float s_grp[kNormT / 32];          // index s * NW + warp
  const int u = threadIdx.x;
  const int lane = u & 31, warp = u >> 5;
  const size_t row = blockIdx.x;
  const int nvec = n / 8;
  const uint16_t *xr = x + row * n;
  auto vidx = [&](int j, int sl) { return j * kNormT + sl * THREADS + u; };

  uint4 v[VPL][LPT];
  // small rows: w is fetched with x, so the scaling pass does not wait on
  // a second memory round trip after the reduction
  constexpr bool PREW = VPL <= 2;
  uint4 wv_pre[PREW ? VPL : 1][LPT];
  float p[LPT];
#pragma unroll
  for (int l = 0; l < LPT; l++) p[l] = 0.0f;
#pragma unroll
  for (int j = 0; j < VPL; j++)
#pragma unroll
    for (int l = 0; l < LPT; l++) {
      const int vi = vidx(j, l);
      v[j][l] = vi < nvec ? ldg128_stream(xr + 8 * vi) : make_uint4(0, 0, 0, 0);
      if constexpr (PREW) wv_pre[j][l] = vi < nvec ? ldg128(w + 8 * vi) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
  for (int j = 0; j < VPL; j++)
#pragma unroll
    for (int l = 0; l < LPT; l++) {
      if (vidx(j, l) < nvec) {
        const uint32_t q[4] = {v[j][l].x, v[j][l].y, v[j][l].z, v[j][l].w};
#pragma unroll
        for (int e = 0; e < 4; e++) {
          const float a = bf16lo(q[e]), b = bf16hi(q[e]);
          p[l] = __fadd_rn(p[l], __fmul_rn(a, a));
          p[l] = __fadd_rn(p[l], __fmul_rn(b, b));
        }
      }
    }
  // each slot: the warp's 32 lanes by the butterfly
#pragma unroll
  for (int l = 0; l < LPT; l++) {
    const float sv = warp_tree_sum(p[l]);
    if (lane == 0) s_grp[l * NW + warp] = sv;
  }
  __syncthreads();
  // the 16 group values in lane order, perfect tree on lanes 0..15
  float q = lane < kNormT / 32 ? s_grp[lane] : 0.0f;
#pragma unroll
  for (int o = 1; o < kNormT / 32; o <<= 1) q = __fadd_rn(q, __shfl_xor_sync(0xffffffffu, q, o));
  q = __shfl_sync(0xffffffffu, q, 0);
  const float inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(q, (float)n), eps)));
  uint16_t *yr = y + row * n;
#pragma unroll
  for (int j = 0; j < VPL; j++)
#pragma unroll
    for (int l = 0; l < LPT; l++) {
      const int vi = vidx(j, l);
      if (vi < nvec) {
        uint4 wv;
        if constexpr (PREW) wv = wv_pre[PREW ? j : 0][l];
        else wv = ldg128(w + 8 * vi);
        const uint32_t q4[4] = {v[j][l].x, v[j][l].y, v[j][l].z, v[j][l].w};
        const uint32_t wq[4] = {wv.x, wv.y, wv.z, wv.w};
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; e++) {
          const float lo = __fmul_rn(__fmul_rn(bf16lo(q4[e]), inv), bf16lo(wq[e]));
          const float hi = __fmul_rn(__fmul_rn(bf16hi(q4[e]), inv), bf16hi(wq[e]));
          o[e] = pack_bf16x2(lo, hi);
        }
        *reinterpret_cast<uint4 *>(yr + 8 * vi) = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
}

// ======================================================================
// mean: T = 1024 lanes of V = 4 fp32.  One CTA of 256 threads per row;
// thread u owns the four lanes u + 256*s (slot s), so each load of a warp
// covers 512 contiguous bytes.  Slot s is the lane block [256s, 256s+256),
// a subtree: a warp's 32 lanes of a slot by the xor butterfly, then the 32
// (slot, warp) values in lane order by a perfect tree in one warp.
// ======================================================================
constexpr int kLaneT = 1024;
constexpr int kMeanClusterRows = 128;        // up to this many rows: mean_cluster_kernel (measured crossover)
constexpr int kMeanThreads = 256;

__global__ void __launch_bounds__(kMeanThreads)
mean_kernel(const float *__restrict__ x, float *__restrict__ out, int n) {
  constexpr int NW = kMeanThreads / 32;
  __shared__ float s_grp[kLaneT / 32];           // index s * NW + warp
  const int u = threadIdx.x;
  const int lane = u & 31, warp = u >> 5;
  const size_t row = blockIdx.x;
  const int nvec = n / 4;
  const float4 *xr = reinterpret_cast<const float4 *>(x + row * n);
  float p[4] = {0.f, 0.f, 0.f, 0.f};
  for (int base = 0; base < nvec; base += kLaneT) {
    float4 v[4];
#pragma unroll
    for (int s = 0; s < 4; s++) {
      const int vi = base + s * kMeanThreads + u;
      v[s] = vi < nvec ? __ldcs(xr + vi) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int s = 0; s < 4; s++) {
      if (base + s * kMeanThreads + u < nvec) {
        p[s] = __fadd_rn(p[s], v[s].x);
        p[s] = __fadd_rn(p[s], v[s].y);
        p[s] = __fadd_rn(p[s], v[s].z);
        p[s] = __fadd_rn(p[s], v[s].w);
      }
    }
  }
#pragma unroll
  for (int s = 0; s < 4; s++) {
    const float sv = warp_tree_sum(p[s]);
    if (lane == 0) s_grp[s * NW + warp] = sv;
  }
  __syncthreads();
  if (u < 32) {
    const float q = warp_tree_sum(s_grp[lane]);
    if (u == 0) out[row] = __fdiv_rn(q, (float)n);
  }
}

// Few rows: one cluster of C CTAs per row, CTA q owning the contiguous lanes
// [q * 1024/C, (q+1) * 1024/C) -- a subtree of the 1024-lane tree, so the
// bits are mean_kernel's.  Each CTA folds its lanes' chains (eight vector
// loads in flight per lane) and its 32-lane groups, and pushes its value
// into slot q of rank 0 by st.async; rank 0 adds the C values by the top
// levels of the tree.  No CTA waits for another's threads.
template <int C>
__global__ void __launch_bounds__(kLaneT / C)
mean_cluster_kernel(const float *__restrict__ x, float *__restrict__ out, int n, unsigned *status) {
  constexpr int T = kLaneT / C, NW = T / 32;
  __shared__ float s_w[NW];
  __shared__ float s_c[C];
  __shared__ __align__(8) uint64_t s_bar;
  cg::cluster_group cluster = cg::this_cluster();
  const int q = (int)cluster.block_rank();
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const size_t row = blockIdx.x / C;
  const int nvec = n / 4;
  if (q == 0 && t == 0) {
    mbar_init(&s_bar, 1);
    mbar_fence_init();
    mbar_arrive_expect_tx(&s_bar, 4u * C);
  }
  // every CTA has started (and rank 0 initialised its barrier) once this
  // arrive is matched; the wait comes before the push
  cluster_arrive_relaxed();
  const float4 *xr = reinterpret_cast<const float4 *>(x + row * n);
  float p = 0.0f;
  int vi = q * T + t;                              // this lane's vectors: vi, vi + 1024, ...
  for (; vi + 7 * kLaneT < nvec; vi += 8 * kLaneT) {
    float4 v[8];
#pragma unroll
    for (int k = 0; k < 8; k++) v[k] = __ldcs(xr + vi + k * kLaneT);
#pragma unroll
    for (int k = 0; k < 8; k++) {
      p = __fadd_rn(p, v[k].x);
      p = __fadd_rn(p, v[k].y);
      p = __fadd_rn(p, v[k].z);
      p = __fadd_rn(p, v[k].w);
    }
  }
  for (; vi < nvec; vi += kLaneT) {
    const float4 v = __ldcs(xr + vi);
    p = __fadd_rn(p, v.x);
    p = __fadd_rn(p, v.y);
    p = __fadd_rn(p, v.z);
    p = __fadd_rn(p, v.w);
  }
  const float g = warp_tree_sum(p);                // one 32-lane group
  if (lane == 0) s_w[warp] = g;
  __syncthreads();
  float cv = 0.0f;                                 // the CTA's groups, perfect tree
  if (warp == 0) {
    cv = lane < NW ? s_w[lane] : 0.0f;
#pragma unroll
    for (int o = 1; o < NW; o <<= 1) cv = __fadd_rn(cv, __shfl_xor_sync(0xffffffffu, cv, o));
  }
  cluster_wait();
  if (t == 0) st_async_f32(&s_c[q], &s_bar, 0u, cv);
  if (q != 0 || warp != 0) return;
  if (!mbar_wait_cluster(&s_bar, 0)) flag_error(status, BI_ERR_TIMEOUT);
  float v = lane < C ? s_c[lane] : 0.0f;           // the top levels over the C CTAs
#pragma unroll
  for (int o = 1; o < C; o <<= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (lane == 0) out[row] = __fdiv_rn(v, (float)n);
}

// ======================================================================
// log_softmax: T = 4096 lanes of V = 4 fp32, two passes over the row
// (max; then the canonical sum of bi_exp(x - max)), then the write.  The
// row is held on chip between the passes so HBM sees one read and one
// write: a cluster of C CTAs shares the row, CTA q owning lanes
// [q*4096/C, (q+1)*4096/C) -- a subtree of the lane tree -- one thread per
// lane, each keeping its lane's vectors in shared memory (slot [j][tau] for
// vector 4096*j + lane).  Maxima and sums meet through distributed shared
// memory: each CTA pushes its value into a slot of every CTA of the cluster
// before a barrier, so after it every CTA reads only its own shared memory
// and no CTA waits for its peers at exit.  The sum pass stores d = x - max
// back into the slot, so the write pass is one subtraction per element.
// ======================================================================
constexpr int kLsmT = 4096;

struct LsmParams {
  const float *x;
  float *out;
  unsigned *status;
  int n;
  int C;      // CTAs per row (cluster size), power of two, 4..16
  int J;      // vector slots per lane = ceil(n/4 / 4096)
};

// bi_exp of the four lanes of d; the packed path when all four lie in
// bi_exp_fast's range (d <= 0 here, so only the lower bound matters).
BI_DEV float4 bi_exp4(float4 d) {
  float4 e;
  float mn;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(mn) : "f"(d.x), "f"(d.y), "f"(d.z));
  if (fminf(mn, d.w) >= -87.0f) {
    const float2 lo = upk2(bi_exp_fast2(pk2(d.x, d.y)));
    const float2 hi = upk2(bi_exp_fast2(pk2(d.z, d.w)));
    e = make_float4(lo.x, lo.y, hi.x, hi.y);
  } else {
    e.x = bi_exp(d.x);
    e.y = bi_exp(d.y);
    e.z = bi_exp(d.z);
    e.w = bi_exp(d.w);
  }
  return e;
}

BI_DEV float max4(float m, float4 v) {
  float a, b;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(a) : "f"(m), "f"(v.x), "f"(v.y));
  asm("max.f32 %0, %1, %2, %3;" : "=f"(b) : "f"(a), "f"(v.z), "f"(v.w));
  return b;
}

// THREADS = 4096 / C.  The minimum-blocks bound keeps the 256-thread form
// (C = 16) at <= 48 registers, so five CTAs (smem-limited) share an SM.
template <int THREADS>
__global__ void __launch_bounds__(THREADS, THREADS == 256 ? 5 : 0)
log_softmax_kernel(const __grid_constant__ LsmParams p) {
  extern __shared__ float4 lsm_smem[];
  __shared__ float s_red[32];
  __shared__ float s_max, s_sum;
  __shared__ float s_maxs[16], s_sums[16];     // the cluster's values, pushed by their owners
  __shared__ __align__(8) uint64_t s_bar[2];   // [0]: all C maxes landed, [1]: all C sums
  cg::cluster_group cluster = cg::this_cluster();
  const int C = p.C;
  const int q = (int)cluster.block_rank();
  const int lpc = kLsmT / C;                   // lanes (= threads) per CTA
  const int tau = threadIdx.x;
  const int lane_id = q * lpc + tau;           // logical lane
  const size_t row = blockIdx.x / C;
  const int nvec = p.n / 4;
  const float4 *xr = reinterpret_cast<const float4 *>(p.x + row * p.n);
  float4 *outr = reinterpret_cast<float4 *>(p.out + row * p.n);
  const int nwarps = lpc / 32;
  // this lane's vectors: 4096*j + lane_id for j < nj
  const int nj = lane_id < nvec ? (nvec - 1 - lane_id) / kLsmT + 1 : 0;

  // Each CTA pushes its max, then its sum, into slot q of every CTA with
  // st.async; a CTA's barrier counts the 4 * C bytes that land in its own
  // slots, so it waits for exactly the values it reads and no CTA waits for
  // another's threads.  The barriers are initialised before the cluster
  // arrive; every CTA has started (and initialised) once it is matched, and
  // the wait comes before the first push.
  if (tau == 0) {
    mbar_init(&s_bar[0], 1);
    mbar_init(&s_bar[1], 1);
    mbar_fence_init();
    mbar_arrive_expect_tx(&s_bar[0], 4u * C);
    mbar_arrive_expect_tx(&s_bar[1], 4u * C);
  }
  cluster_arrive_relaxed();

  // ---- this lane's vectors -> its shared-memory slots: 16-byte cp.async
  // copies, all in flight at once.  Each thread reads back only its own
  // slots, so waiting for its own copies is enough.
  for (int j = 0; j < nj; j++) cp_async16(lsm_smem + (size_t)j * lpc + tau, xr + (size_t)j * kLsmT + lane_id);
  cp_async_commit();
  cp_async_wait<0>();

  // ---- local max
  float m = -INFINITY;
  for (int j = 0; j < nj; j++) {
    m = max4(m, lsm_smem[j * lpc + tau]);
  }
  m = warp_max(m);
  if ((tau & 31) == 0) s_red[tau >> 5] = m;
  __syncthreads();
  if (tau < 32) {
    float v = tau < nwarps ? s_red[tau] : -INFINITY;
    v = warp_max(v);
    if (tau == 0) s_max = v;
  }
  __syncthreads();
  cluster_wait();
  // push this CTA's max into slot q of every CTA of the cluster
  if (tau < C) st_async_f32(&s_maxs[q], &s_bar[0], (uint32_t)tau, s_max);
  if (!mbar_wait_cluster(&s_bar[0], 0)) flag_error(p.status, BI_ERR_TIMEOUT);
  // row max over the cluster (exact in any order), from this CTA's own slots
  float rmax = s_maxs[0];
  for (int t = 1; t < C; t++) rmax = fmaxf(rmax, s_maxs[t]);
  const uint64_t rmax2 = splat2(rmax);

  // ---- lane chain of bi_exp(x - max); d = x - max stays in the slot
  float s = 0.0f;
#pragma unroll 2
  for (int j = 0; j < nj; j++) {
    const float4 xv = lsm_smem[j * lpc + tau];
    const float2 d01 = upk2(sub2_rn(pk2(xv.x, xv.y), rmax2));
    const float2 d23 = upk2(sub2_rn(pk2(xv.z, xv.w), rmax2));
    const float4 d = make_float4(d01.x, d01.y, d23.x, d23.y);
    lsm_smem[j * lpc + tau] = d;
    const float4 e = bi_exp4(d);
    s = __fadd_rn(s, e.x);
    s = __fadd_rn(s, e.y);
    s = __fadd_rn(s, e.z);
    s = __fadd_rn(s, e.w);
  }
  s = warp_tree_sum(s);
  if ((tau & 31) == 0) s_red[tau >> 5] = s;
  __syncthreads();
  if (tau < 32) {
    float v = tau < nwarps ? s_red[tau] : 0.0f;
    for (int o = 1; o < nwarps; o <<= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (tau == 0) s_sum = v;
  }
  __syncthreads();
  // push this CTA's subtree value into slot q of every CTA.  These are the
  // last writes into a peer's memory, and a peer cannot pass its own wait
  // before they land, so no CTA waits for the others before it exits.
  if (tau < C) st_async_f32(&s_sums[q], &s_bar[1], (uint32_t)tau, s_sum);
  if (!mbar_wait_cluster(&s_bar[1], 0)) flag_error(p.status, BI_ERR_TIMEOUT);
  // perfect tree over the C CTA subtrees (lanes 0..C-1, xor butterfly:
  // pairs, then pairs of pairs); every warp computes it from its own copy
  float v = (tau & 31) < C ? s_sums[tau & 31] : 0.0f;
  for (int o = 1; o < C; o <<= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
  v = __shfl_sync(0xffffffffu, v, 0);           // lanes >= C added zeros among themselves
  const uint64_t L2 = splat2(bi_log(v));

  // ---- write out = d - L
  for (int j = 0; j < nj; j++) {
    const float4 d = lsm_smem[j * lpc + tau];
    const float2 o01 = upk2(sub2_rn(pk2(d.x, d.y), L2));
    const float2 o23 = upk2(sub2_rn(pk2(d.z, d.w), L2));
    const float4 o = make_float4(o01.x, o01.y, o23.x, o23.y);
    __stcs(outr + (size_t)j * kLsmT + lane_id, o);
  }
}

// Test and reference hook: the library's exp / log applied elementwise.
__global__ void math_spec_kernel(const float *__restrict__ x, float *__restrict__ y, size_t n,
                                 int which) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    if (which == 3) {                      // packed: elements 2k, 2k+1 share one pair
      const size_t i0 = i & ~size_t(1), i1 = i0 + 1 < n ? i0 + 1 : i0;
      const float2 e = upk2(bi_exp_fast2(pk2(x[i0], x[i1])));
      y[i] = (i & 1) ? e.y : e.x;
    } else {
      y[i] = which == 0 ? bi_exp(x[i]) : (which == 1 ? bi_log(x[i]) : bi_exp_fast(x[i]));
    }
}

}  // namespace bi

// ----------------------------------------------------------------------
extern "C" bi_status bi_rmsnorm(const void *x, const void *w, void *y, int rows, int n, float eps,
                                bi_stream_t stream) {
  if (rows < 0 || n <= 0) return BI_ERR_INVALID_ARG;
  if (rows > 0 && (!x || !w || !y)) return BI_ERR_INVALID_ARG;
  if (n % 8 != 0 || n > 8 * bi::kNormT * 8) return BI_ERR_UNSUPPORTED_SHAPE;
  if (!bi_aligned16(x) || !bi_aligned16(w) || !bi_aligned16(y)) return BI_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0) return BI_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int vpl = (n / 8 + bi::kNormT - 1) / bi::kNormT;
  auto xp = static_cast<const uint16_t *>(x);
  auto wp = static_cast<const uint16_t *>(w);
  auto yp = static_cast<uint16_t *>(y);
  // thread count per row is bit-neutral (lanes are logical); 128 threads
  // with 4 lanes each while the row fits in registers
  if (vpl <= 1) bi::rmsnorm_kernel<128, 1><<<rows, 128, 0, s>>>(xp, wp, yp, n, eps);
  else if (vpl <= 2) bi::rmsnorm_kernel<128, 2><<<rows, 128, 0, s>>>(xp, wp, yp, n, eps);
  else if (vpl <= 4) bi::rmsnorm_kernel<128, 4><<<rows, 128, 0, s>>>(xp, wp, yp, n, eps);
  else bi::rmsnorm_kernel<256, 8><<<rows, 256, 0, s>>>(xp, wp, yp, n, eps);
  return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

extern "C" bi_status bi_mean(const float *x, float *out, int rows, int n, bi_stream_t stream) {
  if (rows < 0 || n <= 0) return BI_ERR_INVALID_ARG;
  if (rows > 0 && (!x || !out)) return BI_ERR_INVALID_ARG;
  if (n % 4 != 0) return BI_ERR_UNSUPPORTED_SHAPE;
  if (!bi_aligned16(x)) return BI_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0) return BI_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // few rows: a 16-CTA cluster per row (bit-neutral: the CTAs own subtrees)
  if (rows <= bi::kMeanClusterRows) {
    constexpr int C = 16;
    auto kern = bi::mean_cluster_kernel<C>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return BI_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)rows * C, 1, 1);
    cfg.blockDim = dim3(bi::kLaneT / C, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    unsigned *status = bi::status_word();
    return cudaLaunchKernelEx(&cfg, kern, x, out, n, status) == cudaSuccess ? BI_OK : BI_ERR_CUDA;
  }
  bi::mean_kernel<<<rows, bi::kMeanThreads, 0, s>>>(x, out, n);
  return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

extern "C" bi_status bi_log_softmax(const float *x, float *out, int rows, int n, bi_stream_t stream) {
  if (rows < 0 || n <= 0) return BI_ERR_INVALID_ARG;
  if (rows > 0 && (!x || !out)) return BI_ERR_INVALID_ARG;
  if (n % 4 != 0 || n > 262144) return BI_ERR_UNSUPPORTED_SHAPE;
  if (!bi_aligned16(x) || !bi_aligned16(out)) return BI_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0) return BI_OK;
  bi::LsmParams p{x, out, bi::status_word(), n, 4, 0};
  const int nvec = n / 4;
  p.J = (nvec + bi::kLsmT - 1) / bi::kLsmT;
  // Smallest cluster (4..16 CTAs, at most 1024 threads each) whose share of
  // the row fits in ~40 KB of shared memory, so that five row slices share
  // an SM and one slice's barriers overlap the others' loads (at 151936
  // columns: C = 16, 8% faster than C = 8).  Bit-neutral.
  int C = 4;
  while (C < 16 && (size_t)p.J * (bi::kLsmT / C) * 16 > 40 * 1024) C *= 2;
  p.C = C;
  const size_t smem = (size_t)p.J * (bi::kLsmT / C) * 16;
  if (smem > 200 * 1024) return BI_ERR_UNSUPPORTED_SHAPE;
  auto launch = [&](auto kern) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (C > 8) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)rows * C, 1, 1);
    cfg.blockDim = dim3(bi::kLsmT / C, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p);
  };
  cudaError_t e;
  switch (C) {
    case 4: e = launch(bi::log_softmax_kernel<1024>); break;
    case 8: e = launch(bi::log_softmax_kernel<512>); break;
    default: e = launch(bi::log_softmax_kernel<256>); break;
  }
  return e == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

extern "C" bi_status bi_math_spec(const float *x, float *y, size_t n, int which, bi_stream_t stream) {
  if ((n > 0 && (!x || !y)) || which < 0 || which > 3) return BI_ERR_INVALID_ARG;
  if (n == 0) return BI_OK;
  const unsigned blocks = (unsigned)std::min<size_t>((n + 255) / 256, (size_t)bi::num_sms() * 16);
  bi::math_spec_kernel<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, y, n, which);
  return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}
