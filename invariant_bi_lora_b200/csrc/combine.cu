// combine.cu -- cross-shard combine of tensor-parallel partials.
//
// "Deterministic Inference across Tensor Parallel Sizes That Eliminates
// Training-Inference Mismatch" (Abstract): the inter-GPU reduction follows
// the same hierarchical binary tree as the intra-GPU one.  With K split into
// s contiguous shards that are subtrees of the canonical tree, the shard
// partials are combined by the top levels of that tree: out[i] =
// tree(partials[0][i], ..., partials[s-1][i]).  The tree is evaluated in
// post order on a small register stack (the merge schedule is computed on
// the host), four elements per thread with 16-byte loads.
#include "common.cuh"

#include <algorithm>

namespace bi {

constexpr int kMaxCombine = 64;

struct CombineParams {
  const float *parts;
  float *out;
  size_t count;
  int s;
  uint8_t merges[kMaxCombine];
};

__global__ void __launch_bounds__(256)
tree_combine_kernel(const __grid_constant__ CombineParams p) {
  constexpr int D = 7;   // stack depth for s <= 64
  const size_t nv = p.count / 4;
  const float4 *src = reinterpret_cast<const float4 *>(p.parts);
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < nv;
       i += (size_t)gridDim.x * blockDim.x) {
    float4 st[D];
#pragma unroll
    for (int d = 0; d < D; d++) st[d] = make_float4(0.f, 0.f, 0.f, 0.f);
    int depth = 0;
    for (int j = 0; j < p.s; j++) {
      const float4 v = __ldcs(src + (size_t)j * nv + i);
#pragma unroll
      for (int d = 0; d < D; d++) {
        const bool hit = d == depth;
        st[d].x = hit ? v.x : st[d].x;
        st[d].y = hit ? v.y : st[d].y;
        st[d].z = hit ? v.z : st[d].z;
        st[d].w = hit ? v.w : st[d].w;
      }
      depth++;
      const int nm = p.merges[j];
#pragma unroll 1
      for (int m = 0; m < nm; m++) {
#pragma unroll
        for (int d = 1; d < D; d++) {
          const bool hit = d == depth - 1;
          const float4 a = st[d - 1], b = st[d];
          st[d - 1].x = hit ? __fadd_rn(a.x, b.x) : a.x;
          st[d - 1].y = hit ? __fadd_rn(a.y, b.y) : a.y;
          st[d - 1].z = hit ? __fadd_rn(a.z, b.z) : a.z;
          st[d - 1].w = hit ? __fadd_rn(a.w, b.w) : a.w;
        }
        depth--;
      }
    }
    reinterpret_cast<float4 *>(p.out)[i] = st[0];
  }
}

// s = S, a power of two: the canonical tree is the perfect tree, so all S
// loads of a thread are issued together and added pairwise afterwards (the
// general kernel's loop issues one load per merge step and waits on each).
template <int S>
__global__ void __launch_bounds__(256)
tree_combine_pow2_kernel(const float *__restrict__ parts, float *__restrict__ out, size_t nv) {
  const float4 *src = reinterpret_cast<const float4 *>(parts);
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < nv;
       i += (size_t)gridDim.x * blockDim.x) {
    float4 v[S];
#pragma unroll
    for (int j = 0; j < S; j++) v[j] = __ldcs(src + (size_t)j * nv + i);
#pragma unroll
    for (int st = 1; st < S; st <<= 1)
#pragma unroll
      for (int q = 0; q + st < S; q += 2 * st) {
        v[q].x = __fadd_rn(v[q].x, v[q + st].x);
        v[q].y = __fadd_rn(v[q].y, v[q + st].y);
        v[q].z = __fadd_rn(v[q].z, v[q + st].z);
        v[q].w = __fadd_rn(v[q].w, v[q + st].w);
      }
    __stcs(reinterpret_cast<float4 *>(out) + i, v[0]);
  }
}

// Post-order merge schedule of the canonical halving tree over n leaves.
void tree_schedule(int n, uint8_t *merges) {
  std::fill(merges, merges + n, 0);
  struct R {
    static void go(int lo, int hi, uint8_t *m) {
      if (hi - lo <= 1) return;
      const int h = lo + (hi - lo + 1) / 2;
      go(lo, h, m);
      go(h, hi, m);
      m[hi - 1]++;
    }
  };
  R::go(0, n, merges);
}

// ---- partials behind s separate pointers (peer GPUs' memory mapped into
// this process, or local buffers): the same tree, element range
// [begin, begin + count) of every partial into the same range of out.
// Plain 16-byte loads through each pointer, no multicast.
struct PeerCombineParams {
  const float4 *ptr[kMaxCombine];
  float4 *out;
  size_t v0, nv;              // first vector and vector count of the range
  int s;
  uint8_t merges[kMaxCombine];
};

template <int S>
__global__ void __launch_bounds__(256)
tree_combine_peers_pow2_kernel(const __grid_constant__ PeerCombineParams p) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < p.nv;
       i += (size_t)gridDim.x * blockDim.x) {
    float4 v[S];
#pragma unroll
    for (int j = 0; j < S; j++) v[j] = p.ptr[j][p.v0 + i];
#pragma unroll
    for (int st = 1; st < S; st <<= 1)
#pragma unroll
      for (int q = 0; q + st < S; q += 2 * st) {
        v[q].x = __fadd_rn(v[q].x, v[q + st].x);
        v[q].y = __fadd_rn(v[q].y, v[q + st].y);
        v[q].z = __fadd_rn(v[q].z, v[q + st].z);
        v[q].w = __fadd_rn(v[q].w, v[q + st].w);
      }
    p.out[p.v0 + i] = v[0];
  }
}

__global__ void __launch_bounds__(256)
tree_combine_peers_kernel(const __grid_constant__ PeerCombineParams p) {
  constexpr int D = 7;   // stack depth for s <= 64
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < p.nv;
       i += (size_t)gridDim.x * blockDim.x) {
    float4 st[D];
#pragma unroll
    for (int d = 0; d < D; d++) st[d] = make_float4(0.f, 0.f, 0.f, 0.f);
    int depth = 0;
    for (int j = 0; j < p.s; j++) {
      const float4 v = p.ptr[j][p.v0 + i];
#pragma unroll
      for (int d = 0; d < D; d++) {
        const bool hit = d == depth;
        st[d].x = hit ? v.x : st[d].x;
        st[d].y = hit ? v.y : st[d].y;
        st[d].z = hit ? v.z : st[d].z;
        st[d].w = hit ? v.w : st[d].w;
      }
      depth++;
      const int nm = p.merges[j];
#pragma unroll 1
      for (int m = 0; m < nm; m++) {
#pragma unroll
        for (int d = 1; d < D; d++) {
          const bool hit = d == depth - 1;
          const float4 a = st[d - 1], b = st[d];
          st[d - 1].x = hit ? __fadd_rn(a.x, b.x) : a.x;
          st[d - 1].y = hit ? __fadd_rn(a.y, b.y) : a.y;
          st[d - 1].z = hit ? __fadd_rn(a.z, b.z) : a.z;
          st[d - 1].w = hit ? __fadd_rn(a.w, b.w) : a.w;
        }
        depth--;
      }
    }
    p.out[p.v0 + i] = st[0];
  }
}

bi_status tree_combine_launch(const float *partials, float *out, int s, size_t count,
                              cudaStream_t stream) {
  if (s < 1 || s > kMaxCombine) return BI_ERR_INVALID_ARG;
  if (count > 0 && (!partials || !out)) return BI_ERR_INVALID_ARG;
  if (count % 4 != 0 || !bi_aligned16(partials) || !bi_aligned16(out)) return BI_ERR_UNSUPPORTED_SHAPE;
  if (count == 0) return BI_OK;
  CombineParams p{};
  p.parts = partials;
  p.out = out;
  p.count = count;
  p.s = s;
  tree_schedule(s, p.merges);
  const size_t nv = count / 4;
  const unsigned blocks = (unsigned)std::min<size_t>((nv + 255) / 256, (size_t)num_sms() * 8);
  switch (s) {
    case 2: tree_combine_pow2_kernel<2><<<blocks, 256, 0, stream>>>(partials, out, nv); break;
    case 4: tree_combine_pow2_kernel<4><<<blocks, 256, 0, stream>>>(partials, out, nv); break;
    case 8: tree_combine_pow2_kernel<8><<<blocks, 256, 0, stream>>>(partials, out, nv); break;
    case 16: tree_combine_pow2_kernel<16><<<blocks, 256, 0, stream>>>(partials, out, nv); break;
    default: tree_combine_kernel<<<blocks, 256, 0, stream>>>(p); break;
  }
  return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

bi_status tree_combine_peers_launch(const float *const *partials, int s, float *out, size_t begin, size_t count,
                                    cudaStream_t stream) {
  if (s < 1 || s > kMaxCombine || !partials) return BI_ERR_INVALID_ARG;
  if (count > 0 && !out) return BI_ERR_INVALID_ARG;
  if (count % 4 != 0 || begin % 4 != 0 || !bi_aligned16(out)) return BI_ERR_UNSUPPORTED_SHAPE;
  PeerCombineParams p{};
  for (int j = 0; j < s; j++) {
    if (count > 0 && !partials[j]) return BI_ERR_INVALID_ARG;
    if (!bi_aligned16(partials[j])) return BI_ERR_UNSUPPORTED_SHAPE;
    p.ptr[j] = reinterpret_cast<const float4 *>(partials[j]);
  }
  if (count == 0) return BI_OK;
  p.out = reinterpret_cast<float4 *>(out);
  p.v0 = begin / 4;
  p.nv = count / 4;
  p.s = s;
  tree_schedule(s, p.merges);
  const unsigned blocks = (unsigned)std::min<size_t>((p.nv + 255) / 256, (size_t)num_sms() * 8);
  switch (s) {
    case 2: tree_combine_peers_pow2_kernel<2><<<blocks, 256, 0, stream>>>(p); break;
    case 4: tree_combine_peers_pow2_kernel<4><<<blocks, 256, 0, stream>>>(p); break;
    case 8: tree_combine_peers_pow2_kernel<8><<<blocks, 256, 0, stream>>>(p); break;
    case 16: tree_combine_peers_pow2_kernel<16><<<blocks, 256, 0, stream>>>(p); break;
    default: tree_combine_peers_kernel<<<blocks, 256, 0, stream>>>(p); break;
  }
  return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

}  // namespace bi

extern "C" bi_status bi_tree_combine_peers(const float *const *partials, int s, float *out, size_t begin,
                                           size_t count, bi_stream_t stream) {
  return bi::tree_combine_peers_launch(partials, s, out, begin, count, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" bi_status bi_tree_combine(const float *partials, float *out, int s, size_t count,
                                     bi_stream_t stream) {
  return bi::tree_combine_launch(partials, out, s, count, reinterpret_cast<cudaStream_t>(stream));
}
