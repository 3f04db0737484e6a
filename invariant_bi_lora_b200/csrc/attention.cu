// attention.cu -- batch-invariant decode attention with a fixed-size KV
// split.
//
// "Restoring AI Reproducibility: Thinking Machines Lab's Challenge to
// Overcome Nondeterminism" (2-3, 3-2): attention must reduce in an order that
// does not depend on the batch; for decoding, where the KV cache is split
// across workers for parallelism, the split has to be by a fixed SIZE, not a
// fixed count chosen from the batch.  Here the KV sequence of every
// (sequence, head) is cut into chunks of 256 key slots whatever the batch,
// and every sum is a fixed tree:
//   s_j  = fl(fl(perfect tree over d of q_d * k_jd) * scale)
//          (a bf16 x bf16 product is exact in fp32; D is a power of two)
//   m_c  = max over the chunk's keys;  p_j = bi_exp(fl(s_j - m_c))
//   l_c  = perfect tree over the 256 slots of p_j (slots past the length
//          hold +0)
//   o_cd = perfect tree over the 256 slots of fl(p_j * v_jd)
// then, over the n = ceil(L/256) chunks padded with zero chunks to the next
// power of two: M = max m_c, a_c = bi_exp(fl(m_c - M)), l and O_d perfect
// trees of fl(a_c * l_c) and fl(a_c * o_cd), out_d = fl(O_d / l).
// The order depends on the sequence's own length only, so a row's bits do
// not depend on the batch, on the row's position in it, or on how many CTAs
// share its chunks.  Decoding reads every K and V element once for a few
// flops, so the work runs on the CUDA cores in exactly this order (the CPU
// oracle reproduces it bit for bit) and is bound by the KV read.
//
// Kernel 1 (one CTA per chunk, kv head, sequence; 256 threads): every lane
// loads one key row into registers and folds its scores; the PV sums read
// V straight from global memory (a warp reads 128 contiguous bytes of one V
// row per slot), so a CTA needs little shared memory (18 KB at D = 128
// with four query heads per kv head) and four share an SM there; the chunk
// partials (m_c, l_c, o_c) of the G query heads that share the kv head go
// to the caller's workspace.  Kernel 2 (one CTA per query head and
// sequence): the combine.
#include "bimath.cuh"
#include "tc.cuh"

namespace bi {

constexpr int kAttnChunk = 256;
constexpr int kAttnThreads = 256;

struct AttnParams {
  const uint16_t *q;       // [B][Hq][D] bf16
  const uint16_t *k, *v;   // [B][Hkv][Lmax][D] bf16
  const int32_t *lens;     // [B]
  float *ws;               // [B][Hq][max_chunks][D + 2]: m, l, o[D]
  float *out;              // [B][Hq][D]
  int B, Hq, Hkv, Lmax, max_chunks;
  float scale;
  unsigned *status;
};

// Perfect-tree fold of value i (0..2^LEVELS-1, in order) into the pending
// subtrees lv: the binary counter of the canonical tree.
template <int LEVELS>
BI_DEV float counter_fold(int i, float x, float (&lv)[LEVELS > 0 ? LEVELS : 1]) {
#pragma unroll
  for (int L = 0; L < LEVELS; L++) {
    if ((i >> L) & 1) {
      x = __fadd_rn(lv[L], x);
    } else {
      lv[L] = x;
      return x;
    }
  }
  return x;
}

// Four CTAs per SM (64 registers) where that costs no spill (G * D <= 512:
// the common D = 128 with up to four query heads per kv head), else two.
template <int D, int G>
__global__ void __launch_bounds__(kAttnThreads, G * D >= 1024 ? 2 : 4)
attn_chunk_kernel(const __grid_constant__ AttnParams p) {
  constexpr int QT = 2 * kAttnThreads / D;          // threads per output column pair
  constexpr int SLOTS = kAttnChunk / QT;            // slots per thread in the PV sum
  constexpr int LV = SLOTS >= 128 ? 7 : SLOTS >= 64 ? 6 : 5;
  constexpr int GP = G >= 4 ? G : 4;                // p row padded to a float4
  __shared__ float s_q[G][D];
  __shared__ float s_p[G][kAttnChunk];             // scores
  __shared__ __align__(16) float s_pt[kAttnChunk][GP];   // p, [slot][head]
  __shared__ float s_red[G][8];
  __shared__ float s_half[G][QT][D];

  const int c = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int L = max(0, min(p.lens[b], p.Lmax));      // a length past Lmax reads nothing beyond it
  const int j0 = c * kAttnChunk;
  // one chunk per sequence at most (max_chunks == 1): this kernel writes the
  // output itself, an empty sequence's included (see the end)
  if (p.max_chunks == 1 && L == 0) {
    for (int e = threadIdx.x; e < G * D; e += kAttnThreads) p.out[((size_t)b * p.Hq + hk * G) * D + e] = 0.0f;
    return;
  }
  if (j0 >= L) return;                              // past this sequence's chunks
  const int nj = min(kAttnChunk, L - j0);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t kvbase = (((size_t)b * p.Hkv + hk) * p.Lmax + j0) * D;

  for (int e = tid; e < G * D; e += kAttnThreads) {
    const int i = e / D, d = e % D;
    s_q[i][d] = __uint_as_float((uint32_t)p.q[((size_t)b * p.Hq + hk * G + i) * D + d] << 16);
  }
  __syncthreads();

  // ---- scores: lane l of warp w owns slot 32w + l and computes the perfect
  // tree over d of q_d * k_d itself, 32 d at a time: each 32-wide block is
  // a subtree (a binary counter, every index known at compile time), and the
  // D/32 block values meet in a perfect tree.  q is read from shared memory
  // by broadcast.
  {
    const int j = warp * 32 + lane;
    constexpr int NBLK = D / 32;
    float blk[G][NBLK];
    const uint4 *kr = reinterpret_cast<const uint4 *>(p.k + kvbase + (size_t)(j < nj ? j : 0) * D);
    uint4 cur[4], nxt[4];
#pragma unroll
    for (int e = 0; e < 4; e++) cur[e] = kr[e];
#pragma unroll
    for (int bk = 0; bk < NBLK; bk++) {
      if (bk + 1 < NBLK)
#pragma unroll
        for (int e = 0; e < 4; e++) nxt[e] = kr[4 * (bk + 1) + e];
#pragma unroll
      for (int i = 0; i < G; i++) {
        float lvd[5];
        float x = 0.0f;
#pragma unroll
        for (int e = 0; e < 4; e++) {
          const uint32_t w[4] = {cur[e].x, cur[e].y, cur[e].z, cur[e].w};
          const float4 qa = *reinterpret_cast<const float4 *>(&s_q[i][32 * bk + 8 * e]);
          const float4 qb = *reinterpret_cast<const float4 *>(&s_q[i][32 * bk + 8 * e + 4]);
          const float qv[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
#pragma unroll
          for (int u = 0; u < 8; u++) {
            const float kf = (u & 1) ? bf16hi(w[u >> 1]) : bf16lo(w[u >> 1]);
            x = counter_fold<5>(8 * e + u, __fmul_rn(qv[u], kf), lvd);        // exact product
          }
        }
        blk[i][bk] = x;
      }
      if (bk + 1 < NBLK)
#pragma unroll
        for (int e = 0; e < 4; e++) cur[e] = nxt[e];
    }
#pragma unroll
    for (int i = 0; i < G; i++) {
#pragma unroll
      for (int w = 1; w < NBLK; w <<= 1)
#pragma unroll
        for (int e = 0; e + w < NBLK; e += 2 * w) blk[i][e] = __fadd_rn(blk[i][e], blk[i][e + w]);
      s_p[i][j] = j < nj ? __fmul_rn(blk[i][0], p.scale) : -INFINITY;
    }
  }
  __syncthreads();

  // ---- chunk max, p = exp(s - m), l = perfect tree over the 256 slots
  // (thread t holds slot t: the butterfly is the tree over 32 slots, then
  // the eight warp values in a perfect tree)
  float m_i[G];
#pragma unroll
  for (int i = 0; i < G; i++) {
    const float mw = warp_max(s_p[i][tid]);
    if (lane == 0) s_red[i][warp] = mw;
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < G; i++) {
    float m = s_red[i][0];
#pragma unroll
    for (int w = 1; w < 8; w++) m = fmaxf(m, s_red[i][w]);
    m_i[i] = m;
  }
  __syncthreads();
  float pv[G];
#pragma unroll
  for (int i = 0; i < G; i++) {
    pv[i] = tid < nj ? bi_exp(__fsub_rn(s_p[i][tid], m_i[i])) : 0.0f;
    s_pt[tid][i] = pv[i];
    const float lw = warp_tree_sum(pv[i]);
    if (lane == 0) s_red[i][warp] = lw;
  }
  __syncthreads();
  float l_i[G];
#pragma unroll
  for (int i = 0; i < G; i++) {
    float r[8];
#pragma unroll
    for (int w = 0; w < 8; w++) r[w] = s_red[i][w];
#pragma unroll
    for (int w = 1; w < 8; w <<= 1)
#pragma unroll
      for (int e = 0; e + w < 8; e += 2 * w) r[e] = __fadd_rn(r[e], r[e + w]);
    l_i[i] = r[0];
  }

  // ---- o_d: thread (part qt, columns 2dp and 2dp + 1) folds slots
  // [qt*SLOTS, +SLOTS) (a subtree) with the binary counter; one vector load
  // gives every head's p of a slot; the QT subtrees meet in order.  V comes
  // straight from global memory: a warp's 32 threads read 128 contiguous
  // bytes of one V row per slot, eight slots' loads in flight ahead.
  const int dp = tid % (D / 2), qt = tid / (D / 2);
  float acc[G][2];
  float lv[G][2][LV];
  const uint32_t *vcol = reinterpret_cast<const uint32_t *>(p.v + kvbase) + dp;   // V[j][2dp, 2dp+1]
  constexpr int VPF = 8;
  uint32_t vbuf[VPF];
#pragma unroll
  for (int s = 0; s < VPF; s++) {
    const int j = qt * SLOTS + s;
    vbuf[s] = j < nj ? __ldg(vcol + (size_t)j * (D / 2)) : 0u;
  }
#pragma unroll
  for (int s = 0; s < SLOTS; s++) {
    const int j = qt * SLOTS + s;
    const uint32_t vw = vbuf[s % VPF];
    if (s + VPF < SLOTS) {
      const int jn = j + VPF;
      vbuf[s % VPF] = jn < nj ? __ldg(vcol + (size_t)jn * (D / 2)) : 0u;
    }
    const float v0 = j < nj ? bf16lo(vw) : 0.0f, v1 = j < nj ? bf16hi(vw) : 0.0f;
    float pj[GP];
#pragma unroll
    for (int u = 0; u < GP; u += 4) {
      const float4 q4 = *reinterpret_cast<const float4 *>(&s_pt[j][u]);
      pj[u] = q4.x; pj[u + 1] = q4.y; pj[u + 2] = q4.z; pj[u + 3] = q4.w;
    }
#pragma unroll
    for (int i = 0; i < G; i++) {
      acc[i][0] = counter_fold<LV>(s, j < nj ? __fmul_rn(pj[i], v0) : 0.0f, lv[i][0]);
      acc[i][1] = counter_fold<LV>(s, j < nj ? __fmul_rn(pj[i], v1) : 0.0f, lv[i][1]);
    }
  }
#pragma unroll
  for (int i = 0; i < G; i++) {
    s_half[i][qt][2 * dp] = acc[i][0];
    s_half[i][qt][2 * dp + 1] = acc[i][1];
  }
  __syncthreads();
  const int d = tid % D;
  float *wsb = p.ws + (((size_t)b * p.Hq + hk * G) * p.max_chunks + c) * (D + 2);
  const size_t head_stride = (size_t)p.max_chunks * (D + 2);
  if (tid < D) {
#pragma unroll
    for (int i = 0; i < G; i++) {
      float r[QT];
#pragma unroll
      for (int e = 0; e < QT; e++) r[e] = s_half[i][e][d];
#pragma unroll
      for (int w = 1; w < QT; w <<= 1)
#pragma unroll
        for (int e = 0; e + w < QT; e += 2 * w) r[e] = __fadd_rn(r[e], r[e + w]);
      if (p.max_chunks == 1) {
        // the combine over one chunk: weight bi_exp(0) = 1 exactly and no
        // tree levels, so out = fl(o / l) -- the same bits as kernel 2
        p.out[((size_t)b * p.Hq + hk * G + i) * D + d] = __fdiv_rn(r[0], l_i[i]);
        continue;
      }
      wsb[i * head_stride + 2 + d] = r[0];
      if (d == 0) {
        wsb[i * head_stride + 0] = m_i[i];
        wsb[i * head_stride + 1] = l_i[i];
      }
    }
  }
}

// One CTA of D threads per (query head, sequence): weights of the chunks,
// then the perfect trees over the chunk count padded to a power of two.
template <int D>
__global__ void __launch_bounds__(D)
attn_combine_kernel(const __grid_constant__ AttnParams p) {
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  const int L = max(0, min(p.lens[b], p.Lmax));
  float *o = p.out + ((size_t)b * p.Hq + h) * D;
  if (L <= 0) {
    o[d] = 0.0f;
    return;
  }
  const int n = (L + kAttnChunk - 1) / kAttnChunk;
  const float *wsb = p.ws + ((size_t)b * p.Hq + h) * p.max_chunks * (D + 2);
  float M = wsb[0];
  for (int c = 1; c < n; c++) M = fmaxf(M, wsb[(size_t)c * (D + 2)]);
  int P = 1;
  while (P < n) P <<= 1;
  constexpr int LVMAX = 16;
  float lvo[LVMAX], lvl[LVMAX];
  float O = 0.0f, l = 0.0f;
  for (int c = 0; c < P; c++) {
    float vo = 0.0f, vl = 0.0f;
    if (c < n) {
      const float a = bi_exp(__fsub_rn(wsb[(size_t)c * (D + 2)], M));
      vl = __fmul_rn(a, wsb[(size_t)c * (D + 2) + 1]);
      vo = __fmul_rn(a, wsb[(size_t)c * (D + 2) + 2 + d]);
    }
    // binary counter with a runtime index (levels held in local arrays)
    int L2 = 0;
    for (; L2 < LVMAX && ((c >> L2) & 1); L2++) {
      vo = __fadd_rn(lvo[L2], vo);
      vl = __fadd_rn(lvl[L2], vl);
    }
    if (L2 < LVMAX) {
      lvo[L2] = vo;
      lvl[L2] = vl;
    }
    O = vo;
    l = vl;
  }
  o[d] = __fdiv_rn(O, l);
}

template <int D, int G>
static cudaError_t attn_chunk_launch(const AttnParams &p, cudaStream_t s) {
  const dim3 g1(p.max_chunks, p.Hkv, p.B);
  attn_chunk_kernel<D, G><<<g1, kAttnThreads, 0, s>>>(p);
  return cudaGetLastError();
}

template <int D>
static bi_status attn_launch_d(const AttnParams &p, int G, cudaStream_t s) {
  cudaError_t e;
  switch (G) {
    case 1: e = attn_chunk_launch<D, 1>(p, s); break;
    case 2: e = attn_chunk_launch<D, 2>(p, s); break;
    case 4: e = attn_chunk_launch<D, 4>(p, s); break;
    case 8: e = attn_chunk_launch<D, 8>(p, s); break;
    default: return BI_ERR_UNSUPPORTED_SHAPE;
  }
  if (e != cudaSuccess) return BI_ERR_CUDA;
  if (p.max_chunks == 1) return BI_OK;              // kernel 1 wrote the output
  attn_combine_kernel<D><<<dim3(p.Hq, p.B), D, 0, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

}  // namespace bi

extern "C" size_t bi_attn_decode_ws_bytes(int B, int Hq, int D, int Lmax) {
  if (B < 0 || Hq < 1 || D < 1 || Lmax < 0) return 0;
  const size_t chunks = (size_t)(Lmax + bi::kAttnChunk - 1) / bi::kAttnChunk;
  return sizeof(float) * (size_t)B * Hq * (chunks > 0 ? chunks : 1) * (size_t)(D + 2);
}

extern "C" bi_status bi_attn_decode(const void *q, const void *k, const void *v, const int32_t *lens, float *out,
                                    int B, int Hq, int Hkv, int D, int Lmax, float scale, void *ws, size_t ws_bytes,
                                    bi_stream_t stream) {
  if (B < 0 || Hq < 1 || Hkv < 1 || D < 1 || Lmax < 0) return BI_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return BI_ERR_UNSUPPORTED_SHAPE;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return BI_ERR_UNSUPPORTED_SHAPE;
  if (D != 64 && D != 128 && D != 256) return BI_ERR_UNSUPPORTED_SHAPE;
  if (B == 0) return BI_OK;
  if (!q || !k || !v || !lens || !out) return BI_ERR_INVALID_ARG;
  if (!bi_aligned16(q) || !bi_aligned16(k) || !bi_aligned16(v) || !bi_aligned16(out)) return BI_ERR_UNSUPPORTED_SHAPE;
  if (!ws || ws_bytes < bi_attn_decode_ws_bytes(B, Hq, D, Lmax)) return BI_ERR_WORKSPACE;
  bi::AttnParams p{};
  p.q = static_cast<const uint16_t *>(q);
  p.k = static_cast<const uint16_t *>(k);
  p.v = static_cast<const uint16_t *>(v);
  p.lens = lens;
  p.ws = static_cast<float *>(ws);
  p.out = out;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Lmax = Lmax;
  p.max_chunks = (Lmax + bi::kAttnChunk - 1) / bi::kAttnChunk;
  if (p.max_chunks == 0) p.max_chunks = 1;
  p.scale = scale;
  p.status = bi::status_word();
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (D == 64) return bi::attn_launch_d<64>(p, G, s);
  if (D == 128) return bi::attn_launch_d<128>(p, G, s);
  return bi::attn_launch_d<256>(p, G, s);
}
