/*
 * oracle.c -- plain, slow, obviously correct CPU reference for the
 * deterministic-reduction kernels.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link,
 * load or call this file: only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark use it.  It shares no code, header,
 * table or constant with the CUDA library; every constant below is written
 * out here from its mathematical definition.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fopenmp -fPIC
 *        -shared oracle.c -lm
 * (-ffp-contract=off: no multiply-add fusion anywhere unless written as
 * fmaf(); float expressions are evaluated in float on x86-64 SSE.)
 *
 * Two kinds of reference live here:
 *   1. EXACT references in double precision (the targets of the tolerance
 *      test).  They also return, per output element, the bound sum
 *      B = sum_k |x_k * a_k| used by the tolerance |gpu - exact| <= 1e-3 * B.
 *   2. CANONICAL fp32 references: the exact sequence of IEEE-754 fp32
 *      round-to-nearest operations that a deterministic kernel must perform
 *      (the fixed reduction tree), for the bit-exact tests.
 *
 * Sources, by page and section:
 *   [LoRA]  "Reproducible LoRA Inference Through Deterministic Split-K
 *           Reduction", Highlights and Q&A: split-K LoRA shrink whose
 *           partials are combined in a fixed order instead of fp32 atomics.
 *   [TBIK]  "Deterministic Inference across Tensor Parallel Sizes That
 *           Eliminates Training-Inference Mismatch", Abstract: one
 *           hierarchical binary tree orders both the intra- and inter-GPU
 *           reduction, so every TP size gives the same bits.
 *   [BI]    "The biggest Mystery of LLMs have just been solved", Detailed
 *           Analysis (fixed reduction tree, locked kernel policy, the
 *           fp32 non-associativity example) and "Restoring AI
 *           Reproducibility", sections 2-3 and 3-1 (RMSNorm / matmul /
 *           attention reductions, one core per batch element).
 *   [BIO]   "Batch Invariant Ops", Highlighted Details: mm, addmm,
 *           log_softmax, mean.
 *
 * Readings where the pages are silent (each one is listed in the design
 * notes of the repository):
 *   - tree shape: halving tree, left half = ceil(n/2)          (tree_f32)
 *   - row reduction: T logical lanes, vectors of V elements,
 *     lane chains then the tree over lanes                     (canon_sum)
 *   - exp / log: Cody-Waite + Taylor, and the atanh series      (or_exp/or_log)
 *   - weights are stored K-contiguous: A as [r][K], W as [N][K],
 *     LoRA-B as [N][r] (the out x in layout of a linear layer).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* bfloat16: the top 16 bits of an IEEE fp32 value.                     */
/* ------------------------------------------------------------------ */

static float bits_to_f32(uint32_t b) { float f; memcpy(&f, &b, 4); return f; }
static uint32_t f32_to_bits(float f) { uint32_t b; memcpy(&b, &f, 4); return b; }

float or_bf16_to_f32(uint16_t h) { return bits_to_f32(((uint32_t)h) << 16); }

/* Round-to-nearest-even from fp32 to bf16.  The 16 discarded bits are
 * compared with one half ulp of the kept part; a tie goes to the even
 * (low bit 0) neighbour.  NaN stays NaN (quiet bit forced). */
uint16_t or_f32_to_bf16(float f)
{
    uint32_t b = f32_to_bits(f);
    if ((b & 0x7f800000u) == 0x7f800000u && (b & 0x007fffffu) != 0)
        return (uint16_t)((b >> 16) | 0x0040u);
    uint32_t keep = b >> 16;
    uint32_t rest = b & 0xffffu;
    if (rest > 0x8000u || (rest == 0x8000u && (keep & 1u)))
        keep += 1u;              /* carries into the exponent correctly */
    return (uint16_t)keep;
}

void or_f32_to_bf16_array(const float *v, long n, uint16_t *out)
{
    for (long i = 0; i < n; i++) out[i] = or_f32_to_bf16(v[i]);
}

static double bf(uint16_t h) { return (double)or_bf16_to_f32(h); }

/* ------------------------------------------------------------------ */
/* The canonical reduction tree [TBIK Abstract; BI Detailed Analysis].  */
/*                                                                      */
/*   tree(v[0..n)) = v[0]                                  if n == 1    */
/*                 = fl( tree(v[0..h)) + tree(v[h..n)) )   h = ceil(n/2)*/
/*                                                                      */
/* For n = 2^k this is the perfect binary tree over contiguous pairs    */
/* (the order of a shfl_xor butterfly 1,2,4,..).  Any power-of-two s    */
/* that divides n cuts v into s contiguous blocks that are exactly the  */
/* subtrees at depth log2(s); that is what makes split counts and       */
/* emulated TP shard counts bitwise irrelevant.                         */
/* ------------------------------------------------------------------ */

float or_tree_f32(const float *v, long n, long stride)
{
    if (n <= 0) return 0.0f;
    if (n == 1) return v[0];
    long h = (n + 1) / 2;
    float left = or_tree_f32(v, h, stride);
    float right = or_tree_f32(v + h * stride, n - h, stride);
    return left + right;
}

/* out[i] = tree over parts[0*count + i], parts[1*count + i], ...,
 * parts[(s-1)*count + i]. */
void or_tree_combine(const float *parts, long s, long count, float *out, int nthreads)
{
    #pragma omp parallel for schedule(static) num_threads(nthreads)
    for (long i = 0; i < count; i++)
        out[i] = or_tree_f32(parts + i, s, count);
}

/* Canonical row sum [BI: one core per row, consistent order]:
 * T logical lanes; lane t starts at +0.0f and adds, in order, the V
 * elements of vectors j = t, t+T, t+2T, ... (j < n/V); the T lane
 * partials are then combined by the tree.  n must be a multiple of V. */
float or_canon_sum(const float *v, long n, int T, int V)
{
    long nvec = n / V;
    float *lane = (float *)malloc(sizeof(float) * (size_t)T);
    for (int t = 0; t < T; t++) {
        float p = 0.0f;
        for (long j = t; j < nvec; j += T)
            for (int e = 0; e < V; e++)
                p = p + v[j * V + e];
        lane[t] = p;
    }
    float s = or_tree_f32(lane, T, 1);
    free(lane);
    return s;
}

/* ------------------------------------------------------------------ */
/* exp and log used by log_softmax.  fp32 exp/log are not correctly     */
/* rounded on any platform, so bitwise agreement needs one written      */
/* method that both sides follow operation by operation.                */
/*                                                                      */
/* or_exp(x): Cody-Waite range reduction x = n*ln2 + r with ln2 split   */
/* into a 16-bit head and a tail, |r| <= ln2/2, then the Taylor series  */
/* of e^r through r^7 in Horner form with fused multiply-adds, then an  */
/* exact scaling by 2^n built from exponent bits.  x < -103 gives +0.   */
/* Domain of use: x <= 88.                                              */
/* ------------------------------------------------------------------ */

static float pow2i(int n)   /* 2^n for -126 <= n <= 127, exact */
{
    return bits_to_f32((uint32_t)(n + 127) << 23);
}

float or_exp(float x)
{
    /* ln2 = 0.693147180559945309...; head = ln2 with the low 8 mantissa
     * bits cleared (0x3f317200), tail = ln2 - head rounded to fp32. */
    const float log2e  = (float)1.4426950408889634074;
    const float ln2_hd = 0.693145751953125f;
    const float ln2_tl = (float)(0.693147180559945309417 - 0.693145751953125);
    const float c7 = (float)(1.0 / 5040.0);
    const float c6 = (float)(1.0 / 720.0);
    const float c5 = (float)(1.0 / 120.0);
    const float c4 = (float)(1.0 / 24.0);
    const float c3 = (float)(1.0 / 6.0);

    if (x < -103.0f) return 0.0f;
    float n = rintf(x * log2e);                 /* nearest, ties to even */
    float r = fmaf(-n, ln2_hd, x);
    r = fmaf(-n, ln2_tl, r);
    float p = c7;
    p = fmaf(p, r, c6);
    p = fmaf(p, r, c5);
    p = fmaf(p, r, c4);
    p = fmaf(p, r, c3);
    p = fmaf(p, r, 0.5f);
    p = fmaf(p, r, 1.0f);
    p = fmaf(p, r, 1.0f);
    int ni = (int)n;
    if (ni > 127) return (p * pow2i(ni - 1)) * 2.0f;
    if (ni < -126) return (p * pow2i(ni + 100)) * pow2i(-100);
    return p * pow2i(ni);
}

/* or_log(x), x a positive normal number: x = 2^e * m with m in
 * [sqrt(1/2), sqrt(2)); log m = 2*atanh(f), f = (m-1)/(m+1), by the odd
 * series 2f + 2f*f^2*(1/3 + f^2/5 + f^4/7 + f^6/9) (the bracket in Horner
 * form in f^2, the leading 2f added last by one fused multiply-add);
 * result = e*ln2_head + (e*ln2_tail + log m). */
float or_log(float x)
{
    const float ln2_hd = 0.693145751953125f;
    const float ln2_tl = (float)(0.693147180559945309417 - 0.693145751953125);
    const float sqrt2  = (float)1.4142135623730950488;
    const float d9 = (float)(1.0 / 9.0);
    const float d7 = (float)(1.0 / 7.0);
    const float d5 = (float)(1.0 / 5.0);
    const float d3 = (float)(1.0 / 3.0);

    uint32_t b = f32_to_bits(x);
    int e = (int)((b >> 23) & 0xffu) - 127;
    float m = bits_to_f32((b & 0x007fffffu) | 0x3f800000u);    /* [1,2) */
    if (m > sqrt2) { m = m * 0.5f; e = e + 1; }
    float f2 = 2.0f * ((m - 1.0f) / (m + 1.0f));      /* 2f, exact doubling */
    float s = f2 * f2 * 0.25f;                           /* f^2 */
    float q = d9;
    q = fmaf(q, s, d7);
    q = fmaf(q, s, d5);
    q = fmaf(q, s, d3);
    float lm = fmaf(f2 * s, q, f2);      /* 2f + 2f*f^2*(1/3 + f^2/5 + ...) */
    float ef = (float)e;
    return fmaf(ef, ln2_hd, fmaf(ef, ln2_tl, lm));
}

/* ------------------------------------------------------------------ */
/* Exact (fp64) LoRA shrink [LoRA Highlights]:                          */
/*   y[m][j] = sum_k x[m][k] * A_{id[m]}[k][j]                          */
/* x bf16 [M][K]; A stored rank-major, at[a][j][k] (a < n_ad, j < r).   */
/* ids == NULL means every token uses adapter 0.  Tokens whose id is    */
/* outside [0, n_ad) get y = 0 and bound = 0.                           */
/* ------------------------------------------------------------------ */

void or_shrink_exact(const uint16_t *x, const uint16_t *at, const int32_t *ids,
                     long n_ad, long M, long K, long r,
                     double *y, double *bound, int nthreads)
{
    #pragma omp parallel for schedule(static) num_threads(nthreads)
    for (long m = 0; m < M; m++) {
        long a = ids ? ids[m] : 0;
        for (long j = 0; j < r; j++) {
            double s = 0.0, b = 0.0;
            if (a >= 0 && a < n_ad) {
                const uint16_t *xr = x + m * K;
                const uint16_t *ar = at + (a * r + j) * K;
                for (long k = 0; k < K; k++) {
                    double p = bf(xr[k]) * bf(ar[k]);
                    s += p;
                    b += fabs(p);
                }
            }
            y[m * r + j] = s;
            if (bound) bound[m * r + j] = b;
        }
    }
}

/* Exact LoRA expand: out[m][n] = prev[m][n] + sum_j bf16(y[m][j]) *
 * B_{id[m]}[j][n], with LoRA-B stored [a][n][j] (K = r contiguous).  y is
 * rounded to bf16 (nearest even) first: the expand consumes bf16 input.
 * prev may be NULL (plain write).  bound = |prev| + sum_j |y_j * b_j|. */
void or_expand_exact(const float *y, const uint16_t *bt, const int32_t *ids,
                     long n_ad, long M, long r, long N, const float *prev,
                     double *out, double *bound, int nthreads)
{
    #pragma omp parallel for schedule(static) num_threads(nthreads)
    for (long m = 0; m < M; m++) {
        long a = ids ? ids[m] : 0;
        double *yb = (double *)malloc(sizeof(double) * (size_t)(r > 0 ? r : 1));
        for (long j = 0; j < r; j++)
            yb[j] = (double)or_bf16_to_f32(or_f32_to_bf16(y[m * r + j]));
        for (long n = 0; n < N; n++) {
            double s = prev ? (double)prev[m * N + n] : 0.0;
            double b = prev ? fabs((double)prev[m * N + n]) : 0.0;
            if (a >= 0 && a < n_ad) {
                const uint16_t *br = bt + (a * N + n) * r;
                for (long j = 0; j < r; j++) {
                    double p = yb[j] * bf(br[j]);
                    s += p;
                    b += fabs(p);
                }
            }
            out[m * N + n] = s;
            if (bound) bound[m * N + n] = b;
        }
        free(yb);
    }
}

/* Exact GEMM [BIO torch.mm; BI locked kernel policy]:
 *   C[m][n] = sum_k A[m][k] * W[n][k]
 * A bf16 [M][K], W bf16 [N][K].  rows == NULL computes every row; else
 * only rows[0..nrows) and C / bound are [nrows][N]. */
void or_gemm_exact(const uint16_t *A, const uint16_t *W, long M, long N, long K,
                   const long *rows, long nrows, double *C, double *bound, int nthreads)
{
    long R = rows ? nrows : M;
    #pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (long i = 0; i < R; i++) {
        long m = rows ? rows[i] : i;
        const uint16_t *ar = A + m * K;
        double *av = (double *)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1));
        for (long k = 0; k < K; k++) av[k] = bf(ar[k]);
        for (long n = 0; n < N; n++) {
            const uint16_t *wr = W + n * K;
            double s = 0.0, b = 0.0;
            for (long k = 0; k < K; k++) {
                double p = av[k] * bf(wr[k]);
                s += p;
                b += fabs(p);
            }
            C[i * N + n] = s;
            if (bound) bound[i * N + n] = b;
        }
        free(av);
    }
}

/* addmm ["Batch Invariant Ops", Highlighted Details: torch.addmm], exact:
 *   C[m][n] = bias[n] + sum_k A[m][k] * W[n][k]
 * bias bf16 [N]; the rest as or_gemm_exact.  bound = |bias| + sum |a*w|. */
void or_addmm_exact(const uint16_t *bias, const uint16_t *A, const uint16_t *W, long M, long N, long K,
                    const long *rows, long nrows, double *C, double *bound, int nthreads)
{
    or_gemm_exact(A, W, M, N, K, rows, nrows, C, bound, nthreads);
    long R = rows ? nrows : M;
    for (long i = 0; i < R; i++)
        for (long n = 0; n < N; n++) {
            C[i * N + n] += bf(bias[n]);
            if (bound) bound[i * N + n] += fabs(bf(bias[n]));
        }
}

/* Segment build: stable counting sort of token indices by adapter id.
 * offsets[a] = number of tokens with id < a (offsets[n_ad] = number of
 * tokens with a valid id); perm[offsets[a] + i] = the i-th token, in
 * increasing token order, whose id is a.  Invalid ids are left out. */
void or_segment(const int32_t *ids, long M, int n_ad, int32_t *perm, int32_t *offsets)
{
    long *count = (long *)calloc((size_t)n_ad + 1, sizeof(long));
    for (long t = 0; t < M; t++)
        if (ids[t] >= 0 && ids[t] < n_ad) count[ids[t]]++;
    long run = 0;
    for (int a = 0; a < n_ad; a++) { offsets[a] = (int32_t)run; run += count[a]; }
    offsets[n_ad] = (int32_t)run;
    for (int a = 0; a < n_ad; a++) count[a] = offsets[a];
    for (long t = 0; t < M; t++)
        if (ids[t] >= 0 && ids[t] < n_ad) perm[count[ids[t]]++] = (int32_t)t;
    free(count);
}

/* ------------------------------------------------------------------ */
/* Decode attention with a fixed-size KV split ["Restoring AI           */
/* Reproducibility", 2-3 (attention) and 3-2 (fixed-size split)].       */
/* One query row per (sequence b, query head h); the kv head is          */
/* h / (Hq / Hkv).  q bf16 [B][Hq][D]; k, v bf16 [B][Hkv][Lmax][D];     */
/* lens int32 [B]; out [B][Hq][D].                                       */
/* ------------------------------------------------------------------ */

/* Exact: out = softmax(scale * q.k_j)_j . v_j over j < lens[b], in
 * double; a sequence of length 0 gives 0. */
void or_attn_decode_exact(const uint16_t *q, const uint16_t *k, const uint16_t *v, const int32_t *lens,
                          long B, long Hq, long Hkv, long D, long Lmax, double scale, double *out, int nthreads)
{
    #pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (long bh = 0; bh < B * Hq; bh++) {
        long b = bh / Hq, h = bh % Hq, hk = h / (Hq / Hkv), L = lens[b];
        const uint16_t *qr = q + bh * D;
        const uint16_t *kb = k + (b * Hkv + hk) * Lmax * D;
        const uint16_t *vb = v + (b * Hkv + hk) * Lmax * D;
        double *o = out + bh * D;
        for (long d = 0; d < D; d++) o[d] = 0.0;
        if (L <= 0) continue;
        double *s = (double *)malloc(sizeof(double) * (size_t)L);
        double m = -INFINITY;
        for (long j = 0; j < L; j++) {
            double t = 0.0;
            for (long d = 0; d < D; d++) t += bf(qr[d]) * bf(kb[j * D + d]);
            s[j] = scale * t;
            if (s[j] > m) m = s[j];
        }
        double den = 0.0;
        for (long j = 0; j < L; j++) { s[j] = exp(s[j] - m); den += s[j]; }
        for (long j = 0; j < L; j++)
            for (long d = 0; d < D; d++) o[d] += s[j] * bf(vb[j * D + d]);
        for (long d = 0; d < D; d++) o[d] /= den;
        free(s);
    }
}

/* Perfect binary tree over n = 2^k fp32 values (stride apart), pairs
 * (0,1), (2,3), ... first: the frame sums of the attention below. */
static float or_frame_tree(float *v, long n)
{
    for (long w = 1; w < n; w *= 2)
        for (long i = 0; i + w < n; i += 2 * w) v[i] = v[i] + v[i + w];
    return v[0];
}

/* Canonical fp32 order.  Chunk c holds keys [256c, 256c + 256) as a frame
 * of 256 slots; slots past the sequence's length hold p = 0 and add +0.
 *   s_j  = fl(fl(perfect tree over d of q_d * k_jd) * scale)  (the
 *          products of two bf16 values are exact in fp32; D = 2^k)
 *   m_c  = max of s_j over the chunk's keys
 *   p_j  = or_exp(fl(s_j - m_c))
 *   l_c  = perfect tree over the 256 slots of p_j
 *   o_cd = perfect tree over the 256 slots of fl(p_j * v_jd)
 * Combine over the n = ceil(L / 256) chunks, padded to the next power of
 * two P with zero chunks:
 *   M = max_c m_c;  a_c = or_exp(fl(m_c - M))
 *   l = perfect tree over P of fl(a_c * l_c);  O_d = same of fl(a_c * o_cd)
 *   out_d = fl(O_d / l)
 * Every order is fixed by the sequence's own length, never by the batch or
 * by how chunks are shared among workers. */
void or_attn_decode_canon(const uint16_t *q, const uint16_t *k, const uint16_t *v, const int32_t *lens,
                          long B, long Hq, long Hkv, long D, long Lmax, float scale, float *out, int nthreads)
{
    #pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (long bh = 0; bh < B * Hq; bh++) {
        long b = bh / Hq, h = bh % Hq, hk = h / (Hq / Hkv), L = lens[b];
        const uint16_t *qr = q + bh * D;
        const uint16_t *kb = k + (b * Hkv + hk) * Lmax * D;
        const uint16_t *vb = v + (b * Hkv + hk) * Lmax * D;
        float *o = out + bh * D;
        for (long d = 0; d < D; d++) o[d] = 0.0f;
        if (L <= 0) continue;
        long n = (L + 255) / 256, P = 1;
        while (P < n) P *= 2;
        float *mc = (float *)calloc((size_t)P, sizeof(float));
        float *lc = (float *)calloc((size_t)P, sizeof(float));
        float *oc = (float *)calloc((size_t)(P * D), sizeof(float));
        float *tmp = (float *)malloc(sizeof(float) * (size_t)(D > 256 ? D : 256));
        float *pj = (float *)malloc(sizeof(float) * 256);
        for (long c = 0; c < n; c++) {
            long j0 = 256 * c, nj = L - j0 < 256 ? L - j0 : 256;
            float m = -INFINITY;
            float s[256];
            for (long i = 0; i < nj; i++) {
                for (long d = 0; d < D; d++) tmp[d] = or_bf16_to_f32(qr[d]) * or_bf16_to_f32(kb[(j0 + i) * D + d]);
                s[i] = or_frame_tree(tmp, D) * scale;
                if (s[i] > m) m = s[i];
            }
            mc[c] = m;
            for (long i = 0; i < 256; i++) pj[i] = i < nj ? or_exp(s[i] - m) : 0.0f;
            for (long i = 0; i < 256; i++) tmp[i] = pj[i];
            lc[c] = or_frame_tree(tmp, 256);
            for (long d = 0; d < D; d++) {
                for (long i = 0; i < 256; i++) tmp[i] = i < nj ? pj[i] * or_bf16_to_f32(vb[(j0 + i) * D + d]) : 0.0f;
                oc[c * D + d] = or_frame_tree(tmp, 256);
            }
        }
        float M = mc[0];
        for (long c = 1; c < n; c++) if (mc[c] > M) M = mc[c];
        float *ac = (float *)calloc((size_t)P, sizeof(float));
        for (long c = 0; c < n; c++) ac[c] = or_exp(mc[c] - M);
        float *col = (float *)malloc(sizeof(float) * (size_t)P);
        for (long c = 0; c < P; c++) col[c] = ac[c] * lc[c];
        float l = or_frame_tree(col, P);
        for (long d = 0; d < D; d++) {
            for (long c = 0; c < P; c++) col[c] = ac[c] * oc[c * D + d];
            o[d] = or_frame_tree(col, P) / l;
        }
        free(col); free(ac); free(pj); free(tmp); free(oc); free(lc); free(mc);
    }
}

/* ------------------------------------------------------------------ */
/* RMSNorm ["Restoring AI Reproducibility" 2-3, 3-1]                    */
/* ------------------------------------------------------------------ */

/* Exact: y = x * w / sqrt(mean(x^2) + eps), in double. */
void or_rmsnorm_exact(const uint16_t *x, const uint16_t *w, long R, long n,
                      double eps, double *y, int nthreads)
{
    #pragma omp parallel for schedule(static) num_threads(nthreads)
    for (long i = 0; i < R; i++) {
        const uint16_t *xr = x + i * n;
        double ss = 0.0;
        for (long k = 0; k < n; k++) ss += bf(xr[k]) * bf(xr[k]);
        double inv = 1.0 / sqrt(ss / (double)n + eps);
        for (long k = 0; k < n; k++) y[i * n + k] = bf(xr[k]) * inv * bf(w[k]);
    }
}

/* Canonical fp32 scale of one row: S = canon_sum(x^2; T=512, V=8)
 * (x^2 is exact in fp32 for bf16 x); ms = S/n; inv = 1/sqrt(ms + eps)
 * with IEEE sqrt and division (no reciprocal-sqrt approximation). */
float or_rmsnorm_inv_canon(const uint16_t *xr, long n, float eps)
{
    float *sq = (float *)malloc(sizeof(float) * (size_t)(n > 0 ? n : 1));
    for (long k = 0; k < n; k++) {
        float v = or_bf16_to_f32(xr[k]);
        sq[k] = v * v;
    }
    float S = or_canon_sum(sq, n, 512, 8);
    free(sq);
    float ms = S / (float)n;
    return 1.0f / sqrtf(ms + eps);
}

/* Canonical fp32 RMSNorm: y = bf16(fl(fl(x * inv) * w)). */
void or_rmsnorm_canon(const uint16_t *x, const uint16_t *w, long R, long n,
                      float eps, uint16_t *y, int nthreads)
{
    #pragma omp parallel for schedule(static) num_threads(nthreads)
    for (long i = 0; i < R; i++) {
        const uint16_t *xr = x + i * n;
        float inv = or_rmsnorm_inv_canon(xr, n, eps);
        for (long k = 0; k < n; k++) {
            float v = or_bf16_to_f32(xr[k]) * inv;
            y[i * n + k] = or_f32_to_bf16(v * or_bf16_to_f32(w[k]));
        }
    }
}

/* ------------------------------------------------------------------ */
/* log_softmax ["Batch Invariant Ops", Highlighted Details]             */
/* ------------------------------------------------------------------ */

/* Exact: out = (x - max) - log(sum exp(x - max)), in double. */
void or_log_softmax_exact(const float *x, long R, long n, double *out, int nthreads)
{
    #pragma omp parallel for schedule(static) num_threads(nthreads)
    for (long i = 0; i < R; i++) {
        const float *xr = x + i * n;
        double m = xr[0];
        for (long k = 1; k < n; k++) if (xr[k] > m) m = xr[k];
        double s = 0.0;
        for (long k = 0; k < n; k++) s += exp((double)xr[k] - m);
        double L = log(s);
        for (long k = 0; k < n; k++) out[i * n + k] = ((double)xr[k] - m) - L;
    }
}

/* Canonical fp32, two passes: m = row max (exact in any order);
 * d_k = x_k - m; S = canon_sum(or_exp(d_k); T=4096, V=4); L = or_log(S);
 * out_k = d_k - L. */
void or_log_softmax_canon(const float *x, long R, long n, float *out, int nthreads)
{
    #pragma omp parallel for schedule(static) num_threads(nthreads)
    for (long i = 0; i < R; i++) {
        const float *xr = x + i * n;
        float m = xr[0];
        for (long k = 1; k < n; k++) if (xr[k] > m) m = xr[k];
        float *e = (float *)malloc(sizeof(float) * (size_t)n);
        for (long k = 0; k < n; k++) e[k] = or_exp(xr[k] - m);
        float S = or_canon_sum(e, n, 4096, 4);
        float L = or_log(S);
        for (long k = 0; k < n; k++) out[i * n + k] = (xr[k] - m) - L;
        free(e);
    }
}

/* ------------------------------------------------------------------ */
/* mean over the last dimension ["Batch Invariant Ops"]                 */
/* ------------------------------------------------------------------ */

void or_mean_exact(const float *x, long R, long n, double *out, int nthreads)
{
    #pragma omp parallel for schedule(static) num_threads(nthreads)
    for (long i = 0; i < R; i++) {
        double s = 0.0;
        for (long k = 0; k < n; k++) s += x[i * n + k];
        out[i] = s / (double)n;
    }
}

/* Canonical fp32: canon_sum(x; T=1024, V=4) / n. */
void or_mean_canon(const float *x, long R, long n, float *out, int nthreads)
{
    #pragma omp parallel for schedule(static) num_threads(nthreads)
    for (long i = 0; i < R; i++)
        out[i] = or_canon_sum(x + i * n, n, 1024, 4) / (float)n;
}

int or_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
