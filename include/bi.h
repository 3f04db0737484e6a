/*
 * bi.h -- C ABI of libbi.so: reduction kernels whose floating-point
 * summation order is fixed, so results are bitwise identical across replays,
 * batch sizes (M), split counts, emulated tensor-parallel shard counts and
 * the position of a row inside a tile.  NVIDIA B200 (sm_100a) only.
 *
 * Sources of the operations (page title, section):
 *   [LoRA] "Reproducible LoRA Inference Through Deterministic Split-K
 *          Reduction", Highlights / Q&A -- split-K LoRA shrink whose
 *          partials are combined by fp32 atomics (nondeterministic) or in a
 *          fixed order (deterministic); unsplit reduction as the baseline.
 *   [TBIK] "Deterministic Inference across Tensor Parallel Sizes That
 *          Eliminates Training-Inference Mismatch", Abstract -- one
 *          hierarchical binary tree orders intra- and inter-GPU reduction.
 *   [BI]   "The biggest Mystery of LLMs have just been solved", Detailed
 *          Analysis / Batch-Variant vs. Batch-Invariant -- locked kernel
 *          policy, deterministic reduction tree; "Restoring AI
 *          Reproducibility", 2-3 / 3-1 / 3-2 -- RMSNorm and matmul reduced
 *          in an order that does not depend on the batch.
 *   [BIO]  "Batch Invariant Ops", Highlighted Details -- mm, log_softmax,
 *          mean.
 *
 * Conventions shared by every entry point
 *   - Every pointer is DEVICE memory owned by the caller, unless stated.
 *     The library allocates no device memory on any call; a caller-sized
 *     workspace is passed where one is needed.
 *   - bf16 arrays are passed as `const void*` (IEEE bfloat16, 2 bytes).
 *     Row-major throughout.  Weights are stored K-contiguous, the
 *     (out_features x in_features) layout of a linear layer:
 *       LoRA A  : [r][K]      (so y = x . A^T-storage = x . A)
 *       GEMM W  : [N][K]      (C = A . W^T)
 *       LoRA B  : [N][r]
 *   - Pointers of vector-loaded arrays must be 16-byte aligned.
 *   - Calls are asynchronous on `stream` (NULL = legacy default stream).
 *     Argument errors are detected on the host before anything is launched
 *     and returned at once; nothing is written then.  Errors seen inside a
 *     kernel (a bounded wait that ran out) are recorded in a device status
 *     word that bi_get_device_status() reads.
 *   - fp32 sums follow the canonical tree: tree(v[0..n)) = v[0] for n = 1,
 *     else fl(tree(v[0..h)) + tree(v[h..n))) with h = ceil(n/2).
 */
#ifndef BI_H
#define BI_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream, without pulling in CUDA headers. */
typedef struct CUstream_st *bi_stream_t;

typedef enum {
    BI_OK = 0,
    BI_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad enum  */
    BI_ERR_UNSUPPORTED_SHAPE = 2, /* shape / split / alignment not handled  */
    BI_ERR_WORKSPACE = 3,         /* workspace missing or too small         */
    BI_ERR_CUDA = 4,              /* a CUDA runtime call failed             */
    BI_ERR_TIMEOUT = 5,           /* a bounded device wait ran out          */
    BI_ERR_NO_DEVICE = 6          /* no sm_100 device current               */
} bi_status;

typedef enum {
    BI_SHRINK_UNSPLIT = 0,  /* one CTA owns all of K for its rows          */
    BI_SHRINK_ATOMIC = 1,   /* split-K, partials added with fp32 atomicAdd
                               in arrival order: NONDETERMINISTIC, kept only
                               to reproduce the variation [LoRA Highlights] */
    BI_SHRINK_TREE = 2      /* split-K, partials combined by the canonical
                               tree inside a thread-block cluster          */
} bi_shrink_mode;

/* ------------------------------------------------------------------ */
/* LoRA shrink [LoRA]:  y[m][j] = sum_k x[m][k] * A[j][k]               */
/*                                                                      */
/* x  bf16 [M][K]; A bf16 [r][K]; y fp32 [M][r] (written).              */
/* K is cut into leaves of 64; each leaf is one tensor-core MMA chain   */
/* started from zero; the K/64 leaves are combined by the canonical     */
/* tree in fp32 (round to nearest).  `splits` CTAs share the K range of */
/* a row tile, each owning a contiguous power-of-two block of leaves =  */
/* one subtree, so in modes UNSPLIT and TREE the result is bitwise the  */
/* same for every M, every splits value and every replay.  ATOMIC adds  */
/* the per-split subtree values with atomicAdd after zeroing y itself.  */
/* Requirements: K % 64 == 0, r % 8 == 0, 8 <= r <= 128, splits a power */
/* of two in [1, 16] dividing K/64 (mode UNSPLIT takes splits = 1),     */
/* x, A 16-byte aligned.  M == 0 is a no-op.                            */
/* ------------------------------------------------------------------ */
bi_status bi_lora_shrink(const void *x, const void *A, float *y,
                         int M, int K, int r, int splits, int mode,
                         bi_stream_t stream);

/* ------------------------------------------------------------------ */
/* Multi-adapter (segmented) LoRA.  A plan groups tokens by adapter:    */
/* a stable counting sort of the token indices by adapter id.          */
/*                                                                      */
/* bi_lora_plan_bytes(M, n_adapters): bytes of plan memory needed.      */
/* bi_lora_plan: ids int32 [M] (device) -> plan (device, caller-owned,  */
/*   at least bi_lora_plan_bytes bytes, 16-byte aligned).  Tokens whose */
/*   id is outside [0, n_adapters) (e.g. -1 = "no adapter") form a last */
/*   segment: their shrink output row is zero and the expand leaves     */
/*   their output row as it was (accumulate) or zero (write).           */
/*   Plan layout (int32): perm[M] (token indices, grouped by adapter,   */
/*   increasing within a group), then offsets[n_adapters + 2] where     */
/*   segment a is perm[offsets[a] .. offsets[a+1]), a = n_adapters being */
/*   the "no adapter" segment; then zero padding up to a multiple of 4  */
/*   words, then a tile table of ceil(M/64) + n_adapters + 1 records of */
/*   68 words, one per 64-row tile of the segments in order: {adapter,  */
/*   rows (1..64), first perm position, 0, token ids[64] (-1 past      */
/*   rows)}; records past the last tile have adapter -1.  The segmented */
/*   kernels read their tile's adapter and rows from one record.       */
/*   1 <= n_adapters <= 256.                                            */
/* ------------------------------------------------------------------ */
size_t bi_lora_plan_bytes(int M, int n_adapters);
bi_status bi_lora_plan(const int32_t *ids, int M, int n_adapters,
                       void *plan, size_t plan_bytes, bi_stream_t stream);

/* Segmented shrink: y[t][j] = sum_k x[t][k] * A_{id[t]}[j][k].
 * A bf16 [n_adapters][r][K]; other arguments and guarantees as
 * bi_lora_shrink (row t of y is bitwise the value bi_lora_shrink gives for
 * that row alone with adapter id[t]'s A, in modes UNSPLIT and TREE). */
bi_status bi_lora_shrink_segmented(const void *x, const void *A, const void *plan,
                                   int n_adapters, float *y, int M, int K, int r,
                                   int splits, int mode, bi_stream_t stream);

/* Segmented shrink for callers that cannot allocate device memory.  The
 * paper has no counterpart: this is a convenience of this library.  Some
 * callers cannot call cudaMalloc -- a plugin inside a host application that
 * owns all device memory through its own pool and lets no library allocate,
 * or a latency-critical loop where an allocation (which may synchronise the
 * device) is not acceptable.  This call takes the adapter ids (int32 [M],
 * device) instead of a plan and builds the plan in a fixed array of the
 * library's own device memory, sized for BI_NOALLOC_MAX_TOKENS tokens and
 * 256 adapters (152,904 int32, about 598 KiB), held by every GPU that loads
 * the library until the process exits.
 * It allocates nothing.  Other arguments, results and guarantees are those of
 * bi_lora_plan followed by bi_lora_shrink_segmented (same bits).
 * M > BI_NOALLOC_MAX_TOKENS or n_adapters > 256 returns
 * BI_ERR_UNSUPPORTED_SHAPE before any work.  The first call on a device looks
 * up the array's device address (cudaGetSymbolAddress) and caches it; make
 * that first call before any stream capture.  All calls share the one array,
 * so calls whose kernels overlap on the GPU (different streams or threads)
 * race on it and must be serialised by the caller. */
#define BI_NOALLOC_MAX_TOKENS 65536
bi_status bi_lora_shrink_segmented_noalloc(const void *x, const void *A, const int32_t *ids,
                                           int n_adapters, float *y, int M, int K, int r,
                                           int splits, int mode, bi_stream_t stream);

/* Fused segmented LoRA [LoRA Q&A: the two low-rank products]: the      */
/* segmented shrink (split-K `splits` in mode TREE, or UNSPLIT when      */
/* splits = 1) and then out[t] (+)= bf16(y[t]) . B_{id[t]}^T, in one     */
/* launch.  y stays on chip (the CTAs of a row tile share it through     */
/* distributed shared memory); it is also written to y when y != NULL.   */
/* Bitwise the same as bi_lora_shrink_segmented followed by              */
/* bi_lora_expand_segmented.  B bf16 [n_adapters][N][r]; out fp32 [M][N] */
/* (16-byte aligned); N % 8 == 0; plan from bi_lora_plan; other          */
/* requirements as those two calls.  Mode ATOMIC has no fused form.      */
bi_status bi_lora_fused(const void *x, const void *A, const void *B, const void *plan,
                        int n_adapters, float *y, float *out, int M, int K, int r, int N,
                        int splits, int accumulate, bi_stream_t stream);

/* ------------------------------------------------------------------ */
/* LoRA expand [LoRA Q&A: the second low-rank product]:                 */
/*   e[t][n] = sum_j bf16(y[t][j]) * B[n][j]                            */
/*   out[t][n] = accumulate ? fl(out[t][n] + e[t][n]) : e[t][n]         */
/* y fp32 [M][r] (rounded to bf16, nearest even, on load); B bf16       */
/* [N][r]; out fp32 [M][N].  K = r is one MMA chain, no split, so each   */
/* output element is computed the same way at every M.                  */
/* Requirements: r % 8 == 0, 8 <= r <= 128, N % 8 == 0, pointers        */
/* 16-byte aligned.                                                     */
/* ------------------------------------------------------------------ */
bi_status bi_lora_expand(const float *y, const void *B, float *out,
                         int M, int r, int N, int accumulate, bi_stream_t stream);

/* Segmented expand: B bf16 [n_adapters][N][r]; plan from bi_lora_plan  */
/* (16-byte aligned, else BI_ERR_UNSUPPORTED_SHAPE).  A CTA reads its 64  */
/* rows' adapter and token ids from one record of the plan's tile table. */
bi_status bi_lora_expand_segmented(const float *y, const void *B, const void *plan,
                                   int n_adapters, float *out, int M, int r, int N,
                                   int accumulate, bi_stream_t stream);

/* ------------------------------------------------------------------ */
/* Batch-invariant GEMM [BI locked kernel policy; BIO torch.mm]:        */
/*   C[m][n] = sum_k A[m][k] * W[n][k]                                  */
/* A bf16 [M][K], W bf16 [N][K]; C fp32 [M][N] (c_bf16 = 0) or bf16     */
/* (c_bf16 = 1, round to nearest even from the fp32 accumulator).       */
/* One locked tcgen05 reduction order (K stepped 0 -> K in 64-wide     */
/* stages, one fp32 TMEM accumulator per element, never split) whatever */
/* M is, so row m of C is bitwise the same for every M.  The output     */
/* tile is 128 x 256, or 128 x 64 / 128 x 32 when M <= 512 / M <= 128 so */
/* that small batches still spread the weight read; the accumulation of */
/* an element does not depend on the tile width.  Requirements: K % 64  */
/* == 0, N % 16 == 0, A / W / C 16-byte aligned.                        */
/* ------------------------------------------------------------------ */
bi_status bi_gemm(const void *A, const void *W, void *C, int M, int N, int K,
                  int c_bf16, bi_stream_t stream);

/* Batch-invariant addmm ["Batch Invariant Ops", Highlighted Details:     */
/* torch.addmm]:  C[m][n] = fl(acc[m][n] + bias[n]), acc being bi_gemm's */
/* fp32 accumulator (same tiles, same K order), so C is bitwise bi_gemm's */
/* fp32 result plus the bias in one IEEE fp32 addition, then the optional */
/* bf16 rounding (c_bf16 = 1).  bias bf16 [N] (device, 16-byte aligned); */
/* everything else as bi_gemm.                                           */
bi_status bi_addmm(const void *bias, const void *A, const void *W, void *C, int M, int N, int K,
                   int c_bf16, bi_stream_t stream);

/* ------------------------------------------------------------------ */
/* TP-invariant tree GEMM [TBIK Abstract]: C = A . W^T with K cut into  */
/* leaves of 256; each leaf is one tensor-core MMA chain from zero; the */
/* leaves are combined by the canonical fp32 tree.  `shards` emulates a */
/* row-parallel tensor-parallel split of K on one GPU: shard s owns the */
/* contiguous leaves [s*L/shards, (s+1)*L/shards) -- one subtree -- and */
/* writes its partial; bi_tree_combine then adds the top log2(shards)   */
/* levels.  The result is bitwise the same for shards = 1, 2, 4, 8, 16. */
/*                                                                      */
/* bi_gemm_tree_partials: partials fp32 [shards][M][N].                */
/* bi_gemm_tree: C fp32 [M][N]; workspace of                            */
/*   bi_gemm_tree_ws_bytes(M, N, shards) bytes for the partials (at     */
/*   least four, so that a shard of 32 or 64 leaves can be folded as    */
/*   power-of-two subtrees of 16 leaves and combined: same bits, faster */
/*   layout).  shards = 1 also runs without a workspace (ws = NULL),    */
/*   folding all leaves in one partial; shards > 1 needs at least       */
/*   shards * M * N * 4 bytes.                                          */
/* Requirements: K % 256 == 0, shards a power of two dividing K/256,    */
/* N % 64 == 0, pointers 16-byte aligned.                               */
/* ------------------------------------------------------------------ */
size_t bi_gemm_tree_ws_bytes(int M, int N, int shards);
bi_status bi_gemm_tree_partials(const void *A, const void *W, float *partials,
                                int M, int N, int K, int shards, bi_stream_t stream);
bi_status bi_gemm_tree(const void *A, const void *W, float *C, int M, int N, int K,
                       int shards, void *ws, size_t ws_bytes, bi_stream_t stream);

/* Cross-shard combine [TBIK]: out[i] = tree(partials[0][i], ...,
 * partials[s-1][i]).  partials fp32 [s][count], out fp32 [count].
 * s in [1, 64]; both pointers 16-byte aligned. */
bi_status bi_tree_combine(const float *partials, float *out, int s, size_t count,
                          bi_stream_t stream);

/* Cross-GPU combine [TBIK Abstract: the inter-GPU reduction follows the  */
/* same tree]: out[i] = tree(partials[0][i], ..., partials[s-1][i]) for   */
/* i in [begin, begin + count), the same tree as bi_tree_combine.         */
/* partials: a HOST array of s device pointers, each to an fp32 [total]   */
/* partial that this device can load from -- its own memory or a peer     */
/* GPU's (peer access or CUDA IPC / symmetric memory); the kernel reads    */
/* them with plain loads (no multicast) and writes out[begin ..) of its    */
/* own memory.  A rank that combines only its share [begin, begin+count)  */
/* gives a reduce-scatter; every rank combining everything, an all-reduce */
/* in the canonical order.  The caller orders the partials' writes before */
/* the call on every GPU (a barrier) and keeps them alive until the call  */
/* has finished on every GPU.  s in [1, 64]; begin and count multiples of */
/* 4; every pointer 16-byte aligned, else BI_ERR_UNSUPPORTED_SHAPE.       */
bi_status bi_tree_combine_peers(const float *const *partials, int s, float *out, size_t begin,
                                size_t count, bi_stream_t stream);

/* ------------------------------------------------------------------ */
/* Batch-invariant row operations, one CTA (or one cluster) per row, so  */
/* row i's bits never depend on how many rows there are.  The row sum S */
/* is canonical: T logical lanes, lane t adds (from +0, in order) the V */
/* elements of vectors t, t+T, t+2T, ...; the T lane values are then    */
/* combined by the canonical tree.                                      */
/* ------------------------------------------------------------------ */

/* RMSNorm ["Restoring AI Reproducibility" 2-3, 3-1]: T = 512, V = 8.
 * S = canonical sum of x^2, inv = 1 / sqrt(S/n + eps) (IEEE sqrt and
 * division), y = bf16(fl(fl(x * inv) * w)).  x, y bf16 [rows][n]; w bf16
 * [n].  n % 8 == 0, 8 <= n <= 32768. */
bi_status bi_rmsnorm(const void *x, const void *w, void *y, int rows, int n,
                     float eps, bi_stream_t stream);

/* log_softmax [BIO]: T = 4096, V = 4.  m = row max; d = x - m;
 * S = canonical sum of bi_exp(d); L = bi_log(S); out = fl(d - L).
 * bi_exp / bi_log are the library's own written methods (Cody-Waite +
 * Taylor; atanh series), bitwise reproducible on any IEEE machine.
 * x, out fp32 [rows][n]; n % 4 == 0, 4 <= n <= 262144. */
bi_status bi_log_softmax(const float *x, float *out, int rows, int n, bi_stream_t stream);

/* mean over the last dimension [BIO]: T = 1024, V = 4; out[i] = fl(S/n).
 * x fp32 [rows][n]; out fp32 [rows]; n % 4 == 0. */
bi_status bi_mean(const float *x, float *out, int rows, int n, bi_stream_t stream);

/* The library's exp (which = 0) or log (which = 1) of bi_log_softmax,
 * applied elementwise: y[i] = bi_exp(x[i]) or bi_log(x[i]).  x, y fp32 [n].
 * bi_log is defined for positive normal x; bi_exp for x <= 88.  which = 2
 * runs the shortcut of bi_exp that log_softmax takes for -87 <= x <= 88
 * (same bits as bi_exp there; undefined outside); which = 3 the same
 * shortcut on packed two-lane fp32 instructions (elements 2k and 2k+1 form
 * one pair).  Other values of which: BI_ERR_INVALID_ARG. */
bi_status bi_math_spec(const float *x, float *y, size_t n, int which, bi_stream_t stream);

/* ------------------------------------------------------------------ */
/* Batch-invariant decode attention with a fixed-size KV split          */
/* ["Restoring AI Reproducibility", 2-3 and 3-2].  One query row per    */
/* (sequence b, query head h) attends to keys [0, lens[b]) of kv head   */
/* h / (Hq / Hkv):  out = softmax(scale * q . k_j) . v_j.  The keys are */
/* cut into chunks of 256 slots whatever the batch; every sum is a      */
/* perfect tree (the dot product over D; the 256 slots of a chunk, zero */
/* past the length; the chunks, padded to a power of two), exp is       */
/* bi_math_spec's, so row (b, h) is bitwise the same for any batch,     */
/* position, Lmax or number of CTAs.  The exact order:                  */
/*   s_j = fl(fl(tree_d q_d k_jd) * scale); m_c = chunk max;            */
/*   p_j = exp(fl(s_j - m_c)); l_c = tree p_j; o_cd = tree fl(p_j v_jd);*/
/*   M = max m_c; a_c = exp(fl(m_c - M)); l = tree fl(a_c l_c);         */
/*   O_d = tree fl(a_c o_cd); out_d = fl(O_d / l); lens[b] = 0 gives 0. */
/* q bf16 [B][Hq][D]; k, v bf16 [B][Hkv][Lmax][D]; lens int32 [B] with  */
/* 0 <= lens[b] <= Lmax (longer lengths are cut at Lmax); out fp32      */
/* [B][Hq][D].  D in {64, 128, 256}; Hq / Hkv in {1, 2, 4, 8}; q, k, v, */
/* out 16-byte aligned.  ws: bi_attn_decode_ws_bytes(B, Hq, D, Lmax)    */
/* bytes of caller memory for the chunk partials.                       */
/* ------------------------------------------------------------------ */
size_t bi_attn_decode_ws_bytes(int B, int Hq, int D, int Lmax);
bi_status bi_attn_decode(const void *q, const void *k, const void *v, const int32_t *lens,
                         float *out, int B, int Hq, int Hkv, int D, int Lmax, float scale,
                         void *ws, size_t ws_bytes, bi_stream_t stream);

/* ------------------------------------------------------------------ */
/* Status                                                               */
/* ------------------------------------------------------------------ */

/* Synchronises `stream`, then returns and clears the device status word of
 * the current device (BI_OK if no kernel recorded an error). */
bi_status bi_get_device_status(bi_stream_t stream);

/* Human-readable name of a status code (static string). */
const char *bi_status_string(int status);

/* Test-only fault injection on the host side.  With fault_code =
 * BI_FAULT_SKIP_STAGE every following bi_gemm / bi_addmm call runs with the
 * TMA producer of its first CTA leaving the first K stage unloaded: the MMA
 * issuer's bounded wait on that stage runs out, the kernel records
 * BI_ERR_TIMEOUT, waits (bounded) for every load and MMA it did issue, frees
 * its tensor memory and returns, so the context stays usable.  While a
 * fault is set the kernels' waits give up after 10 ms instead of 2 s.
 * fault_code = 0 (BI_FAULT_NONE) turns it off.  No GPU fault is involved. */
#define BI_FAULT_NONE 0
#define BI_FAULT_SKIP_STAGE 1
void bi_debug_set_fault(int fault_code);

/* Self-test of the bounded-wait machinery: launches one CTA that waits on
 * a flag nothing sets, giving up after `max_polls` polls; the kernel then
 * records BI_ERR_TIMEOUT in the device status word and returns.  Used to
 * check failure reporting without hanging or faulting the GPU. */
bi_status bi_selftest_bounded_wait(int max_polls, bi_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* BI_H */
