/*
 * xattn.h - C ABI of libxattn.so: XAttention block-sparse prefill attention on
 * NVIDIA B200 (sm_100a).
 *
 * The three steps of the method, one entry point each:
 *   xattn_score        strided antidiagonal block scoring
 *   xattn_select       per-head threshold block selection -> CSR kept lists
 *   xattn_sparse_attn  softmax attention restricted to the kept key blocks
 * plus xattn_dense_attn (every block kept: the dense baseline) and helpers.
 *
 * Sources (page title, section):
 *   [DuSA-Q2]  DuSA rebuttal (paperhub tM5mjMfFmS), "Response to Q2": Q and K of
 *              size (B, H, M, C) are reshaped to (B, H, M//stride, stride*C) and
 *              attention with a softmax over the last two dimensions is computed.
 *   [XA-abs]   XAttention abstract (arXiv 2503.16428): block importance is the sum
 *              of antidiagonal values, lower-left to upper-right.
 *   [XA-app]   XAttention summary (atlas.scime.ai), "Approach": strided
 *              antidiagonal sums inside each block; keep the minimal set of blocks
 *              whose softmax-normalised antidiagonal mass exceeds a per-head
 *              threshold.
 *   [FP-RQ3]   FlexPrefill rebuttal (paperhub OfjIlbelrT), "R Q3": the minimal
 *              set reaching a cumulative threshold is taken in descending order.
 *   [DuSA-W3]  DuSA rebuttal, "Response to W3" / "Response to Q1": sparse
 *              attention is then performed within the important blocks only.
 *   [XA-abl]   XAttention summary, "Measured effects" table: antidiagonal vs
 *              diagonal scoring; threshold selection vs Top K and fixed Ratio.
 *
 * Conventions shared by every entry point:
 *   - Tensors are device memory owned by the caller, dense and row-major, in the
 *     layouts stated per argument. Q, K, V, O must be 16-byte aligned. The
 *     library never allocates or frees device memory; workspaces are sized by
 *     the *_workspace_size functions and passed in.
 *   - bf16 tensors are passed as `const void*` (IEEE bfloat16, 2 bytes).
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). Calls are
 *     asynchronous on that stream and never synchronise, except
 *     xattn_get_device_error.
 *   - Argument errors are detected on the host before any launch and return
 *     XATTN_EINVAL (bad value) or XATTN_EUNSUPPORTED (valid but not built);
 *     nothing is launched then. A failed launch returns XATTN_ECUDA.
 *   - Conditions only the device can see (kept-list capacity, a bounded wait
 *     that ran out) set a per-device error word read by xattn_get_device_error.
 *   - An empty problem (B, H or M equal to 0) returns XATTN_OK and launches
 *     nothing.
 *   - Supported: block = 128; stride in {1, 2, 4, 8, 16, 32, 64}; C in {64, 128};
 *     M a multiple of 128; Hq a multiple of Hkv.
 */
#ifndef XATTN_H
#define XATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define XATTN_API __attribute__((visibility("default")))
#else
#define XATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  XATTN_OK = 0,
  XATTN_EINVAL = 1,       /* bad argument (null/misaligned pointer, bad shape) */
  XATTN_ECAPACITY = 2,    /* col_capacity below the number of kept blocks      */
  XATTN_ECUDA = 3,        /* a CUDA runtime call or launch failed               */
  XATTN_ETIMEOUT = 4,     /* a bounded device-side wait ran out                 */
  XATTN_EUNSUPPORTED = 5  /* valid arguments this build has no kernel for       */
} xattn_status;

/* Static English description of a status code (never NULL). */
XATTN_API const char* xattn_status_string(int status);

/* Library ABI version (major*100 + minor); 200 since the workspace-size
 * functions take the causal flag. */
XATTN_API int xattn_version(void);

/*
 * Workspace bytes xattn_score needs for the given `causal` flag: one fp32
 * partial log-mass per (reshaped row, key block the row can see) plus one fp32
 * log-sum-exp per reshaped row. With rp = M/stride and nb = M/block:
 *   non-causal  B*Hq*rp*(nb + 1)*4 bytes
 *   causal      B*Hq*(rp*(nb + 1)/2 + rp)*4 bytes  (about half: c <= r only)
 * The workspace must be sized with the same `causal` value the scoring call
 * gets. Returns 0 for unsupported arguments.
 */
XATTN_API size_t xattn_score_workspace_size(int B, int Hq, int M, int stride, int block,
                                            int causal);

/*
 * xattn_score - strided antidiagonal block scores [DuSA-Q2, XA-abs, XA-app].
 *
 * For query head h (KV head h/(Hq/Hkv)), with S = stride, g = block/S:
 *   Q'[i'] = q[i'S+S-1], q[i'S+S-2], ..., q[i'S]   (reversed inside the group)
 *   K'[j'] = k[j'S], k[j'S+1], ..., k[j'S+S-1]     (forward)
 *   X[i',j'] = score_scale * <Q'[i'], K'[j']>
 * so X[i',j'] is the S-long lower-left -> upper-right antidiagonal sum of the
 * S x S tile (i',j') of q k^T. Causal: column j' is visible to row i' iff
 * j' <= i'. Each row of X goes through a softmax over its visible columns, and
 *   scores[b,h,r,c] = (1/g) * sum over the g x g entries of block pair (r,c),
 * so every block row sums to 1. Causal entries c > r are written as 0.
 * The (M/S)^2 matrix X is never stored.
 *
 *   Q           bf16 [B, Hq, M, C]
 *   K           bf16 [B, Hkv, M, C]
 *   score_scale the scale of X; the usual value is 1/sqrt(stride*C)
 *   scores      fp32 [B, Hq, M/block, M/block] (output)
 *   workspace   device buffer of at least xattn_score_workspace_size(..., causal)
 *               bytes, 16-byte aligned; contents on entry are ignored
 */
XATTN_API int xattn_score(const void* Q, const void* K, int B, int Hq, int Hkv, int M, int C,
                int stride, int block, int causal, float score_scale,
                float* scores, void* workspace, size_t workspace_bytes, void* stream);

/* Scoring patterns of xattn_score_ex. */
typedef enum {
  XATTN_PATTERN_ANTIDIAGONAL = 0,  /* the method: lower-left -> upper-right sums   */
  XATTN_PATTERN_DIAGONAL = 1       /* the variant the pages compare against        */
} xattn_pattern;

/*
 * xattn_score_ex - xattn_score with a choice of pattern [DuSA-Q2, XA-abl].
 * XATTN_PATTERN_ANTIDIAGONAL is exactly xattn_score. XATTN_PATTERN_DIAGONAL
 * reads the query rows of each stride group forward, so that X[i',j'] sums the
 * main diagonal of the S x S tile (i',j') of q k^T instead:
 *   X[i',j'] = score_scale * sum_s q[i'S+s] . k[j'S+s]
 * (the diagonal-pattern XAttention variant of DuSA's Response to Q2, and the
 * "diagonal scoring" row of the XAttention summary's "Measured effects" table,
 * [XA-abl]). Every other argument, output and error is that of xattn_score;
 * an unknown pattern returns XATTN_EINVAL.
 */
XATTN_API int xattn_score_ex(const void* Q, const void* K, int B, int Hq, int Hkv, int M, int C,
                             int stride, int block, int causal, int pattern, float score_scale,
                             float* scores, void* workspace, size_t workspace_bytes,
                             void* stream);

/*
 * Workspace bytes xattn_select needs: per-row cut (score, index) and count,
 * 12 bytes per (batch, head, query block) row, rounded up to 256 bytes.
 */
XATTN_API size_t xattn_select_workspace_size(int B, int Hq, int nb);

/*
 * xattn_select - threshold block selection [XA-app, FP-RQ3].
 *
 * For each row (b, h, r), candidates are key blocks c <= r (causal) or all
 * c < nb. They are ordered by score descending, ties to the smaller c, and the
 * shortest prefix whose cumulative score reaches tau[h] (>=) is kept; tau[h] >= 1
 * keeps every candidate. The diagonal block c = r is then added if missing. The
 * kept indices of each row are written ascending.
 *
 *   scores       fp32 [B, Hq, nb, nb] as written by xattn_score
 *   tau          fp32 [Hq], device memory; per-head thresholds in (0, 1]
 *   row_ptr      int32 [B*Hq*nb + 1] (output): row (b,h,r) = (b*Hq+h)*nb + r
 *                owns col_idx[row_ptr[row] .. row_ptr[row+1])
 *   col_idx      int32 [col_capacity] (output): kept key-block indices
 *   col_capacity entries col_idx can hold; B*Hq*nb*(nb+1)/2 (causal) or
 *                B*Hq*nb*nb (non-causal) is always enough
 *   nnz          int32 [1], device memory (output): total kept entries
 *   workspace    device buffer of xattn_select_workspace_size() bytes
 * If the kept entries exceed col_capacity, nnz still receives the true count,
 * every row_ptr entry is set to 0 (all rows empty), nothing is written to
 * col_idx, and the device error word is set to XATTN_ECAPACITY.
 */
XATTN_API int xattn_select(const float* scores, const float* tau, int B, int Hq, int nb, int causal,
                 int32_t* row_ptr, int32_t* col_idx, size_t col_capacity, int32_t* nnz,
                 void* workspace, size_t workspace_bytes, void* stream);

/* Selection rules of xattn_select_ex. */
typedef enum {
  XATTN_SELECT_THRESHOLD = 0,  /* the method: shortest prefix reaching tau[h]     */
  XATTN_SELECT_TOPK = 1,       /* the floor(param[h]) highest-ranked candidates   */
  XATTN_SELECT_RATIO = 2       /* ceil(param[h] * candidates) highest-ranked       */
} xattn_select_rule;

/*
 * xattn_select_ex - selection with the rules of the ablation [XA-abl].
 * Candidates are ranked as in xattn_select (score descending, ties to the
 * smaller block index). param is fp32 [Hq] in device memory:
 *   XATTN_SELECT_THRESHOLD  param = tau; identical to xattn_select
 *   XATTN_SELECT_TOPK       keep the first max(1, min(floor(param[h]), n))
 *   XATTN_SELECT_RATIO      keep the first ceil(param[h] * n), computed in fp64
 *                           from the fp32 value and clamped to [1, n]
 * where n is the row's candidate count (r+1 causal, nb otherwise); a NaN param
 * keeps every candidate. The diagonal block is then added if missing. Outputs,
 * workspace and capacity behaviour are those of xattn_select; an unknown rule
 * returns XATTN_EINVAL.
 */
XATTN_API int xattn_select_ex(const float* scores, const float* param, int rule, int B, int Hq,
                              int nb, int causal, int32_t* row_ptr, int32_t* col_idx,
                              size_t col_capacity, int32_t* nnz, void* workspace,
                              size_t workspace_bytes, void* stream);

/*
 * Workspace bytes xattn_score_select needs: the scoring workspace for the same
 * `causal` flag (rounded up to 256 bytes) followed by the selection workspace.
 */
XATTN_API size_t xattn_score_select_workspace_size(int B, int Hq, int M, int stride, int block,
                                                   int causal);

/*
 * xattn_score_select - xattn_score followed by xattn_select_ex, fused
 * [DuSA-Q2, XA-abs, XA-app, FP-RQ3]. The scoring kernel ranks and cuts every
 * query-block row right after writing its scores, while the row is still in L2,
 * so the selection needs only its scan and fill passes: three launches instead
 * of four, and no second read of the score matrix. scores and the CSR
 * (row_ptr, col_idx, nnz) are bit-identical to those of xattn_score with the
 * antidiagonal pattern followed by xattn_select_ex with the same rule and param;
 * every argument, layout and error has the meaning it has there.
 */
XATTN_API int xattn_score_select(const void* Q, const void* K, int B, int Hq, int Hkv, int M,
                                 int C, int stride, int block, int causal, float score_scale,
                                 const float* param, int rule, float* scores, int32_t* row_ptr,
                                 int32_t* col_idx, size_t col_capacity, int32_t* nnz,
                                 void* workspace, size_t workspace_bytes, void* stream);

/*
 * Largest number of selection rows (B*Hq*nb) that xattn_select_noalloc takes.
 */
#define XATTN_SELECT_NOALLOC_MAX_ROWS 262144

/*
 * xattn_select_noalloc - the same selection as xattn_select, for callers that
 * cannot hand the library a workspace. This is a library convenience; the
 * pages describe no counterpart.
 *
 * Some callers cannot allocate device memory when they run this step: a host
 * framework that owns all device memory and forbids allocation inside its
 * execute callbacks (plugins, custom operators with a fixed memory plan), or a
 * latency-critical caller that cannot afford the device-wide synchronisation a
 * cudaMalloc may bring. This entry point takes no workspace and calls no
 * allocator: its per-row scratch (12 bytes per row) lives in a fixed array
 * inside the library, XATTN_SELECT_NOALLOC_MAX_ROWS rows (3 MiB), which every
 * GPU that loads the library holds until the process exits.
 *
 * Arguments, outputs and capacity behaviour are those of xattn_select. The
 * caller still provides every input and output buffer.
 *   - B*Hq*nb above XATTN_SELECT_NOALLOC_MAX_ROWS returns XATTN_EUNSUPPORTED
 *     before any launch.
 *   - The first call on a device looks up the scratch array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it; make that
 *     first call before any stream capture.
 *   - Every call on a device shares the one scratch array, and calls whose work
 *     overlaps on the GPU (different streams, or different host threads) race
 *     on it. Serialise them, e.g. issue them on one stream. The scratch keeps
 *     the last call's contents; each call overwrites every row it reads.
 */
XATTN_API int xattn_select_noalloc(const float* scores, const float* tau, int B, int Hq, int nb,
                                   int causal, int32_t* row_ptr, int32_t* col_idx,
                                   size_t col_capacity, int32_t* nnz, void* stream);

/*
 * xattn_sparse_attn - block-sparse softmax attention [DuSA-W3, XA-app].
 *
 * For query token i of block r of head h (KV head h/(Hq/Hkv)):
 *   O[i] = sum_j softmax_j(softmax_scale * q_i . k_j) v_j
 * over the tokens j of the kept key blocks of row (b,h,r) (and j <= i when
 * causal). Accumulation and softmax are fp32; O is rounded to bf16. The
 * unnormalised weights are taken against one reference per row (its first kept
 * block's maximum; a tile whose logits outgrow it by more than 2^24 is computed
 * again against the true maximum), so they stay below 2^24 and the fp32
 * accumulators stay finite for |V| < 2^86.
 *
 *   Q, O       bf16 [B, Hq, M, C];  K, V  bf16 [B, Hkv, M, C]
 *   row_ptr, col_idx  CSR as produced by xattn_select (device memory). Entries
 *              outside [0, M/block), and entries c > r when causal, are skipped;
 *              any order is accepted; a block listed twice is attended twice
 *              (its keys count twice in the softmax), so lists should not repeat
 *              an entry. The caller guarantees that every
 *              row_ptr[i] .. row_ptr[i+1] range lies inside col_idx (the
 *              kernel reads col_idx there without a bound; a row with
 *              row_ptr[i+1] <= row_ptr[i] is empty).
 *   lse        fp32 [B, Hq, M] natural-log log-sum-exp of each query row's
 *              logits, or NULL. A row with no visible key gets O = 0 and
 *              lse = -inf.
 */
XATTN_API int xattn_sparse_attn(const void* Q, const void* K, const void* V,
                      const int32_t* row_ptr, const int32_t* col_idx,
                      int B, int Hq, int Hkv, int M, int C, int block, int causal,
                      float softmax_scale, void* O, float* lse, void* stream);

/*
 * GQA-shared kept lists - a variant the pages do not define (there every query
 * head keeps its own minimal set [XA-app]). For GQA models the query heads of
 * one KV group share the union of their own kept lists, so that one list of
 * K/V blocks serves the whole group. Each head's own set is contained in the
 * union, so each head still covers at least its own threshold mass.
 *
 * xattn_select_group - every query head's selection exactly as xattn_select_ex
 * (same rule and param), then per (b, kvh, r) the ascending union over the
 * heads h with h / (Hq/Hkv) == kvh. CSR over B*Hkv*nb rows: row_ptr has
 * B*Hkv*nb + 1 entries, row (b*Hkv + kvh)*nb + r. Hq must be a multiple of Hkv
 * and Hq/Hkv <= 64 (else XATTN_EINVAL / XATTN_EUNSUPPORTED). Capacity and
 * error behaviour as in xattn_select; worst case B*Hkv*nb*(nb+1)/2 entries
 * causal, B*Hkv*nb*nb otherwise.
 */
XATTN_API size_t xattn_select_group_workspace_size(int B, int Hq, int Hkv, int nb);
XATTN_API int xattn_select_group(const float* scores, const float* param, int rule, int B,
                                 int Hq, int Hkv, int nb, int causal, int32_t* row_ptr,
                                 int32_t* col_idx, size_t col_capacity, int32_t* nnz,
                                 void* workspace, size_t workspace_bytes, void* stream);

/*
 * xattn_sparse_attn_group - xattn_sparse_attn on GQA-shared lists: query head h
 * of batch b attends over the kept blocks of CSR row (b*Hkv + h/(Hq/Hkv))*nb + r,
 * as produced by xattn_select_group. Everything else as in xattn_sparse_attn.
 */
XATTN_API int xattn_sparse_attn_group(const void* Q, const void* K, const void* V,
                                      const int32_t* row_ptr, const int32_t* col_idx,
                                      int B, int Hq, int Hkv, int M, int C, int block,
                                      int causal, float softmax_scale, void* O, float* lse,
                                      void* stream);

/*
 * xattn_dense_attn - the same attention with every key block kept (all c <= r
 * when causal, all c otherwise); no CSR. Used as the dense baseline.
 */
XATTN_API int xattn_dense_attn(const void* Q, const void* K, const void* V,
                     int B, int Hq, int Hkv, int M, int C, int block, int causal,
                     float softmax_scale, void* O, float* lse, void* stream);

/*
 * xattn_selftest_wait_timeout - diagnostic of the bounded device waits (the
 * pages have no counterpart). Launches one CTA that waits on a barrier nothing
 * will ever complete, for at most limit_ns nanoseconds (1 .. 1e9). The wait must
 * give up, raise XATTN_ETIMEOUT in the device error word and write 1 to
 * *timed_out (int32, device memory). The context stays usable; read the status
 * with xattn_get_device_error. Limits outside the range return XATTN_EINVAL.
 */
XATTN_API int xattn_selftest_wait_timeout(long long limit_ns, int32_t* timed_out, void* stream);

/*
 * xattn_selftest_exp2 - diagnostic of the FMA-pipe base-2 exponential that the
 * attention softmax uses for part of its elements instead of the hardware
 * approximation (the pages have no counterpart). y[i] = 2^x[i] for n fp32
 * values (device arrays, n >= 0): relative error at most 1.1e-4 for x in
 * [-126, 127]; exactly 0 for x <= -127 and for -inf; a value in [0, 2^-126]
 * in between. Larger x are outside its domain. Returns XATTN_EINVAL for n < 0
 * or a null array with n > 0.
 */
XATTN_API int xattn_selftest_exp2(const float* x, float* y, long long n, void* stream);

/*
 * Synchronises `stream`, then returns and clears the current device's error
 * word (XATTN_OK if no device-side condition was raised since the last call).
 * Returns XATTN_ECUDA if the synchronisation itself failed.
 */
XATTN_API int xattn_get_device_error(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* XATTN_H */
