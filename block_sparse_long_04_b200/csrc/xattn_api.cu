// C ABI of libxattn.so: argument validation, workspace sizing and launches.
// The contract of every entry point is documented in include/xattn.h.
#include "xattn.h"

#include <algorithm>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "attn_pair.cuh"
#include "attn_tc.cuh"
#include "common.cuh"
#include "score_tc.cuh"
#include "select.cuh"

using namespace xattn;

namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// cudaFuncSetAttribute is per device: remember, per device ordinal, which
// kernels already have their dynamic shared-memory limit raised.
template <typename F>
int ensure_smem_limit(F* kern, int bytes, unsigned long long* done_mask) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return XATTN_ECUDA;
  const unsigned long long bit = 1ull << (dev & 63);
  if (__atomic_load_n(done_mask, __ATOMIC_ACQUIRE) & bit) return XATTN_OK;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return XATTN_ECUDA;
  __atomic_fetch_or(done_mask, bit, __ATOMIC_RELEASE);
  return XATTN_OK;
}

inline int launch_status() {
  return cudaGetLastError() == cudaSuccess ? XATTN_OK : XATTN_ECUDA;
}

// y = 2^x through ex2_poly2, two elements per thread (grid-stride)
__global__ void exp2_selftest_kernel(const float* __restrict__ x, float* __restrict__ y,
                                     long long n) {
  const long long pairs = (n + 1) / 2;
  for (long long p = blockIdx.x * (long long)blockDim.x + threadIdx.x; p < pairs;
       p += (long long)gridDim.x * blockDim.x) {
    const long long i = 2 * p;
    const bool two = i + 1 < n;
    const float2 e = ex2_poly2(make_float2(x[i], two ? x[i + 1] : 0.f));
    y[i] = e.x;
    if (two) y[i + 1] = e.y;
  }
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D map over a [rows, width] bf16 matrix with box_rows x 64-column boxes and
// 128-byte swizzle (the layout the tensor core's SW128 descriptors read).
bool make_tile_map(CUtensorMap* map, const void* base, uint64_t rows, int width,
                   int box_rows = 128) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)width, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)width * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool stride_supported(int stride) {
  return stride == 1 || stride == 2 || stride == 4 || stride == 8 || stride == 16 ||
         stride == 32 || stride == 64;
}

// Shared shape checks; returns XATTN_OK, XATTN_EINVAL or XATTN_EUNSUPPORTED.
int check_shape(int B, int Hq, int Hkv, int M, int C, int block) {
  if (B < 0 || Hq < 0 || Hkv < 0 || M < 0 || C <= 0 || block <= 0) return XATTN_EINVAL;
  if (Hkv == 0 && Hq > 0) return XATTN_EINVAL;
  if (Hkv > 0 && Hq % Hkv != 0) return XATTN_EINVAL;
  if (M % block != 0) return XATTN_EINVAL;
  if (block != 128) return XATTN_EUNSUPPORTED;
  if (C != 64 && C != 128) return XATTN_EUNSUPPORTED;
  // element offsets stay below 2^62; grid dimensions below their limits
  if ((long long)B * Hq > 65535) return XATTN_EUNSUPPORTED;
  return XATTN_OK;
}

// fp32 partial log-masses of the scoring workspace: one per (reshaped row, key
// block) it can see, i.e. rp * nb per head, or rp * (nb + 1) / 2 when causal.
size_t score_part_entries(int B, int Hq, int M, int stride, int block, int causal) {
  const size_t rp = (size_t)M / stride, nb = (size_t)M / block;
  return (size_t)B * Hq * (causal ? rp * (nb + 1) / 2 : rp * nb);
}

// Optional fused selection of the scoring kernel: rule + per-head parameter, and
// where to put each row's cut (null: scores only).
struct FusedSelect {
  const float* param = nullptr;
  int rule = 0;
  SelCut* cuts = nullptr;
};

// Scoring launches as CTA pairs (cta_group::2) by default; building with
// XATTN_SCORE_PAIR=0 gives the single-CTA kernel.
#ifndef XATTN_SCORE_PAIR
#define XATTN_SCORE_PAIR 1
#endif

template <int C, int G, bool SELECT, int PAIR>
int launch_score_tc_mode(const bf16* Q, const bf16* K, int B, int Hq, int Hkv, int M, int causal,
                         int diagonal, float scale, float* scores, float* part, float* lse_ws,
                         FusedSelect fs, cudaStream_t st) {
  constexpr int BN = 256;
  using L = ScoreTc<BN, PAIR, (PAIR && (128 / G) * C >= 128) ? 2 : 1>;   // the kernel's layout
  auto kern = score_tc_kernel<C, G, BN, SELECT, PAIR>;
  constexpr int smem = L::kSmem;
  static unsigned long long done = 0;
  if (ensure_smem_limit(kern, smem, &done) != XATTN_OK) return XATTN_ECUDA;
  const int S = 128 / G;
  const int rp = M / S;
  const int RT = (rp + 127) / 128;
  CUtensorMap mq, mk;
  if (!make_tile_map(&mq, Q, (uint64_t)B * Hq * rp, S * C, 128) ||
      !make_tile_map(&mk, K, (uint64_t)B * Hkv * rp, S * C, L::kKRows))
    return XATTN_ECUDA;
  const float sl2 = scale * kLog2e;
  if (PAIR == 0) {
    kern<<<dim3(RT, B * Hq), kScoreTcThreads, smem, st>>>(mq, mk, Hq, Hkv, M, causal, diagonal,
                                                         sl2, part, lse_ws, scores, fs.param,
                                                         fs.rule, fs.cuts);
    if (!SELECT)
      score_finalize_kernel<G><<<dim3((unsigned)(M / 128), (unsigned)(B * Hq)), 256, 0, st>>>(
          part, lse_ws, scores, rp, M / 128, causal);
    return launch_status();
  }
  // pairs of heads: grid (2 * RT, B*Hq/2); pairs of row tiles: (2 * ceil(RT/2), B*Hq)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = PAIR == 1 ? dim3(2 * RT, B * Hq / 2) : dim3(2 * ((RT + 1) / 2), B * Hq);
  cfg.blockDim = dim3(kScoreTcThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, mq, mk, Hq, Hkv, M, causal, diagonal, sl2, part, lse_ws,
                         scores, fs.param, fs.rule, fs.cuts) != cudaSuccess)
    return XATTN_ECUDA;
  if (!SELECT) {
    // the block scores from the partials, on every SM at once
    score_finalize_kernel<G><<<dim3((unsigned)(M / 128), (unsigned)(B * Hq)), 256, 0, st>>>(
        part, lse_ws, scores, rp, M / 128, causal);
  }
  return launch_status();
}

template <int C, int G, bool SELECT>
int launch_score_tc(const bf16* Q, const bf16* K, int B, int Hq, int Hkv, int M, int causal,
                    int diagonal, float scale, float* scores, float* part, float* lse_ws,
                    FusedSelect fs, cudaStream_t st) {
#if XATTN_SCORE_PAIR
  // two query heads of one KV group share every key tile; otherwise two row tiles
  if ((Hq / Hkv) % 2 == 0)
    return launch_score_tc_mode<C, G, SELECT, 1>(Q, K, B, Hq, Hkv, M, causal, diagonal, scale,
                                                 scores, part, lse_ws, fs, st);
  return launch_score_tc_mode<C, G, SELECT, 2>(Q, K, B, Hq, Hkv, M, causal, diagonal, scale,
                                               scores, part, lse_ws, fs, st);
#else
  return launch_score_tc_mode<C, G, SELECT, 0>(Q, K, B, Hq, Hkv, M, causal, diagonal, scale,
                                               scores, part, lse_ws, fs, st);
#endif
}

template <int C, bool SELECT>
int launch_score_c(int stride, const bf16* Q, const bf16* K, int B, int Hq, int Hkv, int M,
                   int causal, int diagonal, float scale, float* scores, float* part,
                   float* lse_ws, FusedSelect fs, cudaStream_t st) {
  switch (stride) {
    case 1: return launch_score_tc<C, 128, SELECT>(Q, K, B, Hq, Hkv, M, causal, diagonal, scale, scores, part, lse_ws, fs, st);
    case 2: return launch_score_tc<C, 64, SELECT>(Q, K, B, Hq, Hkv, M, causal, diagonal, scale, scores, part, lse_ws, fs, st);
    case 4: return launch_score_tc<C, 32, SELECT>(Q, K, B, Hq, Hkv, M, causal, diagonal, scale, scores, part, lse_ws, fs, st);
    case 8: return launch_score_tc<C, 16, SELECT>(Q, K, B, Hq, Hkv, M, causal, diagonal, scale, scores, part, lse_ws, fs, st);
    case 16: return launch_score_tc<C, 8, SELECT>(Q, K, B, Hq, Hkv, M, causal, diagonal, scale, scores, part, lse_ws, fs, st);
    case 32: return launch_score_tc<C, 4, SELECT>(Q, K, B, Hq, Hkv, M, causal, diagonal, scale, scores, part, lse_ws, fs, st);
    case 64: return launch_score_tc<C, 2, SELECT>(Q, K, B, Hq, Hkv, M, causal, diagonal, scale, scores, part, lse_ws, fs, st);
  }
  return XATTN_EUNSUPPORTED;
}

// Dense attention at C = 128 runs on CTA pairs (cta_group::2): measured on the
// 128K Llama-shaped layer it is 5% faster than one CTA per query block. Sparse
// attention keeps one CTA per query block: a pair walks the union of its two
// kept lists, and the blocks only one of them keeps (~10% more on the
// Llama-shaped layer) cost more than the pair saves (3% slower at 128K, 25% on
// the video-shaped layer). Building with XATTN_ATTN_PAIR=2 runs the pairs for
// sparse lists too, =0 nowhere.
#ifndef XATTN_ATTN_PAIR
#define XATTN_ATTN_PAIR 1
#endif

template <bool DENSE>
int launch_attn_pair(const bf16* Q, const bf16* K, const bf16* V, const int32_t* row_ptr,
                     const int32_t* col_idx, int B, int Hq, int Hkv, int M, int causal,
                     int group_rows, float scale, bf16* O, float* lse, cudaStream_t st) {
  using L = AttnPair;
  auto kern = attn_pair_kernel<DENSE>;
  constexpr int smem = L::kSmem;
  static unsigned long long done = 0;
  if (ensure_smem_limit(kern, smem, &done) != XATTN_OK) return XATTN_ECUDA;
  CUtensorMap mq, mk, mv;
  if (!make_tile_map(&mq, Q, (uint64_t)B * Hq * M, L::C, 128) ||
      !make_tile_map(&mk, K, (uint64_t)B * Hkv * M, L::C, 64) ||
      !make_tile_map(&mv, V, (uint64_t)B * Hkv * M, L::C, 128))
    return XATTN_ECUDA;
  const int nb = M / 128;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * ((nb + 1) / 2), B * Hq);
  cfg.blockDim = dim3(kAttnTcThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, row_ptr, col_idx, Hq, Hkv, M, causal,
                         group_rows, scale * kLog2e, O, lse) != cudaSuccess)
    return XATTN_ECUDA;
  return launch_status();
}

template <int C, bool DENSE>
int launch_attn_tc(const bf16* Q, const bf16* K, const bf16* V, const int32_t* row_ptr,
                   const int32_t* col_idx, int B, int Hq, int Hkv, int M, int causal,
                   int group_rows, float scale, bf16* O, float* lse, cudaStream_t st) {
  if (C == 128 && (XATTN_ATTN_PAIR >= 2 || (XATTN_ATTN_PAIR == 1 && DENSE)))
    return launch_attn_pair<DENSE>(Q, K, V, row_ptr, col_idx, B, Hq, Hkv, M, causal, group_rows,
                                   scale, O, lse, st);
  auto kern = attn_tc_kernel<C, DENSE>;
  constexpr int smem = AttnTc<C>::kSmem;
  static unsigned long long done = 0;
  if (ensure_smem_limit(kern, smem, &done) != XATTN_OK) return XATTN_ECUDA;
  CUtensorMap mq, mk, mv;
  if (!make_tile_map(&mq, Q, (uint64_t)B * Hq * M, C) ||
      !make_tile_map(&mk, K, (uint64_t)B * Hkv * M, C) ||
      !make_tile_map(&mv, V, (uint64_t)B * Hkv * M, C))
    return XATTN_ECUDA;
  dim3 grid(M / 128, B * Hq);
  kern<<<grid, kAttnTcThreads, smem, st>>>(mq, mk, mv, row_ptr, col_idx, Hq, Hkv, M, causal,
                                           group_rows, scale * kLog2e, O, lse);
  return launch_status();
}

template <bool DENSE>
int attn_common(const void* Q, const void* K, const void* V, const int32_t* row_ptr,
                const int32_t* col_idx, int B, int Hq, int Hkv, int M, int C, int block,
                int causal, float softmax_scale, void* O, float* lse, void* stream,
                int group_rows = 0) {
  int rc = check_shape(B, Hq, Hkv, M, C, block);
  if (rc != XATTN_OK) return rc;
  if (B == 0 || Hq == 0 || M == 0) return XATTN_OK;
  if (!Q || !K || !V || !O) return XATTN_EINVAL;
  if (!DENSE && (!row_ptr || !col_idx)) return XATTN_EINVAL;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return XATTN_EINVAL;
  if (!(softmax_scale > 0.f) || softmax_scale == __builtin_huge_valf()) return XATTN_EINVAL;
  if (M / 128 > 65535) return XATTN_EUNSUPPORTED;
  auto q = static_cast<const bf16*>(Q);
  auto k = static_cast<const bf16*>(K);
  auto v = static_cast<const bf16*>(V);
  auto o = static_cast<bf16*>(O);
  cudaStream_t st = as_stream(stream);
  if (C == 64)
    return launch_attn_tc<64, DENSE>(q, k, v, row_ptr, col_idx, B, Hq, Hkv, M, causal ? 1 : 0,
                                     group_rows, softmax_scale, o, lse, st);
  return launch_attn_tc<128, DENSE>(q, k, v, row_ptr, col_idx, B, Hq, Hkv, M, causal ? 1 : 0,
                                    group_rows, softmax_scale, o, lse, st);
}

template <bool SELECT = false>
int score_common(const void* Q, const void* K, int B, int Hq, int Hkv, int M, int C,
                        int stride, int block, int causal, int pattern, float score_scale,
                        float* scores, void* workspace, size_t workspace_bytes, void* stream,
                        FusedSelect fs = FusedSelect()) {
  int rc = check_shape(B, Hq, Hkv, M, C, block);
  if (rc != XATTN_OK) return rc;
  if (stride <= 0 || block % stride != 0) return XATTN_EINVAL;
  if (pattern != XATTN_PATTERN_ANTIDIAGONAL && pattern != XATTN_PATTERN_DIAGONAL)
    return XATTN_EINVAL;
  if (!stride_supported(stride)) return XATTN_EUNSUPPORTED;
  if (B == 0 || Hq == 0 || M == 0) return XATTN_OK;
  if (!Q || !K || !scores || !workspace) return XATTN_EINVAL;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(workspace) || !aligned16(scores))
    return XATTN_EINVAL;
  if (!(score_scale > 0.f) || score_scale == __builtin_huge_valf()) return XATTN_EINVAL;
  const size_t need = xattn_score_workspace_size(B, Hq, M, stride, block, causal);
  if (workspace_bytes < need) return XATTN_EINVAL;
  const int rp = M / stride;
  if ((rp + 127) / 128 > (1 << 30)) return XATTN_EUNSUPPORTED;
  float* part = static_cast<float*>(workspace);
  float* lse_ws = part + score_part_entries(B, Hq, M, stride, block, causal);
  auto q = static_cast<const bf16*>(Q);
  auto k = static_cast<const bf16*>(K);
  cudaStream_t st = as_stream(stream);
  const int diag = pattern == XATTN_PATTERN_DIAGONAL ? 1 : 0;
  if (C == 64)
    return launch_score_c<64, SELECT>(stride, q, k, B, Hq, Hkv, M, causal ? 1 : 0, diag,
                                      score_scale, scores, part, lse_ws, fs, st);
  return launch_score_c<128, SELECT>(stride, q, k, B, Hq, Hkv, M, causal ? 1 : 0, diag,
                                     score_scale, scores, part, lse_ws, fs, st);
}

}  // namespace

extern "C" {

const char* xattn_status_string(int status) {
  switch (status) {
    case XATTN_OK: return "ok";
    case XATTN_EINVAL: return "invalid argument";
    case XATTN_ECAPACITY: return "kept-block list capacity exceeded";
    case XATTN_ECUDA: return "CUDA runtime error";
    case XATTN_ETIMEOUT: return "device-side wait timed out";
    case XATTN_EUNSUPPORTED: return "unsupported configuration";
  }
  return "unknown status";
}

int xattn_version(void) { return 200; }

size_t xattn_score_workspace_size(int B, int Hq, int M, int stride, int block, int causal) {
  if (B < 0 || Hq < 0 || M < 0 || block != 128 || !stride_supported(stride) || M % block)
    return 0;
  const size_t rp = (size_t)M / stride;
  return (score_part_entries(B, Hq, M, stride, block, causal) + (size_t)B * Hq * rp) *
         sizeof(float);
}

int xattn_score(const void* Q, const void* K, int B, int Hq, int Hkv, int M, int C, int stride,
                int block, int causal, float score_scale, float* scores, void* workspace,
                size_t workspace_bytes, void* stream) {
  return score_common(Q, K, B, Hq, Hkv, M, C, stride, block, causal, XATTN_PATTERN_ANTIDIAGONAL,
                      score_scale, scores, workspace, workspace_bytes, stream);
}

int xattn_score_ex(const void* Q, const void* K, int B, int Hq, int Hkv, int M, int C, int stride,
                   int block, int causal, int pattern, float score_scale, float* scores,
                   void* workspace, size_t workspace_bytes, void* stream) {
  return score_common(Q, K, B, Hq, Hkv, M, C, stride, block, causal, pattern, score_scale, scores,
                      workspace, workspace_bytes, stream);
}

size_t xattn_select_workspace_size(int B, int Hq, int nb) {
  if (B < 0 || Hq < 0 || nb < 0) return 0;
  const size_t bytes = (size_t)B * Hq * nb * sizeof(SelCut);
  return (bytes + 255) & ~(size_t)255;
}

// The count pass of the selection: rows of at most kSelShortRow candidates four
// to a CTA (64 threads each), longer rows one to a CTA.
static int launch_select_count(const float* scores, const float* param, int Hq, int nb, int causal,
                               SelCut* cuts, int rule, long long rows, cudaStream_t st) {
  int P = 1;
  while (P < nb) P <<= 1;
  if (P <= kSelShortRow) {
    static unsigned long long done = 0;
    if (ensure_smem_limit(select_count_kernel<4>, 4 * kSelShortRow * 8, &done) != XATTN_OK)
      return XATTN_ECUDA;
    select_count_kernel<4><<<(unsigned)((rows + 3) / 4), kSelThreads, 4 * P * 8, st>>>(
        scores, param, Hq, nb, causal ? 1 : 0, cuts, rule, (int)rows, P);
  } else {
    static unsigned long long done = 0;
    if (ensure_smem_limit(select_count_kernel<1>, kSelMaxNb * 8, &done) != XATTN_OK)
      return XATTN_ECUDA;
    select_count_kernel<1><<<(unsigned)rows, kSelThreads, P * 8, st>>>(
        scores, param, Hq, nb, causal ? 1 : 0, cuts, rule, (int)rows, P);
  }
  return cudaGetLastError() == cudaSuccess ? XATTN_OK : XATTN_ECUDA;
}

// The fill pass: rows of at most 1024 candidates four to a CTA (at most 16 per
// thread), longer ones one to a CTA.
static void launch_select_fill(const float* scores, const SelCut* cuts, int nb, int causal,
                               const int32_t* row_ptr, int32_t* col_idx, long long rows,
                               cudaStream_t st) {
  if (nb <= 1024)
    select_fill_kernel<4><<<(unsigned)((rows + 3) / 4), kSelThreads, 0, st>>>(
        scores, cuts, nb, causal ? 1 : 0, row_ptr, col_idx, (int)rows);
  else
    select_fill_kernel<1><<<(unsigned)rows, kSelThreads, 0, st>>>(
        scores, cuts, nb, causal ? 1 : 0, row_ptr, col_idx, (int)rows);
}

// Checks and launches of the per-head selection (count, scan, fill) with the
// per-row scratch `cuts` supplied by the caller of this helper: the workspace of
// xattn_select / xattn_select_ex, or the library's fixed array for
// xattn_select_noalloc. `cuts` may be null only when there are no rows.
static int select_launch(const float* scores, const float* param, int rule, int B, int Hq, int nb,
                         int causal, int32_t* row_ptr, int32_t* col_idx, size_t col_capacity,
                         int32_t* nnz, SelCut* cuts, cudaStream_t st) {
  const long long rows = (long long)B * Hq * nb;
  if (rows == 0) {
    // nothing to select: row_ptr = {0}, nnz = 0
    if (cudaMemsetAsync(row_ptr, 0, sizeof(int32_t), st) != cudaSuccess) return XATTN_ECUDA;
    if (cudaMemsetAsync(nnz, 0, sizeof(int32_t), st) != cudaSuccess) return XATTN_ECUDA;
    return XATTN_OK;
  }
  if (!scores || !param || !col_idx) return XATTN_EINVAL;
  if (cuts == nullptr) return XATTN_ECUDA;
  if (launch_select_count(scores, param, Hq, nb, causal, cuts, rule, rows, st) != XATTN_OK)
    return XATTN_ECUDA;
  if (cudaGetLastError() != cudaSuccess) return XATTN_ECUDA;
  const long long cap = col_capacity > (size_t)(1LL << 40) ? (1LL << 40) : (long long)col_capacity;
  select_scan_kernel<<<1, 1024, 0, st>>>(cuts, (int)rows, row_ptr, nnz, cap);
  if (cudaGetLastError() != cudaSuccess) return XATTN_ECUDA;
  launch_select_fill(scores, cuts, nb, causal, row_ptr, col_idx, rows, st);
  return launch_status();
}

// Shape and rule checks shared by every per-head selection entry point.
static int select_check(int rule, int B, int Hq, int nb, int causal, const int32_t* row_ptr,
                        const int32_t* nnz) {
  if (B < 0 || Hq < 0 || nb < 0) return XATTN_EINVAL;
  if (rule != kSelThreshold && rule != kSelTopK && rule != kSelRatio) return XATTN_EINVAL;
  const long long rows = (long long)B * Hq * nb;
  if (nb > kSelMaxNb) return XATTN_EUNSUPPORTED;
  // worst-case kept entries must fit the int32 row_ptr
  const long long worst = causal ? rows * (nb + 1) / 2 : rows * nb;
  if (worst >= (1LL << 31) || rows >= (1LL << 31) - 1) return XATTN_EUNSUPPORTED;
  if (!row_ptr || !nnz) return XATTN_EINVAL;
  return XATTN_OK;
}

static int select_common(const float* scores, const float* param, int rule, int B, int Hq, int nb,
                         int causal, int32_t* row_ptr, int32_t* col_idx, size_t col_capacity,
                         int32_t* nnz, void* workspace, size_t workspace_bytes, void* stream) {
  const int rc = select_check(rule, B, Hq, nb, causal, row_ptr, nnz);
  if (rc != XATTN_OK) return rc;
  if ((long long)B * Hq * nb > 0) {
    if (!workspace) return XATTN_EINVAL;
    if (workspace_bytes < xattn_select_workspace_size(B, Hq, nb)) return XATTN_EINVAL;
    if (((uintptr_t)workspace & 15u) != 0) return XATTN_EINVAL;
  }
  return select_launch(scores, param, rule, B, Hq, nb, causal, row_ptr, col_idx, col_capacity,
                       nnz, static_cast<SelCut*>(workspace), as_stream(stream));
}

int xattn_select(const float* scores, const float* tau, int B, int Hq, int nb, int causal,
                 int32_t* row_ptr, int32_t* col_idx, size_t col_capacity, int32_t* nnz,
                 void* workspace, size_t workspace_bytes, void* stream) {
  return select_common(scores, tau, kSelThreshold, B, Hq, nb, causal, row_ptr, col_idx,
                       col_capacity, nnz, workspace, workspace_bytes, stream);
}

int xattn_select_ex(const float* scores, const float* param, int rule, int B, int Hq, int nb,
                    int causal, int32_t* row_ptr, int32_t* col_idx, size_t col_capacity,
                    int32_t* nnz, void* workspace, size_t workspace_bytes, void* stream) {
  return select_common(scores, param, rule, B, Hq, nb, causal, row_ptr, col_idx, col_capacity,
                       nnz, workspace, workspace_bytes, stream);
}

size_t xattn_select_group_workspace_size(int B, int Hq, int Hkv, int nb) {
  if (B < 0 || Hq < 0 || Hkv <= 0 || nb < 0) return 0;
  const size_t g = (size_t)B * Hkv * nb * sizeof(SelCut);
  return xattn_select_workspace_size(B, Hq, nb) + ((g + 255) & ~(size_t)255);
}

int xattn_select_group(const float* scores, const float* param, int rule, int B, int Hq, int Hkv,
                       int nb, int causal, int32_t* row_ptr, int32_t* col_idx,
                       size_t col_capacity, int32_t* nnz, void* workspace,
                       size_t workspace_bytes, void* stream) {
  if (B < 0 || Hq < 0 || nb < 0 || Hkv <= 0 || Hq % Hkv != 0) return XATTN_EINVAL;
  if (rule != kSelThreshold && rule != kSelTopK && rule != kSelRatio) return XATTN_EINVAL;
  if (Hq / Hkv > kSelMaxGroup || nb > kSelMaxNb) return XATTN_EUNSUPPORTED;
  const long long rows = (long long)B * Hq * nb;
  const long long grows = (long long)B * Hkv * nb;
  const long long worst = causal ? grows * (nb + 1) / 2 : grows * nb;
  if (worst >= (1LL << 31) || rows >= (1LL << 31) - 1) return XATTN_EUNSUPPORTED;
  if (!row_ptr || !nnz) return XATTN_EINVAL;
  cudaStream_t st = as_stream(stream);
  if (rows == 0) {
    if (cudaMemsetAsync(row_ptr, 0, sizeof(int32_t), st) != cudaSuccess) return XATTN_ECUDA;
    if (cudaMemsetAsync(nnz, 0, sizeof(int32_t), st) != cudaSuccess) return XATTN_ECUDA;
    return XATTN_OK;
  }
  if (!scores || !param || !col_idx || !workspace) return XATTN_EINVAL;
  if (workspace_bytes < xattn_select_group_workspace_size(B, Hq, Hkv, nb)) return XATTN_EINVAL;
  if (((uintptr_t)workspace & 15u) != 0) return XATTN_EINVAL;
  SelCut* cuts = static_cast<SelCut*>(workspace);
  SelCut* gcuts = reinterpret_cast<SelCut*>(static_cast<uint8_t*>(workspace) +
                                            xattn_select_workspace_size(B, Hq, nb));
  if (launch_select_count(scores, param, Hq, nb, causal, cuts, rule, rows, st) != XATTN_OK)
    return XATTN_ECUDA;
  if (cudaGetLastError() != cudaSuccess) return XATTN_ECUDA;
  select_group_count_kernel<<<(unsigned)grows, kSelThreads, 0, st>>>(scores, cuts, Hq, Hkv, nb,
                                                                     causal ? 1 : 0, gcuts);
  if (cudaGetLastError() != cudaSuccess) return XATTN_ECUDA;
  const long long cap = col_capacity > (size_t)(1LL << 40) ? (1LL << 40) : (long long)col_capacity;
  select_scan_kernel<<<1, 1024, 0, st>>>(gcuts, (int)grows, row_ptr, nnz, cap);
  if (cudaGetLastError() != cudaSuccess) return XATTN_ECUDA;
  select_group_fill_kernel<<<(unsigned)grows, kSelThreads, 0, st>>>(
      scores, cuts, gcuts, Hq, Hkv, nb, causal ? 1 : 0, row_ptr, col_idx);
  return launch_status();
}

size_t xattn_score_select_workspace_size(int B, int Hq, int M, int stride, int block,
                                         int causal) {
  const size_t a = xattn_score_workspace_size(B, Hq, M, stride, block, causal);
  if (a == 0 && !(B == 0 || Hq == 0 || M == 0)) return 0;
  const size_t a_al = (a + 255) & ~(size_t)255;
  return a_al + xattn_select_workspace_size(B, Hq, block > 0 ? M / block : 0);
}

int xattn_score_select(const void* Q, const void* K, int B, int Hq, int Hkv, int M, int C,
                       int stride, int block, int causal, float score_scale, const float* param,
                       int rule, float* scores, int32_t* row_ptr, int32_t* col_idx,
                       size_t col_capacity, int32_t* nnz, void* workspace,
                       size_t workspace_bytes, void* stream) {
  int rc = check_shape(B, Hq, Hkv, M, C, block);
  if (rc != XATTN_OK) return rc;
  if (rule != kSelThreshold && rule != kSelTopK && rule != kSelRatio) return XATTN_EINVAL;
  const int nb = M / block;
  const long long rows = (long long)B * Hq * nb;
  if (nb > kSelMaxNb) return XATTN_EUNSUPPORTED;
  const long long worst = causal ? rows * (nb + 1) / 2 : rows * nb;
  if (worst >= (1LL << 31) || rows >= (1LL << 31) - 1) return XATTN_EUNSUPPORTED;
  if (!row_ptr || !nnz) return XATTN_EINVAL;
  if (rows > 0 && (!param || !col_idx)) return XATTN_EINVAL;
  if (workspace_bytes < xattn_score_select_workspace_size(B, Hq, M, stride, block, causal))
    return XATTN_EINVAL;
  cudaStream_t st = as_stream(stream);
  if (rows == 0) {
    if (cudaMemsetAsync(row_ptr, 0, sizeof(int32_t), st) != cudaSuccess) return XATTN_ECUDA;
    if (cudaMemsetAsync(nnz, 0, sizeof(int32_t), st) != cudaSuccess) return XATTN_ECUDA;
    return XATTN_OK;
  }
  if (!workspace || ((uintptr_t)workspace & 15u) != 0) return XATTN_EINVAL;
  const size_t a = xattn_score_workspace_size(B, Hq, M, stride, block, causal);
  const size_t a_al = (a + 255) & ~(size_t)255;
  SelCut* cuts = reinterpret_cast<SelCut*>(static_cast<uint8_t*>(workspace) + a_al);
  FusedSelect fs;
  fs.param = param;
  fs.rule = rule;
  fs.cuts = cuts;
  rc = score_common<true>(Q, K, B, Hq, Hkv, M, C, stride, block, causal,
                          XATTN_PATTERN_ANTIDIAGONAL, score_scale, scores, workspace, a, stream,
                          fs);
  if (rc != XATTN_OK) return rc;
  const long long cap = col_capacity > (size_t)(1LL << 40) ? (1LL << 40) : (long long)col_capacity;
  select_scan_kernel<<<1, 1024, 0, st>>>(cuts, (int)rows, row_ptr, nnz, cap);
  if (cudaGetLastError() != cudaSuccess) return XATTN_ECUDA;
  launch_select_fill(scores, cuts, nb, causal, row_ptr, col_idx, rows, st);
  return launch_status();
}

// ---- selection without a caller workspace -------------------------------
// The per-row scratch of xattn_select_noalloc: a fixed device array, so that the
// entry point needs no workspace and calls no allocator.
static __device__ __align__(256) SelCut g_select_scratch[XATTN_SELECT_NOALLOC_MAX_ROWS];

// Device address of g_select_scratch for the current device. The name is a
// host-side stand-in, not a device address, so it is looked up once per device
// (with that device current) and cached.
static SelCut* select_scratch_on_current_device() {
  static SelCut* cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  SelCut* p = __atomic_load_n(&cached[dev], __ATOMIC_ACQUIRE);
  if (p != nullptr) return p;
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_select_scratch) != cudaSuccess || addr == nullptr)
    return nullptr;
  __atomic_store_n(&cached[dev], static_cast<SelCut*>(addr), __ATOMIC_RELEASE);
  return static_cast<SelCut*>(addr);
}

int xattn_select_noalloc(const float* scores, const float* tau, int B, int Hq, int nb, int causal,
                         int32_t* row_ptr, int32_t* col_idx, size_t col_capacity, int32_t* nnz,
                         void* stream) {
  if (B < 0 || Hq < 0 || nb < 0) return XATTN_EINVAL;
  if ((long long)B * Hq * nb > XATTN_SELECT_NOALLOC_MAX_ROWS) return XATTN_EUNSUPPORTED;
  const int rc = select_check(kSelThreshold, B, Hq, nb, causal, row_ptr, nnz);
  if (rc != XATTN_OK) return rc;
  SelCut* cuts = nullptr;
  if ((long long)B * Hq * nb > 0) {
    if (!scores || !tau || !col_idx) return XATTN_EINVAL;
    cuts = select_scratch_on_current_device();
    if (cuts == nullptr) return XATTN_ECUDA;
  }
  return select_launch(scores, tau, kSelThreshold, B, Hq, nb, causal, row_ptr, col_idx,
                       col_capacity, nnz, cuts, as_stream(stream));
}

int xattn_sparse_attn(const void* Q, const void* K, const void* V, const int32_t* row_ptr,
                      const int32_t* col_idx, int B, int Hq, int Hkv, int M, int C, int block,
                      int causal, float softmax_scale, void* O, float* lse, void* stream) {
  return attn_common<false>(Q, K, V, row_ptr, col_idx, B, Hq, Hkv, M, C, block, causal,
                            softmax_scale, O, lse, stream);
}

int xattn_sparse_attn_group(const void* Q, const void* K, const void* V, const int32_t* row_ptr,
                            const int32_t* col_idx, int B, int Hq, int Hkv, int M, int C,
                            int block, int causal, float softmax_scale, void* O, float* lse,
                            void* stream) {
  return attn_common<false>(Q, K, V, row_ptr, col_idx, B, Hq, Hkv, M, C, block, causal,
                            softmax_scale, O, lse, stream, 1);
}

int xattn_dense_attn(const void* Q, const void* K, const void* V, int B, int Hq, int Hkv, int M,
                     int C, int block, int causal, float softmax_scale, void* O, float* lse,
                     void* stream) {
  return attn_common<true>(Q, K, V, nullptr, nullptr, B, Hq, Hkv, M, C, block, causal,
                           softmax_scale, O, lse, stream);
}

int xattn_selftest_wait_timeout(long long limit_ns, int32_t* timed_out, void* stream) {
  if (limit_ns < 1 || limit_ns > 1000000000LL || timed_out == nullptr) return XATTN_EINVAL;
  sm100::wait_timeout_selftest_kernel<<<1, 32, 0, as_stream(stream)>>>(
      (unsigned long long)limit_ns, timed_out);
  return launch_status();
}

int xattn_selftest_exp2(const float* x, float* y, long long n, void* stream) {
  if (n < 0 || (n > 0 && (x == nullptr || y == nullptr))) return XATTN_EINVAL;
  if (n == 0) return XATTN_OK;
  const long long pairs = (n + 1) / 2;
  const unsigned grid = (unsigned)std::min<long long>((pairs + 255) / 256, 148LL * 16);
  exp2_selftest_kernel<<<grid, 256, 0, as_stream(stream)>>>(x, y, n);
  return launch_status();
}

int xattn_get_device_error(void* stream) {
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return XATTN_ECUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess) return XATTN_ECUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return XATTN_ECUDA;
  }
  return v;
}

}  // extern "C"
