// Block-sparse (and dense) softmax attention on the warp-level tensor-core path.
//
// One CTA = one (batch, query head, query block r) of 128 query rows, 8 warps of
// 16 rows. It walks the key blocks of its row (the CSR list, or every block for
// the dense baseline), double-buffering K/V tiles of 128 keys through shared
// memory with cp.async, and keeps the FlashAttention online softmax in fp32
// registers (base-2 domain). Sparse attention over the kept blocks follows the
// DuSA rebuttal (Response to W3/Q1) and the XAttention summary (Approach).
#pragma once
#include "common.cuh"

namespace xattn {

constexpr int kAttnThreads = 256;

template <int C>
constexpr int attn_smem_bytes() { return (128 * C * 2) * 5; }   // Q + 2 x (K, V)

template <int C, bool DENSE>
__global__ void __launch_bounds__(kAttnThreads, 1)
attn_mma_kernel(const bf16* __restrict__ Q, const bf16* __restrict__ K, const bf16* __restrict__ V,
                const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx, int Hq,
                int Hkv, int M, int causal, float scale_log2, bf16* __restrict__ O,
                float* __restrict__ lse) {
  constexpr int RB = C * 2;          // bytes per tile row
  constexpr int NCH = RB / 16;       // 16-byte chunks per row
  constexpr int TILE = 128 * RB;     // bytes per 128-row tile
  constexpr int KD = C / 16;         // k16 steps over the head dim
  constexpr int ND = C / 8;          // n8 tiles over the head dim

  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sQ = smem_u32(smem);
  auto sK = [&](int st) { return smem_u32(smem + TILE * (1 + 2 * st)); };
  auto sV = [&](int st) { return smem_u32(smem + TILE * (2 + 2 * st)); };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nb = M / 128;
  const int r = nb - 1 - (int)blockIdx.x;   // longest rows first
  const int bh = blockIdx.y;
  const int b = bh / Hq, h = bh % Hq, kvh = h / (Hq / Hkv);
  const size_t row = (size_t)bh * nb + r;
  const bf16* Qb = Q + ((size_t)bh * M + (size_t)r * 128) * C;
  const bf16* Kh = K + (size_t)(b * Hkv + kvh) * M * C;
  const bf16* Vh = V + (size_t)(b * Hkv + kvh) * M * C;

  int beg, end;
  if (DENSE) { beg = 0; end = causal ? r + 1 : nb; }
  else { beg = row_ptr[row]; end = row_ptr[row + 1]; }

  // block index of list entry it, or -1 if it must be skipped
  auto block_of = [&](int it) -> int {
    const int c = DENSE ? it : col_idx[it];
    if (c < 0 || c >= nb || (causal && c > r)) return -1;
    return c;
  };

  auto load_tile = [&](uint32_t dst, const bf16* src) {
#pragma unroll
    for (int p = 0; p < (128 * NCH) / kAttnThreads; ++p) {
      const int piece = tid + p * kAttnThreads;
      const int rr = piece / NCH, ch = piece % NCH;
      cp_async16(dst + swz(rr, ch, RB), src + (size_t)rr * C + ch * 8, true);
    }
  };

  // skip leading invalid entries
  int it = beg;
  int cur = -1;
  while (it < end && (cur = block_of(it)) < 0) ++it;

  load_tile(sQ, Qb);
  if (cur >= 0) {
    load_tile(sK(0), Kh + (size_t)cur * 128 * C);
    load_tile(sV(0), Vh + (size_t)cur * 128 * C);
  }
  cp_async_commit();

  float o[ND][4];
#pragma unroll
  for (int n = 0; n < ND; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m_run[2] = {kNegInf, kNegInf}, l_run[2] = {0.f, 0.f};
  uint32_t qf[KD][4];
  bool have_q = false;

  int st = 0;
  while (cur >= 0) {
    // find and prefetch the next valid block
    int nit = it + 1, nxt = -1;
    while (nit < end && (nxt = block_of(nit)) < 0) ++nit;
    if (nxt >= 0) {
      load_tile(sK(st ^ 1), Kh + (size_t)nxt * 128 * C);
      load_tile(sV(st ^ 1), Vh + (size_t)nxt * 128 * C);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();

    if (!have_q) {
#pragma unroll
      for (int kk = 0; kk < KD; ++kk) {
        const int rr = warp * 16 + (lane & 15);
        const int ch = kk * 2 + (lane >> 4);
        ldsm_x4(qf[kk], sQ + swz(rr, ch, RB));
      }
      have_q = true;
    }

    // S = Q K^T for this warp's 16 rows x 128 keys
    float s[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
    const uint32_t kb = sK(st);
#pragma unroll
    for (int kk = 0; kk < KD; ++kk) {
#pragma unroll
      for (int np = 0; np < 8; ++np) {
        uint32_t bb[4];
        const int rr = np * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int ch = kk * 2 + ((lane >> 3) & 1);
        ldsm_x4(bb, kb + swz(rr, ch, RB));
        mma16816(s[2 * np], qf[kk], bb[0], bb[1]);
        mma16816(s[2 * np + 1], qf[kk], bb[2], bb[3]);
      }
    }

    // online softmax (base 2); causal mask on the diagonal block
    const bool diag = causal && (cur == r);
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int qi = warp * 16 + (lane >> 2) + hr * 8;   // query row within the block
      float mx = kNegInf;
#pragma unroll
      for (int n = 0; n < 16; ++n) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int kj = n * 8 + 2 * (lane & 3) + e;
          float x = s[n][hr * 2 + e] * scale_log2;
          if (diag && kj > qi) x = kNegInf;
          s[n][hr * 2 + e] = x;
          mx = fmaxf(mx, x);
        }
      }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m_run[hr], mx);
      const float m_use = (m_new == kNegInf) ? 0.f : m_new;
      const float corr = ex2(m_run[hr] - m_use);
      m_run[hr] = m_new;
      float rs = 0.f;
#pragma unroll
      for (int n = 0; n < 16; ++n) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float p = ex2(s[n][hr * 2 + e] - m_use);
          s[n][hr * 2 + e] = p;
          rs += p;
        }
      }
      l_run[hr] = l_run[hr] * corr + rs;
#pragma unroll
      for (int n = 0; n < ND; ++n) {
        o[n][hr * 2] *= corr;
        o[n][hr * 2 + 1] *= corr;
      }
    }

    // O += P V
    const uint32_t vb = sV(st);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {       // 16 keys per step
      uint32_t a[4];
      a[0] = pack_bf16x2(s[2 * kk][0], s[2 * kk][1]);
      a[1] = pack_bf16x2(s[2 * kk][2], s[2 * kk][3]);
      a[2] = pack_bf16x2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      a[3] = pack_bf16x2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int dp = 0; dp < ND / 2; ++dp) {
        uint32_t bb[4];
        const int rr = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
        const int ch = dp * 2 + (lane >> 4);
        ldsm_x4_t(bb, vb + swz(rr, ch, RB));
        mma16816(o[2 * dp], a, bb[0], bb[1]);
        mma16816(o[2 * dp + 1], a, bb[2], bb[3]);
      }
    }
    __syncthreads();   // stage st is free for the prefetch after next
    st ^= 1;
    it = nit;
    cur = nxt;
  }
  cp_async_wait<0>();

  // epilogue: O / l -> bf16; lse = (m + log2 l) * ln 2
  bf16* Ob = O + ((size_t)bh * M + (size_t)r * 128) * C;
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    float l = l_run[hr];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const int qi = warp * 16 + (lane >> 2) + hr * 8;
#pragma unroll
    for (int n = 0; n < ND; ++n) {
      const int d = n * 8 + 2 * (lane & 3);
      *reinterpret_cast<uint32_t*>(Ob + (size_t)qi * C + d) =
          pack_bf16x2(o[n][hr * 2] * inv, o[n][hr * 2 + 1] * inv);
    }
    if (lse != nullptr && (lane & 3) == 0)
      lse[(size_t)bh * M + (size_t)r * 128 + qi] = l > 0.f ? (m_run[hr] + lg2(l)) * kLn2 : kNegInf;
  }
}

}  // namespace xattn
