// Strided antidiagonal block scoring on the warp-level tensor-core path.
//
// One CTA owns 128 reshaped query rows i' of one (batch, query head) and sweeps
// the reshaped key columns j' in tiles of 128 (only j' <= i' tiles when causal).
// The reduction dimension S*C of the reshaped rows (DuSA rebuttal, Response to
// Q2) is streamed in 64-element chunks: chunk q covers stride slot
// s = (64q)/C, head dims d0 = (64q)%C; the query side reads token i'S+S-1-s
// (rows reversed inside each stride group) and the key side token j'S+s, so
// each dot product is an S-long lower-left -> upper-right antidiagonal of q k^T
// (XAttention abstract). The reversal is pure address arithmetic.
//
// Epilogue per column tile (row softmax + block summation, XAttention summary,
// Approach): for every row and every key block of g = 128/S columns, the block's
// log-sum-exp ell[i', c] (base 2) is formed in registers and written to the
// workspace, and the row's running log-sum-exp is updated online. The (M/S)^2
// logits are never stored. After the sweep the CTA re-reads its own ell values
// (L2-resident) and writes scores[r, c] = (1/g) sum_{i' in r} 2^(ell[i',c] - LSE[i']).
#pragma once
#include "common.cuh"

namespace xattn {

constexpr int kScoreThreads = 256;
constexpr int kScoreStages = 3;
constexpr int kScoreTile = 128;                          // rows and columns per tile
constexpr int kScoreChunk = 64;                          // reduction elements per stage
constexpr int kScoreStageBytes = 2 * kScoreTile * kScoreChunk * 2;  // Q + K chunk
constexpr int kScoreSmem = kScoreStages * kScoreStageBytes + kScoreTile * 4;

// G = block/stride reshaped columns per key block; C = head dim.
template <int C, int G>
__global__ void __launch_bounds__(kScoreThreads, 1)
score_mma_kernel(const bf16* __restrict__ Q, const bf16* __restrict__ K, int Hq, int Hkv, int M,
                 int causal, float scale_log2, float* __restrict__ part, float* __restrict__ lse_ws,
                 float* __restrict__ scores) {
  constexpr int S = 128 / G;
  constexpr int D = S * C;                 // reshaped row width
  constexpr int NCH = D / kScoreChunk;     // chunks per column tile
  constexpr int KB = kScoreTile / G;       // key blocks per column tile
  constexpr int NTB = G / 8 > 0 ? G / 8 : 1;  // n8 tiles per key block
  static_assert(G >= 8 && G <= 128 && (128 % G) == 0, "g must be 8..128");

  extern __shared__ __align__(128) uint8_t smem[];
  float* lse_s = reinterpret_cast<float*>(smem + kScoreStages * kScoreStageBytes);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rp = M / S;                    // reshaped rows
  const int nb = M / 128;
  const int RT = (rp + kScoreTile - 1) / kScoreTile;
  const int t = causal ? (RT - 1 - (int)blockIdx.x) : (int)blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / Hq, h = bh % Hq, kvh = h / (Hq / Hkv);
  const bf16* Qh = Q + (size_t)bh * M * C;
  const bf16* Kh = K + (size_t)(b * Hkv + kvh) * M * C;
  const int i0 = t * kScoreTile;
  const int njt = causal ? (t + 1) : RT;
  const int total = njt * NCH;

  auto stage_q = [&](int st) { return smem_u32(smem + st * kScoreStageBytes); };
  auto stage_k = [&](int st) { return smem_u32(smem + st * kScoreStageBytes + kScoreTile * kScoreChunk * 2); };

  auto load = [&](int st, int it) {
    const int jt = it / NCH, q = it % NCH;
    const int s = (q * kScoreChunk) / C, d0 = (q * kScoreChunk) % C;
    const uint32_t sq = stage_q(st), sk = stage_k(st);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const int piece = tid + p * kScoreThreads;  // 0..1023
      const int row = piece >> 3, ch = piece & 7;
      const int ip = i0 + row;
      const bool okq = ip < rp;
      const bf16* gq = Qh + ((size_t)(okq ? ip : 0) * S + (S - 1 - s)) * C + d0 + ch * 8;
      cp_async16(sq + swz(row, ch, 128), gq, okq);
      const int jp = jt * kScoreTile + row;
      const bool okk = jp < rp;
      const bf16* gk = Kh + ((size_t)(okk ? jp : 0) * S + s) * C + d0 + ch * 8;
      cp_async16(sk + swz(row, ch, 128), gk, okk);
    }
  };

  float acc[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  float m_run[2] = {kNegInf, kNegInf}, l_run[2] = {0.f, 0.f};

#pragma unroll
  for (int st = 0; st < kScoreStages - 1; ++st) {
    if (st < total) load(st, st);
    cp_async_commit();
  }

  for (int it = 0; it < total; ++it) {
    cp_async_wait<kScoreStages - 2>();
    __syncthreads();
    {
      const int nx = it + kScoreStages - 1;
      if (nx < total) load(nx % kScoreStages, nx);
      cp_async_commit();
    }
    const int st = it % kScoreStages;
    const uint32_t sq = stage_q(st), sk = stage_k(st);
#pragma unroll
    for (int kk = 0; kk < kScoreChunk / 16; ++kk) {
      uint32_t a[4];
      {
        const int row = warp * 16 + (lane & 15);
        const int ch = kk * 2 + (lane >> 4);
        ldsm_x4(a, sq + swz(row, ch, 128));
      }
#pragma unroll
      for (int np = 0; np < 8; ++np) {
        uint32_t bb[4];
        const int row = np * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int ch = kk * 2 + ((lane >> 3) & 1);
        ldsm_x4(bb, sk + swz(row, ch, 128));
        mma16816(acc[2 * np], a, bb[0], bb[1]);
        mma16816(acc[2 * np + 1], a, bb[2], bb[3]);
      }
    }

    if ((it % NCH) == NCH - 1) {
      // ---- epilogue for column tile jt: per-(row, key block) log-mass ----
      const int j0 = (it / NCH) * kScoreTile;
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const int ip = i0 + warp * 16 + (lane >> 2) + rr * 8;
#pragma unroll
        for (int kb = 0; kb < KB; ++kb) {
          float v[NTB * 2];
          float vmax = kNegInf;
#pragma unroll
          for (int n = 0; n < NTB; ++n) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int nt = kb * NTB + n;
              const int jp = j0 + nt * 8 + 2 * (lane & 3) + e;
              float x = acc[nt][rr * 2 + e] * scale_log2;
              const bool ok = (jp < rp) && (!causal || jp <= ip);
              x = ok ? x : kNegInf;
              v[n * 2 + e] = x;
              vmax = fmaxf(vmax, x);
            }
          }
          vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, 1));
          vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, 2));
          float sum = 0.f;
          if (vmax != kNegInf) {
#pragma unroll
            for (int n = 0; n < NTB * 2; ++n) sum += ex2(v[n] - vmax);
          }
          sum += __shfl_xor_sync(0xffffffffu, sum, 1);
          sum += __shfl_xor_sync(0xffffffffu, sum, 2);
          if (vmax != kNegInf) {
            const float ell = vmax + lg2(sum);
            const float mn = fmaxf(m_run[rr], ell);
            l_run[rr] = l_run[rr] * ex2(m_run[rr] - mn) + ex2(ell - mn);
            m_run[rr] = mn;
            const int c = (j0 + kb * G) / G;
            if ((lane & 3) == (kb & 3) && ip < rp)
              part[((size_t)bh * rp + ip) * nb + c] = ell;
          }
        }
      }
#pragma unroll
      for (int n = 0; n < 16; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
    }
  }
  cp_async_wait<0>();

  // ---- finalize: row LSE, then block sums over the g rows of each block ----
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const int rl = warp * 16 + (lane >> 2) + rr * 8;
    if ((lane & 3) == 0) {
      const float L = (l_run[rr] > 0.f) ? m_run[rr] + lg2(l_run[rr]) : kNegInf;
      lse_s[rl] = L;
      if (i0 + rl < rp) lse_ws[(size_t)bh * rp + i0 + rl] = L;
    }
  }
  __syncthreads();  // also orders this CTA's part[] writes before the reads below

  const float inv_g = 1.f / (float)G;
  for (int k = 0; k < KB; ++k) {
    const int r = i0 / G + k;
    if (r >= nb) break;
    const int ncand = causal ? r + 1 : nb;
    float* srow = scores + ((size_t)bh * nb + r) * nb;
    for (int c = tid; c < nb; c += kScoreThreads) {
      float acc_s = 0.f;
      if (c < ncand) {
        const float* pr = part + ((size_t)bh * rp + (size_t)r * G) * nb + c;
        // every row i' of block r sees at least one column of each block
        // c <= r (causal) or of every block (non-causal), so ell is defined
#pragma unroll 4
        for (int i = 0; i < G; ++i)
          acc_s += ex2(pr[(size_t)i * nb] - lse_s[r * G + i - i0]);
        acc_s *= inv_g;
      }
      srow[c] = acc_s;
    }
  }
}

}  // namespace xattn
