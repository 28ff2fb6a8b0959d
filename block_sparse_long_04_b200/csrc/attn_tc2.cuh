// Block-sparse (and dense) softmax attention on the 5th-generation tensor cores,
// with two softmax warpgroups working on alternate key blocks of the same query
// tile so that one group's exponentials overlap the other group's MMAs.
//
// Sparse attention over the kept key blocks only (DuSA rebuttal, Response to
// W3/Q1; XAttention summary, Approach). One CTA = one (batch, query head, query
// block r) tile of 128 query rows; GQA maps query head h to KV head h/(Hq/Hkv).
//
// The kept blocks of the row, in list order j = 0, 1, 2, ..., are dealt to two
// streams g = j & 1. Each stream keeps its own running max / sum and its own
// accumulators in TMEM (S_g: 128 fp32 columns, O_g: C fp32 columns), so the
// streams are independent softmax chains over disjoint key sets; at the end the
// two partial results are merged exactly:
//   m = max(m_0, m_1), l = sum_g l_g 2^(m_g - m), O = sum_g O_g 2^(m_g - m) / l.
//
// Warp roles (320 threads):
//   warps 4-7  softmax stream 0 (even list positions); warps 0-3 stream 1 (odd).
//              One query row per thread (TMEM lane = row), online softmax in fp32
//              (base 2, scale folded into one FMA per element, lazy rescaling of
//              O_g only when the running max grows by more than 2^8), P written as
//              bf16 into shared memory in the tensor core's 128-byte-swizzled
//              K-major layout.
//   warp 8     TMA producer (one lane): Q once; K and V of block j into stage j&1
//              (K and V have separate full/empty barriers, so K of block j+2 can
//              load as soon as S of block j has been computed).
//   warp 9     MMA issuer (one lane) and TMEM owner: S_g = Q K_j^T, O_g += P_g V_j.
// Every wait is bounded (sm100::mbar_wait); on a timeout the CTA raises
// XATTN_ETIMEOUT, stops every role, drains its copies and MMAs and frees TMEM.
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace xattn {

constexpr int kAttnTc2Threads = 320;

template <int C>
struct AttnTc2 {
  static constexpr int kRegion = 128 * 128;        // 128 rows x 64 bf16 (128 B) = 16 KB
  static constexpr int kNReg = C / 64;
  static constexpr int kTile = kNReg * kRegion;    // one 128 x C bf16 tile
  static constexpr int kPTile = 2 * kRegion;       // one 128 x 128 bf16 P tile
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kTile;           // [2]
  static constexpr int kOffV = kOffK + 2 * kTile;       // [2]
  static constexpr int kOffP = kOffV + 2 * kTile;       // [2]
  static constexpr int kOffBar = kOffP + 2 * kPTile;
  static constexpr int kSmem = kOffBar + 256 + 1024;     // + alignment slack
  static constexpr int kTmemCols = 512;                 // S_0, S_1, O_0, O_1
  static constexpr int kColS = 0;                       // + g * 128
  static constexpr int kColO = 256;                     // + g * 128
};

template <int C, bool DENSE>
__global__ void __launch_bounds__(kAttnTc2Threads, 1)
attn_tc2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const int32_t* __restrict__ row_ptr,
                const int32_t* __restrict__ col_idx, int Hq, int Hkv, int M, int causal,
                float scale_log2, bf16* __restrict__ O, float* __restrict__ lse) {
  using L = AttnTc2<C>;
  using namespace sm100;

  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const uint32_t sQ = smem_u32(smem + L::kOffQ);
  const uint32_t sK0 = smem_u32(smem + L::kOffK);
  const uint32_t sV0 = smem_u32(smem + L::kOffV);
  const uint32_t sP0 = smem_u32(smem + L::kOffP);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* k_full = bars;          // [2]
  uint64_t* k_empty = bars + 2;     // [2]
  uint64_t* v_full = bars + 4;      // [2]
  uint64_t* v_empty = bars + 6;     // [2]
  uint64_t* s_full = bars + 8;      // [2] per stream
  uint64_t* s_free = bars + 10;     // [2]
  uint64_t* p_full = bars + 12;     // [2]
  uint64_t* o_done = bars + 14;     // [2]
  uint64_t* q_full = bars + 16;
  uint64_t* drain = bars + 17;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 18);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nb = M / 128;
  const int r = nb - 1 - (int)blockIdx.x;   // longest rows first
  const int bh = blockIdx.y;
  const int b = bh / Hq, h = bh % Hq, kvh = h / (Hq / Hkv);
  const size_t row = (size_t)bh * nb + r;
  int beg, end;
  if (DENSE) { beg = 0; end = causal ? r + 1 : nb; }
  else { beg = row_ptr[row]; end = row_ptr[row + 1]; }
  auto block_of = [&](int it) -> int {
    const int c = DENSE ? it : __ldg(col_idx + it);
    return (c < 0 || c >= nb || (causal && c > r)) ? -1 : c;
  };

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1); mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1); mbar_init(&s_free[i], 4);
      mbar_init(&p_full[i], 4); mbar_init(&o_done[i], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  if (tid == 8 * 32) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      mbar_expect_tx(q_full, L::kTile);
      const int yq = bh * M + r * 128;
#pragma unroll
      for (int g = 0; g < L::kNReg; ++g) tma_load_2d(sQ + g * L::kRegion, &tmQ, g * 64, yq, q_full);
      const int ykv = (b * Hkv + kvh) * M;
      int nk = 0, nv = 0;   // K and V loads issued
      for (int it = beg; it < end; ++it) {
        const int c = block_of(it);
        if (c < 0) continue;
        const int st = nk & 1;
        const uint32_t par = ((nk >> 1) - 1) & 1;
        if (nk >= 2 && !mbar_wait(&k_empty[st], par, abort_flag)) break;
        mbar_expect_tx(&k_full[st], L::kTile);
#pragma unroll
        for (int g = 0; g < L::kNReg; ++g)
          tma_load_2d(sK0 + st * L::kTile + g * L::kRegion, &tmK, g * 64, ykv + c * 128, &k_full[st]);
        ++nk;
        if (nv >= 2 && !mbar_wait(&v_empty[st], par, abort_flag)) break;
        mbar_expect_tx(&v_full[st], L::kTile);
#pragma unroll
        for (int g = 0; g < L::kNReg; ++g)
          tma_load_2d(sV0 + st * L::kTile + g * L::kRegion, &tmV, g * 64, ykv + c * 128, &v_full[st]);
        ++nv;
      }
      // drain: every load issued must land before the CTA may exit
      volatile int no_abort = 0;
      mbar_wait(q_full, 0, &no_abort);
      for (int jj = (nk > 2 ? nk - 2 : 0); jj < nk; ++jj)
        mbar_wait(&k_full[jj & 1], (jj >> 1) & 1, &no_abort);
      for (int jj = (nv > 2 ? nv - 2 : 0); jj < nv; ++jj)
        mbar_wait(&v_full[jj & 1], (jj >> 1) & 1, &no_abort);
    }
  } else if (warp == 9) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int n = 0;
      for (int it = beg; it < end; ++it) n += block_of(it) >= 0 ? 1 : 0;
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idPV = idesc_bf16_f32(128, C, false, true);
      auto issue_S = [&](int j) {
        const int g = j & 1;
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kRegion + (kk & 3) * 32;
          mma_f16_ss(tmem + L::kColS + g * 128, smem_desc_sw128(sQ + off, 16, 1024),
                     smem_desc_sw128(sK0 + g * L::kTile + off, 16, 1024), idS, kk > 0);
        }
        mma_commit(&s_full[g]);
        mma_commit(&k_empty[g]);
      };
      bool ok = n > 0 && mbar_wait(q_full, 0, abort_flag);
      for (int j = 0; ok && j < 2 && j < n; ++j) {
        if (!(ok = mbar_wait(&k_full[j], 0, abort_flag))) break;
        tc_fence_after();
        issue_S(j);
      }
      for (int j = 0; ok && j < n; ++j) {
        const int g = j & 1;
        const uint32_t u = (uint32_t)(j >> 1);
        if (j + 2 < n) {
          // S_g may be overwritten once stream g's softmax has read it
          ok = mbar_wait(&s_free[g], u & 1, abort_flag) &&
               mbar_wait(&k_full[g], (u + 1) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          issue_S(j + 2);
        }
        ok = mbar_wait(&p_full[g], u & 1, abort_flag) && mbar_wait(&v_full[g], u & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t a_off = (kk >> 2) * L::kRegion + (kk & 3) * 32;
          mma_f16_ss(tmem + L::kColO + g * 128, smem_desc_sw128(sP0 + g * L::kPTile + a_off, 16, 1024),
                     smem_desc_sw128(sV0 + g * L::kTile + kk * 2048, L::kRegion, 1024), idPV,
                     (u > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&o_done[g]);
        mma_commit(&v_empty[g]);
      }
      mma_commit(drain);
      volatile int no_abort = 0;
      mbar_wait(drain, 0, &no_abort);
    }
  } else {
    // ------------------------------------------------------------- softmax
    const int g = (warp >= 4) ? 0 : 1;                 // stream of this warpgroup
    const int q_row = (warp & 3) * 32 + lane;          // row within the query block
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + L::kColS + g * 128;
    const uint32_t tO = tmem + lane_off + L::kColO + g * 128;
    const uint32_t sP = sP0 + g * L::kPTile;
    float m = kNegInf, l = 0.f;
    int j = 0, u = 0;
    bool ok = true;
    for (int it = beg; it < end; ++it) {
      const int c = block_of(it);
      if (c < 0) continue;
      if ((j++ & 1) != g) continue;
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[g], u & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      const bool diag = causal && c == r;
      // pass 1: row max of this block (raw logits; the scale is positive)
      float mx = kNegInf;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float v[32];
        tmem_ld32(tS + q * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i)
          mx = fmaxf(mx, (diag && q * 32 + i > q_row) ? kNegInf : v[i]);
      }
      const float m_new = fmaxf(m, mx * scale_log2);
      float corr = 1.f;
      bool resc = false;
      if (u == 0) {
        m = m_new;
      } else if (m_new > m + 8.f) {
        corr = ex2(m - m_new);
        m = m_new;
        resc = true;
      }
      // PV of this stream's previous block must be complete: P_g free, O_g stable
      if (u > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(&o_done[g], (u - 1) & 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
      }
      if (__any_sync(0xffffffffu, resc)) {
#pragma unroll
        for (int q = 0; q < C / 32; ++q) {
          float o[32];
          tmem_ld32(tO + q * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= corr;
          tmem_st32(tO + q * 32, o);
        }
        tmem_wait_st();
      }
      // pass 2: P = 2^(s*scale - m) -> bf16, 128-byte-swizzled K-major, 32 keys at a time
      const float neg_m = -m;
      float rs = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float v[32];
        tmem_ld32(tS + q * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float x = (diag && q * 32 + i > q_row) ? kNegInf : v[i];
          v[i] = ex2(fmaf(x, scale_log2, neg_m));
          rs += v[i];
        }
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const int ch = q * 4 + c4;   // 16-byte chunk (8 keys) index, 0..15
          const uint32_t addr =
              sP + (ch >> 3) * L::kRegion + q_row * 128 + (((ch & 7) ^ (q_row & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr),
                       "r"(pack_bf16x2(v[c4 * 8 + 0], v[c4 * 8 + 1])),
                       "r"(pack_bf16x2(v[c4 * 8 + 2], v[c4 * 8 + 3])),
                       "r"(pack_bf16x2(v[c4 * 8 + 4], v[c4 * 8 + 5])),
                       "r"(pack_bf16x2(v[c4 * 8 + 6], v[c4 * 8 + 7]))
                       : "memory");
        }
      }
      l = l * corr + rs;
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&s_free[g]);
        mbar_arrive(&p_full[g]);
      }
      ++u;
    }

    // last PV of this stream
    if (ok && u > 0) {
      ok = __all_sync(0xffffffffu, mbar_wait(&o_done[g], (u - 1) & 1, abort_flag));
      if (ok) tc_fence_after();
    }
    // exchange (m, l) between the two streams of each row, through each stream's
    // own P buffer (free once that stream's last PV has completed)
    float2* xchg0 = reinterpret_cast<float2*>(smem + L::kOffP);
    float2* xchg1 = reinterpret_cast<float2*>(smem + L::kOffP + L::kPTile);
    (g == 0 ? xchg0 : xchg1)[q_row] = make_float2(m, l);
    asm volatile("bar.sync 1, 256;" ::: "memory");
    tc_fence_after();   // the other stream's last PV completed before the barrier
    const float2 s0 = xchg0[q_row];   // stream 0's (m, l)
    const float2 s1 = xchg1[q_row];   // stream 1's (m, l)
    const bool has0 = s0.y > 0.f, has1 = s1.y > 0.f;
    const float mm = fmaxf(has0 ? s0.x : kNegInf, has1 ? s1.x : kNegInf);
    const float f0 = has0 ? ex2(s0.x - mm) : 0.f;
    const float f1 = has1 ? ex2(s1.x - mm) : 0.f;
    const float lt = s0.y * f0 + s1.y * f1;
    const float inv = lt > 0.f ? 1.f / lt : 0.f;
    const bool all_ok = !*abort_flag;

    // epilogue: stream g writes columns [g*C/2, (g+1)*C/2) of the merged row
    bf16* orow = O + ((size_t)bh * M + (size_t)r * 128 + q_row) * C;
    if (all_ok) {
      const uint32_t tO0 = tmem + lane_off + L::kColO;
      const uint32_t tO1 = tmem + lane_off + L::kColO + 128;
#pragma unroll
      for (int q = 0; q < C / 64; ++q) {
        const int col = g * (C / 2) + q * 32;
        float a[32], bb[32];
        tmem_ld32(tO0 + col, a);
        tmem_ld32(tO1 + col, bb);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; i += 8) {
          float vv[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float x0 = has0 ? a[i + e] * f0 : 0.f;
            const float x1 = has1 ? bb[i + e] * f1 : 0.f;
            vv[e] = (x0 + x1) * inv;
          }
          uint4 v;
          v.x = pack_bf16x2(vv[0], vv[1]);
          v.y = pack_bf16x2(vv[2], vv[3]);
          v.z = pack_bf16x2(vv[4], vv[5]);
          v.w = pack_bf16x2(vv[6], vv[7]);
          *reinterpret_cast<uint4*>(orow + col + i) = v;
        }
      }
      if (g == 0 && lse != nullptr)
        lse[(size_t)bh * M + (size_t)r * 128 + q_row] = lt > 0.f ? (mm + lg2(lt)) * kLn2 : kNegInf;
    }
    tc_fence_before();
  }

  __syncthreads();
  if (warp == 9) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace xattn
