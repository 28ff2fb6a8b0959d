// Block-sparse (and dense) softmax attention on a CTA pair (cta_group::2).
//
// The same computation as attn_tc.cuh (attention over the kept key blocks only:
// DuSA rebuttal, Response to W3/Q1; XAttention summary, Approach), with two
// neighbouring query blocks of one (batch, query head) on a pair of SMs. The
// pair walks the union of its two kept lists in ascending block order and shares
// one MMA stream: the leader (cluster rank 0) issues M = 256 MMAs in which each
// CTA contributes its own 128 query rows (Q and P) and half of every K / V tile
// (K: 64 of the 128 keys; V: 64 of the 128 output columns), so each SM loads
// and stores half the K/V bytes of the single-CTA kernel and the pair issues
// half the MMA instructions. A block of the union that is not in a CTA's own
// list (or lies above its diagonal) gets P = 0 in that CTA: its scores are
// computed and dropped. Everything else (warp roles, one fixed reference per row,
// the second pass for rows that outgrow it, bounded waits) is as in attn_tc.cuh;
// the second-pass decision is taken for the pair as a whole.
//
// Warp roles (384 threads per CTA):
//   warp 0, one lane  TMA producer, both CTAs: its own Q tile once, then its
//                     halves of the K and V tiles of the union's blocks into
//                     rings whose completion is counted on the leader's barriers.
//   warp 1, one lane  S issuer (leader only); warp 1 of both CTAs owns the TMEM.
//   warp 2, one lane  PV issuer (leader only).
//   warps 4-11        softmax of the CTA's own rows, two threads per row.
// Kept lists are read into two bitmaps (one per query block of the pair) at the
// start, so any order is accepted and an entry listed twice counts once.
#pragma once
#include "attn_tc.cuh"
#include "common.cuh"
#include "sm100.cuh"

namespace xattn {

struct AttnPair {
  static constexpr int C = 128;
  static constexpr int kStagesK = 4, kStagesV = 4;
  static constexpr int kQTile = 128 * 256;          // 128 rows x 128 bf16: two 16 KB regions
  static constexpr int kQRegion = 128 * 128;
  static constexpr int kKHalf = 64 * 256;           // 64 keys x 128 bf16: two 8 KB regions
  static constexpr int kKRegion = 64 * 128;
  static constexpr int kVHalf = 128 * 128;          // 128 keys x 64 output columns
  static constexpr int kMaxWords = 2048;            // bitmap words: nb <= 65536
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQTile;
  static constexpr int kOffV = kOffK + kStagesK * kKHalf;
  static constexpr int kOffBits = kOffV + kStagesV * kVHalf;           // [2][kMaxWords]
  static constexpr int kOffBar = kOffBits + 2 * kMaxWords * 4;
  static constexpr int kOffX = kOffBar + 512;                          // [2 half][128] float2
  static constexpr int kOffM = kOffX + 2 * 128 * 8;                    // [2 half][128] float
  static constexpr int kSmem = kOffM + 2 * 128 * 4 + 1024;
  static constexpr int kTmemCols = 512;                                // S_0, S_1, S_2, O
  static constexpr int kSBuf = 3;
  static constexpr int kColS = 0;
  static constexpr int kColO = 384;
};

// Walks the union of the pair's two kept-block bitmaps in ascending order.
struct UnionIter {
  const uint32_t* a;   // bitmap of the leader's query block
  const uint32_t* b;   // bitmap of the other CTA's query block
  int nw, w;
  uint32_t wa, wb, rem;
  __device__ __forceinline__ void init(const uint32_t* a_, const uint32_t* b_, int nw_) {
    a = a_; b = b_; nw = nw_; w = -1; rem = 0u; wa = wb = 0u;
  }
  // next block of the union and which CTAs keep it (bit 0: leader, bit 1: other)
  __device__ __forceinline__ bool next(int& c, int& mask) {
    while (rem == 0u) {
      if (++w >= nw) return false;
      wa = a[w];
      wb = b[w];
      rem = wa | wb;
    }
    const int bit = __ffs(rem) - 1;
    rem &= rem - 1u;
    c = w * 32 + bit;
    mask = (int)((wa >> bit) & 1u) | ((int)((wb >> bit) & 1u) << 1);
    return true;
  }
};

template <bool DENSE>
__global__ void __launch_bounds__(kAttnTcThreads, 1)
attn_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const int32_t* __restrict__ row_ptr,
                 const int32_t* __restrict__ col_idx, int Hq, int Hkv, int M, int causal,
                 int group_rows, float scale_log2, bf16* __restrict__ O, float* __restrict__ lse) {
  using L = AttnPair;
  constexpr int C = L::C;
  constexpr int STK = L::kStagesK, STV = L::kStagesV;
  constexpr int SB = L::kSBuf;
  using namespace sm100;

  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const uint32_t sQ = smem_u32(smem + L::kOffQ);
  const uint32_t sK0 = smem_u32(smem + L::kOffK);
  const uint32_t sV0 = smem_u32(smem + L::kOffV);
  uint32_t* bits = reinterpret_cast<uint32_t*>(smem + L::kOffBits);   // [2][kMaxWords]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* k_full = bars;                    // [STK] both CTAs' K halves landed (leader)
  uint64_t* k_empty = bars + STK;             // [STK] its S MMA completed (both CTAs)
  uint64_t* v_full = bars + 2 * STK;          // [STV] both V halves landed (leader)
  uint64_t* v_empty = bars + 2 * STK + STV;   // [STV] its PV MMAs completed (both CTAs)
  uint64_t* q_full = bars + 2 * STK + 2 * STV;
  uint64_t* s_full = q_full + 1;      // [SB] S of the block computed (both CTAs)
  uint64_t* s_free = q_full + 4;      // [SB] the PV MMAs reading P from it completed (leader)
  uint64_t* p_full = q_full + 7;      // [SB] P written by both CTAs' 16 softmax warps (leader)
  uint64_t* o_done = q_full + 10;     // the last PV of a pass completed (both CTAs)
  uint64_t* drain = q_full + 11;      // [2] S issuer, PV issuer (both CTAs)
  uint64_t* x_full = q_full + 13;     // end-of-pass (max, sum) published (8 warps, own CTA)
  uint64_t* m0_full = q_full + 14;    // first-block maxima published (8 warps, own CTA)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_full + 15);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* redo_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);
  volatile int* peer_flags = reinterpret_cast<volatile int*>(tmem_slot + 3);   // written by the other CTA
  float2* xchg = reinterpret_cast<float2*>(smem + L::kOffX);
  float* xm = reinterpret_cast<float*>(smem + L::kOffM);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int crank = (int)cluster_ctarank();
  const bool leader = crank == 0;
  const int nb = M / 128;
  const int nw = (nb + 31) / 32;
  // the pair's query blocks: longest rows first when causal; a CTA past the last
  // block (nb odd) keeps no block and writes nothing
  const int slot0 = (int)blockIdx.x & ~1;
  const int r_of0 = causal ? nb - 1 - slot0 : slot0;
  const int r_of1 = causal ? nb - 2 - slot0 : slot0 + 1;
  const int r = crank == 0 ? r_of0 : r_of1;
  const bool real = r >= 0 && r < nb;
  const int bh = blockIdx.y;
  const int b = bh / Hq, h = bh % Hq, kvh = h / (Hq / Hkv);
  const size_t row_base = (size_t)(group_rows ? b * Hkv + kvh : bh) * nb;

  if (tid == 0) {
    for (int i = 0; i < STK; ++i) { mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1); }
    for (int i = 0; i < STV; ++i) { mbar_init(&v_full[i], 1); mbar_init(&v_empty[i], 1); }
    mbar_init(q_full, 1);
    for (int i = 0; i < SB; ++i) {
      mbar_init(&s_full[i], 1); mbar_init(&s_free[i], 1); mbar_init(&p_full[i], 16);
    }
    mbar_init(o_done, 1);
    mbar_init(&drain[0], 1); mbar_init(&drain[1], 1);
    mbar_init(x_full, 8);
    mbar_init(m0_full, 8);
    *abort_flag = 0;
    *redo_flag = 0;
    peer_flags[0] = 0;
    fence_mbar_init();
  }
  // the two kept-block bitmaps (leader's block, other's block): valid entries only
  for (int i = tid; i < 2 * nw; i += kAttnTcThreads) bits[(i / nw) * L::kMaxWords + i % nw] = 0u;
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, L::kTmemCols);
    tmem_relinquish_pair();
  }
  if (tid == 32 * 2) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  __syncthreads();
#pragma unroll 1
  for (int q = 0; q < 2; ++q) {
    const int rq = q == 0 ? r_of0 : r_of1;
    if (rq < 0 || rq >= nb) continue;
    uint32_t* bm = bits + q * L::kMaxWords;
    const int hi = causal ? rq + 1 : nb;   // visible key blocks: c < hi
    if (DENSE) {
      for (int c = tid; c < hi; c += kAttnTcThreads) atomicOr(&bm[c >> 5], 1u << (c & 31));
    } else {
      const int beg = row_ptr[row_base + rq], end = row_ptr[row_base + rq + 1];
      for (int i = beg + tid; i < end; i += kAttnTcThreads) {
        const int c = __ldg(col_idx + i);
        if (c >= 0 && c < hi) atomicOr(&bm[c >> 5], 1u << (c & 31));
      }
    }
  }
  tc_fence_before();
  cluster_sync();   // bitmaps built; both CTAs' barriers exist before either signals the other's
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t* bm0 = bits;
  const uint32_t* bm1 = bits + L::kMaxWords;
  const int own_bit = 1 << crank;

  int nk = 0, nv = 0;              // producer: K and V tiles issued so far
  int jb = 0;                      // issuers and softmax: blocks of earlier passes
  float m_ref = kNegInf;           // softmax: the row's reference (scaled, base 2)
  bool have_ref = false;
  float m_true = 0.f, l_tot = 0.f; // softmax: the row's largest logit (scaled) and sum of P

  for (int pass = 0; pass < 2; ++pass) {
    if (warp == 0) {
      // ---------------------------------------------------- TMA producer
      if (lane == 0) {
        const uint32_t kf = mapa_shared(k_full, 0), vf = mapa_shared(v_full, 0);
        if (pass == 0) {
          if (leader) mbar_expect_tx(q_full, 2 * L::kQTile);
          // a CTA past the last block loads some valid rows (its scores are dropped)
          const int yq = bh * M + (real ? r : r_of0) * 128;
          const uint32_t qf = mapa_shared(q_full, 0);
          tma_load_2d_pair(sQ, &tmQ, 0, yq, qf);
          tma_load_2d_pair(sQ + L::kQRegion, &tmQ, 64, yq, qf);
        }
        const int ykv = (b * Hkv + kvh) * M;
        auto load_v = [&](int jv, int cv) -> bool {
          const int st = jv % STV;
          if (jv >= STV && !mbar_wait(&v_empty[st], ((jv / STV) - 1) & 1, abort_flag)) return false;
          if (leader) mbar_expect_tx(&v_full[st], 2 * L::kVHalf);
          // V rows of the block, this CTA's 64 output columns
          tma_load_2d_pair(sV0 + st * L::kVHalf, &tmV, crank * 64, ykv + cv * 128, vf + st * 8);
          return true;
        };
        UnionIter it;
        it.init(bm0, bm1, nw);
        int c, mask, c_prev = -1;
        bool ok = true;
        while (it.next(c, mask)) {
          const int st = nk % STK;
          if (nk >= STK && !(ok = mbar_wait(&k_empty[st], ((nk / STK) - 1) & 1, abort_flag))) break;
          if (leader) mbar_expect_tx(&k_full[st], 2 * L::kKHalf);
          // this CTA's 64 keys of the block, both 64-column regions
          const int yk = ykv + c * 128 + crank * 64;
          tma_load_2d_pair(sK0 + st * L::kKHalf, &tmK, 0, yk, kf + st * 8);
          tma_load_2d_pair(sK0 + st * L::kKHalf + L::kKRegion, &tmK, 64, yk, kf + st * 8);
          ++nk;
          if (c_prev >= 0) {
            if (!(ok = load_v(nv, c_prev))) break;
            ++nv;
          }
          c_prev = c;
        }
        if (ok && c_prev >= 0 && load_v(nv, c_prev)) ++nv;
        // drain (leader: its barriers count both CTAs' loads; the other CTA leaves
        // only after the final cluster barrier, which the leader reaches after this)
        if (leader) {
          volatile int no_abort = 0;
          mbar_wait(q_full, 0, &no_abort);
          for (int jj = (nk > STK ? nk - STK : 0); jj < nk; ++jj)
            mbar_wait(&k_full[jj % STK], (jj / STK) & 1, &no_abort);
          for (int jj = (nv > STV ? nv - STV : 0); jj < nv; ++jj)
            mbar_wait(&v_full[jj % STV], (jj / STV) & 1, &no_abort);
        }
      }
    } else if (warp == 1 || warp == 2) {
      // ----------------------------------------------- S and PV issuers (leader)
      if (lane == 0 && leader) {
        const uint64_t dQ = smem_desc_sw128(sQ, 16, 1024);
        const uint64_t dK = smem_desc_sw128(sK0, 16, 1024);
        const uint64_t dV = smem_desc_sw128(sV0, 16, 1024);
        constexpr uint32_t idS = idesc_bf16_f32(256, 128, false, false);
        constexpr uint32_t idPV = idesc_bf16_f32(256, C, false, true);
        UnionIter it;
        it.init(bm0, bm1, nw);
        int c, mask;
        bool have_cur = it.next(c, mask);
        bool ok = true;
        int j = jb;
        if (warp == 1) {
          ok = !have_cur || mbar_wait(q_full, 0, abort_flag);
          for (; ok && have_cur; ++j) {
            const int st = j % STK, sb = j % SB;
            ok = mbar_wait(&k_full[st], (j / STK) & 1, abort_flag) &&
                 (j < SB || mbar_wait(&s_free[sb], ((j / SB) - 1) & 1, abort_flag));
            if (!ok) break;
            tc_fence_after();
            const uint64_t dKs = dK + (uint64_t)((st * L::kKHalf) >> 4);
            const uint32_t tSb = tmem + L::kColS + sb * 128;
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk) {
              const uint32_t offq = ((kk >> 2) * L::kQRegion + (kk & 3) * 32) >> 4;
              const uint32_t offk = ((kk >> 2) * L::kKRegion + (kk & 3) * 32) >> 4;
              mma_f16_ss_pair(tSb, dQ + offq, dKs + offk, idS, kk > 0);
            }
            mma_commit_pair(&s_full[sb]);
            mma_commit_pair(&k_empty[st]);
            have_cur = it.next(c, mask);
          }
        } else {
          for (; ok && have_cur; ++j) {
            const int st = j % STV, sb = j % SB;
            if (!(ok = mbar_wait(&v_full[st], (j / STV) & 1, abort_flag) &&
                       mbar_wait(&p_full[sb], (j / SB) & 1, abort_flag)))
              break;
            tc_fence_after();
            const uint64_t dVs = dV + (uint64_t)((st * L::kVHalf) >> 4);
            const uint32_t tP = tmem + L::kColS + sb * 128;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)   // keys 16kk .. 16kk+15: half kk/4, 8 TMEM columns
              mma_f16_ts_pair(tmem + L::kColO, tP + (kk >> 2) * 64 + (kk & 3) * 8,
                              dVs + (uint64_t)((kk * 2048) >> 4), idPV,
                              (j > jb || kk > 0) ? 1u : 0u);
            mma_commit_pair(&v_empty[st]);
            mma_commit_pair(&s_free[sb]);
            have_cur = it.next(c, mask);
            if (!have_cur) mma_commit_pair(o_done);   // the pass's last PV
          }
        }
        jb = j;
      }
    } else if (warp >= 4) {
      // ----------------------------------------------------------- softmax
      const int g = (warp >= 8) ? 1 : 0;                 // keys [64g, 64g + 64) of each block
      const int q_row = (warp & 3) * 32 + lane;          // row within the query block
      const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
      const uint32_t tSg = tmem + lane_off + L::kColS + g * 64;   // + sb * 128
      const int k0 = g * 64;
      const uint32_t pf = mapa_shared(p_full, 0);
      float l = 0.f, m_seen = kNegInf;
      bool ovf = false;
      int j = jb;
      bool ok = true;
      UnionIter it;
      it.init(bm0, bm1, nw);
      int c, mask;
      for (; it.next(c, mask); ++j) {
        const int sb = j % SB;
        ok = __all_sync(0xffffffffu, mbar_wait(&s_full[sb], (j / SB) & 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
        if (mask & own_bit) {
          float s[64];
          tmem_ld32(tSg + sb * 128, s);
          tmem_ld32(tSg + sb * 128 + 32, s + 32);
          tmem_wait_ld();
          if (causal && c == r) {
#pragma unroll
            for (int i = 0; i < 64; ++i) s[i] = (k0 + i > q_row) ? kNegInf : s[i];
          }
          float pm[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) pm[k] = fmaxf(s[2 * k], s[2 * k + 1]);
          if (pass == 0 && !have_ref) {
            // the row's reference: the maximum over both halves of its first own block
#pragma unroll
            for (int i = 16; i < 64; i += 2) pm[(i >> 1) & 7] = fmax3(pm[(i >> 1) & 7], s[i], s[i + 1]);
            const float mx = fmax3(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], pm[5]),
                                   fmaxf(pm[6], pm[7]));
            xm[g * 128 + q_row] = mx;
            __syncwarp();
            if (lane == 0) mbar_arrive(m0_full);
            ok = __all_sync(0xffffffffu, mbar_wait(m0_full, 0, abort_flag));
            if (!ok) break;
            const float mr = fmaxf(mx, xm[(1 - g) * 128 + q_row]);
            m_ref = (mr == kNegInf) ? 0.f : mr * scale_log2;
            have_ref = true;
          }
          const float2 sc2 = make_float2(scale_log2, scale_log2), nm2 = make_float2(-m_ref, -m_ref);
          float2 ps[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                          make_float2(0.f, 0.f)};
#pragma unroll
          for (int i = 0; i < 64; i += 2) {
            if (i >= 16) pm[(i >> 1) & 7] = fmax3(pm[(i >> 1) & 7], s[i], s[i + 1]);
            const float2 x = ffma2(make_float2(s[i], s[i + 1]), sc2, nm2);
            if (((i >> 1) & 7) < kEmuPer8) {
              const float2 e = ex2_poly2(x);
              s[i] = e.x;
              s[i + 1] = e.y;
            } else {
              s[i] = ex2(x.x);
              s[i + 1] = ex2(x.y);
            }
            ps[(i >> 1) & 3] = fadd2(ps[(i >> 1) & 3], make_float2(s[i], s[i + 1]));
          }
          const float mx = fmax3(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], pm[5]),
                                 fmaxf(pm[6], pm[7]));
          m_seen = fmaxf(m_seen, mx);
          ovf |= mx * scale_log2 > m_ref + kRefHeadroom;
          const float2 pq = fadd2(fadd2(ps[0], ps[1]), fadd2(ps[2], ps[3]));
          l += pq.x + pq.y;
          uint32_t pk[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) pk[i] = pack_bf16x2(s[2 * i], s[2 * i + 1]);
          tmem_st32(tSg + sb * 128, reinterpret_cast<const float*>(pk));
        } else {
          // a block only the other CTA keeps: P = 0 for this CTA's rows
          float z[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) z[i] = 0.f;
          tmem_st32(tSg + sb * 128, z);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(pf + sb * 8);
      }

      if (ok && j > jb) ok = __all_sync(0xffffffffu, mbar_wait(o_done, pass & 1, abort_flag));
      if (ok) {
        xchg[g * 128 + q_row] = make_float2(m_seen, l);
        if (ovf) *redo_flag = 1;
        __syncwarp();
        if (lane == 0) mbar_arrive(x_full);
        ok = __all_sync(0xffffffffu, mbar_wait(x_full, pass & 1, abort_flag));
      }
      if (ok) {
        tc_fence_after();
        // both halves against the same reference; the second pass is decided for
        // the pair (below), with the row's largest logit as its new reference
        const float2 s0 = xchg[q_row], s1 = xchg[128 + q_row];
        const float mr = fmaxf(s0.x, s1.x);
        m_true = (mr == kNegInf) ? 0.f : mr * scale_log2;
        l_tot = s0.y + s1.y;
      }
      tc_fence_before();
      jb = j;
    }

    // pair-wide decision on a second pass (either CTA's rows outgrew their
    // reference) and on an abort (either CTA gave up a wait)
    __syncthreads();
    if (tid == 0) {
      const int mine = (*redo_flag ? 1 : 0) | (*abort_flag ? 2 : 0);
      asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(mapa_shared(
                       const_cast<int*>(peer_flags), (uint32_t)(crank ^ 1))), "r"(mine)
                   : "memory");
    }
    cluster_sync();
    const int both = (*redo_flag ? 1 : 0) | (*abort_flag ? 2 : 0) | peer_flags[0];
    const bool redo = pass == 0 && (both & 1) && !(both & 2);
    if (warp >= 4) {
      const int g = (warp >= 8) ? 1 : 0;
      const int q_row = (warp & 3) * 32 + lane;
      if (!redo && !(both & 2) && !*abort_flag && real) {
        // write the output: O = O_acc / l over this half's output columns
        const float lt = l_tot;
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        bf16* orow = O + ((size_t)bh * M + (size_t)r * 128 + q_row) * C + g * (C / 2);
        const uint32_t tO0 = tmem + lane_off + L::kColO + g * (C / 2);
        tc_fence_after();
#pragma unroll
        for (int qq = 0; qq < C / 64; ++qq) {
          float a[32];
          tmem_ld32(tO0 + qq * 32, a);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            float vv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) vv[e] = lt > 0.f ? a[i + e] * inv : 0.f;
            uint4 v;
            v.x = pack_bf16x2(vv[0], vv[1]);
            v.y = pack_bf16x2(vv[2], vv[3]);
            v.z = pack_bf16x2(vv[4], vv[5]);
            v.w = pack_bf16x2(vv[6], vv[7]);
            *reinterpret_cast<uint4*>(orow + qq * 32 + i) = v;
          }
        }
        if (lse != nullptr && g == 0)
          lse[(size_t)bh * M + (size_t)r * 128 + q_row] =
              lt > 0.f ? (m_ref + lg2(lt)) * kLn2 : kNegInf;
      } else if (redo) {
        m_ref = m_true;   // second pass: the row's largest logit becomes its reference
      }
      tc_fence_before();
    }
    if (!redo) break;
    // every role walks the union again (jb blocks done), its barrier phases carried on
    __syncthreads();
    if (tid == 0) { *redo_flag = 0; peer_flags[0] = 0; }
    cluster_sync();   // neither CTA resets its flags while the other still reads them
  }

  // drain: all MMAs of the pair complete before TMEM is freed
  if ((warp == 1 || warp == 2) && lane == 0) {
    if (leader) mma_commit_pair(&drain[warp - 1]);
    volatile int no_abort = 0;
    mbar_wait(&drain[warp - 1], 0, &no_abort);
  }
  tc_fence_before();
  cluster_sync();   // neither CTA leaves while the other may still touch its memory
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, L::kTmemCols);
  }
}

}  // namespace xattn
