// Block-sparse (and dense) softmax attention on the 5th-generation tensor cores.
//
// Sparse attention over the kept key blocks only (DuSA rebuttal, Response to
// W3/Q1; XAttention summary, Approach). One CTA = one (batch, query head, query
// block r) tile of 128 query rows; GQA maps query head h to KV head h/(Hq/Hkv).
//
// Warp roles (384 threads):
//   warp 0, one lane  TMA producer: Q once, then the K and V tiles of the kept
//                     blocks (in list order) into two rings of kStages stages with
//                     their own full/empty barriers; K runs one block ahead of V.
//   warp 1, one lane  S issuer and TMEM owner: S = Q K^T into one of three TMEM
//                     buffers (128 lanes x 128 fp32 columns each); S of block j
//                     goes to buffer j%3 as soon as the PV MMAs of block j-3,
//                     which read P from that buffer, have completed, so S of the
//                     next two blocks is computed while the softmax works on this one.
//   warp 2, one lane  PV issuer: O += P V into the single TMEM accumulator once
//                     both key halves of P are written.
//   warps 4-11        softmax, two threads per query row (TMEM lane = row): warps
//                     4-7 own keys 0-63 of every block, warps 8-11 keys 64-127.
//                     Both halves exponentiate against one reference m_ref per
//                     row, fixed for the whole row: the maximum over the row's
//                     first kept block, agreed once between the two threads of a
//                     row. P = 2^(s*scale - m_ref) may then exceed 1 where a later
//                     block holds larger logits; fp32 (and bf16) keep the same
//                     relative precision at any magnitude, so this only needs a
//                     bound on the growth: a block whose maximum exceeds m_ref by
//                     more than 2^kRefHeadroom marks the tile, and the whole tile
//                     is computed again with each row's true maximum (seen on the
//                     first pass) as its reference, which cannot be exceeded.
//                     With a fixed reference nothing is ever rescaled, the two
//                     halves never wait for each other inside the loop, and one O
//                     accumulator serves both, which leaves TMEM room for the third
//                     S buffer. Per block: read the half row of S, causal mask on
//                     the diagonal block, fp32 base-2 exponentials with the scale
//                     folded into one FMA, P_g as bf16 over the first 32 columns
//                     of its own half of the S buffer, where the PV MMA reads it
//                     as its A operand. At the end l = l_0 + l_1 and
//                     O = O_acc / l, lse = (m_ref + log2 l) ln 2.
// Every role walks the row's list with the next entry's load already in flight
// (ListIter), so no role waits on a global load inside its loop.
// Every wait is bounded (sm100::mbar_wait); on a timeout the CTA raises
// XATTN_ETIMEOUT, every role stops, in-flight copies and MMAs are drained, and
// TMEM is freed before the CTA exits.
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace xattn {

constexpr int kAttnTcThreads = 384;
#ifndef XATTN_EXP2_EMU_PER8
#define XATTN_EXP2_EMU_PER8 2
#endif
constexpr int kEmuPer8 = XATTN_EXP2_EMU_PER8;   // softmax pairs (of 8) on the FMA pipe
// growth (log2 units) of a row's logits over its reference that one pass accepts:
// P stays below 2^24, the row sum below 2^42 at 256K keys
constexpr float kRefHeadroom = 24.f;

template <int C>
struct AttnTc {
  static constexpr int kStages = (C == 64) ? 3 : 2;
  static constexpr int kRegion = 128 * 128;        // 128 rows x 64 bf16 (128 B) = 16 KB
  static constexpr int kNReg = C / 64;             // regions per 128-row tile
  static constexpr int kTile = kNReg * kRegion;    // one 128 x C bf16 tile
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kTile;
  static constexpr int kOffV = kOffK + kStages * kTile;
  static constexpr int kOffBar = kOffV + kStages * kTile;
  static constexpr int kOffX = kOffBar + 256;             // end-of-row (max, sum) exchange
  static constexpr int kOffM = kOffX + 2 * 128 * 8;       // first-block maxima
  static constexpr int kSmem = kOffM + 2 * 128 * 4 + 1024;  // + alignment slack
  static constexpr int kTmemCols = 512;                   // S_0, S_1, S_2, O
  static constexpr int kSBuf = 3;
  static constexpr int kColS = 0;                         // + b * 128: 128 fp32 columns each
  static constexpr int kColO = 384;                       // C fp32 columns
  // P of the block in S buffer b: for key half g, 64 bf16 keys packed into the
  // first 32 columns of that buffer's half (kColS + b * 128 + g * 64)
};

// Walks the kept-block list of one row, skipping entries outside [0, nb) and,
// when causal, above the diagonal; the load of the following entry is issued as
// soon as the current one is returned, so its latency overlaps the caller's work.
struct ListIter {
  const int32_t* col;
  int it, end, nb, r;
  bool causal, dense;
  int raw;
  __device__ __forceinline__ int fetch(int i) const {
    return i < end ? (dense ? i : __ldg(col + i)) : -1;
  }
  __device__ __forceinline__ void init(const int32_t* c, int beg, int e, int nb_, int r_,
                                       bool causal_, bool dense_) {
    col = c; it = beg; end = e; nb = nb_; r = r_; causal = causal_; dense = dense_;
    raw = fetch(it);
  }
  // next valid key block, or -1 at the end of the list
  __device__ __forceinline__ int next() {
    while (it < end) {
      const int c = raw;
      ++it;
      raw = fetch(it);
      if (c >= 0 && c < nb && !(causal && c > r)) return c;
    }
    return -1;
  }
};

template <int C, bool DENSE>
__global__ void __launch_bounds__(kAttnTcThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const int32_t* __restrict__ row_ptr,
               const int32_t* __restrict__ col_idx, int Hq, int Hkv, int M, int causal,
               int group_rows, float scale_log2, bf16* __restrict__ O, float* __restrict__ lse) {
  using L = AttnTc<C>;
  constexpr int ST = L::kStages;
  constexpr int SB = L::kSBuf;
  using namespace sm100;

  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const uint32_t sQ = smem_u32(smem + L::kOffQ);
  const uint32_t sK0 = smem_u32(smem + L::kOffK);
  const uint32_t sV0 = smem_u32(smem + L::kOffV);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* k_full = bars;            // [ST] K tile of a block landed
  uint64_t* k_empty = bars + ST;      // [ST] its S MMA completed
  uint64_t* v_full = bars + 2 * ST;   // [ST] V tile of a block landed
  uint64_t* v_empty = bars + 3 * ST;  // [ST] its PV MMAs completed
  uint64_t* q_full = bars + 4 * ST;
  uint64_t* s_full = q_full + 1;      // [SB] S of the block computed
  uint64_t* s_free = q_full + 4;      // [SB] the PV MMAs reading P from it completed
  uint64_t* p_full = q_full + 7;      // [SB] P written, both halves (8 warps)
  uint64_t* o_done = q_full + 10;     // the last PV of a pass completed
  uint64_t* drain = q_full + 11;      // [2] S issuer, PV issuer
  uint64_t* x_full = q_full + 13;     // end-of-pass (max, sum) published (8 warps)
  uint64_t* m0_full = q_full + 14;    // first-block maxima published (8 warps)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_full + 15);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* redo_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);
  float2* xchg = reinterpret_cast<float2*>(smem + L::kOffX);   // [2 half][128]
  float* xm = reinterpret_cast<float*>(smem + L::kOffM);       // [2 half][128]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nb = M / 128;
  const int r = nb - 1 - (int)blockIdx.x;   // longest rows first
  const int bh = blockIdx.y;
  const int b = bh / Hq, h = bh % Hq, kvh = h / (Hq / Hkv);
  // the kept list: per (batch, query head) row, or shared by the KV group
  const size_t row = (size_t)(group_rows ? b * Hkv + kvh : bh) * nb + r;
  int beg, end;
  if (DENSE) { beg = 0; end = causal ? r + 1 : nb; }
  else { beg = row_ptr[row]; end = row_ptr[row + 1]; }

  if (tid == 0) {
    for (int i = 0; i < ST; ++i) {
      mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1); mbar_init(&v_empty[i], 1);
    }
    mbar_init(q_full, 1);
    for (int i = 0; i < SB; ++i) {
      mbar_init(&s_full[i], 1); mbar_init(&s_free[i], 1); mbar_init(&p_full[i], 8);
    }
    mbar_init(o_done, 1);
    mbar_init(&drain[0], 1); mbar_init(&drain[1], 1);
    mbar_init(x_full, 8);
    mbar_init(m0_full, 8);
    *abort_flag = 0;
    *redo_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  if (tid == 32 * 2) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // state that carries over into the second pass, if one is needed
  int nk = 0, nv = 0;              // producer: K and V tiles issued so far
  int jb = 0;                      // issuers and softmax: blocks of earlier passes
  float m_ref = kNegInf;           // softmax: the row's reference (scaled, base 2)

  for (int pass = 0; pass < 2; ++pass) {
    if (warp == 0) {
      // ---------------------------------------------------- TMA producer
      if (lane == 0) {
        if (pass == 0) {
          mbar_expect_tx(q_full, L::kTile);
          const int yq = bh * M + r * 128;
#pragma unroll
          for (int g = 0; g < L::kNReg; ++g)
            tma_load_2d(sQ + g * L::kRegion, &tmQ, g * 64, yq, q_full);
        }
        const int ykv = (b * Hkv + kvh) * M;
        // K of block j is issued before V of block j-1: S of a block needs only
        // its K tile, so K loads run one block ahead and are never queued behind
        // the wait for an older PV to free a V stage
        auto load_v = [&](int jv, int cv) -> bool {
          const int st = jv % ST;
          if (jv >= ST && !mbar_wait(&v_empty[st], ((jv / ST) - 1) & 1, abort_flag)) return false;
          mbar_expect_tx(&v_full[st], L::kTile);
#pragma unroll
          for (int g = 0; g < L::kNReg; ++g)
            tma_load_2d(sV0 + st * L::kTile + g * L::kRegion, &tmV, g * 64, ykv + cv * 128,
                        &v_full[st]);
          return true;
        };
        ListIter li;
        li.init(col_idx, beg, end, nb, r, causal != 0, DENSE);
        int c_prev = -1;
        bool ok = true;
        for (int c = li.next(); c >= 0; c = li.next()) {
          const int st = nk % ST;
          if (nk >= ST && !(ok = mbar_wait(&k_empty[st], ((nk / ST) - 1) & 1, abort_flag))) break;
          mbar_expect_tx(&k_full[st], L::kTile);
#pragma unroll
          for (int g = 0; g < L::kNReg; ++g)
            tma_load_2d(sK0 + st * L::kTile + g * L::kRegion, &tmK, g * 64, ykv + c * 128,
                        &k_full[st]);
          ++nk;
          if (c_prev >= 0) {
            if (!(ok = load_v(nv, c_prev))) break;
            ++nv;
          }
          c_prev = c;
        }
        if (ok && c_prev >= 0 && load_v(nv, c_prev)) ++nv;
        // drain: every load issued must land before the CTA may exit
        volatile int no_abort = 0;
        mbar_wait(q_full, 0, &no_abort);
        for (int jj = (nk > ST ? nk - ST : 0); jj < nk; ++jj)
          mbar_wait(&k_full[jj % ST], (jj / ST) & 1, &no_abort);
        for (int jj = (nv > ST ? nv - ST : 0); jj < nv; ++jj)
          mbar_wait(&v_full[jj % ST], (jj / ST) & 1, &no_abort);
      }
    } else if (warp == 1 || warp == 2) {
      // ----------------------------------------------- S and PV issuers
      if (lane == 0) {
        // descriptors built once; per MMA only the start address (16-byte units,
        // low bits) moves, which never carries out of its 14-bit field here
        const uint64_t dQ = smem_desc_sw128(sQ, 16, 1024);
        const uint64_t dK = smem_desc_sw128(sK0, 16, 1024);
        const uint64_t dV = smem_desc_sw128(sV0, L::kRegion, 1024);
        constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);
        constexpr uint32_t idPV = idesc_bf16_f32(128, C, false, true);
        ListIter li;
        li.init(col_idx, beg, end, nb, r, causal != 0, DENSE);
        bool have_cur = li.next() >= 0;
        bool have_nxt = have_cur && li.next() >= 0;
        bool ok = true;
        int j = jb;
        if (warp == 1) {
          ok = !have_cur || mbar_wait(q_full, 0, abort_flag);
          for (; ok && have_cur; ++j) {
            const int st = j % ST, sb = j % SB;
            // buffer j%3 is free once the PV MMAs of block j-3 have read its P
            ok = mbar_wait(&k_full[st], (j / ST) & 1, abort_flag) &&
                 (j < SB || mbar_wait(&s_free[sb], ((j / SB) - 1) & 1, abort_flag));
            if (!ok) break;
            tc_fence_after();
            const uint64_t dKs = dK + (uint64_t)((st * L::kTile) >> 4);
            const uint32_t tSb = tmem + L::kColS + sb * 128;
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk) {
              const uint32_t off = ((kk >> 2) * L::kRegion + (kk & 3) * 32) >> 4;
              mma_f16_ss(tSb, dQ + off, dKs + off, idS, kk > 0);
            }
            mma_commit(&s_full[sb]);
            mma_commit(&k_empty[st]);
            have_cur = have_nxt;
            have_nxt = have_cur && li.next() >= 0;
          }
        } else {
          for (; ok && have_cur; ++j) {
            const int st = j % ST, sb = j % SB;
            if (!(ok = mbar_wait(&v_full[st], (j / ST) & 1, abort_flag) &&
                       mbar_wait(&p_full[sb], (j / SB) & 1, abort_flag)))
              break;
            tc_fence_after();
            const uint64_t dVs = dV + (uint64_t)((st * L::kTile) >> 4);
            const uint32_t tP = tmem + L::kColS + sb * 128;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)   // keys 16kk .. 16kk+15: half kk/4, 8 TMEM columns
              mma_f16_ts(tmem + L::kColO, tP + (kk >> 2) * 64 + (kk & 3) * 8,
                         dVs + (uint64_t)((kk * 2048) >> 4), idPV, (j > jb || kk > 0) ? 1u : 0u);
            mma_commit(&v_empty[st]);
            mma_commit(&s_free[sb]);
            have_cur = have_nxt;
            have_nxt = have_cur && li.next() >= 0;
            if (!have_cur) mma_commit(o_done);   // the pass's last PV
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
      float l = 0.f, m_seen = kNegInf;   // this pass: sum of P, largest raw logit seen
      bool ovf = false;
      int j = jb;
      bool ok = true;
      ListIter li;
      li.init(col_idx, beg, end, nb, r, causal != 0, DENSE);
      for (int c = li.next(); c >= 0; c = li.next(), ++j) {
        const int sb = j % SB;
        ok = __all_sync(0xffffffffu, mbar_wait(&s_full[sb], (j / SB) & 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
        float s[64];
        tmem_ld32(tSg + sb * 128, s);
        tmem_ld32(tSg + sb * 128 + 32, s + 32);
        tmem_wait_ld();
        // masked keys of the diagonal block are set to -inf, on that block only
        if (causal && c == r) {
#pragma unroll
          for (int i = 0; i < 64; ++i) s[i] = (k0 + i > q_row) ? kNegInf : s[i];
        }
        // eight independent partial maxima keep the reduction off one long
        // dependency chain; the three-input max halves its instruction count
        float pm[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) pm[k] = fmaxf(s[2 * k], s[2 * k + 1]);
        if (pass == 0 && j == jb) {
          // the row's reference: the maximum over both halves of its first block
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
        }
        const float2 sc2 = make_float2(scale_log2, scale_log2), nm2 = make_float2(-m_ref, -m_ref);
        float2 ps[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};
        // the exponentials do not depend on this block's maximum, which only
        // checks the headroom, so the two run side by side; kEmuPer8 of every 8
        // pairs take the FMA-pipe exponential, the rest MUFU, so that neither
        // unit alone sets the pace of the block
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
        // P_g half row -> TMEM over the S columns this thread has read (A operand
        // of the PV MMA): 64 bf16 keys packed two per 32-bit column
        {
          uint32_t pk[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) pk[i] = pack_bf16x2(s[2 * i], s[2 * i + 1]);
          tmem_st32(tSg + sb * 128, reinterpret_cast<const float*>(pk));
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[sb]);
      }

      // last PV of the pass, then publish (largest logit, sum) and the headroom check
      if (ok && j > jb) ok = __all_sync(0xffffffffu, mbar_wait(o_done, pass & 1, abort_flag));
      if (ok) {
        xchg[g * 128 + q_row] = make_float2(m_seen, l);
        if (ovf) *redo_flag = 1;
        __syncwarp();
        if (lane == 0) mbar_arrive(x_full);
        ok = __all_sync(0xffffffffu, mbar_wait(x_full, pass & 1, abort_flag));
      }
      if (ok) {
        tc_fence_after();   // the last PV completed before the arrivals
        const float2 s0 = xchg[q_row], s1 = xchg[128 + q_row];
        if (pass == 0 && *redo_flag != 0) {
          // second pass: the row's largest logit becomes its reference
          const float mr = fmaxf(s0.x, s1.x);
          m_ref = (mr == kNegInf) ? 0.f : mr * scale_log2;
        } else {
          const float lt = s0.y + s1.y;     // both halves against the same reference
          const float inv = lt > 0.f ? 1.f / lt : 0.f;
          // this half writes output columns [g*C/2, (g+1)*C/2)
          bf16* orow = O + ((size_t)bh * M + (size_t)r * 128 + q_row) * C + g * (C / 2);
          const uint32_t tO0 = tmem + lane_off + L::kColO + g * (C / 2);
#pragma unroll
          for (int q = 0; q < C / 64; ++q) {
            float a[32];
            tmem_ld32(tO0 + q * 32, a);
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
              *reinterpret_cast<uint4*>(orow + q * 32 + i) = v;
            }
          }
          if (lse != nullptr && g == 0)
            lse[(size_t)bh * M + (size_t)r * 128 + q_row] =
                lt > 0.f ? (m_ref + lg2(lt)) * kLn2 : kNegInf;
        }
      }
      tc_fence_before();
      jb = j;
    }
    __syncthreads();
    // a second pass, only when some row outgrew its reference: every role walks
    // the same list again (jb blocks done), its barrier phases carried on
    if (pass != 0 || *redo_flag == 0 || *abort_flag != 0) break;
  }

  // drain: all MMAs issued by the two issuers complete before TMEM is freed
  if ((warp == 1 || warp == 2) && lane == 0) {
    mma_commit(&drain[warp - 1]);
    volatile int no_abort = 0;
    mbar_wait(&drain[warp - 1], 0, &no_abort);
  }
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace xattn
