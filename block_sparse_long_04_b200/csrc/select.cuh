// Threshold block selection -> CSR kept lists (XAttention summary, Approach;
// FlexPrefill rebuttal, R Q3: the minimal set reaching the cumulative threshold
// is the prefix of the descending order).
//
// Three launches:
//   select_count  one CTA per row (b, h, r): find the cut of the row's candidate
//                 scores (descending, ties to the smaller block index): the first
//                 position whose cumulative sum reaches tau, by a radix search
//                 over the score ranks with exact per-bin masses (no sort), and
//                 record the cut key (score, index) and the kept count (with the
//                 diagonal added if it falls below the cut).
//   select_scan   one CTA: exclusive scan of the counts into row_ptr and nnz;
//                 if nnz exceeds the capacity, every row_ptr entry becomes 0 and
//                 the device error word is set.
//   select_fill   one CTA per row: a block c is kept iff its (score, index) key
//                 ranks at or before the cut key, or c is the diagonal; kept
//                 indices are compacted in ascending order.
#pragma once
#include "common.cuh"

namespace xattn {

constexpr int kSelThreads = 256;

// How the cut of a sorted row is placed.
enum SelRule : int {
  kSelThreshold = 0,   // shortest prefix whose cumulative score reaches param (tau)
  kSelTopK = 1,        // the floor(param) highest-ranked candidates (at least one)
  kSelRatio = 2,       // ceil(param * candidates) highest-ranked, taken in fp64
};
constexpr int kSelMaxNb = 8192;   // candidates per row held in shared memory

struct SelCut {
  float score;   // score of the last block kept by thresholding
  int index;     // its block index
  int count;     // kept entries of the row, diagonal included
};

constexpr int kSelMaxGroup = 64;  // query heads per KV head for GQA-shared lists

// a ranks before b: higher score first, equal scores by smaller index
__device__ __forceinline__ bool ranks_before(float sa, int ia, float sb, int ib) {
  return sa > sb || (sa == sb && ia < ib);
}

__device__ __forceinline__ int block_exclusive_scan_i32(int v, int* red, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) red[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < (int)(blockDim.x >> 5) ? red[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    red[lane] = w;
  }
  __syncthreads();
  const int before = (warp > 0 ? red[warp - 1] : 0) + (x - v);
  total = red[(blockDim.x >> 5) - 1];
  __syncthreads();
  return before;
}

// 32-bit rank of a score for an ascending sort that puts higher scores first:
// the float bits mapped to an order-preserving unsigned, then inverted.
__device__ __forceinline__ uint32_t desc_rank(float s) {
  const uint32_t u = __float_as_uint(s);
  return ~((u & 0x80000000u) ? ~u : (u | 0x80000000u));
}
__device__ __forceinline__ float rank_score(uint32_t rk) {
  const uint32_t o = ~rk;
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o);
}

// Exclusive scan of one fp64 value per thread over a group of NT threads (whole
// warps) that share `sync` as their barrier; red holds NT/32 doubles.
template <int NT, typename Sync>
__device__ __forceinline__ double group_exclusive_scan_f64(double v, double* red, int tid, Sync sync) {
  const int lane = tid & 31, warp = tid >> 5;
  double x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  // the exclusive value is the previous lane's inclusive one (not x - v, which
  // is NaN when v is infinite)
  double before = __shfl_up_sync(0xffffffffu, x, 1);
  if (lane == 0) before = 0.0;
  if (lane == 31) red[warp] = x;
  sync();
  for (int w = 0; w < warp; ++w) before += red[w];
  sync();
  return before;
}

// Ascending bitonic sort of P = 256 * E 64-bit keys by 256 threads, thread t
// holding entries tE .. tE+E-1 in registers: compare-exchange partners at
// distance j < E are in the same thread, at E <= j < 32E in the same warp (a
// shuffle), and only the stages with j >= 32E go through shared memory. Each
// entry keeps the minimum of its pair when it is the pair's lower entry in an
// ascending run (or the upper one in a descending run), else the maximum.
template <int E>
__device__ __forceinline__ void bitonic_sort_256(uint64_t* keys, int tid) {
  constexpr int P = 256 * E;
  uint64_t v[E];
#pragma unroll
  for (int e = 0; e < E; ++e) v[e] = keys[tid * E + e];
#pragma unroll 1
  for (int k = 2; k <= P; k <<= 1) {
    // partners in other threads: shared memory or a shuffle
#pragma unroll 1
    for (int j = k >> 1; j >= E; j >>= 1) {
      if (j >= 32 * E) {
#pragma unroll
        for (int e = 0; e < E; ++e) keys[tid * E + e] = v[e];
        __syncthreads();
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int i = tid * E + e;
          const uint64_t o = keys[i ^ j];
          const bool take_min = ((i & j) == 0) == ((i & k) == 0);
          v[e] = take_min ? (o < v[e] ? o : v[e]) : (o > v[e] ? o : v[e]);
        }
        __syncthreads();
      } else {
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int i = tid * E + e;
          const uint64_t o = __shfl_xor_sync(0xffffffffu, v[e], j / E);
          const bool take_min = ((i & j) == 0) == ((i & k) == 0);
          v[e] = take_min ? (o < v[e] ? o : v[e]) : (o > v[e] ? o : v[e]);
        }
      }
    }
    // partners in the same thread (distance jj < E, known at compile time)
#pragma unroll
    for (int jj = E / 2; jj > 0; jj >>= 1) {
      if (jj < k) {
#pragma unroll
        for (int e = 0; e < E; ++e) {
          if ((e & jj) == 0) {
            const int i = tid * E + e;
            const uint64_t a = v[e], b = v[e ^ jj];
            if ((a > b) == ((i & k) == 0)) {
              v[e] = b;
              v[e ^ jj] = a;
            }
          }
        }
      }
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) keys[tid * E + e] = v[e];
}

// Number of candidates kept by the Top-K / ratio rules (and by a threshold that
// keeps everything): floor(t) (Top-K) or ceil(t * n) (ratio), in fp64 from the
// fp32 parameter, clamped to [1, n]; NaN keeps n.
__device__ __forceinline__ int select_rule_count(int rule, float t, int n) {
  if (rule == kSelThreshold) return n;
  double kk = rule == kSelTopK ? floor((double)t) : ceil((double)t * (double)n);
  kk = kk < 1.0 ? 1.0 : (kk > (double)n ? (double)n : kk);   // NaN -> n
  return (kk >= 1.0 && kk <= (double)n) ? (int)kk : n;
}

// The cut of one row by a full sort (rows holding a negative, infinite or NaN
// score; select_row_cut below handles every other row without sorting):
// bitonic sort of 64-bit keys (descending-score rank, then index) in shared
// memory, i.e. descending score, ascending index; then the cut position of the
// rule: the first prefix whose fp64 cumulative sum reaches t (threshold), or
// select_rule_count. keys holds P entries, P = next power of two >= n. The
// result is valid in thread 0 of the group.
template <int NT, typename Sync>
__device__ SelCut select_row_cut_sorted(const float* __restrict__ srow, int n, int r, float t,
                                        int rule, uint64_t* keys, double* red, int* first_hit,
                                        int tid, Sync sync) {
  int P = 1;
  while (P < n) P <<= 1;
  for (int i = tid; i < P; i += NT)
    keys[i] = i < n ? ((uint64_t)desc_rank(srow[i]) << 32) | (uint32_t)i
                    : ((uint64_t)desc_rank(kNegInf) << 32) | 0x7fffffffu;
  if (tid == 0) *first_hit = n - 1;
  sync();

  // bitonic network over one 64-bit word per entry (one load and one store per
  // side instead of separate score and index arrays); 256-thread groups sort
  // rows of 256 to 2048 entries mostly in registers
  bool sorted = false;
  if (NT == 256 && P >= 256) {
    sorted = true;
    switch (P / 256) {
      case 1: bitonic_sort_256<1>(keys, tid); break;
      case 2: bitonic_sort_256<2>(keys, tid); break;
      case 4: bitonic_sort_256<4>(keys, tid); break;
      case 8: bitonic_sort_256<8>(keys, tid); break;
      default: sorted = false;   // longer rows: the shared-memory network below
    }
    sync();
  }
  for (int k = 2; !sorted && k <= P; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < P; i += NT) {
        const int p = i ^ j;
        if (p > i) {
          const uint64_t a = keys[i], b = keys[p];
          if ((a > b) == ((i & k) == 0)) {
            keys[i] = b;
            keys[p] = a;
          }
        }
      }
      sync();
    }
  }

  if (rule != kSelThreshold) {
    // Top-K / ratio: the cut position follows from the candidate count alone
    if (tid == 0) *first_hit = select_rule_count(rule, t, n) - 1;
    sync();
  }
  // fp64 prefix sums over contiguous per-thread segments of the sorted order
  const int per = (n + NT - 1) / NT;
  const int lo = tid * per, hi = min(n, lo + per);
  double seg = 0.0;
  for (int i = lo; i < hi; ++i) seg += (double)rank_score((uint32_t)(keys[i] >> 32));
  double run = group_exclusive_scan_f64<NT>(seg, red, tid, sync);
  if (rule == kSelThreshold && t < 1.0f) {
    for (int i = lo; i < hi; ++i) {
      run += (double)rank_score((uint32_t)(keys[i] >> 32));
      if (run >= (double)t) { atomicMin(first_hit, i); break; }
    }
  }
  sync();
  SelCut cut;
  if (tid == 0) {
    const int k = *first_hit;
    cut.score = rank_score((uint32_t)(keys[k] >> 32));
    cut.index = (int)(uint32_t)keys[k];
    const bool diag_kept = r == cut.index || ranks_before(srow[r], r, cut.score, cut.index);
    cut.count = k + 1 + (diag_kept ? 0 : 1);
  }
  sync();   // key/idx/first_hit may be reused by the caller's next row
  return cut;
}

// Shared state of one row's cut search (select_row_cut).
struct SelRadix {
  // exact mass of each bin, in units of 2^(e0 - 150): mass_hi * 2^16 + mass_lo,
  // kept as two 32-bit sums so that every update is a native 32-bit atomic (a
  // candidate adds at most 2^25, a row holds at most kSelMaxNb = 2^13 of them)
  unsigned mass_lo[256];
  unsigned mass_hi[256];
  int count[256];                 // candidates in each bin
  double wmass[8];                // per-warp totals of a bin scan (groups of <= 256 threads)
  int wcount[8];
  double before;                  // mass of the candidates ranked before the prefix
  int before_cnt;                 // and their number
  int bin, last_bin;              // crossing bin of the pass; last non-empty bin
  int bin_count;                  // candidates in the crossing bin
  int e0;                         // exponent base of the masses (fixed by the first pass)
  int special;                    // the row holds a negative, infinite or NaN score
  int pick;                       // candidate index of the cut
  SelCut sorted_cut;              // the cut of a row that went to the full sort
};

// 2^k for an integer k in the normal fp64 range, exactly
__device__ __forceinline__ double pow2_f64(int k) {
  return __longlong_as_double((long long)(k + 1023) << 52);
}

// A finite non-negative fp32 score from its descending rank (desc_rank): its
// value is sig * 2^(e - 150) with a 24-bit integer sig and e >= 1.
__device__ __forceinline__ void rank_sig_exp(uint32_t rk, uint32_t& sig, int& e) {
  const uint32_t u = (~rk) & 0x7FFFFFFFu;
  const int E = (int)(u >> 23);
  sig = E ? ((u & 0x7FFFFFu) | 0x800000u) : (u & 0x7FFFFFu);
  e = E ? E : 1;
}

// The cut of one row of block scores (candidates 0..n-1, diagonal r) by a
// group of NT threads (NT a multiple of 32, at most 256), without sorting: a
// radix search over the 32-bit descending-score ranks, eight bits per pass from
// the top. A pass builds a 256-bin histogram of the candidates that share the
// prefix found so far, with each bin's count and its exact mass (the scores are
// added as integers, sig << (e - e0): every candidate left after the first pass
// has one of two neighbouring exponents), scans the bins in rank order in fp64
// (mass before the prefix + bins so far) and takes the first bin that reaches
// the target: the cumulative mass t (threshold) or the kept count of the Top-K /
// ratio rule. A bin holding one candidate ends the search; after four passes the
// remaining candidates share one score, and the cut falls inside that tie group
// (in index order, by adding the score in fp64 until t is reached). The result
// is the same (score, index) cut as taking the shortest prefix of the
// descending order (ties to the smaller index) whose cumulative mass reaches t
// (XAttention summary, Approach; FlexPrefill rebuttal, R Q3), up to the fp64
// rounding of the cumulative sums. A threshold t >= 1 (or NaN), or one that the
// whole row does not reach, keeps every candidate. Rows holding a negative,
// infinite or NaN score go to select_row_cut_sorted. `keys` holds P 64-bit
// entries (P = next power of two >= n); its first n 32-bit words hold the ranks.
// The result is valid in every thread of the group.
template <int NT, typename Sync>
__device__ SelCut select_row_cut(const float* __restrict__ srow, int n, int r, float t, int rule,
                                 uint64_t* keys, double* red, int* first_hit, SelRadix* st,
                                 int tid, Sync sync) {
  static_assert(NT % 32 == 0 && NT <= 256 && 256 % NT == 0, "group of 32..256 threads");
  constexpr int BPT = 256 / NT;                 // bins per thread in a scan
  uint32_t* ranks = reinterpret_cast<uint32_t*>(keys);
  const int lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    st->special = 0;
    st->before = 0.0;
    st->before_cnt = 0;
  }
  sync();
  bool special = false;
  auto rank_one = [&](int i, float s) {
    const uint32_t rk = desc_rank(s);
    special |= (rk & 0x80000000u) != 0 || !(s <= 3.4028234663852886e38f);   // negative, inf, NaN
    ranks[i] = rk;
  };
  // 16-byte loads when the row is 16-byte aligned (the first n & ~3 entries),
  // so that a thread's loads of the row are few and all in flight together
  int n4 = 0;
  if ((reinterpret_cast<uintptr_t>(srow) & 15u) == 0) {
    n4 = n & ~3;
    const float4* s4 = reinterpret_cast<const float4*>(srow);
#pragma unroll 4
    for (int q = tid; q < n4 / 4; q += NT) {
      const float4 v = s4[q];
      rank_one(4 * q, v.x);
      rank_one(4 * q + 1, v.y);
      rank_one(4 * q + 2, v.z);
      rank_one(4 * q + 3, v.w);
    }
  }
  for (int i = n4 + tid; i < n; i += NT) rank_one(i, srow[i]);
  if (special) st->special = 1;
  sync();
  if (st->special) {
    SelCut cut = select_row_cut_sorted<NT>(srow, n, r, t, rule, keys, red, first_hit, tid, sync);
    if (tid == 0) st->sorted_cut = cut;   // valid in thread 0: hand it to the group
    sync();
    cut = st->sorted_cut;
    sync();
    return cut;
  }

  // target: cumulative mass t (threshold rule, t < 1) or a kept count
  bool by_mass = rule == kSelThreshold && t < 1.0f;
  int K = select_rule_count(rule, t, n);
  uint32_t prefix = 0;
  int e0 = 0;
  bool found = false;
  for (int pass = 0; pass < 4 && !found; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int b = tid; b < 256; b += NT) {
      st->mass_lo[b] = 0u;
      st->mass_hi[b] = 0u;
      st->count[b] = 0;
    }
    if (tid == 0) { st->bin = 0x7fffffff; st->last_bin = -1; }
    sync();
    for (int base = 0; base < n; base += NT) {
      const int i = base + tid;
      const uint32_t rk = i < n ? ranks[i] : 0u;
      const bool valid = i < n && (pass == 0 || (rk >> (shift + 8)) == prefix);
      const int bin = (int)((rk >> shift) & 255u);
      uint32_t contrib = 0;
      if (by_mass && valid) {
        uint32_t sig;
        int e;
        rank_sig_exp(rk, sig, e);
        contrib = sig << (e - (pass == 0 ? 2 * (127 - bin) : e0));
      }
      if (pass == 0) {
        // the first pass bins by exponent pairs, so a warp's candidates share a
        // few bins: one set of atomics per group of lanes with the same bin (the
        // match costs more the more distinct values a warp holds)
        const unsigned peers = __match_any_sync(0xffffffffu, valid ? (unsigned)bin : 256u + lane);
        if (valid) {
          const unsigned mlo = by_mass ? __reduce_add_sync(peers, contrib & 0xFFFFu) : 0u;
          const unsigned mhi = by_mass ? __reduce_add_sync(peers, contrib >> 16) : 0u;
          if (lane == __ffs(peers) - 1) {
            atomicAdd(&st->count[bin], __popc(peers));
            if (by_mass) {
              atomicAdd(&st->mass_lo[bin], mlo);
              atomicAdd(&st->mass_hi[bin], mhi);
            }
          }
        }
      } else if (valid) {
        // later passes spread a warp's candidates over many bins: plain atomics
        atomicAdd(&st->count[bin], 1);
        if (by_mass) {
          atomicAdd(&st->mass_lo[bin], contrib & 0xFFFFu);
          atomicAdd(&st->mass_hi[bin], contrib >> 16);
        }
      }
    }
    sync();
    // scan of the bins in rank order: thread tid owns bins tid*BPT .. tid*BPT+BPT-1
    double lm[BPT];
    int lc[BPT];
    double tm = 0.0;
    int tc = 0, my_last = -1;
#pragma unroll
    for (int k = 0; k < BPT; ++k) {
      const int b = tid * BPT + k;
      lc[k] = st->count[b];
      lm[k] = (by_mass && lc[k])
                  ? (double)(((unsigned long long)st->mass_hi[b] << 16) + st->mass_lo[b]) *
                        pow2_f64((pass == 0 ? 2 * (127 - b) : e0) - 150)
                  : 0.0;
      tm += lm[k];
      tc += lc[k];
      if (lc[k]) my_last = b;
    }
    // one shared atomic per warp: the last non-empty bin
    my_last = __reduce_max_sync(0xffffffffu, my_last);
    if (lane == 0 && my_last >= 0) atomicMax(&st->last_bin, my_last);
    double xm = tm;
    int xc = tc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double ym = __shfl_up_sync(0xffffffffu, xm, o);
      const int yc = __shfl_up_sync(0xffffffffu, xc, o);
      if (lane >= o) { xm += ym; xc += yc; }
    }
    if (lane == 31) { st->wmass[warp] = xm; st->wcount[warp] = xc; }
    sync();
    double run = xm - tm;
    int runc = xc - tc;
    for (int w2 = 0; w2 < warp; ++w2) { run += st->wmass[w2]; runc += st->wcount[w2]; }
    const double before = st->before;
    const int before_cnt = st->before_cnt;
    if (pass == 0 && by_mass) {
      // a threshold the whole row does not reach keeps every candidate
      double total = 0.0;
      for (int w2 = 0; w2 < NT / 32; ++w2) total += st->wmass[w2];
      if (!(total >= (double)t)) { by_mass = false; K = n; }
    }
    double excl_m = run;
    int excl_c = runc;
    int my_hit = 0x7fffffff;   // this thread's first bin that reaches the target
#pragma unroll
    for (int k = 0; k < BPT; ++k) {
      const double incl_m = excl_m + lm[k];
      const int incl_c = excl_c + lc[k];
      const bool hit = lc[k] > 0 && (by_mass ? before + incl_m >= (double)t
                                             : before_cnt + incl_c >= K);
      if (hit && my_hit == 0x7fffffff) my_hit = tid * BPT + k;
      excl_m = incl_m;
      excl_c = incl_c;
    }
    // one shared atomic per warp: the first bin of the group that reaches it
    my_hit = (int)__reduce_min_sync(0xffffffffu, (unsigned)my_hit);
    if (lane == 0 && my_hit != 0x7fffffff) atomicMin(&st->bin, my_hit);
    sync();
    // rounding may leave the bin sums just short of what the previous pass saw:
    // the crossing then lies in the last non-empty bin
    const int b = st->bin != 0x7fffffff ? st->bin : st->last_bin;
    if (b / BPT == tid) {
      double em = run;
      int ec = runc;
      for (int k = 0; k < b % BPT; ++k) { em += lm[k]; ec += lc[k]; }
      st->before = before + em;
      st->before_cnt = before_cnt + ec;
      st->bin_count = lc[b % BPT];
      if (pass == 0) st->e0 = 2 * (127 - b);
    }
    sync();
    if (pass == 0) e0 = st->e0;
    prefix = (pass == 0) ? (uint32_t)b : ((prefix << 8) | (uint32_t)b);
    if (st->bin_count == 1) {
      // a single candidate in the crossing bin: it is the cut
      for (int i = tid; i < n; i += NT)
        if ((ranks[i] >> shift) == prefix) st->pick = i;
      found = true;
    }
    sync();
  }
  int j = 1;   // position of the cut inside the tie group (1-based)
  if (!found) {
    // four passes: `prefix` is one exact score shared by bin_count candidates,
    // taken in ascending index order
    const int cnt = st->bin_count;
    if (by_mass) {
      const double sv = (double)rank_score(prefix);
      double cum = st->before;
      j = cnt;
      for (int q = 1; q <= cnt; ++q) {
        cum += sv;
        if (cum >= (double)t) { j = q; break; }
      }
    } else {
      j = K - st->before_cnt;
      j = j < 1 ? 1 : (j > cnt ? cnt : j);
    }
    // the j-th smallest index among the tie group: contiguous segments per thread
    const int per = (n + NT - 1) / NT;
    const int lo = tid * per, hi = min(n, lo + per);
    int mine = 0;
    for (int i = lo; i < hi; ++i) mine += ranks[i] == prefix ? 1 : 0;
    int xs = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, xs, o);
      if (lane >= o) xs += y;
    }
    if (lane == 31) st->wcount[warp] = xs;
    sync();
    int seen = xs - mine;
    for (int w2 = 0; w2 < warp; ++w2) seen += st->wcount[w2];
    if (seen < j && seen + mine >= j) {
      for (int i = lo; i < hi; ++i)
        if (ranks[i] == prefix && ++seen == j) { st->pick = i; break; }
    }
    sync();
  }
  SelCut cut;
  cut.index = st->pick;
  cut.score = rank_score(ranks[cut.index]);
  const bool diag_kept = r == cut.index || ranks_before(srow[r], r, cut.score, cut.index);
  cut.count = st->before_cnt + (found ? 1 : j) + (diag_kept ? 0 : 1);
  sync();   // ranks and the search state may be reused by the caller's next row
  return cut;
}

// block c of row r is kept under the row's cut (the diagonal always is)
__device__ __forceinline__ bool kept_by_cut(float s, int c, int r, const SelCut& cut) {
  return c == r || ranks_before(s, c, cut.score, cut.index) || (s == cut.score && c == cut.index);
}

// Exclusive scan of one int per thread over a group of NT threads (whole warps)
// that share `sync` as their barrier; red holds NT/32 ints. total = the sum.
template <int NT, typename Sync>
__device__ __forceinline__ int group_exclusive_scan_i32(int v, int* red, int tid, Sync sync,
                                                        int& total) {
  const int lane = tid & 31, warp = tid >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) red[warp] = x;
  sync();
  int before = x - v;
  total = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) {
    const int t = red[w];
    if (w < warp) before += t;
    total += t;
  }
  sync();
  return before;
}

// Named barrier of group grp (id 1 + grp, NT threads), or the CTA barrier when
// the CTA holds one group; the ids are constants so that the kernel reserves
// only the barriers it uses.
template <int RPC, int NT>
__device__ __forceinline__ void group_sync(int grp) {
  static_assert(RPC == 1 || RPC == 2 || RPC == 4, "one to four groups per CTA");
  if (RPC == 1) {
    __syncthreads();
    return;
  }
  switch (grp) {
    case 0: asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory"); break;
    case 1: asm volatile("bar.sync 2, %0;" ::"n"(NT) : "memory"); break;
    case 2: asm volatile("bar.sync 3, %0;" ::"n"(NT) : "memory"); break;
    default: asm volatile("bar.sync 4, %0;" ::"n"(NT) : "memory"); break;
  }
}

// One CTA of kSelThreads threads holds RPC rows, a group of NT = kSelThreads /
// RPC threads per row with its own named barrier; `keys` (dynamic shared
// memory) holds P 64-bit entries per group. Short rows run four to a CTA (64
// threads each): the cut search's fixed cost per pass is paid by fewer threads.
template <int RPC>
__global__ void __launch_bounds__(kSelThreads)
select_count_kernel(const float* __restrict__ scores, const float* __restrict__ tau, int Hq, int nb,
                    int causal, SelCut* __restrict__ cuts, int rule, int rows, int P) {
  constexpr int NT = kSelThreads / RPC;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ double red[RPC][NT / 32];
  __shared__ int first_hit[RPC];
  __shared__ SelRadix st[RPC];
  const int grp = (int)threadIdx.x / NT, tid = (int)threadIdx.x % NT;
  const int row = blockIdx.x * RPC + grp;
  if (row >= rows) return;   // whole groups leave; the others sync on their own barriers
  const int bh = row / nb, r = row % nb, h = bh % Hq;
  const int n = causal ? r + 1 : nb;
  uint64_t* keys = reinterpret_cast<uint64_t*>(smem) + (size_t)grp * P;
  auto sync = [grp] { group_sync<RPC, NT>(grp); };   // each group its own barrier
  const SelCut cut = select_row_cut<NT>(scores + (size_t)row * nb, n, r, tau[h], rule, keys,
                                        red[grp], &first_hit[grp], &st[grp], tid, sync);
  if (tid == 0) cuts[row] = cut;
}

// Rows of at most this many candidates run four to a CTA.
constexpr int kSelShortRow = 2048;

// One CTA: the rows' counts go through shared memory in chunks of 8192 (loads
// and stores of consecutive rows by consecutive threads), each thread scanning
// eight neighbouring counts, the running total carried from chunk to chunk.
__global__ void __launch_bounds__(1024)
select_scan_kernel(const SelCut* __restrict__ cuts, int rows, int32_t* __restrict__ row_ptr,
                   int32_t* __restrict__ nnz, long long capacity) {
  constexpr int kPer = 8, kChunk = kPer * 1024;
  __shared__ int cnt[kChunk];
  __shared__ int red[32];
  const int tid = threadIdx.x;
  int carry = 0;
  for (int base = 0; base < rows; base += kChunk) {
    const int m = min(kChunk, rows - base);
    for (int i = tid; i < m; i += 1024) cnt[i] = cuts[base + i].count;
    __syncthreads();
    int loc[kPer], seg = 0;
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      const int i = tid * kPer + e;
      loc[e] = i < m ? cnt[i] : 0;
      seg += loc[e];
    }
    int total;
    int run = carry + block_exclusive_scan_i32(seg, red, total);
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      const int i = tid * kPer + e;
      if (i < m) cnt[i] = run;
      run += loc[e];
    }
    __syncthreads();
    for (int i = tid; i < m; i += 1024) row_ptr[base + i] = cnt[i];
    carry += total;
    __syncthreads();   // cnt is refilled by the next chunk
  }
  // over capacity: every list is withdrawn (row_ptr all 0) and the error raised;
  // each entry is zeroed by the thread that wrote it above
  const bool over = (long long)carry > capacity;
  if (over)
    for (int i = tid; i < rows; i += 1024) row_ptr[i] = 0;
  if (tid == 0) {
    row_ptr[rows] = over ? 0 : carry;
    nnz[0] = carry;
    if (over) raise_device_error(2 /* XATTN_ECAPACITY */);
  }
}

// RPC rows per CTA (a group of NT = kSelThreads / RPC threads per row, each
// thread a contiguous segment of the row), kept indices in ascending order.
template <int RPC>
__global__ void __launch_bounds__(kSelThreads)
select_fill_kernel(const float* __restrict__ scores, const SelCut* __restrict__ cuts, int nb,
                   int causal, const int32_t* __restrict__ row_ptr, int32_t* __restrict__ col_idx,
                   int rows) {
  constexpr int NT = kSelThreads / RPC;
  __shared__ int red[RPC][NT / 32];
  const int grp = (int)threadIdx.x / NT, tid = (int)threadIdx.x % NT;
  const int row = blockIdx.x * RPC + grp;
  if (row >= rows) return;   // whole groups leave; the others sync on their own barriers
  const int r = row % nb;
  const int n = causal ? r + 1 : nb;
  const SelCut cut = cuts[row];
  const int base = row_ptr[row];
  if (row_ptr[row + 1] - base != cut.count) return;   // lists withdrawn (capacity)
  const float* srow = scores + (size_t)row * nb;
  const int per = (n + NT - 1) / NT;
  const int lo = tid * per, hi = min(n, lo + per);
  auto kept = [&](int c) { return kept_by_cut(srow[c], c, r, cut); };
  int cnt = 0;
  for (int c = lo; c < hi; ++c) cnt += kept(c) ? 1 : 0;
  int total;
  int pos = group_exclusive_scan_i32<NT>(cnt, red[grp], tid, [grp] { group_sync<RPC, NT>(grp); },
                                         total);
  // the row's count bounds the writes even if cuts and scores disagree
  for (int c = lo; c < hi && pos < cut.count; ++c)
    if (kept(c)) col_idx[base + pos++] = c;
}

// ---- GQA-shared lists ------------------------------------------------------
// Block c of query block r is kept for KV group (b, kvh) when any query head of
// the group keeps it under its own cut. One CTA per group row
// (b * Hkv + kvh) * nb + r; the G = Hq / Hkv member rows are
// (b * Hq + kvh * G + i) * nb + r.
struct GroupRow {
  int r, n, G;
  size_t row0;   // first member row
  __device__ __forceinline__ GroupRow(int grow, int Hq, int Hkv, int nb, int causal) {
    const int bk = grow / nb;
    r = grow % nb;
    n = causal ? r + 1 : nb;
    G = Hq / Hkv;
    row0 = ((size_t)(bk / Hkv) * Hq + (size_t)(bk % Hkv) * G) * nb + r;
  }
};

__device__ __forceinline__ bool group_keeps(const float* __restrict__ scores, const SelCut* cut_s,
                                            const GroupRow& g, int nb, int c) {
  bool any = false;
  for (int i = 0; i < g.G && !any; ++i)
    any = kept_by_cut(scores[(g.row0 + (size_t)i * nb) * nb + c], c, g.r, cut_s[i]);
  return any;
}

__global__ void __launch_bounds__(kSelThreads)
select_group_count_kernel(const float* __restrict__ scores, const SelCut* __restrict__ cuts,
                          int Hq, int Hkv, int nb, int causal, SelCut* __restrict__ gcuts) {
  __shared__ int red[32];
  __shared__ SelCut cut_s[kSelMaxGroup];
  const GroupRow g((int)blockIdx.x, Hq, Hkv, nb, causal);
  for (int i = threadIdx.x; i < g.G; i += kSelThreads) cut_s[i] = cuts[g.row0 + (size_t)i * nb];
  __syncthreads();
  int cnt = 0;
  for (int c = threadIdx.x; c < g.n; c += kSelThreads) cnt += group_keeps(scores, cut_s, g, nb, c);
  int total;
  block_exclusive_scan_i32(cnt, red, total);
  if (threadIdx.x == 0) gcuts[blockIdx.x] = SelCut{0.f, 0, total};
}

__global__ void __launch_bounds__(kSelThreads)
select_group_fill_kernel(const float* __restrict__ scores, const SelCut* __restrict__ cuts,
                         const SelCut* __restrict__ gcuts, int Hq, int Hkv, int nb, int causal,
                         const int32_t* __restrict__ row_ptr, int32_t* __restrict__ col_idx) {
  __shared__ int red[32];
  __shared__ SelCut cut_s[kSelMaxGroup];
  const int grow = blockIdx.x;
  const GroupRow g(grow, Hq, Hkv, nb, causal);
  const int base = row_ptr[grow];
  const int count = gcuts[grow].count;
  if (row_ptr[grow + 1] - base != count) return;   // lists withdrawn (capacity)
  for (int i = threadIdx.x; i < g.G; i += kSelThreads) cut_s[i] = cuts[g.row0 + (size_t)i * nb];
  __syncthreads();
  const int per = (g.n + kSelThreads - 1) / kSelThreads;
  const int lo = threadIdx.x * per, hi = min(g.n, lo + per);
  int cnt = 0;
  for (int c = lo; c < hi; ++c) cnt += group_keeps(scores, cut_s, g, nb, c);
  int total;
  int pos = block_exclusive_scan_i32(cnt, red, total);
  for (int c = lo; c < hi && pos < count; ++c)
    if (group_keeps(scores, cut_s, g, nb, c)) col_idx[base + pos++] = c;
}

}  // namespace xattn
