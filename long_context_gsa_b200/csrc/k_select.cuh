// k_select.cuh -- top-k chunk selection of one row by a whole CTA, run in the
// prologue of the unfold kernel so that a decode step needs no separate
// selection launch.
//
// Method: "Selectie" on gist.science/nl/paper/2604.20920 ("Het Proces"): the
// k gists of highest relevance s = q.k_g are kept; gist.science/ja section
// 2.1 step 3.  Equal scores go to the lower chunk index (the pages leave ties
// open).
//
// Inputs: the row's scores (fp32, written by the scoring pass and still in
// L2) and its group maxima: the maximum score of every 16 consecutive gists,
// which the scoring pass produces on the side (one shuffle per group).
//
// Fast path (a bound, then a few candidates):
//  1. the kk-th largest group maximum bounds the row's kk-th score from
//     below (kk groups, hence kk distinct gists, reach it).  Two 8-bit radix
//     passes over the order-preserving keys of the group maxima find the
//     bin holding it; L = the lower edge of that bin (16 key bits, about one
//     part in 128 of the score) is a slightly looser bound that needs no
//     further passes.  Rows with fewer than kk groups use the scores
//     themselves as the "groups" of one;
//  2. candidates: the scores >= L inside the groups whose maximum reaches L
//     (in practice about 1.2 kk of them);
//  3. the kk-th largest (score key, inverted index) rank key among them, by
//     two warps sorting 128 each and a merge search, or by counting ranks;
//  4. the candidates reaching that rank key are exactly the kk selected
//     chunks (rank keys are distinct); each one's place in ascending chunk
//     order is the number of selected chunks below it.
// Exact fallback (too many candidates, e.g. long runs of equal scores, or a
// row too long for the group list): an 8-bit radix select over all the
// row's scores finds the kk-th largest key T; the selection is every key
// above T plus the lowest-indexed keys equal to T, written in ascending
// chunk order by a block-wide ordered compaction.
#pragma once

#include "common.cuh"
#include "k_topk.cuh"  // warp_sort_desc

namespace gsa {

constexpr int kSelGroup = 16;       // gists per group maximum
constexpr int kRowSelThreads = 128;    // threads of the selecting CTA
constexpr int kSelGroupCap = 1024;  // group (or score) list the fast path takes
constexpr int kSelCandCap = 1024;   // candidates the fast path ranks

// Scratch of one selection; aliases memory the caller does not use yet.
struct SelectSmem {
  unsigned long long cand[kSelCandCap];
  int cg[kSelGroupCap];
  uint32_t hist[256];
  int wtot[2][kRowSelThreads / 32];
  unsigned long long kth;
  int info[4];
  int ncg, ncand;
};

__device__ __forceinline__ unsigned long long sel_rank_key(uint32_t key, int i) {
  return (static_cast<unsigned long long>(key) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(i));
}

// Warp 0 finds the digit bin of rank `rem` (1-based, from the top) in the
// 256-bin histogram: info[0] = digit, info[1] = entries in higher bins,
// info[2] = entries in the digit's bin.
__device__ __forceinline__ void sel_find_digit(SelectSmem &sm, int rem) {
  const int lane = threadIdx.x & 31;
  uint32_t c[8], tot = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    c[e] = sm.hist[lane * 8 + e];
    tot += c[e];
  }
  uint32_t incl = tot;  // bins of lanes >= lane
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_down_sync(0xffffffffu, incl, o);
    if (lane + o < 32) incl += v;
  }
  uint32_t cum = incl - tot;
#pragma unroll
  for (int e = 7; e >= 0; --e) {
    if (cum < static_cast<uint32_t>(rem) && cum + c[e] >= static_cast<uint32_t>(rem)) {
      sm.info[0] = lane * 8 + e;
      sm.info[1] = static_cast<int>(cum);
      sm.info[2] = static_cast<int>(c[e]);
    }
    cum += c[e];
  }
}

// Exclusive prefix sum over the block's threads (kRowSelThreads).
__device__ __forceinline__ int sel_block_scan(int v, int (&wtot)[kRowSelThreads / 32]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) wtot[warp] = incl;
  __syncthreads();
  int before = 0;
  for (int w = 0; w < warp; ++w) before += wtot[w];
  __syncthreads();
  return before + incl - v;
}

// Exact selection over all n scores (the fallback).  Writes the kk chosen
// chunks in ascending order to out_idx / out_score.
__device__ __noinline__ void select_row_radix(const float *srow, int n, int kk, SelectSmem &sm, int *out_idx,
                                              float *out_score) {
  const int tid = threadIdx.x;
  uint32_t prefix = 0, pmask = 0;
  int rem = kk;
  bool take_all_eq = false;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kRowSelThreads) sm.hist[i] = 0u;
    __syncthreads();
    for (int i = tid; i < n; i += kRowSelThreads) {
      const uint32_t key = float_to_key(__ldcg(srow + i));
      if ((key & pmask) == prefix) atomicAdd(&sm.hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid < 32) sel_find_digit(sm, rem);
    __syncthreads();
    rem -= sm.info[1];
    prefix |= static_cast<uint32_t>(sm.info[0]) << shift;
    pmask |= 0xFFu << shift;
    const bool whole = sm.info[2] == rem;
    __syncthreads();
    if (whole) {
      take_all_eq = true;
      break;
    }
  }
  // ordered compaction over thread-contiguous index ranges
  const int per = (n + kRowSelThreads - 1) / kRowSelThreads;
  const int i0 = min(n, tid * per), i1 = min(n, i0 + per);
  int my_gt = 0, my_eq = 0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t km = float_to_key(__ldcg(srow + i)) & pmask;
    my_gt += km > prefix;
    my_eq += km == prefix;
  }
  const int eq_base = sel_block_scan(my_eq, sm.wtot[0]);
  const int my_take_eq = take_all_eq ? my_eq : max(0, min(my_eq, rem - eq_base));
  int pos = sel_block_scan(my_gt + my_take_eq, sm.wtot[1]);
  int eq_seen = 0;
  for (int i = i0; i < i1; ++i) {
    const float s = __ldcg(srow + i);
    const uint32_t km = float_to_key(s) & pmask;
    bool sel = km > prefix;
    if (km == prefix) sel = eq_seen++ < my_take_eq;
    if (sel && pos < kk) {
      out_idx[pos] = i;
      out_score[pos] = s;
      ++pos;
    }
  }
  __syncthreads();
}

// The kk (0 < kk < n) highest-scoring chunks of a row, in ascending chunk
// order, into out_idx / out_score (shared memory).  srow: the row's n
// scores; gmax: its ceil(n / kSelGroup) group maxima.  Called by the whole
// block (kRowSelThreads threads).
__device__ void select_row(const float *srow, const float *gmax, int n, int kk, SelectSmem &sm, int *out_idx,
                           float *out_score) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_groups = (n + kSelGroup - 1) / kSelGroup;
  const bool by_group = n_groups >= kk;
  const float *vals = by_group ? gmax : srow;
  const int nv = by_group ? n_groups : n;
  const int gsize = by_group ? kSelGroup : 1;
  if (nv > kSelGroupCap) {  // block-uniform
    select_row_radix(srow, n, kk, sm, out_idx, out_score);
    return;
  }
  // 1. bound L from two radix passes over the value keys
  uint32_t prefix = 0, pmask = 0;
  int rem = kk;
  for (int shift = 24; shift >= 16; shift -= 8) {
    for (int i = tid; i < 256; i += kRowSelThreads) sm.hist[i] = 0u;
    __syncthreads();
    for (int i = tid; i < nv; i += kRowSelThreads) {
      const uint32_t key = float_to_key(__ldcg(vals + i));
      if ((key & pmask) == prefix) atomicAdd(&sm.hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (warp == 0) sel_find_digit(sm, rem);
    __syncthreads();
    rem -= sm.info[1];
    prefix |= static_cast<uint32_t>(sm.info[0]) << shift;
    pmask |= 0xFFu << shift;
    __syncthreads();
  }
  const uint32_t L = prefix;  // at least kk values have key >= L
  // 2. candidate groups, then the candidates inside them
  if (tid == 0) {
    sm.ncg = 0;
    sm.ncand = 0;
  }
  __syncthreads();
  for (int i = tid; i < nv; i += kRowSelThreads)
    if (float_to_key(__ldcg(vals + i)) >= L) sm.cg[atomicAdd(&sm.ncg, 1)] = i;
  __syncthreads();
  const int ncg = sm.ncg;
  for (int p = tid; p < ncg * gsize; p += kRowSelThreads) {
    const int m = sm.cg[p / gsize] * gsize + p % gsize;
    if (m < n) {
      const uint32_t key = float_to_key(__ldcg(srow + m));
      if (key >= L) {
        const int slot = atomicAdd(&sm.ncand, 1);
        if (slot < kSelCandCap) sm.cand[slot] = sel_rank_key(key, m);
      }
    }
  }
  __syncthreads();
  const int C = sm.ncand;
  if (C > kSelCandCap || C < kk) {  // block-uniform; C < kk only if the maxima do not match the scores
    select_row_radix(srow, n, kk, sm, out_idx, out_score);
    return;
  }
  // 3. the kk-th largest rank key
  if (C <= 256) {
    if (warp < 2 && 128 * warp < C) {
      unsigned long long v[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = 128 * warp + lane * 4 + e;
        v[e] = i < C ? sm.cand[i] : 0ull;
      }
      warp_sort_desc<4>(v, lane);
#pragma unroll
      for (int e = 0; e < 4; ++e) sm.cand[128 * warp + lane * 4 + e] = v[e];
    }
    __syncthreads();
    if (tid == 0) {  // i entries from the first list, kk - i from the second
      const unsigned long long *A = sm.cand, *Bl = sm.cand + 128;
      const int nA = min(C, 128), nB = C - nA;
      int lo = max(0, kk - nB), hi = min(kk, nA);
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (A[mid] > Bl[kk - mid - 1]) lo = mid + 1;
        else hi = mid;
      }
      const int j = kk - lo;
      const unsigned long long a_last = lo > 0 ? A[lo - 1] : ~0ull, b_last = j > 0 ? Bl[j - 1] : ~0ull;
      sm.kth = min(a_last, b_last);
    }
  } else {
    for (int t = tid; t < C; t += kRowSelThreads) {
      const unsigned long long x = sm.cand[t];
      int rank = 0;
      for (int u = 0; u < C; ++u) rank += sm.cand[u] > x;
      if (rank == kk - 1) sm.kth = x;
    }
  }
  __syncthreads();
  // 4. place the selected ones in ascending chunk order
  const unsigned long long K = sm.kth;
  const int nc = C <= 256 ? (C <= 128 ? 128 : 256) : C;  // sorted lists carry zero padding
  for (int t = tid; t < nc; t += kRowSelThreads) {
    const unsigned long long x = sm.cand[t];
    if (x >= K && x != 0ull) {
      const uint32_t inv = static_cast<uint32_t>(x);
      int pos = 0;
      for (int u = 0; u < nc; ++u) {
        const unsigned long long y = sm.cand[u];
        pos += (y >= K && static_cast<uint32_t>(y) > inv) ? 1 : 0;  // larger inverted index = lower chunk
      }
      if (pos < kk) {  // always, unless the group maxima do not belong to these scores
        out_idx[pos] = static_cast<int>(0xFFFFFFFFu - inv);
        out_score[pos] = key_to_float(static_cast<uint32_t>(x >> 32));
      }
    }
  }
  __syncthreads();
}

}  // namespace gsa
