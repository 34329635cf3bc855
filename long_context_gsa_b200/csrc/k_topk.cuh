// k_topk.cuh -- per-row top-k chunk selection.
//
// Method: "Selectie" on gist.science/nl/paper/2604.20920 ("Het Proces"):
// the k most relevant gists are kept; gist.science/ja section 2.1 step 3.
// Equal scores go to the lower chunk index (the pages leave ties open).
//
// One CTA per row.  Scores become order-preserving uint32 keys.  An 8-bit
// radix select finds the k-th largest key, stopping as soon as the boundary
// digit is taken whole; keys equal to the threshold are taken in index
// order, which is the lower-index tie rule.  The main kernel keeps the keys
// in registers (warp-contiguous index ranges, coalesced loads), aggregates
// the contended first-digit histogram per warp with match.any, and writes
// the selection by ballot compaction, so the output is in ascending chunk
// order and needs no sort.  Rows longer than 16384 use k_topk_mem.
#pragma once

#include "common.cuh"

namespace gsa {

struct TopkArgs {
  const float *scores;    // [rows, stride]
  int32_t stride;
  const int32_t *n_gists; // [B]; row count n = n_gists[b] / count_div ...
  int32_t count_div;
  const int32_t *counts;  // ... unless counts ([rows]) is given
  int32_t hq;             // b = row / hq
  int32_t k;              // <= kTopkMax
  const int32_t *id_map;  // optional [rows, stride]: reported id of position i
  int32_t *sel_idx;       // [rows, k]
  float *sel_score;       // [rows, k] or null
  uint32_t *counters;     // optional: counters[row] is re-armed to 0
  int32_t smem_cap;       // keys kept in shared memory when n <= smem_cap
  uint32_t *status;       // optional: device status word (GSA_DEVERR_* bits)
};

constexpr int kTopkThreads = 512;
constexpr int kTopkMax = 1024;

__device__ __forceinline__ int block_exclusive_scan_512(int v, int *warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int x = lane < kTopkThreads / 32 ? warp_tot[lane] : 0;
    int xi = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, xi, o);
      if (lane >= o) xi += t;
    }
    if (lane < kTopkThreads / 32) warp_tot[lane] = xi - x;
  }
  __syncthreads();
  const int r = incl - v + warp_tot[warp];
  __syncthreads();  // warp_tot may be reused by the next scan
  return r;
}

// Exclusive prefix sum in reversed thread order: for thread t, the sum of v
// over threads t+1 .. 511.
__device__ __forceinline__ int scan_excl_512_rev(int v, int *warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;  // sum over lanes >= lane within the warp
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_down_sync(0xffffffffu, incl, o);
    if (lane + o < 32) incl += t;
  }
  if (lane == 0) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = kTopkThreads / 32;
    int x = lane < nw ? warp_tot[lane] : 0;
    int xi = x;  // sum over warps >= lane
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_down_sync(0xffffffffu, xi, o);
      if (lane + o < 32) xi += t;
    }
    if (lane < nw) warp_tot[lane] = xi - x;  // sum over warps > lane
  }
  __syncthreads();
  const int r = incl - v + warp_tot[warp];
  __syncthreads();
  return r;
}

// Fallback for rows longer than the register-resident kernel handles:
// keys are re-read from shared or global memory on every pass.
__global__ void __launch_bounds__(kTopkThreads) k_topk_mem(const TopkArgs a) {
  constexpr int T = kTopkThreads;
  extern __shared__ __align__(16) uint32_t keys_sm[];
  __shared__ uint32_t hist[256];
  __shared__ unsigned long long cand[kTopkMax];
  __shared__ int info[4];
  __shared__ int warp_tot[32];
  __shared__ int cand_count;

  const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
  pdl_wait();
  const int b = row / a.hq;
  int n = a.counts ? a.counts[row] : a.n_gists[b] / a.count_div;
  n = min(max(n, 0), a.stride);
  const float *srow = a.scores + static_cast<size_t>(row) * a.stride;
  const bool in_smem = n <= a.smem_cap;
  if (in_smem)
    for (int i = tid; i < n; i += T) keys_sm[i] = float_to_key(__ldcg(srow + i));
  if (tid == 0) cand_count = 0;
  __syncthreads();
  auto key_at = [&](int i) -> uint32_t { return in_smem ? keys_sm[i] : float_to_key(__ldcg(srow + i)); };

  const int kk = min(a.k, n);
  uint32_t prefix = 0, pmask = 0;
  int rem = kk;             // still to take among keys matching `prefix`
  bool take_all_eq = kk == n;
  if (kk > 0 && kk < n) {
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += T) hist[i] = 0;
      __syncthreads();
      for (int i = tid; i < n; i += T) {
        const uint32_t key = key_at(i);
        if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (tid < 32) {
        uint32_t c[8], tot = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          c[e] = hist[lane * 8 + e];
          tot += c[e];
        }
        uint32_t incl = tot;  // sum of lanes >= lane
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t v = __shfl_down_sync(0xffffffffu, incl, o);
          if (lane + o < 32) incl += v;
        }
        uint32_t cum = incl - tot;  // keys in higher bins
        int found = -1;
        uint32_t found_above = 0;
#pragma unroll
        for (int e = 7; e >= 0; --e) {
          if (found < 0 && cum < static_cast<uint32_t>(rem) && cum + c[e] >= static_cast<uint32_t>(rem)) {
            found = lane * 8 + e;
            found_above = cum;
          }
          cum += c[e];
        }
        const unsigned ball = __ballot_sync(0xffffffffu, found >= 0);
        const int src = ball ? __ffs(ball) - 1 : 0;
        const int digit = __shfl_sync(0xffffffffu, found, src);
        const uint32_t above = __shfl_sync(0xffffffffu, found_above, src);
        if (lane == 0) {
          info[0] = digit;
          info[1] = static_cast<int>(above);
          info[2] = digit >= 0 ? static_cast<int>(hist[digit]) : 0;
        }
      }
      __syncthreads();
      const int digit = info[0];
      rem -= info[1];
      prefix |= static_cast<uint32_t>(digit & 255) << shift;
      pmask |= 0xFFu << shift;
      if (info[2] == rem) {
        take_all_eq = true;
        break;
      }
      __syncthreads();
    }
  }

  // Collect: keys above the boundary, then boundary keys in index order.
  if (kk > 0) {
    const int per = (n + T - 1) / T;
    const int i0 = min(n, tid * per), i1 = min(n, i0 + per);
    int my_eq = 0;
    if (!take_all_eq)
      for (int i = i0; i < i1; ++i) my_eq += (key_at(i) & pmask) == prefix;
    const int eq_base = block_exclusive_scan_512(my_eq, warp_tot);
    int eq_seen = 0;
    for (int i = i0; i < i1; ++i) {
      const uint32_t key = key_at(i), km = key & pmask;
      bool sel = km > prefix;
      if (km == prefix) {
        sel = take_all_eq || (eq_base + eq_seen < rem);
        ++eq_seen;
      }
      if (sel) {
        const int slot = atomicAdd(&cand_count, 1);
        if (slot < kTopkMax)
          cand[slot] = (static_cast<unsigned long long>(key) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(i));
      }
    }
  }
  __syncthreads();

  // the kk selected entries, sorted to ascending chunk order (descending
  // inverted index; the zero padding sorts last)
  int P = 1;
  while (P < kk) P <<= 1;
  for (int i = kk + tid; i < P; i += T) cand[i] = 0ull;
  __syncthreads();
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < P / 2; i += T) {
        const int lo = 2 * stride * (i / stride) + (i % stride), hi = lo + stride;
        const bool desc = (lo & size) == 0;
        const unsigned long long x = cand[lo], y = cand[hi];
        const uint32_t xi = static_cast<uint32_t>(x), yi = static_cast<uint32_t>(y);  // inverted indices
        if (desc ? (xi < yi) : (xi > yi)) {
          cand[lo] = y;
          cand[hi] = x;
        }
      }
      __syncthreads();
    }
  }

  pdl_trigger();
  int32_t *out_i = a.sel_idx + static_cast<size_t>(row) * a.k;
  float *out_s = a.sel_score ? a.sel_score + static_cast<size_t>(row) * a.k : nullptr;
  for (int i = tid; i < a.k; i += T) {
    int32_t id = -1;
    float sc = neg_inf();
    if (i < kk) {
      const unsigned long long c = cand[i];
      const int pos = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(c & 0xFFFFFFFFull));
      id = a.id_map ? a.id_map[static_cast<size_t>(row) * a.stride + pos] : pos;
      sc = key_to_float(static_cast<uint32_t>(c >> 32));
    }
    out_i[i] = id;
    if (out_s) out_s[i] = sc;
  }
  if (a.counters && tid == 0) a.counters[row] = 0u;
}


constexpr int kTopkRegThreads = 256;

struct BoundSmem {
  unsigned long long cand[1024];
  uint32_t wtop[kTopkRegThreads];       // the full warps' sorted thread maxima
  uint32_t wcnt[kTopkRegThreads / 32];  // per-warp counts of selected entries
  unsigned long long kth;               // the kk-th largest rank key
  uint32_t bound;
  int count;
};

// Rank key of chunk i: the order-preserving score key above, the inverted
// index below, so a larger value ranks first and equal scores go to the
// lower index.  Every valid entry's value is distinct and nonzero.
__device__ __forceinline__ unsigned long long rank_key(uint32_t key, int i) {
  return (static_cast<unsigned long long>(key) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(i));
}

// Descending bitonic sort of 32*E values by one warp, E per lane (element
// i = lane*E + e): pairs closer than E meet in registers, the rest through
// shuffles.
template <int E, typename K>
__device__ __forceinline__ void warp_sort_desc(K (&v)[E], int lane) {
#pragma unroll
  for (int size = 2; size <= 32 * E; size <<= 1)
#pragma unroll
    for (int j = size >> 1; j > 0; j >>= 1) {
      if (j < E) {
#pragma unroll
        for (int e = 0; e < E; ++e)
          if ((e & j) == 0) {
            const bool desc = ((lane * E + e) & size) == 0;
            const K x = v[e], y = v[e | j];
            v[e] = desc ? max(x, y) : min(x, y);
            v[e | j] = desc ? min(x, y) : max(x, y);
          }
      } else {
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int i = lane * E + e;
          const K o = __shfl_xor_sync(0xffffffffu, v[e], j / E);
          const bool keep_max = ((i & size) == 0) == ((i & j) == 0);
          v[e] = keep_max ? max(v[e], o) : min(v[e], o);
        }
      }
    }
}

constexpr int kTopkCandCap = 1024;  // candidates the bound path ranks in shared memory

// Top-k through a lower bound (0 < kk < n, kk <= 256):
//  1. the warps whose 32 lanes all hold entries sort their threads' maximum
//     keys (shuffles); one warp sorts their top R (16, or 32 when fewer
//     than 2 kk maxima would be sorted) and takes the kk-th largest, L: kk
//     distinct entries reach L, so it bounds the row's kk-th score key from
//     below;
//  2. every entry with key >= L is a candidate (in practice under 1.2 kk);
//  3. the candidate of rank kk - 1 among the candidates, by (score desc,
//     index asc), is the row's kk-th rank key: up to 256 candidates are
//     sorted by two warps (128 each) and the kk-th of the two lists found by
//     a binary search; more are ranked by counting (each against all);
//  4. the entries reaching that key (exactly kk: rank keys are distinct)
//     are written in ascending chunk order straight from the registers.
// Returns false (nothing written) when no bound can be taken or the
// candidates exceed the buffer; the caller then runs the radix select.
// Called by the whole block.
template <int KPT>
__device__ __forceinline__ bool topk_by_bound(const TopkArgs &a, int row, int n, int kk, const float *rs, int base,
                                              BoundSmem &sm) {
  constexpr int T = kTopkRegThreads, W = T / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // The loops over this thread's KPT entries (element base + 32 j of the
  // staged row) are only partly unrolled: each phase runs once per block,
  // so its instructions are fetched cold whenever an earlier kernel has
  // streamed through L2, and a fully unrolled body costs more in fetch
  // stalls than the loop does in issue.
  auto key_at = [&](int j) -> uint32_t {
    const int i = base + 32 * j;
    return i < n ? float_to_key(rs[i]) : 0u;  // valid keys are nonzero; 0 marks "no entry"
  };
  uint32_t m = 0u;
#pragma unroll 4
  for (int j = 0; j < KPT; ++j) m = max(m, key_at(j));
  {
    uint32_t v[1] = {m};
    warp_sort_desc<1>(v, lane);
    m = v[0];
  }
  const int w_full = n >= 32 ? min(W, (n - 32) / (32 * KPT) + 1) : 0;  // warps w with w*32*KPT + 31 < n
  const int R = w_full * 16 >= 2 * kk ? 16 : 32;  // sort at least 2 kk maxima when there are enough
  if (w_full * R < kk) return false;              // block-uniform
  if (lane < R) sm.wtop[warp * R + lane] = warp < w_full ? m : 0u;
  if (tid == 0) sm.count = 0;
  __syncthreads();
  if (warp == 0) {  // one warp sorts them
    if (R == 16) {
      uint32_t v[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) v[e] = sm.wtop[lane * 4 + e];
      warp_sort_desc<4>(v, lane);
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (lane * 4 + e == kk - 1) sm.bound = v[e];
    } else {
      uint32_t v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = sm.wtop[lane * 8 + e];
      warp_sort_desc<8>(v, lane);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (lane * 8 + e == kk - 1) sm.bound = v[e];
    }
  }
  __syncthreads();
  const uint32_t L = sm.bound;  // nonzero: at least kk nonzero values were sorted
  // gather the candidates: one shared atomic per warp
  const unsigned lt = (1u << lane) - 1u;
  int w_cnt = 0;
#pragma unroll 4
  for (int j = 0; j < KPT; ++j) w_cnt += __popc(__ballot_sync(0xffffffffu, key_at(j) >= L));
  int w_base = 0;
  if (lane == 0 && w_cnt) w_base = atomicAdd(&sm.count, w_cnt);
  w_base = __shfl_sync(0xffffffffu, w_base, 0);
#pragma unroll 4
  for (int j = 0; j < KPT; ++j) {
    const uint32_t kj = key_at(j);
    const bool c = kj >= L;
    const unsigned bal = __ballot_sync(0xffffffffu, c);
    const int slot = w_base + __popc(bal & lt);
    if (c && slot < kTopkCandCap) sm.cand[slot] = rank_key(kj, base + 32 * j);
    w_base += __popc(bal);
  }
  __syncthreads();
  const int C = sm.count;
  if (C > kTopkCandCap) return false;  // block-uniform
  if (C <= 256) {  // warps 0 and 1 sort 128 candidates each; the kk-th of the two lists
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
    if (tid == 0) {  // i entries from the first list and kk - i from the second (keys are distinct)
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
  } else {  // each candidate's rank is counted against all
    for (int t = tid; t < C; t += T) {
      const unsigned long long x = sm.cand[t];
      int rank = 0;
      for (int u0 = 0; u0 < C; u0 += 8) {  // eight loads in flight per step
        unsigned long long y[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) y[k] = sm.cand[min(u0 + k, C - 1)];
#pragma unroll
        for (int k = 0; k < 8; ++k) rank += (u0 + k < C && y[k] > x) ? 1 : 0;
      }
      if (rank == kk - 1) sm.kth = x;
    }
  }
  __syncthreads();
  // selected: key > the k-th's, or equal with an index at or below its index
  const uint32_t kth_key = static_cast<uint32_t>(sm.kth >> 32);
  const int kth_idx = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(sm.kth));
  auto selected = [&](uint32_t kj, int idx) { return kj > kth_key || (kj == kth_key && idx <= kth_idx); };
  int w_sel = 0;
#pragma unroll 4
  for (int j = 0; j < KPT; ++j) w_sel += __popc(__ballot_sync(0xffffffffu, selected(key_at(j), base + 32 * j)));
  if (lane == 0) sm.wcnt[warp] = w_sel;
  __syncthreads();
  int pos = 0;
  for (int w = 0; w < warp; ++w) pos += sm.wcnt[w];
  pdl_trigger();
  int32_t *out_i = a.sel_idx + static_cast<size_t>(row) * a.k;
  float *out_s = a.sel_score ? a.sel_score + static_cast<size_t>(row) * a.k : nullptr;
#pragma unroll 4
  for (int j = 0; j < KPT; ++j) {
    const int idx = base + 32 * j;
    const uint32_t kj = key_at(j);
    const bool c = selected(kj, idx);
    const unsigned bal = __ballot_sync(0xffffffffu, c);
    if (c) {
      const int o = pos + __popc(bal & lt);
      out_i[o] = a.id_map ? a.id_map[static_cast<size_t>(row) * a.stride + idx] : idx;
      if (out_s) out_s[o] = key_to_float(kj);
    }
    pos += __popc(bal);
  }
  for (int i = kk + tid; i < a.k; i += T) {
    out_i[i] = -1;
    if (out_s) out_s[i] = neg_inf();
  }
  if (a.counters && tid == 0) a.counters[row] = 0u;
  return true;
}

template <int KPT>
__global__ void __launch_bounds__(kTopkRegThreads, KPT <= 16 ? 4 : 1) k_topk(const TopkArgs a) {
  constexpr int T = kTopkRegThreads, W = T / 32;
  __shared__ uint32_t hist[256];
  __shared__ int info[4];
  __shared__ int wtot[2][W];
  __shared__ BoundSmem bsm;

  extern __shared__ __align__(16) float srow_s[];  // [KPT * T]: the row, staged by one bulk copy
  __shared__ uint64_t load_bar;

  const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    mbar_init(&load_bar, 1);
    mbar_fence_init();
  }
  __syncthreads();
  pdl_wait();
  const int b = row / a.hq;
  int n = a.counts ? a.counts[row] : a.n_gists[b] / a.count_div;
  n = min(max(n, 0), min(a.stride, KPT * T));
  const float *srow = a.scores + static_cast<size_t>(row) * a.stride;
  const int base = warp * 32 * KPT + lane;

  // the row's first n & ~3 scores arrive in one bulk copy when the row
  // starts on a 16-byte boundary; the rest (and a timed-out copy) are read
  // from global memory directly
  const int n4 = (reinterpret_cast<uintptr_t>(srow) & 15u) == 0 ? (n & ~3) : 0;
  if (tid == 0) {
    mbar_arrive_expect_tx(&load_bar, static_cast<uint32_t>(n4) * 4u + GSA_TEST_STALL_BYTES);
    if (n4 > 0) bulk_g2s(srow_s, srow, static_cast<uint32_t>(n4) * 4u, &load_bar);
  }
  const bool landed = mbar_wait(&load_bar, 0);
  if (!landed && tid == 0) flag_error(a.status, GSA_DEVERR_TIMEOUT);
  // after a timeout the copy has had kWaitLimitNs to land; the row is read
  // from global memory either way, so a late copy rewrites the same values
  const int staged = landed ? n4 : 0;
  for (int i = staged + tid; i < n; i += T) srow_s[i] = __ldcg(srow + i);  // the tail (and a timed-out copy)
  __syncthreads();

  const int kk = min(a.k, n);
  if (kk > 0 && kk < n && kk <= T && topk_by_bound<KPT>(a, row, n, kk, srow_s, base, bsm)) return;
  uint32_t key[KPT];
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    const int i = base + 32 * j;
    key[j] = i < n ? float_to_key(srow_s[i]) : 0u;
  }

  uint32_t prefix = 0, pmask = 0;
  int rem = kk;
  bool all_eq = kk == n;
  for (int shift = 24; shift >= 0 && !all_eq && kk > 0; shift -= 8) {
    if (tid < 256) hist[tid] = 0u;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
      const bool in = (base + 32 * j < n) && ((key[j] & pmask) == prefix);
      const uint32_t bin = (key[j] >> shift) & 255u;
      if (shift == 24) {
        // first digit: few distinct bins, aggregate per warp
        const unsigned peers = __match_any_sync(0xffffffffu, in ? bin : 0x100u);
        if (in && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], static_cast<uint32_t>(__popc(peers)));
      } else if (in) {
        atomicAdd(&hist[bin], 1u);
      }
    }
    __syncthreads();
    if (warp == 0) {
      uint32_t c[8], tot = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        c[e] = hist[lane * 8 + e];
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
          info[0] = lane * 8 + e;
          info[1] = static_cast<int>(cum);
          info[2] = static_cast<int>(c[e]);
        }
        cum += c[e];
      }
    }
    __syncthreads();
    rem -= info[1];
    prefix |= static_cast<uint32_t>(info[0]) << shift;
    pmask |= 0xFFu << shift;
    all_eq = info[2] == rem;
  }

  // Compaction in index order: ballots within the warp, one small scan
  // across warps for the boundary ranks and the output offsets.
  const unsigned lt = (1u << lane) - 1u;
  int w_gt = 0, w_eq = 0;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    const bool valid = kk > 0 && base + 32 * j < n;
    const uint32_t km = key[j] & pmask;
    w_gt += __popc(__ballot_sync(0xffffffffu, valid && km > prefix));
    w_eq += __popc(__ballot_sync(0xffffffffu, valid && km == prefix));
  }
  if (lane == 0) {
    wtot[0][warp] = w_eq;
  }
  __syncthreads();
  int eq_before = 0;  // boundary keys in lower warps
  for (int w = 0; w < warp; ++w) eq_before += wtot[0][w];
  const int eq_take_w = all_eq ? w_eq : max(0, min(w_eq, rem - eq_before));
  if (lane == 0) wtot[1][warp] = w_gt + eq_take_w;
  __syncthreads();
  int out_base = 0;
  for (int w = 0; w < warp; ++w) out_base += wtot[1][w];
  pdl_trigger();

  int32_t *out_i = a.sel_idx + static_cast<size_t>(row) * a.k;
  float *out_s = a.sel_score ? a.sel_score + static_cast<size_t>(row) * a.k : nullptr;
  int pos = out_base, eq_seen = 0;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    // boundary keys of this j-row taken in lane order while eq_seen < eq_take_w
    const bool valid = kk > 0 && base + 32 * j < n;
    const uint32_t km = key[j] & pmask;
    const unsigned eqs = __ballot_sync(0xffffffffu, valid && km == prefix);
    const int my_eq_rank = eq_seen + __popc(eqs & lt);
    const bool take_eq = ((eqs >> lane) & 1u) && my_eq_rank < eq_take_w;
    const unsigned sel = __ballot_sync(0xffffffffu, (valid && km > prefix) || take_eq);
    if ((sel >> lane) & 1u) {
      const int o = pos + __popc(sel & lt);
      const int idx = base + 32 * j;
      out_i[o] = a.id_map ? a.id_map[static_cast<size_t>(row) * a.stride + idx] : idx;
      if (out_s) out_s[o] = key_to_float(key[j]);
    }
    pos += __popc(sel);
    eq_seen += __popc(eqs);
  }
  for (int i = kk + tid; i < a.k; i += T) {
    out_i[i] = -1;
    if (out_s) out_s[i] = neg_inf();
  }
  if (a.counters && tid == 0) a.counters[row] = 0u;
}

}  // namespace gsa
