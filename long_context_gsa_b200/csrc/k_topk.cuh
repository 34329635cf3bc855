// k_topk.cuh -- per-row top-k chunk selection.
//
// Method: "Selectie" on gist.science/nl/paper/2604.20920 ("Het Proces"):
// the k most relevant gists are kept; gist.science/ja section 2.1 step 3.
// Equal scores go to the lower chunk index (the pages leave ties open).
//
// One CTA per row.  Scores become order-preserving uint32 keys; an 8-bit
// radix select (at most four histogram passes over shared memory, stopping
// as soon as the boundary digit is fully taken) finds the k-th key; keys
// equal to it are taken in index order; a bitonic sort orders the k
// survivors by (key desc, index asc).
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
  return incl - v + warp_tot[warp];
}

__global__ void __launch_bounds__(kTopkThreads) k_topk(const TopkArgs a) {
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
        if (desc ? (x < y) : (x > y)) {
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

}  // namespace gsa
