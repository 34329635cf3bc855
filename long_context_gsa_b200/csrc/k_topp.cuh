// k_topp.cuh -- top-p (nucleus) chunk selection, the variant the pages set
// against top-k: gist.science/ja/paper/2604.20920 section 4 ("Top-k vs
// Top-p") and gist.science/nl/paper/2604.20920 "Stabiliteit" -- a fixed
// probability threshold instead of a fixed chunk budget.  The pages give no
// formula; the reading adopted: the chunk probabilities are the softmax of a
// row's gist scores, and the selection is the shortest prefix of the
// ranking (score desc, index asc) whose probability mass reaches top_p, at
// least one chunk and at most k (the output capacity).
//
// One CTA per (b, h) row, as k_topk: the row is staged in shared memory by
// one bulk copy; the row maximum and the softmax denominator come from block
// reductions; the top-k bound of k_topk gathers the candidates for the k
// best (in practice about 1.2 k), which are put in rank order by counting;
// a block scan of their probabilities gives the prefix length; the entries
// reaching the last chosen rank key are written in ascending chunk order.
// A row with more than kTopkCandCap candidates (heavy exact ties) takes an
// exact slower path: k rounds of a block argmax.
#pragma once

#include "k_topk.cuh"

namespace gsa {

struct ToppArgs {
  const float *scores;    // [rows, stride] natural-unit scores
  int32_t stride;
  const int32_t *n_gists; // [B]
  int32_t hq;             // b = row / hq
  int32_t k;              // output capacity (<= 256)
  float top_p;
  int32_t *sel_idx;       // [rows, k]
  float *sel_score;       // [rows, k] or null
  int32_t *sel_count;     // [rows] or null
  uint32_t *counters;     // optional: counters[row] is re-armed to 0
};

constexpr int kToppMaxK = 256;

struct ToppSmem {
  unsigned long long cand[kTopkCandCap];
  unsigned long long sorted[kToppMaxK];  // the k best rank keys, in rank order
  uint32_t wtop[kTopkRegThreads];
  float wred[kTopkRegThreads / 32];
  int wcnt[kTopkRegThreads / 32];
  unsigned long long pick[kTopkRegThreads / 32];
  uint32_t bound;
  int count;
  float row_max, row_z;
};

// Block-wide reductions over 256 threads (fixed order: the result does not
// depend on timing).
__device__ __forceinline__ float topp_block_max(float v, float *wred) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((threadIdx.x & 31) == 0) wred[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = wred[0];
#pragma unroll
  for (int w = 1; w < kTopkRegThreads / 32; ++w) r = fmaxf(r, wred[w]);
  __syncthreads();
  return r;
}

__device__ __forceinline__ float topp_block_sum(float v, float *wred) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) wred[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = 0.f;
#pragma unroll
  for (int w = 0; w < kTopkRegThreads / 32; ++w) r += wred[w];
  __syncthreads();
  return r;
}

template <int KPT>
__global__ void __launch_bounds__(kTopkRegThreads, KPT <= 16 ? 4 : 1) k_topp(const ToppArgs a) {
  constexpr int T = kTopkRegThreads, W = T / 32;
  extern __shared__ __align__(16) float srow_s[];  // [KPT * T] the row, then [KPT * T / 32] taken bits
  __shared__ ToppSmem sm;
  __shared__ uint64_t load_bar;

  const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    mbar_init(&load_bar, 1);
    mbar_fence_init();
  }
  __syncthreads();
  pdl_wait();
  const int b = row / a.hq;
  const int n = min(max(a.n_gists[b], 0), min(a.stride, KPT * T));
  const float *srow = a.scores + static_cast<size_t>(row) * a.stride;
  const int n4 = (reinterpret_cast<uintptr_t>(srow) & 15u) == 0 ? (n & ~3) : 0;
  if (tid == 0) {
    mbar_arrive_expect_tx(&load_bar, static_cast<uint32_t>(n4) * 4u);
    if (n4 > 0) bulk_g2s(srow_s, srow, static_cast<uint32_t>(n4) * 4u, &load_bar);
  }
  const int staged = mbar_wait(&load_bar, 0) ? n4 : 0;
  for (int i = staged + tid; i < n; i += T) srow_s[i] = __ldcg(srow + i);
  __syncthreads();

  const int kmax = min(a.k, n);
  int32_t *out_i = a.sel_idx + static_cast<size_t>(row) * a.k;
  float *out_s = a.sel_score ? a.sel_score + static_cast<size_t>(row) * a.k : nullptr;
  const int base = warp * 32 * KPT + lane;  // this thread's entries: base + 32 j
  const unsigned lt = (1u << lane) - 1u;
  auto key_at = [&](int j) -> uint32_t {
    const int i = base + 32 * j;
    return i < n ? float_to_key(srow_s[i]) : 0u;  // valid keys are nonzero
  };

  int n_sel = 0;
  if (kmax > 0) {
    // softmax denominator over the whole row
    float mx = neg_inf();
#pragma unroll 4
    for (int j = 0; j < KPT; ++j)
      if (base + 32 * j < n) mx = fmaxf(mx, srow_s[base + 32 * j]);
    const float M = topp_block_max(mx, sm.wred);
    float z = 0.f;
#pragma unroll 4
    for (int j = 0; j < KPT; ++j)
      if (base + 32 * j < n) z += exp2_approx((srow_s[base + 32 * j] - M) * kLog2e);
    const float Z = topp_block_sum(z, sm.wred);

    // a lower bound on the kmax-th key (k_topk's), else every entry
    uint32_t m = 0u;
#pragma unroll 4
    for (int j = 0; j < KPT; ++j) m = max(m, key_at(j));
    {
      uint32_t v[1] = {m};
      warp_sort_desc<1>(v, lane);
      m = v[0];
    }
    const int w_full = n >= 32 ? min(W, (n - 32) / (32 * KPT) + 1) : 0;
    const int R = w_full * 16 >= 2 * kmax ? 16 : 32;
    const bool bounded = kmax < n && w_full * R >= kmax;  // block-uniform
    if (lane < R) sm.wtop[warp * R + lane] = warp < w_full ? m : 0u;
    if (tid == 0) {
      sm.count = 0;
      sm.bound = 0u;
    }
    __syncthreads();
    if (bounded && warp == 0) {
      if (R == 16) {
        uint32_t v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] = sm.wtop[lane * 4 + e];
        warp_sort_desc<4>(v, lane);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (lane * 4 + e == kmax - 1) sm.bound = v[e];
      } else {
        uint32_t v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = sm.wtop[lane * 8 + e];
        warp_sort_desc<8>(v, lane);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if (lane * 8 + e == kmax - 1) sm.bound = v[e];
      }
    }
    __syncthreads();
    const uint32_t L = max(sm.bound, 1u);  // 1: every valid entry
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
    const int nk = min(kmax, C);  // entries in rank order (C >= kmax)
    if (C <= kTopkCandCap) {
      // rank order by counting (rank keys are distinct)
      for (int t = tid; t < C; t += T) {
        const unsigned long long x = sm.cand[t];
        int rank = 0;
        for (int u0 = 0; u0 < C; u0 += 8) {
          unsigned long long y[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) y[k] = sm.cand[min(u0 + k, C - 1)];
#pragma unroll
          for (int k = 0; k < 8; ++k) rank += (u0 + k < C && y[k] > x) ? 1 : 0;
        }
        if (rank < kmax) sm.sorted[rank] = x;
      }
    } else {
      // heavy exact ties: kmax rounds of a block argmax over the row
      uint32_t *taken = reinterpret_cast<uint32_t *>(srow_s + KPT * T);
      for (int i = tid; i < KPT * W; i += T) taken[i] = 0u;
      __syncthreads();
      for (int it = 0; it < kmax; ++it) {
        unsigned long long best = 0ull;
#pragma unroll 4
        for (int j = 0; j < KPT; ++j) {
          const int i = base + 32 * j;
          if (i < n && !((taken[i >> 5] >> (i & 31)) & 1u)) best = max(best, rank_key(key_at(j), i));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) best = max(best, __shfl_xor_sync(0xffffffffu, best, o));
        if (lane == 0) sm.pick[warp] = best;
        __syncthreads();
        if (tid == 0) {
          unsigned long long r = sm.pick[0];
          for (int w = 1; w < W; ++w) r = max(r, sm.pick[w]);
          sm.sorted[it] = r;
          const int i = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(r));
          taken[i >> 5] |= 1u << (i & 31);
        }
        __syncthreads();
      }
    }
    __syncthreads();
    // probabilities in rank order; an entry is chosen while the mass before
    // it is still below top_p (the chosen ones form a prefix)
    float p = 0.f;
    if (tid < nk) p = exp2_approx((key_to_float(static_cast<uint32_t>(sm.sorted[tid] >> 32)) - M) * kLog2e) / Z;
    float incl = p;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) sm.wred[warp] = incl;
    __syncthreads();
    float before = incl - p;
    for (int w = 0; w < warp; ++w) before += sm.wred[w];
    const bool chosen = tid < nk && (tid == 0 || before < a.top_p);
    const int w_chosen = __popc(__ballot_sync(0xffffffffu, chosen));
    if (lane == 0) sm.wcnt[warp] = w_chosen;
    __syncthreads();
    for (int w = 0; w < W; ++w) n_sel += sm.wcnt[w];
  }
  if (a.sel_count && tid == 0) a.sel_count[row] = n_sel;
  if (n_sel > 0) {
    // the entries reaching the last chosen rank key, in ascending chunk order
    const unsigned long long kth = sm.sorted[n_sel - 1];
    __syncthreads();  // every thread has read sorted[] before wcnt is reused
    int w_sel = 0;
#pragma unroll 4
    for (int j = 0; j < KPT; ++j) {
      const uint32_t kj = key_at(j);
      w_sel += __popc(__ballot_sync(0xffffffffu, kj != 0u && rank_key(kj, base + 32 * j) >= kth));
    }
    if (lane == 0) sm.wcnt[warp] = w_sel;
    __syncthreads();
    int pos = 0;
    for (int w = 0; w < warp; ++w) pos += sm.wcnt[w];
    pdl_trigger();
#pragma unroll 4
    for (int j = 0; j < KPT; ++j) {
      const int idx = base + 32 * j;
      const uint32_t kj = key_at(j);
      const bool c = kj != 0u && rank_key(kj, idx) >= kth;
      const unsigned bal = __ballot_sync(0xffffffffu, c);
      if (c) {
        const int o = pos + __popc(bal & lt);
        out_i[o] = idx;
        if (out_s) out_s[o] = key_to_float(kj);
      }
      pos += __popc(bal);
    }
  } else {
    pdl_trigger();
  }
  for (int i = n_sel + tid; i < a.k; i += T) {
    out_i[i] = -1;
    if (out_s) out_s[i] = neg_inf();
  }
  if (a.counters && tid == 0) a.counters[row] = 0u;
}

}  // namespace gsa
