// k_unfold.cuh -- selective unfolding + exact attention (split-K decoding).
//
// Method: "Selectieve Ontvouwing" on gist.science/nl/paper/2604.20920 and
// gist.science/ja section 2.1 steps 3-4: the raw tokens of the selected
// chunks are put back next to their gist tokens and exact softmax attention
// runs over the hybrid set; the own unfinished chunk is raw.  The merge of
// partial softmax results is the online-softmax combination (Milakov and
// Gimelshein, 2018), the same one gist.science/ja/paper/2607.20457 uses to
// merge per-host attention in its second phase.
//
// Grid: (splits, hq, B).  Split s of row (b, h) gathers its share of the
// selected chunks (each a contiguous chunk*D span of K and of V) with bulk
// copies into a shared-memory ring; the last split also takes the own
// chunk.  Each group of lanes that owns one row runs an online softmax; the
// CTA result is a partial (max, sum, acc).  The CTA that arrives last at
// the row's counter (an atomic, no waiting) merges all partials with the
// prior partial (all gists, or the H-GSA levels) and writes out and lse.
#pragma once

#include "common.cuh"

namespace gsa {

struct UnfoldArgs {
  const void *q;             // [B, hq, D]
  const void *raw_k, *raw_v; // [B, hkv, t_max, D]
  const void *gist_v;        // [B, hkv, n_max, D] (exclude mode)
  const int32_t *n_gists, *own_len;
  const int32_t *sel_idx;    // [B*hq, k]
  const float *sel_score;    // [B*hq, k] natural-unit scores (exclude mode)
  int32_t k, chunk, t_max, n_max, hq, hkv, group, exclude;
  float scale_log2;
  float *part;               // [B*hq, n_split, D+4]
  int32_t n_split;
  const float *prior;        // [B*hq, n_prior, D+4] or null
  int32_t n_prior;
  uint32_t *counters;        // [B*hq]
  uint32_t *status;
  void *out;                 // [B*hq, D]
  int32_t out_bf16;
  float *lse;                // [B*hq] or null
};

constexpr int kUnfoldThreads = 128;
constexpr int kUnfoldMaxItems = 1025;

// Merge (m2, l2, acc2) into (m, l, acc): base-2 online-softmax combination.
template <int E>
__device__ __forceinline__ void merge_state(float &m, float &l, float *acc, float m2, float l2, const float *acc2) {
  const float mn = fmaxf(m, m2);
  if (mn == neg_inf()) return;
  const float c1 = exp2_approx(m - mn), c2 = exp2_approx(m2 - mn);
  l = l * c1 + l2 * c2;
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = acc[e] * c1 + acc2[e] * c2;
  m = mn;
}

// Merge `n` partial records and write the normalised output row.
template <int D>
__device__ void combine_records(const float *const *recs, const int *counts, int n_lists, void *out, size_t row,
                                int out_bf16, float *lse) {
  const int tid = threadIdx.x;
  float M = neg_inf();
  for (int li = 0; li < n_lists; ++li)
    for (int i = 0; i < counts[li]; ++i) M = fmaxf(M, __ldcg(recs[li] + static_cast<size_t>(i) * (D + kPartHeader)));
  for (int dim = tid; dim < D; dim += kUnfoldThreads) {
    float L = 0.f, acc = 0.f;
    if (M != neg_inf()) {
      for (int li = 0; li < n_lists; ++li)
        for (int i = 0; i < counts[li]; ++i) {
          const float *r = recs[li] + static_cast<size_t>(i) * (D + kPartHeader);
          const float w = exp2_approx(__ldcg(r) - M);
          L += __ldcg(r + 1) * w;
          acc += __ldcg(r + kPartHeader + dim) * w;
        }
    }
    store_out(out, row * D + dim, L > 0.f ? acc / L : 0.f, out_bf16);
    if (dim == 0 && lse) lse[row] = L > 0.f ? (M + __log2f(L)) * kLn2 : neg_inf();
  }
}

template <int D, typename T>
__global__ void __launch_bounds__(kUnfoldThreads) k_unfold(const UnfoldArgs a) {
  constexpr int kE = Vec16<T>::kElems;          // elements per lane
  constexpr int kLpr = D / kE;                  // lanes per row
  constexpr int kRpw = 32 / kLpr;               // rows per warp pass
  constexpr int kSlots = (kUnfoldThreads / 32) * kRpw;
  constexpr int kRowBytes = D * static_cast<int>(sizeof(T));
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int items[kUnfoldMaxItems];
  __shared__ int item_pos[kUnfoldMaxItems];
  __shared__ int n_items_s;
  __shared__ int is_last_s;
  __shared__ float red[kUnfoldThreads / 32][2 + D];
  __shared__ uint64_t bars[8];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int kvh = h / a.group;
  const size_t row = static_cast<size_t>(b) * a.hq + h;
  const uint32_t chunk_bytes = static_cast<uint32_t>(a.chunk) * kRowBytes;
  const int stages = min(8, max(2, (96 * 1024) / static_cast<int>(2 * chunk_bytes)));

  pdl_wait();
  const int N = min(min(max(a.n_gists[b], 0), a.n_max), a.t_max / a.chunk);
  int own = min(max(a.own_len[b], 0), a.chunk);
  if (static_cast<int64_t>(N) * a.chunk + own > a.t_max) own = max(0, a.t_max - N * a.chunk);

  // Items of this split, in list order: selected chunks, then the own chunk.
  const int per = (a.k + a.n_split - 1) / a.n_split;
  const int i0 = min(a.k, split * per), i1 = min(a.k, i0 + per);
  if (warp == 0) {
    int cnt = 0;
    for (int base = i0; base < i1; base += 32) {
      const int i = base + lane;
      int m = -1;
      if (i < i1) {
        m = a.sel_idx[row * a.k + i];
        if (m >= N) {
          flag_error(a.status, GSA_DEVERR_BAD_INDEX);
          m = -1;
        }
      }
      const unsigned ball = __ballot_sync(0xffffffffu, m >= 0);
      if (m >= 0) {
        const int slot = cnt + __popc(ball & ((1u << lane) - 1u));
        items[slot] = m;
        item_pos[slot] = i;
      }
      cnt += __popc(ball);
    }
    if (lane == 0) {
      if (split == a.n_split - 1 && own > 0) {
        items[cnt] = -1;  // the own chunk
        item_pos[cnt] = -1;
        ++cnt;
      }
      n_items_s = cnt;
      for (int s = 0; s < stages; ++s) mbar_init(&bars[s], 1);
      mbar_fence_init();
    }
  }
  __syncthreads();
  const int n_items = n_items_s;

  const size_t kv_base = (static_cast<size_t>(b) * a.hkv + kvh) * a.t_max;
  const uint8_t *rk = reinterpret_cast<const uint8_t *>(a.raw_k) + kv_base * kRowBytes;
  const uint8_t *rv = reinterpret_cast<const uint8_t *>(a.raw_v) + kv_base * kRowBytes;
  auto item_rows = [&](int it) { return items[it] >= 0 ? a.chunk : own; };
  auto issue = [&](int it) {
    const int st = it % stages;
    const int m = items[it];
    const size_t first = m >= 0 ? static_cast<size_t>(m) * a.chunk : static_cast<size_t>(N) * a.chunk;
    const uint32_t bytes = static_cast<uint32_t>(item_rows(it)) * kRowBytes;
    uint8_t *dst = smem + static_cast<size_t>(st) * 2 * chunk_bytes;
    mbar_arrive_expect_tx(&bars[st], 2 * bytes);
    bulk_g2s(dst, rk + first * kRowBytes, bytes, &bars[st]);
    bulk_g2s(dst + chunk_bytes, rv + first * kRowBytes, bytes, &bars[st]);
  };
  if (tid == 0)
    for (int it = 0; it < min(stages, n_items); ++it) issue(it);

  // Query slice of this lane (dims dd .. dd+kE-1).
  const int slot = warp * kRpw + lane / kLpr;
  const int dd = kE * (lane % kLpr);
  float qf[kE];
  Vec16<T>::unpack(*reinterpret_cast<const uint4 *>(reinterpret_cast<const T *>(a.q) + row * D + dd), qf);

  float m = neg_inf(), l = 0.f, acc[kE];
#pragma unroll
  for (int e = 0; e < kE; ++e) acc[e] = 0.f;

  for (int it = 0; it < n_items; ++it) {
    const int st = it % stages;
    const bool ok = mbar_wait(&bars[st], (it / stages) & 1);
    if (__syncthreads_or(!ok)) {
      if (tid == 0) {
        flag_error(a.status, GSA_DEVERR_TIMEOUT);
        for (int u = it; u < min(it + stages, n_items); ++u) mbar_wait(&bars[u % stages], (u / stages) & 1);
      }
      __syncthreads();
      return;
    }
    const uint8_t *Ks = smem + static_cast<size_t>(st) * 2 * chunk_bytes;
    const uint8_t *Vs = Ks + chunk_bytes;
    const int rows = item_rows(it);
    for (int r0 = 0; r0 < rows; r0 += kSlots) {
      const int r = r0 + slot;
      const bool valid = r < rows;
      float kf[kE], part = 0.f;
      Vec16<T>::unpack(lds_v4(Ks + (valid ? r : 0) * kRowBytes + dd * sizeof(T)), kf);
#pragma unroll
      for (int e = 0; e < kE; ++e) part = fmaf(qf[e], kf[e], part);
#pragma unroll
      for (int o = 1; o < kLpr; o <<= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
      if (valid) {
        const float z = part * a.scale_log2;
        float vf[kE];
        Vec16<T>::unpack(lds_v4(Vs + r * kRowBytes + dd * sizeof(T)), vf);
        const float mn = fmaxf(m, z);
        const float corr = exp2_approx(m - mn), p = exp2_approx(z - mn);
        l = l * corr + p;
#pragma unroll
        for (int e = 0; e < kE; ++e) acc[e] = fmaf(p, vf[e], acc[e] * corr);
        m = mn;
      }
    }
    // Exclude mode: the selected chunk's gist token (logit = its score).
    if (a.exclude && items[it] >= 0 && slot == it % kSlots) {
      const float z = a.sel_score[row * a.k + item_pos[it]] * kLog2e;
      float vf[kE];
      const T *gv = reinterpret_cast<const T *>(a.gist_v) +
                    ((static_cast<size_t>(b) * a.hkv + kvh) * a.n_max + items[it]) * D + dd;
      Vec16<T>::unpack(*reinterpret_cast<const uint4 *>(gv), vf);
      const float mn = fmaxf(m, z);
      const float corr = exp2_approx(m - mn), p = exp2_approx(z - mn);
      l = l * corr + p;
#pragma unroll
      for (int e = 0; e < kE; ++e) acc[e] = fmaf(p, vf[e], acc[e] * corr);
      m = mn;
    }
    __syncthreads();
    if (tid == 0 && it + stages < n_items) issue(it + stages);
  }
  pdl_trigger();

  // Merge the slots of a warp that own the same dims, then the warps.
#pragma unroll
  for (int o = kLpr; o < 32; o <<= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o), l2 = __shfl_xor_sync(0xffffffffu, l, o);
    float acc2[kE];
#pragma unroll
    for (int e = 0; e < kE; ++e) acc2[e] = __shfl_xor_sync(0xffffffffu, acc[e], o);
    merge_state<kE>(m, l, acc, m2, l2, acc2);
  }
  if (lane < kLpr) {
#pragma unroll
    for (int e = 0; e < kE; ++e) red[warp][2 + dd + e] = acc[e];
    if (lane == 0) {
      red[warp][0] = m;
      red[warp][1] = l;
    }
  }
  __syncthreads();
  float *rec = a.part + (row * a.n_split + split) * (D + kPartHeader);
  {
    float M = neg_inf();
#pragma unroll
    for (int w = 0; w < kUnfoldThreads / 32; ++w) M = fmaxf(M, red[w][0]);
    for (int dim = tid; dim < D; dim += kUnfoldThreads) {
      float s = 0.f;
      if (M != neg_inf())
#pragma unroll
        for (int w = 0; w < kUnfoldThreads / 32; ++w) s += red[w][2 + dim] * exp2_approx(red[w][0] - M);
      rec[kPartHeader + dim] = s;
    }
    if (tid == 0) {
      float L = 0.f;
      if (M != neg_inf())
#pragma unroll
        for (int w = 0; w < kUnfoldThreads / 32; ++w) L += red[w][1] * exp2_approx(red[w][0] - M);
      rec[0] = M;
      rec[1] = L;
      rec[2] = 0.f;
      rec[3] = 0.f;
    }
  }
  __syncthreads();
  if (tid == 0) {
    int last = 1;
    if (a.n_split > 1) {
      __threadfence();
      const uint32_t prev = atomicAdd(&a.counters[row], 1u);
      last = prev == static_cast<uint32_t>(a.n_split - 1);
      if (last) {
        __threadfence();
        a.counters[row] = 0u;
      }
    }
    is_last_s = last;
  }
  __syncthreads();
  if (!is_last_s) return;
  const float *recs[2] = {a.part + row * a.n_split * (D + kPartHeader),
                          a.prior ? a.prior + row * a.n_prior * (D + kPartHeader) : nullptr};
  const int counts[2] = {a.n_split, a.prior ? a.n_prior : 0};
  combine_records<D>(recs, counts, 2, a.out, row, a.out_bf16, a.lse);
}

}  // namespace gsa
