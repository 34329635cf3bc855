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
// selected chunks (each a contiguous chunk*D span of K and of V, cut into
// pieces of at most 4 KB) with bulk copies; the last split also takes the
// own chunk.  Each of the 4 warps streams its own pieces through a private
// mbarrier ring, so the main loop has no CTA-wide barrier.  Each group of
// lanes that owns one row runs an online softmax; the CTA result is a
// partial (max, sum, acc).  The CTA that arrives last at
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
constexpr int kUnfoldMaxItems = 1024;

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

// Rows of one bulk-copy piece: at most 4 KB of K (and of V) per piece, so
// long chunks pipeline in several pieces.
template <int D, typename T>
__host__ __device__ __forceinline__ int unfold_piece_rows(int chunk) {
  const int cap = 4096 / (D * static_cast<int>(sizeof(T)));
  return chunk < cap ? chunk : (cap < 1 ? 1 : cap);
}

// Stages of each warp's ring (a stage holds one piece of K and of V).
__host__ __device__ __forceinline__ int unfold_warp_stages(int stage_bytes) {
  const int s = 8192 / stage_bytes;
  return s < 2 ? 2 : (s > 8 ? 8 : s);
}

constexpr int kUnfoldWarps = kUnfoldThreads / 32;

template <int D, typename T>
__global__ void __launch_bounds__(kUnfoldThreads) k_unfold(const UnfoldArgs a) {
  constexpr int kE = Vec16<T>::kElems;          // elements per lane
  constexpr int kLpr = D / kE;                  // lanes per row
  constexpr int kRpw = 32 / kLpr;               // rows per warp pass
  constexpr int kRowBytes = D * static_cast<int>(sizeof(T));
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int items[kUnfoldMaxItems];
  __shared__ int item_pos[kUnfoldMaxItems];
  __shared__ int n_items_s;
  __shared__ int is_last_s;
  __shared__ float red[kUnfoldWarps][2 + D];
  __shared__ uint64_t bars[kUnfoldWarps][8];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int kvh = h / a.group;
  const size_t row = static_cast<size_t>(b) * a.hq + h;
  const int pr = unfold_piece_rows<D, T>(a.chunk);
  const uint32_t piece_bytes = static_cast<uint32_t>(pr) * kRowBytes;
  const int sw = unfold_warp_stages(static_cast<int>(2 * piece_bytes));

  pdl_wait();
  const int N = min(min(max(a.n_gists[b], 0), a.n_max), a.t_max / a.chunk);
  int own = min(max(a.own_len[b], 0), a.chunk);
  if (static_cast<int64_t>(N) * a.chunk + own > a.t_max) own = max(0, a.t_max - N * a.chunk);

  // Selected chunks of this split, in list order (invalid entries dropped).
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
    if (lane == 0) n_items_s = cnt;
    if (lane < kUnfoldWarps)
      for (int s = 0; s < sw; ++s) mbar_init(&bars[lane][s], 1);
    if (lane == 0) mbar_fence_init();
  }
  __syncthreads();

  // Pieces: each selected chunk gives ppc pieces; the own chunk (last split)
  // gives ceil(own / pr) pieces.  Warp w takes pieces w, w + 4, ...
  const int ppc = (a.chunk + pr - 1) / pr;
  const int n_sel = n_items_s;
  const int own_pieces = (split == a.n_split - 1 && own > 0) ? (own + pr - 1) / pr : 0;
  const int n_pieces = n_sel * ppc + own_pieces;
  const int n_mine = n_pieces > warp ? (n_pieces - warp + kUnfoldWarps - 1) / kUnfoldWarps : 0;

  const size_t kv_base = (static_cast<size_t>(b) * a.hkv + kvh) * a.t_max;
  const uint8_t *rk = reinterpret_cast<const uint8_t *>(a.raw_k) + kv_base * kRowBytes;
  const uint8_t *rv = reinterpret_cast<const uint8_t *>(a.raw_v) + kv_base * kRowBytes;
  uint8_t *ring = smem + static_cast<size_t>(warp) * sw * 2 * piece_bytes;
  // piece p -> first raw row and row count
  auto piece = [&](int p, int &first, int &rows) {
    if (p < n_sel * ppc) {
      const int it = p / ppc, sub = p % ppc;
      first = items[it] * a.chunk + sub * pr;
      rows = min(pr, a.chunk - sub * pr);
    } else {
      const int q = p - n_sel * ppc;
      first = N * a.chunk + q * pr;
      rows = min(pr, own - q * pr);
    }
  };
  auto issue = [&](int li) {
    int first, rows;
    piece(warp + kUnfoldWarps * li, first, rows);
    const int st = li % sw;
    const uint32_t bytes = static_cast<uint32_t>(rows) * kRowBytes;
    uint8_t *dst = ring + static_cast<size_t>(st) * 2 * piece_bytes;
    mbar_arrive_expect_tx(&bars[warp][st], 2 * bytes);
    bulk_g2s(dst, rk + static_cast<size_t>(first) * kRowBytes, bytes, &bars[warp][st]);
    bulk_g2s(dst + piece_bytes, rv + static_cast<size_t>(first) * kRowBytes, bytes, &bars[warp][st]);
  };
  if (lane == 0)
    for (int li = 0; li < min(sw, n_mine); ++li) issue(li);

  const int slot = lane / kLpr;
  const int dd = kE * (lane % kLpr);
  float qf[kE];
  Vec16<T>::unpack(*reinterpret_cast<const uint4 *>(reinterpret_cast<const T *>(a.q) + row * D + dd), qf);

  // Online softmax state of this lane's slot; the reference max m is only
  // raised when a logit exceeds it by more than 2^8 (rare after warm-up).
  float m = neg_inf(), l = 0.f, acc[kE];
#pragma unroll
  for (int e = 0; e < kE; ++e) acc[e] = 0.f;
  auto update = [&](float z, const float *vf) {
    if (z > m + 8.0f) {
      const float c = exp2_approx(m - z);
      l *= c;
#pragma unroll
      for (int e = 0; e < kE; ++e) acc[e] *= c;
      m = z;
    }
    const float p = exp2_approx(z - m);
    l += p;
#pragma unroll
    for (int e = 0; e < kE; ++e) acc[e] = fmaf(p, vf[e], acc[e]);
  };

  int stuck = -1;  // first piece whose wait expired
  for (int li = 0; li < n_mine; ++li) {
    const int st = li % sw;
    if (!__all_sync(0xffffffffu, mbar_wait(&bars[warp][st], (li / sw) & 1))) {
      stuck = li;
      break;
    }
    const int p = warp + kUnfoldWarps * li;
    int first, rows;
    piece(p, first, rows);
    const uint8_t *Ks = ring + static_cast<size_t>(st) * 2 * piece_bytes;
    const uint8_t *Vs = Ks + piece_bytes;
    for (int r0 = 0; r0 < rows; r0 += kRpw) {
      const int r = r0 + slot;
      const bool valid = r < rows;
      float kf[kE], part = 0.f;
      Vec16<T>::unpack(lds_v4(Ks + (valid ? r : 0) * kRowBytes + dd * static_cast<int>(sizeof(T))), kf);
#pragma unroll
      for (int e = 0; e < kE; ++e) part = fmaf(qf[e], kf[e], part);
#pragma unroll
      for (int o = 1; o < kLpr; o <<= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
      if (valid) {
        float vf[kE];
        Vec16<T>::unpack(lds_v4(Vs + r * kRowBytes + dd * static_cast<int>(sizeof(T))), vf);
        update(part * a.scale_log2, vf);
      }
    }
    // Exclude mode: the selected chunk's gist token joins with its first piece.
    if (a.exclude && p < n_sel * ppc && p % ppc == 0 && slot == 0) {
      const int it = p / ppc;
      float vf[kE];
      const T *gv = reinterpret_cast<const T *>(a.gist_v) +
                    ((static_cast<size_t>(b) * a.hkv + kvh) * a.n_max + items[it]) * D + dd;
      Vec16<T>::unpack(*reinterpret_cast<const uint4 *>(gv), vf);
      update(a.sel_score[row * a.k + item_pos[it]] * kLog2e, vf);
    }
    __syncwarp();
    if (lane == 0 && li + sw < n_mine) issue(li + sw);
  }
  if (stuck >= 0 && lane == 0) {
    // Let the copies already issued land before the CTA can exit.
    flag_error(a.status, GSA_DEVERR_TIMEOUT);
    for (int li = stuck; li < min(stuck + sw, n_mine); ++li) mbar_wait(&bars[warp][li % sw], (li / sw) & 1);
  }
  pdl_trigger();

  // Merge the slots of the warp that own the same dims, then the warps.
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
    for (int w = 0; w < kUnfoldWarps; ++w) M = fmaxf(M, red[w][0]);
    for (int dim = tid; dim < D; dim += kUnfoldThreads) {
      float s = 0.f;
      if (M != neg_inf())
#pragma unroll
        for (int w = 0; w < kUnfoldWarps; ++w) s += red[w][2 + dim] * exp2_approx(red[w][0] - M);
      rec[kPartHeader + dim] = s;
    }
    if (tid == 0) {
      float L = 0.f;
      if (M != neg_inf())
#pragma unroll
        for (int w = 0; w < kUnfoldWarps; ++w) L += red[w][1] * exp2_approx(red[w][0] - M);
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
