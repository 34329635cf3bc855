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
#include "k_score.cuh"  // mma.sync, ldmatrix and swizzle helpers
#include "tc100.cuh"

namespace gsa {

struct UnfoldArgs {
  CUtensorMap tm_k, tm_v;    // bf16 tensor-core path: raw K/V as [B*hkv*t_max, D], boxes of 64 columns x 8 rows
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
  ReadyList ready;           // w null: CTA (split, h, b) after the previous kernel; else rows as published
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

// The CTA's partial (the warps' states in red) goes to the row's split slot;
// the CTA that arrives last at the row's counter merges all splits with the
// prior partials and writes the output row.  Called by the whole block.
template <int NW, int D>
__device__ void unfold_finish(const UnfoldArgs &a, size_t row, int split, const float (*red)[2 + D], int &is_last_s) {
  const int tid = threadIdx.x;
  constexpr int kUnfoldWarps = NW;
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
  unfold_finish<kUnfoldWarps, D>(a, row, split, red, is_last_s);
}

// ---------------------------------------------------------------------------
// bf16 inputs, D in {64, 128}: the same split and combine, with the rows on
// the tensor cores.  The attended raw rows are cut into half-steps of 8 rows
// (one TMA box of 8 rows x 64 columns per 64 dims, 128-byte swizzle; a chunk
// of c rows gives ceil(c/8) half-steps, the own chunk ceil(own/8)); warp w
// takes steps w, w+4, ... of two half-steps (16 rows) through its own ring.
// Per step: s = q.K^T with mma.sync (the query is row 0 of the A operand), a
// lazy online softmax on lanes 0..3 (the lanes holding row 0), and P.V as
// mma.sync with P split into bf16 high and low parts and V read by
// ldmatrix.trans.  Rows past a half-step's valid count get weight 0 and
// their values are cleared in shared memory first.
template <int D>
struct UnfoldTcCfg {
  static constexpr int kBoxes = D / 64;
  static constexpr uint32_t kHalf = kBoxes * 1024;        // K (or V) of one 8-row half-step
  static constexpr uint32_t kStage = 4 * kHalf;           // K and V of two half-steps
  static constexpr int kStages = D == 64 ? 3 : 2;
  static constexpr uint32_t kRingBytes = kUnfoldWarps * kStages * kStage;
  // ring (1024-aligned) | selected chunks and their list positions [2][per] |
  // half-steps (first raw row, valid rows << 16 | item + 1) [(per + 1) * ceil(chunk / 8) + 1]
  // (the own chunk adds up to ceil(chunk / 8), the last step's pad one)
  static size_t smem_bytes(int per, int chunk) {
    const size_t hpc = static_cast<size_t>((chunk + 7) / 8);
    return kRingBytes + 1024 + 2 * static_cast<size_t>(per) * 4 + ((static_cast<size_t>(per) + 1) * hpc + 1) * 8;
  }
};

// With a ready list (the fused decode step), CTA t takes ticket t in
// arrival order: row = the (t / n_split)-th row published, split = t mod
// n_split.  It waits (bounded) for that row's publication instead of the
// whole scoring grid, so rows whose selection is done unfold while others
// are still being selected.  The last CTA to finish clears the list.
__device__ __forceinline__ int unfold_take_row(const UnfoldArgs &a, int &split) {
  const uint32_t t = atomicAdd(&a.ready.w[a.ready.rows + 1], 1u);
  const uint32_t pos = t / static_cast<uint32_t>(a.n_split);
  split = static_cast<int>(t % static_cast<uint32_t>(a.n_split));
  if (pos >= static_cast<uint32_t>(a.ready.rows)) {
    flag_error(a.status, GSA_DEVERR_CAPACITY);
    return -1;
  }
  uint64_t t0 = 0;
  for (uint32_t it = 0;; ++it) {
    const uint32_t v = ld_acquire_u32(&a.ready.w[pos]);
    if (v != 0u) return v <= static_cast<uint32_t>(a.ready.rows) ? static_cast<int>(v) - 1 : -1;
    if ((it & 15u) == 0) {
      const uint64_t now = global_timer_ns();
      if (!t0) t0 = now;
      else if (now - t0 > kWaitLimitNs) {
        flag_error(a.status, GSA_DEVERR_TIMEOUT);
        return -1;
      }
    }
    __nanosleep(64);
  }
}

__device__ __forceinline__ void unfold_ready_done(const UnfoldArgs &a) {
  __shared__ int last_s;
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t total = gridDim.x * gridDim.y * gridDim.z;
    last_s = atomicAdd(&a.ready.w[a.ready.rows + 2], 1u) == total - 1;
  }
  __syncthreads();
  if (last_s) {  // every CTA has read its entry: clear the list for the next step
    for (int i = threadIdx.x; i < a.ready.rows + 4; i += blockDim.x) a.ready.w[i] = 0u;
    __threadfence();
  }
}

template <int D>
__global__ void __launch_bounds__(kUnfoldThreads) k_unfold_tc(const __grid_constant__ UnfoldArgs a) {
  using Cfg = UnfoldTcCfg<D>;
  constexpr int kNT = D / 8, S = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int per = (a.k + a.n_split - 1) / a.n_split;  // list entries of one split
  int *items = reinterpret_cast<int *>(smem + Cfg::kRingBytes);
  int *item_pos = items + per;
  __shared__ int n_items_s;
  __shared__ int is_last_s;
  __shared__ int take_s[2];
  __shared__ float red[kUnfoldWarps][2 + D];
  __shared__ uint64_t bars[kUnfoldWarps][4];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int split, h, b;
  if (a.ready.w) {
    if (tid == 0) {
      int sp = 0;
      take_s[0] = unfold_take_row(a, sp);
      take_s[1] = sp;
    }
    __syncthreads();
    if (take_s[0] < 0) {  // flagged: nothing to attend
      unfold_ready_done(a);
      return;
    }
    split = take_s[1];
    h = take_s[0] % a.hq;
    b = take_s[0] / a.hq;
  } else {
    pdl_wait();
    split = blockIdx.x;
    h = blockIdx.y;
    b = blockIdx.z;
  }
  const int kvh = h / a.group;
  const size_t row = static_cast<size_t>(b) * a.hq + h;
  const int g = lane >> 2, t4 = lane & 3;

  const int N = min(min(max(__ldcg(a.n_gists + b), 0), a.n_max), a.t_max / a.chunk);
  int own = min(max(__ldcg(a.own_len + b), 0), a.chunk);
  if (static_cast<int64_t>(N) * a.chunk + own > a.t_max) own = max(0, a.t_max - N * a.chunk);

  // Selected chunks of this split, in list order (invalid entries dropped).
  const int i0 = min(a.k, split * per), i1 = min(a.k, i0 + per);
  if (warp == 0) {
    int cnt = 0;
    for (int base = i0; base < i1; base += 32) {
      const int i = base + lane;
      int m = -1;
      if (i < i1) {
        m = __ldcg(a.sel_idx + row * a.k + i);
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
      for (int s = 0; s < S; ++s) mbar_init(&bars[lane][s], 1);
    if (lane == 0) {
      mbar_fence_init();
      tc::prefetch_map(&a.tm_k);
      tc::prefetch_map(&a.tm_v);
    }
  }
  __syncthreads();

  // half-step j -> (first raw row, valid rows, chunk item or -1 for own
  // rows), tabulated once so the per-step issue and compute only look up
  const int hpc = (a.chunk + 7) >> 3;  // half-steps per chunk
  const int n_sel = n_items_s;
  const int own_half = (split == a.n_split - 1 && own > 0) ? (own + 7) >> 3 : 0;
  const int n_half = n_sel * hpc + own_half;
  const int n_steps = (n_half + 1) >> 1;
  const int n_mine = n_steps > warp ? (n_steps - warp + kUnfoldWarps - 1) / kUnfoldWarps : 0;
  int2 *htab = reinterpret_cast<int2 *>(item_pos + per);
  for (int j = tid; j < 2 * n_steps; j += kUnfoldThreads) {
    int first = 0, valid = 0, item = -1;
    if (j < n_sel * hpc) {
      const int it = j / hpc, sub = j - it * hpc;
      first = items[it] * a.chunk + 8 * sub;
      valid = min(8, a.chunk - 8 * sub);
      item = sub == 0 ? it : -1;  // the chunk's gist joins with its first half-step
    } else if (j < n_half) {
      const int q = j - n_sel * hpc;
      first = N * a.chunk + 8 * q;
      valid = min(8, own - 8 * q);
    }
    htab[j] = make_int2(first, (valid << 16) | (item + 1));
  }
  __syncthreads();
  auto half = [&](int j, int &first, int &valid, int &item) {
    const int2 e = htab[j];
    first = e.x;
    valid = e.y >> 16;
    item = (e.y & 0xffff) - 1;
  };
  const int kv_row0 = (b * a.hkv + kvh) * a.t_max;  // tensor-map row of this kv head's first raw row
  uint8_t *ring = smem + static_cast<size_t>(warp) * S * Cfg::kStage;
  auto issue = [&](int li) {
    const int step = warp + kUnfoldWarps * li, st = li % S;
    uint8_t *dst = ring + st * Cfg::kStage;
    mbar_arrive_expect_tx(&bars[warp][st], Cfg::kStage + GSA_TEST_STALL_BYTES);
#pragma unroll
    for (int hs = 0; hs < 2; ++hs) {
      int first, valid, item;
      half(2 * step + hs, first, valid, item);
#pragma unroll
      for (int x = 0; x < Cfg::kBoxes; ++x) {
        tc::tma_load_2d(dst + (hs * Cfg::kBoxes + x) * 1024, &a.tm_k, 64 * x, kv_row0 + first, &bars[warp][st]);
        tc::tma_load_2d(dst + 2 * Cfg::kHalf + (hs * Cfg::kBoxes + x) * 1024, &a.tm_v, 64 * x, kv_row0 + first,
                        &bars[warp][st]);
      }
    }
  };
  if (lane == 0)
    for (int li = 0; li < min(S, n_mine); ++li) issue(li);

  // the query as row 0 of the A operand (k permuted as in the scoring pass)
  uint2 afr[D / 16];
  {
    const uint4 *qrow = reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(a.q) + row * D);
#pragma unroll
    for (int s2 = 0; s2 < D / 32; ++s2) {
      const uint4 w = g == 0 ? qrow[4 * s2 + t4] : make_uint4(0, 0, 0, 0);
      afr[2 * s2] = make_uint2(w.x, w.y);
      afr[2 * s2 + 1] = make_uint2(w.z, w.w);
    }
  }
  float acc[kNT][4];  // row 0 (lanes 0..3): dims 8*nt + 2*t4 (+1); other rows unused
#pragma unroll
  for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
  float mg = neg_inf(), lg = 0.f;  // reference max (base 2, same in every lane) and this lane's sum
  const uint32_t ring_u = smem_u32(ring);
  const __nv_bfloat16 *gv_base =
      reinterpret_cast<const __nv_bfloat16 *>(a.gist_v) + (static_cast<size_t>(b) * a.hkv + kvh) * a.n_max * D;
  int stuck = -1;
  for (int li = 0; li < n_mine; ++li) {
    const int st = li % S, step = warp + kUnfoldWarps * li;
    if (!__all_sync(0xffffffffu, mbar_wait(&bars[warp][st], (li / S) & 1))) {
      stuck = li;
      break;
    }
    const uint32_t kst = ring_u + st * Cfg::kStage, vst = kst + 2 * Cfg::kHalf;
    int valid[2], item[2], first;
    half(2 * step, first, valid[0], item[0]);
    half(2 * step + 1, first, valid[1], item[1]);
    if (valid[0] < 8 || valid[1] < 8) {
      // clear the values of rows past the valid ones (they get weight 0)
#pragma unroll
      for (int hs = 0; hs < 2; ++hs)
        for (int i = lane; i < (8 - valid[hs]) * Cfg::kBoxes * 8; i += 32) {
          const int r = valid[hs] + i / (8 * Cfg::kBoxes), x = (i / 8) % Cfg::kBoxes, ch = i % 8;
          asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(vst + (hs * Cfg::kBoxes + x) * 1024 +
                                                                        sw128(r, ch)),
                       "r"(0u)
                       : "memory");
        }
      tc::fence_proxy_async_smem();
      __syncwarp();
    }
    float s[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int s2 = 0; s2 < D / 32; ++s2) {
        uint4 kb;
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(kb.x), "=r"(kb.y), "=r"(kb.z), "=r"(kb.w)
                     : "r"(kst + (nt * Cfg::kBoxes + (s2 >> 1)) * 1024 + sw128(g, (s2 & 1) * 4 + t4)));
        mma_16816_bf16(c, afr[2 * s2].x, 0u, afr[2 * s2].y, 0u, kb.x, kb.y);
        mma_16816_bf16(c, afr[2 * s2 + 1].x, 0u, afr[2 * s2 + 1].y, 0u, kb.z, kb.w);
      }
#pragma unroll
      for (int e = 0; e < 2; ++e) s[nt][e] = (g == 0 && 2 * t4 + e < valid[nt]) ? c[e] * a.scale_log2 : neg_inf();
    }
    // exclude mode: a selected chunk's gist token joins with its first half-step
    float z[2] = {neg_inf(), neg_inf()};
    if (a.exclude)
#pragma unroll
      for (int hs = 0; hs < 2; ++hs)
        if (item[hs] >= 0) z[hs] = __ldcg(a.sel_score + row * a.k + item_pos[item[hs]]) * kLog2e;
    float qm = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
    qm = fmaxf(qm, __shfl_xor_sync(0xffffffffu, qm, 1));
    qm = fmaxf(qm, __shfl_xor_sync(0xffffffffu, qm, 2));
    qm = fmaxf(__shfl_sync(0xffffffffu, qm, 0), fmaxf(z[0], z[1]));
    if (qm > mg + kRescaleSlack) {  // warp-uniform: raise the reference, rescale
      const float alpha = mg == neg_inf() ? 1.f : exp2_approx(mg - qm);
      lg *= alpha;
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt) {
        acc[nt][0] *= alpha;
        acc[nt][1] *= alpha;
      }
      mg = qm;
    }
    float p[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) p[nt][e] = s[nt][e] > neg_inf() ? exp2_approx(s[nt][e] - mg) : 0.f;
    lg += (p[0][0] + p[0][1]) + (p[1][0] + p[1][1]);
    const uint32_t h0p = pack_bf16(p[0][0], p[0][1]), h1p = pack_bf16(p[1][0], p[1][1]);
    const uint32_t l0p = pack_bf16(p[0][0] - bf16_lo(h0p), p[0][1] - bf16_hi(h0p));
    const uint32_t l1p = pack_bf16(p[1][0] - bf16_lo(h1p), p[1][1] - bf16_hi(h1p));
    const int mi = lane >> 3;
#pragma unroll
    for (int dp = 0; dp < kNT / 2; ++dp) {
      const int dim0 = 8 * (2 * dp + (mi >> 1));
      uint32_t b0, b1, b2, b3;
      ldsm_x4_trans(vst + ((mi & 1) * Cfg::kBoxes + (dim0 >> 6)) * 1024 + sw128(lane & 7, (dim0 & 63) >> 3), b0, b1,
                    b2, b3);
      mma_16816_bf16(acc[2 * dp], h0p, 0u, h1p, 0u, b0, b1);
      mma_16816_bf16(acc[2 * dp], l0p, 0u, l1p, 0u, b0, b1);
      mma_16816_bf16(acc[2 * dp + 1], h0p, 0u, h1p, 0u, b2, b3);
      mma_16816_bf16(acc[2 * dp + 1], l0p, 0u, l1p, 0u, b2, b3);
    }
    if (a.exclude)
#pragma unroll
      for (int hs = 0; hs < 2; ++hs)
        if (item[hs] >= 0 && g == 0) {
          const float pz = exp2_approx(z[hs] - mg);
          if (t4 == 0) lg += pz;
          const __nv_bfloat16 *gv = gv_base + static_cast<size_t>(items[item[hs]]) * D + 2 * t4;
#pragma unroll
          for (int nt = 0; nt < kNT; ++nt) {
            const uint32_t w = *reinterpret_cast<const uint32_t *>(gv + 8 * nt);
            acc[nt][0] = fmaf(pz, bf16_lo(w), acc[nt][0]);
            acc[nt][1] = fmaf(pz, bf16_hi(w), acc[nt][1]);
          }
        }
    __syncwarp();
    if (lane == 0 && li + S < n_mine) issue(li + S);
  }
  if (stuck >= 0 && lane == 0) {
    // Let the copies already issued land before the CTA can exit.
    flag_error(a.status, GSA_DEVERR_TIMEOUT);
    for (int li = stuck; li < min(stuck + S, n_mine); ++li) mbar_wait(&bars[warp][li % S], (li / S) & 1);
  }
  pdl_trigger();
  lg += __shfl_xor_sync(0xffffffffu, lg, 1);
  lg += __shfl_xor_sync(0xffffffffu, lg, 2);
  if (lane < 4) {
#pragma unroll
    for (int nt = 0; nt < kNT; ++nt) {
      red[warp][2 + 8 * nt + 2 * t4] = acc[nt][0];
      red[warp][2 + 8 * nt + 2 * t4 + 1] = acc[nt][1];
    }
    if (lane == 0) {
      red[warp][0] = mg;
      red[warp][1] = lg;
    }
  }
  unfold_finish<kUnfoldWarps, D>(a, row, split, red, is_last_s);
  if (a.ready.w) unfold_ready_done(a);
}

}  // namespace gsa
