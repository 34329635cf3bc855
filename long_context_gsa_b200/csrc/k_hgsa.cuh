// k_hgsa.cuh -- H-GSA second level: score the children of the chosen
// meta-gist groups, and the softmax partial over the coarse levels.
//
// Method: gist.science/ja/paper/2604.20920 section 2.2 and
// gist.science/nl/paper/2604.20920 "Hierarchische Uitbreiding (H-GSA)":
// meta-gists summarise groups of gists; selection runs coarse to fine --
// the top meta groups first, then the top gists among their children, then
// the chosen chunks are unfolded.  Readings adopted where the pages are
// silent: gists of an incomplete trailing group (no meta-gist yet) are
// always candidates; the attended set keeps, besides the unfolded chunks,
// every unselected meta-gist and every unselected candidate gist (unless
// unselected entries are excluded), which keeps the set multi-resolution.
//
// Grid (splits, hq, B).  Candidates are the g rows of each chosen group, in
// ascending gist order (the meta selection is ascending), then the trailing
// gists.  Split s takes candidate pieces s, s+S, ... through per-warp bulk
// copy rings (as in the unfold kernel), writes each candidate's score and
// gist id, and (default mode) folds the candidate gists and its share of
// the unselected meta-gists into an online-softmax partial record.
#pragma once

#include "common.cuh"
#include "k_unfold.cuh"

namespace gsa {

struct HgsaArgs {
  const void *q;                  // [B, hq, D]
  const void *gist_k, *gist_v;    // [B, hkv, n_max, D]
  const void *meta_v;             // [B, hkv, m_max, D]
  const float *meta_scores;       // [B*hq, m_max] natural units
  const int32_t *meta_idx;        // [B*hq, topk_meta] ascending, -1 padded
  const int32_t *n_gists;         // [B]
  int32_t group, topk_meta, m_max, n_max, hq, hkv, gqa, exclude;
  float scale_log2;
  float *cand_scores;             // [B*hq, cap]
  int32_t *cand_ids;              // [B*hq, cap]
  int32_t *cand_count;            // [B*hq]
  int32_t cap;
  float *part;                    // [B*hq, part_stride, D+4] (default mode); this pass: slots part_off ..
  int32_t n_split;
  uint32_t *status;
  // generalisations for a second meta level (zero / null: one level)
  int32_t count_div;              // entries at this level = n_gists[b] / count_div
  int32_t fold_children;          // fold the candidates' values into the partial (the gist level)
  const int32_t *parent_ids;      // parents to attend, as a list [B*hq, parent_cap] (null: all of [0, M))
  const float *parent_scores;     //   their scores (natural units), same layout
  const int32_t *parent_count;    //   list length per row
  int32_t parent_cap;
  int32_t part_stride, part_off;
};

constexpr int kHgsaThreads = 128;
constexpr int kHgsaWarps = kHgsaThreads / 32;
constexpr int kHgsaMaxGroups = 65;  // topk_meta <= 64, plus the trailing group

template <int D, typename T>
__global__ void __launch_bounds__(kHgsaThreads) k_hgsa_children(const HgsaArgs a) {
  constexpr int kE = Vec16<T>::kElems;
  constexpr int kLpr = D / kE;
  constexpr int kRpw = 32 / kLpr;
  constexpr int kRowBytes = D * static_cast<int>(sizeof(T));
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int groups[kHgsaMaxGroups];       // first gist of each candidate group
  __shared__ int group_rows[kHgsaMaxGroups];
  __shared__ int n_groups_s, n_sel_meta_s;
  __shared__ int sel_meta[64];
  __shared__ float red[kHgsaWarps][2 + D];
  __shared__ uint64_t bars[kHgsaWarps][8];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int kvh = h / a.gqa;
  const size_t row = static_cast<size_t>(b) * a.hq + h;
  const int g = a.group;
  const int pr = unfold_piece_rows<D, T>(g);
  const uint32_t piece_bytes = static_cast<uint32_t>(pr) * kRowBytes;
  const int sw = unfold_warp_stages(static_cast<int>(2 * piece_bytes));

  pdl_wait();
  const int N = min(max(a.n_gists[b] / a.count_div, 0), a.n_max);
  const int M = min(N / g, a.m_max);
  if (warp == 0) {
    // chosen groups, ascending (the meta top-k writes them in ascending order)
    int cnt = 0;
    for (int base = 0; base < a.topk_meta; base += 32) {
      const int i = base + lane;
      int j = i < a.topk_meta ? a.meta_idx[row * a.topk_meta + i] : -1;
      if (j >= M) {
        flag_error(a.status, GSA_DEVERR_BAD_INDEX);
        j = -1;
      }
      const unsigned ball = __ballot_sync(0xffffffffu, j >= 0);
      if (j >= 0) {
        const int slot = cnt + __popc(ball & ((1u << lane) - 1u));
        groups[slot] = j * g;
        group_rows[slot] = g;
        sel_meta[slot] = j;
      }
      cnt += __popc(ball);
    }
    if (lane == 0) {
      n_sel_meta_s = cnt;
      if (N > M * g) {
        groups[cnt] = M * g;
        group_rows[cnt] = N - M * g;
        ++cnt;
      }
      n_groups_s = cnt;
      if (split == 0) a.cand_count[row] = n_sel_meta_s * g + (N - M * g);
    }
    if (lane < kHgsaWarps)
      for (int s = 0; s < sw; ++s) mbar_init(&bars[lane][s], 1);
    if (lane == 0) mbar_fence_init();
  }
  __syncthreads();
  const int n_groups = n_groups_s, n_sel_meta = n_sel_meta_s;

  // Pieces: ppg per group (the trailing group may use fewer rows).
  const int ppg = (g + pr - 1) / pr;
  const int n_pieces_total = n_groups * ppg;
  // pieces of this split: p = split + n_split * i
  const int n_split_pieces = n_pieces_total > split ? (n_pieces_total - split + a.n_split - 1) / a.n_split : 0;
  const int n_mine = n_split_pieces > warp ? (n_split_pieces - warp + kHgsaWarps - 1) / kHgsaWarps : 0;
  auto piece_of = [&](int li) { return split + a.n_split * (warp + kHgsaWarps * li); };

  const size_t gbase = (static_cast<size_t>(b) * a.hkv + kvh) * a.n_max;
  const uint8_t *gk = reinterpret_cast<const uint8_t *>(a.gist_k) + gbase * kRowBytes;
  const uint8_t *gv = reinterpret_cast<const uint8_t *>(a.gist_v) + gbase * kRowBytes;
  uint8_t *ring = smem + static_cast<size_t>(warp) * sw * 2 * piece_bytes;
  const bool with_v = !a.exclude && a.fold_children;  // candidate values go into the partial
  auto piece = [&](int p, int &first, int &rows, int &slot0) {
    const int gi = p / ppg, sub = p % ppg;
    first = groups[gi] + sub * pr;
    rows = max(0, min(pr, group_rows[gi] - sub * pr));
    slot0 = gi * g + sub * pr;
  };
  auto issue = [&](int li) {
    int first, rows, slot0;
    piece(piece_of(li), first, rows, slot0);
    const int st = li % sw;
    const uint32_t bytes = static_cast<uint32_t>(rows) * kRowBytes;
    uint8_t *dst = ring + static_cast<size_t>(st) * 2 * piece_bytes;
    mbar_arrive_expect_tx(&bars[warp][st], (with_v ? 2u : 1u) * bytes);
    if (bytes) {
      bulk_g2s(dst, gk + static_cast<size_t>(first) * kRowBytes, bytes, &bars[warp][st]);
      if (with_v) bulk_g2s(dst + piece_bytes, gv + static_cast<size_t>(first) * kRowBytes, bytes, &bars[warp][st]);
    }
  };
  if (lane == 0)
    for (int li = 0; li < min(sw, n_mine); ++li) issue(li);

  const int slot = lane / kLpr;
  const int dd = kE * (lane % kLpr);
  float qf[kE];
  Vec16<T>::unpack(*reinterpret_cast<const uint4 *>(reinterpret_cast<const T *>(a.q) + row * D + dd), qf);
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
    const float pz = exp2_approx(z - m);
    l += pz;
#pragma unroll
    for (int e = 0; e < kE; ++e) acc[e] = fmaf(pz, vf[e], acc[e]);
  };

  int stuck = -1;
  for (int li = 0; li < n_mine; ++li) {
    const int st = li % sw;
    if (!__all_sync(0xffffffffu, mbar_wait(&bars[warp][st], (li / sw) & 1))) {
      stuck = li;
      break;
    }
    int first, rows, slot0;
    piece(piece_of(li), first, rows, slot0);
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
        const float z = part * a.scale_log2;
        if (lane % kLpr == 0) {
          a.cand_scores[row * a.cap + slot0 + r] = z * kLn2;
          a.cand_ids[row * a.cap + slot0 + r] = first + r;
        }
        if (with_v) {
          float vf[kE];
          Vec16<T>::unpack(lds_v4(Vs + r * kRowBytes + dd * static_cast<int>(sizeof(T))), vf);
          update(z, vf);
        }
      }
    }
    __syncwarp();
    if (lane == 0 && li + sw < n_mine) issue(li + sw);
  }
  if (stuck >= 0 && lane == 0) {
    flag_error(a.status, GSA_DEVERR_TIMEOUT);
    for (int li = stuck; li < min(stuck + sw, n_mine); ++li) mbar_wait(&bars[warp][li % sw], (li / sw) & 1);
  }
  if (a.exclude) return;

  // Unselected parents of this split's share: all of [0, M) with logits
  // from the meta scores, or the listed parents (positions of the list)
  // with their own scores; values from meta_v.
  const bool listed = a.parent_ids != nullptr;
  const int P = listed ? min(max(a.parent_count[row], 0), a.parent_cap) : M;
  const int per_m = (P + a.n_split - 1) / a.n_split;
  const int j0 = min(P, split * per_m), j1 = min(P, j0 + per_m);
  auto parent_id = [&](int j) { return listed ? a.parent_ids[row * a.parent_cap + j] : j; };
  const T *mv = reinterpret_cast<const T *>(a.meta_v) + (static_cast<size_t>(b) * a.hkv + kvh) * a.m_max * D;
  const float *ms = a.meta_scores + row * a.m_max;
  constexpr int kU = 8;                          // meta rows in flight per lane group
  constexpr int kStride = kHgsaWarps * kRpw;     // rows between a lane group's consecutive rows
  // a lane group's rows ascend (listed parents are in ascending id order
  // too), so one pointer walks the ascending sel_meta
  int sp = 0;
  {
    const int jfirst = j0 + warp * kRpw + slot;
    const int idfirst = jfirst < j1 ? parent_id(jfirst) : 0x7fffffff;
    int hi = n_sel_meta;
    while (sp < hi) {
      const int mid = (sp + hi) >> 1;
      if (sel_meta[mid] < idfirst) sp = mid + 1; else hi = mid;
    }
  }
  for (int jb = j0 + warp * kRpw + slot; jb - slot < j1; jb += kStride * kU) {
    uint4 w[kU];
    float z[kU];
    bool use[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int j = jb + u * kStride;
      const int id = j < j1 ? parent_id(j) : 0x7fffffff;
      while (sp < n_sel_meta && sel_meta[sp] < id) ++sp;
      const bool chosen = sp < n_sel_meta && sel_meta[sp] == id;
      use[u] = j < j1 && !chosen;
      // every load of the batch is issued before the first is used
      w[u] = use[u] ? *reinterpret_cast<const uint4 *>(mv + static_cast<size_t>(id) * D + dd) : make_uint4(0, 0, 0, 0);
      z[u] = use[u] ? (listed ? __ldcg(a.parent_scores + row * a.parent_cap + j) : __ldcg(ms + id)) * kLog2e : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kU; ++u)
      if (use[u]) {
        float vf[kE];
        Vec16<T>::unpack(w[u], vf);
        update(z[u], vf);
      }
  }
  pdl_trigger();

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
  float *rec = a.part + (row * a.part_stride + a.part_off + split) * (D + kPartHeader);
  float M2 = neg_inf();
#pragma unroll
  for (int w = 0; w < kHgsaWarps; ++w) M2 = fmaxf(M2, red[w][0]);
  for (int dim = tid; dim < D; dim += kHgsaThreads) {
    float s = 0.f;
    if (M2 != neg_inf())
#pragma unroll
      for (int w = 0; w < kHgsaWarps; ++w) s += red[w][2 + dim] * exp2_approx(red[w][0] - M2);
    rec[kPartHeader + dim] = s;
  }
  if (tid == 0) {
    float L = 0.f;
    if (M2 != neg_inf())
#pragma unroll
      for (int w = 0; w < kHgsaWarps; ++w) L += red[w][1] * exp2_approx(red[w][0] - M2);
    rec[0] = M2;
    rec[1] = L;
    rec[2] = 0.f;
    rec[3] = 0.f;
  }
}

}  // namespace gsa
