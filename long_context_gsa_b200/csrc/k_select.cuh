// k_select.cuh -- top-k chunk selection of one row by one warp, run in the
// tail of the scoring kernel: the CTA that finishes a (b, kv head) group
// last selects for the group's query heads, one warp per head, while other
// groups are still streaming.
//
// Method: "Selectie" on gist.science/nl/paper/2604.20920 ("Het Proces"): the
// k gists of highest relevance s = q.k_g are kept; gist.science/ja section
// 2.1 step 3.  Equal scores go to the lower chunk index (the pages leave ties
// open).
//
// Inputs: the row's scores (fp32, just written by the scoring pass and still
// in L2) and its group maxima: the maximum score of every 16 consecutive
// gists, which the scoring pass produces on the side.
//
// Fast path (a bound, then a few candidates in chunk order):
//  1. the kk-th largest group maximum bounds the row's kk-th score from
//     below (kk groups, hence kk distinct gists, reach it).  A histogram of
//     the group maxima's order-preserving keys over 256 equal ranges of
//     [min, max] (from the smallest non-negative one when kk are
//     non-negative: keys are linear in exponent and mantissa, so equal key
//     ranges are equal steps of log |s|, except across zero) finds the range
//     holding it; L = that range's lowest key is a slightly looser bound.
//     Rows with fewer than kk groups use the scores themselves as the
//     "groups" of one;
//  2. candidates: the scores >= L inside the groups whose maximum reaches L,
//     collected in ascending chunk order (about 1.2 kk of them);
//  3. a second histogram over the candidates' keys finds the range holding
//     the kk-th one: candidates above it are all selected, and the few
//     inside it are ranked by (score desc, index asc);
//  4. the selected candidates are written out in the order they were
//     collected, i.e. ascending chunk order.
// Exact fallback (a range too crowded to rank, e.g. long runs of equal
// scores, or a row too long for the group list): an 8-bit radix select over
// all the row's scores finds the kk-th largest key T; the selection is every
// key above T plus the lowest-indexed keys equal to T, in ascending order.
#pragma once

#include "common.cuh"

namespace gsa {

constexpr int kSelGroup = 16;      // gists per group maximum
constexpr int kSelValCap = 1024;   // group (or score) list the fast path takes
constexpr int kSelCandCap = 512;   // candidates the fast path keeps

// Scratch of one warp's selection.
struct WarpSelSmem {
  float vals[kSelValCap];
  unsigned long long cand[kSelCandCap];  // (score key << 32) | chunk index, in chunk order
  unsigned long long mem[32];            // the members of the boundary range, in chunk order
  uint32_t hist[256];
  uint16_t cg[kSelValCap];
};

__device__ __forceinline__ int warp_excl_scan(int v, int lane) {
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  return incl - v;
}

// The bin of rank `rem` (1-based, counted from the top) of a 256-bin
// histogram: returns the bin, *above = entries in higher bins, *inbin =
// entries in the bin (the same in every lane).
__device__ __forceinline__ int warp_find_bin(const uint32_t *hist, int rem, int lane, int *above, int *inbin) {
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
  int bin = -1, ab = 0, in = 0;
#pragma unroll
  for (int e = 7; e >= 0; --e) {
    if (cum < static_cast<uint32_t>(rem) && cum + c[e] >= static_cast<uint32_t>(rem)) {
      bin = lane * 8 + e;
      ab = static_cast<int>(cum);
      in = static_cast<int>(c[e]);
    }
    cum += c[e];
  }
  const unsigned owner = __ballot_sync(0xffffffffu, bin >= 0);
  const int src = owner ? __ffs(owner) - 1 : 0;
  *above = __shfl_sync(0xffffffffu, ab, src);
  *inbin = __shfl_sync(0xffffffffu, in, src);
  return __shfl_sync(0xffffffffu, bin, src);
}

__device__ __forceinline__ void sel_put(int32_t *out_idx, float *out_score, int pos, int idx, float s) {
  out_idx[pos] = idx;
  if (out_score) out_score[pos] = s;
}

// Exact selection over all n scores by one warp (the fallback); writes the
// kk chosen chunks in ascending order.
__device__ __noinline__ void warp_select_radix(const float *srow, int n, int kk, uint32_t *hist, int32_t *out_idx,
                                               float *out_score) {
  const int lane = threadIdx.x & 31;
  uint32_t prefix = 0, pmask = 0;
  int rem = kk;
  bool take_all_eq = false;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = lane; i < 256; i += 32) hist[i] = 0u;
    __syncwarp();
    for (int i = lane; i < n; i += 32) {
      const uint32_t key = float_to_key(__ldcg(srow + i));
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncwarp();
    int above, inbin;
    const int digit = warp_find_bin(hist, rem, lane, &above, &inbin);
    __syncwarp();
    rem -= above;
    prefix |= static_cast<uint32_t>(digit) << shift;
    pmask |= 0xFFu << shift;
    if (inbin == rem) {
      take_all_eq = true;
      break;
    }
  }
  // keys above the prefix, then keys on it in index order while rem lasts
  const unsigned lt = (1u << lane) - 1u;
  int pos = 0, eq_seen = 0;
  for (int base = 0; base < n; base += 32) {
    const int i = base + lane;
    const float s = i < n ? __ldcg(srow + i) : 0.f;
    const uint32_t km = float_to_key(s) & pmask;
    const bool gt = i < n && km > prefix, eq = i < n && km == prefix;
    const unsigned eqs = __ballot_sync(0xffffffffu, eq);
    const bool take = gt || (eq && (take_all_eq || eq_seen + __popc(eqs & lt) < rem));
    const unsigned tk = __ballot_sync(0xffffffffu, take);
    const int o = pos + __popc(tk & lt);
    if (take && o < kk) sel_put(out_idx, out_score, o, i, s);
    pos += __popc(tk);
    eq_seen += __popc(eqs);
  }
}

// The kk (0 < kk < n) highest-scoring chunks of one row, in ascending chunk
// order, written to out_idx / out_score (global).  srow: the row's n
// scores; gmax: its ceil(n / kSelGroup) group maxima.  Called by one whole
// warp; sm is that warp's scratch.
__device__ void warp_select_row(const float *srow, const float *gmax, int n, int kk, WarpSelSmem &sm,
                                int32_t *out_idx, float *out_score) {
  const int lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  const int n_groups = (n + kSelGroup - 1) / kSelGroup;
  const bool by_group = n_groups >= kk;
  const float *vals = by_group ? gmax : srow;
  const int nv = by_group ? n_groups : n;
  const int gsize = by_group ? kSelGroup : 1;
  if (nv > kSelValCap) {  // warp-uniform
    warp_select_radix(srow, n, kk, sm.hist, out_idx, out_score);
    return;
  }
  constexpr uint32_t kZeroKey = 0x80000000u;  // float_to_key(+0)
  // 1. stage the values; their key range; the bound L
  uint32_t lo = 0xFFFFFFFFu, lo_pos = 0xFFFFFFFFu, hi = 0u;
  int npos = 0;
  for (int i = lane; i < nv; i += 32) {
    const float f = __ldcg(vals + i);
    sm.vals[i] = f;
    const uint32_t key = float_to_key(f);
    lo = min(lo, key);
    hi = max(hi, key);
    if (key >= kZeroKey) {
      lo_pos = min(lo_pos, key);
      ++npos;
    }
  }
  for (int i = lane; i < 256; i += 32) sm.hist[i] = 0u;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    lo_pos = min(lo_pos, __shfl_xor_sync(0xffffffffu, lo_pos, o));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    npos += __shfl_xor_sync(0xffffffffu, npos, o);
  }
  if (npos >= kk) lo = lo_pos;
  __syncwarp();
  unsigned long long range = static_cast<unsigned long long>(hi - lo) + 1ull;
  for (int i = lane; i < nv; i += 32) {
    const uint32_t key = float_to_key(sm.vals[i]);
    if (key >= lo) atomicAdd(&sm.hist[static_cast<int>((static_cast<unsigned long long>(key - lo) << 8) / range)], 1u);
  }
  __syncwarp();
  int above, inbin;
  int b = warp_find_bin(sm.hist, kk, lane, &above, &inbin);
  const uint32_t L = lo + static_cast<uint32_t>((static_cast<unsigned long long>(b) * range + 255ull) >> 8);
  // 2. candidate groups in index order, then their scores >= L in index order
  int ncg = 0;
  for (int base = 0; base < nv; base += 32) {
    const int i = base + lane;
    const bool c = i < nv && float_to_key(sm.vals[i]) >= L;
    const unsigned bal = __ballot_sync(0xffffffffu, c);
    if (c) sm.cg[ncg + __popc(bal & lt)] = static_cast<uint16_t>(i);
    ncg += __popc(bal);
  }
  __syncwarp();
  int C = 0;
  const bool vec = gsize == kSelGroup && (reinterpret_cast<uintptr_t>(srow) & 15u) == 0;
  for (int base = 0; base < ncg; base += 32) {  // a round: one candidate group per lane
    const int c = base + lane;
    const int m0 = c < ncg ? static_cast<int>(sm.cg[c]) * gsize : n;
    float f[kSelGroup];
    if (vec && m0 + kSelGroup <= n) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 v4 = __ldcg(reinterpret_cast<const float4 *>(srow + m0) + j);
        f[4 * j] = v4.x;
        f[4 * j + 1] = v4.y;
        f[4 * j + 2] = v4.z;
        f[4 * j + 3] = v4.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < kSelGroup; ++j) f[j] = (j < gsize && m0 + j < n) ? __ldcg(srow + m0 + j) : 0.f;
    }
    uint32_t keep = 0;  // bit j: score j of this lane's group is a candidate
#pragma unroll
    for (int j = 0; j < kSelGroup; ++j)
      if (j < gsize && m0 + j < n && float_to_key(f[j]) >= L) keep |= 1u << j;
    int at = C + warp_excl_scan(__popc(keep), lane);
#pragma unroll
    for (int j = 0; j < kSelGroup; ++j)
      if ((keep >> j) & 1u) {
        if (at < kSelCandCap)
          sm.cand[at] = (static_cast<unsigned long long>(float_to_key(f[j])) << 32) | static_cast<uint32_t>(m0 + j);
        ++at;
      }
    C = __shfl_sync(0xffffffffu, at, 31);  // lane 31 ends at the round's total
  }
  __syncwarp();
  if (C > kSelCandCap || C < kk) {  // C < kk only if the maxima do not match the scores
    warp_select_radix(srow, n, kk, sm.hist, out_idx, out_score);
    return;
  }
  // 3. the candidates' range holding the kk-th one
  for (int i = lane; i < 256; i += 32) sm.hist[i] = 0u;
  __syncwarp();
  range = static_cast<unsigned long long>(hi - L) + 1ull;
  auto bin2 = [&](unsigned long long x) {
    return static_cast<int>((static_cast<unsigned long long>(static_cast<uint32_t>(x >> 32) - L) << 8) / range);
  };
  for (int i = lane; i < C; i += 32) atomicAdd(&sm.hist[bin2(sm.cand[i])], 1u);
  __syncwarp();
  b = warp_find_bin(sm.hist, kk, lane, &above, &inbin);
  const int need = kk - above;  // taken from range b, by (score desc, index asc)
  if (inbin > 32) {  // a crowded range (many equal scores): the exact path
    warp_select_radix(srow, n, kk, sm.hist, out_idx, out_score);
    return;
  }
  int got = 0;  // range b's members, in chunk order
  for (int base = 0; base < C; base += 32) {
    const int i = base + lane;
    const bool inb = i < C && bin2(sm.cand[i]) == b;
    const unsigned bal = __ballot_sync(0xffffffffu, inb);
    if (inb) sm.mem[got + __popc(bal & lt)] = sm.cand[i];
    got += __popc(bal);
  }
  __syncwarp();
  bool taken = false;  // member `lane`: fewer than `need` members rank ahead of it
  if (lane < inbin) {
    const unsigned long long x = sm.mem[lane];
    int rank = 0;
    for (int s = 0; s < inbin; ++s) {
      const unsigned long long y = sm.mem[s];
      const uint32_t yk = static_cast<uint32_t>(y >> 32), xk = static_cast<uint32_t>(x >> 32);
      rank += (yk > xk || (yk == xk && static_cast<uint32_t>(y) < static_cast<uint32_t>(x))) ? 1 : 0;
    }
    taken = rank < need;
  }
  const unsigned taken_mask = __ballot_sync(0xffffffffu, taken);
  // 4. emit in chunk order: candidates above range b, and range b's taken members
  int pos = 0;
  got = 0;
  for (int base = 0; base < C; base += 32) {
    const int i = base + lane;
    const unsigned long long x = i < C ? sm.cand[i] : 0ull;
    const int bx = i < C ? bin2(x) : -1;
    const unsigned inb = __ballot_sync(0xffffffffu, bx == b);
    const bool take = bx > b || (bx == b && ((taken_mask >> (got + __popc(inb & lt))) & 1u));
    got += __popc(inb);
    const unsigned tk = __ballot_sync(0xffffffffu, take);
    const int o = pos + __popc(tk & lt);
    if (take && o < kk)
      sel_put(out_idx, out_score, o, static_cast<int>(static_cast<uint32_t>(x)), key_to_float(static_cast<uint32_t>(x >> 32)));
    pos += __popc(tk);
  }
}

// The selection of one row: kk = min(k, n) chunks in ascending order, then
// -1 / -inf padding up to k.  Called by one whole warp.
__device__ void warp_select(const float *srow, const float *gmax, int n, int k, WarpSelSmem &sm, int32_t *out_idx,
                            float *out_score) {
  const int lane = threadIdx.x & 31;
  const int kk = min(k, n);
  if (kk >= n) {
    for (int i = lane; i < n; i += 32) sel_put(out_idx, out_score, i, i, __ldcg(srow + i));
  } else if (kk > 0) {
    warp_select_row(srow, gmax, n, kk, sm, out_idx, out_score);
  }
  for (int i = kk + lane; i < k; i += 32) sel_put(out_idx, out_score, i, -1, neg_inf());
  __syncwarp();
}

}  // namespace gsa
