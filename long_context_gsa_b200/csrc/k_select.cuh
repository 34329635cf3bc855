// k_select.cuh -- top-k chunk selection of one row by a group of 128
// threads, run in the tail of the scoring kernel.  The last CTAs to finish
// a (b, kv head) group share its query heads' rows, one row per thread group,
// while other groups are still streaming.
//
// Method: "Selectie" on gist.science/nl/paper/2604.20920 ("Het Proces"): the
// k gists of highest relevance s = q.k_g are kept; gist.science/ja section
// 2.1 step 3.  Equal scores go to the lower chunk index (the pages leave ties
// open).
//
// The row (fp32 scores, just written by the scoring pass, still in L2) is
// brought into shared memory by one bulk copy.  Scores become
// order-preserving uint32 keys, linear in exponent and mantissa, so equal
// key ranges are equal steps of log |s| (negative keys sit a factor 2^31
// below the non-negative ones, so a range of non-negative keys starts at the
// smallest non-negative one).
//  1. The maximum of every 16 consecutive scores (a group maximum): the
//     kk-th largest of them bounds the row's kk-th score from below (kk
//     groups, hence kk distinct gists, reach it).  A histogram of the group
//     maxima over 256 equal parts of their key range finds the bin b holding
//     it.  The bin function is monotone, so the scores in bins >= b form an
//     upper set of at least kk scores that contains the top kk: these are
//     the candidates (about 1.2 kk of them).
//  2. A second histogram over the candidates' key range finds the bin b2
//     holding the kk-th: candidates above b2 are taken, and the few in b2 are
//     ranked by (score desc, index asc).
//  3. The taken chunks are marked in a bitmap over the row, which is read
//     out in chunk order.
// Exact path (a crowded bin, e.g. long runs of equal scores): an 8-bit radix
// select over the keys finds the kk-th largest key T; keys above T are
// taken, and keys equal to T in chunk order while they last.
// The code is kept short (rolled loops): it runs once per row after a
// streaming pass, so its instructions are fetched cold.
#pragma once

#include <cstddef>

#include "common.cuh"

namespace gsa {

constexpr int kRowSelThreads = 128;  // threads selecting one row
constexpr int kSelGroup = 16;        // scores per group maximum
constexpr int kSelCandCap = 384;     // candidates of the fast path

// Scratch of one thread group; 16-byte aligned in size and start, because the
// row is the destination of a bulk copy and groups sit back to back.
template <int NMAX>
struct alignas(16) SelSmem {
  float row[NMAX];
  uint32_t gm[NMAX / kSelGroup];
  uint32_t bits[2][NMAX / 32];  // taken; equal to the exact path's threshold
  unsigned long long cand[kSelCandCap];
  unsigned long long mem[32];
  uint32_t hist[256];
  uint32_t red[4][kRowSelThreads / 32];
  uint64_t bar;
  int info[4];
  int ncand, nmem;
  int pad[2];
};
static_assert(sizeof(SelSmem<4096>) % 16 == 0 && sizeof(SelSmem<8192>) % 16 == 0, "groups' rows stay 16-byte aligned");
static_assert(offsetof(SelSmem<4096>, row) == 0 && offsetof(SelSmem<8192>, bar) % 8 == 0, "layout");

// Append from the lanes with want: one shared atomic per warp; returns each
// wanting lane's slot.  Called by all 32 lanes.
__device__ __forceinline__ int warp_append(bool want, int *counter) {
  const int lane = threadIdx.x & 31;
  const unsigned m = __ballot_sync(0xffffffffu, want);
  int base = 0;
  if (m) {
    const int leader = __ffs(m) - 1;
    if (lane == leader) base = atomicAdd(counter, __popc(m));
    base = __shfl_sync(0xffffffffu, base, leader);
  }
  return base + __popc(m & ((1u << lane) - 1u));
}

// hist[bin] += 1 for every lane with bin >= 0, one shared atomic per
// distinct bin of the warp.  Called by all 32 lanes.
__device__ __forceinline__ void warp_hist_add(uint32_t *hist, int bin) {
  const unsigned peers = __match_any_sync(0xffffffffu, bin);
  if (bin >= 0 && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[bin], static_cast<uint32_t>(__popc(peers)));
}

__device__ __forceinline__ void group_bar(int id) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(kRowSelThreads) : "memory");
}

// Bin of rank `rem` (1-based, from the top) of the 256-bin histogram, by the
// group's first warp: info[0] = bin, info[1] = entries above it, info[2] =
// entries in it.
__device__ __forceinline__ void sel_find_bin(const uint32_t *hist, int rem, int lane, int *info) {
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
  for (int e = 7; e >= 0; --e) {
    if (cum < static_cast<uint32_t>(rem) && cum + c[e] >= static_cast<uint32_t>(rem)) {
      info[0] = lane * 8 + e;
      info[1] = static_cast<int>(cum);
      info[2] = static_cast<int>(c[e]);
    }
    cum += c[e];
  }
}

// Group-wide min (a, b), max (c) and sum (d) of one value per thread.
template <int NMAX>
__device__ __forceinline__ void sel_reduce(uint32_t &a, uint32_t &b, uint32_t &c, uint32_t &d, int gtid,
                                           SelSmem<NMAX> &sm, int bar_id) {
  const int lane = gtid & 31, w = gtid >> 5;
  for (int o = 16; o > 0; o >>= 1) {
    a = min(a, __shfl_xor_sync(0xffffffffu, a, o));
    b = min(b, __shfl_xor_sync(0xffffffffu, b, o));
    c = max(c, __shfl_xor_sync(0xffffffffu, c, o));
    d += __shfl_xor_sync(0xffffffffu, d, o);
  }
  if (lane == 0) {
    sm.red[0][w] = a;
    sm.red[1][w] = b;
    sm.red[2][w] = c;
    sm.red[3][w] = d;
  }
  group_bar(bar_id);
  a = b = 0xFFFFFFFFu;
  c = d = 0u;
  for (int i = 0; i < kRowSelThreads / 32; ++i) {
    a = min(a, sm.red[0][i]);
    b = min(b, sm.red[1][i]);
    c = max(c, sm.red[2][i]);
    d += sm.red[3][i];
  }
  group_bar(bar_id);  // red is reused
}


// Keys of unit g (gsz = 16 consecutive scores, or 1) of the row in shared
// memory; 0 (below every valid key) past the row's end or the unit.
__device__ __forceinline__ void sel_unit_keys(const float *row, int g, int gsz, int n, uint32_t (&kv)[kSelGroup]) {
  const int m0 = g * gsz;
  if (gsz == kSelGroup && m0 + kSelGroup <= n) {
    const float4 *p = reinterpret_cast<const float4 *>(row + m0);
    const float4 a = p[0], b = p[1], c = p[2], d = p[3];
    kv[0] = float_to_key(a.x); kv[1] = float_to_key(a.y); kv[2] = float_to_key(a.z); kv[3] = float_to_key(a.w);
    kv[4] = float_to_key(b.x); kv[5] = float_to_key(b.y); kv[6] = float_to_key(b.z); kv[7] = float_to_key(b.w);
    kv[8] = float_to_key(c.x); kv[9] = float_to_key(c.y); kv[10] = float_to_key(c.z); kv[11] = float_to_key(c.w);
    kv[12] = float_to_key(d.x); kv[13] = float_to_key(d.y); kv[14] = float_to_key(d.z); kv[15] = float_to_key(d.w);
  } else {
#pragma unroll
    for (int j = 0; j < kSelGroup; ++j) kv[j] = (j < gsz && m0 + j < n) ? float_to_key(row[m0 + j]) : 0u;
  }
}

// Exclusive scan of v over the group's threads (returned), with the total
// in *total, and the group-wide min of lo and max of hi (in place): one
// barrier.
template <typename Smem>
__device__ __forceinline__ int sel_scan_minmax(int v, uint32_t &lo, uint32_t &hi, int gtid, Smem &sm, int bar_id,
                                               int *total) {
  const int lane = gtid & 31, w = gtid >> 5;
  int inc = v;
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (lane == 31) {
    sm.red[0][w] = static_cast<uint32_t>(inc);
    sm.red[1][w] = lo;
    sm.red[2][w] = hi;
  }
  group_bar(bar_id);
  int before = 0, all = 0;
  for (int i = 0; i < kRowSelThreads / 32; ++i) {
    const int x = static_cast<int>(sm.red[0][i]);
    before += i < w ? x : 0;
    all += x;
    lo = min(lo, sm.red[1][i]);
    hi = max(hi, sm.red[2][i]);
  }
  *total = all;
  return before + inc - v;
}


// Monotone bin of a key: 0 .. 255 for keys >= base, -1 below.  The bins
// are equal power-of-two key ranges (shift chosen so that hi lands in bin
// 255 or below): integer subtract and shift, no conversions.
struct SelBins {
  uint32_t base;
  int shift;
  __device__ __forceinline__ void init(uint32_t lo, uint32_t hi) {
    base = lo;
    const uint32_t span = hi - lo;
    shift = span < 256u ? 0 : 24 - __clz(span);  // (span >> shift) < 256
  }
  __device__ __forceinline__ int operator()(uint32_t key) const {
    return key < base ? -1 : static_cast<int>((key - base) >> shift);
  }
};

// Keys of the rows' group maxima (all, or the scores themselves when there
// are fewer groups than kk): their range and histogram; returns bin b.
template <int NMAX>
__device__ int sel_bound(SelSmem<NMAX> &sm, int nv, bool by_group, int kk, int gtid, int bar_id, SelBins &bins) {
  uint32_t lo = 0xFFFFFFFFu, lo_pos = 0xFFFFFFFFu, hi = 0u, npos = 0u;
  for (int i = gtid; i < nv; i += kRowSelThreads) {
    const uint32_t key = by_group ? sm.gm[i] : float_to_key(sm.row[i]);
    lo = min(lo, key);
    hi = max(hi, key);
    if (key >= 0x80000000u) {  // float_to_key(+0)
      lo_pos = min(lo_pos, key);
      ++npos;
    }
  }
  sel_reduce(lo, lo_pos, hi, npos, gtid, sm, bar_id);
  bins.init(npos >= static_cast<uint32_t>(kk) ? lo_pos : lo, hi);
  for (int i0 = 0; i0 < nv; i0 += kRowSelThreads) {
    const int i = i0 + gtid;
    warp_hist_add(sm.hist, i < nv ? bins(by_group ? sm.gm[i] : float_to_key(sm.row[i])) : -1);
  }
  group_bar(bar_id);
  if (gtid < 32) sel_find_bin(sm.hist, kk, gtid, sm.info);
  group_bar(bar_id);
  const int b = sm.info[0];
  for (int i = gtid; i < 256; i += kRowSelThreads) sm.hist[i] = 0u;
  return b;
}

// Exact path: radix select of the kk-th largest key T; bits[0] marks keys
// above T, bits[1] keys equal to T; returns how many of the latter to take.
template <int NMAX>
__device__ __noinline__ int sel_exact(SelSmem<NMAX> &sm, int n, int kk, int gtid, int bar_id) {
  uint32_t prefix = 0, pmask = 0;
  int rem = kk;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = gtid; i < 256; i += kRowSelThreads) sm.hist[i] = 0u;
    group_bar(bar_id);
    for (int i0 = 0; i0 < n; i0 += kRowSelThreads) {
      const int i = i0 + gtid;
      const uint32_t key = i < n ? float_to_key(sm.row[i]) : 0u;
      warp_hist_add(sm.hist, i < n && (key & pmask) == prefix ? static_cast<int>((key >> shift) & 255u) : -1);
    }
    group_bar(bar_id);
    if (gtid < 32) sel_find_bin(sm.hist, rem, gtid, sm.info);
    group_bar(bar_id);
    rem -= sm.info[1];
    prefix |= static_cast<uint32_t>(sm.info[0]) << shift;
    pmask |= 0xFFu << shift;
    const bool whole = sm.info[2] == rem;
    group_bar(bar_id);
    if (whole) break;
  }
  for (int i = gtid; i < n; i += kRowSelThreads) {
    const uint32_t km = float_to_key(sm.row[i]) & pmask;
    if (km > prefix) atomicOr(&sm.bits[0][i >> 5], 1u << (i & 31));
    if (km == prefix) atomicOr(&sm.bits[1][i >> 5], 1u << (i & 31));
  }
  return rem;
}

// The kk (0 < kk < n <= NMAX) highest-scoring chunks of one row, in
// ascending chunk order, into out_idx / out_score (global).  srow: the
// row's scores (16-byte aligned).  Called by the kRowSelThreads threads of one
// group (gtid 0 .. 127), which synchronise on named barrier bar_id.
template <int NMAX>
__device__ void group_select_row(const float *srow, int n, int kk, int gtid, SelSmem<NMAX> &sm, int bar_id,
                                 int use, uint32_t *status, int32_t *out_idx, float *out_score) {
  // 0. the row into shared memory (one bulk copy), bitmaps and counts
  // cleared, once every thread is done with the group's previous row
  group_bar(bar_id);
  const int nw = (n + 31) >> 5;
  for (int i = gtid; i < 2 * (NMAX / 32); i += kRowSelThreads) (&sm.bits[0][0])[i] = 0u;
  for (int i = gtid; i < 256; i += kRowSelThreads) sm.hist[i] = 0u;
  const int n4 = (reinterpret_cast<uintptr_t>(srow) & 15u) == 0 ? (n & ~3) : 0;
  if (gtid == 0) {
    sm.nmem = 0;
    if (use == 0) {  // the scratch's copy barrier is set up once; each row is one phase of it
      mbar_init(&sm.bar, 1);
      mbar_fence_init();
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // the buffer was last written by this CTA's threads
    mbar_arrive_expect_tx(&sm.bar, static_cast<uint32_t>(n4) * 4u);
    if (n4 > 0) bulk_g2s(sm.row, srow, static_cast<uint32_t>(n4) * 4u, &sm.bar);
  }
  for (int i = n4 + gtid; i < n; i += kRowSelThreads) sm.row[i] = __ldcg(srow + i);
  const uint32_t parity = static_cast<uint32_t>(use) & 1u;
  if (gtid == 0) {
    int ok = mbar_wait(&sm.bar, parity);
    if (!ok) {  // flag it; wait once more so that no copy is left in flight
      flag_error(status, GSA_DEVERR_TIMEOUT);
      mbar_wait(&sm.bar, parity);
    }
    sm.info[3] = ok;
  }
  group_bar(bar_id);
  if (!sm.info[3]) return;     // group-uniform
  mbar_wait(&sm.bar, parity);  // complete already: makes the copied row visible to this thread
  // 1. group maxima (four 16-byte loads per group), the bound
  const int n_groups = (n + kSelGroup - 1) / kSelGroup;
  const bool by_group = n_groups >= kk;
  uint32_t kv[kSelGroup];
  if (by_group)
    for (int g = gtid; g < n_groups; g += kRowSelThreads) {
      sel_unit_keys(sm.row, g, kSelGroup, n, kv);
      uint32_t mx = 0u;  // valid keys are nonzero
#pragma unroll
      for (int j = 0; j < kSelGroup; ++j) mx = max(mx, kv[j]);
      sm.gm[g] = mx;
    }
  group_bar(bar_id);
  SelBins bin1;
  const int nv = by_group ? n_groups : n;
  const int gsz = by_group ? kSelGroup : 1;
  const int b = sel_bound(sm, nv, by_group, kk, gtid, bar_id, bin1);
  // 2. the candidates: each thread scans its own units (groups gtid + 128 r
  // whose maximum reaches bin b, or single scores), counts, takes its slots
  // from a scan over the group, and writes them
  int cnt = 0;
  uint32_t clo = 0xFFFFFFFFu, chi = 0u;
  for (int g = gtid; g < nv; g += kRowSelThreads) {
    if (bin1(by_group ? sm.gm[g] : float_to_key(sm.row[g])) < b) continue;
    sel_unit_keys(sm.row, g, gsz, n, kv);
#pragma unroll
    for (int j = 0; j < kSelGroup; ++j)
      if (kv[j] && bin1(kv[j]) >= b) {
        ++cnt;
        clo = min(clo, kv[j]);
        chi = max(chi, kv[j]);
      }
  }
  int C;
  int slot = sel_scan_minmax(cnt, clo, chi, gtid, sm, bar_id, &C);
  if (C <= kSelCandCap)
    for (int g = gtid; g < nv; g += kRowSelThreads) {
      if (bin1(by_group ? sm.gm[g] : float_to_key(sm.row[g])) < b) continue;
      sel_unit_keys(sm.row, g, gsz, n, kv);
#pragma unroll
      for (int j = 0; j < kSelGroup; ++j)
        if (kv[j] && bin1(kv[j]) >= b) {
          const int i = g * gsz + j;
          sm.cand[slot++] = (static_cast<unsigned long long>(kv[j]) << 32) | static_cast<uint32_t>(i);
        }
    }
  group_bar(bar_id);
  int take_eq = 0;
  // C < kk cannot happen (the bound counts scores of this row)
  bool exact = C > kSelCandCap || C < kk;
  if (!exact) {
    // 2. the candidates' bin b2 holding the kk-th, and its members ranked
    SelBins bin2;
    bin2.init(clo, chi);
    for (int c0 = 0; c0 < C; c0 += kRowSelThreads) {
      const int c = c0 + gtid;
      warp_hist_add(sm.hist, c < C ? bin2(static_cast<uint32_t>(sm.cand[c] >> 32)) : -1);
    }
    group_bar(bar_id);
    if (gtid < 32) sel_find_bin(sm.hist, kk, gtid, sm.info);
    group_bar(bar_id);
    const int b2 = sm.info[0], need = kk - sm.info[1], inbin = sm.info[2];
    exact = inbin > 32;  // a crowded bin
    if (!exact) {
      for (int c0 = 0; c0 < C; c0 += kRowSelThreads) {
        const int c = c0 + gtid;
        const unsigned long long x = c < C ? sm.cand[c] : 0ull;
        const int bx = c < C ? bin2(static_cast<uint32_t>(x >> 32)) : -1;
        const int i = static_cast<int>(static_cast<uint32_t>(x));
        if (bx > b2) atomicOr(&sm.bits[0][i >> 5], 1u << (i & 31));
        const int slot = warp_append(bx == b2, &sm.nmem);
        if (bx == b2) sm.mem[slot] = x;
      }
      group_bar(bar_id);
      if (gtid < inbin) {  // taken: fewer than `need` members ahead (larger key, or equal key and lower index)
        const unsigned long long x = sm.mem[gtid];
        const uint32_t xk = static_cast<uint32_t>(x >> 32), xi = static_cast<uint32_t>(x);
        int rank = 0;
        for (int s = 0; s < inbin; ++s) {
          const unsigned long long y = sm.mem[s];
          const uint32_t yk = static_cast<uint32_t>(y >> 32);
          rank += (yk > xk || (yk == xk && static_cast<uint32_t>(y) < xi)) ? 1 : 0;
        }
        if (rank < need) atomicOr(&sm.bits[0][xi >> 5], 1u << (xi & 31));
      }
    }
  }
  if (exact) {  // group-uniform
    for (int i = gtid; i < nw; i += kRowSelThreads) sm.bits[0][i] = 0u;
    group_bar(bar_id);
    take_eq = sel_exact(sm, n, kk, gtid, bar_id);
  }
  group_bar(bar_id);
  // 3. read the bitmaps out in chunk order: bits[0], and the first take_eq of bits[1]
  const int wpt = (nw + kRowSelThreads - 1) / kRowSelThreads;
  const int w0 = min(nw, gtid * wpt), w1 = min(nw, w0 + wpt);
  uint32_t my_sel = 0u, my_eq = 0u;
  for (int w = w0; w < w1; ++w) {
    my_sel += __popc(sm.bits[0][w]);
    my_eq += __popc(sm.bits[1][w]);
  }
  // exclusive prefix over threads (index order) of my_eq, then of the taken count
  const int lane = gtid & 31, wid = gtid >> 5;
  uint32_t inc = my_eq;
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  if (lane == 31) sm.red[0][wid] = inc;
  group_bar(bar_id);
  uint32_t eq_before = inc - my_eq;
  for (int i = 0; i < wid; ++i) eq_before += sm.red[0][i];
  const uint32_t my_take_eq = min(my_eq, static_cast<uint32_t>(max(0, take_eq - static_cast<int>(eq_before))));
  const uint32_t mine = my_sel + my_take_eq;
  inc = mine;
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  if (lane == 31) sm.red[1][wid] = inc;
  group_bar(bar_id);
  uint32_t pos = inc - mine;
  for (int i = 0; i < wid; ++i) pos += sm.red[1][i];
  uint32_t eq_left = my_take_eq;
  for (int w = w0; w < w1; ++w) {
    uint32_t e = sm.bits[1][w];
    uint32_t t = sm.bits[0][w];
    while (e && eq_left) {  // this thread's equal keys, lowest first, while its share lasts
      const uint32_t low = e & (0u - e);
      t |= low;
      e ^= low;
      --eq_left;
    }
    while (t) {
      const int bit = __ffs(t) - 1;
      t &= t - 1u;
      const int m = (w << 5) + bit;
      if (pos < static_cast<uint32_t>(kk)) {
        out_idx[pos] = m;
        if (out_score) out_score[pos] = sm.row[m];
      }
      ++pos;
    }
  }
}

// The selection of one row: kk = min(k, n) chunks in ascending order, then
// -1 / -inf padding up to k (n <= NMAX).  Called by the 128 threads of one
// group.
// `use` counts the rows this group has selected with this scratch before.
template <int NMAX>
__device__ void group_select(const float *srow, int n, int k, int gtid, SelSmem<NMAX> &sm, int bar_id, int &use,
                             uint32_t *status, int32_t *out_idx, float *out_score) {
  const int kk = min(k, n);
  if (kk >= n) {
    for (int i = gtid; i < n; i += kRowSelThreads) {
      out_idx[i] = i;
      if (out_score) out_score[i] = __ldcg(srow + i);
    }
  } else if (kk > 0) {
    group_select_row<NMAX>(srow, n, kk, gtid, sm, bar_id, use, status, out_idx, out_score);
    ++use;
  }
  for (int i = kk + gtid; i < k; i += kRowSelThreads) {
    out_idx[i] = -1;
    if (out_score) out_score[i] = neg_inf();
  }
}

}  // namespace gsa
