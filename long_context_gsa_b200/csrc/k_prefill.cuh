// k_prefill.cuh -- causal GSA prefill with interleaved gists.
//
// Method: gist.science/nl/paper/2604.20920 "Het Proces": Compressie (a gist
// token sees its own block and the preceding gists), Scoring, Selectie and
// Selectieve Ontvouwing applied at every position of the sequence.  A raw
// query at position i = m*c + j scores the completed gists 0..m-1, keeps
// the top k, and attends their chunks (raw + gist), the other completed
// gists (unless excluded) and its own chunk's raw tokens 0..j.  A gist query
// m attends chunk m's raw tokens and gists 0..m.
//
// Stage 1 (this file, k_prefill_score): the dense part -- every query row
// against every visible gist key -- on the 5th-generation tensor cores.
// Persistent CTAs walk query tiles of 128 rows of one head (gist-query
// tiles, then raw tiles, heaviest first).  Warp 0 issues TMA loads (Q tile,
// then 128-gist key tiles into a 2-stage ring), warp 1 issues tcgen05.mma
// into two 128-column TMEM accumulators, and warps 2..9 (two per TMEM lane
// quadrant, so two threads per query row, each owning half of the key
// columns) read the scores with tcgen05.ld, apply the block-causal mask and
// keep the row maximum.  For raw rows the top-k runs against a lower bound
// on the row's final k-th score: each half keeps the K largest scores it
// has appended (sorted, values only) and the partner half's K-th is read
// once per key tile; only scores above the bound are appended as (score,
// index) candidates to a per-row column in shared memory (column-major, so
// appends of different rows never share a bank).  At the end of the row one
// thread merges both halves' lists into the k-th score and walks both
// columns in ascending index order.
// Outputs: sel_idx/sel_score (ascending chunk order) and the row maximum
// that the attention stage uses as softmax reference.
#pragma once

#include "tc100.cuh"

namespace gsa {

struct PrefillArgs {
  CUtensorMap tm_qraw;   // [B*hq*L, d] bf16, box 128 x 64, SW128
  CUtensorMap tm_qgist;  // [B*hq*N, d]
  CUtensorMap tm_kgist;  // [B*hkv*N, d], box 256 x 64
  CUtensorMap tm_vgist;  // [B*hkv*N, d] fp16 copy of the gist values, box 128 x 64 (attention stage)
  int32_t bh, hq, hkv, group, chunk, n_chunks, L, topk, exclude;
  float scale, scale_log2;
  int32_t *sel_idx;      // [B*hq*L, topk]
  float *sel_score;      // [B*hq*L, topk]
  float *rec_raw;        // [B*hq*L, d+4] partial records; [0] = row max (base 2)
  float *rec_gist;       // [B*hq*N, d+4]
  int32_t gist_tiles;    // query tiles per head over the gist rows
  int32_t raw_tiles;     // query tiles per head over the raw rows
  uint32_t *status;
};

constexpr int kPfRows = 128;        // query rows per tile (TMEM lanes)
constexpr int kPfKeys = 128;        // gist keys per MMA tile (TMEM columns)
constexpr int kPfThreads = 192;     // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr int kPfTopkMax = 16;
constexpr int kPsThreads = 320;     // scoring: warp 0 TMA, warp 1 MMA, warps 2..9 epilogue (2 per row)
constexpr int kPsCap = 38;          // candidate slots per row half (shared memory)

struct PfTile {
  int is_gist, bh, row0, n_kt;
};

// Tile t of the work list: gist-query tiles (heaviest first), then raw
// tiles (heaviest first).  n_kt = gist key tiles the rows can see.
__device__ __forceinline__ PfTile pf_tile(const PrefillArgs &a, int t) {
  PfTile r;
  const int gt = a.bh * a.gist_tiles;
  if (t < gt) {
    r.is_gist = 1;
    r.bh = t % a.bh;
    r.row0 = (a.gist_tiles - 1 - t / a.bh) * kPfRows;
    const int visible = min(a.n_chunks, r.row0 + kPfRows);  // gist m sees 0..m
    r.n_kt = (visible + kPfKeys - 1) / kPfKeys;
  } else {
    const int u = t - gt;
    r.is_gist = 0;
    r.bh = u % a.bh;
    r.row0 = (a.raw_tiles - 1 - u / a.bh) * kPfRows;
    const int last = min(a.L - 1, r.row0 + kPfRows - 1);
    const int visible = min(a.n_chunks, last / a.chunk);    // raw i sees 0..i/c-1
    r.n_kt = (visible + kPfKeys - 1) / kPfKeys;
  }
  return r;
}

struct PfSmem {
  static constexpr uint32_t kQBlock = kPfRows * 128;         // 128 rows x 64 bf16
  static constexpr uint32_t kQBytes = 2 * kQBlock;           // d = 128
  static constexpr uint32_t kKBlock = kPfKeys * 128;
  static constexpr uint32_t kKBytes = 2 * kKBlock;
  static constexpr uint32_t kQOff = 0;                       // 2 Q buffers
  static constexpr uint32_t kKOff = 2 * kQBytes;             // kKStages K stages
  static constexpr int kKStages = 2;
  static constexpr uint32_t kCandOff = kKOff + kKStages * kKBytes;           // [2 halves][kPsCap][128] (score, index)
  static constexpr uint32_t kListOff = kCandOff + 2 * kPsCap * kPfRows * 8;  // [2][kPfTopkMax][128] best values
  static constexpr uint32_t kThrOff = kListOff + 2 * kPfTopkMax * kPfRows * 4;  // [2][128] (threshold, tile tag)
  static constexpr uint32_t kCntOff = kThrOff + 2 * kPfRows * 8;             // [2][128] filtered candidate counts
  static constexpr uint32_t kBarOff = kCntOff + 2 * kPfRows * 4;
  static constexpr uint32_t kBytes = kBarOff + 256 + 1008;   // + alignment slack (base is 16-byte aligned)
};
static_assert(PfSmem::kBytes <= 232448, "prefill scoring shared memory");

constexpr uint32_t kPsSlot = kPfRows * 8;  // bytes between consecutive slots of one row's column

// (score, index) ranking: higher score first, then lower index.
__device__ __forceinline__ bool pf_before(float x, int xi, float y, int yi) { return x > y || (x == y && xi < yi); }

__device__ __forceinline__ uint2 lds_u2(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a) : "memory");
  return v;
}

__device__ __forceinline__ void sts_u2(uint32_t a, uint2 v) {
  asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(a), "r"(v.x), "r"(v.y) : "memory");
}

// Append (v, idx) at the column cursor `cur` when v > thr (GE: v >= thr),
// without a branch: the store and the cursor step are predicated.  NaN
// (a masked score) fails both compares.
template <bool GE>
__device__ __forceinline__ void pf_append(uint32_t &cur, float v, float thr, uint32_t idx) {
  if (GE)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ge.f32 p, %1, %2;\n\t"
        "@p st.shared.v2.u32 [%0], {%3, %4};\n\t"
        "@p add.u32 %0, %0, %5;\n\t}\n"
        : "+r"(cur)
        : "f"(v), "f"(thr), "r"(__float_as_uint(v)), "r"(idx), "n"(kPsSlot)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.gt.f32 p, %1, %2;\n\t"
        "@p st.shared.v2.u32 [%0], {%3, %4};\n\t"
        "@p add.u32 %0, %0, %5;\n\t}\n"
        : "+r"(cur)
        : "f"(v), "f"(thr), "r"(__float_as_uint(v)), "r"(idx), "n"(kPsSlot)
        : "memory");
}

// Values-only insertion into a descending list (the running top K).
template <int K>
__device__ __forceinline__ void pf_insert(float (&b)[K], float x) {
#pragma unroll
  for (int q = 0; q < K; ++q) {
    const float hi = fmaxf(b[q], x);
    x = fminf(b[q], x);
    b[q] = hi;
  }
}

// Descending bitonic sort of 32 values in registers (no NaN inputs).
__device__ __forceinline__ void pf_sort32(float (&w)[32]) {
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1)
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1)
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int l = i ^ j;
        if (l > i) {
          const float x = w[i], y = w[l];
          const bool desc = (i & k) == 0;
          w[i] = desc ? fmaxf(x, y) : fminf(x, y);
          w[l] = desc ? fminf(x, y) : fmaxf(x, y);
        }
      }
}

// Store v at a when p (predicated, no branch).
__device__ __forceinline__ void sts_u2_if(bool p, uint32_t a, uint2 v) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %0, 0;\n\t@q st.shared.v2.u32 [%1], {%2, %3};\n\t}\n" ::"r"(
          static_cast<uint32_t>(p)),
      "r"(a), "r"(v.x), "r"(v.y)
      : "memory");
}

// Keep the column's candidates with score >= lb (order kept).  Called by
// the whole warp (one column per lane): the loop runs to the longest
// column, four slots per step with the loads issued together; a lane's
// slots past its cursor are read but neither kept nor counted (every
// address read lies inside the column's kPsCap slots).  Returns the cursor.
__device__ __forceinline__ uint32_t pf_filter(uint32_t base, uint32_t cur, float lb) {
  const int n = static_cast<int>((cur - base) / kPsSlot);
  const int nmax = __reduce_max_sync(0xffffffffu, n);
  uint32_t w = base;
  for (int s = 0; s < nmax; s += 4) {
    uint2 e[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) e[u] = lds_u2(base + min(s + u, kPsCap - 1) * kPsSlot);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const bool live = s + u < n;
      sts_u2_if(live, w, e[u]);  // w <= s + u: never overwrites an unread slot
      w += (live && __uint_as_float(e[u].x) >= lb) ? kPsSlot : 0u;
    }
  }
  return w;
}

// Rare path (many exactly equal scores): keep the column's best K
// candidates by (score desc, index asc), left in ascending index order;
// returns the new cursor.
template <int K>
__device__ __noinline__ uint32_t pf_reduce(uint32_t base, uint32_t cur) {
  float best[K];
  int bidx[K];
#pragma unroll
  for (int e = 0; e < K; ++e) {
    best[e] = neg_inf();
    bidx[e] = 0x7fffffff;
  }
  int cnt = 0;
  for (uint32_t s = base; s < cur; s += kPsSlot, ++cnt) {
    const uint2 en = lds_u2(s);
    float x = __uint_as_float(en.x);
    int xi = static_cast<int>(en.y);
#pragma unroll
    for (int q = 0; q < K; ++q)
      if (pf_before(x, xi, best[q], bidx[q])) {
        const float tv = best[q];
        const int ti = bidx[q];
        best[q] = x;
        bidx[q] = xi;
        x = tv;
        xi = ti;
      }
  }
  const int n = min(cnt, K);
#pragma unroll
  for (int i = 1; i < K; ++i)
#pragma unroll
    for (int j2 = K - 1; j2 >= i; --j2)
      if (bidx[j2 - 1] > bidx[j2]) {  // unused slots hold INT_MAX and sort last
        const int ti = bidx[j2 - 1];
        bidx[j2 - 1] = bidx[j2];
        bidx[j2] = ti;
        const float tv = best[j2 - 1];
        best[j2 - 1] = best[j2];
        best[j2] = tv;
      }
#pragma unroll
  for (int e = 0; e < K; ++e)
    if (e < n) sts_u2(base + e * kPsSlot, make_uint2(__float_as_uint(best[e]), static_cast<uint32_t>(bidx[e])));
  return base + n * kPsSlot;
}

// A value a little below x (x itself for -inf): comparing v > below(x)
// keeps every v >= x.
__device__ __forceinline__ float pf_below(float x) { return fmaf(-fabsf(x), 1e-6f, x) - 1e-30f; }

// Stage 1, k_prefill_score<K>: scores, row maxima and the top-k selection
// (topk <= K) of every query row.
template <int K>
__global__ void __launch_bounds__(kPsThreads, 1) k_prefill_score(const __grid_constant__ PrefillArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + PfSmem::kBarOff);
  uint64_t *q_full = bars, *q_empty = bars + 2, *k_full = bars + 4, *k_empty = bars + 7;
  uint64_t *acc_full = bars + 10, *acc_empty = bars + 12;
  uint64_t *pair_bar = bars + 14;  // [4]: the two epilogue warps of one TMEM quadrant
  uint32_t *tmem_base_s = reinterpret_cast<uint32_t *>(bars + 18);
  int *abort_s = reinterpret_cast<int *>(bars + 19);
  float *lists = reinterpret_cast<float *>(smem + PfSmem::kListOff);
  float2 *thr_x = reinterpret_cast<float2 *>(smem + PfSmem::kThrOff);
  int *cnt_x = reinterpret_cast<int *>(smem + PfSmem::kCntOff);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = a.bh * (a.gist_tiles + a.raw_tiles);

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 8 * 32);
    }
    for (int i = 0; i < PfSmem::kKStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < 4; ++i) mbar_init(&pair_bar[i], 64);
    *abort_s = 0;
    mbar_fence_init();
    tc::prefetch_map(&a.tm_qraw);
    tc::prefetch_map(&a.tm_qgist);
    tc::prefetch_map(&a.tm_kgist);
  }
  for (int i = threadIdx.x; i < 2 * kPfRows; i += blockDim.x) thr_x[i] = make_float2(neg_inf(), __int_as_float(-1));
  if (warp == 1) tc::tmem_alloc(tmem_base_s, 256);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_base_s;
  pdl_wait();

  auto wait = [&](uint64_t *bar, uint32_t parity) -> bool {
    if (*reinterpret_cast<volatile int *>(abort_s)) return false;
    if (mbar_wait(bar, parity)) return true;
    *reinterpret_cast<volatile int *>(abort_s) = 1;
    flag_error(a.status, GSA_DEVERR_TIMEOUT);
    return false;
  };

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      uint32_t qi = 0, ki = 0;
      for (int t = blockIdx.x; t < total; t += gridDim.x) {
        const PfTile tl = pf_tile(a, t);
        if (tl.n_kt == 0) continue;
        const int qs = qi & 1;
        if (!wait(&q_empty[qs], ((qi >> 1) & 1) ^ 1)) break;
        uint8_t *qdst = smem + PfSmem::kQOff + qs * PfSmem::kQBytes;
        const CUtensorMap *qm = tl.is_gist ? &a.tm_qgist : &a.tm_qraw;
        const int qrow = tl.bh * (tl.is_gist ? a.n_chunks : a.L) + tl.row0;
        mbar_arrive_expect_tx(&q_full[qs], PfSmem::kQBytes);
        tc::tma_load_2d(qdst, qm, 0, qrow, &q_full[qs]);
        tc::tma_load_2d(qdst + PfSmem::kQBlock, qm, 64, qrow, &q_full[qs]);
        const int krow0 = (tl.bh / a.group) * a.n_chunks;
        bool ok = true;
        for (int j = 0; j < tl.n_kt; ++j, ++ki) {
          const int ks = ki % PfSmem::kKStages;
          if (!wait(&k_empty[ks], ((ki / PfSmem::kKStages) & 1) ^ 1)) {
            ok = false;
            break;
          }
          uint8_t *kdst = smem + PfSmem::kKOff + ks * PfSmem::kKBytes;
          mbar_arrive_expect_tx(&k_full[ks], PfSmem::kKBytes);
          tc::tma_load_2d(kdst, &a.tm_kgist, 0, krow0 + j * kPfKeys, &k_full[ks]);
          tc::tma_load_2d(kdst + PfSmem::kKBlock, &a.tm_kgist, 64, krow0 + j * kPfKeys, &k_full[ks]);
        }
        if (!ok) break;
        ++qi;
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_bf16(kPfRows, kPfKeys, false, false);
      uint32_t qi = 0, ki = 0, ai = 0;
      const uint32_t sbase = smem_u32(smem);
      for (int t = blockIdx.x; t < total; t += gridDim.x) {
        const PfTile tl = pf_tile(a, t);
        if (tl.n_kt == 0) continue;
        const int qs = qi & 1;
        if (!wait(&q_full[qs], (qi >> 1) & 1)) break;
        bool ok = true;
        for (int j = 0; j < tl.n_kt; ++j, ++ki, ++ai) {
          const int ks = ki % PfSmem::kKStages, as = ai & 1;
          if (!wait(&k_full[ks], (ki / PfSmem::kKStages) & 1) || !wait(&acc_empty[as], ((ai >> 1) & 1) ^ 1)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t qa = sbase + PfSmem::kQOff + qs * PfSmem::kQBytes;
          const uint32_t ka = sbase + PfSmem::kKOff + ks * PfSmem::kKBytes;
#pragma unroll
          for (int k = 0; k < 8; ++k) {  // d = 128 = 8 x 16
            const uint64_t ad = tc::sw128_desc(qa + (k >> 2) * PfSmem::kQBlock + (k & 3) * 32, 16);
            const uint64_t bd = tc::sw128_desc(ka + (k >> 2) * PfSmem::kKBlock + (k & 3) * 32, 16);
            tc::mma_bf16(tmem + as * kPfKeys, ad, bd, idesc, k > 0);
          }
          tc::commit(&k_empty[ks]);
          tc::commit(&acc_full[as]);
        }
        if (!ok) break;
        tc::commit(&q_empty[qs]);
        ++qi;
      }
    }
  } else {
    // ---------------- epilogue: two threads per query row ----------------
    // Warp w reads TMEM lane quadrant w % 4; half h = (w - 2) / 4 takes
    // columns [64h, 64h + 64) of every key tile, in ascending order.  Each
    // half keeps the K largest scores it has appended (values only, sorted
    // descending); its K-th is a lower bound on the row's final k-th score,
    // and so is the partner half's, published once per key tile.  A score is
    // appended as a (score, index) candidate only when it beats that bound,
    // so after the first key tile few scores are appended at all; appends
    // are predicated stores, never branches.  Equal scores: a score equal
    // to the own bound is not appended (K earlier, lower-index scores of
    // this half already rank ahead of it); one equal to the partner's is.
    const int quad = warp & 3, half = (warp - 2) >> 2;
    const int r = quad * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t base = smem_u32(smem + PfSmem::kCandOff) + (half * kPsCap * kPfRows + r) * 8u;
    const uint32_t base1 = smem_u32(smem + PfSmem::kCandOff) + (kPsCap * kPfRows + r) * 8u;
    const uint32_t room = base + (kPsCap - 8) * kPsSlot;  // a cursor beyond this leaves < 8 free slots
    const float nan = __int_as_float(0x7fffffff);
    uint32_t ai = 0, pair_phase = 0;
    auto pair_sync = [&]() -> bool {
      mbar_arrive(&pair_bar[quad]);
      const bool okp = wait(&pair_bar[quad], pair_phase);
      pair_phase ^= 1;
      return okp;
    };
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      const PfTile tl = pf_tile(a, t);
      const int row = tl.row0 + r;
      const bool row_ok = row < (tl.is_gist ? a.n_chunks : a.L);
      const int limit = !row_ok ? 0 : (tl.is_gist ? min(a.n_chunks, row + 1) : min(a.n_chunks, row / a.chunk));
      const bool want_topk = !tl.is_gist && a.topk > 0;
      float bst[K];
#pragma unroll
      for (int q = 0; q < K; ++q) bst[q] = neg_inf();
      float mx = neg_inf(), thr = neg_inf(), tp = neg_inf();
      uint32_t cur = base, c0 = base;  // column cursor; entries [c0, cur) not yet in bst
      // fold the candidates appended since the last call into bst (whole
      // warp; -inf pads the lanes with fewer, and inserting -inf changes
      // nothing)
      auto absorb = [&]() {
        const int n = static_cast<int>((cur - c0) / kPsSlot);
        const int nmax = __reduce_max_sync(0xffffffffu, n);
        const uint32_t last = base + (kPsCap - 1) * kPsSlot;
        for (int s = 0; s < nmax; s += 4) {
          float x[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float y = __uint_as_float(lds_u2(min(c0 + (s + u) * kPsSlot, last)).x);
            x[u] = s + u < n ? y : neg_inf();
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) pf_insert<K>(bst, x[u]);
        }
        c0 = cur;
      };
      bool ok = true;
      for (int j = 0; j < tl.n_kt; ++j, ++ai) {
        const int as = ai & 1;
        if (!__all_sync(0xffffffffu, wait(&acc_full[as], (ai >> 1) & 1))) {  // warp-uniform outcome
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const bool edge = __any_sync(0xffffffffu, (j + 1) * kPfKeys > limit);  // some row ends in this tile
#pragma unroll 1
        for (int b = 0; b < 2; ++b) {
          const int tb = j * kPfKeys + half * 64 + b * 32;
          float v[32];
          __syncwarp();  // tcgen05.ld is warp-collective
          tc::ld32(lane_addr + as * kPfKeys + half * 64 + b * 32, v);
          if (edge)
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = tb + e < limit ? v[e] : nan;  // masked: fails every compare
          if (!want_topk) {
#pragma unroll
            for (int e = 0; e < 32; ++e) mx = fmaxf(mx, v[e]);
            continue;
          }
          if (j == 0 && b == 0) {
            // first block: its K largest seed the list; append those >= the K-th
            float w[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) w[e] = v[e] == v[e] ? v[e] : neg_inf();
            pf_sort32(w);
#pragma unroll
            for (int q = 0; q < K; ++q) bst[q] = w[q];
#pragma unroll
            for (int e = 0; e < 32; ++e) pf_append<true>(cur, v[e], bst[K - 1], static_cast<uint32_t>(tb + e));
            c0 = cur;
            thr = bst[K - 1];
            continue;
          }
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            if (__any_sync(0xffffffffu, cur > room)) {
              // some lane has fewer than 8 free slots: every lane drops
              // what can no longer be selected (one pass for the warp)
              absorb();
              cur = pf_filter(base, cur, fmaxf(bst[K - 1], tp));
              if (cur > room) cur = pf_reduce<K>(base, cur);  // only under many equal scores
              c0 = cur;
              thr = fmaxf(bst[K - 1], pf_below(tp));
            }
#pragma unroll
            for (int e = 8 * g; e < 8 * g + 8; ++e) pf_append<false>(cur, v[e], thr, static_cast<uint32_t>(tb + e));
          }
        }
        tc::fence_before_sync();
        mbar_arrive(&acc_empty[as]);
        if (want_topk) {  // update the list, publish this half's bound, take the partner's
          absorb();
          thr_x[half * kPfRows + r] = make_float2(bst[K - 1], __int_as_float(t));
          const float2 p = thr_x[(half ^ 1) * kPfRows + r];
          if (__float_as_int(p.y) == t) tp = fmaxf(tp, p.x);
          thr = fmaxf(bst[K - 1], pf_below(tp));
        }
      }
      if (!ok) break;
      // Row end.  Both halves publish their lists; each computes the row's
      // k-th score T from both and keeps the candidates >= T of its own
      // column; half 0 merges the two (ascending index) and writes the row.
      float *mine = lists + half * (kPfTopkMax * kPfRows) + r;
      const float *theirs = lists + (half ^ 1) * (kPfTopkMax * kPfRows) + r;
      if (want_topk) {
#pragma unroll
        for (int q = 0; q < K; ++q) mine[q * kPfRows] = bst[q];
      } else {
        mine[0] = mx;
      }
      if (!pair_sync()) break;
      float T = neg_inf();
      int n_gt = 0;
      if (!want_topk) {
        mx = fmaxf(mx, theirs[0]);
      } else {
        // top K of both lists: elementwise max against the reversed partner
        // list is a bitonic sequence holding them; sort it descending
        float c[K];
#pragma unroll
        for (int q = 0; q < K; ++q) c[q] = fmaxf(bst[q], theirs[(K - 1 - q) * kPfRows]);
#pragma unroll
        for (int j2 = K >> 1; j2 > 0; j2 >>= 1)
#pragma unroll
          for (int i = 0; i < K; ++i)
            if ((i & j2) == 0) {
              const float x = c[i], y = c[i + j2];
              c[i] = fmaxf(x, y);
              c[i + j2] = fminf(x, y);
            }
        mx = c[0];
        T = c[0];
#pragma unroll
        for (int q = 0; q < K; ++q)
          if (q < a.topk) T = c[q];
#pragma unroll
        for (int q = 0; q < K; ++q) n_gt += (q < a.topk && c[q] > T) ? 1 : 0;
        cur = pf_filter(base, cur, T);
        cnt_x[half * kPfRows + r] = static_cast<int>((cur - base) / kPsSlot);
      }
      if (!pair_sync()) break;
      if (half == 0 && row_ok) {
        const size_t orow = static_cast<size_t>(tl.bh) * (tl.is_gist ? a.n_chunks : a.L) + row;
        float *rec = (tl.is_gist ? a.rec_gist : a.rec_raw) + orow * (128 + kPartHeader);
        if (want_topk) {
          // every score > T, then the lowest-index scores == T up to k
          int quota = a.topk - n_gt, n_out = 0;
          const uint32_t end1 = base1 + cnt_x[kPfRows + r] * kPsSlot;
          int32_t *oi = a.sel_idx + orow * a.topk;
          float *os = a.sel_score + orow * a.topk;
          uint32_t p0 = base, p1 = base1;
          while (p0 < cur || p1 < end1) {
            const uint2 e0 = p0 < cur ? lds_u2(p0) : make_uint2(0u, 0x7fffffffu);
            const uint2 e1 = p1 < end1 ? lds_u2(p1) : make_uint2(0u, 0x7fffffffu);
            const bool take0 = e0.y < e1.y;
            const uint2 e = take0 ? e0 : e1;
            p0 += take0 ? kPsSlot : 0u;
            p1 += take0 ? 0u : kPsSlot;
            const float x = __uint_as_float(e.x);
            const bool sel = x > T || (x == T && quota > 0);
            if (sel) {
              quota -= x > T ? 0 : 1;
              oi[n_out] = static_cast<int32_t>(e.y);
              os[n_out] = x * a.scale;
              ++n_out;
            }
          }
          for (int q = n_out; q < a.topk; ++q) {
            oi[q] = -1;
            os[q] = neg_inf();
          }
        }
        rec[0] = mx == neg_inf() ? mx : mx * a.scale_log2;
      }
      if (!pair_sync()) break;
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 256);
  }
}

// ---------------------------------------------------------------------------
// Stage 2a, k_prefill_gist_attn: softmax partial of every row over its
// visible gists, on the tensor cores.  The reference max of each row comes
// from stage 1, so the accumulator never needs rescaling:
//   S = Q K_g^T (TMEM), P = 2^(s*scale*log2e - max) masked (bf16, written
//   to shared memory in the swizzled K-major layout), O += P V_g (TMEM).
// Rows: gist-query rows always; raw rows in default mode (in exclude mode
// unselected gists are not attended and selected ones are added by stage
// 2b).  The P V product runs in fp16 (P in [0, 1] rounds to 2^-11; the
// bf16 gist values are exact in fp16 below 65504 in magnitude), and the sum
// of the rounded weights is the normaliser, so the partial is an exact
// convex combination of the values it weights.
constexpr int kGaKeys = 128;  // gist keys per tile (S is 128 x 128 in TMEM)

struct GaSmem {
  static constexpr uint32_t kBlock = 128 * 128;                 // 128 rows x 64 bf16
  static constexpr uint32_t kTile = 2 * kBlock;                 // 128 x 128 bf16
  static constexpr uint32_t kQOff = 0;
  static constexpr uint32_t kKOff = kTile;                      // 2 stages
  static constexpr uint32_t kVOff = kKOff + 2 * kTile;          // 2 stages
  static constexpr uint32_t kPOff = kVOff + 2 * kTile;          // 2 buffers
  static constexpr uint32_t kBarOff = kPOff + 2 * kTile;
  static constexpr uint32_t kBytes = kBarOff + 256 + 1024;
};

__device__ __forceinline__ PfTile ga_tile(const PrefillArgs &a, int t) {
  // Same order as stage 1; raw tiles are skipped in exclude mode.
  PfTile r = pf_tile(a, t);
  const int visible = r.is_gist ? min(a.n_chunks, r.row0 + kPfRows)
                                : min(a.n_chunks, min(a.L - 1, r.row0 + kPfRows - 1) / a.chunk);
  r.n_kt = (!r.is_gist && a.exclude) ? 0 : (visible + kGaKeys - 1) / kGaKeys;
  return r;
}

__global__ void __launch_bounds__(kPfThreads, 1) k_prefill_gist_attn(const __grid_constant__ PrefillArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + GaSmem::kBarOff);
  uint64_t *q_full = bars, *q_empty = bars + 1, *k_full = bars + 2, *k_empty = bars + 4;
  uint64_t *v_full = bars + 6, *v_empty = bars + 8, *s_full = bars + 10, *s_empty = bars + 12;
  uint64_t *p_full = bars + 14, *p_empty = bars + 16, *o_full = bars + 18, *o_empty = bars + 19;
  uint32_t *tmem_base_s = reinterpret_cast<uint32_t *>(bars + 20);
  int *abort_s = reinterpret_cast<int *>(bars + 21);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = a.bh * (a.gist_tiles + a.raw_tiles);
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(o_full, 1);
    mbar_init(o_empty, 4 * 32);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 4 * 32);
      mbar_init(&p_full[i], 4 * 32);
      mbar_init(&p_empty[i], 1);
    }
    *abort_s = 0;
    mbar_fence_init();
    tc::prefetch_map(&a.tm_qraw);
    tc::prefetch_map(&a.tm_qgist);
    tc::prefetch_map(&a.tm_kgist);
    tc::prefetch_map(&a.tm_vgist);
  }
  if (warp == 1) tc::tmem_alloc(tmem_base_s, 512);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_base_s;  // S buffers at columns 0 and 128, O at 256
  pdl_wait();

  auto wait = [&](uint64_t *bar, uint32_t parity) -> bool {
    if (*reinterpret_cast<volatile int *>(abort_s)) return false;
    if (mbar_wait(bar, parity)) return true;
    *reinterpret_cast<volatile int *>(abort_s) = 1;
    flag_error(a.status, GSA_DEVERR_TIMEOUT);
    return false;
  };

  if (warp == 0) {
    if (lane == 0) {
      uint32_t qi = 0, ki = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const PfTile tl = ga_tile(a, t);
        if (tl.n_kt == 0) continue;
        if (!wait(q_empty, (qi & 1) ^ 1)) break;
        uint8_t *qdst = smem + GaSmem::kQOff;
        const CUtensorMap *qm = tl.is_gist ? &a.tm_qgist : &a.tm_qraw;
        const int qrow = tl.bh * (tl.is_gist ? a.n_chunks : a.L) + tl.row0;
        mbar_arrive_expect_tx(q_full, GaSmem::kTile);
        tc::tma_load_2d(qdst, qm, 0, qrow, q_full);
        tc::tma_load_2d(qdst + GaSmem::kBlock, qm, 64, qrow, q_full);
        const int krow0 = (tl.bh / a.group) * a.n_chunks;
        for (int j = 0; j < tl.n_kt; ++j, ++ki) {
          const int s = ki & 1;
          const uint32_t par = ((ki >> 1) & 1) ^ 1;
          if (!wait(&k_empty[s], par) || !wait(&v_empty[s], par)) {
            ok = false;
            break;
          }
          uint8_t *kdst = smem + GaSmem::kKOff + s * GaSmem::kTile;
          uint8_t *vdst = smem + GaSmem::kVOff + s * GaSmem::kTile;
          mbar_arrive_expect_tx(&k_full[s], GaSmem::kTile);
          tc::tma_load_2d(kdst, &a.tm_kgist, 0, krow0 + j * kGaKeys, &k_full[s]);
          tc::tma_load_2d(kdst + GaSmem::kBlock, &a.tm_kgist, 64, krow0 + j * kGaKeys, &k_full[s]);
          mbar_arrive_expect_tx(&v_full[s], GaSmem::kTile);
          tc::tma_load_2d(vdst, &a.tm_vgist, 0, krow0 + j * kGaKeys, &v_full[s]);
          tc::tma_load_2d(vdst + GaSmem::kBlock, &a.tm_vgist, 64, krow0 + j * kGaKeys, &v_full[s]);
        }
        ++qi;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = tc::idesc_bf16(kPfRows, kGaKeys, false, false);
      constexpr uint32_t idesc_o = tc::idesc_f16kind(kPfRows, 128, false, true, false);  // fp16; B = V, MN-major
      const uint32_t sbase = smem_u32(smem);
      uint32_t qi = 0, ki = 0, si = 0, pi = 0, oi = 0;
      bool ok = true;
      // GEMM1 for key tile j into S buffer (si & 1)
      auto gemm1 = [&](int j) -> bool {
        const int s = ki & 1, sb = si & 1;
        if (!wait(&k_full[s], (ki >> 1) & 1) || !wait(&s_empty[sb], ((si >> 1) & 1) ^ 1)) return false;
        tc::fence_after_sync();
        const uint32_t qa = sbase + GaSmem::kQOff, ka = sbase + GaSmem::kKOff + s * GaSmem::kTile;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t ad = tc::sw128_desc(qa + (k >> 2) * GaSmem::kBlock + (k & 3) * 32, 16);
          const uint64_t bd = tc::sw128_desc(ka + (k >> 2) * GaSmem::kBlock + (k & 3) * 32, 16);
          tc::mma_bf16(tmem + sb * kGaKeys, ad, bd, idesc_s, k > 0);
        }
        tc::commit(&k_empty[s]);
        tc::commit(&s_full[sb]);
        ++ki;
        ++si;
        return true;
      };
      // GEMM2 for key tile j: O += P V
      auto gemm2 = [&](int j, uint32_t vi) -> bool {
        const int s = vi & 1, pb = pi & 1;
        if (!wait(&v_full[s], (vi >> 1) & 1) || !wait(&p_full[pb], (pi >> 1) & 1)) return false;
        tc::fence_after_sync();
        const uint32_t pa = sbase + GaSmem::kPOff + pb * GaSmem::kTile, va = sbase + GaSmem::kVOff + s * GaSmem::kTile;
#pragma unroll
        for (int k = 0; k < 8; ++k) {  // 128 keys = 8 x 16
          const uint64_t ad = tc::sw128_desc(pa + (k >> 2) * GaSmem::kBlock + (k & 3) * 32, 16);
          const uint64_t bd = tc::sw128_desc(va + k * 16 * 128, GaSmem::kBlock);
          tc::mma_bf16(tmem + 2 * kGaKeys, ad, bd, idesc_o, (j > 0 || k > 0) ? 1u : 0u);
        }
        tc::commit(&v_empty[s]);
        tc::commit(&p_empty[pb]);
        ++pi;
        return true;
      };
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const PfTile tl = ga_tile(a, t);
        if (tl.n_kt == 0) continue;
        if (!wait(q_full, qi & 1) || !wait(o_empty, (oi & 1) ^ 1)) break;
        const uint32_t v0 = ki;  // V tiles pair with K tiles
        ok = gemm1(0);
        for (int j = 0; j < tl.n_kt && ok; ++j) {
          if (j + 1 < tl.n_kt) ok = gemm1(j + 1);
          if (ok) ok = gemm2(j, v0 + j);
        }
        if (!ok) break;
        tc::commit(q_empty);
        tc::commit(o_full);
        ++qi;
        ++oi;
      }
    }
  } else {
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    uint32_t si = 0, pi = 0, oi = 0;
    const uint32_t prow = static_cast<uint32_t>(r);
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      const PfTile tl = ga_tile(a, t);
      if (tl.n_kt == 0) continue;
      const int row = tl.row0 + r;
      const bool row_ok = row < (tl.is_gist ? a.n_chunks : a.L);
      const int limit = !row_ok ? 0 : (tl.is_gist ? min(a.n_chunks, row + 1) : min(a.n_chunks, row / a.chunk));
      const size_t orow = static_cast<size_t>(tl.bh) * (tl.is_gist ? a.n_chunks : a.L) + (row_ok ? row : 0);
      float *rec = (tl.is_gist ? a.rec_gist : a.rec_raw) + orow * (128 + kPartHeader);
      const float ref = (row_ok && limit > 0) ? rec[0] : 0.f;
      float l = 0.f;
      bool ok = true;
      for (int j = 0; j < tl.n_kt; ++j) {
        const int sb = si & 1, pb = pi & 1;
        if (!wait(&s_full[sb], (si >> 1) & 1)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        uint32_t packed[64];
#pragma unroll
        for (int c = 0; c < kGaKeys / 32; ++c) {
          float v[32];
          __syncwarp();
          tc::ld32(tmem + lane_addr + sb * kGaKeys + c * 32, v);
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int tt = j * kGaKeys + c * 32 + e;
            const float p0 = tt < limit ? exp2_approx(v[e] * a.scale_log2 - ref) : 0.f;
            const float p1 = tt + 1 < limit ? exp2_approx(v[e + 1] * a.scale_log2 - ref) : 0.f;
            const __half2 ph2 = __floats2half2_rn(p0, p1);
            l += __low2float(ph2) + __high2float(ph2);
            packed[c * 16 + e / 2] = *reinterpret_cast<const uint32_t *>(&ph2);
          }
        }
        tc::fence_before_sync();
        mbar_arrive(&s_empty[sb]);
        ++si;
        if (!wait(&p_empty[pb], ((pi >> 1) & 1) ^ 1)) {
          ok = false;
          break;
        }
        // P row r into the swizzled K-major tile: block kb holds keys 64*kb..
        uint8_t *pbase = smem + GaSmem::kPOff + pb * GaSmem::kTile;
#pragma unroll
        for (int u = 0; u < 16; ++u) {  // 16-byte units along the 128 keys
          const int kb = u >> 3, uu = u & 7;
          uint8_t *dst = pbase + kb * GaSmem::kBlock + (prow >> 3) * 1024 + (prow & 7) * 128 + ((uu ^ (prow & 7)) * 16);
          *reinterpret_cast<uint4 *>(dst) =
              make_uint4(packed[4 * u], packed[4 * u + 1], packed[4 * u + 2], packed[4 * u + 3]);
        }
        tc::fence_proxy_async_smem();
        mbar_arrive(&p_full[pb]);
        ++pi;
      }
      if (!ok) break;
      if (!wait(o_full, oi & 1)) break;
      tc::fence_after_sync();
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float v[32];
        __syncwarp();
        tc::ld32(tmem + lane_addr + 2 * kGaKeys + c * 32, v);
        if (row_ok)
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4 *>(rec + kPartHeader + c * 32 + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
      }
      tc::fence_before_sync();
      mbar_arrive(o_empty);
      ++oi;
      if (row_ok) {
        rec[1] = l;
        if (limit == 0) rec[0] = neg_inf();
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// Stage 2b, k_prefill_gather: per query row, the raw tokens the tensor-core
// stages do not cover -- the selected chunks (with their gist in exclude
// mode) and the own-chunk prefix for raw rows, chunk m's raw tokens for gist
// row m -- merged with the row's gist partial.  One warp per row; a group of
// 16 lanes owns one key row (8 dims per lane), two rows per step.
struct GatherArgs {
  const __nv_bfloat16 *q_raw, *k_raw, *v_raw, *q_gist, *v_gist;
  const int32_t *sel_idx;
  const float *sel_score;
  const float *rec_raw, *rec_gist;
  int32_t bh, hq, group, chunk, n_chunks, L, topk, exclude;
  float scale_log2;
  void *out_raw, *out_gist;
  int32_t out_bf16;
};

constexpr int kGatherWarps = 8;

__global__ void __launch_bounds__(kGatherWarps * 32) k_prefill_gather(const GatherArgs a) {
  constexpr int D = 128, kE = 8, kLpr = 16;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t rows_raw = static_cast<int64_t>(a.bh) * a.L;
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * kGatherWarps + warp;
  const int64_t rows_total = rows_raw + static_cast<int64_t>(a.bh) * a.n_chunks;
  pdl_wait();
  if (gw >= rows_total) return;
  const bool is_gist = gw >= rows_raw;
  const int64_t ridx = is_gist ? gw - rows_raw : gw;
  const int bh = static_cast<int>(is_gist ? ridx / a.n_chunks : ridx / a.L);
  const int pos = static_cast<int>(is_gist ? ridx % a.n_chunks : ridx % a.L);
  const int kvh = bh / a.group;
  const int slot = lane / kLpr, dd = kE * (lane % kLpr);
  const size_t kv0 = static_cast<size_t>(kvh) * a.L;  // raw rows of this kv head
  const __nv_bfloat16 *qrow = is_gist ? a.q_gist + (static_cast<size_t>(bh) * a.n_chunks + pos) * D
                                      : a.q_raw + (static_cast<size_t>(bh) * a.L + pos) * D;
  float qf[kE];
  Vec16<__nv_bfloat16>::unpack(ldg_nc_v4(qrow + dd), qf);
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
  // attend raw rows [first, first + n) of this kv head, 4 rows per lane group in flight
  auto span = [&](int first, int n) {
    for (int r0 = 0; r0 < n; r0 += 8) {
      uint4 kw[4], vw[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int r = r0 + 2 * u + slot;
        const size_t off = (kv0 + first + min(r, n - 1)) * D + dd;
        kw[u] = ldg_nc_v4(a.k_raw + off);
        vw[u] = ldg_nc_v4(a.v_raw + off);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int r = r0 + 2 * u + slot;
        float kf[kE], part = 0.f;
        Vec16<__nv_bfloat16>::unpack(kw[u], kf);
#pragma unroll
        for (int e = 0; e < kE; ++e) part = fmaf(qf[e], kf[e], part);
#pragma unroll
        for (int o = 1; o < kLpr; o <<= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if (r < n) {
          float vf[kE];
          Vec16<__nv_bfloat16>::unpack(vw[u], vf);
          update(part * a.scale_log2, vf);
        }
      }
    }
  };
  if (is_gist) {
    span(pos * a.chunk, a.chunk);
  } else {
    const int mc = pos / a.chunk;
    const int32_t *sel = a.sel_idx + ridx * a.topk;
    for (int e = 0; e < a.topk; ++e) {
      const int t = sel[e];
      if (t < 0 || t >= mc) continue;
      span(t * a.chunk, a.chunk);
      if (a.exclude && slot == 0) {
        float vf[kE];
        Vec16<__nv_bfloat16>::unpack(ldg_nc_v4(a.v_gist + (static_cast<size_t>(kvh) * a.n_chunks + t) * D + dd), vf);
        update(a.sel_score[ridx * a.topk + e] * kLog2e, vf);
      }
    }
    span(mc * a.chunk, pos - mc * a.chunk + 1);
  }
  // merge the two row slots, then the gist partial of the row
  {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, kLpr), l2 = __shfl_xor_sync(0xffffffffu, l, kLpr);
    float acc2[kE];
#pragma unroll
    for (int e = 0; e < kE; ++e) acc2[e] = __shfl_xor_sync(0xffffffffu, acc[e], kLpr);
    merge_state<kE>(m, l, acc, m2, l2, acc2);
  }
  const bool has_prior = is_gist || !a.exclude;
  if (has_prior) {
    const float *rec = (is_gist ? a.rec_gist : a.rec_raw) + ridx * (D + kPartHeader);
    const float pm = rec[0], pl = rec[1];
    if (pm != neg_inf() && pl > 0.f) {
      float pacc[kE];
      const float4 x = *reinterpret_cast<const float4 *>(rec + kPartHeader + dd);
      const float4 y = *reinterpret_cast<const float4 *>(rec + kPartHeader + dd + 4);
      pacc[0] = x.x; pacc[1] = x.y; pacc[2] = x.z; pacc[3] = x.w;
      pacc[4] = y.x; pacc[5] = y.y; pacc[6] = y.z; pacc[7] = y.w;
      merge_state<kE>(m, l, acc, pm, pl, pacc);
    }
  }
  if (lane < kLpr) {
    void *out = is_gist ? a.out_gist : a.out_raw;
    const size_t base = static_cast<size_t>(ridx) * D + dd;
#pragma unroll
    for (int e = 0; e < kE; ++e) store_out(out, base + e, l > 0.f ? acc[e] / l : 0.f, a.out_bf16);
  }
}


// bf16 -> fp16 copy of the gist values for the fp16 P V product (exact for
// magnitudes below 65504; larger values saturate to +-inf).
__global__ void k_bf16_to_f16(const __nv_bfloat16 *__restrict__ src, __half *__restrict__ dst, size_t n8) {
  pdl_wait();
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const uint4 w = ldg_nc_v4(src + 8 * i);
    float f[8];
    Vec16<__nv_bfloat16>::unpack(w, f);
    __half2 h[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) h[e] = __floats2half2_rn(f[2 * e], f[2 * e + 1]);
    *reinterpret_cast<uint4 *>(dst + 8 * i) = *reinterpret_cast<const uint4 *>(h);
  }
}

}  // namespace gsa
