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
// then 128-gist key tiles into a 3-stage ring, 2 stages for the wide
// scorer at d = 128), warp 1 issues tcgen05.mma into three 128-column TMEM
// accumulators, and warps 2..9 (two per TMEM lane
// quadrant, so two threads per query row, each owning a 64-column half of
// every key tile) read the scores with tcgen05.ld and apply the
// block-causal mask.  Raw rows take the key tiles twice: a first pass of
// slot maxima gives the row maximum and a lower bound on its k-th score,
// a second pass appends the few scores above the bound to shared-memory
// candidate columns, from which the exact selection is read off.
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
  int32_t pos0;          // causal position of raw row 0 (0 in prefill; multi-query rows sit after the cache)
  float scale, scale_log2;
  int32_t *sel_idx;      // [B*hq*L, topk]
  float *sel_score;      // [B*hq*L, topk]
  float *rec_raw;        // [B*hq*L, d+4] partial records; [0] = row max (base 2)
  float *rec_gist;       // [B*hq*N, d+4]
  int32_t gist_tiles;    // query tiles per head over the gist rows
  int32_t raw_tiles;     // query tiles per head over the raw rows
  uint32_t *status;
  int32_t *ovf_rows;     // rows whose candidates overflowed (exact pass in k_prefill_select_rows)
  uint32_t *ovf_count;
};

constexpr int kPfRows = 128;        // query rows per tile (TMEM lanes)
constexpr int kPfKeys = 128;        // gist keys per MMA tile (TMEM columns)
constexpr int kPfThreads = 192;     // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr int kPfTopkMax = 16;   // the narrow scorer: k <= 16
constexpr int kPfTopkWide = 64;  // the wide scorer: 16 < k <= 64

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
    const int visible = min(a.n_chunks, (a.pos0 + last) / a.chunk);  // raw i sees 0..i/c-1
    r.n_kt = (visible + kPfKeys - 1) / kPfKeys;
  }
  return r;
}

// Scoring-stage layout: warp 0 TMA, warp 1 MMA, warps 2..9 epilogue; warp
// w reads TMEM lane quadrant w % 4 and owns half h = (w - 2) / 4 of every
// key tile (columns 32h .. 32h+31 and 64+32h .. 95+32h, so short rows still
// spread over both halves); two threads share a query row.
constexpr int kPsEpiWarps = 8;
constexpr int kPsThreads = 64 + 32 * kPsEpiWarps;
// TMEM columns: kPsAcc accumulators of 128 (the MMA runs that many key
// tiles ahead of the epilogue), then the row-end exchange (2 x the sorted
// list length: 16 for the narrow scorer, 64 for the wide one)
constexpr int kPsAcc = 3;
constexpr int kPsXchgCol = kPsAcc * kPfKeys;
static_assert(kPsXchgCol + 2 * 64 <= 512, "TMEM columns");

// Scoring-stage shared memory.  D = 64 or 128: a row is D/64 boxes of 64
// bf16 (128 bytes, swizzled).  K = the largest k the variant selects: the
// narrow scorer (K = 16) keeps 48 candidate slots per row half, the wide
// one (K = 64) 64, and with d = 128 it gives up a key stage to fit them.
template <int D, int K>
struct PfSmem {
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(K == kPfTopkMax || K == kPfTopkWide, "scorer variant");
  static constexpr int kCap = K > 16 ? 64 : 48;  // candidate slots per row half
  static constexpr uint32_t kQBlock = kPfRows * 128;         // 128 rows x 64 bf16
  static constexpr uint32_t kQBytes = (D / 64) * kQBlock;
  static constexpr uint32_t kKBlock = kPfKeys * 128;
  static constexpr uint32_t kKBytes = (D / 64) * kKBlock;
  static constexpr int kQStages = 1;  // the next tile's Q lands during the row end
  static constexpr int kKStages = (K > 16 && D == 128) ? 2 : 3;
  static constexpr uint32_t kQOff = 0;
  static constexpr uint32_t kKOff = kQStages * kQBytes;
  // [2 halves][kCap][128 rows] (score, index); pass A first uses a row
  // half's first slots for its sorted slot maxima (two per slot)
  static constexpr uint32_t kCandOff = kKOff + kKStages * kKBytes;
  static constexpr uint32_t kCntOff = kCandOff + 2 * kCap * kPfRows * 8;  // [2][128] candidate counts (bytes)
  static constexpr uint32_t kSelOff = kCntOff + 2 * kPfRows;               // [2][128] selected counts (bytes)
  static constexpr uint32_t kBarOff = kSelOff + 2 * kPfRows;
  static constexpr uint32_t kBytes = kBarOff + 256 + 1008;   // + alignment slack (base is 16-byte aligned)
  static_assert(kBytes <= 232448, "prefill scoring shared memory");
  static_assert(2 * kCap >= (K > 16 ? 64 : 16), "a column holds the half's sorted slot maxima");
  static_assert(kCap <= 255, "counts are bytes");
};

constexpr uint32_t kPsSlot = kPfRows * 8;  // bytes between consecutive slots of one row's column

__device__ __forceinline__ uint2 lds_u2(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a) : "memory");
  return v;
}

__device__ __forceinline__ void sts_u2(uint32_t a, uint2 v) {
  asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(a), "r"(v.x), "r"(v.y) : "memory");
}

// Append (v, idx) to a row half's column when v >= bound, at the slot
// address `ad`, which then moves on by one slot (the count is (ad - base) /
// kPsSlot).  The store and the step are predicated (no branch).  Past the
// last slot the store lands in the last one while the address keeps
// counting, which the row end reports as an overflow.  NaN (a masked
// score) fails the compare.
__device__ __forceinline__ void ps_append(uint32_t &ad, uint32_t last, float v, float bound, uint32_t idx) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .u32 a2;\n\t"
      "setp.ge.f32 p, %1, %2;\n\t"
      "min.u32 a2, %0, %6;\n\t"
      "@p st.shared.v2.u32 [a2], {%3, %4};\n\t"
      "@p add.u32 %0, %0, %5;\n\t}\n"
      : "+r"(ad)
      : "f"(v), "f"(bound), "r"(__float_as_uint(v)), "r"(idx), "n"(kPsSlot), "r"(last)
      : "memory");
}

__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
  return v;
}

// Descending bitonic sort of N (a power of two) values in registers (no
// NaN inputs).
template <int N>
__device__ __forceinline__ void ps_sort(float (&w)[N]) {
#pragma unroll
  for (int k = 2; k <= N; k <<= 1)
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1)
#pragma unroll
      for (int i = 0; i < N; ++i) {
        const int l = i ^ j;
        if (l > i) {
          const float x = w[i], y = w[l];
          const bool desc = (i & k) == 0;
          w[i] = desc ? fmaxf(x, y) : fminf(x, y);
          w[l] = desc ? fminf(x, y) : fmaxf(x, y);
        }
      }
}

// a <- the N largest of a (sorted descending) and b (sorted descending):
// the elementwise max against b reversed is bitonic; half-cleaners sort it.
template <int N>
__device__ __forceinline__ void ps_merge(float (&a)[N], const float (&b)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) a[i] = fmaxf(a[i], b[N - 1 - i]);
#pragma unroll
  for (int j = N / 2; j > 0; j >>= 1)
#pragma unroll
    for (int i = 0; i < N; ++i)
      if ((i & j) == 0) {
        const float x = a[i], y = a[i + j];
        a[i] = fmaxf(x, y);
        a[i + j] = fminf(x, y);
      }
}

// Stage 1, k_prefill_score: row maxima and the top-k selection of every
// query row, in two passes over the visible key tiles of a query tile (the
// key tiles stream through a ring; Q stays in shared memory).  K = 16 (the
// narrow scorer, k <= 16) or 64 (the wide one, 16 < k <= 64); S = 16 or 64
// slots per row half:
//  A. each thread keeps S slot maxima over its half of the columns (slot =
//     column mod S); the largest of the row's 2S slot maxima are distinct
//     scores, so the k-th largest of them bounds the row's k-th score from
//     below.  The narrow scorer samples every other key tile (0, 2, 4, ...;
//     the bound stays valid, only looser, and the pass's tensor work
//     halves); the wide one takes every tile, which keeps the bound tight
//     at k = 64;
//  B. over all key tiles, every score >= that bound is appended as a
//     (score, index) candidate (about 2k + 10 per row for the narrow
//     scorer, 1.4k for the wide one) by predicated stores, in ascending
//     index order; the largest candidate is the row maximum;
//     at the row end each half sorts its S largest candidate values, the
//     halves exchange them through TMEM and merge them into the row's k-th
//     candidate score T, keep (compact) their entries >= T, and write the
//     two ascending lists merged by index, K/2 output slots per half.
// A row whose candidates overflow a half's slots, or whose k-th score is
// shared by a (k+1)-th (the index rule then decides), is listed for
// k_prefill_select_rows, which recomputes it exactly.
template <int K, int D>
__global__ void __launch_bounds__(kPsThreads, 1) k_prefill_score(const __grid_constant__ PrefillArgs a) {
  using Sm = PfSmem<D, K>;
  constexpr bool kWide = K > 16;
  constexpr int kSl = kWide ? 64 : 16;  // slot maxima (and sorted candidate values) per row half
  constexpr int kCap = Sm::kCap;
  constexpr int kHalfOut = K / 2;       // output slots written by each half
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Sm::kBarOff);
  constexpr int kQS = Sm::kQStages, kKS = Sm::kKStages;
  uint64_t *q_full = bars, *q_empty = bars + kQS, *k_full = bars + 2 * kQS, *k_empty = k_full + kKS;
  uint64_t *acc_full = k_empty + kKS, *acc_empty = acc_full + kPsAcc;
  uint64_t *quad_bar = acc_empty + kPsAcc;  // [4]: the two epilogue warps of one TMEM quadrant
  static_assert(2 * kQS + 2 * kKS + 2 * kPsAcc + 4 <= 24, "barrier block");
  uint32_t *tmem_base_s = reinterpret_cast<uint32_t *>(bars + 24);
  int *abort_s = reinterpret_cast<int *>(bars + 25);
  uint8_t *cnt_x = smem + Sm::kCntOff;                               // [2][128]
  uint8_t *sel_x = smem + Sm::kSelOff;                               // [2][128]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = a.bh * (a.gist_tiles + a.raw_tiles);
  const bool raw_topk = a.topk > 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kQS; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    for (int i = 0; i < kPsAcc; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], kPsEpiWarps * 32);
    }
    for (int i = 0; i < kKS; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < 4; ++i) mbar_init(&quad_bar[i], 2 * 32);
    *abort_s = 0;
    mbar_fence_init();
    tc::prefetch_map(&a.tm_qraw);
    tc::prefetch_map(&a.tm_qgist);
    tc::prefetch_map(&a.tm_kgist);
  }
  if (warp == 1) tc::tmem_alloc(tmem_base_s, 512);  // accumulators + the row-end exchange
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
  // Key tiles of a query tile, in MMA order.  Rows with a selection take
  // pass A (the narrow scorer: over every other key tile, 0, 2, 4, ...; the
  // bound it gives stays exact, only looser) and then pass B over all of
  // them; other rows take pass A over all key tiles (their exact row
  // maximum).
  auto n_pass_a = [&](const PfTile &tl) {
    return (!tl.is_gist && raw_topk && !kWide) ? (tl.n_kt + 1) / 2 : tl.n_kt;
  };
  auto n_steps = [&](const PfTile &tl) { return n_pass_a(tl) + ((!tl.is_gist && raw_topk) ? tl.n_kt : 0); };
  auto step_tile = [&](const PfTile &tl, int jj) {
    const bool sampled = !tl.is_gist && raw_topk && !kWide;
    const int na = n_pass_a(tl);
    return jj < na ? (sampled ? 2 * jj : jj) : jj - na;
  };

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      uint32_t qi = 0, ki = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const PfTile tl = pf_tile(a, t);
        if (tl.n_kt == 0) continue;
        const int qs = qi % kQS;
        if (!wait(&q_empty[qs], ((qi / kQS) & 1) ^ 1)) break;
        uint8_t *qdst = smem + Sm::kQOff + qs * Sm::kQBytes;
        const CUtensorMap *qm = tl.is_gist ? &a.tm_qgist : &a.tm_qraw;
        const int qrow = tl.bh * (tl.is_gist ? a.n_chunks : a.L) + tl.row0;
        mbar_arrive_expect_tx(&q_full[qs], Sm::kQBytes);
#pragma unroll
        for (int x = 0; x < D / 64; ++x) tc::tma_load_2d(qdst + x * Sm::kQBlock, qm, 64 * x, qrow, &q_full[qs]);
        const int krow0 = (tl.bh / a.group) * a.n_chunks;
        for (int jj = 0; jj < n_steps(tl); ++jj, ++ki) {
          const int j = step_tile(tl, jj), ks = ki % kKS;
          if (!wait(&k_empty[ks], ((ki / kKS) & 1) ^ 1)) {
            ok = false;
            break;
          }
          uint8_t *kdst = smem + Sm::kKOff + ks * Sm::kKBytes;
          mbar_arrive_expect_tx(&k_full[ks], Sm::kKBytes);
#pragma unroll
          for (int x = 0; x < D / 64; ++x)
            tc::tma_load_2d(kdst + x * Sm::kKBlock, &a.tm_kgist, 64 * x, krow0 + j * kPfKeys, &k_full[ks]);
        }
        ++qi;
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_bf16(kPfRows, kPfKeys, false, false);
      uint32_t qi = 0, ki = 0, ai = 0;
      const uint32_t sbase = smem_u32(smem);
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const PfTile tl = pf_tile(a, t);
        if (tl.n_kt == 0) continue;
        const int qs = qi % kQS;
        if (!wait(&q_full[qs], (qi / kQS) & 1)) break;
        for (int jj = 0; jj < n_steps(tl); ++jj, ++ki, ++ai) {
          const int ks = ki % kKS, as = ai % kPsAcc;
          if (!wait(&k_full[ks], (ki / kKS) & 1) || !wait(&acc_empty[as], ((ai / kPsAcc) & 1) ^ 1)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t qa = sbase + Sm::kQOff + qs * Sm::kQBytes;
          const uint32_t ka = sbase + Sm::kKOff + ks * Sm::kKBytes;
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {  // 16 dims per MMA
            const uint64_t ad = tc::sw128_desc(qa + (k >> 2) * Sm::kQBlock + (k & 3) * 32, 16);
            const uint64_t bd = tc::sw128_desc(ka + (k >> 2) * Sm::kKBlock + (k & 3) * 32, 16);
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
    const int quad = warp & 3, h = (warp - 2) >> 2;
    const int r = quad * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t cand_u = smem_u32(smem + Sm::kCandOff);
    const uint32_t base = cand_u + (h * kCap * kPfRows + r) * 8u;          // slot s at base + s * kPsSlot
    const uint32_t pbase = cand_u + ((h ^ 1) * kCap * kPfRows + r) * 8u;  // the partner half's column
    const float nan = __int_as_float(0x7fffffff);
    uint32_t ai = 0, pair_phase = 0;
    auto pair_sync = [&]() -> bool {
      mbar_arrive(&quad_bar[quad]);
      const bool okq = wait(&quad_bar[quad], pair_phase);
      pair_phase ^= 1;
      return okq;
    };
    // one accumulator: this thread's 64 scores (columns 32h .. 32h+31 and
    // 64+32h .. 95+32h of the key tile), masked past `limit`, handed to f
    auto take = [&](int j, int limit, auto &&f) -> bool {
      const int as = ai % kPsAcc;
      if (!__all_sync(0xffffffffu, wait(&acc_full[as], (ai / kPsAcc) & 1))) return false;
      tc::fence_after_sync();
      const bool edge = __any_sync(0xffffffffu, (j + 1) * kPfKeys > limit);
      float v[64];
      __syncwarp();  // tcgen05.ld is warp-collective
      tc::ld32x2(lane_addr + as * kPfKeys + 32 * h, lane_addr + as * kPfKeys + 64 + 32 * h, v);
      const int tb = j * kPfKeys + 32 * h;  // v[e] is column tb + e (e < 32) or tb + 32 + e (e >= 32)
      if (edge)
#pragma unroll
        for (int e = 0; e < 64; ++e) v[e] = tb + e + (e >> 5) * 32 < limit ? v[e] : nan;  // masked: fails every compare
      f(v, tb);
      tc::fence_before_sync();
      mbar_arrive(&acc_empty[as]);
      ++ai;
      return true;
    };
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      const PfTile tl = pf_tile(a, t);  // (no key tile: every row sees nothing; still written)
      const int row = tl.row0 + r;
      const bool row_ok = row < (tl.is_gist ? a.n_chunks : a.L);
      const int limit =
          !row_ok ? 0 : (tl.is_gist ? min(a.n_chunks, row + 1) : min(a.n_chunks, (a.pos0 + row) / a.chunk));
      const bool sel_rows = !tl.is_gist && raw_topk;
      const int ksel = min(a.topk, limit);  // entries this row selects
      // ---- pass A: slot maxima ----
      float G[kSl];
#pragma unroll
      for (int q = 0; q < kSl; ++q) G[q] = neg_inf();
      for (int jj = 0; jj < n_pass_a(tl) && ok; ++jj)
        ok = take(step_tile(tl, jj), limit, [&](const float(&v)[64], int) {
#pragma unroll
          for (int e = 0; e < 64; ++e) G[e & (kSl - 1)] = fmaxf(G[e & (kSl - 1)], v[e]);
        });
      if (!ok) break;
      ps_sort<kSl>(G);
      // the sorted slot maxima go to this row half's own candidate column
      // (two per slot); rows of other quadrants, which run ahead or behind,
      // never touch them
#pragma unroll
      for (int q = 0; q < kSl; q += 2)
        sts_u2(base + (q >> 1) * kPsSlot, make_uint2(__float_as_uint(G[q]), __float_as_uint(G[q + 1])));
      if (!pair_sync()) break;
      {
        float o[kSl];
#pragma unroll
        for (int q = 0; q < kSl; q += 2) {
          const uint2 w = lds_u2(pbase + (q >> 1) * kPsSlot);
          o[q] = __uint_as_float(w.x);
          o[q + 1] = __uint_as_float(w.y);
        }
        ps_merge<kSl>(G, o);  // top kSl of the row's 2 kSl slot maxima
      }
      const float mx = G[0];
      float bound = G[0];
#pragma unroll
      for (int q = 1; q < kSl; ++q)
        if (q < ksel) bound = G[q];
      if (!pair_sync()) break;  // the slot maxima area becomes the candidate columns
      const size_t orow = static_cast<size_t>(tl.bh) * (tl.is_gist ? a.n_chunks : a.L) + row;
      float *rec = (tl.is_gist ? a.rec_gist : a.rec_raw) + orow * (D + kPartHeader);
      if (!sel_rows) {  // pass A saw every key tile: its maximum is the row's
        if (h == 0 && row_ok) rec[0] = mx == neg_inf() ? mx : mx * a.scale_log2;
        continue;
      }
      // ---- pass B: candidates >= bound ----
      uint32_t ad = base;
      const uint32_t last = base + (kCap - 1) * kPsSlot;
      for (int j = 0; j < tl.n_kt && ok; ++j)
        ok = take(j, limit, [&](const float(&v)[64], int tb) {
#pragma unroll
          for (int e = 0; e < 64; ++e) ps_append(ad, last, v[e], bound, static_cast<uint32_t>(tb + e + (e >> 5) * 32));
        });
      if (!ok) break;
      const uint32_t cnt = (ad - base) / kPsSlot;
      bool ovf = cnt > static_cast<uint32_t>(kCap);  // the row goes to the exact per-row pass
      const int mine = min(static_cast<int>(cnt), kCap);
      cnt_x[h * kPfRows + r] = static_cast<uint8_t>(ovf ? 255 : mine);
      // The row's k-th candidate score T: each half's kSl largest (values
      // only, sorted kSl at a time) meet through the TMEM exchange columns
      // (lane = row) and are merged by both.
      float top[kSl];
      {
#pragma unroll
        for (int q = 0; q < kSl; ++q) top[q] = q < mine ? __uint_as_float(lds_u32(base + q * kPsSlot)) : neg_inf();
        ps_sort<kSl>(top);
        for (int s0 = kSl; s0 < mine; s0 += kSl) {
          float x[kSl];
#pragma unroll
          for (int q = 0; q < kSl; ++q)
            x[q] = s0 + q < mine ? __uint_as_float(lds_u32(base + (s0 + q) * kPsSlot)) : neg_inf();
          ps_sort<kSl>(x);
          ps_merge<kSl>(top, x);
        }
      }
#pragma unroll
      for (int c = 0; c < kSl / 16; ++c) tc::st16(tmem + lane_addr + kPsXchgCol + kSl * h + 16 * c, top + 16 * c);
      tc::fence_before_sync();
      if (!pair_sync()) break;
      tc::fence_after_sync();
      {
        float o[kSl];
#pragma unroll
        for (int c = 0; c < kSl / 16; ++c) tc::ld16(tmem + lane_addr + kPsXchgCol + kSl * (h ^ 1) + 16 * c, o + 16 * c);
        ps_merge<kSl>(top, o);
      }
      float T = top[0];
#pragma unroll
      for (int q = 1; q < kSl; ++q)
        if (q < ksel) T = top[q];
      // the row maximum: the largest candidate (every score at or above the
      // bound is one); a listed row gets it from the exact per-row pass
      if (h == 0 && row_ok) rec[0] = top[0] == neg_inf() ? top[0] : top[0] * a.scale_log2;
      ovf |= cnt_x[(h ^ 1) * kPfRows + r] == 255;
      // this half's entries >= T, compacted in order to the column's front
      uint32_t w = base;
      for (int s0 = 0; s0 < mine; s0 += 8) {
        uint2 x[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) x[k] = lds_u2(base + min(s0 + k, kCap - 1) * kPsSlot);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (s0 + k < mine && __uint_as_float(x[k].x) >= T) {
            sts_u2(w, x[k]);
            w += kPsSlot;
          }
      }
      const int n_own = static_cast<int>((w - base) / kPsSlot);
      sel_x[h * kPfRows + r] = static_cast<uint8_t>(n_own);
      if (!pair_sync()) break;
      const int n_their = sel_x[(h ^ 1) * kPfRows + r];
      // every entry >= T is selected unless T is shared past the k-th place
      // (then the index rule decides: the exact per-row pass)
      ovf |= n_own + n_their != ksel;
      if (row_ok) {
        if (ovf) {
          if (h == 0) {  // listed for the exact per-row pass
            const uint32_t slot = atomicAdd(a.ovf_count, 1u);
            a.ovf_rows[slot] = static_cast<int32_t>(orow);
          }
        } else {
          // the merged selection in ascending chunk index order; this half
          // writes output slots (K/2) h .. (K/2) h + K/2 - 1 (both lists are
          // ascending)
          int ia = 0, ib = 0;
          for (int q = 0; q < kHalfOut * h; ++q) {
            const uint32_t xa = ia < n_own ? lds_u32(base + ia * kPsSlot + 4) : 0xffffffffu;
            const uint32_t xb = ib < n_their ? lds_u32(pbase + ib * kPsSlot + 4) : 0xffffffffu;
            if (xa < xb) ++ia;
            else ++ib;
          }
          int32_t oid[kHalfOut];
          float osc[kHalfOut];
#pragma unroll
          for (int q = 0; q < kHalfOut; ++q) {
            const uint2 xa = ia < n_own ? lds_u2(base + ia * kPsSlot) : make_uint2(0u, 0xffffffffu);
            const uint2 xb = ib < n_their ? lds_u2(pbase + ib * kPsSlot) : make_uint2(0u, 0xffffffffu);
            const bool ta = xa.y < xb.y;
            const uint2 x = ta ? xa : xb;
            ia += ta ? 1 : 0;
            ib += ta ? 0 : 1;
            const bool valid = x.y != 0xffffffffu;
            oid[q] = valid ? static_cast<int32_t>(x.y) : -1;
            osc[q] = valid ? __uint_as_float(x.x) * a.scale : neg_inf();
          }
          int32_t *oi = a.sel_idx + orow * a.topk + kHalfOut * h;
          float *os = a.sel_score + orow * a.topk + kHalfOut * h;
          if (a.topk == K) {  // rows of K entries: 16-byte aligned stores
#pragma unroll
            for (int q = 0; q < kHalfOut; q += 4) {
              reinterpret_cast<int4 *>(oi)[q / 4] = make_int4(oid[q], oid[q + 1], oid[q + 2], oid[q + 3]);
              reinterpret_cast<float4 *>(os)[q / 4] = make_float4(osc[q], osc[q + 1], osc[q + 2], osc[q + 3]);
            }
          } else {
#pragma unroll
            for (int q = 0; q < kHalfOut; ++q)
              if (kHalfOut * h + q < a.topk) {
                oi[q] = oid[q];
                os[q] = osc[q];
              }
          }
        }
      }
      if (!pair_sync()) break;  // the columns are free for the next tile
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
// Stage 1b, k_prefill_select_rows: the exact selection of the rows that
// k_prefill_score listed (a full candidate column, or scores equal to the
// k-th at the boundary; a handful of rows for most inputs).  One CTA of
// 1024 threads per listed row: its visible gist scores go to shared memory
// (16 lanes per key), each warp picks its k best of its keys by rounds of
// a warp argmax by (score desc, index asc), warp 0 picks the row's k from
// the warps' lists, and they are written in ascending chunk order.  The
// last CTA re-arms the list counter for the next call.
struct SelectRowsArgs {
  const __nv_bfloat16 *q_raw, *k_gist;  // [B*hq*L, D], [B*hkv*N, D]
  const int32_t *rows;                  // listed output rows (b*hq + h)*L + pos
  uint32_t *count, *done;               // list length; CTAs finished
  int32_t group, chunk, n_chunks, L, topk, pos0;
  float scale;
  int32_t *sel_idx;
  float *sel_score;
  float *rec_raw;     // [rows, D + 4]: [0] gets the row maximum (base 2)
  float scale_log2;
};

constexpr int kSelThreads = 1024;  // k_prefill_select_rows: a whole block per listed row
constexpr int kSelWarps = kSelThreads / 32;

template <int D, int K>
__global__ void __launch_bounds__(kSelThreads) k_prefill_select_rows(const SelectRowsArgs a) {
  constexpr int kLpk = D / 8;      // lanes per key (8 dims each)
  constexpr int kKpl = 32 / kLpk;  // keys per warp load
  extern __shared__ float sc[];  // [n_chunks] scores, then [D] query, then the picks' scores
  __shared__ float wl_v[kSelWarps * K];  // each warp's best ksel (score, index), best first
  __shared__ int wl_i[kSelWarps * K];
  __shared__ int picks[K];
  pdl_wait();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t n = *reinterpret_cast<volatile uint32_t *>(a.count);
  float *qs = sc + a.n_chunks;
  for (uint32_t i = blockIdx.x; i < n; i += gridDim.x) {  // one listed row per CTA
    const int orow = a.rows[i];
    const int bh = orow / a.L, pos = orow % a.L;
    const int limit = min(a.n_chunks, (a.pos0 + pos) / a.chunk);
    const int ksel = min(a.topk, limit);
    if (tid < D) qs[tid] = __bfloat162float(a.q_raw[static_cast<size_t>(orow) * D + tid]);
    __syncthreads();
    // Scores: D/8 lanes per key (8 elements each, the query slice in
    // registers), so a warp reads 32/(D/8) whole keys (512 contiguous
    // bytes) per load; eight such loads are issued before the arithmetic.
    const __nv_bfloat16 *kb = a.k_gist + static_cast<size_t>(bh / a.group) * a.n_chunks * D;
    {
      const int sub = lane % kLpk, half = lane / kLpk;
      float qv[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) qv[e] = qs[8 * sub + e];
      constexpr int kU = 8;
      for (int j0 = 0; j0 * kKpl * kSelWarps < limit; j0 += kU) {
        uint4 w[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int t = ((j0 + u) * kSelWarps + warp) * kKpl + half;
          w[u] = t < limit ? ldg_nc_v4(kb + static_cast<size_t>(t) * D + 8 * sub) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int t = ((j0 + u) * kSelWarps + warp) * kKpl + half;
          float f[8];
          Vec16<__nv_bfloat16>::unpack(w[u], f);
          float s = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) s = fmaf(qv[e], f[e], s);
#pragma unroll
          for (int o = kLpk / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
          if (sub == 0 && t < limit) sc[t] = s;
        }
      }
    }
    __syncthreads();
    // Top ksel by (score desc, index asc), in two levels of argmax rounds
    // that stay inside a warp: warp w takes keys w*32 + lane + kSelThreads j
    // (each lane keeps its best untaken key and rescans after losing it)
    // and lists its ksel best in order; warp 0 then merges the 32 ordered
    // lists (lane l holds the head of warp l's list) into the row's ksel.
    // Equal scores keep the lower index at every step.
    auto better = [](float v, int i, float bv, int bi) { return v > bv || (v == bv && i < bi); };
    auto lane_best = [&](float &bv, int &bi) {
      bv = neg_inf();
      bi = 0x7fffffff;
      for (int t = warp * 32 + lane; t < limit; t += kSelThreads) {
        const float v = sc[t];
        if (v > bv) {  // t increases: equal scores keep the lower index
          bv = v;
          bi = t;
        }
      }
    };
    {
      float bv;
      int bi;
      lane_best(bv, bi);
      for (int it = 0; it < ksel; ++it) {
        float wv = bv;
        int wi = bi;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, wv, o);
          const int oi = __shfl_xor_sync(0xffffffffu, wi, o);
          if (better(ov, oi, wv, wi)) {
            wv = ov;
            wi = oi;
          }
        }
        if (lane == 0) {
          wl_v[warp * K + it] = wv;
          wl_i[warp * K + it] = wi;
        }
        if (wi == bi && wi != 0x7fffffff) {  // this lane's key was taken: its next best
          sc[bi] = neg_inf();
          lane_best(bv, bi);
        }
        __syncwarp();
      }
    }
    __syncthreads();
    if (warp == 0) {
      static_assert(kSelWarps == 32, "one list per lane");
      int p = 0;  // this lane's position in warp `lane`'s list
      for (int it = 0; it < ksel; ++it) {
        const float hv = p < ksel ? wl_v[lane * K + p] : neg_inf();
        const int hi = p < ksel ? wl_i[lane * K + p] : 0x7fffffff;
        float wv = hv;
        int wi = hi;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, wv, o);
          const int oi = __shfl_xor_sync(0xffffffffu, wi, o);
          if (better(ov, oi, wv, wi)) {
            wv = ov;
            wi = oi;
          }
        }
        if (p < ksel && hi == wi && hv == wv) ++p;  // this list's head was taken (indices are distinct)
        if (lane == 0) {
          const bool ok = wi < limit;  // false only for non-finite scores
          picks[it] = ok ? wi : 0x7fffffff;
          qs[D + it] = wv;  // pick scores follow the query
        }
      }
    }
    __syncthreads();
    // the first pick is the row maximum
    if (tid == 0)
      a.rec_raw[static_cast<size_t>(orow) * (D + kPartHeader)] = ksel > 0 ? qs[D] * a.scale_log2 : neg_inf();
    // ascending chunk order: a pick's slot is the number of picks below it
    int32_t *oi = a.sel_idx + static_cast<size_t>(orow) * a.topk;
    float *os = a.sel_score + static_cast<size_t>(orow) * a.topk;
    if (tid < ksel) {
      int slot = 0;
      for (int u = 0; u < ksel; ++u) slot += (picks[u] < picks[tid] || (picks[u] == picks[tid] && u < tid)) ? 1 : 0;
      const bool ok = picks[tid] != 0x7fffffff;
      oi[slot] = ok ? picks[tid] : -1;
      os[slot] = ok ? qs[D + tid] * a.scale : neg_inf();
    } else if (tid < a.topk) {
      oi[tid] = -1;
      os[tid] = neg_inf();
    }
    __syncthreads();
  }
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    if (atomicAdd(a.done, 1u) == gridDim.x - 1) {
      *a.count = 0u;
      *a.done = 0u;
      __threadfence();
    }
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

template <int D>
struct GaSmem {
  static constexpr uint32_t kBlock = 128 * 128;                 // 128 rows x 64 16-bit values
  static constexpr uint32_t kTile = (D / 64) * kBlock;          // 128 rows x D (Q, K or V)
  static constexpr uint32_t kPTile = 2 * kBlock;                // 128 rows x 128 keys (P)
  static constexpr uint32_t kQOff = 0;
  static constexpr uint32_t kKOff = kTile;                      // 2 stages
  static constexpr uint32_t kVOff = kKOff + 2 * kTile;          // 2 stages
  static constexpr uint32_t kPOff = kVOff + 2 * kTile;          // 2 buffers
  static constexpr uint32_t kBarOff = kPOff + 2 * kPTile;
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

template <int D>
__global__ void __launch_bounds__(kPfThreads, 1) k_prefill_gist_attn(const __grid_constant__ PrefillArgs a) {
  using Sm = GaSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Sm::kBarOff);
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
        uint8_t *qdst = smem + Sm::kQOff;
        const CUtensorMap *qm = tl.is_gist ? &a.tm_qgist : &a.tm_qraw;
        const int qrow = tl.bh * (tl.is_gist ? a.n_chunks : a.L) + tl.row0;
        mbar_arrive_expect_tx(q_full, Sm::kTile);
#pragma unroll
        for (int x = 0; x < D / 64; ++x) tc::tma_load_2d(qdst + x * Sm::kBlock, qm, 64 * x, qrow, q_full);
        const int krow0 = (tl.bh / a.group) * a.n_chunks;
        for (int j = 0; j < tl.n_kt; ++j, ++ki) {
          const int s = ki & 1;
          const uint32_t par = ((ki >> 1) & 1) ^ 1;
          if (!wait(&k_empty[s], par) || !wait(&v_empty[s], par)) {
            ok = false;
            break;
          }
          uint8_t *kdst = smem + Sm::kKOff + s * Sm::kTile;
          uint8_t *vdst = smem + Sm::kVOff + s * Sm::kTile;
          mbar_arrive_expect_tx(&k_full[s], Sm::kTile);
#pragma unroll
          for (int x = 0; x < D / 64; ++x)
            tc::tma_load_2d(kdst + x * Sm::kBlock, &a.tm_kgist, 64 * x, krow0 + j * kGaKeys, &k_full[s]);
          mbar_arrive_expect_tx(&v_full[s], Sm::kTile);
#pragma unroll
          for (int x = 0; x < D / 64; ++x)
            tc::tma_load_2d(vdst + x * Sm::kBlock, &a.tm_vgist, 64 * x, krow0 + j * kGaKeys, &v_full[s]);
        }
        ++qi;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = tc::idesc_bf16(kPfRows, kGaKeys, false, false);
      constexpr uint32_t idesc_o = tc::idesc_f16kind(kPfRows, D, false, true, false);  // fp16; B = V, MN-major
      const uint32_t sbase = smem_u32(smem);
      uint32_t qi = 0, ki = 0, si = 0, pi = 0, oi = 0;
      bool ok = true;
      // GEMM1 for key tile j into S buffer (si & 1)
      auto gemm1 = [&](int j) -> bool {
        const int s = ki & 1, sb = si & 1;
        if (!wait(&k_full[s], (ki >> 1) & 1) || !wait(&s_empty[sb], ((si >> 1) & 1) ^ 1)) return false;
        tc::fence_after_sync();
        const uint32_t qa = sbase + Sm::kQOff, ka = sbase + Sm::kKOff + s * Sm::kTile;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint64_t ad = tc::sw128_desc(qa + (k >> 2) * Sm::kBlock + (k & 3) * 32, 16);
          const uint64_t bd = tc::sw128_desc(ka + (k >> 2) * Sm::kBlock + (k & 3) * 32, 16);
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
        const uint32_t pa = sbase + Sm::kPOff + pb * Sm::kPTile, va = sbase + Sm::kVOff + s * Sm::kTile;
#pragma unroll
        for (int k = 0; k < 8; ++k) {  // 128 keys = 8 x 16
          const uint64_t ad = tc::sw128_desc(pa + (k >> 2) * Sm::kBlock + (k & 3) * 32, 16);
          const uint64_t bd = tc::sw128_desc(va + k * 16 * 128, Sm::kBlock);
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
      float *rec = (tl.is_gist ? a.rec_gist : a.rec_raw) + orow * (D + kPartHeader);
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
        uint8_t *pbase = smem + Sm::kPOff + pb * Sm::kPTile;
#pragma unroll
        for (int u = 0; u < 16; ++u) {  // 16-byte units along the 128 keys
          const int kb = u >> 3, uu = u & 7;
          uint8_t *dst = pbase + kb * Sm::kBlock + (prow >> 3) * 1024 + (prow & 7) * 128 + ((uu ^ (prow & 7)) * 16);
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
      for (int c = 0; c < D / 32; ++c) {
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
// D/16 lanes owns one key row (16 dims per lane, packed fp32x2 FMAs), so a
// step covers 32/(D/16) rows, and up to two steps' loads are in flight.
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

constexpr int kGatherWarps = 4;

// (d.x, d.y) += (a.x * b.x, a.y * b.y): one packed fp32x2 FMA.
__device__ __forceinline__ void fma2_pair(float2 &d, float ax, float ay, float bx, float by) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rd, {%0, %1};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rd;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "+f"(d.x), "+f"(d.y)
      : "f"(ax), "f"(ay), "f"(bx), "f"(by));
}

template <int D>
__global__ void __launch_bounds__(kGatherWarps * 32) k_prefill_gather(const GatherArgs a) {
  constexpr int kE = 16, kLpr = D / kE, kSlots = 32 / kLpr, kU = 2;  // dims per lane, lanes per row, rows per step
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
  Vec16<__nv_bfloat16>::unpack(ldg_nc_v4(qrow + dd + 8), qf + 8);
  float m = neg_inf(), l = 0.f;
  float2 acc[kE / 2];
#pragma unroll
  for (int e = 0; e < kE / 2; ++e) acc[e] = make_float2(0.f, 0.f);
  // acc += p * v for the 16 values of v (two 16-byte words of bf16 pairs)
  auto add_v = [&](float p, const uint4 &v0, const uint4 &v1) {
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) fma2_pair(acc[e], p, p, bf16_lo(w[e]), bf16_hi(w[e]));
  };
  auto update = [&](float z, const uint4 &v0, const uint4 &v1) {
    if (z > m + 8.0f) {
      const float c = exp2_approx(m - z);
      l *= c;
#pragma unroll
      for (int e = 0; e < kE / 2; ++e) {
        acc[e].x *= c;
        acc[e].y *= c;
      }
      m = z;
    }
    const float p = exp2_approx(z - m);
    l += p;
    add_v(p, v0, v1);
  };
  // q . k for this lane's 16 dims (packed), summed over the row's lanes
  auto dot = [&](const uint4 &k0, const uint4 &k1) {
    const uint32_t w[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
    float2 s = make_float2(0.f, 0.f);
#pragma unroll
    for (int e = 0; e < 8; ++e) fma2_pair(s, qf[2 * e], qf[2 * e + 1], bf16_lo(w[e]), bf16_hi(w[e]));
    float part = s.x + s.y;
#pragma unroll
    for (int o = 1; o < kLpr; o <<= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    return part;
  };
  // attend raw rows [first, first + n) of this kv head: up to kU steps of
  // kSlots rows with their loads in flight (steps past n are skipped)
  auto span = [&](int first, int n) {
    for (int r0 = 0; r0 < n; r0 += kU * kSlots) {
      uint4 kw[kU][2], vw[kU][2];
#pragma unroll
      for (int u = 0; u < kU; ++u)
        if (r0 + kSlots * u < n) {  // warp-uniform
          const int r = r0 + kSlots * u + slot;
          const __nv_bfloat16 *kp = a.k_raw + (kv0 + first + min(r, n - 1)) * D + dd;
          const __nv_bfloat16 *vp = a.v_raw + (kv0 + first + min(r, n - 1)) * D + dd;
          kw[u][0] = ldg_nc_v4(kp);
          kw[u][1] = ldg_nc_v4(kp + 8);
          vw[u][0] = ldg_nc_v4(vp);
          vw[u][1] = ldg_nc_v4(vp + 8);
        }
#pragma unroll
      for (int u = 0; u < kU; ++u)
        if (r0 + kSlots * u < n) {
          const int r = r0 + kSlots * u + slot;
          const float part = dot(kw[u][0], kw[u][1]);
          if (r < n) update(part * a.scale_log2, vw[u][0], vw[u][1]);
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
        const __nv_bfloat16 *gv = a.v_gist + (static_cast<size_t>(kvh) * a.n_chunks + t) * D + dd;
        update(a.sel_score[ridx * a.topk + e] * kLog2e, ldg_nc_v4(gv), ldg_nc_v4(gv + 8));
      }
    }
    span(mc * a.chunk, pos - mc * a.chunk + 1);
  }
  // merge the row slots, then the gist partial of the row
  float accf[kE];
#pragma unroll
  for (int e = 0; e < kE / 2; ++e) {
    accf[2 * e] = acc[e].x;
    accf[2 * e + 1] = acc[e].y;
  }
#pragma unroll
  for (int o = kLpr; o < 32; o <<= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o), l2 = __shfl_xor_sync(0xffffffffu, l, o);
    float acc2[kE];
#pragma unroll
    for (int e = 0; e < kE; ++e) acc2[e] = __shfl_xor_sync(0xffffffffu, accf[e], o);
    merge_state<kE>(m, l, accf, m2, l2, acc2);
  }
  const bool has_prior = is_gist || !a.exclude;
  if (has_prior) {
    const float *rec = (is_gist ? a.rec_gist : a.rec_raw) + ridx * (D + kPartHeader);
    const float pm = rec[0], pl = rec[1];
    if (pm != neg_inf() && pl > 0.f) {
      float pacc[kE];
#pragma unroll
      for (int e = 0; e < kE; e += 4) {
        const float4 x = *reinterpret_cast<const float4 *>(rec + kPartHeader + dd + e);
        pacc[e] = x.x;
        pacc[e + 1] = x.y;
        pacc[e + 2] = x.z;
        pacc[e + 3] = x.w;
      }
      merge_state<kE>(m, l, accf, pm, pl, pacc);
    }
  }
  if (lane < kLpr) {
    void *out = is_gist ? a.out_gist : a.out_raw;
    const size_t base = static_cast<size_t>(ridx) * D + dd;
#pragma unroll
    for (int e = 0; e < kE; ++e) store_out(out, base + e, l > 0.f ? accf[e] / l : 0.f, a.out_bf16);
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
