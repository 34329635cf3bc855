// k_score.cuh -- relevance scoring of gist (or meta-gist) keys, fused with
// the softmax partial over the same rows.
//
// Method: "Scoring" on gist.science/nl/paper/2604.20920 ("Het Proces"):
// s_{t,m} = q_t^T k_{g_m}, here times `scale`; gist.science/ja section 2.1
// step 2.  In the default attended set every completed gist appears (its raw
// tokens too when selected), so the partial (max, sum, sum p*v) over all
// gists does not depend on the selection and is produced in this pass,
// while the gist values stream past anyway.
//
// Work decomposition: one CTA per (split of the gist rows, kv head [x head
// half], batch).  The query heads of one GQA group share every K/V load.
// Rows are staged global->shared by TMA tiled loads (128-byte swizzle) into
// a 3-stage mbarrier ring.  Each warp owns 16 rows of a stage: the scores
// come from mma.sync m16n8k16 (rows = query heads, columns = gists), and
// the same accumulator fragments, exponentiated and split into a bf16 high
// and low part, are the A operand of the P.V mma (k = the 16 rows), so the
// value accumulation also runs on the tensor cores with fp32 accumulators.
#pragma once

#include "common.cuh"
#include "k_select.cuh"
#include "tc100.cuh"

namespace gsa {

struct ScoreArgs {
  CUtensorMap tm_k, tm_v;  // bf16 tensor-core path: [B*hkv*rows_cap, D] boxes of 64 columns x kTile rows
  const void *q;          // [B, hq, D]
  const void *gk, *gv;    // [B, hkv, rows_cap, D]
  const int32_t *n_gists; // [B]
  int32_t count_div;      // rows scored = n_gists[b] / count_div
  int32_t rows_cap;       // rows per (b, kv head) in gk/gv
  float *scores;          // [B*hq, score_stride] natural-unit scores
  int32_t score_stride;
  float *part;            // [B*hq, n_split, D+4] or null
  int32_t n_split;
  uint32_t *zero_rows;    // [B*hq] or null: zeroed for this kernel's heads (re-arms the unfold's counters)
  // Selection in the tail (tensor-core path, needs scores): the last CTAs
  // to finish a (b, kv head) group select the top k of the group's query
  // heads, 128 threads per head.
  uint32_t *unit_counters;  // [2 * B*hkv*head_split] (arrivals, selectors done) or null; re-armed to 0
  int32_t topk;
  int32_t *sel_idx;       // [B*hq, topk]
  float *sel_score;       // [B*hq, topk] or null
  ReadyList ready;        // w null, or each selected row is published there for the unfold
  uint32_t *status;
  int32_t hq, hkv, group;
  int32_t head_split;     // CTAs per kv head along the query heads
  float scale, scale_log2;
};

__device__ __forceinline__ void mma_16816_bf16(float c[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Slice of rows [n0, n1) handled by `split`; slices are multiples of 8.
__device__ __forceinline__ void score_slice(int N, int n_split, int split, int &n0, int &n1) {
  const int per = ((N + n_split - 1) / n_split + 7) & ~7;
  n0 = split * per;
  n1 = min(N, n0 + per);
  if (n1 < n0) n1 = n0;
}

template <int D, int GH, bool WITH_V>
struct ScoreMmaCfg {
  static constexpr int kWarps = D == 64 ? 8 : 4;
  static constexpr int kThreads = 32 * kWarps;
  static constexpr int kTile = 16 * kWarps;         // rows per stage; warp w owns rows 16w .. 16w+15
  static constexpr int kBoxes = D / 64;             // 64-column (128-byte) TMA boxes per row
  static constexpr uint32_t kBoxBytes = kTile * 128;
  static constexpr uint32_t kTileBytes = kBoxes * kBoxBytes;  // K (or V) of one stage
  static constexpr int kStages = 3;
  static constexpr uint32_t kStageBytes = kTileBytes * (WITH_V ? 2 : 1);
  // stages (1024-aligned) | per-warp (max, sum) [2][warps][GH] | query fragments [D/16][32] x uint2 |
  // stage release counters, abort flag, last tile issued per stage | barriers
  static constexpr uint32_t kStateOff = kStages * kStageBytes;
  static constexpr uint32_t kAfOff = kStateOff + 2 * kWarps * GH * 4;
  static constexpr uint32_t kCntOff = kAfOff + (D / 16) * 32 * 8;
  static constexpr uint32_t kBarOff = (kCntOff + (2 * kStages + 1) * 4 + 7) & ~7u;
  static constexpr uint32_t kSmemBytes = kBarOff + kStages * 8 + 1024;  // + alignment slack
  static_assert(kStages * kStageBytes >= kWarps * GH * D * 4 || !WITH_V, "merge buffer fits in the ring");
  // thread groups selecting at once in the tail (their scratch lives in the ring)
  static constexpr int kSelGroups = kThreads / kRowSelThreads;
  // longest row the tail selects (its scratch holds the row)
  static constexpr int kSelMaxN = D == 64 ? 4096 : 8192;
  static_assert(kSelGroups >= 1 && kSelGroups * sizeof(SelSmem<kSelMaxN>) <= kStages * kStageBytes,
                "selection scratch fits in the ring");
};

// The tail's selector CTAs of a group: the last `selectors` to arrive.
__device__ __forceinline__ int score_tail_selectors(int n_split, int nh, int groups) {
  return min(n_split, (nh + groups - 1) / groups);
}

// The rows (query heads j of the group) selector si of S selects: head j
// goes to selector (j / groups) mod S, thread group j mod groups.
__device__ __forceinline__ bool score_tail_mine(int j, int si, int S, int groups) { return (j / groups) % S == si; }

// A selector CTA is done: the last one re-arms the group's two counters.
__device__ __forceinline__ void score_tail_done(uint32_t *cnt, int selectors) {
  if (atomicAdd(&cnt[1], 1u) == static_cast<uint32_t>(selectors - 1)) {
    cnt[0] = 0u;
    cnt[1] = 0u;
  }
}

// Rescaling threshold (base-2 units): the running max used for the
// exponentials is only raised when a score exceeds it by more than this,
// so p <= 2^8 and the rescale of the accumulators is rare.  Numerator and
// denominator use the same reference, so the result is unchanged.
constexpr float kRescaleSlack = 8.0f;

// (acc.x, acc.y) += p * (v.x, v.y) with one packed fp32x2 FMA.
__device__ __forceinline__ void fma2(float &ax, float &ay, float p, float vx, float vy) {
  asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
      "mov.b64 ra, {%0, %1};\n\t"
      "mov.b64 rb, {%2, %3};\n\t"
      "mov.b64 rc, {%4, %4};\n\t"
      "fma.rn.f32x2 ra, rc, rb, ra;\n\t"
      "mov.b64 {%0, %1}, ra;\n\t}"
      : "+f"(ax), "+f"(ay)
      : "f"(vx), "f"(vy), "f"(p));
}

// ldmatrix .x4 .trans: four 8x8 bf16 matrices, row addresses from lanes
// 8i .. 8i+7 for matrix i, each thread receiving the transposed fragment.
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// Two floats -> bf16x2 (lo in the low half), round to nearest.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Byte offset of the 16-byte chunk `c` (0..7) of row `r` in a 128-byte
// swizzled TMA box (chunk index XOR row mod 8).
__device__ __forceinline__ uint32_t sw128(int r, int c) { return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4)); }

// bf16 inputs, D in {64, 128}, up to GH (4 or 8) query heads per CTA.
// Each warp owns 16 rows of every stage from scores to values, with its
// own softmax reference per head, so no block-wide barrier is needed per
// stage: the last warp to finish a stage refills it, and the warps' (max,
// sum, acc) states are merged once at the end.
template <int D, int GH, bool WITH_V>
__global__ void __launch_bounds__(ScoreMmaCfg<D, GH, WITH_V>::kThreads, 2)
    k_score_mma(const __grid_constant__ ScoreArgs a) {
  using Cfg = ScoreMmaCfg<D, GH, WITH_V>;
  constexpr int kTile = Cfg::kTile, kStages = Cfg::kStages, kWarps = Cfg::kWarps;
  constexpr int kNT = D / 8;  // value n-tiles (8 dims each)
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float *st_m = reinterpret_cast<float *>(smem + Cfg::kStateOff);  // [warps][GH]
  float *st_l = st_m + kWarps * GH;                                // [warps][GH]
  uint2 *af_sh = reinterpret_cast<uint2 *>(smem + Cfg::kAfOff);   // [D/16][32]
  int *cnt = reinterpret_cast<int *>(smem + Cfg::kCntOff);         // [kStages] warps done, [kStages] abort
  int *last_issued = cnt + kStages + 1;                            // [kStages]
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kBarOff);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, b = blockIdx.z;
  const int kvh = blockIdx.y / a.head_split, hpart = blockIdx.y % a.head_split;
  const int h0 = kvh * a.group + hpart * GH;
  const int nh = min(GH, a.group - hpart * GH);
  const int g = lane >> 2, t4 = lane & 3;  // mma fragment coordinates: head row g, gist pair t4

  pdl_wait();
  int N = a.n_gists[b] / a.count_div;
  N = min(max(N, 0), a.rows_cap);
  int n0, n1;
  score_slice(N, a.n_split, split, n0, n1);
  const int nrows = n1 - n0;
  const int ntiles = (nrows + kTile - 1) / kTile;
  const int row0 = (b * a.hkv + kvh) * a.rows_cap + n0;  // first tensor-map row of this slice

  if (a.zero_rows && split == 0 && tid < nh) a.zero_rows[static_cast<size_t>(b) * a.hq + h0 + tid] = 0u;
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
    for (int s = 0; s <= kStages; ++s) cnt[s] = 0;
    for (int s = 0; s < kStages; ++s) last_issued[s] = -1;
    mbar_fence_init();
    tc::prefetch_map(&a.tm_k);
    if (WITH_V) tc::prefetch_map(&a.tm_v);
  }
  // Query fragments (same for every warp).  The k dimension is permuted
  // identically in A and B: lane quad t4 reads dims [32*s2 + 8*t4, +8) as
  // two k-steps, so one 16-byte load per row feeds two mma k-steps.
  if (warp == 0) {
    const uint4 *qrow = reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(a.q) +
                                                        (static_cast<size_t>(b) * a.hq + h0 + min(g, nh - 1)) * D);
#pragma unroll
    for (int s2 = 0; s2 < D / 32; ++s2) {
      const uint4 w = g < nh ? qrow[4 * s2 + t4] : make_uint4(0, 0, 0, 0);
      af_sh[(2 * s2) * 32 + lane] = make_uint2(w.x, w.y);
      af_sh[(2 * s2 + 1) * 32 + lane] = make_uint2(w.z, w.w);
    }
  }
  __syncthreads();
  uint2 afr[D / 16];
#pragma unroll
  for (int i = 0; i < D / 16; ++i) afr[i] = af_sh[i * 32 + lane];

  const uint64_t stream_policy = tc::policy_evict_first();  // every gist row is read once
  auto issue = [&](int t) {
    const int st = t % kStages;
    uint8_t *dst = smem + st * Cfg::kStageBytes;
    *reinterpret_cast<volatile int *>(&last_issued[st]) = t;
    mbar_arrive_expect_tx(&bars[st], Cfg::kStageBytes);
#pragma unroll
    for (int x = 0; x < Cfg::kBoxes; ++x) {
      tc::tma_load_2d_hint(dst + x * Cfg::kBoxBytes, &a.tm_k, 64 * x, row0 + t * kTile, &bars[st], stream_policy);
      if (WITH_V)
        tc::tma_load_2d_hint(dst + Cfg::kTileBytes + x * Cfg::kBoxBytes, &a.tm_v, 64 * x, row0 + t * kTile, &bars[st],
                             stream_policy);
    }
  };
  if (tid == 0)
    for (int t = 0; t < min(kStages, ntiles); ++t) issue(t);

  float acc[kNT][4];  // P.V accumulators: rows g (head g) and g+8 (unused), dims 8*nt + 2*t4 (+1)
#pragma unroll
  for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
  float mg = neg_inf();  // this warp's reference max (base 2) for head g
  float lg = 0.f;        // this lane's share of the sum for head g
  const int rw = 16 * warp;
  const uint32_t sbase = smem_u32(smem);
  bool aborted = false;

  for (int t = 0; t < ntiles; ++t) {
    const int st = t % kStages;
    const int rows_t = min(kTile, nrows - t * kTile);
    if (!__all_sync(0xffffffffu, mbar_wait(&bars[st], (t / kStages) & 1))) {
      aborted = true;
      break;
    }
    const uint32_t ks = sbase + st * Cfg::kStageBytes, vs = ks + Cfg::kTileBytes;
    if (rw < rows_t) {
      // scores of rows rw .. rw+15 (two n-tiles of 8) for every head
      float c[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) c[nt][e] = 0.f;
        const int r = rw + 8 * nt + g;
#pragma unroll
        for (int s2 = 0; s2 < D / 32; ++s2) {
          uint4 kb;
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(kb.x), "=r"(kb.y), "=r"(kb.z), "=r"(kb.w)
                       : "r"(ks + (s2 >> 1) * Cfg::kBoxBytes + sw128(r, (s2 & 1) * 4 + t4)));
          mma_16816_bf16(c[nt], afr[2 * s2].x, 0u, afr[2 * s2].y, 0u, kb.x, kb.y);
          mma_16816_bf16(c[nt], afr[2 * s2 + 1].x, 0u, afr[2 * s2 + 1].y, 0u, kb.z, kb.w);
        }
      }
      float s[2][2];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int gi = rw + 8 * nt + 2 * t4 + e;
          s[nt][e] = neg_inf();
          if (g < nh && gi < rows_t) {
            if (a.scores)
              a.scores[(static_cast<size_t>(b) * a.hq + h0 + g) * a.score_stride + n0 + t * kTile + gi] = c[nt][e] * a.scale;
            s[nt][e] = c[nt][e] * a.scale_log2;
          }
        }
      if (WITH_V) {
        // lazy reference: raised only when this warp's rows exceed it by
        // more than kRescaleSlack; the head's accumulators then rescale
        float qm = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
        qm = fmaxf(qm, __shfl_xor_sync(0xffffffffu, qm, 1));
        qm = fmaxf(qm, __shfl_xor_sync(0xffffffffu, qm, 2));
        const bool need = qm > mg + kRescaleSlack;
        if (__any_sync(0xffffffffu, need)) {
          const float mn = need ? qm : mg;
          const float alpha = (mg == neg_inf() || mn == mg) ? 1.f : exp2_approx(mg - mn);
          lg *= alpha;
          mg = mn;
#pragma unroll
          for (int nt = 0; nt < kNT; ++nt) {
            acc[nt][0] *= alpha;
            acc[nt][1] *= alpha;
          }
        }
        float p[2][2];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) p[nt][e] = s[nt][e] > neg_inf() ? exp2_approx(s[nt][e] - mg) : 0.f;
        lg += (p[0][0] + p[0][1]) + (p[1][0] + p[1][1]);
        // A operand of P.V (k = the warp's 16 rows): bf16 high part and the
        // bf16 rounding of the remainder, so the weights keep ~16 bits
        const uint32_t h0p = pack_bf16(p[0][0], p[0][1]), h1p = pack_bf16(p[1][0], p[1][1]);
        const uint32_t l0p = pack_bf16(p[0][0] - bf16_lo(h0p), p[0][1] - bf16_hi(h0p));
        const uint32_t l1p = pack_bf16(p[1][0] - bf16_lo(h1p), p[1][1] - bf16_hi(h1p));
        if (rows_t - rw < 16) {
          // rows past the slice end enter the product with weight 0; clear
          // their values so that whatever the buffer holds there (the next
          // slice, or unwritten memory) cannot turn 0 * v into NaN
          for (int i = lane; i < (rw + 16 - max(rw, rows_t)) * 8 * Cfg::kBoxes; i += 32) {
            const int r = max(rw, rows_t) + i / (8 * Cfg::kBoxes), x = (i / 8) % Cfg::kBoxes, ch = i % 8;
            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(vs + x * Cfg::kBoxBytes + sw128(r, ch)),
                         "r"(0u)
                         : "memory");
          }
          tc::fence_proxy_async_smem();
          __syncwarp();
        }
        const int mi = lane >> 3;               // ldmatrix: matrix fed by this lane's address
        const int vr = rw + (mi & 1) * 8 + (lane & 7);
#pragma unroll
        for (int dp = 0; dp < kNT / 2; ++dp) {
          const int dim0 = 8 * (2 * dp + (mi >> 1));
          uint32_t b0, b1, b2, b3;
          ldsm_x4_trans(vs + (dim0 >> 6) * Cfg::kBoxBytes + sw128(vr, (dim0 & 63) >> 3), b0, b1, b2, b3);
          mma_16816_bf16(acc[2 * dp], h0p, 0u, h1p, 0u, b0, b1);
          mma_16816_bf16(acc[2 * dp], l0p, 0u, l1p, 0u, b0, b1);
          mma_16816_bf16(acc[2 * dp + 1], h0p, 0u, h1p, 0u, b2, b3);
          mma_16816_bf16(acc[2 * dp + 1], l0p, 0u, l1p, 0u, b2, b3);
        }
      }
    }
    // release the stage; the last of the warps to finish it refills it
    __syncwarp();
    if (lane == 0 && atomicAdd(&cnt[st], 1) == (t / kStages + 1) * kWarps - 1 && t + kStages < ntiles)
      issue(t + kStages);
  }
  if (aborted && lane == 0) atomicExch(&cnt[kStages], 1);
  __syncthreads();
  const int unit = blockIdx.z * gridDim.y + blockIdx.y;  // (b, kv head [x head half])
  if (cnt[kStages]) {
    // a wait expired: let every copy that may be in flight land, then leave
    // (still counted at the group's counter, which the last CTA re-arms)
    if (tid == 0) {
      flag_error(a.status, GSA_DEVERR_TIMEOUT);
      for (int s = 0; s < kStages; ++s) {
        const int tl = *reinterpret_cast<volatile int *>(&last_issued[s]);
        if (tl >= 0) mbar_wait(&bars[s], (tl / kStages) & 1);
      }
      if (a.unit_counters) {  // arrive; a selector that cannot select still counts as done
        const int S = score_tail_selectors(gridDim.x, nh, Cfg::kSelGroups);
        const int si = static_cast<int>(atomicAdd(&a.unit_counters[2 * unit], 1u)) - (static_cast<int>(gridDim.x) - S);
        if (si >= 0) {
          if (a.ready.w)  // its rows are published unselected, so the unfold does not wait for them
            for (int j = 0; j < nh; ++j)
              if (score_tail_mine(j, si, S, Cfg::kSelGroups)) ready_publish(a.ready, b * a.hq + h0 + j, a.status);
          score_tail_done(a.unit_counters + 2 * unit, S);
        }
      }
    }
    __syncthreads();
    return;
  }
  pdl_trigger();
  if (WITH_V && a.part) {
    // Per-warp states -> shared memory (the ring is free now), then merge.
    lg += __shfl_xor_sync(0xffffffffu, lg, 1);
    lg += __shfl_xor_sync(0xffffffffu, lg, 2);
    if (t4 == 0 && g < GH) {
      st_m[warp * GH + g] = mg;
      st_l[warp * GH + g] = lg;
    }
    float *red = reinterpret_cast<float *>(smem);  // [warps][GH][D]
    if (g < GH)
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt)
        *reinterpret_cast<float2 *>(red + (warp * GH + g) * D + 8 * nt + 2 * t4) = make_float2(acc[nt][0], acc[nt][1]);
    __syncthreads();
    for (int i = tid; i < nh * D; i += Cfg::kThreads) {
      const int j = i / D, dim = i % D;
      float M = neg_inf();
#pragma unroll
      for (int w = 0; w < kWarps; ++w) M = fmaxf(M, st_m[w * GH + j]);
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float mw = st_m[w * GH + j];
        if (mw > neg_inf()) sum += red[(w * GH + j) * D + dim] * exp2_approx(mw - M);
      }
      a.part[((static_cast<size_t>(b) * a.hq + h0 + j) * a.n_split + split) * (D + kPartHeader) + kPartHeader + dim] =
          sum;
    }
    if (tid < nh) {
      float M = neg_inf();
#pragma unroll
      for (int w = 0; w < kWarps; ++w) M = fmaxf(M, st_m[w * GH + tid]);
      float l = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float mw = st_m[w * GH + tid];
        if (mw > neg_inf()) l += st_l[w * GH + tid] * exp2_approx(mw - M);
      }
      float *hdr = a.part + ((static_cast<size_t>(b) * a.hq + h0 + tid) * a.n_split + split) * (D + kPartHeader);
      hdr[0] = M;
      hdr[1] = l;
      hdr[2] = 0.f;
      hdr[3] = 0.f;
    }
  }
  if (a.unit_counters) {
    // The last S CTAs to arrive at the group's counter select, one query
    // head per 128-thread group: each waits (bounded) until every CTA of
    // the group has arrived, after which all scores are visible to it
    // (writers: fence, then arrive; readers: acquire the count).  The ring
    // is free and holds the groups' selection scratch.
    __shared__ int arrive_s, ok_s;
    uint32_t *cnt2 = a.unit_counters + 2 * unit;
    const int n_split = static_cast<int>(gridDim.x);
    const int S = score_tail_selectors(n_split, nh, Cfg::kSelGroups);
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      arrive_s = static_cast<int>(atomicAdd(&cnt2[0], 1u));
    }
    __syncthreads();
    const int si = arrive_s - (n_split - S);  // selector index; negative: not a selector
    if (si >= 0) {
      if (tid == 0) {
        int ok = 1;
        uint64_t t0 = 0;
        for (uint32_t it = 0; ld_acquire_u32(&cnt2[0]) < static_cast<uint32_t>(n_split); ++it) {
          if ((it & 15u) == 0) {
            const uint64_t now = global_timer_ns();
            if (!t0) t0 = now;
            else if (now - t0 > kWaitLimitNs) {
              ok = 0;
              flag_error(a.status, GSA_DEVERR_TIMEOUT);
              break;
            }
          }
          __nanosleep(100);
        }
        ok_s = ok;
      }
      __syncthreads();
      const int grp = tid / kRowSelThreads;
      if (ok_s) {
        SelSmem<Cfg::kSelMaxN> &ssm = reinterpret_cast<SelSmem<Cfg::kSelMaxN> *>(smem)[grp];
        int use = 0;
        for (int j = si * Cfg::kSelGroups + grp; j < nh; j += S * Cfg::kSelGroups) {
          const size_t row = static_cast<size_t>(b) * a.hq + h0 + j;
          group_select<Cfg::kSelMaxN>(a.scores + row * a.score_stride, N, a.topk, tid % kRowSelThreads, ssm, 1 + grp,
                                      use, a.status, a.sel_idx + row * a.topk,
                                      a.sel_score ? a.sel_score + row * a.topk : nullptr);
          if (a.ready.w) {
            // every writer fences, then the group meets; one thread publishes
            __threadfence();
            group_bar(1 + grp);
            if (tid % kRowSelThreads == 0) ready_publish(a.ready, static_cast<int>(row), a.status);
          }
        }
      } else if (a.ready.w && tid % kRowSelThreads == 0) {
        for (int j = si * Cfg::kSelGroups + grp; j < nh; j += S * Cfg::kSelGroups)
          ready_publish(a.ready, b * a.hq + h0 + j, a.status);  // unselected (TIMEOUT is flagged)
      }
      __syncthreads();
      if (tid == 0) score_tail_done(cnt2, S);
    }
  }
}

// Any input dtype, any group size: plain CUDA-core loops.  Used for fp32
// inputs (small problems); scores must be non-null.
template <int D, typename T, bool WITH_V>
__global__ void __launch_bounds__(128) k_score_generic(const ScoreArgs a) {
  constexpr int kPer = D / 32;  // elements per lane
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  pdl_wait();
  int N = a.n_gists[b] / a.count_div;
  N = min(max(N, 0), a.rows_cap);
  int n0, n1;
  score_slice(N, a.n_split, split, n0, n1);
  const size_t row_base = (static_cast<size_t>(b) * a.hkv + kvh) * a.rows_cap;
  const T *gk = reinterpret_cast<const T *>(a.gk);
  const T *gv = reinterpret_cast<const T *>(a.gv);
  const T *q = reinterpret_cast<const T *>(a.q);
  for (int m = n0 + warp; m < n1; m += 4) {
    float kf[kPer];
#pragma unroll
    for (int e = 0; e < kPer; ++e) kf[e] = static_cast<float>(gk[(row_base + m) * D + lane + 32 * e]);
    for (int j = 0; j < a.group; ++j) {
      const int h = kvh * a.group + j;
      float s = 0.f;
#pragma unroll
      for (int e = 0; e < kPer; ++e) s = fmaf(static_cast<float>(q[(static_cast<size_t>(b) * a.hq + h) * D + lane + 32 * e]), kf[e], s);
      s = warp_sum(s);
      if (lane == 0) a.scores[(static_cast<size_t>(b) * a.hq + h) * a.score_stride + m] = s * a.scale;
    }
  }
  if (!WITH_V || !a.part) return;
  __syncthreads();
  for (int j = warp; j < a.group; j += 4) {
    const int h = kvh * a.group + j;
    const float *srow = a.scores + (static_cast<size_t>(b) * a.hq + h) * a.score_stride;
    float mx = neg_inf();
    for (int m = n0 + lane; m < n1; m += 32) mx = fmaxf(mx, srow[m] * kLog2e);
    mx = warp_max(mx);
    float l = 0.f, acc[kPer];
#pragma unroll
    for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
    for (int m = n0; m < n1; ++m) {
      const float p = exp2_approx(srow[m] * kLog2e - mx);
      l += p;
#pragma unroll
      for (int e = 0; e < kPer; ++e) acc[e] = fmaf(p, static_cast<float>(gv[(row_base + m) * D + lane + 32 * e]), acc[e]);
    }
    float *rec = a.part + ((static_cast<size_t>(b) * a.hq + h) * a.n_split + split) * (D + kPartHeader);
#pragma unroll
    for (int e = 0; e < kPer; ++e) rec[kPartHeader + lane + 32 * e] = acc[e];
    if (lane == 0) {
      rec[0] = mx;
      rec[1] = l;
      rec[2] = 0.f;
      rec[3] = 0.f;
    }
  }
}

}  // namespace gsa
