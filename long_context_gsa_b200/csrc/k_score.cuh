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
// Rows are staged global->shared by bulk copies (TMA engine) into a 3-stage
// mbarrier ring; scores come from mma.sync m16n8k16 (rows = query heads,
// columns = gists); the value accumulation runs on the CUDA cores in fp32.
#pragma once

#include "common.cuh"

namespace gsa {

struct ScoreArgs {
  const void *q;          // [B, hq, D]
  const void *gk, *gv;    // [B, hkv, rows_cap, D]
  const int32_t *n_gists; // [B]
  int32_t count_div;      // rows scored = n_gists[b] / count_div
  int32_t rows_cap;       // rows per (b, kv head) in gk/gv
  float *scores;          // [B*hq, score_stride] natural-unit scores
  int32_t score_stride;
  float *part;            // [B*hq, n_split, D+4] or null
  int32_t n_split;
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
  static constexpr int kThreads = 256;
  static constexpr int kTile = 64;
  static constexpr int kStages = D == 64 ? 4 : 3;
  static constexpr uint32_t kTileBytes = kTile * D * 2;
  static constexpr uint32_t kStageBytes = kTileBytes * (WITH_V ? 2 : 1);
  // stages | p tiles [2][kTile][GH] | per-warp maxima [8][GH] | reference max [GH] | query fragments
  // [D/16][32 lanes] x uint2 | flags | barriers
  static constexpr uint32_t kSmemBytes =
      kStages * kStageBytes + (2 * kTile * GH + 8 * GH + GH) * 4 + (D / 16) * 32 * 8 + 16 + kStages * 8 + 64;
};

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

// bf16 inputs, D in {64, 128}, up to GH (4 or 8) query heads per CTA.
template <int D, int GH, bool WITH_V>
__global__ void __launch_bounds__(256, 2) k_score_mma(const ScoreArgs a) {
  using Cfg = ScoreMmaCfg<D, GH, WITH_V>;
  constexpr int kTile = Cfg::kTile, kStages = Cfg::kStages;
  constexpr int kLpr = D / 8, kRpw = 32 / kLpr, kSlots = 8 * kRpw;
  extern __shared__ __align__(128) uint8_t smem[];
  float *p_tile = reinterpret_cast<float *>(smem + kStages * Cfg::kStageBytes);  // [2][kTile][GH]
  float *wmax = p_tile + 2 * kTile * GH;                                         // [8][GH]
  float *m_sh = wmax + 8 * GH;                                                    // [GH] reference max
  uint2 *af_sh = reinterpret_cast<uint2 *>(m_sh + GH);                            // [D/16][32]
  int *flags = reinterpret_cast<int *>(af_sh + (D / 16) * 32);                    // [0] abort
  uint64_t *bars = reinterpret_cast<uint64_t *>((reinterpret_cast<uintptr_t>(flags + 4) + 7) & ~uintptr_t(7));

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
  const size_t row_base = (static_cast<size_t>(b) * a.hkv + kvh) * a.rows_cap + n0;
  const uint8_t *gk = reinterpret_cast<const uint8_t *>(a.gk) + row_base * D * 2;
  const uint8_t *gv = WITH_V ? reinterpret_cast<const uint8_t *>(a.gv) + row_base * D * 2 : nullptr;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
    mbar_fence_init();
    flags[0] = 0;
  }
  if (tid < GH) m_sh[tid] = neg_inf();
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

  auto issue = [&](int t) {
    const int st = t % kStages;
    const int rows = min(kTile, nrows - t * kTile);
    const uint32_t bytes = static_cast<uint32_t>(rows) * D * 2;
    uint8_t *dst = smem + st * Cfg::kStageBytes;
    mbar_arrive_expect_tx(&bars[st], bytes * (WITH_V ? 2u : 1u));
    bulk_g2s(dst, gk + static_cast<size_t>(t) * Cfg::kTileBytes, bytes, &bars[st]);
    if (WITH_V) bulk_g2s(dst + Cfg::kTileBytes, gv + static_cast<size_t>(t) * Cfg::kTileBytes, bytes, &bars[st]);
  };
  if (tid == 0)
    for (int t = 0; t < min(kStages, ntiles); ++t) issue(t);

  float acc[GH][8];
#pragma unroll
  for (int j = 0; j < GH; ++j)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[j][e] = 0.f;
  // Reference max (base 2) per head lives in m_sh, identical for every
  // thread; mg is this lane's copy for its head g.
  float mg = neg_inf();
  float l_part = 0.f;  // this lane's share of the sum for head g

  for (int t = 0; t < ntiles; ++t) {
    const int st = t % kStages;
    const int rows_t = min(kTile, nrows - t * kTile);
    if (!mbar_wait(&bars[st], (t / kStages) & 1)) flags[0] = 1;
    const uint8_t *Ks = smem + st * Cfg::kStageBytes;
    const uint8_t *Vs = Ks + Cfg::kTileBytes;
    float *pt = p_tile + (t & 1) * kTile * GH;

    // Scores of rows 8*warp .. 8*warp+7 for every head of the group.
    float s0 = neg_inf(), s1 = neg_inf();
    const int gi0 = 8 * warp + 2 * t4, gi1 = gi0 + 1;
    if (8 * warp < rows_t) {
      float c[4] = {0.f, 0.f, 0.f, 0.f};
      const uint8_t *krow = Ks + (8 * warp + g) * D * 2;
#pragma unroll
      for (int s2 = 0; s2 < D / 32; ++s2) {
        const uint4 kb = lds_v4(krow + (32 * s2 + 8 * t4) * 2);
        const uint2 a0 = af_sh[(2 * s2) * 32 + lane], a1 = af_sh[(2 * s2 + 1) * 32 + lane];
        mma_16816_bf16(c, a0.x, 0u, a0.y, 0u, kb.x, kb.y);
        mma_16816_bf16(c, a1.x, 0u, a1.y, 0u, kb.z, kb.w);
      }
      if (g < nh) {
        float *srow = a.scores ? a.scores + (static_cast<size_t>(b) * a.hq + h0 + g) * a.score_stride + n0 + t * kTile
                               : nullptr;
        if (gi0 < rows_t) {
          if (srow) srow[gi0] = c[0] * a.scale;
          s0 = c[0] * a.scale_log2;
        }
        if (gi1 < rows_t) {
          if (srow) srow[gi1] = c[1] * a.scale;
          s1 = c[1] * a.scale_log2;
        }
      }
    }
    bool need = false;
    float tl = 0.f;
    if (WITH_V) {
      need = s0 > mg + kRescaleSlack || s1 > mg + kRescaleSlack;
      if (!need && g < GH) {
        const float p0 = exp2_approx(s0 - mg), p1 = exp2_approx(s1 - mg);
        pt[gi0 * GH + g] = p0;
        pt[gi1 * GH + g] = p1;
        tl = p0 + p1;
      }
    }
    const bool slow = __syncthreads_or(need);
    if (flags[0]) {
      if (tid == 0) {
        flag_error(a.status, GSA_DEVERR_TIMEOUT);
        for (int u = t; u < min(t + kStages, ntiles); ++u) mbar_wait(&bars[u % kStages], (u / kStages) & 1);
      }
      __syncthreads();
      return;
    }
    // Every warp is past the value pass of tile t-1: its stage can refill.
    if (tid == 0 && t >= 1 && t - 1 + kStages < ntiles) issue(t - 1 + kStages);
    if (!WITH_V) continue;

    if (slow) {
      // Raise the reference max to this tile's max, rescale, redo p.
      float qm = fmaxf(s0, s1);
      qm = fmaxf(qm, __shfl_xor_sync(0xffffffffu, qm, 1));
      qm = fmaxf(qm, __shfl_xor_sync(0xffffffffu, qm, 2));
      if (t4 == 0 && g < GH) wmax[warp * GH + g] = qm;
      __syncthreads();
      float m_mine = neg_inf();  // new reference of head `tid` (tid < GH)
#pragma unroll
      for (int j = 0; j < GH; ++j) {
        float tm = neg_inf();
#pragma unroll
        for (int w = 0; w < 8; ++w) tm = fmaxf(tm, wmax[w * GH + j]);
        const float mo = m_sh[j];
        const float mn = fmaxf(mo, tm);
        const float alpha = (mn == neg_inf()) ? 1.f : exp2_approx(mo - mn);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[j][e] *= alpha;
        if (j == g) {
          l_part *= alpha;
          mg = mn;
        }
        if (j == tid) m_mine = mn;
      }
      __syncthreads();  // everyone has read the old reference
      if (tid < GH) m_sh[tid] = m_mine;
      if (g < GH) {
        const float p0 = exp2_approx(s0 - mg), p1 = exp2_approx(s1 - mg);
        pt[gi0 * GH + g] = p0;
        pt[gi1 * GH + g] = p1;
        tl = p0 + p1;
      }
      __syncthreads();
    }
    l_part += tl;

    // Values: slot = (warp, row group); this lane owns dims dd .. dd+7.
    const int slot = warp * kRpw + lane / kLpr;
    const int dd = 8 * (lane % kLpr);
    for (int r = slot; r < rows_t; r += kSlots) {
      const uint4 vw = lds_v4(Vs + (r * D + dd) * 2);
      float v[8];
      Vec16<__nv_bfloat16>::unpack(vw, v);
      float p[GH];
#pragma unroll
      for (int j4 = 0; j4 < GH / 4; ++j4) {
        const float4 pp = reinterpret_cast<const float4 *>(pt + r * GH)[j4];
        p[4 * j4] = pp.x;
        p[4 * j4 + 1] = pp.y;
        p[4 * j4 + 2] = pp.z;
        p[4 * j4 + 3] = pp.w;
      }
#pragma unroll
      for (int j = 0; j < GH; ++j)
#pragma unroll
        for (int e = 0; e < 8; e += 2) fma2(acc[j][e], acc[j][e + 1], p[j], v[e], v[e + 1]);
    }
  }

  pdl_trigger();
  if (WITH_V && a.part) {
    __syncthreads();  // all value passes done before the ring is reused
    // Per-head sums: lanes of quad g across all warps.
    l_part += __shfl_xor_sync(0xffffffffu, l_part, 1);
    l_part += __shfl_xor_sync(0xffffffffu, l_part, 2);
    if (t4 == 0 && g < GH) wmax[warp * GH + g] = l_part;
#pragma unroll
    for (int o = kLpr; o < 32; o <<= 1)
#pragma unroll
      for (int j = 0; j < GH; ++j)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[j][e] += __shfl_xor_sync(0xffffffffu, acc[j][e], o);
    float *red = reinterpret_cast<float *>(smem);  // [8][GH][D]
    if (lane < kLpr) {
#pragma unroll
      for (int j = 0; j < GH; ++j)
#pragma unroll
        for (int e = 0; e < 8; e += 4)
          *reinterpret_cast<float4 *>(red + (warp * GH + j) * D + 8 * lane + e) =
              make_float4(acc[j][e], acc[j][e + 1], acc[j][e + 2], acc[j][e + 3]);
    }
    __syncthreads();
    for (int i = tid; i < nh * D; i += Cfg::kThreads) {
      const int j = i / D, dim = i % D;
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) s += red[(w * GH + j) * D + dim];
      a.part[((static_cast<size_t>(b) * a.hq + h0 + j) * a.n_split + split) * (D + kPartHeader) + kPartHeader + dim] = s;
    }
    if (tid < nh) {
      float l = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) l += wmax[w * GH + tid];
      const float mt = m_sh[tid];
      float *hdr = a.part + ((static_cast<size_t>(b) * a.hq + h0 + tid) * a.n_split + split) * (D + kPartHeader);
      hdr[0] = mt;
      hdr[1] = l;
      hdr[2] = 0.f;
      hdr[3] = 0.f;
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
