// gsa_api.cu -- the extern "C" boundary of libgsa.so (see include/gsa.h).
//
// Host side only: argument checks, workspace layout, split sizing and
// kernel launches.  Every step of the computation runs in the kernels
// included below; nothing here touches tensor data.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "../../include/gsa.h"
#include "common.cuh"
#include "k_backward.cuh"
#include "k_gist_step.cuh"
#include "k_hgsa.cuh"
#include "k_prefill.cuh"
#include "k_score.cuh"
#include "k_select.cuh"
#include "k_topk.cuh"
#include "k_topp.cuh"
#include "k_unfold.cuh"

namespace gsa {
namespace {

constexpr int kScoreSplitMax = 64;   // partial slots per row from the scoring pass
constexpr int kUnfoldSplitMax = 32;  // partial slots per row from the unfold pass
constexpr int kHgsaSplitMax = 32;    // partial slots per row from the H-GSA pass
constexpr int kTopkSmemCap = 16384;  // keys kept in shared memory by the top-k kernel
constexpr int kMaxTopk = kTopkMax;

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t elem_size(int32_t dt) { return dt == GSA_BF16 ? 2 : 4; }
inline float resolve_scale(const gsa_desc *d) {
  return d->scale > 0.f ? d->scale : 1.0f / std::sqrt(static_cast<float>(d->d));
}

struct Layout {
  size_t status = 0, counters = 0, scores = 0, sel_idx = 0, sel_score = 0, part_g = 0, part_u = 0;
  size_t unit_counters = 0, ready = 0;
  size_t meta_scores = 0, meta_idx = 0, cand_scores = 0, cand_ids = 0, cand_count = 0, part_h = 0;
  size_t meta2_scores = 0, meta2_idx = 0, cand1_scores = 0, cand1_ids = 0, cand1_count = 0;
  size_t pf_stats = 0, pf_gist = 0, pf_vh = 0, pf_ovf = 0;
  size_t gs_cur = 0, gs_plus = 0;
  size_t total = 0;
};

gsa_status check_desc(const gsa_desc *d) {
  if (!d) return GSA_ERR_INVALID_ARG;
  if (d->batch < 1 || d->hq < 1 || d->hkv < 1 || d->hq % d->hkv) return GSA_ERR_INVALID_ARG;
  if (d->hq / d->hkv > 16) return GSA_ERR_UNSUPPORTED;
  if (d->d != 64 && d->d != 128) return GSA_ERR_UNSUPPORTED;
  if (d->chunk < 1 || d->chunk > 64) return GSA_ERR_UNSUPPORTED;
  if (d->n_max < 1 || d->t_max < 1 || d->n_max > (1 << 24) || d->t_max > (1 << 28)) return GSA_ERR_INVALID_ARG;
  if (d->topk < 0) return GSA_ERR_INVALID_ARG;
  if (d->topk > kMaxTopk) return GSA_ERR_UNSUPPORTED;
  if (d->exclude_unselected != 0 && d->exclude_unselected != 1) return GSA_ERR_INVALID_ARG;
  if (d->dtype != GSA_F32 && d->dtype != GSA_BF16) return GSA_ERR_INVALID_ARG;
  if (d->out_dtype != GSA_F32 && d->out_dtype != GSA_BF16) return GSA_ERR_INVALID_ARG;
  if (!std::isfinite(d->scale)) return GSA_ERR_INVALID_ARG;
  if (static_cast<size_t>(d->chunk) * d->d * elem_size(d->dtype) > 32768) return GSA_ERR_UNSUPPORTED;
  return GSA_OK;
}

gsa_status check_hdesc(const gsa_desc *d, const gsa_hdesc *h) {
  if (!h) return GSA_ERR_INVALID_ARG;
  if (h->group < 1 || h->topk_meta < 1 || h->m_max < 1) return GSA_ERR_INVALID_ARG;
  if (h->topk_meta > 64 || static_cast<int64_t>(h->topk_meta) * h->group > 4096 || h->group > 4096)
    return GSA_ERR_UNSUPPORTED;
  if (h->m_max < d->n_max / h->group) return GSA_ERR_INVALID_ARG;
  return GSA_OK;
}

inline int hgsa_cand_cap(const gsa_hdesc *h) { return h->topk_meta * h->group + h->group - 1; }

// Two meta levels: level1 groups gists into meta-gists, level2 groups
// level-1 meta-gists into level-2 meta-gists.
gsa_status check_h2desc(const gsa_desc *d, const gsa_h2desc *h) {
  if (!h) return GSA_ERR_INVALID_ARG;
  const gsa_status s1 = check_hdesc(d, &h->level1);
  if (s1 != GSA_OK) return s1;
  const gsa_hdesc &l2 = h->level2;
  if (l2.group < 1 || l2.topk_meta < 1 || l2.m_max < 1) return GSA_ERR_INVALID_ARG;
  if (l2.topk_meta > 64 || static_cast<int64_t>(l2.topk_meta) * l2.group > 4096 || l2.group > 4096)
    return GSA_ERR_UNSUPPORTED;
  if (l2.m_max < h->level1.m_max / l2.group) return GSA_ERR_INVALID_ARG;
  if (h->level1.topk_meta > hgsa_cand_cap(&l2)) return GSA_ERR_INVALID_ARG;
  return GSA_OK;
}

// Whether the scoring kernel can select in its tail: bf16 (tensor-core
// scorer) and rows short enough for the selecting threads' registers.
inline bool tail_select_ok(const gsa_desc *d) {
  return d->dtype == GSA_BF16 && d->n_max <= kRowSelThreads * (d->d == 64 ? 32 : 64);
}

Layout layout(const gsa_desc *d, int32_t op, const gsa_hdesc *h) {
  Layout L;
  const size_t rows = static_cast<size_t>(d->batch) * d->hq;
  const size_t rec = static_cast<size_t>(d->d + kPartHeader) * 4;
  size_t off = 0;
  auto take = [&](size_t &field, size_t bytes) {
    field = off;
    off = align256(off + bytes);
  };
  take(L.status, 256);
  take(L.counters, rows * 4);
  if (op == GSA_OP_MULTIQUERY) {  // t_max = queries per (document, head)
    const size_t prow = rows * static_cast<size_t>(d->t_max);
    take(L.pf_stats, prow * rec);
    take(L.pf_ovf, prow * 4);
    L.total = off;
    return L;
  }
  if (op == GSA_OP_PREFILL) {
    const size_t prow = rows * static_cast<size_t>(d->t_max);
    take(L.sel_idx, prow * d->topk * 4);
    take(L.sel_score, prow * d->topk * 4);
    take(L.pf_stats, prow * rec);
    take(L.pf_gist, rows * static_cast<size_t>(d->n_max) * rec);
    take(L.pf_vh, static_cast<size_t>(d->batch) * d->hkv * d->n_max * d->d * 2);
    take(L.pf_ovf, prow * 4);
    L.total = off;
    return L;
  }
  take(L.unit_counters, rows * 8);
  take(L.ready, (rows + 4) * 4);  // with the status and counters: the prefix a scratch-free call clears
  take(L.scores, rows * d->n_max * 4);
  take(L.sel_idx, rows * d->topk * 4);
  take(L.sel_score, rows * d->topk * 4);
  take(L.part_g, rows * kScoreSplitMax * rec);
  take(L.part_u, rows * kUnfoldSplitMax * rec);
  if ((op == GSA_OP_HGSA || op == GSA_OP_HGSA2) && h) {
    const size_t cap = hgsa_cand_cap(h);
    take(L.meta_scores, rows * h->m_max * 4);
    take(L.meta_idx, rows * h->topk_meta * 4);
    take(L.cand_scores, rows * cap * 4);
    take(L.cand_ids, rows * cap * 4);
    take(L.cand_count, rows * 4);
    take(L.part_h, rows * kHgsaSplitMax * rec);
  }
  if (op == GSA_OP_GIST_STEP) {
    take(L.gs_cur, static_cast<size_t>(d->batch) * 4);
    take(L.gs_plus, static_cast<size_t>(d->batch) * 4);
  }
  if (op == GSA_OP_HGSA2 && h) {  // h points at a gsa_h2desc: level1, then level2
    const gsa_hdesc *l2 = h + 1;
    const size_t cap1 = hgsa_cand_cap(l2);
    take(L.meta2_scores, rows * l2->m_max * 4);
    take(L.meta2_idx, rows * l2->topk_meta * 4);
    take(L.cand1_scores, rows * cap1 * 4);
    take(L.cand1_ids, rows * cap1 * 4);
    take(L.cand1_count, rows * 4);
  }
  L.total = off;
  return L;
}

inline uint8_t *at(void *ws, size_t off) { return static_cast<uint8_t *>(ws) + off; }

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

inline int cdiv(int a, int b) { return (a + b - 1) / b; }
inline int clampi(int x, int lo, int hi) { return x < lo ? lo : (x > hi ? hi : x); }

// Allow `smem` bytes of dynamic shared memory for `kern` (needed above 48 KB).
template <typename Kern>
bool prepare(Kern kern, size_t smem) {
  return smem <= 48 * 1024 ||
         cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) ==
             cudaSuccess;
}

// CTAs of `kern` that fit on the whole GPU at once.
template <typename Kern>
int resident_ctas(Kern kern, int threads, size_t smem) {
  int per_sm = 0;
  if (!prepare(kern, smem) ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem) != cudaSuccess || per_sm < 1) {
    cudaGetLastError();
    per_sm = 1;
  }
  return per_sm * sm_count();
}

// Splits per unit so that all CTAs fit in one wave (at least one split).
inline int one_wave_splits(int units, int slots, int max_splits) {
  return clampi(slots / std::max(units, 1), 1, std::max(1, max_splits));
}

// Launch with programmatic stream serialization: the kernel may start while
// its predecessor drains; it calls griddepcontrol.wait before touching data.
template <typename Kern, typename... Args>
gsa_status launch(Kern kern, dim3 grid, dim3 block, size_t smem, void *stream, const Args &...args) {
  if (grid.x == 0 || grid.y == 0 || grid.z == 0) return GSA_OK;
  if (!prepare(kern, smem)) return GSA_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return GSA_ERR_CUDA;
  }
  return GSA_OK;
}

#define GSA_TRY(x)                     \
  do {                                 \
    const gsa_status _s = (x);         \
    if (_s != GSA_OK) return _s;       \
  } while (0)

gsa_status need_ptr(const void *p) { return (p && aligned16(p)) ? GSA_OK : GSA_ERR_INVALID_ARG; }
gsa_status opt_ptr(const void *p) { return (!p || aligned16(p)) ? GSA_OK : GSA_ERR_INVALID_ARG; }

// ---------------------------------------------------------------- scoring
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
    cudaGetLastError();
  });
  return fn;
}

// 2D 16-bit view [rows, cols] with 64-column, box_rows-row boxes, 128-byte swizzle.
bool map_rows(CUtensorMap *m, const void *base, uint64_t rows, uint32_t box_rows,
              CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, uint64_t cols = 128) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t es[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int GH, bool V>
gsa_status launch_score_mma_t(const ScoreArgs &sa, int splits, int B, void *stream) {
  using Cfg = ScoreMmaCfg<D, GH, V>;
  ScoreArgs ta = sa;
  const uint64_t rows = static_cast<uint64_t>(B) * sa.hkv * sa.rows_cap;
  if (!map_rows(&ta.tm_k, sa.gk, rows, Cfg::kTile, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, D) ||
      (V && !map_rows(&ta.tm_v, sa.gv, rows, Cfg::kTile, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, D)))
    return GSA_ERR_CUDA;
  return launch(k_score_mma<D, GH, V>, dim3(splits, sa.hkv * sa.head_split, B), dim3(Cfg::kThreads), Cfg::kSmemBytes,
                stream, ta);
}

template <int D, int GH, bool V>
int score_mma_slots() {
  using Cfg = ScoreMmaCfg<D, GH, V>;
  return resident_ctas(k_score_mma<D, GH, V>, Cfg::kThreads, Cfg::kSmemBytes);
}

struct ScorePlan {
  bool mma;
  int GH, head_split, splits;
};

// How the scoring pass is cut: CTAs over (row slices, kv head [x head
// half], batch), as many slices as fit the GPU in one wave.
ScorePlan plan_score(const gsa_desc *d, int rows_cap, bool with_v) {
  ScorePlan p;
  const int group = d->hq / d->hkv;
  p.mma = d->dtype == GSA_BF16;
  p.GH = group <= 4 ? 4 : 8;
  p.head_split = p.mma ? cdiv(group, p.GH) : 1;
  int slots;
  if (!p.mma) {
    slots = 4 * sm_count();
  } else if (d->d == 64) {
    slots = p.GH == 4 ? (with_v ? score_mma_slots<64, 4, true>() : score_mma_slots<64, 4, false>())
                      : (with_v ? score_mma_slots<64, 8, true>() : score_mma_slots<64, 8, false>());
  } else {
    slots = p.GH == 4 ? (with_v ? score_mma_slots<128, 4, true>() : score_mma_slots<128, 4, false>())
                      : (with_v ? score_mma_slots<128, 8, true>() : score_mma_slots<128, 8, false>());
  }
  p.splits = one_wave_splits(d->batch * d->hkv * p.head_split, slots,
                             std::min(kScoreSplitMax, cdiv(rows_cap, 64)));
  return p;
}

template <int D, bool V>
gsa_status launch_score_generic_t(const ScoreArgs &sa, int splits, int B, int dtype, void *stream) {
  if (dtype == GSA_BF16)
    return launch(k_score_generic<D, __nv_bfloat16, V>, dim3(splits, sa.hkv, B), dim3(128), 0, stream, sa);
  return launch(k_score_generic<D, float, V>, dim3(splits, sa.hkv, B), dim3(128), 0, stream, sa);
}

// Score rows of `keys` (gists or meta-gists) against q; optional partial.
gsa_status run_score(const gsa_desc *d, const void *q, const void *keys, const void *vals, const int32_t *n_gists,
                     int count_div, int rows_cap, float *scores, int score_stride, float *part, int *splits_out,
                     uint32_t *status, void *stream, uint32_t *zero_rows = nullptr,
                     uint32_t *unit_counters = nullptr, int32_t *sel_idx = nullptr, float *sel_score = nullptr,
                     uint32_t *ready = nullptr) {
  const int group = d->hq / d->hkv;
  const bool with_v = part != nullptr;
  const ScorePlan plan = plan_score(d, rows_cap, with_v);
  const bool mma = plan.mma;
  const int GH = plan.GH;
  const int head_split = plan.head_split;
  const int splits = plan.splits;
  if (splits_out) *splits_out = splits;
  ScoreArgs sa;
  sa.q = q;
  sa.gk = keys;
  sa.gv = vals;
  sa.n_gists = n_gists;
  sa.count_div = count_div;
  sa.rows_cap = rows_cap;
  sa.scores = scores;
  sa.score_stride = score_stride;
  sa.part = part;
  sa.n_split = splits;
  sa.zero_rows = mma ? zero_rows : nullptr;
  sa.unit_counters = mma && scores && sel_idx ? unit_counters : nullptr;
  sa.topk = d->topk;
  sa.sel_idx = sel_idx;
  sa.sel_score = sel_score;
  sa.ready.w = sa.unit_counters ? ready : nullptr;
  sa.ready.rows = d->batch * d->hq;
  sa.status = status;
  sa.hq = d->hq;
  sa.hkv = d->hkv;
  sa.group = group;
  sa.head_split = head_split;
  sa.scale = resolve_scale(d);
  sa.scale_log2 = sa.scale * kLog2e;
  if (!mma) {
    if (d->d == 64)
      return with_v ? launch_score_generic_t<64, true>(sa, splits, d->batch, d->dtype, stream)
                    : launch_score_generic_t<64, false>(sa, splits, d->batch, d->dtype, stream);
    return with_v ? launch_score_generic_t<128, true>(sa, splits, d->batch, d->dtype, stream)
                  : launch_score_generic_t<128, false>(sa, splits, d->batch, d->dtype, stream);
  }
#define GSA_SCORE_CASE(DD, GG)                                                                         \
  if (d->d == DD && GH == GG)                                                                          \
    return with_v ? launch_score_mma_t<DD, GG, true>(sa, splits, d->batch, stream)                     \
                  : launch_score_mma_t<DD, GG, false>(sa, splits, d->batch, stream);
  GSA_SCORE_CASE(64, 4)
  GSA_SCORE_CASE(64, 8)
  GSA_SCORE_CASE(128, 4)
  GSA_SCORE_CASE(128, 8)
#undef GSA_SCORE_CASE
  return GSA_ERR_UNSUPPORTED;
}

gsa_status run_topk(int rows, int hq, const float *scores, int stride, const int32_t *n_gists, int count_div,
                    const int32_t *counts, int k, const int32_t *id_map, int32_t *sel_idx, float *sel_score,
                    uint32_t *counters, void *stream, uint32_t *status = nullptr) {
  TopkArgs ta;
  ta.scores = scores;
  ta.stride = stride;
  ta.n_gists = n_gists;
  ta.count_div = count_div;
  ta.counts = counts;
  ta.hq = hq;
  ta.k = k;
  ta.id_map = id_map;
  ta.sel_idx = sel_idx;
  ta.sel_score = sel_score;
  ta.counters = counters;
  ta.status = status;
  ta.smem_cap = std::min(stride, kTopkSmemCap);
  const dim3 grid(rows), block(kTopkRegThreads);
  constexpr size_t kRowBytes = kTopkRegThreads * 4;  // staged row bytes per key a thread holds
  if (stride <= 4 * kTopkRegThreads) return launch(k_topk<4>, grid, block, 4 * kRowBytes, stream, ta);
  if (stride <= 16 * kTopkRegThreads) return launch(k_topk<16>, grid, block, 16 * kRowBytes, stream, ta);
  if (stride <= 32 * kTopkRegThreads) return launch(k_topk<32>, grid, block, 32 * kRowBytes, stream, ta);
  if (stride <= 64 * kTopkRegThreads) return launch(k_topk<64>, grid, block, 64 * kRowBytes, stream, ta);
  return launch(k_topk_mem, grid, dim3(kTopkThreads), static_cast<size_t>(ta.smem_cap) * 4, stream, ta);
}

template <int D, typename T>
size_t unfold_smem(int chunk) {
  const int piece_bytes = unfold_piece_rows<D, T>(chunk) * D * static_cast<int>(sizeof(T));
  return static_cast<size_t>(kUnfoldWarps) * unfold_warp_stages(2 * piece_bytes) * 2 * piece_bytes;
}

template <int D, typename T>
gsa_status launch_unfold_t(UnfoldArgs ua, int B, void *stream) {
  if (std::is_same<T, __nv_bfloat16>::value) {
    // tensor-core kernel: raw K/V as 2D maps with 8-row boxes
    // residency with the largest list share (one split), then the share of the chosen split count
    const int slots =
        resident_ctas(k_unfold_tc<D>, kUnfoldThreads, UnfoldTcCfg<D>::smem_bytes(std::max(1, ua.k), ua.chunk));
    ua.n_split = one_wave_splits(B * ua.hq, slots, std::min(kUnfoldSplitMax, std::max(1, ua.k)));
    const size_t smem = UnfoldTcCfg<D>::smem_bytes((std::max(1, ua.k) + ua.n_split - 1) / ua.n_split, ua.chunk);
    const uint64_t rows = static_cast<uint64_t>(B) * ua.hkv * ua.t_max;
    if (!map_rows(&ua.tm_k, ua.raw_k, rows, 8, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, D) ||
        !map_rows(&ua.tm_v, ua.raw_v, rows, 8, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, D))
      return GSA_ERR_CUDA;
    return launch(k_unfold_tc<D>, dim3(ua.n_split, ua.hq, B), dim3(kUnfoldThreads), smem, stream, ua);
  }
  ua.ready.w = nullptr;  // the CUDA-core kernel always follows the whole previous kernel
  const size_t smem = unfold_smem<D, T>(ua.chunk);
  const int slots = resident_ctas(k_unfold<D, T>, kUnfoldThreads, smem);
  ua.n_split = one_wave_splits(B * ua.hq, slots, std::min(kUnfoldSplitMax, std::max(1, ua.k)));
  return launch(k_unfold<D, T>, dim3(ua.n_split, ua.hq, B), dim3(kUnfoldThreads), smem, stream, ua);
}

gsa_status run_unfold(const gsa_desc *d, const void *q, const void *raw_k, const void *raw_v, const void *gist_v,
                      const int32_t *n_gists, const int32_t *own_len, const int32_t *sel_idx, const float *sel_score,
                      const float *prior, int n_prior, void *out, float *lse, const Layout &L, void *ws,
                      void *stream, uint32_t *ready = nullptr) {
  UnfoldArgs ua;
  ua.q = q;
  ua.raw_k = raw_k;
  ua.raw_v = raw_v;
  ua.gist_v = gist_v;
  ua.n_gists = n_gists;
  ua.own_len = own_len;
  ua.sel_idx = sel_idx;
  ua.sel_score = sel_score;
  ua.k = d->topk;
  ua.chunk = d->chunk;
  ua.t_max = d->t_max;
  ua.n_max = d->n_max;
  ua.hq = d->hq;
  ua.hkv = d->hkv;
  ua.group = d->hq / d->hkv;
  ua.exclude = d->exclude_unselected;
  ua.scale_log2 = resolve_scale(d) * kLog2e;
  ua.part = reinterpret_cast<float *>(at(ws, L.part_u));
  ua.n_split = 1;  // set by launch_unfold_t
  ua.prior = prior;
  ua.n_prior = prior ? n_prior : 0;
  ua.counters = reinterpret_cast<uint32_t *>(at(ws, L.counters));
  ua.ready.w = ready;
  ua.ready.rows = d->batch * d->hq;
  ua.status = reinterpret_cast<uint32_t *>(at(ws, L.status));
  ua.out = out;
  ua.out_bf16 = d->out_dtype == GSA_BF16;
  ua.lse = lse;
  if (d->dtype == GSA_BF16)
    return d->d == 64 ? launch_unfold_t<64, __nv_bfloat16>(ua, d->batch, stream)
                      : launch_unfold_t<128, __nv_bfloat16>(ua, d->batch, stream);
  return d->d == 64 ? launch_unfold_t<64, float>(ua, d->batch, stream) : launch_unfold_t<128, float>(ua, d->batch, stream);
}

// Splits per row of the H-GSA candidate pass; depends on the descriptor only
// (gsa_unfold_attend needs it without the H-GSA parameters).
int hgsa_splits(const gsa_desc *d) {
  // the children kernel's rings take at most 64 KB per CTA: 3 CTAs per SM
  return one_wave_splits(d->batch * d->hq, 3 * sm_count(), kHgsaSplitMax);
}

template <int D, typename T>
gsa_status launch_hgsa_children_t(const HgsaArgs &ha, int B, void *stream) {
  const int piece_bytes = unfold_piece_rows<D, T>(ha.group) * D * static_cast<int>(sizeof(T));
  const size_t smem = static_cast<size_t>(kHgsaWarps) * unfold_warp_stages(2 * piece_bytes) * 2 * piece_bytes;
  return launch(k_hgsa_children<D, T>, dim3(ha.n_split, ha.hq, B), dim3(kHgsaThreads), smem, stream, ha);
}

gsa_status launch_children(const gsa_desc *d, const HgsaArgs &ha, void *stream) {
  if (d->dtype == GSA_BF16)
    return d->d == 64 ? launch_hgsa_children_t<64, __nv_bfloat16>(ha, d->batch, stream)
                      : launch_hgsa_children_t<128, __nv_bfloat16>(ha, d->batch, stream);
  return d->d == 64 ? launch_hgsa_children_t<64, float>(ha, d->batch, stream)
                    : launch_hgsa_children_t<128, float>(ha, d->batch, stream);
}

gsa_status run_hgsa_select(const gsa_desc *d, const gsa_hdesc *hd, const void *q, const void *meta_k,
                           const void *meta_v, const void *gist_k, const void *gist_v, const int32_t *n_gists,
                           int32_t *meta_idx, int32_t *sel_idx, float *sel_score, const Layout &L, void *ws,
                           void *stream) {
  const int rows = d->batch * d->hq;
  uint32_t *status = reinterpret_cast<uint32_t *>(at(ws, L.status));
  float *meta_scores = reinterpret_cast<float *>(at(ws, L.meta_scores));
  // 1. meta-gist scores; 2. top meta groups (ascending group order)
  GSA_TRY(run_score(d, q, meta_k, nullptr, n_gists, hd->group, hd->m_max, meta_scores, hd->m_max, nullptr, nullptr,
                    status, stream));
  GSA_TRY(run_topk(rows, d->hq, meta_scores, hd->m_max, n_gists, hd->group, nullptr, hd->topk_meta, nullptr, meta_idx,
                   nullptr, nullptr, stream));
  // 3. children of the chosen groups (+ trailing gists): scores, ids, partial
  HgsaArgs ha;
  ha.q = q;
  ha.gist_k = gist_k;
  ha.gist_v = gist_v;
  ha.meta_v = meta_v;
  ha.meta_scores = meta_scores;
  ha.meta_idx = meta_idx;
  ha.n_gists = n_gists;
  ha.group = hd->group;
  ha.topk_meta = hd->topk_meta;
  ha.m_max = hd->m_max;
  ha.n_max = d->n_max;
  ha.hq = d->hq;
  ha.hkv = d->hkv;
  ha.gqa = d->hq / d->hkv;
  ha.exclude = d->exclude_unselected;
  ha.scale_log2 = resolve_scale(d) * kLog2e;
  ha.cand_scores = reinterpret_cast<float *>(at(ws, L.cand_scores));
  ha.cand_ids = reinterpret_cast<int32_t *>(at(ws, L.cand_ids));
  ha.cand_count = reinterpret_cast<int32_t *>(at(ws, L.cand_count));
  ha.cap = hgsa_cand_cap(hd);
  ha.part = reinterpret_cast<float *>(at(ws, L.part_g));
  ha.n_split = hgsa_splits(d);
  ha.status = status;
  ha.count_div = 1;
  ha.fold_children = 1;
  ha.parent_ids = nullptr;
  ha.parent_scores = nullptr;
  ha.parent_count = nullptr;
  ha.parent_cap = 0;
  ha.part_stride = ha.n_split;
  ha.part_off = 0;
  GSA_TRY(launch_children(d, ha, stream));
  // 4. top gists among the candidates, reported as gist (chunk) ids
  if (d->topk > 0)
    return run_topk(rows, d->hq, ha.cand_scores, ha.cap, nullptr, 1, ha.cand_count, d->topk, ha.cand_ids, sel_idx,
                    sel_score, reinterpret_cast<uint32_t *>(at(ws, L.counters)), stream);
  return cudaMemsetAsync(at(ws, L.counters), 0, static_cast<size_t>(rows) * 4, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? GSA_OK
             : GSA_ERR_CUDA;
}

// Two meta levels: level-2 scores -> top level-2 groups -> level-1
// candidates (children pass, partial of the unselected level-2 meta-gists)
// -> top level-1 meta-gists -> gist candidates (children pass, partial of
// the unselected level-1 candidates and all gist candidates) -> top gists.
// The two passes' partials share one prior array: [rows][2 * splits].
gsa_status run_hgsa2_select(const gsa_desc *d, const gsa_h2desc *h2, const void *q, const void *meta2_k,
                            const void *meta2_v, const void *meta_k, const void *meta_v, const void *gist_k,
                            const void *gist_v, const int32_t *n_gists, int32_t *meta2_idx, int32_t *meta_idx,
                            int32_t *sel_idx, float *sel_score, const Layout &L, void *ws, void *stream) {
  const gsa_hdesc &l1 = h2->level1, &l2 = h2->level2;
  const int rows = d->batch * d->hq;
  uint32_t *status = reinterpret_cast<uint32_t *>(at(ws, L.status));
  float *meta2_scores = reinterpret_cast<float *>(at(ws, L.meta2_scores));
  const int g12 = l1.group * l2.group;
  GSA_TRY(run_score(d, q, meta2_k, nullptr, n_gists, g12, l2.m_max, meta2_scores, l2.m_max, nullptr, nullptr, status,
                    stream));
  GSA_TRY(run_topk(rows, d->hq, meta2_scores, l2.m_max, n_gists, g12, nullptr, l2.topk_meta, nullptr, meta2_idx,
                   nullptr, nullptr, stream));
  const int splits = hgsa_splits(d);
  HgsaArgs ha;
  ha.q = q;
  ha.n_gists = n_gists;
  ha.hq = d->hq;
  ha.hkv = d->hkv;
  ha.gqa = d->hq / d->hkv;
  ha.exclude = d->exclude_unselected;
  ha.scale_log2 = resolve_scale(d) * kLog2e;
  ha.part = reinterpret_cast<float *>(at(ws, L.part_g));
  ha.n_split = splits;
  ha.status = status;
  ha.part_stride = 2 * splits;
  // level-1 candidates: children of the chosen level-2 groups
  ha.gist_k = meta_k;
  ha.gist_v = meta_v;
  ha.meta_v = meta2_v;
  ha.meta_scores = meta2_scores;
  ha.meta_idx = meta2_idx;
  ha.group = l2.group;
  ha.topk_meta = l2.topk_meta;
  ha.m_max = l2.m_max;
  ha.n_max = l1.m_max;
  ha.count_div = l1.group;
  ha.fold_children = 0;  // the unselected level-1 candidates enter in the next pass
  ha.parent_ids = nullptr;
  ha.parent_scores = nullptr;
  ha.parent_count = nullptr;
  ha.parent_cap = 0;
  ha.cand_scores = reinterpret_cast<float *>(at(ws, L.cand1_scores));
  ha.cand_ids = reinterpret_cast<int32_t *>(at(ws, L.cand1_ids));
  ha.cand_count = reinterpret_cast<int32_t *>(at(ws, L.cand1_count));
  ha.cap = hgsa_cand_cap(&l2);
  ha.part_off = 0;
  GSA_TRY(launch_children(d, ha, stream));
  GSA_TRY(run_topk(rows, d->hq, ha.cand_scores, ha.cap, nullptr, 1, ha.cand_count, l1.topk_meta, ha.cand_ids,
                   meta_idx, nullptr, nullptr, stream));
  // gist candidates: children of the chosen level-1 meta-gists; the
  // unselected level-1 candidates are the listed parents of this pass
  const float *c1_scores = ha.cand_scores;
  const int32_t *c1_ids = ha.cand_ids, *c1_count = ha.cand_count;
  const int cap1 = ha.cap;
  ha.gist_k = gist_k;
  ha.gist_v = gist_v;
  ha.meta_v = meta_v;
  ha.meta_scores = c1_scores;  // (unused with listed parents)
  ha.meta_idx = meta_idx;
  ha.group = l1.group;
  ha.topk_meta = l1.topk_meta;
  ha.m_max = l1.m_max;
  ha.n_max = d->n_max;
  ha.count_div = 1;
  ha.fold_children = 1;
  ha.parent_ids = c1_ids;
  ha.parent_scores = c1_scores;
  ha.parent_count = c1_count;
  ha.parent_cap = cap1;
  ha.cand_scores = reinterpret_cast<float *>(at(ws, L.cand_scores));
  ha.cand_ids = reinterpret_cast<int32_t *>(at(ws, L.cand_ids));
  ha.cand_count = reinterpret_cast<int32_t *>(at(ws, L.cand_count));
  ha.cap = hgsa_cand_cap(&l1);
  ha.part_off = splits;
  GSA_TRY(launch_children(d, ha, stream));
  if (d->topk > 0)
    return run_topk(rows, d->hq, ha.cand_scores, ha.cap, nullptr, 1, ha.cand_count, d->topk, ha.cand_ids, sel_idx,
                    sel_score, reinterpret_cast<uint32_t *>(at(ws, L.counters)), stream);
  return cudaMemsetAsync(at(ws, L.counters), 0, static_cast<size_t>(rows) * 4, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? GSA_OK
             : GSA_ERR_CUDA;
}

// ---------------------------------------------------------------- prefill
// Words of the 256-byte status block used by the prefill overflow list
// (word 0 is the device status; all are zeroed by gsa_workspace_init).
constexpr int kPfOvfCountWord = 16, kPfOvfDoneWord = 17;
// the exact per-row pass holds a row's scores, the query and its picks in
// dynamic shared memory next to the warps' pick lists (static)
// (k <= K): the static lists are 2 x kSelWarps x K words plus K picks.
constexpr int pf_select_max_chunks(int K) { return (227 << 10) / 4 - 128 - K - (2 * kSelWarps * K + (K > 32 ? K : 32)); }
constexpr int kPfSelectMaxChunks = pf_select_max_chunks(kPfTopkMax);        // 56912
constexpr int kPfSelectMaxChunksWide = pf_select_max_chunks(kPfTopkWide);   // 53760
static_assert(kPfSelectMaxChunks == 56912 && kPfSelectMaxChunksWide == 53760, "documented limits");

// The scorer variant a selection of k entries runs on.
inline bool pf_wide(const gsa_desc *d) { return d->topk > kPfTopkMax; }
inline int pf_max_chunks(const gsa_desc *d) { return pf_wide(d) ? kPfSelectMaxChunksWide : kPfSelectMaxChunks; }

gsa_status check_prefill(const gsa_desc *d) {
  GSA_TRY(check_desc(d));
  if (d->dtype != GSA_BF16 || (d->d != 64 && d->d != 128)) return GSA_ERR_UNSUPPORTED;
  if (d->topk > kPfTopkWide) return GSA_ERR_UNSUPPORTED;  // the wide scorer's lists hold at most 64
  // the exact re-selection of listed rows holds one row's gist scores in shared memory
  if (d->n_max > pf_max_chunks(d)) return GSA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(d->n_max) * d->chunk != d->t_max) return GSA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(d->batch) * d->hq * d->t_max >= (int64_t(1) << 31)) return GSA_ERR_UNSUPPORTED;
  return GSA_OK;
}

// Multi-query scoring runs the prefill scoring kernel: bf16, d = 64 or 128,
// topk 1..64, one row of gist scores in shared memory for the exact re-pass.
gsa_status check_multiquery(const gsa_desc *d) {
  GSA_TRY(check_desc(d));
  if (d->dtype != GSA_BF16 || (d->d != 64 && d->d != 128)) return GSA_ERR_UNSUPPORTED;
  if (d->topk < 1 || d->topk > kPfTopkWide) return GSA_ERR_UNSUPPORTED;
  if (d->n_max > pf_max_chunks(d)) return GSA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(d->batch) * d->hq * d->t_max >= (int64_t(1) << 31)) return GSA_ERR_UNSUPPORTED;
  return GSA_OK;
}

PrefillArgs prefill_args(const gsa_desc *d, int32_t *sel_idx, float *sel_score, const Layout &L, void *ws) {
  PrefillArgs pa;
  std::memset(&pa, 0, sizeof(pa));
  pa.bh = d->batch * d->hq;
  pa.hq = d->hq;
  pa.hkv = d->hkv;
  pa.group = d->hq / d->hkv;
  pa.chunk = d->chunk;
  pa.n_chunks = d->n_max;
  pa.L = d->t_max;
  pa.topk = d->topk;
  pa.exclude = d->exclude_unselected;
  pa.scale = resolve_scale(d);
  pa.scale_log2 = pa.scale * kLog2e;
  pa.sel_idx = sel_idx;
  pa.sel_score = sel_score;
  pa.rec_raw = reinterpret_cast<float *>(at(ws, L.pf_stats));
  pa.rec_gist = reinterpret_cast<float *>(at(ws, L.pf_gist));
  pa.gist_tiles = cdiv(d->n_max, kPfRows);
  pa.raw_tiles = cdiv(d->t_max, kPfRows);
  pa.status = reinterpret_cast<uint32_t *>(at(ws, L.status));
  pa.ovf_rows = reinterpret_cast<int32_t *>(at(ws, L.pf_ovf));
  pa.ovf_count = pa.status + kPfOvfCountWord;
  return pa;
}

// pos0 > 0 (multi-query scoring): the raw rows are queries placed after
// the whole gist cache, and there are no gist-position rows.
gsa_status run_prefill_score(const gsa_desc *d, const void *q_raw, const void *q_gist, const void *k_gist,
                             int32_t *sel_idx, float *sel_score, const Layout &L, void *ws, void *stream,
                             int pos0 = 0) {
  PrefillArgs pa = prefill_args(d, sel_idx, sel_score, L, ws);
  if (pos0 > 0) {
    pa.pos0 = pos0;
    pa.gist_tiles = 0;
  }
  const uint64_t bh = static_cast<uint64_t>(d->batch) * d->hq, bkv = static_cast<uint64_t>(d->batch) * d->hkv;
  const uint64_t qgist_rows = pos0 > 0 ? bh * d->t_max : bh * d->n_max;  // (not read when there are no gist rows)
  const auto bf16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const uint64_t D = static_cast<uint64_t>(d->d);
  if (!map_rows(&pa.tm_qraw, q_raw, bh * d->t_max, kPfRows, bf16, D) ||
      !map_rows(&pa.tm_qgist, q_gist, qgist_rows, kPfRows, bf16, D) ||
      !map_rows(&pa.tm_kgist, k_gist, bkv * d->n_max, kPfKeys, bf16, D))
    return GSA_ERR_CUDA;
  const int total = pa.bh * (pa.gist_tiles + pa.raw_tiles);
  const int grid = std::min(total, sm_count());
  const dim3 ps_grid(grid), ps_block(kPsThreads);
  constexpr int kN = kPfTopkMax, kW = kPfTopkWide;
  if (!pf_wide(d))
    GSA_TRY(d->d == 64 ? launch(k_prefill_score<kN, 64>, ps_grid, ps_block, PfSmem<64, kN>::kBytes, stream, pa)
                       : launch(k_prefill_score<kN, 128>, ps_grid, ps_block, PfSmem<128, kN>::kBytes, stream, pa));
  else
    GSA_TRY(d->d == 64 ? launch(k_prefill_score<kW, 64>, ps_grid, ps_block, PfSmem<64, kW>::kBytes, stream, pa)
                       : launch(k_prefill_score<kW, 128>, ps_grid, ps_block, PfSmem<128, kW>::kBytes, stream, pa));
  if (d->topk <= 0) return GSA_OK;
  // rows whose candidates overflowed: exact per-row selection (usually none)
  SelectRowsArgs sr;
  sr.q_raw = static_cast<const __nv_bfloat16 *>(q_raw);
  sr.k_gist = static_cast<const __nv_bfloat16 *>(k_gist);
  sr.rows = pa.ovf_rows;
  sr.count = pa.ovf_count;
  sr.done = pa.status + kPfOvfDoneWord;
  sr.group = pa.group;
  sr.chunk = d->chunk;
  sr.n_chunks = d->n_max;
  sr.L = d->t_max;
  sr.pos0 = pa.pos0;
  sr.topk = d->topk;
  sr.scale = pa.scale;
  sr.sel_idx = sel_idx;
  sr.sel_score = sel_score;
  sr.rec_raw = pa.rec_raw;
  sr.scale_log2 = pa.scale_log2;
  const int kmax = pf_wide(d) ? kW : kN;
  const size_t sel_smem = (static_cast<size_t>(d->n_max) + 128 + kmax) * 4;  // scores, query (<= 128), pick scores
  const dim3 sr_grid(sm_count()), sr_block(kSelThreads);
  if (!pf_wide(d))
    return d->d == 64 ? launch(k_prefill_select_rows<64, kN>, sr_grid, sr_block, sel_smem, stream, sr)
                      : launch(k_prefill_select_rows<128, kN>, sr_grid, sr_block, sel_smem, stream, sr);
  return d->d == 64 ? launch(k_prefill_select_rows<64, kW>, sr_grid, sr_block, sel_smem, stream, sr)
                    : launch(k_prefill_select_rows<128, kW>, sr_grid, sr_block, sel_smem, stream, sr);
}

gsa_status run_prefill_attend(const gsa_desc *d, const void *q_raw, const void *k_raw, const void *v_raw,
                              const void *q_gist, const void *k_gist, const void *v_gist, const int32_t *sel_idx,
                              const float *sel_score, void *out_raw, void *out_gist, const Layout &L, void *ws,
                              void *stream) {
  PrefillArgs pa = prefill_args(d, nullptr, nullptr, L, ws);
  const uint64_t bh = static_cast<uint64_t>(d->batch) * d->hq, bkv = static_cast<uint64_t>(d->batch) * d->hkv;
  void *vh = at(ws, L.pf_vh);
  const auto bf16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const uint64_t D = static_cast<uint64_t>(d->d);
  if (!map_rows(&pa.tm_qraw, q_raw, bh * d->t_max, kPfRows, bf16, D) ||
      !map_rows(&pa.tm_qgist, q_gist, bh * d->n_max, kPfRows, bf16, D) ||
      !map_rows(&pa.tm_kgist, k_gist, bkv * d->n_max, kGaKeys, bf16, D) ||
      !map_rows(&pa.tm_vgist, vh, bkv * d->n_max, kGaKeys, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, D))
    return GSA_ERR_CUDA;
  const size_t n8 = bkv * d->n_max * D / 8;
  GSA_TRY(launch(k_bf16_to_f16, dim3(static_cast<unsigned>(std::min<size_t>((n8 + 255) / 256, 4 * sm_count()))),
                 dim3(256), 0, stream, static_cast<const __nv_bfloat16 *>(v_gist), static_cast<__half *>(vh), n8));
  const int total = pa.bh * (pa.gist_tiles + pa.raw_tiles);
  const dim3 ga_grid(std::min(total, sm_count()));
  GSA_TRY(d->d == 64 ? launch(k_prefill_gist_attn<64>, ga_grid, dim3(kPfThreads), GaSmem<64>::kBytes, stream, pa)
                     : launch(k_prefill_gist_attn<128>, ga_grid, dim3(kPfThreads), GaSmem<128>::kBytes, stream, pa));
  GatherArgs ga;
  ga.q_raw = static_cast<const __nv_bfloat16 *>(q_raw);
  ga.k_raw = static_cast<const __nv_bfloat16 *>(k_raw);
  ga.v_raw = static_cast<const __nv_bfloat16 *>(v_raw);
  ga.q_gist = static_cast<const __nv_bfloat16 *>(q_gist);
  ga.v_gist = static_cast<const __nv_bfloat16 *>(v_gist);
  ga.sel_idx = sel_idx;
  ga.sel_score = sel_score;
  ga.rec_raw = pa.rec_raw;
  ga.rec_gist = pa.rec_gist;
  ga.bh = pa.bh;
  ga.hq = d->hq;
  ga.group = pa.group;
  ga.chunk = d->chunk;
  ga.n_chunks = d->n_max;
  ga.L = d->t_max;
  ga.topk = d->topk;
  ga.exclude = d->exclude_unselected;
  ga.scale_log2 = pa.scale_log2;
  ga.out_raw = out_raw;
  ga.out_gist = out_gist;
  ga.out_bf16 = d->out_dtype == GSA_BF16;
  const int64_t rows = static_cast<int64_t>(pa.bh) * (d->t_max + d->n_max);
  const dim3 g_grid(static_cast<unsigned>((rows + kGatherWarps - 1) / kGatherWarps));
  return d->d == 64 ? launch(k_prefill_gather<64>, g_grid, dim3(kGatherWarps * 32), 0, stream, ga)
                    : launch(k_prefill_gather<128>, g_grid, dim3(kGatherWarps * 32), 0, stream, ga);
}

// Number of partial records per row the scoring pass writes for these shapes.
int gist_prior_count(const gsa_desc *d) { return plan_score(d, d->n_max, true).splits; }

// The gist-position step runs the decode path with no selection over the
// full gist set (the compression mask has no unselected-gist choice).
gsa_desc gist_step_desc(const gsa_desc *d) {
  gsa_desc g = *d;
  g.topk = 0;
  g.exclude_unselected = 0;
  return g;
}

// Each (batch, kv head) pair is split into the same number of CTAs, chosen
// so the launch is about kBwdWaves full waves of resident CTAs.
template <int D, typename T, int GM>
gsa_status launch_bwd(const BackwardArgs &ba, int B, int hkv, size_t smem, void *stream) {
  const int slots = resident_ctas(k_decode_bwd<D, T, GM>, kBwdWarps * 32, smem);
  const int splits = clampi(kBwdWaves * slots / std::max(1, B * hkv), 1, 256);
  return launch(k_decode_bwd<D, T, GM>, dim3(splits, hkv, B), dim3(kBwdWarps * 32), smem, stream, ba);
}

}  // namespace
}  // namespace gsa

using namespace gsa;

extern "C" {

const char *gsa_status_string(int32_t s) {
  switch (s) {
    case GSA_OK: return "GSA_OK";
    case GSA_ERR_INVALID_ARG: return "GSA_ERR_INVALID_ARG: invalid argument";
    case GSA_ERR_UNSUPPORTED: return "GSA_ERR_UNSUPPORTED: configuration not supported";
    case GSA_ERR_WORKSPACE: return "GSA_ERR_WORKSPACE: workspace too small";
    case GSA_ERR_CUDA: return "GSA_ERR_CUDA: CUDA runtime error";
    case GSA_ERR_TIMEOUT: return "GSA_ERR_TIMEOUT: a bounded device wait expired";
    default: return "unknown gsa_status";
  }
}

int32_t gsa_version(void) { return 100; }

size_t gsa_workspace_bytes(const gsa_desc *desc, int32_t op, const gsa_hdesc *hdesc) {
  if (check_desc(desc) != GSA_OK) return 0;
  if (op != GSA_OP_DECODE && op != GSA_OP_HGSA && op != GSA_OP_PREFILL && op != GSA_OP_HGSA2 &&
      op != GSA_OP_GIST_STEP && op != GSA_OP_MULTIQUERY)
    return 0;
  if (op == GSA_OP_MULTIQUERY && check_multiquery(desc) != GSA_OK) return 0;
  if (op == GSA_OP_GIST_STEP) {
    const gsa_desc g = gist_step_desc(desc);
    return layout(&g, op, nullptr).total;
  }
  if (op == GSA_OP_HGSA && check_hdesc(desc, hdesc) != GSA_OK) return 0;
  if (op == GSA_OP_HGSA2 && (!hdesc || check_h2desc(desc, reinterpret_cast<const gsa_h2desc *>(hdesc)) != GSA_OK))
    return 0;
  return layout(desc, op, hdesc).total;
}

gsa_status gsa_workspace_init(void *ws, size_t ws_bytes, void *stream) {
  if (!ws || !ws_bytes) return GSA_ERR_INVALID_ARG;
  return cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream)) == cudaSuccess ? GSA_OK : GSA_ERR_CUDA;
}

gsa_status gsa_workspace_status(void *ws, size_t ws_bytes, void *stream, uint32_t *flags_out) {
  if (!ws || ws_bytes < 256 || !flags_out) return GSA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  if (cudaMemcpyAsync(&v, ws, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess) return GSA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return GSA_ERR_CUDA;
  if (cudaMemsetAsync(ws, 0, 4, s) != cudaSuccess) return GSA_ERR_CUDA;
  *flags_out = v;
  return (v & GSA_DEVERR_TIMEOUT) ? GSA_ERR_TIMEOUT : GSA_OK;
}

gsa_status gsa_score_gists(const gsa_desc *desc, const void *q, const void *gist_k, const void *gist_v,
                           const int32_t *n_gists, float *scores, void *ws, size_t ws_bytes, void *stream) {
  GSA_TRY(check_desc(desc));
  GSA_TRY(need_ptr(q));
  GSA_TRY(need_ptr(gist_k));
  GSA_TRY(need_ptr(n_gists));
  GSA_TRY(need_ptr(scores));
  GSA_TRY(need_ptr(ws));
  if (!desc->exclude_unselected) GSA_TRY(need_ptr(gist_v));
  const Layout L = layout(desc, GSA_OP_DECODE, nullptr);
  if (ws_bytes < L.total) return GSA_ERR_WORKSPACE;
  float *part = desc->exclude_unselected ? nullptr : reinterpret_cast<float *>(at(ws, L.part_g));
  return run_score(desc, q, gist_k, gist_v, n_gists, 1, desc->n_max, scores, desc->n_max, part, nullptr,
                   reinterpret_cast<uint32_t *>(at(ws, L.status)), stream);
}

gsa_status gsa_topk_select(const gsa_desc *desc, const float *scores, const int32_t *n_gists, int32_t *sel_idx,
                           float *sel_score, void *ws, size_t ws_bytes, void *stream) {
  GSA_TRY(check_desc(desc));
  GSA_TRY(need_ptr(scores));
  GSA_TRY(need_ptr(n_gists));
  GSA_TRY(need_ptr(sel_idx));
  GSA_TRY(opt_ptr(sel_score));
  GSA_TRY(need_ptr(ws));
  const Layout L = layout(desc, GSA_OP_DECODE, nullptr);
  if (ws_bytes < L.total) return GSA_ERR_WORKSPACE;
  if (desc->topk == 0) return GSA_OK;
  return run_topk(desc->batch * desc->hq, desc->hq, scores, desc->n_max, n_gists, 1, nullptr, desc->topk, nullptr,
                  sel_idx, sel_score, reinterpret_cast<uint32_t *>(at(ws, L.counters)), stream,
                  reinterpret_cast<uint32_t *>(at(ws, L.status)));
}

gsa_status gsa_topp_select(const gsa_desc *desc, const float *scores, const int32_t *n_gists, float top_p,
                           int32_t *sel_idx, float *sel_score, int32_t *sel_count, void *ws, size_t ws_bytes,
                           void *stream) {
  GSA_TRY(check_desc(desc));
  GSA_TRY(need_ptr(scores));
  GSA_TRY(need_ptr(n_gists));
  GSA_TRY(need_ptr(sel_idx));
  GSA_TRY(opt_ptr(sel_score));
  GSA_TRY(opt_ptr(sel_count));
  GSA_TRY(need_ptr(ws));
  if (!(top_p == top_p)) return GSA_ERR_INVALID_ARG;  // NaN
  if (desc->topk < 1) return GSA_ERR_INVALID_ARG;
  if (desc->topk > kToppMaxK || desc->n_max > 64 * kTopkRegThreads) return GSA_ERR_UNSUPPORTED;
  const Layout L = layout(desc, GSA_OP_DECODE, nullptr);
  if (ws_bytes < L.total) return GSA_ERR_WORKSPACE;
  ToppArgs ta;
  ta.scores = scores;
  ta.stride = desc->n_max;
  ta.n_gists = n_gists;
  ta.hq = desc->hq;
  ta.k = desc->topk;
  ta.top_p = top_p;
  ta.sel_idx = sel_idx;
  ta.sel_score = sel_score;
  ta.sel_count = sel_count;
  ta.counters = reinterpret_cast<uint32_t *>(at(ws, L.counters));
  const dim3 grid(desc->batch * desc->hq), block(kTopkRegThreads);
  // the staged row, then one bit per entry for the exact tie path
  auto smem = [](int kpt) { return static_cast<size_t>(kpt) * kTopkRegThreads * 4 + kpt * kTopkRegThreads / 8; };
  const int stride = desc->n_max;
  if (stride <= 4 * kTopkRegThreads) return launch(k_topp<4>, grid, block, smem(4), stream, ta);
  if (stride <= 16 * kTopkRegThreads) return launch(k_topp<16>, grid, block, smem(16), stream, ta);
  if (stride <= 32 * kTopkRegThreads) return launch(k_topp<32>, grid, block, smem(32), stream, ta);
  return launch(k_topp<64>, grid, block, smem(64), stream, ta);
}

gsa_status gsa_unfold_attend(const gsa_desc *desc, const void *q, const void *raw_k, const void *raw_v,
                             const void *gist_v, const int32_t *n_gists, const int32_t *own_len,
                             const int32_t *sel_idx, const float *sel_score, int32_t prior, void *out, float *lse,
                             void *ws, size_t ws_bytes, void *stream) {
  GSA_TRY(check_desc(desc));
  GSA_TRY(need_ptr(q));
  GSA_TRY(need_ptr(raw_k));
  GSA_TRY(need_ptr(raw_v));
  GSA_TRY(need_ptr(n_gists));
  GSA_TRY(need_ptr(own_len));
  GSA_TRY(need_ptr(out));
  GSA_TRY(opt_ptr(lse));
  GSA_TRY(need_ptr(ws));
  if (desc->topk > 0) GSA_TRY(need_ptr(sel_idx));
  if (desc->exclude_unselected && desc->topk > 0) {
    GSA_TRY(need_ptr(gist_v));
    GSA_TRY(need_ptr(sel_score));
  }
  if (prior != GSA_PRIOR_NONE && prior != GSA_PRIOR_GISTS && prior != GSA_PRIOR_HGSA && prior != GSA_PRIOR_HGSA2)
    return GSA_ERR_INVALID_ARG;
  if (prior == GSA_PRIOR_NONE && !desc->exclude_unselected) return GSA_ERR_INVALID_ARG;
  const Layout L = layout(desc, GSA_OP_DECODE, nullptr);  // the H-GSA layout extends this one
  if (ws_bytes < L.total) return GSA_ERR_WORKSPACE;
  // The counters must be zero; gsa_topk_select re-arms them, a standalone
  // call re-arms them here.
  if (cudaMemsetAsync(at(ws, L.counters), 0, static_cast<size_t>(desc->batch) * desc->hq * 4,
                      static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return GSA_ERR_CUDA;
  const float *pr = nullptr;
  int n_prior = 0;
  if (prior == GSA_PRIOR_GISTS && !desc->exclude_unselected) {
    pr = reinterpret_cast<const float *>(at(ws, L.part_g));
    n_prior = gist_prior_count(desc);
  } else if (prior == GSA_PRIOR_HGSA && !desc->exclude_unselected) {
    pr = reinterpret_cast<const float *>(at(ws, L.part_g));
    n_prior = hgsa_splits(desc);
  } else if (prior == GSA_PRIOR_HGSA2 && !desc->exclude_unselected) {
    pr = reinterpret_cast<const float *>(at(ws, L.part_g));
    n_prior = 2 * hgsa_splits(desc);
  }
  return run_unfold(desc, q, raw_k, raw_v, gist_v, n_gists, own_len, sel_idx, sel_score, pr, n_prior, out, lse, L,
                    ws, stream);
}

gsa_status gsa_decode(const gsa_desc *desc, const void *q, const void *gist_k, const void *gist_v, const void *raw_k,
                      const void *raw_v, const int32_t *n_gists, const int32_t *own_len, void *out, float *lse,
                      int32_t *sel_idx, float *sel_score, void *ws, size_t ws_bytes, void *stream) {
  GSA_TRY(check_desc(desc));
  GSA_TRY(need_ptr(q));
  GSA_TRY(need_ptr(gist_k));
  GSA_TRY(need_ptr(gist_v));
  GSA_TRY(need_ptr(raw_k));
  GSA_TRY(need_ptr(raw_v));
  GSA_TRY(need_ptr(n_gists));
  GSA_TRY(need_ptr(own_len));
  GSA_TRY(need_ptr(out));
  GSA_TRY(opt_ptr(lse));
  GSA_TRY(opt_ptr(sel_idx));
  GSA_TRY(opt_ptr(sel_score));
  GSA_TRY(need_ptr(ws));
  const Layout L = layout(desc, GSA_OP_DECODE, nullptr);
  if (ws_bytes < L.total) return GSA_ERR_WORKSPACE;
  uint32_t *status = reinterpret_cast<uint32_t *>(at(ws, L.status));
  float *scores = reinterpret_cast<float *>(at(ws, L.scores));
  int32_t *si = sel_idx ? sel_idx : reinterpret_cast<int32_t *>(at(ws, L.sel_idx));
  float *ss = sel_score ? sel_score : reinterpret_cast<float *>(at(ws, L.sel_score));
  float *part = desc->exclude_unselected ? nullptr : reinterpret_cast<float *>(at(ws, L.part_g));
  int n_prior = 0;
  if (tail_select_ok(desc)) {
    // Two launches: scoring with the selection in its tail (it also re-arms
    // the unfold's counters), then the unfold, whose CTAs take the rows as
    // the tail publishes them in the ready list.
    uint32_t *ready = reinterpret_cast<uint32_t *>(at(ws, L.ready));
    GSA_TRY(run_score(desc, q, gist_k, gist_v, n_gists, 1, desc->n_max, scores, desc->n_max, part, &n_prior, status,
                      stream, reinterpret_cast<uint32_t *>(at(ws, L.counters)),
                      reinterpret_cast<uint32_t *>(at(ws, L.unit_counters)), si, ss, ready));
    return run_unfold(desc, q, raw_k, raw_v, gist_v, n_gists, own_len, si, ss, part, part ? n_prior : 0, out, lse, L,
                      ws, stream, ready);
  }
  GSA_TRY(run_score(desc, q, gist_k, gist_v, n_gists, 1, desc->n_max, scores, desc->n_max, part, &n_prior, status,
                    stream));
  if (desc->topk > 0) {
    GSA_TRY(run_topk(desc->batch * desc->hq, desc->hq, scores, desc->n_max, n_gists, 1, nullptr, desc->topk, nullptr,
                     si, ss, reinterpret_cast<uint32_t *>(at(ws, L.counters)), stream));
  } else if (cudaMemsetAsync(at(ws, L.counters), 0, static_cast<size_t>(desc->batch) * desc->hq * 4,
                             static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    return GSA_ERR_CUDA;
  }
  return run_unfold(desc, q, raw_k, raw_v, gist_v, n_gists, own_len, si, ss, part, part ? n_prior : 0, out, lse, L,
                    ws, stream);
}

gsa_status gsa_score_select(const gsa_desc *desc, const void *q, const void *gist_k, const void *gist_v,
                            const int32_t *n_gists, float *scores, int32_t *sel_idx, float *sel_score, void *ws,
                            size_t ws_bytes, void *stream) {
  GSA_TRY(check_desc(desc));
  if (desc->dtype != GSA_BF16) return GSA_ERR_UNSUPPORTED;
  GSA_TRY(need_ptr(q));
  GSA_TRY(need_ptr(gist_k));
  GSA_TRY(need_ptr(n_gists));
  GSA_TRY(opt_ptr(scores));
  GSA_TRY(opt_ptr(sel_idx));
  GSA_TRY(opt_ptr(sel_score));
  GSA_TRY(need_ptr(ws));
  if (!desc->exclude_unselected) GSA_TRY(need_ptr(gist_v));
  const Layout L = layout(desc, GSA_OP_DECODE, nullptr);
  if (ws_bytes < L.total) return GSA_ERR_WORKSPACE;
  float *sc = scores ? scores : reinterpret_cast<float *>(at(ws, L.scores));
  int32_t *si = sel_idx ? sel_idx : reinterpret_cast<int32_t *>(at(ws, L.sel_idx));
  float *ss = sel_score ? sel_score : reinterpret_cast<float *>(at(ws, L.sel_score));
  float *part = desc->exclude_unselected ? nullptr : reinterpret_cast<float *>(at(ws, L.part_g));
  uint32_t *status = reinterpret_cast<uint32_t *>(at(ws, L.status));
  if (!tail_select_ok(desc)) {  // rows too long for the tail: the separate selection kernel
    GSA_TRY(run_score(desc, q, gist_k, gist_v, n_gists, 1, desc->n_max, sc, desc->n_max, part, nullptr, status,
                      stream));
    if (desc->topk == 0) return GSA_OK;
    return run_topk(desc->batch * desc->hq, desc->hq, sc, desc->n_max, n_gists, 1, nullptr, desc->topk, nullptr, si,
                    ss, reinterpret_cast<uint32_t *>(at(ws, L.counters)), stream);
  }
  return run_score(desc, q, gist_k, gist_v, n_gists, 1, desc->n_max, sc, desc->n_max, part, nullptr, status, stream,
                   reinterpret_cast<uint32_t *>(at(ws, L.counters)),
                   reinterpret_cast<uint32_t *>(at(ws, L.unit_counters)), si, ss);
}

gsa_status hgsa_select(const gsa_desc *desc, const gsa_hdesc *hdesc, const void *q, const void *meta_k,
                       const void *meta_v, const void *gist_k, const void *gist_v, const int32_t *n_gists,
                       int32_t *meta_idx, int32_t *sel_idx, float *sel_score, void *ws, size_t ws_bytes,
                       void *stream) {
  GSA_TRY(check_desc(desc));
  GSA_TRY(check_hdesc(desc, hdesc));
  GSA_TRY(need_ptr(q));
  GSA_TRY(need_ptr(meta_k));
  GSA_TRY(need_ptr(gist_k));
  GSA_TRY(need_ptr(n_gists));
  GSA_TRY(need_ptr(meta_idx));
  GSA_TRY(need_ptr(ws));
  if (desc->topk > 0) {
    GSA_TRY(need_ptr(sel_idx));
    GSA_TRY(need_ptr(sel_score));
  }
  if (!desc->exclude_unselected) {
    GSA_TRY(need_ptr(meta_v));
    GSA_TRY(need_ptr(gist_v));
  }
  const Layout L = layout(desc, GSA_OP_HGSA, hdesc);
  if (ws_bytes < L.total) return GSA_ERR_WORKSPACE;
  return run_hgsa_select(desc, hdesc, q, meta_k, meta_v, gist_k, gist_v, n_gists, meta_idx, sel_idx, sel_score, L,
                         ws, stream);
}

gsa_status hgsa_decode(const gsa_desc *desc, const gsa_hdesc *hdesc, const void *q, const void *meta_k,
                       const void *meta_v, const void *gist_k, const void *gist_v, const void *raw_k,
                       const void *raw_v, const int32_t *n_gists, const int32_t *own_len, void *out, float *lse,
                       int32_t *meta_idx, int32_t *sel_idx, float *sel_score, void *ws, size_t ws_bytes,
                       void *stream) {
  GSA_TRY(check_desc(desc));
  GSA_TRY(check_hdesc(desc, hdesc));
  GSA_TRY(need_ptr(q));
  GSA_TRY(need_ptr(meta_k));
  GSA_TRY(need_ptr(meta_v));
  GSA_TRY(need_ptr(gist_k));
  GSA_TRY(need_ptr(gist_v));
  GSA_TRY(need_ptr(raw_k));
  GSA_TRY(need_ptr(raw_v));
  GSA_TRY(need_ptr(n_gists));
  GSA_TRY(need_ptr(own_len));
  GSA_TRY(need_ptr(out));
  GSA_TRY(opt_ptr(lse));
  GSA_TRY(opt_ptr(meta_idx));
  GSA_TRY(opt_ptr(sel_idx));
  GSA_TRY(opt_ptr(sel_score));
  GSA_TRY(need_ptr(ws));
  const Layout L = layout(desc, GSA_OP_HGSA, hdesc);
  if (ws_bytes < L.total) return GSA_ERR_WORKSPACE;
  int32_t *mi = meta_idx ? meta_idx : reinterpret_cast<int32_t *>(at(ws, L.meta_idx));
  int32_t *si = sel_idx ? sel_idx : reinterpret_cast<int32_t *>(at(ws, L.sel_idx));
  float *ss = sel_score ? sel_score : reinterpret_cast<float *>(at(ws, L.sel_score));
  GSA_TRY(run_hgsa_select(desc, hdesc, q, meta_k, meta_v, gist_k, gist_v, n_gists, mi, si, ss, L, ws, stream));
  const float *pr = desc->exclude_unselected ? nullptr : reinterpret_cast<const float *>(at(ws, L.part_g));
  return run_unfold(desc, q, raw_k, raw_v, gist_v, n_gists, own_len, si, ss, pr, pr ? hgsa_splits(desc) : 0, out, lse,
                    L, ws, stream);
}

gsa_status gsa_decode_backward(const gsa_desc *desc, const void *q, const void *gist_k, const void *gist_v,
                               const void *raw_k, const void *raw_v, const int32_t *n_gists, const int32_t *own_len,
                               const int32_t *sel_idx, const float *out, const float *lse, const float *d_out,
                               float *d_q, float *d_gist_k, float *d_gist_v, float *d_raw_k, float *d_raw_v,
                               void *stream) {
  GSA_TRY(check_desc(desc));
  for (const void *p : {q, gist_k, gist_v, raw_k, raw_v, static_cast<const void *>(n_gists),
                        static_cast<const void *>(own_len), static_cast<const void *>(out),
                        static_cast<const void *>(lse), static_cast<const void *>(d_out), static_cast<const void *>(d_q),
                        static_cast<const void *>(d_gist_k), static_cast<const void *>(d_gist_v),
                        static_cast<const void *>(d_raw_k), static_cast<const void *>(d_raw_v)})
    GSA_TRY(need_ptr(p));
  if (desc->topk > 0) GSA_TRY(need_ptr(sel_idx));
  BackwardArgs ba;
  ba.q = q;
  ba.gist_k = gist_k;
  ba.gist_v = gist_v;
  ba.raw_k = raw_k;
  ba.raw_v = raw_v;
  ba.n_gists = n_gists;
  ba.own_len = own_len;
  ba.sel_idx = sel_idx;
  ba.k = desc->topk;
  ba.out = out;
  ba.lse = lse;
  ba.d_out = d_out;
  ba.d_q = d_q;
  ba.d_gist_k = d_gist_k;
  ba.d_gist_v = d_gist_v;
  ba.d_raw_k = d_raw_k;
  ba.d_raw_v = d_raw_v;
  ba.hq = desc->hq;
  ba.hkv = desc->hkv;
  ba.group = desc->hq / desc->hkv;
  ba.chunk = desc->chunk;
  ba.n_max = desc->n_max;
  ba.t_max = desc->t_max;
  ba.exclude = desc->exclude_unselected;
  ba.scale = resolve_scale(desc);
  const size_t smem = bwd_smem_bytes(ba.group, desc->d, ba.k);
  const bool bf = desc->dtype == GSA_BF16;
  const int gm = ba.group <= 4 ? 4 : (ba.group <= 8 ? 8 : 16);
  const int B = desc->batch, hkv = desc->hkv;
#define GSA_BWD_LAUNCH(D_, T_)                                                    \
  return gm == 4   ? launch_bwd<D_, T_, 4>(ba, B, hkv, smem, stream)              \
         : gm == 8 ? launch_bwd<D_, T_, 8>(ba, B, hkv, smem, stream)              \
                   : launch_bwd<D_, T_, 16>(ba, B, hkv, smem, stream)
  if (desc->d == 64) {
    if (bf) GSA_BWD_LAUNCH(64, __nv_bfloat16);
    GSA_BWD_LAUNCH(64, float);
  }
  if (bf) GSA_BWD_LAUNCH(128, __nv_bfloat16);
  GSA_BWD_LAUNCH(128, float);
#undef GSA_BWD_LAUNCH
}

gsa_status gsa_gist_step(const gsa_desc *desc, const void *q, const void *k_new, const void *v_new, void *gist_k,
                         void *gist_v, const void *raw_k, const void *raw_v, int32_t *n_gists, int32_t *own_len,
                         void *out, float *lse, void *ws, size_t ws_bytes, void *stream) {
  GSA_TRY(check_desc(desc));
  for (const void *p : {q, k_new, v_new, static_cast<const void *>(gist_k), static_cast<const void *>(gist_v), raw_k,
                        raw_v, static_cast<const void *>(n_gists), static_cast<const void *>(own_len),
                        static_cast<const void *>(out), static_cast<const void *>(ws)})
    GSA_TRY(need_ptr(p));
  GSA_TRY(opt_ptr(lse));
  const gsa_desc g = gist_step_desc(desc);
  const Layout L = layout(&g, GSA_OP_GIST_STEP, nullptr);
  if (ws_bytes < L.total) return GSA_ERR_WORKSPACE;
  uint32_t *status = reinterpret_cast<uint32_t *>(at(ws, L.status));
  int32_t *n_cur = reinterpret_cast<int32_t *>(at(ws, L.gs_cur));
  int32_t *n_plus = reinterpret_cast<int32_t *>(at(ws, L.gs_plus));
  GistAppendArgs ga;
  ga.k_new = static_cast<const uint4 *>(k_new);
  ga.v_new = static_cast<const uint4 *>(v_new);
  ga.gist_k = static_cast<uint4 *>(gist_k);
  ga.gist_v = static_cast<uint4 *>(gist_v);
  ga.n_gists = n_gists;
  ga.n_cur = n_cur;
  ga.n_plus = n_plus;
  ga.hkv = g.hkv;
  ga.n_max = g.n_max;
  ga.row_vecs = static_cast<int32_t>(static_cast<size_t>(g.d) * elem_size(g.dtype) / 16);
  ga.status = status;
  // 1. the new gist joins the gist arrays at row N (counted as N+1 by the scoring pass)
  GSA_TRY(launch(k_gist_append, dim3(g.hkv, g.batch), dim3(32), 0, stream, ga));
  // 2. the compression-mask attention: gists 0..N through the scoring pass's
  //    partial, chunk N's raw rows through the unfold (no selected chunk)
  float *scores = reinterpret_cast<float *>(at(ws, L.scores));
  float *part = reinterpret_cast<float *>(at(ws, L.part_g));
  int n_prior = 0;
  GSA_TRY(run_score(&g, q, gist_k, gist_v, n_plus, 1, g.n_max, scores, g.n_max, part, &n_prior, status, stream));
  if (cudaMemsetAsync(at(ws, L.counters), 0, static_cast<size_t>(g.batch) * g.hq * 4,
                      static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return GSA_ERR_CUDA;
  GSA_TRY(run_unfold(&g, q, raw_k, raw_v, gist_v, n_cur, own_len, reinterpret_cast<int32_t *>(at(ws, L.sel_idx)),
                     reinterpret_cast<float *>(at(ws, L.sel_score)), part, n_prior, out, lse, L, ws, stream));
  // 3. chunk completion: n_gists = N+1, own_len = 0
  return launch(k_gist_commit, dim3(cdiv(g.batch, 128)), dim3(128), 0, stream, static_cast<const int32_t *>(n_cur),
                static_cast<const int32_t *>(n_plus), n_gists, own_len, static_cast<int>(g.batch));
}

gsa_status hgsa2_select(const gsa_desc *desc, const gsa_h2desc *h2desc, const void *q, const void *meta2_k,
                        const void *meta2_v, const void *meta_k, const void *meta_v, const void *gist_k,
                        const void *gist_v, const int32_t *n_gists, int32_t *meta2_idx, int32_t *meta_idx,
                        int32_t *sel_idx, float *sel_score, void *ws, size_t ws_bytes, void *stream) {
  GSA_TRY(check_desc(desc));
  GSA_TRY(check_h2desc(desc, h2desc));
  GSA_TRY(need_ptr(q));
  GSA_TRY(need_ptr(meta2_k));
  GSA_TRY(need_ptr(meta_k));
  GSA_TRY(need_ptr(gist_k));
  GSA_TRY(need_ptr(n_gists));
  GSA_TRY(need_ptr(meta2_idx));
  GSA_TRY(need_ptr(meta_idx));
  GSA_TRY(need_ptr(ws));
  if (desc->topk > 0) {
    GSA_TRY(need_ptr(sel_idx));
    GSA_TRY(need_ptr(sel_score));
  }
  if (!desc->exclude_unselected) {
    GSA_TRY(need_ptr(meta2_v));
    GSA_TRY(need_ptr(meta_v));
    GSA_TRY(need_ptr(gist_v));
  }
  const Layout L = layout(desc, GSA_OP_HGSA2, &h2desc->level1);
  if (ws_bytes < L.total) return GSA_ERR_WORKSPACE;
  return run_hgsa2_select(desc, h2desc, q, meta2_k, meta2_v, meta_k, meta_v, gist_k, gist_v, n_gists, meta2_idx,
                          meta_idx, sel_idx, sel_score, L, ws, stream);
}

gsa_status hgsa2_decode(const gsa_desc *desc, const gsa_h2desc *h2desc, const void *q, const void *meta2_k,
                        const void *meta2_v, const void *meta_k, const void *meta_v, const void *gist_k,
                        const void *gist_v, const void *raw_k, const void *raw_v, const int32_t *n_gists,
                        const int32_t *own_len, void *out, float *lse, int32_t *meta2_idx, int32_t *meta_idx,
                        int32_t *sel_idx, float *sel_score, void *ws, size_t ws_bytes, void *stream) {
  GSA_TRY(check_desc(desc));
  GSA_TRY(check_h2desc(desc, h2desc));
  GSA_TRY(need_ptr(q));
  GSA_TRY(need_ptr(meta2_k));
  GSA_TRY(need_ptr(meta2_v));
  GSA_TRY(need_ptr(meta_k));
  GSA_TRY(need_ptr(meta_v));
  GSA_TRY(need_ptr(gist_k));
  GSA_TRY(need_ptr(gist_v));
  GSA_TRY(need_ptr(raw_k));
  GSA_TRY(need_ptr(raw_v));
  GSA_TRY(need_ptr(n_gists));
  GSA_TRY(need_ptr(own_len));
  GSA_TRY(need_ptr(out));
  GSA_TRY(opt_ptr(lse));
  GSA_TRY(opt_ptr(meta2_idx));
  GSA_TRY(opt_ptr(meta_idx));
  GSA_TRY(opt_ptr(sel_idx));
  GSA_TRY(opt_ptr(sel_score));
  GSA_TRY(need_ptr(ws));
  const Layout L = layout(desc, GSA_OP_HGSA2, &h2desc->level1);
  if (ws_bytes < L.total) return GSA_ERR_WORKSPACE;
  int32_t *m2 = meta2_idx ? meta2_idx : reinterpret_cast<int32_t *>(at(ws, L.meta2_idx));
  int32_t *mi = meta_idx ? meta_idx : reinterpret_cast<int32_t *>(at(ws, L.meta_idx));
  int32_t *si = sel_idx ? sel_idx : reinterpret_cast<int32_t *>(at(ws, L.sel_idx));
  float *ss = sel_score ? sel_score : reinterpret_cast<float *>(at(ws, L.sel_score));
  GSA_TRY(run_hgsa2_select(desc, h2desc, q, meta2_k, meta2_v, meta_k, meta_v, gist_k, gist_v, n_gists, m2, mi, si,
                           ss, L, ws, stream));
  const float *pr = desc->exclude_unselected ? nullptr : reinterpret_cast<const float *>(at(ws, L.part_g));
  return run_unfold(desc, q, raw_k, raw_v, gist_v, n_gists, own_len, si, ss, pr, pr ? 2 * hgsa_splits(desc) : 0,
                    out, lse, L, ws, stream);
}

gsa_status gsa_prefill_score(const gsa_desc *desc, const void *q_raw, const void *q_gist, const void *k_gist,
                             int32_t *sel_idx, float *sel_score, void *ws, size_t ws_bytes, void *stream) {
  GSA_TRY(check_prefill(desc));
  GSA_TRY(need_ptr(q_raw));
  GSA_TRY(need_ptr(q_gist));
  GSA_TRY(need_ptr(k_gist));
  GSA_TRY(need_ptr(ws));
  if (desc->topk > 0) {
    GSA_TRY(need_ptr(sel_idx));
    GSA_TRY(need_ptr(sel_score));
  }
  const Layout L = layout(desc, GSA_OP_PREFILL, nullptr);
  if (ws_bytes < L.total) return GSA_ERR_WORKSPACE;
  return run_prefill_score(desc, q_raw, q_gist, k_gist, sel_idx, sel_score, L, ws, stream);
}

gsa_status gsa_multiquery_select(const gsa_desc *desc, const void *q, const void *gist_k, int32_t *sel_idx,
                                 float *sel_score, void *ws, size_t ws_bytes, void *stream) {
  GSA_TRY(check_multiquery(desc));
  for (const void *p : {q, gist_k, static_cast<const void *>(sel_idx), static_cast<const void *>(sel_score),
                        static_cast<const void *>(ws)})
    GSA_TRY(need_ptr(p));
  const Layout L = layout(desc, GSA_OP_MULTIQUERY, nullptr);
  if (ws_bytes < L.total) return GSA_ERR_WORKSPACE;
  // the queries are raw rows of a one-token-per-chunk stream placed after
  // the N gists, so each sees all of them: chunk = 1, causal offset N
  gsa_desc m = *desc;
  m.chunk = 1;
  return run_prefill_score(&m, q, q, gist_k, sel_idx, sel_score, L, ws, stream, m.n_max);
}

gsa_status gsa_prefill_attend(const gsa_desc *desc, const void *q_raw, const void *k_raw, const void *v_raw,
                              const void *q_gist, const void *k_gist, const void *v_gist, const int32_t *sel_idx,
                              const float *sel_score, void *out_raw, void *out_gist, void *ws, size_t ws_bytes,
                              void *stream) {
  GSA_TRY(check_prefill(desc));
  GSA_TRY(need_ptr(q_raw));
  GSA_TRY(need_ptr(k_raw));
  GSA_TRY(need_ptr(v_raw));
  GSA_TRY(need_ptr(q_gist));
  GSA_TRY(need_ptr(k_gist));
  GSA_TRY(need_ptr(v_gist));
  GSA_TRY(need_ptr(out_raw));
  GSA_TRY(need_ptr(out_gist));
  GSA_TRY(need_ptr(ws));
  if (desc->topk > 0) {
    GSA_TRY(need_ptr(sel_idx));
    GSA_TRY(need_ptr(sel_score));
  }
  const Layout L = layout(desc, GSA_OP_PREFILL, nullptr);
  if (ws_bytes < L.total) return GSA_ERR_WORKSPACE;
  return run_prefill_attend(desc, q_raw, k_raw, v_raw, q_gist, k_gist, v_gist, sel_idx, sel_score, out_raw, out_gist,
                            L, ws, stream);
}

gsa_status gsa_prefill(const gsa_desc *desc, const void *q_raw, const void *k_raw, const void *v_raw,
                       const void *q_gist, const void *k_gist, const void *v_gist, int32_t *sel_idx,
                       float *sel_score, void *out_raw, void *out_gist, void *ws, size_t ws_bytes, void *stream) {
  GSA_TRY(check_prefill(desc));
  GSA_TRY(opt_ptr(sel_idx));
  GSA_TRY(opt_ptr(sel_score));
  GSA_TRY(need_ptr(ws));
  const Layout L = layout(desc, GSA_OP_PREFILL, nullptr);
  if (ws_bytes < L.total) return GSA_ERR_WORKSPACE;
  int32_t *si = sel_idx ? sel_idx : reinterpret_cast<int32_t *>(at(ws, L.sel_idx));
  float *ss = sel_score ? sel_score : reinterpret_cast<float *>(at(ws, L.sel_score));
  GSA_TRY(gsa_prefill_score(desc, q_raw, q_gist, k_gist, si, ss, ws, ws_bytes, stream));
  return gsa_prefill_attend(desc, q_raw, k_raw, v_raw, q_gist, k_gist, v_gist, si, ss, out_raw, out_gist, ws, ws_bytes,
                            stream);
}

}  // extern "C"

// ---- Scratch-free decode (gsa_decode_noalloc) ------------------------------
// For callers that cannot allocate device memory: the workspace gsa_decode
// needs lives in a file-scope device array instead of a caller buffer.
#include <mutex>

namespace gsa {
namespace {

__device__ __align__(256) uint8_t g_noalloc_scratch[GSA_NOALLOC_SCRATCH_BYTES];

struct NoallocSlot {
  std::once_flag once;
  void *ptr = nullptr;
  cudaError_t err = cudaSuccess;
};
constexpr int kNoallocMaxDevices = 64;
NoallocSlot g_noalloc_slots[kNoallocMaxDevices];

// Device address of g_noalloc_scratch on the current device.  In host code
// the array's name is only a stand-in; the real address is looked up once
// per device, with that device current.
gsa_status noalloc_scratch(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return GSA_ERR_CUDA;
  if (dev < 0 || dev >= kNoallocMaxDevices) return GSA_ERR_UNSUPPORTED;
  NoallocSlot &s = g_noalloc_slots[dev];
  std::call_once(s.once, [&s] { s.err = cudaGetSymbolAddress(&s.ptr, g_noalloc_scratch); });
  if (s.err != cudaSuccess || s.ptr == nullptr) return GSA_ERR_CUDA;
  *out = s.ptr;
  return GSA_OK;
}

}  // namespace
}  // namespace gsa

extern "C" gsa_status gsa_decode_noalloc(const gsa_desc *desc, const void *q, const void *gist_k, const void *gist_v,
                                         const void *raw_k, const void *raw_v, const int32_t *n_gists,
                                         const int32_t *own_len, void *out, float *lse, int32_t *sel_idx,
                                         float *sel_score, void *stream) {
  GSA_TRY(check_desc(desc));
  const Layout L = layout(desc, GSA_OP_DECODE, nullptr);
  if (L.total > GSA_NOALLOC_SCRATCH_BYTES) return GSA_ERR_WORKSPACE;
  GSA_TRY(need_ptr(q));
  GSA_TRY(need_ptr(gist_k));
  GSA_TRY(need_ptr(gist_v));
  GSA_TRY(need_ptr(raw_k));
  GSA_TRY(need_ptr(raw_v));
  GSA_TRY(need_ptr(n_gists));
  GSA_TRY(need_ptr(own_len));
  GSA_TRY(need_ptr(out));
  GSA_TRY(opt_ptr(lse));
  GSA_TRY(opt_ptr(sel_idx));
  GSA_TRY(opt_ptr(sel_score));
  void *ws = nullptr;
  GSA_TRY(noalloc_scratch(&ws));
  // The status word and the per-row and per-group counters must start at
  // zero; the array keeps whatever the previous call (of any shape) left.
  const size_t zero_bytes = L.ready + (static_cast<size_t>(desc->batch) * desc->hq + 4) * 4;
  if (cudaMemsetAsync(ws, 0, zero_bytes, static_cast<cudaStream_t>(stream)) != cudaSuccess) return GSA_ERR_CUDA;
  return gsa_decode(desc, q, gist_k, gist_v, raw_k, raw_v, n_gists, own_len, out, lse, sel_idx, sel_score, ws,
                    GSA_NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" gsa_status gsa_noalloc_status(void *stream, uint32_t *flags_out) {
  if (!flags_out) return GSA_ERR_INVALID_ARG;
  void *ws = nullptr;
  GSA_TRY(noalloc_scratch(&ws));
  // The status word is word 0 of the array (the decode layout starts there);
  // reading it needs no allocation, only a copy into the caller's variable.
  return gsa_workspace_status(ws, GSA_NOALLOC_SCRATCH_BYTES, stream, flags_out);
}
