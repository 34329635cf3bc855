// k_backward.cuh -- backward of the decode attention for a fixed selection.
//
// Selective finetuning trains through this path (gist.science/ja/paper/
// 2604.20920 sections 2.1 and 3: the gist tokens are learned end to end
// with selective unfolding in place).  The top-k choice is piecewise
// constant, so no gradient flows through the selection scores; the
// attention over the attended set (the SG+SR rule of the forward) is
// differentiated exactly.  With w = softmax(z), z_u = scale q.k_u,
// o = sum_u w_u v_u and g = dL/do:
//   dL/dv_u = w_u g,   dL/dz_u = w_u (g.v_u - g.o),
//   dL/dq = scale sum_u dL/dz_u k_u,   dL/dk_u = scale dL/dz_u q.
// The weights come back from the forward's log-sum-exp, g.o from its output.
//
// One CTA set per (batch, kv head) holds the q and g rows of all query heads
// of the GQA group in shared memory and splits two token lists:
//   shared  -- rows every head of the group attends: all gists (default
//              set) and the own rows.  A lane group takes one such row, sums
//              the dk / dv contributions of all heads in registers and adds
//              them to the gradient row with a plain load-add-store: no other
//              CTA touches that row, so no atomics (this is most of the
//              traffic in the default set).
//   per-head -- the rows one head attends through its own selection: the
//              selected chunks' raw rows (and, with exclude, their gists).
//              Heads of a group may select the same chunk, so these rows
//              are added with vector atomics.
// dq is kept per head in registers (shared list) or flushed to shared memory
// when a lane moves to the next head (per-head list), then added to d_q with
// one vector atomic per 4 elements per CTA.  A chunk listed twice in one
// head's selection is counted twice (the selection calls never list one
// twice).
#pragma once

#include "common.cuh"

namespace gsa {

struct BackwardArgs {
  const void *q;                  // [B, hq, D]
  const void *gist_k, *gist_v;    // [B, hkv, n_max, D]
  const void *raw_k, *raw_v;      // [B, hkv, t_max, D]
  const int32_t *n_gists, *own_len;
  const int32_t *sel_idx;         // [B*hq, k] (negative / >= N entries skipped)
  int32_t k;
  const float *out, *lse, *d_out; // [B*hq, D], [B*hq], [B*hq, D]
  float *d_q;                     // [B*hq, D] accumulated
  float *d_gist_k, *d_gist_v;     // accumulated
  float *d_raw_k, *d_raw_v;       // accumulated
  int32_t hq, hkv, group, chunk, n_max, t_max, exclude;
  float scale;
};

constexpr int kBwdWarps = 4;
constexpr int kBwdWaves = 4;  // CTAs per launch: about this many full waves
// Shared-list tokens per lane group per pass: two for groups of up to 4
// heads; larger groups hold more per-head dq registers, and two tokens would
// cost a resident CTA per SM (measured slower on the 7-head Qwen shape).
template <int GM>
constexpr int bwd_unroll() { return GM <= 4 ? 2 : 1; }

// Dynamic shared memory of k_decode_bwd for a group of G heads, D wide, k
// selections per head.
__host__ __device__ constexpr size_t bwd_smem_bytes(int G, int D, int k) {
  return static_cast<size_t>(3 * G * D + 2 * G) * 4 + static_cast<size_t>(2 * G + 1) * 4 +
         static_cast<size_t>(G) * k * 4;
}

__device__ __forceinline__ void red_add4(float *p, float a, float b, float c, float d) {
  atomicAdd(reinterpret_cast<float4 *>(p), make_float4(a, b, c, d));
}

__device__ __forceinline__ float elem_f32(float x) { return x; }
__device__ __forceinline__ float elem_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// GM >= group: the register tile of per-head dq for the shared list.
template <int D, typename T, int GM>
__global__ void __launch_bounds__(kBwdWarps * 32) k_decode_bwd(const BackwardArgs a) {
  constexpr int kE = Vec16<T>::kElems;  // elements per lane (8 bf16 or 4 fp32)
  constexpr int kLpr = D / kE;          // lanes per token
  constexpr int kRpw = 32 / kLpr;       // tokens per warp pass
  extern __shared__ float4 bwd_dyn[];
  const int G = a.group;
  float *q_s = reinterpret_cast<float *>(bwd_dyn);  // [G][D]
  float *g_s = q_s + G * D;                         // [G][D]
  float *dq_s = g_s + G * D;                        // [G][D]
  float *go_s = dq_s + G * D;                       // [G]  g.o
  float *lse_s = go_s + G;                          // [G]  lse * log2(e)
  int *off_s = reinterpret_cast<int *>(lse_s + G);  // [G + 1] per-head list offsets
  int *nsel_s = off_s + G + 1;                      // [G]
  int *sel_s = nsel_s + G;                          // [G][k] valid selections

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kvh = blockIdx.y, b = blockIdx.z;
  const size_t row0 = static_cast<size_t>(b) * a.hq + static_cast<size_t>(kvh) * G;
  const int slot = lane / kLpr, dd = kE * (lane % kLpr);

  pdl_wait();
  // the forward's clamps: N <= n_max, N*chunk + own <= t_max
  const int N = min(min(max(a.n_gists[b], 0), a.n_max), a.t_max / a.chunk);
  int own = min(max(a.own_len[b], 0), a.chunk);
  if (static_cast<int64_t>(N) * a.chunk + own > a.t_max) own = max(0, a.t_max - N * a.chunk);
  for (int i = tid; i < G * D; i += kBwdWarps * 32) {
    const size_t gi = row0 * D + i;
    q_s[i] = elem_f32(reinterpret_cast<const T *>(a.q)[gi]);
    g_s[i] = a.d_out[gi];
    dq_s[i] = 0.f;
  }
  for (int h = warp; h < G; h += kBwdWarps) {
    int n = 0;  // the head's valid selections, in list order
    const int32_t *sr = a.sel_idx + (row0 + h) * a.k;
    for (int i0 = 0; i0 < a.k; i0 += 32) {
      const int i = i0 + lane;
      const int m = i < a.k ? sr[i] : -1;
      const bool ok = m >= 0 && m < N;
      const unsigned bal = __ballot_sync(0xffffffffu, ok);
      if (ok) sel_s[h * a.k + n + __popc(bal & ((1u << lane) - 1u))] = m;
      n += __popc(bal);
    }
    float go = 0.f;
    for (int e = lane; e < D; e += 32) go = fmaf(a.d_out[(row0 + h) * D + e], a.out[(row0 + h) * D + e], go);
    go = warp_sum(go);
    if (lane == 0) {
      nsel_s[h] = n;
      go_s[h] = go;
      lse_s[h] = a.lse[row0 + h] * kLog2e;
    }
  }
  __syncthreads();
  if (tid == 0) {
    int o = 0;
    for (int h = 0; h < G; ++h) {
      off_s[h] = o;
      o += nsel_s[h] * (a.chunk + a.exclude);
    }
    off_s[G] = o;
  }
  __syncthreads();

  const float sl2 = a.scale * kLog2e;
  const size_t gbase = (static_cast<size_t>(b) * a.hkv + kvh) * a.n_max;
  const size_t rbase = (static_cast<size_t>(b) * a.hkv + kvh) * a.t_max;
  const int S = gridDim.x, s = blockIdx.x;

  // ---- shared list: gists (default set), then the own rows
  const int n_gs = a.exclude ? 0 : N;
  const int n_sh = n_gs + own;
  const int per_sh = (n_sh + S - 1) / S;
  const int s0 = min(n_sh, s * per_sh), s1 = min(n_sh, s0 + per_sh);
  float dq[GM][kE];
#pragma unroll
  for (int h = 0; h < GM; ++h)
#pragma unroll
    for (int e = 0; e < kE; ++e) dq[h][e] = 0.f;
  // kBwdU tokens per lane group per pass: their loads are all in flight
  // together and each head's q / g slice is read from shared memory once.
  constexpr int kBwdU = bwd_unroll<GM>();
  for (int tb = s0 + warp * kRpw * kBwdU; tb < s1; tb += kBwdWarps * kRpw * kBwdU) {
    float kf[kBwdU][kE], vf[kBwdU][kE], dk[kBwdU][kE], dv[kBwdU][kE];
    float *dkp[kBwdU], *dvp[kBwdU];
    bool valid[kBwdU];
#pragma unroll
    for (int u = 0; u < kBwdU; ++u) {
      const int t = tb + u * kRpw + slot;
      valid[u] = t < s1;
      const bool gist = t < n_gs;
      const size_t r = gist ? gbase + t : rbase + static_cast<size_t>(N) * a.chunk + (t - n_gs);
      const T *kp = reinterpret_cast<const T *>(gist ? a.gist_k : a.raw_k) + r * D + dd;
      const T *vp = reinterpret_cast<const T *>(gist ? a.gist_v : a.raw_v) + r * D + dd;
      dkp[u] = (gist ? a.d_gist_k : a.d_raw_k) + r * D + dd;
      dvp[u] = (gist ? a.d_gist_v : a.d_raw_v) + r * D + dd;
      Vec16<T>::unpack(valid[u] ? ldg_nc_v4(kp) : make_uint4(0, 0, 0, 0), kf[u]);
      Vec16<T>::unpack(valid[u] ? ldg_nc_v4(vp) : make_uint4(0, 0, 0, 0), vf[u]);
      // the gradient rows' current values, fetched with the keys / values
      // so that the loads overlap instead of following the arithmetic
#pragma unroll
      for (int e = 0; e < kE; e += 4) {
        const float4 x = valid[u] ? *reinterpret_cast<const float4 *>(dkp[u] + e) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 y = valid[u] ? *reinterpret_cast<const float4 *>(dvp[u] + e) : make_float4(0.f, 0.f, 0.f, 0.f);
        dk[u][e] = x.x; dk[u][e + 1] = x.y; dk[u][e + 2] = x.z; dk[u][e + 3] = x.w;
        dv[u][e] = y.x; dv[u][e + 1] = y.y; dv[u][e + 2] = y.z; dv[u][e + 3] = y.w;
      }
    }
#pragma unroll
    for (int h = 0; h < GM; ++h) {
      if (h < G) {
        float qh[kE], gh[kE];
#pragma unroll
        for (int e = 0; e < kE; e += 4) {
          const float4 qv = *reinterpret_cast<const float4 *>(q_s + h * D + dd + e);
          const float4 gw = *reinterpret_cast<const float4 *>(g_s + h * D + dd + e);
          qh[e] = qv.x; qh[e + 1] = qv.y; qh[e + 2] = qv.z; qh[e + 3] = qv.w;
          gh[e] = gw.x; gh[e + 1] = gw.y; gh[e + 2] = gw.z; gh[e + 3] = gw.w;
        }
        const float lh = lse_s[h], goh = go_s[h];
#pragma unroll
        for (int u = 0; u < kBwdU; ++u) {
          float qk = 0.f, gv = 0.f;
#pragma unroll
          for (int e = 0; e < kE; ++e) {
            qk = fmaf(qh[e], kf[u][e], qk);
            gv = fmaf(gh[e], vf[u][e], gv);
          }
#pragma unroll
          for (int o = 1; o < kLpr; o <<= 1) {
            qk += __shfl_xor_sync(0xffffffffu, qk, o);
            gv += __shfl_xor_sync(0xffffffffu, gv, o);
          }
          const float w = valid[u] ? exp2f(qk * sl2 - lh) : 0.f;
          const float sdz = a.scale * w * (gv - goh);
#pragma unroll
          for (int e = 0; e < kE; ++e) {
            dq[h][e] = fmaf(sdz, kf[u][e], dq[h][e]);
            dk[u][e] = fmaf(sdz, qh[e], dk[u][e]);
            dv[u][e] = fmaf(w, gh[e], dv[u][e]);
          }
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kBwdU; ++u) {
      if (valid[u]) {
#pragma unroll
        for (int e = 0; e < kE; e += 4) {
          *reinterpret_cast<float4 *>(dkp[u] + e) = make_float4(dk[u][e], dk[u][e + 1], dk[u][e + 2], dk[u][e + 3]);
          *reinterpret_cast<float4 *>(dvp[u] + e) = make_float4(dv[u][e], dv[u][e + 1], dv[u][e + 2], dv[u][e + 3]);
        }
      }
    }
  }
  // dq of the shared list: over the lane groups of the warp, then into shared memory
#pragma unroll
  for (int h = 0; h < GM; ++h) {
    if (h < G) {
#pragma unroll
      for (int o = kLpr; o < 32; o <<= 1)
#pragma unroll
        for (int e = 0; e < kE; ++e) dq[h][e] += __shfl_xor_sync(0xffffffffu, dq[h][e], o);
      if (lane < kLpr)
#pragma unroll
        for (int e = 0; e < kE; ++e) atomicAdd(dq_s + h * D + dd + e, dq[h][e]);
    }
  }

  // ---- per-head list: [exclude: the selected gists] then the selected chunks' raw rows
  const int n_it = off_s[G];
  const int per_it = (n_it + S - 1) / S;
  const int i0 = min(n_it, s * per_it), i1 = min(n_it, i0 + per_it);
  float dqc[kE];
#pragma unroll
  for (int e = 0; e < kE; ++e) dqc[e] = 0.f;
  int cur = -1;
  for (int tb = i0 + warp * kRpw; tb < i1; tb += kBwdWarps * kRpw) {
    const int t = tb + slot;
    const bool valid = t < i1;
    int h = 0;
    bool gist = false;
    size_t r = 0;
    if (valid) {
      while (h + 1 < G && off_s[h + 1] <= t) ++h;
      int u = t - off_s[h];
      const int nh = nsel_s[h];
      const int *sh = sel_s + h * a.k;
      if (a.exclude && u < nh) {
        gist = true;
        r = gbase + sh[u];
      } else {
        u -= a.exclude ? nh : 0;
        r = rbase + static_cast<size_t>(sh[u / a.chunk]) * a.chunk + u % a.chunk;
      }
    }
    const T *kp = reinterpret_cast<const T *>(gist ? a.gist_k : a.raw_k) + r * D + dd;
    const T *vp = reinterpret_cast<const T *>(gist ? a.gist_v : a.raw_v) + r * D + dd;
    float kf[kE], vf[kE], qh[kE], gh[kE];
    Vec16<T>::unpack(valid ? ldg_nc_v4(kp) : make_uint4(0, 0, 0, 0), kf);
    Vec16<T>::unpack(valid ? ldg_nc_v4(vp) : make_uint4(0, 0, 0, 0), vf);
#pragma unroll
    for (int e = 0; e < kE; e += 4) {
      const float4 qv = *reinterpret_cast<const float4 *>(q_s + h * D + dd + e);
      const float4 gw = *reinterpret_cast<const float4 *>(g_s + h * D + dd + e);
      qh[e] = qv.x; qh[e + 1] = qv.y; qh[e + 2] = qv.z; qh[e + 3] = qv.w;
      gh[e] = gw.x; gh[e + 1] = gw.y; gh[e + 2] = gw.z; gh[e + 3] = gw.w;
    }
    float qk = 0.f, gv = 0.f;
#pragma unroll
    for (int e = 0; e < kE; ++e) {
      qk = fmaf(qh[e], kf[e], qk);
      gv = fmaf(gh[e], vf[e], gv);
    }
#pragma unroll
    for (int o = 1; o < kLpr; o <<= 1) {
      qk += __shfl_xor_sync(0xffffffffu, qk, o);
      gv += __shfl_xor_sync(0xffffffffu, gv, o);
    }
    if (valid) {
      const float w = exp2f(qk * sl2 - lse_s[h]);
      const float sdz = a.scale * w * (gv - go_s[h]);
      if (h != cur) {  // a lane's tokens only move forward, so at most G flushes
        if (cur >= 0)
#pragma unroll
          for (int e = 0; e < kE; ++e) atomicAdd(dq_s + cur * D + dd + e, dqc[e]);
#pragma unroll
        for (int e = 0; e < kE; ++e) dqc[e] = 0.f;
        cur = h;
      }
#pragma unroll
      for (int e = 0; e < kE; ++e) dqc[e] = fmaf(sdz, kf[e], dqc[e]);
      float *dkp = (gist ? a.d_gist_k : a.d_raw_k) + r * D + dd;
      float *dvp = (gist ? a.d_gist_v : a.d_raw_v) + r * D + dd;
#pragma unroll
      for (int e = 0; e < kE; e += 4) {
        red_add4(dkp + e, sdz * qh[e], sdz * qh[e + 1], sdz * qh[e + 2], sdz * qh[e + 3]);
        red_add4(dvp + e, w * gh[e], w * gh[e + 1], w * gh[e + 2], w * gh[e + 3]);
      }
    }
  }
  if (cur >= 0)
#pragma unroll
    for (int e = 0; e < kE; ++e) atomicAdd(dq_s + cur * D + dd + e, dqc[e]);
  __syncthreads();
  pdl_trigger();
  for (int i = tid; i < G * D / 4; i += kBwdWarps * 32) {
    const float4 v = *reinterpret_cast<const float4 *>(dq_s + 4 * i);
    red_add4(a.d_q + row0 * D + 4 * i, v.x, v.y, v.z, v.w);
  }
}

}  // namespace gsa
