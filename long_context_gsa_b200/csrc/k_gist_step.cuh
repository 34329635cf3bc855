// k_gist_step.cuh -- chunk completion: the bookkeeping around the
// gist-position step.
//
// When the raw tokens of chunk N are complete, its gist token is decoded
// under the compression mask (gist.science/nl/paper/2604.20920, "Het
// Proces", Compressie: a gist sees only its own block and the gists before
// it): its query attends the gists 0..N-1, chunk N's raw tokens and itself.
// The library runs that attention with the decode kernels (scoring with the
// gist-set partial, then the unfold with no selected chunk); these two
// kernels put the new gist in place around them:
//   k_gist_append  writes the new gist's key / value at gist row N of each
//                  kv head and records N and N+1 in the workspace, so the
//                  scoring pass sees gists 0..N (itself included) while the
//                  unfold still finds chunk N's raw rows at N*chunk;
//   k_gist_commit  after the attention: n_gists[b] = N+1, own_len[b] = 0.
// A sequence whose gist array is full (N = n_max) is flagged
// (GSA_DEVERR_CAPACITY) and left as it was; its step attends gists 0..N-1
// and the raw rows only.
#pragma once

#include "common.cuh"

namespace gsa {

struct GistAppendArgs {
  const uint4 *k_new, *v_new;    // [B, hkv, row_vecs]
  uint4 *gist_k, *gist_v;        // [B, hkv, n_max, row_vecs]
  const int32_t *n_gists;        // [B]
  int32_t *n_cur, *n_plus;       // workspace [B] each
  int32_t hkv, n_max, row_vecs;  // row_vecs = 16-byte vectors per row
  uint32_t *status;
};

// Grid (hkv, B); one row copy per CTA.
__global__ void __launch_bounds__(64) k_gist_append(const GistAppendArgs a) {
  const int kvh = blockIdx.x, b = blockIdx.y;
  pdl_wait();
  const int N = min(max(a.n_gists[b], 0), a.n_max);
  const bool room = N < a.n_max;
  if (room) {
    const size_t src = (static_cast<size_t>(b) * a.hkv + kvh) * a.row_vecs;
    const size_t dst = ((static_cast<size_t>(b) * a.hkv + kvh) * a.n_max + N) * a.row_vecs;
    for (int i = threadIdx.x; i < a.row_vecs; i += blockDim.x) {
      a.gist_k[dst + i] = a.k_new[src + i];
      a.gist_v[dst + i] = a.v_new[src + i];
    }
  }
  if (kvh == 0 && threadIdx.x == 0) {
    a.n_cur[b] = N;
    a.n_plus[b] = room ? N + 1 : N;
    if (!room) flag_error(a.status, GSA_DEVERR_CAPACITY);
  }
  pdl_trigger();
}

// One thread per sequence.
__global__ void __launch_bounds__(128) k_gist_commit(const int32_t *n_cur, const int32_t *n_plus, int32_t *n_gists,
                                                     int32_t *own_len, int batch) {
  pdl_wait();
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < batch; b += gridDim.x * blockDim.x) {
    if (n_plus[b] == n_cur[b] + 1) {
      n_gists[b] = n_plus[b];
      own_len[b] = 0;
    }
  }
  pdl_trigger();
}

}  // namespace gsa
