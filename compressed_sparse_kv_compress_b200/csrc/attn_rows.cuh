// Row list of one query in hybrid_decode_attn, shared by the CUDA-core and tensor-core kernels.
//
// Query t (position p, sequence b) attends to one virtual list of rows:
//   [0, n_cmp)       CSA: entry idx[t, r] (skipped when < 0; flagged and skipped when not yet
//                    complete at p);  HCA: entry r, r < floor((p+1)/128)
//   [n_cmp, +W)      raw window token p - W + 1 + (r - n_cmp) (skipped when < 0)
// ([SW] shareware.cn/news/167317 §三.1, §八, §十; [TR] trdm.cn/news/516303 §4.3.)
#pragma once

#include "launch.cuh"

namespace cskv {

struct QueryRows {
  int s;          // sequence (-1: invalid query)
  int64_t pos;    // position
  int64_t n_cmp;  // compressed slots
  int64_t vis_c;  // visible CSA entries (index check)
  int64_t cmp0, cmp_cap, raw0, raw_rows, tok0;
  int64_t n_rows;
};

__device__ __forceinline__ QueryRows query_rows(const AttnParams& p, int t) {
  QueryRows q;
  q.s = __ldg(p.q_seq + t);
  if (q.s < 0 || q.s >= p.batch) {
    q.s = -1;
    q.n_rows = 0;
    return q;
  }
  q.pos = __ldg(p.q_pos + t);
  q.cmp0 = __ldg(p.cmp_off + q.s);
  q.cmp_cap = __ldg(p.cmp_off + q.s + 1) - q.cmp0;
  q.raw0 = __ldg(p.raw_off + q.s);
  q.raw_rows = __ldg(p.raw_off + q.s + 1) - q.raw0;
  q.tok0 = p.raw_tok0 ? __ldg(p.raw_tok0 + q.s) : 0;
  const int64_t ratio = p.mode == CSKV_CSA ? 4 : 128;
  const int64_t vis = q.pos >= 0 ? (q.pos + 1) / ratio : 0;
  q.vis_c = vis < q.cmp_cap ? vis : q.cmp_cap;
  q.n_cmp = p.mode == CSKV_CSA ? p.k : q.vis_c;
  q.n_rows = q.n_cmp + p.window;
  return q;
}

// Row pointer (element offset into kv_cmp or kv_raw) of virtual row r, or -1 when the
// row is skipped.  *raw tells which array.  e_pre >= -1: idx[t, r], already loaded (CSA rows
// r < k only; the caller issues that load beside the query's other loads).
__device__ __forceinline__ int64_t resolve_row(const AttnParams& p, const QueryRows& q, int t, int64_t r,
                                               bool* raw, int64_t e_pre = -2) {
  if (r < q.n_cmp) {
    *raw = false;
    int64_t e = r;
    if (p.mode == CSKV_CSA) {
      e = e_pre >= -1 ? e_pre : __ldg(p.idx + (size_t)t * p.k + r);
      if (e < 0) return -1;
      if (e >= q.vis_c) {
        flag(p.st, CSKV_DEV_BAD_INDEX);
        return -1;
      }
    }
    return (q.cmp0 + e) * kRow;
  }
  *raw = true;
  const int64_t tok = q.pos - p.window + 1 + (r - q.n_cmp);
  if (tok < 0) return -1;
  const int64_t row = tok - q.tok0;
  if (row < 0) {
    flag(p.st, CSKV_DEV_TAIL_MISSING);
    return -1;
  }
  if (row >= q.raw_rows) {
    flag(p.st, CSKV_DEV_BAD_INDEX);
    return -1;
  }
  return (q.raw0 + row) * kRow;
}

}  // namespace cskv
