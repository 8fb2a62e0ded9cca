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
  // the query's sequence and position load together with sequence 0's offsets (speculatively:
  // one round trip instead of two dependent ones when the query is in sequence 0)
  q.s = __ldg(p.q_seq + t);
  q.pos = __ldg(p.q_pos + t);
  const int64_t c0 = __ldg(p.cmp_off), c1 = __ldg(p.cmp_off + 1);
  const int64_t w0 = __ldg(p.raw_off), w1 = __ldg(p.raw_off + 1);
  const int64_t k0 = p.raw_tok0 ? __ldg(p.raw_tok0) : 0;
  if (q.s < 0 || q.s >= p.batch) {
    q.s = -1;
    q.n_rows = 0;
    return q;
  }
  const bool s0 = q.s == 0;
  q.cmp0 = s0 ? c0 : __ldg(p.cmp_off + q.s);
  q.cmp_cap = (s0 ? c1 : __ldg(p.cmp_off + q.s + 1)) - q.cmp0;
  q.raw0 = s0 ? w0 : __ldg(p.raw_off + q.s);
  q.raw_rows = (s0 ? w1 : __ldg(p.raw_off + q.s + 1)) - q.raw0;
  q.tok0 = p.raw_tok0 ? (s0 ? k0 : __ldg(p.raw_tok0 + q.s)) : 0;
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

// A pair of adjacent queries (HCA mode, a prefill chunk): q0 at p, q1 at p + 1 of the same
// sequence (q1v false: q0 alone).  Their union row list: the HCA entries [0, nu), nu the larger
// visible count, then the window tokens p - W + 1 .. p + 1.  Returns the row's element offset
// (-1: skipped for both) and whether each query attends to it.
__device__ __forceinline__ int64_t resolve_pair_row(const AttnParams& p, const QueryRows& q0, const QueryRows& q1,
                                                    bool q1v, int64_t nu, int64_t r, bool* raw, bool* ok0,
                                                    bool* ok1) {
  if (r < nu) {
    *raw = false;
    *ok0 = r < q0.n_cmp;
    *ok1 = q1v && r < q1.n_cmp;
    return (*ok0 || *ok1) ? (q0.cmp0 + r) * kRow : -1;
  }
  *raw = true;
  const int64_t tok = q0.pos - p.window + 1 + (r - nu);
  *ok0 = tok >= 0 && tok <= q0.pos;
  *ok1 = q1v && tok >= 0 && tok >= q1.pos - p.window + 1 && tok <= q1.pos;
  if (!*ok0 && !*ok1) return -1;
  const int64_t row = tok - q0.tok0;
  if (row < 0 || row >= q0.raw_rows) {
    flag(p.st, row < 0 ? CSKV_DEV_TAIL_MISSING : CSKV_DEV_BAD_INDEX);
    *ok0 = *ok1 = false;
    return -1;
  }
  return (q0.raw0 + row) * kRow;
}

}  // namespace cskv
