// Hybrid decode attention on CUDA cores: split-KV partials + merge with the sink.
//
// [SW] = shareware.cn/news/167317 (DeepSeek V4 Hybrid Attention essay): §三.1 / §十
// (raw 128-token window, which also covers the query's incomplete block), §六 (main
// attention over the indexer's top-k), §八 (HCA: dense over every entry), §十一 (MQA: all
// query heads share one KV), §十二 (attention sink).  [TR] = trdm.cn/news/516303: §2.2
// (QK^T / sqrt(d_k)), §3.1 (online softmax: running max and sum reproduce the full
// softmax exactly), §4.3 (compressed rows and window rows concatenated; HCA keeps the
// token-granularity window).
//
// Rows of query t (position p, sequence b) form one virtual list:
//   [0, n_cmp)       CSA: idx[t, r] (skipped when < 0);  HCA: entry r (r < floor((p+1)/128))
//   [n_cmp, +W)      window token p - W + 1 + (r - n_cmp) (skipped when < 0)
// CTA (split s, query t) runs an online softmax over rows [s*R, (s+1)*R) in tiles of 32
// and writes (m, l, acc) in the log2 domain; attn_combine merges the splits of a query
// and folds the sink logit in once.  This generic kernel serves fp32 and any head count, and
// FP8 main-KV rows (KV8: kv_cmp rows in the kv8.cuh layout, dequantised as they are loaded;
// the window's raw rows stay bf16 / fp32); bf16 with many heads goes to the tensor-core kernel.
#include "attn_rows.cuh"
#include "kv8.cuh"

namespace cskv {


constexpr int kAttnThreads = 256;
constexpr int kAttnTile = 32;
constexpr int kPsStride = kAttnTile + 1;  // padded row of the probability tile

template <typename T, int HP, bool KV8>
__global__ void __launch_bounds__(kAttnThreads) attn_split_kernel(AttnParams p) {
  constexpr int d = kHeadDim;
  constexpr int TPH = kAttnThreads / HP;  // threads per head in the PV update
  constexpr int ACC = d / TPH;            // accumulators per thread
  extern __shared__ __align__(16) float smf[];
  float* qs = smf;                               // [HP][d]
  float* ks = qs + HP * d;                       // [tile][d + 1]
  float* vs = ks + kAttnTile * (d + 1);          // [tile][d]
  float* ps = vs + kAttnTile * d;                // [HP][tile + 1]
  float* m_run = ps + HP * kPsStride;            // [HP]
  float* l_run = m_run + HP;                     // [HP]
  float* alpha = l_run + HP;                     // [HP]
  __shared__ int valid[kAttnTile];
  pdl_wait();

  const int t = blockIdx.y, split = blockIdx.x, tid = threadIdx.x;
  const QueryRows q = query_rows(p, t);
  if (q.s < 0) {
    if (split == 0 && tid == 0) flag(p.st, CSKV_DEV_BAD_INDEX);
    return;
  }
  const int64_t r0 = (int64_t)split * p.rows_per_split;
  if (r0 >= q.n_rows) return;
  const int64_t r1 = min(q.n_rows, r0 + p.rows_per_split);
  const int H = p.H;
  const T* qg = reinterpret_cast<const T*>(p.q) + (size_t)t * H * d;
  for (int i = tid; i < HP * d; i += kAttnThreads) qs[i] = (i < H * d) ? to_f(qg[i]) : 0.f;
  for (int h = tid; h < HP; h += kAttnThreads) {
    m_run[h] = -INFINITY;
    l_run[h] = 0.f;
  }
  const int hh = tid / TPH, jj = tid % TPH;
  float acc[ACC];
#pragma unroll
  for (int i = 0; i < ACC; ++i) acc[i] = 0.f;
  const T* cmp = reinterpret_cast<const T*>(p.kv_cmp);
  const T* raw = reinterpret_cast<const T*>(p.kv_raw);
  __syncthreads();

  for (int64_t a = r0; a < r1; a += kAttnTile) {
    // ---- load up to 32 rows: thread -> (row tid/8, 32-value part tid%8)
    {
      const int rr = tid >> 3, part = tid & 7;
      const int64_t r = a + rr;
      int64_t off = -1;
      bool is_raw = false;
      if (r < r1) off = resolve_row(p, q, t, r, &is_raw);
      if (part == 0) valid[rr] = off >= 0;
      if (off >= 0) {
        float f[32];
        if (KV8 && !is_raw) {
          kv8_load_part(reinterpret_cast<const uint8_t*>(p.kv_cmp) + (size_t)(off / kRow) * kKv8RowBytes, part, f);
        } else {
          const T* src = (is_raw ? raw : cmp) + off + part * 32;
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            float g[8];
            Vec8<T>::load(src + 8 * v, g);
#pragma unroll
            for (int u = 0; u < 8; ++u) f[8 * v + u] = g[u];
          }
        }
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          const int col = part * 32 + u;
          if (col < d)
            ks[rr * (d + 1) + col] = f[u];
          else
            vs[rr * d + col - d] = f[u];
        }
      }
    }
    __syncthreads();
    // ---- logits (log2 units)
    for (int i = tid; i < H * kAttnTile; i += kAttnThreads) {
      const int h = i / kAttnTile, rr = i % kAttnTile;
      float s = -INFINITY;
      if (valid[rr]) {
        const float* qh = qs + h * d;
        const float* kr = ks + rr * (d + 1);
        float dot = 0.f;
#pragma unroll 8
        for (int c = 0; c < d; ++c) dot = fmaf(qh[c], kr[c], dot);
        s = dot * p.scale_log2;
      }
      ps[h * kPsStride + rr] = s;
    }
    __syncthreads();
    // ---- online softmax per head
    for (int h = tid; h < H; h += kAttnThreads) {
      float mt = -INFINITY;
      for (int rr = 0; rr < kAttnTile; ++rr) mt = fmaxf(mt, ps[h * kPsStride + rr]);
      const float m_old = m_run[h];
      const float m_new = fmaxf(m_old, mt);
      float al = 1.f, sum = 0.f;
      if (m_new != -INFINITY) {
        al = exp2f(m_old - m_new);
        for (int rr = 0; rr < kAttnTile; ++rr) {
          const float e = exp2f(ps[h * kPsStride + rr] - m_new);
          ps[h * kPsStride + rr] = e;
          sum += e;
        }
      } else {
        for (int rr = 0; rr < kAttnTile; ++rr) ps[h * kPsStride + rr] = 0.f;
      }
      m_run[h] = m_new;
      l_run[h] = l_run[h] * al + sum;
      alpha[h] = al;
    }
    __syncthreads();
    // ---- acc = acc * alpha + P V
    if (hh < H) {
      const float al = alpha[hh];
#pragma unroll
      for (int i = 0; i < ACC; ++i) acc[i] *= al;
      for (int rr = 0; rr < kAttnTile; ++rr) {
        if (!valid[rr]) continue;
        const float pr = ps[hh * kPsStride + rr];
        const float* vr = vs + rr * d;
#pragma unroll
        for (int i = 0; i < ACC; ++i) acc[i] = fmaf(pr, vr[jj + TPH * i], acc[i]);
      }
    }
    __syncthreads();
  }
  // ---- partial out, dimension-major: acc[split][j][h], (m, l)[split][2][h]
  const size_t sb = (size_t)t * p.max_splits + split;
  if (hh < H) {
    float* dst = p.part_acc + sb * d * H + hh;
#pragma unroll
    for (int i = 0; i < ACC; ++i) dst[(size_t)(jj + TPH * i) * H] = acc[i];
  }
  for (int h = tid; h < H; h += kAttnThreads) {
    p.part_ml[sb * 2 * H + h] = m_run[h];
    p.part_ml[(sb * 2 + 1) * H + h] = l_run[h];
  }
  pdl_launch_dependents();  // the merge kernel waits for this grid before it reads
}

// Merge the splits of each query ([TR] §3.1), the sink once ([SW] §十二):
//   M = max(max_s m_s, sink), L = sum_s 2^{m_s - M} l_s + 2^{sink - M},
//   o = sum_s 2^{m_s - M} acc_s / L,   lse = ln 2 * (M + log2 L).
// CTA (block of kCombineDims output dimensions, query); thread (head h, split group g), group g
// taking splits g, g + kCombineGroups, ...  With few splits every load is issued at once and
// each group folds its splits under its own max; otherwise two passes with independent loads
// (so many are in flight at once): the max over the splits' m, merged across groups in shared
// memory, then the weighted sums of l and acc under that common max, summed across groups.
constexpr int kCombineDims = 2;
constexpr int kCombineGroups = 4;
constexpr int kFewSplits = 5;  // splits per group folded in one round of loads

__global__ void __launch_bounds__(128 * kCombineGroups) attn_combine_kernel(AttnParams p) {
  __shared__ float sM[kCombineGroups][128], sL[kCombineGroups][128], sO[kCombineGroups][kCombineDims][128];
  const int t = blockIdx.y, j0 = blockIdx.x * kCombineDims;
  const int h = threadIdx.x & 127, g = threadIdx.x >> 7;
  const int H = p.H;
  pdl_launch_dependents();
  pdl_wait();
  const QueryRows q = query_rows(p, t);
  int S = q.s < 0 ? 0 : (int)((q.n_rows + p.rows_per_split - 1) / p.rows_per_split);
  if (S > p.max_splits) {
    if (threadIdx.x == 0 && j0 == 0) flag(p.st, CSKV_DEV_CAPACITY);
    S = p.max_splits;
  }
  const size_t sb0 = (size_t)t * p.max_splits;
  const float* mrow = p.part_ml + sb0 * 2 * H + h;  // m of split s at mrow[s * 2H], l at + H
  const float* acc = p.part_acc + sb0 * kHeadDim * H + (size_t)j0 * H + h;
  if (S <= kFewSplits * kCombineGroups) {
    // ---- few splits (decode): one round of loads; group g folds its <= kFewSplits splits under its
    //      own max, then thread g = 0 rescales the groups to the common max
    float mv[kFewSplits], lv[kFewSplits], av[kFewSplits][kCombineDims];
#pragma unroll
    for (int i = 0; i < kFewSplits; ++i) {
      const int s = g + kCombineGroups * i;
      const bool ok = h < H && s < S;
      mv[i] = ok ? __ldg(mrow + (size_t)s * 2 * H) : -INFINITY;
      lv[i] = ok ? __ldg(mrow + (size_t)s * 2 * H + H) : 0.f;
#pragma unroll
      for (int jj = 0; jj < kCombineDims; ++jj)
        av[i][jj] = ok ? __ldg(acc + (size_t)s * kHeadDim * H + (size_t)jj * H) : 0.f;
    }
    float Mg = -INFINITY;
#pragma unroll
    for (int i = 0; i < kFewSplits; ++i) Mg = fmaxf(Mg, mv[i]);
    float Lg = 0.f, og[kCombineDims] = {};
    if (Mg != -INFINITY) {
#pragma unroll
      for (int i = 0; i < kFewSplits; ++i)
        if (mv[i] != -INFINITY) {
          const float f = exp2f(mv[i] - Mg);
          Lg = fmaf(lv[i], f, Lg);
#pragma unroll
          for (int jj = 0; jj < kCombineDims; ++jj) og[jj] = fmaf(av[i][jj], f, og[jj]);
        }
    }
    sM[g][h] = Mg;
    sL[g][h] = Lg;
#pragma unroll
    for (int jj = 0; jj < kCombineDims; ++jj) sO[g][jj][h] = og[jj];
    __syncthreads();
    if (g != 0 || h >= H) return;
    const float sk = p.sink ? __ldg(p.sink + h) * kLog2e : -INFINITY;
    float Mt = sk;
#pragma unroll
    for (int gg = 0; gg < kCombineGroups; ++gg) Mt = fmaxf(Mt, sM[gg][h]);
    float Lt = 0.f, ot[kCombineDims] = {};
    if (Mt != -INFINITY) {
      Lt = p.sink ? exp2f(sk - Mt) : 0.f;
#pragma unroll
      for (int gg = 0; gg < kCombineGroups; ++gg) {
        if (sM[gg][h] == -INFINITY) continue;
        const float f = exp2f(sM[gg][h] - Mt);
        Lt = fmaf(sL[gg][h], f, Lt);
#pragma unroll
        for (int jj = 0; jj < kCombineDims; ++jj) ot[jj] = fmaf(sO[gg][jj][h], f, ot[jj]);
      }
    }
    const float inv = Lt > 0.f ? 1.f / Lt : 0.f;
    float* dst = p.out + ((size_t)t * H + h) * kHeadDim + j0;
#pragma unroll
    for (int jj = 0; jj < kCombineDims; ++jj) dst[jj] = ot[jj] * inv;
    if (j0 == 0 && p.lse) p.lse[(size_t)t * H + h] = Lt > 0.f ? (Mt + log2f(Lt)) * 0.69314718055994531f : -INFINITY;
    return;
  }
  // ---- pass 1: M = max over all splits of m (log2 units)
  float M = -INFINITY;
  if (h < H) {
#pragma unroll 8
    for (int s = g; s < S; s += kCombineGroups) M = fmaxf(M, __ldg(mrow + (size_t)s * 2 * H));
  }
  sM[g][h] = M;
  __syncthreads();
  M = sM[0][h];
#pragma unroll
  for (int gg = 1; gg < kCombineGroups; ++gg) M = fmaxf(M, sM[gg][h]);
  // ---- pass 2: L = sum_s 2^(m_s - M) l_s, o = sum_s 2^(m_s - M) acc_s
  float L = 0.f, o[kCombineDims] = {};
  if (h < H && M != -INFINITY) {
#pragma unroll 8
    for (int s = g; s < S; s += kCombineGroups) {
      const float ms = __ldg(mrow + (size_t)s * 2 * H);
      const float ls = __ldg(mrow + (size_t)s * 2 * H + H);
      float a[kCombineDims];
#pragma unroll
      for (int jj = 0; jj < kCombineDims; ++jj) a[jj] = __ldg(acc + (size_t)s * kHeadDim * H + (size_t)jj * H);
      if (ms != -INFINITY) {  // a split whose rows were all skipped holds nothing
        const float f = exp2f(ms - M);
        L = fmaf(ls, f, L);
#pragma unroll
        for (int jj = 0; jj < kCombineDims; ++jj) o[jj] = fmaf(a[jj], f, o[jj]);
      }
    }
  }
  sL[g][h] = L;
#pragma unroll
  for (int jj = 0; jj < kCombineDims; ++jj) sO[g][jj][h] = o[jj];
  __syncthreads();
  if (g != 0 || h >= H) return;
  float Ls = 0.f, os[kCombineDims] = {};
#pragma unroll
  for (int gg = 0; gg < kCombineGroups; ++gg) {
    Ls += sL[gg][h];
#pragma unroll
    for (int jj = 0; jj < kCombineDims; ++jj) os[jj] += sO[gg][jj][h];
  }
  // ---- the sink joins the denominator once
  const float sk = p.sink ? __ldg(p.sink + h) * kLog2e : -INFINITY;
  const float Mt = fmaxf(M, sk);
  float Lt = 0.f, fp = 0.f;
  if (Mt != -INFINITY) {
    fp = M == -INFINITY ? 0.f : exp2f(M - Mt);
    Lt = Ls * fp + (p.sink ? exp2f(sk - Mt) : 0.f);
  }
  const float inv = Lt > 0.f ? fp / Lt : 0.f;
  float* dst = p.out + ((size_t)t * H + h) * kHeadDim + j0;
#pragma unroll
  for (int jj = 0; jj < kCombineDims; ++jj) dst[jj] = os[jj] * inv;
  if (j0 == 0 && p.lse) p.lse[(size_t)t * H + h] = Lt > 0.f ? (Mt + log2f(Lt)) * 0.69314718055994531f : -INFINITY;
}

cudaError_t launch_attn_combine(const AttnParams& p, cudaStream_t stream) {
  cudaError_t e = ensure_smem(attn_combine_kernel, 0);
  if (e != cudaSuccess) return e;
  e = launch_dependent(attn_combine_kernel, dim3(kHeadDim / kCombineDims, p.T),
                                         dim3(128 * kCombineGroups), 0, stream, p);
  note_launch();
  return e;
}

// ------------------------------------------------------------------ host side
static int attn_hp(int H) { return H <= 16 ? 16 : H <= 32 ? 32 : H <= 64 ? 64 : 128; }

static size_t attn_smem(int HP) {
  const int d = kHeadDim;
  return sizeof(float) * ((size_t)HP * d + kAttnTile * (d + 1) + kAttnTile * d + HP * kPsStride + 3 * HP);
}

int attn_rows_per_split(int mode, int T, int k, int window, int64_t max_entries, int sms) {
  const int64_t rows_max = (mode == CSKV_CSA ? (int64_t)k : max_entries) + window;
  int64_t R = (rows_max * (int64_t)T + 2 * sms - 1) / (2 * (int64_t)sms);
  R = (R + kAttnTile - 1) / kAttnTile * kAttnTile;
  if (R < kAttnTile) R = kAttnTile;
  if (R > 4096) R = 4096;
  return (int)R;
}

// Tensor-core kernel: a split is a whole number of 128-row chunks, sized so that the
// queries' splits about fill one wave of the SMs (at most 8 chunks per split).
int attn_tc_rows_per_split(int mode, int T, int k, int window, int64_t max_entries, int sms) {
  const int64_t rows_max = (mode == CSKV_CSA ? (int64_t)k : max_entries) + window;
  int64_t R = (rows_max * (int64_t)T + sms - 1) / sms;
  // CSA splits may be a half chunk (64 rows): the few CTAs of a decode query then finish
  // sooner.  HCA splits are two chunks at least: fewer, longer CTAs beside the indexer (the
  // HCA layer runs in its shadow) and half the partials to merge.
  const int64_t g = mode == CSKV_CSA ? 64 : 256;
  R = (R + g - 1) / g * g;
  if (R < g) R = g;
  if (R > 1024) R = 1024;
  return (int)R;
}

int attn_max_splits(int mode, int k, int window, int64_t max_entries, int R) {
  const int64_t rows_max = (mode == CSKV_CSA ? (int64_t)k : max_entries) + window;
  const int64_t s = (rows_max + R - 1) / R;
  return (int)(s > 0 ? s : 1);
}

template <typename T, int HP, bool KV8>
static cudaError_t launch_split_as(const AttnParams& p, cudaStream_t stream) {
  const size_t smem = attn_smem(HP);
  auto kern = attn_split_kernel<T, HP, KV8>;
  cudaError_t e = ensure_smem(kern, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.max_splits, p.T);
  e = launch_dependent(kern, grid, dim3(kAttnThreads), smem, stream, p);
  note_launch();
  return e;
}

template <typename T, int HP>
static cudaError_t launch_split(const AttnParams& p, cudaStream_t stream) {
  return p.kv8 ? launch_split_as<T, HP, true>(p, stream) : launch_split_as<T, HP, false>(p, stream);
}

cudaError_t launch_attn_generic(const AttnParams& p, int dtype, cudaStream_t stream) {
  const int hp = attn_hp(p.H);
  cudaError_t e;
  if (dtype == CSKV_F32) {
    e = hp == 16 ? launch_split<float, 16>(p, stream)
        : hp == 32 ? launch_split<float, 32>(p, stream)
        : hp == 64 ? launch_split<float, 64>(p, stream)
                   : launch_split<float, 128>(p, stream);
  } else {
    e = hp == 16 ? launch_split<__nv_bfloat16, 16>(p, stream)
        : hp == 32 ? launch_split<__nv_bfloat16, 32>(p, stream)
        : hp == 64 ? launch_split<__nv_bfloat16, 64>(p, stream)
                   : launch_split<__nv_bfloat16, 128>(p, stream);
  }
  if (e != cudaSuccess) return e;
  return launch_attn_combine(p, stream);
}

}  // namespace cskv
