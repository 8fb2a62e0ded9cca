// Token-dimension KV compression: CSA (4:1, two streams) and HCA (128:1, one stream).
//
// [SW] = shareware.cn/news/167317 (DeepSeek V4 Hybrid Attention essay), §二, §四, §五;
// [TR] = trdm.cn/news/516303 ("从 MLA 到 CSA ..."), §4.3 改进一/改进二 and the HCA paragraph.
//
// Entry i of a sequence is, for each of the 256 packed K||V dimensions j separately,
// a softmax-weighted sum over its candidate tokens:
//   CSA: tokens of block i through path A (x_a, z_a + B_a[slot]) and of block i-1
//        through path B (x_b, z_b + B_b[slot]) -- one joint softmax over <= 8 candidates;
//   HCA: the 128 tokens of block i (x, z + B_h[slot]).
//
// Both kernels are pure HBM streams (every input row is read once, 512 B bf16 per row):
// lanes own 8 consecutive dimensions, so each warp-wide 16-byte vector load covers one
// whole 512-byte row, and every candidate's loads are in flight before any arithmetic.
// Softmax runs in the log2 domain: l2 = (z + b) * log2(e), w = exp2(l2 - max).
#include "launch.cuh"

namespace cskv {

// Raw 8-value slice of a row kept in registers until used (bf16: one uint4).
template <typename T>
struct Raw8;

template <>
struct Raw8<__nv_bfloat16> {
  uint4 v;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) { v = __ldg(reinterpret_cast<const uint4*>(p)); }
  __device__ __forceinline__ float get(int i) const {
    const uint32_t w = (i < 2) ? v.x : (i < 4) ? v.y : (i < 6) ? v.z : v.w;
    return (i & 1) ? __uint_as_float(w & 0xffff0000u) : __uint_as_float(w << 16);
  }
};

template <>
struct Raw8<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float* p) {
    a = __ldg(reinterpret_cast<const float4*>(p));
    b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  }
  __device__ __forceinline__ float get(int i) const {
    switch (i) {
      case 0: return a.x; case 1: return a.y; case 2: return a.z; case 3: return a.w;
      case 4: return b.x; case 5: return b.y; case 6: return b.z; default: return b.w;
    }
  }
};

__device__ __forceinline__ void load_bias8(const float* bias, int slot, int j0, float (&b)[8]) {
  if (bias == nullptr) {
#pragma unroll
    for (int i = 0; i < 8; ++i) b[i] = 0.f;
    return;
  }
  const float4* p = reinterpret_cast<const float4*>(bias + (size_t)slot * kRow + j0);
  float4 u = __ldg(p), v = __ldg(p + 1);
  b[0] = u.x; b[1] = u.y; b[2] = u.z; b[3] = u.w; b[4] = v.x; b[5] = v.y; b[6] = v.z; b[7] = v.w;
}

struct SeqRange {
  int64_t row0, t0, n, first, num, ent0, ent_cap;
};

__device__ __forceinline__ SeqRange seq_range(int b, int ratio, const int64_t* tok_off, const int64_t* tok0,
                                              const int64_t* ent_off, const int64_t* first_block,
                                              const int64_t* num_blocks) {
  SeqRange r;
  r.row0 = tok_off[b];
  r.t0 = tok0 ? tok0[b] : 0;
  r.n = r.t0 + (tok_off[b + 1] - r.row0);
  const int64_t nent = (r.n + ratio - 1) / ratio;
  r.first = first_block ? first_block[b] : 0;
  r.num = num_blocks ? num_blocks[b] : nent - r.first;
  r.ent0 = ent_off[b];
  r.ent_cap = ent_off[b + 1] - r.ent0;
  return r;
}

// ------------------------------------------------------------------ CSA
// grid (ceil(max_blocks / kCsaWarps), batch), 32 * kCsaWarps threads: warp w of CTA x
// computes entry first + kCsaWarps * x + w of sequence blockIdx.y.  Small CTAs keep the
// register footprint low enough to run beside the indexer in a decode step.
constexpr int kCsaWarps = 2;

template <typename TI, typename TO, bool kTwo>
__global__ void __launch_bounds__(32 * kCsaWarps) csa_compress_kernel(
    const TI* __restrict__ xa, const TI* __restrict__ za, const TI* __restrict__ xb,
    const TI* __restrict__ zb, const float* __restrict__ ba, const float* __restrict__ bb,
    const int64_t* __restrict__ tok_off, const int64_t* __restrict__ tok0,
    const int64_t* __restrict__ ent_off, const int64_t* __restrict__ first_block,
    const int64_t* __restrict__ num_blocks, int64_t max_blocks, TO* __restrict__ out, int* st) {
  constexpr int kC = kTwo ? 8 : 4;  // candidates: 4 path-A (+ 4 path-B)
  const int b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const SeqRange s = seq_range(b, 4, tok_off, tok0, ent_off, first_block, num_blocks);
  if (blockIdx.x == 0 && threadIdx.x == 0 && s.num > max_blocks) flag(st, CSKV_DEV_CAPACITY);
  const int64_t local = (int64_t)blockIdx.x * kCsaWarps + warp;
  if (local >= s.num) return;
  const int64_t i = s.first + local;
  if (i < 0 || 4 * i >= s.n || i >= s.ent_cap) {
    if (lane == 0) flag(st, CSKV_DEV_BAD_INDEX);
    return;
  }
  const int64_t tfirst = (kTwo && i >= 1) ? 4 * (i - 1) : 4 * i;
  if (tfirst < s.t0) {
    if (lane == 0) flag(st, CSKV_DEV_TAIL_MISSING);
    return;
  }
  const int j0 = lane * 8;
  Raw8<TI> xr[kC], zr[kC];
  bool ok[kC];
#pragma unroll
  for (int c = 0; c < kC; ++c) {
    const bool pathA = c < 4;
    const int64_t t = pathA ? 4 * i + c : 4 * (i - 1) + (c - 4);
    ok[c] = pathA ? (t < s.n) : (i >= 1);
    if (ok[c]) {
      const size_t row = (size_t)(s.row0 + (t - s.t0)) * kRow + j0;
      xr[c].load((pathA ? xa : xb) + row);
      zr[c].load((pathA ? za : zb) + row);
    }
  }
  float m[8], den[8], num[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) { m[j] = -INFINITY; den[j] = 0.f; num[j] = 0.f; }
  float bias[kC][8];
#pragma unroll
  for (int c = 0; c < kC; ++c) load_bias8(c < 4 ? ba : bb, c & 3, j0, bias[c]);
#pragma unroll
  for (int c = 0; c < kC; ++c)
    if (ok[c]) {
#pragma unroll
      for (int j = 0; j < 8; ++j) m[j] = fmaxf(m[j], (zr[c].get(j) + bias[c][j]) * kLog2e);
    }
#pragma unroll
  for (int c = 0; c < kC; ++c)
    if (ok[c]) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float w = exp2f((zr[c].get(j) + bias[c][j]) * kLog2e - m[j]);
        den[j] += w;
        num[j] = fmaf(w, xr[c].get(j), num[j]);
      }
    }
  float o[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) o[j] = num[j] / den[j];
  Vec8<TO>::store(out + (size_t)(s.ent0 + i) * kRow + j0, o);
}

// ------------------------------------------------------------------ HCA
// Raw 4-value slice of a row kept in registers until used (bf16: one uint2).
template <typename T>
struct Raw4;

template <>
struct Raw4<__nv_bfloat16> {
  uint2 v;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) { v = __ldg(reinterpret_cast<const uint2*>(p)); }
  __device__ __forceinline__ float get(int i) const {
    const uint32_t w = (i < 2) ? v.x : v.y;
    return (i & 1) ? __uint_as_float(w & 0xffff0000u) : __uint_as_float(w << 16);
  }
};

template <>
struct Raw4<float> {
  float4 a;
  __device__ __forceinline__ void load(const float* p) { a = __ldg(reinterpret_cast<const float4*>(p)); }
  __device__ __forceinline__ float get(int i) const {
    switch (i) {
      case 0: return a.x; case 1: return a.y; case 2: return a.z; default: return a.w;
    }
  }
};

__device__ __forceinline__ void load_bias4(const float* bias, int slot, int j0, float (&b)[4]) {
  if (bias == nullptr) {
    b[0] = b[1] = b[2] = b[3] = 0.f;
    return;
  }
  const float4 u = __ldg(reinterpret_cast<const float4*>(bias + (size_t)slot * kRow + j0));
  b[0] = u.x; b[1] = u.y; b[2] = u.z; b[3] = u.w;
}

// grid (max_blocks, batch), 256 threads: CTA x computes entry first + x.  Warp w covers
// dimension half (w & 1) -- lane l owns its dims 4l .. 4l+3 -- and token quarter (w >> 1),
// 32 tokens streamed eight at a time with a running max; the four quarter partials
// (max, sum, weighted sum) per dimension are merged through shared memory.  The small
// per-thread state keeps the CTA within 64 registers, so it fits beside the indexer.
constexpr int kHcaWarps = 8;
constexpr int kHcaQuarters = 4;

template <typename TI, typename TO>
__global__ void __launch_bounds__(32 * kHcaWarps, 4) hca_compress_kernel(
    const TI* __restrict__ x, const TI* __restrict__ z, const float* __restrict__ bias,
    const int64_t* __restrict__ tok_off, const int64_t* __restrict__ tok0,
    const int64_t* __restrict__ ent_off, const int64_t* __restrict__ first_block,
    const int64_t* __restrict__ num_blocks, int64_t max_blocks, TO* __restrict__ out, int* st) {
  constexpr int kTokPerQuarter = 128 / kHcaQuarters;  // 32
  constexpr int kGroup = sizeof(TI) == 2 ? 8 : 4;     // tokens loaded per round
  __shared__ float sm_m[kHcaQuarters][kRow], sm_s[kHcaQuarters][kRow], sm_a[kHcaQuarters][kRow];
  const int b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const SeqRange s = seq_range(b, 128, tok_off, tok0, ent_off, first_block, num_blocks);
  if (blockIdx.x == 0 && threadIdx.x == 0 && s.num > max_blocks) flag(st, CSKV_DEV_CAPACITY);
  const int64_t local = blockIdx.x;
  if (local >= s.num) return;
  const int64_t i = s.first + local;
  if (i < 0 || 128 * i >= s.n || i >= s.ent_cap) {
    if (threadIdx.x == 0) flag(st, CSKV_DEV_BAD_INDEX);
    return;
  }
  if (128 * i < s.t0) {
    if (threadIdx.x == 0) flag(st, CSKV_DEV_TAIL_MISSING);
    return;
  }
  const int quarter = warp >> 1;
  const int j0 = (warp & 1) * 128 + lane * 4;
  float m[4], den[4], num[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) { m[j] = -INFINITY; den[j] = 0.f; num[j] = 0.f; }
#pragma unroll 1
  for (int g0 = 0; g0 < kTokPerQuarter; g0 += kGroup) {
    Raw4<TI> xr[kGroup], zr[kGroup];
    bool ok[kGroup];
#pragma unroll
    for (int u = 0; u < kGroup; ++u) {
      const int slot = quarter * kTokPerQuarter + g0 + u;
      const int64_t t = 128 * i + slot;
      ok[u] = t < s.n;
      if (ok[u]) {
        const size_t row = (size_t)(s.row0 + (t - s.t0)) * kRow + j0;
        xr[u].load(x + row);
        zr[u].load(z + row);
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float l2[kGroup];
      float mg = m[j];
#pragma unroll
      for (int u = 0; u < kGroup; ++u) {
        const float bb = bias ? __ldg(bias + (size_t)(quarter * kTokPerQuarter + g0 + u) * kRow + j0 + j) : 0.f;
        l2[u] = ok[u] ? (zr[u].get(j) + bb) * kLog2e : -INFINITY;
        mg = fmaxf(mg, l2[u]);
      }
      if (mg != -INFINITY) {
        const float r = exp2f(m[j] - mg);  // rescale of the running sums (0 on the first group)
        den[j] *= r;
        num[j] *= r;
        m[j] = mg;
#pragma unroll
        for (int u = 0; u < kGroup; ++u)
          if (ok[u]) {
            const float w = exp2f(l2[u] - mg);
            den[j] += w;
            num[j] = fmaf(w, xr[u].get(j), num[j]);
          }
      }
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    sm_m[quarter][j0 + j] = m[j];
    sm_s[quarter][j0 + j] = den[j];
    sm_a[quarter][j0 + j] = num[j];
  }
  __syncthreads();
  {
    const int j = threadIdx.x;  // 256 threads, one per dimension
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kHcaQuarters; ++w) M = fmaxf(M, sm_m[w][j]);
    float S = 0.f, A = 0.f;
#pragma unroll
    for (int w = 0; w < kHcaQuarters; ++w) {
      const float mw = sm_m[w][j];
      if (mw != -INFINITY) {
        const float f = exp2f(mw - M);
        S = fmaf(sm_s[w][j], f, S);
        A = fmaf(sm_a[w][j], f, A);
      }
    }
    TO* dst = out + (size_t)(s.ent0 + i) * kRow + j;
    if constexpr (sizeof(TO) == 2)
      *dst = __float2bfloat16_rn(A / S);
    else
      *dst = A / S;
  }
}

// ------------------------------------------------------------------ launchers
template <typename TI, typename TO>
static cudaError_t launch_csa_t(const void* xa, const void* za, const void* xb, const void* zb,
                                const float* ba, const float* bb, const int64_t* tok_off,
                                const int64_t* tok0, int batch, const int64_t* ent_off,
                                const int64_t* first, const int64_t* num, int64_t max_blocks,
                                void* out, int* st, cudaStream_t stream) {
  dim3 grid((unsigned)((max_blocks + kCsaWarps - 1) / kCsaWarps), (unsigned)batch);
  if (xb != nullptr)
    csa_compress_kernel<TI, TO, true><<<grid, 32 * kCsaWarps, 0, stream>>>(
        (const TI*)xa, (const TI*)za, (const TI*)xb, (const TI*)zb, ba, bb, tok_off, tok0, ent_off,
        first, num, max_blocks, (TO*)out, st);
  else
    csa_compress_kernel<TI, TO, false><<<grid, 32 * kCsaWarps, 0, stream>>>(
        (const TI*)xa, (const TI*)za, nullptr, nullptr, ba, bb, tok_off, tok0, ent_off, first, num,
        max_blocks, (TO*)out, st);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_csa_compress(const void* xa, const void* za, const void* xb, const void* zb,
                                const float* ba, const float* bb, const int64_t* tok_off,
                                const int64_t* tok0, int batch, const int64_t* ent_off,
                                const int64_t* first, const int64_t* num, int64_t max_blocks,
                                int in_dt, int out_dt, void* out, int* st, cudaStream_t stream) {
  if (in_dt == CSKV_BF16 && out_dt == CSKV_BF16)
    return launch_csa_t<__nv_bfloat16, __nv_bfloat16>(xa, za, xb, zb, ba, bb, tok_off, tok0, batch,
                                                      ent_off, first, num, max_blocks, out, st, stream);
  if (in_dt == CSKV_BF16 && out_dt == CSKV_F32)
    return launch_csa_t<__nv_bfloat16, float>(xa, za, xb, zb, ba, bb, tok_off, tok0, batch, ent_off,
                                              first, num, max_blocks, out, st, stream);
  if (in_dt == CSKV_F32 && out_dt == CSKV_BF16)
    return launch_csa_t<float, __nv_bfloat16>(xa, za, xb, zb, ba, bb, tok_off, tok0, batch, ent_off,
                                              first, num, max_blocks, out, st, stream);
  return launch_csa_t<float, float>(xa, za, xb, zb, ba, bb, tok_off, tok0, batch, ent_off, first, num,
                                    max_blocks, out, st, stream);
}

template <typename TI, typename TO>
static cudaError_t launch_hca_t(const void* x, const void* z, const float* bias, const int64_t* tok_off,
                                const int64_t* tok0, int batch, const int64_t* ent_off,
                                const int64_t* first, const int64_t* num, int64_t max_blocks,
                                void* out, int* st, cudaStream_t stream) {
  dim3 grid((unsigned)max_blocks, (unsigned)batch);
  hca_compress_kernel<TI, TO><<<grid, 32 * kHcaWarps, 0, stream>>>((const TI*)x, (const TI*)z, bias, tok_off, tok0,
                                                       ent_off, first, num, max_blocks, (TO*)out, st);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_hca_compress(const void* x, const void* z, const float* bias, const int64_t* tok_off,
                                const int64_t* tok0, int batch, const int64_t* ent_off,
                                const int64_t* first, const int64_t* num, int64_t max_blocks,
                                int in_dt, int out_dt, void* out, int* st, cudaStream_t stream) {
  if (in_dt == CSKV_BF16 && out_dt == CSKV_BF16)
    return launch_hca_t<__nv_bfloat16, __nv_bfloat16>(x, z, bias, tok_off, tok0, batch, ent_off, first,
                                                      num, max_blocks, out, st, stream);
  if (in_dt == CSKV_BF16 && out_dt == CSKV_F32)
    return launch_hca_t<__nv_bfloat16, float>(x, z, bias, tok_off, tok0, batch, ent_off, first, num,
                                              max_blocks, out, st, stream);
  if (in_dt == CSKV_F32 && out_dt == CSKV_BF16)
    return launch_hca_t<float, __nv_bfloat16>(x, z, bias, tok_off, tok0, batch, ent_off, first, num,
                                              max_blocks, out, st, stream);
  return launch_hca_t<float, float>(x, z, bias, tok_off, tok0, batch, ent_off, first, num, max_blocks,
                                    out, st, stream);
}

}  // namespace cskv
