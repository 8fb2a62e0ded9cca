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
// Both kernels are pure HBM streams (every input row is read once, 512 B bf16 per row) and
// put every load of a unit of work in flight before any arithmetic.  CSA: a warp per entry,
// lanes own 8 consecutive dimensions, so each warp-wide 16-byte vector load covers one whole
// 512-byte row.  HCA: an entry is cut into 16 slices of 16 dimensions, one small CTA each
// (see below), so one entry's 128 tokens are read by many SMs at once.  Softmax runs in the
// log2 domain: l2 = (z + b) * log2(e), w = exp2(l2 - max).
//
// Also here: the indexer's entry keys pooled from per-token keys ([TR] §4.2), a warp per entry.
#include <cuda_fp8.h>

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
// register footprint low enough to run beside the indexer in a decode step (<= 144 registers).
constexpr int kCsaWarps = 2;
constexpr int64_t kCsaGridCtas = 16384;  // grid bound of whole-cache calls (entries loop)

// Optional epilogues of the CSA kernels: RMSNorm of the entry's K and V halves, and the pooling
// of the per-token indexer keys (rows indexed like x_a) into E4M3 entry keys.
struct CsaExtras {
  int norm;
  const float* gamma;  // [256] (K then V) or NULL = ones
  float eps;
  const void* k_tok;  // [rows, Di] fp32 or bf16, or NULL
  int k_f32;
  int Di;
  uint8_t* k_codes;
  float* k_scale;
  int overlap;  // CSKV_OVERLAP_PREVIOUS: read before the previous kernel completes, wait at the end
};

template <typename TI, typename TO, bool kTwo>
__global__ void __maxnreg__(144) csa_compress_kernel(
    const TI* __restrict__ xa, const TI* __restrict__ za, const TI* __restrict__ xb,
    const TI* __restrict__ zb, const float* __restrict__ ba, const float* __restrict__ bb,
    const int64_t* __restrict__ tok_off, const int64_t* __restrict__ tok0,
    const int64_t* __restrict__ ent_off, const int64_t* __restrict__ first_block,
    const int64_t* __restrict__ num_blocks, int64_t max_blocks, TO* __restrict__ out, CsaExtras ex, int* st) {
  constexpr int kC = kTwo ? 8 : 4;  // candidates: 4 path-A (+ 4 path-B)
  // A few small CTAs: the next kernel may launch at once and sit beside them; it waits for
  // this grid before reading anything.  With ex.overlap the caller guarantees that the kernel
  // before this one neither writes this call's inputs nor reads its outputs: the entries are
  // computed while it runs (in a decode step: beside the indexer), and the wait moves to the
  // end, so this grid still completes after it and a kernel that waits for this grid sees both.
  pdl_launch_dependents();
  if (!ex.overlap) pdl_wait();
  const int b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const SeqRange s = seq_range(b, 4, tok_off, tok0, ent_off, first_block, num_blocks);
  if (blockIdx.x == 0 && threadIdx.x == 0 && s.num > max_blocks) flag(st, CSKV_DEV_CAPACITY);
  // warp-strided over the entries (a decode call has a few; a whole-cache call loops)
  for (int64_t local = (int64_t)blockIdx.x * kCsaWarps + warp; local < s.num && local < max_blocks;
       local += (int64_t)gridDim.x * kCsaWarps) {
    const int64_t i = s.first + local;
    if (i < 0 || 4 * i >= s.n || i >= s.ent_cap) {
      if (lane == 0) flag(st, CSKV_DEV_BAD_INDEX);
      continue;
    }
    const int64_t tfirst = (kTwo && i >= 1) ? 4 * (i - 1) : 4 * i;
    if (tfirst < s.t0) {
      if (lane == 0) flag(st, CSKV_DEV_TAIL_MISSING);
      continue;
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
    if (ex.norm) {
      // RMSNorm over each 128-dim half: lanes 0-15 hold K, lanes 16-31 hold V
      float ss = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) ss = fmaf(o[j], o[j], ss);
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
      const float r = rsqrtf(ss * (1.f / 128.f) + ex.eps);
#pragma unroll
      for (int j = 0; j < 8; ++j) o[j] = o[j] * r * (ex.gamma ? __ldg(ex.gamma + j0 + j) : 1.f);
    }
    Vec8<TO>::store(out + (size_t)(s.ent0 + i) * kRow + j0, o);
    if (ex.k_tok) {
      // the entry's indexer key: mean of its tokens' keys (fp32, token order), E4M3 + scale
      const int cnt = (int)min((int64_t)4, s.n - 4 * i);
      const int dpl = ex.Di / 32;
      const size_t kb = (size_t)ex.Di * (ex.k_f32 ? 4 : 2);
      const uint8_t* krow = reinterpret_cast<const uint8_t*>(ex.k_tok) + (size_t)(s.row0 + 4 * i - s.t0) * kb;
      float key[4] = {0.f, 0.f, 0.f, 0.f};
      float amax = 0.f;
#pragma unroll
      for (int d = 0; d < 4; ++d) {
        if (d < dpl) {
          const int col = lane * dpl + d;
          float acc = 0.f;
          for (int q = 0; q < cnt; ++q) {
            const uint8_t* r = krow + (size_t)q * kb;
            const float v = ex.k_f32 ? __ldg(reinterpret_cast<const float*>(r) + col)
                                     : __bfloat162float(__ldg(reinterpret_cast<const __nv_bfloat16*>(r) + col));
            acc = q == 0 ? v : __fadd_rn(acc, v);
          }
          key[d] = __fdiv_rn(acc, (float)cnt);
          amax = fmaxf(amax, fabsf(key[d]));
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      const float scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
      uint32_t packed = 0;
#pragma unroll
      for (int d = 0; d < 4; ++d)
        if (d < dpl)
          packed |= (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(key[d], scale), __NV_SATFINITE, __NV_E4M3) << (8 * d);
      uint8_t* dst = ex.k_codes + (size_t)(s.ent0 + i) * ex.Di + lane * dpl;
      if (dpl == 2)
        *reinterpret_cast<uint16_t*>(dst) = (uint16_t)packed;
      else
        *reinterpret_cast<uint32_t*>(dst) = packed;
      if (lane == 0) ex.k_scale[s.ent0 + i] = scale;
    }
  }
  if (ex.overlap) pdl_wait();
}

// ------------------------------------------------------------------ HCA
// An entry is cut into kHcaSlices slices of 16 dimensions, one CTA (4 warps) per slice:
// a lane pair covers one token's 16-dimension slice (8 dims per lane, one 16-byte load per
// array for bf16), a warp 16 tokens, the CTA 64 tokens per round, two rounds -- every load
// of the CTA is in flight before any arithmetic.  The per-dimension softmax over the 128
// tokens then takes two reductions (max, then sum and weighted sum): shuffles across the
// 16 lanes that share dimensions, then shared memory across the 4 warps.  Many small CTAs
// keep the latency of one entry short and fit beside the indexer's CTAs.
constexpr int kHcaSlices = 16;
constexpr int64_t kHcaGridEntries = 1024;  // grid bound of whole-cache calls (entries loop)
constexpr int kHcaThreads = 128;

template <typename T>
__device__ __forceinline__ void load8f(const T* p, float (&v)[8]) {
  Raw8<T> r;
  r.load(p);
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = r.get(i);
}

template <typename TI, typename TO>
__global__ void __launch_bounds__(kHcaThreads, 8) hca_compress_kernel(
    const TI* __restrict__ x, const TI* __restrict__ z, const float* __restrict__ bias,
    const int64_t* __restrict__ tok_off, const int64_t* __restrict__ tok0,
    const int64_t* __restrict__ ent_off, const int64_t* __restrict__ first_block,
    const int64_t* __restrict__ num_blocks, int64_t max_blocks, TO* __restrict__ out, int* st) {
  __shared__ float sm_max[4][16], sm_sum[4][16], sm_acc[4][16];
  // the next kernel (the HCA attention in a decode step) may start its set-up at once; it
  // waits for this grid before reading anything
  pdl_launch_dependents();
  pdl_wait();
  const int b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, half = lane & 1;
  const int slice = (int)(blockIdx.x % kHcaSlices);
  const int j0 = slice * 16 + half * 8;  // this lane's first dimension
  const SeqRange s = seq_range(b, 128, tok_off, tok0, ent_off, first_block, num_blocks);
  if (blockIdx.x == 0 && threadIdx.x == 0 && s.num > max_blocks) flag(st, CSKV_DEV_CAPACITY);
  const int64_t stride = gridDim.x / kHcaSlices;
  for (int64_t local = blockIdx.x / kHcaSlices; local < s.num && local < max_blocks; local += stride) {
    const int64_t i = s.first + local;
    if (i < 0 || 128 * i >= s.n || i >= s.ent_cap) {
      if (threadIdx.x == 0) flag(st, CSKV_DEV_BAD_INDEX);
      continue;  // block-uniform
    }
    if (128 * i < s.t0) {
      if (threadIdx.x == 0) flag(st, CSKV_DEV_TAIL_MISSING);
      continue;
    }
    float lg[2][8], xv[2][8];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int slot = r * 64 + warp * 16 + (lane >> 1);
      const int64_t t = 128 * i + slot;
      if (t < s.n) {
        const size_t row = (size_t)(s.row0 + (t - s.t0)) * kRow + j0;
        load8f(x + row, xv[r]);
        load8f(z + row, lg[r]);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          xv[r][e] = 0.f;
          lg[r][e] = -INFINITY;
        }
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int slot = r * 64 + warp * 16 + (lane >> 1);
      float bb[8];
      load_bias8(bias, slot, j0, bb);
#pragma unroll
      for (int e = 0; e < 8; ++e) lg[r][e] = (lg[r][e] + bb[e]) * kLog2e;  // -inf stays -inf
    }
    // ---- per-dimension max over the 128 tokens
    float m[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float v = fmaxf(lg[0][e], lg[1][e]);
#pragma unroll
      for (int o = 2; o < 32; o <<= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
      m[e] = v;
    }
    if (lane < 2)
#pragma unroll
      for (int e = 0; e < 8; ++e) sm_max[warp][half * 8 + e] = m[e];
    __syncthreads();
#pragma unroll
    for (int e = 0; e < 8; ++e)
      m[e] = fmaxf(fmaxf(sm_max[0][half * 8 + e], sm_max[1][half * 8 + e]),
                   fmaxf(sm_max[2][half * 8 + e], sm_max[3][half * 8 + e]));
    // ---- weights, sums and weighted sums (token 128i is present, so every max is finite)
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float w0 = exp2f(lg[0][e] - m[e]), w1 = exp2f(lg[1][e] - m[e]);
      float sw = w0 + w1;
      float sa = fmaf(w0, xv[0][e], w1 * xv[1][e]);
#pragma unroll
      for (int o = 2; o < 32; o <<= 1) {
        sw += __shfl_xor_sync(0xffffffffu, sw, o);
        sa += __shfl_xor_sync(0xffffffffu, sa, o);
      }
      if (lane < 2) {
        sm_sum[warp][half * 8 + e] = sw;
        sm_acc[warp][half * 8 + e] = sa;
      }
    }
    __syncthreads();
    if (threadIdx.x < 16) {
      const int j = threadIdx.x;
      const float S = (sm_sum[0][j] + sm_sum[1][j]) + (sm_sum[2][j] + sm_sum[3][j]);
      const float A = (sm_acc[0][j] + sm_acc[1][j]) + (sm_acc[2][j] + sm_acc[3][j]);
      TO* dst = out + (size_t)(s.ent0 + i) * kRow + slice * 16 + j;
      if constexpr (sizeof(TO) == 2)
        *dst = __float2bfloat16_rn(A / S);
      else
        *dst = A / S;
    }
    __syncthreads();  // the shared arrays are reused by the next entry
  }
}


// ------------------------------------------------------------------ indexer keys of the entries
// The Lightning Indexer's keys are projected per token and pooled to one key per CSA block
// ([TR] §4.2, a 1-D pool with kernel = stride = the block size): the mean over the block's
// tokens (a partial last block: over the tokens it has), stored as E4M3 codes with one fp32
// scale per entry, amax / 448 (1 for an all-zero key).  One warp per entry; lane l holds
// dimensions [l * DPL, l * DPL + DPL).  The codes are integers decided in fp32: tokens summed
// in order, one division by the count, one division by the scale, then the E4M3 conversion
// (round to nearest even, saturating to +-448).
constexpr int kPoolWarps = 4;
constexpr int64_t kPoolGridCtas = 16384;  // grid bound of whole-cache calls (entries loop)

template <int BYTES>
struct RawBytes;
template <>
struct RawBytes<4> { uint32_t v; };
template <>
struct RawBytes<8> { uint2 v; };
template <>
struct RawBytes<16> { uint4 v; };

template <typename TI, int DPL>
__device__ __forceinline__ void load_dims(const TI* p, float (&out)[DPL]) {
  union {
    RawBytes<DPL * sizeof(TI)> r;
    TI e[DPL];
  } u;
  u.r = *reinterpret_cast<const RawBytes<DPL * sizeof(TI)>*>(p);
#pragma unroll
  for (int j = 0; j < DPL; ++j) {
    if constexpr (sizeof(TI) == 2)
      out[j] = __bfloat162float(u.e[j]);
    else
      out[j] = u.e[j];
  }
}

template <typename TI, int DPL>
__global__ void __launch_bounds__(32 * kPoolWarps) pool_keys_kernel(
    const TI* __restrict__ k_tok, const int64_t* __restrict__ tok_off, const int64_t* __restrict__ tok0,
    const int64_t* __restrict__ ent_off, const int64_t* __restrict__ first_block,
    const int64_t* __restrict__ num_blocks, int64_t max_blocks, uint8_t* __restrict__ codes,
    float* __restrict__ scales, int* st) {
  constexpr int Di = 32 * DPL;
  pdl_launch_dependents();  // the indexer after it waits for this grid before reading the keys
  pdl_wait();
  const int b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const SeqRange s = seq_range(b, 4, tok_off, tok0, ent_off, first_block, num_blocks);
  if (blockIdx.x == 0 && threadIdx.x == 0 && s.num > max_blocks) flag(st, CSKV_DEV_CAPACITY);
  for (int64_t local = (int64_t)blockIdx.x * kPoolWarps + warp; local < s.num && local < max_blocks;
       local += (int64_t)gridDim.x * kPoolWarps) {
    const int64_t i = s.first + local;
    if (i < 0 || 4 * i >= s.n || i >= s.ent_cap) {
      if (lane == 0) flag(st, CSKV_DEV_BAD_INDEX);
      continue;
    }
    if (4 * i < s.t0) {
      if (lane == 0) flag(st, CSKV_DEV_TAIL_MISSING);
      continue;
    }
    const int cnt = (int)min((int64_t)4, s.n - 4 * i);
    float v[4][DPL];
#pragma unroll
    for (int c = 0; c < 4; ++c)
      if (c < cnt) load_dims<TI, DPL>(k_tok + (size_t)(s.row0 + (4 * i + c - s.t0)) * Di + lane * DPL, v[c]);
    float key[DPL];
    float amax = 0.f;
#pragma unroll
    for (int j = 0; j < DPL; ++j) {
      float acc = v[0][j];
#pragma unroll
      for (int c = 1; c < 4; ++c)
        if (c < cnt) acc = __fadd_rn(acc, v[c][j]);
      key[j] = __fdiv_rn(acc, (float)cnt);
      amax = fmaxf(amax, fabsf(key[j]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
    uint32_t packed = 0;
#pragma unroll
    for (int j = 0; j < DPL; ++j)
      packed |= (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(key[j], scale), __NV_SATFINITE, __NV_E4M3) << (8 * j);
    uint8_t* dst = codes + (size_t)(s.ent0 + i) * Di + lane * DPL;
    if constexpr (DPL == 2)
      *reinterpret_cast<uint16_t*>(dst) = (uint16_t)packed;
    else
      *reinterpret_cast<uint32_t*>(dst) = packed;
    if (lane == 0) scales[s.ent0 + i] = scale;
  }
}

// ------------------------------------------------------------------ launchers
template <typename TI, typename TO>
static cudaError_t launch_csa_t(const void* xa, const void* za, const void* xb, const void* zb,
                                const float* ba, const float* bb, const int64_t* tok_off,
                                const int64_t* tok0, int batch, const int64_t* ent_off,
                                const int64_t* first, const int64_t* num, int64_t max_blocks,
                                void* out, const CsaExtras& ex, int* st, cudaStream_t stream) {
  // a whole-cache call runs a bounded grid whose warps loop over the entries
  const int64_t ctas = (max_blocks + kCsaWarps - 1) / kCsaWarps;
  dim3 grid((unsigned)(ctas < kCsaGridCtas ? ctas : kCsaGridCtas), (unsigned)batch);
  cudaError_t e = ensure_smem(xb != nullptr ? csa_compress_kernel<TI, TO, true> : csa_compress_kernel<TI, TO, false>, 0);
  if (e != cudaSuccess) return e;
  if (xb != nullptr)
    e = launch_dependent(csa_compress_kernel<TI, TO, true>, grid, dim3(32 * kCsaWarps), 0, stream, (const TI*)xa,
                         (const TI*)za, (const TI*)xb, (const TI*)zb, ba, bb, tok_off, tok0, ent_off, first, num,
                         max_blocks, (TO*)out, ex, st);
  else
    e = launch_dependent(csa_compress_kernel<TI, TO, false>, grid, dim3(32 * kCsaWarps), 0, stream, (const TI*)xa,
                         (const TI*)za, (const TI*)nullptr, (const TI*)nullptr, ba, bb, tok_off, tok0, ent_off,
                         first, num, max_blocks, (TO*)out, ex, st);
  note_launch();
  return e;
}

cudaError_t launch_csa_compress(const void* xa, const void* za, const void* xb, const void* zb,
                                const float* ba, const float* bb, const int64_t* tok_off,
                                const int64_t* tok0, int batch, const int64_t* ent_off,
                                const int64_t* first, const int64_t* num, int64_t max_blocks,
                                int in_dt, int out_dt, void* out, int norm, const float* gamma, float eps,
                                const void* k_tok, int k_dt, int Di, uint8_t* k_codes, float* k_scale, int flags,
                                int* st, cudaStream_t stream) {
  // many entries: the TMA-ring kernel (one CTA per SM); a few (a decode step): warp per entry.
  // (The overlap flag is a permission: the TMA-ring kernel does not use it.)
  if (max_blocks >= kCsaBulkMinEntries)
    return launch_csa_bulk(xa, za, xb, zb, ba, bb, tok_off, tok0, batch, ent_off, first, num, max_blocks, in_dt,
                           out_dt, out, gamma, eps, norm, k_tok, k_dt, Di, k_codes, k_scale, st, stream);
  CsaExtras ex{norm, gamma, eps, k_tok, k_dt == CSKV_F32, Di, k_codes, k_scale, (flags & CSKV_OVERLAP_PREVIOUS) ? 1 : 0};
  if (in_dt == CSKV_BF16 && out_dt == CSKV_BF16)
    return launch_csa_t<__nv_bfloat16, __nv_bfloat16>(xa, za, xb, zb, ba, bb, tok_off, tok0, batch,
                                                      ent_off, first, num, max_blocks, out, ex, st, stream);
  if (in_dt == CSKV_BF16 && out_dt == CSKV_F32)
    return launch_csa_t<__nv_bfloat16, float>(xa, za, xb, zb, ba, bb, tok_off, tok0, batch, ent_off,
                                              first, num, max_blocks, out, ex, st, stream);
  if (in_dt == CSKV_F32 && out_dt == CSKV_BF16)
    return launch_csa_t<float, __nv_bfloat16>(xa, za, xb, zb, ba, bb, tok_off, tok0, batch, ent_off,
                                              first, num, max_blocks, out, ex, st, stream);
  return launch_csa_t<float, float>(xa, za, xb, zb, ba, bb, tok_off, tok0, batch, ent_off, first, num,
                                    max_blocks, out, ex, st, stream);
}

template <typename TI, typename TO>
static cudaError_t launch_hca_t(const void* x, const void* z, const float* bias, const int64_t* tok_off,
                                const int64_t* tok0, int batch, const int64_t* ent_off,
                                const int64_t* first, const int64_t* num, int64_t max_blocks,
                                void* out, int* st, cudaStream_t stream) {
  // slices of one entry are consecutive CTAs; whole-cache calls run a bounded grid whose
  // CTAs loop over the entries (fewer, longer-lived CTAs keep the copy engines of the SMs busy)
  const int64_t entries = max_blocks < kHcaGridEntries ? max_blocks : kHcaGridEntries;
  dim3 grid((unsigned)(entries * kHcaSlices), (unsigned)batch);
  cudaError_t e = ensure_smem(hca_compress_kernel<TI, TO>, 0);
  if (e != cudaSuccess) return e;
  e = launch_dependent(hca_compress_kernel<TI, TO>, grid, dim3(kHcaThreads), 0, stream,
                                         (const TI*)x, (const TI*)z, bias, tok_off, tok0, ent_off, first, num,
                                         max_blocks, (TO*)out, st);
  note_launch();
  return e;
}

cudaError_t launch_hca_compress(const void* x, const void* z, const float* bias, const int64_t* tok_off,
                                const int64_t* tok0, int batch, const int64_t* ent_off,
                                const int64_t* first, const int64_t* num, int64_t max_blocks,
                                int in_dt, int out_dt, void* out, int norm, const float* gamma, float eps, int* st,
                                cudaStream_t stream) {
  // many entries, or RMSNorm (which needs a whole entry in one CTA): the TMA-ring kernel;
  // a few entries (a decode step): sixteen small CTAs per entry
  if (norm || max_blocks >= kHcaBulkMinEntries)
    return launch_hca_bulk(x, z, bias, tok_off, tok0, batch, ent_off, first, num, max_blocks, in_dt, out_dt, out,
                           gamma, eps, norm, st, stream);
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

template <typename TI, int DPL>
static cudaError_t launch_pool_t(const void* k_tok, const int64_t* tok_off, const int64_t* tok0, int batch,
                                 const int64_t* ent_off, const int64_t* first, const int64_t* num,
                                 int64_t max_blocks, uint8_t* codes, float* scales, int* st, cudaStream_t stream) {
  const int64_t ctas = (max_blocks + kPoolWarps - 1) / kPoolWarps;
  dim3 grid((unsigned)(ctas < kPoolGridCtas ? ctas : kPoolGridCtas), (unsigned)batch);
  cudaError_t e = ensure_smem(pool_keys_kernel<TI, DPL>, 0);
  if (e != cudaSuccess) return e;
  e = launch_dependent(pool_keys_kernel<TI, DPL>, grid, dim3(32 * kPoolWarps), 0, stream, (const TI*)k_tok,
                       tok_off, tok0, ent_off, first, num, max_blocks, codes, scales, st);
  note_launch();
  return e;
}

cudaError_t launch_pool_keys(const void* k_tok, int in_dt, int Di, const int64_t* tok_off, const int64_t* tok0,
                             int batch, const int64_t* ent_off, const int64_t* first, const int64_t* num,
                             int64_t max_blocks, uint8_t* codes, float* scales, int* st, cudaStream_t stream) {
  if (in_dt == CSKV_BF16)
    return Di == 64 ? launch_pool_t<__nv_bfloat16, 2>(k_tok, tok_off, tok0, batch, ent_off, first, num, max_blocks,
                                                      codes, scales, st, stream)
                    : launch_pool_t<__nv_bfloat16, 4>(k_tok, tok_off, tok0, batch, ent_off, first, num, max_blocks,
                                                      codes, scales, st, stream);
  return Di == 64 ? launch_pool_t<float, 2>(k_tok, tok_off, tok0, batch, ent_off, first, num, max_blocks, codes,
                                            scales, st, stream)
                  : launch_pool_t<float, 4>(k_tok, tok_off, tok0, batch, ent_off, first, num, max_blocks, codes,
                                            scales, st, stream);
}

}  // namespace cskv

namespace cskv {

// ------------------------------------------------------------------ RMSNorm of head vectors
// [SW] §十四.3: the queries (and the KV, see the compression epilogues) are RMS-normalised so
// that attention logits cannot blow up: y = x / sqrt(mean(x^2) + eps) * gamma over each
// 128-dimension row (a query head).  A warp per row, a lane per 4 dimensions; fp32 inside.
template <typename T>
__global__ void __launch_bounds__(256) rmsnorm_rows_kernel(const T* __restrict__ x, int64_t rows,
                                                           const float* __restrict__ gamma, float eps,
                                                           T* __restrict__ out) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    float v[4];
    const T* src = x + (size_t)r * kHeadDim + 4 * lane;
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = to_f(src[i]);
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) ss = fmaf(v[i], v[i], ss);
    ss = warp_sum(ss);
    const float rr = rsqrtf(ss * (1.f / kHeadDim) + eps);
    T* dst = out + (size_t)r * kHeadDim + 4 * lane;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float y = v[i] * rr * (gamma ? __ldg(gamma + 4 * lane + i) : 1.f);
      if constexpr (sizeof(T) == 2)
        dst[i] = __float2bfloat16_rn(y);
      else
        dst[i] = y;
    }
  }
}

cudaError_t launch_rmsnorm_rows(const void* x, int dtype, int64_t rows, const float* gamma, float eps, void* out,
                                cudaStream_t stream) {
  const int64_t blocks = (rows + 7) / 8;
  const dim3 grid((unsigned)(blocks < 16384 ? blocks : 16384));
  cudaError_t e;
  if (dtype == CSKV_BF16) {
    e = ensure_smem(rmsnorm_rows_kernel<__nv_bfloat16>, 0);
    if (e == cudaSuccess)
      e = launch_dependent(rmsnorm_rows_kernel<__nv_bfloat16>, grid, dim3(256), 0, stream,
                           (const __nv_bfloat16*)x, rows, gamma, eps, (__nv_bfloat16*)out);
  } else {
    e = ensure_smem(rmsnorm_rows_kernel<float>, 0);
    if (e == cudaSuccess)
      e = launch_dependent(rmsnorm_rows_kernel<float>, grid, dim3(256), 0, stream, (const float*)x, rows, gamma, eps,
                           (float*)out);
  }
  note_launch();
  return e;
}

}  // namespace cskv
