// Compression of many entries at once (a whole cache, a prefill chunk) streamed through TMA
// rings, with two optional epilogues: RMSNorm of each entry's K and V halves, and (CSA) the
// pooling of the per-token indexer keys into E4M3 entry keys.
//
// [SW] = shareware.cn/news/167317 (DeepSeek V4 Hybrid Attention essay): §四/§五 (per-dimension
// softmax weights over a block's tokens; CSA mixes block i through path A with block i-1
// through path B), §三.3 (HCA, 128 tokens per entry), §十四.3 (queries and KV are RMS-normalised
// so that attention logits cannot blow up).  [TR] = trdm.cn/news/516303: §4.3 (CSA two-stream
// overlap, HCA single stream), §4.2 (the indexer's per-token keys pooled to block granularity).
//
// Work decomposition: one CTA per SM, a producer warp and sixteen consumer warps.  The producer
// streams the rows a unit of work needs into a ring stage with TMA bulk copies of 16 KB each
// (each fill completes on the stage's mbarrier; consumers hand a stage back through its release
// counter):
//   CSA: eight entries (bf16; four for fp32): 32 rows of each of x_a, z_a, x_b, z_b, and of the
//        per-token keys;
//   HCA: a quarter entry (bf16; an eighth for fp32): 32 rows of x and of z.
// Consumer thread t owns the packed-dimension pair p = t mod 128 (dims 2p, 2p+1, read as one
// 32-bit bf16 pair or 64-bit fp32 pair) and group g = t / 128: CSA entries g and g+4 of a stage
// (bf16); HCA tokens g, g+4, g+8, ... of every stage, with an online per-dimension softmax that
// the four groups merge at the end of an entry.  The per-element work is one fused logit, one
// max, one exp2 and two accumulations: at ~9 instructions per element the SMs keep up with HBM.
//
// RMSNorm (optional): y = x / sqrt(mean(x^2) + eps) * gamma over the K half (dims 0..127) and
// over the V half (128..255) of every entry separately, on the fp32 value before the output's
// rounding.  The key pooling: mean of the block's tokens (fp32, in token order, one division by
// the count), scale = amax / 448 (1 for an all-zero key), codes E4M3(key / scale) rounded to
// nearest even and saturated -- a warp per entry, lane l owning dims [l*Di/32, (l+1)*Di/32).
#include <cuda_fp8.h>

#include "launch.cuh"
#include "sm100.cuh"

namespace cskv {

constexpr int kBkConsumerWarps = 16;
constexpr int kBkConsumers = 32 * kBkConsumerWarps;  // 512: 128 dimension pairs x 4 groups
constexpr int kBkThreads = kBkConsumers + 32;        // + the producer warp
constexpr int kBkRingBudget = 208 * 1024;
constexpr int kBkMaxStages = 8;
constexpr int kBkCopyBytes = 16 * 1024;  // rows per copy: 16 KB (smaller copies stream slower)

// barrier ids (0 is __syncthreads)
constexpr int kBarConsumers = 1;  // all consumer threads
constexpr int kBarVote = 2;       // consumer-wide OR vote
constexpr int kBarGroup0 = 3;     // the 128 threads of consumer group 0

struct BulkShared {
  uint64_t full[kBkMaxStages];
  unsigned released[kBkMaxStages];
  int err;
  int fills;
  float red[2][kBkConsumerWarps][2];  // RMSNorm partial sums, double-buffered
};

struct BulkArgs {
  const uint8_t* x;   // CSA: x_a; HCA: x
  const uint8_t* z;   // CSA: z_a; HCA: z
  const uint8_t* xb;  // CSA path B (NULL: path A only)
  const uint8_t* zb;
  const float* bias;   // CSA: bias_a [4, 256]; HCA: [128, 256]
  const float* biasb;  // CSA: bias_b
  const int64_t* tok_off;
  const int64_t* tok0;
  const int64_t* ent_off;
  const int64_t* first;
  const int64_t* num;
  int64_t max_blocks;
  void* out;
  const float* gamma;  // RMSNorm gains [256] (K then V), NULL = ones
  float eps;
  int norm;
  const uint8_t* k_tok;  // per-token indexer keys [rows, Di] (NULL: no key pooling)
  int k_f32;             // keys are fp32 (else bf16)
  int Di;
  uint8_t* k_codes;
  float* k_scale;
  int* st;
  int stages;
  int stage_bytes;
};

struct SeqSpan {
  int64_t row0, t0, n, first, num, ent0, ent_cap;
};

__device__ __forceinline__ SeqSpan seq_span(const BulkArgs& a, int b, int ratio) {
  SeqSpan r;
  r.row0 = a.tok_off[b];
  r.t0 = a.tok0 ? a.tok0[b] : 0;
  r.n = r.t0 + (a.tok_off[b + 1] - r.row0);
  const int64_t nent = (r.n + ratio - 1) / ratio;
  r.first = a.first ? a.first[b] : 0;
  r.num = a.num ? a.num[b] : nent - r.first;
  r.ent0 = a.ent_off[b];
  r.ent_cap = a.ent_off[b + 1] - r.ent0;
  if (r.num > a.max_blocks) {  // the excess is skipped and flagged once per sequence
    if (blockIdx.x == 0 && threadIdx.x == 0) flag(a.st, CSKV_DEV_CAPACITY);
    r.num = a.max_blocks;
  }
  return r;
}

// A consumer-wide decision: true when any consumer thread passes true (a named barrier with an
// OR reduction over the consumer warps; the producer warp does not take part).
__device__ __forceinline__ bool consumers_any(bool v) {
  unsigned r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((unsigned)v), "n"(kBarVote), "n"(kBkConsumers)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void bar_named(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Dimensions 2p and 2p+1 of a shared-memory row.
template <typename T>
__device__ __forceinline__ void ld_pair(const uint8_t* row, int p, float& a, float& b) {
  if constexpr (sizeof(T) == 2) {
    const uint32_t w = reinterpret_cast<const uint32_t*>(row)[p];
    a = __uint_as_float(w << 16);
    b = __uint_as_float(w & 0xffff0000u);
  } else {
    const float2 v = reinterpret_cast<const float2*>(row)[p];
    a = v.x;
    b = v.y;
  }
}

template <typename TO>
__device__ __forceinline__ void store_pair(void* out, size_t row, int p, float a, float b) {
  if constexpr (sizeof(TO) == 2) {
    reinterpret_cast<__nv_bfloat162*>(out)[row * (kRow / 2) + p] = __floats2bfloat162_rn(a, b);
  } else {
    reinterpret_cast<float2*>(out)[row * (kRow / 2) + p] = make_float2(a, b);
  }
}

// Bounded wait for the last fill of every stage (after a timeout), then the barriers are retired.
__device__ void bulk_drain(BulkShared& S, int stages) {
  if (threadIdx.x != 0) return;
  bool drained = true;
  if (S.err) {
    const int fills = S.fills;
    for (int s = 0; s < stages && drained; ++s) {
      const int n = fills > s ? (fills - s + stages - 1) / stages : 0;
      if (n > 0) drained = mbar_wait_bounded(&S.full[s], (unsigned)((n - 1) & 1));
    }
  }
  if (drained)
    for (int s = 0; s < stages; ++s)
      asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_u32(&S.full[s])) : "memory");
}

__device__ __forceinline__ void bulk_init(BulkShared& S, int stages) {
  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&S.full[s], 1);
      S.released[s] = 0u;
    }
    S.err = 0;
    S.fills = 0;
    fence_mbar_init();
  }
  __syncthreads();
}

// Ring position shared by the producer and the consumers (no division per stage).
struct RingPos {
  int s = 0;
  unsigned phase = 0;
  unsigned wraps = 0;  // completed passes over the ring
  int it = 0;
  __device__ __forceinline__ void next(int stages) {
    ++it;
    if (++s == stages) {
      s = 0;
      phase ^= 1u;
      ++wraps;
    }
  }
};

// Producer side of one fill: waits for the stage's release by every consumer warp (not on the
// first pass over the ring) and arms its barrier with the bytes the copies will bring.
__device__ __forceinline__ bool producer_acquire(BulkShared& S, const RingPos& r, unsigned bytes, int* st) {
  if (r.wraps > 0 && !wait_released(&S.released[r.s], (unsigned)kBkConsumerWarps * r.wraps, &S.err)) {
    flag(st, CSKV_DEV_TIMEOUT);
    S.err = 1;
    return false;
  }
  mbar_arrive_expect_tx(&S.full[r.s], bytes);
  return true;
}

// Consumer side: waits for the fill; with `uniform` all consumers take the same decision.
__device__ __forceinline__ bool consumer_wait(BulkShared& S, const RingPos& r, bool uniform, int* st) {
  bool gave_up = !mbar_wait_bounded(&S.full[r.s], r.phase);
  if (uniform) gave_up = consumers_any(gave_up);
  if (gave_up) {
    flag(st, CSKV_DEV_TIMEOUT);
    *(volatile int*)&S.err = 1;
  }
  return !gave_up;
}

// RMSNorm factor of one entry whose K and V halves are spread over the consumer warps: `ss` is
// this thread's sum of squares, `half_w0` the first of the two warps holding this thread's half
// of the entry; `slot` selects the red buffer entry.  Barrier `bar_id` over `bar_count` threads.
__device__ __forceinline__ float rms_factor(float ss, BulkShared& S, int buf, int slot, int half_w0, int bar_id,
                                            int bar_count, float eps) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  if (lane == 0) S.red[buf][warp][slot] = ss;
  bar_named(bar_id, bar_count);
  const float tot = S.red[buf][half_w0][slot] + S.red[buf][half_w0 + 1][slot];
  return rsqrtf(tot * (1.f / 128.f) + eps);
}

// ------------------------------------------------------------------ CSA (4:1, two streams)
// Stage layout: [x_a 4E rows][z_a 4E rows][x_b 4E rows][z_b 4E rows][keys 4E rows x Di].
// Row r of the A part is token 4*i_lo + r, row r of the B part token 4*i_lo - 4 + r.
template <typename T>
struct CsaTile {
  static constexpr int RB = kRow * (int)sizeof(T);   // row bytes
  static constexpr int E = kBkCopyBytes / (4 * RB);  // entries per stage: 8 (bf16), 4 (fp32)
  static constexpr int AR = 4 * E;                   // rows per part
  static constexpr int EPT = E / 4;                  // entries per consumer thread
};

// Entry i of the sequence can be computed from the rows provided (else flagged once).
__device__ __forceinline__ bool csa_entry_ok(const SeqSpan& sp, int64_t i, bool two, int* st, bool report) {
  if (i < 0 || 4 * i >= sp.n || i >= sp.ent_cap) {
    if (report) flag(st, CSKV_DEV_BAD_INDEX);
    return false;
  }
  if (4 * i < sp.t0 || (two && i >= 1 && 4 * i - 4 < sp.t0)) {
    if (report) flag(st, CSKV_DEV_TAIL_MISSING);
    return false;
  }
  return true;
}

template <typename T, typename TO, bool kTwo>
__global__ void __launch_bounds__(kBkThreads, 1) csa_bulk_kernel(BulkArgs a) {
  using Tl = CsaTile<T>;
  constexpr int RB = Tl::RB, E = Tl::E, AR = Tl::AR, EPT = Tl::EPT;
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ BulkShared S;
  const int b = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  bulk_init(S, a.stages);
  pdl_wait();
  const SeqSpan sp = seq_span(a, b, 4);
  const int kb = a.k_tok ? a.Di * (a.k_f32 ? 4 : 2) : 0;  // key row bytes
  const int64_t nchunks = (sp.num + E - 1) / E;
  RingPos rp;
  if (warp == kBkConsumerWarps) {
    // ---------------- producer
    if (lane == 0) {
      for (int64_t c = blockIdx.x; c < nchunks; c += gridDim.x, rp.next(a.stages)) {
        const int64_t i_lo = sp.first + c * E;
        const int64_t i_hi = i_lo + min((int64_t)E, sp.num - c * E);
        const int64_t a0 = max(max(4 * i_lo, sp.t0), (int64_t)0), a1 = min(4 * i_hi, sp.n);
        const int64_t b0 = max(max(4 * i_lo - 4, sp.t0), (int64_t)0), b1 = min(4 * i_hi - 4, sp.n);
        const unsigned na = a0 < a1 ? (unsigned)(a1 - a0) : 0u;
        const unsigned nb = (kTwo && b0 < b1) ? (unsigned)(b1 - b0) : 0u;
        if (!producer_acquire(S, rp, na * (2u * RB + kb) + nb * 2u * RB, a.st)) break;
        uint8_t* st = ring + (size_t)rp.s * a.stage_bytes;
        uint64_t* bar = &S.full[rp.s];
        if (na) {
          const size_t r = (size_t)(sp.row0 + a0 - sp.t0), o = (size_t)(a0 - 4 * i_lo);
          tma_bulk_g2s(st + o * RB, a.x + r * RB, na * RB, bar);
          tma_bulk_g2s(st + (AR + o) * RB, a.z + r * RB, na * RB, bar);
          if (kb) tma_bulk_g2s(st + 4 * AR * RB + o * kb, a.k_tok + r * kb, na * kb, bar);
        }
        if (nb) {
          const size_t r = (size_t)(sp.row0 + b0 - sp.t0), o = (size_t)(b0 - (4 * i_lo - 4));
          tma_bulk_g2s(st + (2 * AR + o) * RB, a.xb + r * RB, nb * RB, bar);
          tma_bulk_g2s(st + (3 * AR + o) * RB, a.zb + r * RB, nb * RB, bar);
        }
      }
      S.fills = rp.it;
    }
  } else {
    // ---------------- consumers: dimension pair p, entries g, g + 4 of every stage
    const int p = tid & 127, g = tid >> 7;
    // position biases in log2 units: logit * log2(e) = fma(z, log2(e), bias * log2(e))
    float ba[4][2], bb[4][2];
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        ba[c][h] = a.bias ? __ldg(a.bias + c * kRow + 2 * p + h) * kLog2e : 0.f;
        bb[c][h] = (kTwo && a.biasb) ? __ldg(a.biasb + c * kRow + 2 * p + h) * kLog2e : 0.f;
      }
    const float g0 = a.gamma ? __ldg(a.gamma + 2 * p) : 1.f, g1 = a.gamma ? __ldg(a.gamma + 2 * p + 1) : 1.f;
    const bool uniform = a.norm != 0;  // the norm's barriers: leave together on a timeout
    int nbuf = 0;
    for (int64_t c = blockIdx.x; c < nchunks; c += gridDim.x, rp.next(a.stages)) {
      if (!consumer_wait(S, rp, uniform, a.st)) break;
      const uint8_t* st = ring + (size_t)rp.s * a.stage_bytes;
      const int64_t i_lo = sp.first + c * E;
      float o[EPT][2];
      bool ok[EPT];
#pragma unroll
      for (int k = 0; k < EPT; ++k) {
        const int e = g + 4 * k;
        const int64_t i = i_lo + e;
        o[k][0] = o[k][1] = 0.f;
        ok[k] = c * E + e < sp.num && csa_entry_ok(sp, i, kTwo, a.st, p == 0);
        if (!ok[k]) continue;  // warp-uniform
        const int cntA = (int)min((int64_t)4, sp.n - 4 * i);
        const bool hasB = kTwo && i >= 1;
        constexpr int C = kTwo ? 8 : 4;
        float l[C][2], x[C][2];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float z0, z1;
          ld_pair<T>(st + (size_t)(AR + 4 * e + q) * RB, p, z0, z1);
          ld_pair<T>(st + (size_t)(4 * e + q) * RB, p, x[q][0], x[q][1]);
          l[q][0] = fmaf(z0, kLog2e, ba[q][0]);
          l[q][1] = fmaf(z1, kLog2e, ba[q][1]);
          if constexpr (kTwo) {
            ld_pair<T>(st + (size_t)(3 * AR + 4 * e + q) * RB, p, z0, z1);
            ld_pair<T>(st + (size_t)(2 * AR + 4 * e + q) * RB, p, x[4 + q][0], x[4 + q][1]);
            l[4 + q][0] = fmaf(z0, kLog2e, bb[q][0]);
            l[4 + q][1] = fmaf(z1, kLog2e, bb[q][1]);
          }
        }
        if (cntA < 4 || (kTwo && !hasB)) {  // entry 0, or a partial last block: mask absent candidates
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (q >= cntA) l[q][0] = l[q][1] = -INFINITY;
            if constexpr (kTwo)
              if (!hasB) l[4 + q][0] = l[4 + q][1] = -INFINITY;
          }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float m = l[0][h];
#pragma unroll
          for (int q = 1; q < C; ++q) m = fmaxf(m, l[q][h]);
          float den = 0.f, num = 0.f;
#pragma unroll
          for (int q = 0; q < C; ++q) {
            const float w = fast_exp2(l[q][h] - m);  // -inf -> 0
            den += w;
            num = fmaf(w, x[q][h], num);
          }
          o[k][h] = __fdividef(num, den);
        }
      }
      // key pooling: warp w < E pools entry w of the stage
      uint32_t kcodes = 0;
      float kscale = 1.f;
      bool kok = false;
      if (kb && warp < E) {
        const int64_t i = i_lo + warp;
        kok = c * E + warp < sp.num && csa_entry_ok(sp, i, kTwo, a.st, false);
        if (kok) {
          const int cnt = (int)min((int64_t)4, sp.n - 4 * i);
          const int dpl = a.Di / 32;
          float key[4] = {0.f, 0.f, 0.f, 0.f};
          float amax = 0.f;
          const uint8_t* row0 = st + 4 * AR * RB + (size_t)(4 * warp) * kb;
#pragma unroll
          for (int d = 0; d < 4; ++d) {
            if (d < dpl) {
              const int col = lane * dpl + d;
              float acc = 0.f;
              for (int q = 0; q < cnt; ++q) {
                const uint8_t* rq = row0 + (size_t)q * kb;
                const float v = a.k_f32 ? reinterpret_cast<const float*>(rq)[col]
                                        : __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(rq)[col] << 16);
                acc = q == 0 ? v : __fadd_rn(acc, v);
              }
              key[d] = __fdiv_rn(acc, (float)cnt);
              amax = fmaxf(amax, fabsf(key[d]));
            }
          }
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
          kscale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
#pragma unroll
          for (int d = 0; d < 4; ++d)
            if (d < dpl)
              kcodes |= (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(key[d], kscale), __NV_SATFINITE, __NV_E4M3)
                        << (8 * d);
        }
      }
      // every read of the stage is done: hand it back
      __syncwarp();
      if (lane == 0) release_stage(&S.released[rp.s]);
      if (a.norm) {
        // K half: pairs 0..63 (warps 4g, 4g+1 of this group); V half: pairs 64..127
        const int half_w0 = 4 * g + (p >= 64 ? 2 : 0);
        float r[EPT];
#pragma unroll
        for (int k = 0; k < EPT; ++k)
          r[k] = rms_factor(fmaf(o[k][0], o[k][0], o[k][1] * o[k][1]), S, nbuf, k, half_w0, kBarConsumers,
                            kBkConsumers, a.eps);
#pragma unroll
        for (int k = 0; k < EPT; ++k) {
          o[k][0] *= r[k] * g0;
          o[k][1] *= r[k] * g1;
        }
        nbuf ^= 1;
      }
#pragma unroll
      for (int k = 0; k < EPT; ++k)
        if (ok[k]) store_pair<TO>(a.out, (size_t)(sp.ent0 + i_lo + g + 4 * k), p, o[k][0], o[k][1]);
      if (kok) {
        const int64_t row = sp.ent0 + i_lo + warp;
        const int dpl = a.Di / 32;
        uint8_t* dst = a.k_codes + (size_t)row * a.Di + lane * dpl;
        if (dpl == 2)
          *reinterpret_cast<uint16_t*>(dst) = (uint16_t)kcodes;
        else
          *reinterpret_cast<uint32_t*>(dst) = kcodes;
        if (lane == 0) a.k_scale[row] = kscale;
      }
    }
  }
  __syncthreads();
  bulk_drain(S, a.stages);
}

// ------------------------------------------------------------------ HCA (128:1, one stream)
// Work item: R consecutive tokens of one entry (stage layout [x R rows][z R rows]); an entry is
// 128 / R stages (fewer for a partial last block).  Group g of the consumers takes tokens
// g, g+4, ... of every stage and carries its own online softmax (running max, sum and weighted
// sum, log2 units) for dims 2p, 2p+1; at the end of the entry groups 1-3 hand their state to
// group 0 through shared memory, which merges, normalises and stores.
template <typename T>
struct HcaTile {
  static constexpr int RB = kRow * (int)sizeof(T);
  static constexpr int R = kBkCopyBytes / RB;  // tokens per stage: 32 (bf16), 16 (fp32)
  static constexpr int TPG = R / 4;            // tokens per group and stage
};

struct HcaMerge {
  float v[2][3][6][128];  // [entry parity][group 1..3][m0 m1 den0 den1 num0 num1][pair]
};

__device__ __forceinline__ bool hca_entry_ok(const SeqSpan& sp, int64_t i, int* st, bool report) {
  if (i < 0 || 128 * i >= sp.n || i >= sp.ent_cap) {
    if (report) flag(st, CSKV_DEV_BAD_INDEX);
    return false;
  }
  if (128 * i < sp.t0) {
    if (report) flag(st, CSKV_DEV_TAIL_MISSING);
    return false;
  }
  return true;
}

// One stage of one group: tokens g, g+4, ... (< nr) of the stage, dims 2p and 2p+1.
template <typename T, bool kBias>
__device__ __forceinline__ void hca_stage(const uint8_t* st, int p, int g, int nr, int slot0, const float* bias,
                                          float (&m)[2], float (&den)[2], float (&num)[2]) {
  using Tl = HcaTile<T>;
  constexpr int RB = Tl::RB, R = Tl::R, TPG = Tl::TPG;
  float l[TPG][2], x[TPG][2];
  float ms0 = -INFINITY, ms1 = -INFINITY;
#pragma unroll
  for (int k = 0; k < TPG; ++k) {
    const int r = g + 4 * k;
    float z0, z1;
    ld_pair<T>(st + (size_t)(R + r) * RB, p, z0, z1);
    ld_pair<T>(st + (size_t)r * RB, p, x[k][0], x[k][1]);
    float b0 = 0.f, b1 = 0.f;
    if constexpr (kBias) {
      const float2 bv = __ldg(reinterpret_cast<const float2*>(bias + (size_t)(slot0 + r) * kRow) + p);
      b0 = bv.x * kLog2e;
      b1 = bv.y * kLog2e;
    }
    l[k][0] = r < nr ? fmaf(z0, kLog2e, b0) : -INFINITY;
    l[k][1] = r < nr ? fmaf(z1, kLog2e, b1) : -INFINITY;
    ms0 = fmaxf(ms0, l[k][0]);
    ms1 = fmaxf(ms1, l[k][1]);
  }
  const float mn0 = fmaxf(m[0], ms0), mn1 = fmaxf(m[1], ms1);
  // a group may hold no token of a stage (a partial block): its state then stays as it was
  if (mn0 != -INFINITY) {
    const float f = fast_exp2(m[0] - mn0);  // m = -inf before the first token -> 0
    float d = den[0] * f, s = num[0] * f;
#pragma unroll
    for (int k = 0; k < TPG; ++k) {
      const float w = fast_exp2(l[k][0] - mn0);
      d += w;
      s = fmaf(w, x[k][0], s);
    }
    den[0] = d;
    num[0] = s;
    m[0] = mn0;
  }
  if (mn1 != -INFINITY) {
    const float f = fast_exp2(m[1] - mn1);
    float d = den[1] * f, s = num[1] * f;
#pragma unroll
    for (int k = 0; k < TPG; ++k) {
      const float w = fast_exp2(l[k][1] - mn1);
      d += w;
      s = fmaf(w, x[k][1], s);
    }
    den[1] = d;
    num[1] = s;
    m[1] = mn1;
  }
}

template <typename T, typename TO>
__global__ void __launch_bounds__(kBkThreads, 1) hca_bulk_kernel(BulkArgs a) {
  using Tl = HcaTile<T>;
  constexpr int RB = Tl::RB, R = Tl::R;
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ BulkShared S;
  __shared__ HcaMerge M;
  const int b = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  bulk_init(S, a.stages);
  pdl_wait();
  const SeqSpan sp = seq_span(a, b, 128);
  RingPos rp;
  if (warp == kBkConsumerWarps) {
    if (lane == 0) {
      bool stop = false;
      for (int64_t local = blockIdx.x; local < sp.num && !stop; local += gridDim.x) {
        const int64_t i = sp.first + local;
        if (!hca_entry_ok(sp, i, a.st, false)) continue;
        const int64_t ntok = min((int64_t)128, sp.n - 128 * i);
        for (int64_t t = 0; t < ntok; t += R, rp.next(a.stages)) {
          const unsigned nr = (unsigned)min((int64_t)R, ntok - t);
          if (!producer_acquire(S, rp, nr * 2u * RB, a.st)) {
            stop = true;
            break;
          }
          uint8_t* st = ring + (size_t)rp.s * a.stage_bytes;
          const size_t r = (size_t)(sp.row0 + 128 * i + t - sp.t0);
          tma_bulk_g2s(st, a.x + r * RB, nr * RB, &S.full[rp.s]);
          tma_bulk_g2s(st + (size_t)R * RB, a.z + r * RB, nr * RB, &S.full[rp.s]);
        }
      }
      S.fills = rp.it;
    }
  } else {
    const int p = tid & 127, g = tid >> 7;
    const float g0 = a.gamma ? __ldg(a.gamma + 2 * p) : 1.f, g1 = a.gamma ? __ldg(a.gamma + 2 * p + 1) : 1.f;
    int par = 0;  // entry parity: merge and norm buffers
    bool stop = false;
    for (int64_t local = blockIdx.x; local < sp.num && !stop; local += gridDim.x) {
      const int64_t i = sp.first + local;
      if (!hca_entry_ok(sp, i, a.st, tid == 0)) continue;  // uniform across the consumers
      const int64_t ntok = min((int64_t)128, sp.n - 128 * i);
      float m[2] = {-INFINITY, -INFINITY}, den[2] = {0.f, 0.f}, num[2] = {0.f, 0.f};
      for (int64_t t = 0; t < ntok; t += R, rp.next(a.stages)) {
        // the merge barrier below is met every entry: consumers leave together on a timeout
        if (!consumer_wait(S, rp, true, a.st)) {
          stop = true;
          break;
        }
        const uint8_t* st = ring + (size_t)rp.s * a.stage_bytes;
        const int nr = (int)min((int64_t)R, ntok - t);
        if (a.bias)
          hca_stage<T, true>(st, p, g, nr, (int)t, a.bias, m, den, num);
        else
          hca_stage<T, false>(st, p, g, nr, (int)t, nullptr, m, den, num);
        __syncwarp();
        if (lane == 0) release_stage(&S.released[rp.s]);
      }
      if (stop) break;
      // ---- merge the four groups' states into group 0
      if (g > 0) {
        float* v = &M.v[par][g - 1][0][p];
        v[0 * 128] = m[0];
        v[1 * 128] = m[1];
        v[2 * 128] = den[0];
        v[3 * 128] = den[1];
        v[4 * 128] = num[0];
        v[5 * 128] = num[1];
      }
      bar_named(kBarConsumers, kBkConsumers);
      if (g == 0) {
        float o[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float mm = m[h];
#pragma unroll
          for (int q = 0; q < 3; ++q) mm = fmaxf(mm, M.v[par][q][h][p]);  // finite: token 128i is present
          float d = m[h] == -INFINITY ? 0.f : den[h] * fast_exp2(m[h] - mm);
          float s = m[h] == -INFINITY ? 0.f : num[h] * fast_exp2(m[h] - mm);
#pragma unroll
          for (int q = 0; q < 3; ++q) {
            const float mq = M.v[par][q][h][p];
            if (mq != -INFINITY) {
              const float f = fast_exp2(mq - mm);
              d = fmaf(M.v[par][q][2 + h][p], f, d);
              s = fmaf(M.v[par][q][4 + h][p], f, s);
            }
          }
          o[h] = __fdividef(s, d);
        }
        if (a.norm) {
          // group 0 holds the whole entry: K in warps 0-1, V in warps 2-3
          const float r = rms_factor(fmaf(o[0], o[0], o[1] * o[1]), S, par, 0, p >= 64 ? 2 : 0, kBarGroup0, 128,
                                     a.eps);
          o[0] *= r * g0;
          o[1] *= r * g1;
        }
        store_pair<TO>(a.out, (size_t)(sp.ent0 + i), p, o[0], o[1]);
      }
      par ^= 1;
    }
  }
  __syncthreads();
  bulk_drain(S, a.stages);
}

// ------------------------------------------------------------------ host side
static int bulk_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return sms;
}

template <typename K>
static cudaError_t launch_bulk(K kern, BulkArgs a, int batch, int64_t per_seq_units, cudaStream_t stream) {
  const int sms = bulk_sms();
  if (sms == 0) return cudaErrorNoDevice;
  a.stages = kBkRingBudget / a.stage_bytes;
  if (a.stages > kBkMaxStages) a.stages = kBkMaxStages;
  if (a.stages < 2) return cudaErrorInvalidValue;
  const size_t smem = (size_t)a.stages * a.stage_bytes;
  cudaError_t e = ensure_smem(kern, smem);
  if (e != cudaSuccess) return e;
  int64_t gx = batch >= sms ? 1 : sms / batch;
  if (gx > per_seq_units) gx = per_seq_units;
  if (gx < 1) gx = 1;
  e = launch_dependent(kern, dim3((unsigned)gx, (unsigned)batch), dim3(kBkThreads), smem, stream, a);
  note_launch();
  return e;
}

cudaError_t launch_csa_bulk(const void* xa, const void* za, const void* xb, const void* zb, const float* ba,
                            const float* bb, const int64_t* tok_off, const int64_t* tok0, int batch,
                            const int64_t* ent_off, const int64_t* first, const int64_t* num, int64_t max_blocks,
                            int in_dt, int out_dt, void* out, const float* gamma, float eps, int norm,
                            const void* k_tok, int k_dt, int Di, uint8_t* k_codes, float* k_scale, int* st,
                            cudaStream_t stream) {
  BulkArgs a = {};
  a.x = (const uint8_t*)xa;
  a.z = (const uint8_t*)za;
  a.xb = (const uint8_t*)xb;
  a.zb = (const uint8_t*)zb;
  a.bias = ba;
  a.biasb = bb;
  a.tok_off = tok_off;
  a.tok0 = tok0;
  a.ent_off = ent_off;
  a.first = first;
  a.num = num;
  a.max_blocks = max_blocks;
  a.out = out;
  a.gamma = gamma;
  a.eps = eps;
  a.norm = norm;
  a.k_tok = (const uint8_t*)k_tok;
  a.k_f32 = k_dt == CSKV_F32;
  a.Di = Di;
  a.k_codes = k_codes;
  a.k_scale = k_scale;
  a.st = st;
  const bool bf_in = in_dt == CSKV_BF16;
  const int E = bf_in ? CsaTile<__nv_bfloat16>::E : CsaTile<float>::E;
  const int kb = k_tok ? Di * (k_dt == CSKV_F32 ? 4 : 2) : 0;
  a.stage_bytes = 4 * kBkCopyBytes + 4 * E * kb;
  const int64_t units = (max_blocks + E - 1) / E;
  using bf = __nv_bfloat16;
  if (bf_in && out_dt == CSKV_BF16)
    return xb ? launch_bulk(csa_bulk_kernel<bf, bf, true>, a, batch, units, stream)
              : launch_bulk(csa_bulk_kernel<bf, bf, false>, a, batch, units, stream);
  if (bf_in)
    return xb ? launch_bulk(csa_bulk_kernel<bf, float, true>, a, batch, units, stream)
              : launch_bulk(csa_bulk_kernel<bf, float, false>, a, batch, units, stream);
  if (out_dt == CSKV_BF16)
    return xb ? launch_bulk(csa_bulk_kernel<float, bf, true>, a, batch, units, stream)
              : launch_bulk(csa_bulk_kernel<float, bf, false>, a, batch, units, stream);
  return xb ? launch_bulk(csa_bulk_kernel<float, float, true>, a, batch, units, stream)
            : launch_bulk(csa_bulk_kernel<float, float, false>, a, batch, units, stream);
}

cudaError_t launch_hca_bulk(const void* x, const void* z, const float* bias, const int64_t* tok_off,
                            const int64_t* tok0, int batch, const int64_t* ent_off, const int64_t* first,
                            const int64_t* num, int64_t max_blocks, int in_dt, int out_dt, void* out,
                            const float* gamma, float eps, int norm, int* st, cudaStream_t stream) {
  BulkArgs a = {};
  a.x = (const uint8_t*)x;
  a.z = (const uint8_t*)z;
  a.bias = bias;
  a.tok_off = tok_off;
  a.tok0 = tok0;
  a.ent_off = ent_off;
  a.first = first;
  a.num = num;
  a.max_blocks = max_blocks;
  a.out = out;
  a.gamma = gamma;
  a.eps = eps;
  a.norm = norm;
  a.st = st;
  a.stage_bytes = 2 * kBkCopyBytes;
  using bf = __nv_bfloat16;
  if (in_dt == CSKV_BF16 && out_dt == CSKV_BF16)
    return launch_bulk(hca_bulk_kernel<bf, bf>, a, batch, max_blocks, stream);
  if (in_dt == CSKV_BF16) return launch_bulk(hca_bulk_kernel<bf, float>, a, batch, max_blocks, stream);
  if (out_dt == CSKV_BF16) return launch_bulk(hca_bulk_kernel<float, bf>, a, batch, max_blocks, stream);
  return launch_bulk(hca_bulk_kernel<float, float>, a, batch, max_blocks, stream);
}

}  // namespace cskv
