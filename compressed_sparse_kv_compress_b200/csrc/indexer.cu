// Lightning Indexer scan fused with an exact top-k.
//
// [SW] = shareware.cn/news/167317 (DeepSeek V4 Hybrid Attention essay): §六 (cheap
// scoring of every compressed entry, then top-k, then the main attention; low
// precision), §七 (ReLU per head before the heads are summed), §十 (a query sees
// complete blocks only).  [TR] = trdm.cn/news/516303, §4.2 (LightningIndexer:
// scores = relu(q_idx k_idx^T), FP8).  [AM] = aimodeling.com DeepSeek V4 news (k = 1024).
//
// Query t sees CSA entries i < V_t = floor((p_t + 1) / 4) and scores
//     s_i = sum_h w_h * ReLU(sq_h * sk_i * <q_h, k_i>).
// The min(k, V_t) best entries are kept (equal scores: lower index first) and written
// in ascending index order, padded with -1.
//
// Work decomposition.  A query's entries are cut into contiguous segments, one per
// CTA; the CTAs of one query form a group.
//  * split mode (few queries, decode): one round, every CTA of a cooperative grid
//    gets one segment, groups sized in proportion to V_t;
//  * row mode (many queries, prefill): every CTA owns whole queries (group of one)
//    and loops over them.
// A segment's scores never leave shared memory.  Keys are 64-bit (order-preserving score
// bits << 32 | ~index), so a selection "key >= threshold" resolves ties to the lower index
// exactly.
//  * a group of one CTA: most-significant-digit radix select in shared memory;
//  * a group of several CTAs, speculative exchange: every CTA proposes its best keys (the
//    top bins of a linear histogram of its own scores) into fixed slots and publishes the
//    best key it kept back; after one group barrier every CTA gathers all slots, finds the
//    exact k-th proposal T* and, when no CTA kept back a key >= T*, emits its keys >= T* at
//    positions counted from the lower CTAs' proposals;
//  * otherwise (winners crowded into a few segments, massive ties) the exact path: a 12-bit
//    digit histogram of the group (global atomics, group barrier), compaction of the
//    threshold bin's entries when they fit (second barrier), else further 10-bit global
//    passes.  Output positions come from per-CTA counts, so the result needs no sort.
// As kept entries are emitted, their rows of an optional array (the compressed CSA cache that
// the attention gathers next) are prefetched into L2.
//
// Scan of E4M3 keys: a producer warp streams 240-entry tiles (15 KiB at Di = 64) of k_idx into a
// shared-memory ring with TMA bulk copies (each fill completes on the stage's mbarrier; the
// consumers hand a stage back through its release counter); fifteen consumer warps each take 16 entries of
// a tile and run m16n8k32 E4M3 MMAs (entries x dims) x (dims x 8 heads) with fp32
// accumulation -- the head dimension fills N = 8 exactly -- then apply scales, ReLU and
// the head sum in registers.
#include <type_traits>

#include "launch.cuh"
#include "sm100.cuh"

namespace cskv {

// 15 MMA warps + 1 TMA warp = 16 warps, 4 per SM sub-partition: with at most 88 registers a
// thread the indexer leaves 5120 registers on every sub-partition, so a 4-warp attention
// CTA (<= 160 registers) or compression CTAs fit beside it on the same SM.
constexpr int kIdxConsumerWarps = 15;
constexpr int kIdxThreads = 32 * (kIdxConsumerWarps + 1);  // + one producer warp
constexpr int kIdxTile = 16 * kIdxConsumerWarps;          // entries per ring stage
constexpr int kBins0 = 4096;                              // first digit: 12 bits
constexpr int kBinsP = 1024;                              // later digits: 10 bits
constexpr int kMaxPasses = 7;                             // 12 + 5 * 10 + 2 = 64 bits
constexpr int kCandMax = 4096;  // candidates exchanged per query group (global and shared)
constexpr int kMaxGroup = 1024;
constexpr int kMinSeg = 256;
constexpr int kMaxSplitQueries = 128;
constexpr int kIdxMaxHeads = 16;
constexpr int kIdxMaxDim = 128;

enum IdxSrc { kSrcFp8 = 0, kSrcF32 = 1, kSrcScores = 2, kSrcFp4 = 3 };


struct alignas(16) QueryWS {
  unsigned bar_count, spare, done, cand_count;  // bar_count: group barrier (phase bit + arrivals)
  unsigned hist0[kBins0];
  unsigned histp[kMaxPasses - 1][kBinsP];
  unsigned above[kMaxGroup];
  unsigned long long unp[kMaxGroup];   // speculative path: best key each CTA did not propose
  unsigned long long cand[kCandMax];   // speculative path: `cap` proposal slots per CTA
};


// TMA ring depth: at least 64 KiB of k_idx tiles in flight per CTA whatever Di is; deeper (up
// to kIdxMaxStages, the whole segment when it fits) where shared memory allows (run_topk).
__host__ __device__ constexpr int idx_stages(int Di) { return (64 * 1024) / (kIdxTile * Di); }
constexpr int kIdxMaxStages = 16;

// Layout of the shared region after the scan: histogram, candidate keys, then a scratch
// area used first as the owner table of the gathered proposals, then for the keys of the
// threshold bin.
constexpr size_t kUnHist = 0;
constexpr size_t kUnCand = (size_t)kBins0 * 4;
constexpr size_t kUnAux = kUnCand + (size_t)kCandMax * 8;
constexpr int kAuxKeys = 1024;  // 8 KiB: kCandMax owner entries (2 B) or kAuxKeys keys (8 B)
constexpr size_t kUnSelBytes = kUnAux + (size_t)kAuxKeys * 8;

// Bytes of the shared region used first as the TMA ring (`stages` tiles), then for the
// histogram and the candidate keys.
__host__ __device__ constexpr size_t idx_union_bytes(int Di, int stages) {
  return (size_t)stages * kIdxTile * Di > kUnSelBytes ? (size_t)stages * kIdxTile * Di : kUnSelBytes;
}

// ------------------------------------------------------------------ MXFP4 helpers
// Four E2M1 codes (code i in bits 4i..4i+3: sign bit 3, exponent bits 2..1 with bias 1,
// mantissa bit 0; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6) -> the four E4M3 bytes of the same
// values (every E2M1 value is exact in E4M3): a byte permute over the table of the eight
// magnitudes' E4M3 codes, then the sign bits moved to bit 7 of each byte.
__device__ __forceinline__ uint32_t e2m1x4_to_e4m3x4(uint32_t c) {
  const uint32_t mag = __byte_perm(0x3C383000u, 0x4C484440u, c & 0x7777u);
  const uint32_t spread = (c & 0x000Fu) | ((c & 0x00F0u) << 4) | ((c & 0x0F00u) << 8) | ((c & 0xF000u) << 12);
  return mag | ((spread << 4) & 0x80808080u);
}
// E8M0 scale code -> 2^(code - 127) (code 0 is the subnormal 2^-127, 0xFF is NaN).
__device__ __forceinline__ float e8m0_to_float(uint32_t c) {
  return c == 0u ? __uint_as_float(0x00400000u) : (c == 255u ? __uint_as_float(0x7fc00000u) : __uint_as_float(c << 23));
}

// ------------------------------------------------------------------ keys
__device__ __forceinline__ uint32_t score_key(float s) {
  uint32_t u = __float_as_uint(s);
  if (u == 0x80000000u) u = 0u;  // -0 ranks with +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ uint64_t comp_key(float s, int64_t e) {
  return ((uint64_t)score_key(s) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)e);
}
// Score of a composite key (inverse of score_key on the top 32 bits).
__device__ __forceinline__ float key_score(uint64_t c) {
  const uint32_t k = (uint32_t)(c >> 32);
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}
__device__ __forceinline__ bool key_selected(uint64_t c, uint64_t P, int nb) {
  return (c >> (64 - nb)) >= P;
}

// ------------------------------------------------------------------ block helpers
// Copies n values global -> shared with 8 loads in flight per thread (a loop that stores
// each value before loading the next would pay one memory round trip per iteration).
template <bool kCG, typename T>
__device__ __forceinline__ void copy_to_smem(T* dst, const T* src, int n, int tid, int nthr) {
  constexpr int U = 8;
  for (int b = tid; b < n; b += nthr * U) {
    T v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = b + u * nthr;
      if (i < n) v[u] = kCG ? __ldcg(src + i) : __ldg(src + i);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = b + u * nthr;
      if (i < n) dst[i] = v[u];
    }
  }
}

// Exclusive prefix sum over threads in thread order; *total receives the sum.  Two block
// barriers: the warp totals are published once, and `red` is free again on return.
__device__ unsigned block_excl_scan(unsigned v, unsigned* red, unsigned* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int nw = kIdxThreads / 32;
  unsigned x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) red[warp] = x;
  __syncthreads();
  unsigned before = x - v, tot = 0;
  for (int w = 0; w < nw; ++w) {
    const unsigned r = red[w];
    before += w < warp ? r : 0u;
    tot += r;
  }
  if (total) *total = tot;
  __syncthreads();
  return before;
}

// Shared-memory histogram increment (called warp-uniformly).
__device__ __forceinline__ void hist_add(unsigned* hist, unsigned bin, bool active) {
  if (active) atomicAdd(&hist[bin], 1u);
}

struct Crossing {
  unsigned bin, above, cnt;
};

// hist[nbins] in shared memory; finds the bin where the count accumulated from the
// highest bin downwards first reaches r (1 <= r <= sum of hist).  Two block barriers;
// `red` (>= 9 words) must not be used by anything else until the next barrier after return.
__device__ Crossing find_crossing(const unsigned* hist, int nbins, unsigned r, unsigned* red, Crossing* out) {
  const int per = nbins >= 512 ? nbins / 512 : 1;
  const int nthr = nbins / per;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  unsigned local = 0;
  int hi = 0, lo = 0;
  if (tid < nthr) {
    hi = nbins - tid * per;  // exclusive
    lo = hi - per;
    for (int b = hi - 1; b >= lo; --b) local += hist[b];
  }
  unsigned x = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) red[warp] = x;
  if (tid == 0) {  // safe default if a corrupted histogram never reaches r
    out->bin = 0;
    out->above = 0;
    out->cnt = r;
  }
  __syncthreads();
  unsigned excl = x - local;
  for (int w = 0; w < warp; ++w) excl += red[w];
  if (tid < nthr && local > 0 && excl < r && r <= excl + local) {
    unsigned cum = excl;
    for (int b = hi - 1; b >= lo; --b) {
      const unsigned h = hist[b];
      if (cum + h >= r) {
        out->bin = (unsigned)b;
        out->above = cum;
        out->cnt = h;
        break;
      }
      cum += h;
    }
  }
  __syncthreads();
  return *out;
}

// Barrier over the G CTAs of one query group (all co-resident: cooperative launch), on one
// counter whose top bit is the barrier's phase.  Thread 0 arrives with one atomic add that is a
// release (it publishes the CTA's writes) and returns the counter before it, whose phase bit is
// the phase being completed (it cannot change before this CTA arrives): CTA 0 of the group adds
// 2^31 - (G - 1), every other CTA adds 1, so the sum of the G arrivals is exactly 2^31 -- the
// phase bit flips when the last one lands and the low bits are back where they were (zero), for
// any G, with no reset.  Waiters poll (acquire) until the phase differs.  Bounded:
// gives up after a few million polls, about a second (CSKV_DEV_TIMEOUT).
__device__ bool group_barrier(QueryWS* ws, unsigned G, int j, int* st, int* sm_flag) {
  __syncthreads();
  if (threadIdx.x == 0) {
    bool ok = true;
    const unsigned add = j == 0 ? 0x80000000u - (G - 1u) : 1u;
    // the arrival is a release (cumulative over the block barrier before it: every write of the
    // CTA is visible before it) and returns the counter, whose top bit is the phase this CTA
    // arrives in
    unsigned before;
    asm volatile("atom.add.release.gpu.global.u32 %0, [%1], %2;" : "=r"(before) : "l"(&ws->bar_count), "r"(add) : "memory");
    long it = 0;
    while (((ld_acquire_gpu(&ws->bar_count) ^ before) & 0x80000000u) == 0u) {  // an L2 round trip each
      if (++it > (1L << 22)) {
        ok = false;
        flag(st, CSKV_DEV_TIMEOUT);
        break;
      }
    }
    *sm_flag = ok ? 1 : 0;
  }
  __syncthreads();
  return *sm_flag != 0;
}

// ------------------------------------------------------------------ shared state
struct IdxShared {
  uint64_t full[kIdxMaxStages];
  unsigned released[kIdxMaxStages];  // per ring stage: consumer warps done with it, all fills so far
  int fills;              // fills the producer issued (read by the drain after a timeout)
  int scan_err;           // a bounded wait of the scan gave up
  unsigned red[32];
  float fred[64];
  unsigned long long ured[32];
  unsigned long long tstar;
  int fcnt[32];
  Crossing cross;
  int flag;
  unsigned ubuf[4];
  int plan_t, plan_j, plan_G;
  long long plan_V[kMaxSplitQueries];
};

// ------------------------------------------------------------------ scan: E4M3 via TMA + MMA
// Returns false when a bounded wait gave up (CSKV_DEV_TIMEOUT is flagged).  The ring region is
// then left untouched by the caller: every fill the producer issued has been waited for (the
// drain below), or, when even that wait gave up, the barriers are not retired and the caller
// must not touch the ring memory again.
//
// FP4 = false: E4M3 keys and queries ([SW] §六.1 FP8), fp32 scales per entry (kscale) and per
// (query, head).  FP4 = true: OCP MXFP4 keys and queries ([SW] §六.1 / §十三.4 and [TR] §4.2: the
// indexer's QK path may run in FP4): E2M1 codes two per byte (element 2j in the low nibble) with
// one E8M0 scale per 32 elements (kbs: the entry's Di/32 scale bytes; p.q_bs for the queries).
// E2M1 values are exact in E4M3, so the codes are widened in registers and the same E4M3 MMA
// runs once per 32-element block: thread (g, tq) takes elements 32b + 8tq .. 32b + 8tq + 7 of
// block b for its rows and heads (one 32-bit load of codes), which keeps every MMA inside one
// block; the block's dot product is then multiplied by the two power-of-two scales.
template <int KS, int NTILE, bool FP4>
__device__ bool scan_mma(const IdxParams& p, int t, const uint8_t* kbase, const float* kscale, const uint8_t* kbs,
                         int len, float* sc, uint8_t* ring, IdxShared& S) {
  constexpr int Di = KS * 32;
  constexpr int RB = FP4 ? Di / 2 : Di;  // key bytes per entry in the tile
  constexpr int NB = Di / 32;            // MX blocks per key (FP4)
  const int stages = p.stages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = (len + kIdxTile - 1) / kIdxTile;
  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&S.full[s], 1);
      S.released[s] = 0u;
    }
    S.fills = 0;
    S.scan_err = 0;
    fence_mbar_init();
  }
  // generic-proxy writes to the ring region (histograms of a previous segment) must be
  // ordered before the TMA unit writes it
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncthreads();
  if (warp == kIdxConsumerWarps) {
    asm volatile("bar.sync 2, %0;" ::"n"(kIdxThreads) : "memory");  // consumers' scale loads issued
    if (lane == 0) {
      int s = 0, it = 0;
      for (; it < ntiles; ++it) {
        // the stage is refilled once every consumer warp has released its previous fill; a
        // consumer that gave up stops the producer too (no further fills are issued)
        if (it >= stages && !wait_released(&S.released[s], (unsigned)(kIdxConsumerWarps * (it / stages)),
                                           &S.scan_err)) {
          flag(p.st, CSKV_DEV_TIMEOUT);
          S.scan_err = 1;
          break;
        }
        const int rows = min(kIdxTile, len - it * kIdxTile);
        const unsigned bytes = (unsigned)(rows * RB);
        mbar_arrive_expect_tx(&S.full[s], bytes);
        tma_bulk_g2s(ring + (size_t)s * kIdxTile * RB, kbase + (size_t)it * kIdxTile * RB, bytes, &S.full[s]);
        if (++s == stages) s = 0;
      }
      S.fills = it;  // fills issued (the drain below needs the count)
    }
  } else {
    const int g = lane >> 2, tq = lane & 3;
    // B fragments (the query's heads) and per-head scale / weight, loaded once.
    uint32_t bq[NTILE][KS][2];
    float sq[NTILE][2], wh[NTILE][2];
    float fq[NTILE][2][FP4 ? NB : 1];  // FP4: the query heads' block scales
    const uint8_t* qrow = p.q_idx + (size_t)t * p.Hi * RB;
#pragma unroll
    for (int nt = 0; nt < NTILE; ++nt) {
      const int h = nt * 8 + g;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        if (h >= p.Hi) {
          bq[nt][ks][0] = bq[nt][ks][1] = 0u;
        } else if constexpr (FP4) {
          // block ks, elements 32 ks + 8 tq .. + 7: widened to E4M3 (k 4tq.. then 16 + 4tq..)
          const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(qrow + (size_t)h * RB + 16 * ks + 4 * tq));
          bq[nt][ks][0] = e2m1x4_to_e4m3x4(w & 0xFFFFu);
          bq[nt][ks][1] = e2m1x4_to_e4m3x4(w >> 16);
        } else {
          const int chunk = tq + 4 * (ks >> 1), wp = (ks & 1) * 2;
          const uint32_t* src = reinterpret_cast<const uint32_t*>(qrow + (size_t)h * Di + chunk * 16);
          bq[nt][ks][0] = __ldg(src + wp);
          bq[nt][ks][1] = __ldg(src + wp + 1);
        }
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int hh = nt * 8 + 2 * tq + c;
#pragma unroll
        for (int bb = 0; bb < (FP4 ? NB : 1); ++bb)
          fq[nt][c][bb] = (FP4 && hh < p.Hi) ? e8m0_to_float(__ldg(p.q_bs + ((size_t)t * p.Hi + hh) * NB + bb)) : 1.f;
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int h = nt * 8 + 2 * tq + c;
        const bool ok = h < p.Hi;
        sq[nt][c] = ok ? (p.q_scale ? __ldg(p.q_scale + (size_t)t * p.Hi + h) : 1.f) : 0.f;
        wh[nt][c] = ok ? (p.head_w ? __ldg(p.head_w + h) : 1.f) : 0.f;
      }
    }
    // Entry scales of this warp's rows for the next kScalePF tiles, held in registers and
    // shifted along; the first batch is requested before the producer starts streaming, so
    // these small loads are not queued behind the tile traffic.
    // (FP4: the rows' block-scale bytes, NB per entry, instead of an fp32 scale.)
    constexpr int kScalePF = 8;
    const int r0 = warp * 16;
    using SK = typename std::conditional<FP4, uint32_t, float>::type;
    auto ld_sk = [&](int e) -> SK {
      if constexpr (FP4) {
        if (e >= len) return 0u;
        return NB == 2 ? (uint32_t)__ldg(reinterpret_cast<const uint16_t*>(kbs) + e)
                       : __ldg(reinterpret_cast<const uint32_t*>(kbs) + e);
      } else {
        return e < len ? (kscale ? __ldg(kscale + e) : 1.f) : 0.f;
      }
    };
    SK ska[kScalePF], skb[kScalePF];
#pragma unroll
    for (int i = 0; i < kScalePF; ++i) {
      const int e = i * kIdxTile + r0 + g;
      ska[i] = ld_sk(e);
      skb[i] = ld_sk(e + 8);
    }
    asm volatile("bar.arrive 2, %0;" ::"n"(kIdxThreads) : "memory");
    // A fragments of this warp's 16 rows of a tile into registers and the MMAs on them (FP4: the
    // block scales applied to each block's dot product).
    auto mma_tile = [&](const uint8_t* tile, SK skg, SK skg8, float (&acc)[NTILE][4]) {
      if constexpr (FP4) {
        uint32_t wa[NB], wb[NB];
#pragma unroll
        for (int bb = 0; bb < NB; ++bb) {
          wa[bb] = *reinterpret_cast<const uint32_t*>(tile + (size_t)(r0 + g) * RB + 16 * bb + 4 * tq);
          wb[bb] = *reinterpret_cast<const uint32_t*>(tile + (size_t)(r0 + g + 8) * RB + 16 * bb + 4 * tq);
        }
#pragma unroll
        for (int nt = 0; nt < NTILE; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
        for (int bb = 0; bb < NB; ++bb) {
          const uint32_t a0 = e2m1x4_to_e4m3x4(wa[bb] & 0xFFFFu), a2 = e2m1x4_to_e4m3x4(wa[bb] >> 16);
          const uint32_t a1 = e2m1x4_to_e4m3x4(wb[bb] & 0xFFFFu), a3 = e2m1x4_to_e4m3x4(wb[bb] >> 16);
          const float kb0 = e8m0_to_float((skg >> (8 * bb)) & 0xFFu), kb8 = e8m0_to_float((skg8 >> (8 * bb)) & 0xFFu);
#pragma unroll
          for (int nt = 0; nt < NTILE; ++nt) {
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            mma_e4m3_16832(d, a0, a1, a2, a3, bq[nt][bb][0], bq[nt][bb][1]);
            // each block's exact dot product times 2^(key exponent) * 2^(query exponent)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              acc[nt][c] = fmaf(d[c] * kb0, fq[nt][c][bb], acc[nt][c]);
              acc[nt][2 + c] = fmaf(d[2 + c] * kb8, fq[nt][c][bb], acc[nt][2 + c]);
            }
          }
        }
      } else {
        uint4 ra[KS / 2], rb[KS / 2];
#pragma unroll
        for (int c = 0; c < KS / 2; ++c) {
          ra[c] = *reinterpret_cast<const uint4*>(tile + (size_t)(r0 + g) * Di + (tq + 4 * c) * 16);
          rb[c] = *reinterpret_cast<const uint4*>(tile + (size_t)(r0 + g + 8) * Di + (tq + 4 * c) * 16);
        }
#pragma unroll
        for (int nt = 0; nt < NTILE; ++nt) {
          acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
          for (int ks = 0; ks < KS; ++ks) {
            const uint4& A = ra[ks >> 1];
            const uint4& B = rb[ks >> 1];
            const bool hiw = ks & 1;
            mma_e4m3_16832(acc[nt], hiw ? A.z : A.x, hiw ? B.z : B.x, hiw ? A.w : A.y, hiw ? B.w : B.y,
                           bq[nt][ks][0], bq[nt][ks][1]);
          }
        }
      }
    };
    // Scales, ReLU and the weighted head sum of rows g and g + 8; lanes tq 0 / 1 store them.
    auto epilogue = [&](int it, SK skg, SK skg8, const float (&acc)[NTILE][4]) {
      const int e_g = it * kIdxTile + r0 + g, e_g8 = e_g + 8;
      const float kg = FP4 ? 1.f : (float)skg, kg8 = FP4 ? 1.f : (float)skg8;
      float vg = 0.f, vg8 = 0.f;
#pragma unroll
      for (int nt = 0; nt < NTILE; ++nt)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          vg = fmaf(wh[nt][c], fmaxf(0.f, (sq[nt][c] * kg) * acc[nt][c]), vg);
          vg8 = fmaf(wh[nt][c], fmaxf(0.f, (sq[nt][c] * kg8) * acc[nt][2 + c]), vg8);
        }
      vg += __shfl_xor_sync(0xffffffffu, vg, 1);
      vg += __shfl_xor_sync(0xffffffffu, vg, 2);
      vg8 += __shfl_xor_sync(0xffffffffu, vg8, 1);
      vg8 += __shfl_xor_sync(0xffffffffu, vg8, 2);
      if (tq == 0 && e_g < len) sc[e_g] = vg;
      if (tq == 1 && e_g8 < len) sc[e_g8] = vg8;
    };
    // Two ring stages a pass (one when one is left): the two tiles' load -> MMA -> epilogue
    // chains are independent, so the warp overlaps them.  A stage goes back to the producer
    // only after the MMAs have consumed every lane's fragments (a warp-synchronous mma.sync
    // cannot issue before all of its source loads have returned), so the next copy into it
    // cannot overwrite data still being read; the epilogues then overlap the refills.
    bool alive = true;
    int s = 0;
    unsigned ph = 0;
    for (int it = 0; it < ntiles && alive; it += 2) {
      const int n2 = min(2, ntiles - it);
      const int s1 = s + 1 == stages ? 0 : s + 1;
      const unsigned ph1 = s + 1 == stages ? ph ^ 1u : ph;
      if (!mbar_wait_bounded(&S.full[s], ph) || (n2 == 2 && !mbar_wait_bounded(&S.full[s1], ph1))) {
        flag(p.st, CSKV_DEV_TIMEOUT);
        *(volatile int*)&S.scan_err = 1;  // the producer stops issuing fills
        alive = false;
        break;
      }
      const SK ska0 = ska[0], skb0 = skb[0], ska1 = ska[1], skb1 = skb[1];
#pragma unroll
      for (int i = 0; i + 2 < kScalePF; ++i) {
        ska[i] = ska[i + 2];
        skb[i] = skb[i + 2];
      }
      {
        const int e = (it + kScalePF) * kIdxTile + r0 + g;
        ska[kScalePF - 2] = ld_sk(e);
        skb[kScalePF - 2] = ld_sk(e + 8);
        ska[kScalePF - 1] = ld_sk(e + kIdxTile);
        skb[kScalePF - 1] = ld_sk(e + kIdxTile + 8);
      }
      const bool act0 = r0 < min(kIdxTile, len - it * kIdxTile);
      const bool act1 = n2 == 2 && r0 < min(kIdxTile, len - (it + 1) * kIdxTile);
      float acc0[NTILE][4], acc1[NTILE][4];
      if (act0) mma_tile(ring + (size_t)s * kIdxTile * RB, ska0, skb0, acc0);
      if (act1) mma_tile(ring + (size_t)s1 * kIdxTile * RB, ska1, skb1, acc1);
      __syncwarp();
      if (lane == 0) {
        release_stage(&S.released[s]);
        if (n2 == 2) release_stage(&S.released[s1]);
      }
      if (act0) epilogue(it, ska0, skb0, acc0);
      if (act1) epilogue(it + 1, ska1, skb1, acc1);
      s = s1;
      ph = ph1;
      if (n2 == 2 && ++s == stages) {
        s = 0;
        ph ^= 1u;
      }
    }
  }
  __syncthreads();
  // Without a timeout every fill was waited for by the consumers, so the ring can be reused
  // and the barriers retired.  After a timeout some fills may still be in flight: thread 0
  // waits (bounded) for the last fill issued to every stage before the barriers are retired;
  // if that wait gives up too, the barriers stay live and the ring is never touched again.
  if (threadIdx.x == 0) {
    bool drained = true;
    if (S.scan_err) {
      const int fills = S.fills;
      for (int s = 0; s < stages && drained; ++s) {
        const int n = fills > s ? (fills - s + stages - 1) / stages : 0;  // fills of stage s
        if (n > 0) drained = mbar_wait_bounded(&S.full[s], (unsigned)((n - 1) & 1));
      }
    }
    if (drained)
      for (int s = 0; s < stages; ++s)
        asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_u32(&S.full[s])) : "memory");
  }
  __syncthreads();
  return S.scan_err == 0;
}

// ------------------------------------------------------------------ scan: fp32 (CUDA cores)
__device__ void scan_f32(const IdxParams& p, int t, const float* kbase, const float* kscale, int len,
                         float* sc, float* q_f32, IdxShared& S) {
  const int Hi = p.Hi, Di = p.Di;
  copy_to_smem<false>(q_f32, reinterpret_cast<const float*>(p.q_idx) + (size_t)t * Hi * Di, Hi * Di, threadIdx.x,
                      kIdxThreads);
  __syncthreads();
  float sq[kIdxMaxHeads], wh[kIdxMaxHeads];
#pragma unroll
  for (int h = 0; h < kIdxMaxHeads; ++h) {
    sq[h] = (h < Hi) ? (p.q_scale ? __ldg(p.q_scale + (size_t)t * Hi + h) : 1.f) : 0.f;
    wh[h] = (h < Hi) ? (p.head_w ? __ldg(p.head_w + h) : 1.f) : 0.f;
  }
  for (int e = threadIdx.x; e < len; e += kIdxThreads) {
    float acc[kIdxMaxHeads];
#pragma unroll
    for (int h = 0; h < kIdxMaxHeads; ++h) acc[h] = 0.f;
    const float4* kr = reinterpret_cast<const float4*>(kbase + (size_t)e * Di);
    for (int d4 = 0; d4 < Di / 4; ++d4) {
      const float4 kv = __ldg(kr + d4);
#pragma unroll
      for (int h = 0; h < kIdxMaxHeads; ++h)
        if (h < Hi) {
          const float* q = q_f32 + h * Di + 4 * d4;
          acc[h] = fmaf(q[0], kv.x, acc[h]);
          acc[h] = fmaf(q[1], kv.y, acc[h]);
          acc[h] = fmaf(q[2], kv.z, acc[h]);
          acc[h] = fmaf(q[3], kv.w, acc[h]);
        }
    }
    const float sk = kscale ? __ldg(kscale + e) : 1.f;
    float v = 0.f;
#pragma unroll
    for (int h = 0; h < kIdxMaxHeads; ++h)
      if (h < Hi) v = fmaf(wh[h], fmaxf(0.f, (sq[h] * sk) * acc[h]), v);
    sc[e] = v;
  }
  __syncthreads();
}

// ------------------------------------------------------------------ selection helpers
// One local radix pass over `n` keys produced by get(i), restricted to keys whose top nb
// bits equal P (all keys when nb == 0).  The first digit has 12 bits, later ones 10.
// Updates (P, nb, r); returns true when "top nb bits >= P" keeps exactly the r best keys.
template <typename Get>
__device__ bool local_pass(Get get, int n, uint64_t& P, int& nb, unsigned& r, unsigned* hist,
                           IdxShared& S) {
  const int w = nb == 0 ? 12 : min(10, 64 - nb);
  const int nbins = 1 << w;
  for (int i = threadIdx.x; i < nbins; i += kIdxThreads) hist[i] = 0u;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  for (int b0 = threadIdx.x - lane; b0 < n; b0 += kIdxThreads) {  // warp-uniform trip count
    const int i = b0 + lane;
    uint64_t c = 0;
    if (i < n) c = get(i);
    hist_add(hist, (unsigned)((c >> (64 - nb - w)) & (uint64_t)(nbins - 1)),
             i < n && (nb == 0 || (c >> (64 - nb)) == P));
  }
  __syncthreads();
  const Crossing x = find_crossing(hist, nbins, r, S.red, &S.cross);
  P = (P << w) | x.bin;
  nb += w;
  r -= x.above;
  return x.cnt == r || nb == 64;
}

// Exact top-r of n local keys: returns (P, nb) such that exactly r keys satisfy
// "top nb bits >= P".
template <typename Get>
__device__ void local_select(Get get, int n, unsigned r, uint64_t& P, int& nb, unsigned* hist, IdxShared& S) {
  P = 0;
  nb = 0;
  bool done = false;
  while (!done) done = local_pass(get, n, P, nb, r, hist, S);
}

// Writes the selected entries of this segment in ascending order at out[base ...].
// Positions are bounded by k, so even an inconsistent threshold (after a timed-out
// group barrier) cannot write outside the output row.
__device__ void emit(const float* sc, int len, int64_t lo, bool all, uint64_t P, int nb, int64_t base,
                     int64_t k, int32_t* oi, float* os, const IdxParams& p, int64_t ebase, IdxShared& S) {
  const int per = (len + kIdxThreads - 1) / kIdxThreads;
  const int a = min(len, (int)threadIdx.x * per), b = min(len, a + per);
  unsigned c = 0;
  for (int e = a; e < b; ++e) c += (all || key_selected(comp_key(sc[e], lo + e), P, nb)) ? 1u : 0u;
  int64_t pos = base + block_excl_scan(c, S.red, nullptr);
  for (int e = a; e < b; ++e)
    if (all || key_selected(comp_key(sc[e], lo + e), P, nb)) {
      if (pos >= 0 && pos < k) {
        oi[pos] = (int32_t)(lo + e);
        if (os) os[pos] = sc[e];
        if (p.pf_rows) prefetch_l2_bulk(p.pf_rows + (size_t)(ebase + lo + e) * p.pf_row_bytes, (unsigned)p.pf_row_bytes);
      }
      ++pos;
    }
}

__device__ unsigned count_selected(const float* sc, int len, int64_t lo, uint64_t P, int nb, IdxShared& S) {
  unsigned c = 0;
  for (int e = threadIdx.x; e < len; e += kIdxThreads) c += key_selected(comp_key(sc[e], lo + e), P, nb);
  unsigned tot;
  block_excl_scan(c, S.red, &tot);
  return tot;
}

// ---- speculative exchange helpers
// Block-wide max of one 64-bit key per thread.
__device__ uint64_t block_max_u64(uint64_t v, IdxShared& S) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int nw = kIdxThreads / 32;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint64_t y = __shfl_xor_sync(0xffffffffu, v, o);
    v = y > v ? y : v;
  }
  if (lane == 0) S.ured[warp] = v;
  __syncthreads();
  uint64_t m = 0;
  for (int w = 0; w < nw; ++w) m = S.ured[w] > m ? S.ured[w] : m;
  __syncthreads();
  return m;
}

// Log-scale bins below a maximum score key: for scores of one sign the score key grows by 2^23
// per octave, so (key_max - key) >> shift puts 2^(23 - shift) bins in every octave.  Monotone
// (decreasing) in the key; keys more than the range below the maximum share the last bin.
__device__ __forceinline__ unsigned log_bin(uint32_t kmax, uint32_t key, int shift, unsigned nbins) {
  const uint32_t b = (kmax - key) >> shift;
  return b < nbins ? b : nbins - 1u;
}
constexpr int kPropBins = 1024;  // proposal bins below the CTA's best score: 128 per octave
constexpr int kPropShift = 16;
constexpr int kTBins = kBins0;   // T* bins below the group's best proposal, sized to the proposals' range

// Over NB bins ordered from the best scores down, the first bin at which the running count
// exceeds `limit`: *out = {that bin, the count of the bins before it, its count}, or {NB, the
// total, 0} when the count never exceeds the limit.  All threads take part: thread t holds bins
// [t * NB / kIdxThreads, ...) in registers (one or two vector loads: no bank conflicts), one
// block scan, then the thread whose bins hold the cut writes it.  Two block barriers.
template <int NB>
__device__ void block_cut(const unsigned* hist, unsigned limit, Crossing* out, IdxShared& S) {
  constexpr int per = NB / kIdxThreads;
  static_assert(per == 2 || per == 8, "bins per thread");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  unsigned v[per];
  if constexpr (per == 2) {
    const uint2 w = reinterpret_cast<const uint2*>(hist)[tid];
    v[0] = w.x;
    v[1] = w.y;
  } else {
    const uint4 w0 = reinterpret_cast<const uint4*>(hist)[2 * tid], w1 = reinterpret_cast<const uint4*>(hist)[2 * tid + 1];
    v[0] = w0.x; v[1] = w0.y; v[2] = w0.z; v[3] = w0.w;
    v[4] = w1.x; v[5] = w1.y; v[6] = w1.z; v[7] = w1.w;
  }
  unsigned loc = 0;
#pragma unroll
  for (int i = 0; i < per; ++i) loc += v[i];
  unsigned inc = loc;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) S.red[warp] = inc;
  __syncthreads();
  unsigned excl = inc - loc, tot = 0;
#pragma unroll
  for (int w = 0; w < kIdxThreads / 32; ++w) {
    const unsigned r = S.red[w];
    excl += w < warp ? r : 0u;
    tot += r;
  }
  if (excl <= limit && excl + loc > limit) {
    unsigned c = excl;
#pragma unroll
    for (int i = 0; i < per; ++i) {
      if (c + v[i] > limit) {
        out->bin = (unsigned)(tid * per + i);
        out->above = c;
        out->cnt = v[i];
        break;
      }
      c += v[i];
    }
  }
  if (tid == 0 && tot <= limit) {
    out->bin = (unsigned)NB;
    out->above = tot;
    out->cnt = 0u;
  }
  __syncthreads();
}

// Returns the group's synchronisation state (and any global histogram it used) to zero;
// run by the last CTA of the group to finish.  Candidate slots and per-CTA fields are
// scratch: every call writes them before reading them.
__device__ void group_cleanup(QueryWS* ws, int G, bool used_hist0, int used_passes, IdxShared& S) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    S.flag = (atomicAdd(&ws->done, 1u) == (unsigned)(G - 1));
  }
  __syncthreads();
  if (S.flag) {
    __threadfence();
    if (used_hist0)
      for (int i = threadIdx.x; i < kBins0; i += kIdxThreads) ws->hist0[i] = 0u;
    for (int q = 0; q < used_passes; ++q)
      for (int i = threadIdx.x; i < kBinsP; i += kIdxThreads) ws->histp[q][i] = 0u;
    if (threadIdx.x == 0) {
      // every CTA of the group is past its last use of these
      ws->cand_count = 0u;
      ws->done = 0u;
    }
  }
  __syncthreads();
}

// ---- speculative proposals: fill this CTA's first slots (its best keys) in global memory and in
//      `own` (shared), leave their number in S.ubuf[0] (final after the next block barrier), and
//      return an upper bound of every key of the segment that was not proposed (0: none).
// The proposals are the entries in the top bins of a histogram of log-scale bins below the CTA's
// best score (32 per octave), as many bins from the top as keep the count within `limit` (<= cap;
// sized from the CTA's expected share of winners).  Log-scale bins keep a few outlying large
// scores from crowding every other score into one bin.
__device__ uint64_t propose_log(const float* sc, int len, int64_t lo, int cap, unsigned limit,
                                unsigned long long* slots, unsigned long long* own, unsigned* hist, IdxShared& S) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int nw = kIdxThreads / 32;
  float mx = -INFINITY;
  for (int e = threadIdx.x; e < len; e += kIdxThreads) mx = fmaxf(mx, sc[e]);
  for (int i = threadIdx.x; i < kPropBins; i += kIdxThreads) hist[i] = 0u;
  mx = warp_max(mx);
  if (lane == 0) S.fred[warp] = mx;
  if (threadIdx.x == 0) S.ubuf[0] = 0u;  // proposal slot counter
  __syncthreads();
  float gmx = S.fred[0];
#pragma unroll
  for (int w = 1; w < nw; ++w) gmx = fmaxf(gmx, S.fred[w]);
  const uint32_t kmx = score_key(gmx);
  for (int e = threadIdx.x; e < len; e += kIdxThreads)
    atomicAdd(&hist[log_bin(kmx, score_key(sc[e]), kPropShift, kPropBins)], 1u);
  __syncthreads();
  // pb = the number of bins from the top whose entries together stay within the limit
  block_cut<kPropBins>(hist, limit, &S.cross, S);
  const unsigned pb = S.cross.bin;
  for (int b0 = threadIdx.x - lane; b0 < len; b0 += kIdxThreads) {  // warp-uniform trip count
    const int e = b0 + lane;
    const bool valid = e < len;
    const uint32_t k32 = valid ? score_key(sc[e]) : 0u;
    const uint64_t ck = ((uint64_t)k32 << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)(lo + e));
    const bool prop = valid && log_bin(kmx, k32, kPropShift, kPropBins) < pb;
    // one slot reservation per warp
    const unsigned mask = __ballot_sync(0xffffffffu, prop);
    unsigned slot = 0;
    if (mask) {
      unsigned base = 0;
      if (lane == __ffs(mask) - 1) base = atomicAdd(&S.ubuf[0], (unsigned)__popc(mask));
      base = __shfl_sync(0xffffffffu, base, __ffs(mask) - 1);
      slot = base + (unsigned)__popc(mask & ((1u << lane) - 1u));
    }
    if (prop && slot < (unsigned)cap) {
      slots[slot] = ck;
      own[slot] = ck;
    }
  }
  // An upper bound of every key not proposed (no reduction needed): the top of the first bin
  // not proposed; 0 when every entry was proposed.  (A bound a little above the best key kept
  // back can only turn an exact acceptance into the exact path, never the reverse.)
  if (pb >= (unsigned)kPropBins) return 0ull;
  const uint32_t drop = pb << kPropShift;
  const uint32_t top = kmx >= drop ? kmx - drop : kmx;
  return ((uint64_t)top << 32) | 0xFFFFFFFFull;
}

// ---- cold paths, kept out of line: the speculative exchange's code stays compact (a launch
//      runs the selection once, so its instructions come from the instruction caches cold)

// A single CTA owns the query: radix select over the segment's keys, then emission.
__device__ __noinline__ void select_single(const IdxParams& p, const float* sc, int len, int64_t lo, int64_t keff,
                                           int32_t* oi, float* os, int64_t ebase, unsigned* hist, IdxShared& S) {
  uint64_t P = 0;
  int nb = 0;
  local_select([&](int i) { return comp_key(sc[i], lo + i); }, len, (unsigned)keff, P, nb, hist, S);
  emit(sc, len, lo, false, P, nb, 0, keff, oi, os, p, ebase, S);
}

// The rr-th best of the nbk keys of a crowded threshold bin: radix select inside the bin, then
// the smallest selected key exactly (a bare prefix threshold could also admit keys of lower bins).
__device__ __noinline__ uint64_t rank_in_big_bin(const unsigned long long* bin_keys, unsigned nbk, unsigned rr,
                                                 unsigned* hist, IdxShared& S) {
  uint64_t P2;
  int nb2;
  local_select([&](int i) { return (uint64_t)bin_keys[i]; }, nbk, rr, P2, nb2, hist, S);
  uint64_t mnk = ~0ull;
  for (unsigned i = threadIdx.x; i < nbk; i += kIdxThreads) {
    const uint64_t kk = bin_keys[i];
    if (key_selected(kk, P2, nb2) && kk < mnk) mnk = kk;
  }
  return ~block_max_u64(~mnk, S);
}

// The exact path over a group of CTAs (the speculative exchange was rejected: winners crowded
// into a few segments, massive ties).
__device__ __noinline__ void exact_group_select(const IdxParams& p, const float* sc, int len, int64_t lo, int j, int G,
                                                int64_t keff, int32_t* oi, float* os, int64_t ebase, QueryWS* ws,
                                                uint8_t* un, bool ok, IdxShared& S) {
  unsigned* hist = reinterpret_cast<unsigned*>(un + kUnHist);
  unsigned long long* cands = reinterpret_cast<unsigned long long*>(un + kUnCand);
  auto own_key = [&](int i) { return comp_key(sc[i], lo + i); };
  uint64_t P = 0;
  int nb = 0;
  // ---- 12-bit digit histogram of the whole group
  for (int i = threadIdx.x; i < kBins0; i += kIdxThreads) hist[i] = 0u;
  __syncthreads();
  for (int b0 = threadIdx.x - (threadIdx.x & 31); b0 < len; b0 += kIdxThreads) {
    const int e = b0 + (threadIdx.x & 31);
    hist_add(hist, e < len ? score_key(sc[e]) >> 20 : 0u, e < len);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kBins0; i += kIdxThreads)
    if (hist[i]) atomicAdd(&ws->hist0[i], hist[i]);
  ok = group_barrier(ws, G, j, p.st, &S.flag) && ok;
  copy_to_smem<true>(hist, ws->hist0, kBins0, threadIdx.x, kIdxThreads);
  __syncthreads();
  unsigned r = (unsigned)keff;
  Crossing x = find_crossing(hist, kBins0, r, S.red, &S.cross);
  P = x.bin;
  nb = 12;
  r -= x.above;
  bool done = (x.cnt == r);
  int used_passes = 0;
  int64_t base = 0;
  bool have_base = false;
  if (!done && x.cnt <= kCandMax) {
    // compaction of the threshold bin's entries into the group's candidate list
    const unsigned b0 = x.bin;
    unsigned above = 0, mine = 0;
    for (int e = threadIdx.x; e < len; e += kIdxThreads) above += (score_key(sc[e]) >> 20) > b0;
    const int per = (len + kIdxThreads - 1) / kIdxThreads;
    const int a = min(len, (int)threadIdx.x * per), b = min(len, a + per);
    for (int e = a; e < b; ++e) mine += (score_key(sc[e]) >> 20) == b0;
    unsigned tot_above, tot_mine;
    block_excl_scan(above, S.red, &tot_above);
    const unsigned off = block_excl_scan(mine, S.red, &tot_mine);
    if (threadIdx.x == 0) {
      S.ubuf[0] = tot_mine ? atomicAdd(&ws->cand_count, tot_mine) : 0u;
      ws->above[j] = tot_above;
    }
    __syncthreads();
    unsigned slot = S.ubuf[0] + off;
    for (int e = a; e < b; ++e)
      if ((score_key(sc[e]) >> 20) == b0) {
        if (slot < (unsigned)kCandMax) ws->cand[slot] = own_key(e);
        ++slot;
      }
    ok = group_barrier(ws, G, j, p.st, &S.flag) && ok;
    const unsigned n_c = min(__ldcg(&ws->cand_count), (unsigned)kCandMax);
    copy_to_smem<true>(cands, ws->cand, n_c, threadIdx.x, kIdxThreads);
    __syncthreads();
    while (!done) done = local_pass([&](int i) { return (uint64_t)cands[i]; }, n_c, P, nb, r, hist, S);
    // output base = selected entries of lower segments
    unsigned c = 0;
    for (unsigned i = threadIdx.x; i < n_c; i += kIdxThreads) {
      const uint64_t ck = cands[i];
      const int64_t e = (int64_t)(0xFFFFFFFFu - (uint32_t)(ck & 0xFFFFFFFFull));
      c += (e < lo && key_selected(ck, P, nb)) ? 1u : 0u;
    }
    for (int i = threadIdx.x; i < j; i += kIdxThreads) c += __ldcg(&ws->above[i]);
    unsigned tot;
    block_excl_scan(c, S.red, &tot);
    base = tot;
    have_base = true;
  } else if (!done) {
    // massive ties: further digits through the group's global histograms
    while (!done && ok) {
      const int w = min(10, 64 - nb);
      const int nbins = 1 << w;
      for (int i = threadIdx.x; i < nbins; i += kIdxThreads) hist[i] = 0u;
      __syncthreads();
      for (int b0 = threadIdx.x - (threadIdx.x & 31); b0 < len; b0 += kIdxThreads) {
        const int e = b0 + (threadIdx.x & 31);
        const uint64_t c = e < len ? own_key(e) : 0ull;
        hist_add(hist, (unsigned)((c >> (64 - nb - w)) & (uint64_t)(nbins - 1)), e < len && (c >> (64 - nb)) == P);
      }
      __syncthreads();
      unsigned* gh = ws->histp[used_passes];
      for (int i = threadIdx.x; i < nbins; i += kIdxThreads)
        if (hist[i]) atomicAdd(&gh[i], hist[i]);
      ++used_passes;
      ok = group_barrier(ws, G, j, p.st, &S.flag) && ok;
      copy_to_smem<true>(hist, gh, nbins, threadIdx.x, kIdxThreads);
      __syncthreads();
      const Crossing y = find_crossing(hist, nbins, r, S.red, &S.cross);
      P = (P << w) | y.bin;
      nb += w;
      r -= y.above;
      done = (y.cnt == r) || nb == 64;
    }
  }
  if (!have_base) {
    // per-segment selected counts -> output offsets
    const unsigned mine = count_selected(sc, len, lo, P, nb, S);
    if (threadIdx.x == 0) ws->above[j] = mine;
    ok = group_barrier(ws, G, j, p.st, &S.flag) && ok;
    unsigned c = 0;
    for (int i = threadIdx.x; i < j; i += kIdxThreads) c += __ldcg(&ws->above[i]);
    unsigned tot;
    block_excl_scan(c, S.red, &tot);
    base = tot;
  }
  emit(sc, len, lo, false, P, nb, base, keff, oi, os, p, ebase, S);
  group_cleanup(ws, G, true, used_passes, S);
}

// ------------------------------------------------------------------ one segment
template <int SRC, int KS, int NTILE>
__device__ void process_segment(const IdxParams& p, int t, int j, int G, int64_t V, int64_t ebase, QueryWS* ws,
                                float* sc, uint8_t* un, IdxShared& S) {
  const int64_t lo = (int64_t)j * V / G, hi = (int64_t)(j + 1) * V / G;
  int len = (int)min(hi - lo, (int64_t)p.seg_cap);
  const size_t tq = (size_t)t;
  int32_t* oi = p.out_idx + tq * p.k;
  float* os = p.out_score ? p.out_score + tq * p.k : nullptr;
  const int64_t keff = min((int64_t)p.k, V);
  if (j == 0)
    for (int64_t i = keff + threadIdx.x; i < p.k; i += kIdxThreads) {
      oi[i] = -1;
      if (os) os[i] = 0.f;
    }
  if (keff == 0) return;
  if (hi - lo > p.seg_cap && threadIdx.x == 0) flag(p.st, CSKV_DEV_CAPACITY);
  // speculative exchange sizes, computed before the scan (its copies are in flight meanwhile):
  // slots per CTA (group-uniform: every CTA lays out and reads the slots alike), and this CTA's
  // proposal limit -- its expected share of winners, half as many again and 16 more
  const unsigned V32 = (unsigned)min(V, (int64_t)0x7FFFFFFF);
  const int cap = (int)min((unsigned)(kCandMax / G), (V32 + (unsigned)G - 1u) / (unsigned)G);
  const unsigned limit = (unsigned)min((float)cap, 1.5f * (float)keff * (float)len / (float)V32 + 17.f);
  // ---- scores of this segment into shared memory
  if constexpr (SRC == kSrcFp8 || SRC == kSrcFp4) {
    constexpr bool fp4 = SRC == kSrcFp4;
    const uint8_t* kb = p.k_idx + (size_t)(ebase + lo) * (fp4 ? KS * 16 : KS * 32);
    const float* ks = (!fp4 && p.k_scale) ? p.k_scale + ebase + lo : nullptr;
    const uint8_t* kbs = fp4 ? p.k_bs + (size_t)(ebase + lo) * KS : nullptr;
    // after a timeout the ring (and the histograms that share its memory) is not touched
    // again; the other CTAs of the group time out at their next group barrier
    if (!scan_mma<KS, NTILE, fp4>(p, t, kb, ks, kbs, len, sc, un, S)) return;
  } else if constexpr (SRC == kSrcF32) {
    const float* kb = reinterpret_cast<const float*>(p.k_idx) + (size_t)(ebase + lo) * p.Di;
    const float* ks = p.k_scale ? p.k_scale + ebase + lo : nullptr;
    scan_f32(p, t, kb, ks, len, sc, reinterpret_cast<float*>(un), S);
  } else {
    const float* src = p.scores + tq * p.ld_scores + lo;
    copy_to_smem<false>(sc, src, len, threadIdx.x, kIdxThreads);
    __syncthreads();
  }
  // ---- everything kept: output position of entry e is e
  if (keff == V) {
    emit(sc, len, lo, true, 0, 0, lo, keff, oi, os, p, ebase, S);
    return;
  }
  unsigned* hist = reinterpret_cast<unsigned*>(un + kUnHist);
  // ---- a single CTA owns the query: exact selection in shared memory
  if (G == 1) {
    select_single(p, sc, len, lo, keff, oi, os, ebase, hist, S);
    return;
  }
  bool ok = true;
  // ---- speculative exchange (one group barrier).  Every CTA proposes its best entries (at
  //      most `cap`, into its own slots) and reports the best key it did NOT propose.  After
  //      the barrier every CTA finds the exact k-th best proposal T*; when no CTA holds an
  //      unproposed key >= T*, the selection is exactly {key >= T*} and no second exchange is
  //      needed.  Otherwise (winners crowded into one segment, massive ties) the exact path
  //      below runs.
  // slot capacity per CTA: group-uniform (every CTA lays out and reads the slots alike)
  if (G <= kIdxThreads && cap >= 1 && (int64_t)cap * G >= keff) {
    unsigned long long* slots = ws->cand + (size_t)j * cap;
    unsigned long long* own = reinterpret_cast<unsigned long long*>(un + kUnCand);  // this CTA's proposals
    const uint64_t unp = propose_log(sc, len, lo, cap, limit, slots, own, hist, S);
    for (int i = threadIdx.x; i < kTBins; i += kIdxThreads) hist[i] = 0u;  // for T*, set while waiting
    __syncthreads();  // the slot count is final
    const int nprop_own = (int)min(S.ubuf[0], (unsigned)cap);
    for (int i = nprop_own + (int)threadIdx.x; i < cap; i += kIdxThreads) {
      slots[i] = 0ull;  // 0 marks an unused slot
      own[i] = 0ull;
    }
    if (threadIdx.x == 0) ws->unp[j] = unp;
    ok = group_barrier(ws, G, j, p.st, &S.flag);  // its first block barrier orders the writes above
    // -- gather every CTA's slots into registers (thread t: slots t + kIdxThreads * uu, in CTA
    //    order; 0 marks an unused slot), with the best key and the number of proposals
    const unsigned total = (unsigned)G * (unsigned)cap;  // <= kCandMax = 8 * kIdxThreads
    const uint64_t u = (int)threadIdx.x < G ? __ldcg(&ws->unp[threadIdx.x]) : 0ull;
    unsigned long long v[8];
#pragma unroll
    for (int uu = 0; uu < 8; ++uu) {
      const unsigned c = threadIdx.x + uu * kIdxThreads;
      v[uu] = c < total ? __ldcg(ws->cand + c) : 0ull;
    }
    unsigned kmx = 0u, kmn = 0xFFFFFFFFu, cnt = 0u;
#pragma unroll
    for (int uu = 0; uu < 8; ++uu)
      if (v[uu] != 0ull) {
        kmx = max(kmx, (unsigned)(v[uu] >> 32));
        kmn = min(kmn, (unsigned)(v[uu] >> 32));
        ++cnt;
      }
    {
      const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
      kmx = __reduce_max_sync(0xffffffffu, kmx);
      kmn = __reduce_min_sync(0xffffffffu, kmn);
      cnt = __reduce_add_sync(0xffffffffu, cnt);
      if (lane == 0) {
        S.red[warp] = kmx;
        S.ured[warp] = kmn;
        S.fcnt[warp] = (int)cnt;
      }
    }
    if (threadIdx.x == 0) S.ubuf[1] = 0u;
    __syncthreads();
    unsigned gkmx = 0u, gkmn = 0xFFFFFFFFu;
    int nprop = 0;
#pragma unroll
    for (int w = 0; w < kIdxThreads / 32; ++w) {
      gkmx = max(gkmx, S.red[w]);
      gkmn = min(gkmn, (unsigned)S.ured[w]);
      nprop += S.fcnt[w];
    }
    if (nprop >= keff) {  // group-uniform: every CTA gathered the same slots
      // -- exact k-th best proposal: histogram of log-scale bins below the best proposal
      //    (256 per octave), then the rank inside the threshold bin
      // bins from the best proposal down to the worst, as fine as kTBins bins over that range
      // allow (uniform in the score key: about uniform in log(score) for scores of one
      // sign); warp 0 finds the bin holding the k-th best proposal and the count above it
      int tshift = 0;
      while (tshift < 32 && ((gkmx - gkmn) >> tshift) >= (uint32_t)kTBins) ++tshift;
      auto tbin = [&](uint64_t c) { return log_bin(gkmx, (uint32_t)(c >> 32), tshift, kTBins); };
#pragma unroll
      for (int uu = 0; uu < 8; ++uu)
        if (v[uu] != 0ull) atomicAdd(&hist[tbin(v[uu])], 1u);
      __syncthreads();
      block_cut<kTBins>(hist, (unsigned)keff - 1u, &S.cross, S);  // the first bin passing k - 1
      const Crossing x = S.cross;
      const unsigned rr = (unsigned)keff - x.above;  // rank wanted inside bin x.bin (1-based)
      const bool bin_fits = x.bin < (unsigned)kTBins && x.cnt <= (unsigned)kAuxKeys;
      // collect the threshold bin's keys
      unsigned long long* bin_keys = reinterpret_cast<unsigned long long*>(un + kUnAux);
      const unsigned bin_cap = (unsigned)kAuxKeys;
#pragma unroll
      for (int uu = 0; uu < 8; ++uu) {
        const uint64_t c = v[uu];
        if (c != 0ull && tbin(c) == x.bin) {
          const unsigned sl = atomicAdd(&S.ubuf[1], 1u);
          if (sl < bin_cap) bin_keys[sl] = c;
        }
      }
      __syncthreads();
      const unsigned nbk = min(S.ubuf[1], bin_cap);
      uint64_t Tstar = ~0ull;
      if (!bin_fits) {
        // the threshold bin does not fit the scratch: leave T* at "select nothing", which the
        // check below rejects
      } else if (nbk == 1 && rr == 1) {
        Tstar = bin_keys[0];  // the usual case: the threshold bin holds T* alone
      } else if (nbk <= (unsigned)kIdxThreads) {
        // thread i ranks key i against the bin (keys are distinct: exactly one has rank rr-1)
        if (threadIdx.x < nbk) {
          const uint64_t mine = bin_keys[threadIdx.x];
          unsigned rank = 0;
          for (unsigned m = 0; m < nbk; ++m) rank += (uint64_t)bin_keys[m] > mine;
          if (rank + 1 == rr) S.tstar = mine;
        }
        __syncthreads();
        Tstar = S.tstar;
      } else {
        Tstar = rank_in_big_bin(bin_keys, nbk, rr, hist, S);
      }
      // -- accepted when no CTA kept back a key >= T*
      // one block scan carries both the validity count (high bits) and this CTA's output
      // base = proposals of lower CTAs that are kept (low 16 bits; at most kCandMax)
      unsigned packed = 0;
      if ((int)threadIdx.x < G) packed += (unsigned)(u >= Tstar) << 16;
      if (threadIdx.x == 0 && !bin_fits) packed += 1u << 16;
      const unsigned my_off = (unsigned)j * (unsigned)cap;
#pragma unroll
      for (int uu = 0; uu < 8; ++uu)
        packed += (threadIdx.x + uu * kIdxThreads < my_off && v[uu] >= Tstar) ? 1u : 0u;
      unsigned tot;
      block_excl_scan(packed, S.red, &tot);
      if ((tot >> 16) == 0 && ok) {
        const unsigned base = tot & 0xFFFFu;
        if (cap <= 32) {
          // every kept entry of this segment is one of its proposals: its output position is
          // the base plus the kept proposals of this CTA with a lower index; warp 0 holds one
          // proposal a lane and ranks them with shuffles
          if (threadIdx.x < 32) {
            const uint64_t key = (int)threadIdx.x < cap ? own[threadIdx.x] : 0ull;
            const bool kept = key != 0ull && key >= Tstar;
            const uint32_t kl = (uint32_t)key;  // inverted index: larger = lower index
            unsigned pos = base;
#pragma unroll
            for (int m = 0; m < 32; ++m) {
              const uint64_t o = __shfl_sync(0xffffffffu, key, m);
              pos += (o != 0ull && o >= Tstar && (uint32_t)o > kl) ? 1u : 0u;
            }
            if (kept && pos < (unsigned)keff) {
              const uint32_t e = 0xFFFFFFFFu - kl;
              oi[pos] = (int32_t)e;
              if (os) os[pos] = key_score(key);
              if (p.pf_rows)
                prefetch_l2_bulk(p.pf_rows + (size_t)(ebase + e) * p.pf_row_bytes, (unsigned)p.pf_row_bytes);
            }
          }
        } else if (cap <= 64) {
          // as above, a thread a proposal
          if ((int)threadIdx.x < cap) {
            const uint64_t key = own[threadIdx.x];
            if (key >= Tstar) {
              const uint32_t kl = (uint32_t)key;  // inverted index: larger = lower index
              unsigned pos = base;
              for (int m = 0; m < cap; ++m) {
                const uint64_t o = own[m];
                pos += (o >= Tstar && (uint32_t)o > kl) ? 1u : 0u;
              }
              if (pos < (unsigned)keff) {
                const uint32_t e = 0xFFFFFFFFu - kl;
                oi[pos] = (int32_t)e;
                if (os) os[pos] = key_score(key);
                if (p.pf_rows)
                  prefetch_l2_bulk(p.pf_rows + (size_t)(ebase + e) * p.pf_row_bytes, (unsigned)p.pf_row_bytes);
              }
            }
          }
        } else {
          // emit keys >= T*: the rule "top 64 bits >= T*"
          emit(sc, len, lo, false, Tstar, 64, base, keff, oi, os, p, ebase, S);
        }
        return;
      }
    }
    // rejected (uniformly across the group); the next group barrier orders every read of the
    // proposals before the exact path reuses the candidate slots
  }
  exact_group_select(p, sc, len, lo, j, G, keff, oi, os, ebase, ws, un, ok, S);
}

__device__ __forceinline__ int64_t visible_of(const IdxParams& p, int t, int64_t* ebase) {
  if (p.scores) {
    *ebase = 0;
    int64_t v = __ldg(p.n_valid + t);
    if (v < 0 || v > p.ld_scores) {
      flag(p.st, CSKV_DEV_BAD_INDEX);
      v = v < 0 ? 0 : p.ld_scores;
    }
    return v;
  }
  // the query's sequence, position and (speculatively, for sequence 0) entry range are loaded
  // together: one round trip instead of two dependent ones in the common one-sequence case
  const int s = __ldg(p.q_seq + t);
  const int64_t pos = __ldg(p.q_pos + t);
  const int64_t z0 = __ldg(p.ent_off), z1 = __ldg(p.ent_off + 1);
  if (s < 0 || s >= p.batch) {
    flag(p.st, CSKV_DEV_BAD_INDEX);
    *ebase = 0;
    return 0;
  }
  const int64_t e0 = s == 0 ? z0 : __ldg(p.ent_off + s), e1 = s == 0 ? z1 : __ldg(p.ent_off + s + 1);
  *ebase = e0;
  int64_t v = pos >= 0 ? (pos + 1) / 4 : 0;
  if (v > e1 - e0) {
    flag(p.st, CSKV_DEV_BAD_INDEX);
    v = e1 - e0;
  }
  return v;
}

template <int SRC, int KS, int NTILE>
// At most 88 registers per thread (see kIdxConsumerWarps): other kernels of a decode step
// run beside the indexer on the same SMs.
__global__ void __maxnreg__(88) lindex_topk_kernel(IdxParams p) {
  extern __shared__ __align__(128) uint8_t dsm[];
  __shared__ IdxShared S;
  // While the previous kernel finishes: warm L2 with the lines the plan and the first tile
  // need (the query's position, sequence and offsets, its indexer vectors).  Prefetches only
  // move lines into L2, which stays coherent with the writes of the kernel being waited for.
  if (blockIdx.x == 0 && !p.scores) {
    const int t0 = p.t_begin;
    const int lane = threadIdx.x;
    if (lane == 0) asm volatile("prefetch.global.L2 [%0];" ::"l"(p.q_seq + t0));
    if (lane == 1) asm volatile("prefetch.global.L2 [%0];" ::"l"(p.q_pos + t0));
    if (lane == 2) asm volatile("prefetch.global.L2 [%0];" ::"l"(p.ent_off));
    if (lane == 3 && p.q_scale) asm volatile("prefetch.global.L2 [%0];" ::"l"(p.q_scale + (size_t)t0 * p.Hi));
    const size_t qbytes = SRC == kSrcFp4 ? (size_t)p.Hi * p.Di / 2 : (size_t)p.Hi * p.Di * (SRC == kSrcFp8 ? 1 : 4);
    for (size_t off = (size_t)(lane >= 4 ? lane - 4 : 0) * 128; lane >= 4 && off < qbytes; off += 124 * 128)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(p.q_idx + (size_t)t0 * qbytes + off));
  }
  if (threadIdx.x == 0) S.scan_err = 0;  // read only after later block barriers
  pdl_wait();
  // The kernel after the indexer may start now.  Only now: every kernel before the indexer has
  // completed, so a dependent that reads nothing the indexer writes (a compression issued with
  // CSKV_OVERLAP_PREVIOUS) may start reading at once.
  pdl_launch_dependents();
  uint8_t* un = dsm;                                              // ring / histogram / candidates
  float* sc = reinterpret_cast<float*>(dsm + p.un_bytes);  // segment scores
  if (p.split && p.T == 1) {
    // one query: the whole grid is its group (the plan below reduces to this)
    const int t = p.t_begin;
    int64_t eb;
    const int64_t V = visible_of(p, t, &eb);
    const int64_t smax = V > kMinSeg ? (V + kMinSeg - 1) / kMinSeg : 1;
    const int G = V > 0 ? (int)min(min((int64_t)gridDim.x, smax), (int64_t)kMaxGroup) : 1;
    if ((int)blockIdx.x >= G) return;
    process_segment<SRC, KS, NTILE>(p, t, (int)blockIdx.x, G, V, eb, p.ws, sc, un, S);
  } else if (p.split) {
    // plan, in parallel over queries: visible counts, group sizes (one round), CTA ranges
    if (threadIdx.x == 0) S.plan_t = -1;
    int64_t v = 0;
    if ((int)threadIdx.x < p.T) {
      int64_t eb;
      v = visible_of(p, p.t_begin + threadIdx.x, &eb);
    }
    unsigned vt;  // totals fit: the host bounds T * max_entries below 2^31 per launch
    block_excl_scan((unsigned)v, S.red, &vt);
    const int64_t total = vt, avail = (int64_t)gridDim.x - p.T;
    unsigned sz = 0;
    if ((int)threadIdx.x < p.T) {
      int64_t sv = 1 + (total > 0 ? (v * avail) / total : 0);
      const int64_t smax = v > kMinSeg ? (v + kMinSeg - 1) / kMinSeg : 1;
      sv = min(sv, smax);
      sv = min(sv, (int64_t)kMaxGroup);
      sz = (unsigned)sv;
    }
    const unsigned start = block_excl_scan(sz, S.red, nullptr);
    if ((int)threadIdx.x < p.T && blockIdx.x >= start && blockIdx.x < start + sz) {
      S.plan_t = threadIdx.x;
      S.plan_j = (int)(blockIdx.x - start);
      S.plan_G = (int)sz;
    }
    __syncthreads();
    const int i = S.plan_t;
    if (i < 0) return;
    const int t = p.t_begin + i;
    int64_t eb;
    const int64_t V = visible_of(p, t, &eb);
    const int j = S.plan_j, G = S.plan_G;
    process_segment<SRC, KS, NTILE>(p, t, j, G, V, eb, p.ws + i, sc, un, S);
  } else {
    for (int i = blockIdx.x; i < p.T; i += gridDim.x) {
      const int t = p.t_begin + i;
      int64_t eb;
      const int64_t V = visible_of(p, t, &eb);
      process_segment<SRC, KS, NTILE>(p, t, 0, 1, V, eb, nullptr, sc, un, S);
      __syncthreads();
      if (S.scan_err) break;  // a scan gave up: its ring may not be reused (block-uniform)
    }
  }
}

// ------------------------------------------------------------------ host side
struct DevInfo {
  int sms;
  int smem_optin;
};

// SM count and opt-in shared memory of the current device ({0, 0} without a device).
static DevInfo dev_info() {
  static thread_local int cached_dev = -1;
  static thread_local DevInfo info;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return DevInfo{0, 0};
  }
  if (dev != cached_dev) {
    DevInfo d{0, 0};
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) {
      cudaGetLastError();
      return DevInfo{0, 0};
    }
    info = d;
    cached_dev = dev;
  }
  return info;
}

// ring/histogram region + the segment's scores
static size_t idx_dyn_smem(int Di, int64_t seg_cap, int stages) {
  return idx_union_bytes(Di, stages) + (size_t)seg_cap * 4;
}

// Dynamic shared memory an indexer CTA of a split-mode launch may take when choosing a deeper
// ring: a tensor-core attention CTA of a decode step (97 KB dynamic + 3 KB static) must still
// fit on the same SM beside it (228 KB per SM, 1 KB of it reserved per CTA; the indexer's own
// static shared memory is 2 KB): 228 - 101 - 1 - 2 - 1 = 123 KB, rounded down.
constexpr size_t kIdxDeepRingSmem = 123 * 1024;

// Ring stages of a launch: the minimum (64 KiB), deepened towards the whole segment (every
// fill issued at once) while the CTA stays within kIdxDeepRingSmem.
static int idx_ring_stages(int Di, int64_t seg_cap) {
  const int base = idx_stages(Di);
  const int need = (int)min((seg_cap + kIdxTile - 1) / kIdxTile, (int64_t)kIdxMaxStages);
  int st = base;
  while (st < need && idx_dyn_smem(Di, seg_cap, st + 1) <= kIdxDeepRingSmem) ++st;
  return st;
}

static size_t idx_smem_budget() {
  const DevInfo d = dev_info();
  const size_t reserve = sizeof(IdxShared) + 1024;
  return (size_t)d.smem_optin > reserve ? (size_t)d.smem_optin - reserve : 0;
}

// Largest number of queries per split-mode launch for which a segment fits in shared memory.
static int split_queries_per_launch(int T, int64_t max_entries, int Di, int P, int64_t* seg_cap) {
  const size_t budget = idx_smem_budget();
  int Tb = min(T, min(P / 2, kMaxSplitQueries));
  while (Tb >= 1 && (int64_t)Tb * max_entries >= (1LL << 31)) Tb /= 2;  // the plan sums V in 32 bits
  while (Tb >= 1) {
    int64_t cap = (int64_t)Tb * max_entries / (P - Tb) + 1;
    cap = max(cap, (int64_t)2 * kMinSeg);
    cap = min(cap, max_entries);
    if (idx_dyn_smem(Di, cap, idx_stages(Di)) <= budget) {
      *seg_cap = cap;
      return Tb;
    }
    Tb /= 2;
  }
  return 0;
}

// Workspace of one launch: one QueryWS per query handled in split mode (0 without a device).
size_t lindex_ws_bytes(int T, int64_t max_entries) {
  (void)max_entries;
  const DevInfo d = dev_info();
  if (d.sms == 0) return 0;
  const int slots = min(T, min(d.sms / 2, kMaxSplitQueries));
  return (size_t)(slots > 0 ? slots : 1) * sizeof(QueryWS);
}

template <int SRC, int KS, int NTILE>
static cudaError_t launch_one(const IdxParams& p, int grid, bool coop, size_t smem, cudaStream_t stream) {
  auto kern = lindex_topk_kernel<SRC, KS, NTILE>;
  cudaError_t e = ensure_smem(kern, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kIdxThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  // cooperative (the CTAs of a query group wait on one another) and a dependent launch of
  // the previous kernel on the stream (the kernel waits for it before reading any input)
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = coop ? 1 : 0;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, kern, p);
  if (e == cudaSuccess) note_launch();
  return e;
}

template <int SRC, int KS, int NTILE>
static cudaError_t run_topk(IdxParams p, int T, cudaStream_t stream) {
  const DevInfo d = dev_info();
  // Two SMs stay out of the cooperative grid, so the small compression kernels that run
  // beside the indexer in a decode step do not hold up its (all-CTAs-resident) launch.
  const int P = d.sms > 8 ? d.sms - 2 : d.sms;
  // bytes of one key in the scan's tiles ("Di" of the ring and shared-memory plan)
  const int Di = SRC == kSrcFp8 ? KS * 32 : SRC == kSrcFp4 ? KS * 16 : 64;
  int64_t seg_cap = 0;
  const int Tb = split_queries_per_launch(T, p.max_entries, Di, P, &seg_cap);
  const bool row_fits = idx_dyn_smem(Di, p.max_entries, idx_stages(Di)) <= idx_smem_budget();
  if (Tb >= 1 && (Tb == T || !row_fits)) {
    p.split = 1;
    p.seg_cap = seg_cap;
    p.stages = (SRC == kSrcFp8 || SRC == kSrcFp4) ? idx_ring_stages(Di, seg_cap) : idx_stages(Di);
    p.un_bytes = (int64_t)idx_union_bytes(Di, p.stages);
    for (int t0 = 0; t0 < T; t0 += Tb) {
      p.t_begin = t0;
      p.T = min(Tb, T - t0);
      cudaError_t e = launch_one<SRC, KS, NTILE>(p, P, true, idx_dyn_smem(Di, seg_cap, p.stages), stream);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  if (!row_fits) return cudaErrorInvalidValue;
  p.split = 0;
  p.seg_cap = max(p.max_entries, (int64_t)1);
  p.stages = idx_stages(Di);
  p.un_bytes = (int64_t)idx_union_bytes(Di, p.stages);
  p.t_begin = 0;
  p.T = T;
  return launch_one<SRC, KS, NTILE>(p, min(T, P), false, idx_dyn_smem(Di, p.seg_cap, p.stages), stream);
}

bool lindex_shape_supported(int dtype, int Hi, int Di) {
  if (Hi < 1 || Hi > kIdxMaxHeads) return false;
  if (dtype == CSKV_FP8E4M3) return Di == 64 || Di == 128;
  if (dtype == CSKV_F32) return Di >= 4 && Di <= kIdxMaxDim && Di % 4 == 0;
  return false;
}

bool lindex_capacity_ok(int64_t max_entries, int T) {
  const DevInfo d = dev_info();
  if (d.sms < 2) return false;
  int64_t cap;
  const bool split = split_queries_per_launch(T, max_entries, 128, d.sms, &cap) >= 1;
  const bool row = idx_dyn_smem(128, max_entries, idx_stages(128)) <= idx_smem_budget();
  return split || row;
}

cudaError_t launch_lindex(const IdxParams& p0, int dtype, int T, cudaStream_t stream) {
  IdxParams p = p0;
  if (p.scores) return run_topk<kSrcScores, 2, 1>(p, T, stream);
  if (dtype == CSKV_F32) return run_topk<kSrcF32, 2, 1>(p, T, stream);
  const int ks = p.Di / 32;
  const int nt = p.Hi > 8 ? 2 : 1;
  if (p.k_bs) {  // MXFP4
    if (ks == 2 && nt == 1) return run_topk<kSrcFp4, 2, 1>(p, T, stream);
    if (ks == 2 && nt == 2) return run_topk<kSrcFp4, 2, 2>(p, T, stream);
    if (ks == 4 && nt == 1) return run_topk<kSrcFp4, 4, 1>(p, T, stream);
    return run_topk<kSrcFp4, 4, 2>(p, T, stream);
  }
  if (ks == 2 && nt == 1) return run_topk<kSrcFp8, 2, 1>(p, T, stream);
  if (ks == 2 && nt == 2) return run_topk<kSrcFp8, 2, 2>(p, T, stream);
  if (ks == 4 && nt == 1) return run_topk<kSrcFp8, 4, 1>(p, T, stream);
  return run_topk<kSrcFp8, 4, 2>(p, T, stream);
}

}  // namespace cskv
