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

enum IdxSrc { kSrcFp8 = 0, kSrcF32 = 1, kSrcScores = 2 };


struct alignas(16) QueryWS {
  unsigned bar_count, spare, done, cand_count;  // bar_count: group barrier (phase bit + arrivals)
  unsigned hist0[kBins0];
  unsigned histp[kMaxPasses - 1][kBinsP];
  unsigned above[kMaxGroup];
  unsigned long long unp[kMaxGroup];   // speculative path: best key each CTA did not propose
  unsigned long long cand[kCandMax];   // speculative path: `cap` proposal slots per CTA
};


// TMA ring depth: 64 KiB of k_idx tiles in flight per CTA whatever Di is.
__host__ __device__ constexpr int idx_stages(int Di) { return (64 * 1024) / (kIdxTile * Di); }

// Layout of the shared region after the scan: histogram, candidate keys, then a scratch
// area used first as the owner table of the gathered proposals, then for the keys of the
// threshold bin.
constexpr size_t kUnHist = 0;
constexpr size_t kUnCand = (size_t)kBins0 * 4;
constexpr size_t kUnAux = kUnCand + (size_t)kCandMax * 8;
constexpr int kAuxKeys = 1024;  // 8 KiB: kCandMax owner entries (2 B) or kAuxKeys keys (8 B)
constexpr size_t kUnSelBytes = kUnAux + (size_t)kAuxKeys * 8;

// Bytes of the shared region used first as the TMA ring, then for the histogram and the
// candidate keys.
__host__ __device__ constexpr size_t idx_union_bytes(int Di) {
  return (size_t)idx_stages(Di) * kIdxTile * Di > kUnSelBytes ? (size_t)idx_stages(Di) * kIdxTile * Di
                                                                : kUnSelBytes;
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
// counter whose top bit is the barrier's phase.  Thread 0 reads the counter (the phase cannot
// change before this CTA arrives), publishes the CTA's writes with a fence (cumulative over
// the block barrier before it) and arrives with a reduction that needs no reply: CTA 0 of the
// group adds 2^31 - (G - 1), every other CTA adds 1, so the sum of the G arrivals is exactly
// 2^31 -- the phase bit flips when the last one lands and the low bits are back where they
// were (zero), for any G, with no reset.  Waiters poll until the phase differs.  Bounded:
// gives up after a few million polls, about a second (CSKV_DEV_TIMEOUT).
__device__ bool group_barrier(QueryWS* ws, unsigned G, int j, int* st, int* sm_flag) {
  __syncthreads();
  if (threadIdx.x == 0) {
    bool ok = true;
    const unsigned before = ld_acquire_gpu(&ws->bar_count);
    const unsigned add = j == 0 ? 0x80000000u - (G - 1u) : 1u;
    __threadfence();
    asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(&ws->bar_count), "r"(add) : "memory");
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
  uint64_t full[12];
  unsigned released[12];  // per ring stage: consumer warps done with it, all fills so far
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
template <int KS, int NTILE>
__device__ bool scan_fp8(const IdxParams& p, int t, const uint8_t* kbase, const float* kscale, int len,
                         float* sc, uint8_t* ring, IdxShared& S) {
  constexpr int Di = KS * 32;
  constexpr int stages = idx_stages(Di);
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
        const unsigned bytes = (unsigned)(rows * Di);
        mbar_arrive_expect_tx(&S.full[s], bytes);
        tma_bulk_g2s(ring + (size_t)s * kIdxTile * Di, kbase + (size_t)it * kIdxTile * Di, bytes, &S.full[s]);
        if (++s == stages) s = 0;
      }
      S.fills = it;  // fills issued (the drain below needs the count)
    }
  } else {
    const int g = lane >> 2, tq = lane & 3;
    // B fragments (the query's heads) and per-head scale / weight, loaded once.
    uint32_t bq[NTILE][KS][2];
    float sq[NTILE][2], wh[NTILE][2];
    const uint8_t* qrow = p.q_idx + (size_t)t * p.Hi * Di;
#pragma unroll
    for (int nt = 0; nt < NTILE; ++nt) {
      const int h = nt * 8 + g;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const int chunk = tq + 4 * (ks >> 1), wp = (ks & 1) * 2;
        if (h < p.Hi) {
          const uint32_t* src = reinterpret_cast<const uint32_t*>(qrow + (size_t)h * Di + chunk * 16);
          bq[nt][ks][0] = __ldg(src + wp);
          bq[nt][ks][1] = __ldg(src + wp + 1);
        } else {
          bq[nt][ks][0] = bq[nt][ks][1] = 0u;
        }
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
    constexpr int kScalePF = 8;
    const int r0 = warp * 16;
    float ska[kScalePF], skb[kScalePF];
#pragma unroll
    for (int i = 0; i < kScalePF; ++i) {
      const int e = i * kIdxTile + r0 + g;
      ska[i] = e < len ? (kscale ? __ldg(kscale + e) : 1.f) : 0.f;
      skb[i] = e + 8 < len ? (kscale ? __ldg(kscale + e + 8) : 1.f) : 0.f;
    }
    asm volatile("bar.arrive 2, %0;" ::"n"(kIdxThreads) : "memory");
    bool alive = true;
    int s = 0;
    unsigned ph = 0;
    for (int it = 0; it < ntiles && alive; ++it) {
      if (!mbar_wait_bounded(&S.full[s], ph)) {
        flag(p.st, CSKV_DEV_TIMEOUT);
        *(volatile int*)&S.scan_err = 1;  // the producer stops issuing fills
        alive = false;
        break;
      }
      const int rows = min(kIdxTile, len - it * kIdxTile);
      const float skg = ska[0], skg8 = skb[0];
#pragma unroll
      for (int i = 0; i + 1 < kScalePF; ++i) {
        ska[i] = ska[i + 1];
        skb[i] = skb[i + 1];
      }
      {
        const int e = (it + kScalePF) * kIdxTile + r0 + g;
        ska[kScalePF - 1] = e < len ? (kscale ? __ldg(kscale + e) : 1.f) : 0.f;
        skb[kScalePF - 1] = e + 8 < len ? (kscale ? __ldg(kscale + e + 8) : 1.f) : 0.f;
      }
      // A fragments of this warp's 16 rows into registers and the MMAs on them; the stage
      // goes back to the producer only after the MMAs have consumed every lane's fragments
      // (a warp-synchronous mma.sync cannot issue before all of its source loads have
      // returned), so the next copy into the stage cannot overwrite data still being read.
      // The epilogue then overlaps the refill.
      if (r0 >= rows) {
        __syncwarp();
        if (lane == 0) release_stage(&S.released[s]);
      } else {
        uint4 ra[KS / 2], rb[KS / 2];
        const uint8_t* tile = ring + (size_t)s * kIdxTile * Di;
#pragma unroll
        for (int c = 0; c < KS / 2; ++c) {
          ra[c] = *reinterpret_cast<const uint4*>(tile + (size_t)(r0 + g) * Di + (tq + 4 * c) * 16);
          rb[c] = *reinterpret_cast<const uint4*>(tile + (size_t)(r0 + g + 8) * Di + (tq + 4 * c) * 16);
        }
        float acc[NTILE][4];
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
        __syncwarp();
        if (lane == 0) release_stage(&S.released[s]);
        const int e_g = it * kIdxTile + r0 + g, e_g8 = e_g + 8;
        float vg = 0.f, vg8 = 0.f;
#pragma unroll
        for (int nt = 0; nt < NTILE; ++nt)
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            vg = fmaf(wh[nt][c], fmaxf(0.f, (sq[nt][c] * skg) * acc[nt][c]), vg);
            vg8 = fmaf(wh[nt][c], fmaxf(0.f, (sq[nt][c] * skg8) * acc[nt][2 + c]), vg8);
          }
        vg += __shfl_xor_sync(0xffffffffu, vg, 1);
        vg += __shfl_xor_sync(0xffffffffu, vg, 2);
        vg8 += __shfl_xor_sync(0xffffffffu, vg8, 1);
        vg8 += __shfl_xor_sync(0xffffffffu, vg8, 2);
        if (tq == 0 && e_g < len) sc[e_g] = vg;
        if (tq == 1 && e_g8 < len) sc[e_g8] = vg8;
      }
      if (++s == stages) {
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
constexpr int kLinBins = 1024;  // linear score bins (<= kBins0, shares the histogram buffer)

// Block-wide min and max of one float per thread, and the sum of one count per thread.
__device__ void block_minmax(float mn, float mx, IdxShared& S, float& gmn, float& gmx, int cnt = 0,
                             int* gcnt = nullptr) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int nw = kIdxThreads / 32;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  cnt = __reduce_add_sync(0xffffffffu, cnt);
  if (lane == 0) {
    S.fred[warp] = mn;
    S.fred[32 + warp] = mx;
    S.fcnt[warp] = cnt;
  }
  __syncthreads();
  gmn = INFINITY;
  gmx = -INFINITY;
  int c = 0;
  for (int w = 0; w < nw; ++w) {
    gmn = fminf(gmn, S.fred[w]);
    gmx = fmaxf(gmx, S.fred[32 + w]);
    c += S.fcnt[w];
  }
  if (gcnt) *gcnt = c;
  __syncthreads();
}


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

// Bin (of kBins0) of a key by its score bits above the smallest proposal's: the score key
// minus the lowest one, shifted so that the range fits.  Monotone in the key; for scores of
// one sign the bins are about uniform in log(score), so a few outlying large scores (planted
// or real) do not crowd every other proposal into a handful of bins.
__device__ __forceinline__ unsigned key_bin4k(uint64_t c, uint32_t kmin, int shift) {
  const uint32_t d = (uint32_t)(c >> 32) - kmin;
  const uint32_t b = d >> shift;
  return b < (uint32_t)kBins0 ? b : (uint32_t)(kBins0 - 1);
}


// Linear bin of a score inside [lo, lo + 1024/scl]; monotone in s.
__device__ __forceinline__ unsigned lin_bin(float s, float lo, float scl) {
  const float f = (s - lo) * scl;
  return f <= 0.f ? 0u : (f >= (float)(kLinBins - 1) ? (unsigned)(kLinBins - 1) : (unsigned)f);
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

// ---- speculative proposals: fill this CTA's `cap` slots (its best keys; 0 in unused slots)
//      and return the best key of the segment that was not proposed (0: none).

// The proposals are the entries in the top bins of a 1024-bin linear histogram over the CTA's
// own score range, as many bins as keep the count within a limit (<= cap) sized from the CTA's
// expected share of winners.
__device__ uint64_t propose_hist(const float* sc, int len, int64_t lo, int cap, int64_t keff, int64_t V,
                                 unsigned long long* slots, unsigned* hist, IdxShared& S) {
  float mn = INFINITY, mx = -INFINITY;
  for (int e = threadIdx.x; e < len; e += kIdxThreads) {
    mn = fminf(mn, sc[e]);
    mx = fmaxf(mx, sc[e]);
  }
  for (int i = threadIdx.x; i < kLinBins; i += kIdxThreads) hist[i] = 0u;
  float gmn, gmx;
  block_minmax(mn, mx, S, gmn, gmx);
  const float scl = gmx > gmn ? (float)kLinBins / (gmx - gmn) : 0.f;
  for (int e = threadIdx.x; e < len; e += kIdxThreads) atomicAdd(&hist[lin_bin(sc[e], gmn, scl)], 1u);
  __syncthreads();
  // lowest bin whose suffix count stays within the limit: one above the bin where the count
  // from the top first exceeds it
  const unsigned limit = (unsigned)min((int64_t)cap, (3 * keff * len + 2 * V - 1) / (2 * V) + 16);
  if ((unsigned)len <= limit) {
    if (threadIdx.x == 0) S.ubuf[2] = 0u;
  } else {
    const Crossing xl = find_crossing(hist, kLinBins, limit + 1u, S.red, &S.cross);
    if (threadIdx.x == 0) S.ubuf[2] = xl.bin + 1u;
  }
  if (threadIdx.x == 0) S.ubuf[0] = 0u;  // proposal slot counter
  __syncthreads();
  const unsigned pb = S.ubuf[2];
  uint64_t unp = 0;
  for (int e = threadIdx.x; e < len; e += kIdxThreads) {
    const uint64_t ck = comp_key(sc[e], lo + e);
    bool put = false;
    if (lin_bin(sc[e], gmn, scl) >= pb) {
      const unsigned slot = atomicAdd(&S.ubuf[0], 1u);
      if (slot < (unsigned)cap) {
        slots[slot] = ck;
        put = true;
      }
    }
    if (!put) unp = ck > unp ? ck : unp;
  }
  unp = block_max_u64(unp, S);
  for (int i = (int)min(S.ubuf[0], (unsigned)cap) + (int)threadIdx.x; i < cap; i += kIdxThreads) slots[i] = 0ull;
  return unp;
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
  // ---- scores of this segment into shared memory
  if constexpr (SRC == kSrcFp8) {
    const uint8_t* kb = p.k_idx + (size_t)(ebase + lo) * (KS * 32);
    const float* ks = p.k_scale ? p.k_scale + ebase + lo : nullptr;
    // after a timeout the ring (and the histograms that share its memory) is not touched
    // again; the other CTAs of the group time out at their next group barrier
    if (!scan_fp8<KS, NTILE>(p, t, kb, ks, len, sc, un, S)) return;
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
  unsigned long long* cands = reinterpret_cast<unsigned long long*>(un + kUnCand);
  auto own_key = [&](int i) { return comp_key(sc[i], lo + i); };
  uint64_t P = 0;
  int nb = 0;
  // ---- a single CTA owns the query: exact selection in shared memory
  if (G == 1) {
    local_select(own_key, len, (unsigned)keff, P, nb, hist, S);
    emit(sc, len, lo, false, P, nb, 0, keff, oi, os, p, ebase, S);
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
  const int cap = (int)min((int64_t)(kCandMax / G), (V + G - 1) / G);
  if (G <= kIdxThreads && cap >= 1 && (int64_t)cap * G >= keff) {
    unsigned long long* slots = ws->cand + (size_t)j * cap;
    const uint64_t unp = propose_hist(sc, len, lo, cap, keff, V, slots, hist, S);
    if (threadIdx.x == 0) ws->unp[j] = unp;
    for (int i = threadIdx.x; i < kBins0; i += kIdxThreads) hist[i] = 0u;  // for T*, set while waiting
    ok = group_barrier(ws, G, j, p.st, &S.flag);
    // -- gather every CTA's slots (CTA order; 0 marks an unused slot), count the proposals
    //    and find their score range
    const unsigned total = (unsigned)G * (unsigned)cap;
    const uint64_t u = (int)threadIdx.x < G ? __ldcg(&ws->unp[threadIdx.x]) : 0ull;
    float mn = INFINITY, mx = -INFINITY;
    int cnt = 0;
    for (unsigned b0 = threadIdx.x; b0 < total; b0 += kIdxThreads * 8) {
      unsigned long long v[8];
#pragma unroll
      for (int uu = 0; uu < 8; ++uu) {
        const unsigned c = b0 + uu * kIdxThreads;
        v[uu] = c < total ? __ldcg(ws->cand + c) : 0ull;
      }
#pragma unroll
      for (int uu = 0; uu < 8; ++uu) {
        const unsigned c = b0 + uu * kIdxThreads;
        if (c < total) cands[c] = v[uu];
        if (v[uu] != 0ull) {
          const float f = key_score(v[uu]);
          mn = fminf(mn, f);
          mx = fmaxf(mx, f);
          ++cnt;
        }
      }
    }
    float qmn, qmx;
    int nprop;
    block_minmax(mn, mx, S, qmn, qmx, cnt, &nprop);  // its barriers also publish cands[]
    if (nprop >= keff) {  // group-uniform: every CTA gathered the same slots
      // -- exact k-th best proposal: histogram over the proposals' score keys, then rank
      //    inside the threshold bin
      const uint32_t kmin = score_key(qmn), krange = score_key(qmx) - kmin;
      int shift = 0;
      while (shift < 32 && (krange >> shift) >= (uint32_t)kBins0) ++shift;
      for (unsigned i = threadIdx.x; i < total; i += kIdxThreads) {
        const uint64_t c = cands[i];
        if (c != 0ull) atomicAdd(&hist[key_bin4k(c, kmin, shift)], 1u);
      }
      if (threadIdx.x == 0) S.ubuf[1] = 0u;
      __syncthreads();
      const Crossing x = find_crossing(hist, kBins0, (unsigned)keff, S.red, &S.cross);
      const unsigned rr = (unsigned)keff - x.above;  // rank wanted inside bin x.bin (1-based)
      const bool bin_fits = x.cnt <= (unsigned)kAuxKeys;
      // collect the threshold bin's keys
      unsigned long long* bin_keys = reinterpret_cast<unsigned long long*>(un + kUnAux);
      const unsigned bin_cap = (unsigned)kAuxKeys;
      for (unsigned i = threadIdx.x; i < total; i += kIdxThreads) {
        const uint64_t c = cands[i];
        if (c != 0ull && key_bin4k(c, kmin, shift) == x.bin) {
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
        // radix select inside the bin, then T* = the smallest selected key exactly (a bare
        // prefix threshold could also admit keys of lower linear bins)
        uint64_t P2;
        int nb2;
        local_select([&](int i) { return (uint64_t)bin_keys[i]; }, nbk, rr, P2, nb2, hist, S);
        uint64_t mnk = ~0ull;
        for (unsigned i = threadIdx.x; i < nbk; i += kIdxThreads) {
          const uint64_t kk = bin_keys[i];
          if (key_selected(kk, P2, nb2) && kk < mnk) mnk = kk;
        }
        Tstar = ~block_max_u64(~mnk, S);
      }
      // -- accepted when no CTA kept back a key >= T*
      // one block scan carries both the validity count (high bits) and this CTA's output
      // base = proposals of lower CTAs that are kept (low 16 bits; at most kCandMax)
      unsigned packed = 0;
      if ((int)threadIdx.x < G) packed += (unsigned)(u >= Tstar) << 16;
      if (threadIdx.x == 0 && !bin_fits) packed += 1u << 16;
      const unsigned my_off = (unsigned)j * (unsigned)cap;
      for (unsigned i = threadIdx.x; i < my_off; i += kIdxThreads) packed += cands[i] >= Tstar;
      unsigned tot;
      block_excl_scan(packed, S.red, &tot);
      if ((tot >> 16) == 0 && ok) {
        const unsigned base = tot & 0xFFFFu;
        if (cap <= 64) {
          // every kept entry of this segment is one of its proposals: its output position is
          // the base plus the kept proposals of this CTA with a lower index
          const unsigned long long* own = cands + my_off;
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
  // ---- exact path: 12-bit digit histogram of the whole group
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
  unsigned cands_used = 0;
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
    cands_used = n_c;
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
  const int s = __ldg(p.q_seq + t);
  if (s < 0 || s >= p.batch) {
    flag(p.st, CSKV_DEV_BAD_INDEX);
    *ebase = 0;
    return 0;
  }
  const int64_t e0 = __ldg(p.ent_off + s), e1 = __ldg(p.ent_off + s + 1);
  *ebase = e0;
  const int64_t pos = __ldg(p.q_pos + t);
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
  pdl_launch_dependents();  // the kernel after the indexer may start its set-up now
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
    const size_t qbytes = (size_t)p.Hi * p.Di * (SRC == kSrcFp8 ? 1 : 4);
    for (size_t off = (size_t)(lane >= 4 ? lane - 4 : 0) * 128; lane >= 4 && off < qbytes; off += 124 * 128)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(p.q_idx + (size_t)t0 * qbytes + off));
  }
  if (threadIdx.x == 0) S.scan_err = 0;  // read only after later block barriers
  pdl_wait();
  uint8_t* un = dsm;                                              // ring / histogram / candidates
  float* sc = reinterpret_cast<float*>(dsm + idx_union_bytes(KS * 32));  // segment scores
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

// ring/histogram region + the segment's scores + its entry scales
static size_t idx_dyn_smem(int Di, int64_t seg_cap) { return idx_union_bytes(Di) + (size_t)seg_cap * 8; }

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
    if (idx_dyn_smem(Di, cap) <= budget) {
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
  const int Di = SRC == kSrcFp8 ? KS * 32 : 64;
  int64_t seg_cap = 0;
  const int Tb = split_queries_per_launch(T, p.max_entries, Di, P, &seg_cap);
  const bool row_fits = idx_dyn_smem(Di, p.max_entries) <= idx_smem_budget();
  p.stages = idx_stages(Di);
  if (Tb >= 1 && (Tb == T || !row_fits)) {
    p.split = 1;
    p.seg_cap = seg_cap;
    for (int t0 = 0; t0 < T; t0 += Tb) {
      p.t_begin = t0;
      p.T = min(Tb, T - t0);
      cudaError_t e = launch_one<SRC, KS, NTILE>(p, P, true, idx_dyn_smem(Di, seg_cap), stream);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  if (!row_fits) return cudaErrorInvalidValue;
  p.split = 0;
  p.seg_cap = max(p.max_entries, (int64_t)1);
  p.t_begin = 0;
  p.T = T;
  return launch_one<SRC, KS, NTILE>(p, min(T, P), false, idx_dyn_smem(Di, p.seg_cap), stream);
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
  const bool row = idx_dyn_smem(128, max_entries) <= idx_smem_budget();
  return split || row;
}

cudaError_t launch_lindex(const IdxParams& p0, int dtype, int T, cudaStream_t stream) {
  IdxParams p = p0;
  if (p.scores) return run_topk<kSrcScores, 2, 1>(p, T, stream);
  if (dtype == CSKV_F32) return run_topk<kSrcF32, 2, 1>(p, T, stream);
  const int ks = p.Di / 32;
  const int nt = p.Hi > 8 ? 2 : 1;
  if (ks == 2 && nt == 1) return run_topk<kSrcFp8, 2, 1>(p, T, stream);
  if (ks == 2 && nt == 2) return run_topk<kSrcFp8, 2, 2>(p, T, stream);
  if (ks == 4 && nt == 1) return run_topk<kSrcFp8, 4, 1>(p, T, stream);
  return run_topk<kSrcFp8, 4, 2>(p, T, stream);
}

}  // namespace cskv
