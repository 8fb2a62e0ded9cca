// Lightning Indexer scores of many queries at once (a prefill chunk) on the 5th-generation
// tensor cores, reduced to per-query candidate lists for the exact top-k.
//
// [SW] = shareware.cn/news/167317 (DeepSeek V4 Hybrid Attention essay), §六: the indexer scores
// every compressed entry i for query t as
//     s_i = sum_h w_h * ReLU(sq_{t,h} * sk_i * <q_{t,h}, k_i>)
// in low precision (E4M3 codes, fp32 scales); §七: the top-k (k = 1024, [AM]) entries are kept;
// §十: query t sees the entries i < floor((pos_t + 1) / 4) only (the block-24 example).
// [TR] = trdm.cn/news/516303, §4.2: the LightningIndexer is a ReLU'd product of the query heads
// with the pooled keys, weighted and summed over heads.
//
// Across the queries of a chunk the <q_{t,h}, k_i> form a dense product.  A CTA takes QT =
// 128 / Hi consecutive queries -- their (t, h) rows are the N = 128 columns of tcgen05.mma
// kind::f8f6f4 (E4M3 x E4M3 -> fp32 in TMEM) -- and streams its sequence's keys in tiles of
// 256 entries, two MMAs of M = 128 entries (the TMEM lanes): D[i, (t, h)] = K_half Q^T.  Two
// TMEM accumulators of 256 columns let the MMAs of one tile run while the epilogue reads the
// other.  Operands are K-major in the 128-byte swizzle layout (row r at r * 128 bytes, 16-byte
// chunk c at chunk c ^ (r & 7)); key tiles are gathered with 16-byte cp.async copies into a
// ring of four stages (three tiles in flight while one is multiplied), their scales alongside.
//
// Epilogue (16 warps: warp w reads the TMEM lane quarter w % 4 -- 32 entries of each half, one
// per lane -- and the 32 columns 32 (w / 4) .. -- 32 / Hi queries): a lane sums, in
// registers, its entry's score for each of those queries, s = sk_i * sum_h (w_h sq_{t,h})
// max(0, acc) -- factoring the scales out of the ReLU needs sq > 0 and sk > 0 (quantisation
// scales are); a tile or a CTA with a non-positive scale takes the unfactored form
// sum_h w_h max(0, (sq sk) acc).
//
// The k-th best score of a query is not known before all of its entries are scored, so the
// kernel makes two passes over the keys:
//   1. every visible entry's score goes into a per-query histogram (1024 bins, 16 per octave
//      of positive scores, one for scores <= 0), in shared memory;  from it the bin
//      b* holding the k-th best score (k_eff = min(k, visible)) and the count above it;
//   2. the scores are computed again (the same instructions on the same data: the same values)
//      and every visible entry with bin > b*, and the entries of bin b* while the list has
//      room, are appended to the query's candidate list in ascending entry order (a ballot
//      orders the 32 entries of a lane quarter, shared counts the tile's eight segments).
// In pass 1 a per-query floor (raised every 4 tiles to the lowest bin of the 32-bin block in
// which the count from the top reaches k_eff) lets entries far below the k-th score skip the
// histogram: b* is never below the floor, and every bin at or above it is counted exactly.
// The candidate list holds every entry that can be among the k best, in index order, so the
// exact top-k over it (ties to the lower position) is the exact top-k over all entries.  A list
// that overflows its capacity inside bin b* is still exact when every score in b* is equal (a
// pile of equal scores, e.g. zeros: the lowest indices are kept, as ties require); otherwise
// CSKV_DEV_CAPACITY is flagged.
#include <algorithm>

#include "launch.cuh"
#include "sm100.cuh"

namespace cskv {

constexpr int kTcIdxThreads = 512;   // 16 warps: TMEM lanes 32 (w % 4) .. (entries), columns 32 (w / 4) ..
constexpr int kTcIdxN = 256;         // entries per key tile: two MMAs of M = 128 entries
constexpr int kTcIdxBins = 1024;     // histogram bins per query
constexpr uint32_t kTcIdxRow = 128;  // bytes per operand row in the swizzled layout (Di <= 128)
constexpr uint32_t kTcIdxTile = kTcIdxN * kTcIdxRow;  // 32 KiB: one key tile
constexpr int kTcIdxStages = 4;      // key tiles in flight (cp.async groups)

struct TcIdxSmem {
  static constexpr size_t a = 0;                                     // the Q tile: 128 rows x 128 B
  static constexpr size_t b = a + 128 * kTcIdxRow;                   // the key tile ring
  static constexpr size_t ks = b + kTcIdxStages * (size_t)kTcIdxTile;            // key scales
  static constexpr size_t hist = ks + (kTcIdxStages + 1) * kTcIdxN * sizeof(float);  // QT x padded bins
  static size_t bytes(int QT) { return hist + (size_t)QT * (kTcIdxBins + kTcIdxBins / 32) * sizeof(unsigned) + 1024; }
};

// Order-preserving 32-bit key of a float, and its histogram bin: 16 bins per octave (exponent
// and 4 mantissa bits) for positive scores from 2^-30 up (bins 1 .. 1023, the top bin also
// holding everything from 2^34), bin 0 for scores <= 0 and below 2^-30.  Monotone in the score.
__device__ __forceinline__ uint32_t ord_key(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ int score_bin(float f) {
  if (!(f > 0.f)) return 0;
  const int k12 = (int)(__float_as_uint(f) >> 19);  // exponent field * 16 + top 4 mantissa bits
  return min(max(k12 - (127 - 30) * 16 + 1, 0), kTcIdxBins - 1);
}

// The lowest score of bin b (b >= 1; bin 0: -inf): score_bin(f) >= b  <=>  f >= bin_floor(b).
__device__ __forceinline__ float bin_floor(int b) {
  if (b <= 0) return -INFINITY;
  if (b >= kTcIdxBins) return INFINITY;
  return __uint_as_float((uint32_t)(b - 1 + (127 - 30) * 16) << 19);
}

__device__ __forceinline__ uint32_t sw_off_idx(int r, int c) {
  return (uint32_t)r * kTcIdxRow + ((uint32_t)((c & 7) ^ (r & 7)) << 4);
}

// Instruction descriptor of kind::f8f6f4 with E4M3 A and B (format code 0) and fp32 D.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void tc_mma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

struct TcIdxParams {
  const uint8_t* q_idx;   // [T, Hi, Di] E4M3
  const float* q_scale;   // [T, Hi] or null
  const uint8_t* k_idx;   // [entries, Di] E4M3
  const float* k_scale;   // [entries] or null
  const float* head_w;    // [Hi] or null
  const int32_t* q_seq;
  const int64_t* q_pos;
  const int64_t* ent_off;
  int batch, T, Hi, Di, k;
  int64_t cap;            // candidate slots per query
  float* cand_score;      // [T, cap]
  int32_t* cand_idx;      // [T, cap]
  int64_t* cand_n;        // [T]
  int* st;
};

template <int HI, int DI>
__global__ void __launch_bounds__(kTcIdxThreads, 1) lindex_tc_kernel(TcIdxParams p) {
  constexpr int QT = 128 / HI;    // queries per CTA
  constexpr int QPW = 32 / HI;    // queries of a warp's 32 columns
  constexpr int KC = DI / 16;     // 16-byte chunks per operand row
  constexpr int HB = kTcIdxBins + kTcIdxBins / 32;  // a query's histogram row, padded
  static_assert(HI == 8 || HI == 16, "four or two queries per warp");
  extern __shared__ __align__(1024) uint8_t smraw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~(uintptr_t)1023);
  uint8_t* Qs = sm + TcIdxSmem::a;
  uint8_t* Ks = sm + TcIdxSmem::b;
  float* ks_s = reinterpret_cast<float*>(sm + TcIdxSmem::ks);
  unsigned* hist = reinterpret_cast<unsigned*>(sm + TcIdxSmem::hist);
  __shared__ uint64_t bar[2];
  __shared__ uint32_t tmem_base;
  __shared__ int q_seq_s[QT];
  __shared__ int64_t q_vis[QT];
  __shared__ int q_thr[QT];                        // bin b* of the query, or a bin above all (no entry)
  __shared__ unsigned q_bin_lo[QT], q_bin_hi[QT];  // order keys of the lowest / highest score kept from b*
  __shared__ int q_over[QT];
  __shared__ int q_cnt[8][QT];                     // pass 2: candidates of each 32-entry segment of a tile
  __shared__ int q_floor[QT];                      // pass 1: bins below it cannot hold the k_eff-th score
  __shared__ int tile_np[kTcIdxStages + 1];        // the last tile of the scale buffer with a scale <= 0
  __shared__ float sq_s[128], w_s[128];            // per column (t, h): the query scale, the head weight
  __shared__ int seq_cur;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int lq = warp & 3;   // TMEM lane quarter: entries 32 lq .. 32 lq + 31 of a tile
  const int cq = warp >> 2;  // column quarter: (t, h) columns 32 cq .. 32 cq + 31, queries QPW cq ..
  const int q0 = cq * QPW;   // the warp's first query (of the CTA's QT)
  const int t0 = blockIdx.x * QT;
  if (warp == 0) {
    tmem_alloc(&tmem_base, 512);  // two accumulators of 256 columns (two 128-entry halves each)
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
  }
  pdl_wait();
  // ---- the CTA's queries: sequence, visible entries; the Q tile (rows of absent queries: zeros)
  if (tid < QT) {
    const int tq = t0 + tid;
    int s = -1;
    int64_t v = 0;
    if (tq < p.T) {
      s = __ldg(p.q_seq + tq);
      if (s < 0 || s >= p.batch) {
        flag(p.st, CSKV_DEV_BAD_INDEX);
        s = -1;
      } else {
        const int64_t pos = __ldg(p.q_pos + tq);
        const int64_t n = __ldg(p.ent_off + s + 1) - __ldg(p.ent_off + s);
        v = pos >= 0 ? (pos + 1) / 4 : 0;
        if (v > n) {
          flag(p.st, CSKV_DEV_BAD_INDEX);
          v = n;
        }
      }
      if (s < 0) p.cand_n[tq] = 0;
    }
    q_seq_s[tid] = s;
    q_vis[tid] = v;
  }
  if (tid < 128) {
    const int tr = t0 + tid / HI, hh = tid % HI;
    sq_s[tid] = (tr < p.T && p.q_scale) ? __ldg(p.q_scale + (size_t)tr * HI + hh) : 1.f;
    w_s[tid] = p.head_w ? __ldg(p.head_w + hh) : 1.f;
  }
  for (int i = tid; i < 128 * KC; i += kTcIdxThreads) {
    const int r = i / KC, c = i % KC;
    const int tr = t0 + r / HI;
    const bool ok = tr < p.T;
    cp_async16(Qs + sw_off_idx(r, c), p.q_idx + ((size_t)(ok ? tr : 0) * HI + r % HI) * DI + 16 * c, ok ? 16u : 0u);
  }
  cp_async_wait_all();
  if (tid == 0) seq_cur = -2;
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // the factored form's weights w_h * sq_{t,h} of the warp's 32 columns (the same in every lane)
  float crow[32];
  bool sq_pos = true;
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    crow[c] = w_s[cq * 32 + c] * sq_s[cq * 32 + c];
    sq_pos = sq_pos && sq_s[cq * 32 + c] > 0.f;
  }
  sq_pos = __syncthreads_and(sq_pos) != 0;  // every query scale of the CTA is positive

  const uint32_t q_addr = smem_u32(Qs), k_addr = smem_u32(Ks);
  const uint32_t idesc = idesc_e4m3_f32(128, 128);
  const uint32_t lane_base = (uint32_t)(lq * 32) << 16;
  uint32_t uses0 = 0u, uses1 = 0u;  // completed phases of bar[0], bar[1]
  bool alive = true;

  // ---- one sequence of the CTA's queries at a time (a prefill chunk: one)
  for (;;) {
    if (tid == 0) {
      int s = -1;
      for (int i = 0; i < QT; ++i) {
        const int si = q_seq_s[i];
        if (si >= 0 && si > seq_cur && (s < 0 || si < s)) s = si;
      }
      seq_cur = s;
    }
    __syncthreads();
    const int s = seq_cur;
    if (s < 0) break;
    bool mine[QPW];
    int64_t V[QPW];
#pragma unroll
    for (int j = 0; j < QPW; ++j) {
      mine[j] = q_seq_s[q0 + j] == s;
      V[j] = mine[j] ? q_vis[q0 + j] : 0;
    }
    int64_t vmax = 0;
    for (int i = 0; i < QT; ++i)
      if (q_seq_s[i] == s && q_vis[i] > vmax) vmax = q_vis[i];
    const int64_t e_base = __ldg(p.ent_off + s);
    const int ntiles = (int)((vmax + kTcIdxN - 1) / kTcIdxN);

    for (int pass = 0; pass < 2 && alive; ++pass) {
      if (pass == 0) {
        for (int i = tid; i < QT * HB; i += kTcIdxThreads) hist[i] = 0u;
        if (tid < QT) q_floor[tid] = 0;
      }
      int64_t run[QPW];  // pass 2: candidates appended so far for each of the warp's queries
      float thr_lo[QPW], thr_hi[QPW];  // pass 2: the scores of bin b* are thr_lo <= s < thr_hi
#pragma unroll
      for (int j = 0; j < QPW; ++j) {
        run[j] = 0;
        const int thr = pass == 1 ? q_thr[q0 + j] : 0;
        thr_lo[j] = bin_floor(thr);
        thr_hi[j] = bin_floor(thr + 1);
      }
      if (tid < kTcIdxStages + 1) tile_np[tid] = -1;
      __syncthreads();
      auto load_tile = [&](int n) {  // one cp.async group per tile, empty past the last
        if (n >= ntiles) {
          cp_async_commit();
          return;
        }
        const int buf = n % kTcIdxStages;
        const int64_t e0 = (int64_t)n * kTcIdxN;
        // 128 entries x KC chunks of 16 bytes; entries past vmax read nothing (zeros)
        for (int i = tid; i < kTcIdxN * KC; i += kTcIdxThreads) {
          const int r = i / KC, c = i % KC;
          const bool ok = e0 + r < vmax;
          cp_async16(Ks + buf * kTcIdxTile + sw_off_idx(r, c),
                     p.k_idx + (size_t)(e_base + (ok ? e0 + r : 0)) * DI + 16 * c, ok ? 16u : 0u);
        }
        // the scales (kTcIdxStages + 1 buffers, so that the epilogue running beside this load
        // reads another one); a scale <= 0 marks the buffer with the tile's number
        const int kb = n % (kTcIdxStages + 1);
        if (tid < kTcIdxN) {
          const bool ok = e0 + tid < vmax;
          const float v = ok && p.k_scale ? __ldg(p.k_scale + e_base + e0 + tid) : 1.f;
          ks_s[kb * kTcIdxN + tid] = v;
          if (!(v > 0.f)) tile_np[kb] = n;
        }
        static_assert(kTcIdxN <= kTcIdxThreads, "one scale per thread");
        cp_async_commit();
      };
      auto epilogue = [&](int n) {
        const int buf = n & 1;
        const int kb = n % (kTcIdxStages + 1);
        // the factored form needs positive scales: the tile's keys and every query's
        const bool fact = sq_pos && tile_np[kb] != n;
        if (pass == 0 && (n & 3) == 3 && warp < QT) {
          // raise query `warp`'s floor: the lowest bin of the 32-bin block in which the count
          // from the top reaches k_eff (counts only grow, so a floor read from a histogram
          // still being filled is valid)
          const int qq = warp;
          const unsigned keff = (unsigned)min((int64_t)p.k, q_seq_s[qq] == s ? q_vis[qq] : (int64_t)0);
          const unsigned* hq = hist + qq * HB;
          const int blk = 31 - lane;  // lane 0: the top block; bin b at b + b / 32 (padding)
          unsigned c = 0;
#pragma unroll 8
          for (int i = 0; i < 32; ++i) c += *(volatile const unsigned*)(hq + blk * 33 + i);
          unsigned incl = c;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
          }
          const int f = (keff > 0 && incl >= keff && incl - c < keff) ? blk * 32 : 0;
          const int fl = __reduce_max_sync(0xffffffffu, f);
          if (lane == 0 && fl > q_floor[qq]) q_floor[qq] = fl;
        }
        // both 128-entry halves of the tile: TMEM columns buf * 256 + half * 128 + (t, h)
        float sc[2][QPW];
        bool vis[2][QPW];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t v[32];
          tmem_ld32(tmem_base + (uint32_t)(buf * kTcIdxN + hf * 128 + cq * 32) + lane_base, v);
          tmem_ld_wait();
          if (hf == 1) tc_fence_before();
          const int r = hf * 128 + lq * 32 + lane;  // this thread's entry in the tile
          const int64_t e = (int64_t)n * kTcIdxN + r;
          const float ke = ks_s[kb * kTcIdxN + r];
#pragma unroll
          for (int j = 0; j < QPW; ++j) {
            float a = 0.f;
            if (fact) {
#pragma unroll
              for (int hh = 0; hh < HI; ++hh)
                a = fmaf(crow[j * HI + hh], fmaxf(0.f, __uint_as_float(v[j * HI + hh])), a);
              a *= ke;
            } else {
#pragma unroll
              for (int hh = 0; hh < HI; ++hh) {
                const int c = cq * 32 + j * HI + hh;
                a = fmaf(w_s[c], fmaxf(0.f, (sq_s[c] * ke) * __uint_as_float(v[j * HI + hh])), a);
              }
            }
            sc[hf][j] = a;
            vis[hf][j] = mine[j] && e < V[j];
          }
        }
        if (pass == 0) {
          // only scores at or above the query's floor are binned (a comparison first: most fail)
#pragma unroll
          for (int j = 0; j < QPW; ++j) {
            const float flv = bin_floor(*(volatile int*)&q_floor[q0 + j]);
#pragma unroll
            for (int hf = 0; hf < 2; ++hf)
              if (vis[hf][j] && sc[hf][j] >= flv) {
                const int b = score_bin(sc[hf][j]);
                atomicAdd(&hist[(q0 + j) * HB + b + (b >> 5)], 1u);
              }
          }
          return;
        }
        // pass 2: each query's kept entries of this thread's two 32-entry segments (half, lane
        // quarter) in lane order (ballot), after the segments before them in the tile
        unsigned mask[2][QPW];
        bool keep[2][QPW];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
#pragma unroll
          for (int j = 0; j < QPW; ++j) {
            keep[hf][j] = vis[hf][j] && sc[hf][j] >= thr_lo[j];
            mask[hf][j] = __ballot_sync(0xffffffffu, keep[hf][j]);
            if (lane == 0) q_cnt[hf * 4 + lq][q0 + j] = __popc(mask[hf][j]);
          }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < QPW; ++j) {
          int cnt[8];
          int total = 0;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            cnt[c] = q_cnt[c][q0 + j];
            total += cnt[c];
          }
          const int tq = t0 + q0 + j;
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            if (keep[hf][j]) {
              int before = 0;
#pragma unroll
              for (int c = 0; c < 8; ++c) before += c < hf * 4 + lq ? cnt[c] : 0;
              const int64_t pos = run[j] + before + __popc(mask[hf][j] & ((1u << lane) - 1u));
              if (pos < p.cap) {
                p.cand_score[(size_t)tq * p.cap + pos] = sc[hf][j];
                p.cand_idx[(size_t)tq * p.cap + pos] = (int32_t)((int64_t)n * kTcIdxN + hf * 128 + lq * 32 + lane);
              } else {
                q_over[q0 + j] = 1;
              }
              if (sc[hf][j] < thr_hi[j]) {  // in bin b*
                atomicMin(&q_bin_lo[q0 + j], ord_key(sc[hf][j]));
                atomicMax(&q_bin_hi[q0 + j], ord_key(sc[hf][j]));
              }
            }
          }
          run[j] += total;
        }
      };
      for (int n = 0; n < kTcIdxStages - 1; ++n) load_tile(n);
      for (int n = 0; n < ntiles; ++n) {
        cp_async_wait_group<kTcIdxStages - 2>();  // tile n's group has landed
        fence_proxy_async_smem();
        tc_fence_before();
        // one barrier a tile: tile n's keys and scales are visible, the epilogue before has
        // read its TMEM accumulator, and a wait that gave up stops every thread
        if (__syncthreads_or(!alive)) {
          alive = false;
          break;
        }
        tc_fence_after();
        if (tid == 0) {
          // D[entry, (t, h)] = K_half Q^T for both 128-entry halves of the tile: A = the half
          // (M = 128 entries), B = the Q tile (N = 128 columns), D = 128 TMEM columns each
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const uint32_t d = tmem_base + (uint32_t)((n & 1) * kTcIdxN + hf * 128);
            const uint32_t kt = k_addr + (uint32_t)((n % kTcIdxStages) * kTcIdxTile + hf * 128 * kTcIdxRow);
#pragma unroll
            for (int kk = 0; kk < DI / 32; ++kk)  // K = 32 bytes (32 E4M3 elements) per instruction
              tc_mma_f8(d, smem_desc_sw128(kt + kk * 32, 16, 1024), smem_desc_sw128(q_addr + kk * 32, 16, 1024),
                        idesc, kk > 0);
          }
          tc_commit(&bar[n & 1]);
        }
        if (n >= 1) {
          const bool b1 = ((n - 1) & 1) != 0;
          if (!mbar_wait_bounded(&bar[b1 ? 1 : 0], (b1 ? uses1 : uses0) & 1u)) {
            flag(p.st, CSKV_DEV_TIMEOUT);
            alive = false;
          }
          if (b1) ++uses1; else ++uses0;
          tc_fence_after();
        }
        load_tile(n + kTcIdxStages - 1);  // into the stage MMA n - 1 (complete) read
        if (n >= 1) epilogue(n - 1);
      }
      if (ntiles > 0 && __syncthreads_and(alive)) {
        const bool b1 = ((ntiles - 1) & 1) != 0;
        if (!mbar_wait_bounded(&bar[b1 ? 1 : 0], (b1 ? uses1 : uses0) & 1u)) {
          flag(p.st, CSKV_DEV_TIMEOUT);
          alive = false;
        }
        if (b1) ++uses1; else ++uses0;
        tc_fence_after();
        epilogue(ntiles - 1);
      }
      cp_async_wait_all();
      __syncthreads();
      if (!alive) break;
      if (pass == 0) {
        // ---- b*: the bin of the k_eff-th best score of each query, counted from the top
        //      (warp w takes query w; lane j sums the block of 32 bins 31 - j)
        if (warp < QT) {
          const int qq = warp;
          const int64_t vq = q_seq_s[qq] == s ? q_vis[qq] : 0;
          const unsigned keff = (unsigned)min((int64_t)p.k, vq);
          const unsigned* hq = hist + qq * HB;
          const int blk = 31 - lane;
          unsigned c = 0;
          for (int i = 0; i < 32; ++i) c += hq[blk * 33 + i];
          unsigned incl = c;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
          }
          const unsigned excl = incl - c;
          int bstar = kTcIdxBins;  // no entry: a bin above all
          if (keff > 0 && excl < keff && incl >= keff) {
            unsigned cum = excl;
            for (int i = 31; i >= 0; --i) {
              cum += hq[blk * 33 + i];
              if (cum >= keff) {
                bstar = blk * 32 + i;
                break;
              }
            }
          }
          bstar = __reduce_min_sync(0xffffffffu, bstar);
          if (lane == 0) {
            q_thr[qq] = keff > 0 ? bstar : kTcIdxBins;
            q_bin_lo[qq] = 0xFFFFFFFFu;
            q_bin_hi[qq] = 0u;
            q_over[qq] = 0;
          }
        }
        __syncthreads();
      } else {
        // ---- the queries' candidate counts; an overflow is exact only inside a pile of equal
        //      scores (the kept ones are the lowest indices of the pile, as ties require)
        if (lq == 0 && lane == 0) {
#pragma unroll
          for (int j = 0; j < QPW; ++j) {
            const int tq = t0 + q0 + j;
            if (mine[j] && tq < p.T) {
              p.cand_n[tq] = run[j] < p.cap ? run[j] : p.cap;
              if (q_over[q0 + j] && q_bin_lo[q0 + j] != q_bin_hi[q0 + j]) flag(p.st, CSKV_DEV_CAPACITY);
            }
          }
        }
        __syncthreads();
      }
    }
    if (!alive) break;
  }
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// out_idx[t, j] = cand_idx[t, out_idx[t, j]] (positions in the candidate list -> entry indices,
// -1 padding kept); the kept rows can be prefetched into L2 as in the scan path.
__global__ void map_candidates_kernel(int32_t* out_idx, const int32_t* cand_idx, int64_t cap, int T, int k,
                                      const int64_t* q_seq_base, const int32_t* q_seq, const uint8_t* pf_rows,
                                      int64_t pf_row_bytes) {
  pdl_wait();
  const int t = blockIdx.y;
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T || j >= k) return;
  const int32_t pos = out_idx[(size_t)t * k + j];
  if (pos < 0) return;
  const int32_t e = __ldg(cand_idx + (size_t)t * cap + pos);
  out_idx[(size_t)t * k + j] = e;
  if (pf_rows) {
    const int s = __ldg(q_seq + t);
    const uint8_t* r = pf_rows + (size_t)(__ldg(q_seq_base + s) + e) * pf_row_bytes;
    for (int64_t o = 0; o < pf_row_bytes; o += 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(r + o));
  }
}

// ------------------------------------------------------------------ host side
bool lindex_tc_shape(int dtype, int Hi, int Di) {
  return dtype == CSKV_FP8E4M3 && (Hi == 8 || Hi == 16) && (Di == 64 || Di == 128);
}

int64_t lindex_tc_cap(int k, int64_t max_entries) {
  int64_t cap = std::max<int64_t>(8192, 2 * (int64_t)k);
  cap = std::min<int64_t>(cap, std::max<int64_t>(max_entries, 1));
  return (cap + 3) / 4 * 4;
}

template <int HI, int DI>
static cudaError_t launch_tc(const TcIdxParams& p, cudaStream_t stream) {
  constexpr int QT = 128 / HI;
  const size_t smem = TcIdxSmem::bytes(QT);
  auto kern = lindex_tc_kernel<HI, DI>;
  cudaError_t e = ensure_smem(kern, smem);
  if (e != cudaSuccess) return e;
  e = launch_dependent(kern, dim3((p.T + QT - 1) / QT), dim3(kTcIdxThreads), smem, stream, p);
  note_launch();
  return e;
}

cudaError_t launch_lindex_tc_candidates(const uint8_t* q_idx, const float* q_scale, const uint8_t* k_idx,
                                        const float* k_scale, const float* head_w, const int32_t* q_seq,
                                        const int64_t* q_pos, const int64_t* ent_off, int batch, int T, int Hi,
                                        int Di, int k, int64_t cap, float* cand_score, int32_t* cand_idx,
                                        int64_t* cand_n, int* st, cudaStream_t stream) {
  TcIdxParams p{q_idx, q_scale, k_idx, k_scale, head_w, q_seq, q_pos, ent_off, batch, T, Hi, Di, k,
                cap,   cand_score, cand_idx, cand_n, st};
  if (Hi == 8) return Di == 64 ? launch_tc<8, 64>(p, stream) : launch_tc<8, 128>(p, stream);
  return Di == 64 ? launch_tc<16, 64>(p, stream) : launch_tc<16, 128>(p, stream);
}

cudaError_t launch_map_candidates(int32_t* out_idx, const int32_t* cand_idx, int64_t cap, int T, int k,
                                  const int64_t* ent_off, const int32_t* q_seq, const uint8_t* pf_rows,
                                  int64_t pf_row_bytes, cudaStream_t stream) {
  cudaError_t e = ensure_smem(map_candidates_kernel, 0);
  if (e != cudaSuccess) return e;
  e = launch_dependent(map_candidates_kernel, dim3((k + 255) / 256, T), dim3(256), 0, stream, out_idx, cand_idx,
                       cap, T, k, ent_off, q_seq, pf_rows, pf_row_bytes);
  note_launch();
  return e;
}

}  // namespace cskv
