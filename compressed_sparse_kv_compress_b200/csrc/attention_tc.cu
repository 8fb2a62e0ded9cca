// Hybrid decode attention on the 5th-generation tensor cores (tcgen05, TMEM accumulators).
//
// [SW] = shareware.cn/news/167317 (DeepSeek V4 Hybrid Attention essay), §八: after 128:1
// compression a dense pass over every entry is the cheaper, regular kernel; §十一: MQA, all
// query heads read one shared KV.  [TR] = trdm.cn/news/516303, §3.1: the online softmax
// (running max and sum) equals the full softmax exactly.
//
// With MQA every gathered K||V row is shared by all H query heads, so one split of rows is a
// real dense contraction: S = Q K^T is [H x rows] x [rows x 128] and O = P V the same size.
// One CTA (4 warps) takes a split of the query's virtual row list (attn_rows.cuh) in chunks
// of up to 128 rows:
//   1. cp.async gathers the chunk's K||V rows into shared memory, one whole 512-byte row per
//      warp instruction, in the 128-byte-swizzle layout (four 16 KiB regions of 128-byte rows:
//      K dims 0-63, K 64-127, V 0-63, V 64-127; chunk c of row r at chunk c ^ (r & 7), so a
//      row's 32 pieces land on all 32 banks);
//   2. one thread issues tcgen05.mma: S[128 x nc] (fp32, TMEM) = Q[128 x 128] K^T (bf16);
//   3. thread h (TMEM lane h) owns head h's row: masks skipped rows, updates the running
//      max / sum (log2 units), rescales its O row in TMEM when the max grew, and writes
//      P = 2^(s - m) as bf16 into shared memory;
//   4. one thread issues O[128 x 128] (+)= P[128 x nc] V[nc x 128] (V read MN-major).
// Q, K and P are K-major operands, V is MN-major; all four use the same swizzled layout.
// Heads beyond H are zero rows of Q (M is always 128).
//
// Merging the splits of a query ([TR] §3.1; the sink joins once, [SW] §十二):
//  * cluster mode (p.cluster = the split count, at most 16): the query's splits are the CTAs
//    of one thread-block cluster.  Each writes its partial (unnormalised O rows, (m, l)) to
//    the workspace, a cluster barrier publishes them, and each CTA fetches its heads' slices
//    of every split with TMA bulk copies and merges 128 / p.cluster of the heads -- no second
//    kernel and no launch gap.  (Reading the partials from the
//    other CTAs' shared memory instead was slower: every remote load a round trip over the
//    SM-to-SM network.)
//  * otherwise the split's (m, l, O) go to the workspace and attn_combine_kernel merges.
#include <mutex>

#include "attn_rows.cuh"
#include "kv8.cuh"
#include "sm100.cuh"

namespace cskv {

constexpr int kTcThreads = 128;
constexpr int kTcChunk = 128;                      // rows per chunk (MMA N of S, K of PV)
constexpr uint32_t kRegion = 128 * 128;             // 128 rows x 128 bytes: one swizzled region
constexpr uint32_t kTileBytes = 2 * kRegion;        // one 128 x 128 bf16 operand tile
// Q, K||V and P tiles; P takes K's place (K is dead once S = Q K^T has completed), so a CTA
// needs ~97 KB and fits on an SM beside the indexer's CTA.
constexpr size_t kTcSmem = 3 * (size_t)kTileBytes + 1024;

// Byte offset of 16-byte chunk c of row r (c < 16 for a 256-byte row, < 32 for a 512-byte
// K||V row) in the 128-byte-swizzle layout.
__device__ __forceinline__ uint32_t sw_off(int r, int c) {
  return (uint32_t)(c >> 3) * kRegion + (uint32_t)r * 128 + ((uint32_t)((c & 7) ^ (r & 7)) << 4);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Cluster mode: merges the query's splits (the CTAs of this cluster, rank = split) once every
// split has written its partial to the workspace, and writes the output and lse.  Called by
// all threads of every CTA of the cluster.  Partial layout, per (query, split): the
// unnormalised O as float4 groups of 4 dimensions, grouped by merging CTA -- CTA r merges the
// heads r HPC .. r HPC + nh_r - 1 (HPC = 128 / CS, nh_r = min(HPC, H - r HPC)), and its slice
// [group 0..31][head] of nh_r * 512 contiguous bytes sits at offset r HPC * 512 -- and (m, l)
// per head.  After the cluster barrier (release / acquire at cluster scope; the writers'
// proxy fence lets the TMA see their stores) one thread fetches the CS slices of its heads
// with TMA bulk copies into the dead K||V tile (all in flight at once: one round trip), the
// threads load their heads' (m, l) meanwhile, and each thread (head hh, groups g0, g0 + CS,
// ...) folds every split's (m, l) with the sink,
//   M = max(max_s m_s, sink),  L = sum_s 2^(m_s - M) l_s + 2^(sink - M),
// and sums the splits' values, scaled by 2^(m_s - M) / L, from shared memory.
template <int CS>
__device__ __forceinline__ void cluster_merge(const AttnParams& p, int t, float4* stage, uint64_t* bar_m) {
  cluster_sync();
  fence_proxy_async_global();
  const int tid = threadIdx.x, H = p.Hv;  // a pair: 2 p.H heads, its queries' outputs adjacent in memory
  const uint32_t rank = cluster_rank();
  constexpr int HPC = 128 / CS;  // heads merged by a CTA
  constexpr int NG = 32 / CS;    // dimension groups per thread
  const int h0 = (int)rank * HPC;
  const int nh = max(0, min(HPC, H - h0));
  if (nh == 0) return;  // no barrier follows: a CTA without heads is done
  const float4* po = reinterpret_cast<const float4*>(p.part_acc) + (size_t)t * CS * H * 32 + (size_t)h0 * 32;
  const uint32_t slice = (uint32_t)nh * 512u;
  if (tid == 0) {
    mbar_arrive_expect_tx(bar_m, CS * slice);
#pragma unroll
    for (int s = 0; s < CS; ++s) tma_bulk_g2s(stage + (size_t)s * nh * 32, po + (size_t)s * H * 32, slice, bar_m);
  }
  const int hh = tid % HPC, g0 = tid / HPC;
  const int h = h0 + hh;
  // a pair's second query may not exist (an odd T): its heads write nothing
  const bool mine = hh < nh && (!p.pairs || 2 * t + (h >= p.H ? 1 : 0) < p.T);
  float2 mls[CS];
  const float2* ml = reinterpret_cast<const float2*>(p.part_ml) + (size_t)t * CS * H + (mine ? h : h0);
#pragma unroll
  for (int s = 0; s < CS; ++s) mls[s] = __ldcg(ml + (size_t)s * H);
  const float sk = (p.sink && mine) ? __ldg(p.sink + h % p.H) * kLog2e : -INFINITY;
  float M = sk;
#pragma unroll
  for (int s = 0; s < CS; ++s) M = fmaxf(M, mls[s].x);
  float f[CS], L = 0.f;
#pragma unroll
  for (int s = 0; s < CS; ++s) {
    f[s] = mls[s].x == -INFINITY ? 0.f : exp2f(mls[s].x - M);  // a split without rows wrote no O
    L = fmaf(mls[s].y, f[s], L);
  }
  if (M != -INFINITY && p.sink) L += exp2f(sk - M);
  const float inv = L > 0.f ? 1.f / L : 0.f;
  if (!mbar_wait_bounded(bar_m, 0)) flag(p.st, CSKV_DEV_TIMEOUT);
  if (!mine) return;
  float* dst = p.out + ((size_t)t * H + h) * kHeadDim;
#pragma unroll
  for (int k = 0; k < NG; ++k) {
    const int g = g0 + CS * k;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int s = 0; s < CS; ++s)
      if (f[s] != 0.f) {
        const float4 v = stage[(size_t)s * nh * 32 + g * nh + hh];
        a.x = fmaf(v.x, f[s], a.x);
        a.y = fmaf(v.y, f[s], a.y);
        a.z = fmaf(v.z, f[s], a.z);
        a.w = fmaf(v.w, f[s], a.w);
      }
    dst[4 * g] = a.x * inv;
    dst[4 * g + 1] = a.y * inv;
    dst[4 * g + 2] = a.z * inv;
    dst[4 * g + 3] = a.w * inv;
  }
  if (g0 == 0 && p.lse) p.lse[(size_t)t * H + h] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
}

// At most 160 registers a thread: 4 warps x 32 x 160 = 20,480, what an SM has left beside the
// indexer (16 warps x 32 x 88), so the HCA attention and a parked CSA attention fit beside it.
__global__ void __maxnreg__(160) attn_tc_kernel(AttnParams p) {
  extern __shared__ __align__(1024) uint8_t smraw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~(uintptr_t)1023);
  uint8_t* Qs = sm;                   // A of S = Q K^T   [128 heads x 128 d], K-major
  uint8_t* KVs = sm + kTileBytes;     // K: B of S [128 rows x 128 d], K-major (regions 0-1);
                                      // V: B of O = P V [128 rows (K) x 128 d (N)], MN-major (2-3)
  uint8_t* Ps = KVs;                  // A of O = P V     [128 heads x 128 rows], K-major: K's regions,
                                      // written only after the S MMA has read K (bar_s)
  __shared__ uint64_t bar_s, bar_o, bar_m;
  __shared__ uint32_t tmem_base;
  __shared__ const __nv_bfloat16* row_src[kTcChunk];  // address of each chunk row, null = skipped
  __shared__ uint32_t row_mask[2][kTcChunk / 32];  // bit r: chunk row r is attended (by the pair's
                                                   // first / second query; one query: [0])

  // t: the unit of work -- a query, or (pairs) the pair of queries 2t, 2t + 1
  const int t = blockIdx.y, split = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tq0 = p.pairs ? 2 * t : t;
  // ---- set-up that reads no input overlaps the previous kernel (dependent launch)
  if (warp == 0) {
    tmem_alloc(&tmem_base, 256);  // S: columns 0..127, O: columns 128..255
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar_s, 1);
    mbar_init(&bar_o, 1);
    mbar_init(&bar_m, 1);
    fence_mbar_init();
  }
  // warm L2 with the query's metadata and the selected indices of this split's first rows
  // (prefetches only move lines into L2, which stays coherent with the writes being waited for)
  const int64_t r0 = (int64_t)split * p.rows_per_split;
  if (tid == 0) asm volatile("prefetch.global.L2 [%0];" ::"l"(p.q_seq + tq0));
  if (tid == 1) asm volatile("prefetch.global.L2 [%0];" ::"l"(p.q_pos + tq0));
  if (tid == 2) asm volatile("prefetch.global.L2 [%0];" ::"l"(p.cmp_off));
  if (tid == 3) asm volatile("prefetch.global.L2 [%0];" ::"l"(p.raw_off));
  if (tid == 4 && p.raw_tok0) asm volatile("prefetch.global.L2 [%0];" ::"l"(p.raw_tok0));
  if (p.mode == CSKV_CSA && tid >= 32 && tid < 32 + kTcChunk / 32 && r0 + (tid - 32) * 32 < p.k)
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p.idx + (size_t)t * p.k + r0 + (tid - 32) * 32));
  pdl_wait();
  // the first chunk's selected indices load beside the query's metadata
  const int64_t r_pre = r0 + tid;
  const int64_t e_pre = (p.mode == CSKV_CSA && r_pre < p.k && tid < min((int64_t)kTcChunk, (int64_t)p.rows_per_split))
                            ? (int64_t)__ldg(p.idx + (size_t)t * p.k + r_pre)
                            : (int64_t)-2;
  const QueryRows q = query_rows(p, tq0);
  if (q.s < 0 && split == 0 && tid == 0) flag(p.st, CSKV_DEV_BAD_INDEX);
  // a pair: its second query must be the next position of the same sequence (else flagged and
  // left out: its rows then attend to nothing); the union of the two row lists
  QueryRows q1 = q;
  bool q1v = false;
  int64_t nu = 0, n_rows = q.n_rows;
  if (p.pairs) {
    if (tq0 + 1 < p.T) {
      q1 = query_rows(p, tq0 + 1);
      q1v = q.s >= 0 && q1.s == q.s && q1.pos == q.pos + 1;
      if (!q1v && split == 0 && tid == 0) flag(p.st, CSKV_DEV_BAD_INDEX);
    }
    nu = max(q.n_cmp, q1v ? q1.n_cmp : (int64_t)0);
    n_rows = nu + p.window + (q1v ? 1 : 0);
  }
  // a CTA without rows (bad query, or a split past the query's rows) runs no chunk and
  // only releases its TMEM at the end
  const int64_t r1 = q.s < 0 ? r0 : max(r0, min(n_rows, r0 + p.rows_per_split));
  // cluster mode has no merge kernel to notice rows beyond the last split: flag them here
  if (p.cluster && q.s >= 0 && split == p.max_splits - 1 && tid == 0 && n_rows > r0 + p.rows_per_split)
    flag(p.st, CSKV_DEV_CAPACITY);
  const int H = p.Hv;  // heads of the unit: the partials and the merge count in these
  const __nv_bfloat16* cmp = reinterpret_cast<const __nv_bfloat16*>(p.kv_cmp);
  const __nv_bfloat16* raw = reinterpret_cast<const __nv_bfloat16*>(p.kv_raw);
  const __nv_bfloat16* qg = reinterpret_cast<const __nv_bfloat16*>(p.q) + (size_t)tq0 * p.H * kHeadDim;
  // rows of the Q tile that hold a head: h < H for one query; a pair's second query (rows
  // p.H .. 2 p.H - 1) only when it is there
  const int hq = p.pairs ? (q1v ? H : p.H) : H;

  // Q tile: a warp instruction copies two 256-byte head rows (zero rows beyond the heads); the
  // copies complete together with the first chunk's gather, and the barriers of that chunk
  // publish the TMEM address.  A pair's second query follows the first in memory.
  if (r0 < r1)
    for (int it = 0; it < 16; ++it) {
      const int h = warp * 32 + it * 2 + (lane >> 4), c = lane & 15;
      cp_async16(Qs + sw_off(h, c), h < hq ? (const void*)(qg + (size_t)h * kHeadDim + 8 * c) : (const void*)qg,
                 h < hq ? 16u : 0u);
    }
  tc_fence_before();
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;

  const uint32_t qs_a = smem_u32(Qs), ks_a = smem_u32(KVs), vs_a = ks_a + 2 * kRegion, ps_a = smem_u32(Ps);
  float m_run = -INFINITY, l_run = 0.f;
  bool alive = true;
  int c = 0;
  for (int64_t a = r0; a < r1 && alive; a += kTcChunk, ++c) {
    const int rows = (int)min((int64_t)kTcChunk, r1 - a);
    const int nc = (rows + 31) & ~31;  // MMA N / K of this chunk (multiple of 32)
    // ---- resolve the chunk's rows
    {
      int64_t off = -1;
      bool is_raw = false, ok0 = false, ok1 = false;
      if (p.pairs) {
        if (tid < rows) off = resolve_pair_row(p, q, q1, q1v, nu, a + tid, &is_raw, &ok0, &ok1);
      } else {
        if (tid < rows) off = resolve_row(p, q, tq0, a + tid, &is_raw, a == r0 ? e_pre : (int64_t)-2);
        ok0 = off >= 0;
      }
      // an FP8 main-KV row (kv8.cuh) is marked by bit 0 of its address (rows are 16-byte aligned)
      row_src[tid] = off < 0   ? nullptr
                     : is_raw ? raw + off
                     : p.kv8  ? reinterpret_cast<const __nv_bfloat16*>(
                                   reinterpret_cast<uintptr_t>(p.kv_cmp) + (uintptr_t)(off / kRow) * kKv8RowBytes + 1u)
                              : cmp + off;
      const uint32_t b0 = __ballot_sync(0xffffffffu, ok0), b1 = __ballot_sync(0xffffffffu, ok1);
      if (lane == 0) {
        row_mask[0][warp] = b0;
        row_mask[1][warp] = b1;
      }
    }
    __syncthreads();
    // ---- gather: one whole 512-byte K||V row per warp instruction (lane j copies its
    //      16-byte piece j), eight rows in flight per warp; skipped rows up to nc are
    //      zero-filled; an FP8 main-KV row is decoded to bf16 by the lanes and stored
    if (p.kv8) {
#pragma unroll 8
      for (int r = warp; r < nc; r += 4) {
        const __nv_bfloat16* row = row_src[r];
        const uintptr_t ra = reinterpret_cast<uintptr_t>(row);
        if (ra & 1u)
          *reinterpret_cast<uint4*>(KVs + sw_off(r, lane)) =
              kv8_lane_bf16x8(reinterpret_cast<const uint8_t*>(ra - 1u), lane);
        else
          cp_async16(KVs + sw_off(r, lane), row ? (const void*)(row + 8 * lane) : (const void*)qg, row ? 16u : 0u);
      }
    } else {
#pragma unroll 8
      for (int r = warp; r < nc; r += 4) {
        const __nv_bfloat16* row = row_src[r];
        cp_async16(KVs + sw_off(r, lane), row ? (const void*)(row + 8 * lane) : (const void*)qg, row ? 16u : 0u);
      }
    }
    cp_async_wait_all();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tS = tmem_base, tO = tmem_base + 128;
    // ---- S = Q K^T
    if (tid == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, nc, false, false);
      // K steps of 16 elements (32 bytes): region kk / 4, offset 32 * (kk % 4) inside the row
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t koff = (uint32_t)(kk >> 2) * kRegion + (uint32_t)(kk & 3) * 32;
        tc_mma_f16(tS, smem_desc_sw128(qs_a + koff, 16, 1024), smem_desc_sw128(ks_a + koff, 16, 1024), idesc,
                   kk > 0);
      }
      tc_commit(&bar_s);
    }
    if (!mbar_wait_bounded(&bar_s, c & 1)) flag(p.st, CSKV_DEV_TIMEOUT);
    tc_fence_after();
    // ---- online softmax of row tid over the nc columns (log2 units); a pair's rows take the
    //      mask of their query
    const int mhalf = (p.pairs && tid >= p.H) ? 1 : 0;
    const float sl2 = p.scale_log2;
    // pass 1: row max of the raw logits over the attended columns (the scale is positive, so
    // it is applied once, to the max); four independent max chains.  Blocks of 32 columns
    // that are all attended (the common case) skip the mask.
    float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
    for (int cc = 0; cc < nc; cc += 32) {
      const uint32_t vm = row_mask[mhalf][cc >> 5];
      uint32_t v[32];
      tmem_ld32(tS + lane_base + cc, v);
      tmem_ld_wait();
      if (vm == 0xFFFFFFFFu) {
#pragma unroll
        for (int i = 0; i < 32; ++i) mx4[i & 3] = fmaxf(mx4[i & 3], __uint_as_float(v[i]));
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          mx4[i & 3] = fmaxf(mx4[i & 3], ((vm >> i) & 1u) ? __uint_as_float(v[i]) : -INFINITY);
      }
    }
    const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * sl2;
    const float m_new = fmaxf(m_run, mx);
    const float alpha = (m_new == -INFINITY) ? 1.f : fast_exp2(m_run - m_new);
    const float nm = (m_new == -INFINITY) ? 0.f : -m_new;
    // pass 2: P = 2^(s * scale - m) as bf16 into the P tile; four independent partial sums
    float ls4[4] = {0.f, 0.f, 0.f, 0.f};
    for (int cc = 0; cc < nc; cc += 32) {
      const uint32_t vm = row_mask[mhalf][cc >> 5];
      uint32_t v[32];
      tmem_ld32(tS + lane_base + cc, v);
      tmem_ld_wait();
      float pr[32];
      if (vm == 0xFFFFFFFFu) {
#pragma unroll
        for (int i = 0; i < 32; ++i) pr[i] = fast_exp2(fmaf(__uint_as_float(v[i]), sl2, nm));
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) pr[i] = ((vm >> i) & 1u) ? fast_exp2(fmaf(__uint_as_float(v[i]), sl2, nm)) : 0.f;
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) ls4[i & 3] += pr[i];
#pragma unroll
      for (int g = 0; g < 4; ++g)
        *reinterpret_cast<uint4*>(Ps + sw_off(tid, (cc >> 3) + g)) =
            make_uint4(pack_bf16(pr[8 * g], pr[8 * g + 1]), pack_bf16(pr[8 * g + 2], pr[8 * g + 3]),
                       pack_bf16(pr[8 * g + 4], pr[8 * g + 5]), pack_bf16(pr[8 * g + 6], pr[8 * g + 7]));
    }
    const float lsum = (ls4[0] + ls4[1]) + (ls4[2] + ls4[3]);
    // O of the previous chunks is complete (its MMA was waited on).  TMEM loads and stores are
    // warp-collective, so a warp rescales when any of its rows needs it (alpha = 1 elsewhere).
    if (c > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
      for (int cc = 0; cc < 128; cc += 32) {
        uint32_t v[32];
        tmem_ld32(tO + lane_base + cc, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
        tmem_st32(tO + lane_base + cc, v);
      }
      tmem_st_wait();
    }
    l_run = l_run * alpha + lsum;
    m_run = m_new;
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- O (+)= P V
    if (tid == 0) {
      tc_fence_after();
      const uint32_t idesc = idesc_bf16_f32(128, 128, false, true);
      // P: K-major like Q.  V read MN-major: 64-dimension blocks one region apart (leading
      // byte offset), 8-row groups 1024 bytes apart (stride byte offset); a K step of 16 rows
      // advances 2048 bytes.
      for (int kk = 0; kk < nc / 16; ++kk) {
        const uint32_t koff = (uint32_t)(kk >> 2) * kRegion + (uint32_t)(kk & 3) * 32;
        tc_mma_f16(tO, smem_desc_sw128(ps_a + koff, 16, 1024),
                   smem_desc_sw128(vs_a + (uint32_t)kk * 2048, kRegion, 1024), idesc, (c > 0 || kk > 0));
      }
      tc_commit(&bar_o);
    }
    const bool timed_out = !mbar_wait_bounded(&bar_o, c & 1);
    if (timed_out) flag(p.st, CSKV_DEV_TIMEOUT);
    alive = !__syncthreads_or(timed_out);  // block-uniform, so every thread leaves the loop together
    tc_fence_after();
  }
  if (p.cluster) {
    // ---- partial of this split (float4 groups of dimensions, sliced by merging CTA), then the
    //      merge.  Head tid's group j: slice r = tid / HPC (nh_r heads) at r HPC * 32 + j nh_r + hh.
    const size_t sb = (size_t)t * p.max_splits + split;
    if (c > 0) {
      const int hpc = 128 / p.cluster;
      const int r = tid / hpc, hh = tid % hpc;
      const int nh = min(hpc, H - r * hpc);
      const uint32_t tO = tmem_base + 128;
      float4* og = reinterpret_cast<float4*>(p.part_acc) + sb * 32 * H + (size_t)r * hpc * 32 + hh;
      for (int cc = 0; cc < 128; cc += 32) {
        uint32_t v[32];
        tmem_ld32(tO + lane_base + cc, v);
        tmem_ld_wait();
        if (tid < H) {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            og[(size_t)((cc >> 2) + i) * nh] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                                           __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
        }
      }
    }
    if (tid < H)
      reinterpret_cast<float2*>(p.part_ml)[sb * H + tid] = c > 0 ? make_float2(m_run, l_run) : make_float2(-INFINITY, 0.f);
    fence_proxy_async_global();  // the other CTAs' TMA reads these stores after the cluster barrier
    float4* stage = reinterpret_cast<float4*>(KVs);  // the dead K||V tile: 64 KiB
    switch (p.cluster) {
      case 1: cluster_merge<1>(p, t, stage, &bar_m); break;
      case 2: cluster_merge<2>(p, t, stage, &bar_m); break;
      case 4: cluster_merge<4>(p, t, stage, &bar_m); break;
      case 8: cluster_merge<8>(p, t, stage, &bar_m); break;
      default: cluster_merge<16>(p, t, stage, &bar_m); break;
    }
  } else if (c > 0) {
    // ---- partial of this split: O row (unnormalised, relative to m_run), m_run, l_run.
    //      Every lane takes part in the warp-collective TMEM loads; only real heads store.
    //      Partials are stored dimension-major ([split][j][h]), so a warp's stores are contiguous.
    const uint32_t tO = tmem_base + 128;
    const size_t sb = (size_t)t * p.max_splits + split;
    float* dst = p.part_acc + sb * kHeadDim * H + tid;
    for (int cc = 0; cc < 128; cc += 32) {
      uint32_t v[32];
      tmem_ld32(tO + lane_base + cc, v);
      tmem_ld_wait();
      if (tid < H) {
#pragma unroll
        for (int i = 0; i < 32; ++i) dst[(size_t)(cc + i) * H] = __uint_as_float(v[i]);
      }
    }
    if (tid < H) {
      p.part_ml[sb * 2 * H + tid] = m_run;
      p.part_ml[(sb * 2 + 1) * H + tid] = l_run;
    }
  }
  // the next kernel (the merge kernel, without a cluster) may launch now; it waits for this
  // grid to finish before it reads (launching it earlier would park its CTAs on SMs that
  // other kernels of the step need)
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 256);
  }
}

// Largest cluster size (a power of two, at most `want` and 16) at which one cluster of
// attn_tc_kernel CTAs fits on the current device, 0 if none; cached per device.
int attn_tc_cluster_fit(int want) {
  static std::mutex mu;
  static int fit[64][5];  // [device][log2 size]: 0 unknown, 1 fits, -1 does not
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (ensure_smem(attn_tc_kernel, kTcSmem) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lock(mu);
  int best = 0;
  for (int lg = 0; lg < 5 && (1 << lg) <= want; ++lg) {
    if (fit[dev][lg] == 0) {
      const int cs = 1 << lg;
      bool ok = true;
      if (cs > 8)
        ok = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
      int n = 0;
      if (ok) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(cs, 1);
        cfg.blockDim = dim3(kTcThreads);
        cfg.dynamicSmemBytes = kTcSmem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = cs;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        ok = cudaOccupancyMaxActiveClusters(&n, attn_tc_kernel, &cfg) == cudaSuccess && n > 0;
      }
      cudaGetLastError();  // a refused query leaves no sticky error
      fit[dev][lg] = ok ? 1 : -1;
    }
    if (fit[dev][lg] > 0) best = 1 << lg;
  }
  return best;
}

cudaError_t launch_attn_tc(const AttnParams& p, cudaStream_t stream) {
  auto kern = attn_tc_kernel;
  cudaError_t e = ensure_smem(kern, kTcSmem);
  if (e != cudaSuccess) return e;
  // a dependent launch: the CTAs may start (TMEM, barriers) while the previous kernel -- the
  // indexer, or the compression after it -- finishes, and wait for it before reading
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.max_splits, p.pairs ? (p.T + 1) / 2 : p.T);
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = kTcSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = p.cluster ? p.cluster : 1;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.cluster ? 2 : 1;
  e = cudaLaunchKernelEx(&cfg, kern, p);
  note_launch();
  if (e != cudaSuccess || p.cluster) return e;
  return launch_attn_combine(p, stream);
}

}  // namespace cskv
