// C ABI of the cskv library: host-side validation, then dispatch to the launchers.
// Every check here runs before any launch, so an error return means nothing ran.
#include <stdio.h>

#include "launch.cuh"

#include <algorithm>
#include <atomic>
#include <mutex>
#include <vector>

using namespace cskv;

static std::atomic<unsigned long long> g_launches{0};
void cskv::note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

cudaError_t cskv::ensure_smem_raw(const void* kern, size_t bytes) {
  struct Entry {
    const void* kern;
    int dev;
    size_t bytes;
  };
  static std::mutex mu;
  static std::vector<Entry> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (const Entry& x : done)
    if (x.kern == kern && x.dev == dev && x.bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  // Every kernel asks for the largest shared-memory carve-out: an SM runs CTAs of different
  // kernels side by side only under one carve-out, and the decode step relies on the indexer,
  // the attention and the compression CTAs sharing SMs.
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess) done.push_back(Entry{kern, dev, bytes});
  return e;
}

static thread_local char g_cuda_err[256] = "no error";

static int launch_status(cudaError_t e) {
  if (e == cudaSuccess) return CSKV_OK;
  snprintf(g_cuda_err, sizeof(g_cuda_err), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
  return CSKV_ERR_LAUNCH;
}

static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

static int device_sms(int* sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev);
  return launch_status(e);
}

extern "C" {

const char* cskv_status_string(int status) {
  switch (status) {
    case CSKV_OK: return "CSKV_OK";
    case CSKV_ERR_INVALID_ARG: return "CSKV_ERR_INVALID_ARG: null pointer, bad size, misaligned pointer or bad enum";
    case CSKV_ERR_UNSUPPORTED: return "CSKV_ERR_UNSUPPORTED: combination of dtype / head dim / heads not implemented";
    case CSKV_ERR_WORKSPACE: return "CSKV_ERR_WORKSPACE: workspace missing or too small";
    case CSKV_ERR_LAUNCH: return "CSKV_ERR_LAUNCH: the CUDA runtime refused a launch or query";
    default: return "unknown cskv status";
  }
}

const char* cskv_last_cuda_error(void) { return g_cuda_err; }

int cskv_version(void) { return 100; }

int cskv_copy_segments(const void* src, const int64_t* src_off, void* const* dst, const int64_t* len, int n,
                       cskv_stream_t stream) {
  if (n < 0 || n > (1 << 30) || (n > 0 && (!src || !src_off || !dst || !len))) return CSKV_ERR_INVALID_ARG;
  if (n == 0) return CSKV_OK;
  return launch_status(launch_copy_segments(src, src_off, dst, len, n, (cudaStream_t)stream));
}

int cskv_mapped_pointer(const void* p, void** out) {
  if (!out) return CSKV_ERR_INVALID_ARG;
  *out = nullptr;
  if (!p) return CSKV_ERR_INVALID_ARG;
  cudaPointerAttributes at;
  const cudaError_t e = cudaPointerGetAttributes(&at, p);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();  // a failed query leaves no error behind for the next launch
    return launch_status(e);
  }
  if (at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged) {
    *out = const_cast<void*>(p);
    return CSKV_OK;
  }
  // page-locked host memory: the address this device reads it at (none: not mapped here)
  if (at.type == cudaMemoryTypeHost && at.devicePointer) {
    *out = at.devicePointer;
    return CSKV_OK;
  }
  return CSKV_ERR_INVALID_ARG;  // pageable host memory: the device cannot address it
}

unsigned long long cskv_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

static int check_compress_common(const void* x, const void* z, const int64_t* tok_off, int batch,
                                 const int64_t* ent_off, int64_t max_blocks, int in_dtype, int out_dtype,
                                 const void* out) {
  if (!x || !z || !tok_off || !ent_off || !out) return CSKV_ERR_INVALID_ARG;
  if (batch < 1 || batch > 65535 || max_blocks < 0 || max_blocks > (1LL << 31) - 1) return CSKV_ERR_INVALID_ARG;
  if ((in_dtype != CSKV_F32 && in_dtype != CSKV_BF16) || (out_dtype != CSKV_F32 && out_dtype != CSKV_BF16))
    return in_dtype == CSKV_FP8E4M3 || out_dtype == CSKV_FP8E4M3 ? CSKV_ERR_UNSUPPORTED : CSKV_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(z) || !aligned16(out)) return CSKV_ERR_INVALID_ARG;
  return CSKV_OK;
}

// RMSNorm arguments shared by both compressions.
static int check_norm(int rmsnorm, const float* gamma, float eps) {
  if (rmsnorm != 0 && rmsnorm != 1) return CSKV_ERR_INVALID_ARG;
  if (rmsnorm && (!(eps >= 0.f) || !(eps < INFINITY))) return CSKV_ERR_INVALID_ARG;
  if (gamma && (reinterpret_cast<uintptr_t>(gamma) & 3u)) return CSKV_ERR_INVALID_ARG;
  return CSKV_OK;
}

int csa_compress(const void* x_a, const void* z_a, const void* x_b, const void* z_b, const float* bias_a,
                 const float* bias_b, const int64_t* tok_off, const int64_t* tok0, int batch,
                 const int64_t* ent_off, const int64_t* first_block, const int64_t* num_blocks,
                 int64_t max_blocks, int in_dtype, int out_dtype, void* out, int rmsnorm, const float* norm_gamma,
                 float norm_eps, const void* k_tok, int k_dtype, int Di, uint8_t* k_codes, float* k_scale,
                 int flags, int* dev_status, cskv_stream_t stream) {
  int rc = check_compress_common(x_a, z_a, tok_off, batch, ent_off, max_blocks, in_dtype, out_dtype, out);
  if (rc) return rc;
  if (flags & ~CSKV_OVERLAP_PREVIOUS) return CSKV_ERR_INVALID_ARG;
  if ((x_b == nullptr) != (z_b == nullptr)) return CSKV_ERR_INVALID_ARG;
  if (x_b && (!aligned16(x_b) || !aligned16(z_b))) return CSKV_ERR_INVALID_ARG;
  if ((bias_a && !aligned16(bias_a)) || (bias_b && !aligned16(bias_b))) return CSKV_ERR_INVALID_ARG;
  rc = check_norm(rmsnorm, norm_gamma, norm_eps);
  if (rc) return rc;
  if (k_tok) {
    if (!k_codes || !k_scale) return CSKV_ERR_INVALID_ARG;
    if (k_dtype != CSKV_F32 && k_dtype != CSKV_BF16)
      return k_dtype == CSKV_FP8E4M3 ? CSKV_ERR_UNSUPPORTED : CSKV_ERR_INVALID_ARG;
    if (Di != 64 && Di != 128) return Di > 0 ? CSKV_ERR_UNSUPPORTED : CSKV_ERR_INVALID_ARG;
    if (!aligned16(k_tok) || !aligned16(k_codes) || (reinterpret_cast<uintptr_t>(k_scale) & 3u))
      return CSKV_ERR_INVALID_ARG;
  }
  if (max_blocks == 0) return CSKV_OK;
  return launch_status(launch_csa_compress(x_a, z_a, x_b, z_b, bias_a, bias_b, tok_off, tok0, batch, ent_off,
                                           first_block, num_blocks, max_blocks, in_dtype, out_dtype, out, rmsnorm,
                                           norm_gamma, norm_eps, k_tok, k_dtype, k_tok ? Di : 0, k_codes, k_scale,
                                           flags, dev_status, (cudaStream_t)stream));
}

int lindex_pool_keys(const void* k_tok, int in_dtype, int Di, const int64_t* tok_off, const int64_t* tok0,
                     int batch, const int64_t* ent_off, const int64_t* first_block, const int64_t* num_blocks,
                     int64_t max_blocks, uint8_t* out_codes, float* out_scale, int* dev_status,
                     cskv_stream_t stream) {
  if (!k_tok || !tok_off || !ent_off || !out_codes || !out_scale) return CSKV_ERR_INVALID_ARG;
  if (batch < 1 || batch > 65535 || max_blocks < 0 || max_blocks > (1LL << 31) - 1) return CSKV_ERR_INVALID_ARG;
  if (in_dtype != CSKV_F32 && in_dtype != CSKV_BF16)
    return in_dtype == CSKV_FP8E4M3 ? CSKV_ERR_UNSUPPORTED : CSKV_ERR_INVALID_ARG;
  if (Di != 64 && Di != 128) return Di > 0 ? CSKV_ERR_UNSUPPORTED : CSKV_ERR_INVALID_ARG;
  if (!aligned16(k_tok) || !aligned16(out_codes) || (reinterpret_cast<uintptr_t>(out_scale) & 3u))
    return CSKV_ERR_INVALID_ARG;
  if (max_blocks == 0) return CSKV_OK;
  return launch_status(launch_pool_keys(k_tok, in_dtype, Di, tok_off, tok0, batch, ent_off, first_block,
                                        num_blocks, max_blocks, out_codes, out_scale, dev_status,
                                        (cudaStream_t)stream));
}

int hca_compress(const void* x, const void* z, const float* bias, const int64_t* tok_off, const int64_t* tok0,
                 int batch, const int64_t* ent_off, const int64_t* first_block, const int64_t* num_blocks,
                 int64_t max_blocks, int in_dtype, int out_dtype, void* out, int rmsnorm, const float* norm_gamma,
                 float norm_eps, int* dev_status, cskv_stream_t stream) {
  int rc = check_compress_common(x, z, tok_off, batch, ent_off, max_blocks, in_dtype, out_dtype, out);
  if (rc) return rc;
  if (bias && !aligned16(bias)) return CSKV_ERR_INVALID_ARG;
  rc = check_norm(rmsnorm, norm_gamma, norm_eps);
  if (rc) return rc;
  if (max_blocks == 0) return CSKV_OK;
  return launch_status(launch_hca_compress(x, z, bias, tok_off, tok0, batch, ent_off, first_block, num_blocks,
                                           max_blocks, in_dtype, out_dtype, out, rmsnorm, norm_gamma, norm_eps,
                                           dev_status, (cudaStream_t)stream));
}

int kv_quantize_fp8(const void* rows, int dtype, int64_t n, void* out, cskv_stream_t stream) {
  if (n < 0 || n > (int64_t)0x7FFFFFFF * 8) return CSKV_ERR_INVALID_ARG;  // grid.x: 8 rows a CTA
  if (dtype != CSKV_F32 && dtype != CSKV_BF16) return dtype == CSKV_FP8E4M3 ? CSKV_ERR_UNSUPPORTED : CSKV_ERR_INVALID_ARG;
  if (n == 0) return CSKV_OK;
  if (!rows || !out || !aligned16(rows) || !aligned16(out)) return CSKV_ERR_INVALID_ARG;
  return launch_status(cskv::launch_kv_quantize_fp8(rows, dtype, n, (uint8_t*)out, (cudaStream_t)stream));
}

int rmsnorm_heads(const void* x, int dtype, int64_t rows, int d, const float* gamma, float eps, void* out,
                  cskv_stream_t stream) {
  if (dtype != CSKV_F32 && dtype != CSKV_BF16) return dtype == CSKV_FP8E4M3 ? CSKV_ERR_UNSUPPORTED : CSKV_ERR_INVALID_ARG;
  if (d != kHeadDim) return d > 0 ? CSKV_ERR_UNSUPPORTED : CSKV_ERR_INVALID_ARG;
  if (rows < 0 || !(eps >= 0.f) || !(eps < INFINITY)) return CSKV_ERR_INVALID_ARG;
  if (rows == 0) return CSKV_OK;
  if (!x || !out || !aligned16(x) || !aligned16(out) || (gamma && (reinterpret_cast<uintptr_t>(gamma) & 3u)))
    return CSKV_ERR_INVALID_ARG;
  return launch_status(launch_rmsnorm_rows(x, dtype, rows, gamma, eps, out, (cudaStream_t)stream));
}

// Workspace of the tensor-core path (many queries): the candidate lists, then the workspace of
// the exact top-k over them.
static size_t tc_area(size_t b) { return (b + 255) / 256 * 256; }
static size_t lindex_tc_ws_bytes(int T, int k, int64_t max_entries) {
  const int64_t cap = lindex_tc_cap(k, max_entries);
  return tc_area((size_t)T * cap * sizeof(float)) + tc_area((size_t)T * cap * sizeof(int32_t)) +
         tc_area((size_t)T * sizeof(int64_t)) + lindex_ws_bytes(T, cap);
}

size_t lindex_workspace_size_scan(int T, int64_t max_entries) {
  if (T < 1) return 0;
  return lindex_ws_bytes(T, max_entries);
}

size_t lindex_workspace_size(int T, int k, int64_t max_entries) {
  if (T < 1) return 0;
  size_t b = lindex_ws_bytes(T, max_entries);
  if (T >= kLindexTcMinQueries && k >= 1) b = std::max(b, lindex_tc_ws_bytes(T, k, max_entries));
  return b;
}

static int check_topk_common(int T, int k, int64_t max_entries, const int32_t* out_idx, const void* ws,
                             size_t ws_bytes) {
  if (T < 0 || k < 1 || k > (1 << 24) || max_entries < 0 || max_entries >= (1LL << 31)) return CSKV_ERR_INVALID_ARG;
  if (T > 0 && !out_idx) return CSKV_ERR_INVALID_ARG;
  if (T > 0 && !lindex_capacity_ok(max_entries, T)) return CSKV_ERR_UNSUPPORTED;
  if (T > 0 && (!ws || ws_bytes < lindex_ws_bytes(T, max_entries) || !aligned16(ws))) return CSKV_ERR_WORKSPACE;
  return CSKV_OK;
}

int lindex_score_topk(const void* q_idx, const float* q_scale, const void* k_idx, const float* k_scale,
                      const float* head_w, const int32_t* q_seq, const int64_t* q_pos, const int64_t* ent_off,
                      int batch, int T, int Hi, int Di, int k, int dtype, int64_t max_entries, int32_t* out_idx,
                      float* out_score, const void* prefetch_rows, int64_t prefetch_row_bytes, void* workspace,
                      size_t ws_bytes, int* dev_status, cskv_stream_t stream) {
  if (dtype != CSKV_F32 && dtype != CSKV_FP8E4M3 && dtype != CSKV_BF16) return CSKV_ERR_INVALID_ARG;
  if (!lindex_shape_supported(dtype, Hi, Di)) return CSKV_ERR_UNSUPPORTED;
  if (T > 0 && (!q_idx || !k_idx || !q_seq || !q_pos || !ent_off || batch < 1)) return CSKV_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(k_idx)) return CSKV_ERR_INVALID_ARG;
  if (prefetch_rows && (!aligned16(prefetch_rows) || prefetch_row_bytes <= 0 || prefetch_row_bytes % 16 != 0 ||
                        prefetch_row_bytes > (1 << 20)))
    return CSKV_ERR_INVALID_ARG;
  int rc = check_topk_common(T, k, max_entries, out_idx, workspace, ws_bytes);
  if (rc || T == 0) return rc;
  IdxParams p = {};
  p.q_idx = (const uint8_t*)q_idx;
  p.q_scale = q_scale;
  p.k_idx = (const uint8_t*)k_idx;
  p.k_scale = k_scale;
  p.head_w = head_w;
  p.q_seq = q_seq;
  p.q_pos = q_pos;
  p.ent_off = ent_off;
  p.batch = batch;
  p.Hi = Hi;
  p.Di = Di;
  p.k = k;
  p.max_entries = max_entries;
  p.out_idx = out_idx;
  p.out_score = out_score;
  p.pf_rows = prefetch_rows ? (const uint8_t*)prefetch_rows : nullptr;
  p.pf_row_bytes = prefetch_rows ? prefetch_row_bytes : 0;
  p.ws = (QueryWS*)workspace;
  p.st = dev_status;
  if (T >= kLindexTcMinQueries && lindex_tc_shape(dtype, Hi, Di) && ws_bytes >= lindex_tc_ws_bytes(T, k, max_entries)) {
    // many queries: tensor-core scores -> candidate lists -> exact top-k over the lists ->
    // candidate positions mapped back to entry indices
    const int64_t cap = lindex_tc_cap(k, max_entries);
    uint8_t* w = (uint8_t*)workspace;
    float* cand_score = (float*)w;
    w += tc_area((size_t)T * cap * sizeof(float));
    int32_t* cand_idx = (int32_t*)w;
    w += tc_area((size_t)T * cap * sizeof(int32_t));
    int64_t* cand_n = (int64_t*)w;
    w += tc_area((size_t)T * sizeof(int64_t));
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = launch_lindex_tc_candidates(p.q_idx, q_scale, p.k_idx, k_scale, head_w, q_seq, q_pos, ent_off,
                                                batch, T, Hi, Di, k, cap, cand_score, cand_idx, cand_n, dev_status, s);
    if (e != cudaSuccess) return launch_status(e);
    IdxParams ps = {};
    ps.scores = cand_score;
    ps.ld_scores = cap;
    ps.n_valid = cand_n;
    ps.Hi = 1;
    ps.Di = 64;
    ps.k = k;
    ps.max_entries = cap;
    ps.out_idx = out_idx;
    ps.out_score = out_score;
    ps.ws = (QueryWS*)w;
    ps.st = dev_status;
    e = launch_lindex(ps, CSKV_F32, T, s);
    if (e != cudaSuccess) return launch_status(e);
    return launch_status(launch_map_candidates(out_idx, cand_idx, cap, T, k, ent_off, q_seq, p.pf_rows,
                                               p.pf_row_bytes, s));
  }
  return launch_status(launch_lindex(p, dtype, T, (cudaStream_t)stream));
}

int lindex_score_topk_mxfp4(const uint8_t* q_codes, const uint8_t* q_bscale, const float* q_scale,
                            const uint8_t* k_codes, const uint8_t* k_bscale, const float* head_w,
                            const int32_t* q_seq, const int64_t* q_pos, const int64_t* ent_off, int batch, int T,
                            int Hi, int Di, int k, int64_t max_entries, int32_t* out_idx, float* out_score,
                            const void* prefetch_rows, int64_t prefetch_row_bytes, void* workspace, size_t ws_bytes,
                            int* dev_status, cskv_stream_t stream) {
  if (Hi < 1 || Hi > 16 || (Di != 64 && Di != 128)) return Hi >= 1 && Di > 0 ? CSKV_ERR_UNSUPPORTED : CSKV_ERR_INVALID_ARG;
  if (T > 0 && (!q_codes || !q_bscale || !k_codes || !k_bscale || !q_seq || !q_pos || !ent_off || batch < 1))
    return CSKV_ERR_INVALID_ARG;
  // codes are read in 16-byte tiles and 4-byte words; a key's Di/32 scale bytes as one 2- or
  // 4-byte word
  if (!aligned16(q_codes) || !aligned16(k_codes) || (reinterpret_cast<uintptr_t>(k_bscale) % (Di / 32)))
    return CSKV_ERR_INVALID_ARG;
  if (prefetch_rows && (!aligned16(prefetch_rows) || prefetch_row_bytes <= 0 || prefetch_row_bytes % 16 != 0 ||
                        prefetch_row_bytes > (1 << 20)))
    return CSKV_ERR_INVALID_ARG;
  int rc = check_topk_common(T, k, max_entries, out_idx, workspace, ws_bytes);
  if (rc || T == 0) return rc;
  IdxParams p = {};
  p.q_idx = q_codes;
  p.q_scale = q_scale;
  p.k_idx = k_codes;
  p.q_bs = q_bscale;
  p.k_bs = k_bscale;
  p.head_w = head_w;
  p.q_seq = q_seq;
  p.q_pos = q_pos;
  p.ent_off = ent_off;
  p.batch = batch;
  p.Hi = Hi;
  p.Di = Di;
  p.k = k;
  p.max_entries = max_entries;
  p.out_idx = out_idx;
  p.out_score = out_score;
  p.pf_rows = prefetch_rows ? (const uint8_t*)prefetch_rows : nullptr;
  p.pf_row_bytes = prefetch_rows ? prefetch_row_bytes : 0;
  p.ws = (QueryWS*)workspace;
  p.st = dev_status;
  return launch_status(launch_lindex(p, CSKV_FP8E4M3, T, (cudaStream_t)stream));
}

int lindex_topk_from_scores(const float* scores, int64_t ld_scores, const int64_t* n_valid, int T, int k,
                            int64_t max_entries, int32_t* out_idx, float* out_score, void* workspace,
                            size_t ws_bytes, int* dev_status, cskv_stream_t stream) {
  if (T > 0 && (!scores || !n_valid)) return CSKV_ERR_INVALID_ARG;
  if (ld_scores < max_entries || ld_scores < 0) return CSKV_ERR_INVALID_ARG;
  int rc = check_topk_common(T, k, max_entries, out_idx, workspace, ws_bytes);
  if (rc || T == 0) return rc;
  IdxParams p = {};
  p.scores = scores;
  p.ld_scores = ld_scores;
  p.n_valid = n_valid;
  p.Hi = 1;
  p.Di = 64;
  p.k = k;
  p.max_entries = max_entries;
  p.out_idx = out_idx;
  p.out_score = out_score;
  p.ws = (QueryWS*)workspace;
  p.st = dev_status;
  return launch_status(launch_lindex(p, CSKV_F32, T, (cudaStream_t)stream));
}

// Split plan of hybrid_decode_attn for the tensor-core kernel (bf16) or the CUDA-core kernel
// (fp32): rows per split R and split count S; ws_splits = the split count the workspace of
// partials is sized for (the larger of the two plans below).  A tensor-core plan of at most
// kClusterMaxSplits splits instead merges inside a thread-block cluster (cluster = S, a power
// of two <= 16, rows spread evenly over it) when such a cluster fits on the device.
constexpr int kClusterMaxSplits = 18;
struct AttnPlan {
  int R, S, ws_splits, cluster;
};
static int attn_plan(int mode, int T, int k, int window, int64_t max_entries, bool tc, AttnPlan* pl) {
  int sms = 0;
  int rc = device_sms(&sms);
  if (rc) return rc;
  pl->R = tc ? attn_tc_rows_per_split(mode, T, k, window, max_entries, sms)
             : attn_rows_per_split(mode, T, k, window, max_entries, sms);
  pl->S = attn_max_splits(mode, k, window, max_entries, pl->R);
  pl->ws_splits = pl->S;
  pl->cluster = 0;
  if (tc && pl->S <= kClusterMaxSplits) {
    int want = 1;
    while (want < pl->S && want < 16) want <<= 1;
    if (attn_tc_cluster_fit(want) == want) {
      const int64_t rows_max = (mode == CSKV_CSA ? (int64_t)k : max_entries) + window;
      pl->R = (int)std::max<int64_t>(1, (rows_max + want - 1) / want);
      pl->S = want;
      pl->cluster = want;
      pl->ws_splits = std::max(pl->ws_splits, want);
    }
  }
  return CSKV_OK;
}

// Adjacent-query pairs (CSKV_ATTN_PAIRS) for the tensor-core HCA kernel: H == 64 heads, so a
// pair's two queries fill the 128 rows of the tile.
constexpr int kPairHeads = 64;

size_t hybrid_attn_workspace_size(int mode, int T, int H, int d, int k, int window, int64_t max_entries) {
  mode &= ~(CSKV_ATTN_PAIRS | CSKV_ATTN_KV_FP8);
  if (T < 1 || H < 1 || d != kHeadDim || window < 0) return 0;
  size_t best = 0;
  for (int tc = 0; tc < 2; ++tc) {
    AttnPlan pl;
    if (attn_plan(mode, T, k, window, max_entries, tc != 0, &pl)) return 0;
    const size_t need = (size_t)T * pl.ws_splits * H * (kHeadDim + 2) * sizeof(float);
    if (need > best) best = need;
  }
  if (mode == CSKV_HCA && H == kPairHeads && T >= 2) {  // the pair plan: (T + 1) / 2 units of 2H heads
    AttnPlan pl;
    const int Tp = (T + 1) / 2;
    if (attn_plan(mode, Tp, 0, window + 1, max_entries, true, &pl)) return 0;
    const size_t need = (size_t)Tp * pl.ws_splits * 2 * H * (kHeadDim + 2) * sizeof(float);
    if (need > best) best = need;
  }
  return best;
}

}  // extern "C"

// Host-side checks of hybrid_decode_attn's arguments (everything but the workspace), shared
// with the allocation-free variant so that both report the same error for the same mistake.
int cskv::check_attn_args(int mode, const void* q, const void* kv_cmp, const int64_t* cmp_off, const int32_t* idx,
                          int k, const void* kv_raw, const int64_t* raw_off, int window, float scale,
                          const int32_t* q_seq, const int64_t* q_pos, int batch, int T, int H, int d, int dtype,
                          int64_t max_entries, const float* out) {
  constexpr int kFlags = CSKV_ATTN_PAIRS | CSKV_ATTN_KV_FP8;
  if ((mode & ~kFlags) != CSKV_CSA && (mode & ~kFlags) != CSKV_HCA) return CSKV_ERR_INVALID_ARG;
  mode &= ~kFlags;
  if (dtype != CSKV_F32 && dtype != CSKV_BF16) return dtype == CSKV_FP8E4M3 ? CSKV_ERR_UNSUPPORTED : CSKV_ERR_INVALID_ARG;
  if (d != kHeadDim) return CSKV_ERR_UNSUPPORTED;
  if (H < 1 || H > 128 || T < 0 || window < 0 || window > (1 << 20) || batch < 1) return CSKV_ERR_INVALID_ARG;
  if (mode == CSKV_CSA && (k < 1 || k > (1 << 20) || !idx)) return CSKV_ERR_INVALID_ARG;
  if (mode == CSKV_HCA && (max_entries < 0 || max_entries > (1LL << 30))) return CSKV_ERR_INVALID_ARG;
  // the softmax scale must be positive and finite: the kernels take the row maximum of the
  // unscaled logits and scale it once, which is the maximum of the scaled logits only then
  if (!(scale > 0.f) || !(scale < INFINITY)) return CSKV_ERR_INVALID_ARG;
  if (T == 0) return CSKV_OK;
  if (!q || !kv_cmp || !cmp_off || !kv_raw || !raw_off || !q_seq || !q_pos || !out) return CSKV_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kv_cmp) || !aligned16(kv_raw)) return CSKV_ERR_INVALID_ARG;
  return CSKV_OK;
}

extern "C" {

int hybrid_decode_attn(int mode, const void* q, const void* kv_cmp, const int64_t* cmp_off, const int32_t* idx,
                       int k, const void* kv_raw, const int64_t* raw_off, const int64_t* raw_tok0, int window,
                       const float* sink, float scale, const int32_t* q_seq, const int64_t* q_pos, int batch,
                       int T, int H, int d, int dtype, int64_t max_entries, float* out, float* lse,
                       void* workspace, size_t ws_bytes, int* dev_status, cskv_stream_t stream) {
  int arc = check_attn_args(mode, q, kv_cmp, cmp_off, idx, k, kv_raw, raw_off, window, scale, q_seq, q_pos, batch,
                            T, H, d, dtype, max_entries, out);
  if (arc != CSKV_OK || T == 0) return arc;
  const bool want_pairs = (mode & CSKV_ATTN_PAIRS) != 0;
  const bool kv8 = (mode & CSKV_ATTN_KV_FP8) != 0;  // FP8 main-KV rows, decoded as gathered
  mode &= ~(CSKV_ATTN_PAIRS | CSKV_ATTN_KV_FP8);
  const bool tc = dtype == CSKV_BF16;
  AttnPlan pl;
  int rc = attn_plan(mode, T, mode == CSKV_CSA ? k : 0, window, max_entries, tc, &pl);
  if (rc) return rc;
  // adjacent-query pairs: the HCA tensor-core kernel with 64 heads, when the pairs' plan merges
  // inside a cluster (a unit of two queries is one 128-head "query" of the plan)
  int units = T, Hv = H;
  if (want_pairs && tc && mode == CSKV_HCA && H == kPairHeads && T >= 2) {
    AttnPlan pp;
    rc = attn_plan(mode, (T + 1) / 2, 0, window + 1, max_entries, tc, &pp);
    if (rc) return rc;
    if (pp.cluster) {
      pl = pp;
      units = (T + 1) / 2;
      Hv = 2 * H;
    }
  }
  const size_t need = (size_t)units * pl.ws_splits * Hv * (kHeadDim + 2) * sizeof(float);
  if (!workspace || ws_bytes < need || !aligned16(workspace)) return CSKV_ERR_WORKSPACE;
  AttnParams p = {};
  p.mode = mode;
  p.q = q;
  p.kv_cmp = kv_cmp;
  p.cmp_off = cmp_off;
  p.idx = idx;
  p.k = mode == CSKV_CSA ? k : 0;
  p.kv_raw = kv_raw;
  p.raw_off = raw_off;
  p.raw_tok0 = raw_tok0;
  p.window = window;
  p.sink = sink;
  p.scale_log2 = scale * kLog2e;
  p.q_seq = q_seq;
  p.q_pos = q_pos;
  p.batch = batch;
  p.T = T;
  p.H = H;
  p.rows_per_split = pl.R;
  p.max_splits = pl.S;
  p.cluster = pl.cluster;
  p.pairs = Hv != H ? 1 : 0;
  p.Hv = Hv;
  p.kv8 = kv8 ? 1 : 0;
  p.part_acc = (float*)workspace;
  p.part_ml = p.part_acc + (size_t)units * pl.S * Hv * kHeadDim;
  p.out = out;
  p.lse = lse;
  p.st = dev_status;
  if (tc) return launch_status(launch_attn_tc(p, (cudaStream_t)stream));
  return launch_status(launch_attn_generic(p, dtype, (cudaStream_t)stream));
}

}  // extern "C"
