// Parameter blocks and host launchers shared by the kernel files and the C ABI.
#pragma once

#include "common.cuh"

namespace cskv {

struct QueryWS;

// Host-side count of kernels this library has launched (api.cu).
void note_launch();

// Raises a kernel's dynamic shared-memory limit and asks for the largest shared-memory
// carve-out, once per (kernel, device): cudaFuncSetAttribute is a host round trip that
// repeated launches skip (api.cu).  Every kernel calls it before its first launch.
cudaError_t ensure_smem_raw(const void* kern, size_t bytes);
template <typename K>
cudaError_t ensure_smem(K kern, size_t bytes) {
  return ensure_smem_raw(reinterpret_cast<const void*>(kern), bytes);
}

// kern<<<grid, block, smem, stream>>>(args...) as a programmatic dependent launch: the grid
// may be scheduled while the previous kernel on the stream runs; the kernel itself waits
// (pdl_wait) before reading inputs, so stream order is unchanged.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                             Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// compress.cu (a few entries: decode shapes) and compress_bulk.cu (many: TMA rings)
constexpr int64_t kCsaBulkMinEntries = 512;  // at or above: the TMA-ring CSA kernel
constexpr int64_t kHcaBulkMinEntries = 128;  // at or above: the TMA-ring HCA kernel
cudaError_t launch_csa_compress(const void* xa, const void* za, const void* xb, const void* zb,
                                const float* ba, const float* bb, const int64_t* tok_off,
                                const int64_t* tok0, int batch, const int64_t* ent_off,
                                const int64_t* first, const int64_t* num, int64_t max_blocks,
                                int in_dt, int out_dt, void* out, int norm, const float* gamma, float eps,
                                const void* k_tok, int k_dt, int Di, uint8_t* k_codes, float* k_scale, int flags,
                                int* st, cudaStream_t stream);
cudaError_t launch_hca_compress(const void* x, const void* z, const float* bias, const int64_t* tok_off,
                                const int64_t* tok0, int batch, const int64_t* ent_off,
                                const int64_t* first, const int64_t* num, int64_t max_blocks,
                                int in_dt, int out_dt, void* out, int norm, const float* gamma, float eps, int* st,
                                cudaStream_t stream);
cudaError_t launch_csa_bulk(const void* xa, const void* za, const void* xb, const void* zb, const float* ba,
                            const float* bb, const int64_t* tok_off, const int64_t* tok0, int batch,
                            const int64_t* ent_off, const int64_t* first, const int64_t* num, int64_t max_blocks,
                            int in_dt, int out_dt, void* out, const float* gamma, float eps, int norm,
                            const void* k_tok, int k_dt, int Di, uint8_t* k_codes, float* k_scale, int* st,
                            cudaStream_t stream);
cudaError_t launch_hca_bulk(const void* x, const void* z, const float* bias, const int64_t* tok_off,
                            const int64_t* tok0, int batch, const int64_t* ent_off, const int64_t* first,
                            const int64_t* num, int64_t max_blocks, int in_dt, int out_dt, void* out,
                            const float* gamma, float eps, int norm, int* st, cudaStream_t stream);
cudaError_t launch_rmsnorm_rows(const void* x, int dtype, int64_t rows, const float* gamma, float eps, void* out,
                                cudaStream_t stream);
cudaError_t launch_pool_keys(const void* k_tok, int in_dt, int Di, const int64_t* tok_off, const int64_t* tok0,
                             int batch, const int64_t* ent_off, const int64_t* first, const int64_t* num,
                             int64_t max_blocks, uint8_t* codes, float* scales, int* st, cudaStream_t stream);

// indexer.cu
struct IdxParams {
  const uint8_t* q_idx;
  const float* q_scale;
  const uint8_t* k_idx;
  const float* k_scale;
  const uint8_t* q_bs;  // MXFP4: E8M0 block scales of the queries [T, Hi, Di/32] and keys [Nc, Di/32]
  const uint8_t* k_bs;
  const float* head_w;
  const float* scores;
  int64_t ld_scores;
  const int64_t* n_valid;
  const int32_t* q_seq;
  const int64_t* q_pos;
  const int64_t* ent_off;
  int batch;
  int t_begin, T;
  int Hi, Di, k;
  int64_t max_entries;
  int64_t seg_cap;
  int split;
  int stages;        // TMA ring stages of the fp8 scan
  int64_t un_bytes;  // shared bytes of the ring / selection region (the scores follow it)
  int32_t* out_idx;
  float* out_score;
  const uint8_t* pf_rows;  // optional: rows (indexed like k_idx) of kept entries go to L2
  int64_t pf_row_bytes;
  QueryWS* ws;
  int* st;
};
cudaError_t launch_lindex(const IdxParams& p, int dtype, int T, cudaStream_t stream);
size_t lindex_ws_bytes(int T, int64_t max_entries);
bool lindex_shape_supported(int dtype, int Hi, int Di);
bool lindex_capacity_ok(int64_t max_entries, int T);
// indexer_tc.cu: many queries (a prefill chunk) on the tensor cores -> per-query candidate lists
constexpr int kLindexTcMinQueries = 256;
bool lindex_tc_shape(int dtype, int Hi, int Di);
int64_t lindex_tc_cap(int k, int64_t max_entries);
cudaError_t launch_lindex_tc_candidates(const uint8_t* q_idx, const float* q_scale, const uint8_t* k_idx,
                                        const float* k_scale, const float* head_w, const int32_t* q_seq,
                                        const int64_t* q_pos, const int64_t* ent_off, int batch, int T, int Hi,
                                        int Di, int k, int64_t cap, float* cand_score, int32_t* cand_idx,
                                        int64_t* cand_n, int* st, cudaStream_t stream);
cudaError_t launch_map_candidates(int32_t* out_idx, const int32_t* cand_idx, int64_t cap, int T, int k,
                                  const int64_t* ent_off, const int32_t* q_seq, const uint8_t* pf_rows,
                                  int64_t pf_row_bytes, cudaStream_t stream);

// attention.cu
struct AttnParams {
  int mode;
  const void* q;
  const void* kv_cmp;
  const int64_t* cmp_off;
  const int32_t* idx;
  int k;
  const void* kv_raw;
  const int64_t* raw_off;
  const int64_t* raw_tok0;
  int window;
  const float* sink;
  float scale_log2;
  const int32_t* q_seq;
  const int64_t* q_pos;
  int batch, T, H;
  int rows_per_split;
  int max_splits;
  int cluster;  // tensor-core kernel: the splits of a query form a cluster of this size (0: merge kernel)
  int pairs;    // tensor-core HCA kernel: CTA row y takes queries 2y, 2y + 1 (adjacent positions)
  int Hv;       // heads of a unit of work: H, or 2H for a pair (its rows 0..H-1, then H..2H-1)
  int kv8;      // CUDA-core kernel: kv_cmp rows are FP8 main-KV rows (kv8.cuh), kv_raw rows plain
  float* part_acc;
  float* part_ml;
  float* out;
  float* lse;
  int* st;
};
cudaError_t launch_attn_generic(const AttnParams& p, int dtype, cudaStream_t stream);
cudaError_t launch_attn_tc(const AttnParams& p, cudaStream_t stream);
int attn_tc_rows_per_split(int mode, int T, int k, int window, int64_t max_entries, int sms);
int attn_tc_cluster_fit(int want);
cudaError_t launch_attn_combine(const AttnParams& p, cudaStream_t stream);
int attn_rows_per_split(int mode, int T, int k, int window, int64_t max_entries, int sms);
int attn_max_splits(int mode, int k, int window, int64_t max_entries, int R);
// api.cu: host-side argument checks of hybrid_decode_attn (all but the workspace)
int check_attn_args(int mode, const void* q, const void* kv_cmp, const int64_t* cmp_off, const int32_t* idx, int k,
                    const void* kv_raw, const int64_t* raw_off, int window, float scale, const int32_t* q_seq,
                    const int64_t* q_pos, int batch, int T, int H, int d, int dtype, int64_t max_entries,
                    const float* out);
// kv8.cu
cudaError_t launch_kv_quantize_fp8(const void* rows, int dtype, int64_t n, uint8_t* out, cudaStream_t stream);
// staging.cu
cudaError_t launch_copy_segments(const void* src, const int64_t* src_off, void* const* dst, const int64_t* len, int n,
                                 cudaStream_t stream);
}  // namespace cskv
