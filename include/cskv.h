/*
 * cskv -- hybrid compressed sparse KV attention (DeepSeek V4 CSA / HCA) for
 * NVIDIA B200 (sm_100a).  C ABI.
 *
 * Source pages of the method (cited by page and section):
 *   [SW] shareware.cn/news/167317 -- essay on DeepSeek V4 Hybrid Attention.
 *   [TR] trdm.cn/news/516303 -- "从 MLA 到 CSA，聊聊大模型 Attention 的瘦身与闪送".
 *   [AM] aimodeling.com news "DeepSeek V4 混合注意力架构解析：如何在1M上下文下
 *        将计算量降至原来的27%？".
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every pointer argument is a DEVICE pointer unless its comment says host.
 *   The caller owns all memory; the library allocates nothing.
 * - Every call is asynchronous on `stream` (NULL = the legacy default stream)
 *   and may be captured into a CUDA graph.
 * - A KV row is packed K||V: D = 2*d values, K in columns 0..d-1, V in d..2d-1.
 *   d (head dim) must be 128.  Rows are contiguous, row-major.
 * - Sequences are concatenated; int64 CSR offsets give each sequence's rows:
 *   rows of sequence b are [off[b], off[b+1]).
 * - Return value: CSKV_OK, or an error code.  Arguments are validated on the
 *   host before anything is launched, so an error return means nothing ran.
 *   CSKV_ERR_LAUNCH carries a CUDA error; cskv_last_cuda_error() names it.
 * - `dev_status` (optional, may be NULL): device int that kernels OR the
 *   CSKV_DEV_* bits into when a device-side check fails (an index out of
 *   range, a row the caller did not provide, a bounded wait that gave up).
 *   The offending element is skipped; the call still completes.  The caller
 *   zeroes it and reads it back when it wants to know.
 * - Alignment: every row array must start on a 16-byte boundary.
 */
#ifndef CSKV_H
#define CSKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* cskv_stream_t; /* same type as cudaStream_t */

#if defined(__GNUC__)
#define CSKV_API __attribute__((visibility("default")))
#else
#define CSKV_API
#endif

enum cskv_status {
  CSKV_OK = 0,
  CSKV_ERR_INVALID_ARG = 1, /* null pointer, bad size, misaligned pointer, bad enum */
  CSKV_ERR_UNSUPPORTED = 2, /* valid but not implemented combination (dtype, d, Di, Hi) */
  CSKV_ERR_WORKSPACE = 3,   /* workspace missing or smaller than the *_workspace_size() figure */
  CSKV_ERR_LAUNCH = 4,      /* the CUDA runtime refused a launch or a device query */
};

enum cskv_dtype { CSKV_F32 = 0, CSKV_BF16 = 1, CSKV_FP8E4M3 = 2 };
enum cskv_mode { CSKV_CSA = 0, CSKV_HCA = 1 };
/* OR-ed into hybrid_decode_attn's mode (see there): queries 2j and 2j + 1 are adjacent. */
#define CSKV_ATTN_PAIRS 0x100
#define CSKV_ATTN_KV_FP8 0x200  /* hybrid_decode_attn: kv_cmp rows are FP8 main-KV rows */
#define CSKV_KV8_ROW_BYTES 336  /* bytes of one FP8 main-KV row (kv_quantize_fp8) */

/* Bits OR-ed into *dev_status by device-side checks. */
enum cskv_dev_status {
  CSKV_DEV_BAD_INDEX = 1,    /* an index or offset pointed outside its array; element skipped */
  CSKV_DEV_TAIL_MISSING = 2, /* a token row needed lies before the provided tail; element skipped */
  CSKV_DEV_CAPACITY = 4,     /* a size exceeded the host-side bound given to the call */
  CSKV_DEV_TIMEOUT = 8,      /* a bounded cross-block wait gave up; outputs of that call are invalid */
};

CSKV_API const char* cskv_status_string(int status);
CSKV_API const char* cskv_last_cuda_error(void); /* text of the CUDA error behind the last CSKV_ERR_LAUNCH */
CSKV_API int cskv_version(void);
/* Number of kernels this library has launched in this process (host-side count;
 * a captured CUDA graph replays its kernels without adding to it). */
CSKV_API unsigned long long cskv_launch_count(void);

/* ------------------------------------------------------------------------
 * csa_compress -- CSA token-dimension compression, 4 tokens -> 1 entry.
 *
 * [SW] §二/§四/§五, [TR] §4.3 改进一/改进二: entry i of a sequence mixes, for
 * every dimension j separately, the tokens of block i through path A
 * (value x_a[t,j], logit z_a[t,j] + bias_a[t-4i, j]) and the tokens of block
 * i-1 through path B (value x_b[t,j], logit z_b[t,j] + bias_b[t-4(i-1), j]):
 *     w = softmax over the candidates of the logits;  out[i,j] = sum w * value.
 * Entry 0 has no path-B candidates; a partial last block uses the tokens it has.
 *
 * x_a, z_a, x_b, z_b : [rows, 256] in_dtype (CSKV_F32 or CSKV_BF16).  x_b and
 *                      z_b may both be NULL: path A alone.
 * bias_a, bias_b     : [4, 256] fp32, or NULL for zero biases.
 * tok_off            : [batch+1] int64, rows of sequence b are tok_off[b]..tok_off[b+1]-1.
 * tok0               : [batch] int64 or NULL (all 0): the token position of
 *                      sequence b's first provided row.  Its length is
 *                      n_b = tok0[b] + tok_off[b+1] - tok_off[b]; only the tail
 *                      from tok0[b] need be provided.
 * ent_off            : [batch+1] int64, entry i of sequence b is written to row
 *                      ent_off[b] + i of `out` (needs ceil(n_b/4) rows).
 * first_block, num_blocks : [batch] int64 or NULL: entries first..first+num-1
 *                      are computed (NULL: first 0, num ceil(n_b/4) - first).
 * max_blocks         : host, >= every num_blocks[b]; entries beyond it are
 *                      skipped and flagged CSKV_DEV_CAPACITY.
 * out                : [*, 256] out_dtype (CSKV_F32 or CSKV_BF16; bf16 rounds to
 *                      nearest even).  fp32 arithmetic inside.
 * rmsnorm, norm_gamma, norm_eps : [SW] §十四.3 (queries and KV are RMS-normalised
 *                      so that attention logits cannot blow up).  rmsnorm = 1
 *                      normalises every entry written, on its fp32 value before
 *                      the output rounding, over its K half and over its V half
 *                      separately: y = x / sqrt(mean(x^2) + norm_eps) * gamma, with
 *                      norm_gamma [256] fp32 (K gains then V gains; NULL = ones,
 *                      4-byte aligned) and norm_eps >= 0 finite.  rmsnorm = 0: no
 *                      normalisation (norm_gamma / norm_eps unused).
 * k_tok, k_dtype, Di, k_codes, k_scale : optional (k_tok NULL = off): also pool the
 *                      indexer's per-token keys of the same entries, exactly as
 *                      lindex_pool_keys does ([TR] §4.2): k_tok [rows, Di] k_dtype
 *                      (CSKV_F32 / CSKV_BF16; rows indexed like x_a, 16-byte
 *                      aligned), Di 64 or 128; entry i of sequence b writes
 *                      k_codes[ent_off[b] + i, :] (E4M3, 16-byte aligned) and
 *                      k_scale[ent_off[b] + i] (fp32).
 * flags              : 0, or CSKV_OVERLAP_PREVIOUS: the caller guarantees that the
 *                      kernel issued just before this call on `stream` neither
 *                      writes any of its inputs nor reads its outputs, and that
 *                      every kernel before that one has completed by the time that
 *                      one starts its dependents (true right after lindex_score_topk,
 *                      which starts them only after its own wait).  The entries are
 *                      then computed while that kernel still runs (in a decode
 *                      step: beside the indexer), and this call still completes
 *                      after it, so a later kernel that waits for this call sees
 *                      both.  A permission, not a request: the many-entry kernel
 *                      ignores it.  Other bits: CSKV_ERR_INVALID_ARG.
 * Many entries (max_blocks >= 512) run a TMA-ring kernel, one CTA per SM; a few
 * (a decode step) run a warp per entry.  Both give the same results up to fp32
 * rounding order.
 * ------------------------------------------------------------------------ */
#define CSKV_OVERLAP_PREVIOUS 1
CSKV_API int csa_compress(const void* x_a, const void* z_a, const void* x_b, const void* z_b,
                 const float* bias_a, const float* bias_b,
                 const int64_t* tok_off, const int64_t* tok0, int batch,
                 const int64_t* ent_off, const int64_t* first_block, const int64_t* num_blocks,
                 int64_t max_blocks, int in_dtype, int out_dtype, void* out,
                 int rmsnorm, const float* norm_gamma, float norm_eps,
                 const void* k_tok, int k_dtype, int Di, uint8_t* k_codes, float* k_scale,
                 int flags, int* dev_status, cskv_stream_t stream);

/* ------------------------------------------------------------------------
 * hca_compress -- HCA compression, 128 tokens -> 1 entry, one stream.
 *
 * [SW] §三.3, [TR] §4.3 (HCA, no dual stream): entry i mixes the tokens of
 * block i (value x[t,j], logit z[t,j] + bias[t-128i, j]) with one softmax per
 * dimension.  Arguments as csa_compress (no key pooling); bias is [128, 256]
 * fp32 or NULL.  Many entries (max_blocks >= 128) or rmsnorm = 1 run a TMA-ring
 * kernel with one CTA per entry at a time; a few run sixteen small CTAs per entry.
 * ------------------------------------------------------------------------ */
CSKV_API int hca_compress(const void* x, const void* z, const float* bias,
                 const int64_t* tok_off, const int64_t* tok0, int batch,
                 const int64_t* ent_off, const int64_t* first_block, const int64_t* num_blocks,
                 int64_t max_blocks, int in_dtype, int out_dtype, void* out,
                 int rmsnorm, const float* norm_gamma, float norm_eps,
                 int* dev_status, cskv_stream_t stream);

/* ------------------------------------------------------------------------
 * kv_quantize_fp8 -- FP8 main-KV rows from K||V rows.
 *
 * [SW] shareware.cn/news/167317 §十三.4: the main KV may be stored in FP8 while the
 * dimensions most sensitive to position information keep a higher precision.  A
 * compressed row (K dims 0..127 then V dims 0..127) becomes CSKV_KV8_ROW_BYTES (336)
 * bytes: K dims 0..63 as OCP E4M3 codes (64 B) | K dims 64..127, the RoPE dims, as
 * bf16 (128 B) | V dims 0..127 as E4M3 codes (128 B) | scale_k, scale_v fp32 | 8 zero
 * bytes.  A group's scale is amax / 448 over the group (1 when it is all zero); a
 * code is E4M3(value / scale), round to nearest even, saturating; a value is decoded
 * as code x scale.  hybrid_decode_attn reads such rows with CSKV_ATTN_KV_FP8.
 * rows : [n, 256] dtype (CSKV_F32 or CSKV_BF16), 16-byte aligned, device.
 * out  : [n, 336] bytes, 16-byte aligned, device.
 * n == 0 launches nothing.  Errors: CSKV_ERR_INVALID_ARG (null or misaligned pointer
 * with n > 0, n < 0 or n > 8 (2^31 - 1), bad dtype), CSKV_ERR_UNSUPPORTED (FP8 input).
 * ------------------------------------------------------------------------ */
CSKV_API int kv_quantize_fp8(const void* rows, int dtype, int64_t n, void* out, cskv_stream_t stream);

/* ------------------------------------------------------------------------
 * rmsnorm_heads -- RMSNorm of head vectors (the query-side pass).
 *
 * [SW] §十四.3: queries and KV are RMS-normalised so that attention logits cannot
 * blow up.  Every row of x (one query head: d = 128 values) becomes
 *     out = x / sqrt(mean(x^2) + eps) * gamma
 * in fp32, rounded to the storage type.  (The KV side is the compression
 * epilogue: csa_compress / hca_compress with rmsnorm = 1.)
 * x, out : [rows, 128] dtype (CSKV_F32 or CSKV_BF16), 16-byte aligned; out may be x.
 * gamma  : [128] fp32 or NULL (ones), 4-byte aligned.  eps >= 0, finite.
 * rows == 0 launches nothing; d other than 128 is CSKV_ERR_UNSUPPORTED.
 * ------------------------------------------------------------------------ */
CSKV_API int rmsnorm_heads(const void* x, int dtype, int64_t rows, int d, const float* gamma, float eps, void* out,
                           cskv_stream_t stream);

/* ------------------------------------------------------------------------
 * lindex_pool_keys -- the indexer's entry keys from per-token keys.
 *
 * [TR] §4.2 (LightningIndexer: per-token keys, then a 1-D pool whose kernel and
 * stride are the block size): entry i of a sequence gets the mean of the
 * per-token keys of tokens 4i..4i+3 (a partial last block: of the tokens it
 * has), stored as OCP E4M3 codes with one fp32 scale per entry:
 *     scale = amax_j |key_j| / 448 (1 for an all-zero key),
 *     code_j = E4M3(key_j / scale), round to nearest even, saturating to +-448.
 * fp32 arithmetic: the tokens are summed in order, divided once by their
 * count, each element divided once by the scale.  The outputs are the k_idx /
 * k_scale arrays lindex_score_topk reads.
 *
 * k_tok              : [rows, Di] in_dtype (CSKV_F32 or CSKV_BF16; CSKV_FP8E4M3
 *                      is CSKV_ERR_UNSUPPORTED), 16-byte aligned; finite values.
 * Di                 : 64 or 128 (other positive values: CSKV_ERR_UNSUPPORTED).
 * tok_off, tok0, batch, ent_off, first_block, num_blocks, max_blocks : as
 *                      csa_compress (rows of sequence b are its token tail from
 *                      tok0[b]; entry i goes to row ent_off[b] + i).
 * out_codes          : [*, Di] uint8 E4M3 codes, 16-byte aligned.
 * out_scale          : [*] fp32, 4-byte aligned.
 * Device checks: an entry outside the sequence or its ent_off range sets
 * CSKV_DEV_BAD_INDEX, one whose tokens start before the provided tail sets
 * CSKV_DEV_TAIL_MISSING (the entry is skipped), num_blocks above max_blocks
 * sets CSKV_DEV_CAPACITY.  max_blocks == 0 launches nothing.
 * ------------------------------------------------------------------------ */
CSKV_API int lindex_pool_keys(const void* k_tok, int in_dtype, int Di, const int64_t* tok_off,
                 const int64_t* tok0, int batch, const int64_t* ent_off, const int64_t* first_block,
                 const int64_t* num_blocks, int64_t max_blocks, uint8_t* out_codes, float* out_scale,
                 int* dev_status, cskv_stream_t stream);

/* ------------------------------------------------------------------------
 * lindex_score_topk -- Lightning Indexer scan fused with exact top-k.
 *
 * [SW] §六/§七/§十, [TR] §4.2, [AM]: query t (sequence q_seq[t], position
 * q_pos[t]) sees CSA entries i < V_t = floor((q_pos[t]+1)/4); entry i scores
 *     s_i = sum_h head_w[h] * ReLU(q_scale[t,h] * k_scale[i] * <q_idx[t,h,:], k_idx[i,:]>)
 * (fp32 arithmetic; scales and weights default to 1 when NULL).  The
 * min(k, V_t) best entries are kept, equal scores going to the lower index.
 *
 * q_idx   : [T, Hi, Di] dtype;  q_scale: [T, Hi] fp32 or NULL.
 * k_idx   : [sum entries, Di] dtype;  k_scale: [sum entries] fp32 or NULL.
 *           dtype CSKV_FP8E4M3 (OCP E4M3 codes; Hi <= 16, Di in {64, 128}) or
 *           CSKV_F32 (Hi <= 16, Di <= 128, Di % 4 == 0).
 * head_w  : [Hi] fp32 or NULL.
 * q_seq   : [T] int32 sequence of each query; q_pos: [T] int64.
 * ent_off : [batch+1] int64, entries of sequence b are rows ent_off[b].. of k_idx.
 * max_entries : host, >= every V_t (visible entries); sizes the plan.
 * out_idx : [T, k] int32: the kept entries (indices within the sequence) in
 *           ascending index order, then -1 padding.
 * out_score : [T, k] fp32 or NULL: the score of each kept entry (0 on padding).
 * prefetch_rows, prefetch_row_bytes : optional (NULL / 0 for none): a row array
 *           indexed like k_idx (rows ent_off[b] + i, prefetch_row_bytes each, a
 *           multiple of 16, 16-byte aligned) -- e.g. the compressed CSA cache that
 *           the attention call gathers next.  The rows of the kept entries are
 *           prefetched into L2 as they are emitted; a hint with no effect on results.
 *           Issuing the prefetches lengthens the call's tail; on the decode shapes
 *           measured (1-64 queries, k = 1024) it cost more than the gather saved.
 * workspace : lindex_workspace_size(T, k, max_entries) bytes, zero-filled before
 *           its first use; every call leaves it ready for the next (arrival
 *           counters and histograms back at zero, barrier generations advanced,
 *           the rest scratch), so it can be reused as is, unless the call flagged
 *           CSKV_DEV_TIMEOUT (zero-fill it again then).
 *           Calls sharing a workspace must be ordered on one stream.
 * Many queries (T >= 256, E4M3, Hi in {8, 16}, Di in {64, 128}) with that full
 * workspace run on the tensor cores (see lindex_workspace_size): the scores are
 * the same up to fp32 rounding order (the positive scales are applied after the
 * ReLU and head weights, where exact algebra allows it), the selection the same
 * exact top-k of them; an entry list that overflows inside one score bin of
 * unequal scores flags CSKV_DEV_CAPACITY.
 * ------------------------------------------------------------------------ */
CSKV_API int lindex_score_topk(const void* q_idx, const float* q_scale, const void* k_idx, const float* k_scale,
                      const float* head_w, const int32_t* q_seq, const int64_t* q_pos,
                      const int64_t* ent_off, int batch, int T, int Hi, int Di, int k, int dtype,
                      int64_t max_entries, int32_t* out_idx, float* out_score,
                      const void* prefetch_rows, int64_t prefetch_row_bytes,
                      void* workspace, size_t ws_bytes, int* dev_status, cskv_stream_t stream);

/* ------------------------------------------------------------------------
 * lindex_score_topk_mxfp4 -- the same scan and selection on FP4 indexer vectors.
 *
 * [SW] §六.1 / §十三.4, [TR] §4.2: the indexer only ranks entries, so its QK path may run
 * in FP4.  Keys and queries are OCP MXFP4: E2M1 elements (sign, 2 exponent bits with bias
 * 1, 1 mantissa bit: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), two per byte (element 2j in
 * the low nibble of byte j), and one E8M0 scale 2^(e - 127) per 32 elements (e = 0xFF is
 * NaN).  With decoded values q[t,h,:] and k[i,:]:
 *     s_i = sum_h head_w[h] * ReLU(q_scale[t,h] * <q[t,h,:], k[i,:]>)
 * (per-block dot products exact, then fp32), and the selection, outputs and workspace are
 * exactly those of lindex_score_topk.
 * q_codes  : [T, Hi, Di/2] uint8, 16-byte aligned;  q_bscale: [T, Hi, Di/32] uint8.
 * q_scale  : [T, Hi] fp32 or NULL (1).
 * k_codes  : [sum entries, Di/2] uint8, 16-byte aligned;  k_bscale: [sum entries, Di/32]
 *            uint8, aligned to Di/32 bytes (a key's scales are read as one word).
 * Hi in 1..16, Di 64 or 128 (else CSKV_ERR_UNSUPPORTED).  Other arguments: as
 * lindex_score_topk.
 * ------------------------------------------------------------------------ */
CSKV_API int lindex_score_topk_mxfp4(const uint8_t* q_codes, const uint8_t* q_bscale, const float* q_scale,
                      const uint8_t* k_codes, const uint8_t* k_bscale, const float* head_w,
                      const int32_t* q_seq, const int64_t* q_pos, const int64_t* ent_off, int batch, int T,
                      int Hi, int Di, int k, int64_t max_entries, int32_t* out_idx, float* out_score,
                      const void* prefetch_rows, int64_t prefetch_row_bytes,
                      void* workspace, size_t ws_bytes, int* dev_status, cskv_stream_t stream);

/* ------------------------------------------------------------------------
 * lindex_topk_from_scores -- the selection half of lindex_score_topk alone.
 *
 * Keeps, for every row t, the min(k, n_valid[t]) largest of scores[t, 0..n_valid[t]-1]
 * (ties to the lower index), with the same output format and workspace rules.
 * scores : [T, ld_scores] fp32; n_valid : [T] int64 (<= max_entries <= ld_scores).
 * ------------------------------------------------------------------------ */
CSKV_API int lindex_topk_from_scores(const float* scores, int64_t ld_scores, const int64_t* n_valid,
                            int T, int k, int64_t max_entries, int32_t* out_idx, float* out_score,
                            void* workspace, size_t ws_bytes, int* dev_status, cskv_stream_t stream);

/* Workspace bytes of lindex_score_topk / lindex_topk_from_scores for T queries.
 * Many queries (T >= 256) of E4M3 vectors with Hi in {8, 16} and Di in {64, 128} (a
 * prefill chunk) run on the tensor cores: tcgen05 kind::f8f6f4 products of 16 (or 8)
 * queries' heads with 128-entry key tiles, two passes (a per-query histogram of the
 * scores, then every entry that can be among the k best appended to the query's
 * candidate list in index order), and the exact top-k over the lists.  That path needs
 * lindex_workspace_size bytes (about T * 8 * max(8192, 2k) for the lists); with less,
 * but at least lindex_workspace_size_scan(T, max_entries), such calls take the
 * per-query scan instead.  Both give the same selection up to fp32 rounding order. */
CSKV_API size_t lindex_workspace_size(int T, int k, int64_t max_entries);
CSKV_API size_t lindex_workspace_size_scan(int T, int64_t max_entries);

/* ------------------------------------------------------------------------
 * hybrid_decode_attn -- MQA attention over compressed entries + raw window + sink.
 *
 * [SW] §三.1/§六/§八/§十/§十一/§十二, [TR] §2.2/§3.1/§4.3: for query t at
 * position p in sequence b, the rows are
 *   mode CSKV_CSA: the compressed entries idx[t, 0..k-1] (entries < 0 skipped;
 *                  entries not visible at p, i.e. >= floor((p+1)/4), flagged
 *                  CSKV_DEV_BAD_INDEX and skipped),
 *   mode CSKV_HCA: every visible HCA entry i < floor((p+1)/128) (idx unused),
 * followed by the raw window tokens max(0, p-window+1) .. p.  With logits
 * l = scale * <q_h, K_row> and the sink logit sink[h] in the denominator:
 *   o[t,h,:] = sum_rows softmax(l ∪ {sink})_row * V_row,
 *   lse[t,h] = log(sum_rows exp(l) + exp(sink[h])).
 * Split-KV partials are merged on device ([TR] §3.1 online softmax).
 *
 * q       : [T, H, d] dtype (CSKV_F32 or CSKV_BF16), H <= 128, d == 128.
 * kv_cmp  : [sum entries, 2d] dtype; cmp_off: [batch+1] int64 entry offsets.
 * idx     : [T, k] int32 (mode CSA), NULL for HCA.
 * kv_raw  : [rows, 2d] dtype raw window rows; raw_off: [batch+1] int64;
 *           raw_tok0: [batch] int64 or NULL (0): token of sequence b's first row.
 * sink    : [H] fp32 or NULL (no sink).  scale: host float, positive and finite
 *           (1/sqrt(d) typical); anything else is CSKV_ERR_INVALID_ARG.
 * q_seq   : [T] int32; q_pos: [T] int64.
 * max_entries : host; mode HCA: >= every visible HCA entry count; mode CSA: unused.
 * out     : [T, H, d] fp32;  lse: [T, H] fp32 or NULL.
 * workspace : hybrid_attn_workspace_size(...) bytes (no zero-fill needed).
 * mode | CSKV_ATTN_PAIRS : the caller states that queries 2j and 2j + 1 (j < T/2) are the
 *           same sequence's consecutive positions p, p + 1 (a prefill chunk; with an odd T the
 *           last query is alone).  With bf16 and H == 64 the HCA kernel then gives each pair
 *           one pass over the union of the two row lists (the visible entries, then the
 *           window tokens p - window + 1 .. p + 1, each masked for the query that does not
 *           see it): the rows are gathered once and the pair's 128 heads fill the tensor-core
 *           tile.  Results are those of the queries taken one by one.  A pair that is not
 *           adjacent is flagged CSKV_DEV_BAD_INDEX and its second query attends to nothing
 *           (output 0).  Elsewhere (CSA, fp32, other H, or a plan whose splits do not fit
 *           one cluster) the bit is ignored.
 * mode | CSKV_ATTN_KV_FP8 : kv_cmp holds FP8 main-KV rows (kv_quantize_fp8: 336 bytes a
 *           row, indexed by cmp_off like the plain rows); kv_raw stays in dtype.  The rows
 *           are decoded as they are loaded, on the CUDA cores (the tensor-core kernel takes
 *           plain rows only; ignores CSKV_ATTN_PAIRS).  The workspace size is the same.
 * ------------------------------------------------------------------------ */
CSKV_API int hybrid_decode_attn(int mode, const void* q, const void* kv_cmp, const int64_t* cmp_off,
                       const int32_t* idx, int k, const void* kv_raw, const int64_t* raw_off,
                       const int64_t* raw_tok0, int window, const float* sink, float scale,
                       const int32_t* q_seq, const int64_t* q_pos, int batch, int T, int H, int d,
                       int dtype, int64_t max_entries, float* out, float* lse,
                       void* workspace, size_t ws_bytes, int* dev_status, cskv_stream_t stream);

CSKV_API size_t hybrid_attn_workspace_size(int mode, int T, int H, int d, int k, int window, int64_t max_entries);

/* ------------------------------------------------------------------------
 * hybrid_decode_attn_noalloc -- hybrid_decode_attn for callers that cannot allocate.
 *
 * The source pages have no counterpart: this is a library convenience.  Some callers
 * cannot allocate device memory when they run attention (a memory pool that owns all
 * device memory, a plugin host that forbids allocations after start-up, a hot path that
 * must never synchronise, as cudaMalloc/cudaFree can).  This variant takes the same
 * arguments as hybrid_decode_attn minus the workspace, and keeps its split-KV partials
 * in one array of CSKV_NOALLOC_SCRATCH_BYTES that the library declares in device memory.
 * After its first call on a device (below) it allocates nothing.
 * - A call whose hybrid_attn_workspace_size() exceeds CSKV_NOALLOC_SCRATCH_BYTES returns
 *   CSKV_ERR_WORKSPACE and launches nothing.
 * - Every GPU that loads the library holds the array until the process exits.
 * - All calls share the array, which keeps the last call's contents.  Nothing in it needs
 *   clearing (every partial is written before it is read), but calls that overlap on the
 *   GPU (unordered streams) race on it.
 * - The first call on a device looks up the array's address with that device current.
 *   Under lazy module loading (the CUDA 12 default) that first lookup may load the
 *   library's device code and reserve the array, which allocates and may synchronise: make
 *   one warm-up call per device at start-up, before any stream capture and before
 *   allocation becomes forbidden.  Every later call allocates nothing.
 * - Arguments are checked exactly as hybrid_decode_attn checks them (CSKV_ERR_INVALID_ARG /
 *   CSKV_ERR_UNSUPPORTED) before the scratch size is.
 * ------------------------------------------------------------------------ */
#define CSKV_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
CSKV_API int hybrid_decode_attn_noalloc(int mode, const void* q, const void* kv_cmp, const int64_t* cmp_off,
                       const int32_t* idx, int k, const void* kv_raw, const int64_t* raw_off,
                       const int64_t* raw_tok0, int window, const float* sink, float scale,
                       const int32_t* q_seq, const int64_t* q_pos, int batch, int T, int H, int d,
                       int dtype, int64_t max_entries, float* out, float* lse,
                       int* dev_status, cskv_stream_t stream);

/* ------------------------------------------------------------------------
 * cskv_copy_segments -- device-side scatter of byte segments (input staging).
 *
 * Not a step of the method: plumbing for callers that move a decode step's new
 * inputs (queries, the newest token rows, the newest indexer keys) to the GPU from
 * one packed staging buffer and spread them to their places, or read results back.
 * Segment i copies len[i] bytes from src + src_off[i] to dst[i].
 * src     : buffer holding the packed segments: device memory, or page-locked host
 *           memory through the address cskv_mapped_pointer() gives for it (the
 *           kernel then reads the host buffer over the bus: no separate copy).
 * src_off, len : [n] int64 device arrays; dst : [n] device array of pointers the
 *           device can write: device memory, or mapped page-locked host memory
 *           (cskv_mapped_pointer() addresses).  Segments must not overlap their
 *           destinations.  The caller keeps host buffers alive and unchanged until
 *           the stream has passed the copy.
 * n       : number of segments (0 launches nothing).
 * Errors: CSKV_ERR_INVALID_ARG for a null pointer with n > 0 or n < 0.  The
 * pointers inside the arrays are not checked: take host addresses from
 * cskv_mapped_pointer(), never a plain host pointer.
 * ------------------------------------------------------------------------ */
CSKV_API int cskv_copy_segments(const void* src, const int64_t* src_off, void* const* dst, const int64_t* len, int n,
                                cskv_stream_t stream);

/* ------------------------------------------------------------------------
 * cskv_mapped_pointer -- the address at which the current device reaches p.
 *
 * Plumbing for zero-copy staging (cskv_copy_segments).  Device or managed memory:
 * *out = p.  Page-locked host memory mapped into the device's address space:
 * *out = the device-side address of p (under unified addressing, p itself).
 * Pageable host memory, or a null p / out: CSKV_ERR_INVALID_ARG with *out = NULL
 * (when out is not null).  A failed CUDA query: CSKV_ERR_LAUNCH.  Host-side query
 * only: launches nothing, allocates nothing.
 * ------------------------------------------------------------------------ */
CSKV_API int cskv_mapped_pointer(const void* p, void** out);

#ifdef __cplusplus
}
#endif

#endif /* CSKV_H */
