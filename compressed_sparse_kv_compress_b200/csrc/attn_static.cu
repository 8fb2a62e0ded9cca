// hybrid_decode_attn without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the moment they run attention: code that
// sits under a memory pool which owns all device memory, plugin hosts that forbid device
// allocations after start-up, or hot paths that must never synchronise (cudaMalloc and
// cudaFree can synchronise the device).  For them this entry point keeps the split-KV
// partials in one fixed array that the library itself declares in device memory.
//
// Limits and behaviour:
//  * the array holds CSKV_NOALLOC_SCRATCH_BYTES; a call that needs more returns
//    CSKV_ERR_WORKSPACE and launches nothing;
//  * every GPU that loads this library keeps the array until the process exits;
//  * all calls share the array and it keeps the last call's partials; the partials are
//    always written before they are read, so nothing needs clearing, but two calls that
//    overlap on the GPU (different streams, no ordering between them) race on it;
//  * the first call on each device looks up the array's device address with that device
//    current (cudaGetSymbolAddress).  With lazy module loading (the CUDA 12 default) that
//    lookup may be what loads this library's device code on the device and reserves the
//    array, which allocates and can synchronise; so make one warm-up call per device at
//    start-up, before any stream capture and before the point where allocation is
//    forbidden.  Later calls allocate nothing.
#include <mutex>

#include "launch.cuh"

namespace {

constexpr size_t kScratchFloats = CSKV_NOALLOC_SCRATCH_BYTES / sizeof(float);
static __device__ __align__(256) float g_attn_scratch[kScratchFloats];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float* g_scratch_ptr[kMaxDevices] = {};

// Device address of the array for the current device (looked up once per device).
int scratch_for_current_device(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return CSKV_ERR_LAUNCH;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_attn_scratch);
    if (e != cudaSuccess || ptr == nullptr) {
      cudaGetLastError();
      return CSKV_ERR_LAUNCH;
    }
    g_scratch_ptr[dev] = static_cast<float*>(ptr);
  }
  *out = g_scratch_ptr[dev];
  return CSKV_OK;
}

}  // namespace

extern "C" int hybrid_decode_attn_noalloc(int mode, const void* q, const void* kv_cmp, const int64_t* cmp_off,
                                          const int32_t* idx, int k, const void* kv_raw, const int64_t* raw_off,
                                          const int64_t* raw_tok0, int window, const float* sink, float scale,
                                          const int32_t* q_seq, const int64_t* q_pos, int batch, int T, int H,
                                          int d, int dtype, int64_t max_entries, float* out, float* lse,
                                          int* dev_status, cskv_stream_t stream) {
  // the same argument checks as the regular entry point, before the size check, so a bad
  // argument is reported as such and not as a lack of scratch
  const int arc = cskv::check_attn_args(mode, q, kv_cmp, cmp_off, idx, k, kv_raw, raw_off, window, scale, q_seq,
                                        q_pos, batch, T, H, d, dtype, max_entries, out);
  if (arc != CSKV_OK || T == 0) return arc;
  const size_t need = hybrid_attn_workspace_size(mode, T, H, d, (mode & ~(CSKV_ATTN_PAIRS | CSKV_ATTN_KV_FP8)) == CSKV_CSA ? k : 0, window,
                                                 max_entries);
  if (need > CSKV_NOALLOC_SCRATCH_BYTES) return CSKV_ERR_WORKSPACE;
  float* scratch = nullptr;
  const int rc = scratch_for_current_device(&scratch);
  if (rc != CSKV_OK) return rc;
  return hybrid_decode_attn(mode, q, kv_cmp, cmp_off, idx, k, kv_raw, raw_off, raw_tok0, window, sink, scale, q_seq,
                            q_pos, batch, T, H, d, dtype, max_entries, out, lse, scratch,
                            CSKV_NOALLOC_SCRATCH_BYTES, dev_status, stream);
}
