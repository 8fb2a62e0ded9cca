// Device-side scatter of byte segments: the input-staging helper behind cskv_copy_segments.
// One CTA per segment; 16-byte moves when the source, destination and length allow it, else
// 4-byte, else single bytes.
#include "launch.cuh"

namespace cskv {

__global__ void __launch_bounds__(256) copy_segments_kernel(const uint8_t* __restrict__ src,
                                                            const int64_t* __restrict__ src_off,
                                                            void* const* __restrict__ dst,
                                                            const int64_t* __restrict__ len, int n) {
  pdl_wait();
  const int i = blockIdx.x;
  if (i >= n) return;
  const uint8_t* s = src + src_off[i];
  uint8_t* d = static_cast<uint8_t*>(dst[i]);
  const int64_t L = len[i];
  const uintptr_t a = reinterpret_cast<uintptr_t>(s) | reinterpret_cast<uintptr_t>(d) | (uintptr_t)L;
  if ((a & 15) == 0) {
    for (int64_t j = threadIdx.x; j < L / 16; j += blockDim.x)
      reinterpret_cast<uint4*>(d)[j] = reinterpret_cast<const uint4*>(s)[j];
  } else if ((a & 3) == 0) {
    for (int64_t j = threadIdx.x; j < L / 4; j += blockDim.x)
      reinterpret_cast<uint32_t*>(d)[j] = reinterpret_cast<const uint32_t*>(s)[j];
  } else {
    for (int64_t j = threadIdx.x; j < L; j += blockDim.x) d[j] = s[j];
  }
}

cudaError_t launch_copy_segments(const void* src, const int64_t* src_off, void* const* dst, const int64_t* len, int n,
                                 cudaStream_t stream) {
  cudaError_t e = ensure_smem(copy_segments_kernel, 0);
  if (e != cudaSuccess) return e;
  e = launch_dependent(copy_segments_kernel, dim3(n), dim3(256), 0, stream, (const uint8_t*)src, src_off, dst, len,
                       n);
  note_launch();
  return e;
}

}  // namespace cskv
