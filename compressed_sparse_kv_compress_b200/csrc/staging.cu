// Device-side scatter of byte segments: the input-staging helper behind cskv_copy_segments.
// One CTA per segment; 16-byte moves when the source, destination and length allow it, else
// 4-byte, else single bytes.  Either side may be pinned host memory mapped into the device's
// address space (a zero-copy transfer over PCIe): each thread therefore issues a batch of
// independent loads before it stores any of them, so a batch costs one bus round trip.
#include "launch.cuh"

namespace cskv {

template <typename W>
__device__ __forceinline__ void copy_words(const W* __restrict__ s, W* __restrict__ d, int64_t nw) {
  constexpr int kBatch = 8;
  const int64_t step = (int64_t)blockDim.x * kBatch;
  for (int64_t j0 = threadIdx.x; j0 < nw; j0 += step) {
    W v[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int64_t j = j0 + (int64_t)u * blockDim.x;
      if (j < nw) v[u] = s[j];
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int64_t j = j0 + (int64_t)u * blockDim.x;
      if (j < nw) d[j] = v[u];
    }
  }
}

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
  if ((a & 15) == 0)
    copy_words(reinterpret_cast<const uint4*>(s), reinterpret_cast<uint4*>(d), L / 16);
  else if ((a & 3) == 0)
    copy_words(reinterpret_cast<const uint32_t*>(s), reinterpret_cast<uint32_t*>(d), L / 4);
  else
    copy_words(s, d, L);
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
