// Quantiser of FP8 main-KV rows (layout and rule in kv8.cuh; [SW] shareware.cn/news/167317
// §十三.4).  One warp a row: lane l holds values 8l .. 8l + 7 of the 256 K||V values, so lanes
// 0..7 are the E4M3 K dims, 8..15 the bf16 RoPE dims and 16..31 the E4M3 V dims; each group's
// largest magnitude is a shuffle reduction inside its lanes.
#include "kv8.cuh"
#include "launch.cuh"

namespace cskv {

constexpr int kKv8WarpsPerCta = 8;

template <typename T>
__global__ void __launch_bounds__(32 * kKv8WarpsPerCta) kv_quantize_fp8_kernel(const T* __restrict__ rows, int64_t n,
                                                                              uint8_t* __restrict__ out) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * kKv8WarpsPerCta + (threadIdx.x >> 5);
  if (r >= n) return;
  float x[8];
  Vec8<T>::load(rows + (size_t)r * kRow + 8 * lane, x);
  uint8_t* o = out + (size_t)r * kKv8RowBytes;
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(x[i]));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));   // max over the 8-lane group: K (lanes 0..7)
  const float m16 = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));  // 16-lane group: V (16..31)
  if (lane >= 8 && lane < 16) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
      w[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(o + 64 + 16 * (lane - 8)) = make_uint4(w[0], w[1], w[2], w[3]);
    return;
  }
  const float amax = lane < 8 ? m : m16;
  const float scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  uint32_t lo = 0, hi = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    lo |= (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(x[i], scale), __NV_SATFINITE, __NV_E4M3) << (8 * i);
    hi |= (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(x[4 + i], scale), __NV_SATFINITE, __NV_E4M3) << (8 * i);
  }
  *reinterpret_cast<uint2*>(o + (lane < 8 ? 8 * lane : 192 + 8 * (lane - 16))) = make_uint2(lo, hi);
  if (lane == 0 || lane == 16) reinterpret_cast<float*>(o + 320)[lane == 0 ? 0 : 1] = scale;
  if (lane == 1) *reinterpret_cast<uint2*>(o + 328) = make_uint2(0u, 0u);
}

cudaError_t launch_kv_quantize_fp8(const void* rows, int dtype, int64_t n, uint8_t* out, cudaStream_t stream) {
  const dim3 grid((unsigned)((n + kKv8WarpsPerCta - 1) / kKv8WarpsPerCta)), block(32 * kKv8WarpsPerCta);
  cudaError_t e;
  if (dtype == CSKV_F32) {
    e = ensure_smem(kv_quantize_fp8_kernel<float>, 0);
    if (e == cudaSuccess)
      e = launch_dependent(kv_quantize_fp8_kernel<float>, grid, block, 0, stream, (const float*)rows, n, out);
  } else {
    e = ensure_smem(kv_quantize_fp8_kernel<__nv_bfloat16>, 0);
    if (e == cudaSuccess)
      e = launch_dependent(kv_quantize_fp8_kernel<__nv_bfloat16>, grid, block, 0, stream,
                           (const __nv_bfloat16*)rows, n, out);
  }
  note_launch();
  return e;
}

}  // namespace cskv
