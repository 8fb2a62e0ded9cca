// FP8 main-KV rows: the compressed cache in 8-bit floats with the position-sensitive
// dimensions kept in bf16 ([SW] shareware.cn/news/167317 §十三.4: the main KV may be stored in
// FP8, the dimensions most sensitive to position information keep a higher precision).
//
// A row holds K (128 dims) then V (128 dims) of one compressed entry, 336 bytes:
//   [  0,  64) K dims 0..63, OCP E4M3 codes (value = code x scale_k)
//   [ 64, 192) K dims 64..127 (the RoPE dims) as bf16
//   [192, 320) V dims 0..127, OCP E4M3 codes (value = code x scale_v)
//   [320, 328) scale_k, scale_v as fp32;  [328, 336) zero
// scale = amax / 448 over its group (1 for an all-zero group); code = E4M3(value / scale),
// round to nearest even, saturating.
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"

namespace cskv {

constexpr int kKv8RowBytes = 336;
constexpr int kKv8KFp8 = 64;  // K dims stored as E4M3; K dims 64..127 are bf16

__device__ __forceinline__ float e4m3_to_float(uint32_t code) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)code, __NV_E4M3);
  return __half2float(__half(h));
}

// Values 32 * part .. 32 * part + 31 of an FP8 row (part 0..7 over the 256 K||V values), as
// floats: parts 0, 1 are E4M3 K dims, 2, 3 the bf16 RoPE dims, 4..7 E4M3 V dims.
__device__ __forceinline__ void kv8_load_part(const uint8_t* row, int part, float (&f)[32]) {
  if (part == 2 || part == 3) {
    const uint4* src = reinterpret_cast<const uint4*>(row + 64 + (part - 2) * 64);
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const uint4 w = __ldg(src + v);
      const uint32_t x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        f[8 * v + 2 * i] = __uint_as_float(x[i] << 16);
        f[8 * v + 2 * i + 1] = __uint_as_float(x[i] & 0xffff0000u);
      }
    }
    return;
  }
  const bool is_v = part >= 4;
  const float s = __ldg(reinterpret_cast<const float*>(row + 320) + (is_v ? 1 : 0));
  const uint4* src = reinterpret_cast<const uint4*>(row + (is_v ? 192 + (part - 4) * 32 : part * 32));
#pragma unroll
  for (int v = 0; v < 2; ++v) {
    const uint4 w = __ldg(src + v);
    const uint32_t x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int b = 0; b < 4; ++b) f[16 * v + 4 * i + b] = e4m3_to_float((x[i] >> (8 * b)) & 0xFFu) * s;
  }
}

// The 16 bytes of bf16 values 8 * lane .. 8 * lane + 7 (lane 0..31 over the 256 K||V values)
// of an FP8 row, as the tensor-core kernel's gather stores them: lanes 0..7 decode 8 K codes,
// 8..15 copy the RoPE dims, 16..31 decode 8 V codes; a decoded value code x scale is rounded
// to bf16 (nearest even).
__device__ __forceinline__ uint4 kv8_lane_bf16x8(const uint8_t* row, int lane) {
  if (lane >= 8 && lane < 16) return __ldg(reinterpret_cast<const uint4*>(row + 64 + 16 * (lane - 8)));
  const bool is_v = lane >= 16;
  const float s = __ldg(reinterpret_cast<const float*>(row + 320) + (is_v ? 1 : 0));
  const uint2 w = __ldg(reinterpret_cast<const uint2*>(row + (is_v ? 192 + 8 * (lane - 16) : 8 * lane)));
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t x = i < 2 ? w.x : w.y;
    const int b = (i & 1) * 16;
    const __nv_bfloat162 h = __floats2bfloat162_rn(e4m3_to_float((x >> b) & 0xFFu) * s,
                                                   e4m3_to_float((x >> (b + 8)) & 0xFFu) * s);
    o[i] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

}  // namespace cskv
