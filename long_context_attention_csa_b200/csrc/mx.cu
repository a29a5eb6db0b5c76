// MX-FP8 quantization of indexer operands (q_I and the cached K_I).
//
// Method: page "DeepSeek-V4：迈向高效百万 Token 上下文智能", §3.3, last
// paragraph, and §3.6: the indexer's QK path runs in low precision (FP4 with
// quantization-aware training in the model).  Format taken here: OCP
// Microscaling FP8 -- E4M3 elements, one shared power-of-two scale per 32
// consecutive elements of a row, 2^(floor(log2 amax) - 8) (8 = E4M3's largest
// exponent), elements rounded to nearest (ties to even) and saturated at 448.
//
// Layout of the scales, chosen for the block-scaled tensor-core MMA: per 128
// rows of a batch element, one 512-byte tile in which row r (r < 128) and
// 32-element block kb of the 128-element row sit at byte
//   16 (r mod 32) + 4 (r / 32) + kb,
// each byte the UE8M0 exponent + 127.  Copied as is into TMEM (32 lanes x 16
// bytes, replicated over the four lane quarters), it puts row r's four scales
// in the 32-bit word of lane r mod 32, column r / 32.  Rows past the end of
// the tensor get scale bytes 0.
#include <cuda_fp8.h>

#include "common.cuh"
#include "internal.h"
#include "tc.h"

namespace csa {

namespace {

// One warp per (padded) row: lane l holds elements 4l .. 4l + 3 (block l / 8).
template <typename T>
__global__ void __launch_bounds__(256) mxfp8_quantize_kernel(const T* x, uint8_t* codes,
                                                             uint8_t* sf, int64_t B,
                                                             int64_t rows, int64_t tiles) {
  const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t padded = tiles * 128;
  if (gw >= B * padded) return;   // warp-uniform
  const int64_t b = gw / padded, r = gw % padded;
  const int kb = lane >> 3;
  const int64_t sfpos = (b * tiles + r / 128) * 512 + 16 * (r % 32) + 4 * ((r % 128) / 32) + kb;
  if (r >= rows) {   // padding rows of the last tile: scale bytes only
    if ((lane & 7) == 0) sf[sfpos] = 0;
    return;
  }
  const int64_t row = b * rows + r;
  float v[4];
  if constexpr (sizeof(T) == 2) {
    const uint2 u = *reinterpret_cast<const uint2*>(x + row * 128 + 4 * lane);
    v[0] = bf16_bits_to_float(u.x & 0xffffu);
    v[1] = bf16_bits_to_float(u.x >> 16);
    v[2] = bf16_bits_to_float(u.y & 0xffffu);
    v[3] = bf16_bits_to_float(u.y >> 16);
  } else {
    const float4 u = *reinterpret_cast<const float4*>(x + row * 128 + 4 * lane);
    v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
  }
  float am = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
  int e = -127;
  if (am > 0.f) {
    e = ilogbf(am) - 8;          // floor(log2 amax), exact (subnormals included)
    e = e < -127 ? -127 : (e > 127 ? 127 : e);
  }
  // x 2^-e is exact (a power-of-two scaling, |x 2^-e| < 512); the conversion
  // rounds to nearest even and saturates at the largest finite E4M3 value
  const __nv_fp8x2_storage_t c01 = __nv_cvt_float2_to_fp8x2(
      make_float2(ldexpf(v[0], -e), ldexpf(v[1], -e)), __NV_SATFINITE, __NV_E4M3);
  const __nv_fp8x2_storage_t c23 = __nv_cvt_float2_to_fp8x2(
      make_float2(ldexpf(v[2], -e), ldexpf(v[3], -e)), __NV_SATFINITE, __NV_E4M3);
  *reinterpret_cast<uint32_t*>(codes + row * 128 + 4 * lane) =
      (uint32_t)c01 | ((uint32_t)c23 << 16);
  if ((lane & 7) == 0) sf[sfpos] = (uint8_t)(e + 127);
}

}  // namespace

cudaError_t launch_mxfp8_quantize(int dtype, const void* x, void* codes, void* scales, int64_t B,
                                  int64_t rows, cudaStream_t stream) {
  const int64_t tiles = (rows + 127) / 128;
  const int64_t warps = B * tiles * 128;
  if (warps == 0) return cudaSuccess;
  const int64_t blocks = (warps * 32 + 255) / 256;
  if (dtype == CSA_BF16)
    mxfp8_quantize_kernel<bf16><<<(unsigned)blocks, 256, 0, stream>>>(
        static_cast<const bf16*>(x), static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales),
        B, rows, tiles);
  else
    mxfp8_quantize_kernel<float><<<(unsigned)blocks, 256, 0, stream>>>(
        static_cast<const float*>(x), static_cast<uint8_t*>(codes),
        static_cast<uint8_t*>(scales), B, rows, tiles);
  return cudaGetLastError();
}

}  // namespace csa
