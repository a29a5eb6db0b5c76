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
#include <cuda_fp4.h>
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

// MX-FP4: the same rows and scale tiles, E2M1 elements (magnitudes 0 .. 6)
// packed two to a byte (the even element in the low nibble, 64 bytes a row),
// scale 2^(floor(log2 amax) - 2) (2 = E2M1's largest exponent).
template <typename T>
__global__ void __launch_bounds__(256) mxfp4_quantize_kernel(const T* x, uint8_t* codes,
                                                             uint8_t* sf, int64_t B,
                                                             int64_t rows, int64_t tiles) {
  const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t padded = tiles * 128;
  if (gw >= B * padded) return;   // warp-uniform
  const int64_t b = gw / padded, r = gw % padded;
  const int kb = lane >> 3;
  const int64_t sfpos = (b * tiles + r / 128) * 512 + 16 * (r % 32) + 4 * ((r % 128) / 32) + kb;
  if (r >= rows) {
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
    e = ilogbf(am) - 2;
    e = e < -127 ? -127 : (e > 127 ? 127 : e);
  }
  // round to nearest even, saturating at 6
  const __nv_fp4x2_storage_t c01 = __nv_cvt_float2_to_fp4x2(
      make_float2(ldexpf(v[0], -e), ldexpf(v[1], -e)), __NV_E2M1, cudaRoundNearest);
  const __nv_fp4x2_storage_t c23 = __nv_cvt_float2_to_fp4x2(
      make_float2(ldexpf(v[2], -e), ldexpf(v[3], -e)), __NV_E2M1, cudaRoundNearest);
  *reinterpret_cast<uint16_t*>(codes + row * 64 + 2 * lane) =
      (uint16_t)((uint32_t)c01 | ((uint32_t)c23 << 8));
  if ((lane & 7) == 0) sf[sfpos] = (uint8_t)(e + 127);
}

// Mixed storage of compressed entries: one warp per entry; lane l < (c-r)/32
// quantizes 32-element block l of the non-RoPE dims to MX-FP8 (the same rule
// as above), every lane rounds a share of the r RoPE dims to bf16.
template <typename T>
__global__ void __launch_bounds__(256) mixed_store_kernel(const T* x, uint8_t* rec, int64_t n,
                                                          int c, int r, int rec_bytes) {
  const int64_t e = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (e >= n) return;   // warp-uniform
  const int cq = c - r, nblk = cq / 32;
  const T* xe = x + e * c;
  uint8_t* re = rec + e * rec_bytes;
  if (lane < nblk) {
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = to_float(xe[32 * lane + i]);
    float am = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) am = fmaxf(am, fabsf(v[i]));
    int ex = -127;
    if (am > 0.f) {
      ex = ilogbf(am) - 8;
      ex = ex < -127 ? -127 : (ex > 127 ? 127 : ex);
    }
    uint32_t w[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
          make_float2(ldexpf(v[4 * q], -ex), ldexpf(v[4 * q + 1], -ex)), __NV_SATFINITE,
          __NV_E4M3);
      const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
          make_float2(ldexpf(v[4 * q + 2], -ex), ldexpf(v[4 * q + 3], -ex)), __NV_SATFINITE,
          __NV_E4M3);
      w[q] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    uint4* dst = reinterpret_cast<uint4*>(re + 32 * lane);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    re[cq + 2 * r + lane] = (uint8_t)(ex + 127);
  }
  bf16* rope = reinterpret_cast<bf16*>(re + cq);
  for (int d = lane; d < r; d += 32) rope[d] = __float2bfloat16_rn(to_float(xe[cq + d]));
  for (int pb = cq + 2 * r + nblk + lane; pb < rec_bytes; pb += 32) re[pb] = 0;
}

}  // namespace

size_t mixed_record_bytes(int c, int r) {
  const size_t raw = (size_t)(c - r) + 2 * (size_t)r + (size_t)(c - r) / 32;
  return (raw + 15) & ~(size_t)15;
}

cudaError_t launch_mixed_store(int dtype, const void* x, void* rec, int64_t n, int c, int r,
                               cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const int rb = (int)mixed_record_bytes(c, r);
  const int64_t blocks = (n * 32 + 255) / 256;
  if (dtype == CSA_BF16)
    mixed_store_kernel<bf16><<<(unsigned)blocks, 256, 0, stream>>>(
        static_cast<const bf16*>(x), static_cast<uint8_t*>(rec), n, c, r, rb);
  else
    mixed_store_kernel<float><<<(unsigned)blocks, 256, 0, stream>>>(
        static_cast<const float*>(x), static_cast<uint8_t*>(rec), n, c, r, rb);
  return cudaGetLastError();
}

cudaError_t launch_mxfp4_quantize(int dtype, const void* x, void* codes, void* scales, int64_t B,
                                  int64_t rows, cudaStream_t stream) {
  const int64_t tiles = (rows + 127) / 128;
  const int64_t warps = B * tiles * 128;
  if (warps == 0) return cudaSuccess;
  const int64_t blocks = (warps * 32 + 255) / 256;
  if (dtype == CSA_BF16)
    mxfp4_quantize_kernel<bf16><<<(unsigned)blocks, 256, 0, stream>>>(
        static_cast<const bf16*>(x), static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales),
        B, rows, tiles);
  else
    mxfp4_quantize_kernel<float><<<(unsigned)blocks, 256, 0, stream>>>(
        static_cast<const float*>(x), static_cast<uint8_t*>(codes),
        static_cast<uint8_t*>(scales), B, rows, tiles);
  return cudaGetLastError();
}

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
