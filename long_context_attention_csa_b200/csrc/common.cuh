// Shared device helpers of libcsa: vector loads/stores, reductions, RoPE
// angles and the device status word.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "../../include/csa.h"

namespace csa {

typedef __nv_bfloat16 bf16;

// Entry format as the kernels see it.
struct Fmt {
  int c;         // entry / head dim
  int r;         // RoPE dims: the last r of c
  float base;    // RoPE base
  float eps;     // RMSNorm epsilon
  uint32_t flags;
};

// ---- device status word (first 8 bytes of the workspace) -----------------
// The first error wins; later ones are dropped.  Never traps.
__device__ __forceinline__ void report(unsigned* status, unsigned code, unsigned detail) {
  if (status != nullptr) {
    if (atomicCAS(status, 0u, code) == 0u) atomicExch(status + 1, detail);
  }
}

// ---- programmatic dependent launch ---------------------------------------
// A kernel launched with programmatic stream serialization (launch_pdl) may
// start while the previous kernel in the stream is still running.  pdl_wait()
// returns once that kernel has completed and its memory is visible (at once
// for an ordinary launch), so a kernel calls it, in every thread, before its
// first global load or store.  pdl_trigger() lets the next such kernel start
// launching; it waits in its own pdl_wait() for this one to finish.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- 16-byte vector loads/stores as float ------------------------------
template <typename T> struct VecOf;
template <> struct VecOf<float> { static constexpr int N = 4; };
template <> struct VecOf<bf16> { static constexpr int N = 8; };

// A read-only global load the compiler keeps in program order (volatile asm):
// for loads issued well ahead of their first use.
__device__ __forceinline__ int32_t ldg_nc_volatile(const int32_t* p) {
  int32_t v;
  asm volatile("ld.global.nc.s32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits16) {
  return __uint_as_float(bits16 << 16);
}

__device__ __forceinline__ void load_vec(const float* p, float* o) {
  float4 v = __ldg(reinterpret_cast<const float4*>(p));
  o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
}
__device__ __forceinline__ void load_vec(const bf16* p, float* o) {
  uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
  uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    o[2 * i] = bf16_bits_to_float(w[i] & 0xffffu);
    o[2 * i + 1] = bf16_bits_to_float(w[i] >> 16);
  }
}
// streaming (evict-first) variant for data read exactly once
__device__ __forceinline__ void load_vec_stream(const float* p, float* o) {
  float4 v = __ldcs(reinterpret_cast<const float4*>(p));
  o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
}
__device__ __forceinline__ void load_vec_stream(const bf16* p, float* o) {
  uint4 v = __ldcs(reinterpret_cast<const uint4*>(p));
  uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    o[2 * i] = bf16_bits_to_float(w[i] & 0xffffu);
    o[2 * i + 1] = bf16_bits_to_float(w[i] >> 16);
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void store_vec(float* p, const float* v) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
__device__ __forceinline__ void store_vec(bf16* p, const float* v) {
  uint4 u;
  u.x = pack_bf16x2(v[0], v[1]);
  u.y = pack_bf16x2(v[2], v[3]);
  u.z = pack_bf16x2(v[4], v[5]);
  u.w = pack_bf16x2(v[6], v[7]);
  *reinterpret_cast<uint4*>(p) = u;
}

__device__ __forceinline__ float to_float(float x) { return x; }
__device__ __forceinline__ float to_float(bf16 x) { return __bfloat162float(x); }

// ---- RoPE ------------------------------------------------------------------
// cos/sin of pos * base^(-2i/r), the angle formed and reduced in double so that
// positions near 2^20 keep full accuracy, then rounded to float.
__device__ __forceinline__ void rope_cos_sin(int64_t pos, int i, int r, float base, float* cs,
                                             float* sn) {
  double theta = pow((double)base, -2.0 * (double)i / (double)r);
  double a = (double)pos * theta;
  double s, c;
  sincos(a, &s, &c);
  *cs = (float)c;
  *sn = (float)s;
}

// theta_i = base^(-2i/r) of RoPE pair i, in double: the angle pos * theta_i
// needs more than single precision once pos is large.
__device__ __forceinline__ double rope_theta(int i, int r, float base) {
  return pow((double)base, -2.0 * (double)i / (double)r);
}

// cos and sin of pos * theta for a precomputed theta: the angle is formed and
// reduced by a multiple of 2 pi in double (the reduced angle is accurate to
// about 1e-10 rad for |pos| < 2^32), then its sine and cosine are taken in
// single precision.
__device__ __forceinline__ void rope_cos_sin_theta(int64_t pos, double theta, float* cs,
                                                   float* sn) {
  constexpr double kTwoPi = 6.283185307179586;
  const double ang = (double)pos * theta;
  const double turns = rint(ang * (1.0 / kTwoPi));
  const float red = (float)fma(-turns, kTwoPi, ang);
  sincosf(red, sn, cs);
}

// Rotate the pairs of a VEC-wide slice [ch0, ch0+VEC) that fall in the RoPE
// dims [c-r, c) by angle pos * theta_i.
template <int VEC>
__device__ __forceinline__ void rope_slice(float* v, int ch0, const Fmt& f, int64_t pos) {
  int d0 = f.c - f.r;
#pragma unroll
  for (int e = 0; e < VEC; e += 2) {
    int ch = ch0 + e;
    if (ch >= d0) {
      float cs, sn;
      rope_cos_sin(pos, (ch - d0) >> 1, f.r, f.base, &cs, &sn);
      float x0 = v[e], x1 = v[e + 1];
      v[e] = x0 * cs - x1 * sn;
      v[e + 1] = x0 * sn + x1 * cs;
    }
  }
}

// ---- reductions ---------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Sum of `v` over each group of LPR consecutive threads (LPR a power of two,
// blockDim.x a multiple of LPR).  Every thread of the block must call it
// (it contains __syncthreads when LPR > 32).  `red` holds blockDim.x/32 floats.
__device__ __forceinline__ float group_sum(float v, int LPR, float* red) {
  int w = LPR < 32 ? LPR : 32;
  for (int o = w >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (LPR <= 32) return v;
  int tid = threadIdx.x;
  __syncthreads();
  if ((tid & 31) == 0) red[tid >> 5] = v;
  __syncthreads();
  int wpg = LPR >> 5;
  int first = (tid / LPR) * wpg;
  float s = 0.f;
  for (int i = 0; i < wpg; ++i) s += red[first + i];
  return s;
}

}  // namespace csa
