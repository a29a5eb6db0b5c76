// Softmax-gated KV compression (CSA overlapped, rate 1/m; HCA non-overlapped,
// rate 1/m') with the fused RMSNorm + partial-RoPE epilogue and the optional
// window-row output.
//
// Method: page "DeepSeek-V4：迈向高效百万 Token 上下文智能", §3.3 -- two groups
// of per-token KV and compression weights, a softmax over the 2m slots of an
// entry and a weighted sum, the group ranges overlapping so the rate is
// exactly 1/m; HCA uses m' >> m with no overlap; RMSNorm on compressed entries
// and RoPE on their last dims.
//
// Design (HBM-bound streaming kernel): G warps per entry (one for CSA's 2m
// slots, four for HCA's m' slots); lane l owns channels [l*CPL, l*CPL + CPL),
// CPL = c/32, so a warp covers a whole row with one coalesced access and the
// per-channel softmax over the slots needs no cross-lane step (online, one
// exp2 per element).  The only cross-lane operations are the RMSNorm sums of
// squares, done with warp shuffles.  Window rows (the entry's own block, plus
// the tail tokens that form no entry) are normalised and rotated from the
// registers the pooling loaded them into.  Token rows are read exactly once.
#include "common.cuh"
#include "internal.h"

namespace csa {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr double kTwoPi = 6.283185307179586476925286766559;
constexpr int kWarps = 8;   // warps per CTA

// cos/sin of pos * theta: the angle is formed and reduced modulo 2*pi in
// double precision (positions up to 2^20 keep full accuracy), then evaluated
// in single precision on [-pi, pi].
__device__ __forceinline__ void rope_angle(int64_t pos, double theta, float* cs, float* sn) {
  double ang = (double)pos * theta;
  ang -= kTwoPi * rint(ang * (1.0 / kTwoPi));
  sincosf((float)ang, sn, cs);
}

// Load CPL consecutive elements as float (CPL * sizeof(T) bytes, aligned).
template <typename T, int CPL>
__device__ __forceinline__ void load_lane(const T* p, float* o) {
  if constexpr (sizeof(T) == 2) {
    static_assert(CPL % 2 == 0, "bf16 lanes hold pairs");
    if constexpr (CPL >= 8) {
#pragma unroll
      for (int v = 0; v < CPL / 8; ++v) {
        const uint4 u = __ldcs(reinterpret_cast<const uint4*>(p) + v);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          o[8 * v + 2 * i] = bf16_bits_to_float(w[i] & 0xffffu);
          o[8 * v + 2 * i + 1] = bf16_bits_to_float(w[i] >> 16);
        }
      }
    } else {
#pragma unroll
      for (int v = 0; v < CPL / 2; ++v) {
        const uint32_t w = __ldcs(reinterpret_cast<const unsigned int*>(p) + v);
        o[2 * v] = bf16_bits_to_float(w & 0xffffu);
        o[2 * v + 1] = bf16_bits_to_float(w >> 16);
      }
    }
  } else {
    if constexpr (CPL >= 4) {
#pragma unroll
      for (int v = 0; v < CPL / 4; ++v) {
        const float4 u = __ldcs(reinterpret_cast<const float4*>(p) + v);
        o[4 * v] = u.x; o[4 * v + 1] = u.y; o[4 * v + 2] = u.z; o[4 * v + 3] = u.w;
      }
    } else {
#pragma unroll
      for (int v = 0; v < CPL / 2; ++v) {
        const float2 u = __ldcs(reinterpret_cast<const float2*>(p) + v);
        o[2 * v] = u.x; o[2 * v + 1] = u.y;
      }
    }
  }
}

template <typename T, int CPL>
__device__ __forceinline__ void store_lane(T* p, const float* v) {
  if constexpr (sizeof(T) == 2) {
    if constexpr (CPL >= 8) {
#pragma unroll
      for (int i = 0; i < CPL / 8; ++i)
        reinterpret_cast<uint4*>(p)[i] =
            make_uint4(pack_bf16x2(v[8 * i], v[8 * i + 1]), pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                       pack_bf16x2(v[8 * i + 4], v[8 * i + 5]), pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
    } else {
#pragma unroll
      for (int i = 0; i < CPL / 2; ++i)
        reinterpret_cast<unsigned int*>(p)[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
    }
  } else {
    if constexpr (CPL >= 4) {
#pragma unroll
      for (int i = 0; i < CPL / 4; ++i)
        reinterpret_cast<float4*>(p)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    } else {
#pragma unroll
      for (int i = 0; i < CPL / 2; ++i)
        reinterpret_cast<float2*>(p)[i] = make_float2(v[2 * i], v[2 * i + 1]);
    }
  }
}

// RMSNorm over the row held by the warp (sum of squares by shuffles), then
// RoPE of the lane's pairs that fall in the last r dims at position pos.
template <int CPL>
__device__ __forceinline__ void norm_rope_row(float* v, int lane, const Fmt& f, int64_t pos,
                                              const double* theta) {
  if (!(f.flags & CSA_F_NO_NORM)) {
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < CPL; ++e) ss = fmaf(v[e], v[e], ss);
    ss = warp_sum(ss);
    const float inv = rsqrtf(ss / (float)f.c + f.eps);
#pragma unroll
    for (int e = 0; e < CPL; ++e) v[e] *= inv;
  }
  if (!(f.flags & CSA_F_NO_ROPE)) {
    const int ch0 = lane * CPL, d0 = f.c - f.r;
    if (ch0 + CPL > d0) {
#pragma unroll
      for (int e = 0; e < CPL; e += 2) {
        const int ch = ch0 + e;
        if (ch >= d0) {
          float cs, sn;
          rope_angle(pos, theta[(ch - d0) >> 1], &cs, &sn);
          const float x0 = v[e], x1 = v[e + 1];
          v[e] = x0 * cs - x1 * sn;
          v[e + 1] = x0 * sn + x1 * cs;
        }
      }
    }
  }
}

template <typename T, int CPL>
__global__ void __launch_bounds__(kWarps * 32) compress_kernel(CompressParams p) {
  extern __shared__ float smem[];
  double* theta = reinterpret_cast<double*>(smem);        // [r/2] RoPE frequencies
  float* cmb = smem + 2 * 256;                             // [kWarps][3][c] partial states
  const int c = p.f.c;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.G;                  // warps per entry
  const int epc = kWarps / G;         // entries per CTA
  const int64_t b = blockIdx.y;
  for (int i = threadIdx.x; i < (p.f.r >> 1); i += blockDim.x)
    theta[i] = pow((double)p.f.base, -2.0 * (double)i / (double)p.f.r);
  __syncthreads();

  const T* kva = static_cast<const T*>(p.kv_a) + b * p.T * c;
  const T* kvb = p.overlap ? static_cast<const T*>(p.kv_b) + b * p.T * c : nullptr;
  const T* za = static_cast<const T*>(p.z_a) + b * p.T * p.z_cols;
  const T* zb = p.overlap ? static_cast<const T*>(p.z_b) + b * p.T * p.z_cols : nullptr;
  T* win = static_cast<T*>(p.win);
  const int ch0 = lane * CPL;
  const int64_t n_entry_ctas = (p.n_entries + epc - 1) / epc;

  if ((int64_t)blockIdx.x >= n_entry_ctas) {
    // tail tokens: window rows only, one warp per row
    for (int64_t row = p.n_entries * p.m + (int64_t)(blockIdx.x - n_entry_ctas) * kWarps + warp;
         row < p.T; row += (int64_t)(gridDim.x - n_entry_ctas) * kWarps) {
      float v[CPL];
      load_lane<T, CPL>(kva + row * c + ch0, v);
      norm_rope_row<CPL>(v, lane, p.f, p.pos0 + row, theta);
      store_lane<T, CPL>(win + (b * p.T + row) * c + ch0, v);
    }
    return;
  }

  const int e_loc = warp / G, g = warp % G;
  const int64_t s = (int64_t)blockIdx.x * epc + e_loc;
  const bool have = s < p.n_entries;   // warp-uniform
  float mx[CPL], den[CPL], acc[CPL];
#pragma unroll
  for (int e = 0; e < CPL; ++e) { mx[e] = -INFINITY; den[e] = 0.f; acc[e] = 0.f; }

  if (have) {
    const int na = p.m;
    const int ns = na + ((p.overlap && s >= 1) ? p.m : 0);
    constexpr int U = CPL >= 16 ? 2 : 4;   // slots loaded before they are folded in
    for (int j0 = g; j0 < ns; j0 += G * U) {
      float v[U][CPL], z[U][CPL];
      bool ok[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = j0 + u * G;
        ok[u] = j < ns;
        if (ok[u]) {
          const T* row;
          const T* zrow;
          if (j < na) {  // group a: the entry's own block
            const int64_t tok = (int64_t)p.m * s + j;
            row = kva + tok * c;
            zrow = za + tok * p.z_cols;
          } else {       // group b: the previous block (overlap)
            const int64_t tok = (int64_t)p.m * (s - 1) + (j - na);
            row = kvb + tok * c;
            zrow = zb + tok * p.z_cols;
          }
          load_lane<T, CPL>(row + ch0, v[u]);
          if (p.z_cols == 1) {
            const float zz = to_float(zrow[0]);
#pragma unroll
            for (int e = 0; e < CPL; ++e) z[u][e] = zz;
          } else {
            load_lane<T, CPL>(zrow + ch0, z[u]);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (!ok[u]) continue;
#pragma unroll
        for (int e = 0; e < CPL; ++e) {
          // online softmax in base 2, one exp2 per element
          const float zl = z[u][e] * kLog2e;
          const float d = zl - mx[e];
          const float t = exp2f(-fabsf(d));
          const bool gt = d > 0.f;
          const float so = gt ? t : 1.f;
          const float sn = gt ? 1.f : t;
          den[e] = den[e] * so + sn;
          acc[e] = acc[e] * so + sn * v[u][e];
          mx[e] = fmaxf(mx[e], zl);
        }
        // a token row of the entry's own block is also a window row
        const int j = j0 + u * G;
        if (win != nullptr && j < na) {
          const int64_t tok = (int64_t)p.m * s + j;
          float wv[CPL];
#pragma unroll
          for (int e = 0; e < CPL; ++e) wv[e] = v[u][e];
          norm_rope_row<CPL>(wv, lane, p.f, p.pos0 + tok, theta);
          store_lane<T, CPL>(win + (b * p.T + tok) * c + ch0, wv);
        }
      }
    }
  }

  if (G > 1) {  // merge the G partial states of each entry (shared memory)
    float* mine = cmb + (size_t)warp * 3 * c;
#pragma unroll
    for (int e = 0; e < CPL; ++e) {
      mine[ch0 + e] = mx[e];
      mine[c + ch0 + e] = den[e];
      mine[2 * c + ch0 + e] = acc[e];
    }
    __syncthreads();
    if (g != 0 || !have) return;
    for (int gg = 1; gg < G; ++gg) {
      const float* o = cmb + (size_t)(warp + gg) * 3 * c;
#pragma unroll
      for (int e = 0; e < CPL; ++e) {
        const float m2 = o[ch0 + e];
        if (m2 == -INFINITY) continue;
        const float M = fmaxf(mx[e], m2);
        const float a1 = exp2f(mx[e] - M), a2 = exp2f(m2 - M);
        den[e] = den[e] * a1 + o[c + ch0 + e] * a2;
        acc[e] = acc[e] * a1 + o[2 * c + ch0 + e] * a2;
        mx[e] = M;
      }
    }
  } else if (!have) {
    return;
  }

  float val[CPL];
#pragma unroll
  for (int e = 0; e < CPL; ++e) val[e] = acc[e] / den[e];
  norm_rope_row<CPL>(val, lane, p.f, p.pos0 + (int64_t)p.m * s, theta);
  store_lane<T, CPL>(static_cast<T*>(p.entries) + (b * p.n_entries + s) * c + ch0, val);
}

template <typename T, int CPL>
cudaError_t launch_t(CompressParams p, int64_t B, cudaStream_t stream) {
  const int epc = kWarps / p.G;
  const int64_t n_entry_ctas = (p.n_entries + epc - 1) / epc;
  const int64_t tail = p.T - p.n_entries * p.m;
  const int64_t tail_ctas = (p.win != nullptr && tail > 0) ? (tail + kWarps - 1) / kWarps : 0;
  dim3 grid((unsigned)(n_entry_ctas + tail_ctas), (unsigned)B);
  size_t smem = sizeof(float) * (2 * 256 + (p.G > 1 ? (size_t)kWarps * 3 * p.f.c : 0));
  if (grid.x == 0 || B == 0) return cudaSuccess;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(compress_kernel<T, CPL>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  compress_kernel<T, CPL><<<grid, kWarps * 32, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_compress(int dtype, CompressParams p, int64_t B, cudaStream_t stream) {
  const int ns_max = p.overlap ? 2 * p.m : p.m;
  p.G = ns_max >= 32 ? 4 : 1;   // long slot lists are shared by four warps
  const int cpl = p.f.c / 32;
  if (dtype == CSA_BF16) {
    switch (cpl) {
      case 2: return launch_t<bf16, 2>(p, B, stream);
      case 4: return launch_t<bf16, 4>(p, B, stream);
      case 8: return launch_t<bf16, 8>(p, B, stream);
      case 16: return launch_t<bf16, 16>(p, B, stream);
    }
  } else {
    switch (cpl) {
      case 2: return launch_t<float, 2>(p, B, stream);
      case 4: return launch_t<float, 4>(p, B, stream);
      case 8: return launch_t<float, 8>(p, B, stream);
      case 16: return launch_t<float, 16>(p, B, stream);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace csa
