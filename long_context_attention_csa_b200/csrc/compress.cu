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
// Design (HBM-bound streaming kernel): one CTA per (entry, sequence).  Its
// threads form G slot-groups of LPR = c/VEC lanes; lane l owns channels
// [l*VEC, l*VEC+VEC) (one 16-byte vector), so the per-channel softmax over the
// slots needs no shuffles: each lane runs an online softmax over the slots of
// its group with one exp2 per element, the G partial states merge through
// shared memory, and the only cross-lane step is the sum of squares of the
// RMSNorm.  Token rows are read once with streaming (evict-first) 16-byte
// loads, U slots in flight per lane.  The window rows of the entry's own block
// (and, in one extra CTA, the tail tokens that form no entry) are normalised
// and rotated in the same launch.
#include "common.cuh"
#include "internal.h"

namespace csa {

namespace {

constexpr int kSlotBatch = 4;  // slots loaded before they are folded in
constexpr float kLog2e = 1.4426950408889634f;

template <typename T>
__global__ void __launch_bounds__(256) compress_kernel(CompressParams p) {
  constexpr int VEC = VecOf<T>::N;
  const int c = p.f.c;
  const int LPR = c / VEC;
  const int tid = threadIdx.x;
  const int g = tid / LPR;
  const int ch0 = (tid % LPR) * VEC;
  const int64_t b = blockIdx.y;
  const int64_t s = blockIdx.x;

  extern __shared__ float smem[];
  float* red = smem;        // 32 floats for group_sum
  float* cmb = smem + 32;   // [G][3][c] partial softmax states

  const T* kva = static_cast<const T*>(p.kv_a) + b * p.T * c;
  const T* kvb = p.overlap ? static_cast<const T*>(p.kv_b) + b * p.T * c : nullptr;
  const T* za = static_cast<const T*>(p.z_a) + b * p.T * p.z_cols;
  const T* zb = p.overlap ? static_cast<const T*>(p.z_b) + b * p.T * p.z_cols : nullptr;

  if (s < p.n_entries) {
    const int na = p.m;
    const int ns = na + ((p.overlap && s >= 1) ? p.m : 0);
    float mx[VEC], den[VEC], acc[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) { mx[e] = -INFINITY; den[e] = 0.f; acc[e] = 0.f; }

    for (int j0 = g; j0 < ns; j0 += p.G * kSlotBatch) {
      float v[kSlotBatch][VEC], z[kSlotBatch][VEC];
      bool ok[kSlotBatch];
#pragma unroll
      for (int u = 0; u < kSlotBatch; ++u) {
        int j = j0 + u * p.G;
        ok[u] = j < ns;
        if (ok[u]) {
          const T* row;
          const T* zrow;
          if (j < na) {  // group a: the entry's own block
            int64_t tok = (int64_t)p.m * s + j;
            row = kva + tok * c;
            zrow = za + tok * p.z_cols;
          } else {       // group b: the previous block (overlap)
            int64_t tok = (int64_t)p.m * (s - 1) + (j - na);
            row = kvb + tok * c;
            zrow = zb + tok * p.z_cols;
          }
          load_vec_stream(row + ch0, v[u]);
          if (p.z_cols == 1) {
            float zz = to_float(zrow[0]);
#pragma unroll
            for (int e = 0; e < VEC; ++e) z[u][e] = zz;
          } else {
            load_vec_stream(zrow + ch0, z[u]);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kSlotBatch; ++u) {
        if (!ok[u]) continue;
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          // online softmax in base 2, one exp2 per element
          float zl = z[u][e] * kLog2e;
          float d = zl - mx[e];
          float t = exp2f(-fabsf(d));
          bool gt = d > 0.f;
          float so = gt ? t : 1.f;
          float sn = gt ? 1.f : t;
          den[e] = den[e] * so + sn;
          acc[e] = acc[e] * so + sn * v[u][e];
          mx[e] = fmaxf(mx[e], zl);
        }
      }
    }

    if (p.G > 1) {  // merge the G partial states into group 0
      float* mine = cmb + (size_t)g * 3 * c;
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        mine[ch0 + e] = mx[e];
        mine[c + ch0 + e] = den[e];
        mine[2 * c + ch0 + e] = acc[e];
      }
      __syncthreads();
      if (g == 0) {
        for (int gg = 1; gg < p.G; ++gg) {
          const float* o = cmb + (size_t)gg * 3 * c;
#pragma unroll
          for (int e = 0; e < VEC; ++e) {
            float m2 = o[ch0 + e];
            if (m2 == -INFINITY) continue;
            float M = fmaxf(mx[e], m2);
            float a1 = exp2f(mx[e] - M), a2 = exp2f(m2 - M);
            den[e] = den[e] * a1 + o[c + ch0 + e] * a2;
            acc[e] = acc[e] * a1 + o[2 * c + ch0 + e] * a2;
            mx[e] = M;
          }
        }
      }
    }

    float val[VEC];
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      val[e] = acc[e] / den[e];
      ss += val[e] * val[e];
    }
    ss = group_sum(ss, LPR, red);
    if (g == 0) {
      if (!(p.f.flags & CSA_F_NO_NORM)) {
        float inv = rsqrtf(ss / (float)c + p.f.eps);
#pragma unroll
        for (int e = 0; e < VEC; ++e) val[e] *= inv;
      }
      if (!(p.f.flags & CSA_F_NO_ROPE)) rope_slice<VEC>(val, ch0, p.f, p.pos0 + (int64_t)p.m * s);
      T* dst = static_cast<T*>(p.entries) + (b * p.n_entries + s) * c + ch0;
      store_vec(dst, val);
    }
  }

  // window rows of this entry's own block, or of the tail tokens
  if (p.win != nullptr) {
    int64_t r0, r1;
    if (s < p.n_entries) {
      r0 = (int64_t)p.m * s;
      r1 = r0 + p.m;
    } else {
      r0 = (int64_t)p.m * p.n_entries;
      r1 = p.T;
    }
    for (int64_t base = r0; base < r1; base += p.G) {  // uniform trip count
      int64_t row = base + g;
      bool ok = row < r1;
      float v[VEC];
      if (ok) {
        load_vec(kva + row * c + ch0, v);
      } else {
#pragma unroll
        for (int e = 0; e < VEC; ++e) v[e] = 0.f;
      }
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < VEC; ++e) ss += v[e] * v[e];
      ss = group_sum(ss, LPR, red);
      if (ok) {
        if (!(p.f.flags & CSA_F_NO_NORM)) {
          float inv = rsqrtf(ss / (float)c + p.f.eps);
#pragma unroll
          for (int e = 0; e < VEC; ++e) v[e] *= inv;
        }
        if (!(p.f.flags & CSA_F_NO_ROPE)) rope_slice<VEC>(v, ch0, p.f, p.pos0 + row);
        store_vec(static_cast<T*>(p.win) + (b * p.T + row) * c + ch0, v);
      }
    }
  }
}

}  // namespace

cudaError_t launch_compress(int dtype, CompressParams p, int64_t B, cudaStream_t stream) {
  const int vec = dtype == CSA_BF16 ? 8 : 4;
  const int LPR = p.f.c / vec;
  const int ns_max = p.overlap ? 2 * p.m : p.m;
  int G = 256 / LPR;
  if (G < 1) G = 1;
  if (G > ns_max) G = ns_max;
  if (G > 32) G = 32;
  while (G > 1 && LPR * G > 256) G >>= 1;
  if (LPR < 32) {  // whole warps only: round G up to a multiple of 32/LPR
    int q = 32 / LPR;
    G = ((G + q - 1) / q) * q;
  }
  p.G = G;
  dim3 grid((unsigned)(p.n_entries + (p.win ? 1 : 0)), (unsigned)B);
  dim3 block((unsigned)(LPR * G));
  size_t smem = sizeof(float) * (32 + (G > 1 ? (size_t)3 * G * p.f.c : 0));
  if (grid.x == 0 || B == 0) return cudaSuccess;
  if (dtype == CSA_BF16) {
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(compress_kernel<bf16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
    compress_kernel<bf16><<<grid, block, smem, stream>>>(p);
  } else {
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(compress_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
    compress_kernel<float><<<grid, block, smem, stream>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace csa
