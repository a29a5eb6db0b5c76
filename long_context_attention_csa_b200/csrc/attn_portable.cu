// Shared-KV MQA (sparse CSA and dense HCA) on CUDA cores, float32 arithmetic
// with an exact running-maximum softmax.
//
// Method: page "DeepSeek-V4：迈向高效百万 Token 上下文智能", §3.3 -- MQA in which
// each compressed entry is both key and value, over the top-k entries (CSA) or
// all visible entries (HCA); RMSNorm on the query; partial RoPE on the query
// and the output rotated again at position -i; a sliding window of
// uncompressed rows.  Page "DeepSeek V4 完整技术报告", section "混合注意力：CSA +
// HCA": a learnable per-head sink logit lets the total weight fall below one.
// Readings: one joint softmax over sink, selected entries and window rows; the
// sink contributes to the denominator only; the window holds positions
// p-n_win+1 .. p.
//
// Portable path for the float32 workload and for shapes outside the
// tensor-core kernel.  One CTA per (query row, group of 8 heads, sequence);
// warp w owns head w of the group.  Keys are staged 32 at a time in shared
// memory (rows padded to c+1 floats so that lane j reading key j is
// conflict-free); lane j scores key j, the warp runs the online softmax, then
// lane l accumulates output dims l, l+32, ... .
#include <cuda_fp8.h>

#include "common.cuh"
#include "internal.h"

namespace csa {

namespace {

// Element e of a mixed entry record (dims [0, c-r) as E4M3 codes with a
// UE8M0 exponent per 32 dims, dims [c-r, c) as bf16): exact in float.
__device__ __forceinline__ float mixed_elem(const uint8_t* rec, int e, int c, int r) {
  const int cq = c - r;
  if (e >= cq) return __bfloat162float(reinterpret_cast<const bf16*>(rec + cq)[e - cq]);
  const __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)rec[e], __NV_E4M3);
  return ldexpf(__half2float(__half(h)), (int)rec[cq + 2 * r + e / 32] - 127);
}

constexpr int kHG = 8;     // heads per CTA (one warp each)
constexpr int kKT = 32;    // keys per tile (one per lane)
constexpr int kMaxE = 16;  // output dims per lane: c <= 512

__device__ __forceinline__ int64_t visible_count(int64_t pos, int m, int64_t N) {
  if (pos < 0) return 0;
  int64_t v = (pos + 1) / m;
  return v < N ? v : N;
}

template <typename T>
__global__ void __launch_bounds__(256) attn_portable_kernel(AttnParams p) {
  extern __shared__ float sm[];
  const int c = p.f.c;
  const int cs = c + 1;                 // padded key row stride
  float* qh = sm;                       // [kHG][c]
  float* K = qh + kHG * c;              // [kKT][c+1]
  float* P = K + kKT * cs;              // [kHG][kKT]
  int64_t* koff = reinterpret_cast<int64_t*>(P + kHG * kKT);  // [kKT] element offsets (-1 = none)

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t t = blockIdx.x, b = blockIdx.z;
  const int h = blockIdx.y * kHG + warp;
  const int64_t row = b * p.Tq + t;
  const int64_t pos = p.q_pos ? p.q_pos[row] : t;
  const int64_t wp0 = p.win_pos0 ? p.win_pos0[b] : 0;

  // key list: [entry part | window part]
  int64_t n_ent;
  if (p.sparse) n_ent = p.k;
  else n_ent = visible_count(pos, p.m_dense, p.N);
  int64_t jlo = pos - p.n_win + 1;
  if (jlo < wp0) jlo = wp0;
  int64_t jhi = pos;
  if (jhi > wp0 + p.Tw - 1) jhi = wp0 + p.Tw - 1;
  const int64_t n_win = jhi >= jlo ? jhi - jlo + 1 : 0;
  const int64_t n_keys = n_ent + n_win;

  const T* ent = static_cast<const T*>(p.entries) + b * p.N * c;
  // mixed records: the batch offset is added per access (records are not c wide)
  const uint8_t* entm = p.mixed ? static_cast<const uint8_t*>(p.entries) : nullptr;
  const T* win = static_cast<const T*>(p.win) + b * p.Tw * c;
  const float scale = p.scale > 0.f ? p.scale : rsqrtf((float)c);

  // q^ = RoPE_pos(RMSNorm(q)) for this warp's head
  if (h < p.H) {
    const T* q = static_cast<const T*>(p.q) + (row * p.H + h) * c;
    float ss = 0.f;
    for (int e = lane; e < c; e += 32) {
      float x = to_float(q[e]);
      qh[warp * c + e] = x;
      ss += x * x;
    }
    ss = warp_sum(ss);
    float inv = (p.f.flags & CSA_F_NO_NORM) ? 1.f : rsqrtf(ss / (float)c + p.f.eps);
    __syncwarp();
    for (int e2 = 2 * lane; e2 < c; e2 += 64) {
      float x0 = qh[warp * c + e2] * inv, x1 = qh[warp * c + e2 + 1] * inv;
      if (!(p.f.flags & CSA_F_NO_ROPE) && e2 >= c - p.f.r) {
        float co, si;
        rope_cos_sin(pos, (e2 - (c - p.f.r)) >> 1, p.f.r, p.f.base, &co, &si);
        float y0 = x0 * co - x1 * si, y1 = x0 * si + x1 * co;
        x0 = y0;
        x1 = y1;
      }
      qh[warp * c + e2] = x0;
      qh[warp * c + e2 + 1] = x1;
    }
  }

  float o[kMaxE];
#pragma unroll
  for (int i = 0; i < kMaxE; ++i) o[i] = 0.f;
  float run_max = -INFINITY, den = 0.f;
  const int nE = c / 32;

  for (int64_t k0 = 0; k0 < n_keys; k0 += kKT) {
    __syncthreads();
    if (threadIdx.x < kKT) {
      int64_t i = k0 + threadIdx.x;
      int64_t off = -1;
      if (i < n_ent) {
        if (p.sparse) {
          int32_t s = p.idx[row * p.k + i];
          if (s >= 0 && s < p.N) off = (int64_t)s * c;
          else if (s != -1) report(p.status, CSA_DEV_BAD_INDEX, (unsigned)i);
        } else {
          off = i * c;
        }
      } else if (i < n_keys) {
        off = -2 - (jlo - wp0 + (i - n_ent)) * c;  // window row, encoded negative
      }
      koff[threadIdx.x] = off;
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < kKT * c; idx += blockDim.x) {
      int j = idx / c, e = idx - j * c;
      int64_t off = koff[j];
      float v = 0.f;
      if (off >= 0) {
        v = entm ? mixed_elem(entm + (off / c) * p.rec_bytes + (int64_t)b * p.N * p.rec_bytes, e,
                              c, p.f.r)
                 : to_float(ent[off + e]);
      } else if (off <= -2) {
        v = to_float(win[(-2 - off) + e]);
      }
      K[j * cs + e] = v;
    }
    __syncthreads();
    if (h < p.H) {
      const bool valid = koff[lane] != -1 && (k0 + lane) < n_keys;
      float d = 0.f;
      const float* kr = K + lane * cs;
      const float* qr = qh + warp * c;
      for (int e = 0; e < c; ++e) d = fmaf(qr[e], kr[e], d);
      float l = valid ? d * scale : -INFINITY;
      float tmax = l;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, off));
      float new_max = fmaxf(run_max, tmax);
      float pj = 0.f, alpha = 1.f;
      if (new_max != -INFINITY) {
        pj = valid ? expf(l - new_max) : 0.f;
        alpha = run_max == -INFINITY ? 0.f : expf(run_max - new_max);
        run_max = new_max;
      }
      den = den * alpha + warp_sum(pj);
      P[warp * kKT + lane] = pj;
      __syncwarp();
#pragma unroll
      for (int i = 0; i < kMaxE; ++i) {
        if (i < nE) {
          float a = o[i] * alpha;
          const int e = lane + 32 * i;
          for (int j = 0; j < kKT; ++j) a = fmaf(P[warp * kKT + j], K[j * cs + e], a);
          o[i] = a;
        }
      }
    }
  }

  if (h < p.H) {
    float zs = p.sink ? p.sink[h] : -INFINITY;
    float M = fmaxf(run_max, zs);
    float fo = 0.f;
    if (M != -INFINITY) {
      float a = run_max == -INFINITY ? 0.f : expf(run_max - M);
      float dt = den * a + (zs == -INFINITY ? 0.f : expf(zs - M));
      fo = dt > 0.f ? a / dt : 0.f;
    }
    T* out = static_cast<T*>(p.out) + (row * p.H + h) * c;
#pragma unroll
    for (int i = 0; i < kMaxE; ++i) {
      if (i < nE) {
        const int e = lane + 32 * i;
        float v = o[i] * fo;
        float partner = __shfl_xor_sync(0xffffffffu, v, 1);
        if (!(p.f.flags & CSA_F_NO_ROPE) && e >= c - p.f.r) {
          float co, si;
          rope_cos_sin(-pos, (e - (c - p.f.r)) >> 1, p.f.r, p.f.base, &co, &si);
          // pair (x0, x1) = even lane, odd lane
          v = (lane & 1) ? (partner * si + v * co) : (v * co - partner * si);
        }
        if constexpr (sizeof(T) == 4) {
          out[e] = v;
        } else {
          out[e] = __float2bfloat16_rn(v);
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_attn_portable(int dtype, const AttnParams& p, cudaStream_t stream) {
  if (p.B == 0 || p.Tq == 0) return cudaSuccess;
  const int c = p.f.c;
  dim3 grid((unsigned)p.Tq, (unsigned)((p.H + kHG - 1) / kHG), (unsigned)p.B);
  size_t smem = sizeof(float) * ((size_t)kHG * c + (size_t)kKT * (c + 1) + kHG * kKT) +
                sizeof(int64_t) * kKT;
  if (dtype == CSA_BF16) {
    cudaFuncSetAttribute(attn_portable_kernel<bf16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    attn_portable_kernel<bf16><<<grid, 256, smem, stream>>>(p);
  } else {
    cudaFuncSetAttribute(attn_portable_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    attn_portable_kernel<float><<<grid, 256, smem, stream>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace csa
