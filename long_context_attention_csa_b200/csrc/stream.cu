// Streaming compression for decode: one new token per sequence per call, a
// per-sequence tail buffer in HBM, and a compressed entry emitted when the
// token completes a block.
//
// Method: page "DeepSeek-V4：迈向高效百万 Token 上下文智能", §3.3 -- the CSA
// entry of block s pools the block's own group-a rows and the previous
// block's group-b rows under a per-channel softmax over their 2m logits (HCA:
// the block's m' rows, no overlap), then RMSNorm and RoPE at the entry's
// position.  Page "DeepSeek-V4 梗概", the inference-infrastructure table, row
// "Tail buffer": tokens of a block that is not yet complete wait in a tail
// buffer until the block closes.
//
// State of one sequence (`stride` bytes, caller-owned, zero-filled before the
// sequence's first token):
//   [0, 8)    int64 t: tokens appended so far (the next token is token t)
//   [16, ..)  rows in the tensors' dtype:
//             a  [m][c]       group-a rows of the current block
//             b  [2][m][c]    group-b rows of the current and previous block
//                             (CSA only; block s at parity s & 1)
//             za [m][z_cols], zb [2][m][z_cols]   their logits
// Token t lands in slot j = t mod m of block s = t / m; its window row
// RoPE_{pos0+t}(RMSNorm(kv_a)) goes to win_out; when j == m - 1 the entry s
// is pooled from the tail buffer and written to entries[b, s].
//
// Design: latency-bound (a few KB per sequence per call; an HCA block's 256 KB
// once every m' tokens), so one CTA per sequence, thread (pair, g) owning
// channels 2 pair, 2 pair + 1 -- a RoPE pair never leaves its thread -- and
// slot group g of G (long HCA slot lists are split four ways and the partial
// softmax states merged in shared memory).
#include "common.cuh"
#include "internal.h"

namespace csa {

namespace {

constexpr float kLog2e = 1.4426950408889634f;

template <typename T>
__device__ __forceinline__ void load2(const T* p, float& x0, float& x1) {
  if constexpr (sizeof(T) == 2) {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
    x0 = bf16_bits_to_float(w & 0xffffu);
    x1 = bf16_bits_to_float(w >> 16);
  } else {
    const float2 v = *reinterpret_cast<const float2*>(p);
    x0 = v.x;
    x1 = v.y;
  }
}

template <typename T>
__device__ __forceinline__ void store2(T* p, float x0, float x1) {
  if constexpr (sizeof(T) == 2) {
    *reinterpret_cast<uint32_t*>(p) = pack_bf16x2(x0, x1);
  } else {
    *reinterpret_cast<float2*>(p) = make_float2(x0, x1);
  }
}

// Copies two consecutive elements without conversion (exact in either dtype).
template <typename T>
__device__ __forceinline__ void copy2(T* dst, const T* src) {
  if constexpr (sizeof(T) == 2) {
    *reinterpret_cast<uint32_t*>(dst) = *reinterpret_cast<const uint32_t*>(src);
  } else {
    *reinterpret_cast<float2*>(dst) = *reinterpret_cast<const float2*>(src);
  }
}

// Sum over the whole CTA (every thread calls it; `red` holds 32 floats).
__device__ __forceinline__ float cta_sum(float v, float* red) {
  v = warp_sum(v);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float s = 0.f;
  const int nw = (int)(blockDim.x >> 5);
  for (int i = 0; i < nw; ++i) s += red[i];
  return s;
}

// RMSNorm over the c channels held by the pair threads (others pass active =
// false and contribute nothing), then RoPE of the pair at position pos.
__device__ __forceinline__ void norm_rope_pair(float& x0, float& x1, bool active, int pair,
                                               const StreamParams& p, int64_t pos, float* red) {
  if (!(p.f.flags & CSA_F_NO_NORM)) {
    const float ss = cta_sum(active ? fmaf(x0, x0, x1 * x1) : 0.f, red);
    const float inv = rsqrtf(ss / (float)p.f.c + p.f.eps);
    x0 *= inv;
    x1 *= inv;
  }
  const int ch = 2 * pair, d0 = p.f.c - p.f.r;
  if (active && !(p.f.flags & CSA_F_NO_ROPE) && ch >= d0) {
    float cs, sn;
    rope_cos_sin_theta(pos, p.theta[(ch - d0) >> 1], &cs, &sn);
    const float y0 = x0 * cs - x1 * sn, y1 = x0 * sn + x1 * cs;
    x0 = y0;
    x1 = y1;
  }
}

// One slot of the entry's softmax: (value pair, logit pair) of token row
// `row` / logits `zrow` at this thread's channels.
template <typename T>
__device__ __forceinline__ void load_slot(const T* row, const T* zrow, int zc, int ch, float& v0,
                                          float& v1, float& z0, float& z1) {
  load2(row + ch, v0, v1);
  if (zc == 1) {
    z0 = z1 = to_float(zrow[0]);
  } else {
    load2(zrow + ch, z0, z1);
  }
}

// Latency chain: the token count, then in one round every load the call
// needs (the token's own rows; on a block's last token every other slot of
// the entry, which earlier calls stored -- the token's own slot comes from
// its inputs, so nothing waits for this call's stores), then the arithmetic.
template <typename T>
__global__ void __launch_bounds__(1024) stream_append_kernel(const StreamParams p) {
  __shared__ float red[32];
  extern __shared__ float part[];      // [G][c/2][6] partial softmax states (G > 1)
  const int c = p.f.c, m = p.m, zc = p.z_cols;
  const int np = c / 2;
  const int pair = (int)threadIdx.x % np, g = (int)threadIdx.x / np;
  const int G = (int)blockDim.x / np;
  const int ch = 2 * pair;
  const int64_t b = blockIdx.x;
  const T* __restrict__ ka = static_cast<const T*>(p.kv_a) + b * c;
  const T* __restrict__ za = static_cast<const T*>(p.z_a) + b * zc;
  const T* __restrict__ kb = p.overlap ? static_cast<const T*>(p.kv_b) + b * c : nullptr;
  const T* __restrict__ zb = p.overlap ? static_cast<const T*>(p.z_b) + b * zc : nullptr;
  // the token's rows (independent of the state), then the token count
  float x0 = 0.f, x1 = 0.f, az0 = 0.f, az1 = 0.f;
  if (g == 0) load_slot(ka, za, zc, ch, x0, x1, az0, az1);
  uint8_t* st = p.state + (size_t)b * p.stride;
  const int64_t t = *reinterpret_cast<const volatile int64_t*>(st);
  if (t < 0) {   // a corrupt state: nothing of this sequence is touched
    if (threadIdx.x == 0) report(p.status, CSA_DEV_STREAM, (unsigned)b);
    return;
  }
  const int j = (int)(t % m);
  const int64_t s = t / m;
  const int par = (int)(s & 1);
  T* ra = reinterpret_cast<T*>(st + 16);
  T* rb = ra + (size_t)m * c;
  T* rza = rb + (p.overlap ? (size_t)2 * m * c : 0);
  T* rzb = rza + (size_t)m * zc;
  const bool closes = j == m - 1;
  const int ns = closes ? m + ((p.overlap && s >= 1) ? m : 0) : 0;

  // the entry's slots: a(s) (slot j from the inputs), then b(s - 1) for CSA
  constexpr int U = 8;   // slots a thread holds at once
  float v0[U], v1[U], z0[U], z1[U];
  auto load_batch = [&](int i0) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = i0 + u * G;
      if (i < ns) {
        if (i == j)
          load_slot(ka, za, zc, ch, v0[u], v1[u], z0[u], z1[u]);
        else if (i < m)
          load_slot(ra + (size_t)i * c, rza + (size_t)i * zc, zc, ch, v0[u], v1[u], z0[u], z1[u]);
        else
          load_slot(rb + ((size_t)(par ^ 1) * m + (i - m)) * c,
                    rzb + ((size_t)(par ^ 1) * m + (i - m)) * zc, zc, ch, v0[u], v1[u], z0[u],
                    z1[u]);
      }
    }
  };
  if (closes) load_batch(g);

  // 1. this token's rows into the tail buffer (exact copies), window row
  if (g == 0) {
    copy2(ra + (size_t)j * c + ch, ka + ch);
    if (zc == 1) {
      if (pair == 0) rza[j] = za[0];
    } else {
      copy2(rza + (size_t)j * zc + ch, za + ch);
    }
    if (p.overlap) {
      copy2(rb + ((size_t)par * m + j) * c + ch, kb + ch);
      if (zc == 1) {
        if (pair == 0) rzb[par * m + j] = zb[0];
      } else {
        copy2(rzb + ((size_t)par * m + j) * zc + ch, zb + ch);
      }
    }
  }
  if (p.win != nullptr) {   // uniform: every thread takes the reduction
    norm_rope_pair(x0, x1, g == 0, pair, p, p.pos0 + t, red);
    if (g == 0) store2(static_cast<T*>(p.win) + b * c + ch, x0, x1);
  }
  if (!closes) {
    __syncthreads();   // every thread has read the count
    if (threadIdx.x == 0) *reinterpret_cast<int64_t*>(st) = t + 1;
    return;
  }

  // 2. the token completes block s: pool the slots (online softmax in base 2)
  float mx0 = -INFINITY, mx1 = -INFINITY, d0 = 0.f, d1 = 0.f, a0 = 0.f, a1 = 0.f;
  for (int i0 = g; i0 < ns; i0 += G * U) {
    if (i0 != g) load_batch(i0);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (i0 + u * G >= ns) break;
      const float l0 = z0[u] * kLog2e, l1 = z1[u] * kLog2e;
      const float n0 = fmaxf(mx0, l0), n1 = fmaxf(mx1, l1);
      const float s0 = exp2f(mx0 - n0), s1 = exp2f(mx1 - n1);
      const float e0 = exp2f(l0 - n0), e1 = exp2f(l1 - n1);
      d0 = d0 * s0 + e0;
      d1 = d1 * s1 + e1;
      a0 = a0 * s0 + e0 * v0[u];
      a1 = a1 * s1 + e1 * v1[u];
      mx0 = n0;
      mx1 = n1;
    }
  }
  if (G > 1) {   // merge the slot groups' partial states in group order
    float* mine = part + ((size_t)g * np + pair) * 6;
    mine[0] = mx0; mine[1] = mx1; mine[2] = d0; mine[3] = d1; mine[4] = a0; mine[5] = a1;
    __syncthreads();
    if (g == 0) {
      for (int gg = 1; gg < G; ++gg) {
        const float* o = part + ((size_t)gg * np + pair) * 6;
        if (o[0] != -INFINITY) {
          const float n0 = fmaxf(mx0, o[0]);
          const float u0 = exp2f(mx0 - n0), w0 = exp2f(o[0] - n0);
          d0 = d0 * u0 + o[2] * w0;
          a0 = a0 * u0 + o[4] * w0;
          mx0 = n0;
        }
        if (o[1] != -INFINITY) {
          const float n1 = fmaxf(mx1, o[1]);
          const float u1 = exp2f(mx1 - n1), w1 = exp2f(o[1] - n1);
          d1 = d1 * u1 + o[3] * w1;
          a1 = a1 * u1 + o[5] * w1;
          mx1 = n1;
        }
      }
    }
  }
  float y0 = g == 0 ? a0 / d0 : 0.f, y1 = g == 0 ? a1 / d1 : 0.f;
  norm_rope_pair(y0, y1, g == 0, pair, p, p.pos0 + (int64_t)m * s, red);
  if (s < p.n_cap) {
    if (g == 0) store2(static_cast<T*>(p.entries) + ((size_t)b * p.n_cap + s) * c + ch, y0, y1);
  } else if (threadIdx.x == 0) {
    report(p.status, CSA_DEV_STREAM, (unsigned)b);   // entry cache full: entry dropped
  }
  __syncthreads();   // every thread has read the count
  if (threadIdx.x == 0) *reinterpret_cast<int64_t*>(st) = t + 1;
}

}  // namespace

size_t stream_state_bytes(int elem_bytes, int m, int overlap, int c, int z_cols) {
  const size_t groups = overlap ? 3 : 1;   // a + b of two blocks, or a alone
  const size_t raw = 16 + groups * (size_t)m * ((size_t)c + (size_t)z_cols) * elem_bytes;
  return (raw + 255) & ~(size_t)255;
}

cudaError_t launch_stream_append(int dtype, StreamParams p, int64_t B, cudaStream_t stream) {
  if (B == 0) return cudaSuccess;
  if (p.f.r > 2 * kStreamMaxPairs) return cudaErrorInvalidValue;
  for (int i = 0; i < p.f.r / 2; ++i)   // RoPE frequencies base^(-2i/r), in double
    p.theta[i] = pow((double)p.f.base, -2.0 * (double)i / (double)p.f.r);
  const int np = p.f.c / 2;
  const int ns_max = p.overlap ? 2 * p.m : p.m;
  int G = ns_max >= 32 ? 4 : 1;
  while (G > 1 && np * G > 1024) G >>= 1;
  const int threads = np * G;
  const size_t smem = G > 1 ? sizeof(float) * 6 * (size_t)np * G : 0;
  if (dtype == CSA_BF16) {
    if (smem > 48 * 1024) {
      cudaError_t e = cudaFuncSetAttribute(stream_append_kernel<bf16>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
    }
    stream_append_kernel<bf16><<<(unsigned)B, threads, smem, stream>>>(p);
  } else {
    if (smem > 48 * 1024) {
      cudaError_t e = cudaFuncSetAttribute(stream_append_kernel<float>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
    }
    stream_append_kernel<float><<<(unsigned)B, threads, smem, stream>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace csa
