// Lightning indexer + causal top-k on CUDA cores (float32 arithmetic).
//
// Method: page "DeepSeek-V4：迈向高效百万 Token 上下文智能", §3.3 (CSA) --
// I[t,s] = sum_h w[t,h] ReLU(q_I[t,h] . K_I[s]) and the top-k entries of each
// query form its candidate set.  Readings: entry s is visible iff
// s < floor((p+1)/m); ties go to the lower index; the selection is emitted in
// ascending index order and padded with -1.
//
// This is the portable path: the float32 workload and any shape the
// tensor-core kernel does not take.  Two launches: a score kernel (one CTA per
// query row, q_I and w staged in shared memory, each thread scoring entries
// with the key row held in registers) writing the visible prefix of the row
// to scratch, then an exact radix select (four 8-bit passes over the
// order-preserving uint32 image of the scores) and an ordered compaction.
#include "common.cuh"
#include "internal.h"

namespace csa {

namespace {

constexpr int kMaxHI = 64;
constexpr int kChunk = 32;  // key elements held in registers at a time

__device__ __forceinline__ int64_t visible_count(int64_t pos, int m, int64_t N) {
  if (pos < 0) return 0;
  int64_t v = (pos + 1) / m;
  return v < N ? v : N;
}

// Order-preserving map float -> uint32 (larger float, larger key); -0 == +0.
__device__ __forceinline__ unsigned score_key(float f) {
  unsigned u = __float_as_uint(f + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <typename T>
__global__ void __launch_bounds__(256) indexer_scores_kernel(IndexerParams p, float* scores) {
  extern __shared__ float sm[];
  const int HI = p.HI, dI = p.dI;
  float* qs = sm;             // [HI][dI]
  float* ws = sm + HI * dI;   // [HI]
  const int64_t t = blockIdx.x, b = blockIdx.y;
  const int64_t row = b * p.Tq + t;
  const int64_t pos = p.q_pos ? p.q_pos[row] : t;
  const int64_t vis = visible_count(pos, p.m, p.N);
  const T* q = static_cast<const T*>(p.q_I) + row * HI * dI;
  for (int i = threadIdx.x; i < HI * dI; i += blockDim.x) qs[i] = to_float(q[i]);
  for (int i = threadIdx.x; i < HI; i += blockDim.x) ws[i] = p.w[row * HI + i];
  __syncthreads();
  const T* kbase = static_cast<const T*>(p.k_I) + b * p.N * dI;
  float* out = scores + row * p.N;
  for (int64_t s = threadIdx.x; s < vis; s += blockDim.x) {
    float dots[kMaxHI];
#pragma unroll
    for (int h = 0; h < kMaxHI; ++h) dots[h] = 0.f;
    const T* kr = kbase + s * dI;
    for (int d0 = 0; d0 < dI; d0 += kChunk) {
      float kv[kChunk];
      int nd = dI - d0 < kChunk ? dI - d0 : kChunk;
#pragma unroll
      for (int d = 0; d < kChunk; ++d) kv[d] = d < nd ? to_float(kr[d0 + d]) : 0.f;
#pragma unroll
      for (int h = 0; h < kMaxHI; ++h) {
        if (h < HI) {
          const float* qh = qs + h * dI + d0;
          float a = dots[h];
#pragma unroll
          for (int d = 0; d < kChunk; ++d)
            if (d < nd) a = fmaf(qh[d], kv[d], a);
          dots[h] = a;
        }
      }
    }
    float sc = 0.f;
#pragma unroll
    for (int h = 0; h < kMaxHI; ++h)
      if (h < HI) sc = fmaf(ws[h], fmaxf(dots[h], 0.f), sc);
    out[s] = sc;
  }
}

// Exclusive block-wide count of `flag` over threads before this one, and the
// block total.  Every thread must call it.  `tmp` holds 33 unsigned.
__device__ __forceinline__ unsigned block_excl_count(bool flag, unsigned* tmp, unsigned* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  unsigned ball = __ballot_sync(0xffffffffu, flag);
  unsigned in_warp = __popc(ball & ((1u << lane) - 1u));
  __syncthreads();
  if (lane == 0) tmp[warp] = __popc(ball);
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned run = 0;
    for (int i = 0; i < nw; ++i) {
      unsigned c = tmp[i];
      tmp[i] = run;
      run += c;
    }
    tmp[32] = run;
  }
  __syncthreads();
  *total = tmp[32];
  return tmp[warp] + in_warp;
}

__global__ void __launch_bounds__(1024) topk_kernel(IndexerParams p, const float* scores) {
  __shared__ unsigned hist[256];
  __shared__ unsigned tmp[33];
  __shared__ unsigned s_prefix, s_mask;
  __shared__ int s_remaining;
  const int64_t t = blockIdx.x, b = blockIdx.y;
  const int64_t row = b * p.Tq + t;
  const int64_t pos = p.q_pos ? p.q_pos[row] : t;
  const int64_t vis = visible_count(pos, p.m, p.N);
  const float* sc = scores + row * p.N;
  int32_t* out = p.idx_out + row * p.k;
  float* so = p.score_out ? p.score_out + row * p.k : nullptr;
  const int k = p.k;

  if (vis <= k) {  // everything visible is selected
    for (int i = threadIdx.x; i < k; i += blockDim.x) {
      out[i] = i < vis ? i : -1;
      if (so) so[i] = i < vis ? sc[i] : -INFINITY;
    }
    return;
  }

  // radix select of the k-th largest key, most significant digit first
  if (threadIdx.x == 0) { s_prefix = 0u; s_mask = 0u; s_remaining = k; }
  __syncthreads();
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0u;
    __syncthreads();
    const unsigned prefix = s_prefix, mask = s_mask;
    for (int64_t s = threadIdx.x; s < vis; s += blockDim.x) {
      unsigned key = score_key(sc[s]);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int rem = s_remaining;
      unsigned cum = 0;
      int d = 255;
      for (; d > 0; --d) {
        if (cum + hist[d] >= (unsigned)rem) break;
        cum += hist[d];
      }
      s_prefix = prefix | ((unsigned)d << shift);
      s_mask = mask | (255u << shift);
      s_remaining = rem - (int)cum;
    }
    __syncthreads();
  }
  const unsigned tau = s_prefix;
  const unsigned need_eq = (unsigned)s_remaining;  // keys equal to tau to take

  // ordered compaction: every key above tau, and the need_eq lowest-index
  // keys equal to tau
  unsigned run_sel = 0, run_eq = 0;
  for (int64_t base = 0; base < vis; base += blockDim.x) {
    int64_t s = base + threadIdx.x;
    bool in = s < vis;
    unsigned key = in ? score_key(sc[s]) : 0u;
    bool gt = in && key > tau;
    bool eq = in && key == tau;
    unsigned eq_tot;
    unsigned eq_rank = run_eq + block_excl_count(eq, tmp, &eq_tot);
    bool take = gt || (eq && eq_rank < need_eq);
    unsigned sel_tot;
    unsigned at = run_sel + block_excl_count(take, tmp, &sel_tot);
    if (take && at < (unsigned)k) {
      out[at] = (int32_t)s;
      if (so) so[at] = sc[s];
    }
    run_eq += eq_tot;
    run_sel += sel_tot;
  }
}

}  // namespace

size_t indexer_portable_scratch(int64_t B, int64_t Tq, int64_t N, int k) {
  (void)k;
  return (size_t)B * (size_t)Tq * (size_t)N * sizeof(float);
}

cudaError_t launch_indexer_portable(int dtype, const IndexerParams& p, cudaStream_t stream) {
  if (p.B == 0 || p.Tq == 0) return cudaSuccess;
  float* scores = static_cast<float*>(p.scratch);
  dim3 grid((unsigned)p.Tq, (unsigned)p.B);
  size_t smem = sizeof(float) * ((size_t)p.HI * p.dI + p.HI);
  if (dtype == CSA_BF16) {
    cudaFuncSetAttribute(indexer_scores_kernel<bf16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    indexer_scores_kernel<bf16><<<grid, 256, smem, stream>>>(p, scores);
  } else {
    cudaFuncSetAttribute(indexer_scores_kernel<float>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    indexer_scores_kernel<float><<<grid, 256, smem, stream>>>(p, scores);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  topk_kernel<<<grid, 1024, 0, stream>>>(p, scores);
  return cudaGetLastError();
}

}  // namespace csa
