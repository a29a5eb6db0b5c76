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
#include "sm100.cuh"

namespace csa {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kWarps = 8;   // warps per CTA


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
          rope_cos_sin_theta(pos, theta[(ch - d0) >> 1], &cs, &sn);
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

// ---- bf16, c = 512, per-channel logits: streaming fast paths ---------------
// Rows of every input tensor that one chunk of tokens needs are contiguous, so
// persistent CTAs stage them through a ring of shared-memory slots, one bulk
// asynchronous copy per tensor and chunk (several chunks in flight; the copy
// engine, not per-thread 16-byte requests, keeps the bytes in flight), and
// take chunks round-robin; compute reads the staged rows, never global memory.
constexpr int kFC = 512;                    // channels
constexpr int kFRowB = kFC * 2;             // bytes per token row
constexpr int kFThreads = 256;
constexpr int kFTab = 2048 + 64;            // RoPE cos/sin table: [rows][32 pairs] float2
constexpr int kFDelta = 8192;               // (cos, sin) of i * theta, i < 16: [16][32] float2
constexpr int kFBase = kFDelta + 16 * 32 * 8;   // a chunk's row-0 (cos, sin): [32] float2
constexpr int kFBar = kFBase + 32 * 8;      // ring-slot mbarriers: [stages] u64
constexpr int kFHead = 13312;               // frequencies, reductions, tables, barriers
static_assert(kFTab + 17 * 32 * 8 <= kFDelta && kFBar + 4 * 8 <= kFHead, "head layout");

// Fills ring slot `slot_s` with token rows [st, st + rows) of one [B, T, 512]
// tensor of sequence b, clipped to [0, T) (rows outside stay stale and are
// never read); returns the bytes requested.  count_only: no copy is issued.
__device__ __forceinline__ uint32_t stage_rows(uint32_t slot_s, const bf16* src, int64_t b,
                                               int64_t T, int64_t st, int rows, uint64_t* bar,
                                               bool count_only) {
  const int64_t lo = st > 0 ? st : 0, hi = st + rows < T ? st + rows : T;
  if (hi <= lo) return 0u;
  const uint32_t bytes = (uint32_t)(hi - lo) * kFRowB;
  if (!count_only)
    sm100::bulk_load(slot_s + (uint32_t)(lo - st) * kFRowB, src + (b * T + lo) * kFC, bytes, bar);
  return bytes;
}

// Waits for ring phase k (slot k % S); false once a wait ran out on any
// thread of the CTA (the status word then holds the error).
template <int S>
__device__ __forceinline__ bool ring_ready(uint64_t* full, uint32_t k, unsigned* status,
                                           unsigned detail) {
  const bool ok = sm100::mbar_wait(&full[k % S], (k / S) & 1u);
  if (__syncthreads_or(!ok)) {
    if (threadIdx.x == 0) report(status, CSA_DEV_TIMEOUT, detail);
    return false;
  }
  return true;
}

// Before the CTA exits: the copies of every phase issued but not consumed
// ([consumed, issued), at most S of them) have landed (bounded waits;
// thread 0).
template <int S>
__device__ __forceinline__ void ring_drain(uint64_t* full, uint32_t consumed, uint32_t issued) {
  if (threadIdx.x == 0)
    for (uint32_t k = consumed; k < issued; ++k) sm100::mbar_wait(&full[k % S], (k / S) & 1u);
}

// Window row from a staged token row: RoPE_pos(RMSNorm(row)).  Lane l owns the
// 16-byte chunks l and l + 32 (channels 8l..8l+7 and 256+8l..256+8l+7), so a
// warp reads and writes the row as two conflict-free 512-byte sweeps.
__device__ __forceinline__ void window_row_staged(const uint8_t* srow, bf16* dst, int lane,
                                                  const Fmt& f, const float2* tab) {
  float v[16];
  const uint4 u0 = *reinterpret_cast<const uint4*>(srow + lane * 16);
  const uint4 u1 = *reinterpret_cast<const uint4*>(srow + 512 + lane * 16);
  const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[2 * i] = bf16_bits_to_float(w[i] & 0xffffu);
    v[2 * i + 1] = bf16_bits_to_float(w[i] >> 16);
  }
  if (!(f.flags & CSA_F_NO_NORM)) {
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < 16; ++e) ss = fmaf(v[e], v[e], ss);
    ss = warp_sum(ss);
    const float inv = rsqrtf(ss / (float)kFC + f.eps);
#pragma unroll
    for (int e = 0; e < 16; ++e) v[e] *= inv;
  }
  if (!(f.flags & CSA_F_NO_ROPE)) {
    const int d0 = kFC - f.r;
#pragma unroll
    for (int e = 0; e < 16; e += 2) {
      const int ch = (e < 8 ? 8 * lane : 256 + 8 * lane) + (e & 7);
      if (ch >= d0) {
        const float2 cs = tab[(ch - d0) >> 1];
        const float x0 = v[e], x1 = v[e + 1];
        v[e] = x0 * cs.x - x1 * cs.y;
        v[e + 1] = x0 * cs.y + x1 * cs.x;
      }
    }
  }
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
  reinterpret_cast<uint4*>(dst)[lane] = make_uint4(o[0], o[1], o[2], o[3]);
  reinterpret_cast<uint4*>(dst)[32 + lane] = make_uint4(o[4], o[5], o[6], o[7]);
}

// The two bf16 values packed in a 32-bit word, widened exactly.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// One softmax-weighted term in base 2 against a running maximum mxl (in log2
// units, at least z log2(e) up to rounding): e = 2^(z log2 e - mxl).  The
// exponent is never meaningfully positive, so the hardware ex2 (relative
// error ~2^-22, results below 2^-126 flushed to 0) replaces the libm call.
__device__ __forceinline__ void sm_term(float z, float v, float mxl, float& den, float& acc) {
  const float e = sm100::ex2(fmaf(z, kLog2e, -mxl));
  den += e;
  acc = fmaf(e, v, acc);
}

// Per-CTA table of (cos, sin) of i * theta_pr, i < 16: a chunk's table rows are
// positions p0 + i, so each is the row-0 angle rotated by one of these.
__device__ __forceinline__ void fill_delta_table(float2* dtab, int r, const double* theta) {
  for (int q = threadIdx.x; q < 16 * 32; q += kFThreads) {
    const int i = q >> 5, pr = q & 31;
    float cs = 1.f, sn = 0.f;
    if (pr < (r >> 1)) rope_cos_sin_theta(i, theta[pr], &cs, &sn);
    dtab[q] = make_float2(cs, sn);
  }
}

// tab[i][pr] = (cos, sin) of (p0 + delta(i)) theta_pr for i < rows, with
// delta(i) < 16: warp 0 forms the row-0 angles (double-reduced), then every
// thread takes a share of the complex products with the delta table.  Every
// thread of the CTA calls this (it holds a barrier).
template <typename DeltaFn>
__device__ __forceinline__ void fill_rope_rows(float2* tab, float2* base, const float2* dtab,
                                               int rows, int r, const double* theta, int64_t p0,
                                               DeltaFn delta) {
  const int np = r >> 1;
  if (threadIdx.x < np) {
    float cs, sn;
    rope_cos_sin_theta(p0, theta[threadIdx.x], &cs, &sn);
    base[threadIdx.x] = make_float2(cs, sn);
  }
  __syncthreads();
  for (int q = threadIdx.x; q < rows * 32; q += kFThreads) {
    const int i = q >> 5, pr = q & 31;
    if (pr < np) {
      const float2 b = base[pr], d = dtab[delta(i) * 32 + pr];
      tab[q] = make_float2(b.x * d.x - b.y * d.y, b.x * d.y + b.y * d.x);
    }
  }
}

// CSA, m = 4: a chunk is 8 tokens (2 entries); slot = C^a, Z^a rows [t0, t0+8)
// and C^b, Z^b rows [t0-4, t0+4) (group b covers the previous block).
constexpr int kCR = 8;
constexpr int kCStage = 4 * kCR * kFRowB;   // 32 KB
constexpr int kCStages = 3;                 // 96 KB ring: two CTAs per SM

__global__ void __launch_bounds__(kFThreads, 2)
    csa_compress_fast_kernel(CompressParams p, uint32_t n_chunks, uint32_t total) {
  extern __shared__ __align__(1024) uint8_t fsm[];
  double* theta = reinterpret_cast<double*>(fsm);
  float* red = reinterpret_cast<float*>(fsm + 2048);   // [8]
  float2* tab = reinterpret_cast<float2*>(fsm + kFTab); // rows 0-7 window, 8-9 entries
  float2* dtab = reinterpret_cast<float2*>(fsm + kFDelta);
  float2* rbase = reinterpret_cast<float2*>(fsm + kFBase);
  uint64_t* full = reinterpret_cast<uint64_t*>(fsm + kFBar);   // [kCStages] slot landed
  uint8_t* ring = fsm + kFHead;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  if (t == 0) {
    for (int i = 0; i < kCStages; ++i) sm100::mbar_init(&full[i], 1);
    sm100::fence_barrier_init();
  }
  for (int i = t; i < (p.f.r >> 1); i += kFThreads)
    theta[i] = pow((double)p.f.base, -2.0 * (double)i / (double)p.f.r);
  __syncthreads();   // frequencies and barriers complete before the tables
  if (!(p.f.flags & CSA_F_NO_ROPE)) fill_delta_table(dtab, p.f.r, theta);
  __syncthreads();
  const uint32_t ring_s = sm100::smem_u32(ring);
  // slot layout: [kv_a, z_a rows t0..t0+7][kv_b, z_b rows t0-4..t0+3]
  const bf16* src4[4] = {static_cast<const bf16*>(p.kv_a), static_cast<const bf16*>(p.z_a),
                         static_cast<const bf16*>(p.kv_b), static_cast<const bf16*>(p.z_b)};
  // thread 0 fills `slot` with chunk u (past the end: an arrival with no
  // bytes, so the slot's phases stay in step).  The slot was last read in the
  // iteration before, which ended with a CTA barrier.
  uint32_t n_issued = 0;   // ring phases issued (the same count on every thread)
  auto issue = [&](uint32_t u, int slot) {
    ++n_issued;
    if (t != 0) return;
    const uint32_t s0 = ring_s + slot * kCStage;
    const int64_t b = u < total ? u / n_chunks : 0;
    const int64_t t0 = u < total ? (int64_t)(u % n_chunks) * kCR : 0;
    uint32_t bytes = 0;
    if (u < total)
      for (int i = 0; i < 4; ++i)
        bytes += stage_rows(0, src4[i], b, p.T, i < 2 ? t0 : t0 - 4, kCR, nullptr, true);
    sm100::fence_proxy_async_smem();
    sm100::mbar_arrive_expect_tx(&full[slot], bytes);
    if (u < total)
      for (int i = 0; i < 4; ++i)
        stage_rows(s0 + i * kCR * kFRowB, src4[i], b, p.T, i < 2 ? t0 : t0 - 4, kCR, &full[slot],
                   false);
  };
  const int e = t >> 7, cq = t & 127;   // entry of the chunk, channels 4cq .. 4cq+3
  int k = 0;
  for (int i = 0; i < kCStages - 1; ++i) issue(blockIdx.x + i * gridDim.x, i);
  for (uint32_t u = blockIdx.x; u < total; u += gridDim.x, ++k) {
    issue(u + (kCStages - 1) * gridDim.x, (k + kCStages - 1) % kCStages);
    const int64_t b = u / n_chunks, t0 = (int64_t)(u % n_chunks) * kCR;
    // rows 0-7: the chunk's tokens; rows 8-9: its two entries (at t0, t0 + 4)
    if (!(p.f.flags & CSA_F_NO_ROPE))
      fill_rope_rows(tab, rbase, dtab, kCR + 2, p.f.r, theta, p.pos0 + t0,
                     [](int i) { return i < kCR ? i : 4 * (i - kCR); });
    if (!ring_ready<kCStages>(full, (uint32_t)k, p.status, 40u)) break;
    const uint8_t* buf = ring + (k % kCStages) * kCStage;
    const int64_t s = t0 / 4 + e;
    const bool have = s < p.n_entries;   // uniform per warp
    float val[4] = {0.f, 0.f, 0.f, 0.f};
    if (have) {
      // the entry's 2m = 8 slots (group a: its own block; group b: the
      // previous block, absent for entry 0) for channels 4cq .. 4cq+3: the
      // logits' maximum first, then one exp2 per slot
      const int ns = s == 0 ? 4 : 8;   // uniform per warp
      uint2 cv[8], zv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int g = i >> 2, row = 4 * e + (i & 3);
        if (i < ns) {
          cv[i] = *reinterpret_cast<const uint2*>(buf + ((2 * g) * kCR + row) * kFRowB + cq * 8);
          zv[i] = *reinterpret_cast<const uint2*>(buf + ((2 * g + 1) * kCR + row) * kFRowB + cq * 8);
        }
      }
      float mxl[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (i < ns) {
          mxl[0] = fmaxf(mxl[0], bf16_lo(zv[i].x));
          mxl[1] = fmaxf(mxl[1], bf16_hi(zv[i].x));
          mxl[2] = fmaxf(mxl[2], bf16_lo(zv[i].y));
          mxl[3] = fmaxf(mxl[3], bf16_hi(zv[i].y));
        }
      }
      float den[4] = {0.f, 0.f, 0.f, 0.f}, acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 4; ++c) mxl[c] *= kLog2e;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (i < ns) {
          sm_term(bf16_lo(zv[i].x), bf16_lo(cv[i].x), mxl[0], den[0], acc[0]);
          sm_term(bf16_hi(zv[i].x), bf16_hi(cv[i].x), mxl[1], den[1], acc[1]);
          sm_term(bf16_lo(zv[i].y), bf16_lo(cv[i].y), mxl[2], den[2], acc[2]);
          sm_term(bf16_hi(zv[i].y), bf16_hi(cv[i].y), mxl[3], den[3], acc[3]);
        }
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) val[c] = acc[c] / den[c];
    }
    // RMSNorm over the entry's 512 channels (128 threads = warps 4e .. 4e+3)
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) ss = fmaf(val[c], val[c], ss);
    ss = warp_sum(ss);
    if (lane == 0) red[warp] = ss;
    // window rows: warp w normalises and rotates token row t0 + w
    if (p.win != nullptr && t0 + warp < p.T)
      window_row_staged(buf + warp * kFRowB, static_cast<bf16*>(p.win) + (b * p.T + t0 + warp) * kFC,
                        lane, p.f, tab + warp * 32);
    __syncthreads();
    if (have) {
      const float tot = red[4 * e] + red[4 * e + 1] + red[4 * e + 2] + red[4 * e + 3];
      if (!(p.f.flags & CSA_F_NO_NORM)) {
        const float inv = rsqrtf(tot / (float)kFC + p.f.eps);
#pragma unroll
        for (int c = 0; c < 4; ++c) val[c] *= inv;
      }
      const int d0 = kFC - p.f.r;
      if (!(p.f.flags & CSA_F_NO_ROPE)) {
#pragma unroll
        for (int c = 0; c < 4; c += 2) {
          const int ch = 4 * cq + c;
          if (ch >= d0) {
            const float2 cs = tab[(kCR + e) * 32 + ((ch - d0) >> 1)];
            const float x0 = val[c], x1 = val[c + 1];
            val[c] = x0 * cs.x - x1 * cs.y;
            val[c + 1] = x0 * cs.y + x1 * cs.x;
          }
        }
      }
      *reinterpret_cast<uint2*>(static_cast<bf16*>(p.entries) + (b * p.n_entries + s) * kFC + 4 * cq) =
          make_uint2(pack_bf16x2(val[0], val[1]), pack_bf16x2(val[2], val[3]));
    }
    __syncthreads();   // table, reductions and this slot are rewritten next
  }
  ring_drain<kCStages>(full, (uint32_t)k, n_issued);
}

// HCA, m' a multiple of 16: a unit is one block of m' tokens (its entry, when
// complete, plus its window rows) streamed as m'/16 chunks of 16 C and Z rows;
// thread t keeps the online-softmax state of channels 2t, 2t+1 across chunks.
constexpr int kHR = 16;
constexpr int kHStage = 2 * kHR * kFRowB;   // 32 KB
constexpr int kHStages = 3;                 // 96 KB ring: two CTAs per SM

__global__ void __launch_bounds__(kFThreads, 2)
    hca_compress_fast_kernel(CompressParams p, uint32_t n_blocks, uint32_t total) {
  extern __shared__ __align__(1024) uint8_t fsm[];
  double* theta = reinterpret_cast<double*>(fsm);
  float* red = reinterpret_cast<float*>(fsm + 2048);   // [8]
  float2* tab = reinterpret_cast<float2*>(fsm + kFTab); // rows 0-15 window, 16 entry
  float2* dtab = reinterpret_cast<float2*>(fsm + kFDelta);
  float2* rbase = reinterpret_cast<float2*>(fsm + kFBase);
  uint64_t* full = reinterpret_cast<uint64_t*>(fsm + kFBar);   // [kHStages] slot landed
  uint8_t* ring = fsm + kFHead;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  if (t == 0) {
    for (int i = 0; i < kHStages; ++i) sm100::mbar_init(&full[i], 1);
    sm100::fence_barrier_init();
  }
  for (int i = t; i < (p.f.r >> 1); i += kFThreads)
    theta[i] = pow((double)p.f.base, -2.0 * (double)i / (double)p.f.r);
  __syncthreads();   // frequencies and barriers complete before the tables
  if (!(p.f.flags & CSA_F_NO_ROPE)) fill_delta_table(dtab, p.f.r, theta);
  __syncthreads();
  const uint32_t ring_s = sm100::smem_u32(ring);
  const bf16* kv = static_cast<const bf16*>(p.kv_a);
  const bf16* z = static_cast<const bf16*>(p.z_a);
  const int cpu = p.m / kHR;                               // chunks per unit
  const uint32_t n_my = total > blockIdx.x ? (total - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  const uint32_t n_ck = n_my * cpu;                        // this CTA's chunk sequence
  // thread 0 fills `slot` with chunk kk of this CTA's sequence ([kv rows]
  // [z rows], 16 each; past the end: an arrival with no bytes).  The slot was
  // last read in the iteration before, which ended with a CTA barrier.
  uint32_t n_issued = 0;   // ring phases issued (the same count on every thread)
  auto issue = [&](uint32_t kk, int slot) {
    ++n_issued;
    if (t != 0) return;
    const uint32_t s0 = ring_s + slot * kHStage;
    int64_t b = 0, t0 = 0;
    uint32_t bytes = 0;
    if (kk < n_ck) {
      const uint32_t u = blockIdx.x + (kk / cpu) * gridDim.x;
      b = u / n_blocks;
      t0 = (int64_t)(u % n_blocks) * p.m + (int64_t)(kk % cpu) * kHR;
      bytes = 2 * stage_rows(0, kv, b, p.T, t0, kHR, nullptr, true);
    }
    sm100::fence_proxy_async_smem();
    sm100::mbar_arrive_expect_tx(&full[slot], bytes);
    if (kk < n_ck) {
      stage_rows(s0, kv, b, p.T, t0, kHR, &full[slot], false);
      stage_rows(s0 + kHR * kFRowB, z, b, p.T, t0, kHR, &full[slot], false);
    }
  };
  for (int i = 0; i < kHStages - 1; ++i) issue(i, i);
  uint32_t n_done = n_ck;   // phases consumed (the loop's count unless a wait ran out)
  float mx[2], den[2], acc[2];
  for (uint32_t kk = 0; kk < n_ck; ++kk) {
    issue(kk + kHStages - 1, (int)((kk + kHStages - 1) % kHStages));
    const uint32_t u = blockIdx.x + (kk / cpu) * gridDim.x;
    const int j = (int)(kk % cpu);
    const int64_t b = u / n_blocks, s = u % n_blocks, t0 = s * p.m + (int64_t)j * kHR;
    // rows 0-15: the chunk's tokens; row 16: the block's entry (at s m'), on
    // the block's last chunk only, where the entry is finished
    if (!(p.f.flags & CSA_F_NO_ROPE)) {
      fill_rope_rows(tab, rbase, dtab, kHR, p.f.r, theta, p.pos0 + t0, [](int i) { return i; });
      if (j == cpu - 1 && t < (p.f.r >> 1)) {
        float cs, sn;
        rope_cos_sin_theta(p.pos0 + s * p.m, theta[t], &cs, &sn);
        tab[kHR * 32 + t] = make_float2(cs, sn);
      }
    }
    if (!ring_ready<kHStages>(full, kk, p.status, 41u)) {
      n_done = kk;
      break;
    }
    const uint8_t* buf = ring + (kk % kHStages) * kHStage;
    if (j == 0) {
#pragma unroll
      for (int c = 0; c < 2; ++c) { mx[c] = -INFINITY; den[c] = 0.f; acc[c] = 0.f; }
    }
    const bool have = s < p.n_entries;   // a complete block (CTA-uniform)
    if (have) {
      // the chunk's 16 rows of channels 2t, 2t+1: their logits' maximum
      // updates the running one (one rescale of the state per chunk), then
      // one exp2 per row
      uint32_t cw[kHR], zw[kHR];
      float cm0 = -INFINITY, cm1 = -INFINITY;
#pragma unroll
      for (int r = 0; r < kHR; ++r) {
        cw[r] = *reinterpret_cast<const uint32_t*>(buf + r * kFRowB + t * 4);
        zw[r] = *reinterpret_cast<const uint32_t*>(buf + (kHR + r) * kFRowB + t * 4);
        cm0 = fmaxf(cm0, bf16_lo(zw[r]));
        cm1 = fmaxf(cm1, bf16_hi(zw[r]));
      }
      const float cm[2] = {cm0 * kLog2e, cm1 * kLog2e};
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const float mn = fmaxf(mx[c], cm[c]);
        const float sc = sm100::ex2(mx[c] - mn);   // 0 on the block's first chunk
        den[c] *= sc;
        acc[c] *= sc;
        mx[c] = mn;
      }
#pragma unroll
      for (int r = 0; r < kHR; ++r) {
        sm_term(bf16_lo(zw[r]), bf16_lo(cw[r]), mx[0], den[0], acc[0]);
        sm_term(bf16_hi(zw[r]), bf16_hi(cw[r]), mx[1], den[1], acc[1]);
      }
    }
    if (p.win != nullptr) {   // window rows: warp w takes rows 2w, 2w+1 of the chunk
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int r = 2 * warp + h;
        if (t0 + r < p.T)
          window_row_staged(buf + r * kFRowB, static_cast<bf16*>(p.win) + (b * p.T + t0 + r) * kFC,
                            lane, p.f, tab + r * 32);
      }
    }
    if (j == cpu - 1 && have) {   // CTA-uniform: finish the entry
      float v0 = acc[0] / den[0], v1 = acc[1] / den[1];
      float ss = warp_sum(fmaf(v0, v0, v1 * v1));
      if (lane == 0) red[warp] = ss;
      __syncthreads();
      float tot = 0.f;
#pragma unroll
      for (int w = 0; w < kFThreads / 32; ++w) tot += red[w];
      if (!(p.f.flags & CSA_F_NO_NORM)) {
        const float inv = rsqrtf(tot / (float)kFC + p.f.eps);
        v0 *= inv;
        v1 *= inv;
      }
      const int ch = 2 * t, d0 = kFC - p.f.r;
      if (!(p.f.flags & CSA_F_NO_ROPE) && ch >= d0) {
        const float2 cs = tab[kHR * 32 + ((ch - d0) >> 1)];
        const float x0 = v0, x1 = v1;
        v0 = x0 * cs.x - x1 * cs.y;
        v1 = x0 * cs.y + x1 * cs.x;
      }
      reinterpret_cast<uint32_t*>(static_cast<bf16*>(p.entries) + (b * p.n_entries + s) * kFC)[t] =
          pack_bf16x2(v0, v1);
    }
    __syncthreads();   // the slot is refilled next iteration; red reused
  }
  ring_drain<kHStages>(full, n_done, n_issued);
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  return n;
}

// Launches a fast path when the shape has one; *taken tells whether it did.
cudaError_t launch_compress_fast(int dtype, const CompressParams& p, int64_t B, cudaStream_t stream,
                                 bool* taken) {
  *taken = false;
  if (dtype != CSA_BF16 || p.f.c != kFC || p.z_cols != kFC || p.f.r > kFC) return cudaSuccess;
  if (p.overlap ? p.m != 4 : (p.m % kHR != 0)) return cudaSuccess;
  *taken = true;
  const int64_t grid_max = 2 * (int64_t)sm_count();   // two CTAs per SM
  if (p.overlap) {
    const int64_t n_chunks = (p.T + kCR - 1) / kCR;
    const int64_t total = B * n_chunks;
    if (total == 0) return cudaSuccess;
    if (total + grid_max * kCStages >= (1LL << 32)) { *taken = false; return cudaSuccess; }
    const int smem = kFHead + kCStages * kCStage;
    cudaError_t e = cudaFuncSetAttribute(csa_compress_fast_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)(total < grid_max ? total : grid_max);
    csa_compress_fast_kernel<<<grid, kFThreads, smem, stream>>>(p, (uint32_t)n_chunks,
                                                                (uint32_t)total);
  } else {
    const int64_t n_blocks = (p.T + p.m - 1) / p.m;   // the last may be partial (window only)
    const int64_t total = B * n_blocks;
    if (total == 0 || (p.n_entries == 0 && p.win == nullptr)) return cudaSuccess;
    if ((total + grid_max) * (p.m / kHR) >= (1LL << 32)) { *taken = false; return cudaSuccess; }
    const int smem = kFHead + kHStages * kHStage;
    cudaError_t e = cudaFuncSetAttribute(hca_compress_fast_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)(total < grid_max ? total : grid_max);
    hca_compress_fast_kernel<<<grid, kFThreads, smem, stream>>>(p, (uint32_t)n_blocks,
                                                                (uint32_t)total);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_compress(int dtype, CompressParams p, int64_t B, cudaStream_t stream) {
  bool taken = false;
  cudaError_t e = launch_compress_fast(dtype, p, B, stream, &taken);
  if (taken) return e;
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
