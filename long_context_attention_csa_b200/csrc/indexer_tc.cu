// Lightning indexer with a fused causal top-k on the 5th-generation tensor
// cores (tcgen05, accumulators in TMEM, operands staged by TMA).
//
// Method: page "DeepSeek-V4：迈向高效百万 Token 上下文智能", §3.3 (CSA) --
// I[t,s] = sum_h w[t,h] ReLU(q_I[t,h] . K_I[s]); the top-k entries of each
// query are its candidate set.  Readings: entry s is visible iff
// s < floor((p+1)/m); ties go to the lower index; output ascending, -1 padded.
//
// Layout: compressed entries on the MMA's M side (128 per tile, one per TMEM
// lane) and (token, head) pairs on N (TOK tokens x 64 heads), K = d_I = 128.
// Every TMEM lane then holds all heads of one entry for TOK tokens, so the
// epilogue sum_h w ReLU(.) is a per-thread loop with no cross-lane traffic.
//   warp 0      TMA producer: q_I block once, K_I tiles through a ring;
//   warp 1      TMEM owner and single-thread MMA issuer (8 MMAs per tile);
//   warps 2..5  epilogue: TMEM -> registers -> scores in shared memory
//               (two TMEM accumulators so tile i+1's MMAs overlap tile i's
//               epilogue); afterwards one warp per token runs an exact radix
//               select over the scores and an ordered compaction.
// The score matrix never reaches HBM.  A CTA covers the entries of one chunk
// (2048 for 4-token groups, 4096 for single tokens); when the entries span
// several chunks each CTA emits its chunk's top-k as candidates and a merge
// kernel selects the final k (the union of per-chunk top-k sets contains the
// global top-k under the same tie rule).
#include "common.cuh"
#include "sm100.cuh"
#include "tc.h"
#include "tma_host.h"

namespace csa {

namespace {

using namespace sm100;

constexpr int kBM = 128;   // entries per tile
constexpr int kDI = 128;   // indexer dim
constexpr int kHI = 64;    // indexer heads
constexpr int kTileBytes = kBM * kDI * 2;     // 32 KB (two 128-byte-swizzled column halves)
constexpr int kThreads = 192;
constexpr int kBinCap = 64;   // largest boundary bin the value-binned top-k ranks exactly
constexpr int kMergeCap = 2048;   // the same for the chunk-candidate merge

template <int TOK> struct Cfg;
template <> struct Cfg<4> { static constexpr int kStages = 3; static constexpr int kChunk = 2048; };
template <> struct Cfg<1> { static constexpr int kStages = 2; static constexpr int kChunk = 4096; };

// sum_h w[h] ReLU(s[h]) over 64 heads (s: two 32-column TMEM loads) with
// packed fp32 FMAs (two heads per instruction; even and odd heads accumulate
// separately and are added at the end).
__device__ __forceinline__ float relu_weighted_sum64(const float* wt, const uint32_t* r0,
                                                     const uint32_t* r1) {
  unsigned long long acc = 0ull;
  const float2* w2 = reinterpret_cast<const float2*>(wt);
#pragma unroll
  for (int h = 0; h < 64; h += 2) {
    const uint32_t* r = h < 32 ? r0 : r1;
    const float s0 = fmaxf(__uint_as_float(r[h & 31]), 0.f);
    const float s1 = fmaxf(__uint_as_float(r[(h & 31) + 1]), 0.f);
    const float2 wv = w2[h >> 1];
    unsigned long long sp, wp;
    asm("mov.b64 %0, {%1, %2};" : "=l"(sp) : "f"(s0), "f"(s1));
    asm("mov.b64 %0, {%1, %2};" : "=l"(wp) : "f"(wv.x), "f"(wv.y));
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(wp), "l"(sp));
  }
  float a0, a1;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a0), "=f"(a1) : "l"(acc));
  return a0 + a1;
}

// Operand formats: bf16 (FMT 0, rows of 256 bytes in two 128-byte swizzled
// halves), MX-FP8 (FMT 1, 128-byte rows) and MX-FP4 (FMT 2, packed, 64-byte
// rows, 64-byte swizzle); each MX K_I tile and the query block bring a
// 512-byte scale-factor tile.
template <int TOK, int FMT = 0>
struct Smem {
  static constexpr bool MX = FMT != 0;
  static constexpr int kRowB = FMT == 0 ? kDI * 2 : (FMT == 1 ? kDI : kDI / 2);
  static constexpr int kTile = kBM * kRowB;                // one K_I tile
  static constexpr int kB = TOK * kHI * kRowB;             // q_I block
  // smaller tiles: more ring slots keep as many bytes in flight
  static constexpr int kStages = Cfg<TOK>::kStages * (256 / kRowB);
  static constexpr int kChunk = Cfg<TOK>::kChunk;
  static constexpr int off_b = 0;
  static constexpr int off_a = kB;
  static constexpr int off_sf = off_a + kStages * kTile;   // MX: [kStages + 1][512] scales
  static constexpr int off_scores = off_sf + (MX ? (kStages + 1) * 512 : 0);
  static constexpr int off_w = off_scores + TOK * kChunk * 4;
  static constexpr int off_hist = off_w + TOK * kHI * 4;
  static constexpr int off_cand = off_hist + TOK * 256 * 4;   // [TOK][kBinCap] (score, index)
  static constexpr int off_red = off_cand + TOK * kBinCap * 8;  // [16] cooperative top-k
  static constexpr int off_wcnt = off_red + 64;                 // [16]
  static constexpr int off_bar = off_wcnt + 64;
  static constexpr int kBars = 2 * kStages + 6;
  static constexpr int off_misc = off_bar + kBars * 8;
  static constexpr int bytes = off_misc + 64;
};

struct TcIdxArgs {
  int64_t Tq, N;
  int m, k;
  int n_chunks;
  const float* w;
  const int64_t* q_pos;
  int32_t* idx_out;
  float* score_out;
  float* cand_score;   // [B*Tq][n_chunks][k] when n_chunks > 1 ([B*Tq][n_chunks][kChunk] direct)
  int32_t* cand_idx;
  // single-token rows whose whole score row fits one merge cluster: the chunk
  // kernel writes its raw scores (no chunk top-k) and the merge selects
  // among all of them (entry j of a row is a candidate iff j < its visible count)
  int direct;
  unsigned* status;
  // MX-FP8 operands: scale-factor tiles of q_I ([B][Tq][512], one per token)
  // and K_I ([B][ceil(N / 128)][512])
  const uint8_t* q_sf;
  const uint8_t* k_sf;
  int64_t k_sf_tiles;
};

__device__ __forceinline__ int64_t vis_count(int64_t pos, int m, int64_t N) {
  if (pos < 0) return 0;
  int64_t v = (pos + 1) / m;
  return v < N ? v : N;
}

__device__ __forceinline__ unsigned score_key(float f) {
  unsigned u = __float_as_uint(f + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Warp-level exact top-k of sc[0..n) (ties to the lower index), written in
// ascending index order as (e0 + j, sc[j]) and padded to k with (-1, -inf).
__device__ void warp_topk(const float* sc, int n, int k, int64_t e0, unsigned* hist,
                          int32_t* out_idx, float* out_score) {
  const int lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  unsigned tau = 0u, need_eq = 0u;
  bool take_all = n <= k;
  if (!take_all) {
    unsigned prefix = 0u, mask = 0u;
    unsigned rem = (unsigned)k;
    for (int shift = 24; shift >= 0; shift -= 8) {
#pragma unroll
      for (int i = 0; i < 8; ++i) hist[lane * 8 + i] = 0u;
      __syncwarp();
      for (int j = lane; j < n; j += 32) {
        unsigned key = score_key(sc[j]);
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
      }
      __syncwarp();
      // lane L owns digits 255-8L .. 248-8L (descending)
      unsigned c[8], sL = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        c[i] = hist[255 - 8 * lane - i];
        sL += c[i];
      }
      unsigned incl = sL;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        unsigned v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      unsigned pre = incl - sL;  // count of digits above this lane's group
      bool here = pre < rem && rem <= incl;
      unsigned digit = 0, above = 0;
      if (here) {
        unsigned run = pre;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (run + c[i] >= rem) {
            digit = 255u - 8u * lane - i;
            above = run;
            break;
          }
          run += c[i];
        }
      }
      unsigned who = __ballot_sync(0xffffffffu, here);
      int src = __ffs(who) - 1;
      digit = __shfl_sync(0xffffffffu, digit, src);
      above = __shfl_sync(0xffffffffu, above, src);
      prefix |= digit << shift;
      mask |= 255u << shift;
      rem -= above;
      __syncwarp();
    }
    tau = prefix;
    need_eq = rem;
  }
  unsigned run_sel = 0, run_eq = 0;
  for (int base = 0; base < n; base += 32) {
    int j = base + lane;
    bool valid = j < n;
    float s = valid ? sc[j] : 0.f;
    unsigned key = valid ? score_key(s) : 0u;
    bool take;
    if (take_all) {
      take = valid;
    } else {
      bool gt = valid && key > tau;
      bool eq = valid && key == tau;
      unsigned beq = __ballot_sync(0xffffffffu, eq);
      unsigned eq_rank = run_eq + __popc(beq & lt);
      take = gt || (eq && eq_rank < need_eq);
      run_eq += __popc(beq);
    }
    unsigned bt = __ballot_sync(0xffffffffu, take);
    unsigned at = run_sel + __popc(bt & lt);
    if (take) {
      out_idx[at] = (int32_t)(e0 + j);
      if (out_score) out_score[at] = s;
    }
    run_sel += __popc(bt);
  }
  for (int p = (int)run_sel + lane; p < k; p += 32) {
    out_idx[p] = -1;
    if (out_score) out_score[p] = -INFINITY;
  }
}

// Bin of a score in 256 equal-width value bins over [lo, hi]: a monotone map
// (a larger score never lands in a lower bin), evaluated the same way in
// every pass.
__device__ __forceinline__ int value_bin(float s, float lo, float scale) {
  const int b = (int)((s - lo) * scale);
  return b > 255 ? 255 : b;
}

// Inclusive warp prefix sum.
__device__ __forceinline__ unsigned warp_incl_scan(unsigned v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  return v;
}

// Exact warp top-k, the same selection and output as warp_topk: the scores
// are binned by value, every score in a bin above the one holding the k-th
// largest is taken, and that boundary bin's members (at most kBinCap) are
// ranked exactly by (score desc, index asc).  A heavier boundary bin (many
// equal or clustered scores) or a degenerate range falls back to the radix
// select.  Lane l reads scores 4l..4l+3 of each 128-score sweep (16-byte
// loads; sc is 16-byte aligned), so the ordered compactions use a warp
// prefix sum of per-lane counts.
__device__ void warp_topk_binned(const float* sc, int n, int k, int64_t e0, unsigned* hist,
                                 float* cs, int* cj, int32_t* out_idx, float* out_score) {
  const int lane = threadIdx.x & 31;
  if (n <= k) {
    warp_topk(sc, n, k, e0, hist, out_idx, out_score);
    return;
  }
  const float4* sc4 = reinterpret_cast<const float4*>(sc);
  const int n4 = (n + 3) >> 2;
  auto get4 = [&](int i, float* v) {   // scores 4i..4i+3, -inf past n
    const float4 q = sc4[i];
    v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (4 * i + e >= n) v[e] = -INFINITY;
  };
  // every pass takes four independent 32-float4 sweeps per step (latency
  // overlap); the ordered compactions scan the four sweeps' counts at once
  constexpr int U = 4;
  float lo = INFINITY, hi = -INFINITY;
  for (int base = 0; base < n4; base += 32 * U) {
    float v[U][4];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + 32 * u + lane;
      if (i < n4) get4(i, v[u]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (i < n4 && 4 * i + e < n) {
          lo = fminf(lo, v[u][e]);
          hi = fmaxf(hi, v[u][e]);
        }
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  const float scale = 255.99f / (hi - lo);
  if (!(hi > lo) || !(scale < INFINITY)) {
    warp_topk(sc, n, k, e0, hist, out_idx, out_score);
    return;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) hist[lane * 8 + i] = 0u;
  __syncwarp();
  for (int base = 0; base < n4; base += 32 * U) {
    int bins[U][4];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + 32 * u + lane;
      float v[4];
      if (i < n4) get4(i, v);
#pragma unroll
      for (int e = 0; e < 4; ++e)
        bins[u][e] = (i < n4 && 4 * i + e < n) ? value_bin(v[e], lo, scale) : -1;
    }
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (bins[u][e] >= 0) atomicAdd(&hist[bins[u][e]], 1u);
  }
  __syncwarp();
  // boundary bin: lane L owns bins 255-8L .. 248-8L (descending)
  unsigned c[8], sL = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    c[i] = hist[255 - 8 * lane - i];
    sL += c[i];
  }
  const unsigned incl = warp_incl_scan(sL, lane);
  const unsigned pre = incl - sL, rem = (unsigned)k;
  const bool here = pre < rem && rem <= incl;
  unsigned bstar = 0, above = 0, cnt = 0;
  if (here) {
    unsigned run = pre;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (run + c[i] >= rem) {
        bstar = 255u - 8u * lane - i;
        above = run;
        cnt = c[i];
        break;
      }
      run += c[i];
    }
  }
  const int src = __ffs(__ballot_sync(0xffffffffu, here)) - 1;
  bstar = __shfl_sync(0xffffffffu, bstar, src);
  above = __shfl_sync(0xffffffffu, above, src);
  cnt = __shfl_sync(0xffffffffu, cnt, src);
  __syncwarp();
  if (cnt > (unsigned)kBinCap) {
    warp_topk(sc, n, k, e0, hist, out_idx, out_score);
    return;
  }
  const unsigned need = rem - above;   // members of the boundary bin to take, >= 1
  // the boundary bin's members, in ascending index order
  unsigned run = 0;
  for (int base = 0; base < n4; base += 32 * U) {
    float v[U][4];
    unsigned m[U], inc[U];
    bool in[U][4];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + 32 * u + lane;
      if (i < n4) get4(i, v[u]);
      m[u] = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        in[u][e] = i < n4 && 4 * i + e < n && value_bin(v[u][e], lo, scale) == (int)bstar;
        m[u] += in[u][e] ? 1u : 0u;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) inc[u] = warp_incl_scan(m[u], lane);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      unsigned at = run + inc[u] - m[u];
      const int i = base + 32 * u + lane;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (in[u][e]) {
          cs[at] = v[u][e];
          cj[at] = 4 * i + e;
          ++at;
        }
      }
      run += __shfl_sync(0xffffffffu, inc[u], 31);
    }
  }
  __syncwarp();
  // the need-th member by (score desc, index asc) is the threshold
  float ts = 0.f;
  int tj = -1;
  for (unsigned i = lane; i < cnt; i += 32) {
    const float si = cs[i];
    const int ji = cj[i];
    unsigned rank = 0;
    for (unsigned q = 0; q < cnt; ++q) {
      const float sq = cs[q];
      rank += (sq > si || (sq == si && cj[q] < ji)) ? 1u : 0u;
    }
    if (rank == need - 1) {
      ts = si;
      tj = ji;
    }
  }
  const int own = __ffs(__ballot_sync(0xffffffffu, tj >= 0)) - 1;
  ts = __shfl_sync(0xffffffffu, ts, own);
  tj = __shfl_sync(0xffffffffu, tj, own);
  // emit in ascending index order
  unsigned run_sel = 0;
  for (int base = 0; base < n4; base += 32 * U) {
    float v[U][4];
    unsigned m[U], inc[U];
    bool take[U][4];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + 32 * u + lane;
      if (i < n4) get4(i, v[u]);
      m[u] = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = 4 * i + e;
        const bool valid = i < n4 && j < n;
        const int bv = valid ? value_bin(v[u][e], lo, scale) : -1;
        take[u][e] = valid && (bv > (int)bstar || (bv == (int)bstar &&
                                                   (v[u][e] > ts || (v[u][e] == ts && j <= tj))));
        m[u] += take[u][e] ? 1u : 0u;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) inc[u] = warp_incl_scan(m[u], lane);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      unsigned at = run_sel + inc[u] - m[u];
      const int i = base + 32 * u + lane;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (take[u][e]) {
          out_idx[at] = (int32_t)(e0 + 4 * i + e);
          if (out_score) out_score[at] = v[u][e];
          ++at;
        }
      }
      run_sel += __shfl_sync(0xffffffffu, inc[u], 31);
    }
  }
  for (int q = (int)run_sel + lane; q < k; q += 32) {
    out_idx[q] = -1;
    if (out_score) out_score[q] = -INFINITY;
  }
}

// Cooperative exact top-k of one token's scores by G warps: the same
// selection and output as warp_topk (larger score first, ties to the lower
// index, ascending output padded with (-1, -inf)).  Warp w of the group holds
// scores [w R, (w+1) R), R = kMaxN / G, in registers (lane l: 16-byte groups
// l, l+32, ...); value bins as in warp_topk_binned, a histogram in shared
// memory, the boundary bin's members ranked exactly, and an ordered emit with
// per-warp offsets.  With REFINE, a boundary bin of more than kBinCap
// members is narrowed by a radix select on its members' keys first.
// Returns false (nothing written) when the single-warp radix select must run
// instead: n <= k, a degenerate range, or (after any narrowing) more than
// kBinCap members to rank.
template <int G, int kMaxN, bool REFINE = false>
__device__ bool block_topk(const float* sc, int n, int k, int64_t e0, unsigned* hist, float* red,
                           unsigned* wcnt, float* cs, int* cj, int bar_id, int32_t* out_idx,
                           float* out_score) {
  constexpr int R = kMaxN / G;
  constexpr int V = R / 128;
  const int lane = threadIdx.x & 31;
  const int w = (threadIdx.x >> 5) % G;
  const int gt = threadIdx.x % (32 * G);
  auto sync = [&]() { named_bar(bar_id, 32 * G); };
  float v[V][4];
  float lo = INFINITY, hi = -INFINITY;
#pragma unroll
  for (int i = 0; i < V; ++i) {
    const int j0 = w * R + 4 * (32 * i + lane);
    const float4 q = *reinterpret_cast<const float4*>(sc + j0);
    v[i][0] = q.x; v[i][1] = q.y; v[i][2] = q.z; v[i][3] = q.w;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (j0 + e < n) {
        lo = fminf(lo, v[i][e]);
        hi = fmaxf(hi, v[i][e]);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  for (int i = gt; i < 256; i += 32 * G) hist[i] = 0u;
  if (lane == 0) {
    red[w] = lo;
    red[G + w] = hi;
  }
  sync();
#pragma unroll
  for (int i = 0; i < G; ++i) {
    lo = fminf(lo, red[i]);
    hi = fmaxf(hi, red[G + i]);
  }
  const float scale = 255.99f / (hi - lo);
  if (n <= k || !(hi > lo) || !(scale < INFINITY)) return false;
  int bin[V][4];
#pragma unroll
  for (int i = 0; i < V; ++i) {
    const int j0 = w * R + 4 * (32 * i + lane);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      bin[i][e] = j0 + e < n ? value_bin(v[i][e], lo, scale) : -1;
      if (bin[i][e] >= 0) atomicAdd(&hist[bin[i][e]], 1u);
    }
  }
  sync();
  if (w == 0) {   // boundary bin: lane L owns bins 255-8L .. 248-8L (descending)
    unsigned c[8], sL = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      c[i] = hist[255 - 8 * lane - i];
      sL += c[i];
    }
    const unsigned incl = warp_incl_scan(sL, lane);
    const unsigned pre = incl - sL, rem = (unsigned)k;
    if (pre < rem && rem <= incl) {
      unsigned run = pre;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (run + c[i] >= rem) {
          wcnt[G] = 255u - 8u * lane - i;   // boundary bin
          wcnt[G + 1] = run;                // scores above it
          wcnt[G + 2] = c[i];               // its members
          break;
        }
        run += c[i];
      }
    }
    if (lane == 0) wcnt[G + 3] = 0u;        // member slots used
  }
  sync();
  const int bstar = (int)wcnt[G];
  unsigned need = (unsigned)k - wcnt[G + 1], cnt = wcnt[G + 2];
  // A heavier boundary bin is narrowed by a radix select on the members'
  // order-preserving keys (8 bits a pass, every warp of the group counting
  // its own members): afterwards the members whose key equals tau, the key
  // of the need-th largest member, are the ones ranked below, need of them
  // taken (those above tau are taken by value).
  const bool heavy = cnt > (unsigned)kBinCap;
  if (heavy && !REFINE) return false;
  unsigned tau = 0u;
  if (heavy) {
    unsigned mask = 0u;
    for (int shift = 24; shift >= 0; shift -= 8) {
      sync();   // the previous readers of hist and of the boundary slots are done
      for (int i = gt; i < 256; i += 32 * G) hist[i] = 0u;
      sync();
#pragma unroll
      for (int i = 0; i < V; ++i) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (bin[i][e] == bstar) {
            const unsigned key = score_key(v[i][e]);
            if ((key & mask) == tau) atomicAdd(&hist[(key >> shift) & 255u], 1u);
          }
        }
      }
      sync();
      if (w == 0) {   // boundary digit: lane L owns digits 255-8L .. 248-8L
        unsigned c[8], sL = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          c[i] = hist[255 - 8 * lane - i];
          sL += c[i];
        }
        const unsigned incl = warp_incl_scan(sL, lane);
        const unsigned pre = incl - sL;
        if (pre < need && need <= incl) {
          unsigned run = pre;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            if (run + c[i] >= need) {
              wcnt[G] = 255u - 8u * lane - i;   // digit
              wcnt[G + 1] = run;                // members above it
              wcnt[G + 2] = c[i];               // members with it
              break;
            }
            run += c[i];
          }
        }
      }
      sync();
      tau |= wcnt[G] << shift;
      mask |= 255u << shift;
      need -= wcnt[G + 1];
      cnt = wcnt[G + 2];
    }
    // cnt members carry the key tau exactly; more than kBinCap equal
    // scores go to the radix select over all scores
    if (cnt > (unsigned)kBinCap) return false;
  }
  // the members to rank, any order
#pragma unroll
  for (int i = 0; i < V; ++i) {
    const int j0 = w * R + 4 * (32 * i + lane);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (bin[i][e] == bstar && (!heavy || score_key(v[i][e]) == tau)) {
        const unsigned at = atomicAdd(&wcnt[G + 3], 1u);
        cs[at] = v[i][e];
        cj[at] = j0 + e;
      }
    }
  }
  sync();
  // the need-th member by (score desc, index asc) is the threshold
  for (unsigned i = gt; i < cnt; i += 32 * G) {
    const float si = cs[i];
    const int ji = cj[i];
    unsigned rank = 0;
    for (unsigned q = 0; q < cnt; ++q) {
      const float sq = cs[q];
      rank += (sq > si || (sq == si && cj[q] < ji)) ? 1u : 0u;
    }
    if (rank == need - 1) {   // exactly one member
      red[2 * G] = si;
      reinterpret_cast<int*>(red)[2 * G + 1] = ji;
    }
  }
  sync();
  const float ts = red[2 * G];
  const int tj = reinterpret_cast<const int*>(red)[2 * G + 1];
  unsigned mine = 0;
#pragma unroll
  for (int i = 0; i < V; ++i) {
    const int j0 = w * R + 4 * (32 * i + lane);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = j0 + e;
      const bool take = bin[i][e] > bstar ||
                        (bin[i][e] == bstar && (v[i][e] > ts || (v[i][e] == ts && j <= tj)));
      mine += take ? 1u : 0u;
      bin[i][e] = take ? 1 : 0;   // from here: the take flag
    }
  }
  unsigned wtot = mine;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) wtot += __shfl_xor_sync(0xffffffffu, wtot, o);
  if (lane == 0) wcnt[w] = wtot;
  sync();
  unsigned run = 0;
#pragma unroll
  for (int i = 0; i < G; ++i) run += i < w ? wcnt[i] : 0u;
#pragma unroll
  for (int i = 0; i < V; ++i) {
    unsigned m = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) m += (unsigned)bin[i][e];
    const unsigned inc = warp_incl_scan(m, lane);
    unsigned at = run + inc - m;
    const int j0 = w * R + 4 * (32 * i + lane);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (bin[i][e]) {
        out_idx[at] = (int32_t)(e0 + j0 + e);
        if (out_score) out_score[at] = v[i][e];
        ++at;
      }
    }
    run += __shfl_sync(0xffffffffu, inc, 31);
  }
  sync();   // every read of the group's scratch is done before it is reused
  return true;
}

// Block-wide exclusive prefix sum of one value per thread (up to 1024 threads).
__device__ __forceinline__ unsigned block_excl_scan(unsigned v, unsigned* tmp, unsigned* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const unsigned incl = warp_incl_scan(v, lane);
  __syncthreads();
  if (lane == 31) tmp[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    const unsigned wv = lane < (int)(blockDim.x >> 5) ? tmp[lane] : 0u;
    const unsigned wi = warp_incl_scan(wv, lane);
    tmp[lane] = wi - wv;
    if (lane == 31) tmp[32] = wi;
  }
  __syncthreads();
  *total = tmp[32];
  return tmp[wid] + incl - v;
}

// ---------------------------------------------------------------------------
// Cluster top-k: exact selection of the k largest of a list split over the
// CTAs of a cluster, in order (CTA rank, then thread, then element), each
// thread holding R of them in registers (id < 0: not a candidate).  The keys
// are the scores' order-preserving 32-bit images; a radix select on them
// starts below the bits that every valid key shares (the cluster-wide key
// minimum and maximum fix those) and takes at most 11 bits a pass (at most
// three passes), so a pass spreads its keys over up to 2048 bins.  Each CTA
// counts its own keys; every CTA sums the cluster's counts through
// distributed shared memory and so takes the same decisions, and a pass ends
// the select early once the boundary bucket is taken whole.  A candidate is
// then taken if its key prefix is above the boundary, or equal to it and
// among the first `rem` such candidates in list order (ties to the lower
// index, since the list is in ascending index order); one exchange of per-CTA
// (above, equal) counts gives every CTA its output offset, and the output is
// ascending, padded with (-1, -inf).  Every CTA of the cluster runs this with
// all of its threads, which all take the same barriers.
// ---------------------------------------------------------------------------
constexpr int kSelBins = 2048;
constexpr int kSelMaxCluster = 8;   // portable cluster size

struct SelShared {
  unsigned hist[3][kSelBins];   // this CTA's counts, one buffer per pass (read remotely)
  unsigned red[3][32];          // per-warp count / key min / key max (read remotely)
  unsigned tot;                 // packed (above | equal << 16) counts (read remotely)
  unsigned tmp[33];
  unsigned glob[3];
  unsigned dec[3];              // boundary digit, count above it, its bucket size
  unsigned base[2];             // equal-key members before this CTA, output offset
};

template <int R, int NT>
__device__ void cluster_topk_emit(const float (&v)[R], const int32_t (&id)[R], int k,
                                  SelShared& sh, int32_t* out, float* so) {
  static_assert(R * NT < 65536, "per-CTA counts are packed in 16 bits");
  static_assert(NT * 4 == kSelBins, "four bins per thread in the bucket search");
  const uint32_t CL = cluster_nctarank(), rank = cluster_ctarank();
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  constexpr int NW = NT / 32;
  if (k <= 0) return;   // uniform over the cluster
  // a cluster of one CTA: CTA barriers and local loads do
  const bool solo = CL == 1;
  auto csync = [&]() {
    if (solo) __syncthreads(); else cluster_sync();
  };
  auto rd = [&](const unsigned* local, uint32_t r) -> unsigned {
    return solo ? *reinterpret_cast<const volatile unsigned*>(local) : dsmem_ld_u32(local, r);
  };

  for (int i = tid; i < 3 * kSelBins; i += NT) (&sh.hist[0][0])[i] = 0u;
  unsigned cnt = 0, kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
  for (int e = 0; e < R; ++e) {
    if (id[e] >= 0) {
      const unsigned key = score_key(v[e]);
      ++cnt;
      kmin = min(kmin, key);
      kmax = max(kmax, key);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  if (lane == 0) {
    sh.red[0][wid] = cnt;
    sh.red[1][wid] = kmin;
    sh.red[2][wid] = kmax;
  }
  csync();
  if (wid == 0) {
    unsigned c = 0, lo = 0xffffffffu, hi = 0u;
    for (int i = lane; i < (int)CL * NW; i += 32) {
      const uint32_t r = (uint32_t)(i / NW);
      const int w = i % NW;
      c += rd(&sh.red[0][w], r);
      lo = min(lo, rd(&sh.red[1][w], r));
      hi = max(hi, rd(&sh.red[2][w], r));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      c += __shfl_xor_sync(0xffffffffu, c, o);
      lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if (lane == 0) {
      sh.glob[0] = c;
      sh.glob[1] = lo;
      sh.glob[2] = hi;
    }
  }
  __syncthreads();
  const unsigned n_valid = sh.glob[0];
  const bool take_all = n_valid <= (unsigned)k;

  // after the select the taken candidates are those whose key prefix
  // (key & M) is above P, and the first `rem` (in list order) equal to it
  unsigned P = 0u, M = 0u, rem = (unsigned)k;
  if (!take_all) {
    const unsigned gmin = sh.glob[1], gmax = sh.glob[2];
    const unsigned diff = gmin ^ gmax;
    int hb = diff ? 31 - __clz((int)diff) : -1;   // highest bit where valid keys differ
    M = hb < 0 ? 0xffffffffu : (hb == 31 ? 0u : ~((2u << hb) - 1u));
    P = gmin & M;
    for (int pass = 0; hb >= 0; ++pass) {   // uniform over the cluster; at most 3 passes
      const int shift = hb + 1 > 11 ? hb + 1 - 11 : 0;
      const unsigned dmask = (1u << (hb + 1 - shift)) - 1u;
      unsigned* h = sh.hist[pass];
#pragma unroll
      for (int e = 0; e < R; ++e) {
        if (id[e] >= 0) {
          const unsigned key = score_key(v[e]);
          if ((key & M) == P) atomicAdd(&h[(key >> shift) & dmask], 1u);
        }
      }
      csync();
      // bucket search: thread t owns bins 2047-4t .. 2044-4t (descending),
      // summed over the cluster (every rank's load issued before any is used)
      uint4 x[kSelMaxCluster];
      if (solo) {
        x[0] = *reinterpret_cast<const uint4*>(&h[kSelBins - 4 * (tid + 1)]);
      } else {
#pragma unroll
        for (int r = 0; r < kSelMaxCluster; ++r)
          if ((uint32_t)r < CL) x[r] = dsmem_ld_u32x4(&h[kSelBins - 4 * (tid + 1)], (uint32_t)r);
      }
      unsigned c[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int r = 0; r < kSelMaxCluster; ++r) {
        if ((uint32_t)r < CL) {
          c[0] += x[r].w;
          c[1] += x[r].z;
          c[2] += x[r].y;
          c[3] += x[r].x;
        }
      }
      const unsigned sT = c[0] + c[1] + c[2] + c[3];
      unsigned total;
      const unsigned above = block_excl_scan(sT, sh.tmp, &total);
      if (above < rem && rem <= above + sT) {
        unsigned run = above;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if (run + c[i] >= rem) {
            sh.dec[0] = (unsigned)(kSelBins - 1 - 4 * tid - i);
            sh.dec[1] = run;
            sh.dec[2] = c[i];
            break;
          }
          run += c[i];
        }
      }
      __syncthreads();
      const unsigned d = sh.dec[0], bucket = sh.dec[2];
      rem -= sh.dec[1];
      P |= d << shift;
      M |= dmask << shift;
      if (bucket == rem) break;   // the whole bucket is taken
      hb = shift - 1;
    }
  }

  // ordered emit
  unsigned gt = 0, eq = 0;
#pragma unroll
  for (int e = 0; e < R; ++e) {
    if (id[e] >= 0) {
      const unsigned km = score_key(v[e]) & M;
      gt += km > P ? 1u : 0u;
      eq += km == P ? 1u : 0u;
    }
  }
  unsigned tot;
  const unsigned excl = block_excl_scan(gt | (eq << 16), sh.tmp, &tot);
  if (tid == 0) sh.tot = tot;
  csync();
  if (wid == 0) {   // output offset: the lower-ranked CTAs' taken counts, in order
    const unsigned t = (uint32_t)lane < rank ? rd(&sh.tot, lane) : 0u;
    unsigned eq_before = 0u, out_before = 0u;
    for (uint32_t r = 0; r < rank; ++r) {
      const unsigned tr = __shfl_sync(0xffffffffu, t, (int)r);
      const unsigned q = tr >> 16;
      const unsigned left = rem > eq_before ? rem - eq_before : 0u;
      out_before += (tr & 0xffffu) + min(left, q);
      eq_before += q;
    }
    if (lane == 0) {
      sh.base[0] = eq_before;
      sh.base[1] = out_before;
    }
  }
  __syncthreads();
  if (!solo) cluster_arrive();   // this CTA's remote reads are done
  const unsigned eq_base = sh.base[0];
  const unsigned left = rem > eq_base ? rem - eq_base : 0u;
  unsigned at = sh.base[1] + (excl & 0xffffu) + min(left, excl >> 16);
  unsigned eq_rank = eq_base + (excl >> 16);
#pragma unroll
  for (int e = 0; e < R; ++e) {
    if (id[e] >= 0) {
      const unsigned km = score_key(v[e]) & M;
      bool take = km > P;
      if (km == P) {
        take = eq_rank < rem;
        ++eq_rank;
      }
      if (take) {
        out[at] = id[e];
        if (so) so[at] = v[e];
        ++at;
      }
    }
  }
  if (rank == 0) {   // padding after the taken ones
    const unsigned taken = take_all ? n_valid : (unsigned)k;
    for (int p = (int)taken + tid; p < k; p += NT) {
      out[p] = -1;
      if (so) so[p] = -INFINITY;
    }
  }
  if (!solo) cluster_wait();   // no CTA leaves while another may still read its shared memory
}

template <int TOK, int FMT>
__global__ void __launch_bounds__(kThreads, TOK == 1 ? 2 : 1)
    indexer_tc_kernel(const __grid_constant__ CUtensorMap map_q,
                      const __grid_constant__ CUtensorMap map_k, TcIdxArgs a) {
  constexpr bool MX = FMT != 0;
  static_assert(!MX || TOK == 1, "MX operands: single-token groups");
  using L = Smem<TOK, FMT>;
  constexpr int kStages = L::kStages;
  constexpr int kChunk = L::kChunk;
  constexpr int kTile = L::kTile;
  constexpr int kN = TOK * kHI;                 // MMA N
  // two accumulators; MX adds two 4-column K_I scale buffers and the query's
  // scale tile (4 columns), rounded up to a power of two
  constexpr uint32_t kCols = MX ? 256 : 2 * kN;
  constexpr uint32_t kSfa = 2 * kN;
  constexpr uint32_t kSfb = kSfa + 8;
  constexpr uint32_t kIdesc = idesc_bf16_f32(kBM, kN, 0, 0);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sB = sm + L::off_b;
  uint8_t* sA = sm + L::off_a;
  float* scores = reinterpret_cast<float*>(sm + L::off_scores);
  float* sw = reinterpret_cast<float*>(sm + L::off_w);
  unsigned* hist = reinterpret_cast<unsigned*>(sm + L::off_hist);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::off_bar);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* tfull = bars + 2 * kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* bfull = tempty + 2;
  uint64_t* drain = bfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::off_misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::off_misc + 4);

  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x;
  const int group = gridDim.y - 1 - blockIdx.y;   // heaviest causal groups first
  const int b = blockIdx.z;
  const int64_t t0 = (int64_t)group * TOK;
  const int64_t e0 = (int64_t)chunk * kChunk;

  // visibility of the TOK tokens and the entry range this CTA scores
  int64_t vis[TOK];
  int64_t vmax = 0;
#pragma unroll
  for (int i = 0; i < TOK; ++i) {
    int64_t t = t0 + i;
    vis[i] = 0;
    if (t < a.Tq) {
      int64_t row = (int64_t)b * a.Tq + t;
      int64_t pos = a.q_pos ? a.q_pos[row] : t;
      vis[i] = vis_count(pos, a.m, a.N);
    }
    vmax = vis[i] > vmax ? vis[i] : vmax;
  }
  int64_t e_hi = e0 + kChunk < vmax ? e0 + kChunk : vmax;
  const int n_tiles = e_hi > e0 ? (int)((e_hi - e0 + kBM - 1) / kBM) : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 128);
    }
    mbar_init(bfull, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
    if (n_tiles > 0) {   // the q_I block first: its latency overlaps the rest of the setup
      tma_prefetch_desc(&map_q);
      tma_prefetch_desc(&map_k);
      const int32_t qrow = (int32_t)(t0 * kHI);
      if constexpr (MX) {
        // codes (128 bytes a row, one box) and the scale tile holding this token's rows
        mbar_arrive_expect_tx(bfull, L::kB + 512);
        tma_load_3d(sB, &map_q, bfull, 0, qrow, b);
        bulk_load(smem_u32(sm + L::off_sf + kStages * 512),
                  a.q_sf + ((int64_t)b * a.Tq + t0) * 512, 512, bfull);
      } else {
        mbar_arrive_expect_tx(bfull, L::kB);
        tma_load_3d(sB, &map_q, bfull, 0, qrow, b);
        tma_load_3d(sB + L::kB / 2, &map_q, bfull, 64, qrow, b);
      }
    }
  }
  for (int i = threadIdx.x; i < TOK * kHI; i += blockDim.x) {
    int64_t t = t0 + i / kHI;
    sw[i] = t < a.Tq ? a.w[((int64_t)b * a.Tq + t) * kHI + (i % kHI)] : 0.f;
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- TMA producer
    if (n_tiles > 0 && elect_one()) {
      int issued = 0;
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i % kStages;
        const uint32_t ph = (uint32_t)(i / kStages) & 1u;
        if (*abort_flag || !mbar_wait(&empty[s], ph ^ 1u)) {
          *abort_flag = 1;
          report(a.status, CSA_DEV_TIMEOUT, 1u);
          break;
        }
        const int32_t erow = (int32_t)(e0 + (int64_t)i * kBM);
        if constexpr (MX) {
          mbar_arrive_expect_tx(&full[s], kTile + 512);
          tma_load_3d(sA + s * kTile, &map_k, &full[s], 0, erow, b);
          bulk_load(smem_u32(sm + L::off_sf + s * 512),
                    a.k_sf + ((int64_t)b * a.k_sf_tiles + erow / kBM) * 512, 512, &full[s]);
        } else {
          mbar_arrive_expect_tx(&full[s], kTileBytes);
          uint8_t* dst = sA + s * kTileBytes;
          tma_load_3d(dst, &map_k, &full[s], 0, erow, b);
          tma_load_3d(dst + kTileBytes / 2, &map_k, &full[s], 64, erow, b);
        }
        issued = i + 1;
      }
      // drain: every issued copy has landed before the CTA may exit
      for (int i = issued - kStages > 0 ? issued - kStages : 0; i < issued; ++i)
        mbar_wait(&full[i % kStages], (uint32_t)(i / kStages) & 1u);
      mbar_wait(bfull, 0);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (n_tiles > 0 && elect_one()) {
      if (!mbar_wait(bfull, 0)) {
        *abort_flag = 1;
        report(a.status, CSA_DEV_TIMEOUT, 2u);
      } else {
        const uint32_t b_base = smem_u32(sB);
        const uint32_t a_base = smem_u32(sA);
        if constexpr (MX) {
          // the query's scale tile into TMEM (rows 32 j + l: lane l, column j)
          tmem_cp_32x128b_x4(tmem + kSfb,
                             smem_desc(smem_u32(sm + L::off_sf + kStages * 512), 16, 128, 0));
        }
        for (int i = 0; i < n_tiles; ++i) {
          const int s = i % kStages;
          const uint32_t ph = (uint32_t)(i / kStages) & 1u;
          const int buf = i & 1;
          const uint32_t bph = (uint32_t)(i >> 1) & 1u;
          if (*abort_flag || !mbar_wait(&full[s], ph) || !mbar_wait(&tempty[buf], bph ^ 1u)) {
            *abort_flag = 1;
            report(a.status, CSA_DEV_TIMEOUT, 3u);
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem + (uint32_t)(buf * kN);
          if constexpr (MX) {
            // this tile's K_I scales into TMEM (issued before, and executed
            // before, the MMAs below that read them)
            const uint32_t sfa = tmem + kSfa + 4u * (uint32_t)buf;
            tmem_cp_32x128b_x4(sfa, smem_desc(smem_u32(sm + L::off_sf + s * 512), 16, 128, 0));
            const uint32_t sfb = tmem + kSfb;   // the token's own tile: heads on rows 0..63
            if constexpr (FMT == 1) {
#pragma unroll
              for (int kk = 0; kk < kDI / 32; ++kk) {   // K = 32 per MMA, one scale each
                const uint64_t ad = smem_desc(a_base + s * kTile + kk * 32, 16, 1024, 2);
                const uint64_t bd = smem_desc(b_base + kk * 32, 16, 1024, 2);
                mma_mxf8_ss(d, ad, bd, idesc_mxf8_e4m3(kBM, kN, kk, kk),
                            sfa | ((uint32_t)kk << 30), sfb | ((uint32_t)kk << 30),
                            kk > 0 ? 1u : 0u);
              }
            } else {
              // K = 64 per MMA (32 bytes of the 64-byte row), two scales each:
              // bytes 2 kk and 2 kk + 1 of the scale words
#pragma unroll
              for (int kk = 0; kk < kDI / 64; ++kk) {
                const uint64_t ad = smem_desc(a_base + s * kTile + kk * 32, 16, 512, 4);
                const uint64_t bd = smem_desc(b_base + kk * 32, 16, 512, 4);
                mma_mxf4_ss(d, ad, bd, idesc_mxf4_e2m1(kBM, kN, 2 * kk, 2 * kk),
                            sfa | ((uint32_t)(2 * kk) << 30), sfb | ((uint32_t)(2 * kk) << 30),
                            kk > 0 ? 1u : 0u);
              }
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < kDI / 16; ++kk) {
              const uint32_t koff = (uint32_t)((kk & 3) * 32);  // 16 bf16 per K step
              uint64_t ad = smem_desc(a_base + s * kTileBytes + (kk >> 2) * (kTileBytes / 2) +
                                          koff, 16, 1024, 2);
              uint64_t bd = smem_desc(b_base + (kk >> 2) * (L::kB / 2) + koff, 16, 1024, 2);
              mma_bf16_ss(d, ad, bd, kIdesc, kk > 0 ? 1u : 0u);
            }
          }
          mma_commit(&empty[s]);
          mma_commit(&tfull[buf]);
        }
      }
      mma_commit(drain);
      mbar_wait(drain, 0);
    }
  } else {
    // ---------------- epilogue: thread <-> TMEM lane <-> entry
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    for (int i = 0; i < n_tiles; ++i) {
      const int buf = i & 1;
      const uint32_t bph = (uint32_t)(i >> 1) & 1u;
      if (*abort_flag || !mbar_wait(&tfull[buf], bph)) {
        *abort_flag = 1;
        report(a.status, CSA_DEV_TIMEOUT, 4u);
        break;
      }
      tc_fence_after();
      const uint32_t base = tmem_addr(tmem, (uint32_t)(quarter * 32), (uint32_t)(buf * kN));
#pragma unroll
      for (int t = 0; t < TOK; ++t) {
        uint32_t r0[32], r1[32];
        tmem_ld32(base + t * kHI, r0);
        tmem_ld32(base + t * kHI + 32, r1);
        tmem_ld_wait();
        const float sc = relu_weighted_sum64(sw + t * kHI, r0, r1);
        if (TOK == 1 && a.direct)
          a.cand_score[(((int64_t)b * a.Tq + t0) * a.n_chunks + chunk) * kChunk + i * kBM + row] = sc;
        else
          scores[t * kChunk + i * kBM + row] = sc;
      }
      tc_fence_before();
      mbar_arrive(&tempty[buf]);
    }
  }

  __syncthreads();

  // ---------------- top-k: one warp per token (none when the merge selects
  // from the raw scores)
  if (TOK == 1 && warp >= 2 && !*abort_flag && !a.direct) {
    // one token: the four epilogue warps select together (named barrier 1)
    const int64_t tok = t0;
    if (tok < a.Tq) {
      const int64_t row = (int64_t)b * a.Tq + tok;
      int64_t n64 = vis[0] - e0;
      n64 = n64 < 0 ? 0 : (n64 > kChunk ? kChunk : n64);
      int32_t* oi;
      float* os;
      if (a.n_chunks == 1) {
        oi = a.idx_out + row * a.k;
        os = a.score_out ? a.score_out + row * a.k : nullptr;
      } else {
        const int64_t c = (row * a.n_chunks + chunk) * a.k;
        oi = a.cand_idx + c;
        os = a.cand_score + c;
      }
      float* cand = reinterpret_cast<float*>(sm + L::off_cand);
      const bool done = block_topk<4, kChunk, true>(
          scores, (int)n64, a.k, e0, hist, reinterpret_cast<float*>(sm + L::off_red),
          reinterpret_cast<unsigned*>(sm + L::off_wcnt), cand,
          reinterpret_cast<int*>(cand + kBinCap), 1, oi, os);
      if (!done) {
        if (warp == 2) warp_topk(scores, (int)n64, a.k, e0, hist, oi, os);
        named_bar(1, 128);
      }
    }
  } else if (TOK > 1 && warp >= 2 && warp < 2 + TOK && !*abort_flag) {
    const int t = warp - 2;
    const int64_t tok = t0 + t;
    if (tok < a.Tq) {
      const int64_t row = (int64_t)b * a.Tq + tok;
      int64_t n64 = vis[t] - e0;
      n64 = n64 < 0 ? 0 : (n64 > kChunk ? kChunk : n64);
      const int n = (int)n64;
      int32_t* oi;
      float* os;
      if (a.n_chunks == 1) {
        oi = a.idx_out + row * a.k;
        os = a.score_out ? a.score_out + row * a.k : nullptr;
      } else {
        const int64_t c = (row * a.n_chunks + chunk) * a.k;
        oi = a.cand_idx + c;
        os = a.cand_score + c;
      }
      float* cand = reinterpret_cast<float*>(sm + L::off_cand) + t * 2 * kBinCap;
      warp_topk_binned(scores + t * kChunk, n, a.k, e0, hist + t * 256, cand,
                       reinterpret_cast<int*>(cand + kBinCap), oi, os);
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
}

// ---------------------------------------------------------------------------
// Prefill form (4-token groups): persistent CTAs walk (chunk, group) units,
// heaviest causal groups first, and the top-k of one unit runs on its own
// warps while the next unit's tiles stream through the tensor core.
//   warp 0        TMA producer: the unit's q_I block, K_I tiles (2-slot ring)
//   warp 1        TMEM owner, single-thread MMA issuer (8 MMAs per tile)
//   warps 2-5     epilogue: TMEM -> sum_h w ReLU(.) -> the unit's score buffer
//   warps 6-13    top-k, two warps per token (block_topk), on the previous
//                 unit's score buffer (two buffers alternate)
// ---------------------------------------------------------------------------
constexpr int kPTok = 4;
constexpr int kPChunk = 2048;
constexpr int kPN = kPTok * kHI;                  // MMA N = 256
constexpr int kPStages = 2;
constexpr int kPTopkWarps = 2;                    // warps per token in the top-k
constexpr int kPThreads = 32 * (6 + kPTok * kPTopkWarps);   // 448

struct PSmem {
  static constexpr int kB = kPTok * kHI * kDI * 2;              // q_I block, 64 KB
  static constexpr int off_b = 0;
  static constexpr int off_a = kB;                               // K_I tile ring
  static constexpr int off_scores = off_a + kPStages * kTileBytes;   // [2][4][2048] fp32
  static constexpr int off_w = off_scores + 2 * kPTok * kPChunk * 4; // [2][4][64] fp32
  static constexpr int off_hist = off_w + 2 * kPTok * kHI * 4;       // [4][256]
  static constexpr int off_red = off_hist + kPTok * 256 * 4;         // [4][8] fp32
  static constexpr int off_wcnt = off_red + kPTok * 8 * 4;           // [4][8]
  static constexpr int off_cand = off_wcnt + kPTok * 8 * 4;          // [4][kBinCap] (score, index)
  static constexpr int off_bar = off_cand + kPTok * kBinCap * 8;
  static constexpr int kBars = 2 * kPStages + 12;
  static constexpr int off_misc = off_bar + kBars * 8;
  static constexpr int bytes = off_misc + 64;
};
static_assert(PSmem::bytes + 1024 <= 232448, "shared memory budget");


struct PUnit {
  int64_t b, group, chunk, e0;
  int n_tiles;
  int64_t vis[kPTok];
};

// Unit u: heaviest causal groups first (u = (b * n_groups + gi) * n_chunks + c,
// group = n_groups - 1 - gi).  Every role derives it the same way.
__device__ __forceinline__ PUnit punit(const TcIdxArgs& a, int64_t u, int64_t n_groups) {
  PUnit x;
  x.chunk = u % a.n_chunks;
  const int64_t r = u / a.n_chunks;
  x.group = n_groups - 1 - r % n_groups;
  x.b = r / n_groups;
  x.e0 = x.chunk * kPChunk;
  int64_t vmax = 0;
#pragma unroll
  for (int i = 0; i < kPTok; ++i) {
    const int64_t t = x.group * kPTok + i;
    x.vis[i] = 0;
    if (t < a.Tq) {
      const int64_t row = x.b * a.Tq + t;
      const int64_t pos = a.q_pos ? a.q_pos[row] : t;
      x.vis[i] = vis_count(pos, a.m, a.N);
    }
    vmax = x.vis[i] > vmax ? x.vis[i] : vmax;
  }
  const int64_t e_hi = x.e0 + kPChunk < vmax ? x.e0 + kPChunk : vmax;
  x.n_tiles = e_hi > x.e0 ? (int)((e_hi - x.e0 + kBM - 1) / kBM) : 0;
  return x;
}

__global__ void __launch_bounds__(kPThreads, 1)
    indexer_persist_kernel(const __grid_constant__ CUtensorMap map_q,
                           const __grid_constant__ CUtensorMap map_k, TcIdxArgs a,
                           int64_t n_units, int64_t n_groups) {
  using L = PSmem;
  constexpr uint32_t kCols = 2 * kPN;   // two accumulators
  constexpr uint32_t kIdesc = idesc_bf16_f32(kBM, kPN, 0, 0);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sB = sm + L::off_b;
  uint8_t* sA = sm + L::off_a;
  float* scores = reinterpret_cast<float*>(sm + L::off_scores);
  float* sw = reinterpret_cast<float*>(sm + L::off_w);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::off_bar);
  uint64_t* full = bars;                   // [2] K_I tile landed (TMA)
  uint64_t* empty = bars + kPStages;       // [2] tile consumed (MMA)
  uint64_t* tfull = bars + 2 * kPStages;   // [2] accumulator ready (MMA)
  uint64_t* tempty = tfull + 2;            // [2] accumulator read (128 epilogue threads)
  uint64_t* qfull = tempty + 2;            // the unit's q_I block landed (TMA)
  uint64_t* qfree = qfull + 1;             // the unit's last MMA done
  uint64_t* sready = qfree + 1;            // [2] score buffer complete (128 epilogue threads)
  uint64_t* sfree = sready + 2;            // [2] score buffer consumed (8 top-k warps)
  uint64_t* drain = sfree + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::off_misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::off_misc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 128);
      mbar_init(&sready[i], 128);
      mbar_init(&sfree[i], kPTok * kPTopkWarps);
    }
    mbar_init(qfull, 1);
    mbar_init(qfree, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&map_q);
    tma_prefetch_desc(&map_k);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // a timed-out wait marks the thread dead (warp-uniform); dead threads skip
  // work and waits but pass every named barrier
  bool dead = false;
  auto wait_or_die = [&](uint64_t* bar, uint32_t parity, unsigned code) {
    if (!dead) {
      if (!mbar_wait(bar, parity)) {
        *abort_flag = 1;
        report(a.status, CSA_DEV_TIMEOUT, code);
        dead = true;
      }
      dead = dead || *abort_flag;
    }
    dead = __any_sync(0xffffffffu, dead);
  };

  if (warp == 0) {
    // ---------------- TMA producer
    if (elect_one()) {
      int64_t tile = 0;   // tiles issued so far
      int nq = 0;         // q_I blocks loaded so far
      for (int64_t u = blockIdx.x; u < n_units && !dead; u += gridDim.x) {
        const PUnit x = punit(a, u, n_groups);
        if (x.n_tiles == 0) continue;
        if (nq > 0 && !mbar_wait(qfree, (uint32_t)(nq - 1) & 1u)) { dead = true; break; }
        mbar_arrive_expect_tx(qfull, L::kB);
        const int32_t qrow = (int32_t)(x.group * kPTok * kHI);
        tma_load_3d(sB, &map_q, qfull, 0, qrow, (int32_t)x.b);
        tma_load_3d(sB + L::kB / 2, &map_q, qfull, 64, qrow, (int32_t)x.b);
        ++nq;
        for (int i = 0; i < x.n_tiles; ++i, ++tile) {
          const int s = (int)(tile % kPStages);
          if (*abort_flag || !mbar_wait(&empty[s], (uint32_t)((tile / kPStages) & 1) ^ 1u)) {
            dead = true;
            break;
          }
          mbar_arrive_expect_tx(&full[s], kTileBytes);
          uint8_t* dst = sA + s * kTileBytes;
          const int32_t erow = (int32_t)(x.e0 + (int64_t)i * kBM);
          tma_load_3d(dst, &map_k, &full[s], 0, erow, (int32_t)x.b);
          tma_load_3d(dst + kTileBytes / 2, &map_k, &full[s], 64, erow, (int32_t)x.b);
        }
      }
      if (dead) {
        *abort_flag = 1;
        report(a.status, CSA_DEV_TIMEOUT, 1u);
      }
      // drain: the last issued copies land before the CTA may exit
      for (int64_t t = tile - kPStages > 0 ? tile - kPStages : 0; t < tile; ++t)
        mbar_wait(&full[t % kPStages], (uint32_t)((t / kPStages) & 1));
      if (nq > 0) mbar_wait(qfull, (uint32_t)(nq - 1) & 1u);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (elect_one()) {
      const uint64_t dA = smem_desc(smem_u32(sA), 16, 1024, 2);
      const uint64_t dB = smem_desc(smem_u32(sB), 16, 1024, 2);
      int64_t tile = 0;
      int nq = 0;
      bool ok = true;
      for (int64_t u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
        const PUnit x = punit(a, u, n_groups);
        if (x.n_tiles == 0) continue;
        if (*abort_flag || !mbar_wait(qfull, (uint32_t)nq & 1u)) { ok = false; break; }
        ++nq;
        for (int i = 0; i < x.n_tiles; ++i, ++tile) {
          const int s = (int)(tile % kPStages);
          const int buf = (int)(tile & 1);
          if (*abort_flag || !mbar_wait(&full[s], (uint32_t)((tile / kPStages) & 1)) ||
              !mbar_wait(&tempty[buf], (uint32_t)((tile >> 1) & 1) ^ 1u)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem + (uint32_t)(buf * kPN);
          const uint64_t dAs = dA + (uint64_t)((s * kTileBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < kDI / 16; ++kk)
            mma_bf16_ss(d, dAs + (uint64_t)(((kk >> 2) * (kTileBytes / 2) + (kk & 3) * 32) >> 4),
                        dB + (uint64_t)(((kk >> 2) * (L::kB / 2) + (kk & 3) * 32) >> 4), kIdesc,
                        kk > 0 ? 1u : 0u);
          mma_commit(&empty[s]);
          mma_commit(&tfull[buf]);
        }
        if (!ok) break;
        mma_commit(qfree);   // the q_I block may be replaced once these MMAs are done
      }
      if (!ok) {
        *abort_flag = 1;
        report(a.status, CSA_DEV_TIMEOUT, 3u);
      }
      mma_commit(drain);
      mbar_wait(drain, 0);
    }
  } else if (warp < 6) {
    // ---------------- epilogue: thread <-> TMEM lane <-> entry
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int et = threadIdx.x - 64;   // 0..127
    int64_t tile = 0;
    int n = 0;
    for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x, ++n) {
      const PUnit x = punit(a, u, n_groups);
      const int sb = n & 1;
      float* wb = sw + sb * kPTok * kHI;
      // the unit's head weights (this buffer's previous unit is finished: the
      // named barrier below ran after its last tile)
      for (int i = et; i < kPTok * kHI; i += 128) {
        const int64_t t = x.group * kPTok + i / kHI;
        wb[i] = (!dead && t < a.Tq) ? a.w[(x.b * a.Tq + t) * kHI + (i % kHI)] : 0.f;
      }
      wait_or_die(&sfree[sb], (uint32_t)((n >> 1) & 1) ^ 1u, 5u);   // top-k of unit n-2 done
      named_bar(5, 128);   // weights visible
      float* sc = scores + sb * kPTok * kPChunk;
      for (int i = 0; i < x.n_tiles; ++i, ++tile) {
        const int buf = (int)(tile & 1);
        wait_or_die(&tfull[buf], (uint32_t)((tile >> 1) & 1), 4u);
        if (dead) continue;
        tc_fence_after();
        const uint32_t base = tmem_addr(tmem, (uint32_t)(quarter * 32), (uint32_t)(buf * kPN));
#pragma unroll
        for (int t = 0; t < kPTok; ++t) {
          uint32_t r0[32], r1[32];
          tmem_ld32(base + t * kHI, r0);
          tmem_ld32(base + t * kHI + 32, r1);
          tmem_ld_wait();
          sc[t * kPChunk + i * kBM + row] = relu_weighted_sum64(wb + t * kHI, r0, r1);
        }
        tc_fence_before();
        mbar_arrive(&tempty[buf]);
      }
      named_bar(5, 128);   // every epilogue thread is past this unit's weights
      if (!dead) mbar_arrive(&sready[sb]);
    }
  } else {
    // ---------------- top-k: two warps per token
    const int tw = warp - 6;
    const int t = tw / kPTopkWarps;
    const bool lead = tw % kPTopkWarps == 0;
    unsigned* hist = reinterpret_cast<unsigned*>(sm + L::off_hist) + t * 256;
    float* red = reinterpret_cast<float*>(sm + L::off_red) + t * 8;
    unsigned* wcnt = reinterpret_cast<unsigned*>(sm + L::off_wcnt) + t * 8;
    float* cand = reinterpret_cast<float*>(sm + L::off_cand) + t * 2 * kBinCap;
    int n = 0;
    for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x, ++n) {
      const PUnit x = punit(a, u, n_groups);
      const int sb = n & 1;
      wait_or_die(&sready[sb], (uint32_t)(n >> 1) & 1u, 6u);
      const int64_t tok = x.group * kPTok + t;
      if (tok < a.Tq) {
        const int64_t row = x.b * a.Tq + tok;
        int64_t n64 = x.vis[t] - x.e0;
        n64 = n64 < 0 ? 0 : (n64 > kPChunk ? kPChunk : n64);
        int32_t* oi;
        float* os;
        if (a.n_chunks == 1) {
          oi = a.idx_out + row * a.k;
          os = a.score_out ? a.score_out + row * a.k : nullptr;
        } else {
          const int64_t c = (row * a.n_chunks + x.chunk) * a.k;
          oi = a.cand_idx + c;
          os = a.cand_score + c;
        }
        const float* sc = scores + (sb * kPTok + t) * kPChunk;
        // both warps of the token run the same barrier sequence even after a
        // timed-out wait (the selection then reads stale scores; the status
        // word already holds the error)
        const bool done = block_topk<kPTopkWarps, kPChunk>(
            sc, (int)n64, a.k, x.e0, hist, red, wcnt, cand,
            reinterpret_cast<int*>(cand + kBinCap), 1 + t, oi, os);
        if (!done) {
          if (lead) warp_topk(sc, (int)n64, a.k, x.e0, hist, oi, os);
          named_bar(1 + t, 32 * kPTopkWarps);
        }
      }
      if (lane == 0 && !dead) mbar_arrive(&sfree[sb]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
}

struct MergeShared {
  unsigned hist[256];
  unsigned tmp[33];
  unsigned s_prefix, s_mask;
  int s_rem;
  float red[64];          // per-warp min / max
  unsigned info[4];       // boundary bin, scores above it, its members, slots used
  float ts;
  int tj;
  float cs[kMergeCap];    // the boundary bin's members
  int cj[kMergeCap];
};

// Final selection over the per-chunk candidates of one row by exact block
// radix select, then an ordered compaction (candidates are in ascending entry
// order: chunk after chunk, ascending within each chunk).  The fallback of the
// value-binned merge below; the same selection.
__device__ void merge_radix(const TcIdxArgs& a, int64_t row, MergeShared& sh) {
  unsigned* hist = sh.hist;
  unsigned* tmp = sh.tmp;
  unsigned& s_prefix = sh.s_prefix;
  unsigned& s_mask = sh.s_mask;
  int& s_rem = sh.s_rem;
  const int64_t n = (int64_t)a.n_chunks * a.k;
  const float* cs = a.cand_score + row * n;
  const int32_t* ci = a.cand_idx + row * n;
  int32_t* out = a.idx_out + row * a.k;
  float* so = a.score_out ? a.score_out + row * a.k : nullptr;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;

  // number of valid candidates
  unsigned cnt = 0;
  for (int64_t j = threadIdx.x; j < n; j += blockDim.x) cnt += ci[j] >= 0;
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if (lane == 0) tmp[wid] = cnt;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned s = 0;
    for (int i = 0; i < nw; ++i) s += tmp[i];
    tmp[32] = s;
    s_prefix = 0u;
    s_mask = 0u;
    s_rem = a.k;
  }
  __syncthreads();
  const unsigned n_valid = tmp[32];
  const bool take_all = n_valid <= (unsigned)a.k;
  if (!take_all) {
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0u;
      __syncthreads();
      const unsigned prefix = s_prefix, mask = s_mask;
      for (int64_t j = threadIdx.x; j < n; j += blockDim.x) {
        if (ci[j] < 0) continue;
        unsigned key = score_key(cs[j]);
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (threadIdx.x == 0) {
        int rem = s_rem;
        unsigned cum = 0;
        int d = 255;
        for (; d > 0; --d) {
          if (cum + hist[d] >= (unsigned)rem) break;
          cum += hist[d];
        }
        s_prefix = prefix | ((unsigned)d << shift);
        s_mask = mask | (255u << shift);
        s_rem = rem - (int)cum;
      }
      __syncthreads();
    }
  }
  const unsigned tau = s_prefix, need_eq = (unsigned)s_rem;
  unsigned run_sel = 0, run_eq = 0;
  for (int64_t base = 0; base < n; base += blockDim.x) {
    const int64_t j = base + threadIdx.x;
    const bool valid = j < n && ci[j] >= 0;
    const float s = valid ? cs[j] : 0.f;
    const unsigned key = valid ? score_key(s) : 0u;
    const bool gt = valid && (take_all || key > tau);
    const bool eq = valid && !take_all && key == tau;
    // exclusive counts of eq and take over the block, in thread order
    unsigned b1 = __ballot_sync(0xffffffffu, eq);
    __syncthreads();
    if (lane == 0) tmp[wid] = __popc(b1);
    __syncthreads();
    if (threadIdx.x == 0) {
      unsigned r = 0;
      for (int i = 0; i < nw; ++i) { unsigned c = tmp[i]; tmp[i] = r; r += c; }
      tmp[32] = r;
    }
    __syncthreads();
    const unsigned eq_rank = run_eq + tmp[wid] + __popc(b1 & ((1u << lane) - 1u));
    const unsigned eq_tot = tmp[32];
    const bool take = gt || (eq && eq_rank < need_eq);
    unsigned b2 = __ballot_sync(0xffffffffu, take);
    __syncthreads();
    if (lane == 0) tmp[wid] = __popc(b2);
    __syncthreads();
    if (threadIdx.x == 0) {
      unsigned r = 0;
      for (int i = 0; i < nw; ++i) { unsigned c = tmp[i]; tmp[i] = r; r += c; }
      tmp[32] = r;
    }
    __syncthreads();
    const unsigned at = run_sel + tmp[wid] + __popc(b2 & ((1u << lane) - 1u));
    if (take && at < (unsigned)a.k) {
      out[at] = ci[j];
      if (so) so[at] = s;
    }
    run_sel += tmp[32];
    run_eq += eq_tot;
  }
  for (int64_t p = run_sel + threadIdx.x; p < a.k; p += blockDim.x) {
    out[p] = -1;
    if (so) so[p] = -INFINITY;
  }
}



// Final selection over one row's per-chunk candidates (in ascending entry
// order), the same selection as merge_radix: value bins over the valid
// candidates' range, every candidate above the boundary bin taken, the
// boundary bin's members (at most kMergeCap) ranked exactly by (score desc,
// entry asc), and an ordered emit.  The unordered passes stride over the
// candidates (coalesced); the ordered emit gives warp w the contiguous
// segment [w seg, (w+1) seg), compacted with ballots and offset by a block
// scan of the warps' counts.
__global__ void __launch_bounds__(1024)
    indexer_merge_kernel(TcIdxArgs a) {
  __shared__ MergeShared sh;
  const int64_t row = blockIdx.x;
  const int64_t n = (int64_t)a.n_chunks * a.k;
  const float* cs = a.cand_score + row * n;
  const int32_t* ci = a.cand_idx + row * n;
  int32_t* out = a.idx_out + row * a.k;
  float* so = a.score_out ? a.score_out + row * a.k : nullptr;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const unsigned lt = (1u << lane) - 1u;
  unsigned cnt = 0;
  float lo = INFINITY, hi = -INFINITY;
  for (int64_t j = threadIdx.x; j < n; j += blockDim.x) {
    if (ci[j] < 0) continue;
    const float v = cs[j];
    ++cnt;
    lo = fminf(lo, v);
    hi = fmaxf(hi, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (lane == 0) {
    sh.red[wid] = lo;
    sh.red[32 + wid] = hi;
  }
  unsigned n_valid;
  block_excl_scan(cnt, sh.tmp, &n_valid);   // (its barriers also publish red)
  for (int i = 0; i < nw; ++i) {
    lo = fminf(lo, sh.red[i]);
    hi = fmaxf(hi, sh.red[32 + i]);
  }
  const float scale = 255.99f / (hi - lo);
  if (n_valid <= (unsigned)a.k || !(hi > lo) || !(scale < INFINITY)) {
    merge_radix(a, row, sh);
    return;
  }
  for (int i = threadIdx.x; i < 256; i += blockDim.x) sh.hist[i] = 0u;
  __syncthreads();
  for (int64_t j = threadIdx.x; j < n; j += blockDim.x)
    if (ci[j] >= 0) atomicAdd(&sh.hist[value_bin(cs[j], lo, scale)], 1u);
  __syncthreads();
  if (wid == 0) {   // boundary bin: lane L owns bins 255-8L .. 248-8L (descending)
    unsigned c[8], sL = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      c[i] = sh.hist[255 - 8 * lane - i];
      sL += c[i];
    }
    const unsigned incl = warp_incl_scan(sL, lane);
    const unsigned pre = incl - sL, rem = (unsigned)a.k;
    if (pre < rem && rem <= incl) {
      unsigned run = pre;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (run + c[i] >= rem) {
          sh.info[0] = 255u - 8u * lane - i;
          sh.info[1] = run;
          sh.info[2] = c[i];
          break;
        }
        run += c[i];
      }
    }
    if (lane == 0) sh.info[3] = 0u;
  }
  __syncthreads();
  const int bstar = (int)sh.info[0];
  const unsigned need = (unsigned)a.k - sh.info[1], members = sh.info[2];
  if (members > (unsigned)kMergeCap) {
    merge_radix(a, row, sh);
    return;
  }
  for (int64_t j = threadIdx.x; j < n; j += blockDim.x) {
    if (ci[j] >= 0 && value_bin(cs[j], lo, scale) == bstar) {
      const unsigned at = atomicAdd(&sh.info[3], 1u);
      sh.cs[at] = cs[j];
      sh.cj[at] = ci[j];
    }
  }
  __syncthreads();
  for (unsigned i = threadIdx.x; i < members; i += blockDim.x) {
    const float si = sh.cs[i];
    const int ji = sh.cj[i];
    unsigned rank = 0;
    for (unsigned q = 0; q < members; ++q) {
      const float sq = sh.cs[q];
      rank += (sq > si || (sq == si && sh.cj[q] < ji)) ? 1u : 0u;
    }
    if (rank == need - 1) {   // exactly one member
      sh.ts = si;
      sh.tj = ji;
    }
  }
  __syncthreads();
  const float ts = sh.ts;
  const int tj = sh.tj;
  auto take = [&](int64_t j) {
    if (j >= n || ci[j] < 0) return false;
    const float v = cs[j];
    const int bv = value_bin(v, lo, scale);
    return bv > bstar || (bv == bstar && (v > ts || (v == ts && ci[j] <= tj)));
  };
  const int64_t seg = ((n + nw - 1) / nw + 31) / 32 * 32;
  const int64_t s0 = (int64_t)wid * seg, s1 = s0 + seg;
  unsigned mine = 0;
  for (int64_t base = s0; base < s1; base += 32) mine += __popc(__ballot_sync(0xffffffffu, take(base + lane)));
  unsigned total;
  unsigned run = block_excl_scan(lane == 0 ? mine : 0u, sh.tmp, &total);
  run = __shfl_sync(0xffffffffu, run, 0);
  for (int64_t base = s0; base < s1; base += 32) {
    const int64_t j = base + lane;
    const bool t = take(j);
    const unsigned bal = __ballot_sync(0xffffffffu, t);
    if (t) {
      const unsigned at = run + __popc(bal & lt);
      out[at] = ci[j];
      if (so) so[at] = cs[j];
    }
    run += __popc(bal);
  }
}

// Cluster merge of the per-chunk candidates: one row's candidates split over
// a cluster of up to kSelMaxCluster CTAs, 16 contiguous ones per thread.
constexpr int kMThreads = 512;
constexpr int kMRun = 16;
constexpr int kMSlice = kMThreads * kMRun;      // per CTA: 8192

__global__ void __launch_bounds__(kMThreads)
    indexer_merge_cluster_kernel(TcIdxArgs a) {
  __shared__ __align__(16) SelShared sh;
  pdl_wait();
  pdl_trigger();
  const uint32_t CL = cluster_nctarank(), rank = cluster_ctarank();
  const int64_t row = blockIdx.x / CL;
  const int64_t n = (int64_t)a.n_chunks * (a.direct ? Cfg<1>::kChunk : a.k);
  const float* cs = a.cand_score + row * n;
  const int32_t* ci = a.cand_idx + row * n;
  const int64_t j0 = (int64_t)rank * kMSlice + (int64_t)threadIdx.x * kMRun;
  float v[kMRun];
  int32_t id[kMRun];
  if (a.direct) {   // raw scores in entry order: entry j is a candidate iff visible
    const int64_t pos = a.q_pos ? a.q_pos[row] : row % a.Tq;
    const int64_t vis = vis_count(pos, a.m, a.N);
#pragma unroll
    for (int q = 0; q < kMRun / 4; ++q) {
      const int64_t j = j0 + 4 * q;
      float4 s4 = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j < vis) s4 = *reinterpret_cast<const float4*>(cs + j);
      v[4 * q] = s4.x; v[4 * q + 1] = s4.y; v[4 * q + 2] = s4.z; v[4 * q + 3] = s4.w;
#pragma unroll
      for (int e = 0; e < 4; ++e) id[4 * q + e] = j + e < vis ? (int32_t)(j + e) : -1;
    }
  } else if ((n & 3) == 0) {   // 16-byte aligned rows: j0 and n are multiples of 4
#pragma unroll
    for (int q = 0; q < kMRun / 4; ++q) {
      const int64_t j = j0 + 4 * q;
      float4 s4 = make_float4(0.f, 0.f, 0.f, 0.f);
      int4 i4 = make_int4(-1, -1, -1, -1);
      if (j < n) {
        s4 = *reinterpret_cast<const float4*>(cs + j);
        i4 = *reinterpret_cast<const int4*>(ci + j);
      }
      v[4 * q] = s4.x; v[4 * q + 1] = s4.y; v[4 * q + 2] = s4.z; v[4 * q + 3] = s4.w;
      id[4 * q] = i4.x; id[4 * q + 1] = i4.y; id[4 * q + 2] = i4.z; id[4 * q + 3] = i4.w;
    }
  } else {
#pragma unroll
    for (int e = 0; e < kMRun; ++e) {
      const int64_t j = j0 + e;
      id[e] = j < n ? ci[j] : -1;
      v[e] = j < n ? cs[j] : 0.f;
    }
  }
  cluster_topk_emit<kMRun, kMThreads>(v, id, a.k, sh, a.idx_out + row * a.k,
                                      a.score_out ? a.score_out + row * a.k : nullptr);
}

inline int tok_for(int64_t Tq) { return Tq >= 4 ? 4 : 1; }
inline int chunk_for(int tok) { return tok == 4 ? Cfg<4>::kChunk : Cfg<1>::kChunk; }
// Direct selection (no chunk top-k) for single-token rows of 2 to 16 chunks:
// the merge's cluster then holds the whole score row.
inline bool direct_for(int tok, int nc) {
  return tok == 1 && nc > 1 && (int64_t)nc * Cfg<1>::kChunk <= (int64_t)kSelMaxCluster * kMSlice;
}
// Scratch of the candidate lists (or, direct, of the raw score rows).
inline size_t cand_bytes(int64_t B, int64_t Tq, int nc, int k, bool direct) {
  if (nc <= 1) return 0;
  return direct ? (size_t)B * (size_t)Tq * (size_t)nc * (size_t)Cfg<1>::kChunk * 4
                : (size_t)B * (size_t)Tq * (size_t)nc * (size_t)k * 8;
}
inline int n_chunks_for(int64_t N, int tok) {
  int64_t c = chunk_for(tok);
  int64_t n = (N + c - 1) / c;
  return n < 1 ? 1 : (int)n;
}

template <int TOK, int FMT = 0>
cudaError_t launch_tok(const IndexerParams& p, const TcIdxArgs& a, cudaStream_t stream) {
  CUtensorMap mq, mk;
  if constexpr (FMT != 0) {
    constexpr uint32_t rb = Smem<TOK, FMT>::kRowB;
    const CUtensorMapSwizzle swz = FMT == 1 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    if (!make_map_u8_3d(&mq, p.q_I, rb, (uint64_t)p.Tq * kHI, (uint64_t)p.B, rb, TOK * kHI, swz))
      return cudaErrorInvalidValue;
    if (!make_map_u8_3d(&mk, p.k_I, rb, (uint64_t)(p.N > 0 ? p.N : 1), (uint64_t)p.B, rb, kBM,
                        swz))
      return cudaErrorInvalidValue;
  } else {
    if (!make_map_bf16_3d(&mq, p.q_I, kDI, (uint64_t)p.Tq * kHI, (uint64_t)p.B, 64, TOK * kHI))
      return cudaErrorInvalidValue;
    if (!make_map_bf16_3d(&mk, p.k_I, kDI, (uint64_t)(p.N > 0 ? p.N : 1), (uint64_t)p.B, 64,
                          kBM))
      return cudaErrorInvalidValue;
  }
  const int smem = Smem<TOK, FMT>::bytes + 1024;
  cudaError_t e = cudaFuncSetAttribute(indexer_tc_kernel<TOK, FMT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)a.n_chunks, (unsigned)((p.Tq + TOK - 1) / TOK), (unsigned)p.B);
  return launch_pdl(indexer_tc_kernel<TOK, FMT>, grid, dim3(kThreads), (size_t)smem, stream, mq,
                    mk, a);
}

// Rows with no entry at all (N == 0): index -1 and score -inf throughout.
__global__ void topk_padding_kernel(int64_t n, int32_t* idx, float* sc) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    idx[i] = -1;
    if (sc) sc[i] = -INFINITY;
  }
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  return n;
}

// The candidate merge: the cluster kernel when one row's candidates fit a
// cluster of at most kSelMaxCluster CTAs, else one CTA per row.
cudaError_t launch_merge(const TcIdxArgs& a, int64_t rows, cudaStream_t stream) {
  const int64_t n = (int64_t)a.n_chunks * (a.direct ? Cfg<1>::kChunk : a.k);
  const int64_t cl = (n + kMSlice - 1) / kMSlice;
  if (cl > kSelMaxCluster || rows * cl > (int64_t)0x7fffffff) {
    indexer_merge_kernel<<<(unsigned)rows, 1024, 0, stream>>>(a);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)(rows * cl), 1, 1);
  cfg.blockDim = dim3(kMThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = (unsigned)cl;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, indexer_merge_cluster_kernel, a);
}

cudaError_t launch_persist(const IndexerParams& p, const TcIdxArgs& a, cudaStream_t stream) {
  CUtensorMap mq, mk;
  if (!make_map_bf16_3d(&mq, p.q_I, kDI, (uint64_t)p.Tq * kHI, (uint64_t)p.B, 64, kPTok * kHI))
    return cudaErrorInvalidValue;
  if (!make_map_bf16_3d(&mk, p.k_I, kDI, (uint64_t)(p.N > 0 ? p.N : 1), (uint64_t)p.B, 64, kBM))
    return cudaErrorInvalidValue;
  const int smem = PSmem::bytes + 1024;
  cudaError_t e = cudaFuncSetAttribute(indexer_persist_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int64_t n_groups = (p.Tq + kPTok - 1) / kPTok;
  const int64_t n_units = p.B * n_groups * a.n_chunks;
  const int64_t sms = sm_count();
  const unsigned grid = (unsigned)(n_units < sms ? n_units : sms);
  indexer_persist_kernel<<<grid, kPThreads, smem, stream>>>(mq, mk, a, n_units, n_groups);
  return cudaGetLastError();
}

}  // namespace

size_t indexer_mx_scratch(int64_t B, int64_t Tq, int64_t N, int k) {
  const int nc = n_chunks_for(N, 1);
  return cand_bytes(B, Tq, nc, k, direct_for(1, nc));
}

cudaError_t launch_indexer_mx(const IndexerParams& p, int fmt, const void* q_sf,
                              const void* k_sf, cudaStream_t stream,
                              unsigned long long* n_launch) {
  *n_launch = 0;
  if (p.B == 0 || p.Tq == 0) return cudaSuccess;
  if (p.N == 0) {   // nothing to score: every row is padding
    const int64_t n = p.B * p.Tq * (int64_t)p.k;
    const int64_t blocks = (n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096;
    topk_padding_kernel<<<(unsigned)blocks, 256, 0, stream>>>(n, p.idx_out, p.score_out);
    *n_launch = 1;
    return cudaGetLastError();
  }
  TcIdxArgs a{};
  a.Tq = p.Tq;
  a.N = p.N;
  a.m = p.m;
  a.k = p.k;
  a.n_chunks = n_chunks_for(p.N, 1);
  a.w = p.w;
  a.q_pos = p.q_pos;
  a.idx_out = p.idx_out;
  a.score_out = p.score_out;
  a.status = p.status;
  a.q_sf = static_cast<const uint8_t*>(q_sf);
  a.k_sf = static_cast<const uint8_t*>(k_sf);
  a.k_sf_tiles = (p.N + kBM - 1) / kBM;
  a.direct = direct_for(1, a.n_chunks) ? 1 : 0;
  if (a.n_chunks > 1) {
    if (p.scratch_bytes < cand_bytes(p.B, p.Tq, a.n_chunks, p.k, a.direct))
      return cudaErrorInvalidValue;
    const size_t n = (size_t)p.B * p.Tq * a.n_chunks * p.k;
    a.cand_score = static_cast<float*>(p.scratch);
    a.cand_idx = a.direct ? nullptr : reinterpret_cast<int32_t*>(static_cast<float*>(p.scratch) + n);
  }
  cudaError_t e = fmt == 2 ? launch_tok<1, 2>(p, a, stream) : launch_tok<1, 1>(p, a, stream);
  if (e != cudaSuccess) return e;
  *n_launch = 1;
  if (a.n_chunks > 1) {
    e = launch_merge(a, p.B * p.Tq, stream);
    *n_launch = 2;
  }
  return e;
}

bool indexer_tc_supported(const IndexerParams& p) {
  auto al = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
  return p.HI == kHI && p.dI == kDI && p.N >= 0 && p.N < (1LL << 31) &&
         p.Tq * kHI < (1LL << 31) && p.B <= 65535 && al(p.q_I) && (p.N == 0 || al(p.k_I)) &&
         (p.Tq + 3) / 4 <= 65535;
}

size_t indexer_tc_scratch(int64_t B, int64_t Tq, int64_t N, int k) {
  const int tok = tok_for(Tq);
  const int nc = n_chunks_for(N, tok);
  return cand_bytes(B, Tq, nc, k, direct_for(tok, nc));
}

cudaError_t launch_indexer_tc(const IndexerParams& p, cudaStream_t stream,
                              unsigned long long* n_launch) {
  *n_launch = 0;
  if (p.B == 0 || p.Tq == 0) return cudaSuccess;
  if (p.N == 0) {   // nothing to score: every row is padding
    const int64_t n = p.B * p.Tq * (int64_t)p.k;
    const int64_t blocks = (n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096;
    topk_padding_kernel<<<(unsigned)blocks, 256, 0, stream>>>(n, p.idx_out, p.score_out);
    *n_launch = 1;
    return cudaGetLastError();
  }
  const int tok = tok_for(p.Tq);
  TcIdxArgs a{};
  a.Tq = p.Tq;
  a.N = p.N;
  a.m = p.m;
  a.k = p.k;
  a.n_chunks = n_chunks_for(p.N, tok);
  a.w = p.w;
  a.q_pos = p.q_pos;
  a.idx_out = p.idx_out;
  a.score_out = p.score_out;
  a.status = p.status;
  a.direct = direct_for(tok, a.n_chunks) ? 1 : 0;
  if (a.n_chunks > 1) {
    if (p.scratch_bytes < cand_bytes(p.B, p.Tq, a.n_chunks, p.k, a.direct))
      return cudaErrorInvalidValue;
    const size_t n = (size_t)p.B * p.Tq * a.n_chunks * p.k;
    a.cand_score = static_cast<float*>(p.scratch);
    a.cand_idx = a.direct ? nullptr : reinterpret_cast<int32_t*>(static_cast<float*>(p.scratch) + n);
  }
  cudaError_t e = tok == 4 ? launch_persist(p, a, stream) : launch_tok<1>(p, a, stream);
  if (e != cudaSuccess) return e;
  *n_launch = 1;
  if (a.n_chunks > 1) {
    e = launch_merge(a, p.B * p.Tq, stream);
    *n_launch = 2;
  }
  return e;
}

}  // namespace csa
