// Shared-KV MQA (sparse CSA and dense HCA, window and sink merged in one
// pass) on the 5th-generation tensor cores.
//
// Method: page "DeepSeek-V4：迈向高效百万 Token 上下文智能", §3.3 -- MQA in which
// each compressed entry is both key and value, over the top-k entries (CSA) or
// every visible entry (HCA); RMSNorm on the query and on the KV entries, which
// keeps the logits bounded; partial RoPE on query, entries and output, the
// output rotated again at position -i; a sliding window of uncompressed rows.
// Page "DeepSeek V4 完整技术报告", section "混合注意力：CSA + HCA": a learnable
// per-head sink logit lets total attention weight fall below one.
//
// Work item = (query token, group of 64 heads[, key split]).  With c = 512 an
// fp32 accumulator of 64 heads x 512 dims next to the scores would overflow
// TMEM in the usual layout, so the kernel works TRANSPOSED, keys on the MMA's
// M side:
//   S^T[key, h] = K_tile . Q^T      (M = 64 keys, N = 64 heads, K = 512)
//   O^T[c, h]  += V^T . P^T          (M = 128 dims x 4, N = 64, K = 64 keys)
// using 2 x 64 (double-buffered S^T) + 4 x 64 TMEM columns.  A gathered key
// tile (one 1 KB row per selected entry or window row) is stored once,
// 128-byte swizzled, and read by both MMAs: K-major as the A operand of S^T,
// MN-major as the A operand of O^T (K = V).  Two key tiles alternate, so the
// gather of block b+1 and S^T(b+1) overlap the softmax and O^T of block b.
//
// Softmax without a running maximum: q^ and every stored key are RMS-
// normalised (the method's RMSNorm), so |scale q^ . k| <= scale |q^| sqrt(c)
// =: M_h, a per-(token, head) bound known before any key is read.  Weights
// are exp(l - M_h) in (e^-2M_h, 1]: no rescaling of O, no cross-lane max, and
// split partial sums add directly.  A logit more than 60 above the bound (keys
// far from unit RMS) is reported as CSA_DEV_RANGE.
//
// Persistent CTAs (one per SM) walk their items in turn; roles (288 threads):
//   warps 4-7  producer: index compaction, RoPE table, the next item's raw q
//              rows by TMA and their in-place RMSNorm + RoPE, the key gather
//              (cp.async; each warp-instruction moves four 128-byte row pieces);
//   warp 8     TMEM owner and single-thread MMA issuer;
//   warps 0-3  softmax (lanes 0-15: one key each, the M = 64 TMEM layout puts
//              rows 16w..16w+15 in lanes 0-15 of warp w), then the epilogue
//              (thread = output dim), which overlaps the next item's first MMAs.
// Decode rows (one query per sequence) split the key list into fixed 256-key
// pieces whose fp32 partials a combine kernel adds in a fixed order, so a
// row's result does not depend on the batch it runs in.
#include "common.cuh"
#include "sm100.cuh"
#include "tc.h"
#include "tma_host.h"

namespace csa {

namespace {

using namespace sm100;

constexpr int kC = 512;                      // entry / head dim
constexpr int kHG = 64;                      // heads per item (MMA N)
constexpr int kBK = 64;                      // keys per block (MMA M of S^T)
constexpr int kRegions = kC / 64;            // 64-element (128-byte) column chunks
constexpr int kKRegion = kBK * 128;          // 8 KB per key-tile chunk
constexpr int kKTile = kRegions * kKRegion;  // 64 KB
constexpr int kQRegion = kHG * 128;          // 8 KB per query chunk
constexpr int kPTile = kBK * 128;            // 8 KB: P^T [64 keys][64 heads] bf16
constexpr int kSplitKeys = 256;              // decode split size (fixed)
constexpr int kMaxK = 1024;                  // largest top-k the index list holds
constexpr int kThreads = 288;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRangeLog2 = 60.f * kLog2e;  // CSA_DEV_RANGE threshold

constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + kRegions * kQRegion;   // 2 key tiles
constexpr int OFF_P = OFF_K + 2 * kKTile;            // 2 P tiles
constexpr int OFF_LIST = OFF_P + 2 * kPTile;         // 2 index lists
constexpr int OFF_MB = OFF_LIST + 2 * kMaxK * 4;     // [4][64] bounds (log2 units)
constexpr int OFF_ROPE = OFF_MB + 4 * kHG * 4;       // [4][cos 32 | sin 32]
constexpr int OFF_RED = OFF_ROPE + 4 * 64 * 4;       // [4][64] partial denominators
constexpr int OFF_INV = OFF_RED + 4 * kHG * 4;       // [64] 1/denominator
constexpr int OFF_STERM = OFF_INV + kHG * 4;         // [64] sink term
constexpr int OFF_NENT = OFF_STERM + kHG * 4;        // [2] entries per item
constexpr int OFF_BAR = OFF_NENT + 64;
constexpr int kNumBars = 22;
constexpr int OFF_MISC = OFF_BAR + kNumBars * 8;
constexpr int SMEM_BYTES = OFF_MISC + 64;

static_assert(SMEM_BYTES + 1024 <= 232448, "shared memory budget");

struct TcAttnArgs {
  int64_t Tq;
  int H, r;
  float base, eps, scale;
  uint32_t flags;
  const bf16* q;
  const int64_t* q_pos;
  const bf16* entries;
  int64_t N;
  int sparse;
  const int32_t* idx;
  int k;
  int m_dense;
  const bf16* win;
  int64_t Tw;
  const int64_t* win_pos0;
  int n_win;
  const float* sink;
  bf16* out;
  int split, n_splits, n_hg;
  int64_t n_rows, n_items;
  float* o_part;    // [rows][n_hg][n_splits][64][512]
  float* d_part;    // [rows][n_hg][n_splits][64]
  float* mb_part;   // [rows][n_hg][64]
  bf16* qhat;       // [grid][2 slots][64 heads][512]: next items' q^, prepared ahead
  unsigned* status;
};

__device__ __forceinline__ int64_t vis_count(int64_t pos, int m, int64_t N) {
  if (pos < 0) return 0;
  int64_t v = (pos + 1) / m;
  return v < N ? v : N;
}

// Everything about an item that every role derives the same way.
struct Item {
  int64_t row;
  int hg, split;
  int64_t bidx, pos, wp0, jlo, n_w;
};

__device__ __forceinline__ Item decode_item(const TcAttnArgs& a, int64_t it) {
  Item x;
  if (a.split) {
    x.split = (int)(it % a.n_splits);
    const int64_t rest = it / a.n_splits;
    x.hg = (int)(rest % a.n_hg);
    x.row = rest / a.n_hg;
  } else {
    x.split = 0;
    x.hg = (int)(it % a.n_hg);
    x.row = a.n_rows - 1 - it / a.n_hg;   // late (heavier) rows first
  }
  x.bidx = x.row / a.Tq;
  const int64_t t = x.row % a.Tq;
  x.pos = a.q_pos ? a.q_pos[x.row] : t;
  x.wp0 = a.win_pos0 ? a.win_pos0[x.bidx] : 0;
  int64_t jlo = x.pos - a.n_win + 1;
  if (jlo < x.wp0) jlo = x.wp0;
  int64_t jhi = x.pos;
  if (jhi > x.wp0 + a.Tw - 1) jhi = x.wp0 + a.Tw - 1;
  x.jlo = jlo;
  x.n_w = jhi >= jlo ? jhi - jlo + 1 : 0;
  return x;
}

// Key range [lo, hi) of an item and its number of 64-key blocks.
__device__ __forceinline__ int item_blocks(const TcAttnArgs& a, const Item& x, int64_t n_ent,
                                           int64_t* lo, int64_t* hi) {
  const int64_t n_keys = n_ent + x.n_w;
  int64_t l = 0, h = n_keys;
  if (a.split) {
    l = (int64_t)x.split * kSplitKeys;
    h = l + kSplitKeys < n_keys ? l + kSplitKeys : n_keys;
  }
  *lo = l;
  *hi = h;
  return h > l ? (int)((h - l + kBK - 1) / kBK) : 0;
}

// Query preparation by one producer warp, one item ahead of its use: the raw
// q rows of heads [16 w, 16 w + 16) are read from global memory, replaced by
// bf16(RoPE_pos(RMSNorm(q))) and written to the CTA's q^ scratch slot (row h,
// 512 dims), from which a single TMA load brings them into the Q tile when the
// item starts.  mb2[h] = scale |q^| sqrt(c) log2(e) (times 1 + 2^-7) is an
// upper bound of the head's logits against unit-RMS keys.  Lane l owns
// elements [8l, 8l+8) and [256+8l, 256+8l+8); four heads are in flight at once.
__device__ __forceinline__ void prep_query(const TcAttnArgs& a, const bf16* qsrc, bf16* qdst,
                                           int w, int lane, float scale, float* mb2,
                                           const float* rcs, const float* rsn) {
  float rc[8], rs[8];   // this lane's RoPE factors (identity outside the RoPE dims)
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int el = (k >> 2) * 256 + lane * 8 + (k & 3) * 2;
    rc[k] = 1.f;
    rs[k] = 0.f;
    if (!(a.flags & CSA_F_NO_ROPE) && el >= kC - a.r) {
      const int pi = (el - (kC - a.r)) >> 1;
      rc[k] = rcs[pi];
      rs[k] = rsn[pi];
    }
  }
  for (int i0 = 0; i0 < 16; i0 += 4) {
    uint4 raw[4][2];
    float x[4][16], ss[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const bf16* qr = qsrc + (int64_t)(w * 16 + i0 + u) * kC;
      raw[u][0] = __ldg(reinterpret_cast<const uint4*>(qr + lane * 8));
      raw[u][1] = __ldg(reinterpret_cast<const uint4*>(qr + 256 + lane * 8));
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t wr[8] = {raw[u][0].x, raw[u][0].y, raw[u][0].z, raw[u][0].w,
                              raw[u][1].x, raw[u][1].y, raw[u][1].z, raw[u][1].w};
      ss[u] = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        x[u][2 * k] = bf16_bits_to_float(wr[k] & 0xffffu);
        x[u][2 * k + 1] = bf16_bits_to_float(wr[k] >> 16);
        ss[u] = fmaf(x[u][2 * k], x[u][2 * k], ss[u]);
        ss[u] = fmaf(x[u][2 * k + 1], x[u][2 * k + 1], ss[u]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
      for (int u = 0; u < 4; ++u) ss[u] += __shfl_xor_sync(0xffffffffu, ss[u], o);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int h = w * 16 + i0 + u;
      const float inv = (a.flags & CSA_F_NO_NORM) ? 1.f : rsqrtf(ss[u] / (float)kC + a.eps);
      uint32_t wd[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float x0 = x[u][2 * k] * inv, x1 = x[u][2 * k + 1] * inv;
        wd[k] = pack_bf16x2(x0 * rc[k] - x1 * rs[k], x0 * rs[k] + x1 * rc[k]);
      }
      bf16* qd = qdst + (int64_t)h * kC;
      *reinterpret_cast<uint4*>(qd + lane * 8) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
      *reinterpret_cast<uint4*>(qd + 256 + lane * 8) = make_uint4(wd[4], wd[5], wd[6], wd[7]);
      if (lane == 0)
        mb2[h] = scale * sqrtf(ss[u]) * inv * sqrtf((float)kC) * (1.f + 0.0078125f) * kLog2e;
    }
  }
}

// Sum of v[0..63] over the 32 lanes of a warp by recursive halving: after
// the five exchange steps lane L holds the totals of entries 2L and 2L+1.
__device__ __forceinline__ void warp_transpose_sum64(float* v, int lane, float* out2) {
#pragma unroll
  for (int o = 16, n = 64; o >= 1; o >>= 1, n >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < n / 2; ++i) {
      const float lo = v[i], hi = v[i + n / 2];
      const float send = upper ? lo : hi;
      const float keep = upper ? hi : lo;
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  out2[0] = v[0];
  out2[1] = v[1];
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap map_q, TcAttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sQ = sm + OFF_Q;
  float* mb2s = reinterpret_cast<float*>(sm + OFF_MB);
  float* ropes = reinterpret_cast<float*>(sm + OFF_ROPE);
  float* red = reinterpret_cast<float*>(sm + OFF_RED);
  float* sinv = reinterpret_cast<float*>(sm + OFF_INV);
  float* sterm = reinterpret_cast<float*>(sm + OFF_STERM);
  int* nent = reinterpret_cast<int*>(sm + OFF_NENT);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint64_t* kfull = bars;        // [2] key tile landed (128 producer threads)
  uint64_t* bfree = bars + 2;    // [2] O^T of the block done: key tile and P tile free
  uint64_t* sfull = bars + 4;    // [2] S^T of the block done
  uint64_t* pfull = bars + 6;    // [2] P tile written (128 softmax threads)
  uint64_t* iready = bars + 8;   // [2] item's entry count published
  uint64_t* qload = bars + 10;   // the item's q^ rows landed in the Q tile (TMA)
  uint64_t* qfree = bars + 12;   // last S^T of the item done
  uint64_t* ofull = bars + 13;   // last O^T of the item done
  uint64_t* ofree = bars + 14;   // epilogue finished reading O^T (128 threads)
  uint64_t* drain = bars + 15;
  uint64_t* ifree = bars + 16;   // [2] MMA and softmax have read the item slot
  uint64_t* qready = bars + 18;  // [4] the item's bounds and RoPE table ready (softmax)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
  int* wcnt = reinterpret_cast<int*>(sm + OFF_MISC + 8);        // [4]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_MISC + 24);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float scale = a.scale > 0.f ? a.scale : rsqrtf((float)kC);

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kfull[i], 128);
      mbar_init(&bfree[i], 1);
      mbar_init(&sfull[i], 1);
      mbar_init(&pfull[i], 128);
      mbar_init(&iready[i], 1);
      mbar_init(&ifree[i], 2);
    }
    for (int i = 0; i < 4; ++i) mbar_init(&qready[i], 128);
    mbar_init(qload, 1);
    mbar_init(qfree, 1);
    mbar_init(ofull, 1);
    mbar_init(ofree, 128);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 8) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS0 = tmem;          // S^T buffers at columns 0 and 64
  const uint32_t tO = tmem + 128;     // O^T: 4 x 64 columns

  if (warp >= 4 && warp < 8) {
    // ======================= producer
    // Failure handling: a wait that runs out marks the thread `dead` (made
    // warp-uniform); dead threads skip waits and work but still pass every
    // named barrier, so no barrier can be left waiting.
    const int ptid = threadIdx.x - 128, pw = warp - 4, quad = lane >> 3, g8 = lane & 7;
    const uint32_t kbase = smem_u32(sm + OFF_K);
    bf16* qslots = a.qhat + (int64_t)blockIdx.x * 2 * kHG * kC;
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
    // RoPE table, q^ (to scratch slot n&1) and bounds of the CTA's item n
    auto prepare = [&](int64_t it, int n) {
      const Item x = decode_item(a, it);
      float* rcs = ropes + (n & 3) * 64;
      float* rsn = rcs + 32;
      if (!dead && pw == 0 && lane < (a.r >> 1)) {
        float cs, sn;
        rope_cos_sin(x.pos, lane, a.r, a.base, &cs, &sn);
        rcs[lane] = cs;
        rsn[lane] = sn;
      }
      named_bar(2, 128);   // RoPE table complete
      if (!dead) {
        const bf16* qsrc = a.q + (x.row * a.H + (int64_t)x.hg * kHG) * kC;
        prep_query(a, qsrc, qslots + (n & 1) * kHG * kC, pw, lane, scale, mb2s + (n & 3) * kHG,
                   rcs, rsn);
        fence_proxy_async_all();   // q^ stores (generic) -> TMA load (async proxy)
        mbar_arrive(&qready[n & 3]);
      }
      named_bar(2, 128);   // the scratch slot is complete before its TMA load
    };
    int64_t gblk = 0;
    int n = 0;
    if ((int64_t)blockIdx.x < a.n_items) prepare(blockIdx.x, 0);
    for (int64_t it = blockIdx.x; it < a.n_items; it += gridDim.x, ++n) {
      const int ip = n & 1;
      const Item x = decode_item(a, it);
      wait_or_die(&ifree[ip], (uint32_t)((n >> 1) & 1) ^ 1u, 19u);   // item n-2 consumed
      int32_t* list = reinterpret_cast<int32_t*>(sm + OFF_LIST) + ip * kMaxK;
      const int64_t it_next = it + gridDim.x;
      if (!dead && ptid == 0 && it_next < a.n_items) {   // warm L2 with the next item's q rows
        const Item y = decode_item(a, it_next);
        const bf16* qn = a.q + (y.row * a.H + (int64_t)y.hg * kHG) * kC;
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(qn), "r"(kHG * kC * 2)
                     : "memory");
      }
      int64_t n_ent;
      if (a.sparse) {
        // warp pw compacts the contiguous quarter [pw*q4, pw*q4 + q4) of the row
        const int32_t* ir = a.idx + x.row * (int64_t)a.k;
        const int q4 = (a.k + 3) / 4;
        const int lo = pw * q4, hi = lo + q4 < a.k ? lo + q4 : a.k;
        int32_t ev[kMaxK / 128];
#pragma unroll
        for (int u = 0; u < kMaxK / 128; ++u) {
          const int i = lo + u * 32 + lane;
          ev[u] = (!dead && u * 32 < q4 && i < hi) ? ir[i] : -1;
        }
        int cnt = 0;
#pragma unroll
        for (int u = 0; u < kMaxK / 128; ++u) {
          const bool ok = ev[u] >= 0 && ev[u] < a.N;
          if (!ok && ev[u] != -1)
            report(a.status, CSA_DEV_BAD_INDEX, (unsigned)(lo + u * 32 + lane));
          cnt += __popc(__ballot_sync(0xffffffffu, ok));
        }
        named_bar(2, 128);   // previous item's use of wcnt finished
        if (lane == 0) wcnt[pw] = cnt;
        named_bar(2, 128);
        int off = 0;
        for (int w = 0; w < pw; ++w) off += wcnt[w];
        n_ent = wcnt[0] + wcnt[1] + wcnt[2] + wcnt[3];
#pragma unroll
        for (int u = 0; u < kMaxK / 128; ++u) {
          const bool ok = ev[u] >= 0 && ev[u] < a.N;
          const unsigned bal = __ballot_sync(0xffffffffu, ok);
          if (ok) list[off + __popc(bal & ((1u << lane) - 1u))] = ev[u];
          off += __popc(bal);
        }
      } else {
        n_ent = vis_count(x.pos, a.m_dense, a.N);
      }
      named_bar(2, 128);   // the index list is complete
      if (!dead && ptid == 0) {
        nent[ip] = (int)n_ent;
        mbar_arrive(&iready[ip]);
      }
      int64_t k_lo, k_hi;
      const int nb = dead ? 0 : item_blocks(a, x, n_ent, &k_lo, &k_hi);

      // the previous item's last S^T is done with Q: bring in this item's q^
      if (!dead && ptid == 0) {
        if (n > 0 && !mbar_wait(qfree, (uint32_t)(n - 1) & 1u)) {
          *abort_flag = 1;
          report(a.status, CSA_DEV_TIMEOUT, 20u);
        } else {
          mbar_arrive_expect_tx(qload, kRegions * kQRegion);
          const int32_t qr = (int32_t)(((int64_t)blockIdx.x * 2 + (n & 1)) * kHG);
          for (int r = 0; r < kRegions; ++r)
            tma_load_3d(sQ + r * kQRegion, &map_q, qload, r * 64, qr, 0);
        }
      }

      const bf16* ent = a.entries + x.bidx * a.N * kC;
      const bf16* win = a.win + x.bidx * a.Tw * kC;
      for (int b = 0; b < (nb > 0 ? nb : 1); ++b) {
        const int64_t j = gblk + b;
        const int s = (int)(j & 1);
        if (b < nb) {
          wait_or_die(&bfree[s], (uint32_t)((j >> 1) & 1) ^ 1u, 21u);
          if (!dead) {
            const uint32_t tile = kbase + s * kKTile;
            // warp pw fetches rows 16 pw .. 16 pw + 15: four rows per instruction
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int r = pw * 16 + 4 * i + quad;
              const int64_t key = k_lo + (int64_t)b * kBK + r;
              const bf16* src = nullptr;
              if (key < k_hi) {
                if (key < n_ent) src = ent + (int64_t)(a.sparse ? list[key] : key) * kC;
                else src = win + ((x.jlo - x.wp0) + (key - n_ent)) * kC;
              }
              const uint32_t dst =
                  tile + (uint32_t)r * 128u + (((uint32_t)g8 ^ (uint32_t)(r & 7)) << 4);
#pragma unroll
              for (int reg = 0; reg < kRegions; ++reg) {
                const void* sp = src ? (const void*)(src + reg * 64 + g8 * 8) : (const void*)a.q;
                cp_async16(dst + reg * kKRegion, sp, src ? 16u : 0u);
              }
            }
          }
          // the barrier counts this thread's arrival once its copies land
          if (!dead) cp_async_arrive(&kfull[s]);
        }
        // the next item's query, once both key tiles are in flight (the
        // producer would otherwise only wait for a tile to free up)
        if (b == (nb > 1 ? 1 : 0) && it_next < a.n_items) prepare(it_next, n + 1);
      }
      gblk += nb;
    }
    cp_async_wait<0>();
  } else if (warp == 8) {
    // ======================= MMA issuer
    if (elect_one()) {
      constexpr uint32_t idS = idesc_bf16_f32(kBK, kHG, 0, 0);
      constexpr uint32_t idO = idesc_bf16_f32(128, kHG, 1, 1);
      const uint32_t qb = smem_u32(sQ), kb0 = smem_u32(sm + OFF_K), pb0 = smem_u32(sm + OFF_P);
      int64_t gblk = 0;
      int n = 0;
      bool ok = true;
      auto issue_s = [&](int64_t j) -> bool {
        const int s = (int)(j & 1);
        if (*abort_flag || !mbar_wait(&kfull[s], (uint32_t)(j >> 1) & 1u)) return false;
        fence_proxy_async_smem();   // cp.async (generic proxy) writes -> MMA reads
        tc_fence_after();
        const uint32_t kb = kb0 + s * kKTile;
#pragma unroll
        for (int reg = 0; reg < kRegions; ++reg) {
#pragma unroll
          for (int kq = 0; kq < 4; ++kq) {
            const uint64_t ad = smem_desc(kb + reg * kKRegion + kq * 32, 16, 1024, 2);
            const uint64_t bd = smem_desc(qb + reg * kQRegion + kq * 32, 16, 1024, 2);
            mma_bf16_ss(tS0 + 64 * s, ad, bd, idS, (reg | kq) != 0 ? 1u : 0u);
          }
        }
        mma_commit(&sfull[s]);
        return true;
      };
      for (int64_t it = blockIdx.x; ok && it < a.n_items; it += gridDim.x, ++n) {
        const Item x = decode_item(a, it);
        if (!mbar_wait(&iready[n & 1], (uint32_t)(n >> 1) & 1u)) { ok = false; break; }
        int64_t k_lo, k_hi;
        const int nb = item_blocks(a, x, nent[n & 1], &k_lo, &k_hi);
        mbar_arrive(&ifree[n & 1]);
        if (*abort_flag || !mbar_wait(qload, (uint32_t)n & 1u)) { ok = false; break; }
        tc_fence_after();
        if (nb == 0) {
          mma_commit(qfree);
          // keep ofull at most one phase ahead of the epilogue
          if (n > 0 && !mbar_wait(ofree, (uint32_t)(n - 1) & 1u)) { ok = false; break; }
          mma_commit(ofull);
          continue;
        }
        // S^T of the item's block bi; the item's last one releases Q
        auto issue_s_item = [&](int bi) -> bool {
          if (!issue_s(gblk + bi)) return false;
          if (bi == nb - 1) mma_commit(qfree);
          return true;
        };
        if (!issue_s_item(0)) { ok = false; break; }
        int next_s = 1;   // next block whose S^T is still to be issued
        for (int b = 0; b < nb; ++b) {
          const int64_t j = gblk + b;
          const int s = (int)(j & 1);
          // S^T(j+1) ahead of O^T(j) when its key tile is already here (keeps the
          // tensor pipe busy through softmax(j+1)); never block O^T(j) on a gather
          if (next_s == b + 1 && next_s < nb &&
              mbar_try_wait(&kfull[(j + 1) & 1], (uint32_t)((j + 1) >> 1) & 1u)) {
            if (!issue_s_item(next_s)) { ok = false; break; }
            ++next_s;
          }
          if (*abort_flag || !mbar_wait(&pfull[s], (uint32_t)(j >> 1) & 1u)) { ok = false; break; }
          if (b == 0 && n > 0 && !mbar_wait(ofree, (uint32_t)(n - 1) & 1u)) { ok = false; break; }
          tc_fence_after();
          const uint32_t kb = kb0 + s * kKTile, pb = pb0 + s * kPTile;
#pragma unroll 1
          for (int jt = 0; jt < 4; ++jt) {
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              const uint64_t ad = smem_desc(kb + (2 * jt) * kKRegion + kk * 2048, kKRegion, 1024, 2);
              const uint64_t bd = smem_desc(pb + kk * 2048, kKRegion, 1024, 2);
              mma_bf16_ss(tO + 64 * jt, ad, bd, idO, (b > 0 || kk > 0) ? 1u : 0u);
            }
          }
          mma_commit(&bfree[s]);
          if (next_s == b + 1 && next_s < nb) {
            if (!issue_s_item(next_s)) { ok = false; break; }
            ++next_s;
          }
        }
        if (!ok) break;
        mma_commit(ofull);
        gblk += nb;
      }
      if (!ok) {
        *abort_flag = 1;
        report(a.status, CSA_DEV_TIMEOUT, 23u);
      }
      mma_commit(drain);
      mbar_wait(drain, 0);
    }
  } else if (warp < 4) {
    // ======================= softmax + epilogue (same failure handling)
    const int rw = warp * 32 + lane;
    const bool active = lane < 16;      // M = 64: rows 16w..16w+15 in lanes 0..15
    const int kb_row = warp * 16 + lane;
    const float c2 = scale * kLog2e;
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
    int64_t gblk = 0;
    int n = 0;
    for (int64_t it = blockIdx.x; it < a.n_items; it += gridDim.x, ++n) {
      const int ip = n & 1;
      const Item x = decode_item(a, it);
      wait_or_die(&iready[ip], (uint32_t)(n >> 1) & 1u, 24u);
      wait_or_die(&qready[n & 3], (uint32_t)(n >> 2) & 1u, 24u);
      const float* mb2 = mb2s + (n & 3) * kHG;
      int64_t k_lo = 0, k_hi = 0;
      const int nb = dead ? 0 : item_blocks(a, x, nent[ip], &k_lo, &k_hi);
      // values the epilogue needs, copied now (the producer may refill the
      // item-parity buffers before the epilogue runs)
      const int64_t slot = x.row * a.n_hg + x.hg;
      float my_mb2 = 0.f;
      if (rw < kHG) {
        my_mb2 = mb2[rw];
        sterm[rw] = a.sink ? ex2(fmaf(a.sink[x.hg * kHG + rw], kLog2e, -my_mb2)) : 0.f;
      }
      float ecs[4], esn[4];   // RoPE factors of this thread's output pair, per slice
      {
        const float* rcs = ropes + (n & 3) * 64;
#pragma unroll
        for (int jt = 0; jt < 4; ++jt) {
          const int cc = 128 * jt + warp * 32 + (lane & ~1);
          ecs[jt] = 1.f;
          esn[jt] = 0.f;
          if (!(a.flags & CSA_F_NO_ROPE) && cc >= kC - a.r) {
            const int pi = (cc - (kC - a.r)) >> 1;
            ecs[jt] = rcs[pi];
            esn[jt] = rcs[32 + pi];
          }
        }
      }
      named_bar(1, 128);   // every thread has read the item slot
      if (rw == 0 && !dead) mbar_arrive(&ifree[ip]);
      float psum[kHG];
#pragma unroll
      for (int h = 0; h < kHG; ++h) psum[h] = 0.f;
      float xmax = -INFINITY;
      for (int b = 0; b < nb; ++b) {
        const int64_t j = gblk + b;
        const int s = (int)(j & 1);
        const uint32_t ph = (uint32_t)(j >> 1) & 1u;
        wait_or_die(&sfull[s], ph, 25u);
        uint32_t pk[32];
        if (!dead) {
          tc_fence_after();
          const uint32_t ta = tmem_addr(tS0 + 64 * s, (uint32_t)(warp * 32), 0);
          const bool valid = active && (k_lo + (int64_t)b * kBK + kb_row < k_hi);
#pragma unroll
          for (int half = 0; half < 2; ++half) {   // 32 heads at a time
            uint32_t sv[32];
            tmem_ld32(ta + 32 * half, sv);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const int h = 32 * half + e;
              const float x0 = valid ? fmaf(__uint_as_float(sv[e]), c2, -mb2[h]) : -INFINITY;
              const float x1 =
                  valid ? fmaf(__uint_as_float(sv[e + 1]), c2, -mb2[h + 1]) : -INFINITY;
              xmax = fmaxf(xmax, fmaxf(x0, x1));
              const float p0 = ex2(x0), p1 = ex2(x1);
              psum[h] += p0;
              psum[h + 1] += p1;
              pk[h >> 1] = pack_bf16x2(p0, p1);
            }
          }
        }
        wait_or_die(&bfree[s], ph ^ 1u, 25u);   // O^T(j-2) has read this P tile
        if (!dead) {
          if (active) {
            uint8_t* prow = sm + OFF_P + s * kPTile + kb_row * 128;
#pragma unroll
            for (int q8 = 0; q8 < 8; ++q8)
              *reinterpret_cast<uint4*>(prow + ((q8 ^ (kb_row & 7)) << 4)) =
                  make_uint4(pk[4 * q8], pk[4 * q8 + 1], pk[4 * q8 + 2], pk[4 * q8 + 3]);
          }
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive(&pfull[s]);
        }
      }
      if (xmax > kRangeLog2) report(a.status, CSA_DEV_RANGE, (unsigned)x.row);
      wait_or_die(ofull, (uint32_t)n & 1u, 26u);
      tc_fence_after();
      const bool have_o = nb > 0 && !dead;

      // per-head denominators
      float two[2];
      warp_transpose_sum64(psum, lane, two);
      red[warp * kHG + 2 * lane] = two[0];
      red[warp * kHG + 2 * lane + 1] = two[1];
      named_bar(1, 128);
      if (rw < kHG && !dead) {
        const float tot = red[rw] + red[kHG + rw] + red[2 * kHG + rw] + red[3 * kHG + rw];
        if (a.split) {
          a.d_part[(slot * a.n_splits + x.split) * kHG + rw] = tot;
          if (x.split == 0) a.mb_part[slot * kHG + rw] = my_mb2;
        } else {
          const float den = tot + sterm[rw];
          sinv[rw] = den > 0.f ? 1.f / den : 0.f;
        }
      }
      named_bar(1, 128);

      // O^T -> output: thread = dim 128 jt + 32 warp + lane
      float iv[kHG];
#pragma unroll
      for (int h = 0; h < kHG; ++h) iv[h] = a.split ? 1.f : sinv[h];
      const int odd = lane & 1;
#pragma unroll 1
      for (int jt = 0; jt < 4; ++jt) {
        const int c = 128 * jt + warp * 32 + lane;
        const int cc = c - odd;
        const float cs = ecs[jt], sn = esn[jt];
#pragma unroll
        for (int half = 0; half < 2; ++half) {   // heads 32 half .. 32 half + 31
          uint32_t ov[32];
          if (have_o) {
            tmem_ld32(tmem_addr(tO + 64 * jt + 32 * half, (uint32_t)(warp * 32), 0), ov);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = 0u;
          }
          if (jt == 3 && half == 1 && !dead) {   // every TMEM read of this item is done
            tc_fence_before();
            mbar_arrive(ofree);
          }
          if (dead) continue;
          if (a.split) {
            float* op = a.o_part + ((slot * a.n_splits + x.split) * kHG + 32 * half) * kC + c;
#pragma unroll
            for (int e = 0; e < 32; ++e) op[(int64_t)e * kC] = __uint_as_float(ov[e]);
          } else {
            bf16* obase = a.out + (x.row * a.H + (int64_t)x.hg * kHG + 32 * half) * kC + cc;
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const int h = 32 * half + e;
              const float v0 = __uint_as_float(ov[e]) * iv[h];
              const float v1 = __uint_as_float(ov[e + 1]) * iv[h + 1];
              // even lane keeps head h and receives its neighbour's dim; odd lane head h+1
              const float recv = __shfl_xor_sync(0xffffffffu, odd ? v0 : v1, 1);
              const float x0 = odd ? recv : v0;
              const float x1 = odd ? v1 : recv;
              // rotate the pair by -pos: (x0, x1) -> (x0 cs + x1 sn, -x0 sn + x1 cs)
              const float y0 = fmaf(x0, cs, x1 * sn), y1 = fmaf(x1, cs, -x0 * sn);
              *reinterpret_cast<uint32_t*>(obase + (int64_t)(e + odd) * kC) = pack_bf16x2(y0, y1);
            }
          }
        }
      }
      gblk += nb;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Sums the fixed-order split partials of one (row, head group), divides by
// the denominator (sink included) and rotates the output back by -pos.
__global__ void __launch_bounds__(256) attn_combine_kernel(TcAttnArgs a) {
  __shared__ float inv[kHG];
  __shared__ float cs_t[32], sn_t[32];
  const int64_t row = blockIdx.x;
  const int hg = blockIdx.y;
  const int64_t slot = row * a.n_hg + hg;
  const int64_t t = row % a.Tq;
  const int64_t pos = a.q_pos ? a.q_pos[row] : t;
  if (threadIdx.x < kHG) {
    float tot = 0.f;
    for (int s = 0; s < a.n_splits; ++s)
      tot += a.d_part[(slot * a.n_splits + s) * kHG + threadIdx.x];
    if (a.sink) {
      const float z = a.sink[hg * kHG + threadIdx.x];
      tot += ex2(fmaf(z, kLog2e, -a.mb_part[slot * kHG + threadIdx.x]));
    }
    inv[threadIdx.x] = tot > 0.f ? 1.f / tot : 0.f;
  } else if (threadIdx.x >= 64 && threadIdx.x < 64 + (a.r >> 1)) {
    float cs, sn;
    rope_cos_sin(-pos, threadIdx.x - 64, a.r, a.base, &cs, &sn);
    cs_t[threadIdx.x - 64] = cs;
    sn_t[threadIdx.x - 64] = sn;
  }
  __syncthreads();
  for (int pi = threadIdx.x; pi < kHG * kC / 2; pi += blockDim.x) {
    const int h = pi / (kC / 2);
    const int c = (pi % (kC / 2)) * 2;
    float o0 = 0.f, o1 = 0.f;
    for (int s = 0; s < a.n_splits; ++s) {
      const float* op = a.o_part + ((slot * a.n_splits + s) * kHG + h) * kC + c;
      const float2 v = *reinterpret_cast<const float2*>(op);
      o0 += v.x;
      o1 += v.y;
    }
    o0 *= inv[h];
    o1 *= inv[h];
    if (!(a.flags & CSA_F_NO_ROPE) && c >= kC - a.r) {
      const int i = (c - (kC - a.r)) >> 1;
      const float y0 = o0 * cs_t[i] - o1 * sn_t[i], y1 = o0 * sn_t[i] + o1 * cs_t[i];
      o0 = y0;
      o1 = y1;
    }
    *reinterpret_cast<uint32_t*>(a.out + (row * a.H + (int64_t)hg * kHG + h) * kC + c) =
        pack_bf16x2(o0, o1);
  }
}

// Streaming multiprocessors of the current device (one persistent CTA each).
inline int64_t num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  return n;
}

inline int n_splits_for(int64_t max_keys) {
  int64_t n = (max_keys + kSplitKeys - 1) / kSplitKeys;
  return n < 1 ? 1 : (int)n;
}

}  // namespace

bool attn_tc_supported(const AttnParams& p) {
  auto al = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
  if (p.f.c != kC || p.H % kHG != 0 || p.f.r > 64 || (p.f.r & 1)) return false;
  if (p.sparse && p.k > kMaxK) return false;   // the per-item index list holds kMaxK
  if (p.B * p.Tq >= (1LL << 31)) return false;
  if (p.Tq == 1 && p.B > 65535) return false;
  return al(p.q) && al(p.out) && (p.N == 0 || al(p.entries)) && (p.Tw == 0 || al(p.win));
}

// q^ scratch: two 64-head slots per persistent CTA (stays in L2)
inline size_t qhat_bytes() { return (size_t)num_sms() * 2 * kHG * kC * sizeof(bf16); }

size_t attn_tc_scratch(int64_t B, int64_t Tq, int H, int c, int64_t max_keys) {
  if (c != kC || H % kHG != 0) return 0;
  size_t bytes = qhat_bytes();
  if (Tq == 1) {
    const int64_t n_hg = H / kHG;
    const int64_t ns = n_splits_for(max_keys);
    const int64_t slots = B * Tq * n_hg;
    bytes += (size_t)(slots * ns * (kHG * kC + kHG) + slots * kHG) * sizeof(float);
  }
  return bytes;
}

cudaError_t launch_attn_tc(const AttnParams& p, cudaStream_t stream, unsigned long long* n_launch) {
  *n_launch = 0;
  if (p.B == 0 || p.Tq == 0) return cudaSuccess;
  TcAttnArgs a{};
  a.Tq = p.Tq;
  a.H = p.H;
  a.r = p.f.r;
  a.base = p.f.base;
  a.eps = p.f.eps;
  a.scale = p.scale;
  a.flags = p.f.flags;
  a.q = static_cast<const bf16*>(p.q);
  a.q_pos = p.q_pos;
  a.entries = static_cast<const bf16*>(p.entries);
  a.N = p.N;
  a.sparse = p.sparse;
  a.idx = p.idx;
  a.k = p.k;
  a.m_dense = p.m_dense;
  a.win = static_cast<const bf16*>(p.win);
  a.Tw = p.Tw;
  a.win_pos0 = p.win_pos0;
  a.n_win = p.n_win;
  a.sink = p.sink;
  a.out = static_cast<bf16*>(p.out);
  a.status = p.status;
  a.n_hg = p.H / kHG;
  const int64_t rows = p.B * p.Tq;
  a.split = p.Tq == 1 ? 1 : 0;
  const int64_t max_keys = (p.sparse ? (int64_t)p.k : p.N) + p.n_win;
  a.n_rows = rows;
  const size_t need = attn_tc_scratch(p.B, p.Tq, p.H, kC, max_keys);
  if (p.scratch_bytes < need) return cudaErrorInvalidValue;
  a.qhat = static_cast<bf16*>(p.scratch);
  if (a.split) {
    a.n_splits = n_splits_for(max_keys);
    const int64_t slots = rows * a.n_hg;
    a.o_part = reinterpret_cast<float*>(static_cast<char*>(p.scratch) + qhat_bytes());
    a.d_part = a.o_part + slots * a.n_splits * kHG * kC;
    a.mb_part = a.d_part + slots * a.n_splits * kHG;
  } else {
    a.n_splits = 1;
  }
  a.n_items = rows * a.n_hg * a.n_splits;
  const unsigned grid = (unsigned)(a.n_items < num_sms() ? a.n_items : num_sms());
  CUtensorMap mq;   // q^ scratch as [grid*2*64 rows][512] bf16, boxes of 64 rows x 64 dims
  if (!make_map_bf16_3d(&mq, a.qhat, kC, (uint64_t)grid * 2 * kHG, 1, 64, kHG))
    return cudaErrorInvalidValue;
  const int smem = SMEM_BYTES + 1024;
  cudaError_t e =
      cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  attn_tc_kernel<<<grid, kThreads, smem, stream>>>(mq, a);
  if (a.split) {
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    attn_combine_kernel<<<dim3((unsigned)rows, (unsigned)a.n_hg), 256, 0, stream>>>(a);
    *n_launch = 2;
  } else {
    *n_launch = 1;
  }
  return cudaGetLastError();
}

}  // namespace csa
