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
// Query RMSNorm as a per-head scale: the Q tile holds the raw q rows (TMA,
// dims 0..447) and RoPE(q) for the last 64 dims (rotated in place), so
// S^T carries |q| instead of |q^| and the softmax multiplies head h's column
// by scale inv_h log2(e), inv_h = 1/rms(q_h).  RoPE preserves pair norms, so
// inv_h comes from the raw rows.
//
// Softmax without a running maximum: q^ and every stored key are RMS-
// normalised (the method's RMSNorm), so |scale q^ . k| <= scale |q^| sqrt(c)
// =: M_h, a per-(token, head) bound known before any key is read.  Weights
// are exp(l - M_h) in (e^-2M_h, 1]: no rescaling of O, no cross-lane max, and
// split partial sums add directly.  A logit more than 60 above the bound (keys
// far from unit RMS) is reported as CSA_DEV_RANGE.  The per-head sums of the
// bf16 weights come from the tensor core too (a ones tile times P^T), so the
// denominators match the numerators' rounding.
//
// Persistent CTAs (one per SM) walk their items in turn; 512 threads in four
// warpgroups, whose register budgets are rebalanced at the start (softmax and
// epilogue up, producers and issuers down):
//   warps 8-10, 12-14 producer: index compaction, RoPE table, the item's raw
//              q rows by TMA, the key gather (cp.async; each warp-instruction
//              moves four 128-byte row pieces), 128-dim region pair by region
//              pair as the tile's previous block releases them;
//   warp 11    TMEM owner and S^T issuer (each region pair as it lands);
//   warp 15    O^T and row-sum issuer (a commit per 128-dim O^T slice frees
//              that region pair of the key tile);
//   warps 0-3  softmax (all 32 lanes: the 16x64b TMEM load gives each lane
//              one key and the 32 heads of one parity); at an item's start
//              they rotate the Q tile's RoPE dims in place as soon as the raw
//              rows land, then derive the per-head 1/rms while S^T(0) runs;
//   warps 4-7  epilogue (thread = output dim), which runs alongside the next
//              item's softmax; it frees O^T in four 64-column slices, so the
//              next item's first O^T waits only for the slice it overwrites.
// Decode rows (one query per sequence) split the key list into pieces of a
// size fixed by the row's own key count (at least 320 keys, at most 16
// pieces) whose fp32 partials a combine kernel adds in a fixed order, so a
// row's result does not depend on the batch it runs in.
#include <cuda_fp8.h>

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
constexpr int kSplitKeys = 320;              // smallest decode split (five 64-key blocks)
constexpr int kMaxSplits = 16;               // most splits of one decode row
constexpr int kMaxK = 1024;                  // largest top-k the index list holds
// 16 warps in four warpgroups: softmax (0-3), epilogue (4-7), producers
// 8-10 and 12-14, the S^T issuer and TMEM owner (11), the O^T issuer (15).
constexpr int kProdWarps = 6;
constexpr int kProdThreads = 32 * kProdWarps;
constexpr int kMmaWarp = 11;
constexpr int kMmaWarpO = 15;
constexpr int kGatherIters = (kBK / 4 + kProdWarps - 1) / kProdWarps;   // 4-row groups per warp
constexpr int kThreads = 512;
// registers per thread: launched with 128; softmax and epilogue warpgroups
// raise theirs, the producer / issuer warpgroups lower theirs, and the sum
// stays at the launch total (128 threads per warpgroup):
constexpr int kRegHeavy = 136, kRegLight = 120;
static_assert(2 * kRegHeavy + 2 * kRegLight <= 4 * 128, "register split exceeds the launch budget");
__device__ __forceinline__ int prod_index(int warp) {   // producer warp -> 0..5, else -1
  return (warp >= 8 && warp <= 10) ? warp - 8 : (warp >= 12 && warp <= 14) ? warp - 9 : -1;
}
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRangeLog2 = 60.f * kLog2e;  // CSA_DEV_RANGE threshold

constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + kRegions * kQRegion;   // 2 key tiles
constexpr int OFF_P = OFF_K + 2 * kKTile;            // 2 P tiles
constexpr int OFF_ONES = OFF_P + 2 * kPTile;         // 8 rows x 64 bf16 ones (1 KB)
constexpr int OFF_LIST = OFF_ONES + 1024;            // 2 index lists
constexpr int OFF_MB = OFF_LIST + 2 * kMaxK * 4;     // [4][64] bounds (log2 units)
constexpr int OFF_ROPE = OFF_MB + 4 * kHG * 4;       // [4][cos 32 | sin 32]
constexpr int OFF_C2 = OFF_ROPE + 4 * 64 * 4;        // [4][64] scale inv_h log2(e)
constexpr int OFF_INV = OFF_C2 + 4 * kHG * 4;        // [64] 1/denominator
constexpr int OFF_SS7 = OFF_INV + kHG * 4;           // [64] sum of squares of the RoPE dims
constexpr int OFF_NENT = OFF_SS7 + kHG * 4;          // [2] entries per item
constexpr int OFF_BAR = OFF_NENT + 64;
constexpr int kNumBars = 38;
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
  const uint8_t* ent_mixed;   // mixed BF16 / MX-FP8 entry records (mixed != 0)
  int mixed, rec_bytes;
  float* o_part;    // [rows][n_hg][n_splits][64][512]
  float* d_part;    // [rows][n_hg][n_splits][64]
  float* mb_part;   // [rows][n_hg][64]
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

// (query row, head group) of item `it`, from the launch arguments alone.
__device__ __forceinline__ void item_row_hg(const TcAttnArgs& a, int64_t it, int64_t* row,
                                            int64_t* hg) {
  if (a.split) {
    const int64_t rest = it / a.n_splits;
    *hg = rest % a.n_hg;
    *row = rest / a.n_hg;
  } else {
    *hg = it % a.n_hg;
    *row = a.n_rows - 1 - it / a.n_hg;   // late (heavier) rows first
  }
}

__device__ __forceinline__ Item decode_item(const TcAttnArgs& a, int64_t it) {
  Item x;
  int64_t row, hg;
  item_row_hg(a, it, &row, &hg);
  x.row = row;
  x.hg = (int)hg;
  x.split = a.split ? (int)(it % a.n_splits) : 0;
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

// Mixed BF16 / MX-FP8 entries.  One 16-byte piece of a key-tile row: eight
// E4M3 codes (x, y) with their block's scale byte (z), or eight bf16 values
// (the RoPE dims of a record, or a window row).
struct MixedPiece {
  uint4 v;
};

// Loads region pair h (dims 128 h .. 128 h + 127) of this thread's rows of the
// key tile from the entry records or the bf16 window rows.
__device__ __forceinline__ void mixed_load(const TcAttnArgs& a, int h, int pw, int quad, int g8,
                                           int64_t key0, int64_t k_hi, int64_t n_ent,
                                           const int32_t* list, const Item& x,
                                           MixedPiece (&pc)[kGatherIters][2]) {
  constexpr int kCq = kC - 64;               // FP8 dims of a record
  constexpr int kScaleOff = kCq + 2 * 64;    // scale bytes after the bf16 RoPE dims
#pragma unroll
  for (int u = 0; u < kGatherIters; ++u) {
    const int r = 4 * (pw + kProdWarps * u) + quad;
    const int64_t key = key0 + r;
    const bool ok = pw + kProdWarps * u < kBK / 4 && key < k_hi;
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int reg = 2 * h + rr;
      pc[u][rr].v = make_uint4(0u, 0u, 0u, 0u);
      if (!ok) continue;
      if (key < n_ent) {
        const int64_t e = a.sparse ? list[key] : key;
        const uint8_t* rec = a.ent_mixed + (x.bidx * a.N + e) * (int64_t)a.rec_bytes;
        if (reg < kRegions - 1) {
          const uint2 c8 = __ldg(reinterpret_cast<const uint2*>(rec + reg * 64 + g8 * 8));
          pc[u][rr].v = make_uint4(c8.x, c8.y, (uint32_t)rec[kScaleOff + reg * 2 + (g8 >> 2)], 0u);
        } else {
          pc[u][rr].v = __ldg(reinterpret_cast<const uint4*>(rec + kCq + g8 * 16));
        }
      } else {
        const bf16* wr = a.win + (x.bidx * a.Tw + (x.jlo - x.wp0) + (key - n_ent)) * kC;
        pc[u][rr].v = __ldg(reinterpret_cast<const uint4*>(wr + reg * 64 + g8 * 8));
      }
    }
  }
}

// Widens region pair h's pieces exactly to bf16 (E4M3 x 2^(scale - 127)),
// stores them at the swizzled places the cp.async gather fills, fences them
// for the tensor core's async-proxy reads and arrives on the pair's barrier.
// A piece is FP8 when its row is an entry and its region is one of the first
// seven; window rows and region 7 are bf16 as loaded; rows past the key list
// are zeros.
__device__ __forceinline__ void mixed_store(uint32_t tile, int h, int pw, int quad, int g8,
                                            int64_t key0, int64_t k_hi, int64_t n_ent,
                                            const MixedPiece (&pc)[kGatherIters][2],
                                            uint64_t* bar) {
#pragma unroll
  for (int u = 0; u < kGatherIters; ++u) {
    if (pw + kProdWarps * u >= kBK / 4) continue;
    const int r = 4 * (pw + kProdWarps * u) + quad;
    const int64_t key = key0 + r;
    const uint32_t dst = tile + (uint32_t)r * 128u + (((uint32_t)g8 ^ (uint32_t)(r & 7)) << 4);
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      uint4 v = pc[u][rr].v;
      if (key >= k_hi) {
        v = make_uint4(0u, 0u, 0u, 0u);
      } else if (key < n_ent && 2 * h + rr < kRegions - 1) {
        // 2^(byte - 127) as a float: the byte is the exponent field (byte 0 is
        // the subnormal 2^-127); E4M3 x 2^k is exact in float and in bf16
        const float sc = __uint_as_float(v.z ? (v.z << 23) : 0x00400000u);
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t word = q < 2 ? v.x : v.y;
          const __nv_fp8x2_storage_t two = (__nv_fp8x2_storage_t)(word >> (16 * (q & 1)));
          const float2 f = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(two, __NV_E4M3)));
          w[q] = pack_bf16x2(f.x * sc, f.y * sc);
        }
        v = make_uint4(w[0], w[1], w[2], w[3]);
      }
      const uint32_t d = dst + (uint32_t)((2 * h + rr) * kKRegion);
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(d), "r"(v.x), "r"(v.y),
                   "r"(v.z), "r"(v.w)
                   : "memory");
    }
  }
  fence_proxy_async_smem();
  mbar_arrive(bar);
}

// Decode split size of a row with n_keys keys: at least kSplitKeys, and large
// enough (whole 64-key blocks) for at most kMaxSplits splits.  It depends on
// the row's own key count only, so a row's result does not depend on the
// batch it runs in.
__host__ __device__ __forceinline__ int64_t split_keys_for(int64_t n_keys) {
  const int64_t per = (n_keys + kMaxSplits - 1) / kMaxSplits;
  const int64_t blk = (per + kBK - 1) / kBK * kBK;
  return blk > kSplitKeys ? blk : kSplitKeys;
}

// Key range [lo, hi) of an item and its number of 64-key blocks.
__device__ __forceinline__ int item_blocks(const TcAttnArgs& a, const Item& x, int64_t n_ent,
                                           int64_t* lo, int64_t* hi) {
  const int64_t n_keys = n_ent + x.n_w;
  int64_t l = 0, h = n_keys;
  if (a.split) {
    const int64_t sk = split_keys_for(n_keys);
    l = (int64_t)x.split * sk;
    h = l + sk < n_keys ? l + sk : n_keys;
  }
  *lo = l;
  *hi = h;
  return h > l ? (int)((h - l + kBK - 1) / kBK) : 0;
}

// MIXED: the entries are mixed BF16 / MX-FP8 records (a separate instantiation,
// so the bf16 gather compiles exactly as without it).
template <bool MIXED>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap map_q, TcAttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sQ = sm + OFF_Q;
  float* mb2s = reinterpret_cast<float*>(sm + OFF_MB);
  float* c2s = reinterpret_cast<float*>(sm + OFF_C2);
  float* ropes = reinterpret_cast<float*>(sm + OFF_ROPE);
  float* sinv = reinterpret_cast<float*>(sm + OFF_INV);
  float* ss7 = reinterpret_cast<float*>(sm + OFF_SS7);
  int* nent = reinterpret_cast<int*>(sm + OFF_NENT);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  // key tiles move in four region pairs (dims 128 h .. 128 h + 127, regions
  // 2h and 2h+1), the columns one O^T slice reads: barrier [4 s + h]
  uint64_t* kfull = bars;        // [2][4] region pair landed (producer threads)
  uint64_t* bfree = bars + 8;    // [2][4] O^T slice h of the block done: its regions free;
                                 //        [4 s + 3] also frees P tile s (row sums go first)
  uint64_t* sfull = bars + 16;   // [2] S^T of the block done
  uint64_t* pfull = bars + 18;   // [2] P tile written (128 softmax threads)
  uint64_t* iready = bars + 20;  // [2] item's entry count published
  uint64_t* qraw = bars + 22;    // raw q rows landed in the Q tile (TMA)
  uint64_t* qload = bars + 23;   // Q tile complete: RoPE dims rotated (128 softmax threads)
  uint64_t* qfree = bars + 24;   // last S^T of the item done and its Q rows read (2)
  uint64_t* ofull = bars + 25;   // last O^T (and row-sum MMA) of the item done
  uint64_t* drain = bars + 26;
  uint64_t* ifree = bars + 27;   // [2] both issuers, softmax and epilogue have read the item slot
  uint64_t* qready = bars + 29;  // [4] the item's per-head factors ready (epilogue)
  uint64_t* ofree = bars + 33;   // [4] epilogue has read O^T columns 64 jt .. 64 jt + 63
  uint64_t* drain_o = bars + 37;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
  int* wcnt = reinterpret_cast<int*>(sm + OFF_MISC + 8);        // [kProdWarps]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_MISC + 40);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float scale = a.scale > 0.f ? a.scale : rsqrtf((float)kC);

  if (threadIdx.x == 0) {
    for (int i = 0; i < 8; ++i) {
      mbar_init(&kfull[i], kProdThreads);
      mbar_init(&bfree[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sfull[i], 1);
      mbar_init(&pfull[i], 128);
      mbar_init(&iready[i], 1);
      mbar_init(&ifree[i], 4);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&qready[i], 1);
      mbar_init(&ofree[i], 128);
    }
    mbar_init(qraw, 1);
    mbar_init(qload, 128);
    mbar_init(qfree, 2);
    mbar_init(ofull, 1);
    mbar_init(drain, 1);
    mbar_init(drain_o, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  // ones tile of the row-sum MMA: bf16 1.0 everywhere, so the swizzle is moot
  if (threadIdx.x < 256) {
    reinterpret_cast<uint32_t*>(sm + OFF_ONES)[threadIdx.x] = 0x3F803F80u;
    fence_proxy_async_smem();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 0 && (int64_t)blockIdx.x < a.n_items) {
    // the first item's q rows into L2 while the previous kernel may still
    // run: a prefetch reads nothing into this CTA (L2 stays coherent with
    // that kernel's writes) and its address needs only the launch arguments
    int64_t row, hg;
    item_row_hg(a, blockIdx.x, &row, &hg);
    const bf16* q0 = a.q + (row * a.H + hg * kHG) * kC;
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(q0), "r"(kHG * kC * 2)
                 : "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // set-up done without a global load or store: from here on the previous
  // kernel's results are needed (a programmatic launch overlaps only the
  // set-up and the prefetch)
  pdl_wait();
  pdl_trigger();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS0 = tmem;          // S^T buffers at columns 0 and 64
  const uint32_t tO = tmem + 128;     // O^T: 4 x 64 columns
  const uint32_t tL = tmem + 384;     // per-head sums of P (64 columns, rows identical)

  // register budgets per warpgroup (every warp of a warpgroup takes the same)
  if (warp < 8)
    setmaxnreg_inc<kRegHeavy>();
  else
    setmaxnreg_dec<kRegLight>();

  // Failure handling (every role): a wait that runs out marks the thread
  // `dead` (made warp-uniform); dead threads skip waits and work but still
  // pass every named barrier, so no barrier can be left waiting.
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

  if (prod_index(warp) >= 0) {
    // ======================= producer (6 warps)
    // Item n's index list and RoPE table are built while item n-1's keys
    // stream (its index loads are issued early and consumed a block later),
    // so an item starts with its Q tile and first key tiles only.
    const int pw = prod_index(warp), ptid = pw * 32 + lane;
    const int quad = lane >> 3, g8 = lane & 7;
    const uint32_t kbase = smem_u32(sm + OFF_K);
    constexpr int kEv = (kMaxK / kProdWarps + 31) / 32 + 1;   // index words per lane
    int32_t ev[kEv];
    // RoPE frequency of pair `lane` (warp 0 builds the per-item cos/sin table)
    const double theta = rope_theta(lane, a.r > 0 ? a.r : 2, a.base);
    // index loads of item (it, m): warp pw takes the contiguous pw-th share of the row
    auto load_idx = [&](int64_t row) {
      const int32_t* ir = a.idx + row * (int64_t)a.k;
      const int q3 = (a.k + kProdWarps - 1) / kProdWarps;   // this warp's share
      const int lo = pw * q3, hi = lo + q3 < a.k ? lo + q3 : a.k;
#pragma unroll
      for (int u = 0; u < kEv; ++u) {
        const int i = lo + u * 32 + lane;
        // volatile loads: issued here, a block before their use, not sunk to it
        ev[u] = (!dead && a.sparse && u * 32 < q3 && i < hi) ? ldg_nc_volatile(ir + i) : -1;
      }
    };
    // builds item m's index list, RoPE table and entry count (slot m & 1)
    auto compact = [&](const Item& y, int m) -> int64_t {
      wait_or_die(&ifree[m & 1], (uint32_t)((m >> 1) & 1) ^ 1u, 19u);   // item m-2 consumed
      float* rcs = ropes + (m & 3) * 64;
      if (!dead && pw == 0 && lane < (a.r >> 1)) {
        float cs, sn;
        rope_cos_sin_theta(y.pos, theta, &cs, &sn);
        rcs[lane] = cs;
        rcs[32 + lane] = sn;
      }
      int64_t ne;
      if (a.sparse) {
        const int lo = pw * ((a.k + kProdWarps - 1) / kProdWarps);
        int32_t* list = reinterpret_cast<int32_t*>(sm + OFF_LIST) + (m & 1) * kMaxK;
        int cnt = 0;
#pragma unroll
        for (int u = 0; u < kEv; ++u) {
          const bool ok = ev[u] >= 0 && ev[u] < a.N;
          if (!ok && ev[u] != -1)
            report(a.status, CSA_DEV_BAD_INDEX, (unsigned)(lo + u * 32 + lane));
          cnt += __popc(__ballot_sync(0xffffffffu, ok));
        }
        named_bar(2, kProdThreads);   // previous use of wcnt finished
        if (lane == 0) wcnt[pw] = cnt;
        named_bar(2, kProdThreads);
        int off = 0;
        for (int w = 0; w < pw; ++w) off += wcnt[w];
        ne = 0;
        for (int w = 0; w < kProdWarps; ++w) ne += wcnt[w];
#pragma unroll
        for (int u = 0; u < kEv; ++u) {
          const bool ok = ev[u] >= 0 && ev[u] < a.N;
          const unsigned bal = __ballot_sync(0xffffffffu, ok);
          if (ok) list[off + __popc(bal & ((1u << lane) - 1u))] = ev[u];
          off += __popc(bal);
        }
      } else {
        ne = vis_count(y.pos, a.m_dense, a.N);
      }
      named_bar(2, kProdThreads);   // the index list and the RoPE table are complete
      if (!dead && ptid == 0) {
        nent[m & 1] = (int)ne;
        mbar_arrive(&iready[m & 1]);
      }
      return ne;
    };

    int64_t gblk = 0;
    int n = 0;
    int64_t cur_ent = 0;
    if ((int64_t)blockIdx.x < a.n_items) {
      if (ptid == 0) {
        // the first item's raw q rows, before anything else: their load
        // overlaps the item's position reads and index compaction
        int64_t row, hg;
        item_row_hg(a, blockIdx.x, &row, &hg);
        mbar_arrive_expect_tx(qraw, kRegions * kQRegion);
        for (int r = 0; r < kRegions; ++r)
          tma_load_3d(sQ + r * kQRegion, &map_q, qraw, r * 64, (int32_t)(hg * kHG), (int32_t)row);
      }
      const Item y = decode_item(a, blockIdx.x);
      load_idx(y.row);
      cur_ent = compact(y, 0);
    }
    for (int64_t it = blockIdx.x; it < a.n_items; it += gridDim.x, ++n) {
      const Item x = decode_item(a, it);
      const int32_t* list = reinterpret_cast<const int32_t*>(sm + OFF_LIST) + (n & 1) * kMaxK;
      const int64_t n_ent = cur_ent;
      int64_t k_lo = 0, k_hi = 0;
      const int nb = dead ? 0 : item_blocks(a, x, n_ent, &k_lo, &k_hi);
      const int nbl = nb > 0 ? nb : 1;
      const int64_t it_next = it + gridDim.x;
      const bool has_next = it_next < a.n_items;
      const Item y = decode_item(a, has_next ? it_next : it);
      if (!dead && ptid == 0 && has_next) {   // warm L2 with the next item's q rows
        const bf16* qn = a.q + (y.row * a.H + (int64_t)y.hg * kHG) * kC;
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(qn), "r"(kHG * kC * 2)
                     : "memory");
      }
      // the previous item's last S^T is done with Q: the raw q rows by TMA
      // (the first item's were issued before its compaction)
      if (n > 0) wait_or_die(qfree, (uint32_t)(n - 1) & 1u, 20u);
      if (!dead && ptid == 0 && n > 0) {
        mbar_arrive_expect_tx(qraw, kRegions * kQRegion);
        for (int r = 0; r < kRegions; ++r)
          tma_load_3d(sQ + r * kQRegion, &map_q, qraw, r * 64, x.hg * kHG, (int32_t)x.row);
      }

      const bf16* ent = a.entries + x.bidx * a.N * kC;
      const bf16* win = a.win + x.bidx * a.Tw * kC;
      const float* rcs = ropes + (n & 3) * 64;
      for (int b = 0; b < nbl; ++b) {
        const int64_t j = gblk + b;
        const int s = (int)(j & 1);
        if (b < nb) {
          const uint32_t tile = kbase + s * kKTile;
          // groups of four rows (one per 8-lane quad; 128 bytes per lane group
          // and region) dealt round-robin over the producer warps
          const bf16* src[kGatherIters];
#pragma unroll
          for (int u = 0; u < kGatherIters; ++u) {
            const int r = 4 * (pw + kProdWarps * u) + quad;
            const int64_t key = k_lo + (int64_t)b * kBK + r;
            src[u] = nullptr;
            if (!dead && pw + kProdWarps * u < kBK / 4 && key < k_hi)
              src[u] = key < n_ent ? ent + (int64_t)(a.sparse ? list[key] : key) * kC
                                   : win + ((x.jlo - x.wp0) + (key - n_ent)) * kC;
          }
          if constexpr (MIXED) {
            // region pair h + 1's record loads are in flight while pair h is
            // widened and stored (two register sets, the pair loop unrolled)
            MixedPiece ra[kGatherIters][2], rb[kGatherIters][2];
            const int64_t key0 = k_lo + (int64_t)b * kBK;
            if (!dead) mixed_load(a, 0, pw, quad, g8, key0, k_hi, n_ent, list, x, ra);
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              MixedPiece (&cur)[kGatherIters][2] = (h & 1) ? rb : ra;
              MixedPiece (&nxt)[kGatherIters][2] = (h & 1) ? ra : rb;
              if (!dead && h < 3)
                mixed_load(a, h + 1, pw, quad, g8, key0, k_hi, n_ent, list, x, nxt);
              wait_or_die(&bfree[4 * s + h], (uint32_t)((j >> 1) & 1) ^ 1u, 21u);
              if (!dead)
                mixed_store(tile, h, pw, quad, g8, key0, k_hi, n_ent, cur, &kfull[4 * s + h]);
            }
          } else {
          // region pair h as soon as O^T slice h of the tile's previous block
          // has read it
#pragma unroll 1
          for (int h = 0; h < 4; ++h) {
            wait_or_die(&bfree[4 * s + h], (uint32_t)((j >> 1) & 1) ^ 1u, 21u);
            if (!dead) {
#pragma unroll
              for (int u = 0; u < kGatherIters; ++u) {
                if (pw + kProdWarps * u >= kBK / 4) continue;
                const int r = 4 * (pw + kProdWarps * u) + quad;
                const uint32_t dst =
                    tile + (uint32_t)r * 128u + (((uint32_t)g8 ^ (uint32_t)(r & 7)) << 4);
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                  const int reg = 2 * h + rr;
                  const void* sp =
                      src[u] ? (const void*)(src[u] + reg * 64 + g8 * 8) : (const void*)a.q;
                  cp_async16(dst + reg * kKRegion, sp, src[u] ? 16u : 0u);
                }
              }
              // the barrier counts this thread's arrival once its copies land
              cp_async_arrive(&kfull[4 * s + h]);
            }
          }
          }
        }
        if (b == 0) {
          if (has_next) load_idx(y.row);   // consumed by the compaction below
        }
        if (b == (nbl > 2 ? 2 : nbl - 1) && has_next) cur_ent = compact(y, n + 1);
      }
      gblk += nb;
    }
    cp_async_wait<0>();
  } else if (warp == kMmaWarp) {
    // ======================= S^T issuer (TMEM owner)
    if (elect_one()) {
      constexpr uint32_t idS = idesc_bf16_f32(kBK, kHG, 0, 0);
      // descriptors built once; an operand at byte offset o adds o >> 4 to the
      // start-address field (every offset stays inside shared memory)
      const uint64_t dK = smem_desc(smem_u32(sm + OFF_K), 16, 1024, 2);   // A: key tile
      const uint64_t dQ = smem_desc(smem_u32(sQ), 16, 1024, 2);           // B: Q tile
      int64_t gblk = 0;
      int n = 0;
      bool ok = true;
      for (int64_t it = blockIdx.x; ok && it < a.n_items; it += gridDim.x, ++n) {
        const Item x = decode_item(a, it);
        if (!mbar_wait(&iready[n & 1], (uint32_t)(n >> 1) & 1u)) { ok = false; break; }
        int64_t k_lo, k_hi;
        const int nb = item_blocks(a, x, nent[n & 1], &k_lo, &k_hi);
        mbar_arrive(&ifree[n & 1]);
        // the raw q rows suffice for Q regions 0-5; region 7's RoPE dims are
        // rotated in place by the softmax warps (qload) before region pair 3
        if (*abort_flag || !mbar_wait(qraw, (uint32_t)n & 1u)) { ok = false; break; }
        tc_fence_after();
        if (nb == 0 && (*abort_flag || !mbar_wait(qload, (uint32_t)n & 1u))) { ok = false; break; }
        for (int b = 0; b < nb; ++b) {
          const int64_t j = gblk + b;
          const int s = (int)(j & 1);
          // S^T buffer s is free once the softmax has turned S^T(j-2) into P
          if ((j >= 2 && !mbar_wait(&pfull[s], (uint32_t)((j - 2) >> 1) & 1u)) || *abort_flag) {
            ok = false;
            break;
          }
          const uint64_t dKs = dK + (uint64_t)((s * kKTile) >> 4);
          // each region pair as soon as its gather landed
#pragma unroll 1
          for (int h = 0; h < 4 && ok; ++h) {
            if (b == 0 && h == 3 && (*abort_flag || !mbar_wait(qload, (uint32_t)n & 1u))) {
              ok = false;
              break;
            }
            if (*abort_flag || !mbar_wait(&kfull[4 * s + h], (uint32_t)(j >> 1) & 1u)) {
              ok = false;
              break;
            }
            fence_proxy_async_smem();   // cp.async (generic proxy) writes -> MMA reads
            tc_fence_after();
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
              const int reg = 2 * h + rr;
#pragma unroll
              for (int kq = 0; kq < 4; ++kq)
                mma_bf16_ss(tS0 + 64 * s, dKs + (uint64_t)((reg * kKRegion + kq * 32) >> 4),
                            dQ + (uint64_t)((reg * kQRegion + kq * 32) >> 4), idS,
                            (reg | kq) != 0 ? 1u : 0u);
            }
          }
          if (!ok) break;
          mma_commit(&sfull[s]);
        }
        if (!ok) break;
        mma_commit(qfree);   // the item's S^T MMAs are the Q tile's only readers
        gblk += nb;
      }
      if (!ok) {
        *abort_flag = 1;
        report(a.status, CSA_DEV_TIMEOUT, 23u);
      }
      mma_commit(drain);
      mbar_wait(drain, 0);
    }
  } else if (warp == kMmaWarpO) {
    // ======================= O^T and row-sum issuer
    if (elect_one()) {
      constexpr uint32_t idO = idesc_bf16_f32(128, kHG, 1, 1);
      constexpr uint32_t idL = idesc_bf16_f32(kBK, kHG, 0, 1);
      const uint64_t dV = smem_desc(smem_u32(sm + OFF_K), kKRegion, 1024, 2);   // O^T A
      const uint64_t dP = smem_desc(smem_u32(sm + OFF_P), kKRegion, 1024, 2);   // O^T, L B
      const uint64_t dOnes = smem_desc(smem_u32(sm + OFF_ONES), 16, 0, 2);      // L A
      int64_t gblk = 0;
      int n = 0;
      bool ok = true;
      for (int64_t it = blockIdx.x; ok && it < a.n_items; it += gridDim.x, ++n) {
        const Item x = decode_item(a, it);
        if (!mbar_wait(&iready[n & 1], (uint32_t)(n >> 1) & 1u)) { ok = false; break; }
        int64_t k_lo, k_hi;
        const int nb = item_blocks(a, x, nent[n & 1], &k_lo, &k_hi);
        mbar_arrive(&ifree[n & 1]);
        if (nb == 0) {
          // keep ofull at most one phase ahead of the epilogue
          if (n > 0 && !mbar_wait(&ofree[3], (uint32_t)(n - 1) & 1u)) { ok = false; break; }
          mma_commit(ofull);
          continue;
        }
        for (int b = 0; b < nb; ++b) {
          const int64_t j = gblk + b;
          const int s = (int)(j & 1);
          if (*abort_flag || !mbar_wait(&pfull[s], (uint32_t)(j >> 1) & 1u)) { ok = false; break; }
          tc_fence_after();
          const uint64_t dVs = dV + (uint64_t)((s * kKTile) >> 4);
          const uint64_t dPs = dP + (uint64_t)((s * kPTile) >> 4);
          // L[., h] += sum over the block's keys of P^T[key, h]: A = 64 rows of
          // ones (stride 0 repeats one 8-row group), B = the P^T tile.  Issued
          // first, so the last slice's commit covers every reader of P tile s
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_bf16_ss(tL, dOnes + (uint64_t)((kk * 32) >> 4), dPs + (uint64_t)((kk * 2048) >> 4),
                        idL, (b > 0 || kk > 0) ? 1u : 0u);
#pragma unroll 1
          for (int jt = 0; jt < 4; ++jt) {
            // the item's first block overwrites O^T: wait for the epilogue to
            // have read the previous item's columns of this slice
            if (b == 0 && n > 0) {
              if (!mbar_wait(&ofree[jt], (uint32_t)(n - 1) & 1u)) { ok = false; break; }
              tc_fence_after();
            }
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk)
              mma_bf16_ss(tO + 64 * jt, dVs + (uint64_t)((2 * jt * kKRegion + kk * 2048) >> 4),
                          dPs + (uint64_t)((kk * 2048) >> 4), idO, (b > 0 || kk > 0) ? 1u : 0u);
            // regions 2 jt, 2 jt + 1 of key tile s read (S^T(j) finished before P(j))
            mma_commit(&bfree[4 * s + jt]);
          }
          if (!ok) break;
        }
        if (!ok) break;
        mma_commit(ofull);
        gblk += nb;
      }
      if (!ok) {
        *abort_flag = 1;
        report(a.status, CSA_DEV_TIMEOUT, 28u);
      }
      mma_commit(drain_o);
      mbar_wait(drain_o, 0);
    }
  } else if (warp < 4) {
    // ======================= softmax (warps 0-3)
    const int rw = warp * 32 + lane;
    // M = 64 scores read with the 16x64b shape: this lane holds key row kb_row
    // of the block and the heads of parity `par` (head 2 j + par in slot j)
    const int par = (lane >> 1) & 1;
    const int kb_row = warp * 16 + (lane >> 2) + 8 * (lane & 1);
    int64_t gblk = 0;
    int n = 0;
    for (int64_t it = blockIdx.x; it < a.n_items; it += gridDim.x, ++n) {
      const int ip = n & 1;
      const Item x = decode_item(a, it);
      wait_or_die(&iready[ip], (uint32_t)(n >> 1) & 1u, 24u);
      int64_t k_lo = 0, k_hi = 0;
      const int nb = dead ? 0 : item_blocks(a, x, nent[ip], &k_lo, &k_hi);
      // as soon as the raw q rows land, the Q tile's dims 448..511 (region
      // 7): lane `lane` rotates pair `lane` (dims 448 + 2 lane, + 1) of heads
      // warp, warp + 4, ... in place, all of its loads in flight at once (the
      // lanes cover one 128-byte row: no bank conflicts), keeping the raw
      // squares; a transposing butterfly leaves head warp + 4 l's raw sum of
      // squares in lane l < 16.  Then the MMA may read the Q tile.
      wait_or_die(qraw, (uint32_t)n & 1u, 24u);
      if (!dead) {
        const float* rcs = ropes + (n & 3) * 64;
        const int d = (kRegions - 1) * 64 + 2 * lane;   // even dim of the pair
        const bool rot = !(a.flags & CSA_F_NO_ROPE) && d >= kC - a.r;
        const int pi = rot ? (d - (kC - a.r)) >> 1 : 0;
        const float cs = rot ? rcs[pi] : 1.f, sn = rot ? rcs[32 + pi] : 0.f;
        uint8_t* q7 = sQ + (kRegions - 1) * kQRegion + (lane & 3) * 4;
        uint32_t wv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int h = warp + 4 * i;
          wv[i] = *reinterpret_cast<const uint32_t*>(q7 + h * 128 + (((lane >> 2) ^ (h & 7)) << 4));
        }
        float sq[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int h = warp + 4 * i;
          const float x0 = bf16_bits_to_float(wv[i] & 0xffffu);
          const float x1 = bf16_bits_to_float(wv[i] >> 16);
          sq[i] = fmaf(x0, x0, x1 * x1);
          if (rot)
            *reinterpret_cast<uint32_t*>(q7 + h * 128 + (((lane >> 2) ^ (h & 7)) << 4)) =
                pack_bf16x2(x0 * cs - x1 * sn, x0 * sn + x1 * cs);
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) sq[i] += __shfl_xor_sync(0xffffffffu, sq[i], 16);
#pragma unroll
        for (int off = 8; off >= 1; off >>= 1) {
          const bool up = (lane & off) != 0;
#pragma unroll
          for (int i = 0; i < off; ++i) {
            const float send = up ? sq[i] : sq[i + off];
            const float keep = up ? sq[i + off] : sq[i];
            sq[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
          }
        }
        if (lane < 16) ss7[warp + 4 * lane] = sq[0];
        fence_proxy_async_smem();   // generic stores -> the MMA's reads
        mbar_arrive(qload);
      }
      // per-head factors while S^T(0) runs: thread rw sums half of head rw/2's
      // raw dims 0..447 (Q tile regions 0-3 or 4-6, rotated chunk order for the
      // banks) and adds region 7's raw sum from above
      wait_or_die(qload, (uint32_t)n & 1u, 24u);
      if (!dead) {
        const int h = rw >> 1, hh = rw & 1;
        float ss = 0.f;
        for (int r = 4 * hh; r < (hh ? kRegions - 1 : 4); ++r) {
          const uint8_t* qr = sQ + r * kQRegion + h * 128;
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            const uint4 v = *reinterpret_cast<const uint4*>(qr + (((g + h) & 7) << 4));
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float x0 = bf16_bits_to_float(w4[e] & 0xffffu);
              const float x1 = bf16_bits_to_float(w4[e] >> 16);
              ss = fmaf(x0, x0, fmaf(x1, x1, ss));
            }
          }
        }
        ss += __shfl_xor_sync(0xffffffffu, ss, 1);
        if (hh == 0) {
          ss += ss7[h];
          const float inv = (a.flags & CSA_F_NO_NORM) ? 1.f : rsqrtf(ss / (float)kC + a.eps);
          c2s[(n & 3) * kHG + h] = scale * inv * kLog2e;
          // bound of the head's logits against unit-RMS keys (bf16 slack 2^-7)
          mb2s[(n & 3) * kHG + h] =
              scale * sqrtf(ss) * inv * sqrtf((float)kC) * (1.f + 0.0078125f) * kLog2e;
        }
      }
      named_bar(1, 128);   // factors complete; the Q rows are no longer read here
      if (rw == 0 && !dead) {
        mbar_arrive(qfree);
        mbar_arrive(&qready[n & 3]);
      }
      float mbr[32], c2r[32];   // this lane's heads 2 j + par
      {
        const float* mb2 = mb2s + (n & 3) * kHG;
        const float* c2h = c2s + (n & 3) * kHG;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          mbr[j] = mb2[2 * j + par];
          c2r[j] = c2h[2 * j + par];
        }
      }
      named_bar(1, 128);   // every thread has read the item slot
      if (rw == 0 && !dead) mbar_arrive(&ifree[ip]);
      float xmax = -INFINITY;
      for (int b = 0; b < nb; ++b) {
        const int64_t j = gblk + b;
        const int s = (int)(j & 1);
        const uint32_t ph = (uint32_t)(j >> 1) & 1u;
        wait_or_die(&sfull[s], ph, 25u);
        uint32_t wds[16];   // bf16 pairs of P for this lane's half row
        if (!dead) {
          tc_fence_after();
          uint32_t sv[32];
          tmem_ld16x64b_x32(tmem_addr(tS0 + 64 * s, (uint32_t)(warp * 32), 0), sv);
          tmem_ld_wait();
          const bool valid = k_lo + (int64_t)b * kBK + kb_row < k_hi;
          uint32_t mine[16];   // my 32 probabilities as bf16, two per word
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float x0 = valid ? fmaf(__uint_as_float(sv[e]), c2r[e], -mbr[e]) : -INFINITY;
            const float x1 =
                valid ? fmaf(__uint_as_float(sv[e + 1]), c2r[e + 1], -mbr[e + 1]) : -INFINITY;
            xmax = fmaxf(xmax, fmaxf(x0, x1));
            mine[e >> 1] = pack_bf16x2(ex2(x0), ex2(x1));
          }
          // the partner lane (lane ^ 2) holds the other parity of the same key:
          // even-parity lanes assemble heads 0..31, odd-parity lanes 32..63
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint32_t send = par ? mine[q] : mine[8 + q];
            const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, 2);
            // recv holds the partner's slots 2q, 2q+1 (+16 for the odd side)
            const uint32_t m = par ? mine[8 + q] : mine[q];
            // word for slot i = 2q+u: low half = even head, high half = odd head
            const uint32_t ev0 = par ? (recv & 0xffffu) : (m & 0xffffu);
            const uint32_t od0 = par ? (m & 0xffffu) : (recv & 0xffffu);
            const uint32_t ev1 = par ? (recv >> 16) : (m >> 16);
            const uint32_t od1 = par ? (m >> 16) : (recv >> 16);
            wds[2 * q] = ev0 | (od0 << 16);
            wds[2 * q + 1] = ev1 | (od1 << 16);
          }
        }
        wait_or_die(&bfree[4 * s + 3], ph ^ 1u, 25u);   // O^T(j-2) has read this P tile
        if (!dead) {
          uint8_t* prow = sm + OFF_P + s * kPTile + kb_row * 128;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4*>(prow + (((par * 4 + q) ^ (kb_row & 7)) << 4)) =
                make_uint4(wds[4 * q], wds[4 * q + 1], wds[4 * q + 2], wds[4 * q + 3]);
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive(&pfull[s]);
        }
      }
      if (xmax > kRangeLog2) report(a.status, CSA_DEV_RANGE, (unsigned)x.row);
      gblk += nb;
    }
  } else if (warp < 8) {
    // ======================= epilogue (warps 4-7; warp 4 + ew reads TMEM lanes
    // 32 ew .. 32 ew + 31): thread = output dim, overlapping the next item
    const int ew = warp - 4, etid = threadIdx.x - 128;
    int n = 0;
    for (int64_t it = blockIdx.x; it < a.n_items; it += gridDim.x, ++n) {
      const int ip = n & 1;
      const Item x = decode_item(a, it);
      wait_or_die(&iready[ip], (uint32_t)(n >> 1) & 1u, 27u);
      wait_or_die(&qready[n & 3], (uint32_t)(n >> 2) & 1u, 27u);
      int64_t k_lo = 0, k_hi = 0;
      const int nb = dead ? 0 : item_blocks(a, x, nent[ip], &k_lo, &k_hi);
      named_bar(3, 128);   // every epilogue thread has read the entry count
      if (etid == 0 && !dead) mbar_arrive(&ifree[ip]);
      // the item's factor slot stays intact until this item's epilogue ends:
      // the producer refills it four items later, after this role's ifree
      const float* mb2 = mb2s + (n & 3) * kHG;
      const int64_t slot = x.row * a.n_hg + x.hg;
      float ecs[4], esn[4];   // RoPE factors of this thread's output pair, per slice
      {
        const float* rcs = ropes + (n & 3) * 64;
#pragma unroll
        for (int jt = 0; jt < 4; ++jt) {
          const int cc = 128 * jt + ew * 32 + (lane & ~1);
          ecs[jt] = 1.f;
          esn[jt] = 0.f;
          if (!(a.flags & CSA_F_NO_ROPE) && cc >= kC - a.r) {
            const int pi = (cc - (kC - a.r)) >> 1;
            ecs[jt] = rcs[pi];
            esn[jt] = rcs[32 + pi];
          }
        }
      }
      wait_or_die(ofull, (uint32_t)n & 1u, 26u);
      tc_fence_after();
      const bool have_o = nb > 0 && !dead;
      if (x.split == 0 && a.split && etid < kHG && !dead) a.mb_part[slot * kHG + etid] = mb2[etid];

      // per-head denominators: the row-sum MMA's result, the same in every row;
      // warp 4 lanes 0..15 read rows 0..15 and publish heads l, l+16, l+32, l+48
      if (ew == 0) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t lv[32];
          if (have_o) {
            tmem_ld32(tmem_addr(tL + 32 * hf, 0u, 0), lv);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) lv[e] = 0u;
          }
          // lane l < 16 takes heads 32 hf + l and 32 hf + l + 16 (static selects:
          // no dynamically indexed registers)
          float t0 = 0.f, t1 = 0.f;
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            t0 = e == lane ? __uint_as_float(lv[e]) : t0;
            t1 = e == lane ? __uint_as_float(lv[e + 16]) : t1;
          }
          if (!dead && lane < 16) {
            const int h0 = 32 * hf + lane, h1 = h0 + 16;
            if (a.split) {
              a.d_part[(slot * a.n_splits + x.split) * kHG + h0] = t0;
              a.d_part[(slot * a.n_splits + x.split) * kHG + h1] = t1;
            } else {
              // sink: exp(z_h - M_h) joins the denominator only
              const float s0 = a.sink ? ex2(fmaf(a.sink[x.hg * kHG + h0], kLog2e, -mb2[h0])) : 0.f;
              const float s1 = a.sink ? ex2(fmaf(a.sink[x.hg * kHG + h1], kLog2e, -mb2[h1])) : 0.f;
              const float d0 = t0 + s0, d1 = t1 + s1;
              sinv[h0] = d0 > 0.f ? __frcp_rn(d0) : 0.f;
              sinv[h1] = d1 > 0.f ? __frcp_rn(d1) : 0.f;
            }
          }
        }
      }
      named_bar(3, 128);

      // O^T -> output: thread = dim 128 jt + 32 ew + lane
      const int odd = lane & 1;
#pragma unroll 1
      for (int jt = 0; jt < 4; ++jt) {
        const int c = 128 * jt + ew * 32 + lane;
        const int cc = c - odd;
        const float cs = ecs[jt], sn = esn[jt];
#pragma unroll
        for (int half = 0; half < 2; ++half) {   // heads 32 half .. 32 half + 31
          uint32_t ov[32];
          if (have_o) {
            tmem_ld32(tmem_addr(tO + 64 * jt + 32 * half, (uint32_t)(ew * 32), 0), ov);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = 0u;
          }
          if (half == 1 && !dead) {   // this slice's columns are read: O^T may reuse them
            tc_fence_before();
            mbar_arrive(&ofree[jt]);
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
              const float v0 = __uint_as_float(ov[e]) * sinv[h];   // broadcast reads
              const float v1 = __uint_as_float(ov[e + 1]) * sinv[h + 1];
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
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Sums the fixed-order split partials of one (row, head group), divides by
// the denominator (sink included) and rotates the output back by -pos.
constexpr int kCombHeads = 2;   // heads per combine CTA (one 16-byte quad a thread)

__global__ void __launch_bounds__(256, 6) attn_combine_kernel(TcAttnArgs a) {
  static_assert(kCombHeads * kC / 4 == 256, "one 16-byte quad a thread");
  __shared__ float inv[kCombHeads];
  __shared__ float cs_t[32], sn_t[32];
  pdl_wait();
  pdl_trigger();
  const int64_t row = blockIdx.x;
  const int hg = blockIdx.y;
  const int h0 = blockIdx.z * kCombHeads;   // this CTA's heads within the group
  const int64_t slot = row * a.n_hg + hg;
  // thread: 4 consecutive dims of one head; every split's 16-byte load is
  // issued first, then the denominators and the RoPE table are formed while
  // they are in flight (the sum keeps the fixed split order)
  const int hl = threadIdx.x / (kC / 4), c = (threadIdx.x % (kC / 4)) * 4;
  constexpr int kInFlight = 4;   // split loads in flight a thread
  float4 pv[kInFlight];
  auto load = [&](int s0) {
#pragma unroll
    for (int u = 0; u < kInFlight; ++u)
      if (s0 + u < a.n_splits)
        pv[u] = *reinterpret_cast<const float4*>(
            a.o_part + ((slot * a.n_splits + s0 + u) * kHG + h0 + hl) * kC + c);
  };
  load(0);
  const int64_t t = row % a.Tq;
  const int64_t pos = a.q_pos ? a.q_pos[row] : t;
  if (threadIdx.x < kCombHeads) {
    const int h = h0 + threadIdx.x;
    float tot = 0.f;
    for (int s = 0; s < a.n_splits; ++s)   // fixed order: bits independent of the batch
      tot += a.d_part[(slot * a.n_splits + s) * kHG + h];
    if (a.sink) {
      const float z = a.sink[hg * kHG + h];
      tot += ex2(fmaf(z, kLog2e, -a.mb_part[slot * kHG + h]));
    }
    inv[threadIdx.x] = tot > 0.f ? 1.f / tot : 0.f;
  } else if (threadIdx.x >= 32 && threadIdx.x < 32 + (a.r >> 1)) {
    float cs, sn;
    rope_cos_sin_theta(-pos, rope_theta(threadIdx.x - 32, a.r, a.base), &cs, &sn);
    cs_t[threadIdx.x - 32] = cs;
    sn_t[threadIdx.x - 32] = sn;
  }
  __syncthreads();
  float o[4] = {0.f, 0.f, 0.f, 0.f};
  for (int s0 = 0; s0 < a.n_splits; s0 += kInFlight) {
    if (s0 > 0) load(s0);
#pragma unroll
    for (int u = 0; u < kInFlight; ++u) {
      if (s0 + u < a.n_splits) {
        o[0] += pv[u].x;
        o[1] += pv[u].y;
        o[2] += pv[u].z;
        o[3] += pv[u].w;
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) o[e] *= inv[hl];
  if (!(a.flags & CSA_F_NO_ROPE)) {
#pragma unroll
    for (int e = 0; e < 4; e += 2) {
      if (c + e >= kC - a.r) {
        const int i = (c + e - (kC - a.r)) >> 1;
        const float y0 = o[e] * cs_t[i] - o[e + 1] * sn_t[i];
        const float y1 = o[e] * sn_t[i] + o[e + 1] * cs_t[i];
        o[e] = y0;
        o[e + 1] = y1;
      }
    }
  }
  *reinterpret_cast<uint2*>(a.out + (row * a.H + (int64_t)hg * kHG + h0 + hl) * kC + c) =
      make_uint2(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]));
}

// Streaming multiprocessors of the current device (one persistent CTA each).
inline int64_t num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  return n;
}

// Splits per decode row: enough for the row with the most keys (a row with
// fewer keys leaves its last splits empty; their zero partials add exactly).
inline int n_splits_for(int64_t max_keys) {
  int64_t n = (max_keys + kSplitKeys - 1) / kSplitKeys;
  n = n < kMaxSplits ? n : kMaxSplits;
  return n < 1 ? 1 : (int)n;
}

}  // namespace

bool attn_tc_supported(const AttnParams& p) {
  auto al = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
  if (p.f.c != kC || p.H % kHG != 0 || p.f.r > 64 || (p.f.r & 1)) return false;
  if (p.mixed && p.f.r != 64) return false;   // the bf16 part is exactly the last region
  if (p.sparse && p.k > kMaxK) return false;   // the per-item index list holds kMaxK
  if (p.B * p.Tq >= (1LL << 31)) return false;
  if (p.Tq == 1 && p.B > 65535) return false;
  return al(p.q) && al(p.out) && (p.N == 0 || al(p.entries)) && (p.Tw == 0 || al(p.win));
}

size_t attn_tc_scratch(int64_t B, int64_t Tq, int H, int c, int64_t max_keys) {
  if (c != kC || H % kHG != 0) return 0;
  size_t bytes = 0;
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
  a.mixed = p.mixed;
  a.rec_bytes = p.rec_bytes;
  a.ent_mixed = static_cast<const uint8_t*>(p.entries);
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
  if (a.split) {
    a.n_splits = n_splits_for(max_keys);
    const int64_t slots = rows * a.n_hg;
    a.o_part = static_cast<float*>(p.scratch);
    a.d_part = a.o_part + slots * a.n_splits * kHG * kC;
    a.mb_part = a.d_part + slots * a.n_splits * kHG;
  } else {
    a.n_splits = 1;
  }
  a.n_items = rows * a.n_hg * a.n_splits;
  const unsigned grid = (unsigned)(a.n_items < num_sms() ? a.n_items : num_sms());
  CUtensorMap mq;   // q as [rows][H][512] bf16, boxes of 64 heads x 64 dims
  if (!make_map_bf16_3d(&mq, a.q, kC, (uint64_t)p.H, (uint64_t)rows, 64, kHG))
    return cudaErrorInvalidValue;
  const int smem = SMEM_BYTES + 1024;
  cudaError_t e =
      cudaFuncSetAttribute(a.mixed ? attn_tc_kernel<true> : attn_tc_kernel<false>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(a.mixed ? attn_tc_kernel<true> : attn_tc_kernel<false>, dim3(grid),
                 dim3(kThreads), (size_t)smem, stream, mq, a);
  if (e != cudaSuccess) return e;
  *n_launch = 1;
  if (a.split) {
    e = launch_pdl(attn_combine_kernel, dim3((unsigned)rows, (unsigned)a.n_hg, kHG / kCombHeads),
                   dim3(256), 0, stream, a);
    if (e != cudaSuccess) return e;
    *n_launch = 2;
  }
  return cudaSuccess;
}

}  // namespace csa
