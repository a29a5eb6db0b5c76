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
// One CTA takes one query token and 64 heads.  With c = 512 an fp32 output
// accumulator of 64 heads x 512 dims would not fit next to the scores in TMEM
// in the usual layout, so the kernel works TRANSPOSED, keys on the MMA's M
// side:
//   S^T[key, h] = K_tile . Q^T        (M = 128 keys, N = 64 heads, K = 512)
//   O^T[c, h]  += V^T . P^T            (M = 128 dims x 4, N = 64, K = 128 keys)
// which needs 64 + 4 x 64 TMEM columns.  The gathered key tile (one row per
// selected entry or window row, 1 KB each) is stored once, 128-byte swizzled,
// and read by both MMAs: K-major as the A operand of S^T and MN-major as the
// A operand of O^T (K = V).
//
// Softmax without a running maximum: q^ and every stored key are RMS-
// normalised (the method's RMSNorm), so |scale q^ . k| <= scale |q^| sqrt(c)
// =: M_h, a per-(token, head) bound known before any key is read.  Weights
// are exp(l - M_h) in (e^-2M_h, 1]: no rescaling of O, no cross-lane max, and
// split partial sums add directly.  A logit more than 60 above the bound (keys
// far from unit RMS) is reported as CSA_DEV_RANGE.
//
// Roles (288 threads): warps 0-3 softmax + epilogue (thread = TMEM lane =
// key in S^T, = output dim in O^T); warps 4-7 query prologue (RMSNorm, RoPE,
// bf16, swizzle), index compaction and the key gather (cp.async, 16 B per
// copy, region by region so the next block's gather overlaps this block's
// O^T MMAs); warp 8 owns TMEM and issues the MMAs.
// Decode rows (one query per sequence) split the key list into fixed
// 256-key pieces whose fp32 partials a combine kernel adds in a fixed order,
// so a row's result does not depend on the batch it runs in.
#include "common.cuh"
#include "sm100.cuh"
#include "tc.h"

namespace csa {

namespace {

using namespace sm100;

constexpr int kC = 512;                      // entry / head dim
constexpr int kHG = 64;                      // heads per CTA (MMA N)
constexpr int kBK = 128;                     // keys per block (MMA M of S^T)
constexpr int kRegions = kC / 64;            // 64-element (128-byte) column chunks
constexpr int kKRegion = kBK * 128;          // 16 KB per key-tile chunk
constexpr int kQRegion = kHG * 128;          // 8 KB per query chunk
constexpr int kSplitKeys = 256;              // decode split size (fixed)
constexpr int kMaxK = 4096;                  // largest top-k the index list holds
constexpr int kThreads = 288;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRangeLog2 = 60.f * kLog2e;  // CSA_DEV_RANGE threshold

constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + kRegions * kQRegion;   // 64 KB
constexpr int OFF_P = OFF_K + kRegions * kKRegion;   // +128 KB
constexpr int OFF_LIST = OFF_P + kBK * 128;          // +16 KB
constexpr int OFF_MB = OFF_LIST + kMaxK * 4;         // +16 KB
constexpr int OFF_INV = OFF_MB + 256;
constexpr int OFF_ROPE = OFF_INV + 256;
constexpr int OFF_BAR = OFF_ROPE + 256;
constexpr int kNumBars = 8 + 8 + 6;
constexpr int OFF_MISC = OFF_BAR + kNumBars * 8;
constexpr int SMEM_BYTES = OFF_MISC + 64;
constexpr int OFF_RED = OFF_K;                       // epilogue reuse of the key tile
constexpr int OFF_STAGE = OFF_K + 40960;

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

__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(TcAttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sQ = sm + OFF_Q;
  uint8_t* sK = sm + OFF_K;
  uint8_t* sP = sm + OFF_P;
  int32_t* list = reinterpret_cast<int32_t*>(sm + OFF_LIST);
  float* mb2 = reinterpret_cast<float*>(sm + OFF_MB);
  float* sinv = reinterpret_cast<float*>(sm + OFF_INV);
  float* rcs = reinterpret_cast<float*>(sm + OFF_ROPE);        // [32] cos
  float* rsn = rcs + 32;                                        // [32] sin
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint64_t* kfull = bars;
  uint64_t* kfree = bars + 8;
  uint64_t* qfull = bars + 16;
  uint64_t* sfull = bars + 17;
  uint64_t* pfull = bars + 18;
  uint64_t* pfree = bars + 19;
  uint64_t* ofull = bars + 20;
  uint64_t* drain = bars + 21;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
  int* n_ent_slot = reinterpret_cast<int*>(sm + OFF_MISC + 4);
  int* wcnt = reinterpret_cast<int*>(sm + OFF_MISC + 8);        // [4]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_MISC + 24);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int64_t row;
  int split_id, hg;
  if (a.split) {
    split_id = blockIdx.x;
    row = blockIdx.y;
    hg = blockIdx.z;
  } else {
    split_id = 0;
    row = (int64_t)gridDim.x - 1 - blockIdx.x;   // late (heavier) rows first
    hg = blockIdx.y;
  }
  const int64_t bidx = row / a.Tq, t = row % a.Tq;
  const int64_t pos = a.q_pos ? a.q_pos[row] : t;
  const int64_t wp0 = a.win_pos0 ? a.win_pos0[bidx] : 0;
  int64_t jlo = pos - a.n_win + 1;
  if (jlo < wp0) jlo = wp0;
  int64_t jhi = pos;
  if (jhi > wp0 + a.Tw - 1) jhi = wp0 + a.Tw - 1;
  const int64_t n_w = jhi >= jlo ? jhi - jlo + 1 : 0;
  const bf16* ent = a.entries + bidx * a.N * kC;
  const bf16* win = a.win + bidx * a.Tw * kC;
  const float scale = a.scale > 0.f ? a.scale : rsqrtf((float)kC);

  if (threadIdx.x == 0) {
    for (int i = 0; i < 8; ++i) {
      mbar_init(&kfull[i], 128);
      mbar_init(&kfree[i], 1);
    }
    mbar_init(qfull, 128);
    mbar_init(sfull, 1);
    mbar_init(pfull, 128);
    mbar_init(pfree, 1);
    mbar_init(ofull, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 8) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }

  // producer group: RoPE table and the compacted list of selected entries
  if (warp >= 4 && warp < 8) {
    const int ptid = threadIdx.x - 128, pw = warp - 4;
    if (pw == 0 && lane < (a.r >> 1)) {
      float cs, sn;
      rope_cos_sin(pos, lane, a.r, a.base, &cs, &sn);
      rcs[lane] = cs;
      rsn[lane] = sn;
    }
    if (a.sparse) {
      const int32_t* ir = a.idx + row * (int64_t)a.k;
      int base = 0;
      for (int i0 = 0; i0 < a.k; i0 += 128) {
        const int i = i0 + ptid;
        const int32_t e = i < a.k ? ir[i] : -1;
        const bool ok = e >= 0 && e < a.N;
        if (i < a.k && !ok && e != -1) report(a.status, CSA_DEV_BAD_INDEX, (unsigned)i);
        const unsigned bal = __ballot_sync(0xffffffffu, ok);
        if (lane == 0) wcnt[pw] = __popc(bal);
        named_bar(2, 128);
        int off = base;
        for (int w = 0; w < pw; ++w) off += wcnt[w];
        if (ok) list[off + __popc(bal & ((1u << lane) - 1u))] = e;
        base += wcnt[0] + wcnt[1] + wcnt[2] + wcnt[3];
        named_bar(2, 128);
      }
      if (ptid == 0) *n_ent_slot = base;
    } else if (ptid == 0) {
      *n_ent_slot = (int)vis_count(pos, a.m_dense, a.N);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem;          // 64 columns: S^T
  const uint32_t tO = tmem + 64;     // 4 x 64 columns: O^T
  const int64_t n_ent = *n_ent_slot;
  const int64_t n_keys = n_ent + n_w;
  int64_t k_lo = 0, k_hi = n_keys;
  if (a.split) {
    k_lo = (int64_t)split_id * kSplitKeys;
    k_hi = k_lo + kSplitKeys < n_keys ? k_lo + kSplitKeys : n_keys;
  }
  const int n_blocks = k_hi > k_lo ? (int)((k_hi - k_lo + kBK - 1) / kBK) : 0;

  if (warp >= 4 && warp < 8) {
    // ================= query prologue, then the gather
    const int ptid = threadIdx.x - 128, pw = warp - 4;
    for (int i = 0; i < 16; ++i) {
      const int h = pw * 16 + i;
      const bf16* qr = a.q + (row * a.H + (int64_t)hg * kHG + h) * kC;
      float x[16];
      load_vec(qr + lane * 8, x);
      load_vec(qr + 256 + lane * 8, x + 8);
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < 16; ++e) ss += x[e] * x[e];
      ss = warp_sum(ss);
      const float inv = (a.flags & CSA_F_NO_NORM) ? 1.f : rsqrtf(ss / (float)kC + a.eps);
      uint32_t w[8];
      float nq = 0.f;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int e0 = half * 256 + lane * 8;
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          float x0 = x[half * 8 + e] * inv, x1 = x[half * 8 + e + 1] * inv;
          const int el = e0 + e;
          if (!(a.flags & CSA_F_NO_ROPE) && el >= kC - a.r) {
            const int pi = (el - (kC - a.r)) >> 1;
            const float cs = rcs[pi], sn = rsn[pi];
            const float y0 = x0 * cs - x1 * sn, y1 = x0 * sn + x1 * cs;
            x0 = y0;
            x1 = y1;
          }
          const uint32_t pk = pack_bf16x2(x0, x1);
          const float r0 = bf16_bits_to_float(pk & 0xffffu), r1 = bf16_bits_to_float(pk >> 16);
          nq += r0 * r0 + r1 * r1;
          w[half * 4 + e / 2] = pk;
        }
      }
      nq = warp_sum(nq);
      // element lane*8 (+256): chunk region lane/8 (+4), 16-byte chunk lane%8
      const int ch = lane & 7;
      uint8_t* d0 = sQ + (lane >> 3) * kQRegion + h * 128 + ((ch ^ (h & 7)) << 4);
      uint8_t* d1 = sQ + (4 + (lane >> 3)) * kQRegion + h * 128 + ((ch ^ (h & 7)) << 4);
      *reinterpret_cast<uint4*>(d0) = make_uint4(w[0], w[1], w[2], w[3]);
      *reinterpret_cast<uint4*>(d1) = make_uint4(w[4], w[5], w[6], w[7]);
      if (lane == 0) mb2[h] = scale * sqrtf(nq) * sqrtf((float)kC) * kLog2e;
    }
    fence_proxy_async_smem();
    mbar_arrive(qfull);

    // gather: thread ptid fetches key row ptid of every block
    const uint32_t kbase = smem_u32(sK);
    for (int blk = 0; blk < n_blocks && !*abort_flag; ++blk) {
      const int64_t i = k_lo + (int64_t)blk * kBK + ptid;
      const bf16* src = nullptr;
      if (i < k_hi) {
        if (i < n_ent) src = ent + (int64_t)(a.sparse ? list[i] : i) * kC;
        else src = win + ((jlo - wp0) + (i - n_ent)) * kC;
      }
      const uint32_t rowoff = (uint32_t)ptid * 128u;
      int next_arrive = 0;
      for (int reg = 0; reg < kRegions; ++reg) {
        if (blk > 0 && !mbar_try_wait(&kfree[reg], (uint32_t)(blk - 1) & 1u)) {
          // about to block: publish every region already copied
          cp_async_wait<0>();
          fence_proxy_async_smem();
          for (; next_arrive < reg; ++next_arrive) mbar_arrive(&kfull[next_arrive]);
          if (!mbar_wait(&kfree[reg], (uint32_t)(blk - 1) & 1u)) {
            *abort_flag = 1;
            report(a.status, CSA_DEV_TIMEOUT, 10u);
            break;
          }
        }
        const uint32_t dst = kbase + reg * kKRegion + rowoff;
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const void* s = src ? (const void*)(src + reg * 64 + g * 8) : (const void*)a.q;
          cp_async16(dst + (((uint32_t)g ^ (uint32_t)(ptid & 7)) << 4), s, src ? 16u : 0u);
        }
        cp_async_commit();
        if (reg - next_arrive >= 2) {   // keep at most three regions in flight
          cp_async_wait<2>();
          fence_proxy_async_smem();
          mbar_arrive(&kfull[next_arrive]);
          ++next_arrive;
        }
      }
      cp_async_wait<0>();
      fence_proxy_async_smem();
      for (; next_arrive < kRegions; ++next_arrive) mbar_arrive(&kfull[next_arrive]);
    }
    cp_async_wait<0>();
  } else if (warp == 8) {
    // ================= MMA issuer
    if (n_blocks > 0 && elect_one()) {
      constexpr uint32_t idS = idesc_bf16_f32(kBK, kHG, 0, 0);
      constexpr uint32_t idO = idesc_bf16_f32(128, kHG, 1, 1);
      const uint32_t qb = smem_u32(sQ), kb = smem_u32(sK), pb = smem_u32(sP);
      bool ok = mbar_wait(qfull, 0);
      for (int blk = 0; ok && blk < n_blocks; ++blk) {
        const uint32_t ph = (uint32_t)blk & 1u;
        for (int reg = 0; reg < kRegions; ++reg) {
          if (*abort_flag || !mbar_wait(&kfull[reg], ph)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kq = 0; kq < 4; ++kq) {
            const uint64_t ad = smem_desc(kb + reg * kKRegion + kq * 32, 16, 1024, 2);
            const uint64_t bd = smem_desc(qb + reg * kQRegion + kq * 32, 16, 1024, 2);
            mma_bf16_ss(tS, ad, bd, idS, (reg | kq) != 0 ? 1u : 0u);
          }
        }
        if (!ok) break;
        mma_commit(sfull);
        if (*abort_flag || !mbar_wait(pfull, ph)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int j = 0; j < 4; ++j) {
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t ad = smem_desc(kb + (2 * j) * kKRegion + kk * 2048, kKRegion, 1024, 2);
            const uint64_t bd = smem_desc(pb + kk * 2048, kKRegion, 1024, 2);
            mma_bf16_ss(tO + 64 * j, ad, bd, idO, (blk > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&kfree[2 * j]);
          mma_commit(&kfree[2 * j + 1]);
        }
        mma_commit(pfree);
      }
      if (!ok) {
        *abort_flag = 1;
        report(a.status, CSA_DEV_TIMEOUT, 11u);
      }
      mma_commit(ofull);
      mma_commit(drain);
      mbar_wait(drain, 0);
    }
  } else {
    // ================= softmax (warps 0-3): thread = key lane of S^T
    const int rw = warp * 32 + lane;
    const float c2 = scale * kLog2e;
    float psum[kHG];
#pragma unroll
    for (int h = 0; h < kHG; ++h) psum[h] = 0.f;
    float xmax = -INFINITY;
    bool ok = mbar_wait(qfull, 0);   // mb2[] is written by the prologue
    for (int blk = 0; ok && blk < n_blocks; ++blk) {
      const uint32_t ph = (uint32_t)blk & 1u;
      if (*abort_flag || !mbar_wait(sfull, ph)) { ok = false; break; }
      tc_fence_after();
      uint32_t s0[32], s1[32];
      const uint32_t ta = tmem_addr(tS, (uint32_t)(warp * 32), 0);
      tmem_ld32(ta, s0);
      tmem_ld32(ta + 32, s1);
      tmem_ld_wait();
      const bool valid = k_lo + (int64_t)blk * kBK + rw < k_hi;
      uint32_t pk[32];
#pragma unroll
      for (int h = 0; h < kHG; h += 2) {
        const float l0 = __uint_as_float(h < 32 ? s0[h] : s1[h - 32]);
        const float l1 = __uint_as_float(h < 32 ? s0[h + 1] : s1[h + 1 - 32]);
        float x0 = valid ? fmaf(l0, c2, -mb2[h]) : -INFINITY;
        float x1 = valid ? fmaf(l1, c2, -mb2[h + 1]) : -INFINITY;
        xmax = fmaxf(xmax, fmaxf(x0, x1));
        const float p0 = ex2(x0), p1 = ex2(x1);
        psum[h] += p0;
        psum[h + 1] += p1;
        pk[h >> 1] = pack_bf16x2(p0, p1);
      }
      if (!mbar_wait(pfree, ph ^ 1u)) { ok = false; break; }
      uint8_t* prow = sP + rw * 128;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        *reinterpret_cast<uint4*>(prow + ((j ^ (rw & 7)) << 4)) =
            make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(pfull);
    }
    if (!ok) {
      *abort_flag = 1;
      report(a.status, CSA_DEV_TIMEOUT, 12u);
    }
    if (xmax > kRangeLog2) report(a.status, CSA_DEV_RANGE, (unsigned)row);
    bool have_o = n_blocks > 0 && ok && mbar_wait(ofull, 0);
    tc_fence_after();

    // ---- epilogue: per-head denominators, then O^T -> output
    float* red = reinterpret_cast<float*>(sm + OFF_RED);   // [128][65]
#pragma unroll
    for (int h = 0; h < kHG; ++h) red[rw * 65 + h] = psum[h];
    named_bar(1, 128);
    const int64_t slot = (row * a.n_hg + hg);
    if (rw < kHG) {
      float tot = 0.f;
      for (int r = 0; r < 128; ++r) tot += red[r * 65 + rw];
      if (a.split) {
        a.d_part[(slot * a.n_splits + split_id) * kHG + rw] = tot;
        if (split_id == 0) a.mb_part[slot * kHG + rw] = mb2[rw];
      } else {
        float den = tot;
        if (a.sink) {
          const float z = a.sink[hg * kHG + rw];
          den += ex2(fmaf(z, kLog2e, -mb2[rw]));
        }
        sinv[rw] = den > 0.f ? 1.f / den : 0.f;
      }
    }
    named_bar(1, 128);
    bf16* stage = reinterpret_cast<bf16*>(sm + OFF_STAGE);   // [64][512]
    for (int j = 0; j < 4; ++j) {
      uint32_t o0[32], o1[32];
      if (have_o) {
        const uint32_t ta = tmem_addr(tO + 64 * j, (uint32_t)(warp * 32), 0);
        tmem_ld32(ta, o0);
        tmem_ld32(ta + 32, o1);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int h = 0; h < 32; ++h) { o0[h] = 0u; o1[h] = 0u; }
      }
      const int c = 128 * j + rw;
      if (a.split) {
        float* op = a.o_part + ((slot * a.n_splits + split_id) * kHG) * kC + c;
#pragma unroll
        for (int h = 0; h < kHG; ++h)
          op[(int64_t)h * kC] = __uint_as_float(h < 32 ? o0[h] : o1[h - 32]);
      } else {
        const bool rot = !(a.flags & CSA_F_NO_ROPE) && c >= kC - a.r;
        float cs = 1.f, sn = 0.f;
        if (rot) {
          const int pi = (c - (kC - a.r)) >> 1;
          cs = rcs[pi];
          sn = rsn[pi];
        }
#pragma unroll
        for (int h = 0; h < kHG; ++h) {
          float v = __uint_as_float(h < 32 ? o0[h] : o1[h - 32]) * sinv[h];
          const float partner = __shfl_xor_sync(0xffffffffu, v, 1);
          // rotate by -pos: (x0, x1) -> (x0 cs + x1 sn, -x0 sn + x1 cs)
          if (rot) v = (lane & 1) ? fmaf(v, cs, -partner * sn) : fmaf(v, cs, partner * sn);
          stage[h * kC + c] = __float2bfloat16_rn(v);
        }
      }
    }
    if (!a.split) {
      named_bar(1, 128);
      const uint4* s4 = reinterpret_cast<const uint4*>(stage);
      uint4* o4 = reinterpret_cast<uint4*>(a.out + (row * a.H + (int64_t)hg * kHG) * kC);
      for (int i = rw; i < kHG * kC / 8; i += 128) o4[i] = s4[i];
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

inline int n_splits_for(int64_t max_keys) {
  int64_t n = (max_keys + kSplitKeys - 1) / kSplitKeys;
  return n < 1 ? 1 : (int)n;
}

}  // namespace

bool attn_tc_supported(const AttnParams& p) {
  auto al = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
  if (p.f.c != kC || p.H % kHG != 0 || p.f.r > 64 || (p.f.r & 1)) return false;
  if (p.sparse && p.k > kMaxK) return false;
  if (p.B * p.Tq >= (1LL << 31)) return false;
  if (p.Tq == 1 && p.B > 65535) return false;
  return al(p.q) && al(p.out) && (p.N == 0 || al(p.entries)) && (p.Tw == 0 || al(p.win));
}

size_t attn_tc_scratch(int64_t B, int64_t Tq, int H, int c, int64_t max_keys) {
  if (Tq != 1 || c != kC || H % kHG != 0) return 0;
  const int64_t n_hg = H / kHG;
  const int64_t ns = n_splits_for(max_keys);
  const int64_t slots = B * Tq * n_hg;
  return (size_t)(slots * ns * (kHG * kC + kHG) + slots * kHG) * sizeof(float);
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
  if (a.split) {
    a.n_splits = n_splits_for(max_keys);
    const size_t need = attn_tc_scratch(p.B, p.Tq, p.H, kC, max_keys);
    if (p.scratch_bytes < need) return cudaErrorInvalidValue;
    const int64_t slots = rows * a.n_hg;
    a.o_part = static_cast<float*>(p.scratch);
    a.d_part = a.o_part + slots * a.n_splits * kHG * kC;
    a.mb_part = a.d_part + slots * a.n_splits * kHG;
  } else {
    a.n_splits = 1;
  }
  const int smem = SMEM_BYTES + 1024;
  cudaError_t e =
      cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  if (a.split) {
    dim3 grid((unsigned)a.n_splits, (unsigned)rows, (unsigned)a.n_hg);
    attn_tc_kernel<<<grid, kThreads, smem, stream>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    attn_combine_kernel<<<dim3((unsigned)rows, (unsigned)a.n_hg), 256, 0, stream>>>(a);
    *n_launch = 2;
  } else {
    dim3 grid((unsigned)rows, (unsigned)a.n_hg);
    attn_tc_kernel<<<grid, kThreads, smem, stream>>>(a);
    *n_launch = 1;
  }
  return cudaGetLastError();
}

}  // namespace csa
