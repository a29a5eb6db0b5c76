// Grouped output projection of the attention output on the 5th-generation
// tensor cores (tcgen05, accumulators in TMEM, operands staged by TMA).
//
// Method: page "DeepSeek-V4：迈向高效百万 Token 上下文智能", §3.3, CSA paragraph:
// c * n_h is large, so the heads' outputs are first projected group by group
// to an intermediate dim d_g, the g results concatenated and projected back to
// the model dim d.  Reading: the H heads split into g consecutive groups of
// H/g heads.  Two GEMMs, both y = x W^T with bf16 operands, float32
// accumulation and a bf16 result:
//   grouped:  v[:, j d_g : (j+1) d_g] = o[:, group j's (H/g) c columns] . W_j^T
//   output:   y = v . W_out^T
// One kernel serves both: C[:, z n_off + n] = A[:, z k_off + k] . B[z]^T.
//
// Design: persistent CTAs walk 128 x 256 output tiles (z, m-tile, n-tile),
// n fastest so the CTAs running at once share their A tiles through L2 and
// every group's weights stay L2-resident; K in 64-element (128-byte
// swizzled) blocks through a four-slot TMA ring; M = 128, N = 256, K = 16
// MMAs issued by one thread into one of two TMEM accumulators (2 x 256
// columns), so the epilogue of tile i overlaps the MMAs of tile i+1.
//   warp 0     TMA producer (A and B blocks of each K step)
//   warp 1     TMEM owner, single-thread MMA issuer
//   warps 2-5  epilogue: TMEM -> bf16 -> global, thread = output row
#include "common.cuh"
#include "sm100.cuh"
#include "internal.h"
#include "tma_host.h"

namespace csa {

namespace {

using namespace sm100;

constexpr int kGM = 128;                       // tile rows (MMA M)
constexpr int kGN = 256;                       // tile columns (MMA N)
constexpr int kGK = 64;                        // K per stage (one 128-byte swizzle row)
constexpr int kGStages = 4;
constexpr int kGA = kGM * kGK * 2;             // 16 KB
constexpr int kGB = kGN * kGK * 2;             // 32 KB
constexpr int kGStage = kGA + kGB;
constexpr int kGThreads = 192;
constexpr int kGOffBar = kGStages * kGStage;   // after the ring
constexpr int kGSmem = kGOffBar + 256;
static_assert(kGSmem + 1024 <= 232448, "shared memory budget");

struct GemmArgs {
  int64_t M;            // rows of A and C
  int N, K, Z;          // per-z output columns and contraction length; z count
  int a_koff;           // A column offset per z (K for the grouped GEMM, 0 otherwise)
  int c_noff;           // C column offset per z
  int64_t ldc;          // C row stride (elements)
  bf16* C;
  int64_t n_tiles;      // Z * m_tiles * n_tiles
  int m_tiles, n_tiles_n;
  unsigned* status;
};

__global__ void __launch_bounds__(kGThreads, 1)
    gemm_bf16_tc_kernel(const __grid_constant__ CUtensorMap map_a,
                        const __grid_constant__ CUtensorMap map_b, GemmArgs a) {
  constexpr uint32_t kCols = 2 * kGN;
  constexpr uint32_t kIdesc = idesc_bf16_f32(kGM, kGN, 0, 0);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kGOffBar);
  uint64_t* full = bars;                    // [stages] A and B blocks landed
  uint64_t* empty = bars + kGStages;        // [stages] blocks consumed by the MMAs
  uint64_t* tfull = bars + 2 * kGStages;    // [2] accumulator complete
  uint64_t* tempty = tfull + 2;             // [2] accumulator read by the epilogue
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kb_n = (a.K + kGK - 1) / kGK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&map_a);
    tma_prefetch_desc(&map_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto tile_of = [&](int64_t u, int& z, int64_t& m0, int& n0) {
    const int nt = (int)(u % a.n_tiles_n);
    const int64_t r = u / a.n_tiles_n;
    const int mt = (int)(r % a.m_tiles);
    z = (int)(r / a.m_tiles);
    m0 = (int64_t)mt * kGM;
    n0 = nt * kGN;
  };

  if (warp == 0) {
    // ---------------- TMA producer
    if (elect_one()) {
      uint32_t it = 0;
      int64_t issued = 0;
      for (int64_t u = blockIdx.x; u < a.n_tiles && !*abort_flag; u += gridDim.x) {
        int z, n0;
        int64_t m0;
        tile_of(u, z, m0, n0);
        for (int kb = 0; kb < kb_n; ++kb, ++it) {
          const int s = (int)(it % kGStages);
          const uint32_t ph = (it / kGStages) & 1u;
          if (*abort_flag || !mbar_wait(&empty[s], ph ^ 1u)) {
            *abort_flag = 1;
            report(a.status, CSA_DEV_TIMEOUT, 0x701u);
            break;
          }
          mbar_arrive_expect_tx(&full[s], kGStage);
          uint8_t* dst = sm + s * kGStage;
          tma_load_3d(dst, &map_a, &full[s], z * a.a_koff + kb * kGK, (int32_t)m0, 0);
          tma_load_3d(dst + kGA, &map_b, &full[s], kb * kGK, n0, z);
          issued = it + 1;
        }
      }
      // drain: every issued copy has landed before the CTA may exit
      for (int64_t i = issued - kGStages > 0 ? issued - kGStages : 0; i < issued; ++i)
        mbar_wait(&full[i % kGStages], (uint32_t)(i / kGStages) & 1u);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (elect_one()) {
      uint32_t it = 0;
      int n = 0;
      for (int64_t u = blockIdx.x; u < a.n_tiles; u += gridDim.x, ++n) {
        const int buf = n & 1;
        const uint32_t bph = (uint32_t)(n >> 1) & 1u;
        if (*abort_flag || !mbar_wait(&tempty[buf], bph ^ 1u)) {
          *abort_flag = 1;
          report(a.status, CSA_DEV_TIMEOUT, 0x702u);
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(buf * kGN);
        bool ok = true;
        for (int kb = 0; kb < kb_n; ++kb, ++it) {
          const int s = (int)(it % kGStages);
          const uint32_t ph = (it / kGStages) & 1u;
          if (*abort_flag || !mbar_wait(&full[s], ph)) {
            *abort_flag = 1;
            report(a.status, CSA_DEV_TIMEOUT, 0x703u);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(sm + s * kGStage);
#pragma unroll
          for (int kk = 0; kk < kGK / 16; ++kk) {
            const uint64_t ad = smem_desc(sa + kk * 32, 16, 1024, 2);
            const uint64_t bd = smem_desc(sa + kGA + kk * 32, 16, 1024, 2);
            mma_bf16_ss(d, ad, bd, kIdesc, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&empty[s]);
        }
        if (!ok) break;
        mma_commit(&tfull[buf]);
      }
      mma_commit(drain);
      mbar_wait(drain, 0);
    }
  } else {
    // ---------------- epilogue: thread <-> TMEM lane <-> output row
    const int quarter = warp & 3;
    int n = 0;
    for (int64_t u = blockIdx.x; u < a.n_tiles; u += gridDim.x, ++n) {
      int z, n0;
      int64_t m0;
      tile_of(u, z, m0, n0);
      const int buf = n & 1;
      const uint32_t bph = (uint32_t)(n >> 1) & 1u;
      // warp-uniform decision: the TMEM loads below are warp-collective
      const bool ok = __all_sync(0xffffffffu, !*abort_flag && mbar_wait(&tfull[buf], bph));
      if (!ok) {
        *abort_flag = 1;
        report(a.status, CSA_DEV_TIMEOUT, 0x704u);
        break;
      }
      tc_fence_after();
      const int64_t row = m0 + quarter * 32 + lane;
      bf16* crow = a.C + row * a.ldc + (int64_t)z * a.c_noff + n0;
      const uint32_t base = tmem_addr(tmem, (uint32_t)(quarter * 32), (uint32_t)(buf * kGN));
#pragma unroll 1
      for (int cc = 0; cc < kGN; cc += 32) {
        uint32_t r[32];
        tmem_ld32(base + cc, r);
        tmem_ld_wait();
        if (row < a.M && n0 + cc < a.N) {   // N is a multiple of 32
          uint4* dst = reinterpret_cast<uint4*>(crow + cc);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(
                pack_bf16x2(__uint_as_float(r[8 * q]), __uint_as_float(r[8 * q + 1])),
                pack_bf16x2(__uint_as_float(r[8 * q + 2]), __uint_as_float(r[8 * q + 3])),
                pack_bf16x2(__uint_as_float(r[8 * q + 4]), __uint_as_float(r[8 * q + 5])),
                pack_bf16x2(__uint_as_float(r[8 * q + 6]), __uint_as_float(r[8 * q + 7])));
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[buf]);
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
}

int sm_count_proj() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  return n;
}

// C[:, z c_noff + n] = A[:, z a_koff + k] . B[z]^T for z < Z, n < N, k < K.
// A: [M][lda] bf16 (its columns z a_koff .. + K), B: [Z][N][K], C: [M][ldc].
cudaError_t launch_gemm(const void* A, int64_t lda, const void* Bw, void* C, int64_t ldc,
                        int64_t M, int N, int K, int Z, int a_koff, int c_noff, unsigned* status,
                        cudaStream_t stream) {
  GemmArgs a{};
  a.M = M;
  a.N = N;
  a.K = K;
  a.Z = Z;
  a.a_koff = a_koff;
  a.c_noff = c_noff;
  a.ldc = ldc;
  a.C = static_cast<bf16*>(C);
  a.m_tiles = (int)((M + kGM - 1) / kGM);
  a.n_tiles_n = (N + kGN - 1) / kGN;
  a.n_tiles = (int64_t)Z * a.m_tiles * a.n_tiles_n;
  a.status = status;
  if (a.n_tiles == 0) return cudaSuccess;
  CUtensorMap ma, mb;
  if (!make_map_bf16_3d(&ma, A, (uint64_t)lda, (uint64_t)M, 1, kGK, kGM))
    return cudaErrorInvalidValue;
  if (!make_map_bf16_3d(&mb, Bw, (uint64_t)K, (uint64_t)N, (uint64_t)Z, kGK, kGN))
    return cudaErrorInvalidValue;
  const int smem = kGSmem + 1024;
  cudaError_t e = cudaFuncSetAttribute(gemm_bf16_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int64_t sms = sm_count_proj();
  const unsigned grid = (unsigned)(a.n_tiles < sms ? a.n_tiles : sms);
  gemm_bf16_tc_kernel<<<grid, kGThreads, smem, stream>>>(ma, mb, a);
  return cudaGetLastError();
}

}  // namespace

bool proj_supported(const ProjParams& p) {
  const int64_t kg = (int64_t)(p.H / p.g) * p.c;
  return p.H % p.g == 0 && kg % kGK == 0 && ((int64_t)p.g * p.dg) % kGK == 0 && p.dg % 32 == 0 &&
         p.d % 32 == 0 && p.T < (1LL << 31) && (int64_t)p.H * p.c < (1LL << 31) &&
         (int64_t)p.g * p.dg < (1LL << 31);
}

cudaError_t launch_proj(const ProjParams& p, cudaStream_t stream, unsigned long long* n_launch) {
  *n_launch = 0;
  if (p.T == 0) return cudaSuccess;
  const int kg = (p.H / p.g) * p.c;
  const int gd = p.g * p.dg;
  // grouped: v[:, j d_g + n] = sum_k o[:, j kg + k] W_j[n, k]
  cudaError_t e = launch_gemm(p.o, (int64_t)p.H * p.c, p.w_group, p.v, gd, p.T, p.dg, kg, p.g,
                              kg, p.dg, p.status, stream);
  if (e != cudaSuccess) return e;
  *n_launch = 1;
  // output: y = v W_out^T
  e = launch_gemm(p.v, gd, p.w_out, p.y, p.d, p.T, p.d, gd, 1, 0, 0, p.status, stream);
  if (e == cudaSuccess) *n_launch = 2;
  return e;
}

}  // namespace csa
