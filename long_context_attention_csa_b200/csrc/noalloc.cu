// indexer_scores_topk_noalloc: the lightning indexer + top-k with its scratch
// memory in a fixed device array instead of a caller workspace.
//
// Who needs it: callers that cannot allocate device memory at the point of
// the call -- for example a plug-in running inside an inference engine that
// owns every byte of device memory through its own pool, or a latency-
// critical decode loop where a cudaMalloc (which may synchronise the device)
// is not acceptable.  They pass inputs and outputs only.
//
// The scratch is a file-scope __device__ array of kNoAllocScratchBytes,
// resident on every GPU that loads this library until the process exits.
// Host code cannot use the array's name as a device address, so the first
// call on each device looks the address up with cudaGetSymbolAddress (with
// that device current) and caches it; that first call should therefore come
// before any stream capture.  All calls share the array: calls whose
// executions overlap on the GPU (different streams without ordering) race on
// it.  The status word at its start is cleared by every call; device-side
// status from this variant is not reported to the caller.
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "tc.h"

namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)8 << 20;  // 8 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the array on the current device (set up once per device).
cudaError_t noalloc_base(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" csa_status indexer_scores_topk_noalloc(int32_t dtype, int64_t B, int64_t Tq,
                                                  int32_t H_I, int32_t d_I, const void* q_I,
                                                  const float* w, const void* k_I, int64_t N,
                                                  const int64_t* q_pos, int32_t m, int32_t k,
                                                  int32_t* idx_out, float* score_out,
                                                  void* stream) {
  using namespace csa;
  if (dtype != CSA_F32 && dtype != CSA_BF16) return CSA_E_ARG;
  if (B < 0 || Tq < 0 || N < 0 || H_I <= 0 || d_I <= 0 || m < 1 || k < 1) return CSA_E_ARG;
  if (B > 65535 || Tq > 0x7fffffffLL || N > 0x7fffffffLL) return CSA_E_UNSUPPORTED;
  if (H_I > 64 || d_I > 1024) return CSA_E_UNSUPPORTED;
  if (B == 0 || Tq == 0) return CSA_OK;
  if (!q_I || !w || !idx_out || (N > 0 && !k_I)) return CSA_E_ARG;

  IndexerParams p{};
  p.B = B;
  p.Tq = Tq;
  p.HI = H_I;
  p.dI = d_I;
  p.q_I = q_I;
  p.w = w;
  p.k_I = k_I;
  p.N = N;
  p.q_pos = q_pos;
  p.m = m;
  p.k = k;
  p.idx_out = idx_out;
  p.score_out = score_out;
  const bool tc = dtype == CSA_BF16 && indexer_tc_supported(p);
  const size_t need = tc ? indexer_tc_scratch(B, Tq, N, k) : indexer_portable_scratch(B, Tq, N, k);
  if (kWsScratch + need > kNoAllocScratchBytes) return CSA_E_WORKSPACE;  // beyond the fixed array

  void* base = nullptr;
  if (noalloc_base(&base) != cudaSuccess) return CSA_E_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(base, 0, kWsScratch, s) != cudaSuccess) return CSA_E_CUDA;
  p.status = static_cast<unsigned*>(base);
  p.scratch = static_cast<unsigned char*>(base) + kWsScratch;
  p.scratch_bytes = kNoAllocScratchBytes - kWsScratch;
  cudaError_t e;
  if (tc) {
    unsigned long long n = 0;
    e = launch_indexer_tc(p, s, &n);
  } else {
    e = launch_indexer_portable(dtype, p, s);
  }
  return e == cudaSuccess ? CSA_OK : CSA_E_CUDA;
}
