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
// status from this variant is not reported to the caller, so after a device-
// side error (a bounded wait that ran out) the outputs are unspecified and
// nothing says so: callers who must detect that use indexer_scores_topk with a
// workspace and csa_check_status.
//
// Accepted sizes: 256 bytes of status word plus the scratch of the kernels
// the call takes must fit kNoAllocScratchBytes.  bf16 takes the tensor-core
// kernels (H_I = 64, d_I = 128), whose scratch is 8 B x B x Tq x k x chunks
// when the entries span more than one chunk (2048 entries for Tq >= 4, 4096
// for single-token rows) and nothing otherwise; float32 takes the CUDA-core
// kernels, whose scratch is the B x Tq x N float32 score matrix.
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
  // the same checks and kernel choice as indexer_scores_topk
  IndexerParams p{};
  bool tc = false;
  csa_status st = indexer_prepare(dtype, B, Tq, H_I, d_I, q_I, w, k_I, N, q_pos, m, k, idx_out,
                                  score_out, &p, &tc);
  if (st != CSA_OK || B == 0 || Tq == 0) return st;
  // accepted iff the status word plus the chosen kernels' scratch fit the array
  if (kWsScratch + indexer_scratch(tc, p) > kNoAllocScratchBytes) return CSA_E_WORKSPACE;

  void* base = nullptr;
  if (noalloc_base(&base) != cudaSuccess) return CSA_E_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(base, 0, kWsScratch, s) != cudaSuccess) return CSA_E_CUDA;
  p.status = static_cast<unsigned*>(base);
  p.scratch = static_cast<unsigned char*>(base) + kWsScratch;
  p.scratch_bytes = kNoAllocScratchBytes - kWsScratch;
  return indexer_launch(dtype, tc, p, s);
}
