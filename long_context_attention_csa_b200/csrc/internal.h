// Internal launcher interface between the C ABI (abi.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace csa {

// Launches `kernel` with programmatic stream serialization: its CTAs may be
// scheduled while the previous kernel in the stream drains (the kernel must
// call pdl_wait() before touching global memory).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// Offsets inside a caller workspace: the status word lives at byte 0; scratch
// starts at kWsScratch.
constexpr size_t kWsScratch = 256;

struct CompressParams {
  const void* kv_a;   // group a (CSA) or the single group (HCA)
  const void* kv_b;   // group b (CSA only)
  const void* z_a;
  const void* z_b;
  int z_cols;         // c or 1
  int64_t T;          // tokens per sequence
  int64_t n_entries;  // floor(T / m)
  int m;              // rate (m or m')
  int overlap;        // 1 = CSA two overlapping groups
  int G;              // slot groups per CTA (set by the launcher)
  Fmt f;
  int64_t pos0;
  void* entries;
  void* win;          // optional window-row output
  unsigned* status;   // device status word (timed-out copy waits)
};
cudaError_t launch_compress(int dtype, CompressParams p, int64_t B, cudaStream_t stream);

struct IndexerParams {
  int64_t B, Tq;
  int HI, dI;
  const void* q_I;       // [B, Tq, HI, dI]
  const float* w;        // [B, Tq, HI]
  const void* k_I;       // [B, N, dI]
  int64_t N;
  const int64_t* q_pos;  // [B, Tq] or null
  int m, k;
  int32_t* idx_out;      // [B, Tq, k]
  float* score_out;      // [B, Tq, k] or null
  unsigned* status;      // device status word
  void* scratch;         // workspace past the status word
  size_t scratch_bytes;
};
size_t indexer_portable_scratch(int64_t B, int64_t Tq, int64_t N, int k);
cudaError_t launch_indexer_portable(int dtype, const IndexerParams& p, cudaStream_t stream);

struct AttnParams {
  int64_t B, Tq;
  int H;
  Fmt f;
  const void* q;          // [B, Tq, H, c]
  const int64_t* q_pos;   // [B, Tq] or null
  const void* entries;    // [B, N, c]
  int64_t N;
  int sparse;             // 1: keys = idx entries; 0: all visible entries
  const int32_t* idx;     // [B, Tq, k] (sparse; may be null when k == 0)
  int k;
  int m_dense;            // dense visibility rate (dense only)
  const void* win;        // [B, Tw, c]
  int64_t Tw;
  const int64_t* win_pos0;  // [B] or null
  int n_win;
  const float* sink;      // [H] or null
  float scale;
  int mixed;              // entries are mixed BF16 / MX-FP8 records of rec_bytes
  int rec_bytes;
  void* out;              // [B, Tq, H, c]
  unsigned* status;
  void* scratch;
  size_t scratch_bytes;
};
cudaError_t launch_attn_portable(int dtype, const AttnParams& p, cudaStream_t stream);

constexpr int kStreamMaxPairs = 64;   // RoPE pairs the streaming append takes (r <= 128)
struct StreamParams {
  const void* kv_a;   // [B, c] this call's token of each sequence (group a / HCA's group)
  const void* kv_b;   // [B, c] group b (CSA only)
  const void* z_a;    // [B, z_cols]
  const void* z_b;
  int z_cols;
  int m;              // rate
  int overlap;        // 1 = CSA
  Fmt f;
  int64_t pos0;
  uint8_t* state;     // [B][stride] per-sequence tail buffers
  size_t stride;
  void* entries;      // [B, n_cap, c] entry cache
  int64_t n_cap;
  void* win;          // [B, c] window rows of this call's tokens, or null
  unsigned* status;
  double theta[kStreamMaxPairs];   // RoPE frequencies (set by the launcher)
};
size_t stream_state_bytes(int elem_bytes, int m, int overlap, int c, int z_cols);
cudaError_t launch_stream_append(int dtype, StreamParams p, int64_t B, cudaStream_t stream);

struct ProjParams {
  int64_t T;
  int H, c, g, dg, d;
  const void* o;        // [T, H, c]
  const void* w_group;  // [g, dg, (H/g) c]
  const void* w_out;    // [d, g dg]
  void* v;              // [T, g dg] intermediate
  void* y;              // [T, d]
  unsigned* status;
};
bool proj_supported(const ProjParams& p);
cudaError_t launch_proj(const ProjParams& p, cudaStream_t stream, unsigned long long* n_launch);

// Adds n to the library's launch counter (csa_launch_count).
void note_launches(unsigned long long n);

// Indexer entry points' shared steps: argument checks and kernel choice
// (bf16 -> tensor cores, shapes outside that kernel -> CSA_E_UNSUPPORTED;
// float32 -> CUDA cores), the scratch the chosen kernels need past the status
// word, and the launch (counted).
csa_status indexer_prepare(int32_t dtype, int64_t B, int64_t Tq, int32_t H_I, int32_t d_I,
                           const void* q_I, const float* w, const void* k_I, int64_t N,
                           const int64_t* q_pos, int32_t m, int32_t k, int32_t* idx_out,
                           float* score_out, IndexerParams* out, bool* tc);
size_t indexer_scratch(bool tc, const IndexerParams& p);
csa_status indexer_launch(int32_t dtype, bool tc, const IndexerParams& p, cudaStream_t stream);

}  // namespace csa
