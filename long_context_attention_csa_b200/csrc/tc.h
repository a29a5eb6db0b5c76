// Tensor-core (tcgen05 / TMEM / TMA) kernels for the bf16 workloads.
#pragma once

#include "internal.h"

namespace csa {

// Lightning indexer + fused top-k on tcgen05.
bool indexer_tc_supported(const IndexerParams& p);
size_t indexer_tc_scratch(int64_t B, int64_t Tq, int64_t N, int k);
cudaError_t launch_indexer_tc(const IndexerParams& p, cudaStream_t stream,
                              unsigned long long* n_launch);

// The same with MX-FP8 operands (E4M3 codes, UE8M0 scale tiles; p.q_I and
// p.k_I hold the codes), on block-scaled tcgen05 MMAs.
size_t indexer_mx_scratch(int64_t B, int64_t Tq, int64_t N, int k);
// fmt 1: MX-FP8 (128-byte rows), fmt 2: MX-FP4 (64-byte packed rows).
cudaError_t launch_indexer_mx(const IndexerParams& p, int fmt, const void* q_sf,
                              const void* k_sf, cudaStream_t stream,
                              unsigned long long* n_launch);
// MX-FP8 / MX-FP4 quantization of [B][rows][128] rows into codes and scale tiles.
cudaError_t launch_mxfp8_quantize(int dtype, const void* x, void* codes, void* scales, int64_t B,
                                  int64_t rows, cudaStream_t stream);
cudaError_t launch_mxfp4_quantize(int dtype, const void* x, void* codes, void* scales, int64_t B,
                                  int64_t rows, cudaStream_t stream);

// Mixed BF16 / MX-FP8 entry records.
size_t mixed_record_bytes(int c, int r);
cudaError_t launch_mixed_store(int dtype, const void* x, void* rec, int64_t n, int c, int r,
                               cudaStream_t stream);

// Shared-KV MQA (sparse and dense) on tcgen05.
bool attn_tc_supported(const AttnParams& p);
size_t attn_tc_scratch(int64_t B, int64_t Tq, int H, int c, int64_t max_keys);
cudaError_t launch_attn_tc(const AttnParams& p, cudaStream_t stream, unsigned long long* n_launch);

}  // namespace csa
