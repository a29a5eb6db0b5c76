// Tensor-core (tcgen05 / TMEM / TMA) kernels for the bf16 workloads.
#pragma once

#include "internal.h"

namespace csa {

// Lightning indexer + fused top-k on tcgen05.
bool indexer_tc_supported(const IndexerParams& p);
size_t indexer_tc_scratch(int64_t B, int64_t Tq, int64_t N, int k);
cudaError_t launch_indexer_tc(const IndexerParams& p, cudaStream_t stream,
                              unsigned long long* n_launch);

// Shared-KV MQA (sparse and dense) on tcgen05.
bool attn_tc_supported(const AttnParams& p);
size_t attn_tc_scratch(int64_t B, int64_t Tq, int H, int c, int64_t max_keys);
cudaError_t launch_attn_tc(const AttnParams& p, cudaStream_t stream, unsigned long long* n_launch);

}  // namespace csa
