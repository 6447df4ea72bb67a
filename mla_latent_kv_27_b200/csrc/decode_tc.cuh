// Tensor-core decode (decode_tc.cu): dispatch predicates and launcher.
#pragma once
#include "mla_internal.cuh"

namespace mla {
// True when the tcgen05 decode handles these dims (128 heads, d_c 512, d_rope 64, 64-token
// pages, bf16 activations and a bf16 cache).
bool tc_decode_supported(const mla_dims& d, int cache_kind);
// KV chunks per sequence the library picks when the caller passes n_split = 0.
int tc_auto_split(int batch, int s_q, int max_pages);
cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t st);
}  // namespace mla
