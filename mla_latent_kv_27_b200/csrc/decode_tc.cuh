// Tensor-core decode (decode_tc.cu): dispatch predicates, work partition and launcher.
#pragma once
#include "mla_internal.cuh"

namespace mla {
// True when the tcgen05 decode handles these dims (up to 128 heads, d_c 512, d_rope 64,
// 64-token pages, bf16 activations, a bf16 or E4M3 cache).
bool tc_decode_supported(const mla_dims& d, int cache_kind);
// Equal page ranges the length-balanced partition cuts the concatenated rows into (used when
// the caller passes n_split = 0): one per SM pair of a 148-SM B200; each is one persistent
// cluster that walks its range.
constexpr int TC_PLAN_WORKERS = 74;
// Workspace of the length-balanced partition: (workers + rows) partial slots of H x (d_c + 1)
// fp32, then two int32 per row (its first and last slot).
size_t tc_plan_workspace_bytes(const mla_dims& d, int batch, int s_q);
cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t st);
}  // namespace mla
