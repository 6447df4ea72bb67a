// Tensor-core decode (decode_tc.cu): dispatch predicates, work partition and launcher.
#pragma once
#include "mla_internal.cuh"

namespace mla {
// True when the tcgen05 decode handles these dims (up to 128 heads, d_c 512, d_rope 64,
// 64-token pages, bf16 activations, a bf16 or E4M3 cache).
bool tc_decode_supported(const mla_dims& d, int cache_kind);
// Equal page ranges the length-balanced partition cuts the concatenated rows into: one per SM
// pair of a 148-SM B200; each is one persistent cluster that walks its range.  The tensor-core
// path always schedules this way (a caller's n_split only matters on the general path).
constexpr int TC_PLAN_WORKERS = 74;
// Partial slots: the rows cut across ranges (at most workers - 1) write at most 2 workers - 2.
constexpr int TC_PLAN_SLOTS = 2 * TC_PLAN_WORKERS - 2;
// Workspace of the length-balanced partition: TC_PLAN_SLOTS partial slots of H x (d_c + 1)
// fp32, then two int32 per row (its first and last slot).
size_t tc_plan_workspace_bytes(const mla_dims& d, int batch, int s_q);
cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t st);
// The log-sum-exp merge of the rows either partition left cut across ranges (decode_tc.cu),
// launched programmatically after the decode kernel.
cudaError_t launch_plan_combine(const DecodeArgs& a, cudaStream_t st);

// Small-head decode (decode_sh.cu): at most 16 heads, d_c 512, d_rope 64, 64-token pages, bf16
// activations and cache.  Two persistent CTAs per SM of a 148-SM B200, on the same partition.
bool sh_decode_supported(const mla_dims& d, int cache_kind);
constexpr int SH_PLAN_WORKERS = 2 * 148;
constexpr int SH_PLAN_SLOTS = 2 * SH_PLAN_WORKERS - 2;
size_t sh_plan_workspace_bytes(const mla_dims& d, int batch, int s_q);
cudaError_t launch_decode_sh(const DecodeArgs& a, cudaStream_t st);
}  // namespace mla
