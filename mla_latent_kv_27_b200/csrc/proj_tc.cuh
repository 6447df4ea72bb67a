// Tensor-core projection GEMMs (proj_tc.cu).
#pragma once
#include "mla_internal.cuh"

namespace mla {
// True when the bf16 tcgen05 projection kernels handle these dims.
bool tc_proj_supported(const mla_dims& d);
// The whole absorb step in one launch (one CTA per head and 64 tokens): q_packed[t, h] =
// (W_UK[h]^T q_nope[t, h] || RoPE(q_rope[t, h])), bf16.  Shapes: tc_absorb_fused_supported.
bool tc_absorb_fused_supported(const mla_dims& d);
bool absorb_tc_aligned(const void* q_rope, const void* q_packed, const float* rcos, const float* rsin);
cudaError_t launch_absorb_tc(const mla_dims& d, const void* q_nope, const void* q_rope, const int32_t* q_pos,
                             int n_tok, const void* w_uk, const float* rcos, const float* rsin, int rope_rows,
                             void* q_packed, int* err, cudaStream_t st);
// q_packed[t, h, 0:d_c] = W_UK[h]^T q_nope[t, h]  (bf16)
cudaError_t launch_absorb_gemm_tc(const mla_dims& d, const void* q_nope, int n_tok, const void* w_uk,
                                  void* q_packed, int* err, cudaStream_t st);
// out[t, h] = W_UV[h] o_lat[t, h]  (bf16)
cudaError_t launch_output_gemm_tc(const mla_dims& d, const void* o_lat, int n_tok, const void* w_uv, void* out,
                                  int* err, cudaStream_t st);
// The whole append in one launch: [c | k] = [W_DKV ; W_KR] h, split-K partials added in a
// fixed order through distributed shared memory, RoPE on k, rows rounded to bf16 or E4M3
// blocks, stored at each token's page slot.  No workspace.
cudaError_t launch_append_tc(const mla_dims& d, const void* h, int n_tok, const int32_t* seq_idx, const int32_t* pos,
                             const void* w_dkv, const void* w_kr, const float* rcos, const float* rsin,
                             int rope_rows, const CacheView& cv, int* err, cudaStream_t st);
}  // namespace mla
