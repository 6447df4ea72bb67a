// Internal declarations shared by the libmla translation units (not part of the ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/mla.h"

namespace mla {

// ------------------------------------------------------------------ device error word
// kind << 24 | (first bad value & 0xFFFFFF); the first error sticks until cleared.
// ERR_SMEM: a kernel found its dynamic shared memory misaligned for its layout and did nothing.
enum ErrKind : int { ERR_PAGE = 1, ERR_POS = 2, ERR_TIMEOUT = 3, ERR_SEQ = 4, ERR_SMEM = 5 };

__device__ __forceinline__ void record_error(int* err, int kind, int value) {
  if (err) atomicCAS(err, 0, (kind << 24) | (value & 0xFFFFFF));
}

// ------------------------------------------------------------------ element conversion
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float e4m3_to_f32(uint8_t code) {
  __nv_fp8_e4m3 v;
  v.__x = code;
  return float(v);
}
// Round to nearest even, saturating to +-448 (OCP E4M3).
__device__ __forceinline__ uint8_t f32_to_e4m3(float x) {
  return (uint8_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ------------------------------------------------------------------ launchers
// What a launcher returns, never a CUDA runtime code, when the arguments are valid but outside
// what its kernels take (a shape, an alignment, a tensor map the CUDA driver refuses): the ABI
// reports it as MLA_ERR_UNSUPPORTED.  Every CUDA runtime error becomes MLA_ERR_CUDA.
constexpr cudaError_t kUnsupported = static_cast<cudaError_t>(0x4d4c4101);

// Every kernel launch of the library is counted (mla_launch_count in the ABI).
void note_launch(int n = 1);

// Programmatic dependent launch for the projection kernels and the split combine: on unless
// the environment sets MLA_PDL=0 (read once).
bool pdl_enabled();

struct CacheView {
  void* rows;           // f32/bf16 rows [pages, page, d_c + d_rope] or fp8 codes [pages, page, d_c]
  float* scales;        // fp8: [pages, page, d_c / 128]
  void* rope;           // fp8: bf16 [pages, page, d_rope]
  const int32_t* block_table;
  int max_pages;
  int num_pages;
  int num_seqs;         // rows of block_table
  int page_size;
  int kind;             // mla_dtype of the cache
};

cudaError_t launch_rope_table(int d_rope, int max_pos, float theta, float* cos_out, float* sin_out,
                              cudaStream_t st);

cudaError_t launch_append(const mla_dims& d, const void* h, int n_tok, const int32_t* seq_idx,
                          const int32_t* pos, const void* w_dkv, const void* w_kr,
                          const float* rcos, const float* rsin, int rope_rows, const CacheView& cv,
                          float* ws, int* err, cudaStream_t st);
size_t append_workspace_bytes(const mla_dims& d, int n_tok);

cudaError_t launch_absorb(const mla_dims& d, const void* q_nope, const void* q_rope,
                          const int32_t* q_pos, int n_tok, const void* w_uk, const float* rcos,
                          const float* rsin, int rope_rows, void* q_packed, int* err,
                          cudaStream_t st);

cudaError_t launch_output_up(const mla_dims& d, const void* o_lat, int n_tok, const void* w_uv,
                             void* out, int* err, cudaStream_t st);

struct DecodeArgs {
  const void* q;            // [B*s_q, H, d_c + d_rope] act
  CacheView cache;
  const int32_t* seq_lens;
  int batch, s_q, causal, n_split;
  int n_heads, d_c, d_rope, act;  // act: mla_dtype of q / o_lat
  float scale;
  float* o_part;            // [B, n_split, s_q, H, d_c] fp32 (n_split > 1); tensor cores: [slots, H, d_c]
  float* lse_part;          // [B, n_split, s_q, H]; tensor cores: [slots, H]
  int plan;                 // 1: the tensor-core path's length-balanced segments
  int32_t* rowinfo;         // plan: [B * s_q][2] first / last slot of each row, -1 for an empty row
  void* o_lat;              // [B*s_q, H, d_c] act
  float* lse;               // [B*s_q, H] or null
  int* err;
};

cudaError_t launch_decode_simt(const DecodeArgs& a, cudaStream_t st);
cudaError_t launch_combine(const DecodeArgs& a, cudaStream_t st);
int decode_simt_heads_per_cta(int n_heads, int s_q);

}  // namespace mla
