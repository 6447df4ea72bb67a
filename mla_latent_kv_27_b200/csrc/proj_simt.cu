// General (CUDA-core, fp32 FMA) kernels for the projection steps and the RoPE table.
//
//   append:  c = W_DKV h, k = RoPE(W_KR h) -> paged cache   ("DeepSeek-V2 大模型论文原文 PDF" 2.1, 2.3)
//   absorb:  q_lat = W_UK^T q_nope, q_rope rotated          (same page, 2.2)
//   output:  out = W_UV o_lat                               (same page, 2.2)
//
// The fp32-FMA GEMMs are the general path (every dtype and shape, and the only one for fp32
// activations); bf16 shapes the tensor-core kernels of proj_tc.cu support go there, where the
// fused append and absorb kernels also do the RoPE and the finish.  The query RoPE and append
// finish kernels here serve every other case.
#include "mla_internal.cuh"
#include "proj_tc.cuh"

namespace mla {

// ------------------------------------------------------------------ RoPE table
__global__ void rope_table_kernel(int half, int max_pos, double theta, float* cos_out, float* sin_out) {
  int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= half * max_pos) return;
  int p = idx / half, i = idx % half;
  double inv_freq = pow(theta, -2.0 * (double)i / (double)(2 * half));
  double s, c;
  sincos((double)p * inv_freq, &s, &c);
  cos_out[idx] = (float)c;
  sin_out[idx] = (float)s;
}

cudaError_t launch_rope_table(int d_rope, int max_pos, float theta, float* cos_out, float* sin_out,
                              cudaStream_t st) {
  int half = d_rope / 2;
  long n = (long)half * max_pos;
  int blocks = (int)((n + 255) / 256);
  rope_table_kernel<<<blocks, 256, 0, st>>>(half, max_pos, (double)theta, cos_out, sin_out);
  note_launch();
  return cudaGetLastError();
}

// ------------------------------------------------------------------ batched fp32-FMA GEMM
// C[g][t][n] = sum_k A[g][t][k] * B[g](k, n).  A rows are k-contiguous; B(k, n) sits at
// B + k*b_k + n*b_n (either b_k == 1 or b_n == 1).  ATOMIC: fp32 atomicAdd into C (split-K);
// otherwise C gets the act dtype.  Tiles: 64 t x 64 n x 16 k, 256 threads, 4x4 per thread.
constexpr int GB_M = 64, GB_N = 64, GB_K = 16;

template <typename T, bool ATOMIC>
__global__ void __launch_bounds__(256) simt_gemm_kernel(
    const T* __restrict__ A, long a_g, long a_t, const T* __restrict__ B, long b_g, long b_k,
    long b_n, void* __restrict__ C, long c_g, long c_t, int M, int N, int K, int ksplit,
    int k_chunk) {
  __shared__ float As[GB_K][GB_M + 4];
  __shared__ float Bs[GB_K][GB_N + 4];
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const int n0 = blockIdx.x * GB_N, t0 = blockIdx.y * GB_M;
  const int g = blockIdx.z / ksplit, ks = blockIdx.z % ksplit;
  const int k_lo = ks * k_chunk, k_hi = min(K, k_lo + k_chunk);
  const T* Ag = A + g * a_g;
  const T* Bg = B + g * b_g;
  float acc[4][4] = {};
  for (int k0 = k_lo; k0 < k_hi; k0 += GB_K) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int e = tid + 256 * i;
      int t = e / GB_K, k = e % GB_K;
      float v = 0.f;
      if (t0 + t < M && k0 + k < k_hi) v = to_f32(Ag[(long)(t0 + t) * a_t + k0 + k]);
      As[k][t] = v;
    }
    if (b_k == 1) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        int e = tid + 256 * i;
        int n = e / GB_K, k = e % GB_K;
        float v = 0.f;
        if (n0 + n < N && k0 + k < k_hi) v = to_f32(Bg[(long)(k0 + k) + (long)(n0 + n) * b_n]);
        Bs[k][n] = v;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        int e = tid + 256 * i;
        int k = e / GB_N, n = e % GB_N;
        float v = 0.f;
        if (n0 + n < N && k0 + k < k_hi) v = to_f32(Bg[(long)(k0 + k) * b_k + (long)(n0 + n) * b_n]);
        Bs[k][n] = v;
      }
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < GB_K; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[k][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[k][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int t = t0 + ty + 16 * i;
    if (t >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int n = n0 + tx + 16 * j;
      if (n >= N) continue;
      long off = g * c_g + (long)t * c_t + n;
      if (ATOMIC)
        atomicAdd(reinterpret_cast<float*>(C) + off, acc[i][j]);
      else
        reinterpret_cast<T*>(C)[off] = from_f32<T>(acc[i][j]);
    }
  }
}

template <typename T, bool ATOMIC>
static cudaError_t gemm(const T* A, long a_g, long a_t, const T* B, long b_g, long b_k, long b_n,
                        void* C, long c_g, long c_t, int groups, int M, int N, int K, int ksplit,
                        cudaStream_t st) {
  if (M == 0 || N == 0 || groups == 0) return cudaSuccess;
  int k_chunk = ((K + ksplit - 1) / ksplit + GB_K - 1) / GB_K * GB_K;
  ksplit = (K + k_chunk - 1) / k_chunk;
  dim3 grid((N + GB_N - 1) / GB_N, (M + GB_M - 1) / GB_M, groups * ksplit);
  simt_gemm_kernel<T, ATOMIC><<<grid, 256, 0, st>>>(A, a_g, a_t, B, b_g, b_k, b_n, C, c_g, c_t, M,
                                                    N, K, ksplit, k_chunk);
  note_launch();
  return cudaGetLastError();
}

// ------------------------------------------------------------------ append: finish pass
// One CTA (128 threads) per token: RoPE on the k part, then store (f32/bf16 rows, or E4M3
// codes with one fp32 scale per 128-value block) into the token's page slot.
__device__ __forceinline__ bool locate_slot(const CacheView& cv, int seq, int p, int rope_rows,
                                            int* err, long* slot) {
  if (seq < 0) {
    record_error(err, ERR_SEQ, seq);
    return false;
  }
  if (p < 0 || p >= rope_rows || p / cv.page_size >= cv.max_pages) {
    record_error(err, ERR_POS, p);
    return false;
  }
  int pid = cv.block_table[(long)seq * cv.max_pages + p / cv.page_size];
  if (pid < 0 || pid >= cv.num_pages) {
    record_error(err, ERR_PAGE, pid);
    return false;
  }
  *slot = (long)pid * cv.page_size + p % cv.page_size;
  return true;
}

template <typename T>
__global__ void __launch_bounds__(128) append_finish_kernel(
    const float* __restrict__ acc, int d_c, int d_rope, const int32_t* __restrict__ seq_idx,
    const int32_t* __restrict__ pos, const float* __restrict__ rcos,
    const float* __restrict__ rsin, int rope_rows, CacheView cv, int num_seqs, int* err) {
  const int t = blockIdx.x;
  const int W = d_c + d_rope;
  const float* a = acc + (long)t * W;
  const int seq = seq_idx[t], p = pos[t];
  if (seq >= num_seqs) {
    if (threadIdx.x == 0) record_error(err, ERR_SEQ, seq);
    return;
  }
  long slot;
  if (!locate_slot(cv, seq, p, rope_rows, err, &slot)) return;
  const int half = d_rope / 2;
  const float* cs = rcos + (long)p * half;
  const float* sn = rsin + (long)p * half;
  if (cv.kind == MLA_FP8_E4M3) {
    uint8_t* codes = reinterpret_cast<uint8_t*>(cv.rows) + slot * d_c;
    float* scales = cv.scales + slot * (d_c / 128);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    for (int blk = warp; blk < d_c / 128; blk += 4) {
      float x[4], amax = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        x[i] = a[blk * 128 + lane + 32 * i];
        amax = fmaxf(amax, fabsf(x[i]));
      }
      amax = warp_max(amax);
      float s = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
      float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 1.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) codes[blk * 128 + lane + 32 * i] = f32_to_e4m3(__fmul_rn(x[i], inv));
      if (lane == 0) scales[blk] = s;
    }
    __nv_bfloat16* kr = reinterpret_cast<__nv_bfloat16*>(cv.rope) + slot * d_rope;
    for (int i = threadIdx.x; i < half; i += blockDim.x) {
      float x0 = a[d_c + 2 * i], x1 = a[d_c + 2 * i + 1];
      kr[2 * i] = __float2bfloat16_rn(x0 * cs[i] - x1 * sn[i]);
      kr[2 * i + 1] = __float2bfloat16_rn(x0 * sn[i] + x1 * cs[i]);
    }
  } else {
    T* row = reinterpret_cast<T*>(cv.rows) + slot * W;
    for (int i = threadIdx.x; i < d_c; i += blockDim.x) row[i] = from_f32<T>(a[i]);
    for (int i = threadIdx.x; i < half; i += blockDim.x) {
      float x0 = a[d_c + 2 * i], x1 = a[d_c + 2 * i + 1];
      row[d_c + 2 * i] = from_f32<T>(x0 * cs[i] - x1 * sn[i]);
      row[d_c + 2 * i + 1] = from_f32<T>(x0 * sn[i] + x1 * cs[i]);
    }
  }
}

static bool append_fused(const mla_dims& d) { return d.act_dtype == MLA_BF16 && tc_proj_supported(d); }

size_t append_workspace_bytes(const mla_dims& d, int n_tok) {
  if (append_fused(d)) return 0;  // one launch, partial sums reduced on chip
  return (size_t)n_tok * (d.d_c + d.d_rope) * sizeof(float);
}

template <typename T>
static cudaError_t append_impl(const mla_dims& d, const T* h, int n_tok, const int32_t* seq_idx,
                               const int32_t* pos, const T* w_dkv, const T* w_kr,
                               const float* rcos, const float* rsin, int rope_rows,
                               const CacheView& cv, int num_seqs, float* ws, int* err,
                               cudaStream_t st) {
  const int W = d.d_c + d.d_rope;
  if (sizeof(T) == 2 && append_fused(d))
    return launch_append_tc(d, h, n_tok, seq_idx, pos, w_dkv, w_kr, rcos, rsin, rope_rows, cv, err, st);
  cudaError_t e = cudaMemsetAsync(ws, 0, (size_t)n_tok * W * sizeof(float), st);
  if (e != cudaSuccess) return e;
  {
    int tiles = ((n_tok + GB_M - 1) / GB_M) * ((W + GB_N - 1) / GB_N);
    int ksplit = (2 * 148 + tiles - 1) / tiles;
    ksplit = max(1, min(ksplit, d.d_model / 64));
    e = gemm<T, true>(h, 0, d.d_model, w_dkv, 0, 1, d.d_model, ws, 0, W, 1, n_tok, d.d_c, d.d_model,
                      ksplit, st);
    if (e != cudaSuccess) return e;
    e = gemm<T, true>(h, 0, d.d_model, w_kr, 0, 1, d.d_model, ws + d.d_c, 0, W, 1, n_tok, d.d_rope,
                      d.d_model, ksplit, st);
  }
  if (e != cudaSuccess) return e;
  append_finish_kernel<T><<<n_tok, 128, 0, st>>>(ws, d.d_c, d.d_rope, seq_idx, pos, rcos, rsin,
                                                 rope_rows, cv, num_seqs, err);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_append(const mla_dims& d, const void* h, int n_tok, const int32_t* seq_idx,
                          const int32_t* pos, const void* w_dkv, const void* w_kr,
                          const float* rcos, const float* rsin, int rope_rows, const CacheView& cv,
                          float* ws, int* err, cudaStream_t st) {
  if (d.act_dtype == MLA_F32)
    return append_impl<float>(d, (const float*)h, n_tok, seq_idx, pos, (const float*)w_dkv,
                              (const float*)w_kr, rcos, rsin, rope_rows, cv, cv.num_seqs, ws,
                              err, st);
  return append_impl<__nv_bfloat16>(d, (const __nv_bfloat16*)h, n_tok, seq_idx, pos,
                                    (const __nv_bfloat16*)w_dkv, (const __nv_bfloat16*)w_kr, rcos,
                                    rsin, rope_rows, cv, cv.num_seqs, ws, err, st);
}

// ------------------------------------------------------------------ absorb
template <typename T>
__global__ void rope_query_kernel(const T* __restrict__ q_rope, const int32_t* __restrict__ q_pos,
                                  int H, int d_c, int d_rope, const float* __restrict__ rcos,
                                  const float* __restrict__ rsin, int rope_rows,
                                  T* __restrict__ q_packed, int* err) {
  const int t = blockIdx.x;
  const int half = d_rope / 2;
  const int p = q_pos[t];
  const bool ok = p >= 0 && p < rope_rows;
  if (!ok && threadIdx.x == 0 && blockIdx.y == 0) record_error(err, ERR_POS, p);
  const int W = d_c + d_rope;
  for (int idx = blockIdx.y * blockDim.x + threadIdx.x; idx < H * half; idx += gridDim.y * blockDim.x) {
    int h = idx / half, i = idx % half;
    const T* src = q_rope + ((long)t * H + h) * d_rope;
    T* dst = q_packed + ((long)t * H + h) * W + d_c;
    float x0 = to_f32(src[2 * i]), x1 = to_f32(src[2 * i + 1]);
    float c = ok ? rcos[(long)p * half + i] : 1.f, s = ok ? rsin[(long)p * half + i] : 0.f;
    dst[2 * i] = from_f32<T>(x0 * c - x1 * s);
    dst[2 * i + 1] = from_f32<T>(x0 * s + x1 * c);
  }
}

template <typename T>
static cudaError_t absorb_impl(const mla_dims& d, const T* q_nope, const T* q_rope,
                               const int32_t* q_pos, int n_tok, const T* w_uk, const float* rcos,
                               const float* rsin, int rope_rows, T* q_packed, int* err,
                               cudaStream_t st) {
  const int H = d.n_heads, W = d.d_c + d.d_rope;
  if (sizeof(T) == 2 && tc_absorb_fused_supported(d) && absorb_tc_aligned(q_rope, q_packed, rcos, rsin))
    return launch_absorb_tc(d, q_nope, q_rope, q_pos, n_tok, w_uk, rcos, rsin, rope_rows, q_packed, err, st);
  cudaError_t e;
  if (sizeof(T) == 2 && tc_proj_supported(d))
    e = launch_absorb_gemm_tc(d, q_nope, n_tok, w_uk, q_packed, err, st);
  else
    e = gemm<T, false>(q_nope, d.d_nope, (long)H * d.d_nope, w_uk, (long)d.d_nope * d.d_c, d.d_c, 1,
                       q_packed, W, (long)H * W, H, n_tok, d.d_c, d.d_nope, 1, st);
  if (e != cudaSuccess) return e;
  const int pairs = H * (d.d_rope / 2);
  const dim3 rgrid(n_tok, (pairs + 255) / 256);
  rope_query_kernel<T><<<rgrid, 256, 0, st>>>(q_rope, q_pos, H, d.d_c, d.d_rope, rcos, rsin,
                                              rope_rows, q_packed, err);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_absorb(const mla_dims& d, const void* q_nope, const void* q_rope,
                          const int32_t* q_pos, int n_tok, const void* w_uk, const float* rcos,
                          const float* rsin, int rope_rows, void* q_packed, int* err,
                          cudaStream_t st) {
  if (d.act_dtype == MLA_F32)
    return absorb_impl<float>(d, (const float*)q_nope, (const float*)q_rope, q_pos, n_tok,
                              (const float*)w_uk, rcos, rsin, rope_rows, (float*)q_packed, err, st);
  return absorb_impl<__nv_bfloat16>(d, (const __nv_bfloat16*)q_nope, (const __nv_bfloat16*)q_rope,
                                    q_pos, n_tok, (const __nv_bfloat16*)w_uk, rcos, rsin,
                                    rope_rows, (__nv_bfloat16*)q_packed, err, st);
}

// ------------------------------------------------------------------ output up-projection
cudaError_t launch_output_up(const mla_dims& d, const void* o_lat, int n_tok, const void* w_uv,
                             void* out, int* err, cudaStream_t st) {
  const int H = d.n_heads;
  if (d.act_dtype == MLA_BF16 && tc_proj_supported(d))
    return launch_output_gemm_tc(d, o_lat, n_tok, w_uv, out, err, st);
  if (d.act_dtype == MLA_F32)
    return gemm<float, false>((const float*)o_lat, d.d_c, (long)H * d.d_c, (const float*)w_uv,
                              (long)d.d_v * d.d_c, 1, d.d_c, out, d.d_v, (long)H * d.d_v, H, n_tok,
                              d.d_v, d.d_c, 1, st);
  return gemm<__nv_bfloat16, false>((const __nv_bfloat16*)o_lat, d.d_c, (long)H * d.d_c,
                                    (const __nv_bfloat16*)w_uv, (long)d.d_v * d.d_c, 1, d.d_c, out,
                                    d.d_v, (long)H * d.d_v, H, n_tok, d.d_v, d.d_c, 1, st);
}

}  // namespace mla
