// General MLA decode kernel (CUDA cores, fp32 math) and the split-KV log-sum-exp combine.
//
// Attention in the absorbed form ("DeepSeek-V2 大模型论文原文 PDF" 2.2 and 2.3):
//   s_p = (q_lat . c_p + q_rope . k_p) * scale,  o_lat = sum_p softmax(s)_p c_p,
// over the paged latent cache (intelliparadigm.com 6.1), with the online (running max)
// softmax so the cache is read once.  This path handles every dtype and head count; it is
// the only path for the fp32 workload and the reference point for the tensor-core kernels.
//
// CTA = 8 warps, one (sequence b, KV chunk s, group of heads).  Query rows r = (j, h) of the
// group (at most 16) share every cache tile of 32 tokens staged in shared memory as fp32.
// Scores: warp w owns rows w and w + 8, lane = token; row max / sum by warp shuffles.
// PV: thread owns latent dims tid and tid + 256 for all rows.
#include "mla_internal.cuh"

namespace mla {

constexpr int DS_THREADS = 256;
constexpr int DS_TILE = 32;
constexpr int DS_MAX_ROWS = 16;
constexpr int DS_MAX_W = 576;
constexpr int DS_MAX_DC = 512;

int decode_simt_heads_per_cta(int n_heads, int s_q) {
  int hpc = DS_MAX_ROWS / s_q;
  if (hpc > n_heads) hpc = n_heads;
  while (n_heads % hpc) --hpc;
  return hpc;
}

template <typename TQ, int KIND>
__global__ void __launch_bounds__(DS_THREADS) decode_simt_kernel(DecodeArgs a, int hpc) {
  extern __shared__ float smem[];
  const int d_c = a.d_c, d_r = a.d_rope, W = d_c + d_r, H = a.n_heads;
  const int s_q = a.s_q;
  const int R = s_q * hpc;
  float* q_s = smem;                       // [R][W]
  float* kv_s = q_s + R * W;               // [DS_TILE][W + 1]
  float* p_s = kv_s + DS_TILE * (W + 1);   // [R][DS_TILE]
  float* alpha_s = p_s + R * DS_TILE;      // [R]
  float* fin_s = alpha_s + DS_MAX_ROWS;    // [R] 1/l,  [R] lse

  const int split = blockIdx.x, b = blockIdx.y, hg = blockIdx.z;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const CacheView& cv = a.cache;
  const int page = cv.page_size;
  int L = a.seq_lens[b];
  if (L < 0 || L > cv.max_pages * page) {  // keep every block-table read inside its row
    if (tid == 0 && split == 0 && hg == 0) record_error(a.err, ERR_POS, L);
    L = max(0, min(L, cv.max_pages * page));
  }
  const int n_pages = (L + page - 1) / page;
  const int pps = (n_pages + a.n_split - 1) / a.n_split;
  const int lo = min(L, split * pps * page);
  const int hi = min(L, (split + 1) * pps * page);

  // Stage the group's query rows as fp32.
  for (int idx = tid; idx < R * W; idx += DS_THREADS) {
    int r = idx / W, k = idx % W;
    int j = r / hpc, h = hg * hpc + r % hpc;
    q_s[idx] = to_f32(reinterpret_cast<const TQ*>(a.q)[((long)(b * s_q + j) * H + h) * W + k]);
  }

  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  float o[DS_MAX_ROWS][2];
#pragma unroll
  for (int r = 0; r < DS_MAX_ROWS; ++r) o[r][0] = o[r][1] = 0.f;

  for (int t0 = lo; t0 < hi; t0 += DS_TILE) {
    __syncthreads();  // previous tile fully consumed (and q_s staged on the first pass)
    // Stage 32 cache rows as fp32; 8 warps x 4 tokens, lanes stride the row.
    for (int tt = warp; tt < DS_TILE; tt += DS_THREADS / 32) {
      int p = t0 + tt;
      float* dst = kv_s + tt * (W + 1);
      long slot = -1;
      if (p < hi) {
        int pid = cv.block_table[(long)b * cv.max_pages + p / page];
        if (pid >= 0 && pid < cv.num_pages)
          slot = (long)pid * page + p % page;
        else if (lane == 0)
          record_error(a.err, ERR_PAGE, pid);
      }
      if (slot < 0) {
        for (int k = lane; k < W; k += 32) dst[k] = 0.f;
        if (lane == 0) dst[W] = -1.f;  // marks "no token" for the score pass
        continue;
      }
      if (lane == 0) dst[W] = 0.f;
      if (KIND == MLA_FP8_E4M3) {
        const uint8_t* codes = reinterpret_cast<const uint8_t*>(cv.rows) + slot * d_c;
        const float* sc = cv.scales + slot * (d_c / 128);
        const __nv_bfloat16* kr = reinterpret_cast<const __nv_bfloat16*>(cv.rope) + slot * d_r;
        for (int k = lane; k < d_c; k += 32) dst[k] = e4m3_to_f32(codes[k]) * sc[k / 128];
        for (int k = lane; k < d_r; k += 32) dst[d_c + k] = __bfloat162float(kr[k]);
      } else if (KIND == MLA_BF16) {
        const __nv_bfloat16* row = reinterpret_cast<const __nv_bfloat16*>(cv.rows) + slot * W;
        for (int k = lane; k < W; k += 32) dst[k] = __bfloat162float(row[k]);
      } else {
        const float* row = reinterpret_cast<const float*>(cv.rows) + slot * W;
        for (int k = lane; k < W; k += 32) dst[k] = row[k];
      }
    }
    __syncthreads();
    // Scores and the online-softmax update: warp w owns rows w and w + 8.
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int r = warp + 8 * rr;
      if (r < R) {
        const int j = r / hpc;
        const int p = t0 + lane;
        const float* kv = kv_s + lane * (W + 1);
        bool valid = p < hi && kv[W] == 0.f;
        if (a.causal && p > L - s_q + j) valid = false;
        float s = -INFINITY;
        if (valid) {
          const float* q = q_s + r * W;
          float acc = 0.f;
          for (int k = 0; k < W; ++k) acc = fmaf(q[k], kv[k], acc);
          s = acc * a.scale;
        }
        float m_tile = warp_max(s);
        float m_new = fmaxf(m_run[rr], m_tile);
        float alpha, pr;
        if (m_new == -INFINITY) {
          alpha = 1.f;
          pr = 0.f;
        } else {
          alpha = expf(m_run[rr] - m_new);
          pr = expf(s - m_new);
        }
        l_run[rr] = l_run[rr] * alpha + warp_sum(pr);
        m_run[rr] = m_new;
        p_s[r * DS_TILE + lane] = pr;
        if (lane == 0) alpha_s[r] = alpha;
      }
    }
    __syncthreads();
    // O update: thread owns latent dims tid and tid + 256.
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int d = tid + DS_THREADS * i;
      if (d < d_c) {
#pragma unroll
        for (int r = 0; r < DS_MAX_ROWS; ++r) {
          if (r < R) {
            float acc = o[r][i] * alpha_s[r];
            const float* pr = p_s + r * DS_TILE;
#pragma unroll 8
            for (int t = 0; t < DS_TILE; ++t) acc = fmaf(pr[t], kv_s[t * (W + 1) + d], acc);
            o[r][i] = acc;
          }
        }
      }
    }
  }
  __syncthreads();
  // Row statistics to shared memory for the epilogue.
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const int r = warp + 8 * rr;
    if (r < R && lane == 0) {
      bool empty = l_run[rr] == 0.f;
      fin_s[r] = empty ? 0.f : 1.f / l_run[rr];
      fin_s[DS_MAX_ROWS + r] = empty ? -INFINITY : m_run[rr] + logf(l_run[rr]);
    }
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < DS_MAX_ROWS; ++r) {
    if (r >= R) break;
    const int j = r / hpc, h = hg * hpc + r % hpc;
    const float inv_l = fin_s[r];
    const long qrow = (long)(b * s_q + j) * H + h;
    if (a.n_split == 1) {
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int d = tid + DS_THREADS * i;
        if (d < d_c) reinterpret_cast<TQ*>(a.o_lat)[qrow * d_c + d] = from_f32<TQ>(o[r][i] * inv_l);
      }
      if (tid == 0 && a.lse) a.lse[qrow] = fin_s[DS_MAX_ROWS + r];
    } else {
      const long prow = ((long)(b * a.n_split + split) * s_q + j) * H + h;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int d = tid + DS_THREADS * i;
        if (d < d_c) a.o_part[prow * d_c + d] = o[r][i] * inv_l;
      }
      if (tid == 0) a.lse_part[prow] = fin_s[DS_MAX_ROWS + r];
    }
  }
}

static size_t decode_simt_smem(int R, int W) {
  return sizeof(float) * ((size_t)R * W + (size_t)DS_TILE * (W + 1) + (size_t)R * DS_TILE +
                          3 * DS_MAX_ROWS);
}

template <typename TQ, int KIND>
static cudaError_t launch_simt_t(const DecodeArgs& a, int hpc, cudaStream_t st) {
  const int W = a.d_c + a.d_rope;
  const int R = a.s_q * hpc;
  size_t smem = decode_simt_smem(R, W);
  cudaError_t e = cudaFuncSetAttribute(decode_simt_kernel<TQ, KIND>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.n_split, a.batch, a.n_heads / hpc);
  decode_simt_kernel<TQ, KIND><<<grid, DS_THREADS, smem, st>>>(a, hpc);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_decode_simt(const DecodeArgs& a, cudaStream_t st) {
  if (a.d_c + a.d_rope > DS_MAX_W || a.d_c > DS_MAX_DC) return kUnsupported;
  const int hpc = decode_simt_heads_per_cta(a.n_heads, a.s_q);
  if (a.act == MLA_F32) {
    if (a.cache.kind != MLA_F32) return kUnsupported;
    return launch_simt_t<float, MLA_F32>(a, hpc, st);
  }
  if (a.cache.kind == MLA_BF16) return launch_simt_t<__nv_bfloat16, MLA_BF16>(a, hpc, st);
  if (a.cache.kind == MLA_FP8_E4M3) return launch_simt_t<__nv_bfloat16, MLA_FP8_E4M3>(a, hpc, st);
  return kUnsupported;
}

// ------------------------------------------------------------------ split-KV combine
// One warp per query row (b, j, h):  lse = log sum_i exp(lse_i),  o = sum_i exp(lse_i - lse) o_i.
// Empty chunks carry lse_i = -inf and o_i = 0; a row whose chunks are all empty gets o = 0,
// lse = -inf.
template <typename TQ>
__global__ void __launch_bounds__(256) combine_kernel(DecodeArgs a) {
  // the next grid (the output projection) may start streaming its weights meanwhile
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) / 32, lane = threadIdx.x % 32;
  const int H = a.n_heads, s_q = a.s_q, n = a.n_split, d_c = a.d_c;
  const long rows = (long)a.batch * s_q * H;
  if (warp >= rows) return;
  const int h = warp % H;
  const int j = (warp / H) % s_q;
  const int b = warp / (H * s_q);
  auto prow = [&](int i) { return ((long)(b * n + i) * s_q + j) * H + h; };
  float m = -INFINITY;
  for (int i = lane; i < n; i += 32) m = fmaxf(m, a.lse_part[prow(i)]);
  m = warp_max(m);
  TQ* out = reinterpret_cast<TQ*>(a.o_lat) + (long)warp * d_c;
  if (m == -INFINITY) {
    for (int d = lane; d < d_c; d += 32) out[d] = from_f32<TQ>(0.f);
    if (lane == 0 && a.lse) a.lse[warp] = -INFINITY;
    return;
  }
  float sum = 0.f;
  for (int i = lane; i < n; i += 32) sum += expf(a.lse_part[prow(i)] - m);
  sum = warp_sum(sum);
  const float inv = 1.f / sum;
  for (int d0 = lane * 4; d0 < d_c; d0 += 128) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i = 0; i < n; ++i) {
      float w = expf(a.lse_part[prow(i)] - m) * inv;
      if (w == 0.f) continue;
      float4 v = *reinterpret_cast<const float4*>(a.o_part + prow(i) * d_c + d0);
      acc.x = fmaf(w, v.x, acc.x);
      acc.y = fmaf(w, v.y, acc.y);
      acc.z = fmaf(w, v.z, acc.z);
      acc.w = fmaf(w, v.w, acc.w);
    }
    out[d0] = from_f32<TQ>(acc.x);
    out[d0 + 1] = from_f32<TQ>(acc.y);
    out[d0 + 2] = from_f32<TQ>(acc.z);
    out[d0 + 3] = from_f32<TQ>(acc.w);
  }
  if (lane == 0 && a.lse) a.lse[warp] = m + logf(sum);
}

cudaError_t launch_combine(const DecodeArgs& a, cudaStream_t st) {
  const long rows = (long)a.batch * a.s_q * a.n_heads;
  if (rows == 0) return cudaSuccess;
  const int blocks = (int)((rows * 32 + 255) / 256);
  if (a.act == MLA_F32)
    combine_kernel<float><<<blocks, 256, 0, st>>>(a);
  else
    combine_kernel<__nv_bfloat16><<<blocks, 256, 0, st>>>(a);
  note_launch();
  return cudaGetLastError();
}

}  // namespace mla
