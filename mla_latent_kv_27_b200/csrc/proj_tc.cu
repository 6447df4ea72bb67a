// Tensor-core (tcgen05 / TMEM) kernels for the projection steps, bf16 activations:
//
//   append:  [c | k] = [W_DKV ; W_KR] h           ("DeepSeek-V2 大模型论文原文 PDF" 2.1, 2.3)
//   absorb:  q_lat[t, h] = W_UK[h]^T q_nope[t, h]   (same page, 2.2)
//   output:  out[t, h]   = W_UV[h] o_lat[t, h]      (same page, 2.2)
//
// At decode sizes these are weight-bandwidth bound (a few dozen tokens against MBs of
// weights), so the weights are the M = 128 operand of the MMA and the tokens its N operand
// ("swap AB"): every weight byte is read once and the token tile stays resident.  One kernel
// covers all three: D[m, n] = sum_k A[m, k] B[n, k] per group (head), A = weights (K-major,
// or MN-major for W_UK whose rows run along K), B = activations (K-major), fp32 in TMEM.
// TMA stages K in chunks of 64 through a 4-deep ring; one thread issues the MMAs; four warps
// read TMEM (lane = weight row) and write D transposed (coalesced along m), either rounded
// to the output dtype or, for split-K, added into an fp32 workspace with atomics.
// The query RoPE and the append finish (RoPE, E4M3 block quantisation, page scatter) stay on
// the CUDA cores (proj_simt.cu).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "mla_internal.cuh"
#include "proj_tc.cuh"
#include "sm100_ptx.cuh"

namespace mla {
namespace ptc {

using namespace sm100;

constexpr int BK = 64;        // K per stage (one 128-byte swizzle row of bf16)
constexpr int NST = 4;        // stages
constexpr int NTHREADS = 192; // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int A_BYTES = 128 * BK * 2;  // 16384

enum : int { OUT_BF16 = 0, OUT_F32 = 1, OUT_ATOMIC_F32 = 2 };

struct Params {
  int m_total;        // valid rows of A per group
  int n_total;        // tokens
  int k_total;        // reduction length
  int k_chunks_per_split;
  int a_mn;           // A is MN-major (rows of the 2-D view run along K)
  long a_group_rows;  // K-major A: rows per group in the 2-D view; MN-major: K rows per group
  long a_group_cols;  // MN-major A: column offset per group (0 when the group is in the rows)
  long b_group_cols;  // column offset of group g in B's 2-D view
  void* out;
  long out_ld;        // elements between consecutive tokens
  long out_group;     // elements between consecutive groups
  int out_mode;
  int* err;
};

struct Bars {
  uint64_t full[NST], empty[NST], done;
  uint32_t tmem_base;
  int abort_flag;
};

template <int BN>
__global__ void __launch_bounds__(NTHREADS, 1)
    wgemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int B_BYTES = BN * BK * 2;
  constexpr int STAGE = A_BYTES + B_BYTES;
  Bars* bars = reinterpret_cast<Bars*>(smem + NST * STAGE);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int m_blocks = (p.m_total + 127) / 128;
  const int g = blockIdx.x / m_blocks;
  const int m0 = (blockIdx.x % m_blocks) * 128;
  const int n0 = blockIdx.y * BN;
  const int k_chunks = (p.k_total + BK - 1) / BK;
  const int kc0 = blockIdx.z * p.k_chunks_per_split;
  const int kc1 = min(k_chunks, kc0 + p.k_chunks_per_split);
  const int nk = max(0, kc1 - kc0);
  constexpr uint32_t TCOLS = BN < 32 ? 32 : BN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->done, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, TCOLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  bool ok = true;

  if (nk > 0) {
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------------------ TMA producer
      for (int i = 0; i < nk; ++i) {
        const int s = i % NST;
        if (i >= NST && !mbar_wait(&bars->empty[s], ((i / NST) - 1) & 1)) {
          record_error(p.err, ERR_TIMEOUT, 30);
          atomicExch(&bars->abort_flag, 1);
          break;
        }
        const int k = (kc0 + i) * BK;
        uint8_t* st = smem + s * STAGE;
        mbar_arrive_expect_tx(&bars->full[s], STAGE);
        if (p.a_mn) {
          // two boxes of [64 K rows x 64 m] for the 128 rows of this block
          const int y = (int)(g * p.a_group_rows) + k;
          tma_load_2d(st, &tm_a, (int)(g * p.a_group_cols) + m0, y, &bars->full[s]);
          tma_load_2d(st + A_BYTES / 2, &tm_a, (int)(g * p.a_group_cols) + m0 + 64, y, &bars->full[s]);
        } else {
          tma_load_2d(st, &tm_a, k, (int)(g * p.a_group_rows) + m0, &bars->full[s]);
        }
        tma_load_2d(st + A_BYTES, &tm_b, (int)(g * p.b_group_cols) + k, n0, &bars->full[s]);
      }
      for (int i = max(0, nk - NST); i < nk; ++i)
        if (!mbar_wait(&bars->full[i % NST], (i / NST) & 1)) break;
    } else if (warp == 1 && lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      const uint32_t idesc = idesc_bf16(128, BN, p.a_mn, 0);
      for (int i = 0; i < nk; ++i) {
        const int s = i % NST;
        if (!mbar_wait(&bars->full[s], (i / NST) & 1)) {
          record_error(p.err, ERR_TIMEOUT, 31);
          atomicExch(&bars->abort_flag, 1);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_base = smem_addr(smem + s * STAGE);
        const uint32_t b_base = a_base + A_BYTES;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t a = p.a_mn ? umma_desc(a_base + kk * 2048, A_BYTES / 2, 1024, UMMA_SW128)
                                    : umma_desc(a_base + kk * 32, 16, 1024, UMMA_SW128);
          const uint64_t b = umma_desc(b_base + kk * 32, 16, 1024, UMMA_SW128);
          mma_bf16(tmem, a, b, idesc, (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&bars->empty[s]);
      }
      mma_commit(&bars->done);
    } else if (warp >= 2) {
      // ------------------------------------------------------------ epilogue
      const int quarter = warp & 3;
      const int m = m0 + quarter * 32 + lane;
      const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->done, 0, 4000000000ull))) {
        record_error(p.err, ERR_TIMEOUT, 32);
        ok = false;
      }
      tc_fence_after();
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_off + c0, v);
        tmem_wait_ld();
        if (!ok || m >= p.m_total) continue;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int n = n0 + c0 + c;
          if (n >= p.n_total) continue;
          const long off = (long)n * p.out_ld + (long)g * p.out_group + m;
          const float x = __uint_as_float(v[c]);
          if (p.out_mode == OUT_BF16)
            reinterpret_cast<__nv_bfloat16*>(p.out)[off] = __float2bfloat16_rn(x);
          else if (p.out_mode == OUT_F32)
            reinterpret_cast<float*>(p.out)[off] = x;
          else
            atomicAdd(reinterpret_cast<float*>(p.out) + off, x);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TCOLS);
  }
}

}  // namespace ptc

// ------------------------------------------------------------------ host side

static PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D bf16 map: `cols` contiguous elements per row, `rows` rows of `ld` elements.
static bool map2d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t ld, uint32_t box_cols,
                  uint32_t box_rows) {
  auto enc = encoder();
  if (!enc) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15) || (ld * 2) % 16) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {
struct GemmSpec {
  const void* a; uint64_t a_cols, a_rows, a_ld; int a_mn; long a_group_rows, a_group_cols;
  const void* b; uint64_t b_cols, b_rows, b_ld; long b_group_cols;
  int groups, m_total, n_total, k_total, k_splits;
  void* out; long out_ld, out_group; int out_mode;
};
}  // namespace

template <int BN>
static cudaError_t launch_bn(const GemmSpec& g, int* err, cudaStream_t st) {
  CUtensorMap ma, mb;
  const bool ok_a = g.a_mn ? map2d(&ma, g.a, g.a_cols, g.a_rows, g.a_ld, 64, ptc::BK)
                           : map2d(&ma, g.a, g.a_cols, g.a_rows, g.a_ld, ptc::BK, 128);
  if (!ok_a || !map2d(&mb, g.b, g.b_cols, g.b_rows, g.b_ld, ptc::BK, BN)) return cudaErrorInvalidValue;
  ptc::Params p;
  p.m_total = g.m_total;
  p.n_total = g.n_total;
  p.k_total = g.k_total;
  const int k_chunks = (g.k_total + ptc::BK - 1) / ptc::BK;
  p.k_chunks_per_split = (k_chunks + g.k_splits - 1) / g.k_splits;
  const int splits = (k_chunks + p.k_chunks_per_split - 1) / p.k_chunks_per_split;
  p.a_mn = g.a_mn;
  p.a_group_rows = g.a_group_rows;
  p.a_group_cols = g.a_group_cols;
  p.b_group_cols = g.b_group_cols;
  p.out = g.out;
  p.out_ld = g.out_ld;
  p.out_group = g.out_group;
  p.out_mode = g.out_mode;
  p.err = err;
  constexpr int smem = ptc::NST * (ptc::A_BYTES + BN * ptc::BK * 2) + 256 + 1024;
  cudaError_t e = cudaFuncSetAttribute(ptc::wgemm_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)(g.groups * ((g.m_total + 127) / 128)), (unsigned)((g.n_total + BN - 1) / BN), (unsigned)splits);
  ptc::wgemm_kernel<BN><<<grid, ptc::NTHREADS, smem, st>>>(ma, mb, p);
  note_launch();
  return cudaGetLastError();
}

static cudaError_t launch_gemm(const GemmSpec& g, int* err, cudaStream_t st) {
  if (g.n_total <= 0 || g.m_total <= 0 || g.groups <= 0) return cudaSuccess;
  if (g.n_total <= 64) return launch_bn<64>(g, err, st);
  if (g.n_total <= 128) return launch_bn<128>(g, err, st);
  return launch_bn<256>(g, err, st);
}

bool tc_proj_supported(const mla_dims& d) {
  return d.act_dtype == MLA_BF16 && d.d_model % 64 == 0 && d.d_c % 128 == 0 && d.d_nope % 64 == 0 &&
         d.d_v % 128 == 0 && d.d_rope <= 128;
}

cudaError_t launch_absorb_gemm_tc(const mla_dims& d, const void* q_nope, int n_tok, const void* w_uk,
                                  void* q_packed, int* err, cudaStream_t st) {
  // A = W_UK viewed [H * d_nope rows (K), d_c cols (M)], MN-major; B = q_nope [T, H * d_nope].
  GemmSpec g{};
  g.a = w_uk; g.a_cols = d.d_c; g.a_rows = (uint64_t)d.n_heads * d.d_nope; g.a_ld = d.d_c; g.a_mn = 1;
  g.a_group_rows = d.d_nope; g.a_group_cols = 0;
  g.b = q_nope; g.b_cols = (uint64_t)d.n_heads * d.d_nope; g.b_rows = n_tok; g.b_ld = (uint64_t)d.n_heads * d.d_nope;
  g.b_group_cols = d.d_nope;
  g.groups = d.n_heads; g.m_total = d.d_c; g.n_total = n_tok; g.k_total = d.d_nope; g.k_splits = 1;
  g.out = q_packed; g.out_ld = (long)d.n_heads * (d.d_c + d.d_rope); g.out_group = d.d_c + d.d_rope;
  g.out_mode = ptc::OUT_BF16;
  return launch_gemm(g, err, st);
}

cudaError_t launch_output_gemm_tc(const mla_dims& d, const void* o_lat, int n_tok, const void* w_uv, void* out,
                                  int* err, cudaStream_t st) {
  // A = W_UV viewed [H * d_v rows (M), d_c cols (K)], K-major; B = o_lat [T, H * d_c].
  GemmSpec g{};
  g.a = w_uv; g.a_cols = d.d_c; g.a_rows = (uint64_t)d.n_heads * d.d_v; g.a_ld = d.d_c; g.a_mn = 0;
  g.a_group_rows = d.d_v; g.a_group_cols = 0;
  g.b = o_lat; g.b_cols = (uint64_t)d.n_heads * d.d_c; g.b_rows = n_tok; g.b_ld = (uint64_t)d.n_heads * d.d_c;
  g.b_group_cols = d.d_c;
  g.groups = d.n_heads; g.m_total = d.d_v; g.n_total = n_tok; g.k_total = d.d_c; g.k_splits = 1;
  g.out = out; g.out_ld = (long)d.n_heads * d.d_v; g.out_group = d.d_v;
  g.out_mode = ptc::OUT_BF16;
  return launch_gemm(g, err, st);
}

cudaError_t launch_append_gemm_tc(const mla_dims& d, const void* h, int n_tok, const void* w_dkv, const void* w_kr,
                                  float* ws, int* err, cudaStream_t st) {
  // ws[t, 0:d_c] += W_DKV h[t];  ws[t, d_c:] += W_KR h[t]  (fp32, zeroed by the caller)
  const int W = d.d_c + d.d_rope;
  const int k_chunks = d.d_model / ptc::BK;
  const int m_blocks = d.d_c / 128 + 1;
  const int n_tiles = (n_tok + 255) / 256;
  int splits = (2 * 148 + m_blocks * n_tiles - 1) / (m_blocks * n_tiles);
  splits = splits < 1 ? 1 : (splits > k_chunks ? k_chunks : splits);
  GemmSpec g{};
  g.a = w_dkv; g.a_cols = d.d_model; g.a_rows = d.d_c; g.a_ld = d.d_model; g.a_mn = 0;
  g.a_group_rows = 0; g.a_group_cols = 0;
  g.b = h; g.b_cols = d.d_model; g.b_rows = n_tok; g.b_ld = d.d_model; g.b_group_cols = 0;
  g.groups = 1; g.m_total = d.d_c; g.n_total = n_tok; g.k_total = d.d_model; g.k_splits = splits;
  g.out = ws; g.out_ld = W; g.out_group = 0; g.out_mode = ptc::OUT_ATOMIC_F32;
  cudaError_t e = launch_gemm(g, err, st);
  if (e != cudaSuccess) return e;
  g.a = w_kr; g.a_rows = d.d_rope; g.m_total = d.d_rope; g.out = ws + d.d_c;
  return launch_gemm(g, err, st);
}

}  // namespace mla
