// Tensor-core (tcgen05 / TMEM) kernels for the projection steps, bf16 activations:
//
//   append:  [c | k] = [W_DKV ; W_KR] h           ("DeepSeek-V2 大模型论文原文 PDF" 2.1, 2.3)
//   absorb:  q_lat[t, h] = W_UK[h]^T q_nope[t, h]   (same page, 2.2)
//   output:  out[t, h]   = W_UV[h] o_lat[t, h]      (same page, 2.2)
//
// At decode sizes these are weight-bandwidth bound (a few dozen tokens against MBs of
// weights), so the weights are the M = 128 operand of the MMA and the tokens its N operand
// ("swap AB"): every weight byte is read once and the token tile stays resident, fp32 in TMEM.
// Three kernels:
//   wgemm_kernel      D[m, n] = sum_k A[m, k] B[n, k] per group (head), A = weights (K-major, or
//                     MN-major for W_UK whose rows run along K), B = activations; a TMA ring of
//                     up to 8 stages, one MMA-issuing thread, four epilogue warps reading TMEM
//                     (lane = weight row) and writing the bf16 tile through a TMA store.  The
//                     output projection, and the absorb for shapes the fused kernel does not take.
//   append_tc_kernel  both cache projections, split-K over a cluster reduced through distributed
//                     shared memory, and the finish (RoPE, bf16 or E4M3 blocks, page scatter).
//   absorb_tc_kernel  W_UK absorption for one head with the query RoPE in the same launch.
// All three are launched with programmatic stream serialization: weights stream in before the
// wait on the preceding grid, everything else after it.  The general path (fp32, other shapes)
// is in proj_simt.cu.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "mla_internal.cuh"
#include "proj_tc.cuh"
#include "sm100_ptx.cuh"

namespace mla {
namespace ptc {

using namespace sm100;

constexpr int BK = 64;        // K per stage (one 128-byte swizzle row of bf16)
constexpr int A_BYTES = 128 * BK * 2;  // 16384
constexpr int WG_MAX_NST = 8;  // stages: as many as fit in 192 KB (8, 6, 4 for BN = 64, 128, 256)
template <int BN>
__host__ __device__ constexpr int wg_nst() {
  return (192 * 1024) / (A_BYTES + BN * 64 * 2) > WG_MAX_NST ? WG_MAX_NST : (192 * 1024) / (A_BYTES + BN * 64 * 2);
}
constexpr int NTHREADS = 192; // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue

enum : int { OUT_BF16 = 0, OUT_F32 = 1, OUT_ATOMIC_F32 = 2 };

// Named barrier 1 is the epilogue warps' (warps 2-5, 128 threads) in every kernel of this file.
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// Named barrier 1 over the four epilogue warps with an AND of `v` across them.
__device__ __forceinline__ bool epi_sync_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred pi, po;\n setp.ne.u32 pi, %1, 0;\n bar.red.and.pred po, 1, 128, pi;\n"
      " selp.u32 %0, 1, 0, po;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

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
  int tma_out;        // OUT_BF16 tile written by a TMA store (m_total % 128 == 0, aligned output)
  int* err;
};

struct Bars {
  uint64_t full[WG_MAX_NST], empty[WG_MAX_NST], done;
  uint32_t tmem_base;
  int abort_flag;
};

template <int BN>
__global__ void __launch_bounds__(NTHREADS, 1)
    wgemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                 const __grid_constant__ CUtensorMap tm_out, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int B_BYTES = BN * BK * 2;
  constexpr int STAGE = A_BYTES + B_BYTES;
  constexpr int NST = wg_nst<BN>();
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

  griddep_launch_dependents();
  if (nk > 0) {
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------------------ TMA producer
      auto load_a = [&](int i) {
        const int s = i % NST;
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
      };
      auto load_b = [&](int i) {
        tma_load_2d(smem + (i % NST) * STAGE + A_BYTES, &tm_b, (int)(g * p.b_group_cols) + (kc0 + i) * BK, n0,
                    &bars->full[i % NST]);
      };
      // The weights (A) are never written by an earlier grid of the stream: the first ring's
      // worth streams in while that grid finishes.  The activations (B) may be its output.
      const int first = min(nk, NST);
      for (int i = 0; i < first; ++i) load_a(i);
      griddep_wait();
      for (int i = 0; i < first; ++i) load_b(i);
      for (int i = first; i < nk; ++i) {
        const int s = i % NST;
        if (!mbar_wait(&bars->empty[s], ((i / NST) - 1) & 1)) {
          record_error(p.err, ERR_TIMEOUT, 30);
          atomicExch(&bars->abort_flag, 1);
          break;
        }
        load_a(i);
        load_b(i);
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
      griddep_wait();
      const int quarter = warp & 3;
      const int m = m0 + quarter * 32 + lane;
      const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
      if (p.tma_out) {
        // bf16 tile [BN tokens][128 rows] staged in the (now idle) stage ring, one TMA store
        if (!epi_sync_and(mbar_wait(&bars->done, 0, 4000000000ull))) {
          if (threadIdx.x == 64) record_error(p.err, ERR_TIMEOUT, 32);
        } else {
          tc_fence_after();
          __nv_bfloat16* stg = reinterpret_cast<__nv_bfloat16*>(smem);
          for (int c0 = 0; c0 < BN; c0 += 32) {
            uint32_t v[32];
            tmem_ld32(tmem + lane_off + c0, v);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c)
              stg[(c0 + c) * 128 + quarter * 32 + lane] = __float2bfloat16_rn(__uint_as_float(v[c]));
          }
          fence_proxy_async_smem();
          epi_sync();
          if (threadIdx.x == 64) {
            tma_store_2d(&tm_out, stg, (int)(g * p.out_group) + m0, n0);  // rows past n_total not written
            bulk_commit_group();
            bulk_wait_group<0>();
          }
        }
      } else {
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
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TCOLS);
  }
}


// ------------------------------------------------------------------ fused cache append
// [c | k_pre] = [W_DKV ; W_KR] h for a block of tokens, then the finish into the paged cache,
// in one launch.  Grid (S, m_tiles, n_tiles): m-tile mt < d_c / 128 covers 128 rows of W_DKV,
// the last m-tile the d_rope rows of W_KR (the rest of its 128-row A tile is zero).  The S
// CTAs of a cluster split K (d_model) into S ranges, each accumulating its partial tile in
// TMEM; every CTA then sends each token's 128 partial sums to the CTA that owns the token
// (CTA r owns tokens [r * BN / S, (r + 1) * BN / S) of the tile) through distributed shared
// memory, and the owner adds the S partials in rank order, so the result does not depend on
// timing.  The owner finishes its tokens ("DeepSeek-V2 大模型论文原文 PDF" 2.1 and 2.3 for
// what is cached): latent rows rounded to bf16, or E4M3 codes with one fp32 scale (amax / 448)
// per 128-value block - one m-tile is exactly one block -, and k_rope rotated by RoPE at the
// token's position, all stored at the token's page slot.
constexpr int AP_THREADS = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 reduction + finish
constexpr int AP_MAX_ST = 6;

struct ApBars {
  uint64_t full[AP_MAX_ST], empty[AP_MAX_ST], done;
  uint32_t tmem_base;
};

template <int BN>
struct ApCfg {
  static constexpr int NST = BN == 64 ? 6 : 4;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int RECV_OFF = NST * STAGE;                 // [S][128][BN / S] fp32 (split K only)
  static constexpr int RECV_BYTES = BN == 64 ? 128 * 64 * 4 : 0;
  static constexpr int SLOT_OFF = RECV_OFF + RECV_BYTES;      // int64 [BN]
  static constexpr int BAR_OFF = SLOT_OFF + BN * 8;
  static constexpr int SMEM = BAR_OFF + 256 + 1024;
  static_assert(BN * 128 * 4 <= NST * STAGE, "the finished tile aliases the stage ring");
  static_assert(NST <= AP_MAX_ST && sizeof(ApBars) <= 256, "barrier block");
};

struct ApParams {
  int T, d_model, d_c, d_rope, m_tiles_c, kps;
  const int32_t* seq_idx;
  const int32_t* pos;
  const float* rcos;
  const float* rsin;
  int rope_rows;
  CacheView cv;
  int* err;
};

__device__ __forceinline__ void st_cluster_v4(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

template <int BN>
__global__ void __launch_bounds__(AP_THREADS, 1)
    append_tc_kernel(const __grid_constant__ CUtensorMap tm_wc, const __grid_constant__ CUtensorMap tm_wr,
                     const __grid_constant__ CUtensorMap tm_h, const ApParams p) {
  using C = ApCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  ApBars* bars = reinterpret_cast<ApBars*>(smem + C::BAR_OFF);
  float* recv = reinterpret_cast<float*>(smem + C::RECV_OFF);
  float* fin = reinterpret_cast<float*>(smem);  // [tokens][128], after the K loop
  long long* slots = reinterpret_cast<long long*>(smem + C::SLOT_OFF);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int S = gridDim.x, rank = blockIdx.x;
  const int mt = blockIdx.y;
  const bool rope_tile = mt == p.m_tiles_c;
  const int n0 = blockIdx.z * BN;
  const int k_chunks = p.d_model / BK;
  const int kc0 = rank * p.kps;
  const int nk = max(0, min(k_chunks, kc0 + p.kps) - kc0);
  const int own = BN / S;          // tokens of the tile this CTA finishes
  const int t_own = n0 + rank * own;
  const uint32_t a_tx = rope_tile ? (uint32_t)p.d_rope * 128u : (uint32_t)A_BYTES;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->done, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, BN);
    tmem_relinquish();
  }
  if (rope_tile) {
    // rows d_rope .. 127 of the A tile stay zero in every stage (TMA writes only d_rope rows)
    for (int s = 0; s < C::NST; ++s)
      for (int i = p.d_rope * 32 + threadIdx.x; i < A_BYTES / 4; i += AP_THREADS)
        reinterpret_cast<uint32_t*>(smem + s * C::STAGE)[i] = 0u;
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (S > 1) cluster_arrive();  // peers may write into this CTA's receive buffer after this
  griddep_launch_dependents();
  const uint32_t tmem = bars->tmem_base;
  bool ok = true;

  if (warp == 0) {
    if (lane == 0) {
      auto load_w = [&](int i) {
        const int s = i % C::NST;
        const int k = (kc0 + i) * BK;
        uint8_t* st = smem + s * C::STAGE;
        mbar_arrive_expect_tx(&bars->full[s], a_tx + C::B_BYTES);
        if (rope_tile)
          tma_load_2d(st, &tm_wr, k, 0, &bars->full[s]);
        else
          tma_load_2d(st, &tm_wc, k, mt * 128, &bars->full[s]);
      };
      auto load_h = [&](int i) {
        tma_load_2d(smem + (i % C::NST) * C::STAGE + A_BYTES, &tm_h, (kc0 + i) * BK, n0, &bars->full[i % C::NST]);
      };
      // weights first (no earlier grid of the stream writes them), h once that grid is done
      const int first = min(nk, C::NST);
      for (int i = 0; i < first; ++i) load_w(i);
      griddep_wait();
      for (int i = 0; i < first; ++i) load_h(i);
      int issued = first;
      for (int i = first; i < nk; ++i) {
        const int s = i % C::NST;
        if (!mbar_wait(&bars->empty[s], ((i / C::NST) - 1) & 1)) {
          record_error(p.err, ERR_TIMEOUT, 40);
          break;
        }
        load_w(i);
        load_h(i);
        issued = i + 1;
      }
      // no load of this CTA may still be in flight when it exits (bounded wait)
      for (int i = max(0, issued - C::NST); i < issued; ++i)
        if (!mbar_wait(&bars->full[i % C::NST], (i / C::NST) & 1)) break;
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, BN, 0, 0);
      for (int i = 0; i < nk; ++i) {
        const int s = i % C::NST;
        if (!mbar_wait(&bars->full[s], (i / C::NST) & 1)) {
          record_error(p.err, ERR_TIMEOUT, 41);
          break;
        }
        tc_fence_after();
        const uint32_t a_base = smem_addr(smem + s * C::STAGE);
        const uint32_t b_base = a_base + A_BYTES;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          mma_bf16(tmem, umma_desc(a_base + kk * 32, 16, 1024, UMMA_SW128),
                   umma_desc(b_base + kk * 32, 16, 1024, UMMA_SW128), idesc, (i > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars->empty[s]);
      }
      if (nk > 0)
        mma_commit(&bars->done);
      else
        mbar_arrive(&bars->done);  // empty K range: nothing to wait for, the partial is zero
    }
    __syncwarp();
  } else {
    // the cache may still be read by an earlier grid of the stream until it completes
    griddep_wait();
    // page slots of the tokens this CTA finishes (errors reported by the first m-tile only)
    const int e = threadIdx.x - 64;
    for (int i = e; i < own; i += 128) {
      const int t = t_own + i;
      long long slot = -1;
      if (t < p.T) {
        const int seq = p.seq_idx[t], ps = p.pos[t];
        const bool report = mt == 0;
        if (seq < 0 || seq >= p.cv.num_seqs) {
          if (report) record_error(p.err, ERR_SEQ, seq);
        } else if (ps < 0 || ps >= p.rope_rows || ps / p.cv.page_size >= p.cv.max_pages) {
          if (report) record_error(p.err, ERR_POS, ps);
        } else {
          const int pid = p.cv.block_table[(long)seq * p.cv.max_pages + ps / p.cv.page_size];
          if (pid < 0 || pid >= p.cv.num_pages) {
            if (report) record_error(p.err, ERR_PAGE, pid);
          } else {
            slot = (long long)pid * p.cv.page_size + ps % p.cv.page_size;
          }
        }
      }
      slots[i] = slot;
    }
    if (!__all_sync(0xffffffffu, mbar_wait(&bars->done, 0, 4000000000ull))) {
      record_error(p.err, ERR_TIMEOUT, 42);
      ok = false;
    }
    tc_fence_after();
  }
  // every thread reaches both cluster barriers, whatever happened above
  if (S > 1) cluster_wait();

  const int quarter = warp & 3;
  const int m = quarter * 32 + lane;  // TMEM lane = weight row of the tile
  if (warp >= 2) {
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    for (int c0 = 0; c0 < BN; c0 += 32) {
      uint32_t v[32];
      tmem_ld32(tmem + lane_off + c0, v);
      tmem_wait_ld();
      if (nk == 0 || !ok) {
#pragma unroll
        for (int c = 0; c < 32; ++c) v[c] = 0u;
      }
      if (S == 1) {
#pragma unroll
        for (int c = 0; c < 32; ++c) fin[(c0 + c) * 128 + m] = __uint_as_float(v[c]);
      } else {
        // tokens c0 .. c0 + 31 of the tile go to their owners, 4 at a time
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          const int t = c0 + c;
          const int r = t / own, j = t % own;
          const uint32_t dst = map_to_rank(recv, r) + (uint32_t)(((rank * 128 + m) * own + j) * 4);
          st_cluster_v4(dst, __uint_as_float(v[c]), __uint_as_float(v[c + 1]), __uint_as_float(v[c + 2]),
                        __uint_as_float(v[c + 3]));
        }
      }
    }
  }
  if (S > 1) {
    cluster_arrive();
    cluster_wait();
    if (warp >= 2) {
      // sum the S partials of each owned token in rank order
      for (int j = 0; j < own; j += 4) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int r = 0; r < S; ++r) {
          const float4 x = *reinterpret_cast<const float4*>(recv + (r * 128 + m) * own + j);
          acc.x += x.x;
          acc.y += x.y;
          acc.z += x.z;
          acc.w += x.w;
        }
        fin[j * 128 + m] = acc.x;
        fin[(j + 1) * 128 + m] = acc.y;
        fin[(j + 2) * 128 + m] = acc.z;
        fin[(j + 3) * 128 + m] = acc.w;
      }
    }
  }
  if (warp >= 2) {
    epi_sync();
    // finish: one warp per token row; lane l holds features 4l .. 4l + 3 of this m-tile
    const int W = p.d_c + p.d_rope;
    for (int j = warp - 2; j < own; j += 4) {
      const long long slot = slots[j];
      if (slot < 0 || !ok) continue;
      const float4 x = reinterpret_cast<const float4*>(fin + j * 128)[lane];
      const int f = 4 * lane;
      if (!rope_tile) {
        const int col = mt * 128 + f;
        if (p.cv.kind == MLA_FP8_E4M3) {
          const float amax = warp_max(fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(x.z), fabsf(x.w))));
          const float sc = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
          const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 1.f;
          const uint32_t q = (uint32_t)f32_to_e4m3(__fmul_rn(x.x, inv)) |
                             ((uint32_t)f32_to_e4m3(__fmul_rn(x.y, inv)) << 8) |
                             ((uint32_t)f32_to_e4m3(__fmul_rn(x.z, inv)) << 16) |
                             ((uint32_t)f32_to_e4m3(__fmul_rn(x.w, inv)) << 24);
          *reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(p.cv.rows) + slot * p.d_c + col) = q;
          if (lane == 0) p.cv.scales[slot * (p.d_c / 128) + mt] = sc;
        } else {
          __nv_bfloat16* row = reinterpret_cast<__nv_bfloat16*>(p.cv.rows) + slot * W + col;
          *reinterpret_cast<__nv_bfloat162*>(row) = __floats2bfloat162_rn(x.x, x.y);
          *reinterpret_cast<__nv_bfloat162*>(row + 2) = __floats2bfloat162_rn(x.z, x.w);
        }
      } else if (f < p.d_rope) {
        const int half = p.d_rope / 2;
        const int ps = p.pos[t_own + j];
        const float* cs = p.rcos + (long)ps * half;
        const float* sn = p.rsin + (long)ps * half;
        __nv_bfloat16* dst = p.cv.kind == MLA_FP8_E4M3
                                 ? reinterpret_cast<__nv_bfloat16*>(p.cv.rope) + slot * p.d_rope
                                 : reinterpret_cast<__nv_bfloat16*>(p.cv.rows) + slot * W + p.d_c;
        const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int u = 0; u < 4; u += 2) {
          if (f + u >= p.d_rope) break;
          const int i = (f + u) / 2;
          const float x0 = xs[u], x1 = xs[u + 1];
          dst[f + u] = __float2bfloat16_rn(x0 * cs[i] - x1 * sn[i]);
          dst[f + u + 1] = __float2bfloat16_rn(x0 * sn[i] + x1 * cs[i]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, BN);
  }
}


// ------------------------------------------------------------------ fused query absorption
// q_packed[t, h] = ( W_UK[h]^T q_nope[t, h] || RoPE_pos(q_rope[t, h]) ) for one head and 64
// tokens per CTA ("DeepSeek-V2 大模型论文原文 PDF" 2.2, and the decoupled RoPE query of 2.3).
// The head's q_nope tile (64 tokens x d_nope) is loaded once and stays resident as the B
// operand; W_UK[h] (d_nope x d_c, rows along K, so A is MN-major) streams through an 8-deep
// ring of 128 (d_c) x 64 (d_nope) units, each m-block of 128 latent dims accumulating in its
// own 64 TMEM columns.  The four epilogue warps rotate the head's q_rope while the weights are
// in flight, then, as soon as an m-block's MMAs commit, round it to bf16 into one of two
// shared-memory tiles that a TMA bulk store writes out (64 token rows of 256 bytes) while the
// next m-block is converted.
constexpr int AB_THREADS = 192;
constexpr int AB_NST = 8;
constexpr int AB_MAX_KC = 4;   // d_nope <= 256
constexpr int AB_MAX_MB = 8;   // d_c <= 1024 (8 m-blocks x 64 TMEM columns)
constexpr int AB_RING = AB_NST * A_BYTES;
constexpr int AB_B_OFF = AB_RING;
constexpr int AB_STG_OFF = AB_B_OFF + AB_MAX_KC * 64 * BK * 2;  // 2 x [64 tokens][128] bf16 output tiles
constexpr int AB_BAR_OFF = AB_STG_OFF + 2 * 64 * 128 * 2;
constexpr int AB_SMEM = AB_BAR_OFF + 512 + 1024;

struct AbBars {
  uint64_t full[AB_NST], empty[AB_NST], bfull, mb_done[AB_MAX_MB];
  uint32_t tmem_base;
};
static_assert(sizeof(AbBars) <= 512, "barrier block");

struct AbParams {
  int T, H, d_c, d_nope, d_rope, mblocks, kchunks;
  uint32_t tcols;
  const __nv_bfloat16* q_rope;
  const int32_t* q_pos;
  const float* rcos;
  const float* rsin;
  int rope_rows;
  __nv_bfloat16* q_packed;
  int* err;
};

__global__ void __launch_bounds__(AB_THREADS, 1)
    absorb_tc_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_out, const AbParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  AbBars* bars = reinterpret_cast<AbBars*>(smem + AB_BAR_OFF);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int h = blockIdx.x;
  const int n0 = blockIdx.y * 64;
  const int units = p.mblocks * p.kchunks;

  if (threadIdx.x == 0) {
    for (int s = 0; s < AB_NST; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->bfull, 1);
    for (int b = 0; b < AB_MAX_MB; ++b) mbar_init(&bars->mb_done[b], 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, p.tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      // inputs only (weights, q_nope): no earlier grid of the stream writes them
      mbar_arrive_expect_tx(&bars->bfull, (uint32_t)p.kchunks * 64 * BK * 2);
      for (int kc = 0; kc < p.kchunks; ++kc)
        tma_load_2d(smem + AB_B_OFF + kc * 64 * BK * 2, &tm_q, h * p.d_nope + kc * BK, n0, &bars->bfull);
      int issued = 0;
      for (int u = 0; u < units; ++u) {
        const int s = u % AB_NST;
        if (u >= AB_NST && !mbar_wait(&bars->empty[s], ((u / AB_NST) - 1) & 1)) {
          record_error(p.err, ERR_TIMEOUT, 50);
          break;
        }
        const int mb = u / p.kchunks, kc = u % p.kchunks;
        uint8_t* st = smem + s * A_BYTES;
        const int y = h * p.d_nope + kc * BK;
        mbar_arrive_expect_tx(&bars->full[s], A_BYTES);
        tma_load_2d(st, &tm_w, mb * 128, y, &bars->full[s]);
        tma_load_2d(st + A_BYTES / 2, &tm_w, mb * 128 + 64, y, &bars->full[s]);
        issued = u + 1;
      }
      // no load of this CTA may still be in flight when it exits (bounded waits)
      mbar_wait(&bars->bfull, 0);
      for (int u = max(0, issued - AB_NST); u < issued; ++u)
        if (!mbar_wait(&bars->full[u % AB_NST], (u / AB_NST) & 1)) break;
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, 64, 1, 0);
      bool ok = mbar_wait(&bars->bfull, 0);
      if (!ok) record_error(p.err, ERR_TIMEOUT, 51);
      for (int u = 0; ok && u < units; ++u) {
        const int s = u % AB_NST;
        if (!mbar_wait(&bars->full[s], (u / AB_NST) & 1)) {
          record_error(p.err, ERR_TIMEOUT, 52);
          break;
        }
        tc_fence_after();
        const int mb = u / p.kchunks, kc = u % p.kchunks;
        const uint32_t a_base = smem_addr(smem + s * A_BYTES);
        const uint32_t b_base = smem_addr(smem + AB_B_OFF + kc * 64 * BK * 2);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          mma_bf16(tmem + mb * 64, umma_desc(a_base + kk * 2048, A_BYTES / 2, 1024, UMMA_SW128),
                   umma_desc(b_base + kk * 32, 16, 1024, UMMA_SW128), idesc, (kc > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars->empty[s]);
        if (kc == p.kchunks - 1) mma_commit(&bars->mb_done[mb]);
      }
    }
    __syncwarp();
  } else {
    // q_packed may still be read by an earlier grid of the stream until it completes
    griddep_wait();
    // query RoPE: each thread rotates 16 pairs (32 values, 64 bytes) of one token's q_rope,
    // all of its loads in flight at once
    const int e = threadIdx.x - 64;
    const int half = p.d_rope / 2;
    const int W = p.d_c + p.d_rope;
    const int per_tok = p.d_rope / 32;
    for (int idx = e; idx < 64 * per_tok; idx += 128) {
      const int t = n0 + idx / per_tok, i0 = (idx % per_tok) * 16;
      if (t >= p.T) break;
      const int ps = p.q_pos[t];
      const bool pos_ok = ps >= 0 && ps < p.rope_rows;
      if (!pos_ok && h == 0 && i0 == 0) record_error(p.err, ERR_POS, ps);
      const uint4* src = reinterpret_cast<const uint4*>(p.q_rope + ((long)t * p.H + h) * p.d_rope + 2 * i0);
      uint4 x[4];
      float4 c[4], sn[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) x[u] = src[u];
      if (pos_ok) {
        const float4* cp = reinterpret_cast<const float4*>(p.rcos + (long)ps * half + i0);
        const float4* sp = reinterpret_cast<const float4*>(p.rsin + (long)ps * half + i0);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          c[u] = cp[u];
          sn[u] = sp[u];
        }
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          c[u] = make_float4(1.f, 1.f, 1.f, 1.f);
          sn[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      uint4* dst = reinterpret_cast<uint4*>(p.q_packed + ((long)t * p.H + h) * W + p.d_c + 2 * i0);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        // x[u] holds pairs 4u .. 4u+3 of the 16; c[u], sn[u] their angles
        const uint32_t w[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
        const float cc[4] = {c[u].x, c[u].y, c[u].z, c[u].w};
        const float ss[4] = {sn[u].x, sn[u].y, sn[u].z, sn[u].w};
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&w[k]);
          const float x0 = __low2float(v), x1 = __high2float(v);
          const __nv_bfloat162 r =
              __halves2bfloat162(__float2bfloat16_rn(x0 * cc[k] - x1 * ss[k]), __float2bfloat16_rn(x0 * ss[k] + x1 * cc[k]));
          o[k] = *reinterpret_cast<const uint32_t*>(&r);
        }
        dst[u] = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
    const int quarter = warp & 3;
    const int m = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    bool ok = true;
    for (int mb = 0; mb < p.mblocks; ++mb) {
      // the four epilogue warps agree on the outcome, so the named barriers below stay matched
      ok = epi_sync_and(mbar_wait(&bars->mb_done[mb], 0, 4000000000ull));
      if (!ok) {
        if (e == 0) record_error(p.err, ERR_TIMEOUT, 53);
        break;
      }
      tc_fence_after();
      __nv_bfloat16* stg = reinterpret_cast<__nv_bfloat16*>(smem + AB_STG_OFF) + (mb & 1) * 64 * 128;
      if (mb >= 2) {
        if (e == 0) bulk_wait_group_read<1>();  // the store of m-block mb - 2 has read this tile
        epi_sync();
      }
      for (int c0 = 0; c0 < 64; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_off + mb * 64 + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) stg[(c0 + c) * 128 + m] = __float2bfloat16_rn(__uint_as_float(v[c]));
      }
      fence_proxy_async_smem();
      epi_sync();
      if (e == 0) {
        tma_store_2d(&tm_out, stg, h * W + mb * 128, n0);  // rows past T are not written
        bulk_commit_group();
      }
    }
    if (e == 0) bulk_wait_group<0>();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, p.tcols);
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
                  uint32_t box_rows, CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  auto enc = encoder();
  if (!enc) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15) || (ld * 2) % 16) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
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
  CUtensorMap ma, mb, mo;
  const bool ok_a = g.a_mn ? map2d(&ma, g.a, g.a_cols, g.a_rows, g.a_ld, 64, ptc::BK)
                           : map2d(&ma, g.a, g.a_cols, g.a_rows, g.a_ld, ptc::BK, 128);
  if (!ok_a || !map2d(&mb, g.b, g.b_cols, g.b_rows, g.b_ld, ptc::BK, BN)) return kUnsupported;
  // bf16 output through a TMA store when the tile's 128 rows are whole and the layout allows it
  const bool tma_out = g.out_mode == ptc::OUT_BF16 && g.k_splits == 1 && g.m_total % 128 == 0 &&
                       (g.out_group * 2) % 16 == 0 &&
                       map2d(&mo, g.out, (uint64_t)g.out_ld, (uint64_t)g.n_total, (uint64_t)g.out_ld, 128, BN,
                             CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!tma_out) mo = mb;
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
  p.tma_out = tma_out ? 1 : 0;
  p.err = err;
  constexpr int smem = ptc::wg_nst<BN>() * (ptc::A_BYTES + BN * ptc::BK * 2) + 256 + 1024;
  static_assert(BN * 128 * 2 <= ptc::wg_nst<BN>() * (ptc::A_BYTES + BN * ptc::BK * 2), "output tile fits the ring");
  cudaError_t e = cudaFuncSetAttribute(ptc::wgemm_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(g.groups * ((g.m_total + 127) / 128)), (unsigned)((g.n_total + BN - 1) / BN),
                     (unsigned)splits);
  cfg.blockDim = dim3(ptc::NTHREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, ptc::wgemm_kernel<BN>, ma, mb, mo, p);
  note_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
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

bool absorb_tc_aligned(const void* q_rope, const void* q_packed, const float* rcos, const float* rsin) {
  return ((reinterpret_cast<uintptr_t>(q_rope) | reinterpret_cast<uintptr_t>(q_packed) |
           reinterpret_cast<uintptr_t>(rcos) | reinterpret_cast<uintptr_t>(rsin)) & 15) == 0;
}

bool tc_absorb_fused_supported(const mla_dims& d) {
  return d.act_dtype == MLA_BF16 && tc_proj_supported(d) && d.d_c <= 128 * ptc::AB_MAX_MB &&
         d.d_nope <= ptc::BK * ptc::AB_MAX_KC && d.d_rope % 32 == 0 && d.d_rope > 0;
}

cudaError_t launch_absorb_tc(const mla_dims& d, const void* q_nope, const void* q_rope, const int32_t* q_pos,
                             int n_tok, const void* w_uk, const float* rcos, const float* rsin, int rope_rows,
                             void* q_packed, int* err, cudaStream_t st) {
  if (n_tok <= 0) return cudaSuccess;
  if ((n_tok + 63) / 64 > 65535) return kUnsupported;
  // 16-byte vector loads and stores of the RoPE part (callers check with absorb_tc_aligned)
  if (!absorb_tc_aligned(q_rope, q_packed, rcos, rsin)) return kUnsupported;
  CUtensorMap mw, mq, mo;
  const uint64_t W = (uint64_t)d.d_c + d.d_rope;
  if (!map2d(&mw, w_uk, d.d_c, (uint64_t)d.n_heads * d.d_nope, d.d_c, 64, ptc::BK) ||
      !map2d(&mq, q_nope, (uint64_t)d.n_heads * d.d_nope, n_tok, (uint64_t)d.n_heads * d.d_nope, ptc::BK, 64) ||
      !map2d(&mo, q_packed, d.n_heads * W, n_tok, d.n_heads * W, 128, 64, CU_TENSOR_MAP_SWIZZLE_NONE))
    return kUnsupported;
  ptc::AbParams p{};
  p.T = n_tok;
  p.H = d.n_heads;
  p.d_c = d.d_c;
  p.d_nope = d.d_nope;
  p.d_rope = d.d_rope;
  p.mblocks = d.d_c / 128;
  p.kchunks = d.d_nope / ptc::BK;
  uint32_t cols = 32;
  while (cols < (uint32_t)p.mblocks * 64) cols *= 2;
  p.tcols = cols;
  p.q_rope = static_cast<const __nv_bfloat16*>(q_rope);
  p.q_pos = q_pos;
  p.rcos = rcos;
  p.rsin = rsin;
  p.rope_rows = rope_rows;
  p.q_packed = static_cast<__nv_bfloat16*>(q_packed);
  p.err = err;
  cudaError_t e = cudaFuncSetAttribute(ptc::absorb_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, ptc::AB_SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)d.n_heads, (unsigned)((n_tok + 63) / 64), 1);
  cfg.blockDim = dim3(ptc::AB_THREADS);
  cfg.dynamicSmemBytes = ptc::AB_SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, ptc::absorb_tc_kernel, mw, mq, mo, p);
  note_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
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

// Split and tile choice for the fused append: with few token tiles, BN = 64 and the largest
// power-of-two cluster S <= 16 that keeps the grid within one wave of the 148 SMs; otherwise
// no split and the widest token tile.
template <int BN>
static cudaError_t launch_append_bn(const mla_dims& d, const void* h, int T, int S, const void* w_dkv,
                                    const void* w_kr, const ptc::ApParams& p0, cudaStream_t st) {
  using C = ptc::ApCfg<BN>;
  CUtensorMap mc, mr, mh;
  if (!map2d(&mc, w_dkv, d.d_model, d.d_c, d.d_model, ptc::BK, 128) ||
      !map2d(&mr, w_kr, d.d_model, d.d_rope, d.d_model, ptc::BK, d.d_rope) ||
      !map2d(&mh, h, d.d_model, T, d.d_model, ptc::BK, BN))
    return kUnsupported;
  ptc::ApParams p = p0;
  const int k_chunks = d.d_model / ptc::BK;
  p.kps = (k_chunks + S - 1) / S;
  cudaError_t e = cudaFuncSetAttribute(ptc::append_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  if (S > 8) {
    e = cudaFuncSetAttribute(ptc::append_tc_kernel<BN>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)S, (unsigned)(p.m_tiles_c + 1), (unsigned)((T + BN - 1) / BN));
  cfg.blockDim = dim3(ptc::AP_THREADS);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  e = cudaLaunchKernelEx(&cfg, ptc::append_tc_kernel<BN>, mc, mr, mh, p);
  note_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

// Largest cluster size <= want that the device can co-schedule for the BN = 64 kernel.
static int append_cluster_limit(int want) {
  static int cached = 0;
  if (!cached) {
    int best = 1;
    for (int s = 16; s >= 2 && best == 1; s /= 2) {
      if (s > 8 && cudaFuncSetAttribute(ptc::append_tc_kernel<64>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
                       cudaSuccess) {
        cudaGetLastError();
        continue;
      }
      if (cudaFuncSetAttribute(ptc::append_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               ptc::ApCfg<64>::SMEM) != cudaSuccess) {
        cudaGetLastError();
        break;
      }
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)s, 1, 1);
      cfg.blockDim = dim3(ptc::AP_THREADS);
      cfg.dynamicSmemBytes = ptc::ApCfg<64>::SMEM;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = (unsigned)s;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, ptc::append_tc_kernel<64>, &cfg) == cudaSuccess && n > 0)
        best = s;
      else
        cudaGetLastError();
    }
    cached = best;
  }
  return want < cached ? want : cached;
}

cudaError_t launch_append_tc(const mla_dims& d, const void* h, int T, const int32_t* seq_idx, const int32_t* pos,
                             const void* w_dkv, const void* w_kr, const float* rcos, const float* rsin,
                             int rope_rows, const CacheView& cv, int* err, cudaStream_t st) {
  if (T <= 0) return cudaSuccess;
  // 4-byte row stores, 16-byte TMA sources (checked by map2d); same alignment rule as the decode
  if ((reinterpret_cast<uintptr_t>(cv.rows) & 15) ||
      (cv.kind == MLA_FP8_E4M3 && ((reinterpret_cast<uintptr_t>(cv.rope) & 15) ||
                                   (reinterpret_cast<uintptr_t>(cv.scales) & 3))))
    return kUnsupported;
  if ((T + 63) / 64 > 65535) return kUnsupported;
  ptc::ApParams p{};
  p.T = T;
  p.d_model = d.d_model;
  p.d_c = d.d_c;
  p.d_rope = d.d_rope;
  p.m_tiles_c = d.d_c / 128;
  p.seq_idx = seq_idx;
  p.pos = pos;
  p.rcos = rcos;
  p.rsin = rsin;
  p.rope_rows = rope_rows;
  p.cv = cv;
  p.err = err;
  const int m_tiles = p.m_tiles_c + 1;
  const int k_chunks = d.d_model / ptc::BK;
  const int base = m_tiles * ((T + 63) / 64);
  if (2 * base <= 148) {
    int S = 2;
    while (S < 16 && base * S * 2 <= 148 && S * 2 <= k_chunks) S *= 2;
    S = append_cluster_limit(S);
    return launch_append_bn<64>(d, h, T, S, w_dkv, w_kr, p, st);
  }
  if (base <= 296) return launch_append_bn<64>(d, h, T, 1, w_dkv, w_kr, p, st);
  return launch_append_bn<256>(d, h, T, 1, w_dkv, w_kr, p, st);
}

}  // namespace mla
