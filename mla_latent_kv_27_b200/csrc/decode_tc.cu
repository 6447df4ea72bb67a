// Tensor-core (tcgen05 / TMEM) MLA decode for 128 heads over a bf16 latent cache.
//
// What it computes ("DeepSeek-V2 大模型论文原文 PDF" 2.2-2.3; softmax attention of
// intelliparadigm.com 3.3), for one query token (all 128 heads) and one KV chunk:
//   S = (Q_lat C^T + Q_rope K_rope^T) * scale,  online softmax,  O = P C,  lse.
// All heads share one latent cache, so QK^T and PV are dense contractions with the heads as
// the M = 128 dimension of the MMA.
//
// Mapping onto one SM pair (a cluster of two CTAs, rank r = 0, 1):
//  * An fp32 O of 128 heads x 512 latent dims would fill all 512 TMEM columns, and Q alone is
//    147 KB of shared memory, so the pair splits every cached row: CTA r owns latent dims
//    [256r, 256r + 256) and rope dims [32r, 32r + 32).  Each cache byte is loaded once.
//  * CTA r computes the partial S_r = Q_r K_r^T over its 288 dims (tcgen05, fp32 in TMEM),
//    rounds it to fp16 and ships it to its peer over DSMEM (st.async).  Both CTAs form
//    S = f32(f16(S_0)) + f32(f16(S_1)) in the same order of operands, so both see bit-equal
//    scores and take identical softmax decisions.
//  * Each CTA accumulates its half of O (128 x 256 fp32 = 256 TMEM columns) from P and the
//    latent half it already holds: V = C, so PV needs no further loads.
// Roles (192 threads): warp 0 issues TMA loads (Q once, then the cache 32 tokens at a time
// through a 5-stage ring), warp 1 owns TMEM and issues the MMAs (QK of tile i+1 is in flight
// while the softmax of tile i runs), warps 2-5 run the softmax (thread = head row = TMEM lane)
// and the epilogue.  The O rescale is lazy: O is rescaled only when a row's running max grows
// by more than 2^8, which keeps every exponent <= 2^8 and the result exact.
// Every wait is bounded (2 s); on timeout the kernel records MLA_ERR_TIMEOUT and winds down.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>

#include "mla_internal.cuh"
#include "sm100_ptx.cuh"
#include "decode_tc.cuh"

namespace mla {
namespace tc {

using namespace sm100;

constexpr int H = 128, DC = 512, DR = 64, W = 576;
constexpr int HALF_DC = 256, HALF_DR = 32;
constexpr int TILE = 32;     // tokens per pipeline step (half a page)
constexpr int NS = 5;        // cache stages
constexpr int NTHREADS = 192;

// shared-memory layout (bytes from a 1024-aligned base)
constexpr int Q_LAT_BOX = H * 64 * 2;               // 16384: 128 rows x 64 dims, 128B swizzle
constexpr int Q_ROPE_OFF = 4 * Q_LAT_BOX;           // 65536: 128 rows x 32 dims, 64B swizzle
constexpr int KV_OFF = Q_ROPE_OFF + H * HALF_DR * 2;  // 73728
constexpr int KV_LAT_BOX = TILE * 64 * 2;           // 4096: 32 tokens x 64 dims, 128B swizzle
constexpr int KV_ROPE_OFF = 4 * KV_LAT_BOX;         // 16384 within a stage: 32 x 32, 64B swizzle
constexpr int KV_STAGE = KV_ROPE_OFF + TILE * HALF_DR * 2;  // 18432
constexpr int P_OFF = KV_OFF + NS * KV_STAGE;       // 165888: 2 x (128 x 32 bf16, 64B swizzle)
constexpr int P_BUF = H * TILE * 2;                 // 8192
constexpr int RECV_OFF = P_OFF + 2 * P_BUF;         // 182272: 2 x (128 x 32 fp16)
constexpr int RECV_BUF = H * TILE * 2;              // 8192
constexpr int BAR_OFF = RECV_OFF + 2 * RECV_BUF;    // 198656
constexpr int SMEM_BYTES = BAR_OFF + 256 + 1024;    // barriers + alignment slack
constexpr uint32_t Q_BYTES = 4 * Q_LAT_BOX + H * HALF_DR * 2;  // 73728
constexpr uint32_t KV_BYTES = KV_STAGE;                         // 18432
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_O = 0, TM_S = 256;  // O half: cols [0, 256); S buffers: [256, 288), [288, 320)

struct Bars {
  uint64_t kv_full[NS], kv_empty[NS];
  uint64_t q_full;
  uint64_t s_full[2], s_empty[2], p_full[2], pv_done[2];
  uint64_t recv_full[2], peer_free[2];
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

struct Params {
  const int32_t* block_table;
  const int32_t* seq_lens;
  int max_pages, num_pages;
  int batch, s_q, causal, n_split;
  float scale_log2;  // scale * log2(e)
  __nv_bfloat16* o_lat;
  float* lse;
  float* o_part;
  float* lse_part;
  int* err;
};

__device__ __forceinline__ void fail(Bars* bars, int* err, int where) {
  record_error(err, ERR_TIMEOUT, where);
  atomicExch(&bars->abort_flag, 1);
}
__device__ __forceinline__ bool aborted(Bars* bars) {
  return *reinterpret_cast<volatile int*>(&bars->abort_flag) != 0;
}

// Which tokens this unit attends: [lo, hi) of sequence b for query token j.
struct Unit {
  int b, j, split, lo, hi, qrow;
};
__device__ __forceinline__ Unit make_unit(const Params& p, int unit, int* err, bool report) {
  Unit u;
  u.split = unit % p.n_split;
  const int bj = unit / p.n_split;
  u.j = bj % p.s_q;
  u.b = bj / p.s_q;
  u.qrow = u.b * p.s_q + u.j;
  int L = p.seq_lens[u.b];
  if (L < 0 || L > p.max_pages * 64) {
    if (report && u.split == 0 && u.j == 0) record_error(err, ERR_POS, L);
    L = max(0, min(L, p.max_pages * 64));
  }
  int A = L;
  if (p.causal) A = max(0, min(L, L - p.s_q + u.j + 1));
  const int pages = (A + 63) / 64;
  const int pps = (pages + p.n_split - 1) / p.n_split;
  u.lo = min(A, u.split * pps * 64);
  u.hi = min(A, (u.split + 1) * pps * 64);
  return u;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NTHREADS, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_q_lat, const __grid_constant__ CUtensorMap tm_q_rope,
                     const __grid_constant__ CUtensorMap tm_kv_lat, const __grid_constant__ CUtensorMap tm_kv_rope,
                     const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + BAR_OFF);
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int unit = blockIdx.x / 2;
  const Unit u = make_unit(p, unit, p.err, rank == 0 && threadIdx.x == 0);
  const int n_tiles = (u.hi - u.lo + TILE - 1) / TILE;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    mbar_init(&bars->q_full, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->s_empty[b], 4);
      mbar_init(&bars->p_full[b], 4);
      mbar_init(&bars->pv_done[b], 1);
      mbar_init(&bars->recv_full[b], 1);
      mbar_init(&bars->peer_free[b], 4);
    }
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync();  // peer barriers initialised before any remote arrive / st.async
  const uint32_t tmem = bars->tmem_base;

  if (n_tiles > 0) {
    if (warp == 0) {
      // ------------------------------------------------------------ TMA producer
      if (lane == 0) {
        prefetch_tmap(&tm_kv_lat);
        prefetch_tmap(&tm_kv_rope);
        mbar_arrive_expect_tx(&bars->q_full, Q_BYTES);
        const int qy = u.qrow * H;
        for (int jb = 0; jb < 4; ++jb)
          tma_load_2d(smem + jb * Q_LAT_BOX, &tm_q_lat, (int)rank * HALF_DC + jb * 64, qy, &bars->q_full);
        tma_load_2d(smem + Q_ROPE_OFF, &tm_q_rope, DC + (int)rank * HALF_DR, qy, &bars->q_full);
        const int32_t* bt = p.block_table + (long)u.b * p.max_pages;
        for (int i = 0; i < n_tiles; ++i) {
          const int s = i % NS;
          if (i >= NS && !mbar_wait(&bars->kv_empty[s], ((i / NS) - 1) & 1)) {
            fail(bars, p.err, 1);
            break;
          }
          if (aborted(bars)) break;
          const int t0 = u.lo + i * TILE;
          const int page = bt[t0 / 64];
          if ((page < 0 || page >= p.num_pages) && rank == 0) record_error(p.err, ERR_PAGE, page);
          // an out-of-range page reads TMA's zero fill; the softmax masks those tokens
          const int y = page * 64 + (t0 % 64);
          uint8_t* st = smem + KV_OFF + s * KV_STAGE;
          mbar_arrive_expect_tx(&bars->kv_full[s], KV_BYTES);
          for (int jb = 0; jb < 4; ++jb)
            tma_load_2d(st + jb * KV_LAT_BOX, &tm_kv_lat, (int)rank * HALF_DC + jb * 64, y, &bars->kv_full[s]);
          tma_load_2d(st + KV_ROPE_OFF, &tm_kv_rope, DC + (int)rank * HALF_DR, y, &bars->kv_full[s]);
        }
        // drain: every stage still being filled completes before the CTA may exit
        for (int i = max(0, n_tiles - NS); i < n_tiles; ++i)
          if (!mbar_wait(&bars->kv_full[i % NS], (i / NS) & 1)) break;
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        constexpr uint32_t ID_QK = idesc_bf16(128, TILE, 0, 0);
        constexpr uint32_t ID_PV = idesc_bf16(128, HALF_DC, 0, 1);
        const uint32_t q_base = smem_addr(smem);
        bool ok = mbar_wait(&bars->q_full, 0);
        if (!ok) fail(bars, p.err, 2);
        auto issue_pv = [&](int jt) -> bool {
          const int b = jt & 1;
          if (!mbar_wait(&bars->p_full[b], (jt >> 1) & 1)) return false;
          tc_fence_after();
          const uint32_t p_base = smem_addr(smem + P_OFF + b * P_BUF);
          const uint32_t v_base = smem_addr(smem + KV_OFF + (jt % NS) * KV_STAGE);
#pragma unroll
          for (int kt = 0; kt < TILE / 16; ++kt) {
            const uint64_t a = umma_desc(p_base + kt * 32, 16, 512, UMMA_SW64);
            const uint64_t bdesc = umma_desc(v_base + kt * 2048, KV_LAT_BOX, 1024, UMMA_SW128);
            mma_bf16(tmem + TM_O, a, bdesc, ID_PV, (jt > 0 || kt > 0) ? 1u : 0u);
          }
          mma_commit(&bars->pv_done[b]);
          mma_commit(&bars->kv_empty[jt % NS]);
          return true;
        };
        for (int i = 0; ok && i < n_tiles; ++i) {
          const int s = i % NS, b = i & 1;
          if (!mbar_wait(&bars->kv_full[s], (i / NS) & 1) ||
              (i >= 2 && !mbar_wait(&bars->s_empty[b], ((i >> 1) - 1) & 1))) {
            fail(bars, p.err, 3);
            ok = false;
            break;
          }
          if (aborted(bars)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t kv = smem_addr(smem + KV_OFF + s * KV_STAGE);
          const uint32_t d = tmem + TM_S + b * TILE;
#pragma unroll
          for (int ks = 0; ks < 16; ++ks) {  // latent half: 4 boxes x 4 K-steps of 16
            const uint32_t off = (ks & 3) * 32;
            const uint64_t a = umma_desc(q_base + (ks >> 2) * Q_LAT_BOX + off, 16, 1024, UMMA_SW128);
            const uint64_t bd = umma_desc(kv + (ks >> 2) * KV_LAT_BOX + off, 16, 1024, UMMA_SW128);
            mma_bf16(d, a, bd, ID_QK, ks > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) {  // rope half: 2 K-steps of 16
            const uint64_t a = umma_desc(q_base + Q_ROPE_OFF + ks * 32, 16, 512, UMMA_SW64);
            const uint64_t bd = umma_desc(kv + KV_ROPE_OFF + ks * 32, 16, 512, UMMA_SW64);
            mma_bf16(d, a, bd, ID_QK, 1u);
          }
          mma_commit(&bars->s_full[b]);
          if (i >= 1 && !issue_pv(i - 1)) {
            fail(bars, p.err, 4);
            ok = false;
            break;
          }
        }
        if (ok && !issue_pv(n_tiles - 1)) fail(bars, p.err, 5);
      }
    } else {
      // ------------------------------------------------------------ softmax + epilogue
      const int quarter = warp & 3;          // TMEM lane quarter this warp may access
      const int row = quarter * 32 + lane;   // head
      const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
      float m_used = -INFINITY, l_sum = 0.f;
      const int32_t* bt = p.block_table + (long)u.b * p.max_pages;
      uint8_t* recv_row_base = smem + RECV_OFF + row * (TILE * 2);
      bool ok = true;
      for (int i = 0; i < n_tiles; ++i) {
        const int b = i & 1, use = i >> 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[b], use & 1))) {
          fail(bars, p.err, 10);
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sraw[32];
        tmem_ld32(tmem + lane_off + TM_S + b * TILE, sraw);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_empty[b]);
        // own partial, rounded to fp16 exactly as the peer will see it
        uint32_t packed[16];
        float own[32];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          __half2 h2 = __floats2half2_rn(__uint_as_float(sraw[2 * c]), __uint_as_float(sraw[2 * c + 1]));
          packed[c] = *reinterpret_cast<uint32_t*>(&h2);
          float2 f2 = __half22float2(h2);
          own[2 * c] = f2.x;
          own[2 * c + 1] = f2.y;
        }
        // ship it to the peer's receive buffer b (after the peer has freed it)
        if (i >= 2 && !__all_sync(0xffffffffu, mbar_wait(&bars->peer_free[b], (use - 1) & 1))) {
          fail(bars, p.err, 11);
          ok = false;
          break;
        }
        if (threadIdx.x == 64) mbar_arrive_expect_tx(&bars->recv_full[b], RECV_BUF);
        {
          uint8_t* local_row = recv_row_base + b * RECV_BUF;
          const uint32_t remote_row = map_to_rank(local_row, peer);
          const uint32_t remote_bar = map_to_rank(&bars->recv_full[b], peer);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int pc = c ^ ((row >> 1) & 3);
            st_async_v4(remote_row + pc * 16,
                        make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]),
                        remote_bar);
          }
        }
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->recv_full[b], use & 1))) {
          fail(bars, p.err, 12);
          ok = false;
          break;
        }
        float x[32];
        {
          const uint8_t* local_row = recv_row_base + b * RECV_BUF;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int pc = c ^ ((row >> 1) & 3);
            const uint4 v = *reinterpret_cast<const uint4*>(local_row + pc * 16);
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              __half2 h2 = *reinterpret_cast<const __half2*>(&w4[k]);
              float2 f2 = __half22float2(h2);
              // identical operand order on both CTAs: rank-0 partial + rank-1 partial
              const float a0 = own[8 * c + 2 * k], a1 = own[8 * c + 2 * k + 1];
              x[8 * c + 2 * k] = rank == 0 ? a0 + f2.x : f2.x + a0;
              x[8 * c + 2 * k + 1] = rank == 0 ? a1 + f2.y : f2.y + a1;
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(&bars->peer_free[b], peer);
        // mask and scale into the log2 domain
        const int t0 = u.lo + i * TILE;
        const int n_valid = min(TILE, u.hi - t0);
        const int page = bt[t0 / 64];
        const bool page_ok = page >= 0 && page < p.num_pages;
        float m_tile = -INFINITY;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          x[c] = (c < n_valid && page_ok) ? x[c] * p.scale_log2 : -INFINITY;
          m_tile = fmaxf(m_tile, x[c]);
        }
        const float m_new = fmaxf(m_used, m_tile);
        float alpha = 1.f;
        if (m_new > m_used + 8.f) {  // lazy rescale: only when the max grows by more than 2^8
          alpha = exp2f(m_used - m_new);
          m_used = m_new;
        }
        float psum = 0.f;
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          float p0 = m_used == -INFINITY ? 0.f : exp2f(x[2 * c] - m_used);
          float p1 = m_used == -INFINITY ? 0.f : exp2f(x[2 * c + 1] - m_used);
          __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
          pk[c] = *reinterpret_cast<uint32_t*>(&pb);
          float2 pf = __bfloat1622float2(pb);  // sum what the MMA will use
          psum += pf.x + pf.y;
        }
        l_sum = l_sum * alpha + psum;
        // PV(i-1) must be complete before O is rescaled and before P buffer b is rewritten
        // (PV(i-2) used it); waiting for PV(i-1) covers both.
        const bool need_rescale = __any_sync(0xffffffffu, alpha != 1.f) && i > 0;
        if (i >= 1) {
          const int jt = need_rescale ? i - 1 : (i >= 2 ? i - 2 : -1);
          if (jt >= 0 && !__all_sync(0xffffffffu, mbar_wait(&bars->pv_done[jt & 1], (jt >> 1) & 1))) {
            fail(bars, p.err, 13);
            ok = false;
            break;
          }
          tc_fence_after();
        }
        if (need_rescale) {
          for (int cb = 0; cb < HALF_DC / 32; ++cb) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_off + TM_O + cb * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st32(tmem + lane_off + TM_O + cb * 32, o);
          }
          tmem_wait_st();
        }
        // V rows past the valid tokens may hold stale data: zero them so 0 * garbage = 0.
        // Warp q zeroes latent box q of the stage; it arrives on p_full only afterwards.
        if (n_valid < TILE || !page_ok) {
          uint8_t* box = smem + KV_OFF + (i % NS) * KV_STAGE + quarter * KV_LAT_BOX;
          const int first = page_ok ? n_valid : 0;
          for (int e = lane; e < (TILE - first) * 8; e += 32)
            *reinterpret_cast<uint4*>(box + (first + e / 8) * 128 + (e % 8) * 16) = make_uint4(0, 0, 0, 0);
        }
        // P row (bf16), K-major with 64-byte swizzle
        uint8_t* prow = smem + P_OFF + b * P_BUF + row * 64;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int pc = c ^ ((row >> 1) & 3);
          *reinterpret_cast<uint4*>(prow + pc * 16) = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_full[b]);
      }
      // ------------------------------------------------------------ epilogue
      const float inv_l = l_sum > 0.f ? 1.f / l_sum : 0.f;
      const float lse = l_sum > 0.f ? (m_used + log2f(l_sum)) * 0.69314718055994531f : -INFINITY;
      if (ok) {
        const int jt = n_tiles - 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->pv_done[jt & 1], (jt >> 1) & 1))) {
          fail(bars, p.err, 14);
          ok = false;
        }
        tc_fence_after();
      }
      const long qh = (long)u.qrow * H + row;
      const bool final_out = p.n_split == 1;
      const long prow_idx = (((long)u.b * p.n_split + u.split) * p.s_q + u.j) * H + row;
      for (int cb = 0; cb < HALF_DC / 32; ++cb) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_off + TM_O + cb * 32, o);
        tmem_wait_ld();
        const int d0 = (int)rank * HALF_DC + cb * 32;
        if (final_out) {
          uint4* dst = reinterpret_cast<uint4*>(p.o_lat + qh * DC + d0);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t w4[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float a = ok ? __uint_as_float(o[8 * q + 2 * k]) * inv_l : 0.f;
              const float bq = ok ? __uint_as_float(o[8 * q + 2 * k + 1]) * inv_l : 0.f;
              __nv_bfloat162 v = __floats2bfloat162_rn(a, bq);
              w4[k] = *reinterpret_cast<uint32_t*>(&v);
            }
            dst[q] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        } else {
          float4* dst = reinterpret_cast<float4*>(p.o_part + prow_idx * DC + d0);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            float4 v;
            v.x = ok ? __uint_as_float(o[4 * q]) * inv_l : 0.f;
            v.y = ok ? __uint_as_float(o[4 * q + 1]) * inv_l : 0.f;
            v.z = ok ? __uint_as_float(o[4 * q + 2]) * inv_l : 0.f;
            v.w = ok ? __uint_as_float(o[4 * q + 3]) * inv_l : 0.f;
            dst[q] = v;
          }
        }
      }
      if (rank == 0) {
        if (final_out) {
          if (p.lse) p.lse[qh] = ok ? lse : -INFINITY;
        } else {
          p.lse_part[prow_idx] = ok ? lse : -INFINITY;
        }
      }
    }
  } else if (warp >= 2) {
    // empty unit: o = 0, lse = -inf
    const int row = (warp & 3) * 32 + lane;
    const long qh = (long)u.qrow * H + row;
    const long prow_idx = (((long)u.b * p.n_split + u.split) * p.s_q + u.j) * H + row;
    for (int d = 0; d < HALF_DC; d += 8) {
      const int d0 = (int)rank * HALF_DC + d;
      if (p.n_split == 1)
        *reinterpret_cast<uint4*>(p.o_lat + qh * DC + d0) = make_uint4(0, 0, 0, 0);
      else {
        reinterpret_cast<float4*>(p.o_part + prow_idx * DC + d0)[0] = make_float4(0.f, 0.f, 0.f, 0.f);
        reinterpret_cast<float4*>(p.o_part + prow_idx * DC + d0)[1] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    if (rank == 0) {
      if (p.n_split == 1) {
        if (p.lse) p.lse[qh] = -INFINITY;
      } else {
        p.lse_part[prow_idx] = -INFINITY;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
  cluster_sync();  // no CTA leaves while its peer may still touch its shared memory
}

}  // namespace tc

// ------------------------------------------------------------------ host side

static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
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

// 2-D bf16 tensor map over rows of 576 values.
static bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_cols, uint32_t box_rows,
                     CUtensorMapSwizzle sw) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)tc::W, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)tc::W * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool tc_decode_supported(const mla_dims& d, int cache_kind) {
  return d.n_heads == tc::H && d.d_c == tc::DC && d.d_rope == tc::DR && d.page_size == 64 &&
         d.act_dtype == MLA_BF16 && cache_kind == MLA_BF16;
}

int tc_auto_split(int batch, int s_q, int max_pages) {
  // aim at >= 2 clusters per SM pair (74 pairs on 148 SMs)
  const long units = (long)batch * s_q;
  int n = (int)((2 * 74 + units - 1) / units);
  n = n < 1 ? 1 : n;
  const int max_chunks = (max_pages * 64 + tc::TILE - 1) / tc::TILE;
  if (n > max_chunks) n = max_chunks;
  if (n > 64) n = 64;
  return n;
}

cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t st) {
  const CacheView& cv = a.cache;
  tc::Params prm;
  prm.block_table = cv.block_table;
  prm.seq_lens = a.seq_lens;
  prm.max_pages = cv.max_pages;
  prm.num_pages = cv.num_pages;
  prm.batch = a.batch;
  prm.s_q = a.s_q;
  prm.causal = a.causal;
  prm.n_split = a.n_split;
  prm.scale_log2 = a.scale * 1.4426950408889634f;
  prm.o_lat = reinterpret_cast<__nv_bfloat16*>(a.o_lat);
  prm.lse = a.lse;
  prm.o_part = a.o_part;
  prm.lse_part = a.lse_part;
  prm.err = a.err;
  CUtensorMap mq_lat, mq_rope, mkv_lat, mkv_rope;
  const uint64_t q_rows = (uint64_t)a.batch * a.s_q * tc::H;
  const uint64_t kv_rows = (uint64_t)cv.num_pages * 64;
  if (!make_map(&mq_lat, a.q, q_rows, 64, tc::H, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&mq_rope, a.q, q_rows, tc::HALF_DR, tc::H, CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_map(&mkv_lat, cv.rows, kv_rows, 64, tc::TILE, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&mkv_rope, cv.rows, kv_rows, tc::HALF_DR, tc::TILE, CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(tc::decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       tc::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const long units = (long)a.batch * a.s_q * a.n_split;
  if (units == 0) return cudaSuccess;
  tc::decode_tc_kernel<<<dim3((unsigned)(2 * units)), tc::NTHREADS, tc::SMEM_BYTES, st>>>(mq_lat, mq_rope, mkv_lat,
                                                                                           mkv_rope, prm);
  note_launch();
  return cudaGetLastError();
}

}  // namespace mla
