// Small-head MLA decode (at most 16 heads) over a bf16 paged latent cache.
//
// What it computes ("DeepSeek-V2 大模型论文原文 PDF" 2.2-2.3; softmax attention of
// intelliparadigm.com 3.3), for one query token (all heads) and one KV chunk:
//   S = (Q_lat C^T + Q_rope K_rope^T) * scale,  online softmax,  O = P C,  lse.
// With 16 heads the product is 16 rows tall: a tcgen05 MMA (M >= 64) would be three quarters
// padding and would add TMEM commit round trips to a loop that is bound by HBM, not by the tensor
// pipe.  Here the heads are exactly the M = 16 of the warp-level mma.sync.m16n8k16 (bf16 in, fp32
// accumulate), the accumulators stay in registers, and one CTA (two per SM) streams its share of
// the cache:
//  * Work: the length-balanced partition of the tensor-core kernel (decode_plan.cuh), 148 x 2
//    persistent CTAs, each walking its range of pages; rows cut across ranges leave fp32 partials
//    for the same log-sum-exp combine.
//  * Cache: a ring of two 32-token tiles (half a page, 9 TMA boxes of 64 dims x 32 tokens with the
//    128-byte swizzle: 8 latent boxes and the rope box).  A stage is refilled once every warp has
//    passed the next tile's first barrier; nine lanes of warp 0 issue the nine boxes at once.  Q
//    (16 rows x 576) is loaded once per segment the same way.
//  * Per tile, 8 warps:
//    - QK: warp w takes tokens 8 (w % 4) .. + 7 and one half of the 576 dims (w / 4): 18 MMAs
//      on ldmatrix fragments of Q and of the cache tile; the two halves' partial scores meet in
//      shared memory.
//    - Softmax: warp w takes heads 2w, 2w + 1 at once, a half warp each, two tokens per lane:
//      exact running maximum and sum per head (shuffles within the half warp), P rounded to bf16
//      in shared memory, the rescale factor of O.
//    - PV: warp w owns latent dims 64w .. 64w + 63 of O (16 x 64 fp32 in registers), rescales
//      them and adds P V over the tile's 32 tokens (16 MMAs, V fragments by transposing
//      ldmatrix from the same cache tile: V = C).
//  * Every mbarrier wait is bounded (2 s); on a timeout the kernel records MLA_ERR_TIMEOUT and
//    winds down (all threads leave together).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "mla_internal.cuh"
#include "sm100_ptx.cuh"
#include "decode_plan.cuh"
#include "decode_tc.cuh"

namespace mla {
namespace sh {

using namespace sm100;

constexpr int DC = 512, DR = 64, W = 576;
constexpr int HP = 16;                  // head rows of the MMA
constexpr int TS = 32;                  // tokens per tile (half a page)
constexpr int NBOX = W / 64;            // 9 boxes of 64 dims: 8 latent, then the rope dims
constexpr int BOX = TS * 128;           // 4096 bytes: 32 tokens x 128 bytes
constexpr int STAGE = NBOX * BOX;       // 36864
constexpr int NS = 2;                   // cache stages
constexpr int NTHREADS = 256;           // 8 warps
constexpr int ROW_COST = 1;             // a segment boundary (Q reload, ring restart): about a page
constexpr int Q_BOX = HP * 128;         // 2048: 16 rows x 64 dims
constexpr int Q_OFF = 0;
constexpr int ST_OFF = NBOX * Q_BOX;    // 18432
constexpr int S_OFF = ST_OFF + NS * STAGE;       // [dim half][head][token] fp32 partial scores
constexpr int S_BYTES = 2 * HP * TS * 4;
constexpr int P_OFF = S_OFF + S_BYTES;           // [head][token] bf16, 80-byte rows (no bank conflicts)
constexpr int P_ROW = 80;
constexpr int M_OFF = P_OFF + HP * P_ROW;        // running max, sum, rescale factor per head (fp32)
constexpr int LIM_OFF = M_OFF + 3 * HP * 4;      // valid tokens of each stage's tile
constexpr int BAR_OFF = (LIM_OFF + NS * 4 + 15) / 8 * 8;
static_assert(ST_OFF % 1024 == 0 && STAGE % 1024 == 0 && BAR_OFF % 8 == 0, "swizzle and barrier alignment");

struct Bars {
  uint64_t full[NS];
  uint64_t q_full;
  plan::Unit unit, next;
};
constexpr int SMEM_BYTES = BAR_OFF + (int)sizeof(Bars) + 1024;  // + alignment slack
static_assert(2 * (SMEM_BYTES + 1024) <= 233472, "two CTAs per SM");

struct Params {
  const int32_t* block_table;
  const int32_t* seq_lens;
  int H;
  int max_pages, num_pages;
  int batch, s_q, causal;
  float scale_log2;  // scale * log2(e)
  __nv_bfloat16* o_lat;
  float* lse;
  float* o_part;
  float* lse_part;
  int* err;
  int n_workers;     // ranges of the partition (workers = n_workers * s_q)
  int32_t* rowinfo;  // [rows][2] first / last partial slot of each row (-1: no pages)
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr)
               : "memory");
}
// D (16 x 8 fp32) += A (16 x 16 bf16, row-major) B (16 x 8 bf16, column-major)
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// byte address of 16-byte chunk c of row r in a box with 128-byte rows and the 128-byte swizzle
__device__ __forceinline__ uint32_t sw128(uint32_t box, int r, int c) {
  return box + (uint32_t)(r * 128) + (uint32_t)(((c ^ (r & 7)) & 7) << 4);
}

__global__ void __launch_bounds__(NTHREADS, 2)
    decode_sh_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
                     const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + BAR_OFF);
  float* sbuf = reinterpret_cast<float*>(smem + S_OFF);
  float* m_s = reinterpret_cast<float*>(smem + M_OFF);
  float* l_s = m_s + HP;
  float* a_s = l_s + HP;
  int* lim_s = reinterpret_cast<int*>(smem + LIM_OFF);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int worker = blockIdx.x;
  // the combine (launched programmatically) may take each SM this CTA leaves; it waits for the
  // whole grid's writes before it reads any
  griddep_launch_dependents();

  plan::Plan pl;  // warp 0 only
  if (warp == 0) {
    plan::plan_begin<ROW_COST>(p, pl, worker, lane);
    if (worker == 0) plan::write_rowinfo<ROW_COST>(p, pl.T, max(pl.U, 1ll), lane);
    const plan::Unit f = plan::plan_next<ROW_COST>(p, pl, worker, lane);
    __syncwarp();
    if (lane == 0) bars->next = f;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) mbar_init(&bars->full[s], 1);
    mbar_init(&bars->q_full, 1);
    fence_mbar_init();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_kv);
  }
  __syncthreads();

  int gb = 0, seg = 0;   // tiles and segments done (barrier phases run on across segments)
  int issued = 0;        // tiles whose loads were issued, over all segments (warp 0)
  bool ok = true;
  for (;;) {
    if (threadIdx.x == 0) bars->unit = bars->next;
    __syncthreads();
    const plan::Unit u = bars->unit;
    if (!u.valid) break;
    const int n_tiles = (u.hi - u.lo + TS - 1) / TS;
    const int32_t* bt = p.block_table + (long)u.b * p.max_pages;
    // Tile i of the segment: TMA of its 9 boxes (thread 0).  A bad page id reads TMA's zero fill
    // past the end of the cache and counts no tokens.  Page ids are read one issue ahead into
    // registers, so an issue never waits on a global load: pg_next holds tile `next_tile`'s page.
    // (Prefetching tiles into L2 ahead of their TMA was measured 7 % slower: the extra requests
    // compete with the loads the ring is waiting for.)
    auto page_of = [&](int i) -> int { return i < n_tiles ? bt[(u.lo + i * TS) / 64] : -1; };
    int next_tile = 0, pg_next = 0;
    // (warp 0, all lanes: lane 0 arms the barrier, lanes 0-8 issue one box each)
    auto issue = [&]() {
      const int i = next_tile++;
      const int g = gb + i, s = g % NS;
      const int t0 = u.lo + i * TS;
      const int page = pg_next;
      pg_next = page_of(i + 1);
      const bool bad = page < 0 || page >= p.num_pages;
      if (bad && lane == 0) record_error(p.err, ERR_PAGE, page);
      const int y = (bad ? p.num_pages * 64 : page * 64) + t0 % 64;
      uint8_t* st = smem + ST_OFF + s * STAGE;
      if (lane == 0) {
        lim_s[s] = bad ? 0 : min(TS, u.hi - t0);  // published by the arrive below
        mbar_arrive_expect_tx(&bars->full[s], STAGE);
      }
      __syncwarp();
      if (lane < NBOX) tma_load_2d(st + lane * BOX, &tm_kv, lane * 64, y, &bars->full[s]);
      ++issued;
    };
    if (warp == 0) {
      if (lane == 0) mbar_arrive_expect_tx(&bars->q_full, NBOX * Q_BOX);
      __syncwarp();
      const int qy = u.qrow * p.H;  // rows past H: the next query rows or TMA's zero fill
      if (lane < NBOX) tma_load_2d(smem + Q_OFF + lane * Q_BOX, &tm_q, lane * 64, qy, &bars->q_full);
      pg_next = page_of(0);
      for (int i = 0; i < min(NS, n_tiles); ++i) issue();
    }
    // the segment after this one, planned while these loads are in flight
    if (warp == 0) {
      const plan::Unit t2 = plan::plan_next<ROW_COST>(p, pl, worker, lane);
      __syncwarp();
      if (lane == 0) bars->next = t2;
    }
    if (threadIdx.x < HP) {
      m_s[threadIdx.x] = -INFINITY;
      l_s[threadIdx.x] = 0.f;
    }
    // O: rows lane / 4 and lane / 4 + 8, dims 64 warp + 8 nt + 2 (lane % 4) + {0, 1}
    float o[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
    ok = __syncthreads_and(mbar_wait(&bars->q_full, seg & 1) ? 1 : 0) != 0;
    if (!ok) {
      if (threadIdx.x == 0) record_error(p.err, ERR_TIMEOUT, 40);
      break;
    }
    const uint32_t q_base = smem_addr(smem + Q_OFF);
    for (int i = 0; i < n_tiles; ++i) {
      const int g = gb + i, s = g % NS;
      const bool landed = mbar_wait(&bars->full[s], (g / NS) & 1);
      const uint32_t st = smem_addr(smem + ST_OFF + s * STAGE);
      // ---- QK: tokens 8 nb .. 8 nb + 7, k-steps 18 kh .. 18 kh + 17 (16 dims each)
      {
        const int nb = warp & 3, kh = warp >> 2;
        float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
        const int qr = lane & 15, kr = nb * 8 + (lane & 7);
#pragma unroll
        for (int kk = 0; kk < 18; kk += 2) {
          const int ks = kh * 18 + kk;          // k-steps ks, ks + 1 share box ks / 4
          const int jb = ks >> 2, c = (ks & 3) * 2;
          uint32_t a0[4], a1[4], b0, b1, b2, b3;
          const uint32_t qb = q_base + jb * Q_BOX;
          ldsm_x4(sw128(qb, qr, c + (lane >> 4)), a0[0], a0[1], a0[2], a0[3]);
          ldsm_x4(sw128(qb, qr, c + 2 + (lane >> 4)), a1[0], a1[1], a1[2], a1[3]);
          ldsm_x4(sw128(st + jb * BOX, kr, c + (lane >> 3)), b0, b1, b2, b3);
          mma16816(c0, a0, b0, b1);
          mma16816(c1, a1, b2, b3);
        }
        float* sk = sbuf + kh * HP * TS;
        const int r0 = lane >> 2, tc = nb * 8 + 2 * (lane & 3);
        *reinterpret_cast<float2*>(sk + r0 * TS + tc) = make_float2(c0[0] + c1[0], c0[1] + c1[1]);
        *reinterpret_cast<float2*>(sk + (r0 + 8) * TS + tc) = make_float2(c0[2] + c1[2], c0[3] + c1[3]);
      }
      ok = __syncthreads_and(landed ? 1 : 0) != 0;
      if (!ok) {
        if (threadIdx.x == 0) record_error(p.err, ERR_TIMEOUT, 41);
        break;
      }
      // every warp is done with tile i - 1: its stage takes tile i - 1 + NS
      if (warp == 0 && i >= 1 && i - 1 + NS < n_tiles) issue();  // tile i - 1 + NS
      // ---- softmax: head 2 warp + lane / 16 (each half warp one head), tokens 2 (lane % 16), + 1
      {
        const int lim = lim_s[s];
        const int h = 2 * warp + (lane >> 4), t = 2 * (lane & 15);
        const float2 s0 = *reinterpret_cast<const float2*>(sbuf + h * TS + t);
        const float2 s1 = *reinterpret_cast<const float2*>(sbuf + HP * TS + h * TS + t);
        float x0 = (s0.x + s1.x) * p.scale_log2, x1 = (s0.y + s1.y) * p.scale_log2;
        if (t >= lim) x0 = -INFINITY;
        if (t + 1 >= lim) x1 = -INFINITY;
        float mx = fmaxf(x0, x1);
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float m_old = m_s[h];
        const float m_new = fmaxf(m_old, mx);
        const float mu = m_new == -INFINITY ? 0.f : m_new;  // 2^(-inf - 0) = 0
        const float p0 = ex2_approx(x0 - mu), p1 = ex2_approx(x1 - mu);
        float sum = p0 + p1;
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        *reinterpret_cast<__nv_bfloat162*>(smem + P_OFF + h * P_ROW + t * 2) = __floats2bfloat162_rn(p0, p1);
        if ((lane & 15) == 0) {
          // while the maximum is -inf every earlier score was masked: O and l are still zero
          const float alpha = m_old == -INFINITY ? 0.f : ex2_approx(m_old - mu);
          m_s[h] = m_new;
          l_s[h] = l_s[h] * alpha + sum;
          a_s[h] = alpha;
        }
      }
      __syncthreads();
      // ---- PV: dims 64 warp .. 64 warp + 63 (latent box `warp`), 2 k-steps of 16 tokens
      {
        const float al0 = a_s[lane >> 2], al1 = a_s[(lane >> 2) + 8];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          o[nt][0] *= al0;
          o[nt][1] *= al0;
          o[nt][2] *= al1;
          o[nt][3] *= al1;
        }
        const uint32_t pb = smem_addr(smem + P_OFF);
        const uint32_t vbox = st + warp * BOX;
#pragma unroll
        for (int ks = 0; ks < TS / 16; ++ks) {
          uint32_t a[4];
          ldsm_x4(pb + (lane & 15) * P_ROW + (ks * 2 + (lane >> 4)) * 16, a[0], a[1], a[2], a[3]);
          const int vr = ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
          for (int np = 0; np < 4; ++np) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4_trans(sw128(vbox, vr, np * 2 + (lane >> 4)), b0, b1, b2, b3);
            mma16816(o[2 * np], a, b0, b1);
            mma16816(o[2 * np + 1], a, b2, b3);
          }
        }
      }
    }
    if (!ok) break;
    __syncthreads();  // every warp's last PV is done
    // ---- epilogue: O / l, to o_lat (a row this segment covers whole) or to the row's partial slot
    {
      const int r0 = lane >> 2;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int h = r0 + 8 * half;
        if (h >= p.H) continue;
        const float l = l_s[h];
        const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          const int d = warp * 64 + nt * 8 + 2 * (lane & 3);
          const float v0 = o[nt][2 * half] * inv, v1 = o[nt][2 * half + 1] * inv;
          if (u.final_out) {
            *reinterpret_cast<__nv_bfloat162*>(p.o_lat + ((long)u.qrow * p.H + h) * DC + d) =
                __floats2bfloat162_rn(v0, v1);
          } else {
            *reinterpret_cast<float2*>(p.o_part + ((long)u.slot * p.H + h) * DC + d) = make_float2(v0, v1);
          }
        }
      }
      if (warp == 0 && lane < p.H && lane < HP) {
        const float l = l_s[lane];
        const float lse = l > 0.f ? (m_s[lane] + log2f(l)) * 0.69314718055994531f : -INFINITY;
        if (u.final_out) {
          if (p.lse) p.lse[(long)u.qrow * p.H + lane] = lse;
        } else {
          p.lse_part[(long)u.slot * p.H + lane] = lse;
        }
      }
    }
    gb += n_tiles;
    ++seg;
    __syncthreads();  // the state and Q are free for the next segment
  }
  // every load still in flight lands before the CTA may exit
  if (threadIdx.x == 0)
    for (int t = max(0, issued - NS); t < issued; ++t) mbar_wait(&bars->full[t % NS], (t / NS) & 1);
  __syncthreads();
}

}  // namespace sh

bool sh_decode_supported(const mla_dims& d, int cache_kind) {
  return d.n_heads >= 1 && d.n_heads <= sh::HP && d.d_c == sh::DC && d.d_rope == sh::DR && d.page_size == 64 &&
         d.act_dtype == MLA_BF16 && cache_kind == MLA_BF16;
}

size_t sh_plan_workspace_bytes(const mla_dims& d, int batch, int s_q) {
  const size_t rows = (size_t)batch * s_q;
  return (size_t)SH_PLAN_SLOTS * d.n_heads * (d.d_c + 1) * sizeof(float) + rows * 2 * sizeof(int32_t);
}

static bool make_map_sh(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  if (!enc) {
    cudaDriverEntryPointQueryResult q;
    void* fp = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fp, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fp);
  }
  if (reinterpret_cast<uintptr_t>(base) & 15) return false;
  cuuint64_t dims[2] = {(cuuint64_t)sh::W, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(sh::W * 2)};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_decode_sh(const DecodeArgs& a, cudaStream_t st) {
  const CacheView& cv = a.cache;
  sh::Params prm;
  prm.block_table = cv.block_table;
  prm.seq_lens = a.seq_lens;
  prm.H = a.n_heads;
  prm.max_pages = cv.max_pages;
  prm.num_pages = cv.num_pages;
  prm.batch = a.batch;
  prm.s_q = a.s_q;
  prm.causal = a.causal;
  prm.scale_log2 = a.scale * 1.4426950408889634f;
  prm.o_lat = reinterpret_cast<__nv_bfloat16*>(a.o_lat);
  prm.lse = a.lse;
  prm.o_part = a.o_part;
  prm.lse_part = a.lse_part;
  prm.err = a.err;
  prm.n_workers = max(1, SH_PLAN_WORKERS / max(1, a.s_q));
  prm.rowinfo = a.rowinfo;
  if ((reinterpret_cast<uintptr_t>(a.o_lat) & 15) || (reinterpret_cast<uintptr_t>(a.o_part) & 15))
    return kUnsupported;
  const long rows = (long)a.batch * a.s_q;
  if (rows == 0) return cudaSuccess;
  CUtensorMap m_q, m_kv;
  if (!make_map_sh(&m_q, a.q, (uint64_t)rows * a.n_heads, sh::HP) ||
      !make_map_sh(&m_kv, cv.rows, (uint64_t)cv.num_pages * 64, sh::TS))
    return kUnsupported;
  cudaError_t e = cudaFuncSetAttribute(sh::decode_sh_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, sh::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  sh::decode_sh_kernel<<<dim3((unsigned)(prm.n_workers * a.s_q)), sh::NTHREADS, sh::SMEM_BYTES, st>>>(m_q, m_kv, prm);
  note_launch();
  e = cudaGetLastError();
  return e == cudaSuccess ? launch_plan_combine(a, st) : e;
}

}  // namespace mla
