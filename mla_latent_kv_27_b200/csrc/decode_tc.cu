// Tensor-core (tcgen05 / TMEM) MLA decode over a paged latent cache, up to 128 heads.
//
// What it computes ("DeepSeek-V2 大模型论文原文 PDF" 2.2-2.3; softmax attention of
// intelliparadigm.com 3.3), for one query token (all heads) and one KV chunk:
//   S = (Q_lat C^T + Q_rope K_rope^T) * scale,  online softmax,  O = P C,  lse.
// All heads share one latent cache, so QK^T and PV are dense contractions with the heads as
// the M = 128 dimension of the MMA (fewer heads are padded with zero query rows, whose
// results are discarded).
//
// Mapping onto one SM pair (a cluster of two CTAs, rank r = 0, 1):
//  * An fp32 O of 128 heads x 512 latent dims would fill all 512 TMEM columns, so the pair
//    splits every cached row: CTA r owns latent dims [256r, 256r + 256) and rope dims
//    [32r, 32r + 32).  Each cache byte is loaded once.
//  * CTA r computes the partial S_r = Q_r K_r^T over its 288 dims (tcgen05, fp32 in TMEM),
//    rounds it to fp16 and ships it to its peer over DSMEM (st.async).  Both CTAs form
//    S = f16(S_0) + f16(S_1) with one fp16 add, which is commutative, so both see bit-equal
//    scores and take identical softmax decisions.  (fp16 halves the DSMEM bytes of fp32, and
//    the pair's DSMEM bandwidth is what an fp32 exchange runs out of; the three fp16
//    roundings move a score by at most 2^-11 (|S_0| + |S_1| + |S|).)
//  * Each CTA accumulates its half of O (128 x 256 fp32 = 256 TMEM columns) from P and the
//    latent half it already holds: V = C, so PV needs no further loads.
//  * A tile is one 64-token page.  The cost of a tcgen05.mma of M = 128, K = 16 grows slowly
//    with N, so QK (18 instructions per tile whatever N is) wants a wide token tile.
//  * Q's latent half lives in TMEM as the A operand of QK (staged once through two cache
//    stages).  The rows of Q past H (when H < 128) are the next query rows or TMA's zero fill;
//    their results are never stored.  The peer's partial S of tile i lands in exchange buffer
//    i % 2, the softmax overwrites it with P(i) and PV(i) reads P from there.  An S buffer in
//    TMEM is released as soon as its scores have been read, so QK of tile i+2 does not wait
//    for PV of tile i.
//  * FP8 cache (E4M3 codes + one fp32 scale per token per 128 values; intelliparadigm.com 6.3,
//    "8.1 DeepSeek 架构" section 5): TMA brings the codes, the scales and the bf16 rope key of a
//    page; the exchange warps expand the codes in place, exactly to fp16 and times the scale,
//    into a tile with the layout of a bf16 page, which QK and PV read (fp16 MMAs, fp16 P).
//    The rope part of QK stays a bf16 MMA.  The fp16 path needs |c| and |q| below 65504.
// Roles (704 threads): warp 0 issues TMA loads (Q once, then the cache a page at a time
// through a ring of stages); warp 1 owns TMEM and issues the MMAs from an event loop (QK of tile
// i+1 runs while the softmax of tile i does); warps 2-5 move each partial S from TMEM to the
// peer (and expand FP8 pages); warps 6-21 move Q into TMEM, run the softmax (thread = head
// row = TMEM lane; four groups of four warps split each tile's 64 tokens and swap their
// partial row maxima) and the epilogue.  The O
// rescale is lazy: O is rescaled only when a row's running max grows by more than 2^8, which
// keeps every exponent <= 2^8 and the result exact.
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

constexpr int HM = 128, DC = 512, DR = 64, W = 576;
constexpr int HALF_DC = 256, HALF_DR = 32;
constexpr int TILE = 64;     // tokens per pipeline step: one page
constexpr int NSB = 2;       // S buffers in TMEM
constexpr int NXB = 4;       // exchange buffers (peer scores, then P) in shared memory
constexpr int NG = 4;                       // softmax groups: each takes TILE / NG tokens of a tile
constexpr int GT = TILE / NG;               // 16 tokens per softmax thread per tile
constexpr int NSMW = 4 * NG;                // softmax warps
constexpr int NTHREADS = 32 * (6 + NSMW);   // 704

// shared-memory layout (bytes from a 1024-aligned base)
constexpr int Q_ROPE_OFF = 0;                 // Q rope half: 128 rows x 32 dims, 64B swizzle
constexpr int KV_OFF = HM * HALF_DR * 2;      // 8192
constexpr int LAT_BOX = TILE * 128;           // 8192: 64 tokens x 128 bytes, 128B swizzle
constexpr int ROPE_BOX = TILE * HALF_DR * 2;  // 4096: 64 tokens x 32 dims, 64B swizzle
constexpr int Q_LAT_BOX = HM * 128;           // 16384: 128 rows x 64 dims, 128B swizzle

// A stage holds the page's latent half as 16-bit values in 4 boxes of 64 dims, then its rope
// half.  bf16: TMA writes both directly.  FP8: TMA writes the codes (2 boxes of 128 codes)
// into boxes 2-3 and the 4 scales of each token after the rope half; the expansion then
// overwrites boxes 0-3 with fp16 values.
template <bool FP8> struct Cfg {
  static constexpr int NS = 4;  // cache stages
  static constexpr int CODE_OFF = 2 * LAT_BOX;
  static constexpr int ROPE_OFF = 4 * LAT_BOX;
  static constexpr int SCALE_OFF = ROPE_OFF + ROPE_BOX;
  static constexpr int STAGE = SCALE_OFF + (FP8 ? TILE * 16 : 0);  // 36864 / 37888
  static constexpr uint32_t STAGE_TX = FP8 ? 2 * LAT_BOX + ROPE_BOX + TILE * 16 : STAGE;
  // Q's latent half (4 boxes of 16 KB) is staged two boxes per stage in the stages that tiles 2
  // and 3 of the segment will use, moved to TMEM, and only then are those stages filled.
  // Exchange buffers: the peer's partial S of tile i arrives in buffer i % NXB (128 rows x 64
  // fp16), the softmax reads it and then overwrites it with P(i) (128 x 64, 16-bit), which
  // PV(i) reads.  Both use the 128-byte row swizzle (16-byte chunk c of row r at c ^ (r & 7)).
  // The peer may send tile i + NXB only after PV(i) has completed here.
  static constexpr int XB_OFF = KV_OFF + NS * STAGE;
  static constexpr int XB_BUF = HM * TILE * 2;                       // 16384
  static constexpr int MX_OFF = XB_OFF + NXB * XB_BUF;               // group max swap, row sums
  static constexpr int BAR_OFF = MX_OFF + NSB * NG * HM * 4;
  static constexpr int SMEM_BYTES = BAR_OFF + 512 + 1024;            // barriers + alignment slack
  static_assert(STAGE % 1024 == 0, "1024-aligned stages");
  static_assert(STAGE >= 2 * Q_LAT_BOX, "two Q boxes fit one stage");
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
};
constexpr uint32_t Q_BYTES = 4 * Q_LAT_BOX + HM * HALF_DR * 2;  // 73728
constexpr uint32_t TMEM_COLS = 512;
// TMEM: O half in cols [0, 256); S buffers 2 x 64 columns from 256; Q's latent half, the A
// operand of QK, in cols [384, 512) (256 16-bit values per row, two per 32-bit column).
constexpr uint32_t TM_O = 0, TM_S = 256, TM_Q = 384;
static_assert(TM_S + NSB * TILE <= TM_Q && TM_Q + HALF_DC / 2 <= TMEM_COLS, "TMEM budget");

// Which tokens a unit attends: [lo, hi) of sequence b for query token j (row qrow = b s_q + j);
// a partial result goes to slot `slot`, a complete one (final_out) straight to o_lat / lse.
struct Unit {
  int b, j, lo, hi, qrow, slot, final_out, valid;
};

// Barriers of per-tile events that a waiter might otherwise see two phases late are indexed by
// exchange buffer, which no producer can lap (tile i + NXB needs PV(i) done on both CTAs).
struct Bars {
  uint64_t kv_full[4], kv_empty[4], x_full[4];
  uint64_t q_full, q_moved;
  uint64_t s_full[NSB], s_free[NSB], mx_full[NSB];
  uint64_t p_full[NXB], pv_done[NXB], recv_full[NXB], peer_free[NXB];
  uint64_t l_full;
  uint32_t tmem_base;
  int abort_flag;
  Unit unit, next;  // the segment being processed and the one after it
};
static_assert(sizeof(Bars) <= 512, "barrier block");

struct Params {
  const int32_t* block_table;
  const int32_t* seq_lens;
  int H;
  int max_pages, num_pages;
  int batch, s_q, causal, n_split;
  float scale_log2;  // scale * log2(e)
  __nv_bfloat16* o_lat;
  float* lse;
  float* o_part;
  float* lse_part;
  int* err;
  int plan;          // 1: length-balanced segments, 0: n_split equal page ranges per row
  int n_workers;     // plan: equal page ranges of the concatenated rows
  int32_t* rowinfo;  // plan: [rows][2] first / last slot of each row (-1: no pages)
};

__device__ __forceinline__ void fail(Bars* bars, int* err, int where) {
  record_error(err, ERR_TIMEOUT, where);
  atomicExch(&bars->abort_flag, 1);
}
__device__ __forceinline__ bool aborted(Bars* bars) {
  return *reinterpret_cast<volatile int*>(&bars->abort_flag) != 0;
}


// Tokens row r attends (its cached length; with the causal mask, up to its own position).
__device__ __forceinline__ int attended(const Params& p, int r, bool report) {
  const int j = r % p.s_q;
  int L = p.seq_lens[r / p.s_q];
  if (L < 0 || L > p.max_pages * 64) {
    if (report && j == 0) record_error(p.err, ERR_POS, L);
    L = max(0, min(L, p.max_pages * 64));
  }
  return p.causal ? max(0, min(L, L - p.s_q + j + 1)) : L;
}

// n_split equal page ranges per row: unit = (row, split).
__device__ __forceinline__ Unit make_unit(const Params& p, int unit, bool report) {
  Unit u;
  const int split = unit % p.n_split;
  u.qrow = unit / p.n_split;
  u.j = u.qrow % p.s_q;
  u.b = u.qrow / p.s_q;
  const int A = attended(p, u.qrow, report && split == 0);
  const int pages = (A + 63) / 64;
  const int pps = (pages + p.n_split - 1) / p.n_split;
  u.lo = min(A, split * pps * 64);
  u.hi = min(A, (split + 1) * pps * 64);
  u.slot = (u.b * p.n_split + split) * p.s_q + u.j;
  u.final_out = p.n_split == 1;
  u.valid = 1;
  return u;
}

// Length-balanced partition.  Each row with pages costs its pages plus ROW_COST: a segment
// boundary drains and refills the pipeline, about as long as that many pages.  The rows' costs,
// concatenated in row order (T in all), are cut into U = min(n_workers, T) equal ranges; worker w
// (one cluster, launched once per SM pair) takes range [wT/U, (w+1)T/U) and walks it row by row.
// Within row r the first ROW_COST units stand for the boundary and the pages follow; every row
// whose pages meet the range is one segment.  Segment (w, r) writes partial slot c = w + r.
// Along the concatenation the segments form a staircase on which w + r grows by one per step,
// so each slot has one writer and row r owns the consecutive slots [first(r) + r, last(r) + r],
// first / last the workers that hold its first and last page.  The helpers below are warp-
// collective (warp 0 of every CTA; both CTAs of a cluster derive the same plan from the lengths).
constexpr int ROW_COST = 6;

struct Plan {
  long long T, U;   // total cost; ranges in use
  long long w0, w1; // this worker's cost range
  long long S;      // cost offset of the cursor row
  int r;            // cursor row
  bool done;
};

__device__ __forceinline__ int row_pages(const Params& p, int r, bool report) {
  return (attended(p, r, report) + 63) / 64;
}
__device__ __forceinline__ int row_cost(int pages) { return pages > 0 ? pages + ROW_COST : 0; }

__device__ long long total_cost(const Params& p, int lane) {
  const int R = p.batch * p.s_q;
  long long T = 0;
  for (int r0 = 0; r0 < R; r0 += 32) {
    int c = r0 + lane < R ? row_cost(row_pages(p, r0 + lane, false)) : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    T += c;
  }
  return T;
}

__device__ __forceinline__ long long worker_of(long long x, long long T, long long U) {
  return ((x + 1) * U + T - 1) / T - 1;  // the worker whose range holds cost unit x
}

// Each row's slot range for the combine (-1 for a row without pages); also the one place that
// reports an out-of-range sequence length.
__device__ void write_rowinfo(const Params& p, long long T, long long U, int lane) {
  const int R = p.batch * p.s_q;
  long long S = 0;
  for (int r0 = 0; r0 < R; r0 += 32) {
    const int r = r0 + lane;
    const int pr = r < R ? row_pages(p, r, true) : 0;
    const int cr = row_cost(pr);
    int incl = cr;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const long long first = S + incl - cr + ROW_COST;  // cost unit of the row's first page
    if (r < R) {
      int c0 = -1, c1 = -1;
      if (pr > 0) {
        c0 = (int)worker_of(first, T, U) + r;
        c1 = (int)worker_of(first + pr - 1, T, U) + r;
      }
      p.rowinfo[2 * r] = c0;
      p.rowinfo[2 * r + 1] = c1;
    }
    S += __shfl_sync(0xffffffffu, incl, 31);
  }
}

// Position worker w's cursor on the first row whose cost range reaches past its start.
__device__ void plan_begin(const Params& p, Plan& pl, int w, int lane) {
  pl.T = total_cost(p, lane);
  pl.U = min((long long)p.n_workers, pl.T);
  pl.done = w >= pl.U;
  if (pl.done) return;
  pl.w0 = w * pl.T / pl.U;
  pl.w1 = (w + 1) * pl.T / pl.U;
  const int R = p.batch * p.s_q;
  long long S = 0;
  for (int r0 = 0; r0 < R; r0 += 32) {
    const int r = r0 + lane;
    const int cr = r < R ? row_cost(row_pages(p, r, false)) : 0;
    int incl = cr;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const long long st = S + incl - cr;
    const unsigned m = __ballot_sync(0xffffffffu, cr > 0 && st + cr > pl.w0);
    if (m) {
      const int f = __ffs(m) - 1;
      pl.r = __shfl_sync(0xffffffffu, r, f);
      pl.S = __shfl_sync(0xffffffffu, st, f);
      return;
    }
    S += __shfl_sync(0xffffffffu, incl, 31);
  }
  pl.done = true;
}

// The next segment of worker w (rows whose pages meet its range), advancing the cursor.
__device__ Unit plan_next(const Params& p, Plan& pl, int w, int lane) {
  Unit u = {0, 0, 0, 0, 0, 0, 0, 0};
  const int R = p.batch * p.s_q;
  while (!pl.done && pl.S < pl.w1) {
    const int r = pl.r;
    const int A = attended(p, r, false), pr = (A + 63) / 64;
    const long long first = pl.S + ROW_COST;
    const long long g0 = max(pl.w0, first), g1 = min(pl.w1, first + pr);
    const bool hit = g1 > g0;
    if (hit) {
      u.b = r / p.s_q;
      u.j = r % p.s_q;
      u.qrow = r;
      u.lo = (int)(g0 - first) * 64;
      u.hi = min(A, (int)(g1 - first) * 64);
      u.slot = w + r;
      u.final_out = (g0 == first && g1 == first + pr) ? 1 : 0;
      u.valid = 1;
    }
    // move the cursor to the next row with pages
    pl.S += row_cost(pr);
    pl.done = true;
    if (pl.S < pl.w1) {
      for (int r0 = r + 1; r0 < R; r0 += 32) {
        const int rr = r0 + lane;
        const unsigned m = __ballot_sync(0xffffffffu, rr < R && row_pages(p, rr, false) > 0);
        if (m) {
          pl.r = r0 + __ffs(m) - 1;
          pl.done = false;
          break;
        }
      }
    }
    if (hit) return u;
  }
  pl.done = true;
  return u;
}

// bf16 pair -> fp16 pair, saturating to the fp16 range
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
  const float lo = fminf(fmaxf(__uint_as_float(w << 16), -65504.f), 65504.f);
  const float hi = fminf(fmaxf(__uint_as_float(w & 0xFFFF0000u), -65504.f), 65504.f);
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// four E4M3 codes (little-endian in w) -> two fp16 pairs, each times s
__device__ __forceinline__ void e4m3x4_to_f16(uint32_t w, __half2 s, uint32_t& lo, uint32_t& hi) {
  __half2_raw a = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w & 0xFFFFu), __NV_E4M3);
  __half2_raw b = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w >> 16), __NV_E4M3);
  const __half2 x = __hmul2(*reinterpret_cast<__half2*>(&a), s);
  const __half2 y = __hmul2(*reinterpret_cast<__half2*>(&b), s);
  lo = *reinterpret_cast<const uint32_t*>(&x);
  hi = *reinterpret_cast<const uint32_t*>(&y);
}

template <bool FP8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NTHREADS, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_q_lat, const __grid_constant__ CUtensorMap tm_q_rope,
                     const __grid_constant__ CUtensorMap tm_lat, const __grid_constant__ CUtensorMap tm_rope,
                     const __grid_constant__ CUtensorMap tm_scale, const Params p) {
  using C = Cfg<FP8>;
  constexpr int NS = C::NS;
  constexpr int XB_OFF = C::XB_OFF, XB_BUF = C::XB_BUF, MX_OFF = C::MX_OFF;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + C::BAR_OFF);
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int unit = blockIdx.x / 2;
  Plan pl;  // warp 0 only
  if (p.plan && warp == 0) {
    plan_begin(p, pl, unit, lane);
    if (unit == 0 && rank == 0) write_rowinfo(p, pl.T, max(pl.U, 1ll), lane);
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);  // released by PV
      mbar_init(&bars->x_full[s], 4);    // FP8: the 4 expanding warps are done
    }
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_moved, NSMW);
    for (int b = 0; b < NSB; ++b) {
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->s_free[b], 4 + NSMW);  // the exchange and softmax warps have read S
      mbar_init(&bars->mx_full[b], NSMW);
    }
    for (int b = 0; b < NXB; ++b) {
      mbar_init(&bars->p_full[b], NSMW);
      mbar_init(&bars->pv_done[b], 1);
      mbar_init(&bars->recv_full[b], 1);
      mbar_init(&bars->peer_free[b], 4);
    }
    mbar_init(&bars->l_full, NSMW);
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

  // Segment loop: one segment with n_split ranges per row, a worker's whole page range in the
  // balanced partition.  Barrier phases run on across segments (gb = tiles, seg = segments
  // done); both CTAs drain every segment before the next one starts.
  int gb = 0, seg = 0;
  // Warp 0 plans one segment ahead, so the producer can pull the next segment's Q and first
  // pages into L2 while this one drains.
  if (warp == 0) {
    const Unit f = p.plan ? plan_next(p, pl, unit, lane) : make_unit(p, unit, rank == 0 && lane == 0);
    if (lane == 0) bars->next = f;
  }
  for (;;) {
  if (warp == 0) {
    __syncwarp();
    const Unit t = bars->next;
    Unit t2 = {0, 0, 0, 0, 0, 0, 0, 0};
    if (t.valid && p.plan) t2 = plan_next(p, pl, unit, lane);
    __syncwarp();
    if (lane == 0) {
      bars->unit = t;
      bars->next = t2;
    }
  }
  __syncthreads();
  const Unit u = bars->unit;
  if (!u.valid) break;
  const int n_tiles = (u.hi - u.lo + TILE - 1) / TILE;
  const int32_t* bt = p.block_table + (long)u.b * p.max_pages;
  const uint32_t sph = seg & 1;  // phase parity of the once-per-segment barriers
  // Q staging box jb (0..3): stage of the segment's tile 2 + jb / 2, box jb % 2 within it
  auto q_box = [&](int jb) -> uint8_t* {
    return smem + KV_OFF + ((gb + 2 + (jb >> 1)) % NS) * C::STAGE + (jb & 1) * Q_LAT_BOX;
  };

  if (n_tiles > 0) {
    if (warp == 0) {
      // ------------------------------------------------------------ TMA producer
      if (lane == 0) {
        prefetch_tmap(&tm_lat);
        prefetch_tmap(&tm_rope);
        if (FP8) prefetch_tmap(&tm_scale);
        mbar_arrive_expect_tx(&bars->q_full, Q_BYTES);
        const int qy = u.qrow * p.H;
        for (int jb = 0; jb < 4; ++jb)
          tma_load_2d(q_box(jb), &tm_q_lat, (int)rank * HALF_DC + jb * 64, qy,
                      &bars->q_full);
        tma_load_2d(smem + Q_ROPE_OFF, &tm_q_rope, DC + (int)rank * HALF_DR, qy, &bars->q_full);
        // Pages reach L2 one ring ahead of their stage, so a stage refill (which waits for PV of
        // the tile NS earlier) costs an L2 read, not a DRAM round trip.
        // Page ids are read one tile ahead, so their global-load latency overlaps the waits.
        auto page_of = [&](int i) -> int { return i < n_tiles ? bt[(u.lo + i * TILE) / 64] : -1; };
        auto prefetch = [&](int page) {
          if (page < 0 || page >= p.num_pages) return;
          const int y = page * 64;
          if (FP8) {
            for (int k = 0; k < 2; ++k) tma_prefetch_l2_2d(&tm_lat, (int)rank * HALF_DC + k * 128, y);
            tma_prefetch_l2_2d(&tm_rope, (int)rank * HALF_DR, y);
            tma_prefetch_l2_2d(&tm_scale, 0, y);
          } else {
            for (int jb = 0; jb < 4; ++jb) tma_prefetch_l2_2d(&tm_lat, (int)rank * HALF_DC + jb * 64, y);
            tma_prefetch_l2_2d(&tm_rope, DC + (int)rank * HALF_DR, y);
          }
        };
        int page_cur = page_of(0), page_pf = page_of(NS);
        int issued = 0;  // tiles whose loads were issued (the loop may stop early on an abort)
        for (int i = 0; i < n_tiles; ++i) {
          const int g = gb + i, s = g % NS;
          if (g >= NS && !mbar_wait(&bars->kv_empty[s], ((g / NS) - 1) & 1)) {
            fail(bars, p.err, 1);
            break;
          }
          if (i == 2 && !mbar_wait(&bars->q_moved, sph)) {  // the stages of tiles 2, 3 held Q until now
            fail(bars, p.err, 6);
            break;
          }
          if (aborted(bars)) break;
          const int page = page_cur;
          page_cur = page_of(i + 1);
          const bool bad = page < 0 || page >= p.num_pages;
          if (bad && rank == 0) record_error(p.err, ERR_PAGE, page);
          // a bad page reads TMA's zero fill (rows past the end); the softmax masks its tokens
          const int y = bad ? p.num_pages * 64 : page * 64;
          uint8_t* st = smem + KV_OFF + s * C::STAGE;
          mbar_arrive_expect_tx(&bars->kv_full[s], C::STAGE_TX);
          if (FP8) {
            for (int k = 0; k < 2; ++k)
              tma_load_2d(st + C::CODE_OFF + k * LAT_BOX, &tm_lat, (int)rank * HALF_DC + k * 128, y,
                          &bars->kv_full[s]);
            tma_load_2d(st + C::ROPE_OFF, &tm_rope, (int)rank * HALF_DR, y, &bars->kv_full[s]);
            tma_load_2d(st + C::SCALE_OFF, &tm_scale, 0, y, &bars->kv_full[s]);
          } else {
            for (int jb = 0; jb < 4; ++jb)
              tma_load_2d(st + jb * LAT_BOX, &tm_lat, (int)rank * HALF_DC + jb * 64, y, &bars->kv_full[s]);
            tma_load_2d(st + C::ROPE_OFF, &tm_rope, DC + (int)rank * HALF_DR, y, &bars->kv_full[s]);
          }
          issued = i + 1;
          prefetch(page_pf);  // tile i + NS
          page_pf = page_of(i + NS + 1);
        }
        const Unit nxt = bars->next;
        if (nxt.valid) {  // the next segment's Q rows and first pages, into L2
          const int nqy = nxt.qrow * p.H;
          for (int jb = 0; jb < 4; ++jb) tma_prefetch_l2_2d(&tm_q_lat, (int)rank * HALF_DC + jb * 64, nqy);
          tma_prefetch_l2_2d(&tm_q_rope, DC + (int)rank * HALF_DR, nqy);
          const int32_t* nbt = p.block_table + (long)nxt.b * p.max_pages;
          for (int k = 0; k < NS && nxt.lo + k * TILE < nxt.hi; ++k) prefetch(nbt[(nxt.lo + k * TILE) / 64]);
        }
        // drain: every load still in flight lands before the CTA may exit
        for (int i = max(0, issued - NS); i < issued; ++i)
          if (!mbar_wait(&bars->kv_full[(gb + i) % NS], ((gb + i) / NS) & 1)) break;
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        constexpr uint32_t ID_QK = FP8 ? idesc_f16(128, TILE, 0, 0) : idesc_bf16(128, TILE, 0, 0);
        constexpr uint32_t ID_QR = idesc_bf16(128, TILE, 0, 0);
        constexpr uint32_t ID_PV = FP8 ? idesc_f16(128, HALF_DC, 0, 1) : idesc_bf16(128, HALF_DC, 0, 1);
        const uint32_t q_base = smem_addr(smem);
        bool ok = mbar_wait(&bars->q_full, sph) && mbar_wait(&bars->q_moved, sph);
        if (!ok) fail(bars, p.err, 2);
        // i, jt: tile index within the segment; g = gb + i for the rings and barrier phases
        auto lat_tile = [&](int g) -> uint32_t { return smem_addr(smem + KV_OFF + (g % NS) * C::STAGE); };
        auto issue_qk = [&](int i) {
          const int g = gb + i, s = g % NS, b = g % NSB;
          tc_fence_after();
          const uint32_t lat = lat_tile(g);
          const uint32_t rope = smem_addr(smem + KV_OFF + s * C::STAGE + C::ROPE_OFF);
          const uint32_t d = tmem + TM_S + b * TILE;
#pragma unroll
          for (int ks = 0; ks < 16; ++ks) {  // latent half: A = Q from TMEM, 16 K-steps of 16
            const uint64_t bd = umma_desc(lat + (ks >> 2) * LAT_BOX + (ks & 3) * 32, 16, 1024, UMMA_SW128);
            mma_bf16_tmem_a(d, tmem + TM_Q + ks * 8, bd, ID_QK, ks > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) {  // rope half (bf16): 2 K-steps of 16
            const uint64_t a = umma_desc(q_base + Q_ROPE_OFF + ks * 32, 16, 512, UMMA_SW64);
            const uint64_t bd = umma_desc(rope + ks * 32, 16, 512, UMMA_SW64);
            mma_bf16(d, a, bd, ID_QR, 1u);
          }
          mma_commit(&bars->s_full[b]);
        };
        auto issue_pv = [&](int jt) {
          const int g = gb + jt, b = g % NXB;
          tc_fence_after();
          const uint32_t p_base = smem_addr(smem + XB_OFF + b * XB_BUF);
          const uint32_t v_base = lat_tile(g);
#pragma unroll
          for (int kt = 0; kt < TILE / 16; ++kt) {
            const uint64_t a = umma_desc(p_base + kt * 32, 16, 1024, UMMA_SW128);
            const uint64_t bdesc = umma_desc(v_base + kt * 2048, LAT_BOX, 1024, UMMA_SW128);
            mma_bf16(tmem + TM_O, a, bdesc, ID_PV, (jt > 0 || kt > 0) ? 1u : 0u);
          }
          mma_commit(&bars->pv_done[b]);
          mma_commit(&bars->kv_empty[g % NS]);
        };
        // Event loop: QK(j) as soon as its page is loaded (and expanded) and S buffer j%2 has
        // been read by the exchange and softmax warps (tile j-2); PV(k) as soon as P(k) is in
        // shared memory.
        int qk = 0, pv = 0;
        uint64_t t_idle = 0;
        uint32_t spins = 0;
        while (ok && pv < n_tiles) {
          const int gp = gb + pv, gq = gb + qk;
          if (pv < qk && mbar_test(&bars->p_full[gp % NXB], (gp / NXB) & 1)) {
            issue_pv(pv++);
            t_idle = 0;
            continue;
          }
          if (qk < n_tiles && mbar_test(&bars->kv_full[gq % NS], (gq / NS) & 1) &&
              (!FP8 || mbar_test(&bars->x_full[gq % NS], (gq / NS) & 1)) &&
              (gq < NSB || mbar_test(&bars->s_free[gq % NSB], ((gq / NSB) - 1) & 1))) {
            issue_qk(qk++);
            t_idle = 0;
            continue;
          }
          if ((++spins & 63u) == 0) {
            const uint64_t now = globaltimer_ns();
            if (t_idle == 0) t_idle = now;
            else if (now - t_idle > 2000000000ull) {
              fail(bars, p.err, 3);
              ok = false;
            }
            if (aborted(bars)) ok = false;
          }
        }
      }
    } else if (warp < 6) {
      // ------------------------------------------------------------ score exchange (+ FP8 expansion)
      // TMEM partial S -> fp16 -> the peer's receive buffer (st.async).
      const int quarter = warp & 3;
      const int row = quarter * 32 + lane;
      const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
      const int swz = row & 7;
      // FP8: expand page i in place: fp16 (code * scale) into latent boxes 0-3 of its stage,
      // zeros for the tokens the unit does not attend (stale slots may hold any byte).  Warp
      // w owns tokens [16w, 16w + 16) whole: an item is (token t, code box k, 16-code chunk
      // c), and its fp16 output lands over codes of the same token only, so the warp reads
      // all of its items before it writes any.
      auto expand = [&](int i) -> bool {
        const int g = gb + i, s = g % NS;
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->kv_full[s], (g / NS) & 1))) return false;
        const int t0 = u.lo + i * TILE;
        const int page = bt[t0 / 64];
        const int lim = (page >= 0 && page < p.num_pages) ? min(TILE, u.hi - t0) : 0;
        uint8_t* st = smem + KV_OFF + s * C::STAGE;
        const float* sc = reinterpret_cast<const float*>(st + C::SCALE_OFF);
        const int c = lane & 7, k = (lane >> 3) & 1;
        uint4 raw[8];
        float scl[8];
#pragma unroll
        for (int it = 0; it < 8; ++it) {
          const int t = 16 * quarter + 2 * it + (lane >> 4);
          raw[it] = *reinterpret_cast<const uint4*>(st + C::CODE_OFF + k * LAT_BOX + t * 128 + ((c ^ (t & 7)) << 4));
          scl[it] = t < lim ? sc[t * 4 + 2 * (int)rank + k] : 0.f;
        }
        __syncwarp();
#pragma unroll
        for (int it = 0; it < 8; ++it) {
          const int t = 16 * quarter + 2 * it + (lane >> 4);
          uint4 o0 = make_uint4(0, 0, 0, 0), o1 = make_uint4(0, 0, 0, 0);
          if (t < lim) {
            const __half2 s2 = __float2half2_rn(scl[it]);
            e4m3x4_to_f16(raw[it].x, s2, o0.x, o0.y);
            e4m3x4_to_f16(raw[it].y, s2, o0.z, o0.w);
            e4m3x4_to_f16(raw[it].z, s2, o1.x, o1.y);
            e4m3x4_to_f16(raw[it].w, s2, o1.z, o1.w);
          }
          // dims 128k + 16c .. +15 of the CTA's half: box 2k + c/4, 16-byte chunks 2(c%4), +1
          uint8_t* vrow = st + (2 * k + (c >> 2)) * LAT_BOX + t * 128;
          const int cc = 2 * (c & 3);
          *reinterpret_cast<uint4*>(vrow + ((cc ^ (t & 7)) << 4)) = o0;
          *reinterpret_cast<uint4*>(vrow + (((cc + 1) ^ (t & 7)) << 4)) = o1;
        }
        fence_proxy_async_smem();  // the tile is read by the MMA (async proxy)
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->x_full[s]);
        return true;
      };
      bool xok = true;
      // The peer's scores of this segment's first tile go to buffer gb % NXB, whose previous
      // occupant was consumed by PV before the segment boundary: free it for the peer.
      if (gb >= NXB) {
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster_relaxed(&bars->peer_free[gb % NXB], peer);
      }
      if (FP8) {
        for (int i = 0; i < min(2, n_tiles); ++i)
          if (!expand(i)) {
            fail(bars, p.err, 20);
            xok = false;
            break;
          }
      }
      for (int i = 0; xok && i < n_tiles; ++i) {
        const int g = gb + i;
        const int b = g % NXB, use = g / NXB;       // exchange buffer
        const int sb = g % NSB, suse = g / NSB;     // S buffer
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[sb], suse & 1))) {
          fail(bars, p.err, 10);
          break;
        }
        tc_fence_after();
        // read the partial S, round it to fp16 and release the S buffer at once
        uint32_t packed[32];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t sraw[32];
          tmem_ld32(tmem + lane_off + TM_S + sb * TILE + h * 32, sraw);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            __half2 h2 = __floats2half2_rn(__uint_as_float(sraw[2 * c]), __uint_as_float(sraw[2 * c + 1]));
            packed[16 * h + c] = *reinterpret_cast<uint32_t*>(&h2);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_free[sb]);
        // Exchange buffer b holds P(g - NXB) at the peer until the peer's PV(g - NXB) has
        // completed; the peer says so through peer_free[b] (sent a tile ahead, below).
        if (g >= NXB && !__all_sync(0xffffffffu, mbar_wait<true>(&bars->peer_free[b], (use - 1) & 1))) {
          fail(bars, p.err, 15);
          break;
        }
        if (threadIdx.x == 64) mbar_arrive_expect_tx(&bars->recv_full[b], XB_BUF);
        const uint32_t remote_row = map_to_rank(smem + XB_OFF + b * XB_BUF + row * (TILE * 2), peer);
        const uint32_t remote_bar = map_to_rank(&bars->recv_full[b], peer);
#pragma unroll
        for (int c = 0; c < 8; ++c)
          st_async_v4(remote_row + (c ^ swz) * 16,
                      make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]), remote_bar);
        // Free this CTA's buffer for the peer's scores of tile i+1 once its previous occupant,
        // P(i+1 - NXB), has been consumed by PV here.  The MMA completion (pv_done) orders
        // every earlier access to the buffer before this signal, so it can be relaxed.
        if (g + 1 >= NXB && i + 1 < n_tiles) {
          const int j = g + 1 - NXB;
          if (!__all_sync(0xffffffffu, mbar_wait(&bars->pv_done[j % NXB], (j / NXB) & 1))) {
            fail(bars, p.err, 11);
            break;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster_relaxed(&bars->peer_free[(g + 1) % NXB], peer);
        }
        if (FP8 && i + 2 < n_tiles && !expand(i + 2)) {
          fail(bars, p.err, 21);
          break;
        }
      }
    } else {
      // ------------------------------------------------------------ softmax + epilogue
      // NG groups of 4 warps: group g takes token columns [GT g, GT g + GT) of every tile for
      // all 128 rows (the group's warps cover the four TMEM lane quarters).  The groups swap
      // their partial row maxima through shared memory each tile and keep separate partial
      // row sums; group g also owns O columns [64 g, 64 g + 64) for rescales and the epilogue.
      const int quarter = warp & 3;          // TMEM lane quarter this warp may access
      const int grp = (warp - 6) >> 2;       // token slice of the tile
      const int row = quarter * 32 + lane;   // head
      const bool hv = row < p.H;             // rows past H are never stored
      const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
      const int swz = row & 7;
      constexpr int OC = HALF_DC / NG;       // O columns per group
      float* mx_buf = reinterpret_cast<float*>(smem + MX_OFF);  // [NSB][NG][H]
      // Move this row's Q latent dims [64 g, 64 g + 64) of the CTA's 256 from the 128B-swizzled
      // staging box g into TMEM as 16-bit pairs along K (fp16 for FP8 pages).
      {
        bool qok = __all_sync(0xffffffffu, mbar_wait(&bars->q_full, sph));
        if (!qok) fail(bars, p.err, 19);
        uint32_t qv[32];
        const uint8_t* box = q_box(grp) + row * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v = *reinterpret_cast<const uint4*>(box + ((c ^ (row & 7)) * 16));
          qv[4 * c] = FP8 ? bf16x2_to_f16x2(v.x) : v.x;
          qv[4 * c + 1] = FP8 ? bf16x2_to_f16x2(v.y) : v.y;
          qv[4 * c + 2] = FP8 ? bf16x2_to_f16x2(v.z) : v.z;
          qv[4 * c + 3] = FP8 ? bf16x2_to_f16x2(v.w) : v.w;
        }
        tmem_st32(tmem + lane_off + TM_Q + grp * 32, qv);
        tmem_wait_st();
        fence_proxy_async_smem();  // staging reads done before TMA refills those stages
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->q_moved);
      }
      float m_used = -INFINITY, l_sum = 0.f;
      int page_next = bt[u.lo / 64];  // page of tile 0; tile i+1's is fetched during tile i
      bool ok = true;
      for (int i = 0; i < n_tiles; ++i) {
        const int g = gb + i;
        const int b = g % NXB, use = g / NXB;       // exchange buffer
        const int sb = g % NSB, suse = g / NSB;     // S buffer
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[sb], suse & 1))) {
          fail(bars, p.err, 12);
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sr[GT];
        tmem_ld16(tmem + lane_off + TM_S + sb * TILE + grp * GT, sr);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_free[sb]);
        if (!__all_sync(0xffffffffu, mbar_wait<true>(&bars->recv_full[b], use & 1))) {
          fail(bars, p.err, 13);
          ok = false;
          break;
        }
        const int t0 = u.lo + i * TILE;
        const int page = page_next;
        if (i + 1 < n_tiles) page_next = bt[(t0 + TILE) / 64];
        const int lim = (page >= 0 && page < p.num_pages) ? min(TILE, u.hi - t0) - grp * GT : 0;
        // S = f16(S_own) + f16(S_peer), added in fp16 (a commutative IEEE add, so both CTAs get
        // bit-equal scores), max taken on the raw sums
        __half2 xs[GT / 2];
        {
          const uint8_t* peer_row = smem + XB_OFF + b * XB_BUF + row * (TILE * 2);
#pragma unroll
          for (int c = 0; c < GT / 8; ++c) {
            const uint4 vp = *reinterpret_cast<const uint4*>(peer_row + (((GT / 8) * grp + c) ^ swz) * 16);
            const uint32_t wp[4] = {vp.x, vp.y, vp.z, vp.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int e = 8 * c + 2 * k;
              xs[4 * c + k] = __hadd2(__floats2half2_rn(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1])),
                                      *reinterpret_cast<const __half2*>(&wp[k]));
            }
          }
        }
        if (lim < GT) {
          const __half ninf = __ushort_as_half((unsigned short)0xFC00u);
#pragma unroll
          for (int c = 0; c < GT / 2; ++c) {
            if (2 * c >= lim) xs[c].x = ninf;
            if (2 * c + 1 >= lim) xs[c].y = ninf;
          }
        }
        __half2 hm = xs[0];
#pragma unroll
        for (int c = 1; c < GT / 2; ++c) hm = __hmax2(hm, xs[c]);
        // swap partial maxima with the other groups
        mx_buf[(sb * NG + grp) * HM + row] = fmaxf(__low2float(hm), __high2float(hm));
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->mx_full[sb]);
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->mx_full[sb], suse & 1))) {
          fail(bars, p.err, 17);
          ok = false;
          break;
        }
        float m_raw = mx_buf[(sb * NG) * HM + row];
#pragma unroll
        for (int k = 1; k < NG; ++k) m_raw = fmaxf(m_raw, mx_buf[(sb * NG + k) * HM + row]);
        const float m_tile = m_raw * p.scale_log2;
        const float m_new = fmaxf(m_used, m_tile);
        float alpha = 1.f;
        if (m_new > m_used + 8.f) {  // lazy rescale: only when the max grows by more than 2^8
          alpha = ex2_approx(m_used - m_new);
          m_used = m_new;
        }
        // while m_used is still -inf every x is -inf too, and 2^(-inf) = 0
        const float mu = m_used == -INFINITY ? 0.f : m_used;
        float ps0 = 0.f, ps1 = 0.f;
        uint32_t pk[GT / 2];
        const float sc = p.scale_log2;
#pragma unroll
        for (int c = 0; c < GT / 2; ++c) {
          const float2 xf = __half22float2(xs[c]);
          const float p0 = ex2_approx(fmaf(xf.x, sc, -mu)), p1 = ex2_approx(fmaf(xf.y, sc, -mu));
          if (FP8) {
            __half2 ph = __floats2half2_rn(p0, p1);
            pk[c] = *reinterpret_cast<uint32_t*>(&ph);
          } else {
            __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
            pk[c] = *reinterpret_cast<uint32_t*>(&pb);
          }
          ps0 += p0;
          ps1 += p1;
        }
        l_sum = l_sum * alpha + (ps0 + ps1);
        // O may be rescaled only once PV(i-1) has completed.  (The exchange buffer P(i) goes
        // into was released by PV(i - NXB) before the peer's scores of tile i could arrive.)
        const bool need_rescale = __any_sync(0xffffffffu, alpha != 1.f) && i > 0;
        if (need_rescale &&
            !__all_sync(0xffffffffu, mbar_wait(&bars->pv_done[(g - 1) % NXB], ((g - 1) / NXB) & 1))) {
          fail(bars, p.err, 14);
          ok = false;
          break;
        }
        tc_fence_after();
        if (need_rescale) {
#pragma unroll 1
          for (int cb = 0; cb < OC / 32; ++cb) {
            const uint32_t col = TM_O + grp * OC + cb * 32;
            uint32_t o[32];
            tmem_ld32(tmem + lane_off + col, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st32(tmem + lane_off + col, o);
          }
        }
        {  // P row, K-major with 128-byte swizzle: this group's tokens are chunks 2g, 2g + 1
          uint8_t* prow = smem + XB_OFF + b * XB_BUF + row * 128;
#pragma unroll
          for (int c = 0; c < GT / 8; ++c)
            *reinterpret_cast<uint4*>(prow + ((((GT / 8) * grp + c) ^ (row & 7)) * 16)) =
                make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        }
        // bf16 pages: V rows past the valid tokens may hold stale data: zero them so that
        // 0 * garbage = 0.  Warp (quarter q, group g) zeroes latent box q for the token rows of
        // group g.  (FP8 tiles are written with those zeros already.)
        if (!FP8 && lim < GT) {
          uint8_t* box = smem + KV_OFF + (g % NS) * C::STAGE + quarter * LAT_BOX;
          const int first = grp * GT + max(lim, 0);
          for (int e = lane; e < (grp * GT + GT - first) * 8; e += 32)
            *reinterpret_cast<uint4*>(box + (first + e / 8) * 128 + (e % 8) * 16) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();  // P (and any zeroed V rows) visible to the MMA
        if (need_rescale) tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_full[b]);
      }
      // ------------------------------------------------------------ epilogue
      // total row sum = the groups' partial sums, swapped through the max buffer of the parity
      // the last tile did not use (every group has read it before the last tile's swap).
      float* l_buf = mx_buf + ((gb + n_tiles) % NSB) * NG * HM;  // [NG][H]
      l_buf[grp * HM + row] = l_sum;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->l_full);
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->l_full, sph))) {
        fail(bars, p.err, 18);
        ok = false;
      }
      float l_tot = 0.f;
#pragma unroll
      for (int k = 0; k < NG; ++k) l_tot += l_buf[k * HM + row];
      const float inv_l = l_tot > 0.f ? 1.f / l_tot : 0.f;
      const float lse = l_tot > 0.f ? (m_used + log2f(l_tot)) * 0.69314718055994531f : -INFINITY;
      if (ok) {
        const int jt = gb + n_tiles - 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->pv_done[jt % NXB], (jt / NXB) & 1))) {
          fail(bars, p.err, 16);
          ok = false;
        }
        tc_fence_after();
      }
      const long qh = (long)u.qrow * p.H + row;
      const bool final_out = u.final_out != 0;
      const long prow_idx = (long)u.slot * p.H + row;
#pragma unroll 1
      for (int cb = 0; cb < OC / 32; ++cb) {
        const int col = grp * OC + cb * 32;
        uint32_t o[32];
        __syncwarp();
        tmem_ld32(tmem + lane_off + TM_O + col, o);
        tmem_wait_ld();
        const int d0 = (int)rank * HALF_DC + col;
        if (!hv) {
        } else if (final_out) {
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
      if (rank == 0 && grp == 0 && hv) {
        if (final_out) {
          if (p.lse) p.lse[qh] = ok ? lse : -INFINITY;
        } else {
          p.lse_part[prow_idx] = ok ? lse : -INFINITY;
        }
      }
    }
  } else if (warp >= 6) {
    // empty unit: o = 0, lse = -inf (softmax group g clears its rows' columns [64 g, 64 g + 64))
    const int grp = (warp - 6) >> 2;
    const int row = (warp & 3) * 32 + lane;
    if (row < p.H) {
      const long qh = (long)u.qrow * p.H + row;
      const long prow_idx = (long)u.slot * p.H + row;
      for (int d = 0; d < HALF_DC / NG; d += 8) {
        const int d0 = (int)rank * HALF_DC + grp * (HALF_DC / NG) + d;
        if (u.final_out)
          *reinterpret_cast<uint4*>(p.o_lat + qh * DC + d0) = make_uint4(0, 0, 0, 0);
        else {
          reinterpret_cast<float4*>(p.o_part + prow_idx * DC + d0)[0] = make_float4(0.f, 0.f, 0.f, 0.f);
          reinterpret_cast<float4*>(p.o_part + prow_idx * DC + d0)[1] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      if (rank == 0 && grp == 0) {
        if (u.final_out) {
          if (p.lse) p.lse[qh] = -INFINITY;
        } else {
          p.lse_part[prow_idx] = -INFINITY;
        }
      }
    }
  }
  // segment boundary: every role of both CTAs is done with this segment (all loads landed, all
  // MMAs completed, all scores exchanged, O read out)
  gb += n_tiles;
  ++seg;
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  // a CTA that gave up makes its peer stop as well (both read both flags after the barrier)
  if (aborted(bars) || ld_cluster_u32(map_to_rank(&bars->abort_flag, peer)) != 0) break;
  }  // segment loop
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
  cluster_sync();  // no CTA leaves while its peer may still touch its shared memory
}

// Merge the segments of each row of the balanced partition (split-KV by log-sum-exp):
// lse = log sum_s e^{lse_s}, o = sum_s e^{lse_s - lse} o_s.  Rows computed whole by one segment
// were written by the decode kernel; rows with no tokens get o = 0, lse = -inf.
// Block = (row, 8 heads), one warp per head, 16 of the 512 dims per lane.
__global__ void __launch_bounds__(256) combine_plan_kernel(const int32_t* rowinfo, const float* o_part,
                                                           const float* lse_part, int H,
                                                           __nv_bfloat16* o_lat, float* lse) {
  // the next grid (the output projection) may start streaming its weights meanwhile
  griddep_launch_dependents();
  const int r = blockIdx.x, h = blockIdx.y * 8 + threadIdx.x / 32, lane = threadIdx.x % 32;
  if (h >= H) return;
  const int c0 = rowinfo[2 * r], c1 = rowinfo[2 * r + 1];
  if (c0 >= 0 && c0 == c1) return;
  const long qh = (long)r * H + h;
  float m = -INFINITY;
  for (int c = c0; c0 >= 0 && c <= c1; ++c) m = fmaxf(m, lse_part[(long)c * H + h]);
  float4 acc[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  float wsum = 0.f;
  if (m != -INFINITY) {
    for (int c = c0; c <= c1; ++c) {
      const float l = lse_part[(long)c * H + h];
      if (l == -INFINITY) continue;  // empty segment: its o_part is never read
      const float w = expf(l - m);
      wsum += w;
      const float4* src = reinterpret_cast<const float4*>(o_part + ((long)c * H + h) * DC);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float4 v = src[k * 32 + lane];
        acc[k].x += w * v.x;
        acc[k].y += w * v.y;
        acc[k].z += w * v.z;
        acc[k].w += w * v.w;
      }
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  uint2* dst = reinterpret_cast<uint2*>(o_lat + qh * DC);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    __nv_bfloat162 a = __floats2bfloat162_rn(acc[k].x * inv, acc[k].y * inv);
    __nv_bfloat162 b = __floats2bfloat162_rn(acc[k].z * inv, acc[k].w * inv);
    dst[k * 32 + lane] = make_uint2(*reinterpret_cast<uint32_t*>(&a), *reinterpret_cast<uint32_t*>(&b));
  }
  if (lane == 0 && lse) lse[qh] = wsum > 0.f ? m + logf(wsum) : -INFINITY;
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

// 2-D tensor map over `rows` rows of `cols` elements (row pitch cols * elem bytes).
static bool make_map(CUtensorMap* m, CUtensorMapDataType type, uint32_t elem, const void* base, uint64_t cols,
                     uint64_t rows, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw) {
  auto enc = get_encode();
  if (!enc || (reinterpret_cast<uintptr_t>(base) & 15)) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(cols * elem)};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, type, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool tc_decode_supported(const mla_dims& d, int cache_kind) {
  return d.n_heads >= 1 && d.n_heads <= tc::HM && d.d_c == tc::DC && d.d_rope == tc::DR && d.page_size == 64 &&
         d.act_dtype == MLA_BF16 && (cache_kind == MLA_BF16 || cache_kind == MLA_FP8_E4M3);
}

size_t tc_plan_workspace_bytes(const mla_dims& d, int batch, int s_q) {
  const size_t rows = (size_t)batch * s_q, slots = (size_t)TC_PLAN_WORKERS + rows;
  return slots * d.n_heads * (d.d_c + 1) * sizeof(float) + rows * 2 * sizeof(int32_t);
}

template <bool FP8>
static cudaError_t launch_tc(const CUtensorMap& qa, const CUtensorMap& qb, const CUtensorMap& a, const CUtensorMap& b,
                             const CUtensorMap& c, const tc::Params& prm, long units, cudaStream_t st) {
  constexpr int smem = tc::Cfg<FP8>::SMEM_BYTES;
  cudaError_t e = cudaFuncSetAttribute(tc::decode_tc_kernel<FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  tc::decode_tc_kernel<FP8><<<dim3((unsigned)(2 * units)), tc::NTHREADS, smem, st>>>(qa, qb, a, b, c, prm);
  note_launch();
  return cudaGetLastError();
}

static cudaError_t launch_plan_combine(const DecodeArgs& a, cudaStream_t st) {
  const long rows = (long)a.batch * a.s_q;
  tc::combine_plan_kernel<<<dim3((unsigned)rows, (unsigned)((a.n_heads + 7) / 8)), 256, 0, st>>>(
      a.rowinfo, a.o_part, a.lse_part, a.n_heads, reinterpret_cast<__nv_bfloat16*>(a.o_lat), a.lse);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t st) {
  const CacheView& cv = a.cache;
  tc::Params prm;
  prm.block_table = cv.block_table;
  prm.seq_lens = a.seq_lens;
  prm.H = a.n_heads;
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
  prm.plan = a.plan;
  prm.n_workers = TC_PLAN_WORKERS;
  prm.rowinfo = a.rowinfo;
  if ((reinterpret_cast<uintptr_t>(a.q) & 15) || (reinterpret_cast<uintptr_t>(a.o_lat) & 15) ||
      (reinterpret_cast<uintptr_t>(a.o_part) & 15))
    return kUnsupported;
  const long rows = (long)a.batch * a.s_q;
  // balanced partition: one persistent cluster per worker range (one per SM pair)
  const long units = a.plan ? (rows > 0 ? TC_PLAN_WORKERS : 0) : rows * a.n_split;
  const uint64_t kv_rows = (uint64_t)cv.num_pages * 64;
  // Q boxes are 128 rows from row (b * s_q + j) * H: with H < 128 the rows past H belong to
  // the next query rows (or lie past the end, where TMA fills zeros) and are never stored.
  const uint64_t q_rows = (uint64_t)a.batch * a.s_q * a.n_heads;
  CUtensorMap m_q_lat, m_q_rope, m_lat, m_rope, m_scale;
  if (!make_map(&m_q_lat, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.q, tc::W, q_rows, 64, tc::HM,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&m_q_rope, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.q, tc::W, q_rows, tc::HALF_DR, tc::HM,
                CU_TENSOR_MAP_SWIZZLE_64B))
    return kUnsupported;
  if (cv.kind == MLA_FP8_E4M3) {
    if (!make_map(&m_lat, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, cv.rows, tc::DC, kv_rows, 128, tc::TILE,
                  CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&m_rope, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, cv.rope, tc::DR, kv_rows, tc::HALF_DR, tc::TILE,
                  CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_map(&m_scale, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, cv.scales, tc::DC / 128, kv_rows, tc::DC / 128,
                  tc::TILE, CU_TENSOR_MAP_SWIZZLE_NONE))
      return kUnsupported;
    if (units == 0) return cudaSuccess;
    cudaError_t e = launch_tc<true>(m_q_lat, m_q_rope, m_lat, m_rope, m_scale, prm, units, st);
    return e == cudaSuccess && a.plan ? launch_plan_combine(a, st) : e;
  }
  if (!make_map(&m_lat, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, cv.rows, tc::W, kv_rows, 64, tc::TILE,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&m_rope, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, cv.rows, tc::W, kv_rows, tc::HALF_DR, tc::TILE,
                CU_TENSOR_MAP_SWIZZLE_64B))
    return kUnsupported;
  if (units == 0) return cudaSuccess;
  cudaError_t e = launch_tc<false>(m_q_lat, m_q_rope, m_lat, m_rope, m_lat, prm, units, st);
  return e == cudaSuccess && a.plan ? launch_plan_combine(a, st) : e;
}

}  // namespace mla
