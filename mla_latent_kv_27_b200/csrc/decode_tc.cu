// Tensor-core (tcgen05 / TMEM) MLA decode over a paged latent cache, up to 128 heads.
//
// What it computes ("DeepSeek-V2 大模型论文原文 PDF" 2.2-2.3; softmax attention of
// intelliparadigm.com 3.3), for one query token (all heads) and one KV chunk:
//   S = (Q_lat C^T + Q_rope K_rope^T) * scale,  online softmax,  O = P C,  lse.
// All heads share one latent cache, so QK^T and PV are dense contractions with the heads as
// the M = 128 dimension of the MMA (fewer heads are padded with query rows whose results are
// discarded).
//
// Mapping onto one SM pair (a cluster of two CTAs, rank r = 0, 1):
//  * An fp32 O of 128 heads x 512 latent dims would fill all 512 TMEM columns, so the pair
//    splits every cached row: CTA r owns latent dims [256r, 256r + 256) and rope dims
//    [32r, 32r + 32), and each cache byte is loaded once.  CTA r computes the partial scores
//    S_r = Q_r K_r^T over its 288 dims for all 128 heads (tcgen05, fp32 in TMEM) and
//    accumulates its half of O (128 x 256 fp32) from P and the latent half it holds (V = C).
//  * The softmax of a head needs S_0 + S_1.  CTA r owns the softmax of heads [64r, 64r + 64):
//    it sends the peer the fp32 partial scores of the peer's heads (16 KB per page, st.async
//    over DSMEM), adds the ones it receives to its own in fp32 (so the scores are those of an
//    fp32 accumulation over all 576 dims), forms P for its heads and stores those P rows (8 KB)
//    into the peer's P buffer as it writes its own (st.async), so that both CTAs hold P for all
//    128 heads when they run PV.
//  * One thread owns one head row of a page (all 64 tokens): no cross-warp reduction.  The
//    reference maximum m of a row moves lazily: only when a score exceeds it by more than 2^8
//    (log2 units) is m raised and O rescaled; P = 2^(s - m) <= 2^8 otherwise.  The owner
//    rescales its half of O and sends the factor with the P row; the peer applies it to its
//    half before the next PV.  Consecutive pages go to different warps; m is the only state
//    handed from one page to the next.
//  * A tile is one 64-token page.  Q's latent half lives in TMEM as the A operand of QK (staged
//    once per row segment through two stages); the rope half is an A operand in shared memory.
//  * bf16 cache: a page's cache stage feeds QK only and is released when QK completes; its
//    latent half is loaded again, from L2, into a PV stage shortly before PV.  Shared memory
//    then holds a page for its QK and its PV, not through the exchange and softmax between
//    them, and the rings for scores and P rows get the room to be two and three deep.
//  * FP8 cache (E4M3 codes + one fp32 scale per token per 128 values; intelliparadigm.com 6.3,
//    "8.1 DeepSeek 架构" section 5): TMA brings the codes, the scales and the bf16 rope key of a
//    page; the four score-sending warps expand the codes in place, exactly to fp16 and times
//    the scale, into a tile with the layout of a bf16 page, which QK and PV read (fp16 MMAs,
//    fp16 P).  The rope part of QK stays a bf16 MMA.  The fp16 path needs |c| and |q| below
//    65504.
// Roles (512 threads): warps 0-11 are three warps per TMEM lane quarter (a warp reaches the lanes
// of quarter warp % 4, which is also its scheduler).  In the quarters of the CTA's own heads all
// three run the softmax, each on every third page, so that three pages are in flight.  In the
// peer's quarters two warps send the partial scores and one takes the P rows the peer sends (and
// rescales O when asked).  All of them move Q into TMEM and run the epilogue.  Of warps 12-15
// (one per scheduler), the two on the peer quarters' schedulers issue the TMA loads (Q once per
// segment, then the cache a page at a time through a ring of stages) and the MMAs (from an event
// loop that gives PV priority); with a bf16 cache one of the other two loads the PV stages.
// Waiting threads sleep in mbarrier try_wait rather than spin, so the warps that compute keep
// the issue slots.
// Every wait is bounded (2 s); on timeout the kernel records MLA_ERR_TIMEOUT and winds down.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>

#include "mla_internal.cuh"
#include "sm100_ptx.cuh"
#include "decode_tc.cuh"
#include "decode_plan.cuh"

namespace mla {
namespace tc {

using namespace sm100;
using plan::Unit;
using plan::Plan;
constexpr int ROW_COST = 6;  // a segment boundary drains and refills the pipeline: about 6 pages

constexpr int HM = 128, DC = 512, DR = 64, W = 576;
constexpr int HALF_DC = 256, HALF_DR = 32;
constexpr int HO = 64;       // heads whose softmax one CTA of the pair owns
constexpr int TILE = 64;     // tokens per pipeline step: one page
constexpr int NSB = 2;       // partial-score buffers in TMEM
// Ring depths per cache type are in Cfg (cache stages, PV stages, score receive buffers, P
// buffers); the barrier block is sized for the largest.
constexpr int NS_MAX = 4, NV_MAX = 2, NRB_MAX = 2, NPB_MAX = 3;
constexpr int QK_AHEAD = 5;  // QK(j) is issued only while j < (next PV) + QK_AHEAD
constexpr int NROW = 12;     // row warps 0-11: three per TMEM lane quarter (quarter = warp % 4)
// Warps 12-15, one per scheduler (warp % 4): the TMA producer and the MMA issuer on two of the
// peer's lane quarters' schedulers; the other two are spare.  Four warps per scheduler leave 128
// registers per thread.
constexpr int NTHREADS = 32 * (NROW + 4);  // 512
constexpr int NG = 3;        // softmax warps per lane quarter of the CTA's heads (pages g % 3)
// Barriers a softmax warp waits on come in rings of RG = 6 (page g uses slot g % 6): every slot is
// then waited by one warp only, which sees all of its phases in order.  (With two slots a warp that
// skips pages could find a slot two phases away from the one it waits for, where a parity wait
// misreads the phase.)
constexpr int RG = 2 * NG;
static_assert(QK_AHEAD <= RG, "the PV-stage loader's wait on slot g % RG of s6 needs QK(g + RG) after PV(g)");
constexpr float RESCALE_T = 8.f;           // lazy rescale threshold, log2 units

// shared-memory layout (bytes from a 1024-aligned base)
constexpr int Q_ROPE_OFF = 0;                 // Q rope half: 128 rows x 32 dims, 64B swizzle
constexpr int KV_OFF = HM * HALF_DR * 2;      // 8192
constexpr int LAT_BOX = TILE * 128;           // 8192: 64 tokens x 128 bytes, 128B swizzle
constexpr int ROPE_BOX = TILE * HALF_DR * 2;  // 4096: 64 tokens x 32 dims, 64B swizzle
constexpr int Q_LAT_BOX = HM * 128;           // 16384: 128 rows x 64 dims, 128B swizzle
// The peer's partial scores of this CTA's heads: 64 rows x 64 fp32 (256 bytes a row); 16-byte
// chunk c of row o sits at chunk c ^ (o & 15).
constexpr int RECV_BUF = HO * TILE * 4;       // 16384
// P of all 128 heads, K-major with the 128-byte row swizzle (chunk c of row h at c ^ (h & 7)):
// the rows of this CTA's heads written here, the others by the peer.
constexpr int P_BUF = HM * TILE * 2;          // 16384
constexpr uint32_t P_RECV_TX = HO * (TILE * 2 + 4);  // the peer's P rows and their rescale factors

// Barriers of per-tile events are rings indexed by the global tile count g; no producer of a
// barrier can complete it twice before each of its waiters has seen the earlier phase (the
// argument for each is at its use).
struct Bars {
  uint64_t kv_full[NS_MAX], kv_empty[NS_MAX], x_full[NS_MAX];
  uint64_t v_full[NV_MAX], v_empty[NV_MAX];  // PV stages (bf16 pages)
  uint64_t q_full, q_moved;
  uint64_t s_full[NSB], s_free[NSB], s6[RG];
  uint64_t recv6[RG], send_ok[NRB_MAX];
  uint64_t p_recv[NPB_MAX], p_full[NPB_MAX], pv_done[NPB_MAX], p_free[NPB_MAX];
  uint64_t pvs6[RG], pvr6[RG];  // PV done (for the P buffer, for a rescale)
  uint64_t l_full;
  uint64_t hand[2][NG];    // [own quarter][tile % NG]: the reference maximum after that tile is written
  uint32_t sink[4];        // targets of the peer's 4-byte st.async signals (the values are unused)
  uint64_t ls_full[2];     // [own quarter]: the softmax warps' row sums at the end of a segment
  int lim[NS_MAX];         // valid tokens of the stage's page (0 for a bad page id; FP8)
  uint32_t tmem_base;
  int abort_flag;
  Unit unit, next;  // the segment being processed and the one after it
};
static_assert(sizeof(Bars) <= 1024, "barrier block");

// A stage holds the page's latent half as 16-bit values in 4 boxes of 64 dims, then its rope
// half.  bf16: TMA writes both directly.  FP8: TMA writes the codes (2 boxes of 128 codes)
// into boxes 2-3 and the 4 scales of each token after the rope half; the expansion then
// overwrites boxes 0-3 with fp16 values.
// bf16 pages take two rings: a cache stage feeds QK only and is released when QK completes,
// and the latent half is loaded a second time (from L2, where the first load left it) into a
// PV stage shortly before PV needs it.  A cache byte then occupies shared memory for the QK
// and PV steps only, not for the score exchange and softmax in between, so the same shared
// memory keeps about twice as many pages in flight.  FP8 pages are expanded in place once and
// keep one ring of stages that QK and PV both read.
template <bool FP8> struct Cfg {
  static constexpr bool RL = !FP8;       // the PV operand is reloaded into a ring of its own
  static constexpr int NS = RL ? 2 : 4;  // cache stages (QK; FP8: QK and PV)
  static constexpr int NV = RL ? 2 : 0;  // PV stages (latent half only)
  static constexpr int NRB = RL ? 2 : 1; // receive buffers for the peer's partial scores
  static constexpr int NPB = 3;          // P buffers (PV(g) may still read one while later P are written)
  static constexpr int PV_STAGE = 4 * LAT_BOX;
  static constexpr int CODE_OFF = 2 * LAT_BOX;
  static constexpr int ROPE_OFF = 4 * LAT_BOX;
  static constexpr int SCALE_OFF = ROPE_OFF + ROPE_BOX;
  static constexpr int STAGE = SCALE_OFF + (FP8 ? TILE * 16 : 0);  // 36864 / 37888
  static constexpr uint32_t STAGE_TX = FP8 ? 2 * LAT_BOX + ROPE_BOX + TILE * 16 : STAGE;
  // Q's latent half (4 boxes of 16 KB) is staged two boxes per stage, moved to TMEM, and only
  // then are those stages filled: the stages of the segment's tiles 2 and 3 (one ring), or its
  // two PV stages (two rings).
  static constexpr int PV_OFF = KV_OFF + NS * STAGE;
  static constexpr int RECV_OFF = PV_OFF + NV * PV_STAGE;
  static constexpr int P_OFF = RECV_OFF + NRB * RECV_BUF;
  static constexpr int ALPHA_OFF = P_OFF + NPB * P_BUF;   // [NPB][HO] the peer's fp32 rescale factors
  static constexpr int L_OFF = ALPHA_OFF + NPB * HO * 4;  // [HM] fp32 row sums of the segment
  // fp32 per own lane quarter: [NG][32] reference maxima handed from page to page.  (The
  // softmax warps' partial row sums at the end of a segment go to the receive buffer, free by then.)
  static constexpr int MX_OFF = L_OFF + HM * 4;
  static constexpr int BAR_OFF = MX_OFF + 2 * NG * 32 * 4;
  // Two rings: the dynamic shared memory base must be 1024-aligned (the kernel checks it), as
  // the layout leaves no room to align it; one ring: 1 KB of slack to align it.
  static constexpr int SMEM_BYTES = BAR_OFF + (int)(sizeof(Bars) + 127) / 128 * 128 + (RL ? 0 : 1024);
  static_assert(STAGE % 1024 == 0 && RECV_OFF % 1024 == 0 && P_OFF % 1024 == 0, "1024-aligned buffers");
  static_assert((RL ? PV_STAGE : STAGE) >= 2 * Q_LAT_BOX && (RL ? NV : NS) >= 2, "Q staging");
  static_assert(NS <= NS_MAX && NV <= NV_MAX && NRB <= NRB_MAX && NPB <= NPB_MAX, "barrier rings");
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
};
constexpr uint32_t Q_BYTES = 4 * Q_LAT_BOX + HM * HALF_DR * 2;  // 73728
constexpr uint32_t TMEM_COLS = 512;
// TMEM: O half in cols [0, 256); partial-score buffers 2 x 64 columns from 256; Q's latent half,
// the A operand of QK, in cols [384, 512) (256 16-bit values per row, two per 32-bit column).
constexpr uint32_t TM_O = 0, TM_S = 256, TM_Q = 384;
static_assert(TM_S + NSB * TILE <= TM_Q && TM_Q + HALF_DC / 2 <= TMEM_COLS, "TMEM budget");



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
  int n_workers;     // equal page ranges of the concatenated sequences
  int32_t* rowinfo;  // [rows][2] first / last partial slot of each row (-1: no pages)
};

__device__ __forceinline__ void fail(Bars* bars, int* err, int where) {
  record_error(err, ERR_TIMEOUT, where);
  atomicExch(&bars->abort_flag, 1);
}
__device__ __forceinline__ bool aborted(Bars* bars) {
  return *reinterpret_cast<volatile int*>(&bars->abort_flag) != 0;
}



// bf16 pair -> fp16 pair, saturating to the fp16 range
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
  const float lo = fminf(fmaxf(__uint_as_float(w << 16), -65504.f), 65504.f);
  const float hi = fminf(fmaxf(__uint_as_float(w & 0xFFFF0000u), -65504.f), 65504.f);
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// four E4M3 codes (little-endian in w) -> two fp16 pairs, each code times s: the code is exact
// in fp16 and fp32, the product is formed in fp32 and rounded once to fp16
__device__ __forceinline__ void e4m3x4_to_f16(uint32_t w, float s, uint32_t& lo, uint32_t& hi) {
  __half2_raw a = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w & 0xFFFFu), __NV_E4M3);
  __half2_raw b = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w >> 16), __NV_E4M3);
  const float2 fa = __half22float2(*reinterpret_cast<__half2*>(&a));
  const float2 fb = __half22float2(*reinterpret_cast<__half2*>(&b));
  const __half2 x = __floats2half2_rn(fa.x * s, fa.y * s);
  const __half2 y = __floats2half2_rn(fb.x * s, fb.y * s);
  lo = *reinterpret_cast<const uint32_t*>(&x);
  hi = *reinterpret_cast<const uint32_t*>(&y);
}

// FP8 pages: expand tokens [16 eg, 16 eg + 16) of the page in stage st in place, fp16 (code *
// scale, rounded once from fp32) into latent boxes 0-3, zeros for tokens past lim (stale slots
// may hold any byte).  An item is (token t, code box k, 16-code chunk c); its fp16 output lands
// over codes of the same token only, so the warp reads all of its items before it writes any.
template <int CODE_OFF, int SCALE_OFF>
__device__ __forceinline__ void expand_group(uint8_t* st, int lim, int eg, uint32_t rank, int lane) {
  const float* scl_p = reinterpret_cast<const float*>(st + SCALE_OFF);
  const int c = lane & 7, k = (lane >> 3) & 1;
  uint4 raw[8];
  float scl[8];
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int t = 16 * eg + 2 * it + (lane >> 4);
    raw[it] = *reinterpret_cast<const uint4*>(st + CODE_OFF + k * LAT_BOX + t * 128 + ((c ^ (t & 7)) << 4));
    scl[it] = t < lim ? scl_p[t * 4 + 2 * (int)rank + k] : 0.f;
  }
  __syncwarp();
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int t = 16 * eg + 2 * it + (lane >> 4);
    uint4 o0 = make_uint4(0, 0, 0, 0), o1 = make_uint4(0, 0, 0, 0);
    if (t < lim) {
      e4m3x4_to_f16(raw[it].x, scl[it], o0.x, o0.y);
      e4m3x4_to_f16(raw[it].y, scl[it], o0.z, o0.w);
      e4m3x4_to_f16(raw[it].z, scl[it], o1.x, o1.y);
      e4m3x4_to_f16(raw[it].w, scl[it], o1.z, o1.w);
    }
    // dims 128k + 16c .. +15 of the CTA's half: box 2k + c/4, 16-byte chunks 2(c%4), +1
    uint8_t* vrow = st + (2 * k + (c >> 2)) * LAT_BOX + t * 128;
    const int cc = 2 * (c & 3);
    *reinterpret_cast<uint4*>(vrow + ((cc ^ (t & 7)) << 4)) = o0;
    *reinterpret_cast<uint4*>(vrow + (((cc + 1) ^ (t & 7)) << 4)) = o1;
  }
  __syncwarp();
}

template <bool FP8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NTHREADS, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_q_lat, const __grid_constant__ CUtensorMap tm_q_rope,
                     const __grid_constant__ CUtensorMap tm_lat, const __grid_constant__ CUtensorMap tm_rope,
                     const __grid_constant__ CUtensorMap tm_scale, const Params p) {
  using C = Cfg<FP8>;
  constexpr bool RL = C::RL;
  constexpr int NS = C::NS, NRB = C::NRB, NPB = C::NPB;
  constexpr int NV = C::NV > 0 ? C::NV : 1;  // (one ring: no PV stages; kept nonzero for the ring arithmetic)
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if (RL && smem != smem_raw) {  // no room to align (every thread of both CTAs leaves here)
    if (threadIdx.x == 0) record_error(p.err, ERR_SMEM, (int)(smem_addr(smem_raw) & 1023));
    return;
  }
  Bars* bars = reinterpret_cast<Bars*>(smem + C::BAR_OFF);
  // the combine (launched programmatically) may take each SM this CTA leaves; it waits for the
  // whole grid's writes before it reads any
  griddep_launch_dependents();
  float* alpha_buf = reinterpret_cast<float*>(smem + C::ALPHA_OFF);  // [NPB][HO]: the peer's heads
  float* l_buf = reinterpret_cast<float*>(smem + C::L_OFF);          // [HM]
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int unit = blockIdx.x / 2;
  // Row warps (0 .. 11): TMEM lane quarter, set (0 .. 2), and whether the quarter holds heads
  // whose softmax this CTA owns (heads [64 rank, 64 rank + 64) = quarters 2 rank, 2 rank + 1).
  const int quarter = warp & 3;
  const int rset = warp >> 2;
  const int prod_w = NROW + 2 * (int)peer, mma_w = prod_w + 1;  // on the peer quarters' schedulers
  const int vprod_w = NROW + 2 * (int)rank;                      // bf16: loads the PV stages
  const bool own_q = (quarter >> 1) == (int)rank;
  const int row = quarter * 32 + lane;                        // head of this thread's TMEM lane
  const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
  const bool is_softmax = warp < NROW && own_q;              // token group rset of each tile
  const bool is_send = warp < NROW && !own_q && rset < 2;
  const bool is_precv = warp < NROW && !own_q && rset == 2;

  // the thread that arms this CTA's receive barriers for the peer's data
  const bool sm_lead = is_softmax && rset == 0 && quarter == 2 * (int)rank && lane == 0;
  const bool pr_lead = is_precv && quarter == 2 * (int)peer && lane == 0;
  const bool se_lead = is_send && rset == 0 && quarter == 2 * (int)peer && lane == 0;  // arms send_ok
  Plan pl;  // the producer warp only
  if (warp == prod_w) {
    plan::plan_begin<ROW_COST>(p, pl, unit, lane);
    if (unit == 0 && rank == 0) plan::write_rowinfo<ROW_COST>(p, pl.T, max(pl.U, 1ll), lane);
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);  // released by QK (bf16) or PV (FP8)
      mbar_init(&bars->x_full[s], 4);    // FP8: the four send warps expanded their tokens
    }
    for (int v = 0; v < NV; ++v) {
      mbar_init(&bars->v_full[v], 1);
      mbar_init(&bars->v_empty[v], 1);   // released by PV
    }
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_moved, NROW);     // row warp set s moves boxes s and s + 3
    for (int b = 0; b < NSB; ++b) {
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->s_free[b], 2 + 4);  // the tile's two softmax warps and the send warps read S
    }
    // The peer's signals below arrive as 4-byte st.async stores that complete transaction bytes on
    // a barrier armed (one arrival, expect_tx) by the waiting side each phase: unlike a remote
    // arrive, the signalling thread does not wait for the round trip.
    for (int k = 0; k < NRB; ++k) mbar_init(&bars->send_ok[k], 1);  // + 8 bytes: the peer's two readers
    for (int k = 0; k < RG; ++k) {
      mbar_init(&bars->s6[k], 1);          // QK of the slot's tile (a second commit)
      mbar_init(&bars->recv6[k], 1);       // armed by this CTA, completed by the peer's bytes
      mbar_init(&bars->pvs6[k], 1);        // PV of the slot's tile (second and third commits)
      mbar_init(&bars->pvr6[k], 1);
    }
    for (int k = 0; k < NPB; ++k) {
      mbar_init(&bars->p_recv[k], 1);      // armed by pr_lead, completed by the peer's bytes
      mbar_init(&bars->p_full[k], 2 + 2);  // the tile's softmax warps + P-receiving warps
      mbar_init(&bars->pv_done[k], 1);
      mbar_init(&bars->p_free[k], 1);      // + 8 bytes: the peer's PV of the buffer's previous tile
                                           // is done (its two softmax warps of the tile)
    }
    mbar_init(&bars->l_full, 2);         // the two group-0 softmax warps (+ the peer's sums)
    for (int q = 0; q < 2; ++q) {
      for (int j = 0; j < NG; ++j) mbar_init(&bars->hand[q][j], 1);
      mbar_init(&bars->ls_full[q], NG);
    }
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == mma_w) {
    tmem_alloc(&bars->tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Arm the first use of each receive buffer (the peer's bytes may land before or after).
  if (sm_lead) {
    for (int k = 0; k < RG; ++k) mbar_arrive_expect_tx(&bars->recv6[k], RECV_BUF);
    for (int k = 0; k < NPB; ++k) mbar_arrive_expect_tx(&bars->p_free[k], 2 * 4);
  }
  if (pr_lead)
    for (int k = 0; k < NPB; ++k) mbar_arrive_expect_tx(&bars->p_recv[k], P_RECV_TX);
  if (se_lead)
    for (int k = 0; k < NRB; ++k) mbar_arrive_expect_tx(&bars->send_ok[k], 2 * 4);
  cluster_sync();  // peer barriers initialised before any remote arrive / st.async
  const uint32_t tmem = bars->tmem_base;

  // Segment loop: a worker's range of the balanced partition, one row segment at a time.
  // Barrier phases run on across segments (gb = tiles, seg = segments done); both CTAs drain
  // every segment before the next one starts.
  int gb = 0, seg = 0;
  // The producer warp plans one segment ahead, so it can pull the next segment's Q and first
  // pages into L2 while this one drains.
  if (warp == prod_w) {
    const Unit f = plan::plan_next<ROW_COST>(p, pl, unit, lane);
    __syncwarp();
    if (lane == 0) bars->next = f;
  }
  for (;;) {
  if (warp == prod_w) {
    __syncwarp();
    if (lane == 0) bars->unit = bars->next;
  }
  __syncthreads();
  const Unit u = bars->unit;
  if (!u.valid) break;
  const int n_tiles = (u.hi - u.lo + TILE - 1) / TILE;
  const int32_t* bt = p.block_table + (long)u.b * p.max_pages;
  const uint32_t sph = seg & 1;  // phase parity of the once-per-segment barriers
  const long qh = (long)u.qrow * p.H + row;
  const long prow_idx = (long)u.slot * p.H + row;
  const bool hv = row < p.H;  // rows past H are never stored
  // Q staging box jb (0..3): box jb % 2 of the stage of the segment's tile NS - 2 + jb / 2 (one
  // ring: the last two stages the segment fills) or of the PV stage of its tile jb / 2 (two rings)
  auto q_box = [&](int jb) -> uint8_t* {
    if (RL) return smem + C::PV_OFF + ((gb + (jb >> 1)) % NV) * C::PV_STAGE + (jb & 1) * Q_LAT_BOX;
    return smem + KV_OFF + ((gb + NS - 2 + (jb >> 1)) % NS) * C::STAGE + (jb & 1) * Q_LAT_BOX;
  };
  // the segment after this one (the producer warp, all lanes)
  auto plan_ahead = [&]() {
    const Unit t2 = plan::plan_next<ROW_COST>(p, pl, unit, lane);
    __syncwarp();
    if (lane == 0) bars->next = t2;
    __syncwarp();
  };

  if (n_tiles > 0) {
    if (warp == prod_w) {
      // ------------------------------------------------------------ TMA producer
      // Page ids are read one tile ahead, so their global-load latency overlaps the waits.  Only
      // the next segment's first pages are prefetched into L2 (while this segment drains):
      // prefetching every page some tiles ahead of its stage was measured 2-7 % slower.
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
      int page_cur = 0;
      int issued = 0;  // tiles whose loads were issued (the loop may stop early on an abort)
      // Tile i's loads (lane 0).  False when a wait timed out or the kernel is winding down.
      auto issue = [&](int i) -> bool {
        const int g = gb + i, s = g % NS;
        // kv_empty[s] completes once per QK (bf16) or PV (FP8) of a tile using stage s; the next
        // completion needs this tile loaded, so the producer never sees it two phases late.
        if (g >= NS && !mbar_wait(&bars->kv_empty[s], ((g / NS) - 1) & 1)) {
          fail(bars, p.err, 1);
          return false;
        }
        if (!RL && i == NS - 2 && !mbar_wait(&bars->q_moved, sph)) {  // those stages held Q until now
          fail(bars, p.err, 6);
          return false;
        }
        if (aborted(bars)) return false;
        const int page = page_cur;
        page_cur = page_of(i + 1);
        const bool bad = page < 0 || page >= p.num_pages;
        if (bad && rank == 0) record_error(p.err, ERR_PAGE, page);
        // a bad page reads TMA's zero fill (rows past the end); the softmax masks its tokens
        const int y = bad ? p.num_pages * 64 : page * 64;
        uint8_t* st = smem + KV_OFF + s * C::STAGE;
        // the page's valid tokens, for the softmax and the expansion (published by the arrive)
        bars->lim[s] = bad ? 0 : min(TILE, u.hi - (u.lo + i * TILE));
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
        return true;
      };
      bool go = true;
      if (lane == 0) {
        prefetch_tmap(&tm_lat);
        prefetch_tmap(&tm_rope);
        if (FP8) prefetch_tmap(&tm_scale);
        mbar_arrive_expect_tx(&bars->q_full, Q_BYTES);
        const int qy = u.qrow * p.H;
        for (int jb = 0; jb < 4; ++jb)
          tma_load_2d(q_box(jb), &tm_q_lat, (int)rank * HALF_DC + jb * 64, qy, &bars->q_full);
        tma_load_2d(smem + Q_ROPE_OFF, &tm_q_rope, DC + (int)rank * HALF_DR, qy, &bars->q_full);
        page_cur = page_of(0);
        go = issue(0);
      }
      // the following segment is planned while the first loads of this one are in flight
      plan_ahead();
      if (lane == 0) {
        for (int i = 1; go && i < n_tiles; ++i) go = issue(i);
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
    } else if (RL && warp == vprod_w) {
      // ------------------------------------------------------------ PV stage loads (bf16 pages)
      // Tile i's latent half again, into PV stage g % NV, once PV(g - NV) has released the stage
      // and QK(g) has completed (the tile's first load has brought the page into L2).  Slot
      // g % 6 of s6 cannot be a phase ahead here: QK(g + 6) waits for PV(g + 6 - QK_AHEAD) to be
      // issued (QK runs at most QK_AHEAD <= 6 tiles past the next PV), hence for PV(g), which
      // waits for this load.
      if (lane == 0) {
        int vissued = 0;
        for (int i = 0; i < n_tiles; ++i) {
          const int g = gb + i, v = g % NV;
          if (g >= NV && !mbar_wait(&bars->v_empty[v], ((g / NV) - 1) & 1)) {
            fail(bars, p.err, 25);
            break;
          }
          if (i == 0 && !mbar_wait(&bars->q_moved, sph)) {  // the PV stages held Q until now
            fail(bars, p.err, 26);
            break;
          }
          if (!mbar_wait(&bars->s6[g % RG], (g / RG) & 1)) {
            fail(bars, p.err, 27);
            break;
          }
          if (aborted(bars)) break;
          const int page = bt[(u.lo + i * TILE) / 64];
          const int y = (page < 0 || page >= p.num_pages) ? p.num_pages * 64 : page * 64;
          uint8_t* st = smem + C::PV_OFF + v * C::PV_STAGE;
          mbar_arrive_expect_tx(&bars->v_full[v], C::PV_STAGE);
          for (int jb = 0; jb < 4; ++jb)
            tma_load_2d(st + jb * LAT_BOX, &tm_lat, (int)rank * HALF_DC + jb * 64, y, &bars->v_full[v]);
          vissued = i + 1;
        }
        // drain: every load still in flight lands before the CTA may exit
        for (int i = max(0, vissued - NV); i < vissued; ++i)
          if (!mbar_wait(&bars->v_full[(gb + i) % NV], ((gb + i) / NV) & 1)) break;
      }
    } else if (warp == mma_w) {
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
          mma_commit(&bars->s6[g % RG]);
          if (RL) mma_commit(&bars->kv_empty[s]);  // the cache stage is done (PV reads its own)
        };
        auto issue_pv = [&](int jt) {
          const int g = gb + jt, k = g % NPB;
          tc_fence_after();
          const uint32_t p_base = smem_addr(smem + C::P_OFF + k * P_BUF);
          const uint32_t v_base = RL ? smem_addr(smem + C::PV_OFF + (g % NV) * C::PV_STAGE) : lat_tile(g);
#pragma unroll
          for (int kt = 0; kt < TILE / 16; ++kt) {
            const uint64_t a = umma_desc(p_base + kt * 32, 16, 1024, UMMA_SW128);
            const uint64_t bdesc = umma_desc(v_base + kt * 2048, LAT_BOX, 1024, UMMA_SW128);
            mma_bf16(tmem + TM_O, a, bdesc, ID_PV, (jt > 0 || kt > 0) ? 1u : 0u);
          }
          mma_commit(&bars->pv_done[k]);
          mma_commit(RL ? &bars->v_empty[g % NV] : &bars->kv_empty[g % NS]);
          mma_commit(&bars->pvs6[g % RG]);
          mma_commit(&bars->pvr6[g % RG]);
        };
        // Event loop: PV(k) as soon as P(k) is complete in shared memory (and its PV stage loaded);
        // otherwise QK(j) once its page is loaded (and expanded), S buffer j % 2 has been read
        // (tile j - 2) and j is at most QK_AHEAD tiles past the next PV (the tensor pipe runs in
        // order: a QK queued ahead of a PV delays the PV, which releases a stage).
        int qk = 0, pv = 0;
        uint64_t t_idle = 0;
        uint32_t spins = 0;
        while (ok && pv < n_tiles) {
          const int gp = gb + pv, gq = gb + qk;
          if (pv < qk && mbar_test(&bars->p_full[gp % NPB], (gp / NPB) & 1) &&
              (!RL || mbar_test(&bars->v_full[gp % NV], (gp / NV) & 1))) {
            issue_pv(pv++);
            t_idle = 0;
            continue;
          }
          if (qk < n_tiles && qk < pv + QK_AHEAD && mbar_test(&bars->kv_full[gq % NS], (gq / NS) & 1) &&
              (!FP8 || mbar_test(&bars->x_full[gq % NS], (gq / NS) & 1)) &&
              (gq < NSB || mbar_test(&bars->s_free[gq % NSB], ((gq / NSB) - 1) & 1))) {
            issue_qk(qk++);
            t_idle = 0;
            continue;
          }
          __nanosleep(32);  // idle: leave the issue slots to the softmax warps of this SMSP
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
    } else if (warp < NROW) {
      // ------------------------------------------------------------ row warps
      // Move this quarter's 32 Q rows, latent dims [64 jb, 64 jb + 64) of the CTA's 256 (staging box
      // jb) for jb = s and s + 3 (set s), from the 128B-swizzled staging boxes into TMEM as 16-bit
      // pairs along K (fp16 for FP8 pages).
      {
        bool qok = __all_sync(0xffffffffu, mbar_wait(&bars->q_full, sph));
        if (!qok) fail(bars, p.err, 19);
#pragma unroll 1
        for (int jb = rset; jb < 4; jb += NROW / 4) {
          uint32_t qv[32];
          const uint8_t* box = q_box(jb) + row * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 v = *reinterpret_cast<const uint4*>(box + ((c ^ (row & 7)) * 16));
            qv[4 * c] = FP8 ? bf16x2_to_f16x2(v.x) : v.x;
            qv[4 * c + 1] = FP8 ? bf16x2_to_f16x2(v.y) : v.y;
            qv[4 * c + 2] = FP8 ? bf16x2_to_f16x2(v.z) : v.z;
            qv[4 * c + 3] = FP8 ? bf16x2_to_f16x2(v.w) : v.w;
          }
          tmem_st32(tmem + lane_off + TM_Q + jb * 32, qv);
        }
        tmem_wait_st();
        fence_proxy_async_smem();  // staging reads done before TMA refills those stages
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->q_moved);
      }
      bool ok = true;
      if (is_softmax) {
        // ---------------------------------------------------------- softmax (own heads)
        // Thread = head row; the three warps of a lane quarter take turns (warp rset takes the tiles
        // g with g % 3 == rset), whole rows of 64 tokens, so three pages are in flight.  Only the
        // lazy reference maximum m passes from page to page: the warp of tile g reads m after tile
        // g - 1 from the handoff slot (g - 1) % 3 and writes m after tile g to slot g % 3
        // (hand[quarter % 2][slot]).  Each warp keeps its partial row sum with the reference
        // it was accumulated against; they are merged exactly at the end of the segment.
        const int orow = row - HO * (int)rank;  // row in the receive buffers (0..63)
        const int oq = quarter & 1;
        const float sc = p.scale_log2;
        float* hand = reinterpret_cast<float*>(smem + C::MX_OFF);  // [2][NG][32] reference maxima
        // the thread of this quarter's tile-g warp that arms the receive barrier (quarter 2 rank)
        const bool arm_q = quarter == 2 * (int)rank && lane == 0;
        float m_ref = -INFINITY, l_part = 0.f;  // this warp's partial row sum and its reference
        float m_last = -INFINITY;               // reference after the last tile this warp took
        static_assert(RG % NG == 0 && RG % NSB == 0 && RG % NPB == 0, "buffer and slot rings");
        for (int i = 0; i < n_tiles; ++i) {
          const int g = gb + i;
          if (g % NG != rset) continue;
          const int sb = g % NSB, rk = g % NRB, pk = g % NPB;
          // bf16 pages: the tile's page id, for its valid-token count in step (3)
          const int page_id = RL ? bt[(u.lo + i * TILE) / 64] : 0;
          // (1) this CTA's partial scores of the row.  Slot g % 6 of s6 completed QK(g - 6), seen by
          // this warp; QK(g + 6) needs S(g) read (through QK(g + 2), QK(g + 4) and their s_free).
          if (!__all_sync(0xffffffffu, mbar_wait(&bars->s6[g % RG], (g / RG) & 1))) {
            fail(bars, p.err, 12);
            ok = false;
            break;
          }
          tc_fence_after();
          uint32_t sv[TILE];
          tmem_ld32(tmem + lane_off + TM_S + sb * TILE, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
          tmem_ld32(tmem + lane_off + TM_S + sb * TILE + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->s_free[sb]);
          // (2) the peer's partial scores (fp32): S = S_own + S_peer, in log2 units.
          // Slot g % 6 of recv6 is armed again by this warp below, after this tile's bytes.
          if (!__all_sync(0xffffffffu, mbar_wait<true>(&bars->recv6[g % RG], (g / RG) & 1))) {
            fail(bars, p.err, 13);
            ok = false;
            break;
          }
          // x[t] = (S_own + S_peer) * scale * log2(e), kept in place in sv
#define X(t) __uint_as_float(sv[t])
          {
            const uint8_t* rrow = smem + C::RECV_OFF + rk * RECV_BUF + orow * (TILE * 4);
#pragma unroll
            for (int c = 0; c < TILE / 4; ++c) {
              const float4 v = *reinterpret_cast<const float4*>(rrow + ((c ^ (orow & 15)) * 16));
              sv[4 * c] = __float_as_uint((X(4 * c) + v.x) * sc);
              sv[4 * c + 1] = __float_as_uint((X(4 * c + 1) + v.y) * sc);
              sv[4 * c + 2] = __float_as_uint((X(4 * c + 2) + v.z) * sc);
              sv[4 * c + 3] = __float_as_uint((X(4 * c + 3) + v.w) * sc);
            }
          }
          __syncwarp();
          if (arm_q) mbar_arrive_expect_tx(&bars->recv6[g % RG], RECV_BUF);  // tile g + 6
          // the peer may refill the buffer: the values read above have been consumed (x), so the
          // reads are complete and a relaxed arrive suffices
          if (lane == 0)
            st_async_b32(map_to_rank(&bars->sink[0], peer), 0u, map_to_rank(&bars->send_ok[rk], peer));
          // (3) tokens past the unit's end, or of a bad page, do not count.  FP8: the producer wrote
          // the page's count before it armed kv_full for the tile (whose phase QK(g) already passed;
          // its next one needs PV(g)).
          int lim;
          if (RL) {
            const int t0 = u.lo + i * TILE;
            lim = (page_id < 0 || page_id >= p.num_pages) ? 0 : min(TILE, u.hi - t0);
          } else {
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->kv_full[g % NS], (g / NS) & 1))) {
              fail(bars, p.err, 16);
              ok = false;
              break;
            }
            lim = bars->lim[g % NS];
          }
          if (lim < TILE) {
#pragma unroll
            for (int t = 0; t < TILE; ++t)
              if (t >= lim) sv[t] = __float_as_uint(-INFINITY);
          }
          float m8[8];  // the row maximum as a tree: eight independent chains, then three levels
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            m8[j] = X(8 * j);
#pragma unroll
            for (int t = 1; t < 8; ++t) m8[j] = fmaxf(m8[j], X(8 * j + t));
          }
          const float mt = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                 fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
          // (4) the reference after tile g - 1 (none at the segment's first tile), raised only when
          // a score of this tile passes it by more than 2^8.  hand[oq][j] completes once per tile
          // g = j mod NG; its next completion needs NG - 1 more handoffs, the first of which is
          // this warp's.
          float m_prev = -INFINITY;
          if (i > 0) {
            const int j = (g - 1) % NG;
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->hand[oq][j], ((g - 1) / NG) & 1))) {
              fail(bars, p.err, 22);
              ok = false;
              break;
            }
            m_prev = hand[(oq * NG + j) * 32 + lane];
          }
          float m_new = m_prev, alpha = 1.f;
          if (mt > m_prev + RESCALE_T) {
            // while the reference is -inf every earlier score was masked: O is still zero
            if (m_prev != -INFINITY) alpha = ex2_approx(m_prev - mt);
            m_new = mt;
          }
          hand[(oq * NG + g % NG) * 32 + lane] = m_new;
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->hand[oq][g % NG]);
          m_last = m_new;
          // this warp's partial sum moves to the new reference
          if (m_ref != m_new) {
            if (m_ref != -INFINITY) l_part *= ex2_approx(m_ref - m_new);
            m_ref = m_new;
          }
          const float mu = m_new == -INFINITY ? 0.f : m_new;  // 2^(-inf - 0) = 0
          // (5) P buffer pk is free here once PV(g - 3) has completed: the peer is then told that its
          // rows of tile g may land here (p_free).  Slot (g - 3) % 6 of pvs6 is waited only at tiles
          // = g mod 6; PV(g + 3) needs this warp's next tile.
          if (g >= NPB) {
            const int j = (g - NPB) % RG;
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->pvs6[j], ((g - NPB) / RG) & 1))) {
              fail(bars, p.err, 15);
              ok = false;
              break;
            }
          }
          __syncwarp();
          if (lane == 0)
            st_async_b32(map_to_rank(&bars->sink[1], peer), 0u, map_to_rank(&bars->p_free[pk], peer));
          // (5b) the peer's buffer pk takes this CTA's P rows of tile g once the peer's PV(g - 3) is
          // done (p_free: both of the peer's softmax warps of tile g said so).  Buffer pk is used by
          // the tiles g = pk mod 3, all taken by this warp set, which sees every phase; the next
          // completion needs the peer's PV(g), hence these rows.  The quarter-0 warp arms it again.
          if (!__all_sync(0xffffffffu, mbar_wait<true>(&bars->p_free[pk], (g / NPB) & 1))) {
            fail(bars, p.err, 24);
            ok = false;
            break;
          }
          if (oq == 0 && lane == 0) mbar_arrive_expect_tx(&bars->p_free[pk], 2 * 4);  // tile g + 3
          // (6) rescale this CTA's half of the row's O once PV(g - 1) has completed (slot (g - 1) % 6
          // of pvr6: PV(g - 7) is done since PV(g - 3) is, and PV(g + 5) needs the P rows of tile
          // g + 5, which come after this warp's next tile; the peer rescales its half with the
          // factor sent with P)
          const bool need_rescale = __any_sync(0xffffffffu, alpha != 1.f) && i > 0;
          if (need_rescale) {
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->pvr6[(g - 1) % RG], ((g - 1) / RG) & 1))) {
              fail(bars, p.err, 14);
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll 1
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
          // (7) P = 2^(s - m) of the row, rounded to the MMA's 16-bit type, written 16 bytes at a
          // time (128-byte K-major row, 16-byte chunk c at c ^ (row & 7)); l accumulates the
          // unrounded values.  The row's rescale factor goes with the copy to the peer.
          uint8_t* prow = smem + C::P_OFF + pk * P_BUF + row * 128;
          const uint32_t prow_peer = map_to_rank(prow, peer);
          const uint32_t prbar = map_to_rank(&bars->p_recv[pk], peer);
          float ps = 0.f;
#pragma unroll
          for (int c = 0; c < TILE / 8; ++c) {
            uint32_t w4[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float p0 = ex2_approx(X(8 * c + 2 * k) - mu), p1 = ex2_approx(X(8 * c + 2 * k + 1) - mu);
              if (FP8) {
                __half2 ph = __floats2half2_rn(p0, p1);
                w4[k] = *reinterpret_cast<uint32_t*>(&ph);
              } else {
                __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
                w4[k] = *reinterpret_cast<uint32_t*>(&pb);
              }
              ps += p0 + p1;
            }
            const uint4 q4 = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            *reinterpret_cast<uint4*>(prow + ((c ^ (row & 7)) * 16)) = q4;
            st_async_v4(prow_peer + ((c ^ (row & 7)) * 16), q4, prbar);
          }
#undef X
          l_part += ps;
          st_async_b32(map_to_rank(alpha_buf + pk * HO + orow, peer), __float_as_uint(alpha), prbar);
          // (8) bf16 pages: V rows past the valid tokens may hold stale data: zero them, so that
          // 0 * garbage = 0, in the PV stage once it has landed (v_full[g % NV] completes next for
          // tile g + NV, which needs PV(g), hence this warp's P), or in the cache stage (one ring;
          // QK(g) has completed).  The two warps of tile g (one per own quarter) take the rows with
          // their quarter's parity.  FP8 tiles are expanded with zeros already.
          if (!FP8 && lim < TILE) {
            if (RL && !__all_sync(0xffffffffu, mbar_wait(&bars->v_full[g % NV], (g / NV) & 1))) {
              fail(bars, p.err, 28);
              ok = false;
              break;
            }
            uint8_t* st = RL ? smem + C::PV_OFF + (g % NV) * C::PV_STAGE : smem + KV_OFF + (g % NS) * C::STAGE;
            const int first = max(lim, 0) + oq, nrow = (TILE - first + 1) / 2;
            for (int e = lane; e < nrow * 32; e += 32) {  // row, box, 16-byte chunk
              const int r = first + 2 * (e / 32), bx = (e / 8) & 3;
              *reinterpret_cast<uint4*>(st + bx * LAT_BOX + r * 128 + (e % 8) * 16) = make_uint4(0, 0, 0, 0);
            }
          }
          fence_proxy_async_smem();  // P (and any zeroed V rows) visible to the MMA
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->p_full[pk]);
        }
        // The row sum: the three warps' partial sums, each moved to the reference after the
        // segment's last tile (taken by warp (gb + n_tiles - 1) % 3, whose m_last is that
        // reference), and the segment's lse; the row sum goes to both CTAs' epilogues.
        // Slots per own quarter: [warp][2] (partial sum, its reference) and the final reference.
        // They go to receive buffer 0, in the rows of this quarter's heads (read by this quarter's
        // warps only, and sent no more this segment), once the quarter's three warps are done.
        named_bar_sync(1 + oq, 32 * NG);
        float* lp = reinterpret_cast<float*>(smem + C::RECV_OFF + oq * (32 * TILE * 4));
        lp[(rset * 2) * 32 + lane] = l_part;
        lp[(rset * 2 + 1) * 32 + lane] = m_ref;
        const int wl = (gb + n_tiles - 1) % NG;
        if (rset == wl) lp[2 * NG * 32 + lane] = m_last;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->ls_full[oq]);
        if (rset == 0) {
          if (!__all_sync(0xffffffffu, mbar_wait(&bars->ls_full[oq], sph))) {
            fail(bars, p.err, 23);
            ok = false;
          }
          const float m_fin = lp[2 * NG * 32 + lane];
          float l_sum = 0.f;
#pragma unroll
          for (int k = 0; k < NG; ++k) {
            const float lk = lp[(k * 2) * 32 + lane], mk = lp[(k * 2 + 1) * 32 + lane];
            if (mk != -INFINITY) l_sum += lk * ex2_approx(mk - m_fin);
          }
          if (hv) {
            const float lse = (ok && l_sum > 0.f) ? (m_fin + log2f(l_sum)) * 0.69314718055994531f : -INFINITY;
            if (u.final_out) {
              if (p.lse) p.lse[qh] = lse;
            } else {
              p.lse_part[prow_idx] = lse;
            }
          }
          l_buf[row] = l_sum;
          st_async_b32(map_to_rank(l_buf + row, peer), __float_as_uint(l_sum), map_to_rank(&bars->l_full, peer));
          __syncwarp();
          if (lane == 0) {
            if (sm_lead) mbar_arrive_expect_tx(&bars->l_full, HO * 4);
            else mbar_arrive(&bars->l_full);
          }
        }
      } else if (is_send) {
        // ---------------------------------------------------------- partial scores to the peer
        // (FP8 pages: first each of the four send warps expands 16 of the page's tokens; QK(g)
        // waits for all four.  Page g + 1 is expanded after S(g) has gone, so the send is not
        // delayed; QK stays one page ahead of the sends.)
        const int prow = row - HO * (int)peer;  // the head's row in the peer's receive buffers
        const int c0 = rset * 32;               // this warp's 32 token columns
        for (int i = 0; i < n_tiles; ++i) {
          const int g = gb + i, sb = g % NSB, rk = g % NRB;
          if (FP8) {
            const int s = g % NS;
            // kv_full[s] completes next for tile g + NS, which needs PV(g), hence QK(g), hence
            // this warp's x_full arrival.
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->kv_full[s], (g / NS) & 1))) {
              fail(bars, p.err, 20);
              ok = false;
              break;
            }
            expand_group<C::CODE_OFF, C::SCALE_OFF>(smem + KV_OFF + s * C::STAGE, bars->lim[s],
                                                    2 * (quarter & 1) + rset, rank, lane);
            fence_proxy_async_smem();  // the tile is read by the MMA (async proxy)
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->x_full[s]);
          }
          if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[sb], (g / NSB) & 1))) {
            fail(bars, p.err, 10);
            ok = false;
            break;
          }
          tc_fence_after();
          uint32_t v[32];
          tmem_ld32(tmem + lane_off + TM_S + sb * TILE + c0, v);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->s_free[sb]);
          // The peer's buffer rk held tile g - NRB until the peer's softmax read it; send_ok[rk]
          // completes once per such read, and the next one needs this tile's bytes.
          if (g >= NRB &&
              !__all_sync(0xffffffffu, mbar_wait<true>(&bars->send_ok[rk], ((g / NRB) - 1) & 1))) {
            fail(bars, p.err, 11);
            ok = false;
            break;
          }
          if (g >= NRB && se_lead) mbar_arrive_expect_tx(&bars->send_ok[rk], 2 * 4);  // tile g's readers
          const uint32_t rrow = map_to_rank(smem + C::RECV_OFF + rk * RECV_BUF + prow * (TILE * 4), peer);
          const uint32_t rbar = map_to_rank(&bars->recv6[g % RG], peer);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            st_async_v4(rrow + (((c0 / 4 + c) ^ (prow & 15)) * 16),
                        make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]), rbar);
        }
      } else if (is_precv) {
        // ---------------------------------------------------------- the peer's P rows
        for (int i = 0; i < n_tiles; ++i) {
          const int g = gb + i, pk = g % NPB;
          // p_recv[pk] completes again only after this CTA's PV(g) has run (p_free), which needs
          // this warp's p_full arrival.  The rows and their factors arrive by st.async from the
          // peer's softmax warps; a proxy fence below hands the rows to the MMA.
          if (!__all_sync(0xffffffffu, mbar_wait<true>(&bars->p_recv[pk], (g / NPB) & 1))) {
            fail(bars, p.err, 17);
            ok = false;
            break;
          }
          const float alpha = alpha_buf[pk * HO + (row - HO * (int)peer)];
          __syncwarp();
          if (pr_lead) mbar_arrive_expect_tx(&bars->p_recv[pk], P_RECV_TX);  // its next use
          const bool need_rescale = __any_sync(0xffffffffu, alpha != 1.f) && i > 0;
          if (need_rescale) {
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->pv_done[(g - 1) % NPB], ((g - 1) / NPB) & 1))) {
              fail(bars, p.err, 18);
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll 1
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
          fence_proxy_async_smem();  // the peer's P rows (st.async) are read by the MMA
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->p_full[pk]);
        }
      }
      // ------------------------------------------------------------ epilogue (all row warps)
      // O half of every row, normalised by the row sum its owner sent (l_full: the two group-0
      // softmax warps here and the peer's 64 sums), after the last PV.  Warp set s takes the
      // 32-column chunks cb with cb % 3 == s.  l_full comes first: it completes after the softmax warps waited for
      // PV(last - 2), so pv_done of the last tile's buffer is then exactly one phase short of
      // PV(last) (most of these warps never waited on it before and could be two phases behind,
      // where a parity wait passes at once).
      ok = __all_sync(0xffffffffu, ok);
      {
        const int jt = gb + n_tiles - 1;
        const bool w2 = mbar_wait<true>(&bars->l_full, sph);
        const bool w1 = w2 && mbar_wait(&bars->pv_done[jt % NPB], (jt / NPB) & 1);
        if (!__all_sync(0xffffffffu, w1 && w2)) {
          fail(bars, p.err, 21);
          ok = false;
        }
        tc_fence_after();
      }
      if (aborted(bars)) ok = false;
      const float l_row = l_buf[row];
      const float inv_l = l_row > 0.f ? 1.f / l_row : 0.f;
      const bool final_out = u.final_out != 0;
#pragma unroll 1
      for (int cb = rset; cb < HALF_DC / 32; cb += NROW / 4) {
        uint32_t o[32];
        __syncwarp();
        tmem_ld32(tmem + lane_off + TM_O + cb * 32, o);
        tmem_wait_ld();
        const int d0 = (int)rank * HALF_DC + cb * 32;
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
    }
  }
  // segment boundary: every role of both CTAs is done with this segment (all loads landed, all
  // MMAs completed, all scores and P rows exchanged, O read out)
  gb += n_tiles;
  if (n_tiles > 0) ++seg;  // the once-per-segment barriers completed a phase
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  // a CTA that gave up makes its peer stop as well (both read both flags after the barrier)
  if (aborted(bars) || ld_cluster_u32(map_to_rank(&bars->abort_flag, peer)) != 0) break;
  }  // segment loop
  // Every signal the peer sent here has landed before either CTA leaves: the readers' signals of
  // the last NRB tiles (send_ok) are the only ones no later step waits for.
  if (se_lead && !aborted(bars))
    for (int g = max(0, gb - NRB); g < gb; ++g)
      if (!mbar_wait<true>(&bars->send_ok[g % NRB], (g / NRB) & 1)) break;
  tc_fence_before();
  __syncthreads();
  if (warp == mma_w) {
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
                                                           const float* lse_part, int H, int stride,
                                                           __nv_bfloat16* o_lat, float* lse) {
  // launched while the decode kernel drains (programmatic launch): its partials and slot table
  // are complete and visible after this wait
  griddep_wait();
  // the next grid (the output projection) may start streaming its weights meanwhile
  griddep_launch_dependents();
  const int r = blockIdx.x, h = blockIdx.y * 8 + threadIdx.x / 32, lane = threadIdx.x % 32;
  if (h >= H) return;
  const int c0 = rowinfo[2 * r], c1 = rowinfo[2 * r + 1];
  if (c0 >= 0 && c0 == c1) return;
  const long qh = (long)r * H + h;
  float m = -INFINITY;
  for (int c = c0; c0 >= 0 && c <= c1; c += stride) m = fmaxf(m, lse_part[(long)c * H + h]);
  float4 acc[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  float wsum = 0.f;
  if (m != -INFINITY) {
    for (int c = c0; c <= c1; c += stride) {
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
  const size_t rows = (size_t)batch * s_q;
  return (size_t)TC_PLAN_SLOTS * d.n_heads * (d.d_c + 1) * sizeof(float) + rows * 2 * sizeof(int32_t);
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

cudaError_t launch_plan_combine(const DecodeArgs& a, cudaStream_t st) {
  const long rows = (long)a.batch * a.s_q;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)rows, (unsigned)((a.n_heads + 7) / 8));
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, tc::combine_plan_kernel, (const int32_t*)a.rowinfo, (const float*)a.o_part,
                                     (const float*)a.lse_part, a.n_heads, a.s_q,
                                     reinterpret_cast<__nv_bfloat16*>(a.o_lat), a.lse);
  note_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
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
  prm.scale_log2 = a.scale * 1.4426950408889634f;
  prm.o_lat = reinterpret_cast<__nv_bfloat16*>(a.o_lat);
  prm.lse = a.lse;
  prm.o_part = a.o_part;
  prm.lse_part = a.lse_part;
  prm.err = a.err;
  // ranges: one per SM pair for each query token of a sequence (at least one)
  prm.n_workers = max(1, TC_PLAN_WORKERS / max(1, a.s_q));
  prm.rowinfo = a.rowinfo;
  if ((reinterpret_cast<uintptr_t>(a.q) & 15) || (reinterpret_cast<uintptr_t>(a.o_lat) & 15) ||
      (reinterpret_cast<uintptr_t>(a.o_part) & 15))
    return kUnsupported;
  const long rows = (long)a.batch * a.s_q;
  // balanced partition: one persistent cluster per worker range (one per SM pair)
  const long units = rows > 0 ? (long)prm.n_workers * a.s_q : 0;
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
    return e == cudaSuccess ? launch_plan_combine(a, st) : e;
  }
  if (!make_map(&m_lat, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, cv.rows, tc::W, kv_rows, 64, tc::TILE,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&m_rope, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, cv.rows, tc::W, kv_rows, tc::HALF_DR, tc::TILE,
                CU_TENSOR_MAP_SWIZZLE_64B))
    return kUnsupported;
  if (units == 0) return cudaSuccess;
  cudaError_t e = launch_tc<false>(m_q_lat, m_q_rope, m_lat, m_rope, m_lat, prm, units, st);
  return e == cudaSuccess ? launch_plan_combine(a, st) : e;
}

}  // namespace mla
