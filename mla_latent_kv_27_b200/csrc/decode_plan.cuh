// Length-balanced work partition of the paged decode kernels (decode_tc.cu, decode_sh.cu): which
// cached tokens each persistent worker attends, and where a row cut across workers leaves its
// partial result for the log-sum-exp combine.  Device helpers, warp-collective where stated; both
// kernels instantiate them with their own parameter block and boundary cost.
#pragma once
#include "mla_internal.cuh"

namespace mla {
namespace plan {

// Which tokens a unit attends: [lo, hi) of sequence b for query token j (row qrow = b s_q + j);
// a partial result goes to slot `slot`, a complete one (final_out) straight to o_lat / lse.
struct Unit {
  int b, j, lo, hi, qrow, slot, final_out, valid;
};

// Tokens row r attends (its cached length; with the causal mask, up to its own position).
template <class P>
__device__ __forceinline__ int attended(const P& p, int r, bool report) {
  const int j = r % p.s_q;
  int L = p.seq_lens[r / p.s_q];
  if (L < 0 || L > p.max_pages * 64) {
    if (report && j == 0) record_error(p.err, ERR_POS, L);
    L = max(0, min(L, p.max_pages * 64));
  }
  return p.causal ? max(0, min(L, L - p.s_q + j + 1)) : L;
}

// Length-balanced partition.  A sequence with pages costs its pages plus RC (the kernel's boundary cost): a segment
// boundary drains and refills the pipeline, about as long as that many pages.  The sequences'
// costs, concatenated in order (T in all), are cut into U = min(n_workers, T) equal ranges.  The
// grid holds n_workers * s_q workers: worker w takes range R = w / s_q for query token j = w % s_q,
// so the s_q query tokens of a sequence (whose rows attend the same pages) are walked by s_q
// neighbouring workers at the same time and each page comes from DRAM once.  Range R is walked
// sequence by sequence; within a sequence the first RC units stand for the boundary and the
// pages follow, and every sequence whose pages (those row b s_q + j attends) meet the range is
// one segment.  A row whose pages lie in one range is computed whole (final_out); a row cut across
// ranges a .. c writes, in range R, partial slot (R + k) s_q + j, k the number of sequences before
// b cut across ranges.  The next cut sequence starts in range c or later with k one higher, so
// each slot has one writer, slots stay below (2U - 2) s_q <= 2 n_workers s_q - 2 s_q, and the
// cut row (b, j) owns slots (a + k) s_q + j .. (c + k) s_q + j with stride s_q.  The helpers below
// are warp-collective (one warp of every CTA; all CTAs of a worker derive the same plan
// from the lengths).

struct Plan {
  long long T, U;   // total cost; ranges in use
  long long w0, w1; // this worker's cost range
  long long S;      // cost offset of the cursor sequence
  int b;            // cursor sequence
  int j;            // this worker's query token
  int k;            // sequences cut across ranges before the cursor sequence
  bool done;
};

// pages of row (b, j); a sequence's pages are those of its last query token (the longest row)
template <class P>
__device__ __forceinline__ int row_pages(const P& p, int r, bool report) {
  return (attended(p, r, report) + 63) / 64;
}
template <class P>
__device__ __forceinline__ int seq_pages(const P& p, int b, bool report) {
  return row_pages(p, b * p.s_q + p.s_q - 1, report);
}
template <int RC>
__device__ __forceinline__ int seq_cost(int pages) { return pages > 0 ? pages + RC : 0; }

template <int RC, class P>
__device__ long long total_cost(const P& p, int lane) {
  long long T = 0;
  for (int b0 = 0; b0 < p.batch; b0 += 32) {
    int c = b0 + lane < p.batch ? seq_cost<RC>(seq_pages(p, b0 + lane, false)) : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    T += c;
  }
  return T;
}

__device__ __forceinline__ long long worker_of(long long x, long long T, long long U) {
  return ((x + 1) * U + T - 1) / T - 1;  // the range that holds cost unit x
}
// whether pages [first, first + pages) of the cost line span more than one range
__device__ __forceinline__ bool is_split(long long first, int pages, long long T, long long U) {
  return pages > 0 && worker_of(first, T, U) != worker_of(first + pages - 1, T, U);
}

// Walk the sequences 32 at a time with their cost offsets; f(b, pages, first page's cost unit,
// cut sequences before b) for each sequence, lane-parallel.  f returns true for the sequence
// where the walk should stop (the lowest such sequence wins); the walk returns it (or -1).
template <int RC, class P, class F>
__device__ int walk_seqs(const P& p, long long T, long long U, int lane, F f) {
  long long S = 0;
  int K = 0;
  for (int b0 = 0; b0 < p.batch; b0 += 32) {
    const int b = b0 + lane;
    const int pb = b < p.batch ? seq_pages(p, b, false) : 0;
    const int cb = seq_cost<RC>(pb);
    int incl = cb;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const long long first = S + incl - cb + RC;
    const bool sp = b < p.batch && T > 0 && is_split(first, pb, T, U);
    const unsigned sm = __ballot_sync(0xffffffffu, sp);
    const int k = K + __popc(sm & ((1u << lane) - 1u));
    const bool stop = b < p.batch && f(b, pb, first, k);
    const unsigned m = __ballot_sync(0xffffffffu, stop);
    if (m) return b0 + __ffs(m) - 1;
    S += __shfl_sync(0xffffffffu, incl, 31);
    K += __popc(sm);
  }
  return -1;
}

// Each row's slots for the combine: first and last (stride s_q), -1 for a row without pages,
// the same slot twice for a row computed whole.  Also the one place that reports an
// out-of-range sequence length.
template <int RC, class P>
__device__ void write_rowinfo(const P& p, long long T, long long U, int lane) {
  walk_seqs<RC>(p, T, U, lane, [&](int b, int, long long first, int k) {
    for (int j = 0; j < p.s_q; ++j) {
      const int r = b * p.s_q + j;
      const int pr = row_pages(p, r, true);  // reports a bad length (once per sequence)
      int c0 = -1, c1 = -1;
      if (pr > 0) {
        const int a = (int)worker_of(first, T, U), c = (int)worker_of(first + pr - 1, T, U);
        c0 = a != c ? (a + k) * p.s_q + j : a;
        c1 = a != c ? (c + k) * p.s_q + j : a;
      }
      p.rowinfo[2 * r] = c0;
      p.rowinfo[2 * r + 1] = c1;
    }
    return false;
  });
}

// Position worker w's cursor on the first sequence whose cost range reaches past its start.
template <int RC, class P>
__device__ void plan_begin(const P& p, Plan& pl, int w, int lane) {
  pl.T = total_cost<RC>(p, lane);
  pl.U = min((long long)p.n_workers, pl.T);
  const int R = w / p.s_q;
  pl.j = w % p.s_q;
  pl.done = R >= pl.U;
  if (pl.done) return;
  pl.w0 = R * pl.T / pl.U;
  pl.w1 = (R + 1) * pl.T / pl.U;
  long long st_found = 0;
  int k_found = 0;
  const long long w0 = pl.w0;
  const int b = walk_seqs<RC>(p, pl.T, pl.U, lane, [&](int b, int pb, long long first, int k) {
    const bool hit = pb > 0 && first + pb > w0;  // (its boundary units, then its pages)
    if (hit) {
      st_found = first - RC;
      k_found = k;
    }
    return hit;
  });
  if (b < 0) {
    pl.done = true;
    return;
  }
  pl.b = b;
  pl.S = __shfl_sync(0xffffffffu, st_found, b & 31);
  pl.k = __shfl_sync(0xffffffffu, k_found, b & 31);
}

// The next segment of worker w (the sequences whose pages for its query token meet its range),
// advancing the cursor.  Every segment it returns holds at least one page.
template <int RC, class P>
__device__ Unit plan_next(const P& p, Plan& pl, int w, int lane) {
  Unit u = {0, 0, 0, 0, 0, 0, 0, 0};
  const int R = w / p.s_q;
  while (!pl.done && pl.S < pl.w1) {
    const int b = pl.b, r = b * p.s_q + pl.j;
    const int pb = seq_pages(p, b, false);
    const int A = attended(p, r, false), pr = (A + 63) / 64;
    const long long first = pl.S + RC;
    const long long g0 = max(pl.w0, first), g1 = min(pl.w1, first + pr);
    const bool hit = g1 > g0;
    if (hit) {
      u.b = b;
      u.j = pl.j;
      u.qrow = r;
      u.lo = (int)(g0 - first) * 64;
      u.hi = min(A, (int)(g1 - first) * 64);
      u.slot = (R + pl.k) * p.s_q + pl.j;
      u.final_out = is_split(first, pr, pl.T, pl.U) ? 0 : 1;
      u.valid = 1;
    }
    // move the cursor to the next sequence with pages
    pl.S += seq_cost<RC>(pb);
    if (is_split(first, pb, pl.T, pl.U)) ++pl.k;
    pl.done = true;
    if (pl.S < pl.w1) {
      for (int b0 = b + 1; b0 < p.batch; b0 += 32) {
        const int bb = b0 + lane;
        const unsigned m = __ballot_sync(0xffffffffu, bb < p.batch && seq_pages(p, bb, false) > 0);
        if (m) {
          pl.b = b0 + __ffs(m) - 1;
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

}  // namespace plan
}  // namespace mla
