// Row generators: the key blocks of one query-block row computed from an
// analytic description instead of read from a column list, so the attention
// kernel needs no col_idx at all (the Sparse-vDiT skill page, "CUDA kernel
// invocation (pseudo-code)", runs pattern-specialised kernels; the Compact
// Attention abstract's tile-aligned windows; the radial rule of the "Radial
// Attention" skill page, Step 1, and of the thismoment.ai blog, "How Radial
// Attention Works").
//
// Each generator returns a row's key blocks in ascending order, exactly the
// blocks the list builders (patterns.cuh, lists.cuh) would write for that row,
// and answers membership of one block (used for the ragged last key block).
// Row lengths still come from the builders' count pass (row_ptr only).
#pragma once

#include <climits>
#include <cstdint>

#include "bsa.h"
#include "lists.cuh"
#include "patterns.cuh"

namespace bsa {

// ------------------------------------------------------------ tile patterns

// Row qb of one tile pattern: the union of the diagonal bands
// qb + lo <= kb <= qb + hi, the axial term ((kb - qb) within a of a multiple
// of the period P) and the stripe columns, over key blocks [0, nkb). The
// descriptor may sit in shared or global memory; malformed fields are clamped
// (the count pass reports them). Blocks come out in ascending order; the walk
// only moves forward, so each term keeps its next candidate.
struct PatternRow {
  const bsa_tile_pattern *pat;
  const int32_t *columns;
  int qb, nkb, x;  // x: the smallest key block not yet returned
  int run_end;     // blocks [x, run_end] are known to be in the row (one band)
  int nbands, cb, ce;
  // Each term's smallest block >= x found so far (INT_MAX: none left); a term
  // is searched again only once the walk has passed its candidate.
  int c_band, band_until, c_axial, c_stripe;

  __device__ __forceinline__ void reset(const bsa_tile_pattern *p, const int32_t *cols,
                                        long long num_columns, int q, int n) {
    pat = p;
    columns = cols;
    qb = q;
    nkb = n;
    x = 0;
    run_end = -1;
    c_band = c_axial = c_stripe = -1;
    band_until = -1;
    nbands = min(max(p->num_bands, 0), BSA_TILE_PATTERN_MAX_BANDS);
    cb = static_cast<int>(min(max(static_cast<long long>(p->columns_begin), 0LL), num_columns));
    ce = static_cast<int>(min(max(static_cast<long long>(p->columns_end), 0LL), num_columns));
  }

  // Smallest band block >= from (INT_MAX when none); `until` gets the end of
  // the band that holds it (every block of a band is in the row).
  __device__ __forceinline__ int band_from(int from, int &until) const {
    int best = INT_MAX;
    until = -1;
#pragma unroll 4
    for (int t = 0; t < nbands; ++t) {
      const long long lo = max(static_cast<long long>(qb) + pat->band_lo[t], 0LL);
      const long long hi = min(static_cast<long long>(qb) + pat->band_hi[t],
                               static_cast<long long>(nkb) - 1);
      if (lo <= hi && from <= hi) {
        const int c = static_cast<int>(max(lo, 1LL * from));
        if (c < best) {
          best = c;
          until = static_cast<int>(hi);
        } else if (c == best) {
          until = max(until, static_cast<int>(hi));
        }
      }
    }
    return best;
  }

  // Smallest block >= from with (kb - qb) within a of a multiple of P.
  __device__ __forceinline__ int axial_from(int from) const {
    const int P = pat->axial_period, a = pat->axial_halfwidth;
    if (P <= 0 || a < 0) return INT_MAX;
    if (2LL * a + 1 >= P) return from;  // every residue
    int d = (from - qb) % P;
    if (d < 0) d += P;
    const long long c = (d <= a || d >= P - a) ? from : 1LL * from + (P - a - d);
    return c < nkb ? static_cast<int>(c) : INT_MAX;
  }

  // Smallest stripe column >= from.
  __device__ __forceinline__ int stripe_from(int from) const {
    int best = INT_MAX;
    for (int e = cb; e < ce; ++e) {
      const int c = columns[e];
      if (c >= from && c < nkb) best = min(best, c);
    }
    return best;
  }

  __device__ __forceinline__ int next() {
    if (x <= run_end) return x++;  // inside a band run found earlier
    if (x >= nkb) return INT_MAX;
    if (c_band != INT_MAX && c_band < x) c_band = band_from(x, band_until);
    if (c_axial != INT_MAX && c_axial < x) c_axial = axial_from(x);
    if (c_stripe != INT_MAX && c_stripe < x) c_stripe = stripe_from(x);
    const int best = min(c_band, min(c_axial, c_stripe));
    if (best == INT_MAX || best >= nkb) return INT_MAX;
    run_end = best == c_band ? band_until : best;
    x = best + 1;
    return best;
  }

  __device__ __forceinline__ bool has(int kb) const {
    if (kb < 0 || kb >= nkb) return false;
    int until;
    return band_from(kb, until) == kb || axial_from(kb) == kb || stripe_from(kb) == kb;
  }
};

// ------------------------------------------------------------------- radial

// Bits, relative to key block `base`, of the key blocks that query positions
// [s_lo, s_hi] of frame fi admit in key frame fj (radial_mark_row's
// interval); 0 for a thinned frame.
// The generated path runs at block 128 (the two-tile kernel's block), so the
// block divisions are shifts.
constexpr int kGenBlockShift = 7;

__device__ __forceinline__ uint64_t radial_frame_bits(const RadialGeom &g, int fi, int fj,
                                                      int s_lo, int s_hi, int base) {
  const int d = abs(fi - fj);
  const int r = band_of(d);
  if (r > g.rstar && (d & ((1 << (r - g.rstar)) - 1)) != 0) return 0ull;
  const int w = max(1, g.tpf >> min(r, g.rstar));
  const int st_lo = min(max(s_lo - (w >> 1), 0), g.tpf - w);
  const int st_hi = min(max(s_hi - (w >> 1), 0), g.tpf - w);
  const int b0 = ((fj * g.tpf + st_lo) >> kGenBlockShift) - base;
  const int b1 = ((fj * g.tpf + st_hi + w - 1) >> kGenBlockShift) - base;
  const uint64_t upto = b1 >= 63 ? ~0ull : ((2ull << b1) - 1ull);
  return upto & ~((1ull << b0) - 1ull);
}

// Row qb of the joint radial mask (video tokens frame-major, then text
// tokens attended globally). Key frame by key frame, the blocks a frame's
// admitted windows touch are gathered in a 64-bit mask (a frame spans at most
// tokens_per_frame / block + 2 blocks, checked on the host) and returned in
// ascending order; a block shared by two frames is returned once.
struct RadialRow {
  RadialGeom g;
  int qb, fa, fb, t0, t1;  // the query block's frames and tokens [t0, t1)
  bool dense;              // the block holds a text token: every key block
  int fj, base, last;      // next key frame, the mask's first block, last returned
  uint64_t mask;

  __device__ __forceinline__ void reset(const RadialGeom &geo, int q) {
    g = geo;
    qb = q;
    t0 = q << kGenBlockShift;
    t1 = min(g.n, t0 + (1 << kGenBlockShift));
    dense = t1 > g.nv;
    fa = t0 / g.tpf;
    fb = (min(t1, g.nv) - 1) / g.tpf;
    fj = 0;
    base = 0;
    last = -1;
    mask = 0ull;
  }

  // Query positions of frame fi inside this block.
  __device__ __forceinline__ void span(int fi, int &s_lo, int &s_hi) const {
    s_lo = max(t0, fi * g.tpf) - fi * g.tpf;
    s_hi = min(t1, (fi + 1) * g.tpf) - 1 - fi * g.tpf;
  }

  __device__ __forceinline__ int next() {
    if (dense) {
      if (last + 1 >= g.nb) return INT_MAX;
      return ++last;
    }
    for (;;) {
      if (mask) {
        const int i = __ffsll(static_cast<long long>(mask)) - 1;
        mask &= mask - 1ull;
        const int kb = base + i;
        if (kb > last) {
          last = kb;
          return kb;
        }
        continue;
      }
      if (fj < g.frames) {
        base = (fj * g.tpf) >> kGenBlockShift;
        for (int fi = fa; fi <= fb; ++fi) {
          int s_lo, s_hi;
          span(fi, s_lo, s_hi);
          mask |= radial_frame_bits(g, fi, fj, s_lo, s_hi, base);
        }
        ++fj;
        continue;
      }
      if (g.nv < g.n) {  // text key blocks come last, in every row
        const int kb = max(last + 1, g.nv >> kGenBlockShift);
        if (kb < g.nb) {
          last = kb;
          return kb;
        }
      }
      return INT_MAX;
    }
  }

  // Whether key block kb is in the row (for the ragged last block).
  __device__ __forceinline__ bool has(int kb) const {
    if (kb < 0 || kb >= g.nb) return false;
    if (dense) return true;
    const int k0 = kb << kGenBlockShift, k1 = min(g.n, k0 + (1 << kGenBlockShift));  // key tokens
    if (k1 > g.nv) return true;                              // holds a text token
    const int kf0 = k0 / g.tpf, kf1 = (k1 - 1) / g.tpf;
    for (int fj = kf0; fj <= kf1; ++fj) {
      const int fbase = (fj * g.tpf) >> kGenBlockShift;
      for (int fi = fa; fi <= fb; ++fi) {
        int s_lo, s_hi;
        span(fi, s_lo, s_hi);
        if ((radial_frame_bits(g, fi, fj, s_lo, s_hi, fbase) >> (kb - fbase)) & 1ull) return true;
      }
    }
    return false;
  }
};

// ------------------------------------------------------------ work orders

// Union sizes of the query-block pairs (2p, 2p+1), one CTA per pair: the two
// rows' bitmaps (the list builders' own row marking) OR-ed and counted.
// cost[list * npairs + p]. Shared memory: one bitmap of nkb bits per row.
__global__ void radial_pair_union_kernel(RadialGeom g, int32_t *cost) {
  extern __shared__ uint32_t bits[];
  __shared__ int scratch[32];
  const int pr = blockIdx.x, words = (g.nb + 31) >> 5;
  for (int i = threadIdx.x; i < words; i += blockDim.x) bits[i] = 0u;
  __syncthreads();
  radial_mark_row(g, 2 * pr, bits, threadIdx.x, blockDim.x);
  if (2 * pr + 1 < g.nb) radial_mark_row(g, 2 * pr + 1, bits, threadIdx.x, blockDim.x);
  __syncthreads();
  int c = 0;
  for (int i = threadIdx.x; i < words; i += blockDim.x) c += __popc(bits[i]);
  int total;
  cta_inclusive_scan(c, scratch, total);
  if (threadIdx.x == 0) cost[pr] = total;
}

__global__ void pattern_pair_union_kernel(const bsa_tile_pattern *patterns,
                                          const int32_t *columns, long long num_columns, int nqb,
                                          int32_t *cost) {
  extern __shared__ uint32_t bits[];
  __shared__ int scratch[32];
  __shared__ bsa_tile_pattern p;
  const int npairs = (nqb + 1) / 2;
  const int list = blockIdx.x / npairs, pr = blockIdx.x % npairs;
  if (threadIdx.x == 0) p = patterns[list];
  __syncthreads();
  const int words = (nqb + 31) >> 5;
  const bool ok = pattern_ok(p, num_columns);
  pattern_row_bitmap(p, ok, columns, 2 * pr, nqb, bits, words);
  int c = 0;
  if (2 * pr + 1 < nqb) {
    // the second row's bitmap after the first, OR-ed into the count
    uint32_t *row2 = bits + words;
    pattern_row_bitmap(p, ok, columns, 2 * pr + 1, nqb, row2, words);
    for (int i = threadIdx.x; i < words; i += blockDim.x) c += __popc(bits[i] | row2[i]);
  } else {
    for (int i = threadIdx.x; i < words; i += blockDim.x) c += __popc(bits[i]);
  }
  int total;
  cta_inclusive_scan(c, scratch, total);
  if (threadIdx.x == 0) cost[blockIdx.x] = total;
}

// One CTA per list: order[list * npairs + rank] = the pair with the rank-th
// largest union (ties: lower pair first); lists with more pairs than fit in
// shared memory keep natural order. Also zeroes the work counter.
__global__ void rank_pairs_kernel(const int32_t *cost, int npairs, int32_t *order,
                                  int max_smem_rows, int32_t *item_counter) {
  extern __shared__ int c[];
  if (item_counter && blockIdx.x == 0 && threadIdx.x == 0) *item_counter = 0;
  int32_t *ord = order + static_cast<long long>(blockIdx.x) * npairs;
  if (npairs > max_smem_rows) {
    for (int r = threadIdx.x; r < npairs; r += blockDim.x) ord[r] = r;
    return;
  }
  for (int r = threadIdx.x; r < npairs; r += blockDim.x)
    c[r] = cost[static_cast<long long>(blockIdx.x) * npairs + r];
  __syncthreads();
  rank_by_cost(c, npairs, ord);
}

}  // namespace bsa
