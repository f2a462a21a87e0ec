// Block-list kernels: the radial mask builder, list validation and the
// longest-row-first work order used by the attention kernel.
#pragma once

#include <climits>
#include <cstdint>

#include "device_status.cuh"

namespace bsa {

// ----------------------------------------------------------- block helpers --

// Inclusive prefix sum over the CTA (blockDim.x a multiple of 32, <= 1024).
// `scratch` holds 32 ints. Returns this thread's inclusive sum; `total` gets
// the CTA total.
template <typename T>
__device__ T cta_inclusive_scan(T x, T *scratch, T &total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    T y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[warp] = x;
  __syncthreads();
  if (warp == 0) {
    T w = lane < nwarps ? scratch[lane] : T(0);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      T y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    scratch[lane] = w;
  }
  __syncthreads();
  if (warp > 0) x += scratch[warp - 1];
  total = scratch[nwarps - 1];
  __syncthreads();
  return x;
}

// ------------------------------------------------------------ radial mask --

// n = nv + text: the frames * tpf video tokens, then `text` text tokens.
struct RadialGeom {
  int32_t frames, tpf, block, n, nb, rstar, nv;
};

__device__ __forceinline__ int band_of(int d) { return 31 - __clz(d < 1 ? 1 : d); }

// Sets, in the shared bitmap `bits`, every key block of query block `qb`.
//
// For one query frame f_i and one key frame f_j the admitted keys of query
// in-frame position s form the window [st(s), st(s) + w) with
// st(s) = clamp(s - w/2, 0, S - w). st is non-decreasing in s and moves by at
// most one per step, so the union over the query block's positions
// [s_lo, s_hi] in that frame is the single interval [st(s_lo), st(s_hi) + w).
// Its key blocks are marked; the threads of the CTA share the (f_i, f_j) pairs.
//
// Text tokens (after the video tokens) are global: a query block holding a
// text token lists every key block, and every query block lists the key
// blocks that hold text tokens.
// Threads tid of nthr share the work (a CTA, or one warp of the attention
// kernel that generates rows ahead of its producer).
__device__ void radial_mark_row(const RadialGeom g, int qb, uint32_t *bits, int tid, int nthr) {
  const int t0 = qb * g.block;
  const int t1 = min(g.n, t0 + g.block);  // query tokens [t0, t1)
  if (t1 > g.nv) {
    for (int b = tid; b < g.nb; b += nthr) atomicOr(&bits[b >> 5], 1u << (b & 31));
    return;
  }
  for (int b = g.nv / g.block + tid; g.nv < g.n && b < g.nb; b += nthr)
    atomicOr(&bits[b >> 5], 1u << (b & 31));
  const int fa = t0 / g.tpf, fb = (t1 - 1) / g.tpf;
  const int pairs = (fb - fa + 1) * g.frames;
  for (int p = tid; p < pairs; p += nthr) {
    const int fi = fa + p / g.frames, fj = p % g.frames;
    const int d = abs(fi - fj);
    const int r = band_of(d);
    if (r > g.rstar && (d & ((1 << (r - g.rstar)) - 1)) != 0) continue;  // thinned frame
    const int w = max(1, g.tpf >> min(r, g.rstar));
    const int s_lo = max(t0, fi * g.tpf) - fi * g.tpf;
    const int s_hi = min(t1, (fi + 1) * g.tpf) - 1 - fi * g.tpf;
    const int st_lo = min(max(s_lo - w / 2, 0), g.tpf - w);
    const int st_hi = min(max(s_hi - w / 2, 0), g.tpf - w);
    const int b0 = (fj * g.tpf + st_lo) / g.block;
    const int b1 = (fj * g.tpf + st_hi + w - 1) / g.block;
    for (int b = b0; b <= b1; ++b) atomicOr(&bits[b >> 5], 1u << (b & 31));
  }
}

__device__ void radial_row_bitmap(const RadialGeom g, int qb, uint32_t *bits, int words) {
  for (int i = threadIdx.x; i < words; i += blockDim.x) bits[i] = 0u;
  __syncthreads();
  radial_mark_row(g, qb, bits, threadIdx.x, blockDim.x);
  __syncthreads();
}

// One CTA per query block: row length into row_ptr[row0 + qb + 1]. `row0` is
// the first row of this mask in a concatenation of several items' lists (0
// for a single mask).
__global__ void radial_count_kernel(RadialGeom g, int32_t *row_ptr, int row0) {
  extern __shared__ uint32_t bits[];
  __shared__ int scratch[32];
  const int words = (g.nb + 31) >> 5;
  radial_row_bitmap(g, blockIdx.x, bits, words);
  int c = 0;
  for (int i = threadIdx.x; i < words; i += blockDim.x) c += __popc(bits[i]);
  int total;
  cta_inclusive_scan(c, scratch, total);
  if (threadIdx.x == 0) {
    row_ptr[row0 + blockIdx.x + 1] = total;
    if (row0 == 0 && blockIdx.x == 0) row_ptr[0] = 0;
  }
}

// Single CTA: in-place inclusive scan of row_ptr[1..rows]; row_ptr[0] = 0.
__global__ void scan_rows_kernel(int32_t *row_ptr, int rows) {
  __shared__ long long scratch[32];
  long long carry = 0;
  for (int base = 0; base < rows; base += blockDim.x) {
    const int i = base + threadIdx.x;
    long long x = i < rows ? row_ptr[i + 1] : 0;
    long long total;
    long long inc = cta_inclusive_scan(x, scratch, total);
    const long long v = carry + inc;
    if (i < rows) {
      if (v > 0x7fffffffLL) record_status(6u /* BSA_ERR_CAPACITY */);
      row_ptr[i + 1] = static_cast<int32_t>(v > 0x7fffffffLL ? 0x7fffffffLL : v);
    }
    carry += total;
  }
}

// Writes the set bits of a row bitmap (`words` words) as ascending key-block
// indices from col_idx[start]; entries at or beyond `capacity` are not written
// and record BSA_ERR_CAPACITY. Each thread owns a contiguous run of words, so
// ascending thread order is ascending block order. `scratch` holds 32 ints.
__device__ void write_row_ascending(const uint32_t *bits, int words, long long start,
                                    int32_t *col_idx, long long capacity, int *scratch) {
  const int per = (words + blockDim.x - 1) / blockDim.x;
  const int w0 = min(words, threadIdx.x * per), w1 = min(words, w0 + per);
  int c = 0;
  for (int i = w0; i < w1; ++i) c += __popc(bits[i]);
  int total;
  const int inc = cta_inclusive_scan(c, scratch, total);
  long long pos = start + (inc - c);
  for (int i = w0; i < w1; ++i) {
    uint32_t b = bits[i];
    while (b) {
      const int t = __ffs(b) - 1;
      b &= b - 1;
      if (pos < capacity) {
        col_idx[pos] = i * 32 + t;
      } else {
        record_status(6u /* BSA_ERR_CAPACITY */);
      }
      ++pos;
    }
  }
}

// One CTA per query block: write the row's key blocks in ascending order
// (key blocks of this mask's own item, from 0).
__global__ void radial_fill_kernel(RadialGeom g, const int32_t *row_ptr, int row0,
                                   int32_t *col_idx, long long capacity) {
  extern __shared__ uint32_t bits[];
  __shared__ int scratch[32];
  const int words = (g.nb + 31) >> 5;
  radial_row_bitmap(g, blockIdx.x, bits, words);
  write_row_ascending(bits, words, row_ptr[row0 + blockIdx.x], col_idx, capacity, scratch);
}

// ------------------------------------------------------------- validation --

// Grid-stride over rows; row_ptr has already been checked on the host to be
// monotone and bounded by nnz, so every read here is in bounds.
__global__ void validate_cols_kernel(const int32_t *row_ptr, const int32_t *col_idx, int rows,
                                     int nkb) {
  for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < rows; r += gridDim.x * blockDim.x) {
    const int a = row_ptr[r], b = row_ptr[r + 1];
    int prev = -1;
    for (int e = a; e < b; ++e) {
      const int c = col_idx[e];
      if (c <= prev || c >= nkb) {
        record_status(5u /* BSA_ERR_BAD_LISTS */);
        break;
      }
      prev = c;
    }
  }
}

// ------------------------------------------------------------ work order --

// ord[rank] = the index with the rank-th largest cost (ties: lower index
// first), ranked by counting so the order is deterministic. The CTA's threads
// share the work; `cost` is complete before the call.
__device__ __forceinline__ void rank_by_cost(const int *cost, int count, int32_t *ord) {
  for (int r = threadIdx.x; r < count; r += blockDim.x) {
    const int c = cost[r];
    int rank = 0;
    for (int o = 0; o < count; ++o) {
      const int co = cost[o];
      rank += (co > c) || (co == c && o < r);
    }
    ord[rank] = r;
  }
}

// One CTA per list. order[list * nqb + rank] = query block with the rank-th
// longest row (ties: lower block first). Rows are ranked by counting, which
// keeps the order deterministic. Lists with more rows than fit in shared
// memory keep their natural order.
__global__ void lpt_order_kernel(const int32_t *row_ptr, int nqb, int nnz, int32_t *order,
                                 int max_smem_rows) {
  extern __shared__ int cost[];
  const int list = blockIdx.x;
  const int32_t *rp = row_ptr + static_cast<long long>(list) * nqb;
  int32_t *ord = order + static_cast<long long>(list) * nqb;
  if (nqb > max_smem_rows) {
    for (int r = threadIdx.x; r < nqb; r += blockDim.x) ord[r] = r;
    return;
  }
  for (int r = threadIdx.x; r < nqb; r += blockDim.x) {
    const int a = min(max(rp[r], 0), nnz), b = min(max(rp[r + 1], 0), nnz);
    cost[r] = max(b - a, 0);
  }
  __syncthreads();
  for (int r = threadIdx.x; r < nqb; r += blockDim.x) {
    const int c = cost[r];
    int rank = 0;
    for (int o = 0; o < nqb; ++o) {
      const int co = cost[o];
      rank += (co > c) || (co == c && o < r);
    }
    ord[rank] = r;
  }
}

// One CTA per list: order[list * npairs + rank] = query-block pair (2p, 2p+1)
// with the rank-th longest union of key blocks (ties: lower pair first).
// Lists whose pair count does not fit in shared memory keep natural order.
// Also zeroes `item_counter` (when given), the attention kernel's work
// counter (this kernel runs before it in stream order).
__global__ void pair_order_kernel(const int32_t *row_ptr, const int32_t *col_idx, int nqb,
                                  int nnz, int32_t *order, int max_smem_rows,
                                  int32_t *item_counter) {
  extern __shared__ int cost[];
  if (item_counter && blockIdx.x == 0 && threadIdx.x == 0) *item_counter = 0;
  const int list = blockIdx.x;
  const int npairs = (nqb + 1) / 2;
  const int32_t *rp = row_ptr + static_cast<long long>(list) * nqb;
  int32_t *ord = order + static_cast<long long>(list) * npairs;
  if (npairs > max_smem_rows) {
    for (int r = threadIdx.x; r < npairs; r += blockDim.x) ord[r] = r;
    return;
  }
  // one warp per pair: |A u B| = |A| + |B| - |A n B|, the lanes looking
  // A's entries up in B (sorted) by binary search
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  for (int pr = warp; pr < npairs; pr += nwarps) {
    const int qa = 2 * pr;
    const int ia = min(max(rp[qa], 0), nnz), ea = max(ia, min(max(rp[qa + 1], 0), nnz));
    int ib = 0, eb = 0;
    if (qa + 1 < nqb) {
      ib = min(max(rp[qa + 1], 0), nnz);
      eb = max(ib, min(max(rp[qa + 2], 0), nnz));
    }
    int common = 0;
    for (int e = ia + lane; e < ea; e += 32) {
      const int v = col_idx[e];
      int lo = ib, hi = eb;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (col_idx[mid] < v) lo = mid + 1;
        else hi = mid;
      }
      common += (lo < eb && col_idx[lo] == v) ? 1 : 0;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) common += __shfl_xor_sync(0xffffffffu, common, o);
    if (lane == 0) cost[pr] = (ea - ia) + (eb - ib) - common;
  }
  __syncthreads();
  rank_by_cost(cost, npairs, ord);
}

}  // namespace bsa
