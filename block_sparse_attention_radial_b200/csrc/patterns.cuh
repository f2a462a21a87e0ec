// Tile-pattern list builder: one pattern per head (diagonal bands, an axial
// term and vertical-stripe columns; the families of the Sparse-vDiT skill
// page, "Sparse attention patterns", and the Compact Attention abstract's
// dual window) expanded into CSR block lists, one CTA per row.
#pragma once

#include <cstdint>

#include "bsa.h"
#include "device_status.cuh"
#include "lists.cuh"

namespace bsa {

// Bits of the key-block interval [lo, hi] that fall in bitmap word `word`.
__device__ __forceinline__ uint32_t interval_word(long long lo, long long hi, int word) {
  const long long base = 32LL * word;
  const long long a = lo > base ? lo : base;
  const long long b = hi < base + 31 ? hi : base + 31;
  if (a > b) return 0u;
  const int s = static_cast<int>(a - base), e = static_cast<int>(b - base);
  const uint32_t upto = e == 31 ? 0xffffffffu : ((1u << (e + 1)) - 1u);
  return upto & ~((1u << s) - 1u);
}

__device__ __forceinline__ bool pattern_ok(const bsa_tile_pattern &p, long long num_columns) {
  return p.num_bands >= 0 && p.num_bands <= BSA_TILE_PATTERN_MAX_BANDS && p.axial_period >= 0 &&
         p.axial_halfwidth >= 0 && p.columns_begin >= 0 && p.columns_begin <= p.columns_end &&
         p.columns_end <= num_columns;
}

// The words [tid, tid + nthr, ...) of a row's bitmap from its bands and
// axial term (no stripe columns yet); key blocks >= nkb stay clear.
__device__ void pattern_row_words(const bsa_tile_pattern &p, bool ok, int qb, int nkb,
                                  uint32_t *bits, int words, int tid, int nthr) {
  for (int wd = tid; wd < words; wd += nthr) {
    uint32_t m = 0u;
    if (ok) {
      for (int t = 0; t < p.num_bands; ++t)
        m |= interval_word(static_cast<long long>(qb) + p.band_lo[t],
                           static_cast<long long>(qb) + p.band_hi[t], wd);
      const int P = p.axial_period, a = p.axial_halfwidth;
      if (P > 0) {
        if (2LL * a + 1 >= P) {
          m = 0xffffffffu;  // every residue is within a of a multiple of P
        } else {
          for (int i = 0; i < 32; ++i) {
            int r = (wd * 32 + i - qb) % P;
            if (r < 0) r += P;
            if (r <= a || r >= P - a) m |= 1u << i;
          }
        }
      }
    }
    const long long left = static_cast<long long>(nkb) - 32LL * wd;  // key blocks in this word
    if (left < 32) m &= left <= 0 ? 0u : ((1u << left) - 1u);
    bits[wd] = m;
  }
}

// The stripe columns OR-ed into the row's bitmap (after its words are
// written); a column outside [0, nkb) is an argument error when `report`.
__device__ void pattern_row_columns(const bsa_tile_pattern &p, const int32_t *columns, int nkb,
                                    uint32_t *bits, int tid, int nthr, bool report) {
  for (long long e = static_cast<long long>(p.columns_begin) + tid; e < p.columns_end; e += nthr) {
    const int c = columns[e];
    if (c >= 0 && c < nkb) atomicOr(&bits[c >> 5], 1u << (c & 31));
    else if (report) record_status(1u /* BSA_ERR_INVALID_ARG */);
  }
}

// Row qb of pattern p as a bitmap over the nkb key blocks. Each thread builds
// whole words from the band and axial terms; the stripe columns are then OR-ed
// in. Ends with the CTA synchronised.
__device__ void pattern_row_bitmap(const bsa_tile_pattern &p, bool ok, const int32_t *columns,
                                   int qb, int nkb, uint32_t *bits, int words) {
  pattern_row_words(p, ok, qb, nkb, bits, words, threadIdx.x, blockDim.x);
  __syncthreads();
  if (ok) {
    pattern_row_columns(p, columns, nkb, bits, threadIdx.x, blockDim.x, true);
  } else if (threadIdx.x == 0) {
    record_status(1u /* BSA_ERR_INVALID_ARG */);
  }
  __syncthreads();
}

// One CTA per row (list * nqb + qb): row length into row_ptr[row + 1].
__global__ void pattern_count_kernel(const bsa_tile_pattern *patterns, const int32_t *columns,
                                     long long num_columns, int nqb, int32_t *row_ptr) {
  extern __shared__ uint32_t bits[];
  __shared__ int scratch[32];
  __shared__ bsa_tile_pattern p;
  const int row = blockIdx.x, list = row / nqb, qb = row % nqb;
  if (threadIdx.x == 0) p = patterns[list];
  __syncthreads();
  const int words = (nqb + 31) >> 5;
  pattern_row_bitmap(p, pattern_ok(p, num_columns), columns, qb, nqb, bits, words);
  int c = 0;
  for (int i = threadIdx.x; i < words; i += blockDim.x) c += __popc(bits[i]);
  int total;
  cta_inclusive_scan(c, scratch, total);
  if (threadIdx.x == 0) {
    row_ptr[row + 1] = total;
    if (row == 0) row_ptr[0] = 0;
  }
}

// One CTA per row: the row's key blocks in ascending order at row_ptr[row].
__global__ void pattern_fill_kernel(const bsa_tile_pattern *patterns, const int32_t *columns,
                                    long long num_columns, int nqb, const int32_t *row_ptr,
                                    int32_t *col_idx, long long capacity) {
  extern __shared__ uint32_t bits[];
  __shared__ int scratch[32];
  __shared__ bsa_tile_pattern p;
  const int row = blockIdx.x, list = row / nqb, qb = row % nqb;
  if (threadIdx.x == 0) p = patterns[list];
  __syncthreads();
  const int words = (nqb + 31) >> 5;
  pattern_row_bitmap(p, pattern_ok(p, num_columns), columns, qb, nqb, bits, words);
  write_row_ascending(bits, words, row_ptr[row], col_idx, capacity, scratch);
}

}  // namespace bsa
