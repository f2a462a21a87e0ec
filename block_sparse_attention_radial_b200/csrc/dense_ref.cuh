// Dense-masked reference kernel: fp32 scalar arithmetic on the CUDA cores.
//
// For every query row it visits the key blocks in order, looks each one up in
// a per-row bitmap built from the row's list, and for a listed block scores
// every key j < n, then folds the block into a running max / sum / output in
// fp32. It shares no code with the tensor-core kernel and exists to check it
// on full tensors. Two threads serve one query row, each holding half of the
// head dimension.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "device_status.cuh"

namespace bsa {

struct RefParams {
  const __nv_bfloat16 *q, *k, *v;
  __nv_bfloat16 *out;
  float *lse;
  const int32_t *row_ptr, *col_idx;
  int32_t heads, n, nqb, nkb, num_lists, nnz;
  float scale;
};

template <int D, int BLK>
__global__ void __launch_bounds__(2 * BLK) dense_masked_ref_kernel(RefParams p) {
  constexpr int HD = D / 2;           // dims per thread
  constexpr int KS = D + 4;           // padded smem row stride (floats)
  constexpr int SS = BLK + 1;         // padded score row stride
  extern __shared__ float4 smem_f4[];
  float *ks = reinterpret_cast<float *>(smem_f4);
  float *vs = ks + BLK * KS;
  float *ss = vs + BLK * KS;
  uint32_t *bits = reinterpret_cast<uint32_t *>(ss + BLK * SS);

  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int r = threadIdx.x >> 1, half = threadIdx.x & 1;
  const int row = qb * BLK + r;
  const long long head_off = (static_cast<long long>(b) * p.heads + h) * p.n;

  float q[HD], o[HD];
#pragma unroll
  for (int d = 0; d < HD; ++d) {
    q[d] = row < p.n ? __bfloat162float(p.q[(head_off + row) * D + half * HD + d]) : 0.f;
    o[d] = 0.f;
  }

  const int words = (p.nkb + 31) >> 5;
  for (int i = threadIdx.x; i < words; i += blockDim.x) bits[i] = 0u;
  __syncthreads();
  const int list = p.num_lists > 1 ? h : 0;
  const long long lr = static_cast<long long>(list) * p.nqb + qb;
  const int a = min(max(p.row_ptr[lr], 0), p.nnz), e = min(max(p.row_ptr[lr + 1], 0), p.nnz);
  for (int i = a + threadIdx.x; i < e; i += blockDim.x) {
    const int kb = min(max(p.col_idx[i], 0), p.nkb - 1);
    atomicOr(&bits[kb >> 5], 1u << (kb & 31));
  }
  __syncthreads();

  float m = -INFINITY, l = 0.f;
  for (int kb = 0; kb < p.nkb; ++kb) {
    if (!((bits[kb >> 5] >> (kb & 31)) & 1u)) continue;  // block not listed
    const int valid = min(BLK, p.n - kb * BLK);
    __syncthreads();
    for (int i = threadIdx.x; i < BLK * D; i += blockDim.x) {
      const int j = i / D, d = i % D;
      const bool ok = j < valid;
      const long long g = (head_off + kb * BLK + j) * D + d;
      ks[j * KS + d] = ok ? __bfloat162float(p.k[g]) : 0.f;
      vs[j * KS + d] = ok ? __bfloat162float(p.v[g]) : 0.f;
    }
    __syncthreads();
    float mx = -INFINITY;
    for (int j = 0; j < valid; ++j) {
      const float4 *kr = reinterpret_cast<const float4 *>(ks + j * KS + half * HD);
      float part = 0.f;
#pragma unroll
      for (int c = 0; c < HD / 4; ++c) {
        const float4 kv = kr[c];
        part = fmaf(q[4 * c], kv.x, part);
        part = fmaf(q[4 * c + 1], kv.y, part);
        part = fmaf(q[4 * c + 2], kv.z, part);
        part = fmaf(q[4 * c + 3], kv.w, part);
      }
      const float s = (part + __shfl_xor_sync(0xffffffffu, part, 1)) * p.scale;
      if (half == 0) ss[r * SS + j] = s;
      mx = fmaxf(mx, s);
    }
    __syncwarp();
    const float mn = fmaxf(m, mx);
    const float alpha = expf(m - mn);  // m = -inf on the first listed block: alpha = 0
    l *= alpha;
#pragma unroll
    for (int d = 0; d < HD; ++d) o[d] *= alpha;
    for (int j = 0; j < valid; ++j) {
      const float pj = expf(ss[r * SS + j] - mn);
      l += pj;
      const float4 *vr = reinterpret_cast<const float4 *>(vs + j * KS + half * HD);
#pragma unroll
      for (int c = 0; c < HD / 4; ++c) {
        const float4 vv = vr[c];
        o[4 * c] = fmaf(pj, vv.x, o[4 * c]);
        o[4 * c + 1] = fmaf(pj, vv.y, o[4 * c + 1]);
        o[4 * c + 2] = fmaf(pj, vv.z, o[4 * c + 2]);
        o[4 * c + 3] = fmaf(pj, vv.w, o[4 * c + 3]);
      }
    }
    m = mn;
  }

  if (row < p.n) {
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int d = 0; d < HD; ++d)
      p.out[(head_off + row) * D + half * HD + d] = __float2bfloat16_rn(o[d] * inv);
    if (half == 0 && p.lse) p.lse[head_off + row] = l > 0.f ? m + logf(l) : -INFINITY;
  }
}

template <int D, int BLK>
constexpr size_t dense_ref_smem_bytes(int nkb) {
  return static_cast<size_t>(2 * BLK * (D + 4) + BLK * (BLK + 1)) * sizeof(float) +
         static_cast<size_t>((nkb + 31) / 32) * sizeof(uint32_t);
}

}  // namespace bsa
