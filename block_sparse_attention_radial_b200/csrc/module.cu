// libbsa: the radial attention module forward and backward
// (bsa_attn_module_fwd, bsa_attn_module_bwd).
//
// The skill page's RadialAttention module ("Radial Attention" skill page,
// Step 2, RadialAttention.__init__ / forward) projects x with three
// nn.Linear layers, views each result as [batch, n, heads, head_dim] and
// transposes it to [batch, heads, n, head_dim], runs the masked softmax
// attention, transposes back, merges the heads and applies out_proj.
//
// Here the three projections are one GEMM against the stacked weight
// [q_proj; k_proj; v_proj] (bias in the GEMM epilogue), whose token-major
// output [batch*n, 3*heads*head_dim] the attention kernels read in place
// through strided TMA descriptors; the attention writes its output in
// [batch, n, heads, head_dim] order, which is already the row-major
// [batch*n, C] operand of out_proj. No transpose or copy runs between the
// three launches. Every GEMM, forward and backward, is the library's tcgen05
// GEMM (gemm_sm100.cuh: bf16 inputs, fp32 accumulation in tensor memory,
// bf16 output), which reads either operand in either orientation, so the
// backward's transposed products need no transposed copies either.

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>

#include "bsa.h"
#include "gemm.h"

namespace {

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Scratch layout inside the caller's forward workspace: the attention's work
// order, the q/k/v projection, the attention output and lse (kept for the
// backward).
struct ModuleLayout {
  size_t order, qkv, attn, lse, total;
};

ModuleLayout module_layout(int32_t batch, int32_t n, int32_t heads, int32_t head_dim,
                           const bsa_block_lists *l) {
  ModuleLayout w;
  const size_t rows = static_cast<size_t>(batch) * n;
  const size_t C = static_cast<size_t>(heads) * head_dim;
  w.order = 0;
  w.qkv = align256(bsa_attn_fwd_workspace_bytes(batch, heads, l));
  w.attn = w.qkv + align256(rows * 3 * C * 2);
  w.lse = w.attn + align256(rows * C * 2);
  w.total = w.lse + align256(rows * heads * sizeof(float));
  return w;
}

// Scratch layout of the backward's own workspace: the attention output's
// gradient, the q/k/v gradients, the attention backward's scratch, the
// column-sum partials.
constexpr int kColsumChunks = 32;  // row chunks of the bias-gradient sums

struct ModuleBwdLayout {
  size_t dattn, dqkv, attn_ws, partial, total;
};

ModuleBwdLayout module_bwd_layout(int32_t batch, int32_t n, int32_t heads, int32_t head_dim,
                                  const bsa_block_lists *l) {
  ModuleBwdLayout w;
  const size_t rows = static_cast<size_t>(batch) * n;
  const size_t C = static_cast<size_t>(heads) * head_dim;
  w.dattn = 0;
  w.dqkv = align256(rows * C * 2);
  w.attn_ws = w.dqkv + align256(rows * 3 * C * 2);
  w.partial = w.attn_ws + align256(bsa_attn_bwd_workspace_bytes(batch, heads, n, l));
  w.total = w.partial + align256(static_cast<size_t>(kColsumChunks) * 3 * C * sizeof(float));
  return w;
}

// Bias gradients: out[c] = sum over rows r of x[r, c] (bf16 [rows, cols]
// row-major, cols even), in a fixed order. Pass 1: CTA (strip, chunk) sums
// 64 columns over one chunk of rows (eight warps on interleaved rows, each
// lane two adjacent columns, loads unrolled four deep), the warps' partials
// combined in warp order; pass 2: one thread per column adds the chunks in
// chunk order.
__global__ void colsum_partial_kernel(const __nv_bfloat16 *x, long long rows, int cols,
                                      float *partial) {
  __shared__ float2 red[8][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x * 64 + 2 * lane;
  const long long per = (rows + gridDim.y - 1) / gridDim.y;
  const long long r0 = blockIdx.y * per, r1 = min(rows, r0 + per);
  float2 acc = make_float2(0.f, 0.f);
  if (c < cols) {
    long long r = r0 + warp;
    for (; r + 24 < r1; r += 32) {
      __nv_bfloat162 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        v[u] = *reinterpret_cast<const __nv_bfloat162 *>(x + (r + 8 * u) * cols + c);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 f = __bfloat1622float2(v[u]);
        acc.x += f.x;
        acc.y += f.y;
      }
    }
    for (; r < r1; r += 8) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(x + r * cols + c));
      acc.x += f.x;
      acc.y += f.y;
    }
  }
  red[warp][lane] = acc;
  __syncthreads();
  if (warp == 0 && c < cols) {
    float2 t = red[0][lane];
    for (int w = 1; w < 8; ++w) {
      t.x += red[w][lane].x;
      t.y += red[w][lane].y;
    }
    partial[static_cast<long long>(blockIdx.y) * cols + c] = t.x;
    partial[static_cast<long long>(blockIdx.y) * cols + c + 1] = t.y;
  }
}

__global__ void colsum_final_kernel(const float *partial, int chunks, int cols,
                                    __nv_bfloat16 *out) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= cols) return;
  float t = 0.f;
  for (int i = 0; i < chunks; ++i) t += partial[static_cast<long long>(i) * cols + c];
  out[c] = __float2bfloat16(t);
}

int colsum_bf16(const void *x, long long rows, int cols, float *partial, void *out,
                cudaStream_t stream) {
  dim3 grid((cols + 63) / 64, kColsumChunks);
  colsum_partial_kernel<<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16 *>(x), rows,
                                                  cols, partial);
  if (cudaGetLastError() != cudaSuccess) return BSA_ERR_CUDA;
  colsum_final_kernel<<<(cols + 255) / 256, 256, 0, stream>>>(partial, kColsumChunks, cols,
                                                              static_cast<__nv_bfloat16 *>(out));
  return cudaGetLastError() == cudaSuccess ? BSA_OK : BSA_ERR_CUDA;
}

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return na && nb && x < y + nb && y < x + na;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// out[rows, m] (row-major) = a[rows, k] (row-major) * w[m, k]^T + bias[m]:
// an nn.Linear layer, weight [out, in].
int linear_bf16(const void *a, const void *w, const void *bias, void *out, int64_t rows,
                int64_t m, int64_t k, cudaStream_t stream) {
  return bsa::gemm_bf16(a, k, false, w, k, false, bias, out, m, rows, m, k, stream);
}

}  // namespace

extern "C" {

size_t bsa_attn_module_workspace_bytes(int32_t batch, int32_t n, int32_t heads,
                                       int32_t head_dim, const bsa_block_lists *l) {
  if (!l || batch < 1 || n < 1 || heads < 1 || head_dim < 1) return 0;
  if (bsa_attn_fwd_workspace_bytes(batch, heads, l) == 0) return 0;
  return module_layout(batch, n, heads, head_dim, l).total;
}

int bsa_attn_module_fwd(const void *x, const void *w_qkv, const void *b_qkv, const void *w_out,
                        const void *b_out, int32_t batch, int32_t n, int32_t heads,
                        int32_t head_dim, float softmax_scale, const bsa_block_lists *l, void *y,
                        void *workspace, size_t workspace_bytes, bsa_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (!x || !w_qkv || !w_out || !y || !l || !workspace) return BSA_ERR_INVALID_ARG;
  if (batch < 1 || n < 1 || heads < 1) return BSA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return BSA_ERR_UNSUPPORTED;
  const ModuleLayout w = module_layout(batch, n, heads, head_dim, l);
  if (bsa_attn_fwd_workspace_bytes(batch, heads, l) == 0) return BSA_ERR_INVALID_ARG;
  if (workspace_bytes < w.total) return BSA_ERR_INVALID_ARG;
  const void *const ptrs[5] = {x, w_qkv, w_out, y, workspace};
  for (const void *p : ptrs)
    if (!aligned16(p)) return BSA_ERR_INVALID_ARG;
  if ((b_qkv && !aligned16(b_qkv)) || (b_out && !aligned16(b_out))) return BSA_ERR_INVALID_ARG;
  const int64_t rows = static_cast<int64_t>(batch) * n;
  const int64_t C = static_cast<int64_t>(heads) * head_dim;
  const size_t xb = static_cast<size_t>(rows * C * 2);
  const size_t wqb = static_cast<size_t>(3 * C * C * 2), wob = static_cast<size_t>(C * C * 2);
  if (overlaps(y, xb, x, xb) || overlaps(y, xb, workspace, w.total) ||
      overlaps(y, xb, w_qkv, wqb) || overlaps(y, xb, w_out, wob) ||
      overlaps(x, xb, workspace, w.total) || overlaps(w_qkv, wqb, workspace, w.total) ||
      overlaps(w_out, wob, workspace, w.total))
    return BSA_ERR_INVALID_ARG;

  uint8_t *ws = static_cast<uint8_t *>(workspace);
  uint16_t *qkv = reinterpret_cast<uint16_t *>(ws + w.qkv);
  void *attn = ws + w.attn;
  int st;

  // (1) qkv[b*n + i, :] = x[b, i, :] [q_proj; k_proj; v_proj]^T + bias
  if ((st = linear_bf16(x, w_qkv, b_qkv, qkv, rows, 3 * C, C, stream)) != BSA_OK) return st;
  // (2) attention on the q / k / v column slices of qkv, output token-major
  bsa_layout lqkv, lo;
  lqkv.batch_stride = static_cast<int64_t>(n) * 3 * C;
  lqkv.head_stride = head_dim;
  lqkv.token_stride = 3 * C;
  lo.batch_stride = static_cast<int64_t>(n) * C;
  lo.head_stride = head_dim;
  lo.token_stride = C;
  if ((st = bsa_attn_fwd_strided(qkv, &lqkv, qkv + C, &lqkv, qkv + 2 * C, &lqkv, batch, heads, n,
                                 head_dim, softmax_scale, l, attn, &lo,
                                 reinterpret_cast<float *>(ws + w.lse), ws + w.order, w.qkv,
                                 stream_)) != BSA_OK)
    return st;
  // (3) y = attn out_proj^T + bias
  return linear_bf16(attn, w_out, b_out, y, rows, C, C, stream);
}

size_t bsa_attn_module_bwd_workspace_bytes(int32_t batch, int32_t n, int32_t heads,
                                           int32_t head_dim, const bsa_block_lists *l) {
  if (!l || batch < 1 || n < 1 || heads < 1 || head_dim < 1) return 0;
  if (bsa_attn_bwd_workspace_bytes(batch, heads, n, l) == 0) return 0;
  return module_bwd_layout(batch, n, heads, head_dim, l).total;
}

int bsa_attn_module_bwd(const void *x, const void *w_qkv, const void *w_out, const void *dy,
                        int32_t batch, int32_t n, int32_t heads, int32_t head_dim,
                        float softmax_scale, const bsa_block_lists *l, const void *fwd_workspace,
                        size_t fwd_workspace_bytes, void *dx, void *dw_qkv, void *db_qkv,
                        void *dw_out, void *db_out, void *workspace, size_t workspace_bytes,
                        bsa_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (!x || !w_qkv || !w_out || !dy || !l || !fwd_workspace || !dx || !dw_qkv || !dw_out ||
      !workspace)
    return BSA_ERR_INVALID_ARG;
  if (batch < 1 || n < 1 || heads < 1) return BSA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return BSA_ERR_UNSUPPORTED;
  if (bsa_attn_fwd_workspace_bytes(batch, heads, l) == 0 ||
      bsa_attn_bwd_workspace_bytes(batch, heads, n, l) == 0)
    return BSA_ERR_INVALID_ARG;
  const ModuleLayout fw = module_layout(batch, n, heads, head_dim, l);
  const ModuleBwdLayout w = module_bwd_layout(batch, n, heads, head_dim, l);
  if (fwd_workspace_bytes < fw.total || workspace_bytes < w.total) return BSA_ERR_INVALID_ARG;
  const void *const ptrs[9] = {x, w_qkv, w_out, dy, fwd_workspace, dx, dw_qkv, dw_out, workspace};
  for (const void *p : ptrs)
    if (!aligned16(p)) return BSA_ERR_INVALID_ARG;
  if ((db_qkv && !aligned16(db_qkv)) || (db_out && !aligned16(db_out))) return BSA_ERR_INVALID_ARG;
  const int64_t rows = static_cast<int64_t>(batch) * n;
  const int64_t C = static_cast<int64_t>(heads) * head_dim;
  // outputs against everything else (inputs, both workspaces, each other)
  const size_t xb = static_cast<size_t>(rows * C * 2);
  const size_t wqb = static_cast<size_t>(3 * C * C * 2), wob = static_cast<size_t>(C * C * 2);
  const void *ins[6] = {x, w_qkv, w_out, dy, fwd_workspace, workspace};
  const size_t in_bytes[6] = {xb, wqb, wob, xb, fw.total, w.total};
  void *outs[5] = {dx, dw_qkv, dw_out, db_qkv, db_out};
  const size_t out_bytes[5] = {xb, wqb, wob, static_cast<size_t>(3 * C * 2),
                               static_cast<size_t>(C * 2)};
  for (int a = 0; a < 5; ++a) {
    if (!outs[a]) continue;
    for (int b = 0; b < 6; ++b)
      if (overlaps(outs[a], out_bytes[a], ins[b], in_bytes[b])) return BSA_ERR_INVALID_ARG;
    for (int b = a + 1; b < 5; ++b)
      if (outs[b] && overlaps(outs[a], out_bytes[a], outs[b], out_bytes[b]))
        return BSA_ERR_INVALID_ARG;
  }
  if (overlaps(workspace, w.total, fwd_workspace, fw.total)) return BSA_ERR_INVALID_ARG;

  const uint8_t *fws = static_cast<const uint8_t *>(fwd_workspace);
  const uint16_t *qkv = reinterpret_cast<const uint16_t *>(fws + fw.qkv);
  const void *attn = fws + fw.attn;
  const float *lse = reinterpret_cast<const float *>(fws + fw.lse);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  uint16_t *dattn = reinterpret_cast<uint16_t *>(ws + w.dattn);
  uint16_t *dqkv = reinterpret_cast<uint16_t *>(ws + w.dqkv);
  float *partial = reinterpret_cast<float *>(ws + w.partial);
  int st;

  // Row-major products; "MN-major" operands are read transposed in place.
  // (1) d_attn[rows, C] = dy[rows, C] w_out[C, C]
  if ((st = bsa::gemm_bf16(dy, C, false, w_out, C, true, nullptr, dattn, C, rows, C, C,
                           stream)) != BSA_OK)
    return st;
  // (2) dw_out[C, C] = dy^T attn   (both read from their [rows, C] storage)
  if ((st = bsa::gemm_bf16(dy, C, true, attn, C, true, nullptr, dw_out, C, C, C, rows,
                           stream)) != BSA_OK)
    return st;
  // (3) db_out = column sums of dy
  if (db_out && (st = colsum_bf16(dy, rows, static_cast<int>(C), partial, db_out, stream)) != BSA_OK)
    return st;
  // (4) attention backward on the strided views; dq, dk, dv land in the
  //     q / k / v column slices of dqkv [rows, 3C]
  bsa_layout lqkv, ltok;
  lqkv.batch_stride = static_cast<int64_t>(n) * 3 * C;
  lqkv.head_stride = head_dim;
  lqkv.token_stride = 3 * C;
  ltok.batch_stride = static_cast<int64_t>(n) * C;
  ltok.head_stride = head_dim;
  ltok.token_stride = C;
  if ((st = bsa_attn_bwd_strided(qkv, &lqkv, qkv + C, &lqkv, qkv + 2 * C, &lqkv, attn, &ltok,
                                 dattn, &ltok, lse, batch, heads, n, head_dim, softmax_scale, l,
                                 dqkv, &lqkv, dqkv + C, &lqkv, dqkv + 2 * C, &lqkv,
                                 ws + w.attn_ws, w.partial - w.attn_ws, stream_)) != BSA_OK)
    return st;
  // (5) dw_qkv[3C, C] = dqkv^T x   (both read from their [rows, .] storage)
  if ((st = bsa::gemm_bf16(dqkv, 3 * C, true, x, C, true, nullptr, dw_qkv, C, 3 * C, C, rows,
                           stream)) != BSA_OK)
    return st;
  // (6) db_qkv = column sums of dqkv
  if (db_qkv &&
      (st = colsum_bf16(dqkv, rows, static_cast<int>(3 * C), partial, db_qkv, stream)) != BSA_OK)
    return st;
  // (7) dx[rows, C] = dqkv[rows, 3C] w_qkv[3C, C]
  return bsa::gemm_bf16(dqkv, 3 * C, false, w_qkv, C, true, nullptr, dx, C, rows, C, 3 * C,
                        stream);
}

}  // extern "C"
