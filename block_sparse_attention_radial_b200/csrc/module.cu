// libbsa: the radial attention module forward (bsa_attn_module_fwd).
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
// three launches. The two projections are plain dense GEMMs and run on
// cuBLASLt (bf16 inputs, fp32 accumulation, bf16 output).

#include <cublasLt.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <map>
#include <mutex>
#include <tuple>

#include "bsa.h"

namespace {

constexpr size_t kGemmScratch = size_t(32) << 20;  // cuBLASLt workspace
constexpr int kMaxDevices = 64;

std::mutex g_lt_mu;
cublasLtHandle_t g_lt[kMaxDevices] = {};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Scratch layout inside the caller's forward workspace: the attention's work
// order, the q/k/v projection, the attention output and lse (kept for the
// backward), the GEMM scratch.
struct ModuleLayout {
  size_t order, qkv, attn, lse, gemm, total;
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
  w.gemm = w.lse + align256(rows * heads * sizeof(float));
  w.total = w.gemm + kGemmScratch;
  return w;
}

// Scratch layout of the backward's own workspace: the attention output's
// gradient, the q/k/v gradients, the attention backward's scratch, the
// column-sum partials, the GEMM scratch.
constexpr int kColsumChunks = 32;  // row chunks of the bias-gradient sums

struct ModuleBwdLayout {
  size_t dattn, dqkv, attn_ws, partial, gemm, total;
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
  w.gemm = w.partial + align256(static_cast<size_t>(kColsumChunks) * 3 * C * sizeof(float));
  w.total = w.gemm + kGemmScratch;
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

int lt_handle(cublasLtHandle_t *h) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BSA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_lt_mu);
  if (!g_lt[dev] && cublasLtCreate(&g_lt[dev]) != CUBLAS_STATUS_SUCCESS) return BSA_ERR_CUDA;
  *h = g_lt[dev];
  return BSA_OK;
}

// Column-major GEMM on cuBLASLt: D (m x n, leading dimension ldd) =
// op(A) (m x k) * op(B) (k x n) [+ bias[m] on every column], bf16 operands,
// fp32 accumulation, bf16 D. Row-major matrices are their transposes in
// these terms (see the callers).
//
// The descriptors and the algorithm cuBLASLt's heuristic picks are built once
// per (device, shape, transposes, bias or not) and reused, so a call costs one
// enqueue on the host (the heuristic query alone takes longer than a small
// GEMM).
struct GemmPlan {
  int status = BSA_ERR_CUDA;
  cublasLtMatmulDesc_t op = nullptr;
  cublasLtMatrixLayout_t la = nullptr, lb = nullptr, lc = nullptr;
  cublasLtMatmulAlgo_t algo;
};

struct GemmKey {
  int dev;
  bool ta, tb, bias;
  int64_t m, n, k, lda, ldb, ldd;
  bool operator<(const GemmKey &o) const {
    return std::tie(dev, ta, tb, bias, m, n, k, lda, ldb, ldd) <
           std::tie(o.dev, o.ta, o.tb, o.bias, o.m, o.n, o.k, o.lda, o.ldb, o.ldd);
  }
};

std::mutex g_plan_mu;
std::map<GemmKey, GemmPlan> g_plans;

GemmPlan make_plan(cublasLtHandle_t h, const GemmKey &g) {
  GemmPlan p;
  if (cublasLtMatmulDescCreate(&p.op, CUBLAS_COMPUTE_32F, CUDA_R_32F) != CUBLAS_STATUS_SUCCESS)
    return p;
  const cublasOperation_t tA = g.ta ? CUBLAS_OP_T : CUBLAS_OP_N;
  const cublasOperation_t tB = g.tb ? CUBLAS_OP_T : CUBLAS_OP_N;
  cublasLtMatmulDescSetAttribute(p.op, CUBLASLT_MATMUL_DESC_TRANSA, &tA, sizeof(tA));
  cublasLtMatmulDescSetAttribute(p.op, CUBLASLT_MATMUL_DESC_TRANSB, &tB, sizeof(tB));
  if (g.bias) {
    const cublasLtEpilogue_t ep = CUBLASLT_EPILOGUE_BIAS;
    const cudaDataType_t bt = CUDA_R_16BF;
    cublasLtMatmulDescSetAttribute(p.op, CUBLASLT_MATMUL_DESC_EPILOGUE, &ep, sizeof(ep));
    cublasLtMatmulDescSetAttribute(p.op, CUBLASLT_MATMUL_DESC_BIAS_DATA_TYPE, &bt, sizeof(bt));
  }
  // stored shapes: A is (ta ? k x m : m x k), B is (tb ? n x k : k x n)
  if (cublasLtMatrixLayoutCreate(&p.la, CUDA_R_16BF, g.ta ? g.k : g.m, g.ta ? g.m : g.k, g.lda) !=
          CUBLAS_STATUS_SUCCESS ||
      cublasLtMatrixLayoutCreate(&p.lb, CUDA_R_16BF, g.tb ? g.n : g.k, g.tb ? g.k : g.n, g.ldb) !=
          CUBLAS_STATUS_SUCCESS ||
      cublasLtMatrixLayoutCreate(&p.lc, CUDA_R_16BF, g.m, g.n, g.ldd) != CUBLAS_STATUS_SUCCESS)
    return p;
  cublasLtMatmulPreference_t pref = nullptr;
  if (cublasLtMatmulPreferenceCreate(&pref) != CUBLAS_STATUS_SUCCESS) return p;
  const size_t scratch = kGemmScratch;
  cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES, &scratch,
                                       sizeof(scratch));
  cublasLtMatmulHeuristicResult_t res;
  int found = 0;
  const cublasStatus_t hs =
      cublasLtMatmulAlgoGetHeuristic(h, p.op, p.la, p.lb, p.lc, p.lc, pref, 1, &res, &found);
  cublasLtMatmulPreferenceDestroy(pref);
  if (hs != CUBLAS_STATUS_SUCCESS || found < 1) {
    p.status = BSA_ERR_UNSUPPORTED;
    return p;
  }
  p.algo = res.algo;
  p.status = BSA_OK;
  return p;
}

int gemm_bf16(cublasLtHandle_t h, bool ta, bool tb, int64_t m, int64_t n, int64_t k,
              const void *A, int64_t lda, const void *B, int64_t ldb, void *D, int64_t ldd,
              const void *bias, void *scratch, cudaStream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BSA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_plan_mu);  // the bias pointer is set on the shared desc
  const GemmKey key{dev, ta, tb, bias != nullptr, m, n, k, lda, ldb, ldd};
  auto it = g_plans.find(key);
  if (it == g_plans.end()) it = g_plans.emplace(key, make_plan(h, key)).first;
  GemmPlan &p = it->second;
  if (p.status != BSA_OK) return p.status;
  if (bias)
    cublasLtMatmulDescSetAttribute(p.op, CUBLASLT_MATMUL_DESC_BIAS_POINTER, &bias, sizeof(bias));
  const float alpha = 1.f, beta = 0.f;
  if (cublasLtMatmul(h, p.op, &alpha, A, p.la, B, p.lb, &beta, D, p.lc, D, p.lc, &p.algo, scratch,
                     kGemmScratch, stream) != CUBLAS_STATUS_SUCCESS)
    return BSA_ERR_CUDA;
  return BSA_OK;
}

// out[rows, m] (row-major) = a[rows, k] (row-major) * w[m, k]^T + bias[m]:
// column-major out^T (m x rows) = op_T(w^T) * a^T, w's row-major storage being
// the k x m column-major matrix w^T.
int linear_bf16(cublasLtHandle_t h, const void *a, const void *w, const void *bias, void *out,
                int64_t rows, int64_t m, int64_t k, void *scratch, cudaStream_t stream) {
  return gemm_bf16(h, true, false, m, rows, k, w, k, a, k, out, m, bias, scratch, stream);
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
  cublasLtHandle_t h;
  int st;
  if ((st = lt_handle(&h)) != BSA_OK) return st;

  // (1) qkv[b*n + i, :] = x[b, i, :] [q_proj; k_proj; v_proj]^T + bias
  if ((st = linear_bf16(h, x, w_qkv, b_qkv, qkv, rows, 3 * C, C, ws + w.gemm, stream)) !=
      BSA_OK)
    return st;
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
  return linear_bf16(h, attn, w_out, b_out, y, rows, C, C, ws + w.gemm, stream);
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
  void *scratch = ws + w.gemm;
  cublasLtHandle_t h;
  int st;
  if ((st = lt_handle(&h)) != BSA_OK) return st;

  // Row-major [r, c] matrices are column-major [c, r] below.
  // (1) d_attn = dy w_out            : d_attn^T (C x rows) = w_out^T dy^T
  if ((st = gemm_bf16(h, false, false, C, rows, C, w_out, C, dy, C, dattn, C, nullptr, scratch,
                      stream)) != BSA_OK)
    return st;
  // (2) dw_out = dy^T attn           : dw_out^T (C x C) = attn^T dy
  if ((st = gemm_bf16(h, false, true, C, C, rows, attn, C, dy, C, dw_out, C, nullptr, scratch,
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
  // (5) dw_qkv = dqkv^T x            : dw_qkv^T (C x 3C) = x^T dqkv
  if ((st = gemm_bf16(h, false, true, C, 3 * C, rows, x, C, dqkv, 3 * C, dw_qkv, C, nullptr,
                      scratch, stream)) != BSA_OK)
    return st;
  // (6) db_qkv = column sums of dqkv
  if (db_qkv &&
      (st = colsum_bf16(dqkv, rows, static_cast<int>(3 * C), partial, db_qkv, stream)) != BSA_OK)
    return st;
  // (7) dx = dqkv w_qkv              : dx^T (C x rows) = w_qkv^T dqkv^T
  return gemm_bf16(h, false, false, C, rows, 3 * C, w_qkv, C, dqkv, 3 * C, dx, C, nullptr,
                   scratch, stream);
}

}  // extern "C"
