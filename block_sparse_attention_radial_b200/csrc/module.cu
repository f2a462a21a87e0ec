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

// Scratch layout inside the caller's workspace.
struct ModuleLayout {
  size_t order, qkv, attn, gemm, total;
};

ModuleLayout module_layout(int32_t batch, int32_t n, int32_t heads, int32_t head_dim,
                           const bsa_block_lists *l) {
  ModuleLayout w;
  const size_t rows = static_cast<size_t>(batch) * n;
  const size_t C = static_cast<size_t>(heads) * head_dim;
  w.order = 0;
  w.qkv = align256(bsa_attn_fwd_workspace_bytes(batch, heads, l));
  w.attn = w.qkv + align256(rows * 3 * C * 2);
  w.gemm = w.attn + align256(rows * C * 2);
  w.total = w.gemm + kGemmScratch;
  return w;
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

// out[rows, m] (row-major) = a[rows, k] (row-major) * w[m, k]^T + bias[m].
// In cuBLASLt's column-major terms: out^T (m x rows) = op_T(w^T) * a^T, where
// w^T is w's row-major storage read as a k x m column-major matrix.
//
// The descriptors and the algorithm cuBLASLt's heuristic picks are built once
// per (device, shape, bias or not) and reused, so a call costs one enqueue on
// the host (the heuristic query alone takes longer than a small GEMM).
struct GemmPlan {
  int status = BSA_ERR_CUDA;
  cublasLtMatmulDesc_t op = nullptr;
  cublasLtMatrixLayout_t la = nullptr, lb = nullptr, lc = nullptr;
  cublasLtMatmulAlgo_t algo;
};

struct GemmKey {
  int dev;
  int64_t rows, m, k;
  bool bias;
  bool operator<(const GemmKey &o) const {
    return std::tie(dev, rows, m, k, bias) < std::tie(o.dev, o.rows, o.m, o.k, o.bias);
  }
};

std::mutex g_plan_mu;
std::map<GemmKey, GemmPlan> g_plans;

GemmPlan make_plan(cublasLtHandle_t h, int64_t rows, int64_t m, int64_t k, bool bias) {
  GemmPlan p;
  if (cublasLtMatmulDescCreate(&p.op, CUBLAS_COMPUTE_32F, CUDA_R_32F) != CUBLAS_STATUS_SUCCESS)
    return p;
  const cublasOperation_t tA = CUBLAS_OP_T, tB = CUBLAS_OP_N;
  cublasLtMatmulDescSetAttribute(p.op, CUBLASLT_MATMUL_DESC_TRANSA, &tA, sizeof(tA));
  cublasLtMatmulDescSetAttribute(p.op, CUBLASLT_MATMUL_DESC_TRANSB, &tB, sizeof(tB));
  if (bias) {
    const cublasLtEpilogue_t ep = CUBLASLT_EPILOGUE_BIAS;
    const cudaDataType_t bt = CUDA_R_16BF;
    cublasLtMatmulDescSetAttribute(p.op, CUBLASLT_MATMUL_DESC_EPILOGUE, &ep, sizeof(ep));
    cublasLtMatmulDescSetAttribute(p.op, CUBLASLT_MATMUL_DESC_BIAS_DATA_TYPE, &bt, sizeof(bt));
  }
  if (cublasLtMatrixLayoutCreate(&p.la, CUDA_R_16BF, k, m, k) != CUBLAS_STATUS_SUCCESS ||
      cublasLtMatrixLayoutCreate(&p.lb, CUDA_R_16BF, k, rows, k) != CUBLAS_STATUS_SUCCESS ||
      cublasLtMatrixLayoutCreate(&p.lc, CUDA_R_16BF, m, rows, m) != CUBLAS_STATUS_SUCCESS)
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

int linear_bf16(cublasLtHandle_t h, const void *a, const void *w, const void *bias, void *out,
                int64_t rows, int64_t m, int64_t k, void *scratch, cudaStream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BSA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_plan_mu);  // the bias pointer is set on the shared desc
  const GemmKey key{dev, rows, m, k, bias != nullptr};
  auto it = g_plans.find(key);
  if (it == g_plans.end()) it = g_plans.emplace(key, make_plan(h, rows, m, k, bias)).first;
  GemmPlan &p = it->second;
  if (p.status != BSA_OK) return p.status;
  if (bias)
    cublasLtMatmulDescSetAttribute(p.op, CUBLASLT_MATMUL_DESC_BIAS_POINTER, &bias, sizeof(bias));
  const float alpha = 1.f, beta = 0.f;
  if (cublasLtMatmul(h, p.op, &alpha, w, p.la, a, p.lb, &beta, out, p.lc, out, p.lc, &p.algo,
                     scratch, kGemmScratch, stream) != CUBLAS_STATUS_SUCCESS)
    return BSA_ERR_CUDA;
  return BSA_OK;
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
                                 head_dim, softmax_scale, l, attn, &lo, nullptr, ws + w.order,
                                 w.qkv, stream_)) != BSA_OK)
    return st;
  // (3) y = attn out_proj^T + bias
  return linear_bf16(h, attn, w_out, b_out, y, rows, C, C, ws + w.gemm, stream);
}

}  // extern "C"
