// libbsa: host side of the C ABI declared in include/bsa.h.
//
// Argument checking, TMA descriptor encoding and kernel launches. The library
// keeps no device allocations; per-device state is limited to the status word
// (a __device__ variable) and a few cached device attributes.

#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "bsa.h"

#include "attn_bwd_fused_sm100.cuh"
#include "attn_bwd_sm100.cuh"
#include "attn_fwd_pair_sm100.cuh"
#include "attn_fwd_sm100.cuh"
#include "dense_ref.cuh"
#include "device_status.cuh"
#include "gemm.h"
#include "gemm_sm100.cuh"
#include "lists.cuh"
#include "patterns.cuh"

namespace bsa {
namespace {

thread_local char t_last_error[256] = "";

int cuda_fail(cudaError_t e, const char *what) {
  std::snprintf(t_last_error, sizeof(t_last_error), "%s: %s (%s)", what, cudaGetErrorName(e),
                cudaGetErrorString(e));
  return BSA_ERR_CUDA;
}

#define BSA_CUDA(call)                                  \
  do {                                                  \
    cudaError_t e_ = (call);                            \
    if (e_ != cudaSuccess) return cuda_fail(e_, #call); \
  } while (0)

// Test hooks (bsa_set_test_hooks).
std::mutex g_hook_mu;
unsigned long long g_wait_limit_ns = 2000000000ull;
int g_fault_flags = 0;
bool g_force_one_tile = false;  // test hook: run block-128 problems on the one-tile kernel

constexpr int kMaxDevices = 64;
struct DeviceInfo {
  bool probed = false;
  int cc_major = 0, cc_minor = 0, sms = 0;
  bool attrs_set[18] = {};
  bool ref_attrs_set[4] = {false, false, false, false};
  bool gemm_attrs_set[4] = {false, false, false, false};
  bool pair_attrs_set[12] = {};
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

int current_device(DeviceInfo **info) {
  int dev = 0;
  BSA_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return BSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo &d = g_dev[dev];
  if (!d.probed) {
    BSA_CUDA(cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev));
    BSA_CUDA(cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev));
    BSA_CUDA(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev));
    d.probed = true;
  }
  *info = &d;
  return BSA_OK;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// A [batch, heads, n, D] bf16 view with arbitrary batch / head / token strides
// (elements; D contiguous) as a 5-D tensor {64 columns, n rows, D/64 column
// halves, heads, batch}. One box {64, rows, D/64, 1, 1} brings a whole
// rows x D tile with 128-byte swizzling, laid out in shared memory as D/64
// consecutive [rows][64] blocks (the K-major layout the MMA descriptors use):
// one large box per tile, since the TMA unit's cost is mostly per box. Rows
// past n read as zeros. Head and batch stay separate coordinates, so
// token-major layouts (the [batch, n, heads, D] output of a fused projection)
// load without a transpose. An axis of extent 1 gets a placeholder stride
// (never used).
int make_map_strided(CUtensorMap *map, const void *ptr, const bsa_layout &L, int batch,
                     int heads, int n, int D, int rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    std::snprintf(t_last_error, sizeof(t_last_error), "cuTensorMapEncodeTiled not available");
    return BSA_ERR_CUDA;
  }
  cuuint64_t dims[5] = {64, static_cast<cuuint64_t>(n), static_cast<cuuint64_t>(D / 64),
                        static_cast<cuuint64_t>(heads), static_cast<cuuint64_t>(batch)};
  cuuint64_t strides[4] = {static_cast<cuuint64_t>(L.token_stride) * 2, 128,
                           heads > 1 ? static_cast<cuuint64_t>(L.head_stride) * 2 : 128,
                           batch > 1 ? static_cast<cuuint64_t>(L.batch_stride) * 2 : 128};
  cuuint32_t box[5] = {64, static_cast<cuuint32_t>(rows), static_cast<cuuint32_t>(D / 64), 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(ptr), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::snprintf(t_last_error, sizeof(t_last_error), "cuTensorMapEncodeTiled failed (%d)",
                  static_cast<int>(r));
    return BSA_ERR_CUDA;
  }
  return BSA_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bsa_layout contiguous_layout(int heads, int n, int D) {
  bsa_layout L;
  L.token_stride = D;
  L.head_stride = static_cast<int64_t>(n) * D;
  L.batch_stride = static_cast<int64_t>(heads) * n * D;
  return L;
}

// A layout the kernels can use: every stride of an axis longer than one is
// positive, a multiple of 8 elements (16 bytes, for TMA and the 16-byte
// output stores) and below 2^39 elements (TMA's 2^40-byte stride limit).
bool layout_ok(const bsa_layout &L, int batch, int heads, int n) {
  const int64_t lim = int64_t(1) << 39;
  auto good = [&](int64_t st, int extent) {
    return extent <= 1 || (st > 0 && st % 8 == 0 && st < lim);
  };
  return good(L.token_stride, n) && good(L.head_stride, heads) && good(L.batch_stride, batch);
}

// Bytes from the first to one past the last element a layout addresses.
size_t layout_span_bytes(const bsa_layout &L, int batch, int heads, int n, int D) {
  const int64_t last = (batch > 1 ? (batch - 1) * L.batch_stride : 0) +
                       (heads > 1 ? (heads - 1) * L.head_stride : 0) +
                       (n > 1 ? (n - 1) * L.token_stride : 0) + D;
  return static_cast<size_t>(last) * 2;
}

// No two (batch, head, token) rows of the layout share an element: sorted by
// stride, each axis steps past everything the inner axes span. Required of
// the output, whose rows are written concurrently.
bool layout_disjoint(const bsa_layout &L, int batch, int heads, int n, int D) {
  struct Ax {
    int64_t st;
    int ext;
  } ax[3] = {{L.token_stride, n}, {L.head_stride, heads}, {L.batch_stride, batch}};
  for (int i = 0; i < 3; ++i)
    for (int j = i + 1; j < 3; ++j)
      if (ax[j].st < ax[i].st) {
        const Ax t = ax[i];
        ax[i] = ax[j];
        ax[j] = t;
      }
  int64_t inner = D;  // elements spanned by the axes already placed
  for (int i = 0; i < 3; ++i) {
    if (ax[i].ext <= 1) continue;
    if (ax[i].st < inner) return false;
    inner = ax[i].st * (ax[i].ext - 1) + inner;
  }
  return true;
}

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

int ceil_div(long long a, long long b) { return static_cast<int>((a + b - 1) / b); }

// Shared argument checks of the two attention entry points.
int check_attn_args(const void *q, const void *k, const void *v, int32_t batch, int32_t heads,
                    int32_t n, int32_t head_dim, const bsa_block_lists *l, const void *out) {
  if (!q || !k || !v || !out || !l || !l->row_ptr || (l->nnz > 0 && !l->col_idx))
    return BSA_ERR_INVALID_ARG;
  if (batch < 1 || heads < 1 || n < 1) return BSA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return BSA_ERR_UNSUPPORTED;
  if (l->block != 64 && l->block != 128) return BSA_ERR_UNSUPPORTED;
  const long long nb = (static_cast<long long>(n) + l->block - 1) / l->block;
  if (l->num_q_blocks != nb || l->num_k_blocks != nb) return BSA_ERR_INVALID_ARG;
  if (l->num_lists != 1 && l->num_lists != heads) return BSA_ERR_INVALID_ARG;
  if (l->nnz < 0) return BSA_ERR_INVALID_ARG;
  const long long bh = static_cast<long long>(batch) * heads;
  if (bh * nb > 0x7fffffffLL || bh * n > 0x7fffffffLL) return BSA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return BSA_ERR_INVALID_ARG;
  const size_t bytes = static_cast<size_t>(bh) * n * head_dim * 2;
  if (overlaps(out, bytes, q, bytes) || overlaps(out, bytes, k, bytes) ||
      overlaps(out, bytes, v, bytes))
    return BSA_ERR_INVALID_ARG;
  return BSA_OK;
}

// Argument checks of the strided entry point: those of check_attn_args (with
// the overlap test made layout-aware) plus the layouts themselves.
int check_strided_args(const void *q, const bsa_layout *lq, const void *k, const bsa_layout *lk,
                       const void *v, const bsa_layout *lv, int32_t batch, int32_t heads,
                       int32_t n, int32_t head_dim, const bsa_block_lists *l, const void *out,
                       const bsa_layout *lo) {
  if (!lq || !lk || !lv || !lo) return BSA_ERR_INVALID_ARG;
  if (!q || !k || !v || !out || !l || !l->row_ptr || (l->nnz > 0 && !l->col_idx))
    return BSA_ERR_INVALID_ARG;
  if (batch < 1 || heads < 1 || n < 1) return BSA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return BSA_ERR_UNSUPPORTED;
  if (l->block != 64 && l->block != 128) return BSA_ERR_UNSUPPORTED;
  const long long nb = (static_cast<long long>(n) + l->block - 1) / l->block;
  if (l->num_q_blocks != nb || l->num_k_blocks != nb) return BSA_ERR_INVALID_ARG;
  if (l->num_lists != 1 && l->num_lists != heads) return BSA_ERR_INVALID_ARG;
  if (l->nnz < 0) return BSA_ERR_INVALID_ARG;
  const long long bh = static_cast<long long>(batch) * heads;
  if (bh * nb > 0x7fffffffLL || bh * n > 0x7fffffffLL) return BSA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return BSA_ERR_INVALID_ARG;
  for (const bsa_layout *L : {lq, lk, lv, lo})
    if (!layout_ok(*L, batch, heads, n)) return BSA_ERR_INVALID_ARG;
  if (!layout_disjoint(*lo, batch, heads, n, head_dim)) return BSA_ERR_INVALID_ARG;
  const size_t so = layout_span_bytes(*lo, batch, heads, n, head_dim);
  if (overlaps(out, so, q, layout_span_bytes(*lq, batch, heads, n, head_dim)) ||
      overlaps(out, so, k, layout_span_bytes(*lk, batch, heads, n, head_dim)) ||
      overlaps(out, so, v, layout_span_bytes(*lv, batch, heads, n, head_dim)))
    return BSA_ERR_INVALID_ARG;
  return BSA_OK;
}

// Whether two [batch, heads, n, D] views share no element. Exact for what
// callers use: spans that do not overlap, or identical token-major layouts
// (the heads of a token inside one token row, token rows of every batch item
// one after another) whose bases sit at least one row footprint apart inside
// a token row, as the q / k / v slices of one [batch, n, 3, heads, D] buffer
// do. Anything else counts as overlapping.
bool views_disjoint(const void *a, const bsa_layout &La, const void *b, const bsa_layout &Lb,
                    int batch, int heads, int n, int D) {
  if (!overlaps(a, layout_span_bytes(La, batch, heads, n, D), b,
                layout_span_bytes(Lb, batch, heads, n, D)))
    return true;
  if (La.batch_stride != Lb.batch_stride || La.head_stride != Lb.head_stride ||
      La.token_stride != Lb.token_stride)
    return false;
  const int64_t sn = La.token_stride;
  const int64_t foot = (heads > 1 ? (heads - 1) * La.head_stride : 0) + D;
  if (heads > 1 && La.head_stride < D) return false;
  if (batch > 1 && La.batch_stride != static_cast<int64_t>(n) * sn) return false;
  if (foot > sn) return false;
  const int64_t bytes = static_cast<int64_t>(reinterpret_cast<uintptr_t>(b)) -
                        static_cast<int64_t>(reinterpret_cast<uintptr_t>(a));
  if (bytes % 2) return false;
  const int64_t r = ((bytes / 2) % sn + sn) % sn;
  return r >= foot && sn - r >= foot;
}

// Forward scratch: the work order, then (256 bytes on) the work counter;
// at block 64 then the 128-row tile lists the two-tile kernel runs on (tile
// row pointers, tile columns, quarter masks).
size_t order_only_bytes(const bsa_block_lists *l) {
  return (static_cast<size_t>(l->num_lists) * l->num_q_blocks * sizeof(int32_t) + 255) & ~size_t(255);
}

struct TileScratch {
  size_t ptr, col, mask, total;  // offsets from the start of the tile lists
};

TileScratch tile_scratch(const bsa_block_lists *l) {
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t nt = (static_cast<size_t>(l->num_q_blocks) + 1) / 2;
  const size_t cap = l->nnz > 0 ? static_cast<size_t>(l->nnz) : 1;
  TileScratch t;
  t.ptr = 0;
  t.col = up((static_cast<size_t>(l->num_lists) * nt + 1) * sizeof(int32_t));
  t.mask = t.col + up(cap * sizeof(int32_t));
  t.total = t.mask + up(cap);
  return t;
}

size_t order_bytes(const bsa_block_lists *l) {
  return order_only_bytes(l) + 256 + (l->block == 64 ? tile_scratch(l).total : 0);
}

constexpr int kLptMaxRows = 12288;  // rows whose costs fit in 48 KB of shared memory

// q, k, v, their layouts, batch and heads of one forward call.
struct QkvViews {
  const void *q, *k, *v;
  bsa_layout lq, lk, lv;
  int batch, heads;
};

template <int D, int BN>
int launch_fwd(const QkvViews &x, int32_t n, const FwdParams &p, DeviceInfo *dev, int slot,
               cudaStream_t stream) {
  using C = FwdCfg<D, BN>;
  CUtensorMap tq, tk, tv;
  int st;
  if ((st = make_map_strided(&tq, x.q, x.lq, x.batch, x.heads, n, D, C::BM)) != BSA_OK) return st;
  if ((st = make_map_strided(&tk, x.k, x.lk, x.batch, x.heads, n, D, C::STAGE_ROWS)) != BSA_OK)
    return st;
  if ((st = make_map_strided(&tv, x.v, x.lv, x.batch, x.heads, n, D, C::STAGE_ROWS)) != BSA_OK)
    return st;
  {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!dev->attrs_set[slot]) {
      BSA_CUDA(cudaFuncSetAttribute(attn_fwd_sm100_kernel<D, BN>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, C::DSMEM));
      dev->attrs_set[slot] = true;
    }
  }
  const int grid = p.total_items < dev->sms ? p.total_items : dev->sms;
  attn_fwd_sm100_kernel<D, BN><<<grid, C::THREADS, C::DSMEM, stream>>>(tq, tk, tv, p);
  BSA_CUDA(cudaGetLastError());
  return BSA_OK;
}

template <int D, int BLK>
int launch_ref(const RefParams &p, int batch, DeviceInfo *dev, int slot, cudaStream_t stream) {
  const size_t smem = dense_ref_smem_bytes<D, BLK>(p.nkb);
  if (smem > static_cast<size_t>(kSmemLimit) - 64) return BSA_ERR_UNSUPPORTED;
  {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!dev->ref_attrs_set[slot]) {
      BSA_CUDA(cudaFuncSetAttribute(dense_masked_ref_kernel<D, BLK>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    kSmemLimit - 64));
      dev->ref_attrs_set[slot] = true;
    }
  }
  dim3 grid(p.nqb, p.heads, batch);
  dense_masked_ref_kernel<D, BLK><<<grid, 2 * BLK, smem, stream>>>(p);
  BSA_CUDA(cudaGetLastError());
  return BSA_OK;
}

int slot_of(int D, int BN) { return (D == 128 ? 2 : 0) + (BN == 128 ? 1 : 0); }

// The two-tile kernel in one of its row modes (kModeLists, kModeVarlen with
// `vt`, kModePatterns, kModeRadial). For a variable-length batch, x.batch is 1
// and n the total tokens.
template <int D, int MODE>
int launch_pair_mode(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                     const FwdParams &p, DeviceInfo *dev, const VarlenTable &vt,
                     cudaStream_t stream) {
  using C = PairCfg<D>;
  const int slot = MODE * 2 + (D == 128 ? 1 : 0);
  {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!dev->pair_attrs_set[slot]) {
      BSA_CUDA(cudaFuncSetAttribute(attn_fwd_pair_sm100_kernel<D, MODE>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, C::DSMEM));
      dev->pair_attrs_set[slot] = true;
    }
  }
  const int grid = p.total_items < dev->sms ? p.total_items : dev->sms;
  attn_fwd_pair_sm100_kernel<D, MODE><<<grid, C::THREADS, C::DSMEM, stream>>>(tq, tk, tv, p, vt);
  BSA_CUDA(cudaGetLastError());
  return BSA_OK;
}

template <int D>
int launch_pair(const QkvViews &x, int32_t n, const FwdParams &p, DeviceInfo *dev, int mode,
                const VarlenTable *vt, cudaStream_t stream) {
  using C = PairCfg<D>;
  CUtensorMap tq, tk, tv;
  int st;
  if ((st = make_map_strided(&tq, x.q, x.lq, x.batch, x.heads, n, D, C::BN)) != BSA_OK) return st;
  if ((st = make_map_strided(&tk, x.k, x.lk, x.batch, x.heads, n, D, C::BN)) != BSA_OK) return st;
  if ((st = make_map_strided(&tv, x.v, x.lv, x.batch, x.heads, n, D, C::BN)) != BSA_OK) return st;
  VarlenTable none;
  none.num_items = 0;
  const VarlenTable &t = vt ? *vt : none;
  switch (mode) {
    case kModeVarlen: return launch_pair_mode<D, kModeVarlen>(tq, tk, tv, p, dev, t, stream);
    case kModePatterns: return launch_pair_mode<D, kModePatterns>(tq, tk, tv, p, dev, t, stream);
    case kModeRadial: return launch_pair_mode<D, kModeRadial>(tq, tk, tv, p, dev, t, stream);
    case kModeQuarters: return launch_pair_mode<D, kModeQuarters>(tq, tk, tv, p, dev, t, stream);
    case kModeVarlenQuarters:
      return launch_pair_mode<D, kModeVarlenQuarters>(tq, tk, tv, p, dev, t, stream);
    default: return launch_pair_mode<D, kModeLists>(tq, tk, tv, p, dev, t, stream);
  }
}

// Work order into `order`, then the attention kernel. Block-128 problems run
// on the two-tile kernel (adjacent query blocks share K/V loads); block 64 on
// the one-tile kernel. Arguments were checked by the caller.
int run_fwd(const QkvViews &x, int32_t n, int32_t head_dim, float softmax_scale,
            const bsa_block_lists *l, void *out, const bsa_layout &lo, float *lse,
            int32_t *order, int32_t *item_counter, DeviceInfo *dev, int fault_flags,
            cudaStream_t stream, uint8_t *tile_lists = nullptr) {
  const int batch = x.batch, heads = x.heads;
  const int nqb = l->num_q_blocks;
  bool pair, force_one_tile;
  {
    std::lock_guard<std::mutex> lk(g_hook_mu);
    force_one_tile = g_force_one_tile;
    pair = l->block == 128 && !force_one_tile;
  }
  if (l->block == 64 && tile_lists && !force_one_tile) {
    // Block 64 on the two-tile kernel: the lists merged into 128-row tile
    // lists (each entry with its listed 64 x 64 quarters), the work order over
    // tile-row pairs, then the kernel masking the unlisted quarters.
    const TileScratch ts = tile_scratch(l);
    int32_t *tile_ptr = reinterpret_cast<int32_t *>(tile_lists + ts.ptr);
    int32_t *tile_col = reinterpret_cast<int32_t *>(tile_lists + ts.col);
    uint8_t *tile_mask = tile_lists + ts.mask;
    const int nt = (nqb + 1) / 2, ntk = (l->num_k_blocks + 1) / 2;
    const int rows_t = l->num_lists * nt;
    const long long cap = l->nnz > 0 ? l->nnz : 1;
    tile_count_kernel<<<(rows_t + 127) / 128, 128, 0, stream>>>(
        l->row_ptr, l->col_idx, nqb, l->num_k_blocks, l->nnz, nt, rows_t, tile_ptr, 1);
    BSA_CUDA(cudaGetLastError());
    scan_rows_kernel<<<1, 1024, 0, stream>>>(tile_ptr, rows_t);
    BSA_CUDA(cudaGetLastError());
    tile_fill_kernel<<<(rows_t + 127) / 128, 128, 0, stream>>>(
        l->row_ptr, l->col_idx, nqb, l->num_k_blocks, l->nnz, nt, rows_t, tile_ptr, tile_col,
        tile_mask, cap);
    BSA_CUDA(cudaGetLastError());
    const int npairs = (nt + 1) / 2;
    const size_t smem = static_cast<size_t>(npairs <= kLptMaxRows ? npairs : 0) * sizeof(int);
    pair_order_kernel<<<l->num_lists, 1024, smem, stream>>>(tile_ptr, tile_col, nt,
                                                           static_cast<int>(cap), order,
                                                           kLptMaxRows, item_counter);
    BSA_CUDA(cudaGetLastError());
    FwdParams p;
    p.row_ptr = tile_ptr;
    p.col_idx = tile_col;
    p.tile_mask = tile_mask;
    p.order = order;
    p.item_counter = item_counter;
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.o_sb = lo.batch_stride;
    p.o_sh = lo.head_stride;
    p.o_sn = lo.token_stride;
    p.lse = lse;
    p.heads = heads;
    p.n = n;
    p.nqb = nt;
    p.nkb = ntk;
    p.num_lists = l->num_lists;
    p.nnz = static_cast<int32_t>(cap);
    p.total_items = batch * heads * npairs;
    const float scale =
        softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(head_dim));
    p.scale_log2 = scale * 1.4426950408889634f;
    {
      std::lock_guard<std::mutex> lk(g_hook_mu);
      p.wait_limit_ns = g_wait_limit_ns;
    }
    p.fault_flags = fault_flags;
    if (head_dim == 128) return launch_pair<128>(x, n, p, dev, kModeQuarters, nullptr, stream);
    return launch_pair<64>(x, n, p, dev, kModeQuarters, nullptr, stream);
  }
  if (pair) {
    const int npairs = (nqb + 1) / 2;
    const size_t smem = static_cast<size_t>(npairs <= kLptMaxRows ? npairs : 0) * sizeof(int);
    pair_order_kernel<<<l->num_lists, 1024, smem, stream>>>(l->row_ptr, l->col_idx, nqb, l->nnz,
                                                           order, kLptMaxRows, item_counter);
  } else {
    const size_t smem = static_cast<size_t>(nqb <= kLptMaxRows ? nqb : 0) * sizeof(int);
    lpt_order_kernel<<<l->num_lists, 1024, smem, stream>>>(l->row_ptr, nqb, l->nnz, order,
                                                          kLptMaxRows);
  }
  BSA_CUDA(cudaGetLastError());

  FwdParams p;
  p.row_ptr = l->row_ptr;
  p.col_idx = l->col_idx;
  p.order = order;
  p.item_counter = item_counter;
  p.out = static_cast<__nv_bfloat16 *>(out);
  p.o_sb = lo.batch_stride;
  p.o_sh = lo.head_stride;
  p.o_sn = lo.token_stride;
  p.lse = lse;
  p.heads = heads;
  p.n = n;
  p.nqb = nqb;
  p.nkb = l->num_k_blocks;
  p.num_lists = l->num_lists;
  p.nnz = l->nnz;
  p.total_items = batch * heads * (pair ? (nqb + 1) / 2 : nqb);
  const float scale =
      softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(head_dim));
  p.scale_log2 = scale * 1.4426950408889634f;
  {
    std::lock_guard<std::mutex> lk(g_hook_mu);
    p.wait_limit_ns = g_wait_limit_ns;
  }
  p.fault_flags = fault_flags;
  if (pair) {
    if (head_dim == 128) return launch_pair<128>(x, n, p, dev, kModeLists, nullptr, stream);
    return launch_pair<64>(x, n, p, dev, kModeLists, nullptr, stream);
  }
  const int slot = slot_of(head_dim, l->block);
  if (head_dim == 128 && l->block == 128) return launch_fwd<128, 128>(x, n, p, dev, slot, stream);
  if (head_dim == 128 && l->block == 64) return launch_fwd<128, 64>(x, n, p, dev, slot, stream);
  if (head_dim == 64 && l->block == 128) return launch_fwd<64, 128>(x, n, p, dev, slot, stream);
  return launch_fwd<64, 64>(x, n, p, dev, slot, stream);
}

// ----------------------------------------------------- variable-length batches

// Per-item table of a variable-length batch from the host's cu_seqlens
// (item b = tokens [cu[b], cu[b+1])), for block-128 lists with `heads`
// work-item rows per query-block pair. Returns BSA_ERR_INVALID_ARG for a
// malformed cu_seqlens.
int varlen_table(int32_t num_items, const int32_t *cu, int32_t heads, int block, VarlenTable *vt,
                 int32_t *max_nqb) {
  if (num_items < 1 || num_items > kMaxVarlenItems || !cu || cu[0] != 0) return BSA_ERR_INVALID_ARG;
  long long rows = 0, pairs = 0, work = 0;
  int mx = 0;
  vt->num_items = num_items;
  for (int b = 0; b <= num_items; ++b) {
    if (b > 0 && cu[b] < cu[b - 1]) return BSA_ERR_INVALID_ARG;
    vt->tok0[b] = cu[b];
    vt->row0[b] = static_cast<int32_t>(rows);
    vt->pair0[b] = static_cast<int32_t>(pairs);
    vt->work0[b] = static_cast<int32_t>(work);
    if (b == num_items) break;
    const int nqb = ceil_div(static_cast<long long>(cu[b + 1]) - cu[b], block);
    mx = nqb > mx ? nqb : mx;
    rows += nqb;
    pairs += (nqb + 1) / 2;
    work += static_cast<long long>(heads) * ((nqb + 1) / 2);
    if (work > 0x7fffffffLL) return BSA_ERR_UNSUPPORTED;
  }
  if (cu[num_items] < 1) return BSA_ERR_INVALID_ARG;
  *max_nqb = mx;
  return BSA_OK;
}

size_t varlen_order_bytes(const VarlenTable &vt, int num_lists) {
  return ((static_cast<size_t>(num_lists) * vt.pair0[vt.num_items] * sizeof(int32_t) + 255) &
          ~size_t(255)) + 256;
}

// Scratch of a variable-length forward: the work order and counter over the
// 128-row tables' pairs (vt128), then, for block-64 lists, the items' tile
// lists (offsets of num_lists * sum_b nt_b rows, entries and quarter masks,
// at most one tile entry per 64-block entry).
struct VarlenFwdLayout {
  size_t tile_ptr, tile_col, tile_mask, total;
};
VarlenFwdLayout varlen_fwd_layout(const VarlenTable &vt128, const bsa_block_lists *l) {
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  VarlenFwdLayout w;
  w.tile_ptr = w.tile_col = w.tile_mask = w.total = varlen_order_bytes(vt128, l->num_lists);
  if (l->block == 64) {
    const size_t cap = l->nnz > 0 ? static_cast<size_t>(l->nnz) : 1;
    w.tile_col = w.tile_ptr + up((static_cast<size_t>(l->num_lists) * vt128.row0[vt128.num_items] + 1) *
                                 sizeof(int32_t));
    w.tile_mask = w.tile_col + up(cap * sizeof(int32_t));
    w.total = w.tile_mask + up(cap);
  }
  return w;
}

// ------------------------------------------------ rows generated in-kernel

// Scratch of the generated-row entries: row lengths (row_ptr of the count
// pass), the work order and the work counter.
constexpr int kMaxGeneratedLists = 4096;
struct GeneratedLayout {
  size_t row_ptr, order, cost, counter, total;
};
GeneratedLayout generated_layout(int num_lists, int nqb) {
  GeneratedLayout w;
  const size_t pairs = static_cast<size_t>(num_lists) * ((nqb + 1) / 2) * sizeof(int32_t);
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  w.row_ptr = 0;
  w.order = up((static_cast<size_t>(num_lists) * nqb + 1) * sizeof(int32_t));
  w.cost = w.order + up(pairs);
  w.counter = w.cost + up(pairs);
  w.total = w.counter + 256;
  return w;
}

// Parameters of the two-tile kernel for rows generated in the kernel
// (contiguous [batch, heads, n, head_dim] views, block 128).
FwdParams generated_params(int batch, int heads, int n, int nqb, int num_lists,
                           const int32_t *row_ptr, const int32_t *order, int32_t *counter,
                           void *out, int head_dim, float *lse, float softmax_scale) {
  FwdParams p;
  p.row_ptr = row_ptr;
  p.col_idx = nullptr;
  p.order = order;
  p.item_counter = counter;
  p.out = static_cast<__nv_bfloat16 *>(out);
  const bsa_layout lo = contiguous_layout(heads, n, head_dim);
  p.o_sb = lo.batch_stride;
  p.o_sh = lo.head_stride;
  p.o_sn = lo.token_stride;
  p.lse = lse;
  p.heads = heads;
  p.n = n;
  p.nqb = nqb;
  p.nkb = nqb;
  p.num_lists = num_lists;
  p.nnz = 0x7fffffff;  // row_ptr comes from this call's own count pass
  p.total_items = batch * heads * ((nqb + 1) / 2);
  const float scale =
      softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(head_dim));
  p.scale_log2 = scale * 1.4426950408889634f;
  {
    std::lock_guard<std::mutex> lk(g_hook_mu);
    p.wait_limit_ns = g_wait_limit_ns;
    p.fault_flags = g_fault_flags;
    g_fault_flags = 0;
  }
  return p;
}

QkvViews contiguous_views(const void *q, const void *k, const void *v, int batch, int heads,
                          int n, int D) {
  QkvViews x;
  x.q = q;
  x.k = k;
  x.v = v;
  x.lq = x.lk = x.lv = contiguous_layout(heads, n, D);
  x.batch = batch;
  x.heads = heads;
  return x;
}

// ---------------------------------------------------------------- backward

// Workspace of the backward pass: lse2 and delta per padded query row, then
// the transposed lists; for block-64 lists also the per-entry masks of the
// transposed lists and the 128-row tile lists (pointers, entries, masks); for
// block-128 lists of a regular call (the one-pass kernel) the key blocks'
// positions in their query rows, the dQ part counters and the fp32 dQ
// accumulator rows (sized for head_dim 128, the largest). Offsets are
// 256-byte aligned (the bulk copies of lse2 / delta rows need 16-byte
// aligned 512-byte rows).
struct BwdLayout {
  size_t lse2, delta, counters, col_ptr, row_idx, cmask, tile_ptr, tile_col, tile_mask;
  size_t row_pos, dq_sem, dq_acc, total;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

BwdLayout bwd_layout(int32_t batch, int32_t heads, int32_t n, const bsa_block_lists *l,
                     bool one_pass = false) {
  BwdLayout w;
  const size_t nt = static_cast<size_t>(ceil_div(n, kBwdBlock));  // 128-row tiles
  const size_t rows = static_cast<size_t>(batch) * heads * nt * kBwdBlock;
  const size_t ptrs = (static_cast<size_t>(l->num_lists) * nt + 1) * sizeof(int32_t);
  const size_t entries = static_cast<size_t>(l->nnz > 0 ? l->nnz : 1);
  w.lse2 = 0;
  w.delta = align256(rows * sizeof(float));
  w.counters = w.delta + align256(rows * sizeof(float));  // the two kernels' work counters
  w.col_ptr = w.counters + 256;
  w.row_idx = w.col_ptr + align256(ptrs);
  w.cmask = w.tile_ptr = w.tile_col = w.tile_mask = w.total =
      w.row_idx + align256(entries * sizeof(int32_t));
  if (l->block != kBwdBlock) {
    w.tile_ptr = w.cmask + align256(entries);
    w.tile_col = w.tile_ptr + align256(ptrs);
    w.tile_mask = w.tile_col + align256(entries * sizeof(int32_t));
    w.total = w.tile_mask + align256(entries);
  }
  w.row_pos = w.dq_sem = w.dq_acc = w.total;
  if (one_pass && l->block == kBwdBlock) {
    const size_t qblocks = static_cast<size_t>(batch) * heads * nt;
    w.dq_sem = w.row_pos + align256(entries * sizeof(int32_t));
    w.dq_acc = w.dq_sem + align256(qblocks * 4 * sizeof(int32_t));
    w.total = w.dq_acc + align256(qblocks * kBwdBlock * 128 * sizeof(float));
  }
  return w;
}

// Inputs, outputs and their layouts of one backward call.
struct BwdViews {
  const void *q, *k, *v, *out, *dout;
  void *dq, *dk, *dv;
  bsa_layout lq, lk, lv, lo, ldo, ldq, ldk, ldv;
  int batch, heads;
  long long lse_sb = -1, lse_sh = -1;  // lse's batch / head strides; -1: contiguous [B, H, n]
};

// The dK/dV and dQ kernels of one backward call, once the prep and the
// transposed lists are in place: TMA maps over the views ([batch, heads,
// n_map] tokens), the instance for the masks and for a variable-length
// batch (vt non-null: its items are the problems), dkdv_items and dq_items
// work items.
template <int D>
int launch_bwd_kernels(const BwdViews &x, int32_t n_map, BwdParams &p, bool masked,
                       const VarlenTable *vt, long long dkdv_items, long long dq_items,
                       DeviceInfo *dev, cudaStream_t stream) {
  CUtensorMap tq, tk, tv, td;
  int st;
  if ((st = make_map_strided(&tq, x.q, x.lq, x.batch, x.heads, n_map, D, kBwdBlock)) != BSA_OK)
    return st;
  if ((st = make_map_strided(&tk, x.k, x.lk, x.batch, x.heads, n_map, D, kBwdBlock)) != BSA_OK)
    return st;
  if ((st = make_map_strided(&tv, x.v, x.lv, x.batch, x.heads, n_map, D, kBwdBlock)) != BSA_OK)
    return st;
  if ((st = make_map_strided(&td, x.dout, x.ldo, x.batch, x.heads, n_map, D, kBwdBlock)) != BSA_OK)
    return st;
  const bool varlen = vt != nullptr;
  using DkdvFn = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, BwdParams,
                          VarlenTable);
  DkdvFn dkdv = varlen   ? (masked ? attn_bwd_dkdv_kernel<D, true, true>
                                   : attn_bwd_dkdv_kernel<D, false, true>)
                : masked ? attn_bwd_dkdv_kernel<D, true, false>
                         : attn_bwd_dkdv_kernel<D, false, false>;
  DkdvFn dq = varlen   ? (masked ? attn_bwd_dq_kernel<D, true, true>
                                 : attn_bwd_dq_kernel<D, false, true>)
              : masked ? attn_bwd_dq_kernel<D, true, false>
                       : attn_bwd_dq_kernel<D, false, false>;
  const int slot = varlen && masked ? 16 + (D == 128 ? 1 : 0)
                                    : 8 + (D == 128 ? 3 : 0) + (varlen ? 2 : masked ? 1 : 0);
  {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!dev->attrs_set[slot]) {
      BSA_CUDA(cudaFuncSetAttribute(dkdv, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    DkdvCfg<D>::DSMEM));
      BSA_CUDA(cudaFuncSetAttribute(dq, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    DqCfg<D>::DSMEM));
      dev->attrs_set[slot] = true;
    }
  }
  static const VarlenTable kNoItems{};
  const VarlenTable &table = varlen ? *vt : kNoItems;
  int32_t *counters = p.item_counter;
  p.total_items = static_cast<int32_t>(dkdv_items);
  int grid = p.total_items < dev->sms ? p.total_items : dev->sms;
  if (grid > 0) {
    dkdv<<<grid, DkdvCfg<D>::THREADS, DkdvCfg<D>::DSMEM, stream>>>(tq, tk, tv, td, p, table);
    BSA_CUDA(cudaGetLastError());
  }
  p.total_items = static_cast<int32_t>(dq_items);
  p.item_counter = counters + 1;
  grid = p.total_items < dev->sms ? p.total_items : dev->sms;
  if (grid > 0) {
    dq<<<grid, DqCfg<D>::THREADS, DqCfg<D>::DSMEM, stream>>>(tq, tk, tv, td, p, table);
    BSA_CUDA(cudaGetLastError());
  }
  p.item_counter = counters;
  return BSA_OK;
}

// The one-pass backward (block 128): counters and dq of empty rows
// initialised, then one kernel for dK, dV and dQ over `items` (batch*head,
// key block) work items; rows = batch*heads*nqb*128 padded query rows.
template <int D>
int launch_bwd_one_pass(const BwdViews &x, int32_t n_map, BwdParams &p, long long items,
                        long long rows, DeviceInfo *dev, cudaStream_t stream) {
  CUtensorMap tq, tk, tv, td;
  int st;
  if ((st = make_map_strided(&tq, x.q, x.lq, x.batch, x.heads, n_map, D, kBwdBlock)) != BSA_OK)
    return st;
  if ((st = make_map_strided(&tk, x.k, x.lk, x.batch, x.heads, n_map, D, kBwdBlock)) != BSA_OK)
    return st;
  if ((st = make_map_strided(&tv, x.v, x.lv, x.batch, x.heads, n_map, D, kBwdBlock)) != BSA_OK)
    return st;
  if ((st = make_map_strided(&td, x.dout, x.ldo, x.batch, x.heads, n_map, D, kBwdBlock)) != BSA_OK)
    return st;
  const int slot = 14 + (D == 128 ? 1 : 0);
  {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!dev->attrs_set[slot]) {
      BSA_CUDA(cudaFuncSetAttribute(attn_bwd_fused_kernel<D>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    FusedCfg<D>::DSMEM));
      dev->attrs_set[slot] = true;
    }
  }
  const long long sems = rows / kBwdBlock * 4;
  const long long threads = rows > sems ? rows : sems;
  fused_init_kernel<D><<<static_cast<unsigned>((threads + 255) / 256), 256, 0, stream>>>(
      p, rows, sems);
  BSA_CUDA(cudaGetLastError());
  p.total_items = static_cast<int32_t>(items);
  const int grid = p.total_items < dev->sms ? p.total_items : dev->sms;
  if (grid > 0) {
    attn_bwd_fused_kernel<D><<<grid, FusedCfg<D>::THREADS, FusedCfg<D>::DSMEM, stream>>>(
        tq, tk, tv, td, p);
    BSA_CUDA(cudaGetLastError());
  }
  return BSA_OK;
}

// Parameters shared by every backward launch of a call.
template <int D>
BwdParams bwd_params(const BwdViews &x, const bsa_block_lists *l, float softmax_scale) {
  BwdParams p;
  p.row_ptr = l->row_ptr;
  p.col_idx = l->col_idx;
  p.dq = static_cast<__nv_bfloat16 *>(x.dq);
  p.dk = static_cast<__nv_bfloat16 *>(x.dk);
  p.dv = static_cast<__nv_bfloat16 *>(x.dv);
  const bsa_layout *outl[3] = {&x.ldq, &x.ldk, &x.ldv};
  long long *outs[3] = {p.dq_s, p.dk_s, p.dv_s};
  for (int i = 0; i < 3; ++i) {
    outs[i][0] = outl[i]->batch_stride;
    outs[i][1] = outl[i]->head_stride;
    outs[i][2] = outl[i]->token_stride;
  }
  p.heads = x.heads;
  p.num_lists = l->num_lists;
  p.nnz = l->nnz;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(D));
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  {
    std::lock_guard<std::mutex> lk(g_hook_mu);
    p.wait_limit_ns = g_wait_limit_ns;
  }
  return p;
}

// one_pass (block 128 only): dK, dV and dQ from the one-pass kernel with the
// dQ parts added in order; otherwise the dK/dV and dQ kernels.
template <int D>
int launch_bwd(const BwdViews &x, const float *lse, int32_t n, float softmax_scale,
               const bsa_block_lists *l_in, uint8_t *ws, DeviceInfo *dev, cudaStream_t stream,
               bool one_pass = false) {
  const int32_t bh = x.batch * x.heads;
  const BwdLayout w = bwd_layout(1, bh, n, l_in, one_pass);
  float *lse2 = reinterpret_cast<float *>(ws + w.lse2);
  float *delta = reinterpret_cast<float *>(ws + w.delta);
  int32_t *col_ptr = reinterpret_cast<int32_t *>(ws + w.col_ptr);
  int32_t *row_idx = reinterpret_cast<int32_t *>(ws + w.row_idx);
  // The kernels walk 128 x 128 tiles. Block-64 lists become tile lists with a
  // 4-bit mask per entry (the listed 64 x 64 pairs of the tile pair).
  bsa_block_lists tiles = *l_in;
  const bsa_block_lists *l = &tiles;
  const uint8_t *rmask = nullptr;
  uint8_t *cmask = nullptr;
  if (l_in->block != kBwdBlock) {
    const int nt = ceil_div(n, kBwdBlock);
    const int rows_t = l_in->num_lists * nt;
    int32_t *tile_ptr = reinterpret_cast<int32_t *>(ws + w.tile_ptr);
    int32_t *tile_col = reinterpret_cast<int32_t *>(ws + w.tile_col);
    uint8_t *tile_mask = ws + w.tile_mask;
    const long long cap = l_in->nnz > 0 ? l_in->nnz : 1;
    tile_count_kernel<<<(rows_t + 127) / 128, 128, 0, stream>>>(
        l_in->row_ptr, l_in->col_idx, l_in->num_q_blocks, l_in->num_k_blocks, l_in->nnz, nt,
        rows_t, tile_ptr, 1);
    BSA_CUDA(cudaGetLastError());
    scan_rows_kernel<<<1, 1024, 0, stream>>>(tile_ptr, rows_t);
    BSA_CUDA(cudaGetLastError());
    tile_fill_kernel<<<(rows_t + 127) / 128, 128, 0, stream>>>(
        l_in->row_ptr, l_in->col_idx, l_in->num_q_blocks, l_in->num_k_blocks, l_in->nnz, nt,
        rows_t, tile_ptr, tile_col, tile_mask, cap);
    BSA_CUDA(cudaGetLastError());
    tiles.num_q_blocks = tiles.num_k_blocks = nt;
    tiles.block = kBwdBlock;
    tiles.row_ptr = tile_ptr;
    tiles.col_idx = tile_col;  // nnz stays the 64-list size: a bound on the tile entries
    rmask = tile_mask;
    cmask = ws + w.cmask;
  }
  const int nqb = l->num_q_blocks, nkb = l->num_k_blocks;

  const long long rows = static_cast<long long>(bh) * nqb * kBwdBlock;
  const long long l_sh = x.lse_sh >= 0 ? x.lse_sh : n;
  const long long l_sb = x.lse_sb >= 0 ? x.lse_sb : static_cast<long long>(x.heads) * n;
  bwd_prep_kernel<D><<<static_cast<unsigned>((rows + 255) / 256), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16 *>(x.out), static_cast<const __nv_bfloat16 *>(x.dout), lse,
      lse2, delta, n, nqb, x.heads, x.lo.batch_stride, x.lo.head_stride, x.lo.token_stride,
      x.ldo.batch_stride, x.ldo.head_stride, x.ldo.token_stride, l_sb, l_sh, rows,
      reinterpret_cast<int32_t *>(ws + w.counters));
  BSA_CUDA(cudaGetLastError());
  const int cols = l->num_lists * nkb;
  csc_count_kernel<<<cols, 256, 0, stream>>>(l->row_ptr, l->col_idx, nqb, nkb, l->nnz, col_ptr,
                                             1);
  BSA_CUDA(cudaGetLastError());
  scan_rows_kernel<<<1, 1024, 0, stream>>>(col_ptr, cols);
  BSA_CUDA(cudaGetLastError());
  int32_t *row_pos = one_pass ? reinterpret_cast<int32_t *>(ws + w.row_pos) : nullptr;
  csc_fill_kernel<<<cols, 256, 0, stream>>>(l->row_ptr, l->col_idx, nqb, nkb, l->nnz, col_ptr,
                                            row_idx, l->nnz > 0 ? l->nnz : 1, rmask, cmask,
                                            row_pos);
  BSA_CUDA(cudaGetLastError());

  BwdParams p = bwd_params<D>(x, l, softmax_scale);
  p.col_ptr = col_ptr;
  p.row_idx = row_idx;
  p.rmask = rmask;
  p.cmask = cmask;
  p.lse2 = lse2;
  p.delta = delta;
  p.n = n;
  p.nqb = nqb;
  p.nkb = nkb;
  p.row_ptr = l->row_ptr;
  p.col_idx = l->col_idx;
  p.item_counter = reinterpret_cast<int32_t *>(ws + w.counters);
  if (one_pass) {
    p.row_pos = row_pos;
    p.dq_sem = reinterpret_cast<int32_t *>(ws + w.dq_sem);
    p.dq_acc = reinterpret_cast<float *>(ws + w.dq_acc);
    return launch_bwd_one_pass<D>(x, n, p, static_cast<long long>(bh) * nkb, rows, dev, stream);
  }
  return launch_bwd_kernels<D>(x, n, p, rmask != nullptr, nullptr,
                               static_cast<long long>(bh) * nkb, static_cast<long long>(bh) * nqb,
                               dev, stream);
}

// Backward of a variable-length batch (block-128 lists concatenated item by
// item, packed [1, heads, total] views, lse [heads, total]): per item the
// prep (lse2 / delta laid out item by item, head by head) and the item's
// columns of the transposed lists (one scan over all of them); then one
// dK/dV and one dQ launch over every item's work.
template <int D>
int launch_bwd_varlen(const BwdViews &x, const float *lse, int32_t total, float softmax_scale,
                      const bsa_block_lists *l, const VarlenTable &vt_l, const VarlenTable &vt,
                      uint8_t *ws, DeviceInfo *dev, cudaStream_t stream) {
  // vt_l: the items in blocks of the lists; vt: in 128-row tiles (the
  // kernels' blocks; the same table at block 128)
  const int R = vt.row0[vt.num_items];
  const BwdLayout w = bwd_layout(1, x.heads, R * kBwdBlock, l);
  float *lse2 = reinterpret_cast<float *>(ws + w.lse2);
  float *delta = reinterpret_cast<float *>(ws + w.delta);
  int32_t *col_ptr = reinterpret_cast<int32_t *>(ws + w.col_ptr);
  int32_t *row_idx = reinterpret_cast<int32_t *>(ws + w.row_idx);
  int32_t *counters = reinterpret_cast<int32_t *>(ws + w.counters);
  const int L = l->num_lists;
  const long long cap = l->nnz > 0 ? l->nnz : 1;
  // block-64 lists: the items' tile lists with the quarter masks, as in the
  // forward (counts per item, one scan, fills per item)
  const int32_t *rows = l->row_ptr, *cols = l->col_idx;
  const uint8_t *rmask = nullptr;
  uint8_t *cmask = nullptr;
  if (l->block != kBwdBlock) {
    int32_t *tile_ptr = reinterpret_cast<int32_t *>(ws + w.tile_ptr);
    int32_t *tile_col = reinterpret_cast<int32_t *>(ws + w.tile_col);
    uint8_t *tile_mask = ws + w.tile_mask;
    bool first_seg = true;
    for (int b = 0; b < vt.num_items; ++b) {
      const int nq = vt_l.row0[b + 1] - vt_l.row0[b], nt = vt.row0[b + 1] - vt.row0[b];
      if (nt == 0) continue;
      const int rows_t = L * nt;
      tile_count_kernel<<<(rows_t + 127) / 128, 128, 0, stream>>>(
          l->row_ptr + static_cast<long long>(L) * vt_l.row0[b], l->col_idx, nq, nq, l->nnz, nt,
          rows_t, tile_ptr + static_cast<long long>(L) * vt.row0[b], first_seg ? 1 : 0);
      BSA_CUDA(cudaGetLastError());
      first_seg = false;
    }
    scan_rows_kernel<<<1, 1024, 0, stream>>>(tile_ptr, L * R);
    BSA_CUDA(cudaGetLastError());
    for (int b = 0; b < vt.num_items; ++b) {
      const int nq = vt_l.row0[b + 1] - vt_l.row0[b], nt = vt.row0[b + 1] - vt.row0[b];
      if (nt == 0) continue;
      const int rows_t = L * nt;
      tile_fill_kernel<<<(rows_t + 127) / 128, 128, 0, stream>>>(
          l->row_ptr + static_cast<long long>(L) * vt_l.row0[b], l->col_idx, nq, nq, l->nnz, nt,
          rows_t, tile_ptr + static_cast<long long>(L) * vt.row0[b], tile_col, tile_mask, cap);
      BSA_CUDA(cudaGetLastError());
    }
    rows = tile_ptr;
    cols = tile_col;
    rmask = tile_mask;
    cmask = ws + w.cmask;
  }
  const int nnz = static_cast<int>(l->block != kBwdBlock ? cap : l->nnz);
  bool first = true;
  for (int b = 0; b < vt.num_items; ++b) {
    const int nq = vt.row0[b + 1] - vt.row0[b];
    if (nq == 0) continue;
    const int32_t t0 = vt.tok0[b], n_b = vt.tok0[b + 1] - t0;
    const long long base = static_cast<long long>(x.heads) * vt.row0[b] * kBwdBlock;
    const long long prow = static_cast<long long>(x.heads) * nq * kBwdBlock;
    bwd_prep_kernel<D><<<static_cast<unsigned>((prow + 255) / 256), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(x.out) + static_cast<long long>(t0) * x.lo.token_stride,
        static_cast<const __nv_bfloat16 *>(x.dout) + static_cast<long long>(t0) * x.ldo.token_stride,
        lse + t0, lse2 + base, delta + base, n_b, nq, x.heads, 0, x.lo.head_stride,
        x.lo.token_stride, 0, x.ldo.head_stride, x.ldo.token_stride, 0, total, prow, counters);
    BSA_CUDA(cudaGetLastError());
    const long long lr = static_cast<long long>(L) * vt.row0[b];
    csc_count_kernel<<<L * nq, 256, 0, stream>>>(rows + lr, cols, nq, nq, nnz, col_ptr + lr,
                                                 first ? 1 : 0);
    BSA_CUDA(cudaGetLastError());
    first = false;
  }
  scan_rows_kernel<<<1, 1024, 0, stream>>>(col_ptr, L * R);
  BSA_CUDA(cudaGetLastError());
  for (int b = 0; b < vt.num_items; ++b) {
    const int nq = vt.row0[b + 1] - vt.row0[b];
    if (nq == 0) continue;
    const long long lr = static_cast<long long>(L) * vt.row0[b];
    csc_fill_kernel<<<L * nq, 256, 0, stream>>>(rows + lr, cols, nq, nq, nnz, col_ptr + lr,
                                                row_idx, nnz > 0 ? nnz : 1, rmask, cmask,
                                                nullptr);
    BSA_CUDA(cudaGetLastError());
  }
  BwdParams p = bwd_params<D>(x, l, softmax_scale);
  p.row_ptr = rows;
  p.col_idx = cols;
  p.nnz = nnz;
  p.col_ptr = col_ptr;
  p.row_idx = row_idx;
  p.rmask = rmask;
  p.cmask = cmask;
  p.lse2 = lse2;
  p.delta = delta;
  p.n = total;
  p.nqb = p.nkb = 0;  // per item, from the table
  p.item_counter = counters;
  const long long items = static_cast<long long>(x.heads) * R;
  return launch_bwd_kernels<D>(x, total, p, rmask != nullptr, &vt, items, items, dev, stream);
}

// Self-test of the two exp2 paths of the attention softmax against exp2f.
__global__ void exp2_selftest_kernel(const float *x, float *y_poly, float *y_mufu,
                                     float *y_ref, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (2 * i + 1 >= n) return;
  const float2 v = make_float2(x[2 * i], x[2 * i + 1]);
  const float2 p = exp2_poly2(v);
  y_poly[2 * i] = p.x;
  y_poly[2 * i + 1] = p.y;
  y_mufu[2 * i] = ex2_approx(v.x);
  y_mufu[2 * i + 1] = ex2_approx(v.y);
  y_ref[2 * i] = exp2f(v.x);
  y_ref[2 * i + 1] = exp2f(v.y);
}

// A row-major bf16 matrix [outer][inner] (row stride `stride` elements) as a
// 2-D tensor map with 128-byte swizzling and box {64, box_outer}: a K-major
// operand tile (64 K values per row) or one 64-wide chunk of an MN-major one.
// Out-of-range rows and columns read as zeros.
int make_map_2d(CUtensorMap *map, const void *ptr, int64_t inner, int64_t outer, int64_t stride,
                int box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    std::snprintf(t_last_error, sizeof(t_last_error), "cuTensorMapEncodeTiled not available");
    return BSA_ERR_CUDA;
  }
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(stride) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_outer)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::snprintf(t_last_error, sizeof(t_last_error), "cuTensorMapEncodeTiled failed (%d)",
                  static_cast<int>(r));
    return BSA_ERR_CUDA;
  }
  return BSA_OK;
}

template <bool A_MN, bool B_MN>
int launch_gemm(const CUtensorMap &ta, const CUtensorMap &tb, const GemmParams &p,
                DeviceInfo *dev, cudaStream_t stream) {
  const int slot = (A_MN ? 2 : 0) + (B_MN ? 1 : 0);
  {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!dev->gemm_attrs_set[slot]) {
      BSA_CUDA(cudaFuncSetAttribute(gemm_bf16_sm100_kernel<A_MN, B_MN>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, GemmCfg::DSMEM));
      dev->gemm_attrs_set[slot] = true;
    }
  }
  const int grid = p.total_tiles < dev->sms ? p.total_tiles : dev->sms;
  gemm_bf16_sm100_kernel<A_MN, B_MN><<<grid, GemmCfg::THREADS, GemmCfg::DSMEM, stream>>>(ta, tb,
                                                                                       p);
  BSA_CUDA(cudaGetLastError());
  return BSA_OK;
}

}  // namespace

int gemm_bf16(const void *a, int64_t lda, bool a_mn_major, const void *b, int64_t ldb,
              bool b_mn_major, const void *bias, void *d, int64_t ldd, int64_t m, int64_t n,
              int64_t k, cudaStream_t stream) {
  if (!a || !b || !d) return BSA_ERR_INVALID_ARG;
  constexpr int64_t kMaxDim = (int64_t(1) << 31) - 256;
  if (m < 1 || n < 1 || k < 1 || m > kMaxDim || n > kMaxDim || k > kMaxDim)
    return BSA_ERR_INVALID_ARG;
  // 16-byte aligned bases and row strides (TMA, 16-byte output vectors);
  // output rows hold whole 8-element vectors
  if (!aligned16(a) || !aligned16(b) || !aligned16(d) || (lda & 7) || (ldb & 7) || (ldd & 7) ||
      (n & 7))
    return BSA_ERR_INVALID_ARG;
  if (lda < (a_mn_major ? m : k) || ldb < (b_mn_major ? n : k) || ldd < n)
    return BSA_ERR_INVALID_ARG;
  if (lda >= (int64_t(1) << 39) || ldb >= (int64_t(1) << 39)) return BSA_ERR_INVALID_ARG;
  const size_t a_span = static_cast<size_t>(((a_mn_major ? k : m) - 1) * lda + (a_mn_major ? m : k)) * 2;
  const size_t b_span = static_cast<size_t>(((b_mn_major ? k : n) - 1) * ldb + (b_mn_major ? n : k)) * 2;
  const size_t d_span = static_cast<size_t>((m - 1) * ldd + n) * 2;
  if (overlaps(d, d_span, a, a_span) || overlaps(d, d_span, b, b_span) ||
      (bias && overlaps(d, d_span, bias, static_cast<size_t>(n) * 2)))
    return BSA_ERR_INVALID_ARG;
  DeviceInfo *dev = nullptr;
  int st;
  if ((st = current_device(&dev)) != BSA_OK) return st;
  if (dev->cc_major != 10) return BSA_ERR_UNSUPPORTED;
  CUtensorMap ta, tb;
  if ((st = a_mn_major ? make_map_2d(&ta, a, m, k, lda, GemmCfg::BK)
                       : make_map_2d(&ta, a, k, m, lda, GemmCfg::BM)) != BSA_OK)
    return st;
  if ((st = b_mn_major ? make_map_2d(&tb, b, n, k, ldb, GemmCfg::BK)
                       : make_map_2d(&tb, b, k, n, ldb, GemmCfg::BN)) != BSA_OK)
    return st;
  GemmParams p;
  p.M = static_cast<int>(m);
  p.N = static_cast<int>(n);
  p.K = static_cast<int>(k);
  p.d = static_cast<__nv_bfloat16 *>(d);
  p.ldd = ldd;
  p.bias = static_cast<const __nv_bfloat16 *>(bias);
  p.tiles_m = static_cast<int>((m + GemmCfg::BM - 1) / GemmCfg::BM);
  p.tiles_n = static_cast<int>((n + GemmCfg::BN - 1) / GemmCfg::BN);
  if (static_cast<int64_t>(p.tiles_m) * p.tiles_n > INT32_MAX) return BSA_ERR_INVALID_ARG;
  p.total_tiles = p.tiles_m * p.tiles_n;
  p.k_blocks = static_cast<int>((k + GemmCfg::BK - 1) / GemmCfg::BK);
  {
    std::lock_guard<std::mutex> lk(g_hook_mu);
    p.wait_limit_ns = g_wait_limit_ns;
  }
  if (a_mn_major)
    return b_mn_major ? launch_gemm<true, true>(ta, tb, p, dev, stream)
                      : launch_gemm<true, false>(ta, tb, p, dev, stream);
  return b_mn_major ? launch_gemm<false, true>(ta, tb, p, dev, stream)
                    : launch_gemm<false, false>(ta, tb, p, dev, stream);
}

}  // namespace bsa

using namespace bsa;

extern "C" {

int bsa_joint_mask_build(int32_t frames, int32_t tokens_per_frame, int32_t text_tokens,
                         int32_t block, int32_t *row_ptr, int32_t *col_idx,
                         int64_t col_capacity, int64_t *nnz_out, bsa_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (frames < 1 || tokens_per_frame < 1 || text_tokens < 0 || !row_ptr)
    return BSA_ERR_INVALID_ARG;
  if (block != 64 && block != 128) return BSA_ERR_UNSUPPORTED;
  const long long nv = static_cast<long long>(frames) * tokens_per_frame;
  const long long n = nv + text_tokens;
  if (n > 0x7fffffffLL) return BSA_ERR_INVALID_ARG;
  const int nb = ceil_div(n, block);
  if (nb > 262144) return BSA_ERR_UNSUPPORTED;
  if (col_idx && col_capacity < 0) return BSA_ERR_INVALID_ARG;
  RadialGeom g;
  g.frames = frames;
  g.tpf = tokens_per_frame;
  g.block = block;
  g.nv = static_cast<int>(nv);
  g.n = static_cast<int>(n);
  g.nb = nb;
  int rs = 0;
  if (tokens_per_frame >= block)
    while ((tokens_per_frame >> (rs + 1)) >= block) ++rs;
  g.rstar = rs;
  const size_t smem = static_cast<size_t>((nb + 31) / 32) * sizeof(uint32_t);
  radial_count_kernel<<<nb, 128, smem, stream>>>(g, row_ptr, 0);
  BSA_CUDA(cudaGetLastError());
  scan_rows_kernel<<<1, 1024, 0, stream>>>(row_ptr, nb);
  BSA_CUDA(cudaGetLastError());
  if (nnz_out) {
    int32_t last = 0;
    BSA_CUDA(cudaMemcpyAsync(&last, row_ptr + nb, sizeof(int32_t), cudaMemcpyDeviceToHost, stream));
    BSA_CUDA(cudaStreamSynchronize(stream));
    *nnz_out = last;
    if (col_idx && last > col_capacity) return BSA_ERR_CAPACITY;
  }
  if (col_idx) {
    radial_fill_kernel<<<nb, 128, smem, stream>>>(g, row_ptr, 0, col_idx, col_capacity);
    BSA_CUDA(cudaGetLastError());
  }
  return BSA_OK;
}

int bsa_joint_mask_build_varlen(int32_t num_items, const int32_t *frames,
                                const int32_t *tokens_per_frame, const int32_t *text_tokens,
                                int32_t block, int32_t *row_ptr, int32_t *col_idx,
                                int64_t col_capacity, int64_t *nnz_out, bsa_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (num_items < 1 || num_items > kMaxVarlenItems || !frames || !tokens_per_frame || !row_ptr)
    return BSA_ERR_INVALID_ARG;
  if (block != 64 && block != 128) return BSA_ERR_UNSUPPORTED;
  if (col_idx && col_capacity < 0) return BSA_ERR_INVALID_ARG;
  RadialGeom g[kMaxVarlenItems];
  int row0[kMaxVarlenItems + 1];
  long long rows = 0;
  for (int b = 0; b < num_items; ++b) {
    const int T = text_tokens ? text_tokens[b] : 0;
    if (frames[b] < 1 || tokens_per_frame[b] < 1 || T < 0) return BSA_ERR_INVALID_ARG;
    const long long nv = static_cast<long long>(frames[b]) * tokens_per_frame[b];
    const long long n = nv + T;
    if (n > 0x7fffffffLL) return BSA_ERR_INVALID_ARG;
    const int nb = ceil_div(n, block);
    if (nb > 262144) return BSA_ERR_UNSUPPORTED;
    g[b].frames = frames[b];
    g[b].tpf = tokens_per_frame[b];
    g[b].block = block;
    g[b].nv = static_cast<int>(nv);
    g[b].n = static_cast<int>(n);
    g[b].nb = nb;
    int rs = 0;
    if (tokens_per_frame[b] >= block)
      while ((tokens_per_frame[b] >> (rs + 1)) >= block) ++rs;
    g[b].rstar = rs;
    row0[b] = static_cast<int>(rows);
    rows += nb;
    if (rows > 0x7fffffffLL - 1) return BSA_ERR_UNSUPPORTED;
  }
  row0[num_items] = static_cast<int>(rows);
  for (int b = 0; b < num_items; ++b) {
    const size_t smem = static_cast<size_t>((g[b].nb + 31) / 32) * sizeof(uint32_t);
    radial_count_kernel<<<g[b].nb, 128, smem, stream>>>(g[b], row_ptr, row0[b]);
    BSA_CUDA(cudaGetLastError());
  }
  scan_rows_kernel<<<1, 1024, 0, stream>>>(row_ptr, row0[num_items]);
  BSA_CUDA(cudaGetLastError());
  if (nnz_out) {
    int32_t last = 0;
    BSA_CUDA(cudaMemcpyAsync(&last, row_ptr + row0[num_items], sizeof(int32_t),
                             cudaMemcpyDeviceToHost, stream));
    BSA_CUDA(cudaStreamSynchronize(stream));
    *nnz_out = last;
    if (col_idx && last > col_capacity) return BSA_ERR_CAPACITY;
  }
  if (col_idx) {
    for (int b = 0; b < num_items; ++b) {
      const size_t smem = static_cast<size_t>((g[b].nb + 31) / 32) * sizeof(uint32_t);
      radial_fill_kernel<<<g[b].nb, 128, smem, stream>>>(g[b], row_ptr, row0[b], col_idx,
                                                         col_capacity);
      BSA_CUDA(cudaGetLastError());
    }
  }
  return BSA_OK;
}

int bsa_radial_mask_build(int32_t frames, int32_t tokens_per_frame, int32_t block,
                          int32_t *row_ptr, int32_t *col_idx, int64_t col_capacity,
                          int64_t *nnz_out, bsa_stream_t stream_) {
  return bsa_joint_mask_build(frames, tokens_per_frame, 0, block, row_ptr, col_idx, col_capacity,
                              nnz_out, stream_);
}

static_assert(sizeof(bsa_tile_pattern) == (5 + 2 * BSA_TILE_PATTERN_MAX_BANDS) * sizeof(int32_t),
              "bsa_tile_pattern is a plain array of int32 fields");

int bsa_tile_pattern_lists_build(int32_t num_lists, int32_t num_q_blocks,
                                 const bsa_tile_pattern *patterns, const int32_t *columns,
                                 int64_t num_columns, int32_t *row_ptr, int32_t *col_idx,
                                 int64_t col_capacity, int64_t *nnz_out, bsa_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (num_lists < 1 || num_q_blocks < 1 || !patterns || !row_ptr || num_columns < 0 ||
      (num_columns > 0 && !columns))
    return BSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(patterns) | reinterpret_cast<uintptr_t>(row_ptr) |
       reinterpret_cast<uintptr_t>(columns) | reinterpret_cast<uintptr_t>(col_idx)) & 3u)
    return BSA_ERR_INVALID_ARG;
  if (num_q_blocks > 262144) return BSA_ERR_UNSUPPORTED;
  const long long rows = static_cast<long long>(num_lists) * num_q_blocks;
  if (rows >= 0x7fffffffLL) return BSA_ERR_INVALID_ARG;
  if (col_idx && col_capacity < 0) return BSA_ERR_INVALID_ARG;
  const size_t smem = static_cast<size_t>((num_q_blocks + 31) / 32) * sizeof(uint32_t);
  pattern_count_kernel<<<static_cast<unsigned>(rows), 128, smem, stream>>>(
      patterns, columns, num_columns, num_q_blocks, row_ptr);
  BSA_CUDA(cudaGetLastError());
  scan_rows_kernel<<<1, 1024, 0, stream>>>(row_ptr, static_cast<int>(rows));
  BSA_CUDA(cudaGetLastError());
  if (nnz_out) {
    int32_t last = 0;
    BSA_CUDA(cudaMemcpyAsync(&last, row_ptr + rows, sizeof(int32_t), cudaMemcpyDeviceToHost,
                             stream));
    BSA_CUDA(cudaStreamSynchronize(stream));
    *nnz_out = last;
    if (col_idx && last > col_capacity) return BSA_ERR_CAPACITY;
  }
  if (col_idx) {
    pattern_fill_kernel<<<static_cast<unsigned>(rows), 128, smem, stream>>>(
        patterns, columns, num_columns, num_q_blocks, row_ptr, col_idx, col_capacity);
    BSA_CUDA(cudaGetLastError());
  }
  return BSA_OK;
}

size_t bsa_attn_fwd_workspace_bytes(int32_t batch, int32_t heads, const bsa_block_lists *l) {
  if (!l || batch < 1 || heads < 1 || l->num_q_blocks < 1) return 0;
  if (l->num_lists != 1 && l->num_lists != heads) return 0;
  return order_bytes(l);
}

int bsa_attn_fwd(const void *q, const void *k, const void *v, int32_t batch, int32_t heads,
                 int32_t n, int32_t head_dim, float softmax_scale, const bsa_block_lists *l,
                 void *out, float *lse, void *workspace, size_t workspace_bytes,
                 bsa_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  int st = check_attn_args(q, k, v, batch, heads, n, head_dim, l, out);
  if (st != BSA_OK) return st;
  if (!workspace || !aligned16(workspace) || workspace_bytes < order_bytes(l))
    return BSA_ERR_INVALID_ARG;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return BSA_ERR_INVALID_ARG;
  DeviceInfo *dev = nullptr;
  if ((st = current_device(&dev)) != BSA_OK) return st;
  if (dev->cc_major != 10) return BSA_ERR_UNSUPPORTED;

  int fault_flags;
  {
    std::lock_guard<std::mutex> lk(g_hook_mu);
    fault_flags = g_fault_flags;
    g_fault_flags = 0;
  }
  int32_t *order = static_cast<int32_t *>(workspace);
  int32_t *counter = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(workspace) +
                                                 order_only_bytes(l));
  return run_fwd(contiguous_views(q, k, v, batch, heads, n, head_dim), n, head_dim,
                 softmax_scale, l, out, contiguous_layout(heads, n, head_dim), lse, order,
                 counter, dev, fault_flags, stream,
                 static_cast<uint8_t *>(workspace) + order_only_bytes(l) + 256);
}

int bsa_attn_fwd_strided(const void *q, const bsa_layout *q_layout, const void *k,
                         const bsa_layout *k_layout, const void *v, const bsa_layout *v_layout,
                         int32_t batch, int32_t heads, int32_t n, int32_t head_dim,
                         float softmax_scale, const bsa_block_lists *l, void *out,
                         const bsa_layout *out_layout, float *lse, void *workspace,
                         size_t workspace_bytes, bsa_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  int st = check_strided_args(q, q_layout, k, k_layout, v, v_layout, batch, heads, n, head_dim,
                              l, out, out_layout);
  if (st != BSA_OK) return st;
  if (!workspace || !aligned16(workspace) || workspace_bytes < order_bytes(l))
    return BSA_ERR_INVALID_ARG;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return BSA_ERR_INVALID_ARG;
  DeviceInfo *dev = nullptr;
  if ((st = current_device(&dev)) != BSA_OK) return st;
  if (dev->cc_major != 10) return BSA_ERR_UNSUPPORTED;
  int fault_flags;
  {
    std::lock_guard<std::mutex> lk(g_hook_mu);
    fault_flags = g_fault_flags;
    g_fault_flags = 0;
  }
  QkvViews x;
  x.q = q;
  x.k = k;
  x.v = v;
  x.lq = *q_layout;
  x.lk = *k_layout;
  x.lv = *v_layout;
  x.batch = batch;
  x.heads = heads;
  int32_t *order = static_cast<int32_t *>(workspace);
  int32_t *counter = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(workspace) +
                                                 order_only_bytes(l));
  return run_fwd(x, n, head_dim, softmax_scale, l, out, *out_layout, lse, order, counter, dev,
                 fault_flags, stream, static_cast<uint8_t *>(workspace) + order_only_bytes(l) + 256);
}

size_t bsa_attn_fwd_varlen_workspace_bytes(int32_t num_items, const int32_t *cu_seqlens,
                                           int32_t heads, const bsa_block_lists *l) {
  if (!l || heads < 1 || (l->num_lists != 1 && l->num_lists != heads)) return 0;
  if (l->block != 64 && l->block != 128) return 0;
  VarlenTable vt;
  int32_t mx = 0;
  if (varlen_table(num_items, cu_seqlens, heads, 128, &vt, &mx) != BSA_OK) return 0;
  return varlen_fwd_layout(vt, l).total;
}

int bsa_attn_fwd_varlen(const void *q, const bsa_layout *q_layout, const void *k,
                        const bsa_layout *k_layout, const void *v, const bsa_layout *v_layout,
                        int32_t num_items, const int32_t *cu_seqlens, int32_t heads,
                        int32_t head_dim, float softmax_scale, const bsa_block_lists *l,
                        void *out, const bsa_layout *out_layout, float *lse, void *workspace,
                        size_t workspace_bytes, bsa_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (!q_layout || !k_layout || !v_layout || !out_layout) return BSA_ERR_INVALID_ARG;
  if (!q || !k || !v || !out || !l || !l->row_ptr || (l->nnz > 0 && !l->col_idx))
    return BSA_ERR_INVALID_ARG;
  if (heads < 1) return BSA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return BSA_ERR_UNSUPPORTED;
  if (l->block != 64 && l->block != 128) return BSA_ERR_UNSUPPORTED;
  if (l->num_lists != 1 && l->num_lists != heads) return BSA_ERR_INVALID_ARG;
  if (l->nnz < 0) return BSA_ERR_INVALID_ARG;
  // vt: the items in blocks of the lists; vt128: in 128-row tiles (the
  // kernel's pairs and work items; the same table at block 128)
  VarlenTable vt, vt128;
  int32_t max_nqb = 0, max_nt = 0;
  int st;
  if ((st = varlen_table(num_items, cu_seqlens, heads, l->block, &vt, &max_nqb)) != BSA_OK)
    return st;
  if ((st = varlen_table(num_items, cu_seqlens, heads, 128, &vt128, &max_nt)) != BSA_OK)
    return st;
  const int32_t total = cu_seqlens[num_items];
  if (l->num_q_blocks != vt.row0[num_items] || l->num_k_blocks != max_nqb)
    return BSA_ERR_INVALID_ARG;
  if (static_cast<long long>(heads) * total > 0x7fffffffLL ||
      static_cast<long long>(l->num_lists) * l->num_q_blocks > 0x7fffffffLL)
    return BSA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return BSA_ERR_INVALID_ARG;
  // the packed sequence is a batch of one: [1, heads, total, head_dim] views
  for (const bsa_layout *L : {q_layout, k_layout, v_layout, out_layout})
    if (!layout_ok(*L, 1, heads, total)) return BSA_ERR_INVALID_ARG;
  if (!layout_disjoint(*out_layout, 1, heads, total, head_dim)) return BSA_ERR_INVALID_ARG;
  const size_t so = layout_span_bytes(*out_layout, 1, heads, total, head_dim);
  if (overlaps(out, so, q, layout_span_bytes(*q_layout, 1, heads, total, head_dim)) ||
      overlaps(out, so, k, layout_span_bytes(*k_layout, 1, heads, total, head_dim)) ||
      overlaps(out, so, v, layout_span_bytes(*v_layout, 1, heads, total, head_dim)))
    return BSA_ERR_INVALID_ARG;
  const VarlenFwdLayout wl = varlen_fwd_layout(vt128, l);
  if (!workspace || !aligned16(workspace) || workspace_bytes < wl.total)
    return BSA_ERR_INVALID_ARG;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return BSA_ERR_INVALID_ARG;
  DeviceInfo *dev = nullptr;
  if ((st = current_device(&dev)) != BSA_OK) return st;
  if (dev->cc_major != 10) return BSA_ERR_UNSUPPORTED;
  int fault_flags;
  {
    std::lock_guard<std::mutex> lk(g_hook_mu);
    fault_flags = g_fault_flags;
    g_fault_flags = 0;
  }
  const int L = l->num_lists;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  int32_t *order = reinterpret_cast<int32_t *>(ws);
  int32_t *counter = reinterpret_cast<int32_t *>(ws + varlen_order_bytes(vt128, L) - 256);
  // The kernel walks 128-row tiles: block-128 lists as they are; block-64
  // lists merged item by item into tile lists with the quarter masks
  // (counts per item, one scan over every item's tile rows, fills per item)
  const int32_t *rows = l->row_ptr;
  const int32_t *cols = l->col_idx;
  const uint8_t *masks = nullptr;
  int32_t nnz = l->nnz;
  if (l->block == 64) {
    int32_t *tile_ptr = reinterpret_cast<int32_t *>(ws + wl.tile_ptr);
    int32_t *tile_col = reinterpret_cast<int32_t *>(ws + wl.tile_col);
    uint8_t *tile_mask = ws + wl.tile_mask;
    const long long cap = l->nnz > 0 ? l->nnz : 1;
    bool first_seg = true;
    for (int b = 0; b < num_items; ++b) {
      const int nq = vt.row0[b + 1] - vt.row0[b], nt = vt128.row0[b + 1] - vt128.row0[b];
      if (nt == 0) continue;
      const int rows_t = L * nt;
      tile_count_kernel<<<(rows_t + 127) / 128, 128, 0, stream>>>(
          l->row_ptr + static_cast<long long>(L) * vt.row0[b], l->col_idx, nq, nq, l->nnz, nt,
          rows_t, tile_ptr + static_cast<long long>(L) * vt128.row0[b], first_seg ? 1 : 0);
      BSA_CUDA(cudaGetLastError());
      first_seg = false;
    }
    const int all_rows = L * vt128.row0[num_items];
    scan_rows_kernel<<<1, 1024, 0, stream>>>(tile_ptr, all_rows);
    BSA_CUDA(cudaGetLastError());
    for (int b = 0; b < num_items; ++b) {
      const int nq = vt.row0[b + 1] - vt.row0[b], nt = vt128.row0[b + 1] - vt128.row0[b];
      if (nt == 0) continue;
      const int rows_t = L * nt;
      tile_fill_kernel<<<(rows_t + 127) / 128, 128, 0, stream>>>(
          l->row_ptr + static_cast<long long>(L) * vt.row0[b], l->col_idx, nq, nq, l->nnz, nt,
          rows_t, tile_ptr + static_cast<long long>(L) * vt128.row0[b], tile_col, tile_mask, cap);
      BSA_CUDA(cudaGetLastError());
    }
    rows = tile_ptr;
    cols = tile_col;
    masks = tile_mask;
    nnz = static_cast<int32_t>(cap);
  }
  // work order per item: each item's pairs longest union first, per list;
  // the first launch also zeroes the work counter
  bool first = true;
  for (int b = 0; b < num_items; ++b) {
    const int nqb = vt128.row0[b + 1] - vt128.row0[b];
    if (nqb == 0) continue;
    const int npairs = (nqb + 1) / 2;
    const size_t smem = static_cast<size_t>(npairs <= kLptMaxRows ? npairs : 0) * sizeof(int);
    pair_order_kernel<<<L, 1024, smem, stream>>>(
        rows + static_cast<long long>(L) * vt128.row0[b], cols, nqb, nnz,
        order + static_cast<long long>(L) * vt128.pair0[b], kLptMaxRows,
        first ? counter : nullptr);
    BSA_CUDA(cudaGetLastError());
    first = false;
  }
  FwdParams p;
  p.row_ptr = rows;
  p.col_idx = cols;
  p.tile_mask = masks;
  p.order = order;
  p.item_counter = counter;
  p.out = static_cast<__nv_bfloat16 *>(out);
  p.o_sb = out_layout->batch_stride;
  p.o_sh = out_layout->head_stride;
  p.o_sn = out_layout->token_stride;
  p.lse = lse;
  p.heads = heads;
  p.n = total;
  p.nqb = vt128.row0[num_items];
  p.nkb = max_nt;
  p.num_lists = L;
  p.nnz = nnz;
  p.total_items = vt128.work0[num_items];
  const float scale =
      softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(head_dim));
  p.scale_log2 = scale * 1.4426950408889634f;
  {
    std::lock_guard<std::mutex> lk(g_hook_mu);
    p.wait_limit_ns = g_wait_limit_ns;
  }
  p.fault_flags = fault_flags;
  QkvViews x;
  x.q = q;
  x.k = k;
  x.v = v;
  x.lq = *q_layout;
  x.lk = *k_layout;
  x.lv = *v_layout;
  x.batch = 1;
  x.heads = heads;
  const int mode = l->block == 64 ? kModeVarlenQuarters : kModeVarlen;
  if (head_dim == 128) return launch_pair<128>(x, total, p, dev, mode, &vt128, stream);
  return launch_pair<64>(x, total, p, dev, mode, &vt128, stream);
}

size_t bsa_attn_fwd_patterns_workspace_bytes(int32_t num_patterns, int32_t num_q_blocks) {
  if (num_patterns < 1 || num_q_blocks < 1) return 0;
  return generated_layout(num_patterns, num_q_blocks).total;
}

int bsa_attn_fwd_patterns(const void *q, const void *k, const void *v, int32_t batch,
                          int32_t heads, int32_t n, int32_t head_dim, float softmax_scale,
                          int32_t num_patterns, const bsa_tile_pattern *patterns,
                          const int32_t *columns, int64_t num_columns,
                          const int32_t *head_pattern, void *out, float *lse, void *workspace,
                          size_t workspace_bytes, bsa_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (!patterns || num_columns < 0 || (num_columns > 0 && !columns)) return BSA_ERR_INVALID_ARG;
  if (num_patterns < 1 || num_patterns > kMaxGeneratedLists) return BSA_ERR_INVALID_ARG;
  if (!head_pattern && num_patterns != 1 && num_patterns != heads) return BSA_ERR_INVALID_ARG;
  if (n < 1) return BSA_ERR_INVALID_ARG;
  const int nqb = ceil_div(n, 128);
  // the argument checks of bsa_attn_fwd, on stand-in lists of the same shape
  bsa_block_lists shape;
  shape.num_lists = 1;
  shape.num_q_blocks = nqb;
  shape.num_k_blocks = nqb;
  shape.block = 128;
  shape.nnz = 0;
  shape.row_ptr = static_cast<const int32_t *>(workspace);
  shape.col_idx = nullptr;
  int st = check_attn_args(q, k, v, batch, heads, n, head_dim, &shape, out);
  if (st != BSA_OK) return st;
  const GeneratedLayout w = generated_layout(num_patterns, nqb);
  if (!workspace || !aligned16(workspace) || workspace_bytes < w.total) return BSA_ERR_INVALID_ARG;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return BSA_ERR_INVALID_ARG;
  if (static_cast<long long>(num_patterns) * nqb > 0x7fffffffLL) return BSA_ERR_UNSUPPORTED;
  DeviceInfo *dev = nullptr;
  if ((st = current_device(&dev)) != BSA_OK) return st;
  if (dev->cc_major != 10) return BSA_ERR_UNSUPPORTED;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  int32_t *row_ptr = reinterpret_cast<int32_t *>(ws + w.row_ptr);
  int32_t *order = reinterpret_cast<int32_t *>(ws + w.order);
  int32_t *counter = reinterpret_cast<int32_t *>(ws + w.counter);
  // row lengths of every pattern (the count pass of the list builder), then
  // the work order from the generated rows; no column list is written
  const int rows = num_patterns * nqb;
  const size_t bits = static_cast<size_t>((nqb + 31) / 32) * sizeof(uint32_t);
  pattern_count_kernel<<<rows, 128, bits, stream>>>(patterns, columns, num_columns, nqb, row_ptr);
  BSA_CUDA(cudaGetLastError());
  scan_rows_kernel<<<1, 1024, 0, stream>>>(row_ptr, rows);
  BSA_CUDA(cudaGetLastError());
  const int npairs = (nqb + 1) / 2;
  int32_t *cost = reinterpret_cast<int32_t *>(ws + w.cost);
  pattern_pair_union_kernel<<<num_patterns * npairs, 128, 2 * bits, stream>>>(
      patterns, columns, num_columns, nqb, cost);
  BSA_CUDA(cudaGetLastError());
  const size_t smem = static_cast<size_t>(npairs <= kLptMaxRows ? npairs : 0) * sizeof(int);
  rank_pairs_kernel<<<num_patterns, 1024, smem, stream>>>(cost, npairs, order, kLptMaxRows,
                                                          counter);
  BSA_CUDA(cudaGetLastError());
  FwdParams p = generated_params(batch, heads, n, nqb, num_patterns, row_ptr, order, counter,
                                 out, head_dim, lse, softmax_scale);
  p.patterns = patterns;
  p.pattern_columns = columns;
  p.num_pattern_columns = num_columns;
  p.head_list = head_pattern;
  const QkvViews x = contiguous_views(q, k, v, batch, heads, n, head_dim);
  if (head_dim == 128) return launch_pair<128>(x, n, p, dev, kModePatterns, nullptr, stream);
  return launch_pair<64>(x, n, p, dev, kModePatterns, nullptr, stream);
}

size_t bsa_attn_fwd_radial_workspace_bytes(int32_t frames, int32_t tokens_per_frame,
                                           int32_t text_tokens) {
  if (frames < 1 || tokens_per_frame < 1 || text_tokens < 0) return 0;
  const long long n = static_cast<long long>(frames) * tokens_per_frame + text_tokens;
  if (n > 0x7fffffffLL) return 0;
  return generated_layout(1, ceil_div(n, 128)).total;
}

int bsa_attn_fwd_radial(const void *q, const void *k, const void *v, int32_t batch,
                        int32_t heads, int32_t frames, int32_t tokens_per_frame,
                        int32_t text_tokens, int32_t head_dim, float softmax_scale, void *out,
                        float *lse, void *workspace, size_t workspace_bytes,
                        bsa_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (frames < 1 || tokens_per_frame < 1 || text_tokens < 0) return BSA_ERR_INVALID_ARG;
  // a key frame must fit the generator's 64-block window: it touches at most
  // (tokens_per_frame - 1) / 128 + 2 key blocks
  if ((tokens_per_frame - 1) / 128 + 2 > 64) return BSA_ERR_UNSUPPORTED;
  const long long nl = static_cast<long long>(frames) * tokens_per_frame + text_tokens;
  if (nl > 0x7fffffffLL) return BSA_ERR_INVALID_ARG;
  const int n = static_cast<int>(nl);
  const int nqb = ceil_div(n, 128);
  bsa_block_lists shape;
  shape.num_lists = 1;
  shape.num_q_blocks = nqb;
  shape.num_k_blocks = nqb;
  shape.block = 128;
  shape.nnz = 0;
  shape.row_ptr = static_cast<const int32_t *>(workspace);
  shape.col_idx = nullptr;
  int st = check_attn_args(q, k, v, batch, heads, n, head_dim, &shape, out);
  if (st != BSA_OK) return st;
  const GeneratedLayout w = generated_layout(1, nqb);
  if (!workspace || !aligned16(workspace) || workspace_bytes < w.total) return BSA_ERR_INVALID_ARG;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return BSA_ERR_INVALID_ARG;
  DeviceInfo *dev = nullptr;
  if ((st = current_device(&dev)) != BSA_OK) return st;
  if (dev->cc_major != 10) return BSA_ERR_UNSUPPORTED;
  RadialGeom g;
  g.frames = frames;
  g.tpf = tokens_per_frame;
  g.block = 128;
  g.nv = frames * tokens_per_frame;
  g.n = n;
  g.nb = nqb;
  int rs = 0;
  if (tokens_per_frame >= 128)
    while ((tokens_per_frame >> (rs + 1)) >= 128) ++rs;
  g.rstar = rs;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  int32_t *row_ptr = reinterpret_cast<int32_t *>(ws + w.row_ptr);
  int32_t *order = reinterpret_cast<int32_t *>(ws + w.order);
  int32_t *counter = reinterpret_cast<int32_t *>(ws + w.counter);
  const size_t bits = static_cast<size_t>((nqb + 31) / 32) * sizeof(uint32_t);
  radial_count_kernel<<<nqb, 128, bits, stream>>>(g, row_ptr, 0);
  BSA_CUDA(cudaGetLastError());
  scan_rows_kernel<<<1, 1024, 0, stream>>>(row_ptr, nqb);
  BSA_CUDA(cudaGetLastError());
  const int npairs = (nqb + 1) / 2;
  int32_t *cost = reinterpret_cast<int32_t *>(ws + w.cost);
  radial_pair_union_kernel<<<npairs, 128, bits, stream>>>(g, cost);
  BSA_CUDA(cudaGetLastError());
  const size_t smem = static_cast<size_t>(npairs <= kLptMaxRows ? npairs : 0) * sizeof(int);
  rank_pairs_kernel<<<1, 1024, smem, stream>>>(cost, npairs, order, kLptMaxRows, counter);
  BSA_CUDA(cudaGetLastError());
  FwdParams p = generated_params(batch, heads, n, nqb, 1, row_ptr, order, counter, out,
                                 head_dim, lse, softmax_scale);
  p.radial = g;
  const QkvViews x = contiguous_views(q, k, v, batch, heads, n, head_dim);
  if (head_dim == 128) return launch_pair<128>(x, n, p, dev, kModeRadial, nullptr, stream);
  return launch_pair<64>(x, n, p, dev, kModeRadial, nullptr, stream);
}

}  // extern "C"

namespace {

// Argument checks shared by the strided and variable-length backward entries:
// the eight views of [batch, heads, n, head_dim] (q, k, v, out, dout, dq, dk,
// dv), lse (lbytes bytes) and `need` bytes of workspace.
int check_bwd_views(const void *const ptrs[8], const bsa_layout *const lays[8], const float *lse,
                    int32_t batch, int32_t heads, int32_t n, int32_t head_dim, size_t lbytes,
                    const void *workspace, size_t workspace_bytes, size_t need) {
  for (int i = 0; i < 8; ++i) {
    if (!aligned16(ptrs[i])) return BSA_ERR_INVALID_ARG;
    if (!layout_ok(*lays[i], batch, heads, n)) return BSA_ERR_INVALID_ARG;
  }
  if (reinterpret_cast<uintptr_t>(lse) & 3u) return BSA_ERR_INVALID_ARG;
  size_t span[8];
  for (int i = 0; i < 8; ++i) span[i] = layout_span_bytes(*lays[i], batch, heads, n, head_dim);
  for (int a = 5; a < 8; ++a) {  // the gradients
    if (!layout_disjoint(*lays[a], batch, heads, n, head_dim)) return BSA_ERR_INVALID_ARG;
    for (int b = 0; b < 5; ++b)
      if (overlaps(ptrs[a], span[a], ptrs[b], span[b])) return BSA_ERR_INVALID_ARG;
    if (overlaps(ptrs[a], span[a], lse, lbytes)) return BSA_ERR_INVALID_ARG;
    for (int b = a + 1; b < 8; ++b)
      if (!views_disjoint(ptrs[a], *lays[a], ptrs[b], *lays[b], batch, heads, n, head_dim))
        return BSA_ERR_INVALID_ARG;
  }
  if (!workspace || !aligned16(workspace) || workspace_bytes < need) return BSA_ERR_INVALID_ARG;
  for (int i = 0; i < 8; ++i)
    if (overlaps(workspace, need, ptrs[i], span[i])) return BSA_ERR_INVALID_ARG;
  if (overlaps(workspace, need, lse, lbytes)) return BSA_ERR_INVALID_ARG;
  return BSA_OK;
}

BwdViews bwd_views(const void *const ptrs[8], const bsa_layout *const lays[8], int batch,
                   int heads) {
  BwdViews x;
  x.q = ptrs[0];
  x.k = ptrs[1];
  x.v = ptrs[2];
  x.out = ptrs[3];
  x.dout = ptrs[4];
  x.dq = const_cast<void *>(ptrs[5]);
  x.dk = const_cast<void *>(ptrs[6]);
  x.dv = const_cast<void *>(ptrs[7]);
  x.lq = *lays[0];
  x.lk = *lays[1];
  x.lv = *lays[2];
  x.lo = *lays[3];
  x.ldo = *lays[4];
  x.ldq = *lays[5];
  x.ldk = *lays[6];
  x.ldv = *lays[7];
  x.batch = batch;
  x.heads = heads;
  return x;
}

// lse2 / delta for every item's padded rows (item by item, head by head),
// the transposed lists of all items, the work counters.
size_t varlen_bwd_bytes(const VarlenTable &vt, int heads, const bsa_block_lists *l) {
  return bwd_layout(1, heads, vt.row0[vt.num_items] * kBwdBlock, l).total;
}

}  // namespace

extern "C" {

int bsa_attn_bwd_strided(const void *q, const bsa_layout *q_layout, const void *k,
                         const bsa_layout *k_layout, const void *v, const bsa_layout *v_layout,
                         const void *out, const bsa_layout *out_layout, const void *dout,
                         const bsa_layout *dout_layout, const float *lse, int32_t batch,
                         int32_t heads, int32_t n, int32_t head_dim, float softmax_scale,
                         const bsa_block_lists *l, void *dq, const bsa_layout *dq_layout,
                         void *dk, const bsa_layout *dk_layout, void *dv,
                         const bsa_layout *dv_layout, void *workspace, size_t workspace_bytes,
                         bsa_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const bsa_layout *lays[8] = {q_layout, k_layout,  v_layout,  out_layout,
                               dout_layout, dq_layout, dk_layout, dv_layout};
  const void *ptrs[8] = {q, k, v, out, dout, dq, dk, dv};
  for (int i = 0; i < 8; ++i)
    if (!lays[i] || !ptrs[i]) return BSA_ERR_INVALID_ARG;
  if (!lse || !l || !l->row_ptr || (l->nnz > 0 && !l->col_idx)) return BSA_ERR_INVALID_ARG;
  if (batch < 1 || heads < 1 || n < 1) return BSA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return BSA_ERR_UNSUPPORTED;
  if (l->block != 64 && l->block != 128) return BSA_ERR_UNSUPPORTED;
  const long long nb = (static_cast<long long>(n) + l->block - 1) / l->block;
  if (l->num_q_blocks != nb || l->num_k_blocks != nb) return BSA_ERR_INVALID_ARG;
  if (l->num_lists != 1 && l->num_lists != heads) return BSA_ERR_INVALID_ARG;
  if (l->nnz < 0) return BSA_ERR_INVALID_ARG;
  const long long bhl = static_cast<long long>(batch) * heads;
  if (bhl * nb > 0x7fffffffLL || bhl * n > 0x7fffffffLL) return BSA_ERR_UNSUPPORTED;
  const size_t lbytes = static_cast<size_t>(bhl) * n * sizeof(float);
  const size_t need = bwd_layout(batch, heads, n, l).total;
  int st = check_bwd_views(ptrs, lays, lse, batch, heads, n, head_dim, lbytes, workspace,
                           workspace_bytes, need);
  if (st != BSA_OK) return st;
  DeviceInfo *dev = nullptr;
  if ((st = current_device(&dev)) != BSA_OK) return st;
  if (dev->cc_major != 10) return BSA_ERR_UNSUPPORTED;
  const BwdViews x = bwd_views(ptrs, lays, batch, heads);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  if (head_dim == 128) return launch_bwd<128>(x, lse, n, softmax_scale, l, ws, dev, stream);
  return launch_bwd<64>(x, lse, n, softmax_scale, l, ws, dev, stream);
}

size_t bsa_attn_bwd_varlen_workspace_bytes(int32_t num_items, const int32_t *cu_seqlens,
                                           int32_t heads, const bsa_block_lists *l) {
  if (!l || heads < 1 || (l->block != 64 && l->block != 128) ||
      (l->num_lists != 1 && l->num_lists != heads))
    return 0;
  VarlenTable vt;
  int32_t mx = 0;
  if (varlen_table(num_items, cu_seqlens, heads, 128, &vt, &mx) != BSA_OK) return 0;
  if (static_cast<long long>(heads) * vt.row0[num_items] * kBwdBlock > 0x7fffffffLL) return 0;
  return varlen_bwd_bytes(vt, heads, l);
}

int bsa_attn_bwd_varlen(const void *q, const bsa_layout *q_layout, const void *k,
                        const bsa_layout *k_layout, const void *v, const bsa_layout *v_layout,
                        const void *out, const bsa_layout *out_layout, const void *dout,
                        const bsa_layout *dout_layout, const float *lse, int32_t num_items,
                        const int32_t *cu_seqlens, int32_t heads, int32_t head_dim,
                        float softmax_scale, const bsa_block_lists *l, void *dq,
                        const bsa_layout *dq_layout, void *dk, const bsa_layout *dk_layout,
                        void *dv, const bsa_layout *dv_layout, void *workspace,
                        size_t workspace_bytes, bsa_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const bsa_layout *lays[8] = {q_layout, k_layout,  v_layout,  out_layout,
                               dout_layout, dq_layout, dk_layout, dv_layout};
  const void *ptrs[8] = {q, k, v, out, dout, dq, dk, dv};
  for (int i = 0; i < 8; ++i)
    if (!lays[i] || !ptrs[i]) return BSA_ERR_INVALID_ARG;
  if (!lse || !l || !l->row_ptr || (l->nnz > 0 && !l->col_idx)) return BSA_ERR_INVALID_ARG;
  if (heads < 1) return BSA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return BSA_ERR_UNSUPPORTED;
  if (l->block != 64 && l->block != 128) return BSA_ERR_UNSUPPORTED;
  if (l->num_lists != 1 && l->num_lists != heads) return BSA_ERR_INVALID_ARG;
  if (l->nnz < 0) return BSA_ERR_INVALID_ARG;
  // vt_l: the items in blocks of the lists; vt: in 128-row tiles
  VarlenTable vt_l, vt;
  int32_t max_nqb = 0, max_nt = 0;
  int st;
  if ((st = varlen_table(num_items, cu_seqlens, heads, l->block, &vt_l, &max_nqb)) != BSA_OK)
    return st;
  if ((st = varlen_table(num_items, cu_seqlens, heads, kBwdBlock, &vt, &max_nt)) != BSA_OK)
    return st;
  const int32_t total = cu_seqlens[num_items];
  if (l->num_q_blocks != vt_l.row0[num_items] || l->num_k_blocks != max_nqb)
    return BSA_ERR_INVALID_ARG;
  if (static_cast<long long>(heads) * total > 0x7fffffffLL ||
      static_cast<long long>(l->num_lists) * l->num_q_blocks > 0x7fffffffLL ||
      static_cast<long long>(heads) * vt.row0[num_items] * kBwdBlock > 0x7fffffffLL)
    return BSA_ERR_UNSUPPORTED;
  // the packed sequence is a batch of one: [1, heads, total, head_dim] views
  const size_t lbytes = static_cast<size_t>(heads) * total * sizeof(float);
  const size_t need = varlen_bwd_bytes(vt, heads, l);
  if ((st = check_bwd_views(ptrs, lays, lse, 1, heads, total, head_dim, lbytes, workspace,
                            workspace_bytes, need)) != BSA_OK)
    return st;
  DeviceInfo *dev = nullptr;
  if ((st = current_device(&dev)) != BSA_OK) return st;
  if (dev->cc_major != 10) return BSA_ERR_UNSUPPORTED;
  const BwdViews x = bwd_views(ptrs, lays, 1, heads);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  if (head_dim == 128)
    return launch_bwd_varlen<128>(x, lse, total, softmax_scale, l, vt_l, vt, ws, dev, stream);
  return launch_bwd_varlen<64>(x, lse, total, softmax_scale, l, vt_l, vt, ws, dev, stream);
}

size_t bsa_attn_bwd_workspace_bytes(int32_t batch, int32_t heads, int32_t n,
                                    const bsa_block_lists *l) {
  if (!l || batch < 1 || heads < 1 || n < 1 || l->num_q_blocks < 1 || l->num_k_blocks < 1)
    return 0;
  if (l->num_lists != 1 && l->num_lists != heads) return 0;
  if ((l->block != 64 && l->block != 128) || l->num_q_blocks != ceil_div(n, l->block)) return 0;
  return bwd_layout(batch, heads, n, l).total;
}

}  // extern "C"

namespace {

// bsa_attn_bwd and bsa_attn_bwd_one_pass: contiguous views, the two-kernel
// or (one_pass, block 128) the one-pass backward.
int attn_bwd_contiguous(const void *q, const void *k, const void *v, const void *out,
                        const void *dout, const float *lse, int32_t batch, int32_t heads,
                        int32_t n, int32_t head_dim, float softmax_scale,
                        const bsa_block_lists *l, void *dq, void *dk, void *dv, void *workspace,
                        size_t workspace_bytes, bsa_stream_t stream_, bool one_pass) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  int st = check_attn_args(q, k, v, batch, heads, n, head_dim, l, dq);
  if (st != BSA_OK) return st;
  if (!out || !dout || !lse || !dk || !dv) return BSA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(dout) || !aligned16(dk) || !aligned16(dv) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return BSA_ERR_INVALID_ARG;
  const size_t bytes = static_cast<size_t>(batch) * heads * n * head_dim * 2;
  const size_t lbytes = static_cast<size_t>(batch) * heads * n * sizeof(float);
  const void *ins[6] = {q, k, v, out, dout, lse};
  const size_t in_bytes[6] = {bytes, bytes, bytes, bytes, bytes, lbytes};
  void *outs[3] = {dq, dk, dv};
  for (int a = 0; a < 3; ++a) {
    for (int b = 0; b < 6; ++b)
      if (overlaps(outs[a], bytes, ins[b], in_bytes[b])) return BSA_ERR_INVALID_ARG;
    for (int b = a + 1; b < 3; ++b)
      if (overlaps(outs[a], bytes, outs[b], bytes)) return BSA_ERR_INVALID_ARG;
  }
  if (one_pass && l->block != kBwdBlock) return BSA_ERR_UNSUPPORTED;
  const size_t need = bwd_layout(batch, heads, n, l, one_pass).total;
  if (!workspace || !aligned16(workspace) || workspace_bytes < need) return BSA_ERR_INVALID_ARG;
  if (overlaps(workspace, need, ins[0], bytes) || overlaps(workspace, need, dq, bytes) ||
      overlaps(workspace, need, dk, bytes) || overlaps(workspace, need, dv, bytes))
    return BSA_ERR_INVALID_ARG;
  DeviceInfo *dev = nullptr;
  if ((st = current_device(&dev)) != BSA_OK) return st;
  if (dev->cc_major != 10) return BSA_ERR_UNSUPPORTED;
  BwdViews x;
  x.q = q;
  x.k = k;
  x.v = v;
  x.out = out;
  x.dout = dout;
  x.dq = dq;
  x.dk = dk;
  x.dv = dv;
  x.lq = x.lk = x.lv = x.lo = x.ldo = x.ldq = x.ldk = x.ldv =
      contiguous_layout(heads, n, head_dim);
  x.batch = batch;
  x.heads = heads;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  if (head_dim == 128)
    return launch_bwd<128>(x, lse, n, softmax_scale, l, ws, dev, stream, one_pass);
  return launch_bwd<64>(x, lse, n, softmax_scale, l, ws, dev, stream, one_pass);
}

}  // namespace

extern "C" {

int bsa_attn_bwd(const void *q, const void *k, const void *v, const void *out, const void *dout,
                 const float *lse, int32_t batch, int32_t heads, int32_t n, int32_t head_dim,
                 float softmax_scale, const bsa_block_lists *l, void *dq, void *dk, void *dv,
                 void *workspace, size_t workspace_bytes, bsa_stream_t stream) {
  return attn_bwd_contiguous(q, k, v, out, dout, lse, batch, heads, n, head_dim, softmax_scale, l,
                             dq, dk, dv, workspace, workspace_bytes, stream, false);
}

size_t bsa_attn_bwd_one_pass_workspace_bytes(int32_t batch, int32_t heads, int32_t n,
                                             const bsa_block_lists *l) {
  if (bsa_attn_bwd_workspace_bytes(batch, heads, n, l) == 0 || l->block != kBwdBlock) return 0;
  return bwd_layout(batch, heads, n, l, true).total;
}

int bsa_attn_bwd_one_pass(const void *q, const void *k, const void *v, const void *out,
                          const void *dout, const float *lse, int32_t batch, int32_t heads,
                          int32_t n, int32_t head_dim, float softmax_scale,
                          const bsa_block_lists *l, void *dq, void *dk, void *dv, void *workspace,
                          size_t workspace_bytes, bsa_stream_t stream) {
  return attn_bwd_contiguous(q, k, v, out, dout, lse, batch, heads, n, head_dim, softmax_scale, l,
                             dq, dk, dv, workspace, workspace_bytes, stream, true);
}

int bsa_attn_dense_masked_ref(const void *q, const void *k, const void *v, int32_t batch,
                              int32_t heads, int32_t n, int32_t head_dim, float softmax_scale,
                              const bsa_block_lists *l, void *out, float *lse,
                              bsa_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  int st = check_attn_args(q, k, v, batch, heads, n, head_dim, l, out);
  if (st != BSA_OK) return st;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return BSA_ERR_INVALID_ARG;
  if (batch > 65535 || heads > 65535) return BSA_ERR_UNSUPPORTED;
  DeviceInfo *dev = nullptr;
  if ((st = current_device(&dev)) != BSA_OK) return st;
  RefParams p;
  p.q = static_cast<const __nv_bfloat16 *>(q);
  p.k = static_cast<const __nv_bfloat16 *>(k);
  p.v = static_cast<const __nv_bfloat16 *>(v);
  p.out = static_cast<__nv_bfloat16 *>(out);
  p.lse = lse;
  p.row_ptr = l->row_ptr;
  p.col_idx = l->col_idx;
  p.heads = heads;
  p.n = n;
  p.nqb = l->num_q_blocks;
  p.nkb = l->num_k_blocks;
  p.num_lists = l->num_lists;
  p.nnz = l->nnz;
  p.scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(head_dim));
  const int slot = slot_of(head_dim, l->block);
  if (head_dim == 128 && l->block == 128) return launch_ref<128, 128>(p, batch, dev, slot, stream);
  if (head_dim == 128 && l->block == 64) return launch_ref<128, 64>(p, batch, dev, slot, stream);
  if (head_dim == 64 && l->block == 128) return launch_ref<64, 128>(p, batch, dev, slot, stream);
  return launch_ref<64, 64>(p, batch, dev, slot, stream);
}

int bsa_validate_lists(const bsa_block_lists *l, bsa_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (!l || !l->row_ptr || l->num_lists < 1 || l->num_q_blocks < 1 || l->num_k_blocks < 1 ||
      l->nnz < 0 || (l->nnz > 0 && !l->col_idx))
    return BSA_ERR_INVALID_ARG;
  const long long rows = static_cast<long long>(l->num_lists) * l->num_q_blocks;
  if (rows > (1LL << 28)) return BSA_ERR_INVALID_ARG;
  int32_t *host = static_cast<int32_t *>(std::malloc(static_cast<size_t>(rows + 1) * sizeof(int32_t)));
  if (!host) return BSA_ERR_INVALID_ARG;
  cudaError_t e = cudaMemcpyAsync(host, l->row_ptr, static_cast<size_t>(rows + 1) * sizeof(int32_t),
                                  cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) {
    std::free(host);
    return cuda_fail(e, "bsa_validate_lists: read row_ptr");
  }
  bool bad = host[0] != 0 || host[rows] != l->nnz;
  for (long long r = 0; r < rows && !bad; ++r) bad = host[r + 1] < host[r];
  std::free(host);
  if (bad) return BSA_ERR_BAD_LISTS;
  // The device check reports through the status word; keep whatever another
  // kernel recorded before and restore it afterwards.
  unsigned int prior = 0, zero = 0, after = 0;
  BSA_CUDA(cudaStreamSynchronize(stream));
  BSA_CUDA(cudaMemcpyFromSymbol(&prior, g_status, sizeof(prior)));
  BSA_CUDA(cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)));
  const int threads = 256;
  const long long blocks = (rows + threads - 1) / threads;
  validate_cols_kernel<<<static_cast<int>(blocks < 4096 ? blocks : 4096), threads, 0, stream>>>(
      l->row_ptr, l->col_idx, static_cast<int>(rows), l->num_k_blocks);
  BSA_CUDA(cudaGetLastError());
  BSA_CUDA(cudaStreamSynchronize(stream));
  BSA_CUDA(cudaMemcpyFromSymbol(&after, g_status, sizeof(after)));
  BSA_CUDA(cudaMemcpyToSymbol(g_status, &prior, sizeof(prior)));
  return after == BSA_ERR_BAD_LISTS ? BSA_ERR_BAD_LISTS : BSA_OK;
}

int bsa_get_device_status(bsa_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  BSA_CUDA(cudaStreamSynchronize(stream));
  unsigned int v = 0, zero = 0;
  BSA_CUDA(cudaMemcpyFromSymbol(&v, g_status, sizeof(v)));
  BSA_CUDA(cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)));
  return static_cast<int>(v);
}

int bsa_get_timeout_detail(int32_t *out4) {
  if (!out4) return BSA_ERR_INVALID_ARG;
  unsigned int d[4];
  BSA_CUDA(cudaMemcpyFromSymbol(d, g_status_detail, sizeof(d)));
  for (int i = 0; i < 4; ++i) out4[i] = static_cast<int32_t>(d[i]);
  return BSA_OK;
}

const char *bsa_status_string(int status) {
  switch (status) {
    case BSA_OK: return "ok";
    case BSA_ERR_INVALID_ARG: return "invalid argument";
    case BSA_ERR_UNSUPPORTED: return "unsupported head_dim, block or device";
    case BSA_ERR_CUDA: return "CUDA runtime error";
    case BSA_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case BSA_ERR_BAD_LISTS: return "malformed block lists";
    case BSA_ERR_CAPACITY: return "col_idx capacity too small";
    case BSA_ERR_SCRATCH_LIMIT: return "problem exceeds the fixed scratch of bsa_attn_fwd_noalloc";
    default: return "unknown status";
  }
}

const char *bsa_last_cuda_error(void) { return t_last_error; }

int bsa_selftest_exp2(const float *x, float *y_poly, float *y_mufu, float *y_ref, int32_t n,
                      bsa_stream_t stream_) {
  if (!x || !y_poly || !y_mufu || !y_ref || n < 2 || (n & 1)) return BSA_ERR_INVALID_ARG;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const int pairs = n / 2;
  exp2_selftest_kernel<<<(pairs + 255) / 256, 256, 0, stream>>>(x, y_poly, y_mufu, y_ref, n);
  BSA_CUDA(cudaGetLastError());
  return BSA_OK;
}

int bsa_gemm_bf16(const void *a, int64_t lda, int32_t a_mn_major, const void *b, int64_t ldb,
                  int32_t b_mn_major, const void *bias, void *d, int64_t ldd, int64_t m,
                  int64_t n, int64_t k, bsa_stream_t stream) {
  return gemm_bf16(a, lda, a_mn_major != 0, b, ldb, b_mn_major != 0, bias, d, ldd, m, n, k,
                   reinterpret_cast<cudaStream_t>(stream));
}

int bsa_set_test_hooks(int64_t wait_limit_ns, int32_t fault_flags) {
  if (wait_limit_ns < 0) return BSA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_hook_mu);
  g_wait_limit_ns = wait_limit_ns == 0 ? 2000000000ull : static_cast<unsigned long long>(wait_limit_ns);
  g_fault_flags = fault_flags & 1;
  g_force_one_tile = (fault_flags & 2) != 0;
  return BSA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free entry point. Its scratch (the work order, then the work
// counter) is this fixed array instead of a caller-provided workspace. In host code `g_noalloc_order`
// names a host-side stand-in, not device memory, so the device address is
// resolved once per device with cudaGetSymbolAddress and cached.
// ---------------------------------------------------------------------------

static __device__ __align__(256) int32_t g_noalloc_order[BSA_NOALLOC_MAX_ORDER_ENTRIES + 64];

namespace bsa {
namespace {
std::mutex g_noalloc_mu;
int32_t *g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_order on the current device (set up on first use).
int noalloc_scratch(int32_t **out) {
  int dev = 0;
  BSA_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return BSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void *p = nullptr;
    BSA_CUDA(cudaGetSymbolAddress(&p, g_noalloc_order));
    g_noalloc_ptr[dev] = static_cast<int32_t *>(p);
  }
  *out = g_noalloc_ptr[dev];
  return BSA_OK;
}
}  // namespace
}  // namespace bsa

extern "C" int bsa_attn_fwd_noalloc(const void *q, const void *k, const void *v, int32_t batch,
                                    int32_t heads, int32_t n, int32_t head_dim,
                                    float softmax_scale, const bsa_block_lists *l, void *out,
                                    float *lse, bsa_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  int st = check_attn_args(q, k, v, batch, heads, n, head_dim, l, out);
  if (st != BSA_OK) return st;
  if (static_cast<long long>(l->num_lists) * l->num_q_blocks > BSA_NOALLOC_MAX_ORDER_ENTRIES)
    return BSA_ERR_SCRATCH_LIMIT;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return BSA_ERR_INVALID_ARG;
  DeviceInfo *dev = nullptr;
  if ((st = current_device(&dev)) != BSA_OK) return st;
  if (dev->cc_major != 10) return BSA_ERR_UNSUPPORTED;
  int32_t *order = nullptr;
  if ((st = noalloc_scratch(&order)) != BSA_OK) return st;

  return run_fwd(contiguous_views(q, k, v, batch, heads, n, head_dim), n, head_dim,
                 softmax_scale, l, out, contiguous_layout(heads, n, head_dim), lse, order,
                 order + BSA_NOALLOC_MAX_ORDER_ENTRIES, dev, 0, stream);
}
