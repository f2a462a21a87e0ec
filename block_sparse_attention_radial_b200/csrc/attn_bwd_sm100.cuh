// Block-sparse attention backward for sm_100a (block 128, head_dim 64/128).
//
// Gradients of O = softmax(Q K^T * scale restricted to the listed blocks) V,
// given dO and the forward's lse (the derivative of the forward definition;
// the pages fine-tune the radial attention module with LoRA, [RA-skill]
// Step 4, which runs this pass):
//   P = exp(S * scale - lse),  dV = P^T dO,  dP = dO V^T,
//   delta_i = sum_d dO_id O_id,  dS = P * (dP - delta),
//   dQ = dS K * scale,  dK = dS^T Q * scale.
//
// Three steps:
//   bwd_prep_kernel    delta and lse * log2(e) per query row, padded to whole
//                      blocks (padding: delta 0, lse +inf, so P = 0 there)
//   csc_*_kernel       the lists transposed: per key block, its query blocks
//                      in ascending order (deterministic accumulation order)
//   attn_bwd_dkdv_kernel  one item = (batch*head, key block): K and V stay in
//                      shared memory while the key block's query blocks
//                      stream through; dK and dV accumulate in TMEM
//   attn_bwd_dq_kernel    one item = (batch*head, query block): Q and dO stay
//                      in shared memory while the row's key blocks stream
//                      through; dQ accumulates in TMEM
// No atomics: every output row is written once by one CTA, so the result is
// deterministic. dQ recomputes S and dP (7 block products per listed block
// instead of the 5 an atomic dQ needs).
//
// Both kernels use the forward's two MMA shapes (M128 N128 K16 with K-major
// operands from shared memory; M128 N=D with A from TMEM and an MN-major B),
// the same 4-D TMA boxes, and the same bounded waits (a timeout records
// BSA_ERR_DEVICE_TIMEOUT, raises the CTA abort flag and every role leaves).
#pragma once

#include <climits>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "attn_fwd_sm100.cuh"
#include "lists.cuh"

namespace bsa {

struct BwdParams {
  const int32_t *row_ptr, *col_idx;  // lists: query block -> key blocks
  const int32_t *col_ptr, *row_idx;  // transposed: key block -> query blocks
  const float *lse2;                 // [bh][nqb * 128]: lse * log2(e), +inf padding
  const float *delta;                // [bh][nqb * 128]: sum_d dO * O, 0 padding
  __nv_bfloat16 *dq, *dk, *dv;
  // element strides (batch, head, token) of dq, dk, dv; head_dim contiguous
  long long dq_s[3], dk_s[3], dv_s[3];
  // Block-64 lists run as 128-row tiles: a 4-bit mask per list entry, bit
  // qi * 2 + kj set when 64-row query block qi of the tile lists 64-key block
  // kj of the key tile (rmask per CSR entry, cmask per transposed entry).
  // Both null for block-128 lists (every pair of the tile is listed); read
  // only by the MASKED instances of the kernels.
  const uint8_t *rmask, *cmask;
  int32_t heads, n, nqb, nkb, num_lists, nnz;  // heads: per batch item
  int32_t total_items;
  int32_t *item_counter;  // next work item; zeroed by bwd_prep_kernel
  float scale, scale_log2;
  unsigned long long wait_limit_ns;
  // one-pass kernel only: the dQ accumulator rows ([bh][nqb * 128][D] fp32),
  // the part counters ([bh][nqb][4]) and, per transposed entry, the key
  // block's position in its query block's row
  float *dq_acc = nullptr;
  int32_t *dq_sem = nullptr;
  const int32_t *row_pos = nullptr;
};

constexpr int kBwdBlock = 128;
constexpr int kBwdItemN = 4;  // work items in flight between the producer and the consumers

// ------------------------------------------------------------------ prep --

// One thread per padded query row of one (batch*head): delta and lse2.
// out and dout are read through their (batch, head, token) element strides,
// lse through its (batch, head) strides l_sb, l_sh (rows contiguous).
template <int D>
__global__ void bwd_prep_kernel(const __nv_bfloat16 *out, const __nv_bfloat16 *dout,
                                const float *lse, float *lse2, float *delta, int n, int nqb,
                                int heads, long long o_sb, long long o_sh, long long o_sn,
                                long long d_sb, long long d_sh, long long d_sn, long long l_sb,
                                long long l_sh, long long rows_total, int32_t *item_counters) {
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx < 2) item_counters[idx] = 0;  // the dK/dV and the dQ kernel's work counters
  if (idx >= rows_total) return;
  const long long padded = static_cast<long long>(nqb) * kBwdBlock;
  const long long bh = idx / padded;
  const int i = static_cast<int>(idx - bh * padded);
  if (i >= n) {
    lse2[idx] = INFINITY;
    delta[idx] = 0.f;
    return;
  }
  const long long b = bh / heads, h = bh - b * heads;
  const long long row = b * l_sb + h * l_sh + i;
  const uint4 *o4 = reinterpret_cast<const uint4 *>(out + b * o_sb + h * o_sh + i * o_sn);
  const uint4 *d4 = reinterpret_cast<const uint4 *>(dout + b * d_sb + h * d_sh + i * d_sn);
  float acc = 0.f;
#pragma unroll 4
  for (int c = 0; c < D / 8; ++c) {
    const uint4 a = o4[c], b = d4[c];
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&aw[w]));
      const float2 fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&bw[w]));
      acc = fmaf(fa.x, fb.x, acc);
      acc = fmaf(fa.y, fb.y, acc);
    }
  }
  delta[idx] = acc;
  const float l = lse[row];
  lse2[idx] = l > -INFINITY ? l * 1.4426950408889634f : INFINITY;
}

// ------------------------------------------------------- transposed lists --

// Position of kb in the sorted row [a, b) of col_idx, or -1.
__device__ __forceinline__ int row_find(const int32_t *col_idx, int a, int b, int kb) {
  while (a < b) {
    const int m = (a + b) >> 1;
    const int v = col_idx[m];
    if (v == kb) return m;
    if (v < kb) a = m + 1;
    else b = m;
  }
  return -1;
}

__device__ __forceinline__ bool row_has(const int32_t *col_idx, int a, int b, int kb) {
  return row_find(col_idx, a, b, kb) >= 0;
}

// One CTA per (list, key block): how many query blocks list it.
// (first: also write col_cnt[0] = 0; later segments of a concatenation
// leave the entry before them alone)
__global__ void csc_count_kernel(const int32_t *row_ptr, const int32_t *col_idx, int nqb, int nkb,
                                 int nnz, int32_t *col_cnt, int first) {
  __shared__ int scratch[32];
  const int list = blockIdx.x / nkb, kb = blockIdx.x - list * nkb;
  const int32_t *rp = row_ptr + static_cast<long long>(list) * nqb;
  int c = 0;
  for (int qb = threadIdx.x; qb < nqb; qb += blockDim.x) {
    const int a = min(max(rp[qb], 0), nnz), b = min(max(rp[qb + 1], 0), nnz);
    c += row_has(col_idx, a, b, kb) ? 1 : 0;
  }
  int total;
  cta_inclusive_scan(c, scratch, total);
  if (threadIdx.x == 0) col_cnt[blockIdx.x + 1] = total;
  if (first && blockIdx.x == 0 && threadIdx.x == 0) col_cnt[0] = 0;
}

// One CTA per (list, key block): its query blocks in ascending order, at
// col_ptr (the inclusive scan of the counts), and with rmask given each
// entry's mask into cmask and (row_pos non-null) the key block's position in
// the query block's row into row_pos. Writes stay below `cap` (the entries
// row_idx holds) even for lists the validator would reject.
__global__ void csc_fill_kernel(const int32_t *row_ptr, const int32_t *col_idx, int nqb, int nkb,
                                int nnz, const int32_t *col_ptr, int32_t *row_idx, int cap,
                                const uint8_t *rmask, uint8_t *cmask, int32_t *row_pos) {
  __shared__ int scratch[32];
  const int list = blockIdx.x / nkb, kb = blockIdx.x - list * nkb;
  const int32_t *rp = row_ptr + static_cast<long long>(list) * nqb;
  int base = col_ptr[blockIdx.x];
  const int end = col_ptr[blockIdx.x + 1];
  for (int q0 = 0; q0 < nqb; q0 += blockDim.x) {
    const int qb = q0 + threadIdx.x;
    int at = -1, a = 0;
    if (qb < nqb) {
      a = min(max(rp[qb], 0), nnz);
      const int b = min(max(rp[qb + 1], 0), nnz);
      at = row_find(col_idx, a, b, kb);
    }
    const bool has = at >= 0;
    int total;
    const int inc = cta_inclusive_scan(has ? 1 : 0, scratch, total);
    const int pos = base + inc - 1;
    if (has && pos >= 0 && pos < end && pos < cap) {
      row_idx[pos] = qb;
      if (rmask) cmask[pos] = rmask[at];
      if (row_pos) row_pos[pos] = at - a;
    }
    base += total;
  }
}

// ------------------------------------------------- block-64 lists as tiles --
//
// The backward kernels work on 128 x 128 tiles. Lists at block 64 become tile
// lists: tile row t covers query blocks 2t and 2t+1, tile column u key blocks
// 2u and 2u+1; entry (t, u) exists when any of its four pairs is listed and
// carries the 4-bit mask of the listed pairs (bit qi * 2 + kj). One thread
// per tile row merges the two sorted rows; counts first, then (after a scan
// of the counts) the entries.
__device__ int merge_tile_row(const int32_t *col_idx, int a0, int a1, int b0, int b1, int nkb,
                              int32_t *cols, uint8_t *masks, long long cap) {
  int cnt = 0;
  while (a0 < a1 || b0 < b1) {
    const int ka = a0 < a1 ? min(max(col_idx[a0], 0), nkb - 1) >> 1 : 0x7fffffff;
    const int kb = b0 < b1 ? min(max(col_idx[b0], 0), nkb - 1) >> 1 : 0x7fffffff;
    const int u = min(ka, kb);
    uint32_t bits = 0;
    while (a0 < a1 && (min(max(col_idx[a0], 0), nkb - 1) >> 1) == u) {
      bits |= 1u << (min(max(col_idx[a0], 0), nkb - 1) & 1);
      ++a0;
    }
    while (b0 < b1 && (min(max(col_idx[b0], 0), nkb - 1) >> 1) == u) {
      bits |= 1u << (2 + (min(max(col_idx[b0], 0), nkb - 1) & 1));
      ++b0;
    }
    if (cols && cnt < cap) {
      cols[cnt] = u;
      masks[cnt] = static_cast<uint8_t>(bits);
    }
    ++cnt;
  }
  return cnt;
}

// rows = num_lists * nt tile rows; nqb, nkb count 64-blocks.
// (first: also write tile_ptr[0] = 0; later segments of a concatenation
// leave the entry before them alone)
__global__ void tile_count_kernel(const int32_t *row_ptr, const int32_t *col_idx, int nqb, int nkb,
                                  int nnz, int nt, int rows, int32_t *tile_ptr, int first) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (first && i == 0) tile_ptr[0] = 0;
  if (i >= rows) return;
  const int list = i / nt, t = i - list * nt;
  const int32_t *rp = row_ptr + static_cast<long long>(list) * nqb;
  const int q0 = 2 * t, q1 = 2 * t + 1;
  const int a0 = min(max(rp[q0], 0), nnz), a1 = min(max(rp[q0 + 1], 0), nnz);
  const int b0 = q1 < nqb ? min(max(rp[q1], 0), nnz) : 0;
  const int b1 = q1 < nqb ? min(max(rp[q1 + 1], 0), nnz) : 0;
  tile_ptr[i + 1] = merge_tile_row(col_idx, a0, max(a0, a1), b0, max(b0, b1), nkb, nullptr,
                                   nullptr, 0);
}

__global__ void tile_fill_kernel(const int32_t *row_ptr, const int32_t *col_idx, int nqb, int nkb,
                                 int nnz, int nt, int rows, const int32_t *tile_ptr,
                                 int32_t *tile_col, uint8_t *tile_mask, long long cap) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= rows) return;
  const int list = i / nt, t = i - list * nt;
  const int32_t *rp = row_ptr + static_cast<long long>(list) * nqb;
  const int q0 = 2 * t, q1 = 2 * t + 1;
  const int a0 = min(max(rp[q0], 0), nnz), a1 = min(max(rp[q0 + 1], 0), nnz);
  const int b0 = q1 < nqb ? min(max(rp[q1], 0), nnz) : 0;
  const int b1 = q1 < nqb ? min(max(rp[q1 + 1], 0), nnz) : 0;
  const long long at = tile_ptr[i];
  merge_tile_row(col_idx, a0, max(a0, a1), b0, max(b0, b1), nkb, tile_col + at, tile_mask + at,
                 cap - at);
}

// tcgen05.st of 16 columns (32x32b shape: thread t writes TMEM lane t).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

// 1-D bulk copy global -> shared (16-byte aligned, size a multiple of 16),
// completing on `bar`'s transaction count.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes,
                                          uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// ------------------------------------------------------------ dK / dV --

template <int D>
struct DkdvCfg {
  static constexpr int T = kBwdBlock * D * 2;        // one 128 x D bf16 tile
  static constexpr int STAGE = 2 * T + 1024;         // Q, dO, lse2 and delta of a query block
  static constexpr int NS_FIT = (kSmemLimit - 1024 - 1024 - 2 * T) / STAGE;
  static constexpr int NS = NS_FIT > 4 ? 4 : NS_FIT;
  static constexpr int DSMEM = 1024 + 2 * T + NS * STAGE;
  static constexpr uint32_t ST_COL = 0;              // S^T, then P^T (bf16) over its first 64
  static constexpr uint32_t DPT_COL = 128;           // dP^T, then dS^T (bf16) over its first 64
  static constexpr uint32_t DV_COL = 256;
  static constexpr uint32_t DK_COL = 256 + D;
  static constexpr int THREADS = 192;
  static_assert(NS >= 2, "stage ring needs two stages");
};

struct BwdItem {
  int blk, a, len;           // block; rows [a, a + len) of the (transposed) list
  int ib, ih;                // batch item and head of the views
  int n, nqb, nkb, tok0;     // the problem's tokens, query and key blocks, first token
  long long lbase;           // lse2 / delta index of the problem's first query row
};

// Work item idx (one per (batch*head, block) of `nblk` blocks) of a regular
// call, or of a variable-length batch (one per (item, head, block); items
// from the table, each its own problem of nqb_b = nkb_b blocks): everything
// but the list rows. Returns the list row (query-block row, or transposed
// key-block column) that the item's entries are at.
template <bool VARLEN>
__device__ __forceinline__ long long bwd_decode(int idx, bool by_key, const BwdParams &p,
                                                const VarlenTable &vt, BwdItem &it) {
  long long lrow;
  if (!VARLEN) {
    const int nblk = by_key ? p.nkb : p.nqb;
    const int bh = idx / nblk;
    it.blk = idx - bh * nblk;
    it.ib = bh / p.heads;
    it.ih = bh - it.ib * p.heads;
    it.n = p.n;
    it.nqb = p.nqb;
    it.nkb = p.nkb;
    it.tok0 = 0;
    it.lbase = static_cast<long long>(bh) * p.nqb * kBwdBlock;
    lrow = 0;
  } else {
    const int b = varlen_item_of_row(vt, idx / p.heads);
    const int nq = vt.row0[b + 1] - vt.row0[b];
    const int local = idx - p.heads * vt.row0[b];
    it.ih = local / nq;
    it.blk = local - it.ih * nq;
    it.ib = 0;
    it.tok0 = vt.tok0[b];
    it.n = vt.tok0[b + 1] - it.tok0;
    it.nqb = it.nkb = nq;
    // lse2 / delta: per item, per head, its padded rows
    it.lbase = (static_cast<long long>(p.heads) * vt.row0[b] + static_cast<long long>(it.ih) * nq) *
               kBwdBlock;
    lrow = static_cast<long long>(p.num_lists) * vt.row0[b];
  }
  const int list = p.num_lists > 1 ? it.ih : 0;
  return lrow + static_cast<long long>(list) * (by_key ? it.nkb : it.nqb) + it.blk;
}

// Warps 0-3: elementwise (thread = key row = TMEM lane) and the dK/dV
// epilogue; warp 4: TMA producer (lane 0); warp 5: MMA issuer (lane 0).
// Per query block e of the key block's column, the MMA issuer runs
//   S^T = K Q_e^T,  dP^T = V dO_e^T        (then the elementwise warps write
//                                           P^T and dS^T as bf16 over them)
//   dV += P^T dO_e, dK += dS^T Q_e         (issued before the next S^T, so the
//                                           TMEM they read is not overwritten)
template <int D, bool MASKED, bool VARLEN>
__global__ void __launch_bounds__(192, 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_do, const BwdParams p,
                         const __grid_constant__ VarlenTable vt) {
  using C = DkdvCfg<D>;
  constexpr int BN = kBwdBlock;
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t bar_st_full[C::NS], bar_st_empty[C::NS];
  __shared__ __align__(8) uint64_t bar_kv_full, bar_kv_empty, bar_s_full, bar_dp_full;
  __shared__ __align__(8) uint64_t bar_p_part[4], bar_ds_part[4];
  __shared__ __align__(8) uint64_t bar_acc_full, bar_acc_empty, bar_final;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  // work items from the global counter (natural order, served dynamically):
  // the producer takes them and hands them to the MMA issuer and the four
  // elementwise warps
  __shared__ int item_ring[kBwdItemN];
  __shared__ __align__(8) uint64_t bar_item_full[kBwdItemN], bar_item_empty[kBwdItemN];

  const uint32_t raw = smem_addr(dsmem);
  uint8_t *base = dsmem + (((raw + 1023u) & ~1023u) - raw);
  uint8_t *sK = base;
  uint8_t *sV = base + C::T;
  uint8_t *sStage = base + 2 * C::T;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&bar_st_full[s], 1);
      mbar_init(&bar_st_empty[s], 1);
    }
    mbar_init(&bar_kv_full, 1);
    mbar_init(&bar_kv_empty, 1);
    mbar_init(&bar_s_full, 1);
    mbar_init(&bar_dp_full, 1);
    for (int h = 0; h < 4; ++h) {
      mbar_init(&bar_p_part[h], 4);  // one arrival per elementwise warp
      mbar_init(&bar_ds_part[h], 4);
    }
    mbar_init(&bar_acc_full, 1);
    mbar_init(&bar_acc_empty, 4);
    mbar_init(&bar_final, 1);
    for (int i = 0; i < kBwdItemN; ++i) {
      mbar_init(&bar_item_full[i], 1);
      mbar_init(&bar_item_empty[i], 5);  // the MMA lane and one lane per elementwise warp
    }
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(&tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  WaitCtx wc{&abort_flag, p.wait_limit_ns, 0};

  // Item k of this CTA: (batch*head, key block) and its column of the
  // transposed lists.
  auto decode = [&](int idx) {
    BwdItem it;
    const long long c = bwd_decode<VARLEN>(idx, true, p, vt, it);
    const int a = min(max(p.col_ptr[c], 0), p.nnz), b = min(max(p.col_ptr[c + 1], 0), p.nnz);
    it.a = a;
    it.len = max(b - a, 0);
    return it;
  };

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      wc.role = kRoleProducer;
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      uint32_t ring = 0, kvcount = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int slot = k % kBwdItemN;
        if (!(ok = lane_wait(&bar_item_empty[slot], ((k / kBwdItemN) & 1) ^ 1, wc, kBarItem, k)))
          break;
        int idx = atomicAdd(p.item_counter, 1);
        if (idx >= p.total_items) idx = -1;
        item_ring[slot] = idx;
        mbar_arrive(&bar_item_full[slot]);
        if (idx < 0) break;
        const BwdItem it = decode(idx);
        if (it.len == 0) continue;
        if (!(ok = lane_wait(&bar_kv_empty, (kvcount & 1u) ^ 1u, wc, kBarQEmpty, kvcount))) break;
        mbar_arrive_expect_tx(&bar_kv_full, 2 * C::T);
        const int ib = it.ib, ih = it.ih;
        tma_load_5d(sK, &tm_k, &bar_kv_full, 0, it.tok0 + it.blk * BN, 0, ih, ib);
        tma_load_5d(sV, &tm_v, &bar_kv_full, 0, it.tok0 + it.blk * BN, 0, ih, ib);
        ++kvcount;
        for (int e = 0; e < it.len && ok; ++e) {
          const int qb = min(max(__ldg(p.row_idx + it.a + e), 0), it.nqb - 1);
          const uint32_t s = ring % C::NS;
          if (!(ok = lane_wait(&bar_st_empty[s], ((ring / C::NS) & 1u) ^ 1u, wc, kBarKvEmpty,
                               ring)))
            break;
          uint8_t *st = sStage + s * C::STAGE;
          mbar_arrive_expect_tx(&bar_st_full[s], 2 * C::T + 1024);
          tma_load_5d(st, &tm_q, &bar_st_full[s], 0, it.tok0 + qb * BN, 0, ih, ib);
          tma_load_5d(st + C::T, &tm_do, &bar_st_full[s], 0, it.tok0 + qb * BN, 0, ih, ib);
          const long long off = it.lbase + static_cast<long long>(qb) * BN;
          bulk_load(st + 2 * C::T, p.lse2 + off, 512, &bar_st_full[s]);
          bulk_load(st + 2 * C::T + 512, p.delta + off, 512, &bar_st_full[s]);
          ++ring;
        }
      }
      WaitCtx drain{&abort_flag, p.wait_limit_ns, kRoleProducer};
      int zero = 0;
      drain.abort = &zero;
      const uint32_t first = ring > C::NS ? ring - C::NS : 0;
      for (uint32_t r = first; r < ring; ++r)
        wait_bounded(&bar_st_full[r % C::NS], (r / C::NS) & 1u, drain, kBarKvFull, r);
      if (kvcount > 0) wait_bounded(&bar_kv_full, (kvcount - 1) & 1u, drain, kBarQFull, kvcount);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      wc.role = kRoleMma;
      constexpr uint32_t idesc_ss = idesc_bf16_f32(128, BN, false);
      constexpr uint32_t idesc_ts = idesc_bf16_f32(128, D, true);
      constexpr uint32_t kHi = (1024u >> 4) | (1u << 14) | (2u << 29);
      constexpr uint32_t kLboK = 1u << 16;
      constexpr uint32_t kLboMN = static_cast<uint32_t>(BN * 128 / 16) << 16;
      const uint32_t k_lo = (smem_addr(sK) >> 4) | kLboK;
      const uint32_t v_lo = (smem_addr(sV) >> 4) | kLboK;
      const uint32_t st_base = smem_addr(sStage) >> 4;
      uint32_t ring = 0, kvcount = 0, pcount = 0, items = 0;
      bool ok = true;
      // Schedule per query block e (stage s_e):
      //   S^T_e, dP^T_e                       (S^T_0, dP^T_0 before the loop)
      //   dV += P^T_e dO_e   part by part, as the elementwise warps hand
      //                      P^T over (p_part[0..3]); they compute P^T while
      //                      dP^T_e is still on the tensor pipe
      //   S^T_{e+1}          the S^T region is free once the dV MMAs that
      //                      read P^T_e are issued; it runs while the
      //                      elementwise warps compute dS^T_e
      //   dK += dS^T_e Q_e   part by part (ds_part[0..3])
      //   dP^T_{e+1}         after the dK MMAs that read dS^T_e
      auto issue_s = [&](uint32_t r) -> bool {  // S^T = K Q^T for ring slot r
        const uint32_t s = r % C::NS;
        if (!lane_wait(&bar_st_full[s], (r / C::NS) & 1u, wc, kBarKvFull, r)) return false;
        tc_fence_after();
        const uint32_t q_k = (st_base + s * (C::STAGE >> 4)) | kLboK;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (BN * 128 >> 4) + (kk & 3) * 2;
          mma_ss_lh(tmem + C::ST_COL, k_lo + off, kHi, q_k + off, kHi, idesc_ss, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bar_s_full);
        return true;
      };
      auto issue_dp = [&](uint32_t r) {  // dP^T = V dO^T (slot already waited)
        const uint32_t s = r % C::NS;
        const uint32_t do_k = (st_base + s * (C::STAGE >> 4) + (C::T >> 4)) | kLboK;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (BN * 128 >> 4) + (kk & 3) * 2;
          mma_ss_lh(tmem + C::DPT_COL, v_lo + off, kHi, do_k + off, kHi, idesc_ss,
                    kk > 0 ? 1u : 0u);
        }
        mma_commit(&bar_dp_full);
      };
      for (int k = 0; ok; ++k) {
        const int slot = k % kBwdItemN;
        if (!(ok = lane_wait(&bar_item_full[slot], (k / kBwdItemN) & 1, wc, kBarItem, k))) break;
        const int idx = *static_cast<volatile int *>(&item_ring[slot]);
        mbar_arrive(&bar_item_empty[slot]);
        if (idx < 0) break;
        const BwdItem it = decode(idx);
        if (it.len == 0) continue;
        if (!(ok = lane_wait(&bar_kv_full, kvcount & 1u, wc, kBarQFull, kvcount))) break;
        ++kvcount;
        tc_fence_after();
        if (!(ok = issue_s(ring))) break;
        issue_dp(ring);
        bool first = true;
        for (int e = 0; e < it.len; ++e) {
          const uint32_t s = ring % C::NS;
          const uint32_t q_mn = (st_base + s * (C::STAGE >> 4)) | kLboMN;
          const uint32_t do_mn = (st_base + s * (C::STAGE >> 4) + (C::T >> 4)) | kLboMN;
          if (first && items > 0) {  // the previous item's epilogue has read dV, dK
            if (!(ok = lane_wait(&bar_acc_empty, (items - 1) & 1u, wc, kBarOEmpty, items))) break;
            tc_fence_after();
          }
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            if (!(ok = lane_wait(&bar_p_part[h], pcount & 1u, wc, kBarPFull, pcount))) break;
            tc_fence_after();
#pragma unroll
            for (int kk = h * BN / 64; kk < (h + 1) * BN / 64; ++kk)
              mma_ts_lh(tmem + C::DV_COL, tmem + C::ST_COL + kk * 8,
                        do_mn + kk * (16 * 128 >> 4), kHi, idesc_ts,
                        (!first || kk > 0) ? 1u : 0u);
          }
          if (!ok) break;
          if (e + 1 < it.len && !(ok = issue_s(ring + 1))) break;
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            if (!(ok = lane_wait(&bar_ds_part[h], pcount & 1u, wc, kBarPFull, pcount))) break;
            tc_fence_after();
#pragma unroll
            for (int kk = h * BN / 64; kk < (h + 1) * BN / 64; ++kk)
              mma_ts_lh(tmem + C::DK_COL, tmem + C::DPT_COL + kk * 8,
                        q_mn + kk * (16 * 128 >> 4), kHi, idesc_ts,
                        (!first || kk > 0) ? 1u : 0u);
          }
          if (!ok) break;
          mma_commit(&bar_st_empty[s]);  // Q_e and dO_e read for the last time
          ++pcount;
          ++ring;
          first = false;
          if (e + 1 < it.len) issue_dp(ring);
        }
        if (!ok) break;
        mma_commit(&bar_kv_empty);  // K and V read for the last time
        mma_commit(&bar_acc_full);
        ++items;
      }
      mma_commit(&bar_final);
      WaitCtx drain{&abort_flag, p.wait_limit_ns, kRoleMma};
      int zero = 0;
      drain.abort = &zero;
      wait_bounded(&bar_final, 0, drain, kBarFinal, items);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ elementwise + epilogue
    wc.role = kRoleSoftmax;
    const int r = warp * 32 + lane;  // key row within the tile = TMEM lane
    const uint32_t lane_tmem = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float sl2 = p.scale_log2;
    uint32_t ring = 0, scount = 0, dcount = 0, acount = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int slot = k % kBwdItemN;
      if (!(ok = warp_wait(&bar_item_full[slot], (k / kBwdItemN) & 1, wc, kBarItem, k))) break;
      const int idx = *static_cast<volatile int *>(&item_ring[slot]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_item_empty[slot]);
      if (idx < 0) break;
      const BwdItem it = decode(idx);
      const int key = it.blk * BN + r;
      const bool store = key < it.n;
      const long long ib = it.ib, ih = it.ih, tk = it.tok0 + key;
      __nv_bfloat16 *const dk_row = p.dk + ib * p.dk_s[0] + ih * p.dk_s[1] + tk * p.dk_s[2];
      __nv_bfloat16 *const dv_row = p.dv + ib * p.dv_s[0] + ih * p.dv_s[1] + tk * p.dv_s[2];
      if (it.len == 0) {  // no query attends these keys
        if (store) {
          uint4 *a = reinterpret_cast<uint4 *>(dk_row);
          uint4 *b = reinterpret_cast<uint4 *>(dv_row);
#pragma unroll
          for (int c = 0; c < D / 8; ++c) {
            a[c] = make_uint4(0, 0, 0, 0);
            b[c] = make_uint4(0, 0, 0, 0);
          }
        }
        continue;
      }
      for (int e = 0; e < it.len; ++e) {
        const uint32_t s = ring % C::NS, spar = (ring / C::NS) & 1u;
        ++ring;
        if (!(ok = warp_wait(&bar_s_full, scount & 1u, wc, kBarSFull, scount))) break;
        // the stage's lse2 / delta rows came by TMA: acquire them from the
        // stage barrier itself (complete long before S^T is; the stage is
        // not released before this warp's dS^T arrives)
        if (!(ok = warp_wait(&bar_st_full[s], spar, wc, kBarKvFull, ring))) break;
        tc_fence_after();
        const float *lse_s = reinterpret_cast<const float *>(sStage + s * C::STAGE + 2 * C::T);
        const float *del_s = lse_s + 128;
        // listed (query half, key half) pairs of this tile pair; this thread's
        // key half is warp / 2, chunk c's query half c / 2
        const uint32_t bits = MASKED ? __ldg(p.cmask + it.a + e) : 0xFu;
        // P^T (fp32, kept for dS^T), handed over as bf16 in four parts while
        // dP^T is still being computed
        float pf[BN];
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t sr[32];
          tmem_ld32(lane_tmem + C::ST_COL + c * 32, sr);
          tmem_wait_ld();
          reg_fence32(sr);
          const bool on = !MASKED || ((bits >> ((c >> 1) * 2 + (warp >> 1))) & 1u);
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float4 l4 = *reinterpret_cast<const float4 *>(lse_s + c * 32 + (i & ~1) * 2);
            const float la = (i & 1) ? l4.z : l4.x, lb = (i & 1) ? l4.w : l4.y;
            const float pa = ex2_approx(fmaf(__uint_as_float(sr[2 * i]), sl2, -la));
            const float pb = ex2_approx(fmaf(__uint_as_float(sr[2 * i + 1]), sl2, -lb));
            pf[c * 32 + 2 * i] = on ? pa : 0.f;
            pf[c * 32 + 2 * i + 1] = on ? pb : 0.f;
            pk[i] = pack_bf16x2(pf[c * 32 + 2 * i], pf[c * 32 + 2 * i + 1]);
          }
          // chunk c lands on columns [16c, 16c + 16): already read back
          tmem_st16(lane_tmem + C::ST_COL + c * 16, pk);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar_p_part[c]);
        }
        ++scount;
        if (!(ok = warp_wait(&bar_dp_full, dcount & 1u, wc, kBarSFull, dcount))) break;
        ++dcount;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t dr[32];
          tmem_ld32(lane_tmem + C::DPT_COL + c * 32, dr);
          tmem_wait_ld();
          reg_fence32(dr);
          uint32_t g16[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float4 d4 = *reinterpret_cast<const float4 *>(del_s + c * 32 + (i & ~1) * 2);
            const float da = (i & 1) ? d4.z : d4.x, db = (i & 1) ? d4.w : d4.y;
            g16[i] = pack_bf16x2(pf[c * 32 + 2 * i] * (__uint_as_float(dr[2 * i]) - da),
                                 pf[c * 32 + 2 * i + 1] * (__uint_as_float(dr[2 * i + 1]) - db));
          }
          tmem_st16(lane_tmem + C::DPT_COL + c * 16, g16);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar_ds_part[c]);
        }
      }
      if (!ok) break;
      // epilogue: dV and dK (times scale) of this key row
      if (!(ok = warp_wait(&bar_acc_full, acount & 1u, wc, kBarODone, acount))) break;
      ++acount;
      tc_fence_after();
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        const uint32_t col = part == 0 ? C::DV_COL : C::DK_COL;
        const float mul = part == 0 ? 1.f : p.scale;
        __nv_bfloat16 *dst = part == 0 ? dv_row : dk_row;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(lane_tmem + col + c * 32, v);
          tmem_wait_ld();
          reg_fence32(v);
          if (store) {
            uint4 *o4 = reinterpret_cast<uint4 *>(dst + c * 32);
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              uint4 x;
              x.x = pack_bf16x2(__uint_as_float(v[8 * w + 0]) * mul, __uint_as_float(v[8 * w + 1]) * mul);
              x.y = pack_bf16x2(__uint_as_float(v[8 * w + 2]) * mul, __uint_as_float(v[8 * w + 3]) * mul);
              x.z = pack_bf16x2(__uint_as_float(v[8 * w + 4]) * mul, __uint_as_float(v[8 * w + 5]) * mul);
              x.w = pack_bf16x2(__uint_as_float(v[8 * w + 6]) * mul, __uint_as_float(v[8 * w + 7]) * mul);
              o4[w] = x;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_acc_empty);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ dQ --

template <int D>
struct DqCfg {
  static constexpr int T = kBwdBlock * D * 2;
  static constexpr int STAGE = 2 * T;                // K and V of a key block
  static constexpr int NS_FIT = (kSmemLimit - 1024 - 1024 - 2 * T) / STAGE;
  static constexpr int NS = NS_FIT > 4 ? 4 : NS_FIT;
  static constexpr int DSMEM = 1024 + 2 * T + NS * STAGE;
  static constexpr uint32_t S_COL = 0;               // S of even steps
  static constexpr uint32_t DP_COL = 128;            // dP, then dS (bf16) over its first 64
  static constexpr uint32_t DQ_COL = 256;
  static constexpr uint32_t S1_COL = 256 + D;        // S of odd steps
  static constexpr int THREADS = 192;
  static_assert(NS >= 2, "stage ring needs two stages");
  static_assert(S1_COL + 128 <= 512, "TMEM columns");
  __host__ __device__ static constexpr uint32_t s_col(int e) { return (e & 1) ? S1_COL : S_COL; }
};

// Warps 0-3: elementwise (thread = query row = TMEM lane) and the dQ
// epilogue; warp 4: TMA producer (lane 0); warp 5: MMA issuer (lane 0).
// Per key block e of the row: S_e = Q K_e^T (double-buffered, issued one
// block ahead so it runs during the previous elementwise step), dP = dO V_e^T,
// the elementwise warps write dS (bf16) over dP, then dQ += dS K_e (issued
// before the next dP, which overwrites the dS it reads).
template <int D, bool MASKED, bool VARLEN>
__global__ void __launch_bounds__(192, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_do, const BwdParams p,
                       const __grid_constant__ VarlenTable vt) {
  using C = DqCfg<D>;
  constexpr int BN = kBwdBlock;
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t bar_st_full[C::NS], bar_st_empty[C::NS];
  // one S-ready barrier per S buffer: with S issued a block ahead, a single
  // barrier could complete two phases before the elementwise warps wait for
  // the first (at an item's start), and a parity wait cannot tell them apart
  __shared__ __align__(8) uint64_t bar_qd_full, bar_qd_empty, bar_s_full[2], bar_dp_full;
  __shared__ __align__(8) uint64_t bar_ds_part[4];
  __shared__ __align__(8) uint64_t bar_acc_full, bar_acc_empty, bar_final;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  // work items from the global counter (natural order, served dynamically):
  // the producer takes them and hands them to the MMA issuer and the four
  // elementwise warps
  __shared__ int item_ring[kBwdItemN];
  __shared__ __align__(8) uint64_t bar_item_full[kBwdItemN], bar_item_empty[kBwdItemN];

  const uint32_t raw = smem_addr(dsmem);
  uint8_t *base = dsmem + (((raw + 1023u) & ~1023u) - raw);
  uint8_t *sQ = base;
  uint8_t *sDO = base + C::T;
  uint8_t *sStage = base + 2 * C::T;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&bar_st_full[s], 1);
      mbar_init(&bar_st_empty[s], 1);
    }
    mbar_init(&bar_qd_full, 1);
    mbar_init(&bar_qd_empty, 1);
    mbar_init(&bar_s_full[0], 1);
    mbar_init(&bar_s_full[1], 1);
    mbar_init(&bar_dp_full, 1);
    for (int h = 0; h < 4; ++h) mbar_init(&bar_ds_part[h], 4);
    mbar_init(&bar_acc_full, 1);
    mbar_init(&bar_acc_empty, 4);
    mbar_init(&bar_final, 1);
    for (int i = 0; i < kBwdItemN; ++i) {
      mbar_init(&bar_item_full[i], 1);
      mbar_init(&bar_item_empty[i], 5);  // the MMA lane and one lane per elementwise warp
    }
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(&tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  WaitCtx wc{&abort_flag, p.wait_limit_ns, 0};

  auto decode = [&](int idx) {
    BwdItem it;
    const long long r = bwd_decode<VARLEN>(idx, false, p, vt, it);
    const int a = min(max(p.row_ptr[r], 0), p.nnz), b = min(max(p.row_ptr[r + 1], 0), p.nnz);
    it.a = a;
    it.len = max(b - a, 0);
    return it;
  };

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      wc.role = kRoleProducer;
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      uint32_t ring = 0, qdcount = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int slot = k % kBwdItemN;
        if (!(ok = lane_wait(&bar_item_empty[slot], ((k / kBwdItemN) & 1) ^ 1, wc, kBarItem, k)))
          break;
        int idx = atomicAdd(p.item_counter, 1);
        if (idx >= p.total_items) idx = -1;
        item_ring[slot] = idx;
        mbar_arrive(&bar_item_full[slot]);
        if (idx < 0) break;
        const BwdItem it = decode(idx);
        if (it.len == 0) continue;
        if (!(ok = lane_wait(&bar_qd_empty, (qdcount & 1u) ^ 1u, wc, kBarQEmpty, qdcount))) break;
        mbar_arrive_expect_tx(&bar_qd_full, 2 * C::T);
        const int ib = it.ib, ih = it.ih;
        tma_load_5d(sQ, &tm_q, &bar_qd_full, 0, it.tok0 + it.blk * BN, 0, ih, ib);
        tma_load_5d(sDO, &tm_do, &bar_qd_full, 0, it.tok0 + it.blk * BN, 0, ih, ib);
        ++qdcount;
        for (int e = 0; e < it.len && ok; ++e) {
          const int kb = min(max(__ldg(p.col_idx + it.a + e), 0), it.nkb - 1);
          const uint32_t s = ring % C::NS;
          if (!(ok = lane_wait(&bar_st_empty[s], ((ring / C::NS) & 1u) ^ 1u, wc, kBarKvEmpty,
                               ring)))
            break;
          uint8_t *st = sStage + s * C::STAGE;
          mbar_arrive_expect_tx(&bar_st_full[s], 2 * C::T);
          tma_load_5d(st, &tm_k, &bar_st_full[s], 0, it.tok0 + kb * BN, 0, ih, ib);
          tma_load_5d(st + C::T, &tm_v, &bar_st_full[s], 0, it.tok0 + kb * BN, 0, ih, ib);
          ++ring;
        }
      }
      WaitCtx drain{&abort_flag, p.wait_limit_ns, kRoleProducer};
      int zero = 0;
      drain.abort = &zero;
      const uint32_t first = ring > C::NS ? ring - C::NS : 0;
      for (uint32_t r = first; r < ring; ++r)
        wait_bounded(&bar_st_full[r % C::NS], (r / C::NS) & 1u, drain, kBarKvFull, r);
      if (qdcount > 0) wait_bounded(&bar_qd_full, (qdcount - 1) & 1u, drain, kBarQFull, qdcount);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      wc.role = kRoleMma;
      constexpr uint32_t idesc_ss = idesc_bf16_f32(128, BN, false);
      constexpr uint32_t idesc_ts = idesc_bf16_f32(128, D, true);
      constexpr uint32_t kHi = (1024u >> 4) | (1u << 14) | (2u << 29);
      constexpr uint32_t kLboK = 1u << 16;
      constexpr uint32_t kLboMN = static_cast<uint32_t>(BN * 128 / 16) << 16;
      const uint32_t q_lo = (smem_addr(sQ) >> 4) | kLboK;
      const uint32_t do_lo = (smem_addr(sDO) >> 4) | kLboK;
      const uint32_t st_base = smem_addr(sStage) >> 4;
      uint32_t ring = 0, qdcount = 0, pcount = 0, items = 0;
      bool ok = true;
      // Schedule per key block e (stage s_e):
      //   S_{e+1}           into the other S buffer (its previous user, the
      //                     elementwise step of block e-1, is done): runs
      //                     while block e's elementwise step works
      //   dQ += dS_e K_e    part by part, as the elementwise warps hand dS
      //                     over (ds_part[0..3]); they compute P_e from S_e
      //                     while dP_e is still on the tensor pipe
      //   dP_{e+1}          after the dQ MMAs that read dS_e from its region
      // (S_0 and dP_0 before the loop.)
      auto issue_s = [&](int e, uint32_t r) -> bool {  // S_e = Q K_e^T
        const uint32_t s = r % C::NS;
        if (!lane_wait(&bar_st_full[s], (r / C::NS) & 1u, wc, kBarKvFull, r)) return false;
        tc_fence_after();
        const uint32_t k_k = (st_base + s * (C::STAGE >> 4)) | kLboK;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (BN * 128 >> 4) + (kk & 3) * 2;
          mma_ss_lh(tmem + C::s_col(e), q_lo + off, kHi, k_k + off, kHi, idesc_ss,
                    kk > 0 ? 1u : 0u);
        }
        mma_commit(&bar_s_full[e & 1]);
        return true;
      };
      auto issue_dp = [&](uint32_t r) {  // dP = dO V^T (slot already waited)
        const uint32_t s = r % C::NS;
        const uint32_t v_k = (st_base + s * (C::STAGE >> 4) + (C::T >> 4)) | kLboK;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (BN * 128 >> 4) + (kk & 3) * 2;
          mma_ss_lh(tmem + C::DP_COL, do_lo + off, kHi, v_k + off, kHi, idesc_ss,
                    kk > 0 ? 1u : 0u);
        }
        mma_commit(&bar_dp_full);
      };
      for (int k = 0; ok; ++k) {
        const int slot = k % kBwdItemN;
        if (!(ok = lane_wait(&bar_item_full[slot], (k / kBwdItemN) & 1, wc, kBarItem, k))) break;
        const int idx = *static_cast<volatile int *>(&item_ring[slot]);
        mbar_arrive(&bar_item_empty[slot]);
        if (idx < 0) break;
        const BwdItem it = decode(idx);
        if (it.len == 0) continue;
        if (!(ok = lane_wait(&bar_qd_full, qdcount & 1u, wc, kBarQFull, qdcount))) break;
        ++qdcount;
        tc_fence_after();
        if (!(ok = issue_s(0, ring))) break;
        issue_dp(ring);
        bool first = true;
        for (int e = 0; e < it.len; ++e) {
          const uint32_t s = ring % C::NS;
          if (e + 1 < it.len && !(ok = issue_s(e + 1, ring + 1))) break;
          if (first && items > 0) {  // the previous item's epilogue has read dQ
            if (!(ok = lane_wait(&bar_acc_empty, (items - 1) & 1u, wc, kBarOEmpty, items))) break;
            tc_fence_after();
          }
          const uint32_t k_mn = (st_base + s * (C::STAGE >> 4)) | kLboMN;
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            if (!(ok = lane_wait(&bar_ds_part[h], pcount & 1u, wc, kBarPFull, pcount))) break;
            tc_fence_after();
#pragma unroll
            for (int kk = h * BN / 64; kk < (h + 1) * BN / 64; ++kk)
              mma_ts_lh(tmem + C::DQ_COL, tmem + C::DP_COL + kk * 8,
                        k_mn + kk * (16 * 128 >> 4), kHi, idesc_ts,
                        (!first || kk > 0) ? 1u : 0u);
          }
          if (!ok) break;
          mma_commit(&bar_st_empty[s]);  // K_e and V_e read for the last time
          ++pcount;
          ++ring;
          first = false;
          if (e + 1 < it.len) issue_dp(ring);
        }
        if (!ok) break;
        mma_commit(&bar_qd_empty);  // Q and dO read for the last time
        mma_commit(&bar_acc_full);
        ++items;
      }
      mma_commit(&bar_final);
      WaitCtx drain{&abort_flag, p.wait_limit_ns, kRoleMma};
      int zero = 0;
      drain.abort = &zero;
      wait_bounded(&bar_final, 0, drain, kBarFinal, items);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ elementwise + epilogue
    wc.role = kRoleSoftmax;
    const int r = warp * 32 + lane;  // query row within the tile = TMEM lane
    const uint32_t lane_tmem = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float sl2 = p.scale_log2;
    uint32_t scount[2] = {0u, 0u}, dcount = 0, acount = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int slot = k % kBwdItemN;
      if (!(ok = warp_wait(&bar_item_full[slot], (k / kBwdItemN) & 1, wc, kBarItem, k))) break;
      const int idx = *static_cast<volatile int *>(&item_ring[slot]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_item_empty[slot]);
      if (idx < 0) break;
      const BwdItem it = decode(idx);
      const int row = it.blk * BN + r;
      const bool store = row < it.n;
      const long long ib = it.ib, ih = it.ih, tq = it.tok0 + row;
      __nv_bfloat16 *const dq_row = p.dq + ib * p.dq_s[0] + ih * p.dq_s[1] + tq * p.dq_s[2];
      if (it.len == 0) {  // no key: dQ = 0
        if (store) {
          uint4 *a = reinterpret_cast<uint4 *>(dq_row);
#pragma unroll
          for (int c = 0; c < D / 8; ++c) a[c] = make_uint4(0, 0, 0, 0);
        }
        continue;
      }
      const long long prow = it.lbase + static_cast<long long>(it.blk) * BN + r;
      const float lse2 = p.lse2[prow], del = p.delta[prow];
      // lists are sorted: only the row's last block can be the ragged final
      // key block (its columns >= n hold zero keys, or the next item's keys
      // in a variable-length batch; they are masked out)
      const int last_kb = min(max(__ldg(p.col_idx + it.a + it.len - 1), 0), it.nkb - 1);
      const int last_valid = min(it.n - last_kb * BN, BN);
      for (int e = 0; e < it.len; ++e) {
        const int sb = e & 1;
        if (!(ok = warp_wait(&bar_s_full[sb], scount[sb] & 1u, wc, kBarSFull, scount[sb]))) break;
        ++scount[sb];
        tc_fence_after();
        const int valid = e == it.len - 1 ? last_valid : BN;
        // listed (query half, key half) pairs of this tile pair; this thread's
        // query half is warp / 2, chunk c's key half c / 2
        const uint32_t bits = MASKED ? __ldg(p.rmask + it.a + e) : 0xFu;
        // P from S (fp32, kept for dS) while dP is still being computed
        float pf[BN];
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t sr[32];
          tmem_ld32(lane_tmem + C::s_col(e) + c * 32, sr);
          tmem_wait_ld();
          reg_fence32(sr);
          const bool on = !MASKED || ((bits >> ((warp >> 1) * 2 + (c >> 1))) & 1u);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float pv = ex2_approx(fmaf(__uint_as_float(sr[i]), sl2, -lse2));
            pf[c * 32 + i] = (!on || (valid < BN && c * 32 + i >= valid)) ? 0.f : pv;
          }
        }
        if (!(ok = warp_wait(&bar_dp_full, dcount & 1u, wc, kBarSFull, dcount))) break;
        ++dcount;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t dr[32];
          tmem_ld32(lane_tmem + C::DP_COL + c * 32, dr);
          tmem_wait_ld();
          reg_fence32(dr);
          uint32_t g16[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            g16[i] = pack_bf16x2(pf[c * 32 + 2 * i] * (__uint_as_float(dr[2 * i]) - del),
                                 pf[c * 32 + 2 * i + 1] * (__uint_as_float(dr[2 * i + 1]) - del));
          // chunk c lands on dP columns [16c, 16c + 16): already read back
          tmem_st16(lane_tmem + C::DP_COL + c * 16, g16);
          tmem_wait_st();  // part c of the key columns handed over
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar_ds_part[c]);
        }
      }
      if (!ok) break;
      if (!(ok = warp_wait(&bar_acc_full, acount & 1u, wc, kBarODone, acount))) break;
      ++acount;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(lane_tmem + C::DQ_COL + c * 32, v);
        tmem_wait_ld();
        reg_fence32(v);
        if (store) {
          const float mul = p.scale;
          uint4 *o4 = reinterpret_cast<uint4 *>(dq_row + c * 32);
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            uint4 x;
            x.x = pack_bf16x2(__uint_as_float(v[8 * w + 0]) * mul, __uint_as_float(v[8 * w + 1]) * mul);
            x.y = pack_bf16x2(__uint_as_float(v[8 * w + 2]) * mul, __uint_as_float(v[8 * w + 3]) * mul);
            x.z = pack_bf16x2(__uint_as_float(v[8 * w + 4]) * mul, __uint_as_float(v[8 * w + 5]) * mul);
            x.w = pack_bf16x2(__uint_as_float(v[8 * w + 6]) * mul, __uint_as_float(v[8 * w + 7]) * mul);
            o4[w] = x;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_acc_empty);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace bsa
