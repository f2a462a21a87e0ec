// Block-sparse softmax attention forward for sm_100a: TMA-staged tiles,
// tcgen05 MMAs accumulating in tensor memory, exp2 online softmax.
//
// One CTA per SM (persistent). Work items are (batch*head, query block); the
// host-side prepass orders each list's query blocks longest row first and the
// CTAs walk that order head-major in a static snake, so concurrently running
// CTAs share the K/V of one or two heads in L2 and the cheapest rows finish
// the job.
//
// Warp roles (192 threads):
//   warps 0-3  softmax: thread t owns query row t of the 128-row tile
//              (TMEM lane t); exp2 online softmax, P written back to TMEM as
//              bf16, O rescaled in TMEM when the running max jumps, epilogue.
//   warp 4     producer (one thread): TMA loads of Q and of the listed K and
//              V tiles through an NS-stage ring, in the order the MMA warp
//              consumes them.
//   warp 5     MMA issuer (one thread): S = Q K^T into one of two TMEM S
//              buffers, then O += P V with P read from TMEM.
//
// TMEM columns (512 allocated): S0 [0,128), S1 [128,256), O [256, 256+D),
// Q [384, 384+D/2) (copied from shared memory once per item).
// Per block g (global counter) the MMA warp issues QK(g+1) before PV(g), so
// the tensor core computes the next scores while the softmax warps work.
//
// Every wait is bounded (globaltimer). On expiry the thread records
// BSA_ERR_DEVICE_TIMEOUT, raises a CTA-wide abort flag, and all roles leave
// their loops; the producer waits (bounded) for its copies in flight, the MMA
// thread waits for its MMAs, and TMEM is freed before the CTA exits.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "bsa.h"
#include "device_status.cuh"
#include "lists.cuh"
#include "ptx_sm100.cuh"

namespace bsa {

// Variable-length batches: the batch is one packed token sequence (batch
// extent 1 in the views) holding num_items items one after the other; item b
// owns tokens [tok0[b], tok0[b+1]), query-block rows [row0[b], row0[b+1]) of
// every list (its key blocks counted from 0 inside the item), work-order
// entries [pair0[b], pair0[b+1]) of every list and work items
// [work0[b], work0[b+1]) (heads x its query-block pairs; the backward
// derives its own work items from row0). Passed by value as a kernel
// parameter.
constexpr int kMaxVarlenItems = 64;
struct VarlenTable {
  int32_t num_items;
  int32_t tok0[kMaxVarlenItems + 1];
  int32_t row0[kMaxVarlenItems + 1];
  int32_t pair0[kMaxVarlenItems + 1];
  int32_t work0[kMaxVarlenItems + 1];
};

// The item holding query-block row r of a variable-length batch: the last b
// with row0[b] <= r (an item without rows shares its row0 with the next item
// and is skipped).
__device__ __forceinline__ int varlen_item_of_row(const VarlenTable &vt, int r) {
  int lo = 0, hi = vt.num_items - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (vt.row0[mid] <= r)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

struct FwdParams {
  const int32_t *row_ptr, *col_idx, *order;
  int32_t *item_counter;  // next work item (two-tile kernel); zeroed by the work-order kernel
  __nv_bfloat16 *out;
  // element strides of out's batch, head and token axes (head_dim contiguous)
  long long o_sb, o_sh, o_sn;
  float *lse;
  int32_t heads, n, nqb, nkb, num_lists, nnz;
  int32_t total_items;
  float scale_log2;  // softmax_scale * log2(e)
  unsigned long long wait_limit_ns;
  int32_t fault_flags;
  // Rows generated in the kernel instead of read from col_idx (two-tile
  // kernel): per-list tile patterns (list of head h = head_list[h] when given)
  // or the radial geometry shared by every head.
  const bsa_tile_pattern *patterns = nullptr;
  const int32_t *pattern_columns = nullptr;
  long long num_pattern_columns = 0;
  const int32_t *head_list = nullptr;
  RadialGeom radial = {};
  // Block-64 lists packed as 128-row tiles (two-tile kernel): per tile-list
  // entry, bit qi * 2 + kj set when query half qi lists key half kj.
  const uint8_t *tile_mask = nullptr;
};

constexpr int kSmemLimit = 232448;  // 227 KB dynamic + static per CTA on sm_100

template <int D, int BN>
struct FwdCfg {
  static constexpr int BM = 128;                 // tile rows (MMA M)
  static constexpr int NCB = D / 64;             // 128-byte column blocks per row
  static constexpr int Q_BYTES = BM * D * 2;
  // A ring stage holds two consecutive key blocks of K (or of V), loaded by
  // one TMA box of 2*BN rows: the TMA unit's cost is mostly per box, and
  // radial lists are made of runs of consecutive blocks. A lone block still
  // takes a whole stage (its second half is simply not used). Layout: D/64
  // column blocks of [2*BN rows][128 B], block h of the pair at h*BN rows.
  static constexpr int SEG = 2;                  // key blocks per stage
  static constexpr int STAGE_ROWS = SEG * BN;
  static constexpr int CB_BYTES = STAGE_ROWS * 128;  // one 64-column block of a stage
  static constexpr int STAGE_BYTES = STAGE_ROWS * D * 2;
  static constexpr int NS_FIT = (kSmemLimit - 1024 - 512 - Q_BYTES) / STAGE_BYTES;
  static constexpr int NS = NS_FIT > 8 ? 8 : NS_FIT;
  // At least 120 KB so that a second CTA never fits on an SM: every CTA then
  // owns its SM's tensor memory and the persistent grid covers all SMs.
  static constexpr int DSMEM_USED = 1024 + Q_BYTES + NS * STAGE_BYTES;
  static constexpr int DSMEM = DSMEM_USED > 122880 ? DSMEM_USED : 122880;
  static constexpr uint32_t S_COL = 0;           // S buffer b at S_COL + 128 b
  static constexpr uint32_t O_COL = 256;
  static constexpr uint32_t P_COL = 384;         // P buffer b at P_COL + 64 b (bf16 pairs)
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int THREADS = 192;
  static_assert(NS >= 2, "K/V ring needs at least two stages");
  static_assert(D == 64 || D == 128, "head_dim");
  static_assert(BN == 64 || BN == 128, "block");
};

enum : int { kRoleProducer = 1, kRoleMma = 2, kRoleSoftmax = 3 };
enum : int {
  kBarKvFull = 1, kBarKvEmpty, kBarQFull, kBarQEmpty, kBarSFull, kBarPFull, kBarODone,
  kBarOEmpty, kBarFinal, kBarSFree, kBarPlan, kBarItem
};

struct WaitCtx {
  volatile int *abort;
  unsigned long long limit;
  int role;
};

// Bounded parity wait. Returns false when the CTA is aborting or the limit ran
// out (the first thread to run out records the timeout and raises the flag).
__device__ __forceinline__ bool wait_bounded(uint64_t *bar, uint32_t parity, const WaitCtx &w,
                                          int bar_id, uint32_t counter) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*w.abort) return false;
    if (global_timer_ns() - t0 > w.limit) {
      if (atomicCAS(&g_status, 0u, 4u /* BSA_ERR_DEVICE_TIMEOUT */) == 0u) {
        g_status_detail[0] = w.role;
        g_status_detail[1] = bar_id;
        g_status_detail[2] = counter;
        g_status_detail[3] = blockIdx.x;
      }
      *w.abort = 1;
      return false;
    }
  }
}

// Whole-warp wait: a fast inline test, the bounded slow path only on a miss,
// and a warp vote so every lane takes the same branch afterwards.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, const WaitCtx &w,
                                          int bar_id, uint32_t counter) {
  bool r = mbar_try_wait(bar, parity);
  if (!r) r = wait_bounded(bar, parity, w, bar_id, counter);
  return __all_sync(0xffffffffu, r);
}

// Single-thread wait, for the roles that run on one lane (no warp vote).
__device__ __forceinline__ bool lane_wait(uint64_t *bar, uint32_t parity, const WaitCtx &w,
                                          int bar_id, uint32_t counter) {
  return mbar_try_wait(bar, parity) || wait_bounded(bar, parity, w, bar_id, counter);
}

// Work item k of this CTA (static snake over the ordered item list); -1 when
// the CTA has no item k.
__device__ __forceinline__ int snake_item(int k, int total) {
  const int G = gridDim.x;
  const long long base = static_cast<long long>(k) * G;
  if (base >= total) return -2;  // past the end for every CTA
  const int idx = static_cast<int>(base) + ((k & 1) ? (G - 1 - static_cast<int>(blockIdx.x))
                                                    : static_cast<int>(blockIdx.x));
  return idx < total ? idx : -1;
}

struct Item {
  int bh, qb, a, len;
};

__device__ __forceinline__ Item decode_item(int idx, const FwdParams &p) {
  Item it;
  it.bh = idx / p.nqb;
  const int rank = idx - it.bh * p.nqb;
  const int list = p.num_lists > 1 ? (it.bh % p.heads) : 0;
  const long long lbase = static_cast<long long>(list) * p.nqb;
  it.qb = min(max(p.order[lbase + rank], 0), p.nqb - 1);
  const int a = min(max(p.row_ptr[lbase + it.qb], 0), p.nnz);
  const int e = min(max(p.row_ptr[lbase + it.qb + 1], 0), p.nnz);
  it.a = a;
  it.len = max(e - a, 0);
  return it;
}

__device__ __forceinline__ int key_block(const FwdParams &p, int e) {
  return min(max(p.col_idx[e], 0), p.nkb - 1);
}

// A warp's register cache of one row's key blocks: lane i holds entry
// base + i, and the next 32 entries are already in flight, so reading the
// list costs a shuffle instead of a dependent global load on the critical
// path. Lookups must be warp-uniform and non-decreasing in b.
struct ListCache {
  int base, cur, nxt;
  __device__ __forceinline__ static int load(const FwdParams &p, int a, int len, int chunk) {
    const int i = chunk + static_cast<int>(threadIdx.x & 31);
    return i < len ? min(max(__ldg(p.col_idx + a + i), 0), p.nkb - 1) : 0;
  }
  __device__ __forceinline__ void reset(const FwdParams &p, int a, int len) {
    base = 0;
    cur = load(p, a, len, 0);
    nxt = load(p, a, len, 32);
  }
  __device__ __forceinline__ int get(const FwdParams &p, int a, int len, int b) {
    while (b >= base + 32) {
      base += 32;
      cur = nxt;
      nxt = load(p, a, len, base + 32);
    }
    return __shfl_sync(0xffffffffu, cur, b - base);
  }
};

// Walks a row's key blocks as segments of one or two consecutive blocks (the
// unit one ring stage holds). The producer and the MMA warp run identical
// walkers, so they agree on which ring position holds which block.
struct SegWalker {
  int first = 0, count = 0, kb = 0;
  ListCache cache;
  __device__ __forceinline__ void reset(const FwdParams &p, int a, int len) {
    first = 0;
    count = 0;
    cache.reset(p, a, len);
  }
  // True when block b opens a new segment (b is past the current one).
  __device__ __forceinline__ bool advance(const FwdParams &p, int a, int len, int b) {
    if (b < first + count) return false;
    first = b;
    kb = cache.get(p, a, len, b);
    const int next = b + 1 < len ? cache.get(p, a, len, b + 1) : -1;
    count = next == kb + 1 ? 2 : 1;
    return true;
  }
};

#ifndef BSA_EMU_PAIRS
#define BSA_EMU_PAIRS 0
#endif
// Of every 8 column pairs, this many take 2^x on the FMA pipe (exp2_poly2)
// and the rest on the MUFU unit, so the two units share the softmax's
// exponentials.
constexpr int kEmuPairsPer8 = BSA_EMU_PAIRS;

// p = 2^(s * sl2 + neg) for one row of BN scores: returns the fp32 row sum and
// the values packed as bf16 pairs. EMU of every 8 pairs use the polynomial.
// Column pairs [C0, C1) of the row into the four partial sums acc (pair c
// into acc[c % 4]); a whole row is [0, BN / 2) and then exp2_row_sum.
template <int BN, int EMU, int C0, int C1>
__device__ __forceinline__ void exp2_pack_pairs(const float (&s)[BN], float sl2, float neg,
                                                uint32_t (&pk)[BN / 2], float2 (&acc)[4]) {
  const float2 neg2 = make_float2(neg, neg);
  const float2 sl2v = make_float2(sl2, sl2);
#pragma unroll
  for (int c = C0; c < C1; ++c) {
    const float2 x = ffma2(make_float2(s[2 * c], s[2 * c + 1]), sl2v, neg2);
    float2 pp;
    if ((c & 7) < EMU) {
      pp = exp2_poly2(x);
    } else {
      pp = make_float2(ex2_approx(x.x), ex2_approx(x.y));
    }
    acc[c & 3] = fadd2(acc[c & 3], pp);
    pk[c] = pack_bf16x2(pp.x, pp.y);
  }
}

__device__ __forceinline__ float exp2_row_sum(const float2 (&acc)[4]) {
  const float2 a = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
  return a.x + a.y;
}

template <int BN, int EMU>
__device__ __forceinline__ float exp2_pack_row(const float (&s)[BN], float sl2, float neg,
                                               uint32_t (&pk)[BN / 2]) {
  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                   make_float2(0.f, 0.f)};
  exp2_pack_pairs<BN, EMU, 0, BN / 2>(s, sl2, neg, pk, acc);
  return exp2_row_sum(acc);
}

template <int D, int BN>
__global__ void __launch_bounds__(192, 1)
    attn_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = FwdCfg<D, BN>;
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t bar_kv_full[C::NS];
  __shared__ __align__(8) uint64_t bar_kv_empty[C::NS];
  __shared__ __align__(8) uint64_t bar_q_full, bar_q_empty, bar_o_empty, bar_final;
  __shared__ __align__(8) uint64_t bar_o_done[2];
  __shared__ __align__(8) uint64_t bar_s_full[2], bar_s_free[2], bar_p_full[2];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const uint32_t raw = smem_addr(dsmem);
  uint8_t *base = dsmem + (((raw + 1023u) & ~1023u) - raw);
  uint8_t *sQ = base;
  uint8_t *sKV = base + C::Q_BYTES;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&bar_kv_full[s], 1);
      mbar_init(&bar_kv_empty[s], 1);
    }
    mbar_init(&bar_q_full, 1);
    mbar_init(&bar_q_empty, 1);
    mbar_init(&bar_o_empty, 4);  // one arrival per softmax warp
    mbar_init(&bar_final, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar_s_full[b], 1);
      mbar_init(&bar_s_free[b], 4);
      mbar_init(&bar_o_done[b], 1);
      mbar_init(&bar_p_full[b], 4);
    }
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(&tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  WaitCtx wc{&abort_flag, p.wait_limit_ns, 0};

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    // The whole warp walks the schedule; lane 0 issues the copies.
    wc.role = kRoleProducer;
    const bool leader = lane == 0;
    if (leader) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    uint32_t ring = 0, qcount = 0;
    bool skip_next_k = (p.fault_flags & 1) && blockIdx.x == 0;
    int skipped_ring = -1;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int idx = snake_item(k, p.total_items);
      if (idx == -2) break;
      if (idx < 0) continue;
      const Item it = decode_item(idx, p);
      if (it.len == 0) continue;
      if (!(ok = warp_wait(&bar_q_empty, (qcount & 1u) ^ 1u, wc, kBarQEmpty, qcount))) break;
      const int ib = it.bh / p.heads, ih = it.bh - ib * p.heads;
      if (leader) {
        mbar_arrive_expect_tx(&bar_q_full, C::Q_BYTES);
        tma_load_5d(sQ, &tm_q, &bar_q_full, 0, it.qb * BN, 0, ih, ib);
      }
      ++qcount;
      // Walk the blocks as the MMA warp does (step j: QK(j+1), then PV(j),
      // after QK(0)) and load each K or V segment at its first use, so the
      // ring fills in exactly the order the MMA warp consumes it.
      SegWalker ks, vs;
      ks.reset(p, it.a, it.len);
      vs.reset(p, it.a, it.len);
      for (int t = -1; ok && t < it.len; ++t) {
#pragma unroll
        for (int side = 0; side < 2; ++side) {
          const bool is_k = side == 0;
          const int b = is_k ? t + 1 : t;
          if (is_k ? b >= it.len : t < 0) continue;
          SegWalker &w = is_k ? ks : vs;
          if (!w.advance(p, it.a, it.len, b)) continue;
          const uint32_t s = ring % C::NS;
          if (!(ok = warp_wait(&bar_kv_empty[s], ((ring / C::NS) & 1u) ^ 1u, wc, kBarKvEmpty,
                               ring)))
            break;
          if (is_k && skip_next_k) {  // test hook: this stage's barrier never gets its arrival
            skip_next_k = false;
            skipped_ring = static_cast<int>(ring);
            ++ring;
            continue;
          }
          if (leader) {
            mbar_arrive_expect_tx(&bar_kv_full[s], C::STAGE_BYTES);
            tma_load_5d(sKV + s * C::STAGE_BYTES, is_k ? &tm_k : &tm_v, &bar_kv_full[s], 0,
                        w.kb * BN, 0, ih, ib);
          }
          ++ring;
        }
      }
    }
    // Copies still in flight must land before the CTA exits: wait for the
    // latest use of every stage and for the last Q tile (bounded, even when
    // aborting).
    if (leader) {
      WaitCtx drain{&abort_flag, p.wait_limit_ns, kRoleProducer};
      int zero = 0;
      drain.abort = &zero;
      const uint32_t first = ring > C::NS ? ring - C::NS : 0;
      for (uint32_t r = first; r < ring; ++r) {
        if (static_cast<int>(r) == skipped_ring) continue;
        wait_bounded(&bar_kv_full[r % C::NS], (r / C::NS) & 1u, drain, kBarKvFull, r);
      }
      if (qcount > 0) wait_bounded(&bar_q_full, (qcount - 1) & 1u, drain, kBarQFull, qcount);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp walks the schedule and waits; lane 0 issues the MMAs.
    // Descriptors are kept as 32-bit halves: the high half is the same for
    // every operand (stride 1024 B, version 1, 128-byte swizzle) and the low
    // half is the start address >> 4 plus the leading byte offset, so each
    // k-step is one add on a precomputed base.
    wc.role = kRoleMma;
    const bool leader = lane == 0;
    constexpr uint32_t idesc_qk = idesc_bf16_f32(128, BN, false);
    constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, true);
    constexpr uint32_t kHi = (1024u >> 4) | (1u << 14) | (2u << 29);
    constexpr uint32_t kLboK = 1u << 16;                          // 16 B (unused for K-major SW128)
    constexpr uint32_t kLboV = static_cast<uint32_t>(C::CB_BYTES / 16) << 16;  // 64-wide D chunks
    const uint32_t q_lo = (smem_addr(sQ) >> 4) | kLboK;
    const uint32_t kv_base = smem_addr(sKV) >> 4;
    uint32_t ring = 0, qcount = 0, g = 0, items_done = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int idx = snake_item(k, p.total_items);
      if (idx == -2) break;
      if (idx < 0) continue;
      const Item it = decode_item(idx, p);
      if (it.len == 0) continue;
      if (!(ok = warp_wait(&bar_q_full, qcount & 1u, wc, kBarQFull, qcount))) break;
      tc_fence_after();

      SegWalker ks, vs;
      ks.reset(p, it.a, it.len);
      vs.reset(p, it.a, it.len);
      uint32_t kstage = 0, vstage = 0;
      // Step t (from -1): QK(t+1) as soon as its S buffer has been read by
      // the softmax, then PV(t) once P(t) is ready. QK for the next block
      // thus never waits on a PV, and the softmax finds S ready.
      for (int t = -1; ok && t < it.len; ++t) {
        const int bq = t + 1;
        if (bq < it.len) {
          const uint32_t gq = g + bq;
          if (gq >= 2) {  // S buffer of block gq-2 must have been loaded by the softmax
            if (!(ok = warp_wait(&bar_s_free[gq & 1u], ((gq - 2) >> 1) & 1u, wc, kBarSFree, gq)))
              break;
            tc_fence_after();
          }
          if (ks.advance(p, it.a, it.len, bq)) {
            kstage = ring % C::NS;
            if (!(ok = warp_wait(&bar_kv_full[kstage], (ring / C::NS) & 1u, wc, kBarKvFull, ring)))
              break;
            tc_fence_after();
            ++ring;
          }
          if (leader) {
            const uint32_t d_tmem = tmem + C::S_COL + (gq & 1u) * 128u;
            const uint32_t k_lo = (kv_base + kstage * (C::STAGE_BYTES >> 4) +
                                   (bq - ks.first) * (BN * 128 >> 4)) | kLboK;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off_a = (kk >> 2) * (C::BM * 128 >> 4) + (kk & 3) * 2;
              const uint32_t off_b = (kk >> 2) * (C::CB_BYTES >> 4) + (kk & 3) * 2;
              mma_ss_lh(d_tmem, q_lo + off_a, kHi, k_lo + off_b, kHi, idesc_qk, kk > 0 ? 1u : 0u);
            }
            if (bq == ks.first + ks.count - 1) mma_commit(&bar_kv_empty[kstage]);
            mma_commit(&bar_s_full[gq & 1u]);
            if (bq == it.len - 1) mma_commit(&bar_q_empty);  // last QK: Q may refill
          }
          __syncwarp();
        }
        if (t >= 0) {
          const int j = t;
          const uint32_t gg = g + j;
          if (!(ok = warp_wait(&bar_p_full[gg & 1u], (gg >> 1) & 1u, wc, kBarPFull, gg))) break;
          tc_fence_after();
          if (j == 0 && items_done > 0) {
            if (!(ok = warp_wait(&bar_o_empty, (items_done - 1) & 1u, wc, kBarOEmpty, items_done)))
              break;
            tc_fence_after();
          }
          if (vs.advance(p, it.a, it.len, j)) {
            vstage = ring % C::NS;
            if (!(ok = warp_wait(&bar_kv_full[vstage], (ring / C::NS) & 1u, wc, kBarKvFull, ring)))
              break;
            tc_fence_after();
            ++ring;
          }
          if (leader) {
            const uint32_t v_lo = (kv_base + vstage * (C::STAGE_BYTES >> 4) +
                                   (j - vs.first) * (BN * 128 >> 4)) | kLboV;
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk) {
              // V rows of 128 bytes (64 head-dim values); 64-wide head-dim
              // chunks one stage column block apart (MN-major operand)
              mma_ts_lh(tmem + C::O_COL, tmem + C::P_COL + (gg & 1u) * 64u + kk * 8,
                        v_lo + kk * (16 * 128 >> 4),
                        kHi, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
            }
            if (j == vs.first + vs.count - 1) mma_commit(&bar_kv_empty[vstage]);
            mma_commit(&bar_o_done[gg & 1u]);
          }
          __syncwarp();
        }
      }
      g += it.len;
      ++qcount;
      ++items_done;
    }
    // Let every issued MMA finish before TMEM is released.
    if (leader) {
      mma_commit(&bar_final);
      WaitCtx drain{&abort_flag, p.wait_limit_ns, kRoleMma};
      int zero = 0;
      drain.abort = &zero;
      wait_bounded(&bar_final, 0, drain, kBarFinal, g);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    wc.role = kRoleSoftmax;
    const int row_in_tile = warp * 32 + lane;
    const uint32_t lane_tmem = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float sl2 = p.scale_log2;
    uint32_t g = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int idx = snake_item(k, p.total_items);
      if (idx == -2) break;
      if (idx < 0) continue;
      const Item it = decode_item(idx, p);
      const int row = it.qb * BN + row_in_tile;
      const bool store = row_in_tile < BN && row < p.n;
      const long long orow = static_cast<long long>(it.bh) * p.n + row;
      const int ib = it.bh / p.heads, ih = it.bh - ib * p.heads;
      __nv_bfloat16 *const orow_ptr = p.out + ib * p.o_sb + ih * p.o_sh + row * p.o_sn;
      if (it.len == 0) {
        if (store) {
          uint4 *dst = reinterpret_cast<uint4 *>(orow_ptr);
#pragma unroll
          for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
          if (p.lse) p.lse[orow] = -INFINITY;
        }
        continue;
      }
      float m_ref = 0.f, l = 0.f;
      ListCache lc;
      lc.reset(p, it.a, it.len);
      for (int j = 0; j < it.len; ++j) {
        const uint32_t gg = g + j;
        const uint32_t s_tmem = lane_tmem + C::S_COL + (gg & 1u) * 128u;
        if (!(ok = warp_wait(&bar_s_full[gg & 1u], (gg >> 1) & 1u, wc, kBarSFull, gg))) break;
        tc_fence_after();
        float s[BN];
        {
          uint32_t sr[BN / 32][32];
#pragma unroll
          for (int c = 0; c < BN / 32; ++c) tmem_ld32(s_tmem + c * 32, sr[c]);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < BN / 32; ++c) {
            reg_fence32(sr[c]);
#pragma unroll
            for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(sr[c][i]);
          }
        }
        // S is in registers: its TMEM buffer may take QK(gg+2) right away.
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_s_free[gg & 1u]);
        const int kb = lc.get(p, it.a, it.len, j);
        const int valid = p.n - kb * BN;
        if (valid < BN) {
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (c >= valid) s[c] = -INFINITY;
        }
        // row max: eight independent chains of three-input max
        float m8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) m8[i] = fmaxf(s[i], s[i + 8]);
#pragma unroll
        for (int c = 16; c < BN; c += 16) {
#pragma unroll
          for (int i = 0; i < 8; ++i) m8[i] = fmax3(m8[i], s[c + i], s[c + 8 + i]);
        }
        const float mx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]),
                               fmaxf(m8[6], m8[7]));
        const float mblk = mx * sl2;
        float alpha = 1.f;
        bool rescale = false;
        if (j == 0) {
          m_ref = mblk;
        } else if (mblk > m_ref + 8.f) {
          // lazy rescale: the reference max only moves when the block max
          // exceeds it by more than 2^8; the final O / l is exact either way
          alpha = ex2_approx(m_ref - mblk);
          m_ref = mblk;
          rescale = true;
        }
        uint32_t pk[BN / 2];
        const float sum = valid < BN ? exp2_pack_row<BN, 0>(s, sl2, -m_ref, pk)
                                     : exp2_pack_row<BN, kEmuPairsPer8>(s, sl2, -m_ref, pk);
        l = l * alpha + sum;
        // P buffer gg&1 was last read by PV(gg-2). Waiting for that PV at
        // every block keeps each o_done wait phase-exact (PV(gg-4) was waited
        // for two blocks ago) and is cheap: PV(gg-2) was issued a whole block
        // earlier. Only a rescale of O also needs PV(gg-1); that wait is
        // phase-exact too, since PV(gg-3) is complete once PV(gg-2) is.
        if (gg >= 2) {
          if (!(ok = warp_wait(&bar_o_done[gg & 1u], ((gg - 2) >> 1) & 1u, wc, kBarODone, gg)))
            break;
          tc_fence_after();
        }
        if (__any_sync(0xffffffffu, rescale)) {
          if (!(ok = warp_wait(&bar_o_done[(gg - 1) & 1u], ((gg - 1) >> 1) & 1u, wc, kBarODone,
                               gg)))
            break;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(lane_tmem + C::O_COL + c * 32, r);
            tmem_wait_ld();
            reg_fence32(r);
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st32(lane_tmem + C::O_COL + c * 32, r);
          }
        }
        // P (bf16 pairs) into its TMEM buffer
#pragma unroll
        for (int c = 0; c < BN / 64; ++c) {
          uint32_t r[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = pk[c * 32 + i];
          tmem_st32(lane_tmem + C::P_COL + (gg & 1u) * 64u + c * 32, r);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_p_full[gg & 1u]);
      }
      if (!ok) break;
      const uint32_t gl = g + it.len - 1;
      if (!(ok = warp_wait(&bar_o_done[gl & 1u], (gl >> 1) & 1u, wc, kBarODone, gl))) break;
      tc_fence_after();
      const float inv_l = 1.f / l;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(lane_tmem + C::O_COL + c * 32, r);
        tmem_wait_ld();
        reg_fence32(r);
        if (store) {
          uint4 *dst = reinterpret_cast<uint4 *>(orow_ptr + c * 32);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(r[8 * v4 + 0]) * inv_l, __uint_as_float(r[8 * v4 + 1]) * inv_l);
            w.y = pack_bf16x2(__uint_as_float(r[8 * v4 + 2]) * inv_l, __uint_as_float(r[8 * v4 + 3]) * inv_l);
            w.z = pack_bf16x2(__uint_as_float(r[8 * v4 + 4]) * inv_l, __uint_as_float(r[8 * v4 + 5]) * inv_l);
            w.w = pack_bf16x2(__uint_as_float(r[8 * v4 + 6]) * inv_l, __uint_as_float(r[8 * v4 + 7]) * inv_l);
            dst[v4] = w;
          }
        }
      }
      if (store && p.lse) p.lse[orow] = (m_ref + log2f(l)) * 0.69314718055994531f;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_o_empty);
      g += it.len;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) {
    __syncwarp();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace bsa
