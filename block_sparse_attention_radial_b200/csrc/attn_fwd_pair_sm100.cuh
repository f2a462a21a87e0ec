// Block-sparse attention forward for sm_100a, two query tiles per CTA.
//
// A work item is a pair of adjacent query blocks (2p, 2p+1) of one
// (batch, head). The CTA walks the union of the two rows' key-block lists:
// each K and V tile is loaded once and used by both tiles when both list it,
// by one tile otherwise, so the L2 -> shared-memory stream per unit of tensor
// work drops to (union length) / (sum of the two lengths) of a one-tile
// kernel. Each tile runs its own softmax warpgroup, and while one tile's
// softmax works the tensor core runs the other tile's MMAs.
//
// Warp roles (384 threads, three warpgroups):
//   warps 0-3  softmax of tile A (thread = row = TMEM lane)
//   warps 4-7  softmax of tile B
//   warp 8     producer: Q_A, Q_B, then the union's K and V tiles (TMA)
//   warp 9     MMA issuer
//   warps 10-11 no role (they complete the third warpgroup)
// Register budgets: each SM sub-partition holds one warp of each warpgroup,
// launched at 168 registers per thread. The third warpgroup gives up all but
// 88 and the two softmax warpgroups take 208 each (208 + 208 + 88 = 3 x 168),
// so a softmax thread keeps its 128 scores and the packed P in registers
// without spilling, and the producer and MMA lanes still fit theirs. Each
// budget change sits inside its role's branch: the compiler allocates the
// code a change dominates within that budget, and code after a join of the
// branches would get the smallest one.
//
// TMEM: S_A [0,128), S_B [128,256), O_A [256, 256+D), O_B [256+D, 256+2D).
// P of a tile overwrites the first 64 columns of its S buffer.
//
// MMA schedule, per union step j with flags a (tile A lists block j) and b:
//   PV_A(j-1) if A listed j-1;  QK_A(j) if a;  PV_B(j-1) if B listed j-1;
//   QK_B(j) if b;  then K(j) and V(j-1) are released.
// PV_X(prev) is always issued before QK_X(next), so when S_X is complete the
// previous PV_X is complete too: the softmax can rescale O_X without waiting.
//
// Work items come from a global counter, in the longest-first order of
// pair_order_kernel: the producer takes each index and passes it to the MMA
// issuer and the softmax warps through a small ring in shared memory.
// Softmax: the row maximum of an item's first block is the reference for
// the whole item; later blocks rescale only when a row sum of P leaves
// [0, 2^64].
#pragma once

#include <climits>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "attn_fwd_sm100.cuh"
#include "rowgen.cuh"

namespace bsa {

template <int D>
struct PairCfg {
  static constexpr int BN = 128;                 // block = tile rows = MMA M and N
  static constexpr int Q_BYTES = BN * D * 2;     // one tile's Q
  static constexpr int TILE_BYTES = BN * D * 2;  // one K or V tile (one TMA box)
  // room for the alignment pad, the ring and the Q tiles, with 512 bytes kept
  // for static shared memory; the ring's stages are whole tiles, so the
  // remainder left for static use is 2 KB at D = 128 (the generated rows'
  // bitmaps and the barriers take 1.6 KB) and more at D = 64
  static constexpr int NS_FIT = (kSmemLimit - 1024 - 512 - 2 * Q_BYTES) / TILE_BYTES;
  static constexpr int NS = NS_FIT > 8 ? 8 : NS_FIT;
  static constexpr int DSMEM_USED = 1024 + 2 * Q_BYTES + NS * TILE_BYTES;
  static constexpr int DSMEM = DSMEM_USED > 122880 ? DSMEM_USED : 122880;
  static constexpr uint32_t S_COL = 0;           // S of tile t at S_COL + 128 t
  static constexpr uint32_t O_COL = 256;         // O of tile t at O_COL + D t
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int THREADS = 384;
  static constexpr uint32_t REGS_LAUNCH = 168;  // 65536 / 384, rounded down to a multiple of 8
  static constexpr uint32_t REGS_SOFTMAX = 208;
  static constexpr uint32_t REGS_OTHER = 88;
  static_assert(2 * REGS_SOFTMAX + REGS_OTHER <= 3 * REGS_LAUNCH, "register budgets");
  static_assert(NS >= 3, "K/V ring needs at least three stages");
};

// One row's key blocks read in order by a single thread. The next entry is
// loaded one call ahead, so its latency overlaps the caller's work.
struct RowReader {
  const int32_t *ptr;
  int left, nxt, hi;
  __device__ __forceinline__ int fetch() const {
    return left > 0 ? min(max(__ldg(ptr), 0), hi) : INT_MAX;
  }
  __device__ __forceinline__ void reset(const FwdParams &p, int a, int len, int nkb) {
    ptr = p.col_idx + a;
    left = len;
    hi = nkb - 1;
    nxt = fetch();
  }
  __device__ __forceinline__ void pop() {
    ++ptr;
    --left;
    nxt = fetch();
  }
};

// Where the rows' key blocks come from: the CSR lists (col_idx), or
// generated in the kernel from per-list tile patterns or the radial geometry.
// kModeQuarters: block-64 lists merged into 128-row tile lists, each entry
// with the mask of its listed 64 x 64 quarters (the softmax masks the rest).
enum : int {
  kModeLists = 0, kModeVarlen = 1, kModePatterns = 2, kModeRadial = 3, kModeQuarters = 4,
  kModeVarlenQuarters = 5  // a variable-length batch of block-64 lists as quarter tiles
};

__host__ __device__ constexpr bool mode_varlen(int m) {
  return m == kModeVarlen || m == kModeVarlenQuarters;
}
__host__ __device__ constexpr bool mode_quarters(int m) {
  return m == kModeQuarters || m == kModeVarlenQuarters;
}

// One row's key blocks in ascending order, by mode; next() returns INT_MAX
// past the end.
template <int MODE>
struct RowSource;

template <>
struct RowSource<kModeLists> {
  RowReader r;
  __device__ __forceinline__ void reset(const FwdParams &p, int list, int qb, int a0, int len,
                                        int nkb, const bsa_tile_pattern *) {
    r.reset(p, a0, len, nkb);
  }
  __device__ __forceinline__ int next() {
    const int v = r.nxt;
    if (v != INT_MAX) r.pop();
    return v;
  }
};

template <>
struct RowSource<kModeVarlen> : RowSource<kModeLists> {};

template <>
struct RowSource<kModeQuarters> : RowSource<kModeLists> {};

template <>
struct RowSource<kModeVarlenQuarters> : RowSource<kModeLists> {};

template <>
struct RowSource<kModePatterns> {
  PatternRow r;
  int left;  // the row's length from the count pass: never walk past it
  // `pat`: the item's pattern, staged in shared memory by the producer
  __device__ __forceinline__ void reset(const FwdParams &p, int list, int qb, int a0, int len,
                                        int nkb, const bsa_tile_pattern *pat) {
    r.reset(pat, p.pattern_columns, p.num_pattern_columns, qb, nkb);
    left = len;
  }
  __device__ __forceinline__ int next() {
    if (left <= 0) return INT_MAX;
    --left;
    return r.next();
  }
};

template <>
struct RowSource<kModeRadial> {
  RadialRow r;
  int left;
  __device__ __forceinline__ void reset(const FwdParams &p, int list, int qb, int a0, int len,
                                        int nkb, const bsa_tile_pattern *) {
    r.reset(p.radial, qb);
    left = len;
  }
  __device__ __forceinline__ int next() {
    if (left <= 0) return INT_MAX;
    --left;
    return r.next();
  }
};

// Key blocks of one query-block pair, walked as the sorted union of the two
// rows by one thread (the producer; the MMA issuer reads its step plans).
template <int MODE>
struct UnionWalker {
  RowSource<MODE> ra, rb;
  int va, vb;
  __device__ __forceinline__ void reset(const FwdParams &p, int list, int qa, int a0, int lenA,
                                        int b0, int lenB, int nkb, const bsa_tile_pattern *pat) {
    ra.reset(p, list, qa, a0, lenA, nkb, pat);
    rb.reset(p, list, qa + 1, b0, lenB, nkb, pat);
    va = ra.next();
    vb = rb.next();
  }
  // Next union block: false when both rows are exhausted.
  __device__ __forceinline__ bool next(int &kb, bool &inA, bool &inB) {
    if (va == INT_MAX && vb == INT_MAX) return false;
    kb = min(va, vb);
    inA = va == kb;
    inB = vb == kb;
    if (inA) va = ra.next();
    if (inB) vb = rb.next();
    return true;
  }
};

// Key blocks of one query-block pair from the two rows' bitmaps in shared
// memory, walked as their union (rows generated ahead by the item fetcher).
struct BitmapWalker {
  const volatile uint32_t *a, *b;
  int w, nw;
  uint32_t cur;
  __device__ __forceinline__ void reset(const uint32_t *ba, const uint32_t *bb, int nwords) {
    a = ba;
    b = bb;
    nw = nwords;
    w = 0;
    cur = nwords > 0 ? (a[0] | b[0]) : 0u;
  }
  __device__ __forceinline__ bool next(int &kb, bool &inA, bool &inB) {
    while (cur == 0u) {
      if (++w >= nw) return false;
      cur = a[w] | b[w];
    }
    const int bit = __ffs(cur) - 1;
    cur &= cur - 1u;
    kb = w * 32 + bit;
    inA = ((a[w] >> bit) & 1u) != 0u;
    inB = ((b[w] >> bit) & 1u) != 0u;
    return true;
  }
};

constexpr int kItemN = 4;  // work items in flight between the producer and the consumers

struct PairItem {
  int bh, qa, a0, lenA, b0, lenB;  // tile B absent (lenB = 0) past the last block
  int n, nqb, nkb, tok0;           // the item's tokens, query and key blocks, first token
  int list;                        // the list (pattern) the item's rows belong to
};

// Rows qa and qa + 1 (when it exists) of the list starting at row lbase.
__device__ __forceinline__ void pair_rows(const FwdParams &p, long long lbase, PairItem &it) {
  const int a = min(max(p.row_ptr[lbase + it.qa], 0), p.nnz);
  const int ae = min(max(p.row_ptr[lbase + it.qa + 1], 0), p.nnz);
  it.a0 = a;
  it.lenA = max(ae - a, 0);
  if (it.qa + 1 < it.nqb) {
    const int b = min(max(p.row_ptr[lbase + it.qa + 1], 0), p.nnz);
    const int be = min(max(p.row_ptr[lbase + it.qa + 2], 0), p.nnz);
    it.b0 = b;
    it.lenB = max(be - b, 0);
  } else {
    it.b0 = 0;
    it.lenB = 0;
  }
}

template <int MODE>
__device__ __forceinline__ PairItem decode_pair(int idx, const FwdParams &p, int npairs,
                                                const VarlenTable &vt) {
  PairItem it;
  if (!mode_varlen(MODE)) {
    it.n = p.n;
    it.nqb = p.nqb;
    it.nkb = p.nkb;
    it.tok0 = 0;
    it.bh = idx / npairs;
    const int rank = idx - it.bh * npairs;
    const int h = it.bh % p.heads;
    const int list = p.head_list ? min(max(p.head_list[h], 0), p.num_lists - 1)
                                 : (p.num_lists > 1 ? h : 0);
    it.list = list;
    const long long lbase = static_cast<long long>(list) * p.nqb;
    const int pr = min(max(p.order[static_cast<long long>(list) * npairs + rank], 0), npairs - 1);
    it.qa = 2 * pr;
    pair_rows(p, lbase, it);
    return it;
  }
  // the item holding work index idx: the last b with work0[b] <= idx (items
  // without work share their work0 with the next item and are skipped)
  int lo = 0, hi = vt.num_items - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (vt.work0[mid] <= idx)
      lo = mid;
    else
      hi = mid - 1;
  }
  const int b = lo;
  it.tok0 = vt.tok0[b];
  it.n = vt.tok0[b + 1] - it.tok0;
  it.nqb = vt.row0[b + 1] - vt.row0[b];
  it.nkb = it.nqb;
  const int np = vt.pair0[b + 1] - vt.pair0[b];
  const int local = idx - vt.work0[b];
  it.bh = local / np;  // the head (batch extent 1)
  const int rank = local - it.bh * np;
  const int list = p.num_lists > 1 ? it.bh : 0;
  it.list = list;
  const long long lbase = static_cast<long long>(p.num_lists) * vt.row0[b] +
                          static_cast<long long>(list) * it.nqb;
  const long long obase = static_cast<long long>(p.num_lists) * vt.pair0[b] +
                          static_cast<long long>(list) * np;
  const int pr = min(max(p.order[obase + rank], 0), np - 1);
  it.qa = 2 * pr;
  pair_rows(p, lbase, it);
  return it;
}

// Step plans: the producer, which walks the schedule anyway, writes one
// 32-bit record per step into a small shared ring, so the MMA issuer reads
// its step instead of walking the lists itself (the issuer's time between
// MMA groups is tensor-pipe idle time). Record bits:
//   1 PV of tile A, 2 QK of tile A, 3 PV of tile B, 4 QK of tile B,
//   5 last step of the item, 8-10 V stage, 11 its fill parity,
//   12-14 K stage, 15 its fill parity, 24-31 generation tag (never 0).
// The producer runs at most a few steps ahead (it is held by the K/V ring and
// by the Q buffers), far less than kPlanN steps, so a record is never
// overwritten before it is read.
constexpr int kPlanN = 32;

__device__ __forceinline__ uint32_t plan_tag(uint32_t step) {
  return ((step / kPlanN) & 0x7fu) + 1u;
}

// Bounded wait for step `step`'s record.
__device__ __forceinline__ bool plan_wait(const volatile uint32_t *ring, uint32_t step,
                                          uint32_t &rec, const WaitCtx &w) {
  const volatile uint32_t *slot = ring + step % kPlanN;
  const uint32_t tag = plan_tag(step);
  rec = *slot;
  if ((rec >> 24) == tag) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i) {
      rec = *slot;
      if ((rec >> 24) == tag) return true;
    }
    if (*w.abort) return false;
    if (global_timer_ns() - t0 > w.limit) {
      if (atomicCAS(&g_status, 0u, 4u /* BSA_ERR_DEVICE_TIMEOUT */) == 0u) {
        g_status_detail[0] = w.role;
        g_status_detail[1] = kBarPlan;
        g_status_detail[2] = step;
        g_status_detail[3] = blockIdx.x;
      }
      *w.abort = 1;
      return false;
    }
  }
}

template <int D, int MODE>
__global__ void __launch_bounds__(384, 1)
    attn_fwd_pair_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                               const __grid_constant__ CUtensorMap tm_k,
                               const __grid_constant__ CUtensorMap tm_v, const FwdParams p,
                               const __grid_constant__ VarlenTable vt) {
  using C = PairCfg<D>;
  constexpr int BN = C::BN;
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t bar_kv_full[C::NS];
  __shared__ __align__(8) uint64_t bar_kv_empty[C::NS];
  __shared__ __align__(8) uint64_t bar_q_full, bar_q_empty, bar_final;
  __shared__ __align__(8) uint64_t bar_s_full[2], bar_p_full[2], bar_o_final[2], bar_o_empty[2];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ uint32_t plan_ring[kPlanN];
  // Work items are taken from a global counter by the producer, in the work
  // order, and handed to the MMA issuer and the softmax warps through this
  // ring (a longest-first order served dynamically keeps the CTAs' finishing
  // times within about one item of each other).
  __shared__ int item_ring[kItemN];
  // the producer's copy of the current item's tile pattern (rows generated
  // from tile patterns only)
  __shared__ bsa_tile_pattern prod_pat;
  __shared__ __align__(8) uint64_t bar_item_full[kItemN], bar_item_empty[kItemN];
  // Rows generated in the kernel: warp 10 takes the work items instead of
  // the producer and generates each item's two rows into bitmaps here
  // (rows of up to kGenRowWords * 32 key blocks; longer rows are generated
  // by the producer as it walks them), a few items ahead of the walk.
  constexpr bool kGen = MODE == kModePatterns || MODE == kModeRadial;
  constexpr int kGenRowWords = 32;
  __shared__ uint32_t row_bits[kGen ? kItemN : 1][2][kGen ? kGenRowWords : 1];
  __shared__ int row_len[kGen ? kItemN : 1][2];
  const bool bitmaps = kGen && p.nkb <= kGenRowWords * 32;

  const uint32_t raw = smem_addr(dsmem);
  uint8_t *base = dsmem + (((raw + 1023u) & ~1023u) - raw);
  uint8_t *sQ = base;                      // Q_A, then Q_B at + Q_BYTES
  uint8_t *sKV = base + 2 * C::Q_BYTES;
  const int npairs = (p.nqb + 1) / 2;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x < kPlanN) plan_ring[threadIdx.x] = 0u;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&bar_kv_full[s], 1);
      mbar_init(&bar_kv_empty[s], 1);
    }
    mbar_init(&bar_q_full, 1);
    mbar_init(&bar_q_empty, 1);
    mbar_init(&bar_final, 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bar_s_full[t], 1);
      mbar_init(&bar_p_full[t], 4);   // one arrival per softmax warp
      mbar_init(&bar_o_final[t], 1);
      mbar_init(&bar_o_empty[t], 4);
    }
    for (int i = 0; i < kItemN; ++i) {
      mbar_init(&bar_item_full[i], 1);
      // the MMA lane and one lane per softmax warp (and, for generated rows,
      // the producer once it has walked the item's bitmaps)
      mbar_init(&bar_item_empty[i], kGen ? 10 : 9);
    }
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(&tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  WaitCtx wc{&abort_flag, p.wait_limit_ns, 0};

  // Each budget change sits inside its role's branch, so that the role's code
  // is dominated by it and the compiler allocates that role's registers
  // within its own budget (after a join of the branches it would have to
  // assume the smallest).
  if (warp >= 8) {
    regs_shrink<C::REGS_OTHER>();
    if (warp == 8) {
      // ------------------------------------------------------------ producer
      // One lane: TMA issue needs no warp, and warp-wide bookkeeping between
      // issues only adds latency.
      if (lane == 0) {
        wc.role = kRoleProducer;
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        uint32_t ring = 0, qcount = 0, gstep = 0;
        volatile uint32_t *plans = plan_ring;
        bool skip_next_k = (p.fault_flags & 1) && blockIdx.x == 0;
        int skipped_ring = -1;
        bool ok = true;
        for (int k = 0; ok; ++k) {
          const int slot = k % kItemN;
          int idx;
          if (kGen) {  // warp 10 takes the items
            if (!(ok = lane_wait(&bar_item_full[slot], (k / kItemN) & 1, wc, kBarItem, k))) break;
            idx = *static_cast<volatile int *>(&item_ring[slot]);
          } else {
            if (!(ok = lane_wait(&bar_item_empty[slot], ((k / kItemN) & 1) ^ 1, wc, kBarItem, k)))
              break;
            idx = atomicAdd(p.item_counter, 1);
            if (idx >= p.total_items) idx = -1;
            item_ring[slot] = idx;
            mbar_arrive(&bar_item_full[slot]);
          }
          if (idx < 0) break;
          PairItem it = decode_pair<MODE>(idx, p, npairs, vt);
          if (bitmaps) {
            it.lenA = *static_cast<volatile int *>(&row_len[slot][0]);
            it.lenB = *static_cast<volatile int *>(&row_len[slot][1]);
          }
          if (it.lenA == 0 && it.lenB == 0) {
            if (kGen) mbar_arrive(&bar_item_empty[slot]);
            continue;
          }
          if (!(ok = lane_wait(&bar_q_empty, (qcount & 1u) ^ 1u, wc, kBarQEmpty, qcount))) break;
          mbar_arrive_expect_tx(&bar_q_full, 2 * C::Q_BYTES);
          const int ib = it.bh / p.heads, ih = it.bh - ib * p.heads;
          tma_load_5d(sQ, &tm_q, &bar_q_full, 0, it.tok0 + it.qa * BN, 0, ih, ib);
          tma_load_5d(sQ + C::Q_BYTES, &tm_q, &bar_q_full, 0, it.tok0 + (it.qa + 1) * BN, 0, ih,
                      ib);
          ++qcount;
          // Same walk and same first-use order as the MMA issuer: at step j it
          // needs V(j-1) first when tile A listed j-1 or A skips j, and K(j)
          // first otherwise.
          UnionWalker<MODE> uw;
          BitmapWalker bw;
          if (bitmaps) {
            bw.reset(row_bits[slot][0], row_bits[slot][1], (it.nkb + 31) >> 5);
          } else {
            if (MODE == kModePatterns) prod_pat = p.patterns[it.list];
            uw.reset(p, it.list, it.qa, it.a0, it.lenA, it.b0, it.lenB, it.nkb, &prod_pat);
          }
          bool pa = false, pb = false;
          int prev_kb = 0;
          while (ok) {
            int kb = 0;
            bool a = false, b = false;
            const bool more = bitmaps ? bw.next(kb, a, b) : uw.next(kb, a, b);
            const bool need_v = pa || pb;
            if (!more && !need_v) break;
            const bool v_first = pa || !a;
            {
              const bool need_k = more;
              const uint32_t vpos = ring + ((need_k && !v_first) ? 1u : 0u);
              const uint32_t kpos = ring + ((need_v && v_first) ? 1u : 0u);
              const uint32_t rec =
                  (pa ? 2u : 0u) | (a ? 4u : 0u) | (pb ? 8u : 0u) | (b ? 16u : 0u) |
                  (more ? 0u : 32u) | ((vpos % C::NS) << 8) | (((vpos / C::NS) & 1u) << 11) |
                  ((kpos % C::NS) << 12) | (((kpos / C::NS) & 1u) << 15) | (plan_tag(gstep) << 24);
              plans[gstep % kPlanN] = rec;
              ++gstep;
            }
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const bool is_v = (e == 0) == v_first;
              if (is_v ? !need_v : !more) continue;
              const uint32_t s = ring % C::NS;
              if (!(ok = lane_wait(&bar_kv_empty[s], ((ring / C::NS) & 1u) ^ 1u, wc, kBarKvEmpty,
                                   ring)))
                break;
              if (!is_v && skip_next_k) {  // test hook: this stage's barrier never gets its arrival
                skip_next_k = false;
                skipped_ring = static_cast<int>(ring);
                ++ring;
                continue;
              }
              mbar_arrive_expect_tx(&bar_kv_full[s], C::TILE_BYTES);
              tma_load_5d(sKV + s * C::TILE_BYTES, is_v ? &tm_v : &tm_k, &bar_kv_full[s], 0,
                          it.tok0 + (is_v ? prev_kb : kb) * BN, 0, ih, ib);
              ++ring;
            }
            pa = a;
            pb = b;
            prev_kb = kb;
            if (!more) break;
          }
          // the item's rows are walked: its slot may take the next item
          if (kGen && ok) mbar_arrive(&bar_item_empty[slot]);
        }
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
    }
    else if (warp == 9) {
      // ------------------------------------------------------------ MMA issuer
      // One lane issues everything. tcgen05.mma and tcgen05.commit issued from
      // a single thread go back to back; issued under a lane-0 branch of a
      // whole warp that also votes on its waits, each MMA and commit costs
      // tens of extra cycles. Descriptors as 32-bit halves (see the one-tile
      // kernel): shared high half, low half = address >> 4 | LBO.
      if (lane == 0) {
        wc.role = kRoleMma;
        constexpr uint32_t idesc_qk = idesc_bf16_f32(128, BN, false);
        constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, true);
        constexpr uint32_t kHi = (1024u >> 4) | (1u << 14) | (2u << 29);
        constexpr uint32_t kLboK = 1u << 16;
        constexpr uint32_t kLboV = static_cast<uint32_t>(BN * 128 / 16) << 16;  // 64-wide D chunks
        const uint32_t q_lo0 = (smem_addr(sQ) >> 4) | kLboK;
        const uint32_t kv_base = smem_addr(sKV) >> 4;
        uint32_t gstep = 0, qcount = 0;
        const volatile uint32_t *plans = plan_ring;
        uint32_t rec_next = 0u;
        uint32_t pcnt[2] = {0u, 0u};     // p_full phases consumed, per tile
        uint32_t items_t[2] = {0u, 0u};  // items in which the tile had blocks
        bool ok = true;
        for (int k = 0; ok; ++k) {
          const int slot = k % kItemN;
          if (!(ok = lane_wait(&bar_item_full[slot], (k / kItemN) & 1, wc, kBarItem, k))) break;
          const int idx = *static_cast<volatile int *>(&item_ring[slot]);
          int glen[2] = {0, 0};
          if (bitmaps && idx >= 0) {  // read before the slot is released
            glen[0] = *static_cast<volatile int *>(&row_len[slot][0]);
            glen[1] = *static_cast<volatile int *>(&row_len[slot][1]);
          }
          mbar_arrive(&bar_item_empty[slot]);
          if (idx < 0) break;
          PairItem it = decode_pair<MODE>(idx, p, npairs, vt);
          if (bitmaps) {
            it.lenA = glen[0];
            it.lenB = glen[1];
          }
          if (it.lenA == 0 && it.lenB == 0) continue;
          if (!(ok = lane_wait(&bar_q_full, qcount & 1u, wc, kBarQFull, qcount))) break;
          tc_fence_after();
          const int len_t[2] = {it.lenA, it.lenB};
          bool first_pv[2] = {true, true};
          bool q_released = false;
          while (ok) {
            // this step's record (usually already there: the producer runs ahead)
            uint32_t rec = rec_next;
            if ((rec >> 24) != plan_tag(gstep) && !(ok = plan_wait(plan_ring, gstep, rec, wc)))
              break;
            ++gstep;
            const bool pv[2] = {(rec & 2u) != 0u, (rec & 8u) != 0u};
            const bool qk[2] = {(rec & 4u) != 0u, (rec & 16u) != 0u};
            const bool last = (rec & 32u) != 0u;
            const uint32_t vstage = (rec >> 8) & 7u, vpar = (rec >> 11) & 1u;
            const uint32_t kstage = (rec >> 12) & 7u, kpar = (rec >> 15) & 1u;
            if (last && !q_released) {  // no QK left in this item: the Q buffers may refill
              mma_commit(&bar_q_empty);
              q_released = true;
            }
            // Early non-blocking checks of this step's barriers: a check of
            // even a completed mbarrier takes about as long as two MMAs and the
            // tensor pipe accepts one MMA at a time, so checks issued together
            // (and ahead of the MMAs that precede their use) keep that latency
            // off the tensor pipe.
            const bool need_v = pv[0] || pv[1];
            const bool need_k = qk[0] || qk[1];
            bool p_ready[2];
            p_ready[0] = pv[0] && mbar_test(&bar_p_full[0], pcnt[0] & 1u);
            const bool v_ready = need_v && mbar_test(&bar_kv_full[vstage], vpar);
            const bool k_ready = need_k && mbar_test(&bar_kv_full[kstage], kpar);
            p_ready[1] = false;
            bool have_k = false, have_v = false;
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              if (!ok) break;
              if (t == 1) rec_next = plans[gstep % kPlanN];  // next step's record, read ahead
              if (pv[t]) {
                if (!p_ready[t] &&
                    !(ok = lane_wait(&bar_p_full[t], pcnt[t] & 1u, wc, kBarPFull, pcnt[t])))
                  break;
                ++pcnt[t];
                if (first_pv[t] && items_t[t] > 0) {
                  if (!(ok = lane_wait(&bar_o_empty[t], (items_t[t] - 1) & 1u, wc, kBarOEmpty,
                                       items_t[t])))
                    break;
                }
                if (!have_v) {
                  if (!v_ready &&
                      !(ok = lane_wait(&bar_kv_full[vstage], vpar, wc, kBarKvFull, gstep)))
                    break;
                  have_v = true;
                }
                tc_fence_after();
                // tile B's P, checked while tile A's MMAs go out
                if (t == 0 && pv[1]) p_ready[1] = mbar_test(&bar_p_full[1], pcnt[1] & 1u);
                const uint32_t v_lo = (kv_base + vstage * (C::TILE_BYTES >> 4)) | kLboV;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk)
                  mma_ts_lh(tmem + C::O_COL + t * D, tmem + C::S_COL + t * 128 + kk * 8,
                            v_lo + kk * (16 * 128 >> 4), kHi, idesc_pv,
                            (!first_pv[t] || kk > 0) ? 1u : 0u);
                first_pv[t] = false;
              } else if (t == 0 && pv[1]) {
                p_ready[1] = mbar_test(&bar_p_full[1], pcnt[1] & 1u);
              }
              if (qk[t]) {
                if (!have_k) {
                  if (!k_ready &&
                      !(ok = lane_wait(&bar_kv_full[kstage], kpar, wc, kBarKvFull, gstep)))
                    break;
                  tc_fence_after();
                  have_k = true;
                }
                const uint32_t q_lo = q_lo0 + t * (C::Q_BYTES >> 4);
                const uint32_t k_lo = (kv_base + kstage * (C::TILE_BYTES >> 4)) | kLboK;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                  const uint32_t off = (kk >> 2) * (BN * 128 >> 4) + (kk & 3) * 2;
                  mma_ss_lh(tmem + C::S_COL + t * 128, q_lo + off, kHi, k_lo + off, kHi, idesc_qk,
                            kk > 0 ? 1u : 0u);
                }
                mma_commit(&bar_s_full[t]);
              }
            }
            if (!ok) break;
            if (have_k) mma_commit(&bar_kv_empty[kstage]);
            if (have_v) mma_commit(&bar_kv_empty[vstage]);
            if (last) break;
          }
          if (!ok) break;
#pragma unroll
          for (int t = 0; t < 2; ++t)
            if (len_t[t] > 0) mma_commit(&bar_o_final[t]);
          if (!q_released) mma_commit(&bar_q_empty);
#pragma unroll
          for (int t = 0; t < 2; ++t) items_t[t] += len_t[t] > 0 ? 1u : 0u;
          ++qcount;
        }
        mma_commit(&bar_final);
        WaitCtx drain{&abort_flag, p.wait_limit_ns, kRoleMma};
        int zero = 0;
        drain.abort = &zero;
        wait_bounded(&bar_final, 0, drain, kBarFinal, qcount);
      }
      __syncwarp();
    } else if (kGen && warp == 10) {
      // ------------------------------------------------- item fetcher (rows
      // generated in the kernel): takes the work items from the counter and,
      // a few items ahead of the producer's walk, generates each item's two
      // rows into bitmaps (lane r generates row r; every lane clears a word)
      wc.role = kRoleProducer;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int slot = k % kItemN;
        if (!(ok = warp_wait(&bar_item_empty[slot], ((k / kItemN) & 1) ^ 1, wc, kBarItem, k)))
          break;
        int idx = 0;
        if (lane == 0) {
          idx = atomicAdd(p.item_counter, 1);
          if (idx >= p.total_items) idx = -1;
        }
        idx = __shfl_sync(0xffffffffu, idx, 0);
        if (idx >= 0 && bitmaps) {
          // the list builders' own row marking, spread over the warp's lanes
          const PairItem it = decode_pair<MODE>(idx, p, npairs, vt);
          const int words = (it.nkb + 31) >> 5;
#pragma unroll 1
          for (int r = 0; r < 2; ++r) {
            uint32_t *bits = row_bits[slot][r];
            const int qb = it.qa + r;
            bits[lane] = 0u;
            __syncwarp();
            if (qb < it.nqb) {
              if (MODE == kModeRadial) {
                radial_mark_row(p.radial, qb, bits, lane, 32);
              } else {
                const bsa_tile_pattern &pat = p.patterns[it.list];
                const bool pok = pattern_ok(pat, p.num_pattern_columns);
                pattern_row_words(pat, pok, qb, it.nkb, bits, words, lane, 32);
                __syncwarp();
                if (pok) pattern_row_columns(pat, p.pattern_columns, it.nkb, bits, lane, 32, false);
              }
            }
            __syncwarp();
            const int cnt = __reduce_add_sync(0xffffffffu, __popc(bits[lane]));
            if (lane == 0) row_len[slot][r] = cnt;
          }
          __syncwarp();
        }
        if (lane == 0) {
          item_ring[slot] = idx;
          mbar_arrive(&bar_item_full[slot]);
        }
        __syncwarp();
        if (idx < 0) break;
      }
    }
    // warp 11 (and warp 10 when rows come from lists) has no role: it waits
    // at the final barrier
  } else {
    // ------------------------------------------------------------ softmax
    // Warpgroup t (warps 4t..4t+3) serves tile t; thread = row = TMEM lane.
    regs_grow<C::REGS_SOFTMAX>();
    wc.role = kRoleSoftmax;
    const int t = warp >> 2;
    const int wq = warp & 3;
    const int row_in_tile = wq * 32 + lane;
    const uint32_t lane_tmem = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t s_tmem = lane_tmem + C::S_COL + t * 128;
    const uint32_t o_tmem = lane_tmem + C::O_COL + t * D;
    const float sl2 = p.scale_log2;
    uint32_t scnt = 0, icnt = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int slot = k % kItemN;
      if (!(ok = warp_wait(&bar_item_full[slot], (k / kItemN) & 1, wc, kBarItem, k))) break;
      const int idx = *static_cast<volatile int *>(&item_ring[slot]);
      const int glen = bitmaps && idx >= 0 ? *static_cast<volatile int *>(&row_len[slot][t]) : 0;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_item_empty[slot]);
      if (idx < 0) break;
      const PairItem it = decode_pair<MODE>(idx, p, npairs, vt);
      const int qb = it.qa + t;
      if (qb >= it.nqb) continue;
      const int len = bitmaps ? glen : (t == 0 ? it.lenA : it.lenB);
      const int a0 = t == 0 ? it.a0 : it.b0;
      const int row = qb * BN + row_in_tile;
      const bool store = row < it.n;
      const long long orow = static_cast<long long>(it.bh) * p.n + it.tok0 + row;
      const int ib = it.bh / p.heads, ih = it.bh - ib * p.heads;
      __nv_bfloat16 *const orow_ptr =
          p.out + ib * p.o_sb + ih * p.o_sh + static_cast<long long>(it.tok0 + row) * p.o_sn;
      if (len == 0) {
        if (store) {
          uint4 *dst = reinterpret_cast<uint4 *>(orow_ptr);
#pragma unroll
          for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
          if (p.lse) p.lse[orow] = -INFINITY;
        }
        continue;
      }
      // Lists are sorted, so only the row's last block can be the ragged
      // final key block; its valid column count is taken once per item.
      int last_valid;
      if (MODE == kModeLists || mode_varlen(MODE) || mode_quarters(MODE)) {
        const int last_kb = min(max(__ldg(p.col_idx + a0 + len - 1), 0), it.nkb - 1);
        last_valid = min(it.n - last_kb * BN, BN);
      } else {
        // generated rows: the last block is ragged iff the row holds the
        // final key block
        bool has_final;
        if (MODE == kModePatterns) {
          PatternRow r;
          r.reset(p.patterns + it.list, p.pattern_columns, p.num_pattern_columns, qb, it.nkb);
          has_final = r.has(it.nkb - 1);
        } else {
          RadialRow r;
          r.reset(p.radial, qb);
          has_final = r.has(it.nkb - 1);
        }
        last_valid = has_final ? min(it.n - (it.nkb - 1) * BN, BN) : BN;
      }
      // With quarter masks a row half may have nothing listed in its first
      // blocks: it then carries no reference maximum (-inf) until it does.
      float m_ref = mode_quarters(MODE) ? -INFINITY : 0.f, l = 0.f;
      const int qhalf = wq >> 1;  // the 64-row half of the tile this warp's rows are in
      for (int j = 0; j < len; ++j) {
        // this block's listed key halves for the warp's query half
        const uint32_t qbits =
            mode_quarters(MODE) ? (__ldg(p.tile_mask + a0 + j) >> (2 * qhalf)) & 3u : 3u;
        if (!(ok = warp_wait(&bar_s_full[t], scnt & 1u, wc, kBarSFull, scnt))) break;
        ++scnt;
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
        const int valid = j == len - 1 ? last_valid : BN;
        if (valid < BN) {
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (c >= valid) s[c] = -INFINITY;
        }
        if (mode_quarters(MODE) && qbits != 3u) {  // an unlisted key half
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (!((qbits >> (c >> 6)) & 1u)) s[c] = -INFINITY;
        }
        // a column the row attends in this block (used when S is re-read)
        auto col_ok = [&](int c) { return c < valid && ((qbits >> (c >> 6)) & 1u); };
        auto row_max = [&]() {
          float m8[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) m8[i] = fmaxf(s[i], s[i + 8]);
#pragma unroll
          for (int c = 16; c < BN; c += 16) {
#pragma unroll
            for (int i = 0; i < 8; ++i) m8[i] = fmax3(m8[i], s[c + i], s[c + 8 + i]);
          }
          return fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]),
                       fmaxf(m8[6], m8[7]));
        };
        uint32_t pk[BN / 2];
        auto exp_row = [&]() {
          // a row without a reference maximum has every column at -inf here
          // (its block maximum is -inf): any finite bias gives P = 0, sum 0
          const float bias = mode_quarters(MODE) && m_ref == -INFINITY ? 0.f : -m_ref;
          if (mode_quarters(MODE)) {
            // the exponentials of a key half this warp's query half does not
            // list are not computed (P = 0 there); both halves listed: the
            // same operations in the same order as a whole row
            float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                             make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            if (qbits & 1u) {
              exp2_pack_pairs<BN, 0, 0, BN / 4>(s, sl2, bias, pk, acc);
            } else {
#pragma unroll
              for (int c = 0; c < BN / 4; ++c) pk[c] = 0u;
            }
            if (qbits & 2u) {
              exp2_pack_pairs<BN, 0, BN / 4, BN / 2>(s, sl2, bias, pk, acc);
            } else {
#pragma unroll
              for (int c = BN / 4; c < BN / 2; ++c) pk[c] = 0u;
            }
            return exp2_row_sum(acc);
          }
          return valid < BN ? exp2_pack_row<BN, 0>(s, sl2, bias, pk)
                            : exp2_pack_row<BN, kEmuPairsPer8>(s, sl2, bias, pk);
        };
        float alpha = 1.f;
        bool rescale = false;
        float sum;
        if (mode_quarters(MODE)) {
          // rows without a reference yet take this block's maximum (still
          // -inf when none of the row's columns here is listed); the vote
          // keeps the branch warp-uniform
          if (__any_sync(0xffffffffu, m_ref == -INFINITY)) {
            const float mb = row_max() * sl2;
            if (m_ref == -INFINITY) m_ref = mb;
          }
        } else if (j == 0) {
          m_ref = row_max() * sl2;
        }
        sum = exp_row();
        // (at j = 0, and at a row's first block with a reference, the
        // reference is the block's own maximum: every P <= 1, no rescale)
        if (j > 0) {
          // The reference stays the first block's maximum: P may exceed 1 by
          // far (bf16 keeps its relative precision and the fp32 sums stay
          // finite), so the row maximum is only taken again when the row sum
          // leaves [0, 2^64]; then O and l are rescaled (the final O / l and
          // lse are exact either way).
          // Warp-uniform: the TMEM reads below are warp-collective
          // (.sync.aligned), so when any row of the warp needs the rescale
          // every lane takes this path (a rescale is valid for any row).
          if (__any_sync(0xffffffffu, !(sum <= 0x1p64f))) {
            // S is still in TMEM (P has not been stored over it yet): take the
            // row maximum from it, then recompute P 32 columns at a time, so
            // that no more than one chunk of scores is live next to P
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < BN / 32; ++c) {
              uint32_t sr[32];
              tmem_ld32(s_tmem + c * 32, sr);
              tmem_wait_ld();
              reg_fence32(sr);
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (col_ok(c * 32 + i)) mx = fmaxf(mx, __uint_as_float(sr[i]));
            }
            const float m_new = fmaxf(m_ref, mx * sl2);
            // (a row with nothing listed so far keeps P = 0 and alpha = 1)
            const bool has_ref = m_new != -INFINITY;
            alpha = has_ref ? ex2_approx(m_ref - m_new) : 1.f;
            m_ref = m_new;
            rescale = has_ref;
            float2 acc = make_float2(0.f, 0.f);
#pragma unroll
            for (int c = 0; c < BN / 32; ++c) {
              uint32_t sr[32];
              tmem_ld32(s_tmem + c * 32, sr);
              tmem_wait_ld();
              reg_fence32(sr);
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const int col = c * 32 + 2 * i;
                const float a = has_ref && col_ok(col)
                                    ? ex2_approx(fmaf(__uint_as_float(sr[2 * i]), sl2, -m_ref))
                                    : 0.f;
                const float b = has_ref && col_ok(col + 1)
                                    ? ex2_approx(fmaf(__uint_as_float(sr[2 * i + 1]), sl2, -m_ref))
                                    : 0.f;
                acc.x += a;
                acc.y += b;
                pk[c * 16 + i] = pack_bf16x2(a, b);
              }
            }
            sum = acc.x + acc.y;
          }
        }
        l = l * alpha + sum;
        // S being complete means QK of this block is complete, and the
        // previous PV of this tile was issued before it: O is settled.
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(o_tmem + c * 32, r);
            tmem_wait_ld();
            reg_fence32(r);
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st32(o_tmem + c * 32, r);
          }
        }
        // P (bf16 pairs) over the first BN/2 columns of this tile's S buffer
#pragma unroll
        for (int c = 0; c < BN / 64; ++c) {
          uint32_t r[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = pk[c * 32 + i];
          tmem_st32(s_tmem + c * 32, r);
        }
        // the warp-collective wait covers every lane's stores; one arrival
        // per warp (128 arrivals on one barrier would serialise)
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_p_full[t]);
      }
      if (!ok) break;
      if (!(ok = warp_wait(&bar_o_final[t], icnt & 1u, wc, kBarODone, icnt))) break;
      ++icnt;
      tc_fence_after();
      // l = 0 only for a row with nothing listed in any block (a row half
      // whose quarters are all unlisted): out 0, lse -inf, like an empty row
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(o_tmem + c * 32, r);
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
      if (store && p.lse)
        p.lse[orow] = l > 0.f ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_o_empty[t]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) {
    __syncwarp();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace bsa
