// One-pass block-sparse attention backward for sm_100a (block 128, head_dim
// 64/128): dK, dV and dQ from one kernel, each listed block pair's products
// computed once.
//
// Same definitions as attn_bwd_sm100.cuh (the derivative of the forward; the
// radial attention module is fine-tuned with LoRA in [RA-skill] Step 4):
//   P = exp(S * scale - lse),  dV = P^T dO,  dP = dO V^T,
//   delta_i = sum_d dO_id O_id,  dS = P * (dP - delta),
//   dQ = dS K * scale,  dK = dS^T Q * scale.
//
// One work item = (batch*head, key block): K and V stay in shared memory
// while the key block's query blocks stream through. Per query block e the
// MMA warp runs S^T = K Q_e^T and dP^T = V dO_e^T; the elementwise warps
// write P^T (bf16) into TMEM over S^T and dS^T (bf16) into shared memory;
// then dV += P^T dO_e (A from TMEM), dK += dS^T Q_e and dQ_e = dS_e K (A and
// B from shared memory: the same dS^T tile read K-major for dK and MN-major
// for dQ). Five block products per listed pair, against seven for the
// two-kernel backward, which recomputes S and dP for dQ.
//
// dQ_e is this key block's part of query block e's gradient. The parts of a
// query block are summed in a fixed order, the order of the keys in the
// query block's row (ascending): the elementwise warp that holds part p
// waits until a per-(query block, warp) counter reaches p, adds its part to
// an fp32 accumulator row in the workspace (the first part stores, middle
// parts add with red.global.add, the last part reads the sum, scales, rounds
// to bf16 and writes dq), fences and advances the counter. The result is
// deterministic and does not depend on which CTA runs which key block.
// Progress: work items are served in ascending (batch*head, key block)
// order and each waits only for parts of smaller key blocks of the same
// batch*head, all served earlier to running CTAs; the smallest key block in
// flight never waits, so every wait ends. Each wait is also bounded in time
// (the kernel's wait limit): when one runs out the CTA records
// BSA_ERR_DEVICE_TIMEOUT and leaves, like every other bounded wait here.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "attn_bwd_sm100.cuh"

namespace bsa {

constexpr int kBarDqSem = 13;  // timeout detail: the dQ part counter

template <int D>
struct FusedCfg {
  static constexpr int T = kBwdBlock * D * 2;        // one 128 x D bf16 tile
  static constexpr int STAGE = 2 * T;                // Q and dO of a query block
  static constexpr int DS = kBwdBlock * kBwdBlock * 2;  // dS^T, bf16
  static constexpr int NS_FIT = (kSmemLimit - 1024 - 1024 - 2 * T - DS) / STAGE;
  static constexpr int NS = NS_FIT > 4 ? 4 : NS_FIT;
  static constexpr int DSMEM = 1024 + 2 * T + NS * STAGE + DS;
  static constexpr uint32_t ST_COL = 0;              // S^T, then P^T (bf16) over its first 64
  static constexpr uint32_t DPT_COL = 128;           // dP^T
  static constexpr uint32_t DV_COL = 256;
  static constexpr uint32_t DK_COL = 256 + D;
  // dQ_e: in the dP^T columns at D = 128 (TMEM is full), so dP^T of the next
  // query block waits until dQ_e is read out; its own columns at D = 64
  static constexpr bool SHARED_DQ = D == 128;
  static constexpr uint32_t DQ_COL = SHARED_DQ ? DPT_COL : 256 + 2 * D;
  static constexpr int THREADS = 192;
  static_assert(NS >= 2, "stage ring needs two stages");
  static_assert(DQ_COL + D <= 512, "TMEM columns");
};

__device__ __forceinline__ int ld_acquire_gpu(const int32_t *p) {
  int32_t v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_gpu(int32_t *p, int32_t v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void red_add_v4(float *p, float a, float b, float c, float d) {
  asm volatile("red.relaxed.gpu.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a),
               "f"(b), "f"(c), "f"(d)
               : "memory");
}

__device__ __forceinline__ float4 ld_cg_v4(const float *p) {
  float4 v;
  asm volatile("ld.global.cg.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p)
               : "memory");
  return v;
}

// Drops a 128-byte line of the accumulator from L2 without writing it back
// (it is dead once the last part has read it).
__device__ __forceinline__ void discard_l2_line(const void *p) {
  asm volatile("discard.global.L2 [%0], 128;" ::"l"(p) : "memory");
}

// Bounded spin of one lane until *sem == want. False when the CTA is aborting
// or the limit ran out (then the timeout is recorded and the flag raised).
__device__ __forceinline__ bool wait_counter(const int32_t *sem, int32_t want, const WaitCtx &w,
                                             uint32_t counter) {
  if (ld_acquire_gpu(sem) == want) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 16; ++i) {
      __nanosleep(64);
      if (ld_acquire_gpu(sem) == want) return true;
    }
    if (*w.abort) return false;
    if (global_timer_ns() - t0 > w.limit) {
      if (atomicCAS(&g_status, 0u, 4u /* BSA_ERR_DEVICE_TIMEOUT */) == 0u) {
        g_status_detail[0] = w.role;
        g_status_detail[1] = kBarDqSem;
        g_status_detail[2] = counter;
        g_status_detail[3] = blockIdx.x;
      }
      *w.abort = 1;
      return false;
    }
  }
}

// Zeroes the dQ part counters and writes dq = 0 for the query rows whose
// block lists no key block (no part will ever reach them). One thread per
// padded query row of every batch*head.
template <int D>
__global__ void fused_init_kernel(const BwdParams p, long long rows_total, long long num_sems) {
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx < num_sems) p.dq_sem[idx] = 0;
  if (idx >= rows_total) return;
  const long long padded = static_cast<long long>(p.nqb) * kBwdBlock;
  const long long bh = idx / padded;
  const int i = static_cast<int>(idx - bh * padded);
  if (i >= p.n) return;
  const int qb = i / kBwdBlock;
  const int list = p.num_lists > 1 ? static_cast<int>(bh % p.heads) : 0;
  const long long r = static_cast<long long>(list) * p.nqb + qb;
  const int a = min(max(p.row_ptr[r], 0), p.nnz), b = min(max(p.row_ptr[r + 1], 0), p.nnz);
  if (b > a) return;
  const long long ib = bh / p.heads, ih = bh - ib * p.heads;
  uint4 *dst = reinterpret_cast<uint4 *>(p.dq + ib * p.dq_s[0] + ih * p.dq_s[1] + i * p.dq_s[2]);
#pragma unroll
  for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
}

// Warps 0-3: elementwise (thread = key row = TMEM lane for S^T, dP^T; thread
// = query row for the dQ part) and the dK/dV epilogue; warp 4: TMA producer
// (lane 0); warp 5: MMA issuer (lane 0).
template <int D>
__global__ void __launch_bounds__(192, 1)
    attn_bwd_fused_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v,
                          const __grid_constant__ CUtensorMap tm_do, const BwdParams p) {
  using C = FusedCfg<D>;
  constexpr int BN = kBwdBlock;
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t bar_st_full[C::NS], bar_st_empty[C::NS];
  __shared__ __align__(8) uint64_t bar_kv_full, bar_kv_empty, bar_s_full, bar_dp_full;
  __shared__ __align__(8) uint64_t bar_p_part[4], bar_ds_part[4];
  __shared__ __align__(8) uint64_t bar_dq_full, bar_dq_drained, bar_ds_free;
  __shared__ __align__(8) uint64_t bar_acc_full, bar_acc_empty, bar_final;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ int item_ring[kBwdItemN];
  __shared__ __align__(8) uint64_t bar_item_full[kBwdItemN], bar_item_empty[kBwdItemN];

  const uint32_t raw = smem_addr(dsmem);
  uint8_t *base = dsmem + (((raw + 1023u) & ~1023u) - raw);
  uint8_t *sK = base;
  uint8_t *sV = base + C::T;
  uint8_t *sStage = base + 2 * C::T;
  uint8_t *sDS = base + 2 * C::T + C::NS * C::STAGE;

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
    mbar_init(&bar_dq_full, 1);
    mbar_init(&bar_dq_drained, 4);
    mbar_init(&bar_ds_free, 1);
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

  // Item: (batch*head, key block) and its column of the transposed lists.
  auto decode = [&](int idx) {
    BwdItem it;
    const long long c = bwd_decode<false>(idx, true, p, VarlenTable{}, it);
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
        tma_load_5d(sK, &tm_k, &bar_kv_full, 0, it.blk * BN, 0, it.ih, it.ib);
        tma_load_5d(sV, &tm_v, &bar_kv_full, 0, it.blk * BN, 0, it.ih, it.ib);
        ++kvcount;
        for (int e = 0; e < it.len && ok; ++e) {
          const int qb = min(max(__ldg(p.row_idx + it.a + e), 0), it.nqb - 1);
          const uint32_t s = ring % C::NS;
          if (!(ok = lane_wait(&bar_st_empty[s], ((ring / C::NS) & 1u) ^ 1u, wc, kBarKvEmpty,
                               ring)))
            break;
          uint8_t *st = sStage + s * C::STAGE;
          mbar_arrive_expect_tx(&bar_st_full[s], 2 * C::T);
          tma_load_5d(st, &tm_q, &bar_st_full[s], 0, qb * BN, 0, it.ih, it.ib);
          tma_load_5d(st + C::T, &tm_do, &bar_st_full[s], 0, qb * BN, 0, it.ih, it.ib);
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
      // dK: A = dS^T K-major, B = Q MN-major; dQ: A = dS MN-major (bit 15),
      // B = K MN-major
      constexpr uint32_t idesc_dk = idesc_bf16_f32(128, D, true);
      constexpr uint32_t idesc_dq = idesc_bf16_f32(128, D, true) | (1u << 15);
      constexpr uint32_t kHi = (1024u >> 4) | (1u << 14) | (2u << 29);
      constexpr uint32_t kLboK = 1u << 16;
      constexpr uint32_t kLboMN = static_cast<uint32_t>(BN * 128 / 16) << 16;
      const uint32_t k_lo = (smem_addr(sK) >> 4) | kLboK;
      const uint32_t v_lo = (smem_addr(sV) >> 4) | kLboK;
      const uint32_t k_mn = (smem_addr(sK) >> 4) | kLboMN;
      const uint32_t ds_k = (smem_addr(sDS) >> 4) | kLboK;
      const uint32_t ds_mn = (smem_addr(sDS) >> 4) | kLboMN;
      const uint32_t st_base = smem_addr(sStage) >> 4;
      uint32_t ring = 0, kvcount = 0, pcount = 0, items = 0, blocks = 0;
      bool ok = true;
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
      // waits until the dQ part of block b (this CTA's count) has been read
      // out of TMEM
      auto wait_drained = [&](uint32_t b) -> bool {
        if (!lane_wait(&bar_dq_drained, b & 1u, wc, kBarSFree, b)) return false;
        tc_fence_after();
        return true;
      };
      auto issue_dp = [&](uint32_t r) -> bool {  // dP^T = V dO^T (slot already waited)
        if (C::SHARED_DQ && blocks > 0 && !wait_drained(blocks - 1)) return false;
        const uint32_t s = r % C::NS;
        const uint32_t do_k = (st_base + s * (C::STAGE >> 4) + (C::T >> 4)) | kLboK;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (BN * 128 >> 4) + (kk & 3) * 2;
          mma_ss_lh(tmem + C::DPT_COL, v_lo + off, kHi, do_k + off, kHi, idesc_ss,
                    kk > 0 ? 1u : 0u);
        }
        mma_commit(&bar_dp_full);
        return true;
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
        if (!(ok = issue_dp(ring))) break;
        bool first = true;
        for (int e = 0; e < it.len; ++e) {
          const uint32_t s = ring % C::NS;
          const uint32_t q_mn = (st_base + s * (C::STAGE >> 4)) | kLboMN;
          const uint32_t do_mn = (st_base + s * (C::STAGE >> 4) + (C::T >> 4)) | kLboMN;
          if (first && items > 0) {  // the previous item's epilogue has read dV, dK
            if (!(ok = lane_wait(&bar_acc_empty, (items - 1) & 1u, wc, kBarOEmpty, items))) break;
            tc_fence_after();
          }
          // dV += P^T dO_e as the elementwise warps hand P^T over
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
          // the S^T columns are free once the dV MMAs that read P^T_e ran
          if (e + 1 < it.len && !(ok = issue_s(ring + 1))) break;
          // dK += dS^T Q_e as dS^T lands in shared memory, part by part
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            if (!(ok = lane_wait(&bar_ds_part[h], pcount & 1u, wc, kBarPFull, pcount))) break;
            tc_fence_after();
#pragma unroll
            for (int kk = h * BN / 64; kk < (h + 1) * BN / 64; ++kk) {
              const uint32_t off = (kk >> 2) * (BN * 128 >> 4) + (kk & 3) * 2;
              mma_ss_lh(tmem + C::DK_COL, ds_k + off, kHi, q_mn + kk * (16 * 128 >> 4), kHi,
                        idesc_dk, (!first || kk > 0) ? 1u : 0u);
            }
          }
          if (!ok) break;
          mma_commit(&bar_st_empty[s]);  // Q_e and dO_e read for the last time
          // dQ_e = dS_e K over all key rows (every part has landed)
          if (!C::SHARED_DQ && blocks > 0 && !(ok = wait_drained(blocks - 1))) break;
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk)
            mma_ss_lh(tmem + C::DQ_COL, ds_mn + kk * (16 * 128 >> 4), kHi,
                      k_mn + kk * (16 * 128 >> 4), kHi, idesc_dq, kk > 0 ? 1u : 0u);
          mma_commit(&bar_dq_full);
          mma_commit(&bar_ds_free);  // dS^T read by dK and dQ
          ++pcount;
          ++ring;
          ++blocks;
          first = false;
          if (e + 1 < it.len && !(ok = issue_dp(ring))) break;
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
    const int r = warp * 32 + lane;  // TMEM lane: key row (S^T, dP^T), query row (dQ part)
    const uint32_t lane_tmem = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float sl2 = p.scale_log2;
    // this thread's dS^T row in shared memory: 128-byte swizzled rows of 64
    // query columns, two column halves 16 KB apart (the layout TMA gives Q)
    uint8_t *const ds_row = sDS + (r >> 3) * 1024 + (r & 7) * 128;
    uint32_t scount = 0, dcount = 0, acount = 0, blocks = 0;
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
      const long long ib = it.ib, ih = it.ih;
      __nv_bfloat16 *const dk_row = p.dk + ib * p.dk_s[0] + ih * p.dk_s[1] + key * p.dk_s[2];
      __nv_bfloat16 *const dv_row = p.dv + ib * p.dv_s[0] + ih * p.dv_s[1] + key * p.dv_s[2];
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
      const int list = p.num_lists > 1 ? it.ih : 0;
      const long long bhq = static_cast<long long>(it.ib) * p.heads + it.ih;
      for (int e = 0; e < it.len; ++e) {
        const int qb = min(max(__ldg(p.row_idx + it.a + e), 0), it.nqb - 1);
        const float *lse_g = p.lse2 + it.lbase + static_cast<long long>(qb) * BN;
        const float *del_g = p.delta + it.lbase + static_cast<long long>(qb) * BN;
        if (!(ok = warp_wait(&bar_s_full, scount & 1u, wc, kBarSFull, scount))) break;
        tc_fence_after();
        // P^T (fp32, kept for dS^T), handed over as bf16 in four parts while
        // dP^T is still being computed
        float pf[BN];
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t sr[32];
          tmem_ld32(lane_tmem + C::ST_COL + c * 32, sr);
          tmem_wait_ld();
          reg_fence32(sr);
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float4 l4 = __ldg(reinterpret_cast<const float4 *>(lse_g + c * 32) + (i >> 1));
            const float la = (i & 1) ? l4.z : l4.x, lb = (i & 1) ? l4.w : l4.y;
            pf[c * 32 + 2 * i] = ex2_approx(fmaf(__uint_as_float(sr[2 * i]), sl2, -la));
            pf[c * 32 + 2 * i + 1] = ex2_approx(fmaf(__uint_as_float(sr[2 * i + 1]), sl2, -lb));
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
        // the dK and dQ MMAs of the previous block have read dS^T
        if (blocks > 0) {
          if (!(ok = warp_wait(&bar_ds_free, (blocks - 1) & 1u, wc, kBarSFree, blocks))) break;
        }
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t dr[32];
          tmem_ld32(lane_tmem + C::DPT_COL + c * 32, dr);
          tmem_wait_ld();
          reg_fence32(dr);
          uint32_t g16[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float4 d4 = __ldg(reinterpret_cast<const float4 *>(del_g + c * 32) + (i >> 1));
            const float da = (i & 1) ? d4.z : d4.x, db = (i & 1) ? d4.w : d4.y;
            g16[i] = pack_bf16x2(pf[c * 32 + 2 * i] * (__uint_as_float(dr[2 * i]) - da),
                                 pf[c * 32 + 2 * i + 1] * (__uint_as_float(dr[2 * i + 1]) - db));
          }
          // query columns [32c, 32c + 32): four 16-byte units of this row,
          // in column half c / 2, swizzled by the row within its 8-row group
          uint8_t *half = ds_row + (c >> 1) * (BN * 128);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const int u = ((c & 1) * 4 + v) ^ (r & 7);
            *reinterpret_cast<uint4 *>(half + u * 16) =
                make_uint4(g16[4 * v], g16[4 * v + 1], g16[4 * v + 2], g16[4 * v + 3]);
          }
          fence_proxy_async_smem();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar_ds_part[c]);
        }
        // dQ part of query block qb from this key block: read it out of TMEM
        // (thread = query row qb * 128 + r), free the columns, then add it in
        // the row's order
        if (!(ok = warp_wait(&bar_dq_full, blocks & 1u, wc, kBarODone, blocks))) break;
        tc_fence_after();
        float g[D];
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(lane_tmem + C::DQ_COL + c * 32, v);
          tmem_wait_ld();
          reg_fence32(v);
#pragma unroll
          for (int i = 0; i < 32; ++i) g[c * 32 + i] = __uint_as_float(v[i]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_dq_drained);
        ++blocks;
        // this key block's position among the row's keys, and the row length
        const long long rrow = static_cast<long long>(list) * p.nqb + qb;
        const int ra = min(max(__ldg(p.row_ptr + rrow), 0), p.nnz);
        const int rb = min(max(__ldg(p.row_ptr + rrow + 1), 0), p.nnz);
        const int m = max(rb - ra, 1);
        const int pos = min(max(__ldg(p.row_pos + it.a + e), 0), m - 1);
        const int qrow = qb * BN + r;
        const bool qstore = qrow < it.n;
        __nv_bfloat16 *const dq_row =
            p.dq + ib * p.dq_s[0] + ih * p.dq_s[1] + static_cast<long long>(qrow) * p.dq_s[2];
        float *const acc = p.dq_acc + ((bhq * p.nqb + qb) * BN + r) * static_cast<long long>(D);
        int32_t *const sem = p.dq_sem + (bhq * p.nqb + qb) * 4 + warp;
        if (m > 1) {
          bool got = true;
          if (lane == 0) got = wait_counter(sem, pos, wc, blocks);
          if (!(ok = __all_sync(0xffffffffu, __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0)))
            break;
        }
        if (pos + 1 < m) {  // not the last part: into the accumulator
          if (pos == 0) {
#pragma unroll
            for (int c = 0; c < D / 4; ++c)
              *reinterpret_cast<float4 *>(acc + 4 * c) =
                  make_float4(g[4 * c], g[4 * c + 1], g[4 * c + 2], g[4 * c + 3]);
          } else {
#pragma unroll
            for (int c = 0; c < D / 4; ++c)
              red_add_v4(acc + 4 * c, g[4 * c], g[4 * c + 1], g[4 * c + 2], g[4 * c + 3]);
          }
          __threadfence();
          __syncwarp();
          if (lane == 0) st_release_gpu(sem, pos + 1);
        } else {  // the last part: the sum, scaled, as bf16
          if (m > 1) {
#pragma unroll
            for (int c = 0; c < D / 4; ++c) {
              const float4 a = ld_cg_v4(acc + 4 * c);
              g[4 * c] += a.x;
              g[4 * c + 1] += a.y;
              g[4 * c + 2] += a.z;
              g[4 * c + 3] += a.w;
            }
#pragma unroll
            for (int c = 0; c < D / 32; ++c) discard_l2_line(acc + 32 * c);
          }
          if (qstore) {
            const float mul = p.scale;
            uint4 *o4 = reinterpret_cast<uint4 *>(dq_row);
#pragma unroll
            for (int c = 0; c < D / 8; ++c)
              o4[c] = make_uint4(pack_bf16x2(g[8 * c] * mul, g[8 * c + 1] * mul),
                                 pack_bf16x2(g[8 * c + 2] * mul, g[8 * c + 3] * mul),
                                 pack_bf16x2(g[8 * c + 4] * mul, g[8 * c + 5] * mul),
                                 pack_bf16x2(g[8 * c + 6] * mul, g[8 * c + 7] * mul));
          }
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

}  // namespace bsa
