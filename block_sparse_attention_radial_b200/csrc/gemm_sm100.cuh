// Dense bf16 GEMM for sm_100a: D[M, N] = A[M, K] B[K, N] (+ bias[N]), fp32
// accumulation in tensor memory, bf16 output. It serves the linear layers
// around the attention (the "Radial Attention" skill page's RadialAttention
// module, Step 2: q_proj, k_proj, v_proj, out_proj, and their gradients).
//
// Operands are row-major matrices read through TMA in either orientation:
//   A K-major:  stored [M][K] (K contiguous);  A MN-major: stored [K][M].
//   B K-major:  stored [N][K] (an nn.Linear weight [out, in]);
//   B MN-major: stored [K][N].
// Every tile lands in shared memory with 128-byte swizzling in the layout the
// MMA descriptors name: a K-major tile as [rows][64 K] (one 128-byte row per
// M or N index), an MN-major tile as 64-wide MN chunks of [64 K rows][64 MN].
//
// Persistent kernel, one CTA per SM, 128 x 256 output tiles, 64-deep K blocks
// through a 4-stage ring (48 KB per stage). Warp roles (192 threads):
//   warp 0      TMA producer (one lane)
//   warp 1      MMA issuer (one lane): 4 x tcgen05.mma M=128 N=256 K=16 per
//               K block into one of two TMEM accumulators (2 x 256 columns)
//   warps 2-5   epilogue: thread = output row = TMEM lane; loads 32 columns
//               at a time, adds the bias, rounds to bf16, stores 16-byte
//               vectors; the accumulator is released for the tile after next
// so that a tile's epilogue overlaps the next tile's MMAs. Tiles are taken
// in groups of 8 column blocks (all row blocks of a group before the next
// group), so the A and B tiles that the CTAs running at the same time read
// stay in L2. Every wait is bounded like the attention kernels' waits.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "attn_fwd_sm100.cuh"

namespace bsa {

struct GemmParams {
  int M, N, K;
  __nv_bfloat16 *d;
  long long ldd;               // row stride of D (elements)
  const __nv_bfloat16 *bias;   // [N] or null
  int tiles_m, tiles_n, total_tiles, k_blocks;
  unsigned long long wait_limit_ns;
};

struct GemmCfg {
  static constexpr int BM = 128, BN = 256, BK = 64;
  static constexpr int A_BYTES = BM * BK * 2;           // 16 KB
  static constexpr int B_BYTES = BN * BK * 2;           // 32 KB
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int NS = 4;
  static constexpr int DSMEM = 1024 + NS * STAGE_BYTES;
  static constexpr int CHUNK_BYTES = BK * 128;          // one 64-wide MN chunk of 64 K rows
  static constexpr int GROUP_N = 8;                     // column blocks per raster group
  static constexpr uint32_t TMEM_COLS = 512;            // two 256-column accumulators
  static constexpr int THREADS = 192;
};

// Tile t -> (row block, column block): groups of GROUP_N column blocks, every
// row block of a group before the next group, column fastest inside it.
__device__ __forceinline__ void gemm_tile_coords(int t, const GemmParams &p, int &mb, int &nb) {
  const int per_group = GemmCfg::GROUP_N * p.tiles_m;
  const int g = t / per_group;
  const int r = t - g * per_group;
  const int gn = min(GemmCfg::GROUP_N, p.tiles_n - g * GemmCfg::GROUP_N);
  nb = g * GemmCfg::GROUP_N + r % gn;
  mb = r / gn;
}

template <bool A_MN, bool B_MN>
__global__ void __launch_bounds__(192, 1)
    gemm_bf16_sm100_kernel(const __grid_constant__ CUtensorMap tm_a,
                           const __grid_constant__ CUtensorMap tm_b, const GemmParams p) {
  using C = GemmCfg;
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t bar_full[C::NS], bar_empty[C::NS];
  __shared__ __align__(8) uint64_t bar_acc_full[2], bar_acc_empty[2], bar_final;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const uint32_t raw = smem_addr(dsmem);
  uint8_t *base = dsmem + (((raw + 1023u) & ~1023u) - raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&bar_full[s], 1);
      mbar_init(&bar_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar_acc_full[b], 1);
      mbar_init(&bar_acc_empty[b], 4);  // one arrival per epilogue warp
    }
    mbar_init(&bar_final, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  WaitCtx wc{&abort_flag, p.wait_limit_ns, 0};

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      wc.role = kRoleProducer;
      tma_prefetch_desc(&tm_a);
      tma_prefetch_desc(&tm_b);
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < p.total_tiles; t += gridDim.x) {
        int mb, nb;
        gemm_tile_coords(t, p, mb, nb);
        const int m0 = mb * C::BM, n0 = nb * C::BN;
        for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
          const uint32_t s = it % C::NS;
          if (!(ok = lane_wait(&bar_empty[s], ((it / C::NS) & 1u) ^ 1u, wc, kBarKvEmpty, it)))
            break;
          uint8_t *sa = base + s * C::STAGE_BYTES;
          uint8_t *sb = sa + C::A_BYTES;
          const int k0 = kb * C::BK;
          mbar_arrive_expect_tx(&bar_full[s], C::STAGE_BYTES);
          if (A_MN) {
#pragma unroll
            for (int c = 0; c < C::BM / 64; ++c)
              tma_load_2d(sa + c * C::CHUNK_BYTES, &tm_a, &bar_full[s], m0 + 64 * c, k0);
          } else {
            tma_load_2d(sa, &tm_a, &bar_full[s], k0, m0);
          }
          if (B_MN) {
#pragma unroll
            for (int c = 0; c < C::BN / 64; ++c)
              tma_load_2d(sb + c * C::CHUNK_BYTES, &tm_b, &bar_full[s], n0 + 64 * c, k0);
          } else {
            tma_load_2d(sb, &tm_b, &bar_full[s], k0, n0);
          }
        }
      }
      // copies still in flight complete before the CTA exits
      WaitCtx drain{&abort_flag, p.wait_limit_ns, kRoleProducer};
      int zero = 0;
      drain.abort = &zero;
      const uint32_t first = it > C::NS ? it - C::NS : 0;
      for (uint32_t r = first; r < it; ++r)
        wait_bounded(&bar_full[r % C::NS], (r / C::NS) & 1u, drain, kBarKvFull, r);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      wc.role = kRoleMma;
      // M = 128, N = 256, bf16 x bf16 -> fp32; bit 15 / 16: A / B MN-major
      constexpr uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((A_MN ? 1u : 0u) << 15) |
                                 ((B_MN ? 1u : 0u) << 16) | ((C::BN >> 3) << 17) |
                                 ((C::BM >> 4) << 24);
      // high half of every descriptor: stride byte offset 1024 (8 rows of
      // 128 bytes), version 1, 128-byte swizzling
      constexpr uint32_t kHi = (1024u >> 4) | (1u << 14) | (2u << 29);
      // low half: start address >> 4 | leading byte offset >> 4 << 16; the
      // leading offset is the distance between 64-wide MN chunks for an
      // MN-major tile (unused for a K-major one)
      constexpr uint32_t kLboMN = static_cast<uint32_t>(C::CHUNK_BYTES >> 4) << 16;
      constexpr uint32_t kLboK = 1u << 16;
      const uint32_t ring_base = smem_addr(base) >> 4;
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < p.total_tiles; t += gridDim.x, ++tcount) {
        const uint32_t buf = tcount & 1u;
        if (tcount >= 2 &&
            !(ok = lane_wait(&bar_acc_empty[buf], ((tcount >> 1) - 1) & 1u, wc, kBarOEmpty,
                             tcount)))
          break;
        tc_fence_after();
        const uint32_t acc = tmem + buf * C::BN;
        for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
          const uint32_t s = it % C::NS;
          if (!(ok = lane_wait(&bar_full[s], (it / C::NS) & 1u, wc, kBarKvFull, it))) break;
          tc_fence_after();
          const uint32_t a_lo = (ring_base + s * (C::STAGE_BYTES >> 4)) | (A_MN ? kLboMN : kLboK);
          const uint32_t b_lo =
              (ring_base + s * (C::STAGE_BYTES >> 4) + (C::A_BYTES >> 4)) | (B_MN ? kLboMN : kLboK);
#pragma unroll
          for (int kk = 0; kk < C::BK / 16; ++kk) {
            // K step of 16: 32 bytes along a K-major row, 16 rows (2 KB) down
            // an MN-major chunk
            const uint32_t a_off = A_MN ? kk * (16 * 128 >> 4) : kk * 2;
            const uint32_t b_off = B_MN ? kk * (16 * 128 >> 4) : kk * 2;
            mma_ss_lh(acc, a_lo + a_off, kHi, b_lo + b_off, kHi, idesc,
                      (kb > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&bar_empty[s]);
        }
        if (!ok) break;
        mma_commit(&bar_acc_full[buf]);
      }
      mma_commit(&bar_final);
      WaitCtx drain{&abort_flag, p.wait_limit_ns, kRoleMma};
      int zero = 0;
      drain.abort = &zero;
      wait_bounded(&bar_final, 0, drain, kBarFinal, tcount);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    wc.role = kRoleSoftmax;
    const int q = warp & 3;  // TMEM lane quarter of this warp
    const uint32_t lane_tmem = tmem + (static_cast<uint32_t>(q * 32) << 16);
    uint32_t tcount = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.total_tiles; t += gridDim.x, ++tcount) {
      int mb, nb;
      gemm_tile_coords(t, p, mb, nb);
      const uint32_t buf = tcount & 1u;
      if (!(ok = warp_wait(&bar_acc_full[buf], (tcount >> 1) & 1u, wc, kBarODone, tcount))) break;
      tc_fence_after();
      const int row = mb * C::BM + q * 32 + lane;
      const int n0 = nb * C::BN;
      __nv_bfloat16 *drow = p.d + static_cast<long long>(row) * p.ldd + n0;
#pragma unroll 1
      for (int c = 0; c < C::BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(lane_tmem + buf * C::BN + c * 32, r);
        tmem_wait_ld();
        reg_fence32(r);
        const int col0 = n0 + c * 32;
        if (col0 >= p.N) break;  // warp-uniform
        if (p.bias) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (col0 + i < p.N)
              r[i] = __float_as_uint(__uint_as_float(r[i]) + __bfloat162float(p.bias[col0 + i]));
        }
        if (row < p.M) {
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            if (col0 + 8 * v4 >= p.N) break;
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(r[8 * v4 + 0]), __uint_as_float(r[8 * v4 + 1]));
            w.y = pack_bf16x2(__uint_as_float(r[8 * v4 + 2]), __uint_as_float(r[8 * v4 + 3]));
            w.z = pack_bf16x2(__uint_as_float(r[8 * v4 + 4]), __uint_as_float(r[8 * v4 + 5]));
            w.w = pack_bf16x2(__uint_as_float(r[8 * v4 + 6]), __uint_as_float(r[8 * v4 + 7]));
            *reinterpret_cast<uint4 *>(drow + c * 32 + 8 * v4) = w;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_acc_empty[buf]);
    }
    (void)ok;
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace bsa
