// The GEMM of gemm.cuh on a pair of SMs (a cluster of two CTAs and the
// tensor cores' two-SM mode, cta_group::2): one 256 x 256 output tile per
// pair, each CTA holding 128 of its rows in its own tensor memory. Each CTA
// loads its own 128 rows of A and HALF of B (128 of the 256 columns); one
// MMA instruction, issued by the pair's leader (rank 0), multiplies the
// pair's A (256 rows) by the whole B tile. Per SM and K step, shared memory
// takes 32 KB of copies instead of the single-SM kernel's 48 KB, and L2
// serves half as much of B.
//
// Protocol (rank 0 = leader, rank 1 = follower):
//   full[s]   leader only: the leader's producer posts the pair's bytes; the
//             copies of both CTAs complete on it (the follower's copies name
//             the leader's barrier through its cluster address).
//   empty[s]  both: the leader's MMA commit arrives on both (multicast).
//   tfull[a]  both: the leader commits a finished accumulator to both.
//   tempty[a] leader only: all eight epilogue warps of the pair arrive (the
//             follower's through the cluster address).
// Both CTAs walk the same tile list. Every mbarrier wait is bounded as in the
// other kernels; cluster barriers after the barrier set-up and before the
// tensor memory is freed keep either CTA from touching the other's shared
// memory after it has left.
#pragma once

#include "gemm.cuh"

namespace bpt {

constexpr int GP_BM = 256;  // rows of a pair tile (128 per CTA)
constexpr int GP_BN = 256;
constexpr int GP_STAGES = 6;
constexpr int GP_A_BYTES = 128 * GEMM_BK * 2;           // this CTA's 128 rows: 16 KB
constexpr int GP_B_BYTES = GEMM_BK * (GP_BN / 2) * 2;   // this CTA's 128 columns: two [64 k][64 n] boxes, 16 KB
constexpr int GP_STAGE_BYTES = GP_A_BYTES + GP_B_BYTES;
constexpr int GP_GROUP_M = 8;                            // raster: 8 pair tiles (2048 rows) share B in L2
constexpr int GP_SMEM_BYTES = GP_STAGES * GP_STAGE_BYTES + 1024 + 256;

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Cluster address of the same shared-memory location in CTA `rank`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// A tile copy of this CTA whose completion counts on the pair leader's barrier.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster, int c0,
                                                 int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void mma_bf16_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                 uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on the barrier at this shared-memory offset in both CTAs of the
// pair when the leader's earlier MMAs have completed.
__device__ __forceinline__ void mma_commit_pair(uint32_t bar) {
  const uint16_t mask = 0x3;
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
               "h"(mask)
               : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void pair_tile_coords(int t, int m_tiles, int n_tiles, int& mt, int& nt) {
  const int group_size = GP_GROUP_M * n_tiles;
  const int group = t / group_size;
  const int first_m = group * GP_GROUP_M;
  const int gm = min(GP_GROUP_M, m_tiles - first_m);
  const int r = t - group * group_size;
  mt = first_m + r % gm;
  nt = r / gm;
}

// args.m_tiles / n_tiles count 256 x 256 pair tiles; grid = 2 x pairs.
// Operand layouts as in gemm_bf16_tcgen05: A_MN = 1, A stored [K, M] (this
// CTA's 128 rows as two [64 k][64 m] boxes), else [M, K] (one [128 m][64 k]
// box); B_MN = 1, B stored [K, N] (this CTA's 128 columns as two [64 k][64 n]
// boxes), else [N, K] (one [128 n][64 k] box).
template <int MODE, int A_MN = 0, int B_MN = 1>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(GEMM_THREADS, 1)
    gemm_pair_tcgen05(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + GP_STAGES * GP_STAGE_BYTES);
  const uint32_t full0 = smem_addr(bars);
  const uint32_t empty0 = smem_addr(bars + GP_STAGES);
  const uint32_t tfull0 = smem_addr(bars + 2 * GP_STAGES);
  const uint32_t tempty0 = smem_addr(bars + 2 * GP_STAGES + 2);
  const uint32_t mma_done = smem_addr(bars + 2 * GP_STAGES + 4);  // both: the leader's last commit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * GP_STAGES + 5);
  const Abort abort_flag{reinterpret_cast<volatile int*>(bars + 2 * GP_STAGES + 6), args.status};

  const int warp = warp_id();
  const int lane = lane_id();
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const uint32_t smem_base = smem_addr(smem);

  if (warp == 0 && lane == 0) {
    for (int i = 0; i < GP_STAGES; ++i) {
      mbar_init(full0 + 8 * i, 1);
      mbar_init(empty0 + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(tfull0 + 8 * i, 1);
      mbar_init(tempty0 + 8 * i, 8);
    }
    mbar_init(mma_done, 1);
    *abort_flag.flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_addr(tmem_slot), GEMM_TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers exist before either signals the other
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int pairs = gridDim.x / 2;
  const int pair = blockIdx.x / 2;
  const int num_tiles = args.m_tiles * args.n_tiles;
  const int k_blocks = args.K / GEMM_BK;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, last_parity = 0;
      const uint32_t full_leader0 = mapa_shared(full0, 0);
      for (int t = pair; t < num_tiles; t += pairs) {
        int mt, nt;
        pair_tile_coords(t, args.m_tiles, args.n_tiles, mt, nt);
        const int m0 = mt * GP_BM + (int)rank * 128;        // this CTA's rows
        const int n0 = nt * GP_BN + (int)rank * (GP_BN / 2);  // this CTA's half of B
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1, abort_flag)) goto producer_done;
          if (leader) mbar_arrive_expect_tx(full0 + 8 * stage, 2 * GP_STAGE_BYTES);
          const uint32_t fb = full_leader0 + 8 * stage;
          const uint32_t sa = smem_base + stage * GP_STAGE_BYTES;
          if constexpr (A_MN) {
#pragma unroll
            for (int j = 0; j < 128 / 64; ++j)
              tma_load_2d_pair(sa + j * GEMM_B_BOX_BYTES, &tmA, fb, m0 + 64 * j, kb * GEMM_BK);
          } else {
            tma_load_2d_pair(sa, &tmA, fb, kb * GEMM_BK, m0);
          }
          if constexpr (B_MN) {
#pragma unroll
            for (int j = 0; j < GP_BN / 2 / 64; ++j)
              tma_load_2d_pair(sa + GP_A_BYTES + j * GEMM_B_BOX_BYTES, &tmB, fb, n0 + 64 * j, kb * GEMM_BK);
          } else {
            tma_load_2d_pair(sa + GP_A_BYTES, &tmB, fb, kb * GEMM_BK, n0);
          }
          issued |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == GP_STAGES) { stage = 0; phase ^= 1; }
        }
      }
    producer_done:
      // never leave with copies still landing: the leader waits for the pair's
      // last copies on its full barriers; the follower for the leader's last
      // MMA commits, which come after every copy the MMAs read
      for (int i = 0; i < GP_STAGES; ++i)
        if (issued & (1u << i)) {
          volatile int dummy = 0;
          if (leader)
            mbar_wait(full0 + 8 * i, (last_parity >> i) & 1u, Abort{&dummy, args.status});
          else
            mbar_wait(empty0 + 8 * i, (last_parity >> i) & 1u, Abort{&dummy, args.status});
        }
    }
  } else if (warp == 1) {
    if (leader && lane == 0) {
      // ------------------------------------------------------------ MMA issuer (leader)
      const uint32_t idesc = idesc_bf16_f32(GP_BM, GP_BN, A_MN, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      for (int t = pair; t < num_tiles; t += pairs, ++it) {
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!mbar_wait(tempty0 + 8 * acc, acc_phase ^ 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + acc * GEMM_BN;
        bool ok = true;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(full0 + 8 * stage, phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_base + stage * GP_STAGE_BYTES;
          const uint32_t sb = sa + GP_A_BYTES;
#pragma unroll
          for (int kk = 0; kk < GEMM_BK / 16; ++kk) {
            const uint64_t adesc = A_MN ? smem_desc_sw128(sa + kk * 16 * 128, GEMM_B_BOX_BYTES, 1024)
                                        : smem_desc_sw128(sa + kk * 32, 16, 1024);
            const uint64_t bdesc = B_MN ? smem_desc_sw128(sb + kk * 16 * 128, GEMM_B_BOX_BYTES, 1024)
                                        : smem_desc_sw128(sb + kk * 32, 16, 1024);
            mma_bf16_ss_pair(d, adesc, bdesc, idesc, (kb | kk) != 0);
          }
          mma_commit_pair(empty0 + 8 * stage);
          if (++stage == GP_STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        mma_commit_pair(tfull0 + 8 * acc);
      }
      mma_commit_pair(mma_done);  // on every path, so that both CTAs can free their tensor memory
    }
  } else {
    // -------------------------------------------------------------- epilogue (both CTAs)
    const int quarter = warp & 3;
    const uint32_t tempty_leader0 = mapa_shared(tempty0, 0);
    int it = 0;
    for (int t = pair; t < num_tiles; t += pairs, ++it) {
      int mt, nt;
      pair_tile_coords(t, args.m_tiles, args.n_tiles, mt, nt);
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      if (!warp_wait(tfull0 + 8 * acc, acc_phase, abort_flag)) break;
      tc_fence_after();
      const int row = mt * GP_BM + (int)rank * 128 + quarter * 32 + lane;
      const uint32_t taddr = tmem_base + acc * GEMM_BN + ((uint32_t)(quarter * 32) << 16);
#pragma unroll 1
      for (int c = 0; c < GP_BN / 32; ++c) {
        uint32_t r[32];
        tmem_load32(taddr + c * 32, r);
        const int col = nt * GP_BN + c * 32;
        if (row < args.M && col < args.N) {
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
          gemm_epilogue<MODE>(args, row, col, v);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader0 + 8 * acc);
    }
  }

  // both CTAs free their tensor memory once the leader's MMAs (which write
  // both) have completed, and neither leaves while the other may still
  // signal its barriers
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) {
      volatile int dummy = 0;
      mbar_wait(mma_done, 0, Abort{&dummy, args.status});
    }
    __syncwarp();
  }
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, GEMM_TMEM_COLS);
  }
}

}  // namespace bpt
