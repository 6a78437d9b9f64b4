// The blockwise attention of attention.cuh (Eq. 3 and Algorithm 1 steps 4-10
// of the BPT paper review) on a pair of SMs: a cluster of two CTAs shares
// every key/value tile, and the tensor cores run in their two-SM mode
// (cta_group::2), each MMA producing 256 query rows, 128 in each CTA's tensor
// memory. Each CTA loads half of each K tile (64 of its 128 keys) and half of
// each V tile (64 of its 128 head columns); the MMAs read the other half from
// the peer. Per SM, the S MMA's shared-memory reads fall from 8 KB to 6 KB
// per 64 tensor clocks and the K/V copies from 64 KB to 32 KB per key/value
// tile; the single-SM kernel's S MMAs sit at the shared memory's bandwidth.
//
// A cluster covers four consecutive 128-row query tiles of one head of one
// sequence: rank 0 holds tiles 0 and 3, rank 1 tiles 1 and 2. MMA slot q
// multiplies the pair's tiles in slot q (slot 0: tiles 0 and 1, slot 1: tiles
// 3 and 2), so that the two tiles of a slot need key/value ranges that differ
// by at most one tile when causal; the slot runs over the longer range, and
// the shorter tile's extra keys are masked (weight exactly 0).
//
// Roles per CTA (as in attention.cuh): warp 0 copies Q (both tiles, once)
// and its halves of the K/V tiles into a ring of 16 KB slots; one thread of
// the leader's (rank 0) warp 1 issues the MMAs for the pair; warpgroups 1 and
// 2 run the softmax of slot 0 and slot 1, one row per thread, over the CTA's
// own tensor memory. Barriers:
//   q_full, ring_full[i]  leader only: the leader posts the pair's bytes and
//                         both CTAs' copies complete on it;
//   ring_empty[i], s_full[q], o_done[q], mma_done
//                         both: the leader's MMA commits arrive on both;
//   p_full[q]             leader only: the 4 softmax warps of slot q in each
//                         CTA arrive (8 arrivals), the follower's through the
//                         cluster address.
// Every mbarrier wait is bounded (kWaitTimeoutNs, then BPT_ERR_TIMEOUT);
// cluster barriers after the set-up and before the tensor memory is freed
// keep either CTA from signalling the other after it has left.
#pragma once

#include "attention.cuh"
#include "gemm_pair.cuh"

namespace bpt {

// Warpgroup 0's register budget in this kernel (the leader's MMA issuer keeps
// the cluster addresses of its barriers): 128 x 64 + 256 x ATT_REGS_SOFTMAX =
// 63488 <= 384 x ATT_REGS_LAUNCH.
constexpr int ATT_PAIR_REGS_CONTROL = 64;
static_assert(ATT_THREADS * ATT_REGS_LAUNCH >= 128 * ATT_PAIR_REGS_CONTROL + 256 * ATT_REGS_SOFTMAX,
              "register split exceeds the block's launch allocation");

struct AttnPairCfg {
  static constexpr int DH = 128;
  static constexpr int Q_BYTES = ATT_BM * DH * 2;       // one query tile: 32 KB
  static constexpr int Q_ATOM = 128 * 128;              // [128 rows][64 bf16] box: 16 KB
  static constexpr int K_ATOM = 64 * 128;               // [64 keys][64 bf16] box: 8 KB
  static constexpr int SLOT_BYTES = 16384;              // a K half (two K atoms) or a V half (one box)
  static constexpr int RING = 10;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_RING = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_BAR = OFF_RING + RING * SLOT_BYTES;
  static constexpr int USED = OFF_BAR + 512 + 1024;
  static constexpr int SMEM_BYTES = USED;
  static_assert(USED <= 232448, "shared memory budget");
};

struct AttnPairArgs {
  int s, heads, causal;
  int beta0;
  int t_start, t_len;
  int n_quads;       // ceil(t_len / 512): clusters per (sequence, head)
  __nv_bfloat16* o;  // output rows: (beta - beta0) * t_len + (t - t_start)
  long long ldo;
  float scale_log2;
  int* status;
};

__device__ __forceinline__ void mma_bf16_ts_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                                 uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster, int c0,
                                                 int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// Query tile (within the cluster's four) held by `rank` in `slot`.
__host__ __device__ __forceinline__ int pair_tile_of(int rank, int slot) {
  return rank == 0 ? (slot == 0 ? 0 : 3) : (slot == 0 ? 1 : 2);
}

// tmQ: box [128 rows][64 cols]; tmK: box [64 rows][64 cols]; tmV: box
// [128 rows][64 cols]; all over [b, s, h] bf16.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(ATT_THREADS, 1)
    attention_pair_tcgen05(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, const AttnPairArgs args) {
  using C = AttnPairCfg;
  constexpr int DH = C::DH;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  const uint32_t q_full = smem_addr(bars + 0);
  const uint32_t s_full0 = smem_addr(bars + 1);   // [2] per slot
  const uint32_t p_full0 = smem_addr(bars + 3);   // [2] per slot
  const uint32_t o_done0 = smem_addr(bars + 5);   // [2] per slot
  const uint32_t mma_done = smem_addr(bars + 9);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 10);
  const Abort abort_flag{reinterpret_cast<volatile int*>(bars + 11), args.status};
  const uint32_t ring_full0 = smem_addr(bars + 12);             // [RING]
  const uint32_t ring_empty0 = smem_addr(bars + 12 + C::RING);  // [RING]

  const int warp = warp_id();
  const int lane = lane_id();
  const uint32_t sbase = smem_addr(smem);
  const int rank = (int)cluster_ctarank();
  const bool leader = rank == 0;

  // ------------------------------------------------------------ geometry
  // as attention.cuh, with a cluster of two CTAs per four query tiles: x / 2
  // enumerates (head, quad) in groups of ATT_HEAD_GROUP heads, heaviest quads
  // first when causal; z = sequence
  const int cl = (int)blockIdx.x / 2;
  const int per_group = ATT_HEAD_GROUP * args.n_quads;
  const int group = cl / per_group;
  const int within = cl - group * per_group;
  const int heads_in_group = min(ATT_HEAD_GROUP, args.heads - group * ATT_HEAD_GROUP);
  const int quad_rank = within / heads_in_group;
  const int head = group * ATT_HEAD_GROUP + (within - quad_rank * heads_in_group);
  const int quad = args.causal ? (args.n_quads - 1 - quad_rank) : quad_rank;
  const int beta = args.beta0 + blockIdx.z;
  const int tq = args.t_start + quad * 4 * ATT_BM;  // first row of the cluster's four tiles
  const int t_end = args.t_start + args.t_len;
  // key/value tiles a query tile needs (0 for a tile past the end)
  auto tile_n_kv = [&](int tile) {
    const int r0 = tq + tile * ATT_BM;
    const int rv = max(0, min(ATT_BM, t_end - r0));
    if (rv == 0) return 0;
    const int kv_end = args.causal ? min(args.s, r0 + rv) : args.s;
    return (kv_end + ATT_BN - 1) / ATT_BN;
  };
  int n_slot[2], rows_valid[2], my_t0[2];
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    n_slot[q] = max(tile_n_kv(pair_tile_of(0, q)), tile_n_kv(pair_tile_of(1, q)));
    my_t0[q] = tq + pair_tile_of(rank, q) * ATT_BM;
    rows_valid[q] = max(0, min(ATT_BM, t_end - my_t0[q]));
  }
  const int n_tiles = max(n_slot[0], n_slot[1]);

  if (warp == 0 && lane == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full0 + 8 * i, 1);
      mbar_init(p_full0 + 8 * i, 8);
      mbar_init(o_done0 + 8 * i, 1);
    }
    for (int i = 0; i < C::RING; ++i) {
      mbar_init(ring_full0 + 8 * i, 1);
      mbar_init(ring_empty0 + 8 * i, 1);
    }
    mbar_init(mma_done, 1);
    *abort_flag.flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_addr(tmem_slot), ATT_TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers exist before either signals the other
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < 4) {
    regs_decrease<ATT_PAIR_REGS_CONTROL>();
    if (warp == 0) {
      if (lane == 0) {
        // ---------------------------------------------------------- TMA producer (both CTAs)
        // load n of the ring: this CTA's half of K_j for n = 2j, of V_j for n = 2j + 1
        const uint32_t q_full_l = mapa_shared(q_full, 0);
        const uint32_t ring_full_l0 = mapa_shared(ring_full0, 0);
        uint32_t issued = 0, par = 0;
        if (leader) mbar_arrive_expect_tx(q_full, 4 * C::Q_BYTES);
        for (int q = 0; q < 2; ++q)
#pragma unroll
          for (int a = 0; a < DH / 64; ++a)
            tma_load_3d_pair(sbase + C::OFF_Q + q * C::Q_BYTES + a * C::Q_ATOM, &tmQ, q_full_l, head * DH + a * 64,
                             my_t0[q], beta);
        for (int n = 0; n < 2 * n_tiles; ++n) {
          const int slot = n % C::RING;
          const uint32_t ph = (uint32_t)(n / C::RING) & 1u;
          if (!mbar_wait(ring_empty0 + 8 * slot, ph ^ 1, abort_flag)) break;
          if (leader) mbar_arrive_expect_tx(ring_full0 + 8 * slot, 2 * C::SLOT_BYTES);
          const uint32_t dst = sbase + C::OFF_RING + slot * C::SLOT_BYTES;
          const int j = n >> 1;
          if ((n & 1) == 0) {
            // K_j, keys j*128 + rank*64 .. +63, all head columns (two boxes)
#pragma unroll
            for (int a = 0; a < DH / 64; ++a)
              tma_load_3d_pair(dst + a * C::K_ATOM, &tmK, ring_full_l0 + 8 * slot, head * DH + a * 64,
                               j * ATT_BN + rank * 64, beta);
          } else {
            // V_j, all 128 keys, head columns rank*64 .. +63 (one box)
            tma_load_3d_pair(dst, &tmV, ring_full_l0 + 8 * slot, head * DH + rank * 64, j * ATT_BN, beta);
          }
          issued |= 1u << slot;
          par = (par & ~(1u << slot)) | (ph << slot);
        }
        // never leave with copies still landing in shared memory: the leader
        // waits for the pair's last copies on its full barriers; the follower
        // for the leader's commits, which follow every copy the MMAs read
        volatile int dummy = 0;
        const Abort drain{&dummy, args.status};
        if (leader) mbar_wait(q_full, 0, drain);
        for (int i = 0; i < C::RING; ++i)
          if (issued & (1u << i)) {
            if (leader)
              mbar_wait(ring_full0 + 8 * i, (par >> i) & 1u, drain);
            else
              mbar_wait(ring_empty0 + 8 * i, (par >> i) & 1u, drain);
          }
      }
    } else if (warp == 1) {
      if (leader && lane == 0) {
        // ---------------------------------------------------------- MMA issuer (leader)
        const uint32_t idesc_s = idesc_bf16_f32(2 * ATT_BM, ATT_BN, 0, 0);  // Q K-major, K half K-major
        const uint32_t idesc_o = idesc_bf16_f32(2 * ATT_BM, DH, 0, 1);      // P (TMEM), V half MN-major
        int k_waited = -1, v_waited = -1;
        bool ok = mbar_wait(q_full, 0, abort_flag);
        auto last_user = [&](int j) { return j < n_slot[1] ? 1 : 0; };
        auto slot_of = [&](int n) { return n % C::RING; };
        auto parity_of = [&](int n) { return (uint32_t)(n / C::RING) & 1u; };
        auto issue_s = [&](int q, int j) -> bool {
          const int sl = slot_of(2 * j);
          if (k_waited < j) {
            if (!mbar_wait(ring_full0 + 8 * sl, parity_of(2 * j), abort_flag)) return false;
            k_waited = j;
          }
          tc_fence_after();
          const uint32_t q_s = sbase + C::OFF_Q + q * C::Q_BYTES;
          const uint32_t k_s = sbase + C::OFF_RING + sl * C::SLOT_BYTES;
#pragma unroll
          for (int kk = 0; kk < DH / 16; ++kk) {
            mma_bf16_ss_pair(tmem_base + q * 128,
                             smem_desc_sw128(q_s + (kk >> 2) * C::Q_ATOM + (kk & 3) * 32, 16, 1024),
                             smem_desc_sw128(k_s + (kk >> 2) * C::K_ATOM + (kk & 3) * 32, 16, 1024), idesc_s, kk > 0);
          }
          mma_commit_pair(s_full0 + 8 * q);
          if (last_user(j) == q) mma_commit_pair(ring_empty0 + 8 * sl);
          return true;
        };
        auto issue_pv = [&](int q, int j) -> bool {
          const int sl = slot_of(2 * j + 1);
          if (v_waited < j) {
            if (!mbar_wait(ring_full0 + 8 * sl, parity_of(2 * j + 1), abort_flag)) return false;
            v_waited = j;
          }
          const uint32_t v_s = sbase + C::OFF_RING + sl * C::SLOT_BYTES;
          const uint32_t p_t = tmem_base + q * 128;
          const uint32_t o_t = tmem_base + 256 + q * 128;
          if (!mbar_wait(p_full0 + 8 * q, j & 1, abort_flag)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < ATT_BN / 16; ++kk)
            mma_bf16_ts_pair(o_t, p_t + kk * 8, smem_desc_sw128(v_s + kk * 16 * 128, C::SLOT_BYTES, 1024), idesc_o,
                             (j | kk) != 0);
          if (last_user(j) == q) mma_commit_pair(ring_empty0 + 8 * sl);
          if (j == n_slot[q] - 1) mma_commit_pair(o_done0 + 8 * q);
          return true;
        };
        for (int q = 0; ok && q < 2; ++q)
          if (n_slot[q] > 0) ok = issue_s(q, 0);
        for (int j = 0; ok && j < n_tiles; ++j) {
          for (int q = 0; ok && q < 2; ++q) {
            if (j < n_slot[q]) ok = issue_pv(q, j);
            if (ok && j + 1 < n_slot[q]) ok = issue_s(q, j + 1);
          }
        }
        mma_commit_pair(mma_done);  // on every path, so that both CTAs can free their tensor memory
      }
    }
  } else {
    regs_increase<ATT_REGS_SOFTMAX>();
    // ------------------------------------------------------------ softmax (both CTAs)
    const int q = (warp - 4) >> 2;  // slot of this warpgroup
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int tq0 = my_t0[q];
    const int t = tq0 + r;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem_base + q * 128 + lane_base;
    const uint32_t tO = tmem_base + 256 + q * 128 + lane_base;
    const uint32_t p_full_l = mapa_shared(p_full0 + 8 * q, 0);
    const float sl2 = args.scale_log2;
    const int nk = n_slot[q];
    const int lim = args.causal ? min(args.s - 1, t) : args.s - 1;  // last visible key of this row
    float m = -INFINITY, l = 0.0f;
    bool ok = true;
    for (int j = 0; j < nk; ++j) {
      if (!warp_wait(s_full0 + 8 * q, j & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      float sv[ATT_BN];
      tmem_load128f(tS, sv);
      const int key0 = j * ATT_BN;
      const bool need_mask = (key0 + ATT_BN > args.s) || (args.causal && key0 + ATT_BN - 1 > tq0);
      if (need_mask) {
#pragma unroll
        for (int i = 0; i < ATT_BN; ++i) sv[i] = (key0 + i <= lim) ? sv[i] : -INFINITY;
      }
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int i = 0; i < ATT_BN; i += 8) {
#pragma unroll
        for (int k = 0; k < 4; ++k) mx4[k] = max3f(mx4[k], sv[i + 2 * k], sv[i + 2 * k + 1]);
      }
      float mx = max3f(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3]));
      mx *= sl2;
      float m_new = m, alpha = 1.0f;
      if (mx > m + ATT_RESCALE_THRESHOLD) {
        m_new = mx;
        alpha = ex2_approx(m - mx);  // 0 on the first tile (m = -inf)
      }
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll 1
        for (int c = 0; c < DH / 32; ++c) {
          uint32_t o[32];
          tmem_load32(tO + c * 32, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_store32(tO + c * 32, o);
        }
      }
      // P = 2^(S*scale - m) in bf16 over the first 64 columns of S; l sums the
      // bf16 weights the P V product uses. A row whose tile ends before this
      // key/value tile (the shorter tile of a causal slot) sees every key
      // masked: its weights are exactly 0 and m, l do not change.
      const uint64_t sl2x2 = f2_pack(sl2, sl2);
      const uint64_t negm2 = f2_pack(m_new == -INFINITY ? 0.0f : -m_new, m_new == -INFINITY ? 0.0f : -m_new);
      float sum4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      auto exp_phase = [&]() {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t pk[32];
#pragma unroll
          for (int i2 = 0; i2 < 32; ++i2) {
            const int i = 32 * half + i2;
            const uint64_t x2 = f2_fma(f2_pack(sv[2 * i], sv[2 * i + 1]), sl2x2, negm2);
            float x0, x1;
            f2_unpack(x2, x0, x1);
            const uint32_t pp = pack_bf16x2(ex2_approx(x0), ex2_approx(x1));
            pk[i2] = pp;
            add_bf16x2_to(pp, sum4[i & 3], sum4[(i + 2) & 3]);
          }
          tmem_store32(tS + 32 * half, pk);
        }
      };
      exp_phase();
      // hand P to the leader's MMA issuer
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(p_full_l);
      const float sum = (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]);
      l = l * alpha + sum;
      m = m_new;
    }

    // ------------------------------------------------------------ epilogue
    if (ok && nk > 0 && warp_wait(o_done0 + 8 * q, 0, abort_flag)) {
      tc_fence_after();
      const float inv_l = 1.0f / l;
      const bool row_ok = r < rows_valid[q];
      __nv_bfloat16* orow =
          args.o + ((long long)(beta - args.beta0) * args.t_len + (t - args.t_start)) * args.ldo + head * DH;
#pragma unroll 1
      for (int c = 0; c < DH / 32; ++c) {
        uint32_t o[32];
        tmem_load32(tO + c * 32, o);
        if (row_ok) {
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(o[i]) * inv_l;
#pragma unroll
          for (int i = 0; i < 4; ++i)
            st_global_v4(orow + c * 32 + 8 * i, pack_bf16x2(v[8 * i], v[8 * i + 1]),
                         pack_bf16x2(v[8 * i + 2], v[8 * i + 3]), pack_bf16x2(v[8 * i + 4], v[8 * i + 5]),
                         pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
        }
      }
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
    tmem_dealloc_pair(tmem_base, ATT_TMEM_COLS);
  }
}

}  // namespace bpt
