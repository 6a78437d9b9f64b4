// Fused blockwise attention: one CTA computes two query tiles (2 x 128 rows of
// one head of one sequence) over all of their key/value tiles, with
// online-softmax rescaling.
//
// Follows Eq. 3 and Algorithm 1 (steps 4-10) of the BPT paper review: scores
// of a query block against each key/value block, normalisation statistics per
// row (running max m and running sum l, fp32 registers), the block's
// exp-weights applied to V, and a final rescale by 1/l. The s x s score matrix
// never leaves the SM: S and P live in tensor memory.
//
// Roles (384 threads = three warpgroups): warp 0 loads Q (both tiles, once)
// and the K/V tiles into a ring of shared-memory slots with TMA; one thread of warp 1 issues
// the MMAs; warps 2-3 idle; warpgroup 1 (warps 4-7) runs the softmax of query
// tile 0 and warpgroup 2 (warps 8-11) that of tile 1, one row per thread =
// one TMEM lane (warp w reaches lanes 32*(w%4) .. +31). Registers are split
// per warpgroup: the kernel is built for 168 per thread (384 x 168 = 64512),
// warpgroup 0 gives back down to ATT_REGS_CONTROL and the softmax warpgroups
// grow to ATT_REGS_SOFTMAX (128 x 56 + 256 x 216 = 62464 <= 64512). The host
// launches the kernel only if it was built with exactly ATT_REGS_LAUNCH. While one warpgroup computes exponentials the
// tensor core works on the other tile, in the order
//     PV0(j), S0(j+1), PV1(j), S1(j+1), PV0(j+1), ...
// Tensor memory (512 columns): S0 [0,128), S1 [128,256), O0 [256, 256+dh),
// O1 [384, 384+dh). The softmax writes P (bf16 pairs) over the first 64
// columns of its S; the P V product reads it from there (A operand in TMEM);
// the next S MMA of that tile, issued after it, overwrites it (MMAs of one
// thread execute in issue order). P is handed over whole: splitting it in
// two halves, each with its own barrier, measured about 3% slower, since the
// extra wait delays the issuing thread more than the early half gains.
#pragma once

#include "ptx.cuh"

namespace bpt {

constexpr int ATT_BM = 128;  // query rows per tile; two tiles per CTA
constexpr int ATT_BN = 128;  // keys per key/value tile
constexpr int ATT_THREADS = 384;
constexpr int ATT_REGS_LAUNCH = 168;   // registers per thread the kernel is built with
constexpr int ATT_REGS_CONTROL = 56;   // warpgroup 0: TMA producer and MMA issuer
constexpr int ATT_REGS_SOFTMAX = 216;  // warpgroups 1 and 2
static_assert(ATT_THREADS * ATT_REGS_LAUNCH >= 128 * ATT_REGS_CONTROL + 256 * ATT_REGS_SOFTMAX,
              "register split exceeds the block's launch allocation");
constexpr int ATT_TMEM_COLS = 512;
// Heads scheduled together (see the grid order below). Two: at s = 32768 a
// group of four heads' K/V (67 MB) and the next group's exceeded L2 (DRAM
// reads 1.48x Q + K + V); groups of two read 1.01x and ran ~1% faster, and
// single heads ran ~1.5% slower (fewer CTAs share each K/V tile).
constexpr int ATT_HEAD_GROUP = 2;
// Skip rescaling O until the running max has grown by more than this (log2
// units); P then holds values up to 2^8, well inside bf16 and fp32 range. The
// final division by l uses the same stale max, so the result is exact.
constexpr float ATT_RESCALE_THRESHOLD = 8.0f;

template <int DH>
struct AttnCfg {
  static constexpr int Q_BYTES = ATT_BM * DH * 2;   // one query tile
  static constexpr int KV_BYTES = ATT_BN * DH * 2;  // one K or V tile
  static constexpr int ATOM_BYTES = 128 * 128;      // [128 rows][64 bf16] 128B-swizzled box
  // K and V tiles share one ring of slots (K_j, V_j, K_j+1, ...), as deep as
  // shared memory allows, so that several tiles are in flight from L2
  static constexpr int RING = DH == 128 ? 5 : 8;
  static constexpr int OFF_Q = 0;                   // two query tiles
  static constexpr int OFF_RING = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_BAR = OFF_RING + RING * KV_BYTES;
  static constexpr int USED = OFF_BAR + 512 + 1024;
  // at least 116 KB so that one CTA holds an SM (all 512 TMEM columns are
  // allocated)
  static constexpr int SMEM_BYTES = USED > 118784 ? USED : 118784;
  static_assert(USED <= 232448, "shared memory budget");
};

struct AttnArgs {
  int s, heads, causal;
  int beta0;        // first sequence of this launch
  int t_start;      // query positions [t_start, t_start + t_len) of each sequence
  int t_len;
  int n_pairs;      // ceil(t_len / 256): CTAs per (sequence, head)
  __nv_bfloat16* o; // output rows: (beta - beta0) * t_len + (t - t_start)
  long long ldo;
  float scale_log2; // log2(e) / sqrt(dh)
  int* status;      // status word of the launching stream
  float* lse2;      // [n_seq][heads][t_len]: m + log2(l) of each row (log2 units); written by the LSE build only
  unsigned* grp_cnt;  // one-launch layer only: per group of grp_rows output rows (flat over the sequences), one
  int grp_rows;       // count per warp whose 32 rows of one head are stored (release order after the stores)
};

// D[tmem] (+)= A[tmem] * B[smem]: bf16 A read from tensor memory (K-major).
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Work item `item` of the one-launch layer: query-tile pairs in row order, every
// head of a pair before the next pair (host code, the schedule's tests, uses it too).
__host__ __device__ __forceinline__ void mega_item_coords(const AttnArgs& a, int item, int& beta, int& head,
                                                          int& pair) {
  head = item % a.heads;
  const int bp = item / a.heads;
  pair = bp % a.n_pairs;
  beta = a.beta0 + bp / a.n_pairs;
}

// The first of the output rows (flat over the call's sequences) that a warp of
// a query tile stores, and so the group whose count it raises.
__host__ __device__ __forceinline__ long long mega_warp_row(const AttnArgs& a, int beta, int tq0, int quarter) {
  return (long long)(beta - a.beta0) * a.t_len + (tq0 - a.t_start) + quarter * 32;
}

// One CTA's work: query-tile pair `item` of sequence beta0 + zseq (the
// attention kernel below), or, with MEGA (the one-launch layer), work item
// `item` in row order with every warp's stored rows counted in args.grp_cnt.
// LSE: also write each row's log-sum-exp (args.lse2), for the backward; a
// separate build so that the forward alone carries nothing for it.
template <int DH, bool LSE, bool MEGA>
__device__ __forceinline__ void attention_fwd_body(const CUtensorMap& tmQ, const CUtensorMap& tmK,
                                                   const CUtensorMap& tmV, const AttnArgs& args, int item, int zseq) {
  using C = AttnCfg<DH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  const uint32_t q_full = smem_addr(bars + 0);
  const uint32_t s_full0 = smem_addr(bars + 1);   // [2] per query tile
  const uint32_t p_full0 = smem_addr(bars + 3);   // [2] per query tile
  const uint32_t o_done0 = smem_addr(bars + 5);   // [2] per query tile
  const uint32_t mma_done = smem_addr(bars + 9);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 10);
  const Abort abort_flag{reinterpret_cast<volatile int*>(bars + 11), args.status};
  const uint32_t ring_full0 = smem_addr(bars + 12);             // [RING]
  const uint32_t ring_empty0 = smem_addr(bars + 12 + C::RING);  // [RING]

  const int warp = warp_id();
  const int lane = lane_id();
  const uint32_t sbase = smem_addr(smem);

  // ------------------------------------------------------------ geometry
  // grid: x enumerates (head, query-tile pair) in groups of ATT_HEAD_GROUP
  // heads; inside a group the pairs go heaviest first (causal), cycling over
  // the group's heads. CTAs resident together then touch a few heads, whose
  // K/V stay in L2, and the end of the grid holds the lightest pairs.
  // z = sequence.
  // (MEGA: items in row order, every head of a pair before the next pair, so
  // that the rows a later out-projection tile needs are finished early.)
  int head, pair, beta;
  if constexpr (MEGA) {
    mega_item_coords(args, item, beta, head, pair);
  } else {
    const int per_group = ATT_HEAD_GROUP * args.n_pairs;
    const int group = item / per_group;
    const int within = item - group * per_group;
    const int heads_in_group = min(ATT_HEAD_GROUP, args.heads - group * ATT_HEAD_GROUP);
    const int pair_rank = within / heads_in_group;
    head = group * ATT_HEAD_GROUP + (within - pair_rank * heads_in_group);
    pair = args.causal ? (args.n_pairs - 1 - pair_rank) : pair_rank;
    beta = args.beta0 + zseq;
  }
  const int t0 = args.t_start + pair * 2 * ATT_BM;  // first row of query tile 0
  const int t_end = args.t_start + args.t_len;
  int rows_valid[2], n_kv[2];
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    rows_valid[q] = max(0, min(ATT_BM, t_end - (t0 + q * ATT_BM)));
    const int kv_end = args.causal ? min(args.s, t0 + q * ATT_BM + rows_valid[q]) : args.s;
    n_kv[q] = rows_valid[q] > 0 ? (kv_end + ATT_BN - 1) / ATT_BN : 0;
  }
  const int n_tiles = max(n_kv[0], n_kv[1]);
  const bool has1 = rows_valid[1] > 0;

  if (warp == 0 && lane == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full0 + 8 * i, 1);
      mbar_init(p_full0 + 8 * i, 4);
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
    tmem_alloc(smem_addr(tmem_slot), ATT_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < 4) {
    // each role stays inside the branch that set its register budget
    regs_decrease<ATT_REGS_CONTROL>();
    if (warp == 0) {
      if (lane == 0) {
        // ---------------------------------------------------------- TMA producer
        // load n of the ring: K_j for n = 2j, V_j for n = 2j + 1
        uint32_t issued = 0, par = 0;
        const int nq = has1 ? 2 : 1;
        mbar_arrive_expect_tx(q_full, nq * C::Q_BYTES);
        for (int q = 0; q < nq; ++q)
#pragma unroll
          for (int a = 0; a < DH / 64; ++a)
            tma_load_3d(sbase + C::OFF_Q + q * C::Q_BYTES + a * C::ATOM_BYTES, &tmQ, q_full, head * DH + a * 64,
                        t0 + q * ATT_BM, beta);
        for (int n = 0; n < 2 * n_tiles; ++n) {
          const int slot = n % C::RING;
          const uint32_t ph = (uint32_t)(n / C::RING) & 1u;
          if (!mbar_wait(ring_empty0 + 8 * slot, ph ^ 1, abort_flag)) break;
          mbar_arrive_expect_tx(ring_full0 + 8 * slot, C::KV_BYTES);
          const CUtensorMap* map = (n & 1) ? &tmV : &tmK;
#pragma unroll
          for (int a = 0; a < DH / 64; ++a)
            tma_load_3d(sbase + C::OFF_RING + slot * C::KV_BYTES + a * C::ATOM_BYTES, map, ring_full0 + 8 * slot,
                        head * DH + a * 64, (n >> 1) * ATT_BN, beta);
          issued |= 1u << slot;
          par = (par & ~(1u << slot)) | (ph << slot);
        }
        // never leave with copies still landing in shared memory
        volatile int dummy = 0;
        const Abort drain{&dummy, args.status};
        mbar_wait(q_full, 0, drain);
        for (int i = 0; i < C::RING; ++i)
          if (issued & (1u << i)) mbar_wait(ring_full0 + 8 * i, (par >> i) & 1u, drain);
      }
    } else if (warp == 1) {
      if (lane == 0) {
        // ---------------------------------------------------------- MMA issuer
        const uint32_t idesc_s = idesc_bf16_f32(ATT_BM, ATT_BN, 0, 0);  // Q K-major, K tile K-major
        const uint32_t idesc_o = idesc_bf16_f32(ATT_BM, DH, 0, 1);      // P K-major (TMEM), V MN-major
        int k_waited = -1, v_waited = -1;
        bool ok = mbar_wait(q_full, 0, abort_flag);
        // the last query tile that uses key/value tile j releases its slots
        auto last_user = [&](int j) { return (has1 && j < n_kv[1]) ? 1 : 0; };
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
          const uint32_t k_s = sbase + C::OFF_RING + sl * C::KV_BYTES;
#pragma unroll
          for (int kk = 0; kk < DH / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::ATOM_BYTES + (kk & 3) * 32;
            mma_bf16_ss(tmem_base + q * 128, smem_desc_sw128(q_s + off, 16, 1024),
                        smem_desc_sw128(k_s + off, 16, 1024), idesc_s, kk > 0);
          }
          mma_commit(s_full0 + 8 * q);
          if (last_user(j) == q) mma_commit(ring_empty0 + 8 * sl);
          return true;
        };
        auto issue_pv = [&](int q, int j) -> bool {
          const int sl = slot_of(2 * j + 1);
          if (v_waited < j) {
            if (!mbar_wait(ring_full0 + 8 * sl, parity_of(2 * j + 1), abort_flag)) return false;
            v_waited = j;
          }
          const uint32_t v_s = sbase + C::OFF_RING + sl * C::KV_BYTES;
          const uint32_t p_t = tmem_base + q * 128;
          const uint32_t o_t = tmem_base + 256 + q * 128;
          if (!mbar_wait(p_full0 + 8 * q, j & 1, abort_flag)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < ATT_BN / 16; ++kk)
            mma_bf16_ts(o_t, p_t + kk * 8, smem_desc_sw128(v_s + kk * 16 * 128, C::ATOM_BYTES, 1024), idesc_o,
                        (j | kk) != 0);
          if (last_user(j) == q) mma_commit(ring_empty0 + 8 * sl);
          if (j == n_kv[q] - 1) mma_commit(o_done0 + 8 * q);
          return true;
        };
        for (int q = 0; ok && q < 2; ++q)
          if (n_kv[q] > 0) ok = issue_s(q, 0);
        for (int j = 0; ok && j < n_tiles; ++j) {
          for (int q = 0; ok && q < 2; ++q) {
            if (j < n_kv[q]) ok = issue_pv(q, j);
            if (ok && j + 1 < n_kv[q]) ok = issue_s(q, j + 1);
          }
        }
        mma_commit(mma_done);
      }
    }
  } else {
    regs_increase<ATT_REGS_SOFTMAX>();
    // ------------------------------------------------------------ softmax
    const int q = (warp - 4) >> 2;  // query tile of this warpgroup
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // row within the tile == TMEM lane
    const int tq0 = t0 + q * ATT_BM;    // first row of the tile
    const int t = tq0 + r;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem_base + q * 128 + lane_base;
    const uint32_t tO = tmem_base + 256 + q * 128 + lane_base;
    const float sl2 = args.scale_log2;
    const int nk = n_kv[q];
    const int lim = args.causal ? min(args.s - 1, t) : args.s - 1;  // last visible key of this row
    float m = -INFINITY, l = 0.0f;
    bool ok = true;
    for (int j = 0; j < nk; ++j) {
      if (!warp_wait(s_full0 + 8 * q, j & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      float sv[ATT_BN];
      tmem_load128f(tS, sv);
      // mask and row max of the raw scores (the scale is positive)
      const int key0 = j * ATT_BN;
      const bool need_mask = (key0 + ATT_BN > args.s) || (args.causal && key0 + ATT_BN - 1 > tq0);
      // four independent chains of three-input max operations (a single
      // dependent chain would serialise on latency)
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
      // O may be rescaled now: the MMA that produced this S was committed after
      // every earlier P V product of this tile, so those have completed
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
      // P = 2^(S*scale - m) in bf16, written over the first 64 columns of S.
      // l sums the bf16 weights that the P V product uses, so that
      // O = sum(P V) / l is an exact weighted mean (V == 1 gives exactly 1).
      const uint64_t sl2x2 = f2_pack(sl2, sl2);
      const uint64_t negm2 = f2_pack(-m_new, -m_new);
      float sum4[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // independent partial sums
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
      // hand P to the MMA issuer
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full0 + 8 * q);
      const float sum = (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]);
      l = l * alpha + sum;
      m = m_new;
    }

    // ------------------------------------------------------------ epilogue
    if (ok && nk > 0 && warp_wait(o_done0 + 8 * q, 0, abort_flag)) {
      tc_fence_after();
      const float inv_l = 1.0f / l;
      const bool row_ok = r < rows_valid[q];
      // the row's log-sum-exp of the scaled scores, in log2 units: the
      // (possibly stale) max m plus log2 of the sum l taken against it
      if constexpr (LSE) {
        if (row_ok)
          args.lse2[((long long)(beta - args.beta0) * args.heads + head) * args.t_len + (t - args.t_start)] =
              m + log2f(l);
      }
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
      if constexpr (MEGA) {
        // publish this warp's 32 rows of this head (the rows of a 128-row tile lie
        // in one group: groups are whole tiles)
        __threadfence();
        __syncwarp();
        if (lane == 0) red_release_add(args.grp_cnt + mega_warp_row(args, beta, tq0, quarter) / args.grp_rows, 1u);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) {
      volatile int dummy = 0;
      mbar_wait(mma_done, 0, Abort{&dummy, args.status});
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, ATT_TMEM_COLS);
  }
}

template <int DH, bool LSE = false>
__global__ void __launch_bounds__(ATT_THREADS, 1)
    attention_fwd_tcgen05(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const AttnArgs args) {
  attention_fwd_body<DH, LSE, false>(tmQ, tmK, tmV, args, (int)blockIdx.x, (int)blockIdx.z);
}

}  // namespace bpt
