// Fused blockwise attention for one query tile (128 rows of one head of one
// sequence) over all of its key/value tiles, with online-softmax rescaling.
//
// Follows Eq. 3 and Algorithm 1 (steps 4-10) of the BPT paper review: scores of
// the query block against each key/value block, normalisation statistics kept
// per row (running max m and running sum l in fp32 registers), the block's
// exp-weights applied to V, and a final rescale by 1/l. The s x s score matrix
// never leaves the SM: S lives in tensor memory, P in shared memory.
//
// Roles (192 threads): warp 0 loads Q once and K/V tiles into a two-stage
// ring with TMA; one thread of warp 1 issues S = Q K^T into one of two TMEM
// score buffers and O += P V into the TMEM output accumulator; warps 2-5 own
// one query row each (TMEM lane), run the softmax, write P (bf16) to shared
// memory in the operand layout of the next MMA, rescale O when the running
// max grows, and write the normalised output row.
#pragma once

#include "ptx.cuh"

namespace bpt {

constexpr int ATT_BM = 128;  // query rows per CTA
constexpr int ATT_BN = 128;  // keys per key/value tile
constexpr int ATT_THREADS = 192;
constexpr int ATT_TMEM_COLS = 512;  // S0 [0,128), S1 [128,256), O [256, 256+dh)
// Skip rescaling O until the running max has grown by more than this (log2
// units); P then holds values up to 2^8, which bf16 and fp32 carry exactly in
// range. The final division by l uses the same stale max, so the result is exact.
constexpr float ATT_RESCALE_THRESHOLD = 8.0f;

template <int DH>
struct AttnCfg {
  static constexpr int Q_BYTES = ATT_BM * DH * 2;
  static constexpr int KV_BYTES = ATT_BN * DH * 2;
  static constexpr int P_BYTES = ATT_BM * ATT_BN * 2;
  static constexpr int ATOM_BYTES = 128 * 128;  // [128 rows][64 bf16] swizzle-128B box
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + 2 * KV_BYTES;
  static constexpr int OFF_P = OFF_V + 2 * KV_BYTES;
  static constexpr int OFF_BAR = OFF_P + P_BYTES;
  static constexpr int USED = OFF_BAR + 256 + 1024;
  // at least 116 KB so that one CTA holds an SM (the 512 TMEM columns are
  // allocated whole)
  static constexpr int SMEM_BYTES = USED > 118784 ? USED : 118784;
};

struct AttnArgs {
  int s, heads, causal;
  int beta0;        // first sequence of this launch
  int t_start;      // query positions [t_start, t_start + t_len) of each sequence
  int t_len;
  int n_qtiles;     // ceil(t_len / 128)
  __nv_bfloat16* o; // output rows: (beta - beta0) * t_len + (t - t_start)
  long long ldo;
  float scale_log2; // log2(e) / sqrt(dh)
};

template <int DH>
__global__ void __launch_bounds__(ATT_THREADS, 1)
    attention_fwd_tcgen05(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const AttnArgs args) {
  using C = AttnCfg<DH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  const uint32_t q_full = smem_addr(bars + 0);
  const uint32_t k_full0 = smem_addr(bars + 1);   // [2]
  const uint32_t k_empty0 = smem_addr(bars + 3);  // [2]
  const uint32_t v_full0 = smem_addr(bars + 5);   // [2]
  const uint32_t v_empty0 = smem_addr(bars + 7);  // [2]
  const uint32_t s_full0 = smem_addr(bars + 9);   // [2]
  const uint32_t s_free0 = smem_addr(bars + 11);  // [2]
  const uint32_t p_full = smem_addr(bars + 13);
  const uint32_t pv_done = smem_addr(bars + 14);
  const uint32_t mma_done = smem_addr(bars + 15);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 17);

  const int warp = warp_id();
  const int lane = lane_id();
  const uint32_t sbase = smem_addr(smem);

  // ------------------------------------------------------------ tile geometry
  const int head = blockIdx.x;
  const int qt = args.causal ? (args.n_qtiles - 1 - (int)blockIdx.y) : (int)blockIdx.y;  // heavy tiles first
  const int beta = args.beta0 + blockIdx.z;
  const int t0 = args.t_start + qt * ATT_BM;
  const int rows_valid = min(ATT_BM, args.t_start + args.t_len - t0);
  const int kv_end = args.causal ? min(args.s, t0 + rows_valid) : args.s;  // keys [0, kv_end)
  const int n_kv = (kv_end + ATT_BN - 1) / ATT_BN;

  if (warp == 0 && lane == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(k_full0 + 8 * i, 1);
      mbar_init(k_empty0 + 8 * i, 1);
      mbar_init(v_full0 + 8 * i, 1);
      mbar_init(v_empty0 + 8 * i, 1);
      mbar_init(s_full0 + 8 * i, 1);
      mbar_init(s_free0 + 8 * i, 4);
    }
    mbar_init(p_full, 4);
    mbar_init(pv_done, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
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
  const uint32_t tS0 = tmem_base, tO = tmem_base + 256;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- TMA producer
      uint32_t k_issued = 0, v_issued = 0, k_par = 0, v_par = 0;
      mbar_arrive_expect_tx(q_full, C::Q_BYTES);
#pragma unroll
      for (int a = 0; a < DH / 64; ++a)
        tma_load_3d(sbase + C::OFF_Q + a * C::ATOM_BYTES, &tmQ, q_full, head * DH + a * 64, t0, beta);
      for (int j = 0; j < n_kv; ++j) {
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!mbar_wait(k_empty0 + 8 * st, ph ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(k_full0 + 8 * st, C::KV_BYTES);
#pragma unroll
        for (int a = 0; a < DH / 64; ++a)
          tma_load_3d(sbase + C::OFF_K + st * C::KV_BYTES + a * C::ATOM_BYTES, &tmK, k_full0 + 8 * st,
                      head * DH + a * 64, j * ATT_BN, beta);
        k_issued |= 1u << st;
        k_par = (k_par & ~(1u << st)) | (ph << st);
        if (!mbar_wait(v_empty0 + 8 * st, ph ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(v_full0 + 8 * st, C::KV_BYTES);
#pragma unroll
        for (int a = 0; a < DH / 64; ++a)
          tma_load_3d(sbase + C::OFF_V + st * C::KV_BYTES + a * C::ATOM_BYTES, &tmV, v_full0 + 8 * st,
                      head * DH + a * 64, j * ATT_BN, beta);
        v_issued |= 1u << st;
        v_par = (v_par & ~(1u << st)) | (ph << st);
      }
      // never leave with copies still landing in shared memory
      volatile int dummy = 0;
      mbar_wait(q_full, 0, &dummy);
      for (int i = 0; i < 2; ++i) {
        if (k_issued & (1u << i)) mbar_wait(k_full0 + 8 * i, (k_par >> i) & 1u, &dummy);
        if (v_issued & (1u << i)) mbar_wait(v_full0 + 8 * i, (v_par >> i) & 1u, &dummy);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      const uint32_t idesc_s = idesc_bf16_f32(ATT_BM, ATT_BN, 0, 0);  // Q K-major, K tile K-major
      const uint32_t idesc_o = idesc_bf16_f32(ATT_BM, DH, 0, 1);      // P K-major, V tile MN-major
      const uint32_t q_s = sbase + C::OFF_Q;
      const uint32_t p_s = sbase + C::OFF_P;
      bool ok = mbar_wait(q_full, 0, abort_flag);
      // S(n) = Q K_n^T into score buffer n % 2
      auto issue_s = [&](int n) -> bool {
        const int sb = n & 1;
        if (n >= 2 && !mbar_wait(s_free0 + 8 * sb, ((n >> 1) - 1) & 1, abort_flag)) return false;
        if (!mbar_wait(k_full0 + 8 * sb, (n >> 1) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t k_s = sbase + C::OFF_K + sb * C::KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::ATOM_BYTES + (kk & 3) * 32;
          mma_bf16_ss(tS0 + sb * ATT_BN, smem_desc_sw128(q_s + off, 16, 1024), smem_desc_sw128(k_s + off, 16, 1024),
                      idesc_s, kk > 0);
        }
        mma_commit(s_full0 + 8 * sb);
        mma_commit(k_empty0 + 8 * sb);
        return true;
      };
      if (ok && n_kv > 0) ok = issue_s(0);
      for (int j = 0; ok && j < n_kv; ++j) {
        if (j + 1 < n_kv && !issue_s(j + 1)) break;
        const int st = j & 1;
        if (!mbar_wait(p_full, j & 1, abort_flag)) break;
        if (!mbar_wait(v_full0 + 8 * st, (j >> 1) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t v_s = sbase + C::OFF_V + st * C::KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < ATT_BN / 16; ++kk) {
          const uint64_t pdesc = smem_desc_sw128(p_s + (kk >> 2) * C::ATOM_BYTES + (kk & 3) * 32, 16, 1024);
          const uint64_t vdesc = smem_desc_sw128(v_s + kk * 16 * 128, C::ATOM_BYTES, 1024);
          mma_bf16_ss(tO, pdesc, vdesc, idesc_o, (j | kk) != 0);
        }
        mma_commit(pv_done);
        mma_commit(v_empty0 + 8 * st);
      }
      mma_commit(mma_done);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // query row within the tile == TMEM lane
    const int t = t0 + r;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const float sl2 = args.scale_log2;
    float m = -INFINITY, l = 0.0f;
    bool ok = true;
    const uint32_t p_row = sbase + C::OFF_P + r * 128;
    for (int j = 0; j < n_kv; ++j) {
      const int sb = j & 1;
      if (!warp_wait(s_full0 + 8 * sb, (j >> 1) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      float sv[ATT_BN];
      {
        uint32_t a[32], b[32];
        tmem_load32x2(tS0 + sb * ATT_BN + lane_base, tS0 + sb * ATT_BN + 32 + lane_base, a, b);
#pragma unroll
        for (int i = 0; i < 32; ++i) { sv[i] = __uint_as_float(a[i]); sv[32 + i] = __uint_as_float(b[i]); }
        tmem_load32x2(tS0 + sb * ATT_BN + 64 + lane_base, tS0 + sb * ATT_BN + 96 + lane_base, a, b);
#pragma unroll
        for (int i = 0; i < 32; ++i) { sv[64 + i] = __uint_as_float(a[i]); sv[96 + i] = __uint_as_float(b[i]); }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free0 + 8 * sb);

      // scale into log2 units, mask, row max
      const int key0 = j * ATT_BN;
      const bool need_mask = (key0 + ATT_BN > args.s) || (args.causal && key0 + ATT_BN - 1 > t0);
      float mx = -INFINITY;
      if (need_mask) {
        const int lim = args.causal ? min(args.s - 1, t) : args.s - 1;  // last visible key
#pragma unroll
        for (int i = 0; i < ATT_BN; ++i) {
          const float v = (key0 + i <= lim) ? sv[i] * sl2 : -INFINITY;
          sv[i] = v;
          mx = fmaxf(mx, v);
        }
      } else {
#pragma unroll
        for (int i = 0; i < ATT_BN; ++i) {
          sv[i] *= sl2;
          mx = fmaxf(mx, sv[i]);
        }
      }
      float m_new = m, alpha = 1.0f;
      if (mx > m + ATT_RESCALE_THRESHOLD) {
        m_new = mx;
        alpha = ex2_approx(m - mx);  // 0 on the first tile (m = -inf)
      }
      uint32_t pk[ATT_BN / 2];
      float sum = 0.0f;
#pragma unroll
      for (int i = 0; i < ATT_BN; i += 2) {
        const float p0 = ex2_approx(sv[i] - m_new);
        const float p1 = ex2_approx(sv[i + 1] - m_new);
        const uint32_t pp = pack_bf16x2(p0, p1);
        pk[i / 2] = pp;
        // l sums the bf16 weights the P V product uses, so that O = sum(P V) / l
        // is an exact weighted mean (V == 1 gives exactly 1)
        sum += __uint_as_float(pp << 16) + __uint_as_float(pp & 0xffff0000u);
      }
      l = l * alpha + sum;
      m = m_new;

      // P buffer and O are free once the previous P V product has completed
      if (j > 0) {
        if (!warp_wait(pv_done, (j - 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll 1
          for (int c = 0; c < DH / 32; ++c) {
            uint32_t o[32];
            tmem_load32(tO + c * 32 + lane_base, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_store32(tO + c * 32 + lane_base, o);
          }
        }
      }
      // P row -> shared memory, K-major 128B-swizzled: two [128][64] atoms
#pragma unroll
      for (int c16 = 0; c16 < 16; ++c16) {
        const uint32_t addr = p_row + (c16 >> 3) * C::ATOM_BYTES + (((c16 & 7) ^ (r & 7)) << 4);
        st_shared_v4(addr, pk[4 * c16], pk[4 * c16 + 1], pk[4 * c16 + 2], pk[4 * c16 + 3]);
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }

    // ------------------------------------------------------------ epilogue
    if (ok && n_kv > 0 && warp_wait(pv_done, (n_kv - 1) & 1, abort_flag)) {
      tc_fence_after();
      const float inv_l = 1.0f / l;
      const bool row_ok = r < rows_valid;
      __nv_bfloat16* orow =
          args.o + ((long long)(beta - args.beta0) * args.t_len + (t - args.t_start)) * args.ldo + head * DH;
#pragma unroll 1
      for (int c = 0; c < DH / 32; ++c) {
        uint32_t o[32];
        tmem_load32(tO + c * 32 + lane_base, o);
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

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) {
      volatile int dummy = 0;
      mbar_wait(mma_done, 0, &dummy);
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, ATT_TMEM_COLS);
  }
}

}  // namespace bpt
