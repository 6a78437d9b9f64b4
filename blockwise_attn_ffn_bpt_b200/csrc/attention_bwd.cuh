// Attention backward: gradients dQ, dK, dV of O = softmax(Q K^T / sqrt(dh)) V
// for one head, blockwise, from the forward's per-row log-sum-exp.
//
// Follows the blockwise backward of the BPT paper review (section 3: the
// blockwise computation is rematerialised for training; Eq. 3 and Algorithm 1
// give the forward it inverts). One CTA owns one key/value tile of 128 keys of
// one head of one sequence and visits every query tile that sees it (causal:
// from the diagonal on). Per query tile i it recomputes
//     S^T  = K_j Q_i^T                 (scores, keys x queries)
//     P^T  = 2^(S^T * scale_log2 - lse2_i)   (0 where masked)
//     dP^T = V_j dO_i^T
//     dS^T = scale x P^T (dP^T - D_i),  D_i = rowsum(dO_i O_i),  scale = 1/sqrt(dh)
// and accumulates dV_j += P^T dO_i and dK_j += dS^T Q_i in tensor memory; the
// query gradient dQ_i += dS K_j is added to an fp32 accumulator in global
// memory by the TMA engine (bulk reduce-add of whole boxes staged in shared
// memory). At the end dK_j and dV_j are written as bf16. (The score scale sits
// in dS, where it costs nothing: dS = P (scale dP - scale D), one fused
// multiply-add and one multiply per element as without it.)
//
// Roles (640 threads): warp 0 copies K_j, V_j once and Q_i, dO_i per query
// tile (two-stage ring) with TMA; one thread of warp 1 issues the MMAs; one
// thread of warp 2 issues the dQ reduce-adds and returns each ring stage to the
// copies once they have read it; four warpgroups (warps 4-19, one row per
// thread = one tensor-memory lane) form P, then dS, for the query columns
// [32g, 32g + 32) of the tile (warpgroup g), stage the dQ partial, and finally
// write dK and dV, one 32-column chunk per warpgroup.
//
// Per query tile the products are issued as
//     S^T_i, dP^T_i, dV_i, dK_i, dQ_i
// and the elementwise warps form P_i as soon as S^T_i has landed (while dP^T_i
// runs), then dS_i (while dV_i runs), then read out and stage dQ_i (while
// S^T_(i+1) runs). P stays in registers (fp32) from the P step to the dS step.
// Tensor memory: dV [0, 128), dK [128, 256), S^T [256, 384), dP^T [384, 512).
// Each warpgroup writes its P^T (bf16 pairs) over the first 16 of its own 32 S^T
// columns and its dS^T likewise in dP^T, so that none overwrites scores another
// has not loaded yet; the dQ partial then goes over dP^T (after the dK product
// has read dS^T there), so that the next tile's S^T product need not wait for
// it to be read out.
// Shared memory: K_j, V_j; per ring stage Q_i and dO_i; dS (bf16, the dQ
// product's operand); the statistics. The dQ partial of tile i (fp32 [128
// rows][32] boxes) is staged in tile i's own ring stage, whose Q and dO every
// product of the tile has read by then; the stage takes the copies of tile i + 2
// once the TMA engine has read the boxes (which takes thousands of clocks: a
// buffer reused within one tile would stall on it).
#pragma once

#include "ptx.cuh"

namespace bpt {

constexpr int AB_BM = 128;  // query rows per tile
constexpr int AB_BN = 128;  // keys per CTA
constexpr int AB_THREADS = 640;
constexpr int AB_EW_WARPS = 16;  // elementwise warps (four warpgroups)
constexpr int AB_T_DV = 0, AB_T_DK = 128, AB_T_ST = 256, AB_T_DP = 384;

template <int DH>
struct AttnBwdCfg {
  static_assert(DH == 64 || DH == 128, "dh must be 64 or 128");
  static constexpr int ATOM = 128 * 128;            // [128 rows][64 bf16] swizzled box
  static constexpr int TILE = 128 * DH * 2;         // one K, V, Q or dO tile
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_QDO = OFF_V + TILE;      // [2 stages][Q, dO]
  static constexpr int OFF_DS = OFF_QDO + 4 * TILE;  // dS^T [128 keys][128 queries] bf16, two atoms
  static constexpr int OFF_LD = OFF_DS + 2 * ATOM;   // lse2 and D of the query tile, 2 x 128 fp32
  static constexpr int OFF_BAR = OFF_LD + 2 * 128 * 4;
  static constexpr int USED = OFF_BAR + 256 + 1024;
  static constexpr int SMEM_BYTES = USED;
  static_assert(USED <= 232448, "shared memory budget");
};

struct AttnBwdArgs {
  int s, heads, causal;
  int beta0;                // first sequence of this launch
  int n_kv;                 // key/value tiles per (sequence, head)
  const float* lse2;        // [b][heads][s]: max + log2(sum) of the forward, in log2 units
  const float* dsum;        // [b][heads][s]: D = rowsum(dO O)
  float* dq;                // [b][s][h] fp32 accumulator (zeroed by the caller; reached through its tensor map)
  __nv_bfloat16* dk;        // rows (beta * s + t), ld_kv elements apart, head columns
  __nv_bfloat16* dv;
  long long ld_kv;
  int h;
  float scale;              // 1 / sqrt(dh)
  float scale_log2;         // log2(e) / sqrt(dh)
  int* status;
};

__device__ __forceinline__ void ab_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 16 columns of this thread's lane, waited for.
__device__ __forceinline__ void ab_tmem_load16(uint32_t ta, uint32_t (&a)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), "=r"(a[6]), "=r"(a[7]),
        "=r"(a[8]), "=r"(a[9]), "=r"(a[10]), "=r"(a[11]), "=r"(a[12]), "=r"(a[13]), "=r"(a[14]), "=r"(a[15])
      : "r"(ta)
      : "memory");
}

// 8 columns of this thread's lane, waited for.
__device__ __forceinline__ void ab_tmem_store8(uint32_t ta, const uint32_t (&a)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(ta),
      "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(a[4]), "r"(a[5]), "r"(a[6]), "r"(a[7])
      : "memory");
}

__device__ __forceinline__ void ab_named_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Bulk reduce-add of a shared-memory box into global memory by the TMA engine
// (the tensor map gives the global layout, here fp32 with 128B swizzle).
__device__ __forceinline__ void ab_tma_reduce_add_3d(const CUtensorMap* map, uint32_t src, int c0, int c1, int c2) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void ab_bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// the shared-memory sources of every committed bulk group have been read
__device__ __forceinline__ void ab_bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// every committed bulk group has completed
__device__ __forceinline__ void ab_bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }


template <int DH>
__global__ void __launch_bounds__(AB_THREADS, 1)
    attention_bwd_tcgen05(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                          const __grid_constant__ CUtensorMap tmdQ, const AttnBwdArgs args) {
  using C = AttnBwdCfg<DH>;
  constexpr int BOX = 128 * 128;  // one staged dQ box: [128 rows][32 fp32], 128B-swizzled
  constexpr int NBOX = DH / 32;   // dQ boxes per query tile, one per warpgroup g < NBOX
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  const uint32_t kv_full = smem_addr(bars + 0);
  const uint32_t qdo_full0 = smem_addr(bars + 1);   // [2] per ring stage: Q_i and dO_i have landed
  const uint32_t qdo_empty0 = smem_addr(bars + 3);  // [2] the dQ boxes staged over them have been read
  const uint32_t s_ready = smem_addr(bars + 5);     // S^T_i in tensor memory
  const uint32_t p_ready = smem_addr(bars + 6);     // P^T_i in tensor memory
  const uint32_t dp_ready = smem_addr(bars + 7);    // dP^T_i in tensor memory
  const uint32_t ds_ready = smem_addr(bars + 8);    // dS^T_i in tensor memory and dS_i in shared memory
  const uint32_t dq_ready = smem_addr(bars + 9);    // dQ partial of tile i in tensor memory
  const uint32_t dq_free = smem_addr(bars + 10);    // ... read out of tensor memory
  // [2] per ring stage: the dQ boxes of the stage's tile are in place (the next
  // arrival on a stage's barrier needs that stage refilled, which warp 2 allows only
  // after its wait, so a wait can never fall a phase behind)
  const uint32_t dq_staged0 = smem_addr(bars + 11);
  const uint32_t kv_done = smem_addr(bars + 13);
  const uint32_t mma_done = smem_addr(bars + 14);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 15);
  const Abort abort_flag{reinterpret_cast<volatile int*>(bars + 16), args.status};
  float* s_lse = reinterpret_cast<float*>(smem + C::OFF_LD);
  float* s_dsum = s_lse + 128;

  const int warp = warp_id();
  const int lane = lane_id();
  const uint32_t sbase = smem_addr(smem);
  const uint32_t ds_s = sbase + C::OFF_DS;
  auto q_stage = [&](int st) { return sbase + C::OFF_QDO + st * 2 * C::TILE; };
  auto do_stage = [&](int st) { return sbase + C::OFF_QDO + st * 2 * C::TILE + C::TILE; };

  // grid: x = (head, key tile), heaviest key tiles first when causal; z = sequence
  const int head = (int)blockIdx.x % args.heads;
  const int rank = (int)blockIdx.x / args.heads;
  const int jt = rank;  // key tile 0 sees the most query tiles
  const int beta = args.beta0 + blockIdx.z;
  const int j0 = jt * AB_BN;
  const int n_q = (args.s + AB_BM - 1) / AB_BM;
  const int i_first = args.causal ? jt : 0;  // query tiles before the key tile's diagonal see none of its keys
  const int n_it = n_q - i_first;

  if (warp == 0 && lane == 0) {
    mbar_init(kv_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(qdo_full0 + 8 * i, 1);
      mbar_init(qdo_empty0 + 8 * i, 1);
      mbar_init(dq_staged0 + 8 * i, AB_EW_WARPS);
    }
    mbar_init(s_ready, 1);
    mbar_init(p_ready, AB_EW_WARPS);
    mbar_init(dp_ready, 1);
    mbar_init(ds_ready, AB_EW_WARPS);
    mbar_init(dq_ready, 1);
    mbar_init(dq_free, AB_EW_WARPS);
    mbar_init(kv_done, 1);
    mbar_init(mma_done, 1);
    *abort_flag.flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmdO);
    tma_prefetch_desc(&tmdQ);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0 && n_it > 0) {
      // ------------------------------------------------------------ TMA producer
      mbar_arrive_expect_tx(kv_full, 2 * C::TILE);
#pragma unroll
      for (int a = 0; a < DH / 64; ++a) {
        tma_load_3d(sbase + C::OFF_K + a * C::ATOM, &tmK, kv_full, head * DH + a * 64, j0, beta);
        tma_load_3d(sbase + C::OFF_V + a * C::ATOM, &tmV, kv_full, head * DH + a * 64, j0, beta);
      }
      uint32_t issued = 0, par = 0;  // bit st: a copy into stage st was issued / the parity it completes
      for (int it = 0; it < n_it; ++it) {
        const int st = it & 1;
        const uint32_t ph = (uint32_t)(it >> 1) & 1u;
        if (!mbar_wait(qdo_empty0 + 8 * st, ph ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(qdo_full0 + 8 * st, 2 * C::TILE);
        const int i0 = (i_first + it) * AB_BM;
#pragma unroll
        for (int a = 0; a < DH / 64; ++a) {
          tma_load_3d(q_stage(st) + a * C::ATOM, &tmQ, qdo_full0 + 8 * st, head * DH + a * 64, i0, beta);
          tma_load_3d(do_stage(st) + a * C::ATOM, &tmdO, qdo_full0 + 8 * st, head * DH + a * 64, i0, beta);
        }
        issued |= 1u << st;
        par = (par & ~(1u << st)) | (ph << st);
      }
      // no copy may still be writing shared memory when the CTA exits
      volatile int dummy = 0;
      const Abort drain{&dummy, args.status};
      mbar_wait(kv_full, 0, drain);
      for (int i = 0; i < 2; ++i)
        if (issued & (1u << i)) mbar_wait(qdo_full0 + 8 * i, (par >> i) & 1u, drain);
    }
  } else if (warp == 1) {
    if (lane == 0 && n_it > 0) {
      // ------------------------------------------------------------ MMA issuer
      const uint32_t id_kmaj = idesc_bf16_f32(128, 128, 0, 0);  // S^T, dP^T: both operands K-major (dh)
      const uint32_t id_bmn = idesc_bf16_f32(128, DH, 0, 1);    // dV, dK: A from tensor memory, B MN-major
      const uint32_t id_amn = idesc_bf16_f32(128, DH, 1, 1);    // dQ: dS and K both MN-major
      const uint32_t k_s = sbase + C::OFF_K, v_s = sbase + C::OFF_V;
      bool ok = mbar_wait(kv_full, 0, abort_flag);
      for (int it = 0; ok && it < n_it; ++it) {
        const int st = it & 1;
        if (!mbar_wait(qdo_full0 + 8 * st, (uint32_t)(it >> 1) & 1u, abort_flag)) break;
        tc_fence_after();
        // S^T = K Q^T (may overwrite the previous tile's P^T at once: its dV product was issued earlier)
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::ATOM + (kk & 3) * 32;
          mma_bf16_ss(tmem_base + AB_T_ST, smem_desc_sw128(k_s + off, 16, 1024),
                      smem_desc_sw128(q_stage(st) + off, 16, 1024), id_kmaj, kk > 0);
        }
        mma_commit(s_ready);
        // dP^T = V dO^T, once the previous tile's dQ partial (in the dP^T columns) is read out
        if (it > 0 && !mbar_wait(dq_free, (uint32_t)(it - 1) & 1u, abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::ATOM + (kk & 3) * 32;
          mma_bf16_ss(tmem_base + AB_T_DP, smem_desc_sw128(v_s + off, 16, 1024),
                      smem_desc_sw128(do_stage(st) + off, 16, 1024), id_kmaj, kk > 0);
        }
        mma_commit(dp_ready);
        // dV += P^T dO (A from tensor memory: 16 queries = 8 columns per step;
        // queries [32g, 32g + 32) in warpgroup g's columns [32g, 32g + 16))
        if (!mbar_wait(p_ready, (uint32_t)it & 1u, abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < AB_BM / 16; ++kk)
          ab_mma_ts(tmem_base + AB_T_DV, tmem_base + AB_T_ST + (kk >> 1) * 32 + (kk & 1) * 8,
                    smem_desc_sw128(do_stage(st) + kk * 16 * 128, C::ATOM, 1024), id_bmn, (it | kk) != 0);
        // dK += dS^T Q, then the dQ partial = dS K over this key tile (16 keys per
        // step) into the dP^T columns (after the dK product, which reads dS^T there)
        if (!mbar_wait(ds_ready, (uint32_t)it & 1u, abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < AB_BM / 16; ++kk)
          ab_mma_ts(tmem_base + AB_T_DK, tmem_base + AB_T_DP + (kk >> 1) * 32 + (kk & 1) * 8,
                    smem_desc_sw128(q_stage(st) + kk * 16 * 128, C::ATOM, 1024), id_bmn, (it | kk) != 0);
#pragma unroll
        for (int kk = 0; kk < AB_BN / 16; ++kk)
          mma_bf16_ss(tmem_base + AB_T_DP, smem_desc_sw128(ds_s + kk * 16 * 128, C::ATOM, 1024),
                      smem_desc_sw128(k_s + kk * 16 * 128, C::ATOM, 1024), id_amn, kk > 0);
        mma_commit(dq_ready);
      }
      mma_commit(kv_done);
      mma_commit(mma_done);
    }
  } else if (warp == 2) {
    if (lane == 0 && n_it > 0) {
      // ------------------------------------------------------------ dQ reduce-adds
      for (int it = 0; it < n_it; ++it) {
        const int st = it & 1;
        if (!mbar_wait(dq_staged0 + 8 * st, (uint32_t)(it >> 1) & 1u, abort_flag)) break;
        const int i0 = (i_first + it) * AB_BM;
#pragma unroll
        for (int bx = 0; bx < NBOX; ++bx)
          ab_tma_reduce_add_3d(&tmdQ, q_stage(st) + bx * BOX, head * DH + 32 * bx, i0, beta);
        ab_bulk_commit();
        ab_bulk_wait_read();
        mbar_arrive(qdo_empty0 + 8 * st);  // the stage may take the next copies
      }
      ab_bulk_wait_all();  // the last reduce-adds have landed
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ P, dS, dQ, epilogue
    const int g = (warp - 4) >> 2;  // warpgroup: query columns [32g, 32g + 32) of the tile
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // tensor-memory lane: a key (P, dS) or a query (dQ)
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int key = j0 + r;
    const float sl2 = args.scale_log2;
    const long long bh = (long long)beta * args.heads + head;
    // Every warp runs every iteration and every named barrier of it; a wait
    // that gives up only switches the work off (the waits are bounded, and the
    // barriers never see a warp missing).
    // the query tile's statistics: row r of warpgroup 0 holds -lse2, of warpgroup 1
    // scale x D; loaded one tile ahead into a register and staged in shared memory at the
    // top of each tile
    auto stat_of = [&](int i0_) {
      const int t = i0_ + r;
      if (t >= args.s || g > 1) return 0.0f;
      return g == 0 ? -args.lse2[bh * args.s + t] : args.scale * args.dsum[bh * args.s + t];
    };
    // dQ partial of tile t (lane = query row): warpgroup g < NBOX stages
    // its 32 columns as box g, after releasing the tensor memory; warp 2 then adds
    // the boxes into the accumulator. Rows past the sequence are clipped by the
    // tensor map (and hold zeros: their dS is zero).
    auto dq_out = [&](int t, bool run) -> bool {
      const bool got = run && warp_wait(dq_ready, (uint32_t)t & 1u, abort_flag);
      if (!got) return false;
      tc_fence_after();
      // 16 columns at a time; the tensor memory is released once both halves are loaded
      const uint32_t row = q_stage(t & 1) + g * BOX + r * 128;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t o[16];
        if (g < NBOX) ab_tmem_load16(tmem_base + AB_T_DP + g * 32 + 16 * hf + lane_base, o);
        if (hf == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(dq_free);
        }
        if (g < NBOX) {
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const int c = 4 * hf + x;  // 16-byte chunk of the box row
            st_shared_v4(row + (uint32_t)((c ^ (r & 7)) * 16), o[4 * x], o[4 * x + 1], o[4 * x + 2], o[4 * x + 3]);
          }
        }
      }
      if (g < NBOX) fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(dq_staged0 + 8 * (t & 1));
      return true;
    };
    float stat_next = n_it > 0 ? stat_of(i_first * AB_BM) : 0.0f;
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int i0 = (i_first + it) * AB_BM;
      ab_named_sync(1, 32 * AB_EW_WARPS);  // the previous tile's readers of the statistics are done
      if (g == 0)
        s_lse[r] = stat_next;
      else if (g == 1)
        s_dsum[r] = stat_next;
      ok = ok && warp_wait(s_ready, (uint32_t)it & 1u, abort_flag);
      ab_named_sync(1, 32 * AB_EW_WARPS);  // the statistics are in place
      if (it + 1 < n_it) stat_next = stat_of(i0 + AB_BM);
      // ---- P: this row's 32 columns, kept in registers for the dS step
      float pf[32];
      if (ok) {
        tc_fence_after();
        // a query column q is used when it is a real row and (causal) not before this
        // key; in most tiles every column of every row is, and no test is needed
        const bool key_ok = key < args.s;
        const bool all_used = key_ok && i0 + AB_BM <= args.s && (!args.causal || j0 + AB_BN - 1 <= i0);
        const float4* nl4 = reinterpret_cast<const float4*>(s_lse + 32 * g);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t sv[16];
          ab_tmem_load16(tmem_base + AB_T_ST + 32 * g + 16 * hf + lane_base, sv);
          float* pp = pf + 16 * hf;
          uint32_t pk[8];
#pragma unroll
          for (int x4 = 0; x4 < 4; ++x4) {
            const float4 nl = nl4[4 * hf + x4];
            const float nlv[4] = {nl.x, nl.y, nl.z, nl.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) pp[4 * x4 + e] = ex2_approx(fmaf(__uint_as_float(sv[4 * x4 + e]), sl2, nlv[e]));
            if (!all_used) {
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int q = i0 + 32 * g + 16 * hf + 4 * x4 + e;
                const bool use = key_ok && q < args.s && (!args.causal || key <= q);
                pp[4 * x4 + e] = use ? pp[4 * x4 + e] : 0.0f;
              }
            }
            pk[2 * x4] = pack_bf16x2(pp[4 * x4], pp[4 * x4 + 1]);
            pk[2 * x4 + 1] = pack_bf16x2(pp[4 * x4 + 2], pp[4 * x4 + 3]);
          }
          // P^T (bf16 pairs) over the first 16 of this warpgroup's 32 S^T columns:
          // the first half's pairs only overwrite columns loaded already
          ab_tmem_store8(tmem_base + AB_T_ST + 32 * g + 8 * hf + lane_base, pk);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_ready);
      }
      // ---- dS = P (dP - D): into the dP^T columns (the dK product's A) and into
      // the dS buffer (the dQ product's A; the previous tile's dQ product has read it)
      ok = ok && warp_wait(dp_ready, (uint32_t)it & 1u, abort_flag);
      if (ok) {
        tc_fence_after();
        // two 16-column halves (registers: P is live here); dS carries the score scale
        // (scale x P (dP - D)), so that the dK and dQ products need no rescaling
        const float sc = args.scale;
        const float4* d4 = reinterpret_cast<const float4*>(s_dsum + 32 * g);
        const uint32_t row = ds_s + (g >> 1) * C::ATOM + r * 128;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t dp[16];
          ab_tmem_load16(tmem_base + AB_T_DP + 32 * g + 16 * hf + lane_base, dp);
          uint32_t dk[8];
#pragma unroll
          for (int x4 = 0; x4 < 4; ++x4) {
            const float4 dd = d4[4 * hf + x4];
            const float ddv[4] = {dd.x, dd.y, dd.z, dd.w};
            const float* pp = pf + 16 * hf + 4 * x4;
            dk[2 * x4] = pack_bf16x2(pp[0] * fmaf(__uint_as_float(dp[4 * x4]), sc, -ddv[0]),
                                     pp[1] * fmaf(__uint_as_float(dp[4 * x4 + 1]), sc, -ddv[1]));
            dk[2 * x4 + 1] = pack_bf16x2(pp[2] * fmaf(__uint_as_float(dp[4 * x4 + 2]), sc, -ddv[2]),
                                         pp[3] * fmaf(__uint_as_float(dp[4 * x4 + 3]), sc, -ddv[3]));
          }
          // dS^T (bf16 pairs) over the first 16 of this warpgroup's 32 dP^T columns:
          // the first half's pairs only overwrite columns loaded already
          ab_tmem_store8(tmem_base + AB_T_DP + 32 * g + 8 * hf + lane_base, dk);
          // dS^T row of this key into the 128B-swizzled [keys][queries] layout of the dQ operand
#pragma unroll
          for (int t2 = 0; t2 < 2; ++t2) {
            const int chunk = 4 * (g & 1) + 2 * hf + t2;
            st_shared_v4(row + (uint32_t)((chunk ^ (r & 7)) * 16), dk[4 * t2], dk[4 * t2 + 1], dk[4 * t2 + 2],
                         dk[4 * t2 + 3]);
          }
        }
        fence_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(ds_ready);
      }
      // ---- this tile's dQ partial, read out while the next tile's S^T product runs
      ok = dq_out(it, ok);
    }
    // dK and dV of this key tile: lane = key; warpgroup g < DH / 32 the
    // 32-column chunk g
    if (ok && n_it > 0 && warp_wait(kv_done, 0, abort_flag)) {
      tc_fence_after();
      // the loads are warp-collective: every lane loads, only real keys store
      const bool key_row = key < args.s;
      __nv_bfloat16* dkr = args.dk + ((long long)beta * args.s + key) * args.ld_kv + head * DH;
      __nv_bfloat16* dvr = args.dv + ((long long)beta * args.s + key) * args.ld_kv + head * DH;
#pragma unroll 1
      for (int c = g; c < g + 1 && c < DH / 32; ++c) {
        uint32_t a[32], b[32];
        tmem_load32x2(tmem_base + AB_T_DK + c * 32 + lane_base, tmem_base + AB_T_DV + c * 32 + lane_base, a, b);
        if (key_row) {
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const float* fa = reinterpret_cast<const float*>(a) + 8 * x;
            const float* fb = reinterpret_cast<const float*>(b) + 8 * x;
            st_global_v4(dkr + c * 32 + 8 * x, pack_bf16x2(fa[0], fa[1]), pack_bf16x2(fa[2], fa[3]),
                         pack_bf16x2(fa[4], fa[5]), pack_bf16x2(fa[6], fa[7]));
            st_global_v4(dvr + c * 32 + 8 * x, pack_bf16x2(fb[0], fb[1]), pack_bf16x2(fb[2], fb[3]),
                         pack_bf16x2(fb[4], fb[5]), pack_bf16x2(fb[6], fb[7]));
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0 && n_it > 0) {
      volatile int dummy = 0;
      mbar_wait(mma_done, 0, Abort{&dummy, args.status});
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace bpt
