// The FFN side of the BPT layer (Algorithm 1 step 11 of the BPT paper review:
// output projection, first residual, the position-wise FFN and the second
// residual) for every query block of a call in ONE persistent launch.
//
// Rows are taken in groups of gm M-tiles (at most CHAIN_GROUP_MT = 16, i.e.
// 2048 rows; the host picks the largest group whose scratch fits where the
// keys and values were). Each
// group passes through three GEMMs -- out-projection (OP: O Wo + bo + x -> fp32
// hid and its bf16 copy), FFN-up (UP: relu(hid W1 + b1) -> bf16 U) and
// FFN-down (DN: U W2 + b2 + hid -> out) -- whose 128 x 256 output tiles form
// one queue. Step k of the queue holds the DN tiles of group k - 2, the UP
// tiles of group k - 1 and the OP tiles of group k, so a group's three GEMMs
// overlap those of its neighbours and no GEMM's tail idles the SMs. Within a
// segment the tiles run N-major over the group's M-tiles, which then share
// each weight tile in L2.
//
// CTA c takes tiles c, c + grid, c + 2 grid, ... in order; one CTA per SM, all
// resident. A tile waits only on tiles earlier in the queue: the UP tiles of
// a group wait until every OP tile of the group has been stored (they sit a
// whole step later), the DN tiles until every UP tile of the group has, and a
// group reusing a scratch slot waits until the DN tiles of the slot's
// previous group have read it. So the smallest unfinished tile always has its
// inputs and progress is guaranteed. Each CTA remembers the latest group it
// has seen complete for each GEMM, so it polls a counter about once per group
// instead of once per tile. The waits are bounded (the kernel records
// BPT_ERR_TIMEOUT and stops, like every wait of this library).
//
// Hand-over between CTAs: an epilogue warp stores its part of a tile, fences
// (device scope) and adds 1 with release semantics to the tile's counter; the
// producer of a dependent tile polls the counter with acquire semantics, then
// orders the generic-proxy stores before its tensor-memory-access (async
// proxy) loads with a proxy fence. The residual hid is read with L2-only
// loads, since its slot held another group's rows earlier in the launch.
//
// Scratch: CHAIN_HID_SLOTS slots of a group's fp32 hid and bf16 hid copy and
// CHAIN_U_SLOTS slots of its bf16 U, used round-robin by group (fewer when the
// call has fewer groups). With three hid slots the OP tiles of group g wait
// for the DN tiles of group g - 3, which sit a whole step earlier in the
// queue; with two U slots the UP tiles of group g wait for the DN tiles of
// group g - 2, also a step earlier, so these waits rarely stall.
#pragma once

#include "gemm.cuh"

namespace bpt {

constexpr int CHAIN_GROUP_MT = 16;  // largest group: 16 M-tiles (2048 rows)
constexpr int CHAIN_HID_SLOTS = 3;
constexpr int CHAIN_U_SLOTS = 2;

enum ChainKind { CK_OP = 0, CK_UP = 1, CK_DN = 2 };

struct ChainArgs {
  long long M;     // rows of the call (b * s)
  int h, f;        // model width and FFN width
  int m_tiles;     // ceil(M / 128)
  int gm;          // M-tiles per group (1 .. CHAIN_GROUP_MT)
  int groups;      // ceil(m_tiles / gm)
  int hid_slots, u_slots;
  int n_op, n_up, n_dn;  // N-tiles of each GEMM
  const __nv_bfloat16* x;  // residual input [M, h]
  const __nv_bfloat16 *bo, *b1, *b2;
  float* hid;              // [hid_slots * gm * 128, h] fp32
  __nv_bfloat16* hb;       // [hid_slots * gm * 128, h] bf16
  __nv_bfloat16* u;        // [u_slots * gm * 128, f] bf16
  float* out;              // [M, h] fp32
  unsigned* op_cnt;        // [groups]: epilogue warps done with the group's OP tiles
  unsigned* up_cnt;        // [groups]
  unsigned* dn_cnt;        // [groups]
  int* status;
  // one-launch layer only (else null): attention's count of stored warps per
  // group, complete at 4 x (the group's M-tiles) x att_heads
  const unsigned* att_cnt;
  int att_heads;
};

struct ChainTile {
  int kind, g, mt, nt;  // mt: M-tile within the group
};

// The queue is a pure function of the arguments; host code (the schedule's
// tests) evaluates the same functions.
__host__ __device__ __forceinline__ int chain_group_mt(const ChainArgs& a, int g) {
  const int rest = a.m_tiles - g * a.gm;
  return rest < a.gm ? rest : a.gm;
}

__host__ __device__ __forceinline__ long long chain_step_size(const ChainArgs& a, int k) {
  long long n = 0;
  if (k - 2 >= 0 && k - 2 < a.groups) n += (long long)chain_group_mt(a, k - 2) * a.n_dn;
  if (k - 1 >= 0 && k - 1 < a.groups) n += (long long)chain_group_mt(a, k - 1) * a.n_up;
  if (k < a.groups) n += (long long)chain_group_mt(a, k) * a.n_op;
  return n;
}

// Tile at position r of step k: the DN tiles of group k - 2, then the UP
// tiles of group k - 1, then the OP tiles of group k.
__host__ __device__ __forceinline__ ChainTile chain_in_step(const ChainArgs& a, int k, long long r) {
  ChainTile t{};
#pragma unroll
  for (int s = 0; s < 3; ++s) {
    const int g = k - 2 + s;
    if (g < 0 || g >= a.groups) continue;
    const int n = s == 0 ? a.n_dn : (s == 1 ? a.n_up : a.n_op);
    const int gm = chain_group_mt(a, g);
    const long long sz = (long long)gm * n;
    if (r < sz) {
      t.kind = s == 0 ? CK_DN : (s == 1 ? CK_UP : CK_OP);
      t.g = g;
      t.nt = (int)(r / gm);
      t.mt = (int)(r - (long long)t.nt * gm);
      return t;
    }
    r -= sz;
  }
  t.kind = -1;
  return t;
}

// Tile number `idx` of the queue. Steps 2 .. k_full all have three whole
// groups and the same size, so they are skipped by one division.
__host__ __device__ __forceinline__ ChainTile chain_tile(const ChainArgs& a, long long idx) {
  const bool last_full = a.m_tiles % a.gm == 0;
  const int k_full = last_full ? a.groups - 1 : a.groups - 2;  // last step whose three groups are whole
  long long off = 0;
  for (int k = 0; k <= a.groups + 1; ++k) {
    if (k == 2 && k_full >= 2) {
      const long long S = (long long)a.gm * (a.n_dn + a.n_up + a.n_op);
      const long long n = k_full - 1;  // steps 2 .. k_full
      if (idx < off + n * S) {
        const long long q = (idx - off) / S;
        return chain_in_step(a, 2 + (int)q, idx - off - q * S);
      }
      off += n * S;
      k = k_full;
      continue;
    }
    const long long sz = chain_step_size(a, k);
    if (idx < off + sz) return chain_in_step(a, k, idx - off);
    off += sz;
  }
  ChainTile t{};
  t.kind = -1;
  return t;
}

__host__ __device__ __forceinline__ long long chain_num_tiles(const ChainArgs& a) {
  return (long long)a.m_tiles * (a.n_op + a.n_up + a.n_dn);
}

// 32 fp32 values read through L2 only (the line may have been written by
// another SM since this SM last cached it).
__device__ __forceinline__ void load32_f32_cg(const float* p, float (&v)[32]) {
  const float4* s = reinterpret_cast<const float4*>(p);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 t = __ldcg(s + i);
    v[4 * i] = t.x; v[4 * i + 1] = t.y; v[4 * i + 2] = t.z; v[4 * i + 3] = t.w;
  }
}

// One CTA's share of the queue: CTA `cta` of `n_ctas` takes tiles cta,
// cta + n_ctas, ... Warps 0-5 work (producer, MMA issuer, four epilogue warps);
// any further warps of the block only pass the final barrier.
__device__ __forceinline__ void ffn_chain_body(const CUtensorMap& tmO, const CUtensorMap& tmHb, const CUtensorMap& tmU,
                                               const CUtensorMap& tmWo, const CUtensorMap& tmW1,
                                               const CUtensorMap& tmW2, const ChainArgs& args, int cta, int n_ctas) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + GEMM_STAGES * GEMM_STAGE_BYTES);
  const uint32_t full0 = smem_addr(bars);
  const uint32_t empty0 = smem_addr(bars + GEMM_STAGES);
  const uint32_t tfull0 = smem_addr(bars + 2 * GEMM_STAGES);
  const uint32_t tempty0 = smem_addr(bars + 2 * GEMM_STAGES + 2);
  const uint32_t mma_done = smem_addr(bars + 2 * GEMM_STAGES + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * GEMM_STAGES + 5);
  const Abort abort_flag{reinterpret_cast<volatile int*>(bars + 2 * GEMM_STAGES + 6), args.status};

  const int warp = warp_id();
  const int lane = lane_id();
  const uint32_t smem_base = smem_addr(smem);
  const int group_rows = args.gm * GEMM_BM;

  if (warp == 0 && lane == 0) {
    for (int i = 0; i < GEMM_STAGES; ++i) {
      mbar_init(full0 + 8 * i, 1);
      mbar_init(empty0 + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(tfull0 + 8 * i, 1);
      mbar_init(tempty0 + 8 * i, 4);
    }
    mbar_init(mma_done, 1);
    *abort_flag.flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmO);
    tma_prefetch_desc(&tmHb);
    tma_prefetch_desc(&tmU);
    tma_prefetch_desc(&tmWo);
    tma_prefetch_desc(&tmW1);
    tma_prefetch_desc(&tmW2);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), GEMM_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const long long num_tiles = chain_num_tiles(args);
  auto k_blocks_of = [&](int kind) { return (kind == CK_DN ? args.f : args.h) / GEMM_BK; };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, last_parity = 0;
      // latest group seen complete, per GEMM (groups complete in order of the
      // queue's steps, so "group g complete" covers the groups before it)
      int done_op = -1, done_up = -1, done_dn = -1, done_att = -1;
      auto need = [&](int& done, const unsigned* cnt, int g, int n_tiles_per_mt) -> bool {
        if (g <= done) return true;
        if (!counter_wait(cnt + g, 4u * chain_group_mt(args, g) * n_tiles_per_mt, abort_flag)) return false;
        done = g;
        return true;
      };
      for (long long t = cta; t < num_tiles; t += n_ctas) {
        const ChainTile ct = chain_tile(args, t);
        // inputs of this tile, and the scratch slot it writes, are ready
        const int d0 = done_op, d1 = done_up, d2 = done_dn, d3 = done_att;
        bool ok = true;
        if (ct.kind == CK_OP) {
          if (args.att_cnt != nullptr) ok = need(done_att, args.att_cnt, ct.g, args.att_heads);
          if (ok && ct.g >= args.hid_slots) ok = need(done_dn, args.dn_cnt, ct.g - args.hid_slots, args.n_dn);
        } else if (ct.kind == CK_UP) {
          ok = need(done_op, args.op_cnt, ct.g, args.n_op);
          if (ok && ct.g >= args.u_slots) ok = need(done_dn, args.dn_cnt, ct.g - args.u_slots, args.n_dn);
        } else {
          ok = need(done_up, args.up_cnt, ct.g, args.n_up);
        }
        if (!ok) break;
        // another CTA's stores become visible to this thread's tensor-memory-
        // access loads once a counter has been acquired
        if (d0 != done_op || d1 != done_up || d2 != done_dn || d3 != done_att) fence_proxy_async_global();
        const CUtensorMap* ta = ct.kind == CK_OP ? &tmO : (ct.kind == CK_UP ? &tmHb : &tmU);
        const CUtensorMap* tb = ct.kind == CK_OP ? &tmWo : (ct.kind == CK_UP ? &tmW1 : &tmW2);
        const int a_row = ct.kind == CK_OP ? ct.g * group_rows + ct.mt * GEMM_BM
                                           : (ct.g % (ct.kind == CK_UP ? args.hid_slots : args.u_slots)) * group_rows +
                                                 ct.mt * GEMM_BM;
        const int n0 = ct.nt * GEMM_BN;
        const int kbs = k_blocks_of(ct.kind);
        for (int kb = 0; kb < kbs; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1, abort_flag)) { ok = false; break; }
          const uint32_t fb = full0 + 8 * stage;
          const uint32_t sa = smem_base + stage * GEMM_STAGE_BYTES;
          mbar_arrive_expect_tx(fb, GEMM_STAGE_BYTES);
          tma_load_2d(sa, ta, fb, kb * GEMM_BK, a_row);
#pragma unroll
          for (int j = 0; j < GEMM_BN / 64; ++j)
            tma_load_2d(sa + GEMM_A_BYTES + j * GEMM_B_BOX_BYTES, tb, fb, n0 + 64 * j, kb * GEMM_BK);
          issued |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == GEMM_STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
      }
      // never leave with tile copies still landing in shared memory
      for (int i = 0; i < GEMM_STAGES; ++i)
        if (issued & (1u << i)) {
          volatile int dummy = 0;
          mbar_wait(full0 + 8 * i, (last_parity >> i) & 1u, Abort{&dummy, args.status});
        }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      const uint32_t idesc = idesc_bf16_f32(GEMM_BM, GEMM_BN, 0, 1);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      for (long long t = cta; t < num_tiles; t += n_ctas, ++it) {
        const ChainTile ct = chain_tile(args, t);
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!mbar_wait(tempty0 + 8 * acc, acc_phase ^ 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + acc * GEMM_BN;
        bool ok = true;
        const int kbs = k_blocks_of(ct.kind);
        for (int kb = 0; kb < kbs; ++kb) {
          if (!mbar_wait(full0 + 8 * stage, phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_base + stage * GEMM_STAGE_BYTES;
          const uint32_t sb = sa + GEMM_A_BYTES;
#pragma unroll
          for (int kk = 0; kk < GEMM_BK / 16; ++kk) {
            const uint64_t adesc = smem_desc_sw128(sa + kk * 32, 16, 1024);
            const uint64_t bdesc = smem_desc_sw128(sb + kk * 16 * 128, GEMM_B_BOX_BYTES, 1024);
            mma_bf16_ss(d, adesc, bdesc, idesc, (kb | kk) != 0);
          }
          mma_commit(empty0 + 8 * stage);
          if (++stage == GEMM_STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        mma_commit(tfull0 + 8 * acc);
      }
      mma_commit(mma_done);
    }
  } else if (warp < 6) {
    // -------------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    int it = 0;
    for (long long t = cta; t < num_tiles; t += n_ctas, ++it) {
      const ChainTile ct = chain_tile(args, t);
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      if (!warp_wait(tfull0 + 8 * acc, acc_phase, abort_flag)) break;
      tc_fence_after();
      const int r_local = ct.mt * GEMM_BM + quarter * 32 + lane;  // row within the group
      const long long grow = (long long)ct.g * group_rows + r_local;  // row of the call
      const long long hrow = (long long)(ct.g % args.hid_slots) * group_rows + r_local;
      const long long urow = (long long)(ct.g % args.u_slots) * group_rows + r_local;
      const int n_cols = ct.kind == CK_UP ? args.f : args.h;
      const uint32_t taddr = tmem_base + acc * GEMM_BN + ((uint32_t)(quarter * 32) << 16);
#pragma unroll 1
      for (int c = 0; c < GEMM_BN / 32; ++c) {
        uint32_t r[32];
        tmem_load32(taddr + c * 32, r);
        const int col = ct.nt * GEMM_BN + c * 32;
        if (grow < args.M && col < n_cols) {
          float v[32], bias[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
          if (ct.kind == CK_OP) {
            float x[32];
            load32(args.bo, 0, col, bias);
            load32(args.x, 0, grow * args.h + col, x);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] += bias[i] + x[i];
            store32_f32(args.hid + hrow * args.h + col, v);
            store32_bf16(args.hb + hrow * args.h + col, v);
          } else if (ct.kind == CK_UP) {
            load32(args.b1, 0, col, bias);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = fmaxf(v[i] + bias[i], 0.0f);
            store32_bf16(args.u + urow * args.f + col, v);
          } else {
            float hid[32];
            load32(args.b2, 0, col, bias);
            load32_f32_cg(args.hid + hrow * args.h + col, hid);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] += bias[i] + hid[i];
            store32_f32(args.out + grow * args.h + col, v);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty0 + 8 * acc);
      // publish this warp's part of the tile
      __threadfence();
      __syncwarp();
      if (lane == 0)
        red_release_add((ct.kind == CK_OP ? args.op_cnt : (ct.kind == CK_UP ? args.up_cnt : args.dn_cnt)) + ct.g, 1u);
    }
  }

  __syncthreads();
  if (warp == 1) {
    if (lane == 0) {
      volatile int dummy = 0;
      mbar_wait(mma_done, 0, Abort{&dummy, args.status});
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, GEMM_TMEM_COLS);
  }
}

__global__ void __launch_bounds__(GEMM_THREADS, 1)
    ffn_chain_tcgen05(const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmHb,
                      const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmWo,
                      const __grid_constant__ CUtensorMap tmW1, const __grid_constant__ CUtensorMap tmW2,
                      const ChainArgs args) {
  ffn_chain_body(tmO, tmHb, tmU, tmWo, tmW1, tmW2, args, (int)blockIdx.x, (int)gridDim.x);
}

}  // namespace bpt
