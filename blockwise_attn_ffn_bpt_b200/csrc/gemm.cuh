// Persistent tcgen05 GEMM with fused epilogues for the projections of the BPT
// layer and of its FFN block's backward: D[M, N] = A[M, K] * B[K, N], bf16
// operands, fp32 accumulation in tensor memory. Forward: A row-major [M, K]
// (K-major operand), B = [in, out] weights row-major [K, N] (MN-major
// operand). Backward: B = a weight used transposed, stored [N, K] (K-major,
// B_MN = 0), and, for weight gradients, A = an activation used transposed,
// stored [K, M] (MN-major, A_MN = 1).
//
// Roles (192 threads): warp 0 issues TMA tile loads into a STAGES-deep ring,
// one thread of warp 1 issues tcgen05.mma into one of two TMEM accumulators,
// warps 2-5 read the finished accumulator (warp w owns TMEM lanes
// 32*(w%4) .. +31, one output row per thread) and run the epilogue while the
// next tile's MMAs proceed into the other accumulator.
#pragma once

#include "ptx.cuh"

namespace bpt {

constexpr int GEMM_BM = 128;
constexpr int GEMM_BN = 256;
constexpr int GEMM_BK = 64;
constexpr int GEMM_STAGES = 4;
constexpr int GEMM_THREADS = 192;
constexpr int GEMM_A_BYTES = GEMM_BM * GEMM_BK * 2;  // 16 KB, one 128B-swizzle atom column
constexpr int GEMM_B_BOX_BYTES = GEMM_BK * 64 * 2;   // 8 KB: 64 K-rows x 64 N-columns
constexpr int GEMM_B_BYTES = GEMM_BK * GEMM_BN * 2;  // 32 KB: four boxes along N
constexpr int GEMM_STAGE_BYTES = GEMM_A_BYTES + GEMM_B_BYTES;
constexpr int GEMM_TMEM_COLS = 2 * GEMM_BN;          // two fp32 accumulators
constexpr int GEMM_GROUP_M = 16;                     // raster: 16 M-tiles share B tiles in L2
constexpr int GEMM_SMEM_BYTES = GEMM_STAGES * GEMM_STAGE_BYTES + 1024 + 256;

enum EpiMode {
  EPI_QKV = 0,       // + bqkv -> bf16 Q | K | V
  EPI_OUTPROJ = 1,   // + bo + x (first residual) -> fp32 hid and its bf16 copy (wave scratch)
  EPI_FFN_UP = 2,    // + b1, ReLU -> bf16 U
  EPI_FFN_DOWN = 3,  // + b2 + hid (second residual) -> fp32 out
  EPI_BWD_DA = 4,    // (dy W2^T) masked by U > 0 (the ReLU's derivative; no mask without U) -> bf16 da
  EPI_BWD_DHID = 5,  // + dy (the residual's gradient) -> fp32 dhid
  EPI_GRAD = 6,      // -> fp32 weight gradient, added to what is there when accumulate is set
};

struct GemmArgs {
  int M, N, K;
  int m_tiles, n_tiles;
  const void* bias;  // [N], bf16 or fp32
  int bias_f32;
  // EPI_QKV
  __nv_bfloat16* q;
  long long ldq;     // elements between Q rows
  __nv_bfloat16* k;
  __nv_bfloat16* v;
  long long ldkv;
  int h;
  // EPI_OUTPROJ residual input x
  const void* resid;
  int resid_f32;
  long long ld_resid;
  // fp32 hid of the wave's rows (OUTPROJ writes it, FFN_DOWN reads it)
  float* hid;
  long long ld_hid;
  // fp32 layer output (FFN_DOWN)
  float* out;
  long long ld_out;
  long long row0;    // flat row of local row 0 (for x and out)
  // bf16 destination of OUTPROJ (hid copy) and FFN_UP (U)
  __nv_bfloat16* dst;
  long long ld_dst;
  // Split products (fp32 inputs): B stacks bf16 parts of the weights along K
  // and A is read again for each part. a_split 0: A's K block = kb; 1: kb
  // modulo a_kb (A against [W_hi; W_lo]); 2: kb modulo a_kb for the first
  // 2 a_kb blocks, then kb - a_kb (A = [x_hi | x_lo] against [W_hi; W_lo; W_hi]).
  int a_split;
  int a_kb;  // K blocks of one copy of A
  // backward: U (EPI_BWD_DA's mask), dy fp32 (EPI_BWD_DHID), accumulate (EPI_GRAD)
  const __nv_bfloat16* mask_u;
  long long ld_mask;
  const float* dy;
  long long ld_dy;
  int accumulate;
  int* status;  // status word of the launching stream
};

// K block of A that pairs with K block kb of B
__device__ __forceinline__ int a_block(const GemmArgs& a, int kb) {
  if (a.a_split == 0) return kb;
  if (a.a_split == 1 || kb < 2 * a.a_kb) return kb % a.a_kb;
  return kb - a.a_kb;
}

// 32 consecutive values (columns col .. col+31) of one row.
__device__ __forceinline__ void load32(const void* p, int f32, long long off, float (&v)[32]) {
  if (f32) {
    const float4* s = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p) + off);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float4 t = s[i];
      v[4 * i] = t.x; v[4 * i + 1] = t.y; v[4 * i + 2] = t.z; v[4 * i + 3] = t.w;
    }
  } else {
    const uint4* s = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p) + off);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint4 t = s[i];
      const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        __nv_bfloat162 b2 = *reinterpret_cast<const __nv_bfloat162*>(&w[j]);
        float2 f = __bfloat1622float2(b2);
        v[8 * i + 2 * j] = f.x;
        v[8 * i + 2 * j + 1] = f.y;
      }
    }
  }
}

__device__ __forceinline__ void store32_bf16(__nv_bfloat16* dst, const float (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
    st_global_v4(dst + 8 * i, pack_bf16x2(v[8 * i], v[8 * i + 1]), pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                 pack_bf16x2(v[8 * i + 4], v[8 * i + 5]), pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
}

__device__ __forceinline__ void store32_f32(float* dst, const float (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 8; ++i)
    st_global_v4(dst + 4 * i, __float_as_uint(v[4 * i]), __float_as_uint(v[4 * i + 1]), __float_as_uint(v[4 * i + 2]),
                 __float_as_uint(v[4 * i + 3]));
}

template <int MODE>
__device__ __forceinline__ void gemm_epilogue(const GemmArgs& a, int row, int col, float (&v)[32]) {
  float bias[32];
  if constexpr (MODE <= EPI_FFN_DOWN) load32(a.bias, a.bias_f32, col, bias);
  if constexpr (MODE == EPI_QKV) {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] += bias[i];
    const int part = col / a.h;
    const int c = col - part * a.h;
    __nv_bfloat16* dst = part == 0 ? a.q + (long long)row * a.ldq + c
                                   : (part == 1 ? a.k : a.v) + (long long)row * a.ldkv + c;
    store32_bf16(dst, v);
  } else if constexpr (MODE == EPI_OUTPROJ) {
    float x[32];
    const long long grow = a.row0 + row;
    load32(a.resid, a.resid_f32, grow * a.ld_resid + col, x);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] += bias[i] + x[i];
    store32_f32(a.hid + (long long)row * a.ld_hid + col, v);
    store32_bf16(a.dst + (long long)row * a.ld_dst + col, v);
  } else if constexpr (MODE == EPI_FFN_UP) {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = fmaxf(v[i] + bias[i], 0.0f);
    store32_bf16(a.dst + (long long)row * a.ld_dst + col, v);
  } else if constexpr (MODE == EPI_FFN_DOWN) {
    float hid[32];
    load32(a.hid + (long long)row * a.ld_hid + col, 1, 0, hid);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] += bias[i] + hid[i];
    float* o = a.out + (a.row0 + row) * a.ld_out + col;
    store32_f32(o, v);
  } else if constexpr (MODE == EPI_BWD_DA) {
    if (a.mask_u != nullptr) {
      float u[32];
      load32(a.mask_u, 0, (long long)row * a.ld_mask + col, u);
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = u[i] > 0.0f ? v[i] : 0.0f;
    }
    store32_bf16(a.dst + (long long)row * a.ld_dst + col, v);
  } else if constexpr (MODE == EPI_BWD_DHID) {
    float dy[32];
    load32(a.dy, 1, (long long)row * a.ld_dy + col, dy);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] += dy[i];
    store32_f32(a.out + (long long)row * a.ld_out + col, v);
    if (a.dst != nullptr) store32_bf16(a.dst + (long long)row * a.ld_dst + col, v);  // its bf16 copy, if asked
  } else {
    float* o = a.out + (long long)row * a.ld_out + col;
    if (a.accumulate) {
      float old[32];
      load32(o, 1, 0, old);
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] += old[i];
    }
    store32_f32(o, v);
  }
}

__device__ __forceinline__ void gemm_tile_coords(int t, int m_tiles, int n_tiles, int& mt, int& nt) {
  const int group_size = GEMM_GROUP_M * n_tiles;
  const int group = t / group_size;
  const int first_m = group * GEMM_GROUP_M;
  const int gm = min(GEMM_GROUP_M, m_tiles - first_m);
  const int r = t - group * group_size;
  mt = first_m + r % gm;
  nt = r / gm;
}

// A_MN = 1: A stored [K, M] (M contiguous), loaded as two [64 k][64 m] boxes
// per stage; otherwise [M, K], one [128 m][64 k] box. B_MN = 1: B stored [K,
// N], four [64 k][64 n] boxes; otherwise [N, K], one [256 n][64 k] box. Both
// are 128-byte swizzled; the descriptors follow the operand's majorness.
template <int MODE, int A_MN = 0, int B_MN = 1>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_bf16_tcgen05(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + GEMM_STAGES * GEMM_STAGE_BYTES);
  // barrier slots
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
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), GEMM_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int num_tiles = args.m_tiles * args.n_tiles;
  const int k_blocks = args.K / GEMM_BK;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, last_parity = 0;
      for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
        int mt, nt;
        gemm_tile_coords(t, args.m_tiles, args.n_tiles, mt, nt);
        const int m0 = mt * GEMM_BM, n0 = nt * GEMM_BN;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1, abort_flag)) goto producer_done;
          const uint32_t fb = full0 + 8 * stage;
          const uint32_t sa = smem_base + stage * GEMM_STAGE_BYTES;
          mbar_arrive_expect_tx(fb, GEMM_STAGE_BYTES);
          if constexpr (A_MN) {
#pragma unroll
            for (int j = 0; j < GEMM_BM / 64; ++j)
              tma_load_2d(sa + j * GEMM_B_BOX_BYTES, &tmA, fb, m0 + 64 * j, kb * GEMM_BK);
          } else {
            tma_load_2d(sa, &tmA, fb, a_block(args, kb) * GEMM_BK, m0);
          }
          if constexpr (B_MN) {
#pragma unroll
            for (int j = 0; j < GEMM_BN / 64; ++j)
              tma_load_2d(sa + GEMM_A_BYTES + j * GEMM_B_BOX_BYTES, &tmB, fb, n0 + 64 * j, kb * GEMM_BK);
          } else {
            tma_load_2d(sa + GEMM_A_BYTES, &tmB, fb, kb * GEMM_BK, n0);
          }
          issued |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == GEMM_STAGES) { stage = 0; phase ^= 1; }
        }
      }
    producer_done:
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
      const uint32_t idesc = idesc_bf16_f32(GEMM_BM, GEMM_BN, A_MN, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++it) {
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!mbar_wait(tempty0 + 8 * acc, acc_phase ^ 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + acc * GEMM_BN;
        bool ok = true;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(full0 + 8 * stage, phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_base + stage * GEMM_STAGE_BYTES;
          const uint32_t sb = sa + GEMM_A_BYTES;
#pragma unroll
          for (int kk = 0; kk < GEMM_BK / 16; ++kk) {
            // K-major: the 16-deep slice starts 32 bytes further along each
            // 128-byte row; MN-major: 16 rows (of 128 bytes) further, with the
            // 64-wide boxes GEMM_B_BOX_BYTES apart
            const uint64_t adesc = A_MN ? smem_desc_sw128(sa + kk * 16 * 128, GEMM_B_BOX_BYTES, 1024)
                                        : smem_desc_sw128(sa + kk * 32, 16, 1024);
            const uint64_t bdesc = B_MN ? smem_desc_sw128(sb + kk * 16 * 128, GEMM_B_BOX_BYTES, 1024)
                                        : smem_desc_sw128(sb + kk * 32, 16, 1024);
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
  } else {
    // -------------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    int it = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++it) {
      int mt, nt;
      gemm_tile_coords(t, args.m_tiles, args.n_tiles, mt, nt);
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      if (!warp_wait(tfull0 + 8 * acc, acc_phase, abort_flag)) break;
      tc_fence_after();
      const int row = mt * GEMM_BM + quarter * 32 + lane;
      const uint32_t taddr = tmem_base + acc * GEMM_BN + ((uint32_t)(quarter * 32) << 16);
#pragma unroll 1
      for (int c = 0; c < GEMM_BN / 32; ++c) {
        uint32_t r[32];
        tmem_load32(taddr + c * 32, r);
        const int col = nt * GEMM_BN + c * 32;
        if (row < args.M && col < args.N) {
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
          gemm_epilogue<MODE>(args, row, col, v);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty0 + 8 * acc);
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

}  // namespace bpt
