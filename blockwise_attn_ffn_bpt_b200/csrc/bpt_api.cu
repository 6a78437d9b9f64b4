// C ABI of the BPT layer forward: argument checks, workspace layout, TMA
// descriptors, the wave schedule and the kernel launches.
//
// Schedule of one call (Algorithm 1 of the BPT paper review, section 3):
//   1. QKV projection over the whole sequence (step 1): K and V go to the
//      workspace, Q is parked inside `out` (a bf16 Q row fits in the first half
//      of its fp32 output row and is consumed before that row is written).
//   2. Blockwise attention of every query tile over all of its key/value tiles
//      (steps 4-10) in one launch; each CTA writes its output O over the Q of
//      its own rows and head inside `out`.
//   3. For each wave of query blocks (a whole number of q_block rows, sized
//      by a tile-round model of the GEMMs): Wo + bo + x (first residual, fp32
//      hid in the wave scratch), W1 + b1 + ReLU (bf16 U) and W2 + b2 + hid
//      (second residual, into `out`) on the wave's rows (step 11). Scratch is
//      bounded by the wave, not by s, and reuses the K/V region, dead once
//      attention has run: the full-sequence 4h FFN intermediate and the s x s
//      scores never exist.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "attention.cuh"
#include "attention_bwd.cuh"
#include "layer_mega.cuh"
#include "attention_pair.cuh"
#include "bpt.h"
#include "ffn_chain.cuh"
#include "gemm.cuh"
#include "gemm_pair.cuh"
#include "row_pieces.h"

// The bf16 forward GEMMs run on SM pairs (gemm_pair.cuh) when this is 1, on
// single SMs (gemm.cuh) when it is 0. Measured on B200 at b=1, s=32768,
// h=4096: QKV 2.46 -> 2.15 ms, FFN-up 3.39 -> 2.92 ms, FFN-down 3.34 -> 2.90
// ms, out-projection 1.03 -> 0.95 ms (the single-SM kernel's copies and MMA
// reads exceed what shared memory delivers per clock; a pair halves B's).
#ifndef BPT_PAIR_GEMM
#define BPT_PAIR_GEMM 1
#endif
// Attention with dh = 128 runs on SM pairs (attention_pair.cuh) when this is
// 1, on single SMs (attention.cuh) when it is 0. The pair form passes the same
// parity tests but measured 20-30% slower on B200 (b=1, s=32768, h=4096:
// 10.8 ms against 8.7-9.0 ms): each of its MMA steps waits for the slower of
// two CTAs' softmax, which costs more than the halved shared-memory traffic
// of its S MMAs gains.
#ifndef BPT_PAIR_ATTENTION
#define BPT_PAIR_ATTENTION 0
#endif

namespace bpt {
namespace {

std::atomic<uint64_t> g_launches{0};

// ------------------------------------------------------------- timing log
struct TimedLaunch {
  const char* name;
  cudaEvent_t start, stop;
};
std::mutex g_timing_mu;
bool g_timing = false;
std::vector<TimedLaunch> g_timed;

struct LaunchScope {
  TimedLaunch rec{};
  bool on = false;
  cudaStream_t stream;
  LaunchScope(const char* name, cudaStream_t st) : stream(st) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    std::lock_guard<std::mutex> lk(g_timing_mu);
    if (!g_timing) return;
    on = true;
    rec.name = name;
    cudaEventCreate(&rec.start);
    cudaEventCreate(&rec.stop);
    cudaEventRecord(rec.start, stream);
  }
  ~LaunchScope() {
    if (!on) return;
    cudaEventRecord(rec.stop, stream);
    std::lock_guard<std::mutex> lk(g_timing_mu);
    g_timed.push_back(rec);
  }
};

// ------------------------------------------------------------- driver entry
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// bf16 tensor map with 128-byte swizzle; dims/strides innermost first,
// strides in bytes for dims 1.. (dim 0 is contiguous).
bool make_map(CUtensorMap* map, const void* base, int rank, const uint64_t* dims, const uint64_t* strides,
              const uint32_t* box, CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t gd[3], gs[2];
  cuuint32_t bx[3], es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) gs[i] = strides[i];
  CUresult r = enc(map, dtype, rank, const_cast<void*>(base), gd, gs, bx, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// [rows, cols] bf16 row-major with `ld` elements between rows, loaded as
// [box_rows][64] boxes.
bool map_rows(CUtensorMap* m, const void* base, long long rows, long long cols, long long ld, uint32_t box_rows) {
  const uint64_t dims[2] = {(uint64_t)cols, (uint64_t)rows};
  const uint64_t strides[1] = {(uint64_t)ld * 2};
  const uint32_t box[2] = {64, box_rows};
  return make_map(m, base, 2, dims, strides, box);
}

// [b, s, cols] bf16 with `ld` elements between rows, [box_rows][64] boxes;
// rows past s of a sequence read as zero.
bool map_seq(CUtensorMap* m, const void* base, int b, int s, int cols, long long ld, uint32_t box_rows = 128) {
  const uint64_t dims[3] = {(uint64_t)cols, (uint64_t)s, (uint64_t)b};
  const uint64_t strides[2] = {(uint64_t)ld * 2, (uint64_t)ld * 2 * (uint64_t)s};
  const uint32_t box[3] = {64, box_rows, 1};
  return make_map(m, base, 3, dims, strides, box);
}

// [b, s, cols] fp32 (rows `cols` apart) as [128 rows][32] boxes: the dQ
// accumulator of the attention backward, which the TMA engine adds into (rows
// past s of a sequence are clipped).
bool map_seq_f32(CUtensorMap* m, float* base, int b, int s, int cols) {
  const uint64_t dims[3] = {(uint64_t)cols, (uint64_t)s, (uint64_t)b};
  const uint64_t strides[2] = {(uint64_t)cols * 4, (uint64_t)cols * 4 * (uint64_t)s};
  const uint32_t box[3] = {32, 128, 1};
  return make_map(m, base, 3, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_FLOAT32);
}

// ------------------------------------------------------------- device info
struct DeviceInfo {
  bool checked = false;
  bool ok = false;
  bool mega_ok = false;  // the one-launch layer kernel was built with the attention's register count
  int sms = 0;
};
std::mutex g_dev_mu;
DeviceInfo g_dev[64];

int check_device(int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return BPT_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.checked) {
    int major = 0, minor = 0, n = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return BPT_ERR_CUDA;
    d.ok = (major == 10 && minor == 0);
    d.sms = n;
    if (d.ok) {
      bool attrs = cudaFuncSetAttribute(gemm_bf16_tcgen05<EPI_QKV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        GEMM_SMEM_BYTES) == cudaSuccess &&
                   cudaFuncSetAttribute(gemm_bf16_tcgen05<EPI_OUTPROJ>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, GEMM_SMEM_BYTES) == cudaSuccess &&
                   cudaFuncSetAttribute(gemm_bf16_tcgen05<EPI_FFN_UP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        GEMM_SMEM_BYTES) == cudaSuccess &&
                   cudaFuncSetAttribute(gemm_bf16_tcgen05<EPI_FFN_DOWN>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, GEMM_SMEM_BYTES) == cudaSuccess &&
                   cudaFuncSetAttribute(gemm_bf16_tcgen05<EPI_BWD_DA, 0, 0>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, GEMM_SMEM_BYTES) == cudaSuccess &&
                   cudaFuncSetAttribute(gemm_bf16_tcgen05<EPI_BWD_DHID, 0, 0>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, GEMM_SMEM_BYTES) == cudaSuccess &&
                   cudaFuncSetAttribute(gemm_bf16_tcgen05<EPI_GRAD, 1, 1>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, GEMM_SMEM_BYTES) == cudaSuccess &&
                   cudaFuncSetAttribute(gemm_pair_tcgen05<EPI_QKV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        GP_SMEM_BYTES) == cudaSuccess &&
                   cudaFuncSetAttribute(gemm_pair_tcgen05<EPI_OUTPROJ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        GP_SMEM_BYTES) == cudaSuccess &&
                   cudaFuncSetAttribute(gemm_pair_tcgen05<EPI_FFN_UP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        GP_SMEM_BYTES) == cudaSuccess &&
                   cudaFuncSetAttribute(gemm_pair_tcgen05<EPI_FFN_DOWN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        GP_SMEM_BYTES) == cudaSuccess &&
                   cudaFuncSetAttribute(gemm_pair_tcgen05<EPI_BWD_DA, 0, 0>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, GP_SMEM_BYTES) == cudaSuccess &&
                   cudaFuncSetAttribute(gemm_pair_tcgen05<EPI_BWD_DHID, 0, 0>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, GP_SMEM_BYTES) == cudaSuccess &&
                   cudaFuncSetAttribute(gemm_pair_tcgen05<EPI_GRAD, 1, 1>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, GP_SMEM_BYTES) == cudaSuccess &&
                   cudaFuncSetAttribute(ffn_chain_tcgen05, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        GEMM_SMEM_BYTES) == cudaSuccess &&
                   cudaFuncSetAttribute(attention_pair_tcgen05, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        AttnPairCfg::SMEM_BYTES) == cudaSuccess &&
                   cudaFuncSetAttribute(attention_fwd_tcgen05<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        AttnCfg<64>::SMEM_BYTES) == cudaSuccess &&
                   cudaFuncSetAttribute(attention_fwd_tcgen05<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        AttnCfg<128>::SMEM_BYTES) == cudaSuccess &&
                   cudaFuncSetAttribute(attention_fwd_tcgen05<64, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        AttnCfg<64>::SMEM_BYTES) == cudaSuccess &&
                   cudaFuncSetAttribute(attention_fwd_tcgen05<128, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        AttnCfg<128>::SMEM_BYTES) == cudaSuccess &&
                   cudaFuncSetAttribute(attention_bwd_tcgen05<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        AttnBwdCfg<64>::SMEM_BYTES) == cudaSuccess &&
                   cudaFuncSetAttribute(attention_bwd_tcgen05<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        AttnBwdCfg<128>::SMEM_BYTES) == cudaSuccess &&
                   cudaFuncSetAttribute(layer_mega_tcgen05<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        mega_smem_bytes<64>()) == cudaSuccess &&
                   cudaFuncSetAttribute(layer_mega_tcgen05<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        mega_smem_bytes<128>()) == cudaSuccess;
      if (!attrs) return BPT_ERR_CUDA;
      // the attention kernel splits its registers between warpgroups assuming
      // it was built with exactly ATT_REGS_LAUNCH per thread; any other build
      // is never launched (its register requests could not be met)
      cudaFuncAttributes fa64{}, fa128{}, fl64{}, fl128{}, fap{};
      if (cudaFuncGetAttributes(&fa64, attention_fwd_tcgen05<64>) != cudaSuccess ||
          cudaFuncGetAttributes(&fa128, attention_fwd_tcgen05<128>) != cudaSuccess ||
          cudaFuncGetAttributes(&fl64, attention_fwd_tcgen05<64, true>) != cudaSuccess ||
          cudaFuncGetAttributes(&fl128, attention_fwd_tcgen05<128, true>) != cudaSuccess ||
          cudaFuncGetAttributes(&fap, attention_pair_tcgen05) != cudaSuccess)
        return BPT_ERR_CUDA;
      if (fa64.numRegs != ATT_REGS_LAUNCH || fa128.numRegs != ATT_REGS_LAUNCH || fl64.numRegs != ATT_REGS_LAUNCH ||
          fl128.numRegs != ATT_REGS_LAUNCH || fap.numRegs != ATT_REGS_LAUNCH)
        d.ok = false;
      cudaFuncAttributes fm64{}, fm128{};
      if (cudaFuncGetAttributes(&fm64, layer_mega_tcgen05<64>) != cudaSuccess ||
          cudaFuncGetAttributes(&fm128, layer_mega_tcgen05<128>) != cudaSuccess)
        return BPT_ERR_CUDA;
      d.mega_ok = fm64.numRegs == ATT_REGS_LAUNCH && fm128.numRegs == ATT_REGS_LAUNCH;
    }
    d.checked = true;
  }
  if (!d.ok) return BPT_ERR_UNSUPPORTED;
  *sms = d.sms;
  return BPT_OK;
}

// Whether the one-launch layer kernel may run on the current device (after check_device).
bool mega_available() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  return g_dev[dev].checked && g_dev[dev].mega_ok;
}

// ------------------------------------------------------------- stream status
// Each (device, stream) that launches this library's kernels owns one word of
// g_status_slots on that device, assigned at its first call and kept for the
// life of the process; word 0 is shared by every stream past the first
// kStatusSlots - 1 of a device. The table of stream handles is a fixed array
// (open addressing), so assigning a word allocates nothing. The device address
// of the array is looked up on every call (a symbol lookup, no allocation), so
// it stays right after a cudaDeviceReset recreates the module.
std::mutex g_status_mu;
uintptr_t g_status_key[64][kStatusSlots];
bool g_status_used[64][kStatusSlots];

int status_base(int** base) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_status_slots) != cudaSuccess || !p) {
    cudaGetLastError();
    return BPT_ERR_CUDA;
  }
  *base = reinterpret_cast<int*>(p);
  return BPT_OK;
}

// Index of the stream's word on the current device; -1 if it has none and
// `create` is false.
int status_index(int dev, cudaStream_t st, bool create) {
  const uintptr_t key = reinterpret_cast<uintptr_t>(st);
  constexpr int n = kStatusSlots - 1;  // words 1 .. kStatusSlots - 1
  const int start = (int)((key >> 4) * 0x9E3779B97F4A7C15ull >> 40) % n;
  std::lock_guard<std::mutex> lk(g_status_mu);
  for (int i = 0; i < n; ++i) {
    const int idx = 1 + (start + i) % n;
    if (!g_status_used[dev][idx]) {
      if (!create) return -1;
      g_status_used[dev][idx] = true;
      g_status_key[dev][idx] = key;
      return idx;
    }
    if (g_status_key[dev][idx] == key) return idx;
  }
  return 0;  // table full: the shared word
}

// Device address of the status word of `st` on the current device.
int stream_status_word(cudaStream_t st, int** word) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return BPT_ERR_CUDA;
  int* base = nullptr;
  const int r = status_base(&base);
  if (r != BPT_OK) return r;
  *word = base + status_index(dev, st, true);
  return BPT_OK;
}

// A single thread waits until *flag == value, at most timeout_ns; if it gives
// up it records BPT_ERR_TIMEOUT in the stream's status word.
__global__ void wait_flag_kernel(const int* flag, int value, unsigned long long timeout_ns, int* status) {
  if (threadIdx.x != 0) return;
  const unsigned long long t0 = global_timer_ns();
  while (*reinterpret_cast<const volatile int*>(flag) != value) {
    if (global_timer_ns() - t0 > timeout_ns) {
      atomicExch(status, (int)BPT_ERR_TIMEOUT);
      return;
    }
    __nanosleep(1000);
  }
}

// ------------------------------------------------------------- workspace pool
// The allocating entry points take their workspace from a library-owned,
// stream-ordered memory pool per device that keeps freed memory for the next
// call (release threshold: never), so a call does not map and unmap hundreds
// of MB each time. The pool holds at most the largest workspace requested by
// concurrent calls.
std::mutex g_pool_mu;
cudaMemPool_t g_pool[64] = {};

int workspace_pool(cudaMemPool_t* pool) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return BPT_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_pool_mu);
  if (!g_pool[dev]) {
    cudaMemPoolProps props{};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t p = nullptr;
    if (cudaMemPoolCreate(&p, &props) != cudaSuccess) {
      cudaGetLastError();
      return BPT_ERR_CUDA;
    }
    uint64_t keep = UINT64_MAX;
    cudaMemPoolSetAttribute(p, cudaMemPoolAttrReleaseThreshold, &keep);
    g_pool[dev] = p;
  }
  *pool = g_pool[dev];
  return BPT_OK;
}

// ------------------------------------------------------------- argument checks
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Range {
  uintptr_t lo, hi;
};
bool overlap(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi && a.lo < a.hi && b.lo < b.hi; }
Range rng(const void* p, size_t bytes) {
  return Range{reinterpret_cast<uintptr_t>(p), reinterpret_cast<uintptr_t>(p) + bytes};
}

int check_shape(int b, int s, int h, int heads) {
  if (b < 0 || s < 0 || h <= 0 || heads <= 0) return BPT_ERR_SHAPE;
  if (h % heads) return BPT_ERR_SHAPE;
  const int dh = h / heads;
  if (dh != 64 && dh != 128) return BPT_ERR_SHAPE;
  if ((long long)b * s > 0x7fffffffLL) return BPT_ERR_SHAPE;
  if ((long long)h * 4 > 0x7fffffffLL / 4) return BPT_ERR_SHAPE;
  return BPT_OK;
}

int check_blocks(int s, int q_block, int kv_block) {
  if (s == 0) return BPT_OK;
  if (q_block <= 0 || kv_block <= 0 || q_block > s || kv_block > s) return BPT_ERR_BLOCK;
  if (s % q_block || s % kv_block) return BPT_ERR_BLOCK;
  return BPT_OK;
}

// ------------------------------------------------------------- wave plan
struct Wave {
  long long row0;  // flat row of the wave's first row
  int beta0, n_seq, t_start, t_len;
  long long rows() const { return (long long)n_seq * t_len; }
};

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Bytes of the K and V copies of the whole sequence (bf16, 1 KB aligned).
size_t kv_bytes(int b, int s, int h) { return 2 * align_up((size_t)b * s * h * 2, 1024); }

// Bytes of one wave's scratch: fp32 hid, its bf16 copy and the bf16 FFN
// intermediate U (ffn wide), each 1 KB aligned.
size_t wave_scratch_bytes(long long wr, int h, int ffn) {
  return align_up((size_t)wr * h * 4, 1024) + align_up((size_t)wr * h * 2, 1024) +
         align_up((size_t)wr * ffn * 2, 1024);
}

// Modelled duration of the three FFN-side GEMMs of one wave of `rows` rows,
// in units of one 128 x 256 x 64 tile step: a persistent launch takes
// ceil(tiles / SMs) rounds of K/64 steps each, plus a fixed fill/drain cost.
constexpr int kModelSms = 148;
constexpr long long kLaunchSteps = 24;
long long gemm_steps(long long rows, long long n, long long k) {
  const long long tiles = ((rows + GEMM_BM - 1) / GEMM_BM) * ((n + GEMM_BN - 1) / GEMM_BN);
  return (tiles + kModelSms - 1) / kModelSms * (k / GEMM_BK) + kLaunchSteps;
}
long long wave_steps(long long rows, int h, int ffn) {
  if (rows <= 0) return 0;
  return gemm_steps(rows, h, h) + gemm_steps(rows, ffn, h) + gemm_steps(rows, h, ffn);
}

// Default wave: the whole number of query blocks (or, when a sequence fits,
// of whole sequences) whose modelled GEMM time over the layer is within 1% of
// the best, taking the smallest such wave. The scratch of a wave aliases the
// K/V copies (dead once attention has run), and is held to 1.5x their size,
// or to the scratch of a ~4096-row wave where that is larger (small problems).
int default_wave_rows(int b, int s, int h, int ffn, int q_block) {
  const size_t per_row = 6 * (size_t)h + 2 * (size_t)ffn;  // 4h + 2h + 2 ffn bytes per row
  const long long floor_rows = s >= 4096 ? std::max<long long>(q_block, 4096 / q_block * q_block)
                                         : (long long)std::min(b, 4096 / s) * s;
  const size_t budget = std::max(kv_bytes(b, s, h) / 2 * 3, wave_scratch_bytes(floor_rows, h, ffn));
  const long long max_rows = std::max<long long>(q_block, (long long)(budget / per_row));
  // candidates (modelled steps, wave rows): whole numbers of query blocks
  // shorter than a sequence, then whole numbers of sequences; two passes over
  // them (the best time, then the smallest wave within 1% of it) keep this
  // free of allocations
  auto visit = [&](auto&& f) {
    bool any = false;
    for (long long wr = q_block; wr < s && wr <= max_rows; wr += q_block, any = true)
      f(b * ((s / wr) * wave_steps(wr, h, ffn) + wave_steps(s % wr, h, ffn)), wr);
    for (long long g = 1; g <= b && (g * s <= max_rows || !any); ++g, any = true)
      f((b / g) * wave_steps(g * s, h, ffn) + wave_steps((b % g) * s, h, ffn), g * s);
  };
  long long best = -1;
  visit([&](long long steps, long long) { best = best < 0 ? steps : std::min(best, steps); });
  long long pick = 0;
  visit([&](long long steps, long long wr) {
    if (steps * 100 <= best * 101 && (pick == 0 || wr < pick)) pick = wr;
  });
  return (int)std::min<long long>(pick, 0x7fffffffLL);
}

int wave_rows_for(int b, int s, int h, int ffn, int q_block, int wave_rows) {
  if (wave_rows <= 0) return default_wave_rows(b, s, h, ffn, q_block);  // BPT_WAVE_DEFAULT(_WAVES)
  long long wr = std::max<long long>(q_block, ((long long)wave_rows / q_block) * q_block);
  if (wr >= s) {
    const long long g = std::max<long long>(1, std::min<long long>(b, wr / s));
    return (int)std::min<long long>(g * s, 0x7fffffffLL);
  }
  return (int)wr;
}

// Calls f(wave) for each wave of the FFN side in order and returns the first
// status other than BPT_OK (or BPT_OK).
template <class F>
int for_each_wave(int b, int s, int h, int ffn, int q_block, int wave_rows, F&& f) {
  const int wr = wave_rows_for(b, s, h, ffn, q_block, wave_rows);
  if (wr >= s) {
    const int g = wr / s;
    for (int beta = 0; beta < b; beta += g) {
      const int r = f(Wave{(long long)beta * s, beta, std::min(g, b - beta), 0, s});
      if (r != BPT_OK) return r;
    }
  } else {
    for (int beta = 0; beta < b; ++beta)
      for (int ts = 0; ts < s; ts += wr) {
        const int r = f(Wave{(long long)beta * s + ts, beta, 1, ts, std::min(wr, s - ts)});
        if (r != BPT_OK) return r;
      }
  }
  return BPT_OK;
}

// Rows per chunk of the FFN block's backward: the caller's, rounded down to a
// multiple of 128 (at least 128), or 16384 by default (measured against 4096, 8192
// and 32768 rows: the fp32 weight-gradient epilogues read and write dW1 and dW2 once
// per chunk, so short chunks cost traffic, and 16384 was 10% faster than 4096 at
// rows 32768, h 4096, ffn 16384); never more than rows.
long long ffn_bwd_chunk(int rows, int chunk_rows) {
  long long r = chunk_rows > 0 ? std::max(128, chunk_rows / 128 * 128) : 16384;
  return std::min<long long>(r, rows);
}

// ------------------------------------------------------------- FFN chain plan
// Groups of the one-launch FFN side (ffn_chain.cuh): the largest group of
// 16, 8, 4, 2 or 1 M-tiles whose slots (fp32 hid, its bf16 copy, bf16 U) take
// at most 1.5x the K/V bytes (or 32 MiB, for small problems); one M-tile
// when none does. The slots alias the K/V region, dead once attention has
// run, so the workspace is the larger of the two. Slots are 1 KB aligned.
struct ChainPlan {
  int m_tiles, gm, groups, hs, us;
  size_t hid, hb, u, bytes;
};

ChainPlan chain_plan(int b, int s, int h, int ffn) {
  const long long M = (long long)b * s;
  const size_t kv = kv_bytes(b, s, h);
  const size_t budget = std::max(kv / 2 * 3, (size_t)32 << 20);
  ChainPlan p{};
  p.m_tiles = (int)((M + GEMM_BM - 1) / GEMM_BM);
  for (int gm = CHAIN_GROUP_MT; gm >= 1; gm /= 2) {
    p.gm = gm;
    p.groups = (p.m_tiles + gm - 1) / gm;
    p.hs = std::min(CHAIN_HID_SLOTS, p.groups);
    p.us = std::min(CHAIN_U_SLOTS, p.groups);
    const size_t rows = (size_t)gm * GEMM_BM;
    p.hid = 0;
    p.hb = align_up((size_t)p.hs * rows * h * 4, 1024);
    p.u = p.hb + align_up((size_t)p.hs * rows * h * 2, 1024);
    p.bytes = p.u + align_up((size_t)p.us * rows * ffn * 2, 1024);
    if (p.bytes <= budget) break;
  }
  return p;
}

// ------------------------------------------------------------- workspace layout
// Region 0 holds K and V during the projection and attention, then the
// scratch of the FFN side: the chain's group slots (default bf16 path) or one
// wave's hid, hb and U (explicit wave size, fp32 inputs); the chain's
// completion counters, then the f32 entry's bf16 copies of x and the weights
// follow it.
struct Layout {
  size_t k, v, hid, hb, u, xb, wqkv, wo, w1, w2, cnt, total;
  int wave_rows;
  bool chain;
  bool mega;  // attention and the chain in one launch: the chain's slots follow K/V instead of aliasing them
  ChainPlan cp;
};

// wave_rows selects the FFN side's schedule: BPT_WAVE_CHAINED runs it in one
// launch (bf16 inputs), BPT_WAVE_DEFAULT_WAVES and any positive size in one
// launch per GEMM and wave, and BPT_WAVE_DEFAULT (0) takes kChainByDefault.
// fp32 inputs (split products) always run per wave.
// BPT_WAVE_MEGA (bf16, s a multiple of 128) runs attention and the chain in
// one launch; otherwise it runs as BPT_WAVE_CHAINED (bf16) or per wave (fp32).
constexpr bool kChainByDefault = false;
bool use_mega(int dtype, int s, int wave_rows) {
  return dtype == BPT_DTYPE_BF16 && wave_rows == BPT_WAVE_MEGA && s % ATT_BM == 0;
}
bool use_chain(int dtype, int wave_rows) {
  if (dtype != BPT_DTYPE_BF16) return false;
  return wave_rows == BPT_WAVE_CHAINED || wave_rows == BPT_WAVE_MEGA ||
         (wave_rows == BPT_WAVE_DEFAULT && kChainByDefault);
}

// With ffn_after_kv (per-GEMM waves only), the wave scratch follows the K/V
// copies instead of aliasing them, so that a wave's FFN side can run while
// later rows still need K and V.
Layout layout_for(int dtype, int b, int s, int h, int ffn, int q_block, int wave_rows, bool ffn_after_kv = false) {
  Layout L{};
  const size_t tok = (size_t)b * s;
  L.k = 0;
  L.v = align_up(tok * h * 2, 1024);
  size_t off;
  if (use_chain(dtype, wave_rows)) {
    L.chain = true;
    L.mega = use_mega(dtype, s, wave_rows);
    L.cp = chain_plan(b, s, h, ffn);
    L.wave_rows = L.cp.gm * GEMM_BM;
    // the slots alias K/V (dead once attention has run), or follow them when
    // attention runs in the same launch
    const size_t base = L.mega ? align_up(kv_bytes(b, s, h), 1024) : 0;
    L.hid = base + L.cp.hid;
    L.hb = base + L.cp.hb;
    L.u = base + L.cp.u;
    off = L.mega ? base + L.cp.bytes : std::max(kv_bytes(b, s, h), L.cp.bytes);
    L.cnt = off;
    // the chain's three counters per group; with mega, attention's per group and the ticket
    off = align_up(off + (3 * (size_t)L.cp.groups + (L.mega ? (size_t)L.cp.groups + 1 : 0)) * sizeof(unsigned), 1024);
  } else {
    const int wr = wave_rows_for(b, s, h, ffn, q_block, wave_rows);
    const size_t base = ffn_after_kv ? align_up(kv_bytes(b, s, h), 1024) : 0;
    L.wave_rows = wr;
    L.hid = base;
    L.hb = base + align_up((size_t)wr * h * 4, 1024);
    L.u = L.hb + align_up((size_t)wr * h * 2, 1024);
    off = ffn_after_kv ? base + wave_scratch_bytes(wr, h, ffn) : std::max(kv_bytes(b, s, h), wave_scratch_bytes(wr, h, ffn));
  }
  auto take = [&](size_t bytes) {
    size_t at = off;
    off = align_up(off + bytes, 1024);
    return at;
  };
  if (dtype == BPT_DTYPE_F32) {
    // split bf16 parts: x as rows [x_hi | x_lo]; Wqkv as [hi; lo; hi] and
    // Wo, W1, W2 as [hi; lo], stacked along K
    L.xb = take(tok * 2 * h * 2);
    L.wqkv = take((size_t)3 * h * 3 * h * 2);
    L.wo = take((size_t)2 * h * h * 2);
    L.w1 = take((size_t)2 * h * ffn * 2);
    L.w2 = take((size_t)2 * ffn * h * 2);
  }
  L.total = off;
  return L;
}

// ------------------------------------------------------------- launches
struct LayerPtrs {
  const void *x, *Wqkv, *bqkv, *Wo, *bo, *W1, *b1, *W2, *b2;
};

// A [M, a_cols] (row stride lda) times B [K, N]; with a_split != 0 the K
// blocks of B pair with A's blocks as a_block() maps them (split products).
template <int MODE>
int launch_gemm_split(const void* A, long long M, long long a_cols, long long lda, const void* B, long long K,
                      long long N, int a_split, int a_kb, GemmArgs args, int sms, cudaStream_t st, int* status,
                      const char* name) {
  if (M <= 0) return BPT_OK;
  args.status = status;
  CUtensorMap ta, tb;
  if (!map_rows(&ta, A, M, a_cols, lda, GEMM_BM)) return BPT_ERR_CUDA;
  if (!map_rows(&tb, B, K, N, N, 64)) return BPT_ERR_CUDA;
  args.a_split = a_split;
  args.a_kb = a_kb;
  args.M = (int)M;
  args.N = (int)N;
  args.K = (int)K;
  args.m_tiles = (int)((M + GEMM_BM - 1) / GEMM_BM);
  args.n_tiles = (int)((N + GEMM_BN - 1) / GEMM_BN);
  if (BPT_PAIR_GEMM && a_split == 0) {
    // 256 x 256 tiles on SM pairs: each CTA maps its own 128 rows of A and its
    // 128-column half of B
    CUtensorMap tb2;
    if (!map_rows(&ta, A, M, a_cols, lda, 128) || !map_rows(&tb2, B, K, N, N, 64)) return BPT_ERR_CUDA;
    args.m_tiles = (int)((M + GP_BM - 1) / GP_BM);
    args.n_tiles = (int)((N + GP_BN - 1) / GP_BN);
    const int pairs = std::min(args.m_tiles * args.n_tiles, sms / 2);
    {
      LaunchScope ls(name, st);
      gemm_pair_tcgen05<MODE><<<2 * pairs, GEMM_THREADS, GP_SMEM_BYTES, st>>>(ta, tb2, args);
    }
    return cudaGetLastError() == cudaSuccess ? BPT_OK : BPT_ERR_CUDA;
  }
  const int tiles = args.m_tiles * args.n_tiles;
  const int grid = std::min(tiles, sms);
  {
    LaunchScope ls(name, st);
    gemm_bf16_tcgen05<MODE><<<grid, GEMM_THREADS, GEMM_SMEM_BYTES, st>>>(ta, tb, args);
  }
  return cudaGetLastError() == cudaSuccess ? BPT_OK : BPT_ERR_CUDA;
}

template <int MODE>
int launch_gemm(const void* A, long long M, long long K, long long lda, const void* B, long long N,
                GemmArgs args, int sms, cudaStream_t st, int* status, const char* name) {
  return launch_gemm_split<MODE>(A, M, K, lda, B, K, N, 0, 0, args, sms, st, status, name);
}

// D[M, N] = A B for the backward's products: A is [M, K] (lda elements apart)
// or, with A_MN, stored [K, M]; B is [K, N] (ldb apart) with B_MN or stored
// [N, K] without. K need not be a multiple of 64: the copies zero-fill past
// the last row of an operand.
template <int MODE, int A_MN, int B_MN>
int launch_gemm_t(const void* A, long long lda, const void* B, long long ldb, long long M, long long N, long long K,
                  GemmArgs args, int sms, cudaStream_t st, int* status, const char* name) {
  if (M <= 0 || N <= 0) return BPT_OK;
  args.status = status;
  args.M = (int)M;
  args.N = (int)N;
  args.K = (int)((K + GEMM_BK - 1) / GEMM_BK * GEMM_BK);
  CUtensorMap ta, tb;
  if (BPT_PAIR_GEMM) {
    // 256 x 256 tiles on SM pairs: each CTA maps its own 128 rows of A and its
    // 128-column half of B
    const bool ok_a = A_MN ? map_rows(&ta, A, K, M, lda, 64) : map_rows(&ta, A, M, K, lda, 128);
    const bool ok_b = B_MN ? map_rows(&tb, B, K, N, ldb, 64) : map_rows(&tb, B, N, K, ldb, 128);
    if (!ok_a || !ok_b) return BPT_ERR_CUDA;
    args.m_tiles = (int)((M + GP_BM - 1) / GP_BM);
    args.n_tiles = (int)((N + GP_BN - 1) / GP_BN);
    const int pairs = std::min(args.m_tiles * args.n_tiles, sms / 2);
    {
      LaunchScope ls(name, st);
      gemm_pair_tcgen05<MODE, A_MN, B_MN><<<2 * pairs, GEMM_THREADS, GP_SMEM_BYTES, st>>>(ta, tb, args);
    }
    return cudaGetLastError() == cudaSuccess ? BPT_OK : BPT_ERR_CUDA;
  }
  const bool ok_a = A_MN ? map_rows(&ta, A, K, M, lda, 64) : map_rows(&ta, A, M, K, lda, GEMM_BM);
  const bool ok_b = B_MN ? map_rows(&tb, B, K, N, ldb, 64) : map_rows(&tb, B, N, K, ldb, GEMM_BN);
  if (!ok_a || !ok_b) return BPT_ERR_CUDA;
  args.m_tiles = (int)((M + GEMM_BM - 1) / GEMM_BM);
  args.n_tiles = (int)((N + GEMM_BN - 1) / GEMM_BN);
  const int grid = std::min(args.m_tiles * args.n_tiles, sms);
  {
    LaunchScope ls(name, st);
    gemm_bf16_tcgen05<MODE, A_MN, B_MN><<<grid, GEMM_THREADS, GEMM_SMEM_BYTES, st>>>(ta, tb, args);
  }
  return cudaGetLastError() == cudaSuccess ? BPT_OK : BPT_ERR_CUDA;
}

// out[c] (+)= sum over rows r of src[r * ld + c], fp32: one block of 32 warps
// per 32 columns; lane l of warp w sums column c0 + l over the rows r = w, w + 32,
// ... (each row read as one coalesced line by the warp), then the 32 partial sums
// of a column are added in warp order. Same order every run (deterministic).
template <typename T>
__global__ void __launch_bounds__(1024) colsum_kernel(const T* __restrict__ src, long long rows, int cols, long long ld,
                                                      float* out, int accumulate) {
  __shared__ float part[32][33];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int c = blockIdx.x * 32 + lane;
  float acc = 0.0f;
  if (c < cols) {
    long long r = w;
#pragma unroll 4
    for (; r < rows; r += 32) {
      if constexpr (sizeof(T) == 2)
        acc += __bfloat162float(src[r * ld + c]);
      else
        acc += src[r * ld + c];
    }
  }
  part[w][lane] = acc;
  __syncthreads();
  if (w == 0 && c < cols) {
    float t = 0.0f;
    for (int i = 0; i < 32; ++i) t += part[i][lane];
    out[c] = accumulate ? out[c] + t : t;
  }
}

// The same column sums with 16-byte loads: a cluster of CS_SPLIT CTAs shares one
// strip of 32 x (16 / sizeof(T)) columns, each CTA a contiguous eighth of the
// rows; in a CTA, warp w takes rows w, w + CS_WARPS, ... and each lane one
// 16-byte vector of a row (a warp reads 512 contiguous bytes per row). The sums
// are taken in a fixed order (rows in order within a thread, then the warps in
// order, then the CTAs of the cluster in rank order, read by rank 0 from the
// others' shared memory), so results are the same on every run.
constexpr int CS_SPLIT = 8;
constexpr int CS_WARPS = 32;
template <typename T>
__global__ void __cluster_dims__(1, CS_SPLIT, 1) __launch_bounds__(CS_WARPS * 32)
    colsum_vec_kernel(const T* __restrict__ src, long long rows, int cols, long long ld, float* out, int accumulate) {
  constexpr int VEC = 16 / (int)sizeof(T);
  constexpr int CW = 32 * VEC;  // columns of the strip
  __shared__ float part[CS_WARPS][CW];  // [warp][i * 32 + lane]: column lane * VEC + i
  __shared__ float csum[CW];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int rank = (int)blockIdx.y;  // the cluster spans grid.y (= CS_SPLIT)
  const long long c0 = (long long)blockIdx.x * CW + lane * VEC;
  const long long per = (rows + CS_SPLIT - 1) / CS_SPLIT;
  const long long rb = rank * per, re = rows < rb + per ? rows : rb + per;
  float acc[VEC];
#pragma unroll
  for (int i = 0; i < VEC; ++i) acc[i] = 0.0f;
  if (c0 < cols) {
#pragma unroll 4
    for (long long r = rb + w; r < re; r += CS_WARPS) {
      const uint4 q = __ldg(reinterpret_cast<const uint4*>(src + r * ld + c0));
      const uint32_t u[4] = {q.x, q.y, q.z, q.w};
      if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[2 * i] += __uint_as_float(u[i] << 16);
          acc[2 * i + 1] += __uint_as_float(u[i] & 0xffff0000u);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i] += __uint_as_float(u[i]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < VEC; ++i) part[w][i * 32 + lane] = acc[i];
  __syncthreads();
  for (int t = threadIdx.x; t < CW; t += blockDim.x) {
    float v = 0.0f;
    for (int k = 0; k < CS_WARPS; ++k) v += part[k][t];
    csum[t] = v;
  }
  cluster_sync_all();  // every CTA's strip sum is in its shared memory
  if (rank == 0) {
    for (int t = threadIdx.x; t < CW; t += blockDim.x) {
      const long long col = (long long)blockIdx.x * CW + (t & 31) * VEC + (t >> 5);
      float v = 0.0f;
      for (int k = 0; k < CS_SPLIT; ++k) {
        float x;
        asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(x) : "r"(mapa_shared(smem_addr(csum + t), k)) : "memory");
        v += x;
      }
      if (col < cols) out[col] = accumulate ? out[col] + v : v;
    }
  }
  cluster_sync_all();  // no CTA leaves while rank 0 may still read its shared memory
}

// Column sums (deterministic): the vector kernel when rows are 16-byte aligned
// vectors, else one thread per column.
template <typename T>
int launch_colsum(const T* src, long long rows, int cols, long long ld, float* out, int accumulate, cudaStream_t st) {
  if (cols <= 0) return BPT_OK;
  LaunchScope ls("colsum", st);
  constexpr int VEC = 16 / (int)sizeof(T);
  if (cols % VEC == 0 && ld % VEC == 0 && aligned16(src)) {
    const dim3 grid((unsigned)((cols + 32 * VEC - 1) / (32 * VEC)), CS_SPLIT);
    colsum_vec_kernel<T><<<grid, CS_WARPS * 32, 0, st>>>(src, rows, cols, ld, out, accumulate);
  } else {
    colsum_kernel<T><<<(cols + 31) / 32, 1024, 0, st>>>(src, rows, cols, ld, out, accumulate);
  }
  return cudaGetLastError() == cudaSuccess ? BPT_OK : BPT_ERR_CUDA;
}

// Attention of the query rows [t_start, t_start + t_len) of sequences
// beta0 .. beta0 + n_seq - 1; q rows have `ldq` elements between them.
int launch_attention(const void* q, long long ldq, const void* k, const void* v, int b, int s, int h, int heads,
                     int causal, int beta0, int n_seq, int t_start, int t_len, __nv_bfloat16* o, long long ldo,
                     cudaStream_t st, int* status, float* lse2 = nullptr) {
  const int dh = h / heads;
  CUtensorMap tq, tk, tv;
  if (BPT_PAIR_ATTENTION && dh == 128 && lse2 == nullptr) {
    // K halves are [64 keys][64 cols] boxes, Q and the V halves [128][64]
    if (!map_seq(&tq, q, b, s, h, ldq, 128) || !map_seq(&tk, k, b, s, h, h, 64) || !map_seq(&tv, v, b, s, h, h, 128))
      return BPT_ERR_CUDA;
    AttnPairArgs a{};
    a.s = s;
    a.heads = heads;
    a.causal = causal ? 1 : 0;
    a.t_start = t_start;
    a.t_len = t_len;
    a.n_quads = (t_len + 4 * ATT_BM - 1) / (4 * ATT_BM);
    a.ldo = ldo;
    a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)dh));
    a.status = status;
    for (int z0 = 0; z0 < n_seq; z0 += 65535) {
      const int nz = std::min(65535, n_seq - z0);
      a.beta0 = beta0 + z0;
      a.o = o + (long long)z0 * t_len * ldo;
      dim3 grid(2u * (unsigned)a.n_quads * (unsigned)heads, 1, nz);
      LaunchScope ls("attention", st);
      attention_pair_tcgen05<<<grid, ATT_THREADS, AttnPairCfg::SMEM_BYTES, st>>>(tq, tk, tv, a);
    }
    return cudaGetLastError() == cudaSuccess ? BPT_OK : BPT_ERR_CUDA;
  }
  if (!map_seq(&tq, q, b, s, h, ldq) || !map_seq(&tk, k, b, s, h, h) || !map_seq(&tv, v, b, s, h, h))
    return BPT_ERR_CUDA;
  AttnArgs a{};
  a.s = s;
  a.heads = heads;
  a.causal = causal ? 1 : 0;
  a.t_start = t_start;
  a.t_len = t_len;
  a.n_pairs = (t_len + 2 * ATT_BM - 1) / (2 * ATT_BM);
  a.ldo = ldo;
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)dh));
  a.status = status;
  for (int z0 = 0; z0 < n_seq; z0 += 65535) {
    const int nz = std::min(65535, n_seq - z0);
    a.beta0 = beta0 + z0;
    a.o = o + (long long)z0 * t_len * ldo;
    a.lse2 = lse2 ? lse2 + (long long)z0 * heads * t_len : nullptr;
    dim3 grid((unsigned)a.n_pairs * (unsigned)heads, 1, nz);
    LaunchScope ls("attention", st);
    if (lse2 != nullptr) {
      if (dh == 64)
        attention_fwd_tcgen05<64, true><<<grid, ATT_THREADS, AttnCfg<64>::SMEM_BYTES, st>>>(tq, tk, tv, a);
      else
        attention_fwd_tcgen05<128, true><<<grid, ATT_THREADS, AttnCfg<128>::SMEM_BYTES, st>>>(tq, tk, tv, a);
    } else if (dh == 64) {
      attention_fwd_tcgen05<64><<<grid, ATT_THREADS, AttnCfg<64>::SMEM_BYTES, st>>>(tq, tk, tv, a);
    } else {
      attention_fwd_tcgen05<128><<<grid, ATT_THREADS, AttnCfg<128>::SMEM_BYTES, st>>>(tq, tk, tv, a);
    }
  }
  return cudaGetLastError() == cudaSuccess ? BPT_OK : BPT_ERR_CUDA;
}

// D = rowsum(dO O) of every (row, head): dsum[(beta * heads + head) * s + t],
// fp32 sums of the bf16 products, one thread per (row, head).
__global__ void attn_dsum_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dO,
                                 long long ld, long long rows, int s, int heads, int dh, float* __restrict__ dsum) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= rows * heads) return;
  const int head = (int)(i % heads);
  const long long row = i / heads;
  const __nv_bfloat16* po = o + row * ld + (long long)head * dh;
  const __nv_bfloat16* pd = dO + row * ld + (long long)head * dh;
  float acc = 0.0f;
  for (int c = 0; c < dh; c += 8) {
    const uint4 a = *reinterpret_cast<const uint4*>(po + c);
    const uint4 d = *reinterpret_cast<const uint4*>(pd + c);
    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&d);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 fa = __bfloat1622float2(a2[k]), fd = __bfloat1622float2(d2[k]);
      acc = fmaf(fa.x, fd.x, acc);
      acc = fmaf(fa.y, fd.y, acc);
    }
  }
  const long long beta = row / s, t = row - beta * s;
  dsum[(beta * heads + head) * s + t] = acc;
}

// dst[r * ld_dst + c] = bf16(src[r * cols + c]) for c < cols (cols a multiple of 8).
__global__ void rows_f32_to_bf16_kernel(const float* __restrict__ src, long long rows, int cols,
                                        __nv_bfloat16* __restrict__ dst, long long ld_dst) {
  const long long per_row = cols / 8;
  const long long n = rows * per_row;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const long long r = i / per_row, c = (i - r * per_row) * 8;
    const float4 a = *reinterpret_cast<const float4*>(src + r * cols + c);
    const float4 b = *reinterpret_cast<const float4*>(src + r * cols + c + 4);
    st_global_v4(dst + r * ld_dst + c, pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y),
                 pack_bf16x2(b.z, b.w));
  }
}

// Gradients of the attention of b sequences: dK, dV (bf16, ld_kv apart) and
// the fp32 dQ accumulator (rows h apart, zero on entry) from Q, K, V (ld_in
// apart), dO (ld_do apart), the forward's lse2 and D = rowsum(dO O).
int launch_attention_bwd(const void* q, const void* k, const void* v, long long ld_in, const void* dO,
                         long long ld_do, const float* lse2, const float* dsum, float* dq, __nv_bfloat16* dk,
                         __nv_bfloat16* dv, long long ld_kv, int b, int s, int h, int heads, int causal,
                         cudaStream_t st, int* status) {
  if ((long long)b * s == 0) return BPT_OK;
  const int dh = h / heads;
  CUtensorMap tq, tk, tv, td, tdq;
  if (!map_seq(&tq, q, b, s, h, ld_in) || !map_seq(&tk, k, b, s, h, ld_in) || !map_seq(&tv, v, b, s, h, ld_in) ||
      !map_seq(&td, dO, b, s, h, ld_do) || !map_seq_f32(&tdq, dq, b, s, h))
    return BPT_ERR_CUDA;
  AttnBwdArgs a{};
  a.s = s;
  a.heads = heads;
  a.causal = causal ? 1 : 0;
  a.n_kv = (s + AB_BN - 1) / AB_BN;
  a.lse2 = lse2;
  a.dsum = dsum;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.ld_kv = ld_kv;
  a.h = h;
  a.scale = (float)(1.0 / std::sqrt((double)dh));
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)dh));
  a.status = status;
  for (int z0 = 0; z0 < b; z0 += 65535) {
    a.beta0 = z0;
    dim3 grid((unsigned)a.n_kv * (unsigned)heads, 1, std::min(65535, b - z0));
    LaunchScope ls("attention_bwd", st);
    if (dh == 64)
      attention_bwd_tcgen05<64><<<grid, AB_THREADS, AttnBwdCfg<64>::SMEM_BYTES, st>>>(tq, tk, tv, td, tdq, a);
    else
      attention_bwd_tcgen05<128><<<grid, AB_THREADS, AttnBwdCfg<128>::SMEM_BYTES, st>>>(tq, tk, tv, td, tdq, a);
  }
  return cudaGetLastError() == cudaSuccess ? BPT_OK : BPT_ERR_CUDA;
}

int launch_dsum(const void* o, const void* dO, long long ld, long long rows, int s, int heads, int dh, float* dsum,
                cudaStream_t st) {
  const long long n = rows * heads;
  if (n <= 0) return BPT_OK;
  LaunchScope ls("attention_dsum", st);
  attn_dsum_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(o),
                                                                 reinterpret_cast<const __nv_bfloat16*>(dO), ld, rows,
                                                                 s, heads, dh, dsum);
  return cudaGetLastError() == cudaSuccess ? BPT_OK : BPT_ERR_CUDA;
}

int launch_rows_to_bf16(const float* src, long long rows, int cols, void* dst, long long ld_dst, int sms,
                        cudaStream_t st) {
  if (rows <= 0) return BPT_OK;
  const long long n = rows * (cols / 8);
  const long long blocks = std::min<long long>((n + 255) / 256, (long long)sms * 8);
  LaunchScope ls("f32_to_bf16", st);
  rows_f32_to_bf16_kernel<<<(int)blocks, 256, 0, st>>>(src, rows, cols, reinterpret_cast<__nv_bfloat16*>(dst),
                                                       ld_dst);
  return cudaGetLastError() == cudaSuccess ? BPT_OK : BPT_ERR_CUDA;
}

// The FFN side of every query block in one launch (ffn_chain.cuh): O (bf16
// rows inside out, `ldq` elements apart) -> hid, U -> out.
int launch_chain(const __nv_bfloat16* O, long long ldq, const LayerPtrs& p, long long M, int h, int ffn,
                 const Layout& L, uint8_t* ws, float* out, int sms, cudaStream_t st, int* status) {
  if (M <= 0) return BPT_OK;
  const ChainPlan& cp = L.cp;
  const long long rows = (long long)cp.gm * GEMM_BM;
  ChainArgs a{};
  a.M = M;
  a.h = h;
  a.f = ffn;
  a.m_tiles = cp.m_tiles;
  a.gm = cp.gm;
  a.groups = cp.groups;
  a.hid_slots = cp.hs;
  a.u_slots = cp.us;
  a.n_op = (h + GEMM_BN - 1) / GEMM_BN;
  a.n_up = (ffn + GEMM_BN - 1) / GEMM_BN;
  a.n_dn = a.n_op;
  a.x = reinterpret_cast<const __nv_bfloat16*>(p.x);
  a.bo = reinterpret_cast<const __nv_bfloat16*>(p.bo);
  a.b1 = reinterpret_cast<const __nv_bfloat16*>(p.b1);
  a.b2 = reinterpret_cast<const __nv_bfloat16*>(p.b2);
  a.hid = reinterpret_cast<float*>(ws + L.hid);
  a.hb = reinterpret_cast<__nv_bfloat16*>(ws + L.hb);
  a.u = reinterpret_cast<__nv_bfloat16*>(ws + L.u);
  a.out = out;
  unsigned* cnt = reinterpret_cast<unsigned*>(ws + L.cnt);
  a.op_cnt = cnt;
  a.up_cnt = cnt + cp.groups;
  a.dn_cnt = cnt + 2 * (size_t)cp.groups;
  a.status = status;
  CUtensorMap tO, tHb, tU, tWo, tW1, tW2;
  if (!map_rows(&tO, O, M, h, ldq, GEMM_BM) || !map_rows(&tHb, a.hb, cp.hs * rows, h, h, GEMM_BM) ||
      !map_rows(&tU, a.u, cp.us * rows, ffn, ffn, GEMM_BM) || !map_rows(&tWo, p.Wo, h, h, h, 64) ||
      !map_rows(&tW1, p.W1, h, ffn, ffn, 64) || !map_rows(&tW2, p.W2, ffn, h, h, 64))
    return BPT_ERR_CUDA;
  if (cudaMemsetAsync(cnt, 0, 3 * (size_t)cp.groups * sizeof(unsigned), st) != cudaSuccess)
    return BPT_ERR_CUDA;
  const long long tiles = (long long)cp.m_tiles * (a.n_op + a.n_up + a.n_dn);
  const int grid = (int)std::min<long long>(tiles, sms);
  {
    LaunchScope ls("ffn_chain", st);
    ffn_chain_tcgen05<<<grid, GEMM_THREADS, GEMM_SMEM_BYTES, st>>>(tO, tHb, tU, tWo, tW1, tW2, a);
  }
  return cudaGetLastError() == cudaSuccess ? BPT_OK : BPT_ERR_CUDA;
}

// Attention and the chain in one launch (layer_mega.cuh): the same arguments
// as launch_attention (every sequence, every row, O over Q) and launch_chain.
int launch_mega(const __nv_bfloat16* QO, long long ldq, const __nv_bfloat16* K, const __nv_bfloat16* V,
                const LayerPtrs& p, int b, int s, int h, int heads, int ffn, int causal, const Layout& L, uint8_t* ws,
                float* out, int sms, cudaStream_t st, int* status) {
  const long long M = (long long)b * s;
  if (M <= 0) return BPT_OK;
  const int dh = h / heads;
  const ChainPlan& cp = L.cp;
  const long long rows = (long long)cp.gm * GEMM_BM;
  // attention: every sequence in one grid, items in row order
  CUtensorMap tq, tk, tv;
  if (!map_seq(&tq, QO, b, s, h, ldq) || !map_seq(&tk, K, b, s, h, h) || !map_seq(&tv, V, b, s, h, h))
    return BPT_ERR_CUDA;
  unsigned* cnt = reinterpret_cast<unsigned*>(ws + L.cnt);
  AttnArgs aa{};
  aa.s = s;
  aa.heads = heads;
  aa.causal = causal ? 1 : 0;
  aa.beta0 = 0;
  aa.t_start = 0;
  aa.t_len = s;
  aa.n_pairs = (s + 2 * ATT_BM - 1) / (2 * ATT_BM);
  aa.o = const_cast<__nv_bfloat16*>(QO);
  aa.ldo = ldq;
  aa.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)dh));
  aa.status = status;
  aa.grp_cnt = cnt + 3 * (size_t)cp.groups;
  aa.grp_rows = (int)rows;
  // the chain, waiting per group on attention's count
  ChainArgs a{};
  a.M = M;
  a.h = h;
  a.f = ffn;
  a.m_tiles = cp.m_tiles;
  a.gm = cp.gm;
  a.groups = cp.groups;
  a.hid_slots = cp.hs;
  a.u_slots = cp.us;
  a.n_op = (h + GEMM_BN - 1) / GEMM_BN;
  a.n_up = (ffn + GEMM_BN - 1) / GEMM_BN;
  a.n_dn = a.n_op;
  a.x = reinterpret_cast<const __nv_bfloat16*>(p.x);
  a.bo = reinterpret_cast<const __nv_bfloat16*>(p.bo);
  a.b1 = reinterpret_cast<const __nv_bfloat16*>(p.b1);
  a.b2 = reinterpret_cast<const __nv_bfloat16*>(p.b2);
  a.hid = reinterpret_cast<float*>(ws + L.hid);
  a.hb = reinterpret_cast<__nv_bfloat16*>(ws + L.hb);
  a.u = reinterpret_cast<__nv_bfloat16*>(ws + L.u);
  a.out = out;
  a.op_cnt = cnt;
  a.up_cnt = cnt + cp.groups;
  a.dn_cnt = cnt + 2 * (size_t)cp.groups;
  a.status = status;
  a.att_cnt = aa.grp_cnt;
  a.att_heads = heads;
  CUtensorMap tO, tHb, tU, tWo, tW1, tW2;
  if (!map_rows(&tO, QO, M, h, ldq, GEMM_BM) || !map_rows(&tHb, a.hb, cp.hs * rows, h, h, GEMM_BM) ||
      !map_rows(&tU, a.u, cp.us * rows, ffn, ffn, GEMM_BM) || !map_rows(&tWo, p.Wo, h, h, h, 64) ||
      !map_rows(&tW1, p.W1, h, ffn, ffn, 64) || !map_rows(&tW2, p.W2, ffn, h, h, 64))
    return BPT_ERR_CUDA;
  MegaArgs mg{};
  mg.ticket = cnt + 4 * (size_t)cp.groups;
  const long long n_att = (long long)b * aa.n_pairs * heads;
  const long long tiles = (long long)cp.m_tiles * (a.n_op + a.n_up + a.n_dn);
  const long long n_chain = std::min<long long>(tiles, sms);
  if (n_att + n_chain > 0x7fffffffLL) return BPT_ERR_SHAPE;
  mg.n_att = (int)n_att;
  if (cudaMemsetAsync(cnt, 0, (4 * (size_t)cp.groups + 1) * sizeof(unsigned), st) != cudaSuccess)
    return BPT_ERR_CUDA;
  {
    LaunchScope ls("layer_mega", st);
    const unsigned grid = (unsigned)(n_att + n_chain);
    if (dh == 64)
      layer_mega_tcgen05<64><<<grid, ATT_THREADS, mega_smem_bytes<64>(), st>>>(tq, tk, tv, tO, tHb, tU, tWo, tW1,
                                                                               tW2, aa, a, mg);
    else
      layer_mega_tcgen05<128><<<grid, ATT_THREADS, mega_smem_bytes<128>(), st>>>(tq, tk, tv, tO, tHb, tU, tWo, tW1,
                                                                                 tW2, aa, a, mg);
  }
  return cudaGetLastError() == cudaSuccess ? BPT_OK : BPT_ERR_CUDA;
}

__global__ void f32_to_bf16_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst, long long n) {
  const long long n4 = n / 4;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    const float4 f = reinterpret_cast<const float4*>(src)[i];
    uint2 o;
    o.x = pack_bf16x2(f.x, f.y);
    o.y = pack_bf16x2(f.z, f.w);
    reinterpret_cast<uint2*>(dst)[i] = o;
  }
  for (long long i = n4 * 4 + blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x)
    dst[i] = __float2bfloat16_rn(src[i]);
}

int launch_convert(const float* src, void* dst, long long n, int sms, cudaStream_t st) {
  if (n <= 0) return BPT_OK;
  const long long blocks = std::min<long long>((n / 4 + 255) / 256 + 1, (long long)sms * 8);
  LaunchScope ls("f32_to_bf16", st);
  f32_to_bf16_kernel<<<(int)blocks, 256, 0, st>>>(src, reinterpret_cast<__nv_bfloat16*>(dst), n);
  return cudaGetLastError() == cudaSuccess ? BPT_OK : BPT_ERR_CUDA;
}

// The two bf16 parts of fp32 values: hi = bf16(v), lo = bf16(v - hi), so that
// hi + lo carries v to about 16 significant bits. hi is also written to hi2
// when it is given.
__global__ void split_bf16_kernel(const float* __restrict__ src, long long n, __nv_bfloat16* hi,
                                  __nv_bfloat16* lo, __nv_bfloat16* hi2) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const float v = src[i];
    const __nv_bfloat16 a = __float2bfloat16_rn(v);
    const __nv_bfloat16 b = __float2bfloat16_rn(v - __bfloat162float(a));
    hi[i] = a;
    lo[i] = b;
    if (hi2) hi2[i] = a;
  }
}

// Rows of x as [x_hi | x_lo]: dst row r = hi parts of src row r, then lo parts.
__global__ void split_rows_bf16_kernel(const float* __restrict__ src, long long rows, int cols,
                                       __nv_bfloat16* dst) {
  const long long n = rows * cols;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const long long r = i / cols, c = i - r * cols;
    const float v = src[i];
    const __nv_bfloat16 a = __float2bfloat16_rn(v);
    dst[r * 2 * cols + c] = a;
    dst[r * 2 * cols + cols + c] = __float2bfloat16_rn(v - __bfloat162float(a));
  }
}

int launch_split(const float* src, long long n, void* hi, void* lo, void* hi2, int sms, cudaStream_t st) {
  if (n <= 0) return BPT_OK;
  const long long blocks = std::min<long long>((n + 255) / 256, (long long)sms * 8);
  LaunchScope ls("split_bf16", st);
  split_bf16_kernel<<<(int)blocks, 256, 0, st>>>(src, n, reinterpret_cast<__nv_bfloat16*>(hi),
                                                 reinterpret_cast<__nv_bfloat16*>(lo),
                                                 reinterpret_cast<__nv_bfloat16*>(hi2));
  return cudaGetLastError() == cudaSuccess ? BPT_OK : BPT_ERR_CUDA;
}

int launch_split_rows(const float* src, long long rows, int cols, void* dst, int sms, cudaStream_t st) {
  const long long n = rows * cols;
  if (n <= 0) return BPT_OK;
  const long long blocks = std::min<long long>((n + 255) / 256, (long long)sms * 8);
  LaunchScope ls("split_bf16", st);
  split_rows_bf16_kernel<<<(int)blocks, 256, 0, st>>>(src, rows, cols, reinterpret_cast<__nv_bfloat16*>(dst));
  return cudaGetLastError() == cudaSuccess ? BPT_OK : BPT_ERR_CUDA;
}

#define BPT_TRY(expr)            \
  do {                           \
    int _r = (expr);             \
    if (_r != BPT_OK) return _r; \
  } while (0)


// FFN width: a positive multiple of 64 (one K step of the GEMMs, one TMA box)
int check_ffn(int ffn) { return (ffn <= 0 || ffn % 64) ? BPT_ERR_SHAPE : BPT_OK; }

int validate_layer(int dtype, const LayerPtrs& p, int b, int s, int h, int heads, int ffn, int q_block,
                   int kv_block, const float* out) {
  if (dtype != BPT_DTYPE_BF16 && dtype != BPT_DTYPE_F32) return BPT_ERR_DTYPE;
  BPT_TRY(check_shape(b, s, h, heads));
  BPT_TRY(check_ffn(ffn));
  BPT_TRY(check_blocks(s, q_block, kv_block));
  if ((long long)b * s == 0) return BPT_OK;
  const void* ptrs[10] = {p.x, p.Wqkv, p.bqkv, p.Wo, p.bo, p.W1, p.b1, p.W2, p.b2, out};
  for (const void* q : ptrs)
    if (!q) return BPT_ERR_NULL;
  for (const void* q : ptrs)
    if (!aligned16(q)) return BPT_ERR_ALIGN;
  const size_t es = dtype == BPT_DTYPE_F32 ? 4 : 2;
  const size_t tok = (size_t)b * s;
  const Range ro = rng(out, tok * h * 4);
  const Range in[9] = {rng(p.x, tok * h * es),      rng(p.Wqkv, (size_t)h * 3 * h * es), rng(p.bqkv, 3 * (size_t)h * es),
                       rng(p.Wo, (size_t)h * h * es), rng(p.bo, (size_t)h * es),          rng(p.W1, (size_t)h * ffn * es),
                       rng(p.b1, (size_t)ffn * es), rng(p.W2, (size_t)ffn * h * es),       rng(p.b2, (size_t)h * es)};
  for (const Range& r : in)
    if (overlap(ro, r)) return BPT_ERR_ALIAS;
  return BPT_OK;
}

// Called after the launches that finish rows [row0, row0 + rows) of out (each
// FFN wave's FFN-down), so that a caller can start copying them out. With
// split_last, the last wave runs as two halves, each followed by the call, so
// that only the second half's copy waits for the last launch.
struct WaveHook {
  int (*fn)(void* ctx, long long row0, long long rows) = nullptr;
  void* ctx = nullptr;
  bool split_last = false;
};

// x arriving in row chunks (bf16 inputs): chunk c, rows [c rows, (c + 1) rows),
// is in place once ev[c] has completed; the projection then runs chunk by
// chunk, each launch after its chunk's event, instead of after all of x.
struct XChunks {
  int n = 0;
  long long rows = 0;
  const cudaEvent_t* ev = nullptr;
};

// Whether a layer can run wave by wave (attention of a wave's rows, then its
// FFN side): causal attention (a row needs only the keys at or before it)
// and the per-GEMM wave schedule.
bool interleavable(int dtype, int causal, int wave_rows) { return causal && !use_chain(dtype, wave_rows); }

// interleave_req, where interleavable(): attention runs wave by wave, each
// wave's rows just before that wave's FFN side, and the first input's row
// chunks (xc) are projected as the waves need them, so that results start to
// come out early in the layer rather than after all of attention. The caller
// then sizes ws with layout_for(..., interleavable(dtype, causal, wave_rows)),
// whose FFN scratch lies beside K/V; that workspace also holds the layout
// without interleave.
int run_layer(int dtype, const LayerPtrs& p, int b, int s, int h, int heads, int ffn, int q_block, int causal,
              int wave_rows, uint8_t* ws, float* out, cudaStream_t st, int sms, const WaveHook* hook = nullptr,
              const XChunks* xc = nullptr, __nv_bfloat16* o_save = nullptr, float* lse2_save = nullptr,
              bool interleave_req = false) {
  int* status = nullptr;
  BPT_TRY(stream_status_word(st, &status));
  const bool interleave = interleave_req && interleavable(dtype, causal, wave_rows) && o_save == nullptr;
  const Layout L = layout_for(dtype, b, s, h, ffn, q_block, wave_rows, interleave);
  const long long tok = (long long)b * s;
  __nv_bfloat16* K = reinterpret_cast<__nv_bfloat16*>(ws + L.k);
  __nv_bfloat16* V = reinterpret_cast<__nv_bfloat16*>(ws + L.v);
  float* HID = reinterpret_cast<float*>(ws + L.hid);
  __nv_bfloat16* HB = reinterpret_cast<__nv_bfloat16*>(ws + L.hb);
  __nv_bfloat16* U = reinterpret_cast<__nv_bfloat16*>(ws + L.u);
  // Q, then the attention output O, live in out: bf16 row r in the first half
  // of out's fp32 row r
  __nv_bfloat16* QO = reinterpret_cast<__nv_bfloat16*>(out);
  const long long ldq = 2LL * h;

  const void *xa = p.x, *wqkv = p.Wqkv, *wo = p.Wo, *w1 = p.W1, *w2 = p.W2;
  const int f32 = dtype == BPT_DTYPE_F32 ? 1 : 0;
  const bool mega = L.mega && mega_available() && o_save == nullptr;
  const __nv_bfloat16* O = o_save != nullptr ? o_save : QO;
  const long long ldo = o_save != nullptr ? (long long)h : ldq;
  // Attention of the flat rows [r0, r0 + m), one launch per piece (whole
  // sequences, or one sequence's run of rows). Every row's arithmetic is the
  // same as in one launch over all rows.
  auto attend_rows = [&](long long r0, long long m) -> int {
    return for_each_row_piece(r0, m, b, s, [&](const RowPiece& pc) -> int {
      const long long r = (long long)pc.beta * s + pc.t_start;
      return launch_attention(QO, ldq, K, V, b, s, h, heads, causal, pc.beta, pc.n_seq, pc.t_start, pc.t_len,
                              const_cast<__nv_bfloat16*>(O) + r * ldo, ldo, st, status);
    });
  };
  // the first input's row chunks, projected in order up to a given row
  const bool chunked = !f32 && xc != nullptr && xc->n > 0;
  int next_chunk = 0;
  long long projected = 0;
  if (f32) {
    // fp32 inputs: split bf16 products, so that neither x nor the weights
    // lose more than about 16 significant bits (x W = x_hi W_hi + x_hi W_lo +
    // x_lo W_hi for the projection; a W_hi + a W_lo for the other GEMMs,
    // whose A is a bf16 activation of the path)
    const long long q3 = 3LL * h * h;
    BPT_TRY(launch_split_rows((const float*)p.x, tok, h, ws + L.xb, sms, st));
    BPT_TRY(launch_split((const float*)p.Wqkv, q3, ws + L.wqkv, ws + L.wqkv + q3 * 2, ws + L.wqkv + q3 * 4, sms, st));
    BPT_TRY(launch_split((const float*)p.Wo, 1LL * h * h, ws + L.wo, ws + L.wo + 2LL * h * h, nullptr, sms, st));
    BPT_TRY(launch_split((const float*)p.W1, (long long)h * ffn, ws + L.w1, ws + L.w1 + 2LL * h * ffn, nullptr, sms,
                         st));
    BPT_TRY(launch_split((const float*)p.W2, (long long)ffn * h, ws + L.w2, ws + L.w2 + 2LL * ffn * h, nullptr, sms,
                         st));
    xa = ws + L.xb;
    wqkv = ws + L.wqkv;
    wo = ws + L.wo;
    w1 = ws + L.w1;
    w2 = ws + L.w2;
  }

  // step 1: projection of the whole sequence
  GemmArgs qa{};
  qa.bias = p.bqkv;
  qa.bias_f32 = f32;
  qa.q = QO;
  qa.ldq = ldq;
  qa.k = K;
  qa.v = V;
  qa.ldkv = h;
  qa.h = h;
  auto project_to = [&](long long end) -> int {
    for (; next_chunk < xc->n && projected < end; ++next_chunk) {
      const long long r0 = (long long)next_chunk * xc->rows, m = std::min(xc->rows, tok - r0);
      if (m <= 0) {
        projected = tok;
        break;
      }
      if (cudaStreamWaitEvent(st, xc->ev[next_chunk], 0) != cudaSuccess) return BPT_ERR_CUDA;
      GemmArgs ac = qa;
      ac.q = QO + r0 * ldq;
      ac.k = K + r0 * h;
      ac.v = V + r0 * h;
      BPT_TRY(launch_gemm<EPI_QKV>(reinterpret_cast<const __nv_bfloat16*>(xa) + r0 * h, m, h, h, wqkv, 3LL * h, ac,
                                   sms, st, status, "gemm_qkv"));
      projected = r0 + m;
    }
    return BPT_OK;
  };
  {
    const GemmArgs& a = qa;
    if (f32) {
      BPT_TRY(launch_gemm_split<EPI_QKV>(xa, tok, 2LL * h, 2LL * h, wqkv, 3LL * h, 3LL * h, 2, h / GEMM_BK, a, sms,
                                         st, status, "gemm_qkv"));
    } else if (chunked) {
      if (!interleave) BPT_TRY(project_to(tok));
    } else {
      BPT_TRY(launch_gemm<EPI_QKV>(xa, tok, h, h, wqkv, 3LL * h, a, sms, st, status, "gemm_qkv"));
    }
  }

  // steps 4-10 for every query block at once: each CTA overwrites the Q of its
  // own rows and head with their attention output (or, in the one-launch
  // schedule, attention and the whole FFN side together)
  // (With o_save, for a later backward: O goes to o_save, h apart, and each row's
  // log-sum-exp to lse2_save; the FFN side then reads O from there.)
  if (mega) return launch_mega(QO, ldq, K, V, p, b, s, h, heads, ffn, causal, L, ws, out, sms, st, status);
  if (!interleave)
    BPT_TRY(launch_attention(QO, ldq, K, V, b, s, h, heads, causal, 0, b, 0, s, const_cast<__nv_bfloat16*>(O), ldo,
                             st, status, lse2_save));

  // step 11 for every query block: out-projection, residuals and FFN
  if (L.chain) return launch_chain(O, ldo, p, tok, h, ffn, L, ws, out, sms, st, status);
  auto ffn_side = [&](const Wave& w) -> int {
    const long long rows = w.rows();
    GemmArgs a{};
    a.resid = p.x;
    a.resid_f32 = f32;
    a.ld_resid = h;
    a.hid = HID;
    a.ld_hid = h;
    a.out = out;
    a.ld_out = h;
    a.row0 = w.row0;
    a.bias_f32 = f32;
    a.bias = p.bo;
    a.dst = HB;
    a.ld_dst = h;
    const int sp = f32 ? 1 : 0, kf = f32 ? 2 : 1;  // fp32 inputs: A against [W_hi; W_lo]
    BPT_TRY(launch_gemm_split<EPI_OUTPROJ>(O + w.row0 * ldo, rows, h, ldo, wo, (long long)kf * h, h, sp,
                                           h / GEMM_BK, a, sms, st, status, "gemm_outproj"));
    a.bias = p.b1;
    a.dst = U;
    a.ld_dst = ffn;
    BPT_TRY(launch_gemm_split<EPI_FFN_UP>(HB, rows, h, h, w1, (long long)kf * h, ffn, sp, h / GEMM_BK, a, sms, st,
                                          status, "gemm_ffn_up"));
    a.bias = p.b2;
    BPT_TRY(launch_gemm_split<EPI_FFN_DOWN>(U, rows, ffn, ffn, w2, (long long)kf * ffn, h, sp, ffn / GEMM_BK, a, sms,
                                            st, status, "gemm_ffn_down"));
    return hook ? hook->fn(hook->ctx, w.row0, rows) : BPT_OK;
  };
  return for_each_wave(b, s, h, ffn, q_block, wave_rows, [&](const Wave& w) -> int {
    // The last wave as two halves (hook->split_last): the first half's rows are
    // copied out while the second half computes. Each row's arithmetic is the
    // same either way.
    const long long rows = w.rows();
    if (interleave) {
      if (chunked) BPT_TRY(project_to(w.row0 + rows));
      BPT_TRY(attend_rows(w.row0, rows));
    }
    if (hook != nullptr && hook->split_last && w.n_seq == 1 && w.row0 + rows == tok && rows >= 2 * GEMM_BM) {
      const int half = (int)((rows / 2 + GEMM_BM - 1) / GEMM_BM * GEMM_BM);
      BPT_TRY(ffn_side(Wave{w.row0, w.beta0, 1, w.t_start, half}));
      return ffn_side(Wave{w.row0 + half, w.beta0, 1, w.t_start + half, w.t_len - half});
    }
    return ffn_side(w);
  });
}

int layer_entry(int dtype, const LayerPtrs& p, int b, int s, int h, int heads, int ffn, int q_block, int kv_block,
                int causal, int wave_rows, void* workspace, size_t ws_bytes, bool caller_ws, float* out,
                void* stream, __nv_bfloat16* o_save = nullptr, float* lse2_save = nullptr) {
  BPT_TRY(validate_layer(dtype, p, b, s, h, heads, ffn, q_block, kv_block, out));
  if ((long long)b * s == 0) return BPT_OK;
  const Layout L = layout_for(dtype, b, s, h, ffn, q_block, wave_rows);
  if (caller_ws) {
    if (!workspace) return BPT_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return BPT_ERR_ALIGN;
    if (ws_bytes < L.total) return BPT_ERR_NOMEM;
    const size_t es = dtype == BPT_DTYPE_F32 ? 4 : 2;
    const size_t tok = (size_t)b * s;
    const Range rw = rng(workspace, L.total);
    const Range others[10] = {rng(out, tok * h * 4),      rng(p.x, tok * h * es),        rng(p.Wqkv, (size_t)3 * h * h * es),
                              rng(p.bqkv, (size_t)3 * h * es), rng(p.Wo, (size_t)h * h * es), rng(p.bo, (size_t)h * es),
                              rng(p.W1, (size_t)h * ffn * es), rng(p.b1, (size_t)ffn * es), rng(p.W2, (size_t)ffn * h * es),
                              rng(p.b2, (size_t)h * es)};
    for (const Range& r : others)
      if (overlap(rw, r)) return BPT_ERR_ALIAS;
  }
  int sms = 0;
  BPT_TRY(check_device(&sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  if (!caller_ws) {
    cudaMemPool_t pool = nullptr;
    BPT_TRY(workspace_pool(&pool));
    void* m = nullptr;
    if (cudaMallocFromPoolAsync(&m, L.total, pool, st) != cudaSuccess) {
      cudaGetLastError();
      return BPT_ERR_NOMEM;
    }
    ws = reinterpret_cast<uint8_t*>(m);
  }
  const int r =
      run_layer(dtype, p, b, s, h, heads, ffn, q_block, causal, wave_rows, ws, out, st, sms, nullptr, nullptr, o_save,
                lse2_save);
  if (!caller_ws) cudaFreeAsync(ws, st);
  return r;
}

// Scratch of bpt_layer_forward_noalloc: one fixed array in device memory,
// created with the library image on every device that loads it. In host code
// the name g_static_ws denotes a host-side stand-in, never the device address.
static __device__ __align__(256) unsigned char g_static_ws[BPT_STATIC_WORKSPACE_BYTES];

// Device address of g_static_ws on the current device. It is looked up on
// every call, with the device current: a symbol lookup allocates nothing, and
// an address saved from an earlier call would be stale once cudaDeviceReset
// (or a new context on the device) has recreated the module. The first call
// on a device also loads the library's device image there.
int static_workspace(void** ptr) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess || !p) {
    cudaGetLastError();
    return BPT_ERR_CUDA;
  }
  *ptr = p;
  return BPT_OK;
}

// n independent inputs from host memory: input i is copied in while input
// i - 1 computes, and its result is copied out while input i + 1 computes.
// Two device buffers each for x and out plus one workspace come from the
// library's pool; non-blocking copy streams are ordered against the compute
// stream with events; every copy is one cudaMemcpyAsync. Each input comes
// in, and each result goes out, in two halves on two streams, so that two
// copy engines share every transfer.
struct HostPipe {
  static constexpr int kCopy = 2;  // streams per direction
  cudaStream_t h2d[kCopy] = {}, d2h[kCopy] = {};
  cudaEvent_t ready = nullptr, comp_done[2] = {}, h2d_done[2][kCopy] = {}, d2h_done[2][kCopy] = {};
  cudaEvent_t wave_done = nullptr;  // re-recorded after each FFN wave (waits take its latest record)
  static constexpr int kXChunks = 4;  // the first input arrives in this many row chunks
  cudaEvent_t x_chunk[kXChunks] = {};
  bool create() {
    for (int c = 0; c < kCopy; ++c)
      if (cudaStreamCreateWithFlags(&h2d[c], cudaStreamNonBlocking) != cudaSuccess ||
          cudaStreamCreateWithFlags(&d2h[c], cudaStreamNonBlocking) != cudaSuccess)
        return false;
    cudaEvent_t* all[4] = {&ready, &comp_done[0], &comp_done[1], &wave_done};
    for (cudaEvent_t* e : all)
      if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) return false;
    for (int k = 0; k < 2; ++k)
      for (int c = 0; c < kCopy; ++c)
        if (cudaEventCreateWithFlags(&h2d_done[k][c], cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&d2h_done[k][c], cudaEventDisableTiming) != cudaSuccess)
          return false;
    for (cudaEvent_t& e : x_chunk)
      if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return false;
    return true;
  }
  bool sync_copies() {
    bool ok = true;
    for (int c = 0; c < kCopy; ++c) {
      if (h2d[c]) ok = cudaStreamSynchronize(h2d[c]) == cudaSuccess && ok;
      if (d2h[c]) ok = cudaStreamSynchronize(d2h[c]) == cudaSuccess && ok;
    }
    return ok;
  }
  void destroy() {
    sync_copies();
    for (int c = 0; c < kCopy; ++c) {
      if (h2d[c]) cudaStreamDestroy(h2d[c]);
      if (d2h[c]) cudaStreamDestroy(d2h[c]);
    }
    cudaEvent_t all[4] = {ready, comp_done[0], comp_done[1], wave_done};
    for (cudaEvent_t e : all)
      if (e) cudaEventDestroy(e);
    for (int k = 0; k < 2; ++k)
      for (int c = 0; c < kCopy; ++c) {
        if (h2d_done[k][c]) cudaEventDestroy(h2d_done[k][c]);
        if (d2h_done[k][c]) cudaEventDestroy(d2h_done[k][c]);
      }
    for (cudaEvent_t e : x_chunk)
      if (e) cudaEventDestroy(e);
  }
};

// Copies the rows of one finished FFN wave from device to host memory, half on
// each copy stream, after the launches queued so far on the compute stream.
struct WaveCopy {
  HostPipe* pp;
  cudaStream_t st;
  const uint8_t* dev;  // result rows on the device
  uint8_t* host;       // result rows in host memory
  size_t row_bytes;
  int waves;
  static int on_wave(void* ctx, long long row0, long long rows) {
    WaveCopy& c = *reinterpret_cast<WaveCopy*>(ctx);
    ++c.waves;
    if (cudaEventRecord(c.pp->wave_done, c.st) != cudaSuccess) return BPT_ERR_CUDA;
    const long long half = rows / 2;
    for (int k = 0; k < HostPipe::kCopy; ++k) {
      const long long r0 = row0 + (k == 0 ? 0 : half), n = k == 0 ? half : rows - half;
      if (n <= 0) continue;
      const size_t off = (size_t)r0 * c.row_bytes, bytes = (size_t)n * c.row_bytes;
      if (cudaStreamWaitEvent(c.pp->d2h[k], c.pp->wave_done, 0) != cudaSuccess ||
          cudaMemcpyAsync(c.host + off, c.dev + off, bytes, cudaMemcpyDeviceToHost, c.pp->d2h[k]) != cudaSuccess)
        return BPT_ERR_CUDA;
    }
    return BPT_OK;
  }
};

int host_entry(int dtype, const void* x_host, long long x_stride, const LayerPtrs& w, int b, int s, int h,
               int heads, int q_block, int kv_block, int causal, float* out_host, long long out_stride, int n,
               void* stream) {
  if (dtype != BPT_DTYPE_BF16 && dtype != BPT_DTYPE_F32) return BPT_ERR_DTYPE;
  BPT_TRY(check_shape(b, s, h, heads));
  BPT_TRY(check_blocks(s, q_block, kv_block));
  if (n < 0) return BPT_ERR_SHAPE;
  const size_t es = dtype == BPT_DTYPE_F32 ? 4 : 2;
  const size_t tok = (size_t)b * s;
  const size_t xb = tok * h * es, ob = tok * h * 4;
  if (n == 0 || tok == 0) return BPT_OK;
  const void* dev_ptrs[8] = {w.Wqkv, w.bqkv, w.Wo, w.bo, w.W1, w.b1, w.W2, w.b2};
  if (!x_host || !out_host) return BPT_ERR_NULL;
  for (const void* q : dev_ptrs)
    if (!q) return BPT_ERR_NULL;
  for (const void* q : dev_ptrs)
    if (!aligned16(q)) return BPT_ERR_ALIGN;
  if (x_stride < 0 || out_stride < 0 || (x_stride && (size_t)x_stride < xb) || (out_stride && (size_t)out_stride < ob))
    return BPT_ERR_SHAPE;
  // the host ranges must be addressable: stride * (n - 1) + size without overflow
  const size_t lim = (size_t)1 << 62;
  if ((x_stride && (size_t)(n - 1) > (lim - xb) / (size_t)x_stride) ||
      (out_stride && (size_t)(n - 1) > (lim - ob) / (size_t)out_stride))
    return BPT_ERR_SHAPE;
  // host ranges: every input against every output (both are arithmetic progressions)
  const Range xr = rng(x_host, (size_t)x_stride * (n - 1) + xb), orr = rng(out_host, (size_t)out_stride * (n - 1) + ob);
  if (overlap(xr, orr)) return BPT_ERR_ALIAS;
  int sms = 0;
  BPT_TRY(check_device(&sms));
  // causal: attention and the FFN side wave by wave for the first and last
  // input (run_layer's interleave), with one wave's FFN scratch beside the K/V
  // copies (the inputs between them use the same workspace with the scratch
  // over K/V)
  const Layout L = layout_for(dtype, b, s, h, 4 * h, q_block, 0, interleavable(dtype, causal, 0));
  const size_t xa = align_up(xb, 1024), oa = align_up(ob, 1024);
  const size_t total = 2 * xa + 2 * oa + L.total;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaMemPool_t pool = nullptr;
  BPT_TRY(workspace_pool(&pool));
  void* mem = nullptr;
  if (cudaMallocFromPoolAsync(&mem, total, pool, st) != cudaSuccess) {
    cudaGetLastError();
    return BPT_ERR_NOMEM;
  }
  uint8_t* base = reinterpret_cast<uint8_t*>(mem);
  uint8_t* xdev[2] = {base, base + xa};
  float* odev[2] = {reinterpret_cast<float*>(base + 2 * xa), reinterpret_cast<float*>(base + 2 * xa + oa)};
  uint8_t* ws = base + 2 * xa + 2 * oa;
  HostPipe pp;
  int r = pp.create() ? BPT_OK : BPT_ERR_CUDA;
  if (r == BPT_OK) {
    bool cu = cudaEventRecord(pp.ready, st) == cudaSuccess;
    for (int c = 0; c < HostPipe::kCopy; ++c)
      cu = cu && cudaStreamWaitEvent(pp.h2d[c], pp.ready, 0) == cudaSuccess &&
           cudaStreamWaitEvent(pp.d2h[c], pp.ready, 0) == cudaSuccess;
    // transfers split at a row boundary: [0, half) and [half, end)
    const size_t x_half = (tok / 2) * h * es, o_half = (tok / 2) * h * 4;
    for (int i = 0; cu && r == BPT_OK && i < n; ++i) {
      const int k = i & 1;
      const uint8_t* xi = reinterpret_cast<const uint8_t*>(x_host) + (size_t)x_stride * i;
      uint8_t* oi = reinterpret_cast<uint8_t*>(out_host) + (size_t)out_stride * i;
      // The first input (bf16) comes in row chunks and the projection starts on each
      // chunk as it lands, so that only the first chunk's copy is exposed; later
      // inputs arrive while the previous one computes.
      XChunks xc;
      const long long xrows = ((long long)tok + HostPipe::kXChunks - 1) / HostPipe::kXChunks;
      const long long crows = (xrows + 127) / 128 * 128;
      if (i == 0 && dtype == BPT_DTYPE_BF16 && (long long)tok > crows) {
        xc.n = (int)(((long long)tok + crows - 1) / crows);
        xc.rows = crows;
        xc.ev = pp.x_chunk;
        for (int c = 0; cu && c < xc.n; ++c) {
          const size_t lo = (size_t)(c * crows) * h * es;
          const size_t bytes = (size_t)std::min<long long>(crows, (long long)tok - c * crows) * h * es;
          // in order on one stream: the link's bandwidth is shared by every copy in
          // flight in a direction, so chunk 0 lands soonest when it goes alone
          cu = cudaMemcpyAsync(xdev[k] + lo, xi + lo, bytes, cudaMemcpyHostToDevice, pp.h2d[0]) == cudaSuccess &&
               cudaEventRecord(pp.x_chunk[c], pp.h2d[0]) == cudaSuccess;
        }
        // the copy streams' completion events still mark the whole input
        for (int c = 0; cu && c < HostPipe::kCopy; ++c)
          cu = cudaEventRecord(pp.h2d_done[k][c], pp.h2d[c]) == cudaSuccess;
      } else {
        // x buffer k is free once input i - 2 has been computed
        for (int c = 0; c < HostPipe::kCopy; ++c) {
          const size_t lo = c == 0 ? 0 : x_half, bytes = c == 0 ? x_half : xb - x_half;
          if (i >= 2) cu = cu && cudaStreamWaitEvent(pp.h2d[c], pp.comp_done[k], 0) == cudaSuccess;
          cu = cu && (bytes == 0 || cudaMemcpyAsync(xdev[k] + lo, xi + lo, bytes, cudaMemcpyHostToDevice,
                                                    pp.h2d[c]) == cudaSuccess) &&
               cudaEventRecord(pp.h2d_done[k][c], pp.h2d[c]) == cudaSuccess;
          cu = cu && cudaStreamWaitEvent(st, pp.h2d_done[k][c], 0) == cudaSuccess;
        }
      }
      // out buffer k is free once result i - 2 has been copied out
      for (int c = 0; i >= 2 && c < HostPipe::kCopy; ++c)
        cu = cu && cudaStreamWaitEvent(st, pp.d2h_done[k][c], 0) == cudaSuccess;
      if (!cu) break;
      LayerPtrs p = w;
      p.x = xdev[k];
      // each FFN wave's rows of the result are copied out as soon as they are final
      // (split over the copy streams), overlapping the waves still to run
      WaveCopy wc{&pp, st, reinterpret_cast<const uint8_t*>(odev[k]), oi, (size_t)h * 4, 0};
      // the last input's last wave in halves: its copy out is the call's tail
      const WaveHook hook{&WaveCopy::on_wave, &wc, i == n - 1};
      // wave by wave only where it shortens the call: the first input (whose
      // copy in is not hidden) and the last (whose copy out is the call's tail);
      // between them one attention launch per input leaves fewer launch tails,
      // and the copies are hidden by the neighbouring inputs' compute
      r = run_layer(dtype, p, b, s, h, heads, 4 * h, q_block, causal, 0, ws, odev[k], st, sms, &hook,
                    xc.n > 0 ? &xc : nullptr, nullptr, nullptr, i == 0 || i == n - 1);
      if (r != BPT_OK) break;
      cu = cudaEventRecord(pp.comp_done[k], st) == cudaSuccess;
      for (int c = 0; c < HostPipe::kCopy; ++c) {
        // a schedule without waves (one FFN launch) copies the whole result here
        const size_t lo = c == 0 ? 0 : o_half, bytes = c == 0 ? o_half : ob - o_half;
        if (wc.waves == 0)
          cu = cu && cudaStreamWaitEvent(pp.d2h[c], pp.comp_done[k], 0) == cudaSuccess &&
               (bytes == 0 || cudaMemcpyAsync(oi + lo, reinterpret_cast<uint8_t*>(odev[k]) + lo, bytes,
                                              cudaMemcpyDeviceToHost, pp.d2h[c]) == cudaSuccess);
        cu = cu && cudaEventRecord(pp.d2h_done[k][c], pp.d2h[c]) == cudaSuccess;
      }
    }
    if (!cu && r == BPT_OK) r = BPT_ERR_CUDA;
  }
  // the buffers go back to the pool only after every copy has finished
  if (!pp.sync_copies() && r == BPT_OK) r = BPT_ERR_CUDA;
  cudaFreeAsync(mem, st);
  if (cudaStreamSynchronize(st) != cudaSuccess && r == BPT_OK) r = BPT_ERR_CUDA;
  pp.destroy();
  return r;
}

}  // namespace
}  // namespace bpt

using namespace bpt;

extern "C" {

const char* bpt_status_string(int status) {
  switch (status) {
    case BPT_OK: return "BPT_OK";
    case BPT_ERR_NULL: return "BPT_ERR_NULL: a required pointer is NULL";
    case BPT_ERR_SHAPE: return "BPT_ERR_SHAPE: bad b, s, h or heads (dh = h/heads must be 64 or 128)";
    case BPT_ERR_BLOCK: return "BPT_ERR_BLOCK: q_block/kv_block must be in [1, s] and divide s";
    case BPT_ERR_ALIGN: return "BPT_ERR_ALIGN: pointers must be 16-byte aligned (workspace 256-byte)";
    case BPT_ERR_ALIAS: return "BPT_ERR_ALIAS: out or workspace overlaps another argument";
    case BPT_ERR_NOMEM: return "BPT_ERR_NOMEM: workspace allocation failed or ws_bytes too small";
    case BPT_ERR_CUDA: return "BPT_ERR_CUDA: a CUDA call failed";
    case BPT_ERR_TIMEOUT: return "BPT_ERR_TIMEOUT: a kernel gave up a bounded wait";
    case BPT_ERR_UNSUPPORTED: return "BPT_ERR_UNSUPPORTED: the current device is not sm_100";
    case BPT_ERR_DTYPE: return "BPT_ERR_DTYPE: unknown dtype";
    default: return "unknown bpt status";
  }
}

int bpt_layer_forward(const void* x, const void* Wqkv, const void* bqkv, const void* Wo, const void* bo,
                      const void* W1, const void* b1, const void* W2, const void* b2, int b, int s, int h,
                      int heads, int q_block, int kv_block, int causal, float* out, void* stream) {
  const LayerPtrs p{x, Wqkv, bqkv, Wo, bo, W1, b1, W2, b2};
  if (check_shape(b, s, h, heads) != BPT_OK) return BPT_ERR_SHAPE;
  return layer_entry(BPT_DTYPE_BF16, p, b, s, h, heads, 4 * h, q_block, kv_block, causal, 0, nullptr, 0, false, out,
                     stream);
}

int bpt_layer_forward_f32(const float* x, const float* Wqkv, const float* bqkv, const float* Wo, const float* bo,
                          const float* W1, const float* b1, const float* W2, const float* b2, int b, int s, int h,
                          int heads, int q_block, int kv_block, int causal, float* out, void* stream) {
  const LayerPtrs p{x, Wqkv, bqkv, Wo, bo, W1, b1, W2, b2};
  if (check_shape(b, s, h, heads) != BPT_OK) return BPT_ERR_SHAPE;
  return layer_entry(BPT_DTYPE_F32, p, b, s, h, heads, 4 * h, q_block, kv_block, causal, 0, nullptr, 0, false, out,
                     stream);
}

size_t bpt_layer_workspace_bytes_ffn(int dtype, int b, int s, int h, int heads, int ffn, int q_block, int kv_block,
                                     int wave_rows) {
  if (dtype != BPT_DTYPE_BF16 && dtype != BPT_DTYPE_F32) return 0;
  if (check_shape(b, s, h, heads) != BPT_OK || check_blocks(s, q_block, kv_block) != BPT_OK) return 0;
  if (check_ffn(ffn) != BPT_OK) return 0;
  if ((long long)b * s == 0) return 0;
  return layout_for(dtype, b, s, h, ffn, q_block, wave_rows).total;
}

size_t bpt_layer_workspace_bytes(int dtype, int b, int s, int h, int heads, int q_block, int kv_block,
                                 int wave_rows) {
  if (check_shape(b, s, h, heads) != BPT_OK) return 0;
  return bpt_layer_workspace_bytes_ffn(dtype, b, s, h, heads, 4 * h, q_block, kv_block, wave_rows);
}

int bpt_layer_forward_ws(int dtype, const void* x, const void* Wqkv, const void* bqkv, const void* Wo,
                         const void* bo, const void* W1, const void* b1, const void* W2, const void* b2, int b,
                         int s, int h, int heads, int q_block, int kv_block, int causal, int wave_rows,
                         void* workspace, size_t ws_bytes, float* out, void* stream) {
  const LayerPtrs p{x, Wqkv, bqkv, Wo, bo, W1, b1, W2, b2};
  if (check_shape(b, s, h, heads) != BPT_OK) return BPT_ERR_SHAPE;
  return layer_entry(dtype, p, b, s, h, heads, 4 * h, q_block, kv_block, causal, wave_rows, workspace, ws_bytes, true,
                     out, stream);
}

int bpt_layer_forward_ffn(int dtype, const void* x, const void* Wqkv, const void* bqkv, const void* Wo,
                          const void* bo, const void* W1, const void* b1, const void* W2, const void* b2, int b,
                          int s, int h, int heads, int ffn, int q_block, int kv_block, int causal, int wave_rows,
                          void* workspace, size_t ws_bytes, float* out, void* stream) {
  const LayerPtrs p{x, Wqkv, bqkv, Wo, bo, W1, b1, W2, b2};
  const bool caller_ws = workspace != nullptr || ws_bytes != 0;
  return layer_entry(dtype, p, b, s, h, heads, ffn, q_block, kv_block, causal, wave_rows, workspace, ws_bytes,
                     caller_ws, out, stream);
}

int bpt_layer_forward_save(const void* x, const void* Wqkv, const void* bqkv, const void* Wo, const void* bo,
                           const void* W1, const void* b1, const void* W2, const void* b2, int b, int s, int h,
                           int heads, int ffn, int q_block, int kv_block, int causal, float* out, void* o_save,
                           float* lse2_save, void* stream) {
  const LayerPtrs p{x, Wqkv, bqkv, Wo, bo, W1, b1, W2, b2};
  BPT_TRY(validate_layer(BPT_DTYPE_BF16, p, b, s, h, heads, ffn, q_block, kv_block, out));
  if ((long long)b * s == 0) return BPT_OK;
  if (!o_save || !lse2_save) return BPT_ERR_NULL;
  if (!aligned16(o_save) || !aligned16(lse2_save)) return BPT_ERR_ALIGN;
  const size_t rows = (size_t)b * s;
  const Range ro = rng(o_save, rows * h * 2), rl = rng(lse2_save, (size_t)b * heads * s * 4);
  const Range others[10] = {rng(out, rows * h * 4), rng(x, rows * h * 2), rng(Wqkv, (size_t)3 * h * h * 2),
                            rng(bqkv, (size_t)3 * h * 2), rng(Wo, (size_t)h * h * 2), rng(bo, (size_t)h * 2),
                            rng(W1, (size_t)h * ffn * 2), rng(b1, (size_t)ffn * 2), rng(W2, (size_t)ffn * h * 2),
                            rng(b2, (size_t)h * 2)};
  if (overlap(ro, rl)) return BPT_ERR_ALIAS;
  for (const Range& r : others)
    if (overlap(ro, r) || overlap(rl, r)) return BPT_ERR_ALIAS;
  return layer_entry(BPT_DTYPE_BF16, p, b, s, h, heads, ffn, q_block, kv_block, causal, BPT_WAVE_DEFAULT_WAVES,
                     nullptr, 0, false, out, stream, reinterpret_cast<__nv_bfloat16*>(o_save), lse2_save);
}

int bpt_layer_forward_noalloc(const void* x, const void* Wqkv, const void* bqkv, const void* Wo, const void* bo,
                              const void* W1, const void* b1, const void* W2, const void* b2, int b, int s, int h,
                              int heads, int q_block, int kv_block, int causal, float* out, void* stream) {
  const LayerPtrs p{x, Wqkv, bqkv, Wo, bo, W1, b1, W2, b2};
  BPT_TRY(check_shape(b, s, h, heads));
  BPT_TRY(validate_layer(BPT_DTYPE_BF16, p, b, s, h, heads, 4 * h, q_block, kv_block, out));
  if ((long long)b * s == 0) return BPT_OK;
  const Layout L = layout_for(BPT_DTYPE_BF16, b, s, h, 4 * h, q_block, 0);
  if (L.total > BPT_STATIC_WORKSPACE_BYTES) return BPT_ERR_NOMEM;
  int sms = 0;
  BPT_TRY(check_device(&sms));
  void* ws = nullptr;
  BPT_TRY(static_workspace(&ws));
  return run_layer(BPT_DTYPE_BF16, p, b, s, h, heads, 4 * h, q_block, causal, 0, reinterpret_cast<uint8_t*>(ws),
                   out, reinterpret_cast<cudaStream_t>(stream), sms);
}

int bpt_layer_forward_host(int dtype, const void* x_host, long long x_stride, const void* Wqkv, const void* bqkv,
                           const void* Wo, const void* bo, const void* W1, const void* b1, const void* W2,
                           const void* b2, int b, int s, int h, int heads, int q_block, int kv_block, int causal,
                           float* out_host, long long out_stride, int n_inputs, void* stream) {
  const LayerPtrs w{nullptr, Wqkv, bqkv, Wo, bo, W1, b1, W2, b2};
  return host_entry(dtype, x_host, x_stride, w, b, s, h, heads, q_block, kv_block, causal, out_host, out_stride,
                    n_inputs, stream);
}

int bpt_convert_f32_to_bf16(const float* src, void* dst, long long n, void* stream) {
  if (n < 0 || n > (1LL << 60)) return BPT_ERR_SHAPE;
  if (n == 0) return BPT_OK;
  if (!src || !dst) return BPT_ERR_NULL;
  if (!aligned16(src) || !aligned16(dst)) return BPT_ERR_ALIGN;
  if (overlap(rng(src, (size_t)n * 4), rng(dst, (size_t)n * 2))) return BPT_ERR_ALIAS;
  int sms = 0;
  BPT_TRY(check_device(&sms));
  return launch_convert(src, dst, n, sms, reinterpret_cast<cudaStream_t>(stream));
}

// The FFN block's backward over `rows` rows in chunks of R rows (workspace as
// bpt_ffn_backward_workspace_bytes sizes it for R). hid_bf16, when given, is
// hid already rounded to bf16 (every row, h apart), used instead of converting
// each chunk; dhid_bf16, when given, receives dhid rounded to bf16 as well.
int ffn_backward_impl(const float* hid, const void* W1, const void* b1, const void* W2, const float* dy,
                      long long rows, int h, int ffn, long long R, float* dhid, float* dW1, float* db1, float* dW2,
                      float* db2, void* workspace, int sms, cudaStream_t st, int* status,
                      const __nv_bfloat16* hid_bf16 = nullptr, __nv_bfloat16* dhid_bf16 = nullptr) {
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  __nv_bfloat16* hb = reinterpret_cast<__nv_bfloat16*>(ws);
  __nv_bfloat16* dyb = reinterpret_cast<__nv_bfloat16*>(ws + align_up((size_t)R * h * 2, 1024));
  __nv_bfloat16* U = reinterpret_cast<__nv_bfloat16*>(ws + 2 * align_up((size_t)R * h * 2, 1024));
  __nv_bfloat16* da = reinterpret_cast<__nv_bfloat16*>(ws + 2 * align_up((size_t)R * h * 2, 1024) +
                                                       align_up((size_t)R * ffn * 2, 1024));
  for (long long r0 = 0; r0 < rows; r0 += R) {
    const long long n = std::min<long long>(R, rows - r0);
    const int acc = r0 > 0 ? 1 : 0;
    const __nv_bfloat16* hbp = hid_bf16 != nullptr ? hid_bf16 + r0 * h : hb;
    if (hid_bf16 == nullptr) BPT_TRY(launch_convert(hid + r0 * h, hb, n * h, sms, st));
    BPT_TRY(launch_convert(dy + r0 * h, dyb, n * h, sms, st));
    // the chunk's FFN intermediate again (rematerialised, not stored by the forward)
    GemmArgs a{};
    a.bias = b1;
    a.dst = U;
    a.ld_dst = ffn;
    BPT_TRY((launch_gemm_t<EPI_FFN_UP, 0, 1>(hbp, h, W1, ffn, n, ffn, h, a, sms, st, status, "bwd_ffn_up")));
    // da = (dy W2^T) [U > 0]
    a = GemmArgs{};
    a.mask_u = U;
    a.ld_mask = ffn;
    a.dst = da;
    a.ld_dst = ffn;
    BPT_TRY((launch_gemm_t<EPI_BWD_DA, 0, 0>(dyb, h, W2, h, n, ffn, h, a, sms, st, status, "bwd_da")));
    // dhid = dy + da W1^T
    a = GemmArgs{};
    a.dy = dy + r0 * h;
    a.ld_dy = h;
    a.out = dhid + r0 * h;
    a.ld_out = h;
    a.dst = dhid_bf16 != nullptr ? dhid_bf16 + r0 * h : nullptr;
    a.ld_dst = h;
    BPT_TRY((launch_gemm_t<EPI_BWD_DHID, 0, 0>(da, ffn, W1, ffn, n, h, ffn, a, sms, st, status, "bwd_dhid")));
    // dW1 (+)= hid^T da and dW2 (+)= U^T dy over the chunk's rows
    a = GemmArgs{};
    a.accumulate = acc;
    a.out = dW1;
    a.ld_out = ffn;
    BPT_TRY((launch_gemm_t<EPI_GRAD, 1, 1>(hbp, h, da, ffn, h, ffn, n, a, sms, st, status, "bwd_dW1")));
    a.out = dW2;
    a.ld_out = h;
    BPT_TRY((launch_gemm_t<EPI_GRAD, 1, 1>(U, ffn, dyb, h, ffn, h, n, a, sms, st, status, "bwd_dW2")));
    BPT_TRY(launch_colsum(da, n, ffn, ffn, db1, acc, st));
    BPT_TRY(launch_colsum(dy + r0 * h, n, h, h, db2, acc, st));
  }
  return BPT_OK;
}


size_t bpt_ffn_backward_workspace_bytes(int rows, int h, int ffn, int chunk_rows) {
  if (rows <= 0 || h <= 0 || h % 64 || ffn <= 0 || ffn % 64 || chunk_rows < 0) return 0;
  const long long R = ffn_bwd_chunk(rows, chunk_rows);
  return 2 * align_up((size_t)R * h * 2, 1024) + 2 * align_up((size_t)R * ffn * 2, 1024);
}

int bpt_ffn_backward(const float* hid, const void* W1, const void* b1, const void* W2, const float* dy, int rows,
                     int h, int ffn, int chunk_rows, float* dhid, float* dW1, float* db1, float* dW2, float* db2,
                     void* workspace, size_t ws_bytes, void* stream) {
  if (rows < 0 || h <= 0 || h % 64 || ffn <= 0 || ffn % 64 || chunk_rows < 0) return BPT_ERR_SHAPE;
  if ((long long)h * ffn > 0x7fffffffLL || (long long)rows * std::max(h, ffn) > (1LL << 40)) return BPT_ERR_SHAPE;
  if (rows == 0) return BPT_OK;
  const void* ptrs[12] = {hid, W1, b1, W2, dy, dhid, dW1, db1, dW2, db2, workspace, nullptr};
  for (int i = 0; i < 11; ++i)
    if (!ptrs[i]) return BPT_ERR_NULL;
  for (int i = 0; i < 11; ++i)
    if (!aligned16(ptrs[i])) return BPT_ERR_ALIGN;
  const long long R = ffn_bwd_chunk(rows, chunk_rows);
  const size_t need = bpt_ffn_backward_workspace_bytes(rows, h, ffn, chunk_rows);
  if (ws_bytes < need) return BPT_ERR_NOMEM;
  // outputs must not overlap the inputs or one another
  const Range in[5] = {rng(hid, (size_t)rows * h * 4), rng(W1, (size_t)h * ffn * 2), rng(b1, (size_t)ffn * 2),
                       rng(W2, (size_t)ffn * h * 2), rng(dy, (size_t)rows * h * 4)};
  const Range outs[6] = {rng(dhid, (size_t)rows * h * 4), rng(dW1, (size_t)h * ffn * 4), rng(db1, (size_t)ffn * 4),
                         rng(dW2, (size_t)ffn * h * 4), rng(db2, (size_t)h * 4), rng(workspace, need)};
  for (int i = 0; i < 6; ++i) {
    for (const Range& r : in)
      if (overlap(outs[i], r)) return BPT_ERR_ALIAS;
    for (int j = i + 1; j < 6; ++j)
      if (overlap(outs[i], outs[j])) return BPT_ERR_ALIAS;
  }
  int sms = 0;
  BPT_TRY(check_device(&sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int* status = nullptr;
  BPT_TRY(stream_status_word(st, &status));
  return ffn_backward_impl(hid, W1, b1, W2, dy, rows, h, ffn, R, dhid, dW1, db1, dW2, db2, workspace, sms, st,
                           status);
}

int bpt_attention_lse(const void* q, const void* k, const void* v, int b, int s, int h, int heads, int causal,
                      void* o, float* lse2, void* stream) {
  BPT_TRY(check_shape(b, s, h, heads));
  if ((long long)b * s == 0) return BPT_OK;
  const void* ptrs[5] = {q, k, v, o, lse2};
  for (const void* p : ptrs)
    if (!p) return BPT_ERR_NULL;
  for (const void* p : ptrs)
    if (!aligned16(p)) return BPT_ERR_ALIGN;
  const size_t act = (size_t)b * s * h * 2;
  if (overlap(rng(lse2, (size_t)b * heads * s * 4), rng(o, act))) return BPT_ERR_ALIAS;
  int sms = 0;
  BPT_TRY(check_device(&sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int* status = nullptr;
  BPT_TRY(stream_status_word(st, &status));
  return launch_attention(q, h, k, v, b, s, h, heads, causal, 0, b, 0, s, reinterpret_cast<__nv_bfloat16*>(o), h,
                          st, status, lse2);
}

size_t bpt_attention_backward_workspace_bytes(int b, int s, int h, int heads) {
  if (check_shape(b, s, h, heads) != BPT_OK) return 0;
  return align_up((size_t)b * heads * s * 4, 1024) + align_up((size_t)b * s * h * 4, 1024);
}

int bpt_attention_backward(const void* q, const void* k, const void* v, const void* o, const void* dO,
                           const float* lse2, int b, int s, int h, int heads, int causal, void* dq, void* dk,
                           void* dv, void* workspace, size_t ws_bytes, void* stream) {
  BPT_TRY(check_shape(b, s, h, heads));
  if ((long long)b * s == 0) return BPT_OK;
  const void* ptrs[10] = {q, k, v, o, dO, lse2, dq, dk, dv, workspace};
  for (const void* p : ptrs)
    if (!p) return BPT_ERR_NULL;
  for (const void* p : ptrs)
    if (!aligned16(p)) return BPT_ERR_ALIGN;
  const size_t need = bpt_attention_backward_workspace_bytes(b, s, h, heads);
  if (ws_bytes < need) return BPT_ERR_NOMEM;
  const size_t act = (size_t)b * s * h * 2;
  const Range in[6] = {rng(q, act), rng(k, act), rng(v, act), rng(o, act), rng(dO, act),
                       rng(lse2, (size_t)b * heads * s * 4)};
  const Range outs[4] = {rng(dq, act), rng(dk, act), rng(dv, act), rng(workspace, need)};
  for (int i = 0; i < 4; ++i) {
    for (const Range& r : in)
      if (overlap(outs[i], r)) return BPT_ERR_ALIAS;
    for (int j = i + 1; j < 4; ++j)
      if (overlap(outs[i], outs[j])) return BPT_ERR_ALIAS;
  }
  int sms = 0;
  BPT_TRY(check_device(&sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int* status = nullptr;
  BPT_TRY(stream_status_word(st, &status));
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  float* dsum = reinterpret_cast<float*>(ws);
  float* dq32 = reinterpret_cast<float*>(ws + align_up((size_t)b * heads * s * 4, 1024));
  const long long rows = (long long)b * s;
  if (cudaMemsetAsync(dq32, 0, (size_t)rows * h * 4, st) != cudaSuccess) return BPT_ERR_CUDA;
  BPT_TRY(launch_dsum(o, dO, h, rows, s, heads, h / heads, dsum, st));
  BPT_TRY(launch_attention_bwd(q, k, v, h, dO, h, lse2, dsum, dq32, reinterpret_cast<__nv_bfloat16*>(dk),
                               reinterpret_cast<__nv_bfloat16*>(dv), h, b, s, h, heads, causal, st, status));
  return launch_rows_to_bf16(dq32, rows, h, dq, h, sms, st);
}

// Workspace of the layer backward: the recomputed forward (Q, K, V, O, the
// log-sum-exp, hid and its bf16 copy), the gradients on the way (dhid and its
// bf16 copy, dO, D, the fp32 dQ accumulator, [dQ | dK | dV]) and the FFN
// backward's chunk buffers.
struct LayerBwdLayout {
  size_t q, k, v, o, lse, hid, hb, dhid, dhb, dO, dsum, dq32, dqkv, ffn, total;
  long long R;
};

LayerBwdLayout layer_bwd_layout(int b, int s, int h, int heads, int ffn) {
  LayerBwdLayout L{};
  const size_t rows = (size_t)b * s;
  const size_t act = align_up(rows * h * 2, 1024), act32 = align_up(rows * h * 4, 1024);
  const size_t stat = align_up((size_t)b * heads * s * 4, 1024);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += bytes;
    return o;
  };
  L.q = take(act);
  L.k = take(act);
  L.v = take(act);
  L.o = take(act);
  L.lse = take(stat);
  L.hid = take(act32);  // later the fp32 dQ accumulator (hid is dead once dhid is known)
  L.dq32 = L.hid;
  L.hb = take(act);
  L.dhid = take(act32);
  L.dhb = take(act);
  L.dO = take(act);
  L.dsum = take(stat);
  L.dqkv = take(align_up(rows * 3 * h * 2, 1024));
  L.R = ffn_bwd_chunk((int)std::min<size_t>(rows, 0x7fffffff), 0);
  L.ffn = take(bpt_ffn_backward_workspace_bytes((int)std::min<size_t>(rows, 0x7fffffff), h, ffn, 0));
  L.total = off;
  return L;
}

size_t bpt_layer_backward_workspace_bytes(int b, int s, int h, int heads, int ffn) {
  if (check_shape(b, s, h, heads) != BPT_OK || ffn <= 0 || ffn % 64 || (long long)b * s == 0) return 0;
  return layer_bwd_layout(b, s, h, heads, ffn).total;
}

// The layer backward; with o_saved and lse2_saved (the forward's O and per-row
// log-sum-exp, bpt_layer_forward_save) the attention is not recomputed.
static int layer_backward_impl(const void* x, const void* Wqkv, const void* bqkv, const void* Wo,
                               const void* bo, const void* W1, const void* b1, const void* W2, const void* b2,
                               const float* dy, int b, int s, int h, int heads, int ffn, int causal, float* dx,
                               float* dWqkv, float* dbqkv, float* dWo, float* dbo, float* dW1, float* db1, float* dW2,
                               float* db2, void* workspace, size_t ws_bytes, void* stream, const void* o_saved,
                               const float* lse2_saved) {
  BPT_TRY(check_shape(b, s, h, heads));
  if (ffn <= 0 || ffn % 64 || (long long)h * ffn > 0x7fffffffLL) return BPT_ERR_SHAPE;
  if ((long long)b * s == 0) return BPT_OK;
  const void* ptrs[20] = {x, Wqkv, bqkv, Wo, bo, W1, b1, W2, b2, dy, dx, dWqkv, dbqkv, dWo, dbo, dW1, db1, dW2, db2,
                          workspace};
  for (const void* p : ptrs)
    if (!p) return BPT_ERR_NULL;
  for (const void* p : ptrs)
    if (!aligned16(p)) return BPT_ERR_ALIGN;
  const LayerBwdLayout L = layer_bwd_layout(b, s, h, heads, ffn);
  if (ws_bytes < L.total) return BPT_ERR_NOMEM;
  const long long rows = (long long)b * s;
  const bool saved = o_saved != nullptr;
  if (saved != (lse2_saved != nullptr)) return BPT_ERR_NULL;
  if (saved && (!aligned16(o_saved) || !aligned16(lse2_saved))) return BPT_ERR_ALIGN;
  // (without saved inputs the two extra ranges are empty)
  const Range in[12] = {rng(x, (size_t)rows * h * 2),     rng(Wqkv, (size_t)h * 3 * h * 2), rng(bqkv, (size_t)3 * h * 2),
                        rng(Wo, (size_t)h * h * 2),       rng(bo, (size_t)h * 2),           rng(W1, (size_t)h * ffn * 2),
                        rng(b1, (size_t)ffn * 2),         rng(W2, (size_t)ffn * h * 2),     rng(b2, (size_t)h * 2),
                        rng(dy, (size_t)rows * h * 4),
                        rng(o_saved, saved ? (size_t)rows * h * 2 : 0),
                        rng(lse2_saved, saved ? (size_t)b * heads * s * 4 : 0)};
  const Range outs[10] = {rng(dx, (size_t)rows * h * 4), rng(dWqkv, (size_t)h * 3 * h * 4), rng(dbqkv, (size_t)3 * h * 4),
                          rng(dWo, (size_t)h * h * 4),   rng(dbo, (size_t)h * 4),           rng(dW1, (size_t)h * ffn * 4),
                          rng(db1, (size_t)ffn * 4),     rng(dW2, (size_t)ffn * h * 4),     rng(db2, (size_t)h * 4),
                          rng(workspace, L.total)};
  for (int i = 0; i < 10; ++i) {
    for (const Range& r : in)
      if (overlap(outs[i], r)) return BPT_ERR_ALIAS;
    for (int j = i + 1; j < 10; ++j)
      if (overlap(outs[i], outs[j])) return BPT_ERR_ALIAS;
  }
  int sms = 0;
  BPT_TRY(check_device(&sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int* status = nullptr;
  BPT_TRY(stream_status_word(st, &status));
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  auto bf = [&](size_t off) { return reinterpret_cast<__nv_bfloat16*>(ws + off); };
  auto f32 = [&](size_t off) { return reinterpret_cast<float*>(ws + off); };
  const int dh = h / heads;

  // the forward again (rematerialised): Q, K, V; O and each row's log-sum-exp (or the
  // forward's own, saved); hid
  const __nv_bfloat16* Osrc = saved ? reinterpret_cast<const __nv_bfloat16*>(o_saved) : bf(L.o);
  const float* lse = saved ? lse2_saved : f32(L.lse);
  {
    GemmArgs a{};
    a.bias = bqkv;
    a.q = bf(L.q);
    a.ldq = h;
    a.k = bf(L.k);
    a.v = bf(L.v);
    a.ldkv = h;
    a.h = h;
    BPT_TRY(launch_gemm<EPI_QKV>(x, rows, h, h, Wqkv, 3LL * h, a, sms, st, status, "bwd_qkv"));
  }
  if (!saved)
    BPT_TRY(launch_attention(bf(L.q), h, bf(L.k), bf(L.v), b, s, h, heads, causal, 0, b, 0, s, bf(L.o), h, st,
                             status, f32(L.lse)));
  {
    GemmArgs a{};
    a.resid = x;
    a.ld_resid = h;
    a.hid = f32(L.hid);
    a.ld_hid = h;
    a.bias = bo;
    a.dst = bf(L.hb);
    a.ld_dst = h;
    BPT_TRY(launch_gemm<EPI_OUTPROJ>(Osrc, rows, h, h, Wo, h, a, sms, st, status, "bwd_outproj"));
  }
  // FFN block: dhid, dW1, db1, dW2, db2
  // (hid's bf16 copy is the out-projection's; dhid's bf16 copy comes from the dhid product's epilogue)
  BPT_TRY(ffn_backward_impl(f32(L.hid), W1, b1, W2, dy, rows, h, ffn, L.R, f32(L.dhid), dW1, db1, dW2, db2,
                            ws + L.ffn, sms, st, status, bf(L.hb), bf(L.dhb)));
  // out-projection: dbo = sum dhid, dWo = O^T dhid, dO = dhid Wo^T
  BPT_TRY(launch_colsum(f32(L.dhid), rows, h, h, dbo, 0, st));
  {
    GemmArgs a{};
    a.out = dWo;
    a.ld_out = h;
    BPT_TRY((launch_gemm_t<EPI_GRAD, 1, 1>(Osrc, h, bf(L.dhb), h, h, h, rows, a, sms, st, status, "bwd_dWo")));
    a = GemmArgs{};
    a.dst = bf(L.dO);
    a.ld_dst = h;
    BPT_TRY((launch_gemm_t<EPI_BWD_DA, 0, 0>(bf(L.dhb), h, Wo, h, rows, h, h, a, sms, st, status, "bwd_dO")));
  }
  // attention: dQ, dK, dV into [dQ | dK | dV]
  float* dq32 = f32(L.dq32);
  __nv_bfloat16* dqkv = bf(L.dqkv);
  if (cudaMemsetAsync(dq32, 0, (size_t)rows * h * 4, st) != cudaSuccess) return BPT_ERR_CUDA;
  BPT_TRY(launch_dsum(Osrc, bf(L.dO), h, rows, s, heads, dh, f32(L.dsum), st));
  BPT_TRY(launch_attention_bwd(bf(L.q), bf(L.k), bf(L.v), h, bf(L.dO), h, lse, f32(L.dsum), dq32, dqkv + h,
                               dqkv + 2 * h, 3LL * h, b, s, h, heads, causal, st, status));
  BPT_TRY(launch_rows_to_bf16(dq32, rows, h, dqkv, 3LL * h, sms, st));
  // projection: dbqkv = sum dqkv, dWqkv = x^T dqkv, dx = dhid + dqkv Wqkv^T
  BPT_TRY(launch_colsum(dqkv, rows, 3 * h, 3LL * h, dbqkv, 0, st));
  {
    GemmArgs a{};
    a.out = dWqkv;
    a.ld_out = 3LL * h;
    BPT_TRY((launch_gemm_t<EPI_GRAD, 1, 1>(x, h, dqkv, 3LL * h, h, 3LL * h, rows, a, sms, st, status, "bwd_dWqkv")));
    a = GemmArgs{};
    a.dy = f32(L.dhid);
    a.ld_dy = h;
    a.out = dx;
    a.ld_out = h;
    BPT_TRY((launch_gemm_t<EPI_BWD_DHID, 0, 0>(dqkv, 3LL * h, Wqkv, 3LL * h, rows, h, 3LL * h, a, sms, st, status,
                                               "bwd_dx")));
  }
  return BPT_OK;
}

int bpt_layer_backward(const void* x, const void* Wqkv, const void* bqkv, const void* Wo, const void* bo,
                       const void* W1, const void* b1, const void* W2, const void* b2, const float* dy, int b, int s,
                       int h, int heads, int ffn, int causal, float* dx, float* dWqkv, float* dbqkv, float* dWo,
                       float* dbo, float* dW1, float* db1, float* dW2, float* db2, void* workspace,
                       size_t ws_bytes, void* stream) {
  return layer_backward_impl(x, Wqkv, bqkv, Wo, bo, W1, b1, W2, b2, dy, b, s, h, heads, ffn, causal, dx, dWqkv, dbqkv,
                             dWo, dbo, dW1, db1, dW2, db2, workspace, ws_bytes, stream, nullptr, nullptr);
}

int bpt_layer_backward_saved(const void* x, const void* Wqkv, const void* bqkv, const void* Wo, const void* bo,
                             const void* W1, const void* b1, const void* W2, const void* b2, const void* o_saved,
                             const float* lse2_saved, const float* dy, int b, int s, int h, int heads, int ffn,
                             int causal, float* dx, float* dWqkv, float* dbqkv, float* dWo, float* dbo, float* dW1,
                             float* db1, float* dW2, float* db2, void* workspace, size_t ws_bytes, void* stream) {
  if ((long long)b * s > 0 && (!o_saved || !lse2_saved)) return BPT_ERR_NULL;
  return layer_backward_impl(x, Wqkv, bqkv, Wo, bo, W1, b1, W2, b2, dy, b, s, h, heads, ffn, causal, dx, dWqkv, dbqkv,
                             dWo, dbo, dW1, db1, dW2, db2, workspace, ws_bytes, stream, o_saved, lse2_saved);
}

int bpt_qkv_projection(const void* x, const void* Wqkv, const void* bqkv, int b, int s, int h, void* q, void* k,
                       void* v, void* stream) {
  if (b < 0 || s < 0 || h <= 0 || h % 64 || (long long)b * s > 0x7fffffffLL) return BPT_ERR_SHAPE;
  if ((long long)b * s == 0) return BPT_OK;
  const void* ptrs[6] = {x, Wqkv, bqkv, q, k, v};
  for (const void* p : ptrs)
    if (!p) return BPT_ERR_NULL;
  for (const void* p : ptrs)
    if (!aligned16(p)) return BPT_ERR_ALIGN;
  int sms = 0;
  BPT_TRY(check_device(&sms));
  GemmArgs a{};
  a.bias = bqkv;
  a.q = reinterpret_cast<__nv_bfloat16*>(q);
  a.ldq = h;
  a.k = reinterpret_cast<__nv_bfloat16*>(k);
  a.v = reinterpret_cast<__nv_bfloat16*>(v);
  a.ldkv = h;
  a.h = h;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int* status = nullptr;
  BPT_TRY(stream_status_word(st, &status));
  return launch_gemm<EPI_QKV>(x, (long long)b * s, h, h, Wqkv, 3LL * h, a, sms, st, status, "gemm_qkv");
}

int bpt_attention(const void* q, const void* k, const void* v, int b, int s, int h, int heads, int q_block,
                  int kv_block, int causal, void* o, void* stream) {
  BPT_TRY(check_shape(b, s, h, heads));
  BPT_TRY(check_blocks(s, q_block, kv_block));
  if ((long long)b * s == 0) return BPT_OK;
  const void* ptrs[4] = {q, k, v, o};
  for (const void* p : ptrs)
    if (!p) return BPT_ERR_NULL;
  for (const void* p : ptrs)
    if (!aligned16(p)) return BPT_ERR_ALIGN;
  int sms = 0;
  BPT_TRY(check_device(&sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int* status = nullptr;
  BPT_TRY(stream_status_word(st, &status));
  return launch_attention(q, h, k, v, b, s, h, heads, causal, 0, b, 0, s, reinterpret_cast<__nv_bfloat16*>(o), h,
                          st, status);
}

int bpt_stream_status(void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return BPT_ERR_CUDA;
  }
  if (cudaStreamSynchronize(st) != cudaSuccess) {
    cudaGetLastError();
    return BPT_ERR_CUDA;
  }
  const int idx = status_index(dev, st, false);
  if (idx < 0) return BPT_OK;  // no call of this library ever ran on the stream
  int* base = nullptr;
  BPT_TRY(status_base(&base));
  int v = 0;
  if (cudaMemcpyAsync(&v, base + idx, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess) {
    cudaGetLastError();
    return BPT_ERR_CUDA;
  }
  if (v != BPT_OK && (cudaMemsetAsync(base + idx, 0, sizeof(int), st) != cudaSuccess ||
                      cudaStreamSynchronize(st) != cudaSuccess)) {
    cudaGetLastError();
    return BPT_ERR_CUDA;
  }
  return v;
}

int bpt_device_status(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    return BPT_ERR_CUDA;
  }
  static int words[kStatusSlots];
  static std::mutex mu;
  std::lock_guard<std::mutex> lk(mu);
  if (cudaMemcpyFromSymbol(words, g_status_slots, sizeof(words)) != cudaSuccess) {
    cudaGetLastError();
    return BPT_ERR_CUDA;
  }
  int v = BPT_OK;
  for (int w : words)
    if (w != BPT_OK && v == BPT_OK) v = w;
  if (v != BPT_OK) {
    std::memset(words, 0, sizeof(words));
    if (cudaMemcpyToSymbol(g_status_slots, words, sizeof(words)) != cudaSuccess) {
      cudaGetLastError();
      return BPT_ERR_CUDA;
    }
  }
  return v;
}

int bpt_wait_flag(const int* flag, int value, int timeout_us, void* stream) {
  if (!flag) return BPT_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(flag) & 3u) != 0) return BPT_ERR_ALIGN;
  if (timeout_us < 0 || timeout_us > 10000000) return BPT_ERR_SHAPE;
  int sms = 0;
  BPT_TRY(check_device(&sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int* status = nullptr;
  BPT_TRY(stream_status_word(st, &status));
  {
    LaunchScope ls("wait_flag", st);
    wait_flag_kernel<<<1, 32, 0, st>>>(flag, value, (unsigned long long)timeout_us * 1000ull, status);
  }
  return cudaGetLastError() == cudaSuccess ? BPT_OK : BPT_ERR_CUDA;
}

uint64_t bpt_launch_count(void) { return g_launches.load(); }

int bpt_set_kernel_timing(int enable) {
  std::lock_guard<std::mutex> lk(g_timing_mu);
  g_timing = enable != 0;
  return BPT_OK;
}

int bpt_kernel_times(bpt_kernel_time* out, int max) {
  std::vector<TimedLaunch> recs;
  {
    std::lock_guard<std::mutex> lk(g_timing_mu);
    recs.swap(g_timed);
  }
  std::map<std::string, std::pair<int, double>> agg;
  std::vector<std::string> order;
  int rc = BPT_OK;
  for (auto& r : recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess)
      rc = BPT_ERR_CUDA;
    cudaEventDestroy(r.start);
    cudaEventDestroy(r.stop);
    auto it = agg.find(r.name);
    if (it == agg.end()) {
      order.push_back(r.name);
      agg[r.name] = {1, ms};
    } else {
      it->second.first += 1;
      it->second.second += ms;
    }
  }
  if (rc != BPT_OK) return rc;
  int n = 0;
  for (const auto& name : order) {
    if (n >= max || !out) break;
    std::memset(out[n].name, 0, sizeof(out[n].name));
    std::strncpy(out[n].name, name.c_str(), sizeof(out[n].name) - 1);
    out[n].launches = agg[name].first;
    out[n].total_ms = agg[name].second;
    ++n;
  }
  return n;
}

}  // extern "C"
