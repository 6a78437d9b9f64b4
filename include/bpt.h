/*
 * bpt.h - C ABI of the B200 (sm_100a) Blockwise Parallel Transformer layer forward.
 *
 * One call computes, for every query block Q_i of the sequence, exact
 * multi-head attention over all key/value blocks with a running max and
 * running sum (online-softmax rescaling), then the output projection, the
 * first residual, the position-wise FFN max(0, y W1 + b1) W2 + b2 and the
 * second residual:
 *
 *     [Q | K | V] = x Wqkv + bqkv
 *     O_i         = concat_k softmax(Q_i,k K_k^T / sqrt(dh)) V_k      (per head k)
 *     hid_i       = x_i + O_i Wo + bo
 *     out_i       = hid_i + max(0, hid_i W1 + b1) W2 + b2
 *
 * Sources: "Blockwise Parallel Transformer for Large Context Models" (paper
 * review of arXiv:2305.19370), section 3: core formulas (standard attention,
 * standard FFN, Eq. 3 blockwise attention and its scaling operation, the
 * blockwise FFN with residuals) and Algorithm 1 (input sequence x, query block
 * count B_q, key/value block count B_kv). Head split and concatenation follow
 * "PyTorch 2.3 multi-head self-attention from QKV to 8 heads", sections 2-4;
 * the fused QKV projection follows "Transformer QKV matrix computation and 3
 * parallel strategies", section 2.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - All tensor pointers are CUDA device pointers owned by the caller unless a
 *   function says otherwise. The library keeps no pointer after a call returns
 *   (work it queued on the stream still reads them until it completes).
 * - Layouts are row-major. x and out are [b, s, h] (token-major). Weights are
 *   [in, out] so that a projection reads x W: Wqkv [h, 3h] with columns
 *   [W_Q | W_K | W_V] and head k of each third in columns k*dh .. k*dh+dh-1;
 *   Wo [h, h]; W1 [h, 4h]; W2 [4h, h]. Biases are vectors of the output width.
 * - bf16 entry points take bf16 x, weights and biases. The f32 entry points
 *   take fp32 x, weights and biases; their matrix products round operands to
 *   bf16 (fp32 accumulation) while the residual and bias additions use the
 *   fp32 values.
 * - out is fp32 [b, s, h]. It is written entirely and is also used as scratch
 *   during the call (it must not overlap any input).
 * - Shapes: b >= 0, s >= 0 (b*s == 0 is a no-op), h = heads * dh with
 *   dh in {64, 128}, b*s <= 2^31 - 1. The FFN width is fixed at 4h.
 * - Blocks: 1 <= q_block <= s, 1 <= kv_block <= s, s % q_block == 0,
 *   s % kv_block == 0 (equal-length blocks). The result does not depend on the
 *   block sizes (the blockwise computation is exact). The kernels tile by the
 *   hardware instead: attention by 128 query rows x 128 keys, the FFN side by
 *   waves of whole query blocks (or, on request, by groups of 128-row tiles
 *   that all run in one launch: BPT_WAVE_CHAINED).
 * - causal != 0: key u is visible to query t iff u <= t in the same sequence.
 * - Pointers must be 16-byte aligned (tensor-memory-access tiles).
 * - Errors: argument errors return a negative bpt_status synchronously, with
 *   nothing launched and nothing written. Otherwise the call is asynchronous on
 *   `stream` (a cudaStream_t; NULL means the legacy default stream) and
 *   returns BPT_OK once all kernels are queued. Device-side failures (a
 *   bounded wait that gave up) are recorded in a status word owned by the
 *   stream the kernels ran on, and bpt_stream_status(stream) reports them.
 * - Reentrancy: calls on different streams may run concurrently; each stream
 *   has its own device status word. The other process-wide state is the
 *   launch counter and the optional kernel timing log.
 */
#ifndef BPT_H_
#define BPT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum bpt_status {
  BPT_OK = 0,
  BPT_ERR_NULL = -1,        /* a required pointer is NULL */
  BPT_ERR_SHAPE = -2,       /* b, s, h, heads out of range; h % heads; dh not 64 or 128 */
  BPT_ERR_BLOCK = -3,       /* q_block / kv_block <= 0, > s, or not dividing s */
  BPT_ERR_ALIGN = -4,       /* a pointer is not 16-byte aligned */
  BPT_ERR_ALIAS = -5,       /* out overlaps an input, or workspace overlaps out or an input */
  BPT_ERR_NOMEM = -6,       /* workspace allocation failed, or ws_bytes too small */
  BPT_ERR_CUDA = -7,        /* a CUDA runtime / driver call failed */
  BPT_ERR_TIMEOUT = -8,     /* a kernel gave up a bounded wait (device-side) */
  BPT_ERR_UNSUPPORTED = -9, /* the current device is not sm_100 */
  BPT_ERR_DTYPE = -10       /* unknown dtype code */
} bpt_status;

typedef enum bpt_dtype {
  BPT_DTYPE_BF16 = 0,
  BPT_DTYPE_F32 = 1
} bpt_dtype;

/* Schedules of the FFN side (the wave_rows argument of the _ws and _ffn entry
 * points and of bpt_layer_workspace_bytes(_ffn)); any positive value is an
 * explicit wave of that many rows, one launch per GEMM and wave. */
#define BPT_WAVE_DEFAULT 0         /* the library's choice (per-GEMM waves) */
#define BPT_WAVE_CHAINED (-1)      /* every query block's FFN side in one launch (bf16 inputs) */
#define BPT_WAVE_DEFAULT_WAVES (-2) /* one launch per GEMM and wave, waves of the library's default size */
#define BPT_WAVE_MEGA (-3)         /* attention and the FFN side in one persistent launch (bf16, s % 128 == 0;
                                      otherwise as BPT_WAVE_CHAINED, or per wave for fp32 inputs) */

/* Human-readable name of a status code (static string, never NULL). A library
 * utility; the pages have no counterpart. */
const char* bpt_status_string(int status);

/* ------------------------------------------------------------------------
 * The layer forward (Algorithm 1 of the BPT paper review, section 3).
 * ------------------------------------------------------------------------ */

/* The layer as the pages define it: Algorithm 1 steps 1-12 with Eq. 3 and its
 * scaling operation for the attention and the blockwise FFN-with-residuals
 * formula (paper review section 3), bf16 matmul inputs with fp32
 * accumulation (paper review section 5, precision).
 *
 * bf16 inputs. Allocates its workspace stream-ordered on `stream` from a
 * library-owned memory pool of the current device and frees it stream-ordered
 * after the last kernel; the pool keeps freed memory for later calls (so
 * repeated calls do not map device memory again). Returns BPT_ERR_NOMEM if the
 * allocation fails. */
int bpt_layer_forward(const void* x, const void* Wqkv, const void* bqkv, const void* Wo, const void* bo,
                      const void* W1, const void* b1, const void* W2, const void* b2, int b, int s, int h,
                      int heads, int q_block, int kv_block, int causal, float* out, void* stream);

/* The same layer (Algorithm 1, paper review section 3) for fp32 inputs; the
 * small fp32 workload of the test suite uses it. The pages fix bf16 matmul
 * inputs with fp32 accumulation (section 5); this entry keeps more of the fp32
 * inputs' precision than a plain bf16 rounding would.
 *
 * fp32 inputs (same arguments, fp32 tensors). The GEMMs keep about 16
 * significant bits of x and of the weights: each fp32 value v is split on the
 * device into bf16 parts hi = bf16(v) and lo = bf16(v - hi), and the products
 * x W_hi + x W_lo (projection: x_hi W_hi + x_hi W_lo + x_lo W_hi) accumulate in
 * fp32. Attention and the FFN activations are bf16 as in the bf16 entry. */
int bpt_layer_forward_f32(const float* x, const float* Wqkv, const float* bqkv, const float* Wo, const float* bo,
                          const float* W1, const float* b1, const float* W2, const float* b2, int b, int s, int h,
                          int heads, int q_block, int kv_block, int causal, float* out, void* stream);

/* Workspace of one layer call. The pages' memory analysis (paper review
 * section 3, "memory analysis": 2bsh of activations per layer, FFN scratch
 * per chunk of c rows, never per sequence) is what it is sized against.
 * Departure from the plain (b, s, h, heads, q_block, kv_block) signature:
 * dtype selects the element type of the inputs and wave_rows the FFN chunk.
 *
 * Bytes of workspace a caller must pass to bpt_layer_forward_ws for these
 * arguments (0 if they are invalid or b*s == 0): one region that holds the bf16
 * K and V of the whole input (2 * b*s*h * 2 bytes) until attention is done and
 * then the FFN scratch, so its size is the larger of the two, plus a few KiB.
 * wave_rows = BPT_WAVE_CHAINED with bf16 inputs runs the FFN side of every
 * query block in one launch over groups of 128-row tiles: the scratch is 3
 * slots of a group's fp32 residual stream and its bf16 copy and 2 slots of
 * its FFN intermediate (ffn wide, bf16), with the largest group of 16, 8, 4,
 * 2 or 1 tiles whose slots take at most 1.5x the K/V bytes (or 32 MiB); at
 * b=1, s=32768, h=4096 that is 2048-row groups inside the K/V region, 512 MiB
 * in all (1.0x 2bsh read as elements). BPT_WAVE_DEFAULT (the library's
 * choice: per-GEMM waves, which measured as fast as the chained launch at
 * the large workloads and faster at the small ones), BPT_WAVE_DEFAULT_WAVES,
 * wave_rows > 0 and fp32 inputs run one launch per GEMM and FFN wave: the
 * scratch is one
 * wave's (14 * h bytes per wave row: fp32 residual stream, its bf16 copy and
 * the 4h-wide bf16 intermediate); wave_rows is rounded down to a multiple of
 * q_block (at least q_block), and a value of s or more groups whole
 * sequences; otherwise the library picks the whole number of query
 * blocks (or of whole sequences) that its model of its GEMM tile
 * rounds finds fastest, with scratch of at most 1.5x the K/V bytes (or of
 * about 4096 rows). BPT_WAVE_MEGA (bf16 inputs, s a multiple of 128) runs
 * attention and the chained FFN side in one persistent launch whose
 * out-projection tiles wait (bounded) for their rows' attention output; the
 * chain's slots then follow the K/V region instead of aliasing it (K and V are
 * still read while the FFN side of earlier rows runs). The fp32 entry adds
 * bf16 copies of x and the weights. */
size_t bpt_layer_workspace_bytes(int dtype, int b, int s, int h, int heads, int q_block, int kv_block,
                                 int wave_rows);

/* The standard FFN max(0, x W1 + b1) W2 + b2 (paper review section 3, core
 * formulas) has a hidden width the formula leaves open; the memory analysis'
 * 8bch activation input implies 4h, which every other entry point uses.
 *
 * The layer with an FFN of any width ffn (the pages fix ffn = 4h; every
 * other entry point uses 4h): W1 is [h, ffn], b1 [ffn], W2 [ffn, h], in the
 * element type dtype. ffn must be a positive multiple of 64 (BPT_ERR_SHAPE
 * otherwise). workspace == NULL with ws_bytes == 0 takes the workspace from
 * the library's stream-ordered pool, as bpt_layer_forward does; otherwise it
 * is caller-owned with the rules of bpt_layer_forward_ws and must hold
 * bpt_layer_workspace_bytes_ffn(...) bytes. All other arguments, the result
 * and the error behaviour are those of bpt_layer_forward_ws. */
size_t bpt_layer_workspace_bytes_ffn(int dtype, int b, int s, int h, int heads, int ffn, int q_block, int kv_block,
                                     int wave_rows);
int bpt_layer_forward_ffn(int dtype, const void* x, const void* Wqkv, const void* bqkv, const void* Wo,
                          const void* bo, const void* W1, const void* b1, const void* W2, const void* b2, int b,
                          int s, int h, int heads, int ffn, int q_block, int kv_block, int causal, int wave_rows,
                          void* workspace, size_t ws_bytes, float* out, void* stream);

/* Algorithm 1 (paper review section 3) with the caller's workspace; same
 * departure as bpt_layer_workspace_bytes (dtype, wave_rows).
 *
 * The layer with a caller-owned workspace (device memory, 256-byte aligned,
 * at least bpt_layer_workspace_bytes(...) bytes, not overlapping any argument;
 * BPT_ERR_NOMEM if ws_bytes is too small). dtype is a bpt_dtype and gives the
 * element type of x, the weights and the biases. Allocates nothing. */
int bpt_layer_forward_ws(int dtype, const void* x, const void* Wqkv, const void* bqkv, const void* Wo,
                         const void* bo, const void* W1, const void* b1, const void* W2, const void* b2, int b,
                         int s, int h, int heads, int q_block, int kv_block, int causal, int wave_rows,
                         void* workspace, size_t ws_bytes, float* out, void* stream);

/* Algorithm 1 (paper review section 3) from its input sequence x in host
 * memory to the layer's output in host memory; the copy pipeline has no
 * counterpart in the pages.
 *
 * End to end from host memory: for i in [0, n_inputs), out_host + i *
 * out_stride receives the layer applied to x_host + i * x_stride (strides in
 * bytes; 0 reuses the same input, or writes every result to the same place).
 * x is [b, s, h] of dtype (bf16 or fp32) in host memory; out is fp32 [b, s, h]
 * in host memory; the weights and biases are device pointers as for
 * bpt_layer_forward. Host buffers should be pinned (page-locked) for the
 * copies to overlap the compute; pageable memory works, slower. Input i is
 * copied in while input i - 1 computes and its result copied out while input
 * i + 1 computes (two device buffers each for x and out and one workspace,
 * from the library's pool; four internal copy streams, two each way, that
 * move every input and every result in two halves, ordered by events
 * against `stream`, which runs the layer). The first bf16 input arrives in
 * four row chunks, each projected when the rows it holds are needed. With
 * causal attention (a row needs only the keys at or before it) the first and
 * the last input run wave by wave: the attention of an FFN wave's rows, then
 * that wave's FFN side, whose scratch then lies beside the K/V copies instead
 * of over them (one wave's, 14 h bytes a row, more device memory), so that the
 * first input's compute starts with its first chunk and the last input's
 * results start to come out early in the layer. Each wave's rows are copied out as soon as
 * the wave is done, and the last input's last wave runs in two halves so that
 * only the second half's copy follows the last launch. None of this changes a
 * result: every row is computed as in bpt_layer_forward, bit for bit. Returns after every result has reached host memory. Errors as
 * bpt_layer_forward; BPT_ERR_SHAPE also for
 * n_inputs < 0 or a nonzero stride smaller than one input (output); and
 * BPT_ERR_ALIAS if the input and output host ranges overlap. */
int bpt_layer_forward_host(int dtype, const void* x_host, long long x_stride, const void* Wqkv, const void* bqkv,
                           const void* Wo, const void* bo, const void* W1, const void* b1, const void* W2,
                           const void* b2, int b, int s, int h, int heads, int q_block, int kv_block, int causal,
                           float* out_host, long long out_stride, int n_inputs, void* stream);

/* Between the layers of a stack (the pages' models are stacks of BPT layers:
 * paper review section 6, 1B-70B models) the fp32 output becomes the next
 * layer's bf16 input, the matmul input precision of section 5.
 *
 * dst[i] = src[i] rounded to bf16 (nearest, ties to even), i < n; device
 * pointers, 16-byte aligned, not overlapping; asynchronous on `stream`.
 * Chains layers: one layer's fp32 out becomes the next layer's bf16 x (a
 * stack of BPT layers, as the pages' models are). Errors: BPT_ERR_SHAPE for
 * n < 0, BPT_ERR_NULL, BPT_ERR_ALIGN, BPT_ERR_ALIAS; nothing launched then. */
int bpt_convert_f32_to_bf16(const float* src, void* dst, long long n, void* stream);

/* Allocation-free variant of bpt_layer_forward (bf16 inputs, same arguments
 * and result). The paper has no counterpart: this entry point exists for
 * callers that cannot call cudaMalloc (or any allocator) while they run, for
 * example code executing inside an inference engine's enqueue/execute hook
 * where allocating is forbidden, or a process whose device memory is reserved
 * up front by another memory manager, and that also cannot lend the library a
 * workspace buffer. Its scratch is one fixed array of
 * BPT_STATIC_WORKSPACE_BYTES in the library's device memory: every GPU on
 * which the library is loaded holds that array until the process exits.
 *
 * - Allocates nothing: no cudaMalloc / cudaMallocAsync / cudaFree, and no
 *   allocating library routine (nor host heap memory). The caller still owns
 *   x, the weights, the biases and out.
 * - Size limit: returns BPT_ERR_NOMEM, with nothing launched, when the
 *   workspace the layer needs (bpt_layer_workspace_bytes(BPT_DTYPE_BF16, b, s,
 *   h, heads, q_block, kv_block, 0)) exceeds BPT_STATIC_WORKSPACE_BYTES; for
 *   example b=1, s=2048, h=1024 needs 28 MiB and fits, s=8192, h=2048 does not.
 * - Every call looks up the current device's address of the array (one
 *   cudaGetSymbolAddress with that device current, which allocates nothing),
 *   so the address is right even after cudaDeviceReset has recreated the
 *   library's device image. The first call of this library on a device also
 *   loads that image there; make it before any stream capture on the device.
 * - Every call on a device uses the same array, and it keeps whatever the last
 *   call left in it. No part of it needs to start at zero: each byte a call
 *   reads was written earlier in the same call. Calls whose work overlaps on
 *   the GPU (different streams, or different host threads, without ordering
 *   between them) race on the array and corrupt each other's results; order
 *   them on one stream or with events. */
#define BPT_STATIC_WORKSPACE_BYTES ((size_t)64 << 20)

int bpt_layer_forward_noalloc(const void* x, const void* Wqkv, const void* bqkv, const void* Wo, const void* bo,
                              const void* W1, const void* b1, const void* W2, const void* b2, int b, int s, int h,
                              int heads, int q_block, int kv_block, int causal, float* out, void* stream);

/* ------------------------------------------------------------------------
 * Single steps of Algorithm 1, for checking intermediate results.
 * ------------------------------------------------------------------------ */

/* Algorithm 1 step 1 (paper review section 3), with the fused projection of
 * "Transformer QKV matrix computation and 3 parallel strategies", section 2.
 *
 * Step 1: [Q | K | V] = x Wqkv + bqkv with bf16 x [b*s, h], Wqkv [h, 3h],
 * bqkv [3h]; writes bf16 q, k, v, each [b*s, h] row-major. */
int bpt_qkv_projection(const void* x, const void* Wqkv, const void* bqkv, int b, int s, int h, void* q, void* k,
                       void* v, void* stream);

/* Algorithm 1 steps 2-10 with Eq. 3 and its scaling operation (paper review
 * section 3); heads split and concatenated as in "PyTorch 2.3 multi-head
 * self-attention from QKV to 8 heads", sections 2-4.
 *
 * Steps 2-10: O = concat_k softmax(Q_k K_k^T / sqrt(dh)) V_k over all key
 * blocks with online-softmax rescaling; bf16 q, k, v [b, s, h] in, bf16 o
 * [b, s, h] out. q_block / kv_block are validated as for the layer. */
int bpt_attention(const void* q, const void* k, const void* v, int b, int s, int h, int heads, int q_block,
                  int kv_block, int causal, void* o, void* stream);

/* ------------------------------------------------------------------------
 * Backward of the FFN block (part of the layer's backward pass).
 * ------------------------------------------------------------------------ */

/* Gradients of the FFN block with its residual, out = hid + max(0, hid W1 +
 * b1) W2 + b2 (paper review section 3: the standard FFN and the second
 * residual of the blockwise FFN formula), for the upstream gradient dy =
 * dL/dout. The pages train with this layer and rematerialise the blockwise
 * FFN in the backward pass (the scanned blockwise FFN of section 3): the
 * intermediate max(0, hid W1 + b1) is recomputed here, chunk by chunk of
 * rows, never stored for the whole sequence.
 *
 *     u = max(0, hid W1 + b1)       (recomputed per chunk)
 *     da = (dy W2^T) * [u > 0]
 *     dhid = dy + da W1^T           dW1 = hid^T da    db1 = sum_rows da
 *     dW2 = u^T dy                  db2 = sum_rows dy
 *
 * hid, dy: fp32 [rows, h] device memory; W1 [h, ffn], b1 [ffn], W2 [ffn, h]
 * bf16 (the layer's weights). Outputs, fp32, written entirely (not
 * accumulated into): dhid [rows, h], dW1 [h, ffn], db1 [ffn], dW2 [ffn, h],
 * db2 [h]. The matrix products take bf16 operands (hid and dy rounded to
 * nearest even) with fp32 accumulation; the weight gradients sum the chunks
 * in fp32. chunk_rows: rows per chunk, rounded down to a multiple of 128 (0 =
 * 16384). workspace: device memory of at least
 * bpt_ffn_backward_workspace_bytes(...) bytes (bf16 copies of a chunk's hid
 * and dy, its recomputed intermediate and da). h and ffn must be multiples of
 * 64. Errors: BPT_ERR_SHAPE, BPT_ERR_NULL, BPT_ERR_ALIGN (16 bytes),
 * BPT_ERR_NOMEM (workspace too small), BPT_ERR_ALIAS (an output or the
 * workspace overlaps an input or another output); nothing launched then.
 * Asynchronous on `stream`; device-side failures through
 * bpt_stream_status. */
size_t bpt_ffn_backward_workspace_bytes(int rows, int h, int ffn, int chunk_rows);
int bpt_ffn_backward(const float* hid, const void* W1, const void* b1, const void* W2, const float* dy, int rows,
                     int h, int ffn, int chunk_rows, float* dhid, float* dW1, float* db1, float* dW2, float* db2,
                     void* workspace, size_t ws_bytes, void* stream);

/* Attention forward (as bpt_attention) that also writes each row's
 * log-sum-exp of the scaled scores, the statistic the backward recomputes the
 * attention weights from (Algorithm 1 records each query block's
 * normalisation statistics, step 10; the backward of the paper review's
 * section 3 rematerialises the blockwise computation from them).
 * lse2: fp32 [b, heads, s] device memory, lse2[(beta * heads + k) * s + t] =
 * log2(sum_u exp2(c S_tu)) for head k, with c = log2(e) / sqrt(dh) and S the
 * scores Q K^T (masked keys left out); it must not overlap o. Other arguments,
 * errors and stream semantics as for bpt_attention (no block sizes: the
 * result does not depend on them). */
int bpt_attention_lse(const void* q, const void* k, const void* v, int b, int s, int h, int heads, int causal,
                      void* o, float* lse2, void* stream);

/* ------------------------------------------------------------------------
 * Backward of the attention and of the whole layer.
 * ------------------------------------------------------------------------ */

/* Gradients of O = softmax(Q K^T / sqrt(dh)) V per head (Eq. 3 and Algorithm 1
 * steps 4-10 of the paper review, inverted blockwise as its section 3
 * rematerialises the blockwise computation for training): for dO = dL/dO,
 *
 *     P = 2^(c S - lse2) (0 where masked),  D = rowsum(dO O)
 *     dV = P^T dO,  dS = P (dO V^T - D),  dQ = dS K / sqrt(dh),  dK = dS^T Q / sqrt(dh)
 *
 * computed per key/value tile of 128 keys over the query tiles that see it,
 * with P recomputed from lse2 (from bpt_attention_lse) and never stored.
 * q, k, v, o, dO: bf16 [b, s, h] device memory (o the forward's output);
 * lse2 fp32 [b, heads, s]. Outputs dq, dk, dv: bf16 [b, s, h], written
 * entirely. P and dS enter the products as bf16; dQ is summed over the key
 * tiles in fp32. workspace: at least bpt_attention_backward_workspace_bytes
 * bytes of device memory (D and the fp32 dQ sums). Errors: BPT_ERR_SHAPE
 * (dh not 64 or 128, ...), BPT_ERR_NULL, BPT_ERR_ALIGN (16 bytes),
 * BPT_ERR_NOMEM, BPT_ERR_ALIAS (an output or the workspace overlaps an input
 * or another output); nothing launched then. Asynchronous on `stream`;
 * device-side failures through bpt_stream_status. */
size_t bpt_attention_backward_workspace_bytes(int b, int s, int h, int heads);
int bpt_attention_backward(const void* q, const void* k, const void* v, const void* o, const void* dO,
                           const float* lse2, int b, int s, int h, int heads, int causal, void* dq, void* dk,
                           void* dv, void* workspace, size_t ws_bytes, void* stream);

/* Gradients of one BPT layer's output with respect to its input and every
 * parameter (the layer of bpt_layer_forward_ffn, FFN width ffn), for the
 * upstream gradient dy = dL/dout: the chain rule through the forward of
 * Algorithm 1 and Eq. 3 of the paper review,
 *
 *     qkv = x Wqkv + bqkv;  O = attention(Q, K, V);  hid = x + O Wo + bo
 *     out = hid + max(0, hid W1 + b1) W2 + b2
 *     FFN block as bpt_ffn_backward -> dhid, dW1, db1, dW2, db2
 *     dbo = sum dhid;  dWo = O^T dhid;  dO = dhid Wo^T
 *     attention as bpt_attention_backward -> dQ, dK, dV
 *     dbqkv = sum [dQ|dK|dV];  dWqkv = x^T [dQ|dK|dV];  dx = dhid + [dQ|dK|dV] Wqkv^T
 *
 * The forward is rematerialised here (the pages' training recipe stores none
 * of it): the projection, the attention with its per-row statistics, and the
 * out-projection are recomputed, and the FFN intermediate chunk by chunk.
 * x and the weights bf16 as for bpt_layer_forward_ffn; dy fp32 [b, s, h].
 * Outputs fp32, written entirely: dx [b, s, h], dWqkv [h, 3h], dbqkv [3h],
 * dWo [h, h], dbo [h], dW1 [h, ffn], db1 [ffn], dW2 [ffn, h], db2 [h]. Products
 * take bf16 operands with fp32 accumulation. workspace: at least
 * bpt_layer_backward_workspace_bytes bytes of device memory (about 20 bytes
 * per element of [b, s, h] plus the FFN backward's chunk buffers). Causal
 * masking as for the forward. Errors as for bpt_attention_backward, plus
 * BPT_ERR_SHAPE for ffn not a positive multiple of 64; nothing launched then.
 * Asynchronous on `stream`; device-side failures through bpt_stream_status. */
size_t bpt_layer_backward_workspace_bytes(int b, int s, int h, int heads, int ffn);
int bpt_layer_backward(const void* x, const void* Wqkv, const void* bqkv, const void* Wo, const void* bo,
                       const void* W1, const void* b1, const void* W2, const void* b2, const float* dy, int b, int s,
                       int h, int heads, int ffn, int causal, float* dx, float* dWqkv, float* dbqkv, float* dWo,
                       float* dbo, float* dW1, float* db1, float* dW2, float* db2, void* workspace,
                       size_t ws_bytes, void* stream);

/* The forward for a later backward: bpt_layer_forward_ffn (bf16 inputs, FFN
 * width ffn, one launch per GEMM and FFN wave, workspace from the library's
 * pool) that also keeps what the backward would otherwise recompute with a
 * second attention pass -- the attention output O and, per row and head, the
 * normalisation statistic that Algorithm 1 of the paper review records for
 * each query block (the running max m and sum l, kept as m + log2 l in log2
 * units, as bpt_attention_lse writes it). The pages rematerialise the
 * blockwise FFN for training; attention's P is never stored either way, and O
 * is the layer's own activation (the out-projection's input).
 * o_save: bf16 [b, s, h] (head k in columns k*dh ..), lse2_save: fp32
 * [b][heads][s]; both caller-owned device memory, written entirely. out as for
 * bpt_layer_forward_ffn (the same values). Errors as for bpt_layer_forward_ffn,
 * plus BPT_ERR_NULL / BPT_ERR_ALIGN (16 bytes) for o_save and lse2_save and
 * BPT_ERR_ALIAS where they overlap each other, out or an input. */
int bpt_layer_forward_save(const void* x, const void* Wqkv, const void* bqkv, const void* Wo, const void* bo,
                           const void* W1, const void* b1, const void* W2, const void* b2, int b, int s, int h,
                           int heads, int ffn, int q_block, int kv_block, int causal, float* out, void* o_save,
                           float* lse2_save, void* stream);

/* bpt_layer_backward from the forward's saved O and statistics
 * (bpt_layer_forward_save) instead of recomputing the attention: the
 * projection and the out-projection are still recomputed, and the FFN
 * intermediate chunk by chunk. The same arguments, workspace and results as
 * bpt_layer_backward (equal bit for bit when o_saved and lse2_saved come from
 * bpt_layer_forward_save on the same x and weights), plus o_saved bf16 [b, s, h]
 * and lse2_saved fp32 [b][heads][s], read only. Errors as for
 * bpt_layer_backward, plus BPT_ERR_NULL / BPT_ERR_ALIGN for the saved inputs and
 * BPT_ERR_ALIAS where an output or the workspace overlaps them. */
int bpt_layer_backward_saved(const void* x, const void* Wqkv, const void* bqkv, const void* Wo, const void* bo,
                             const void* W1, const void* b1, const void* W2, const void* b2, const void* o_saved,
                             const float* lse2_saved, const float* dy, int b, int s, int h, int heads, int ffn,
                             int causal, float* dx, float* dWqkv, float* dbqkv, float* dWo, float* dbo, float* dW1,
                             float* db1, float* dW2, float* db2, void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Status and measurement.
 * ------------------------------------------------------------------------ */

/* Status of the work queued on one stream (library plumbing; the pages have
 * no counterpart). Synchronises `stream` only (other streams keep running),
 * then returns the status word owned by that stream on the current device --
 * BPT_OK, or BPT_ERR_TIMEOUT if a kernel of this library launched on it gave
 * up a bounded wait since the word was last read -- and resets the word to
 * BPT_OK. A status recorded on another stream is neither returned nor cleared.
 * Call it with the device current on which the work was queued. Returns
 * BPT_ERR_CUDA if the synchronisation or the read fails (for example when no
 * GPU is present). Words are assigned to streams at their first call and kept
 * for the life of the process; past 1023 distinct streams on one device the
 * further ones share one word. A destroyed stream's word passes to a later
 * stream that gets the same handle, so read a stream's status before
 * destroying it. */
int bpt_stream_status(void* stream);

/* Every stream of the current device at once: synchronises the whole device,
 * returns the first status word that is not BPT_OK (or BPT_OK) and resets all
 * words of the device. It stalls every stream of the device; prefer
 * bpt_stream_status. */
int bpt_device_status(void);

/* A check of the status path (library plumbing; the pages have no
 * counterpart): one thread, queued on `stream`, waits until the int at `flag`
 * (device or host-mapped memory, 4-byte aligned) equals `value`, for at most
 * timeout_us microseconds; if it gives up it records BPT_ERR_TIMEOUT in the
 * stream's status word, exactly as the layer's kernels do when one of their
 * bounded waits runs out. The wait ends either way, so it never hangs the
 * stream. Errors: BPT_ERR_NULL, BPT_ERR_ALIGN, BPT_ERR_SHAPE (timeout_us
 * outside [0, 10^7]), with nothing launched. */
int bpt_wait_flag(const int* flag, int value, int timeout_us, void* stream);

/* Number of kernels this library has launched in this process (measurement
 * support; the pages have no counterpart). */
uint64_t bpt_launch_count(void);

/* Kernel timing log (measurement support; the pages have no counterpart).
 * While enabled, every launch is bracketed by CUDA events
 * recorded on its own stream. bpt_kernel_times synchronises and writes, for at
 * most `max` kernel kinds, the name, launch count and summed milliseconds,
 * then clears the log; it returns the number of kinds written. */
typedef struct bpt_kernel_time {
  char name[32];
  int launches;
  double total_ms;
} bpt_kernel_time;

int bpt_set_kernel_timing(int enable);
int bpt_kernel_times(bpt_kernel_time* out, int max);

#ifdef __cplusplus
}
#endif

#endif /* BPT_H_ */
