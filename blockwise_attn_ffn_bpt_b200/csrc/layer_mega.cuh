// The layer's attention and its FFN side (Algorithm 1 steps 4-11 of the BPT
// paper review, for every query block) in ONE persistent launch, with bounded
// device-side dependency waits.
//
// The block size and the per-CTA resources are the attention kernel's (384
// threads, its register split, all 512 tensor-memory columns; shared memory
// the larger of the two layouts, so one CTA per SM). Each CTA first takes a
// ticket from a global counter. Tickets 0 .. n_att - 1 are attention work
// items (two query tiles of one head), in row order with every head of a
// tile pair before the next pair, so that early rows finish first; the
// attention epilogue counts, per group of output rows, the warps whose rows
// are stored. The remaining tickets make CTAs of the FFN side's queue
// (ffn_chain.cuh), whose out-projection tiles of row group g wait until all
// of g's attention rows are counted; from there the queue runs as in its own
// launch. While the heaviest attention items finish, SMs that are done with
// attention already run the FFN side of the first row groups.
//
// Progress: tickets go to CTAs in the order they start, so every attention
// item is held by a CTA that has started before any FFN-side CTA exists; an
// attention item waits on nothing outside its CTA, and an FFN-side tile only on
// attention items and on earlier tiles of the queue. Every wait is bounded
// (BPT_ERR_TIMEOUT on the launching stream's status word).
#pragma once

#include "attention.cuh"
#include "ffn_chain.cuh"

namespace bpt {

template <int DH>
constexpr int mega_smem_bytes() {
  return AttnCfg<DH>::SMEM_BYTES > GEMM_SMEM_BYTES ? AttnCfg<DH>::SMEM_BYTES : GEMM_SMEM_BYTES;
}

struct MegaArgs {
  unsigned* ticket;  // zeroed before the launch
  int n_att;         // attention work items
};

template <int DH>
__global__ void __launch_bounds__(ATT_THREADS, 1)
    layer_mega_tcgen05(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                       const __grid_constant__ CUtensorMap tmHb, const __grid_constant__ CUtensorMap tmU,
                       const __grid_constant__ CUtensorMap tmWo, const __grid_constant__ CUtensorMap tmW1,
                       const __grid_constant__ CUtensorMap tmW2, const AttnArgs att, const ChainArgs chain,
                       const MegaArgs mega) {
  extern __shared__ uint8_t smem_raw[];
  volatile int* slot = reinterpret_cast<volatile int*>(smem_raw);
  if (threadIdx.x == 0) *slot = (int)atomicAdd(mega.ticket, 1u);
  __syncthreads();
  const int ticket = *slot;
  __syncthreads();  // read by every thread before the work reuses the memory
  if (ticket < mega.n_att)
    attention_fwd_body<DH, false, true>(tmQ, tmK, tmV, att, ticket, 0);
  else
    ffn_chain_body(tmO, tmHb, tmU, tmWo, tmW1, tmW2, chain, ticket - mega.n_att, (int)gridDim.x - mega.n_att);
}

}  // namespace bpt
