// blocks.cu -- block-management steps around the paged cache: copy-on-write
// block copies and the slot of each token from (request, position).
//
// "第三部分 · 推理系统与基础设施" (llm-learning-path part 3), chapter map 3.3:
// block tables with copy-on-write -- requests sharing physical blocks keep
// sharing them until one writes, and the writer first gets its own copy of
// the block.  "AI Infra入门干货总结：大模型是如何高效推理的", "Paged Attention":
// slot = block_table[request][pos / block_size] * block_size + pos % block_size.
#include "internal.h"
#include "ptx.cuh"

namespace pa {

// One CTA per (pair, pool): the block's bytes as 16-byte vectors, eight loads
// in flight per thread before their stores.
__global__ void __launch_bounds__(256) copy_blocks_kernel(uint4* __restrict__ kc,
                                                          uint4* __restrict__ vc,
                                                          const int64_t* __restrict__ mapping,
                                                          int64_t num_pairs, int64_t block_vec,
                                                          int64_t num_blocks, int32_t* err) {
  grid_launch_dependents();
  grid_dependency_wait();
  constexpr int U = 8;
  for (int64_t w = blockIdx.x; w < 2 * num_pairs; w += gridDim.x) {
    const int64_t pair = w >> 1;
    const int64_t src = __ldg(mapping + 2 * pair), dst = __ldg(mapping + 2 * pair + 1);
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
      if (threadIdx.x == 0 && (w & 1) == 0 && err) atomicOr(err, PA_ERRBIT_BLOCK_OOB);
      continue;
    }
    if (src == dst) continue;
    uint4* pool = (w & 1) ? vc : kc;
    const uint4* s = pool + src * block_vec;
    uint4* d = pool + dst * block_vec;
    const int nvec = static_cast<int>(block_vec);  // a block is far below 2^31 vectors
    for (int i0 = threadIdx.x; i0 < nvec; i0 += U * blockDim.x) {
      uint4 r[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = i0 + u * blockDim.x;
        if (i < nvec) r[u] = __ldcs(s + i);  // streamed: neither block is re-read here
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = i0 + u * blockDim.x;
        if (i < nvec) __stcs(d + i, r[u]);
      }
    }
  }
}

__global__ void __launch_bounds__(256) slot_positions_kernel(
    const int32_t* __restrict__ block_tables, int32_t max_blocks, int32_t num_seqs,
    const int32_t* __restrict__ token_req, const int64_t* __restrict__ positions,
    int64_t num_tokens, int32_t block_size, int64_t num_blocks, int64_t* __restrict__ slots,
    int32_t* err) {
  grid_launch_dependents();
  grid_dependency_wait();
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < num_tokens;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int32_t b = token_req[t];
    const int64_t p = positions[t];
    int64_t slot = -1;
    int bits = 0;
    if (b >= 0) {
      if (b >= num_seqs || p < 0 || p >= static_cast<int64_t>(max_blocks) * block_size) {
        bits = PA_ERRBIT_POS_OOB;
      } else {
        const int32_t phys = block_tables[static_cast<int64_t>(b) * max_blocks + p / block_size];
        if (phys < 0 || phys >= num_blocks)
          bits = PA_ERRBIT_BLOCK_OOB;
        else
          slot = static_cast<int64_t>(phys) * block_size + p % block_size;
      }
    }
    slots[t] = slot;
    if (bits && err) atomicOr(err, bits);
  }
}

cudaError_t launch_copy_blocks(void* kc, void* vc, const int64_t* mapping, int64_t num_pairs,
                               int64_t block_bytes, int64_t num_blocks, int32_t* err, int num_sms,
                               cudaStream_t s) {
  const int64_t blocks = std::max<int64_t>(
      1, std::min<int64_t>(2 * num_pairs, static_cast<int64_t>(num_sms) * 32));
  return launch_pdl<copy_blocks_kernel>(dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s,
                                        static_cast<uint4*>(kc), static_cast<uint4*>(vc), mapping,
                                        num_pairs, block_bytes / 16, num_blocks, err);
}

cudaError_t launch_slot_positions(const int32_t* block_tables, int32_t max_blocks,
                                  int32_t num_seqs, const int32_t* token_req,
                                  const int64_t* positions, int64_t num_tokens,
                                  int32_t block_size, int64_t num_blocks, int64_t* slots,
                                  int32_t* err, int num_sms, cudaStream_t s) {
  const int64_t blocks = std::max<int64_t>(
      1, std::min<int64_t>((num_tokens + 255) / 256, static_cast<int64_t>(num_sms) * 8));
  return launch_pdl<slot_positions_kernel>(dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s,
                                           block_tables, max_blocks, num_seqs, token_req,
                                           positions, num_tokens, block_size, num_blocks, slots,
                                           err);
}

}  // namespace pa
