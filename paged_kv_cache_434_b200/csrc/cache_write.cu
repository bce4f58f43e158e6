// cache_write.cu -- slot mapping and reshape_and_cache for the paged KV pools.
//
// "AI Infra入门干货总结：大模型是如何高效推理的", section "Paged Attention":
// slot_idx = block_idx * block_size + block_offset; the kernel recovers
// block_idx = slot / block_size and block_offset = slot % block_size.  With the
// pool laid out [num_blocks, block_size, num_kv_heads, head_dim], the whole
// [num_kv_heads, head_dim] row of a token is contiguous at element offset
// slot * num_kv_heads * head_dim, so the scatter is one contiguous row copy per
// token, done with 16-byte vector loads and stores.
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"
#include "slot_write.cuh"

namespace pa {

// One warp per request: tokens query_start_loc[b] .. [b+1]-1 are the request's
// last q_b positions.  Invalid requests get slot -1 for all their tokens.
__global__ void __launch_bounds__(256) slot_mapping_kernel(
    const int32_t* __restrict__ block_tables, int32_t max_blocks,
    const int32_t* __restrict__ qsl, const int32_t* __restrict__ seq_lens, int32_t num_seqs,
    int64_t num_tokens, int32_t block_size, int64_t num_blocks, int64_t* __restrict__ slots,
    int32_t* __restrict__ err) {
  grid_launch_dependents();
  grid_dependency_wait();  // tables and lengths may come from the previous launch
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (b >= num_seqs) return;
  const int32_t t0 = qsl[b], t1 = qsl[b + 1];
  const int32_t q_b = t1 - t0;
  const int32_t L = seq_lens[b];
  int32_t bits = 0;
  if (q_b < 0 || q_b > L) bits |= PA_ERRBIT_QUERY_TOO_LONG;
  if (L > max_blocks * block_size) bits |= PA_ERRBIT_SEQ_TOO_LONG;
  if (t0 < 0) {
    if (lane == 0 && err) atomicOr(err, PA_ERRBIT_QUERY_TOO_LONG);
    return;
  }
  const int32_t* table = block_tables + static_cast<int64_t>(b) * max_blocks;
  for (int32_t i = lane; i < q_b && t0 + static_cast<int64_t>(i) < num_tokens; i += 32) {
    int64_t slot = -1;
    if (bits == 0) {
      const int32_t pos = L - q_b + i;
      const int32_t phys = table[pos / block_size];
      if (phys < 0 || phys >= num_blocks) {
        bits |= PA_ERRBIT_BLOCK_OOB;
      } else {
        slot = static_cast<int64_t>(phys) * block_size + pos % block_size;
      }
    }
    slots[t0 + i] = slot;
  }
  if (bits && err) atomicOr(err, bits);
}

// One warp per (token, K|V): copies row_bytes (a multiple of 16) with uint4.
__global__ void __launch_bounds__(256) cache_write_kernel(
    const uint4* __restrict__ k, const uint4* __restrict__ v, uint4* __restrict__ kc,
    uint4* __restrict__ vc, const int64_t* __restrict__ slots, int64_t num_tokens,
    int64_t row_vec, int64_t num_slots, int32_t* __restrict__ err) {
  grid_launch_dependents();
  grid_dependency_wait();  // the slots usually come from the previous launch
  const int lane = threadIdx.x & 31;
  const int64_t w = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t t = w >> 1;
  if (t >= num_tokens) return;
  const int64_t slot = slots[t];
  if (slot < 0) return;  // padding token
  if (slot >= num_slots) {
    if (lane == 0 && (w & 1) == 0 && err) atomicOr(err, PA_ERRBIT_SLOT_OOB);
    return;
  }
  copy_row(((w & 1) ? v : k) + t * row_vec, ((w & 1) ? vc : kc) + slot * row_vec, row_vec, lane);
}

// FP8 pools: one warp per (token, K|V); a lane turns 16 bf16 entries into 16
// e4m3 codes of the float32 quotients x / scale (IEEE division, the rounding
// the oracle reproduces) per step.
__global__ void __launch_bounds__(256) cache_write_fp8_kernel(
    const uint4* __restrict__ k, const uint4* __restrict__ v, uint4* __restrict__ kc,
    uint4* __restrict__ vc, const int64_t* __restrict__ slots, int64_t num_tokens,
    int64_t row_chunks /* 16-entry chunks per row */, int64_t num_slots, float k_scale,
    float v_scale, int32_t* __restrict__ err) {
  grid_launch_dependents();
  grid_dependency_wait();  // the slots usually come from the previous launch
  const int lane = threadIdx.x & 31;
  const int64_t w = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t t = w >> 1;
  if (t >= num_tokens) return;
  const int64_t slot = slots[t];
  if (slot < 0) return;  // padding token
  if (slot >= num_slots) {
    if (lane == 0 && (w & 1) == 0 && err) atomicOr(err, PA_ERRBIT_SLOT_OOB);
    return;
  }
  const bool is_v = (w & 1) != 0;
  quantize_row((is_v ? v : k) + t * row_chunks * 2,  // 2 uint4 of bf16 per chunk
               (is_v ? vc : kc) + slot * row_chunks,  // 1 uint4 of codes per chunk
               row_chunks, is_v ? v_scale : k_scale, lane);
}

// Slot mapping and the cache write in one launch: one warp per (token, K|V).
template <bool F8>
__global__ void __launch_bounds__(256) slot_cache_write_kernel(SlotWrite a) {
  grid_launch_dependents();
  grid_dependency_wait();  // tables, lengths and rows may come from the previous launch
  const int64_t w = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  slot_write_warp<F8>(a, w, threadIdx.x & 31);
}

cudaError_t launch_slot_cache_write(const void* k, const void* v, void* kc, void* vc,
                                    const int32_t* block_tables, int32_t max_blocks,
                                    const int32_t* qsl, const int32_t* seq_lens, int32_t num_seqs,
                                    int64_t num_tokens, int32_t block_size, int64_t num_blocks,
                                    int64_t row_elems, int32_t elt_bytes, bool fp8,
                                    float k_scale, float v_scale, int64_t* slots, int32_t* err,
                                    cudaStream_t s) {
  if (num_tokens == 0) return cudaSuccess;
  const int warps = 8;
  const int64_t nwarps = 2 * num_tokens;
  dim3 grid(static_cast<unsigned>((nwarps + warps - 1) / warps));
  const SlotWrite a = make_slot_write(k, v, kc, vc, block_tables, max_blocks, qsl, seq_lens,
                                      num_seqs, num_tokens, block_size, num_blocks, row_elems,
                                      elt_bytes, fp8, k_scale, v_scale, slots, err);
  if (fp8) return launch_pdl<slot_cache_write_kernel<true>>(grid, dim3(warps * 32), 0, s, a);
  return launch_pdl<slot_cache_write_kernel<false>>(grid, dim3(warps * 32), 0, s, a);
}

cudaError_t launch_cache_write_fp8(const void* k, const void* v, void* kc, void* vc,
                                   const int64_t* slots, int64_t num_tokens, int64_t row_elems,
                                   int64_t num_slots, float k_scale, float v_scale, int32_t* err,
                                   cudaStream_t s) {
  if (num_tokens == 0) return cudaSuccess;
  const int warps = 8;
  const int64_t nwarps = 2 * num_tokens;
  dim3 grid(static_cast<unsigned>((nwarps + warps - 1) / warps));
  return launch_pdl<cache_write_fp8_kernel>(
      grid, dim3(warps * 32), 0, s, static_cast<const uint4*>(k), static_cast<const uint4*>(v),
      static_cast<uint4*>(kc), static_cast<uint4*>(vc), slots, num_tokens, row_elems / 16,
      num_slots, k_scale, v_scale, err);
}

cudaError_t launch_slot_mapping(const int32_t* block_tables, int32_t max_blocks,
                                const int32_t* qsl, const int32_t* seq_lens, int32_t num_seqs,
                                int64_t num_tokens, int32_t block_size, int64_t num_blocks,
                                int64_t* slots, int32_t* err, cudaStream_t s) {
  if (num_seqs == 0) return cudaSuccess;
  const int warps = 8;
  dim3 grid((num_seqs + warps - 1) / warps);
  return launch_pdl<slot_mapping_kernel>(grid, dim3(warps * 32), 0, s, block_tables, max_blocks,
                                         qsl, seq_lens, num_seqs, num_tokens, block_size,
                                         num_blocks, slots, err);
}

cudaError_t launch_cache_write(const void* k, const void* v, void* kc, void* vc,
                               const int64_t* slots, int64_t num_tokens, int64_t row_bytes,
                               int64_t num_slots, int32_t* err, cudaStream_t s) {
  if (num_tokens == 0) return cudaSuccess;
  const int warps = 8;
  const int64_t nwarps = 2 * num_tokens;
  dim3 grid(static_cast<unsigned>((nwarps + warps - 1) / warps));
  return launch_pdl<cache_write_kernel>(
      grid, dim3(warps * 32), 0, s, static_cast<const uint4*>(k), static_cast<const uint4*>(v),
      static_cast<uint4*>(kc), static_cast<uint4*>(vc), slots, num_tokens, row_bytes / 16,
      num_slots, err);
}

}  // namespace pa
