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

// A warp copies one row of row_vec 16-byte vectors, 4 loads in flight per lane
// before the stores.
__device__ __forceinline__ void copy_row(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                         int64_t row_vec, int lane) {
  int64_t i = lane;
  for (; i + 96 < row_vec; i += 128) {
    uint4 a = __ldg(src + i), b = __ldg(src + i + 32), c = __ldg(src + i + 64),
          d = __ldg(src + i + 96);
    dst[i] = a;
    dst[i + 32] = b;
    dst[i + 64] = c;
    dst[i + 96] = d;
  }
  for (; i < row_vec; i += 32) dst[i] = __ldg(src + i);
}

// A warp quantises one row of bf16 entries to e4m3 codes of the float32
// quotients x / sc (IEEE division, the rounding the oracle reproduces), 16
// entries (two uint4 in, one out) per lane and step.
__device__ __forceinline__ void quantize_row(const uint4* __restrict__ src,
                                             uint4* __restrict__ dst, int64_t row_chunks, float sc,
                                             int lane) {
  for (int64_t c = lane; c < row_chunks; c += 32) {
    const uint4 a = __ldg(src + 2 * c), b = __ldg(src + 2 * c + 1);
    const uint32_t in[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t out[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 p0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&in[2 * j]));
      const float2 p1 =
          __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&in[2 * j + 1]));
      const uint16_t lo = f32x2_to_e4m3x2(__fdiv_rn(p0.x, sc), __fdiv_rn(p0.y, sc));
      const uint16_t hi = f32x2_to_e4m3x2(__fdiv_rn(p1.x, sc), __fdiv_rn(p1.y, sc));
      out[j] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
    }
    dst[c] = make_uint4(out[0], out[1], out[2], out[3]);
  }
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

// The request owning flattened token t: the largest b < num_seqs with
// qsl[b] <= t (requests with no token are passed over).  The warp probes 32
// positions at once, so a batch of up to ~1000 requests takes two rounds.
__device__ __forceinline__ int request_of_token(const int32_t* __restrict__ qsl, int num_seqs,
                                                int64_t t, int lane) {
  int lo = 0, hi = num_seqs;  // qsl[lo] <= t < qsl[hi] for a well-formed qsl
  while (hi - lo > 1) {
    const int span = hi - lo;
    const int probe = span <= 33 ? lo + 1 + lane
                                 : lo + static_cast<int>(static_cast<int64_t>(span) * (lane + 1) / 33);
    const bool valid = probe > lo && probe < hi;
    const bool le = valid && __ldg(qsl + probe) <= t;
    const unsigned m = __ballot_sync(0xffffffffu, le);
    const unsigned gt = __ballot_sync(0xffffffffu, valid && !le);
    const int nlo = m ? __shfl_sync(0xffffffffu, probe, 31 - __clz(m)) : lo;
    const int nhi = gt ? __shfl_sync(0xffffffffu, probe, __ffs(gt) - 1) : hi;
    lo = nlo;
    hi = nhi;
  }
  return lo;
}

// Slot mapping and the cache write in one launch: one warp per (token, K|V)
// finds the token's request, its position and slot (the checks of
// slot_mapping_kernel), and copies (or, F8, quantises) the row.  The K warp
// of a token writes its slot and reports the error bits.  qsl == nullptr: one
// new token per request (a decode step), token t of request t.
template <bool F8>
__global__ void __launch_bounds__(256) slot_cache_write_kernel(
    const uint4* __restrict__ k, const uint4* __restrict__ v, uint4* __restrict__ kc,
    uint4* __restrict__ vc, const int32_t* __restrict__ block_tables, int32_t max_blocks,
    const int32_t* __restrict__ qsl, const int32_t* __restrict__ seq_lens, int32_t num_seqs,
    int64_t num_tokens, int32_t block_size, int64_t num_blocks, int64_t row_units,
    float k_scale, float v_scale, int64_t* __restrict__ slots, int32_t* __restrict__ err) {
  grid_launch_dependents();
  grid_dependency_wait();  // tables, lengths and rows may come from the previous launch
  const int lane = threadIdx.x & 31;
  const int64_t w = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t t = w >> 1;
  if (t >= num_tokens) return;
  const int b = qsl ? request_of_token(qsl, num_seqs, t, lane) : static_cast<int>(t);
  const int32_t t0 = qsl ? __ldg(qsl + b) : b;
  const int32_t q_b = qsl ? __ldg(qsl + b + 1) - t0 : 1;
  const int32_t L = __ldg(seq_lens + b);
  int32_t bits = 0;
  if (q_b < 0 || q_b > L || t < t0 || t - t0 >= q_b) bits |= PA_ERRBIT_QUERY_TOO_LONG;
  if (L > max_blocks * block_size) bits |= PA_ERRBIT_SEQ_TOO_LONG;
  int64_t slot = -1;
  if (bits == 0) {
    const int32_t pos = L - q_b + static_cast<int32_t>(t - t0);
    const int32_t phys = __ldg(block_tables + static_cast<int64_t>(b) * max_blocks + pos / block_size);
    if (phys < 0 || phys >= num_blocks) bits |= PA_ERRBIT_BLOCK_OOB;
    else slot = static_cast<int64_t>(phys) * block_size + pos % block_size;
  }
  if ((w & 1) == 0 && lane == 0) {
    if (slots) slots[t] = slot;
    if (bits && err) atomicOr(err, bits);
  }
  if (slot < 0) return;
  const bool is_v = (w & 1) != 0;
  if constexpr (F8)
    quantize_row((is_v ? v : k) + t * row_units * 2, (is_v ? vc : kc) + slot * row_units,
                 row_units, is_v ? v_scale : k_scale, lane);
  else
    copy_row((is_v ? v : k) + t * row_units, (is_v ? vc : kc) + slot * row_units, row_units, lane);
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
  const uint4* k4 = static_cast<const uint4*>(k);
  const uint4* v4 = static_cast<const uint4*>(v);
  uint4* kc4 = static_cast<uint4*>(kc);
  uint4* vc4 = static_cast<uint4*>(vc);
  if (fp8)
    return launch_pdl<slot_cache_write_kernel<true>>(
        grid, dim3(warps * 32), 0, s, k4, v4, kc4, vc4, block_tables, max_blocks, qsl, seq_lens,
        num_seqs, num_tokens, block_size, num_blocks, row_elems / 16, k_scale, v_scale, slots,
        err);
  return launch_pdl<slot_cache_write_kernel<false>>(
      grid, dim3(warps * 32), 0, s, k4, v4, kc4, vc4, block_tables, max_blocks, qsl, seq_lens,
      num_seqs, num_tokens, block_size, num_blocks, row_elems * elt_bytes / 16, k_scale, v_scale,
      slots, err);
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
