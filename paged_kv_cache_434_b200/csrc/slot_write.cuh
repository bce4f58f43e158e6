// slot_write.cuh -- the per-warp body of the slot mapping + cache write,
// shared by its own launch (cache_write.cu) and by the decode step's first
// launch, where it runs beside the work planner (attn_common.cu).
//
// "AI Infra入门干货总结：大模型是如何高效推理的", sections "Paged Attention"
// and "Reshape & Cache": a token at position pos of request b goes to slot
// block_tables[b][pos / block_size] * block_size + pos % block_size, and its
// [num_kv_heads, head_dim] K and V rows are copied there.
#pragma once

#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace pa {

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

// Arguments of one slot mapping + cache write.  row_units: uint4 of a pool
// row (16 bytes of entries, or 16 e4m3 codes -- 32 bytes of bf16 input -- F8).
// qsl == nullptr: one new token per request (a decode step), token t of
// request t.
struct SlotWrite {
  const uint4* k;
  const uint4* v;
  uint4* kc;
  uint4* vc;
  const int32_t* block_tables;
  const int32_t* qsl;
  const int32_t* seq_lens;
  int64_t* slots;
  int32_t* err;
  int64_t num_tokens;
  int64_t num_blocks;
  int64_t row_units;
  int32_t max_blocks;
  int32_t num_seqs;
  int32_t block_size;
  float k_scale, v_scale;
};

// Warp w of the write handles (token w / 2, K if w is even else V): it finds
// the token's request, its position and slot (the checks of the separate slot
// mapping), and copies (or, F8, quantises) the row.  The K warp of a token
// writes its slot and reports the error bits.
template <bool F8>
__device__ __forceinline__ void slot_write_warp(const SlotWrite& a, int64_t w, int lane) {
  const int64_t t = w >> 1;
  if (t >= a.num_tokens) return;
  const int32_t* qsl = a.qsl;
  const int b = qsl ? request_of_token(qsl, a.num_seqs, t, lane) : static_cast<int>(t);
  const int32_t t0 = qsl ? __ldg(qsl + b) : b;
  const int32_t q_b = qsl ? __ldg(qsl + b + 1) - t0 : 1;
  const int32_t L = __ldg(a.seq_lens + b);
  int32_t bits = 0;
  if (q_b < 0 || q_b > L || t < t0 || t - t0 >= q_b) bits |= PA_ERRBIT_QUERY_TOO_LONG;
  if (L > a.max_blocks * a.block_size) bits |= PA_ERRBIT_SEQ_TOO_LONG;
  int64_t slot = -1;
  if (bits == 0) {
    const int32_t pos = L - q_b + static_cast<int32_t>(t - t0);
    const int32_t phys =
        __ldg(a.block_tables + static_cast<int64_t>(b) * a.max_blocks + pos / a.block_size);
    if (phys < 0 || phys >= a.num_blocks) bits |= PA_ERRBIT_BLOCK_OOB;
    else slot = static_cast<int64_t>(phys) * a.block_size + pos % a.block_size;
  }
  if ((w & 1) == 0 && lane == 0) {
    if (a.slots) a.slots[t] = slot;
    if (bits && a.err) atomicOr(a.err, bits);
  }
  if (slot < 0) return;
  const bool is_v = (w & 1) != 0;
  if constexpr (F8)
    quantize_row((is_v ? a.v : a.k) + t * a.row_units * 2, (is_v ? a.vc : a.kc) + slot * a.row_units,
                 a.row_units, is_v ? a.v_scale : a.k_scale, lane);
  else
    copy_row((is_v ? a.v : a.k) + t * a.row_units, (is_v ? a.vc : a.kc) + slot * a.row_units,
             a.row_units, lane);
}

// One launch's SlotWrite for these sizes (host side).
inline SlotWrite make_slot_write(const void* k, const void* v, void* kc, void* vc,
                                 const int32_t* block_tables, int32_t max_blocks,
                                 const int32_t* qsl, const int32_t* seq_lens, int32_t num_seqs,
                                 int64_t num_tokens, int32_t block_size, int64_t num_blocks,
                                 int64_t row_elems, int32_t elt_bytes, bool fp8, float k_scale,
                                 float v_scale, int64_t* slots, int32_t* err) {
  SlotWrite a;
  a.k = static_cast<const uint4*>(k);
  a.v = static_cast<const uint4*>(v);
  a.kc = static_cast<uint4*>(kc);
  a.vc = static_cast<uint4*>(vc);
  a.block_tables = block_tables;
  a.qsl = qsl;
  a.seq_lens = seq_lens;
  a.slots = slots;
  a.err = err;
  a.num_tokens = num_tokens;
  a.num_blocks = num_blocks;
  a.row_units = fp8 ? row_elems / 16 : row_elems * elt_bytes / 16;
  a.max_blocks = max_blocks;
  a.num_seqs = num_seqs;
  a.block_size = block_size;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  return a;
}

}  // namespace pa
