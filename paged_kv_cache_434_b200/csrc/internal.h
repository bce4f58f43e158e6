// internal.h -- structures shared by the C-ABI layer and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <atomic>
#include <utility>

#include <cuda_runtime.h>

#include "pa.h"  // include/ is on the include path

namespace pa {

constexpr int kStageTokens = 16;     // keys per pipeline stage / partition granule
constexpr int kMaxGroup = 16;        // query heads per KV head handled in one tile
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bounded device waits: 2 s

// ---------------------------------------------------------------- workspace
// One attention call's scratch, carved from the caller's workspace buffer.
//   ctrl      int32[64]   [0] dynamic work counter, [1] number of items,
//                         [2] partition length in tokens, [3] tile counter,
//                         [4] number of tensor-core tiles, [5] rows to merge,
//                         [6] shared-prefix tokens (decode cascade, 0: none),
//                         [7] key chunks the shared prefix is split into,
//                         [8] CTAs of the tensor-core tile kernel that work,
//                         [9] rows to merge with more than kMergeWarpParts partitions
//                         (listed from the back of merge_rows)
//   qrow_info int4[R]     {request b, key_len, valid, key_start}: the row's
//                         partitions cover keys [key_start, key_len); keys
//                         below key_start (a shared prefix) come from tiles
//   nparts    int32[R]    partitions of the row (0: empty -> zero row;
//                         -1: invalid -> row left unwritten)
//   qrow_bad  int32[R]    set when a block id outside the pool was met
//   merge_rows int32[R]   rows the merge pass must write (0 or >1 partitions):
//                         up to kMergeWarpParts partitions from the front, more from the back
//   items     int4[I]     {qrow, head group | partition << 16, stages, first
//                         stage}: keys [key_start + 16 first, + 16 stages) of
//                         the row, clipped to its length
//   part_ml   float2[R*H*P]   per (row, query head, partition): (m, l),
//                         m in log2 units (score * scale * log2 e)
//   part_o    float[R*H*P*D]  unnormalised partial outputs
//   tiles     int4[Tl]    tensor-core tiles: prefill {request b, kv head, first
//                         token, tokens}; shared prefix {first request, kv
//                         head, requests, key chunk}
struct WsLayout {
  size_t ctrl, qrow_info, nparts, qrow_bad, merge_rows, items, part_ml, part_o, tiles, total;
  int64_t num_qrows, max_parts, max_items, max_tiles;
};

// Item field packing: head group in the low 16 bits of .y, the partition index
// in the high 16 (partitions per row stay far below 2^15).
constexpr int kItemPartShift = 16;
constexpr int kItemHgMask = (1 << kItemPartShift) - 1;

struct WsView {
  int32_t* ctrl;
  int4* qrow_info;
  int32_t* nparts;
  int32_t* qrow_bad;
  int32_t* merge_rows;
  int4* items;
  float2* part_ml;
  float* part_o;
  int4* tiles;
  int64_t max_parts;
  int64_t max_items;
  int64_t max_tiles;
};

WsLayout ws_layout(int64_t num_qrows, int num_heads, int head_dim, int head_groups,
                   int64_t max_parts, int64_t max_tiles);
WsView ws_view(void* base, const WsLayout& L);

// ---------------------------------------------------------------- geometry
struct AttnGeom {
  const void* q;          // [R, Hq, D]
  const void* k_cache;    // [NB, bs, Hkv, D]
  const void* v_cache;
  const int32_t* block_tables;
  const int32_t* seq_lens;
  const int32_t* query_start_loc;  // nullptr for decode
  void* out;              // [R, Hq, D]
  int64_t num_blocks;
  int32_t num_seqs;
  int32_t num_qrows;
  int32_t num_heads;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t block_size;
  int32_t max_blocks;
  int32_t dtype;          // pa_dtype of q / caches
  int32_t out_dtype;
  float scale_log2;       // scale * log2(e) (* k_scale for an FP8 cache)
  float v_scale;          // FP8 cache: value entry = code * v_scale; 1 otherwise
  int32_t* err_word;
};

// ---------------------------------------------------------------- planner
struct PlanArgs {
  int32_t head_groups;      // items per (row, partition)
  int32_t heads_per_group;  // KV heads per item
  int32_t target_items;     // aim for about this many items in total
  int32_t min_part_stages;  // lower bound of a partition, in 16-key stages
  int32_t expand_prefill;   // 1: every query of a q_b>1 request is its own row
  int32_t tile_tokens;      // tokens (rows of a request) per tensor-core tile pair
  int32_t cascade;          // decode: attend a prefix shared by all requests once
  int32_t num_sms;
};

// Shared-prefix cascade: only worth it for long prefixes and enough requests.
constexpr int kCascadeMinPrefix = 256;
constexpr int kCascadeMinSeqs = 16;
constexpr int kMaxPrefixChunks = 8;  // partitions reserved per row for the shared prefix
// rows with at most this many split-KV partitions are merged by one warp per
// (row, head); the others by one CTA per (row, head)
constexpr int kMergeWarpParts = 64;

// ---------------------------------------------------------------- launchers
// Each returns cudaSuccess or the launch error.
// Every kernel of a step is launched with programmatic dependent launch
// allowed: it may become resident while the previous kernel on the stream
// drains, and reads nothing that kernel wrote before griddepcontrol.wait.
// Kernels ask for the largest shared-memory carveout, so that a kernel
// launched early can share an SM with the one before it instead of waiting
// for the SM to be reconfigured.
// Each kernel's dynamic shared memory is fixed by its template arguments.
template <auto Kern, typename... Args>
inline cudaError_t launch_pdl(dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args&&... args) {
  static std::atomic<unsigned long long> attrs_set{0};  // one bit per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attrs_set.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(Kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e == cudaSuccess && smem > 48 * 1024)
      e = cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    attrs_set.fetch_or(bit, std::memory_order_acq_rel);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, Kern, std::forward<Args>(args)...);
}

struct RopeLaunch {
  const void* q_in;
  const void* k;
  const void* v;
  int64_t q_stride, kv_stride;
  void* q_out;
  void* kc;
  void* vc;
  const int64_t* positions;
  const int64_t* slots;
  const float* cs;
  int32_t max_position, rot, neox;
  int64_t num_tokens;
  int32_t hq, hkv, d, dtype;
  int64_t num_slots;
  int32_t* err;
};
cudaError_t launch_rope_table(float* cache, int32_t max_position, int32_t rotary_dim, double theta,
                              int num_sms, cudaStream_t s);
cudaError_t launch_rope_cache_write(const RopeLaunch& l, int num_sms, cudaStream_t s);
cudaError_t launch_copy_blocks(void* kc, void* vc, const int64_t* mapping, int64_t num_pairs,
                               int64_t block_bytes, int64_t num_blocks, int32_t* err, int num_sms,
                               cudaStream_t s);
cudaError_t launch_slot_positions(const int32_t* block_tables, int32_t max_blocks,
                                  int32_t num_seqs, const int32_t* token_req,
                                  const int64_t* positions, int64_t num_tokens,
                                  int32_t block_size, int64_t num_blocks, int64_t* slots,
                                  int32_t* err, int num_sms, cudaStream_t s);
cudaError_t launch_slot_cache_write(const void* k, const void* v, void* kc, void* vc,
                                    const int32_t* block_tables, int32_t max_blocks,
                                    const int32_t* qsl, const int32_t* seq_lens, int32_t num_seqs,
                                    int64_t num_tokens, int32_t block_size, int64_t num_blocks,
                                    int64_t row_elems, int32_t elt_bytes, bool fp8,
                                    float k_scale, float v_scale, int64_t* slots, int32_t* err,
                                    cudaStream_t s);
cudaError_t launch_cache_write_fp8(const void* k, const void* v, void* kc, void* vc,
                                   const int64_t* slots, int64_t num_tokens, int64_t row_elems,
                                   int64_t num_slots, float k_scale, float v_scale, int32_t* err,
                                   cudaStream_t s);
cudaError_t launch_slot_mapping(const int32_t* block_tables, int32_t max_blocks,
                                const int32_t* qsl, const int32_t* seq_lens, int32_t num_seqs,
                                int64_t num_tokens, int32_t block_size, int64_t num_blocks,
                                int64_t* slots, int32_t* err, cudaStream_t s);
cudaError_t launch_cache_write(const void* k, const void* v, void* kc, void* vc,
                               const int64_t* slots, int64_t num_tokens, int64_t row_bytes,
                               int64_t num_slots, int32_t* err, cudaStream_t s);
cudaError_t launch_plan(const AttnGeom& g, const PlanArgs& a, const WsView& ws, cudaStream_t s);
struct SlotWrite;
// The planner on CTA 0 and the slot mapping + cache write of sw on the others.
cudaError_t launch_write_plan(const AttnGeom& g, const PlanArgs& a, const WsView& ws,
                              const SlotWrite& sw, bool fp8, cudaStream_t s);
cudaError_t launch_attn_generic(const AttnGeom& g, const WsView& ws, int num_sms,
                                cudaStream_t s);
cudaError_t launch_attn_mma(const AttnGeom& g, const WsView& ws, int num_sms, int heads_per_group,
                            int after_tiles, cudaStream_t s);
cudaError_t launch_merge(const AttnGeom& g, const WsView& ws, int num_sms, cudaStream_t s);
cudaError_t launch_attn_tc(const AttnGeom& g, const WsView& ws, int grid, cudaStream_t s);

bool mma_path_supported(const AttnGeom& g);
bool tc_path_supported(const AttnGeom& g);
int tc_tokens_per_tile(const AttnGeom& g);
int device_num_sms();

}  // namespace pa
