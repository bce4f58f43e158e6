// pa_api.cu -- the extern "C" entry points declared in include/pa.h.
//
// Host side only: validates arguments, sizes and carves the workspace, picks the
// kernel path and enqueues the launches.  No allocation, no host<->device
// synchronisation except in pa_read_error.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "internal.h"
#include "slot_write.cuh"

namespace pa {

int device_num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 0;
  if (dev < 64 && cache[dev]) return cache[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev < 64) cache[dev] = n;
  return n;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static pa_status check_cache(const pa_cache_desc* c) {
  if (!c) return PA_ERR_INVALID_ARG;
  if (c->num_blocks < 1 || c->num_kv_heads < 1) return PA_ERR_INVALID_ARG;
  const int bs = c->block_size;
  if (!(bs == 8 || bs == 16 || bs == 32 || bs == 64 || bs == 128 || bs == 256))
    return PA_ERR_UNSUPPORTED;
  if (c->head_dim != 64 && c->head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (c->dtype != PA_F32 && c->dtype != PA_BF16 && c->dtype != PA_FP8_E4M3)
    return PA_ERR_UNSUPPORTED;
  if (c->dtype == PA_FP8_E4M3 &&
      !(c->k_scale > 0.f && c->k_scale < INFINITY && c->v_scale > 0.f && c->v_scale < INFINITY))
    return PA_ERR_INVALID_ARG;
  return PA_OK;
}

// bytes of one element of q / new k, v rows (bf16 for an FP8 cache)
static int elt_bytes(int dtype) { return dtype == PA_F32 ? 4 : 2; }
// bytes of one pool entry
static int pool_elt_bytes(int dtype) { return dtype == PA_F32 ? 4 : dtype == PA_BF16 ? 2 : 1; }

// Largest workspace the library plans for: far beyond any device's memory,
// and small enough that none of the size terms of ws_layout can wrap.
constexpr double kMaxWorkspaceBytes = 70368744177664.0;  // 2^46

// Launch plan of one attention call (decode or mixed step); identical in the
// workspace-size query and in the call itself.
struct AttnPlan {
  bool size_ok;      // the workspace stays within kMaxWorkspaceBytes
  bool use_mma;
  bool use_tc;       // tcgen05 tiles: prefill requests, or a decode batch's shared prefix
  bool cascade;      // decode: shared-prefix tiles + suffix partitions
  int tile_tokens;
  int tc_grid;       // CTAs of the tensor-core tile launch
  int heads_per_group;
  int head_groups;
  int num_sms;
  int64_t num_qrows;
  int64_t max_parts;
  int target_items;
  int64_t max_tiles;
};

static AttnPlan make_plan(int64_t num_qrows, int num_heads, int max_blocks,
                          const pa_cache_desc* c, bool bf16_fast_ok, int num_seqs = 0,
                          bool mixed = false) {
  AttnPlan p{};
  AttnGeom probe{};
  probe.num_heads = num_heads;
  probe.num_kv_heads = c->num_kv_heads;
  probe.head_dim = c->head_dim;
  probe.block_size = c->block_size;
  probe.dtype = c->dtype;
  probe.num_blocks = c->num_blocks;
  p.use_mma = bf16_fast_ok && mma_path_supported(probe);
  if (p.use_mma) {
    int hg = 8;
    while (c->num_kv_heads % hg) hg >>= 1;
    p.heads_per_group = hg;
  } else {
    p.heads_per_group = 1;
  }
  p.head_groups = c->num_kv_heads / p.heads_per_group;
  p.num_sms = device_num_sms();
  if (p.num_sms <= 0) p.num_sms = 148;
  p.num_qrows = num_qrows;
  p.target_items = p.num_sms * (p.use_mma ? 8 : 16);
  const int64_t max_units =
      (static_cast<int64_t>(max_blocks) * c->block_size + kStageTokens - 1) / kStageTokens;
  const int64_t denom = num_qrows * p.head_groups;
  int64_t mp = denom > 0 ? (p.target_items + denom - 1) / denom : 1;
  if (mp > max_units) mp = max_units;
  if (mp < 1) mp = 1;
  const bool tc_ok = p.use_mma && tc_path_supported(probe);
  p.cascade = !mixed && tc_ok && num_qrows >= kCascadeMinSeqs;
  p.use_tc = (mixed && tc_ok) || p.cascade;
  p.max_parts = mp + (p.cascade ? kMaxPrefixChunks : 0);  // shared-prefix chunks
  p.tile_tokens = p.use_tc ? tc_tokens_per_tile(probe) : 0;
  // A decode batch's shared-prefix tiles take at most one SM in two (the
  // suffix partitions stream on the others from the start) unless there are
  // more (request group, KV head) tiles than that: a grid of half the SMs
  // leaves the other half to the partitions at once, also when the planner
  // finds no shared prefix and the tile CTAs only exit.
  p.tc_grid = p.num_sms;
  if (p.cascade && p.tile_tokens > 0) {
    const int64_t base =
        (num_qrows + p.tile_tokens - 1) / p.tile_tokens * static_cast<int64_t>(c->num_kv_heads);
    if (2 * base <= p.num_sms) p.tc_grid = (p.num_sms + 1) / 2;
  }
  // ws_layout's terms in double first: arguments whose exact workspace would
  // not fit a size_t are refused instead of getting a wrapped, too small size
  const double rows = static_cast<double>(num_qrows), parts = static_cast<double>(p.max_parts);
  const double tiles =
      p.use_tc ? (std::ceil(rows / p.tile_tokens) + num_seqs) * c->num_kv_heads *
                     (p.cascade ? kMaxPrefixChunks : 1)
               : 0.0;
  const double bytes = 64.0 * 4 + rows * (16 + 3 * 4) + rows * p.head_groups * parts * 16 +
                       rows * num_heads * parts * (8 + 4.0 * c->head_dim) + tiles * 16 +
                       9 * 256;
  p.size_ok = bytes <= kMaxWorkspaceBytes;
  p.max_tiles = (p.use_tc && p.size_ok)
                    ? ((num_qrows + p.tile_tokens - 1) / p.tile_tokens + num_seqs) *
                          static_cast<int64_t>(c->num_kv_heads) *
                          (p.cascade ? kMaxPrefixChunks : 1)
                    : 0;
  return p;
}

static AttnGeom make_geom(const void* q, const void* kc, const void* vc, const int32_t* bt,
                          const int32_t* sl, const int32_t* qsl, float scale, void* out,
                          int32_t num_seqs, int64_t num_qrows, int32_t num_heads,
                          int32_t max_blocks, int32_t out_dtype, const pa_cache_desc* c,
                          int32_t* err) {
  AttnGeom g{};
  g.q = q;
  g.k_cache = kc;
  g.v_cache = vc;
  g.block_tables = bt;
  g.seq_lens = sl;
  g.query_start_loc = qsl;
  g.out = out;
  g.num_blocks = c->num_blocks;
  g.num_seqs = num_seqs;
  g.num_qrows = static_cast<int32_t>(num_qrows);
  g.num_heads = num_heads;
  g.num_kv_heads = c->num_kv_heads;
  g.head_dim = c->head_dim;
  g.block_size = c->block_size;
  g.max_blocks = max_blocks;
  g.dtype = c->dtype;
  g.out_dtype = out_dtype;
  g.scale_log2 = scale * 1.4426950408889634f;
  g.v_scale = 1.f;
  if (c->dtype == PA_FP8_E4M3) {  // scores see code * k_scale, outputs code * v_scale
    g.scale_log2 *= c->k_scale;
    g.v_scale = c->v_scale;
  }
  g.err_word = err;
  return g;
}

static pa_status check_attn_args(int32_t num_seqs, int64_t num_qrows, int32_t num_heads,
                                  int32_t max_blocks, int32_t out_dtype,
                                  const pa_cache_desc* c) {
  pa_status st = check_cache(c);
  if (st != PA_OK) return st;
  if (num_seqs < 0 || num_qrows < 0 || num_qrows > (1LL << 30) || max_blocks < 0)
    return PA_ERR_INVALID_ARG;
  if (num_heads < 1 || num_heads % c->num_kv_heads) return PA_ERR_INVALID_ARG;
  if (num_heads / c->num_kv_heads > kMaxGroup) return PA_ERR_UNSUPPORTED;
  if (out_dtype != PA_F32 && out_dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(max_blocks) * c->block_size > (1LL << 30)) return PA_ERR_UNSUPPORTED;
  return PA_OK;
}

// Per-launch device timing (a measurement aid): one event pair per launch kind,
// recorded on the call's stream while timing is on for the current device.
struct LaunchTimer {
  std::mutex mu;
  bool on = false;
  bool pending = false;
  bool failed = false;
  int device = -1;
  bool launched[PA_TIMED_KERNELS] = {};
  cudaEvent_t ev[2 * PA_TIMED_KERNELS] = {};
};
static LaunchTimer g_timer;

class TimedCall {
 public:
  explicit TimedCall(cudaStream_t s) : s_(s) {
    std::lock_guard<std::mutex> lk(g_timer.mu);
    int dev = -1;
    if (!g_timer.on || cudaGetDevice(&dev) != cudaSuccess || dev != g_timer.device) return;
    active_ = true;
    g_timer.pending = true;
    g_timer.failed = false;
    for (bool& l : g_timer.launched) l = false;
  }
  void begin(int k) { record(2 * k, k); }
  void end(int k) { record(2 * k + 1, k); }

 private:
  void record(int i, int k) {
    if (!active_) return;
    if (cudaEventRecord(g_timer.ev[i], s_) != cudaSuccess) g_timer.failed = true;
    g_timer.launched[k] = true;
  }
  cudaStream_t s_;
  bool active_ = false;
};

// sw != nullptr: the call also writes the step's new K/V rows (decode form),
// in the planner's launch.
static pa_status run_attention(const AttnGeom& g, const AttnPlan& p, void* workspace,
                               size_t ws_bytes, cudaStream_t s, const SlotWrite* sw = nullptr,
                               bool fp8 = false) {
  const WsLayout L = ws_layout(p.num_qrows, g.num_heads, g.head_dim, p.head_groups, p.max_parts,
                               p.max_tiles);
  if (!workspace || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return PA_ERR_WORKSPACE;
  if (g.num_qrows == 0 || g.num_seqs == 0) return PA_OK;
  const WsView ws = ws_view(workspace, L);
  PlanArgs a{};
  a.head_groups = p.head_groups;
  a.heads_per_group = p.heads_per_group;
  a.target_items = p.target_items;
  a.min_part_stages = 2;
  a.expand_prefill = (p.use_tc && !p.cascade) ? 0 : 1;
  a.tile_tokens = p.tile_tokens;
  a.cascade = p.cascade ? 1 : 0;
  a.num_sms = p.num_sms;
  TimedCall tm(s);
  tm.begin(PA_TK_PLAN);
  if ((sw ? launch_write_plan(g, a, ws, *sw, fp8, s) : launch_plan(g, a, ws, s)) != cudaSuccess)
    return PA_ERR_CUDA;
  tm.end(PA_TK_PLAN);
  if (p.use_tc) {
    tm.begin(PA_TK_TILES);
    if (launch_attn_tc(g, ws, p.tc_grid, s) != cudaSuccess) return PA_ERR_CUDA;
    tm.end(PA_TK_TILES);
  }
  tm.begin(PA_TK_DECODE);
  cudaError_t e = p.use_mma ? launch_attn_mma(g, ws, p.num_sms, p.heads_per_group,
                                              p.use_tc ? 1 : 0, s)
                            : launch_attn_generic(g, ws, p.num_sms, s);
  if (e != cudaSuccess) return PA_ERR_CUDA;
  tm.end(PA_TK_DECODE);
  tm.begin(PA_TK_MERGE);
  if (launch_merge(g, ws, p.num_sms, s) != cudaSuccess) return PA_ERR_CUDA;
  tm.end(PA_TK_MERGE);
  return PA_OK;
}

}  // namespace pa

using namespace pa;

extern "C" {

const char* pa_status_str(int status) {
  switch (status) {
    case PA_OK: return "ok";
    case PA_ERR_INVALID_ARG: return "invalid argument";
    case PA_ERR_UNSUPPORTED: return "unsupported configuration";
    case PA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case PA_ERR_CUDA: return "CUDA runtime error";
    case PA_ERR_DEVICE_OOB: return "device found out-of-range input (error bits set)";
    case PA_ERR_TIMEOUT: return "a bounded device wait gave up";
    default: return "unknown status";
  }
}

int pa_version(void) { return 101; }

pa_status pa_slot_mapping(const int32_t* block_tables, int32_t max_blocks_per_seq,
                          const int32_t* query_start_loc, const int32_t* seq_lens,
                          int32_t num_seqs, int64_t num_tokens, int32_t block_size,
                          int64_t num_blocks, int64_t* slot_mapping, int32_t* err_word,
                          void* stream) {
  if (num_seqs < 0 || num_tokens < 0 || max_blocks_per_seq < 0 || block_size < 1 ||
      num_blocks < 0)
    return PA_ERR_INVALID_ARG;
  if (num_seqs == 0 || num_tokens == 0) return PA_OK;
  if (!block_tables || !query_start_loc || !seq_lens || !slot_mapping) return PA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(max_blocks_per_seq) * block_size > (1LL << 30))
    return PA_ERR_UNSUPPORTED;
  cudaError_t e = launch_slot_mapping(block_tables, max_blocks_per_seq, query_start_loc, seq_lens,
                                      num_seqs, num_tokens, block_size, num_blocks, slot_mapping,
                                      err_word, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_cache_write(const void* k, const void* v, void* key_cache, void* value_cache,
                         const int64_t* slot_mapping, int64_t num_tokens,
                         const pa_cache_desc* cache, int32_t* err_word, void* stream) {
  pa_status st = check_cache(cache);
  if (st != PA_OK) return st;
  if (num_tokens < 0) return PA_ERR_INVALID_ARG;
  if (num_tokens == 0) return PA_OK;
  if (!k || !v || !key_cache || !value_cache || !slot_mapping) return PA_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(key_cache) || !aligned16(value_cache))
    return PA_ERR_INVALID_ARG;
  const int64_t row_elems = static_cast<int64_t>(cache->num_kv_heads) * cache->head_dim;
  cudaError_t e;
  if (cache->dtype == PA_FP8_E4M3)
    e = launch_cache_write_fp8(k, v, key_cache, value_cache, slot_mapping, num_tokens, row_elems,
                               cache->num_blocks * cache->block_size, cache->k_scale,
                               cache->v_scale, err_word, static_cast<cudaStream_t>(stream));
  else
    e = launch_cache_write(k, v, key_cache, value_cache, slot_mapping, num_tokens,
                           row_elems * elt_bytes(cache->dtype),
                           cache->num_blocks * cache->block_size, err_word,
                           static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_slot_mapping_cache_write(const void* k, const void* v, void* key_cache,
                                      void* value_cache, const int32_t* block_tables,
                                      int32_t max_blocks_per_seq, const int32_t* query_start_loc,
                                      const int32_t* seq_lens, int32_t num_seqs,
                                      int64_t num_tokens, const pa_cache_desc* cache,
                                      int64_t* slot_mapping, int32_t* err_word, void* stream) {
  pa_status st = check_cache(cache);
  if (st != PA_OK) return st;
  if (num_seqs < 0 || num_tokens < 0 || max_blocks_per_seq < 0) return PA_ERR_INVALID_ARG;
  if (!query_start_loc && num_tokens != num_seqs) return PA_ERR_INVALID_ARG;
  if (num_seqs == 0 || num_tokens == 0) return PA_OK;
  if (!k || !v || !key_cache || !value_cache || !block_tables || !seq_lens)
    return PA_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(key_cache) || !aligned16(value_cache))
    return PA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(max_blocks_per_seq) * cache->block_size > (1LL << 30))
    return PA_ERR_UNSUPPORTED;
  const int64_t row_elems = static_cast<int64_t>(cache->num_kv_heads) * cache->head_dim;
  const bool fp8 = cache->dtype == PA_FP8_E4M3;
  cudaError_t e = launch_slot_cache_write(
      k, v, key_cache, value_cache, block_tables, max_blocks_per_seq, query_start_loc, seq_lens,
      num_seqs, num_tokens, cache->block_size, cache->num_blocks, row_elems,
      fp8 ? 1 : elt_bytes(cache->dtype), fp8, cache->k_scale, cache->v_scale, slot_mapping,
      err_word, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_heads, int32_t max_blocks_per_seq,
                                const pa_cache_desc* cache) {
  if (check_attn_args(num_seqs, num_seqs, num_heads, max_blocks_per_seq, PA_F32, cache) != PA_OK)
    return 0;
  const AttnPlan p = make_plan(num_seqs, num_heads, max_blocks_per_seq, cache, true);
  if (!p.size_ok) return 0;
  return ws_layout(p.num_qrows, num_heads, cache->head_dim, p.head_groups, p.max_parts,
                   p.max_tiles)
      .total;
}

pa_status pa_decode(const void* q, const void* key_cache, const void* value_cache,
                    const int32_t* block_tables, const int32_t* seq_lens, float scale,
                    void* out, int32_t num_seqs, int32_t num_heads, int32_t max_blocks_per_seq,
                    int32_t out_dtype, const pa_cache_desc* cache, void* workspace,
                    size_t workspace_bytes, int32_t* err_word, void* stream) {
  pa_status st =
      check_attn_args(num_seqs, num_seqs, num_heads, max_blocks_per_seq, out_dtype, cache);
  if (st != PA_OK) return st;
  if (num_seqs == 0) return PA_OK;
  if (!q || !key_cache || !value_cache || !block_tables || !seq_lens || !out)
    return PA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(key_cache) || !aligned16(value_cache) || !aligned16(out))
    return PA_ERR_INVALID_ARG;
  const AttnPlan p = make_plan(num_seqs, num_heads, max_blocks_per_seq, cache, true);
  if (!p.size_ok) return PA_ERR_UNSUPPORTED;
  const AttnGeom g = make_geom(q, key_cache, value_cache, block_tables, seq_lens, nullptr, scale,
                               out, num_seqs, num_seqs, num_heads, max_blocks_per_seq, out_dtype,
                               cache, err_word);
  return run_attention(g, p, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

pa_status pa_decode_step(const void* q, const void* k, const void* v, void* key_cache,
                         void* value_cache, const int32_t* block_tables, const int32_t* seq_lens,
                         float scale, void* out, int32_t num_seqs, int32_t num_heads,
                         int32_t max_blocks_per_seq, int32_t out_dtype, const pa_cache_desc* cache,
                         int64_t* slot_mapping, void* workspace, size_t workspace_bytes,
                         int32_t* err_word, void* stream) {
  pa_status st =
      check_attn_args(num_seqs, num_seqs, num_heads, max_blocks_per_seq, out_dtype, cache);
  if (st != PA_OK) return st;
  if (num_seqs == 0) return PA_OK;
  if (!q || !k || !v || !key_cache || !value_cache || !block_tables || !seq_lens || !out)
    return PA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(key_cache) ||
      !aligned16(value_cache) || !aligned16(out))
    return PA_ERR_INVALID_ARG;
  const AttnPlan p = make_plan(num_seqs, num_heads, max_blocks_per_seq, cache, true);
  if (!p.size_ok) return PA_ERR_UNSUPPORTED;
  const AttnGeom g = make_geom(q, key_cache, value_cache, block_tables, seq_lens, nullptr, scale,
                               out, num_seqs, num_seqs, num_heads, max_blocks_per_seq, out_dtype,
                               cache, err_word);
  const bool fp8 = cache->dtype == PA_FP8_E4M3;
  const SlotWrite sw = make_slot_write(
      k, v, key_cache, value_cache, block_tables, max_blocks_per_seq, nullptr, seq_lens,
      num_seqs, num_seqs, cache->block_size, cache->num_blocks,
      static_cast<int64_t>(cache->num_kv_heads) * cache->head_dim,
      fp8 ? 1 : elt_bytes(cache->dtype), fp8, cache->k_scale, cache->v_scale, slot_mapping,
      err_word);
  return run_attention(g, p, workspace, workspace_bytes, static_cast<cudaStream_t>(stream), &sw,
                       fp8);
}

size_t pa_mixed_step_workspace_size(int32_t num_seqs, int64_t num_tokens, int32_t num_heads,
                                    int32_t max_blocks_per_seq, const pa_cache_desc* cache) {
  if (check_attn_args(num_seqs, num_tokens, num_heads, max_blocks_per_seq, PA_F32, cache) !=
      PA_OK)
    return 0;
  const AttnPlan p =
      make_plan(num_tokens, num_heads, max_blocks_per_seq, cache, true, num_seqs, true);
  if (!p.size_ok) return 0;
  return ws_layout(p.num_qrows, num_heads, cache->head_dim, p.head_groups, p.max_parts,
                   p.max_tiles)
      .total;
}

pa_status pa_mixed_step(const void* q, const void* key_cache, const void* value_cache,
                        const int32_t* block_tables, const int32_t* query_start_loc,
                        const int32_t* seq_lens, float scale, void* out, int32_t num_seqs,
                        int64_t num_tokens, int32_t num_heads, int32_t max_blocks_per_seq,
                        int32_t out_dtype, const pa_cache_desc* cache, void* workspace,
                        size_t workspace_bytes, int32_t* err_word, void* stream) {
  pa_status st =
      check_attn_args(num_seqs, num_tokens, num_heads, max_blocks_per_seq, out_dtype, cache);
  if (st != PA_OK) return st;
  if (num_seqs == 0 || num_tokens == 0) return PA_OK;
  if (!q || !key_cache || !value_cache || !block_tables || !query_start_loc || !seq_lens || !out)
    return PA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(key_cache) || !aligned16(value_cache) || !aligned16(out))
    return PA_ERR_INVALID_ARG;
  const AttnPlan p =
      make_plan(num_tokens, num_heads, max_blocks_per_seq, cache, true, num_seqs, true);
  if (!p.size_ok) return PA_ERR_UNSUPPORTED;
  const AttnGeom g = make_geom(q, key_cache, value_cache, block_tables, seq_lens,
                               query_start_loc, scale, out, num_seqs, num_tokens, num_heads,
                               max_blocks_per_seq, out_dtype, cache, err_word);
  return run_attention(g, p, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

pa_status pa_copy_blocks(void* key_cache, void* value_cache, const int64_t* block_mapping,
                         int64_t num_pairs, const pa_cache_desc* cache, int32_t* err_word,
                         void* stream) {
  pa_status st = check_cache(cache);
  if (st != PA_OK) return st;
  if (num_pairs < 0) return PA_ERR_INVALID_ARG;
  if (num_pairs == 0) return PA_OK;
  if (!key_cache || !value_cache || !block_mapping) return PA_ERR_INVALID_ARG;
  if (!aligned16(key_cache) || !aligned16(value_cache)) return PA_ERR_INVALID_ARG;
  const int64_t block_bytes = static_cast<int64_t>(cache->block_size) * cache->num_kv_heads *
                              cache->head_dim * pool_elt_bytes(cache->dtype);
  return launch_copy_blocks(key_cache, value_cache, block_mapping, num_pairs, block_bytes,
                            cache->num_blocks, err_word, device_num_sms(),
                            static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? PA_OK
             : PA_ERR_CUDA;
}

pa_status pa_slot_mapping_positions(const int32_t* block_tables, int32_t max_blocks_per_seq,
                                    int32_t num_seqs, const int32_t* token_req,
                                    const int64_t* positions, int64_t num_tokens,
                                    int32_t block_size, int64_t num_blocks,
                                    int64_t* slot_mapping, int32_t* err_word, void* stream) {
  if (num_seqs < 0 || num_tokens < 0 || max_blocks_per_seq < 0 || block_size < 1 ||
      num_blocks < 0)
    return PA_ERR_INVALID_ARG;
  if (num_tokens == 0) return PA_OK;
  if (!token_req || !positions || !slot_mapping || (num_seqs > 0 && !block_tables))
    return PA_ERR_INVALID_ARG;
  return launch_slot_positions(block_tables, max_blocks_per_seq, num_seqs, token_req, positions,
                               num_tokens, block_size, num_blocks, slot_mapping, err_word,
                               device_num_sms(), static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? PA_OK
             : PA_ERR_CUDA;
}

pa_status pa_rope_cos_sin_cache(float* cache, int32_t max_position, int32_t rotary_dim,
                                double theta, void* stream) {
  if (!cache || max_position <= 0 || rotary_dim <= 0 || (rotary_dim & 1) || !(theta > 0.0))
    return PA_ERR_INVALID_ARG;
  return launch_rope_table(cache, max_position, rotary_dim, theta, device_num_sms(),
                           static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? PA_OK
             : PA_ERR_CUDA;
}

pa_status pa_rope_cache_write(const void* q_in, const void* k, const void* v, int64_t q_stride,
                              int64_t kv_stride, void* q_out, void* key_cache, void* value_cache,
                              const int64_t* positions, const int64_t* slot_mapping,
                              const float* cos_sin_cache, int32_t max_position,
                              int32_t rotary_dim, int32_t neox, int64_t num_tokens,
                              int32_t num_heads, const pa_cache_desc* cache, int32_t* err_word,
                              void* stream) {
  pa_status st = check_cache(cache);
  if (st != PA_OK) return st;
  if (cache->dtype == PA_FP8_E4M3) return PA_ERR_UNSUPPORTED;
  if (num_tokens < 0 || num_heads < 1 || max_position < 1) return PA_ERR_INVALID_ARG;
  if (rotary_dim < 16 || rotary_dim % 16 || rotary_dim > cache->head_dim)
    return PA_ERR_UNSUPPORTED;
  const int64_t D = cache->head_dim;
  if (q_stride < num_heads * D || kv_stride < cache->num_kv_heads * D || q_stride % 8 ||
      kv_stride % 8)
    return PA_ERR_INVALID_ARG;
  if (num_tokens == 0) return PA_OK;
  if (!q_in || !k || !v || !q_out || !key_cache || !value_cache || !positions || !slot_mapping ||
      !cos_sin_cache)
    return PA_ERR_INVALID_ARG;
  if (!aligned16(q_in) || !aligned16(k) || !aligned16(v) || !aligned16(q_out) ||
      !aligned16(key_cache) || !aligned16(value_cache) || !aligned16(cos_sin_cache))
    return PA_ERR_INVALID_ARG;
  // q_out either is q_in (contiguous rows, rotated in place) or does not overlap it
  const uintptr_t qi = reinterpret_cast<uintptr_t>(q_in), qo = reinterpret_cast<uintptr_t>(q_out);
  const int64_t eb = elt_bytes(cache->dtype);
  const uintptr_t q_in_end = qi + static_cast<uintptr_t>(((num_tokens - 1) * q_stride + num_heads * D) * eb);
  const uintptr_t q_out_end = qo + static_cast<uintptr_t>(num_tokens * num_heads * D * eb);
  if (qi == qo ? q_stride != num_heads * D : (qo < q_in_end && qi < q_out_end))
    return PA_ERR_INVALID_ARG;
  RopeLaunch l{};
  l.q_in = q_in;
  l.k = k;
  l.v = v;
  l.q_stride = q_stride;
  l.kv_stride = kv_stride;
  l.q_out = q_out;
  l.kc = key_cache;
  l.vc = value_cache;
  l.positions = positions;
  l.slots = slot_mapping;
  l.cs = cos_sin_cache;
  l.max_position = max_position;
  l.rot = rotary_dim;
  l.neox = neox ? 1 : 0;
  l.num_tokens = num_tokens;
  l.hq = num_heads;
  l.hkv = cache->num_kv_heads;
  l.d = cache->head_dim;
  l.dtype = cache->dtype;
  l.num_slots = cache->num_blocks * cache->block_size;
  l.err = err_word;
  return launch_rope_cache_write(l, device_num_sms(), static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? PA_OK
             : PA_ERR_CUDA;
}

pa_status pa_kernel_timing_enable(int32_t enable) {
  std::lock_guard<std::mutex> lk(g_timer.mu);
  if (g_timer.on) {
    int prev = -1;
    cudaGetDevice(&prev);
    cudaSetDevice(g_timer.device);
    for (cudaEvent_t& e : g_timer.ev) {
      if (e) cudaEventDestroy(e);
      e = nullptr;
    }
    cudaSetDevice(prev);
    g_timer.on = false;
    g_timer.pending = false;
  }
  if (!enable) return PA_OK;
  if (cudaGetDevice(&g_timer.device) != cudaSuccess) return PA_ERR_CUDA;
  for (cudaEvent_t& e : g_timer.ev) {
    if (cudaEventCreate(&e) != cudaSuccess) {
      for (cudaEvent_t& f : g_timer.ev) {
        if (f) cudaEventDestroy(f);
        f = nullptr;
      }
      return PA_ERR_CUDA;
    }
  }
  g_timer.on = true;
  return PA_OK;
}

pa_status pa_kernel_timing_read(float* ms) {
  std::lock_guard<std::mutex> lk(g_timer.mu);
  if (!ms || !g_timer.on || !g_timer.pending) return PA_ERR_INVALID_ARG;
  g_timer.pending = false;
  if (g_timer.failed) return PA_ERR_CUDA;
  for (int k = 0; k < PA_TIMED_KERNELS; ++k) {
    ms[k] = -1.f;
    if (!g_timer.launched[k]) continue;
    if (cudaEventSynchronize(g_timer.ev[2 * k + 1]) != cudaSuccess ||
        cudaEventElapsedTime(&ms[k], g_timer.ev[2 * k], g_timer.ev[2 * k + 1]) != cudaSuccess)
      return PA_ERR_CUDA;
  }
  return PA_OK;
}

pa_status pa_read_error(int32_t* err_word, int32_t* host_bits, void* stream) {
  if (!err_word || !host_bits) return PA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t h = 0;
  if (cudaMemcpyAsync(&h, err_word, sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return PA_ERR_CUDA;
  if (cudaMemsetAsync(err_word, 0, sizeof(int32_t), s) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return PA_ERR_CUDA;
  *host_bits = h;
  if (h & PA_ERRBIT_TIMEOUT) return PA_ERR_TIMEOUT;
  return h ? PA_ERR_DEVICE_OOB : PA_OK;
}

}  // extern "C"
