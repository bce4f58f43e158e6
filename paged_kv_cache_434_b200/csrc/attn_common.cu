// attn_common.cu -- work planner, CUDA-core attention kernel and the split-KV
// log-sum-exp merge, shared by pa_decode and pa_mixed_step.
//
// What is computed ("AI Infra入门干货总结：大模型是如何高效推理的", section
// "Attention (FlashAttention, Scaled Dot-Product Attention)"): for every query
// row r of request b and query head h, with kv = h / (Hq / Hkv),
//     o = sum_j softmax_j(scale * <q_rh, k_j,kv>) v_j,kv   over j < key_len(r)
// where key_len(r) = seq_len_b - q_b + i + 1 for the i-th new token of b
// (causal inside the chunk, full over the cached prefix).  K/V row j lives in
// physical block block_tables[b][j / block_size] at offset j % block_size.
//
// Flash-Decoding ("总结": split the KV axis for SM utilisation, re-normalise
// across pieces with log-sum-exp): the key range of a row is cut into
// partitions of P keys; each (row, head group, partition) is one work item
// producing (m, l, o) with the online softmax (running max m, running sum l,
// rescale by exp(m_old - m_new), as in the ursb.me Field Note blurb); a second
// pass merges the partitions: O = sum_k 2^(m_k - M) o_k / sum_k 2^(m_k - M) l_k.
// Scores are kept in log2 units (scale * log2 e folded in) so exp becomes ex2.
#include <cuda_bf16.h>

#include <cmath>
#include <type_traits>

#include "internal.h"
#include "ptx.cuh"
#include "slot_write.cuh"

namespace pa {

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

WsLayout ws_layout(int64_t num_qrows, int num_heads, int head_dim, int head_groups,
                   int64_t max_parts, int64_t max_tiles) {
  WsLayout L{};
  L.num_qrows = num_qrows;
  L.max_parts = max_parts;
  L.max_items = num_qrows * head_groups * max_parts;
  L.max_tiles = max_tiles;
  size_t off = 0;
  L.ctrl = off;
  off = align_up(off + 64 * sizeof(int32_t), 256);
  L.qrow_info = off;
  off = align_up(off + num_qrows * sizeof(int4), 256);
  L.nparts = off;
  off = align_up(off + num_qrows * sizeof(int32_t), 256);
  L.qrow_bad = off;
  off = align_up(off + num_qrows * sizeof(int32_t), 256);
  L.merge_rows = off;
  off = align_up(off + num_qrows * sizeof(int32_t), 256);
  L.items = off;
  off = align_up(off + L.max_items * sizeof(int4), 256);
  L.part_ml = off;
  off = align_up(off + num_qrows * num_heads * max_parts * sizeof(float2), 256);
  L.part_o = off;
  off = align_up(off + num_qrows * num_heads * max_parts * head_dim * sizeof(float), 256);
  L.tiles = off;
  off = align_up(off + max_tiles * sizeof(int4), 256);
  L.total = off;
  return L;
}

WsView ws_view(void* base, const WsLayout& L) {
  char* p = static_cast<char*>(base);
  WsView v;
  v.ctrl = reinterpret_cast<int32_t*>(p + L.ctrl);
  v.qrow_info = reinterpret_cast<int4*>(p + L.qrow_info);
  v.nparts = reinterpret_cast<int32_t*>(p + L.nparts);
  v.qrow_bad = reinterpret_cast<int32_t*>(p + L.qrow_bad);
  v.merge_rows = reinterpret_cast<int32_t*>(p + L.merge_rows);
  v.items = reinterpret_cast<int4*>(p + L.items);
  v.part_ml = reinterpret_cast<float2*>(p + L.part_ml);
  v.part_o = reinterpret_cast<float*>(p + L.part_o);
  v.tiles = reinterpret_cast<int4*>(p + L.tiles);
  v.max_parts = L.max_parts;
  v.max_items = L.max_items;
  v.max_tiles = L.max_tiles;
  return v;
}

// ======================================================================= planner
// One CTA of 1024 threads, all loops parallel:
//   0. every row starts "unassigned" (left unwritten);
//   1. requests in parallel: validation (error bits), rows of small requests
//      filled inline, larger per-row requests and prefill-tile requests listed;
//   1b. listed per-row requests: their rows filled cooperatively;
//   1c. prefill-tile requests: block table validated cooperatively, tiles
//      counted per 128-key-tile bin;
//   the partition length P is then chosen so that the item count is near
//   target_items and no row needs more than max_parts partitions;
//   2./3. rows in parallel: items counted, scanned, written; rows whose result
//      the merge pass writes (0 or > 1 partitions) listed;
//   4. tiles scattered longest-first (descending bin order).
constexpr int kPlanThreads = 1024;
constexpr int kMaxPrefill = 512;  // prefill requests served by tensor-core tiles per call
constexpr int kTileBins = 2048;   // longest-first ordering of tiles by 128-key tile count
constexpr int kInlineRows = 8;    // requests with at most this many rows: one thread
constexpr int kMaxBig = 1024;     // larger per-row requests: whole CTA, one at a time
constexpr int kInlineItems = 32;  // rows with more work items: written by the whole CTA

__device__ __forceinline__ int tile_bin(int n_kv) { return n_kv < kTileBins ? n_kv : kTileBins - 1; }

__device__ __forceinline__ void request_rows(const AttnGeom& g, int b, int& r0, int& q_b) {
  if (g.query_start_loc) {
    r0 = g.query_start_loc[b];
    q_b = g.query_start_loc[b + 1] - r0;
  } else {
    r0 = b;
    q_b = 1;
  }
}

__device__ __forceinline__ void fill_row(const AttnGeom& g, const WsView& ws, bool decode_mode,
                                         int b, int r, int i, int q_b, int L,
                                         long long& units_sum, int& units_max) {
  const int key_len = decode_mode ? L : L - q_b + i + 1;
  ws.qrow_info[r] = make_int4(b, key_len, 1, 0);
  const int units = (key_len + kStageTokens - 1) / kStageTokens;
  units_sum += units;
  units_max = max(units_max, units);
}

// Longest run of leading block-table entries shared by every request (decode
// batches), limited so that each request keeps at least one key of its own.
// Cooperative over the CTA: column 0 alone first (most batches already differ
// there), then as many columns at once as keeps 16 loads in flight per thread.
__device__ int shared_prefix_blocks(const AttnGeom& g, int max_cols, int* s_bad) {
  constexpr int kPer = 16;
  if (threadIdx.x == 0) *s_bad = max_cols;
  __syncthreads();
  int c0 = 0, width = 1;
  while (c0 < max_cols) {
    const int c1 = min(c0 + width, max_cols);
    const int pairs = (c1 - c0) * g.num_seqs;
    int v[kPer], ref[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int idx = threadIdx.x + u * blockDim.x;
      v[u] = ref[u] = 0;
      if (idx < pairs) {  // consecutive threads: consecutive columns of one table row
        const int w = c1 - c0;
        const int j = c0 + idx % w, b = idx / w;
        v[u] = g.block_tables[static_cast<int64_t>(b) * g.max_blocks + j];
        ref[u] = g.block_tables[j];
      }
    }
    int first = 0x7fffffff;  // first differing column this thread saw
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int idx = threadIdx.x + u * blockDim.x;
      if (idx < pairs && v[u] != ref[u]) first = min(first, c0 + idx % (c1 - c0));
    }
    first = __reduce_min_sync(0xffffffffu, first);  // one shared atomic per warp
    if ((threadIdx.x & 31) == 0 && first != 0x7fffffff) atomicMin(s_bad, first);
    __syncthreads();
    // later atomics only lower s_bad to columns >= c1, so every thread sees the
    // same answer to this test
    if (*s_bad < c1) break;
    c0 = c1;
    width = max(1, kPer * static_cast<int>(blockDim.x) / max(g.num_seqs, 1));
  }
  const int r = *s_bad;
  __syncthreads();
  return r;
}

// Exclusive prefix of v over the CTA's threads in thread order; *total gets
// the sum.  s_scan holds 33 values.
template <typename T>
__device__ __forceinline__ T block_exclusive_scan(T v, T* s_scan, T* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  T incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const T n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) s_scan[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const T w = s_scan[lane];
    T wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const T n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    s_scan[lane] = wi - w;
    if (lane == 31) s_scan[32] = wi;
  }
  __syncthreads();
  *total = s_scan[32];
  return s_scan[warp] + incl - v;
}

// Decode batches of up to kFastRows requests, in one pass: each thread holds
// up to kFastPerThread consecutive requests' lengths in registers, so the
// plan needs no re-reads of the workspace and few barriers.
//   * Shared prefix (batches of >= kCascadeMinSeqs requests whose tables all
//     start with the same block): the longest common run of leading blocks is
//     found by comparing (request, column) pairs against row 0; a run of
//     >= kCascadeMinPrefix tokens is attended by tensor-core tiles (listed
//     here) and the rows keep only their suffix.
//   * Partitions in decreasing sizes: work W = stages x head groups; each row
//     is cut into big pieces of Pb ~ 0.4 W / SMs stages (within 80 % of its
//     stages, whole pieces only) and small pieces of Ps ~ 0.05 W / SMs for
//     the rest: about two big and four small pieces per SM overall.
//     The item list holds every big piece before every small one, and the
//     partition kernel takes items in list order from a global counter: the
//     big pieces spread the work, the small ones even out the end, whatever
//     the SMs' start times and streaming rates.  Rows that would need more
//     pieces than the partial slots hold fall back to uniform pieces.
//   * Items are written by the whole CTA: item i finds its row by binary
//     search over the rows' first items in shared memory.
constexpr int kFastPerThread = 4;
constexpr int kFastRows = kPlanThreads * kFastPerThread;
constexpr int kMinSmallStages = 8;

// The pieces of a row of n stages: nb big ones of pb stages (whole pieces
// within 80 % of the row), then ns small ones of ps.  A row that would need
// more than `cap` pieces gets larger pieces of its own (at most cap / 2 big
// and the rest small).  The same arithmetic wherever a row's pieces are
// counted or listed.
struct RowPieces {
  int pb, nb, ps, ns;
};
// (one out-of-line copy: the planner runs it cold once per call, and six inlined
// copies cost more instruction fetches than the calls)
__device__ __noinline__ RowPieces row_pieces(int n, int Pb, int Ps, int cap) {
  RowPieces p;
  if (cap < 2) {  // one piece per row
    p.pb = max(n, 1), p.nb = n > 0 ? 1 : 0, p.ps = 1, p.ns = 0;
    return p;
  }
  const int big = static_cast<int>(static_cast<float>(n) * 0.8f);
  p.pb = Pb;
  p.nb = big / Pb;
  p.ps = Ps;
  p.ns = (n - p.nb * Pb + Ps - 1) / Ps;
  if (p.nb + p.ns <= cap) return p;
  const int hb = cap / 2, hs = cap - hb;
  p.pb = max(Pb, (big + hb - 1) / hb);
  p.nb = big / p.pb;
  const int rem = n - p.nb * p.pb;
  p.ps = max(Ps, (rem + hs - 1) / hs);
  p.ns = (rem + p.ps - 1) / p.ps;
  return p;
}

__device__ void plan_decode_fast(const AttnGeom& g, const PlanArgs& a, const WsView& ws,
                                 int* s_rowpos, int* s_scan,
                                 int* s_max, int* s_P, int* s_merge,
                                 int* s_merge_big) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int B = g.num_seqs;
  const int per = (B + kPlanThreads - 1) / kPlanThreads;  // <= kFastPerThread
  const int r0 = tid * per;
  const int64_t max_keys = static_cast<int64_t>(g.max_blocks) * g.block_size;
  const bool look_shared = a.cascade && B >= kCascadeMinSeqs && g.max_blocks > 0;
  const int ref0 = look_shared ? g.block_tables[0] : 0;
  int L[kFastPerThread], c0[kFastPerThread];
#pragma unroll
  for (int k = 0; k < kFastPerThread; ++k) {
    const int r = r0 + k;
    L[k] = 0;
    c0[k] = ref0;
    if (k < per && r < B) {
      L[k] = g.seq_lens[r];
      if (look_shared) c0[k] = g.block_tables[static_cast<int64_t>(r) * g.max_blocks];
    }
  }
  bool same = true, all_ok = true;
  int min_len = 0x7fffffff;
#pragma unroll
  for (int k = 0; k < kFastPerThread; ++k) {
    if (k >= per || r0 + k >= B) continue;
    const bool ok = L[k] >= 0 && L[k] <= max_keys;
    all_ok &= ok;
    same &= c0[k] == ref0;
    if (ok) min_len = min(min_len, L[k]);
  }

  // Shared prefix: the (request, column) pairs are compared with row 0 column
  // chunk by column chunk -- each thread loads both entries of its pairs, 16
  // pairs per thread in a chunk, the chunks growing fourfold -- until a chunk
  // holds a mismatch (the tables are often cold: one round trip per chunk).
  // The run is limited so that each request keeps at least one key of its own.
  __shared__ int s_first, s_minlen;
  int prefix_blocks = 0;
  // (the shortest row is looked up only when every table starts with row 0's
  // first block: most batches leave after one barrier)
  if (look_shared && __syncthreads_and(same && all_ok)) {
    const int w_min = __reduce_min_sync(0xffffffffu, min_len);
    if (tid == 0) s_minlen = 0x7fffffff;
    __syncthreads();
    if (lane == 0) atomicMin(&s_minlen, w_min);
    __syncthreads();
    if (s_minlen > kCascadeMinPrefix && s_minlen != 0x7fffffff) {
      const int max_cols = min((s_minlen - 1) / g.block_size, g.max_blocks);
      if (tid == 0) s_first = max_cols;
      __syncthreads();
      constexpr int kPairs = 8;  // pairs per thread and pass
      // a chunk's pairs are laid out as B rows x 2^lw columns (the chunk's width
      // rounded up to a power of two), so that a pair's request and column are
      // a shift and a mask of its index
      int W = max(1, 2 * kPairs * kPlanThreads / B);  // columns per chunk (two passes)
      for (int cb = 1; cb < max_cols; cb += W, W = min(W * 4, 1 << 24)) {
        const int ce = min(cb + W, max_cols);
        const int lw = 32 - __clz(max(ce - cb - 1, 0));  // 2^lw >= ce - cb
        const int64_t slots = static_cast<int64_t>(B) << lw;
        int mine = 0x7fffffff;
        for (int64_t i0 = 0; i0 < slots; i0 += kPairs * kPlanThreads) {
          // every load is issued unconditionally (addresses clamped into the
          // table, pairs outside the chunk masked afterwards), so that all of
          // a thread's loads are in flight at once
          int v[kPairs], ref[kPairs];
#pragma unroll
          for (int k = 0; k < kPairs; ++k) {
            const int64_t idx = i0 + tid + static_cast<int64_t>(k) * kPlanThreads;
            const int j = min(cb + static_cast<int>(idx & ((1 << lw) - 1)), ce - 1);
            const int64_t b = min(idx >> lw, static_cast<int64_t>(B - 1));
            v[k] = __ldg(g.block_tables + b * g.max_blocks + j);
            ref[k] = __ldg(g.block_tables + j);
          }
#pragma unroll
          for (int k = 0; k < kPairs; ++k) {
            const int64_t idx = i0 + tid + static_cast<int64_t>(k) * kPlanThreads;
            const int j = cb + static_cast<int>(idx & ((1 << lw) - 1));
            if ((idx >> lw) < B && j < ce && v[k] != ref[k]) mine = min(mine, j);
          }
        }
        mine = __reduce_min_sync(0xffffffffu, mine);
        if (lane == 0 && mine != 0x7fffffff) atomicMin(&s_first, mine);
        __syncthreads();
        if (s_first < ce) break;  // s_first only falls: every thread sees the same answer
      }
      const int pb = s_first;
      if (pb * g.block_size >= kCascadeMinPrefix) prefix_blocks = pb;
    }
  }
  const int prefix = prefix_blocks * g.block_size;

  // invalid requests: error bits, rows left unwritten (L = -1 from here on);
  // the stage total only sizes the pieces, so it is summed in float
  float units_sum = 0.f;
  int units_max = 0;
#pragma unroll
  for (int k = 0; k < kFastPerThread; ++k) {
    if (k >= per || r0 + k >= B) continue;
    int bits = 0;
    if (L[k] < 0) bits |= PA_ERRBIT_QUERY_TOO_LONG;
    if (L[k] > max_keys) bits |= PA_ERRBIT_SEQ_TOO_LONG;
    if (bits) {
      if (g.err_word) atomicOr(g.err_word, bits);
      L[k] = -1;
      continue;
    }
    const int units = (L[k] - prefix + kStageTokens - 1) / kStageTokens;
    units_sum += static_cast<float>(units);
    units_max = max(units_max, units);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) units_sum += __shfl_xor_sync(0xffffffffu, units_sum, o);
  units_max = __reduce_max_sync(0xffffffffu, units_max);
  __shared__ float s_fsum[32];
  if (lane == 0) {
    s_fsum[warp] = units_sum;
    s_max[warp] = units_max;
  }
  __shared__ int s_Pb, s_Ps;
  __syncthreads();
  // partial slots a row's own pieces may use (the last kMaxPrefixChunks are
  // the shared prefix's, when there is one)
  const int cap = static_cast<int>(
      max(1LL, static_cast<long long>(ws.max_parts) - (prefix > 0 ? kMaxPrefixChunks : 0)));
  if (warp == 0) {
    float total = s_fsum[lane];
#pragma unroll
    for (int o = 16; o; o >>= 1) total += __shfl_xor_sync(0xffffffffu, total, o);
    const int mx = __reduce_max_sync(0xffffffffu, s_max[lane]);
    if (lane == 0) {
      // the sizes are heuristics: single precision with fast divisions (no
      // double or 64-bit division routines in this once-per-call, cold code)
      const float work = total * static_cast<float>(a.head_groups);
      const float by_target = ceilf(__fdividef(work, static_cast<float>(max(a.target_items, 1))));
      const int by_cap = (mx + cap - 1) / cap;
      const float P = fmaxf(static_cast<float>(a.min_part_stages),
                            fmaxf(by_target, static_cast<float>(by_cap)));
      *s_P = static_cast<int>(fminf(fmaxf(P, 1.f), 1e9f));
      // big pieces: 80 % of the work, about two per SM; small pieces: the
      // rest, about four per SM
      const float per_sm = __fdividef(work, static_cast<float>(max(a.num_sms, 1)));
      s_Pb = static_cast<int>(fminf(fmaxf(0.4f * per_sm, static_cast<float>(a.min_part_stages)), 1e9f));
      // (at least kMinSmallStages: smaller pieces cost more, in the merge and
      // in each item's start, than they gain at the end)
      s_Ps = static_cast<int>(fminf(fmaxf(0.05f * per_sm, static_cast<float>(kMinSmallStages)),
                                    static_cast<float>(s_Pb)));
      *s_merge = 0;
      *s_merge_big = 0;
    }
  }
  __syncthreads();
  // pieces per row: whole big pieces within 80 % of its stages, small pieces
  // for the rest
  const int Pb = s_Pb, Ps = s_Ps;
  int nb[kFastPerThread], ns[kFastPerThread];
#pragma unroll
  for (int k = 0; k < kFastPerThread; ++k) {
    nb[k] = ns[k] = 0;
    if (k >= per || r0 + k >= B || L[k] < 0) continue;
    const RowPieces rp = row_pieces((L[k] - prefix + kStageTokens - 1) / kStageTokens, Pb, Ps, cap);
    nb[k] = rp.nb;
    ns[k] = rp.ns;
  }
  // item positions: every big piece first, then every small piece
  int my_big = 0, my_small = 0;
#pragma unroll
  for (int k = 0; k < kFastPerThread; ++k) {
    my_big += nb[k] * a.head_groups;
    my_small += ns[k] * a.head_groups;
  }
  // both offsets from one scan: big counts in the high 32 bits, small in the low
  __shared__ unsigned long long s_scan64[33];
  unsigned long long both = 0;
  const unsigned long long pre = block_exclusive_scan<unsigned long long>(
      (static_cast<unsigned long long>(my_big) << 32) | static_cast<unsigned long long>(my_small),
      s_scan64, &both);
  const int n_big = static_cast<int>(both >> 32), n_small = static_cast<int>(both & 0xffffffffull);
  const int big0 = static_cast<int>(pre >> 32), small0 = static_cast<int>(pre & 0xffffffffull);
  // big items, spread over the CTA by binary search over the rows' first items
  {
    int pos = big0;
#pragma unroll
    for (int k = 0; k < kFastPerThread; ++k) {
      const int r = r0 + k;
      if (k >= per || r >= B) continue;
      s_rowpos[r] = pos;
      pos += nb[k] * a.head_groups;
    }
    if (tid == 0) s_rowpos[B] = n_big;
    __syncthreads();
    for (int i = tid; i < n_big; i += kPlanThreads) {
      int lo = 0, hi = B;  // the row r with s_rowpos[r] <= i < s_rowpos[r + 1]
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_rowpos[mid] <= i) lo = mid;
        else hi = mid;
      }
      const int k = i - s_rowpos[lo], piece = k / a.head_groups;
      const int n = (g.seq_lens[lo] - prefix + kStageTokens - 1) / kStageTokens;
      const RowPieces rp = row_pieces(n, Pb, Ps, cap);
      ws.items[i] = make_int4(lo, (k % a.head_groups) | (piece << kItemPartShift), rp.pb,
                              piece * rp.pb);
    }
    __syncthreads();
  }
  // small items, after them
  {
    int pos = small0;
#pragma unroll
    for (int k = 0; k < kFastPerThread; ++k) {
      const int r = r0 + k;
      if (k >= per || r >= B) continue;
      s_rowpos[r] = pos;
      pos += ns[k] * a.head_groups;
    }
    if (tid == 0) s_rowpos[B] = n_small;
    __syncthreads();
    for (int i = tid; i < n_small; i += kPlanThreads) {
      int lo = 0, hi = B;
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_rowpos[mid] <= i) lo = mid;
        else hi = mid;
      }
      const int row = lo, k = i - s_rowpos[row], piece = k / a.head_groups;
      // the row's piece sizes, from the owning thread's registers, are not at
      // hand here: recompute them from its length
      const int n = (g.seq_lens[row] - prefix + kStageTokens - 1) / kStageTokens;
      const RowPieces rp = row_pieces(n, Pb, Ps, cap);
      ws.items[n_big + i] =
          make_int4(row, (k % a.head_groups) | ((rp.nb + piece) << kItemPartShift), rp.ps,
                    rp.nb * rp.pb + piece * rp.ps);
    }
  }
  // shared-prefix tiles: groups of tile_tokens requests x one KV head x a
  // chunk of the prefix keys, at most one tile per two SMs, so that the suffix
  // partitions start at once on the SMs the tiles leave free (longer tiles on
  // half the SMs measured 11 % faster than one wave of shorter tiles)
  int prefix_chunks = 0, n_tiles = 0;
  if (prefix > 0) {
    const int per_tile = a.tile_tokens;
    const int groups = (B + per_tile - 1) / per_tile;
    const int kv_tiles = (prefix + 127) / 128;
    const int base = groups * g.num_kv_heads;
    const int want = min(min(kMaxPrefixChunks, kv_tiles), max(1, a.num_sms / (2 * base)));
    const int per_chunk = (kv_tiles + want - 1) / want;
    prefix_chunks = (kv_tiles + per_chunk - 1) / per_chunk;  // no empty chunk
    n_tiles = static_cast<int>(min(static_cast<int64_t>(base) * prefix_chunks, ws.max_tiles));
    for (int idx = tid; idx < n_tiles; idx += kPlanThreads) {
      const int c = idx / base, rest = idx % base;
      const int grp = rest / g.num_kv_heads, hk = rest % g.num_kv_heads;
      ws.tiles[idx] = make_int4(grp * per_tile, hk, min(per_tile, B - grp * per_tile), c);
    }
  }
  // rows: info, partition counts, and the merge pass's list (rows with no key
  // get zeros there; rows of more than one partition are merged)
#pragma unroll
  for (int k = 0; k < kFastPerThread; ++k) {
    const int r = r0 + k;
    if (k >= per || r >= B) continue;
    const int n = L[k] < 0 ? -1 : nb[k] + ns[k] + (prefix > 0 ? prefix_chunks : 0);
    ws.qrow_bad[r] = 0;
    ws.nparts[r] = n;
    ws.qrow_info[r] = n >= 0 ? make_int4(r, L[k], 1, prefix) : make_int4(-1, 0, 0, 0);
    if (n > kMergeWarpParts) ws.merge_rows[g.num_qrows - 1 - atomicAdd(s_merge_big, 1)] = r;
    else if (n >= 0 && n != 1) ws.merge_rows[atomicAdd(s_merge, 1)] = r;
  }
  __syncthreads();
  if (tid == 0) {
    ws.ctrl[0] = 0;
    ws.ctrl[1] = n_big + n_small;
    ws.ctrl[2] = Pb * kStageTokens;  // (informative: items carry their own length)
    ws.ctrl[3] = 0;
    ws.ctrl[4] = n_tiles;
    ws.ctrl[5] = *s_merge;
    ws.ctrl[6] = prefix;
    ws.ctrl[7] = prefix_chunks;
    ws.ctrl[8] = prefix > 0 ? a.num_sms : 0;  // every tile CTA works
    ws.ctrl[9] = *s_merge_big;
  }
}

// The planner: one CTA of kPlanThreads threads.
__device__ __forceinline__ void plan_body(const AttnGeom& g, const PlanArgs& a, const WsView& ws) {
  __shared__ long long s_sum[32];
  __shared__ int s_max[32];
  __shared__ int s_scan[32];
  __shared__ int s_P, s_merge, s_merge_big, s_npref, s_nbig, s_badpref, s_minL, s_nbad, s_pbad,
      s_ntc;
  __shared__ unsigned long long s_tile_kv;
  __shared__ int s_pref[kMaxPrefill];
  __shared__ int s_big[kMaxBig];
  __shared__ int s_bigpos[kMaxBig];
  __shared__ int s_hist[kTileBins];
  __shared__ int s_rowpos[kFastRows + 1];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool decode_mode = g.query_start_loc == nullptr;
  const int64_t max_keys = static_cast<int64_t>(g.max_blocks) * g.block_size;

  if (decode_mode && g.num_seqs <= kFastRows && g.num_qrows == g.num_seqs) {
    __shared__ int s_scan33[33];
    plan_decode_fast(g, a, ws, s_rowpos, s_scan33, s_max, &s_P,
                     &s_merge, &s_merge_big);
    return;
  }

  // 0. rows no request covers stay unwritten
  for (int r = tid; r < g.num_qrows; r += kPlanThreads) {
    ws.nparts[r] = -1;
    ws.qrow_bad[r] = 0;
    ws.qrow_info[r] = make_int4(-1, 0, 0, 0);
  }
  if (tid == 0) {
    s_merge = 0;
    s_merge_big = 0;
    s_npref = 0;
    s_nbig = 0;
    s_minL = 0x7fffffff;
    s_nbad = 0;
    s_tile_kv = 0;
  }
  for (int i = tid; i < kTileBins; i += kPlanThreads) s_hist[i] = 0;
  __syncthreads();

  // 1. requests
  long long my_units = 0;
  int my_max = 0;
  for (int b = tid; b < g.num_seqs; b += kPlanThreads) {
    int r0, q_b;
    request_rows(g, b, r0, q_b);
    const int L = g.seq_lens[b];
    if (r0 < 0 || r0 > g.num_qrows) {
      if (g.err_word) atomicOr(g.err_word, PA_ERRBIT_QUERY_TOO_LONG);
      continue;
    }
    int bits = 0;
    if (decode_mode) {
      if (L < 0) bits |= PA_ERRBIT_QUERY_TOO_LONG;
    } else if (q_b < 0 || q_b > L) {
      bits |= PA_ERRBIT_QUERY_TOO_LONG;
    }
    if (L > max_keys) bits |= PA_ERRBIT_SEQ_TOO_LONG;
    if (bits) {
      if (g.err_word) atomicOr(g.err_word, bits);
      atomicAdd(&s_nbad, 1);
      continue;  // its rows stay unwritten
    }
    if (decode_mode && a.cascade) {
      // units as if no prefix is shared; recounted below if one is
      atomicMin(&s_minL, L);
      ws.qrow_info[r0] = make_int4(b, L, 1, 0);
      const int units = (L + kStageTokens - 1) / kStageTokens;
      my_units += units;
      my_max = max(my_max, units);
      continue;
    }
    const bool tile = !(decode_mode || q_b == 1 || a.expand_prefill);
    if (tile) {
      const int slot = atomicAdd(&s_npref, 1);
      if (slot < kMaxPrefill) {
        s_pref[slot] = b;
        continue;
      }  // beyond the tile list's capacity: per-row path below
    }
    const int nrows = min(q_b, g.num_qrows - r0);
    if (nrows > kInlineRows) {
      const int slot = atomicAdd(&s_nbig, 1);
      if (slot < kMaxBig) {
        s_big[slot] = b;
        continue;
      }
    }
    for (int i = 0; i < nrows; ++i)
      fill_row(g, ws, decode_mode, b, r0 + i, i, q_b, L, my_units, my_max);
  }
  __syncthreads();

  // 1b. large per-row requests, cooperatively
  const int nbig = min(s_nbig, kMaxBig);
  for (int k = 0; k < nbig; ++k) {
    const int b = s_big[k];
    int r0, q_b;
    request_rows(g, b, r0, q_b);
    const int L = g.seq_lens[b];
    const int nrows = min(q_b, g.num_qrows - r0);
    for (int i = tid; i < nrows; i += kPlanThreads)
      fill_row(g, ws, decode_mode, b, r0 + i, i, q_b, L, my_units, my_max);
  }

  // 1c. prefill requests on tensor-core tiles: block tables validated
  // cooperatively, rows marked, tiles counted per bin
  const int npref = min(s_npref, kMaxPrefill);
  int n_tiles_total = 0;
  unsigned long long my_tile_kv = 0;  // summed per warp below (one shared atomic per warp)
  for (int pi = 0; pi < npref; ++pi) {
    const int b = s_pref[pi];
    const int L = g.seq_lens[b];
    const int nblk = (L + g.block_size - 1) / g.block_size;
    if (tid == 0) s_badpref = 0;
    __syncthreads();
    const int32_t* table = g.block_tables + static_cast<int64_t>(b) * g.max_blocks;
    for (int k = tid; k < nblk; k += kPlanThreads) {
      const int phys = table[k];
      if (phys < 0 || phys >= g.num_blocks) s_badpref = 1;
    }
    __syncthreads();
    int r0, q_b;
    request_rows(g, b, r0, q_b);
    if (s_badpref) {
      if (tid == 0) {
        s_pref[pi] = -1;
        if (g.err_word) atomicOr(g.err_word, PA_ERRBIT_BLOCK_OOB);
      }
    } else {
      for (int i = tid; i < q_b && r0 + i < g.num_qrows; i += kPlanThreads)
        ws.nparts[r0 + i] = -2;  // written by the tile kernel
      const int ntb = (q_b + a.tile_tokens - 1) / a.tile_tokens;
      for (int idx = tid; idx < ntb * g.num_kv_heads; idx += kPlanThreads) {
        const int tb = idx / g.num_kv_heads;
        const int last = min((tb + 1) * a.tile_tokens, q_b) - 1;
        const int n_kv = (L - q_b + last) / 128 + 1;
        atomicAdd(&s_hist[tile_bin(n_kv)], 1);
        // (query tile, key tile) products of this item: one or two query tiles
        const int halves = last + 1 - tb * a.tile_tokens > a.tile_tokens / 2 ? 2 : 1;
        my_tile_kv += static_cast<unsigned long long>(n_kv * halves);
      }
      n_tiles_total += ntb * g.num_kv_heads;
    }
    __syncthreads();
  }

  if (npref > 0) {
#pragma unroll
    for (int o = 16; o; o >>= 1) my_tile_kv += __shfl_xor_sync(0xffffffffu, my_tile_kv, o);
    if (lane == 0 && my_tile_kv) atomicAdd(&s_tile_kv, my_tile_kv);
  }

  // 1d. decode cascade: a prefix of blocks shared by every request is attended
  // once by tensor-core tiles; each row keeps only its own suffix
  int prefix_tokens = 0, prefix_chunks = 0;
  if (decode_mode && a.cascade) {
    __syncthreads();
    if (s_nbad == 0 && g.num_seqs >= kCascadeMinSeqs && s_minL > kCascadeMinPrefix) {
      const int max_cols = min((s_minL - 1) / g.block_size, g.max_blocks);
      const int pb = shared_prefix_blocks(g, max_cols, &s_pbad);
      if (pb * g.block_size >= kCascadeMinPrefix) prefix_tokens = pb * g.block_size;
    }
    if (prefix_tokens > 0) {
      // rows keep only their suffix (thread tid filled rows tid, tid + 1024, ...)
      my_units = 0;
      my_max = 0;
      for (int r = tid; r < g.num_qrows; r += kPlanThreads) {
        int4 info = ws.qrow_info[r];
        if (info.z == 0) continue;
        info.w = prefix_tokens;
        ws.qrow_info[r] = info;
        const int units = (info.y - prefix_tokens + kStageTokens - 1) / kStageTokens;
        my_units += units;
        my_max = max(my_max, units);
      }
      // tiles of (requests x heads) rows; the prefix keys are split into chunks
      const int per = a.tile_tokens;  // requests per tile pair
      const int groups = (g.num_seqs + per - 1) / per;
      const int kv_tiles = (prefix_tokens + 127) / 128;
      const int base = groups * g.num_kv_heads;
      // at most one tile per two SMs: the suffix partitions start at once on
      // the SMs the tiles leave free (longer tiles on half the SMs measured
      // 11 % faster than one wave of shorter tiles, a quarter 13 % slower)
      const int want = min(min(kMaxPrefixChunks, kv_tiles), max(1, a.num_sms / (2 * base)));
      const int per_chunk = (kv_tiles + want - 1) / want;
      prefix_chunks = (kv_tiles + per_chunk - 1) / per_chunk;  // no empty chunk
      for (int idx = tid; idx < base * prefix_chunks; idx += kPlanThreads) {
        const int c = idx / base, rest = idx % base;
        const int grp = rest / g.num_kv_heads, hk = rest % g.num_kv_heads;
        if (idx < ws.max_tiles)
          ws.tiles[idx] = make_int4(grp * per, hk, min(per, g.num_seqs - grp * per), c);
      }
      n_tiles_total = base * prefix_chunks;
    }
  }

  // partition length
  for (int o = 16; o; o >>= 1) {
    my_units += __shfl_xor_sync(0xffffffffu, my_units, o);
    my_max = max(my_max, __shfl_xor_sync(0xffffffffu, my_max, o));
  }
  if (lane == 0) {
    s_sum[warp] = my_units;
    s_max[warp] = my_max;
  }
  __syncthreads();
  if (tid == 0) {
    long long total = 0;
    int mx = 0;
    for (int w = 0; w < kPlanThreads / 32; ++w) {
      total += s_sum[w];
      mx = max(mx, s_max[w]);
    }
    long long by_target = (total * a.head_groups + a.target_items - 1) / max(a.target_items, 1);
    const long long cap =
        max(1LL, static_cast<long long>(ws.max_parts) - (prefix_tokens > 0 ? kMaxPrefixChunks : 0));
    long long by_cap = (mx + cap - 1) / cap;
    long long P = max(static_cast<long long>(a.min_part_stages), max(by_target, by_cap));
    s_P = static_cast<int>(max(P, 1LL));
    // CTAs the tensor-core tiles run on.  With decode partitions in the same
    // call, the tiles take only as many SMs as finish them in about half the
    // time the (HBM-bound) partitions need, and the partitions start at once
    // on the other SMs (rough B200 rates: a 128 x 128 query x key product of
    // head_dim 128 takes ~1.9 us on one SM; decode streams ~6.5 TB/s).
    int ntc = a.num_sms;
    if (!a.cascade && total > 0 && s_tile_kv > 0) {
      const double tile_sm_us = static_cast<double>(s_tile_kv) * 1.9 * g.head_dim / 128.0;
      const double dec_us = static_cast<double>(total) * kStageTokens * g.num_kv_heads *
                            g.head_dim * 4.0 / 6.5e6;
      const double want = 2.0 * tile_sm_us / max(dec_us, 1.0);
      ntc = static_cast<int>(min(static_cast<double>(a.num_sms), ceil(want)));
      ntc = max(ntc, min(8, a.num_sms));
    }
    s_ntc = ntc;
  }
  __syncthreads();
  const int P = s_P;

  // 2. items per thread (rows in parallel)
  int my_items = 0;
  for (int r = tid; r < g.num_qrows; r += kPlanThreads) {
    const int4 info = ws.qrow_info[r];
    if (info.z == 0) continue;
    const int units = (info.y - info.w + kStageTokens - 1) / kStageTokens;
    my_items += (units + P - 1) / P * a.head_groups;
  }
  int incl = my_items;
  for (int o = 1; o < 32; o <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) s_scan[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int v = s_scan[lane];
    int vi = v;
    for (int o = 1; o < 32; o <<= 1) {
      int n = __shfl_up_sync(0xffffffffu, vi, o);
      if (lane >= o) vi += n;
    }
    s_scan[lane] = vi - v;  // exclusive prefix of warp totals
    if (lane == 31) {
      ws.ctrl[0] = 0;
      ws.ctrl[1] = vi;
      ws.ctrl[2] = P * kStageTokens;
      ws.ctrl[3] = 0;
    }
  }
  __syncthreads();
  int pos = s_scan[warp] + incl - my_items;

  // 3. items, partition counts, rows to merge; a row with many items is listed
  // and its items written by the whole CTA below (one thread storing hundreds
  // of items one after another takes tens of microseconds)
  if (tid == 0) s_nbig = 0;
  __syncthreads();
  for (int r = tid; r < g.num_qrows; r += kPlanThreads) {
    const int4 info = ws.qrow_info[r];
    if (info.z == 0) continue;
    const int units = (info.y - info.w + kStageTokens - 1) / kStageTokens;
    const int np = (units + P - 1) / P;
    ws.nparts[r] = np + (info.w > 0 ? prefix_chunks : 0);  // the last ones: shared-prefix chunks
    // rows to merge: those a warp merges from the front of the list, those
    // with more than kMergeWarpParts partitions (a CTA each) from the back
    if (ws.nparts[r] > kMergeWarpParts)
      ws.merge_rows[g.num_qrows - 1 - atomicAdd(&s_merge_big, 1)] = r;
    else if (ws.nparts[r] != 1)
      ws.merge_rows[atomicAdd(&s_merge, 1)] = r;
    const int n_it = np * a.head_groups;
    if (n_it > kInlineItems) {
      const int slot = atomicAdd(&s_nbig, 1);
      if (slot < kMaxBig) {
        s_big[slot] = r;
        s_bigpos[slot] = pos;
        pos += n_it;
        continue;
      }
    }
    for (int p = 0; p < np; ++p)
      for (int hg = 0; hg < a.head_groups; ++hg)
        ws.items[pos++] = make_int4(r, hg | (p << kItemPartShift), P, p * P);
  }
  __syncthreads();
  const int nbig_rows = min(s_nbig, kMaxBig);
  for (int k = 0; k < nbig_rows; ++k) {
    const int r = s_big[k];
    const int4 info = ws.qrow_info[r];
    const int units = (info.y - info.w + kStageTokens - 1) / kStageTokens;
    const int n_it = (units + P - 1) / P * a.head_groups;
    for (int i = tid; i < n_it; i += kPlanThreads)
      ws.items[s_bigpos[k] + i] =
          make_int4(r, (i % a.head_groups) | ((i / a.head_groups) << kItemPartShift), P,
                    (i / a.head_groups) * P);
  }

  // 4. tiles, longest first
  if (npref > 0) {
    // exclusive scan of the bins from the longest down: two bins per thread
    static_assert(kTileBins == 2 * kPlanThreads, "two bins per thread");
    const int b0 = kTileBins - 1 - 2 * tid, b1 = b0 - 1;
    const int c0 = s_hist[b0], c1 = s_hist[b1];
    int incl = c0 + c1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    if (lane == 31) s_scan[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int v = s_scan[lane];
      int vi = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, vi, o);
        if (lane >= o) vi += n;
      }
      s_scan[lane] = vi - v;  // warps before this one
    }
    __syncthreads();
    const int before = s_scan[warp] + incl - (c0 + c1);
    s_hist[b0] = before;
    s_hist[b1] = before + c0;
    __syncthreads();
    for (int pi = 0; pi < npref; ++pi) {
      const int b = s_pref[pi];
      if (b < 0) continue;
      int r0, q_b;
      request_rows(g, b, r0, q_b);
      const int L = g.seq_lens[b];
      const int ntb = (q_b + a.tile_tokens - 1) / a.tile_tokens;
      for (int idx = tid; idx < ntb * g.num_kv_heads; idx += kPlanThreads) {
        const int tb = idx / g.num_kv_heads, hk = idx % g.num_kv_heads;
        const int tok0 = tb * a.tile_tokens;
        const int ntok = min(a.tile_tokens, q_b - tok0);
        const int at = atomicAdd(&s_hist[tile_bin((L - q_b + tok0 + ntok - 1) / 128 + 1)], 1);
        if (at < ws.max_tiles) ws.tiles[at] = make_int4(b, hk, tok0, ntok);
      }
    }
  }
  __syncthreads();
  if (tid == 0) {
    ws.ctrl[4] = static_cast<int>(min(static_cast<int64_t>(n_tiles_total), ws.max_tiles));
    ws.ctrl[5] = s_merge;
    ws.ctrl[9] = s_merge_big;
    ws.ctrl[6] = prefix_tokens;
    ws.ctrl[7] = prefix_chunks;
    ws.ctrl[8] = s_ntc;
  }
}

__global__ void __launch_bounds__(kPlanThreads) plan_kernel(AttnGeom g, PlanArgs a, WsView ws) {
  grid_launch_dependents();
  grid_dependency_wait();  // seq_lens / tables / the workspace may come from the previous launch
  plan_body(g, a, ws);
}

// A decode step's first launch: CTA 0 plans the attention while the other
// CTAs write the step's new K/V rows into the pools (one warp per token and
// K|V).  Neither half reads what the other writes -- the planner reads the
// lengths and tables, the write reads those and the new rows and writes slots
// and pool rows -- and the attention launches after this one read both
// results only after griddepcontrol.wait, i.e. after the whole grid.
template <bool F8>
__global__ void __launch_bounds__(kPlanThreads) write_plan_kernel(AttnGeom g, PlanArgs a,
                                                                  WsView ws, SlotWrite sw) {
  grid_launch_dependents();
  grid_dependency_wait();  // every input and the workspace may come from the previous launch
  if (blockIdx.x == 0) {
    plan_body(g, a, ws);
    return;
  }
  const int64_t w =
      static_cast<int64_t>(blockIdx.x - 1) * (kPlanThreads / 32) + (threadIdx.x >> 5);
  slot_write_warp<F8>(sw, w, threadIdx.x & 31);
}

cudaError_t launch_plan(const AttnGeom& g, const PlanArgs& a, const WsView& ws, cudaStream_t s) {
  return launch_pdl<plan_kernel>(dim3(1), dim3(kPlanThreads), 0, s, g, a, ws);
}

cudaError_t launch_write_plan(const AttnGeom& g, const PlanArgs& a, const WsView& ws,
                              const SlotWrite& sw, bool fp8, cudaStream_t s) {
  constexpr int64_t kWarps = kPlanThreads / 32;
  const int64_t write_ctas = (2 * sw.num_tokens + kWarps - 1) / kWarps;
  if (write_ctas + 1 > 0x7fffffffLL) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(1 + write_ctas));
  if (fp8) return launch_pdl<write_plan_kernel<true>>(grid, dim3(kPlanThreads), 0, s, g, a, ws, sw);
  return launch_pdl<write_plan_kernel<false>>(grid, dim3(kPlanThreads), 0, s, g, a, ws, sw);
}

// ======================================================================= generic
// CUDA-core path (any dtype, D in {64,128}, group <= 16): one CTA of 4 warps per
// item (row, KV head, partition).  Each warp walks every 4th key; the 32 lanes
// split head_dim, the q.k partial sums are combined with xor shuffles, and
// each warp keeps its own running (m, l, o) per query head of the group.  The
// four warps are merged through shared memory at the end of the item.
template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

template <typename T, int V>
__device__ __forceinline__ void load_row(const T* p, float (&x)[V]) {
#pragma unroll
  for (int e = 0; e < V; ++e) x[e] = to_f32(p[e]);
}
// FP8 pool entries: e4m3 codes, decoded exactly (the scales are applied to the
// scores and to the output instead)
struct e4m3_t {
  uint8_t code;
};
template <int V>
__device__ __forceinline__ void load_row_e4m3(const e4m3_t* p, float (&x)[V]) {
  static_assert(V % 2 == 0, "pairs of codes");
  const uint8_t* b = reinterpret_cast<const uint8_t*>(p);
#pragma unroll
  for (int e = 0; e < V; e += 2) {
    const uint16_t c = static_cast<uint16_t>(b[e]) | (static_cast<uint16_t>(b[e + 1]) << 8);
    const float2 f = f16x2_to_f32x2(e4m3x2_to_f16x2(c));
    x[e] = f.x;
    x[e + 1] = f.y;
  }
}
template <typename T>
struct QueryType {
  using type = T;
};
template <>
struct QueryType<e4m3_t> {
  using type = __nv_bfloat16;  // queries of an FP8 cache are bf16
};

__device__ __forceinline__ void store_out(void* out, int out_dtype, int64_t idx, float v) {
  if (out_dtype == PA_F32)
    static_cast<float*>(out)[idx] = v;
  else
    static_cast<__nv_bfloat16*>(out)[idx] = __float2bfloat16_rn(v);
}

constexpr int kGenWarps = 4;

template <typename T, int D>
__global__ void __launch_bounds__(kGenWarps * 32) attn_generic_kernel(AttnGeom g, WsView ws) {
  constexpr int V = D / 32;
  __shared__ float s_q[kMaxGroup][D];
  __shared__ float s_o[kGenWarps][kMaxGroup][D];
  __shared__ float s_m[kGenWarps][kMaxGroup];
  __shared__ float s_l[kGenWarps][kMaxGroup];
  __shared__ int s_item;
  __shared__ int s_bad;
  grid_dependency_wait();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = g.num_heads / g.num_kv_heads;
  const int n_items = ws.ctrl[1];
  using QT = typename QueryType<T>::type;
  const QT* q = static_cast<const QT*>(g.q);
  const T* kc = static_cast<const T*>(g.k_cache);
  const T* vc = static_cast<const T*>(g.v_cache);

  for (;;) {
    if (tid == 0) {
      s_item = atomicAdd(&ws.ctrl[0], 1);
      s_bad = 0;
    }
    __syncthreads();
    const int it = s_item;
    if (it >= n_items) break;
    const int4 item = ws.items[it];
    const int r = item.x, hk = item.y & kItemHgMask, p = item.y >> kItemPartShift;
    const int4 info = ws.qrow_info[r];
    const int b = info.x, key_len = info.y;
    const int64_t lo64 = info.w + static_cast<int64_t>(item.w) * kStageTokens;
    const int lo = static_cast<int>(lo64);
    const int hi = static_cast<int>(min(lo64 + static_cast<int64_t>(item.z) * kStageTokens,
                                        static_cast<int64_t>(key_len)));
    for (int idx = tid; idx < G * D; idx += blockDim.x) {
      const int gq = idx / D, d = idx % D;
      s_q[gq][d] = to_f32(q[(static_cast<int64_t>(r) * g.num_heads + hk * G + gq) * D + d]);
    }
    __syncthreads();

    float m[kMaxGroup], l[kMaxGroup], o[kMaxGroup][V];
#pragma unroll
    for (int gq = 0; gq < kMaxGroup; ++gq) {
      m[gq] = -INFINITY;
      l[gq] = 0.f;
#pragma unroll
      for (int e = 0; e < V; ++e) o[gq][e] = 0.f;
    }
    const int32_t* table = g.block_tables + static_cast<int64_t>(b) * g.max_blocks;
    bool bad = false;
    for (int j = lo + warp; j < hi; j += kGenWarps) {
      const int phys = table[j / g.block_size];
      if (phys < 0 || phys >= g.num_blocks) {
        bad = true;
        continue;
      }
      const int64_t row = static_cast<int64_t>(phys) * g.block_size + j % g.block_size;
      const int64_t off = (row * g.num_kv_heads + hk) * D + lane * V;
      float kx[V], vx[V];
      if constexpr (std::is_same<T, e4m3_t>::value) {
        load_row_e4m3<V>(kc + off, kx);
        load_row_e4m3<V>(vc + off, vx);
      } else {
        load_row<T, V>(kc + off, kx);
        load_row<T, V>(vc + off, vx);
      }
#pragma unroll
      for (int gq = 0; gq < kMaxGroup; ++gq) {
        if (gq < G) {
          float dot = 0.f;
#pragma unroll
          for (int e = 0; e < V; ++e) dot = fmaf(s_q[gq][lane * V + e], kx[e], dot);
#pragma unroll
          for (int o2 = 16; o2; o2 >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o2);
          const float s = dot * g.scale_log2;
          const float m_new = fmaxf(m[gq], s);
          const float alpha = fast_exp2(m[gq] - m_new);
          const float pe = fast_exp2(s - m_new);
          l[gq] = l[gq] * alpha + pe;
#pragma unroll
          for (int e = 0; e < V; ++e) o[gq][e] = fmaf(o[gq][e], alpha, pe * vx[e]);
          m[gq] = m_new;
        }
      }
    }
    if (bad) s_bad = 1;
#pragma unroll
    for (int gq = 0; gq < kMaxGroup; ++gq) {
      if (gq < G) {
        if (lane == 0) {
          s_m[warp][gq] = m[gq];
          s_l[warp][gq] = l[gq];
        }
#pragma unroll
        for (int e = 0; e < V; ++e) s_o[warp][gq][lane * V + e] = o[gq][e];
      }
    }
    __syncthreads();
    const bool row_bad = s_bad != 0;
    if (row_bad) {
      if (tid == 0) {
        ws.qrow_bad[r] = 1;
        if (g.err_word) atomicOr(g.err_word, PA_ERRBIT_BLOCK_OOB);
      }
    }
    const int np = ws.nparts[r];
    for (int idx = tid; idx < G * D; idx += blockDim.x) {
      const int gq = idx / D, d = idx % D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kGenWarps; ++w) M = fmaxf(M, s_m[w][gq]);
      float Ls = 0.f, O = 0.f;
#pragma unroll
      for (int w = 0; w < kGenWarps; ++w) {
        const float c = (s_m[w][gq] == -INFINITY) ? 0.f : fast_exp2(s_m[w][gq] - M);
        Ls = fmaf(s_l[w][gq], c, Ls);
        O = fmaf(s_o[w][gq][d], c, O);
      }
      const int h = hk * G + gq;
      if (np == 1) {
        if (!row_bad)
          store_out(g.out, g.out_dtype, (static_cast<int64_t>(r) * g.num_heads + h) * D + d,
                    O * g.v_scale / Ls);
      } else {
        const int64_t slot = (static_cast<int64_t>(r) * g.num_heads + h) * ws.max_parts + p;
        if (d == 0) ws.part_ml[slot] = make_float2(M, Ls);
        ws.part_o[slot * D + d] = O * g.v_scale;
      }
    }
    __syncthreads();
  }
}

cudaError_t launch_attn_generic(const AttnGeom& g, const WsView& ws, int num_sms,
                                cudaStream_t s) {
  const dim3 grid(num_sms * 8), block(kGenWarps * 32);
  if (g.dtype == PA_F32) {
    if (g.head_dim == 64) return launch_pdl<attn_generic_kernel<float, 64>>(grid, block, 0, s, g, ws);
    return launch_pdl<attn_generic_kernel<float, 128>>(grid, block, 0, s, g, ws);
  }
  if (g.dtype == PA_FP8_E4M3) {
    if (g.head_dim == 64)
      return launch_pdl<attn_generic_kernel<e4m3_t, 64>>(grid, block, 0, s, g, ws);
    return launch_pdl<attn_generic_kernel<e4m3_t, 128>>(grid, block, 0, s, g, ws);
  }
  if (g.head_dim == 64)
    return launch_pdl<attn_generic_kernel<__nv_bfloat16, 64>>(grid, block, 0, s, g, ws);
  return launch_pdl<attn_generic_kernel<__nv_bfloat16, 128>>(grid, block, 0, s, g, ws);
}

// ======================================================================= merge
// Rows with a single partition were written by the attention kernel; rows with
// none get zeros; invalid rows are skipped.  The rows to merge come from the
// planner's list.  Pass 1: one warp per (row, query head) with at most
// kMergeWarpParts (64) partitions: lane k holds partitions k and k + 32 (m, l),
// the weights 2^(m_k - M) are shuffled to all lanes and each lane accumulates
// D/32 output columns.  Pass 2: one 32-warp CTA per remaining (row, head): max and
// denominator reduced over the CTA, then each warp accumulates every 8th
// partition (4 in flight) and the warp sums are combined.
constexpr int kMergeWarps = 32;
constexpr int kMergeCached = 2048;  // partition weights kept in shared memory

template <int D>
__device__ __forceinline__ void merge_pair_warp(const AttnGeom& g, const WsView& ws, int64_t idx,
                                                int np, int lane) {
  constexpr int V = D / 32;
  const int64_t out_base = idx * D + lane * V;
  if (np == 0) {
#pragma unroll
    for (int e = 0; e < V; ++e) store_out(g.out, g.out_dtype, out_base + e, 0.f);
    return;
  }
  const int64_t base = idx * ws.max_parts;
  const float* po = ws.part_o + base * D + lane * V;
  // up to 8 partial rows in flight per lane (and 32 warps per SM); the first
  // batch is requested before the weights, so that its round trip to L2
  // overlaps the one of the (m, l) pairs
  constexpr int kBatch = 8;
  float x[kBatch][V];
  auto load_batch = [&](int k0) {
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const bool ok = k0 + u < np;
      if constexpr (V == 4) {
        const float4 t4 = ok ? *reinterpret_cast<const float4*>(po + static_cast<int64_t>(k0 + u) * D)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
        x[u][0] = t4.x, x[u][1] = t4.y, x[u][2] = t4.z, x[u][3] = t4.w;
      } else {
#pragma unroll
        for (int e = 0; e < V; ++e) x[u][e] = ok ? po[static_cast<int64_t>(k0 + u) * D + e] : 0.f;
      }
    }
  };
  load_batch(0);
  const float2 ml0 = lane < np ? ws.part_ml[base + lane] : make_float2(-INFINITY, 0.f);
  const float2 ml1 = lane + 32 < np ? ws.part_ml[base + lane + 32] : make_float2(-INFINITY, 0.f);
  float M = fmaxf(ml0.x, ml1.x);
#pragma unroll
  for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float c0 = (ml0.x == -INFINITY) ? 0.f : fast_exp2(ml0.x - M);
  const float c1 = (ml1.x == -INFINITY) ? 0.f : fast_exp2(ml1.x - M);
  float den = c0 * ml0.y + c1 * ml1.y;
#pragma unroll
  for (int o = 16; o; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  float acc[V];
#pragma unroll
  for (int e = 0; e < V; ++e) acc[e] = 0.f;
  for (int k0 = 0; k0 < np; k0 += kBatch) {
    if (k0 > 0) load_batch(k0);
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int k = min(k0 + u, kMergeWarpParts - 1);  // warp-uniform
      const float cu = __shfl_sync(0xffffffffu, k < 32 ? c0 : c1, k & 31);
#pragma unroll
      for (int e = 0; e < V; ++e) acc[e] = fmaf(x[u][e], cu, acc[e]);
    }
  }
  const float inv = 1.f / den;
#pragma unroll
  for (int e = 0; e < V; ++e) store_out(g.out, g.out_dtype, out_base + e, acc[e] * inv);
}

template <int D>
__global__ void __launch_bounds__(kMergeWarps * 32, 1) merge_kernel(AttnGeom g, WsView ws) {
  constexpr int V = D / 32;
  __shared__ float s_c[kMergeCached];
  __shared__ float s_red[kMergeWarps];
  __shared__ float s_acc[kMergeWarps][D];
  grid_dependency_wait();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t pairs = static_cast<int64_t>(ws.ctrl[5]) * g.num_heads;
  const int64_t big_pairs = static_cast<int64_t>(ws.ctrl[9]) * g.num_heads;
  // pass 1: (row, head) pairs with at most kMergeWarpParts partitions, one warp
  // each, spread over the CTAs first (pair i on CTA i % grid): a batch of few
  // pairs then loads its partials through every SM, not through a few
  for (int64_t pi = static_cast<int64_t>(warp) * gridDim.x + blockIdx.x; pi < pairs;
       pi += static_cast<int64_t>(gridDim.x) * kMergeWarps) {
    const int r = ws.merge_rows[pi / g.num_heads];
    const int np = ws.nparts[r];
    if (np == 1 || np < 0 || np > kMergeWarpParts || ws.qrow_bad[r]) continue;
    merge_pair_warp<D>(g, ws, static_cast<int64_t>(r) * g.num_heads + pi % g.num_heads, np, lane);
  }
  // pass 2: pairs with more partitions (listed from the back), one CTA each
  for (int64_t pi = blockIdx.x; pi < big_pairs; pi += gridDim.x) {
    const int r = ws.merge_rows[g.num_qrows - 1 - pi / g.num_heads];
    const int64_t idx = static_cast<int64_t>(r) * g.num_heads + pi % g.num_heads;
    const int np = ws.nparts[r];
    if (np <= kMergeWarpParts || ws.qrow_bad[r]) continue;
    const int64_t out_base = idx * D;
    const int64_t base = idx * ws.max_parts;
    // M
    float M = -INFINITY;
    for (int k = tid; k < np; k += blockDim.x) M = fmaxf(M, ws.part_ml[base + k].x);
#pragma unroll
    for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    if (lane == 0) s_red[warp] = M;
    __syncthreads();
    M = s_red[0];
#pragma unroll
    for (int w = 1; w < kMergeWarps; ++w) M = fmaxf(M, s_red[w]);
    __syncthreads();
    // denominator and weights
    float den = 0.f;
    for (int k = tid; k < np; k += blockDim.x) {
      const float2 ml = ws.part_ml[base + k];
      const float c = (ml.x == -INFINITY) ? 0.f : fast_exp2(ml.x - M);
      if (k < kMergeCached) s_c[k] = c;
      den = fmaf(ml.y, c, den);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    if (lane == 0) s_red[warp] = den;
    __syncthreads();
    den = 0.f;
#pragma unroll
    for (int w = 0; w < kMergeWarps; ++w) den += s_red[w];
    // weighted sum of the partial outputs
    float acc[V];
#pragma unroll
    for (int e = 0; e < V; ++e) acc[e] = 0.f;
    const float* po = ws.part_o + base * D + lane * V;
    int k = warp;
    for (; k + 3 * kMergeWarps < np; k += 4 * kMergeWarps) {
      float x[4][V], c[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int kk = k + u * kMergeWarps;
        c[u] = kk < kMergeCached ? s_c[kk]
                                 : (ws.part_ml[base + kk].x == -INFINITY
                                        ? 0.f
                                        : fast_exp2(ws.part_ml[base + kk].x - M));
#pragma unroll
        for (int e = 0; e < V; ++e) x[u][e] = po[static_cast<int64_t>(kk) * D + e];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] = fmaf(x[u][e], c[u], acc[e]);
    }
    for (; k < np; k += kMergeWarps) {
      const float c = k < kMergeCached ? s_c[k]
                                       : (ws.part_ml[base + k].x == -INFINITY
                                              ? 0.f
                                              : fast_exp2(ws.part_ml[base + k].x - M));
#pragma unroll
      for (int e = 0; e < V; ++e) acc[e] = fmaf(po[static_cast<int64_t>(k) * D + e], c, acc[e]);
    }
#pragma unroll
    for (int e = 0; e < V; ++e) s_acc[warp][lane * V + e] = acc[e];
    __syncthreads();
    const float inv = 1.f / den;
    for (int d = tid; d < D; d += blockDim.x) {
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < kMergeWarps; ++w) sum += s_acc[w][d];
      store_out(g.out, g.out_dtype, out_base + d, sum * inv);
    }
    __syncthreads();  // s_c / s_red / s_acc are reused by the next pair
  }
}

cudaError_t launch_merge(const AttnGeom& g, const WsView& ws, int num_sms, cudaStream_t s) {
  // one CTA of 32 warps per SM, warps looping over the pairs: a grid of
  // eight small CTAs per SM took ~10 us just to be launched
  int64_t blocks = static_cast<int64_t>(g.num_qrows) * g.num_heads;
  if (blocks == 0) return cudaSuccess;
  if (blocks > num_sms) blocks = num_sms;
  const dim3 grid(static_cast<unsigned>(blocks)), block(kMergeWarps * 32);
  if (g.head_dim == 64) return launch_pdl<merge_kernel<64>>(grid, block, 0, s, g, ws);
  return launch_pdl<merge_kernel<128>>(grid, block, 0, s, g, ws);
}

}  // namespace pa
