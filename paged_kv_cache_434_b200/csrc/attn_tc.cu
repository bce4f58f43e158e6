// attn_tc.cu -- tensor-core (tcgen05 / TMEM) tiles for the chunked-prefill
// requests of a mixed continuous-batching step.
//
// What is computed ("AI Infra入门干货总结：大模型是如何高效推理的", section
// "Attention (FlashAttention, Scaled Dot-Product Attention)"): for the q_b new
// tokens of a request with seq_len L (q_b > 1), query i at position
// L - q_b + i attends causally to keys 0 .. L - q_b + i through the block table
// (the v1 unified varlen path reads every K/V from the paged cache).  The
// online softmax keeps a running max m and sum l and rescales the output by
// exp(m_old - m_new); here the rescale is skipped while the new row max stays
// within 2^8 of the one in use (the weights then stay below 256, which bf16
// and fp32 represent exactly enough), an exact reformulation.
//
// A work item is a pair of 128-row query tiles A and B (each 128/G
// consecutive tokens x the G query heads of one KV head) that share every
// 128-key K/V tile: one K/V read serves 256 query rows, which halves the
// bytes per FLOP that must come from L2.
//
// The same kernel serves the shared-prefix cascade of a decode batch: when
// every request's block table starts with the same blocks, the rows of an
// item are 256/G requests x G heads, all see the whole prefix (no causal
// mask), and the result is written as a split-KV partial (m, l, unnormalised
// o) that the log-sum-exp merge combines with the requests' own suffixes
// ("总结": partials re-normalised with log-sum-exp; "Paged Attention": blocks
// shared through the block table).
//
// CTA (persistent, one per SM, 12 warps in three warpgroups; the first gives
// registers to the two softmax warpgroups: 128 x 104 + 256 x 200 = 384 x 168):
//   warp 3   scheduler: takes the next item from the planner's longest-first
//            list, publishes it in a 2-slot ring and TMA-loads the 256 query
//            rows (128-byte swizzle) once the previous item's QK^T are done.
//   warps 0-1  loaders: warp 0 fills the K stages (three), warp 1 the V stages
//            (two), with 16-byte cp.async copies gathered through the block
//            table into the 128B-swizzled layout the MMA reads (blocks of 16
//            keys are too small for efficient TMA boxes).  A K stage is free
//            again once its QK^T are done, a V stage once its PVs are done;
//            each loader keeps two tiles in flight and announces a tile when
//            it has issued the next one.
//   warp 2   allocates TMEM (S_A, S_B, O_A, O_B: 128 columns each); one thread
//            issues S_X = Q_X K^T (M=128, N=128, K=D) and O_X += P_X V (N=D,
//            K=128, P from TMEM, V an MN-major shared-memory operand) in the
//            order QK_A(t), QK_B(t), PV_A(t), QK_A(t+1), PV_B(t), QK_B(t+1),
//            ... so that the tensor core works on one tile while the softmax
//            handles the other.  MMAs of one thread complete in issue order.
//   warps 4-7 (tile A) and 8-11 (tile B)  softmax, the two tiles concurrently:
//            thread i owns row i (TMEM lane i), reads its S row straight from
//            TMEM (row max and sum need no shuffles), writes bf16 P over the
//            first 64 columns of the same S buffer, rescales O in TMEM when the
//            max moved (S_X(t) being complete implies PV_X(t-1) is), and
//            finally writes O / l.
#include <cuda.h>
#include <cuda_bf16.h>

#include <cmath>

#include "internal.h"
#include "ptx.cuh"

namespace pa {
namespace tck {

constexpr int kRows = 128;     // query rows per tile
constexpr int kKeys = 128;     // keys per KV tile
constexpr int kThreads = 384;  // 12 warps
constexpr int kHalfBytes = 128 * 128;  // [128 rows x 64 bf16]
constexpr float kRescaleLog2 = 8.f;

struct Item {
  int b, hk, tok0, ntok;  // request, KV head, first token (within the request), tokens
  int n_kv;               // 128-key tiles to visit (0: end of work)
  int first_pos;          // position of the first token
  int row0;               // flattened row of the first token
  int L;                  // keys [0, L) exist: seq_len, or the shared prefix length
  int causal;             // 0: shared-prefix item (every row sees all L keys)
  int kv0;                // first 128-key tile (shared-prefix chunks)
  int chunk;              // shared-prefix chunk index
  int end;                // 1: no more work
};

template <int D>
struct Cfg {
  static constexpr int NH = D / 64;
  static constexpr int kQTile = NH * kHalfBytes;     // one 128-row query tile
  static constexpr int kKVBytes = NH * kHalfBytes;   // one K (or V) tile
  static constexpr int kKStages = 3, kVStages = 2;
  static constexpr int kOffQ = 0;                    // 256 query rows: per half, A then B
  static constexpr int kOffK = 2 * kQTile;
  static constexpr int kOffV = kOffK + kKStages * kKVBytes;
  static constexpr int kOffMeta = kOffV + kVStages * kKVBytes;
  // meta + alignment slack; at least 120 KB so that one CTA runs per SM (each
  // CTA takes all 512 TMEM columns)
  static constexpr int kSmem0 = kOffMeta + 1024 + 1024;
  static constexpr int kSmem = kSmem0 > 120 * 1024 ? kSmem0 : 120 * 1024;
};

struct Meta {
  Item ring[2];
  uint64_t item_full[2], item_empty[2];
  uint64_t q_full, q_empty;
  uint64_t k_full[3], k_empty[3], v_full[2], v_empty[2];
  uint64_t s_full[2], p_full[2], o_ready[2];  // [tile A, tile B]
  uint64_t o_empty, drain;
  uint32_t tmem_base;
};

__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity) {
  bool ok = mbar_wait_bounded(bar, parity, kWaitLimitNs);
  return __all_sync(0xffffffffu, ok);
}

}  // namespace tck

template <int D>
__global__ void __launch_bounds__(tck::kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, AttnGeom g, WsView ws) {
  using namespace tck;
  using C = Cfg<D>;
  constexpr int NH = C::NH;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  Meta* meta = reinterpret_cast<Meta*>(smem + C::kOffMeta);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = g.num_heads / g.num_kv_heads;
  const int Tq = kRows / G;  // tokens per query tile

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&meta->item_full[i], 1);
      mbar_init(&meta->item_empty[i], 32 + 32 + 1 + 256);
      mbar_init(&meta->v_full[i], 32);
      mbar_init(&meta->v_empty[i], 1);
      mbar_init(&meta->s_full[i], 1);
      mbar_init(&meta->p_full[i], 128);
      mbar_init(&meta->o_ready[i], 1);
    }
    for (int i = 0; i < 3; ++i) {
      mbar_init(&meta->k_full[i], 32);
      mbar_init(&meta->k_empty[i], 1);
    }
    mbar_init(&meta->q_full, 1);
    mbar_init(&meta->q_empty, 1);
    mbar_init(&meta->o_empty, 256);
    mbar_init(&meta->drain, 1);
    fence_mbar_init();
    prefetch_tmap(&tmQ);
  }
  if (warp == 2) {
    tmem_alloc(&meta->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  grid_dependency_wait();
  // after the wait: the next launch may start while tiles run, and relies on
  // the plan being complete by then
  grid_launch_dependents();
  const uint32_t tmem = meta->tmem_base;
  const int n_tiles = ws.ctrl[4];
  const int prefix = ws.ctrl[6];  // > 0: decode cascade over a shared prefix
  const int prefix_chunks = ws.ctrl[7];
  const uint32_t sQ = smem_u32(smem + C::kOffQ);
  const uint32_t sK = smem_u32(smem + C::kOffK);
  const uint32_t sV = smem_u32(smem + C::kOffV);
  // the planner may leave part of the SMs to the decode partitions that run
  // beside the tiles, or find no tile at all: such CTAs only release their TMEM
  const bool working = static_cast<int>(blockIdx.x) < ws.ctrl[8] && n_tiles > 0;

  if (!working) {
  } else if (warp == 3) {
    // ---------------------------------------------------------- scheduler
    regs_dec<104>();
    if (lane == 0) {
      for (int n = 0;; ++n) {
        // claim item n only once every role has taken item n - 1 (at most one
        // item ahead of the work): items are handed out longest first, and a
        // CTA that held two claimed items at the end would stretch the tail
        if (n >= 1 && !mbar_wait_bounded(&meta->item_empty[(n - 1) & 1], ((n - 1) >> 1) & 1,
                                         kWaitLimitNs)) {
          if (g.err_word) atomicOr(g.err_word, PA_ERRBIT_TIMEOUT);
          break;
        }
        const int it = atomicAdd(&ws.ctrl[3], 1);
        Item info{};
        info.end = it >= n_tiles;
        if (it < n_tiles && prefix > 0) {
          const int4 t = ws.tiles[it];  // {first request, kv head, requests}
          info.b = t.x;
          info.hk = t.y;
          info.tok0 = 0;
          info.ntok = t.z;
          info.L = prefix;
          info.first_pos = prefix - 1;
          info.row0 = t.x;
          const int kv_all = (prefix + kKeys - 1) / kKeys;
          const int per_chunk = (kv_all + prefix_chunks - 1) / prefix_chunks;
          info.kv0 = t.w * per_chunk;
          info.n_kv = max(0, min(per_chunk, kv_all - info.kv0));
          info.causal = 0;
          info.chunk = t.w;
        } else if (it < n_tiles) {
          const int4 t = ws.tiles[it];
          const int qs = g.query_start_loc[t.x];
          const int qb = g.query_start_loc[t.x + 1] - qs;
          info.b = t.x;
          info.hk = t.y;
          info.tok0 = t.z;
          info.ntok = t.w;
          info.L = g.seq_lens[t.x];
          info.first_pos = info.L - qb + t.z;
          info.row0 = qs + t.z;
          info.n_kv = (info.first_pos + t.w - 1) / kKeys + 1;
          info.causal = 1;
          info.kv0 = 0;
        }
        // an entry that does not describe a valid tile is reported and skipped
        const int64_t max_keys = static_cast<int64_t>(g.max_blocks) * g.block_size;
        if (!info.end &&
            (info.b < 0 || info.b >= g.num_seqs || info.hk < 0 || info.hk >= g.num_kv_heads ||
             info.ntok < 1 || info.ntok > 2 * Tq || info.n_kv < 1 || info.L > max_keys ||
             static_cast<int64_t>(info.kv0 + info.n_kv) * kKeys > max_keys + kKeys ||
             info.row0 < 0 || info.row0 + info.ntok > g.num_qrows)) {
          if (g.err_word) atomicOr(g.err_word, PA_ERRBIT_QUERY_TOO_LONG);
          --n;
          continue;
        }
        const int slot = n & 1;
        if (n >= 2 && !mbar_wait_bounded(&meta->item_empty[slot], ((n >> 1) - 1) & 1,
                                         kWaitLimitNs)) {
          if (g.err_word) atomicOr(g.err_word, PA_ERRBIT_TIMEOUT);
          break;
        }
        meta->ring[slot] = info;
        mbar_arrive(&meta->item_full[slot]);
        if (info.end) break;
        // the 256 query rows: box [64 dims x G heads x 2Tq tokens] per half
        if (n >= 1 && !mbar_wait_bounded(&meta->q_empty, (n - 1) & 1, kWaitLimitNs)) {
          if (g.err_word) atomicOr(g.err_word, PA_ERRBIT_TIMEOUT);
          break;
        }
        mbar_arrive_expect_tx(&meta->q_full, 2 * C::kQTile);
#pragma unroll
        for (int dh = 0; dh < NH; ++dh)
          tma_load_3d(smem + C::kOffQ + dh * 2 * kHalfBytes, &tmQ, &meta->q_full, dh * 64,
                      info.hk * G, info.row0);
      }
    }
  } else if (warp < 2) {
    // ---------------------------------------------------------- loaders
    regs_dec<104>();
    const bool is_v = warp == 1;
    const int tg = lane;
    const int bshift = __ffs(g.block_size) - 1;  // block sizes are powers of two
    const __nv_bfloat16* src_pool = static_cast<const __nv_bfloat16*>(is_v ? g.v_cache : g.k_cache);
    const uint32_t sbase = is_v ? sV : sK;
    uint64_t* full = is_v ? meta->v_full : meta->k_full;
    uint64_t* empty = is_v ? meta->v_empty : meta->k_empty;
    const int nst = is_v ? C::kVStages : C::kKStages;
    int tile_base = 0, pending = -1;
    bool ok = true;
    for (int n = 0; ok; ++n) {
      const int slot = n & 1;
      if (!wait_warp(&meta->item_full[slot], (n >> 1) & 1)) {
        ok = false;
        break;
      }
      const Item info = meta->ring[slot];
      mbar_arrive(&meta->item_empty[slot]);
      if (info.end) break;
      const int32_t* table = g.block_tables + static_cast<int64_t>(info.b) * g.max_blocks;
      for (int j = 0; j < info.n_kv; ++j) {
        const int t = tile_base + j;
        const int st = t % nst, use = t / nst;  // stage and how often it was used before
        const uint32_t dst = sbase + st * C::kKVBytes;
        // Lanes are paired (D = 128) or grouped by four (D = 64) on a key so
        // that one warp instruction copies whole 32-byte sectors of 16 (8)
        // keys.  Each lane first resolves its keys' pool rows through the block
        // table (-1: past the request or outside the pool), then copies fixed
        // chunk offsets of those rows into the 128B-swizzled tile.
        constexpr int kChunks = 8 * NH;                 // 16-byte chunks per key row
        constexpr int kKPI = D == 128 ? 16 : 8;          // keys per warp instruction
        constexpr int kLPK = 32 / kKPI;                  // lanes per key
        constexpr int kKeysPerLane = kKeys / kKPI;
        constexpr int kCPL = kChunks / kLPK;             // chunks per lane per key
        const int ksub = tg / kLPK, csub = tg % kLPK;
        const __nv_bfloat16* rowp[kKeysPerLane];
#pragma unroll
        for (int q = 0; q < kKeysPerLane; ++q) {
          const int kpos = (info.kv0 + j) * kKeys + q * kKPI + ksub;
          rowp[q] = nullptr;
          if (kpos < info.L) {
            const int phys = table[kpos >> bshift];
            if (phys >= 0 && phys < g.num_blocks)
              rowp[q] = src_pool + ((static_cast<int64_t>(phys << bshift) + (kpos & (g.block_size - 1))) *
                                        g.num_kv_heads + info.hk) * D;
          }
        }
        if (use >= 1 && !wait_warp(&empty[st], (use - 1) & 1)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int q = 0; q < kKeysPerLane; ++q) {
          const int key = q * kKPI + ksub;
          const uint32_t rbase = dst + key * 128;
          const bool valid = rowp[q] != nullptr;
#pragma unroll
          for (int p = 0; p < kCPL; ++p) {
            const int chunk = p * kLPK + csub, dh = chunk >> 3, c = chunk & 7;
            cp_async16(rbase + dh * kHalfBytes + ((c ^ (key & 7)) << 4),
                       valid ? rowp[q] + chunk * 8 : src_pool, valid ? 16u : 0u);
          }
        }
        cp_async_commit();
        if (pending >= 0) {
          // the previous tile's copies are complete once at most this group is in flight
          cp_async_wait<1>();
          fence_proxy_async_smem();
          mbar_arrive(&full[pending % nst]);
        }
        pending = t;
      }
      tile_base += info.n_kv;
    }
    cp_async_wait<0>();
    if (pending >= 0) {
      fence_proxy_async_smem();
      mbar_arrive(&full[pending % nst]);
    }
    if (!ok && g.err_word && tg == 0) atomicOr(g.err_word, PA_ERRBIT_TIMEOUT);
  } else if (warp == 2) {
    // ---------------------------------------------------------- MMA issuer
    regs_dec<104>();
    if (lane == 0) {
      const uint32_t id_qk = idesc_bf16_f32(kRows, kKeys, 0, 0);
      const uint32_t id_pv = idesc_bf16_f32(kRows, D, 0, 1);
      int tile_base = 0;
      int sfa = 0, sfb = 0;  // P tiles consumed per query tile (p_full parity)
      bool ok = true;
      // S_X = Q_X K_t^T, X = 0 (A) or 1 (B)
      auto qk = [&](int X, int t) {
        const uint32_t qx = sQ + X * (kRows * 128);
        const uint32_t kst = sK + (t % 3) * C::kKVBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t qo = (kk >> 2) * 2 * kHalfBytes + (kk & 3) * 32;
          const uint32_t ko = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
          umma_bf16(tmem + X * 128, smem_desc(qx + qo, 16, 1024, 2), smem_desc(kst + ko, 16, 1024, 2),
                    id_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(&meta->s_full[X]);
      };
      // O_X += P_X V_t
      auto pv = [&](int X, int t, bool first) -> bool {
        int& cnt = X ? sfb : sfa;
        if (!mbar_wait_bounded(&meta->p_full[X], cnt & 1, kWaitLimitNs)) return false;
        ++cnt;
        tc_fence_after();
        const uint32_t vst = sV + (t & 1) * C::kKVBytes;
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk)
          umma_bf16_tmem_a(tmem + 256 + X * 128, tmem + X * 128 + kk * 8,
                           smem_desc(vst + kk * 2048, kHalfBytes, 1024, 2), id_pv,
                           (!first || kk > 0) ? 1u : 0u);
        return true;
      };
      auto wait_k = [&](int t) {
        return mbar_wait_bounded(&meta->k_full[t % 3], (t / 3) & 1, kWaitLimitNs);
      };
      for (int n = 0; ok; ++n) {
        const int slot = n & 1;
        if (!mbar_wait_bounded(&meta->item_full[slot], (n >> 1) & 1, kWaitLimitNs)) {
          ok = false;
          break;
        }
        const Item info = meta->ring[slot];
        mbar_arrive(&meta->item_empty[slot]);
        if (info.end) break;
        const bool hasB = info.ntok > Tq;
        // (the first QK^T only writes S: it runs while the softmax warps still
        // store the previous item's O; the first PV, which overwrites O,
        // waits for them below)
        if (!mbar_wait_bounded(&meta->q_full, n & 1, kWaitLimitNs) || !wait_k(tile_base)) {
          ok = false;
          break;
        }
        tc_fence_after();
        qk(0, tile_base);
        if (hasB) qk(1, tile_base);
        umma_commit(&meta->k_empty[tile_base % 3]);
        for (int j = 0; j < info.n_kv && ok; ++j) {
          const int t = tile_base + j;
          const bool more = j + 1 < info.n_kv;
          if (j == 0 && n >= 1) {
            if (!mbar_wait_bounded(&meta->o_empty, (n - 1) & 1, kWaitLimitNs)) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
          if (!mbar_wait_bounded(&meta->v_full[t & 1], (t >> 1) & 1, kWaitLimitNs) ||
              !pv(0, t, j == 0)) {
            ok = false;
            break;
          }
          if (!more) umma_commit(&meta->o_ready[0]);
          if (more) {
            if (!wait_k(t + 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
            qk(0, t + 1);
          }
          if (hasB) {
            if (!pv(1, t, j == 0)) {
              ok = false;
              break;
            }
            if (!more) umma_commit(&meta->o_ready[1]);
          }
          umma_commit(&meta->v_empty[t & 1]);
          if (more) {
            if (hasB) qk(1, t + 1);
            umma_commit(&meta->k_empty[(t + 1) % 3]);
          } else {
            umma_commit(&meta->q_empty);
          }
        }
        tile_base += info.n_kv;
      }
      // every MMA issued so far has completed before TMEM is released
      umma_commit(&meta->drain);
      mbar_wait_bounded(&meta->drain, 0, kWaitLimitNs);
      if (!ok && g.err_word) atomicOr(g.err_word, PA_ERRBIT_TIMEOUT);
    }
  } else {
    // ---------------------------------------------------------- softmax
    regs_inc<200>();
    const int X = warp >= 8 ? 1 : 0;  // query tile of this warpgroup
    const int row = (tid - 128) & 127;  // query row = TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_addr + X * 128;
    const uint32_t tO = tmem + lane_addr + 256 + X * 128;
    int cnt = 0;      // S tiles consumed (s_full parity)
    int items_x = 0;  // items that had this query tile (o_ready parity)
    bool ok = true;
    for (int n = 0; ok; ++n) {
      const int slot = n & 1;
      if (!wait_warp(&meta->item_full[slot], (n >> 1) & 1)) {
        ok = false;
        break;
      }
      const Item info = meta->ring[slot];
      mbar_arrive(&meta->item_empty[slot]);
      if (info.end) break;
      const bool active = X == 0 || info.ntok > Tq;  // tile B may be empty
      float m = -INFINITY, l = 0.f;
      for (int j = 0; active && j < info.n_kv && ok; ++j) {
        {
          if (!wait_warp(&meta->s_full[X], cnt & 1)) {
            ok = false;
            break;
          }
          ++cnt;
          tc_fence_after();
          // last visible key of this row (causal) or of every row (shared prefix)
          const int pos = info.causal ? info.first_pos + X * Tq + row / G : info.L - 1;
          const int kbase = (info.kv0 + j) * kKeys;
          const bool masked = kbase + kKeys - 1 > (info.causal ? info.first_pos + X * Tq : info.L - 1);
          const int lim = pos - kbase;  // keys c <= lim are visible
          // the whole S row in one round trip: 4 loads of 32 columns, one wait
          uint32_t sr[4][32];
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, sr[c]);
          tmem_ld_wait();
          if (masked) {
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (c * 32 + e > lim) sr[c][e] = 0xff800000u;  // -inf
          }
          // row max: four independent chains of 3-input maxima
          float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int e = 0; e < 32; e += 8)
#pragma unroll
              for (int k = 0; k < 4; ++k)
                mq[k] = fmax3(mq[k], __uint_as_float(sr[c][e + 2 * k]), __uint_as_float(sr[c][e + 2 * k + 1]));
          float mx = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
          mx *= g.scale_log2;
          const bool rescale = mx > m + kRescaleLog2;
          const float m_use = rescale ? mx : m;
          const float alpha = rescale ? fast_exp2(m - m_use) : 1.f;
          // S_X(t) complete implies PV_X(t-1) complete: O_X is stable here
          if (j >= 1 && __any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
              uint32_t orr[32];
              tmem_ld32(tO + c * 32, orr);
              tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
              tmem_st32(tO + c * 32, orr);
            }
            tmem_st_wait();
          }
          // P = 2^(s * scale_log2 - m_use) as bf16 over columns 0..63 of S_X;
          // scaling and the row sum on packed f32x2 pairs, four sum chains
          const uint64_t sl2 = f2_pack(g.scale_log2, g.scale_log2);
          const uint64_t nm2 = f2_pack(-m_use, -m_use);
          uint64_t acc[4] = {0, 0, 0, 0};
          uint32_t pk[2][32];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              float x0, x1;
              f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[c][e]), __uint_as_float(sr[c][e + 1])), sl2, nm2),
                        x0, x1);
              // every exponential on the XU (ex2.approx): sending a quarter, three
              // eighths or half of them (by column pairs) to a cubic on the FMA pipe
              // measured 3 %, 15 % and 20 % slower -- the softmax is not XU-bound
              const float p0 = fast_exp2(x0);
              const float p1 = fast_exp2(x1);
              acc[(e >> 1) & 3] = f2_add(acc[(e >> 1) & 3], f2_pack(p0, p1));
              pk[c >> 1][(c & 1) * 16 + (e >> 1)] = pack_bf16x2(p0, p1);
            }
          }
          float a0, a1, b0, b1;
          f2_unpack(f2_add(acc[0], acc[1]), a0, a1);
          f2_unpack(f2_add(acc[2], acc[3]), b0, b1);
          const float psum = (a0 + b0) + (a1 + b1);
          tmem_st32(tS, pk[0]);
          tmem_st32(tS + 32, pk[1]);
          tmem_st_wait();
          l = l * alpha + psum;
          m = m_use;
          tc_fence_before();
          mbar_arrive(&meta->p_full[X]);
        }
      }
      if (!ok) break;
      // epilogue: O_X / l_X for the rows of real tokens
      if (active) {
        if (!wait_warp(&meta->o_ready[X], items_x++ & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int tok = X * Tq + row / G;
        const float inv = 1.f / l;
        const bool store = tok < info.ntok;
        const int64_t obase =
            (static_cast<int64_t>(info.row0 + tok) * g.num_heads + info.hk * G + row % G) * D;
        if (!info.causal) {
          // shared prefix: one of the request's last split-KV partitions (m, l, o).
          // Every lane takes part in the TMEM loads; only the stores depend on the row.
          const int r = info.row0 + tok;
          const int part = store && r < g.num_qrows ? ws.nparts[r] - prefix_chunks + info.chunk : -1;
          const bool put = part >= 0 && part < ws.max_parts;
          if (store && !put && g.err_word) atomicOr(g.err_word, PA_ERRBIT_BLOCK_OOB);
          const int64_t slot =
              (static_cast<int64_t>(r) * g.num_heads + info.hk * G + row % G) * ws.max_parts + part;
          if (put) ws.part_ml[slot] = make_float2(m, l);
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r32[32];
            tmem_ld32(tO + c * 32, r32);
            tmem_ld_wait();
            if (put) {
              float4* po = reinterpret_cast<float4*>(ws.part_o + slot * D + c * 32);
#pragma unroll
              for (int e = 0; e < 8; ++e)
                po[e] = make_float4(__uint_as_float(r32[4 * e]), __uint_as_float(r32[4 * e + 1]),
                                    __uint_as_float(r32[4 * e + 2]), __uint_as_float(r32[4 * e + 3]));
            }
          }
        } else {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(tO + c * 32, r);
            tmem_ld_wait();
            if (store) {
              if (g.out_dtype == PA_F32) {
                float4* o4 = reinterpret_cast<float4*>(static_cast<float*>(g.out) + obase + c * 32);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                  o4[e] = make_float4(__uint_as_float(r[4 * e]) * inv, __uint_as_float(r[4 * e + 1]) * inv,
                                      __uint_as_float(r[4 * e + 2]) * inv,
                                      __uint_as_float(r[4 * e + 3]) * inv);
              } else {
                uint4* o4 =
                    reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(g.out) + obase + c * 32);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  o4[e] = make_uint4(
                      pack_bf16x2(__uint_as_float(r[8 * e]) * inv, __uint_as_float(r[8 * e + 1]) * inv),
                      pack_bf16x2(__uint_as_float(r[8 * e + 2]) * inv, __uint_as_float(r[8 * e + 3]) * inv),
                      pack_bf16x2(__uint_as_float(r[8 * e + 4]) * inv, __uint_as_float(r[8 * e + 5]) * inv),
                      pack_bf16x2(__uint_as_float(r[8 * e + 6]) * inv, __uint_as_float(r[8 * e + 7]) * inv));
              }
            }
          }
        }
      }
      if (!ok) break;
      tc_fence_before();
      mbar_arrive(&meta->o_empty);
    }
    if (!ok && g.err_word && row == 0) atomicOr(g.err_word, PA_ERRBIT_TIMEOUT);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ----------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFnTc)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                    const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                    const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                    CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFnTc encode_fn_tc() {
  static EncodeTiledFnTc fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFnTc>(p);
  }
  return fn;
}

bool tc_path_supported(const AttnGeom& g) {
  const int G = g.num_kv_heads > 0 ? g.num_heads / g.num_kv_heads : 0;
  return g.dtype == PA_BF16 && (g.head_dim == 64 || g.head_dim == 128) && G >= 1 && G <= 16 &&
         (tck::kRows % G) == 0 && encode_fn_tc() != nullptr &&
         static_cast<int64_t>(g.num_blocks) * g.block_size < (1LL << 31);
}

int tc_tokens_per_tile(const AttnGeom& g) {
  return 2 * tck::kRows / (g.num_heads / g.num_kv_heads);  // a pair of query tiles
}

template <int D>
static cudaError_t launch_tc_t(const AttnGeom& g, const WsView& ws, int num_sms, cudaStream_t s) {
  using C = tck::Cfg<D>;
  const int G = g.num_heads / g.num_kv_heads;
  // q viewed as (dim, head, token); one box = 64 dims x G heads x 256/G tokens
  CUtensorMap tq;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(g.num_heads),
                        static_cast<cuuint64_t>(g.num_qrows)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2,
                           static_cast<cuuint64_t>(D) * 2 * g.num_heads};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(G), static_cast<cuuint32_t>(2 * tck::kRows / G)};
  cuuint32_t estr[3] = {1, 1, 1};
  if (encode_fn_tc()(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(g.q), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  return launch_pdl<attn_tc_kernel<D>>(dim3(num_sms), dim3(tck::kThreads), C::kSmem, s, tq, g,
                                       ws);
}

cudaError_t launch_attn_tc(const AttnGeom& g, const WsView& ws, int grid, cudaStream_t s) {
  if (g.head_dim == 128) return launch_tc_t<128>(g, ws, grid, s);
  return launch_tc_t<64>(g, ws, grid, s);
}

}  // namespace pa
