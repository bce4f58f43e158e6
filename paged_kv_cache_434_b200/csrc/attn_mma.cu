// attn_mma.cu -- bf16 paged attention for query rows that see a long key range
// (decode rows, split-KV partitions): TMA-staged K/V tiles, one K/V read serving
// all query heads of a GQA group, tensor-core (mma.sync m16n8k16) products.
//
// Math as in attn_common.cu ("AI Infra入门干货总结：大模型是如何高效推理的",
// "Attention (FlashAttention, Scaled Dot-Product Attention)" and "总结").
//
// Layout and work split
//   * Pools are [num_blocks, block_size, Hkv, D] bf16.  A stage is 16
//     consecutive keys of one request.  In shared memory each (64-column
//     half of D, KV head) pair holds a [16 keys x 64 dims] tile (2 KiB,
//     128-byte swizzle), tiles of one half stored head after head.  With
//     block_size >= 16 the tensor map walks (dim, token, head), so ONE TMA box
//     [64 dims x 16 tokens x HG heads] fills a whole half (16 KiB per copy, 4
//     copies per stage); with block_size 8 a stage spans two blocks and each
//     head's tile takes two [64 x 8] boxes from a (dim, head, token) map.
//   * A persistent CTA = HG consumer warps (warp w owns KV head w of the
//     group) + 1 producer warp.  The producer pulls items from a global
//     counter, walks their block tables and keeps NS stages in flight
//     (full/empty mbarriers); stage descriptors travel with the stage.
//   * Consumer warp: the G query heads of its KV head are the rows of a
//     16-row A tile (rows >= G are zero), S = Q K^T uses K as the col-major B
//     operand (ldmatrix), P V uses V through ldmatrix.trans.  Row max and
//     row sums are reduced over the 4 lanes of a quad with xor shuffles; the
//     running (m, l, O) live in registers for the whole item.
#include <cuda.h>
#include <cuda_bf16.h>

#include <cmath>

#include "internal.h"
#include "ptx.cuh"

namespace pa {

namespace mmak {

enum : int { kFirst = 1, kLast = 2, kBad = 4, kEnd = 8 };
constexpr float kRescaleLog2 = 8.f;  // lazy O rescale threshold (log2 units)

struct StageInfo {
  int qrow;
  int b;
  int hg;
  int part;
  int nvalid;
  int flags;
  int np;  // partitions of the item's row
  int pad1;
};

// F8: e4m3 pools (head_dim 128).  A stage then holds [16 keys x 128 codes]
// per head and tensor (one 128-byte swizzled row per key, the same 2 KiB tile
// size).  K fragments are widened in registers straight from an ldmatrix of
// the codes (the dimension order inside each 16-dim step is permuted, and the
// query fragments follow the same order).  V fragments come from a transposed
// ldmatrix of the codes too: a lane receives the code pairs (dims 2g, 2g+1)
// of keys 2t and 2t+1, and one byte permute turns them into the key pairs of
// dim 2g and of dim 2g+1 -- the B operands of two n8 tiles that hold the even
// and the odd dims of a 16-dim chunk.  The output rows are put back in dim
// order when they are stored.
template <int D, int HG, bool F8 = false>
struct Cfg {
  static constexpr int NH = F8 ? 1 : D / 64;            // tiles per head and tensor in a stage
  static constexpr int kTile = 2048;                    // [16 keys x 128 bytes]
  static constexpr int kTensorBytes = HG * NH * kTile;  // K (or V) part of a stage
  static constexpr int kStageBytes = 2 * kTensorBytes;
  static constexpr int kBudget = 200 * 1024;
  static constexpr int NS0 = kBudget / kStageBytes;
  static constexpr int NS = NS0 > 6 ? 6 : (NS0 < 2 ? 2 : NS0);
  static constexpr int kThreads = (HG + 1) * 32;
  static constexpr int kSmem = NS * kStageBytes + 1024 /*align*/ + 1024 /*info+bars*/;
};

// byte offset of (key, 16-byte chunk) inside one 128B-swizzled [16 x 64] tile
__device__ __forceinline__ uint32_t swz(int key, int chunk) {
  return static_cast<uint32_t>(key * 128 + ((chunk ^ (key & 7)) << 4));
}

}  // namespace mmak

template <int D, int HG, bool F8>
__global__ void __launch_bounds__((HG + 1) * 32, 1)
    attn_mma_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    AttnGeom g, WsView ws, int box_rows, int by_token, int after_tiles) {
  static_assert(!F8 || D == 128, "e4m3 pools: head_dim 128");
  using C = mmak::Cfg<D, HG, F8>;
  constexpr int NS = C::NS;
  constexpr int NH = C::NH;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* stages = smem;
  mmak::StageInfo* info = reinterpret_cast<mmak::StageInfo*>(smem + NS * C::kStageBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(info + NS);
  uint64_t* empty = full + NS;
  __shared__ int s_abort;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], HG);
    }
    s_abort = 0;
    fence_mbar_init();
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  __syncthreads();
  // (no early launch_dependents: the merge has no prologue to overlap, and an
  // early launch of it measured slower than launching it at our completion)
  // Launched right after the tensor-core tile kernel (after_tiles), this grid
  // starts once every tile CTA has passed its own wait on the planner, so the
  // plan is complete; the tiles' results are not read here.  It then runs
  // beside the tile CTAs still at work and waits for them only before it
  // exits, so that the merge (which waits for this grid) sees both.
  if (!after_tiles) grid_dependency_wait();

  const int n_items = __ldcg(&ws.ctrl[1]);
  const int G = g.num_heads / g.num_kv_heads;

  if (warp == HG) {
    // ------------------------------------------------------------- producer
    if (lane != 0) return;
    const uint64_t policy = l2_policy_evict_first();
    int stage = 0;
    uint32_t phase = 0;
    int round = 0;  // completed passes over the ring
    bool ok = true;
    for (;;) {
      const int it = atomicAdd(&ws.ctrl[0], 1);
      const bool done = it >= n_items;
      int4 item = make_int4(0, 0, 0, 0), qi = make_int4(0, 0, 0, 0);
      int np = 1;
      if (!done) {
        item = __ldcg(&ws.items[it]);
        qi = __ldcg(&ws.qrow_info[item.x]);
        np = __ldcg(&ws.nparts[item.x]);
      }
      // keys [key_start + 16 first, + 16 stages) of the row (after a shared
      // prefix, if any); lo >= hi: empty item, skipped; never past the table
      const int lo = qi.w + item.w * kStageTokens;
      const int hi =
          done ? lo + 1
               : static_cast<int>(min(static_cast<int64_t>(lo) + static_cast<int64_t>(item.z) *
                                                                   kStageTokens,
                                      static_cast<int64_t>(min(qi.y, g.max_blocks * g.block_size))));
      const int hg = item.y & kItemHgMask, part = item.y >> kItemPartShift;
      const int32_t* table = g.block_tables + static_cast<int64_t>(qi.x) * g.max_blocks;
      for (int key0 = lo; key0 < hi; key0 += kStageTokens) {
        if (round > 0 && !mbar_wait_bounded(&empty[stage], phase ^ 1, kWaitLimitNs)) {
          ok = false;
          break;
        }
        mmak::StageInfo si;
        si.qrow = item.x;
        si.b = qi.x;
        si.hg = hg;
        si.part = part;
        si.np = np;
        si.nvalid = min(kStageTokens, hi - key0);
        si.flags = done ? mmak::kEnd
                        : ((key0 == lo ? mmak::kFirst : 0) |
                           (key0 + kStageTokens >= hi ? mmak::kLast : 0));
        int rows0 = 0, rows1 = -1;
        if (!done) {
          const int phys0 = table[key0 / g.block_size];
          if (phys0 < 0 || phys0 >= g.num_blocks) si.flags |= mmak::kBad;
          rows0 = phys0 * g.block_size + key0 % g.block_size;
          if (box_rows < kStageTokens && si.nvalid > box_rows) {
            const int phys1 = table[(key0 + box_rows) / g.block_size];
            if (phys1 < 0 || phys1 >= g.num_blocks) si.flags |= mmak::kBad;
            rows1 = phys1 * g.block_size + (key0 + box_rows) % g.block_size;
          }
        }
        info[stage] = si;
        if (done || (si.flags & mmak::kBad)) {
          mbar_arrive(&full[stage]);
        } else {
          uint8_t* kbase = stages + stage * C::kStageBytes;
          uint8_t* vbase = kbase + C::kTensorBytes;
          const int head0 = hg * HG;
          // The branch follows the kind of map the host encoded (by_token), and
          // each branch announces exactly the bytes of the boxes it issues.
          if (by_token) {
            // (dim, token, head) map, box [64 | 128 codes, 16 tokens, HG heads]:
            // one box per half and tensor
            mbar_arrive_expect_tx(&full[stage], 2u * NH * HG * C::kTile);
#pragma unroll
            for (int dh = 0; dh < NH; ++dh) {
              const int toff = dh * HG * C::kTile;
              tma_load_3d_hint(kbase + toff, &tmK, &full[stage], dh * 64, rows0, head0, policy);
              tma_load_3d_hint(vbase + toff, &tmV, &full[stage], dh * 64, rows0, head0, policy);
            }
          } else {
            // (dim, head, token) map, box [64 | 128 codes, 1 head, box_rows
            // tokens]: one box per head, half, tensor and block
            const int boxes = rows1 >= 0 ? 2 : 1;
            const uint32_t box_bytes = static_cast<uint32_t>(box_rows) * 128u;
            mbar_arrive_expect_tx(&full[stage], 2u * HG * NH * boxes * box_bytes);
#pragma unroll
            for (int hh = 0; hh < HG; ++hh) {
#pragma unroll
              for (int dh = 0; dh < NH; ++dh) {
                const int toff = (dh * HG + hh) * C::kTile;
                tma_load_3d_hint(kbase + toff, &tmK, &full[stage], dh * 64, head0 + hh, rows0,
                                 policy);
                tma_load_3d_hint(vbase + toff, &tmV, &full[stage], dh * 64, head0 + hh, rows0,
                                 policy);
                if (rows1 >= 0) {
                  tma_load_3d_hint(kbase + toff + box_bytes, &tmK, &full[stage], dh * 64,
                                   head0 + hh, rows1, policy);
                  tma_load_3d_hint(vbase + toff + box_bytes, &tmV, &full[stage], dh * 64,
                                   head0 + hh, rows1, policy);
                }
              }
            }
          }
        }
        if (++stage == NS) {
          stage = 0;
          phase ^= 1;
          ++round;
        }
      }
      if (!ok || done) break;
    }
    if (!ok) {
      s_abort = 1;
      if (g.err_word) atomicOr(g.err_word, PA_ERRBIT_TIMEOUT);
    }
    return;
  }

  // --------------------------------------------------------------- consumers
  const int hh = warp;  // KV head within the group
  const int qr = lane >> 2;      // fragment row (and row + 8)
  const int qc = (lane & 3) * 2; // fragment column pair
  uint32_t qa[D / 16][4];
  float o[D / 8][4];
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  bool bad = false;
  int stage = 0;
  uint32_t phase = 0;
  const __nv_bfloat16* qbase = static_cast<const __nv_bfloat16*>(g.q);
  // score and output scales (the pools' k_scale / v_scale are already in g)
  const float sl2 = g.scale_log2;
  const float vsc = g.v_scale;
  constexpr bool kPair = F8;

  for (;;) {
    if (!mbar_wait_bounded(&full[stage], phase, kWaitLimitNs)) {
      if (g.err_word && lane == 0) atomicOr(g.err_word, PA_ERRBIT_TIMEOUT);
      break;
    }
    const mmak::StageInfo si = info[stage];
    if (si.flags & mmak::kEnd) break;
    const int head = (si.hg * HG + hh) * G;  // first query head of this warp's group
    if (si.flags & mmak::kFirst) {
      const __nv_bfloat16* qrow = qbase + (static_cast<int64_t>(si.qrow) * g.num_heads + head) * D;
      // F8: k slots (2j, 2j+1 | 2j+8, 2j+9) of a 16-dim step hold dims
      // (4j, 4j+1 | 4j+2, 4j+3), the order the widened K fragments come in
      const int c_lo = F8 ? 4 * (lane & 3) : qc, c_hi = F8 ? c_lo + 2 : qc + 8;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int c = kk * 16 + c_lo, ch = kk * 16 + c_hi;
        qa[kk][0] = qr < G ? *reinterpret_cast<const uint32_t*>(qrow + qr * D + c) : 0u;
        qa[kk][1] = qr + 8 < G ? *reinterpret_cast<const uint32_t*>(qrow + (qr + 8) * D + c) : 0u;
        qa[kk][2] = qr < G ? *reinterpret_cast<const uint32_t*>(qrow + qr * D + ch) : 0u;
        qa[kk][3] =
            qr + 8 < G ? *reinterpret_cast<const uint32_t*>(qrow + (qr + 8) * D + ch) : 0u;
      }
      if constexpr (F8) {
        // f16 operands: bf16 queries are exact in f16 within +-65504
        bool out_of_range = false;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f =
                __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qa[kk][i]));
            out_of_range |= fabsf(f.x) > 65504.f || fabsf(f.y) > 65504.f;
            qa[kk][i] = pack_f16x2(f.x, f.y);
          }
        if (out_of_range && g.err_word) atomicOr(g.err_word, PA_ERRBIT_Q_RANGE);
      }
#pragma unroll
      for (int j = 0; j < D / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
      m0 = m1 = -INFINITY;
      l0 = l1 = 0.f;
      bad = false;
    }
    // F8: the next stage, when it belongs to the same item, is taken with this
    // one: one softmax pass over 32 keys and twice the independent products
    // per pass (the e4m3 path is bound by the latency of each warp's chain)
    int stage2 = -1;
    mmak::StageInfo si2 = si;
    if (kPair && !(si.flags & (mmak::kLast | mmak::kBad))) {
      const int s2 = stage + 1 == NS ? 0 : stage + 1;
      const uint32_t ph2 = stage + 1 == NS ? phase ^ 1u : phase;
      if (!mbar_wait_bounded(&full[s2], ph2, kWaitLimitNs)) {
        if (g.err_word && lane == 0) atomicOr(g.err_word, PA_ERRBIT_TIMEOUT);
        break;
      }
      si2 = info[s2];
      if (!(si2.flags & mmak::kBad)) stage2 = s2;  // a bad stage is taken alone
      else si2 = si;
    }
    if (si.flags & mmak::kBad) {
      bad = true;
    } else {
      constexpr uint32_t kHalf = HG * C::kTile;  // between the two halves (bf16)
      // ---- S = Q K^T over the 16 keys of stage stg
      auto qk = [&](int stg, float* a0, float* a1) {
        const uint32_t kt = smem_u32(stages + stg * C::kStageBytes) + hh * C::kTile;
        if constexpr (F8) {
          // one ldmatrix of the code tile gives two 16-dim steps x 16 keys: a
          // lane holds 4 codes (dims 4j..4j+3) of one key per matrix
          const int mi = lane >> 3;
          const int key = (lane & 7) + ((mi & 1) << 3);
          // two accumulator chains per half (even and odd 16-dim steps): the
          // dependent mma chain of a stage is half as long
          float t0[4] = {0.f, 0.f, 0.f, 0.f}, t1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int kk = 0; kk < D / 16; kk += 2) {
            uint32_t r[4];
            ldmatrix_x4(kt + mmak::swz(key, kk + (mi >> 1)), r[0], r[1], r[2], r[3]);
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              const uint32_t lo = e4m3x2_to_f16x2(static_cast<uint16_t>(r[m] & 0xffffu));
              const uint32_t hi = e4m3x2_to_f16x2(static_cast<uint16_t>(r[m] >> 16));
              float* acc = (m >> 1) ? ((m & 1) ? t1 : t0) : ((m & 1) ? a1 : a0);
              mma_f16_16816(acc, qa[kk + (m >> 1)], lo, hi);
            }
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            a0[e] += t0[e];
            a1[e] += t1[e];
          }
        } else {
          const int mi = lane >> 3;
          const int key = (lane & 7) + ((mi >> 1) << 3);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int dh = kk >> 2, c16 = kk & 3;
            const int chunk = 2 * c16 + (mi & 1);
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4(kt + dh * kHalf + mmak::swz(key, chunk), b0, b1, b2, b3);
            mma_bf16_16816(a0, qa[kk], b0, b1);
            mma_bf16_16816(a1, qa[kk], b2, b3);
          }
        }
      };
      // ---- O += P V over the 16 keys of stage stg (nv of them valid)
      auto pv = [&](int stg, const uint32_t* pa, int nv) {
        const uint32_t vt = smem_u32(stages + stg * C::kStageBytes) + hh * C::kTile + C::kTensorBytes;
        // keys past the end of the request: zero their V rows (P is 0 there,
        // but the pool may hold non-finite garbage and 0 * inf is NaN)
        if (!F8 && nv < kStageTokens) {
          uint8_t* vrow = stages + stg * C::kStageBytes + C::kTensorBytes + hh * C::kTile;
          for (int idx = lane; idx < (kStageTokens - nv) * 8 * NH; idx += 32) {
            const int dh = idx / ((kStageTokens - nv) * 8);
            const int rem = idx % ((kStageTokens - nv) * 8);
            const int key = nv + rem / 8, chunk = rem % 8;
            *reinterpret_cast<uint4*>(vrow + dh * HG * C::kTile + mmak::swz(key, chunk)) =
                make_uint4(0, 0, 0, 0);
          }
          __syncwarp();
        }
        if constexpr (F8) {
          // matrices: keys 0-7 / 8-15 of code chunk 2q, then of chunk 2q + 1
          const int mi = lane >> 3;
          const int key = (lane & 7) + ((mi & 1) << 3);
          // keys past the end of the request: their (possibly NaN) codes are
          // zeroed after widening, as halves of the key pairs (2t, 2t+1) and
          // (2t+8, 2t+9) this lane holds
          const int t2 = 2 * (lane & 3);
          const bool tail = nv < kStageTokens;  // only a request's last stage
          const uint32_t mk0 = (t2 < nv ? 0x0000ffffu : 0u) | (t2 + 1 < nv ? 0xffff0000u : 0u);
          const uint32_t mk1 = (t2 + 8 < nv ? 0x0000ffffu : 0u) | (t2 + 9 < nv ? 0xffff0000u : 0u);
#pragma unroll
          for (int q = 0; q < D / 32; ++q) {
            uint32_t r[4];
            ldmatrix_x4_trans(vt + mmak::swz(key, 2 * q + (mi >> 1)), r[0], r[1], r[2], r[3]);
#pragma unroll
            for (int h = 0; h < 2; ++h) {  // code chunk 2q + h: even dims, then odd dims
              const uint32_t lo = prmt_b32(r[2 * h], 0x3120u), hi = prmt_b32(r[2 * h + 1], 0x3120u);
              uint32_t e0 = e4m3x2_to_f16x2(static_cast<uint16_t>(lo & 0xffffu));
              uint32_t e1 = e4m3x2_to_f16x2(static_cast<uint16_t>(hi & 0xffffu));
              uint32_t d0 = e4m3x2_to_f16x2(static_cast<uint16_t>(lo >> 16));
              uint32_t d1 = e4m3x2_to_f16x2(static_cast<uint16_t>(hi >> 16));
              if (tail) {
                e0 &= mk0, d0 &= mk0;
                e1 &= mk1, d1 &= mk1;
              }
              mma_f16_16816(o[2 * (2 * q + h)], pa, e0, e1);
              mma_f16_16816(o[2 * (2 * q + h) + 1], pa, d0, d1);
            }
          }
        } else {
          const int mi = lane >> 3;
          const int key = (lane & 7) + ((mi & 1) << 3);
#pragma unroll
          for (int n2 = 0; n2 < D / 16; ++n2) {
            const int dh = n2 >> 2, c16 = n2 & 3;
            const int chunk = 2 * c16 + (mi >> 1);
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4_trans(vt + dh * kHalf + mmak::swz(key, chunk), b0, b1, b2, b3);
            mma_bf16_16816(o[2 * n2], pa, b0, b1);
            mma_bf16_16816(o[2 * n2 + 1], pa, b2, b3);
          }
        }
        if (!F8 && nv < kStageTokens) fence_proxy_async_smem();
      };
      float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
      float u0[4] = {0.f, 0.f, 0.f, 0.f}, u1[4] = {0.f, 0.f, 0.f, 0.f};
      if (kPair && stage2 >= 0) {
        // both stages' products in one unrolled loop: independent chains interleave
        const uint32_t ka = smem_u32(stages + stage * C::kStageBytes) + hh * C::kTile;
        const uint32_t kb = smem_u32(stages + stage2 * C::kStageBytes) + hh * C::kTile;
        const int mi = lane >> 3;
        const int key = (lane & 7) + ((mi & 1) << 3);
#pragma unroll
        for (int kk = 0; kk < D / 16; kk += 2) {
          uint32_t ra[4], rb[4];
          ldmatrix_x4(ka + mmak::swz(key, kk + (mi >> 1)), ra[0], ra[1], ra[2], ra[3]);
          ldmatrix_x4(kb + mmak::swz(key, kk + (mi >> 1)), rb[0], rb[1], rb[2], rb[3]);
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const int step = kk + (m >> 1);
            mma_f16_16816((m & 1) ? s1 : s0, qa[step],
                          e4m3x2_to_f16x2(static_cast<uint16_t>(ra[m] & 0xffffu)),
                          e4m3x2_to_f16x2(static_cast<uint16_t>(ra[m] >> 16)));
            mma_f16_16816((m & 1) ? u1 : u0, qa[step],
                          e4m3x2_to_f16x2(static_cast<uint16_t>(rb[m] & 0xffffu)),
                          e4m3x2_to_f16x2(static_cast<uint16_t>(rb[m] >> 16)));
          }
        }
      } else {
        qk(stage, s0, s1);
      }
      // ---- mask, scale, online softmax (over both stages when paired)
      const int nv = si.nvalid, nv2 = stage2 >= 0 ? si2.nvalid : 0;
      float p[8], p2[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = qc + (e & 1);
        p[e] = key < nv ? s0[e] * sl2 : -INFINITY;
        p[4 + e] = key + 8 < nv ? s1[e] * sl2 : -INFINITY;
        p2[e] = key < nv2 ? u0[e] * sl2 : -INFINITY;
        p2[4 + e] = key + 8 < nv2 ? u1[e] * sl2 : -INFINITY;
      }
      float mx0 = fmaxf(fmaxf(fmaxf(p[0], p[1]), fmaxf(p[4], p[5])),
                        fmaxf(fmaxf(p2[0], p2[1]), fmaxf(p2[4], p2[5])));
      float mx1 = fmaxf(fmaxf(fmaxf(p[2], p[3]), fmaxf(p[6], p[7])),
                        fmaxf(fmaxf(p2[2], p2[3]), fmaxf(p2[6], p2[7])));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      // lazy rescale: the reference max moves only when a row's max grows by
      // more than 2^8 (the weights then stay <= 256, exact enough in bf16 / f16
      // and fp32), so in steady state O is not touched; (m, l, o) stay
      // consistent for any reference, and the merge re-normalises partials
      const bool up0 = mx0 > m0 + mmak::kRescaleLog2, up1 = mx1 > m1 + mmak::kRescaleLog2;
      const float mn0 = up0 ? mx0 : m0, mn1 = up1 ? mx1 : m1;
      const float a0 = up0 ? fast_exp2(m0 - mn0) : 1.f, a1 = up1 ? fast_exp2(m1 - mn1) : 1.f;
      const bool rescale = __any_sync(0xffffffffu, up0 || up1);
      m0 = mn0;
      m1 = mn1;
      // P as the A fragment of the PV product; the row sums use the same
      // rounded weights the product sees
      auto weights = [&](const float* q, uint32_t* pa, float& ps0, float& ps1) {
        const float e0 = fast_exp2(q[0] - mn0), e1 = fast_exp2(q[1] - mn0);
        const float e2 = fast_exp2(q[2] - mn1), e3 = fast_exp2(q[3] - mn1);
        const float e4 = fast_exp2(q[4] - mn0), e5 = fast_exp2(q[5] - mn0);
        const float e6 = fast_exp2(q[6] - mn1), e7 = fast_exp2(q[7] - mn1);
        float2 f0, f1, f2, f3;
        if constexpr (F8) {
          pa[0] = pack_f16x2(e0, e1);
          pa[1] = pack_f16x2(e2, e3);
          pa[2] = pack_f16x2(e4, e5);
          pa[3] = pack_f16x2(e6, e7);
          f0 = f16x2_to_f32x2(pa[0]), f1 = f16x2_to_f32x2(pa[1]);
          f2 = f16x2_to_f32x2(pa[2]), f3 = f16x2_to_f32x2(pa[3]);
        } else {
          pa[0] = pack_bf16x2(e0, e1);
          pa[1] = pack_bf16x2(e2, e3);
          pa[2] = pack_bf16x2(e4, e5);
          pa[3] = pack_bf16x2(e6, e7);
          const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(pa);
          f0 = __bfloat1622float2(h[0]), f1 = __bfloat1622float2(h[1]);
          f2 = __bfloat1622float2(h[2]), f3 = __bfloat1622float2(h[3]);
        }
        ps0 += f0.x + f0.y + f2.x + f2.y;
        ps1 += f1.x + f1.y + f3.x + f3.y;
      };
      uint32_t pa[4], pa2[4];
      float ps0 = 0.f, ps1 = 0.f;
      weights(p, pa, ps0, ps1);
      if (stage2 >= 0) weights(p2, pa2, ps0, ps1);
      l0 = l0 * a0 + ps0;
      l1 = l1 * a1 + ps1;
      if (rescale) {
#pragma unroll
        for (int j = 0; j < D / 8; ++j) {
          o[j][0] *= a0;
          o[j][1] *= a0;
          o[j][2] *= a1;
          o[j][3] *= a1;
        }
      }
      if (kPair && stage2 >= 0) {
        // both stages in one unrolled loop (the first is whole: it is not an
        // item's last stage; the second may end the request)
        const uint32_t va = smem_u32(stages + stage * C::kStageBytes) + hh * C::kTile + C::kTensorBytes;
        const uint32_t vb = smem_u32(stages + stage2 * C::kStageBytes) + hh * C::kTile + C::kTensorBytes;
        const int mi = lane >> 3;
        const int key = (lane & 7) + ((mi & 1) << 3);
        const int t2 = 2 * (lane & 3);
        const bool tail = nv2 < kStageTokens;
        const uint32_t mk0 = (t2 < nv2 ? 0x0000ffffu : 0u) | (t2 + 1 < nv2 ? 0xffff0000u : 0u);
        const uint32_t mk1 = (t2 + 8 < nv2 ? 0x0000ffffu : 0u) | (t2 + 9 < nv2 ? 0xffff0000u : 0u);
#pragma unroll
        for (int q = 0; q < D / 32; ++q) {
          uint32_t ra[4], rb[4];
          ldmatrix_x4_trans(va + mmak::swz(key, 2 * q + (mi >> 1)), ra[0], ra[1], ra[2], ra[3]);
          ldmatrix_x4_trans(vb + mmak::swz(key, 2 * q + (mi >> 1)), rb[0], rb[1], rb[2], rb[3]);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t la = prmt_b32(ra[2 * h], 0x3120u), ha = prmt_b32(ra[2 * h + 1], 0x3120u);
            const uint32_t lb = prmt_b32(rb[2 * h], 0x3120u), hb = prmt_b32(rb[2 * h + 1], 0x3120u);
            uint32_t e0 = e4m3x2_to_f16x2(static_cast<uint16_t>(lb & 0xffffu));
            uint32_t e1 = e4m3x2_to_f16x2(static_cast<uint16_t>(hb & 0xffffu));
            uint32_t d0 = e4m3x2_to_f16x2(static_cast<uint16_t>(lb >> 16));
            uint32_t d1 = e4m3x2_to_f16x2(static_cast<uint16_t>(hb >> 16));
            if (tail) {
              e0 &= mk0, d0 &= mk0;
              e1 &= mk1, d1 &= mk1;
            }
            mma_f16_16816(o[2 * (2 * q + h)], pa, e4m3x2_to_f16x2(static_cast<uint16_t>(la & 0xffffu)),
                          e4m3x2_to_f16x2(static_cast<uint16_t>(ha & 0xffffu)));
            mma_f16_16816(o[2 * (2 * q + h) + 1], pa, e4m3x2_to_f16x2(static_cast<uint16_t>(la >> 16)),
                          e4m3x2_to_f16x2(static_cast<uint16_t>(ha >> 16)));
            mma_f16_16816(o[2 * (2 * q + h)], pa2, e0, e1);
            mma_f16_16816(o[2 * (2 * q + h) + 1], pa2, d0, d1);
          }
        }
      } else {
        pv(stage, pa, nv);
      }
    }
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&empty[stage]);
      if (stage2 >= 0) mbar_arrive(&empty[stage2]);
    }
    if (stage2 >= 0) {  // the paired stage is consumed too
      if (++stage == NS) {
        stage = 0;
        phase ^= 1;
      }
    }

    if (si2.flags & mmak::kLast) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
      l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
      const int r = si.qrow;
      if (bad) {
        if (lane == 0) {
          ws.qrow_bad[r] = 1;
          if (g.err_word) atomicOr(g.err_word, PA_ERRBIT_BLOCK_OOB);
        }
      } else {
        const int np = si.np;
        if (F8) {
          // o[2c] holds the even dims of chunk c, o[2c + 1] the odd ones: this
          // lane's four values of a row are dims 16c + 4t .. 16c + 4t + 3
          const int t4 = 4 * (lane & 3);
          const bool direct = np == 1;
          const float i0 = direct ? vsc / l0 : vsc, i1 = direct ? vsc / l1 : vsc;
          float* dst0 = nullptr;
          float* dst1 = nullptr;
          __nv_bfloat16* bdst0 = nullptr;
          __nv_bfloat16* bdst1 = nullptr;
          if (direct) {
            const int64_t ob = (static_cast<int64_t>(r) * g.num_heads + head) * D;
            if (g.out_dtype == PA_F32) {
              dst0 = static_cast<float*>(g.out) + ob + qr * D;
              dst1 = dst0 + 8 * D;
            } else {
              bdst0 = static_cast<__nv_bfloat16*>(g.out) + ob + qr * D;
              bdst1 = bdst0 + 8 * D;
            }
          } else {
            const int64_t slot0 =
                (static_cast<int64_t>(r) * g.num_heads + head) * ws.max_parts + si.part;
            const int64_t sl0 = slot0 + static_cast<int64_t>(qr) * ws.max_parts;
            const int64_t sl1 = slot0 + static_cast<int64_t>(qr + 8) * ws.max_parts;
            if ((lane & 3) == 0 && qr < G) ws.part_ml[sl0] = make_float2(m0, l0);
            if ((lane & 3) == 0 && qr + 8 < G) ws.part_ml[sl1] = make_float2(m1, l1);
            dst0 = ws.part_o + sl0 * D;
            dst1 = ws.part_o + sl1 * D;
          }
#pragma unroll
          for (int c = 0; c < D / 16; ++c) {
            const float4 v0 = make_float4(o[2 * c][0] * i0, o[2 * c + 1][0] * i0,
                                          o[2 * c][1] * i0, o[2 * c + 1][1] * i0);
            const float4 v1 = make_float4(o[2 * c][2] * i1, o[2 * c + 1][2] * i1,
                                          o[2 * c][3] * i1, o[2 * c + 1][3] * i1);
            if (bdst0) {
              if (qr < G)
                *reinterpret_cast<uint2*>(bdst0 + c * 16 + t4) =
                    make_uint2(pack_bf16x2(v0.x, v0.y), pack_bf16x2(v0.z, v0.w));
              if (qr + 8 < G)
                *reinterpret_cast<uint2*>(bdst1 + c * 16 + t4) =
                    make_uint2(pack_bf16x2(v1.x, v1.y), pack_bf16x2(v1.z, v1.w));
            } else {
              if (qr < G) *reinterpret_cast<float4*>(dst0 + c * 16 + t4) = v0;
              if (qr + 8 < G) *reinterpret_cast<float4*>(dst1 + c * 16 + t4) = v1;
            }
          }
        } else if (np == 1) {
          const float i0 = vsc / l0, i1 = vsc / l1;
          const int64_t ob = (static_cast<int64_t>(r) * g.num_heads + head) * D;
          if (g.out_dtype == PA_F32) {
            float* out = static_cast<float*>(g.out) + ob;
#pragma unroll
            for (int j = 0; j < D / 8; ++j) {
              if (qr < G)
                *reinterpret_cast<float2*>(out + qr * D + j * 8 + qc) =
                    make_float2(o[j][0] * i0, o[j][1] * i0);
              if (qr + 8 < G)
                *reinterpret_cast<float2*>(out + (qr + 8) * D + j * 8 + qc) =
                    make_float2(o[j][2] * i1, o[j][3] * i1);
            }
          } else {
            __nv_bfloat16* out = static_cast<__nv_bfloat16*>(g.out) + ob;
#pragma unroll
            for (int j = 0; j < D / 8; ++j) {
              if (qr < G)
                *reinterpret_cast<uint32_t*>(out + qr * D + j * 8 + qc) =
                    pack_bf16x2(o[j][0] * i0, o[j][1] * i0);
              if (qr + 8 < G)
                *reinterpret_cast<uint32_t*>(out + (qr + 8) * D + j * 8 + qc) =
                    pack_bf16x2(o[j][2] * i1, o[j][3] * i1);
            }
          }
        } else {
          const int64_t slot0 = (static_cast<int64_t>(r) * g.num_heads + head) * ws.max_parts + si.part;
          if (qr < G) {
            const int64_t sl = slot0 + static_cast<int64_t>(qr) * ws.max_parts;
            if ((lane & 3) == 0) ws.part_ml[sl] = make_float2(m0, l0);
            float* po = ws.part_o + sl * D;
#pragma unroll
            for (int j = 0; j < D / 8; ++j)
              *reinterpret_cast<float2*>(po + j * 8 + qc) =
                  make_float2(o[j][0] * vsc, o[j][1] * vsc);
          }
          if (qr + 8 < G) {
            const int64_t sl = slot0 + static_cast<int64_t>(qr + 8) * ws.max_parts;
            if ((lane & 3) == 0) ws.part_ml[sl] = make_float2(m1, l1);
            float* po = ws.part_o + sl * D;
#pragma unroll
            for (int j = 0; j < D / 8; ++j)
              *reinterpret_cast<float2*>(po + j * 8 + qc) =
                  make_float2(o[j][2] * vsc, o[j][3] * vsc);
          }
        }
      }
    }
    if (++stage == NS) {
      stage = 0;
      phase ^= 1;
    }
  }
  if (after_tiles) grid_dependency_wait();
}

// ----------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Pool views for TMA.  heads_per_box == 1: (dim, head, token) with box
// [64, 1, box_rows]; heads_per_box > 1: (dim, token, head) with box
// [64, 16, heads_per_box] -- the same memory walked with the token stride as
// the second dimension, so one box holds 16 tokens of several heads.
static bool make_pool_map(CUtensorMap* m, const void* base, const AttnGeom& g, int box_rows,
                          int heads_per_box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  // e4m3 pools: bytes; a box row is the head's 128 codes (one 128-byte row)
  const bool f8 = g.dtype == PA_FP8_E4M3;
  const cuuint64_t head_stride = static_cast<cuuint64_t>(g.head_dim) * (f8 ? 1 : 2);
  const cuuint64_t token_stride = head_stride * g.num_kv_heads;
  const cuuint64_t tokens = static_cast<cuuint64_t>(g.num_blocks) * g.block_size;
  const bool by_token = heads_per_box > 1;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(g.head_dim),
                        by_token ? tokens : static_cast<cuuint64_t>(g.num_kv_heads),
                        by_token ? static_cast<cuuint64_t>(g.num_kv_heads) : tokens};
  cuuint64_t strides[2] = {by_token ? token_stride : head_stride,
                           by_token ? head_stride : token_stride};
  cuuint32_t box[3] = {f8 ? 128u : 64u, by_token ? static_cast<cuuint32_t>(box_rows) : 1u,
                       by_token ? static_cast<cuuint32_t>(heads_per_box)
                                : static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, f8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                  const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool mma_path_supported(const AttnGeom& g) {
  const int G = g.num_kv_heads > 0 ? g.num_heads / g.num_kv_heads : 0;
  const bool bs_ok = g.block_size == 8 || (g.block_size % 16 == 0 && g.block_size <= 256);
  const bool type_ok = g.dtype == PA_BF16 ||
                       (g.dtype == PA_FP8_E4M3 && g.head_dim == 128 && g.block_size % 16 == 0);
  return type_ok && (g.head_dim == 64 || g.head_dim == 128) && G >= 1 && G <= kMaxGroup &&
         bs_ok && encode_fn() != nullptr &&
         static_cast<int64_t>(g.num_blocks) * g.block_size < (1LL << 31);
}

template <int D, int HG, bool F8 = false>
static cudaError_t launch_mma_t(const AttnGeom& g, const WsView& ws, int num_sms, int after_tiles,
                                cudaStream_t s) {
  using C = mmak::Cfg<D, HG, F8>;
  const int box_rows = g.block_size < kStageTokens ? g.block_size : kStageTokens;
  CUtensorMap tk, tv;
  int heads_per_box = (box_rows == kStageTokens && HG > 1) ? HG : 1;
  if (heads_per_box > 1 && !(make_pool_map(&tk, g.k_cache, g, box_rows, heads_per_box) &&
                             make_pool_map(&tv, g.v_cache, g, box_rows, heads_per_box)))
    heads_per_box = 1;  // the driver refused the token-major view: one box per head
  if (heads_per_box == 1 && !(make_pool_map(&tk, g.k_cache, g, box_rows, 1) &&
                              make_pool_map(&tv, g.v_cache, g, box_rows, 1)))
    return cudaErrorInvalidValue;
  auto kern = attn_mma_kernel<D, HG, F8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, C::kThreads, C::kSmem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  // the kernel's choice of box coordinates must follow the map just encoded
  const int by_token = heads_per_box > 1 ? 1 : 0;
  return launch_pdl<attn_mma_kernel<D, HG, F8>>(dim3(num_sms * per_sm), dim3(C::kThreads),
                                                C::kSmem, s, tk, tv, g, ws, box_rows, by_token,
                                                after_tiles);
}

cudaError_t launch_attn_mma(const AttnGeom& g, const WsView& ws, int num_sms, int heads_per_group,
                            int after_tiles, cudaStream_t s) {
  if (g.dtype == PA_FP8_E4M3) {  // head_dim 128 (mma_path_supported)
    switch (heads_per_group) {
      case 8: return launch_mma_t<128, 8, true>(g, ws, num_sms, after_tiles, s);
      case 4: return launch_mma_t<128, 4, true>(g, ws, num_sms, after_tiles, s);
      case 2: return launch_mma_t<128, 2, true>(g, ws, num_sms, after_tiles, s);
      default: return launch_mma_t<128, 1, true>(g, ws, num_sms, after_tiles, s);
    }
  }
  if (g.head_dim == 128) {
    switch (heads_per_group) {
      case 8: return launch_mma_t<128, 8>(g, ws, num_sms, after_tiles, s);
      case 4: return launch_mma_t<128, 4>(g, ws, num_sms, after_tiles, s);
      case 2: return launch_mma_t<128, 2>(g, ws, num_sms, after_tiles, s);
      default: return launch_mma_t<128, 1>(g, ws, num_sms, after_tiles, s);
    }
  }
  switch (heads_per_group) {
    case 8: return launch_mma_t<64, 8>(g, ws, num_sms, after_tiles, s);
    case 4: return launch_mma_t<64, 4>(g, ws, num_sms, after_tiles, s);
    case 2: return launch_mma_t<64, 2>(g, ws, num_sms, after_tiles, s);
    default: return launch_mma_t<64, 1>(g, ws, num_sms, after_tiles, s);
  }
}

}  // namespace pa
