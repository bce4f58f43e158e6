/*
 * pa.h -- C ABI of the paged-KV attention library (libpa_b200.so, sm_100a).
 *
 * Operations (names after the vLLM v1 walkthrough "AI Infra入门干货总结：大模型
 * 是如何高效推理的"):
 *   pa_slot_mapping   slot of every new token from the block tables
 *                     ("Paged Attention": slot = block_idx * block_size + offset,
 *                     worked example: block_size 16, table [5,8,12], pos 25 -> 137)
 *   pa_cache_write    reshape_and_cache: scatter each new token's K/V row to
 *                     its slot ("Reshape & Cache"; "Paged Attention")
 *   pa_slot_mapping_cache_write
 *                     the two above in one launch
 *   pa_decode         GQA decode attention over the paged cache, FlashAttention
 *                     online softmax, split-KV partitions merged by log-sum-exp
 *                     ("Attention (FlashAttention, Scaled Dot-Product Attention)";
 *                     "总结": Flash-Decoding re-normalises with log-sum-exp)
 *   pa_decode_step    a decode step's cache write and attention in one call:
 *                     pa_slot_mapping_cache_write (one new token per request)
 *                     then pa_decode, the write done in the planner's launch
 *   pa_mixed_step     causal varlen attention of a flattened continuous-batching
 *                     step mixing chunked-prefill tokens and decode tokens, every
 *                     K/V read through the block table (same section: the v1
 *                     unified varlen call over the paged cache)
 *   pa_rope_cos_sin_cache, pa_rope_cache_write
 *                     rotary position embedding of Q/K fused with the cache
 *                     write ("Reshape & Cache")
 *   pa_copy_blocks    copy-on-write block copies ("第三部分 · 推理系统与基础设施",
 *                     chapter map 3.3)
 *   pa_slot_mapping_positions
 *                     slots from explicit (request, position) pairs
 *   PA_FP8_E4M3       e4m3 cache pools with one scale per pool ("从零构建LLM
 *                     推理引擎", card "量化")
 *   pa_decode_no_alloc, pa_kernel_timing_enable / _read,
 *   pa_selftest_wait_timeout
 *                     entry points with no counterpart on the pages (a decode
 *                     for callers that cannot allocate; per-launch timing; a
 *                     check that a bounded device wait ends and reports)
 *
 * Conventions shared by every call
 *   - All tensor arguments are DEVICE pointers of the current CUDA device,
 *     row-major and densely packed, owned by the caller.  The library never
 *     allocates, frees or retains them, and keeps no state between calls
 *     other than a per-device cache of launch attributes (and, where those
 *     entry points are used, the no-alloc scratch and the timing events).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call
 *     is asynchronous: it validates on the host, enqueues kernels on `stream`
 *     and returns.  Host-detectable errors return a non-zero pa_status and
 *     enqueue nothing.
 *   - Cache pools: key_cache and value_cache are each
 *     [num_blocks, block_size, num_kv_heads, head_dim] (one layer), dtype
 *     cache->dtype (e4m3 codes for PA_FP8_E4M3, whose queries and new K/V
 *     rows are bf16).
 *   - Index arrays are int32 (block_tables, seq_lens, query_start_loc) except
 *     slot_mapping (int64, as in the page's reshape_and_cache code).
 *   - Device-detected errors never trap: the offending item is skipped and a
 *     PA_ERRBIT_* bit is OR-ed into *err_word (an int32 in device memory;
 *     may be NULL to discard).  pa_read_error() collects it.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pa_status {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, inconsistent shapes        */
  PA_ERR_UNSUPPORTED = 2,  /* valid but unsupported (dtype, head_dim, ...)       */
  PA_ERR_WORKSPACE = 3,    /* workspace pointer NULL or smaller than required    */
  PA_ERR_CUDA = 4,         /* a CUDA runtime call failed (launch, attribute ...) */
  PA_ERR_DEVICE_OOB = 5,   /* pa_read_error: the device found out-of-range input
                              (any error bit but PA_ERRBIT_TIMEOUT)              */
  PA_ERR_TIMEOUT = 6       /* pa_read_error: a bounded device wait gave up
                              (PA_ERRBIT_TIMEOUT set, whatever else is)          */
} pa_status;

/* PA_FP8_E4M3: the pools hold e4m3 codes (1 sign, 4 exponent bits with bias
 * 7, 3 mantissa bits; no infinities; 448 the largest magnitude) with one
 * float scale per pool (pa_cache_desc.k_scale / v_scale): an entry stands for
 * code * scale.  Queries, new K/V rows and rotated queries are bf16 then.
 * ("从零构建LLM 推理引擎", card "量化": halving the bits of every KV entry
 * nearly halves the bytes, and so the time, of each decoded token.) */
typedef enum pa_dtype { PA_F32 = 0, PA_BF16 = 1, PA_FP8_E4M3 = 2 } pa_dtype;

/* Device error bits (OR-ed into *err_word). */
#define PA_ERRBIT_SLOT_OOB 0x1        /* slot >= num_blocks * block_size           */
#define PA_ERRBIT_BLOCK_OOB 0x2       /* a needed block_tables entry not in [0,NB) */
#define PA_ERRBIT_SEQ_TOO_LONG 0x4    /* seq_len > max_blocks_per_seq * block_size */
#define PA_ERRBIT_QUERY_TOO_LONG 0x8  /* query_len > seq_len (or negative)         */
#define PA_ERRBIT_TIMEOUT 0x10        /* a bounded device wait gave up             */
#define PA_ERRBIT_POS_OOB 0x20        /* a rotary position outside the cos/sin table */
#define PA_ERRBIT_Q_RANGE 0x40        /* FP8 cache: a query entry beyond +-65504 (the
                                         tensor-core path takes queries as f16)  */

/* One layer's cache pools. */
typedef struct pa_cache_desc {
  int64_t num_blocks;    /* physical blocks in each pool                 */
  int32_t block_size;    /* tokens per block: 8, 16, 32, 64, 128 or 256  */
  int32_t num_kv_heads;  /* >= 1                                        */
  int32_t head_dim;      /* 64 or 128                                   */
  int32_t dtype;         /* pa_dtype of pools, q, k and v (FP8: pools
                            e4m3, q / k / v bf16)                       */
  float k_scale;         /* PA_FP8_E4M3: key entry = code * k_scale;
                            positive and finite; ignored otherwise      */
  float v_scale;         /* PA_FP8_E4M3: value entry = code * v_scale   */
} pa_cache_desc;

/* Static description of a status code; never NULL. */
const char* pa_status_str(int status);

/* Library ABI version (major * 100 + minor). */
int pa_version(void);

/*
 * pa_slot_mapping -- slot of every new token of a flattened step.
 * Request b owns flattened tokens query_start_loc[b] .. query_start_loc[b+1]-1;
 * its q_b new tokens are its last q_b positions, token i at position
 * p = seq_lens[b] - q_b + i, and
 *     slot = block_tables[b][p / block_size] * block_size + p % block_size.
 *   block_tables    int32 [num_seqs, max_blocks_per_seq]
 *   query_start_loc int32 [num_seqs + 1], non-decreasing, [num_seqs] == num_tokens
 *   seq_lens        int32 [num_seqs]
 *   slot_mapping    int64 [num_tokens] (output)
 * Tokens of a request whose q_b > seq_len or seq_len > max_blocks_per_seq *
 * block_size, or whose table entry is outside [0, num_blocks), get slot -1
 * and set the matching error bit.
 */
pa_status pa_slot_mapping(const int32_t* block_tables, int32_t max_blocks_per_seq,
                          const int32_t* query_start_loc, const int32_t* seq_lens,
                          int32_t num_seqs, int64_t num_tokens, int32_t block_size,
                          int64_t num_blocks, int64_t* slot_mapping, int32_t* err_word,
                          void* stream);

/*
 * pa_cache_write -- reshape_and_cache.
 * For every t < num_tokens with s = slot_mapping[t] >= 0:
 *     key_cache[s / block_size][s % block_size][:][:]   = k[t][:][:]
 *     value_cache[s / block_size][s % block_size][:][:] = v[t][:][:]
 *   k, v         [num_tokens, num_kv_heads, head_dim], dtype cache->dtype
 *   slot_mapping int64 [num_tokens]; a negative slot marks padding (skipped)
 * Bit-exact copy.  s >= num_blocks * block_size is skipped and sets
 * PA_ERRBIT_SLOT_OOB.  Two tokens with the same slot in one call: undefined.
 * PA_FP8_E4M3 pools: k and v are bf16 and each entry is stored as the e4m3
 * code of the float32 quotient x / scale, rounded to nearest (ties to even)
 * and saturated to +-448.
 */
pa_status pa_cache_write(const void* k, const void* v, void* key_cache, void* value_cache,
                         const int64_t* slot_mapping, int64_t num_tokens,
                         const pa_cache_desc* cache, int32_t* err_word, void* stream);

/*
 * pa_slot_mapping_cache_write -- pa_slot_mapping and pa_cache_write in one
 * launch (the walkthrough's two steps before attention: the slot of each new
 * token, then reshape_and_cache into it).  The same results as the two calls:
 * the slots (written to slot_mapping when it is not NULL), the pools, and the
 * error bits of both (a token whose request fails the slot checks, or whose
 * table entry is outside the pool, gets slot -1 and is not written).
 *   k, v, key_cache, value_cache, cache: as for pa_cache_write
 *   block_tables, max_blocks_per_seq, seq_lens, num_seqs: as for pa_slot_mapping
 *   query_start_loc int32 [num_seqs + 1] as for pa_slot_mapping, or NULL for a
 *                   decode step: one new token per request, token b of
 *                   request b (num_tokens must then equal num_seqs)
 *   slot_mapping    int64 [num_tokens] (output), may be NULL
 * Returns PA_ERR_INVALID_ARG for NULL or misaligned buffers, negative sizes or
 * a NULL query_start_loc with num_tokens != num_seqs; PA_ERR_UNSUPPORTED when
 * max_blocks_per_seq * block_size exceeds 2^30.
 */
pa_status pa_slot_mapping_cache_write(const void* k, const void* v, void* key_cache,
                                      void* value_cache, const int32_t* block_tables,
                                      int32_t max_blocks_per_seq, const int32_t* query_start_loc,
                                      const int32_t* seq_lens, int32_t num_seqs,
                                      int64_t num_tokens, const pa_cache_desc* cache,
                                      int64_t* slot_mapping, int32_t* err_word, void* stream);

/*
 * pa_copy_blocks -- copy-on-write block copies ("第三部分 · 推理系统与基础设施",
 * chapter map 3.3: requests that share physical blocks keep sharing them until
 * one writes; the writer first gets its own copy of the block).
 * For each pair i < num_pairs with (src, dst) = block_mapping[2i], [2i+1]:
 *     key_cache[dst] = key_cache[src] and value_cache[dst] = value_cache[src]
 * (whole blocks: block_size x num_kv_heads x head_dim elements, bit-exact).
 *   block_mapping int64 [num_pairs, 2], device memory
 * A pair naming a block outside [0, num_blocks) is skipped and sets
 * PA_ERRBIT_BLOCK_OOB.  A block that is the destination of one pair and the
 * source or destination of another pair of the same call: undefined.
 */
pa_status pa_copy_blocks(void* key_cache, void* value_cache, const int64_t* block_mapping,
                         int64_t num_pairs, const pa_cache_desc* cache, int32_t* err_word,
                         void* stream);

/*
 * pa_slot_mapping_positions -- slot of each token from an explicit request
 * index and position ("AI Infra入门干货总结：大模型是如何高效推理的", "Paged
 * Attention": slot = block_tables[b][p / block_size] * block_size +
 * p % block_size), for callers whose tokens are not the last q_b positions
 * of each request (pa_slot_mapping covers that case).
 *   token_req   int32 [num_tokens]: request index b, < 0 = padding (slot -1)
 *   positions   int64 [num_tokens]
 *   slot_mapping int64 [num_tokens] (output)
 * b >= num_seqs or p outside [0, max_blocks_per_seq * block_size): slot -1,
 * PA_ERRBIT_POS_OOB; a table entry outside [0, num_blocks): slot -1,
 * PA_ERRBIT_BLOCK_OOB.
 */
pa_status pa_slot_mapping_positions(const int32_t* block_tables, int32_t max_blocks_per_seq,
                                    int32_t num_seqs, const int32_t* token_req,
                                    const int64_t* positions, int64_t num_tokens,
                                    int32_t block_size, int64_t num_blocks,
                                    int64_t* slot_mapping, int32_t* err_word, void* stream);

/*
 * pa_rope_cos_sin_cache -- the rotary table, built once at start-up
 * ("AI Infra入门干货总结：大模型是如何高效推理的", section "Reshape & Cache":
 * cos_sin_cache of shape [max_position_embeddings, rotary_dim], indexed by
 * position at run time so that no sin/cos is evaluated per token).
 *   cache  float32 [max_position, rotary_dim] (output).  Row p holds
 *          cos(p * f_i) for i < rotary_dim / 2, then sin(p * f_i), with
 *          f_i = theta ** (-2 i / rotary_dim); angles, cos and sin in float64,
 *          rounded once to float32.  rope_theta is 500000 for Llama-3-8B
 *          (same article, "附1：模型配置参数").
 * rotary_dim must be even and > 0, max_position > 0, theta > 0.
 */
pa_status pa_rope_cos_sin_cache(float* cache, int32_t max_position, int32_t rotary_dim,
                                double theta, void* stream);

/*
 * pa_rope_cache_write -- rotary position embedding fused with reshape_and_cache
 * (same article, "Reshape & Cache": Q and K rotated by the position's rotation,
 * V unchanged, then K and V scattered into the pools through slot_mapping).
 * For token t with position p = positions[t] and each rotated pair (x1, x2)
 * of a Q or K head (angle a_i = p * f_i, cos/sin read from cos_sin_cache):
 *     (x1, x2) -> (x1 cos a_i - x2 sin a_i, x2 cos a_i + x1 sin a_i)
 * in float32, rounded to the cache dtype.  Pairs: neox != 0 pairs dimension i
 * with i + rotary_dim / 2, neox == 0 pairs 2i with 2i + 1; dimensions
 * >= rotary_dim are copied unchanged.
 *   q_in   token t's [num_heads, head_dim] row at q_in + t * q_stride
 *   k, v   token t's [num_kv_heads, head_dim] rows at k / v + t * kv_stride
 *          (strides in elements; the three may be column slices of one fused
 *          QKV projection output, e.g. q_stride = kv_stride =
 *          (num_heads + 2 * num_kv_heads) * head_dim)
 *   q_out  [num_tokens, num_heads, head_dim] rotated queries; may be q_in
 *          itself when q_stride == num_heads * head_dim, must not otherwise
 *          overlap it
 *   key_cache / value_cache, slot_mapping: as pa_cache_write (rotated K and
 *          plain V stored at the slot; negative slot = padding, skipped;
 *          slot past the pool: skipped, PA_ERRBIT_SLOT_OOB)
 *   positions int64 [num_tokens]; a position outside [0, max_position) sets
 *          PA_ERRBIT_POS_OOB, copies the token's queries unrotated to q_out
 *          and writes nothing to the pools
 *   cos_sin_cache float32 [max_position, rotary_dim] (pa_rope_cos_sin_cache)
 * rotary_dim: a multiple of 16, at most head_dim.  Strides: multiples of 8
 * elements.  dtype of q/k/v/q_out: cache->dtype.
 */
pa_status pa_rope_cache_write(const void* q_in, const void* k, const void* v, int64_t q_stride,
                              int64_t kv_stride, void* q_out, void* key_cache, void* value_cache,
                              const int64_t* positions, const int64_t* slot_mapping,
                              const float* cos_sin_cache, int32_t max_position,
                              int32_t rotary_dim, int32_t neox, int64_t num_tokens,
                              int32_t num_heads, const pa_cache_desc* cache, int32_t* err_word,
                              void* stream);

/* Bytes of workspace pa_decode needs for these sizes; 0 on bad arguments and
 * for sizes whose workspace would exceed 2^46 bytes (pa_decode then returns
 * PA_ERR_UNSUPPORTED). */
size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_heads,
                                int32_t max_blocks_per_seq, const pa_cache_desc* cache);

/*
 * pa_decode -- one query per request attends to all seq_lens[b] keys.
 *   q            [num_seqs, num_heads, head_dim], dtype cache->dtype
 *   block_tables int32 [num_seqs, max_blocks_per_seq]; entries past
 *                ceil(seq_lens[b] / block_size) are never read
 *   seq_lens     int32 [num_seqs]; the new token (already written by
 *                pa_cache_write) is position seq_lens[b] - 1
 *   scale        multiplies q.k before the softmax (1/sqrt(head_dim) usually)
 *   out          [num_seqs, num_heads, head_dim] of out_dtype (PA_F32 or PA_BF16)
 *   workspace    device buffer of >= pa_decode_workspace_size(...) bytes,
 *                256-byte aligned; contents need no initialisation.  One
 *                workspace must not be used by two calls that overlap on the GPU.
 * Query head h uses KV head h / (num_heads / num_kv_heads) (GQA).
 * seq_lens[b] == 0 writes a zero row.  Rows of requests with an error bit
 * (table entry outside the pool, seq_len too long) are left unwritten.
 */
pa_status pa_decode(const void* q, const void* key_cache, const void* value_cache,
                    const int32_t* block_tables, const int32_t* seq_lens, float scale,
                    void* out, int32_t num_seqs, int32_t num_heads, int32_t max_blocks_per_seq,
                    int32_t out_dtype, const pa_cache_desc* cache, void* workspace,
                    size_t workspace_bytes, int32_t* err_word, void* stream);

/*
 * pa_decode_step -- one decode step of one layer: each request's new K/V row
 * goes to its slot, then its query attends to all seq_lens[b] keys
 * ("AI Infra入门干货总结：大模型是如何高效推理的", sections "Reshape & Cache",
 * "Paged Attention" and "Attention (FlashAttention, Scaled Dot-Product
 * Attention)": the step writes the token's K/V into the paged cache before
 * the attention reads it).
 * Results, error bits and the rows left unwritten are exactly those of
 *     pa_slot_mapping_cache_write(k, v, key_cache, value_cache, block_tables,
 *         max_blocks_per_seq, NULL, seq_lens, num_seqs, num_seqs, cache,
 *         slot_mapping, err_word, stream)
 *     pa_decode(q, key_cache, value_cache, block_tables, seq_lens, scale, out,
 *         ..., workspace, workspace_bytes, err_word, stream)
 * made back to back; the write runs in the CTAs beside the work planner, in
 * the same launch, so it costs no launch of its own.
 *   k, v          [num_seqs, num_kv_heads, head_dim] new rows, token b of
 *                 request b at position seq_lens[b] - 1 (bf16 for PA_FP8_E4M3)
 *   slot_mapping  int64 [num_seqs] (output), may be NULL
 *   workspace     >= pa_decode_workspace_size(num_seqs, num_heads,
 *                 max_blocks_per_seq, cache) bytes, as for pa_decode
 *   other arguments as for pa_decode.
 * Returns what pa_decode returns for the same arguments, and PA_ERR_INVALID_ARG
 * for a NULL or misaligned k or v.  A status found on the host (every one but
 * PA_ERR_CUDA) launches nothing, so the pools are left as they were; after
 * PA_ERR_CUDA the launches before the failing one may have run.
 */
pa_status pa_decode_step(const void* q, const void* k, const void* v, void* key_cache,
                         void* value_cache, const int32_t* block_tables, const int32_t* seq_lens,
                         float scale, void* out, int32_t num_seqs, int32_t num_heads,
                         int32_t max_blocks_per_seq, int32_t out_dtype, const pa_cache_desc* cache,
                         int64_t* slot_mapping, void* workspace, size_t workspace_bytes,
                         int32_t* err_word, void* stream);

/* Bytes of workspace pa_mixed_step needs; 0 on bad arguments and beyond
 * 2^46 bytes, as for pa_decode_workspace_size. */
size_t pa_mixed_step_workspace_size(int32_t num_seqs, int64_t num_tokens, int32_t num_heads,
                                    int32_t max_blocks_per_seq, const pa_cache_desc* cache);

/*
 * pa_mixed_step -- causal varlen attention of a flattened step.
 *   q               [num_tokens, num_heads, head_dim]
 *   query_start_loc int32 [num_seqs + 1] (cu_seqlens of the queries)
 *   seq_lens        int32 [num_seqs], KV length after this step
 *   out             [num_tokens, num_heads, head_dim] of out_dtype
 * Query i of request b (flattened row query_start_loc[b] + i) sits at
 * position seq_lens[b] - q_b + i and attends to keys 0 .. that position
 * (causal inside the new tokens, full over the cached prefix).  The new
 * tokens' K/V must already be in the cache (pa_cache_write).  Requests may
 * appear in any order and with any mix of q_b == 1 (decode) and q_b > 1
 * (prefill chunk).  Rows of a request with q_b > seq_len are left unwritten
 * and set PA_ERRBIT_QUERY_TOO_LONG.  Workspace rules as for pa_decode.
 */
pa_status pa_mixed_step(const void* q, const void* key_cache, const void* value_cache,
                        const int32_t* block_tables, const int32_t* query_start_loc,
                        const int32_t* seq_lens, float scale, void* out, int32_t num_seqs,
                        int64_t num_tokens, int32_t num_heads, int32_t max_blocks_per_seq,
                        int32_t out_dtype, const pa_cache_desc* cache, void* workspace,
                        size_t workspace_bytes, int32_t* err_word, void* stream);

/*
 * pa_decode_no_alloc -- pa_decode without a caller-provided workspace.
 * The pages have no counterpart: this entry point exists for callers that
 * can't allocate device memory (a plug-in inside a host engine that owns all
 * device allocations and hands it no workspace; a runtime that forbids
 * cudaMalloc after start-up).  Its scratch is a static device array of
 * PA_DECODE_NO_ALLOC_MAX_BYTES that every GPU loading this library holds
 * until the process exits; the call itself allocates nothing.
 *   Arguments, layouts and results: exactly those of pa_decode (same kernels,
 *   same partition plan), minus workspace / workspace_bytes.
 *   Returns PA_ERR_WORKSPACE when pa_decode_workspace_size(...) for these
 *   sizes exceeds PA_DECODE_NO_ALLOC_MAX_BYTES (nothing is launched).
 *   The first call on a device looks up the array's address on that device
 *   (cudaGetSymbolAddress) and caches it; make that first call before any
 *   stream capture.  The cached address belongs to the device's current
 *   context: after a cudaDeviceReset of that device, this entry point must
 *   not be called again in the same process (it would hand the kernels the
 *   old context's address).  All calls share the array: two calls whose
 *   kernels overlap on the GPU race.  Nothing in it needs clearing between
 *   calls.
 */
#define PA_DECODE_NO_ALLOC_MAX_BYTES (32u << 20) /* 32 MiB of device memory per GPU */

pa_status pa_decode_no_alloc(const void* q, const void* key_cache, const void* value_cache,
                             const int32_t* block_tables, const int32_t* seq_lens, float scale,
                             void* out, int32_t num_seqs, int32_t num_heads,
                             int32_t max_blocks_per_seq, int32_t out_dtype,
                             const pa_cache_desc* cache, int32_t* err_word, void* stream);

/*
 * pa_kernel_timing_enable / pa_kernel_timing_read -- a measurement aid with no
 * counterpart on the pages: device time of each launch of one attention call.
 *   pa_kernel_timing_enable(1) creates PA_TIMED_KERNELS pairs of CUDA events on
 *   the current device; from then on every pa_decode / pa_mixed_step call made
 *   on that device records one pair around each of its launches, on the call's
 *   stream.  A recorded event between two launches ends the overlap that
 *   programmatic dependent launch otherwise gives them, so timed calls run each
 *   launch on its own: use it in a pass of its own, not in the timed steps.
 *   pa_kernel_timing_enable(0) destroys the events.  Not for concurrent use
 *   from several host threads.
 *   pa_kernel_timing_read waits for the last timed call's events and writes
 *   ms[PA_TIMED_KERNELS] (index PA_TK_*); -1 for a launch the call did not
 *   make.  Returns PA_ERR_INVALID_ARG when timing is off, nothing was timed
 *   since the last read, or ms is NULL; PA_ERR_CUDA if an event call failed.
 */
#define PA_TIMED_KERNELS 4
#define PA_TK_PLAN 0    /* work planner                                  */
#define PA_TK_TILES 1   /* tensor-core tiles (prefill or shared prefix)  */
#define PA_TK_DECODE 2  /* decode partitions                             */
#define PA_TK_MERGE 3   /* split-KV merge                                */

pa_status pa_kernel_timing_enable(int32_t enable);
pa_status pa_kernel_timing_read(float* ms);

/*
 * pa_read_error -- synchronise `stream`, copy *err_word to *host_bits and
 * reset it to 0.  Returns PA_OK when no bit was set, PA_ERR_TIMEOUT when
 * PA_ERRBIT_TIMEOUT was set, PA_ERR_DEVICE_OOB when only other bits were,
 * PA_ERR_CUDA if a CUDA call failed (e.g. an earlier kernel faulted).
 */
pa_status pa_read_error(int32_t* err_word, int32_t* host_bits, void* stream);

/*
 * pa_selftest_wait_timeout -- a check of the library's failure detection
 * (the pages have no counterpart).  Every mbarrier wait in the attention
 * kernels is bounded: when it runs out it sets PA_ERRBIT_TIMEOUT and the
 * kernel leaves its role, so a stalled pipeline ends its launch instead of
 * hanging the device.  A correct call never reaches that exit; this entry
 * point does, on purpose and harmlessly: it launches one warp whose lane 0
 * waits, through the same bounded-wait routine, on a shared-memory mbarrier
 * that nothing arrives at.
 *   limit_us   the wait's limit in microseconds, 1 .. 100000 (100 ms)
 *   err_word   device int32; PA_ERRBIT_TIMEOUT is OR-ed into it when the
 *              wait gives up (required)
 *   waited_ns  device uint64 or NULL: the wait's duration by the GPU's global
 *              timer, from its start to its end
 * Returns PA_ERR_INVALID_ARG for a limit outside the range or a NULL
 * err_word (nothing is launched), PA_ERR_CUDA if the launch failed, PA_OK
 * otherwise.  Asynchronous on `stream`; pa_read_error collects the bit.
 */
pa_status pa_selftest_wait_timeout(uint32_t limit_us, int32_t* err_word,
                                   unsigned long long* waited_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
