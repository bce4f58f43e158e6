"""float64 NumPy oracle: slot mapping, cache write, paged gather, attention.

TEST INFRASTRUCTURE ONLY (see the package docstring).  Plain loops over
sequences and heads, NumPy matmul as the only library primitive, no blocking
or fusion beyond what the definitions state.

Notation follows "AI Infra入门干货总结：大模型是如何高效推理的", sections
"Paged Attention" and "Attention (FlashAttention, Scaled Dot-Product
Attention)":
  key_cache / value_cache : [num_blocks, block_size, num_kv_heads, head_dim]
  block_table             : [num_reqs, max_num_blocks_per_req] physical ids
  slot_mapping            : one slot per new token,
                            slot = block_idx * block_size + block_offset
  seq_lens                : KV length of a request after this step
                            (num_computed_tokens + new tokens)
  query_lens              : new tokens of the request in this step
  cu_seqlens / query_start_loc : offsets of each request in the flattened
                            [num_sched_tokens, ...] query array
"""

from __future__ import annotations

import numpy as np

# Error conditions the oracle reports (names, not bit values: the CUDA library
# numbers its own error bits and the tests translate).
ERR_SLOT_OOB = "slot_out_of_range"          # slot >= num_blocks * block_size
ERR_BLOCK_OOB = "block_id_out_of_range"     # block_table entry outside the pool
ERR_SEQ_TOO_LONG = "seq_len_exceeds_table"  # seq_len > max_blocks * block_size
ERR_QUERY_TOO_LONG = "query_len_exceeds_seq_len"  # q_b > L_b


# --------------------------------------------------------------------------
# Slot arithmetic ("Paged Attention": slot_mapping code and worked example)
# --------------------------------------------------------------------------

def slot_of(block_table_row, pos: int, block_size: int) -> int:
    """Slot of logical token position `pos` of one request.

    The logical block is pos // block_size; the request's block table turns it
    into a physical block id; the offset inside the block is pos % block_size;
    slot = physical_block * block_size + offset.  (Worked example on the page:
    block_size 16, table [5, 8, 12], position 25 -> logical 1 -> physical 8,
    offset 9, slot 137.)
    """
    logical_block = pos // block_size
    physical_block = int(block_table_row[logical_block])
    offset = pos % block_size
    return physical_block * block_size + offset


def slot_mapping(block_tables, query_start_loc, seq_lens, block_size: int):
    """Slot of every new token of a flattened step.

    Request b owns the flattened tokens query_start_loc[b] .. query_start_loc[b+1]-1.
    Its q_b new tokens are the LAST q_b positions of its sequence of length
    L_b, i.e. token i sits at position L_b - q_b + i (seq_lens counts the
    computed tokens plus the new ones; "附2：推理运行时变量": 105 computed + 1
    new -> seq_lens 106).
    """
    qsl = np.asarray(query_start_loc, dtype=np.int64)
    lens = np.asarray(seq_lens, dtype=np.int64)
    num_tokens = int(qsl[-1])
    out = np.full(num_tokens, -1, dtype=np.int64)
    for b in range(len(lens)):
        q_b = int(qsl[b + 1] - qsl[b])
        L_b = int(lens[b])
        for i in range(q_b):
            pos = L_b - q_b + i
            out[qsl[b] + i] = slot_of(block_tables[b], pos, block_size)
    return out


# --------------------------------------------------------------------------
# Cache write (reshape_and_cache: scatter each new K/V row to its slot)
# --------------------------------------------------------------------------

def cache_write(k_cache, v_cache, k, v, slots):
    """Return copies of the two pools with row t of k / v stored at slots[t].

    block_idx = slot // block_size, block_offset = slot % block_size, and the
    whole [num_kv_heads, head_dim] row is copied.  Works on any dtype
    (including raw bit patterns), so the result can be compared byte for byte.

    A negative slot marks a padding token and is skipped; a slot beyond the
    pool is reported and skipped.  Returns (k_cache', v_cache', errors).
    """
    num_blocks, block_size = k_cache.shape[0], k_cache.shape[1]
    k_out = k_cache.copy()
    v_out = v_cache.copy()
    errors = set()
    for t, slot in enumerate(np.asarray(slots, dtype=np.int64)):
        slot = int(slot)
        if slot < 0:
            continue
        if slot >= num_blocks * block_size:
            errors.add(ERR_SLOT_OOB)
            continue
        block_idx, block_offset = divmod(slot, block_size)
        k_out[block_idx, block_offset] = k[t]
        v_out[block_idx, block_offset] = v[t]
    return k_out, v_out, errors


# --------------------------------------------------------------------------
# Gather through the block table into a contiguous [L, num_kv_heads, head_dim]
# --------------------------------------------------------------------------

def gather(cache, block_table_row, length: int):
    """Logical K (or V) of one request: row p is cache[table[p // bs], p % bs].

    Source: "AI Infra入门干货总结：大模型是如何高效推理的", "Paged Attention" (the block table maps a logical block to
    its physical block; the offset inside the block is p % block_size).
    """
    block_size = cache.shape[1]
    rows = [cache[int(block_table_row[p // block_size]), p % block_size]
            for p in range(length)]
    if not rows:
        return np.zeros((0,) + cache.shape[2:], dtype=np.float64)
    return np.stack(rows).astype(np.float64)


# --------------------------------------------------------------------------
# Attention on contiguous K/V (scaled dot product, causal mask, GQA)
# --------------------------------------------------------------------------

def _kv_head(h: int, num_heads: int, num_kv_heads: int) -> int:
    """GQA map: kv_head_idx = q_head_idx // (num_heads // num_kv_heads)."""
    return h // (num_heads // num_kv_heads)


def _scores(q_h, K_kv, scale, first_pos):
    """Masked scores of one head: s[i, j] = scale * <q_i, k_j>, -inf if j > first_pos + i.

    Query i of the chunk is at absolute position first_pos + i and may see
    keys 0 .. first_pos + i (causal within the new tokens, full over the
    cached prefix).
    """
    s = scale * (q_h @ K_kv.T)
    n_q, L = s.shape
    allowed = np.arange(L)[None, :] <= (first_pos + np.arange(n_q))[:, None]
    return np.where(allowed, s, -np.inf)


def attend_two_pass(q, K, V, scale: float, first_pos: int):
    """softmax(Q K^T * scale + M) V with the max / sum taken over the full row.

    q: [n_q, num_heads, D]; K, V: [L, num_kv_heads, D]; returns [n_q, num_heads, D].
    Pass 1 takes m = max_j s_ij; pass 2 forms w_ij = exp(s_ij - m_i),
    l_i = sum_j w_ij and o_i = sum_j w_ij v_j / l_i.

    Source: "AI Infra入门干货总结：大模型是如何高效推理的", "Attention (FlashAttention, Scaled Dot-Product Attention)"
    (its table of steps: GQA head map, Q K^T, scale, mask, softmax, P V).
    """
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    n_q, num_heads, D = q.shape
    num_kv_heads = K.shape[1]
    out = np.zeros((n_q, num_heads, D), dtype=np.float64)
    if K.shape[0] == 0:
        return out
    for h in range(num_heads):
        kv = _kv_head(h, num_heads, num_kv_heads)
        s = _scores(q[:, h, :], K[:, kv, :], scale, first_pos)
        m = s.max(axis=1, keepdims=True)                     # pass 1
        w = np.exp(s - m)                                    # pass 2 (exp(-inf) = 0)
        l = w.sum(axis=1, keepdims=True)
        out[:, h, :] = (w @ V[:, kv, :]) / l
    return out


def attend_online(q, K, V, scale: float, first_pos: int, tile: int = 16):
    """The same attention computed with the online (streaming) softmax.

    Keys are consumed `tile` at a time.  Per query row the running max m, the
    running denominator l and the unnormalised output o are kept; when a tile
    raises the max from m_old to m_new, l and o are rescaled by
    exp(m_old - m_new) before the tile's exp(s - m_new) terms are added.  The
    final output is o / l.
    """
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    n_q, num_heads, D = q.shape
    L, num_kv_heads = K.shape[0], K.shape[1]
    out = np.zeros((n_q, num_heads, D), dtype=np.float64)
    if L == 0:
        return out
    for h in range(num_heads):
        kv = _kv_head(h, num_heads, num_kv_heads)
        s_all = _scores(q[:, h, :], K[:, kv, :], scale, first_pos)
        m = np.full(n_q, -np.inf)
        l = np.zeros(n_q)
        o = np.zeros((n_q, D))
        for j0 in range(0, L, tile):
            s = s_all[:, j0:j0 + tile]
            m_new = np.maximum(m, s.max(axis=1))
            # rows that have seen no allowed key yet keep m = -inf; use 0 there
            m_safe = np.where(np.isfinite(m_new), m_new, 0.0)
            alpha = np.where(np.isfinite(m), np.exp(m - m_safe), 0.0)
            p = np.exp(s - m_safe[:, None])
            l = alpha * l + p.sum(axis=1)
            o = alpha[:, None] * o + p @ V[j0:j0 + tile, kv, :]
            m = m_new
        out[:, h, :] = o / l[:, None]
    return out


def attend_partial(q, K, V, scale: float, first_pos: int, key_lo: int, key_hi: int):
    """Flash-Decoding partial over keys [key_lo, key_hi): (m, l, o_unnormalised).

    m[i, h] = max of the allowed scores in the range (-inf if none),
    l[i, h] = sum exp(s - m), o[i, h] = sum exp(s - m) v.

    Source: "AI Infra入门干货总结：大模型是如何高效推理的", "总结" (Flash-Decoding splits the key axis across SMs);
    "第三部分 · 推理系统与基础设施", chapter map 3.4.
    """
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    n_q, num_heads, D = q.shape
    num_kv_heads = K.shape[1]
    m_out = np.full((n_q, num_heads), -np.inf)
    l_out = np.zeros((n_q, num_heads))
    o_out = np.zeros((n_q, num_heads, D))
    for h in range(num_heads):
        kv = _kv_head(h, num_heads, num_kv_heads)
        s = _scores(q[:, h, :], K[:, kv, :], scale, first_pos)[:, key_lo:key_hi]
        if s.shape[1] == 0:
            continue
        m = s.max(axis=1)
        m_safe = np.where(np.isfinite(m), m, 0.0)
        w = np.exp(s - m_safe[:, None])
        m_out[:, h] = m
        l_out[:, h] = w.sum(axis=1)
        o_out[:, h, :] = w @ V[key_lo:key_hi, kv, :]
    return m_out, l_out, o_out


def merge_partials(parts):
    """Log-sum-exp merge of Flash-Decoding partials.

    With M = max_k m_k and weights c_k = exp(m_k - M):
    O = sum_k c_k o_k / sum_k c_k l_k.  Partials whose m_k is -inf (no
    allowed key) have c_k = 0.

    Source: "AI Infra入门干货总结：大模型是如何高效推理的", "总结" (the partial results are re-normalised with
    log-sum-exp).
    """
    ms = np.stack([p[0] for p in parts])            # [P, n_q, H]
    ls = np.stack([p[1] for p in parts])
    os_ = np.stack([p[2] for p in parts])           # [P, n_q, H, D]
    M = ms.max(axis=0)
    M_safe = np.where(np.isfinite(M), M, 0.0)
    c = np.where(np.isfinite(ms), np.exp(ms - M_safe[None]), 0.0)
    num = (c[..., None] * os_).sum(axis=0)
    den = (c * ls).sum(axis=0)
    return num / den[..., None]


def attend_split(q, K, V, scale: float, first_pos: int, num_parts: int):
    """Attention with the key axis cut into `num_parts` near-equal ranges and
    the partials merged by log-sum-exp (split-KV / Flash-Decoding)."""
    L = K.shape[0]
    edges = np.linspace(0, L, num_parts + 1).round().astype(int)
    parts = [attend_partial(q, K, V, scale, first_pos, int(edges[i]), int(edges[i + 1]))
             for i in range(num_parts)]
    return merge_partials(parts)


# --------------------------------------------------------------------------
# Paged attention over a whole flattened step
# --------------------------------------------------------------------------

def paged_mixed_step(q, k_cache, v_cache, block_tables, query_start_loc, seq_lens,
                     scale: float):
    """Causal varlen attention of a flattened continuous-batching step.

    q: [num_tokens, num_heads, D].  Request b's queries are rows
    query_start_loc[b] .. query_start_loc[b+1]-1 (q_b of them); its K/V are
    the first L_b = seq_lens[b] logical positions, gathered through
    block_tables[b] (the new tokens must already be in the cache).  Query i of
    b sits at position L_b - q_b + i.

    Returns (out [num_tokens, num_heads, D] float64, errors, valid_rows) where
    valid_rows marks the tokens whose output is defined: rows of a request
    with q_b > L_b or with L_b larger than the table are left as NaN and
    reported; a request with L_b == 0 (and q_b == 0) has no rows.
    """
    q = np.asarray(q, dtype=np.float64)
    num_tokens, num_heads, D = q.shape
    num_blocks, block_size = k_cache.shape[0], k_cache.shape[1]
    max_blocks = block_tables.shape[1]
    qsl = np.asarray(query_start_loc, dtype=np.int64)
    lens = np.asarray(seq_lens, dtype=np.int64)
    out = np.full((num_tokens, num_heads, D), np.nan)
    valid = np.zeros(num_tokens, dtype=bool)
    errors = set()
    for b in range(len(lens)):
        t0, t1 = int(qsl[b]), int(qsl[b + 1])
        q_b, L_b = t1 - t0, int(lens[b])
        if q_b == 0:
            continue
        if q_b > L_b:
            errors.add(ERR_QUERY_TOO_LONG)
            continue
        if L_b > max_blocks * block_size:
            errors.add(ERR_SEQ_TOO_LONG)
            continue
        needed = block_tables[b, : (L_b + block_size - 1) // block_size]
        if np.any((needed < 0) | (needed >= num_blocks)):
            errors.add(ERR_BLOCK_OOB)
            continue
        K = gather(k_cache, block_tables[b], L_b)
        V = gather(v_cache, block_tables[b], L_b)
        out[t0:t1] = attend_two_pass(q[t0:t1], K, V, scale, L_b - q_b)
        valid[t0:t1] = True
    return out, errors, valid


def paged_decode(q, k_cache, v_cache, block_tables, seq_lens, scale: float):
    """Decode: one query per request at position L_b - 1, seeing all L_b keys.

    q: [num_seqs, num_heads, D] -> (out [num_seqs, num_heads, D], errors, valid).
    A request with L_b == 0 attends to nothing; its output row is zero.

    Source: "AI Infra入门干货总结：大模型是如何高效推理的", "附2：推理运行时变量" (seq_lens counts the computed tokens
    plus the new one, so the decode query is the last position).
    """
    lens = np.asarray(seq_lens, dtype=np.int64)
    num_seqs = len(lens)
    q = np.asarray(q, dtype=np.float64)
    out = np.zeros_like(q)
    valid = np.ones(num_seqs, dtype=bool)
    errors = set()
    nonempty = lens > 0
    if nonempty.any():
        idx = np.nonzero(nonempty)[0]
        qsl = np.arange(len(idx) + 1, dtype=np.int64)
        o, errors, v = paged_mixed_step(q[idx], k_cache, v_cache, block_tables[idx],
                                        qsl, lens[idx], scale)
        out[idx] = o
        valid[idx] = v
    return out, errors, valid


def kv_cache_bytes(num_layers: int, num_kv_heads: int, head_dim: int,
                   bytes_per_elt: int, context_len: int) -> int:
    """Bytes of K and V cache for one sequence: layers x 2 x heads x dim x elt x tokens.

    Source: ursb.me Field Note "llm-inference-life", blurb (Llama-3-8B holds
    about 1 GB of KV cache at 8K context); "AI Infra入门干货总结：大模型是如何高效推理的", "附1：模型配置参数".
    """
    return num_layers * 2 * num_kv_heads * head_dim * bytes_per_elt * context_len
