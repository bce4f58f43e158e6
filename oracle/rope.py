"""float64 oracle for rotary position embedding fused with the cache write.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Sources (page title, section):
  * "AI Infra入门干货总结：大模型是如何高效推理的", section "Reshape & Cache":
    the fused QKV output is split by columns into Q [tokens, num_heads*head_dim],
    K and V [tokens, num_kv_heads*head_dim]; Q and K are rotated by the
    block-diagonal rotation R_pos of the token's position (computed
    element-wise with sin/cos, dimensions unchanged); V is not rotated; then
    reshape_and_cache scatters K and V into the paged pools through
    slot_mapping.  The sin/cos values come from a cos_sin_cache of shape
    [max_position_embeddings, rotary_dim] built once at start-up and indexed
    by position.
  * same article, "附1：模型配置参数": rope_theta = 500000 for Llama-3-8B.
  * ursb.me Field Note "llm-inference-life", blurb (C06): every pair of Q/K
    dimensions is a point of the complex plane rotated by the angle m*theta,
    so that q.k depends on the positions only through m - n.

Readings (the pages leave these open):
  * Frequencies: the pair i (0 <= i < rotary_dim/2) turns by
    position * rope_theta ** (-2 i / rotary_dim) radians, the standard
    rotary schedule the "base theta" parameter names.
  * cos_sin_cache row p holds cos of the rotary_dim/2 angles followed by
    their sin (rotary_dim values, the page's [max_position, rotary_dim]).
  * Which dimensions form a pair: both conventions are provided.  neox=True
    pairs dimension i with i + rotary_dim/2 (the split-half layout Llama
    checkpoints use); neox=False pairs 2i with 2i+1 (adjacent dimensions).
    Dimensions at or past rotary_dim are left unchanged (partial rotary).
"""

from __future__ import annotations

import numpy as np

ERR_POS_OOB = "position_out_of_range"  # position < 0 or >= max_position


def inv_freq(rotary_dim: int, theta: float) -> np.ndarray:
    """theta ** (-2 i / rotary_dim) for i < rotary_dim / 2, float64.

    Source: "AI Infra入门干货总结：大模型是如何高效推理的", "附1：模型配置参数" (rope_theta); the schedule itself is the
    reading stated in this module's header.
    """
    i = np.arange(rotary_dim // 2, dtype=np.float64)
    return np.power(np.float64(theta), -2.0 * i / rotary_dim)


def cos_sin_table(max_position: int, rotary_dim: int, theta: float) -> np.ndarray:
    """[max_position, rotary_dim] float64: cos of every angle, then sin.

    Source: "AI Infra入门干货总结：大模型是如何高效推理的", "Reshape & Cache" (a cos_sin_cache of shape
    [max_position, rotary_dim] indexed by position).
    """
    ang = np.outer(np.arange(max_position, dtype=np.float64), inv_freq(rotary_dim, theta))
    return np.concatenate([np.cos(ang), np.sin(ang)], axis=1)


def pair_index(rotary_dim: int, neox: bool):
    """(first, second) dimension of each rotated pair i < rotary_dim / 2.

    Source: ursb.me Field Note "llm-inference-life", blurb (dimensions taken
    in pairs, each pair turned like a complex number); which dimensions form
    a pair is the reading stated in this module's header.
    """
    half = rotary_dim // 2
    i = np.arange(half)
    if neox:
        return i, i + half
    return 2 * i, 2 * i + 1


def rotate(x, positions, table, rotary_dim: int, neox: bool):
    """Rotate the heads of x [tokens, heads, head_dim] (float64) by each
    token's position: for pair i with angle a, (x1, x2) ->
    (x1 cos a - x2 sin a, x2 cos a + x1 sin a)."""
    x = np.asarray(x, dtype=np.float64)
    out = x.copy()
    half = rotary_dim // 2
    a, b = pair_index(rotary_dim, neox)
    for t, p in enumerate(np.asarray(positions)):
        c = table[int(p), :half]
        s = table[int(p), half:rotary_dim]
        x1 = x[t][:, a]
        x2 = x[t][:, b]
        out[t][:, a] = x1 * c - x2 * s
        out[t][:, b] = x2 * c + x1 * s
    return out


def rope_cache_write(q, k, v, positions, slots, k_pool, v_pool, table, rotary_dim: int,
                     neox: bool):
    """What the fused step produces: rotated queries, and the pools with each
    token's rotated K and plain V row placed at its slot.

    q [T, Hq, D], k/v [T, Hkv, D], positions/slots [T] ints, pools
    [num_blocks, block_size, Hkv, D] (float64 copies are returned).
    Tokens whose position is outside the table are reported and left alone
    (their q row unchanged, nothing written); negative slots are padding
    (q still rotated, nothing written); slots past the pool are reported.
    Returns (q_rot, k_pool, v_pool, errors, rotated_mask).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    kp = np.array(k_pool, dtype=np.float64, copy=True)
    vp = np.array(v_pool, dtype=np.float64, copy=True)
    nb, bs = kp.shape[0], kp.shape[1]
    errors = set()
    ok = np.array([0 <= int(p) < table.shape[0] for p in positions], dtype=bool)
    if not ok.all():
        errors.add(ERR_POS_OOB)
    pos_safe = np.where(ok, np.asarray(positions), 0)
    q_rot = np.where(ok[:, None, None], rotate(q, pos_safe, table, rotary_dim, neox), q)
    k_rot = rotate(k, pos_safe, table, rotary_dim, neox)
    for t, s in enumerate(np.asarray(slots)):
        s = int(s)
        if not ok[t] or s < 0:
            continue
        if s >= nb * bs:
            errors.add("slot_out_of_range")
            continue
        kp[s // bs, s % bs] = k_rot[t]
        vp[s // bs, s % bs] = v[t]
    return q_rot, kp, vp, errors, ok
