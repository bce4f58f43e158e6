"""float64/bit-level oracle for the block-management steps around the paged
cache -- TEST INFRASTRUCTURE ONLY (see the package docstring).

Sources (page title, section):
  * "第三部分 · 推理系统与基础设施" (liuzhe1218.github.io llm-learning-path,
    part 3), chapter map, 3.3 "批处理与内存管理": PagedAttention block
    tables with copy-on-write -- requests that share physical blocks (after a
    fork, or a shared prefix) keep sharing them until one of them writes; the
    writer first gets its own copy of the block.
  * "AI Infra入门干货总结：大模型是如何高效推理的", section "Paged Attention":
    a token's slot is block_table[request][pos // block_size] * block_size +
    pos % block_size (the slot function in oracle/attention.py, pinned by the
    page's worked example).

Readings:
  * A copy request is a (source block, destination block) pair; the whole
    block (every offset, every KV head, every dimension) of both pools is
    copied.  Pairs of one call are applied as if one after another; a block
    that is the destination of one pair and the source of another in the same
    call is outside the contract (the tests never build one).
  * Building slot_mapping from explicit (request, position) pairs is the
    same slot function applied per token; a negative request index marks a
    padding token (slot -1, no error).
"""

from __future__ import annotations

import numpy as np

from .attention import ERR_BLOCK_OOB, slot_of

ERR_POS_OOB_TABLE = "position_outside_block_table"


def copy_blocks(k_pool, v_pool, mapping):
    """Return copies of the pools with block dst := block src for each
    (src, dst) row of mapping; pairs naming a block outside the pool are
    reported and skipped.  Works on any dtype (bit-exact).

    Source: "第三部分 · 推理系统与基础设施", chapter map 3.3 (copy-on-write:
    a request about to write into a shared block first gets its own copy).
    """
    kp = np.array(k_pool, copy=True)
    vp = np.array(v_pool, copy=True)
    nb = kp.shape[0]
    errors = set()
    for src, dst in np.asarray(mapping).reshape(-1, 2):
        src, dst = int(src), int(dst)
        if not (0 <= src < nb and 0 <= dst < nb):
            errors.add(ERR_BLOCK_OOB)
            continue
        kp[dst] = kp[src]
        vp[dst] = vp[src]
    return kp, vp, errors


def slot_mapping_positions(block_tables, token_req, positions, block_size: int, num_blocks: int):
    """slot of every token from its request's block table and its position."""
    block_tables = np.asarray(block_tables)
    n_req, width = block_tables.shape
    out = np.full(len(positions), -1, dtype=np.int64)
    errors = set()
    for t, (b, p) in enumerate(zip(np.asarray(token_req), np.asarray(positions))):
        b, p = int(b), int(p)
        if b < 0:
            continue                                   # padding token
        if b >= n_req or p < 0 or p >= width * block_size:
            errors.add(ERR_POS_OOB_TABLE)
            continue
        phys = int(block_tables[b, p // block_size])
        if not 0 <= phys < num_blocks:
            errors.add(ERR_BLOCK_OOB)
            continue
        out[t] = slot_of(block_tables[b], p, block_size)
    return out, errors
