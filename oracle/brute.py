"""Brute-force attention in pure Python (lists, math.exp) -- TEST INFRASTRUCTURE ONLY.

Deliberately naive restatement of softmax(Q K^T * scale + M) V for tiny
inputs, written without NumPy so that it cannot share a mistake with the
vectorised oracle in attention.py.  Follows "AI Infra入门干货总结：大模型是如何
高效推理的", section "Attention (FlashAttention, Scaled Dot-Product
Attention)": GQA map kv = h // (num_heads // num_kv_heads), scaled scores,
future keys masked, softmax over the allowed keys, weighted sum of V.
"""

from __future__ import annotations

import math


def brute_attention(q, K, V, scale, first_pos):
    """q: nested lists [n_q][num_heads][D]; K, V: [L][num_kv_heads][D].

    Query i is at position first_pos + i and sees keys 0 .. first_pos + i.
    Returns nested lists [n_q][num_heads][D] of Python floats.

    Source: "AI Infra入门干货总结：大模型是如何高效推理的", "Attention (FlashAttention, Scaled Dot-Product Attention)",
    written out with loops and math.exp only.
    """
    n_q = len(q)
    num_heads = len(q[0])
    D = len(q[0][0])
    L = len(K)
    num_kv_heads = len(K[0]) if L else 1
    group = num_heads // num_kv_heads
    out = []
    for i in range(n_q):
        row = []
        for h in range(num_heads):
            kv = h // group
            visible = min(L, first_pos + i + 1)
            scores = []
            for j in range(visible):
                dot = 0.0
                for d in range(D):
                    dot += float(q[i][h][d]) * float(K[j][kv][d])
                scores.append(scale * dot)
            if not scores:
                row.append([0.0] * D)
                continue
            biggest = max(scores)
            weights = [math.exp(s - biggest) for s in scores]
            total = sum(weights)
            o = []
            for d in range(D):
                acc = 0.0
                for j in range(visible):
                    acc += weights[j] * float(V[j][kv][d])
                o.append(acc / total)
            row.append(o)
        out.append(row)
    return out
