"""Algorithmic byte accounting for decode attention (host logic, no kernels).

The unit of work is one (sequence, attended position) pair of one layer.  The
bytes that must cross HBM for it are the cached key row and value row of every KV
head: ``n_kv_heads * head_dim * 2 bytes`` for K, the same again for V unless K
serves as V, in which case the one tensor is read once.  Queries, outputs, LSE
and split partials are overhead and are not counted.

The per-token formula of the "Gemma 4 12B" record (KV GEOMETRY paragraph) counts
K and V for every layer; ``count_shared_twice=True`` reproduces that figure.

An fp8 cache row is ``head_dim`` one-byte e4m3 codes plus its 4-byte scale.

A multi-token (verify) step of T tokens whose union of windows is read once
counts the positions of that union: min(L, w + T - 1) for a sliding layer.
"""
from __future__ import annotations

BF16_BYTES = 2


def kv_bytes_per_position(spec, count_shared_twice: bool = False) -> int:
    """KV bytes read for one attended position of one sequence in one layer."""
    tensors = 2 if (not spec.kv_shared or count_shared_twice) else 1
    return spec.n_kv_heads * spec.head_dim * BF16_BYTES * tensors


def attended_positions(spec, seqlen: int) -> int:
    """Positions one decode step attends: min(L, w) for a sliding layer, L otherwise."""
    return min(seqlen, spec.window) if spec.window > 0 else seqlen


def layer_kv_bytes(spec, seqlens) -> int:
    """Algorithmic KV bytes for one decode step of one layer over a batch."""
    per = kv_bytes_per_position(spec)
    return sum(attended_positions(spec, int(L)) * per for L in seqlens)


def union_positions(spec, seqlen: int, tokens: int) -> int:
    """Positions the T tokens of a verify step attend together: token t at
    position L - T + t attends min(w, ...) positions ending at its own, so the
    union is the last min(L, w + T - 1) positions (all L for a global layer)."""
    return min(seqlen, spec.window + tokens - 1) if spec.window > 0 else seqlen


def layer_multi_kv_bytes(spec, seqlens, tokens: int) -> int:
    """Algorithmic KV bytes of a T-token step that reads each position of the
    union of its tokens' windows once."""
    per = kv_bytes_per_position(spec)
    return sum(union_positions(spec, int(L), tokens) * per for L in seqlens)


def multi_attended_pairs(spec, seqlen: int, tokens: int) -> int:
    """(query token, attended position) pairs of one query head in a T-token step:
    token t at p = L - T + t attends min(p + 1, w) positions (p + 1 without a
    window)."""
    total = 0
    for t in range(tokens):
        p = seqlen - tokens + t
        if p < 0:
            continue
        total += min(p + 1, spec.window) if spec.window > 0 else p + 1
    return total


def layer_prefill_flops(spec, seqlens, tokens: int) -> int:
    """Useful flops of a T-token step (prefill chunk) of one layer: 2 D for the
    score and 2 D for the weighted value of every (query head, token, attended
    position)."""
    per = 4 * spec.head_dim * spec.n_q_heads
    return sum(multi_attended_pairs(spec, int(L), tokens) * per for L in seqlens)


FP8_ROW_EXTRA = 4  # the fp32 scale stored with every fp8 cache row


def fp8_kv_bytes_per_position(spec) -> int:
    """fp8-cache bytes read for one attended position of one sequence in one layer."""
    tensors = 1 if spec.kv_shared else 2
    return spec.n_kv_heads * (spec.head_dim + FP8_ROW_EXTRA) * tensors


def layer_fp8_kv_bytes(spec, seqlens) -> int:
    """Algorithmic fp8-cache bytes (codes and row scales) for one decode step of one layer."""
    per = fp8_kv_bytes_per_position(spec)
    return sum(attended_positions(spec, int(L)) * per for L in seqlens)
