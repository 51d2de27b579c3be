"""Paged single-query decode attention, computed the plain way (oracle; test infrastructure only).

What the pages fix:

* The KV cache of a sequence is split into fixed-size blocks of B tokens; a
  per-sequence block table maps logical block j to a physical block anywhere in
  the GPU pool ([digest] "Method (PagedAttention + vLLM)"; [velog] "PagedAttention",
  the table logical 0 -> physical 4, 1 -> 1, 2 -> 7).
* Attention follows the block table, gathers the non-contiguous blocks and
  computes softmax(Q K^T) V ([digest] "Method (PagedAttention + vLLM)").
* Logical blocks are contiguous from the sequence's point of view while physical
  blocks sit anywhere ([digest] framework-overview flowchart and the note under it).

So the oracle does exactly that and nothing more: it rebuilds the contiguous K
and V rows of each (sequence, head) by following the table, token by token in
logical order, and applies the textbook definition of attention for one query
vector.  Decode means one query token per sequence ([video] "쉽게 이해하기": the
decode phase produces one token at a time and re-reads the cached context).

Readings where the pages are silent:

* Pool layout: K and V are two pools, each ``[num_blocks, num_heads, B, head_dim]``;
  token ``t`` of a sequence is element ``(table[t // B], h, t % B, :)``.
* The scale multiplies q.k before the softmax (1/sqrt(head_dim) in the workloads).
* A context of length 0 gives an all-zero output.
* Slots at or beyond the context length, and blocks not in the table, are never read.
* Grouped-query attention (fewer K/V heads than query heads, named on the digest's
  related-work list as an orthogonal way to shrink the KV cache): with Hq query
  heads and Hkv K/V heads, G = Hq / Hkv consecutive query heads share one K/V head,
  query head h reading K/V head h // G.  Hkv = Hq is ordinary multi-head attention.
* Several query tokens per sequence (a prefill chunk appended to a cached prefix,
  or draft tokens checked in one pass; the video summary's "주요 인사이트" names
  chunked prefill and speculative decoding): the Lq new tokens are the last Lq of
  the context, and query token j (0-based) attends the positions before and at its
  own, i.e. the first ctx - Lq + j + 1 tokens.  Lq = 1 is decode.
"""

import numpy as np

from .storage import to_f64


def gather_rows(pool, table_row, ctx, head, block_size):
    """Stored rows ``[ctx, head_dim]`` of one head of one sequence, in logical order.

    ``pool`` is ``[num_blocks, num_heads, block_size, head_dim]`` (stored elements);
    ``table_row`` lists the physical block of each logical block.  Logical token
    ``t`` lives in physical block ``table_row[t // block_size]`` at slot
    ``t % block_size``.  Raises ``IndexError`` if the table points outside the pool.
    """
    ctx = int(ctx)
    num_blocks = pool.shape[0]
    if ctx < 0:
        raise ValueError("negative context length")
    need = -(-ctx // block_size)
    if need > len(table_row):
        raise IndexError("context needs more logical blocks than the table has")
    t = np.arange(ctx)
    phys = np.asarray(table_row, dtype=np.int64)[t // block_size]
    if ctx and (phys.min() < 0 or phys.max() >= num_blocks):
        raise IndexError("block table entry outside the pool")
    slot = t % block_size
    return pool[phys, head, slot, :]


def softmax_weights(logits):
    """Softmax of a 1-D float64 vector; subtracting the max changes nothing mathematically."""
    logits = np.asarray(logits, dtype=np.float64)
    e = np.exp(logits - logits.max())
    w = e / e.sum()
    if abs(w.sum() - 1.0) >= 1e-12:
        raise AssertionError("softmax weights do not sum to 1")
    return w


def attend(q, K, V, scale):
    """softmax(scale * K q) V for one query vector over the rows of K and V (float64).

    An empty context (no rows) returns zeros.
    """
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    if K.shape[0] == 0:
        return np.zeros(V.shape[1], dtype=np.float64)
    logits = scale * (K @ q)
    w = softmax_weights(logits)
    return w @ V


def paged_decode_selected(q, k_pool, v_pool, block_tables, context_lens, scale,
                          block_size, dtype, selection):
    """Decode outputs for the listed (sequence, query head) pairs: float64 ``[len(selection), D]``.

    ``q`` is ``[S, Hq, D]`` and the pools ``[NB, Hkv, B, D]``, all stored in ``dtype``;
    Hq must be a multiple of Hkv and query head h reads K/V head h // (Hq // Hkv).
    """
    Hq, D = q.shape[1], q.shape[2]
    Hkv = k_pool.shape[1]
    if Hq % Hkv:
        raise ValueError("query heads must be a multiple of K/V heads")
    group = Hq // Hkv
    out = np.zeros((len(selection), D), dtype=np.float64)
    for i, (s, h) in enumerate(selection):
        ctx = int(context_lens[s])
        kvh = h // group
        K = to_f64(gather_rows(k_pool, block_tables[s], ctx, kvh, block_size), dtype)
        V = to_f64(gather_rows(v_pool, block_tables[s], ctx, kvh, block_size), dtype)
        qv = to_f64(q[s, h], dtype)
        out[i] = attend(qv, K, V, scale)
    return out


def paged_decode(q, k_pool, v_pool, block_tables, context_lens, scale, block_size, dtype):
    """Decode outputs for every sequence and query head: float64 ``[S, Hq, D]``."""
    S, H, D = q.shape
    sel = [(s, h) for s in range(S) for h in range(H)]
    flat = paged_decode_selected(q, k_pool, v_pool, block_tables, context_lens, scale,
                                 block_size, dtype, sel)
    return flat.reshape(S, H, D)


def paged_multi_query(q, k_pool, v_pool, block_tables, context_lens, scale, block_size, dtype):
    """Outputs for Lq query tokens per sequence: float64 ``[S, Lq, Hq, D]``.

    ``q`` is ``[S, Lq, Hq, D]``; the context of sequence s (``context_lens[s]``
    tokens) already holds the Lq new tokens as its last Lq positions, and query
    token j attends the first ``context_lens[s] - Lq + j + 1`` tokens (none when
    that count is not positive).
    """
    S, Lq, Hq, D = q.shape
    Hkv = k_pool.shape[1]
    group = Hq // Hkv
    out = np.zeros((S, Lq, Hq, D), dtype=np.float64)
    for s in range(S):
        ctx = int(context_lens[s])
        for j in range(Lq):
            visible = max(0, ctx - Lq + j + 1)
            for h in range(Hq):
                K = to_f64(gather_rows(k_pool, block_tables[s], visible, h // group, block_size), dtype)
                V = to_f64(gather_rows(v_pool, block_tables[s], visible, h // group, block_size), dtype)
                out[s, j, h] = attend(to_f64(q[s, j, h], dtype), K, V, scale)
    return out
