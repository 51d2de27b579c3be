"""KV append into slots, copy-on-write block copy and the plain gather (oracle; test infrastructure only).

What the pages fix:

* Each new token's K and V are computed and added to the cache, then reused by
  later steps ([velog] "KV Cache의 메모리 문제", steps 1-4).  Physical blocks are
  taken only when needed: store the token's K/V, and when the current block is
  full take a new block and update the table ([velog] "PagedAttention의 동작 방식",
  steps 1-5; [blog] section 2, on-demand allocation).
* Sequences with a common prefix share physical blocks; when one of them writes,
  only that block is copied, e.g. P3 -> P9 in the framework-overview flowchart
  ([digest] "Method (PagedAttention + vLLM)" and the flowchart under "방법 (Method)";
  [blog] section 2, copy-on-write sharing).

Readings where the pages are silent:

* A slot number addresses block ``slot // B`` at offset ``slot % B``; a negative
  slot means "no write" for that token.
* A block copy copies the whole block (every head, every one of the B slots) of
  both K and V, reading the pre-call pool; pairs must not overlap.
* A slot or block id outside the pool is skipped and counted as an error.
"""

import numpy as np


def kv_append(k_pool, v_pool, k_new, v_new, slot_mapping, block_size):
    """Return ``(k_pool', v_pool', n_bad)`` after writing token t's rows into slot t.

    ``k_new``/``v_new`` are ``[T, H, D]``; ``slot_mapping`` is ``[T]``.  For each t with
    ``slot >= 0``: ``pool'[slot // B, :, slot % B, :] = new[t]``.  Slots at or past
    ``num_blocks * B`` are skipped and counted in ``n_bad``.  Inputs are not modified.
    """
    k = np.array(k_pool, copy=True)
    v = np.array(v_pool, copy=True)
    num_slots = k.shape[0] * block_size
    n_bad = 0
    for t, slot in enumerate(np.asarray(slot_mapping).tolist()):
        if slot < 0:
            continue
        if slot >= num_slots:
            n_bad += 1
            continue
        blk, off = divmod(int(slot), block_size)
        k[blk, :, off, :] = k_new[t]
        v[blk, :, off, :] = v_new[t]
    return k, v, n_bad


def kv_block_copy(k_pool, v_pool, pairs):
    """Return ``(k_pool', v_pool', n_bad)`` with ``pool'[dst] = pool[src]`` for every pair.

    ``pairs`` is ``[n, 2]`` of (src, dst) physical block ids.  Every copy reads the
    pools as they were before the call.  A pair with an id outside the pool is
    skipped and counted in ``n_bad``.  Inputs are not modified.
    """
    k = np.array(k_pool, copy=True)
    v = np.array(v_pool, copy=True)
    num_blocks = k.shape[0]
    n_bad = 0
    for src, dst in np.asarray(pairs).reshape(-1, 2).tolist():
        if not (0 <= src < num_blocks and 0 <= dst < num_blocks):
            n_bad += 1
            continue
        k[dst] = k_pool[src]
        v[dst] = v_pool[src]
    return k, v, n_bad


def gather_kv(pool, table_row, ctx, block_size):
    """Stored rows of every head of one sequence, ``[H, ctx, D]``, in logical order.

    Token t of head h is ``pool[table_row[t // B], h, t % B, :]``, copied bit for bit.
    """
    ctx = int(ctx)
    num_blocks, num_heads, _, head_dim = pool.shape
    out = np.empty((num_heads, ctx, head_dim), dtype=pool.dtype)
    for t in range(ctx):
        phys = int(table_row[t // block_size])
        if not (0 <= phys < num_blocks):
            raise IndexError("block table entry outside the pool")
        out[:, t, :] = pool[phys, :, t % block_size, :]
    return out


def kv_swap_out(k_pool, v_pool, block_ids):
    """Return ``(host_k, host_v, n_bad)`` with ``host[i] = pool[block_ids[i]]`` (all heads and slots).

    Swapping a preempted sequence's blocks to host memory ("PagedAttention - Efficient
    Memory Management for LLM Serving with vLLM", section "Method", scheduling).  An id
    outside the pool leaves its host slot zero and is counted in ``n_bad``.
    """
    ids = np.asarray(block_ids).reshape(-1)
    hk = np.zeros((len(ids),) + k_pool.shape[1:], dtype=k_pool.dtype)
    hv = np.zeros((len(ids),) + v_pool.shape[1:], dtype=v_pool.dtype)
    n_bad = 0
    for i, b in enumerate(ids.tolist()):
        if not (0 <= b < k_pool.shape[0]):
            n_bad += 1
            continue
        hk[i] = k_pool[b]
        hv[i] = v_pool[b]
    return hk, hv, n_bad


def kv_swap_in(k_pool, v_pool, host_k, host_v, block_ids):
    """Return ``(k_pool', v_pool', n_bad)`` with ``pool'[block_ids[i]] = host[i]``."""
    k = np.array(k_pool, copy=True)
    v = np.array(v_pool, copy=True)
    n_bad = 0
    for i, b in enumerate(np.asarray(block_ids).reshape(-1).tolist()):
        if not (0 <= b < k.shape[0]):
            n_bad += 1
            continue
        k[b] = host_k[i]
        v[b] = host_v[i]
    return k, v, n_bad
