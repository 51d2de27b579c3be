"""Block-size advice for a paged KV pool (host logic).

The block size B is fixed when the pool is laid out, so it cannot be tuned per
call the way the partition size is (``tune_partition_tokens``).  The pages frame
B as a trade-off: small blocks waste less memory in each sequence's last,
partly filled block, large blocks let the attention kernel read longer
contiguous runs ("PagedAttention - Efficient Memory Management for LLM Serving
with vLLM", Zettelkasten note on block size and Figure 18; "vLLM PagedAttention
and continuous batching", section 5: 8-16 for little waste, 32-64 for bandwidth
on long contexts).  ``recommend_block_size`` puts numbers on both sides for a
sample of context lengths:

* waste(B): the fraction of reserved slots left empty, 1 - sum(ctx) / sum(ceil(ctx/B) B);
* rate(B): the decode kernel's measured K/V bandwidth at that block size;

and ranks the block sizes by rate(B) * (1 - waste(B)): how fast the kernel
streams the cache times how much of the reserved memory holds context (more
sequences fit in the same pool).
"""

import numpy as np

# paged_attn_decode on one B200 (batch-256 OPT-13B layer, bf16, contexts U[1,2048],
# bench.py --block-size sweep, the attention call's roofline.achieved): effective
# K/V GB/s per block size, measured with the current decode kernel (one sweep, one box).
B200_DECODE_GBS = {8: 7186.0, 16: 7330.0, 32: 7392.0, 64: 7400.0, 128: 7447.0}


def last_block_waste(context_lens, block_size):
    """Fraction of reserved slots left empty: only each sequence's last block is partly filled."""
    ctx = np.asarray(context_lens, dtype=np.int64)
    reserved = int((-(-ctx // block_size)).sum()) * block_size
    return 0.0 if reserved == 0 else 1.0 - int(ctx.sum()) / reserved


def recommend_block_size(context_lens, rates=None):
    """Rank block sizes for these context lengths: returns (best B, rows) where each
    row is (B, waste, rate GB/s, score = rate * (1 - waste))."""
    rates = B200_DECODE_GBS if rates is None else dict(rates)
    rows = []
    for B in sorted(rates):
        w = last_block_waste(context_lens, B)
        rows.append((B, w, rates[B], rates[B] * (1.0 - w)))
    best = max(rows, key=lambda r: r[3])[0]
    return best, rows
