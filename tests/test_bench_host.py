"""Host-side helpers of bench.py (no GPU): the unique-byte count of a step whose
sequences share blocks, the spread statistics, and the oracle sample shared by
the two CPU timings."""

import types

import numpy as np

import bench


def fake(tables, ctx, B=4, H=2, D=8, e=2):
    return types.SimpleNamespace(block_tables=np.array(tables, dtype=np.int32),
                                 context_lens=np.array(ctx, dtype=np.int32), B=B, Hkv=H, D=D, elem_bytes=e)


def test_unique_bytes_count_shared_blocks_once():
    # two samples share prompt blocks 5 and 6 (8 tokens); sample 0 reads 3 more
    # tokens in block 7, sample 1 reads 1 more in block 9; block 6 is read whole
    w = fake([[5, 6, 7, -1], [5, 6, 9, -1]], [11, 9])
    row = 2 * 8 * 2 * 2  # H * D * e * (K + V)
    assert bench.unique_kv_bytes(w) == (4 + 4 + 3 + 1) * row
    # the logical count reads the shared blocks twice
    assert (11 + 9) * row > bench.unique_kv_bytes(w)


def test_unique_bytes_takes_the_longest_prefix_of_a_block():
    # a block read partly by one sequence and whole by another counts whole
    w = fake([[3, -1], [3, 4]], [2, 6])
    assert bench.unique_kv_bytes(w) == (4 + 2) * 2 * 8 * 2 * 2
    # no context reads nothing
    assert bench.unique_kv_bytes(fake([[-1]], [0])) == 0


def test_unique_bytes_of_the_sampling_layout_closed_form():
    """32 prompts of 512 tokens shared by 4 samples, each non-owner reading its own
    copy of the last prompt block, plus private tails: unique tokens =
    groups * (prompt - B) + samples * B + sum(tail + 1)."""
    B, groups, n, prompt = 16, 32, 4, 512
    pb = prompt // B
    rng = np.random.default_rng(0)
    tails = rng.integers(1, 257, size=groups * n)
    tb = -(-(tails + 1) // B)
    mb = pb + int(tb.max())
    tables = np.full((groups * n, mb), -1, dtype=np.int64)
    nxt = 0
    for g in range(groups):
        shared = np.arange(nxt, nxt + pb)
        nxt += pb
        for i in range(n):
            s = g * n + i
            tables[s, :pb] = shared
            if i:
                tables[s, pb - 1] = nxt
                nxt += 1
            tables[s, pb:pb + tb[s]] = np.arange(nxt, nxt + tb[s])
            nxt += tb[s]
    w = fake(tables, prompt + tails + 1, B=B, H=40, D=128, e=2)
    tokens = groups * (prompt - B) + groups * n * B + int((tails + 1).sum())
    assert bench.unique_kv_bytes(w) == tokens * 40 * 128 * 2 * 2


def test_spread():
    s = bench.spread([float(x) for x in range(1, 12)])
    assert s["median"] == 6.0 and s["p10"] == 2.0 and s["p90"] == 10.0 and s["mean"] == 6.0


def test_both_oracle_timings_use_one_sample_size():
    # cpu_baseline and the reference arm draw the same bounded sample
    assert bench.oracle_sample_seqs("opt13b") == 32
    assert bench.oracle_sample_seqs("longctx") == 2
