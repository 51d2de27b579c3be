"""Pins for the block-manager model and the swap functions of the oracle (CPU only).

The expected values come from the pages' worked example written out by hand
(tests/golden/block_manager_flowchart.json), from invariants of reference
counting (every block is either free or referenced by exactly as many tables as
its count says), and from flat-offset brute force for the swap copies.
"""

import json
import os
import random

import numpy as np
import pytest

import oracle
from oracle import BlockManager, BlockManagerError


def load(golden_dir):
    with open(os.path.join(golden_dir, "block_manager_flowchart.json")) as f:
        return json.load(f)


def check_invariants(bm, num_blocks):
    counts = [0] * num_blocks
    for s in bm.seqs.values():
        assert len(s["table"]) == -(-s["tokens"] // bm.B)  # on demand: ceil(tokens / B) blocks
        for b in s["table"]:
            counts[b] += 1
    assert counts == bm.ref
    assert sorted(bm.free) == [b for b in range(num_blocks) if counts[b] == 0]


def test_flowchart_tables(golden_dir):
    g = load(golden_dir)
    sc = g["scenario_tables"]
    bm = BlockManager(10, g["block_size"], free_order=sc["free_order"])
    bm.add_sequence(2, 16)
    bm.fork(2, 1)
    for _ in range(21):
        bm.append_tokens([1])
    for _ in range(4):
        bm.append_tokens([2])
    e = sc["expected"]
    assert bm.block_table(1) == (e["seq1"]["table"], e["seq1"]["tokens"])
    assert bm.block_table(2) == (e["seq2"]["table"], e["seq2"]["tokens"])
    for b, c in e["ref_counts"].items():
        assert bm.ref[int(b)] == c
    assert bm.free == e["free"]
    check_invariants(bm, 10)


def test_flowchart_copy_on_write(golden_dir):
    g = load(golden_dir)
    sc = g["scenario_cow"]
    e = sc["expected"]
    bm = BlockManager(10, g["block_size"], free_order=sc["free_order"])
    bm.add_sequence(1, 10)
    bm.fork(1, 2)
    slots, pairs = bm.append_tokens([2])
    assert slots == e["append_seq2"]["slots"] and [list(p) for p in pairs] == e["append_seq2"]["pairs"]
    slots, pairs = bm.append_tokens([1])
    assert slots == e["append_seq1"]["slots"] and [list(p) for p in pairs] == e["append_seq1"]["pairs"]
    assert bm.block_table(1) == (e["seq1"]["table"], e["seq1"]["tokens"])
    assert bm.block_table(2) == (e["seq2"]["table"], e["seq2"]["tokens"])
    for b, c in e["ref_counts"].items():
        assert bm.ref[int(b)] == c
    check_invariants(bm, 10)


def test_out_of_blocks_changes_nothing():
    bm = BlockManager(3, 4)
    bm.add_sequence(0, 8)          # 2 blocks
    bm.add_sequence(1, 3)          # 1 block, pool full
    with pytest.raises(BlockManagerError):
        bm.append_tokens([1, 0])   # seq 1 fits its block, seq 0 needs a new one
    assert bm.block_table(0) == ([0, 1], 8) and bm.block_table(1) == ([2], 3)
    check_invariants(bm, 3)


def test_siblings_sharing_a_last_block_need_one_copy():
    """Two forks that share a partly filled last block append in one batch: the
    first copies it (copy-on-write), after which the block has one holder left and
    the second writes in place, so one free block serves the batch.  Worked out by
    hand: B = 4, FIFO order 0, 1, 2, ..."""
    bm = BlockManager(3, 4)
    bm.add_sequence(0, 6)                      # blocks [0, 1], 2 tokens in block 1
    bm.fork(0, 1)                              # blocks 0 and 1 held twice
    assert bm.num_free() == 1
    slots, pairs = bm.append_tokens([0, 1])
    assert pairs == [(1, 2)]                   # seq 0 copies block 1 into block 2
    assert slots == [2 * 4 + 2, 1 * 4 + 2]     # seq 1 writes block 1 in place
    assert bm.block_table(0) == ([0, 2], 7) and bm.block_table(1) == ([0, 1], 7)
    assert bm.ref == [2, 1, 1] and bm.num_free() == 0
    check_invariants(bm, 3)
    # three holders, two free blocks: two copies, the last writer in place
    bm = BlockManager(4, 4)
    bm.add_sequence(0, 6)
    bm.fork(0, 1)
    bm.fork(0, 2)
    slots, pairs = bm.append_tokens([2, 0, 1])
    assert pairs == [(1, 2), (1, 3)] and slots == [10, 14, 6]
    assert bm.num_free() == 0
    check_invariants(bm, 4)
    # three holders, one free block: two of them writing need two copies (the
    # block keeps a third holder), so the batch is refused and nothing changes
    bm = BlockManager(3, 4)
    bm.add_sequence(0, 6)
    bm.fork(0, 1)
    bm.fork(0, 2)
    with pytest.raises(BlockManagerError):
        bm.append_tokens([0, 1])
    assert bm.ref == [3, 3, 0] and bm.num_free() == 1
    check_invariants(bm, 3)


def test_random_operations_keep_invariants():
    rng = random.Random(5)
    nb = 40
    bm = BlockManager(nb, 4)
    next_id = 0
    for _ in range(2000):
        op = rng.random()
        live = list(bm.seqs)
        try:
            if op < 0.2 or not live:
                bm.add_sequence(next_id, rng.randint(0, 9))
                next_id += 1
            elif op < 0.35:
                bm.fork(rng.choice(live), next_id)
                next_id += 1
            elif op < 0.8:
                bm.append_tokens(rng.sample(live, k=min(len(live), rng.randint(1, 4))))
            elif op < 0.9:
                bm.free_sequence(rng.choice(live))
            elif op < 0.95:
                bm.swap_out(rng.choice(live))
            elif bm.swapped:
                bm.swap_in(rng.choice(list(bm.swapped)))
        except BlockManagerError:
            pass
        check_invariants(bm, nb)


def test_swap_round_trip_and_brute_force():
    rng = np.random.default_rng(3)
    nb, H, B, D = 9, 2, 4, 8
    k = rng.standard_normal((nb, H, B, D)).astype(np.float32)
    v = rng.standard_normal((nb, H, B, D)).astype(np.float32)
    ids = np.array([7, 2, 5, nb + 1])
    hk, hv, bad = oracle.kv_swap_out(k, v, ids)
    assert bad == 1
    size = H * B * D
    for i, b in enumerate(ids[:3]):
        assert np.array_equal(hk.reshape(len(ids), -1)[i], k.reshape(-1)[b * size:(b + 1) * size])
        assert np.array_equal(hv.reshape(len(ids), -1)[i], v.reshape(-1)[b * size:(b + 1) * size])
    assert not hk[3].any()
    # back into different blocks: pool'[new[i]] = pool[old[i]], everything else unchanged
    new = np.array([0, 8, 3, -1])
    k2, v2, bad = oracle.kv_swap_in(k, v, hk, hv, new)
    assert bad == 1
    for o, n in zip(ids[:3], new[:3]):
        assert np.array_equal(k2[n], k[o]) and np.array_equal(v2[n], v[o])
    for b in set(range(nb)) - set(new[:3].tolist()):
        assert np.array_equal(k2[b], k[b]) and np.array_equal(v2[b], v[b])
