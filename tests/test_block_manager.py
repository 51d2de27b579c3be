"""The native block manager (C ABI, host code) against the oracle's model, on CPU.

Both are driven with the same operations; every slot, copy-on-write pair, block
table, token count, reference count and free count must be identical, and a
failing operation must fail on both and change nothing on either.
"""

import json
import os
import random

import pytest

import oracle
import paged_kv_cache_328_b200 as pkv
from paged_kv_cache_328_b200 import build as builder

PKV_ENOMEM, PKV_ESEQ = -9, -10


@pytest.fixture(scope="module", autouse=True)
def lib():
    builder.build()
    return pkv.load()


def same_state(native, model, nb):
    for seq in model.seqs:
        assert native.block_table(seq) == model.block_table(seq)
    assert native.num_free() == model.num_free()
    assert [native.ref_count(b) for b in range(nb)] == model.ref


def test_flowchart_fixture(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "block_manager_flowchart.json")))
    sc = g["scenario_cow"]
    bm = pkv.BlockManager(10, 16, free_order=sc["free_order"])
    bm.add_sequence(1, 10)
    bm.fork(1, 2)
    slots, pairs = bm.append_tokens([2])
    assert slots == sc["expected"]["append_seq2"]["slots"]
    assert [list(p) for p in pairs] == sc["expected"]["append_seq2"]["pairs"]
    slots, pairs = bm.append_tokens([1])
    assert slots == sc["expected"]["append_seq1"]["slots"] and pairs == []
    assert bm.block_table(2) == (sc["expected"]["seq2"]["table"], sc["expected"]["seq2"]["tokens"])


@pytest.mark.parametrize("seed", range(6))
def test_native_matches_model(seed):
    rng = random.Random(seed)
    nb, B = rng.choice([(16, 4), (40, 8), (64, 16)])
    order = list(range(nb))
    rng.shuffle(order)
    native = pkv.BlockManager(nb, B, free_order=order)
    model = oracle.BlockManager(nb, B, free_order=order)
    next_id = 1000 * seed
    for _ in range(1500):
        live = list(model.seqs)
        op = rng.random()
        if op < 0.18 or not live:
            call = ("add", next_id, rng.randint(0, 3 * B))
            next_id += 1
        elif op < 0.32:
            call = ("fork", rng.choice(live), next_id)
            next_id += 1
        elif op < 0.8:
            k = min(len(live), rng.randint(1, 5))
            batch = rng.sample(live, k)
            if rng.random() < 0.05:
                batch = batch + batch[:1]          # a repeated sequence is rejected
            call = ("append", batch)
        elif op < 0.9:
            call = ("free", rng.choice(live + list(model.swapped)))
        elif op < 0.95:
            call = ("swap_out", rng.choice(live))
        else:
            call = ("swap_in", rng.choice(list(model.swapped) or [10 ** 9]))
        results = []
        for impl in (model, native):
            try:
                if call[0] == "add":
                    impl.add_sequence(call[1], call[2])
                    results.append(None)
                elif call[0] == "fork":
                    impl.fork(call[1], call[2])
                    results.append(None)
                elif call[0] == "append":
                    slots, pairs = impl.append_tokens(call[1])
                    results.append((list(slots), [tuple(p) for p in pairs]))
                    # a step's outputs never overlap: they pass the debug checks
                    assert pkv.check_slots(list(slots)) == 0
                    assert pkv.check_copy_pairs([list(p) for p in pairs]) == 0
                elif call[0] == "free":
                    impl.free_sequence(call[1])
                    results.append(None)
                elif call[0] == "swap_out":
                    results.append(list(impl.swap_out(call[1])))
                else:
                    results.append(list(impl.swap_in(call[1])))
            except (oracle.BlockManagerError, pkv.PagedKVError) as e:
                results.append(("error", type(e).__name__))
        m, n = results
        if isinstance(m, tuple) and m and m[0] == "error":
            assert isinstance(n, tuple) and n[0] == "error", (call, n)
        else:
            assert m == n, call
        same_state(native, model, nb)


def test_error_codes_and_no_change():
    bm = pkv.BlockManager(3, 4)
    bm.add_sequence(0, 8)
    bm.add_sequence(1, 3)
    with pytest.raises(pkv.PagedKVError) as e:
        bm.append_tokens([1, 0])        # seq 0 needs a fourth block
    assert e.value.code == PKV_ENOMEM
    assert bm.block_table(0) == ([0, 1], 8) and bm.block_table(1) == ([2], 3)
    with pytest.raises(pkv.PagedKVError) as e:
        bm.add_sequence(0, 1)
    assert e.value.code == PKV_ESEQ
    with pytest.raises(pkv.PagedKVError) as e:
        bm.append_tokens([7])
    assert e.value.code == PKV_ESEQ
    tables, lens = bm.fill_tables([1, 0], 4)
    assert tables.tolist() == [[2, -1, -1, -1], [0, 1, -1, -1]] and lens.tolist() == [3, 8]


@pytest.mark.parametrize("holders,free,writers", [(2, 1, 2), (3, 2, 3), (3, 1, 2), (3, 2, 2), (4, 2, 4),
                                                   (4, 3, 4), (2, 0, 2), (2, 0, 1)])
def test_shared_last_block_batches_agree(holders, free, writers):
    """Forks sharing a partly filled last block append together: k writers of a
    block with r holders take min(k, r - 1) free blocks; native and model agree on
    success, slots, pairs and state, and on refusing batches that do not fit."""
    nb = 2 + free
    impls = [pkv.BlockManager(nb, 4), oracle.BlockManager(nb, 4)]
    for bm in impls:
        bm.add_sequence(0, 6)
        for c in range(1, holders):
            bm.fork(0, c)
    batch = list(range(holders))[::-1][:writers]
    got = []
    for bm in impls:
        try:
            slots, pairs = bm.append_tokens(batch)
            got.append((list(slots), [tuple(p) for p in pairs]))
        except (oracle.BlockManagerError, pkv.PagedKVError):
            got.append("refused")
    assert got[0] == got[1]
    fits = min(writers, holders - 1) <= free
    assert (got[0] != "refused") == fits
    same_state(impls[0], impls[1], nb)
