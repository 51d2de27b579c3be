"""Host-side checks of the seeded input generator (no GPU)."""

import math

import numpy as np
import torch

import oracle
from paged_kv_cache_328_b200 import workloads as wl


def _raw(w, t):
    return w.host(t)


def test_tiny_structure():
    w = wl.make_tiny(preappend=True)
    assert w.context_lens.tolist() == [2, 16, 17, 38]
    used = w.block_tables[w.block_tables >= 0]
    assert len(used) == 7 and len(set(used.tolist())) == 7          # 1+1+2+3 blocks, distinct
    assert w.num_blocks == 16 and w.max_blocks == 3
    for s in range(w.S):
        c = int(w.context_lens[s])
        pos = c - 1
        assert w.slot_mapping[s] == w.block_tables[s, pos // 16] * 16 + pos % 16
    # unused blocks are all NaN; the step's slot is NaN before the append
    k = _raw(w, w.k_pool)
    unused = [b for b in range(16) if b not in set(used.tolist())]
    assert np.all(np.isnan(k[unused]))
    for s in range(w.S):
        blk, off = divmod(int(w.slot_mapping[s]), 16)
        assert np.all(np.isnan(k[blk, :, off]))
    src, dst = w.cow_pairs[0]
    assert src == w.block_tables[3, 2] and dst in unused


def test_preappend_plus_append_equals_full():
    full = wl.make_tiny(preappend=False)
    pre = wl.make_tiny(preappend=True)
    k, v, bad = oracle.kv_append(_raw(pre, pre.k_pool), _raw(pre, pre.v_pool),
                                 _raw(pre, pre.k_new), _raw(pre, pre.v_new), pre.slot_mapping, pre.B)
    assert bad == 0
    kf, vf = _raw(full, full.k_pool), _raw(full, full.v_pool)
    assert np.array_equal(k, kf, equal_nan=True) and np.array_equal(v, vf, equal_nan=True)


def test_same_tokens_for_every_block_size():
    S = 6
    ctx = np.array([1, 7, 16, 40, 129, 300])
    logical = wl.draw_logical(int(ctx.sum()), S, 2, 64, "bf16", 5, "cpu")
    ref = None
    for B in (8, 16, 32, 64, 128):
        w = wl.build_paged(ctx, 2, 64, B, "bf16", 5, logical=logical, placement_seed=B)
        rows = [oracle.gather_kv(_raw(w, w.k_pool), w.block_tables[s], ctx[s], B) for s in range(S)]
        if ref is None:
            ref = rows
        for a, b in zip(rows, ref):
            assert np.array_equal(a, b)


def test_lognormal_lengths():
    x = wl.lognormal_lengths(200000, 1)
    assert x.min() >= 1 and x.max() <= 2048
    # mean 340 before the clip; clipping at 2048 removes about 1% of the mass
    # (ln 2048 is 2.3 sd above the log-mean) and about 3.6% of the mean
    assert 0.95 < x.mean() / 340 < 0.99
    assert abs(np.std(np.log(x[(x > 1) & (x < 2048)])) - 1.0) < 0.05


def test_uniform_lengths():
    x = wl.opt13b_lengths()
    assert len(x) == 256 and x.min() >= 1 and x.max() <= 2048


def test_cow_structure():
    w = wl.make_cow(groups=3, n=4, prompt=32, tail_max=20, H=2, D=8, B=16, dtype="f16")
    pb = 2
    assert w.S == 12 and len(w.cow_pairs) == 9
    dsts = w.cow_pairs[:, 1].tolist()
    assert len(set(dsts)) == len(dsts)
    srcs = set(w.cow_pairs[:, 0].tolist())
    assert not (set(dsts) & srcs)
    for g in range(3):
        owner = w.block_tables[g * 4]
        for i in range(4):
            t = w.block_tables[g * 4 + i]
            assert np.array_equal(t[:pb - 1], owner[:pb - 1])            # shared prompt blocks
            if i > 0:
                assert [owner[pb - 1], t[pb - 1]] in w.cow_pairs.tolist()  # its own copy
    # copying then reading through the samples' tables gives the owner's prompt tokens
    k, v, bad = oracle.kv_block_copy(_raw(w, w.k_pool), _raw(w, w.v_pool), w.cow_pairs)
    assert bad == 0
    for g in range(3):
        ref = oracle.gather_kv(k, w.block_tables[g * 4], 32, 16)
        for i in range(1, 4):
            assert np.array_equal(oracle.gather_kv(k, w.block_tables[g * 4 + i], 32, 16), ref)
    assert 0 < w.info["cow_saving"] < 1


def test_last_block_waste():
    w = wl.make_tiny()
    blocks = 1 + 1 + 2 + 3
    assert math.isclose(wl.last_block_waste(w), 1 - (2 + 16 + 17 + 38) / (blocks * 16))


def test_all_empty_contexts():
    """A batch whose contexts are all empty has nothing to append: every slot is -1
    and the append rows are zeros (no logical token exists to take them from)."""
    for ctx in ([0], [0, 0, 0]):
        w = wl.build_paged(np.array(ctx), 2, 64, 16, "f16", 3)
        assert w.slot_mapping.tolist() == [-1] * len(ctx)
        assert tuple(w.k_new.shape) == (len(ctx), 2, 64) and not bool(w.k_new.float().abs().sum())
        assert bool(torch.isnan(w.k_pool.float()).all())
