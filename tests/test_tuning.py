"""Block-size advice (host logic) and the partition tuner's host-side checks (no GPU).

The waste figure is pinned to brute force (lay the sequences out block by block and
count the empty slots) and to the pages' closed forms: a sequence wastes fewer than
B slots, none when its length is a multiple of B ("vLLM PagedAttention and
continuous batching", section 2; "PagedAttention - Efficient Memory Management for
LLM Serving with vLLM", note on block size).
"""

import ctypes

import numpy as np
import pytest

from paged_kv_cache_328_b200 import _lib, tuning
from paged_kv_cache_328_b200 import build as builder


def brute_waste(ctx, B):
    used = empty = 0
    for c in ctx:
        filled = 0
        while filled < c:                 # take a block, fill up to B slots
            n = min(B, c - filled)
            used += B
            empty += B - n
            filled += n
    return 0.0 if used == 0 else empty / used


@pytest.mark.parametrize("B", [8, 16, 32, 64, 128])
def test_waste_matches_brute_force(B):
    rng = np.random.default_rng(B)
    ctx = rng.integers(0, 700, 200)
    assert tuning.last_block_waste(ctx, B) == pytest.approx(brute_waste(ctx.tolist(), B), abs=1e-12)


def test_waste_closed_forms():
    assert tuning.last_block_waste([64, 128, 1024], 16) == 0.0       # multiples of B: no waste
    assert tuning.last_block_waste([1], 16) == pytest.approx(15 / 16)  # one token in a block of 16
    assert tuning.last_block_waste([], 16) == 0.0
    assert tuning.last_block_waste([0, 0], 16) == 0.0
    # under B-1 empty slots per sequence: waste < S (B-1) / sum(ctx)
    rng = np.random.default_rng(0)
    ctx = rng.integers(1, 4096, 500)
    for B in (8, 16, 32, 64, 128):
        assert tuning.last_block_waste(ctx, B) * (-(-ctx // B)).sum() * B < len(ctx) * B


def test_recommendation_follows_the_trade_off():
    rates = {8: 100.0, 16: 110.0, 32: 115.0, 64: 120.0}
    # lengths that are multiples of every B: no waste, the fastest block size wins
    best, rows = tuning.recommend_block_size([128, 256, 64], rates)
    assert best == 64 and [r[0] for r in rows] == [8, 16, 32, 64]
    # one-token sequences: waste 1 - 1/B dominates, the smallest block wins
    best, _ = tuning.recommend_block_size([1] * 10, rates)
    assert best == 8
    # scores are rate x (1 - waste)
    _, rows = tuning.recommend_block_size([20], rates)
    for B, w, r, sc in rows:
        assert w == pytest.approx(1 - 20 / (-(-20 // B) * B)) and sc == pytest.approx(r * (1 - w))


def test_default_rates_cover_the_supported_block_sizes():
    assert sorted(tuning.B200_DECODE_GBS) == [8, 16, 32, 64, 128]


@pytest.fixture(scope="module")
def lib():
    builder.build()
    return _lib.load()


A = 0x10000  # an aligned fake device address; rejected calls never dereference it


def tune_args(**over):
    a = dict(q=A, k=A, v=A, bt=A, cl=A, S=4, H=8, Hkv=2, D=128, B=16, MB=64, NB=512, dt=2, scale=0.1, out=A,
             ws=A, wsb=1 << 30, reps=3, times=None, cands=None, maxc=0, nc=None, stream=None)
    a.update(over)
    return [a[k] for k in ("q", "k", "v", "bt", "cl", "S", "H", "Hkv", "D", "B", "MB", "NB", "dt", "scale", "out",
                           "ws", "wsb", "reps", "times", "cands", "maxc", "nc", "stream")]


@pytest.mark.parametrize("over, code", [
    (dict(reps=0), -1),
    (dict(reps=5000), -1),
    (dict(ws=None), -1),
    (dict(maxc=-1), -1),
    (dict(MB=0), -1),
    (dict(D=80), -1),            # workspace query fails first: -1
    (dict(wsb=64), -6),          # PKV_EWORKSPACE
])
def test_tuner_rejects_on_host(lib, over, code):
    assert lib.paged_attn_decode_tune(*tune_args(**over)) == code


def test_tuner_workspace_is_the_largest_candidate(lib):
    S, H, Hkv, D, B, MB = 8, 32, 8, 128, 16, 256       # contexts up to 4096: candidates 4096 ... 64
    n = lib.paged_attn_decode_tune_workspace_size(S, H, Hkv, D, B, MB)
    sizes = [lib.paged_attn_decode_gqa_workspace_size(S, H, Hkv, D, B, MB, pt) for pt in (4096, 2048, 1024, 512,
                                                                                            256, 128, 64)]
    assert n == max(sizes) == sizes[-1]
    assert lib.paged_attn_decode_tune_workspace_size(S, H, Hkv, D, B, 0) == ctypes.c_size_t(-1).value
    # block size 128: 64 is not a multiple of B and is not a candidate
    n128 = lib.paged_attn_decode_tune_workspace_size(S, H, Hkv, D, 128, 32)
    assert n128 == lib.paged_attn_decode_gqa_workspace_size(S, H, Hkv, D, 128, 32, 128)
