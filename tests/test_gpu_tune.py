"""GPU: the partition tuner (paged_attn_decode_tune through the C ABI).

It must time every documented candidate, return the fastest, and leave in `out`
the decode result for that size, which is compared with the oracle like any
decode call (2e-3 for fp16/bf16, 1e-5 for fp32).
"""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_328_b200 as pkv
from paged_kv_cache_328_b200 import workloads as wl
from paritykit import TOL, Snapshot, dev_indices, max_err, sample_pairs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    pkv.load()
    return torch.device("cuda", 0)


def expected_candidates(B, max_ctx):
    c = [max_ctx]
    pt = 4096
    while pt >= 64:
        if pt % B == 0 and pt < max_ctx:
            c.append(pt)
        pt //= 2
    return c


@pytest.mark.parametrize("dtype, Hkv, G, B", [("bf16", 4, 1, 16), ("f16", 2, 4, 16), ("f32", 2, 1, 32),
                                              ("bf16", 2, 8, 128)])
def test_tuner_picks_a_candidate_and_leaves_its_result(dev, dtype, Hkv, G, B):
    lens = [0, 1, 17, 129, 700, 1500, 2049, 333, 64, 5]
    mb = -(-max(lens) // B) + 1
    w = wl.build_paged(lens, Hkv, 128, B, dtype, 90 + G + B, device=dev, max_blocks=mb, num_q_heads=Hkv * G)
    ix = dev_indices(w, dev)
    out = torch.full((w.S, w.H, w.D), float("nan"), device=dev)
    best, times = pkv.tune_partition_tokens(w.q, w.k_pool, w.v_pool, ix["bt"], ix["ctx"], w.scale, reps=3, out=out)
    assert sorted(times) == sorted(expected_candidates(B, mb * B))
    assert best in times and times[best] == min(times.values())
    assert all(t > 0 for t in times.values())
    want = oracle.paged_decode(w.host(w.q), w.host(w.k_pool), w.host(w.v_pool), w.block_tables, w.context_lens,
                               w.scale, w.B, w.dtype)
    got = out.cpu().numpy()
    assert np.all(np.isfinite(got)) and max_err(got, want) <= TOL[dtype]
    code, reason = pkv.get_device_error(dev)
    assert code == 0, (code, reason)


def test_tuner_on_a_large_batch(dev):
    # batch-256 OPT-13B layer (40 heads, D 128, bf16): the tuner's choice runs and matches
    # sampled oracle rows
    w = wl.make_opt13b(B=16, device=dev, S=64)
    bt = torch.from_numpy(w.block_tables).to(dev)
    ctx = torch.from_numpy(w.context_lens).to(dev)
    best, times = pkv.tune_partition_tokens(w.q, w.k_pool, w.v_pool, bt, ctx, w.scale, reps=2)
    assert best in times and len(times) == len(expected_candidates(16, w.max_blocks * 16))
    got = pkv.paged_attn_decode(w.q, w.k_pool, w.v_pool, bt, ctx, w.scale, partition_tokens=best).cpu().numpy()
    for s, h in sample_pairs(w, 24, 3):
        want = Snapshot(w, s, h).expected(w, copy=False, append=False)
        assert max_err(got[s, h], want) <= TOL["bf16"], (s, h)
