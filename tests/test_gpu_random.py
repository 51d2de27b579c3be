"""Seeded random configurations of the attention entry points against the oracle.

Each case draws a storage dtype, head_dim, block size, K/V heads, query heads per
K/V head G, query tokens per sequence Lq, a batch of ragged context lengths (with
empty, one-token, block-edge and table-maximum lengths mixed in) and a partition
size (the library's choice or a random multiple of the block size).  Decode runs
through ``paged_attn_decode`` (multi-head or grouped-query), Lq > 1 through
``paged_attn_multi_query``, so that every kernel and its routing boundaries
(fewer than 8, 8 to 64 and more than 64 query rows per K/V head; split and
unsplit contexts) meet inputs that no hand-written case chose.  Outputs start as
NaN and are compared element by element with the oracle; the device error word
must stay clear.
"""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_328_b200 as pkv
from paged_kv_cache_328_b200 import workloads as wl
from paritykit import TOL

pytestmark = pytest.mark.gpu

N_CASES = 48


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    pkv.load()
    return torch.device("cuda", 0)


def draw(i):
    rng = np.random.default_rng(7100 + i)
    dtype = str(rng.choice(["f16", "bf16", "f32"], p=[0.4, 0.5, 0.1]))
    D = int(rng.choice([64, 128], p=[0.25, 0.75]))
    B = int(rng.choice([8, 16, 32, 64, 128]))
    G = int(rng.choice([1, 2, 4, 8, 16, 32, 64]))
    Hkv = int(rng.integers(1, 4)) if G >= 16 else int(rng.integers(1, 7))
    Lq = 1 if dtype == "f32" else int(rng.choice([1, 1, 2, 3, 4, 8, 16, 32]))
    S = int(rng.integers(1, 24 if Lq * G <= 64 else 8))
    mb = -(-int(rng.choice([40, 300, 700])) // B)
    ctx = rng.integers(0, mb * B + 1, S)
    for c in (0, 1, B - 1, B, B + 1, mb * B, Lq - 1, Lq):
        if rng.random() < 0.3:
            ctx[int(rng.integers(0, S))] = max(0, min(c, mb * B))
    pt = 0 if rng.random() < 0.5 else B * int(rng.integers(1, max(2, 1024 // B)))
    return dict(dtype=dtype, D=D, B=B, G=G, Hkv=Hkv, Lq=Lq, S=S, mb=mb, ctx=ctx, pt=pt, seed=7200 + i)


@pytest.mark.parametrize("i", range(N_CASES))
def test_random_configuration(dev, i):
    c = draw(i)
    w = wl.build_paged(c["ctx"], H=c["Hkv"], D=c["D"], B=c["B"], dtype=c["dtype"], seed=c["seed"], device=dev,
                       max_blocks=c["mb"], num_q_heads=c["Hkv"] * c["G"])
    bt = torch.from_numpy(w.block_tables).to(dev)
    cl = torch.from_numpy(w.context_lens).to(dev)
    if c["Lq"] == 1:
        q = w.q
        want = oracle.paged_decode(w.host(q), w.host(w.k_pool), w.host(w.v_pool), w.block_tables, w.context_lens,
                                   w.scale, w.B, w.dtype)
        out = torch.full((w.S, w.H, w.D), float("nan"), dtype=torch.float32, device=dev)
        pkv.paged_attn_decode(q, w.k_pool, w.v_pool, bt, cl, w.scale, out=out, partition_tokens=c["pt"])
    else:
        g = torch.Generator().manual_seed(c["seed"])
        qc = torch.randn((w.S, c["Lq"], w.H, w.D), generator=g).to(w.q.dtype)
        want = oracle.paged_multi_query(w.host(qc), w.host(w.k_pool), w.host(w.v_pool), w.block_tables,
                                        w.context_lens, w.scale, w.B, w.dtype)
        out = torch.full((w.S, c["Lq"], w.H, w.D), float("nan"), dtype=torch.float32, device=dev)
        pkv.paged_attn_multi_query(qc.to(dev), w.k_pool, w.v_pool, bt, cl, w.scale, out=out,
                                   partition_tokens=c["pt"])
    torch.cuda.synchronize()
    code, reason = pkv.get_device_error(dev)
    assert code == 0, (code, reason)
    got = out.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got))
    err = float(np.max(np.abs(got - want))) if got.size else 0.0
    assert err <= TOL[c["dtype"]], (err, {k: v for k, v in c.items() if k != "ctx"})
