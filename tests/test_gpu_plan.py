"""GPU tests of the decode plan: the work list the plan kernel leaves in the
workspace, and decode through every ordering path with a NaN-filled output.

The plan turns context_lens into one unit per (sequence, partition) and orders
them longest first so that the dynamically scheduled CTAs end together ("vLLM
PagedAttention and continuous batching", section 5: partitioned long contexts;
the ordering itself is a scheduling choice of this library).  The workspace
starts with the unit counter and the number of units (two int32), then the unit
list at byte 16: per unit {(s << 16) | p, clamped context length}.

The sort key of a unit of n tokens: 8-token buckets up to 512 tokens, 256-token
buckets above, the last bucket (127) taking everything longer.  Every partition
but a sequence's last holds partition_tokens tokens.  Up to 1024 sequences the
list is exactly the stable sort of the (sequence, partition) order by decreasing
key; longer lists that are sorted (at most 4096 units) keep every unit with keys
non-increasing; the rest are in (sequence, partition) order.
"""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_328_b200 as pkv
from paged_kv_cache_328_b200 import workloads as wl
from paritykit import TOL, dev_indices, max_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    pkv.load()
    return torch.device("cuda", 0)


def bucket(n):
    return (n + 7) >> 3 if n <= 512 else min(127, 64 + ((n - 512 + 255) >> 8))


def all_units(ctx, pt):
    """(s, p, ctx, key) in (sequence, partition) order."""
    units = []
    for s, c in enumerate(ctx):
        n = max(1, -(-int(c) // pt))
        for p in range(n):
            units.append((s, p, int(c), bucket(pt) if p < n - 1 else bucket(int(c) - (n - 1) * pt)))
    return units


def plan_list(ws, n_max):
    head = ws[:8].view(torch.int32).cpu().numpy()
    n = int(head[1])
    assert 0 < n <= n_max
    u = ws[16:16 + 8 * n].view(torch.int32).cpu().numpy().reshape(n, 2).astype(np.int64)
    return [(int(x) >> 16, int(x) & 0xFFFF, int(c)) for x, c in u]


def run(w, ix, pt, dev):
    ws = pkv.alloc_workspace(w.q, w.k_pool, ix["bt"], pt)
    ws.fill_(0xFF)
    out = torch.full((w.S, w.H, w.D), float("nan"), dtype=torch.float32, device=dev)
    pkv.paged_attn_decode(w.q, w.k_pool, w.v_pool, ix["bt"], ix["ctx"], w.scale, out=out,
                          partition_tokens=pt, workspace=ws)
    torch.cuda.synchronize()
    code, reason = pkv.get_device_error(dev)
    assert code == 0, (code, reason)
    return out.cpu().numpy(), ws


def contexts(S, mb, B, pt, seed):
    """Random lengths plus the special ones: empty, one token, exact multiples of
    the partition, the table's maximum."""
    rng = np.random.default_rng(seed)
    ctx = rng.integers(0, mb * B + 1, S)
    special = [0, 1, pt, 2 * pt, pt - 1, pt + 1, mb * B, 512, 513, 8, 9]
    for i, c in enumerate(special[:S]):
        ctx[(7 * i) % S] = min(c, mb * B)
    return ctx


@pytest.mark.parametrize("S,pt", [(1, 64), (7, 128), (256, 512), (256, 128), (1000, 256), (1024, 64),
                                  (1024, 608)])
def test_one_pass_plan_is_the_stable_longest_first_order(dev, S, pt):
    B, mb = 16, 38  # contexts up to 608 tokens
    ctx = contexts(S, mb, B, pt, 900 + S + pt)
    w = wl.build_paged(ctx, H=2, D=64, B=B, dtype="f16", seed=901 + S, device=dev, max_blocks=mb)
    ix = dev_indices(w, dev)
    got, ws = run(w, ix, pt, dev)
    units = all_units(ctx, pt)
    want = [(s, p, c) for s, p, c, _ in sorted(units, key=lambda u: -u[3])]
    assert plan_list(ws, len(units)) == want
    ref = oracle.paged_decode(w.host(w.q), w.host(w.k_pool), w.host(w.v_pool), w.block_tables, w.context_lens,
                              w.scale, B, "f16")
    assert np.all(np.isfinite(got))
    assert max_err(got, ref) <= TOL["f16"]


@pytest.mark.parametrize("S,pt,sorted_list", [(1500, 608, True), (1500, 512, True), (1500, 256, False)])
def test_long_lists(dev, S, pt, sorted_list):
    """Above 1024 sequences: the warp sort (up to 4096 units) keeps keys
    non-increasing; longer lists keep (sequence, partition) order."""
    B, mb = 16, 38
    ctx = contexts(S, mb, B, pt, 950 + pt)
    w = wl.build_paged(ctx, H=2, D=64, B=B, dtype="f16", seed=951, device=dev, max_blocks=mb)
    ix = dev_indices(w, dev)
    got, ws = run(w, ix, pt, dev)
    units = all_units(ctx, pt)
    lst = plan_list(ws, len(units))
    assert sorted(lst) == [(s, p, c) for s, p, c, _ in units]
    key = {(s, p): k for s, p, _, k in units}
    keys = [key[(s, p)] for s, p, _ in lst]
    if sorted_list:
        assert all(a >= b for a, b in zip(keys, keys[1:]))
    else:
        assert lst == [(s, p, c) for s, p, c, _ in units]
    ref = oracle.paged_decode(w.host(w.q), w.host(w.k_pool), w.host(w.v_pool), w.block_tables, w.context_lens,
                              w.scale, B, "f16")
    assert np.all(np.isfinite(got))
    assert max_err(got, ref) <= TOL["f16"]


@pytest.mark.parametrize("H,Hq", [(8, 8), (2, 64), (2, 16)])
def test_back_to_back_calls_share_one_workspace(dev, H, Hq):
    """Calls queued back to back on one stream and one workspace, with different context
    lengths and partition sizes: each call's plan reads its lengths while the previous
    call's kernels may still run and must not change the unit list or the counters under
    them (the plan waits for its predecessor before writing).  MHA, the token-major and the
    warp-level grouped-query kernels; every output against the oracle."""
    B, mb, S = 16, 64, 96
    rng = np.random.default_rng(1200 + Hq)
    ctx_sets = [rng.integers(0, mb * B + 1, S) for _ in range(3)]
    ctx_sets[1][:5] = 0
    # tables and pool cover the longest of the three lengths of every sequence
    w = wl.build_paged(np.maximum.reduce(ctx_sets), H=H, D=128, B=B, dtype="bf16", seed=1201 + Hq, device=dev, max_blocks=mb,
                       num_q_heads=Hq)
    ix = dev_indices(w, dev)
    ws = pkv.alloc_workspace(w.q, w.k_pool, ix["bt"], 64)  # the largest of the plans below
    calls = [(ctx_sets[i % 3], pt) for i, pt in enumerate([0, 64, 256, 0, 512, 64, 0, 256, 1024])]
    # inputs and outputs made first, so nothing but the calls themselves sits between them
    ctx_dev = [torch.from_numpy(c.astype(np.int32)).to(dev) for c in ctx_sets]
    outs = [torch.full((w.S, w.H, w.D), float("nan"), dtype=torch.float32, device=dev) for _ in calls]
    ws.fill_(0xFF)
    torch.cuda.synchronize()
    for k, (_, pt) in enumerate(calls):
        pkv.paged_attn_decode(w.q, w.k_pool, w.v_pool, ix["bt"], ctx_dev[k % 3], w.scale, out=outs[k],
                              partition_tokens=pt, workspace=ws)
    torch.cuda.synchronize()
    code, reason = pkv.get_device_error(dev)
    assert code == 0, (code, reason)
    want = {i: oracle.paged_decode(w.host(w.q), w.host(w.k_pool), w.host(w.v_pool), w.block_tables, c, w.scale,
                                   B, "bf16") for i, c in enumerate(ctx_sets)}
    for k, ((c, pt), out) in enumerate(zip(calls, outs)):
        got = out.cpu().numpy()
        assert np.all(np.isfinite(got)), (k, pt)
        assert max_err(got, want[k % 3]) <= TOL["bf16"], (k, pt, max_err(got, want[k % 3]))
