"""GPU parity of the tcgen05 attention kernels at the benchmarked full sizes, against
the CPU oracle on sampled rows.

The batch-256 layer (8 K/V heads x 128, bf16, contexts U[1, 2048], block size 16)
with G = 32 and G = 64 query heads per K/V head, and the multi-token query shapes
that the benchmark times: G = 8 with 16 query tokens (128 rows per K/V head),
G = 8 with 32 query tokens (256 rows: two row tiles), and the OPT-13B geometry
(40 heads, G = 1) with 32 query tokens.  At these sizes every CTA runs many
units, so the pipelines' barrier phases and tensor-memory buffers turn over many
times.  Each sampled (sequence, query token, query head) row is recomputed by the
oracle from host copies of just the blocks that row reads, taken before any
library kernel runs (the decode step appends first; the snapshot replays that
append on the host).
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


def clean(dev):
    code, reason = pkv.get_device_error(dev)
    assert code == 0, (code, reason)


@pytest.mark.parametrize("G", [32, 64])
def test_gqa_decode_full_size_tcgen05(dev, G):
    """Append, then decode the batch-256 layer with G query heads per K/V head."""
    w = wl.make_gqa(G, device=dev, preappend=True)
    ix = dev_indices(w, dev)
    sel = sample_pairs(w, 28, 100 + G)
    # the last query head of the longest context: the last row of the tile
    sel.append((int(np.argmax(w.context_lens)), w.H - 1))
    snaps = [Snapshot(w, s, h) for s, h in sel]
    pkv.kv_cache_append(w.k_new, w.v_new, w.k_pool, w.v_pool, ix["slots"])
    out = pkv.paged_attn_decode(w.q, w.k_pool, w.v_pool, ix["bt"], ix["ctx"], w.scale)
    torch.cuda.synchronize()
    clean(dev)
    assert bool(torch.isfinite(out).all())
    got = out.cpu().numpy()
    for sn in snaps:
        assert max_err(got[sn.s, sn.h], sn.expected(w)) <= TOL["bf16"], (G, sn.s, sn.h, sn.ctx)
    # split into 512-token partitions: the same rows through the partial states and the merge
    out2 = pkv.paged_attn_decode(w.q, w.k_pool, w.v_pool, ix["bt"], ix["ctx"], w.scale, partition_tokens=512)
    torch.cuda.synchronize()
    clean(dev)
    got2 = out2.cpu().numpy()
    for sn in snaps:
        assert max_err(got2[sn.s, sn.h], sn.expected(w)) <= TOL["bf16"], (G, sn.s, sn.h, sn.ctx, 512)


def draw_q(S, Lq, H, D, seed, dev):
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    return torch.randn((S, Lq, H, D), generator=g, device=dev).to(torch.bfloat16)


def sampled_rows(w, Lq, n, seed):
    """(sequence, query token, query head) rows: the longest and the shortest context
    (first and last query token), the last head of the last query token (the last row
    of the last row tile), then random rows."""
    rng = np.random.default_rng(seed)
    s_long, s_short = int(np.argmax(w.context_lens)), int(np.argmin(w.context_lens))
    rows = {(s_long, Lq - 1, int(rng.integers(w.H))), (s_long, 0, int(rng.integers(w.H))),
            (s_short, Lq - 1, int(rng.integers(w.H))), (s_short, 0, 0),
            (int(rng.integers(w.S)), Lq - 1, w.H - 1)}
    while len(rows) < n:
        rows.add((int(rng.integers(w.S)), int(rng.integers(Lq)), int(rng.integers(w.H))))
    return sorted(rows)


def expected_row(w, qh, s, j, h, Lq):
    """Oracle output of query token j of sequence s, head h: it sees the first
    ctx - Lq + j + 1 positions, read through the sequence's own blocks."""
    vis = max(0, int(w.context_lens[s]) - Lq + j + 1)
    nblk = -(-vis // w.B)
    kvh = h // (w.H // w.Hkv)
    blocks = [int(b) for b in w.block_tables[s, :nblk]]
    idx = torch.tensor(blocks if blocks else [0], dtype=torch.long, device=w.k_pool.device)
    kc = w.host(w.k_pool.index_select(0, idx)[:, kvh:kvh + 1].contiguous())
    vc = w.host(w.v_pool.index_select(0, idx)[:, kvh:kvh + 1].contiguous())
    table = np.arange(max(1, nblk)).reshape(1, -1)
    return oracle.paged_decode(qh[s:s + 1, j, h:h + 1], kc, vc, table, np.array([vis]), w.scale, w.B, "bf16")[0, 0]


@pytest.mark.parametrize("name,G,Lq", [("gqa8", 8, 16), ("gqa8", 8, 32), ("opt13b", 1, 32)])
def test_multi_query_full_size_tcgen05(dev, name, G, Lq):
    """Verify / chunked-prefill shapes at full size: Lq new query tokens per sequence."""
    if name == "opt13b":
        w = wl.build_paged(wl.opt13b_lengths(), 40, 128, 16, "bf16", wl.BASE_SEED + 3, device=dev,
                           max_blocks=128)
    else:
        w = wl.make_gqa(G, device=dev)
    ix = dev_indices(w, dev)
    q = draw_q(w.S, Lq, w.H, w.D, 4242 + G + Lq, dev)
    qh = w.host(q)
    rows = sampled_rows(w, Lq, 28, 7 * G + Lq)
    want = [expected_row(w, qh, s, j, h, Lq) for s, j, h in rows]
    for pt in (0, 512):
        out = pkv.paged_attn_multi_query(q, w.k_pool, w.v_pool, ix["bt"], ix["ctx"], w.scale,
                                         partition_tokens=pt)
        torch.cuda.synchronize()
        clean(dev)
        got = out.cpu().numpy()
        assert np.all(np.isfinite(got))
        for (s, j, h), ref in zip(rows, want):
            assert max_err(got[s, j, h], ref) <= TOL["bf16"], (name, Lq, pt, s, j, h, int(w.context_lens[s]))
