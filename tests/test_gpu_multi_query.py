"""GPU parity of paged_attn_multi_query (several query tokens per sequence, causal
within the new tokens) against the CPU oracle, through the C ABI."""

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


def clean(dev):
    code, reason = pkv.get_device_error(dev)
    assert code == 0, (code, reason)


def draw_q(S, Lq, H, D, dtype, seed, dev):
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    return torch.randn((S, Lq, H, D), generator=g, device=dev).to(wl.TORCH_DTYPES[dtype])


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("Lq,G", [(1, 1), (2, 1), (7, 1), (16, 1), (33, 1), (3, 2), (4, 8), (5, 4), (9, 2)])
def test_multi_query_small(dev, dtype, Lq, G):
    Hkv, D = 2, 128
    ctx = [max(0, Lq - 2), Lq, Lq + 1, 20, 100, 700]
    for B in (16, 128):
        mb = -(-max(ctx) // B) + 1
        w = wl.build_paged(ctx, Hkv, D, B, dtype, 300 + Lq + G + B, device=dev, max_blocks=mb)
        ix = dev_indices(w, dev)
        q = draw_q(w.S, Lq, Hkv * G, D, dtype, Lq * 10 + G, dev)
        want = oracle.paged_multi_query(w.host(q), w.host(w.k_pool), w.host(w.v_pool), w.block_tables,
                                        w.context_lens, w.scale, B, dtype)
        for pt in sorted({0, max(B, 64), 512, mb * B}):
            got = pkv.paged_attn_multi_query(q, w.k_pool, w.v_pool, ix["bt"], ix["ctx"], w.scale,
                                             partition_tokens=pt).cpu().numpy()
            assert np.all(np.isfinite(got)), (B, pt)
            assert max_err(got, want) <= TOL[dtype], (B, pt, max_err(got, want))
    clean(dev)


@pytest.mark.parametrize("D", [64, 128])
def test_multi_query_one_token_is_decode(dev, D):
    """q_len = 1 runs exactly the grouped-query decode (same kernel, same result)."""
    w = wl.build_paged([1, 50, 333, 1024, 0], 2, D, 16, "bf16", 31, device=dev, num_q_heads=8)
    ix = dev_indices(w, dev)
    a = pkv.paged_attn_decode(w.q, w.k_pool, w.v_pool, ix["bt"], ix["ctx"], w.scale)
    b = pkv.paged_attn_multi_query(w.q[:, None], w.k_pool, w.v_pool, ix["bt"], ix["ctx"], w.scale)
    assert torch.equal(a, b[:, 0])
    clean(dev)


def test_multi_query_last_row_matches_multi_head_decode(dev):
    """With G = 1 the last query token sees the whole context: it must agree with the
    CUDA-core multi-head decode of that token (different kernels, same tolerance)."""
    w = wl.build_paged([8, 300, 1500, 2048], 4, 128, 16, "f16", 32, device=dev)
    ix = dev_indices(w, dev)
    q = draw_q(w.S, 6, 4, 128, "f16", 33, dev)
    mq = pkv.paged_attn_multi_query(q, w.k_pool, w.v_pool, ix["bt"], ix["ctx"], w.scale)
    dec = pkv.paged_attn_decode(q[:, -1].contiguous(), w.k_pool, w.v_pool, ix["bt"], ix["ctx"], w.scale)
    assert max_err(mq[:, -1].cpu(), dec.cpu().numpy().astype(np.float64)) <= 2e-3
    clean(dev)


@pytest.mark.parametrize("G,Lq", [(1, 4), (4, 4), (8, 2)])
def test_multi_query_full_size(dev, G, Lq):
    """Verify-step shape: batch-256 layer (8 K/V heads, contexts U[1,2048]), Lq draft tokens."""
    w = wl.make_gqa(G, device=dev) if G > 1 else wl.build_paged(wl.opt13b_lengths(), 8, 128, 16, "bf16", 34,
                                                                device=dev, max_blocks=128)
    ix = dev_indices(w, dev)
    q = draw_q(w.S, Lq, w.H, 128, "bf16", 35 + G, dev)
    out = pkv.paged_attn_multi_query(q, w.k_pool, w.v_pool, ix["bt"], ix["ctx"], w.scale).cpu().numpy()
    clean(dev)
    assert np.all(np.isfinite(out))
    rng = np.random.default_rng(G * 100 + Lq)
    qh = w.host(q)
    for _ in range(16):
        s, j, h = int(rng.integers(w.S)), int(rng.integers(Lq)), int(rng.integers(w.H))
        vis = max(0, int(w.context_lens[s]) - Lq + j + 1)
        nblk = -(-vis // w.B)
        kvh = h // (w.H // w.Hkv)
        blocks = [int(b) for b in w.block_tables[s, :nblk]]
        idx = torch.tensor(blocks if blocks else [0], dtype=torch.long, device=dev)
        kc = w.host(w.k_pool.index_select(0, idx)[:, kvh:kvh + 1].contiguous())
        vc = w.host(w.v_pool.index_select(0, idx)[:, kvh:kvh + 1].contiguous())
        table = np.arange(max(1, nblk)).reshape(1, -1)
        want = oracle.paged_decode(qh[s:s + 1, j, h:h + 1], kc, vc, table, np.array([vis]), w.scale, w.B, "bf16")
        assert max_err(out[s, j, h], want[0, 0]) <= TOL["bf16"], (s, j, h, vis)
