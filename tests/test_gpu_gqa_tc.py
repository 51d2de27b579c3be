"""GPU parity of the token-major tcgen05 kernel (17 to 64 query rows per K/V head,
head_dim 128, 16-bit K/V: S^T = K Q^T with the tile's 128 tokens as M) against the
CPU oracle, through the C ABI.

Covers grouped-query decode with G = 17..64 and multi-token queries with Lq * G in
(16, 64]: every row tile size (16, 32 and 64 rows), groups and query lengths that
leave padding rows, contexts shorter than Lq, every block size, every partition
size, large logit scales (the per-row reference maximum is raised and O rescaled
on many tiles), one-token contexts (V returned exactly), and enough units that
every CTA turns its barriers and tensor memory over many times.
"""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_328_b200 as pkv
from paged_kv_cache_328_b200 import workloads as wl
from paritykit import TOL, dev_indices, max_err

pytestmark = pytest.mark.gpu

RAGGED = [0, 1, 2, 63, 127, 128, 129, 255, 256, 300, 513, 1000]


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
@pytest.mark.parametrize("G", [17, 24, 32, 40, 64])
def test_decode_groups(dev, dtype, G):
    for B in (8, 16, 128):
        mb = -(-max(RAGGED) // B) + 1
        w = wl.build_paged(RAGGED, 2, 128, B, dtype, 600 + G + B, device=dev, max_blocks=mb, num_q_heads=2 * G)
        ix = dev_indices(w, dev)
        want = oracle.paged_decode(w.host(w.q), w.host(w.k_pool), w.host(w.v_pool), w.block_tables,
                                   w.context_lens, w.scale, B, dtype)
        for pt in sorted({0, 128, 256, max(B, 64), mb * B}):
            got = pkv.paged_attn_decode(w.q, w.k_pool, w.v_pool, ix["bt"], ix["ctx"], w.scale,
                                        partition_tokens=pt).cpu().numpy()
            assert np.all(np.isfinite(got)), (B, pt)
            assert max_err(got, want) <= TOL[dtype], (B, pt, max_err(got, want))
            assert np.all(got[[i for i, c in enumerate(RAGGED) if c == 0]] == 0.0)
    clean(dev)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("Lq,G", [(17, 1), (32, 1), (64, 1), (3, 8), (8, 8), (2, 16), (4, 16), (9, 7), (5, 12),
                                  (2, 32), (1, 20)])
def test_multi_query_rows(dev, dtype, Lq, G):
    ctx = [max(0, Lq - 3), Lq, Lq + 1, 127, 128, 129, 400, 1500]
    for B in (16, 64):
        mb = -(-max(ctx) // B) + 1
        w = wl.build_paged(ctx, 2, 128, B, dtype, 700 + 3 * Lq + G + B, device=dev, max_blocks=mb)
        ix = dev_indices(w, dev)
        q = draw_q(w.S, Lq, 2 * G, 128, dtype, 701 + Lq + G, dev)
        want = oracle.paged_multi_query(w.host(q), w.host(w.k_pool), w.host(w.v_pool), w.block_tables,
                                        w.context_lens, w.scale, B, dtype)
        for pt in sorted({0, 128, 512, mb * B}):
            got = pkv.paged_attn_multi_query(q, w.k_pool, w.v_pool, ix["bt"], ix["ctx"], w.scale,
                                             partition_tokens=pt).cpu().numpy()
            assert np.all(np.isfinite(got)), (B, pt)
            assert max_err(got, want) <= TOL[dtype], (B, pt, max_err(got, want))
    clean(dev)


@pytest.mark.parametrize("scale", [0.5, 2.0, 8.0])
@pytest.mark.parametrize("G,Lq", [(32, 1), (16, 2), (64, 1)])
def test_large_logits_rescale(dev, scale, G, Lq):
    """Logits with spreads of tens to hundreds: the rows' maxima keep growing past
    the first tile's, so the reference maxima are raised and O is rescaled."""
    ctx = [1, 200, 777, 1500, 2048]
    w = wl.build_paged(ctx, 2, 128, 16, "bf16", 800 + G, device=dev, max_blocks=129)
    ix = dev_indices(w, dev)
    q = draw_q(w.S, Lq, 2 * G, 128, "bf16", 801 + G, dev)
    want = oracle.paged_multi_query(w.host(q), w.host(w.k_pool), w.host(w.v_pool), w.block_tables,
                                    w.context_lens, scale, 16, "bf16")
    for pt in (0, 256):
        got = pkv.paged_attn_multi_query(q, w.k_pool, w.v_pool, ix["bt"], ix["ctx"], scale,
                                         partition_tokens=pt).cpu().numpy()
        assert np.all(np.isfinite(got)), pt
        assert max_err(got, want) <= TOL["bf16"], (pt, max_err(got, want))
    clean(dev)


def test_one_token_contexts_return_v_exactly(dev):
    for dtype in ("f16", "bf16"):
        for G in (17, 32, 64):
            w = wl.build_paged([1] * 7, 3, 128, 16, dtype, 9, device=dev, num_q_heads=3 * G)
            ix = dev_indices(w, dev)
            got = pkv.paged_attn_decode(w.q, w.k_pool, w.v_pool, ix["bt"], ix["ctx"], w.scale).cpu().numpy()
            v = w.v_pool.float().cpu().numpy()
            for s in range(w.S):
                blk = w.block_tables[s, 0]
                for h in range(w.H):
                    assert np.array_equal(got[s, h], v[blk, h // G, 0, :]), (dtype, G, s, h)
    clean(dev)


def test_many_units_per_cta(dev):
    """400 sequences x 4 K/V heads: about 11 units per CTA, through the partial
    states and the merge as well."""
    rng = np.random.default_rng(11)
    ctx = rng.integers(0, 1200, 400).tolist()
    w = wl.build_paged(ctx, 4, 128, 16, "bf16", 12, device=dev, max_blocks=76, num_q_heads=4 * 32)
    ix = dev_indices(w, dev)
    want = oracle.paged_decode(w.host(w.q), w.host(w.k_pool), w.host(w.v_pool), w.block_tables,
                               w.context_lens, w.scale, 16, "bf16")
    for pt in (0, 256):
        got = pkv.paged_attn_decode(w.q, w.k_pool, w.v_pool, ix["bt"], ix["ctx"], w.scale,
                                    partition_tokens=pt).cpu().numpy()
        assert np.all(np.isfinite(got))
        assert max_err(got, want) <= TOL["bf16"], (pt, max_err(got, want))
    clean(dev)


def test_permutation_and_block_size_identical(dev):
    """The kernel follows logical order only: every placement and block size gives
    bit-identical output."""
    ctx = np.array([3, 77, 300, 129, 1000, 16])
    logical = wl.draw_logical(int(ctx.sum()), len(ctx), 2, 128, "bf16", 19, dev)
    logical = (logical[0], logical[1], wl.draw_logical(1, len(ctx), 64, 128, "bf16", 20, dev)[2])
    ref = None
    for B in (8, 16, 32, 64, 128):
        for placement in (1, 2):
            w = wl.build_paged(ctx, 2, 128, B, "bf16", 19, device=dev, logical=logical, num_q_heads=64,
                               placement_seed=1000 * B + placement, max_blocks=-(-1024 // B))
            ix = dev_indices(w, dev)
            got = pkv.paged_attn_decode(w.q, w.k_pool, w.v_pool, ix["bt"], ix["ctx"], w.scale,
                                        partition_tokens=256).cpu()
            if ref is None:
                ref = got
                want = oracle.paged_decode(w.host(w.q), w.host(w.k_pool), w.host(w.v_pool), w.block_tables,
                                           w.context_lens, w.scale, B, "bf16")
                assert max_err(ref, want) <= TOL["bf16"]
            assert torch.equal(got, ref), (B, placement)
    clean(dev)
