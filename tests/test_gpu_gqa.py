"""GPU parity of grouped-query paged decode (paged_attn_decode_gqa through the C ABI).

Query head h reads K/V head h // G.  16-bit K/V with G < 8 runs on the warp-level
tensor-core kernel, 8 <= G <= 64 (head_dim 128) on the token-major tcgen05 kernel,
more on the 128-row tcgen05 kernel (head_dim 64 above 16 as well); fp32 K/V and
G = 1 run on the CUDA-core kernel.
Tolerances as for multi-head decode: 2e-3 (fp16/bf16), 1e-5 (fp32).
"""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_328_b200 as pkv
from paged_kv_cache_328_b200 import workloads as wl
from paritykit import TOL, dev_indices, max_err, sample_pairs, Snapshot

pytestmark = pytest.mark.gpu

RAGGED = [0, 1, 2, 15, 16, 17, 63, 64, 65, 127, 128, 129, 200, 513, 700]


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    pkv.load()
    return torch.device("cuda", 0)


def clean(dev):
    code, reason = pkv.get_device_error(dev)
    assert code == 0, (code, reason)


def full_oracle(w):
    return oracle.paged_decode(w.host(w.q), w.host(w.k_pool), w.host(w.v_pool), w.block_tables, w.context_lens,
                               w.scale, w.B, w.dtype)


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("G", [2, 3, 4, 7, 8, 16, 32, 48, 128])
@pytest.mark.parametrize("D", [64, 128])
def test_gqa_small_ragged(dev, dtype, G, D):
    Hkv = 2
    for B in (8, 16, 128):
        mb = -(-max(RAGGED) // B) + 1
        w = wl.build_paged(RAGGED, Hkv, D, B, dtype, 200 + G + D + B, device=dev, max_blocks=mb, num_q_heads=Hkv * G)
        ix = dev_indices(w, dev)
        want = full_oracle(w)
        for pt in sorted({0, max(B, 64), 256, mb * B}):
            got = pkv.paged_attn_decode(w.q, w.k_pool, w.v_pool, ix["bt"], ix["ctx"], w.scale,
                                        partition_tokens=pt).cpu().numpy()
            assert np.all(np.isfinite(got)), (B, pt)
            assert max_err(got, want) <= TOL[dtype], (B, pt, max_err(got, want))
            assert np.all(got[[i for i, c in enumerate(RAGGED) if c == 0]] == 0.0)
    clean(dev)


def test_gqa_one_token_returns_v_exactly(dev):
    for dtype in ("f16", "bf16"):
        for G in (2, 8, 16):
            w = wl.build_paged([1] * 9, 3, 128, 16, dtype, 7, device=dev, num_q_heads=3 * G)
            ix = dev_indices(w, dev)
            got = pkv.paged_attn_decode(w.q, w.k_pool, w.v_pool, ix["bt"], ix["ctx"], w.scale).cpu().numpy()
            v = w.v_pool.float().cpu().numpy()
            for s in range(w.S):
                blk = w.block_tables[s, 0]
                for h in range(w.H):
                    assert np.array_equal(got[s, h], v[blk, h // G, 0, :]), (dtype, G, s, h)
    clean(dev)


def test_gqa_group_of_one_is_multi_head(dev):
    w = wl.build_paged([5, 300, 77, 1024], 4, 128, 16, "bf16", 8, device=dev)
    ix = dev_indices(w, dev)
    a = pkv.paged_attn_decode(w.q, w.k_pool, w.v_pool, ix["bt"], ix["ctx"], w.scale)
    lib = pkv.load()
    b = torch.empty_like(a)
    ws = pkv.alloc_workspace(w.q, w.k_pool, ix["bt"])
    rc = lib.paged_attn_decode_gqa(w.q.data_ptr(), w.k_pool.data_ptr(), w.v_pool.data_ptr(), ix["bt"].data_ptr(),
                                   ix["ctx"].data_ptr(), w.S, 4, 4, 128, 16, w.max_blocks, w.num_blocks, 2,
                                   w.scale, b.data_ptr(), 0, ws.data_ptr(), ws.numel(),
                                   torch.cuda.current_stream(dev).cuda_stream)
    assert rc == 0
    assert torch.equal(a, b)
    clean(dev)


def test_gqa_permutation_and_block_size_identical(dev):
    """The tensor-core kernel also follows logical order only: every placement and
    block size gives bit-identical output."""
    ctx = np.array([3, 77, 300, 129, 1000, 16])
    logical = wl.draw_logical(int(ctx.sum()), len(ctx), 2, 128, "bf16", 9, dev)
    logical = (logical[0], logical[1], wl.draw_logical(1, len(ctx), 16, 128, "bf16", 10, dev)[2])
    ref = None
    for B in (8, 16, 32, 64, 128):
        for placement in (1, 2):
            w = wl.build_paged(ctx, 2, 128, B, "bf16", 9, device=dev, logical=logical, num_q_heads=16,
                               placement_seed=1000 * B + placement, max_blocks=-(-1024 // B))
            ix = dev_indices(w, dev)
            got = pkv.paged_attn_decode(w.q, w.k_pool, w.v_pool, ix["bt"], ix["ctx"], w.scale,
                                        partition_tokens=256).cpu()
            if ref is None:
                ref = got
                assert max_err(ref, full_oracle(w)) <= TOL["bf16"]
            assert torch.equal(got, ref), (B, placement)
    clean(dev)


@pytest.mark.parametrize("G", [4, 8])
def test_gqa_full_size(dev, G):
    """Batch-256 layer with 8 K/V heads and G query heads each: append, then decode."""
    w = wl.make_gqa(G, device=dev, preappend=True)
    ix = dev_indices(w, dev)
    sel = sample_pairs(w, 24, G)
    snaps = [Snapshot(w, s, h) for s, h in sel]
    pkv.kv_cache_append(w.k_new, w.v_new, w.k_pool, w.v_pool, ix["slots"])
    out = pkv.paged_attn_decode(w.q, w.k_pool, w.v_pool, ix["bt"], ix["ctx"], w.scale)
    torch.cuda.synchronize()
    clean(dev)
    assert bool(torch.isfinite(out).all())
    got = out.cpu().numpy()
    for sn in snaps:
        assert max_err(got[sn.s, sn.h], sn.expected(w)) <= TOL["bf16"], (sn.s, sn.h, sn.ctx)
