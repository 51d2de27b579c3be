"""GPU parity of the tcgen05 multi-query kernels (more than 16 query rows per K/V head:
Lq * G > 16) against the CPU oracle, through the C ABI: with head_dim 128 up to 64
rows run on the token-major kernel, more on the 128-row kernel; head_dim 64 always
on the 128-row kernel.

Covers query rows spanning several 128-row tiles (Lq * G > 128), groups that do not
divide 128 (padding rows in every tile), contexts shorter than Lq (query rows that
see no token), every partition size, block sizes below and above the 64-token
tile, head sizes 64 and 128, fp16 and bf16.  Tolerance 2e-3 as for every 16-bit
path.
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


def clean(dev):
    code, reason = pkv.get_device_error(dev)
    assert code == 0, (code, reason)


def draw_q(S, Lq, H, D, dtype, seed, dev):
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    return torch.randn((S, Lq, H, D), generator=g, device=dev).to(wl.TORCH_DTYPES[dtype])


def check(dev, dtype, D, Lq, G, Hkv, ctx, blocks, seed):
    for B in blocks:
        mb = -(-max(ctx) // B) + 1
        w = wl.build_paged(ctx, Hkv, D, B, dtype, seed + B, device=dev, max_blocks=mb)
        ix = dev_indices(w, dev)
        q = draw_q(w.S, Lq, Hkv * G, D, dtype, seed + 1, dev)
        want = oracle.paged_multi_query(w.host(q), w.host(w.k_pool), w.host(w.v_pool), w.block_tables,
                                        w.context_lens, w.scale, B, dtype)
        for pt in sorted({0, max(B, 64), 512, mb * B}):
            got = pkv.paged_attn_multi_query(q, w.k_pool, w.v_pool, ix["bt"], ix["ctx"], w.scale,
                                             partition_tokens=pt).cpu().numpy()
            assert np.all(np.isfinite(got)), (B, pt)
            assert max_err(got, want) <= TOL[dtype], (B, pt, max_err(got, want))
    clean(dev)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Lq,G", [(17, 1), (128, 1), (200, 1), (3, 8), (16, 8), (40, 8), (2, 16), (9, 16),
                                  (1, 32), (5, 32), (1, 128), (2, 128), (7, 3), (11, 5), (6, 12)])
def test_tcgen05_multi_query(dev, dtype, D, Lq, G):
    ctx = [max(0, Lq - 3), Lq, Lq + 1, 63, 64, 65, 129, 700]
    check(dev, dtype, D, Lq, G, 2, ctx, (16, 128), 500 + Lq * 7 + G)


def test_tcgen05_block_sizes_and_many_units(dev):
    # every block size, 40 sequences x 4 K/V heads x several row tiles: many units per CTA
    rng = np.random.default_rng(9)
    ctx = rng.integers(0, 900, 40).tolist()
    check(dev, "bf16", 128, 24, 8, 4, ctx, (8, 32, 64), 77)


def test_tcgen05_long_context_split(dev):
    # 32K-token contexts split into partitions, chunk of 64 query tokens, G = 4
    ctx = [32768, 20000, 1]
    check(dev, "f16", 128, 64, 4, 1, ctx, (16,), 91)
