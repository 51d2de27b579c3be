"""GPU parity of kv_cache_append, kv_block_copy and paged_kv_gather (bit-exact) and
of the device-side error word, through the C ABI."""

import json
import os

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_328_b200 as pkv
from paged_kv_cache_328_b200 import workloads as wl

pytestmark = pytest.mark.gpu

TD = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    pkv.load()
    return torch.device("cuda", 0)


def host(t):
    t = t.detach().cpu().contiguous()
    return t.numpy() if t.dtype == torch.float32 else t.view(torch.int16).numpy().view(np.uint16)


def nan_pool(nb, H, B, D, dtype, dev, seed):
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    p = torch.randn((nb, H, B, D), generator=g, device=dev).to(TD[dtype])
    p[::3] = float("nan")
    return p


def clean(dev):
    code, reason = pkv.get_device_error(dev)
    assert code == 0, (code, reason)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("B", [8, 16, 128])
def test_append_bit_exact(dev, dtype, D, B):
    nb, H, T = 12, 3, 40
    kc, vc = nan_pool(nb, H, B, D, dtype, dev, 1), nan_pool(nb, H, B, D, dtype, dev, 2)
    g = torch.Generator(device=dev)
    g.manual_seed(3)
    k = torch.randn((T, H, D), generator=g, device=dev).to(TD[dtype])
    v = torch.randn((T, H, D), generator=g, device=dev).to(TD[dtype])
    rng = np.random.default_rng(B + D)
    slots = rng.choice(nb * B, size=T, replace=False).astype(np.int64)
    slots[::7] = -1
    k0, v0 = host(kc), host(vc)
    pkv.kv_cache_append(k, v, kc, vc, torch.from_numpy(slots).to(dev))
    ke, ve, bad = oracle.kv_append(k0, v0, host(k), host(v), slots, B)
    assert bad == 0
    assert np.array_equal(host(kc), ke, equal_nan=True) and np.array_equal(host(vc), ve, equal_nan=True)
    clean(dev)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("B", [8, 16, 128])
def test_block_copy_bit_exact(dev, dtype, B):
    nb, H, D = 20, 5, 128
    kc, vc = nan_pool(nb, H, B, D, dtype, dev, 4), nan_pool(nb, H, B, D, dtype, dev, 5)
    perm = np.random.default_rng(B).permutation(nb)
    pairs = np.stack([perm[:7], perm[7:14]], axis=1).astype(np.int64)  # no dst repeats or is a src
    k0, v0 = host(kc), host(vc)
    pkv.kv_block_copy(kc, vc, torch.from_numpy(pairs).to(dev))
    ke, ve, bad = oracle.kv_block_copy(k0, v0, pairs)
    assert bad == 0
    assert np.array_equal(host(kc), ke, equal_nan=True) and np.array_equal(host(vc), ve, equal_nan=True)
    clean(dev)


def test_block_copy_large_blocks(dev):
    # config-4 geometry: 40 heads x 16 x 128 fp16 = 160 KB per block, 96 pairs
    nb, H, B, D = 300, 40, 16, 128
    kc, vc = nan_pool(nb, H, B, D, "f16", dev, 6), nan_pool(nb, H, B, D, "f16", dev, 7)
    perm = np.random.default_rng(0).permutation(nb)
    pairs = np.stack([perm[:96], perm[96:192]], axis=1).astype(np.int64)
    k0, v0 = host(kc), host(vc)
    pkv.kv_block_copy(kc, vc, torch.from_numpy(pairs).to(dev))
    ke, ve, _ = oracle.kv_block_copy(k0, v0, pairs)
    assert np.array_equal(host(kc), ke, equal_nan=True) and np.array_equal(host(vc), ve, equal_nan=True)
    clean(dev)


def encoded_pool(nb, H, B, D, dev):
    p = np.arange(nb)[:, None, None, None]
    h = np.arange(H)[None, :, None, None]
    o = np.arange(B)[None, None, :, None]
    d = np.arange(D)[None, None, None, :]
    return torch.from_numpy((10000.0 * h + 100.0 * p + o + d / 8.0).astype(np.float32)).to(dev)


@pytest.mark.parametrize("fixture", ["velog_block_table.json", "digest_flowchart.json"])
def test_gather_pages_block_tables(dev, golden_dir, fixture):
    g = json.load(open(os.path.join(golden_dir, fixture)))
    B, nb, H = g["block_size"], g["num_blocks"], g["num_heads"]
    D = 64  # the library's smallest head size; the fixtures' encoding does not depend on D
    pool = encoded_pool(nb, H, B, D, dev)
    tables = g["tables"] if "tables" in g else {"seq": g["table"]}
    lens = g["context_lens"] if "context_lens" in g else {"seq": g["context_len"]}
    expect = g["expected_gather"] if "expected_gather" in g else {"seq": g["expected"]}
    for seq, table in tables.items():
        ctx = lens[seq]
        got = host(pkv.paged_kv_gather(pool, torch.tensor(table, dtype=torch.int32, device=dev), ctx))
        want = oracle.gather_kv(host(pool), table, ctx, B)
        assert np.array_equal(got, want)
        for r in expect[seq]:
            t0, t1 = r["logical_tokens"]
            for i, t in enumerate(range(t0, t1 + 1)):
                for h in range(H):
                    assert got[h, t, 0] == 10000.0 * h + 100.0 * r["physical_block"] + r["first_slot"] + i
    clean(dev)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_gather_random(dev, dtype):
    w = wl.build_paged([1, 17, 300, 1000], 4, 128, 16, dtype, 21, device=dev)
    for s in range(w.S):
        row = torch.from_numpy(w.block_tables[s]).to(dev)
        got = host(pkv.paged_kv_gather(w.k_pool, row, int(w.context_lens[s])))
        want = oracle.gather_kv(host(w.k_pool), w.block_tables[s], int(w.context_lens[s]), w.B)
        assert np.array_equal(got, want)
    clean(dev)


# ---------------------------------------------------------------------------
# Device-side checks: skip the bad access, set the error word, never fault
# ---------------------------------------------------------------------------

def test_bad_slot_is_skipped_and_flagged(dev):
    nb, H, B, D = 6, 2, 16, 64
    kc, vc = nan_pool(nb, H, B, D, "f16", dev, 8), nan_pool(nb, H, B, D, "f16", dev, 9)
    k = torch.ones((3, H, D), dtype=torch.float16, device=dev)
    slots = np.array([5, nb * B + 3, 40], dtype=np.int64)
    k0, v0 = host(kc), host(vc)
    pkv.kv_cache_append(k, k, kc, vc, torch.from_numpy(slots).to(dev))
    code, reason = pkv.get_device_error(dev)
    assert code == -7 and reason == 3
    ke, ve, bad = oracle.kv_append(k0, v0, host(k), host(k), slots, B)
    assert bad == 1
    assert np.array_equal(host(kc), ke, equal_nan=True)
    clean(dev)


def test_bad_copy_pair_is_skipped_and_flagged(dev):
    nb, H, B, D = 6, 2, 16, 64
    kc, vc = nan_pool(nb, H, B, D, "f16", dev, 10), nan_pool(nb, H, B, D, "f16", dev, 11)
    pairs = np.array([[0, 4], [1, nb]], dtype=np.int64)
    k0, v0 = host(kc), host(vc)
    pkv.kv_block_copy(kc, vc, torch.from_numpy(pairs).to(dev))
    code, reason = pkv.get_device_error(dev)
    assert code == -7 and reason == 4
    ke, _, _ = oracle.kv_block_copy(k0, v0, pairs)
    assert np.array_equal(host(kc), ke, equal_nan=True)
    clean(dev)


def test_bad_block_id_and_context_are_flagged(dev):
    w = wl.build_paged([40, 20], 2, 64, 16, "f16", 12, device=dev, max_blocks=4)
    bt = torch.from_numpy(w.block_tables).to(dev)
    ctx = torch.from_numpy(w.context_lens).to(dev)
    bad_bt = bt.clone()
    bad_bt[0, 1] = w.num_blocks + 5
    pkv.paged_attn_decode(w.q, w.k_pool, w.v_pool, bad_bt, ctx, w.scale)
    code, reason = pkv.get_device_error(dev)
    assert code == -7 and reason == 1
    bad_ctx = ctx.clone()
    bad_ctx[1] = 4 * 16 + 1
    pkv.paged_attn_decode(w.q, w.k_pool, w.v_pool, bt, bad_ctx, w.scale)
    code, reason = pkv.get_device_error(dev)
    assert code == -7 and reason == 2
    # the context stays usable: a clean call afterwards is correct
    out = pkv.paged_attn_decode(w.q, w.k_pool, w.v_pool, bt, ctx, w.scale)
    want = oracle.paged_decode(w.host(w.q), w.host(w.k_pool), w.host(w.v_pool), w.block_tables,
                               w.context_lens, w.scale, w.B, w.dtype)
    assert float(np.max(np.abs(out.cpu().numpy() - want))) <= 2e-3
    clean(dev)


def test_debug_checks_reject_overlaps_before_launch(dev):
    """With the debug checks on, overlapping copy pairs and duplicate append slots
    are rejected on the host (PKV_EOVERLAP) and the pools are left untouched;
    valid inputs still copy bit-exactly."""
    nb, H, B, D = 16, 2, 16, 128
    kc, vc = nan_pool(nb, H, B, D, "bf16", dev, 21), nan_pool(nb, H, B, D, "bf16", dev, 22)
    k0, v0 = host(kc), host(vc)
    before = pkv.set_debug_checks(True)
    try:
        for bad in ([[2, 2]], [[1, 7], [3, 7]], [[1, 7], [7, 9]]):
            with pytest.raises(pkv.PagedKVError) as e:
                pkv.kv_block_copy(kc, vc, torch.tensor(bad, dtype=torch.int64, device=dev))
            assert e.value.code == -11, bad
        g = torch.Generator(device=dev)
        g.manual_seed(23)
        k = torch.randn((3, H, D), generator=g, device=dev).to(torch.bfloat16)
        v = torch.randn((3, H, D), generator=g, device=dev).to(torch.bfloat16)
        with pytest.raises(pkv.PagedKVError) as e:
            pkv.kv_cache_append(k, v, kc, vc, torch.tensor([5, 40, 5], dtype=torch.int64, device=dev))
        assert e.value.code == -11
        torch.cuda.synchronize()
        assert np.array_equal(host(kc), k0) and np.array_equal(host(vc), v0)
        # one source forked into three fresh blocks passes, and copies bit-exactly
        pairs = np.array([[4, 10], [4, 11], [5, 12]], dtype=np.int64)
        pkv.kv_block_copy(kc, vc, torch.from_numpy(pairs).to(dev))
        ke, ve, nbad = oracle.kv_block_copy(k0, v0, pairs)
        assert nbad == 0
        assert np.array_equal(host(kc), ke) and np.array_equal(host(vc), ve)
        slots = np.array([5, 40, -1], dtype=np.int64)
        pkv.kv_cache_append(k, v, kc, vc, torch.from_numpy(slots).to(dev))
        ka, va, nbad = oracle.kv_append(ke, ve, host(k), host(v), slots, B)
        assert nbad == 0
        assert np.array_equal(host(kc), ka) and np.array_equal(host(vc), va)
    finally:
        pkv.set_debug_checks(before)
    clean(dev)
