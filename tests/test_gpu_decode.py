"""GPU parity of paged_attn_decode (through the C ABI) against the CPU oracle.

Tolerances (max abs error): 1e-5 for fp32 KV, 2e-3 for fp16/bf16 KV, fp32
accumulation and fp32 output.  Cases span several tiles, ragged last blocks and
tiles, empty contexts, every supported block size and head size, split and
unsplit execution, and the five workload shapes at full size (sampled outputs).
"""

import math

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


def no_device_error(dev):
    code, reason = pkv.get_device_error(dev)
    assert code == 0, f"device error word: code {code}, reason {reason}"


def decode(w, ix, pt=0, ctx=None, ws=None):
    return pkv.paged_attn_decode(w.q, w.k_pool, w.v_pool, ix["bt"], ix["ctx"] if ctx is None else ctx,
                                 w.scale, partition_tokens=pt, workspace=ws)


def full_oracle(w, ctx=None):
    c = w.context_lens if ctx is None else ctx
    return oracle.paged_decode(w.host(w.q), w.host(w.k_pool), w.host(w.v_pool), w.block_tables, c,
                               w.scale, w.B, w.dtype)


# ---------------------------------------------------------------------------
# Tiny case: the whole step (copy-on-write, append, decode) against the oracle
# ---------------------------------------------------------------------------

def test_tiny_step(dev):
    w = wl.make_tiny(device=dev, preappend=True)
    ix = dev_indices(w, dev)
    k0, v0 = w.host(w.k_pool), w.host(w.v_pool)
    pre = w.context_lens - 1
    got_pre = decode(w, ix, ctx=torch.from_numpy(pre).to(dev))
    want_pre = oracle.paged_decode(w.host(w.q), k0, v0, w.block_tables, pre, w.scale, w.B, w.dtype)
    assert max_err(got_pre.cpu(), want_pre) <= TOL["f32"]

    pkv.kv_block_copy(w.k_pool, w.v_pool, ix["pairs"])
    pkv.kv_cache_append(w.k_new, w.v_new, w.k_pool, w.v_pool, ix["slots"])
    k1, v1, _ = oracle.kv_block_copy(k0, v0, w.cow_pairs)
    k2, v2, _ = oracle.kv_append(k1, v1, w.host(w.k_new), w.host(w.v_new), w.slot_mapping, w.B)
    assert np.array_equal(w.host(w.k_pool), k2, equal_nan=True)
    assert np.array_equal(w.host(w.v_pool), v2, equal_nan=True)

    want = oracle.paged_decode(w.host(w.q), k2, v2, w.block_tables, w.context_lens, w.scale, w.B, w.dtype)
    for pt in (0, 16, 32, 48):
        got = decode(w, ix, pt=pt)
        assert max_err(got.cpu(), want) <= TOL["f32"], pt
    no_device_error(dev)


# ---------------------------------------------------------------------------
# Small ragged cases, every dtype / head size / block size / partition size
# ---------------------------------------------------------------------------

RAGGED = [0, 1, 2, 15, 16, 17, 63, 64, 65, 127, 128, 129, 200, 513, 700]


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("B", [8, 16, 32, 64, 128])
def test_small_ragged(dev, dtype, D, B):
    mb = -(-max(RAGGED) // B) + 1
    w = wl.build_paged(RAGGED, H=3, D=D, B=B, dtype=dtype, seed=100 + D + B, device=dev, max_blocks=mb)
    ix = dev_indices(w, dev)
    want = full_oracle(w)
    outs = {}
    for pt in sorted({0, B, max(B, 64), 256, 512, mb * B}):
        got = decode(w, ix, pt=pt).cpu().numpy()
        assert np.all(np.isfinite(got)), pt
        assert max_err(got, want) <= TOL[dtype], (pt, max_err(got, want))
        outs[pt] = got
    zero = [i for i, c in enumerate(RAGGED) if c == 0]
    for pt, got in outs.items():
        assert np.all(got[zero] == 0.0)
    no_device_error(dev)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("B", [8, 16, 128])
@pytest.mark.parametrize("H", [36, 37])
def test_ring_depth_boundary_ragged(dev, dtype, D, B, H):
    # 16-bit decode runs a two-stage ring (three CTAs per SM) from 8 x 296 = 2368
    # (sequence, head, partition) units up, a three-stage ring below: 64 x 36 units
    # unsplit run the deep ring, 64 x 37 and every split run the shallow one
    ctx = np.array([RAGGED[i % len(RAGGED)] for i in range(64)])
    mb = -(-max(RAGGED) // B) + 1
    w = wl.build_paged(ctx, H=H, D=D, B=B, dtype=dtype, seed=300 + H + D + B, device=dev, max_blocks=mb)
    ix = dev_indices(w, dev)
    want = full_oracle(w)
    for pt in sorted({0, max(B, 64), 256, mb * B}):
        got = decode(w, ix, pt=pt).cpu().numpy()
        assert np.all(np.isfinite(got)), pt
        assert max_err(got, want) <= TOL[dtype], (pt, max_err(got, want))
        assert np.all(got[ctx == 0] == 0.0)
    no_device_error(dev)


def test_plan_sort_many_sequences(dev):
    # 1500 sequences: the plan's sorted path with several runs of 32 sequences per warp,
    # unsplit (1500 entries) and with full + last 512-token partitions (3000 entries);
    # 256-token partitions (4500 entries) take the unsorted path
    rng = np.random.default_rng(77)
    ctx = rng.integers(0, 601, 1500)
    w = wl.build_paged(ctx, H=2, D=64, B=16, dtype="f16", seed=77, device=dev, max_blocks=38)
    ix = dev_indices(w, dev)
    want = full_oracle(w)
    for pt in (0, 512, 256):
        got = decode(w, ix, pt=pt).cpu().numpy()
        assert max_err(got, want) <= TOL["f16"], pt
        assert np.all(got[ctx == 0] == 0.0)
    no_device_error(dev)


def test_one_token_contexts_return_v_exactly(dev):
    for dtype in ("f32", "f16", "bf16"):
        w = wl.build_paged([1] * 7, H=4, D=128, B=16, dtype=dtype, seed=7, device=dev)
        ix = dev_indices(w, dev)
        got = decode(w, ix).cpu().numpy()
        v = w.v_pool.float().cpu().numpy()
        for s in range(w.S):
            blk = w.block_tables[s, 0]
            assert np.array_equal(got[s], v[blk, :, 0, :]), dtype
    no_device_error(dev)


def test_maximum_context_and_empty(dev):
    # contexts at the table's maximum (max_blocks * B), empty ones, and one block
    B, mb = 16, 40
    ctx = [mb * B, 0, mb * B, B, 0, mb * B - 1]
    for dtype in ("f16", "bf16", "f32"):
        w = wl.build_paged(ctx, H=2, D=128, B=B, dtype=dtype, seed=8, device=dev, max_blocks=mb)
        ix = dev_indices(w, dev)
        want = full_oracle(w)
        for pt in (0, 64, mb * B):
            got = decode(w, ix, pt=pt).cpu().numpy()
            assert max_err(got, want) <= TOL[dtype]
            assert np.all(got[[1, 4]] == 0.0)
    no_device_error(dev)


def test_permutation_and_block_size_give_identical_results(dev):
    """Paging changes only where tokens live: the kernel's arithmetic follows the
    logical order, so every placement and block size gives bit-identical output."""
    ctx = np.array([3, 77, 300, 129, 1000, 16])
    for dtype in ("f16", "bf16"):
        logical = wl.draw_logical(int(ctx.sum()), len(ctx), 4, 128, dtype, 9, dev)
        ref = None
        for B in (8, 16, 32, 64, 128):
            for placement in (1, 2):
                w = wl.build_paged(ctx, 4, 128, B, dtype, 9, device=dev, logical=logical,
                                   placement_seed=1000 * B + placement, max_blocks=-(-1024 // B))
                ix = dev_indices(w, dev)
                got = decode(w, ix, pt=256).cpu()
                if ref is None:
                    ref = got
                    assert max_err(ref, full_oracle(w)) <= TOL[dtype]
                assert torch.equal(got, ref), (dtype, B, placement)
    no_device_error(dev)


def test_split_matches_unsplit(dev):
    ctx = np.array([5000, 4096, 1, 2500, 333])
    w = wl.build_paged(ctx, 8, 128, 16, "bf16", 10, device=dev, max_blocks=320)
    ix = dev_indices(w, dev)
    want = full_oracle(w)
    base = decode(w, ix, pt=320 * 16).cpu().numpy()
    assert max_err(base, want) <= TOL["bf16"]
    for pt in (16, 64, 128, 512, 1024, 4096):
        got = decode(w, ix, pt=pt).cpu().numpy()
        assert max_err(got, want) <= TOL["bf16"], pt
        assert max_err(got, base) <= TOL["bf16"], pt
    no_device_error(dev)


@pytest.mark.parametrize("S,H", [(5000, 2), (65535, 1)])
def test_many_sequences(dev, S, H):
    rng = np.random.default_rng(S)
    ctx = rng.integers(0, 81, size=S)
    w = wl.build_paged(ctx, H, 64, 16, "f16", 11, device=dev, max_blocks=6)
    ix = dev_indices(w, dev)
    for pt in (0, 32):
        got = decode(w, ix, pt=pt).cpu().numpy()
        sel = sample_pairs(w, 64, 12) + [(S - 1, H - 1), (0, 0)]
        want = oracle.paged_decode_selected(w.host(w.q), w.host(w.k_pool), w.host(w.v_pool), w.block_tables,
                                            w.context_lens, w.scale, w.B, w.dtype, sel)
        assert max_err(np.stack([got[s, h] for s, h in sel]), want) <= TOL["f16"]
        assert np.all(np.isfinite(got))
    no_device_error(dev)


def test_caller_workspace_and_library_workspace_agree(dev):
    w = wl.build_paged([900, 10, 2048, 0], 4, 128, 16, "f16", 13, device=dev, max_blocks=128)
    ix = dev_indices(w, dev)
    ws = pkv.alloc_workspace(w.q, w.k_pool, ix["bt"], 256)
    ws.fill_(0xAB)  # contents on entry must not matter
    a = decode(w, ix, pt=256, ws=ws)
    b = decode(w, ix, pt=256)
    assert torch.equal(a, b)
    assert max_err(a.cpu(), full_oracle(w)) <= TOL["f16"]
    no_device_error(dev)


# ---------------------------------------------------------------------------
# Full-size workloads: the bench step (copy -> append -> decode), sampled outputs
# ---------------------------------------------------------------------------

def run_step_and_check(w, dev, n_samples=24, seed=0, pt=None):
    ix = dev_indices(w, dev)
    sel = sample_pairs(w, n_samples, seed)
    snaps = [Snapshot(w, s, h) for s, h in sel]
    pair_src = None
    if len(w.cow_pairs):
        j = np.random.default_rng(seed).integers(len(w.cow_pairs), size=4)
        pair_src = [(int(w.cow_pairs[i, 0]), int(w.cow_pairs[i, 1]),
                     w.host(w.k_pool[int(w.cow_pairs[i, 0])]), w.host(w.v_pool[int(w.cow_pairs[i, 0])]))
                    for i in j]
        pkv.kv_block_copy(w.k_pool, w.v_pool, ix["pairs"])
    pkv.kv_cache_append(w.k_new, w.v_new, w.k_pool, w.v_pool, ix["slots"])
    ws = pkv.alloc_workspace(w.q, w.k_pool, ix["bt"], w.partition_tokens if pt is None else pt)
    out = decode(w, ix, pt=w.partition_tokens if pt is None else pt, ws=ws)
    torch.cuda.synchronize()
    no_device_error(dev)
    assert bool(torch.isfinite(out).all())
    got = out.cpu().numpy()
    for sn in snaps:
        want = sn.expected(w)
        err = max_err(got[sn.s, sn.h], want)
        assert err <= TOL[w.dtype], (w.name, sn.s, sn.h, sn.ctx, err)
    # appended rows landed bit for bit
    for s in range(0, w.S, max(1, w.S // 16)):
        slot = int(w.slot_mapping[s])
        blk, off = divmod(slot, w.B)
        assert torch.equal(w.k_pool[blk, :, off], w.k_new[s]) and torch.equal(w.v_pool[blk, :, off], w.v_new[s])
    if pair_src:
        for src, dst, ksrc, vsrc in pair_src:
            kd, vd = w.host(w.k_pool[dst]), w.host(w.v_pool[dst])
            # the copy equals the pre-step source, except rows the append then wrote
            written = [divmod(int(x), w.B)[1] for x in w.slot_mapping if int(x) // w.B == dst]
            keep = [o for o in range(w.B) if o not in written]
            assert np.array_equal(kd[:, keep], ksrc[:, keep], equal_nan=True)
            assert np.array_equal(vd[:, keep], vsrc[:, keep], equal_nan=True)
    return out


@pytest.mark.parametrize("name", ["llama7b", "cow", "longctx"])
def test_full_size_workload(dev, name):
    w = wl.make(name, device=dev, preappend=True)
    run_step_and_check(w, dev)


def test_opt13b_block_size_sweep(dev):
    """Batch-256 OPT-13B layer: the same token data under B = 8..128, each its own placement."""
    ctx = wl.opt13b_lengths()
    logical = wl.draw_logical(int(ctx.sum()), 256, 40, 128, "bf16", wl.BASE_SEED + 3, dev)
    ref = None
    for B in (8, 16, 32, 64, 128):
        w = wl.make_opt13b(B=B, device=dev, preappend=True, logical=logical)
        out = run_step_and_check(w, dev, n_samples=12, seed=B)
        if ref is None:
            ref = out
        else:
            assert torch.equal(out, ref), B
        del w, out
        torch.cuda.empty_cache()
