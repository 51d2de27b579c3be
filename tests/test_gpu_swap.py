"""GPU parity of the block swaps (kv_blocks_to_host / kv_blocks_from_host) and a
decode loop driven by the native block manager, against the oracle."""

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


def clean(dev):
    code, reason = pkv.get_device_error(dev)
    assert code == 0, (code, reason)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("B", [8, 16, 128])
def test_swap_out_and_in_bit_exact(dev, dtype, B):
    nb, H, D = 24, 4, 128
    g = torch.Generator(device=dev)
    g.manual_seed(B)
    kc = torch.randn((nb, H, B, D), generator=g, device=dev).to(TD[dtype])
    vc = torch.randn((nb, H, B, D), generator=g, device=dev).to(TD[dtype])
    ids = np.array([5, 17, 2, 9, 23], dtype=np.int64)
    hk = torch.empty((len(ids), H, B, D), dtype=TD[dtype]).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    k0, v0 = host(kc), host(vc)
    pkv.kv_blocks_to_host(kc, vc, torch.from_numpy(ids).to(dev), hk, hv)
    torch.cuda.synchronize()
    ek, ev, bad = oracle.kv_swap_out(k0, v0, ids)
    assert bad == 0 and np.array_equal(host(hk), ek) and np.array_equal(host(hv), ev)
    # bring them back into other blocks
    new = np.array([0, 1, 11, 12, 20], dtype=np.int64)
    pkv.kv_blocks_from_host(hk, hv, kc, vc, torch.from_numpy(new).to(dev))
    ek2, ev2, bad = oracle.kv_swap_in(k0, v0, ek, ev, new)
    assert bad == 0 and np.array_equal(host(kc), ek2) and np.array_equal(host(vc), ev2)
    clean(dev)


def test_swap_bad_id_is_flagged_and_unpinned_memory_rejected(dev):
    nb, H, B, D = 6, 2, 16, 64
    kc = torch.zeros((nb, H, B, D), dtype=torch.float16, device=dev)
    hk = torch.zeros((2, H, B, D), dtype=torch.float16).pin_memory()
    pkv.kv_blocks_to_host(kc, kc, torch.tensor([1, nb], device=dev), hk, hk.clone().pin_memory())
    code, reason = pkv.get_device_error(dev)
    assert code == -7 and reason == 4
    with pytest.raises(ValueError):
        pkv.kv_blocks_to_host(kc, kc, torch.tensor([1], device=dev), torch.zeros((1, H, B, D), dtype=torch.float16),
                              hk[:1].clone().pin_memory())
    lib = pkv.load()
    plain = torch.zeros((1, H, B, D), dtype=torch.float16)   # not page-locked: the C ABI refuses it
    ids = torch.tensor([1], device=dev)
    rc = lib.kv_blocks_to_host(kc.data_ptr(), kc.data_ptr(), ids.data_ptr(), 1, plain.data_ptr(), plain.data_ptr(),
                               H, D, B, nb, 1, torch.cuda.current_stream(dev).cuda_stream)
    assert rc == -1
    clean(dev)


def test_sampling_loop_with_native_manager(dev):
    """Prompts forked into samples, a few decode steps: the native manager's slots and
    copy-on-write pairs drive the append / copy / decode kernels, one sample is swapped
    out and back in, and every output matches the oracle run on the oracle's manager."""
    H, D, B, NB, dtype = 4, 64, 16, 96, "bf16"
    rng = np.random.default_rng(7)
    native = pkv.BlockManager(NB, B)
    model = oracle.BlockManager(NB, B)
    kc = torch.full((NB, H, B, D), float("nan"), dtype=TD[dtype], device=dev)
    vc = torch.full_like(kc, float("nan"))
    k_host = host(kc)
    v_host = host(vc)
    seqs = []
    for p, plen in enumerate([10, 16, 33]):                     # prompts, then 3 samples each
        for impl in (native, model):
            impl.add_sequence(100 * p, plen)
        table, _ = model.block_table(100 * p)
        kp = rng.standard_normal((plen, H, D)).astype(np.float32)
        vp = rng.standard_normal((plen, H, D)).astype(np.float32)
        for t in range(plen):
            k_host[table[t // B], :, t % B] = (torch.from_numpy(kp[t]).to(TD[dtype])).view(torch.int16).numpy().view(np.uint16)
            v_host[table[t // B], :, t % B] = (torch.from_numpy(vp[t]).to(TD[dtype])).view(torch.int16).numpy().view(np.uint16)
        seqs.append(100 * p)
        for j in range(1, 4):
            for impl in (native, model):
                impl.fork(100 * p, 100 * p + j)
            seqs.append(100 * p + j)
    kc.copy_(torch.from_numpy(k_host.view(np.int16)).view(TD[dtype]).to(dev))
    vc.copy_(torch.from_numpy(v_host.view(np.int16)).view(TD[dtype]).to(dev))
    ws = None
    for step in range(20):
        if step == 7:                                              # swap one sample out and back
            blocks = native.swap_out(seqs[5])
            assert blocks == model.swap_out(seqs[5])
            hk = torch.empty((len(blocks), H, B, D), dtype=TD[dtype]).pin_memory()
            hv = torch.empty_like(hk).pin_memory()
            pkv.kv_blocks_to_host(kc, vc, torch.tensor(blocks, device=dev), hk, hv)
            hk_o, hv_o, _ = oracle.kv_swap_out(k_host, v_host, blocks)
            back = native.swap_in(seqs[5])
            assert back == model.swap_in(seqs[5])
            pkv.kv_blocks_from_host(hk, hv, kc, vc, torch.tensor(back, device=dev))
            k_host, v_host, _ = oracle.kv_swap_in(k_host, v_host, hk_o, hv_o, back)
        slots, pairs = native.append_tokens(seqs)
        slots_m, pairs_m = model.append_tokens(seqs)
        assert slots == slots_m and [tuple(p) for p in pairs] == [tuple(p) for p in pairs_m]
        knew = torch.randn((len(seqs), H, D), device=dev).to(TD[dtype])
        vnew = torch.randn((len(seqs), H, D), device=dev).to(TD[dtype])
        q = torch.randn((len(seqs), H, D), device=dev).to(TD[dtype])
        if pairs:
            pkv.kv_block_copy(kc, vc, torch.tensor(pairs, device=dev))
            k_host, v_host, _ = oracle.kv_block_copy(k_host, v_host, np.array(pairs))
        pkv.kv_cache_append(knew, vnew, kc, vc, torch.tensor(slots, device=dev))
        k_host, v_host, _ = oracle.kv_append(k_host, v_host, host(knew), host(vnew), np.array(slots), B)
        tables, lens = native.fill_tables(seqs, 8)
        out = pkv.paged_attn_decode(q, kc, vc, tables.to(dev), lens.to(dev), 0.125)
        want = oracle.paged_decode(host(q), k_host, v_host, tables.numpy(), lens.numpy(), 0.125, B, dtype)
        assert float(np.max(np.abs(out.cpu().numpy() - want))) <= 2e-3, step
        assert np.array_equal(host(kc), k_host, equal_nan=True)
    clean(dev)
