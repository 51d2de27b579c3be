"""The allocation-free decode entry point, paged_attn_decode_noalloc.

Some callers cannot allocate device memory: a host framework may own all of it
and hand a plugin nothing but a stream and its buffers, and a latency-critical
serving loop may not afford an allocation's implicit synchronisation.  For them
the library offers a decode that takes its scratch from a static device array
inside the library instead of a caller workspace.

These tests call that entry point through the C ABI (ctypes, no Python wrapper),
twice in a row on different inputs, so that the second call starts from the
scratch contents the first one left behind, and compare each output with the
CPU oracle (float64, from host copies of the inputs) and with the ordinary
entry point's output on the same inputs.  The file is named so that
pytest collects it after every other test file; it also passes on its own in a
fresh process (the first call on a device does the scratch set-up).
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_328_b200 as pkv
from paged_kv_cache_328_b200 import _lib
from paged_kv_cache_328_b200 import workloads as wl
from paritykit import TOL, max_err

pytestmark = pytest.mark.gpu

PKV_EWORKSPACE = -6


def call_noalloc(lib, w, bt, ctx, out, partition_tokens, stream):
    return lib.paged_attn_decode_noalloc(
        w.q.data_ptr(), w.k_pool.data_ptr(), w.v_pool.data_ptr(), bt.data_ptr(), ctx.data_ptr(),
        w.S, w.H, w.D, w.B, w.max_blocks, w.num_blocks, _lib.DTYPE_CODE[w.k_pool.dtype], ctypes.c_float(w.scale),
        out.data_ptr(), partition_tokens, ctypes.c_void_p(stream.cuda_stream))


def test_noalloc_matches_the_workspace_entry_point_on_two_calls_in_a_row():
    assert torch.cuda.is_available()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    lib = pkv.load()
    stream = torch.cuda.current_stream(dev)
    cases = [
        # split into 512-token partitions: the scratch holds the work list and partial states
        (wl.build_paged([5000, 1, 3100, 700, 0, 4096], 8, 128, 16, "f16", 31, device=dev, max_blocks=320), 512),
        # a different shape and dtype, library-chosen partitions, over the first call's leftovers
        (wl.build_paged(np.random.default_rng(32).integers(0, 900, size=40), 4, 64, 32, "bf16", 32,
                        device=dev, max_blocks=32), 0),
    ]
    for w, pt in cases:
        bt = torch.from_numpy(w.block_tables).to(dev)
        ctx = torch.from_numpy(w.context_lens).to(dev)
        want = oracle.paged_decode(w.host(w.q), w.host(w.k_pool), w.host(w.v_pool), w.block_tables,
                                   w.context_lens, w.scale, w.B, w.dtype)
        ref = pkv.paged_attn_decode(w.q, w.k_pool, w.v_pool, bt, ctx, w.scale, partition_tokens=pt)
        out = torch.full((w.S, w.H, w.D), float("nan"), dtype=torch.float32, device=dev)
        assert _lib.workspace_size(w.S, w.H, w.D, w.B, w.max_blocks, pt) <= _lib.NOALLOC_SCRATCH_BYTES
        rc = call_noalloc(lib, w, bt, ctx, out, pt, stream)
        assert rc == 0, _lib.strerror(rc)
        code, reason = pkv.get_device_error(dev)
        assert code == 0, (code, reason)
        assert bool(torch.isfinite(out).all())
        assert max_err(out.cpu(), want) <= TOL[w.dtype]
        assert max_err(out.cpu(), ref.cpu().numpy()) <= TOL[w.dtype]
        assert np.all(out.cpu().numpy()[w.context_lens == 0] == 0.0)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = pkv.load()
    # 64 sequences x 64 heads x 2048 partitions of 16 tokens need far more than 32 MiB
    S, H, D, B, MB, pt = 64, 64, 128, 16, 2048, 16
    assert _lib.workspace_size(S, H, D, B, MB, pt) > _lib.NOALLOC_SCRATCH_BYTES
    fake = 0x10000  # rejected on the host before any pointer is used
    rc = lib.paged_attn_decode_noalloc(fake, fake, fake, fake, fake, S, H, D, B, MB, 100000, 1,
                                       ctypes.c_float(0.088), fake, pt, None)
    assert rc == PKV_EWORKSPACE
    assert "workspace" in _lib.strerror(rc)
